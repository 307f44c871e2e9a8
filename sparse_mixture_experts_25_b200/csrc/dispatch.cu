// Capacity check, token-order dispatch and the row gather.
//
// What it computes (Algorithm 36.1 steps 3-4 of "LLM from scratch" ch. 36;
// ch. 36.3 dispatch matrices D_e as index lists and prefix sums; auturnal
// review equations for O and rho_max): paths (t, e) are taken in token order;
// path (t, e) gets slot c = number of earlier requests for e and is accepted
// iff c < C.
//
// Design: a stable counting sort in three short launches, with no cross-CTA
// waiting:
//   hist   one CTA per tile of tokens counts its requests per expert
//          (shared-memory atomics; order does not matter for counts);
//   scan   a warp per expert turns its row of the [E][tiles] counts into
//          exclusive per-tile bases (each lane a contiguous run of tiles);
//          the block that finishes last (a ticket, no waiting) scans the
//          accepted counts min(L_e, C) over experts into row offsets and the
//          M-tile prefix used by the grouped GEMMs, and writes the statistics;
//   assign one warp per tile walks its requests in token order, 32 at a
//          time; __match_any_sync groups equal experts so a lane's slot is
//          base + running count + its rank among earlier equal lanes.
// gather then copies x rows into the per-expert row buffer, a warp per row
// with 16-byte vector loads (HBM-bound, coalesced along each row).
#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Exclusive scan over blockDim.x (<= 1024, multiple of 32) values; returns
// the exclusive prefix and writes the block total to *total (all threads).
__device__ int block_excl_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int inc = warp_incl_scan(v, lane);
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int wv = lane < nw ? warp_tot[lane] : 0;
        const int wi = warp_incl_scan(wv, lane);
        if (lane < nw) warp_tot[lane] = wi - wv;
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    const int ex = inc - v + warp_tot[warp];
    *total = warp_tot[32];
    __syncthreads();
    return ex;
}

__global__ void hist_kernel(const int32_t* __restrict__ ids, int64_t N, int k, int E,
                            int tile_tokens, int n_tiles, int32_t* __restrict__ hist,
                            unsigned long long* counters) {
    extern __shared__ int h[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {  // the scans that follow count finished blocks from 0
        counters[CNT_SCAN_TICKET] = 0;
        counters[CNT_SCAN_ANY] = 0;
    }
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * tile_tokens;
    const int64_t t1 = min64(N, t0 + tile_tokens);
    bool oob = false;
    for (int64_t i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) {
        const int e = ids[i];
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        else if (e >= E) oob = true;
    }
    if (oob) atomicOr(reinterpret_cast<unsigned long long*>(counters + CNT_DEVICE_ERROR), (unsigned long long)DEVERR_BOUNDS);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)e * n_tiles + blockIdx.x] = h[e];
}

// Per expert (one warp each), the per-tile request counts become exclusive
// bases in place; sL[e] receives the expert's total.  Each lane owns a
// contiguous segment of the expert's tiles: it sums the segment (independent
// loads), one warp scan turns the sums into segment bases, and the lane
// rewrites its segment as running bases.  A warp takes its experts four at a
// time so that the loads of all four are in flight together.
__device__ void tile_scan(int32_t* __restrict__ hist, int n_tiles, int E, int* sL) {
    constexpr int G = 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int seg = (n_tiles + 31) / 32;
    const int i0 = min(n_tiles, lane * seg), i1 = min(n_tiles, i0 + seg);
    for (int e0 = warp; e0 < E; e0 += G * nw) {
        int sum[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
            sum[j] = 0;
            const int e = e0 + j * nw;
            if (e < E) {
                const int32_t* row = hist + (int64_t)e * n_tiles;
#pragma unroll 8
                for (int i = i0; i < i1; ++i) sum[j] += row[i];
            }
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const int e = e0 + j * nw;  // warp-uniform
            if (e >= E) break;
            int32_t* row = hist + (int64_t)e * n_tiles;
            const int inc = warp_incl_scan(sum[j], lane);
            int run = inc - sum[j];
#pragma unroll 8
            for (int i = i0; i < i1; ++i) {
                const int v = row[i];
                row[i] = run;
                run += v;
            }
            if (lane == 31) sL[e] = inc;
        }
    }
}

// Expert e's per-tile request counts (one row of hist) become exclusive bases
// in place, by one warp: each lane sums a contiguous run of tiles (independent
// loads), one warp scan turns the sums into run bases, and each lane rewrites
// its run.  Returns the expert's total in every lane.
__device__ int warp_tile_scan(int32_t* __restrict__ row, int n_tiles, int lane) {
    const int seg = (n_tiles + 31) / 32;
    const int i0 = min(n_tiles, lane * seg), i1 = min(n_tiles, i0 + seg);
    int sum = 0;
#pragma unroll 8
    for (int i = i0; i < i1; ++i) sum += row[i];
    const int inc = warp_incl_scan(sum, lane);
    int run = inc - sum;
#pragma unroll 8
    for (int i = i0; i < i1; ++i) {
        const int v = row[i];
        row[i] = run;
        run += v;
    }
    return __shfl_sync(0xffffffffu, inc, 31);
}

// True in the block that finishes last (each block fences its global writes
// before taking a ticket, so the last one sees them all).  No block waits for
// another.  The last block puts the ticket back to 0 for the next launch.
__device__ bool last_block_done(unsigned long long* ticket) {
    __shared__ int last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        last = atomicAdd(ticket, 1ull) == (unsigned long long)gridDim.x - 1;
        if (last) *ticket = 0;
    }
    __syncthreads();
    if (last) __threadfence();
    return last;
}

constexpr int kScanWarps = 8;  // experts per scan block (one warp each)

// Per-tile bases (one warp per expert, kScanWarps experts per block), then,
// in the block that finishes last, the scans over experts: accepted counts
// min(L_e, C) into row offsets, M-tiles into the prefix used by the grouped
// GEMMs, requests into all_offsets (acceptance by weight), and the
// statistics.
__global__ void scan_kernel(int32_t* __restrict__ hist, int n_tiles, int E, int64_t C, int bm,
                            int32_t* __restrict__ L, int32_t* __restrict__ acc,
                            int32_t* __restrict__ offsets, int32_t* __restrict__ mt_start,
                            int32_t* __restrict__ all_offsets, unsigned long long* counters) {
    __shared__ int warp_tot[33];
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * kScanWarps + (threadIdx.x >> 5);
    if (e < E) {
        const int tot = warp_tile_scan(hist + (int64_t)e * n_tiles, n_tiles, lane);
        if (lane == 0) L[e] = tot;
    }
    if (!last_block_done(counters + CNT_SCAN_TICKET)) return;
    int car_a = 0, car_mt = 0, car_L = 0, car_O = 0, lmax = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {  // uniform over the block
        const int ex = e0 + (int)threadIdx.x;
        const int Le = ex < E ? __ldcg(L + ex) : 0;
        const int a = (int)min64(Le, C);
        const int mt = (a + bm - 1) / bm;
        int t_a, t_mt, t_L, t_O;
        const int ex_a = block_excl_scan(a, warp_tot, &t_a);
        const int ex_mt = block_excl_scan(mt, warp_tot, &t_mt);
        const int ex_L = block_excl_scan(Le, warp_tot, &t_L);
        block_excl_scan(Le > C ? (int)(Le - C) : 0, warp_tot, &t_O);
        if (ex < E) {
            acc[ex] = a;
            offsets[ex] = car_a + ex_a;
            mt_start[ex] = car_mt + ex_mt;
            if (all_offsets) all_offsets[ex] = car_L + ex_L;
        }
        lmax = max(lmax, Le);
        car_a += t_a;
        car_mt += t_mt;
        car_L += t_L;
        car_O += t_O;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if (lane == 0 && lmax > 0) atomicMax(counters + CNT_L_MAX, (unsigned long long)lmax);
    if (threadIdx.x == 0) {
        if (all_offsets) all_offsets[E] = car_L;
        offsets[E] = car_a;
        mt_start[E] = car_mt;
        counters[CNT_REQUESTED] = (unsigned long long)car_L;
        counters[CNT_ACCEPTED] = (unsigned long long)car_a;
        counters[CNT_REJECTED] = (unsigned long long)(car_L - car_a);
        counters[CNT_O] = (unsigned long long)car_O;
        counters[CNT_C] = (unsigned long long)C;
    }
}

// Sharded routing group, first half: this rank's per-tile bases and its
// per-expert request counts (written to L and, when given, counts_out for the
// exchange between ranks).
__global__ void count_scan_kernel(int32_t* __restrict__ hist, int n_tiles, int E,
                                  int32_t* __restrict__ L, int32_t* __restrict__ counts_out) {
    __shared__ int sL[kMaxExperts];
    tile_scan(hist, n_tiles, E, sL);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        L[e] = sL[e];
        if (counts_out) counts_out[e] = sL[e];
    }
}

// Sharded routing group, second half: from the gathered request counts of
// every rank ([n_ranks][E], ranks in token order) this rank's requests for e
// are requests base_e .. base_e + L_e - 1 of the whole group, base_e = sum of
// the earlier ranks' counts; the first C of the group are accepted, so this
// rank keeps acc_e = clamp(C - base_e, 0, L_e) of them.  Statistics: counts
// of this rank's requests, plus O, the maximum load and (in L) the loads of
// the whole group.
__global__ void expert_scan_ranked_kernel(int E, int64_t C, int bm, const int32_t* __restrict__ table,
                                          int rank, int n_ranks, int64_t n_group,
                                          int32_t* __restrict__ L, int32_t* __restrict__ acc,
                                          int32_t* __restrict__ offsets,
                                          int32_t* __restrict__ mt_start,
                                          int32_t* __restrict__ base_out,
                                          unsigned long long* counters) {
    __shared__ int warp_tot[33];
    const int e = threadIdx.x;
    int64_t base = 0, Lg = 0, Le = 0;
    if (e < E) {
        for (int r = 0; r < n_ranks; ++r) {
            const int64_t v = table[(int64_t)r * E + e];
            if (r < rank) base += v;
            if (r == rank) Le = v;
            Lg += v;
        }
    }
    int64_t a64 = C - base;
    a64 = a64 < 0 ? 0 : (a64 > Le ? Le : a64);
    const int a = (int)a64;
    const int mt = (a + bm - 1) / bm;
    int tot_a, tot_mt, tot_L, tot_O;
    const int ex_a = block_excl_scan(a, warp_tot, &tot_a);
    const int ex_mt = block_excl_scan(mt, warp_tot, &tot_mt);
    block_excl_scan((int)Le, warp_tot, &tot_L);
    block_excl_scan(Lg > C ? (int)(Lg - C) : 0, warp_tot, &tot_O);
    if (e < E) {
        L[e] = (int32_t)Lg;
        acc[e] = a;
        offsets[e] = ex_a;
        mt_start[e] = ex_mt;
        base_out[e] = (int32_t)base;
        atomicMax(counters + CNT_L_MAX, (unsigned long long)Lg);
    }
    if (threadIdx.x == 0) {
        offsets[E] = tot_a;
        mt_start[E] = tot_mt;
        counters[CNT_REQUESTED] = (unsigned long long)tot_L;
        counters[CNT_ACCEPTED] = (unsigned long long)tot_a;
        counters[CNT_REJECTED] = (unsigned long long)(tot_L - tot_a);
        counters[CNT_O] = (unsigned long long)tot_O;
        counters[CNT_C] = (unsigned long long)C;
        counters[CNT_N_GROUP] = (unsigned long long)n_group;
    }
}

// rank_base (nullable): per-expert requests of earlier ranks of a sharded group;
// a request's group-wide slot is base + its slot among this rank's requests.
__device__ void token_pass(const int32_t* __restrict__ ids, const float* __restrict__ w, int k, int E,
                           int64_t tb, int64_t te, const int32_t* __restrict__ offsets,
                           const int32_t* __restrict__ rank_base, int renorm_rejected,
                           const int32_t* __restrict__ slot, float* __restrict__ slot_w,
                           unsigned long long* counters);

// slots_only: write slot[] only (first round of rerouting: the rows and the
// per-token statistics are written once every round is done)
__global__ void assign_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                              int64_t N, int k, int E, int64_t C, int tile_tokens, int n_tiles,
                              const int32_t* __restrict__ hist, const int32_t* __restrict__ offsets,
                              const int32_t* __restrict__ rank_base, int renorm_rejected,
                              int store_request, int slots_only, int32_t* __restrict__ slot,
                              int32_t* __restrict__ slot_token, float* __restrict__ slot_w,
                              unsigned long long* counters) {
    extern __shared__ int run[];
    const int lane = threadIdx.x;
    const int tile = blockIdx.x;
    for (int e = lane; e < E; e += 32) run[e] = hist[(int64_t)e * n_tiles + tile];
    __syncwarp();
    const int64_t tb = (int64_t)tile * tile_tokens;
    const int64_t te = min64(N, tb + tile_tokens);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t base = tb * k; base < te * k; base += 32) {
        const int64_t i = base + lane;
        const bool valid = i < te * k;
        int e = valid ? ids[i] : -1;
        if (e >= E || e < 0) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int s = e >= 0 ? run[e] + rank : -1;
        __syncwarp();
        if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
        __syncwarp();
        if (valid) {
            const int64_t sg = e >= 0 ? (rank_base ? (int64_t)rank_base[e] + s : (int64_t)s) : -1;
            if (e >= 0 && sg < C) {
                if (!slots_only) {
                    const int64_t pos = (int64_t)offsets[e] + s;
                    slot_token[pos] = store_request ? (int32_t)i : (int32_t)(i / k);
                    slot_w[pos] = w[i];
                }
                slot[i] = (int32_t)sg;
            } else {
                slot[i] = -1;
            }
        }
    }
    __syncwarp();
    if (store_request || slots_only) return;  // no statistics yet
    token_pass(ids, w, k, E, tb, te, offsets, rank_base, renorm_rejected, slot, slot_w, counters);
}

// Per token of [tb, te) (one warp): tokens with a rejected path, tokens with
// every path rejected, and (reject policy 1) the rescaling of the accepted
// paths' combine weights to sum to one.
__device__ void token_pass(const int32_t* __restrict__ ids, const float* __restrict__ w, int k, int E,
                           int64_t tb, int64_t te, const int32_t* __restrict__ offsets,
                           const int32_t* __restrict__ rank_base, int renorm_rejected,
                           const int32_t* __restrict__ slot, float* __restrict__ slot_w,
                           unsigned long long* counters) {
    const int lane = threadIdx.x & 31;
    unsigned long long affected = 0, skipped = 0;
    for (int64_t t = tb + lane; t < te; t += 32) {
        int req = 0, rej = 0;
        for (int j = 0; j < k; ++j) {
            const int e = ids[t * k + j];
            if (e >= 0 && e < E) {
                ++req;
                if (slot[t * k + j] < 0) ++rej;
            }
        }
        affected += rej > 0;
        skipped += (req > 0 && rej == req);
        if (renorm_rejected && rej > 0 && rej < req) {
            // the token's accepted paths share its weight: rescale them to sum to one
            float sum = 0.f;
            for (int j = 0; j < k; ++j)
                if (slot[t * k + j] >= 0) sum += w[t * k + j];
            for (int j = 0; j < k; ++j) {
                const int sg = slot[t * k + j];
                if (sg < 0) continue;
                const int e = ids[t * k + j];
                const int64_t local = rank_base ? (int64_t)sg - rank_base[e] : (int64_t)sg;
                slot_w[(int64_t)offsets[e] + local] = w[t * k + j] / sum;
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        affected += __shfl_xor_sync(0xffffffffu, affected, o);
        skipped += __shfl_xor_sync(0xffffffffu, skipped, o);
    }
    if (lane == 0) {
        if (affected) atomicAdd(counters + CNT_AFFECTED, affected);
        if (skipped) atomicAdd(counters + CNT_SKIPPED, skipped);
    }
}

// --- acceptance by routing weight ------------------------------------------
// After the placement pass (assign_kernel with no capacity, storing request
// indices), expert e's requests sit in token order at seg_req / seg_w
// [all_offsets[e], all_offsets[e+1]).  An expert with more than C requests
// accepts the C with the largest weight, equal weights to the earlier
// request.  prio_accept_kernel (one block per expert) finds the C-th largest
// weight W* by a radix select over the order-preserving bit pattern of the
// fp32 weights (four passes of 8-bit digits into a 256-bin shared-memory
// histogram) and how many of the requests equal to W* are taken; requests
// above W* are all accepted, and those equal to W* in token order up to that
// count.  It then numbers the accepted requests in token order and writes the
// routing records.

// fp32 bits -> unsigned integer with the same order as the floats
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One block of 1024 threads per expert.
//   select  per pass, lanes of a warp with the same digit add to the
//           histogram once (match_any), and warp 0 finds the digit that holds
//           the rem-th largest candidate with a scan over 8 bins per lane;
//   number  each thread takes a contiguous run of the expert's requests, so
//           the whole numbering costs two block scans (equal keys before the
//           run, accepted requests before the run) whatever the request count.
// An expert with at most C requests accepts them all: slot = position.
__global__ void __launch_bounds__(1024)
    prio_accept_kernel(int k, int64_t C, const int32_t* __restrict__ all_offsets,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ seg_req,
                       const float* __restrict__ seg_w, const float* __restrict__ w,
                       uint32_t* __restrict__ sel_key, int32_t* __restrict__ sel_take,
                       int32_t* __restrict__ slot, int32_t* __restrict__ slot_token,
                       float* __restrict__ slot_w) {
    __shared__ int hist[256];
    __shared__ int warp_tot[33];
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem;
    const int e = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s0 = all_offsets[e], Le = all_offsets[e + 1] - s0;
    const int64_t o = offsets[e];
    if (Le <= C) {
        for (int i = threadIdx.x; i < Le; i += blockDim.x) {
            const int req = seg_req[s0 + i];
            slot[req] = i;
            slot_token[o + i] = req / k;
            slot_w[o + i] = w[req];
        }
        return;
    }
    uint32_t prefix = 0, mask = 0;
    int rem = (int)C;  // rank (1-based, from the top) of the wanted key among the candidates
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < Le; i0 += blockDim.x) {  // warp-uniform trip count
            const int i = i0 + threadIdx.x;
            bool cand = false;
            uint32_t dg = 0;
            if (i < Le) {
                const uint32_t key = order_key(seg_w[s0 + i]);
                cand = (key & mask) == prefix;
                dg = (key >> shift) & 255u;
            }
            const unsigned act = __ballot_sync(0xffffffffu, cand);
            if (cand) {
                const unsigned peers = __match_any_sync(act, dg);
                if (__ffs(peers) - 1 == lane) atomicAdd(&hist[dg], __popc(peers));
            }
        }
        __syncthreads();
        if (warp == 0) {
            // lane l holds digits 255 - 8l down to 248 - 8l (largest first)
            int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[255 - 8 * lane - j];
                sum += c[j];
            }
            const int incl = warp_incl_scan(sum, lane);
            const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);
            // the candidates always number at least rem; lane 31 if not
            const int l0 = hit ? __ffs(hit) - 1 : 31;
            if (lane == l0) {
                int cum = incl - sum, d = 248 - 8 * lane;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum + c[j] >= rem) {
                        d = 255 - 8 * lane - j;
                        break;
                    }
                    cum += c[j];
                }
                s_rem = rem - cum;
                s_prefix = prefix | ((uint32_t)d << shift);
            }
        }
        __syncthreads();
        prefix = s_prefix;
        rem = s_rem;
        mask |= 255u << shift;
    }
    const uint32_t T = prefix;  // key of the C-th largest weight
    const int take = rem;       // requests with exactly that key to accept, earliest first
    if (threadIdx.x == 0) {
        sel_key[e] = T;
        sel_take[e] = take;
    }
    const int per = (Le + blockDim.x - 1) / blockDim.x;
    const int b0 = min(Le, (int)threadIdx.x * per), b1 = min(Le, b0 + per);
    int n_eq = 0;
    for (int i = b0; i < b1; ++i) n_eq += order_key(seg_w[s0 + i]) == T ? 1 : 0;
    int tot;
    const int eq0 = block_excl_scan(n_eq, warp_tot, &tot);
    int n_f = 0;
    for (int i = b0, eq = eq0; i < b1; ++i) {
        const uint32_t key = order_key(seg_w[s0 + i]);
        if (key > T) ++n_f;
        else if (key == T && eq++ < take) ++n_f;
    }
    int sl = block_excl_scan(n_f, warp_tot, &tot);
    // accepted rows of e: C (the cap also keeps a caller's NaN weight, whose
    // key is arbitrary, from numbering a row past the expert's block)
    for (int i = b0, eq = eq0; i < b1; ++i) {
        const uint32_t key = order_key(seg_w[s0 + i]);
        const bool f = key > T || (key == T && eq++ < take);
        const int req = seg_req[s0 + i];
        if (f && sl < C) {
            slot[req] = sl;
            slot_token[o + sl] = req / k;
            slot_w[o + sl] = w[req];
        } else {
            slot[req] = -1;
        }
        if (f) ++sl;
    }
}

// Unrequested paths (-1 ids) get slot -1, then the per-token statistics and
// the reject policy; one warp per tile of tokens.
__global__ void prio_token_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                  int64_t N, int k, int E, int tile_tokens,
                                  const int32_t* __restrict__ offsets, int renorm_rejected,
                                  int32_t* __restrict__ slot, float* __restrict__ slot_w,
                                  unsigned long long* counters) {
    const int64_t tb = (int64_t)blockIdx.x * tile_tokens;
    const int64_t te = min64(N, tb + tile_tokens);
    for (int64_t i = tb * k + threadIdx.x; i < te * k; i += 32) {
        const int e = ids[i];
        if (e < 0 || e >= E) slot[i] = -1;
    }
    __syncwarp();
    token_pass(ids, w, k, E, tb, te, offsets, nullptr, renorm_rejected, slot, slot_w, counters);
}

// --- rerouting of rejected paths (MOE_REJECT_REROUTE) ----------------------
// After the first-choice acceptance (assign_kernel, slots only), each round:
//   offer   per token (one thread each): every path still without an expert
//           takes the token's next unused candidate whose expert was not full
//           at the start of the round (acc[] as the previous round left it);
//           offers are counted per tile and expert, like first choices;
//   scan    per-tile bases of the offers, base[e] = acc[e], and acc[e] grows
//           by the offers it can take (at most C in all);
//   assign  one warp per tile walks the offers in token order: an offer for e
//           gets slot base[e] + (earlier offers for e) and is accepted iff
//           that is < C.
// Then the final offsets (prefix of acc), and the rows of every served path
// (first choices at offsets[e] + slot, rerouted ones at offsets[e] + rr_slot)
// with the per-token statistics.
// rr_stop: set by the scan of a round that had no offers; every later round
// returns at once (a round without offers leaves nothing for the next).
__global__ void reroute_offer_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ slot,
                                     const int32_t* __restrict__ cand, int X, const int32_t* __restrict__ acc,
                                     int64_t C, int64_t N, int k, int E, int tile_tokens, int n_tiles,
                                     const int32_t* __restrict__ rr_e, int32_t* __restrict__ rr_next,
                                     int32_t* __restrict__ rr_offer, int32_t* __restrict__ hist,
                                     const int32_t* __restrict__ rr_stop) {
    if (*rr_stop) return;
    extern __shared__ int h[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * tile_tokens;
    const int64_t t1 = min64(N, t0 + tile_tokens);
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        int q = rr_next[t];
        for (int j = 0; j < k; ++j) {
            const int64_t i = t * k + j;
            int off = -1;
            const int e0 = ids[i];
            if (e0 >= 0 && e0 < E && slot[i] < 0 && rr_e[i] < 0) {
                while (q < X) {
                    const int c = cand[t * X + q];
                    if (c < 0 || c >= E) {  // no further candidate
                        q = X;
                        break;
                    }
                    if (acc[c] < C) break;
                    ++q;
                }
                if (q < X) {
                    off = q;
                    atomicAdd(&h[cand[t * X + q]], 1);
                    ++q;
                }
            }
            rr_offer[i] = off;
        }
        rr_next[t] = q;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)e * n_tiles + blockIdx.x] = h[e];
}

// One rerouting round's offers per expert (one warp each): per-tile bases of
// the offers, base[e] = slots taken before the round, acc[e] grows by the
// offers it accepts.  The block that finishes last sets rr_stop when no
// expert received an offer (the later rounds then return at once).
__global__ void reroute_scan_kernel(int32_t* __restrict__ hist, int n_tiles, int E, int64_t C,
                                    int32_t* __restrict__ acc, int32_t* __restrict__ base,
                                    int32_t* __restrict__ rr_stop, unsigned long long* counters) {
    if (*rr_stop) return;  // uniform: every thread reads the same flag
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * kScanWarps + (threadIdx.x >> 5);
    if (e < E) {
        const int offers = warp_tile_scan(hist + (int64_t)e * n_tiles, n_tiles, lane);
        if (lane == 0) {
            const int a = acc[e];
            base[e] = a;
            acc[e] = (int)min64((int64_t)a + offers, C);
            if (offers) atomicAdd(counters + CNT_SCAN_ANY, 1ull);
        }
    }
    if (!last_block_done(counters + CNT_SCAN_TICKET)) return;
    if (threadIdx.x == 0) {
        if (atomicExch(counters + CNT_SCAN_ANY, 0ull) == 0ull) *rr_stop = 1;
    }
}

__global__ void reroute_assign_kernel(const int32_t* __restrict__ rr_offer, const int32_t* __restrict__ cand,
                                      int X, int64_t N, int k, int E, int64_t C, int tile_tokens, int n_tiles,
                                      const int32_t* __restrict__ hist, const int32_t* __restrict__ base,
                                      int32_t* __restrict__ rr_e, int32_t* __restrict__ rr_slot,
                                      int32_t* __restrict__ rr_q, const int32_t* __restrict__ rr_stop) {
    if (*rr_stop) return;
    extern __shared__ int run[];
    const int lane = threadIdx.x;
    const int tile = blockIdx.x;
    for (int e = lane; e < E; e += 32) run[e] = hist[(int64_t)e * n_tiles + tile];
    __syncwarp();
    const int64_t tb = (int64_t)tile * tile_tokens;
    const int64_t te = min64(N, tb + tile_tokens);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t b = tb * k; b < te * k; b += 32) {
        const int64_t i = b + lane;
        const bool valid = i < te * k;
        const int q = valid ? rr_offer[i] : -1;
        int e = q >= 0 ? cand[(i / k) * X + q] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int s = e >= 0 ? run[e] + rank : -1;
        __syncwarp();
        if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
        __syncwarp();
        if (e >= 0) {
            const int64_t sg = (int64_t)base[e] + s;
            if (sg < C) {
                rr_e[i] = e;
                rr_slot[i] = (int32_t)sg;
                rr_q[i] = q;
            }
        }
    }
}

// Offsets and M-tile prefix from the final rows per expert; accepted and
// rejected counters (requested, O, the maximum load and C were written by the
// first-choice scan).
__global__ void reroute_final_scan_kernel(int E, int bm, const int32_t* __restrict__ acc,
                                          int32_t* __restrict__ offsets, int32_t* __restrict__ mt_start,
                                          unsigned long long* counters) {
    __shared__ int warp_tot[33];
    const int e = threadIdx.x;  // blockDim.x >= E
    const int a = e < E ? acc[e] : 0;
    const int mt = (a + bm - 1) / bm;
    int tot_a, tot_mt;
    const int ex_a = block_excl_scan(a, warp_tot, &tot_a);
    const int ex_mt = block_excl_scan(mt, warp_tot, &tot_mt);
    if (e < E) {
        offsets[e] = ex_a;
        mt_start[e] = ex_mt;
    }
    if (threadIdx.x == 0) {
        offsets[E] = tot_a;
        mt_start[E] = tot_mt;
        const unsigned long long req = counters[CNT_REQUESTED];
        counters[CNT_ACCEPTED] = (unsigned long long)tot_a;
        counters[CNT_REJECTED] = req - (unsigned long long)tot_a;
    }
}

// Rows of every served path and the per-token statistics (one warp per tile):
// tokens with a requested path left without an expert, tokens with every
// requested path left without one, and the rerouted paths.
__global__ void reroute_rows_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                    const int32_t* __restrict__ slot, const int32_t* __restrict__ rr_e,
                                    const int32_t* __restrict__ rr_slot, const int32_t* __restrict__ rr_q,
                                    const float* __restrict__ cand_w, int X, int64_t N, int k, int E,
                                    int tile_tokens, const int32_t* __restrict__ offsets,
                                    int32_t* __restrict__ slot_token, float* __restrict__ slot_w,
                                    unsigned long long* counters) {
    const int lane = threadIdx.x & 31;
    const int64_t tb = (int64_t)blockIdx.x * tile_tokens;
    const int64_t te = min64(N, tb + tile_tokens);
    const int total = offsets[E];
    for (int64_t i = tb * k + lane; i < te * k; i += 32) {
        const int64_t t = i / k;
        const int e0 = ids[i];
        if (e0 < 0 || e0 >= E) continue;
        int64_t row = -1;
        float wr = 0.f;
        if (slot[i] >= 0) {
            row = (int64_t)offsets[e0] + slot[i];
            wr = w[i];
        } else if (rr_e[i] >= 0) {
            row = (int64_t)offsets[rr_e[i]] + rr_slot[i];
            wr = cand_w[t * X + rr_q[i]];
        }
        if (row >= 0 && row < total) {
            slot_token[row] = (int32_t)t;
            slot_w[row] = wr;
        }
    }
    unsigned long long affected = 0, skipped = 0, moved = 0;
    for (int64_t t = tb + lane; t < te; t += 32) {
        int req = 0, lost = 0;
        for (int j = 0; j < k; ++j) {
            const int64_t i = t * k + j;
            const int e0 = ids[i];
            if (e0 < 0 || e0 >= E) continue;
            ++req;
            if (rr_e[i] >= 0) ++moved;
            else if (slot[i] < 0) ++lost;
        }
        affected += lost > 0;
        skipped += (req > 0 && lost == req);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        affected += __shfl_xor_sync(0xffffffffu, affected, o);
        skipped += __shfl_xor_sync(0xffffffffu, skipped, o);
        moved += __shfl_xor_sync(0xffffffffu, moved, o);
    }
    if (lane == 0) {
        if (affected) atomicAdd(counters + CNT_AFFECTED, affected);
        if (skipped) atomicAdd(counters + CNT_SKIPPED, skipped);
        if (moved) atomicAdd(counters + CNT_REROUTED, moved);
    }
}

// One warp copies a row of row_vec 16-byte words; four loads per lane are in
// flight before their stores, so that each SM keeps enough bytes outstanding
// to draw the HBM rate.  The source rows are read with an evict-last L2
// policy and the destination written evict-first: a token's row is read once
// per path (k times), and the copies streaming out must not push the source
// rows out of L2 between those reads.
__device__ __forceinline__ uint4 ld_keep(const uint4* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ void st_stream(uint4* p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void copy_row_warp(const uint4* __restrict__ src, uint4* __restrict__ dst, int row_vec,
                                              int lane) {
    uint64_t keep, stream;
#ifndef MOE_GATHER_HINTS
#define MOE_GATHER_HINTS 1
#endif
    if (MOE_GATHER_HINTS) {
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(stream));
    } else {  // both normal priority
        asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(keep));
        stream = keep;
    }
    int i = lane;
    for (; i + 96 < row_vec; i += 128) {
        const uint4 v0 = ld_keep(src + i, keep), v1 = ld_keep(src + i + 32, keep);
        const uint4 v2 = ld_keep(src + i + 64, keep), v3 = ld_keep(src + i + 96, keep);
        st_stream(dst + i, v0, stream);
        st_stream(dst + i + 32, v1, stream);
        st_stream(dst + i + 64, v2, stream);
        st_stream(dst + i + 96, v3, stream);
    }
    for (; i < row_vec; i += 32) st_stream(dst + i, ld_keep(src + i, keep), stream);
}

constexpr int kGatherThreads = 256;

__global__ void gather_kernel(const uint4* __restrict__ x, uint4* __restrict__ x_perm,
                              const int32_t* __restrict__ slot_token,
                              const int32_t* __restrict__ offsets, int E, int row_vec) {
    const int total = offsets[E];
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < total; r += gridDim.x * wpb) {
        const int64_t t = slot_token[r];
        copy_row_warp(x + t * row_vec, x_perm + (int64_t)r * row_vec, row_vec, lane);
    }
}

// dst[i] = src[index[i]], rows of row_vec 16-byte words (expert-parallel
// regrouping of exchanged rows)
__global__ void gather_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ index, int64_t n,
                                   int row_vec, uint4* __restrict__ dst) {
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    for (int64_t r = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += (int64_t)gridDim.x * wpb)
        copy_row_warp(src + (int64_t)index[r] * row_vec, dst + r * row_vec, row_vec, lane);
}

__global__ void combine_kernel(const float* __restrict__ H, const int32_t* __restrict__ offsets,
                               int E, const int32_t* __restrict__ slot_token,
                               const float* __restrict__ slot_w, float* Y, int d, int64_t N,
                               int64_t max_rows) {
    const int total = (int)min64(offsets[E], max_rows);
    for (int r = blockIdx.x; r < total; r += gridDim.x) {
        const int64_t t = slot_token[r];
        if (t < 0 || t >= N) continue;
        const float a = slot_w[r];
        const float4* h = reinterpret_cast<const float4*>(H + (int64_t)r * d);
        for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
            const float4 v = h[c];
            red_add_v4(Y + t * d + 4 * c, a * v.x, a * v.y, a * v.z, a * v.w);
        }
    }
}

__global__ void mtile_prefix_kernel(int E, int bm, const int32_t* __restrict__ offsets,
                                    int32_t* __restrict__ mt_start) {
    __shared__ int warp_tot[33];
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        const int a = e < E ? offsets[e + 1] - offsets[e] : 0;
        const int mt = (a + bm - 1) / bm;
        int tot;
        const int ex = block_excl_scan(mt, warp_tot, &tot);
        if (e < E) mt_start[e] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) mt_start[E] = carry;
}

__global__ void zero_kernel(float4* __restrict__ Y, int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x)
        Y[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace

cudaError_t launch_dispatch(const moe_params& p, int64_t C, int bm, const int32_t* ids,
                            const float* w, int32_t* slot, int32_t* offsets, int32_t* L,
                            int32_t* acc, int32_t* slot_token, float* slot_w, const void* x,
                            void* x_perm, unsigned long long* counters, const Scratch& sc,
                            cudaStream_t st, const char** where) {
    const int E = p.E_r, k = p.k;
    const int n_tiles = sc.n_tiles;
    cudaError_t e;
    *where = "hist";
    hist_kernel<<<n_tiles, 256, sizeof(int) * E, st>>>(ids, p.N, k, E, sc.tile_tokens, n_tiles,
                                                        sc.hist, counters);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 32 warps share the per-expert tile scans; the expert-level scans need
    // one thread per expert (E <= kMaxExperts = 1024)
    *where = "scan";
    const bool by_weight = p.accept_order == MOE_ACCEPT_WEIGHT;
    const int scan_blocks = (E + kScanWarps - 1) / kScanWarps;
    scan_kernel<<<scan_blocks, 32 * kScanWarps, 0, st>>>(sc.hist, n_tiles, E, C, bm, L, acc, offsets, sc.mt_start,
                                                         by_weight ? sc.all_offsets : nullptr, counters);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int renorm = p.reject_policy == MOE_REJECT_RENORM;
    const bool reroute = p.reject_policy == MOE_REJECT_REROUTE;
    if (reroute) {
        // first choices (slots only), then reroute_depth rounds of offers for
        // the slots left free, then the final offsets, rows and statistics
        const int X = p.reroute_depth;
        *where = "assign";
        assign_kernel<<<n_tiles, 32, sizeof(int) * E, st>>>(ids, w, p.N, k, E, C, sc.tile_tokens, n_tiles, sc.hist,
                                                             offsets, nullptr, 0, 0, 1, slot, slot_token, slot_w,
                                                             counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        *where = "reroute init";
        const size_t nk = (size_t)p.N * k;
        if ((e = cudaMemsetAsync(sc.rr_e, 0xff, nk * 4, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(sc.rr_slot, 0xff, nk * 4, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(sc.rr_q, 0xff, nk * 4, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(sc.rr_next, 0, (size_t)p.N * 4, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(sc.rr_stop, 0, 4, st)) != cudaSuccess) return e;
        for (int r = 0; r < X; ++r) {
            *where = "reroute offer";
            reroute_offer_kernel<<<n_tiles, 256, sizeof(int) * E, st>>>(ids, slot, sc.cand, X, acc, C, p.N, k, E,
                                                                         sc.tile_tokens, n_tiles, sc.rr_e,
                                                                         sc.rr_next, sc.rr_offer, sc.hist, sc.rr_stop);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            *where = "reroute scan";
            reroute_scan_kernel<<<scan_blocks, 32 * kScanWarps, 0, st>>>(sc.hist, n_tiles, E, C, acc, sc.base,
                                                                          sc.rr_stop, counters);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            *where = "reroute assign";
            reroute_assign_kernel<<<n_tiles, 32, sizeof(int) * E, st>>>(sc.rr_offer, sc.cand, X, p.N, k, E, C,
                                                                         sc.tile_tokens, n_tiles, sc.hist, sc.base,
                                                                         sc.rr_e, sc.rr_slot, sc.rr_q, sc.rr_stop);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        *where = "reroute offsets";
        reroute_final_scan_kernel<<<1, 1024, 0, st>>>(E, bm, acc, offsets, sc.mt_start, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        *where = "reroute rows";
        reroute_rows_kernel<<<n_tiles, 32, 0, st>>>(ids, w, slot, sc.rr_e, sc.rr_slot, sc.rr_q, sc.cand_w, X, p.N,
                                                    k, E, sc.tile_tokens, offsets, slot_token, slot_w, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else if (!by_weight) {
        *where = "assign";
        assign_kernel<<<n_tiles, 32, sizeof(int) * E, st>>>(ids, w, p.N, k, E, C, sc.tile_tokens,
                                                             n_tiles, sc.hist, offsets, nullptr, renorm, 0, 0,
                                                             slot, slot_token, slot_w, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
        // every request placed in its expert's segment in token order, then
        // the C-th largest weight of each over-full expert selected, then the
        // accepted requests numbered and scattered
        *where = "place";
        assign_kernel<<<n_tiles, 32, sizeof(int) * E, st>>>(ids, w, p.N, k, E, INT64_MAX, sc.tile_tokens,
                                                             n_tiles, sc.hist, sc.all_offsets, nullptr, 0, 1, 0,
                                                             slot, sc.seg_req, sc.seg_w, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        *where = "select";
        prio_accept_kernel<<<E, 1024, 0, st>>>(k, C, sc.all_offsets, offsets, sc.seg_req, sc.seg_w, w,
                                               sc.sel_key, sc.sel_take, slot, slot_token, slot_w);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        *where = "tokens";
        prio_token_kernel<<<n_tiles, 32, 0, st>>>(ids, w, p.N, k, E, sc.tile_tokens, offsets, renorm, slot,
                                                  slot_w, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (x && x_perm) {
        *where = "gather";
        const int row_vec = (int)(p.d * esize(p.dtype) / 16);
        const int64_t rows = p.N * p.k;
        const int blocks = (int)min64((rows + kGatherThreads / 32 - 1) / (kGatherThreads / 32), (int64_t)num_sms() * 8);
        gather_kernel<<<blocks, kGatherThreads, 0, st>>>(static_cast<const uint4*>(x),
                                              static_cast<uint4*>(x_perm), slot_token, offsets, E,
                                              row_vec);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_count(const moe_params& p, const int32_t* ids, int32_t* L, int32_t* counts_out,
                         unsigned long long* counters, const Scratch& sc, cudaStream_t st) {
    const int E = p.E_r;
    hist_kernel<<<sc.n_tiles, 256, sizeof(int) * E, st>>>(ids, p.N, p.k, E, sc.tile_tokens,
                                                           sc.n_tiles, sc.hist, counters);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_scan_kernel<<<1, 1024, 0, st>>>(sc.hist, sc.n_tiles, E, L, counts_out);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_ranked(const moe_params& p, int64_t C, int bm, const int32_t* table,
                                   int rank, int n_ranks, int64_t n_group, const int32_t* ids,
                                   const float* w, int32_t* slot, int32_t* offsets, int32_t* L,
                                   int32_t* acc, int32_t* slot_token, float* slot_w,
                                   const void* x, void* x_perm, unsigned long long* counters,
                                   const Scratch& sc, cudaStream_t st, const char** where) {
    const int E = p.E_r, k = p.k;
    cudaError_t e;
    *where = "expert scan";
    const int threads = ((E + 31) / 32) * 32 < 64 ? 64 : ((E + 31) / 32) * 32;
    expert_scan_ranked_kernel<<<1, threads, 0, st>>>(E, C, bm, table, rank, n_ranks, n_group, L, acc,
                                                     offsets, sc.mt_start, sc.base, counters);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    *where = "assign";
    assign_kernel<<<sc.n_tiles, 32, sizeof(int) * E, st>>>(ids, w, p.N, k, E, C, sc.tile_tokens,
                                                            sc.n_tiles, sc.hist, offsets, sc.base,
                                                            p.reject_policy == MOE_REJECT_RENORM, 0, 0,
                                                            slot, slot_token, slot_w, counters);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (x && x_perm) {
        *where = "gather";
        const int row_vec = (int)(p.d * esize(p.dtype) / 16);
        const int64_t rows = p.N * p.k;
        const int blocks = (int)min64((rows + kGatherThreads / 32 - 1) / (kGatherThreads / 32), (int64_t)num_sms() * 8);
        gather_kernel<<<blocks, kGatherThreads, 0, st>>>(static_cast<const uint4*>(x),
                                              static_cast<uint4*>(x_perm), slot_token, offsets, E,
                                              row_vec);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gather_rows(const void* src, const int32_t* index, int64_t n_rows, int64_t row_bytes, void* dst,
                               cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    const int blocks =
        (int)min64((n_rows + kGatherThreads / 32 - 1) / (kGatherThreads / 32), (int64_t)num_sms() * 8);
    gather_rows_kernel<<<blocks, kGatherThreads, 0, st>>>(static_cast<const uint4*>(src), index, n_rows, (int)(row_bytes / 16),
                                               static_cast<uint4*>(dst));
    return cudaGetLastError();
}

cudaError_t launch_combine(const moe_params& p, const float* H, const int32_t* offsets,
                           const int32_t* slot_token, const float* slot_w, float* Y,
                           cudaStream_t st) {
    const int64_t rows = p.N * p.k;
    const int blocks = (int)min64(rows, (int64_t)num_sms() * 8);
    combine_kernel<<<blocks, 256, 0, st>>>(H, offsets, p.E_r, slot_token, slot_w, Y, p.d, p.N, rows);
    return cudaGetLastError();
}

cudaError_t launch_mtile_prefix(int E, int bm, const int32_t* offsets, int32_t* mt_start,
                                cudaStream_t st) {
    mtile_prefix_kernel<<<1, 1024, 0, st>>>(E, bm, offsets, mt_start);
    return cudaGetLastError();
}

cudaError_t launch_zero_f32(float* Y, int64_t n, cudaStream_t st) {
    const int64_t n4 = n / 4;
    const int blocks = (int)min64((n4 + 255) / 256, (int64_t)num_sms() * 8);
    if (blocks > 0) zero_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<float4*>(Y), n4);
    return cudaGetLastError();
}

}  // namespace moe
