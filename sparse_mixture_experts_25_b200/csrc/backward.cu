// Backward pass of the sparse-MoE layer: gradients of
//   L = sum dY (.) Y + aux_coef * aux
// with the routing decisions of the forward held fixed ("LLM from scratch"
// ch. 36.3 combine, ch. 36.4 balance objective whose gradient reaches the
// router through the mean probabilities and the softmax Jacobian, ch. 36.6
// shared expert; vegetog "MoE token routing" sec. 3 SwiGLU expert).
//
// Per accepted path (row r of expert e, token t, combine weight wc):
//   z = W_g x, u = W_u x        recomputed on the tensor cores (fp32)
//   Gd = W_d^T dY_t             one grouped GEMM on the bf16 dY rows
//   dwc = <Gd, h>               = <dY_t, W_d h>, the combine-weight gradient
//   dh = wc Gd; dz = dh u SiLU'(z), du = dh SiLU(z)   (bf16 operands)
//   dx_perm = [dz | du] [W_g ; W_u]                   one grouped GEMM
//   dW_d = (wc dY)^T h, dW_g = dz^T x, dW_u = du^T x  per-expert GEMMs over
//                                                     the expert's rows (K)
// Router (one warp per token): dwc -> routing-weight gradient (overflow
// policy, renormalisation) -> probability gradient -> score gradient dG
// (softmax Jacobian) + the balance objective's term; dx += dG W_r,
// dW_r = dG^T X, db = column sums of dG.  With E_r a multiple of 64 (bf16)
// the two contractions run on the tensor cores, dG split into bf16 hi + lo
// parts (two K segments of one launch, W_r and X read as stored); otherwise
// fp32 CUDA-core kernels.  dx gathers the expert rows' dx_perm in token order.
//
// Layout choices for the tcgen05 GEMM (out = A B^T, A K-major): z and u run
// on the grouped kernel in store mode with the dimensions relabelled (its
// "d_f" is K, its "d" the output width; W_g, W_u are K-major as stored); W_d^T
// dY and [dz | du] [W_g ; W_u] read W_d, W_g and W_u as stored, as MN-major B
// operands (launch_tc_store_bmn), so no weight is transposed.  The shared
// expert's dense contractions still read transposed copies of its three
// matrices (one expert: small).  The weight gradients contract over an
// expert's rows, so their operands are transposed into blocks [E][C][Kmax]
// (expert e's C rows hold its R_e row values as columns, zero-padded to whole
// 64-wide K blocks; Kmax = the largest padded R_e, from the host offsets).
// Read as a grouped GEMM whose group e owns rows e C .. e C + C - 1, one
// launch per gradient computes every expert's dW_e = A_e B_e^T, each group
// contracting over its own K blocks only.
#include <cuda_bf16.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kTT = 64;  // transposition tile

__device__ __forceinline__ void ld8(const bf16* p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

unsigned grid_blocks(int64_t n) {  // 256-thread blocks for a grid-stride loop over n items
    const int64_t b = std::min<int64_t>((n + 255) / 256, (int64_t)num_sms() * 8);
    return (unsigned)std::max<int64_t>(b, 1);
}

// four consecutive elements as fp32 (8-byte bf16 or 16-byte fp32 accesses)
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const bf16* p) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st4(bf16* p, float4 v) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pk2(v.x, v.y), pk2(v.z, v.w));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// tstart[g]: first 64-row transposition tile of group g; nkb[g]: its 64-wide
// K blocks, max(1, ceil(R_g / 64)) (an empty group still gets one block of
// zeros, so its gradient tile is written).  One thread: G <= 1024.
__global__ void bwd_tables_kernel(int G, const int32_t* __restrict__ offsets, int32_t* __restrict__ tstart,
                                  int32_t* __restrict__ nkb) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t t = 0;
    for (int g = 0; g < G; ++g) {
        int32_t R = offsets[g + 1] - offsets[g];
        if (R < 0) R = 0;
        const int32_t n = R > 0 ? (R + kTT - 1) / kTT : 1;
        tstart[g] = t;
        nkb[g] = n;
        t += n;
    }
    tstart[G] = t;
}

// The caller's host copy of the forward's offsets, passed by value.
struct HostOffsets {
    int32_t v[kMaxRouterExperts + 1];
};

// The launches, the operand blocks and the fp32 per-expert contractions are
// sized from the caller's host copy of the offsets; the kernels read the
// device copy.  A copy that differs (stale, or from another forward) would
// give wrong gradients without any fault: record it as DEVERR_BOUNDS, which
// moe_backward_check reports.
__global__ void bwd_offsets_check_kernel(int G, const int32_t* __restrict__ offsets, HostOffsets host,
                                         unsigned long long* counters) {
    bool bad = false;
    for (int g = threadIdx.x; g <= G; g += blockDim.x) bad |= offsets[g] != host.v[g];
    if (__syncthreads_or(bad) && threadIdx.x == 0)
        atomicOr(counters + CNT_DEVICE_ERROR, (unsigned long long)DEVERR_BOUNDS);
}
// off[e] = e C for e = 0..E: groups of C consecutive rows
__global__ void bwd_strided_offsets_kernel(int E, int32_t C, int32_t* __restrict__ off) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) off[e] = e * C;
}

__global__ void bwd_single_group_kernel(int32_t n, int32_t* __restrict__ off) {
    if (threadIdx.x == 0) {
        off[0] = 0;
        off[1] = n;
    }
}

// Group-wise transposition: for group g (rows offsets[g] .. offsets[g+1]-1 of
// src [*, ld], columns 0..C-1), block g = dst + g gstride is [C, kstride]
// row-major with dst[c, r] = bf16(scale[row] src[row, c]) (scale optional)
// for r < R_g and zeros for r in [R_g, 64 nkb_g) (the group's K blocks).
// 64 x 64 tiles through shared memory, 16-byte global accesses; C, ld and
// kstride multiples of 8.
template <bool SCALE>
__global__ void __launch_bounds__(256)
    bwd_group_transpose_kernel(const bf16* __restrict__ src, int64_t ld, int64_t C, const int32_t* __restrict__ offsets,
                               const int32_t* __restrict__ tstart, int G, const float* __restrict__ scale,
                               bf16* __restrict__ dst, int64_t kstride, int64_t gstride) {
    __shared__ float tile[kTT][kTT + 1];
    const int bx = blockIdx.x;
    if (bx >= tstart[G]) return;
    int lo = 0, hi = G - 1;  // last group whose first tile is <= bx
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tstart[mid] <= bx) lo = mid;
        else hi = mid - 1;
    }
    const int g = lo;
    const int64_t R = offsets[g + 1] - offsets[g];
    const int64_t lr0 = (int64_t)(bx - tstart[g]) * kTT;
    const int64_t c0 = (int64_t)blockIdx.y * kTT;
    const int t = threadIdx.x, cc = (t & 7) * 8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = (t >> 3) + h * 32;
        const int64_t lr = lr0 + rr, c = c0 + cc;
        float v[8];
        if (lr < R && c < C) {
            const int64_t row = offsets[g] + lr;
            ld8(src + row * ld + c, v);
            if (SCALE) {
                const float s = scale[row];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] *= s;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) tile[rr][cc + i] = v[i];
    }
    __syncthreads();
    bf16* base = dst + (int64_t)g * gstride;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int oc = (t >> 3) + h * 32;
        const int64_t c = c0 + oc, lr = lr0 + cc;
        if (c < C && lr + 8 <= kstride) {
            uint4 q;
            q.x = pk2(tile[cc][oc], tile[cc + 1][oc]);
            q.y = pk2(tile[cc + 2][oc], tile[cc + 3][oc]);
            q.z = pk2(tile[cc + 4][oc], tile[cc + 5][oc]);
            q.w = pk2(tile[cc + 6][oc], tile[cc + 7][oc]);
            *reinterpret_cast<uint4*>(base + c * kstride + lr) = q;
        }
    }
}

// dst[b][c][r] (row stride ld_dst, batch stride bs_dst) = src[b][r][c] for a
// contiguous batch of [R, C] matrices; R, C, ld_dst multiples of 8.
__global__ void __launch_bounds__(256)
    bwd_batched_transpose_kernel(const bf16* __restrict__ src, int64_t R, int64_t C, bf16* __restrict__ dst,
                                 int64_t ld_dst, int64_t bs_dst) {
    __shared__ float tile[kTT][kTT + 1];
    const int64_t b = blockIdx.z;
    const bf16* s = src + b * R * C;
    bf16* o = dst + b * bs_dst;
    const int64_t r0 = (int64_t)blockIdx.x * kTT, c0 = (int64_t)blockIdx.y * kTT;
    const int t = threadIdx.x, cc = (t & 7) * 8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = (t >> 3) + h * 32;
        const int64_t r = r0 + rr, c = c0 + cc;
        float v[8];
        if (r < R && c < C) {
            ld8(s + r * C + c, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) tile[rr][cc + i] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int oc = (t >> 3) + h * 32;
        const int64_t c = c0 + oc, r = r0 + cc;
        if (c < C && r < R) {
            uint4 q;
            q.x = pk2(tile[cc][oc], tile[cc + 1][oc]);
            q.y = pk2(tile[cc + 2][oc], tile[cc + 3][oc]);
            q.z = pk2(tile[cc + 4][oc], tile[cc + 5][oc]);
            q.w = pk2(tile[cc + 6][oc], tile[cc + 7][oc]);
            *reinterpret_cast<uint4*>(o + c * ld_dst + r) = q;
        }
    }
}

// out[r, :] = scale[r] dY[tok(r), :] in T (bf16: rounded) for r < n (tok =
// slot_token[r], or r when slot_token is null; scale null: 1; n = *n_dev
// clamped to max_rows, or n_fixed).  One warp per row, 4 columns per step.
template <typename T>
__global__ void __launch_bounds__(256)
    bwd_gather_dy_kernel(const float* __restrict__ dY, int64_t d, const int32_t* __restrict__ slot_token,
                         const int32_t* __restrict__ n_dev, int64_t n_fixed, int64_t max_rows, int64_t n_tokens,
                         const float* __restrict__ scale, T* __restrict__ out) {
    int64_t n = n_fixed;
    if (n_dev) {
        n = *n_dev;
        if (n > max_rows) n = max_rows;
    }
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += (int64_t)gridDim.x * wpb) {
        const int64_t tok = slot_token ? (int64_t)slot_token[r] : r;
        const bool ok = tok >= 0 && tok < n_tokens;
        const float s = scale ? scale[r] : 1.f;
        const float* src = dY + (ok ? tok : 0) * d;
#pragma unroll 4
        for (int64_t c = lane; c < d / 4; c += 32) {
            float4 v = ok ? ld4(src + 4 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
            v.x *= s; v.y *= s; v.z *= s; v.w *= s;
            st4(out + r * d + 4 * c, v);
        }
    }
}

// SwiGLU backward of routed (or shared) rows r < n: with dh = wc[r] Gd[r],
//   dz = dh u SiLU'(z), du = dh SiLU(z)  ->  dzu[r] = [dz | du] (TO, 2 d_f)
//   dwc[r] = <Gd[r], h[r]>                  (fp32; skipped when dwc is null)
// SiLU(z) = z s(z), SiLU'(z) = s(z) (1 + z (1 - s(z))), s the logistic
// function.  wc null: weight 1.  TH: the forward's h type; TO: bf16 (rounded
// tensor-core operands) or fp32.  One warp per row.
template <typename TH, typename TO>
__global__ void __launch_bounds__(256)
    bwd_swiglu_kernel(const float* __restrict__ Z, const float* __restrict__ U, const float* __restrict__ Gd,
                      const TH* __restrict__ H, int64_t d_f, const float* __restrict__ wc,
                      const int32_t* __restrict__ n_dev, int64_t n_fixed, int64_t max_rows, TO* __restrict__ dzu,
                      float* __restrict__ dwc) {
    int64_t n = n_fixed;
    if (n_dev) {
        n = *n_dev;
        if (n > max_rows) n = max_rows;
    }
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += (int64_t)gridDim.x * wpb) {
        const float w = wc ? wc[r] : 1.f;
        float acc = 0.f;
        for (int64_t c = 4 * lane; c < d_f; c += 128) {
            const float4 z = ld4(Z + r * d_f + c), u = ld4(U + r * d_f + c), g = ld4(Gd + r * d_f + c);
            const float4 h = ld4(H + r * d_f + c);
            acc += g.x * h.x + g.y * h.y + g.z * h.z + g.w * h.w;
            const float zz[4] = {z.x, z.y, z.z, z.w}, uu[4] = {u.x, u.y, u.z, u.w}, gg[4] = {g.x, g.y, g.z, g.w};
            float dz[4], du[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float s = 1.f / (1.f + expf(-zz[i]));
                const float dh = w * gg[i];
                du[i] = dh * (zz[i] * s);
                dz[i] = dh * uu[i] * (s * (1.f + zz[i] * (1.f - s)));
            }
            st4(dzu + r * 2 * d_f + c, make_float4(dz[0], dz[1], dz[2], dz[3]));
            st4(dzu + r * 2 * d_f + d_f + c, make_float4(du[0], du[1], du[2], du[3]));
        }
        acc = warp_sum(acc);
        if (dwc && lane == 0) dwc[r] = acc;
    }
}

// Score gradient, one warp per token (see moe_backward in moe.h):
//   da_j  = dwc_j                     (policy 0, or no partial rejection)
//         = (dwc_j - sum_i dwc_i wc_i) / A,  wc = a / A,  A = sum_acc a   (policy 1)
//   RENORM / WLR: a_j = m_j p_j / s (s = sum over the chosen experts of p,
//                 m_j = 0 where the forward's weight is 0);
//                 dp_j = (m_j da_j - sum_i da_i a_i) / s
//   FULLPROB:     a_j = p_j, dp_j = da_j
//   dg_e = p_e (dp_e - sum_i p_i dp_i)
//        + aux_coef (E_r / N_valid) p_e (f_e - sum_i f_i p_i),  f = L / sum L
// Tokens with a non-finite score get dg = 0.
struct RouterBwd {
    const float* logits;  // [N, E] scores without bias
    const float* b_r;     // [E] or null
    const int32_t* ids;
    const float* w;
    const int32_t* slot;
    const int32_t* offsets;
    const float* dwc;     // [rows] per routed row
    const int32_t* L;     // [E] requests per expert
    const unsigned long long* counters;
    float* dG;            // [N, E]
    int64_t N;
    int E, k, norm, policy;
    float aux_coef;
    int64_t max_rows;
};

__global__ void __launch_bounds__(256) bwd_router_kernel(RouterBwd a) {
    __shared__ float sp[8][kMaxRouterExperts];
    __shared__ float sdp[8][kMaxRouterExperts];
    __shared__ float sf[kMaxRouterExperts];
    __shared__ float s_coef;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
    const bool aux = a.aux_coef != 0.f;
    if (threadIdx.x == 0) {
        const double req = (double)a.counters[CNT_REQUESTED];
        const double nv = (double)(a.N - (int64_t)a.counters[CNT_NONFINITE]);
        s_coef = (aux && req > 0 && nv > 0) ? (float)(a.aux_coef * E / nv) : 0.f;
    }
    __syncthreads();
    if (aux) {
        const double req = (double)a.counters[CNT_REQUESTED];
        for (int e = threadIdx.x; e < E; e += blockDim.x) sf[e] = req > 0 ? (float)(a.L[e] / req) : 0.f;
    }
    __syncthreads();
    const float coef = s_coef;
    float* p = sp[warp];
    float* dp = sdp[warp];
    for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < a.N; t += (int64_t)gridDim.x * 8) {
        float m = -INFINITY;
        bool bad = false;
        for (int e = lane; e < E; e += 32) {
            const float g = a.logits[t * E + e] + (a.b_r ? a.b_r[e] : 0.f);
            p[e] = g;
            bad |= !isfinite(g);
            m = fmaxf(m, g);
        }
        bad = __any_sync(0xffffffffu, bad);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (bad) {
            for (int e = lane; e < E; e += 32) a.dG[t * E + e] = 0.f;
            __syncwarp();
            continue;
        }
        float z = 0.f;
        for (int e = lane; e < E; e += 32) {
            const float v = expf(p[e] - m);
            p[e] = v;
            dp[e] = 0.f;
            z += v;
        }
        z = warp_sum(z);
        const float inv = 1.f / z;
        for (int e = lane; e < E; e += 32) p[e] *= inv;
        __syncwarp();
        // this lane's routing record
        int ej = -1;
        float aj = 0.f, dw = 0.f;
        bool acc = false;
        if (lane < a.k) {
            ej = a.ids[t * a.k + lane];
            if (ej >= E) ej = -1;
            if (ej >= 0) {
                aj = a.w[t * a.k + lane];
                const int s = a.slot[t * a.k + lane];
                if (s >= 0) {
                    const int64_t row = (int64_t)a.offsets[ej] + s;
                    if (row < a.max_rows) {
                        acc = true;
                        dw = a.dwc[row];
                    }
                }
            }
        }
        const bool chosen = ej >= 0;
        const float pj = chosen ? p[ej] : 0.f;
        const float ssel = warp_sum(pj);
        const float mj = (chosen && aj != 0.f) ? 1.f : 0.f;
        const float ap = a.norm == MOE_NORM_FULLPROB ? pj : (ssel > 0.f ? mj * pj / ssel : 0.f);
        const int req = __popc(__ballot_sync(0xffffffffu, chosen));
        const int rej = __popc(__ballot_sync(0xffffffffu, chosen && !acc));
        float da = acc ? dw : 0.f;
        if (a.policy == MOE_REJECT_RENORM && rej > 0 && rej < req) {
            const float A = warp_sum(acc ? ap : 0.f);
            const float S = warp_sum(acc && A > 0.f ? dw * (ap / A) : 0.f);
            da = (acc && A > 0.f) ? (dw - S) / A : 0.f;
        }
        float dpj;
        if (a.norm == MOE_NORM_FULLPROB) {
            dpj = da;
        } else {
            const float T = warp_sum(da * ap);
            dpj = ssel > 0.f ? (mj * da - T) / ssel : 0.f;
        }
        if (chosen) dp[ej] = dpj;
        __syncwarp();
        float spd = 0.f, sfp = 0.f;
        for (int e = lane; e < E; e += 32) {
            spd += p[e] * dp[e];
            if (aux) sfp += sf[e] * p[e];
        }
        spd = warp_sum(spd);
        if (aux) sfp = warp_sum(sfp);
        for (int e = lane; e < E; e += 32) {
            float g = p[e] * (dp[e] - spd);
            if (aux) g += coef * p[e] * (sf[e] - sfp);
            a.dG[t * E + e] = g;
        }
        __syncwarp();
    }
}

// db[e] = sum_t dG[t, e] in two deterministic phases: block (x, y) sums the
// rows of chunk y for 32 columns (8 warps over the rows, then shared memory)
// into part[y][e]; bwd_reduce_kernel then adds the chunks in order.
__global__ void __launch_bounds__(256) bwd_colsum_kernel(const float* __restrict__ dG, int64_t N, int E,
                                                         int64_t chunk, float* __restrict__ part) {
    __shared__ float sm[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const int64_t t0 = (int64_t)blockIdx.y * chunk;
    const int64_t t1 = min64(N, t0 + chunk);
    float s = 0.f;
    if (e < E)
        for (int64_t t = t0 + warp; t < t1; t += 8) s += dG[t * E + e];
    sm[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && e < E) {
        float v = 0.f;
        for (int i = 0; i < 8; ++i) v += sm[i][lane];
        part[(int64_t)blockIdx.y * E + e] = v;
    }
}

// out[i] = sum_{z < S} part[z n + i], z in order
__global__ void bwd_reduce_kernel(const float* __restrict__ part, int S, int64_t n, float* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int z = 0; z < S; ++z) v += part[(int64_t)z * n + i];
        out[i] = v;
    }
}

// dx[t] += sum over the token's accepted paths (rank order) of
// dxp[offsets[e] + slot] (+ dxs[t] when the shared expert ran).  One warp
// per token, float4 columns.
__global__ void __launch_bounds__(256)
    bwd_dx_kernel(float* __restrict__ dx, const float* __restrict__ dxp, const float* __restrict__ dxs,
                  const int32_t* __restrict__ ids, const int32_t* __restrict__ slot, const int32_t* __restrict__ offsets,
                  int64_t N, int64_t d, int k, int E, int64_t max_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t t = blockIdx.x * wpb + (threadIdx.x >> 5); t < N; t += (int64_t)gridDim.x * wpb) {
        float4* o = reinterpret_cast<float4*>(dx + t * d);
        // the token's accepted rows, resolved once: lane j holds path j's row
        // (-1: rejected), for paths j0 .. j0 + 31
        for (int j0 = 0; j0 < k; j0 += 32) {
            int64_t my_row = -1;
            if (j0 + lane < k) {
                const int e = ids[t * k + j0 + lane];
                const int s = slot[t * k + j0 + lane];
                if (e >= 0 && e < E && s >= 0) {
                    const int64_t row = (int64_t)offsets[e] + s;
                    if (row < max_rows) my_row = row;
                }
            }
            const int nj = min(32, k - j0);
            // every lane runs the same trip count (the shuffles need the whole warp)
            for (int64_t c0 = 0; c0 < d / 4; c0 += 32) {
                const int64_t c = c0 + lane;
                const bool in = c < d / 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (in) v = o[c];
                if (in && dxs && j0 == 0) {
                    const float4 q = reinterpret_cast<const float4*>(dxs + t * d)[c];
                    v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
                }
#pragma unroll 4
                for (int j = 0; j < nj; ++j) {
                    const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
                    if (row < 0 || !in) continue;
                    const float4 q = reinterpret_cast<const float4*>(dxp + row * d)[c];
                    v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
                }
                if (in) o[c] = v;
            }
        }
    }
}

// C[m, n] = sum_k A(m, k) B(n, k) with A(m, k) = A[m sam + k sak] and
// B(n, k) = B[n sbn + k sbk] (fp32 accumulate, C row-major with ldc): 64 x 64
// tiles, K steps of 16 through shared memory, 4 x 4 outputs per thread.  For
// the router's small contractions (one side is E_r wide).
__device__ __forceinline__ float as_f32(float v) { return v; }
__device__ __forceinline__ float as_f32(bf16 v) { return __bfloat162float(v); }

// blockIdx.z = K slice: slice z sums k in [z kchunk, (z+1) kchunk) into
// C + z cz (kchunk a multiple of 16; one slice: kchunk >= K, cz unused).
template <typename TA, typename TB>
__global__ void __launch_bounds__(256)
    bwd_simt_gemm_kernel(int64_t M, int64_t N, int64_t K, const TA* __restrict__ A, int64_t sam, int64_t sak,
                         const TB* __restrict__ B, int64_t sbn, int64_t sbk, float* __restrict__ C, int64_t ldc,
                         int64_t kchunk, int64_t cz, int accumulate) {
    __shared__ float As[16][64 + 4];
    __shared__ float Bs[16][64 + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t m0 = (int64_t)blockIdx.y * 64, n0 = (int64_t)blockIdx.x * 64;
    const int64_t kbeg = (int64_t)blockIdx.z * kchunk;
    K = min64(K, kbeg + kchunk);
    C += (int64_t)blockIdx.z * cz;
    float acc[4][4] = {};
    for (int64_t k0 = kbeg; k0 < K; k0 += 16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid + i * 256;
            int mm, kk;
            if (sak == 1) { kk = idx & 15; mm = idx >> 4; }
            else { mm = idx & 63; kk = idx >> 6; }
            const int64_t m = m0 + mm, kq = k0 + kk;
            As[kk][mm] = (m < M && kq < K) ? as_f32(A[m * sam + kq * sak]) : 0.f;
            int nn, kb;
            if (sbk == 1) { kb = idx & 15; nn = idx >> 4; }
            else { nn = idx & 63; kb = idx >> 6; }
            const int64_t n = n0 + nn, kr = k0 + kb;
            Bs[kb][nn] = (n < N && kr < K) ? as_f32(B[n * sbn + kr * sbk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[kk][ty * 4 + i];
                bv[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] += av[i] * bv[j];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = n0 + tx * 4 + j;
            if (n < N) C[m * ldc + n] = accumulate ? C[m * ldc + n] + acc[i][j] : acc[i][j];
        }
    }
}

// accumulate: C += the product instead of C = the product
template <typename TA, typename TB>
cudaError_t simt_gemm(int64_t M, int64_t N, int64_t K, const TA* A, int64_t sam, int64_t sak, const TB* B,
                      int64_t sbn, int64_t sbk, float* C, int64_t ldc, cudaStream_t st, int accumulate = 0) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64), 1);
    bwd_simt_gemm_kernel<TA, TB><<<grid, 256, 0, st>>>(M, N, K, A, sam, sak, B, sbn, sbk, C, ldc, K + 16, 0,
                                                       accumulate);
    return cudaGetLastError();
}

// K slices of a long contraction with few output tiles: enough slices for
// about two waves, at least 256 K per slice, at most kMaxSlices
constexpr int kMaxSlices = 16;

int k_slices(int64_t M, int64_t N, int64_t K) {
    const int64_t tiles = ((M + 63) / 64) * ((N + 63) / 64);
    int64_t s = (2 * (int64_t)num_sms() + tiles - 1) / tiles;
    s = std::min<int64_t>(s, std::max<int64_t>(1, K / 256));
    return (int)std::max<int64_t>(1, std::min<int64_t>(s, kMaxSlices));
}

// C [M, N] (row-major, ldc = N) = the K-sliced contraction: slices into
// part [S, M, N], then added in slice order (deterministic)
template <typename TA, typename TB>
cudaError_t simt_gemm_sliced(int64_t M, int64_t N, int64_t K, const TA* A, int64_t sam, int64_t sak, const TB* B,
                             int64_t sbn, int64_t sbk, float* C, float* part, cudaStream_t st) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    const int S = k_slices(M, N, K);
    if (S == 1) return simt_gemm(M, N, K, A, sam, sak, B, sbn, sbk, C, N, st);
    const int64_t kchunk = ((K + S - 1) / S + 15) / 16 * 16;
    const dim3 grid((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64), (unsigned)S);
    bwd_simt_gemm_kernel<TA, TB><<<grid, 256, 0, st>>>(M, N, K, A, sam, sak, B, sbn, sbk, part, N, kchunk, M * N, 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_reduce_kernel<<<grid_blocks(M * N), 256, 0, st>>>(part, S, M * N, C);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Workspace
// ---------------------------------------------------------------------------
bool router_on_tensor_cores(const moe_params& p);

struct BwdLayout {
    size_t tstart, nkb, mt_start, offs_d, offs_f, mt_d, mt_f, sh_off, sh_tstart, sh_nkb, counters;
    size_t logits, dG, part, part_db, dwc, doP, mt128, rsplit, rtab, dYp, Z, U, Gd, dzu, dxp, doT, xT, hT, dzT, duT;
    size_t dYs, Zs, Us, Gs, dzus, dxs, WsT_d, WsT_gu, dYsT, xsT, hsT, dzsT, dusT;
    int64_t Kmax, Kmax_sh;
    size_t total;
};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

int64_t up64(int64_t v) { return (v + kTT - 1) / kTT * kTT; }

// Kmax: the widest expert block of the weight-gradient operands (64 times the
// largest nkb), from the host offsets, else the bound min(capacity, N).
int64_t kmax_of(const moe_params& p, const int32_t* offsets_host) {
    int64_t m = kTT;
    if (p.dtype != MOE_BF16) return m;  // no transposed operands
    if (offsets_host) {
        for (int64_t g = 0; g < p.E_r; ++g) m = std::max(m, up64((int64_t)offsets_host[g + 1] - offsets_host[g]));
        return m;
    }
    int64_t C = p.N;
    moe_capacity(&p, &C);
    return std::max(m, up64(std::min<int64_t>(C, p.N)));
}

// bf16 layers: tensor-core operands in bf16, transposed weights and the
// [E][C][Kmax] weight-gradient operands.  fp32 layers: fp32 rows only (their
// CUDA-core contractions read any layout through strides).
BwdLayout bwd_layout(const moe_params& p, int64_t Kmax) {
    const bool b16 = p.dtype == MOE_BF16;
    const size_t N = (size_t)p.N, d = (size_t)p.d, df = (size_t)p.d_f, E = (size_t)p.E_r;
    const size_t rows = N * (size_t)p.k;
    const size_t ds = p.d_f_shared > 0 ? (size_t)p.d_f_shared : 0;
    const size_t es = b16 ? 2 : 4;     // element size of the operand buffers
    const size_t tb = b16 ? 1 : 0;     // bf16-only buffers
    BwdLayout L{};
    L.Kmax = Kmax;
    L.Kmax_sh = std::max<int64_t>(kTT, up64(p.N));
    const size_t K = (size_t)Kmax, Ks = (size_t)L.Kmax_sh;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = up256(off + bytes);
        return o;
    };
    L.tstart = take((E + 1) * 4);
    L.nkb = take(E * 4);
    L.mt_start = take((E + 1) * 4);
    L.offs_d = take((E + 1) * 4);
    L.offs_f = take((E + 1) * 4);
    L.mt_d = take((E + 1) * 4);
    L.mt_f = take((E + 1) * 4);
    L.sh_off = take(2 * 4);
    L.sh_tstart = take(2 * 4);
    L.sh_nkb = take(4);
    L.counters = take(CNT_COUNT * 8);
    L.logits = take(N * E * 4);
    L.dG = take(N * E * 4);
    L.part = take((size_t)kMaxSlices * E * d * 4);
    L.part_db = take((size_t)kMaxSlices * E * 4);
    L.dwc = take(rows * 4);
    L.doP = take((1 - tb) * rows * d * 4);
    L.mt128 = take((E + 1) * 4);  // 128-row tile prefix for the MN-major weight contractions
    // the score gradient's bf16 parts for the tensor-core router contractions
    L.rsplit = take(router_on_tensor_cores(p) ? 4 * N * E * 2 : 0);
    L.rtab = take(8 * 4);
    L.dYp = take(rows * d * es);
    L.Z = take(rows * df * 4);
    L.U = take(rows * df * 4);
    L.Gd = take(rows * df * 4);
    L.dzu = take(rows * 2 * df * es);
    L.dxp = take(rows * d * 4);
    L.doT = take(tb * E * d * K * 2);
    L.xT = take(tb * E * d * K * 2);
    L.hT = take(tb * E * df * K * 2);
    L.dzT = take(tb * E * df * K * 2);
    L.duT = take(tb * E * df * K * 2);
    if (ds) {
        L.dYs = take(tb * N * d * 2);
        L.Zs = take(N * ds * 4);
        L.Us = take(N * ds * 4);
        L.Gs = take(N * ds * 4);
        L.dzus = take(N * 2 * ds * es);
        L.dxs = take(N * d * 4);
        L.WsT_d = take(tb * ds * d * 2);
        L.WsT_gu = take(tb * d * 2 * ds * 2);
        L.dYsT = take(tb * d * Ks * 2);
        L.xsT = take(tb * d * Ks * 2);
        L.hsT = take(tb * ds * Ks * 2);
        L.dzsT = take(tb * ds * Ks * 2);
        L.dusT = take(tb * ds * Ks * 2);
    }
    L.total = off;
    return L;
}

thread_local char g_bwd_error[256] = "";

moe_status bwd_fail(cudaError_t e, const char* where) {
    snprintf(g_bwd_error, sizeof(g_bwd_error), "moe_backward %s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    record_error(g_bwd_error);
    return MOE_ERR_CUDA;
}

bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

moe_status bwd_check(const moe_params* p) {
    size_t ws = 0;
    const moe_status s = moe_workspace_size(p, &ws);  // the forward's parameter checks
    if (s != MOE_OK) return s;
    if (p->E_r > kMaxRouterExperts || p->k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;  // rerouted weights: no backward
    if (p->N > (int64_t)65535 * 64) return MOE_ERR_UNSUPPORTED;  // grid rows of the router contractions
    // rows of the grouped weight-gradient GEMMs (E_r groups of d or d_f rows)
    if ((int64_t)p->E_r * std::max(p->d, p->d_f) >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// blocks of 8 warps for one warp per item, at most 16 per SM (grid-stride)
unsigned grid_for(int64_t items_per_block_units, int64_t n) {
    int64_t b = (n + items_per_block_units - 1) / items_per_block_units;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (b > cap) b = cap;
    if (b < 1) b = 1;
    return (unsigned)b;
}

// Router chain of the backward: score gradient dG (bwd_router_kernel), then
// dx = dG W_r (written), dW_r = dG^T X (sliced over the tokens) and db_r.
// The score gradient dG [N, E] (fp32) as two bf16 parts, hi = bf16(dG) and
// lo = bf16(dG - hi), each also transposed to [E, N]: the tensor-core router
// contractions multiply both parts by the exact bf16 W_r or x and add them, so
// dG enters with about 16 mantissa bits instead of 8.  32 x 32 tiles through
// shared memory, so both layouts are written row-contiguously.
__global__ void __launch_bounds__(256)
    bwd_split_scores_kernel(const float* __restrict__ dG, int64_t N, int E, bf16* __restrict__ hi,
                            bf16* __restrict__ lo, bf16* __restrict__ hiT, bf16* __restrict__ loT) {
    __shared__ float tile[32][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
    const int64_t t0 = (int64_t)blockIdx.y * 32;
    const int e0 = blockIdx.x * 32;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t t = t0 + ty + 8 * i;
        const int e = e0 + tx;
        float v = 0.f;
        if (t < N && e < E) {
            v = dG[t * E + e];
            const bf16 h = __float2bfloat16_rn(v);
            hi[t * E + e] = h;
            lo[t * E + e] = __float2bfloat16_rn(v - __bfloat162float(h));
        }
        tile[ty + 8 * i][tx] = v;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = e0 + ty + 8 * i;
        const int64_t t = t0 + tx;
        if (t < N && e < E) {
            const float v = tile[tx][ty + 8 * i];
            const bf16 h = __float2bfloat16_rn(v);
            hiT[(int64_t)e * N + t] = h;
            loT[(int64_t)e * N + t] = __float2bfloat16_rn(v - __bfloat162float(h));
        }
    }
}

// One-group row offsets and 128-row tile prefixes for the two router
// contractions: t[0..1] = {0, N}, t[2..3] = {0, tiles(N)}, t[4..5] = {0, E},
// t[6..7] = {0, tiles(E)}.
__global__ void bwd_router_tables_kernel(int32_t* t, int32_t N, int32_t E) {
    if (threadIdx.x == 0) {
        t[0] = 0;
        t[1] = N;
        t[2] = 0;
        t[3] = (N + 127) / 128;
        t[4] = 0;
        t[5] = E;
        t[6] = 0;
        t[7] = (E + 127) / 128;
    }
}

// Whether the bf16 router contractions run on the tensor cores: E_r a
// multiple of the 64-wide K block and 16-byte rows of the transposed scores.
bool router_on_tensor_cores(const moe_params& p) {
    return p.dtype == MOE_BF16 && p.E_r % 64 == 0 && p.N % 8 == 0 && p.N > 0 && p.d % 8 == 0;
}

template <typename T>
moe_status router_backward(const moe_params& p, float aux_coef, const T* x, const T* W_r, const float* b_r,
                           const WsView& v, const float* logits, const float* dwc, float* dG, float* part,
                           float* part_db, const moe_grads* gr, cudaStream_t st, bf16* split = nullptr,
                           int32_t* tables = nullptr, unsigned long long* counters = nullptr) {
    const int64_t N = p.N, d = p.d, E = p.E_r;
    RouterBwd ra{};
    ra.logits = logits;
    ra.b_r = b_r;
    ra.ids = v.ids;
    ra.w = v.w;
    ra.slot = v.slot;
    ra.offsets = v.offsets;
    ra.dwc = dwc;
    ra.L = v.L;
    ra.counters = v.counters;
    ra.dG = dG;
    ra.N = N;
    ra.E = (int)E;
    ra.k = p.k;
    ra.norm = p.norm;
    ra.policy = p.reject_policy;
    ra.aux_coef = aux_coef;
    ra.max_rows = N * p.k;
    bwd_router_kernel<<<grid_for(8, N), 256, 0, st>>>(ra);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return bwd_fail(e, "router");
    if (split && tables) {
        // tensor cores: dx = dG W_r and dW_r = dG^T x, each as hi + lo parts of
        // dG in two K segments of one launch, W_r and x read as stored (MN-major)
        bf16 *hi = split, *lo = split + N * E, *hiT = split + 2 * N * E, *loT = split + 3 * N * E;
        bwd_split_scores_kernel<<<dim3((unsigned)((E + 31) / 32), (unsigned)((N + 31) / 32)), 256, 0, st>>>(
            dG, N, (int)E, hi, lo, hiT, loT);
        bwd_router_tables_kernel<<<1, 32, 0, st>>>(tables, (int32_t)N, (int32_t)E);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "score split");
        int status = MOE_OK;
        moe_params q = p;  // one group of N rows, K = E_r
        q.E_r = 1;
        q.k = 1;
        q.d_f_shared = 0;
        e = launch_tc_store_bmn(q, d, E, hi, E, W_r, lo, E, W_r, tables, tables + 2, gr->dx, counters, st, &status);
        if (e != cudaSuccess) return bwd_fail(e, "router dx (tcgen05)");
        q.N = E;  // one group of E_r rows, K = N tokens, split over the tokens
        const bool split_k = tc_store_bmn_split(q, d, N, true) > 1;
        if (split_k && (e = cudaMemsetAsync(gr->dW_r, 0, sizeof(float) * E * d, st)) != cudaSuccess)
            return bwd_fail(e, "memset");
        e = launch_tc_store_bmn(q, d, N, hiT, N, x, loT, N, x, tables + 4, tables + 6, gr->dW_r, counters, st,
                                &status, split_k);
        if (e != cudaSuccess) return bwd_fail(e, "router dW_r (tcgen05)");
    } else {
        e = simt_gemm<float, T>(N, d, E, dG, E, 1, W_r, 1, d, gr->dx, d, st);
        if (e == cudaSuccess)  // K = N tokens, few output tiles: sliced over the tokens
            e = simt_gemm_sliced<float, T>(E, d, N, dG, 1, E, x, 1, d, gr->dW_r, part, st);
        if (e != cudaSuccess) return bwd_fail(e, "router contractions");
    }
    if (gr->db_r) {
        const int64_t chunk = (N + kMaxSlices - 1) / kMaxSlices;
        bwd_colsum_kernel<<<dim3((unsigned)((E + 31) / 32), (unsigned)kMaxSlices), 256, 0, st>>>(dG, N, (int)E, chunk,
                                                                                                 part_db);
        bwd_reduce_kernel<<<grid_blocks(E), 256, 0, st>>>(part_db, kMaxSlices, E, gr->db_r);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "db");
    }
    return MOE_OK;
}

// The fp32 layer: every contraction on the CUDA cores (bwd_simt_gemm_kernel
// reads the weights and rows in place through strides), one launch per expert
// and contraction; nothing is rounded.
moe_status backward_f32(const moe_params& p, float aux_coef, const int32_t* off_h, const float* x, const float* W_r,
                        const float* b_r, const float* W_g, const float* W_u, const float* W_d, const float* Ws_g,
                        const float* Ws_u, const float* Ws_d, const float* dY, const WsView& v, const moe_grads* gr,
                        char* b, const BwdLayout& L, cudaStream_t st) {
    const int64_t N = p.N, d = p.d, df = p.d_f, E = p.E_r, rows = N * p.k;
    auto F32 = [&](size_t o) { return reinterpret_cast<float*>(b + o); };
    float *logits = F32(L.logits), *dG = F32(L.dG), *dwc = F32(L.dwc), *dYp = F32(L.dYp), *doP = F32(L.doP);
    float *Z = F32(L.Z), *U = F32(L.U), *Gd = F32(L.Gd), *dzu = F32(L.dzu), *dxp = F32(L.dxp);
    const float* xp = static_cast<const float*>(v.x_perm);
    const float* hp = static_cast<const float*>(v.h);
    const int32_t* n_rows = v.offsets + E;
    cudaError_t e = simt_gemm<float, float>(N, E, d, x, d, 1, W_r, d, 1, logits, E, st);
    if (e != cudaSuccess) return bwd_fail(e, "scores");
    // dY rows of the accepted paths, and wc dY for dW_d
    bwd_gather_dy_kernel<float><<<grid_for(8, rows), 256, 0, st>>>(dY, d, v.slot_token, n_rows, 0, rows, N, nullptr,
                                                                   dYp);
    bwd_gather_dy_kernel<float><<<grid_for(8, rows), 256, 0, st>>>(dY, d, v.slot_token, n_rows, 0, rows, N, v.slot_w,
                                                                   doP);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "dY rows");
    for (int64_t g = 0; g < E; ++g) {
        const int64_t o = off_h[g], R = off_h[g + 1] - off_h[g];
        if (R == 0) continue;
        const float* Wg = W_g + g * df * d;
        const float* Wu = W_u + g * df * d;
        const float* Wd = W_d + g * d * df;
        e = simt_gemm<float, float>(R, df, d, xp + o * d, d, 1, Wg, d, 1, Z + o * df, df, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(R, df, d, xp + o * d, d, 1, Wu, d, 1, U + o * df, df, st);
        // W_d^T dY: B(j, i) = W_d[i, j]
        if (e == cudaSuccess) e = simt_gemm<float, float>(R, df, d, dYp + o * d, d, 1, Wd, 1, df, Gd + o * df, df, st);
        if (e != cudaSuccess) return bwd_fail(e, "z, u, W_d^T dY");
    }
    bwd_swiglu_kernel<float, float><<<grid_for(8, rows), 256, 0, st>>>(Z, U, Gd, hp, df, v.slot_w, n_rows, 0, rows,
                                                                       dzu, dwc);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "SwiGLU backward");
    for (int64_t g = 0; g < E; ++g) {  // dx rows = dz W_g + du W_u: B(i, j) = W[j, i]
        const int64_t o = off_h[g], R = off_h[g + 1] - off_h[g];
        if (R == 0) continue;
        e = simt_gemm<float, float>(R, d, df, dzu + o * 2 * df, 2 * df, 1, W_g + g * df * d, 1, d, dxp + o * d, d, st);
        if (e == cudaSuccess)
            e = simt_gemm<float, float>(R, d, df, dzu + o * 2 * df + df, 2 * df, 1, W_u + g * df * d, 1, d,
                                        dxp + o * d, d, st, 1);
        if (e != cudaSuccess) return bwd_fail(e, "dx rows");
    }
    moe_status s = router_backward<float>(p, aux_coef, x, W_r, b_r, v, logits, dwc, dG, F32(L.part), F32(L.part_db),
                                          gr, st);
    if (s != MOE_OK) return s;
    float* dxs = nullptr;
    if (p.d_f_shared > 0) {
        const int64_t ds = p.d_f_shared;
        const float* hs = static_cast<const float*>(v.h_shared);
        float *Zs = F32(L.Zs), *Us = F32(L.Us), *Gs = F32(L.Gs), *dzus = F32(L.dzus);
        dxs = F32(L.dxs);
        e = simt_gemm<float, float>(N, ds, d, x, d, 1, Ws_g, d, 1, Zs, ds, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(N, ds, d, x, d, 1, Ws_u, d, 1, Us, ds, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(N, ds, d, dY, d, 1, Ws_d, 1, ds, Gs, ds, st);
        if (e != cudaSuccess) return bwd_fail(e, "shared z, u, W_d^T dY");
        bwd_swiglu_kernel<float, float><<<grid_for(8, N), 256, 0, st>>>(Zs, Us, Gs, hs, ds, nullptr, nullptr, N, N,
                                                                        dzus, nullptr);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = simt_gemm<float, float>(N, d, ds, dzus, 2 * ds, 1, Ws_g, 1, d, dxs, d, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(N, d, ds, dzus + ds, 2 * ds, 1, Ws_u, 1, d, dxs, d, st, 1);
        // weight gradients over the tokens: A(m, t) and B(n, t) read column-wise
        if (e == cudaSuccess) e = simt_gemm<float, float>(d, ds, N, dY, 1, d, hs, 1, ds, gr->dWs_d, ds, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(ds, d, N, dzus, 1, 2 * ds, x, 1, d, gr->dWs_g, d, st);
        if (e == cudaSuccess) e = simt_gemm<float, float>(ds, d, N, dzus + ds, 1, 2 * ds, x, 1, d, gr->dWs_u, d, st);
        if (e != cudaSuccess) return bwd_fail(e, "shared expert");
    }
    bwd_dx_kernel<<<grid_for(8, N), 256, 0, st>>>(gr->dx, dxp, dxs, v.ids, v.slot, v.offsets, N, d, p.k, (int)E, rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "dx");
    for (int64_t g = 0; g < E; ++g) {  // weight gradients over the expert's rows
        const int64_t o = off_h[g], R = off_h[g + 1] - off_h[g];
        float* gWd = gr->dW_d + g * d * df;
        float* gWg = gr->dW_g + g * df * d;
        float* gWu = gr->dW_u + g * df * d;
        if (R == 0) {
            e = cudaMemsetAsync(gWd, 0, sizeof(float) * d * df, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(gWg, 0, sizeof(float) * d * df, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(gWu, 0, sizeof(float) * d * df, st);
        } else {
            e = simt_gemm<float, float>(d, df, R, doP + o * d, 1, d, hp + o * df, 1, df, gWd, df, st);
            if (e == cudaSuccess)
                e = simt_gemm<float, float>(df, d, R, dzu + o * 2 * df, 1, 2 * df, xp + o * d, 1, d, gWg, d, st);
            if (e == cudaSuccess)
                e = simt_gemm<float, float>(df, d, R, dzu + o * 2 * df + df, 1, 2 * df, xp + o * d, 1, d, gWu, d, st);
        }
        if (e != cudaSuccess) return bwd_fail(e, "weight gradients");
    }
    return MOE_OK;
}

// offsets_host: a non-decreasing prefix from 0 to at most N k
bool offsets_valid(const moe_params& p, const int32_t* o) {
    if (o[0] != 0) return false;
    for (int64_t e = 0; e < p.E_r; ++e)
        if (o[e + 1] < o[e]) return false;
    return (int64_t)o[p.E_r] <= p.N * p.k;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_backward_workspace_size(const moe_params* p, const int32_t* offsets_host, size_t* bytes) {
    const moe_status s = bwd_check(p);
    if (s != MOE_OK) return s;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    if (offsets_host && p->N > 0 && !offsets_valid(*p, offsets_host)) return MOE_ERR_INVALID_ARG;
    *bytes = bwd_layout(*p, kmax_of(*p, p->N > 0 ? offsets_host : nullptr)).total;
    return MOE_OK;
}

moe_status moe_backward(const moe_params* p, float aux_coef, const int32_t* offsets_host, const void* x,
                        const void* W_r, const float* b_r, const void* W_g, const void* W_u, const void* W_d,
                        const void* Ws_g, const void* Ws_u, const void* Ws_d, const float* dY, const void* ws,
                        const moe_grads* gr, void* bws, size_t bws_bytes, moe_stream_t stream) {
    moe_status s = bwd_check(p);
    if (s != MOE_OK) return s;
    if (!ws || !al16(ws) || !bws || !al16(bws)) return MOE_ERR_WORKSPACE;
    if (!gr || !offsets_host) return MOE_ERR_INVALID_ARG;
    const bool sh = p->d_f_shared > 0;
    if ((p->N > 0 && !gr->dx) || !gr->dW_r || !gr->dW_g || !gr->dW_u || !gr->dW_d) return MOE_ERR_INVALID_ARG;
    if (sh && (!gr->dWs_g || !gr->dWs_u || !gr->dWs_d)) return MOE_ERR_INVALID_ARG;
    if (!(aux_coef == aux_coef)) return MOE_ERR_INVALID_ARG;
    const int64_t N = p->N, d = p->d, df = p->d_f, E = p->E_r, k = p->k;
    const int64_t rows = N * k;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    const int64_t dfs = sh ? p->d_f_shared : 0;
    if (N == 0) {  // no tokens: every weight gradient is zero
        (void)cudaGetLastError();
        e = cudaMemsetAsync(gr->dW_r, 0, sizeof(float) * E * d, st);
        if (e == cudaSuccess && gr->db_r) e = cudaMemsetAsync(gr->db_r, 0, sizeof(float) * E, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gr->dW_g, 0, sizeof(float) * E * df * d, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gr->dW_u, 0, sizeof(float) * E * df * d, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gr->dW_d, 0, sizeof(float) * E * df * d, st);
        if (e == cudaSuccess && sh) e = cudaMemsetAsync(gr->dWs_g, 0, sizeof(float) * dfs * d, st);
        if (e == cudaSuccess && sh) e = cudaMemsetAsync(gr->dWs_u, 0, sizeof(float) * dfs * d, st);
        if (e == cudaSuccess && sh) e = cudaMemsetAsync(gr->dWs_d, 0, sizeof(float) * dfs * d, st);
        return e == cudaSuccess ? MOE_OK : bwd_fail(e, "memset");
    }
    if (!x || !W_r || !W_g || !W_u || !W_d || !dY) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(W_r) || !al16(W_g) || !al16(W_u) || !al16(W_d) || !al16(dY) || !al16(gr->dx) ||
        !al16(gr->dW_g) || !al16(gr->dW_u) || !al16(gr->dW_d))
        return MOE_ERR_INVALID_ARG;
    if (sh && (!Ws_g || !Ws_u || !Ws_d || !al16(Ws_g) || !al16(Ws_u) || !al16(Ws_d) || !al16(gr->dWs_g) ||
               !al16(gr->dWs_u) || !al16(gr->dWs_d)))
        return MOE_ERR_INVALID_ARG;
    // (an empty forward writes no offsets, so they are checked only now)
    if (!offsets_valid(*p, offsets_host)) return MOE_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(*p, kmax_of(*p, offsets_host));
    if (bws_bytes < L.total) return MOE_ERR_WORKSPACE;
    (void)cudaGetLastError();  // clear a stale non-sticky error left by earlier unrelated calls

    WsView v;
    make_view(*p, const_cast<void*>(ws), v);
    char* b = static_cast<char*>(bws);
    e = cudaMemsetAsync(b + L.counters, 0, CNT_COUNT * 8, st);
    if (e != cudaSuccess) return bwd_fail(e, "memset");
    {
        HostOffsets ho;
        for (int64_t g = 0; g <= p->E_r; ++g) ho.v[g] = offsets_host[g];
        bwd_offsets_check_kernel<<<1, 256, 0, st>>>(p->E_r, v.offsets,
                                                    ho, reinterpret_cast<unsigned long long*>(b + L.counters));
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "offsets check");
    }
    if (p->dtype == MOE_F32)
        return backward_f32(*p, aux_coef, offsets_host, static_cast<const float*>(x), static_cast<const float*>(W_r),
                            b_r, static_cast<const float*>(W_g), static_cast<const float*>(W_u),
                            static_cast<const float*>(W_d), static_cast<const float*>(Ws_g),
                            static_cast<const float*>(Ws_u), static_cast<const float*>(Ws_d), dY, v, gr, b, L, st);
    auto I32 = [&](size_t o) { return reinterpret_cast<int32_t*>(b + o); };
    auto F32 = [&](size_t o) { return reinterpret_cast<float*>(b + o); };
    auto B16 = [&](size_t o) { return reinterpret_cast<bf16*>(b + o); };
    int32_t *tstart = I32(L.tstart), *nkb = I32(L.nkb), *mt_start = I32(L.mt_start);
    int32_t *offs_d = I32(L.offs_d), *offs_f = I32(L.offs_f), *mt_d = I32(L.mt_d), *mt_f = I32(L.mt_f);
    auto* counters = reinterpret_cast<unsigned long long*>(b + L.counters);
    float* logits = F32(L.logits);
    float* dG = F32(L.dG);
    float* dwc = F32(L.dwc);
    bf16 *dYp = B16(L.dYp), *dzu = B16(L.dzu);
    int32_t* mt128 = I32(L.mt128);
    float *Z = F32(L.Z), *U = F32(L.U), *Gd = F32(L.Gd), *dxp = F32(L.dxp);
    bf16 *doT = B16(L.doT), *xT = B16(L.xT), *hT = B16(L.hT), *dzT = B16(L.dzT), *duT = B16(L.duT);
    const bf16* xp = static_cast<const bf16*>(v.x_perm);
    const bf16* hp = static_cast<const bf16*>(v.h);
    const int32_t* n_rows = v.offsets + E;  // accepted rows, on the device
    const int64_t Kmax = L.Kmax;
    int status = MOE_OK;
    // transposition tiles of the routed rows (host count, same rule as bwd_tables_kernel)
    int64_t n_tiles = 0;
    for (int64_t g = 0; g < E; ++g) {
        const int64_t R = offsets_host[g + 1] - offsets_host[g];
        n_tiles += R > 0 ? (R + kTT - 1) / kTT : 1;
    }

    bwd_tables_kernel<<<1, 32, 0, st>>>((int)E, v.offsets, tstart, nkb);
    bwd_strided_offsets_kernel<<<1, 256, 0, st>>>((int)E, (int32_t)d, offs_d);
    bwd_strided_offsets_kernel<<<1, 256, 0, st>>>((int)E, (int32_t)df, offs_f);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "tables");
    e = launch_mtile_prefix((int)E, tc_tile_rows(*p), v.offsets, mt_start, st);
    if (e == cudaSuccess) e = launch_mtile_prefix((int)E, 128, v.offsets, mt128, st);
    if (e != cudaSuccess) return bwd_fail(e, "tables");
    // router scores (bias added in the router kernel): tensor cores when the
    // fp32 epilogue's 4-column groups tile E_r, else the CUDA-core GEMM
    if (E % 4 == 0)
        e = launch_tc_dense(N, E, d, x, W_r, logits, counters, st, &status);
    else
        e = simt_gemm<bf16, bf16>(N, E, d, static_cast<const bf16*>(x), d, 1, static_cast<const bf16*>(W_r), d, 1,
                                  logits, E, st);
    if (e != cudaSuccess) return bwd_fail(e, "scores");
    // dY rows of the accepted paths, bf16
    bwd_gather_dy_kernel<bf16><<<grid_for(8, rows), 256, 0, st>>>(dY, d, v.slot_token, n_rows, 0, rows, N, nullptr,
                                                                  dYp);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "dY rows");

    // row-grouped contractions on the grouped tcgen05 kernel (store mode):
    // its output width is q.d and its K is q.d_f
    ExpertWeights W0{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    moe_params q = *p;
    q.d_f_shared = 0;
    q.d = (int32_t)df;
    q.d_f = (int32_t)d;
    W0.W_d = W_g;
    e = launch_tc_down(q, DOWN_STORE, N, xp, nullptr, v.offsets, mt_start, W0, nullptr, nullptr, nullptr, Z, counters,
                       st, &status);
    if (e != cudaSuccess) return bwd_fail(e, "z (tcgen05)");
    W0.W_d = W_u;
    e = launch_tc_down(q, DOWN_STORE, N, xp, nullptr, v.offsets, mt_start, W0, nullptr, nullptr, nullptr, U, counters,
                       st, &status);
    if (e != cudaSuccess) return bwd_fail(e, "u (tcgen05)");
    // W_d^T dY: W_d [E, d, d_f] read as stored (MN-major B operand)
    e = launch_tc_store_bmn(*p, df, d, dYp, d, W_d, nullptr, 0, nullptr, v.offsets, mt128, Gd, counters, st,
                            &status);
    if (e != cudaSuccess) return bwd_fail(e, "W_d^T dY (tcgen05)");
    bwd_swiglu_kernel<bf16, bf16><<<grid_for(8, rows), 256, 0, st>>>(Z, U, Gd, hp, df, v.slot_w, n_rows, 0, rows, dzu,
                                                                     dwc);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "SwiGLU backward");
    // dx rows = dz W_g + du W_u: W_g, W_u [E, d_f, d] read as stored (MN-major
    // B operands), dz and du the two halves of each [dz | du] row
    e = launch_tc_store_bmn(*p, d, df, dzu, 2 * df, W_g, dzu + df, 2 * df, W_u, v.offsets, mt128, dxp, counters,
                            st, &status);
    if (e != cudaSuccess) return bwd_fail(e, "dx rows (tcgen05)");

    const bf16* xb = static_cast<const bf16*>(x);
    const bool rtc = router_on_tensor_cores(*p);
    if ((s = router_backward<bf16>(*p, aux_coef, xb, static_cast<const bf16*>(W_r), b_r, v, logits, dwc, dG,
                                   F32(L.part), F32(L.part_db), gr, st, rtc ? B16(L.rsplit) : nullptr,
                                   rtc ? I32(L.rtab) : nullptr, counters)) != MOE_OK)
        return s;

    // shared expert: weight 1 on every token
    float* dxs = nullptr;
    if (sh) {
        const int64_t Ks = L.Kmax_sh;
        bf16 *dYs = B16(L.dYs), *dzus = B16(L.dzus), *WsT_d = B16(L.WsT_d), *WsT_gu = B16(L.WsT_gu);
        float *Zs = F32(L.Zs), *Us = F32(L.Us), *Gs = F32(L.Gs);
        dxs = F32(L.dxs);
        int32_t *sh_off = I32(L.sh_off), *sh_ts = I32(L.sh_tstart), *sh_nkb = I32(L.sh_nkb);
        bwd_single_group_kernel<<<1, 32, 0, st>>>((int32_t)N, sh_off);
        bwd_tables_kernel<<<1, 32, 0, st>>>(1, sh_off, sh_ts, sh_nkb);
        bwd_gather_dy_kernel<bf16><<<grid_for(8, N), 256, 0, st>>>(dY, d, nullptr, nullptr, N, N, N, nullptr, dYs);
        bwd_batched_transpose_kernel<<<dim3((unsigned)((d + kTT - 1) / kTT), (unsigned)((dfs + kTT - 1) / kTT), 1), 256,
                                       0, st>>>(static_cast<const bf16*>(Ws_d), d, dfs, WsT_d, d, 0);
        bwd_batched_transpose_kernel<<<dim3((unsigned)((dfs + kTT - 1) / kTT), (unsigned)((d + kTT - 1) / kTT), 1), 256,
                                       0, st>>>(static_cast<const bf16*>(Ws_g), dfs, d, WsT_gu, 2 * dfs, 0);
        bwd_batched_transpose_kernel<<<dim3((unsigned)((dfs + kTT - 1) / kTT), (unsigned)((d + kTT - 1) / kTT), 1), 256,
                                       0, st>>>(static_cast<const bf16*>(Ws_u), dfs, d, WsT_gu + dfs, 2 * dfs, 0);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "shared transposes");
        e = launch_tc_dense(N, dfs, d, x, Ws_g, Zs, counters, st, &status);
        if (e == cudaSuccess) e = launch_tc_dense(N, dfs, d, x, Ws_u, Us, counters, st, &status);
        if (e == cudaSuccess) e = launch_tc_dense(N, dfs, d, dYs, WsT_d, Gs, counters, st, &status);
        if (e != cudaSuccess) return bwd_fail(e, "shared z, u, W_d^T dY (tcgen05)");
        bwd_swiglu_kernel<bf16, bf16><<<grid_for(8, N), 256, 0, st>>>(Zs, Us, Gs, static_cast<const bf16*>(v.h_shared),
                                                                      dfs, nullptr, nullptr, N, N, dzus, nullptr);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "shared SwiGLU backward");
        e = launch_tc_dense(N, d, 2 * dfs, dzus, WsT_gu, dxs, counters, st, &status);
        if (e != cudaSuccess) return bwd_fail(e, "shared dx (tcgen05)");
        // weight gradients over all tokens (K = N, zero-padded to whole 64-wide blocks)
        bf16 *dYsT = B16(L.dYsT), *xsT = B16(L.xsT), *hsT = B16(L.hsT), *dzsT = B16(L.dzsT), *dusT = B16(L.dusT);
        const unsigned tiles_sh = (unsigned)(Ks / kTT);
        bwd_group_transpose_kernel<false><<<dim3(tiles_sh, (unsigned)((d + kTT - 1) / kTT)), 256, 0, st>>>(
            dYs, d, d, sh_off, sh_ts, 1, nullptr, dYsT, Ks, 0);
        bwd_group_transpose_kernel<false><<<dim3(tiles_sh, (unsigned)((d + kTT - 1) / kTT)), 256, 0, st>>>(
            xb, d, d, sh_off, sh_ts, 1, nullptr, xsT, Ks, 0);
        bwd_group_transpose_kernel<false><<<dim3(tiles_sh, (unsigned)((dfs + kTT - 1) / kTT)), 256, 0, st>>>(
            static_cast<const bf16*>(v.h_shared), dfs, dfs, sh_off, sh_ts, 1, nullptr, hsT, Ks, 0);
        bwd_group_transpose_kernel<false><<<dim3(tiles_sh, (unsigned)((dfs + kTT - 1) / kTT)), 256, 0, st>>>(
            dzus, 2 * dfs, dfs, sh_off, sh_ts, 1, nullptr, dzsT, Ks, 0);
        bwd_group_transpose_kernel<false><<<dim3(tiles_sh, (unsigned)((dfs + kTT - 1) / kTT)), 256, 0, st>>>(
            dzus + dfs, 2 * dfs, dfs, sh_off, sh_ts, 1, nullptr, dusT, Ks, 0);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "shared row transposes");
        e = launch_tc_dense(d, dfs, Ks, dYsT, hsT, gr->dWs_d, counters, st, &status);
        if (e == cudaSuccess) e = launch_tc_dense(dfs, d, Ks, dzsT, xsT, gr->dWs_g, counters, st, &status);
        if (e == cudaSuccess) e = launch_tc_dense(dfs, d, Ks, dusT, xsT, gr->dWs_u, counters, st, &status);
        if (e != cudaSuccess) return bwd_fail(e, "shared weight gradients (tcgen05)");
    }

    // dx: router part (written above) + expert rows + shared expert
    bwd_dx_kernel<<<grid_for(8, N), 256, 0, st>>>(gr->dx, dxp, dxs, v.ids, v.slot, v.offsets, N, d, (int)k, (int)E,
                                                  rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "dx");

    // weight gradients: operands transposed into [E][C][Kmax] blocks (expert
    // e's rows as columns, zeros up to its last K block), then one grouped
    // GEMM per gradient whose group e is the expert's C rows
    {
        const dim3 gd((unsigned)n_tiles, (unsigned)((d + kTT - 1) / kTT));
        const dim3 gf((unsigned)n_tiles, (unsigned)((df + kTT - 1) / kTT));
        bwd_group_transpose_kernel<true><<<gd, 256, 0, st>>>(dYp, d, d, v.offsets, tstart, (int)E, v.slot_w, doT, Kmax,
                                                             d * Kmax);
        bwd_group_transpose_kernel<false><<<gd, 256, 0, st>>>(xp, d, d, v.offsets, tstart, (int)E, nullptr, xT, Kmax,
                                                              d * Kmax);
        bwd_group_transpose_kernel<false><<<gf, 256, 0, st>>>(hp, df, df, v.offsets, tstart, (int)E, nullptr, hT, Kmax,
                                                              df * Kmax);
        bwd_group_transpose_kernel<false><<<gf, 256, 0, st>>>(dzu, 2 * df, df, v.offsets, tstart, (int)E, nullptr, dzT,
                                                              Kmax, df * Kmax);
        bwd_group_transpose_kernel<false><<<gf, 256, 0, st>>>(dzu + df, 2 * df, df, v.offsets, tstart, (int)E, nullptr,
                                                              duT, Kmax, df * Kmax);
        if ((e = cudaGetLastError()) != cudaSuccess) return bwd_fail(e, "row transposes");
    }
    moe_params qw = *p;  // groups of d rows (dW_d) or d_f rows (dW_g, dW_u), K = Kmax
    qw.d_f_shared = 0;
    qw.k = 1;
    qw.d_f = (int32_t)Kmax;
    qw.N = E * d;
    qw.d = (int32_t)df;
    e = launch_mtile_prefix((int)E, tc_tile_rows(qw), offs_d, mt_d, st);
    if (e != cudaSuccess) return bwd_fail(e, "tables");
    W0.W_d = hT;
    e = launch_tc_down(qw, DOWN_STORE, qw.N, doT, nullptr, offs_d, mt_d, W0, nullptr, nullptr, nullptr, gr->dW_d,
                       counters, st, &status, nkb);
    if (e != cudaSuccess) return bwd_fail(e, "dW_d (tcgen05)");
    qw.N = E * df;
    qw.d = (int32_t)d;
    e = launch_mtile_prefix((int)E, tc_tile_rows(qw), offs_f, mt_f, st);
    if (e != cudaSuccess) return bwd_fail(e, "tables");
    W0.W_d = xT;
    e = launch_tc_down(qw, DOWN_STORE, qw.N, dzT, nullptr, offs_f, mt_f, W0, nullptr, nullptr, nullptr, gr->dW_g,
                       counters, st, &status, nkb);
    if (e == cudaSuccess)
        e = launch_tc_down(qw, DOWN_STORE, qw.N, duT, nullptr, offs_f, mt_f, W0, nullptr, nullptr, nullptr, gr->dW_u,
                           counters, st, &status, nkb);
    if (e != cudaSuccess) return bwd_fail(e, "dW_g, dW_u (tcgen05)");
    return MOE_OK;
}

moe_status moe_backward_check(const moe_params* p, const void* bws, moe_stream_t stream) {
    const moe_status s = bwd_check(p);
    if (s != MOE_OK) return s;
    if (!bws || !al16(bws)) return MOE_ERR_WORKSPACE;
    unsigned long long cnt[CNT_COUNT];
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the counters sit at the same offset whatever Kmax is
    cudaError_t e = cudaMemcpyAsync(cnt, static_cast<const char*>(bws) + bwd_layout(*p, kTT).counters, sizeof(cnt),
                                    cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return bwd_fail(e, "check");
    if (cnt[CNT_DEVICE_ERROR] & DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (cnt[CNT_DEVICE_ERROR] & DEVERR_BOUNDS) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // extern "C"
