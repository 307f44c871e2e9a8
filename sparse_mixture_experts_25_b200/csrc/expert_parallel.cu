// Expert parallelism ("LLM from scratch" ch. 36.7: expert parameters placed on
// different devices; after routing, token rows travel to the device of their
// expert and the expert outputs travel back).
//
// Rank r of R owns experts [r El, (r+1) El), El = E_r / R, and holds a
// contiguous shard of the routing group's tokens (rank order = token order).
// Acceptance is token order over the whole group (Algorithm 36.1), so with
// cum_s[e] = requests for e by ranks 0..s, rank s's accepted requests for e
// number acc[s][e] = min(C, cum_s[e]) - min(C, cum_{s-1}[e]).  Every rank
// derives the same table from the exchanged counts [R][E_r].
//
// The owner of expert e keeps its rows expert-major: owned expert j's rows
// from source 0, then source 1, ..., in token order within a source.  So the
// row a source s sends for expert e lands at
//   dest_base[e] + i,   dest_base[e] = (rows of the owner's earlier experts)
//                                      + min(C, cum_{s-1}[e]),
// i = its index among s's accepted rows of e.  ep_plan_kernel writes
// dest_base, the owner's expert offsets, the send / receive row counts per
// rank (the split sizes of an all-to-all) and, for an exchange that delivers
// rows source-major, the index that regroups them expert-major.
//
// The fused exchange writes each accepted row straight to its position in the
// owner's buffer (ep_dispatch_kernel; the buffer may be a peer GPU's memory
// reached over NVLink) and reads each expert output straight from the owner's
// output buffer into the weighted combine (ep_combine_kernel): no all-to-all,
// no regrouping, and no host round trip for split sizes.
#include <stdio.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ int plan_warp_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Block-wide exclusive scan over kPlanThreads values (returns the exclusive
// prefix; *total gets the sum).
__device__ int plan_block_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int inc = plan_warp_scan(v, lane);
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int wv = warp_tot[lane];
        const int wi = plan_warp_scan(wv, lane);
        warp_tot[lane] = wi - wv;
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    const int ex = inc - v + warp_tot[warp];
    *total = warp_tot[32];
    __syncthreads();
    return ex;
}

// One block, thread e = expert (E <= 1024).
//   dest_base [E]        position of this rank's first row of e in e's owner's buffer
//   local_offsets [El+1] the owned experts' rows in this rank's (owner's) buffer
//   send_rows [R]        rows this rank sends to each rank
//   recv_rows [R]        rows this rank receives from each rank
//   recv_base [R][El]    (scratch) source-major position of source s's first row of owned expert j
__global__ void ep_plan_kernel(const int32_t* __restrict__ counts_all, int R, int E, int rank, int64_t C,
                               int32_t* __restrict__ dest_base, int32_t* __restrict__ local_offsets,
                               int32_t* __restrict__ send_rows, int32_t* __restrict__ recv_rows,
                               int32_t* __restrict__ recv_base) {
    __shared__ int warp_tot[33];
    __shared__ int s_send[kMaxEpRanks], s_recv[kMaxEpRanks], s_seg0[kMaxEpRanks];
    const int e = threadIdx.x;
    const int El = E / R;
    if (threadIdx.x < kMaxEpRanks) {
        s_send[threadIdx.x] = 0;
        s_recv[threadIdx.x] = 0;
    }
    __syncthreads();
    int64_t cum = 0;
    int before = 0, mine = 0, tot = 0;
    if (e < E) {
        for (int s = 0; s < R; ++s) {
            const int64_t prev = cum < C ? cum : C;
            cum += counts_all[(int64_t)s * E + e];
            const int64_t now = cum < C ? cum : C;
            const int a = (int)(now - prev);  // acc[s][e]
            if (s < rank) before += a;
            if (s == rank) mine = a;
            if (e / El == rank) atomicAdd(&s_recv[s], a);
        }
        tot = (int)(cum < C ? cum : C);
        atomicAdd(&s_send[e / El], mine);
    }
    // exclusive prefix of tot within each owner's segment of El experts
    int seg_total;
    const int ex = plan_block_scan(e < E ? tot : 0, warp_tot, &seg_total);
    if (e < E && e % El == 0) s_seg0[e / El] = ex;
    __syncthreads();
    if (e < E) {
        const int local = ex - s_seg0[e / El];
        dest_base[e] = local + before;
        if (e / El == rank) local_offsets[e % El] = local;
        if (e / El == rank && e % El == El - 1) local_offsets[El] = local + tot;
    }
    if (threadIdx.x < R) {
        send_rows[threadIdx.x] = s_send[threadIdx.x];
        recv_rows[threadIdx.x] = s_recv[threadIdx.x];
    }
    // source-major layout of the received rows: source s's rows for owned
    // experts j = 0..El-1 follow each other; recv_base[s][j] = first of them
    if (recv_base && threadIdx.x == 0) {
        int pos = 0;
        for (int s = 0; s < R; ++s) {
            for (int j = 0; j < El; ++j) {
                const int eo = rank * El + j;
                int64_t c0 = 0;
                for (int q = 0; q < s; ++q) c0 += counts_all[(int64_t)q * E + eo];
                const int64_t c1 = c0 + counts_all[(int64_t)s * E + eo];
                recv_base[s * El + j] = pos;
                pos += (int)((c1 < C ? c1 : C) - (c0 < C ? c0 : C));
            }
        }
    }
}

// regroup[i] = the received (source-major) row that is row i of the owner's
// expert-major buffer, regroup_inv its inverse; one block per (owned expert
// j, source s).
__global__ void ep_regroup_kernel(const int32_t* __restrict__ counts_all, int R, int E, int rank, int64_t C,
                                  const int32_t* __restrict__ local_offsets, const int32_t* __restrict__ recv_base,
                                  int32_t* __restrict__ regroup, int32_t* __restrict__ regroup_inv) {
    const int El = E / R;
    const int j = blockIdx.x, s = blockIdx.y;
    const int eo = rank * El + j;
    int64_t c0 = 0;
    for (int q = 0; q < s; ++q) c0 += counts_all[(int64_t)q * E + eo];
    const int64_t c1 = c0 + counts_all[(int64_t)s * E + eo];
    const int before = (int)(c0 < C ? c0 : C);
    const int a = (int)((c1 < C ? c1 : C) - before);
    const int dst0 = local_offsets[j] + before;
    const int src0 = recv_base[s * El + j];
    for (int i = threadIdx.x; i < a; i += blockDim.x) {
        regroup[dst0 + i] = src0 + i;
        regroup_inv[src0 + i] = dst0 + i;
    }
}

// expert of row r of this rank's expert-grouped rows (offsets [E+1])
__device__ __forceinline__ int row_expert(const int32_t* __restrict__ offsets, int E, int r) {
    int lo = 0, hi = E - 1;  // last e with offsets[e] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= r) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Each accepted row of this rank (offsets / slot_token of its dispatch) is
// copied from x to its position in the owning rank's buffer recv_bufs[owner]
// (16-byte vectors; a peer GPU's memory when the owner is another GPU).
__global__ void ep_dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ offsets,
                                   const int32_t* __restrict__ slot_token, const int32_t* __restrict__ dest_base,
                                   int E, int El, int row_vec, void* const* __restrict__ recv_bufs, int64_t N) {
    __shared__ int s_e;
    const int total = offsets[E];
    for (int r = blockIdx.x; r < total; r += gridDim.x) {
        if (threadIdx.x == 0) s_e = row_expert(offsets, E, r);
        __syncthreads();
        const int e = s_e;
        __syncthreads();
        const int64_t t = slot_token[r];
        if (t < 0 || t >= N) continue;
        const int64_t pos = (int64_t)dest_base[e] + (r - offsets[e]);
        uint4* dst = static_cast<uint4*>(recv_bufs[e / El]) + pos * row_vec;
        const uint4* src = x + t * row_vec;
        for (int i = threadIdx.x; i < row_vec; i += blockDim.x) dst[i] = src[i];
    }
    // the rows are read by another GPU after this kernel: make them visible
    // beyond this device before the kernel completes
    __threadfence_system();
}

// Y[token] += weight * out_bufs[owner][position] for each accepted row of this
// rank (fp32 rows of d; Y zeroed by the caller or accumulated into).
__global__ void ep_combine_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ slot_token,
                                  const float* __restrict__ slot_w, const int32_t* __restrict__ dest_base, int E,
                                  int El, int d, const float* const* __restrict__ out_bufs, float* Y, int64_t N) {
    __shared__ int s_e;
    const int total = offsets[E];
    for (int r = blockIdx.x; r < total; r += gridDim.x) {
        if (threadIdx.x == 0) s_e = row_expert(offsets, E, r);
        __syncthreads();
        const int e = s_e;
        __syncthreads();
        const int64_t t = slot_token[r];
        if (t < 0 || t >= N) continue;
        const float a = slot_w[r];
        const int64_t pos = (int64_t)dest_base[e] + (r - offsets[e]);
        const float4* h = reinterpret_cast<const float4*>(out_bufs[e / El] + pos * d);
        for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
            const float4 v = h[c];
            red_add_v4(Y + t * d + 4 * c, a * v.x, a * v.y, a * v.z, a * v.w);
        }
    }
}

}  // namespace

cudaError_t launch_ep_plan(const moe_params& p, const int32_t* counts_all, int R, int rank, int64_t C,
                           int32_t* dest_base, int32_t* local_offsets, int32_t* send_rows, int32_t* recv_rows,
                           int32_t* recv_base, int32_t* regroup, int32_t* regroup_inv, cudaStream_t st) {
    ep_plan_kernel<<<1, kPlanThreads, 0, st>>>(counts_all, R, p.E_r, rank, C, dest_base, local_offsets, send_rows,
                                               recv_rows, recv_base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !regroup) return e;
    const int El = p.E_r / R;
    ep_regroup_kernel<<<dim3((unsigned)El, (unsigned)R), 128, 0, st>>>(counts_all, R, p.E_r, rank, C, local_offsets,
                                                                        recv_base, regroup, regroup_inv);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const moe_params& p, int R, const void* x, const int32_t* offsets,
                               const int32_t* slot_token, const int32_t* dest_base, void* const* recv_bufs,
                               cudaStream_t st) {
    const int row_vec = (int)(p.d * esize(p.dtype) / 16);
    const int blocks = (int)min64(p.N * p.k, (int64_t)num_sms() * 8);
    if (blocks <= 0) return cudaSuccess;
    ep_dispatch_kernel<<<blocks, 128, 0, st>>>(static_cast<const uint4*>(x), offsets, slot_token, dest_base, p.E_r,
                                               p.E_r / R, row_vec, recv_bufs, p.N);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const moe_params& p, int R, const int32_t* offsets, const int32_t* slot_token,
                              const float* slot_w, const int32_t* dest_base, const float* const* out_bufs, float* Y,
                              cudaStream_t st) {
    const int blocks = (int)min64(p.N * p.k, (int64_t)num_sms() * 8);
    if (blocks <= 0) return cudaSuccess;
    ep_combine_kernel<<<blocks, 256, 0, st>>>(offsets, slot_token, slot_w, dest_base, p.E_r, p.E_r / R, p.d, out_bufs,
                                              Y, p.N);
    return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

namespace {

moe_status ep_fail(cudaError_t e, const char* where) {
    char msg[192];
    snprintf(msg, sizeof(msg), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    record_error(msg);
    return MOE_ERR_CUDA;
}

moe_status ep_check(const moe_params* p, int32_t n_ranks) {
    size_t bytes = 0;
    moe_status s = moe_workspace_size(p, &bytes);  // the layer's parameter checks
    if (s != MOE_OK) return s;
    if (n_ranks < 1 || n_ranks > kMaxEpRanks || p->E_r % n_ranks) return MOE_ERR_INVALID_ARG;
    if (p->accept_order != MOE_ACCEPT_TOKEN || p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_ep_plan(const moe_params* p, const int32_t* counts_all, int32_t rank, int32_t n_ranks, int64_t C,
                       int32_t* local_offsets, int32_t* send_rows, int32_t* recv_rows, int32_t* regroup,
                       int32_t* regroup_inv, void* ws, moe_stream_t stream) {
    moe_status s = ep_check(p, n_ranks);
    if (s != MOE_OK) return s;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u)) return MOE_ERR_WORKSPACE;
    if (rank < 0 || rank >= n_ranks || C < 1 || !counts_all || !local_offsets || !send_rows || !recv_rows)
        return MOE_ERR_INVALID_ARG;
    if ((regroup != nullptr) != (regroup_inv != nullptr)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e = launch_ep_plan(*p, counts_all, n_ranks, rank, C, v.scratch.ep_dest, local_offsets, send_rows,
                                   recv_rows, v.scratch.ep_recv_base, regroup, regroup_inv, st);
    return e == cudaSuccess ? MOE_OK : ep_fail(e, "moe_ep_plan");
}

moe_status moe_ep_dispatch(const moe_params* p, int32_t n_ranks, const void* x, void* const* recv_bufs,
                           const void* ws, moe_stream_t stream) {
    moe_status s = ep_check(p, n_ranks);
    if (s != MOE_OK) return s;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u)) return MOE_ERR_WORKSPACE;
    if (p->N == 0) return MOE_OK;
    if (!x || !recv_bufs || (reinterpret_cast<uintptr_t>(x) & 15u)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, const_cast<void*>(ws), v);
    (void)cudaGetLastError();
    cudaError_t e = launch_ep_dispatch(*p, n_ranks, x, v.offsets, v.slot_token, v.scratch.ep_dest, recv_bufs, st);
    return e == cudaSuccess ? MOE_OK : ep_fail(e, "moe_ep_dispatch");
}

moe_status moe_ep_combine(const moe_params* p, int32_t n_ranks, const float* const* out_bufs, float* Y,
                          const void* ws, moe_stream_t stream) {
    moe_status s = ep_check(p, n_ranks);
    if (s != MOE_OK) return s;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u)) return MOE_ERR_WORKSPACE;
    if (p->N == 0) return MOE_OK;
    if (!out_bufs || !Y || (reinterpret_cast<uintptr_t>(Y) & 15u)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, const_cast<void*>(ws), v);
    (void)cudaGetLastError();
    cudaError_t e = launch_ep_combine(*p, n_ranks, v.offsets, v.slot_token, v.slot_w, v.scratch.ep_dest, out_bufs, Y,
                                      st);
    return e == cudaSuccess ? MOE_OK : ep_fail(e, "moe_ep_combine");
}

}  // extern "C"
