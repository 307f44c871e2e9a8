// Soft MoE forward ("LLM from scratch" ch. 36.6, Soft Mixture of Experts).
//
// What it computes: S = E_r p slots, slot s = e p + i belongs to expert e;
//   Z  = X Phi^T                      [N, S]  slot scores
//   D  = softmax of Z over tokens     (each slot's column sums to one)
//   C  = softmax of Z over slots      (each token's row sums to one)
//   Xs = D^T X                        [S, d]  slot inputs (token mixtures)
//   Ys_s = E_{e(s)}(Xs_s)             SwiGLU expert of the slot's owner
//   Y  = C Ys                         [N, d]
//
// Design: the three contractions run on the tcgen05 dense GEMM
// (out = A B^T with both operands K-major), so the operands are laid out for
// it: D is written transposed ([S, N], K = tokens), X is transposed once
// ([d, N]), and the slot outputs are transposed ([d, S], K = slots).  The
// experts run on the grouped tcgen05 GEMMs with p rows per expert (the slot
// rows are already grouped by expert).  D, C, Xs and Ys enter the tensor cores
// as bf16; scores, softmax statistics and every accumulation are fp32.
// Small kernels: column statistics of Z (per-chunk max / sum, merged), the
// transposed dispatch weights, the row softmax, bf16 transposes in 64 x 64
// shared-memory tiles, an fp32 -> bf16 conversion.
#include <cuda_bf16.h>
#include <stdio.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kT = 32;  // grid limit unit of the slot dimension

// Column statistics of Z in two steps.  Partial: one block per 32 slots x
// 256 tokens; each warp takes 32 tokens (independent loads, lane = slot),
// computes their max and sum of exp, and the 8 warps merge into one partial
// (max, sum) per slot and chunk.  Merge: one thread per slot combines its
// chunks into m_s = max_t Z[t, s] and l_s = sum_t exp(Z[t, s] - m_s).
constexpr int kColChunk = 256;

__global__ void soft_colstat_partial_kernel(const float* __restrict__ Z, int64_t N, int S,
                                            float* __restrict__ pmax, float* __restrict__ psum) {
    __shared__ float sm[8][32], sl[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s = blockIdx.x * 32 + lane;
    const int64_t t0 = (int64_t)blockIdx.y * kColChunk + warp * 32;
    float v[32];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int64_t t = t0 + i;
        v[i] = (s < S && t < N) ? Z[t * S + s] : -INFINITY;
        m = fmaxf(m, v[i]);
    }
    float l = 0.f;
    if (m != -INFINITY) {
#pragma unroll
        for (int i = 0; i < 32; ++i) l += expf(v[i] - m);
    }
    sm[warp][lane] = m;
    sl[warp][lane] = l;
    __syncthreads();
    if (warp == 0 && s < S) {
        float M = -INFINITY;
        for (int w = 0; w < 8; ++w) M = fmaxf(M, sm[w][lane]);
        float L = 0.f;
        if (M != -INFINITY)
            for (int w = 0; w < 8; ++w)
                if (sl[w][lane] > 0.f) L += sl[w][lane] * expf(sm[w][lane] - M);
        pmax[(int64_t)blockIdx.y * S + s] = M;
        psum[(int64_t)blockIdx.y * S + s] = L;
    }
}

__global__ void soft_colstat_merge_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                          int n_chunks, int S, float* __restrict__ colmax,
                                          float* __restrict__ colsum) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= S) return;
    float M = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, pmax[(int64_t)c * S + s]);
    float L = 0.f;
    if (M != -INFINITY)
        for (int c = 0; c < n_chunks; ++c) {
            const float l = psum[(int64_t)c * S + s];
            if (l > 0.f) L += l * expf(pmax[(int64_t)c * S + s] - M);
        }
    colmax[s] = M;
    colsum[s] = L;
}

// C[t, s] = exp(Z[t, s] - m_t) / l_t in bf16; one warp per token, three
// passes over the token's row in 16-byte loads (max, sum of exp, write)
__global__ void soft_combine_w_kernel(const float* __restrict__ Z, int64_t N, int S,
                                      __nv_bfloat16* __restrict__ Cw) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= N) return;
    const float4* z = reinterpret_cast<const float4*>(Z + t * S);
    const int S4 = S / 4;
    float m = -INFINITY;
#pragma unroll 4
    for (int i = lane; i < S4; i += 32) {
        const float4 v = z[i];
        m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
#pragma unroll 4
    for (int i = lane; i < S4; i += 32) {
        const float4 v = z[i];
        l += expf(v.x - m) + expf(v.y - m) + expf(v.z - m) + expf(v.w - m);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    const float inv = 1.f / l;
    uint2* out = reinterpret_cast<uint2*>(Cw + t * S);
#pragma unroll 4
    for (int i = lane; i < S4; i += 32) {
        const float4 v = z[i];
        __nv_bfloat162 a = __floats2bfloat162_rn(expf(v.x - m) * inv, expf(v.y - m) * inv);
        __nv_bfloat162 b = __floats2bfloat162_rn(expf(v.z - m) * inv, expf(v.w - m) * inv);
        out[i] = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    }
}

// out[c, r] = f(in[r, c]) in bf16 for a row-major [R, Cc] input (R, Cc
// multiples of 8): 64 x 64 tiles through shared memory, every global access a
// 16-byte chunk of 8 elements (a warp covers four 128-byte row segments).
// SOFTMAX: f(z) = exp(z - colmax[c]) / colsum[c] (the dispatch weights, read
// from the scores), else the identity.
constexpr int kTT = 64;

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename Tin, bool SOFTMAX>
__global__ void __launch_bounds__(256) soft_transpose_kernel(const Tin* __restrict__ in, int64_t R, int64_t Cc,
                                                             const float* __restrict__ colmax,
                                                             const float* __restrict__ colsum,
                                                             __nv_bfloat16* __restrict__ out) {
    __shared__ float tile[kTT][kTT + 1];
    const int64_t r0 = (int64_t)blockIdx.x * kTT, c0 = (int64_t)blockIdx.y * kTT;
    const int t = threadIdx.x;
    const int cc = (t & 7) * 8;  // chunk column inside the tile
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = (t >> 3) + h * 32;
        const int64_t r = r0 + rr, c = c0 + cc;
        float v[8];
        if (r < R && c < Cc) {
            load8(in + r * Cc + c, v);
            if (SOFTMAX) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = expf(v[i] - colmax[c + i]) / colsum[c + i];
            }
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
        const int oc = (t >> 3) + h * 32;   // output row = input column
        const int64_t c = c0 + oc, r = r0 + cc;
        if (c < Cc && r < R) {
            uint4 q;
            __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = __floats2bfloat162_rn(tile[cc + 2 * i][oc], tile[cc + 2 * i + 1][oc]);
            *reinterpret_cast<uint4*>(out + c * R + r) = q;
        }
    }
}

__global__ void soft_to_bf16_kernel(const float4* __restrict__ in, uint2* __restrict__ out, int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = in[i];
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        out[i] = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    }
}

__global__ void soft_offsets_kernel(int E, int p, int32_t* __restrict__ offsets) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = e * p;
}

struct SoftLayout {
    size_t counters, offsets, mt_start, Z, colmax, colsum, pmax, psum, Dt, Cw, Xt, S32, Xs, h, Yst, total;
};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

SoftLayout soft_layout(const moe_soft_params& p) {
    const size_t N = (size_t)p.N, S = (size_t)p.E_r * p.p, d = (size_t)p.d, df = (size_t)p.d_f;
    const size_t E = (size_t)p.E_r;
    SoftLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = up256(off + bytes);
        return o;
    };
    L.counters = take(CNT_COUNT * 8);
    L.offsets = take((E + 1) * 4);
    L.mt_start = take((E + 1) * 4);
    L.Z = take(N * S * 4);
    L.colmax = take(S * 4);
    L.colsum = take(S * 4);
    L.pmax = take((N + kColChunk - 1) / kColChunk * S * 4);
    L.psum = take((N + kColChunk - 1) / kColChunk * S * 4);
    L.Dt = take(S * N * 2);
    L.Cw = take(N * S * 2);
    L.Xt = take(d * N * 2);
    L.S32 = take(S * d * 4);  // slot inputs, then slot outputs, fp32
    L.Xs = take(S * d * 2);
    L.h = take(S * df * 2);
    L.Yst = take(d * S * 2);
    L.total = off;
    return L;
}

moe_status soft_check(const moe_soft_params* p) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (p->N < 0 || p->d <= 0 || p->d_f <= 0 || p->E_r <= 0 || p->p <= 0) return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_F32 && p->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;  // the slot contractions are bf16 tcgen05 GEMMs
    if (p->E_r > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    const int64_t S = (int64_t)p->E_r * p->p;
    // 16-byte rows for every tensor-core operand (K = d, tokens, slots)
    if (p->d % 8 || p->d_f % 8 || p->N % 8 || S % 8) return MOE_ERR_UNSUPPORTED;
    // grid limits of the column-statistics and transposition launches
    if (p->N > (int64_t)65535 * kColChunk || S > (int64_t)65535 * kT) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

thread_local char g_soft_error[256] = "";

moe_status soft_fail(cudaError_t e, const char* where) {
    snprintf(g_soft_error, sizeof(g_soft_error), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    record_error(g_soft_error);
    return MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_soft_workspace_size(const moe_soft_params* p, size_t* bytes) {
    moe_status s = soft_check(p);
    if (s != MOE_OK) return s;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = soft_layout(*p).total;
    return MOE_OK;
}

moe_status moe_soft_forward(const moe_soft_params* p, const void* x, const void* Phi, const void* W_g,
                            const void* W_u, const void* W_d, float* Y, void* ws, moe_stream_t stream) {
    moe_status s = soft_check(p);
    if (s != MOE_OK) return s;
    auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!ws || !al16(ws)) return MOE_ERR_WORKSPACE;
    if (p->N == 0) return MOE_OK;
    if (!x || !Phi || !W_g || !W_u || !W_d || !Y) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(Phi) || !al16(W_g) || !al16(W_u) || !al16(W_d) || !al16(Y)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const SoftLayout L = soft_layout(*p);
    char* b = static_cast<char*>(ws);
    auto* counters = reinterpret_cast<unsigned long long*>(b + L.counters);
    auto* offsets = reinterpret_cast<int32_t*>(b + L.offsets);
    auto* mt_start = reinterpret_cast<int32_t*>(b + L.mt_start);
    auto* Z = reinterpret_cast<float*>(b + L.Z);
    auto* colmax = reinterpret_cast<float*>(b + L.colmax);
    auto* colsum = reinterpret_cast<float*>(b + L.colsum);
    auto* Dt = reinterpret_cast<__nv_bfloat16*>(b + L.Dt);
    auto* Cw = reinterpret_cast<__nv_bfloat16*>(b + L.Cw);
    auto* Xt = reinterpret_cast<__nv_bfloat16*>(b + L.Xt);
    auto* S32 = reinterpret_cast<float*>(b + L.S32);
    auto* Xs = reinterpret_cast<__nv_bfloat16*>(b + L.Xs);
    auto* h = b + L.h;
    auto* Yst = reinterpret_cast<__nv_bfloat16*>(b + L.Yst);
    const int64_t N = p->N;
    const int S = p->E_r * p->p;
    const int d = p->d;
    (void)cudaGetLastError();
    cudaError_t e = cudaMemsetAsync(counters, 0, CNT_COUNT * 8, st);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward memset");
    int status = MOE_OK;
    // slot scores
    e = launch_tc_dense(N, S, d, x, Phi, Z, counters, st, &status);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward scores (tcgen05)");
    // dispatch weights (transposed) and combine weights
    const int n_chunks = (int)((N + kColChunk - 1) / kColChunk);
    soft_colstat_partial_kernel<<<dim3((unsigned)((S + 31) / 32), (unsigned)n_chunks), 256, 0, st>>>(
        Z, N, S, reinterpret_cast<float*>(b + L.pmax), reinterpret_cast<float*>(b + L.psum));
    soft_colstat_merge_kernel<<<(S + 255) / 256, 256, 0, st>>>(reinterpret_cast<const float*>(b + L.pmax),
                                                                reinterpret_cast<const float*>(b + L.psum),
                                                                n_chunks, S, colmax, colsum);
    soft_transpose_kernel<float, true><<<dim3((unsigned)((N + kTT - 1) / kTT), (unsigned)((S + kTT - 1) / kTT)),
                                         256, 0, st>>>(Z, N, S, colmax, colsum, Dt);
    soft_combine_w_kernel<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(Z, N, S, Cw);
    // slot inputs Xs = D^T X: X transposed so that K = tokens is contiguous
    soft_transpose_kernel<__nv_bfloat16, false><<<dim3((unsigned)((N + kTT - 1) / kTT),
                                                        (unsigned)((d + kTT - 1) / kTT)), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), N, d, nullptr, nullptr, Xt);
    if ((e = cudaGetLastError()) != cudaSuccess) return soft_fail(e, "moe_soft_forward weights");
    e = launch_tc_dense(S, d, N, Dt, Xt, S32, counters, st, &status);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward slot inputs (tcgen05)");
    const int64_t n4 = (int64_t)S * d / 4;
    soft_to_bf16_kernel<<<(unsigned)min64((n4 + 255) / 256, (int64_t)num_sms() * 8), 256, 0, st>>>(
        reinterpret_cast<const float4*>(S32), reinterpret_cast<uint2*>(Xs), n4);
    // experts on their slots: p consecutive slot rows per expert
    moe_params q{};
    q.N = S;
    q.d = d;
    q.d_f = p->d_f;
    q.E_r = p->E_r;
    q.k = 1;
    q.dtype = MOE_BF16;
    soft_offsets_kernel<<<1, 256, 0, st>>>(p->E_r, p->p, offsets);
    if ((e = cudaGetLastError()) != cudaSuccess) return soft_fail(e, "moe_soft_forward slots");
    e = launch_mtile_prefix(p->E_r, tc_tile_rows(q), offsets, mt_start, st);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward prefix");
    ExpertWeights W{W_g, W_u, W_d, nullptr, nullptr, nullptr};
    e = launch_tc_gate_up(q, Xs, nullptr, offsets, mt_start, W, h, nullptr, nullptr, counters, st, &status);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward gate/up (tcgen05)");
    e = launch_tc_down(q, DOWN_STORE, S, h, nullptr, offsets, mt_start, W, nullptr, nullptr, nullptr, S32,
                       counters, st, &status);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward down (tcgen05)");
    // Y = C Ys: slot outputs transposed so that K = slots is contiguous
    soft_transpose_kernel<float, false><<<dim3((unsigned)((S + kTT - 1) / kTT), (unsigned)((d + kTT - 1) / kTT)),
                                          256, 0, st>>>(S32, S, d, nullptr, nullptr, Yst);
    if ((e = cudaGetLastError()) != cudaSuccess) return soft_fail(e, "moe_soft_forward transpose");
    e = launch_tc_dense(N, d, S, Cw, Yst, Y, counters, st, &status);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_forward combine (tcgen05)");
    return MOE_OK;
}

moe_status moe_soft_check(const moe_soft_params* p, const void* ws, moe_stream_t stream) {
    moe_status s = soft_check(p);
    if (s != MOE_OK) return s;
    if (!ws) return MOE_ERR_WORKSPACE;
    const SoftLayout L = soft_layout(*p);
    unsigned long long cnt[CNT_COUNT];
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(cnt, static_cast<const char*>(ws) + L.counters, sizeof(cnt),
                                    cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return soft_fail(e, "moe_soft_check");
    if (cnt[CNT_DEVICE_ERROR] & DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    return MOE_OK;
}

}  // extern "C"
