// Router scores, softmax, top-k and routing weights, fused in one kernel.
//
// What it computes ("LLM from scratch" ch. 36.1-36.2, Algorithm 36.1 steps
// 1-2; vegetog "MoE token routing" sec. 2; WDMoE note on WLR pruning):
//   g_te = sum_i x_ti W_r[e,i] + b_e            (fp32 accumulation)
//   p_te = exp(g_te - max_e g_te) / sum_e exp(...)
//   S_t  = k largest scores, ties to the lower expert index
//   a_te = p_te / sum_{S_t} p (renorm) | p_te (full prob) | WLR pruning
//
// Design: one CTA of 256 threads owns 32 tokens.  The score tile
// [32 tokens x E_r] is a small FFMA GEMM staged through shared memory in
// 64-wide K chunks, with a (TT tokens x TE experts) register tile per thread
// chosen from E_r.  The selection then runs warp-wide: each lane holds
// ceil(E_r/32) scores and k rounds of a (value desc, index asc) warp argmax
// pick the experts in rank order.  For the narrow routers of the pages'
// layers (E_r = 8 on a d = 4096 model) the kernel is bound by reading x
// once; for E_r = 128-256 it is FFMA-bound.
#include "moe_internal.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int kTok = 32;
constexpr int kThreads = 256;
constexpr int kKC = 64;

struct RouterArgs {
    const void* x;
    const void* W_r;
    const float* b_r;
    const float* lat;
    int32_t* ids;
    float* w;
    float* margin;
    unsigned long long* counters;
    float* Y_zero;
    float* psum;  // [E] sum over tokens of the full-softmax probabilities (nullable)
    int32_t* cand;  // [N, X] rerouting candidates: experts of rank k .. k+X-1 (X > 0 only)
    float* cand_w;  // [N, X] their weights under the layer's normalisation
    int64_t N;
    int d, E, k, norm;
    int X;          // rerouting candidates per token (0: none)
    float theta;
};

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Softmax, top-k in rank order (score descending, ties to the lower expert
// index), weights and records for one token.  The calling warp holds the
// token's scores (bias included) as v[i] = g[lane + 32 i], -inf past E_r.
// ps (shared memory, nullable) accumulates the token's full-softmax
// probabilities per expert, for the mean router probability of the batch.
template <int PER>
__device__ __forceinline__ void select_token(const RouterArgs& a, int64_t t, int lane, float (&v)[PER],
                                             float* ps) {
    const int E = a.E, k = a.k;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !isfinite(v[i])) bad = true;
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < PER; ++i) m = fmaxf(m, v[i]);
    m = warp_max(m);
    unsigned taken = 0;
    int my_e = -1;
    float my_g = 0.f, next_g = -INFINITY;
    // ranks 0..k-1 are the chosen experts; rank k gives the margin; ranks
    // k..k+X-1 are the rerouting candidates (lane r holds rank r)
    const int want = k + (a.X > 1 ? a.X : 1);
    const int rounds = want < E ? want : E;
    if (!__any_sync(0xffffffffu, bad)) {
        for (int r = 0; r < rounds; ++r) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = lane + 32 * i;
                if (!((taken >> i) & 1u) && e < E && (v[i] > bv || (v[i] == bv && e < be))) {
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (lane == r) {
                my_e = be;
                my_g = bv;
            }
            if (r == k) next_g = bv;
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
        }
    }
    float z = 0.f;
    float ev[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        ev[i] = e < E ? expf(v[i] - m) : 0.f;
        z += ev[i];
    }
    z = warp_sum(z);
    const bool pick = lane < k;
    const float ex = pick && !bad ? expf(my_g - m) : 0.f;
    float wv = 0.f;
    bool active = pick;
    bool lat_bad = false;
    float te = 1.f;
    if (a.norm == MOE_NORM_WLR && pick && !bad) {
        te = a.lat[t * E + my_e];
        lat_bad = !(te > 0.f);  // NaN or non-positive latency
    }
    bad = __any_sync(0xffffffffu, bad || lat_bad);
    const bool is_cand = lane >= k && lane < k + a.X;
    if (bad) {
        if (pick) {
            a.ids[t * k + lane] = -1;
            a.w[t * k + lane] = 0.f;
        }
        if (is_cand) {
            a.cand[t * a.X + (lane - k)] = -1;
            a.cand_w[t * a.X + (lane - k)] = 0.f;
        }
        if (lane == 0) {
            if (a.margin) a.margin[t] = NAN;
            atomicAdd(a.counters + CNT_NONFINITE, 1ull);
        }
        return;
    }
    if (ps) {
        const float iz = 1.f / z;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            if (e < E) atomicAdd(&ps[e], ev[i] * iz);
        }
    }
    float sel_sum = 1.f;  // sum of the chosen experts' exp(g - m) (renormalisation)
    if (a.norm == MOE_NORM_FULLPROB) {
        wv = ex / z;
    } else if (a.norm == MOE_NORM_RENORM) {
        sel_sum = warp_sum(ex);
        wv = ex / sel_sum;
    } else {
        const float wlr = (ex / z) / te;  // p_e / t_e (0 when t_e = inf)
        for (;;) {
            const unsigned am = __ballot_sync(0xffffffffu, active);
            if (__popc(am) < 2) break;
            // smallest WLR (on equal WLR the higher expert index) and largest WLR
            float mn = active ? wlr : INFINITY;
            int mne = active ? my_e : -1;
            float mx = active ? wlr : -INFINITY;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, mn, o);
                const int oe = __shfl_xor_sync(0xffffffffu, mne, o);
                if (ov < mn || (ov == mn && oe > mne)) {
                    mn = ov;
                    mne = oe;
                }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            const float ratio = mn / (mn + mx);
            if (ratio <= a.theta) {
                if (active && my_e == mne) active = false;
            } else {
                break;
            }
        }
        const float s = warp_sum(active ? ex : 0.f);
        wv = active ? ex / s : 0.f;
        if (active && isinf(te)) wv = 0.f;  // disconnected expert: weight 0
    }
    if (pick) {
        a.ids[t * k + lane] = active ? my_e : -1;
        a.w[t * k + lane] = wv;
    }
    if (is_cand) {
        // the expert of rank `lane`, weighted against the chosen set as the
        // chosen experts are (full probability: p; renormalised: p / sum_S p)
        const bool have = lane < E;
        const float exc = have ? expf(my_g - m) : 0.f;
        a.cand[t * a.X + (lane - k)] = have ? my_e : -1;
        a.cand_w[t * a.X + (lane - k)] = have ? (a.norm == MOE_NORM_FULLPROB ? exc / z : exc / sel_sum) : 0.f;
    }
    const float kth = __shfl_sync(0xffffffffu, my_g, k - 1);
    const float mg = k < E ? kth - next_g : INFINITY;
    if (lane == 0) {
        if (a.margin) a.margin[t] = mg;
        if (mg < kNearTie) atomicAdd(a.counters + CNT_NEAR_TIE, 1ull);
    }
}

template <int TT, int TE, typename Tin>
__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a) {
    constexpr int EG = 8 * TT;       // expert groups across the CTA
    constexpr int EPAD = EG * TE;    // padded expert count
    constexpr int PER = (EPAD + 31) / 32;
    static_assert((kTok / TT) * EG == kThreads, "thread grid");
    extern __shared__ float smem[];
    float* xs = smem;                 // [kKC][kTok]
    float* wsm = smem + kKC * kTok;   // [kKC][EPAD]

    __shared__ float ps[kMaxRouterExperts];
    const int tid = threadIdx.x;
    const int tg = tid / EG, eg = tid % EG;
    const int64_t t0 = (int64_t)blockIdx.x * kTok;
    for (int e = tid; e < a.E; e += kThreads) ps[e] = 0.f;
    const Tin* X = static_cast<const Tin*>(a.x);
    const Tin* W = static_cast<const Tin*>(a.W_r);

    float acc[TT][TE];
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < a.d; k0 += kKC) {
        for (int i = tid; i < kTok * (kKC / 8); i += kThreads) {
            const int tt = i / (kKC / 8), kc = (i % (kKC / 8)) * 8;
            const int64_t t = t0 + tt;
            float v[8];
            if (t < a.N && k0 + kc < a.d) {
                load8(X + t * a.d + k0 + kc, v);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) xs[(kc + j) * kTok + tt] = v[j];
        }
        for (int i = tid; i < EPAD * (kKC / 8); i += kThreads) {
            const int e = i / (kKC / 8), kc = (i % (kKC / 8)) * 8;
            float v[8];
            if (e < a.E && k0 + kc < a.d) {
                load8(W + (int64_t)e * a.d + k0 + kc, v);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) wsm[(kc + j) * EPAD + e] = v[j];
        }
        __syncthreads();
        // two-level fp32 summation: a fresh partial per 64-wide chunk, then
        // added to the running score (error ~ (64 + d/64) ulp instead of d ulp)
        float part[TT][TE];
#pragma unroll
        for (int i = 0; i < TT; ++i)
#pragma unroll
            for (int j = 0; j < TE; ++j) part[i][j] = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < kKC; ++kk) {
            float xv[TT], wv[TE];
#pragma unroll
            for (int i = 0; i < TT; ++i) xv[i] = xs[kk * kTok + tg * TT + i];
#pragma unroll
            for (int j = 0; j < TE; ++j) wv[j] = wsm[kk * EPAD + eg + EG * j];
#pragma unroll
            for (int i = 0; i < TT; ++i)
#pragma unroll
                for (int j = 0; j < TE; ++j) part[i][j] = fmaf(xv[i], wv[j], part[i][j]);
        }
#pragma unroll
        for (int i = 0; i < TT; ++i)
#pragma unroll
            for (int j = 0; j < TE; ++j) acc[i][j] += part[i][j];
        __syncthreads();
    }

    // scores -> shared memory
    constexpr int LD = EPAD + 1;
    float* lg = smem;  // [kTok][LD], fits inside the staging buffers
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            const int e = eg + EG * j;
            if (e < a.E) lg[(tg * TT + i) * LD + e] = acc[i][j] + (a.b_r ? a.b_r[e] : 0.f);
        }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    for (int q = 0; q < kTok / 8; ++q) {
        const int tt = warp * (kTok / 8) + q;
        const int64_t t = t0 + tt;
        if (t >= a.N) break;
        const float* g = lg + tt * LD;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < a.E ? g[e] : -INFINITY;
        }
        select_token<PER>(a, t, lane, v, a.psum ? ps : nullptr);
    }
    if (a.psum) {
        __syncthreads();
        for (int e = tid; e < a.E; e += kThreads)
            if (ps[e] != 0.f) atomicAdd(&a.psum[e], ps[e]);
    }

    if (a.Y_zero) {
        const int64_t t_end = min64(a.N, t0 + kTok);
        float4* Y4 = reinterpret_cast<float4*>(a.Y_zero + t0 * a.d);
        const int64_t n4 = (t_end - t0) * a.d / 4;
        for (int64_t i = tid; i < n4; i += kThreads) Y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

__device__ __forceinline__ void zero_row(float* Y, int64_t t, int d, int lane) {
    float4* y4 = reinterpret_cast<float4*>(Y + t * d);
    for (int i = lane; i < d / 4; i += 32) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Eight consecutive inputs kept in their storage format until used (bf16
// stays packed in one 16-byte register quad, halving register pressure).
template <typename Tin>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void ldg(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void ldcs(const __nv_bfloat16* p) { u = __ldcs(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ float get(int j) const {
        const uint32_t w = j < 2 ? u.x : j < 4 ? u.y : j < 6 ? u.z : u.w;
        return (j & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
    }
};
template <>
struct Vec8<float> {
    float4 a, b;
    __device__ __forceinline__ void ldg(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p + 4));
    }
    __device__ __forceinline__ void ldcs(const float* p) {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p + 4));
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float get(int j) const {
        const float4& q = j < 4 ? a : b;
        const int i = j & 3;
        return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w;
    }
};

// Narrow routers (E_r <= EMAX <= 32), one warp per token: the lanes stream the
// token's row of x in 16-byte vectors (each lane a strided slice of d), keep
// E_r partial scores, and a butterfly reduction gives every lane all scores.
// W_r (E_r x d) is read through L1.  All loads of one step (x and eight
// experts' weights, two steps per iteration) are issued before their FMAs so
// that the warp waits for memory once per iteration rather than once per
// expert.  Bound by reading x once.
template <int EMAX, typename Tin>
__device__ __forceinline__ void narrow_token(const RouterArgs& a, int64_t t, int lane, float* ps) {
    const Tin* X = static_cast<const Tin*>(a.x) + t * a.d;
    const Tin* W = static_cast<const Tin*>(a.W_r);
    const int E = a.E;
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    for (int i0 = lane * 8; i0 < a.d; i0 += 512) {
        const int i1 = i0 + 256;
        const bool has1 = i1 < a.d;
        Vec8<Tin> x0, x1;
        x0.ldcs(X + i0);
        if (has1) x1.ldcs(X + i1);
        else x1.zero();
#pragma unroll
        for (int g = 0; g < EMAX; g += 8) {
            Vec8<Tin> w0[8], w1[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int ee = min(g + e, E - 1);  // clamped: loads are unconditional
                const Tin* row = W + (int64_t)ee * a.d;
                w0[e].ldg(row + i0);
                if (has1) w1[e].ldg(row + i1);
                else w1[e].zero();
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float part = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) part = fmaf(x0.get(j), w0[e].get(j), part);
#pragma unroll
                for (int j = 0; j < 8; ++j) part = fmaf(x1.get(j), w1[e].get(j), part);
                acc[g + e] += part;
            }
        }
    }
    float v[1] = {-INFINITY};
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
        float s = acc[e];
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == e && e < E) v[0] = s + (a.b_r ? a.b_r[e] : 0.f);
    }
    select_token<1>(a, t, lane, v, ps);
    if (a.Y_zero) zero_row(a.Y_zero, t, a.d, lane);
}

template <int EMAX, typename Tin>
__global__ void __launch_bounds__(256) router_narrow_kernel(RouterArgs a) {
    __shared__ float ps[EMAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    if (threadIdx.x < EMAX) ps[threadIdx.x] = 0.f;
    __syncthreads();
    if (t < a.N) narrow_token<EMAX, Tin>(a, t, lane, a.psum ? ps : nullptr);
    if (a.psum) {
        __syncthreads();
        if (threadIdx.x < a.E && ps[threadIdx.x] != 0.f) atomicAdd(&a.psum[threadIdx.x], ps[threadIdx.x]);
    }
}

// Selection from precomputed scores [N, E_r] (tensor-core score path), one
// warp per token.
template <int PER>
__global__ void __launch_bounds__(256) logits_topk_kernel(RouterArgs a, const float* __restrict__ logits) {
    __shared__ float ps[32 * PER];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    for (int e = threadIdx.x; e < 32 * PER; e += blockDim.x) ps[e] = 0.f;
    __syncthreads();
    if (t < a.N) {
        const float* g = logits + t * a.E;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < a.E ? g[e] + (a.b_r ? a.b_r[e] : 0.f) : -INFINITY;
        }
        select_token<PER>(a, t, lane, v, a.psum ? ps : nullptr);
        if (a.Y_zero) zero_row(a.Y_zero, t, a.d, lane);
    }
    if (a.psum) {
        __syncthreads();
        for (int e = threadIdx.x; e < a.E; e += blockDim.x)
            if (ps[e] != 0.f) atomicAdd(&a.psum[e], ps[e]);
    }
}

template <int TT, int TE, typename Tin>
cudaError_t launch_one(const RouterArgs& a, cudaStream_t st) {
    constexpr int EPAD = 8 * TT * TE;
    const size_t smem = sizeof(float) * (kKC * kTok + kKC * EPAD);
    auto kern = router_kernel<TT, TE, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (a.N + kTok - 1) / kTok;
    kern<<<(unsigned)blocks, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_typed(const RouterArgs& a, cudaStream_t st) {
    if (a.E <= 8) return launch_one<1, 1, Tin>(a, st);
    if (a.E <= 16) return launch_one<1, 2, Tin>(a, st);
    if (a.E <= 32) return launch_one<2, 2, Tin>(a, st);
    if (a.E <= 64) return launch_one<2, 4, Tin>(a, st);
    if (a.E <= 128) return launch_one<4, 4, Tin>(a, st);
    return launch_one<4, 8, Tin>(a, st);
}

}  // namespace

cudaError_t launch_router(const moe_params& p, const void* x, const void* W_r, const float* b_r,
                          const float* lat, int32_t* ids, float* w, float* margin,
                          unsigned long long* counters, float* Y_zero, float* logits, float* psum,
                          cudaStream_t st, int32_t* cand, float* cand_w) {
    RouterArgs a;
    a.x = x;
    a.W_r = W_r;
    a.b_r = b_r;
    a.lat = lat;
    a.ids = ids;
    a.w = w;
    a.margin = margin;
    a.counters = counters;
    a.Y_zero = Y_zero;
    a.psum = psum;
    a.N = p.N;
    a.d = p.d;
    a.E = p.E_r;
    a.k = p.k;
    a.norm = p.norm;
    a.theta = p.theta;
    a.X = (p.reject_policy == MOE_REJECT_REROUTE && cand && cand_w) ? p.reroute_depth : 0;
    a.cand = cand;
    a.cand_w = cand_w;
    if (p.N == 0) return cudaSuccess;
    const unsigned warps_blocks = (unsigned)((p.N + 7) / 8);
    const bool bf16 = p.dtype == MOE_BF16;
    if (p.E_r <= 32 && !(bf16 && logits && p.E_r % 4 == 0)) {
        if (p.E_r <= 8) {
            if (bf16) router_narrow_kernel<8, __nv_bfloat16><<<warps_blocks, 256, 0, st>>>(a);
            else router_narrow_kernel<8, float><<<warps_blocks, 256, 0, st>>>(a);
        } else if (p.E_r <= 16) {
            if (bf16) router_narrow_kernel<16, __nv_bfloat16><<<warps_blocks, 256, 0, st>>>(a);
            else router_narrow_kernel<16, float><<<warps_blocks, 256, 0, st>>>(a);
        } else {
            if (bf16) router_narrow_kernel<32, __nv_bfloat16><<<warps_blocks, 256, 0, st>>>(a);
            else router_narrow_kernel<32, float><<<warps_blocks, 256, 0, st>>>(a);
        }
        return cudaGetLastError();
    }
    if (bf16 && logits && p.E_r % 4 == 0) {
        // bf16 routers: scores on the tensor cores (K split over SMs for small
        // batches), then one warp per token selects
        int status = 0;
        cudaError_t e = launch_tc_logits(p, x, W_r, logits, counters, st, &status);
        if (e != cudaSuccess) return e;
        if (p.E_r <= 32) logits_topk_kernel<1><<<warps_blocks, 256, 0, st>>>(a, logits);
        else if (p.E_r <= 64) logits_topk_kernel<2><<<warps_blocks, 256, 0, st>>>(a, logits);
        else if (p.E_r <= 128) logits_topk_kernel<4><<<warps_blocks, 256, 0, st>>>(a, logits);
        else logits_topk_kernel<8><<<warps_blocks, 256, 0, st>>>(a, logits);
        return cudaGetLastError();
    }
    if (bf16) return launch_typed<__nv_bfloat16>(a, st);
    return launch_typed<float>(a, st);
}

}  // namespace moe
