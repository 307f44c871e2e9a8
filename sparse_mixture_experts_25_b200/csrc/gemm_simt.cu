// Grouped expert GEMMs in fp32 on the CUDA cores (no TF32), for fp32 layers.
//
// Same functions as the tensor-core path (vegetog "MoE token routing" sec. 3
// SwiGLU expert; "LLM from scratch" ch. 36.3 combine and ch. 36.6 shared
// expert), computed with fp32 FFMA so that fp32 layers keep fp32 accuracy:
//   gate/up  h[r, :] = SiLU(x_r W_g^T) (.) (x_r W_u^T)
//   down     Y[tok(r), :] += a(r) * (h[r, :] W_d^T)   (or H[r, :] = ...)
//
// Design: 64 x 64 output tiles, 256 threads with a 4 x 4 register tile each
// (gate/up keeps a gate and an up tile), K staged through shared memory in
// chunks of 16, tiles scheduled grid-stride over the same group-ordered list
// as the tensor-core kernels (M-tile prefix from the dispatch with BM = 64).
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256, PAD = 4;

enum Epi { EPI_SWIGLU = 0, EPI_COMBINE = 1, EPI_STORE = 2 };

struct SimtArgs {
    const float* A;        // routed A [rows, K]
    const float* A_sh;     // shared A [N, K_sh]
    const float* B0;       // routed: gate (or down) weights, [E * b_rows, K]
    const float* B1;       // routed: up weights (SWIGLU)
    const float* B0_sh;
    const float* B1_sh;
    const int32_t* mt_start;
    const int32_t* offsets;
    int E, K, K_sh, b_rows;
    int n_out, n_out_sh;   // output columns (d_f / d_f_sh for SWIGLU; d for down)
    int M_sh;
    float* out;            // SWIGLU: h; STORE: H
    float* out_sh;         // SWIGLU: h_shared
    const int32_t* slot_token;
    const float* slot_w;
    float* Y;
    int ldY;
    int max_rows;          // rows of the routed A / output buffers (N k)
    int n_tokens;
};

template <int EPI>
__global__ void __launch_bounds__(THREADS) simt_grouped_kernel(const SimtArgs a) {
    constexpr bool TWO = EPI == EPI_SWIGLU;
    __shared__ float As[BK][BM + PAD];
    __shared__ float Bs0[BK][BN + PAD];
    __shared__ float Bs1[TWO ? BK : 1][BN + PAD];
    __shared__ int mt[kMaxExperts + 1];
    __shared__ int off[kMaxExperts + 1];
    for (int i = threadIdx.x; i <= a.E; i += THREADS) {
        mt[i] = a.mt_start[i];
        off[i] = a.offsets[i];
    }
    __syncthreads();
    const int nt_r = (a.n_out + BN - 1) / BN;
    const int routed_tiles = mt[a.E] * nt_r;
    const int nt_sh = a.M_sh > 0 ? (a.n_out_sh + BN - 1) / BN : 0;
    const int mt_sh = (a.M_sh + BM - 1) / BM;
    const int total = routed_tiles + mt_sh * nt_sh;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;

    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        int g = 0, n_tile, a_row, rows, K, b_row0, n_out;
        const float *A, *B0, *B1;
        bool shared;
        if (t < routed_tiles) {
            const int q = t / nt_r;
            int lo = 0, hi = a.E - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (mt[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            g = lo;
            const int mtiles = mt[g + 1] - mt[g];
            if (mtiles > 0) {
                const int local = t - mt[g] * nt_r;
                n_tile = local / mtiles;
                a_row = off[g] + (local % mtiles) * BM;
                rows = max(0, min(min(BM, off[g + 1] - a_row), a.max_rows - a_row));
                if (a_row < 0) rows = 0;
            } else {  // inconsistent prefix (caller-supplied offsets): no rows
                n_tile = 0;
                a_row = 0;
                rows = 0;
            }
            K = a.K;
            A = a.A;
            B0 = a.B0 + (int64_t)g * a.b_rows * a.K;
            B1 = TWO ? a.B1 + (int64_t)g * a.b_rows * a.K : nullptr;
            n_out = a.n_out;
            shared = false;
        } else {
            const int local = t - routed_tiles;
            n_tile = local / mt_sh;
            a_row = (local % mt_sh) * BM;
            rows = min(BM, a.M_sh - a_row);
            K = a.K_sh;
            A = a.A_sh;
            B0 = a.B0_sh;
            B1 = a.B1_sh;
            n_out = a.n_out_sh;
            shared = true;
        }
        b_row0 = n_tile * BN;
        float acc0[4][4] = {}, acc1[4][4] = {};
        for (int k0 = 0; k0 < K; k0 += BK) {
            {   // A: 64 rows x 16 k as float4 along k
                const int r = threadIdx.x / 4, kc = (threadIdx.x % 4) * 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (r < rows && k0 + kc < K)
                    v = *reinterpret_cast<const float4*>(A + (int64_t)(a_row + r) * K + k0 + kc);
                As[kc + 0][r] = v.x;
                As[kc + 1][r] = v.y;
                As[kc + 2][r] = v.z;
                As[kc + 3][r] = v.w;
            }
            {
                const int n = threadIdx.x / 4, kc = (threadIdx.x % 4) * 4;
                float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
                if (b_row0 + n < n_out && k0 + kc < K) {
                    v0 = *reinterpret_cast<const float4*>(B0 + (int64_t)(b_row0 + n) * K + k0 + kc);
                    if (TWO) v1 = *reinterpret_cast<const float4*>(B1 + (int64_t)(b_row0 + n) * K + k0 + kc);
                }
                Bs0[kc + 0][n] = v0.x;
                Bs0[kc + 1][n] = v0.y;
                Bs0[kc + 2][n] = v0.z;
                Bs0[kc + 3][n] = v0.w;
                if (TWO) {
                    Bs1[kc + 0][n] = v1.x;
                    Bs1[kc + 1][n] = v1.y;
                    Bs1[kc + 2][n] = v1.z;
                    Bs1[kc + 3][n] = v1.w;
                }
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < BK; ++kk) {
                const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
                const float4 b0 = *reinterpret_cast<const float4*>(&Bs0[kk][tx * 4]);
                const float ar[4] = {av.x, av.y, av.z, av.w};
                const float br0[4] = {b0.x, b0.y, b0.z, b0.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc0[i][j] = fmaf(ar[i], br0[j], acc0[i][j]);
                if (TWO) {
                    const float4 b1 = *reinterpret_cast<const float4*>(&Bs1[kk][tx * 4]);
                    const float br1[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc1[i][j] = fmaf(ar[i], br1[j], acc1[i][j]);
                }
            }
            __syncthreads();
        }
        const int c0 = b_row0 + tx * 4;
        if (c0 >= n_out) continue;  // n_out % 4 == 0: a 4-column group is all in or all out
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (r >= rows) continue;
            const int grow = a_row + r;
            if (EPI == EPI_SWIGLU) {
                float4 h;
                h.x = acc0[i][0] / (1.f + expf(-acc0[i][0])) * acc1[i][0];
                h.y = acc0[i][1] / (1.f + expf(-acc0[i][1])) * acc1[i][1];
                h.z = acc0[i][2] / (1.f + expf(-acc0[i][2])) * acc1[i][2];
                h.w = acc0[i][3] / (1.f + expf(-acc0[i][3])) * acc1[i][3];
                float* o = shared ? a.out_sh : a.out;
                *reinterpret_cast<float4*>(o + (int64_t)grow * n_out + c0) = h;
            } else if (EPI == EPI_COMBINE) {
                int tok;
                float wgt;
                if (shared) {
                    tok = grow;
                    wgt = 1.f;
                } else {
                    tok = a.slot_token[grow];
                    wgt = a.slot_w[grow];
                }
                if (tok < 0 || tok >= a.n_tokens) continue;
                red_add_v4(a.Y + (int64_t)tok * a.ldY + c0, wgt * acc0[i][0], wgt * acc0[i][1],
                           wgt * acc0[i][2], wgt * acc0[i][3]);
            } else {
                *reinterpret_cast<float4*>(a.out + (int64_t)grow * n_out + c0) =
                    make_float4(acc0[i][0], acc0[i][1], acc0[i][2], acc0[i][3]);
            }
        }
    }
}

template <int EPI>
cudaError_t launch(const SimtArgs& a, int64_t max_tiles, cudaStream_t st) {
    const int grid = (int)min64(max_tiles, (int64_t)num_sms() * 4);
    if (grid <= 0) return cudaSuccess;
    simt_grouped_kernel<EPI><<<grid, THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

int64_t routed_mtile_bound(const moe_params& p) { return (p.N * p.k + BM - 1) / BM + p.E_r; }

}  // namespace

cudaError_t launch_simt_gate_up(const moe_params& p, const void* x_perm, const void* x_shared,
                                const int32_t* offsets, const int32_t* mt_start,
                                const ExpertWeights& W, void* h, void* h_shared,
                                cudaStream_t st) {
    SimtArgs a{};
    a.A = static_cast<const float*>(x_perm);
    a.A_sh = static_cast<const float*>(x_shared);
    a.B0 = static_cast<const float*>(W.W_g);
    a.B1 = static_cast<const float*>(W.W_u);
    a.B0_sh = static_cast<const float*>(W.Ws_g);
    a.B1_sh = static_cast<const float*>(W.Ws_u);
    a.mt_start = mt_start;
    a.offsets = offsets;
    a.E = p.E_r;
    a.K = p.d;
    a.K_sh = p.d;
    a.b_rows = p.d_f;
    a.n_out = p.d_f;
    a.n_out_sh = p.d_f_shared;
    a.M_sh = p.d_f_shared > 0 ? (int)p.N : 0;
    a.out = static_cast<float*>(h);
    a.out_sh = static_cast<float*>(h_shared);
    a.max_rows = (int)(p.N * p.k);
    a.n_tokens = (int)p.N;
    const int64_t nt = (p.d_f + BN - 1) / BN;
    const int64_t tiles = routed_mtile_bound(p) * nt +
                          (a.M_sh ? ((p.N + BM - 1) / BM) * ((p.d_f_shared + BN - 1) / BN) : 0);
    return launch<EPI_SWIGLU>(a, tiles, st);
}

cudaError_t launch_simt_down(const moe_params& p, int mode, const void* h, const void* h_shared,
                             const int32_t* offsets, const int32_t* mt_start,
                             const ExpertWeights& W, const int32_t* slot_token,
                             const float* slot_w, float* Y, float* H_out, cudaStream_t st) {
    SimtArgs a{};
    const bool sh = p.d_f_shared > 0 && mode == DOWN_COMBINE;
    a.A = static_cast<const float*>(h);
    a.A_sh = static_cast<const float*>(h_shared);
    a.B0 = static_cast<const float*>(W.W_d);
    a.B0_sh = static_cast<const float*>(W.Ws_d);
    a.mt_start = mt_start;
    a.offsets = offsets;
    a.E = p.E_r;
    a.K = p.d_f;
    a.K_sh = p.d_f_shared;
    a.b_rows = p.d;
    a.n_out = p.d;
    a.n_out_sh = p.d;
    a.M_sh = sh ? (int)p.N : 0;
    a.out = H_out;
    a.slot_token = slot_token;
    a.slot_w = slot_w;
    a.Y = Y;
    a.ldY = p.d;
    a.max_rows = (int)(p.N * p.k);
    a.n_tokens = (int)p.N;
    const int64_t nt = (p.d + BN - 1) / BN;
    const int64_t tiles = routed_mtile_bound(p) * nt + (sh ? ((p.N + BM - 1) / BM) * nt : 0);
    if (mode == DOWN_COMBINE) return launch<EPI_COMBINE>(a, tiles, st);
    return launch<EPI_STORE>(a, tiles, st);
}

}  // namespace moe
