// Internal declarations shared by the CUDA sources of libmoe (not installed).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------------------
// Limits and workspace constants
// ---------------------------------------------------------------------------
constexpr int kMaxExperts = 1024;     // E_r limit of dispatch and the GEMM schedule
constexpr int kMaxRouterExperts = 256;  // E_r limit of the fused router kernel
constexpr int kMaxK = 32;             // k limit (warp-wide selection)
constexpr int kTcBM = 128;            // M tile of the tcgen05 grouped GEMM
constexpr int kSimtBM = 64;           // M tile of the fp32 grouped GEMM

// indices into the int64 device counter block (moe_ws_layout.counters)
enum Counter {
    CNT_REQUESTED = 0,
    CNT_ACCEPTED = 1,
    CNT_REJECTED = 2,
    CNT_O = 3,
    CNT_AFFECTED = 4,
    CNT_SKIPPED = 5,
    CNT_NONFINITE = 6,
    CNT_NEAR_TIE = 7,
    CNT_L_MAX = 8,
    CNT_C = 9,
    CNT_DEVICE_ERROR = 10,  // bit flags, see DevErr
    CNT_N_GROUP = 11,       // tokens of the whole routing group (sharded runs; 0 = N)
    CNT_REROUTED = 12,      // rejected paths served by a rerouted expert
    CNT_SCAN_TICKET = 13,   // dispatch scans: blocks finished (reset by hist_kernel and the last block)
    CNT_SCAN_ANY = 14,      // rerouting scan: experts that received offers this round
    CNT_COUNT = 16
};

enum DevErr { DEVERR_TIMEOUT = 1, DEVERR_BOUNDS = 2 };

constexpr float kNearTie = 1e-5f;

// Scratch region of the workspace (int32 unless noted)
struct Scratch {
    int32_t* hist;        // [E][n_tiles] per-tile request counts -> exclusive bases
    int32_t* mt_start;    // [E+1] prefix of M tiles (BM of the GEMM in use)
    float* logits;        // [N][E] router scores (tensor-core score path)
    int32_t* base;        // [E] requests of earlier ranks (sharded routing group)
    int32_t* all_offsets; // [E+1] start of each expert's requests (acceptance by weight)
    uint32_t* sel_key;    // [E] order key of the C-th largest weight of an over-full expert
    int32_t* sel_take;    // [E] requests with exactly that key to accept
    int32_t* seg_req;     // [N k] requests grouped by expert, token order (acceptance by weight)
    float* seg_w;         // [N k] their routing weights
    float* psum;          // [E] sum over tokens of the full-softmax probabilities
    // rerouting (MOE_REJECT_REROUTE): candidates and results (workspace
    // records), then the rounds' state
    const int32_t* cand;  // [N, X] candidate experts (rank k + q), -1 none
    const float* cand_w;  // [N, X] their weights
    int32_t* rr_e;        // [N k] expert a rejected path was rerouted to, -1
    int32_t* rr_slot;     // [N k] its slot
    int32_t* rr_q;        // [N k] candidate index used
    int32_t* rr_offer;    // [N k] candidate index offered in the current round, -1
    int32_t* rr_next;     // [N] next unused candidate of each token
    int32_t* rr_stop;     // [1] set once a round made no offer
    // expert parallelism: position of this rank's first row of each expert in
    // its owner's buffer, and (receiving side) source-major row starts [R][El]
    int32_t* ep_dest;     // [E]
    int32_t* ep_recv_base;  // [E]
    int n_tiles;          // dispatch tiles
    int tile_tokens;      // tokens per dispatch tile
};

struct WsView {
    moe_ws_layout lay;
    char* base;
    int32_t* ids;
    float* w;
    float* margin;
    int32_t* slot;
    int32_t* offsets;
    int32_t* L;
    int32_t* acc;
    int32_t* slot_token;
    float* slot_w;
    unsigned long long* counters;
    void* x_perm;
    void* h;
    void* h_shared;
    int32_t* cand;
    float* cand_w;
    int32_t* rr_e;
    int32_t* rr_slot;
    Scratch scratch;
};

// Host helpers (moe_api.cu)
void record_error(const char* msg);  // text returned by moe_last_error on this thread
int dispatch_tile_tokens(int k);
size_t esize(int dtype);
bool make_view(const moe_params& p, void* ws, WsView& v);

// ---------------------------------------------------------------------------
// Launchers (each returns cudaGetLastError() of its launch)
// ---------------------------------------------------------------------------
// router.cu
// logits: [N, E_r] fp32 scratch for the tensor-core score path (may be null)
// psum: [E_r] fp32 sums of the full-softmax probabilities, accumulated (may be null)
// cand / cand_w (MOE_REJECT_REROUTE, nullable): [N, reroute_depth] rerouting candidates
cudaError_t launch_router(const moe_params& p, const void* x, const void* W_r, const float* b_r,
                          const float* lat, int32_t* ids, float* w, float* margin,
                          unsigned long long* counters, float* Y_zero, float* logits, float* psum,
                          cudaStream_t st, int32_t* cand = nullptr, float* cand_w = nullptr);
// dispatch.cu
cudaError_t launch_dispatch(const moe_params& p, int64_t C, int bm, const int32_t* ids,
                            const float* w, int32_t* slot, int32_t* offsets, int32_t* L,
                            int32_t* acc, int32_t* slot_token, float* slot_w, const void* x,
                            void* x_perm, unsigned long long* counters, const Scratch& sc,
                            cudaStream_t st, const char** where);
// sharded routing group: per-rank request counts, then dispatch against the
// gathered counts of all ranks
cudaError_t launch_count(const moe_params& p, const int32_t* ids, int32_t* L, int32_t* counts_out,
                         unsigned long long* counters, const Scratch& sc, cudaStream_t st);
cudaError_t launch_dispatch_ranked(const moe_params& p, int64_t C, int bm, const int32_t* table,
                                   int rank, int n_ranks, int64_t n_group, const int32_t* ids,
                                   const float* w, int32_t* slot, int32_t* offsets, int32_t* L,
                                   int32_t* acc, int32_t* slot_token, float* slot_w,
                                   const void* x, void* x_perm, unsigned long long* counters,
                                   const Scratch& sc, cudaStream_t st, const char** where);
cudaError_t launch_combine(const moe_params& p, const float* H, const int32_t* offsets,
                           const int32_t* slot_token, const float* slot_w, float* Y,
                           cudaStream_t st);
cudaError_t launch_mtile_prefix(int E, int bm, const int32_t* offsets, int32_t* mt_start,
                                cudaStream_t st);
cudaError_t launch_zero_f32(float* Y, int64_t n, cudaStream_t st);

// gemm_tc.cu (bf16, tcgen05)
struct ExpertWeights {
    const void* W_g;
    const void* W_u;
    const void* W_d;
    const void* Ws_g;
    const void* Ws_u;
    const void* Ws_d;
};
enum DownMode { DOWN_COMBINE = 0, DOWN_STORE = 1 };
// Y_zero (nullable): fp32 [N, d] that the kernel zeroes before the down projection adds into it
cudaError_t launch_tc_gate_up(const moe_params& p, const void* x_perm, const void* x_shared,
                              const int32_t* offsets, const int32_t* mt_start,
                              const ExpertWeights& W, void* h, void* h_shared, float* Y_zero,
                              unsigned long long* counters, cudaStream_t st, int* status);
// grp_nkb (DOWN_STORE only, nullable): [E] K blocks of 64 that each group
// contracts over (at least 1); the rest of K is skipped for that group
cudaError_t launch_tc_down(const moe_params& p, int mode, int64_t C, const void* h,
                           const void* h_shared, const int32_t* offsets, const int32_t* mt_start,
                           const ExpertWeights& W, const int32_t* slot_token,
                           const float* slot_w, float* Y, float* H_out,
                           unsigned long long* counters, cudaStream_t st, int* status,
                           const int32_t* grp_nkb = nullptr);
// out[r, :] = A0[r, :K] B0[e] (+ A1[r, :K] B1[e]) for the rows r of each group e
// (offsets), with B0, B1 [E_r][K][n_out] read as stored (MN-major operands:
// no transposed copies); A rows K-major with leading dimensions ldA0 / ldA1;
// fp32 out [N k, n_out].  Single-CTA 128-row tiles: mt_start128 is the
// 128-row tile prefix of offsets.  split_k: when the output tiles fill less
// than one wave, the K blocks are split across CTAs and added into `out`
// with red.add, so the caller zeroes it first (the function returns the
// split it chose in *ks_out when that is not null; pass split_k = false to
// keep one CTA per tile).
cudaError_t launch_tc_store_bmn(const moe_params& p, int64_t n_out, int64_t K, const void* A0, int64_t ldA0,
                                const void* B0, const void* A1, int64_t ldA1, const void* B1,
                                const int32_t* offsets, const int32_t* mt_start128, float* out,
                                unsigned long long* counters, cudaStream_t st, int* status,
                                bool split_k = false, int* ks_out = nullptr);
// K blocks split that launch_tc_store_bmn uses for these sizes with split_k
int tc_store_bmn_split(const moe_params& p, int64_t n_out, int64_t K, bool two_segments);
// rows of one output tile of the tcgen05 grouped GEMMs for these params
// (256 when CTA pairs are used, else 128): the dispatch's M-tile prefix unit
int tc_tile_rows(const moe_params& p);
// CTA-pair layers run each expert's tail of at most 128 rows past its last
// 256-row boundary as one weight-stationary tile (tokens rounded up to 32)
bool tc_swap_tails(const moe_params& p);
// out[M, Nc] (fp32, row-major) = A[M, K] B[Nc, K]^T, bf16 operands with rows
// of K elements (K % 8 == 0, 16-byte aligned bases), tcgen05 tiles of 128 x 256
cudaError_t launch_tc_dense(int64_t M, int64_t Nc, int64_t K, const void* A, const void* B, float* out,
                            unsigned long long* counters, cudaStream_t st, int* status);
cudaError_t launch_gather_rows(const void* src, const int32_t* index, int64_t n_rows, int64_t row_bytes, void* dst,
                               cudaStream_t st);
// expert_parallel.cu: plan of an expert-parallel step from the exchanged
// request counts, and the exchange fused into the dispatch and the combine
constexpr int kMaxEpRanks = 64;
cudaError_t launch_ep_plan(const moe_params& p, const int32_t* counts_all, int R, int rank, int64_t C,
                           int32_t* dest_base, int32_t* local_offsets, int32_t* send_rows, int32_t* recv_rows,
                           int32_t* recv_base, int32_t* regroup, int32_t* regroup_inv, cudaStream_t st);
cudaError_t launch_ep_dispatch(const moe_params& p, int R, const void* x, const int32_t* offsets,
                               const int32_t* slot_token, const int32_t* dest_base, void* const* recv_bufs,
                               cudaStream_t st);
cudaError_t launch_ep_combine(const moe_params& p, int R, const int32_t* offsets, const int32_t* slot_token,
                              const float* slot_w, const int32_t* dest_base, const float* const* out_bufs, float* Y,
                              cudaStream_t st);
cudaError_t launch_wait_selftest(unsigned long long* counters, unsigned long long limit_ns, cudaStream_t st);
// router scores G = x W_r^T (bf16 in, fp32 out [N, E_r]) on the tensor cores
cudaError_t launch_tc_logits(const moe_params& p, const void* x, const void* W_r, float* logits,
                             unsigned long long* counters, cudaStream_t st, int* status);

// gemm_simt.cu (fp32 CUDA-core path)
cudaError_t launch_simt_gate_up(const moe_params& p, const void* x_perm, const void* x_shared,
                                const int32_t* offsets, const int32_t* mt_start,
                                const ExpertWeights& W, void* h, void* h_shared,
                                cudaStream_t st);
cudaError_t launch_simt_down(const moe_params& p, int mode, const void* h, const void* h_shared,
                             const int32_t* offsets, const int32_t* mt_start,
                             const ExpertWeights& W, const int32_t* slot_token,
                             const float* slot_w, float* Y, float* H_out, cudaStream_t st);

int num_sms();

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

}  // namespace moe
