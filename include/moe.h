/*
 * moe.h — C ABI of the B200 (sm_100a) sparse Mixture-of-Experts layer
 * forward pass: router, softmax, top-k, weighting, capacity-limited
 * token-order dispatch, SwiGLU experts, optional shared expert, weighted
 * combine.
 *
 * Notation follows the pages' notation table ("LLM from scratch" ch. 36.1):
 * N tokens in the routing group, model width d, expert hidden width d_f,
 * E_r routed experts, k experts per token, capacity factor c (gamma on that
 * page), router W_r and bias b_r, routing weights a_te, requested load n_e
 * (L_e in the auturnal review), capacity C_e, expert outputs H_e, output Y.
 *
 * Conventions for every entry point
 *  - Memory: every pointer argument is DEVICE memory unless marked "host".
 *    The caller allocates and owns all buffers, including the workspace
 *    (size from moe_workspace_size).  The library never allocates device
 *    memory and never frees caller memory.
 *  - Execution: every call enqueues its kernels on `stream` and returns
 *    without waiting, except moe_get_stats, which waits for the stream.
 *    Host-side argument checks return synchronously; a non-MOE_OK status
 *    means nothing was enqueued (except MOE_ERR_CUDA: a launch failed).
 *  - Layout: row-major.  Weights are stored output-major ("K-major"), the
 *    transposes of the pages' x W convention, which ch. 36.8 of
 *    "LLM from scratch" names an allowed transposition:
 *      W_r [E_r, d]; W_g, W_u [E_r, d_f, d]; W_d [E_r, d, d_f];
 *      shared Ws_g, Ws_u [d_f_shared, d]; Ws_d [d, d_f_shared].
 *    Element type of x and all weights: params.dtype (fp32, or bf16 stored
 *    as raw 16-bit patterns).  b_r, lat, routing weights and Y are fp32.
 *  - Alignment: device pointers to x, weights, x_perm, H and the workspace
 *    must be 16-byte aligned (256 recommended); d and d_f must be multiples
 *    of 8, else MOE_ERR_UNSUPPORTED.
 *  - Threads: calls on different streams with different workspaces may run
 *    concurrently; one workspace must not be shared by calls in flight.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  NULL selects the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* a size, mode or pointer violates the contract */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement */
    MOE_ERR_NONFINITE = 3,    /* a router score (or WLR latency) was not finite */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    MOE_ERR_WORKSPACE = 5,    /* workspace missing or too small / misaligned */
    MOE_ERR_TIMEOUT = 6       /* a bounded device wait gave up (kernel fault guard) */
} moe_status;

/* Weighting of the chosen experts ("LLM from scratch" ch. 36.2; WDMoE note). */
typedef enum moe_norm {
    MOE_NORM_RENORM = 0,   /* a_te = p_te / sum_{j in S_t} p_tj  (sums to 1)        */
    MOE_NORM_FULLPROB = 1, /* a_te = p_te, the full-softmax probability (Switch)   */
    MOE_NORM_WLR = 2       /* WDMoE weight-latency-ratio pruning with threshold theta,
                              then softmax over the surviving scores               */
} moe_norm;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* What a path rejected by the capacity limit does to the token's other paths
 * ("LLM from scratch" ch. 36.3-36.4: the overflow policy is part of the
 * function; the worked example prints both outcomes). */
typedef enum moe_reject_policy {
    MOE_REJECT_ZERO = 0,    /* rejected path adds 0, the others keep their weights
                               (Algorithm 36.1)                                     */
    MOE_REJECT_RENORM = 1,  /* the token's accepted paths are rescaled to sum to 1  */
    MOE_REJECT_REROUTE = 2  /* a rejected path is rerouted to the token's next-ranked
                               expert with a free slot (below); a path that finds
                               none adds 0                                          */
} moe_reject_policy;

/* Rerouting (MOE_REJECT_REROUTE; "LLM from scratch" ch. 36.3: a rejected path
 * may be rerouted, which calls another expert's parameters; vegetog "MoE
 * token routing" sec. 5).  The pages leave the target open; this library
 * reads it as follows.  A token's candidates are its experts of ranks k .. k
 * + reroute_depth - 1 in the router's order (score descending, ties to the
 * lower index), each weighted as the router's normalisation weights it
 * against the token's chosen set S (p_e / sum_S p under MOE_NORM_RENORM, p_e
 * under MOE_NORM_FULLPROB).  After Algorithm 36.1's token-order acceptance of
 * the first choices, the rejected paths fill the slots left free in rounds:
 * each path still without an expert takes its token's next unused candidate
 * whose expert was not full at the start of the round (a token's paths in
 * rank order take consecutive candidates), and the round's offers are
 * accepted in token order while the expert has a free slot.  A refused path
 * tries the next candidate in the next round.  An expert's rows are its
 * first-choice rows in token order, then each round's rerouted rows in token
 * order.  Requires MOE_NORM_RENORM or MOE_NORM_FULLPROB and
 * MOE_ACCEPT_TOKEN, a single routing group (not moe_forward_begin/end,
 * moe_dispatch_ranked or moe_dispatch_noalloc: MOE_ERR_UNSUPPORTED), and no
 * backward pass (moe_backward returns MOE_ERR_UNSUPPORTED). */

/* Which requests an over-full expert accepts ("LLM from scratch" ch. 36.3,
 * on how the acceptance rule makes outputs depend on the batch: first come
 * first served in token order, or ordering by gate weight, under which the
 * low-weight paths lose their computation).
 *
 * Expert-choice routing (ch. 36.6 table of routing styles: each expert picks
 * a limited number of tokens by its column of scores; a token may get several
 * experts or none) is this library with k = E_r, MOE_NORM_FULLPROB and
 * MOE_ACCEPT_WEIGHT: every token requests every expert with weight p_te and
 * each expert keeps the C largest, C = ceil(c N) (c = C / N). */
typedef enum moe_accept_order {
    MOE_ACCEPT_TOKEN = 0,  /* the first C requests in token order (Algorithm 36.1) */
    MOE_ACCEPT_WEIGHT = 1  /* the C requests with the largest routing weight a_te,
                              equal weights to the earlier token; accepted rows
                              keep token order in the expert's buffer.  Single
                              routing group only (moe_forward_begin/end and
                              moe_dispatch_noalloc return MOE_ERR_UNSUPPORTED). */
} moe_accept_order;

typedef struct moe_params {
    int64_t N;          /* tokens in the routing group, N >= 0                      */
    int32_t d;          /* model width                                               */
    int32_t d_f;        /* routed expert hidden width                                */
    int32_t E_r;        /* routed experts, 1..1024                                   */
    int32_t k;          /* experts per token, 1 <= k <= min(E_r, 32)                 */
    double c;           /* capacity factor; c <= 0 means no limit (C = N)            */
    int32_t norm;       /* moe_norm                                                  */
    float theta;        /* WLR threshold in [0, 1) (MOE_NORM_WLR only)               */
    int32_t dtype;      /* moe_dtype of x and of every weight                        */
    int32_t d_f_shared; /* hidden width of the always-on shared expert; 0 = none     */
    int32_t reject_policy; /* moe_reject_policy                                      */
    int32_t accept_order;  /* moe_accept_order                                       */
    int32_t reroute_depth; /* MOE_REJECT_REROUTE: candidates per token, 1 ..
                              min(E_r - k, 32 - k); ignored by the other policies   */
    int32_t reserved;      /* 0                                                      */
} moe_params;

/* Routing statistics of the last moe_dispatch / moe_forward on a workspace
 * ("LLM from scratch" ch. 36.4 load statistics and Algorithm 36.1 outputs;
 * auturnal review equations for O and rho_max). */
typedef struct moe_stats {
    int64_t C;               /* capacity used                                     */
    int64_t requested;       /* sum_e L_e (paths that asked for an expert)        */
    int64_t accepted;        /* paths given a slot                                */
    int64_t rejected;        /* requested - accepted                              */
    int64_t O;               /* sum_e max(0, L_e - C)                             */
    int64_t tokens_affected; /* tokens with at least one rejected path            */
    int64_t tokens_skipped;  /* tokens whose every requested path was rejected    */
    int64_t nonfinite;       /* tokens whose scores were not finite (no paths)    */
    int64_t near_tie;        /* tokens whose k-th vs (k+1)-th score margin < 1e-5 */
    int64_t L_max, L_p50, L_p90, L_p99; /* requested load: max, nearest-rank pct  */
    double rho_max;          /* max_e L_e / (N k / E_r)                           */
    double reject_rate;      /* rejected / requested                              */
    int32_t device_error;    /* nonzero: a bounded device wait timed out (bit 0)
                                or a routing id was out of range (bit 1)           */
    int32_t rerouted;        /* MOE_REJECT_REROUTE: rejected paths served by a
                                rerouted expert (included in accepted; rejected and
                                tokens_affected / tokens_skipped then count the
                                paths left without any expert); 0 otherwise       */
    int64_t padded_rows;     /* rows the routed gate/up GEMM computes: each expert's
                                accepted rows rounded up to the GEMM's row tile (on
                                CTA pairs a tail of at most 128 rows past the last
                                256-row boundary rounded up to 32 instead; on single
                                CTAs a last tile of at most 64 rows to 64)         */
    double padding_ratio;    /* padded_rows / accepted (0 when nothing accepted)  */
    double aux_balance;      /* E_r sum_e f_e pbar_e ("LLM from scratch" ch. 36.4
                                balance objective, value only): f_e = L_e / sum L,
                                the requests' shares before capacity; pbar_e = the
                                mean full-softmax probability over the tokens with
                                finite scores (this rank's tokens in a sharded
                                group); 1 when both are uniform                    */
} moe_stats;

/* Byte offsets of the regions inside the workspace (for inspection and
 * tests; every region is 256-byte aligned). */
typedef struct moe_ws_layout {
    size_t ids;        /* int32 [N, k]  chosen expert per rank, -1 = none         */
    size_t w;          /* fp32  [N, k]  weight a_te                                */
    size_t margin;     /* fp32  [N]     score margin g_(k) - g_(k+1)               */
    size_t slot;       /* int32 [N, k]  slot in the expert buffer, -1 = rejected   */
    size_t offsets;    /* int32 [E_r+1] start row of each expert's accepted rows   */
    size_t L;          /* int32 [E_r]   requested load per expert                  */
    size_t acc;        /* int32 [E_r]   accepted rows per expert                   */
    size_t slot_token; /* int32 [N k]   token of each accepted row                 */
    size_t slot_w;     /* fp32  [N k]   weight of each accepted row                */
    size_t counters;   /* int64 [16]    device counters                            */
    size_t x_perm;     /* dtype [N k, d] gathered expert inputs                    */
    size_t h;          /* dtype [N k, d_f] expert hidden activations               */
    size_t h_shared;   /* dtype [N, d_f_shared]                                    */
    size_t cand;       /* int32 [N, reroute_depth] rerouting candidates (rank k + q),
                          -1 past E_r or for an invalid token (MOE_REJECT_REROUTE)  */
    size_t cand_w;     /* fp32  [N, reroute_depth] their weights                    */
    size_t rr_e;       /* int32 [N, k] expert a rejected path was rerouted to, -1   */
    size_t rr_slot;    /* int32 [N, k] its slot in that expert's buffer, -1        */
    size_t scratch;    /* internal                                                 */
    size_t total;      /* bytes required                                           */
} moe_ws_layout;

/* Capacity C = ceil(c N k / E_r) (auturnal review, C_e equation; "LLM from
 * scratch" ch. 36.3 capacity rule; vegetog sec. 6 example), on the exact
 * value of c, taking an integer within 1e-9 (relative) of c N k / E_r as
 * exact.  c <= 0 gives C = N.  *C is host memory. */
MOE_API moe_status moe_capacity(const moe_params* p, int64_t* C);

/* Bytes of device workspace that moe_route/moe_dispatch/moe_expert_ffn/
 * moe_forward need for these params (host call, no device work). */
MOE_API moe_status moe_workspace_size(const moe_params* p, size_t* bytes);

/* Region offsets inside the workspace (host call). */
MOE_API moe_status moe_workspace_layout(const moe_params* p, moe_ws_layout* out);

/*
 * Router scores G = x W_r^T + b_r, softmax over experts, top-k with ties to
 * the lower expert index, and weights by params.norm ("LLM from scratch"
 * ch. 36.1-36.2 and Algorithm 36.1 steps 1-2; vegetog sec. 2; WDMoE note).
 *   x   [N, d] dtype;  W_r [E_r, d] dtype;  b_r [E_r] fp32 or NULL
 *   lat [N, E_r] fp32 per-token per-expert latency t = t_up + t_comp + t_down,
 *       required for MOE_NORM_WLR, ignored otherwise
 * Outputs (rank order j = 0..k-1, score descending):
 *   ids [N, k] int32 expert, -1 for a path pruned by WLR or an invalid token
 *   w   [N, k] fp32 weight a_te (0 where ids = -1)
 *   margin [N] fp32 g_(k) - g_(k+1) (+inf if k = E_r; NaN if invalid), nullable
 * Scores are accumulated in fp32.  A token with a non-finite score (or,
 * under WLR, a chosen expert whose latency is not a positive number) gets no
 * paths and is counted in the workspace counters (MOE_ERR_NONFINITE from
 * moe_get_stats).  ws: workspace of moe_workspace_size bytes.  Under
 * MOE_REJECT_REROUTE the call also writes each token's rerouting candidates
 * and their weights into ws (moe_ws_layout.cand, cand_w), which
 * moe_dispatch on the same workspace reads.
 */
MOE_API moe_status moe_route(const moe_params* p, const void* x, const void* W_r, const float* b_r,
                     const float* lat, int32_t* ids, float* w, float* margin, void* ws,
                     moe_stream_t stream);

/*
 * Capacity check and dispatch (Algorithm 36.1 steps 3-4; ch. 36.3 dispatch
 * matrix D_e as index lists and prefix sums).  Requests are taken in token
 * order t = 0..N-1: path (t, e) gets slot c = number of earlier requests for
 * e, and is accepted iff c < C.  Deterministic (a stable counting sort).
 *   ids, w     [N, k] from moe_route (ids -1 = no request)
 *   C          capacity, >= 1 (see moe_capacity)
 *   slot       [N, k] int32 out: slot, or -1 if rejected / not requested
 *   offsets    [E_r + 1] int32 out: accepted rows of expert e are rows
 *              offsets[e] .. offsets[e+1]-1 of the expert buffers, in slot order
 *   slot_token [N k] int32 out: source token of each accepted row
 *   slot_w     [N k] fp32 out: combine weight of each accepted row: a_te, or
 *              under MOE_REJECT_RENORM a_te / (sum of the token's accepted a)
 *              for tokens that lost a path
 *   x          [N, d] dtype, nullable; with x_perm [N k, d] dtype, gathers
 *              x_perm[r] = x[slot_token[r]] for every accepted row r
 * Statistics (L_e, accepted, O, ...) go to the workspace counters.
 * MOE_REJECT_REROUTE: the rejected paths are then rerouted (see
 * moe_reject_policy) to the candidates moe_route wrote into ws; slot keeps the
 * first-choice slots (-1 for a rejected path), the rerouted paths' experts and
 * slots go to ws (moe_ws_layout.rr_e, rr_slot), and the rows, offsets,
 * slot_token and slot_w cover both (a rerouted row's weight is its
 * candidate's weight).  The rounds are launched reroute_depth times.
 */
MOE_API moe_status moe_dispatch(const moe_params* p, const int32_t* ids, const float* w, int64_t C,
                        int32_t* slot, int32_t* offsets, int32_t* slot_token, float* slot_w,
                        const void* x, void* x_perm, void* ws, moe_stream_t stream);

/*
 * moe_dispatch without a workspace, for callers that cannot allocate device
 * memory where they dispatch: code running under a memory pool that may not
 * grow, embedders whose allocator is not reachable from the call site, and
 * call sites that must not call cudaMalloc because it can synchronise the
 * device.  The pages have no counterpart of this entry point; it computes
 * exactly what moe_dispatch computes (same arguments, minus ws) and fills
 * the same outputs.
 *
 * Its scratch (per-tile request counts, per-expert loads, M-tile prefix,
 * counters) lives in a 1 MiB array inside the library, which every GPU that
 * loads the library holds until the process exits.  Limit:
 * E_r * n_tiles + 3 E_r + 33 four-byte words must fit in 1 MiB, with
 * n_tiles = ceil(N / max(8, floor(128 / k))) (for example N = 8192, k = 8,
 * E_r = 128 needs 258 KB); larger sizes return MOE_ERR_UNSUPPORTED with the
 * required size in moe_last_error.  The routing statistics of this call
 * stay inside the array and are not readable through moe_get_stats.
 *
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * With lazy module loading (the CUDA 12 default) that first lookup may be
 * what loads the library onto the device: a one-time reservation of the
 * 1 MiB array that can synchronise the device.  Make the first call early
 * (for example at start-up, with N = 0), outside any region that must not
 * allocate.  The address is looked up again after the device's context was
 * destroyed and re-created (cudaDeviceReset).
 * Every call shares the array: a call clears the counters it accumulates and
 * overwrites the rest, and the array keeps the last call's contents.  Calls
 * that overlap on the GPU (unordered streams or threads) race on it.  After
 * that first call the entry point allocates no memory, host or device.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_params* p, const int32_t* ids, const float* w,
                                        int64_t C, int32_t* slot, int32_t* offsets,
                                        int32_t* slot_token, float* slot_w, const void* x,
                                        void* x_perm, moe_stream_t stream);

/*
 * Routed SwiGLU experts on the dispatched rows (vegetog sec. 3:
 * E_i(x) = [SiLU(x W_gate,i) (.) (x W_up,i)] W_down,i; ch. 36.3: each expert
 * runs only on its accepted slots).
 *   x_perm  [N k, d] dtype (rows offsets[e] .. offsets[e+1]-1 belong to e)
 *   offsets [E_r + 1] from moe_dispatch
 *   H       [N k, d] fp32 out: H[r] = E_e(x_perm[r]) for r < offsets[E_r]
 * bf16 layers keep h = SiLU(.)(.)(.) in bf16 and accumulate in fp32; fp32
 * layers compute in fp32 throughout (no TF32).
 */
MOE_API moe_status moe_expert_ffn(const moe_params* p, const void* x_perm, const int32_t* offsets,
                          const void* W_g, const void* W_u, const void* W_d, float* H, void* ws,
                          moe_stream_t stream);

/*
 * Weighted combine (Algorithm 36.1 last step; ch. 36.3 combine matrix A_e):
 * Y[slot_token[r]] += slot_w[r] * H[r] for every accepted row r.  Y [N, d]
 * fp32 is accumulated into (the caller zeroes it first); rejected paths add
 * nothing and weights are not renormalised.  Summation order is free (fp32
 * atomics).
 */
MOE_API moe_status moe_combine(const moe_params* p, const float* H, const int32_t* offsets,
                       const int32_t* slot_token, const float* slot_w, float* Y,
                       moe_stream_t stream);

/*
 * The whole layer: route, dispatch, experts and combine, with the combine
 * fused into the down-projection epilogue, plus the shared expert
 * (ch. 36.6; DeepSeek-V3 form y = FFN_shared(x) + sum_i g_i FFN_i(x)) when
 * params.d_f_shared > 0.  Y [N, d] fp32 is overwritten.  Routing records
 * and statistics stay in the workspace (moe_workspace_layout, moe_get_stats).
 * Ws_g/Ws_u/Ws_d are required when d_f_shared > 0 and ignored otherwise.
 * The call only enqueues kernels and memsets on `stream` (no host wait, no
 * allocation), so it can be captured into a CUDA graph and replayed with new
 * contents of the same buffers; make the first call on a device outside a
 * capture (it sets the kernels' shared-memory attributes).
 */
MOE_API moe_status moe_forward(const moe_params* p, const void* x, const void* W_r, const float* b_r,
                       const float* lat, const void* W_g, const void* W_u, const void* W_d,
                       const void* Ws_g, const void* Ws_u, const void* Ws_d, float* Y, void* ws,
                       moe_stream_t stream);

/*
 * A routing group split over ranks (data parallel: each GPU holds a shard of
 * the group's tokens, ranks in token order, weights replicated).  Capacity
 * competition is defined over the whole routing group ("LLM from scratch"
 * ch. 36.3-36.4 and Algorithm 36.1; auturnal review: C from the group's token
 * count), so the shards exchange one small table: each rank's per-expert
 * request counts.  Two calls around that exchange give exactly the routing,
 * slots and outputs of one GPU running the concatenated batch:
 *
 * moe_forward_begin: route this rank's N = params.N tokens (as moe_route) and
 * count its requests per expert: counts [E_r] int32 (device, nullable; also
 * kept in the workspace).  The caller then all-gathers the counts of every
 * rank into counts_all [n_ranks][E_r] (for example with NCCL on the same
 * stream).
 *
 * moe_forward_end: with counts_all, this rank's requests for expert e are the
 * requests base_e .. base_e + L_e - 1 of the whole group (base_e = sum of the
 * counts of earlier ranks); the first C of the group are accepted.  Then it
 * dispatches, runs the experts and the combine as moe_forward does (same
 * x, weights, workspace; Y [N, d] overwritten).  C is the group's capacity
 * (moe_capacity with N = N_group, the group's token count).  slot records
 * hold group-wide slots.  moe_get_stats then reports this rank's request
 * counts (requested, accepted, rejected, tokens_affected, tokens_skipped) and
 * the group's loads (O, L_max, percentiles, rho_max over N_group).
 */
MOE_API moe_status moe_forward_begin(const moe_params* p, const void* x, const void* W_r,
                                     const float* b_r, const float* lat, int32_t* counts,
                                     void* ws, moe_stream_t stream);
MOE_API moe_status moe_forward_end(const moe_params* p, const int32_t* counts_all, int32_t rank,
                                   int32_t n_ranks, int64_t N_group, int64_t C, const void* x,
                                   const void* W_g, const void* W_u, const void* W_d,
                                   const void* Ws_g, const void* Ws_u, const void* Ws_d, float* Y,
                                   void* ws, moe_stream_t stream);

/*
 * Reads the routing statistics of the last dispatch on this workspace into
 * *out (host memory); waits for `stream`.  Returns MOE_ERR_NONFINITE when a
 * token had non-finite scores, MOE_ERR_TIMEOUT when a device wait gave up,
 * else MOE_OK (out is filled in every case).
 */
MOE_API moe_status moe_get_stats(const moe_params* p, const void* ws, moe_stats* out, moe_stream_t stream);

/*
 * Optional stage timing for moe_forward on the calling host thread: with
 * n >= 5 events (cudaEvent_t handles created by the caller), the next
 * moe_forward calls record events[0] at the start of the call's device work
 * (before the statistics counters are reset), [1] after routing,
 * [2] after dispatch, [3] after the gate/up expert GEMM and [4] after the
 * down-projection + combine, on the call's stream (moe_forward_begin records
 * [0] and [1], moe_forward_end [2] to [4]).  n = 0 turns it off.
 */
MOE_API moe_status moe_set_stage_events(void* const* events, int n);

/*
 * Dispatch step of a routing group sharded over ranks, on its own (the first
 * half of moe_forward_end): after moe_forward_begin on this workspace and
 * the exchange of the per-expert request counts (counts_all [n_ranks, E_r],
 * ranks in token order), accepts this rank's requests by their group-wide
 * token order, writes the routing records (slot, offsets, L, acc, slot_token,
 * slot_w in the workspace) and gathers the accepted rows of x into x_perm
 * (moe_workspace_layout), grouped by expert.  Used by expert parallelism
 * ("LLM from scratch" ch. 36.7: experts placed on different devices, token
 * rows sent to the device of their expert and the outputs sent back), where
 * x_perm's expert blocks are what each rank sends.  Token-order acceptance
 * only (MOE_ERR_UNSUPPORTED for MOE_ACCEPT_WEIGHT).  x may be NULL: the
 * routing records are written and no rows are gathered (the fused exchange,
 * moe_ep_dispatch, reads x itself).
 */
MOE_API moe_status moe_dispatch_ranked(const moe_params* p, const int32_t* counts_all, int32_t rank,
                                       int32_t n_ranks, int64_t N_group, int64_t C, const void* x, void* ws,
                                       moe_stream_t stream);

/*
 * Expert parallelism ("LLM from scratch" ch. 36.7: experts on different
 * devices; token rows go to their expert's device and the outputs come back).
 * Rank r of n_ranks owns experts [r El, (r+1) El), El = E_r / n_ranks; the
 * routing group's tokens are sharded over the ranks in token order.  Every
 * rank derives the same plan from the all-gathered request counts
 * counts_all [n_ranks][E_r] (moe_forward_begin): rank s's accepted requests for
 * expert e are acc[s][e] = min(C, cum_s[e]) - min(C, cum_{s-1}[e]), cum_s the
 * requests of ranks 0..s (token-order acceptance over the group).  An owner
 * keeps its rows expert-major: owned expert j's rows from rank 0, then rank 1,
 * ..., token order within a rank.
 *
 * moe_ep_plan: after moe_dispatch_ranked on this workspace.  Writes (device,
 * caller-owned) local_offsets [El + 1] (the owned experts' rows in this rank's
 * expert-major buffer), send_rows [n_ranks] and recv_rows [n_ranks] (the
 * split sizes of an all-to-all of x_perm's expert blocks), and, when given,
 * regroup / regroup_inv [rows received] (row i of the expert-major buffer is
 * received row regroup[i] of a source-major all-to-all; regroup_inv is the
 * inverse, for the return trip).  It also stores, in ws, where each of this
 * rank's expert blocks lands in its owner's expert-major buffer.
 *
 * moe_ep_dispatch: the exchange fused into the dispatch.  Copies each of this
 * rank's accepted rows of x [N, d] straight to its place in its owner's
 * expert-major buffer: recv_bufs is a DEVICE array of n_ranks device pointers
 * (rank r's buffer, of at least El C rows of d elements; another GPU's memory
 * reachable by peer access, or this GPU's own).  The kernel ends with a
 * system-scope fence; the caller orders the owners' expert computation
 * (moe_expert_ffn on their buffer with local_offsets) after every rank's
 * dispatch (a barrier across the ranks).
 *
 * moe_ep_combine: the return trip fused into the combine.  After the owners'
 * outputs are complete (a barrier across the ranks), Y[t] += a_te out[row] for
 * each of this rank's accepted rows, reading the output row from its owner's
 * buffer out_bufs[owner] (DEVICE array of n_ranks pointers to fp32 [rows, d]
 * expert-major outputs, peer or local).  Y is accumulated into (zero it
 * first); the shared expert, if any, is the caller's (replicated per rank).
 *
 * Token-order acceptance, overflow policies 0 and 1; n_ranks <= 64 dividing
 * E_r.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE,
 * MOE_ERR_CUDA (moe_last_error).  All three are asynchronous on `stream`.
 */
MOE_API moe_status moe_ep_plan(const moe_params* p, const int32_t* counts_all, int32_t rank, int32_t n_ranks,
                               int64_t C, int32_t* local_offsets, int32_t* send_rows, int32_t* recv_rows,
                               int32_t* regroup, int32_t* regroup_inv, void* ws, moe_stream_t stream);
MOE_API moe_status moe_ep_dispatch(const moe_params* p, int32_t n_ranks, const void* x, void* const* recv_bufs,
                                   const void* ws, moe_stream_t stream);
MOE_API moe_status moe_ep_combine(const moe_params* p, int32_t n_ranks, const float* const* out_bufs, float* Y,
                                  const void* ws, moe_stream_t stream);

/*
 * dst[i] = src[index[i]] for i < n_rows, rows of row_bytes bytes (a multiple
 * of 16; 16-byte aligned src and dst): the regrouping of rows exchanged
 * between ranks under expert parallelism (ch. 36.7).  No bounds checks on
 * index beyond the caller's contract (0 <= index[i] < rows of src).
 */
MOE_API moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t n_rows, int64_t row_bytes,
                                   void* dst, moe_stream_t stream);

/*
 * Soft MoE ("LLM from scratch" ch. 36.6, Soft Mixture of Experts): tokens are
 * mixed into S = E_r p slots, each expert processes its p slots, and the slot
 * outputs are mixed back into the tokens.
 *   Z  = X Phi^T [N, S]; D = softmax of Z over the tokens (each slot's column
 *   sums to one); C = softmax of Z over the slots (each token's row sums to
 *   one); Xs = D^T X [S, d]; Ys_s = E_{e(s)}(Xs_s) with e(s) = s / p (SwiGLU
 *   expert as in moe_forward); Y = C Ys [N, d].
 * Layouts: x [N, d] bf16; Phi [S, d] bf16 (slot s's score vector, slots of
 * expert e at rows e p .. e p + p - 1); W_g, W_u [E_r, d_f, d], W_d
 * [E_r, d, d_f] bf16 as in moe_forward; Y [N, d] fp32, overwritten.
 * Precision: scores, softmax statistics and all accumulations fp32; D, C, the
 * slot inputs and the slot outputs are bf16 operands of the tensor-core
 * contractions; the experts' hidden activations are bf16.
 * Constraints: dtype MOE_BF16 (fp32 soft layers are not built:
 * MOE_ERR_UNSUPPORTED); N, d, d_f and S multiples of 8 (16-byte operand rows),
 * N <= 65535 * 256 and S <= 65535 * 32 (else MOE_ERR_UNSUPPORTED).  Every token mixes into every slot, so this is
 * not causal across the batch.  Non-finite scores are not detected (they
 * propagate into Y).
 */
typedef struct moe_soft_params {
    int64_t N;          /* tokens                                                   */
    int32_t d;          /* model width                                              */
    int32_t d_f;        /* expert hidden width                                      */
    int32_t E_r;        /* experts, 1..1024                                         */
    int32_t p;          /* slots per expert (S = E_r p)                             */
    int32_t dtype;      /* MOE_BF16                                                 */
    int32_t reserved;
} moe_soft_params;

/* Workspace bytes of moe_soft_forward (caller-allocated, 16-byte aligned). */
MOE_API moe_status moe_soft_workspace_size(const moe_soft_params* p, size_t* bytes);

/* The Soft MoE forward pass above, asynchronous on `stream`; the library
 * allocates nothing.  Errors: MOE_ERR_INVALID_ARG (null or misaligned
 * pointers), MOE_ERR_WORKSPACE, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA (with
 * moe_last_error).  N = 0 returns MOE_OK with nothing launched. */
MOE_API moe_status moe_soft_forward(const moe_soft_params* p, const void* x, const void* Phi,
                                    const void* W_g, const void* W_u, const void* W_d, float* Y, void* ws,
                                    moe_stream_t stream);

/* Waits for `stream` and reports MOE_ERR_TIMEOUT if a device wait of the
 * last moe_soft_forward on `ws` gave up, else MOE_OK. */
MOE_API moe_status moe_soft_check(const moe_soft_params* p, const void* ws, moe_stream_t stream);

/*
 * Backward pass: gradients of
 *     L = sum_{t,o} dY[t,o] Y[t,o] + aux_coef * aux
 * for the forward pass that moe_forward last ran on `ws` (single routing
 * group, bf16 layer).  Y is the layer output ("LLM from scratch" ch. 36.3,
 * Algorithm 36.1; ch. 36.6 shared expert; vegetog "MoE token routing" sec. 3
 * SwiGLU expert) and aux the balance objective E_r sum_e f_e pbar_e of
 * ch. 36.4 (the value moe_stats.aux_balance reports).  The routing decisions
 * (top-k sets, WLR pruning, capacity acceptance) are held fixed: they are
 * piecewise constant in the inputs.  The objective's gradient reaches the
 * router only through the mean probabilities pbar_e (the hard shares f_e are
 * constants, ch. 36.4), via the softmax Jacobian.
 *
 * Chain (per accepted path j of token t with expert e, combine weight wc):
 *   dwc = <dY_t, o>, o = W_d h;  dh = wc W_d^T dY_t;  dW_d += wc dY_t h^T;
 *   dz = dh u SiLU'(z), du = dh SiLU(z);  dx_t += W_g^T dz + W_u^T du;
 *   dW_g += dz x_t^T, dW_u += du x_t^T;  combine weight -> routing weight
 *   (overflow policy, renormalisation over the chosen or surviving experts)
 *   -> probability -> score (softmax Jacobian) -> dx_t += W_r^T dg_t,
 *   dW_r = dg^T X, db_r = sum_t dg_t; the shared expert as an expert with
 *   weight 1 on every token.
 * Precision (bf16 layers): dY enters rounded to bf16; the forward's bf16 h is used as
 * stored (its rounding passes the gradient through); wc dY, dz and du are
 * rounded to bf16 as tensor-core operands; every accumulation and all router
 * arithmetic are fp32.  Gradients are fp32.
 *
 * Arguments: p, x, W_r, b_r and the weights exactly as given to that
 * moe_forward (b_r nullable); dY [N, d] fp32 (device); ws the forward's
 * workspace, unchanged since (its routing records, gathered rows x_perm and
 * hidden activations are read); offsets_host a HOST copy of the forward's
 * offsets [E_r + 1] (ws's "offsets" array, read after the forward finished:
 * the per-expert weight-gradient launches are sized by it); grads the output
 * buffers (device, fp32, overwritten; see moe_grads); bws, bws_bytes the
 * backward workspace (at least moe_backward_workspace_size bytes for these
 * offsets, 256-byte aligned recommended); aux_coef the objective's
 * coefficient (0: none).
 * fp32 layers: the same chain on the CUDA cores, nothing rounded.
 * Constraints: E_r <=
 * 256, k <= 32, N <= 65535 * 64; single routing group (not after
 * moe_forward_end).
 * Errors: MOE_ERR_INVALID_ARG (null or misaligned pointers, offsets_host not
 * a non-decreasing prefix from 0 to at most N k), MOE_ERR_WORKSPACE (missing,
 * misaligned or smaller than needed),
 * MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA (with moe_last_error).  Asynchronous on
 * `stream`; the library allocates nothing.  N = 0 zeroes the weight
 * gradients and returns.
 */
typedef struct moe_grads {
    float* dx;      /* [N, d]                       required (may be null when N = 0) */
    float* dW_r;    /* [E_r, d]                                        required */
    float* db_r;    /* [E_r]                                           nullable */
    float* dW_g;    /* [E_r, d_f, d]                                   required */
    float* dW_u;    /* [E_r, d_f, d]                                   required */
    float* dW_d;    /* [E_r, d, d_f]                                   required */
    float* dWs_g;   /* [d_f_shared, d]     required when d_f_shared > 0          */
    float* dWs_u;   /* [d_f_shared, d]     required when d_f_shared > 0          */
    float* dWs_d;   /* [d, d_f_shared]     required when d_f_shared > 0          */
} moe_grads;

/* Bytes of the backward workspace for p and the forward's offsets (host,
 * [E_r + 1]; the weight-gradient operands take E_r x max_e ceil64(rows of
 * expert e) columns).  offsets_host NULL: the bound for any routing (every
 * expert at min(capacity, N) rows).  MOE_ERR_INVALID_ARG for invalid
 * offsets. */
MOE_API moe_status moe_backward_workspace_size(const moe_params* p, const int32_t* offsets_host,
                                               size_t* bytes);

MOE_API moe_status moe_backward(const moe_params* p, float aux_coef, const int32_t* offsets_host,
                                const void* x, const void* W_r, const float* b_r, const void* W_g,
                                const void* W_u, const void* W_d, const void* Ws_g, const void* Ws_u,
                                const void* Ws_d, const float* dY, const void* ws, const moe_grads* grads,
                                void* bws, size_t bws_bytes, moe_stream_t stream);

/* Waits for `stream` and reports MOE_ERR_TIMEOUT if a bounded device wait of
 * the last moe_backward on `bws` gave up (its tensor-core GEMMs record that in
 * the backward workspace), MOE_ERR_INVALID_ARG if the offsets_host given to
 * that call differed from the forward's offsets on the device (a stale or
 * foreign host copy: the launches were sized from it, so the gradients are
 * not valid), else MOE_OK. */
MOE_API moe_status moe_backward_check(const moe_params* p, const void* bws, moe_stream_t stream);

/*
 * Self-test of the library's bounded device waits (no counterpart on the
 * pages).  Launches one CTA that waits on a shared-memory mbarrier nothing
 * ever arrives on, with the same bounded-wait routine the tensor-core GEMMs
 * use but a limit of limit_ns nanoseconds (1e6 .. 5e9) instead of 2 s; on
 * expiry the routine records the timeout in the counters of `ws` exactly as a
 * GEMM would, and the CTA returns.  `ws` is a workspace laid out for `p`; its
 * counters are reset first.  moe_get_stats then returns MOE_ERR_TIMEOUT with
 * device_error bit 0 set, and the CUDA context stays usable.  Asynchronous on
 * `stream`.  Errors: MOE_ERR_INVALID_ARG (limit out of range),
 * MOE_ERR_WORKSPACE (ws missing or misaligned), MOE_ERR_CUDA (launch).
 */
MOE_API moe_status moe_selftest_wait_timeout(const moe_params* p, void* ws, int64_t limit_ns,
                                             moe_stream_t stream);

/* Text of the last CUDA failure seen by an entry point on the calling host
 * thread ("" if none): the failing step and cudaGetErrorString's text. */
MOE_API const char* moe_last_error(void);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
