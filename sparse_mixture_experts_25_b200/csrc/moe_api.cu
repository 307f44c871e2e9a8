// C ABI of the sparse-MoE layer: argument checks, workspace layout and the
// stream-ordered launch sequence.  See include/moe.h for the contract of
// every entry point.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.cuh"

namespace moe {

size_t esize(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

int dispatch_tile_tokens(int k) {
    // about 128 requests per dispatch tile (one warp walks a tile)
#ifndef MOE_DISPATCH_TILE_REQUESTS
#define MOE_DISPATCH_TILE_REQUESTS 128
#endif
    int t = MOE_DISPATCH_TILE_REQUESTS / (k > 0 ? k : 1);
    return t < 8 ? 8 : t;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    if (dev < 64) cache[dev] = n;
    return n;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static bool layout(const moe_params& p, moe_ws_layout& L, int& n_tiles, int& tile_tokens) {
    const size_t Nk = (size_t)p.N * (size_t)p.k;
    const size_t E = (size_t)p.E_r;
    const size_t es = esize(p.dtype);
    tile_tokens = dispatch_tile_tokens(p.k);
    n_tiles = (int)((p.N + tile_tokens - 1) / tile_tokens);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    L.ids = take(Nk * 4);
    L.w = take(Nk * 4);
    L.margin = take((size_t)p.N * 4);
    L.slot = take(Nk * 4);
    L.offsets = take((E + 1) * 4);
    L.L = take(E * 4);
    L.acc = take(E * 4);
    L.slot_token = take(Nk * 4);
    L.slot_w = take(Nk * 4);
    L.counters = take(CNT_COUNT * 8);
    L.x_perm = take(Nk * (size_t)p.d * es);
    L.h = take(Nk * (size_t)p.d_f * es);
    L.h_shared = take((size_t)p.N * (size_t)(p.d_f_shared > 0 ? p.d_f_shared : 0) * es);
    const bool rr = p.reject_policy == MOE_REJECT_REROUTE;
    const size_t X = rr ? (size_t)p.reroute_depth : 0;
    L.cand = take((size_t)p.N * X * 4);
    L.cand_w = take((size_t)p.N * X * 4);
    L.rr_e = take(rr ? Nk * 4 : 0);
    L.rr_slot = take(rr ? Nk * 4 : 0);
    // scratch: per-tile histograms, M-tile prefix, earlier ranks' requests,
    // then (256-byte aligned) router scores, then the acceptance-by-weight
    // arrays (all-request offsets, selected keys and counts, requests, weights),
    // the per-expert probability sums and (rerouting) the rounds' state
    L.scratch = take(align_up(E * (size_t)std::max(n_tiles, 1) * 4 + (E + 1) * 4 + E * 4, 256) +
                     align_up((size_t)p.N * E * 4, 256) + align_up((3 * E + 1) * 4, 256) + align_up(2 * Nk * 4, 256) +
                     align_up(E * 4, 256) + (rr ? align_up(2 * Nk * 4 + (size_t)p.N * 4 + 16, 256) : 0) +
                     align_up(2 * E * 4, 256));
    L.total = off;
    return true;
}

bool make_view(const moe_params& p, void* ws, WsView& v) {
    int n_tiles, tile_tokens;
    layout(p, v.lay, n_tiles, tile_tokens);
    char* b = static_cast<char*>(ws);
    v.base = b;
    v.ids = reinterpret_cast<int32_t*>(b + v.lay.ids);
    v.w = reinterpret_cast<float*>(b + v.lay.w);
    v.margin = reinterpret_cast<float*>(b + v.lay.margin);
    v.slot = reinterpret_cast<int32_t*>(b + v.lay.slot);
    v.offsets = reinterpret_cast<int32_t*>(b + v.lay.offsets);
    v.L = reinterpret_cast<int32_t*>(b + v.lay.L);
    v.acc = reinterpret_cast<int32_t*>(b + v.lay.acc);
    v.slot_token = reinterpret_cast<int32_t*>(b + v.lay.slot_token);
    v.slot_w = reinterpret_cast<float*>(b + v.lay.slot_w);
    v.counters = reinterpret_cast<unsigned long long*>(b + v.lay.counters);
    v.x_perm = b + v.lay.x_perm;
    v.h = b + v.lay.h;
    v.h_shared = b + v.lay.h_shared;
    v.scratch.hist = reinterpret_cast<int32_t*>(b + v.lay.scratch);
    v.scratch.mt_start = v.scratch.hist + (size_t)p.E_r * std::max(n_tiles, 1);
    v.scratch.base = v.scratch.mt_start + p.E_r + 1;
    v.scratch.logits = reinterpret_cast<float*>(
        b + v.lay.scratch +
        align_up((size_t)p.E_r * std::max(n_tiles, 1) * 4 + ((size_t)p.E_r + 1) * 4 +
                     (size_t)p.E_r * 4, 256));
    {
        const size_t Nk = (size_t)p.N * p.k;
        char* pr = reinterpret_cast<char*>(v.scratch.logits) + align_up((size_t)p.N * p.E_r * 4, 256);
        v.scratch.all_offsets = reinterpret_cast<int32_t*>(pr);
        v.scratch.sel_key = reinterpret_cast<uint32_t*>(v.scratch.all_offsets + p.E_r + 1);
        v.scratch.sel_take = reinterpret_cast<int32_t*>(v.scratch.sel_key + p.E_r);
        pr += align_up((3 * (size_t)p.E_r + 1) * 4, 256);
        v.scratch.seg_req = reinterpret_cast<int32_t*>(pr);
        v.scratch.seg_w = reinterpret_cast<float*>(pr + Nk * 4);
        v.scratch.psum = reinterpret_cast<float*>(pr + align_up(2 * Nk * 4, 256));
        char* rq = reinterpret_cast<char*>(v.scratch.psum) + align_up((size_t)p.E_r * 4, 256);
        v.scratch.rr_q = reinterpret_cast<int32_t*>(rq);
        v.scratch.rr_offer = v.scratch.rr_q + Nk;
        v.scratch.rr_next = v.scratch.rr_offer + Nk;
        v.scratch.rr_stop = v.scratch.rr_next + p.N;
        const bool rr = p.reject_policy == MOE_REJECT_REROUTE;
        char* ep = rq + (rr ? align_up(2 * Nk * 4 + (size_t)p.N * 4 + 16, 256) : 0);
        v.scratch.ep_dest = reinterpret_cast<int32_t*>(ep);
        v.scratch.ep_recv_base = v.scratch.ep_dest + p.E_r;
    }
    v.cand = reinterpret_cast<int32_t*>(b + v.lay.cand);
    v.cand_w = reinterpret_cast<float*>(b + v.lay.cand_w);
    v.rr_e = reinterpret_cast<int32_t*>(b + v.lay.rr_e);
    v.rr_slot = reinterpret_cast<int32_t*>(b + v.lay.rr_slot);
    v.scratch.cand = v.cand;
    v.scratch.cand_w = v.cand_w;
    v.scratch.rr_e = v.rr_e;
    v.scratch.rr_slot = v.rr_slot;
    v.scratch.n_tiles = n_tiles;
    v.scratch.tile_tokens = tile_tokens;
    return true;
}

}  // namespace moe

using namespace moe;

namespace {

thread_local cudaEvent_t g_stage_events[8];
thread_local char g_last_error[256] = "";

moe_status fail(cudaError_t e, const char* where) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    return MOE_ERR_CUDA;
}
thread_local int g_stage_event_count = 0;

// Stage boundaries of moe_forward / moe_forward_begin + moe_forward_end:
// 0 before routing, 1 after routing, 2 after dispatch, 3 after gate/up,
// 4 after down + combine.  Each boundary records the caller's stage event (if
// any) and closes / opens an NVTX range named after the stage, so a timeline
// profiler shows the host-side enqueue of each stage.
thread_local nvtxRangeId_t g_nvtx_range = 0;

inline cudaError_t stage_mark(int i, cudaStream_t st) {
    static const char* const kStageNames[4] = {"moe route", "moe dispatch", "moe gate/up + SwiGLU",
                                               "moe down + combine"};
    if (g_nvtx_range) {
        nvtxRangeEnd(g_nvtx_range);
        g_nvtx_range = 0;
    }
    if (i < 4) g_nvtx_range = nvtxRangeStartA(kStageNames[i]);
    if (g_stage_event_count >= 5 && i < g_stage_event_count) return cudaEventRecord(g_stage_events[i], st);
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status check_params(const moe_params* p) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (p->N < 0 || p->d < 1 || p->d_f < 1 || p->E_r < 1 || p->k < 1 || p->k > p->E_r)
        return MOE_ERR_INVALID_ARG;
    if (p->norm < MOE_NORM_RENORM || p->norm > MOE_NORM_WLR) return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_F32 && p->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (p->d_f_shared < 0) return MOE_ERR_INVALID_ARG;
    if (p->reject_policy != MOE_REJECT_ZERO && p->reject_policy != MOE_REJECT_RENORM &&
        p->reject_policy != MOE_REJECT_REROUTE)
        return MOE_ERR_INVALID_ARG;
    if (p->reject_policy == MOE_REJECT_REROUTE) {
        // candidates are ranks k .. k + depth - 1, held one per lane of a warp
        if (p->reroute_depth < 1 || p->reroute_depth > p->E_r - p->k || p->k + p->reroute_depth > kMaxK)
            return MOE_ERR_INVALID_ARG;
        if (p->norm == MOE_NORM_WLR || p->accept_order != MOE_ACCEPT_TOKEN) return MOE_ERR_UNSUPPORTED;
    }
    if (p->accept_order != MOE_ACCEPT_TOKEN && p->accept_order != MOE_ACCEPT_WEIGHT)
        return MOE_ERR_INVALID_ARG;
    if (!(p->c == p->c) || p->c > 1e6) return MOE_ERR_INVALID_ARG;
    if (p->norm == MOE_NORM_WLR && !(p->theta >= 0.f && p->theta < 1.f)) return MOE_ERR_INVALID_ARG;
    if (p->E_r > kMaxExperts || p->k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (p->d % 8 || p->d_f % 8 || p->d_f_shared % 8) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)p->N * p->k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status cuda_status(cudaError_t e, const char* where) {
    return e == cudaSuccess ? MOE_OK : fail(e, where);
}

// exact capacity on the binary value of c (see moe.h)
int64_t capacity_exact(double c, int64_t N, int k, int E) {
    if (c <= 0.0) return N;
    int ex = 0;
    const double m = frexp(c, &ex);                      // c = m 2^ex, m in [0.5, 1)
    const __int128 mant = (__int128)ldexp(m, 53);        // c = mant 2^(ex-53), exact
    const int sh = ex - 53;
    __int128 num = mant * (__int128)N * (__int128)k;
    __int128 den = (__int128)E;
    if (sh >= 0) {
        num <<= sh;
    } else {
        int s = -sh;
        while (s > 0 && (num & 1) == 0) {  // strip common powers of two
            num >>= 1;
            --s;
        }
        den <<= s;
    }
    const __int128 fl = num / den;
    const __int128 rem = num - fl * den;
    const __int128 r = (2 * rem >= den) ? fl + 1 : fl;   // nearest integer
    const long double q = (long double)num / (long double)den;
    const long double dist = fabsl(q - (long double)r);
    const long double tol = 1e-9L * (q > 1.0L ? q : 1.0L);
    int64_t C = (dist <= tol) ? (int64_t)r : (int64_t)(rem ? fl + 1 : fl);
    if (N > 0 && C < 1) C = 1;
    return C;
}

}  // namespace

namespace moe {
void record_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
}  // namespace moe

extern "C" {

const char* moe_last_error(void) { return g_last_error; }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported size or mode";
        case MOE_ERR_NONFINITE: return "non-finite router score (input failure)";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_WORKSPACE: return "workspace missing or misaligned";
        case MOE_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

moe_status moe_capacity(const moe_params* p, int64_t* C) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (!C) return MOE_ERR_INVALID_ARG;
    *C = capacity_exact(p->c, p->N, p->k, p->E_r);
    return MOE_OK;
}

moe_status moe_workspace_layout(const moe_params* p, moe_ws_layout* out) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (!out) return MOE_ERR_INVALID_ARG;
    int n_tiles, tile_tokens;
    layout(*p, *out, n_tiles, tile_tokens);
    return MOE_OK;
}

moe_status moe_workspace_size(const moe_params* p, size_t* bytes) {
    moe_ws_layout L;
    moe_status s = moe_workspace_layout(p, &L);
    if (s != MOE_OK) return s;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = L.total;
    return MOE_OK;
}

moe_status moe_set_stage_events(void* const* events, int n) {
    if (n < 0 || n > 8 || (n > 0 && !events)) return MOE_ERR_INVALID_ARG;
    if (n > 0 && n < 5) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_event_count = n;
    return MOE_OK;
}

moe_status moe_route(const moe_params* p, const void* x, const void* W_r, const float* b_r,
                     const float* lat, int32_t* ids, float* w, float* margin, void* ws,
                     moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->E_r > kMaxRouterExperts) return MOE_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (p->N == 0) return MOE_OK;
    if (!x || !W_r || !ids || !w || !aligned16(x) || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
    if (p->norm == MOE_NORM_WLR && !lat) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e = cudaMemsetAsync(v.counters, 0, CNT_COUNT * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.scratch.psum, 0, sizeof(float) * p->E_r, st);
    if (e != cudaSuccess) return fail(e, "moe_route memset");
    return cuda_status(launch_router(*p, x, W_r, b_r, p->norm == MOE_NORM_WLR ? lat : nullptr, ids,
                                     w, margin, v.counters, nullptr, v.scratch.logits, v.scratch.psum, st,
                                     v.cand, v.cand_w),
                       "moe_route router");
}

moe_status moe_dispatch(const moe_params* p, const int32_t* ids, const float* w, int64_t C,
                        int32_t* slot, int32_t* offsets, int32_t* slot_token, float* slot_w,
                        const void* x, void* x_perm, void* ws, moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (C < 1) return MOE_ERR_INVALID_ARG;
    if (!offsets) return MOE_ERR_INVALID_ARG;
    if ((x != nullptr) != (x_perm != nullptr)) return MOE_ERR_INVALID_ARG;
    if (x && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    if (p->N == 0) {
        cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p->E_r + 1), st);
        if (e != cudaSuccess) return fail(e, "moe_dispatch memset");
        return MOE_OK;
    }
    if (!ids || !w || !slot || !slot_token || !slot_w) return MOE_ERR_INVALID_ARG;
    (void)cudaGetLastError();
    // dispatch-side counters start from zero; router counters are kept
    cudaError_t e = cudaMemsetAsync(v.counters + CNT_REQUESTED, 0, 6 * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.counters + CNT_L_MAX, 0, 2 * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.counters + CNT_REROUTED, 0, 8, st);
    if (e != cudaSuccess) return fail(e, "moe_dispatch memset");
    const int bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
    const char* where = "";
    e = launch_dispatch(*p, C, bm, ids, w, slot, offsets, v.L, v.acc, slot_token, slot_w, x, x_perm,
                        v.counters, v.scratch, st, &where);
    if (e != cudaSuccess) {
        char buf[96];
        snprintf(buf, sizeof(buf), "moe_dispatch %s", where);
        return fail(e, buf);
    }
    return MOE_OK;
}

moe_status moe_expert_ffn(const moe_params* p, const void* x_perm, const int32_t* offsets,
                          const void* W_g, const void* W_u, const void* W_d, float* H, void* ws,
                          moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (p->N == 0) return MOE_OK;
    if (!x_perm || !offsets || !W_g || !W_u || !W_d || !H) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(W_g) || !aligned16(W_u) || !aligned16(W_d) || !aligned16(H))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    moe_params q = *p;
    q.d_f_shared = 0;  // routed experts only
    ExpertWeights W{W_g, W_u, W_d, nullptr, nullptr, nullptr};
    const int bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
    (void)cudaGetLastError();
    cudaError_t e0 = launch_mtile_prefix(p->E_r, bm, offsets, v.scratch.mt_start, st);
    if (e0 != cudaSuccess) return fail(e0, "moe_expert_ffn prefix");
    int status = MOE_OK;
    cudaError_t e;
    if (p->dtype == MOE_BF16) {
        e = launch_tc_gate_up(q, x_perm, nullptr, offsets, v.scratch.mt_start, W, v.h, nullptr,
                              nullptr, v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, status != MOE_OK ? "moe_expert_ffn gate/up: tensor map encode" : "moe_expert_ffn gate/up (tcgen05)");
        e = launch_tc_down(q, DOWN_STORE, p->N, v.h, nullptr, offsets, v.scratch.mt_start, W, nullptr,
                           nullptr, nullptr, H, v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, status != MOE_OK ? "moe_expert_ffn down: tensor map encode" : "moe_expert_ffn down (tcgen05)");
    } else {
        e = launch_simt_gate_up(q, x_perm, nullptr, offsets, v.scratch.mt_start, W, v.h, nullptr, st);
        if (e != cudaSuccess) return fail(e, "moe_expert_ffn gate/up (fp32)");
        e = launch_simt_down(q, DOWN_STORE, v.h, nullptr, offsets, v.scratch.mt_start, W, nullptr,
                             nullptr, nullptr, H, st);
        if (e != cudaSuccess) return fail(e, "moe_expert_ffn down (fp32)");
    }
    return MOE_OK;
}

moe_status moe_combine(const moe_params* p, const float* H, const int32_t* offsets,
                       const int32_t* slot_token, const float* slot_w, float* Y,
                       moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->N == 0) return MOE_OK;
    if (!H || !offsets || !slot_token || !slot_w || !Y || !aligned16(H) || !aligned16(Y))
        return MOE_ERR_INVALID_ARG;
    (void)cudaGetLastError();
    return cuda_status(launch_combine(*p, H, offsets, slot_token, slot_w, Y,
                                      reinterpret_cast<cudaStream_t>(stream)), "moe_combine");
}

moe_status moe_forward(const moe_params* p, const void* x, const void* W_r, const float* b_r,
                       const float* lat, const void* W_g, const void* W_u, const void* W_d,
                       const void* Ws_g, const void* Ws_u, const void* Ws_d, float* Y, void* ws,
                       moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->E_r > kMaxRouterExperts) return MOE_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();  // clear a stale non-sticky error left by earlier unrelated calls
    cudaError_t e0;
    if (p->N > 0 && (e0 = stage_mark(0, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
    e0 = cudaMemsetAsync(v.counters, 0, CNT_COUNT * 8, st);
    if (e0 == cudaSuccess) e0 = cudaMemsetAsync(v.scratch.psum, 0, sizeof(float) * p->E_r, st);
    if (e0 != cudaSuccess) return fail(e0, "moe_forward memset");
    if (p->N == 0) return MOE_OK;
    if (!x || !W_r || !W_g || !W_u || !W_d || !Y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_r) || !aligned16(W_g) || !aligned16(W_u) || !aligned16(W_d) ||
        !aligned16(Y))
        return MOE_ERR_INVALID_ARG;
    if (p->norm == MOE_NORM_WLR && !lat) return MOE_ERR_INVALID_ARG;
    const bool sh = p->d_f_shared > 0;
    if (sh && (!Ws_g || !Ws_u || !Ws_d || !aligned16(Ws_g) || !aligned16(Ws_u) || !aligned16(Ws_d)))
        return MOE_ERR_INVALID_ARG;
    const int64_t C = capacity_exact(p->c, p->N, p->k, p->E_r);
    ExpertWeights W{W_g, W_u, W_d, sh ? Ws_g : nullptr, sh ? Ws_u : nullptr, sh ? Ws_d : nullptr};

    // bf16 layers zero Y inside the gate/up kernel (hidden behind its first
    // tile); fp32 layers zero it in the router
    const bool bf16 = p->dtype == MOE_BF16;
    cudaError_t e = launch_router(*p, x, W_r, b_r, p->norm == MOE_NORM_WLR ? lat : nullptr, v.ids,
                                  v.w, v.margin, v.counters, bf16 ? nullptr : Y, v.scratch.logits,
                                  v.scratch.psum, st, v.cand, v.cand_w);
    if (e != cudaSuccess) return fail(e, "moe_forward router");
    if ((e0 = stage_mark(1, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
    const int bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
    const char* where = "";
    e = launch_dispatch(*p, C, bm, v.ids, v.w, v.slot, v.offsets, v.L, v.acc, v.slot_token, v.slot_w,
                        x, v.x_perm, v.counters, v.scratch, st, &where);
    if (e != cudaSuccess) {
        char buf[96];
        snprintf(buf, sizeof(buf), "moe_forward dispatch %s", where);
        return fail(e, buf);
    }
    if ((e0 = stage_mark(2, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
    int status = MOE_OK;
    if (p->dtype == MOE_BF16) {
        e = launch_tc_gate_up(*p, v.x_perm, x, v.offsets, v.scratch.mt_start, W, v.h, v.h_shared,
                              Y, v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, status != MOE_OK ? "moe_forward gate/up: tensor map encode" : "moe_forward gate/up (tcgen05)");
        if ((e0 = stage_mark(3, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
        e = launch_tc_down(*p, DOWN_COMBINE, C, v.h, v.h_shared, v.offsets, v.scratch.mt_start, W,
                           v.slot_token, v.slot_w, Y, nullptr, v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, status != MOE_OK ? "moe_forward down: tensor map encode" : "moe_forward down+combine (tcgen05)");
    } else {
        e = launch_simt_gate_up(*p, v.x_perm, x, v.offsets, v.scratch.mt_start, W, v.h, v.h_shared, st);
        if (e != cudaSuccess) return fail(e, "moe_forward gate/up (fp32)");
        if ((e0 = stage_mark(3, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
        e = launch_simt_down(*p, DOWN_COMBINE, v.h, v.h_shared, v.offsets, v.scratch.mt_start, W,
                             v.slot_token, v.slot_w, Y, nullptr, st);
        if (e != cudaSuccess) return fail(e, "moe_forward down+combine (fp32)");
    }
    if ((e0 = stage_mark(4, st)) != cudaSuccess) return fail(e0, "moe_forward stage event");
    return MOE_OK;
}

moe_status moe_forward_begin(const moe_params* p, const void* x, const void* W_r, const float* b_r,
                             const float* lat, int32_t* counts, void* ws, moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->accept_order == MOE_ACCEPT_WEIGHT) return MOE_ERR_UNSUPPORTED;  // needs every rank's weights
    if (p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;  // single routing group only
    if (p->E_r > kMaxRouterExperts) return MOE_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e;
    if (p->N > 0 && (e = stage_mark(0, st)) != cudaSuccess) return fail(e, "moe_forward_begin stage event");
    e = cudaMemsetAsync(v.counters, 0, CNT_COUNT * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.scratch.psum, 0, sizeof(float) * p->E_r, st);
    if (e != cudaSuccess) return fail(e, "moe_forward_begin memset");
    if (p->N == 0) {
        if (counts) {
            e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * p->E_r, st);
            if (e != cudaSuccess) return fail(e, "moe_forward_begin memset");
        }
        return MOE_OK;
    }
    if (!x || !W_r || !aligned16(x) || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
    if (p->norm == MOE_NORM_WLR && !lat) return MOE_ERR_INVALID_ARG;
    e = launch_router(*p, x, W_r, b_r, p->norm == MOE_NORM_WLR ? lat : nullptr, v.ids, v.w, v.margin,
                      v.counters, nullptr, v.scratch.logits, v.scratch.psum, st);
    if (e != cudaSuccess) return fail(e, "moe_forward_begin router");
    if ((e = stage_mark(1, st)) != cudaSuccess) return fail(e, "moe_forward_begin stage event");
    e = launch_count(*p, v.ids, v.L, counts, v.counters, v.scratch, st);
    if (e != cudaSuccess) return fail(e, "moe_forward_begin counts");
    return MOE_OK;
}

moe_status moe_dispatch_ranked(const moe_params* p, const int32_t* counts_all, int32_t rank, int32_t n_ranks,
                               int64_t N_group, int64_t C, const void* x, void* ws, moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->accept_order == MOE_ACCEPT_WEIGHT) return MOE_ERR_UNSUPPORTED;  // needs every rank's weights
    if (p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;  // single routing group only
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks || !counts_all || C < 1 || N_group < p->N)
        return MOE_ERR_INVALID_ARG;
    if (p->N == 0) return MOE_OK;
    if (x && !aligned16(x)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e = cudaMemsetAsync(v.counters + CNT_REQUESTED, 0, 6 * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.counters + CNT_L_MAX, 0, 2 * 8, st);
    if (e != cudaSuccess) return fail(e, "moe_dispatch_ranked memset");
    const int bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
    const char* where = "";
    e = launch_dispatch_ranked(*p, C, bm, counts_all, rank, n_ranks, N_group, v.ids, v.w, v.slot, v.offsets, v.L,
                               v.acc, v.slot_token, v.slot_w, x, x ? v.x_perm : nullptr, v.counters, v.scratch, st,
                               &where);
    if (e != cudaSuccess) {
        char buf[96];
        snprintf(buf, sizeof(buf), "moe_dispatch_ranked %s", where);
        return fail(e, buf);
    }
    return MOE_OK;
}

moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t n_rows, int64_t row_bytes, void* dst,
                           moe_stream_t stream) {
    if (n_rows < 0 || row_bytes <= 0 || row_bytes % 16) return MOE_ERR_INVALID_ARG;
    if (n_rows == 0) return MOE_OK;
    if (!src || !index || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
    (void)cudaGetLastError();
    cudaError_t e = launch_gather_rows(src, index, n_rows, row_bytes, dst, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(e, "moe_gather_rows");
    return MOE_OK;
}

moe_status moe_forward_end(const moe_params* p, const int32_t* counts_all, int32_t rank,
                           int32_t n_ranks, int64_t N_group, int64_t C, const void* x,
                           const void* W_g, const void* W_u, const void* W_d, const void* Ws_g,
                           const void* Ws_u, const void* Ws_d, float* Y, void* ws,
                           moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (p->accept_order == MOE_ACCEPT_WEIGHT) return MOE_ERR_UNSUPPORTED;  // needs every rank's weights
    if (p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;  // single routing group only
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks || !counts_all || C < 1 || N_group < p->N)
        return MOE_ERR_INVALID_ARG;
    if (p->N == 0) return MOE_OK;
    if (!x || !W_g || !W_u || !W_d || !Y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_g) || !aligned16(W_u) || !aligned16(W_d) || !aligned16(Y))
        return MOE_ERR_INVALID_ARG;
    const bool sh = p->d_f_shared > 0;
    if (sh && (!Ws_g || !Ws_u || !Ws_d || !aligned16(Ws_g) || !aligned16(Ws_u) || !aligned16(Ws_d)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e = cudaMemsetAsync(v.counters + CNT_REQUESTED, 0, 6 * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.counters + CNT_L_MAX, 0, 2 * 8, st);
    if (e != cudaSuccess) return fail(e, "moe_forward_end memset");
    const bool bf16 = p->dtype == MOE_BF16;
    const int bm = bf16 ? tc_tile_rows(*p) : kSimtBM;
    const char* where = "";
    e = launch_dispatch_ranked(*p, C, bm, counts_all, rank, n_ranks, N_group, v.ids, v.w, v.slot,
                               v.offsets, v.L, v.acc, v.slot_token, v.slot_w, x, v.x_perm,
                               v.counters, v.scratch, st, &where);
    if (e != cudaSuccess) {
        char buf[96];
        snprintf(buf, sizeof(buf), "moe_forward_end dispatch %s", where);
        return fail(e, buf);
    }
    ExpertWeights W{W_g, W_u, W_d, sh ? Ws_g : nullptr, sh ? Ws_u : nullptr, sh ? Ws_d : nullptr};
    if ((e = stage_mark(2, st)) != cudaSuccess) return fail(e, "moe_forward_end stage event");
    int status = MOE_OK;
    if (bf16) {
        e = launch_tc_gate_up(*p, v.x_perm, x, v.offsets, v.scratch.mt_start, W, v.h, v.h_shared, Y,
                              v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, "moe_forward_end gate/up (tcgen05)");
        if ((e = stage_mark(3, st)) != cudaSuccess) return fail(e, "moe_forward_end stage event");
        e = launch_tc_down(*p, DOWN_COMBINE, C, v.h, v.h_shared, v.offsets, v.scratch.mt_start, W,
                           v.slot_token, v.slot_w, Y, nullptr, v.counters, st, &status);
        if (e != cudaSuccess) return fail(e, "moe_forward_end down+combine (tcgen05)");
    } else {
        e = launch_zero_f32(Y, p->N * (int64_t)p->d, st);
        if (e != cudaSuccess) return fail(e, "moe_forward_end zero");
        e = launch_simt_gate_up(*p, v.x_perm, x, v.offsets, v.scratch.mt_start, W, v.h, v.h_shared, st);
        if (e != cudaSuccess) return fail(e, "moe_forward_end gate/up (fp32)");
        if ((e = stage_mark(3, st)) != cudaSuccess) return fail(e, "moe_forward_end stage event");
        e = launch_simt_down(*p, DOWN_COMBINE, v.h, v.h_shared, v.offsets, v.scratch.mt_start, W,
                             v.slot_token, v.slot_w, Y, nullptr, st);
        if (e != cudaSuccess) return fail(e, "moe_forward_end down+combine (fp32)");
    }
    if ((e = stage_mark(4, st)) != cudaSuccess) return fail(e, "moe_forward_end stage event");
    return MOE_OK;
}

moe_status moe_selftest_wait_timeout(const moe_params* p, void* ws, int64_t limit_ns, moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (limit_ns < 1000000 || limit_ns > 5000000000LL) return MOE_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, ws, v);
    (void)cudaGetLastError();
    cudaError_t e = cudaMemsetAsync(v.counters, 0, CNT_COUNT * 8, st);
    if (e == cudaSuccess) e = launch_wait_selftest(v.counters, (unsigned long long)limit_ns, st);
    if (e != cudaSuccess) return fail(e, "moe_selftest_wait_timeout");
    return MOE_OK;
}

moe_status moe_get_stats(const moe_params* p, const void* ws, moe_stats* out, moe_stream_t stream) {
    moe_status s = check_params(p);
    if (s != MOE_OK) return s;
    if (!ws || !out) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsView v;
    make_view(*p, const_cast<void*>(ws), v);
    unsigned long long cnt[CNT_COUNT];
    std::vector<int32_t> L((size_t)p->E_r), acc((size_t)p->E_r);
    std::vector<float> psum((size_t)p->E_r);
    memset(out, 0, sizeof(*out));
    cudaError_t e = cudaMemcpyAsync(cnt, v.counters, sizeof(cnt), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(L.data(), v.L, sizeof(int32_t) * L.size(), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(acc.data(), v.acc, sizeof(int32_t) * acc.size(), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(psum.data(), v.scratch.psum, sizeof(float) * psum.size(), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(e, "moe_get_stats");
    out->C = (int64_t)cnt[CNT_C];
    out->requested = (int64_t)cnt[CNT_REQUESTED];
    out->accepted = (int64_t)cnt[CNT_ACCEPTED];
    out->rejected = (int64_t)cnt[CNT_REJECTED];
    out->O = (int64_t)cnt[CNT_O];
    out->tokens_affected = (int64_t)cnt[CNT_AFFECTED];
    out->tokens_skipped = (int64_t)cnt[CNT_SKIPPED];
    out->nonfinite = (int64_t)cnt[CNT_NONFINITE];
    out->near_tie = (int64_t)cnt[CNT_NEAR_TIE];
    out->L_max = (int64_t)cnt[CNT_L_MAX];
    out->device_error = (int32_t)cnt[CNT_DEVICE_ERROR];
    out->rerouted = (int32_t)cnt[CNT_REROUTED];
    if (p->N > 0) {
        std::vector<int32_t> srt(L);
        std::sort(srt.begin(), srt.end());
        auto pct = [&](double q) {
            size_t rank = (size_t)ceil(q / 100.0 * (double)srt.size());
            if (rank < 1) rank = 1;
            return (int64_t)srt[rank - 1];
        };
        out->L_p50 = pct(50);
        out->L_p90 = pct(90);
        out->L_p99 = pct(99);
        const double n_group = cnt[CNT_N_GROUP] ? (double)cnt[CNT_N_GROUP] : (double)p->N;
        out->rho_max = (double)out->L_max * (double)p->E_r / (n_group * (double)p->k);
        out->reject_rate = out->requested ? (double)out->rejected / (double)out->requested : 0.0;
        // rows the routed GEMMs compute: accepted rows per expert rounded up
        // to the row tile of the kernels that run them
        const int64_t bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
        const bool swap = p->dtype == MOE_BF16 && tc_swap_tails(*p);
        int64_t padded = 0, accepted = 0;
        for (int32_t a : acc) {
            const int64_t rem = a % 256, tail = swap && rem <= 128 ? rem : 0;
            // a tail of at most 128 rows runs as one tile of its tokens rounded up to 32
            padded += (a - tail + bm - 1) / bm * bm + (tail + 31) / 32 * 32;
            // single-CTA tcgen05 tiles: a last tile of at most 64 rows is an M=64 MMA
            if (p->dtype == MOE_BF16 && bm == 128 && a % 128 > 0 && a % 128 <= 64) padded -= 64;
            accepted += a;
        }
        out->padded_rows = padded;
        out->padding_ratio = accepted ? (double)padded / (double)accepted : 0.0;
        // balance statistic: E_r sum_e f_e pbar_e, f_e = L_e / sum L (requests
        // before capacity), pbar_e = mean full-softmax probability over the
        // tokens with finite scores
        const double n_valid = (double)(p->N - (int64_t)cnt[CNT_NONFINITE]);
        double req = 0.0;
        for (int32_t l : L) req += l;
        double aux = 0.0;
        if (req > 0 && n_valid > 0)
            for (int e2 = 0; e2 < p->E_r; ++e2) aux += ((double)L[e2] / req) * ((double)psum[e2] / n_valid);
        out->aux_balance = aux * p->E_r;
    }
    if (cnt[CNT_DEVICE_ERROR] & DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (cnt[CNT_NONFINITE]) return MOE_ERR_NONFINITE;
    return MOE_OK;
}

}  // extern "C"
