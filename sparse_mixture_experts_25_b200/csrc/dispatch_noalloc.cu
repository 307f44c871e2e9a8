// moe_dispatch_noalloc: the dispatch step with its scratch memory in a fixed,
// library-owned device buffer instead of a caller-provided workspace.
//
// Why it exists: some callers cannot allocate device memory at the point
// where they dispatch.  Examples are code running inside a memory pool that
// forbids growth, embedders whose allocator is not reachable from the call
// site, and call sites that must not call cudaMalloc because it can
// synchronise the device.  This variant takes only the inputs and outputs of
// moe_dispatch; its per-tile histograms, per-expert counts, M-tile prefix and
// counters live in a file-scope __device__ array of kScratchBytes (1 MiB).
// Every GPU that loads the library holds that array until the process exits.
//
// The array is shared by every call: each call overwrites it and clears the
// counters that must start at zero, and the buffer keeps the last call's
// contents afterwards.  Calls that overlap on the GPU (different streams or
// threads without ordering between them) race on it.
//
// The array's device address is looked up once per device and context: the
// first call on a device (and the first after that device's context was
// destroyed and re-created, e.g. by cudaDeviceReset) queries it with the
// device current.  With lazy module loading (the CUDA 12 default) that first
// query can be what loads the library's kernels onto the device, which
// reserves the 1 MiB array and may synchronise; later calls do neither.
#include <cudaTypedefs.h>
#include <mutex>
#include <stdio.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB

// Scratch layout (bytes from the start of the array):
//   [0, 128)                          int64 counters[16]
//   [128, 128 + 4 E)                  int32 L[E]
//   next 4 E                          int32 acc[E]
//   next 4 (E + 1)                    int32 M-tile prefix[E + 1]
//   next 4 E n_tiles                  int32 per-tile histograms [E][n_tiles]
static __device__ __align__(256) unsigned char g_dispatch_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};  // id of the context the address belongs to
std::mutex g_setup_mutex;

// Unique id of the calling thread's current context (0 if it cannot be read,
// in which case the address is looked up again on every call).
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

size_t scratch_needed(const moe_params& p, int n_tiles) {
    const size_t E = (size_t)p.E_r;
    return 128 + 4 * E + 4 * E + 4 * (E + 1) + 4 * E * (size_t)(n_tiles > 0 ? n_tiles : 1);
}

// Device address of the scratch array for the current device (set-up on the
// first call per device and context: a symbol-address query with that device
// current).  A cached address is dropped when the device's context changed
// since it was taken (a reset frees the array with the old context).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const unsigned long long ctx = current_context_id();  // 0 before the runtime made one current
    if (!g_scratch_addr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_dispatch_scratch);  // makes the primary context current
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = ptr;
        g_scratch_ctx[dev] = current_context_id();
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_dispatch_noalloc(const moe_params* p, const int32_t* ids, const float* w, int64_t C,
                                int32_t* slot, int32_t* offsets, int32_t* slot_token,
                                float* slot_w, const void* x, void* x_perm, moe_stream_t stream) {
    if (!p) return MOE_ERR_INVALID_ARG;
    moe_ws_layout lay;
    moe_status s = moe_workspace_layout(p, &lay);  // validates the parameters
    if (s != MOE_OK) return s;
    if (C < 1 || !offsets) return MOE_ERR_INVALID_ARG;
    if (p->accept_order == MOE_ACCEPT_WEIGHT) return MOE_ERR_UNSUPPORTED;  // token order only
    if (p->reject_policy == MOE_REJECT_REROUTE) return MOE_ERR_UNSUPPORTED;  // needs the workspace's candidates
    if ((x != nullptr) != (x_perm != nullptr)) return MOE_ERR_INVALID_ARG;
    if (x && ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u)))
        return MOE_ERR_INVALID_ARG;
    const int tile_tokens = dispatch_tile_tokens(p->k);
    const int n_tiles = (int)((p->N + tile_tokens - 1) / tile_tokens);
    const size_t need = scratch_needed(*p, n_tiles);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "moe_dispatch_noalloc: these sizes need %zu bytes of scratch, the static buffer "
                 "holds %zu (E_r per-tile counts for each tile of max(8, 128/k) tokens); use moe_dispatch",
                 need, kScratchBytes);
        record_error(msg);
        return MOE_ERR_UNSUPPORTED;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "moe_dispatch_noalloc set-up: %s", cudaGetErrorString(e));
        record_error(msg);
        return MOE_ERR_CUDA;
    }
    if (p->N == 0) {
        e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p->E_r + 1), st);
        if (e != cudaSuccess) {
            record_error("moe_dispatch_noalloc: memset of offsets failed");
            return MOE_ERR_CUDA;
        }
        return MOE_OK;
    }
    if (!ids || !w || !slot || !slot_token || !slot_w) return MOE_ERR_INVALID_ARG;
    char* b = static_cast<char*>(base);
    const size_t E = (size_t)p->E_r;
    unsigned long long* counters = reinterpret_cast<unsigned long long*>(b);
    int32_t* L = reinterpret_cast<int32_t*>(b + 128);
    int32_t* acc = L + E;
    Scratch sc{};
    sc.mt_start = acc + E;
    sc.hist = sc.mt_start + E + 1;
    sc.n_tiles = n_tiles;
    sc.tile_tokens = tile_tokens;
    (void)cudaGetLastError();
    // the counters are accumulated with atomics: start them at zero each call
    e = cudaMemsetAsync(counters, 0, CNT_COUNT * sizeof(unsigned long long), st);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "moe_dispatch_noalloc: %s", cudaGetErrorString(e));
        record_error(msg);
        return MOE_ERR_CUDA;
    }
    const int bm = p->dtype == MOE_BF16 ? tc_tile_rows(*p) : kSimtBM;
    const char* where = "";
    e = launch_dispatch(*p, C, bm, ids, w, slot, offsets, L, acc, slot_token, slot_w, x, x_perm,
                        counters, sc, st, &where);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "moe_dispatch_noalloc %s: %s", where, cudaGetErrorString(e));
        record_error(msg);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // extern "C"
