// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// What they compute (vegetog "MoE token routing" sec. 3, SwiGLU expert
// E_i(x) = [SiLU(x W_gate,i) (.) (x W_up,i)] W_down,i; "LLM from scratch"
// ch. 36.3: each expert runs only on its accepted slots, then
// Y_t += a_te (H_e)_c; ch. 36.6: the shared expert adds F_sh(x) with weight 1):
//   gate/up  h[r, :] = SiLU(x_r W_g^T) (.) (x_r W_u^T)        bf16 out
//   down     Y[tok(r), :] += a(r) * (h[r, :] W_d^T)            fp32 atomics
//            (or H[r, :] = h[r, :] W_d^T for the unfused entry point)
//
// Design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0     TMA producer: per 64-wide K block it loads the A tile
//              (128 rows x 64, bf16) and two 128-row B tiles into one
//              shared-memory stage (4 stages of 48 KB, 128-byte swizzle).
//   warp 1     MMA issuer: one elected thread issues tcgen05.mma
//              (cta_group::1, kind::f16, M=128, N=256, K=16, fp32 accumulate)
//              into one of two TMEM accumulators (2 x 256 columns), commits
//              each stage back to the producer and each finished tile to the
//              epilogue.
//   warps 2-5  epilogue: tcgen05.ld of the accumulator rows (one TMEM lane
//              per row), then SwiGLU -> bf16 h (gate/up) or the weighted
//              scatter-combine with 16-byte fp32 red.global.add (down), each
//              32-column chunk transposed through a per-warp 128-byte-swizzled
//              shared-memory tile so one warp instruction adds 4 rows x 128
//              contiguous bytes.  Plain fp32 outputs (the store epilogue)
//              leave that tile by TMA store, 32 rows x 32 columns at a time,
//              when all 32 rows of the warp's slab are valid.
// For gate/up the two B tiles are the gate and up rows of the same 128
// output columns, so one N=256 MMA yields both and the SwiGLU is local to a
// thread.  For the down projection they are two consecutive 128-row halves
// of a 256-column output tile.
//
// Layers with many rows per expert run on CTA pairs instead (cluster of 2,
// cta_group::2 MMAs issued by the leader): a 256 x 256 tile, each CTA loading
// its 128 A rows and half of B (6 stages of 32 KB), so each SM reads half the
// B bytes per MMA.  A pair tile of at most 128 rows uses the M=128 pair MMA
// (64 A rows per CTA).  On pairs the gate/up B half of a CTA is 64 gate rows
// followed by the 64 up rows of the same columns, which keeps gate and up of
// one output column in one TMEM lane for both tile heights.
//
// Tiles are scheduled statically (tile = blockIdx.x + i * gridDim.x) over a
// list ordered group by group, output-column tile by column tile, with the
// row tiles of one group fastest, so CTAs running at the same time share
// the B (weight) tile through L2 and each weight byte leaves HBM about once.
// The row count of each group is read from device memory (offsets and the
// M-tile prefix written by the dispatch), so no host synchronisation is
// needed.  Rows past a group's end are loaded (TMA zero-fills past the
// tensor) but masked in the epilogue.
//
// Every wait on an mbarrier is bounded (about 2 s of %globaltimer): on
// timeout the CTA raises an abort flag, records DEVERR_TIMEOUT, drains its
// outstanding copies and MMAs with bounded waits, frees TMEM and returns.
#include "moe_internal.cuh"

#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;   // MMA N (gate+up, or output columns of the down tile)
constexpr int BK = 64;    // 64 bf16 = 128 bytes = one swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_HALF_BYTES = 128 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + 2 * B_HALF_BYTES;
constexpr int STAGES_PAIR = 6;                            // CTA pair: A + one B half per CTA
constexpr int STAGE_BYTES_PAIR = A_BYTES + B_HALF_BYTES;
constexpr int NUM_THREADS = 192;
// Per epilogue warp, a 32 x 32 fp32 staging tile (4 KB, 1024-byte aligned) in
// the 128-byte-swizzle layout: row r at byte r * 128, its 16-byte chunk j at
// chunk j ^ (r & 7).  Row-wise writes and 4-rows-at-a-time reads are both
// conflict-free, and it is the layout a TMA store of a 32 x 32 fp32 box reads.
constexpr int kStgTile = 32 * 32 * 4;
constexpr size_t kStgBytes = 4 * kStgTile + 1024;  // + alignment slack
constexpr int TMEM_COLS = 512;
constexpr unsigned long long kTimeoutNs = 2000000000ull;

enum Epi { EPI_SWIGLU = 0, EPI_COMBINE = 1, EPI_STORE = 2 };

struct TcArgs {
    const int32_t* mt_start;  // [E+1] routed M-tile prefix
    const int32_t* offsets;   // [E+1] routed row offsets
    int E;
    int nt_r, nkb_r;          // routed: output-column tiles, K blocks
    int b_rows_r;             // routed B rows per expert (d_f for gate/up, d for down)
    int M_sh, nt_sh, nkb_sh;  // shared group (M_sh = 0: none)
    int n_valid_r, n_valid_sh;  // valid output columns
    void* out;                // SWIGLU: h bf16 [rows, ld_out]; STORE: H fp32 [rows, ld_out]
    void* out_sh;             // SWIGLU: h_sh bf16 [N, ld_out_sh]
    int ld_out, ld_out_sh;
    const int32_t* slot_token;
    const float* slot_w;
    float* Y;
    int ldY;
    int max_rows;             // rows of the routed A / output buffers (N k)
    int n_tokens;             // N
    int has_routed;           // 0: only the second (dense) segment runs
    float* zero_ptr;          // optional fp32 buffer the epilogue warps zero first
    int64_t zero_n4;          // its size in float4
    int ks;                   // K splits per output tile (partial sums reduced with red.add)
    const int32_t* grp_nkb;   // [E] K blocks of each routed group (null: nkb_r for all; ks must be 1)
    int b_mn;                 // 1: B is read MN-major (single-CTA store mode): per K block,
                              //    four 64 x 64 boxes of a [K rows, N cols] matrix
    int nkb_split;            // b_mn: K blocks >= nkb_split take A from mA_h and B from mB1
                              //    (a second K segment); 0: one segment
    int tma_out;              // store epilogue without K split: warp slabs whose 32 rows
                              //    are all valid leave by TMA store (tensor map mOut)
    int a_h64;                // single CTA: mA_h / mA_sh_h hold the A rows in 64-row boxes,
                              //    so tiles of at most 64 rows run as M=64 MMAs
    int swap_tails;           // CTA pairs: the rows of each group past its last 256-row
                              //    boundary, when at most 128, run as one weight-stationary
                              //    tile (see group_tail_rows); the M-tile prefix is then
                              //    built from offsets inside the kernel, and mOut holds the
                              //    A rows in 16-row boxes
    unsigned long long* counters;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: true when the phase with `parity` completed; false on abort
// (flag raised elsewhere) or timeout (raises the flag and records it).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long* counters,
                                             unsigned long long limit = kTimeoutNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit) {
                *abort_flag = 1;
                atomicOr(counters + CNT_DEVICE_ERROR, (unsigned long long)DEVERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Warp-collective bounded wait: every lane returns the same result, so the
// .sync.aligned tcgen05 loads that follow are executed by the whole warp.
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  unsigned long long* counters) {
    const uint32_t a = smem_u32(bar);
    const int lane = threadIdx.x & 31;
    unsigned long long t0 = 0;
    if (lane == 0) t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        const bool done = mbar_try_wait(a, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 63u) == 63u) {
            int stop = 0;
            if (lane == 0) {
                if (*abort_flag) {
                    stop = 1;
                } else if (global_timer_ns() - t0 > kTimeoutNs) {
                    *abort_flag = 1;
                    atomicOr(counters + CNT_DEVICE_ERROR, (unsigned long long)DEVERR_TIMEOUT);
                    stop = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// TMA store of one box from shared memory (bulk async-group completion)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// this thread's bulk stores have read their shared-memory source
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// this thread's bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// orders this thread's shared-memory writes before reads by the async proxy (TMA)
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle,
// 8-row core groups 1024 bytes apart (SBO), leading offset 16 bytes (unused
// by the swizzled K-major layout), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Shared-memory matrix descriptor of an MN-major operand, 128-byte swizzle:
// each 128-byte row holds 64 consecutive N (or M) elements of one K index,
// 8-row atoms of 1024 bytes follow each other along K (SBO = 1024 bytes), and
// the next 64 N elements start 8 KB further (LBO = 8 KB: one 64 x 64 box).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(8192 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// M = 64 (one CTA): accumulator row i in TMEM lane (i mod 16) + 32 (i / 16),
// lanes 0-15 of each 32-lane quarter; the other lanes are not written
constexpr uint32_t kIdescM64 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                               ((uint32_t)(64 >> 4) << 24);

__device__ __forceinline__ void umma_bf16_id(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// the same MMA with B MN-major (instruction descriptor bit 16)
constexpr uint32_t kIdescBmn = kIdesc | (1u << 16);

__device__ __forceinline__ void umma_bf16_bmn(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdescBmn), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// --- CTA-pair (cta_group::2) forms -------------------------------------------
// M = 256 across the pair (128 A rows in each CTA), N = 256 (128 B rows in each).
constexpr uint32_t kIdescPair = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(256 >> 4) << 24);
// M = 128 across the pair (64 A rows in each CTA), N = 256: for tiles of at
// most 128 rows.  Each CTA's accumulator then holds its 64 rows twice as
// wide: TMEM lanes 0-63 carry MMA columns 0-127, lanes 64-127 columns
// 128-255, both at TMEM columns 0-127.
constexpr uint32_t kIdescPairHalf = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in the peer CTA of the pair (each CTA fetches only
// the tiles it stores itself).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on the same barrier in both CTAs of the pair once the MMAs issued
// so far complete
__device__ __forceinline__ void umma_commit_pair_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives on; the wait gives up after limit_ns and records DEVERR_TIMEOUT.
__global__ void wait_selftest_kernel(unsigned long long* counters, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        wait_bounded(&bar, 0u, &abort_flag, counters, limit_ns);
    }
}

// ---------------------------------------------------------------------------
// Tile schedule
// ---------------------------------------------------------------------------
struct Tile {
    int shared;     // 0 routed, 1 shared expert
    int g;          // expert
    int a_row;      // first row of the tile's rows in its A matrix
    int rows;       // valid rows of the tile (<= TM)
    int n_tile;     // output-column tile
    int kb0, kb1;   // K blocks [kb0, kb1) of this tile
    int swap;       // 1: weight-stationary tail tile (CTA pairs with swap_tails)
    int m64;        // 1: single-CTA tile of at most 64 rows, run as an M=64 MMA
};

struct SchedSmem {
    int32_t mt[kMaxExperts + 1];
    int32_t off[kMaxExperts + 1];
};

// Weight-stationary tail tiles (CTA pairs, swap_tails).  A pair tile of at
// most 128 rows costs as long as a full one: an M=128 pair MMA uses half of
// each SM's tensor datapath.  So the rows of a group of L rows past its last
// 256-row boundary, when there are at most 128 of them, run as one tile with
// the operands swapped: the 256 weight rows of the output-column tile on the
// MMA's M side (128 per CTA, the same boxes a row tile loads as B) and the
// tail's tokens on its N side, rounded up to 32, so the tile costs in
// proportion to its rows.  The group's other rows run in 256-row tiles (the
// last of 129..255 rows).
__device__ __forceinline__ int group_tail_rows(int L) {
    const int rem = L > 0 ? (L & 255) : 0;
    return rem <= 128 ? rem : 0;
}

__device__ __forceinline__ int group_swap_tiles(int L) {
    const int tail = group_tail_rows(L);
    return ((max(L, 0) - tail + 255) >> 8) + (tail > 0 ? 1 : 0);
}

// MMA N of a tail tile: its rows rounded up to 32 (each CTA loads half)
__device__ __forceinline__ int swap_tile_n(int rows) {
    const int n = (rows + 31) / 32 * 32;
    return n < 32 ? 32 : (n > 128 ? 128 : n);
}

// kind::f16, D fp32, A and B bf16 K-major, M = 256 across the pair; N per tile
constexpr uint32_t kIdescSwapBase = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 4) << 24);

// TM: rows of one output tile (128 for one CTA, 256 for a CTA pair); the
// M-tile prefix in `s.mt` counts tiles of TM rows.
template <int TM>
__device__ __forceinline__ bool decode_tile(int t_in, const SchedSmem& s, const TcArgs& a,
                                            int routed_tiles, Tile& ti) {
    // K split fastest: consecutive tiles are the K slices of one output tile
    const int kq = t_in % a.ks;
    const int t = t_in / a.ks;
    if (t < routed_tiles) {
        const int q = t / a.nt_r;
        // last group g with mt[g] <= q (non-empty, since mt[g+1] > q)
        int lo = 0, hi = a.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s.mt[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int g = lo;
        const int mtiles = s.mt[g + 1] - s.mt[g];
        ti.shared = 0;
        ti.g = g;
        ti.kb0 = (int)((int64_t)kq * a.nkb_r / a.ks);
        ti.kb1 = (int)((int64_t)(kq + 1) * a.nkb_r / a.ks);
        if (a.grp_nkb) {  // a group's own K extent (at least one block: its tiles are always written)
            const int nk = min(max(a.grp_nkb[g], 1), a.nkb_r);
            if (ti.kb1 > nk) ti.kb1 = nk;
        }
        if (mtiles <= 0) {  // inconsistent prefix (caller-supplied offsets): no rows
            ti.n_tile = 0;
            ti.a_row = 0;
            ti.rows = 0;
            ti.swap = 0;
            ti.m64 = 0;
            return true;
        }
        const int local = t - s.mt[g] * a.nt_r;
        const int m_tile = local % mtiles;
        ti.n_tile = local / mtiles;
        ti.a_row = s.off[g] + m_tile * TM;
        int r_end = s.off[g + 1];
        ti.swap = 0;
        if (a.swap_tails) {
            const int tail = group_tail_rows(r_end - s.off[g]);
            if (tail > 0 && ti.a_row >= r_end - tail) {  // the group's last tile
                ti.swap = 1;
                ti.a_row = r_end - tail;
            } else {
                r_end -= tail;
            }
        }
        // rows of this tile inside the group and inside the row buffer
        ti.rows = max(0, min(min(TM, r_end - ti.a_row), a.max_rows - ti.a_row));
        if (ti.a_row < 0) ti.rows = 0;
        ti.m64 = (TM == 128 && a.a_h64 && !a.b_mn && ti.rows > 0 && ti.rows <= 64) ? 1 : 0;
        return true;
    }
    const int mt_sh = (a.M_sh + TM - 1) / TM;
    const int local = t - routed_tiles;
    if (a.M_sh <= 0 || local >= mt_sh * a.nt_sh) return false;
    ti.shared = 1;
    ti.swap = 0;
    ti.g = 0;
    ti.n_tile = local / mt_sh;
    ti.a_row = (local % mt_sh) * TM;
    ti.rows = min(TM, a.M_sh - ti.a_row);
    ti.m64 = (TM == 128 && a.a_h64 && !a.b_mn && ti.rows > 0 && ti.rows <= 64) ? 1 : 0;
    ti.kb0 = (int)((int64_t)kq * a.nkb_sh / a.ks);
    ti.kb1 = (int)((int64_t)(kq + 1) * a.nkb_sh / a.ks);
    return true;
}

__device__ __forceinline__ int warp_incl_sum(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Epilogue of one accumulator segment.  The calling thread owns one output
// row (`row_ok`, global row `grow`) in TMEM lane `t_row`'s quarter; the
// segment spans TMEM columns [cb, cb + width) of that lane, which hold the
// output columns starting at `ob`.
//   SwiGLU: the gate value of output column ob + c sits at TMEM column
//           cb + c and the up value at cb + up_off + c (c < width).
//   fp32:   TMEM column cb + c is output column ob + c.
template <int EPI>
__device__ __forceinline__ void epilogue_segment(const TcArgs& a, const Tile& ti, uint32_t t_row,
                                                 int lane, bool row_ok, int grow, int cb, int ob,
                                                 int width, int up_off, float* stg, const CUtensorMap* mOut) {
    const int n_valid = ti.shared ? a.n_valid_sh : a.n_valid_r;
    if (EPI == EPI_SWIGLU) {
        const int ld = ti.shared ? a.ld_out_sh : a.ld_out;
        __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(ti.shared ? a.out_sh : a.out);
#pragma unroll 1
        for (int c = 0; c < width; c += 32) {
            uint32_t g[32], u[32];
            tmem_ld32(t_row + (uint32_t)(cb + c), g);
            tmem_ld32(t_row + (uint32_t)(cb + up_off + c), u);
            tmem_ld_wait();
            const int col0 = ob + c;
            if (row_ok) {
                uint4* dst = reinterpret_cast<uint4*>(outp + (int64_t)grow * ld + col0);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    if (col0 + v * 8 < n_valid) {
                        uint4 pk;
                        float h[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            h[j] = silu_f(__uint_as_float(g[v * 8 + j])) * __uint_as_float(u[v * 8 + j]);
                        pk.x = pack_bf16(h[0], h[1]);
                        pk.y = pack_bf16(h[2], h[3]);
                        pk.z = pack_bf16(h[4], h[5]);
                        pk.w = pack_bf16(h[6], h[7]);
                        dst[v] = pk;
                    }
                }
            }
        }
    } else {
        // fp32 rows (combine into Y, or plain stores), 32 columns at a time
        // through this warp's swizzled staging tile: each lane writes its row;
        // then one TMA store takes the 32 x 32 box (store epilogue, every row
        // of the warp's slab valid), or each warp instruction covers 4 rows x
        // 128 contiguous bytes (8 lanes per row) instead of 32 rows x 16 bytes
        float wgt = 1.f;
        long long dst_off = -1;  // element offset of this row in the destination, -1: none
        float* dst_base = EPI == EPI_COMBINE ? a.Y : static_cast<float*>(a.out);
        if (row_ok) {
            if (EPI == EPI_COMBINE) {
                int tok;
                if (ti.shared) {
                    tok = grow;
                } else {
                    tok = a.slot_token[grow];
                    wgt = a.slot_w[grow];
                }
                if (tok >= 0 && tok < a.n_tokens) dst_off = (long long)tok * a.ldY;
            } else {
                dst_off = (long long)grow * a.ld_out;
            }
        }
        const bool reduce = EPI == EPI_COMBINE || a.ks > 1;
        const bool tma_path = EPI == EPI_STORE && !reduce && a.tma_out;
        const bool use_tma = tma_path && __all_sync(0xffffffffu, dst_off >= 0);
        const int row0 = __shfl_sync(0xffffffffu, grow, 0);
        uint8_t* sbuf = reinterpret_cast<uint8_t*>(stg);
        const uint32_t sbuf_u = smem_u32(sbuf);
        const int jj = lane & 7;
#pragma unroll 1
        for (int c = 0; c < width; c += 32) {
            uint32_t v[32];
            tmem_ld32(t_row + (uint32_t)(cb + c), v);
            tmem_ld_wait();
            if (tma_path) {  // the last TMA store from the tile has read it
                if (lane == 0) bulk_wait_read();
                __syncwarp();
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(sbuf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                    make_float4(__uint_as_float(v[4 * q]) * wgt, __uint_as_float(v[4 * q + 1]) * wgt,
                                __uint_as_float(v[4 * q + 2]) * wgt, __uint_as_float(v[4 * q + 3]) * wgt);
            const int col0 = ob + c;
            if (use_tma) {
                fence_proxy_async_smem();
                __syncwarp();
                // columns past n_valid are outside the tensor map and not written
                if (lane == 0 && col0 < n_valid) tma_store_2d(mOut, sbuf_u, col0, row0);
                continue;
            }
            __syncwarp();
            const int cg = jj * 4;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rr = i * 4 + (lane >> 3);
                const long long off = __shfl_sync(0xffffffffu, dst_off, rr);
                if (off >= 0 && col0 + cg < n_valid) {
                    const float4 val =
                        *reinterpret_cast<const float4*>(sbuf + rr * 128 + ((jj ^ (rr & 7)) << 4));
                    float* p = dst_base + off + col0 + cg;
                    if (reduce) red_add_v4(p, val.x, val.y, val.z, val.w);
                    else *reinterpret_cast<float4*>(p) = val;
                }
            }
            __syncwarp();
        }
    }
}

// --- tail tiles (CTA pairs): TMEM lane = weight row, column = token --------
// Exchange handshake of the two epilogue warps of a gate/up column group: all
// 64 threads arrive on the group's mbarrier, then wait (bounded) for its
// phase; xk counts this warp's handshakes (both warps of a group make the same
// number).  A wait that gives up leaves through the abort path.
__device__ __forceinline__ bool xch_sync(uint64_t* bar, uint32_t& xk, volatile int* abort_flag,
                                         unsigned long long* counters) {
    __syncwarp();
    mbar_arrive(bar);
    const bool ok = warp_wait_bounded(bar, xk & 1u, abort_flag, counters);
    ++xk;
    return ok;
}

constexpr int kXchLd = 17;  // floats per lane row of the exchange buffers (conflict-free)

// Gate/up tail tile: CTA c holds gate rows of output columns
// j0 + 64 c .. + 63 in TMEM lanes 0-63 and the up rows of the same columns in
// lanes 64-127.  The gate and up warps of a column group (lane quarters 0/2
// and 1/3) trade half of each 32-token chunk through shared memory, and each
// writes h for 16 tokens: 32 lanes store 32 consecutive columns of a token.
__device__ __forceinline__ bool tail_epilogue_swiglu(const TcArgs& a, const Tile& ti, uint32_t t_row, int quarter,
                                                     int lane, uint32_t crank, float* xch, uint64_t* xbar,
                                                     uint32_t& xk, volatile int* abort_flag) {
    const int nt = swap_tile_n(ti.rows);
    const bool gate = quarter < 2;
    const int grp = quarter & 1;
    const int j = ti.n_tile * 128 + (int)crank * 64 + grp * 32 + lane;  // output column of this lane
    const bool col_ok = j < a.n_valid_r;
    __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(a.out);
    float* xg = xch + grp * (2 * 32 * kXchLd);  // gate of tokens 16-31 (from the gate warp)
    float* xu = xg + 32 * kXchLd;               // up of tokens 0-15 (from the up warp)
#pragma unroll 1
    for (int c0 = 0; c0 < nt; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(t_row + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (gate) xg[lane * kXchLd + i] = __uint_as_float(v[16 + i]);
            else xu[lane * kXchLd + i] = __uint_as_float(v[i]);
        }
        if (!xch_sync(&xbar[grp], xk, abort_flag, a.counters)) return false;
        const int tb = c0 + (gate ? 0 : 16);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float g = gate ? __uint_as_float(v[i]) : xg[lane * kXchLd + i];
            const float u = gate ? xu[lane * kXchLd + i] : __uint_as_float(v[16 + i]);
            const int tok = tb + i;
            if (col_ok && tok < ti.rows)
                outp[(int64_t)(ti.a_row + tok) * a.ld_out + j] = __float2bfloat16_rn(silu_f(g) * u);
        }
        // the exchange rows are free for the next chunk
        if (!xch_sync(&xbar[grp], xk, abort_flag, a.counters)) return false;
    }
    return true;
}

// Down + combine tail tile: CTA c holds output features n0 + 128 c .. + 127
// (lane quarter q: 32 of them), a column per token.  Each 32-token chunk is
// transposed through the warp's swizzled staging tile (row = token) and added
// into Y[token] with 16-byte red.add, 4 tokens x 128 bytes per instruction.
__device__ __forceinline__ void tail_epilogue_combine(const TcArgs& a, const Tile& ti, uint32_t t_row, int quarter,
                                                      int lane, uint32_t crank, float* stg) {
    const int nt = swap_tile_n(ti.rows);
    const int nf = ti.n_tile * BN + (int)crank * 128 + quarter * 32;  // first feature of this warp
    uint8_t* sbuf = reinterpret_cast<uint8_t*>(stg);
    const int jj = lane & 7;
#pragma unroll 1
    for (int c0 = 0; c0 < nt; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(t_row + (uint32_t)c0, v);
        tmem_ld_wait();
        // token and combine weight of column c0 + lane
        long long dst_off = -1;
        float wt = 0.f;
        const int tt = c0 + lane;
        if (tt < ti.rows) {
            const int row = ti.a_row + tt;
            if (row < a.max_rows) {
                const int tok = a.slot_token[row];
                wt = a.slot_w[row];
                if (tok >= 0 && tok < a.n_tokens) dst_off = (long long)tok * a.ldY;
            }
        }
        // staging row = token t, column = this lane's feature
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const float val = __uint_as_float(v[t]) * __shfl_sync(0xffffffffu, wt, t);
            *reinterpret_cast<float*>(sbuf + t * 128 + (((lane >> 2) ^ (t & 7)) << 4) + ((lane & 3) << 2)) = val;
        }
        __syncwarp();
        const int cg = jj * 4;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int rr = i * 4 + (lane >> 3);
            const long long off = __shfl_sync(0xffffffffu, dst_off, rr);
            if (off >= 0 && nf + cg < a.n_valid_r) {
                const float4 val = *reinterpret_cast<const float4*>(sbuf + rr * 128 + ((jj ^ (rr & 7)) << 4));
                red_add_v4(a.Y + off + nf + cg, val.x, val.y, val.z, val.w);
            }
        }
        __syncwarp();
    }
}

// PAIR = false: one CTA computes a 128 x 256 tile (A 128 rows, B 256 rows:
//   4 stages of 48 KB).
// PAIR = true: a cluster of two CTAs computes a 256 x 256 tile with
//   cta_group::2 MMAs issued by the leader (cluster rank 0): each CTA loads
//   its 128 A rows and its 128-row half of B (6 stages of 32 KB), the
//   leader's full barrier counts both CTAs' bytes, and the leader's commits
//   arrive on the empty / accumulator-full barriers of both CTAs.  Each CTA
//   drains its own TMEM rows; the leader's accumulator-empty barrier counts
//   the epilogue warps of both CTAs.
template <int EPI, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_grouped_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
                      const __grid_constant__ CUtensorMap mB1,
                      const __grid_constant__ CUtensorMap mA_sh,
                      const __grid_constant__ CUtensorMap mB0_sh,
                      const __grid_constant__ CUtensorMap mB1_sh,
                      const __grid_constant__ CUtensorMap mA_h,
                      const __grid_constant__ CUtensorMap mA_sh_h,
                      const __grid_constant__ CUtensorMap mOut, const TcArgs a) {
    constexpr int NST = PAIR ? STAGES_PAIR : STAGES;
    constexpr int SBYTES = PAIR ? STAGE_BYTES_PAIR : STAGE_BYTES;
    constexpr int TM = PAIR ? 256 : 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned stage buffers (the 128-byte swizzle atom spans 8 rows)
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * SBYTES);
    uint64_t* empty = full + NST;
    uint64_t* tfull = empty + NST;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint64_t* xbar = done + 1;  // [2] tail-tile gate/up exchange handshakes (CTA pairs)
    uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(xbar + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_s + 1);
    SchedSmem* sched = reinterpret_cast<SchedSmem*>(smem + NST * SBYTES + 256);
    // per-epilogue-warp staging tiles (kStgTile bytes each, 1024-byte aligned)
    float* stg_all = reinterpret_cast<float*>(
        (reinterpret_cast<uintptr_t>(sched) + sizeof(SchedSmem) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = crank == 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // tile-processing unit
    const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    const bool swap_tails = PAIR && a.swap_tails;
    if (a.has_routed) {
        for (int i = threadIdx.x; i <= a.E; i += NUM_THREADS) {
            if (!swap_tails) sched->mt[i] = a.mt_start[i];
            sched->off[i] = a.offsets[i];
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], PAIR ? 8 : 4);  // one arrival per epilogue warp (of both CTAs)
        }
        mbar_init(done, 1);
        mbar_init(&xbar[0], 64);  // the two epilogue warps of a column group
        mbar_init(&xbar[1], 64);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        if (PAIR) tmem_alloc_pair(tmem_base_s, TMEM_COLS);
        else tmem_alloc(tmem_base_s, TMEM_COLS);
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mA);
        tma_prefetch_desc(&mB0);
        tma_prefetch_desc(&mB1);
        if (a.M_sh > 0) {
            tma_prefetch_desc(&mA_sh);
            tma_prefetch_desc(&mB0_sh);
            tma_prefetch_desc(&mB1_sh);
        }
        if (PAIR) {
            tma_prefetch_desc(&mA_h);
            if (a.M_sh > 0) tma_prefetch_desc(&mA_sh_h);
        }
    }
    tc_fence_before();
    if (PAIR) cluster_sync_all();  // the peer's barriers exist before any remote arrival
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_s;
    if (a.has_routed && swap_tails) {
        // M-tile prefix with tail tiles, from the row offsets (both CTAs of a
        // pair compute the same one)
        if (warp == 2) {
            int carry = 0;
            for (int base = 0; base < a.E; base += 32) {
                const int g = base + lane;
                const int c = g < a.E ? group_swap_tiles(sched->off[g + 1] - sched->off[g]) : 0;
                const int v = warp_incl_sum(c, lane);
                if (g < a.E) sched->mt[g] = carry + v - c;
                carry += __shfl_sync(0xffffffffu, v, 31);
            }
            if (lane == 0) sched->mt[a.E] = carry;
        }
        __syncthreads();
    }

    const int routed_tiles = a.has_routed ? sched->mt[a.E] * a.nt_r : 0;
    const int total_tiles =
        (routed_tiles + (a.M_sh > 0 ? ((a.M_sh + TM - 1) / TM) * a.nt_sh : 0)) * a.ks;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[NST];
            for (int s = 0; s < NST; ++s) issued_parity[s] = -1;
            bool ok = true;
            for (int t = unit; t < total_tiles && ok; t += n_units) {
                Tile ti;
                decode_tile<TM>(t, *sched, a, routed_tiles, ti);
                // pair tiles of at most 128 rows load 64 A rows per CTA
                const bool half = PAIR && ti.rows <= 128;
                const CUtensorMap* pa = ti.shared ? (half ? &mA_sh_h : &mA_sh) : (half ? &mA_h : &mA);
                const CUtensorMap* pb0 = ti.shared ? &mB0_sh : &mB0;
                const CUtensorMap* pb1 = ti.shared ? &mB1_sh : &mB1;
                int b_row0, b_row1;
                if (EPI == EPI_SWIGLU) {  // gate rows and up rows of the same 128 columns
                    b_row0 = (ti.shared ? 0 : ti.g * a.b_rows_r) + ti.n_tile * 128;
                    b_row1 = b_row0;
                } else {                  // two 128-column halves of a 256-column tile
                    b_row0 = (ti.shared ? 0 : ti.g * a.b_rows_r) + ti.n_tile * 256;
                    b_row1 = b_row0 + 128;
                }
                const int a_row = ti.a_row + (PAIR ? (int)crank * (half ? 64 : 128) : 0);
                const uint32_t a_bytes = half ? A_BYTES / 2 : A_BYTES;
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.counters)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = stage_base + stage * SBYTES;
                    uint8_t* sb = sa + A_BYTES;
                    if (PAIR && ti.swap) {
                        // tail tile: this CTA's 128 weight rows (the row tile's B
                        // boxes) as A, half of the tail's token rows (16-row
                        // boxes; rows past the tail only feed unused columns) as B
                        const uint32_t fb = map_shared_rank(smem_u32(&full[stage]), 0);
                        const int hrows = swap_tile_n(ti.rows) / 2;
                        if (leader) mbar_expect_tx(&full[stage], 2u * (uint32_t)(A_BYTES + hrows * BK * 2));
                        if (EPI == EPI_SWIGLU) {
                            tma_load_2d_pair(sa, pb0, fb, kb * BK, b_row0 + (int)crank * 64);
                            tma_load_2d_pair(sa + A_BYTES / 2, pb1, fb, kb * BK, b_row0 + (int)crank * 64);
                        } else {
                            tma_load_2d_pair(sa, crank == 0 ? pb0 : pb1, fb, kb * BK, crank == 0 ? b_row0 : b_row1);
                        }
                        const int x_row = ti.a_row + (int)crank * hrows;
                        for (int r16 = 0; r16 < hrows; r16 += 16)
                            tma_load_2d_pair(sb + r16 * BK * 2, &mOut, fb, kb * BK, x_row + r16);
                    } else if (PAIR) {
                        // both CTAs' bytes complete on the leader's full barrier
                        const uint32_t fb = map_shared_rank(smem_u32(&full[stage]), 0);
                        if (leader) mbar_expect_tx(&full[stage], 2 * (a_bytes + B_HALF_BYTES));
                        tma_load_2d_pair(sa, pa, fb, kb * BK, a_row);
                        if (EPI == EPI_SWIGLU) {
                            // this CTA's B half: 64 gate rows, then the 64 up
                            // rows of the same output columns
                            const int br = b_row0 + (int)crank * 64;
                            tma_load_2d_pair(sb, pb0, fb, kb * BK, br);
                            tma_load_2d_pair(sb + B_HALF_BYTES / 2, pb1, fb, kb * BK, br);
                        } else if (crank == 0) {
                            tma_load_2d_pair(sb, pb0, fb, kb * BK, b_row0);
                        } else {
                            tma_load_2d_pair(sb, pb1, fb, kb * BK, b_row1);
                        }
                    } else if (a.b_mn) {
                        // B MN-major: rows of the group's [K, N] matrix; a second
                        // K segment (nkb_split) takes A from mA_h and B from mB1
                        const bool seg1 = a.nkb_split > 0 && kb >= a.nkb_split;
                        const int kbs = seg1 ? kb - a.nkb_split : kb;
                        const CUtensorMap* pbm = seg1 ? &mB1 : &mB0;
                        const int brow = ti.g * a.b_rows_r + kbs * BK;
                        mbar_expect_tx(&full[stage], SBYTES);
                        tma_load_2d(sa, seg1 ? &mA_h : pa, &full[stage], kbs * BK, a_row);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_2d(sb + c * (B_HALF_BYTES / 2), pbm, &full[stage], ti.n_tile * 256 + c * BK,
                                        brow);
                    } else if (ti.m64) {
                        // at most 64 rows: the first 64 A rows of the stage (an M=64 MMA)
                        mbar_expect_tx(&full[stage], SBYTES - A_BYTES / 2);
                        tma_load_2d(sa, ti.shared ? &mA_sh_h : &mA_h, &full[stage], kb * BK, a_row);
                        tma_load_2d(sb, pb0, &full[stage], kb * BK, b_row0);
                        tma_load_2d(sb + B_HALF_BYTES, pb1, &full[stage], kb * BK, b_row1);
                    } else {
                        mbar_expect_tx(&full[stage], SBYTES);
                        tma_load_2d(sa, pa, &full[stage], kb * BK, a_row);
                        tma_load_2d(sb, pb0, &full[stage], kb * BK, b_row0);
                        tma_load_2d(sb + B_HALF_BYTES, pb1, &full[stage], kb * BK, b_row1);
                    }
                    issued_parity[stage] = (int)phase;
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag && (!PAIR || leader)) {
                // drain copies still in flight into shared memory
                for (int s = 0; s < NST; ++s)
                    if (issued_parity[s] >= 0)
                        wait_bounded(&full[s], (uint32_t)issued_parity[s], abort_flag, a.counters,
                                     kTimeoutNs / 4);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && (!PAIR || leader)) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = unit; t < total_tiles && ok; t += n_units) {
                Tile ti;
                decode_tile<TM>(t, *sched, a, routed_tiles, ti);
                const uint32_t idesc_pair =
                    ti.swap ? (kIdescSwapBase | ((uint32_t)(swap_tile_n(ti.rows) >> 3) << 17))
                            : (ti.rows <= 128 ? kIdescPairHalf : kIdescPair);
                if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, a.counters)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!wait_bounded(&full[stage], phase, abort_flag, a.counters)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage_base + stage * SBYTES);
                    const uint32_t sb = sa + A_BYTES;
                    const uint64_t ad = smem_desc_sw128(sa);
                    if (!PAIR && a.b_mn) {
                        // B MN-major: 16 K indices are 16 rows of 128 bytes (2 KB)
                        const uint64_t bd = smem_desc_mn_sw128(sb);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16_bmn(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 128),
                                          (kb > ti.kb0 || kk > 0) ? 1u : 0u);
                    } else {
                        const uint64_t bd = smem_desc_sw128(sb);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            // advance 16 elements (32 bytes) along K inside the swizzled row
                            const uint32_t accum = (kb > ti.kb0 || kk > 0) ? 1u : 0u;
                            if (PAIR)
                                umma_bf16_pair(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc_pair,
                                               accum);
                            else
                                umma_bf16_id(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2),
                                             ti.m64 ? kIdescM64 : kIdesc, accum);
                        }
                    }
                    if (PAIR) umma_commit_pair_both(&empty[stage]);
                    else umma_commit(&empty[stage]);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (PAIR) umma_commit_pair_both(&tfull[acc]);
                else umma_commit(&tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // all MMAs issued by this thread have completed once `done` fires
            if (PAIR) umma_commit_pair_local(done);
            else umma_commit(done);
            wait_bounded(done, 0, abort_flag, a.counters, kTimeoutNs / 4);
        }
    } else {
        // epilogue warps 2..5: TMEM lane quarter = warp % 4
        if (a.zero_ptr) {
            // zero this CTA's share of the combine output while the first
            // accumulator is being computed (the down projection adds into it)
            const int64_t per = (a.zero_n4 + gridDim.x - 1) / gridDim.x;
            const int64_t lo = per * blockIdx.x;
            const int64_t hi = min64(a.zero_n4, lo + per);
            float4* z = reinterpret_cast<float4*>(a.zero_ptr);
            for (int64_t i = lo + (threadIdx.x - 64); i < hi; i += 128) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        float* stg = stg_all + (warp - 2) * (kStgTile / 4);
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t xk = 0;  // tail-tile exchange handshakes of this warp
        for (int t = unit; t < total_tiles; t += n_units) {
            Tile ti;
            decode_tile<TM>(t, *sched, a, routed_tiles, ti);
            if (!warp_wait_bounded(&tfull[acc], acc_phase, abort_flag, a.counters)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            if (PAIR && ti.swap) {
                if (EPI == EPI_SWIGLU) {
                    if (!tail_epilogue_swiglu(a, ti, t_row, quarter, lane, crank, stg_all, xbar, xk, abort_flag))
                        break;
                } else if (EPI == EPI_COMBINE) {
                    tail_epilogue_combine(a, ti, t_row, quarter, lane, crank, stg);
                }
            } else if (!PAIR) {
                // lane r = row r (M=64 tiles: lanes 0-15 of quarter q hold rows
                // 16 q .. 16 q + 15); gate/up: gate columns 0-127, up 128-255
                const int rr = ti.m64 ? (lane < 16 ? quarter * 16 + lane : TM) : r;
                const bool ok = rr < ti.rows;
                if (EPI == EPI_SWIGLU)
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + rr, 0, ti.n_tile * 128, 128, 128, stg, &mOut);
                else
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + rr, 0, ti.n_tile * BN, BN, 0, stg, &mOut);
            } else if (ti.rows > 128) {
                // 256-row tile: lane r = row crank * 128 + r, all 256 columns
                const int lr = (int)crank * 128 + r;
                const bool ok = lr < ti.rows;
                if (EPI == EPI_SWIGLU) {
                    // each CTA's B half is 64 gate rows then 64 up rows
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + lr, 0, ti.n_tile * 128, 64, 64, stg, &mOut);
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + lr, 128, ti.n_tile * 128 + 64, 64,
                                          64, stg, &mOut);
                } else {
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + lr, 0, ti.n_tile * BN, BN, 0, stg, &mOut);
                }
            } else {
                // 128-row tile (64 rows per CTA): lanes 0-63 hold the first
                // 128 MMA columns of rows 0-63, lanes 64-127 the last 128
                const int lr = (int)crank * 64 + (quarter & 1) * 32 + lane;
                const int hf = quarter >> 1;
                const bool ok = lr < ti.rows;
                if (EPI == EPI_SWIGLU)
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + lr, 0, ti.n_tile * 128 + hf * 64, 64,
                                          64, stg, &mOut);
                else
                    epilogue_segment<EPI>(a, ti, t_row, lane, ok, ti.a_row + lr, 0, ti.n_tile * BN + hf * 128, 128,
                                          0, stg, &mOut);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_cluster(map_shared_rank(smem_u32(&tempty[acc]), 0));
                else mbar_arrive(&tempty[acc]);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        // this warp's TMA stores are complete before its shared memory goes away
        if (EPI == EPI_STORE && a.tma_out && lane == 0) bulk_wait_all();
    }

    __syncwarp();
    if (PAIR && *abort_flag) {
        // copies of the peer CTA complete on the leader's barriers: give any
        // still in flight time to land before the pair leaves
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    tc_fence_before();
    if (PAIR) cluster_sync_all();  // the leader's MMAs into the peer's TMEM are complete
    else __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 row-major matrix [rows, cols] (row stride ld elements, default
// cols) read in boxes of box_rows rows x 64 columns
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows = 128,
              uint64_t ld = 0) {
    auto enc = get_encode();
    if (!enc || rows == 0 || cols == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(ld ? ld : cols) * 2};
    cuuint32_t box[2] = {BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// fp32 output [rows, cols] (row stride ld elements) written by TMA stores of
// 32 x 32 boxes from the epilogue's swizzled staging tiles; false (plain
// stores) when the address or the stride is not 16-byte aligned
bool make_map_out(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld) {
    auto enc = get_encode();
    if (!enc || !ptr || rows == 0 || cols == 0 || (reinterpret_cast<uintptr_t>(ptr) & 15) || (ld * 4) % 16)
        return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// the fp32 epilogues stage through shared memory, and on CTA pairs the tail
// tiles' SwiGLU epilogue trades values through the same area; the single-CTA
// SwiGLU epilogue needs none
constexpr size_t smem_bytes(int epi, bool pair) {
    return 1024 + (pair ? (size_t)STAGES_PAIR * STAGE_BYTES_PAIR : (size_t)STAGES * STAGE_BYTES) + 256 +
           sizeof(SchedSmem) + (epi == EPI_SWIGLU && !pair ? 0 : kStgBytes);
}
static_assert(smem_bytes(EPI_SWIGLU, true) <= 232448 &&
                  smem_bytes(EPI_COMBINE, false) <= 232448 && smem_bytes(EPI_COMBINE, true) <= 232448 &&
                  smem_bytes(EPI_STORE, false) <= 232448 && smem_bytes(EPI_STORE, true) <= 232448,
              "shared memory per CTA");

// mA_h / mA_sh_h: the A matrices again in 64-row boxes (CTA-pair tiles of at
// most 128 rows); unused by single-CTA launches.
template <int EPI, bool PAIR>
cudaError_t launch_tc(const CUtensorMap& mA, const CUtensorMap& mB0, const CUtensorMap& mB1,
                      const CUtensorMap& mA_sh, const CUtensorMap& mB0_sh, const CUtensorMap& mB1_sh,
                      const CUtensorMap& mA_h, const CUtensorMap& mA_sh_h, const CUtensorMap& mOut,
                      const TcArgs& a, int64_t max_tiles, cudaStream_t st) {
    auto kern = tc_grouped_kernel<EPI, PAIR>;
    const size_t smem = smem_bytes(EPI, PAIR);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (!PAIR) {
        const int grid = (int)min64(max_tiles, num_sms());
        if (grid <= 0) return cudaSuccess;
        kern<<<grid, NUM_THREADS, smem, st>>>(mA, mB0, mB1, mA_sh, mB0_sh, mB1_sh, mA_h, mA_sh_h, mOut, a);
        return cudaGetLastError();
    }
    // clusters of two CTAs, one tile per cluster at a time
    const int pairs = (int)min64(max_tiles, num_sms() / 2);
    if (pairs <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mA, mB0, mB1, mA_sh, mB0_sh, mB1_sh, mA_h, mA_sh_h, mOut, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int64_t routed_mtile_bound(const moe_params& p, int tm) {
    return (p.N * p.k + tm - 1) / tm + p.E_r;
}

// Expected routed M tiles: each expert gets about mu = N k / E_r rows (at most
// C); a group of r rows takes ceil(r / 128) tiles, about r / 128 + 1/2 on average.
double routed_mtile_estimate(const moe_params& p, int64_t C, int tm) {
    double mu = (double)p.N * p.k / p.E_r;
    if (mu > (double)C) mu = (double)C;
    if (mu <= 0) return 0;
    const double per = mu / tm + 0.5;
    return p.E_r * (per < 1.0 ? 1.0 : per);
}

// K splits for an output-tile count: only when the tiles fill less than one
// wave of SMs (splitting a multi-wave launch measured slower on the
// Mixtral-shaped down projection: the extra red.add traffic costs more than
// the last partial wave), minimise ceil(tiles * ks / SMs) / ks, keeping >= 8 K
// blocks per slice.
int choose_ksplit(double tiles, int nkb_min) {
    const int sms = num_sms();
    if (tiles >= sms) return 1;
    int best = 1;
    double best_cost = 1e30;
    for (int ks = 1; ks <= 8; ++ks) {
        if (ks > 1 && nkb_min / ks < 8) break;
        const double waves = ceil(tiles * ks / sms - 1e-9);
        const double cost = waves / ks;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = ks;
        }
    }
    return best;
}

}  // namespace

#ifndef MOE_TC_PAIR_MIN_ROWS
#define MOE_TC_PAIR_MIN_ROWS 768
#endif
#ifndef MOE_TC_SWAP_TAILS
#define MOE_TC_SWAP_TAILS 1
#endif
#ifndef MOE_TC_COMBINE_PAIR_MIN_ROWS
#define MOE_TC_COMBINE_PAIR_MIN_ROWS 384
#endif

int tc_tile_rows(const moe_params& p) {
    // CTA pairs (256-row tiles) when experts average enough rows to fill them
    const double mu = (double)p.N * p.k / p.E_r;
    return (p.dtype == MOE_BF16 && mu >= (double)MOE_TC_PAIR_MIN_ROWS) ? 256 : 128;
}

bool tc_swap_tails(const moe_params& p) { return MOE_TC_SWAP_TAILS && tc_tile_rows(p) == 256; }

cudaError_t launch_tc_gate_up(const moe_params& p, const void* x_perm, const void* x_shared,
                              const int32_t* offsets, const int32_t* mt_start,
                              const ExpertWeights& W, void* h, void* h_shared, float* Y_zero,
                              unsigned long long* counters, cudaStream_t st, int* status) {
    *status = MOE_OK;
    CUtensorMap mA, mB0, mB1, mA_sh, mB0_sh, mB1_sh, mA_h, mA_sh_h;
    const bool pair = tc_tile_rows(p) == 256;
    // CTA pairs: each CTA loads 64 gate rows and 64 up rows per 128 columns
    const uint32_t b_box = pair ? 64 : 128;
    const uint64_t rows = (uint64_t)(p.N * p.k);
    bool ok = make_map(&mA, x_perm, rows, p.d) && make_map(&mA_h, x_perm, rows, p.d, 64) &&
              make_map(&mB0, W.W_g, (uint64_t)p.E_r * p.d_f, p.d, b_box) &&
              make_map(&mB1, W.W_u, (uint64_t)p.E_r * p.d_f, p.d, b_box);
    const bool sh = p.d_f_shared > 0;
    if (ok && sh) {
        ok = make_map(&mA_sh, x_shared, (uint64_t)p.N, p.d) &&
             make_map(&mA_sh_h, x_shared, (uint64_t)p.N, p.d, 64) &&
             make_map(&mB0_sh, W.Ws_g, (uint64_t)p.d_f_shared, p.d, b_box) &&
             make_map(&mB1_sh, W.Ws_u, (uint64_t)p.d_f_shared, p.d, b_box);
    } else {
        mA_sh = mA;
        mA_sh_h = mA_h;
        mB0_sh = mB0;
        mB1_sh = mB1;
    }
    if (!ok) {
        *status = MOE_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    TcArgs a{};
    a.mt_start = mt_start;
    a.offsets = offsets;
    a.E = p.E_r;
    a.nt_r = (p.d_f + 127) / 128;
    a.nkb_r = (p.d + BK - 1) / BK;
    a.b_rows_r = p.d_f;
    a.M_sh = sh ? (int)p.N : 0;
    a.nt_sh = sh ? (p.d_f_shared + 127) / 128 : 0;
    a.nkb_sh = a.nkb_r;
    a.n_valid_r = p.d_f;
    a.n_valid_sh = p.d_f_shared;
    a.out = h;
    a.out_sh = h_shared;
    a.ld_out = p.d_f;
    a.ld_out_sh = p.d_f_shared;
    a.max_rows = (int)(p.N * p.k);
    a.n_tokens = (int)p.N;
    a.has_routed = 1;
    a.a_h64 = 1;
    a.ks = 1;  // the SwiGLU epilogue needs the whole K sum
    a.zero_ptr = Y_zero;
    a.zero_n4 = Y_zero ? p.N * (int64_t)p.d / 4 : 0;
    a.counters = counters;
    const int tm = pair ? 256 : 128;
    int64_t max_tiles =
        routed_mtile_bound(p, tm) * a.nt_r + (sh ? ((p.N + tm - 1) / tm) * a.nt_sh : 0);
    const int units = pair ? num_sms() / 2 : num_sms();
    if (Y_zero && max_tiles < units) max_tiles = units;  // every CTA zeroes a share
    if (pair) {
        // tail tiles read the gathered rows in 16-row boxes (the mOut slot)
        CUtensorMap mX16 = mA;
        if (tc_swap_tails(p)) {
            if (!make_map(&mX16, x_perm, rows, p.d, 16)) {
                *status = MOE_ERR_CUDA;
                return cudaErrorInvalidValue;
            }
            a.swap_tails = 1;
        }
        return launch_tc<EPI_SWIGLU, true>(mA, mB0, mB1, mA_sh, mB0_sh, mB1_sh, mA_h, mA_sh_h, mX16, a, max_tiles,
                                           st);
    }
    return launch_tc<EPI_SWIGLU, false>(mA, mB0, mB1, mA_sh, mB0_sh, mB1_sh, mA_h, mA_sh_h, mA, a, max_tiles,
                                        st);
}

cudaError_t launch_tc_down(const moe_params& p, int mode, int64_t C, const void* h,
                           const void* h_shared, const int32_t* offsets, const int32_t* mt_start,
                           const ExpertWeights& W, const int32_t* slot_token,
                           const float* slot_w, float* Y, float* H_out,
                           unsigned long long* counters, cudaStream_t st, int* status,
                           const int32_t* grp_nkb) {
    *status = MOE_OK;
    if (grp_nkb && mode != DOWN_STORE) return cudaErrorInvalidValue;
    CUtensorMap mA, mB0, mA_sh, mB0_sh, mA_h, mA_sh_h;
    const uint64_t rows = (uint64_t)(p.N * p.k);
    bool ok = make_map(&mA, h, rows, p.d_f) && make_map(&mA_h, h, rows, p.d_f, 64) &&
              make_map(&mB0, W.W_d, (uint64_t)p.E_r * p.d, p.d_f);
    const bool sh = p.d_f_shared > 0 && mode == DOWN_COMBINE;
    if (ok && sh) {
        ok = make_map(&mA_sh, h_shared, (uint64_t)p.N, p.d_f_shared) &&
             make_map(&mA_sh_h, h_shared, (uint64_t)p.N, p.d_f_shared, 64) &&
             make_map(&mB0_sh, W.Ws_d, (uint64_t)p.d, p.d_f_shared);
    } else {
        mA_sh = mA;
        mA_sh_h = mA_h;
        mB0_sh = mB0;
    }
    if (!ok) {
        *status = MOE_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    TcArgs a{};
    a.mt_start = mt_start;
    a.offsets = offsets;
    a.E = p.E_r;
    a.nt_r = (p.d + BN - 1) / BN;
    a.nkb_r = (p.d_f + BK - 1) / BK;
    a.b_rows_r = p.d;
    a.M_sh = sh ? (int)p.N : 0;
    a.nt_sh = sh ? a.nt_r : 0;
    a.nkb_sh = sh ? (p.d_f_shared + BK - 1) / BK : 0;
    a.n_valid_r = p.d;
    a.n_valid_sh = p.d;
    a.out = H_out;
    a.ld_out = p.d;
    a.slot_token = slot_token;
    a.slot_w = slot_w;
    a.Y = Y;
    a.ldY = p.d;
    a.max_rows = (int)(p.N * p.k);
    a.n_tokens = (int)p.N;
    a.has_routed = 1;
    a.a_h64 = 1;
    a.ks = 1;
    a.grp_nkb = grp_nkb;
    // the combine runs on CTA pairs with tail tiles also where the layer's row
    // tiles are 128 rows (its tile list comes from the offsets, not from the
    // dispatch's M-tile prefix): measured faster than single CTAs on layers of
    // 384..767 requests per expert, whose gate/up stays on single CTAs
    const bool combine_swap = mode == DOWN_COMBINE && MOE_TC_SWAP_TAILS && p.dtype == MOE_BF16 &&
                              (double)p.N * p.k >= (double)MOE_TC_COMBINE_PAIR_MIN_ROWS * p.E_r;
    const bool pair = tc_tile_rows(p) == 256 || combine_swap;
    const int tm = pair ? 256 : 128;
    if (mode == DOWN_COMBINE) {
        // the combine reduces with red.add into a zeroed Y, so K slices of one
        // output tile can run on different SMs: split K to fill the last wave
        const double tiles = routed_mtile_estimate(p, C, tm) * a.nt_r +
                             (sh ? (double)((p.N + tm - 1) / tm) * a.nt_sh : 0.0);
        a.ks = choose_ksplit(pair ? 2.0 * tiles : tiles, sh ? std::min(a.nkb_r, a.nkb_sh) : a.nkb_r);
    }
    a.counters = counters;
    int64_t max_tiles =
        (routed_mtile_bound(p, tm) * a.nt_r + (sh ? ((p.N + tm - 1) / tm) * a.nt_sh : 0)) * a.ks;
    if (mode == DOWN_COMBINE) {
        if (pair) {
            // tail tiles read the h rows in 16-row boxes (the mOut slot)
            CUtensorMap mX16 = mA;
            if (tc_swap_tails(p) || combine_swap) {
                if (!make_map(&mX16, h, rows, p.d_f, 16)) {
                    *status = MOE_ERR_CUDA;
                    return cudaErrorInvalidValue;
                }
                a.swap_tails = 1;
            }
            return launch_tc<EPI_COMBINE, true>(mA, mB0, mB0, mA_sh, mB0_sh, mB0_sh, mA_h, mA_sh_h, mX16, a,
                                                max_tiles, st);
        }
        return launch_tc<EPI_COMBINE, false>(mA, mB0, mB0, mA_sh, mB0_sh, mB0_sh, mA_h, mA_sh_h, mA, a, max_tiles,
                                             st);
    }
    // plain stores: whole 32-row slabs of the output leave by TMA store
    CUtensorMap mOut = mA;
    a.tma_out = (a.ks == 1 && make_map_out(&mOut, H_out, (uint64_t)a.max_rows, (uint64_t)a.n_valid_r,
                                           (uint64_t)a.ld_out))
                    ? 1
                    : 0;
    if (pair)
        return launch_tc<EPI_STORE, true>(mA, mB0, mB0, mA_sh, mB0_sh, mB0_sh, mA_h, mA_sh_h, mOut, a, max_tiles,
                                          st);
    return launch_tc<EPI_STORE, false>(mA, mB0, mB0, mA_sh, mB0_sh, mB0_sh, mA_h, mA_sh_h, mOut, a, max_tiles, st);
}

int tc_store_bmn_split(const moe_params& p, int64_t n_out, int64_t K, bool two_segments) {
    const int nkb = (int)((K + BK - 1) / BK) * (two_segments ? 2 : 1);
    const double tiles = (double)((p.N * p.k + 127) / 128 + p.E_r - 1) * (double)((n_out + BN - 1) / BN);
    return choose_ksplit(tiles, nkb);
}

cudaError_t launch_tc_store_bmn(const moe_params& p, int64_t n_out, int64_t K, const void* A0, int64_t ldA0,
                                const void* B0, const void* A1, int64_t ldA1, const void* B1,
                                const int32_t* offsets, const int32_t* mt_start128, float* out,
                                unsigned long long* counters, cudaStream_t st, int* status, bool split_k,
                                int* ks_out) {
    *status = MOE_OK;
    CUtensorMap mA, mA2, mB0, mB1;
    const uint64_t rows = (uint64_t)(p.N * p.k);
    const bool two = A1 && B1;
    bool ok = make_map(&mA, A0, rows, (uint64_t)K, 128, (uint64_t)ldA0) &&
              make_map(&mB0, B0, (uint64_t)p.E_r * K, (uint64_t)n_out, 64);
    if (ok && two)
        ok = make_map(&mA2, A1, rows, (uint64_t)K, 128, (uint64_t)ldA1) &&
             make_map(&mB1, B1, (uint64_t)p.E_r * K, (uint64_t)n_out, 64);
    if (!two) {
        mA2 = mA;
        mB1 = mB0;
    }
    if (!ok) {
        *status = MOE_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    const int nkb = (int)((K + BK - 1) / BK);
    TcArgs a{};
    a.mt_start = mt_start128;
    a.offsets = offsets;
    a.E = p.E_r;
    a.nt_r = (int)((n_out + BN - 1) / BN);
    a.nkb_r = two ? 2 * nkb : nkb;
    a.b_rows_r = (int)K;
    a.b_mn = 1;
    a.nkb_split = two ? nkb : 0;
    a.n_valid_r = (int)n_out;
    a.out = out;
    a.ld_out = (int)n_out;
    a.max_rows = (int)(p.N * p.k);
    a.n_tokens = (int)p.N;
    a.has_routed = 1;
    a.ks = split_k ? tc_store_bmn_split(p, n_out, K, two) : 1;
    if (ks_out) *ks_out = a.ks;
    a.counters = counters;
    const int64_t max_tiles = routed_mtile_bound(p, 128) * a.nt_r * a.ks;
    CUtensorMap mOut = mA;
    a.tma_out = (a.ks == 1 && make_map_out(&mOut, out, (uint64_t)a.max_rows, (uint64_t)n_out, (uint64_t)n_out))
                    ? 1
                    : 0;
    return launch_tc<EPI_STORE, false>(mA, mB0, mB1, mA, mB0, mB1, mA2, mA, mOut, a, max_tiles, st);
}

cudaError_t launch_tc_dense(int64_t M, int64_t Nc, int64_t K, const void* A, const void* B, float* out,
                            unsigned long long* counters, cudaStream_t st, int* status) {
    *status = MOE_OK;
    if (M <= 0 || Nc <= 0) return cudaSuccess;
    CUtensorMap mA, mB;
    if (!make_map(&mA, A, (uint64_t)M, (uint64_t)K) || !make_map(&mB, B, (uint64_t)Nc, (uint64_t)K)) {
        *status = MOE_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    TcArgs a{};
    a.E = 0;
    a.has_routed = 0;
    a.M_sh = (int)M;
    a.nt_sh = (int)((Nc + BN - 1) / BN);
    a.nkb_sh = (int)((K + BK - 1) / BK);
    a.n_valid_sh = (int)Nc;
    a.out = out;
    a.ld_out = (int)Nc;
    a.max_rows = (int)M;
    a.n_tokens = (int)M;
    const int64_t tiles = ((M + 127) / 128) * a.nt_sh;
    a.ks = choose_ksplit((double)tiles, a.nkb_sh);
    a.counters = counters;
    if (a.ks > 1) {  // K slices add into the output with red.add
        cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)M * (size_t)Nc, st);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mOut = mA;
    a.tma_out = (a.ks == 1 && make_map_out(&mOut, out, (uint64_t)M, (uint64_t)Nc, (uint64_t)Nc)) ? 1 : 0;
    return launch_tc<EPI_STORE, false>(mA, mB, mB, mA, mB, mB, mA, mA, mOut, a, tiles * a.ks, st);
}

cudaError_t launch_tc_logits(const moe_params& p, const void* x, const void* W_r, float* logits,
                             unsigned long long* counters, cudaStream_t st, int* status) {
    return launch_tc_dense(p.N, p.E_r, p.d, x, W_r, logits, counters, st, status);
}

cudaError_t launch_wait_selftest(unsigned long long* counters, unsigned long long limit_ns, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(counters, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
