// Paged GQA decode attention for B200 (sm_100a): the split kernel, the merge
// and the decode entry points of the C ABI (include/pkv.h).
//
// Method: "PersistentKV: Page-Aware Decode Scheduling for Long-Context LLM
// Serving on Commodity GPUs" (gist.science explainer), Technical summary >
// Methodology > 1 "Native block-table decode engine":
//   - GQA: the G = H_q / H_kv query heads of one KV head are handled by one
//     block, so every K/V byte is read from HBM once;
//   - layout: K/V pages are read through the block table in place, never
//     repacked into a contiguous tensor;
//   - sequence splitting: a row's token range is cut into disjoint chunks;
//     each chunk yields a partial online-softmax state (running max m,
//     denominator l, fp32 accumulator) and a merge combines them exactly;
//   - row-local bounds: chunk ranges come from each row's real length; an
//     empty chunk writes the neutral state (m = -inf, l = 0, acc = 0) and
//     reads nothing;
//   - compact work queue: a 1D grid over the non-empty (row, KV head, chunk)
//     items only.
//
// B200 design (the pages' kernels were written for an RTX 3060):
//   - one producer warp streams whole 16-token pages of K and V for one KV
//     head (4 KiB each at D = 128) with TMA tensor copies (one rank-5 copy per
//     page and tensor, four lanes issuing at once) into an NST-stage
//     shared-memory ring, completion tracked by mbarriers; the copies use the
//     128-byte swizzle so the tensor-core fragment loads below are free of
//     bank conflicts;
//   - NW consumer warps take pages round robin; per page a warp computes
//     S^T = K Q^T (16 tokens x 8 heads, mma.sync m16n8k16, bf16 in, fp32
//     accumulate), the online-softmax update with warp shuffles, transposes
//     P in registers (movmatrix) and accumulates O^T += V^T P^T on the tensor
//     cores.  Decode does G flops per K/V byte, far below any tensor-core
//     ridge: the kernel is HBM-bound and the warp-level MMAs keep the math
//     off the critical path for every G <= 16 at the same cost per page;
//   - the warps' states are combined in shared memory; a chunk that covers
//     the whole (row, KV head) writes the bf16 output directly, otherwise it
//     writes its partial state and the last block to finish that (row, KV
//     head) (an atomic ticket) merges all states in ascending chunk order,
//     so the result is deterministic and no second launch is needed.
//   - every device-side wait is bounded (2 s); on a timeout the kernel
//     records an error bit in the workspace and gives up instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>

#include "pkv_internal.h"

// One rank-5 TMA copy per K (or V) page; 0 selects one rank-4 copy per
// 64-wide half of head_dim.
#ifndef PKV_TMA_5D
#define PKV_TMA_5D 1
#endif
// Pages per block that the split kernel prefetches into L2 while it waits for
// the kernel before it (0 turns the prefetch off).
#ifndef PKV_L2_PREFETCH_PAGES
#define PKV_L2_PREFETCH_PAGES 16
#endif
static_assert(PKV_L2_PREFETCH_PAGES >= 0 && PKV_L2_PREFETCH_PAGES <= 32, "one page per lane of the producer warp");

namespace pkv {

constexpr int kBoxD = 64;                   // head-dim elements per TMA box row (128 bytes)
constexpr int kBoxBytes = kBoxD * kPage * 2; // one [16 tokens][64 d] bf16 box = 2 KiB
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kWaitLimitIters = 1u << 30;

struct __align__(64) Params {
    CUtensorMap tm_k;  // pool views [pages][H_kv][P][D] -> boxes of [1][1][16][64]
    CUtensorMap tm_v;
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int4 *items;
    const int32_t *indptr;
    float *ws_m;
    float *ws_l;
    float *ws_acc;
    uint32_t *ws_counters;
    uint32_t *ws_error;
    float scale_log2;  // scale * log2(e): logits are kept in the log2 domain
    int32_t B, H_q, H_kv, G, max_pages, num_pool_pages;
    int32_t mode, num_splits, chunk_pages, separate_merge;
    int32_t pdl_early;  // may read lengths, table and KV pages (but a row's last) before the dependency wait
    int32_t n_items;
    int32_t prefetch_blocks;  // blocks below this index warm L2 before the wait (the grid's first wave)
    uint32_t *host_err;       // or NULL: per error bit k, a flag word host_err[k] in mapped host memory
    int32_t n_units;          // prefix-sharing queue: units (the grid); their offsets follow the pair offsets
    int32_t device_fill;      // WORK_QUEUE: every block derives its own item from the device lengths
    int32_t fill_blocks;      // ... of the queue whose chunk fills one wave of this many blocks
#ifdef PKV_TRACE
    int32_t trace_epoch;
#endif
};

// Record an error bit the kernel met on device data: in the workspace's error
// word and, for a call whose caller reads the result straight from host
// memory, as a plain store of 1 into that bit's own flag word there (one word
// per bit, so no read-modify-write crosses the bus).
__device__ __forceinline__ void raise_error(const Params &p, uint32_t bit)
{
    atomicOr(p.ws_error, bit);
    if (p.host_err)
        *reinterpret_cast<volatile uint32_t *>(p.host_err + (__ffs(bit) - 1)) = 1u;
}

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Optional timeline tracing (build with -DPKV_TRACE): thread 0 of each block
// records global-timer stamps at fixed points of the kernel.
#ifdef PKV_TRACE
// Two epochs (launch parity) so that consecutive launches can be compared.
constexpr int kTraceBlocks = 16384;
__device__ unsigned long long g_pkv_trace_buf[2][kTraceBlocks][16];
#define g_pkv_trace (g_pkv_trace_buf[p.trace_epoch & 1])
#define PKV_TRACE_POINT(slot)                                                  \
    do {                                                                       \
        if (threadIdx.x == 0 && blockIdx.x < kTraceBlocks)                     \
            g_pkv_trace[blockIdx.x][slot] = global_timer_ns();                 \
    } while (0)
#else
#define PKV_TRACE_POINT(slot) \
    do {                      \
    } while (0)
#endif

// Wait for phase `parity` of an mbarrier, giving up after kWaitLimitNs (or
// kWaitLimitIters polls) with the timeout bit set in the error word (and,
// when host_flags is not NULL, the timeout's flag word set in host memory).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t *err, uint64_t limit_ns = kWaitLimitNs,
                                       uint32_t *host_flags = nullptr)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1; i < kWaitLimitIters; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255u) == 0 && global_timer_ns() - t0 > limit_ns)
            break;
    }
    atomicOr(err, kErrTimeout);
    if (host_flags)
        *reinterpret_cast<volatile uint32_t *>(host_flags) = 1u;  // bit 0: timeout
    return false;
}

__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// TMA tiled copy of one [1][1][16][64] box of a pool view into shared memory.
__device__ __forceinline__ void tma_load_box(uint32_t dst, const CUtensorMap *tm, uint32_t bar, int d0, int head,
                                             int page, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(d0), "r"(0), "r"(head), "r"(page), "r"(bar), "l"(policy)
        : "memory");
}

// Bulk (non-tensor) async copy global -> shared, completion on an mbarrier.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Per-thread asynchronous copies global -> shared that bypass L1 (16 or 4
// bytes), and the wait for all of this thread's copies.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most the most recently committed group of this thread's
// async copies is still in flight.
__device__ __forceinline__ void cp_async_wait_but_last() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Ticket: atomic add with release (orders this block's earlier writes, made
// visible to thread 0 by the preceding __syncthreads) and acquire (the last
// arriver sees every other block's released writes).
__device__ __forceinline__ uint32_t ticket_acq_rel(uint32_t *ctr)
{
    uint32_t prev;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(prev) : "l"(ctr) : "memory");
    return prev;
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Programmatic dependent launch: wait for the grids this one depends on
// (complete, memory visible); allow dependents to be scheduled.  Both are
// no-ops when the kernel was launched without the PDL attribute.
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Thread-block clusters: rank in the cluster, a full cluster barrier
// (release / acquire), and loads from a peer block's shared memory.
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Barrier among the first `threads` threads of the block (named barrier `id`).
__device__ __forceinline__ void named_barrier(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// TMA tiled copy of a whole (page, head) block [d_hi][16 tokens][64 d] of a
// rank-5 pool view (head_dim split as 64 x d_hi) in one instruction.
__device__ __forceinline__ void tma_load_page(uint32_t dst, const CUtensorMap *tm, uint32_t bar, int head, int page,
                                              uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(0), "r"(0), "r"(0), "r"(head), "r"(page), "r"(bar), "l"(policy)
        : "memory");
}

// L2 prefetch of one (page, head) block through the same tensor map: no
// shared memory, no barrier; coordinates outside the tensor fetch nothing.
template <int D>
__device__ __forceinline__ void tma_prefetch_page_l2(const CUtensorMap *tm, int head, int page)
{
#if PKV_TMA_5D
    asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(0), "r"(0), "r"(0), "r"(head), "r"(page)
                 : "memory");
#else
    for (int d0 = 0; d0 < D; d0 += kBoxD)
        asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                         reinterpret_cast<uint64_t>(tm)),
                     "r"(d0), "r"(0), "r"(head), "r"(page)
                     : "memory");
#endif
}

// Loads that are cached in L2 only (never in L1), for reads of data that a
// kernel still running may be writing: a later load of the same address
// after the dependency wait cannot hit a stale L1 line.
__device__ __forceinline__ int ld_l2_only(const int32_t *ptr)
{
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(ptr));
    return v;
}

__device__ __forceinline__ int4 ld_l2_only(const int4 *ptr)
{
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(ptr));
    return v;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *tm)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                              uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held one row pair per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// 2^x on the SFU (ex2.approx: relative error ~2^-22); 2^-inf = +0.
__device__ __forceinline__ float exp2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16 *dst, float4 v)
{
    uint2 u;
    u.x = pack_bf16(v.x, v.y);
    u.y = pack_bf16(v.z, v.w);
    *reinterpret_cast<uint2 *>(dst) = u;
}

__device__ __forceinline__ float4 fma4(float4 a, float s, float4 b)  // a * s + b
{
    return make_float4(fmaf(a.x, s, b.x), fmaf(a.y, s, b.y), fmaf(a.z, s, b.z), fmaf(a.w, s, b.w));
}

__device__ __forceinline__ float4 scale4(float4 a, float s)
{
    return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}

// ---------------------------------------------------------------------------
// Kernel configuration

template <int D, int NT, int NW, int NST>
struct Cfg {
    static_assert(D == 64 || D == 128, "head_dim");
    // Pages go to warps round robin and to stages round robin; when NST is a
    // multiple of NW every use of a stage belongs to the same warp, so a
    // stage's mbarrier can never be more than one phase ahead of its waiter
    // (otherwise phase parities could alias).
    static_assert(NST % NW == 0, "stages must be a multiple of consumer warps");
    static constexpr int kHalves = D / kBoxD;
    static constexpr int kStageBytes = D * kPage * 2;  // one K (or V) page of one KV head
    static constexpr int kThreads = (NW + 1) * 32;     // NW consumer warps + 1 producer warp
    static constexpr int kGP = 8 * NT;                 // query heads per block, padded to the MMA's n = 8
    static constexpr int kOStride = D + 4;             // floats per (warp, head) row in the combine buffer
    static constexpr int kCombineBytes = NW * kGP * (kOStride + 2) * 4;
    static constexpr int kRingBytes = 2 * NST * kStageBytes;
    static constexpr int kBarOff = ((kRingBytes > kCombineBytes ? kRingBytes : kCombineBytes) + 63) / 64 * 64;
    static constexpr int kMiscOff = kBarOff + 2 * NST * 8;  // int flag, merge mbarriers at +8, +16, a guessed item at +32
    static constexpr int kFillResOff = kMiscOff + 64;       // a block's self-derived work item (8 int32)
    static constexpr int kSmemBytes = kMiscOff + 96 + 1024;  // + slack to align the base to 1024
    static constexpr int kMaxMergeTasks = (kGP * (D / 4) + kThreads - 1) / kThreads;
    // cluster merge: this block's final state [m: 16][l: 16][acc: kGP][D] in the idle ring
    static constexpr int kClusterOff = (kCombineBytes + 127) / 128 * 128;
    static constexpr int kClusterBytes = 128 + kGP * D * 4;
    static_assert(kClusterOff + kClusterBytes <= kRingBytes, "cluster state must fit in the ring");
};

// The producer's issue rate bounds a block's bandwidth: one rank-5 TMA copy
// per K (or V) page instead of one per 64-wide half (PKV_TMA_5D, defined
// above), issued by several lanes at once.
#ifndef PKV_ISSUE_LANES
#define PKV_ISSUE_LANES 4
#endif


// Producer: copy the K and V blocks of cnt consecutive pages of one KV head
// into the ring, page j's physical id held by lane j of `e`; pages get ring
// positions gp, gp+1, ... (stage = position % NST).  PKV_ISSUE_LANES lanes
// issue in parallel, each waiting for its own stage to be released.
// Returns false (after setting the error bit) when a wait timed out.
// Pages before `start` of the batch are already in the ring (copied ahead,
// see the split kernel's speculative start) and are skipped.
template <int D, int NST>
__device__ __forceinline__ bool issue_pages(const Params &p, int lane, int e, int cnt, int &gp, int head,
                                            uint32_t k_ring, uint32_t v_ring, uint32_t bar_full, uint32_t bar_empty,
                                            uint64_t policy, int gate = INT_MAX, int start = 0)
{
    constexpr int kStage = D * kPage * 2;
    bool ok = true;
    gp -= start;  // ring position of page j of the batch: gp + j
    for (int j0 = start; j0 < cnt && ok; j0 += PKV_ISSUE_LANES) {
        // the page at ring position `gate` may be written by the previous
        // kernel: wait for it (whole warp) before copying it
        if (gp + j0 <= gate && gate < gp + j0 + PKV_ISSUE_LANES)
            grid_dependency_wait();
        const int j = j0 + lane;
        const int phys = __shfl_sync(0xffffffffu, e, j & 31);
        bool my_ok = true;
        if (lane < PKV_ISSUE_LANES && j < cnt) {
            const int g = gp + j;
            const int st = g % NST;
            const int k = g / NST;
            if (k > 0 && !mbar_wait(bar_empty + 8 * st, (k - 1) & 1, p.ws_error, kWaitLimitNs, p.host_err))
                my_ok = false;
            if (my_ok) {
                const uint32_t fb = bar_full + 8 * st;
                mbar_expect_tx(fb, 2 * kStage);
#if PKV_TMA_5D
                tma_load_page(k_ring + st * kStage, &p.tm_k, fb, head, phys, policy);
                tma_load_page(v_ring + st * kStage, &p.tm_v, fb, head, phys, policy);
#else
#pragma unroll
                for (int hf = 0; hf < D / kBoxD; ++hf) {
                    tma_load_box(k_ring + st * kStage + hf * kBoxBytes, &p.tm_k, fb, hf * kBoxD, head, phys, policy);
                    tma_load_box(v_ring + st * kStage + hf * kBoxBytes, &p.tm_v, fb, hf * kBoxD, head, phys, policy);
                }
#endif
            }
        }
        ok = __all_sync(0xffffffffu, my_ok);
    }
    gp += cnt;
    return ok;
}

// Attention over one 16-token page in ring stage (ks_base, vs_base) for the
// G heads of one KV head: S^T = K Q^T on the tensor cores, the stage handed
// back to the producer as soon as the K/V fragments are in registers, the
// online-softmax update of (m, l, o) in the log2 domain with tokens >= nvalid
// masked, and O^T += V^T P^T.
template <int D, int NT>
__device__ __forceinline__ void attend_page(uint8_t *smem, uint32_t sbase, uint32_t ks_base, uint32_t vs_base,
                                            uint32_t bar_empty_s, int nvalid, int lane, int r, int ri,
                                            uint32_t k_off, int k_hi, uint32_t v_off, int v_hi, float sl2,
                                            const uint32_t (&qf)[D / 16][NT][2], float (&m_run)[NT][2],
                                            float (&l_run)[NT][2], float (&o)[D / 16][NT][4])
{
    constexpr int kHalves = D / kBoxD;
    if (nvalid < kPage) {
        // Tail page: zero V rows past the row's end, so that stale or
        // NaN slots cannot leak through P = 0 in the PV product.
        uint8_t *vs = smem + (vs_base - sbase);
        const int dead = kPage - nvalid;
        for (int i = lane; i < dead * kHalves * 8; i += 32) {
            const int rr = i >> 3;
            const int hf = rr / dead;
            const int t = nvalid + rr % dead;
            *reinterpret_cast<uint4 *>(vs + hf * kBoxBytes + t * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
    }
    // S^T[t][g] = K[t] . q[g]
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
        sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const int chunk = (((ks & 3) << 1) + k_hi) ^ ri;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(ks_base + (ks >> 2) * kBoxBytes + k_off + (chunk << 4), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            mma_bf16(sacc[nt], a0, a1, a2, a3, qf[ks][nt][0], qf[ks][nt][1]);
    }
    // V^T fragments to registers, then hand the stage back to the
    // producer before the softmax and PV math.
    uint32_t vf[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        const int chunk = (((mt & 3) << 1) + v_hi) ^ ri;
        ldsm_x4_trans(vs_base + (mt >> 2) * kBoxBytes + v_off + (chunk << 4), vf[mt][0], vf[mt][1],
                      vf[mt][2], vf[mt][3]);
    }
    __syncwarp();
    if (nvalid < kPage)
        fence_proxy_async_smem();  // our zero stores precede the next TMA write of this stage
    if (lane == 0)
        mbar_arrive(bar_empty_s);  // release: orders the fragment loads before the refill
    // Online softmax over this page (log2 domain), tokens past the end masked.
    const bool lo_ok = r < nvalid;
    const bool hi_ok = r + 8 < nvalid;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float x0 = lo_ok ? sacc[nt][0] * sl2 : -INFINITY;
        const float x1 = lo_ok ? sacc[nt][1] * sl2 : -INFINITY;
        const float x2 = hi_ok ? sacc[nt][2] * sl2 : -INFINITY;
        const float x3 = hi_ok ? sacc[nt][3] * sl2 : -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
        }
        const float mn0 = fmaxf(m_run[nt][0], mx0);
        const float mn1 = fmaxf(m_run[nt][1], mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
        const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2_approx(m_run[nt][0] - mu0);
        const float al1 = exp2_approx(m_run[nt][1] - mu1);
        const float p0 = exp2_approx(x0 - mu0);
        const float p1 = exp2_approx(x1 - mu1);
        const float p2 = exp2_approx(x2 - mu0);
        const float p3 = exp2_approx(x3 - mu1);
        l_run[nt][0] = fmaf(l_run[nt][0], al0, p0 + p2);
        l_run[nt][1] = fmaf(l_run[nt][1], al1, p1 + p3);
        m_run[nt][0] = mn0;
        m_run[nt][1] = mn1;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][nt][0] *= al0;
            o[mt][nt][1] *= al1;
            o[mt][nt][2] *= al0;
            o[mt][nt][3] *= al1;
        }
        // P^T as the B operand (k = token, n = head): transpose the two 8x8 halves.
        pb[nt][0] = movmatrix_trans(pack_bf16(p0, p1));
        pb[nt][1] = movmatrix_trans(pack_bf16(p2, p3));
    }
    // O^T[d][g] += V^T[d][t] P^T[t][g]
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            mma_bf16(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], pb[nt][0], pb[nt][1]);
}

// (M, L, O) <- (M, L, O) merged with the state (m2, l2, o2); neutral states
// (max = -inf) carry no weight.
__device__ __forceinline__ void merge_into(float &M, float &L, float4 &O, float m2, float l2, float4 o2)
{
    if (m2 == -INFINITY)
        return;
    if (M == -INFINITY) {
        M = m2;
        L = l2;
        O = o2;
        return;
    }
    const float Mn = fmaxf(M, m2);
    const float a = exp2_approx(M - Mn);
    const float b = exp2_approx(m2 - Mn);
    L = fmaf(L, a, l2 * b);
    O = fma4(O, a, scale4(o2, b));
    M = Mn;
}

// The same merge straight from L2 into registers: each thread owns (head g,
// 4 columns) tasks and walks the slots in batches of 4, the loads of batch
// k+1 in flight while batch k is merged (online: running max M, the sum L
// and the accumulator O rescaled as the max grows), in ascending slot order.
template <int D>
__device__ void merge_pair_direct(const Params &p, int row, int h, int slot0, int nslots, int tid, int nthreads)
{
    constexpr int kB = 4;
    const int G = p.G;
    constexpr int D4 = D / 4;
    for (int e = tid; e < G * D4; e += nthreads) {
        const int g = e / D4;
        const int d4 = (e % D4) * 4;
        float M = -INFINITY, L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        float ms[2][kB], ls[2][kB];
        float4 as[2][kB];
        auto load = [&](int buf, int s0) {
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                ms[buf][u] = -INFINITY;
                ls[buf][u] = 0.f;
                as[buf][u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s0 + u < nslots) {
                    const int64_t idx = (int64_t)(slot0 + s0 + u) * G + g;
                    ms[buf][u] = __ldcg(p.ws_m + idx);
                    ls[buf][u] = __ldcg(p.ws_l + idx);
                    as[buf][u] = __ldcg(reinterpret_cast<const float4 *>(p.ws_acc + idx * D + d4));
                }
            }
        };
        load(0, 0);
        for (int s0 = 0, buf = 0; s0 < nslots; s0 += kB, buf ^= 1) {
            if (s0 + kB < nslots) {
                if (buf == 0)
                    load(1, s0 + kB);
                else
                    load(0, s0 + kB);
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const float mu = buf == 0 ? ms[0][u] : ms[1][u];
                const float lu = buf == 0 ? ls[0][u] : ls[1][u];
                const float4 au = buf == 0 ? as[0][u] : as[1][u];
                if (mu == -INFINITY)
                    continue;  // neutral state: weight 0
                const float Mn = fmaxf(M, mu);
                const float a = exp2_approx(M - Mn);
                const float b = exp2_approx(mu - Mn);
                L = fmaf(L, a, lu * b);
                O = fma4(O, a, scale4(au, b));
                M = Mn;
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
    }
}

// Merge of one (row, KV head)'s n partial states by the block that finished
// it last, staged through the idle shared-memory ring.  The weights
// w_s = 2^(m_s - M) (M = max_s m_s, 0 for a neutral state) and the
// denominator L = sum_s w_s l_s are computed once per head; the fp32
// accumulators arrive in chunks by bulk async copies (double buffered), and
// out = sum_s w_s acc_s / L is accumulated in ascending slot order.
// Returns false when the ring cannot hold the weights plus two slots.
template <int D, int NT, int NW, int NST>
__device__ bool merge_pair_staged(const Params &p, uint8_t *smem, uint32_t mbar0, int row, int h, int slot0, int n,
                                  int tid, uint32_t (&uses)[2])
{
    using C = Cfg<D, NT, NW, NST>;
    const int G = p.G;
    constexpr int D4 = D / 4;
    const int slot_bytes = G * D * 4;
    const int wbytes = ((2 * n * G + 32) * 4 + 1023) / 1024 * 1024;
    const int half = (C::kRingBytes - wbytes) / 2 / 1024 * 1024;
    const int hs = half > 0 ? half / slot_bytes : 0;  // slots per buffer
    if (hs < 1)
        return false;
    float *w_s = reinterpret_cast<float *>(smem);  // [n][G]: m, then the weights
    float *l_s = w_s + n * G;                      // [n][G]
    float *ML = l_s + n * G;                       // M[16], L[16]
    const uint32_t stage0 = smem_addr(smem) + wbytes;
    const int nch = (n + hs - 1) / hs;
    if (tid == 0) {
        fence_proxy_async_smem();    // earlier generic accesses to the ring precede the copies
        fence_proxy_async_global();  // the states were written by other blocks' generic stores
        for (int ch = 0; ch < 2 && ch < nch; ++ch) {
            const int cnt = min(hs, n - ch * hs);
            mbar_expect_tx(mbar0 + 8 * ch, cnt * slot_bytes);
            bulk_g2s(stage0 + ch * half, p.ws_acc + (int64_t)(slot0 + ch * hs) * G * D, cnt * slot_bytes,
                     mbar0 + 8 * ch);
        }
    }
    for (int i = tid; i < n * G; i += C::kThreads) {
        w_s[i] = __ldcg(p.ws_m + (int64_t)slot0 * G + i);
        l_s[i] = __ldcg(p.ws_l + (int64_t)slot0 * G + i);
    }
    __syncthreads();
    // One warp per head: M = max_s m_s, the weights, and L = sum_s w_s l_s,
    // each reduced over the lanes by a fixed xor-shuffle tree.
    const int lane = tid & 31;
    for (int g = tid >> 5; g < G; g += C::kThreads / 32) {
        float M = -INFINITY;
        for (int s = lane; s < n; s += 32)
            M = fmaxf(M, w_s[s * G + g]);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1)
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
        float L = 0.f;
        for (int s = lane; s < n; s += 32) {
            const float m = w_s[s * G + g];
            const float wgt = m == -INFINITY ? 0.f : exp2_approx(m - M);
            w_s[s * G + g] = wgt;
            L = fmaf(wgt, l_s[s * G + g], L);
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1)
            L += __shfl_xor_sync(0xffffffffu, L, sh);
        if (lane == 0)
            ML[16 + g] = L;
    }
    __syncthreads();
    float4 O[C::kMaxMergeTasks];
#pragma unroll
    for (int k = 0; k < C::kMaxMergeTasks; ++k)
        O[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int ch = 0; ch < nch; ++ch) {
        mbar_wait(mbar0 + 8 * (ch & 1), (uses[ch & 1] + (ch >> 1)) & 1, p.ws_error, kWaitLimitNs, p.host_err);
        const float *st = reinterpret_cast<const float *>(smem + wbytes + (ch & 1) * half);
        const int first = ch * hs;
        const int cnt = min(hs, n - first);
#pragma unroll
        for (int k = 0; k < C::kMaxMergeTasks; ++k) {
            const int e = tid + k * C::kThreads;
            if (e < G * D4) {
                const int g = e / D4;
                const int d4 = (e % D4) * 4;
                float4 O2 = make_float4(0.f, 0.f, 0.f, 0.f);  // second chain for ILP
                int s = 0;
                for (; s + 1 < cnt; s += 2) {
                    O[k] = fma4(*reinterpret_cast<const float4 *>(st + (s * G + g) * D + d4),
                                w_s[(first + s) * G + g], O[k]);
                    O2 = fma4(*reinterpret_cast<const float4 *>(st + ((s + 1) * G + g) * D + d4),
                              w_s[(first + s + 1) * G + g], O2);
                }
                if (s < cnt)
                    O[k] = fma4(*reinterpret_cast<const float4 *>(st + (s * G + g) * D + d4), w_s[(first + s) * G + g],
                                O[k]);
                O[k] = make_float4(O[k].x + O2.x, O[k].y + O2.y, O[k].z + O2.z, O[k].w + O2.w);
            }
        }
        __syncthreads();
        if (tid == 0 && ch + 2 < nch) {
            fence_proxy_async_smem();  // our reads of this buffer precede its refill
            const int c2 = ch + 2;
            const int cnt2 = min(hs, n - c2 * hs);
            mbar_expect_tx(mbar0 + 8 * (c2 & 1), cnt2 * slot_bytes);
            bulk_g2s(stage0 + (c2 & 1) * half, p.ws_acc + (int64_t)(slot0 + c2 * hs) * G * D, cnt2 * slot_bytes,
                     mbar0 + 8 * (c2 & 1));
        }
    }
#pragma unroll
    for (int k = 0; k < C::kMaxMergeTasks; ++k) {
        const int e = tid + k * C::kThreads;
        if (e < G * D4) {
            const int g = e / D4;
            const int d4 = (e % D4) * 4;
            const float L = ML[16 + g];
            const float inv = L > 0.f ? 1.f / L : 0.f;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O[k], inv));
        }
    }
    uses[0] += (nch + 1) / 2;  // barrier 0 carried the even chunks, barrier 1 the odd ones
    uses[1] += nch / 2;
    __syncthreads();  // the ring is free again once every thread has left it
    return true;
}

// Merge of a pair's states landed in the idle ring by per-thread async
// copies: every thread issues the copies of its own (head g, 4 columns) tasks
// for all n states (and the (m, l) pairs are shared out), so every load of the
// merge is in flight at once without holding registers; then each thread
// merges its tasks alone, in ascending slot order: M = max_s m_s,
// w_s = 2^(m_s - M) (0 for a neutral state), L = sum w_s l_s,
// out = sum w_s acc_s / L.  With kPasses, states too large for the ring go
// through merge_pair_landed_passes; returns false when they cannot land.
template <int D, int NT, int NW, int NST>
__device__ __noinline__ bool merge_pair_landed_passes(const Params &p, uint8_t *smem, int row, int h, int slot0,
                                                      int n, int tid);

// The merge weights of a pair's n landed states, once per head rather than
// once per column task: warp w takes the heads g = w, w + warps, ...; for
// each it finds M_g = max_s m_s, overwrites m_s with w_s = 2^(m_s - M_g)
// (0 for a neutral state) and writes L_g = sum_s w_s l_s to lsum[g].
template <int kThreads>
__device__ __forceinline__ void merge_weights(float *m_s, const float *l_s, float *lsum, int n, int G, int tid)
{
    const int warp = tid >> 5, lane = tid & 31;
    for (int g = warp; g < G; g += kThreads / 32) {
        float M = -INFINITY;
        for (int s = lane; s < n; s += 32)
            M = fmaxf(M, m_s[s * G + g]);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1)
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
        float L = 0.f;
        for (int s = lane; s < n; s += 32) {
            const float m = m_s[s * G + g];
            const float w = m == -INFINITY ? 0.f : exp2_approx(m - M);
            m_s[s * G + g] = w;
            L = fmaf(w, l_s[s * G + g], L);
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1)
            L += __shfl_xor_sync(0xffffffffu, L, sh);
        if (lane == 0)
            lsum[g] = L;
    }
}

// One (head g, 4 columns) task of a landed merge: sum_s w_s acc_s over the
// n states in ascending slot order (two interleaved chains), divided by L_g.
__device__ __forceinline__ float4 merge_task(const float *acc_s, const float *w_s, int n, int G, int g, int stride,
                                             int d4, float L)
{
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f), O2 = O;
    int s = 0;
    for (; s + 1 < n; s += 2) {
        O = fma4(*reinterpret_cast<const float4 *>(acc_s + (s * G + g) * stride + d4), w_s[s * G + g], O);
        O2 = fma4(*reinterpret_cast<const float4 *>(acc_s + ((s + 1) * G + g) * stride + d4), w_s[(s + 1) * G + g],
                  O2);
    }
    if (s < n)
        O = fma4(*reinterpret_cast<const float4 *>(acc_s + (s * G + g) * stride + d4), w_s[s * G + g], O);
    O = make_float4(O.x + O2.x, O.y + O2.y, O.z + O2.z, O.w + O2.w);
    return scale4(O, L > 0.f ? 1.f / L : 0.f);
}

template <int D, int NT, int NW, int NST, bool kPasses>
__device__ bool merge_pair_landed(const Params &p, uint8_t *smem, int row, int h, int slot0, int n, int tid)
{
    using C = Cfg<D, NT, NW, NST>;
    const int G = p.G;
    constexpr int D4 = D / 4;
    const int acc_bytes = n * G * D * 4;
    if (acc_bytes + (2 * n * G + G) * 4 > C::kRingBytes)
        return kPasses && merge_pair_landed_passes<D, NT, NW, NST>(p, smem, row, h, slot0, n, tid);
    float *acc_s = reinterpret_cast<float *>(smem);  // [n][G][D]
    float *m_s = acc_s + n * G * D;                  // [n][G], then the weights
    float *l_s = m_s + n * G;                        // [n][G]
    float *lsum = l_s + n * G;                       // [G]
    const uint32_t base = smem_addr(smem);
    const float *acc_g = p.ws_acc + (int64_t)slot0 * G * D;
    // m and l land first, the accumulators behind them: the weights are
    // computed while the accumulators are still in flight
    for (int i = tid; i < n * G; i += C::kThreads) {
        cp_async_4(smem_addr(m_s + i), p.ws_m + (int64_t)slot0 * G + i);
        cp_async_4(smem_addr(l_s + i), p.ws_l + (int64_t)slot0 * G + i);
    }
    cp_async_commit();
#pragma unroll
    for (int k = 0; k < C::kMaxMergeTasks; ++k) {
        const int e = tid + k * C::kThreads;
        if (e < G * D4) {
            const int g = e / D4;
            const int d4 = (e % D4) * 4;
            for (int s = 0; s < n; ++s) {
                const int off = (s * G + g) * D + d4;
                cp_async_16(base + 4 * off, acc_g + off);
            }
        }
    }
    cp_async_commit();
    cp_async_wait_but_last();
    __syncthreads();
    merge_weights<C::kThreads>(m_s, l_s, lsum, n, G, tid);
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int k = 0; k < C::kMaxMergeTasks; ++k) {
        const int e = tid + k * C::kThreads;
        if (e < G * D4) {
            const int g = e / D4;
            const int d4 = (e % D4) * 4;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4,
                         merge_task(acc_s, m_s, n, G, g, D, d4, lsum[g]));
        }
    }
    __syncthreads();  // the ring is free again once every thread has left it
    return true;
}

// The landed merge in two or four passes over the columns, for states whose
// D columns do not fit the ring at once: each pass lands D/2 or D/4 columns
// of all n states (the m and l of all states land once, behind them) and
// merges them as above.  A call of its own, so that the kernels' main loops
// keep their registers.  Returns false (the caller stages the states instead)
// when a quarter of the columns does not fit either, or when a pass would
// leave most threads idle.
template <int D, int NT, int NW, int NST>
__device__ __noinline__ bool merge_pair_landed_passes(const Params &p, uint8_t *smem, int row, int h, int slot0,
                                                      int n, int tid)
{
    using C = Cfg<D, NT, NW, NST>;
    const int G = p.G;
    const int ml_bytes = (2 * n * G + G) * 4;
    int parts = 2;
    if (n * G * (D / 2) * 4 + ml_bytes > C::kRingBytes)
        parts = 4;
    // Each pass merges G * D / (4 * parts) (head, 4-column) tasks, one per
    // thread, with n dependent steps each; with fewer than 128 tasks (G = 4,
    // or G = 8 in four passes) the staged merge, whose chunks keep all 128
    // consumer threads busy, measured faster (long context at G = 4 with the
    // 8-page ring: 25.2 against 26.6 us per step).
    if (n * G * (D / parts) * 4 + ml_bytes > C::kRingBytes || G * D / (4 * parts) < 128)
        return false;
    const int Dp = D / parts;  // columns per pass
    const int Dp4 = Dp / 4;
    float *acc_s = reinterpret_cast<float *>(smem);  // [n][G][Dp]
    float *m_s = acc_s + n * G * Dp;                 // [n][G], then the weights
    float *l_s = m_s + n * G;                        // [n][G]
    float *lsum = l_s + n * G;                       // [G]
    const uint32_t base = smem_addr(smem);
    const float *acc_g = p.ws_acc + (int64_t)slot0 * G * D;
    for (int i = tid; i < n * G; i += C::kThreads) {
        cp_async_4(smem_addr(m_s + i), p.ws_m + (int64_t)slot0 * G + i);
        cp_async_4(smem_addr(l_s + i), p.ws_l + (int64_t)slot0 * G + i);
    }
    cp_async_commit();
    for (int part = 0; part < parts; ++part) {
        const int c0 = part * Dp;
        for (int e = tid; e < G * Dp4; e += C::kThreads) {
            const int g = e / Dp4;
            const int d4 = (e % Dp4) * 4;
            for (int s = 0; s < n; ++s)
                cp_async_16(base + 4 * ((s * G + g) * Dp + d4), acc_g + (int64_t)(s * G + g) * D + c0 + d4);
        }
        cp_async_commit();
        if (part == 0) {
            cp_async_wait_but_last();
            __syncthreads();
            merge_weights<C::kThreads>(m_s, l_s, lsum, n, G, tid);
        }
        cp_async_wait_all();
        __syncthreads();
        for (int e = tid; e < G * Dp4; e += C::kThreads) {
            const int g = e / Dp4;
            const int d4 = (e % Dp4) * 4;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + c0 + d4,
                         merge_task(acc_s, m_s, n, G, g, Dp, d4, lsum[g]));
        }
        __syncthreads();  // the next pass refills the ring; after the last one it is free again
    }
    return true;
}

// The last block's merge of a pair: through per-thread async copies into the
// ring whenever the ring holds a quarter of the columns of all n states
// ("landed", in one, two or four passes), else staged through the ring in
// double-buffered bulk copies, else straight into registers.
// Timed on B200 with the step's own blocks merging: landed beat staged at 17
// states (mixed batch, 18.3 -> 17.5 us per step) and at 32 (long context,
// 24.2 -> 23.2 us per step).  The balanced grid merges without the column
// passes (kPasses false): the out-of-line call cost its main loop registers
// (128 with spills instead of 140) and 0.7-2.9 us per step.
template <int D, int NT, int NW, int NST, bool kPasses = true>
__device__ void merge_pair_last_block(const Params &p, uint8_t *smem, uint32_t mbar0, int row, int h, int slot0,
                                      int n, int tid, uint32_t (&uses)[2])
{
    using C = Cfg<D, NT, NW, NST>;
    if (merge_pair_landed<D, NT, NW, NST, kPasses>(p, smem, row, h, slot0, n, tid))
        return;
    if (!merge_pair_staged<D, NT, NW, NST>(p, smem, mbar0, row, h, slot0, n, tid, uses))
        merge_pair_direct<D>(p, row, h, slot0, n, tid, C::kThreads);
}

// The guessed range of the block, for the L2 prefetch and the speculative
// start: its (row, KV head), first page, page count (0: no guess) and, in
// lane j, the block-table entry of page pg0 + j (j < PKV_L2_PREFETCH_PAGES).
struct PageGuess {
    int row = 0, h = 0, pg0 = 0, np = 0, e = -1;
};

// L2 prefetch of pages [pg0, pg_end) of (row, KV head h), at most
// PKV_L2_PREFETCH_PAGES of them, one page per lane of the calling warp; the
// block-table entries are read speculatively through L2 (see above).  With
// `g`, the range and the entries are also kept as the block's guess.
template <int D>
__device__ __forceinline__ void l2_prefetch_range(const Params &p, int lane, int row, int h, int64_t pg0,
                                                  int64_t pg_end, PageGuess *g = nullptr)
{
#if PKV_L2_PREFETCH_PAGES > 0
    const int64_t j = pg0 + lane;
    int e = -1;
    if (lane < PKV_L2_PREFETCH_PAGES && j < pg_end && j < p.max_pages) {
        e = ld_l2_only(p.block_table + (int64_t)row * p.max_pages + j);
        if (e >= 0 && e < p.num_pool_pages) {
            tma_prefetch_page_l2<D>(&p.tm_k, h, e);
            tma_prefetch_page_l2<D>(&p.tm_v, h, e);
        }
    }
    if (g) {
        g->row = row;
        g->h = h;
        g->pg0 = (int)pg0;
        g->np = pg_end > pg0 ? (int)(pg_end - pg0) : 0;
        g->e = e;
    }
#endif
}

// Before its dependency wait the split kernel may read nothing that the
// kernel before it might still be writing.  What it may do is warm L2: the
// producer warp reads its range (work item or row length) and the first
// block-table entries speculatively, through L2 only, and asks the TMA unit to
// prefetch the first PKV_L2_PREFETCH_PAGES K/V pages of the range into L2.
// A stale or torn value costs only a useless prefetch (page ids are range
// checked, and a prefetch moves no data into the block); everything the block
// uses is read again after the wait, and L2 is coherent with the writes of
// the kernel before.  In a back-to-back decode loop this streams the first
// pages while the previous step finishes its merges.
// In the work-queue grid the producer also hands the speculatively read
// item to the block (*spec, set when it is a well-formed item): after the
// wait the block then issues the loads that depend on the item (the pair's
// slot range, the first block-table entries) at the addresses the guess
// gives, together with the item itself, and keeps them only if the item
// read after the wait equals the guess.  Every value used is read after the
// wait; the guess only saves one round trip to L2 when it is right.
template <int D>
__device__ __forceinline__ void l2_prefetch_first_pages(const Params &p, int lane, int64_t row_cap, int4 *spec,
                                                        PageGuess &g)
{
#if PKV_L2_PREFETCH_PAGES > 0
    int row, h;
    int64_t pg0, pg_end;
    if (p.mode == PKV_WORK_QUEUE) {
        const int4 it = ld_l2_only(p.items + blockIdx.x);
        if (!(it.x >= 0 && it.x < p.B && it.y >= 0 && it.y < p.H_kv && it.z >= 0 && it.z <= it.w && it.w <= row_cap &&
              (it.z % kPage) == 0))
            return;
        if (lane == 0)
            *spec = it;
        row = it.x;
        h = it.y;
        pg0 = it.z / kPage;
        pg_end = (it.w + kPage - 1) / kPage;
    } else {
        const int S = p.mode == PKV_SPLIT_S ? p.num_splits : 1;
        const int pair = blockIdx.x / S;
        row = pair / p.H_kv;
        h = pair % p.H_kv;
        int64_t N = ld_l2_only(p.seq_lens + row);
        N = N < 0 ? 0 : (N > row_cap ? row_cap : N);
        pg_end = (N + kPage - 1) / kPage;
        pg0 = 0;
        if (p.mode == PKV_SPLIT_S) {
            pg0 = (int64_t)(blockIdx.x % S) * p.chunk_pages;
            pg_end = pg_end < pg0 + p.chunk_pages ? pg_end : pg0 + p.chunk_pages;
        }
    }
    l2_prefetch_range<D>(p, lane, row, h, pg0, pg_end, &g);
#endif
}

// Rows a block can plan for itself (PKV_FLAG_DEVICE_FILL): the derivation
// keeps three int32 per row in the idle shared-memory ring.
constexpr int kFillMaxRows = 1024;

struct FillItem {
    int row, h, tb, te, slot0, nslots, len;
    bool valid;
};

__device__ __forceinline__ int warp_sum_i32(int v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ int warp_max_i32(int v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// The compact work queue whose chunk fills one wave of T = p.fill_blocks
// blocks [PKV, Methodology 1 "Compact work queue", "Row-local bounds"; the
// fill rule is this library's], derived by each block for itself from the
// device lengths, so that no builder kernel runs before the decode: the
// same items, in the same (row, KV head, chunk) order, as
// pkv_build_work_queue at the chunk C that pkv_select_policy's fill rule
// picks.  C is the smallest chunk (pages) with
//   count(C) = H_kv * sum_i max(1, ceil(pages_i / C)) <= T,
// or pages_max when one item per (row, KV head) already exceeds T.  Since
// ceil(x) lies in [x, x + 1), C lies in [ceil(H_kv * U / T),
// ceil(H_kv * U / (T - H_kv * B))] (U = sum_i pages_i): the 32 lanes of
// warp 0 test 32 candidates of that range at a time, so the search takes one
// round whenever the range holds at most 32 chunk sizes (it does when the
// wave is large against B * H_kv).  Then a prefix sum over the rows' chunk
// counts places block b's item.  Warp 0 does the work in 32-bit arithmetic
// (the host checks H_kv * B * max_pages < 2^31): up to 32 rows in registers
// (lane i holds row i, shuffles carry the rest), more through `sm`, 3 * B + 1
// int32 of the idle ring.  The item reaches the block through `res` (8
// int32 outside the ring): called by every thread (one block barrier).
// speculative: lengths read through L2 before the dependency wait, for the
// L2 prefetch only; no error is recorded.
__device__ __forceinline__ uint32_t fill_row_len(const Params &p, int i, bool speculative)
{
    const uint32_t cap = (uint32_t)p.max_pages * kPage;
    const int n = speculative ? ld_l2_only(p.seq_lens + i) : __ldg(p.seq_lens + i);
    if (n >= 0 && (uint32_t)n <= cap)
        return (uint32_t)n;
    if (!speculative)
        raise_error(p, kErrSeqLen);
    return n < 0 ? 0u : cap;
}

// The smallest chunk in [lo, hi] that satisfies the fill rule (hi does),
// given count(c) (items of one KV head at chunk c) for the lane's candidate;
// called by a whole warp, every lane calling count() in step.
template <typename Count>
__device__ __forceinline__ uint32_t fill_search(uint32_t lo, uint32_t hi, uint32_t limit, int lane, Count count)
{
    while (lo < hi) {
        const uint32_t step = (hi - lo + 32) / 32;
        const uint32_t c = lo + (uint32_t)lane * step;
        const uint32_t n = count(c < hi ? c : hi);  // every lane counts: count() may shuffle
        const bool ok = c < hi && n <= limit;
        const uint32_t hits = __ballot_sync(0xffffffffu, ok);
        const uint32_t b = hits ? lo + (uint32_t)(__ffs(hits) - 1) * step : hi;
        lo = b + 1 > lo + step ? b + 1 - step : lo;
        hi = b;
    }
    return lo;
}

template <int NTHREADS>
__device__ __forceinline__ FillItem fill_queue_item(const Params &p, int32_t *sm, int32_t *res, bool speculative)
{
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int B = p.B;
    if (tid < 32) {
        const uint32_t T = (uint32_t)p.fill_blocks;
        const uint32_t H = (uint32_t)p.H_kv;
        const uint32_t HB = H * (uint32_t)B;
        const uint32_t b = blockIdx.x;
        uint32_t pmax = 0, U = 0;
        uint32_t my_len = 0, my_pg = 0;  // row `lane` (B <= 32)
        if (B <= 32) {
            if (lane < B) {
                my_len = fill_row_len(p, lane, speculative);
                my_pg = (my_len + kPage - 1) / kPage;
            }
            pmax = my_pg;
            U = my_pg;
        } else {
            for (int i = lane; i < B; i += 32) {
                const uint32_t N = fill_row_len(p, i, speculative);
                const uint32_t pg = (N + kPage - 1) / kPage;
                sm[B + i] = (int32_t)N;
                sm[i] = (int32_t)pg;
                pmax = max(pmax, pg);
                U += pg;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            pmax = max(pmax, __shfl_xor_sync(0xffffffffu, pmax, off));
            U += __shfl_xor_sync(0xffffffffu, U, off);
        }
        __syncwarp();
        if (!speculative)
            PKV_TRACE_POINT(15);
        // items of one head at chunk c
        auto count = [&](uint32_t c) {
            uint32_t n = 0;
            for (int i = 0; i < B; ++i) {
                const uint32_t pg = B <= 32 ? __shfl_sync(0xffffffffu, my_pg, i) : (uint32_t)sm[i];
                const uint32_t k = (pg + c - 1) / c;
                n += k > 1 ? k : 1;
            }
            return n;
        };
        uint32_t C;
        if (pmax == 0) {
            C = 1;  // every row is empty: one empty item per (row, KV head)
        } else if (HB > T) {
            C = pmax;
        } else {
            uint32_t lo = (H * U + T - 1) / T;
            uint32_t hi = HB < T ? (H * U + (T - HB) - 1) / (T - HB) : pmax;
            lo = lo < 1 ? 1 : (lo > pmax ? pmax : lo);
            hi = hi > pmax ? pmax : (hi < lo ? lo : hi);
            C = fill_search(lo, hi, T / H, lane, count);  // count(c) * H <= T  <=>  count(c) <= T / H
        }
        int row = -1;
        uint32_t row_start = 0, row_cnt = 1, row_len = 0;
        if (B <= 32) {
            // one KV head's item offset of row `lane`, then the row whose items hold b
            uint32_t cnt = 0;
            if (lane < B) {
                const uint32_t k = (my_pg + C - 1) / C;
                cnt = k > 1 ? k : 1;
            }
            uint32_t incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t add = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off)
                    incl += add;
            }
            const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
            const uint32_t start = incl - cnt;
            if (b < total * H) {
                row = __popc(__ballot_sync(0xffffffffu, lane < B && start * H <= b)) - 1;
                row_start = __shfl_sync(0xffffffffu, start, row);
                row_cnt = __shfl_sync(0xffffffffu, cnt, row);
                row_len = __shfl_sync(0xffffffffu, my_len, row);
            }
        } else {
            int32_t *rs = sm + 2 * B;  // [B + 1]: items of one KV head before row i
            uint32_t carry = 0;
            for (int base = 0; base < B; base += 32) {
                const int i = base + lane;
                uint32_t cnt = 0;
                if (i < B) {
                    const uint32_t k = ((uint32_t)sm[i] + C - 1) / C;
                    cnt = k > 1 ? k : 1;
                }
                uint32_t incl = cnt;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t add = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off)
                        incl += add;
                }
                if (i < B)
                    rs[i] = (int32_t)(carry + incl - cnt);
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0)
                rs[B] = (int32_t)carry;
            __syncwarp();
            if (b < carry * H) {
                int below = 0;
                for (int base = 0; base < B; base += 32) {
                    const int i = base + lane;
                    below += __popc(__ballot_sync(0xffffffffu, i < B && (uint32_t)rs[i] * H <= b));
                }
                row = below - 1;
                row_start = (uint32_t)rs[row];
                row_cnt = (uint32_t)(rs[row + 1] - rs[row]);
                row_len = (uint32_t)sm[B + row];
            }
            fence_proxy_async_smem();  // these generic writes precede later TMA writes into the ring
        }
        if (lane == 0) {
            res[0] = row;
            if (row >= 0) {
                const uint32_t j = b - row_start * H;
                const uint32_t h = j / row_cnt, c = j - h * row_cnt;
                const uint32_t span = C * kPage;
                res[1] = (int32_t)h;
                res[2] = row_len > 0 ? (int32_t)(c * span) : 0;
                res[3] = row_len > 0 ? (int32_t)((c + 1) * span < row_len ? (c + 1) * span : row_len) : 0;
                res[4] = (int32_t)(row_start * H + h * row_cnt);
                res[5] = (int32_t)row_cnt;
                res[6] = (int32_t)row_len;
            }
        }
    }
    __syncthreads();
    FillItem f;
    f.row = res[0];
    f.valid = f.row >= 0;
    f.h = res[1];
    f.tb = res[2];
    f.te = res[3];
    f.slot0 = res[4];
    f.nslots = res[5];
    f.len = res[6];
    __syncthreads();  // every thread has read res before it is written again
    return f;
}

// One block = one work item (row, KV head, token range) for all G query heads.
// The launch bounds say how many blocks share an SM: two for the deep ring
// (by shared memory), three for the 8-page ring.  The three-block hint keeps
// the 8-stage D = 128, G <= 8 variant at 128 registers; without it the
// kernel grew to 134 registers, which fit only two blocks of five warps per
// SM (registers are handed out per SM sub-partition), and many-wave queues
// ran up to 25 % slower.
// FILL: the self-planned queue (PKV_FLAG_DEVICE_FILL) and its speculative
// start are compiled into a variant of their own: in the other variants
// their code cost the main loop 6 registers and 0.1-0.3 us per step.
template <int D, int NT, int NW, int NST, bool CL, bool FILL>
__global__ void __launch_bounds__((NW + 1) * 32, (NST >= 12 ? 2 : 3)) split_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<D, NT, NW, NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t k_ring = sbase;
    const uint32_t v_ring = sbase + NST * C::kStageBytes;
    const uint32_t bar_full = sbase + C::kBarOff;
    const uint32_t bar_empty = bar_full + NST * 8;
    volatile int *misc = reinterpret_cast<volatile int *>(smem + C::kMiscOff);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t row_cap = (int64_t)p.max_pages * kPage;
    PKV_TRACE_POINT(0);
    // Set-up that reads no global data comes first: the ring's barriers and
    // the tensor maps (kernel parameters).
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(sbase + C::kMiscOff + 8, 1);
        mbar_init(sbase + C::kMiscOff + 16, 1);
        mbar_init(sbase + C::kMiscOff + 24, 1);  // the speculative start's verdict
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == NW && lane == 0) {
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
    }
    // Under programmatic dependent launch this block may start while the
    // previous kernel on the stream is still running: wait before reading
    // any global memory it may have written (after warming L2 with the
    // first pages, see l2_prefetch_first_pages).  With pdl_early the caller
    // promises that kernel writes neither the lengths, the table, the queue
    // nor any KV page but a row's last, so those are read first and the wait
    // comes before q, the last page and any global write.
    // guessed work item (row = -1: none), see l2_prefetch_first_pages
    int4 *spec_item = reinterpret_cast<int4 *>(smem + C::kMiscOff + 32);
    if (tid == 0)
        *spec_item = make_int4(-1, 0, 0, 0);
    int32_t *fill_scratch = reinterpret_cast<int32_t *>(smem);  // the idle ring, before any page copy
    int32_t *fill_res = reinterpret_cast<int32_t *>(smem + C::kFillResOff);
    const uint32_t verify_bar = sbase + C::kMiscOff + 24;
    PageGuess guess;  // the producer warp's guess of its range (np = 0: none)
    const uint64_t policy = evict_first_policy();
    int spec_k = 0;   // producer: pages copied ahead into ring positions 0 .. spec_k - 1
    if (!p.pdl_early) {
        __syncthreads();
        const bool warm = (int)blockIdx.x < p.prefetch_blocks;
        if (FILL && p.mode == PKV_WORK_QUEUE) {
            if (warm) {
                const FillItem g = fill_queue_item<C::kThreads>(p, fill_scratch, fill_res, true);
                if (g.valid && tid == 0)
                    *spec_item = make_int4(g.row, g.h, g.tb, g.te);
                if (g.valid && warp == NW)
                    l2_prefetch_range<D>(p, lane, g.row, g.h, g.tb / kPage, (g.te + kPage - 1) / kPage, &guess);
            }
        } else if (warm && warp == NW) {
            l2_prefetch_first_pages<D>(p, lane, row_cap, spec_item, guess);
        }
        __syncthreads();
        grid_dependency_wait();
        PKV_TRACE_POINT(13);
        // Speculative start of the self-planned queue: copy the guessed
        // range's first pages now, before the block has derived its real
        // range from the lengths (≈ 1.5 µs).  The copies read K/V after the
        // dependency wait, so only the guessed page ids can be wrong; the
        // producer checks them against the real ones before the consumers
        // touch the ring, and on any difference those ring positions are
        // drained and skipped.  Only there: where the range is one round trip
        // away (a host-built queue, split-S), copies issued this early
        // measured slower, since they queue ahead of that round trip.  Not
        // either when the queue has more rows than a warp holds in registers:
        // its derivation then keeps its arrays in the ring.
        if (FILL && warp == NW && p.mode == PKV_WORK_QUEUE && p.B <= 32) {
            int k = guess.np < PKV_L2_PREFETCH_PAGES ? guess.np : PKV_L2_PREFETCH_PAGES;
            k = (k < NST ? k : NST) & ~(NW - 1);  // whole rounds of the consumer warps
            const bool ok = lane >= k || (guess.e >= 0 && guess.e < p.num_pool_pages);
            if (!__all_sync(0xffffffffu, ok))
                k = 0;
            spec_k = k;
            if (k > 0) {
                int gp = 0;
                issue_pages<D, NST>(p, lane, guess.e, k, gp, guess.h, k_ring, v_ring, bar_full, bar_empty, policy);
            }
        }
    }
    // a block that leaves before streaming first waits for its speculative copies
    auto drain = [&]() {
        if (warp == NW && lane < spec_k)
            mbar_wait(bar_full + 8 * lane, 0, p.ws_error, kWaitLimitNs, p.host_err);
    };

    // ---- which (row, KV head, token range) this block owns ----
    // The producer warp fetches the first 32 block-table entries of the
    // range as soon as the range's first page is known, which for the
    // no-split and split-S grids is before the row length arrives.
    int row, h, tb, te, slot0 = 0, nslots = 1, my_slot = 0;
    int e_first = 0;
    bool hit = false;  // the guessed work item was the real one
    int row_len = -1;  // the row's length where known (for the early dependency gate)
    if (FILL && p.mode == PKV_WORK_QUEUE) {
        // the block's own item, derived from the device lengths; the
        // table entries at the guessed item's first page go out first
        const int4 guess = p.pdl_early ? make_int4(-1, 0, 0, 0) : *spec_item;
        int g_entry = 0;
        if (guess.x >= 0 && warp == NW) {
            const int idx = guess.z / kPage + lane;
            if (idx < p.max_pages)
                g_entry = __ldg(p.block_table + (int64_t)guess.x * p.max_pages + idx);
        }
        const FillItem f = fill_queue_item<C::kThreads>(p, fill_scratch, fill_res, false);
        PKV_TRACE_POINT(14);
        if (!f.valid) {
            drain();
            return;
        }
        hit = guess.x == f.row && guess.y == f.h && guess.z == f.tb && guess.w == f.te;
        row = f.row;
        h = f.h;
        tb = f.tb;
        te = f.te;
        slot0 = f.slot0;
        nslots = f.nslots;
        my_slot = blockIdx.x;
        e_first = g_entry;
        if (slot0 + nslots > p.n_items) {
            if (tid == 0)
                raise_error(p, kErrItem);
            drain();
            return;
        }
        if (warp == NW) {
            const int idx = tb / kPage + lane;
            if (!hit && idx < p.max_pages)
                e_first = __ldg(p.block_table + (int64_t)row * p.max_pages + idx);
            row_len = f.len;
        }
    } else if (p.mode == PKV_WORK_QUEUE) {
        // a queue built on the device may hold fewer items than the grid has
        // blocks (the buffer holds one per block); the item, the item count
        // and the loads at the guessed item's addresses go out at once
        const int4 guess = p.pdl_early ? make_int4(-1, 0, 0, 0) : *spec_item;  // written before the last barrier
        const int n_real = __ldg(p.indptr + p.B * p.H_kv);
        const int4 it = __ldg(p.items + blockIdx.x);
        int g_slot0 = 0, g_slot1 = 0, g_entry = 0;
        if (guess.x >= 0) {
            const int gpair = guess.x * p.H_kv + guess.y;
            g_slot0 = __ldg(p.indptr + gpair);
            g_slot1 = __ldg(p.indptr + gpair + 1);
            const int idx = guess.z / kPage + lane;
            if (warp == NW && idx < p.max_pages)
                g_entry = __ldg(p.block_table + (int64_t)guess.x * p.max_pages + idx);
        }
        if ((int)blockIdx.x >= n_real) {
            drain();
            return;
        }
        hit = guess.x >= 0 && guess.x == it.x && guess.y == it.y && guess.z == it.z && guess.w == it.w;
        row = it.x;
        h = it.y;
        tb = it.z;
        te = it.w;
        bool ok = row >= 0 && row < p.B && h >= 0 && h < p.H_kv && tb >= 0 && tb <= te && te <= row_cap &&
                  (tb % kPage) == 0;
        if (ok) {
            const int pair = row * p.H_kv + h;
            slot0 = hit ? g_slot0 : __ldg(p.indptr + pair);
            nslots = (hit ? g_slot1 : __ldg(p.indptr + pair + 1)) - slot0;
            e_first = g_entry;
            my_slot = blockIdx.x;
            ok = nslots >= 1 && slot0 >= 0 && my_slot >= slot0 && my_slot < slot0 + nslots &&
                 slot0 + nslots <= p.n_items;
        }
        if (!ok) {
            if (tid == 0)
                raise_error(p, kErrItem);
            drain();
            return;
        }
        if (warp == NW) {
            const int idx = tb / kPage + lane;
            if (!hit && idx < p.max_pages)
                e_first = __ldg(p.block_table + (int64_t)row * p.max_pages + idx);
            if (p.pdl_early)
                row_len = __ldg(p.seq_lens + row);
        }
    } else {
        const int S = p.mode == PKV_SPLIT_S ? p.num_splits : 1;
        const int pair = blockIdx.x / S;
        const int c = blockIdx.x % S;
        row = pair / p.H_kv;
        h = pair % p.H_kv;
        if (warp == NW) {
            const int64_t idx = (p.mode == PKV_SPLIT_S ? (int64_t)c * p.chunk_pages : 0) + lane;
            if (idx < p.max_pages)
                e_first = __ldg(p.block_table + (int64_t)row * p.max_pages + idx);
        }
        int N = __ldg(p.seq_lens + row);
        if (N < 0 || N > row_cap) {
            if (tid == 0)
                raise_error(p, kErrSeqLen);
            N = N < 0 ? 0 : (int)row_cap;
        }
        row_len = N;
        if (p.mode == PKV_SPLIT_S) {
            const int64_t span = (int64_t)p.chunk_pages * kPage;
            if (c == 0 && tid == 0 && (int64_t)S * span < N)
                raise_error(p, kErrItem);  // the plan's S * C pages do not cover this row
            const int64_t b = (int64_t)c * span;
            tb = (int)(b < N ? b : N);
            te = (int)(b < N ? (b + span < N ? b + span : N) : N);  // empty chunk: tb == te
            nslots = S;
            slot0 = pair * S;
            my_slot = slot0 + c;
        } else {
            tb = 0;
            te = N;
        }
    }
    const int pair = row * p.H_kv + h;
    const int pg0 = tb / kPage;
    const int npages = te > tb ? (te + kPage - 1) / kPage - pg0 : 0;

    __syncthreads();  // the barriers' initialisation is visible to all warps
    PKV_TRACE_POINT(1);
#ifdef PKV_TRACE
    if (tid == 0 && blockIdx.x < kTraceBlocks) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        g_pkv_trace[blockIdx.x][6] = smid;
        g_pkv_trace[blockIdx.x][7] = npages;
    }
#endif

    // Per-warp softmax state for the heads g = 8*nt + 2*(lane%4) + j.
    float m_run[NT][2], l_run[NT][2];
    float o[D / 16][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
            o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }
    const int r = lane >> 2;  // fragment row group
    const int c4 = lane & 3;  // fragment column pair

    if (warp == NW) {
        // ================= producer: block table -> TMA page copies =================
        const int32_t *bt = p.block_table + (int64_t)row * p.max_pages + pg0;
        // the speculative copies hold pages 0 .. spec_k - 1 when the guess was
        // right (same pair, same first page, enough pages, same page ids);
        // otherwise the pages start at ring position spec_k
        const bool right = __all_sync(0xffffffffu, spec_k > 0 && row == guess.row && h == guess.h &&
                                                       pg0 == guess.pg0 && npages >= spec_k &&
                                                       (lane >= spec_k || e_first == guess.e));
        if (FILL && lane == 0) {
            misc[1] = spec_k | ((spec_k > 0 && !right) ? 0x100 : 0);
            mbar_arrive(verify_bar);  // release: the verdict precedes the consumers' reads
        }
        const int skip = right ? spec_k : 0;  // pages already in the ring
#ifdef PKV_TRACE
        long long prod_wait = 0;
        const long long prod_t0 = clock64();
#endif
        int e_next = lane < npages ? e_first : 0;
        bool ok = true;
        int gp = spec_k;  // the first ring position not holding a speculative copy
        // ring position of the row's last page, which the previous kernel may write
        int gate = INT_MAX;
        if (p.pdl_early) {
            const int last = row_len > 0 ? (row_len - 1) / kPage : (row_len < 0 ? pg0 : -1);
            if (last >= pg0 && last < pg0 + npages)
                gate = last - pg0;
            else if (row_len < 0 || row_len > row_cap)
                gate = 0;  // unknown or invalid length: wait before the first copy
        }
        for (int base = 0; base < npages && ok; base += 32) {
            int e = e_next;
            e_next = base + 32 + lane < npages ? __ldg(bt + base + 32 + lane) : 0;
            const bool bad = base + lane < npages && (e < 0 || e >= p.num_pool_pages);
            if (__any_sync(0xffffffffu, bad) && lane == 0)
                raise_error(p, kErrPageId);
            if (bad)
                e = 0;  // read a real page instead; the error bit reports the bad entry
            const int cnt = npages - base < 32 ? npages - base : 32;
#ifdef PKV_TRACE
            const long long tw0 = clock64();
#endif
            ok = issue_pages<D, NST>(p, lane, e, cnt, gp, h, k_ring, v_ring, bar_full, bar_empty, policy, gate,
                                     base == 0 ? skip : 0);
#ifdef PKV_TRACE
            prod_wait += clock64() - tw0;
#endif
        }
        if (p.pdl_early)
            grid_dependency_wait();  // before this warp's share of the global writes below
#ifdef PKV_TRACE
        if (lane == 0 && blockIdx.x < kTraceBlocks) {
            g_pkv_trace[blockIdx.x][10] = prod_wait;
            g_pkv_trace[blockIdx.x][11] = clock64() - prod_t0;
        }
#endif
    } else {
        // ================= consumers: tensor-core attention over pages =================
        // Q as the MMA's B operand (k = head_dim, n = query head), loaded once.
        if (p.pdl_early)
            grid_dependency_wait();  // q may come from the previous kernel
        uint32_t qf[D / 16][NT][2];
        const __nv_bfloat16 *qb = p.q + ((int64_t)row * p.H_q + (int64_t)h * p.G) * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int g = nt * 8 + r;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t lo = 0, hi = 0;
                if (g < p.G) {
                    const uint32_t *src = reinterpret_cast<const uint32_t *>(qb + (int64_t)g * D + ks * 16 + 2 * c4);
                    lo = __ldg(src);
                    hi = __ldg(src + 4);
                }
                qf[ks][nt][0] = lo;
                qf[ks][nt][1] = hi;
            }
        }
        // ldmatrix lane roles: matrix mi = lane / 8, row ri = lane % 8 (= token % 8).
        const int mi = lane >> 3;
        const int ri = lane & 7;
        const uint32_t k_off = (uint32_t)((8 * (mi & 1) + ri) * 128);   // K as A (rows = tokens)
        const int k_hi = mi >> 1;
        const uint32_t v_off = (uint32_t)((8 * (mi >> 1) + ri) * 128);  // V^T as A via .trans
        const int v_hi = mi & 1;
        const float sl2 = p.scale_log2;
#ifdef PKV_TRACE
        long long cons_wait = 0;
        const long long cons_t0 = clock64();
#endif
        // the speculative start's verdict: on a wrong guess, release the ring
        // positions its copies took (each once they landed) and read the pages
        // from position `spec` on
        int offset = 0;
        if (FILL && !p.pdl_early && mbar_wait(verify_bar, 0, p.ws_error, kWaitLimitNs, p.host_err)) {
            const int v = misc[1];
            const int spec = v & 0xff;
            if (v & 0x100) {
                offset = spec;
                for (int q = warp; q < spec; q += NW) {
                    mbar_wait(bar_full + 8 * (q % NST), (q / NST) & 1, p.ws_error, kWaitLimitNs, p.host_err);
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar_empty + 8 * (q % NST));
                }
            }
        }

        for (int pidx = warp; pidx < npages; pidx += NW) {
            const int qpos = pidx + offset;
            const int s = qpos % NST;
#ifdef PKV_TRACE
            const long long tw0 = clock64();
#endif
            const bool ready = mbar_wait(bar_full + 8 * s, (qpos / NST) & 1, p.ws_error, kWaitLimitNs, p.host_err);
#ifdef PKV_TRACE
            cons_wait += clock64() - tw0;
#endif
            if (!__all_sync(0xffffffffu, ready))
                break;
            const uint32_t ks_base = k_ring + s * C::kStageBytes;
            const uint32_t vs_base = v_ring + s * C::kStageBytes;
            const int tok0 = (pg0 + pidx) * kPage;
            const int nvalid = te - tok0 < kPage ? te - tok0 : kPage;
            attend_page<D, NT>(smem, sbase, ks_base, vs_base, bar_empty + 8 * s, nvalid, lane, r, ri, k_off, k_hi,
                               v_off, v_hi, sl2, qf, m_run, l_run, o);
            if (pidx == 0)
                PKV_TRACE_POINT(2);
        }
#ifdef PKV_TRACE
        if (tid == 0 && blockIdx.x < kTraceBlocks) {
            g_pkv_trace[blockIdx.x][8] = cons_wait;
            g_pkv_trace[blockIdx.x][9] = clock64() - cons_t0;
        }
#endif
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1)
                    l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], sh);
    }

    // ---- combine the warps' states (the ring is idle now; reuse it) ----
    grid_launch_dependents();  // the next kernel may start its prologue
    __syncthreads();
    PKV_TRACE_POINT(3);
    float *cb_o = reinterpret_cast<float *>(smem);
    float *cb_m = cb_o + NW * C::kGP * C::kOStride;
    float *cb_l = cb_m + NW * C::kGP;
    if (warp < NW) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int g = nt * 8 + 2 * c4 + j;
                float *dst = cb_o + (warp * C::kGP + g) * C::kOStride;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    dst[mt * 16 + r] = o[mt][nt][j];
                    dst[mt * 16 + r + 8] = o[mt][nt][2 + j];
                }
                if (r == 0) {
                    cb_m[warp * C::kGP + g] = m_run[nt][j];
                    cb_l[warp * C::kGP + g] = l_run[nt][j];
                }
            }
    }
    __syncthreads();

    constexpr int D4 = D / 4;
    const int G = p.G;
    for (int e = tid; e < G * D4; e += C::kThreads) {
        const int g = e / D4;
        const int d4 = (e % D4) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, cb_m[w * C::kGP + g]);
        float L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = cb_m[w * C::kGP + g];
            if (mw == -INFINITY)
                continue;
            const float sc = exp2_approx(mw - M);
            L = fmaf(cb_l[w * C::kGP + g], sc, L);
            O = fma4(*reinterpret_cast<const float4 *>(cb_o + (w * C::kGP + g) * C::kOStride + d4), sc, O);
        }
        if (CL) {
            float *cs = reinterpret_cast<float *>(smem + C::kClusterOff);
            *reinterpret_cast<float4 *>(cs + 32 + g * D + d4) = O;
            if (d4 == 0) {
                cs[g] = M;
                cs[16 + g] = L;
            }
        } else if (nslots == 1) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
        } else {
            const int64_t idx = (int64_t)my_slot * G + g;
            *reinterpret_cast<float4 *>(p.ws_acc + idx * D + d4) = O;
            if (d4 == 0) {
                p.ws_m[idx] = M;
                p.ws_l[idx] = L;
            }
        }
    }

    PKV_TRACE_POINT(4);
    if (CL) {
        // ---- cluster merge: the S blocks of this (row, KV head) form one
        // cluster; each merges a slice of the (head, 4-column) tasks over all
        // S states, read from the peers' shared memory in rank order ----
        cluster_sync_all();
        const uint32_t cs_addr = sbase + C::kClusterOff;
        const int S = nslots;
        const int T = G * D4;
        const int per = (T + S - 1) / S;
        const int e0 = (int)cluster_ctarank() * per;
        const int e1 = e0 + per < T ? e0 + per : T;
        for (int e = e0 + tid; e < e1; e += C::kThreads) {
            const int g = e / D4;
            const int d4 = (e % D4) * 4;
            float ms[16], ls[16];
            float4 as[16];
#pragma unroll
            for (int src = 0; src < 16; ++src) {
                ms[src] = -INFINITY;
                ls[src] = 0.f;
                as[src] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src < S) {
                    const uint32_t base = map_shared_rank(cs_addr, (uint32_t)src);
                    ms[src] = ld_cluster_f32(base + 4 * g);
                    ls[src] = ld_cluster_f32(base + 64 + 4 * g);
                    as[src] = ld_cluster_f32x4(base + 128 + 4 * (g * D + d4));
                }
            }
            float M = -INFINITY, L = 0.f;
            float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int src = 0; src < 16; ++src)
                merge_into(M, L, O, ms[src], ls[src], as[src]);
            const float inv = L > 0.f ? 1.f / L : 0.f;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
        }
        cluster_sync_all();  // peers may still be reading this block's state
    }
    // ---- the last block of a split (row, KV head) merges its states ----
    if (!CL && nslots > 1 && !p.separate_merge) {
        __syncthreads();
        if (tid == 0) {
            const uint32_t prev = ticket_acq_rel(p.ws_counters + pair);
            misc[0] = prev == (uint32_t)(nslots - 1);
        }
        __syncthreads();
        if (misc[0]) {
            uint32_t uses[2] = {0, 0};
            merge_pair_last_block<D, NT, NW, NST>(p, smem, sbase + C::kMiscOff + 8, row, h, slot0, nslots, tid,
                                                  uses);
            if (tid == 0)
                p.ws_counters[pair] = 0u;  // ready for the next call
            PKV_TRACE_POINT(5);
        }
    }
    PKV_TRACE_POINT(12);
}

// ---------------------------------------------------------------------------
// Prefix-sharing grid (PKV_FLAG_SHARED_PREFIX): one block per unit of the
// prefix-sharing queue.  A unit's members are items of up to 16 / G rows
// that cover the same tokens of the same KV head on the same physical pages
// (a prefix their block tables share ["Chapter 8 - Next-generation KV cache
// management", 8.1 and 8.3]): each page is staged once and the tensor-core
// tile carries the G query heads of every member (16 columns, two n = 8
// tiles), so the shared K/V bytes cross HBM once per unit instead of once per
// row.  Each member's partial state goes to its own slot (its item), and the
// last block to finish a member's (row, KV head) merges that pair as in the
// plain queue.  Units of one member are plain work items.

constexpr int kMaxMembers = 16;
constexpr int kPrefixSmemExtra = (8 * kMaxMembers + 16) * 4;  // member table of a unit

// The prefix grid's counterpart of l2_prefetch_first_pages: the unit's first
// member, read speculatively through L2 before the dependency wait.
template <int D>
__device__ __forceinline__ void l2_prefetch_unit(const Params &p, int lane, int64_t row_cap)
{
#if PKV_L2_PREFETCH_PAGES > 0
    const int32_t *unit_ptr = p.indptr + p.B * p.H_kv + 1;
    const int32_t *unit_items = unit_ptr + p.n_units + 1;
    const int u0 = ld_l2_only(unit_ptr + blockIdx.x);
    if (u0 < 0 || u0 >= p.n_items)
        return;
    const int x = ld_l2_only(unit_items + u0);
    if (x < 0 || x >= p.n_items)
        return;
    const int4 it = ld_l2_only(p.items + x);
    if (!(it.x >= 0 && it.x < p.B && it.y >= 0 && it.y < p.H_kv && it.z >= 0 && it.z <= it.w && it.w <= row_cap))
        return;
    l2_prefetch_range<D>(p, lane, it.x, it.y, it.z / kPage, (it.w + kPage - 1) / kPage);
#endif
}

template <int D, int NW, int NST>
__global__ void __launch_bounds__((NW + 1) * 32, (NST >= 12 ? 2 : 1)) prefix_kernel(const __grid_constant__ Params p)
{
    constexpr int NT = 2;  // 16 query columns: the G heads of up to 16 / G members
    using C = Cfg<D, NT, NW, NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // the members' table past the misc area (kPrefixSmemExtra bytes; no static shared memory, so the
    // dynamic size may use everything an SM offers a block)
    int *s_row = reinterpret_cast<int *>(smem + C::kMiscOff + 96);
    int *s_item = s_row + kMaxMembers, *s_slot0 = s_item + kMaxMembers, *s_nslots = s_slot0 + kMaxMembers;
    int *s_h = s_nslots + kMaxMembers, *s_tb = s_h + kMaxMembers, *s_te = s_tb + kMaxMembers;
    int *s_last = s_te + kMaxMembers;
    volatile int &s_bad = s_last[kMaxMembers];
    const uint32_t sbase = smem_addr(smem);
    const uint32_t k_ring = sbase;
    const uint32_t v_ring = sbase + NST * C::kStageBytes;
    const uint32_t bar_full = sbase + C::kBarOff;
    const uint32_t bar_empty = bar_full + NST * 8;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t row_cap = (int64_t)p.max_pages * kPage;
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(sbase + C::kMiscOff + 8, 1);
        mbar_init(sbase + C::kMiscOff + 16, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
        s_bad = 0;
    }
    if (warp == NW && lane == 0) {
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
    }
    __syncthreads();
    if (warp == NW && (int)blockIdx.x < p.prefetch_blocks)
        l2_prefetch_unit<D>(p, lane, row_cap);
    __syncthreads();
    grid_dependency_wait();

    // ---- the unit's members: same KV head, same tokens, own rows and slots ----
    const int pairs = p.B * p.H_kv;
    const int32_t *unit_ptr = p.indptr + pairs + 1;
    const int32_t *unit_items = unit_ptr + p.n_units + 1;
    const int u0 = __ldg(unit_ptr + blockIdx.x);
    const int k = __ldg(unit_ptr + blockIdx.x + 1) - u0;
    const int G = p.G;
    if (u0 < 0 || k < 1 || k > kMaxMembers || k * G > 8 * NT || u0 + k > p.n_items) {
        if (tid == 0)
            raise_error(p, kErrItem);
        return;
    }
    if (tid < k) {
        const int x = __ldg(unit_items + u0 + tid);
        bool ok = x >= 0 && x < p.n_items;
        const int4 it = ok ? __ldg(p.items + x) : make_int4(-1, 0, 0, 0);
        ok = ok && it.x >= 0 && it.x < p.B && it.y >= 0 && it.y < p.H_kv && it.z >= 0 && it.z <= it.w &&
             it.w <= row_cap && (it.z % kPage) == 0;
        int slot0 = 0, nslots = 0;
        if (ok) {
            const int pair = it.x * p.H_kv + it.y;
            slot0 = __ldg(p.indptr + pair);
            nslots = __ldg(p.indptr + pair + 1) - slot0;
            ok = nslots >= 1 && slot0 >= 0 && x >= slot0 && x < slot0 + nslots && slot0 + nslots <= p.n_items;
        }
        s_row[tid] = it.x;
        s_item[tid] = x;
        s_h[tid] = it.y;
        s_tb[tid] = it.z;
        s_te[tid] = it.w;
        s_slot0[tid] = slot0;
        s_nslots[tid] = nslots;
        if (!ok)
            s_bad = 1;
    }
    __syncthreads();
    if (tid < k && (s_h[tid] != s_h[0] || s_tb[tid] != s_tb[0] || s_te[tid] != s_te[0]))
        s_bad = 1;
    __syncthreads();
    if (s_bad) {
        if (tid == 0)
            raise_error(p, kErrItem);
        return;
    }
    const int h = s_h[0];
    const int tb = s_tb[0];
    const int te = s_te[0];
    const int row0 = s_row[0];
    const int pg0 = tb / kPage;
    const int npages = te > tb ? (te + kPage - 1) / kPage - pg0 : 0;

    float m_run[NT][2], l_run[NT][2];
    float o[D / 16][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
            o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }
    const int r = lane >> 2;
    const int c4 = lane & 3;

    if (warp == NW) {
        // ================= producer: the first member's table (the pages are shared) =================
        const int32_t *bt = p.block_table + (int64_t)row0 * p.max_pages + pg0;
        const uint64_t policy = evict_first_policy();
        int e_next = lane < npages ? __ldg(bt + lane) : 0;
        bool ok = true;
        int gp = 0;
        for (int base = 0; base < npages && ok; base += 32) {
            int e = e_next;
            e_next = base + 32 + lane < npages ? __ldg(bt + base + 32 + lane) : 0;
            const bool bad = base + lane < npages && (e < 0 || e >= p.num_pool_pages);
            if (__any_sync(0xffffffffu, bad) && lane == 0)
                raise_error(p, kErrPageId);
            if (bad)
                e = 0;
            const int cnt = npages - base < 32 ? npages - base : 32;
            ok = issue_pages<D, NST>(p, lane, e, cnt, gp, h, k_ring, v_ring, bar_full, bar_empty, policy);
        }
    } else {
        // ================= consumers: column j = member (j / G), head (j % G) =================
        uint32_t qf[D / 16][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int j = nt * 8 + r;
            const int m = j / G;
            const bool live = m < k;
            const __nv_bfloat16 *qb =
                p.q + ((int64_t)(live ? s_row[m] : 0) * p.H_q + (int64_t)h * G + (live ? j % G : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t lo = 0, hi = 0;
                if (live) {
                    const uint32_t *src = reinterpret_cast<const uint32_t *>(qb + ks * 16 + 2 * c4);
                    lo = __ldg(src);
                    hi = __ldg(src + 4);
                }
                qf[ks][nt][0] = lo;
                qf[ks][nt][1] = hi;
            }
        }
        const int mi = lane >> 3;
        const int ri = lane & 7;
        const uint32_t k_off = (uint32_t)((8 * (mi & 1) + ri) * 128);
        const int k_hi = mi >> 1;
        const uint32_t v_off = (uint32_t)((8 * (mi >> 1) + ri) * 128);
        const int v_hi = mi & 1;
        const float sl2 = p.scale_log2;
        for (int pidx = warp; pidx < npages; pidx += NW) {
            const int s = pidx % NST;
            const bool ready = mbar_wait(bar_full + 8 * s, (pidx / NST) & 1, p.ws_error, kWaitLimitNs, p.host_err);
            if (!__all_sync(0xffffffffu, ready))
                break;
            const int tok0 = (pg0 + pidx) * kPage;
            const int nvalid = te - tok0 < kPage ? te - tok0 : kPage;
            attend_page<D, NT>(smem, sbase, k_ring + s * C::kStageBytes, v_ring + s * C::kStageBytes,
                               bar_empty + 8 * s, nvalid, lane, r, ri, k_off, k_hi, v_off, v_hi, sl2, qf, m_run,
                               l_run, o);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1)
                    l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], sh);
    }

    // ---- combine the warps' states per column; each member's to its own slot ----
    grid_launch_dependents();
    __syncthreads();
    float *cb_o = reinterpret_cast<float *>(smem);
    float *cb_m = cb_o + NW * C::kGP * C::kOStride;
    float *cb_l = cb_m + NW * C::kGP;
    if (warp < NW) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int g = nt * 8 + 2 * c4 + j;
                float *dst = cb_o + (warp * C::kGP + g) * C::kOStride;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    dst[mt * 16 + r] = o[mt][nt][j];
                    dst[mt * 16 + r + 8] = o[mt][nt][2 + j];
                }
                if (r == 0) {
                    cb_m[warp * C::kGP + g] = m_run[nt][j];
                    cb_l[warp * C::kGP + g] = l_run[nt][j];
                }
            }
    }
    __syncthreads();
    constexpr int D4 = D / 4;
    for (int e = tid; e < k * G * D4; e += C::kThreads) {
        const int col = e / D4;
        const int d4 = (e % D4) * 4;
        const int m = col / G;
        const int g = col % G;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, cb_m[w * C::kGP + col]);
        float L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = cb_m[w * C::kGP + col];
            if (mw == -INFINITY)
                continue;
            const float sc = exp2_approx(mw - M);
            L = fmaf(cb_l[w * C::kGP + col], sc, L);
            O = fma4(*reinterpret_cast<const float4 *>(cb_o + (w * C::kGP + col) * C::kOStride + d4), sc, O);
        }
        if (s_nslots[m] == 1) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            store_bf16x4(p.out + ((int64_t)s_row[m] * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
        } else {
            const int64_t idx = (int64_t)s_item[m] * G + g;
            *reinterpret_cast<float4 *>(p.ws_acc + idx * D + d4) = O;
            if (d4 == 0) {
                p.ws_m[idx] = M;
                p.ws_l[idx] = L;
            }
        }
    }
    if (p.separate_merge)
        return;
    // ---- tickets: the last block of a member's (row, KV head) merges it ----
    __syncthreads();
    if (tid < k) {
        s_last[tid] = 0;
        if (s_nslots[tid] > 1) {
            const uint32_t prev = ticket_acq_rel(p.ws_counters + s_row[tid] * p.H_kv + h);
            s_last[tid] = prev == (uint32_t)(s_nslots[tid] - 1);
        }
    }
    __syncthreads();
    uint32_t uses[2] = {0, 0};
    for (int m = 0; m < k; ++m) {
        if (!s_last[m])
            continue;
        merge_pair_last_block<D, NT, NW, NST>(p, smem, sbase + C::kMiscOff + 8, s_row[m], h, s_slot0[m], s_nslots[m],
                                              tid, uses);
        if (tid == 0)
            p.ws_counters[s_row[m] * p.H_kv + h] = 0u;  // ready for the next call
    }
}

// ---------------------------------------------------------------------------
// Balanced persistent grid: block b streams the items of its equal page share
// (the balanced queue) back to back through one ring.  The producer never
// stops at item boundaries; the consumer warps close each item with a combine
// in a dedicated buffer, and the merges this block owns (it was the last to
// finish a pair) run at the end, when the ring is idle.

template <int D, int NT, int NW, int NST>
struct BCfg {
    using Base = Cfg<D, NT, NW, NST>;
    static constexpr int kThreads = Base::kThreads;
    static constexpr int kStageBytes = Base::kStageBytes;
    static constexpr int kRingBytes = Base::kRingBytes;
    static constexpr int kGP = Base::kGP;
    static constexpr int kOStride = Base::kOStride;
    static constexpr int kCombOff = kRingBytes;
    static constexpr int kCombBytes = NW * kGP * (kOStride + 2) * 4;
    static constexpr int kBarOff = (kCombOff + kCombBytes + 63) / 64 * 64;
    static constexpr int kMiscOff = kBarOff + 2 * NST * 8;  // flags, two merge mbarriers, deferred merges
    static constexpr int kMaxDeferred = 32;
    static constexpr int kListOff = kMiscOff + 64;
    static constexpr int kSmemBytes = kListOff + 16 * kMaxDeferred + 1024;
};

// Page range of one balanced-queue item; false (and no pages) for an item
// that does not describe a valid range of a valid (row, KV head).
__device__ __forceinline__ bool item_pages(const Params &p, const int4 &it, int &pg0, int &np)
{
    const int64_t row_cap = (int64_t)p.max_pages * kPage;
    const bool ok = it.x >= 0 && it.x < p.B && it.y >= 0 && it.y < p.H_kv && it.z >= 0 && it.z <= it.w &&
                    it.w <= row_cap && (it.z % kPage) == 0;
    pg0 = ok ? it.z / kPage : 0;
    np = ok && it.w > it.z ? (it.w + kPage - 1) / kPage - pg0 : 0;
    return ok;
}

// The balanced grid's counterpart of l2_prefetch_first_pages: the first
// PKV_L2_PREFETCH_PAGES pages of this block's share, walked through its first
// work items, all read speculatively through L2 before the dependency wait.
template <int D>
__device__ __forceinline__ void l2_prefetch_block_share(const Params &p, int lane)
{
#if PKV_L2_PREFETCH_PAGES > 0
    const int32_t *block_ptr = p.indptr + p.B * p.H_kv + 1;
    const int it0 = ld_l2_only(block_ptr + blockIdx.x);
    const int it1 = ld_l2_only(block_ptr + blockIdx.x + 1);
    if (it0 < 0 || it1 < it0 || it1 > p.n_items)
        return;
    int got = 0;
    for (int it = it0; it < it1 && it < it0 + PKV_L2_PREFETCH_PAGES && got < PKV_L2_PREFETCH_PAGES; ++it) {
        const int4 item = ld_l2_only(p.items + it);
        int pg0, np;
        if (!item_pages(p, item, pg0, np))
            return;
        const int cnt = np < PKV_L2_PREFETCH_PAGES - got ? np : PKV_L2_PREFETCH_PAGES - got;
        if (lane >= got && lane < got + cnt) {
            const int e = ld_l2_only(p.block_table + (int64_t)item.x * p.max_pages + pg0 + (lane - got));
            if (e >= 0 && e < p.num_pool_pages) {
                tma_prefetch_page_l2<D>(&p.tm_k, item.y, e);
                tma_prefetch_page_l2<D>(&p.tm_v, item.y, e);
            }
        }
        got += cnt;
    }
#endif
}

template <int D, int NT, int NW, int NST>
__global__ void __launch_bounds__((NW + 1) * 32) balanced_kernel(const __grid_constant__ Params p)
{
    using C = BCfg<D, NT, NW, NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t k_ring = sbase;
    const uint32_t v_ring = sbase + NST * C::kStageBytes;
    const uint32_t bar_full = sbase + C::kBarOff;
    const uint32_t bar_empty = bar_full + NST * 8;
    volatile int *misc = reinterpret_cast<volatile int *>(smem + C::kMiscOff);  // [0] deferred count, [1] merge now
    int4 *deferred = reinterpret_cast<int4 *>(smem + C::kListOff);
    float *cb_o = reinterpret_cast<float *>(smem + C::kCombOff);
    float *cb_m = cb_o + NW * C::kGP * C::kOStride;
    float *cb_l = cb_m + NW * C::kGP;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    constexpr int kConsumers = NW * 32;
    // set-up that reads no global data, then the dependency wait (see split_kernel)
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(sbase + C::kMiscOff + 8, 1);
        mbar_init(sbase + C::kMiscOff + 16, 1);
        misc[0] = 0;
        misc[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == NW && lane == 0) {
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
    }
    if (warp == NW && (int)blockIdx.x < p.prefetch_blocks)
        l2_prefetch_block_share<D>(p, lane);
    grid_dependency_wait();

    const int pairs = p.B * p.H_kv;
    const int32_t *block_ptr = p.indptr + pairs + 1;
    const int it0 = __ldg(block_ptr + blockIdx.x);
    const int it1 = __ldg(block_ptr + blockIdx.x + 1);
    if (it0 < 0 || it1 < it0 || it1 > p.n_items) {
        if (tid == 0)
            raise_error(p, kErrItem);
        return;
    }
    __syncthreads();  // the barriers' initialisation is visible to all warps

    const int r = lane >> 2;
    const int c4 = lane & 3;
    if (warp == NW) {
        // ================= producer =================
        const uint64_t policy = evict_first_policy();
        int gp = 0;
        bool ok = true;
        for (int it = it0; it < it1 && ok; ++it) {
            const int4 item = __ldg(p.items + it);
            int pg0, np;
            if (!item_pages(p, item, pg0, np) && lane == 0)
                raise_error(p, kErrItem);
            const int32_t *bt = p.block_table + (int64_t)item.x * p.max_pages + pg0;
            for (int base = 0; base < np && ok; base += 32) {
                int e = base + lane < np ? __ldg(bt + base + lane) : 0;
                const bool bad = base + lane < np && (e < 0 || e >= p.num_pool_pages);
                if (__any_sync(0xffffffffu, bad) && lane == 0)
                    raise_error(p, kErrPageId);
                if (bad)
                    e = 0;
                const int cnt = np - base < 32 ? np - base : 32;
                ok = issue_pages<D, NST>(p, lane, e, cnt, gp, item.y, k_ring, v_ring, bar_full, bar_empty, policy);
            }
        }
    } else {
        // ================= consumers =================
        const int mi = lane >> 3;
        const int ri = lane & 7;
        const uint32_t k_off = (uint32_t)((8 * (mi & 1) + ri) * 128);
        const int k_hi = mi >> 1;
        const uint32_t v_off = (uint32_t)((8 * (mi >> 1) + ri) * 128);
        const int v_hi = mi & 1;
        const float sl2 = p.scale_log2;
        const int G = p.G;
        constexpr int D4 = D / 4;
        int gp_base = 0;
        bool alive = true;
        for (int it = it0; it < it1; ++it) {
            const int4 item = __ldg(p.items + it);
            int pg0, np;
            const bool item_ok = item_pages(p, item, pg0, np);
            const int row = item.x, h = item.y, te = item.w;
            uint32_t qf[D / 16][NT][2];
            float m_run[NT][2], l_run[NT][2];
            float o[D / 16][NT][4];
            const __nv_bfloat16 *qb = p.q + ((int64_t)(item_ok ? row : 0) * p.H_q + (int64_t)(item_ok ? h : 0) * G) * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int g = nt * 8 + r;
                m_run[nt][0] = m_run[nt][1] = -INFINITY;
                l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt)
                    o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t lo = 0, hi = 0;
                    if (g < G) {
                        const uint32_t *src =
                            reinterpret_cast<const uint32_t *>(qb + (int64_t)g * D + ks * 16 + 2 * c4);
                        lo = __ldg(src);
                        hi = __ldg(src + 4);
                    }
                    qf[ks][nt][0] = lo;
                    qf[ks][nt][1] = hi;
                }
            }
            // this warp's pages of the item: global page index gp with gp % NW == warp
            for (int gp = gp_base + ((warp - gp_base % NW) + NW) % NW; alive && gp < gp_base + np; gp += NW) {
                const int s = gp % NST;
                const bool ready = mbar_wait(bar_full + 8 * s, (gp / NST) & 1, p.ws_error, kWaitLimitNs, p.host_err);
                if (!__all_sync(0xffffffffu, ready)) {
                    alive = false;
                    break;
                }
                const int pidx = gp - gp_base;
                const int tok0 = (pg0 + pidx) * kPage;
                const int nvalid = te - tok0 < kPage ? te - tok0 : kPage;
                attend_page<D, NT>(smem, sbase, k_ring + s * C::kStageBytes, v_ring + s * C::kStageBytes,
                                   bar_empty + 8 * s, nvalid, lane, r, ri, k_off, k_hi, v_off, v_hi, sl2, qf, m_run,
                                   l_run, o);
            }
            gp_base += np;
            // ---- close the item: combine the consumer warps' states ----
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int sh = 4; sh < 32; sh <<= 1)
                        l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], sh);
                    const int g = nt * 8 + 2 * c4 + j;
                    float *dst = cb_o + (warp * C::kGP + g) * C::kOStride;
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        dst[mt * 16 + r] = o[mt][nt][j];
                        dst[mt * 16 + r + 8] = o[mt][nt][2 + j];
                    }
                    if (r == 0) {
                        cb_m[warp * C::kGP + g] = m_run[nt][j];
                        cb_l[warp * C::kGP + g] = l_run[nt][j];
                    }
                }
            named_barrier(1, kConsumers);
            const int pair = item_ok ? row * p.H_kv + h : 0;
            int slot0 = 0, nslots = 0;
            if (item_ok) {
                slot0 = __ldg(p.indptr + pair);
                nslots = __ldg(p.indptr + pair + 1) - slot0;
            }
            const bool slot_ok = item_ok && nslots >= 1 && slot0 >= 0 && it >= slot0 && it < slot0 + nslots &&
                                 slot0 + nslots <= p.n_items;
            if (!slot_ok && item_ok && tid == 0)
                raise_error(p, kErrItem);
            if (slot_ok) {
                for (int e = tid; e < G * D4; e += kConsumers) {
                    const int g = e / D4;
                    const int d4 = (e % D4) * 4;
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < NW; ++w)
                        M = fmaxf(M, cb_m[w * C::kGP + g]);
                    float L = 0.f;
                    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        const float mw = cb_m[w * C::kGP + g];
                        if (mw == -INFINITY)
                            continue;
                        const float sc = exp2_approx(mw - M);
                        L = fmaf(cb_l[w * C::kGP + g], sc, L);
                        O = fma4(*reinterpret_cast<const float4 *>(cb_o + (w * C::kGP + g) * C::kOStride + d4), sc, O);
                    }
                    if (nslots == 1) {
                        const float inv = L > 0.f ? 1.f / L : 0.f;
                        store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
                    } else {
                        const int64_t idx = (int64_t)it * G + g;
                        *reinterpret_cast<float4 *>(p.ws_acc + idx * D + d4) = O;
                        if (d4 == 0) {
                            p.ws_m[idx] = M;
                            p.ws_l[idx] = L;
                        }
                    }
                }
            }
            named_barrier(1, kConsumers);  // partial stored by all consumers; combine buffer free
            if (slot_ok && nslots > 1 && !p.separate_merge) {
                if (tid == 0) {
                    const uint32_t prev = ticket_acq_rel(p.ws_counters + pair);
                    if (prev == (uint32_t)(nslots - 1)) {
                        const int k = misc[0];
                        if (k < C::kMaxDeferred) {
                            deferred[k] = make_int4(row, h, slot0, nslots);
                            misc[0] = k + 1;
                        } else {
                            misc[1] = 1;  // list full: merge right away
                        }
                    }
                }
                named_barrier(1, kConsumers);
                if (misc[1]) {
                    merge_pair_direct<D>(p, row, h, slot0, nslots, tid, kConsumers);
                    named_barrier(1, kConsumers);
                    if (tid == 0) {
                        p.ws_counters[pair] = 0u;
                        misc[1] = 0;
                    }
                    named_barrier(1, kConsumers);
                }
            }
        }
    }

    // ---- merges this block owns, through the now idle ring ----
    grid_launch_dependents();
    __syncthreads();
    const int nd = misc[0];
    uint32_t uses[2] = {0, 0};
    for (int k = 0; k < nd; ++k) {
        const int4 d = deferred[k];
        merge_pair_last_block<D, NT, NW, NST, false>(p, smem, sbase + C::kMiscOff + 8, d.x, d.y, d.z, d.w, tid,
                                                     uses);
        __syncthreads();
        if (tid == 0)
            p.ws_counters[d.x * p.H_kv + d.y] = 0u;  // ready for the next call
    }
}

// Separate merge (chained to the split kernel by programmatic dependent
// launch): one block per (row, KV head); pairs with one slot were finalized
// by the split kernel.  Four threads share each (head, 4-column) task; a
// thread loads the m, l and acc of its slots (every fourth one, 8 slots per
// batch) all at once, so a pair of up to 32 slots costs one memory round
// trip, then the four partial merges are combined by a fixed xor tree.
constexpr int kMergeThreads = 512;
constexpr int kMergeTPT = 4;
constexpr int kMergeBatch = 8;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ Params p)
{
    grid_dependency_wait();  // the split kernel's partial states are complete and visible
    const int pair = blockIdx.x;
    const int row = pair / p.H_kv;
    const int h = pair % p.H_kv;
    int slot0, nslots;
    if (p.mode == PKV_SPLIT_S) {
        slot0 = pair * p.num_splits;
        nslots = p.num_splits;
    } else {
        slot0 = __ldg(p.indptr + pair);
        nslots = __ldg(p.indptr + pair + 1) - slot0;
        if (slot0 < 0 || nslots < 0 || slot0 + nslots > p.n_items) {
            if (threadIdx.x == 0)
                raise_error(p, kErrItem);
            return;
        }
    }
    if (nslots <= 1)
        return;
    const int G = p.G;
    constexpr int D4 = D / 4;
    const int sub = threadIdx.x % kMergeTPT;
    for (int t = threadIdx.x / kMergeTPT; t < G * D4; t += kMergeThreads / kMergeTPT) {
        const int g = t / D4;
        const int d4 = (t % D4) * 4;
        float M = -INFINITY, L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = sub; s0 < nslots; s0 += kMergeTPT * kMergeBatch) {
            float ms[kMergeBatch], ls[kMergeBatch];
            float4 as[kMergeBatch];
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u) {
                const int s = s0 + u * kMergeTPT;
                ms[u] = -INFINITY;
                ls[u] = 0.f;
                as[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s < nslots) {
                    const int64_t idx = (int64_t)(slot0 + s) * G + g;
                    ms[u] = __ldcg(p.ws_m + idx);
                    ls[u] = __ldcg(p.ws_l + idx);
                    as[u] = __ldcg(reinterpret_cast<const float4 *>(p.ws_acc + idx * D + d4));
                }
            }
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u)
                merge_into(M, L, O, ms[u], ls[u], as[u]);
        }
#pragma unroll
        for (int off = 1; off < kMergeTPT; off <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, M, off);
            const float l2 = __shfl_xor_sync(0xffffffffu, L, off);
            float4 o2;
            o2.x = __shfl_xor_sync(0xffffffffu, O.x, off);
            o2.y = __shfl_xor_sync(0xffffffffu, O.y, off);
            o2.z = __shfl_xor_sync(0xffffffffu, O.z, off);
            o2.w = __shfl_xor_sync(0xffffffffu, O.w, off);
            merge_into(M, L, O, m2, l2, o2);
        }
        if (sub == 0) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            store_bf16x4(p.out + ((int64_t)row * p.H_q + (int64_t)h * G + g) * D + d4, scale4(O, inv));
        }
    }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that no
// one arrives at; the wait must give up after limit_ns and set the timeout bit.
__global__ void wait_timeout_selftest_kernel(uint32_t *err, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_wait(b, 0, err, limit_ns);
    }
}

// ---------------------------------------------------------------------------
// Device-side builder of the balanced queue, so that a decode step whose
// lengths change on the device (a CUDA graph replayed every step) needs no
// host planning.  Same output as pkv_build_balanced_queue for the same
// lengths: the (row, KV head) pairs laid end to end, U pages in all, block b
// of T owning pages [floor(bU/T), floor((b+1)U/T)); every maximal run of one
// pair's pages in one share is an item, a row with no tokens gets one empty
// item per head owned by the last block whose share starts at or before the
// pair's position; indptr holds the pair offsets, then the block offsets.
// One block of threads: the row page counts and the per-pair item counts are
// each prefix-summed over the block, then the items are emitted one per
// thread (each finds its pair by a binary search of the pair offsets), so a
// pair spread over many shares no longer costs one thread a serial loop.

constexpr int kBuildThreads = 256;
constexpr int kBuildWarps = kBuildThreads / 32;
constexpr int kBuildMaxRows = 4096;

__device__ __forceinline__ int64_t share_start(int64_t U, int64_t T, int64_t b) { return (b * U) / T; }

// Last block whose share starts at or before page u: the largest b < T with
// floor(bU/T) <= u, i.e. bU < (u+1)T, i.e. b = ceil((u+1)T / U) - 1.
__device__ __forceinline__ int64_t share_owner(int64_t U, int64_t T, int64_t u)
{
    if (U == 0)
        return T - 1;
    const int64_t b = ((u + 1) * T + U - 1) / U - 1;
    return b < T - 1 ? b : T - 1;
}

// Block-wide primitives of the queue builders (all threads call them):
// shuffles inside each warp, one shared-memory pass over the warps' values,
// two barriers in all.  `scan` holds kBuildWarps values.
__device__ int64_t block_inclusive_scan(int64_t v, int64_t *scan)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int64_t add = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off)
            v += add;
    }
    if (lane == 31)
        scan[warp] = v;
    __syncthreads();
    int64_t before = 0;
    for (int w = 0; w < warp; ++w)
        before += scan[w];
    __syncthreads();  // scan[] is free again
    return v + before;
}

__device__ int64_t block_sum(int64_t v, int64_t *scan)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0)
        scan[threadIdx.x >> 5] = v;
    __syncthreads();
    int64_t r = 0;
    for (int w = 0; w < kBuildWarps; ++w)
        r += scan[w];
    __syncthreads();
    return r;
}

__device__ int64_t block_max(int64_t v, int64_t *scan)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const int64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    if ((threadIdx.x & 31) == 0)
        scan[threadIdx.x >> 5] = v;
    __syncthreads();
    int64_t r = scan[0];
    for (int w = 1; w < kBuildWarps; ++w)
        r = scan[w] > r ? scan[w] : r;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kBuildThreads)
    balanced_queue_kernel(const int32_t *lens, int32_t B, int32_t H_kv, int32_t P, int32_t max_pages, int32_t T,
                          int4 *items, int32_t capacity, int32_t *indptr, uint32_t *err)
{
    __shared__ int64_t row_start[kBuildMaxRows + 1];  // pages of one head's rows before row i
    __shared__ int64_t scan[kBuildWarps];
    __shared__ int64_t total;
    grid_dependency_wait();     // the lengths may come from the kernel before
    grid_launch_dependents();  // the decode kernel may start its set-up
    const int tid = threadIdx.x;
    const int64_t cap_tokens = (int64_t)max_pages * P;
    auto clamped_len = [&](int i) {
        int64_t N = lens[i];
        if (N < 0 || N > cap_tokens) {
            atomicOr(err, kErrSeqLen);
            N = N < 0 ? 0 : cap_tokens;
        }
        return N;
    };
    int64_t carry = 0;
    for (int base = 0; base < B; base += kBuildThreads) {
        const int i = base + tid;
        const int64_t pg = i < B ? (clamped_len(i) + P - 1) / P : 0;
        const int64_t incl = block_inclusive_scan(pg, scan);
        if (i < B)
            row_start[i] = carry + incl - pg;
        if (tid == kBuildThreads - 1)
            total = carry + incl;
        __syncthreads();
        carry = total;
        __syncthreads();
    }
    if (tid == 0)
        row_start[B] = carry;
    __syncthreads();
    const int64_t U = carry * H_kv;
    const int64_t pairs = (int64_t)B * H_kv;
    int32_t *block_ptr = indptr + pairs + 1;
    // position and page count of pair q; the owner of its last item
    auto pair_span = [&](int64_t q, int64_t &a, int64_t &n) {
        const int iq = (int)(q / H_kv);
        n = row_start[iq + 1] - row_start[iq];
        a = row_start[iq] * H_kv + (q % H_kv) * n;
    };
    auto last_owner = [&](int64_t q) {
        int64_t a, n;
        pair_span(q, a, n);
        return share_owner(U, T, n == 0 ? a : a + n - 1);
    };
    // the pairs' item counts and offsets
    carry = 0;
    for (int64_t base = 0; base < pairs; base += kBuildThreads) {
        const int64_t p = base + tid;
        int64_t a = 0, n = 0, cnt = 0;
        if (p < pairs) {
            pair_span(p, a, n);
            // distinct owners of the pair's pages: every share holds a page when U >= T,
            // exactly one page or none when U < T
            const int64_t span = share_owner(U, T, a + n - 1) - share_owner(U, T, a) + 1;
            cnt = n == 0 ? 1 : (span < n ? span : n);
        }
        const int64_t incl = block_inclusive_scan(cnt, scan);
        if (p < pairs)
            indptr[p] = (int32_t)(carry + incl - cnt);
        if (tid == kBuildThreads - 1)
            total = carry + incl;
        __syncthreads();
        carry = total;
        __syncthreads();
    }
    const int64_t n_items = carry;
    if (tid == 0)
        indptr[pairs] = (int32_t)n_items;
    __syncthreads();  // the offsets are visible to every thread
    // The items, one thread per item: item k of pair p covers the pair's pages
    // [x_k, x_{k+1}) of share b_k; when every share holds a page (U >= T) the
    // pair's owners are consecutive, b_k = b_0 + k and x_k = max(a, start(b_k)),
    // otherwise every share holds at most one page and item k is page a + k.
    // Each item also sets the block offsets of the shares after the previous
    // item's owner up to its own.
    auto item_owner = [&](int64_t a, int64_t n, int64_t k) {
        if (n == 0)
            return share_owner(U, T, a);
        return U >= T ? share_owner(U, T, a) + k : share_owner(U, T, a + k);
    };
    for (int64_t idx = tid; idx < n_items; idx += kBuildThreads) {
        int64_t lo = 0, hi = pairs - 1;  // the pair: the last offset <= idx (offsets rise strictly)
        while (lo < hi) {
            const int64_t mid = (lo + hi + 1) / 2;
            if (indptr[mid] <= idx)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t p = lo;
        const int64_t k = idx - indptr[p];
        int64_t a, n;
        pair_span(p, a, n);
        const int i = (int)(p / H_kv), h = (int)(p % H_kv);
        const int64_t b = item_owner(a, n, k);
        int4 it = make_int4(i, h, 0, 0);
        if (n > 0) {
            const int64_t N = clamped_len(i);
            int64_t x, y;
            if (U >= T) {
                x = k == 0 ? a : share_start(U, T, b);
                const int64_t end = share_start(U, T, b + 1);
                y = a + n < end ? a + n : end;
            } else {
                x = a + k;
                y = x + 1;
            }
            it.z = (int)((x - a) * P);
            it.w = (int)((y - a) * P < N ? (y - a) * P : N);
        }
        if (idx < capacity)
            items[idx] = it;
        else
            atomicOr(err, kErrItem);
        const int64_t prev = k > 0 ? item_owner(a, n, k - 1) : (p == 0 ? -1 : last_owner(p - 1));
        for (int64_t c = prev + 1; c <= b; ++c)
            block_ptr[c] = (int32_t)idx;
        if (idx == n_items - 1)
            for (int64_t c = b + 1; c <= T; ++c)
                block_ptr[c] = (int32_t)n_items;
    }
}

// The compact queue whose chunk fills one wave of T blocks, built on the
// device: the same items and pair offsets as pkv_select_policy's fill rule
// followed by pkv_build_work_queue.  C is the smallest chunk (in pages) with
// H_kv * sum_i max(1, ceil(pages_i / C)) <= T, found by bisection over block
// sums (the count only falls as C grows), or the longest row's page count
// when whole rows already exceed T.
__global__ void __launch_bounds__(kBuildThreads)
    fill_queue_kernel(const int32_t *lens, int32_t B, int32_t H_kv, int32_t P, int32_t max_pages, int32_t T,
                      int4 *items, int32_t capacity, int32_t *indptr, uint32_t *err)
{
    __shared__ int32_t pages[kBuildMaxRows];
    // items of one head's rows before row i (the whole queue is bounded by the
    // int32 capacity, so 32 bits hold it)
    __shared__ int32_t row_start[kBuildMaxRows + 1];
    __shared__ int64_t scan[kBuildWarps];
    __shared__ int64_t total;
    grid_dependency_wait();
    grid_launch_dependents();
    const int tid = threadIdx.x;
    const int64_t cap_tokens = (int64_t)max_pages * P;
    auto clamped_len = [&](int i) {
        int64_t N = lens[i];
        if (N < 0 || N > cap_tokens) {
            atomicOr(err, kErrSeqLen);
            N = N < 0 ? 0 : cap_tokens;
        }
        return N;
    };
    int64_t pmax = 0;
    for (int i = tid; i < B; i += kBuildThreads) {
        pages[i] = (int32_t)((clamped_len(i) + P - 1) / P);
        pmax = pmax > pages[i] ? pmax : pages[i];
    }
    __syncthreads();  // pages[] complete
    int64_t pages_max = block_max(pmax, scan);
    pages_max = pages_max > 0 ? pages_max : 1;
    // items of one head at chunk size C, summed over the block
    auto head_items = [&](int64_t C) {
        int64_t n = 0;
        for (int i = tid; i < B; i += kBuildThreads) {
            const int64_t c = (pages[i] + C - 1) / C;
            n += c > 1 ? c : 1;
        }
        return block_sum(n, scan);
    };
    int64_t C = pages_max;
    if (head_items(pages_max) * H_kv <= T) {
        int64_t lo = 1, hi = pages_max;
        while (lo < hi) {
            const int64_t mid = lo + (hi - lo) / 2;
            if (head_items(mid) * H_kv <= T)
                hi = mid;
            else
                lo = mid + 1;
        }
        C = lo;
    }
    // row offsets of the items (one head), then every pair's items
    int64_t carry = 0;
    for (int base = 0; base < B; base += kBuildThreads) {
        const int i = base + tid;
        int64_t cnt = 0;
        if (i < B) {
            cnt = (pages[i] + C - 1) / C;
            cnt = cnt > 1 ? cnt : 1;
        }
        const int64_t incl = block_inclusive_scan(cnt, scan);
        if (i < B)
            row_start[i] = (int32_t)(carry + incl - cnt);
        if (tid == kBuildThreads - 1)
            total = carry + incl;
        __syncthreads();
        carry = total;
        __syncthreads();
    }
    if (tid == 0)
        row_start[B] = (int32_t)carry;
    __syncthreads();
    const int64_t pairs = (int64_t)B * H_kv;
    const int64_t span = C * P;
    for (int64_t p = tid; p < pairs; p += kBuildThreads) {
        const int i = (int)(p / H_kv), h = (int)(p % H_kv);
        const int64_t cnt = (int64_t)row_start[i + 1] - row_start[i];
        const int64_t o = (int64_t)row_start[i] * H_kv + h * cnt;
        indptr[p] = (int32_t)o;
        const int64_t N = pages[i] == 0 ? 0 : clamped_len(i);
        for (int64_t c = 0; c < cnt; ++c) {
            int4 it = make_int4(i, h, 0, 0);
            if (N > 0) {
                it.z = (int)(c * span);
                it.w = (int)((c + 1) * span < N ? (c + 1) * span : N);
            }
            if (o + c < capacity)
                items[o + c] = it;
            else
                atomicOr(err, kErrItem);
        }
    }
    if (tid == 0)
        indptr[pairs] = (int32_t)(carry * H_kv);
}

// ---------------------------------------------------------------------------
// Host side

namespace {

// Block shapes: kNW consumer warps and a ring of kNST pages (three blocks fit
// per SM), or the deep ring of kNSTDeep pages (two blocks per SM, more bytes in
// flight per block; chosen per plan with PKV_FLAG_DEEP_RING).
#ifndef PKV_NW
#define PKV_NW 4
#endif
#ifndef PKV_NST
#define PKV_NST 8
#endif
#ifndef PKV_NST_DEEP
#define PKV_NST_DEEP 12
#endif
constexpr int kNW = PKV_NW;
constexpr int kNST = PKV_NST;
constexpr int kNSTDeep = PKV_NST_DEEP;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

struct MapKey {
    const void *base;
    int64_t dims[4];
    int64_t strides[3];
    bool operator==(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

// Tensor maps are pure host encodings; a small cache saves re-encoding the
// same pool every step.
int pool_tensor_map(CUtensorMap *out, const void *base, const pkv_shape &s)
{
    static std::mutex mu;
    static MapKey keys[8];
    static CUtensorMap maps[8];
    static int used = 0, next = 0;
    MapKey key;
    std::memset(&key, 0, sizeof key);
    key.base = base;
    key.dims[0] = s.head_dim;
    key.dims[1] = s.page_size;
    key.dims[2] = s.H_kv;
    key.dims[3] = s.num_pool_pages;
    key.strides[0] = s.kv_stride_token * 2;
    key.strides[1] = s.kv_stride_head * 2;
    key.strides[2] = s.kv_stride_page * 2;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (keys[i] == key) {
                *out = maps[i];
                return PKV_OK;
            }
    }
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return PKV_ERR_CUDA;
    CUtensorMap tm;
#if PKV_TMA_5D
    // [pages][H_kv][d_hi][P][64] view: one box = one whole (page, head) block,
    // laid out [d_hi][token][64 d] in shared memory like two rank-4 boxes.
    cuuint64_t dims[5] = {(cuuint64_t)kBoxD, (cuuint64_t)s.page_size, (cuuint64_t)(s.head_dim / kBoxD),
                          (cuuint64_t)s.H_kv, (cuuint64_t)s.num_pool_pages};
    cuuint64_t strides[4] = {(cuuint64_t)key.strides[0], (cuuint64_t)(kBoxD * 2), (cuuint64_t)key.strides[1],
                             (cuuint64_t)key.strides[2]};
    cuuint32_t box[5] = {(cuuint32_t)kBoxD, (cuuint32_t)s.page_size, (cuuint32_t)(s.head_dim / kBoxD), 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult rc = enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
#else
    cuuint64_t dims[4], strides[3];
    for (int i = 0; i < 4; ++i)
        dims[i] = (cuuint64_t)key.dims[i];
    for (int i = 0; i < 3; ++i)
        strides[i] = (cuuint64_t)key.strides[i];
    cuuint32_t box[4] = {(cuuint32_t)kBoxD, (cuuint32_t)s.page_size, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult rc = enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
#endif
    if (rc != CUDA_SUCCESS)
        return PKV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    keys[next] = key;
    maps[next] = tm;
    next = (next + 1) % 8;
    if (used < 8)
        ++used;
    *out = tm;
    return PKV_OK;
}

// Largest dynamic shared memory a block may request (227 KiB on sm_100).
constexpr int kMaxDynSmem = 227 * 1024;

// cudaFuncSetAttribute is per kernel and per device; `done_mask` (one per
// kernel instantiation) remembers the devices already configured.
template <typename K>
cudaError_t set_smem(K kernel, int bytes, std::atomic<uint64_t> &done_mask)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (bit && (done_mask.load() & bit))
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit)
        done_mask.fetch_or(bit);
    return e;
}

// Launch geometry of one kernel instantiation on one device: its blocks
// per SM at its own shared-memory size, the SM count and the shared memory
// an SM offers (per-block reservation included).
struct Occupancy {
    int per_sm = 0, sms = 0, smem_per_sm = 0, reserved = 0;
};

template <typename K>
Occupancy occupancy(K kernel, int threads, int smem, std::atomic<uint64_t> (&cache)[64])
{
    Occupancy o;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return o;
    uint64_t packed = cache[dev].load();
    if (packed == 0) {
        int per_sm = 0, sms = 0, smem_sm = 0, reserved = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            return o;
        packed = (uint64_t)(per_sm & 0xff) | ((uint64_t)(sms & 0xffff) << 8) | ((uint64_t)(reserved & 0xffff) << 24) |
                 ((uint64_t)(smem_sm & 0xffffff) << 40);
        cache[dev].store(packed);
    }
    o.per_sm = (int)(packed & 0xff);
    o.sms = (int)((packed >> 8) & 0xffff);
    o.reserved = (int)((packed >> 24) & 0xffff);
    o.smem_per_sm = (int)((packed >> 40) & 0xffffff);
    return o;
}

// Dynamic shared memory to launch a grid with.  A grid that fits in fewer
// blocks per SM than the kernel allows gets just enough extra shared memory
// that no SM can hold more than ceil(grid / SMs) of its blocks, so the
// blocks spread over every SM instead of piling onto some of them.  Timed
// on B200: a one-wave work-queue grid (216 blocks) ran about 1 us faster per
// step spread two per SM than where three per SM were allowed.
int spread_smem(const Occupancy &o, int smem, int64_t grid)
{
    if (o.sms <= 0 || o.per_sm <= 1)
        return smem;
    const int64_t want = (grid + o.sms - 1) / o.sms;
    if (want >= o.per_sm)
        return smem;
    const int t = want < 1 ? 1 : (int)want;
    // t + 1 blocks of this size no longer fit in the SM's shared memory
    const int padded = o.smem_per_sm / (t + 1) - o.reserved + 16;
    return padded > smem && padded <= kMaxDynSmem ? padded : smem;
}

template <typename... Args>
cudaError_t launch_ex(void (*kernel)(Args...), unsigned grid, unsigned block, size_t smem, cudaStream_t st, bool pdl,
                      const Params &prm, unsigned cluster = 0)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, prm);
}

template <int D, int NT, int NST, bool CL, bool FILL>
cudaError_t launch_split(const Params &prm, int64_t grid, cudaStream_t st, bool pdl, unsigned cluster)
{
    using C = Cfg<D, NT, kNW, NST>;
    static std::atomic<uint64_t> configured{0};
    auto kernel = split_kernel<D, NT, kNW, NST, CL, FILL>;
    cudaError_t e = set_smem(kernel, kMaxDynSmem, configured);
    if (e != cudaSuccess)
        return e;
    if (CL && cluster > 8) {
        static std::atomic<uint64_t> wide{0};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess)
            return e;
        const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
        if (!(bit && (wide.load() & bit))) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess)
                return e;
            wide.fetch_or(bit);
        }
    }
    static std::atomic<uint64_t> occ_cache[64] = {};
    const Occupancy o = occupancy(kernel, C::kThreads, C::kSmemBytes, occ_cache);
    const int smem = CL ? C::kSmemBytes : spread_smem(o, C::kSmemBytes, grid);
    Params q = prm;
    q.prefetch_blocks = o.per_sm * o.sms;  // the first wave (see l2_prefetch_first_pages)
    e = launch_ex(kernel, (unsigned)grid, C::kThreads, smem, st, pdl, q, CL ? cluster : 0);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int NST, bool CL, bool FILL>
cudaError_t launch_split_nst(int D, int NT, const Params &prm, int64_t grid, cudaStream_t st, bool pdl,
                             unsigned cluster)
{
    if (D == 128) {
        if (NT == 1)
            return launch_split<128, 1, NST, CL, FILL>(prm, grid, st, pdl, cluster);
        if constexpr (NST >= 12)
            return launch_split<128, 2, NST, CL, FILL>(prm, grid, st, pdl, cluster);
        else
            return cudaErrorInvalidConfiguration;  // launch_split_any gives this tile the deep ring
    }
    return NT == 1 ? launch_split<64, 1, NST, CL, FILL>(prm, grid, st, pdl, cluster)
                   : launch_split<64, 2, NST, CL, FILL>(prm, grid, st, pdl, cluster);
}

#ifndef PKV_NST_BAL
#define PKV_NST_BAL 8
#endif
#ifndef PKV_NST_BAL_DEEP
#define PKV_NST_BAL_DEEP 20
#endif

template <int D, int NT, int NST>
cudaError_t launch_balanced(const Params &prm, int64_t grid, cudaStream_t st, bool pdl)
{
    using C = BCfg<D, NT, kNW, NST>;
    static std::atomic<uint64_t> configured{0};
    auto kernel = balanced_kernel<D, NT, kNW, NST>;
    cudaError_t e = set_smem(kernel, kMaxDynSmem, configured);
    if (e != cudaSuccess)
        return e;
    static std::atomic<uint64_t> occ_cache[64] = {};
    const Occupancy o = occupancy(kernel, C::kThreads, C::kSmemBytes, occ_cache);
    Params q = prm;
    q.prefetch_blocks = o.per_sm * o.sms;
    e = launch_ex(kernel, (unsigned)grid, C::kThreads, spread_smem(o, C::kSmemBytes, grid), st, pdl, q);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int NST>
cudaError_t launch_balanced_nst(int D, int NT, const Params &prm, int64_t grid, cudaStream_t st, bool pdl)
{
    if (D == 128)
        return NT == 1 ? launch_balanced<128, 1, NST>(prm, grid, st, pdl)
                       : launch_balanced<128, 2, NST>(prm, grid, st, pdl);
    return NT == 1 ? launch_balanced<64, 1, NST>(prm, grid, st, pdl) : launch_balanced<64, 2, NST>(prm, grid, st, pdl);
}

template <int D, int NST>
cudaError_t launch_prefix(const Params &prm, int64_t grid, cudaStream_t st, bool pdl)
{
    using C = Cfg<D, 2, kNW, NST>;
    static std::atomic<uint64_t> configured{0};
    auto kernel = prefix_kernel<D, kNW, NST>;
    cudaError_t e = set_smem(kernel, kMaxDynSmem, configured);
    if (e != cudaSuccess)
        return e;
    static std::atomic<uint64_t> occ_cache[64] = {};
    const Occupancy o = occupancy(kernel, C::kThreads, C::kSmemBytes + kPrefixSmemExtra, occ_cache);
    Params q = prm;
    q.prefetch_blocks = o.per_sm * o.sms;
    e = launch_ex(kernel, (unsigned)grid, C::kThreads, spread_smem(o, C::kSmemBytes + kPrefixSmemExtra, grid), st,
                  pdl, q);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// The prefix grid always runs the 12-page ring: its 16-column tile needs
// about 190 registers, and only the deep variant's launch bounds (two blocks
// per SM) keep two blocks resident; with the 8-page ring one block per SM ran
// a 64-row batch 1.6x slower than the split kernel.
cudaError_t launch_prefix_any(int D, const Params &prm, int64_t grid, cudaStream_t st, bool pdl)
{
    return D == 128 ? launch_prefix<128, kNSTDeep>(prm, grid, st, pdl) : launch_prefix<64, kNSTDeep>(prm, grid, st, pdl);
}

// Head dim 128 with the 16-column tile (G > 8) also takes the 12-page ring
// whatever the plan's flags say: with the 8-page ring's launch bounds it needs
// 193 registers, which leaves one block per SM.
cudaError_t launch_split_any(int D, int NT, bool deep, const Params &prm, int64_t grid, cudaStream_t st, bool pdl,
                             unsigned cluster)
{
    deep = deep || (D == 128 && NT == 2);
    if (cluster > 0)
        return deep ? launch_split_nst<kNSTDeep, true, false>(D, NT, prm, grid, st, pdl, cluster)
                    : launch_split_nst<kNST, true, false>(D, NT, prm, grid, st, pdl, cluster);
    if (prm.device_fill)
        return deep ? launch_split_nst<kNSTDeep, false, true>(D, NT, prm, grid, st, pdl, 0)
                    : launch_split_nst<kNST, false, true>(D, NT, prm, grid, st, pdl, 0);
    return deep ? launch_split_nst<kNSTDeep, false, false>(D, NT, prm, grid, st, pdl, 0)
                : launch_split_nst<kNST, false, false>(D, NT, prm, grid, st, pdl, 0);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_fast_path(const pkv_shape &s)
{
    const int G = s.H_q / s.H_kv;
    if (s.page_size != kPage || (s.head_dim != 64 && s.head_dim != 128) || G < 1 || G > 16)
        return PKV_ERR_UNSUPPORTED;
    if (s.kv_stride_token % 8 || s.kv_stride_head % 8 || s.kv_stride_page % 8 || s.kv_stride_token <= 0 ||
        s.kv_stride_head <= 0 || s.kv_stride_page <= 0)
        return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}

}  // namespace

// Device addresses of the workspace sections (error word, completion
// counters, partial states); normally carved out of one workspace by
// ws_layout, placed one by one by pkv_decode_host.
struct WsPtrs {
    uint32_t *error;
    uint32_t *counters;
    float *m, *l, *acc;
    uint32_t *host_err = nullptr;  // flag words in mapped host memory (pkv_decode_host), or NULL
};

// Internal entry shared by pkv_paged_decode, pkv_paged_decode_noalloc and
// pkv_decode_host.  With `sections` NULL the workspace sections are carved
// out of `workspace` (checked against workspace_bytes); otherwise they are
// taken from `sections` and workspace/workspace_bytes are ignored.  With
// zero_bytes > 0 the first zero_bytes of the workspace (error word and
// completion counters) are cleared on the stream once every argument check
// has passed, right before the launch, so a rejected call queues nothing.
int paged_decode_impl(const void *q, const void *k_pool, const void *v_pool, const int32_t *block_table,
                      const int32_t *seq_lens, int32_t page_size, float scale, void *out, const pkv_shape *shape,
                      const pkv_plan *plan, const pkv_work_item *items, const int32_t *indptr, int32_t n_items,
                      void *workspace, size_t workspace_bytes, cudaStream_t st, const WsPtrs *sections = nullptr,
                      size_t zero_bytes = 0)
{
    if (check_shape(shape) != PKV_OK || !plan || page_size != shape->page_size)
        return PKV_ERR_INVALID;
    const pkv_shape &s = *shape;
    const pkv_plan &pl = *plan;
    if (pl.mode != PKV_NO_SPLIT && pl.mode != PKV_SPLIT_S && pl.mode != PKV_WORK_QUEUE && pl.mode != PKV_BALANCED)
        return PKV_ERR_INVALID;
    if (pl.mode == PKV_SPLIT_S && (pl.num_splits < 1 || pl.chunk_pages < 1))
        return PKV_ERR_INVALID;
    const bool device_fill = (pl.flags & PKV_FLAG_DEVICE_FILL) != 0;
    const bool shared_prefix = (pl.flags & PKV_FLAG_SHARED_PREFIX) != 0;
    if (shared_prefix) {
        // the prefix-sharing queue: num_splits carries the unit count (the grid)
        if (pl.mode != PKV_WORK_QUEUE || device_fill || (pl.flags & PKV_FLAG_PDL_EARLY))
            return PKV_ERR_UNSUPPORTED;
        if (!items || !indptr || n_items < (int64_t)s.B * s.H_kv || pl.num_splits < 1 || pl.num_splits > n_items)
            return PKV_ERR_INVALID;
    } else if (device_fill) {
        // each block derives its item: the grid must hold the longest queue the fill rule allows
        if (pl.mode != PKV_WORK_QUEUE || (pl.flags & PKV_FLAG_SEPARATE_MERGE) || s.B > kFillMaxRows)
            return PKV_ERR_UNSUPPORTED;
        if (pl.num_splits < 1 || pl.chunk_pages != 0)
            return PKV_ERR_INVALID;
        if ((int64_t)s.B * s.max_pages_per_seq * s.H_kv > INT32_MAX)
            return PKV_ERR_UNSUPPORTED;
        if (n_items < std::max<int64_t>(pl.num_splits, (int64_t)s.B * s.H_kv))
            return PKV_ERR_INVALID;
    } else if ((pl.mode == PKV_WORK_QUEUE || pl.mode == PKV_BALANCED) &&
               (!items || !indptr || n_items < (int64_t)s.B * s.H_kv)) {
        return PKV_ERR_INVALID;
    }
    if (pl.mode == PKV_BALANCED && pl.num_splits < 1)
        return PKV_ERR_INVALID;
    if ((pl.flags & PKV_FLAG_CLUSTER_MERGE) && (pl.mode != PKV_SPLIT_S || pl.num_splits > 16))
        return PKV_ERR_UNSUPPORTED;
    int rc = check_fast_path(s);
    if (rc != PKV_OK)
        return rc;
    if (s.B == 0)
        return PKV_OK;
    if (!q || !k_pool || !v_pool || !seq_lens || !out || (!workspace && !sections) ||
        (!block_table && s.max_pages_per_seq > 0))
        return PKV_ERR_INVALID;
    if (s.num_pool_pages < 1 || s.max_pages_per_seq < 1)
        return PKV_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        (!sections && !aligned(workspace, 256)) || !aligned(block_table, 4) || !aligned(seq_lens, 4) ||
        (items && !aligned(items, 16)) || (indptr && !aligned(indptr, 4)))
        return PKV_ERR_UNSUPPORTED;
    WsPtrs wp;
    if (sections) {
        wp = *sections;
    } else {
        const WsLayout ws = ws_layout(s, pl, n_items);
        if (workspace_bytes < ws.total)
            return PKV_ERR_CAPACITY;
        uint8_t *wsb = static_cast<uint8_t *>(workspace);
        wp.error = reinterpret_cast<uint32_t *>(wsb + ws.error_off);
        wp.counters = reinterpret_cast<uint32_t *>(wsb + ws.counters_off);
        wp.m = reinterpret_cast<float *>(wsb + ws.m_off);
        wp.l = reinterpret_cast<float *>(wsb + ws.l_off);
        wp.acc = reinterpret_cast<float *>(wsb + ws.acc_off);
    }

    Params prm;
    std::memset(&prm, 0, sizeof prm);
    if ((rc = pool_tensor_map(&prm.tm_k, k_pool, s)) != PKV_OK)
        return rc;
    if ((rc = pool_tensor_map(&prm.tm_v, v_pool, s)) != PKV_OK)
        return rc;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.block_table = block_table;
    prm.seq_lens = seq_lens;
    prm.items = reinterpret_cast<const int4 *>(items);
    prm.indptr = indptr;
    prm.ws_error = wp.error;
    prm.host_err = wp.host_err;
    prm.ws_counters = wp.counters;
    prm.ws_m = wp.m;
    prm.ws_l = wp.l;
    prm.ws_acc = wp.acc;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.B = s.B;
    prm.H_q = s.H_q;
    prm.H_kv = s.H_kv;
    prm.G = s.H_q / s.H_kv;
    prm.max_pages = s.max_pages_per_seq;
    prm.num_pool_pages = s.num_pool_pages;
    prm.mode = pl.mode;
    prm.num_splits = pl.mode == PKV_SPLIT_S ? pl.num_splits : 1;
    prm.chunk_pages = pl.chunk_pages;
    prm.separate_merge = (pl.flags & PKV_FLAG_SEPARATE_MERGE) ? 1 : 0;
    prm.pdl_early = (pl.flags & PKV_FLAG_PDL_EARLY) && !(pl.flags & PKV_FLAG_NO_PDL) ? 1 : 0;
    prm.n_items = n_items;
    prm.device_fill = device_fill ? 1 : 0;
    prm.n_units = shared_prefix ? pl.num_splits : 0;
    prm.fill_blocks = device_fill ? pl.num_splits : 0;
#ifdef PKV_TRACE
    static std::atomic<int32_t> trace_launches{0};
    prm.trace_epoch = trace_launches.fetch_add(1);
#endif

    const int64_t pairs = (int64_t)s.B * s.H_kv;
    const int64_t grid = pl.mode == PKV_NO_SPLIT ? pairs
                         : pl.mode == PKV_SPLIT_S ? pairs * pl.num_splits
                         : pl.mode == PKV_BALANCED || shared_prefix ? (int64_t)pl.num_splits
                                                                     : n_items;
    if (grid > INT32_MAX || pairs > INT32_MAX)
        return PKV_ERR_UNSUPPORTED;
    const int NT = prm.G <= 8 ? 1 : 2;
    const bool pdl = (pl.flags & PKV_FLAG_NO_PDL) == 0;
    const bool deep = (pl.flags & PKV_FLAG_DEEP_RING) != 0;
    // cluster merge: the S blocks of each (row, KV head) form one cluster
    const unsigned cluster = (pl.flags & PKV_FLAG_CLUSTER_MERGE) ? (unsigned)pl.num_splits : 0u;
    if (zero_bytes > 0 && cudaMemsetAsync(wp.error, 0, zero_bytes, st) != cudaSuccess)
        return PKV_ERR_CUDA;
    cudaError_t le;
    if (pl.mode == PKV_BALANCED)
        le = deep ? launch_balanced_nst<PKV_NST_BAL_DEEP>(s.head_dim, NT, prm, grid, st, pdl)
                  : launch_balanced_nst<PKV_NST_BAL>(s.head_dim, NT, prm, grid, st, pdl);
    else if (shared_prefix)
        le = launch_prefix_any(s.head_dim, prm, grid, st, pdl);
    else
        le = launch_split_any(s.head_dim, NT, deep, prm, grid, st, pdl, cluster);
    if (le != cudaSuccess)
        return PKV_ERR_CUDA;
    const bool need_merge = pl.mode != PKV_NO_SPLIT && prm.separate_merge && cluster == 0;
    if (need_merge) {
        cudaError_t e = s.head_dim == 128
                            ? launch_ex(merge_kernel<128>, (unsigned)pairs, kMergeThreads, 0, st, pdl, prm)
                            : launch_ex(merge_kernel<64>, (unsigned)pairs, kMergeThreads, 0, st, pdl, prm);
        if (e != cudaSuccess || cudaGetLastError() != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

int status_from_error_word(uint32_t w)
{
    if (w & kErrTimeout)
        return PKV_ERR_TIMEOUT;
    if (w)
        return PKV_ERR_DEVICE_INPUT;
    return PKV_OK;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_paged_decode(const void *q, const void *k_pool, const void *v_pool, const int32_t *block_table,
                     const int32_t *seq_lens, int32_t page_size, float scale, void *out, const pkv_shape *shape,
                     const pkv_plan *plan, const pkv_work_item *items, const int32_t *indptr, int32_t n_items,
                     void *workspace, size_t workspace_bytes, void *stream)
{
    return paged_decode_impl(q, k_pool, v_pool, block_table, seq_lens, page_size, scale, out, shape, plan, items,
                             indptr, n_items, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

#ifdef PKV_TRACE
// Copy the timeline of the first blocks (16 uint64 per block) to the host.
__attribute__((visibility("default"))) int pkv_trace_read(void *host, size_t bytes)
{
    return cudaMemcpyFromSymbol(host, g_pkv_trace_buf, bytes) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
#endif

int pkv_build_balanced_queue_device(const int32_t *seq_lens, const pkv_shape *shape, int32_t n_blocks,
                                    pkv_work_item *items, int32_t capacity, int32_t *indptr, void *workspace,
                                    void *stream)
{
    int32_t need = 0;
    int rc = pkv_balanced_queue_capacity(shape, n_blocks, &need);
    if (rc != PKV_OK)
        return rc;
    const pkv_shape &s = *shape;
    if (s.B == 0)
        return PKV_OK;
    if (s.B > kBuildMaxRows)
        return PKV_ERR_UNSUPPORTED;
    if (capacity < need)
        return PKV_ERR_CAPACITY;
    if (!seq_lens || !items || !indptr || !workspace)
        return PKV_ERR_INVALID;
    if (!aligned(items, 16) || !aligned(indptr, 4) || !aligned(seq_lens, 4) || !aligned(workspace, 256))
        return PKV_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kBuildThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, balanced_queue_kernel, seq_lens, s.B, s.H_kv, s.page_size,
                                             s.max_pages_per_seq, n_blocks, reinterpret_cast<int4 *>(items),
                                             capacity, indptr, static_cast<uint32_t *>(workspace));
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_build_fill_queue_device(const int32_t *seq_lens, const pkv_shape *shape, int32_t n_blocks,
                                pkv_work_item *items, int32_t capacity, int32_t *indptr, void *workspace,
                                void *stream)
{
    int32_t need = 0;
    int rc = pkv_fill_queue_capacity(shape, n_blocks, &need);
    if (rc != PKV_OK)
        return rc;
    const pkv_shape &s = *shape;
    if (s.B == 0)
        return PKV_OK;
    if (s.B > kBuildMaxRows)
        return PKV_ERR_UNSUPPORTED;
    if (capacity < need)
        return PKV_ERR_CAPACITY;
    if (!seq_lens || !items || !indptr || !workspace)
        return PKV_ERR_INVALID;
    if (!aligned(items, 16) || !aligned(indptr, 4) || !aligned(seq_lens, 4) || !aligned(workspace, 256))
        return PKV_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kBuildThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fill_queue_kernel, seq_lens, s.B, s.H_kv, s.page_size,
                                             s.max_pages_per_seq, n_blocks, reinterpret_cast<int4 *>(items),
                                             capacity, indptr, static_cast<uint32_t *>(workspace));
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_selftest_wait_timeout(void *workspace, size_t workspace_bytes, uint32_t limit_us, void *stream)
{
    if (!workspace || workspace_bytes < kWsAlign || limit_us == 0 || limit_us > 1000000u)
        return PKV_ERR_INVALID;
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint32_t *>(workspace), (uint64_t)limit_us * 1000u);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace || workspace_bytes < kWsAlign)
        return PKV_ERR_INVALID;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

int pkv_workspace_status(const void *workspace, void *stream, int32_t *device_error)
{
    if (!workspace)
        return PKV_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t w = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (cudaMemcpy(&w, workspace, sizeof w, cudaMemcpyDeviceToHost) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (device_error)
        *device_error = (int32_t)w;
    return status_from_error_word(w);
}

namespace {

// ---------------------------------------------------------------------------
// Scratch for pkv_paged_decode_noalloc: a fixed array in the library's device
// image, so that callers without an allocator can still run split plans.
// Every GPU that loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current CUDA context.  In host
// code the symbol is only a host-side handle: the address is looked up with
// cudaGetSymbolAddress (the device in question current) the first time a
// context calls, and cached per context, so a caller that makes a context of
// its own current on the same device gets that context's copy.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

void *noalloc_scratch_address()
{
    static std::mutex mu;
    static CUcontext ctxs[64] = {};
    static void *addrs[64] = {};
    static int used = 0;
    CtxGetCurrentFn current = ctx_get_current();
    if (!current)
        return nullptr;
    CUcontext ctx = nullptr;
    if (current(&ctx) != CUDA_SUCCESS)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; ctx && i < used; ++i)
        if (ctxs[i] == ctx)
            return addrs[i];
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
        return nullptr;
    // the lookup makes the device's primary context current if none was
    if (!ctx && (current(&ctx) != CUDA_SUCCESS || !ctx))
        return ptr;
    const int slot = used < 64 ? used++ : 63;
    ctxs[slot] = ctx;
    addrs[slot] = ptr;
    return ptr;
}

// pkv_decode_host moves a step's inputs in one host->device copy and its
// result in one device->host copy.  The device buffer is laid out so that the
// inputs and the zeroed error word / completion counters form one contiguous
// upload, and the error word and `out` one contiguous download:
//
//   [q*] [seq_lens] [items] [indptr] [block_table*] [counters] [error] [out*] [m] [l] [acc] [q**] [block_table**]
//   '------------------------ upload --------------------------------'
//                                                           '-- download --'
//
// The host staging buffer holds the same upload image, then the download.
// q, block_table and out travel inside the packed copies (*) up to
// kInlineBytes each; larger ones are copied straight from / to the caller's
// buffers with their own copy (**), where a host-side memcpy into the
// staging buffer would cost more than one extra copy command.
constexpr size_t kInlineBytes = size_t(64) << 10;

struct HostLayout {
    pkv_plan plan;
    int32_t n_items = 0, n_indptr = 0;
    bool q_inline, bt_inline, out_inline;
    size_t q_bytes, bt_bytes;
    size_t q_off, lens_off, items_off, indptr_off, bt_off, counters_off, err_off, out_off, m_off, l_off, acc_off;
    size_t up_bytes, down_bytes, dev_total;
    size_t h_down_off, host_total;
};

// The device address of host memory the GPU can reach (page-locked and
// mapped, as every page-locked allocation is under unified addressing), or
// NULL for any other pointer.
void *device_view(const void *host)
{
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
        cudaGetLastError();  // an unregistered pointer is not an error here
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

// Four timing events per device for pkv_decode_host_timed, made on first use.
cudaEvent_t *timing_events()
{
    static std::mutex mu;
    static cudaEvent_t events[64][4] = {};
    static bool made[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!made[dev]) {
        for (int i = 0; i < 4; ++i)
            if (cudaEventCreate(&events[dev][i]) != cudaSuccess)
                return nullptr;
        made[dev] = true;
    }
    return events[dev];
}

// Everything the work a pkv_decode_host call enqueues depends on, apart from
// the contents of the buffers: calls with equal keys enqueue the same copies
// and launches with the same arguments.
struct HostGraphKey {
    int device;
    const void *dev, *hst, *out_dev, *stage_dev, *k_pool, *v_pool;
    float scale;
    pkv_shape shape;
    pkv_plan plan;
    int32_t n_items;
    size_t up_bytes;
};

// The calling thread's replayable step: a CUDA graph of the upload copy and
// the decode launches, captured the second time in a row that a call comes
// with the same key and replayed while the key stays the same.  A serving
// loop with steady buffers and plan then queues one graph launch per step
// instead of a copy and a kernel launch.
struct HostGraph {
    HostGraphKey key{}, last{};
    bool have_key = false, have_last = false, failed = false;
    cudaGraphExec_t exec = nullptr;
    int64_t replays = 0;
};

HostGraph &host_graph()
{
    static thread_local HostGraph hg;
    return hg;
}

bool same_key(const HostGraphKey &a, const HostGraphKey &b) { return std::memcmp(&a, &b, sizeof a) == 0; }

// A non-blocking stream of the current device to capture on (capture only
// records work, so its stream never runs anything).
cudaStream_t capture_stream(int dev)
{
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    if (dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();
        streams[dev] = nullptr;
    }
    return streams[dev];
}

int host_layout(const int32_t *lens, const pkv_shape *shape, const pkv_policy_rule *rules, int32_t n_rules,
                HostLayout *L)
{
    int rc = pkv_select_policy(lens, shape, rules, n_rules, &L->plan);
    if (rc != PKV_OK)
        return rc;
    const pkv_shape &s = *shape;
    const size_t pairs = (size_t)s.B * s.H_kv;
    L->n_items = 0;
    L->n_indptr = 0;
    if (L->plan.mode == PKV_WORK_QUEUE && (L->plan.flags & PKV_FLAG_DEVICE_FILL)) {
        // no queue travels: the blocks derive their items; the grid holds the longest queue
        L->n_items = (int32_t)std::max<int64_t>(L->plan.num_splits, (int64_t)pairs);
    } else if (L->plan.mode == PKV_WORK_QUEUE) {
        rc = pkv_work_queue_size(lens, shape, L->plan.chunk_pages, &L->n_items);
        L->n_indptr = (int32_t)pairs + 1;
    } else if (L->plan.mode == PKV_BALANCED) {
        rc = pkv_balanced_queue_size(lens, shape, L->plan.num_splits, &L->n_items);
        L->n_indptr = (int32_t)pairs + 2 + L->plan.num_splits;
    }
    if (rc != PKV_OK)
        return rc;
    const WsLayout ws = ws_layout(s, L->plan, L->n_items);
    L->q_bytes = (size_t)s.B * s.H_q * s.head_dim * 2;
    L->bt_bytes = (size_t)s.B * s.max_pages_per_seq * 4;
    L->q_inline = L->q_bytes <= kInlineBytes;
    L->out_inline = L->q_inline;
    L->bt_inline = L->bt_bytes <= kInlineBytes;
    size_t off = 0;
    auto take = [&off](size_t bytes) {
        const size_t at = off;
        off += round_up(bytes, kWsAlign);
        return at;
    };
    L->q_off = L->q_inline ? take(L->q_bytes) : 0;
    L->lens_off = take((size_t)s.B * 4);
    L->items_off = take(L->n_indptr > 0 ? (size_t)L->n_items * sizeof(pkv_work_item) : 0);
    L->indptr_off = take((size_t)L->n_indptr * 4);
    L->bt_off = L->bt_inline ? take(L->bt_bytes) : 0;
    L->counters_off = take(ws.m_off - ws.counters_off);
    L->err_off = take(kWsAlign);
    L->up_bytes = L->err_off + 16;
    L->out_off = take(L->q_bytes);
    L->down_bytes = L->out_inline ? L->out_off + L->q_bytes - L->err_off : 16;
    L->m_off = take(ws.l_off - ws.m_off);
    L->l_off = take(ws.acc_off - ws.l_off);
    L->acc_off = take(ws.total - ws.acc_off);
    if (!L->q_inline)
        L->q_off = take(L->q_bytes);
    if (!L->bt_inline)
        L->bt_off = take(L->bt_bytes);
    L->dev_total = off;
    L->h_down_off = round_up(L->up_bytes, kWsAlign);
    L->host_total = L->h_down_off + round_up(L->down_bytes, kWsAlign);
    return PKV_OK;
}
}  // namespace

int pkv_paged_decode_noalloc(const void *q, const void *k_pool, const void *v_pool, const int32_t *block_table,
                             const int32_t *seq_lens, int32_t page_size, float scale, void *out,
                             const pkv_shape *shape, const pkv_plan *plan, const pkv_work_item *items,
                             const int32_t *indptr, int32_t n_items, void *stream)
{
    if (check_shape(shape) != PKV_OK || !plan || n_items < 0)
        return PKV_ERR_INVALID;
    const WsLayout ws = ws_layout(*shape, *plan, n_items);
    if (ws.total > kNoAllocScratchBytes)
        return PKV_ERR_CAPACITY;  // the plan needs more scratch than the library holds
    if (shape->B == 0)
        return PKV_OK;
    void *scratch = noalloc_scratch_address();
    if (!scratch)
        return PKV_ERR_CUDA;
    // The array keeps whatever the previous call left in it: the error word
    // and the completion counters must start at zero (cleared on the stream
    // after the argument checks, just before the launch), the partial states not.
    return paged_decode_impl(q, k_pool, v_pool, block_table, seq_lens, page_size, scale, out, shape, plan, items,
                             indptr, n_items, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream),
                             nullptr, ws.m_off);
}

int pkv_noalloc_status(void *stream, int32_t *device_error)
{
    void *scratch = noalloc_scratch_address();
    if (!scratch)
        return PKV_ERR_CUDA;
    return pkv_workspace_status(scratch, stream, device_error);
}

int pkv_decode_host_bytes(const int32_t *seq_lens_host, const pkv_shape *shape, const pkv_policy_rule *rules,
                          int32_t n_rules, size_t *device_bytes, size_t *host_bytes)
{
    if (!device_bytes || !host_bytes)
        return PKV_ERR_INVALID;
    HostLayout L;
    int rc = host_layout(seq_lens_host, shape, rules, n_rules, &L);
    if (rc != PKV_OK)
        return rc;
    *device_bytes = L.dev_total;
    *host_bytes = L.host_total;
    return PKV_OK;
}

int pkv_decode_host(const void *q_host, const int32_t *block_table_host, const int32_t *seq_lens_host,
                    void *out_host, const void *k_pool, const void *v_pool, float scale, const pkv_shape *shape,
                    const pkv_policy_rule *rules, int32_t n_rules, void *device_buffer, size_t device_buffer_bytes,
                    void *host_staging, size_t host_staging_bytes, void *stream, pkv_plan *plan_out)
{
    return pkv_decode_host_timed(q_host, block_table_host, seq_lens_host, out_host, k_pool, v_pool, scale, shape,
                                 rules, n_rules, device_buffer, device_buffer_bytes, host_staging,
                                 host_staging_bytes, stream, plan_out, nullptr);
}

int64_t pkv_decode_host_replays(void) { return host_graph().replays; }

int pkv_decode_host_call(const pkv_host_call *c)
{
    if (c == nullptr)
        return PKV_ERR_INVALID;
    return pkv_decode_host_timed(c->q_host, c->block_table_host, c->seq_lens_host, c->out_host, c->k_pool,
                                 c->v_pool, c->scale, c->shape, c->rules, c->n_rules, c->device_buffer,
                                 c->device_buffer_bytes, c->host_staging, c->host_staging_bytes, c->stream,
                                 c->plan_out, c->timing);
}

int pkv_decode_host_timed(const void *q_host, const int32_t *block_table_host, const int32_t *seq_lens_host,
                          void *out_host, const void *k_pool, const void *v_pool, float scale,
                          const pkv_shape *shape, const pkv_policy_rule *rules, int32_t n_rules,
                          void *device_buffer, size_t device_buffer_bytes, void *host_staging,
                          size_t host_staging_bytes, void *stream, pkv_plan *plan_out, pkv_host_timing *timing)
{
    using clock = std::chrono::steady_clock;
    const clock::time_point t0 = clock::now();
    cudaEvent_t *ev = nullptr;
    if (timing) {
        std::memset(timing, 0, sizeof *timing);
        if (!(ev = timing_events()))
            return PKV_ERR_CUDA;
    }
    HostLayout L;
    int rc = host_layout(seq_lens_host, shape, rules, n_rules, &L);
    if (rc != PKV_OK)
        return rc;
    if (plan_out)
        *plan_out = L.plan;
    const pkv_shape &s = *shape;
    if (s.B == 0)
        return PKV_OK;
    if (!q_host || !block_table_host || !out_host || !device_buffer || !host_staging)
        return PKV_ERR_INVALID;
    if (device_buffer_bytes < L.dev_total || host_staging_bytes < L.host_total)
        return PKV_ERR_CAPACITY;
    if (!aligned(device_buffer, kWsAlign))
        return PKV_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *dev = static_cast<uint8_t *>(device_buffer);
    uint8_t *hst = static_cast<uint8_t *>(host_staging);
    // When out_host and the staging buffer are page-locked, the kernels write
    // out straight into out_host and report errors as flag words in the
    // staging buffer: the result needs no device->host copy.
    void *out_dev = device_view(out_host);
    uint8_t *stage_dev = out_dev ? static_cast<uint8_t *>(device_view(hst)) : nullptr;
    const bool direct = out_dev && stage_dev && aligned(out_dev, 16);
    volatile uint32_t *h_flags = reinterpret_cast<volatile uint32_t *>(hst + L.h_down_off);
    if (direct)
        for (int k = 0; k < 4; ++k)
            h_flags[k] = 0u;
    // upload image: inputs, queue, zeroed counters and error word
    if (L.q_inline)
        std::memcpy(hst + L.q_off, q_host, L.q_bytes);
    std::memcpy(hst + L.lens_off, seq_lens_host, (size_t)s.B * 4);
    if (L.bt_inline)
        std::memcpy(hst + L.bt_off, block_table_host, L.bt_bytes);
    std::memset(hst + L.counters_off, 0, L.up_bytes - L.counters_off);
    pkv_work_item *h_items = reinterpret_cast<pkv_work_item *>(hst + L.items_off);
    int32_t *h_indptr = reinterpret_cast<int32_t *>(hst + L.indptr_off);
    int32_t n = 0;
    if (L.plan.mode == PKV_WORK_QUEUE && !(L.plan.flags & PKV_FLAG_DEVICE_FILL))
        rc = pkv_build_work_queue(seq_lens_host, shape, L.plan.chunk_pages, h_items, L.n_items, h_indptr, &n);
    else if (L.plan.mode == PKV_BALANCED)
        rc = pkv_build_balanced_queue(seq_lens_host, shape, L.plan.num_splits, h_items, L.n_items, h_indptr, &n);
    if (rc != PKV_OK)
        return rc;
    const clock::time_point t1 = clock::now();
    uint8_t *h_down = hst + L.h_down_off;
    // The step's device work on stream `ss`, with the timing events when `evs`.
    auto enqueue = [&](cudaStream_t ss, cudaEvent_t *evs) -> int {
        bool ok = !evs || cudaEventRecord(evs[0], ss) == cudaSuccess;
        ok = ok && cudaMemcpyAsync(dev, hst, L.up_bytes, cudaMemcpyHostToDevice, ss) == cudaSuccess;
        if (ok && !L.q_inline)
            ok = cudaMemcpyAsync(dev + L.q_off, q_host, L.q_bytes, cudaMemcpyHostToDevice, ss) == cudaSuccess;
        if (ok && !L.bt_inline)
            ok = cudaMemcpyAsync(dev + L.bt_off, block_table_host, L.bt_bytes, cudaMemcpyHostToDevice, ss) ==
                 cudaSuccess;
        if (ok && evs)
            ok = cudaEventRecord(evs[1], ss) == cudaSuccess;
        if (!ok)
            return PKV_ERR_CUDA;
        const WsPtrs wp{reinterpret_cast<uint32_t *>(dev + L.err_off),
                        reinterpret_cast<uint32_t *>(dev + L.counters_off), reinterpret_cast<float *>(dev + L.m_off),
                        reinterpret_cast<float *>(dev + L.l_off), reinterpret_cast<float *>(dev + L.acc_off),
                        direct ? reinterpret_cast<uint32_t *>(stage_dev + L.h_down_off) : nullptr};
        const int r = paged_decode_impl(dev + L.q_off, k_pool, v_pool, reinterpret_cast<const int32_t *>(dev + L.bt_off),
                                        reinterpret_cast<const int32_t *>(dev + L.lens_off), s.page_size, scale,
                                        direct ? out_dev : dev + L.out_off, shape, &L.plan,
                                        reinterpret_cast<const pkv_work_item *>(dev + L.items_off),
                                        reinterpret_cast<const int32_t *>(dev + L.indptr_off), L.n_items, nullptr, 0,
                                        ss, &wp);
        if (r != PKV_OK)
            return r;
        ok = !evs || cudaEventRecord(evs[2], ss) == cudaSuccess;
        if (!direct) {
            ok = ok &&
                 cudaMemcpyAsync(h_down, dev + L.err_off, L.down_bytes, cudaMemcpyDeviceToHost, ss) == cudaSuccess;
            if (ok && !L.out_inline)
                ok = cudaMemcpyAsync(out_host, dev + L.out_off, L.q_bytes, cudaMemcpyDeviceToHost, ss) ==
                     cudaSuccess;
        }
        if (ok && evs)
            ok = cudaEventRecord(evs[3], ss) == cudaSuccess;
        return ok ? PKV_OK : PKV_ERR_CUDA;
    };
    // Untimed calls whose whole step sits in page-locked buffers replay a
    // graph of it once the same key has come twice in a row.
    HostGraph &hg = host_graph();
    HostGraphKey key;
    std::memset(&key, 0, sizeof key);
    const bool graphable = !ev && direct && L.q_inline && L.bt_inline && cudaGetDevice(&key.device) == cudaSuccess;
    bool launched = false;
    if (graphable) {
        key.dev = dev;
        key.hst = hst;
        key.out_dev = out_dev;
        key.stage_dev = stage_dev;
        key.k_pool = k_pool;
        key.v_pool = v_pool;
        key.scale = scale;
        key.shape = s;
        key.plan = L.plan;
        key.n_items = L.n_items;
        key.up_bytes = L.up_bytes;
        if (!(hg.have_key && same_key(hg.key, key)) && hg.have_last && same_key(hg.last, key)) {
            // second call in a row with this key: capture its step
            cudaGraphExec_t exec = nullptr;
            cudaStream_t cs = capture_stream(key.device);
            if (cs && cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) == cudaSuccess) {
                const int r = enqueue(cs, nullptr);
                cudaGraph_t graph = nullptr;
                const bool ended = cudaStreamEndCapture(cs, &graph) == cudaSuccess;
                if (r == PKV_OK && ended && graph && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess)
                    exec = nullptr;
                if (graph)
                    cudaGraphDestroy(graph);
            }
            cudaGetLastError();  // a step that cannot be captured runs as before
            if (hg.exec)
                cudaGraphExecDestroy(hg.exec);  // freed once any launch of it in flight ends
            hg.exec = exec;
            hg.key = key;
            hg.have_key = true;
            hg.failed = exec == nullptr;
        }
        hg.last = key;
        hg.have_last = true;
        if (hg.have_key && same_key(hg.key, key) && !hg.failed) {
            if (cudaGraphLaunch(hg.exec, st) != cudaSuccess)
                return PKV_ERR_CUDA;
            launched = true;
            ++hg.replays;
        }
    }
    if (!launched && (rc = enqueue(st, ev)) != PKV_OK)
        return rc;
    const clock::time_point t2 = clock::now();
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return PKV_ERR_CUDA;
    const clock::time_point t3 = clock::now();
    uint32_t err = 0;
    if (direct) {
        for (int k = 0; k < 4; ++k)
            err |= h_flags[k] ? (1u << k) : 0u;
    } else {
        if (L.out_inline)
            std::memcpy(out_host, h_down + (L.out_off - L.err_off), L.q_bytes);
        std::memcpy(&err, h_down, 4);
    }
    if (timing) {
        const clock::time_point t4 = clock::now();
        auto us = [](clock::duration d) { return std::chrono::duration<double, std::micro>(d).count(); };
        timing->host_plan_us = us(t1 - t0);
        timing->host_enqueue_us = us(t2 - t1);
        timing->host_wait_us = us(t3 - t2);
        timing->host_unpack_us = us(t4 - t3);
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, ev[0], ev[1]) == cudaSuccess)
            timing->dev_h2d_us = ms * 1e3;
        if (cudaEventElapsedTime(&ms, ev[1], ev[2]) == cudaSuccess)
            timing->dev_kernel_us = ms * 1e3;
        if (cudaEventElapsedTime(&ms, ev[2], ev[3]) == cudaSuccess)
            timing->dev_d2h_us = ms * 1e3;
        timing->host_events_us = us(clock::now() - t4);
    }
    return status_from_error_word(err);
}

}  // extern "C"
