// Shared definitions of the sm_100a MoE kernels: workspace layout, tile
// descriptors, and thin inline-PTX wrappers for mbarrier, TMA (bulk tensor
// copies) and the 5th-generation tensor cores (tcgen05 + tensor memory).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe.h"  // include/ is on the include path

namespace moe {

// ------------------------------------------------------------------ tiling --
constexpr int kScanChunk = 1024;     // routed pairs per histogram / rank block
constexpr int kLookback = 16;        // predecessor chunks read at once by the scan's look-back
constexpr int kScanThreads = 256;
constexpr int kMaxExperts = 256;
constexpr int kTileRows = 256;       // largest UMMA N: most permuted rows a GEMM tile holds
constexpr int kPieceAlign = 16;      // rows of one B-operand TMA box

// Scan look-back state: a 64-bit word per (block, expert): flag << 32 | value.
constexpr uint32_t kFlagAggregate = 1u;
constexpr uint32_t kFlagPrefix = 2u;

// ---------------------------------------------------------------- workspace --
// Byte offsets inside the caller's workspace.  The "reset" range (ticket +
// look-back state) is zeroed by a memset node before every histogram launch;
// the status word lives outside it and is sticky.
struct WsLayout {
    size_t status, num_tiles, total_spill, tile_rows;
    size_t counts, offsets, cap_cnt, spill_cnt, spill_off, order, grp_tile_start;
    size_t chunk_excl;            // int32[nchunks * E] exclusive per-block prefix
    size_t reset_begin;           // start of the memset range
    size_t ticket;                // uint32 dynamic block ticket, then uint32 router completion count
    size_t scan_state;            // uint64[nchunks * E]
    size_t reset_end;
    size_t tile_map;              // int4[max_tiles]
    size_t dispatch_end;          // end of what the dispatch step uses (the router's buffers follow)
    size_t router_planes;         // bf16[3][H][router_plane_cols(E)] (tensor-core router only)
    size_t router_part;           // fp32[q][T][E] partial logits of the K ranges (tensor-core router only)
    size_t combine_cnt;           // int32[T][H/128] arrival counts of the combine fused into the down GEMM
    size_t total;
    int nchunks, max_tiles;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Router logits go to the tensor cores (three bf16 planes of W_r) for large
// batches; below this many tokens the fp32 SIMT router is faster.
constexpr int kTcRouterMinTokens = 2048;
inline bool use_tc_router(int T) { return T >= kTcRouterMinTokens; }
// Columns of one router-weight plane: E rounded up to the 64-column TMA box.
inline int router_plane_cols(int E) { return (E + 63) / 64 * 64; }

// Work split of the tensor-core router.  A unit is `rows` tokens times one
// range of `kb` 64-wide K blocks; the hidden dimension is cut into q ranges
// (each written as a partial-logit plane and added in range order by the
// top-k kernel), and inside a unit the K blocks rotate over `groups`
// accumulators.  Every logit is thus the fixed-order sum of q * groups >=
// kRouteChains independent accumulation chains of at most ceil(H/64/8) K
// blocks each, the accuracy the exact three-plane split needs from the
// tensor cores' fp32 accumulator.  Tokens per unit: as many as one MMA takes
// (256, or 128 with a second 128-expert accumulator), so that each weight
// tile read from L2 feeds the most tokens (256; with a second 128-expert
// accumulator 64, so that two stages of both operands still fit in shared
// memory); the K split then fills the SMs.
constexpr int kRouteChains = 8;
constexpr int kRouteMaxQ = 16;
constexpr int kRoutePlanMaxSms = 160;  // the workspace is sized for up to this many SMs
struct RouterTcPlan {
    int rows, groups, q, kb;
};
inline RouterTcPlan router_tc_plan(int T, int H, int E, int num_sms) {
    const int nacc = E > 128 ? 2 : 1;
    RouterTcPlan p;
    p.rows = nacc == 1 ? 256 : 64;
    p.groups = 512 / (nacc * p.rows);
    if (p.groups > kRouteChains) p.groups = kRouteChains;
    const int nk = H / 64;
    const int ntb = (T + p.rows - 1) / p.rows;
    if (num_sms > kRoutePlanMaxSms) num_sms = kRoutePlanMaxSms;
    const int qmin = (kRouteChains + p.groups - 1) / p.groups;
    int q = num_sms / ntb;
    if (q < qmin) q = qmin;
    if (q > kRouteMaxQ) q = kRouteMaxQ;
    if (q > nk) q = nk;
    if (q < 1) q = 1;
    p.kb = (nk + q - 1) / q;
    p.q = (nk + p.kb - 1) / p.kb;  // no empty range
    return p;
}

// Routed pairs up to which moe_forward lets the router's last CTA build the
// dispatch (histogram, scan, schedule, ranks) instead of separate kernels.
constexpr int kFusedDispatchMaxPairs = 4096;

// Outputs of the dispatch step when the router builds it (see above).
struct FusedDispatch {
    int32_t *counts, *offsets, *src_token, *dest_row;
};

// Inputs and output of the combine when it runs in the down GEMM's epilogue.
struct CombineOut {
    const int32_t *src_token, *dest_row;
    const float *topk_w;
    void *out;
};

inline int64_t permuted_rows(int T, int E, int k, int C, bool capped) {
    if (!capped) return (int64_t)T * k;
    return (int64_t)E * C + (int64_t)k * (T > C ? T - C : 0);
}

// Upper bound on the tiles the schedule builder emits.  Its row cap is either
// below kTileRows, and then every expert fits one tile (<= E tiles), or equal
// to kTileRows; then every tile of an expert but the first holds only
// overflow rows and closes only when full, so an expert needs at most
// 2 + spill/kTileRows tiles (uncapped: 1 + n_e/kTileRows).  Summed:
// 2E + P/kTileRows.
inline int max_tiles_for(int64_t P, int E) { return (int)(2 * (int64_t)E + P / kTileRows + 1); }

inline WsLayout ws_layout(int T, int H, int E, int k, int C, bool capped) {
    WsLayout L{};
    const int64_t R = (int64_t)T * k;
    const int64_t P = permuted_rows(T, E, k, C, capped);
    L.nchunks = (int)((R + kScanChunk - 1) / kScanChunk);
    L.max_tiles = max_tiles_for(P, E);
    size_t o = 0;
    L.status = o;
    L.num_tiles = o + 4;
    L.total_spill = o + 8;
    L.tile_rows = o + 12;
    o += 256;
    auto arr = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    L.counts = arr(4 * (size_t)E);
    L.offsets = arr(4 * (size_t)(E + 1));
    L.cap_cnt = arr(4 * (size_t)E);
    L.spill_cnt = arr(4 * (size_t)E);
    L.spill_off = arr(4 * (size_t)(E + 1));
    L.order = arr(4 * (size_t)E);
    L.grp_tile_start = arr(4 * (size_t)(E + 1));
    L.chunk_excl = arr(4 * (size_t)L.nchunks * E);
    L.reset_begin = o;
    L.ticket = o;
    o += 256;
    L.scan_state = arr(8 * (size_t)L.nchunks * E);
    L.reset_end = o;
    L.tile_map = arr(16 * (size_t)L.max_tiles);
    L.dispatch_end = o;
    L.router_planes = L.router_part = 0;
    if (use_tc_router(T)) {
        L.router_planes = arr(3 * (size_t)H * router_plane_cols(E) * 2);
        // q grows with the SM count: the bound of the largest device planned for
        L.router_part = arr(4 * (size_t)router_tc_plan(T, H, E, kRoutePlanMaxSms).q * T * E);
    }
    // zero after moe_workspace_init; every fused down+combine launch leaves it zero again
    L.combine_cnt = arr(4 * (size_t)T * (H / 128));
    L.total = o;
    return L;
}

// Device-side view of the workspace (pointers resolved on the host).
struct WsPtrs {
    uint32_t *status;
    int *num_tiles, *total_spill, *tile_rows;
    int *counts, *offsets, *cap_cnt, *spill_cnt, *spill_off, *order, *grp_tile_start;
    int *chunk_excl;
    uint32_t *ticket;
    uint32_t *route_done;  // router CTAs that finished their top-k (fused dispatch)
    unsigned long long *scan_state;
    int4 *tile_map;
    int nchunks, max_tiles;
};

inline WsPtrs ws_ptrs(void *ws, const WsLayout &L) {
    char *b = (char *)ws;
    WsPtrs p;
    p.status = (uint32_t *)(b + L.status);
    p.num_tiles = (int *)(b + L.num_tiles);
    p.total_spill = (int *)(b + L.total_spill);
    p.tile_rows = (int *)(b + L.tile_rows);
    p.counts = (int *)(b + L.counts);
    p.offsets = (int *)(b + L.offsets);
    p.cap_cnt = (int *)(b + L.cap_cnt);
    p.spill_cnt = (int *)(b + L.spill_cnt);
    p.spill_off = (int *)(b + L.spill_off);
    p.order = (int *)(b + L.order);
    p.grp_tile_start = (int *)(b + L.grp_tile_start);
    p.chunk_excl = (int *)(b + L.chunk_excl);
    p.ticket = (uint32_t *)(b + L.ticket);
    p.route_done = p.ticket + 1;
    p.scan_state = (unsigned long long *)(b + L.scan_state);
    p.tile_map = (int4 *)(b + L.tile_map);
    p.nchunks = L.nchunks;
    p.max_tiles = L.max_tiles;
    return p;
}

// ------------------------------------------- programmatic dependent launch --
// The kernels after the first one of the layer are launched with the
// programmatic-serialization attribute: such a kernel may be scheduled while
// the kernel before it on the stream is still running, once every CTA of that
// kernel has called pdl_trigger (or exited).  It calls pdl_wait -- which
// returns when the kernel before it has completed and its memory is visible --
// before its first global-memory access, so only its launch and its prologue
// (barrier set-up, tensor-memory allocation, descriptor prefetch) overlap the
// previous kernel.  Launched without the attribute, both calls do nothing.
#if defined(__CUDACC__)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
#endif

// ------------------------------------------------------------ device helpers --
#if defined(__CUDACC__)

// End of a block's stores into other GPUs' memory: a block barrier (every
// thread's stores happen before it), then one system-scope fence by thread 0,
// which is cumulative over them.  All threads of the block call it.
__device__ __forceinline__ void fence_block_stores_system() {
    __syncthreads();
    if (threadIdx.x == 0) __threadfence_system();
}

// One row of H8 16-byte vectors copied by one warp, eight loads per lane in
// flight before their stores (one memory round trip per 4 KB of row).
__device__ __forceinline__ void copy_row_warp(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int H8,
                                              int lane) {
    int v = lane;
    for (; v + 224 < H8; v += 256) {
        uint4 q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __ldg(src + v + 32 * i);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[v + 32 * i] = q[i];
    }
    for (; v < H8; v += 32) dst[v] = __ldg(src + v);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---- cp.async: 16-byte asynchronous global -> shared copies ----
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most `n` of this thread's most recent copy groups are pending.
__device__ __forceinline__ void cp_async_wait_pending(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    }
}

// ---- mbarrier ----
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of parity `parity` to complete.  Gives up (returns
// false) when *abort becomes non-zero or after timeout_ns; the clock is only
// read once the wait has already spun for a while.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                                  volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t deadline = 0;
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 255u) == 0) {
            if (*abort) return false;
            const uint64_t now = globaltimer_ns();
            if (deadline == 0) deadline = now + timeout_ns;
            else if (now > deadline) return false;
        }
    }
}

// ---- TMA: 2-D tiled bulk tensor load into this CTA's shared memory ----
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, uint64_t *bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
// Same, with an L2 cache policy (from createpolicy) for the loaded lines.
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const void *tmap, uint64_t *bar, int x, int y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}
// Four rows (tensor-map row coordinates r0..r3) of one tensor-map box column
// range starting at column x, into 4 consecutive box rows at dst.  The tensor
// map's box must be one row high; with the 128-byte swizzle each row lands in
// its own 128-byte line, swizzled by its shared-memory address.
__device__ __forceinline__ void tma_gather4(void *dst, const void *tmap, uint64_t *bar, int x, int r0, int r1,
                                            int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---- tcgen05: tensor memory and the 5th-generation MMA ----
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrives once on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc], both operands 8-bit floats of the
// kind the instruction descriptor names (kind::f8f6f4), fp32 accumulate;
// K = 32 per instruction.
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 lanes x 32 bits, 16 consecutive columns: register i <- column (col + i)
// of the lane this thread maps to (warp w reads lanes 32*(w%4) .. +31).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// Lanes [l, l + 16) x 16 columns from taddr (lane l in bits 31-16, l a
// multiple of 16 inside the warp's quarter), twice (lanes l and l + 16) in the
// 16x256b layout: with t the thread's lane in the warp, r[8 i + 4 k + e] holds
// tensor-memory lane l + 16 i + (t >> 2) + 8 (e >> 1), column
// 8 k + 2 (t & 3) + (e & 1) -- the m8n8 fragments that stmatrix takes.
__device__ __forceinline__ void tmem_ld_frag16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15])
                 : "r"(taddr + (16u << 16))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Four 8x8 b16 matrices, transposed, into shared memory (thread 8i + j gives
// the address of row j of matrix i).
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Shared-memory matrix descriptor of a tcgen05 operand laid out with the
// 128-byte swizzle: bits 0-13 start address >> 4, 16-29 leading-dimension
// byte offset >> 4, 32-45 stride-dimension byte offset >> 4, 46-47 version
// (1 on sm_100), 61-63 layout (2 = SWIZZLE_128B).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

#endif  // __CUDACC__

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 and 10-12 = 1), A/B major-ness (bit 15 /
// 16: 0 = K-major, 1 = MN-major), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor of tcgen05.mma kind::f8f6f4 with both operands E4M3
// (type code 0 in bits 7-9 and 10-12), both K-major (bits 15, 16 clear), fp32
// accumulator (bits 4-5 = 1), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace moe
