// Expert-parallel dispatch and return by device-initiated peer stores: the
// all-to-all of the layer written as two kernels that store rows straight
// into the other ranks' buffers over NVLink (peer pointers from symmetric
// memory or CUDA IPC), instead of collective passes over fixed-size slots.
//
// G ranks, E experts, rank d owns experts [d E_g, (d + 1) E_g), E_g = E / G.
// Each rank routes its T tokens with the uncapped dispatch (expert-contiguous
// rows, pair i of expert e at row offsets[e] + its rank among e's pairs), and
// the ranks all-gather their per-expert counts cnt[G][E].  From the same
// counts every rank derives the same layouts:
//   destination d's local rows: per local expert, each source's pairs in
//     source order, each source's in its own dispatch order (so an expert's
//     rows are its tokens in (source, token) order, as on one GPU);
//   source s's row for pair i of expert e in d's local rows:
//     base_d[e] + sum over s' < s of cnt[s'][e] + (dest_row[i] - offsets_s[e]);
//   the way back: local row -> (source, its uncapped row offsets_s[e] + j).
// Only the routed rows cross the links (no padding), the receiver needs no
// copy into its layout, and the return stores land in each source's y rows,
// where moe_combine reads them.  The counts are clamped the same way on every
// rank (each source's rows to one destination to at most T min(k, E_g), each
// (source, expert) to at most T), so corrupt counts never move a store outside
// a buffer; such counts set MOE_DEV_BAD_ROW.
//
// k_ep_direct_plan    one block: clamped counts, this rank's send bases, its
//                     local layout, GEMM schedule and return segments.
// k_ep_direct_put     source: a warp per routed pair, x[t] -> the
//                     destination's x_loc row.
// k_ep_direct_plan_put  both in one launch: every block derives the send
//                     positions itself; one extra block lays out the local
//                     rows while the others store.
// k_ep_direct_return  destination: a warp per local row, y_loc -> the
//                     source's y row.
// Every block of a kernel that stores into peer memory ends with a block
// barrier and one system-scope fence (cumulative over the block's stores), so
// a stream-ordered collective after it (a barrier) orders its peer stores
// before any later work on every rank.
#include <cuda_bf16.h>

#include "dispatch_block.cuh"
#include "fp8_rows.cuh"

namespace moe {

namespace {

constexpr int kDirThreads = 256;
constexpr int kDirWarps = kDirThreads / 32;

// At most kDirMaxCounts (source, expert) counts; the return kernel keeps up
// to kDirSmemSegs segment starts in shared memory.
constexpr int kDirMaxCounts = 4096;
constexpr int kDirSmemSegs = 1024;

struct DirPlanArgs {
    const int32_t *cnt_all;  // [G][E] as gathered
    int G, E, T, k, rank;
    int32_t *send_base, *send_cnt;               // [E]
    int32_t *seg_start, *seg_cnt, *seg_ysrc;     // [G][E_g]
    int32_t *loc_counts, *loc_offsets;           // [E_g], [E_g + 1]
    const unsigned long long *peer_y;            // [G] or null
    unsigned long long *row_addr;                // [local T]: byte address of each local row's result
    int H, P;
    WsPtrs lws;
};

// Shared-memory state of a planning block.
struct DirPlanSmem {
    DispatchSmem sm;
    int c[kDirMaxCounts];      // gathered counts, clamped
    int base[kMaxExperts];     // per expert: this rank's first row in its owner's x_loc; later segment starts
    int cnt[kMaxExperts];      // per expert: this rank's rows for it
    int sstart[kMaxExperts];   // return segments' first local rows
    int any_bad;
};

// The gathered counts, clamped identically on every rank ((source s,
// destination d): its experts' counts to [0, T] and their running sum to the
// per-destination bound T min(k, E_g), in expert order), and this rank's
// send positions: base[e] = rows of expert e's owner before expert e's rows
// from this rank, cnt[e] = this rank's rows for e.  All threads of the block.
__device__ void plan_send(const DirPlanArgs &a, DirPlanSmem &p) {
    const int tid = threadIdx.x, G = a.G, E = a.E, Eg = E / G, r = a.rank;
    const int per_dest = a.T * (a.k < Eg ? a.k : Eg);
    if (tid == 0) p.any_bad = 0;
    for (int i = tid; i < G * E; i += kScanThreads) p.c[i] = a.cnt_all[i];
    __syncthreads();
    for (int sd = tid; sd < G * G; sd += kScanThreads) {
        const int s = sd / G, d = sd % G;
        int run = 0;
        bool bad = false;
        for (int el = 0; el < Eg; ++el) {
            const int i = s * E + d * Eg + el, v = p.c[i];
            const int w = min(min(max(v, 0), a.T), per_dest - run);
            bad |= w != v;
            p.c[i] = w;
            run += w;
        }
        if (bad) p.any_bad = 1;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kScanThreads) {
        const int d = e / Eg, el = e % Eg;
        int off = 0;
        for (int e2 = d * Eg; e2 < d * Eg + el; ++e2)
            for (int s = 0; s < G; ++s) off += p.c[s * E + e2];
        for (int s = 0; s < r; ++s) off += p.c[s * E + e];
        p.base[e] = off;
        p.cnt[e] = p.c[r * E + e];
    }
    __syncthreads();
}

// This rank as a destination: the local layout and its GEMM schedule, the
// return segments and each local row's destination address.  All threads of
// the block, after plan_send (base[] and cnt[] are left as they were).
__device__ void plan_local(const DirPlanArgs &a, DirPlanSmem &p) {
    DispatchSmem &sm = p.sm;
    const int tid = threadIdx.x, G = a.G, E = a.E, Eg = E / G, r = a.rank;
    if (tid == 0 && p.any_bad) atomicOr(a.lws.status, MOE_DEV_BAD_ROW);
    for (int el = tid; el < Eg; el += kScanThreads) {
        int n = 0;
        for (int s = 0; s < G; ++s) n += p.c[s * E + r * Eg + el];
        sm.hist[el] = n;
    }
    __syncthreads();
    build_schedule_block(sm, Eg, 0, false, a.loc_counts, a.loc_offsets, a.lws);
    // Return segments: (source s, local expert el) -> first local row, rows,
    // first row in the source's y (its uncapped offset of the expert).
    int *sstart = p.sstart;
    for (int i = tid; i < G * Eg; i += kScanThreads) {
        const int s = i / Eg, el = i % Eg, e = r * Eg + el;
        int start = sm.offs[el];
        for (int s2 = 0; s2 < s; ++s2) start += p.c[s2 * E + e];
        int ysrc = 0;
        for (int e2 = 0; e2 < e; ++e2) ysrc += p.c[s * E + e2];
        a.seg_start[i] = start;
        a.seg_cnt[i] = p.c[s * E + e];
        a.seg_ysrc[i] = ysrc;
        sstart[i] = start;
        sm.running[i] = ysrc;  // scratch: the segment's first row in the source's y
    }
    __syncthreads();
    // Each local row's destination: the byte address of its row in its
    // token's rank's y (0 without peer addresses), for the down projection
    // that stores its results there itself.
    const int total = sm.offs[Eg];
    for (int row = tid; row < total; row += kScanThreads) {
        int lo = 0, hi = Eg - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sm.offs[mid] <= row) lo = mid;
            else hi = mid - 1;
        }
        const int el = lo;
        lo = 0;
        hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sstart[mid * Eg + el] <= row) lo = mid;
            else hi = mid - 1;
        }
        const int i = lo * Eg + el;
        const int yrow = sm.running[i] + (row - sstart[i]);
        a.row_addr[row] = (a.peer_y && (unsigned)yrow < (unsigned)a.P)
                              ? a.peer_y[lo] + (unsigned long long)yrow * (unsigned long long)a.H * 2ull
                              : 0ull;
    }
}

__global__ void __launch_bounds__(kScanThreads) k_ep_direct_plan(DirPlanArgs a) {
    __shared__ DirPlanSmem p;
    pdl_trigger();
    pdl_wait();
    plan_send(a, p);
    for (int e = threadIdx.x; e < a.E; e += kScanThreads) {
        a.send_base[e] = p.base[e];
        a.send_cnt[e] = p.cnt[e];
    }
    plan_local(a, p);
}

// Source side: pair i = t k + j of expert e goes to row base[e] +
// (dest_row[i] - offsets[e]) of rank e / E_g's x_loc.  Rows of H8 16-byte
// vectors (bf16 rows, or e4m3 code rows); with x_scale, the row's scale goes
// to the same row of the rank's scale array (peer_scale).
struct DirPutArgs {
    const uint4 *x;
    const int32_t *topk_idx, *dest_row, *offsets;
    const unsigned long long *peer_x_loc;
    int R, k, E, Eg, Tloc, H8;
    uint32_t *status;
    const float *x_scale;
    const unsigned long long *peer_scale;
    int quantize;  // x: bf16 rows, quantized on the way (codes and scale into peer_x_loc / peer_scale)
};

// One bf16 row of H8 16-byte vectors stored as e4m3 codes (H8 8-byte groups)
// with its scale, by one warp, exactly as the row quantizer does it: the
// row's largest magnitude (eight loads per lane in flight), then the codes
// from a second read of the row, which comes from L1 or L2.
__device__ __forceinline__ void put_row_quantized(const uint4 *__restrict__ src, uint2 *__restrict__ dst, int H8,
                                                  int lane, float *scale_dst) {
    __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
    int v = lane;
    for (; v + 224 < H8; v += 256) {
        uint4 t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = __ldg(src + v + 32 * j);
#pragma unroll
        for (int j = 0; j < 8; ++j) m2 = amax8(t[j], m2);
    }
    for (; v < H8; v += 32) m2 = amax8(__ldg(src + v), m2);
    float m = amax_of(m2);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const Fp8Scale sc = fp8_scale(m);
    v = lane;
    for (; v + 224 < H8; v += 256) {
        uint4 t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = __ldg(src + v + 32 * j);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[v + 32 * j] = quant8(t[j], sc);
    }
    for (; v < H8; v += 32) dst[v] = quant8(__ldg(src + v), sc);
    if (lane == 0) *scale_dst = sc.s;
}

// A routed pair's expert (-1 past the end or for an id the router reported)
// and its rank among the expert's pairs on this rank.
struct PairRef {
    int e, ri;
};
__device__ __forceinline__ PairRef load_pair(const DirPutArgs &q, int i) {
    PairRef r = {-1, 0};
    if (i < q.R) {
        const int e = q.topk_idx[i];
        if ((unsigned)e < (unsigned)q.E) {
            r.e = e;
            r.ri = q.dest_row[i] - q.offsets[e];
        }
    }
    return r;
}

// Blocks [0, nblocks) of the grid share the pairs, a warp per pair; `first`
// is the warp's first pair, loaded by the caller.
__device__ void put_rows(const DirPutArgs &q, const int *base, const int *cnt, int nblocks, PairRef first) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    PairRef pr = first;
    for (int i = blockIdx.x * kDirWarps + (threadIdx.x >> 5); i < q.R; i += nblocks * kDirWarps) {
        if (i != blockIdx.x * kDirWarps + (threadIdx.x >> 5)) pr = load_pair(q, i);
        const int e = pr.e, ri = pr.ri;
        if (e < 0) continue;  // reported by the router
        const int pos = base[e] + ri;
        if (ri < 0 || ri >= cnt[e] || (unsigned)pos >= (unsigned)q.Tloc) {
            bad = true;
            continue;
        }
        if (q.quantize) {
            put_row_quantized(q.x + (size_t)(i / q.k) * q.H8,
                              reinterpret_cast<uint2 *>(q.peer_x_loc[e / q.Eg]) + (size_t)pos * q.H8, q.H8, lane,
                              reinterpret_cast<float *>(q.peer_scale[e / q.Eg]) + pos);
            continue;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(q.peer_x_loc[e / q.Eg]) + (size_t)pos * q.H8;
        copy_row_warp(q.x + (size_t)(i / q.k) * q.H8, dst, q.H8, lane);
        if (q.x_scale && lane == 0) reinterpret_cast<float *>(q.peer_scale[e / q.Eg])[pos] = q.x_scale[i / q.k];
    }
    if (bad && lane == 0) atomicOr(q.status, MOE_DEV_BAD_ROW);
    fence_block_stores_system();
}

// The dispatch after a separate plan (send positions from the workspace).
__global__ void __launch_bounds__(kDirThreads) k_ep_direct_put(DirPutArgs q, const int32_t *send_base,
                                                                const int32_t *send_cnt) {
    pdl_trigger();
    pdl_wait();
    put_rows(q, send_base, send_cnt, (int)gridDim.x, load_pair(q, blockIdx.x * kDirWarps + (threadIdx.x >> 5)));
}

// Plan and dispatch in one launch: every block derives this rank's send
// positions from the gathered counts itself (its warps' first pairs loaded
// meanwhile), so the stores start at once; the last block instead lays out
// this rank's local rows (schedule, return segments, row addresses) for the
// kernels after the barrier, alongside the stores.
__global__ void __launch_bounds__(kDirThreads) k_ep_direct_plan_put(DirPlanArgs a, DirPutArgs q) {
    __shared__ DirPlanSmem p;
    pdl_trigger();
    pdl_wait();
    const bool planner = blockIdx.x == gridDim.x - 1;
    const PairRef first = planner ? PairRef{-1, 0} : load_pair(q, blockIdx.x * kDirWarps + (threadIdx.x >> 5));
    plan_send(a, p);
    if (planner)
        plan_local(a, p);
    else
        put_rows(q, p.base, p.cnt, (int)gridDim.x - 1, first);
}

// Destination side: local row r of segment (s, el) goes to row seg_ysrc +
// (r - seg_start) of rank s's y.
__global__ void __launch_bounds__(kDirThreads) k_ep_direct_return(const uint4 *y_loc, const int32_t *seg_start,
                                                                   const int32_t *seg_cnt, const int32_t *seg_ysrc,
                                                                   const int32_t *loc_offsets,
                                                                   const unsigned long long *peer_y, int G, int Eg,
                                                                   int Tloc, int P, int H8) {
    __shared__ int offs[kMaxExperts + 1];
    __shared__ int sstart[kDirSmemSegs];
    pdl_trigger();
    pdl_wait();
    for (int i = threadIdx.x; i <= Eg; i += kDirThreads) offs[i] = loc_offsets[i];
    const bool staged = G * Eg <= kDirSmemSegs;  // segment starts searched in shared memory
    if (staged)
        for (int i = threadIdx.x; i < G * Eg; i += kDirThreads) sstart[i] = seg_start[i];
    __syncthreads();
    const int *starts = staged ? sstart : seg_start;
    const int lane = threadIdx.x & 31;
    const int total = min(offs[Eg], Tloc);
    for (int r = blockIdx.x * kDirWarps + (threadIdx.x >> 5); r < total; r += gridDim.x * kDirWarps) {
        int lo = 0, hi = Eg - 1;  // local expert: last el with offs[el] <= r
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offs[mid] <= r) lo = mid;
            else hi = mid - 1;
        }
        const int el = lo;
        lo = 0;
        hi = G - 1;  // source: last s with seg_start[s][el] <= r (empty segments share a start)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid * Eg + el] <= r) lo = mid;
            else hi = mid - 1;
        }
        const int i = lo * Eg + el, j = r - starts[i];
        const int yrow = seg_ysrc[i] + j;
        if (j >= seg_cnt[i] || (unsigned)yrow >= (unsigned)P) continue;  // cannot happen: the plan's layout
        uint4 *dst = reinterpret_cast<uint4 *>(peer_y[lo]) + (size_t)yrow * H8;
        copy_row_warp(y_loc + (size_t)r * H8, dst, H8, lane);
    }
    fence_block_stores_system();
}

int dir_grid(int64_t rows, int num_sms) {
    const int64_t g = (rows + kDirWarps - 1) / kDirWarps;
    return (int)(g < 1 ? 1 : (g > 2 * num_sms ? 2 * num_sms : g));
}

}  // namespace

// Local rows of one rank at most: every source sends it at most T min(k, E/G)
// pairs.
int64_t ep_direct_local_rows(const moe_shape &s, int G) {
    const int Eg = s.E / G;
    return (int64_t)G * s.T * (s.k < Eg ? s.k : Eg);
}

bool ep_direct_counts_fit(const moe_shape &s, int G) { return (int64_t)G * s.E <= kDirMaxCounts; }

// Direct EP workspace (int32 arrays, each padded to 16 bytes): send bases and
// counts [E] each, return segments (start, rows, source row) [G E_g] each,
// local counts [E_g], local offsets [E_g + 1].
struct DirWs {
    unsigned long long *row_addr;
    int32_t *send_base, *send_cnt, *seg_start, *seg_cnt, *seg_ysrc, *loc_counts, *loc_offsets;
};
static DirWs dir_ptrs(void *ep_ws, const moe_shape &s, int G) {
    const size_t E4 = align_up((size_t)s.E, 4), Eg = (size_t)(s.E / G);
    DirWs p;
    p.row_addr = (unsigned long long *)ep_ws;
    int32_t *b = (int32_t *)(p.row_addr + align_up((size_t)ep_direct_local_rows(s, G), 2));
    p.send_base = b;
    p.send_cnt = p.send_base + E4;
    p.seg_start = p.send_cnt + E4;
    p.seg_cnt = p.seg_start + E4;
    p.seg_ysrc = p.seg_cnt + E4;
    p.loc_counts = p.seg_ysrc + E4;
    p.loc_offsets = p.loc_counts + align_up(Eg, 4);
    return p;
}

size_t ep_direct_workspace_bytes(const moe_shape &s, int G) {
    const size_t E4 = align_up((size_t)s.E, 4), Eg = (size_t)(s.E / G);
    return 8 * align_up((size_t)ep_direct_local_rows(s, G), 2) + 4 * (5 * E4 + align_up(Eg, 4) + align_up(Eg + 1, 4));
}

const unsigned long long *ep_direct_row_addr(void *ep_ws, const moe_shape &s, int G) {
    return dir_ptrs(ep_ws, s, G).row_addr;
}

// The number of local rows the plan laid out (device int).
const int32_t *ep_direct_local_total(void *ep_ws, const moe_shape &s, int G) {
    return dir_ptrs(ep_ws, s, G).loc_offsets + s.E / G;
}

static DirPlanArgs plan_args(const moe_shape &s, int G, int rank, const int32_t *cnt_all, const void *peer_y,
                             const WsLayout &Lloc, void *ws_loc, void *ep_ws) {
    const DirWs p = dir_ptrs(ep_ws, s, G);
    DirPlanArgs a;
    a.cnt_all = cnt_all;
    a.G = G;
    a.E = s.E;
    a.T = s.T;
    a.k = s.k;
    a.rank = rank;
    a.send_base = p.send_base;
    a.send_cnt = p.send_cnt;
    a.seg_start = p.seg_start;
    a.seg_cnt = p.seg_cnt;
    a.seg_ysrc = p.seg_ysrc;
    a.loc_counts = p.loc_counts;
    a.loc_offsets = p.loc_offsets;
    a.peer_y = (const unsigned long long *)peer_y;
    a.row_addr = p.row_addr;
    a.H = s.H;
    a.P = s.T * s.k;
    a.lws = ws_ptrs(ws_loc, Lloc);
    return a;
}

// x: bf16 rows (x_scale null), or e4m3 code rows with their scales.
static DirPutArgs put_args(const moe_shape &s, int G, const void *x, const int32_t *topk_idx, const int32_t *dest_row,
                           const int32_t *offsets, const void *peer_x_loc, uint32_t *status, const float *x_scale,
                           const void *peer_scale, bool quantize = false) {
    DirPutArgs q;
    q.x = (const uint4 *)x;
    q.topk_idx = topk_idx;
    q.dest_row = dest_row;
    q.offsets = offsets;
    q.peer_x_loc = (const unsigned long long *)peer_x_loc;
    q.R = s.T * s.k;
    q.k = s.k;
    q.E = s.E;
    q.Eg = s.E / G;
    q.Tloc = (int)ep_direct_local_rows(s, G);
    q.H8 = x_scale ? s.H / 16 : s.H / 8;
    q.status = status;
    q.x_scale = x_scale;
    q.peer_scale = (const unsigned long long *)peer_scale;
    q.quantize = quantize ? 1 : 0;  // H8 = H / 8: bf16 vectors in, 8-byte code groups out
    return q;
}

cudaError_t launch_ep_direct_plan(const moe_shape &s, int G, int rank, const int32_t *cnt_all, const void *peer_y,
                                  const WsLayout &Lloc, void *ws_loc, void *ep_ws, cudaStream_t stream) {
    return launch_pdl(k_ep_direct_plan, dim3(1), dim3(kScanThreads), 0, stream,
                      plan_args(s, G, rank, cnt_all, peer_y, Lloc, ws_loc, ep_ws));
}

cudaError_t launch_ep_direct_put(const moe_shape &s, int G, const void *x, const int32_t *topk_idx,
                                 const int32_t *dest_row, const int32_t *offsets, const void *peer_x_loc,
                                 void *ep_ws, uint32_t *status, int num_sms, cudaStream_t stream,
                                 const float *x_scale, const void *peer_scale) {
    const DirWs p = dir_ptrs(ep_ws, s, G);
    return launch_pdl(k_ep_direct_put, dim3(dir_grid((int64_t)s.T * s.k, num_sms)), dim3(kDirThreads), 0, stream,
                      put_args(s, G, x, topk_idx, dest_row, offsets, peer_x_loc, status, x_scale, peer_scale),
                      (const int32_t *)p.send_base, (const int32_t *)p.send_cnt);
}

cudaError_t launch_ep_direct_plan_put(const moe_shape &s, int G, int rank, const int32_t *cnt_all,
                                      const void *peer_y, const WsLayout &Lloc, void *ws_loc, const void *x,
                                      const int32_t *topk_idx, const int32_t *dest_row, const int32_t *offsets,
                                      const void *peer_x_loc, void *ep_ws, uint32_t *status, int num_sms,
                                      cudaStream_t stream, const float *x_scale, const void *peer_scale,
                                      bool quantize) {
    return launch_pdl(k_ep_direct_plan_put, dim3(dir_grid((int64_t)s.T * s.k, num_sms) + 1), dim3(kDirThreads), 0,
                      stream, plan_args(s, G, rank, cnt_all, peer_y, Lloc, ws_loc, ep_ws),
                      put_args(s, G, x, topk_idx, dest_row, offsets, peer_x_loc, status, quantize ? nullptr : x_scale,
                               peer_scale, quantize));
}

cudaError_t launch_ep_direct_return(const moe_shape &s, int G, const void *y_loc, const void *peer_y, void *ep_ws,
                                    int num_sms, cudaStream_t stream) {
    const DirWs p = dir_ptrs(ep_ws, s, G);
    const int64_t Tloc = ep_direct_local_rows(s, G);
    return launch_pdl(k_ep_direct_return, dim3(dir_grid(Tloc, num_sms)), dim3(kDirThreads), 0, stream,
                      (const uint4 *)y_loc, (const int32_t *)p.seg_start, (const int32_t *)p.seg_cnt,
                      (const int32_t *)p.seg_ysrc, (const int32_t *)p.loc_offsets,
                      (const unsigned long long *)peer_y, G, s.E / G, (int)Tloc, s.T * s.k, s.H / 8);
}

}  // namespace moe
