// Expert-parallel Cap-and-Spill dispatch: the data movement around two
// all-to-all passes ("Cap-and-Spill" critique, juhe.plus, section
// "Cap-and-Spill": a first pass with C slots per expert, then a second pass
// for the compacted overflow, whose buffer is sized for the largest possible
// overflow so that it can be allocated ahead of time and no token is dropped;
// no host synchronisation between the passes).
//
// G ranks, E experts, rank d owns experts [d E_g, (d + 1) E_g), E_g = E / G.
// Each rank routes its own T tokens with the capacity layout of
// moe_permute: rows [0, E C) are the capacity slots, expert-major, so the
// slots of rank d's experts are the contiguous rows [d E_g C, (d+1) E_g C) --
// pass 1 is an equal-split all-to-all of x_perm[0, E C).  The overflow rows
// follow, compacted and expert-major, so rank d's overflow rows are contiguous
// too; pass 2 moves each destination's rows in a fixed slot of S rows, S =
// min(k, E_g) max(0, T - C) (one source's tokens send at most min(k, E_g)
// pairs each to one destination, and an expert's overflow is at most T - C),
// an equal-split all-to-all as well.
//
// k_ep_spill_rows  the overflow rows between x_perm's compacted overflow
//                  region and the per-destination slots (pack: also the
//                  counts sent ahead of the rows; unpack: the same copies
//                  reversed), a warp per row over every block.
// k_ep_receive     on the receiving rank, from the counts of every source:
//                  an expert-contiguous local layout (per expert, each
//                  source's capacity rows then its overflow rows), the
//                  received rows copied into it (a warp per row, every block
//                  deriving the layout itself) and, by one extra block, its
//                  GEMM schedule (the block schedule builder of the dispatch)
//                  and the source of every local row.
// k_ep_local_rows  the local results back to the return buffers, a warp per
//                  row.
#include <cuda_bf16.h>

#include "dispatch_block.cuh"

namespace moe {

namespace {

constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;

// Overflow row q of x_perm (row E C + q) belongs to destination d, the last
// with starts[d * stride] <= q, and sits at row d S + (q - starts[d * stride])
// of the slots.  pack (reverse = 0): a = x_perm, b = send slots, b <- a, and
// block 0 writes meta (per destination: its experts' capacity counts, then
// their overflow counts) and the destination starts into ep_starts for
// unpack; unpack (reverse = 1): a = y, b = received slots, a <- b, with the
// starts read back from ep_starts.
__global__ void __launch_bounds__(kRowThreads) k_ep_spill_rows(WsPtrs ws, const int32_t *ep_starts_in, int E, int G,
                                                               int C, int S, int P, int H8, uint4 *a, uint4 *b,
                                                               int reverse, int32_t *meta, int32_t *ep_starts_out) {
    __shared__ int starts[kMaxExperts + 1];
    pdl_trigger();
    pdl_wait();
    const int Eg = E / G, tid = threadIdx.x;
    for (int d = tid; d <= G; d += kRowThreads) starts[d] = reverse ? ep_starts_in[d] : ws.spill_off[d * Eg];
    if (!reverse && blockIdx.x == 0) {
        for (int i = tid; i < E; i += kRowThreads) {
            const int d = i / Eg, e = i % Eg;
            meta[(size_t)d * 2 * Eg + e] = ws.cap_cnt[i];
            meta[(size_t)d * 2 * Eg + Eg + e] = ws.spill_cnt[i];
        }
        for (int d = tid; d <= G; d += kRowThreads) ep_starts_out[d] = ws.spill_off[d * Eg];
    }
    __syncthreads();
    const int total = min(starts[G], P - E * C);
    const int lane = tid & 31;
    for (int q = blockIdx.x * kRowWarps + (tid >> 5); q < total; q += gridDim.x * kRowWarps) {
        int lo = 0, hi = G - 1;  // last d with starts[d] <= q
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int j = q - starts[lo];
        if (j >= S) {  // cannot happen for a valid routing; never touch past the slot
            if (lane == 0 && !reverse) atomicOr(ws.status, MOE_DEV_BAD_ROW);  // unpack: flagged by the pack
            continue;
        }
        uint4 *ra = a + (size_t)(E * C + q) * H8, *rb = b + (size_t)(lo * S + j) * H8;
        if (reverse)
            copy_row_warp(rb, ra, H8, lane);
        else
            copy_row_warp(ra, rb, H8, lane);
    }
}

// The row copy of the dispatch and the pack in one launch: capacity slot
// rows of x_perm from x (zero rows for unfilled slots), overflow rows
// straight into their destination's slot of `send` (x_perm's overflow region
// is not written); block 0 also writes the counts sent ahead (meta) and the
// destination starts, as the pack does.  A warp per row, eight 16-byte loads
// per lane in flight, streaming stores (each row is read once, by the
// exchange).
__global__ void __launch_bounds__(kRowThreads) k_ep_gather_pack(WsPtrs ws, const uint4 *__restrict__ x,
                                                                const int32_t *__restrict__ src_token, int T, int E,
                                                                int G, int C, int S, int P, int H8, uint4 *x_perm,
                                                                uint4 *send, int32_t *meta, int32_t *ep_starts_out) {
    __shared__ int starts[kMaxExperts + 1];
    pdl_trigger();
    pdl_wait();
    const int Eg = E / G, tid = threadIdx.x;
    for (int d = tid; d <= G; d += kRowThreads) starts[d] = ws.spill_off[d * Eg];
    if (blockIdx.x == 0) {
        for (int i = tid; i < E; i += kRowThreads) {
            const int d = i / Eg, e = i % Eg;
            meta[(size_t)d * 2 * Eg + e] = ws.cap_cnt[i];
            meta[(size_t)d * 2 * Eg + Eg + e] = ws.spill_cnt[i];
        }
        for (int d = tid; d <= G; d += kRowThreads) ep_starts_out[d] = ws.spill_off[d * Eg];
    }
    __syncthreads();
    const int cap = E * C, rows = min(cap + starts[G], P);
    const int lane = tid & 31;
    for (int row = blockIdx.x * kRowWarps + (tid >> 5); row < rows; row += gridDim.x * kRowWarps) {
        uint4 *dst;
        if (row < cap) {
            dst = x_perm + (size_t)row * H8;
        } else {
            const int q = row - cap;
            int lo = 0, hi = G - 1;  // last d with starts[d] <= q
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (starts[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            const int j = q - starts[lo];
            if (j >= S) {  // cannot happen for a valid routing; never touch past the slot
                if (lane == 0) atomicOr(ws.status, MOE_DEV_BAD_ROW);
                continue;
            }
            dst = send + (size_t)(lo * S + j) * H8;
        }
        const int t = src_token[row];
        if ((unsigned)t < (unsigned)T) {
            const uint4 *src = x + (size_t)t * H8;
            int v = lane;
            for (; v + 224 < H8; v += 256) {
                uint4 q8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q8[i] = __ldg(src + v + 32 * i);
#pragma unroll
                for (int i = 0; i < 8; ++i) __stcs(dst + v + 32 * i, q8[i]);
            }
            for (; v < H8; v += 32) __stcs(dst + v, __ldg(src + v));
        } else {
            for (int v = lane; v < H8; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

// Receiving rank, one block.  meta[s][0][e], meta[s][1][e]: capacity and
// overflow rows source s sent for local expert e, clamped to what the buffers
// hold (capacity rows to C, each source's overflow rows to its slot of S
// rows; counts from a pack never need it).  Local row order: expert, then
// source, then the capacity rows before the overflow rows; the local rows
// total at most G (E_g C + S), the local shape's T.  row_src[r] = the row of
// the received capacity buffer that local row r comes from, or -1 - its row
// in the received overflow buffer.
// Shared-memory state of a receiving block: the received counts of every
// (source s, local expert e), indexed s E_g + e, clamped.
struct RecvSmem {
    DispatchSmem sm;
    int nc[kMaxExperts], no[kMaxExperts], ovf_pre[kMaxExperts], seg[kMaxExperts];
    int m[2 * kMaxExperts];
    int any_bad;
};

// The received counts (all loads in one round trip), clamped to what the
// buffers hold (capacity rows to C, each source's overflow rows to S in
// expert order); all threads of the block.
__device__ void recv_counts(const int32_t *meta, int G, int Eg, int C, int S, RecvSmem &p) {
    const int tid = threadIdx.x;
    if (tid == 0) p.any_bad = 0;
    for (int i = tid; i < 2 * G * Eg; i += kScanThreads) p.m[i] = meta[i];
    __syncthreads();
    for (int s = tid; s < G; s += kScanThreads) {
        int pre = 0;
        bool bad = false;
        for (int e = 0; e < Eg; ++e) {
            const int rc = p.m[s * 2 * Eg + e], ro = p.m[s * 2 * Eg + Eg + e];
            const int c = min(max(rc, 0), C), o = min(max(ro, 0), S - pre);
            bad |= c != rc || o != ro;
            p.nc[s * Eg + e] = c;
            p.no[s * Eg + e] = o;
            p.ovf_pre[s * Eg + e] = pre;
            pre += o;
        }
        if (bad) p.any_bad = 1;
    }
    __syncthreads();
}

// First local row of each (source, expert) segment: expert e's rows are its
// sources' rows in source order from offs[e].  All threads of the block.
__device__ void recv_segments(RecvSmem &p, const int *offs, int G, int Eg) {
    for (int e = threadIdx.x; e < Eg; e += kScanThreads) {
        int row = offs[e];
        for (int s = 0; s < G; ++s) {
            p.seg[s * Eg + e] = row;
            row += p.nc[s * Eg + e] + p.no[s * Eg + e];
        }
    }
    __syncthreads();
}

// Received row of local row r: capacity buffer row (>= 0) or -1 - overflow
// buffer row.
__device__ __forceinline__ int recv_row_source(const RecvSmem &p, const int *offs, int r, int G, int Eg, int C,
                                               int S) {
    int lo = 0, hi = Eg - 1;  // expert: last e with offs[e] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] <= r) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo;
    lo = 0;
    hi = G - 1;  // source: last s with seg[s][e] <= r (empty segments share a start)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.seg[mid * Eg + e] <= r) lo = mid;
        else hi = mid - 1;
    }
    const int i = lo * Eg + e, j = r - p.seg[i];
    return j < p.nc[i] ? lo * Eg * C + e * C + j : -1 - (lo * S + p.ovf_pre[i] + (j - p.nc[i]));
}

// The receiving side in one launch.  Every block derives the local layout
// from the received counts itself and copies its share of the received rows
// into x_loc (a warp per local row); the last block instead builds what the
// later kernels read: the local counts, offsets and GEMM schedule (uncapped
// layout of the local experts) and the source of every local row (row_src,
// for the return).
__global__ void __launch_bounds__(kScanThreads) k_ep_receive(const int32_t *meta, int G, int Eg, int C, int S,
                                                             int32_t *loc_counts, int32_t *loc_offsets,
                                                             int32_t *row_src, WsPtrs lws, int Tloc, int H8,
                                                             const uint4 *cap, const uint4 *ovf, uint4 *loc) {
    __shared__ RecvSmem p;
    DispatchSmem &sm = p.sm;
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x;
    recv_counts(meta, G, Eg, C, S, p);
    const int n = tid < Eg ? [&] {
        int v = 0;
        for (int s = 0; s < G; ++s) v += p.nc[s * Eg + tid] + p.no[s * Eg + tid];
        return v;
    }() : 0;
    if (blockIdx.x == gridDim.x - 1) {
        if (tid == 0 && p.any_bad) atomicOr(lws.status, MOE_DEV_BAD_ROW);
        if (tid < Eg) sm.hist[tid] = n;
        __syncthreads();
        build_schedule_block(sm, Eg, 0, false, loc_counts, loc_offsets, lws);
        recv_segments(p, sm.offs, G, Eg);
        const int total = sm.offs[Eg];
        for (int r = tid; r < total; r += kScanThreads) row_src[r] = recv_row_source(p, sm.offs, r, G, Eg, C, S);
        return;
    }
    // exclusive offsets of the local experts (the schedule builder's own)
    int incl = n, unused = 0;
    block_inclusive_scan2(sm, incl, unused);
    if (tid < Eg) sm.offs[tid] = incl - n;
    if (tid == Eg - 1) sm.offs[Eg] = incl;
    __syncthreads();
    recv_segments(p, sm.offs, G, Eg);
    const int lane = tid & 31;
    const int total = min(sm.offs[Eg], Tloc);
    for (int r = blockIdx.x * kRowWarps + (tid >> 5); r < total; r += ((int)gridDim.x - 1) * kRowWarps) {
        const int src = recv_row_source(p, sm.offs, r, G, Eg, C, S);
        const uint4 *rx = src >= 0 ? cap + (size_t)src * H8 : ovf + (size_t)(-1 - src) * H8;
        copy_row_warp(rx, loc + (size_t)r * H8, H8, lane);
    }
}

// Local row r <-> its received row (row_src[r]: capacity buffer row, or
// -1 - overflow buffer row); forward: loc <- cap / ovf, reverse: cap / ovf
// <- loc.  total = loc_offsets[E_g], at most Tloc.
__global__ void __launch_bounds__(kRowThreads) k_ep_local_rows(const int32_t *row_src, const int32_t *loc_total,
                                                               int Tloc, int H8, uint4 *cap, uint4 *ovf, uint4 *loc,
                                                               int reverse) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int total = min(*loc_total, Tloc);
    for (int r = blockIdx.x * kRowWarps + (threadIdx.x >> 5); r < total; r += gridDim.x * kRowWarps) {
        const int src = row_src[r];
        uint4 *rx = src >= 0 ? cap + (size_t)src * H8 : ovf + (size_t)(-1 - src) * H8;
        uint4 *rl = loc + (size_t)r * H8;
        if (reverse)
            copy_row_warp(rl, rx, H8, lane);
        else
            copy_row_warp(rx, rl, H8, lane);
    }
}

int row_grid(int64_t rows, int num_sms) {
    const int64_t g = (rows + kRowWarps - 1) / kRowWarps;
    return (int)(g < 1 ? 1 : (g > 2 * num_sms ? 2 * num_sms : g));
}

}  // namespace

// Overflow slot rows per (source, destination): min(k, E/G) * max(0, T - C).
int64_t ep_overflow_rows(const moe_shape &s, int G) {
    const int Eg = s.E / G;
    return (int64_t)(s.k < Eg ? s.k : Eg) * (s.T > s.C ? s.T - s.C : 0);
}

static int64_t ep_local_rows(const moe_shape &s, int G) {
    return (int64_t)G * ((int64_t)(s.E / G) * s.C + ep_overflow_rows(s, G));
}

// EP workspace (int32 arrays, each padded to 16 bytes): destination starts
// [G + 1], local counts [E/G], local offsets [E/G + 1], row sources [local T].
struct EpWs {
    int32_t *starts, *loc_counts, *loc_offsets, *row_src;
};
static EpWs ep_ptrs(void *ep_ws, const moe_shape &s, int G) {
    int32_t *b = (int32_t *)ep_ws;
    const int Eg = s.E / G;
    EpWs p;
    p.starts = b;
    p.loc_counts = p.starts + align_up((size_t)G + 1, 4);
    p.loc_offsets = p.loc_counts + align_up((size_t)Eg, 4);
    p.row_src = p.loc_offsets + align_up((size_t)Eg + 1, 4);
    return p;
}

size_t ep_workspace_bytes(const moe_shape &s, int G) {
    const int Eg = s.E / G;
    return 4 * (align_up((size_t)G + 1, 4) + align_up((size_t)Eg, 4) + align_up((size_t)Eg + 1, 4) +
                align_up((size_t)ep_local_rows(s, G), 4));
}

// Source side: counts per destination into send_meta, each destination's
// overflow rows of x_perm into its slot of send_ovf ([G][S] rows).
cudaError_t launch_ep_pack(const moe_shape &s, int G, const void *x_perm, const WsLayout &L, void *ws, void *send_ovf,
                           int32_t *send_meta, void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G);
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, true);
    return launch_pdl(k_ep_spill_rows, dim3(row_grid(P - (int64_t)s.E * s.C, num_sms)), dim3(kRowThreads), 0, stream,
                      ws_ptrs(ws, L), (const int32_t *)nullptr, s.E, G, s.C, S, (int)P, s.H / 8, (uint4 *)x_perm,
                      (uint4 *)send_ovf, 0, send_meta, p.starts);
}

// Source side, the row copy and the pack in one launch.
cudaError_t launch_ep_gather_pack(const moe_shape &s, int G, const void *x, const int32_t *src_token, void *x_perm,
                                  const WsLayout &L, void *ws, void *send_ovf, int32_t *send_meta, void *ep_ws,
                                  int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G);
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, true);
    const int64_t rows_hint = (int64_t)s.E * s.C + (int64_t)s.k * (s.T > s.C ? s.T - s.C : 0);
    return launch_pdl(k_ep_gather_pack, dim3(row_grid(rows_hint < P ? rows_hint : P, num_sms)), dim3(kRowThreads), 0,
                      stream, ws_ptrs(ws, L), (const uint4 *)x, src_token, s.T, s.E, G, s.C, S, (int)P, s.H / 8,
                      (uint4 *)x_perm, (uint4 *)send_ovf, send_meta, p.starts);
}

// Receiving side: the local layout, its GEMM schedule in the local workspace,
// and the received rows gathered into x_loc.
cudaError_t launch_ep_local_dispatch(const moe_shape &s, int G, const int32_t *recv_meta, const void *recv_cap,
                                     const void *recv_ovf, void *x_loc, const WsLayout &Lloc, void *ws_loc,
                                     void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G), Eg = s.E / G;
    const int64_t Tloc = ep_local_rows(s, G);
    return launch_pdl(k_ep_receive, dim3(row_grid(Tloc, num_sms) + 1), dim3(kScanThreads), 0, stream, recv_meta, G,
                      Eg, s.C, S, p.loc_counts, p.loc_offsets, p.row_src, ws_ptrs(ws_loc, Lloc), (int)Tloc, s.H / 8,
                      (const uint4 *)recv_cap, (const uint4 *)recv_ovf, (uint4 *)x_loc);
}

// Receiving side, after the local experts: y_loc rows back to where their
// inputs came from (the capacity and overflow send buffers of the return
// passes).
cudaError_t launch_ep_local_return(const moe_shape &s, int G, const void *y_loc, void *back_cap, void *back_ovf,
                                   void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int64_t Tloc = ep_local_rows(s, G);
    return launch_pdl(k_ep_local_rows, dim3(row_grid(Tloc, num_sms)), dim3(kRowThreads), 0, stream,
                      (const int32_t *)p.row_src, (const int32_t *)(p.loc_offsets + s.E / G), (int)Tloc, s.H / 8,
                      (uint4 *)back_cap, (uint4 *)back_ovf, (uint4 *)y_loc, 1);
}

// Source side, after the return passes: the overflow rows' results from
// their slots back into y's overflow region (the pack copies reversed).
cudaError_t launch_ep_unpack(const moe_shape &s, int G, const void *recv_back_ovf, void *y, void *ep_ws, int num_sms,
                             cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G);
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, true);
    const WsPtrs none = {};  // no status word: the pack already flagged a bad row
    return launch_pdl(k_ep_spill_rows, dim3(row_grid(P - (int64_t)s.E * s.C, num_sms)), dim3(kRowThreads), 0, stream,
                      none, (const int32_t *)p.starts, s.E, G, s.C, S, (int)P, s.H / 8, (uint4 *)y,
                      (uint4 *)recv_back_ovf, 1, (int32_t *)nullptr, (int32_t *)nullptr);
}

// The unpack folded into the combine: overflow results read from the
// received return slots where the unpack would have copied them from.
cudaError_t launch_combine_ovf(const moe_shape &s, int G, int S, const void *y, const void *ovf,
                               const int32_t *starts, const int32_t *dest_row, const float *topk_w, void *out,
                               cudaStream_t stream);
cudaError_t launch_ep_unpack_combine(const moe_shape &s, int G, const void *recv_back_ovf, const void *y,
                                     const int32_t *dest_row, const float *topk_w, void *out, void *ep_ws,
                                     cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    return launch_combine_ovf(s, G, (int)ep_overflow_rows(s, G), y, recv_back_ovf, p.starts, dest_row, topk_w, out,
                              stream);
}

}  // namespace moe
