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
// k_ep_plan_send   per destination: its experts' capacity and overflow
//                  counts (sent ahead of the rows) and the range of its
//                  overflow rows (the pack and unpack copies).
// k_ep_plan_recv   on the receiving rank, from the counts of every source:
//                  an expert-contiguous local layout (per expert, each
//                  source's capacity rows then its overflow rows), the copy
//                  segments into it and back, and the local grouped-GEMM
//                  schedule (the block schedule builder of the dispatch).
// k_copy_segments  row copies by segment list, forward or reversed.
#include <cuda_bf16.h>

#include "dispatch_block.cuh"

namespace moe {

namespace {

constexpr int kSegThreads = 256;

// Per destination d: meta[d][0][e] = capacity count, meta[d][1][e] =
// overflow count of its expert d E_g + e; seg[d] = {first overflow row in
// x_perm, first row of d's slot in the send buffer, rows, 0}.
__global__ void __launch_bounds__(kSegThreads) k_ep_plan_send(WsPtrs ws, int E, int G, int C, int S,
                                                              int32_t *meta, int4 *seg) {
    pdl_trigger();
    pdl_wait();
    const int Eg = E / G;
    for (int i = threadIdx.x; i < E; i += kSegThreads) {
        const int d = i / Eg, e = i % Eg;
        meta[(size_t)d * 2 * Eg + e] = ws.cap_cnt[i];
        meta[(size_t)d * 2 * Eg + Eg + e] = ws.spill_cnt[i];
    }
    for (int d = threadIdx.x; d < G; d += kSegThreads) {
        const int a = ws.spill_off[d * Eg], b = ws.spill_off[(d + 1) * Eg];
        int len = b - a;
        if (len > S) {  // cannot happen for a valid routing; never copy past the slot
            atomicOr(ws.status, MOE_DEV_BAD_ROW);
            len = S;
        }
        seg[d] = make_int4(E * C + a, d * S, len, 0);
    }
}

// Rows source s sent for local expert e, clamped to what the buffers hold
// (capacity rows to C, each source's overflow rows to its slot of S rows);
// counts from moe_ep_pack never need the clamp.  ovf: the source's overflow
// rows before expert e's in its slot.
__device__ inline void ep_recv_counts(const int32_t *meta, int s, int e, int Eg, int C, int S, int &nc, int &no,
                                      int &ovf, bool &bad) {
    const int32_t *m = meta + (size_t)s * 2 * Eg;
    ovf = 0;
    for (int e2 = 0; e2 < e; ++e2) ovf += min(max(m[Eg + e2], 0), S - ovf);
    const int rc = m[e], ro = m[Eg + e];
    nc = min(max(rc, 0), C);
    no = min(max(ro, 0), S - ovf);
    bad = nc != rc || no != ro;
}

// Receiving rank, one block.  meta[s][0][e], meta[s][1][e]: capacity and
// overflow rows source s sent for local expert e.  Local row order: expert,
// then source, then the capacity rows before the overflow rows.
// cap_seg[s E_g + e] = {row in the received capacity buffer, local row, len};
// ovf_seg[s E_g + e] = {row in the received overflow buffer, local row, len}.
// The local rows total at most G (E_g C + S), the local shape's T.
__global__ void __launch_bounds__(kScanThreads) k_ep_plan_recv(const int32_t *meta, int G, int Eg, int C, int S,
                                                               int4 *cap_seg, int4 *ovf_seg, int32_t *loc_counts,
                                                               int32_t *loc_offsets, WsPtrs lws) {
    __shared__ DispatchSmem sm;
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x;
    bool any_bad = false;
    for (int e = tid; e < Eg; e += kScanThreads) {
        int n = 0;
        for (int s = 0; s < G; ++s) {
            int nc, no, ovf;
            bool bad;
            ep_recv_counts(meta, s, e, Eg, C, S, nc, no, ovf, bad);
            n += nc + no;
            any_bad |= bad;
        }
        sm.hist[e] = n;
    }
    if (any_bad) atomicOr(lws.status, MOE_DEV_BAD_ROW);
    __syncthreads();
    // offsets, local schedule (uncapped layout of the local experts)
    build_schedule_block(sm, Eg, 0, false, loc_counts, loc_offsets, lws);
    for (int i = tid; i < G * Eg; i += kScanThreads) {
        const int s = i / Eg, e = i % Eg;
        int row = sm.offs[e];
        int nc, no, ovf;
        bool bad;
        for (int s2 = 0; s2 < s; ++s2) {
            ep_recv_counts(meta, s2, e, Eg, C, S, nc, no, ovf, bad);
            row += nc + no;
        }
        ep_recv_counts(meta, s, e, Eg, C, S, nc, no, ovf, bad);
        cap_seg[i] = make_int4(s * Eg * C + e * C, row, nc, 0);
        ovf_seg[i] = make_int4(s * S + ovf, row + nc, no, 0);
    }
}

// Row copies: segment i moves rows [src, src + len) of `a` to [dst, dst + len)
// of `b` (reverse: from b's dst rows to a's src rows).  A block per segment
// (grid-stride), a warp per row, 16-byte vectors.
__global__ void __launch_bounds__(kSegThreads) k_copy_segments(const uint4 *a, uint4 *b, const uint4 *rb, uint4 *ra,
                                                               int H8, const int4 *seg, int nseg, int reverse) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = blockIdx.x; i < nseg; i += gridDim.x) {
        const int4 sg = seg[i];
        for (int r = warp; r < sg.z; r += kSegThreads / 32) {
            const uint4 *src = reverse ? rb + (size_t)(sg.y + r) * H8 : a + (size_t)(sg.x + r) * H8;
            uint4 *dst = reverse ? ra + (size_t)(sg.x + r) * H8 : b + (size_t)(sg.y + r) * H8;
            for (int v = lane; v < H8; v += 32) dst[v] = __ldg(src + v);
        }
    }
}

}  // namespace

// Overflow slot rows per (source, destination): min(k, E/G) * max(0, T - C).
int64_t ep_overflow_rows(const moe_shape &s, int G) {
    const int Eg = s.E / G;
    return (int64_t)(s.k < Eg ? s.k : Eg) * (s.T > s.C ? s.T - s.C : 0);
}

// EP workspace: pack segments [G], capacity and overflow receive segments
// [E] each, local counts [E/G], local offsets [E/G + 1] (all 16-byte units).
size_t ep_workspace_bytes(const moe_shape &s, int G) {
    const int Eg = s.E / G;
    return 16 * ((size_t)G + 2 * (size_t)s.E) + 4 * align_up((size_t)(2 * Eg + 1), 4);
}

struct EpWs {
    int4 *pack_seg, *cap_seg, *ovf_seg;
    int32_t *loc_counts, *loc_offsets;
};
static EpWs ep_ptrs(void *ep_ws, const moe_shape &s, int G) {
    char *b = (char *)ep_ws;
    EpWs p;
    p.pack_seg = (int4 *)b;
    p.cap_seg = p.pack_seg + G;
    p.ovf_seg = p.cap_seg + s.E;
    p.loc_counts = (int32_t *)(p.ovf_seg + s.E);
    p.loc_offsets = p.loc_counts + s.E / G;
    return p;
}

// Source side: counts per destination into send_meta, each destination's
// overflow rows of x_perm into its slot of send_ovf ([G][S] rows).
cudaError_t launch_ep_pack(const moe_shape &s, int G, const void *x_perm, const WsLayout &L, void *ws, void *send_ovf,
                           int32_t *send_meta, void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G);
    cudaError_t e = launch_pdl(k_ep_plan_send, dim3(1), dim3(kSegThreads), 0, stream, ws_ptrs(ws, L), s.E, G, s.C, S,
                               send_meta, p.pack_seg);
    if (e != cudaSuccess) return e;
    int grid = G < num_sms ? G : num_sms;
    return launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)x_perm,
                      (uint4 *)send_ovf, (const uint4 *)nullptr, (uint4 *)nullptr, s.H / 8, (const int4 *)p.pack_seg, G,
                      0);
}

// Receiving side: the local layout, its GEMM schedule in the local workspace,
// and the received rows gathered into x_loc.
cudaError_t launch_ep_local_dispatch(const moe_shape &s, int G, const int32_t *recv_meta, const void *recv_cap,
                                     const void *recv_ovf, void *x_loc, const WsLayout &Lloc, void *ws_loc,
                                     void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int S = (int)ep_overflow_rows(s, G), Eg = s.E / G;
    cudaError_t e = launch_pdl(k_ep_plan_recv, dim3(1), dim3(kScanThreads), 0, stream, recv_meta, G, Eg, s.C, S,
                               p.cap_seg, p.ovf_seg, p.loc_counts, p.loc_offsets, ws_ptrs(ws_loc, Lloc));
    if (e != cudaSuccess) return e;
    const int grid = s.E < 4 * num_sms ? s.E : 4 * num_sms;
    e = launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)recv_cap, (uint4 *)x_loc,
                   (const uint4 *)nullptr, (uint4 *)nullptr, s.H / 8, (const int4 *)p.cap_seg, s.E, 0);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)recv_ovf,
                      (uint4 *)x_loc, (const uint4 *)nullptr, (uint4 *)nullptr, s.H / 8, (const int4 *)p.ovf_seg, s.E,
                      0);
}

// Receiving side, after the local experts: y_loc rows back to where their
// inputs came from (the capacity and overflow send buffers of the return
// passes).
cudaError_t launch_ep_local_return(const moe_shape &s, int G, const void *y_loc, void *back_cap, void *back_ovf,
                                   void *ep_ws, int num_sms, cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int grid = s.E < 4 * num_sms ? s.E : 4 * num_sms;
    cudaError_t e = launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)nullptr,
                               (uint4 *)nullptr, (const uint4 *)y_loc, (uint4 *)back_cap, s.H / 8,
                               (const int4 *)p.cap_seg, s.E, 1);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)nullptr,
                      (uint4 *)nullptr, (const uint4 *)y_loc, (uint4 *)back_ovf, s.H / 8, (const int4 *)p.ovf_seg, s.E,
                      1);
}

// Source side, after the return passes: the overflow rows' results from
// their slots back into y's overflow rows (the pack copies reversed).
cudaError_t launch_ep_unpack(const moe_shape &s, int G, const void *recv_back_ovf, void *y, void *ep_ws, int num_sms,
                             cudaStream_t stream) {
    const EpWs p = ep_ptrs(ep_ws, s, G);
    const int grid = G < num_sms ? G : num_sms;
    return launch_pdl(k_copy_segments, dim3(grid), dim3(kSegThreads), 0, stream, (const uint4 *)nullptr,
                      (uint4 *)nullptr, (const uint4 *)recv_back_ovf, (uint4 *)y, s.H / 8, (const int4 *)p.pack_seg, G,
                      1);
}

}  // namespace moe
