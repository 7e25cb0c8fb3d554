// Block-level pieces of the dispatch step (steps 2-3), shared by the
// multi-block dispatch kernels and by the router's fused tail for small
// batches: the schedule builder (offsets, capacity-plus-overflow layout,
// row cap, expert order, tile map) and the stable rank of a range of routed
// pairs.  Every function here is called by all kScanThreads threads of one
// block and synchronises that block only.
//
// Definitions followed: "TritonMoE" verdict page, arXiv 2605.23911 (tokens
// reordered onto experts by a histogram, an exclusive scan and a stable
// permutation) and the "Cap-and-Spill" critique, juhe.plus, section
// "Cap-and-Spill" (the first C rows of an expert in its capacity slots, the
// rest appended to one compacted overflow region, none dropped).
#pragma once

#include "common.cuh"

namespace moe {

// Shared-memory scratch of one dispatching block (16-byte aligned: the
// expert order reads hist as int4).
struct alignas(16) DispatchSmem {
    int hist[kMaxExperts];        // per-expert totals (-1 past E, up to a multiple of 4)
    int offs[kMaxExperts + 1];    // exclusive offsets of the uncapped layout
    int spoff[kMaxExperts + 1];   // exclusive offsets in the overflow region
    int tstart[kMaxExperts + 1];  // first tile of the g-th expert of the schedule order
    int rank[kMaxExperts];        // expert -> position in schedule order
    int order[kMaxExperts];       // position -> expert
    int ntiles[kMaxExperts];      // tiles per expert
    int running[kMaxExperts];     // rank: pairs of each expert before the current range
    int wcnt[kScanThreads / 32][kMaxExperts];  // rank: per-warp counts, then per-warp bases
    int wsum[2][kScanThreads / 32];            // block scan: warp totals
    int cap;                      // row cap of the tiles
    int flag;                     // scratch flag (bad expert id seen)
};

// Inclusive sum over the block of (a, b), one pair per thread (all
// kScanThreads threads call it; it synchronises the block twice).
__device__ __forceinline__ void block_inclusive_scan2(DispatchSmem &sm, int &a, int &b) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int ua = __shfl_up_sync(0xffffffffu, a, off), ub = __shfl_up_sync(0xffffffffu, b, off);
        if (lane >= off) {
            a += ua;
            b += ub;
        }
    }
    if (lane == 31) {
        sm.wsum[0][warp] = a;
        sm.wsum[1][warp] = b;
    }
    __syncthreads();
    for (int w = 0; w < warp; ++w) {
        a += sm.wsum[0][w];
        b += sm.wsum[1][w];
    }
    __syncthreads();  // wsum may be reused by the next scan
}

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

// Tiles of one expert: its row segments (uncapped: one; capacity layout:
// capacity slots then overflow) are cut into pieces and packed into tiles of
// at most `cap` rows, each piece starting on a 16-row boundary of the tile and
// at most two pieces per tile.  Emits if `out` is non-null; returns the tile
// count.
__device__ inline int pack_expert_tiles(int e, int seg0_start, int seg0_len, int seg1_start, int seg1_len, int cap,
                                        int4 *out) {
    int ntiles = 0, used = 0, np = 0;
    int p_start[2] = {0, 0}, p_len[2] = {0, 0};
    const int seg_start[2] = {seg0_start, seg1_start};
    const int seg_len[2] = {seg0_len, seg1_len};
    for (int s = 0; s < 2; ++s) {
        int start = seg_start[s], len = seg_len[s];
        while (len > 0) {
            if (used == cap || np == 2) {
                if (out) out[ntiles] = make_int4(e, p_start[0], p_len[0] | (p_len[1] << 16), p_start[1]);
                ++ntiles;
                used = 0;
                np = 0;
                p_len[1] = 0;
                p_start[1] = 0;
            }
            const int take = len < cap - used ? len : cap - used;
            p_start[np] = start;
            p_len[np] = take;
            ++np;
            used += round16(take);
            start += take;
            len -= take;
        }
    }
    if (np > 0) {
        if (out) out[ntiles] = make_int4(e, p_start[0], p_len[0] | (p_len[1] << 16), p_start[1]);
        ++ntiles;
    }
    return ntiles;
}

// From the per-expert totals in sm.hist: the exclusive offsets, the capacity
// layout (capacity count, overflow count and overflow offset per expert), the
// tile row cap, the expert order (descending count, ties by index) and the
// tile map, written to the caller's counts/offsets and to the workspace.  The
// offsets stay in sm.offs / sm.spoff for rank_pairs_block.
__device__ inline void build_schedule_block(DispatchSmem &sm, int E, int C, bool capped, int *counts_out,
                                            int *offsets_out, const WsPtrs &ws) {
    static_assert(kMaxExperts == kScanThreads, "one expert per thread");
    const int tid = threadIdx.x;
    const int E4 = (E + 3) & ~3;
    if (tid >= E && tid < E4) sm.hist[tid] = -1;  // never counted by the order below
    if (tid == 0) sm.cap = 16;
    const int n = tid < E ? sm.hist[tid] : 0;
    const int capn = capped ? min(n, C) : n;
    int incl_n = n, incl_s = n - capn;
    block_inclusive_scan2(sm, incl_n, incl_s);
    if (tid < E) {
        sm.offs[tid] = incl_n - n;
        sm.spoff[tid] = incl_s - (n - capn);
        offsets_out[tid] = incl_n - n;
        ws.offsets[tid] = incl_n - n;
        ws.spill_off[tid] = incl_s - (n - capn);
        counts_out[tid] = n;
        ws.counts[tid] = n;
        ws.cap_cnt[tid] = capn;
        ws.spill_cnt[tid] = n - capn;
        // Row cap of the tiles: the largest padded row count of one expert
        // (its capacity piece and its overflow piece each start on a 16-row
        // boundary), capped at kTileRows.  Below the cap every expert is one
        // tile, and the GEMM uses the spare shared memory for deeper
        // pipelining.
        atomicMax(&sm.cap, min(round16(capn) + round16(n - capn), kTileRows));
    }
    if (tid == E - 1) {
        sm.offs[E] = incl_n;
        sm.spoff[E] = incl_s;
        offsets_out[E] = incl_n;
        ws.offsets[E] = incl_n;
        ws.spill_off[E] = incl_s;
        *ws.total_spill = incl_s;
    }
    __syncthreads();
    const int row_cap = sm.cap;
    if (tid == 0) *ws.tile_rows = row_cap;
    // Expert order: descending count, ties by index (largest work first).
    int nt = 0;
    if (tid < E) {
        int r = 0;
        const int4 *h4 = reinterpret_cast<const int4 *>(sm.hist);
        for (int f4 = 0; f4 < E4 / 4; ++f4) {
            const int4 m = h4[f4];
            const int f = 4 * f4;
            r += (m.x > n) || (m.x == n && f < tid);
            r += (m.y > n) || (m.y == n && f + 1 < tid);
            r += (m.z > n) || (m.z == n && f + 2 < tid);
            r += (m.w > n) || (m.w == n && f + 3 < tid);
        }
        sm.rank[tid] = r;
        sm.order[r] = tid;
        ws.order[r] = tid;
        if (n > 0)
            nt = capped ? pack_expert_tiles(tid, tid * C, capn, E * C + sm.spoff[tid], n - capn, row_cap, nullptr)
                        : pack_expert_tiles(tid, sm.offs[tid], n, 0, 0, row_cap, nullptr);
        sm.ntiles[tid] = nt;
    }
    __syncthreads();
    // First tile of each expert in schedule order.
    const int ng = tid < E ? sm.ntiles[sm.order[tid]] : 0;
    int incl_t = ng, unused = 0;
    block_inclusive_scan2(sm, incl_t, unused);
    if (tid < E) {
        sm.tstart[tid] = incl_t - ng;
        ws.grp_tile_start[tid] = incl_t - ng;
    }
    if (tid == E - 1) {
        sm.tstart[E] = incl_t;
        ws.grp_tile_start[E] = incl_t;
        *ws.num_tiles = incl_t;
    }
    __syncthreads();
    if (tid < E && n > 0) {
        int4 *dst = ws.tile_map + sm.tstart[sm.rank[tid]];
        if (capped)
            pack_expert_tiles(tid, tid * C, capn, E * C + sm.spoff[tid], n - capn, row_cap, dst);
        else
            pack_expert_tiles(tid, sm.offs[tid], n, 0, 0, row_cap, dst);
    }
    __syncthreads();
}

// Stable rank of the routed pairs [begin, end) (flat index i = t * k + j)
// among the pairs of their expert, given sm.running[e] = pairs of expert e
// before `begin` and the offsets in sm.offs / sm.spoff; writes dest_row[i] and
// src_token[dest_row[i]] = i / k.  expert_of(i) returns the expert of pair i,
// or -1 for an invalid id.  Each warp takes a contiguous slice of the range:
// one pass counts its pairs per expert (warp match masks), a block-wide
// prefix over the warps turns the counts into bases, and a second pass
// assigns the ranks; `running` ends up advanced past the range.
template <class ExpertOf>
__device__ inline void rank_pairs_block(DispatchSmem &sm, ExpertOf expert_of, int begin, int end, int E, int k, int C,
                                        bool capped, int P, int *dest_row, int *src_token, const WsPtrs &ws) {
    constexpr int W = kScanThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (((end - begin) + W - 1) / W + 31) & ~31;
    const int w0 = begin + warp * per, w1 = min(end, w0 + per);
    int *cnt = sm.wcnt[warp];
    for (int e = lane; e < E; e += 32) cnt[e] = 0;
    __syncwarp();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
        const int i = base + lane;
        const int e = i < w1 ? expert_of(i) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & lt_mask) == 0) cnt[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < E; e += kScanThreads) {
        int run = sm.running[e];
        for (int w = 0; w < W; ++w) {
            const int c = sm.wcnt[w][e];
            sm.wcnt[w][e] = run;
            run += c;
        }
        sm.running[e] = run;
    }
    __syncthreads();
    for (int base = w0; base < w1; base += 32) {
        const int i = base + lane;
        const int e = i < w1 ? expert_of(i) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
            const int r = cnt[e] + __popc(peers & lt_mask);
            int row;
            if (!capped)
                row = sm.offs[e] + r;
            else if (r < C)
                row = e * C + r;
            else
                row = E * C + sm.spoff[e] + (r - C);
            if ((unsigned)row < (unsigned)P) {
                dest_row[i] = row;
                src_token[row] = i / k;
            } else {
                dest_row[i] = -1;
                atomicOr(ws.status, MOE_DEV_BAD_ROW);
            }
        } else if (i < w1) {
            dest_row[i] = -1;
        }
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) cnt[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
}

}  // namespace moe
