// Steps 2-3: per-expert histogram, exclusive scan and stable permutation of
// the routed (token, slot) pairs into expert-contiguous order ("TritonMoE"
// verdict page, arXiv 2605.23911: tokens reordered onto experts), with the
// optional capacity-plus-compacted-overflow layout ("Cap-and-Spill" critique,
// juhe.plus, section "Cap-and-Spill"), and the device-built tile schedule of
// the grouped GEMMs.
//
// k_hist_scan  one pass over topk_idx.  Each block takes a ticket (its block
//              index in launch-independent order), histograms its chunk of
//              1024 pairs in shared memory and resolves, per expert, the count
//              of that expert in all earlier chunks by decoupled look-back
//              over per-(chunk, expert) flag words, kLookback chunks per
//              read.  The block holding the
//              last chunk owns the totals and builds the per-expert offsets,
//              the capacity/overflow offsets and the GEMM tile schedule, all
//              on the device: nothing goes back to the host.
// k_rank       each block re-reads its chunk and ranks every pair among the
//              pairs of its expert (stable: earlier flat index = lower rank),
//              using warp match masks and per-warp counts, and writes
//              dest_row / src_token.
// k_gather     x_perm[row] = x[src_token[row]] with 16-byte loads and stores,
//              zero rows for unfilled capacity slots.
#include <cuda_bf16.h>

#include "dispatch_block.cuh"

namespace moe {

namespace {

struct ScanArgs {
    const int *topk_idx;
    int T, E, k, C, capped, R;
    int stall_first_block;  // test hook: block 0 never publishes
    unsigned long long timeout_ns;
    int *counts_out;   // caller's expert_counts [E]
    int *offsets_out;  // caller's expert_offsets [E+1]
    WsPtrs ws;
};

__global__ void __launch_bounds__(kScanThreads) k_hist_scan(ScanArgs a) {
    __shared__ DispatchSmem sm;
    int *hist = sm.hist;
    __shared__ int s_chunk, s_bad, s_timeout;
    const int tid = threadIdx.x, E = a.E;
    pdl_trigger();
    if (tid == 0) {
        s_chunk = (int)atomicAdd(a.ws.ticket, 1u);
        s_bad = 0;
        s_timeout = 0;
    }
    for (int e = tid; e < E; e += kScanThreads) hist[e] = 0;
    __syncthreads();
    const int chunk = s_chunk;
    const int begin = chunk * kScanChunk;
    const int end = min(a.R, begin + kScanChunk);
    for (int i = begin + tid; i < end; i += kScanThreads) {
        const int e = a.topk_idx[i];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&hist[e], 1);
        else
            s_bad = 1;
    }
    __syncthreads();
    if (tid == 0 && s_bad) atomicOr(a.ws.status, MOE_DEV_BAD_EXPERT);

    // Decoupled look-back, one thread per expert.
    const bool last = (chunk == a.ws.nchunks - 1);
    for (int e = tid; e < E; e += kScanThreads) {
        const int agg = hist[e];
        unsigned long long *mine = a.ws.scan_state + (size_t)chunk * E + e;
        const bool publish = !(a.stall_first_block && chunk == 0);
        int excl = 0;
        if (chunk == 0) {
            if (publish) st_release_u64(mine, ((unsigned long long)kFlagPrefix << 32) | (uint32_t)agg);
        } else {
            st_release_u64(mine, ((unsigned long long)kFlagAggregate << 32) | (uint32_t)agg);
            // Look back over windows of kLookback predecessors, all of a
            // window's words read at once: add the aggregates from the
            // nearest chunk backwards until an inclusive prefix (chunk 0
            // always publishes one).  A predecessor that has not published
            // yet stops the walk there, and the window is read again after a
            // short sleep (bounded by the timeout).  Every word holds its flag
            // and value together, so relaxed loads suffice.
            int p = chunk - 1;
            uint64_t deadline = 0;
            while (true) {
                unsigned long long v[kLookback];
#pragma unroll
                for (int i = 0; i < kLookback; ++i)
                    v[i] = p - i >= 0 ? ld_relaxed_u64(a.ws.scan_state + (size_t)(p - i) * E + e)
                                      : ((unsigned long long)kFlagPrefix << 32);  // before chunk 0: prefix 0
                int used = 0;
                bool done = false, blocked = false;
#pragma unroll
                for (int i = 0; i < kLookback; ++i) {
                    const uint32_t flag = (uint32_t)(v[i] >> 32);
                    if (done || blocked) continue;
                    if (flag == 0u) {
                        blocked = true;
                        continue;
                    }
                    excl += (int)(uint32_t)v[i];
                    ++used;
                    done = flag == kFlagPrefix;
                }
                p -= used;
                if (done) break;
                if (blocked) {
                    const uint64_t now = globaltimer_ns();
                    if (deadline == 0) {
                        deadline = now + a.timeout_ns;
                    } else if (now > deadline) {
                        s_timeout = 1;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            st_release_u64(mine, ((unsigned long long)kFlagPrefix << 32) | (uint32_t)(excl + agg));
        }
        a.ws.chunk_excl[(size_t)chunk * E + e] = excl;
        if (last) hist[e] = excl + agg;  // totals
    }
    __syncthreads();
    if (tid == 0 && s_timeout) atomicOr(a.ws.status, MOE_DEV_SCAN_TIMEOUT);
    if (!last) return;

    // ---- the block with the last chunk: offsets, capacity layout, schedule ----
    build_schedule_block(sm, E, a.C, a.capped != 0, a.counts_out, a.offsets_out, a.ws);
}

struct RankArgs {
    const int *topk_idx;
    int E, k, C, capped, R, P;
    int *dest_row;
    int *src_token;
    WsPtrs ws;
};

__global__ void __launch_bounds__(kScanThreads) k_rank(RankArgs a) {
    __shared__ DispatchSmem sm;
    pdl_trigger();
    pdl_wait();
    const int chunk = blockIdx.x;
    for (int e = threadIdx.x; e <= a.E; e += kScanThreads) {
        if (e < a.E) sm.running[e] = a.ws.chunk_excl[(size_t)chunk * a.E + e];
        sm.offs[e] = a.ws.offsets[e];
        sm.spoff[e] = a.ws.spill_off[e];
    }
    const int begin = chunk * kScanChunk, end = min(a.R, begin + kScanChunk);
    const int *topk_idx = a.topk_idx;
    const int E = a.E;
    auto expert_of = [topk_idx, E](int i) {
        const int e = topk_idx[i];
        return (unsigned)e < (unsigned)E ? e : -1;
    };
    rank_pairs_block(sm, expert_of, begin, end, a.E, a.k, a.C, a.capped != 0, a.P, a.dest_row, a.src_token, a.ws);
}

// One warp per permuted row; rows are [0, R) uncapped, or the E*C capacity
// slots plus the used part of the overflow region.  The rows are written with
// streaming (evict-first) stores: x_perm is k times larger than x, and a
// token's k copies are made at different times, so ordinary stores would
// evict x from L2 between them and every copy would re-read it from DRAM.
__global__ void __launch_bounds__(256) k_gather(const uint4 *__restrict__ x, const int *__restrict__ src_token,
                                                uint4 *__restrict__ x_perm, int H8, int T, int P, int fixed_rows,
                                                int cap_rows, const int *total_spill) {
    pdl_trigger();
    pdl_wait();
    int rows = fixed_rows >= 0 ? fixed_rows : cap_rows + *total_spill;
    if (rows > P) rows = P;
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    for (int row = gw; row < rows; row += nw) {
        const int t = src_token[row];
        uint4 *dst = x_perm + (size_t)row * H8;
        if ((unsigned)t < (unsigned)T) {
            const uint4 *src = x + (size_t)t * H8;
            int v = lane;
            // eight 16-byte loads per lane in flight before the stores
            for (; v + 224 < H8; v += 256) {
                uint4 q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __ldg(src + v + 32 * i);
#pragma unroll
                for (int i = 0; i < 8; ++i) __stcs(dst + v + 32 * i, q[i]);
            }
            for (; v < H8; v += 32) __stcs(dst + v, __ldg(src + v));
        } else {
            for (int v = lane; v < H8; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

}  // namespace

// x_perm[row] = x[src_token[row]] for every filled permuted row.
cudaError_t launch_gather(const moe_shape &s, const void *x, const int32_t *src_token, void *x_perm,
                          const WsLayout &L, void *ws, int num_sms, cudaStream_t stream) {
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int R = s.T * s.k;
    const int P = (int)permuted_rows(s.T, s.E, s.k, s.C, capped);
    WsPtrs p = ws_ptrs(ws, L);
    const int H8 = s.H / 8;
    const int fixed = capped ? -1 : R;
    const int rows_hint = capped ? s.E * s.C + s.k * (s.T > s.C ? s.T - s.C : 0) : R;
    int blocks = (rows_hint + 7) / 8;  // 8 warps per block, one row each
    const int cap_blocks = num_sms * 8;
    if (blocks > cap_blocks) blocks = cap_blocks;
    if (blocks < 1) blocks = 1;
    return launch_pdl(k_gather, dim3(blocks), dim3(256), 0, stream, (const uint4 *)x, src_token, (uint4 *)x_perm, H8,
                      s.T, P, fixed, s.E * s.C, (const int *)p.total_spill);
}

// Histogram, scan, schedule and ranks (moe_permute without the row copy).
cudaError_t launch_dispatch_index(const moe_shape &s, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                                  int32_t *src_token, int32_t *dest_row, const WsLayout &L, void *ws,
                                  uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
    (void)num_sms;
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int R = s.T * s.k;
    WsPtrs p = ws_ptrs(ws, L);
    cudaError_t err = cudaMemsetAsync((char *)ws + L.reset_begin, 0, L.reset_end - L.reset_begin, stream);
    if (err != cudaSuccess) return err;
    if (capped) {
        const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, true);
        err = cudaMemsetAsync(src_token, 0xFF, sizeof(int32_t) * (size_t)P, stream);
        if (err != cudaSuccess) return err;
    }
    ScanArgs sa;
    sa.topk_idx = topk_idx;
    sa.T = s.T;
    sa.E = s.E;
    sa.k = s.k;
    sa.C = s.C;
    sa.capped = capped;
    sa.R = R;
    sa.stall_first_block = (s.flags & MOE_FLAG_TEST_STALL_SCAN) ? 1 : 0;
    sa.timeout_ns = timeout_ns;
    sa.counts_out = counts;
    sa.offsets_out = offsets;
    sa.ws = p;
    k_hist_scan<<<L.nchunks, kScanThreads, 0, stream>>>(sa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    RankArgs ra;
    ra.topk_idx = topk_idx;
    ra.E = s.E;
    ra.k = s.k;
    ra.C = s.C;
    ra.capped = capped;
    ra.R = R;
    ra.P = (int)permuted_rows(s.T, s.E, s.k, s.C, capped);
    ra.dest_row = dest_row;
    ra.src_token = src_token;
    ra.ws = p;
    return launch_pdl(k_rank, dim3(L.nchunks), dim3(kScanThreads), 0, stream, ra);
}

cudaError_t launch_permute(const moe_shape &s, const void *x, const int32_t *topk_idx, int32_t *counts,
                           int32_t *offsets, int32_t *src_token, int32_t *dest_row, void *x_perm, const WsLayout &L,
                           void *ws, uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
    cudaError_t err =
        launch_dispatch_index(s, topk_idx, counts, offsets, src_token, dest_row, L, ws, timeout_ns, num_sms, stream);
    if (err != cudaSuccess) return err;
    return launch_gather(s, x, src_token, x_perm, L, ws, num_sms, stream);
}

}  // namespace moe
