// Step 1: router scoring ("TritonMoE" verdict page, arXiv 2605.23911, referee
// report summary).  logits = x * W_r (+ bias) in fp32, then per token the k
// largest logits (equal logits to the lower expert index, NaN lowest) and the
// softmax over the k selected logits.
//
// The logits are a small fp32 GEMM (T x H times H x E, E <= 256) that is
// latency-bound at decode sizes and FMA-bound at prefill sizes:
// - A CTA of 8 warps owns TB tokens (16, 8 or 4: fewer for more experts) and
//   all E experts for a slice of the hidden dimension.  When there are few
//   token blocks, the hidden dimension is split over a thread-block cluster of
//   CL CTAs (CL <= 8) so that about 3/4 of the SMs get a CTA; rank r of the
//   cluster sums the CL partial logits of tokens r, r + CL, ... through
//   distributed shared memory, in rank order (deterministic), and runs their
//   top-k.
// - x and W_r stream through shared memory in chunks of HC hidden units with
//   a 2-4 stage cp.async pipeline.  The 8 warps split each chunk's hidden
//   units; inside a warp ES lanes split the experts (EJ consecutive experts
//   each) and HS = 32/ES lanes the hidden pairs.  Each thread holds a TB x EJ
//   tile of sums, so every weight value it reads feeds TB multiply-adds; the
//   warps' partial sums are added in warp order.
// - Top-k: one warp per token, each lane holding ceil(E/32) candidates,
//   sorted once per lane; k rounds of a warp max of the lanes' first orderable
//   logit and a warp min of the expert index among the lanes holding that
//   maximum (redux.sync), the winning lane dropping its first candidate.
// - Logits computed elsewhere (given by the caller, or the tensor-core
//   router's partial planes for large batches) go to k_topk: one warp per
//   token loads its logits straight into registers, no CTA-wide staging.
// - Fused dispatch (small batches, called from moe_forward): every CTA that
//   finished its top-k takes a ticket after a memory fence; the CTA that takes
//   the last one (no CTA ever waits for another) builds the whole dispatch of
//   steps 2-3 for all T*k pairs in its shared memory: histogram, scan,
//   capacity layout, GEMM schedule and stable ranks.
#include <cuda_bf16.h>

#include "dispatch_block.cuh"

namespace moe {

namespace {

// Dynamic shared memory of a router CTA, at most.
constexpr int kRouteSmemMax = 200 * 1024;

struct RouteArgs {
    const __nv_bfloat16 *x;
    const float *w_router;
    const float *bias;
    float *logits;  // output (or input with logits_in and no lparts); may be null when output
    const float *lparts;  // logits_in from the tensor cores: lq partial planes [lq][T][E] (bias not added)
    int lq;
    int *topk_idx;
    float *topk_w;
    uint32_t *status;
    int T, H, E, k;
    int logits_in;
    int hc;           // hidden units per pipeline chunk (power of two, >= 64, divides slice)
    int stages;       // cp.async pipeline depth (2..4)
    int stage_bytes;  // bytes of one stage (16-byte multiple)
    int cl;           // CTAs per cluster splitting the hidden dimension
    int slice;        // hidden units per CTA = H / cl
    int es;           // lanes across experts (power of two <= 32)
    int part_off;     // byte offset of the partial-logit tile in dynamic shared memory
    // fused dispatch (fuse != 0)
    int fuse;
    int C, capped, P;
    FusedDispatch out;
    WsPtrs ws;
};

// The last router CTA to finish: the dispatch of all T*k routed pairs, in the
// dynamic shared memory (DispatchSmem, then the pairs' experts).
__device__ void fused_dispatch_tail(const RouteArgs &a, uint8_t *smem) {
    DispatchSmem &sm = *reinterpret_cast<DispatchSmem *>(smem);
    int *pairs = reinterpret_cast<int *>(smem + sizeof(DispatchSmem));
    const int tid = threadIdx.x, E = a.E, R = a.T * a.k;
    for (int e = tid; e < E; e += kScanThreads) {
        sm.hist[e] = 0;
        sm.running[e] = 0;
    }
    if (tid == 0) sm.flag = 0;
    __syncthreads();
    // All loads first (one L2 round trip), then the histogram.  The pairs were
    // written by other CTAs: read them from L2.
    constexpr int kPer = kFusedDispatchMaxPairs / kScanThreads;
    int v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * kScanThreads;
        v[j] = i < R ? __ldcg(a.topk_idx + i) : 0;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = tid + j * kScanThreads;
        if (i >= R) break;
        const int e = v[j];
        if ((unsigned)e < (unsigned)E) {
            pairs[i] = e;
            atomicAdd(&sm.hist[e], 1);
        } else {
            pairs[i] = -1;
            sm.flag = 1;
        }
    }
    __syncthreads();
    if (tid == 0 && sm.flag) atomicOr(a.status, MOE_DEV_BAD_EXPERT);
    build_schedule_block(sm, E, a.C, a.capped != 0, a.out.counts, a.out.offsets, a.ws);
    if (a.capped) {
        // Rows no pair fills: the capacity slots past each expert's count and
        // the overflow rows past the total overflow.
        for (int i = tid; i < E * a.C; i += kScanThreads)
            if (i % a.C >= min(sm.hist[i / a.C], a.C)) a.out.src_token[i] = -1;
        for (int i = E * a.C + sm.spoff[E] + tid; i < a.P; i += kScanThreads) a.out.src_token[i] = -1;
    }
    auto expert_of = [pairs](int i) { return pairs[i]; };
    rank_pairs_block(sm, expert_of, 0, R, E, a.k, a.C, a.capped != 0, a.P, a.out.dest_row, a.out.src_token, a.ws);
    // Every router CTA has taken its ticket: the count starts at zero again.
    if (tid == 0) *a.ws.route_done = 0;
}

// Monotone map of a float onto uint32 (larger float -> larger key); -0 is
// folded onto +0 and NaN maps to 1, below -inf (whose key is 0x007FFFFF);
// key 0 marks an empty candidate slot.
__device__ __forceinline__ uint32_t orderable(float f) {
    if (f != f) return 1u;
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// The float of a key (+0 for a folded -0, a quiet NaN for the NaN key).
__device__ __forceinline__ float orderable_value(uint32_t k) {
    if (k == 1u) return __uint_as_float(0x7FC00000u);
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Reads a float at the same shared-memory offset in cluster CTA `rank`.
__device__ __forceinline__ float ld_cluster_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// logit = sum over q < lq of part[q * plane + i], in order q = 0, 1, ...,
// then + bias[0] when bias is given (the tensor-core router's partial
// planes of the hidden ranges).
__device__ __forceinline__ float sum_partials(const float *__restrict__ part, size_t plane, int lq, size_t i,
                                              const float *bias) {
    float l = part[i];
#pragma unroll 4
    for (int q = 1; q < lq; ++q) l += part[(size_t)q * plane + i];
    if (bias) l = l + *bias;
    return l;
}

// Top-k and softmax of one token by one warp.  Lane l holds the logits of
// experts l, l + 32, ..., l + 32 (MPL - 1) in v[] (MPL = 1, 2, 4 or 8 with
// E <= 32 MPL; entries past E are ignored).  Each lane first sorts its
// candidates (larger key first; a lane's candidates are in index order and
// the insertion sort is stable, so equal keys keep the lower index first).
// A round then takes the largest head key over the warp (redux max) and the
// lowest expert index among the lanes whose head holds it (redux min) -- the
// larger logit, ties to the lower index, NaN below every number -- and the
// winning lane pops its head.  Selected slot j lives in register j / 32 of
// lane j % 32, so the softmax needs no round trip through memory.  Writes
// idx[0..k) and w[0..k); returns true (in every lane) if a logit was NaN.
template <int MPL>
__device__ __forceinline__ bool warp_topk_softmax(const float (&v)[MPL], int E, int k, int *idx, float *w) {
    const int lane = threadIdx.x & 31;
    uint32_t key[MPL];
    int ix[MPL];
    bool nan = false;
#pragma unroll
    for (int m = 0; m < MPL; ++m) {
        const int e = lane + 32 * m;
        key[m] = 0u;
        ix[m] = 0x7FFFFFFF;
        if (e < E) {
            nan |= (v[m] != v[m]);
            key[m] = orderable(v[m]);
            ix[m] = e;
        }
    }
#pragma unroll
    for (int i = 1; i < MPL; ++i)
#pragma unroll
        for (int j = i; j > 0; --j)
            if (key[j] > key[j - 1]) {
                const uint32_t tk = key[j];
                key[j] = key[j - 1];
                key[j - 1] = tk;
                const int ti = ix[j];
                ix[j] = ix[j - 1];
                ix[j - 1] = ti;
            }
    float sel[MPL];  // k <= E <= 32 MPL slots
#pragma unroll
    for (int m = 0; m < MPL; ++m) sel[m] = 0.0f;
    float lmax = 0.0f;
    for (int j = 0; j < k; ++j) {
        const uint32_t wk = __reduce_max_sync(0xffffffffu, key[0]);
        const int e = (int)__reduce_min_sync(0xffffffffu, key[0] == wk ? (uint32_t)ix[0] : 0xFFFFFFFFu);
        if (ix[0] == e) {  // the owner pops its head
#pragma unroll
            for (int m = 0; m + 1 < MPL; ++m) {
                key[m] = key[m + 1];
                ix[m] = ix[m + 1];
            }
            key[MPL - 1] = 0u;
            ix[MPL - 1] = 0x7FFFFFFF;
        }
        const float l = orderable_value(wk);
        if (j == 0) lmax = l;
        if ((j & 31) == lane) {
#pragma unroll
            for (int m = 0; m < MPL; ++m)
                if (m == (j >> 5)) sel[m] = l;
        }
        if (lane == 0) idx[j] = e;
    }
    // Softmax over the k selected logits, reference = the largest (slot 0):
    // per-lane partial sums over slots lane, lane + 32, ..., then a butterfly
    // over the warp.
    float ex[MPL];
    float sum = 0.0f;
#pragma unroll
    for (int m = 0; m < MPL; ++m) {
        ex[m] = 0.0f;
        if (lane + 32 * m < k) {
            ex[m] = expf(sel[m] - lmax);
            sum += ex[m];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
    for (int m = 0; m < MPL; ++m)
        if (lane + 32 * m < k) w[lane + 32 * m] = ex[m] / sum;
    return __any_sync(0xffffffffu, nan);
}

// Candidates per lane for E experts: 1, 2, 4 or 8.
__host__ __device__ inline int topk_mpl(int E) { return E <= 32 ? 1 : (E <= 64 ? 2 : (E <= 128 ? 4 : 8)); }

// Top-k of logits already computed (caller-given, or the tensor-core
// router's partial planes), without the fused dispatch: one warp per token,
// the logits straight into registers (all of a lane's loads issued before
// the first is used), no shared-memory staging.
template <int MPL>
__global__ void __launch_bounds__(256) k_topk(RouteArgs a) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (t >= a.T) return;  // warp-uniform
    const int E = a.E;
    float v[MPL];
    if (a.lparts) {
        const size_t plane = (size_t)a.T * E;
#pragma unroll
        for (int m = 0; m < MPL; ++m) v[m] = lane + 32 * m < E ? a.lparts[(size_t)t * E + lane + 32 * m] : 0.0f;
#pragma unroll 4
        for (int q = 1; q < a.lq; ++q) {
            const float *pq = a.lparts + (size_t)q * plane + (size_t)t * E;
#pragma unroll
            for (int m = 0; m < MPL; ++m)
                if (lane + 32 * m < E) v[m] += pq[lane + 32 * m];
        }
#pragma unroll
        for (int m = 0; m < MPL; ++m) {
            const int e = lane + 32 * m;
            if (e < E) {
                if (a.bias) v[m] = v[m] + a.bias[e];
                if (a.logits) a.logits[(size_t)t * E + e] = v[m];
            }
        }
    } else {
#pragma unroll
        for (int m = 0; m < MPL; ++m) v[m] = lane + 32 * m < E ? a.logits[(size_t)t * E + lane + 32 * m] : 0.0f;
    }
    if (warp_topk_softmax<MPL>(v, E, a.k, a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k) && lane == 0)
        atomicOr(a.status, MOE_DEV_NAN_LOGIT);
}

// A lane's EJ consecutive experts of one weight row: one 8- or 16-byte load
// when they all exist (the row start and es * EJ are multiples of EJ floats),
// else clamped scalar loads (ecol[j] = min(es * EJ + j, E - 1); the values
// past E are never used).
template <int EJ>
__device__ __forceinline__ void load_weights(const float *row, int E, int es, const int *ecol, float *w) {
    if constexpr (EJ == 2 || EJ == 4) {
        if (es * EJ + EJ <= E && (E % EJ) == 0) {
            if constexpr (EJ == 2) {
                const float2 v = *reinterpret_cast<const float2 *>(row + es * EJ);
                w[0] = v.x;
                w[1] = v.y;
            } else {
                const float4 v = *reinterpret_cast<const float4 *>(row + es * EJ);
                w[0] = v.x;
                w[1] = v.y;
                w[2] = v.z;
                w[3] = v.w;
            }
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < EJ; ++j) w[j] = row[ecol[j]];
}

template <int TB, int EJ>
__global__ void __launch_bounds__(256) k_route(RouteArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_nan;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();  // the next kernel may set up while the router runs
    const int CL = a.cl;
    const int rank = CL > 1 ? (int)cluster_rank() : 0;
    const int t0 = (blockIdx.x / CL) * TB;
    const int E = a.E;
    if (tid == 0) s_nan = 0;
    // rank 0: the logits tile for the top-k, over the (finished) pipeline buffers
    float(*lg)[kMaxExperts + 1] = reinterpret_cast<float(*)[kMaxExperts + 1]>(smem);

    if (!a.logits_in) {
        float *part = reinterpret_cast<float *>(smem + a.part_off);  // [TB][E] partials of this slice
        const int HC = a.hc, S = a.stages, stage_bytes = a.stage_bytes;
        const int xbytes = TB * HC * 2;
        const int h_begin = rank * a.slice;
        const int nchunks = a.slice / HC;
        auto issue = [&](int c, int st) {
            uint8_t *sx = smem + (size_t)st * stage_bytes;
            float *sw = reinterpret_cast<float *>(sx + xbytes);
            const int h0 = h_begin + c * HC;
            const int vpr = HC / 8;  // 16-byte vectors per token row
            for (int i = tid; i < TB * vpr; i += 256) {
                const int tok = i / vpr, v = i % vpr, t = t0 + tok;
                void *dst = sx + ((size_t)tok * HC + v * 8) * 2;
                if (t < a.T)
                    cp_async16(dst, a.x + (size_t)t * a.H + h0 + v * 8);
                else
                    *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
            }
            const float *src = a.w_router + (size_t)h0 * E;  // rows h0 .. h0+HC: contiguous
            for (int i = tid; i < HC * E / 4; i += 256) cp_async16(sw + 4 * i, src + 4 * i);
        };
        // All 8 warps share the CTA's TB tokens and split each chunk's hidden
        // units (warp w takes pairs [w * PPW, (w + 1) * PPW)); inside a warp ES
        // lanes split the experts (EJ consecutive experts each) and HS = 32/ES
        // lanes the hidden pairs.  Each thread keeps a TB x EJ tile of sums, so
        // every weight value read from shared memory feeds TB multiply-adds.
        const int ES = a.es, HS = 32 / ES;
        const int es = lane % ES, hs = lane / ES;
        const int PPW = HC / 2 / 8;
        int ecol[EJ];
#pragma unroll
        for (int j = 0; j < EJ; ++j) ecol[j] = min(es * EJ + j, E - 1);  // reads past E are clamped, unused
        // sums of tokens 2i and 2i + 1 side by side: one packed fp32 FMA
        // (fma.rn.f32x2) updates both, each element rounded exactly as a
        // scalar fmaf would round it
        static_assert(TB % 2 == 0, "tokens are processed in pairs");
        float2 acc2[TB / 2][EJ];
#pragma unroll
        for (int i = 0; i < TB / 2; ++i)
#pragma unroll
            for (int j = 0; j < EJ; ++j) acc2[i][j] = make_float2(0.0f, 0.0f);

        for (int s = 0; s < S - 1; ++s) {
            if (s < nchunks) issue(s, s);
            cp_async_commit();
        }
        // x of the chunk in fp32, token pairs interleaved: x2[i][p] =
        // (x[2i][2p], x[2i+1][2p], x[2i][2p+1], x[2i+1][2p+1]), the two packed
        // operands of hidden units 2p and 2p+1 in one 16-byte load
        float4 *x2 = reinterpret_cast<float4 *>(smem + (size_t)S * stage_bytes);
        const int HP = HC / 2;
        for (int c = 0; c < nchunks; ++c) {
            if (c + S - 1 < nchunks) issue(c + S - 1, (c + S - 1) % S);
            cp_async_commit();
            cp_async_wait_pending(S - 1);  // this thread's copies of chunk c have landed
            __syncthreads();               // ... and everyone else's
            const uint8_t *sx = smem + (size_t)(c % S) * stage_bytes;
            const __nv_bfloat16 *xs = reinterpret_cast<const __nv_bfloat16 *>(sx);
            const float *wsm = reinterpret_cast<const float *>(sx + xbytes);
            for (int idx = tid; idx < (TB / 2) * HP; idx += 256) {
                const int i = idx / HP, p = idx - i * HP;
                const float2 xa =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(xs + (size_t)(2 * i) * HC + 2 * p));
                const float2 xb = __bfloat1622float2(
                    *reinterpret_cast<const __nv_bfloat162 *>(xs + (size_t)(2 * i + 1) * HC + 2 * p));
                x2[idx] = make_float4(xa.x, xb.x, xa.y, xb.y);
            }
            __syncthreads();
            // Pairs of hidden units 2p, 2p+1 of this warp's range; this lane
            // takes p = p0 + hs, p0 + hs + HS, ...
            const int p0 = warp * PPW;
            for (int p = p0 + hs; p < p0 + PPW; p += HS) {
                const float *w0 = wsm + (size_t)(2 * p) * E;
                float wa[EJ], wb[EJ];
                load_weights<EJ>(w0, E, es, ecol, wa);
                load_weights<EJ>(w0 + E, E, es, ecol, wb);
#pragma unroll
                for (int i = 0; i < TB / 2; ++i) {
                    const float4 xv = x2[i * HP + p];
                    const float2 x0 = make_float2(xv.x, xv.y), x1 = make_float2(xv.z, xv.w);
#pragma unroll
                    for (int j = 0; j < EJ; ++j) {
                        acc2[i][j] = __ffma2_rn(x0, make_float2(wa[j], wa[j]), acc2[i][j]);
                        acc2[i][j] = __ffma2_rn(x1, make_float2(wb[j], wb[j]), acc2[i][j]);
                    }
                }
            }
            __syncthreads();  // stage c % S and the fp32 tile may be refilled from here on
        }
        float acc[TB][EJ];
#pragma unroll
        for (int i = 0; i < TB / 2; ++i)
#pragma unroll
            for (int j = 0; j < EJ; ++j) {
                acc[2 * i][j] = acc2[i][j].x;
                acc[2 * i + 1][j] = acc2[i][j].y;
            }
        // Fold the hidden-pair split inside the warp, then the warps' partial
        // sums in warp order (deterministic) through shared memory, which the
        // pipeline no longer needs.
        for (int off = ES; off < 32; off <<= 1)
#pragma unroll
            for (int i = 0; i < TB; ++i)
#pragma unroll
                for (int j = 0; j < EJ; ++j) acc[i][j] += __shfl_xor_sync(0xffffffffu, acc[i][j], off);
        float *wpart = reinterpret_cast<float *>(smem);  // [8][TB][E]
        if (hs == 0) {
#pragma unroll
            for (int i = 0; i < TB; ++i)
#pragma unroll
                for (int j = 0; j < EJ; ++j) {
                    const int e = es * EJ + j;
                    if (e < E) wpart[(warp * TB + i) * E + e] = acc[i][j];
                }
        }
        __syncthreads();
        for (int i = tid; i < TB * E; i += 256) {
            float v = wpart[i];
            for (int w = 1; w < 8; ++w) v += wpart[w * TB * E + i];
            part[i] = v;
        }
        if (CL > 1)
            cluster_sync_all();
        else
            __syncthreads();
        // Rank r of the cluster takes tokens r, r + CL, ...: it sums their
        // slices in rank order (every token in the same order), adds the
        // bias, publishes their logits and runs their top-k below.
        const int mine = (TB - rank + CL - 1) / CL;  // tokens of this rank
        for (int i = tid; i < mine * E; i += 256) {
            const int tok = rank + CL * (i / E), e = i % E, t = t0 + tok;
            const int pi = tok * E + e;
            float l = CL > 1 ? ld_cluster_f32(part + pi, 0u) : part[pi];
            for (int r = 1; r < CL; ++r) l += ld_cluster_f32(part + pi, (uint32_t)r);
            if (a.bias) l = l + a.bias[e];
            lg[tok][e] = l;
            if (t < a.T && a.logits) a.logits[(size_t)t * E + e] = l;
        }
    } else if (a.lparts) {
        // Partial planes of the hidden ranges, added in range order, then
        // the bias; the logits are published for the caller.
        for (int i = tid; i < TB * E; i += 256) {
            const int tok = i / E, e = i % E, t = t0 + tok;
            float l = 0.0f;
            if (t < a.T) {
                l = sum_partials(a.lparts, (size_t)a.T * E, a.lq, (size_t)t * E + e, a.bias ? a.bias + e : nullptr);
                if (a.logits) a.logits[(size_t)t * E + e] = l;
            }
            lg[tok][e] = l;
        }
    } else {
        for (int i = tid; i < TB * E; i += 256) {
            const int tok = i / E, e = i % E, t = t0 + tok;
            lg[tok][e] = t < a.T ? a.logits[(size_t)t * E + e] : 0.0f;
        }
    }
    __syncthreads();

    // Top-k, one warp per token (with a cluster: this rank's tokens).
    for (int tok = rank + CL * warp; tok < TB; tok += 8 * CL) {
        const int t = t0 + tok;
        if (t >= a.T) break;
        float v[EJ];
#pragma unroll
        for (int m = 0; m < EJ; ++m) v[m] = lane + 32 * m < E ? lg[tok][lane + 32 * m] : 0.0f;
        // EJ experts per lane in the sums above = ceil(E/32) rounded up to a power of two
        if (warp_topk_softmax<EJ>(v, E, a.k, a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k) && lane == 0)
            s_nan = 1;
    }
    __syncthreads();
    if (tid == 0 && s_nan) atomicOr(a.status, MOE_DEV_NAN_LOGIT);
    if (CL > 1) cluster_sync_all();  // every slice stays readable until the cluster has summed it
    if (a.fuse) {
        // Publish this CTA's top-k, then take a ticket; the last CTA sees every
        // other CTA's results after its own fence.
        __threadfence();
        __syncthreads();
        __shared__ int s_last;
        if (tid == 0) s_last = atomicAdd(a.ws.route_done, 1u) == gridDim.x - 1;
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        fused_dispatch_tail(a, smem);
    }
}

template <int TB, int EJ>
cudaError_t launch_one(const RouteArgs &a, int smem_bytes, int tiles, cudaStream_t stream) {
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(k_route<TB, EJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouteSmemMax);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * a.cl));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (size_t)smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cl > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_route<TB, EJ>, a);
}

// Tokens per CTA by experts per lane: a thread keeps at most 32 sums.
constexpr int route_tile_tokens(int ej) { return ej <= 2 ? 16 : (ej == 4 ? 8 : 4); }

cudaError_t launch_ej(const RouteArgs &a, int ej, int tb, int smem, int tiles, cudaStream_t st) {
    switch (ej) {
        case 1: return tb == 8 ? launch_one<8, 1>(a, smem, tiles, st) : launch_one<16, 1>(a, smem, tiles, st);
        case 2: return tb == 8 ? launch_one<8, 2>(a, smem, tiles, st) : launch_one<16, 2>(a, smem, tiles, st);
        case 4: return launch_one<route_tile_tokens(4), 4>(a, smem, tiles, st);
        default: return launch_one<route_tile_tokens(8), 8>(a, smem, tiles, st);
    }
}

}  // namespace

cudaError_t launch_router_logits_tc(const moe_shape &s, const void *x, const float *w_router, float *part, int *q,
                                    const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                    cudaStream_t stream);

cudaError_t launch_route(const moe_shape &s0, const void *x, const float *w_router, const float *bias, float *logits,
                         int32_t *topk_idx, float *topk_w, const WsLayout &L, void *ws, uint64_t timeout_ns,
                         int num_sms, cudaStream_t stream, const FusedDispatch *fused) {
    uint32_t *status = (uint32_t *)((char *)ws + L.status);
    moe_shape s = s0;
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, capped);
    // The fused path needs no clearing launch: the CTA that builds the
    // dispatch resets the completion count it used and writes the empty
    // capacity slots' src_token itself.
    if (fused && (int64_t)s.T * s.k > kFusedDispatchMaxPairs) return cudaErrorInvalidValue;
    const float *lparts = nullptr;
    int lq = 0;
    if (!(s.flags & MOE_FLAG_LOGITS_IN) && use_tc_router(s.T)) {
        // Partial logits on the tensor cores, then the top-k below adds them.
        float *part = (float *)((char *)ws + L.router_part);
        cudaError_t err = launch_router_logits_tc(s, x, w_router, part, &lq, L, ws, timeout_ns, num_sms, stream);
        if (err != cudaSuccess) return err;
        lparts = part;
        s.flags |= MOE_FLAG_LOGITS_IN;
    }
    RouteArgs a;
    a.x = (const __nv_bfloat16 *)x;
    a.w_router = w_router;
    a.bias = bias;
    a.logits = logits;
    a.lparts = lparts;
    a.lq = lq;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.status = status;
    a.T = s.T;
    a.H = s.H;
    a.E = s.E;
    a.k = s.k;
    a.logits_in = (s.flags & MOE_FLAG_LOGITS_IN) ? 1 : 0;
    a.fuse = fused ? 1 : 0;
    a.C = s.C;
    a.capped = capped ? 1 : 0;
    a.P = (int)P;
    a.out = fused ? *fused : FusedDispatch{nullptr, nullptr, nullptr, nullptr};
    a.ws = ws_ptrs(ws, L);
    if (a.logits_in && !fused) {
        const int blocks = (int)(((int64_t)s.T * 32 + 255) / 256);
        if (blocks > 0) {
            switch (topk_mpl(s.E)) {
                case 1: return launch_pdl(k_topk<1>, dim3(blocks), dim3(256), 0, stream, a);
                case 2: return launch_pdl(k_topk<2>, dim3(blocks), dim3(256), 0, stream, a);
                case 4: return launch_pdl(k_topk<4>, dim3(blocks), dim3(256), 0, stream, a);
                default: return launch_pdl(k_topk<8>, dim3(blocks), dim3(256), 0, stream, a);
            }
        }
        return cudaGetLastError();
    }
    int es = 1;
    while (es < s.E && es < 32) es <<= 1;
    a.es = es;
    int ej = (s.E + es - 1) / es;
    ej = ej <= 1 ? 1 : ej <= 2 ? 2 : ej <= 4 ? 4 : 8;
    int TB = route_tile_tokens(ej);
    // Small batches: halve the tile while 8-CTA clusters of full tiles would
    // leave more than a quarter of the SMs idle.  (32-token tiles, which read
    // each weight slice for more tokens, measured slower: smaller slices and
    // longer top-k per CTA.)
    if (TB == 16 && !a.logits_in && ((s.T + 15) / 16) * 8 < (3 * num_sms) / 4) TB = 8;
    const int tiles = (s.T + TB - 1) / TB;
    // Split the hidden dimension over a cluster until there are about 3/4 as
    // many blocks as SMs (measured best at 8 and 64 experts).
    int cl = 1;
    if (!a.logits_in)
        while (cl < 8 && tiles * cl < (3 * num_sms) / 4 && s.H % (64 * 2 * cl) == 0) cl *= 2;
    a.cl = cl;
    a.slice = s.H / cl;
    // Chunk: the largest power of two dividing the slice with the stage <= 40 KiB, >= 64.
    int hc = 1024;
    while (hc > 64 && (a.slice % hc != 0 || hc * (4 * s.E + 2 * TB) > 40 * 1024)) hc >>= 1;
    const int stage_bytes = (int)align_up((size_t)TB * hc * 2, 16) + (int)align_up((size_t)hc * s.E * 4, 16);
    const int nchunks = a.slice / hc;
    int stages = (160 * 1024) / stage_bytes;
    stages = stages < 2 ? 2 : (stages > 4 ? 4 : stages);
    if (stages > nchunks + 1) stages = nchunks + 1 < 2 ? 2 : nchunks + 1;
    a.hc = hc;
    a.stages = stages;
    a.stage_bytes = stage_bytes;
    const int lg_bytes = TB * (kMaxExperts + 1) * 4;
    int smem;
    if (a.logits_in) {
        a.part_off = 0;
        smem = lg_bytes;
    } else {
        // the pipeline stages and the chunk's fp32 x tile, later the per-warp
        // partial sums [8][TB][E] and then rank 0's logits tile share the
        // front of shared memory; fewer stages if it would not fit
        const int x2_bytes = TB * hc * 4;
        auto front_of = [&](int st) {
            int f = st * stage_bytes + x2_bytes;
            if (f < lg_bytes) f = lg_bytes;
            if (f < 8 * TB * s.E * 4) f = 8 * TB * s.E * 4;
            return (int)align_up((size_t)f, 16);
        };
        while (a.stages > 2 && front_of(a.stages) + TB * s.E * 4 > kRouteSmemMax) --a.stages;
        a.part_off = front_of(a.stages);
        smem = a.part_off + TB * s.E * 4;
    }
    if (fused) {
        const int need = (int)align_up(sizeof(DispatchSmem) + sizeof(int) * (size_t)s.T * s.k, 16);
        if (smem < need) smem = need;
    }
    return launch_ej(a, ej, TB, smem, tiles, stream);
}

}  // namespace moe
