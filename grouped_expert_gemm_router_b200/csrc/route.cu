// Step 1: router scoring ("TritonMoE" verdict page, arXiv 2605.23911, referee
// report summary).  logits = x * W_r (+ bias) in fp32, then per token the k
// largest logits (equal logits to the lower expert index, NaN lowest) and the
// softmax over the k selected logits.
//
// One CTA of 8 warps owns a block of TB = 8*TW tokens and all E experts.  The
// logits are a small fp32 GEMM: x and W_r are staged through shared memory in
// chunks of 32 hidden units, and each lane accumulates TW tokens x EJ experts
// in registers.  When E < 32 the spare lanes split the hidden dimension and
// are folded together with shuffles at the end.  The top-k then runs one warp
// per token: each lane holds ceil(E/32) candidates as 64-bit keys
// (orderable logit << 32 | ~expert) and k rounds of a warp-wide max pick the
// winners.
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr int kHC = 32;  // hidden units per staged chunk

struct RouteArgs {
    const __nv_bfloat16 *x;
    const float *w_router;
    const float *bias;
    float *logits;       // output (or input with logits_in); may be null when not logits_in
    int *topk_idx;
    float *topk_w;
    uint32_t *status;
    int T, H, E, k;
    int logits_in;
};

// Monotone map of a float onto uint32 (larger float -> larger key); -0 is
// folded onto +0 and NaN maps to 0, below -inf (whose key is 0x007FFFFF).
__device__ __forceinline__ uint32_t orderable(float f) {
    if (f != f) return 0u;
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    return v;
}

template <int TW>
__global__ void __launch_bounds__(256) k_route(RouteArgs a) {
    constexpr int TB = 8 * TW;
    // x chunk, transposed; rows padded by 4 floats so lanes reading different
    // rows hit different banks while float4 reads stay 16-byte aligned.
    __shared__ __align__(16) float xs[kHC][TB + 4];
    // W_r chunk during the GEMM phase (dense [32][Wcols]), then the logits
    // tile for the top-k.
    __shared__ __align__(16) float pool[(kHC * kMaxExperts > TB * (kMaxExperts + 1)) ? kHC * kMaxExperts
                                                                                       : TB * (kMaxExperts + 1)];
    __shared__ int s_nan;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * TB;
    const int E = a.E, H = a.H;
    if (tid == 0) s_nan = 0;

    float *wsm = pool;
    float(*lg)[kMaxExperts + 1] = reinterpret_cast<float(*)[kMaxExperts + 1]>(pool);

    if (!a.logits_in) {
        // Lane split: ES lanes across experts, HS = 32/ES lanes across hidden units.
        int ES = 1;
        while (ES < E && ES < 32) ES <<= 1;
        const int HS = 32 / ES;
        const int es = lane % ES, hs = lane / ES;
        const int EJ = (E + ES - 1) / ES;  // <= 8
        // W chunk columns incl. zero padding.  With ES < 32 this is ES (EJ = 1),
        // so lanes (hs, es) read word hs*ES + es of a 32-word window: no bank
        // conflicts; with ES = 32 all lanes read one row.
        const int Wcols = ES * EJ;
        float acc[TW][8];
#pragma unroll
        for (int i = 0; i < TW; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

        for (int h0 = 0; h0 < H; h0 += kHC) {
            __syncthreads();
            // x chunk: TB tokens x 32 hidden units, transposed into xs[h][token].
            for (int i = tid; i < TB * (kHC / 2); i += 256) {
                const int tok = i / (kHC / 2), hp = (i % (kHC / 2)) * 2;
                const int t = t0 + tok;
                float2 v = make_float2(0.f, 0.f);
                if (t < a.T) {
                    const __nv_bfloat162 b =
                        *reinterpret_cast<const __nv_bfloat162 *>(a.x + (size_t)t * H + h0 + hp);
                    v = __bfloat1622float2(b);
                }
                xs[hp][tok] = v.x;
                xs[hp + 1][tok] = v.y;
            }
            // W_r chunk: rows h0..h0+31, E columns, zero-padded to Wcols.
            for (int i = tid; i < kHC * Wcols; i += 256) {
                const int hh = i / Wcols, e = i % Wcols;
                wsm[hh * Wcols + e] = e < E ? a.w_router[(size_t)(h0 + hh) * E + e] : 0.0f;
            }
            __syncthreads();
            for (int hh = hs; hh < kHC; hh += HS) {
                float xv[TW];
                if constexpr (TW == 4) {
                    const float4 q = *reinterpret_cast<const float4 *>(&xs[hh][warp * 4]);
                    xv[0] = q.x;
                    xv[1] = q.y;
                    xv[2] = q.z;
                    xv[3] = q.w;
                } else {
#pragma unroll
                    for (int i = 0; i < TW; ++i) xv[i] = xs[hh][warp * TW + i];
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j < EJ) {
                        const float wv = wsm[hh * Wcols + es + ES * j];
#pragma unroll
                        for (int i = 0; i < TW; ++i) acc[i][j] = fmaf(xv[i], wv, acc[i][j]);
                    }
                }
            }
        }
        // Fold the hidden-unit split.
        for (int off = ES; off < 32; off <<= 1)
#pragma unroll
            for (int i = 0; i < TW; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] += __shfl_xor_sync(0xffffffffu, acc[i][j], off);
        __syncthreads();  // everyone is done with wsm; pool becomes lg
        if (hs == 0) {
#pragma unroll
            for (int i = 0; i < TW; ++i) {
                const int tok = warp * TW + i, t = t0 + tok;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = es + ES * j;
                    if (j < EJ && e < E) {
                        float l = acc[i][j];
                        if (a.bias) l = l + a.bias[e];
                        lg[tok][e] = l;
                        if (t < a.T && a.logits) a.logits[(size_t)t * E + e] = l;
                    }
                }
            }
        }
    } else {
        for (int i = tid; i < TB * E; i += 256) {
            const int tok = i / E, e = i % E, t = t0 + tok;
            lg[tok][e] = t < a.T ? a.logits[(size_t)t * E + e] : 0.0f;
        }
    }
    __syncthreads();

    // Top-k, one warp per token.
    for (int i = 0; i < TW; ++i) {
        const int tok = warp * TW + i, t = t0 + tok;
        if (t >= a.T) break;
        unsigned long long key[8];
        bool nan = false;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int e = lane + 32 * m;
            key[m] = 0ull;
            if (e < E) {
                const float l = lg[tok][e];
                nan |= (l != l);
                key[m] = ((unsigned long long)orderable(l) << 32) | (0xFFFFFFFFu - (uint32_t)e);
            }
        }
        if (__any_sync(0xffffffffu, nan) && lane == 0) s_nan = 1;
        for (int j = 0; j < a.k; ++j) {
            unsigned long long best = 0ull;
#pragma unroll
            for (int m = 0; m < 8; ++m) best = key[m] > best ? key[m] : best;
            best = warp_max_u64(best);
            const int e = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
            if ((e & 31) == lane) {
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    if (m == (e >> 5)) key[m] = 0ull;
            }
            if (lane == 0) {
                a.topk_idx[(size_t)t * a.k + j] = e;
                a.topk_w[(size_t)t * a.k + j] = lg[tok][e];  // selected logit, replaced below
            }
        }
        __syncwarp();
        // Softmax over the k selected logits, reference = the largest (slot 0).
        const float lmax = a.topk_w[(size_t)t * a.k];
        float s = 0.0f;
        for (int j = lane; j < a.k; j += 32) s += expf(a.topk_w[(size_t)t * a.k + j] - lmax);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        // k <= E <= 256: at most 8 slots per lane.
        float ex[8];
        int n = 0;
        for (int j = lane; j < a.k; j += 32) ex[n++] = expf(a.topk_w[(size_t)t * a.k + j] - lmax);
        __syncwarp();
        n = 0;
        for (int j = lane; j < a.k; j += 32) a.topk_w[(size_t)t * a.k + j] = ex[n++] / s;
        __syncwarp();
    }
    __syncthreads();
    if (tid == 0 && s_nan) atomicOr(a.status, MOE_DEV_NAN_LOGIT);
}

}  // namespace

cudaError_t launch_route(const moe_shape &s, const void *x, const float *w_router, const float *bias, float *logits,
                         int32_t *topk_idx, float *topk_w, uint32_t *status, int num_sms, cudaStream_t stream) {
    RouteArgs a;
    a.x = (const __nv_bfloat16 *)x;
    a.w_router = w_router;
    a.bias = bias;
    a.logits = logits;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.status = status;
    a.T = s.T;
    a.H = s.H;
    a.E = s.E;
    a.k = s.k;
    a.logits_in = (s.flags & MOE_FLAG_LOGITS_IN) ? 1 : 0;
    // Four tokens per warp when that still gives every SM a block.
    if ((s.T + 31) / 32 >= num_sms) {
        k_route<4><<<(s.T + 31) / 32, 256, 0, stream>>>(a);
    } else {
        k_route<1><<<(s.T + 7) / 8, 256, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace moe
