// fp8 (e4m3) operands of the expert GEMMs ("TEMPO" verdict page, arXiv
// 2608.13057, referee report summary: the per-expert cost law is measured on
// an fp8 grouped GEMM, whose flat regime streams the expert's weights from
// HBM, so 8-bit weights halve the bytes that bound it).
//
// Format: OCP E4M3 codes and one power-of-two scale per vector,
// s = 2^(c - 8) with c the smallest integer such that max|v| <= 2^c (s = 1 for
// an all-zero vector); code = nearest e4m3 value of v / s, ties to even.  So
// |v| / s <= 256 (below e4m3's 448), v / s is exact, and code * s is exactly a
// bf16 value.  Expert weights get one scale per expert and output column and
// are stored with the reduction dimension contiguous (the K-major operand of
// the MMA); activations get one scale per row.
//
// k_quant_weights  w [E][K][N] bf16 -> codes, scales [E][N] (one-time
//                  preparation of a layer's weights).  The codes are K-major
//                  inside tiles of 128 output columns x 128 K, each tile 16 KB
//                  contiguous: code (e, n, k) at byte
//                  ((e (N/128) + n/128) (K/128) + k/128) 16384 + (n%128) 128 + k%128,
//                  so each weight load of the GEMM streams one contiguous
//                  16 KB tile from HBM.
// k_quant_rows     rows of a bf16 matrix -> codes + one scale per row: a row
//                  is held in registers by 32-256 threads (all its loads in
//                  flight at once), its largest magnitude comes from warp and
//                  block reductions, the codes go out with streaming 8-byte
//                  stores.  Optionally reads row r from src[idx[r]] (the row
//                  copy of the dispatch, x_perm) or skips rows whose idx is
//                  negative (h: unfilled slots).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "fp8_rows.cuh"

namespace moe {

namespace {

// Block of 256 threads: expert e = blockIdx.y, columns [32 blockIdx.x, +32).
__global__ void __launch_bounds__(256) k_quant_weights(const __nv_bfloat16 *__restrict__ w, uint8_t *__restrict__ q,
                                                       float *__restrict__ scale, int K, int N) {
    __shared__ float s_red[8][32];
    __shared__ Fp8Scale s_scale[32];
    __shared__ __nv_bfloat16 tile[128][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int e = blockIdx.y, n0 = blockIdx.x * 32;
    const __nv_bfloat16 *we = w + (size_t)e * K * N;
    float m = 0.0f;
    for (int k = ty; k < K; k += 8) m = fmaxf(m, fabsf(__bfloat162float(we[(size_t)k * N + n0 + tx])));
    s_red[ty][tx] = m;
    __syncthreads();
    if (ty == 0) {
        for (int i = 1; i < 8; ++i) m = fmaxf(m, s_red[i][tx]);
        const Fp8Scale sc = fp8_scale(m);
        s_scale[tx] = sc;
        scale[(size_t)e * N + n0 + tx] = sc.s;
    }
    __syncthreads();
    // codes (e, n0 + i, k0 + 16 c ...): thread (i = t / 8, c = t % 8) writes 16
    // bytes into row (n0 + i) % 128 of tile (e, (n0 + i) / 128, k0 / 128)
    const int i = threadIdx.x >> 3, c = threadIdx.x & 7;
    const Fp8Scale s = s_scale[i];
    const int n = n0 + i, KB = K / 128;
    uint8_t *qe = q + ((size_t)e * (N / 128) + n / 128) * (size_t)KB * 16384 + (size_t)(n % 128) * 128;
    for (int k0 = 0; k0 < K; k0 += 128) {
        for (int r = ty; r < 128; r += 8) tile[r][tx] = we[(size_t)(k0 + r) * N + n0 + tx];
        __syncthreads();
        uint32_t word[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int kk = 16 * c + 4 * v;
            const uint32_t lo = e4m3x2<false>(__bfloat162float(tile[kk][i]), __bfloat162float(tile[kk + 1][i]), s);
            const uint32_t hi = e4m3x2<false>(__bfloat162float(tile[kk + 2][i]), __bfloat162float(tile[kk + 3][i]), s);
            word[v] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4 *>(qe + (size_t)(k0 / 128) * 16384 + 16 * c) = make_uint4(word[0], word[1], word[2], word[3]);
        __syncthreads();
    }
}

// Rows of TPR threads (TPR = 32 << g, 256 / TPR rows per block): row r < rows
// (rows = fixed_rows, or cap_rows + *total_spill when fixed_rows < 0).
// gather: row r is src[idx[r]] (idx outside [0, src_rows): a zero row with
// scale 1); otherwise row r is src[r], skipped when idx != nullptr and
// idx[r] < 0.  Each thread loads its VPT 16-byte vectors of the row into
// registers (all loads in flight at once), the row's largest magnitude comes
// from a warp reduction and, for TPR > 32, a reduction over the row's warps in
// shared memory; the codes are written from the registers with streaming
// stores (the codes are read once, by the GEMM).
template <int TPR, int VPT, int RPG>
__global__ void __launch_bounds__(256) k_quant_rows(const uint4 *__restrict__ src, const int *__restrict__ idx,
                                                    int gather, uint2 *__restrict__ q, float *__restrict__ scale,
                                                    int K8, int src_rows, int P, int fixed_rows, int cap_rows,
                                                    const int *total_spill) {
    // RPG rows per thread group and iteration (all their loads in flight
    // before the first reduction; rows of a few vectors per thread are
    // otherwise bound by one load latency per row)
    static_assert(RPG == 1 || TPR == 32, "several rows per group only for one-warp rows");
    constexpr int kRowsPerBlock = 256 / TPR, kWarpsPerRow = TPR / 32;
    __shared__ float s_max[8];
    pdl_trigger();
    pdl_wait();
    int rows = fixed_rows >= 0 ? fixed_rows : cap_rows + *total_spill;
    if (rows > P) rows = P;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = threadIdx.x / TPR, tr = threadIdx.x % TPR;
    // every thread of the block runs the same number of iterations (the
    // shared-memory reduction below needs the whole block)
    for (int base = blockIdx.x * kRowsPerBlock * RPG; base < rows; base += gridDim.x * kRowsPerBlock * RPG) {
        int row[RPG];
        bool active[RPG], valid[RPG];
        uint4 v[RPG][VPT];
        float m[RPG];
#pragma unroll
        for (int j = 0; j < RPG; ++j) {
            row[j] = base + j * kRowsPerBlock + g;
            active[j] = row[j] < rows;
            int sr = row[j];
            if (active[j] && idx) {
                const int t = idx[row[j]];
                if (!gather && t < 0) active[j] = false;
                if (gather) sr = t;
            }
            valid[j] = active[j] && (unsigned)sr < (unsigned)src_rows;
            if (valid[j]) {
                const uint4 *s_row = src + (size_t)sr * K8;
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int c = tr + i * TPR;
                    v[j][i] = c < K8 ? __ldg(s_row + c) : make_uint4(0, 0, 0, 0);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < RPG; ++j) {
            m[j] = 0.0f;
            if (valid[j]) {
                __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
#pragma unroll
                for (int i = 0; i < VPT; ++i) m2 = amax8(v[j][i], m2);
                m[j] = amax_of(m2);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
        }
        if (kWarpsPerRow > 1) {
            if (lane == 0) s_max[warp] = m[0];
            __syncthreads();
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) m[0] = fmaxf(m[0], s_max[g * kWarpsPerRow + w]);
            __syncthreads();
        }
#pragma unroll
        for (int j = 0; j < RPG; ++j) {
            if (!active[j]) continue;
            uint2 *dst = q + (size_t)row[j] * K8;
            if (!valid[j]) {
                for (int c = tr; c < K8; c += TPR) dst[c] = make_uint2(0, 0);
                if (tr == 0) scale[row[j]] = 1.0f;
                continue;
            }
            const Fp8Scale sc = fp8_scale(m[j]);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int c = tr + i * TPR;
                if (c < K8) __stcs(dst + c, quant8(v[j][i], sc));
            }
            if (tr == 0) scale[row[j]] = sc.s;
        }
    }
}

// Two passes over the row (rows longer than 256 threads x 16 vectors).
__global__ void __launch_bounds__(256) k_quant_rows_long(const uint4 *__restrict__ src, const int *__restrict__ idx,
                                                         int gather, uint2 *__restrict__ q, float *__restrict__ scale,
                                                         int K8, int src_rows, int P, int fixed_rows, int cap_rows,
                                                         const int *total_spill) {
    __shared__ float s_max[8];
    pdl_trigger();
    pdl_wait();
    int rows = fixed_rows >= 0 ? fixed_rows : cap_rows + *total_spill;
    if (rows > P) rows = P;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        int sr = row;
        if (idx) {
            const int t = idx[row];
            if (!gather && t < 0) continue;  // block-uniform
            if (gather) sr = t;
        }
        uint2 *dst = q + (size_t)row * K8;
        if ((unsigned)sr >= (unsigned)src_rows) {
            for (int c = threadIdx.x; c < K8; c += 256) dst[c] = make_uint2(0, 0);
            if (threadIdx.x == 0) scale[row] = 1.0f;
            continue;
        }
        const uint4 *s_row = src + (size_t)sr * K8;
        __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
        for (int c = threadIdx.x; c < K8; c += 256) m2 = amax8(__ldg(s_row + c), m2);
        float m = amax_of(m2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_max[warp] = m;
        __syncthreads();
        for (int w = 0; w < 8; ++w) m = fmaxf(m, s_max[w]);
        __syncthreads();
        const Fp8Scale sc = fp8_scale(m);
        for (int c = threadIdx.x; c < K8; c += 256) __stcs(dst + c, quant8(__ldg(s_row + c), sc));
        if (threadIdx.x == 0) scale[row] = sc.s;
    }
}

// Row quantization launch: threads per row chosen so that a row's vectors fit
// 8 (up to 16) registers per thread.
cudaError_t launch_rows(const uint4 *src, const int *idx, int gather, uint2 *q, float *scale, int K8, int src_rows,
                        int P, int fixed_rows, int cap_rows, const int *total_spill, int row_hint, int num_sms,
                        cudaStream_t stream) {
    int tpr = 32;
    while (tpr < 256 && K8 > tpr * 8) tpr <<= 1;
    const int rpb = 256 / tpr;
    int blocks = (row_hint + rpb - 1) / rpb;
    const int cap = num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
#define MOE_QROWS(T, V, R)                                                                                  \
    return launch_pdl(k_quant_rows<T, V, R>, dim3(blocks), dim3(256), 0, stream, src, idx, gather, q, scale, K8,    \
                      src_rows, P, fixed_rows, cap_rows, total_spill)
    if (K8 <= 32 * 4) MOE_QROWS(32, 4, 2);  // short rows: two rows per warp in flight
    if (K8 <= 32 * 8) MOE_QROWS(32, 8, 1);
    if (K8 <= 64 * 8) MOE_QROWS(64, 8, 1);
    if (K8 <= 128 * 8) MOE_QROWS(128, 8, 1);
    if (K8 <= 256 * 8) MOE_QROWS(256, 8, 1);
    if (K8 <= 256 * 16) MOE_QROWS(256, 16, 1);
#undef MOE_QROWS
    return launch_pdl(k_quant_rows_long, dim3(blocks), dim3(256), 0, stream, src, idx, gather, q, scale, K8, src_rows,
                      P, fixed_rows, cap_rows, total_spill);
}

}  // namespace

// Expert weights w [E][K][N] bf16 -> codes [E][N][K] and scales [E][N].
cudaError_t launch_quant_weights(int E, int K, int N, const void *w, void *q, float *scale, cudaStream_t stream) {
    const dim3 grid((unsigned)(N / 32), (unsigned)E);
    k_quant_weights<<<grid, 256, 0, stream>>>((const __nv_bfloat16 *)w, (uint8_t *)q, scale, K, N);
    return cudaGetLastError();
}

// Codes + row scales of the rows of the permuted buffers (P rows of length
// K, the used rows only).  gather: row r = src[idx[r]] with src holding
// src_rows rows (the row copy of x); otherwise row r = src[r], rows with
// idx[r] < 0 skipped (h).
cudaError_t launch_quant_rows(const moe_shape &s, int K, const void *src, int src_rows, const int32_t *idx,
                              bool gather, void *q, float *scale, const WsLayout &L, void *ws, int num_sms,
                              cudaStream_t stream) {
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int R = s.T * s.k;
    const int P = (int)permuted_rows(s.T, s.E, s.k, s.C, capped);
    WsPtrs p = ws_ptrs(ws, L);
    return launch_rows((const uint4 *)src, idx, gather ? 1 : 0, (uint2 *)q, scale, K / 8, src_rows, P,
                       capped ? -1 : R, s.E * s.C, p.total_spill, P, num_sms, stream);
}

// Codes + scales of rows [0, *rows_dev) of src [rows_cap, K] (rows_dev: a
// device count, at most rows_cap; the rest are left unwritten).
cudaError_t launch_quant_rows_counted(const void *src, int K, int rows_cap, const int *rows_dev, void *q,
                                      float *scale, int num_sms, cudaStream_t stream) {
    return launch_rows((const uint4 *)src, nullptr, 0, (uint2 *)q, scale, K / 8, rows_cap, rows_cap, -1, 0, rows_dev,
                       rows_cap, num_sms, stream);
}

// Codes + scales of every token row of x [T, K] (the form the row-gathering
// SwiGLU GEMM reads).
cudaError_t launch_quant_tokens(const moe_shape &s, const void *x, void *q, float *scale, int num_sms,
                                cudaStream_t stream) {
    return launch_rows((const uint4 *)x, nullptr, 0, (uint2 *)q, scale, s.H / 8, s.T, s.T, s.T, 0, nullptr, s.T,
                       num_sms, stream);
}

}  // namespace moe
