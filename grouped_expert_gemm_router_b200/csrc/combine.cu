// Step 5: weighted unpermutation ("TritonMoE" verdict page, arXiv 2605.23911,
// referee report summary):
//   out[t] = bf16( sum_{j<k} topk_w[t,j] * y[dest_row[t*k+j]] )
// summed in fp32 in slot order with each product and each sum rounded on its
// own (no fused multiply-add), so that given the same y the result is
// bit-identical to a plain sequential fp32 loop.
//
// HBM-bound gather: each thread owns 8 consecutive features (one 16-byte
// vector) of one token, reads the k expert rows with 16-byte loads (for
// k <= 8 all of them issued before the first is used) and writes one 16-byte
// vector.  Grid: tokens x ceil(H/8 / 256) blocks of 256 threads.
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void unpack8(const uint4 &q, float (&v)[8]) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Overflow rows read from where an expert-parallel exchange left them: row
// E C + q of y is row d S + (q - starts[d]) of `ovf`, d the last destination
// with starts[d] <= q (the rows the unpack would copy into y); any other row
// is read from y.
struct OvfRows {
    const uint4 *ovf;
    const int32_t *starts;  // [G + 1]
    int cap_rows, S, G;
};

// KMAX > 0: k <= KMAX, all k row loads issued before any is used; KMAX = 0:
// any k, one row at a time.  REDIR: overflow rows through OvfRows.
template <int KMAX, bool REDIR = false>
__global__ void __launch_bounds__(256) k_combine(const uint4 *__restrict__ y, const int *__restrict__ dest_row,
                                                 const float *__restrict__ w, uint4 *__restrict__ out, int k, int H8,
                                                 int P, OvfRows orw) {
    __shared__ int st[REDIR ? kMaxExperts + 1 : 1];
    pdl_trigger();
    pdl_wait();
    if (REDIR) {
        for (int d = threadIdx.x; d <= orw.G; d += blockDim.x) st[d] = orw.starts[d];
        __syncthreads();
    }
    const int total = REDIR ? min(st[REDIR ? orw.G : 0], P - orw.cap_rows) : 0;
    auto row_ptr = [&](int r) -> const uint4 * {
        if (REDIR && r >= orw.cap_rows && r - orw.cap_rows < total) {
            const int q = r - orw.cap_rows;
            int lo = 0, hi = orw.G - 1;  // last d with st[d] <= q
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (st[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            const int j = q - st[lo];
            if (j < orw.S) return orw.ovf + (size_t)(lo * orw.S + j) * H8;
        }
        return y + (size_t)r * H8;
    };
    const int t = blockIdx.x;
    const int v = blockIdx.y * blockDim.x + threadIdx.x;
    if (v >= H8) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    if (KMAX > 0) {
        int r[KMAX > 0 ? KMAX : 1];
        float wj[KMAX > 0 ? KMAX : 1];
        uint4 q[KMAX > 0 ? KMAX : 1];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            r[j] = j < k ? __ldg(dest_row + (size_t)t * k + j) : -1;
            wj[j] = j < k ? __ldg(w + (size_t)t * k + j) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)  // an index outside [0, P) only after an earlier device error
            q[j] = (unsigned)r[j] < (unsigned)P ? __ldg(row_ptr(r[j]) + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if ((unsigned)r[j] >= (unsigned)P) continue;
            float yv[8];
            unpack8(q[j], yv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(wj[j], yv[i]));
        }
    } else {
        for (int j = 0; j < k; ++j) {
            const int r = __ldg(dest_row + (size_t)t * k + j);
            if ((unsigned)r >= (unsigned)P) continue;  // only after an earlier device error
            const float wj = __ldg(w + (size_t)t * k + j);
            float yv[8];
            unpack8(__ldg(row_ptr(r) + v), yv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(wj, yv[i]));
        }
    }
    uint4 o;
    __nv_bfloat162 *ob = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) ob[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    out[(size_t)t * H8 + v] = o;
}

}  // namespace

cudaError_t launch_combine(const moe_shape &s, const void *y, const int32_t *dest_row, const float *topk_w, void *out,
                           cudaStream_t stream) {
    const int H8 = s.H / 8;
    const dim3 grid((unsigned)s.T, (unsigned)((H8 + 255) / 256));
    const int P = (int)permuted_rows(s.T, s.E, s.k, s.C, (s.flags & MOE_FLAG_CAPACITY) != 0);
    if (s.k <= 2)
        return launch_pdl(k_combine<2>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w, (uint4 *)out,
                          s.k, H8, P, OvfRows{});
    else if (s.k <= 8)
        return launch_pdl(k_combine<8>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w, (uint4 *)out,
                          s.k, H8, P, OvfRows{});
    else
        return launch_pdl(k_combine<0>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w, (uint4 *)out,
                          s.k, H8, P, OvfRows{});
    return cudaGetLastError();
}

// The combine reading each overflow row from the received return slots
// (ovf [G][S] rows, destination starts [G + 1] from the expert-parallel
// workspace) instead of from y: the unpack and the combine in one launch,
// bit-identical to the two.
cudaError_t launch_combine_ovf(const moe_shape &s, int G, int S, const void *y, const void *ovf,
                               const int32_t *starts, const int32_t *dest_row, const float *topk_w, void *out,
                               cudaStream_t stream) {
    const int H8 = s.H / 8;
    const dim3 grid((unsigned)s.T, (unsigned)((H8 + 255) / 256));
    const int P = (int)permuted_rows(s.T, s.E, s.k, s.C, (s.flags & MOE_FLAG_CAPACITY) != 0);
    const OvfRows o = {(const uint4 *)ovf, starts, s.E * s.C, S, G};
    if (s.k <= 2)
        return launch_pdl(k_combine<2, true>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w,
                          (uint4 *)out, s.k, H8, P, o);
    else if (s.k <= 8)
        return launch_pdl(k_combine<8, true>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w,
                          (uint4 *)out, s.k, H8, P, o);
    return launch_pdl(k_combine<0, true>, grid, dim3(256), 0, stream, (const uint4 *)y, dest_row, topk_w,
                      (uint4 *)out, s.k, H8, P, o);
}

}  // namespace moe
