// Step 4: grouped expert GEMMs on the sm_100a tensor cores.
//   mode 0, fused gate+up SwiGLU ("TritonMoE" verdict page, arXiv 2605.23911,
//           pith extraction key machinery: both projections from one load of
//           each input tile, SiLU in registers, the two intermediates never
//           written to global memory):
//           h[r, f] = bf16( silu(x_perm[r] . Wg[e][:, f]) * (x_perm[r] . Wu[e][:, f]) )
//   mode 1, down projection (same page, desk editor letter):
//           y[r, c] = bf16( h[r] . Wd[e][:, c] )
//   mode 2, router logits of step 1 on the tensor cores (for large batches):
//           part[q, t, e] = fp32( x[t, Kq] . (P0 + P1 + P2)[Kq, e] ) over the
//           q-th range Kq of the hidden dimension, where P0 + P1 + P2 is the
//           exact three-way bf16 split of the fp32 router weights (to 2^-27
//           relative); every product of two bf16 values is exact in fp32.  The
//           top-k kernel adds the ranges in order and the bias.  The tensor
//           cores' fp32 accumulator loses low bits on every accumulate, so
//           inside a unit the K blocks rotate over route_groups accumulators
//           (block j of the range to accumulator j mod route_groups) and the
//           epilogue adds them in fp32 in a fixed order.
//
// Design (B200 first, not the page's Triton kernel):
// - Swap-AB.  The MMA computes D[feature, row] = W^T[feature, k] * X^T[k, row]:
//   the expert weights are the M = 128 operand (MN-major, read straight from
//   the [E, K, N] weight tensors) and up to 256 permuted rows of one expert
//   are the N operand (K-major).  An expert with <= 256 routed rows therefore
//   streams each weight tile from HBM exactly once, which is what the
//   weight-streaming regime of small per-expert batches needs, and N is
//   rounded only to 16 rows, not to a 128-row M tile.
// - Two accumulators per work unit share every B tile: gate and up for the
//   same 128 features (mode 0), or two adjacent 128-feature blocks (mode 1).
//   Units of <= 128 rows take one 256-column half of tensor memory each, in
//   turn, so the epilogue of one overlaps the MMAs of the next; larger units
//   take both halves.  The epilogue finishes the values into registers and
//   hands the accumulator back before its global stores whenever the
//   results fit in 64 registers; it stores 16-byte vectors of eight features
//   of one row, transposed through a small per-warp staging block
//   (stmatrix), since its time is set by its store instructions.
// - Persistent, warp-specialised: warp 0 streams weight tiles and warp 2
//   token tiles with TMA into two rings of shared-memory stages (mbarrier
//   expect-tx), warp 1 issues tcgen05.mma from one thread and commits each
//   pair of stages back to the producers, warps 3-18 drain tensor memory with
//   tcgen05.ld (four warps per lane quarter, taking 16-column chunks in
//   turn) and write bf16 results.  The more epilogue warps, the sooner a
//   finished accumulator is handed back to the MMA warp.
// - Stage sizes follow the routing.  A weight stage holds the two 128-feature
//   A tiles of 64 K rows; a token stage holds tile_rows rows of B (loaded in
//   TMA boxes of up to 256 rows, so that one producer thread keeps up), where
//   tile_rows (chosen on the device by the schedule builder from the actual
//   counts) is the largest padded row count of any expert, capped at 256.
//   The token ring has four stages while that leaves room for four weight
//   stages, else three, and the weight ring takes the rest of shared
//   memory: the fewer rows per tile, the more weight bytes are in flight per
//   SM, which is what the weight-streaming regime of small per-expert
//   batches is bound by (4 + 4 stages at 144 rows, 6 + 4 at 32 rows, 3 + 3
//   at 256).
// - The schedule is the device-built tile map: work unit u -> (expert group
//   in descending-count order, feature block, row tile), feature-block-major
//   inside an expert so that the row tiles of one expert that share a weight
//   tile run next to each other.  Nothing depends on the host knowing the
//   routing, so the kernel is launched with one CTA per SM and can be
//   captured in a CUDA graph; the CTAs count the units on the device and
//   only as many take work as balance the rounds.
// - Every wait is bounded: on expiry the kernel records MOE_DEV_GEMM_TIMEOUT,
//   tells the other roles to stop, lets in-flight copies and MMAs land, frees
//   its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr int kBK = 64;                        // K per stage: one 128-byte swizzle row of bf16
constexpr int kMaxAStages = 16;
constexpr int kMaxBStages = 4;                 // token stages: 4 while >= 4 weight stages still fit, else 3
constexpr uint32_t kABox = 64 * 64 * 2;        // TMA box: 64 K rows x 64 features (8 KiB)
constexpr uint32_t kATile = 2 * kABox;         // one accumulator's A: 128 features x 64 K
constexpr uint32_t kBRowBytes = kBK * 2;       // one B row of a stage: 128 bytes
constexpr uint32_t kBBox = 16 * kBRowBytes;    // TMA box: 16 rows x 64 K (2 KiB)
constexpr int kRowBoxes = 5;                   // token-tile boxes of 16, 32, 64, 128 and 256 rows
constexpr uint32_t kCtrlBytes = 3072;
constexpr uint32_t kSmemBytes = 226 * 1024;
constexpr uint32_t kEpiStageBytes = 512;      // per epilogue warp: one 8-row x 32-feature bf16 block
constexpr uint32_t kRingBytes = (kSmemBytes - 1024 - kCtrlBytes - 16 * kEpiStageBytes) & ~1023u;
// The largest token stages still leave room for a weight stage of both
// accumulators, so the ring geometry below never runs out of space (its
// unsigned arithmetic relies on it).
static_assert((uint32_t)kMaxBStages * kTileRows * kBRowBytes + 2u * kATile <= kRingBytes, "ring too small");
static_assert(3 * 2 * kATile + 3 * kTileRows * kBRowBytes <= kRingBytes,
              "three weight stages and three token stages of 256 rows must fit");
constexpr int kEpiWarp0 = 3;                   // warps 0-2 load and issue, 3-10 drain tensor memory
constexpr int kEpiWarps = 16;                  // four per tensor-memory lane quarter
constexpr int kEpiSub = kEpiWarps / 4;         // warps sharing one lane quarter
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
    const int4 *tile_map;
    const int *grp_tile_start;
    const int *num_tiles;
    const int *tile_rows;  // row cap of the tiles, chosen by the schedule builder
    uint32_t *status;
    __nv_bfloat16 *out;
    int n_out;   // row length of `out`: F (mode 0) or H (mode 1)
    // mode 1 without the fused combine: when set, row r of the result goes to
    // row_addr[r] (a byte address, anywhere the GPU can store: another GPU's
    // memory included) instead of out + r * n_out; entries of 0 are skipped
    const unsigned long long *row_addr;
    int K;       // reduction length: H (mode 0) or F (mode 1)
    int num_fb;  // feature blocks per row tile
    int E;
    int P;          // rows of the permuted buffers
    int max_tiles;  // capacity of the tile map
    unsigned long long timeout_ns;
    // mode 2 (router logits)
    float *logits;      // partial planes [route_q][T][E]
    int T;              // tokens
    // mode 0 with the row gather: the B rows come from x[src_token[row]]
    const int *src_token;
    int route_rows;     // tokens per unit (multiple of 16, <= 256)
    int route_q;        // K ranges (units per token block)
    int route_kb;       // K blocks per range
    int route_groups;   // accumulators per unit: route_groups * nacc * route_rows <= 512 columns
    uint32_t row_boxes; // bit i: RowMaps::m[i] (boxes of 16 << i rows) is valid; bit 0 always
    int stall_first_stage;  // test hook: CTA 0's token producer never loads its first stage
    // FP8 (e4m3 operands): value = code * scale, one power-of-two scale per
    // expert and output feature (w_scale0/1: [E][n_out], for the weights of
    // accumulators 0 and 1) and one per row of the token matrix (row_scale,
    // indexed by permuted row, or by token when the rows are gathered)
    const float *w_scale0, *w_scale1, *row_scale;
    // COMBINE (mode 1): step 5 fused into the down projection's epilogue.
    // comb_cnt [T][n_out / 128] counts, per token and 128-feature block, the
    // (row, lane-quarter warp) pieces of y stored so far; the warp whose piece
    // completes a token's block (4 k pieces) combines that block from y into
    // comb_out and sets the count back to zero.
    const int *dest_row;
    const float *topk_w;
    __nv_bfloat16 *comb_out;
    int *comb_cnt;
    int k;
};

// Tensor maps of the token matrix (B operand) with boxes of 16 << i rows x 64
// K; the row gather uses m[0] alone, with one-row boxes.
struct RowMaps {
    CUtensorMap m[kRowBoxes];
};

// Rows [row0, row0 + n) (n a multiple of 16, <= 256) of the token matrix at
// K offset kx into consecutive 128-byte shared-memory rows from dst, largest
// boxes first: a 256-row tile is one copy instead of sixteen, which keeps the
// single producer thread's TMA issue off the critical path.
__device__ __forceinline__ void tma_load_rows(uint8_t *dst, const RowMaps &rm, uint32_t boxes, uint64_t *bar, int kx,
                                              int row0, int n) {
#pragma unroll
    for (int i = kRowBoxes - 1; i >= 0; --i) {
        const int h = 16 << i;
        if (!((boxes >> i) & 1u)) continue;
        while (n >= h) {
            tma_load_2d(dst, &rm.m[i], bar, kx, row0);
            dst += h * kBRowBytes;
            row0 += h;
            n -= h;
        }
    }
}

struct Unit {
    int e, fb, fx, nacc, N, n0p, p0s, p0l, p1s, p1l;  // fx: first output feature of accumulator 0
    bool valid;  // false only for a corrupt schedule: every role then skips the unit
};

template <int MODE>
// num_fb / fbw: feature blocks per row tile and their width (mode 0: 128
// features, gate and up; mode 1: 256 features in two accumulators, or 128 in
// one when that still fits one wave).
__device__ __forceinline__ void decode_unit(int u, const int *gts, const GemmArgs &a, int trows, int num_fb, int fbw,
                                            Unit &U) {
    if (MODE == 2) {  // unit u = tokens [tb * route_rows, ...) x K range fb, all experts
        const int tb = u / a.route_q;
        U.e = 0;
        U.fb = u - tb * a.route_q;
        U.fx = 0;
        U.p0s = tb * a.route_rows;
        U.p0l = min(a.route_rows, a.T - U.p0s);
        U.p1s = 0;
        U.p1l = 0;
        U.n0p = (U.p0l + 15) & ~15;
        U.N = U.n0p;
        U.nacc = a.E > 128 ? 2 : 1;
        U.valid = U.p0l > 0;
        return;
    }
    int lo = 0, hi = a.E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gts[mid] * num_fb <= u)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int g0 = gts[lo], nt = gts[lo + 1] - g0;
    U.valid = false;
    U.N = 0;
    if (nt <= 0 || g0 < 0) return;
    const int local = u - g0 * num_fb;
    U.fb = local / nt;
    const int tile = g0 + local % nt;
    if (tile >= a.max_tiles) return;
    const int4 d = a.tile_map[tile];
    U.e = d.x;
    U.p0s = d.y;
    U.p0l = d.z & 0xFFFF;
    U.p1l = (d.z >> 16) & 0xFFFF;
    U.p1s = d.w;
    U.n0p = (U.p0l + 15) & ~15;
    U.N = U.n0p + ((U.p1l + 15) & ~15);
    U.fx = U.fb * fbw;
    U.nacc = (MODE == 0) ? 2 : ((fbw == 256 && U.fx + 128 < a.n_out) ? 2 : 1);
    U.valid = (unsigned)U.e < (unsigned)a.E && U.N > 0 && U.N <= trows && U.p0s >= 0 && U.p1s >= 0 &&
              U.p0s + U.p0l <= a.P && U.p1s + U.p1l <= a.P && U.fb < num_fb;
}

__device__ __forceinline__ int unit_row(const Unit &U, int c) {
    if (c < U.n0p) return c < U.p0l ? U.p0s + c : -1;
    const int c1 = c - U.n0p;
    return c1 < U.p1l ? U.p1s + c1 : -1;
}

// Stores a 32-feature x 16-row block of bf16 results held by one warp in the
// fragment layout of tmem_ld_frag16 (w[m] = the pair r[2m], r[2m + 1]: feature
// 16 (m >> 2) + 8 (m & 1) + (t >> 2), rows 8 ((m >> 1) & 1) + 2 (t & 3) + {0, 1}
// of unit rows c0 ..): per 8-row group one transposing stmatrix into the
// warp's 512-byte staging block (rows of four 16-byte feature groups, the
// group index XORed with bits 1-2 of the row so that neither side conflicts
// on banks), then each lane reads back one 16-byte vector (8 features of one
// row) and stores it.  Two 16-byte store instructions per warp for the
// block instead of sixteen 2-byte ones.
__device__ __forceinline__ void store_block_frag(const uint32_t (&w)[8], uint8_t *stg, __nv_bfloat16 *out, int n_out,
                                                 const unsigned long long *row_addr, int fbase, const Unit &U,
                                                 int c0) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3, mj = lane & 7;  // stmatrix: row mj of matrix (feature group) mi
    const int r = lane >> 2, c = lane & 3;    // read-back: row r, feature group c
    const uint32_t st_addr = smem_u32(stg) + mj * 64 + 16 * (mi ^ ((mj >> 1) & 3));
    const uint32_t ld_addr = smem_u32(stg) + r * 64 + 16 * (c ^ ((r >> 1) & 3));
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        stmatrix_x4_trans(st_addr, w[2 * k], w[2 * k + 1], w[4 + 2 * k], w[5 + 2 * k]);
        __syncwarp();
        const uint4 v = lds128(ld_addr);
        __syncwarp();  // the block is rewritten by the next group
        const int row = unit_row(U, c0 + 8 * k + r);
        if (row < 0) continue;
        if (row_addr) {  // the row's own destination (another GPU's memory, say); 0 = none
            const unsigned long long d = row_addr[row];
            if (d) *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(d) + fbase + 8 * c) = v;
        } else {
            *reinterpret_cast<uint4 *>(out + (size_t)row * n_out + fbase + 8 * c) = v;
        }
    }
}

// silu(z) = z * sigmoid(z) = z/2 + (z/2) tanh(z/2): one MUFU operation
// (tanh.approx, relative error below 2^-10, far inside the bf16 rounding of
// h) instead of an exponential and a reciprocal.  The epilogue of the SwiGLU
// GEMM holds the accumulator while it evaluates 32,768 of these per unit.
__device__ __forceinline__ float silu_f(float z) {
    const float hz = 0.5f * z;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hz));
    return fmaf(hz, t, hz);
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Rows of the placement rule below: a unit needs N columns per accumulator;
// the rule takes half the columns the unit occupies.  Mode 2 fills all of
// tensor memory.
template <int MODE>
__device__ __forceinline__ int tmem_width(const Unit &U) {
    if (MODE == 2) return 256;
    return MODE == 1 && U.nacc == 1 ? (U.N + 1) / 2 : U.N;
}

// Tensor memory is two halves of 256 columns.  A unit with <= 128 rows keeps
// both accumulators in one half (columns +0 and +128) and takes the halves in
// turn, so the epilogue of one such unit overlaps the MMAs of the next; a
// larger unit takes both halves (accumulator 0 in half 0, 1 in half 1).  The
// MMA issuer and the epilogue walk the same sequence of units, so they derive
// the same placement and barrier phases from this state.
struct TmemPlan {
    uint32_t uses[2] = {0u, 0u};  // completed uses of each half
    uint32_t next = 0u;           // half for the next small unit
    // Placement of a unit: first half and whether it spans both.
    __device__ __forceinline__ void place(int N, uint32_t &h, bool &big) const {
        big = N > 128;
        h = big ? 0u : next;
    }
    __device__ __forceinline__ void advance(bool big, uint32_t h) {
        if (big) {
            ++uses[0];
            ++uses[1];
            next = 0u;
        } else {
            ++uses[h];
            next = h ^ 1u;
        }
    }
};

// FP8 epilogue: in the fragment layout of tmem_ld_frag16, register j of a
// 16-column chunk holds feature (lane >> 2) + 8 * fidx(j) of the warp's lane
// quarter and unit row c0 + 2 * (lane & 3) + 8 * ((j >> 2) & 1) + (j & 1):
// four features and four rows per thread.
__device__ __forceinline__ int frag_fidx(int j) { return 2 * (j >> 3) + ((j >> 1) & 1); }
__device__ __forceinline__ int frag_ridx(int j) { return 2 * ((j >> 2) & 1) + (j & 1); }
__device__ __forceinline__ int frag_row_offset(int ri, int lane) { return 2 * (lane & 3) + 8 * (ri >> 1) + (ri & 1); }

// Scales of the four rows a thread holds in the chunk at unit column c0
// (0 for padding rows, whose results are never stored).
template <bool GATHER>
__device__ __forceinline__ void load_row_scales(const GemmArgs &a, const Unit &U, int c0, int lane, float (&rs)[4]) {
#pragma unroll
    for (int ri = 0; ri < 4; ++ri) {
        const int row = unit_row(U, c0 + frag_row_offset(ri, lane));
        float v = 0.0f;
        if (row >= 0) {
            if (GATHER) {
                const int t = __ldg(a.src_token + row);
                v = (unsigned)t < (unsigned)a.T ? __ldg(a.row_scale + t) : 0.0f;
            } else {
                v = __ldg(a.row_scale + row);
            }
        }
        rs[ri] = v;
    }
}

// Multiplies the 16 accumulator values of a chunk by their feature's and
// row's scales (powers of two: exact).
__device__ __forceinline__ void scale_frag(uint32_t (&r)[16], const float (&fs)[4], const float (&rs)[4]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * fs[frag_fidx(j)] * rs[frag_ridx(j)]);
}

// Step 5 for one token t and one 128-feature block b, by 16 lanes (lane l of
// the half-warp owns features 128 b + 8 l .. + 7): out[t] = bf16( sum_j
// w[t,j] * y[dest_row[t,j]] ) in fp32, in slot order, each product and each
// sum rounded on its own -- the arithmetic of the separate combine kernel, so
// the results are identical.  The rows were stored by other warps and other
// SMs: read through L2, all of them in flight at once (k <= 8 per pass).
__device__ __forceinline__ void combine_block_half(const GemmArgs &a, int t, int b, int hl) {
    const int H = a.n_out;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    const int *dr = a.dest_row + (size_t)t * a.k;
    const float *wr = a.topk_w + (size_t)t * a.k;
    for (int j0 = 0; j0 < a.k; j0 += 8) {
        const int nj = min(8, a.k - j0);
        uint4 v[8];
        float w[8];
        int r[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            r[j] = j < nj ? __ldg(dr + j0 + j) : -1;
            w[j] = j < nj ? __ldg(wr + j0 + j) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = (unsigned)r[j] < (unsigned)a.P
                       ? __ldcg(reinterpret_cast<const uint4 *>(a.out + (size_t)r[j] * H + 128 * b + 8 * hl))
                       : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((unsigned)r[j] >= (unsigned)a.P) continue;
            const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p[i]);
                acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w[j], f.x));
                acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w[j], f.y));
            }
        }
    }
    uint4 o;
    uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 pk = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        ow[i] = *reinterpret_cast<const uint32_t *>(&pk);
    }
    *reinterpret_cast<uint4 *>(a.comb_out + (size_t)t * H + 128 * b + 8 * hl) = o;
}

// After a warp has stored its pieces of a down-projection unit (its lane
// quarter's 32 features of every 128-feature block, for its chunks of 16
// rows): one arrival per (row, block), all issued before any result is used
// (one round trip to L2); the warp whose arrival completes a token's block
// combines it, two tokens at a time (one per half-warp).  Every lane fences
// its own stores first, so a combining warp that sees the full count also sees
// every piece of y.
__device__ __forceinline__ void arrive_and_combine(const GemmArgs &a, const Unit &U, int sub, int lane) {
    constexpr int kChunks = (16 + kEpiSub - 1) / kEpiSub;
    __threadfence();
    __syncwarp();
    const int nblk = a.n_out / 128;
    const int b0 = U.fx / 128;
    int tok[kChunks];
    int old[kChunks][2];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int c0 = (sub + kEpiSub * i) * 16;
        tok[i] = -1;
        old[i][0] = old[i][1] = -1;
        if (c0 < U.N && lane < 16) {
            const int row = unit_row(U, c0 + lane);
            if (row >= 0) {
                const int t = __ldg(a.src_token + row);
                if ((unsigned)t < (unsigned)a.T) {
                    tok[i] = t;
                    old[i][0] = atomicAdd(a.comb_cnt + (size_t)t * nblk + b0, 1);
                    if (U.nacc == 2) old[i][1] = atomicAdd(a.comb_cnt + (size_t)t * nblk + b0 + 1, 1);
                }
            }
        }
    }
    const int full = 4 * a.k - 1;
    bool fenced = false;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        for (int acc = 0; acc < U.nacc; ++acc) {
            unsigned mask = __ballot_sync(0xffffffffu, old[i][acc] == full);
            if (mask && !fenced) {
                __threadfence();
                fenced = true;
            }
            while (mask) {
                const int sa = __ffs(mask) - 1;
                mask &= mask - 1;
                int sb = -1;
                if (mask) {
                    sb = __ffs(mask) - 1;
                    mask &= mask - 1;
                }
                const int ta = __shfl_sync(0xffffffffu, tok[i], sa);
                const int tb = __shfl_sync(0xffffffffu, tok[i], sb < 0 ? sa : sb);
                const int t = lane < 16 ? ta : tb;
                if (lane < 16 || sb >= 0) {
                    combine_block_half(a, t, b0 + acc, lane & 15);
                    if ((lane & 15) == 0) a.comb_cnt[(size_t)t * nblk + b0 + acc] = 0;
                }
            }
        }
    }
}

__device__ __forceinline__ void raise_abort(volatile int *abort, uint32_t *status) {
    *abort = 1;
    atomicOr(status, MOE_DEV_GEMM_TIMEOUT);
}

// GATHER (mode 0 only): tmB maps the tokens x [T, H] with one-row boxes and
// the token-tile producer gathers each unit's rows x[src_token[row]] with
// tile::gather4 loads, so the permuted copy x_perm is never materialised.
// FP8 (modes 0 and 1): weights and tokens are e4m3 codes, both K-major (the
// weights stored [E][n_out][K]), 128 K per stage (still 128-byte rows), MMAs
// of kind::f8f6f4; the epilogue multiplies each accumulator by its row's and
// its feature's power-of-two scales (exact) before the bf16 results.
// COMBINE (mode 1 only): the weighted combine of step 5 in the epilogue (see
// arrive_and_combine).
template <int MODE, bool GATHER = false, bool FP8 = false, bool COMBINE = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ RowMaps tmB, GemmArgs a) {
    static_assert(!GATHER || MODE == 0, "the row gather feeds the SwiGLU GEMM");
    static_assert(!COMBINE || MODE == 1, "the combine follows the down projection");
    static_assert(!FP8 || MODE != 2, "the router runs on bf16 planes");
    constexpr int kStageK = FP8 ? 128 : kBK;  // K elements per stage: 128 bytes of each row
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // SW128 tiles need 1 KiB alignment
    uint8_t *ctrl = smem + kRingBytes;
    uint64_t *fullA = reinterpret_cast<uint64_t *>(ctrl);  // weight stage s has landed
    uint64_t *emptyA = fullA + kMaxAStages;                  // weight stage s was read by its MMAs
    uint64_t *fullB = emptyA + kMaxAStages;                  // token stage s has landed
    uint64_t *emptyB = fullB + kMaxBStages;                  // token stage s was read by its MMAs
    uint64_t *tfull = emptyB + kMaxBStages;                    // [2] accumulator half h is ready
    uint64_t *tempty = tfull + 2;                            // [2] accumulator half h is drained
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_gts = reinterpret_cast<int *>(tmem_slot + 2);  // E + 1 <= 257 ints
    int *s_rows = s_gts + 260;                             // GATHER: token of each row of the unit (<= 256)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    // Set-up that reads nothing an earlier kernel writes: barriers, tensor-map
    // prefetch, tensor memory (overlaps the previous kernel's tail when this
    // kernel is launched as its programmatic dependent).
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxAStages; ++s) {
            mbar_init(&fullA[s], 1);
            mbar_init(&emptyA[s], 1);
        }
        for (int s = 0; s < kMaxBStages; ++s) {
            mbar_init(&fullB[s], 1);
            mbar_init(&emptyB[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(mma_done, 1);
        *s_abort = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmA1);
        for (int b = 0; b < kRowBoxes; ++b)
            if ((a.row_boxes >> b) & 1u) tma_prefetch_desc(&tmB.m[b]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the schedule and the token rows come from earlier kernels
    int total, trows;
    int num_fb = a.num_fb, fbw = MODE == 0 ? 128 : 256;
    if (MODE == 2) {
        total = (a.T + a.route_rows - 1) / a.route_rows * a.route_q;
        trows = a.route_rows;
    } else {
        const int ntiles = *a.num_tiles;
        const int nt = ntiles < a.max_tiles ? ntiles : a.max_tiles;
        // Down projection: 128-feature units (one accumulator of up to 256
        // columns: half of tensor memory, so a unit's epilogue overlaps the
        // next unit's MMAs) when they give each CTA fewer operand bytes to
        // load -- rounds x (weight columns + token rows) per K row -- else
        // 256-feature units, which read each token tile once for two
        // accumulators (also with e4m3 operands: 128-feature units for full
        // tiles measured 13% slower on the 8192-token prefill).
        const int grid = (int)gridDim.x;
        const int tr = *a.tile_rows;
        const int r256 = (nt * a.num_fb + grid - 1) / grid, r128 = (nt * (a.n_out / 128) + grid - 1) / grid;
        if (MODE == 1 && r128 * (128 + tr) < r256 * (256 + tr)) {
            num_fb = a.n_out / 128;
            fbw = 128;
        }
        total = nt * num_fb;
        trows = *a.tile_rows;  // the schedule's row cap
    }
    // Balanced waves for the expert GEMMs: with R = ceil(total / grid) units
    // for the busiest CTA, only ceil(total / R) CTAs take units (R or R - 1
    // each), so the last round is not left to a few SMs while the rest idle
    // (896 units on 148 SMs: 128 CTAs x 7 instead of 8 CTAs running a 7th).
    const int rounds = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int stride = MODE == 2 || rounds == 0 ? (int)gridDim.x : (total + rounds - 1) / rounds;
    if ((int)blockIdx.x >= total || (int)blockIdx.x >= stride) {  // uniform: this CTA has no work
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem, kTmemCols);
        }
        return;
    }
    // Two rings: weight stages (the A tiles of both accumulators; mode 2:
    // three weight planes per accumulator), streamed from HBM, and token
    // stages of trows rows (multiple of 16, <= 256).  Four token stages
    // while that leaves at least four weight stages, else three; the weight
    // ring takes the rest, so that as many weight bytes as possible are in
    // flight.  Mode 2 reads both operands from L2 and consumes one stage of
    // each per K block: equally deep rings.
    trows = trows < 16 ? 16 : (trows > kTileRows ? kTileRows : (trows + 15) & ~15);
    // weight tiles per stage: both accumulators' (gate and up, or two
    // 128-feature blocks), one for 128-feature down units (twice the stages)
    const uint32_t a_tiles = MODE == 2 ? 3u * (a.E > 128 ? 2u : 1u) : (MODE == 1 && fbw == 128 ? 1u : 2u);
    const uint32_t a_bytes = a_tiles * kATile, b_bytes = (uint32_t)trows * kBRowBytes;
    int nb = kMaxBStages;
    int fit = (int)((kRingBytes - (uint32_t)nb * b_bytes) / a_bytes);
    if (MODE == 2) {
        nb = (int)(kRingBytes / (a_bytes + b_bytes));
        nb = nb > kMaxBStages ? kMaxBStages : nb;
        fit = nb;
    } else if (fit < 4) {
        nb = 3;
        fit = (int)((kRingBytes - (uint32_t)nb * b_bytes) / a_bytes);
    }
    const int na = fit > kMaxAStages ? kMaxAStages : fit;
    uint8_t *ringB = smem + (uint32_t)na * a_bytes;  // a_bytes is a multiple of 16 KiB: 1 KiB aligned

    if (MODE != 2)
        for (int i = threadIdx.x; i <= a.E; i += kThreads) s_gts[i] = a.grp_tile_start[i];
    __syncthreads();
    const int nk = a.K / kStageK;

    if (GATHER && warp == 2) {
        // ------------------- token rows gathered from x by src_token (warp 2) ----
        // tile::gather4 loads of four rows x[src_token[r]] each (one-row
        // boxes, 128-byte swizzle by shared-memory address, so the rows land
        // exactly where a tiled load of x_perm would put them).  The TMA unit
        // moves these at a lower rate than whole tiles, so this pays off when
        // units have few rows (the gather pass it replaces dominates then).
        int stage = 0;
        uint32_t ph = 0;
        int issued_ph[kMaxBStages];
        for (int s = 0; s < kMaxBStages; ++s) issued_ph[s] = -1;
        for (int u = blockIdx.x; u < total; u += stride) {
            Unit U;
            decode_unit<MODE>(u, s_gts, a, trows, num_fb, fbw, U);
            if (!U.valid) continue;
            // The unit's tokens, one per tile row; padding rows repeat the
            // first row (their results are never stored).  Loads already
            // issued took their row coordinates from registers.
            __syncwarp();
            bool bad = false;
            for (int c = lane; c < U.N; c += 32) {
                int r = unit_row(U, c);
                if (r < 0) r = U.p0s;
                int t = a.src_token[r];
                if ((unsigned)t >= (unsigned)a.T) {
                    bad = true;
                    t = 0;
                }
                s_rows[c] = t;
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.status, MOE_DEV_BAD_ROW);
            __syncwarp();
            const uint32_t bytes = (uint32_t)U.N * kBRowBytes;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                int got = 1;
                if (lane == 0) got = mbar_wait_bounded(&emptyB[stage], ph ^ 1u, a.timeout_ns, s_abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&fullB[stage], bytes);
                    uint8_t *sb = ringB + stage * b_bytes;
                    const int kx = kb * kStageK;
                    for (int g = 0; g < U.N; g += 4)
                        tma_gather4(sb + g * kBRowBytes, &tmB.m[0], &fullB[stage], kx, s_rows[g], s_rows[g + 1],
                                    s_rows[g + 2], s_rows[g + 3]);
                    issued_ph[stage] = (int)ph;
                }
                if (++stage == nb) {
                    stage = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) {
                if (lane == 0 && !*s_abort) raise_abort(s_abort, a.status);
                break;
            }
        }
        // Every issued copy must land before the CTA may leave.
        if (lane == 0) {
            int never = 0;
            for (int s = 0; s < nb; ++s)
                if (issued_ph[s] >= 0) mbar_wait_bounded(&fullB[s], (uint32_t)issued_ph[s], a.timeout_ns, &never);
        }
        __syncwarp();
    } else if (warp == 0 || warp == 2) {
        // ----------------------------- TMA producers: warp 0 weights, warp 2 tokens ----
        if (lane == 0) {
            const bool is_a = warp == 0;
            const int nst = is_a ? na : nb;
            uint64_t *full = is_a ? fullA : fullB;
            uint64_t *empty = is_a ? emptyA : emptyB;
            int stage = 0;
            uint32_t ph = 0;
            int issued_ph[kMaxAStages];
            for (int s = 0; s < kMaxAStages; ++s) issued_ph[s] = -1;
            for (int u = blockIdx.x; u < total; u += stride) {
                Unit U;
                decode_unit<MODE>(u, s_gts, a, trows, num_fb, fbw, U);
                if (!U.valid) {
                    if (is_a) atomicOr(a.status, MOE_DEV_BAD_ROW);
                    continue;
                }
                const int fx0 = U.fx;
                const int fx1 = MODE == 0 ? U.fx : U.fx + 128;
                const int nb0 = (U.p0l + 15) >> 4, nb1 = (U.p1l + 15) >> 4;
                const uint32_t bytes = is_a ? (MODE == 2 ? 3u : 1u) * (uint32_t)U.nacc * kATile
                                            : (uint32_t)(nb0 + nb1) * kBBox;
                const int krow = U.e * a.K;
                const int kb0 = MODE == 2 ? U.fb * a.route_kb : 0;
                const int kb1 = MODE == 2 ? min(nk, kb0 + a.route_kb) : nk;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], ph ^ 1u, a.timeout_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    if (!is_a && a.stall_first_stage && blockIdx.x == 0 && u == (int)blockIdx.x && kb == kb0) {
                        // test hook: this stage is never loaded (no copy is in
                        // flight for it), so the MMA issuer's wait expires
                        if (++stage == nst) {
                            stage = 0;
                            ph ^= 1u;
                        }
                        continue;
                    }
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    const int ky = krow + kb * kBK, kx = kb * kStageK;
                    if (!is_a) {
                        uint8_t *sb = ringB + stage * b_bytes;
                        tma_load_rows(sb, tmB, a.row_boxes, &full[stage], kx, U.p0s, 16 * nb0);
                        if (nb1) tma_load_rows(sb + U.n0p * kBRowBytes, tmB, a.row_boxes, &full[stage], kx, U.p1s, 16 * nb1);
                    } else if (MODE == 2) {
                        // tile (plane p, accumulator c) at index p * nacc + c;
                        // plane p holds rows [p*K, (p+1)*K) of the plane tensor
                        uint8_t *sa0 = smem + stage * a_bytes;
                        for (int pl = 0; pl < 3; ++pl)
                            for (int c = 0; c < U.nacc; ++c) {
                                uint8_t *dst = sa0 + (uint32_t)(pl * U.nacc + c) * kATile;
                                tma_load_2d(dst, &tmA0, &full[stage], c * 128, pl * a.K + kx);
                                tma_load_2d(dst + kABox, &tmA0, &full[stage], c * 128 + 64, pl * a.K + kx);
                            }
                    } else if (FP8) {
                        // one 128-feature x 128-K tile of codes per accumulator,
                        // 16 KB contiguous (tile-blocked, K-major inside: rows
                        // of 128 bytes, tile (e, n / 128, k / 128) at row
                        // ((e * n_out / 128 + n / 128) * K / 128 + k / 128) * 128)
                        uint8_t *sa0 = smem + stage * a_bytes;
                        const int nbk = a.n_out / 128, kbk = a.K / 128;
                        const int trow0 = ((U.e * nbk + fx0 / 128) * kbk + kx / 128) * 128;
                        tma_load_2d(sa0, &tmA0, &full[stage], 0, trow0);
                        if (U.nacc == 2)
                            tma_load_2d(sa0 + kATile, &tmA1, &full[stage], 0,
                                        ((U.e * nbk + fx1 / 128) * kbk + kx / 128) * 128);
                    } else {
                        uint8_t *sa0 = smem + stage * a_bytes, *sa1 = sa0 + kATile;
                        tma_load_2d(sa0, &tmA0, &full[stage], fx0, ky);
                        tma_load_2d(sa0 + kABox, &tmA0, &full[stage], fx0 + 64, ky);
                        if (U.nacc == 2) {
                            tma_load_2d(sa1, &tmA1, &full[stage], fx1, ky);
                            tma_load_2d(sa1 + kABox, &tmA1, &full[stage], fx1 + 64, ky);
                        }
                    }
                    issued_ph[stage] = (int)ph;
                    if (++stage == nst) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    if (!*s_abort) raise_abort(s_abort, a.status);
                    break;
                }
            }
            // Every issued copy must land before the CTA may leave.
            int never = 0;
            for (int s = 0; s < nst; ++s)
                if (issued_ph[s] >= 0) mbar_wait_bounded(&full[s], (uint32_t)issued_ph[s], a.timeout_ns, &never);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (lane == 0) {
            int sa = 0, sb = 0;
            uint32_t pha = 0, phb = 0;
            TmemPlan plan;
            const uint32_t baseA = smem_u32(smem), baseB = smem_u32(ringB);
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += stride) {
                Unit U;
                decode_unit<MODE>(u, s_gts, a, trows, num_fb, fbw, U);
                if (!U.valid) continue;
                const uint32_t idesc = FP8 ? idesc_e4m3_f32(128, U.N) : idesc_bf16_f32(128, U.N, 1, 0);
                uint32_t h;
                bool big;
                plan.place(tmem_width<MODE>(U), h, big);  // mode 2 uses all of tensor memory
                const uint32_t d0 = tmem + h * 256u, d1 = big ? tmem + 256u : d0 + 128u;
                // wait until the epilogue has drained the half(s) this unit takes
                ok = mbar_wait_bounded(&tempty[h], (plan.uses[h] & 1u) ^ 1u, a.timeout_ns, s_abort);
                if (ok && big) ok = mbar_wait_bounded(&tempty[1], (plan.uses[1] & 1u) ^ 1u, a.timeout_ns, s_abort);
                if (!ok) break;
                tc_fence_after();
                const int kb0 = MODE == 2 ? U.fb * a.route_kb : 0;
                const int kb1 = MODE == 2 ? min(nk, kb0 + a.route_kb) : nk;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&fullA[sa], pha, a.timeout_ns, s_abort) ||
                        !mbar_wait_bounded(&fullB[sb], phb, a.timeout_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa0 = baseA + sa * a_bytes, sa1 = sa0 + kATile, sbt = baseB + sb * b_bytes;
                    if (MODE == 2) {
                        // accumulator (group g, expert block c) at column (g * nacc + c) * trows
                        const int j = kb - kb0, g = j % a.route_groups;
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint64_t bdesc = sdesc_sw128(sbt + kk * 32, 16, 1024);
                            for (int pl = 0; pl < 3; ++pl)
                                for (int c = 0; c < U.nacc; ++c) {
                                    const uint32_t at = sa0 + (uint32_t)(pl * U.nacc + c) * kATile + kk * 2048;
                                    const uint32_t dst = tmem + (uint32_t)((g * U.nacc + c) * trows);
                                    const uint32_t accum = (j >= a.route_groups || kk || pl) ? 1u : 0u;
                                    tc_mma_bf16(dst, sdesc_sw128(at, kABox, 1024), bdesc, idesc, accum);
                                }
                        }
                    } else if (FP8) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            // A and B K-major: 32 K (32 bytes) per MMA inside the 128-byte rows
                            const uint64_t bdesc = sdesc_sw128(sbt + kk * 32, 16, 1024);
                            const uint32_t accum = (kb | kk) ? 1u : 0u;
                            tc_mma_f8(d0, sdesc_sw128(sa0 + kk * 32, 16, 1024), bdesc, idesc, accum);
                            if (U.nacc == 2) tc_mma_f8(d1, sdesc_sw128(sa1 + kk * 32, 16, 1024), bdesc, idesc, accum);
                        }
                    } else
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // B: K-major, 16 K-elements (32 bytes) per MMA inside the 128-byte row.
                        const uint64_t bdesc = sdesc_sw128(sbt + kk * 32, 16, 1024);
                        // A: MN-major, 16 K-rows (2 KiB) per MMA; the two 64-feature halves 8 KiB apart.
                        const uint64_t a0desc = sdesc_sw128(sa0 + kk * 2048, kABox, 1024);
                        const uint32_t accum = (kb | kk) ? 1u : 0u;
                        tc_mma_bf16(d0, a0desc, bdesc, idesc, accum);
                        if (U.nacc == 2) {
                            const uint64_t a1desc = sdesc_sw128(sa1 + kk * 2048, kABox, 1024);
                            tc_mma_bf16(d1, a1desc, bdesc, idesc, accum);
                        }
                    }
                    // each stage is freed once these MMAs have read it
                    tc_commit(&emptyA[sa]);
                    tc_commit(&emptyB[sb]);
                    if (++sa == na) {
                        sa = 0;
                        pha ^= 1u;
                    }
                    if (++sb == nb) {
                        sb = 0;
                        phb ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tfull[h]);
                if (big) tc_commit(&tfull[1]);
                plan.advance(big, h);
            }
            if (!ok && !*s_abort) raise_abort(s_abort, a.status);
            // All MMAs issued by this thread complete before tensor memory is freed.
            int never = 0;
            tc_commit(mma_done);
            mbar_wait_bounded(mma_done, 0, a.timeout_ns, &never);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- epilogue ----
        const int q = warp & 3;              // tensor-memory lane quarter of this warp
        const int sub = (warp - kEpiWarp0) >> 2;  // which 16-column chunks: sub, sub + kEpiSub, ...
        const int L = q * 32 + lane;         // feature within a 128-feature accumulator
        uint8_t *stg = smem + kRingBytes + kCtrlBytes + (warp - kEpiWarp0) * kEpiStageBytes;
        const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
        TmemPlan plan;
        for (int u = blockIdx.x; u < total; u += stride) {
            Unit U;
            decode_unit<MODE>(u, s_gts, a, trows, num_fb, fbw, U);
            if (!U.valid) continue;
            // FP8: the scales of this thread's four features in each accumulator
            float fs0[4] = {1.0f, 1.0f, 1.0f, 1.0f}, fs1[4] = {1.0f, 1.0f, 1.0f, 1.0f};
            if (FP8) {
                const size_t fb0 = (size_t)U.e * a.n_out + U.fx + q * 32 + (lane >> 2);
                const size_t fb1 = MODE == 0 ? fb0 : fb0 + 128;
#pragma unroll
                for (int fi = 0; fi < 4; ++fi) {
                    fs0[fi] = __ldg(a.w_scale0 + fb0 + 8 * fi);
                    if (MODE == 0 || U.nacc == 2) fs1[fi] = __ldg(a.w_scale1 + fb1 + 8 * fi);
                }
            }
            uint32_t h;
            bool big;
            plan.place(tmem_width<MODE>(U), h, big);
            // The whole warp takes one decision, so the .sync.aligned loads
            // below never run with part of the warp.
            bool got = mbar_wait_bounded(&tfull[h], plan.uses[h] & 1u, a.timeout_ns, s_abort);
            if (got && big) got = mbar_wait_bounded(&tfull[1], plan.uses[1] & 1u, a.timeout_ns, s_abort);
            const bool ready = __all_sync(0xffffffffu, got);
            if (!ready) {
                if (lane == 0 && !*s_abort) raise_abort(s_abort, a.status);
                break;
            }
            tc_fence_after();
            const uint32_t t0 = tq + h * 256u, t1 = big ? tq + 256u : t0 + 128u;
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&tempty[h]);
                    if (big) mbar_arrive(&tempty[1]);
                }
            };
            if (MODE == 2) {
                // fp32 partial logits of K range U.fb: lane L of expert block c
                // is expert c*128 + L; the groups' sums are added in order
                // g = 0, 1, ...
                const int kb0 = U.fb * a.route_kb;
                const int nkr = min(nk, kb0 + a.route_kb) - kb0;
                const int ng = nkr < a.route_groups ? nkr : a.route_groups;
                float *part = a.logits + (size_t)U.fb * a.T * a.E;
                for (int c0 = sub * 16; c0 < U.N; c0 += 16 * kEpiSub) {
                    for (int c = 0; c < U.nacc; ++c) {
                        float acc[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
                        for (int g = 0; g < ng; ++g) {
                            uint32_t r[16];
                            tmem_ld16(tq + (uint32_t)((g * U.nacc + c) * trows + c0), r);
                            tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 16; ++j) acc[j] += __uint_as_float(r[j]);
                        }
                        const int e = c * 128 + L;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int row = unit_row(U, c0 + j);
                            if (row >= 0 && e < a.E) part[(size_t)row * a.E + e] = acc[j];
                        }
                    }
                }
                release();
                plan.advance(big, h);
                continue;
            }
            if (MODE == 1 && big) {
                // Two accumulators of up to 256 columns each: accumulator 0 of
                // every chunk and accumulator 1 of the first kHold1 chunks go to
                // registers as packed bf16; the rest of accumulator 1 is stored
                // while the accumulator is held.  Then the accumulator goes back
                // to the MMA warp and the registers are stored, overlapping the
                // next unit's MMAs (when every CTA stores its whole unit while
                // holding it, the stores of all SMs collide and the tensor cores
                // wait for them).
                constexpr int kBigChunks = (16 + kEpiSub - 1) / kEpiSub;
                constexpr int kHold1 = 1;
                uint32_t h0[kBigChunks][8], h1[kHold1 > 0 ? kHold1 : 1][8];
#pragma unroll
                for (int i = 0; i < kBigChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) {
                        uint32_t r[16];
                        float rs[4];
                        if (FP8) load_row_scales<GATHER>(a, U, c0, lane, rs);
                        tmem_ld_frag16(t0 + (uint32_t)c0, r);
                        tmem_ld_wait();
                        if (FP8) scale_frag(r, fs0, rs);
#pragma unroll
                        for (int m = 0; m < 8; ++m) h0[i][m] = pack_bf16x2(r[2 * m], r[2 * m + 1]);
                    }
                }
                if (U.nacc == 2) {
#pragma unroll
                    for (int i = 0; i < kBigChunks; ++i) {
                        const int c0 = (sub + kEpiSub * i) * 16;
                        if (c0 < U.N) {
                            uint32_t r[16];
                            float rs[4];
                            if (FP8) load_row_scales<GATHER>(a, U, c0, lane, rs);
                            tmem_ld_frag16(t1 + (uint32_t)c0, r);
                            tmem_ld_wait();
                            if (FP8) scale_frag(r, fs1, rs);
                            if (i < kHold1) {
#pragma unroll
                                for (int m = 0; m < 8; ++m) h1[i][m] = pack_bf16x2(r[2 * m], r[2 * m + 1]);
                            } else {
                                uint32_t w[8];
#pragma unroll
                                for (int m = 0; m < 8; ++m) w[m] = pack_bf16x2(r[2 * m], r[2 * m + 1]);
                                store_block_frag(w, stg, a.out, a.n_out, a.row_addr, U.fx + 128 + q * 32, U, c0);
                            }
                        }
                    }
                }
                release();
#pragma unroll
                for (int i = 0; i < kBigChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) {
                        store_block_frag(h0[i], stg, a.out, a.n_out, a.row_addr, U.fx + q * 32, U, c0);
                        if (i < kHold1 && U.nacc == 2) store_block_frag(h1[i], stg, a.out, a.n_out, a.row_addr, U.fx + 128 + q * 32, U, c0);
                    }
                }
                if (COMBINE) arrive_and_combine(a, U, sub, lane);
                plan.advance(big, h);
                continue;
            }
            if (MODE == 1 && U.nacc == 1) {
                // One accumulator of up to 256 columns in one half: up to four
                // 16-column chunks per warp, packed into registers, then handed
                // back before the stores.
                constexpr int kOneChunks = (16 + kEpiSub - 1) / kEpiSub;
                uint32_t h0[kOneChunks][8];
#pragma unroll
                for (int i = 0; i < kOneChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) {
                        uint32_t r[16];
                        float rs[4];
                        if (FP8) load_row_scales<GATHER>(a, U, c0, lane, rs);
                        tmem_ld_frag16(t0 + (uint32_t)c0, r);
                        tmem_ld_wait();
                        if (FP8) scale_frag(r, fs0, rs);
#pragma unroll
                        for (int m = 0; m < 8; ++m) h0[i][m] = pack_bf16x2(r[2 * m], r[2 * m + 1]);
                    }
                }
                release();
#pragma unroll
                for (int i = 0; i < kOneChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) store_block_frag(h0[i], stg, a.out, a.n_out, a.row_addr, U.fx + q * 32, U, c0);
                }
                if (COMBINE) arrive_and_combine(a, U, sub, lane);
                plan.advance(big, h);
                continue;
            }
            // Phase 1 (holds the accumulator): load this warp's 16-column
            // chunks (sub, sub + kEpiSub, ...), finish the values and keep them as
            // packed bf16 pairs in registers.
            constexpr int kHoldChunks = MODE == 0 ? (16 + kEpiSub - 1) / kEpiSub   // N <= 256
                                                  : (8 + kEpiSub - 1) / kEpiSub;   // mode 1 here: N <= 128
            constexpr int kHoldWords = MODE == 0 ? 8 : 16;
            uint32_t hold[kHoldChunks][kHoldWords];
#pragma unroll
            for (int i = 0; i < kHoldChunks; ++i) {
                const int c0 = (sub + kEpiSub * i) * 16;
                if (c0 < U.N) {
                    uint32_t r0[16], r1[16];
                    float rs[4];
                    if (FP8) load_row_scales<GATHER>(a, U, c0, lane, rs);
                    tmem_ld_frag16(t0 + (uint32_t)c0, r0);
                    if (U.nacc == 2) tmem_ld_frag16(t1 + (uint32_t)c0, r1);
                    tmem_ld_wait();
                    if (FP8) {
                        scale_frag(r0, fs0, rs);
                        if (U.nacc == 2) scale_frag(r1, fs1, rs);
                    }
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        if (MODE == 0) {
                            const float g0 = __uint_as_float(r0[j]), v0 = __uint_as_float(r1[j]);
                            const float g1 = __uint_as_float(r0[j + 1]), v1 = __uint_as_float(r1[j + 1]);
                            const __nv_bfloat162 p = __floats2bfloat162_rn(silu_f(g0) * v0, silu_f(g1) * v1);
                            hold[i][j / 2] = *reinterpret_cast<const uint32_t *>(&p);
                        } else {
                            const __nv_bfloat162 p0 =
                                __floats2bfloat162_rn(__uint_as_float(r0[j]), __uint_as_float(r0[j + 1]));
                            hold[i][j / 2] = *reinterpret_cast<const uint32_t *>(&p0);
                            if (U.nacc == 2) {
                                const __nv_bfloat162 p1 =
                                    __floats2bfloat162_rn(__uint_as_float(r1[j]), __uint_as_float(r1[j + 1]));
                                hold[i][8 + j / 2] = *reinterpret_cast<const uint32_t *>(&p1);
                            }
                        }
                    }
                }
            }
            // Hand the accumulator back to the MMA warp before the stores.
            release();
            // Phase 2: the stores, 16-byte vectors of eight features per row.
#pragma unroll
            for (int i = 0; i < kHoldChunks; ++i) {
                const int c0 = (sub + kEpiSub * i) * 16;
                if (c0 < U.N) {
                    uint32_t w[8];
#pragma unroll
                    for (int m = 0; m < 8; ++m) w[m] = hold[i][m];
                    store_block_frag(w, stg, a.out, a.n_out, a.row_addr, U.fx + q * 32, U, c0);
                    if (MODE == 1 && U.nacc == 2) {
#pragma unroll
                        for (int m = 0; m < 8; ++m) w[m] = hold[i][8 + m];
                        store_block_frag(w, stg, a.out, a.n_out, a.row_addr, U.fx + 128 + q * 32, U, c0);
                    }
                }
            }
            if (COMBINE) arrive_and_combine(a, U, sub, lane);
            plan.advance(big, h);
        }
    }

    tc_fence_before();
    __syncthreads();
    // Results stored into other GPUs' memory (row addresses): one
    // system-scope fence, cumulative over the block's stores, before the
    // collective that follows the kernel.
    if (MODE == 1 && a.row_addr && threadIdx.x == 0) __threadfence_system();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Exact three-way bf16 split of the router weights: p0 = bf16(w),
// p1 = bf16(w - p0), p2 = bf16(w - p0 - p1) (each difference is exact in
// fp32), written as planes[3][H][Ep]; columns e >= E are zero.
__global__ void __launch_bounds__(256) k_router_planes(const float *__restrict__ w, __nv_bfloat16 *__restrict__ planes,
                                                       int H, int E, int Ep) {
    pdl_trigger();
    const size_t n = (size_t)H * Ep;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int h = (int)(i / Ep), e = (int)(i % Ep);
        const float v = e < E ? w[(size_t)h * E + e] : 0.0f;
        const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(p1);
        planes[i] = p0;
        planes[n + i] = p1;
        planes[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D tensor map over a row-major [rows, cols] matrix of bf16 (or, with
// bytes = true, of 8-bit codes) with the 128-byte swizzle; box = box_cols x
// box_rows (box_cols elements must span 128 bytes).
bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows, bool bytes = false) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (bytes ? 1 : 2)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void *>(ptr), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The token matrix with boxes of 16, 32, ... 256 rows; returns the mask of the
// maps that could be encoded (bit 0 is required).
uint32_t make_row_maps(RowMaps *rm, const void *ptr, uint64_t rows, uint64_t cols, uint32_t min_rows = 16,
                       bool bytes = false) {
    uint32_t boxes = 0;
    for (int i = 0; i < kRowBoxes; ++i)
        if (make_tmap(&rm->m[i], ptr, rows, cols, bytes ? 128 : 64, min_rows << i, bytes)) boxes |= 1u << i;
    return (boxes & 1u) ? boxes : 0u;
}

}  // namespace

// Router logits on the tensor cores: planes of W_r into the workspace, then
// mode 2 of the grouped GEMM (one unit per block of route_rows tokens and
// range of the hidden dimension), which writes the partial-logit planes
// `part` [q][T][E]; returns q.
cudaError_t launch_router_logits_tc(const moe_shape &s, const void *x, const float *w_router, float *part, int *q,
                                    const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                    cudaStream_t stream) {
    const int Ep = router_plane_cols(s.E);
    __nv_bfloat16 *planes = (__nv_bfloat16 *)((char *)ws + L.router_planes);
    const size_t n = (size_t)s.H * Ep;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 4 * num_sms) blocks = 4 * num_sms;
    k_router_planes<<<blocks, 256, 0, stream>>>(w_router, planes, s.H, s.E, Ep);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    CUtensorMap tA;
    RowMaps tB;
    if (!make_tmap(&tA, planes, 3 * (uint64_t)s.H, (uint64_t)Ep, 64, 64)) return cudaErrorInvalidValue;
    const uint32_t boxes = make_row_maps(&tB, x, (uint64_t)s.T, (uint64_t)s.H);
    if (!boxes) return cudaErrorInvalidValue;
    WsPtrs p = ws_ptrs(ws, L);
    GemmArgs a = {};
    a.status = p.status;
    a.K = s.H;
    a.E = s.E;
    a.timeout_ns = timeout_ns;
    a.logits = part;
    a.T = s.T;
    const RouterTcPlan plan = router_tc_plan(s.T, s.H, s.E, num_sms);
    a.route_rows = plan.rows;
    a.route_q = plan.q;
    a.route_kb = plan.kb;
    a.route_groups = plan.groups;
    a.row_boxes = boxes;
    static bool attr_done = false;
    if (!attr_done) {
        err = cudaFuncSetAttribute(k_grouped_gemm<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (err != cudaSuccess) return err;
        attr_done = true;
    }
    *q = plan.q;
    return launch_pdl(k_grouped_gemm<2>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA, tA, tB, a);
}

// mode 0: act = x_perm [P,H], w0 = gate, w1 = up, out = h [P,F]
//         (with src_token: act = x [T,H], rows gathered as x[src_token[row]])
// mode 1: act = h [P,F],      w0 = w1 = down,   out = y [P,H]
// comb (mode 1, nullable): the combine of step 5 in the epilogue, into comb->out.
cudaError_t launch_grouped_gemm(int mode, const moe_shape &s, const void *act, const void *w0, const void *w1,
                                void *out, const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                cudaStream_t stream, const int32_t *src_token, const CombineOut *comb,
                                const unsigned long long *row_addr) {
    const bool gather = mode == 0 && src_token != nullptr;
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, capped);
    const int K = mode == 0 ? s.H : s.F;
    const int n_out = mode == 0 ? s.F : s.H;
    CUtensorMap tA0, tA1;
    RowMaps tB;
    uint32_t boxes = 0;
    if (!make_tmap(&tA0, w0, (uint64_t)s.E * K, (uint64_t)n_out, 64, 64) ||
        !make_tmap(&tA1, w1, (uint64_t)s.E * K, (uint64_t)n_out, 64, 64))
        return cudaErrorInvalidValue;
    if (gather) {
        if (!make_tmap(&tB.m[0], act, (uint64_t)s.T, (uint64_t)K, 64, 1)) return cudaErrorInvalidValue;
        boxes = 1u;
    } else if (!(boxes = make_row_maps(&tB, act, (uint64_t)P, (uint64_t)K))) {
        return cudaErrorInvalidValue;
    }
    WsPtrs p = ws_ptrs(ws, L);
    GemmArgs a = {};
    a.tile_map = p.tile_map;
    a.grp_tile_start = p.grp_tile_start;
    a.num_tiles = p.num_tiles;
    a.tile_rows = p.tile_rows;
    a.status = p.status;
    a.out = (__nv_bfloat16 *)out;
    a.n_out = n_out;
    a.K = K;
    a.num_fb = mode == 0 ? s.F / 128 : (s.H + 255) / 256;
    a.E = s.E;
    a.P = (int)P;
    a.max_tiles = L.max_tiles;
    a.timeout_ns = timeout_ns;
    a.T = s.T;
    a.src_token = src_token;
    a.row_boxes = boxes;
    a.stall_first_stage = (mode == 0 && !gather && (s.flags & MOE_FLAG_TEST_STALL_GEMM)) ? 1 : 0;
    a.row_addr = (mode == 1 && !comb) ? row_addr : nullptr;
    static bool attr_done[6] = {false, false, false, false, false, false};
    cudaError_t err;
    if (mode == 1 && comb) {
        a.src_token = comb->src_token;
        a.dest_row = comb->dest_row;
        a.topk_w = comb->topk_w;
        a.comb_out = (__nv_bfloat16 *)comb->out;
        a.comb_cnt = (int *)((char *)ws + L.combine_cnt);
        a.k = s.k;
        if (!attr_done[5]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<1, false, false, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[5] = true;
        }
        err = launch_pdl(k_grouped_gemm<1, false, false, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else if (gather) {
        if (!attr_done[2]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[2] = true;
        }
        err = launch_pdl(k_grouped_gemm<0, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else if (mode == 0) {
        if (!attr_done[0]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[0] = true;
        }
        err = launch_pdl(k_grouped_gemm<0>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else {
        if (!attr_done[1]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[1] = true;
        }
        err = launch_pdl(k_grouped_gemm<1>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    }
    return cudaGetLastError();
}

// FP8 expert GEMMs.  mode 0: act = the e4m3 token rows (x_perm codes [P,H],
// or with src_token the per-token codes [T,H] gathered by row), w0/w1 = gate/
// up codes [E][F][H] with scales [E][F]; mode 1: act = h codes [P,F], w0 = w1
// = down codes [E][H][F] with scales [E][H].  row_scale: one per row of act.
cudaError_t launch_grouped_gemm_fp8(int mode, const moe_shape &s, const void *act, const float *row_scale,
                                    const void *w0, const float *w0_scale, const void *w1, const float *w1_scale,
                                    void *out, const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                    cudaStream_t stream, const int32_t *src_token, const CombineOut *comb,
                                    const unsigned long long *row_addr) {
    const bool gather = mode == 0 && src_token != nullptr;
    const bool capped = (s.flags & MOE_FLAG_CAPACITY) != 0;
    const int64_t P = permuted_rows(s.T, s.E, s.k, s.C, capped);
    const int K = mode == 0 ? s.H : s.F;
    const int n_out = mode == 0 ? s.F : s.H;
    CUtensorMap tA0, tA1;
    RowMaps tB;
    uint32_t boxes = 0;
    // the tile-blocked codes as rows of 128 bytes (E * n_out * K / 128 rows,
    // addressed with int32 coordinates)
    if ((int64_t)s.E * n_out * (K / 128) >= (1ll << 31)) return cudaErrorInvalidValue;
    if (!make_tmap(&tA0, w0, (uint64_t)s.E * n_out * (K / 128), 128, 128, 128, true) ||
        !make_tmap(&tA1, w1, (uint64_t)s.E * n_out * (K / 128), 128, 128, 128, true))
        return cudaErrorInvalidValue;
    if (gather) {
        if (!make_tmap(&tB.m[0], act, (uint64_t)s.T, (uint64_t)K, 128, 1, true)) return cudaErrorInvalidValue;
        boxes = 1u;
    } else if (!(boxes = make_row_maps(&tB, act, (uint64_t)P, (uint64_t)K, 16, true))) {
        return cudaErrorInvalidValue;
    }
    WsPtrs p = ws_ptrs(ws, L);
    GemmArgs a = {};
    a.tile_map = p.tile_map;
    a.grp_tile_start = p.grp_tile_start;
    a.num_tiles = p.num_tiles;
    a.tile_rows = p.tile_rows;
    a.status = p.status;
    a.out = (__nv_bfloat16 *)out;
    a.n_out = n_out;
    a.K = K;
    a.num_fb = mode == 0 ? s.F / 128 : (s.H + 255) / 256;
    a.E = s.E;
    a.P = (int)P;
    a.max_tiles = L.max_tiles;
    a.timeout_ns = timeout_ns;
    a.T = s.T;
    a.src_token = src_token;
    a.row_boxes = boxes;
    a.w_scale0 = w0_scale;
    a.w_scale1 = w1_scale;
    a.row_scale = row_scale;
    a.row_addr = (mode == 1 && !comb) ? row_addr : nullptr;
    static bool attr_done[4] = {false, false, false, false};
    cudaError_t err;
    auto setup = [&](const void *fn, int i) -> cudaError_t {
        if (attr_done[i]) return cudaSuccess;
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e == cudaSuccess) attr_done[i] = true;
        return e;
    };
    if (mode == 1 && comb) {
        a.src_token = comb->src_token;
        a.dest_row = comb->dest_row;
        a.topk_w = comb->topk_w;
        a.comb_out = (__nv_bfloat16 *)comb->out;
        a.comb_cnt = (int *)((char *)ws + L.combine_cnt);
        a.k = s.k;
        if ((err = setup((const void *)k_grouped_gemm<1, false, true, true>, 3)) != cudaSuccess) return err;
        err = launch_pdl(k_grouped_gemm<1, false, true, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else if (gather) {
        if ((err = setup((const void *)k_grouped_gemm<0, true, true>, 0)) != cudaSuccess) return err;
        err = launch_pdl(k_grouped_gemm<0, true, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else if (mode == 0) {
        if ((err = setup((const void *)k_grouped_gemm<0, false, true>, 1)) != cudaSuccess) return err;
        err = launch_pdl(k_grouped_gemm<0, false, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    } else {
        if ((err = setup((const void *)k_grouped_gemm<1, false, true>, 2)) != cudaSuccess) return err;
        err = launch_pdl(k_grouped_gemm<1, false, true>, dim3(num_sms), dim3(kThreads), kSmemBytes, stream, tA0, tA1, tB, a);
        if (err != cudaSuccess) return err;
    }
    return cudaGetLastError();
}

}  // namespace moe
