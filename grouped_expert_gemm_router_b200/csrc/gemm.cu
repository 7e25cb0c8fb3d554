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
constexpr int kMaxAStages = 8;
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
// features per CTA, 256 per CTA pair; mode 1: 256 features in two
// accumulators, or 128 in one when that still fits one wave).
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

// Stores a 32-feature x 16-row block of bf16 results held by one warp: lane l
// holds feature fbase + l of unit rows c0 .. c0 + 15 as w[m] = (row 2m, row
// 2m + 1).  Three butterfly exchanges (lanes ^1, ^2, ^4) leave each lane eight
// consecutive features of unit rows c0 + (l & 7) and c0 + 8 + (l & 7), stored
// as two 16-byte vectors: a warp writes the block with 2 store instructions
// instead of 16, and the epilogue's time is set by its store instructions.
__device__ __forceinline__ void store_block_32x16(const uint32_t (&w)[8], __nv_bfloat16 *out, int n_out, int fbase,
                                                  const Unit &U, int c0) {
    const int lane = threadIdx.x & 31;
    const bool p = lane & 1, P = (lane >> 1) & 1, Q = (lane >> 2) & 1;
    // (two rows, one feature) -> (one row, two features): x[m] = row 2m + p,
    // features (l & ~1) and (l & ~1) + 1
    uint32_t x[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, w[m], 1);
        x[m] = p ? __byte_perm(o, w[m], 0x7632) : __byte_perm(w[m], o, 0x5410);
    }
    // keep m = 2t + P: y[t] = row 4t + 2P + p, features (l & ~3) .. + 3
    uint32_t y[4][2];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint32_t keep = P ? x[2 * t + 1] : x[2 * t];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, P ? x[2 * t] : x[2 * t + 1], 2);
        y[t][0] = P ? recv : keep;
        y[t][1] = P ? keep : recv;
    }
    // keep t = 2s + Q: row 8s + (l & 7), features (l & ~7) .. + 7
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const uint32_t k0 = Q ? y[2 * s + 1][0] : y[2 * s][0], k1 = Q ? y[2 * s + 1][1] : y[2 * s][1];
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, Q ? y[2 * s][0] : y[2 * s + 1][0], 4);
        const uint32_t r1 = __shfl_xor_sync(0xffffffffu, Q ? y[2 * s][1] : y[2 * s + 1][1], 4);
        const int row = unit_row(U, c0 + 8 * s + (lane & 7));
        if (row >= 0)
            *reinterpret_cast<uint4 *>(out + (size_t)row * n_out + fbase + (lane & ~7)) =
                Q ? make_uint4(r0, r1, k0, k1) : make_uint4(k0, k1, r0, r1);
    }
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
                                                 int fbase, const Unit &U, int c0) {
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
        if (row >= 0) *reinterpret_cast<uint4 *>(out + (size_t)row * n_out + fbase + 8 * c) = v;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t *>(&v);
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

__device__ __forceinline__ void raise_abort(volatile int *abort, uint32_t *status) {
    *abort = 1;
    atomicOr(status, MOE_DEV_GEMM_TIMEOUT);
}

// GATHER (mode 0 only): tmB maps the tokens x [T, H] with one-row boxes and
// the token-tile producer gathers each unit's rows x[src_token[row]] with
// tile::gather4 loads, so the permuted copy x_perm is never materialised.
template <int MODE, bool GATHER = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ RowMaps tmB, GemmArgs a) {
    static_assert(!GATHER || MODE == 0, "the row gather feeds the SwiGLU GEMM");
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
    int total, trows;
    int num_fb = a.num_fb, fbw = MODE == 0 ? 128 : 256;
    if (MODE == 2) {
        total = (a.T + a.route_rows - 1) / a.route_rows * a.route_q;
        trows = a.route_rows;
    } else {
        const int ntiles = *a.num_tiles;
        const int nt = ntiles < a.max_tiles ? ntiles : a.max_tiles;
        // Down projection with few row tiles: 128-feature units, twice as many,
        // when they still fit one wave (otherwise 256-feature units, which read
        // each token tile once for two accumulators).
        if (MODE == 1 && nt * a.num_fb * 2 <= (int)gridDim.x) {
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
    if ((int)blockIdx.x >= total || (int)blockIdx.x >= stride) return;  // uniform: this CTA has no work
    // Two rings: weight stages (the A tiles of both accumulators; mode 2:
    // three weight planes per accumulator), streamed from HBM, and token
    // stages of trows rows (multiple of 16, <= 256).  Four token stages
    // while that leaves at least four weight stages, else three; the weight
    // ring takes the rest, so that as many weight bytes as possible are in
    // flight.  Mode 2 reads both operands from L2 and consumes one stage of
    // each per K block: equally deep rings.
    trows = trows < 16 ? 16 : (trows > kTileRows ? kTileRows : (trows + 15) & ~15);
    const uint32_t a_tiles = MODE == 2 ? 3u * (a.E > 128 ? 2u : 1u) : 2u;
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
    const int nk = a.K / kBK;

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
                    const int kx = kb * kBK;
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
                    const int ky = krow + kb * kBK, kx = kb * kBK;
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
                const uint32_t idesc = idesc_bf16_f32(128, U.N, 1, 0);
                uint32_t h;
                bool big;
                plan.place(MODE == 2 ? 256 : U.N, h, big);  // mode 2 uses all of tensor memory
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
            uint32_t h;
            bool big;
            plan.place(MODE == 2 ? 256 : U.N, h, big);
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
                // Two accumulators of up to 256 columns do not fit in
                // registers: store while holding the accumulator.
                for (int c0 = sub * 16; c0 < U.N; c0 += 16 * kEpiSub) {
                    uint32_t r0[16], r1[16];
                    tmem_ld_frag16(t0 + (uint32_t)c0, r0);
                    if (U.nacc == 2) tmem_ld_frag16(t1 + (uint32_t)c0, r1);
                    tmem_ld_wait();
                    uint32_t w[8];
#pragma unroll
                    for (int m = 0; m < 8; ++m) w[m] = pack_bf16x2(r0[2 * m], r0[2 * m + 1]);
                    store_block_frag(w, stg, a.out, a.n_out, U.fx + q * 32, U, c0);
                    if (U.nacc == 2) {
#pragma unroll
                        for (int m = 0; m < 8; ++m) w[m] = pack_bf16x2(r1[2 * m], r1[2 * m + 1]);
                        store_block_frag(w, stg, a.out, a.n_out, U.fx + 128 + q * 32, U, c0);
                    }
                }
                release();
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
                    tmem_ld_frag16(t0 + (uint32_t)c0, r0);
                    if (U.nacc == 2) tmem_ld_frag16(t1 + (uint32_t)c0, r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        if (MODE == 0) {
                            const float g0 = __uint_as_float(r0[j]), v0 = __uint_as_float(r1[j]);
                            const float g1 = __uint_as_float(r0[j + 1]), v1 = __uint_as_float(r1[j + 1]);
                            const __nv_bfloat162 p = __floats2bfloat162_rn(__fdividef(g0, 1.0f + __expf(-g0)) * v0,
                                                                           __fdividef(g1, 1.0f + __expf(-g1)) * v1);
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
                    store_block_frag(w, stg, a.out, a.n_out, U.fx + q * 32, U, c0);
                    if (MODE == 1 && U.nacc == 2) {
#pragma unroll
                        for (int m = 0; m < 8; ++m) w[m] = hold[i][8 + m];
                        store_block_frag(w, stg, a.out, a.n_out, U.fx + 128 + q * 32, U, c0);
                    }
                }
            }
            plan.advance(big, h);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Pairs of CTAs sharing one MMA (tcgen05 cta_group::2), modes 0 and 1.
// A cluster of two CTAs takes units (expert group, 256-feature block, row
// tile): CTA r of the pair holds the weights of features [256 fb + 128 r, +128)
// (the MMA's M = 256 is split by CTA) and rows [r N/2, (r+1) N/2) of the token
// tile (N split by CTA), so each CTA streams only half of every token tile.
// Both CTAs' copies complete on the leader's (rank 0) barriers, which count
// both halves' bytes; the leader alone issues the MMAs and multicasts their
// commits to both CTAs' stage and accumulator barriers; each CTA drains its
// own tensor memory (its 128 features for all N rows) and hands it back by
// arriving on the leader's barrier.  Mode 0 keeps gate and up for the CTA's
// 128 features (two accumulators); mode 1 one accumulator of up to 256
// columns, so its units always alternate between the tensor-memory halves.
// Selected by MOE_FLAG_GEMM_PAIRS.  Measured on B200 it is not faster than the
// single-CTA kernel for the shapes of this library's benchmarks (the
// weight-streaming shapes stream no faster per SM with the deeper weight ring
// it allows, and the down projection of a 128-unit layer loses half of its
// per-CTA rate), so it is off by default.
constexpr int kPairMaxAStages = 12;
constexpr int kPairMaxBStages = 8;

// Rows [row0, row0 + n) (n a multiple of 8, <= 128) of the token matrix into
// this CTA's shared memory from dst, completing on the leader's barrier;
// boxes of 128, 64, 32, 16 and 8 rows (RowMaps with heights 8 << i), largest
// first.
__device__ __forceinline__ void tma_load_rows_pair(uint8_t *dst, const RowMaps &rm, uint32_t boxes, uint32_t bar,
                                                   int kx, int row0, int n) {
#pragma unroll
    for (int i = kRowBoxes - 1; i >= 0; --i) {
        const int h = 8 << i;
        if (!((boxes >> i) & 1u)) continue;
        while (n >= h) {
            tma_load_2d_pair(dst, &rm.m[i], bar, kx, row0);
            dst += h * kBRowBytes;
            row0 += h;
            n -= h;
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) __cluster_dims__(2, 1, 1)
    k_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ RowMaps tmB, GemmArgs a) {
    static_assert(MODE == 0 || MODE == 1, "pairs run the expert GEMMs");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *ctrl = smem + kRingBytes;
    uint64_t *fullA = reinterpret_cast<uint64_t *>(ctrl);
    uint64_t *emptyA = fullA + kPairMaxAStages;
    uint64_t *fullB = emptyA + kPairMaxAStages;
    uint64_t *emptyB = fullB + kPairMaxBStages;
    uint64_t *tfull = emptyB + kPairMaxBStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_gts = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
    const int ntiles = *a.num_tiles;
    const int nt = ntiles < a.max_tiles ? ntiles : a.max_tiles;
    const int num_fb = (a.n_out + 255) / 256;
    const int total = nt * num_fb;
    if (pair >= total) return;  // uniform over the pair: neither CTA has work
    int trows = *a.tile_rows;
    trows = trows < 16 ? 16 : (trows > kTileRows ? kTileRows : (trows + 15) & ~15);
    const uint32_t a_tiles = MODE == 0 ? 2u : 1u;
    const uint32_t a_bytes = a_tiles * kATile, b_bytes = (uint32_t)(trows / 2) * kBRowBytes;
    // Both rings equally deep (a pipeline stage waits for its weight and its
    // token tile alike, and both can come from HBM), then the rest of shared
    // memory for more weight stages.
    int nb = (int)(kRingBytes / (a_bytes + b_bytes));
    nb = nb > kPairMaxBStages ? kPairMaxBStages : (nb < 2 ? 2 : nb);
    int fit = (int)((kRingBytes - (uint32_t)nb * b_bytes) / a_bytes);
    const int na = fit > kPairMaxAStages ? kPairMaxAStages : fit;
    uint8_t *ringB = smem + (uint32_t)na * a_bytes;

    for (int i = threadIdx.x; i <= a.E; i += kThreads) s_gts[i] = a.grp_tile_start[i];
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairMaxAStages; ++s) {
            mbar_init(&fullA[s], 1);
            mbar_init(&emptyA[s], 1);
        }
        for (int s = 0; s < kPairMaxBStages; ++s) {
            mbar_init(&fullB[s], 1);
            mbar_init(&emptyB[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kEpiWarps);  // both CTAs' epilogue warps (the leader's count)
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
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_arrive_wait();  // both CTAs' barriers are initialised before any remote use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nk = a.K / kBK;

    if (warp == 0 || warp == 2) {
        // ------------- TMA producers (both CTAs): warp 0 weights, warp 2 token rows ----
        if (lane == 0) {
            const bool is_a = warp == 0;
            const int nst = is_a ? na : nb;
            uint64_t *full = is_a ? fullA : fullB;
            uint64_t *empty = is_a ? emptyA : emptyB;
            const uint32_t full_leader = mapa_shared(full, 0);  // the leader's barrier array
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = pair; u < total && ok; u += npairs) {
                Unit U;
                decode_unit<MODE>(u, s_gts, a, trows, num_fb, 256, U);
                if (!U.valid) {
                    if (is_a && leader) atomicOr(a.status, MOE_DEV_BAD_ROW);
                    continue;
                }
                const int fx = U.fx + 128 * (int)rank;  // this CTA's first feature
                const int half_rows = U.N / 2;          // rows of the token tile this CTA holds
                const uint32_t my_bytes = is_a ? a_tiles * kATile : (uint32_t)half_rows * kBRowBytes;
                const int krow = U.e * a.K;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], ph ^ 1u, a.timeout_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    // the leader expects both CTAs' bytes of this stage
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2u * my_bytes);
                    const uint32_t bar = full_leader + 8u * (uint32_t)stage;
                    const int ky = krow + kb * kBK, kx = kb * kBK;
                    if (is_a) {
                        uint8_t *sa0 = smem + stage * a_bytes;
                        tma_load_2d_pair(sa0, &tmA0, bar, fx, ky);
                        tma_load_2d_pair(sa0 + kABox, &tmA0, bar, fx + 64, ky);
                        if (MODE == 0) {
                            tma_load_2d_pair(sa0 + kATile, &tmA1, bar, fx, ky);
                            tma_load_2d_pair(sa0 + kATile + kABox, &tmA1, bar, fx + 64, ky);
                        }
                    } else {
                        // tile rows [rank * N/2, (rank + 1) * N/2): the part in
                        // row piece 0 (tile rows [0, n0p)), then the part in
                        // piece 1 (all lengths multiples of 8)
                        uint8_t *sb = ringB + stage * b_bytes;
                        const int cb = (int)rank * half_rows, ce = cb + half_rows;
                        const int l0 = max(0, min(ce, U.n0p) - cb);
                        const int c1 = max(cb, U.n0p);
                        if (l0) tma_load_rows_pair(sb, tmB, a.row_boxes, bar, kx, U.p0s + cb, l0);
                        if (ce > c1) tma_load_rows_pair(sb + l0 * kBRowBytes, tmB, a.row_boxes, bar, kx,
                                                        U.p1s + (c1 - U.n0p), ce - c1);
                    }
                    if (++stage == nst) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok && !*s_abort) raise_abort(s_abort, a.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------- MMA issuer (the leader only) ----
        if (lane == 0 && leader) {
            int sa = 0, sb = 0;
            uint32_t pha = 0, phb = 0;
            TmemPlan plan;
            const uint32_t baseA = smem_u32(smem), baseB = smem_u32(ringB);
            bool ok = true;
            for (int u = pair; u < total && ok; u += npairs) {
                Unit U;
                decode_unit<MODE>(u, s_gts, a, trows, num_fb, 256, U);
                if (!U.valid) continue;
                const uint32_t idesc = idesc_bf16_f32(256, U.N, 1, 0);
                uint32_t h;
                bool big;
                plan.place(MODE == 0 ? U.N : 0, h, big);  // mode 1: one accumulator fits a half
                const uint32_t d0 = tmem + h * 256u, d1 = big ? tmem + 256u : d0 + 128u;
                ok = mbar_wait_bounded(&tempty[h], (plan.uses[h] & 1u) ^ 1u, a.timeout_ns, s_abort);
                if (ok && big) ok = mbar_wait_bounded(&tempty[1], (plan.uses[1] & 1u) ^ 1u, a.timeout_ns, s_abort);
                if (!ok) break;
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(&fullA[sa], pha, a.timeout_ns, s_abort) ||
                        !mbar_wait_bounded(&fullB[sb], phb, a.timeout_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa0 = baseA + sa * a_bytes, sa1 = sa0 + kATile, sbt = baseB + sb * b_bytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = sdesc_sw128(sbt + kk * 32, 16, 1024);
                        const uint32_t accum = (kb | kk) ? 1u : 0u;
                        tc_mma_bf16_pair(d0, sdesc_sw128(sa0 + kk * 2048, kABox, 1024), bdesc, idesc, accum);
                        if (MODE == 0)
                            tc_mma_bf16_pair(d1, sdesc_sw128(sa1 + kk * 2048, kABox, 1024), bdesc, idesc, accum);
                    }
                    tc_commit_pair(&emptyA[sa], 3);  // both CTAs' stages are free once read
                    tc_commit_pair(&emptyB[sb], 3);
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
                tc_commit_pair(&tfull[h], 3);
                if (big) tc_commit_pair(&tfull[1], 3);
                plan.advance(big, h);
            }
            if (!ok && !*s_abort) raise_abort(s_abort, a.status);
            int never = 0;
            tc_commit_pair(mma_done, 1);
            mbar_wait_bounded(mma_done, 0, a.timeout_ns, &never);
        }
        __syncwarp();
    } else {
        // -------------------------------------------- epilogue (both CTAs) ----
        const int q = warp & 3;
        const int sub = (warp - kEpiWarp0) >> 2;
        const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
        const uint32_t tempty_leader = mapa_shared(tempty, 0);
        TmemPlan plan;
        for (int u = pair; u < total; u += npairs) {
            Unit U;
            decode_unit<MODE>(u, s_gts, a, trows, num_fb, 256, U);
            if (!U.valid) continue;
            uint32_t h;
            bool big;
            plan.place(MODE == 0 ? U.N : 0, h, big);
            bool got = mbar_wait_bounded(&tfull[h], plan.uses[h] & 1u, a.timeout_ns, s_abort);
            if (got && big) got = mbar_wait_bounded(&tfull[1], plan.uses[1] & 1u, a.timeout_ns, s_abort);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0 && !*s_abort) raise_abort(s_abort, a.status);
                break;
            }
            tc_fence_after();
            const uint32_t t0 = tq + h * 256u, t1 = big ? tq + 256u : t0 + 128u;
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_cluster(tempty_leader + 8u * h);
                    if (big) mbar_arrive_cluster(tempty_leader + 8u);
                }
            };
            const int fb0 = U.fx + 128 * (int)rank + q * 32;  // this warp's first feature
            const bool inside = fb0 < a.n_out;  // the last block may have no second half (warp-uniform)
            if (MODE == 1) {
                // one accumulator of up to 256 columns: hold up to 4 chunks per warp
                constexpr int kChunks = (16 + kEpiSub - 1) / kEpiSub;
                uint32_t hold[kChunks][8];
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) {
                        uint32_t r0[16];
                        tmem_ld16(t0 + (uint32_t)c0, r0);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            const __nv_bfloat162 pk =
                                __floats2bfloat162_rn(__uint_as_float(r0[j]), __uint_as_float(r0[j + 1]));
                            hold[i][j / 2] = *reinterpret_cast<const uint32_t *>(&pk);
                        }
                    }
                }
                release();
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N && inside) store_block_32x16(hold[i], a.out, a.n_out, fb0, U, c0);
                }
            } else {
                constexpr int kChunks = (16 + kEpiSub - 1) / kEpiSub;
                uint32_t hold[kChunks][8];
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N) {
                        uint32_t r0[16], r1[16];
                        tmem_ld16(t0 + (uint32_t)c0, r0);
                        tmem_ld16(t1 + (uint32_t)c0, r1);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            const float g0 = __uint_as_float(r0[j]), v0 = __uint_as_float(r1[j]);
                            const float g1 = __uint_as_float(r0[j + 1]), v1 = __uint_as_float(r1[j + 1]);
                            const __nv_bfloat162 pk = __floats2bfloat162_rn(__fdividef(g0, 1.0f + __expf(-g0)) * v0,
                                                                            __fdividef(g1, 1.0f + __expf(-g1)) * v1);
                            hold[i][j / 2] = *reinterpret_cast<const uint32_t *>(&pk);
                        }
                    }
                }
                release();
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    const int c0 = (sub + kEpiSub * i) * 16;
                    if (c0 < U.N && inside) store_block_32x16(hold[i], a.out, a.n_out, fb0, U, c0);
                }
            }
            plan.advance(big, h);
        }
    }

    // Neither CTA leaves (or frees tensor memory) while the other may still
    // read its shared memory, write its tensor memory or signal its barriers.
    tc_fence_before();
    __syncthreads();
    cluster_arrive_wait();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// Exact three-way bf16 split of the router weights: p0 = bf16(w),
// p1 = bf16(w - p0), p2 = bf16(w - p0 - p1) (each difference is exact in
// fp32), written as planes[3][H][Ep]; columns e >= E are zero.
__global__ void __launch_bounds__(256) k_router_planes(const float *__restrict__ w, __nv_bfloat16 *__restrict__ planes,
                                                       int H, int E, int Ep) {
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

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with the 128-byte
// swizzle; box = box_cols x box_rows (box_cols * 2 bytes must be 128).
bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The token matrix with boxes of 16, 32, ... 256 rows; returns the mask of the
// maps that could be encoded (bit 0 is required).
uint32_t make_row_maps(RowMaps *rm, const void *ptr, uint64_t rows, uint64_t cols, uint32_t min_rows = 16) {
    uint32_t boxes = 0;
    for (int i = 0; i < kRowBoxes; ++i)
        if (make_tmap(&rm->m[i], ptr, rows, cols, 64, min_rows << i)) boxes |= 1u << i;
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
    k_grouped_gemm<2><<<num_sms, kThreads, kSmemBytes, stream>>>(tA, tA, tB, a);
    return cudaGetLastError();
}

// mode 0: act = x_perm [P,H], w0 = gate, w1 = up, out = h [P,F]
//         (with src_token: act = x [T,H], rows gathered as x[src_token[row]])
// mode 1: act = h [P,F],      w0 = w1 = down,   out = y [P,H]
cudaError_t launch_grouped_gemm(int mode, const moe_shape &s, const void *act, const void *w0, const void *w1,
                                void *out, const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                cudaStream_t stream, const int32_t *src_token) {
    const bool gather = mode == 0 && src_token != nullptr;
    // Pairs of CTAs sharing one MMA for the expert GEMMs, on request (not for
    // the row gather).
    const bool pairs = (s.flags & MOE_FLAG_GEMM_PAIRS) && !gather && num_sms >= 2;
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
    } else if (pairs) {
        if (!(boxes = make_row_maps(&tB, act, (uint64_t)P, (uint64_t)K, 8))) return cudaErrorInvalidValue;
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
    static bool attr_done[5] = {false, false, false, false, false};
    cudaError_t err;
    if (pairs) {
        const int grid = num_sms & ~1;
        if (mode == 0) {
            if (!attr_done[3]) {
                err = cudaFuncSetAttribute(k_grouped_gemm_pair<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
                if (err != cudaSuccess) return err;
                attr_done[3] = true;
            }
            k_grouped_gemm_pair<0><<<grid, kThreads, kSmemBytes, stream>>>(tA0, tA1, tB, a);
        } else {
            if (!attr_done[4]) {
                err = cudaFuncSetAttribute(k_grouped_gemm_pair<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
                if (err != cudaSuccess) return err;
                attr_done[4] = true;
            }
            k_grouped_gemm_pair<1><<<grid, kThreads, kSmemBytes, stream>>>(tA0, tA1, tB, a);
        }
    } else if (gather) {
        if (!attr_done[2]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[2] = true;
        }
        k_grouped_gemm<0, true><<<num_sms, kThreads, kSmemBytes, stream>>>(tA0, tA1, tB, a);
    } else if (mode == 0) {
        if (!attr_done[0]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[0] = true;
        }
        k_grouped_gemm<0><<<num_sms, kThreads, kSmemBytes, stream>>>(tA0, tA1, tB, a);
    } else {
        if (!attr_done[1]) {
            err = cudaFuncSetAttribute(k_grouped_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[1] = true;
        }
        k_grouped_gemm<1><<<num_sms, kThreads, kSmemBytes, stream>>>(tA0, tA1, tB, a);
    }
    return cudaGetLastError();
}

}  // namespace moe
