/*
 * moe.h - C ABI of the B200 (sm_100a) MoE-layer forward dispatch library.
 *
 * The library computes, on one GPU, the five-step forward path of a
 * Mixture-of-Experts layer described on the "TritonMoE" verdict page
 * (pith.science, arXiv 2605.23911; referee report summary and pith summary):
 * router scoring, permutation of the routed tokens onto experts, the grouped
 * expert GEMMs (a fused gate+up SwiGLU projection, then the down projection)
 * and a weighted unpermutation.  The optional capacity layout follows the
 * "Cap-and-Spill" critique page (juhe.plus), section "Cap-and-Spill": C slots
 * per expert plus a compacted overflow buffer sized for the largest possible
 * overflow, so no routed token is ever dropped.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Ownership: the CALLER allocates and owns every buffer (inputs, outputs,
 *   intermediates and the workspace `ws`).  The library never allocates,
 *   frees or synchronises, except moe_read_status, which synchronises.
 * - Memory: every data pointer is a DEVICE pointer on the current CUDA
 *   device; bf16 tensors and w_router are 16-byte aligned, int32/fp32
 *   vectors 4-byte aligned, `ws` 256-byte aligned.  bf16 tensors are
 *   passed as `void *` holding IEEE bfloat16 values.  All matrices are dense
 *   and row-major with the leading dimension equal to the row length.
 * - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  Each
 *   call only enqueues work on it and returns; every call other than
 *   moe_read_status and moe_permute_static is stream-ordered, performs no
 *   host synchronisation and may be captured in a CUDA graph (this header
 *   states nothing about graphs for moe_permute_static, whose section below
 *   gives its own rules).  Grid sizes depend only on the shape and the SM count,
 *   never on the routing, so a captured graph stays valid for any input
 *   values of the same shape.
 * - Errors: a bad argument or an unsupported shape returns a non-zero
 *   moe_status before anything is enqueued.  A failed launch returns
 *   MOE_ERR_CUDA.  Faults found on the device (a bounded wait that expired,
 *   an expert index out of range) are OR-ed into a sticky status word in
 *   `ws`; read it with moe_read_status.  No kernel traps.
 * - Workspace: size it with moe_workspace_bytes and zero it once after
 *   allocating it (moe_workspace_init, or a plain memset); afterwards every
 *   call keeps it consistent by itself.
 * - Workspace coupling: moe_permute leaves the per-expert offsets and the
 *   tile schedule of the grouped GEMMs in `ws`; moe_grouped_swiglu and
 *   moe_grouped_down read them.  A workspace must not be used by two
 *   streams at once.
 *
 * Supported shapes: T >= 1, H and F multiples of 128, 1 <= E <= 256,
 * 1 <= k <= E, C >= 0, and the permuted row count below 2^31.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,       /* null/misaligned pointer, bad flag */
    MOE_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the supported set above */
    MOE_ERR_WORKSPACE = 3,         /* workspace pointer unusable */
    MOE_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
    MOE_ERR_DEVICE = 5             /* current device is not sm_100 */
} moe_status;

/* Bits of the device status word (sticky until cleared by moe_read_status). */
#define MOE_DEV_SCAN_TIMEOUT 0x1u  /* histogram look-back wait expired */
#define MOE_DEV_GEMM_TIMEOUT 0x2u  /* a grouped-GEMM pipeline wait expired */
#define MOE_DEV_BAD_EXPERT 0x4u    /* a routed expert index was outside [0, E) */
#define MOE_DEV_NAN_LOGIT 0x8u     /* warning: a router logit was NaN */
#define MOE_DEV_BAD_ROW 0x10u      /* a row index fell outside its buffer and the
                                      access was skipped (follows another error) */

/* moe_shape.flags */
#define MOE_FLAG_CAPACITY 0x1u  /* capacity layout: C slots per expert + overflow */
#define MOE_FLAG_LOGITS_IN 0x2u /* moe_route/moe_forward read the caller's fp32
                                   logits instead of computing x * W_r + bias */
#define MOE_FLAG_FUSED_COMBINE 0x8u /* moe_forward / moe_forward_fp8 run the
                                   combine of step 5 inside the down GEMM
                                   (moe_grouped_down_combine): same out, bit
                                   for bit, and y is still written */
#define MOE_FLAG_TEST_STALL_SCAN 0x40000000u /* test only: the first histogram
                                   block never publishes, so its successor's
                                   bounded wait expires and reports
                                   MOE_DEV_SCAN_TIMEOUT */
#define MOE_FLAG_TEST_STALL_GEMM 0x20000000u /* test only: in moe_grouped_swiglu
                                   (tiled form) the token-tile producer of
                                   CTA 0 never loads its first stage, so the
                                   MMA issuer's bounded wait expires; the
                                   kernel reports MOE_DEV_GEMM_TIMEOUT, lets
                                   its copies in flight land, frees its
                                   tensor memory and returns */

typedef struct {
    int32_t T;      /* tokens */
    int32_t H;      /* hidden size */
    int32_t F;      /* expert FFN size */
    int32_t E;      /* experts */
    int32_t k;      /* experts per token */
    int32_t C;      /* capacity slots per expert (used with MOE_FLAG_CAPACITY) */
    uint32_t flags; /* MOE_FLAG_* */
} moe_shape;

/* Every pointer argument of the whole layer, for moe_forward. */
typedef struct {
    const void *x;         /* [T,H]   bf16 tokens */
    const float *w_router; /* [H,E]   fp32 router weights (unused with LOGITS_IN) */
    const float *bias;     /* [E]     fp32 additive logit bias, or NULL */
    const void *w_gate;    /* [E,H,F] bf16 */
    const void *w_up;      /* [E,H,F] bf16 */
    const void *w_down;    /* [E,F,H] bf16 */
    float *logits;         /* [T,E]   fp32 (input with LOGITS_IN, else output; may be NULL without LOGITS_IN) */
    int32_t *topk_idx;     /* [T,k]   expert ids in rank order */
    float *topk_w;         /* [T,k]   gate weights */
    int32_t *expert_counts;  /* [E]   routed pairs per expert */
    int32_t *expert_offsets; /* [E+1] exclusive prefix sum of expert_counts */
    int32_t *src_token;    /* [P]     token of each permuted row, -1 = empty slot */
    int32_t *dest_row;     /* [T*k]   permuted row of each routed pair */
    void *x_perm;          /* [P,H]   bf16 permuted tokens, or NULL: not produced (see moe_forward) */
    void *h;               /* [P,F]   bf16 SwiGLU activations */
    void *y;               /* [P,H]   bf16 expert outputs */
    void *out;             /* [T,H]   bf16 layer output */
} moe_forward_args;

/* Byte offsets of the workspace sections a caller may inspect (tests do). */
typedef struct {
    size_t total;          /* bytes the workspace must hold */
    size_t status;         /* uint32 sticky device status word */
    size_t num_tiles;      /* int32 number of GEMM row tiles */
    size_t total_spill;    /* int32 rows used in the overflow region */
    size_t cap_cnt;        /* int32[E] min(n_e, C) (n_e when uncapped) */
    size_t spill_cnt;      /* int32[E] n_e - cap_cnt[e] */
    size_t spill_off;      /* int32[E+1] exclusive prefix sum of spill_cnt */
    size_t order;          /* int32[E] experts by descending count, ties by index */
    size_t grp_tile_start; /* int32[E+1] first tile of the g-th expert of `order` */
    size_t tile_map;       /* int32[4*max_tiles] tiles: {e, row0, len0 | len1<<16, row1} */
    int32_t max_tiles;     /* capacity of tile_map */
    int32_t tile_rows;     /* largest number of rows any tile can hold (256) */
    size_t row_cap;        /* int32 row cap of the last schedule's tiles (<= tile_rows):
                              the largest padded row count of one expert */
} moe_ws_layout;

/* Rows of the permuted buffers x_perm, h, y: T*k uncapped; with the capacity
 * layout E*C + k*max(0, T-C) (the overflow is at most k*(T-C): it is largest
 * when k experts take every token).  Returns -1 for an unsupported shape. */
MOE_API int64_t moe_permuted_rows(const moe_shape *shape);

/* Workspace bytes for `shape`, or 0 for an unsupported shape. */
MOE_API size_t moe_workspace_bytes(const moe_shape *shape);

/* Fills `layout` for `shape`; MOE_ERR_UNSUPPORTED_SHAPE if unsupported. */
MOE_API moe_status moe_workspace_layout(const moe_shape *shape, moe_ws_layout *layout);

/* Zero-fills `ws` (moe_workspace_bytes(shape) bytes) on `stream`.  Needed
 * once per newly allocated workspace; clears the sticky status word too. */
MOE_API moe_status moe_workspace_init(const moe_shape *shape, void *ws, void *stream);

/* Step 1, router scoring ("TritonMoE" verdict page, referee report summary):
 *   logits[t,e] = fp32(sum_h x[t,h] * w_router[h,e]) + bias[e]
 *   topk_idx[t,:] = the k experts of largest logit, in rank order, equal
 *                   logits to the lower index, NaN below every number;
 *   topk_w[t,j]   = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k selected.
 * With MOE_FLAG_LOGITS_IN, `logits` is read (w_router, bias unused).
 * Otherwise `logits` may be NULL (not written).  From 2048 tokens the dot
 * products run on the tensor cores against an exact three-way bf16 split of
 * w_router, summed over at least eight fp32 partial accumulations in a fixed
 * order (within 1e-5 relative of the fp32 definition; deterministic); the
 * workspace then also holds the split weights and the partial logits. */
MOE_API moe_status moe_route(const moe_shape *shape, const void *x, const float *w_router, const float *bias, float *logits,
                     int32_t *topk_idx, float *topk_w, void *ws, void *stream);

/* Steps 2-3, histogram + exclusive scan + stable permutation ("TritonMoE"
 * verdict page: tokens reordered onto experts; "Cap-and-Spill" page for the
 * capacity layout):
 *   expert_counts[e]  = #{(t,j): topk_idx[t,j] == e}
 *   expert_offsets    = exclusive prefix sum of expert_counts
 *   the r-th pair of expert e in flat order t*k+j goes to row
 *     uncapped:  expert_offsets[e] + r
 *     capacity:  r < C ? e*C + r : E*C + spill_off[e] + (r - C)
 *   dest_row[t*k+j] = its row; src_token[row] = t (-1 for an unfilled row);
 *   x_perm[row] = x[src_token[row]] (zeros for unfilled capacity slots).
 * Also leaves the grouped-GEMM tile schedule in `ws`. */
MOE_API moe_status moe_permute(const moe_shape *shape, const void *x, const int32_t *topk_idx, int32_t *expert_counts,
                       int32_t *expert_offsets, int32_t *src_token, int32_t *dest_row, void *x_perm, void *ws,
                       void *stream);

/* Steps 1-3 without the row copy: moe_route, then the index part of
 * moe_permute (expert_counts, expert_offsets, src_token, dest_row and the
 * tile schedule in `ws`; x_perm is not written), with the same arguments,
 * checks and results as those two calls.  For up to 4096 routed pairs
 * (T*k <= 4096) the router's last CTA builds the dispatch in its shared
 * memory (one kernel after a memset instead of three); above that the
 * histogram and rank kernels of moe_permute run. */
MOE_API moe_status moe_route_dispatch(const moe_shape *shape, const void *x, const float *w_router, const float *bias,
                                      float *logits, int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                                      int32_t *expert_offsets, int32_t *src_token, int32_t *dest_row, void *ws,
                                      void *stream);

/* The row copy of step 3: x_perm[row] = x[src_token[row]] for every permuted
 * row (zeros where src_token is -1), as moe_permute writes it; reads the
 * overflow size moe_permute / moe_route_dispatch left in `ws`. */
MOE_API moe_status moe_gather(const moe_shape *shape, const void *x, const int32_t *src_token, void *x_perm, void *ws,
                              void *stream);

/* Step 4a, fused gate+up SwiGLU over every filled permuted row r of expert e
 * ("TritonMoE" verdict page, pith extraction key machinery):
 *   h[r,f] = bf16( silu(x_perm[r] . w_gate[e][:,f]) * (x_perm[r] . w_up[e][:,f]) ),
 *   silu(z) = z / (1 + exp(-z)), fp32 accumulation.  Rows not filled are
 *   left unwritten.  Reads the tile schedule moe_permute left in `ws`. */
MOE_API moe_status moe_grouped_swiglu(const moe_shape *shape, const void *x_perm, const void *w_gate, const void *w_up,
                              void *h, void *ws, void *stream);

/* Step 4a with the row copy of step 3 folded in: the same h as
 * moe_grouped_swiglu on x_perm, reading each permuted row r straight from
 * x[src_token[r]] (TMA gather of four token rows per load), so x_perm is
 * neither written nor read.  It saves the row copy and the P x H buffer;
 * the gathers move fewer bytes per cycle than whole tiles, so with many rows
 * per expert (more than about 32 on average) moe_gather + moe_grouped_swiglu
 * is faster.  src_token as moe_permute / moe_route_dispatch
 * leave it; a row outside [0, T) is read as token 0 and reported as
 * MOE_DEV_BAD_ROW. */
MOE_API moe_status moe_grouped_swiglu_gather(const moe_shape *shape, const void *x, const int32_t *src_token,
                                             const void *w_gate, const void *w_up, void *h, void *ws, void *stream);

/* Step 4b, down projection ("TritonMoE" verdict page, desk editor letter):
 *   y[r,c] = bf16( h[r] . w_down[e][:,c] ), fp32 accumulation. */
MOE_API moe_status moe_grouped_down(const moe_shape *shape, const void *h, const void *w_down, void *y, void *ws,
                            void *stream);

/* Steps 4b and 5 in one kernel: the down projection of moe_grouped_down
 * (y is written as there), and, in its epilogue, the weighted combine of
 * moe_combine.  The "TritonMoE" verdict page (desk editor letter) notes that
 * its fused kernel stops before the down projection; here the combine follows
 * the down projection's stores without another launch: after a warp has
 * stored its piece of a unit's rows it counts one arrival per (token,
 * 128-feature block) in the workspace, and the warp whose arrival completes a
 * token's block (all k of its rows stored) combines that block, in slot
 * order, with exactly moe_combine's arithmetic: `out` is bit-identical to
 * moe_combine's on the same y.  The counts start at zero after
 * moe_workspace_init and every complete call leaves them at zero; after a
 * device-side fault (status word non-zero) re-initialise the workspace.
 * src_token and dest_row as moe_permute / moe_route_dispatch leave them. */
MOE_API moe_status moe_grouped_down_combine(const moe_shape *shape, const void *h, const void *w_down,
                                            const int32_t *src_token, const int32_t *dest_row, const float *topk_w,
                                            void *y, void *out, void *ws, void *stream);

/* Step 5, weighted unpermutation ("TritonMoE" verdict page, referee report
 * summary):  out[t] = bf16( sum_j topk_w[t,j] * y[dest_row[t*k+j]] ), the
 * sum in fp32 in slot order j, products and sums rounded separately. */
MOE_API moe_status moe_combine(const moe_shape *shape, const void *y, const int32_t *dest_row, const float *topk_w, void *out,
                       void *stream);

/* The five steps in order on one stream (no host sync; graph-capturable):
 * moe_route_dispatch, moe_gather, moe_grouped_swiglu, moe_grouped_down,
 * moe_combine (with MOE_FLAG_FUSED_COMBINE: moe_grouped_down_combine in place
 * of the last two).  With args->x_perm == NULL the row copy is folded into the
 * SwiGLU GEMM (moe_grouped_swiglu_gather) and x_perm is not produced: the
 * faster choice for decode-sized batches (about 32 or fewer routed rows per
 * expert), the slower one for large batches. */
MOE_API moe_status moe_forward(const moe_shape *shape, const moe_forward_args *args, void *ws, void *stream);

/* Synchronises `stream`, copies the sticky device status word of `ws` to
 * *device_status and, if clear != 0, resets it.  Not graph-capturable. */
MOE_API moe_status moe_read_status(void *ws, void *stream, uint32_t *device_status, int clear);

/* Dispatch for callers that cannot allocate device memory.  (This entry
 * point has no counterpart on the source pages; it is an interface
 * convenience.)  Some callers cannot call cudaMalloc: a plug-in whose host
 * application owns every device allocation, for instance, and hands it only
 * the tensors it works on.  moe_permute_static computes exactly what moe_permute computes
 * (same arguments, minus `ws`) but takes its scratch from an array of
 * MOE_STATIC_WS_BYTES bytes compiled into the library, which every GPU that
 * loads the library holds until the process exits.
 *   - It allocates nothing and calls no allocating routine.
 *   - Shapes whose dispatch scratch exceeds MOE_STATIC_WS_BYTES are rejected
 *     with MOE_ERR_WORKSPACE (see moe_last_error_string).  The dispatch
 *     scratch is moe_workspace_bytes without the router buffers that large
 *     batches add (it grows with T*k/1024 and E).
 *   - The first call on each device (with that device current) looks up the
 *     array's device address and zero-fills it on `stream`.  (A context that
 *     was torn down and recreated gets the same set-up again on its first
 *     call.)
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears what must start at zero.  Calls that overlap on the GPU
 *     (other streams, other host threads) race on the array: order them.
 *   - The GEMM schedule it builds stays inside the array, so the grouped GEMM
 *     entry points still need the workspace form (moe_permute).
 *   - Device-side faults cannot be reported: there is no caller workspace to
 *     hold the status word.  After one (an expert index outside [0, E), an
 *     expired look-back wait) the outputs are undefined; a pair that cannot
 *     be placed gets dest_row = -1.  MOE_FLAG_TEST_STALL_SCAN is refused
 *     with MOE_ERR_INVALID_ARG. */
#define MOE_STATIC_WS_BYTES (1u << 20)
MOE_API moe_status moe_permute_static(const moe_shape *shape, const void *x, const int32_t *topk_idx,
                                      int32_t *expert_counts, int32_t *expert_offsets, int32_t *src_token,
                                      int32_t *dest_row, void *x_perm, void *stream);

/* ------------------------------------------------------------------------
 * fp8 (e4m3) expert GEMMs ("TEMPO" verdict page, pith.science, arXiv
 * 2608.13057, referee report summary: its per-expert cost law is measured on
 * an fp8 grouped GEMM, whose flat regime streams the expert's weights from
 * HBM; 8-bit weights halve those bytes).
 *
 * Format (the pages fix none; this is the plainest reading): OCP E4M3 codes
 * (uint8: sign, 4 exponent bits with bias 7, 3 mantissa bits, max 448) with
 * one power-of-two fp32 scale per vector, s = 2^(c - 8) for the smallest
 * integer c with max|v| <= 2^c (s = 1 for an all-zero vector); code = the
 * nearest e4m3 value of v / s, ties to even.  value = code * s, which is
 * exactly a bf16 value, so the fp8 layer is the bf16 layer applied to the
 * dequantized weights and activations.  Expert weights: one scale per expert
 * and output column, codes stored with the reduction dimension contiguous.
 * Activations: one scale per row.  The GEMMs multiply products of codes on
 * the tensor cores (tcgen05 kind::f8f6f4, fp32 accumulation) and apply the
 * row and column scales in the epilogue; h and y stay bf16, the combine is
 * the bf16 one.
 * Weight codes are tile-blocked: for N output columns and reduction length K
 * (gate/up: N = F, K = H; down: N = H, K = F), the code of expert e, column n,
 * index k is byte ((e*(N/128) + n/128)*(K/128) + k/128)*16384 + (n%128)*128 +
 * k%128 -- tiles of 128 columns x 128 K, each 16 KB contiguous and K-major
 * inside, so each load of the GEMMs streams one contiguous 16 KB tile.
 * ------------------------------------------------------------------------ */
#define MOE_WEIGHTS_GATE_UP 0 /* w [E,H,F] bf16 -> E*F*H codes (N = F, K = H), scales [E,F] */
#define MOE_WEIGHTS_DOWN 1    /* w [E,F,H] bf16 -> E*H*F codes (N = H, K = F), scales [E,H] */
#define MOE_ROWS_X_PERM 0     /* codes [P,H] of x[src_token[r]] (the row copy of step 3; zero codes
                                 with scale 1 where src_token is -1), scales [P] */
#define MOE_ROWS_TOKENS 1     /* codes [T,H] of every token row of x, scales [T] */
#define MOE_ROWS_H 2          /* codes [P,F] of h[r] for every filled row r (src_token[r] >= 0; the
                                 other rows are left unwritten; src_token null: every row), scales [P] */

/* One-time preparation of expert weights: `which` = MOE_WEIGHTS_GATE_UP (w is
 * w_gate or w_up, [E,H,F]) or MOE_WEIGHTS_DOWN (w is w_down, [E,F,H]).
 * w_q: 16-byte aligned device buffer of E*H*F bytes; w_scale: E*F (gate/up)
 * or E*H (down) floats. */
MOE_API moe_status moe_quantize_weights_fp8(const moe_shape *shape, int which, const void *w, void *w_q,
                                            float *w_scale, void *stream);

/* Row quantization (see MOE_ROWS_*): `src` is x ([T,H] bf16) for X_PERM and
 * TOKENS, h ([P,F] bf16) for H; src_token as moe_permute / moe_route_dispatch
 * leave it (unused for TOKENS).  X_PERM and H read the overflow size from
 * `ws`. */
MOE_API moe_status moe_quantize_rows_fp8(const moe_shape *shape, int which, const void *src, const int32_t *src_token,
                                         void *q, float *scale, void *ws, void *stream);

/* Step 4a on fp8 operands: the same h as moe_grouped_swiglu on the
 * dequantized operands (up to fp32 summation order):
 *   h[r,f] = bf16( silu(g) * u ),  g = sx[r] * swg[e,f] * sum_k xq[r,k] * wgq[e,f,k]
 * (u likewise with the up weights).  With src_token == NULL, x_q / x_scale
 * hold the permuted rows ([P,H] codes, [P] scales: MOE_ROWS_X_PERM);
 * otherwise they hold the token rows ([T,H], [T]: MOE_ROWS_TOKENS) and row r
 * is gathered from token src_token[r] (like moe_grouped_swiglu_gather). */
MOE_API moe_status moe_grouped_swiglu_fp8(const moe_shape *shape, const void *x_q, const float *x_scale,
                                          const int32_t *src_token, const void *wg_q, const float *wg_scale,
                                          const void *wu_q, const float *wu_scale, void *h, void *ws, void *stream);

/* Step 4b on fp8 operands: y[r,c] = bf16( sh[r] * swd[e,c] * sum_f hq[r,f] * wdq[e,c,f] ),
 * h_q / h_scale as MOE_ROWS_H writes them. */
MOE_API moe_status moe_grouped_down_fp8(const moe_shape *shape, const void *h_q, const float *h_scale,
                                        const void *wd_q, const float *wd_scale, void *y, void *ws, void *stream);

/* moe_grouped_down_fp8 with the combine of step 5 in its epilogue, as
 * moe_grouped_down_combine does for the bf16 projection. */
MOE_API moe_status moe_grouped_down_fp8_combine(const moe_shape *shape, const void *h_q, const float *h_scale,
                                                const void *wd_q, const float *wd_scale, const int32_t *src_token,
                                                const int32_t *dest_row, const float *topk_w, void *y, void *out,
                                                void *ws, void *stream);

/* Every pointer argument of the fp8 layer, for moe_forward_fp8. */
typedef struct {
    const void *x;           /* [T,H]   bf16 tokens */
    const float *w_router;   /* [H,E]   fp32 */
    const float *bias;       /* [E]     fp32, or NULL */
    const void *wg_q;        /* [E,F,H] e4m3 gate codes */
    const float *wg_scale;   /* [E,F] */
    const void *wu_q;        /* [E,F,H] e4m3 up codes */
    const float *wu_scale;   /* [E,F] */
    const void *wd_q;        /* [E,H,F] e4m3 down codes */
    const float *wd_scale;   /* [E,H] */
    float *logits;           /* [T,E]   as in moe_forward_args */
    int32_t *topk_idx;       /* [T,k] */
    float *topk_w;           /* [T,k] */
    int32_t *expert_counts;  /* [E] */
    int32_t *expert_offsets; /* [E+1] */
    int32_t *src_token;      /* [P] */
    int32_t *dest_row;       /* [T*k] */
    void *x_q;               /* [P,H] codes (x_q_per_token == 0) or [T,H] (== 1) */
    float *x_scale;          /* [P] or [T] */
    int32_t x_q_per_token;   /* 1: token rows gathered by the SwiGLU GEMM (no row copy) */
    void *h;                 /* [P,F]   bf16 */
    void *h_q;               /* [P,F]   e4m3 codes */
    float *h_scale;          /* [P] */
    void *y;                 /* [P,H]   bf16 */
    void *out;               /* [T,H]   bf16 layer output */
} moe_forward_fp8_args;

/* The fp8 layer on one stream (no host sync; graph-capturable):
 * moe_route_dispatch, moe_quantize_rows_fp8 (X_PERM, or TOKENS with
 * x_q_per_token), moe_grouped_swiglu_fp8, moe_quantize_rows_fp8 (H),
 * moe_grouped_down_fp8, moe_combine (with MOE_FLAG_FUSED_COMBINE:
 * moe_grouped_down_fp8_combine in place of the last two).  Weights must have been prepared with
 * moe_quantize_weights_fp8. */
MOE_API moe_status moe_forward_fp8(const moe_shape *shape, const moe_forward_fp8_args *args, void *ws, void *stream);

/* ------------------------------------------------------------------------
 * Expert-parallel Cap-and-Spill dispatch ("Cap-and-Spill" critique page,
 * juhe.plus, section "Cap-and-Spill": a capacity pass with C slots per
 * expert, then a pass for the compacted overflow, whose buffer is sized for
 * the largest possible overflow so that it exists before the routing is
 * known; no token is dropped and no host synchronisation sits between the
 * passes).
 *
 * G ranks, E experts (E divisible by G); rank d owns experts
 * [d*E/G, (d+1)*E/G) and its local expert weights are the [E/G, ...] slices of
 * the layer's weights.  `shape` is the global shape of one rank's batch (its
 * T tokens over all E experts) and must carry MOE_FLAG_CAPACITY.  One layer on
 * rank r, buffers as moe_forward's plus the EP ones (rows of H bf16 values):
 *   1. moe_route_dispatch + moe_gather: x_perm in the capacity layout.
 *   2. moe_ep_pack: send_meta [G][2][E/G] int32 (each destination's capacity
 *      and overflow counts) and send_ovf [G][S] rows (each destination's
 *      compacted overflow rows at the start of its slot), S =
 *      moe_ep_overflow_rows.
 *   3. all-to-all (equal splits) of x_perm[0, E*C) into recv_cap
 *      [G][E/G*C] rows (pass 1), of send_meta into recv_meta, and of
 *      send_ovf into recv_ovf [G][S] rows (pass 2).
 *   4. moe_ep_local_dispatch: the received rows in expert-contiguous order in
 *      x_loc and the local GEMM schedule in ws_loc, a workspace of the local
 *      shape (moe_ep_local_shape: T = G*(E/G*C + S), E/G experts, k = 1).
 *   5. moe_grouped_swiglu / moe_grouped_down (or their fp8 forms) on the
 *      local shape: x_loc -> h_loc -> y_loc with the local weights.
 *   6. moe_ep_local_return: y_loc rows into back_cap [G][E/G*C] and back_ovf
 *      [G][S] at the positions their inputs arrived at.
 *   7. all-to-all of back_cap into y[0, E*C) and of back_ovf into
 *      recv_back_ovf [G][S] rows.
 *   8. moe_ep_unpack: the overflow rows' results into y's overflow region.
 *   9. moe_combine: out from y, dest_row, topk_w -- the result equals
 *      moe_forward's on the rank's tokens with all E experts.
 * ep_ws: moe_ep_workspace_bytes bytes, 16-byte aligned; written by
 * moe_ep_pack and moe_ep_local_dispatch and read by the later steps of the
 * same layer.  Row buffers are caller-owned device memory, 16-byte aligned;
 * the capacity buffers (recv_cap, back_cap) may be null when C = 0 and the
 * overflow buffers (send_ovf, recv_ovf, back_ovf, recv_back_ovf) when S = 0.
 * Errors: MOE_ERR_UNSUPPORTED_SHAPE (no MOE_FLAG_CAPACITY, G < 1, E not
 * divisible by G, local T >= 2^30), MOE_ERR_INVALID_ARG (null or misaligned
 * pointer), MOE_ERR_CUDA (launch failure).  Counts in recv_meta that exceed
 * what the buffers hold (never produced by moe_ep_pack) are clamped and set
 * MOE_DEV_BAD_ROW in ws_loc's status.
 * ------------------------------------------------------------------------ */

/* S: rows of one (source, destination) overflow slot, min(k, E/G) *
 * max(0, T - C) (one source's tokens send at most min(k, E/G) pairs each to
 * one destination, and an expert overflows by at most T - C).  -1 for an
 * unsupported shape or G. */
MOE_API int64_t moe_ep_overflow_rows(const moe_shape *shape, int32_t G);

/* Bytes of the EP workspace, or 0 for an unsupported shape or G. */
MOE_API size_t moe_ep_workspace_bytes(const moe_shape *shape, int32_t G);

/* The local shape of step 5: T = G*(E/G*C + S), H, F, E/G experts, k = 1,
 * C = 0, flags 0. */
MOE_API moe_status moe_ep_local_shape(const moe_shape *shape, int32_t G, moe_shape *local);

/* Step 2 (reads the capacity and overflow counts moe_route_dispatch /
 * moe_permute left in ws). */
MOE_API moe_status moe_ep_pack(const moe_shape *shape, int32_t G, const void *x_perm, const void *ws,
                               void *send_ovf, int32_t *send_meta, void *ep_ws, void *stream);

/* The row copy of step 1 and step 2 in one launch: x_perm's capacity slots
 * filled from x by src_token (zero rows for unfilled slots), each overflow
 * row copied from x straight into its destination's slot of send_ovf (so
 * x_perm's overflow region is not written and may be as short as E*C rows),
 * send_meta and the destination starts as moe_ep_pack writes them.  Replaces
 * moe_gather + moe_ep_pack after moe_route_dispatch; x: device bf16 [T,H],
 * src_token: from moe_route_dispatch; ws: the routing workspace (read: the
 * capacity and overflow counts; its status word gets MOE_DEV_BAD_ROW for a
 * row that does not fit a slot). */
MOE_API moe_status moe_ep_gather_pack(const moe_shape *shape, int32_t G, const void *x, const int32_t *src_token,
                                      void *x_perm, void *ws, void *send_ovf, int32_t *send_meta, void *ep_ws,
                                      void *stream);

/* Step 4.  ws_loc: a workspace of the local shape, initialised once
 * (moe_workspace_init with the local shape). */
MOE_API moe_status moe_ep_local_dispatch(const moe_shape *shape, int32_t G, const int32_t *recv_meta,
                                         const void *recv_cap, const void *recv_ovf, void *x_loc, void *ws_loc,
                                         void *ep_ws, void *stream);

/* Step 6. */
MOE_API moe_status moe_ep_local_return(const moe_shape *shape, int32_t G, const void *y_loc, void *back_cap,
                                       void *back_ovf, void *ep_ws, void *stream);

/* Step 8. */
MOE_API moe_status moe_ep_unpack(const moe_shape *shape, int32_t G, const void *recv_back_ovf, void *y, void *ep_ws,
                                 void *stream);

/* Steps 8 and 9 in one launch: moe_combine (y, dest_row, topk_w -> out) that
 * reads each overflow row's result from recv_back_ovf, where moe_ep_unpack
 * would have copied it from, instead of from y (y's overflow region is left
 * as it was).  out equals that of moe_ep_unpack + moe_combine bit for bit.
 * dest_row, topk_w: device [T*k]; out: device bf16 [T,H], 16-byte aligned. */
MOE_API moe_status moe_ep_unpack_combine(const moe_shape *shape, int32_t G, const void *recv_back_ovf,
                                         const void *y, const int32_t *dest_row, const float *topk_w, void *out,
                                         void *ep_ws, void *stream);

/* ------------------------------------------------------------------------
 * Expert parallelism by device-initiated peer stores ("direct" form).
 *
 * The same layer and the same result per rank as above, with the all-to-all
 * written as two kernels that store rows straight into the other ranks'
 * buffers (peer pointers, e.g. from symmetric memory or CUDA IPC over
 * NVLink): only the routed rows cross the links (no worst-case slots), the
 * receiver needs no copy into its layout, and the results land in each
 * source's y rows.  The Cap-and-Spill page's two passes move a buffer sized
 * for the worst case (the critique's point that they send as much as one
 * padded pass); here the receive buffers are still sized for the worst case,
 * but only the real rows move.
 *
 * `shape`: one rank's batch (T tokens, all E experts), uncapped layout (no
 * MOE_FLAG_CAPACITY); E divisible by G; G * E <= 4096.  One layer on rank r:
 *   1. moe_route_dispatch (uncapped): topk_idx, expert_counts, expert_offsets,
 *      dest_row on rank r.
 *   2. all-gather of expert_counts into cnt_all [G][E] int32 (every rank the
 *      same array).
 *   3. moe_ep_direct_plan(rank r): this rank's send positions, its local
 *      layout and GEMM schedule (ws_loc: a workspace of the local shape,
 *      moe_ep_direct_local_shape, initialised once) and its return segments.
 *   4. moe_ep_direct_dispatch: each routed pair's x row into the x_loc of its
 *      expert's rank; then a barrier over the ranks (a stream-ordered
 *      collective), after which every rank's x_loc holds its rows.
 *   5. moe_grouped_swiglu / moe_grouped_down on the local shape with the
 *      local weights: x_loc -> h_loc -> y_loc.
 *   6. moe_ep_direct_return: each local result row into its source's y row;
 *      then a barrier.
 *   7. moe_combine on rank r (y, dest_row, topk_w): equals moe_forward's out
 *      on the rank's tokens with all E experts.
 * peer_x_loc, peer_y: DEVICE arrays of G pointers (uint64), entry d = rank
 * d's x_loc / y as this rank's kernels address it (its own entry included).
 * x_loc holds moe_ep_direct_local_rows rows; y is moe_forward's y (T*k rows).
 * Every kernel that stores into peer memory (the puts, the return, the down
 * projection with its return) ends each block with a block barrier and one
 * system-scope fence.  ep_ws:
 * moe_ep_direct_workspace_bytes bytes, written by the plan, read by the two
 * puts of the same layer.  Errors as for the Cap-and-Spill calls; counts in
 * cnt_all beyond what the buffers hold (each (source, expert) above T, each
 * source's rows for one rank above T*min(k, E/G)) are clamped identically on
 * every rank and set MOE_DEV_BAD_ROW in ws_loc's status.
 * ------------------------------------------------------------------------ */

/* Local rows of one rank, G*T*min(k, E/G); -1 for an unsupported shape or G. */
MOE_API int64_t moe_ep_direct_local_rows(const moe_shape *shape, int32_t G);

/* Bytes of the direct-form EP workspace, or 0 for an unsupported shape or G. */
MOE_API size_t moe_ep_direct_workspace_bytes(const moe_shape *shape, int32_t G);

/* The local shape of step 5: T = moe_ep_direct_local_rows, H, F, E/G experts,
 * k = 1, C = 0, flags 0. */
MOE_API moe_status moe_ep_direct_local_shape(const moe_shape *shape, int32_t G, moe_shape *local);

/* Step 3.  cnt_all: device [G][E] int32; rank in [0, G); peer_y: the device
 * array of step 6 (may be null when moe_ep_direct_down_return is not used):
 * the plan also records each local row's destination address for it. */
MOE_API moe_status moe_ep_direct_plan(const moe_shape *shape, int32_t G, int32_t rank, const int32_t *cnt_all,
                                      const void *peer_y, void *ws_loc, void *ep_ws, void *stream);

/* Steps 3 and 4 in one launch (the form the layer uses): every block of the
 * dispatch derives this rank's send positions from cnt_all itself, so the
 * stores start at once, and one block also lays out the local rows as
 * moe_ep_direct_plan does.  x_scale null: x is bf16 [T,H] and peer_x_loc the
 * owners' x_loc; else x holds e4m3 codes [T,H] with scales x_scale [T], and
 * peer_x_loc / peer_scale_loc the owners' x_loc_q / scale_loc (the fp8 form).
 * ws: the rank's routing workspace; ws_loc: its local workspace. */
MOE_API moe_status moe_ep_direct_plan_dispatch(const moe_shape *shape, int32_t G, int32_t rank,
                                               const int32_t *cnt_all, const void *peer_y, const void *x,
                                               const float *x_scale, const int32_t *topk_idx, const int32_t *dest_row,
                                               const int32_t *expert_offsets, const void *peer_x_loc,
                                               const void *peer_scale_loc, void *ws, void *ws_loc, void *ep_ws,
                                               void *stream);

/* Steps 3 and 4 of the fp8 form in one launch, the token rows quantized on
 * the way: x is the rank's bf16 token rows [T,H]; each routed pair's row is
 * quantized by the warp that sends it, with the arithmetic of
 * moe_quantize_rows_fp8 (the same codes and scale bit for bit), and its e4m3
 * code row and scale are stored into the owner's x_loc_q and scale_loc
 * (peer_x_loc_q, peer_scale_loc: device arrays of G addresses).  Replaces
 * moe_quantize_rows_fp8 (MOE_ROWS_TOKENS) + moe_ep_direct_plan_dispatch with
 * codes; a token sent to k experts is quantized k times.  Other arguments and
 * errors as moe_ep_direct_plan_dispatch. */
MOE_API moe_status moe_ep_direct_plan_dispatch_quantize(const moe_shape *shape, int32_t G, int32_t rank,
                                                        const int32_t *cnt_all, const void *peer_y, const void *x,
                                                        const int32_t *topk_idx, const int32_t *dest_row,
                                                        const int32_t *expert_offsets, const void *peer_x_loc_q,
                                                        const void *peer_scale_loc, void *ws, void *ws_loc,
                                                        void *ep_ws, void *stream);

/* Step 4 (ws: the rank's routing workspace, for its status word). */
MOE_API moe_status moe_ep_direct_dispatch(const moe_shape *shape, int32_t G, const void *x, const int32_t *topk_idx,
                                          const int32_t *dest_row, const int32_t *expert_offsets,
                                          const void *peer_x_loc, void *ws, void *ep_ws, void *stream);

/* Step 6. */
MOE_API moe_status moe_ep_direct_return(const moe_shape *shape, int32_t G, const void *y_loc, const void *peer_y,
                                        void *ep_ws, void *stream);

/* Steps 5b and 6 in one kernel: the local down projection (h_loc [local T][F]
 * bf16, w_down: the rank's [E/G][F][H] slice) whose epilogue stores each
 * result row straight into its token's rank's y, at the address the plan
 * recorded from peer_y (rows without one are not stored).  Replaces
 * moe_grouped_down + moe_ep_direct_return; the plan must have been given
 * peer_y.  A barrier over the ranks follows, as after step 6. */
MOE_API moe_status moe_ep_direct_down_return(const moe_shape *shape, int32_t G, const void *h_loc,
                                             const void *w_down, void *ws_loc, void *ep_ws, void *stream);

/* The fp8 layer in the peer-store form: e4m3 rows on the links (half the
 * bytes of bf16 rows).  Each rank quantizes its token rows once
 * (moe_quantize_rows_fp8, MOE_ROWS_TOKENS: x_q [T,H] codes, x_scale [T]);
 * step 4 becomes moe_ep_direct_dispatch_fp8, which stores each routed pair's
 * code row into its expert's rank's x_loc_q [local T, H] and the row's scale
 * into that rank's scale_loc [local T] (peer_x_loc_q, peer_scale_loc: device
 * arrays of G addresses); step 5 is moe_grouped_swiglu_fp8 on the local shape
 * (x_loc_q, scale_loc, no src_token; the rank's weight codes and scales, as
 * moe_quantize_weights_fp8 leaves them, sliced to its experts), then
 * moe_ep_direct_quantize_h (or moe_quantize_rows_fp8, MOE_ROWS_H, no
 * src_token: every row) and moe_ep_direct_down_return_fp8, the fp8 down projection storing each result
 * row straight into its token's rank's y.  Each rank's out equals
 * moe_forward_fp8's on its tokens. */
MOE_API moe_status moe_ep_direct_dispatch_fp8(const moe_shape *shape, int32_t G, const void *x_q,
                                              const float *x_scale, const int32_t *topk_idx, const int32_t *dest_row,
                                              const int32_t *expert_offsets, const void *peer_x_loc_q,
                                              const void *peer_scale_loc, void *ws, void *ep_ws, void *stream);

MOE_API moe_status moe_ep_direct_down_return_fp8(const moe_shape *shape, int32_t G, const void *h_q,
                                                 const float *h_scale, const void *wd_q, const float *wd_scale,
                                                 void *ws_loc, void *ep_ws, void *stream);

/* The fp8 form's h quantization limited to the local rows the plan laid out
 * (the received rows, read from ep_ws on the device): h_loc [local T, F] bf16
 * -> h_q [local T, F] codes, h_scale [local T]; rows past them are left
 * unwritten.  Same codes as moe_quantize_rows_fp8 (MOE_ROWS_H) on those rows. */
MOE_API moe_status moe_ep_direct_quantize_h(const moe_shape *shape, int32_t G, const void *h_loc, void *h_q,
                                            float *h_scale, void *ep_ws, void *stream);

/* Upper bound, in nanoseconds, of every bounded device wait (default 1e9). */
MOE_API void moe_set_wait_timeout_ns(uint64_t ns);

MOE_API const char *moe_status_string(moe_status status);

/* Text of the last CUDA failure seen by this thread's calls ("no error" if none). */
MOE_API const char *moe_last_error_string(void);

/* Library version, major*10000 + minor*100 + patch. */
MOE_API int32_t moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
