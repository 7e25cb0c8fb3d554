// extern "C" entry points declared in include/moe.h: argument validation,
// workspace carving and kernel launches.  No entry point allocates, frees or
// synchronises except moe_read_status.
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdio>

#include "common.cuh"

namespace moe {
cudaError_t launch_route(const moe_shape &s, const void *x, const float *w_router, const float *bias, float *logits,
                         int32_t *topk_idx, float *topk_w, const WsLayout &L, void *ws, uint64_t timeout_ns,
                         int num_sms, cudaStream_t stream, const FusedDispatch *fused);
cudaError_t launch_gather(const moe_shape &s, const void *x, const int32_t *src_token, void *x_perm,
                          const WsLayout &L, void *ws, int num_sms, cudaStream_t stream);
cudaError_t launch_dispatch_index(const moe_shape &s, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                                  int32_t *src_token, int32_t *dest_row, const WsLayout &L, void *ws,
                                  uint64_t timeout_ns, int num_sms, cudaStream_t stream);
cudaError_t launch_permute(const moe_shape &s, const void *x, const int32_t *topk_idx, int32_t *counts,
                           int32_t *offsets, int32_t *src_token, int32_t *dest_row, void *x_perm, const WsLayout &L,
                           void *ws, uint64_t timeout_ns, int num_sms, cudaStream_t stream);
cudaError_t launch_grouped_gemm(int mode, const moe_shape &s, const void *act, const void *w0, const void *w1,
                                void *out, const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                cudaStream_t stream, const int32_t *src_token, const CombineOut *comb = nullptr,
                                const unsigned long long *row_addr = nullptr);
cudaError_t launch_combine(const moe_shape &s, const void *y, const int32_t *dest_row, const float *topk_w, void *out,
                           cudaStream_t stream);
cudaError_t launch_grouped_gemm_fp8(int mode, const moe_shape &s, const void *act, const float *row_scale,
                                    const void *w0, const float *w0_scale, const void *w1, const float *w1_scale,
                                    void *out, const WsLayout &L, void *ws, uint64_t timeout_ns, int num_sms,
                                    cudaStream_t stream, const int32_t *src_token, const CombineOut *comb = nullptr,
                                    const unsigned long long *row_addr = nullptr);
cudaError_t launch_quant_weights(int E, int K, int N, const void *w, void *q, float *scale, cudaStream_t stream);
cudaError_t launch_quant_rows(const moe_shape &s, int K, const void *src, int src_rows, const int32_t *idx,
                              bool gather, void *q, float *scale, const WsLayout &L, void *ws, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_quant_tokens(const moe_shape &s, const void *x, void *q, float *scale, int num_sms,
                                cudaStream_t stream);
int64_t ep_overflow_rows(const moe_shape &s, int G);
size_t ep_workspace_bytes(const moe_shape &s, int G);
cudaError_t launch_ep_pack(const moe_shape &s, int G, const void *x_perm, const WsLayout &L, void *ws, void *send_ovf,
                           int32_t *send_meta, void *ep_ws, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_gather_pack(const moe_shape &s, int G, const void *x, const int32_t *src_token, void *x_perm,
                                  const WsLayout &L, void *ws, void *send_ovf, int32_t *send_meta, void *ep_ws,
                                  int num_sms, cudaStream_t stream);
cudaError_t launch_ep_unpack_combine(const moe_shape &s, int G, const void *recv_back_ovf, const void *y,
                                     const int32_t *dest_row, const float *topk_w, void *out, void *ep_ws,
                                     cudaStream_t stream);
cudaError_t launch_ep_local_dispatch(const moe_shape &s, int G, const int32_t *recv_meta, const void *recv_cap,
                                     const void *recv_ovf, void *x_loc, const WsLayout &Lloc, void *ws_loc,
                                     void *ep_ws, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_local_return(const moe_shape &s, int G, const void *y_loc, void *back_cap, void *back_ovf,
                                   void *ep_ws, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_unpack(const moe_shape &s, int G, const void *recv_back_ovf, void *y, void *ep_ws, int num_sms,
                             cudaStream_t stream);
int64_t ep_direct_local_rows(const moe_shape &s, int G);
bool ep_direct_counts_fit(const moe_shape &s, int G);
size_t ep_direct_workspace_bytes(const moe_shape &s, int G);
cudaError_t launch_ep_direct_plan(const moe_shape &s, int G, int rank, const int32_t *cnt_all, const void *peer_y,
                                  const WsLayout &Lloc, void *ws_loc, void *ep_ws, cudaStream_t stream);
const unsigned long long *ep_direct_row_addr(void *ep_ws, const moe_shape &s, int G);
const int32_t *ep_direct_local_total(void *ep_ws, const moe_shape &s, int G);
cudaError_t launch_ep_direct_plan_put(const moe_shape &s, int G, int rank, const int32_t *cnt_all,
                                      const void *peer_y, const WsLayout &Lloc, void *ws_loc, const void *x,
                                      const int32_t *topk_idx, const int32_t *dest_row, const int32_t *offsets,
                                      const void *peer_x_loc, void *ep_ws, uint32_t *status, int num_sms,
                                      cudaStream_t stream, const float *x_scale, const void *peer_scale,
                                      bool quantize);
cudaError_t launch_quant_rows_counted(const void *src, int K, int rows_cap, const int *rows_dev, void *q,
                                      float *scale, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_direct_put(const moe_shape &s, int G, const void *x, const int32_t *topk_idx,
                                 const int32_t *dest_row, const int32_t *offsets, const void *peer_x_loc,
                                 void *ep_ws, uint32_t *status, int num_sms, cudaStream_t stream,
                                 const float *x_scale = nullptr, const void *peer_scale = nullptr);
cudaError_t launch_ep_direct_return(const moe_shape &s, int G, const void *y_loc, const void *peer_y, void *ep_ws,
                                    int num_sms, cudaStream_t stream);
}  // namespace moe

using namespace moe;

namespace {

std::atomic<uint64_t> g_timeout_ns{1000000000ull};
thread_local char g_last_error[160] = "no error";

constexpr uint32_t kKnownFlags = MOE_FLAG_CAPACITY | MOE_FLAG_LOGITS_IN | MOE_FLAG_FUSED_COMBINE |
                                  MOE_FLAG_TEST_STALL_SCAN | MOE_FLAG_TEST_STALL_GEMM;

bool aligned(const void *p, uintptr_t a) { return p != nullptr && ((uintptr_t)p % a) == 0; }
// A buffer of zero rows may be null.
bool aligned_or_empty(const void *p, uintptr_t a, bool empty) { return (empty && p == nullptr) || aligned(p, a); }

moe_status cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

moe_status check_shape(const moe_shape *s) {
    if (!s) return MOE_ERR_INVALID_ARG;
    if (s->flags & ~kKnownFlags) return MOE_ERR_INVALID_ARG;
    if (s->T < 1 || s->E < 1 || s->E > kMaxExperts || s->k < 1 || s->k > s->E || s->C < 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (s->H < 128 || s->H % 128 || s->H > 65536 || s->F < 128 || s->F % 128 || s->F > 65536)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    const bool capped = (s->flags & MOE_FLAG_CAPACITY) != 0;
    const int64_t R = (int64_t)s->T * s->k;
    const int64_t P = permuted_rows(s->T, s->E, s->k, s->C, capped);
    if (R >= (1ll << 30) || P >= (1ll << 30) || (int64_t)s->E * s->C >= (1ll << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int64_t units = (int64_t)max_tiles_for(P, s->E) * (s->F / 128 > s->H / 256 + 1 ? s->F / 128 : s->H / 256 + 1);
    if (units >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

WsLayout layout_of(const moe_shape *s) {
    return ws_layout(s->T, s->H, s->E, s->k, s->C, (s->flags & MOE_FLAG_CAPACITY) != 0);
}

// sm_100 check and SM count of the current device, cached per device.
moe_status device_info(int *num_sms) {
    static std::atomic<int> cache[64];  // 0 unknown, -1 not sm_100, else SM count
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    int v = (dev >= 0 && dev < 64) ? cache[dev].load() : 0;
    if (v == 0) {
        int major = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        v = (major == 10 && sms > 0) ? sms : -1;
        if (dev >= 0 && dev < 64) cache[dev].store(v);
    }
    if (v < 0) {
        std::snprintf(g_last_error, sizeof(g_last_error), "current device is not sm_100");
        return MOE_ERR_DEVICE;
    }
    *num_sms = v;
    return MOE_OK;
}

moe_status check_ws(void *ws) { return aligned(ws, 256) ? MOE_OK : MOE_ERR_WORKSPACE; }

}  // namespace

// Shared with the other entry-point file of the library (static_ws.cu).
moe_status moe_internal_check_shape(const moe_shape *s) { return check_shape(s); }
moe_status moe_internal_device_info(int *num_sms) { return device_info(num_sms); }
moe_status moe_internal_cuda_fail(cudaError_t e, const char *where) { return cuda_fail(e, where); }
void moe_internal_set_error(const char *msg) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
uint64_t moe_internal_timeout_ns() { return g_timeout_ns.load(); }

extern "C" {

int64_t moe_permuted_rows(const moe_shape *s) {
    if (check_shape(s) != MOE_OK) return -1;
    return permuted_rows(s->T, s->E, s->k, s->C, (s->flags & MOE_FLAG_CAPACITY) != 0);
}

size_t moe_workspace_bytes(const moe_shape *s) {
    if (check_shape(s) != MOE_OK) return 0;
    return layout_of(s).total;
}

moe_status moe_workspace_layout(const moe_shape *s, moe_ws_layout *out) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!out) return MOE_ERR_INVALID_ARG;
    const WsLayout L = layout_of(s);
    out->total = L.total;
    out->status = L.status;
    out->num_tiles = L.num_tiles;
    out->total_spill = L.total_spill;
    out->cap_cnt = L.cap_cnt;
    out->spill_cnt = L.spill_cnt;
    out->spill_off = L.spill_off;
    out->order = L.order;
    out->grp_tile_start = L.grp_tile_start;
    out->tile_map = L.tile_map;
    out->max_tiles = L.max_tiles;
    out->tile_rows = kTileRows;
    out->row_cap = L.tile_rows;
    return MOE_OK;
}

moe_status moe_workspace_init(const moe_shape *s, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    cudaError_t e = cudaMemsetAsync(ws, 0, layout_of(s).total, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_workspace_init");
}

moe_status moe_route(const moe_shape *s, const void *x, const float *w_router, const float *bias, float *logits,
                     int32_t *topk_idx, float *topk_w, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    const bool logits_in = (s->flags & MOE_FLAG_LOGITS_IN) != 0;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
    if (logits_in) {
        if (!aligned(logits, 4)) return MOE_ERR_INVALID_ARG;
    } else {
        if (!aligned(x, 16) || !aligned(w_router, 16)) return MOE_ERR_INVALID_ARG;
        if (bias && !aligned(bias, 4)) return MOE_ERR_INVALID_ARG;
        if (logits && !aligned(logits, 4)) return MOE_ERR_INVALID_ARG;
    }
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_route(*s, x, w_router, bias, logits, topk_idx, topk_w, L, ws, g_timeout_ns.load(), sms,
                                 (cudaStream_t)stream, nullptr);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route");
}

moe_status moe_permute(const moe_shape *s, const void *x, const int32_t *topk_idx, int32_t *expert_counts,
                       int32_t *expert_offsets, int32_t *src_token, int32_t *dest_row, void *x_perm, void *ws,
                       void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 4) || !aligned(expert_counts, 4) ||
        !aligned(expert_offsets, 4) || !aligned(src_token, 4) || !aligned(dest_row, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_permute(*s, x, topk_idx, expert_counts, expert_offsets, src_token, dest_row, x_perm, L, ws,
                                   g_timeout_ns.load(), sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_permute");
}

moe_status moe_grouped_swiglu(const moe_shape *s, const void *x_perm, const void *w_gate, const void *w_up, void *h,
                              void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(x_perm, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(h, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_grouped_gemm(0, *s, x_perm, w_gate, w_up, h, L, ws, g_timeout_ns.load(), sms,
                                        (cudaStream_t)stream, nullptr);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_swiglu");
}

moe_status moe_grouped_swiglu_gather(const moe_shape *s, const void *x, const int32_t *src_token, const void *w_gate,
                                     const void *w_up, void *h, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(x, 16) || !aligned(src_token, 4) || !aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(h, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_grouped_gemm(0, *s, x, w_gate, w_up, h, L, ws, g_timeout_ns.load(), sms,
                                        (cudaStream_t)stream, src_token);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_swiglu_gather");
}

moe_status moe_grouped_down(const moe_shape *s, const void *h, const void *w_down, void *y, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(h, 16) || !aligned(w_down, 16) || !aligned(y, 16)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_grouped_gemm(1, *s, h, w_down, w_down, y, L, ws, g_timeout_ns.load(), sms,
                                        (cudaStream_t)stream, nullptr);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_down");
}

moe_status moe_grouped_down_combine(const moe_shape *s, const void *h, const void *w_down, const int32_t *src_token,
                                    const int32_t *dest_row, const float *topk_w, void *y, void *out, void *ws,
                                    void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(h, 16) || !aligned(w_down, 16) || !aligned(y, 16) || !aligned(out, 16) || !aligned(src_token, 4) ||
        !aligned(dest_row, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    const CombineOut comb{src_token, dest_row, topk_w, out};
    cudaError_t e = launch_grouped_gemm(1, *s, h, w_down, w_down, y, L, ws, g_timeout_ns.load(), sms,
                                        (cudaStream_t)stream, nullptr, &comb);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_down_combine");
}

moe_status moe_combine(const moe_shape *s, const void *y, const int32_t *dest_row, const float *topk_w, void *out,
                       void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(dest_row, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e = launch_combine(*s, y, dest_row, topk_w, out, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine");
}

moe_status moe_route_dispatch(const moe_shape *s, const void *x, const float *w_router, const float *bias,
                              float *logits, int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                              int32_t *expert_offsets, int32_t *src_token, int32_t *dest_row, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if ((int64_t)s->T * s->k > kFusedDispatchMaxPairs || (s->flags & MOE_FLAG_TEST_STALL_SCAN)) {
        st = moe_route(s, x, w_router, bias, logits, topk_idx, topk_w, ws, stream);
        if (st != MOE_OK) return st;
        if (!aligned(x, 16) || !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) ||
            !aligned(src_token, 4) || !aligned(dest_row, 4))
            return MOE_ERR_INVALID_ARG;
        int sms = 0;
        if ((st = device_info(&sms)) != MOE_OK) return st;
        const WsLayout L = layout_of(s);
        cudaError_t e = launch_dispatch_index(*s, topk_idx, expert_counts, expert_offsets, src_token, dest_row, L, ws,
                                              g_timeout_ns.load(), sms, (cudaStream_t)stream);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_dispatch");
    }
    const bool logits_in = (s->flags & MOE_FLAG_LOGITS_IN) != 0;
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) ||
        !aligned(src_token, 4) || !aligned(dest_row, 4))
        return MOE_ERR_INVALID_ARG;
    if (logits_in) {
        if (!aligned(logits, 4)) return MOE_ERR_INVALID_ARG;
    } else {
        if (!aligned(x, 16) || !aligned(w_router, 16)) return MOE_ERR_INVALID_ARG;
        if (bias && !aligned(bias, 4)) return MOE_ERR_INVALID_ARG;
        if (logits && !aligned(logits, 4)) return MOE_ERR_INVALID_ARG;
    }
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    const FusedDispatch fd{expert_counts, expert_offsets, src_token, dest_row};
    cudaError_t e = launch_route(*s, x, w_router, bias, logits, topk_idx, topk_w, L, ws, g_timeout_ns.load(), sms,
                                 (cudaStream_t)stream, &fd);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_dispatch");
}

moe_status moe_gather(const moe_shape *s, const void *x, const int32_t *src_token, void *x_perm, void *ws,
                      void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(src_token, 4)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_gather(*s, x, src_token, x_perm, L, ws, sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_gather");
}

moe_status moe_forward(const moe_shape *s, const moe_forward_args *a, void *ws, void *stream) {
    if (!a) return MOE_ERR_INVALID_ARG;
    moe_status st = moe_route_dispatch(s, a->x, a->w_router, a->bias, a->logits, a->topk_idx, a->topk_w,
                                       a->expert_counts, a->expert_offsets, a->src_token, a->dest_row, ws, stream);
    if (st != MOE_OK) return st;
    if (a->x_perm) {
        st = moe_gather(s, a->x, a->src_token, a->x_perm, ws, stream);
        if (st != MOE_OK) return st;
        st = moe_grouped_swiglu(s, a->x_perm, a->w_gate, a->w_up, a->h, ws, stream);
    } else {
        st = moe_grouped_swiglu_gather(s, a->x, a->src_token, a->w_gate, a->w_up, a->h, ws, stream);
    }
    if (st != MOE_OK) return st;
    if (s->flags & MOE_FLAG_FUSED_COMBINE)
        return moe_grouped_down_combine(s, a->h, a->w_down, a->src_token, a->dest_row, a->topk_w, a->y, a->out, ws,
                                        stream);
    st = moe_grouped_down(s, a->h, a->w_down, a->y, ws, stream);
    if (st != MOE_OK) return st;
    return moe_combine(s, a->y, a->dest_row, a->topk_w, a->out, stream);
}

moe_status moe_quantize_weights_fp8(const moe_shape *s, int which, const void *w, void *w_q, float *w_scale,
                                    void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if ((which != MOE_WEIGHTS_GATE_UP && which != MOE_WEIGHTS_DOWN) || !aligned(w, 16) || !aligned(w_q, 16) ||
        !aligned(w_scale, 4))
        return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const int K = which == MOE_WEIGHTS_GATE_UP ? s->H : s->F;
    const int N = which == MOE_WEIGHTS_GATE_UP ? s->F : s->H;
    cudaError_t e = launch_quant_weights(s->E, K, N, w, w_q, w_scale, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_quantize_weights_fp8");
}

moe_status moe_quantize_rows_fp8(const moe_shape *s, int which, const void *src, const int32_t *src_token, void *q,
                                 float *scale, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (which != MOE_ROWS_X_PERM && which != MOE_ROWS_TOKENS && which != MOE_ROWS_H) return MOE_ERR_INVALID_ARG;
    if (!aligned(src, 16) || !aligned(q, 16) || !aligned(scale, 4)) return MOE_ERR_INVALID_ARG;
    if (which == MOE_ROWS_X_PERM && !aligned(src_token, 4)) return MOE_ERR_INVALID_ARG;
    if (which == MOE_ROWS_H && src_token && !aligned(src_token, 4)) return MOE_ERR_INVALID_ARG;
    if (which != MOE_ROWS_TOKENS && (st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e;
    if (which == MOE_ROWS_TOKENS) {
        e = launch_quant_tokens(*s, src, q, scale, sms, (cudaStream_t)stream);
    } else {
        const WsLayout L = layout_of(s);
        const bool xp = which == MOE_ROWS_X_PERM;
        e = launch_quant_rows(*s, xp ? s->H : s->F, src, xp ? s->T : INT32_MAX, src_token, xp, q, scale, L, ws, sms,
                              (cudaStream_t)stream);
    }
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_quantize_rows_fp8");
}

moe_status moe_grouped_swiglu_fp8(const moe_shape *s, const void *x_q, const float *x_scale, const int32_t *src_token,
                                  const void *wg_q, const float *wg_scale, const void *wu_q, const float *wu_scale,
                                  void *h, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(x_q, 16) || !aligned(x_scale, 4) || !aligned(wg_q, 16) || !aligned(wg_scale, 4) ||
        !aligned(wu_q, 16) || !aligned(wu_scale, 4) || !aligned(h, 16))
        return MOE_ERR_INVALID_ARG;
    if (src_token && !aligned(src_token, 4)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_grouped_gemm_fp8(0, *s, x_q, x_scale, wg_q, wg_scale, wu_q, wu_scale, h, L, ws,
                                            g_timeout_ns.load(), sms, (cudaStream_t)stream, src_token);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_swiglu_fp8");
}

moe_status moe_grouped_down_fp8(const moe_shape *s, const void *h_q, const float *h_scale, const void *wd_q,
                                const float *wd_scale, void *y, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(h_q, 16) || !aligned(h_scale, 4) || !aligned(wd_q, 16) || !aligned(wd_scale, 4) || !aligned(y, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_grouped_gemm_fp8(1, *s, h_q, h_scale, wd_q, wd_scale, wd_q, wd_scale, y, L, ws,
                                            g_timeout_ns.load(), sms, (cudaStream_t)stream, nullptr);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_down_fp8");
}

moe_status moe_grouped_down_fp8_combine(const moe_shape *s, const void *h_q, const float *h_scale, const void *wd_q,
                                        const float *wd_scale, const int32_t *src_token, const int32_t *dest_row,
                                        const float *topk_w, void *y, void *out, void *ws, void *stream) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!aligned(h_q, 16) || !aligned(h_scale, 4) || !aligned(wd_q, 16) || !aligned(wd_scale, 4) || !aligned(y, 16) ||
        !aligned(out, 16) || !aligned(src_token, 4) || !aligned(dest_row, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    const CombineOut comb{src_token, dest_row, topk_w, out};
    cudaError_t e = launch_grouped_gemm_fp8(1, *s, h_q, h_scale, wd_q, wd_scale, wd_q, wd_scale, y, L, ws,
                                            g_timeout_ns.load(), sms, (cudaStream_t)stream, nullptr, &comb);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_grouped_down_fp8_combine");
}

moe_status moe_forward_fp8(const moe_shape *s, const moe_forward_fp8_args *a, void *ws, void *stream) {
    if (!a) return MOE_ERR_INVALID_ARG;
    moe_status st = moe_route_dispatch(s, a->x, a->w_router, a->bias, a->logits, a->topk_idx, a->topk_w,
                                       a->expert_counts, a->expert_offsets, a->src_token, a->dest_row, ws, stream);
    if (st != MOE_OK) return st;
    if (a->x_q_per_token) {
        st = moe_quantize_rows_fp8(s, MOE_ROWS_TOKENS, a->x, nullptr, a->x_q, a->x_scale, ws, stream);
        if (st != MOE_OK) return st;
        st = moe_grouped_swiglu_fp8(s, a->x_q, a->x_scale, a->src_token, a->wg_q, a->wg_scale, a->wu_q, a->wu_scale,
                                    a->h, ws, stream);
    } else {
        st = moe_quantize_rows_fp8(s, MOE_ROWS_X_PERM, a->x, a->src_token, a->x_q, a->x_scale, ws, stream);
        if (st != MOE_OK) return st;
        st = moe_grouped_swiglu_fp8(s, a->x_q, a->x_scale, nullptr, a->wg_q, a->wg_scale, a->wu_q, a->wu_scale, a->h,
                                    ws, stream);
    }
    if (st != MOE_OK) return st;
    st = moe_quantize_rows_fp8(s, MOE_ROWS_H, a->h, a->src_token, a->h_q, a->h_scale, ws, stream);
    if (st != MOE_OK) return st;
    if (s->flags & MOE_FLAG_FUSED_COMBINE)
        return moe_grouped_down_fp8_combine(s, a->h_q, a->h_scale, a->wd_q, a->wd_scale, a->src_token, a->dest_row,
                                            a->topk_w, a->y, a->out, ws, stream);
    st = moe_grouped_down_fp8(s, a->h_q, a->h_scale, a->wd_q, a->wd_scale, a->y, ws, stream);
    if (st != MOE_OK) return st;
    return moe_combine(s, a->y, a->dest_row, a->topk_w, a->out, stream);
}

// ------------------------------------------------------------ expert parallel --
namespace {
moe_status check_ep(const moe_shape *s, int32_t G) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if (!(s->flags & MOE_FLAG_CAPACITY) || G < 1 || s->E % G != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int64_t S = ep_overflow_rows(*s, G);
    const int64_t Tloc = (int64_t)G * ((int64_t)(s->E / G) * s->C + S);
    if (Tloc < 1 || Tloc >= (1ll << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}
moe_shape ep_local(const moe_shape *s, int32_t G) {
    const int64_t S = ep_overflow_rows(*s, G);
    moe_shape l;
    l.T = (int32_t)((int64_t)G * ((int64_t)(s->E / G) * s->C + S));
    l.H = s->H;
    l.F = s->F;
    l.E = s->E / G;
    l.k = 1;
    l.C = 0;
    l.flags = 0;
    return l;
}
}  // namespace

int64_t moe_ep_overflow_rows(const moe_shape *s, int32_t G) {
    if (check_ep(s, G) != MOE_OK) return -1;
    return ep_overflow_rows(*s, G);
}

size_t moe_ep_workspace_bytes(const moe_shape *s, int32_t G) {
    if (check_ep(s, G) != MOE_OK) return 0;
    return ep_workspace_bytes(*s, G);
}

moe_status moe_ep_local_shape(const moe_shape *s, int32_t G, moe_shape *local) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    if (!local) return MOE_ERR_INVALID_ARG;
    *local = ep_local(s, G);
    return check_shape(local);
}

moe_status moe_ep_pack(const moe_shape *s, int32_t G, const void *x_perm, const void *ws, void *send_ovf,
                       int32_t *send_meta, void *ep_ws, void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    const bool no_ovf = ep_overflow_rows(*s, G) == 0;
    if (!aligned(x_perm, 16) || !aligned_or_empty(send_ovf, 16, no_ovf) || !aligned(send_meta, 4) ||
        !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(const_cast<void *>(ws))) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_ep_pack(*s, G, x_perm, L, const_cast<void *>(ws), send_ovf, send_meta, ep_ws, sms,
                                   (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_pack");
}

moe_status moe_ep_gather_pack(const moe_shape *s, int32_t G, const void *x, const int32_t *src_token, void *x_perm,
                              void *ws, void *send_ovf, int32_t *send_meta, void *ep_ws, void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    const bool no_ovf = ep_overflow_rows(*s, G) == 0;
    if (!aligned(x, 16) || !aligned(src_token, 4) || !aligned_or_empty(x_perm, 16, s->C == 0) ||
        !aligned_or_empty(send_ovf, 16, no_ovf) || !aligned(send_meta, 4) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    cudaError_t e = launch_ep_gather_pack(*s, G, x, src_token, x_perm, L, ws, send_ovf, send_meta, ep_ws, sms,
                                          (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_gather_pack");
}

moe_status moe_ep_local_dispatch(const moe_shape *s, int32_t G, const int32_t *recv_meta, const void *recv_cap,
                                 const void *recv_ovf, void *x_loc, void *ws_loc, void *ep_ws, void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(recv_meta, 4) || !aligned_or_empty(recv_cap, 16, s->C == 0) ||
        !aligned_or_empty(recv_ovf, 16, ep_overflow_rows(*s, G) == 0) || !aligned(x_loc, 16) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws_loc)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const moe_shape l = ep_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    cudaError_t e = launch_ep_local_dispatch(*s, G, recv_meta, recv_cap, recv_ovf, x_loc, Lloc, ws_loc, ep_ws, sms,
                                             (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_local_dispatch");
}

moe_status moe_ep_local_return(const moe_shape *s, int32_t G, const void *y_loc, void *back_cap, void *back_ovf,
                               void *ep_ws, void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(y_loc, 16) || !aligned_or_empty(back_cap, 16, s->C == 0) ||
        !aligned_or_empty(back_ovf, 16, ep_overflow_rows(*s, G) == 0) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e = launch_ep_local_return(*s, G, y_loc, back_cap, back_ovf, ep_ws, sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_local_return");
}

moe_status moe_ep_unpack_combine(const moe_shape *s, int32_t G, const void *recv_back_ovf, const void *y,
                                 const int32_t *dest_row, const float *topk_w, void *out, void *ep_ws, void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    if (!aligned_or_empty(recv_back_ovf, 16, ep_overflow_rows(*s, G) == 0) || !aligned(y, 16) ||
        !aligned(dest_row, 4) || !aligned(topk_w, 4) || !aligned(out, 16) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    cudaError_t e = launch_ep_unpack_combine(*s, G, recv_back_ovf, y, dest_row, topk_w, out, ep_ws,
                                             (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_unpack_combine");
}

moe_status moe_ep_unpack(const moe_shape *s, int32_t G, const void *recv_back_ovf, void *y, void *ep_ws,
                         void *stream) {
    moe_status st = check_ep(s, G);
    if (st != MOE_OK) return st;
    if (!aligned_or_empty(recv_back_ovf, 16, ep_overflow_rows(*s, G) == 0) || !aligned(y, 16) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e = launch_ep_unpack(*s, G, recv_back_ovf, y, ep_ws, sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_unpack");
}

moe_status moe_read_status(void *ws, void *stream, uint32_t *device_status, int clear) {
    if (!aligned(ws, 256) || !device_status) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "moe_read_status");
    *device_status = v;
    return MOE_OK;
}

void moe_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns ? ns : 1); }

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_WORKSPACE: return "unusable workspace";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE: return "device is not sm_100";
    }
    return "unknown status";
}

const char *moe_last_error_string(void) { return g_last_error; }

int32_t moe_version(void) { return 100; }

}  // extern "C"

// ------------------------------------------- expert parallel, peer stores --
namespace {
moe_status check_ep_direct(const moe_shape *s, int32_t G) {
    moe_status st = check_shape(s);
    if (st != MOE_OK) return st;
    if ((s->flags & MOE_FLAG_CAPACITY) || G < 1 || s->E % G != 0 || !ep_direct_counts_fit(*s, G))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    const int64_t Tloc = ep_direct_local_rows(*s, G);
    if (Tloc < 1 || Tloc >= (1ll << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}
moe_shape ep_direct_local(const moe_shape *s, int32_t G) {
    moe_shape l;
    l.T = (int32_t)ep_direct_local_rows(*s, G);
    l.H = s->H;
    l.F = s->F;
    l.E = s->E / G;
    l.k = 1;
    l.C = 0;
    l.flags = 0;
    return l;
}
}  // namespace

int64_t moe_ep_direct_local_rows(const moe_shape *s, int32_t G) {
    if (check_ep_direct(s, G) != MOE_OK) return -1;
    return ep_direct_local_rows(*s, G);
}

size_t moe_ep_direct_workspace_bytes(const moe_shape *s, int32_t G) {
    if (check_ep_direct(s, G) != MOE_OK) return 0;
    return ep_direct_workspace_bytes(*s, G);
}

moe_status moe_ep_direct_local_shape(const moe_shape *s, int32_t G, moe_shape *local) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!local) return MOE_ERR_INVALID_ARG;
    *local = ep_direct_local(s, G);
    return check_shape(local);
}

moe_status moe_ep_direct_plan(const moe_shape *s, int32_t G, int32_t rank, const int32_t *cnt_all,
                              const void *peer_y, void *ws_loc, void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (rank < 0 || rank >= G) return MOE_ERR_INVALID_ARG;
    if (!aligned(cnt_all, 4) || !aligned(ep_ws, 16) || (peer_y && !aligned(peer_y, 8))) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws_loc)) != MOE_OK) return st;
    const moe_shape l = ep_direct_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    cudaError_t e = launch_ep_direct_plan(*s, G, rank, cnt_all, peer_y, Lloc, ws_loc, ep_ws, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_plan");
}

moe_status moe_ep_direct_dispatch(const moe_shape *s, int32_t G, const void *x, const int32_t *topk_idx,
                                  const int32_t *dest_row, const int32_t *expert_offsets, const void *peer_x_loc,
                                  void *ws, void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(dest_row, 4) || !aligned(expert_offsets, 4) ||
        !aligned(peer_x_loc, 8) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    uint32_t *status = (uint32_t *)((char *)ws + L.status);
    cudaError_t e = launch_ep_direct_put(*s, G, x, topk_idx, dest_row, expert_offsets, peer_x_loc, ep_ws, status, sms,
                                         (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_dispatch");
}

moe_status moe_ep_direct_return(const moe_shape *s, int32_t G, const void *y_loc, const void *peer_y, void *ep_ws,
                                void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(y_loc, 16) || !aligned(peer_y, 8) || !aligned(ep_ws, 16)) return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e = launch_ep_direct_return(*s, G, y_loc, peer_y, ep_ws, sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_return");
}

moe_status moe_ep_direct_down_return(const moe_shape *s, int32_t G, const void *h_loc, const void *w_down,
                                     void *ws_loc, void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(h_loc, 16) || !aligned(w_down, 16) || !aligned(ep_ws, 16)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws_loc)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const moe_shape l = ep_direct_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    cudaError_t e = launch_grouped_gemm(1, l, h_loc, w_down, w_down, nullptr, Lloc, ws_loc, g_timeout_ns.load(), sms,
                                        (cudaStream_t)stream, nullptr, nullptr, ep_direct_row_addr(ep_ws, *s, G));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_down_return");
}

moe_status moe_ep_direct_dispatch_fp8(const moe_shape *s, int32_t G, const void *x_q, const float *x_scale,
                                      const int32_t *topk_idx, const int32_t *dest_row, const int32_t *expert_offsets,
                                      const void *peer_x_loc_q, const void *peer_scale_loc, void *ws, void *ep_ws,
                                      void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(x_q, 16) || !aligned(x_scale, 4) || !aligned(topk_idx, 4) || !aligned(dest_row, 4) ||
        !aligned(expert_offsets, 4) || !aligned(peer_x_loc_q, 8) || !aligned(peer_scale_loc, 8) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    uint32_t *status = (uint32_t *)((char *)ws + L.status);
    cudaError_t e = launch_ep_direct_put(*s, G, x_q, topk_idx, dest_row, expert_offsets, peer_x_loc_q, ep_ws, status,
                                         sms, (cudaStream_t)stream, x_scale, peer_scale_loc);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_dispatch_fp8");
}

moe_status moe_ep_direct_down_return_fp8(const moe_shape *s, int32_t G, const void *h_q, const float *h_scale,
                                         const void *wd_q, const float *wd_scale, void *ws_loc, void *ep_ws,
                                         void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(h_q, 16) || !aligned(h_scale, 4) || !aligned(wd_q, 16) || !aligned(wd_scale, 4) ||
        !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws_loc)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const moe_shape l = ep_direct_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    cudaError_t e = launch_grouped_gemm_fp8(1, l, h_q, h_scale, wd_q, wd_scale, wd_q, wd_scale, nullptr, Lloc, ws_loc,
                                            g_timeout_ns.load(), sms, (cudaStream_t)stream, nullptr, nullptr,
                                            ep_direct_row_addr(ep_ws, *s, G));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_down_return_fp8");
}

moe_status moe_ep_direct_quantize_h(const moe_shape *s, int32_t G, const void *h_loc, void *h_q, float *h_scale,
                                    void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (!aligned(h_loc, 16) || !aligned(h_q, 16) || !aligned(h_scale, 4) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    cudaError_t e = launch_quant_rows_counted(h_loc, s->F, (int)ep_direct_local_rows(*s, G),
                                              ep_direct_local_total(ep_ws, *s, G), h_q, h_scale, sms,
                                              (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_quantize_h");
}

moe_status moe_ep_direct_plan_dispatch(const moe_shape *s, int32_t G, int32_t rank, const int32_t *cnt_all,
                                       const void *peer_y, const void *x, const float *x_scale,
                                       const int32_t *topk_idx, const int32_t *dest_row, const int32_t *expert_offsets,
                                       const void *peer_x_loc, const void *peer_scale_loc, void *ws, void *ws_loc,
                                       void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (rank < 0 || rank >= G) return MOE_ERR_INVALID_ARG;
    if (!aligned(cnt_all, 4) || (peer_y && !aligned(peer_y, 8)) || !aligned(x, 16) || !aligned(topk_idx, 4) ||
        !aligned(dest_row, 4) || !aligned(expert_offsets, 4) || !aligned(peer_x_loc, 8) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if (x_scale && (!aligned(x_scale, 4) || !aligned(peer_scale_loc, 8))) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK || (st = check_ws(ws_loc)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    const moe_shape l = ep_direct_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    uint32_t *status = (uint32_t *)((char *)ws + L.status);
    cudaError_t e = launch_ep_direct_plan_put(*s, G, rank, cnt_all, peer_y, Lloc, ws_loc, x, topk_idx, dest_row,
                                              expert_offsets, peer_x_loc, ep_ws, status, sms, (cudaStream_t)stream,
                                              x_scale, x_scale ? peer_scale_loc : nullptr, false);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_plan_dispatch");
}

moe_status moe_ep_direct_plan_dispatch_quantize(const moe_shape *s, int32_t G, int32_t rank, const int32_t *cnt_all,
                                                const void *peer_y, const void *x, const int32_t *topk_idx,
                                                const int32_t *dest_row, const int32_t *expert_offsets,
                                                const void *peer_x_loc_q, const void *peer_scale_loc, void *ws,
                                                void *ws_loc, void *ep_ws, void *stream) {
    moe_status st = check_ep_direct(s, G);
    if (st != MOE_OK) return st;
    if (rank < 0 || rank >= G) return MOE_ERR_INVALID_ARG;
    if (!aligned(cnt_all, 4) || (peer_y && !aligned(peer_y, 8)) || !aligned(x, 16) || !aligned(topk_idx, 4) ||
        !aligned(dest_row, 4) || !aligned(expert_offsets, 4) || !aligned(peer_x_loc_q, 8) ||
        !aligned(peer_scale_loc, 8) || !aligned(ep_ws, 16))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(ws)) != MOE_OK || (st = check_ws(ws_loc)) != MOE_OK) return st;
    int sms = 0;
    if ((st = device_info(&sms)) != MOE_OK) return st;
    const WsLayout L = layout_of(s);
    const moe_shape l = ep_direct_local(s, G);
    const WsLayout Lloc = layout_of(&l);
    uint32_t *status = (uint32_t *)((char *)ws + L.status);
    cudaError_t e = launch_ep_direct_plan_put(*s, G, rank, cnt_all, peer_y, Lloc, ws_loc, x, topk_idx, dest_row,
                                              expert_offsets, peer_x_loc_q, ep_ws, status, sms, (cudaStream_t)stream,
                                              nullptr, peer_scale_loc, true);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_direct_plan_dispatch_quantize");
}

