// moe_permute_static: the dispatch step (histogram, scan, stable permutation,
// gather) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: a plug-in whose host
// application owns every device allocation and hands it only the tensors it
// works on, for instance.  Such a caller can
// still provide its inputs and outputs, but not the scratch workspace that
// moe_permute needs.  This entry point takes its scratch from a fixed-size
// array compiled into the library instead.
//
// The array is a file-scope __device__ object of kStaticWsBytes bytes: every
// GPU that loads the library holds it until the process exits.  Host code
// cannot use the array's name as a device address (it names a host-side
// stand-in), so the first call on each device, with that device current,
// looks its address up with cudaGetSymbolAddress and zero-fills it; later
// calls reuse the cached address.  The cache is keyed by the device's current
// context, so a context that was torn down and recreated (cudaDeviceReset)
// gets a fresh look-up and zero-fill instead of a stale address.  Every call
// shares the array and leaves its contents behind, so each call clears what
// must start at zero (the look-back flags and block ticket) before its
// kernels run.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace moe {
cudaError_t launch_permute(const moe_shape &s, const void *x, const int32_t *topk_idx, int32_t *counts,
                           int32_t *offsets, int32_t *src_token, int32_t *dest_row, void *x_perm, const WsLayout &L,
                           void *ws, uint64_t timeout_ns, int num_sms, cudaStream_t stream);
}  // namespace moe

namespace {

constexpr size_t kStaticWsBytes = MOE_STATIC_WS_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_static_ptr[kMaxDevices] = {nullptr};
void *g_static_ctx[kMaxDevices] = {nullptr};  // context the cached address belongs to

// The current context of the calling thread (a CUcontext), through the
// driver entry point, so the library needs no link-time driver dependency.
void *current_context() {
    using Fn = int (*)(void **);
    static Fn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<Fn>(p);
        tried = true;
    }
    void *ctx = nullptr;
    if (fn && fn(&ctx) != 0) ctx = nullptr;
    return ctx;
}

// Device address of g_static_ws on the current device (set-up on the first
// use in each context: look-up and zero-fill).
cudaError_t static_ws_address(int dev, cudaStream_t stream, void **out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    void *ctx = current_context();
    if (g_static_ptr[dev] == nullptr || g_static_ctx[dev] != ctx) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(p, 0, kStaticWsBytes, stream);
        if (e != cudaSuccess) return e;
        g_static_ptr[dev] = p;
        g_static_ctx[dev] = ctx;
    }
    *out = g_static_ptr[dev];
    return cudaSuccess;
}

}  // namespace

// Declared in moe_abi.cu: shared validation helpers.
moe_status moe_internal_check_shape(const moe_shape *s);
moe_status moe_internal_device_info(int *num_sms);
moe_status moe_internal_cuda_fail(cudaError_t e, const char *where);
void moe_internal_set_error(const char *msg);
uint64_t moe_internal_timeout_ns();

extern "C" MOE_API moe_status moe_permute_static(const moe_shape *s, const void *x, const int32_t *topk_idx,
                                                 int32_t *expert_counts, int32_t *expert_offsets,
                                                 int32_t *src_token, int32_t *dest_row, void *x_perm,
                                                 void *stream) {
    moe_status st = moe_internal_check_shape(s);
    if (st != MOE_OK) return st;
    // The test hook that stalls the histogram's look-back would leave
    // outputs this entry point has no way to flag: refused here.
    if (s->flags & MOE_FLAG_TEST_STALL_SCAN) return MOE_ERR_INVALID_ARG;
    auto al = [](const void *p, uintptr_t a) { return p != nullptr && ((uintptr_t)p % a) == 0; };
    if (!al(x, 16) || !al(x_perm, 16) || !al(topk_idx, 4) || !al(expert_counts, 4) || !al(expert_offsets, 4) ||
        !al(src_token, 4) || !al(dest_row, 4))
        return MOE_ERR_INVALID_ARG;
    const moe::WsLayout L = moe::ws_layout(s->T, s->H, s->E, s->k, s->C, (s->flags & MOE_FLAG_CAPACITY) != 0);
    // The dispatch uses the workspace up to the GEMM's and the router's buffers, which come last.
    const size_t need = L.dispatch_end;
    if (need > kStaticWsBytes) {
        char msg[160];
        std::snprintf(msg, sizeof(msg), "moe_permute_static: shape needs %zu bytes of scratch, the static area holds %zu",
                      need, kStaticWsBytes);
        moe_internal_set_error(msg);
        return MOE_ERR_WORKSPACE;
    }
    int sms = 0;
    if ((st = moe_internal_device_info(&sms)) != MOE_OK) return st;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moe_internal_cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
    void *ws = nullptr;
    e = static_ws_address(dev, (cudaStream_t)stream, &ws);
    if (e != cudaSuccess) return moe_internal_cuda_fail(e, "moe_permute_static set-up");
    e = moe::launch_permute(*s, x, topk_idx, expert_counts, expert_offsets, src_token, dest_row, x_perm, L, ws,
                            moe_internal_timeout_ns(), sms, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : moe_internal_cuda_fail(e, "moe_permute_static");
}
