"""Python binding of the B200 MoE-layer forward library (include/moe.h).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libmoe_b200.so``.  Functions carry the C names; tensors are torch CUDA
tensors (their ``data_ptr()`` is passed through), ``stream`` defaults to the
current torch stream.  There is no fallback: if the library is missing or the
device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_DEV_SCAN_TIMEOUT = 0x1
MOE_DEV_GEMM_TIMEOUT = 0x2
MOE_DEV_BAD_EXPERT = 0x4
MOE_DEV_NAN_LOGIT = 0x8
MOE_DEV_BAD_ROW = 0x10
MOE_FLAG_CAPACITY = 0x1
MOE_FLAG_LOGITS_IN = 0x2
MOE_FLAG_FUSED_COMBINE = 0x8
MOE_FLAG_TEST_STALL_SCAN = 0x40000000
MOE_FLAG_TEST_STALL_GEMM = 0x20000000
MOE_WEIGHTS_GATE_UP = 0
MOE_WEIGHTS_DOWN = 1
MOE_ROWS_X_PERM = 0
MOE_ROWS_TOKENS = 1
MOE_ROWS_H = 2

# Every symbol include/moe.h declares (the CPU tests check the library exports each).
ABI_FUNCTIONS = (
    "moe_permuted_rows", "moe_workspace_bytes", "moe_workspace_layout", "moe_workspace_init", "moe_route",
    "moe_permute", "moe_grouped_swiglu", "moe_grouped_down", "moe_combine", "moe_forward", "moe_read_status",
    "moe_set_wait_timeout_ns", "moe_status_string", "moe_last_error_string", "moe_version", "moe_permute_static",
    "moe_route_dispatch", "moe_gather", "moe_grouped_swiglu_gather", "moe_quantize_weights_fp8",
    "moe_quantize_rows_fp8", "moe_grouped_swiglu_fp8", "moe_grouped_down_fp8", "moe_forward_fp8",
    "moe_grouped_down_combine", "moe_grouped_down_fp8_combine", "moe_ep_overflow_rows", "moe_ep_workspace_bytes",
    "moe_ep_local_shape", "moe_ep_pack", "moe_ep_local_dispatch", "moe_ep_local_return", "moe_ep_unpack",
    "moe_ep_direct_local_rows", "moe_ep_direct_workspace_bytes", "moe_ep_direct_local_shape", "moe_ep_direct_plan",
    "moe_ep_direct_dispatch", "moe_ep_direct_return", "moe_ep_direct_down_return", "moe_ep_direct_dispatch_fp8",
    "moe_ep_direct_down_return_fp8", "moe_ep_direct_quantize_h", "moe_ep_direct_plan_dispatch",
    "moe_ep_direct_plan_dispatch_quantize", "moe_ep_unpack_combine", "moe_ep_gather_pack",
)
MOE_STATIC_WS_BYTES = 1 << 20


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("F", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("C", ctypes.c_int32), ("flags", ctypes.c_uint32)]

    def __repr__(self):
        return "MoeShape(T=%d, H=%d, F=%d, E=%d, k=%d, C=%d, flags=%#x)" % (
            self.T, self.H, self.F, self.E, self.k, self.C, self.flags)


class MoeForwardArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "x", "w_router", "bias", "w_gate", "w_up", "w_down", "logits", "topk_idx", "topk_w", "expert_counts",
        "expert_offsets", "src_token", "dest_row", "x_perm", "h", "y", "out")]


class MoeForwardFp8Args(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "x", "w_router", "bias", "wg_q", "wg_scale", "wu_q", "wu_scale", "wd_q", "wd_scale", "logits", "topk_idx",
        "topk_w", "expert_counts", "expert_offsets", "src_token", "dest_row", "x_q", "x_scale")] + [
        ("x_q_per_token", ctypes.c_int32)] + [(n, ctypes.c_void_p) for n in ("h", "h_q", "h_scale", "y", "out")]


class MoeWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total", "status", "num_tiles", "total_spill", "cap_cnt", "spill_cnt", "spill_off", "order",
        "grp_tile_start", "tile_map")] + [("max_tiles", ctypes.c_int32), ("tile_rows", ctypes.c_int32),
                                          ("row_cap", ctypes.c_size_t)]


class MoeError(RuntimeError):
    pass


_lib = None


def load_library(path: str = LIB_PATH):
    """Load (once) and declare the C ABI.  Raises if the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise MoeError("CUDA library %s is missing: build it with "
                       "`python -m grouped_expert_gemm_router_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, sp = ctypes.c_void_p, ctypes.POINTER(MoeShape)
    st = ctypes.c_int
    lib.moe_permuted_rows.argtypes = [sp]
    lib.moe_permuted_rows.restype = ctypes.c_int64
    lib.moe_workspace_bytes.argtypes = [sp]
    lib.moe_workspace_bytes.restype = ctypes.c_size_t
    lib.moe_workspace_layout.argtypes = [sp, ctypes.POINTER(MoeWsLayout)]
    lib.moe_workspace_layout.restype = st
    lib.moe_workspace_init.argtypes = [sp, vp, vp]
    lib.moe_workspace_init.restype = st
    lib.moe_route.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.moe_route.restype = st
    lib.moe_permute.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.moe_permute.restype = st
    lib.moe_route_dispatch.argtypes = [sp] + [vp] * 12
    lib.moe_route_dispatch.restype = st
    lib.moe_gather.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.moe_gather.restype = st
    lib.moe_grouped_swiglu_gather.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp]
    lib.moe_grouped_swiglu_gather.restype = st
    lib.moe_grouped_swiglu.argtypes = [sp, vp, vp, vp, vp, vp, vp]
    lib.moe_grouped_swiglu.restype = st
    lib.moe_grouped_down.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.moe_grouped_down.restype = st
    lib.moe_combine.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.moe_combine.restype = st
    lib.moe_forward.argtypes = [sp, ctypes.POINTER(MoeForwardArgs), vp, vp]
    lib.moe_forward.restype = st
    lib.moe_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    lib.moe_read_status.restype = st
    lib.moe_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.moe_set_wait_timeout_ns.restype = None
    lib.moe_status_string.argtypes = [st]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_last_error_string.argtypes = []
    lib.moe_last_error_string.restype = ctypes.c_char_p
    lib.moe_version.argtypes = []
    lib.moe_version.restype = ctypes.c_int32
    lib.moe_permute_static.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.moe_permute_static.restype = st
    lib.moe_quantize_weights_fp8.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp]
    lib.moe_quantize_weights_fp8.restype = st
    lib.moe_quantize_rows_fp8.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, vp, vp]
    lib.moe_quantize_rows_fp8.restype = st
    lib.moe_grouped_swiglu_fp8.argtypes = [sp] + [vp] * 10
    lib.moe_grouped_swiglu_fp8.restype = st
    lib.moe_grouped_down_fp8.argtypes = [sp] + [vp] * 7
    lib.moe_grouped_down_fp8.restype = st
    lib.moe_forward_fp8.argtypes = [sp, ctypes.POINTER(MoeForwardFp8Args), vp, vp]
    lib.moe_forward_fp8.restype = st
    lib.moe_grouped_down_combine.argtypes = [sp] + [vp] * 9
    lib.moe_grouped_down_combine.restype = st
    lib.moe_grouped_down_fp8_combine.argtypes = [sp] + [vp] * 11
    lib.moe_grouped_down_fp8_combine.restype = st
    i32 = ctypes.c_int32
    lib.moe_ep_overflow_rows.argtypes = [sp, i32]
    lib.moe_ep_overflow_rows.restype = ctypes.c_int64
    lib.moe_ep_workspace_bytes.argtypes = [sp, i32]
    lib.moe_ep_workspace_bytes.restype = ctypes.c_size_t
    lib.moe_ep_local_shape.argtypes = [sp, i32, sp]
    lib.moe_ep_local_shape.restype = st
    lib.moe_ep_pack.argtypes = [sp, i32] + [vp] * 6
    lib.moe_ep_pack.restype = st
    lib.moe_ep_local_dispatch.argtypes = [sp, i32] + [vp] * 7
    lib.moe_ep_local_dispatch.restype = st
    lib.moe_ep_local_return.argtypes = [sp, i32] + [vp] * 5
    lib.moe_ep_local_return.restype = st
    lib.moe_ep_unpack.argtypes = [sp, i32] + [vp] * 4
    lib.moe_ep_unpack.restype = st
    lib.moe_ep_unpack_combine.argtypes = [sp, i32] + [vp] * 7
    lib.moe_ep_unpack_combine.restype = st
    lib.moe_ep_gather_pack.argtypes = [sp, i32] + [vp] * 8
    lib.moe_ep_gather_pack.restype = st
    lib.moe_ep_direct_local_rows.argtypes = [sp, i32]
    lib.moe_ep_direct_local_rows.restype = ctypes.c_int64
    lib.moe_ep_direct_workspace_bytes.argtypes = [sp, i32]
    lib.moe_ep_direct_workspace_bytes.restype = ctypes.c_size_t
    lib.moe_ep_direct_local_shape.argtypes = [sp, i32, sp]
    lib.moe_ep_direct_local_shape.restype = st
    lib.moe_ep_direct_plan.argtypes = [sp, i32, i32] + [vp] * 5
    lib.moe_ep_direct_plan.restype = st
    lib.moe_ep_direct_dispatch.argtypes = [sp, i32] + [vp] * 8
    lib.moe_ep_direct_dispatch.restype = st
    lib.moe_ep_direct_return.argtypes = [sp, i32] + [vp] * 4
    lib.moe_ep_direct_return.restype = st
    lib.moe_ep_direct_down_return.argtypes = [sp, i32] + [vp] * 5
    lib.moe_ep_direct_down_return.restype = st
    lib.moe_ep_direct_dispatch_fp8.argtypes = [sp, i32] + [vp] * 10
    lib.moe_ep_direct_dispatch_fp8.restype = st
    lib.moe_ep_direct_down_return_fp8.argtypes = [sp, i32] + [vp] * 7
    lib.moe_ep_direct_down_return_fp8.restype = st
    lib.moe_ep_direct_quantize_h.argtypes = [sp, i32] + [vp] * 5
    lib.moe_ep_direct_quantize_h.restype = st
    lib.moe_ep_direct_plan_dispatch.argtypes = [sp, i32, i32] + [vp] * 13
    lib.moe_ep_direct_plan_dispatch.restype = st
    lib.moe_ep_direct_plan_dispatch_quantize.argtypes = [sp, i32, i32] + [vp] * 12
    lib.moe_ep_direct_plan_dispatch_quantize.restype = st
    _lib = lib
    return lib


def make_shape(T, H, F, E, k, C=0, capacity=False, logits_in=False, flags=0) -> MoeShape:
    f = flags | (MOE_FLAG_CAPACITY if capacity else 0) | (MOE_FLAG_LOGITS_IN if logits_in else 0)
    return MoeShape(T, H, F, E, k, C, f)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc, what):
    if rc != MOE_OK:
        lib = load_library()
        raise MoeError("%s failed: %s (%s)" % (what, lib.moe_status_string(rc).decode(),
                                               lib.moe_last_error_string().decode()))


def moe_permuted_rows(shape: MoeShape) -> int:
    return int(load_library().moe_permuted_rows(ctypes.byref(shape)))


def moe_workspace_bytes(shape: MoeShape) -> int:
    return int(load_library().moe_workspace_bytes(ctypes.byref(shape)))


def moe_workspace_layout(shape: MoeShape) -> MoeWsLayout:
    out = MoeWsLayout()
    _check(load_library().moe_workspace_layout(ctypes.byref(shape), ctypes.byref(out)), "moe_workspace_layout")
    return out


def moe_workspace_init(shape, ws, stream=None):
    _check(load_library().moe_workspace_init(ctypes.byref(shape), _ptr(ws), _stream(stream)), "moe_workspace_init")


def moe_route(shape, x, w_router, bias, logits, topk_idx, topk_w, ws, stream=None):
    _check(load_library().moe_route(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits),
                                    _ptr(topk_idx), _ptr(topk_w), _ptr(ws), _stream(stream)), "moe_route")


def moe_permute(shape, x, topk_idx, expert_counts, expert_offsets, src_token, dest_row, x_perm, ws, stream=None):
    _check(load_library().moe_permute(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(expert_counts),
                                      _ptr(expert_offsets), _ptr(src_token), _ptr(dest_row), _ptr(x_perm),
                                      _ptr(ws), _stream(stream)), "moe_permute")


def moe_route_dispatch(shape, x, w_router, bias, logits, topk_idx, topk_w, expert_counts, expert_offsets, src_token,
                       dest_row, ws, stream=None):
    _check(load_library().moe_route_dispatch(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits),
                                             _ptr(topk_idx), _ptr(topk_w), _ptr(expert_counts), _ptr(expert_offsets),
                                             _ptr(src_token), _ptr(dest_row), _ptr(ws), _stream(stream)),
           "moe_route_dispatch")


def moe_gather(shape, x, src_token, x_perm, ws, stream=None):
    _check(load_library().moe_gather(ctypes.byref(shape), _ptr(x), _ptr(src_token), _ptr(x_perm), _ptr(ws),
                                     _stream(stream)), "moe_gather")


def moe_grouped_swiglu_gather(shape, x, src_token, w_gate, w_up, h, ws, stream=None):
    _check(load_library().moe_grouped_swiglu_gather(ctypes.byref(shape), _ptr(x), _ptr(src_token), _ptr(w_gate),
                                                    _ptr(w_up), _ptr(h), _ptr(ws), _stream(stream)),
           "moe_grouped_swiglu_gather")


def moe_permute_static(shape, x, topk_idx, expert_counts, expert_offsets, src_token, dest_row, x_perm, stream=None):
    """moe_permute without a caller workspace, for callers that cannot
    allocate device memory: the scratch is a fixed array inside the library
    (MOE_STATIC_WS_BYTES).  Make the first call on a device before any stream
    capture; calls that overlap on the GPU race on the shared array."""
    _check(load_library().moe_permute_static(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(expert_counts),
                                             _ptr(expert_offsets), _ptr(src_token), _ptr(dest_row), _ptr(x_perm),
                                             _stream(stream)), "moe_permute_static")


def moe_grouped_swiglu(shape, x_perm, w_gate, w_up, h, ws, stream=None):
    _check(load_library().moe_grouped_swiglu(ctypes.byref(shape), _ptr(x_perm), _ptr(w_gate), _ptr(w_up), _ptr(h),
                                             _ptr(ws), _stream(stream)), "moe_grouped_swiglu")


def moe_grouped_down(shape, h, w_down, y, ws, stream=None):
    _check(load_library().moe_grouped_down(ctypes.byref(shape), _ptr(h), _ptr(w_down), _ptr(y), _ptr(ws),
                                           _stream(stream)), "moe_grouped_down")


def moe_grouped_down_combine(shape, h, w_down, src_token, dest_row, topk_w, y, out, ws, stream=None):
    _check(load_library().moe_grouped_down_combine(ctypes.byref(shape), _ptr(h), _ptr(w_down), _ptr(src_token),
                                                   _ptr(dest_row), _ptr(topk_w), _ptr(y), _ptr(out), _ptr(ws),
                                                   _stream(stream)), "moe_grouped_down_combine")


def moe_grouped_down_fp8_combine(shape, h_q, h_scale, wd_q, wd_scale, src_token, dest_row, topk_w, y, out, ws,
                                 stream=None):
    _check(load_library().moe_grouped_down_fp8_combine(ctypes.byref(shape), _ptr(h_q), _ptr(h_scale), _ptr(wd_q),
                                                       _ptr(wd_scale), _ptr(src_token), _ptr(dest_row), _ptr(topk_w),
                                                       _ptr(y), _ptr(out), _ptr(ws), _stream(stream)),
           "moe_grouped_down_fp8_combine")


def moe_combine(shape, y, dest_row, topk_w, out, stream=None):
    _check(load_library().moe_combine(ctypes.byref(shape), _ptr(y), _ptr(dest_row), _ptr(topk_w), _ptr(out),
                                      _stream(stream)), "moe_combine")


def forward_args(bufs: dict) -> MoeForwardArgs:
    a = MoeForwardArgs()
    for name, _ in MoeForwardArgs._fields_:
        setattr(a, name, _ptr(bufs.get(name)))
    return a


def moe_forward(shape, bufs: dict, ws, stream=None, args: MoeForwardArgs | None = None):
    """bufs: dict with the moe_forward_args field names -> tensors (or None)."""
    a = args if args is not None else forward_args(bufs)
    _check(load_library().moe_forward(ctypes.byref(shape), ctypes.byref(a), _ptr(ws), _stream(stream)), "moe_forward")


class ForwardGraph:
    """moe_forward on fixed buffers, captured once as a CUDA graph (its launch
    grid depends only on the shape, so one capture serves any inputs written
    into the same buffers); replay() enqueues the whole layer on a stream."""

    def __init__(self, shape, bufs: dict, ws, stream=None):
        import torch
        self.args = forward_args(bufs)
        self.keep = (bufs, ws)  # the graph holds their addresses
        moe_forward(shape, bufs, ws, stream, args=self.args)  # first launches outside the capture
        self.graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream() if stream is None else stream)
        with torch.cuda.graph(self.graph, stream=cap):
            moe_forward(shape, bufs, ws, cap, args=self.args)

    def replay(self, stream=None):
        import torch
        if stream is None:
            self.graph.replay()
        else:
            with torch.cuda.stream(stream):
                self.graph.replay()


def moe_read_status(ws, stream=None, clear=True) -> int:
    v = ctypes.c_uint32(0)
    _check(load_library().moe_read_status(_ptr(ws), _stream(stream), ctypes.byref(v), int(bool(clear))),
           "moe_read_status")
    return int(v.value)


def moe_set_wait_timeout_ns(ns: int) -> None:
    load_library().moe_set_wait_timeout_ns(int(ns))


def moe_version() -> int:
    return int(load_library().moe_version())


def alloc_buffers(shape: MoeShape, device="cuda"):
    """Allocate (with torch) every intermediate/output buffer of moe_forward
    and a zeroed workspace.  Returns a dict keyed like moe_forward_args plus
    'ws'."""
    import torch
    T, H, F, E, k = shape.T, shape.H, shape.F, shape.E, shape.k
    P = moe_permuted_rows(shape)
    if P < 0:
        raise MoeError("unsupported shape %r" % (shape,))
    dev = torch.device(device)
    b = dict(
        logits=torch.empty((T, E), dtype=torch.float32, device=dev),
        topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
        topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
        expert_counts=torch.empty((E,), dtype=torch.int32, device=dev),
        expert_offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
        src_token=torch.empty((P,), dtype=torch.int32, device=dev),
        dest_row=torch.empty((T * k,), dtype=torch.int32, device=dev),
        x_perm=torch.empty((P, H), dtype=torch.bfloat16, device=dev),
        h=torch.empty((P, F), dtype=torch.bfloat16, device=dev),
        y=torch.empty((P, H), dtype=torch.bfloat16, device=dev),
        out=torch.empty((T, H), dtype=torch.bfloat16, device=dev),
    )
    ws = torch.empty((moe_workspace_bytes(shape) + 255) // 256 * 256, dtype=torch.uint8, device=dev)
    moe_workspace_init(shape, ws)
    b["ws"] = ws
    return b


# ---------------------------------------------------------------- fp8 (e4m3) --

def moe_quantize_weights_fp8(shape, which, w, w_q, w_scale, stream=None):
    _check(load_library().moe_quantize_weights_fp8(ctypes.byref(shape), int(which), _ptr(w), _ptr(w_q), _ptr(w_scale),
                                                   _stream(stream)), "moe_quantize_weights_fp8")


def moe_quantize_rows_fp8(shape, which, src, src_token, q, scale, ws, stream=None):
    _check(load_library().moe_quantize_rows_fp8(ctypes.byref(shape), int(which), _ptr(src), _ptr(src_token), _ptr(q),
                                                _ptr(scale), _ptr(ws), _stream(stream)), "moe_quantize_rows_fp8")


def moe_grouped_swiglu_fp8(shape, x_q, x_scale, src_token, wg_q, wg_scale, wu_q, wu_scale, h, ws, stream=None):
    _check(load_library().moe_grouped_swiglu_fp8(ctypes.byref(shape), _ptr(x_q), _ptr(x_scale), _ptr(src_token),
                                                 _ptr(wg_q), _ptr(wg_scale), _ptr(wu_q), _ptr(wu_scale), _ptr(h),
                                                 _ptr(ws), _stream(stream)), "moe_grouped_swiglu_fp8")


def moe_grouped_down_fp8(shape, h_q, h_scale, wd_q, wd_scale, y, ws, stream=None):
    _check(load_library().moe_grouped_down_fp8(ctypes.byref(shape), _ptr(h_q), _ptr(h_scale), _ptr(wd_q),
                                               _ptr(wd_scale), _ptr(y), _ptr(ws), _stream(stream)),
           "moe_grouped_down_fp8")


def forward_fp8_args(bufs: dict, per_token=False) -> MoeForwardFp8Args:
    a = MoeForwardFp8Args()
    for name, _ in MoeForwardFp8Args._fields_:
        if name != "x_q_per_token":
            setattr(a, name, _ptr(bufs.get(name)))
    a.x_q_per_token = 1 if per_token else 0
    return a


def moe_forward_fp8(shape, bufs: dict, ws, stream=None, args: MoeForwardFp8Args | None = None, per_token=False):
    a = args if args is not None else forward_fp8_args(bufs, per_token)
    _check(load_library().moe_forward_fp8(ctypes.byref(shape), ctypes.byref(a), _ptr(ws), _stream(stream)),
           "moe_forward_fp8")


def alloc_fp8_buffers(shape: MoeShape, per_token=False, device="cuda"):
    """Device buffers of the fp8 layer that moe_forward's buffers do not hold:
    weight codes and scales, token-row codes and scales, h codes and scales."""
    import torch
    T, H, F, E = shape.T, shape.H, shape.F, shape.E
    P = moe_permuted_rows(shape)
    dev = torch.device(device)
    xr = T if per_token else P
    return dict(
        # weight codes tile-blocked (see fp8_weight_codes_plain): [E][N/128][K/128][128][128]
        wg_q=torch.empty((E, F, H), dtype=torch.uint8, device=dev),
        wg_scale=torch.empty((E, F), dtype=torch.float32, device=dev),
        wu_q=torch.empty((E, F, H), dtype=torch.uint8, device=dev),
        wu_scale=torch.empty((E, F), dtype=torch.float32, device=dev),
        wd_q=torch.empty((E, H, F), dtype=torch.uint8, device=dev),
        wd_scale=torch.empty((E, H), dtype=torch.float32, device=dev),
        x_q=torch.empty((xr, H), dtype=torch.uint8, device=dev),
        x_scale=torch.empty((xr,), dtype=torch.float32, device=dev),
        h_q=torch.empty((P, F), dtype=torch.uint8, device=dev),
        h_scale=torch.empty((P,), dtype=torch.float32, device=dev),
    )


def quantize_layer_weights_fp8(shape, bufs, stream=None):
    """Codes and scales of w_gate, w_up, w_down (bufs as alloc_buffers +
    alloc_fp8_buffers fill it)."""
    moe_quantize_weights_fp8(shape, MOE_WEIGHTS_GATE_UP, bufs["w_gate"], bufs["wg_q"], bufs["wg_scale"], stream)
    moe_quantize_weights_fp8(shape, MOE_WEIGHTS_GATE_UP, bufs["w_up"], bufs["wu_q"], bufs["wu_scale"], stream)
    moe_quantize_weights_fp8(shape, MOE_WEIGHTS_DOWN, bufs["w_down"], bufs["wd_q"], bufs["wd_scale"], stream)


# ---------------------------------------------------- expert-parallel dispatch --

def moe_ep_overflow_rows(shape, G) -> int:
    return int(load_library().moe_ep_overflow_rows(ctypes.byref(shape), int(G)))


def moe_ep_workspace_bytes(shape, G) -> int:
    return int(load_library().moe_ep_workspace_bytes(ctypes.byref(shape), int(G)))


def moe_ep_local_shape(shape, G) -> MoeShape:
    out = MoeShape()
    _check(load_library().moe_ep_local_shape(ctypes.byref(shape), int(G), ctypes.byref(out)), "moe_ep_local_shape")
    return out


def moe_ep_pack(shape, G, x_perm, ws, send_ovf, send_meta, ep_ws, stream=None):
    _check(load_library().moe_ep_pack(ctypes.byref(shape), int(G), _ptr(x_perm), _ptr(ws), _ptr(send_ovf),
                                      _ptr(send_meta), _ptr(ep_ws), _stream(stream)), "moe_ep_pack")


def moe_ep_local_dispatch(shape, G, recv_meta, recv_cap, recv_ovf, x_loc, ws_loc, ep_ws, stream=None):
    _check(load_library().moe_ep_local_dispatch(ctypes.byref(shape), int(G), _ptr(recv_meta), _ptr(recv_cap),
                                                _ptr(recv_ovf), _ptr(x_loc), _ptr(ws_loc), _ptr(ep_ws),
                                                _stream(stream)), "moe_ep_local_dispatch")


def moe_ep_local_return(shape, G, y_loc, back_cap, back_ovf, ep_ws, stream=None):
    _check(load_library().moe_ep_local_return(ctypes.byref(shape), int(G), _ptr(y_loc), _ptr(back_cap),
                                              _ptr(back_ovf), _ptr(ep_ws), _stream(stream)), "moe_ep_local_return")


def moe_ep_unpack(shape, G, recv_back_ovf, y, ep_ws, stream=None):
    _check(load_library().moe_ep_unpack(ctypes.byref(shape), int(G), _ptr(recv_back_ovf), _ptr(y), _ptr(ep_ws),
                                        _stream(stream)), "moe_ep_unpack")


def moe_ep_gather_pack(shape, G, x, src_token, x_perm, ws, send_ovf, send_meta, ep_ws, stream=None):
    """moe_gather + moe_ep_pack in one launch (overflow rows straight into
    the send slots)."""
    _check(load_library().moe_ep_gather_pack(ctypes.byref(shape), int(G), _ptr(x), _ptr(src_token), _ptr(x_perm),
                                              _ptr(ws), _ptr(send_ovf), _ptr(send_meta), _ptr(ep_ws),
                                              _stream(stream)), "moe_ep_gather_pack")


def moe_ep_unpack_combine(shape, G, recv_back_ovf, y, dest_row, topk_w, out, ep_ws, stream=None):
    """moe_ep_unpack + moe_combine in one launch (overflow results read from
    the return slots)."""
    _check(load_library().moe_ep_unpack_combine(ctypes.byref(shape), int(G), _ptr(recv_back_ovf), _ptr(y),
                                                 _ptr(dest_row), _ptr(topk_w), _ptr(out), _ptr(ep_ws),
                                                 _stream(stream)), "moe_ep_unpack_combine")


def moe_ep_direct_local_rows(shape, G) -> int:
    return int(load_library().moe_ep_direct_local_rows(ctypes.byref(shape), int(G)))


def moe_ep_direct_workspace_bytes(shape, G) -> int:
    return int(load_library().moe_ep_direct_workspace_bytes(ctypes.byref(shape), int(G)))


def moe_ep_direct_local_shape(shape, G) -> MoeShape:
    out = MoeShape()
    _check(load_library().moe_ep_direct_local_shape(ctypes.byref(shape), int(G), ctypes.byref(out)),
           "moe_ep_direct_local_shape")
    return out


def moe_ep_direct_plan(shape, G, rank, cnt_all, peer_y, ws_loc, ep_ws, stream=None):
    """peer_y: a device tensor of G int64 addresses, or None."""
    _check(load_library().moe_ep_direct_plan(ctypes.byref(shape), int(G), int(rank), _ptr(cnt_all), _ptr(peer_y),
                                             _ptr(ws_loc), _ptr(ep_ws), _stream(stream)), "moe_ep_direct_plan")


def moe_ep_direct_dispatch(shape, G, x, topk_idx, dest_row, expert_offsets, peer_x_loc, ws, ep_ws, stream=None):
    """peer_x_loc: a device tensor of G int64 addresses (rank d's x_loc)."""
    _check(load_library().moe_ep_direct_dispatch(ctypes.byref(shape), int(G), _ptr(x), _ptr(topk_idx),
                                                 _ptr(dest_row), _ptr(expert_offsets), _ptr(peer_x_loc), _ptr(ws),
                                                 _ptr(ep_ws), _stream(stream)), "moe_ep_direct_dispatch")


def moe_ep_direct_return(shape, G, y_loc, peer_y, ep_ws, stream=None):
    """peer_y: a device tensor of G int64 addresses (rank s's y)."""
    _check(load_library().moe_ep_direct_return(ctypes.byref(shape), int(G), _ptr(y_loc), _ptr(peer_y), _ptr(ep_ws),
                                                _stream(stream)), "moe_ep_direct_return")


def moe_ep_direct_down_return(shape, G, h_loc, w_down, ws_loc, ep_ws, stream=None):
    _check(load_library().moe_ep_direct_down_return(ctypes.byref(shape), int(G), _ptr(h_loc), _ptr(w_down),
                                                    _ptr(ws_loc), _ptr(ep_ws), _stream(stream)),
           "moe_ep_direct_down_return")


def fp8_weight_codes_plain(q, N, K):
    """Host-side view of expert weight codes as moe_quantize_weights_fp8 leaves
    them (tile-blocked: tiles of 128 output columns x 128 K, each 16 KB
    contiguous, K-major inside) as a plain [E, N, K] numpy array (code of
    expert e, output column n, reduction index k).  q: a numpy array or CPU
    tensor holding the codes of one or more whole experts."""
    import numpy as np
    a = np.asarray(q).reshape(-1, N // 128, K // 128, 128, 128)
    return np.ascontiguousarray(a.transpose(0, 1, 3, 2, 4)).reshape(-1, N, K)


def moe_ep_direct_dispatch_fp8(shape, G, x_q, x_scale, topk_idx, dest_row, expert_offsets, peer_x_loc_q,
                               peer_scale_loc, ws, ep_ws, stream=None):
    _check(load_library().moe_ep_direct_dispatch_fp8(ctypes.byref(shape), int(G), _ptr(x_q), _ptr(x_scale),
                                                     _ptr(topk_idx), _ptr(dest_row), _ptr(expert_offsets),
                                                     _ptr(peer_x_loc_q), _ptr(peer_scale_loc), _ptr(ws), _ptr(ep_ws),
                                                     _stream(stream)), "moe_ep_direct_dispatch_fp8")


def moe_ep_direct_down_return_fp8(shape, G, h_q, h_scale, wd_q, wd_scale, ws_loc, ep_ws, stream=None):
    _check(load_library().moe_ep_direct_down_return_fp8(ctypes.byref(shape), int(G), _ptr(h_q), _ptr(h_scale),
                                                        _ptr(wd_q), _ptr(wd_scale), _ptr(ws_loc), _ptr(ep_ws),
                                                        _stream(stream)), "moe_ep_direct_down_return_fp8")


def moe_ep_direct_quantize_h(shape, G, h_loc, h_q, h_scale, ep_ws, stream=None):
    _check(load_library().moe_ep_direct_quantize_h(ctypes.byref(shape), int(G), _ptr(h_loc), _ptr(h_q),
                                                   _ptr(h_scale), _ptr(ep_ws), _stream(stream)),
           "moe_ep_direct_quantize_h")


def moe_ep_direct_plan_dispatch(shape, G, rank, cnt_all, peer_y, x, x_scale, topk_idx, dest_row, expert_offsets,
                                peer_x_loc, peer_scale_loc, ws, ws_loc, ep_ws, stream=None):
    """x_scale None: bf16 rows; else e4m3 code rows with their scales."""
    _check(load_library().moe_ep_direct_plan_dispatch(
        ctypes.byref(shape), int(G), int(rank), _ptr(cnt_all), _ptr(peer_y), _ptr(x), _ptr(x_scale), _ptr(topk_idx),
        _ptr(dest_row), _ptr(expert_offsets), _ptr(peer_x_loc), _ptr(peer_scale_loc), _ptr(ws), _ptr(ws_loc),
        _ptr(ep_ws), _stream(stream)), "moe_ep_direct_plan_dispatch")


def moe_ep_direct_plan_dispatch_quantize(shape, G, rank, cnt_all, peer_y, x, topk_idx, dest_row, expert_offsets,
                                         peer_x_loc_q, peer_scale_loc, ws, ws_loc, ep_ws, stream=None):
    """x: bf16 token rows, quantized to e4m3 rows on the way to the owners."""
    _check(load_library().moe_ep_direct_plan_dispatch_quantize(
        ctypes.byref(shape), int(G), int(rank), _ptr(cnt_all), _ptr(peer_y), _ptr(x), _ptr(topk_idx), _ptr(dest_row),
        _ptr(expert_offsets), _ptr(peer_x_loc_q), _ptr(peer_scale_loc), _ptr(ws), _ptr(ws_loc), _ptr(ep_ws),
        _stream(stream)), "moe_ep_direct_plan_dispatch_quantize")

