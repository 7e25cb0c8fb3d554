"""Python handle on the CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  The CUDA library never imports,
links or calls it, and it shares no code with the CUDA library.

The oracle is compiled with ``gcc -O2`` (no fast-math, no OpenMP, no SIMD
intrinsics) and runs single-threaded.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

EXPERT_SWIGLU, EXPERT_IDENTITY = 0, 1


def build(force: bool = False, src: str | None = None, out: str | None = None) -> str:
    """Compile the oracle.  ``src``/``out`` let a test compile a modified copy."""
    src = src or os.path.join(_HERE, "oracle.c")
    out = out or _SO
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def _declare(lib):
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.oracle_router_logits.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_topk_softmax.argtypes = [i32, i32, i32, vp, vp, vp]
    lib.oracle_topk_softmax.restype = i32
    lib.oracle_permuted_rows.argtypes = [i32, i32, i32, i32, i32]
    lib.oracle_permuted_rows.restype = i64
    lib.oracle_dispatch.argtypes = [i32, i32, i32, i32, i32] + [vp] * 8
    lib.oracle_dispatch.restype = i32
    lib.oracle_swiglu_row.argtypes = [i32, i32, vp, vp, vp, vp]
    lib.oracle_down_row.argtypes = [i32, i32, vp, vp, vp]
    lib.oracle_combine.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_forward.argtypes = [i32] * 8 + [vp] * 21
    lib.oracle_forward.restype = i32
    lib.oracle_token_outputs.argtypes = [i32, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_fp8_scale.argtypes = [ctypes.c_float]
    lib.oracle_fp8_scale.restype = ctypes.c_float
    lib.oracle_quantize_rows.argtypes = [i32, i32, vp, vp, vp]
    lib.oracle_quantize_weights.argtypes = [i32, i32, i32, vp, vp, vp]
    lib.oracle_dequantize.argtypes = [i64, i32, vp, vp, vp]
    return lib


def load(path: str | None = None):
    """Load the oracle library (a fresh handle when ``path`` is given)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


class Oracle:
    """numpy-level wrappers; arrays of bf16 are uint16 bit patterns."""

    def __init__(self, lib=None):
        self.lib = lib or load()

    def permuted_rows(self, T, E, k, C=0, capped=False) -> int:
        return int(self.lib.oracle_permuted_rows(T, E, k, C, int(bool(capped))))

    def router_logits(self, x, w_router, bias=None):
        x = _c(x, np.uint16)
        wr = _c(w_router, np.float32)
        b = _c(bias, np.float32)
        T, H = x.shape
        E = wr.shape[1]
        logits = np.empty((T, E), dtype=np.float32)
        self.lib.oracle_router_logits(T, H, E, _p(x), _p(wr), _p(b), _p(logits))
        return logits

    def topk_softmax(self, logits, k):
        logits = _c(logits, np.float32)
        T, E = logits.shape
        idx = np.empty((T, k), dtype=np.int32)
        w = np.empty((T, k), dtype=np.float32)
        nan = self.lib.oracle_topk_softmax(T, E, k, _p(logits), _p(idx), _p(w))
        return idx, w, int(nan)

    def dispatch(self, idx, E, C=0, capped=False):
        idx = _c(idx, np.int32)
        T, k = idx.shape
        P = self.permuted_rows(T, E, k, C, capped)
        counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        cap_cnt = np.empty(E, np.int32)
        spill_cnt = np.empty(E, np.int32)
        spill_off = np.empty(E + 1, np.int32)
        dest_row = np.empty(T * k, np.int32)
        src_token = np.empty(max(P, 1), np.int32)
        rc = self.lib.oracle_dispatch(T, E, k, C, int(bool(capped)), _p(idx), _p(counts), _p(offsets), _p(cap_cnt),
                                      _p(spill_cnt), _p(spill_off), _p(dest_row), _p(src_token))
        if rc != 0:
            raise ValueError("expert index out of range")
        return dict(counts=counts, offsets=offsets, cap_cnt=cap_cnt, spill_cnt=spill_cnt, spill_off=spill_off,
                    dest_row=dest_row, src_token=src_token[:P], P=P)

    def swiglu_row(self, xrow, wg_e, wu_e):
        xrow = _c(xrow, np.uint16)
        wg_e = _c(wg_e, np.uint16)
        wu_e = _c(wu_e, np.uint16)
        H, F = wg_e.shape
        h = np.empty(F, np.uint16)
        self.lib.oracle_swiglu_row(H, F, _p(xrow), _p(wg_e), _p(wu_e), _p(h))
        return h

    def down_row(self, hrow, wd_e):
        hrow = _c(hrow, np.uint16)
        wd_e = _c(wd_e, np.uint16)
        F, H = wd_e.shape
        y = np.empty(H, np.uint16)
        self.lib.oracle_down_row(H, F, _p(hrow), _p(wd_e), _p(y))
        return y

    def combine(self, y, dest_row, w):
        y = _c(y, np.uint16)
        w = _c(w, np.float32)
        T, k = w.shape
        H = y.shape[1]
        dest_row = _c(dest_row, np.int32)
        out = np.empty((T, H), np.uint16)
        self.lib.oracle_combine(T, H, k, _p(y), _p(dest_row), _p(w), _p(out))
        return out

    def forward(self, x, w_router, bias, w_gate, w_up, w_down, k, C=0, capped=False,
                expert=EXPERT_SWIGLU, w_in=None):
        x = _c(x, np.uint16)
        wr = _c(w_router, np.float32)
        b = _c(bias, np.float32)
        T, H = x.shape
        E = wr.shape[1]
        if expert == EXPERT_IDENTITY:
            F = 0
            wg = wu = wd = None
        else:
            wg, wu, wd = _c(w_gate, np.uint16), _c(w_up, np.uint16), _c(w_down, np.uint16)
            F = wg.shape[2]
        P = self.permuted_rows(T, E, k, C, capped)
        r = dict(
            logits=np.empty((T, E), np.float32), idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float32),
            counts=np.empty(E, np.int32), offsets=np.empty(E + 1, np.int32), cap_cnt=np.empty(E, np.int32),
            spill_cnt=np.empty(E, np.int32), spill_off=np.empty(E + 1, np.int32),
            dest_row=np.empty(T * k, np.int32), src_token=np.empty(max(P, 1), np.int32),
            x_perm=np.empty((max(P, 1), H), np.uint16), h=np.empty((max(P, 1), max(F, 1)), np.uint16),
            y=np.empty((max(P, 1), H), np.uint16), out=np.empty((T, H), np.uint16))
        w_in = _c(w_in, np.float32)
        rc = self.lib.oracle_forward(
            T, H, F, E, k, C, int(bool(capped)), expert, _p(x), _p(wr), _p(b), _p(wg), _p(wu), _p(wd), _p(w_in),
            _p(r["logits"]), _p(r["idx"]), _p(r["w"]), _p(r["counts"]), _p(r["offsets"]), _p(r["cap_cnt"]),
            _p(r["spill_cnt"]), _p(r["spill_off"]), _p(r["dest_row"]), _p(r["src_token"]), _p(r["x_perm"]),
            _p(r["h"]), _p(r["y"]), _p(r["out"]))
        if rc != 0:
            raise ValueError("expert index out of range")
        r["P"] = P
        for key in ("src_token", "x_perm", "h", "y"):
            r[key] = r[key][:P]
        if F == 0:
            r["h"] = r["h"][:, :0]
        return r

    def token_outputs(self, tokens, x, idx, w, w_gate, w_up, w_down):
        tokens = _c(tokens, np.int32)
        x = _c(x, np.uint16)
        idx = _c(idx, np.int32)
        w = _c(w, np.float32)
        H = x.shape[1]
        F = w_gate.shape[2]
        k = idx.shape[1]
        out = np.empty((len(tokens), H), np.uint16)
        self.lib.oracle_token_outputs(len(tokens), _p(tokens), H, F, k, _p(x), _p(idx), _p(w),
                                      _p(_c(w_gate, np.uint16)), _p(_c(w_up, np.uint16)),
                                      _p(_c(w_down, np.uint16)), _p(out))
        return out

    # ---- fp8 (e4m3) variant: codes are uint8, scales float32 powers of two ----

    def e4m3_decode(self, q: int) -> float:
        return float(self.lib.oracle_e4m3_decode(int(q)))

    def e4m3_encode(self, v: float) -> int:
        return int(self.lib.oracle_e4m3_encode(float(v)))

    def fp8_scale(self, amax: float) -> float:
        return float(self.lib.oracle_fp8_scale(float(amax)))

    def quantize_rows(self, v):
        """bf16 [rows, n] -> (codes [rows, n] uint8, scales [rows] float32)."""
        v = _c(v, np.uint16)
        rows, n = v.shape
        q = np.empty((rows, n), np.uint8)
        s = np.empty(rows, np.float32)
        self.lib.oracle_quantize_rows(rows, n, _p(v), _p(q), _p(s))
        return q, s

    def quantize_weights(self, w):
        """bf16 [E, K, N] -> (codes [E, N, K] uint8, scales [E, N] float32)."""
        w = _c(w, np.uint16)
        E, K, N = w.shape
        q = np.empty((E, N, K), np.uint8)
        s = np.empty((E, N), np.float32)
        self.lib.oracle_quantize_weights(E, K, N, _p(w), _p(q), _p(s))
        return q, s

    def dequantize(self, q, scale):
        """codes with one scale per last-axis vector -> bf16 bits of the same shape."""
        q = _c(q, np.uint8)
        scale = _c(scale, np.float32)
        out = np.empty(q.shape, np.uint16)
        group = q.shape[-1] if q.ndim else 1
        self.lib.oracle_dequantize(q.size, group, _p(q), _p(scale), _p(out))
        return out

    def dequantize_weights(self, q, scale):
        """codes [E, N, K] + scales [E, N] -> bf16 weights [E, K, N] (the layout the
        bf16 expert functions take)."""
        return np.ascontiguousarray(self.dequantize(q, scale).transpose(0, 2, 1))
