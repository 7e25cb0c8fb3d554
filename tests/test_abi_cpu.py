"""The C-ABI library on the CPU: it loads, exports every symbol include/moe.h
declares, and answers the host-only queries (no kernel is launched here)."""
import ctypes
import os
import re

import pytest

import grouped_expert_gemm_router_b200 as moe
from grouped_expert_gemm_router_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(moe.ABI_FUNCTIONS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen("nm -D --defined-only %s" % moe.LIB_PATH).read()
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert set(declared_functions()) <= exported


def test_library_is_sm100a(lib):
    # The fat binary carries sm_100a code only (checked from the build flags, not by disassembly).
    assert "arch=compute_100a,code=sm_100a" in " ".join(moe_build.NVCC_FLAGS)
    assert lib.moe_version() == 100


def test_permuted_rows_and_workspace(lib):
    s = moe.make_shape(512, 4096, 14336, 8, 2)
    assert moe.moe_permuted_rows(s) == 1024
    s = moe.make_shape(128, 2048, 1408, 64, 6, C=16, capacity=True)
    assert moe.moe_permuted_rows(s) == 64 * 16 + 6 * 112
    L = moe.moe_workspace_layout(s)
    assert L.total == moe.moe_workspace_bytes(s) and L.total > 0
    assert L.status == 0 and L.tile_rows == 256
    assert L.tile_map % 256 == 0 and L.tile_map + 16 * L.max_tiles <= L.total
    # the tile bound: 2E + P/256 + 1
    assert L.max_tiles == 2 * 64 + (64 * 16 + 6 * 112) // 256 + 1


@pytest.mark.parametrize("bad", [
    dict(T=0), dict(H=96), dict(F=100), dict(E=0), dict(E=257), dict(k=0), dict(k=9), dict(C=-1),
])
def test_unsupported_shapes_rejected(lib, bad):
    d = dict(T=64, H=128, F=256, E=8, k=2, C=0)
    d.update(bad)
    s = moe.make_shape(**d)
    assert moe.moe_permuted_rows(s) == -1
    assert moe.moe_workspace_bytes(s) == 0
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_layout(s)


def test_unknown_flag_rejected(lib):
    s = moe.make_shape(64, 128, 256, 8, 2, flags=0x100)
    assert lib.moe_workspace_bytes(ctypes.byref(s)) == 0


def test_null_pointers_rejected_before_any_launch(lib):
    # Argument validation happens on the host before any CUDA call.
    s = moe.make_shape(64, 128, 256, 8, 2)
    rc = lib.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None)
    assert rc == 1  # MOE_ERR_INVALID_ARG
    rc = lib.moe_combine(ctypes.byref(s), None, None, None, None, None)
    assert rc == 1
    rc = lib.moe_forward(ctypes.byref(s), None, None, None)
    assert rc == 1
    assert lib.moe_status_string(2) == b"unsupported shape"


def _pack_expert(seg, tile_rows=256):
    """Python restatement of the tile packing rule (for the bound test)."""
    tiles, used, pieces = 0, 0, 0
    for start, n in seg:
        while n > 0:
            if used == tile_rows or pieces == 2:
                tiles += 1
                used, pieces = 0, 0
            take = min(n, tile_rows - used)
            pieces += 1
            used += (take + 15) // 16 * 16
            n -= take
    return tiles + (1 if pieces else 0)


def test_tile_bound_holds_for_adversarial_counts():
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(300):
        E = int(rng.integers(1, 65))
        T = int(rng.integers(1, 3000))
        k = int(rng.integers(1, E + 1))
        C = int(rng.integers(0, 300))
        # counts with n_e <= T and sum = T*k, skewed
        n = np.zeros(E, int)
        left = T * k
        for e in rng.permutation(E):
            take = min(T, left) if rng.random() < 0.5 else min(T, left, int(rng.integers(0, T + 1)))
            n[e] = take
            left -= take
        n[np.argmin(n)] += left if left <= T - n.min() else 0
        for capped in (False, True):
            P = E * C + k * max(0, T - C) if capped else T * k
            tiles = 0
            for e in range(E):
                if n[e] == 0:
                    continue
                if capped:
                    cap = min(n[e], C)
                    tiles += _pack_expert([(0, cap), (0, n[e] - cap)])
                else:
                    tiles += _pack_expert([(0, n[e])])
            assert tiles <= 2 * E + P // 256 + 1


def test_static_dispatch_refuses_the_scan_stall_hook(lib):
    # the no-workspace dispatch has no status word to report the stalled
    # look-back through, so it refuses the test hook before any CUDA call
    s = moe.make_shape(64, 128, 256, 8, 2, flags=moe.MOE_FLAG_TEST_STALL_SCAN)
    rc = lib.moe_permute_static(ctypes.byref(s), None, None, None, None, None, None, None, None)
    assert rc == 1  # MOE_ERR_INVALID_ARG


def test_test_hook_flags_are_known(lib):
    for f in (moe.MOE_FLAG_TEST_STALL_SCAN, moe.MOE_FLAG_TEST_STALL_GEMM):
        s = moe.make_shape(64, 128, 256, 8, 2, flags=f)
        assert lib.moe_workspace_bytes(ctypes.byref(s)) > 0


def test_fp8_weight_codes_plain_follows_the_tile_layout():
    """The host view of the tile-blocked fp8 weight codes: the code of expert
    e, column n, index k sits at the byte the header gives."""
    import numpy as np
    E, N, K = 2, 256, 384
    plain = np.random.default_rng(0).integers(0, 256, (E, N, K)).astype(np.uint8)
    e, n, k = np.meshgrid(np.arange(E), np.arange(N), np.arange(K), indexing="ij")
    off = ((e * (N // 128) + n // 128) * (K // 128) + k // 128) * 16384 + (n % 128) * 128 + k % 128
    blocked = np.zeros(E * N * K, np.uint8)
    blocked[off.reshape(-1)] = plain.reshape(-1)
    assert np.array_equal(moe.fp8_weight_codes_plain(blocked, N, K), plain)

