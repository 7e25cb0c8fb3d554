"""moe_permute_static, the dispatch entry point for callers that cannot
allocate device memory (for example a plug-in whose host application owns all
device memory).

It must give exactly what moe_permute gives with a caller-allocated
workspace, call after call: the second call below routes different tokens
over the same shared scratch array, so left-over state from the first call
would show up as a mismatch.  This file is collected last so that a failure
here cannot stop the rest of the suite; it passes alone or after the rest."""
import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import DeviceLayer, shape_of

pytestmark = pytest.mark.gpu

FIELDS = ("expert_counts", "expert_offsets", "dest_row", "src_token", "x_perm")


def _route(dl, shape):
    b = dl.bufs(shape)
    moe.moe_route(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"], b["ws"])
    return b


def _static_outputs(shape, b):
    P = moe.moe_permuted_rows(shape)
    o = dict(expert_counts=torch.empty_like(b["expert_counts"]), expert_offsets=torch.empty_like(b["expert_offsets"]),
             dest_row=torch.empty_like(b["dest_row"]), src_token=torch.full((P,), 7, dtype=torch.int32, device="cuda"),
             x_perm=torch.empty_like(b["x_perm"]))
    moe.moe_permute_static(shape, b["x"], b["topk_idx"], o["expert_counts"], o["expert_offsets"], o["src_token"],
                           o["dest_row"], o["x_perm"])
    return o


def _compare(shape, b, o):
    torch.cuda.synchronize()
    filled = b["src_token"] >= 0
    for f in FIELDS:
        ref, got = b[f], o[f]
        if f in ("x_perm",):
            ref, got = ref[filled], got[filled]
        if f == "src_token" and not (shape.flags & moe.MOE_FLAG_CAPACITY):
            ref, got = ref[filled], got[filled]
        assert torch.equal(ref.view(torch.int16) if ref.dtype == torch.bfloat16 else ref,
                           got.view(torch.int16) if got.dtype == torch.bfloat16 else got), f


@pytest.mark.parametrize("first,second", [
    (synth.LayerConfig("a", 700, 256, 128, 8, 2, alpha=1.0, seed=21),
     synth.LayerConfig("b", 2100, 128, 128, 16, 3, alpha=0.3, seed=22)),
    (synth.LayerConfig("c", 128, 256, 128, 64, 6, C=16, alpha=0.25634765625, seed=23),
     synth.LayerConfig("d", 300, 256, 128, 64, 6, C=4, alpha=1.5, seed=24)),
])
def test_static_scratch_matches_workspace_form(first, second):
    for cfg in (first, second):
        L = synth.make_layer(cfg, with_experts=False)
        L.w_gate = L.w_up = L.w_down = np.zeros((cfg.E, 1, 1), np.uint16)
        dl = DeviceLayer(L)
        shape = shape_of(cfg)
        b = _route(dl, shape)
        moe.moe_permute(shape, b["x"], b["topk_idx"], b["expert_counts"], b["expert_offsets"], b["src_token"],
                        b["dest_row"], b["x_perm"], b["ws"])
        o = _static_outputs(shape, b)
        _compare(shape, b, o)


def test_static_scratch_rejects_oversized_shape():
    # 2^20 routed pairs over 256 experts need more scratch than the static area holds
    shape = moe.make_shape(1 << 17, 128, 128, 256, 8)
    lay = moe.moe_workspace_layout(shape)
    assert lay.tile_map > moe.MOE_STATIC_WS_BYTES  # the dispatch part alone is too big
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError, match="static area"):
        moe.moe_permute_static(shape, dummy, dummy, dummy, dummy, dummy, dummy, dummy)
