"""Router logits on the tensor cores (batches of >= 2048 tokens): the exact
three-way bf16 split of W_r must give logits within the fp32 tolerance of the
oracle, and the top-k on those logits must match the oracle's bit for bit."""
import numpy as np
import pytest

import synth
from gpu_util import LOGIT_TOL, WEIGHT_TOL, DeviceLayer, host, run_steps, shape_of, assert_close_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H,E,k,alpha", [
    (2048, 256, 8, 2, 0.0),      # one accumulator, plane padded 8 -> 64 columns
    (2100, 384, 128, 8, 1.0),    # ragged last token block, full 128-expert accumulator
    (4096, 128, 200, 6, 2.0),    # two accumulators (experts 128..199), padded planes
])
def test_tensor_core_router(orc, T, H, E, k, alpha):
    cfg = synth.LayerConfig("t", T, H, 128, E, k, alpha=alpha, seed=31)
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    r = host(run_steps(DeviceLayer(L), shape), shape)
    assert r["status"] == 0, hex(r["status"])
    ref = orc.router_logits(L.x, L.w_router, L.bias)
    err = np.abs(r["logits"] - ref) / np.maximum(1.0, np.abs(ref))
    assert err.max() <= LOGIT_TOL, err.max()
    idx, w, _ = orc.topk_softmax(r["logits"], k)
    assert np.array_equal(r["topk_idx"], idx)
    assert np.max(np.abs(r["topk_w"] - w)) <= WEIGHT_TOL
    # the rest of the layer on a few tokens
    tk = np.array([0, T // 2, T - 1], np.int32)
    out_ref = orc.token_outputs(tk, L.x, idx, w, L.w_gate, L.w_up, L.w_down)
    assert_close_bf16(r["out"][tk], out_ref, "out")
