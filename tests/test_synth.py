"""The seeded input generator: determinism, distribution and thread independence."""
import math

import numpy as np

import synth


def test_counter_based_equals_sequential_splitmix():
    lib = synth._load()
    key = lib.synth_stream_key(0, 3)
    # sequential SplitMix64 seeded with `key`: state += gamma, then mix
    state, seq = key, []
    for _ in range(5):
        state = (state + 0x9E3779B97F4A7C15) & (2 ** 64 - 1)
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2 ** 64 - 1)
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2 ** 64 - 1)
        seq.append(z ^ (z >> 31))
    assert [lib.synth_draw(key, i) for i in range(5)] == seq


def test_thread_count_does_not_change_values():
    n = 300_001
    a = np.empty(n, np.uint16)
    b = np.empty(n, np.uint16)
    synth.fill_bf16_normal(a.ctypes.data, n, 0, 5, 0.02, nthreads=1)
    synth.fill_bf16_normal(b.ctypes.data, n, 0, 5, 0.02, nthreads=7)
    assert np.array_equal(a, b)


def test_normal_moments():
    z = synth.f32_normal((1_000_000,), 0, 1, 1.0).astype(np.float64)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    assert abs((z ** 4).mean() - 3) < 0.05
    w = synth.bf16_bits_to_f32(synth.bf16_normal((200_000,), 0, 3, 0.02)).astype(np.float64)
    assert abs(w.std() - 0.02) < 5e-4


def test_streams_and_seeds_differ():
    a = synth.bf16_normal((1000,), 0, 1, 1.0)
    assert not np.array_equal(a, synth.bf16_normal((1000,), 0, 2, 1.0))
    assert not np.array_equal(a, synth.bf16_normal((1000,), 1, 1, 1.0))
    assert np.array_equal(a, synth.bf16_normal((1000,), 0, 1, 1.0))


def test_rank_permutation_and_bias():
    r = synth.rank_permutation(64, 0)
    assert sorted(r.tolist()) == list(range(1, 65))
    b = synth.skew_bias(64, 2.0, 0)
    assert b.dtype == np.float32 and b.max() == 0.0
    assert abs(float(b.min()) - (-2.0 * math.log(64))) < 1e-5
    assert synth.skew_bias(8, 0.0, 0) is None


def test_bf16_rounding_helper():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e38, np.inf], dtype=np.float32)
    b = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(b)
    assert back[0] == 1.0 and back[1] == 1.0          # halfway: ties to even
    assert back[2] == 1.0078125                         # above halfway: up
    assert back[3] == -2.5 and np.isinf(back[5])


def test_config4_alpha_gives_gini_0_3(orc):
    """The frozen skew of the decode layer yields a token-count Gini of 0.30
    (the MLA band of the "DODOCO" abstract), with routing from the oracle."""
    cfg = synth.CONFIGS[4]
    L = synth.make_layer(cfg, with_experts=False)
    idx, _, _ = orc.topk_softmax(orc.router_logits(L.x, L.w_router, L.bias), cfg.k)
    n = np.bincount(idx.reshape(-1), minlength=cfg.E).astype(np.float64)
    g = np.abs(n[:, None] - n[None, :]).sum() / (2 * cfg.E ** 2 * n.mean())
    assert 0.29 <= g <= 0.31
