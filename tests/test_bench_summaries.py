"""bench.py's host-side arithmetic on made-up measurements (CPU): the
algorithmic work of each kernel, the expert-parallel summaries (per-rank
totals, the fused-return total, the bytes of each pass, the bound the local
GEMMs are held to)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def test_algorithmic_work_of_the_mixtral_layer():
    cfg = synth.CONFIGS[2]
    w = bench.algorithmic_work(cfg, [128] * 8)
    R = 512 * 2
    assert w["swiglu_bytes"] == 8 * 2 * 4096 * 14336 * 2 + R * 4096 * 2 + R * 14336 * 2
    assert w["swiglu_flops"] == 4 * R * 4096 * 14336
    assert w["down_flops"] == 2 * R * 14336 * 4096
    # untouched experts' weights are not work
    w2 = bench.algorithmic_work(cfg, [256, 256, 256, 256, 0, 0, 0, 0])
    assert w["swiglu_bytes"] - w2["swiglu_bytes"] == 4 * 2 * 4096 * 14336 * 2


def test_two_pass_summary():
    cfg = synth.CONFIGS[4]  # T 128, H 2048, F 1408, E 64, k 6, C 16
    G = 8
    S = min(6, 8) * (128 - 16)
    phases = {"route_and_pack": 240.0, "receive": 120.0, "experts_swiglu": 264.0, "experts_down": 200.0,
              "send_back": 64.0, "finish": 112.0}
    e = {"G": G, "S": S, "per_phase_us_all_ranks": phases, "overflow_rows": [87] * G, "device_status": [0] * G,
         "single_gpu_layer_us": 215.0}
    s = bench.summarize_ep(cfg, e, PEAKS)
    assert s["per_rank_us"]["route_and_pack"] == pytest.approx(30.0)
    assert s["per_rank_kernels_us"] == pytest.approx(sum(phases.values()) / G)
    row = 2048 * 2
    x = s["exchange_per_rank"]
    assert x["pass1_bytes"] == 64 * 16 * row and x["pass2_bytes"] == G * S * row
    assert x["real_overflow_bytes"] == pytest.approx(87 * row)
    assert x["nvlink_model_us"] == pytest.approx(2 * (64 * 16 * row + G * S * row + G * 2 * 8 * 4) / 770e9 * 1e6)
    assert s["experts_roofline"]["bound"] == "hbm"


def test_peer_store_summary_and_bound():
    G = 8
    phases = {"route": 80.0, "plan": 40.0, "dispatch": 48.0, "plan_dispatch": 72.0, "experts_swiglu": 1600.0,
              "experts_down": 1200.0,
              "send_back": 120.0, "down_return_fused": 1240.0, "finish": 64.0}
    e = {"G": G, "per_phase_us_all_ranks": phases, "device_status": [0] * G, "single_gpu_layer_us": 500.0}
    cfg = synth.CONFIGS[2]  # one expert per rank: the local GEMMs are tensor-bound
    s = bench.summarize_ep_direct(cfg, e, PEAKS)
    per = {k: v / G for k, v in phases.items()}
    sep = ("route", "plan", "dispatch", "experts_swiglu", "experts_down", "send_back", "finish")
    fused = ("route", "plan_dispatch", "experts_swiglu", "down_return_fused", "finish")
    assert s["per_rank_kernels_us"] == pytest.approx(sum(per[k] for k in sep))
    assert s["per_rank_kernels_fused_return_us"] == pytest.approx(sum(per[k] for k in fused))
    assert s["exchange_per_rank"]["dispatch_bytes"] == 512 * 2 * 4096 * 2
    assert s["experts_roofline"]["bound"] == "tensor"
    t = (per["experts_swiglu"] + per["experts_down"]) * 1e-6
    assert s["experts_roofline"]["achieved"] == pytest.approx(2.0 * 512 * 2 * 4096 * 14336 * 3 / t / 1e12)
    # the decode layer's eight experts per rank stream their weights: HBM-bound
    r = bench.experts_roofline(synth.CONFIGS[4], G, 60e-6, PEAKS)
    assert r["bound"] == "hbm" and r["bytes"] == 3 * 8 * 2048 * 1408 * 2


def test_peer_store_fp8_summary():
    G = 8
    phases = {"route": 80.0, "plan_dispatch_quantize": 104.0, "experts_swiglu": 160.0,
              "quantize_h": 32.0, "down_return_fused": 120.0, "finish": 64.0}
    e = {"G": G, "fp8": True, "per_phase_us_all_ranks": phases, "device_status": [0] * G,
         "single_gpu_layer_us": 150.0}
    cfg = synth.CONFIGS[4]
    s = bench.summarize_ep_direct(cfg, e, PEAKS)
    assert s["per_rank_kernels_us"] == pytest.approx(sum(phases.values()) / G)
    assert s["exchange_per_rank"]["dispatch_bytes"] == 128 * 6 * (2048 + 4)   # code rows and a scale each
    assert s["exchange_per_rank"]["return_bytes"] == 128 * 6 * 2048 * 2       # bf16 results
    r = s["experts_roofline"]
    assert r["bound"] == "hbm" and r["bytes"] == 3 * 8 * 2048 * 1408           # one-byte weights
