"""bench.py's algorithmic work per stage (the roofline numerators), checked
against closed forms on CPU: the FLOPs of the full-width prefill workload and
the bytes a decode step must move."""
import importlib.util
import os

import pytest

from synthetic import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_prefill_work_closed_forms():
    b = _bench()
    cfg = get_config("prefill_4k")
    M, H, I, R = 4096, 2048, 2048, 256
    routed, pairs = 4093, 8390656
    w = b.stage_work(cfg, routed, pairs)
    assert w["qkv_gemm"] == ("tensor", 2.0 * M * H * 1536, "FLOP")          # 25.8 GF
    assert w["o_proj_merge"] == ("tensor", 2.0 * M * 1024 * H, "FLOP")      # 17.2 GF
    assert w["router_down"] == ("tensor", 2.0 * M * H * R, "FLOP")          # 4.3 GF
    assert w["attention"] == ("tensor", 4.0 * 128 * pairs * 8, "FLOP")      # 34.4 GF
    assert w["experts_gate_up"] == ("tensor", 2.0 * routed * H * 2 * I, "FLOP")
    assert w["experts_down_merge"] == ("tensor", 2.0 * routed * I * H, "FLOP")
    tc = sum(v[1] for v in w.values() if v[0] == "tensor")
    # the TC total for routed = M is the 184.7 GF of the scope table
    w_all = b.stage_work(cfg, M, pairs)
    tc_all = sum(v[1] for v in w_all.values() if v[0] == "tensor")
    assert tc_all == pytest.approx(184.7e9, rel=2e-3)
    assert tc < tc_all


def test_attention_pairs_is_the_causal_window_count():
    b = _bench()
    cfg = get_config("prefill_4k")
    # window = S: plain causal, S(S+1)/2 pairs
    assert b.attention_pairs(cfg, None) == 4096 * 4097 // 2
    small = cfg.with_(seq=10, window=3)
    # rows 0, 1 see 1 and 2 keys, the other 8 rows see 3
    assert b.attention_pairs(small, None) == 1 + 2 + 8 * 3


def test_decode_bytes_closed_forms():
    b = _bench()
    cfg = get_config("decode_stack_b64")
    w = b.stage_work_decode(cfg, routed=64, distinct=16)
    kv = 64 * 2 * 4096 * 128 * 2 * 2             # window K and V of every sequence
    assert w["attention_decode"][1] == kv + 2 * 64 * 1024 * 2
    expert = 2 * 2048 * 2048 * 2 + 2048 * 2048 * 2  # gate/up + down of one expert (bf16)
    gate_up, down = w["experts_gate_up"][1], w["experts_down_merge"][1]
    assert gate_up - 64 * 2048 * 2 - 64 * 2048 * 2 == 16 * 2 * 2048 * 2048 * 2
    assert gate_up + down > 16 * expert
    assert w["lm_head"][1] == 262144 * 2048 * 2 + 64 * 2048 * 2 + 64 * 262144 * 2
    assert all(v[0] == "hbm" for v in w.values())


def test_fp8_variants_work_and_peaks():
    """The fp8 variants' algorithmic work: the E4M3 cache halves the window's
    K/V bytes, FP8 experts halve their weight bytes in decode and are held
    against twice the bf16 dense peak in prefill (the nominal E4M3 / bf16
    ratio times the measured bf16 figure)."""
    b = _bench()
    d16 = b.stage_work_decode(get_config("decode_stack_b64"), routed=64, distinct=6)
    dkv = b.stage_work_decode(get_config("decode_stack_b64_fp8kv"), routed=64, distinct=6)
    dx = b.stage_work_decode(get_config("decode_stack_b64_fp8x"), routed=64, distinct=6)
    kv = 64 * 2 * 4096 * 128 * 2 * 2
    assert d16["attention_decode"][1] - dkv["attention_decode"][1] == kv // 2
    assert d16["experts_gate_up"][1] - dx["experts_gate_up"][1] == 6 * 2 * 2048 * 2048
    assert d16["experts_down_merge"][1] - dx["experts_down_merge"][1] == 6 * 2048 * 2048
    w = b.stage_work(get_config("prefill_4k_fp8x"), 4093, 8390656)
    assert w["experts_gate_up"][0] == "tensor_f8" and w["qkv_gemm"][0] == "tensor"
    peaks = {"bf16_tflops": 1665.3, "bf16_tflops_sustained": 1404.1, "hbm_gbs": 6455.6}
    cfg = get_config("prefill_4k_fp8x")
    r = b.roofline({"experts_gate_up": (0.0604, 1)}, w, peaks, "measured", cfg, 0.314)
    assert r["peak"] == round(2 * 1665.3, 1) and r["bound"] == "tensor"
    assert abs(r["achieved"] - w["experts_gate_up"][1] / 60.4e-6 / 1e12) < 0.01
