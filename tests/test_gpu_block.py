"""GPU parity of one block (prefill and decode) against the CPU oracle,
through the C ABI.  See tests/harness.py for the comparison protocol."""
import numpy as np
import pytest
import torch

from synthetic import gen_block_weights, gen_prefill_inputs, get_config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from top_moe_block_b200 import build
    build.build()


def _run_prefill(cfg, block_idx=None):
    from tests import harness as Hn
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    gpu = Hn.gpu_prefill(cfg, Hn.dev_weights(W), inp["x"], inp["attn_mask"], inp["router_state_in"],
                         block_idx=block_idx)
    res = Hn.check_prefill_block(cfg, W, inp, gpu, block_idx=block_idx)
    return res


@pytest.mark.parametrize("seq,batch", [(64, 1), (61, 1), (129, 2), (1, 3), (200, 1)])
def test_tiny_prefill(seq, batch):
    """Tiny block (hidden 256, 4/1 heads of 64, 4 experts + skip, window 32):
    several tiles plus ragged tails, a batch, and S = 1."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(seq=seq, batch=batch)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    assert res["cache_len_ok"]
    for key in ("k_cache", "v_cache", "attention_queries", "attention_output", "mlp_output"):
        assert res[key]["bf16_ok"], (key, res[key])


def test_tiny_block0_no_carried_state():
    from tests import harness as Hn
    cfg = get_config("tiny").with_(block_idx=0)
    Hn.assert_block_ok(_run_prefill(cfg))


def test_tiny_padding():
    """Left padding: pads take no part; the real rows match the oracle."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(batch=3, seq=80, pad_max=40)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)


def test_tiny_split_kv_attention():
    """Long causal rows against a short launch: the attention cuts the longest
    row tiles into key chunks and merges their partials (B2 x S1000, window
    1024, a ragged last tile and left padding)."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(batch=2, seq=1000, window=1024, pad_max=100)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    for key in ("attention_queries", "attention_output"):
        assert res[key]["bf16_ok"], (key, res[key])


def test_full_prefill_4k():
    """Full-width block, B1 x S4096 (the benchmark workload)."""
    from tests import harness as Hn
    res = _run_prefill(get_config("prefill_4k"))
    Hn.assert_block_ok(res)
    assert res["flips"] <= 0.001 * res["tokens"] + 2, res


def test_full_prefill_skewed_8x2k():
    """B8 x S2048 with left pads U{0..256}, Zipf(1.1) expert loads, ~20% skip."""
    from tests import harness as Hn
    cfg = get_config("prefill_skewed_8x2k")
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)


@pytest.mark.parametrize("name", ["tiny", "prefill_4k"])
def test_decode_after_prefill(name):
    """prefill(S) on the GPU, then one decode step: the decode output is
    compared with the oracle's decode on the GPU's own state."""
    from oracle import zaya_oracle as Z
    from tests import harness as Hn
    cfg = get_config(name)
    S = 256 if name == "prefill_4k" else 40
    cfg = cfg.with_(seq=S)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + 1))
    x, rin = inp["x"], inp["router_state_in"]
    st = Hn.new_state(cfg, 1, S + 8)
    Hn.gpu_prefill(cfg, Wd, x[:, :S], None, rin[:, :S], state=st)
    host_state = {k: v.cpu().clone() for k, v in st.items()}
    dec = Hn.gpu_decode(cfg, Wd, x[:, S], st, rin[:, S])
    g_cls = Hn.gpu_classes(cfg, dec)
    ref = Z.block_decode(cfg, Hn.eff(W), x[:, S], host_state, rin[:, S], force_cls=g_cls)
    t_cls, gap, _, _ = Hn.router_teacher_forced(cfg, Hn.eff(W), dec["mlp_norm_output"], rin[:, S], cfg.block_idx)
    assert ((t_cls == g_cls) | (gap < Hn.NEAR_TIE)).all()
    lo = Hn.report("layer_output", dec["layer_output"].numpy(), ref["layer_output"])
    assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, lo
    assert int(st["cache_len"][0]) == S + 1
    k_new = st["k_cache"][0, :, S].float().cpu().numpy()
    assert Hn.rel_max(k_new, ref["state"]["k_cache"][0, :, S]) <= 2e-2
    np.testing.assert_array_equal(st["prev_hs"].cpu().float().numpy(), dec["attention_norm_output"].float().numpy())


@pytest.mark.parametrize("name", ["tiny", "prefill_4k"])
def test_key_temperature_stress(name):
    """Key temperatures drawn U(0.8, 12.9) per kv head, the range of the
    ZAYA1-8B checkpoint (zaya page, 'Queries and keys are convolved ...'):
    softmax logits reach ~146, where the attention's lazy rescale of O
    does its work."""
    from tests import harness as Hn
    cfg = get_config(name).with_(temp_mode="stress")
    if name == "prefill_4k":
        cfg = cfg.with_(seq=1024)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    for key in ("attention_output", "k_cache"):
        assert res[key]["bf16_ok"], (key, res[key])


def test_tiny_partial_rope_not_multiple_of_16():
    """rot_dim = 24 (not a multiple of 16) takes the CCA kernel's general
    form instead of the streaming one."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(rot_dim=24, seq=77)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    for key in ("k_cache", "attention_queries"):
        assert res[key]["bf16_ok"], (key, res[key])


def test_full_prefill_8k_window_edge_sampled():
    """Full width at S = 8192 with window 4096 < S: from row 4096 on, every
    query tile's window starts inside a key tile (head_dim 128).  Sampled
    row ranges against the oracle's windowed evaluation: across the first
    window edge, in the middle, and the last rows."""
    from tests import harness as Hn
    cfg = get_config("prefill_4k").with_(seq=8192)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    gpu = Hn.gpu_prefill(cfg, Hn.dev_weights(W), inp["x"], None, inp["router_state_in"])
    ranges = [(4088, 4104), (6000, 6020), (8192 - 40, 8192)]
    res = Hn.check_prefill_rows(cfg, W, inp["x"][0], inp["router_state_in"][0], gpu, ranges, cfg.block_idx)
    print(res)
    Hn.assert_rows_ok(res)


def test_decode_position_outside_cache_is_reported():
    """A decode step whose position equals cache_cap for one sequence
    records ZAYA_ERR_DEVICE_RANGE and writes no sequence's cache,
    conv_state, prev_hs or cache_len."""
    import top_moe_block_b200 as ZB
    from tests import harness as Hn
    cfg = get_config("tiny")
    B, S = 3, 20
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + 1, batch=B))
    st = Hn.new_state(cfg, B, S + 2)
    Hn.gpu_prefill(cfg, Wd, inp["x"][:, :S], None, inp["router_state_in"][:, :S], state=st, taps=False)
    st["cache_len"][1] = S + 2                       # == cache_cap
    before = {k: v.clone() for k, v in st.items()}
    c = ZB.make_config(cfg)
    ws = Hn.workspace(ZB.zaya_workspace_size(c, ZB.ZAYA_DECODE, B, 1))
    h = inp["x"][:, S].cuda().contiguous()
    r_out = torch.empty(B, cfg.router_hidden, device="cuda")
    ZB.zaya_block_decode(c, ZB.make_weights(Wd), cfg.block_idx, B, h, inp["router_state_in"][:, S].cuda().contiguous(),
                         r_out, ZB.make_state(st), None, ws)
    assert ZB.zaya_device_status(ws) == ZB._abi.ZAYA_ERR_DEVICE_RANGE
    assert ZB.zaya_device_status(ws) == 0             # read and cleared
    for k in before:
        assert torch.equal(st[k], before[k]), k


def test_wait_timeout_is_reported_and_the_context_recovers():
    """With a 1 ns wait limit in the workspace header the bounded waits run
    out: the call records ZAYA_ERR_TIMEOUT (nothing hangs or faults).  With
    the header cleared, the same call on the same context matches the
    oracle."""
    import top_moe_block_b200 as ZB
    from tests import harness as Hn
    cfg = get_config("tiny")
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg)
    B, S = cfg.batch, cfg.seq
    c = ZB.make_config(cfg)
    ws = Hn.workspace(ZB.zaya_workspace_size(c, ZB.ZAYA_PREFILL, B, S))
    ZB.set_wait_limit_ns(ws, 1)
    hidden = inp["x"].cuda().contiguous()
    r_out = torch.empty(B, S, cfg.router_hidden, device="cuda")
    st = Hn.new_state(cfg, B, S)
    ZB.zaya_block_prefill(c, ZB.make_weights(Wd), cfg.block_idx, B, S, hidden, None,
                          inp["router_state_in"].cuda().contiguous(), r_out, ZB.make_state(st), None, ws)
    assert ZB.zaya_device_status(ws) == ZB._abi.ZAYA_ERR_TIMEOUT
    ZB.set_wait_limit_ns(ws, 0)
    torch.cuda.synchronize()
    gpu = Hn.gpu_prefill(cfg, Wd, inp["x"], None, inp["router_state_in"])
    Hn.assert_block_ok(Hn.check_prefill_block(cfg, W, inp, gpu, verbose=False))


@pytest.mark.parametrize("block_idx", [1, 2])
def test_full_prefill_hybrid_8k_sampled(block_idx):
    """The 74B preview's hybrid at full width, S = 8192: block 1 slides over
    4097 keys, block 2 attends to every earlier token (zaya page, 'Queries
    and keys are convolved ...', last sentence); sampled rows against the
    oracle's windowed evaluation."""
    from tests import harness as Hn
    cfg = get_config("prefill_4k").with_(seq=8192, window=4097, sliding_period=2, sliding_phase=1,
                                         block_idx=block_idx)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    gpu = Hn.gpu_prefill(cfg, Hn.dev_weights(W), inp["x"], None, inp["router_state_in"])
    ranges = [(4090, 4106), (8192 - 24, 8192)]
    res = Hn.check_prefill_rows(cfg, W, inp["x"][0], inp["router_state_in"][0], gpu, ranges, block_idx)
    print(res)
    Hn.assert_rows_ok(res)


@pytest.mark.parametrize("seq,batch,pad", [(64, 1, 0), (129, 2, 0), (80, 3, 40)])
def test_tiny_two_stage_conv(seq, batch, pad):
    """The printout's two convs (depthwise k=2, then grouped k=2 with one
    group per head) in place of the width-3 conv: tiles with ragged tails, a
    batch, and left padding."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(seq=seq, batch=batch, pad_max=pad, conv_width=2, conv_groups=5)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    for key in ("k_cache", "attention_queries", "conv_state"):
        assert res[key]["rel_max"] <= Hn.TOL_REL_MAX, (key, res[key])


def test_full_prefill_4k_two_stage_conv():
    """Full width with the two-stage conv_qk (10 groups of 128 channels)."""
    from tests import harness as Hn
    res = _run_prefill(get_config("prefill_4k_conv2"))
    Hn.assert_block_ok(res)
    for key in ("k_cache", "attention_queries"):
        assert res[key]["bf16_ok"], (key, res[key])


@pytest.mark.parametrize("name", ["tiny", "prefill_4k_conv2"])
def test_two_stage_conv_decode_after_prefill(name):
    """prefill(S) then one decode step with the two-stage conv: the decode's
    grouped conv takes u(t-2), u(t-1) from conv_state."""
    from oracle import zaya_oracle as Z
    from tests import harness as Hn
    cfg = get_config(name)
    if name == "tiny":
        cfg = cfg.with_(conv_width=2, conv_groups=5)
    S = 40
    cfg = cfg.with_(seq=S, batch=2)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + 1))
    x, rin = inp["x"], inp["router_state_in"]
    st = Hn.new_state(cfg, 2, S + 8)
    Hn.gpu_prefill(cfg, Wd, x[:, :S], None, rin[:, :S], state=st)
    host_state = {k: v.cpu().clone() for k, v in st.items()}
    dec = Hn.gpu_decode(cfg, Wd, x[:, S], st, rin[:, S])
    g_cls = Hn.gpu_classes(cfg, dec)
    ref = Z.block_decode(cfg, Hn.eff(W), x[:, S], host_state, rin[:, S], force_cls=g_cls)
    lo = Hn.report("layer_output", dec["layer_output"].numpy(), ref["layer_output"])
    assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, lo
    k_new = st["k_cache"][:, :, S].float().cpu().numpy()
    assert Hn.rel_max(k_new, ref["state"]["k_cache"][:, :, S]) <= 2e-2


def _ring_matches_linear(lin, ring, n, cap):
    """The ring's kept rows (positions max(0, n - cap) .. n-1 at slots p % cap)
    equal the linear cache's rows, bit for bit; the other state too."""
    for p in range(max(0, n - cap), n):
        for key in ("k_cache", "v_cache"):
            assert torch.equal(lin[key][:, :, p], ring[key][:, :, p % cap]), (key, p)
    for key in ("cache_len", "conv_state", "prev_hs"):
        assert torch.equal(lin[key], ring[key]), key


@pytest.mark.parametrize("name", ["tiny", "prefill_4k"])
def test_window_ring_cache_matches_linear_cache(name):
    """kv_ring: a window-sized cache that keeps position p at slot p % cap.
    A prompt longer than the ring, then decode steps across the ring's wrap:
    every output equals the linear-cache run bit for bit (the same kernels
    add the same keys in the same order; only the rows' addresses differ),
    and the kept K / V rows equal the linear cache's.  The decode outputs are
    also held against the oracle's decode on a dense state rebuilt from the
    ring (positions outside the window are not read)."""
    from oracle import zaya_oracle as Z
    from tests import harness as Hn
    cfg = get_config(name)
    S, steps = (50, 5) if name == "tiny" else (300, 3)
    if name == "prefill_4k":
        cfg = cfg.with_(window=128)
    cfg = cfg.with_(seq=S)
    cap = cfg.window
    rcfg = cfg.with_(kv_ring=1)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + steps))
    x, rin = inp["x"], inp["router_state_in"]
    r_at = (lambda i: None) if rin is None else (lambda i: rin[:, i])
    lin = Hn.new_state(cfg, 1, S + steps)
    ring = Hn.new_state(cfg, 1, cap)
    a = Hn.gpu_prefill(cfg, Wd, x[:, :S], None, None if rin is None else rin[:, :S], state=lin, taps=False)
    b = Hn.gpu_prefill(rcfg, Wd, x[:, :S], None, None if rin is None else rin[:, :S], state=ring, taps=False)
    assert torch.equal(a["layer_output"], b["layer_output"])
    assert torch.equal(a["router_state"], b["router_state"])
    _ring_matches_linear(lin, ring, S, cap)
    for k in range(steps):
        n = S + k
        host = {key: v.cpu().clone() for key, v in ring.items()}
        dense = dict(host)
        for key in ("k_cache", "v_cache"):
            full = torch.zeros(host[key].shape[0], host[key].shape[1], n + 1, host[key].shape[3], dtype=host[key].dtype)
            for p in range(max(0, n - cap), n):
                full[:, :, p] = host[key][:, :, p % cap]
            dense[key] = full
        da = Hn.gpu_decode(cfg, Wd, x[:, n], lin, r_at(n))
        db = Hn.gpu_decode(rcfg, Wd, x[:, n], ring, r_at(n))
        assert torch.equal(da["layer_output"], db["layer_output"]), k
        _ring_matches_linear(lin, ring, n + 1, cap)
        g_cls = Hn.gpu_classes(cfg, db)
        ref = Z.block_decode(cfg, Hn.eff(W), x[:, n], dense, r_at(n), force_cls=g_cls)
        lo = Hn.report("layer_output", db["layer_output"].numpy(), ref["layer_output"])
        assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, (k, lo)


@pytest.mark.parametrize("name", ["tiny", "prefill_4k"])
def test_fp8_cache_prefill_and_decode(name):
    """kv_fp8 (E4M3 K/V cache, the NVFP4 README's --kv-cache-dtype fp8): the
    prompt attends over its bf16 keys / values, so every prefill output equals
    the bf16-cache run bit for bit; the cache bytes are the E4M3 codes of the
    bf16 run's keys and values, exactly; decode steps then read the E4M3 cache
    and match the oracle's fp8-cache decode on the GPU's own state."""
    from oracle import zaya_oracle as Z
    from tests import harness as Hn
    cfg = get_config(name)
    S, steps = (40, 3) if name == "tiny" else (256, 2)
    cfg = cfg.with_(seq=S)
    c8 = cfg.with_(kv_fp8=1)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + steps))
    x, rin = inp["x"], inp["router_state_in"]
    r_at = (lambda i: None) if rin is None else (lambda i: rin[:, i])
    st16 = Hn.new_state(cfg, 1, S + steps)
    st8 = Hn.new_state(c8, 1, S + steps)
    a = Hn.gpu_prefill(cfg, Wd, x[:, :S], None, None if rin is None else rin[:, :S], state=st16, taps=False)
    b = Hn.gpu_prefill(c8, Wd, x[:, :S], None, None if rin is None else rin[:, :S], state=st8, taps=False)
    assert torch.equal(a["layer_output"], b["layer_output"])
    assert torch.equal(a["router_state"], b["router_state"])
    for key in ("k_cache", "v_cache"):
        got = Hn.e4m3_values(st8[key][:, :, :S]).numpy()
        want = Z.round_e4m3(st16[key][:, :, :S].float().cpu().numpy())
        np.testing.assert_array_equal(got, want)
    for key in ("cache_len", "conv_state", "prev_hs"):
        assert torch.equal(st8[key], st16[key]), key
    for k in range(steps):
        n = S + k
        host = {key: v.cpu().clone() for key, v in st8.items()}
        host["k_cache"] = Hn.e4m3_values(host["k_cache"])
        host["v_cache"] = Hn.e4m3_values(host["v_cache"])
        dec = Hn.gpu_decode(c8, Wd, x[:, n], st8, r_at(n))
        g_cls = Hn.gpu_classes(cfg, dec)
        ref = Z.block_decode(c8, Hn.eff(W), x[:, n], host, r_at(n), force_cls=g_cls)
        lo = Hn.report("layer_output", dec["layer_output"].numpy(), ref["layer_output"])
        assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, (k, lo)
        ao = Hn.report("attention_output", dec["attention_output"].float().numpy(), ref["attention_output"])
        assert ao["cos"] >= 0.999, (k, ao)
        new = Hn.e4m3_values(st8["k_cache"][:, :, n]).numpy()
        want = ref["state"]["k_cache"][:, :, n]
        step = np.ldexp(1.0, np.maximum(np.frexp(np.abs(want) + (want == 0))[1] - 1, -6) - 3)
        assert (np.abs(new - want) <= step).all()   # one E4M3 step: the keys' bf16 inputs differ in rounding


def test_fp8_window_ring_matches_linear_fp8_cache():
    """kv_fp8 with kv_ring: a prompt longer than the ring and decode steps
    across the wrap equal the linear fp8-cache run bit for bit."""
    from tests import harness as Hn
    cfg = get_config("tiny").with_(seq=50, kv_fp8=1)
    S, steps, cap = 50, 4, cfg.window
    rcfg = cfg.with_(kv_ring=1)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + steps))
    x, rin = inp["x"], inp["router_state_in"]
    lin = Hn.new_state(cfg, 1, S + steps)
    ring = Hn.new_state(cfg, 1, cap)
    a = Hn.gpu_prefill(cfg, Wd, x[:, :S], None, rin[:, :S], state=lin, taps=False)
    b = Hn.gpu_prefill(rcfg, Wd, x[:, :S], None, rin[:, :S], state=ring, taps=False)
    assert torch.equal(a["layer_output"], b["layer_output"])
    _ring_matches_linear(lin, ring, S, cap)
    for k in range(steps):
        da = Hn.gpu_decode(cfg, Wd, x[:, S + k], lin, rin[:, S + k])
        db = Hn.gpu_decode(rcfg, Wd, x[:, S + k], ring, rin[:, S + k])
        assert torch.equal(da["layer_output"], db["layer_output"]), k
        _ring_matches_linear(lin, ring, S + k + 1, cap)


@pytest.mark.parametrize("name", ["tiny", "prefill_4k"])
def test_fp8_experts_prefill(name):
    """expert_fp8: the experts as an FP8 W8A8 checkpoint (E4M3 weight codes
    with per-row scales, E4M3 activations with static scales) on tcgen05
    kind::f8f6f4 swapped pair tiles, against the oracle's FP8 expert at the
    block tolerances (every step before the experts is the bf16 block's)."""
    from tests import harness as Hn
    cfg = get_config(name).with_(expert_fp8=1)
    if name == "prefill_4k":
        cfg = cfg.with_(seq=1024)
    res = _run_prefill(cfg)
    Hn.assert_block_ok(res)
    assert res["mlp_output"]["cos"] >= 0.999, res["mlp_output"]


def test_fp8_experts_decode_after_prefill():
    """expert_fp8 in decode: a few tokens per expert on 16-token swapped
    tiles, E4M3 operands, against the oracle's decode."""
    from oracle import zaya_oracle as Z
    from tests import harness as Hn
    cfg = get_config("prefill_4k").with_(seq=128, expert_fp8=1)
    S = 128
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + 1))
    x, rin = inp["x"], inp["router_state_in"]
    st = Hn.new_state(cfg, 1, S + 4)
    Hn.gpu_prefill(cfg, Wd, x[:, :S], None, None if rin is None else rin[:, :S], state=st, taps=False)
    host = {k: v.cpu().clone() for k, v in st.items()}
    r1 = None if rin is None else rin[:, S]
    dec = Hn.gpu_decode(cfg, Wd, x[:, S], st, r1)
    g_cls = Hn.gpu_classes(cfg, dec)
    ref = Z.block_decode(cfg, Hn.eff(W), x[:, S], host, r1, force_cls=g_cls)
    lo = Hn.report("layer_output", dec["layer_output"].numpy(), ref["layer_output"])
    assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, lo
