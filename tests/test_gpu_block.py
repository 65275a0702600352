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
    ref = Z.block_decode(cfg, W, x[:, S], host_state, rin[:, S], force_cls=g_cls)
    t_cls, gap, _, _ = Hn.router_teacher_forced(cfg, W, dec["mlp_norm_output"], rin[:, S], cfg.block_idx)
    assert ((t_cls == g_cls) | (gap < Hn.NEAR_TIE)).all()
    lo = Hn.report("layer_output", dec["layer_output"].numpy(), ref["layer_output"])
    assert lo["rel_max"] <= Hn.TOL_REL_MAX and lo["cos"] >= Hn.TOL_COS, lo
    assert int(st["cache_len"][0]) == S + 1
    k_new = st["k_cache"][0, :, S].float().cpu().numpy()
    assert Hn.rel_max(k_new, ref["state"]["k_cache"][0, :, S]) <= 2e-2
    np.testing.assert_array_equal(st["prev_hs"].cpu().float().numpy(), dec["attention_norm_output"].float().numpy())
