"""Pins of the CPU oracle to what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-worked example (tests/golden/worked_examples.json), an identity the
zaya page prints, a textbook routine the block reduces to in a special
case, or a brute-force structural property (causality, window reach).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import zaya_oracle as Z
from synthetic import gen_block_weights, gen_prefill_inputs, get_config

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def tiny():
    cfg = get_config("tiny")
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    out = Z.block_prefill(cfg, W, inp["x"], inp["attn_mask"], inp["router_state_in"])
    return cfg, W, inp, out


# ---------------------------------------------------------------- worked examples

def test_conv_worked_examples():
    g = _load("worked_examples.json")
    for key in ("conv_fresh", "conv_with_state"):
        ex = g[key]
        w = np.array([ex["taps_t-2_t-1_t"]])
        y = Z.causal_conv(np.array(ex["u"])[:, None], w, np.array([ex["bias"]]), np.array(ex["hist"])[:, None])
        np.testing.assert_allclose(y[:, 0], ex["y"], rtol=0, atol=1e-12)


def test_cca_residual_worked_example():
    ex = _load("worked_examples.json")["cca_mean_residual"]
    q = np.array(ex["q_pre"])[None, :, None]
    k = np.array(ex["k_pre"])[None, :, None]
    qr, kr = Z.cca_mean_residual(q, k, ex["n_q"], ex["n_kv"])
    np.testing.assert_allclose(qr.ravel(), ex["q_res"], atol=1e-12)
    np.testing.assert_allclose(kr.ravel(), ex["k_res"], atol=1e-12)


def test_norms_rope_merge_worked_examples():
    g = _load("worked_examples.json")
    ex = g["l2_to_sqrt_d"]
    np.testing.assert_allclose(Z.l2_to_sqrt_d(np.array(ex["x"]), 1e-6), ex["y"], atol=1e-12)
    ex = g["rms_norm"]
    np.testing.assert_allclose(Z.rms_norm(np.array(ex["x"]), np.array(ex["w"]), ex["eps"]), ex["y"], atol=1e-12)
    ex = g["rope_half"]
    for a, b in (("x_a", "y_a"), ("x_b", "y_b")):
        y = Z.rope(np.array(ex[a])[None, None, :], [ex["pos"]], ex["rot"], ex["theta"])
        np.testing.assert_allclose(y.ravel(), ex[b], atol=1e-12)
    ex = g["merge"]
    p = np.array([[ex["hb"]], [ex["hs"]], [ex["rb"]], [ex["rs"]]])
    c, s = Z.merge(np.array([ex["o"]]), np.array([ex["r"]]), p)
    assert c[0] == ex["contribution"] and s[0] == ex["stream"]


def test_activations_closed_form():
    ex = _load("worked_examples.json")["activations"]
    for x, y in ex["gelu"]:
        assert Z.gelu(np.array(x)) == pytest.approx(y, abs=1e-15)
    for x, y in ex["silu"]:
        assert Z.silu(np.array(x)) == pytest.approx(y, abs=1e-15)


def test_selection_worked_examples():
    ex = _load("worked_examples.json")["selection"]
    for c in ex["cases"]:
        cls, idx, w, p, gap = Z.select(np.array([c["logits"]]), np.array(c["bias"]), ex["n_experts"])
        assert int(cls[0]) == c["cls"], c["note"]
        assert int(idx[0]) == c["idx"], c["note"]
        assert w[0] == pytest.approx(c["w"], abs=1e-7), c["note"]


# ---------------------------------------------------------------- page identities

def test_contribution_identity(tiny):
    """layer_output == (layer_mid + m.rb) * m.rs + mlp_output and
    layer_mid == (layer_input + a.rb) * a.rs + attention_output, in float32
    (zaya page, 'The contributions are the merges' scaled terms')."""
    cfg, W, inp, o = tiny
    f = lambda a: torch.tensor(a, dtype=torch.float32)
    a, m = W["merge_a"], W["merge_m"]
    h = (f(o["layer_input"]) + a[2]) * a[3] + f(o["attention_output"])
    torch.testing.assert_close(h, f(o["layer_mid"]))
    out = (f(o["layer_mid"]) + m[2]) * m[3] + f(o["mlp_output"])
    torch.testing.assert_close(out, f(o["layer_output"]))


def test_router_identity_and_skip(tiny):
    """softmax(router_logits.float()).gather(idx) == expert_weights where an
    expert was chosen; skip slots read (0, 0) and leave mlp_output =
    hidden_states_bias * hidden_states_scale (zaya page, 'One expert per
    token' and 'Ablating an expert leaves the merge's bias')."""
    cfg, W, inp, o = tiny
    E = cfg.n_experts
    logits = torch.tensor(o["router_logits"], dtype=torch.float32)
    probs = logits.softmax(-1)
    idx = torch.tensor(o["expert_indices"]).long()
    w = torch.tensor(o["expert_weights"], dtype=torch.float32)
    cls = o["expert_cls"]
    chose = torch.tensor(cls != E)
    assert chose.any() and (~chose).any(), "the tiny workload must route some tokens to skip"
    g = probs.gather(-1, idx[..., None])[..., 0]
    torch.testing.assert_close(g[chose], w[chose])
    assert (idx[~chose] == 0).all() and (w[~chose] == 0).all()
    skip = cls == E
    assert np.all(o["routed_output"][skip] == 0)
    hb, hs = Z.as64(W["merge_m"][0]), Z.as64(W["merge_m"][1])
    np.testing.assert_array_equal(o["mlp_output"][skip], np.broadcast_to(Z.round_bf16(hb * hs), o["mlp_output"][skip].shape))


def test_expert_ablation(tiny):
    """Zeroing expert e's weight changes mlp_output exactly at the tokens
    with (idx == e) & (w > 0) (zaya page, 'Ablating an expert ...')."""
    cfg, W, inp, o = tiny
    m_in = o["mlp_norm_output"][0]
    cls, w = o["expert_cls"][0], o["expert_weights"][0]
    h = o["layer_mid"][0]
    for e in range(cfg.n_experts):
        w_abl = np.where(o["expert_indices"][0] == e, 0.0, w)
        routed = Z.moe(cfg, W, m_in, cls, w_abl)
        ablated, _ = Z.merge(routed, h, Z.as64(W["merge_m"]))
        changed = (ablated != o["mlp_output"][0]).any(-1)
        chose = (o["expert_indices"][0] == e) & (w > 0)
        np.testing.assert_array_equal(changed, chose)


def test_zero_attention_contribution(tiny):
    """hidden_states_scale = 0 on the first merge leaves (x + rb) * rs
    (zaya page, 'Zeroing attention_output removes the term ...')."""
    cfg, W, inp, _ = tiny
    W2 = dict(W)
    ma = W["merge_a"].clone()
    ma[1] = 0.0
    W2["merge_a"] = ma
    o = Z.block_prefill(cfg, W2, inp["x"], None, inp["router_state_in"])
    assert np.all(o["attention_output"] == 0)
    x = Z.as64(inp["x"])
    np.testing.assert_array_equal(o["layer_mid"], Z.round_f32((x + Z.as64(ma[2])) * Z.as64(ma[3])))


# ---------------------------------------------------------------- special cases

def test_temp_zero_uniform_attention():
    """temp = 0 zeroes every key, so each query mixes the values of its
    visible window uniformly (zaya page, family docstring: 'at its initial
    value of zero every key is zero and the pattern uniform').  Uses 2 kv
    heads with 2 query heads each, so the head -> kv-head map is pinned."""
    cfg = get_config("tiny").with_(n_q=4, n_kv=2, temp_mode="zero", window=8, seq=20)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    o = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"])
    assert np.all(o["attention_keys"] == 0)
    v = o["attention_values"][0]            # [nkv, S, d]
    S, d = cfg.seq, cfg.head_dim
    prem = o["attention_premix"][0].reshape(S, cfg.n_q, d)
    for i in range(S):
        lo = max(0, i - cfg.window + 1)
        for h in range(cfg.n_q):
            np.testing.assert_allclose(prem[i, h], v[h // 2, lo:i + 1].mean(axis=0), rtol=1e-12, atol=1e-12)


def test_plain_gqa_special_case():
    """With conv taps (0,0,1), zero conv bias, no CCA residual, no delayed
    values, no rotation and a window >= S, the attention half is plain
    L2-normed causal GQA: compared with torch's scaled_dot_product_attention
    in float64."""
    cfg = get_config("tiny").with_(n_q=4, n_kv=2, cca_mean_residual=0, v_delayed=0, rot_dim=0,
                                   window=1000, seq=24)
    W = dict(gen_block_weights(cfg))
    cw = torch.zeros_like(W["conv_w"])
    cw[:, 2] = 1.0
    W["conv_w"], W["conv_b"] = cw, torch.zeros_like(W["conv_b"])
    inp = gen_prefill_inputs(cfg)
    o = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"])
    S, d, H = cfg.seq, cfg.head_dim, cfg.hidden
    a_in = torch.tensor(o["attention_norm_output"][0])
    proj = a_in @ W["w_qkv"].double().T
    proj = torch.tensor(Z.round_bf16(proj.numpy()))
    q = proj[:, :cfg.q_dim].reshape(S, cfg.n_q, d).transpose(0, 1)
    k = proj[:, cfg.q_dim:cfg.q_dim + cfg.kv_dim].reshape(S, cfg.n_kv, d).transpose(0, 1)
    vc = proj[:, cfg.q_dim + cfg.kv_dim:cfg.q_dim + cfg.kv_dim + cfg.v_half]
    vd = proj[:, cfg.q_dim + cfg.kv_dim + cfg.v_half:]
    hd = d // 2
    v = torch.stack([torch.cat([vc[:, g * hd:(g + 1) * hd], vd[:, g * hd:(g + 1) * hd]], -1)
                     for g in range(cfg.n_kv)])
    q = torch.nn.functional.normalize(q, dim=-1) * math.sqrt(d)
    k = torch.nn.functional.normalize(k, dim=-1) * math.sqrt(d)
    k = torch.tensor(Z.round_bf16(k.numpy()))
    v = torch.tensor(Z.round_bf16(v.numpy()))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None], k[None], v[None], is_causal=True, enable_gqa=True)[0]
    np.testing.assert_allclose(o["attention_premix"][0], ref.transpose(0, 1).reshape(S, -1).numpy(),
                               rtol=1e-10, atol=1e-10)


def test_rope_is_complex_rotation_and_relative():
    """Rotate-half RoPE on dims (i, i+rot/2) is multiplication of
    x_i + j x_{i+rot/2} by exp(j * pos * inv_freq_i); scores depend only on
    the position difference."""
    rng = np.random.default_rng(0)
    rot, theta = 32, 1e4
    x = rng.standard_normal((5, 1, 64))
    pos = np.array([0, 1, 7, 30, 63])
    y = Z.rope(x, pos, rot, theta)
    inv = Z.rope_inv_freq(rot, theta)
    ang = Z.round_f32(pos[:, None] * inv[None, :])
    z = (x[:, 0, :16] + 1j * x[:, 0, 16:32]) * np.exp(1j * ang)
    np.testing.assert_allclose(y[:, 0, :16], z.real, atol=1e-12)
    np.testing.assert_allclose(y[:, 0, 16:32], z.imag, atol=1e-12)
    np.testing.assert_array_equal(y[:, 0, 32:], x[:, 0, 32:])
    q, k = rng.standard_normal((1, 1, 64)), rng.standard_normal((1, 1, 64))
    s0 = (Z.rope(q, [10], rot, theta) * Z.rope(k, [3], rot, theta)).sum()
    s1 = (Z.rope(q, [50], rot, theta) * Z.rope(k, [43], rot, theta)).sum()
    assert s0 == pytest.approx(s1, rel=1e-5)


def test_expert_permutation_closed_form():
    """An expert whose gate is a permutation sigma, up the identity and down
    a permutation tau gives y_i = silu(x[sigma(tau(i))]) * x[tau(i)];
    sigma and tau are not involutions, so a transposed operand fails."""
    n = 6
    sigma = np.array([1, 2, 3, 4, 5, 0])
    tau = np.array([2, 0, 4, 1, 5, 3])
    P = lambda perm: np.eye(n)[perm]                 # (P @ x)[j] = x[perm[j]]
    wgu = np.concatenate([P(sigma), np.eye(n)], axis=0)
    x = np.array([[0.3, -1.2, 2.0, 0.7, -0.4, 1.5]])
    y = Z.expert_ffn(x, wgu, P(tau), n)
    expect = [Z.silu(x[0, sigma[tau[i]]]) * x[0, tau[i]] for i in range(n)]
    np.testing.assert_allclose(y[0], expect, atol=1e-14)


# ---------------------------------------------------------------- brute force

def _perturbed(cfg, W, inp, t):
    x2 = inp["x"].clone()
    x2[0, t] += 0.5
    return Z.block_prefill(cfg, W, x2, None, inp["router_state_in"])


def test_causality_brute_force(tiny):
    """Perturbing token t leaves every output before t bit-identical."""
    cfg, W, inp, o = tiny
    for t in (0, 5, 31, 63):
        o2 = _perturbed(cfg, W, inp, t)
        for key in ("layer_output", "router_state", "router_logits", "attention_premix"):
            np.testing.assert_array_equal(o2[key][0, :t], o[key][0, :t])
        assert not np.array_equal(o2["layer_output"][0, t], o["layer_output"][0, t])


def test_window_and_conv_reach(tiny):
    """Keys j in {t, t+1, t+2} depend on token t (width-3 conv and the
    delayed value half), and a query i sees keys with 0 <= i-j < W.  So
    outputs at i >= t+W+2 are bit-identical and the output at t+W+1
    changes; reading the window as i-j <= W would move that edge by one."""
    cfg, W, inp, o = tiny
    Wn = cfg.window
    for t in (0, 10, 20):
        o2 = _perturbed(cfg, W, inp, t)
        edge = t + Wn + 1
        assert edge < cfg.seq - 1
        np.testing.assert_array_equal(o2["attention_premix"][0, edge + 1:], o["attention_premix"][0, edge + 1:])
        np.testing.assert_array_equal(o2["layer_output"][0, edge + 1:], o["layer_output"][0, edge + 1:])
        assert not np.array_equal(o2["attention_premix"][0, edge], o["attention_premix"][0, edge])


def test_decode_continues_prefill(tiny):
    """prefill(S) then one decode step equals prefill(S+1) at position S,
    for the outputs and the state it leaves (KV, conv_state, prev_hs)."""
    cfg, W, inp, _ = tiny
    S = cfg.seq
    x = inp["x"]
    r = inp["router_state_in"]
    full = Z.block_prefill(cfg, W, x, None, r)
    part = Z.block_prefill(cfg.with_(seq=S - 1), W, x[:, :S - 1], None, r[:, :S - 1])
    st = part["state"]
    cap = S + 3
    B = 1
    kc = np.zeros((B, cfg.n_kv, cap, cfg.head_dim))
    vc = np.zeros_like(kc)
    kc[:, :, :S - 1] = st["k_cache"]
    vc[:, :, :S - 1] = st["v_cache"]
    state = dict(k_cache=kc, v_cache=vc, conv_state=st["conv_state"], prev_hs=st["prev_hs"],
                 cache_len=st["cache_len"])
    dec = Z.block_decode(cfg, W, x[:, S - 1], state, r[:, S - 1])
    for key in ("layer_output", "router_state", "attention_output", "mlp_output"):
        np.testing.assert_allclose(dec[key], full[key][:, S - 1], rtol=1e-9, atol=1e-9)
    np.testing.assert_array_equal(dec["expert_cls"], full["expert_cls"][:, S - 1])
    np.testing.assert_allclose(dec["state"]["k_cache"][:, :, :S], full["state"]["k_cache"], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(dec["state"]["v_cache"][:, :, :S], full["state"]["v_cache"], rtol=1e-9, atol=1e-9)
    np.testing.assert_array_equal(dec["state"]["conv_state"], full["state"]["conv_state"])
    np.testing.assert_array_equal(dec["state"]["prev_hs"], full["state"]["prev_hs"])
    assert int(dec["state"]["cache_len"][0]) == S


@pytest.mark.parametrize("rot", [0, 32])
def test_left_padding_equals_unpadded(tiny, rot):
    """A left-padded sequence's real rows equal the unpadded sequence's
    (padding is absent; RoPE sees only position differences).  Without
    rotation the match is exact up to summation order; with it, the fp32
    angles differ by rounding, which can move a bf16-rounded contribution
    by one unit in the last place."""
    cfg, W, inp, _ = tiny
    cfg = cfg.with_(rot_dim=rot)
    S, P = cfg.seq, 9
    x = inp["x"][:, :S - P]
    r = inp["router_state_in"][:, :S - P]
    ref = Z.block_prefill(cfg.with_(seq=S - P), W, x, None, r)
    g = torch.Generator().manual_seed(5)
    xp = torch.cat([torch.randn(1, P, cfg.hidden, generator=g), x], dim=1)
    rp = torch.cat([torch.randn(1, P, cfg.router_hidden, generator=g), r], dim=1)
    mask = torch.ones(1, S, dtype=torch.int32)
    mask[0, :P] = 0
    o = Z.block_prefill(cfg, W, xp, mask, rp)
    tol = 1e-9 if rot == 0 else 8e-3
    np.testing.assert_allclose(o["layer_output"][0, P:], ref["layer_output"][0], rtol=tol, atol=tol)
    np.testing.assert_array_equal(o["expert_cls"][0, P:], ref["expert_cls"][0])
    np.testing.assert_array_equal(o["expert_cls"][0, :P], cfg.n_experts)


# ---------------------------------------------------------------- printed sizes

def test_page_sizes():
    facts = _load("page_facts.json")
    cfg = get_config("prefill_4k")
    kv = facts["kv_cache_bytes_per_token"]
    assert kv["layers"] * 2 * cfg.n_kv * cfg.head_dim * 2 == kv["value"]
    e = facts["embed_bytes"]
    assert e["shape"][0] * e["shape"][1] * e["dtype_bytes"] == e["value"]
    assert e["shape"][1] == cfg.hidden
    pr = facts["projections"]
    assert pr["q"][1] == cfg.q_dim and pr["k"][1] == cfg.kv_dim
    assert pr["v_current"][1] == cfg.v_half and pr["v_delayed"][1] == cfg.v_half
    assert pr["o"] == [cfg.q_dim, cfg.hidden]
    assert pr["router_down"][1] == cfg.router_hidden and pr["router_out"][1] == cfg.n_experts + 1
    assert facts["conv_channels"]["value"] == cfg.qk_channels
    assert facts["conv_state_shape"]["value"][1] == cfg.qk_channels
    assert facts["prev_hs_shape"]["value"][1] == cfg.hidden


# ---------------------------------------------------------------- router MLP order, stack

def test_router_mlp_order_special_case():
    """With fc1 = 2*I, fc2 = I, zero biases, unit norm weight, out_proj
    = the first E+1 unit rows and a constant router state, the router MLP
    reduces to gelu(gelu(2 * 1)) in every logit (norm -> fc1 -> GELU ->
    fc2 -> GELU -> out_proj); computed here with math.erf."""
    R, E = 8, 3
    W = {"router_norm_w": np.ones(R), "fc1_w": 2 * np.eye(R), "fc1_b": np.zeros(R),
         "fc2_w": np.eye(R), "fc2_b": np.zeros(R), "out_w": np.eye(R)[:E + 1]}
    r = np.full((2, R), 3.7)
    g = lambda x: 0.5 * x * (1 + math.erf(x / math.sqrt(2)))
    expect = np.float32(g(g(2.0)))
    logits = Z.router_mlp(r, W, 0.0)
    np.testing.assert_allclose(logits, np.full((2, E + 1), expect), rtol=1e-6)


def test_embed_and_head_closed_form():
    """stream0 = fp32((E[id] + shift) * mult); logits = norm(x) @ E^T with
    the tied table: for x = c * e_k, norm(x) = sqrt(H) * w_k * e_k."""
    cfg = get_config("tiny").with_(emb_shift=0.25)
    V, H = 7, cfg.hidden
    table = np.arange(V, dtype=np.float64)[:, None] * np.ones((1, H)) / 8.0
    ids = np.array([[3, 0, 6]])
    te, x = Z.embed(cfg, table, ids)
    np.testing.assert_array_equal(x[0, :, 0], Z.round_f32((np.array([3, 0, 6]) / 8.0 + 0.25) * cfg.emb_mult))
    k = 5
    xs = np.zeros((1, H))
    xs[0, k] = 3.0
    wn = np.ones(H)
    wn[k] = 0.5
    tab = np.zeros((V, H))
    tab[:, k] = np.arange(V) / 4.0
    fn, logits = Z.lm_head(cfg, tab, wn, xs)
    expect = Z.round_bf16(Z.round_bf16(math.sqrt(H) * 0.5 / math.sqrt(1 + cfg.rms_eps * H / 9.0)) * np.arange(V) / 4.0)
    np.testing.assert_allclose(logits[0], expect, rtol=1e-12)


def test_stack_with_silent_sublayers():
    """With hidden_states_scale = 0 on both merges of every block, each
    block maps the stream to ((x + a.rb) * a.rs + m.rb) * m.rs (each merge
    rounded to fp32), block after block in order."""
    cfg = get_config("tiny").with_(seq=6)
    blocks = []
    for i in range(3):
        W = dict(gen_block_weights(cfg, block=i))
        for m in ("merge_a", "merge_m"):
            t = W[m].clone()
            t[1] = 0.0
            W[m] = t
        blocks.append(W)
    V = cfg.vocab
    extra = {"embed": torch.randn(V, cfg.hidden, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16),
             "final_norm_w": torch.ones(cfg.hidden, dtype=torch.bfloat16)}
    ids = np.array([[1, 2, 3, 4, 5, 6]])
    out = Z.stack_prefill(cfg, blocks, extra, ids)
    _, x = Z.embed(cfg, extra["embed"], ids)
    for W in blocks:
        a, m = Z.as64(W["merge_a"]), Z.as64(W["merge_m"])
        x = Z.round_f32((x + a[2]) * a[3])
        x = Z.round_f32((x + m[2]) * m[3])
    np.testing.assert_array_equal(out["final_stream"], x)


def test_prefill_rows_equals_full_prefill():
    """The windowed evaluation of a row range (used for long sequences)
    equals the full prefill at those rows, including ranges whose window and
    conv history start mid-sequence."""
    cfg = get_config("tiny").with_(seq=120, window=20)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    full = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"])
    for r0, r1 in ((0, 5), (30, 47), (100, 120), (21, 22)):
        part = Z.block_prefill_rows(cfg, W, inp["x"][0], r0, r1, inp["router_state_in"][0])
        for key in ("layer_output", "router_state", "attention_premix", "mlp_output"):
            np.testing.assert_allclose(part[key], full[key][0, r0:r1], rtol=1e-9, atol=1e-9, err_msg=key)
        np.testing.assert_array_equal(part["expert_cls"], full["expert_cls"][0, r0:r1])
        np.testing.assert_allclose(part["attention_keys"].transpose(1, 0, 2),
                                   full["attention_keys"][0][:, r0:r1], rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- carried router state

def _carry_case(block_idx):
    """The hand-worked carried-state example through the oracle's mlp half."""
    ex = _load("worked_examples.json")["router_state_carry"]
    R, H, E = ex["router_hidden"], ex["hidden"], ex["n_experts"]
    cfg = get_config("tiny").with_(hidden=H, router_hidden=R, n_experts=E, inter=1, rms_eps=ex["rms_eps"])
    W = {"ln2_w": np.array(ex["ln2_w"]), "router_down_w": np.array(ex["router_down_w"]),
         "router_down_b": np.array(ex["router_down_b"]), "router_state_scale": np.array(ex["router_state_scale"]),
         "router_norm_w": np.ones(R), "fc1_w": np.eye(R), "fc1_b": np.zeros(R), "fc2_w": np.eye(R),
         "fc2_b": np.zeros(R), "out_w": np.eye(R)[:E + 1], "balancing": np.zeros(E + 1),
         "w_gate_up": np.zeros((E, 2, H)), "w_down": np.zeros((E, H, 1)),
         "merge_m": np.array([[0.0] * H, [1.0] * H, [0.0] * H, [1.0] * H])}
    h = np.array([ex["stream_h"]])
    rin = np.array([ex["router_state_in"]])
    return ex, Z._mlp_half(cfg, W, h, rin, block_idx, np.ones(1, dtype=bool))


def test_router_state_carry_worked_example():
    """Block > 0: the state out is down_proj + bias + prev * router_states_scale
    (after the add, the scale on the previous state), and the router MLP reads
    that same state: its logits are gelu(gelu(rmsnorm(state))) for identity
    fc1 / fc2 / out_proj, computed here with math.erf (zaya page, 'One expert
    per token, chosen beside a skip class')."""
    ex, o = _carry_case(block_idx=1)
    np.testing.assert_array_equal(o["router_state"][0], ex["state_out_block1"])
    g = lambda x: 0.5 * x * (1 + math.erf(x / math.sqrt(2)))
    r = np.array(ex["state_out_block1"])
    z = r / math.sqrt(np.mean(r * r))
    np.testing.assert_allclose(o["router_logits"][0], [np.float32(g(g(v))) for v in z], rtol=1e-6)


def test_router_state_not_carried_on_block0():
    """Block 0 adds no carried state, even when one is passed in."""
    ex, o = _carry_case(block_idx=0)
    np.testing.assert_array_equal(o["router_state"][0], ex["state_out_block0"])


def _silent_expert_stack(cfg, n_blocks, scale_zero=False):
    """Blocks whose experts output zero (w_down = 0), so the stream does not
    depend on the routing and only the carried router state links the
    blocks' routers."""
    blocks = []
    for i in range(n_blocks):
        W = dict(gen_block_weights(cfg, block=i))
        W["w_down"] = torch.zeros_like(W["w_down"])
        if scale_zero:
            W["router_state_scale"] = torch.zeros_like(W["router_state_scale"])
        blocks.append(W)
    return blocks


def _bump_block0_router(blocks):
    out = [dict(W) for W in blocks]
    out[0]["router_down_b"] = out[0]["router_down_b"] + 0.5
    return out


def test_router_state_reaches_every_later_block():
    """An edit to block 0's routing input (its down_proj bias) changes the
    router logits of blocks 1 and 2 through the carried state; with
    router_states_scale = 0 on every block the later blocks' logits are
    bit-identical (zaya page, 'One expert per token ...': the state carries
    from block to block)."""
    cfg = get_config("tiny").with_(seq=12, batch=1)
    ids = np.arange(1, 13)[None, :] * 7 % cfg.vocab
    extra = {"embed": torch.randn(cfg.vocab, cfg.hidden, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16),
             "final_norm_w": torch.ones(cfg.hidden, dtype=torch.bfloat16)}

    def logits_per_block(blocks):
        te, x = Z.embed(cfg, extra["embed"], ids)
        r, out = None, []
        for i, W in enumerate(blocks):
            o = Z.block_prefill(cfg, W, x, None, r, block_idx=i)
            x, r = o["layer_output"], o["router_state"]
            out.append((o["router_logits"], o["layer_output"]))
        return out

    for scale_zero in (False, True):
        base = _silent_expert_stack(cfg, 3, scale_zero)
        a = logits_per_block(base)
        b = logits_per_block(_bump_block0_router(base))
        assert not np.array_equal(a[0][0], b[0][0])            # block 0's own router sees the edit
        for i in (1, 2):
            np.testing.assert_array_equal(a[i][1], b[i][1])     # the stream is the same
            if scale_zero:
                np.testing.assert_array_equal(a[i][0], b[i][0])
            else:
                assert (a[i][0] != b[i][0]).any(axis=-1).all(), i   # every token's logits moved


def test_router_state_chain_in_decode():
    """The decode stack chains the router state the same way: block 2's
    router logits follow an edit to block 0's down_proj bias only through a
    nonzero router_states_scale."""
    cfg = get_config("tiny").with_(seq=10, batch=2)
    extra = {"embed": torch.randn(cfg.vocab, cfg.hidden, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16),
             "final_norm_w": torch.ones(cfg.hidden, dtype=torch.bfloat16)}
    ids = (np.arange(20).reshape(2, 10) * 5 + 1) % cfg.vocab
    for scale_zero in (False, True):
        base = _silent_expert_stack(cfg, 3, scale_zero)
        pre = Z.stack_prefill(cfg, base, extra, ids)
        states = [dict(s, cache_len=s["cache_len"]) for s in pre["states"]]
        for s in states:
            s["k_cache"] = np.concatenate([s["k_cache"], np.zeros_like(s["k_cache"][:, :, :1])], axis=2)
            s["v_cache"] = np.concatenate([s["v_cache"], np.zeros_like(s["v_cache"][:, :, :1])], axis=2)
        new_ids = np.array([3, 9])

        def last_block_logits(blocks):
            te, x = Z.embed(cfg, extra["embed"], new_ids)
            r = None
            for i, W in enumerate(blocks):
                o = Z.block_decode(cfg, W, x, states[i], r, block_idx=i)
                x, r = o["layer_output"], o["router_state"]
            return o["router_logits"]

        a = last_block_logits(base)
        b = last_block_logits(_bump_block0_router(base))
        if scale_zero:
            np.testing.assert_array_equal(a, b)
        else:
            assert (a != b).any(axis=-1).all()


# ---------------------------------------------------------------- hybrid sliding / full blocks

def test_hybrid_blocks_window_reach():
    """With sliding_period = 2, sliding_phase = 1 (ZAYA1-74B-preview: a
    window on every other block; zaya page, 'Queries and keys are convolved
    ...', last sentence), an odd block keeps the window's reach (outputs at
    i >= t+W+2 bit-identical after perturbing token t), an even block
    attends to every earlier token (the output far beyond the window moves),
    and a stack without the setting slides on every block."""
    cfg = get_config("tiny").with_(seq=48, window=8, sliding_period=2, sliding_phase=1)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    t = 3
    far = t + cfg.window + 20
    for bidx, slides in ((1, True), (3, True), (0, False), (2, False)):
        assert (Z.block_window(cfg, bidx) == cfg.window) == slides
        o = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"], block_idx=bidx)
        x2 = inp["x"].clone()
        x2[0, t] += 1.0
        o2 = Z.block_prefill(cfg, W, x2, None, inp["router_state_in"], block_idx=bidx)
        same = np.array_equal(o2["attention_premix"][0, t + cfg.window + 2:], o["attention_premix"][0, t + cfg.window + 2:])
        assert same == slides, bidx
        assert np.array_equal(o2["attention_premix"][0, far], o["attention_premix"][0, far]) == slides, bidx
    plain = cfg.with_(sliding_period=0)
    assert all(Z.block_window(plain, b) == cfg.window for b in range(4))


def test_hybrid_full_block_is_plain_causal():
    """A full-attention block equals the same block with a window longer
    than the sequence, and its windowed row evaluation (keys back to 0)
    equals the full prefill at those rows."""
    cfg = get_config("tiny").with_(seq=60, window=8, sliding_period=2, sliding_phase=1)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    o = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"], block_idx=2)
    ref = Z.block_prefill(cfg.with_(window=10**6, sliding_period=0), W, inp["x"], None, inp["router_state_in"],
                          block_idx=2)
    np.testing.assert_array_equal(o["layer_output"], ref["layer_output"])
    part = Z.block_prefill_rows(cfg, W, inp["x"][0], 40, 60, inp["router_state_in"][0], block_idx=2)
    np.testing.assert_allclose(part["layer_output"], o["layer_output"][0, 40:60], rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- two-stage conv_qk

def test_conv_two_stage_worked_example():
    """The printout's two causal convolutions (depthwise k=2, then grouped
    k=2), hand-worked for one group of two channels, fresh and with a
    conv_state history, and for two groups of one channel."""
    ex = _load("worked_examples.json")["conv_two_stage"]
    dw, db = np.array(ex["dw_taps_t-1_t"]), np.array(ex["db"])
    gw = np.stack([np.array(ex["gw_tap_t-1"]), np.array(ex["gw_tap_t"])], axis=-1)   # [out, in, tap]
    u = np.array(ex["u"])
    y = Z.causal_conv_two_stage(u, dw, db, gw, np.array(ex["gb"]), np.zeros((2, 2)), 1)
    np.testing.assert_allclose(y, ex["y_fresh"], atol=1e-12)
    y = Z.causal_conv_two_stage(u, dw, db, gw, np.array(ex["gb"]), np.array(ex["hist"]), 1)
    np.testing.assert_allclose(y, ex["y_with_state"], atol=1e-12)
    g2 = ex["two_groups"]
    y = Z.causal_conv_two_stage(u, dw, db, np.array(g2["gw"]), np.array(g2["gb"]), np.zeros((2, 2)), 2)
    np.testing.assert_allclose(y, g2["y_fresh"], atol=1e-12)


def test_conv_two_stage_reduces_to_the_depthwise_conv():
    """With the grouped stage the identity on the current token (zero on the
    previous one, no bias), the two-stage conv is the depthwise conv of
    width 2: the width-3 conv with taps (0, dw0, dw1), itself pinned above."""
    rng = np.random.default_rng(7)
    T, C, G = 9, 12, 3
    u, hist = rng.standard_normal((T, C)), rng.standard_normal((2, C))
    dw, db = rng.standard_normal((C, 2)), rng.standard_normal(C)
    gw = np.zeros((C, C // G, 2))
    for o in range(C):
        gw[o, o % (C // G), 1] = 1.0
    y = Z.causal_conv_two_stage(u, dw, db, gw, np.zeros(C), hist, G)
    ref = Z.causal_conv(u, np.concatenate([np.zeros((C, 1)), dw], axis=1), db, hist)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_conv_two_stage_block_reach_and_decode():
    """A block with the two-stage conv keeps the width-3 reach (outputs at
    i >= t+W+2 bit-identical after perturbing token t, the one at t+W+1
    moved), and prefill(S) then decode equals prefill(S+1) at S."""
    cfg = get_config("tiny").with_(seq=48, conv_width=2, conv_groups=5)
    W = gen_block_weights(cfg)
    inp = gen_prefill_inputs(cfg)
    o = Z.block_prefill(cfg, W, inp["x"], None, inp["router_state_in"])
    t = 4
    x2 = inp["x"].clone()
    x2[0, t] += 0.5
    o2 = Z.block_prefill(cfg, W, x2, None, inp["router_state_in"])
    edge = t + cfg.window + 1
    np.testing.assert_array_equal(o2["attention_premix"][0, edge + 1:], o["attention_premix"][0, edge + 1:])
    assert not np.array_equal(o2["attention_premix"][0, edge], o["attention_premix"][0, edge])
    S = 30
    pre = Z.block_prefill(cfg.with_(seq=S), W, inp["x"][:, :S], None, inp["router_state_in"][:, :S])
    st = {k: v for k, v in pre["state"].items()}
    st["k_cache"] = np.concatenate([st["k_cache"], np.zeros_like(st["k_cache"][:, :, :1])], axis=2)
    st["v_cache"] = np.concatenate([st["v_cache"], np.zeros_like(st["v_cache"][:, :, :1])], axis=2)
    dec = Z.block_decode(cfg, W, inp["x"][:, S], st, inp["router_state_in"][:, S],
                         force_cls=o["expert_cls"][:, S])
    full = Z.block_prefill(cfg.with_(seq=S + 1), W, inp["x"][:, :S + 1], None, inp["router_state_in"][:, :S + 1],
                           force_cls=o["expert_cls"][:, :S + 1])
    np.testing.assert_allclose(dec["layer_output"], full["layer_output"][:, S], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(dec["attention_keys"], full["attention_keys"][:, :, S], rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- fp8 KV cache

def _e4m3_table():
    """Every finite OCP FP8 E4M3 code and its value, decoded from the format's
    definition: sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN (no infinities)."""
    codes, vals = [], []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        codes.append(code)
        vals.append(-v if s else v)
    return np.array(codes), np.array(vals)


def test_e4m3_rounding_against_the_format():
    """round_e4m3 against the code table: every finite value is a fixed point;
    a point just inside either neighbour's half goes to that neighbour; an
    exact midpoint goes to the neighbour with the even mantissa; magnitudes
    past 448 saturate; the largest value is 448 and the smallest subnormal
    2^-9 (NVFP4 README, "--kv-cache-dtype fp8": keys and values stored in
    8-bit floating point)."""
    codes, vals = _e4m3_table()
    assert vals.max() == 448.0 and vals[(vals > 0)].min() == 2.0 ** -9
    np.testing.assert_array_equal(Z.round_e4m3(vals), vals)
    pos = np.unique(vals[vals >= 0])
    code_of = {v: c for c, v in zip(codes, vals) if v >= 0}
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = 0.5 * (lo + hi)
        gap = hi - lo
        assert Z.round_e4m3(mid - gap * 1e-3) == lo
        assert Z.round_e4m3(mid + gap * 1e-3) == hi
        even = lo if code_of[lo] % 2 == 0 else hi
        assert Z.round_e4m3(mid) == even, (lo, hi)
        assert Z.round_e4m3(-mid) == -even
    for big in (448.5, 463.9, 464.0, 500.0, 1e9):
        assert Z.round_e4m3(big) == 448.0 and Z.round_e4m3(-big) == -448.0


def test_fp8_cache_prefill_and_decode(tiny):
    """kv_fp8: the prompt attends over its bf16 keys / values, so every
    prefill output is the bf16 cache's; the cache then holds E4M3 values
    within half a step of the bf16 ones; a decode step computes its token's
    keys as the bf16 run does and writes them in E4M3 before attending over
    the cache, so its attention differs from the bf16 decode's by about
    E4M3's precision (three mantissa bits), no more."""
    cfg, W, inp, out = tiny
    c8 = cfg.with_(kv_fp8=1)
    x, r = inp["x"], inp["router_state_in"]
    S = cfg.seq
    p16 = Z.block_prefill(cfg, W, x[:, :S - 1], None, r[:, :S - 1])
    p8 = Z.block_prefill(c8, W, x[:, :S - 1], None, r[:, :S - 1])
    for key in ("layer_output", "router_state", "attention_output", "mlp_output"):
        np.testing.assert_array_equal(p8[key], p16[key])
    for key in ("k_cache", "v_cache"):
        c16, c8v = p16["state"][key], p8["state"][key]
        np.testing.assert_array_equal(Z.round_e4m3(c8v), c8v)
        step = np.ldexp(1.0, np.maximum(np.frexp(np.abs(c16) + (c16 == 0))[1] - 1, -6) - 3)
        assert (np.abs(c8v - c16) <= 0.5 * step + 1e-300).all()
        assert (c8v != c16).any()
    cap = S + 2

    def state_of(st):
        kc = np.zeros((1, cfg.n_kv, cap, cfg.head_dim))
        vc = np.zeros_like(kc)
        kc[:, :, :S - 1] = st["k_cache"]
        vc[:, :, :S - 1] = st["v_cache"]
        return dict(k_cache=kc, v_cache=vc, conv_state=st["conv_state"], prev_hs=st["prev_hs"],
                    cache_len=st["cache_len"])

    d8 = Z.block_decode(c8, W, x[:, S - 1], state_of(p8["state"]), r[:, S - 1])
    d16 = Z.block_decode(cfg, W, x[:, S - 1], state_of(p16["state"]), r[:, S - 1])
    # the token's own K / V entered the cache rounded to E4M3
    np.testing.assert_array_equal(d8["state"]["k_cache"][:, :, S - 1], Z.round_e4m3(d16["state"]["k_cache"][:, :, S - 1]))
    np.testing.assert_array_equal(d8["attention_keys"], d16["attention_keys"])
    rel = np.abs(d8["attention_premix"] - d16["attention_premix"]).max() / np.abs(d16["attention_premix"]).max()
    assert 1e-4 < rel < 0.1, rel


# ---------------------------------------------------------------- FP8 experts

def test_e4m3_decode_against_the_format():
    """e4m3_decode of every code equals the table decoded from the format's
    definition, and every finite value is a fixed point of round_e4m3."""
    codes, vals = _e4m3_table()
    np.testing.assert_array_equal(Z.e4m3_decode(codes), vals)
    assert np.isnan(Z.e4m3_decode([0x7F, 0xFF])).all()
    np.testing.assert_array_equal(Z.round_e4m3(Z.e4m3_decode(codes)), vals)


def test_fp8_expert_brute_force():
    """expert_ffn_fp8 on tiny shapes against a per-element loop: the input
    quantised as E4M3(x / s_in), each gate / up dot product of E4M3 values
    times s_in and its row's scale, SwiGLU, the activation quantised as
    E4M3(act / s_act), the down dot products times s_act and their rows'
    scales (an FP8 W8A8 expert; NVFP4 README, "Quantization details", for
    the pages' quantised experts)."""
    rng = np.random.default_rng(7)
    T, H, I = 3, 5, 4
    codes_gu = rng.integers(0, 256, size=(2 * I, H))
    codes_dn = rng.integers(0, 256, size=(H, I))
    codes_gu[(codes_gu & 0x7F) == 0x7F] = 0x12     # no NaN codes
    codes_dn[(codes_dn & 0x7F) == 0x7F] = 0x21
    wgu, wdn = Z.e4m3_decode(codes_gu), Z.e4m3_decode(codes_dn)
    sgu = rng.uniform(0.001, 0.01, size=2 * I)
    sdn = rng.uniform(0.001, 0.01, size=H)
    s_in, s_act = 2.0 ** -5, 2.0 ** -3
    x = rng.normal(0, 2.0, size=(T, H))
    got = Z.expert_ffn_fp8(x, wgu, sgu, wdn, sdn, s_in, s_act, I)
    for t in range(T):
        xq = [float(Z.round_e4m3(x[t, h] / s_in)) for h in range(H)]
        gu = [sum(xq[h] * wgu[j, h] for h in range(H)) * s_in * sgu[j] for j in range(2 * I)]
        act = [gu[i] / (1.0 + math.exp(-gu[i])) * gu[I + i] for i in range(I)]
        aq = [float(Z.round_e4m3(a / s_act)) for a in act]
        for o in range(H):
            want = sum(aq[i] * wdn[o, i] for i in range(I)) * s_act * sdn[o]
            assert abs(got[t, o] - want) <= 1e-12 * max(1.0, abs(want)), (t, o)
