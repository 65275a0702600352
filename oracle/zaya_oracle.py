"""CPU oracle of the ZAYA1 decoder block -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module.  The product path (``top_moe_block_b200``) never
imports, links or calls it, and shares no code with it: the two meet only in
the seeded inputs drawn by ``synthetic/``.

What it computes is the block as the nnterp encyclopedia's "zaya" family page
defines it (sections "The block, in order", "The stream is float32 whatever
the load", "Queries and keys are convolved, normed to sqrt(head_dim) and the
keys scaled", "One expert per token, chosen beside a skip class", and the
family-module docstring), with the conv_state / prev_hs state contract of the
ZAYA1-8B-JANGTQ2 README ("Architecture Summary").

Precision.  Arithmetic is float64 (numpy), written as plain per-definition
steps; a matmul is the only library primitive used for a contraction.  Values
are rounded where the pages fix a dtype and nowhere else:

* the residual stream is float32 (zaya page, "The stream is float32 whatever
  the load"): every merge result and the embedding are rounded to fp32;
* each norm casts the stream to its weight's dtype (bf16) first, and its
  output is in that dtype (same section);
* token_embeddings, attention_output, mlp_output and logits keep the load's
  dtype, bf16 (same section);
* q_proj / k_proj / v_proj_current / v_proj_delayed outputs are in the load
  dtype (bf16), as every Linear's under a bf16 load; this is also what the
  conv_state [B,1280,2] carries (JANGTQ2 README, "Architecture Summary");
* the KV cache holds bf16 keys and values (llm-atlas card, "kvCacheText":
  40 KiB per token = 40 layers x (K+V) x 2 heads x 128 x 2 bytes), so keys
  and values are rounded to bf16 where they enter the attention; with the
  fp8 cache option (``kv_fp8``, the NVFP4 README's ``--kv-cache-dtype fp8``)
  the cache holds them rounded on to E4M3 and a decode step reads those;
* with the FP8 expert option (``expert_fp8``) the experts take E4M3 weight
  codes with per-row scales and quantise their inputs to E4M3 with static
  scales (``expert_ffn_fp8``);
* the router's choice is taken on float32 softmax scores
  (``logits.float().softmax(-1)``, zaya page, "One expert per token"), so the
  logits are rounded to fp32 and the softmax, the bias add and the argmax run
  in float32.

Readings of points the pages leave open are the fields of
``synthetic.BlockConfig`` and the notes on each function below.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

# ---------------------------------------------------------------------------
# dtype rounding at the points the pages fix
# ---------------------------------------------------------------------------


def as64(t) -> np.ndarray:
    """Any torch tensor / array (bf16, fp32, ...) as a float64 ndarray."""
    if hasattr(t, "detach"):
        t = t.detach().cpu()
        if str(t.dtype) in ("torch.bfloat16", "torch.float16"):
            t = t.float()
        t = t.numpy()
    return np.asarray(t, dtype=np.float64)


def round_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 (ties to even) from the fp32 value."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


E4M3_MAX = 448.0   # the largest finite OCP FP8 E4M3 value, 1.75 * 2^8


def round_e4m3(x) -> np.ndarray:
    """Round to the nearest OCP FP8 E4M3 value (4 exponent bits, bias 7, 3
    mantissa bits; normals down to 2^-6, subnormals k * 2^-9), ties to an
    even mantissa, magnitudes beyond the largest finite value saturating to
    +-448 (the fp8 KV cache of the NVFP4 README's serving command,
    "--kv-cache-dtype fp8", stores keys and values in this format).

    The step between neighbours is 2^(e - 3) in the binade [2^e, 2^(e+1))
    for e >= -6 and 2^-9 below it; rounding |x| / step to an integer (ties
    to even) and scaling back lands on the nearest value, a carry into the
    next binade included."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))      # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)
    step = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.round(a / step) * step                    # numpy rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(q, x))


def e4m3_decode(codes) -> np.ndarray:
    """Values of OCP FP8 E4M3 codes (uint8): sign bit, 4 exponent bits (bias
    7), 3 mantissa bits; exponent 0 holds the subnormals m/8 * 2^-6; code
    S.1111.111 is NaN."""
    c = np.asarray(codes).astype(np.int64)
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    v = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(s == 1, -v, v)


def cache_kv(cfg, t):
    """Keys / values as the cache holds them: bf16, or with ``cfg.kv_fp8``
    the bf16 value rounded on to E4M3."""
    return round_e4m3(t) if getattr(cfg, "kv_fp8", 0) else t


# ---------------------------------------------------------------------------
# elementwise pieces
# ---------------------------------------------------------------------------


def silu(x):
    """SiLU, x * sigmoid(x) (ZayaExperts act_fn, zaya page "Printout")."""
    return x / (1.0 + np.exp(-x))


def gelu(x):
    """Exact GELU, x * Phi(x) (router_mlp act_fn, GELU(approximate='none'))."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def rms_norm(x, w, eps):
    """w * x / sqrt(mean(x^2) + eps) over the last axis (ZayaRMSNorm)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return w * (x / np.sqrt(ms + eps))


def block_norm(stream, w, eps):
    """A block norm as the zaya page states it: cast the fp32 stream to the
    weight's dtype (bf16), norm, output in bf16."""
    return round_bf16(rms_norm(round_bf16(stream), w, eps))


def merge(o, r, p):
    """ZayaResidualScaling: (o + hidden_states_bias) * hidden_states_scale
    + (r + residual_bias) * residual_scale (zaya page, "The block, in
    order").  p rows are (hb, hs, rb, rs).  Returns (contribution in bf16,
    merged stream in fp32): the contribution (attention_output / mlp_output)
    keeps the load dtype and the stream is fp32."""
    hb, hs, rb, rs = p[0], p[1], p[2], p[3]
    contrib = round_bf16((o + hb) * hs)
    return contrib, round_f32(contrib + (r + rb) * rs)


# ---------------------------------------------------------------------------
# CCA attention pieces (zaya page, "Queries and keys are convolved ...")
# ---------------------------------------------------------------------------


def causal_conv(u, w, b, hist):
    """Depthwise causal conv over tokens, width 3, per channel c:
    y[t,c] = w[c,0]*u[t-2,c] + w[c,1]*u[t-1,c] + w[c,2]*u[t,c] + b[c].
    u [T,C]; hist [2,C] holds u[-2], u[-1] (zeros for a fresh sequence,
    conv_state in decode)."""
    ext = np.concatenate([hist, u], axis=0)
    T = u.shape[0]
    return w[:, 0] * ext[0:T] + w[:, 1] * ext[1:T + 1] + w[:, 2] * ext[2:T + 2] + b


def causal_conv_two_stage(u, dw, db, gw, gb, hist, groups):
    """ZayaCCAProjection's two causal convolutions as the ZAYA1-8B printout
    lists them (zaya page, "Printout": conv_qk_depthwise Conv1d(C, C, k=2,
    groups=C), then conv_qk_grouped Conv1d(C, C, k=2, groups=G); "Queries
    and keys are convolved ...": the current and two previous tokens):

      z[s, c] = dw[c, 0] u[s-1, c] + dw[c, 1] u[s, c] + db[c]
      y[t, o] = sum_i gw[o, i, 0] z[t-1, g(o) Cg + i] + gw[o, i, 1] z[t, g(o) Cg + i] + gb[o]

    with Cg = C / G and g(o) = o // Cg (PyTorch's Conv1d weight layout
    [out, in / groups, k]).  u before the sequence is ``hist`` (u[-2],
    u[-1]: zeros for a fresh sequence, conv_state in decode), and z[-1] is
    computed from it the same way, so prefill and decode agree.  u [T,C];
    hist [2,C]; dw [C,2]; gw [C,Cg,2]."""
    ext = np.concatenate([hist, u], axis=0)                  # u[-2] .. u[T-1]
    T, C = u.shape
    z = dw[:, 0] * ext[:-1] + dw[:, 1] * ext[1:] + db       # z[-1] .. z[T-1]
    Cg = C // groups
    y = np.empty((T, C))
    for g in range(groups):
        sl = slice(g * Cg, (g + 1) * Cg)
        y[:, sl] = z[:-1, sl] @ gw[sl, :, 0].T + z[1:, sl] @ gw[sl, :, 1].T + gb[sl]
    return y


def cca_mean_residual(q_pre, k_pre, n_q, n_kv):
    """Each query head gets the mean of its own projection and its key head's
    projection; each key head gets the mean of those query residuals over the
    query heads it serves.  q_pre [T,nq,d], k_pre [T,nkv,d]."""
    rep = n_q // n_kv
    q_res = np.empty_like(q_pre)
    for h in range(n_q):
        q_res[:, h] = 0.5 * (q_pre[:, h] + k_pre[:, h // rep])
    k_res = np.empty_like(k_pre)
    for g in range(n_kv):
        k_res[:, g] = q_res[:, g * rep:(g + 1) * rep].mean(axis=1)
    return q_res, k_res


def l2_to_sqrt_d(x, eps):
    """Normalise each head vector (last axis) to length sqrt(d)."""
    d = x.shape[-1]
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x * math.sqrt(d) / np.maximum(n, eps)


def rope_inv_freq(rot, theta):
    """inv_freq[i] = theta^(-2i/rot), i < rot/2, held in fp32 as Llama's
    rotary does."""
    i = np.arange(0, rot, 2, dtype=np.float64)
    return round_f32(1.0 / (theta ** (i / rot)))


def rope(x, pos, rot, theta):
    """Rotate the first ``rot`` dims of each head, pairing dim i with
    i + rot/2 (Llama's rotate-half), angle = fp32(pos * inv_freq[i]).
    x [T,heads,d]; pos [T]."""
    if rot == 0:
        return x
    half = rot // 2
    ang = round_f32(np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(rot, theta)[None, :])
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    y = x.copy()
    x1 = x[..., :half]
    x2 = x[..., half:rot]
    y[..., :half] = x1 * c - x2 * s
    y[..., half:rot] = x2 * c + x1 * s
    return y


def attention(q, k, v, q_pos, k_pos, k_valid, window, scale):
    """Eager softmax attention of one sequence, GQA with kv head h // rep.
    q [Tq,nq,d], k/v [Tk,nkv,d]; key j is visible to query i iff
    0 <= pos_i - pos_j < window and key j is not padding.  A query with no
    visible key (a padding row) outputs 0."""
    Tq, nq, d = q.shape
    nkv = k.shape[1]
    rep = nq // nkv
    dist = np.asarray(q_pos)[:, None] - np.asarray(k_pos)[None, :]
    vis = (dist >= 0) & (dist < window) & np.asarray(k_valid, dtype=bool)[None, :]
    any_vis = vis.any(axis=1)
    out = np.zeros((Tq, nq, d))
    for h in range(nq):
        g = h // rep
        s = (q[:, h] @ k[:, g].T) * scale
        s = np.where(vis, s, -np.inf)
        m = np.where(any_vis, s.max(axis=1), 0.0)
        p = np.where(vis, np.exp(s - m[:, None]), 0.0)
        den = p.sum(axis=1)
        p = p / np.where(den > 0, den, 1.0)[:, None]
        out[:, h] = p @ v[:, g]
    return out


FULL_ATTENTION = 1 << 62   # a window no sequence reaches


def block_window(cfg, block_idx):
    """Keys (its own included) a query of block ``block_idx`` attends over.
    Every block slides over ``cfg.window`` keys unless ``cfg.sliding_period``
    is set: then only the blocks with block_idx % period == phase slide and
    the others attend to every earlier token -- ZAYA1-74B-preview's hybrid,
    a 4097-token window on every other block (zaya page, "Queries and keys
    are convolved ...", last sentence)."""
    period = getattr(cfg, "sliding_period", 0)
    if period <= 0 or block_idx % period == cfg.sliding_phase:
        return cfg.window
    return FULL_ATTENTION


# ---------------------------------------------------------------------------
# router and experts (zaya page, "One expert per token, chosen beside a skip
# class"; "Printout" for the router's modules)
# ---------------------------------------------------------------------------


def router_mlp(r, W, eps):
    """router_mlp: RMSNorm(R) -> fc1 -> GELU -> fc2 -> GELU -> out_proj
    (no bias).  Returns router_logits [T,E+1] rounded to fp32."""
    z = rms_norm(r, as64(W["router_norm_w"]), eps)
    g1 = gelu(z @ as64(W["fc1_w"]).T + as64(W["fc1_b"]))
    g2 = gelu(g1 @ as64(W["fc2_w"]).T + as64(W["fc2_b"]))
    return round_f32(g2 @ as64(W["out_w"]).T)


def select(logits, balancing, n_experts):
    """Scoring and top-1 choice, in float32: p = softmax(logits); class
    c = argmax(p + balancing_biases), the lowest index on exact ties; the
    weight is p[c] (not renormalised).  A token that picks skip (the last
    class) gets index 0 and weight 0.  Returns (cls, idx, w, p, gap), gap
    being the relative distance between the two best selection scores."""
    l32 = np.asarray(logits, dtype=np.float32)
    m = l32.max(axis=-1, keepdims=True)
    e = np.exp(l32 - m, dtype=np.float32)
    p = (e / e.sum(axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)
    s = (p + np.asarray(balancing, dtype=np.float32)[None, :]).astype(np.float32)
    cls = np.argmax(s, axis=-1)
    srt = np.sort(s.astype(np.float64), axis=-1)
    gap = (srt[:, -1] - srt[:, -2]) / np.maximum(np.abs(srt[:, -1]), 1e-30)
    w = p[np.arange(len(cls)), cls].astype(np.float64)
    skip = cls == n_experts
    idx = np.where(skip, 0, cls)
    w = np.where(skip, 0.0, w)
    return cls, idx.astype(np.int32), w, p, gap


def expert_ffn(x, w_gate_up_e, w_down_e, inter):
    """SwiGLU expert: down(silu(gate x) * up x); w_gate_up_e rows [0,I) are
    the gate, [I,2I) the up projection."""
    gu = x @ w_gate_up_e.T
    return (silu(gu[:, :inter]) * gu[:, inter:]) @ w_down_e.T


def expert_ffn_fp8(x, wgu_e, sgu_e, wdn_e, sdn_e, s_in, s_act, inter):
    """The SwiGLU expert with FP8 (E4M3) weights and activations, the scheme
    of an FP8 W8A8 checkpoint (the pages' own deployments quantise the
    experts, NVFP4 README "Quantization details"): weights are
    E4M3 values wgu_e [2I,H], wdn_e [H,I] with one fp32 scale per output row
    (sgu_e [2I], sdn_e [H]); each input is quantised with a static per-expert
    scale, x_q = E4M3(x / s_in) and act_q = E4M3(act / s_act); a product
    is the E4M3 dot product times its input's and its row's scales."""
    xq = round_e4m3(x / s_in)
    gu = (xq @ wgu_e.T) * (s_in * sgu_e[None, :])
    act = silu(gu[:, :inter]) * gu[:, inter:]
    aq = round_e4m3(act / s_act)
    return (aq @ wdn_e.T) * (s_act * sdn_e[None, :])


def moe(cfg, W, m_in, cls, w):
    """routed_output: w_t * expert_{c_t}(m_in_t); zero where c_t is skip."""
    E, I = cfg.n_experts, cfg.inter
    y = np.zeros_like(m_in)
    wgu = W["w_gate_up"]
    wdn = W["w_down"]
    fp8 = getattr(cfg, "expert_fp8", 0)
    for e in range(E):
        rows = np.nonzero(cls == e)[0]
        if rows.size == 0:
            continue
        if fp8:   # E4M3 codes with per-row scales and the expert's static input scales
            sc = as64(W["expert_act_scale"])[e]
            f = expert_ffn_fp8(m_in[rows], e4m3_decode(np.asarray(wgu[e])), as64(W["w_gate_up_scale"])[e],
                               e4m3_decode(np.asarray(wdn[e])), as64(W["w_down_scale"])[e], sc[0], sc[1], I)
        else:
            f = expert_ffn(m_in[rows], as64(wgu[e]), as64(wdn[e]), I)
        y[rows] = w[rows, None] * f
    return y


# ---------------------------------------------------------------------------
# the block
# ---------------------------------------------------------------------------


def _split_proj(cfg, proj):
    """Stacked projection rows: q (nq*d), k (nkv*d), v_current, v_delayed."""
    qd, kd, vh = cfg.q_dim, cfg.kv_dim, cfg.v_half
    return proj[:, :qd], proj[:, qd:qd + kd], proj[:, qd + kd:qd + kd + vh], proj[:, qd + kd + vh:]


def _values(cfg, vc, vd_prev):
    """Value head g = [v_current[g*d/2:(g+1)*d/2] (token t) ||
    v_delayed[g*d/2:(g+1)*d/2] (token t-1)]."""
    T = vc.shape[0]
    hd = cfg.head_dim // 2
    v = np.empty((T, cfg.n_kv, cfg.head_dim))
    for g in range(cfg.n_kv):
        v[:, g, :hd] = vc[:, g * hd:(g + 1) * hd]
        v[:, g, hd:] = vd_prev[:, g * hd:(g + 1) * hd]
    return v


def _qk(cfg, W, q_pre, k_pre, hist, pos):
    """conv_qk over q||k, CCA mean residual, qk_norm (+ temp), partial RoPE."""
    T = q_pre.shape[0]
    d = cfg.head_dim
    u = np.concatenate([q_pre, k_pre], axis=1)
    if getattr(cfg, "conv_groups", 0):
        y = causal_conv_two_stage(u, as64(W["conv_w"]), as64(W["conv_b"]), as64(W["conv2_w"]), as64(W["conv2_b"]),
                                  hist, cfg.conv_groups)
    else:
        y = causal_conv(u, as64(W["conv_w"]), as64(W["conv_b"]), hist)
    q = y[:, :cfg.q_dim].reshape(T, cfg.n_q, d)
    k = y[:, cfg.q_dim:].reshape(T, cfg.n_kv, d)
    if cfg.cca_mean_residual:
        q_res, k_res = cca_mean_residual(q_pre.reshape(T, cfg.n_q, d), k_pre.reshape(T, cfg.n_kv, d),
                                         cfg.n_q, cfg.n_kv)
        q = q + q_res
        k = k + k_res
    q = l2_to_sqrt_d(q, cfg.qk_norm_eps)
    k = l2_to_sqrt_d(k, cfg.qk_norm_eps) * as64(W["k_temp"])[None, :, None]
    q = rope(q, pos, cfg.rot_dim, cfg.rope_theta)
    k = rope(k, pos, cfg.rot_dim, cfg.rope_theta)
    return q, k, u


def _mlp_half(cfg, W, h, router_state_in, block_idx, real, force_cls=None):
    """post_attention_layernorm -> router (down_proj + carried state, MLP,
    scoring) -> experts -> merge 2.  Rows where ``real`` is False (padding)
    are routed to skip."""
    m_in = block_norm(h, as64(W["ln2_w"]), cfg.rms_eps)
    r = m_in @ as64(W["router_down_w"]).T + as64(W["router_down_b"])
    if block_idx > 0 and router_state_in is not None:
        r = r + router_state_in * as64(W["router_state_scale"])
    r = round_f32(r)
    logits = router_mlp(r, W, cfg.rms_eps)
    cls, idx, w, p, gap = select(logits, as64(W["balancing"]), cfg.n_experts)
    own_cls = cls.copy()
    if force_cls is not None:
        cls = np.asarray(force_cls).copy()
        skip = cls == cfg.n_experts
        idx = np.where(skip, 0, cls).astype(np.int32)
        w = np.where(skip, 0.0, p[np.arange(len(cls)), cls].astype(np.float64))
    pad = ~real
    cls = np.where(pad, cfg.n_experts, cls)
    idx = np.where(pad, 0, idx).astype(np.int32)
    w = np.where(pad, 0.0, w)
    routed = moe(cfg, W, m_in, cls, w)
    mlp_out, out = merge(routed, h, as64(W["merge_m"]))
    return dict(mlp_norm_output=m_in, router_state=r, router_logits=logits, expert_cls=cls,
                expert_indices=idx, expert_weights=w, router_probs=p, router_gap=gap,
                router_own_cls=own_cls, routed_output=routed, mlp_output=mlp_out, layer_output=out)


def block_prefill(cfg, W, x, attn_mask=None, router_state_in=None, block_idx=None, force_cls=None):
    """One block over fresh sequences (empty cache).

    x [B,S,H] fp32 stream; attn_mask [B,S] (1 = token, 0 = left padding) or
    None; router_state_in [B,S,R] or None.  Padding tokens take no part:
    their pre-conv q/k and their delayed-value input are zero, keys at pads
    are masked, pad queries output 0 and pads are routed to skip.
    Positions are 0..S-1 for every sequence.  Returns the taps (nnterp
    names, [B,S,...]) and the decode state the prefill leaves behind."""
    x = as64(x)
    B, S, H = x.shape
    bidx = cfg.block_idx if block_idx is None else block_idx
    mask = np.ones((B, S), dtype=bool) if attn_mask is None else as64(attn_mask) != 0
    rin = None if router_state_in is None else as64(router_state_in)
    d, nq, nkv = cfg.head_dim, cfg.n_q, cfg.n_kv
    taps = {k: [] for k in ("attention_norm_output", "attention_queries", "attention_keys",
                            "attention_values", "attention_premix", "attention_output", "layer_mid")}
    mlp_taps = []
    state = dict(k_cache=[], v_cache=[], conv_state=[], prev_hs=[])
    pos = np.arange(S)
    for b in range(B):
        real = mask[b]
        a_in = block_norm(x[b], as64(W["ln1_w"]), cfg.rms_eps)
        proj = round_bf16(a_in @ as64(W["w_qkv"]).T)
        q_pre, k_pre, vc, vd = _split_proj(cfg, proj)
        q_pre = q_pre * real[:, None]
        k_pre = k_pre * real[:, None]
        vd = vd * real[:, None]
        hist = np.zeros((2, cfg.qk_channels))
        q, k, u = _qk(cfg, W, q_pre, k_pre, hist, pos)
        vd_prev = np.concatenate([np.zeros((1, cfg.v_half)), vd[:-1]], axis=0)
        if not cfg.v_delayed:
            vd_prev = vd
        v = _values(cfg, vc, vd_prev)
        k = round_bf16(k)
        v = round_bf16(v)
        o = attention(q, k, v, pos, pos, real, block_window(cfg, bidx), cfg.scale)
        premix = o.reshape(S, nq * d)
        attn_o = premix @ as64(W["w_o"]).T
        attn_out, h = merge(attn_o, x[b], as64(W["merge_a"]))
        mt = _mlp_half(cfg, W, h, None if rin is None else rin[b], bidx, real,
                       None if force_cls is None else np.asarray(force_cls)[b])
        mlp_taps.append(mt)
        for name, val in (("attention_norm_output", a_in), ("attention_queries", q.transpose(1, 0, 2)),
                          ("attention_keys", k.transpose(1, 0, 2)), ("attention_values", v.transpose(1, 0, 2)),
                          ("attention_premix", premix), ("attention_output", attn_out), ("layer_mid", h)):
            taps[name].append(val)
        # the prompt attended over its bf16 keys and values above; the cache
        # keeps them in its own format (E4M3 with kv_fp8)
        state["k_cache"].append(cache_kv(cfg, k).transpose(1, 0, 2))
        state["v_cache"].append(cache_kv(cfg, v).transpose(1, 0, 2))
        last2 = np.concatenate([hist, u], axis=0)[-2:]          # pre-conv q||k at S-2, S-1
        state["conv_state"].append(last2.T)                     # [C, 2]
        state["prev_hs"].append(a_in[-1])
    out = {k: np.stack(v) for k, v in taps.items()}
    for key in mlp_taps[0]:
        out[key] = np.stack([mt[key] for mt in mlp_taps])
    out["layer_input"] = x
    out["state"] = {k: np.stack(v) for k, v in state.items()}
    out["state"]["cache_len"] = np.full(B, S, dtype=np.int64)
    return out


def block_prefill_rows(cfg, W, x, r0, r1, router_state_in=None, block_idx=None, force_cls=None):
    """The block outputs of rows [r0, r1) of one unpadded sequence, computed
    from only the tokens those rows depend on: keys back to r0 - window + 1
    and two more tokens of conv history.  Positions are the rows' own, so the
    result is the full prefill's at those rows (up to summation order).
    x [S,H]; router_state_in [S,R] or None; force_cls [r1-r0] or None.
    Returns taps of the rows (no decode state)."""
    x = as64(x)
    bidx = cfg.block_idx if block_idx is None else block_idx
    d, nq = cfg.head_dim, cfg.n_q
    window = block_window(cfg, bidx)
    lo = max(0, r0 - window + 1)         # first key any of the rows sees
    t0 = max(0, lo - 3)                  # plus the conv / delayed-value history
    seg = x[t0:r1]
    a_in = block_norm(seg, as64(W["ln1_w"]), cfg.rms_eps)
    proj = round_bf16(a_in @ as64(W["w_qkv"]).T)
    q_pre, k_pre, vc, vd = _split_proj(cfg, proj)
    pos = np.arange(t0, r1)
    q, k, u = _qk(cfg, W, q_pre, k_pre, np.zeros((2, cfg.qk_channels)), pos)
    vd_prev = np.concatenate([np.zeros((1, cfg.v_half)), vd[:-1]], axis=0)
    if not cfg.v_delayed:
        vd_prev = vd
    v = round_bf16(_values(cfg, vc, vd_prev))
    k = round_bf16(k)
    # rows whose conv / delayed-value history starts before t0 were computed with zeros
    # there: they are keys only if >= lo, and lo >= t0 + 2 whenever t0 > 0
    kl = lo - t0
    qi = np.arange(r0, r1) - t0
    o = attention(q[qi], k[kl:], v[kl:], np.arange(r0, r1), np.arange(lo, r1), np.ones(r1 - lo, dtype=bool),
                  window, cfg.scale)
    premix = o.reshape(r1 - r0, nq * d)
    attn_o = premix @ as64(W["w_o"]).T
    attn_out, h = merge(attn_o, x[r0:r1], as64(W["merge_a"]))
    rin = None if router_state_in is None else as64(router_state_in)[r0:r1]
    mt = _mlp_half(cfg, W, h, rin, bidx, np.ones(r1 - r0, dtype=bool), force_cls)
    out = dict(attention_norm_output=a_in[r0 - t0:], attention_premix=premix, attention_output=attn_out,
               layer_mid=h, layer_input=x[r0:r1], attention_keys=k[r0 - t0:], attention_values=v[r0 - t0:])
    out.update(mt)
    return out


def block_decode(cfg, W, x, state, router_state_in=None, block_idx=None, force_cls=None):
    """One new token per sequence through a block with a cache.

    x [B,H] fp32 stream; state: k_cache / v_cache [B,nkv,cap,d] (bf16
    values), conv_state [B,C,2] (pre-conv q||k at t-2, t-1), prev_hs [B,H]
    (attention_norm_output at t-1), cache_len [B] (the new token's
    position).  Returns the taps ([B,...]) and the updated state (copies)."""
    x = as64(x)
    B, H = x.shape
    bidx = cfg.block_idx if block_idx is None else block_idx
    d, nq, nkv = cfg.head_dim, cfg.n_q, cfg.n_kv
    kc = as64(state["k_cache"]).copy()
    vcache = as64(state["v_cache"]).copy()
    conv_state = as64(state["conv_state"]).copy()
    prev_hs = as64(state["prev_hs"]).copy()
    clen = np.asarray(state["cache_len"]).astype(np.int64).copy()
    rin = None if router_state_in is None else as64(router_state_in)
    a_in = block_norm(x, as64(W["ln1_w"]), cfg.rms_eps)
    proj = round_bf16(a_in @ as64(W["w_qkv"]).T)
    q_pre, k_pre, vc, _ = _split_proj(cfg, proj)
    vd_prev = round_bf16(prev_hs @ as64(W["w_qkv"])[cfg.q_dim + cfg.kv_dim + cfg.v_half:].T)
    if not cfg.v_delayed:
        vd_prev = _split_proj(cfg, proj)[3]
    premix = np.zeros((B, nq * d))
    qs, ks, vs = [], [], []
    for b in range(B):
        t = int(clen[b])
        hist = conv_state[b].T                                   # [2, C]
        q, k, u = _qk(cfg, W, q_pre[b:b + 1], k_pre[b:b + 1], hist, np.array([t]))
        v = _values(cfg, vc[b:b + 1], vd_prev[b:b + 1])
        k = round_bf16(k)
        v = round_bf16(v)
        # the token's keys / values go into the cache first, in its format,
        # and the attention reads every position from the cache
        kc[b, :, t] = cache_kv(cfg, k[0])
        vcache[b, :, t] = cache_kv(cfg, v[0])
        window = block_window(cfg, bidx)
        lo = max(0, t - window + 1)
        kpos = np.arange(lo, t + 1)
        o = attention(q, kc[b, :, lo:t + 1].transpose(1, 0, 2), vcache[b, :, lo:t + 1].transpose(1, 0, 2),
                      np.array([t]), kpos, np.ones(len(kpos), dtype=bool), window, cfg.scale)
        premix[b] = o.reshape(nq * d)
        conv_state[b] = np.stack([hist[1], u[0]], axis=1)
        qs.append(q[0]); ks.append(k[0]); vs.append(v[0])
    prev_hs = a_in.copy()
    clen = clen + 1
    attn_o = premix @ as64(W["w_o"]).T
    attn_out, h = merge(attn_o, x, as64(W["merge_a"]))
    mt = _mlp_half(cfg, W, h, rin, bidx, np.ones(B, dtype=bool), force_cls)
    out = dict(attention_norm_output=a_in, attention_queries=np.stack(qs), attention_keys=np.stack(ks),
               attention_values=np.stack(vs), attention_premix=premix, attention_output=attn_out,
               layer_mid=h, layer_input=x)
    out.update(mt)
    out["state"] = dict(k_cache=kc, v_cache=vcache, conv_state=conv_state, prev_hs=prev_hs, cache_len=clen)
    return out


# ---------------------------------------------------------------------------
# the stack: embedding -> blocks (router state chained) -> final norm -> head
# ---------------------------------------------------------------------------


def embed(cfg, emb, ids):
    """token_embeddings = E[id] (bf16); the stream entering block 0 is
    fp32((E[id] + shift) * multiplier) (zaya page, "The stream is float32
    whatever the load"; family docstring, last sentence)."""
    te = as64(emb[np.asarray(ids).reshape(-1)]).reshape(*np.asarray(ids).shape, -1)
    return te, round_f32((te + cfg.emb_shift) * cfg.emb_mult)


def lm_head(cfg, emb, final_norm_w, stream):
    """logits = lm_head(norm(stream)) with the tied embedding, no cap or
    scale (zaya page, "The readout and the tokenizer"); bf16."""
    fn = block_norm(stream, as64(final_norm_w), cfg.rms_eps)
    return fn, round_bf16(fn @ as64(emb).T)


def stack_prefill(cfg, blocks, extra, ids, attn_mask=None, logits_rows=None):
    """Full stack over fresh sequences.  blocks: list of weight dicts;
    extra: embed + final_norm_w.  logits_rows: None = every position, else a
    list of positions whose logits are computed."""
    te, x = embed(cfg, extra["embed"], ids)
    r = None
    states = []
    for i, W in enumerate(blocks):
        o = block_prefill(cfg, W, x, attn_mask, r, block_idx=i)
        x, r = o["layer_output"], o["router_state"]
        states.append(o["state"])
    rows = slice(None) if logits_rows is None else logits_rows
    fn, logits = lm_head(cfg, extra["embed"], extra["final_norm_w"], x[:, rows])
    return dict(token_embeddings=te, final_stream=x, final_norm_output=fn, logits=logits, states=states)


def stack_decode(cfg, blocks, extra, ids, states):
    """One decode step through the stack: ids [B]; states: per-block state
    dicts.  Returns logits [B,V] and the updated states."""
    te, x = embed(cfg, extra["embed"], ids)
    r = None
    new_states = []
    for i, W in enumerate(blocks):
        o = block_decode(cfg, W, x, states[i], r, block_idx=i)
        x, r = o["layer_output"], o["router_state"]
        new_states.append(o["state"])
    fn, logits = lm_head(cfg, extra["embed"], extra["final_norm_w"], x)
    return dict(token_embeddings=te, final_stream=x, final_norm_output=fn, logits=logits, states=new_states)
