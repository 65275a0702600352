"""Test harness: runs the CUDA path through the C ABI and compares it with
the CPU oracle on the same seeded inputs.

Comparison protocol (the block's tolerances):
  * router choices, teacher-forced: the oracle's router (down_proj, router
    MLP, fp32 scoring) is run on the GPU's own mlp_norm_output and incoming
    router state; its class must equal the GPU's for every token except
    near-ties (top-two selection scores within 1e-5 relative), which are
    counted and reported;
  * floating point, per block: the oracle block is run on the GPU's block
    input (and state), with the GPU's expert choices forced where the
    oracle's own choice flips from upstream rounding (flips counted);
    layer_output must satisfy max|err| / rms(oracle) <= 2e-2 and
    cosine >= 0.9995.
"""
from __future__ import annotations

import numpy as np
import torch

import top_moe_block_b200 as ZB
from oracle import zaya_oracle as Z

TOL_REL_MAX = 2e-2
TOL_COS = 0.9995
NEAR_TIE = 1e-5


# Weight fields the C ABI reads in bf16 (the rest are fp32).
BF16_FIELDS = ("ln1_w", "ln2_w", "w_qkv", "w_o", "router_down_w", "w_gate_up", "w_down")


def dev_weights(W: dict, dev="cuda") -> dict:
    """The block's weights on the device in the C ABI's dtypes: unrounded
    fp32 matrices (the tiny workload) become bf16-rounded copies."""
    return {k: v.to(dev, _abi_dtype(k, v)).contiguous() for k, v in W.items()}


def _abi_dtype(name, t):
    """The dtype the C ABI reads a weight in: bf16 for the block's matrices
    and norm weights, fp32 for its small parameters; other tensors (the
    stack's bf16 embedding and final norm) keep theirs."""
    if t.dtype == torch.uint8:   # E4M3 codes (FP8 experts) stay bytes
        return torch.uint8
    if name in BF16_FIELDS:
        return torch.bfloat16
    if name in ZB._abi.WEIGHT_FIELDS:
        return torch.float32
    return t.dtype


def eff(W: dict) -> dict:
    """The weights as the GPU reads them (host copies): the matrices the C
    ABI takes in bf16 rounded to bf16.  Unchanged for a bf16 checkpoint; for
    the tiny workload's unrounded fp32 weights this is what the kernels see."""
    return {k: v.detach().cpu().to(_abi_dtype(k, v)) for k, v in W.items()}


def _fp32_matrices(W: dict) -> bool:
    return any(W[k].dtype == torch.float32 and not torch.equal(W[k], W[k].to(torch.bfloat16).float())
               for k in BF16_FIELDS if k in W and W[k].dtype != torch.uint8)


def new_state(cfg, B, cap, dev="cuda") -> dict:
    kv = torch.uint8 if getattr(cfg, "kv_fp8", 0) else torch.bfloat16   # E4M3 bytes with kv_fp8
    return dict(
        k_cache=torch.zeros(B, cfg.n_kv, cap, cfg.head_dim, dtype=kv, device=dev),
        v_cache=torch.zeros(B, cfg.n_kv, cap, cfg.head_dim, dtype=kv, device=dev),
        cache_len=torch.zeros(B, dtype=torch.int32, device=dev),
        conv_state=torch.zeros(B, cfg.qk_channels, 2, dtype=torch.bfloat16, device=dev),
        prev_hs=torch.zeros(B, cfg.hidden, dtype=torch.bfloat16, device=dev))


def new_taps(cfg, B, S, dev="cuda") -> dict:
    M, H, E1 = B * S, cfg.hidden, cfg.n_experts + 1
    bf, f32 = torch.bfloat16, torch.float32
    return dict(
        router_logits=torch.full((M, E1), float("nan"), dtype=f32, device=dev),
        expert_indices=torch.full((M,), -1, dtype=torch.int32, device=dev),
        expert_weights=torch.full((M,), float("nan"), dtype=f32, device=dev),
        attention_norm_output=torch.empty(M, H, dtype=bf, device=dev),
        attention_output=torch.empty(M, H, dtype=bf, device=dev),
        layer_mid=torch.empty(M, H, dtype=f32, device=dev),
        mlp_norm_output=torch.empty(M, H, dtype=bf, device=dev),
        mlp_output=torch.empty(M, H, dtype=bf, device=dev),
        attention_queries=torch.empty(B, cfg.n_q, S, cfg.head_dim, dtype=bf, device=dev))


def workspace(nbytes, dev="cuda", poison=True) -> torch.Tensor:
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if poison:
        ws.fill_(0xFF)           # NaN bit patterns: a read before write shows up as a mismatch
    ws[:256].zero_()             # status word
    return ws


def gpu_prefill(cfg, Wd, x, mask=None, rin=None, block_idx=None, cap=None, taps=True, state=None):
    """One block prefill on the GPU; returns outputs and taps as CPU tensors."""
    bidx = cfg.block_idx if block_idx is None else block_idx
    B, S, H, R = x.shape[0], x.shape[1], cfg.hidden, cfg.router_hidden
    cap = cap or S
    hidden = x.to("cuda", torch.float32).contiguous().clone()
    m = None if mask is None else mask.to("cuda", torch.int32).contiguous()
    r_in = None if (rin is None or bidx == 0) else rin.to("cuda", torch.float32).contiguous()
    r_out = torch.full((B, S, R), float("nan"), dtype=torch.float32, device="cuda")
    st = state if state is not None else new_state(cfg, B, cap)
    tp = new_taps(cfg, B, S) if taps else None
    c = ZB.make_config(cfg)
    ws = workspace(ZB.zaya_workspace_size(c, ZB.ZAYA_PREFILL, B, S))
    ZB.zaya_block_prefill(c, ZB.make_weights(Wd), bidx, B, S, hidden, m, r_in, r_out, ZB.make_state(st),
                          ZB.make_taps(tp), ws)
    status = ZB.zaya_device_status(ws)
    assert status == 0, f"device status {status}: {ZB.zaya_status_string(status)}"
    out = dict(layer_output=hidden.cpu(), router_state=r_out.cpu(), state={k: v.cpu() for k, v in st.items()})
    if tp:
        out.update({k: v.cpu() for k, v in tp.items()})
    return out


def gpu_decode(cfg, Wd, x, state, rin=None, block_idx=None, taps=True):
    """One decode step of one block on the GPU; `state` (device tensors) is updated in place."""
    bidx = cfg.block_idx if block_idx is None else block_idx
    B, H, R = x.shape[0], cfg.hidden, cfg.router_hidden
    hidden = x.to("cuda", torch.float32).contiguous().clone()
    r_in = None if (rin is None or bidx == 0) else rin.to("cuda", torch.float32).contiguous()
    r_out = torch.full((B, R), float("nan"), dtype=torch.float32, device="cuda")
    tp = new_taps(cfg, B, 1) if taps else None
    c = ZB.make_config(cfg)
    ws = workspace(ZB.zaya_workspace_size(c, ZB.ZAYA_DECODE, B, 1))
    ZB.zaya_block_decode(c, ZB.make_weights(Wd), bidx, B, hidden, r_in, r_out, ZB.make_state(state),
                         ZB.make_taps(tp), ws)
    status = ZB.zaya_device_status(ws)
    assert status == 0, f"device status {status}: {ZB.zaya_status_string(status)}"
    out = dict(layer_output=hidden.cpu(), router_state=r_out.cpu())
    if tp:
        out.update({k: v.cpu() for k, v in tp.items()})
    return out


def gpu_classes(cfg, gpu) -> np.ndarray:
    """Class per token from the GPU taps: expert index, or E (skip) where the weight is 0."""
    idx = gpu["expert_indices"].numpy().astype(np.int64)
    w = gpu["expert_weights"].numpy()
    return np.where(w > 0, idx, cfg.n_experts)


def router_teacher_forced(cfg, W, m_in, rin, block_idx, real=None):
    """The oracle's router on the GPU's mlp_norm_output: returns (cls, gap, r, logits)."""
    m = Z.as64(m_in)
    r = m @ Z.as64(W["router_down_w"]).T + Z.as64(W["router_down_b"])
    if block_idx > 0 and rin is not None:
        r = r + Z.as64(rin) * Z.as64(W["router_state_scale"])
    r = Z.round_f32(r)
    logits = Z.router_mlp(r, W, cfg.rms_eps)
    cls, idx, w, p, gap = Z.select(logits, Z.as64(W["balancing"]), cfg.n_experts)
    if real is not None:
        cls = np.where(real, cls, cfg.n_experts)
    return cls, gap, r, logits


def rel_max(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    rms = np.sqrt(np.mean(b * b))
    return float(np.max(np.abs(a - b)) / max(rms, 1e-30))


def cosine(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))


def report(name, gpu, ref) -> dict:
    return {"name": name, "rel_max": rel_max(gpu, ref), "cos": cosine(gpu, ref)}


def check_prefill_block(cfg, W, inp, gpu, block_idx=None, verbose=True):
    """Full comparison of one GPU prefill block against the oracle, on the
    weights as the GPU reads them.  When the workload's weights are
    unrounded fp32 (the tiny workload), layer_output is also compared with
    the oracle run on those fp32 weights (same expert choices), with the
    block tolerances."""
    W_given = W
    W = eff(W)
    bidx = cfg.block_idx if block_idx is None else block_idx
    B, S = inp["x"].shape[:2]
    M = B * S
    E = cfg.n_experts
    real = np.ones(M, dtype=bool) if inp.get("attn_mask") is None else inp["attn_mask"].numpy().reshape(-1) != 0
    rin = inp.get("router_state_in")
    rin2 = None if rin is None else rin.reshape(M, -1)
    g_cls = gpu_classes(cfg, gpu)
    t_cls, gap, t_r, t_logits = router_teacher_forced(cfg, W, gpu["mlp_norm_output"], rin2, bidx, real)
    near = gap < NEAR_TIE
    mism = (t_cls != g_cls) & ~near
    res = {"tokens": M, "near_ties": int((near & real).sum()), "router_mismatch": int(mism.sum())}
    res["router_state"] = report("router_state", gpu["router_state"].reshape(M, -1).numpy(), t_r)
    res["router_logits"] = report("router_logits", gpu["router_logits"].numpy(), t_logits)
    o = Z.block_prefill(cfg, W, inp["x"], inp.get("attn_mask"), rin, bidx, force_cls=g_cls.reshape(B, S))
    res["flips"] = int((o["router_own_cls"].reshape(-1) != g_cls)[real].sum())
    for key in ("layer_output", "attention_output", "mlp_output", "layer_mid", "attention_norm_output",
                "mlp_norm_output"):
        gv = gpu[key].float().numpy().reshape(M, -1)
        ov = o[key].reshape(M, -1)
        res[key] = report(key, gv, ov)
        res[key]["bf16_ok"] = close_bf16(gv, ov)
    res["attention_queries"] = report("q", gpu["attention_queries"].float().numpy(), o["attention_queries"])
    st = gpu["state"]
    res["attention_queries"]["bf16_ok"] = close_bf16(gpu["attention_queries"].float().numpy(), o["attention_queries"])
    res["k_cache"] = report("k", st["k_cache"][:, :, :S].float().numpy(), o["state"]["k_cache"])
    res["k_cache"]["bf16_ok"] = close_bf16(st["k_cache"][:, :, :S].float().numpy(), o["state"]["k_cache"])
    res["v_cache"] = report("v", st["v_cache"][:, :, :S].float().numpy(), o["state"]["v_cache"])
    res["v_cache"]["bf16_ok"] = close_bf16(st["v_cache"][:, :, :S].float().numpy(), o["state"]["v_cache"])
    res["conv_state"] = report("conv", st["conv_state"].float().numpy(), o["state"]["conv_state"])
    res["prev_hs"] = report("prev_hs", st["prev_hs"].float().numpy(), o["state"]["prev_hs"])
    res["cache_len_ok"] = bool((st["cache_len"].numpy() == S).all())
    if _fp32_matrices(W_given):
        o32 = Z.block_prefill(cfg, W_given, inp["x"], inp.get("attn_mask"), rin, bidx, force_cls=g_cls.reshape(B, S))
        res["fp32_weights"] = report("layer_output", gpu["layer_output"].float().numpy().reshape(M, -1),
                                     o32["layer_output"].reshape(M, -1))
    if verbose:
        print({k: (round(v["rel_max"], 5), round(v["cos"], 6)) if isinstance(v, dict) else v for k, v in res.items()})
    return res


def close_bf16(gpu, ref) -> bool:
    """For a tensor the block stores in bf16: every element within the block
    tolerance (2e-2 of the reference rms) plus one bf16 unit in the last place
    of the element (rounding of the two sides may land on neighbouring bf16
    values), and cosine >= 0.9995."""
    g = np.asarray(gpu, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(o * o))
    ok = np.abs(g - o) <= TOL_REL_MAX * rms + 2.0 ** -7 * np.abs(o)
    return bool(ok.all()) and cosine(g, o) >= TOL_COS


def assert_block_ok(res):
    assert res["router_mismatch"] == 0, res
    lo = res["layer_output"]
    assert lo["rel_max"] <= TOL_REL_MAX and lo["cos"] >= TOL_COS, lo
    if "fp32_weights" in res:
        lo = res["fp32_weights"]
        assert lo["rel_max"] <= TOL_REL_MAX and lo["cos"] >= TOL_COS, ("against the fp32-weight oracle", lo)


def check_prefill_rows(cfg, W, x_seq, rin_seq, gpu, ranges, block_idx, b=0):
    """Sampled-row comparison of one GPU prefill block of a long unpadded
    sequence (sequence b of the batch): for each row range, the oracle's
    windowed evaluation of those rows (teacher-forced with the GPU's expert
    choices) against the GPU's layer_output, and the oracle's router on the
    GPU's mlp_norm_output against the GPU's choices.  Returns a list of
    per-range results (near-ties counted, not failed)."""
    S = x_seq.shape[0]
    W = eff(W)
    g_cls = gpu_classes(cfg, gpu).reshape(-1, S)[b]
    m_in = gpu["mlp_norm_output"].reshape(-1, S, cfg.hidden)[b]
    out = []
    for r0, r1 in ranges:
        ref = Z.block_prefill_rows(cfg, W, x_seq, r0, r1, rin_seq, block_idx=block_idx, force_cls=g_cls[r0:r1])
        rin_rows = None if rin_seq is None else rin_seq[r0:r1]
        t_cls, gap, _, _ = router_teacher_forced(cfg, W, m_in[r0:r1], rin_rows, block_idx)
        near = gap < NEAR_TIE
        res = {"rows": (r0, r1), "near_ties": int(near.sum()),
               "router_mismatch": int(((t_cls != g_cls[r0:r1]) & ~near).sum())}
        lo = gpu["layer_output"].reshape(-1, S, cfg.hidden)[b, r0:r1].numpy()
        res["layer_output"] = report("layer_output", lo, ref["layer_output"])
        out.append(res)
    return out


def assert_rows_ok(results):
    for res in results:
        assert res["router_mismatch"] == 0, res
        lo = res["layer_output"]
        assert lo["rel_max"] <= TOL_REL_MAX and lo["cos"] >= TOL_COS, res


def _e4m3_lut() -> torch.Tensor:
    """The value of every OCP FP8 E4M3 code (sign, 4 exponent bits with bias
    7, 3 mantissa bits; exponent 0 subnormal; S.1111.111 NaN)."""
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            v = float("nan")
        else:
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(-v if s else v)
    return torch.tensor(vals, dtype=torch.float64)


def e4m3_values(t: torch.Tensor) -> torch.Tensor:
    """E4M3 bytes (uint8) as their float64 values."""
    return _e4m3_lut()[t.cpu().long()]
