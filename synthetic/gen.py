"""Seeded tensors for the ZAYA1 block workloads.

Every tensor is drawn from its own torch generator whose seed is derived
from (workload seed, block index, tensor name), so any one block's weights
can be drawn without drawing the others.  Values that the C ABI takes in
bf16 are returned as torch.bfloat16; the small per-channel parameters the
ABI takes in fp32 are returned as float32 but hold bf16-representable
values, as a bf16 checkpoint would.

Draws depend on the device they are made on (CPU and CUDA generators are
different streams); every consumer takes the same returned tensors.
"""
from __future__ import annotations

import json
import os
import zlib

import torch

from .configs import BlockConfig

_HERE = os.path.dirname(os.path.abspath(__file__))


def _seed(cfg_seed: int, block: int, tag: str) -> int:
    return zlib.crc32(f"{cfg_seed}/{block}/{tag}".encode()) & 0x7FFFFFFF


def _gen(cfg: BlockConfig, block: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(cfg.seed, block, tag))
    return g


def bf16_values(t: torch.Tensor) -> torch.Tensor:
    """The float32 tensor holding t's values rounded to bf16."""
    return t.to(torch.bfloat16).to(torch.float32)


_bf16_values = bf16_values


def _identity(t: torch.Tensor) -> torch.Tensor:
    return t


def _normal(cfg, block, tag, shape, std, device, mean=0.0):
    g = _gen(cfg, block, tag, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std + mean


def _uniform(cfg, block, tag, shape, lo, hi, device):
    g = _gen(cfg, block, tag, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def balancing_biases(cfg: BlockConfig) -> torch.Tensor:
    """[E+1] fp32 balancing biases of the router's selection (last = skip).

    Calibrated workloads read the values written by
    ``oracle/calibrate_balancing.py`` (a seeded fixed-point fit of the loads
    to Zipf(s) with the requested skip share); the others are 0 on every
    expert and ``skip_bias`` on skip.
    """
    E = cfg.n_experts
    if cfg.calibrated:
        path = os.path.join(_HERE, f"balancing_{cfg.calib or cfg.name}.json")
        with open(path) as f:
            vals = json.load(f)["balancing_biases"]
        assert len(vals) == E + 1
        return torch.tensor(vals, dtype=torch.float32)
    b = torch.zeros(E + 1, dtype=torch.float32)
    b[E] = cfg.skip_bias
    return b


def gen_block_weights(cfg: BlockConfig, block: int | None = None, device="cpu") -> dict:
    """One block's parameters, keyed by the C ABI's field names.  With
    ``weight_dtype == "fp32"`` every tensor is float32 and unrounded (the
    caller rounds the matrices the C ABI takes in bf16); otherwise matrices
    are bf16 and the small parameters hold bf16 values in float32."""
    blk = cfg.block_idx if block is None else block
    H, R, E, I, C = cfg.hidden, cfg.router_hidden, cfg.n_experts, cfg.inter, cfg.qk_channels
    if cfg.weight_dtype == "fp32":
        bf = torch.float32
        bf16_values = _identity
    else:
        bf = torch.bfloat16
        bf16_values = _bf16_values
    n = lambda tag, shape, std, mean=0.0: _normal(cfg, blk, tag, shape, std, device, mean)
    u = lambda tag, shape, lo, hi: _uniform(cfg, blk, tag, shape, lo, hi, device)
    w = {}
    w["ln1_w"] = n("ln1_w", (H,), 0.02, 1.0).to(bf)
    w["ln2_w"] = n("ln2_w", (H,), 0.02, 1.0).to(bf)
    w["w_qkv"] = n("w_qkv", (cfg.n_qkv, H), cfg.w_std).to(bf)
    w["conv_w"] = bf16_values(n("conv_w", (C, cfg.conv_width), 0.5))
    w["conv_b"] = bf16_values(n("conv_b", (C,), 0.02))
    if cfg.conv_groups:   # the grouped conv: [C, C/G, 2] (Conv1d layout), std 1/sqrt(2 C/G)
        cg = C // cfg.conv_groups
        w["conv2_w"] = bf16_values(n("conv2_w", (C, cg, 2), 1.0 / (2 * cg) ** 0.5))
        w["conv2_b"] = bf16_values(n("conv2_b", (C,), 0.02))
    if cfg.temp_mode == "one":
        w["k_temp"] = torch.ones(cfg.n_kv, dtype=torch.float32, device=device)
    elif cfg.temp_mode == "zero":
        w["k_temp"] = torch.zeros(cfg.n_kv, dtype=torch.float32, device=device)
    else:
        w["k_temp"] = bf16_values(u("k_temp", (cfg.n_kv,), 0.8, 12.9))
    w["w_o"] = n("w_o", (H, cfg.q_dim), cfg.w_std).to(bf)
    for m in ("merge_a", "merge_m"):
        hb = n(m + ".hb", (H,), 0.1)
        hs = u(m + ".hs", (H,), 0.5, 1.5)
        rb = n(m + ".rb", (H,), 0.1)
        rs = u(m + ".rs", (H,), 0.5, 1.5)
        w[m] = bf16_values(torch.stack([hb, hs, rb, rs]))      # rows: hb, hs, rb, rs
    w["router_down_w"] = n("router_down_w", (R, H), cfg.w_std).to(bf)
    w["router_down_b"] = bf16_values(n("router_down_b", (R,), cfg.router_b_std))
    w["router_state_scale"] = bf16_values(u("router_state_scale", (R,), 0.25, 0.75))
    w["router_norm_w"] = bf16_values(n("router_norm_w", (R,), 0.02, 1.0))
    w["fc1_w"] = bf16_values(n("fc1_w", (R, R), cfg.router_w_std))
    w["fc1_b"] = bf16_values(n("fc1_b", (R,), cfg.router_b_std))
    w["fc2_w"] = bf16_values(n("fc2_w", (R, R), cfg.router_w_std))
    w["fc2_b"] = bf16_values(n("fc2_b", (R,), cfg.router_b_std))
    w["out_w"] = bf16_values(n("out_w", (E + 1, R), cfg.router_w_std))
    w["balancing"] = balancing_biases(cfg).to(device)
    w["w_gate_up"] = n("w_gate_up", (E, 2 * I, H), cfg.w_std).to(bf)   # rows [0,I) gate, [I,2I) up
    w["w_down"] = n("w_down", (E, H, I), cfg.w_std).to(bf)
    if cfg.expert_fp8:
        # an FP8 checkpoint of the same draws: E4M3 codes (uint8) with one fp32
        # scale per output row (its absolute maximum over 448), and static
        # per-expert input scales (powers of two: inputs of |x| <= 14 fit)
        for name in ("w_gate_up", "w_down"):
            full = w[name].float()
            scale = full.abs().amax(dim=-1).clamp_min(1e-30) / 448.0
            w[name] = (full / scale[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
            w[name + "_scale"] = scale.to(torch.float32)
        w["expert_act_scale"] = torch.full((E, 2), 2.0 ** -5, dtype=torch.float32, device=device)
    return w


def gen_prefill_inputs(cfg: BlockConfig, device="cpu", stream: int = -1) -> dict:
    """Stream input x [B,S,H] fp32 ~ N(0,1), the left-padding mask, and the
    router state carried in from the previous block ([B,S,R] ~ N(0,1)) when
    the workload runs as a block > 0.  ``stream`` selects an independent
    draw of the same distribution (-1: the workload's own inputs)."""
    B, S, H, R = cfg.batch, cfg.seq, cfg.hidden, cfg.router_hidden
    out = {"x": _normal(cfg, stream, "x", (B, S, H), 1.0, device)}
    if cfg.pad_max > 0:
        g = _gen(cfg, stream, "pads", "cpu")
        pads = torch.randint(0, cfg.pad_max + 1, (B,), generator=g)
        mask = torch.ones(B, S, dtype=torch.int32)
        for b in range(B):
            mask[b, : int(pads[b])] = 0
        out["attn_mask"] = mask.to(device)
        out["pads"] = pads
    else:
        out["attn_mask"] = None
    out["router_state_in"] = (_normal(cfg, stream, "router_state_in", (B, S, R), 1.0, device)
                              if cfg.block_idx > 0 else None)
    return out


def gen_decode_state(cfg: BlockConfig, block: int, cap: int, device="cpu") -> dict:
    """A block's decode state with ``cache_prior`` tokens already cached:
    K/V cache [B,n_kv,cap,d] bf16, conv_state [B,C,2] bf16 and prev_hs [B,H]
    bf16, all N(0,1), and cache_len [B] int32 = cache_prior."""
    B, d = cfg.batch, cfg.head_dim
    L = cfg.cache_prior
    k = torch.zeros(B, cfg.n_kv, cap, d, dtype=torch.bfloat16, device=device)
    v = torch.zeros_like(k)
    k[:, :, :L] = _normal(cfg, block, "k_cache", (B, cfg.n_kv, L, d), 1.0, device).to(torch.bfloat16)
    v[:, :, :L] = _normal(cfg, block, "v_cache", (B, cfg.n_kv, L, d), 1.0, device).to(torch.bfloat16)
    if cfg.kv_fp8:   # an fp8 cache holds E4M3 codes (uint8) of the same draws
        k = k.to(torch.float8_e4m3fn).view(torch.uint8)
        v = v.to(torch.float8_e4m3fn).view(torch.uint8)
    return {
        "k_cache": k, "v_cache": v,
        "conv_state": _normal(cfg, block, "conv_state", (B, cfg.qk_channels, 2), 1.0,
                              device).to(torch.bfloat16),
        "prev_hs": _normal(cfg, block, "prev_hs", (B, cfg.hidden), 1.0, device).to(torch.bfloat16),
        "cache_len": torch.full((B,), L, dtype=torch.int32, device=device),
    }


def gen_stack_weights_extra(cfg: BlockConfig, device="cpu") -> dict:
    """Tied embedding / lm_head [V,H] bf16 and the final norm weight."""
    return {
        "embed": _normal(cfg, -2, "embed", (cfg.vocab, cfg.hidden), cfg.w_std, device).to(torch.bfloat16),
        "final_norm_w": _normal(cfg, -2, "final_norm_w", (cfg.hidden,), 0.02, device, 1.0).to(torch.bfloat16),
    }


def gen_token_ids(cfg: BlockConfig, device="cpu") -> torch.Tensor:
    """Token ids [B,S] int32, uniform over the vocabulary."""
    g = _gen(cfg, -1, "ids", "cpu")
    return torch.randint(0, cfg.vocab, (cfg.batch, cfg.seq), generator=g, dtype=torch.int64).to(
        torch.int32).to(device)
