"""The five ZAYA1 block workloads, named by what they are.

Shapes follow the ZAYA1-8B printout and config (nnterp encyclopedia, "zaya"
family page, "Printout" and "Config"): hidden 2048, 8 query heads and 2
key/value heads of dim 128, 16 experts of width 2048, a 17-class router
(16 experts + skip) over a 256-wide router hidden state, 1280 convolved
query+key channels.  Every detail the pages leave open is a field here, set
once, with the reading it encodes stated beside it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class BlockConfig:
    name: str
    # ---- block shape (zaya page, "Config" and "Printout") ----
    hidden: int
    n_q: int
    n_kv: int
    head_dim: int
    rot_dim: int                 # partial_rotary_factor 0.5 -> head_dim / 2
    n_experts: int
    inter: int                   # moe_intermediate_size
    router_hidden: int           # router down_proj width (256 on ZAYA1-8B)
    window: int                  # key j visible to query i iff 0 <= i-j < window
    rope_theta: float
    conv_width: int = 3          # taps (t-2, t-1, t) over the q||k channels
    conv_groups: int = 0         # 0: that one depthwise conv; G: the printout's two convs of width 2
                                 # (depthwise, then grouped with G groups; conv_width = 2)
    rms_eps: float = 1e-5
    qk_norm_eps: float = 1e-6    # x * sqrt(d) / max(|x|, eps)
    attn_scale: float = 0.0      # 0 -> 1/sqrt(head_dim)
    cca_mean_residual: int = 1   # add the CCA mean residual after the conv
    v_delayed: int = 1           # half of each value head from token t-1
    sliding_period: int = 0      # 0: every block slides over `window` keys; P > 0: only blocks with
    sliding_phase: int = 0       # block % P == phase slide, the others attend to every earlier token
    kv_ring: int = 0             # 1: K/V caches as window rings (slot = position % cache_cap)
    kv_fp8: int = 0              # 1: K/V caches hold OCP FP8 E4M3 (the prompt attends over bf16)
    expert_fp8: int = 0          # 1: expert weights as E4M3 codes + per-row scales, E4M3 activations
    calib: str = ""              # calibrated: the workload whose fitted balancing biases apply (default: own)
    vocab: int = 0
    emb_mult: float = 1.0
    emb_shift: float = 0.0
    # ---- workload ----
    batch: int = 1
    seq: int = 1
    n_blocks: int = 1
    block_idx: int = 1           # single-block workloads run as a block > 0 (router state carried in)
    mode: str = "prefill"        # "prefill" | "decode"
    cache_prior: int = 0         # decode: tokens already in each sequence's cache
    pad_max: int = 0             # left padding drawn U{0..pad_max} per sequence
    calibrated: int = 0          # 1: balancing biases fitted to target loads (file beside this one)
    zipf_s: float = 0.0          # target expert loads ~ Zipf(s) (0 -> uniform)
    skip_frac: float = 0.0       # target skip share for the calibrated biases
    seed: int = 0
    # ---- value distributions (open on the pages; written down here) ----
    w_std: float = 0.02          # every projection / expert / embedding weight N(0, w_std)
    router_w_std: float = 0.02   # router MLP (fc1, fc2, out_proj) weights
    router_b_std: float = 0.02   # router Linear biases (down_proj, fc1, fc2)
    skip_bias: float = 0.0       # balancing bias of the skip class when not calibrated
    temp_mode: str = "one"       # "one" -> temp = 1; "stress" -> U(0.8, 12.9) per kv head
    input_dtype: str = "fp32"    # "fp32": tiny workload (GPU takes bf16-rounded copies)
    weight_dtype: str = "bf16"   # "bf16": drawn values rounded to bf16 (a bf16 checkpoint);
                                 # "fp32": unrounded fp32 weights (the tiny workload); the GPU
                                 # takes bf16-rounded copies of the matrices it reads in bf16

    # ---- derived sizes ----
    @property
    def q_dim(self) -> int:
        return self.n_q * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv * self.head_dim

    @property
    def v_half(self) -> int:
        """Width of v_proj_current and of v_proj_delayed (n_kv * d / 2)."""
        return self.n_kv * self.head_dim // 2

    @property
    def qk_channels(self) -> int:
        """Channels the causal conv runs over: q || k (1280 on ZAYA1-8B)."""
        return self.q_dim + self.kv_dim

    @property
    def n_qkv(self) -> int:
        """Rows of the stacked projection weight: q, k, v_current, v_delayed."""
        return self.q_dim + self.kv_dim + 2 * self.v_half

    @property
    def scale(self) -> float:
        return self.attn_scale if self.attn_scale > 0 else 1.0 / math.sqrt(self.head_dim)

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    def with_(self, **kw) -> "BlockConfig":
        return replace(self, **kw)


_FULL = dict(hidden=2048, n_q=8, n_kv=2, head_dim=128, rot_dim=64, n_experts=16,
             inter=2048, router_hidden=256, window=4096, rope_theta=5e6,
             router_w_std=1.0 / 16.0, router_b_std=0.5)

CONFIGS = {
    # Tiny single block, fp32 inputs and weights (unrounded), seed 0.
    "tiny": BlockConfig(
        name="tiny", hidden=256, n_q=4, n_kv=1, head_dim=64, rot_dim=32, n_experts=4,
        inter=256, router_hidden=32, window=32, rope_theta=1e4, batch=1, seq=64,
        seed=0, vocab=512, emb_mult=math.sqrt(256.0),
        # N(0, 0.02) router-MLP weights make the 5 logits equal to ~1e-3 and send
        # every token to one class; 1/sqrt(R) keeps the choice token-dependent.
        router_w_std=1.0 / math.sqrt(32.0), calibrated=1, skip_frac=0.25, weight_dtype="fp32"),
    # Full-width single block prefill, B1 x S4096; balancing biases fitted to
    # roughly uniform expert loads with no skip (the random-init router alone
    # sends half the tokens to one expert).
    "prefill_4k": BlockConfig(
        name="prefill_4k", batch=1, seq=4096, seed=1, calibrated=1, skip_frac=0.0,
        input_dtype="bf16", **_FULL),
    # Batched prefill, B8 x S2048, left pads U{0..256}, Zipf(1.1) loads, ~20% skip.
    "prefill_skewed_8x2k": BlockConfig(
        name="prefill_skewed_8x2k", batch=8, seq=2048, seed=2, pad_max=256,
        calibrated=1, zipf_s=1.1, skip_frac=0.2, input_dtype="bf16", **_FULL),
    # Decode step through 40 blocks, B64, 8192 cached tokens per sequence.
    "decode_stack_b64": BlockConfig(
        name="decode_stack_b64", batch=64, seq=1, n_blocks=40, block_idx=0, mode="decode",
        cache_prior=8192, seed=3, skip_bias=-1.0, input_dtype="bf16",
        vocab=262144, emb_mult=math.sqrt(2048.0), **_FULL),
    # The prefill block and the decode step with the experts as an FP8 W8A8
    # checkpoint (E4M3 codes, per-row scales, static input scales).
    "prefill_4k_fp8x": BlockConfig(
        name="prefill_4k_fp8x", batch=1, seq=4096, seed=1, calibrated=1, skip_frac=0.0,
        input_dtype="bf16", expert_fp8=1, calib="prefill_4k", **_FULL),
    "decode_stack_b64_fp8x": BlockConfig(
        name="decode_stack_b64_fp8x", batch=64, seq=1, n_blocks=40, block_idx=0, mode="decode",
        cache_prior=8192, seed=3, skip_bias=-1.0, input_dtype="bf16", expert_fp8=1,
        vocab=262144, emb_mult=math.sqrt(2048.0), **_FULL),
    # The decode step with an fp8 (E4M3) KV cache, as the NVFP4 README serves
    # the model (--kv-cache-dtype fp8).
    "decode_stack_b64_fp8kv": BlockConfig(
        name="decode_stack_b64_fp8kv", batch=64, seq=1, n_blocks=40, block_idx=0, mode="decode",
        cache_prior=8192, seed=3, skip_bias=-1.0, input_dtype="bf16", kv_fp8=1,
        vocab=262144, emb_mult=math.sqrt(2048.0), **_FULL),
    # The same stack with the 74B preview's hybrid attention: a 4097-token
    # window on every other block (the odd ones), every earlier token on the others.
    "prefill_stack_hybrid_32k": BlockConfig(
        name="prefill_stack_hybrid_32k", batch=1, seq=32768, n_blocks=40, block_idx=0, seed=5,
        skip_bias=-1.0, input_dtype="bf16", vocab=262144, emb_mult=math.sqrt(2048.0),
        sliding_period=2, sliding_phase=1, **dict(_FULL, window=4097)),
    # The full-width block with the printout's two-stage conv_qk (depthwise
    # k=2, then grouped k=2 with 10 groups), B1 x S4096.
    "prefill_4k_conv2": BlockConfig(
        name="prefill_4k_conv2", batch=1, seq=4096, seed=6, calibrated=1, skip_frac=0.0,
        input_dtype="bf16", conv_width=2, conv_groups=10, **_FULL),
    # Long prefill through the 40-block stack with embedding and tied lm_head.
    "prefill_stack_32k": BlockConfig(
        name="prefill_stack_32k", batch=1, seq=32768, n_blocks=40, block_idx=0, seed=4,
        skip_bias=-1.0, input_dtype="bf16", vocab=262144, emb_mult=math.sqrt(2048.0), **_FULL),
}


def get_config(name: str, **overrides) -> BlockConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg
