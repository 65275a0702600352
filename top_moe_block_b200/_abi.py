"""ctypes mirror of include/zaya.h: structures, status codes and the entry
points, with the same names.  Argument marshalling only; every step of the
block runs in the CUDA kernels of libzaya.so."""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzaya.so")

ZAYA_OK = 0
ZAYA_ERR_INVALID_ARG = 1
ZAYA_ERR_MISALIGNED = 2
ZAYA_ERR_UNSUPPORTED = 3
ZAYA_ERR_WORKSPACE = 4
ZAYA_ERR_CUDA = 5
ZAYA_ERR_TIMEOUT = 6
ZAYA_ERR_DEVICE_RANGE = 7
ZAYA_PREFILL = 0
ZAYA_DECODE = 1


class zaya_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "hidden", "n_q", "n_kv", "head_dim", "rot_dim", "conv_width", "n_experts", "inter",
        "router_hidden", "window", "vocab", "cca_mean_residual", "v_delayed", "sliding_period",
        "sliding_phase", "conv_groups", "kv_ring", "expert_fp8", "kv_fp8")] + [
        (n, C.c_float) for n in ("rope_theta", "rms_eps", "qk_norm_eps", "attn_scale", "emb_mult", "emb_shift")]


WEIGHT_FIELDS = ("ln1_w", "ln2_w", "w_qkv", "conv_w", "conv_b", "k_temp", "w_o", "merge_a", "merge_m",
                 "router_down_w", "router_down_b", "router_state_scale", "router_norm_w", "fc1_w", "fc1_b",
                 "fc2_w", "fc2_b", "out_w", "balancing", "w_gate_up", "w_down", "conv2_w", "conv2_b",
                 "w_gate_up_scale", "w_down_scale", "expert_act_scale")


class zaya_block_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


class zaya_block_state(C.Structure):
    _fields_ = [("k_cache", C.c_void_p), ("v_cache", C.c_void_p), ("cache_cap", C.c_int32),
                ("cache_len", C.c_void_p), ("conv_state", C.c_void_p), ("prev_hs", C.c_void_p)]


TAP_FIELDS = ("router_logits", "expert_indices", "expert_weights", "attention_norm_output", "attention_output",
              "layer_mid", "mlp_norm_output", "mlp_output", "attention_queries")


class zaya_taps(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in TAP_FIELDS]


_lib = None


def lib() -> C.CDLL:
    """The loaded libzaya.so; raises if the CUDA library has not been built
    (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libzaya.so not built ({LIB_PATH}); run top_moe_block_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        P = C.POINTER
        vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        L.zaya_workspace_size.argtypes = [P(zaya_config), i32, i32, i32]
        L.zaya_workspace_size.restype = sz
        L.zaya_stack_workspace_size.argtypes = [P(zaya_config), i32, i32, i32]
        L.zaya_stack_workspace_size.restype = sz
        L.zaya_block_prefill.argtypes = [P(zaya_config), P(zaya_block_weights), i32, i32, i32, vp, vp, vp, vp,
                                         P(zaya_block_state), P(zaya_taps), vp, sz, vp]
        L.zaya_block_prefill.restype = C.c_int
        L.zaya_block_decode.argtypes = [P(zaya_config), P(zaya_block_weights), i32, i32, vp, vp, vp,
                                        P(zaya_block_state), P(zaya_taps), vp, sz, vp]
        L.zaya_block_decode.restype = C.c_int
        L.zaya_block_decode_noalloc.argtypes = [P(zaya_config), P(zaya_block_weights), i32, i32, vp, vp, vp,
                                                P(zaya_block_state), P(zaya_taps), vp]
        L.zaya_block_decode_noalloc.restype = C.c_int
        L.zaya_stack_forward.argtypes = [P(zaya_config), i32, P(zaya_block_weights), vp, vp, i32, i32, i32, vp, vp,
                                         P(zaya_block_state), vp, i32, vp, sz, vp]
        L.zaya_stack_forward.restype = C.c_int
        L.zaya_device_status.argtypes = [vp, vp]
        L.zaya_device_status.restype = C.c_int
        L.zaya_noalloc_status.argtypes = [vp]
        L.zaya_noalloc_status.restype = C.c_int
        L.zaya_status_string.argtypes = [C.c_int]
        L.zaya_status_string.restype = C.c_char_p
        L.zaya_profile_enable.argtypes = [C.c_int]
        L.zaya_profile_enable.restype = None
        L.zaya_profile_reset.argtypes = []
        L.zaya_profile_reset.restype = None
        L.zaya_profile_read.argtypes = [i32, P(C.c_char_p), P(C.c_double), P(C.c_int64)]
        L.zaya_profile_read.restype = C.c_int
        L.zaya_launch_count.argtypes = []
        L.zaya_launch_count.restype = C.c_int64
        L.zaya_abi_version.argtypes = []
        L.zaya_abi_version.restype = C.c_int
        _lib = L
    return _lib
