"""ZAYA1 decoder-block forward on B200 (sm_100a): Python binding of the C ABI.

The functions below carry the C entry points' names (include/zaya.h) and do
argument marshalling only: torch tensors in, device pointers out.  PyTorch
supplies device memory and streams; every step of the block runs in the
library's CUDA kernels, and a missing library raises instead of falling
back to anything else.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _abi
from ._abi import (ZAYA_DECODE, ZAYA_OK, ZAYA_PREFILL, zaya_block_state,  # noqa: F401
                   zaya_block_weights, zaya_config, zaya_taps)

__all__ = ["make_config", "make_weights", "make_state", "make_taps", "zaya_workspace_size",
           "zaya_stack_workspace_size", "zaya_block_prefill", "zaya_block_decode", "zaya_block_decode_noalloc",
           "zaya_stack_forward",
           "zaya_device_status", "zaya_noalloc_status", "set_wait_limit_ns", "zaya_status_string", "zaya_abi_version", "zaya_profile_enable",
           "zaya_profile_reset", "zaya_profile_read", "zaya_launch_count", "ZayaError", "ZAYA_PREFILL",
           "ZAYA_DECODE"]


class ZayaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {zaya_status_string(code)} (code {code})")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_config(cfg) -> zaya_config:
    """zaya_config from any object with the same attribute names."""
    c = zaya_config()
    for name, _ in zaya_config._fields_:
        if hasattr(cfg, name):
            setattr(c, name, getattr(cfg, name))
    c.conv_width = getattr(cfg, "conv_width", 3)
    return c


def make_weights(w: dict) -> zaya_block_weights:
    s = zaya_block_weights()
    for n in _abi.WEIGHT_FIELDS:
        setattr(s, n, _ptr(w.get(n)))
    return s


def make_state(st: dict) -> zaya_block_state:
    s = zaya_block_state()
    s.k_cache = _ptr(st["k_cache"])
    s.v_cache = _ptr(st["v_cache"])
    s.cache_cap = int(st["k_cache"].shape[2])
    s.cache_len = _ptr(st["cache_len"])
    s.conv_state = _ptr(st["conv_state"])
    s.prev_hs = _ptr(st["prev_hs"])
    return s


def make_taps(t: dict | None) -> zaya_taps | None:
    if not t:
        return None
    s = zaya_taps()
    for n in _abi.TAP_FIELDS:
        setattr(s, n, _ptr(t.get(n)))
    return s


def _ref(x):
    return C.byref(x) if x is not None else None


def zaya_status_string(code: int) -> str:
    return _abi.lib().zaya_status_string(code).decode()


def zaya_abi_version() -> int:
    return _abi.lib().zaya_abi_version()


def zaya_workspace_size(cfg: zaya_config, mode: int, B: int, S: int) -> int:
    return _abi.lib().zaya_workspace_size(C.byref(cfg), mode, B, S)


def zaya_stack_workspace_size(cfg: zaya_config, mode: int, B: int, S: int) -> int:
    return _abi.lib().zaya_stack_workspace_size(C.byref(cfg), mode, B, S)


def _check(rc: int, where: str, check: bool) -> int:
    if check and rc != ZAYA_OK:
        raise ZayaError(rc, where)
    return rc


def zaya_block_prefill(cfg, weights, block_idx, B, S, hidden, attn_mask, router_state_in, router_state_out,
                       state, taps, workspace, workspace_bytes=None, stream=None, check=True) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    rc = _abi.lib().zaya_block_prefill(
        C.byref(cfg), C.byref(weights), block_idx, B, S, _ptr(hidden), _ptr(attn_mask), _ptr(router_state_in),
        _ptr(router_state_out), C.byref(state), _ref(taps), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    return _check(rc, "zaya_block_prefill", check)


def zaya_block_decode(cfg, weights, block_idx, B, hidden, router_state_in, router_state_out, state, taps,
                      workspace, workspace_bytes=None, stream=None, check=True) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    rc = _abi.lib().zaya_block_decode(
        C.byref(cfg), C.byref(weights), block_idx, B, _ptr(hidden), _ptr(router_state_in), _ptr(router_state_out),
        C.byref(state), _ref(taps), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    return _check(rc, "zaya_block_decode", check)


def zaya_block_decode_noalloc(cfg, weights, block_idx, B, hidden, router_state_in, router_state_out, state,
                              taps=None, stream=None, check=True) -> int:
    """zaya_block_decode with the library's own fixed scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    rc = _abi.lib().zaya_block_decode_noalloc(
        C.byref(cfg), C.byref(weights), block_idx, B, _ptr(hidden), _ptr(router_state_in), _ptr(router_state_out),
        C.byref(state), _ref(taps), _stream_ptr(stream))
    return _check(rc, "zaya_block_decode_noalloc", check)


def zaya_stack_forward(cfg, blocks, embed, final_norm_w, mode, B, S, ids, attn_mask, states, logits,
                       logits_last_only, workspace, workspace_bytes=None, stream=None, check=True) -> int:
    """blocks / states: sequences of zaya_block_weights / zaya_block_state."""
    n = len(blocks)
    barr = (zaya_block_weights * n)(*blocks)
    sarr = (zaya_block_state * n)(*states)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    rc = _abi.lib().zaya_stack_forward(
        C.byref(cfg), n, barr, _ptr(embed), _ptr(final_norm_w), mode, B, S, _ptr(ids), _ptr(attn_mask), sarr,
        _ptr(logits), int(logits_last_only), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    return _check(rc, "zaya_stack_forward", check)


def zaya_device_status(workspace, stream=None) -> int:
    return _abi.lib().zaya_device_status(_ptr(workspace), _stream_ptr(stream))


def zaya_noalloc_status(stream=None) -> int:
    """Status word of zaya_block_decode_noalloc's fixed scratch (read and cleared)."""
    return _abi.lib().zaya_noalloc_status(_stream_ptr(stream))


def set_wait_limit_ns(workspace, ns: int) -> None:
    """Write the wait limit into the workspace header (bytes 8..16; 0 = the
    default 2 s), stream-ordered on the current stream."""
    workspace[8:16].copy_(torch.tensor([int(ns)], dtype=torch.int64).view(torch.uint8))


def zaya_profile_enable(on: bool = True) -> None:
    _abi.lib().zaya_profile_enable(1 if on else 0)


def zaya_profile_reset() -> None:
    _abi.lib().zaya_profile_reset()


def zaya_profile_read(max_stages: int = 64) -> dict:
    """{stage name: (total milliseconds, stage calls)} since the last reset."""
    names = (C.c_char_p * max_stages)()
    ms = (C.c_double * max_stages)()
    n_l = (C.c_int64 * max_stages)()
    n = _abi.lib().zaya_profile_read(max_stages, names, ms, n_l)
    return {names[i].decode(): (ms[i], n_l[i]) for i in range(min(n, max_stages))}


def zaya_launch_count() -> int:
    return _abi.lib().zaya_launch_count()
