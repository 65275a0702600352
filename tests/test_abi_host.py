"""Host-side checks of the C ABI (no GPU): the library loads and exports
every entry point include/zaya.h declares, the ctypes structures have the
C layout, and argument errors come back as the documented status codes
before anything touches a device."""
import ctypes as C
import os
import re
import subprocess

import pytest

import top_moe_block_b200 as ZB
from top_moe_block_b200 import _abi, build
from synthetic import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zaya.h")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    return _abi.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|void|int64_t|size_t|char)\s*\*?\s*(zaya_\w+)\s*\(",
                                 src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"zaya_block_prefill", "zaya_block_decode", "zaya_stack_forward", "zaya_workspace_size",
            "zaya_status_string", "zaya_device_status"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (zaya_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing


def test_struct_layout_matches_header(tmp_path):
    """Compile a C program against include/zaya.h that prints sizeof/offsetof
    of every field, and compare with the ctypes mirror."""
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "zaya.h"', 'int main(void){']
    structs = [("zaya_config", _abi.zaya_config), ("zaya_block_weights", _abi.zaya_block_weights),
               ("zaya_block_state", _abi.zaya_block_state), ("zaya_taps", _abi.zaya_taps)]
    for cname, ct in structs:
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in ct._fields_:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    for cname, ct in structs:
        assert int(got[cname]) == C.sizeof(ct), cname
        for f, _ in ct._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(ct, f).offset, (cname, f)


def test_status_strings_and_version():
    assert ZB.zaya_abi_version() == 3
    for code in range(8):
        assert isinstance(ZB.zaya_status_string(code), str)
    assert ZB.zaya_status_string(0) == "ok"
    assert "unknown" in ZB.zaya_status_string(99)


def test_workspace_size_and_config_checks():
    cfg = get_config("prefill_4k")
    c = ZB.make_config(cfg)
    n1 = ZB.zaya_workspace_size(c, ZB.ZAYA_PREFILL, 1, 4096)
    n2 = ZB.zaya_workspace_size(c, ZB.ZAYA_PREFILL, 2, 4096)
    assert 0 < n1 < n2
    assert ZB.zaya_workspace_size(c, ZB.ZAYA_DECODE, 64, 1) > 0
    assert ZB.zaya_stack_workspace_size(c, ZB.ZAYA_PREFILL, 1, 4096) > n1
    assert ZB.zaya_workspace_size(c, ZB.ZAYA_PREFILL, 0, 4096) == 0
    assert ZB.zaya_workspace_size(c, 7, 1, 1) == 0
    for bad in (dict(head_dim=96), dict(conv_width=2), dict(hidden=1000), dict(n_kv=3), dict(router_hidden=48)):
        assert ZB.zaya_workspace_size(ZB.make_config(cfg.with_(**bad)) if "conv_width" not in bad else
                                      _with_conv(c, bad["conv_width"]), ZB.ZAYA_PREFILL, 1, 8) == 0, bad


def _with_conv(c, w):
    c2 = _abi.zaya_config.from_buffer_copy(c)
    c2.conv_width = w
    return c2


def test_argument_errors_are_reported_before_launch():
    """Invalid arguments return their status on a machine without a GPU."""
    cfg = get_config("tiny")
    c = ZB.make_config(cfg)
    w = _abi.zaya_block_weights()
    st = _abi.zaya_block_state()
    L = _abi.lib()
    fake = C.c_void_p(256)
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st), None,
                              fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # NULL weights
    for name in _abi.WEIGHT_FIELDS:
        setattr(w, name, 4096)
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st), None,
                              fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # NULL state
    st.k_cache = st.v_cache = st.conv_state = st.prev_hs = st.cache_len = 4096
    st.cache_cap = 4
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st), None,
                              fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # cache too small for S
    st.cache_cap = 8
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, fake, C.byref(st), None,
                              fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # router state in aliases out
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, None, C.c_void_p(512), C.byref(st),
                              None, fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # block > 0 needs the carried state
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st),
                              None, C.c_void_p(4096), 16, None)
    assert rc == ZB._abi.ZAYA_ERR_WORKSPACE                    # workspace too small
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st),
                              None, C.c_void_p(4100), 1 << 30, None)
    assert rc == ZB._abi.ZAYA_ERR_MISALIGNED                   # workspace not 256-byte aligned
    setattr(w, "w_qkv", 4098)
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st),
                              None, fake, 1 << 30, None)
    assert rc == ZB._abi.ZAYA_ERR_MISALIGNED                   # bf16 operand off a 16-byte boundary
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 0, 8, fake, None, fake, C.c_void_p(512), C.byref(st),
                              None, fake, 1 << 30, None)
    assert rc in (ZB._abi.ZAYA_ERR_INVALID_ARG, ZB._abi.ZAYA_ERR_MISALIGNED)   # B = 0
    rc = L.zaya_stack_forward(C.byref(c), 0, None, None, None, 0, 1, 8, None, None, None, None, 0, None, 0, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG
    rc = L.zaya_device_status(None, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG


def test_noalloc_checks_arguments_before_enqueueing_anything():
    """The entry point without a caller workspace checks every argument
    before it touches a device (it clears its scratch header only after):
    on a machine without a GPU an invalid call returns its code, and a
    well-formed call too large for the fixed scratch returns
    ZAYA_ERR_WORKSPACE."""
    cfg = get_config("tiny")
    c = ZB.make_config(cfg)
    L = _abi.lib()
    w = _abi.zaya_block_weights()
    st = _abi.zaya_block_state()
    fake = C.c_void_p(256)
    rc = L.zaya_block_decode_noalloc(C.byref(c), C.byref(w), 1, 2, fake, fake, C.c_void_p(512), C.byref(st), None,
                                     None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # NULL weights
    for name in _abi.WEIGHT_FIELDS:
        setattr(w, name, 4096)
    rc = L.zaya_block_decode_noalloc(C.byref(c), C.byref(w), 1, 2, fake, fake, C.c_void_p(512), C.byref(st), None,
                                     None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # NULL state
    st.k_cache = st.v_cache = st.conv_state = st.prev_hs = st.cache_len = 4096
    st.cache_cap = 4
    rc = L.zaya_block_decode_noalloc(C.byref(c), C.byref(w), 1, 2, fake, fake, fake, C.byref(st), None, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # router state in aliases out
    rc = L.zaya_block_decode_noalloc(C.byref(c), C.byref(w), 1, 2, C.c_void_p(260), fake, C.c_void_p(512),
                                     C.byref(st), None, None)
    assert rc == ZB._abi.ZAYA_ERR_MISALIGNED                   # stream not 16-byte aligned
    big = ZB.make_config(get_config("prefill_4k"))
    rc = L.zaya_block_decode_noalloc(C.byref(big), C.byref(w), 1, 4096, fake, fake, C.c_void_p(512), C.byref(st),
                                     None, None)
    assert rc == ZB._abi.ZAYA_ERR_WORKSPACE                    # beyond the fixed scratch


def test_window_ring_arguments():
    """kv_ring: a window ring needs every block to slide (no full-attention
    blocks) and a cache of at least a window; both are checked before any
    launch."""
    cfg = get_config("tiny")
    assert ZB.zaya_workspace_size(ZB.make_config(cfg.with_(kv_ring=1)), ZB.ZAYA_DECODE, 2, 1) > 0
    assert ZB.zaya_workspace_size(ZB.make_config(cfg.with_(kv_ring=2)), ZB.ZAYA_DECODE, 2, 1) == 0
    assert ZB.zaya_workspace_size(ZB.make_config(cfg.with_(kv_fp8=2)), ZB.ZAYA_DECODE, 2, 1) == 0
    assert (ZB.zaya_workspace_size(ZB.make_config(cfg.with_(kv_fp8=1)), ZB.ZAYA_PREFILL, 1, 64)
            > ZB.zaya_workspace_size(ZB.make_config(cfg), ZB.ZAYA_PREFILL, 1, 64))
    hybrid = cfg.with_(kv_ring=1, sliding_period=2, sliding_phase=1)
    assert ZB.zaya_workspace_size(ZB.make_config(hybrid), ZB.ZAYA_DECODE, 2, 1) == 0
    # the prefill workspace of a ring also holds the prompt's linear K / V
    assert (ZB.zaya_workspace_size(ZB.make_config(cfg.with_(kv_ring=1)), ZB.ZAYA_PREFILL, 1, 64)
            > ZB.zaya_workspace_size(ZB.make_config(cfg), ZB.ZAYA_PREFILL, 1, 64))
    c = ZB.make_config(cfg.with_(kv_ring=1))
    L = _abi.lib()
    w = _abi.zaya_block_weights()
    for name in _abi.WEIGHT_FIELDS:
        setattr(w, name, 4096)
    st = _abi.zaya_block_state()
    st.k_cache = st.v_cache = st.conv_state = st.prev_hs = st.cache_len = 4096
    st.cache_cap = cfg.window - 1
    fake = C.c_void_p(256)
    rc = L.zaya_block_decode(C.byref(c), C.byref(w), 1, 2, fake, fake, C.c_void_p(512), C.byref(st), None,
                             fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # ring shorter than the window
    rc = L.zaya_block_prefill(C.byref(c), C.byref(w), 1, 1, 8, fake, None, fake, C.c_void_p(512), C.byref(st), None,
                              fake, 1 << 20, None)
    assert rc == ZB._abi.ZAYA_ERR_INVALID_ARG                  # the same in prefill
