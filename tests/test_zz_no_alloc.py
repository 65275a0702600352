"""zaya_block_decode_noalloc: the decode step for callers that cannot
allocate device memory (no workspace argument; the library's fixed scratch is
used instead).  Two decode steps in a row through the no-allocation entry
point must give what two steps through zaya_block_decode give.

This file is collected last on purpose, and holds up both alone in a fresh
process and after every other test (the scratch keeps earlier contents)."""
import ctypes as C

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


@pytest.mark.parametrize("name,B", [("tiny", 3), ("prefill_4k", 64)])
def test_noalloc_decode_matches_workspace_decode(name, B):
    import top_moe_block_b200 as ZB
    from tests import harness as Hn
    S = 48
    cfg = get_config(name).with_(seq=S, batch=B)
    W = gen_block_weights(cfg)
    Wd = Hn.dev_weights(W)
    inp = gen_prefill_inputs(cfg.with_(seq=S + 2))
    x, rin = inp["x"], inp["router_state_in"]
    st = Hn.new_state(cfg, B, S + 4)
    Hn.gpu_prefill(cfg, Wd, x[:, :S], None, rin[:, :S], state=st, taps=False)
    st_ref = {k: v.clone() for k, v in st.items()}
    st_new = {k: v.clone() for k, v in st.items()}
    c = ZB.make_config(cfg)
    w = ZB.make_weights(Wd)
    ws = Hn.workspace(ZB.zaya_workspace_size(c, ZB.ZAYA_DECODE, B, 1))
    for step in range(2):
        xs = x[:, S + step].cuda().contiguous()
        rs = rin[:, S + step].cuda().contiguous()
        h_ref, h_new = xs.clone(), xs.clone()
        r_ref = torch.full((B, cfg.router_hidden), float("nan"), device="cuda")
        r_new = torch.full((B, cfg.router_hidden), float("nan"), device="cuda")
        ZB.zaya_block_decode(c, w, cfg.block_idx, B, h_ref, rs, r_ref, ZB.make_state(st_ref), None, ws)
        ZB.zaya_block_decode_noalloc(c, w, cfg.block_idx, B, h_new, rs, r_new, ZB.make_state(st_new))
        torch.cuda.synchronize()
        assert ZB.zaya_device_status(ws) == 0
        assert ZB.zaya_noalloc_status() == 0        # the fixed scratch's own status word
        a, b = h_new.cpu().numpy(), h_ref.cpu().numpy()
        assert Hn.rel_max(a, b) <= Hn.TOL_REL_MAX and Hn.cosine(a, b) >= Hn.TOL_COS
        np.testing.assert_allclose(r_new.cpu().numpy(), r_ref.cpu().numpy(), rtol=1e-6, atol=1e-6)
        for k in ("k_cache", "v_cache", "conv_state", "prev_hs"):
            assert Hn.rel_max(st_new[k].float().cpu().numpy(), st_ref[k].float().cpu().numpy()) <= Hn.TOL_REL_MAX, k
        assert torch.equal(st_new["cache_len"], st_ref["cache_len"])
        assert int(st_new["cache_len"][0]) == S + step + 1


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A decode step whose workspace would exceed the fixed 8 MiB returns
    ZAYA_ERR_WORKSPACE before launching anything."""
    import top_moe_block_b200 as ZB
    from top_moe_block_b200 import _abi
    cfg = get_config("prefill_4k")
    c = ZB.make_config(cfg)
    B = 4096
    assert ZB.zaya_workspace_size(c, ZB.ZAYA_DECODE, B, 1) > 8 << 20
    w = _abi.zaya_block_weights()
    for n in _abi.WEIGHT_FIELDS:
        setattr(w, n, 4096)
    st = _abi.zaya_block_state()   # well-formed but never dereferenced: the call must stop at the size
    st.k_cache, st.v_cache, st.cache_len, st.conv_state, st.prev_hs = 1024, 2048, 3072, 4096, 5120
    st.cache_cap = 8
    rc = _abi.lib().zaya_block_decode_noalloc(C.byref(c), C.byref(w), 1, B, C.c_void_p(256), C.c_void_p(512),
                                              C.c_void_p(768), C.byref(st), None, None)
    assert rc == _abi.ZAYA_ERR_WORKSPACE
