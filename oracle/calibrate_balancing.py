"""Fit a workload's router balancing biases to target expert loads.

Writes ``synthetic/balancing_<workload>.json``.  Runs the CPU oracle only:
the router logits of a calibration batch (an independent draw of the
workload's input distribution, never the batch that is later measured) are
computed once, then the biases follow the fixed-point update
``b_e += eta * (target_e - load_e)`` for at most 200 iterations, on the
selection rule of the zaya page ("One expert per token, chosen beside a
skip class": argmax of softmax + balancing_biases).  The achieved load
histogram is stored beside the biases.

Usage:  python oracle/calibrate_balancing.py tiny prefill_skewed_8x2k
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import zaya_oracle as Z  # noqa: E402
from synthetic import get_config, gen_block_weights, gen_prefill_inputs  # noqa: E402

CALIB_STREAM = 1000


def target_loads(cfg) -> np.ndarray:
    """[E+1] target shares: experts ~ Zipf(s) (uniform when s = 0) over the
    routed share, skip = skip_frac."""
    E = cfg.n_experts
    ranks = np.arange(1, E + 1, dtype=np.float64)
    z = ranks ** (-cfg.zipf_s) if cfg.zipf_s > 0 else np.ones(E)
    t = np.empty(E + 1)
    t[:E] = (1.0 - cfg.skip_frac) * z / z.sum()
    t[E] = cfg.skip_frac
    return t


def calibration_logits(cfg, W) -> np.ndarray:
    calib_cfg = cfg.with_(batch=1, seq=min(cfg.seq, 2048), pad_max=0)
    inp = gen_prefill_inputs(calib_cfg, stream=CALIB_STREAM)
    W0 = dict(W)
    W0["balancing"] = np.zeros(cfg.n_experts + 1)
    o = Z.block_prefill(calib_cfg, W0, inp["x"], None, inp["router_state_in"])
    return o["router_logits"].reshape(-1, cfg.n_experts + 1)


def fit(cfg, logits, iters=200, eta=0.05):
    E = cfg.n_experts
    tgt = target_loads(cfg)
    b = np.zeros(E + 1, dtype=np.float32)
    best = (np.inf, b.copy(), None)
    for _ in range(iters):
        cls = Z.select(logits, b, E)[0]
        load = np.bincount(cls, minlength=E + 1) / len(cls)
        err = np.abs(load - tgt).sum()
        if err < best[0]:
            best = (err, b.copy(), load)
        b = (b + eta * (tgt - load)).astype(np.float32)
        b = (b - b[:E].mean()).astype(np.float32)
    return best


def main(names):
    for name in names:
        cfg = get_config(name).with_(calibrated=0)
        W = gen_block_weights(cfg)
        logits = calibration_logits(cfg, W)
        err, b, load = fit(cfg, logits)
        b = [float(np.float32(v)) for v in b]
        out = {"workload": name, "balancing_biases": b,
               "target_loads": [float(v) for v in target_loads(cfg)],
               "calibration_loads": [float(v) for v in load], "l1_error": float(err),
               "calibration_tokens": int(logits.shape[0]),
               "method": "fixed-point b += 0.05*(target-load), 200 iters, best L1 kept; "
                         "calibration batch = independent input draw (stream 1000)"}
        path = os.path.join(ROOT, "synthetic", f"balancing_{name}.json")
        with open(path, "w") as f:
            json.dump(out, f, indent=1)
        print(name, "L1 err", round(err, 4), "loads", np.round(load, 3))


if __name__ == "__main__":
    main(sys.argv[1:] or ["tiny", "prefill_skewed_8x2k"])
