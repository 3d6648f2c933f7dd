"""Calibrate the generator's amplitude factor so the long workloads hit their target density.

TEST INFRASTRUCTURE (calls only the oracle and the seeded input generator).
Writes ``block_sparse_long_blocks_b200/workloads_calibration.json``.

The 128K workload is tuned so that about 5% of causal (KV group, query block,
key block) pairs pass discovery, and the 256K one to 3-4%, the retention the
FlashPrefill summary page reports at 256K (Results: 3.5% of blocks retained).
Density is measured with the oracle's own discovery (float64 block pooling,
per-head threshold, union over the group, sink/window forcing) on the exact
bfloat16 tensors the generator emits, and the factor is found by bisection.

Usage:  python -m oracle.calibrate_workloads [--only NAME]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_long_blocks_b200 import workloads as wl  # noqa: E402
from oracle import flashprefill_oracle as fo  # noqa: E402

OUT = os.path.join(ROOT, "block_sparse_long_blocks_b200", "workloads_calibration.json")

TARGETS = {"qwen30b_128k": (0.045, 0.055), "extreme_256k": (0.030, 0.040)}


def pooled(t, B, chunk=4):
    """Block means of a bfloat16 tensor [L, H, d], converted to float64 a few heads at a time."""
    H = t.shape[1]
    parts = []
    for h0 in range(0, H, chunk):
        parts.append(fo.pool_blocks(t[:, h0:h0 + chunk].double().numpy(), B))
    return np.concatenate(parts, axis=1)


def density(w) -> float:
    inp = wl.make_inputs(w)
    q, k = inp.q[0], inp.k[0]
    B = w.block
    qbar, kbar = pooled(q, B), pooled(k, B)
    Sb, Wb = fo.forced_blocks(w.sink_tokens, w.window_tokens, B)
    mask = fo.block_mask(qbar, kbar, fo.default_scale(w.head_dim), w.alpha, Sb, Wb)
    N = mask.shape[1]
    return float(mask.sum()) / (w.hkv * N * (N + 1) / 2)


def calibrate(name: str, lo: float = 1.0, hi: float = 4.0, iters: int = 14):
    base = wl.workloads()[name]
    tlo, thi = TARGETS[name]
    target = 0.5 * (tlo + thi)
    log = []
    # density decreases as the amplitude (hence the heavy/noise score gap) grows
    dlo = density(base.with_(amp_scale=lo))
    dhi = density(base.with_(amp_scale=hi))
    log += [(lo, dlo), (hi, dhi)]
    if not (dlo > target > dhi):
        raise RuntimeError(f"{name}: target {target} not bracketed: {log}")
    c = hi
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        d = density(base.with_(amp_scale=mid))
        log.append((mid, d))
        print(f"  {name}: amp_scale={mid:.6f} density={d:.5f}", flush=True)
        if tlo <= d <= thi:
            c = mid
            break
        if d > target:
            lo = mid
        else:
            hi = mid
        c = mid
    return c, log


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", default=None)
    args = ap.parse_args()
    try:
        with open(OUT) as f:
            data = json.load(f)
    except OSError:
        data = {}
    data["about"] = ("Amplitude factor of the synthetic generator per workload, found by "
                     "bisection on the oracle's discovery density (written by "
                     "oracle/calibrate_workloads.py). Targets: 128K ~5% of causal blocks, "
                     "256K 3-4%.")
    data.setdefault("amp_scale", {})
    data.setdefault("density", {})
    for name in TARGETS:
        if args.only and name != args.only:
            continue
        t0 = time.time()
        c, log = calibrate(name)
        data["amp_scale"][name] = c
        data["density"][name] = [d for (a, d) in log if a == c][-1]
        print(f"{name}: amp_scale={c} ({time.time() - t0:.0f}s)")
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1)


if __name__ == "__main__":
    main()
