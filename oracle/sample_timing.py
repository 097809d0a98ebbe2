"""Timing of the CPU oracle on a bounded sample — TEST INFRASTRUCTURE.

Only ``bench.py`` (its CPU-baseline leg and its reference arm) runs this
module.  It times the oracle's functions as they stand; nothing here is
tuned, and nothing here is used by the CUDA path.

One sample is one (sequence, KV head) group of one decode step: append one
token, score the pages, select, attend over the selection, and project the
group's heads through their share of the folded out-projection.

As a worker process:

    python -m oracle.sample_timing SAMPLE.npz START_EPOCH SECONDS

waits until the wall clock reaches START_EPOCH (so that several workers
time the same window), runs sample steps for SECONDS, and prints one JSON
line {"n": steps, "s": elapsed seconds}.
"""
from __future__ import annotations

import json
import sys
import time

import numpy as np

from oracle import basiskv_oracle as O

_SCALARS = ("T", "S", "top_k", "fp8", "r_b", "r_q", "n_sink", "n_recent")


def save_sample(path: str, arrays: dict, **scalars) -> None:
    """Writes one sample: arrays q [G][d], k, v [d], K [cap][d], Z [cap][r_v],
    E [cap][r_k], A_V [d][r_v], P_K [r_v][d], U_K [d][r_k], W [G][r_v][H]
    (the group's folded out-projection), and the scalars of _SCALARS."""
    np.savez(path, **arrays, **{k: np.asarray(scalars[k]) for k in _SCALARS})


def load_sample(path: str) -> dict:
    with np.load(path) as f:
        s = {k: f[k] for k in f.files}
    for k in _SCALARS:
        s[k] = int(s[k])
    return s


def group_step(s: dict) -> None:
    """One decode step of the sample's group through the oracle."""
    T = s["T"]
    z, e = O.append_latents(s["k"][None], s["v"][None], s["A_V"], s["P_K"], s["U_K"])
    Z, E, K = s["Z"].copy(), s["E"].copy(), s["K"].copy()
    store = O.to_e4m3 if s["fp8"] else O.to_bf16
    Z[T], E[T] = store(z[0]), store(e[0])
    K[T] = O.to_e4m3(s["k"]) if s["fp8"] else s["k"]
    sc = O.page_scores(s["q"], Z, E, s["P_K"], s["U_K"], T + 1, s["S"], s["r_b"], s["r_q"])
    sel, _ = O.select_pages(sc, s["top_k"], s["n_sink"], s["n_recent"])
    a, _ = O.attend(s["q"], K, Z, sel, T + 1, s["S"])
    O.outproj(a, s["W"])


def time_steps(s: dict, seconds: float) -> tuple:
    """Runs group steps for at least `seconds` (and at least one); returns
    (steps, elapsed seconds)."""
    n, t0 = 0, time.perf_counter()
    while n == 0 or time.perf_counter() - t0 < seconds:
        group_step(s)
        n += 1
    return n, time.perf_counter() - t0


def main(argv) -> None:
    path, start, seconds = argv[0], float(argv[1]), float(argv[2])
    s = load_sample(path)
    group_step(s)  # warm
    while time.time() < start:
        time.sleep(0.01)
    n, dt = time_steps(s, seconds)
    print(json.dumps({"n": n, "s": dt}), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
