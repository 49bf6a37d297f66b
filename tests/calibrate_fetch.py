#!/usr/bin/env python
"""Writes synth/fetch_calibration.json: for each workload, seed and sequence, the target handed to
the generator's head-weight model (synth.model_target) that makes the fetch rate of the whole path
on that sequence's own inputs equal the wanted rate.  The whole path is stage 1 (c = h W^DQ,
q = c W^IUQ, w = h W^w), the index score, the threshold and the OR over the indexer layers (blog
review, sections 3.1 and 4.2); the rates are measured with the CPU oracle only.

The wanted rates are the workloads' own: about 13.5 % of the entries (blog review, section 5
table: 0.10 GB of 0.93 GB), 15 % for the tiny workload, and 1-40 % per sequence for the ragged mix
(spanning the review's 8.4 % background fetch, section 6.1, and 30-49 % with eight indexer layers,
section 4.2).  Per sequence the model target is adjusted by secant steps in logit space until the
measured rate is within tolerance; long sequences are measured on a fixed seeded sample of their
entries (all entries up to `--sample`).

    python tests/calibrate_fetch.py [--workloads a,b,...] [--sample 16384]
"""
import argparse
import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

CHUNK_ENTRIES = 1 << 20      # sequences generated together (bounds host memory)


def logit(p):
    p = min(max(p, 1e-6), 1 - 1e-6)
    return math.log(p / (1 - p))


def sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


def sample_entries(wl, b, n):
    S = wl.S[b]
    if S <= n:
        return np.arange(S, dtype=np.int64)
    rng = np.random.default_rng([wl.seed, 4242, wl._ids()[b]])
    return np.sort(rng.choice(S, n, replace=False)).astype(np.int64)


def measure(base, model_targets, samples):
    """Fetch rate of every sequence of `base` through the whole path, with the head weights drawn
    for the given model targets (the workload is renamed so that no calibration entry applies)."""
    wl = synth.workload(base.name, fetch=tuple(model_targets), name=base.name + "#calibrating")
    rates = np.zeros(wl.B)
    b0 = 0
    while b0 < wl.B:
        b1 = b0
        n = 0
        while b1 < wl.B and (b1 == b0 or n + wl.S[b1] <= CHUNK_ENTRIES):
            n += wl.S[b1]
            b1 += 1
        sub = wl.subset(range(b0, b1))
        inp = synth.make_inputs(sub, parts=("proj", "score"))
        q, w = oracle.project(inp.h, inp.W_dq, inp.W_iuq, inp.W_w, sub.n_h, sub.d_I)
        offs = inp.seq_offsets.numpy()
        eb = np.concatenate([np.full(samples[b].size, b - b0, dtype=np.int32) for b in range(b0, b1)])
        es = np.concatenate([samples[b] for b in range(b0, b1)])
        x = oracle.score_entries(q, w, inp.K, inp.k_scale, offs, eb, es)     # [L][n] logits
        fetched = (x >= 0.0).any(axis=0)
        pos = 0
        for b in range(b0, b1):
            m = samples[b].size
            rates[b] = fetched[pos:pos + m].mean()
            pos += m
        b0 = b1
    return rates


def calibrate(name, sample, max_iter=8, verbose=True):
    base = synth.WORKLOADS[name]
    wanted = np.asarray(base.fetch, dtype=np.float64)
    samples = [sample_entries(base, b, sample) for b in range(base.B)]
    tol = np.maximum(0.001, np.array([2.0 / math.sqrt(s.size) * math.sqrt(p * (1 - p)) for s, p in zip(samples, wanted)]))
    x_prev = None
    y_prev = None
    x = np.array([logit(p) for p in wanted])
    for it in range(max_iter):
        t0 = time.time()
        r = measure(base, [sigmoid(v) for v in x], samples)
        y = np.array([logit(max(v, 0.5 / s.size)) for v, s in zip(r, samples)])
        err = r - wanted
        if verbose:
            print(f"{name} iteration {it}: mean rate {r.mean():.4f} (wanted {wanted.mean():.4f}), "
                  f"max |rate - wanted| {np.abs(err).max():.4f}, {time.time() - t0:.0f} s", flush=True)
        done = np.abs(err) <= tol
        if done.all():
            break
        yw = np.array([logit(p) for p in wanted])
        if x_prev is None:
            x_new = x + (yw - y)
        else:
            slope = (y - y_prev) / np.where(np.abs(x - x_prev) > 1e-9, x - x_prev, 1e-9)
            slope = np.clip(np.where(np.isfinite(slope), slope, 1.0), 0.2, 5.0)
            x_new = x + (yw - y) / slope
        x_new = np.where(done, x, x_new)
        x_prev, y_prev, x = x, y, x_new
    return {"seed": base.seed, "target": [float(v) for v in base.fetch],
            "model_target": [float(sigmoid(v)) for v in x], "measured": [float(v) for v in r],
            "sample_entries": [int(s.size) for s in samples]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default="tiny_fp32,ctx128k_bf16,ctx500k_bf16_b8,ctx1m_fp8_b32,ragged_mix_b64")
    ap.add_argument("--sample", type=int, default=16384)
    ap.add_argument("--out", default=synth.CALIBRATION_FILE)
    a = ap.parse_args()
    try:
        with open(a.out) as f:
            table = json.load(f)
    except (OSError, ValueError):
        table = {}
    for name in a.workloads.split(","):
        table[name] = calibrate(name, a.sample)
        with open(a.out, "w") as f:
            json.dump(table, f, indent=1)
            f.write("\n")
    print("wrote", a.out)


if __name__ == "__main__":
    main()
