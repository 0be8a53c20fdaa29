"""Writes tests/golden/tiny_trajectory.json from the CPU oracle alone.

Run:  python tests/golden/make_golden.py
The file records, for the tiny fp32 workload (d=64, 4 heads of 16, FFN 256,
N=64, rank-8 proxy, cosine > 0.99 lock, 20 steps, seed 0), the active count
of every step and a SHA-256 of each step's lock mask, so that a change in the
oracle's trajectory shows up as a diff of this file.
"""
import hashlib
import json
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def tiny_records():
    D = synth.TINY
    W = synth.layer_weights(D, 1.0 / math.sqrt(D.d))
    X0 = synth.hidden_states(D)
    Ut = synth.proxy_basis(D.d, synth.TINY_RANK, dtype="f32").astype(np.float64)
    lock0 = synth.bernoulli_active(D.B, D.N, synth.TINY_P_ACTIVE)
    noises = [synth.step_noise((D.B, D.N, D.d), synth.TINY_NOISE_VAR, step=t)
              for t in range(synth.TINY_STEPS)]
    recs = oracle.tiny_run(D, W, X0, Ut, lock0, noises, synth.TINY_TAU,
                           lambda X, e, m: synth.perturb_rows(X, e, m, "f32"))
    return lock0, recs


def main():
    lock0, recs = tiny_records()
    out = {
        "workload": "tiny fp32 layer, d=64, H=4x16, F=256, N=64, r=8, tau=0.99, 20 steps, seed 0",
        "initial_active": int((lock0 == 0).sum()),
        "active_per_step": [int(r["idx"].size) for r in recs],
        "lock_sha256": [hashlib.sha256(r["lock"].tobytes()).hexdigest()[:16] for r in recs],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_trajectory.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path, out["active_per_step"])


if __name__ == "__main__":
    main()
