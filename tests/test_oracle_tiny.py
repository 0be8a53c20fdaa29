"""The tiny fp32 workload through the oracle: invariants of the SureLock page
("Stopping Computation for Converged Tokens in Masked Diffusion-LM Decoding",
Sec. 2 "Permanent Deactivation" and "Algorithmic Complexity": M_t is monotone
non-increasing, locked rows are frozen) and the recorded trajectory."""
import hashlib
import json
import os

import numpy as np

from tests.golden.make_golden import tiny_records

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_trajectory_invariants_and_golden():
    lock0, recs = tiny_records()
    prev_lock = lock0
    prev_state = None
    for r in recs:
        lock = r["lock"]
        assert np.all(lock >= prev_lock), "locking is permanent"
        active_before = prev_lock == 0
        # the decision margin: every score that decided a lock is far from tau,
        # so fp32 and fp64 take the same decision
        s = r["score"][active_before]
        if s.size:
            assert np.min(np.abs(s - 0.99)) > 1e-4
        if prev_state is not None:
            frozen = lock.astype(bool)
            for key in ("K", "V", "Y"):
                assert np.array_equal(r[key][frozen], prev_state[key][frozen])
            np.testing.assert_array_equal(r["proxy"][frozen], prev_state["proxy"][frozen])
        prev_lock, prev_state = lock, r
    counts = [int(r["idx"].size) for r in recs]
    assert all(a >= b for a, b in zip(counts, counts[1:]))
    with open(os.path.join(HERE, "golden", "tiny_trajectory.json")) as f:
        g = json.load(f)
    assert g["initial_active"] == int((lock0 == 0).sum())
    assert g["active_per_step"] == counts
    assert g["lock_sha256"] == [hashlib.sha256(r["lock"].tobytes()).hexdigest()[:16] for r in recs]
