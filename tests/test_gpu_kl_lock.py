"""GPU parity of the SureLock KL lock rule (plk_kl_lock) against the oracle.

Tolerances: KL and H are fp32 results of sums over the V vocabulary entries;
the fp32 parity bound of this library (1e-4 relative) applies, with an absolute floor for KL
values near zero (2e-7) and for H (1e-5 nats: H = lse - E_p[z] carries the
rounding of lse ~ |max z|).  The lock bit is decided on the GPU's own fp32 KL
and H, so it is checked bit-exactly against the rule applied to those values,
and against the oracle's decision wherever the oracle's KL is not within the
tolerance band of eps.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import Guarded, check_guards, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plk():
    import partial_recompute_kv_b200 as m
    return m


def _run(plk, zt, zp, lock_in, eps, h_max, dtype):
    B, N, V = zt.shape
    dm = plk.dims(B, N, 256, 2, 128, 512, dtype=plk.BF16 if dtype == "bf16" else plk.F32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = {"lock": Guarded((B, N), torch.uint8, init=lock_in), "kl": Guarded((B, N), torch.float32, fill=-7.0),
         "h": Guarded((B, N), torch.float32, fill=-7.0)}
    lk, kl, h = g["lock"].t, g["kl"].t, g["h"].t
    plk.kl_lock(dm, V, dev(zt, tdt), dev(zp, tdt), lk, lk, eps, h_max, kl, h)  # lock in place
    assert plk.get_status() == plk.OK
    check_guards(g, "kl_lock")
    return host(lk), host(kl), host(h)


CASES = [  # (B, N, V, dtype, gate)
    (2, 7, 50, "f32", False),        # V not a multiple of the vector width: scalar path
    (1, 64, 4096, "bf16", False),
    (2, 24, 1004, "bf16", True),     # 2008-byte rows: not 16-byte aligned, scalar path
    (1, 12, synth.VOCAB_8B, "bf16", True),
]


@pytest.mark.parametrize("B,N,V,dtype,gate", CASES, ids=[f"{c[3]}-V{c[2]}" for c in CASES])
def test_kl_lock_matches_oracle(plk, B, N, V, dtype, gate):
    zt, zp = synth.logits_pair(B, N, V, seed=V, dtype=dtype)
    lock_in = synth.bernoulli_active(B, N, 0.75, seed=V) if B * N > 4 else np.zeros((B, N), np.uint8)
    act = lock_in == 0
    kl_ref = oracle.kl_divergence(zt.astype(np.float64), zp.astype(np.float64))
    h_ref = oracle.entropy(zt.astype(np.float64))
    eps = float(np.median(kl_ref[act]))
    h_max = float(np.median(h_ref[act])) if gate else math.inf
    ref_lock, _, _ = oracle.kl_lock(zt, zp, lock_in, eps, h_max)
    lock, kl, h = _run(plk, zt, zp, lock_in, eps, h_max, dtype)
    # values at examined rows
    kl_tol = 1e-4 * np.abs(kl_ref[act]) + 2e-7
    h_tol = 1e-4 * np.abs(h_ref[act]) + 1e-5
    assert np.all(np.abs(kl[act] - kl_ref[act]) <= kl_tol), np.max(np.abs(kl[act] - kl_ref[act]) - kl_tol)
    assert np.all(np.abs(h[act] - h_ref[act]) <= h_tol), np.max(np.abs(h[act] - h_ref[act]) - h_tol)
    # locked rows: not examined (outputs untouched), still locked
    assert np.all(lock[~act] == 1) and np.all(kl[~act] == -7.0) and np.all(h[~act] == -7.0)
    # the bit follows the rule on the GPU's own fp32 values
    np.testing.assert_array_equal(lock[act], ((kl[act] <= np.float32(eps)) & (h[act] <= np.float32(h_max))))
    # and the oracle's decision away from the threshold band
    clear = act & (np.abs(kl_ref - eps) > 1e-4 * abs(eps) + 2e-7)
    if gate:
        clear &= np.abs(h_ref - h_max) > 1e-4 * abs(h_max) + 1e-5
    np.testing.assert_array_equal(lock[clear], ref_lock[clear])
    assert 0 < int(lock[act].sum()) < int(act.sum())  # the threshold splits the rows


def test_kl_lock_identical_steps_lock_everything(plk):
    zt, _ = synth.logits_pair(1, 16, 2048, seed=3, dtype="bf16")
    lock, kl, h = _run(plk, zt, zt, np.zeros((1, 16), np.uint8), 0.0, math.inf, "bf16")
    assert np.all(lock == 1) and np.all(np.abs(kl) <= 2e-7)
