"""GPU parity of the SlowFast span policy against the oracle (bit-exact).

Every step of a decoding trajectory runs on both sides from the same seeded
confidences; the masked rows, the unmasked positions, the lock rows and the
per-sequence state (phase, s, e, slow-step count and the valid end points of
the ring) must agree exactly.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import plk_oracle as po
from tests.parity_util import Guarded, check_guards

pytestmark = pytest.mark.gpu

plk = pytest.importorskip("partial_recompute_kv_b200")


def _dims(B, N):
    return plk.dims(B, N, 64, 4, 16, 64, dtype=plk.F32)  # only B and N are read


def _check_state(row, ost, w, where):
    row = [int(v) for v in row]
    assert row[:4] == [ost.phase, ost.s, ost.e, ost.nslow], (where, row[:4], vars(ost))
    for n in range(max(0, ost.nslow - w), ost.nslow):  # the ring slots written in this cycle
        assert row[4 + n % w] == ost.hist[n], (where, n, row[4:4 + w], ost.hist)


def _trajectory(B, N, prompt, steps, seed, rate=16.0, nan_every=0, outputs=True, **kw):
    prm = dict(k=1, tau_conv=0.5, tau_high=0.9, var_stable=1.0, w_hist=2, k_max=8)
    prm.update(kw)
    dm, params, op = _dims(B, N), plk.sf_params(**prm), po.SpanParams(**prm)
    m_or = synth.generation_mask(B, N, prompt)
    guards = {"masked": Guarded((B, N), torch.uint8, init=m_or), "state": Guarded((B, plk.SF_STATE_WORDS), torch.int32,
                                                                                  fill=0)}
    if outputs:
        guards["unmask"] = Guarded((B, N), torch.uint8, fill=7)
        guards["lock"] = Guarded((B, N), torch.uint8, fill=7)
    m_dev, st_dev = guards["masked"].t, guards["state"].t
    un = guards["unmask"].t if outputs else None
    lk = guards["lock"].t if outputs else None
    states = [po.SpanState() for _ in range(B)]
    phases = set()
    for t in range(steps):
        conf = synth.span_confidences(B, N, t, seed=seed, prompt=prompt, rate=rate)
        if nan_every:
            conf[:, t % nan_every::nan_every] = np.nan
        plk.slowfast_step(dm, params, torch.from_numpy(conf).cuda(), m_dev, st_dev, un, lk)
        m_or, u_or, l_or, states = po.slowfast_step(conf, m_or, states, op)
        torch.cuda.synchronize()
        assert np.array_equal(m_dev.cpu().numpy(), m_or), t
        if outputs:
            assert np.array_equal(un.cpu().numpy(), u_or), t
            assert np.array_equal(lk.cpu().numpy(), l_or), t
        st_np = st_dev.cpu().numpy()
        for b in range(B):
            _check_state(st_np[b], states[b], op.w_hist, (t, b))
            phases.add(states[b].phase)
        if not m_or.any():
            break
    check_guards(guards, "slowfast trajectory")
    return t + 1, phases, m_or


@pytest.mark.parametrize("B,N,prompt,kw", [
    (3, 2500, 100, dict(k=2, tau_conv=0.6, tau_high=0.85)),                 # ragged N, several tiles
    (2, 1000, 0, dict(k=1, w_hist=3, k_max=4, var_stable=50.0)),
    (5, 77, 5, dict(k=100, w_hist=1, k_max=1, tau_high=-np.inf)),            # k above the masked count
    (5, 77, 5, dict(k=3, w_hist=1, k_max=1, tau_high=-np.inf)),              # every span decoded at once
    (2, 300, 30, dict(k=3, tau_high=np.inf, var_stable=np.inf)),             # always the fallback
    (4, 1024, 64, dict(k=4, w_hist=16, k_max=16, var_stable=400.0)),         # the largest window
    (2, 600, 40, dict(k=20, k_max=3, tau_conv=0.3, tau_high=0.97)),          # k > 16: radix select
    (1, 20000, 19000, dict(k=3)),                                            # too long to stage in smem
])
def test_slowfast_trajectory_matches_oracle(B, N, prompt, kw):
    steps, phases, left = _trajectory(B, N, prompt, 600, seed=B + N, **kw)
    assert not left.any(), "trajectory did not finish"
    assert phases == {po.SF_SLOW, po.SF_FAST} or kw.get("k_max") == 1


def test_slowfast_nan_and_ties():
    _trajectory(2, 700, 50, 300, seed=3, nan_every=11, k=5, tau_conv=0.5, tau_high=0.75)


def test_slowfast_without_outputs():
    _trajectory(2, 500, 20, 120, seed=4, outputs=False, k=2)


@pytest.mark.parametrize("B,N,prompt", [(4, 2048, 1024), (1, 8192, 7936)])
def test_slowfast_workload_shapes(B, N, prompt):
    # the 32-layer stack's batch (4 x 2048) and the long-context sequence (8192 with
    # 256 generated positions), at K_max = 8, W_hist = 2, variance threshold 1.0
    _trajectory(B, N, prompt, 80, seed=N, k=2, tau_conv=0.7, tau_high=0.9)


def test_slowfast_single_position():
    _trajectory(1, 1, 0, 3, seed=9)


def test_slowfast_edge_states():
    B, N = 4, 40
    dm, params, op = _dims(B, N), plk.sf_params(k=2), po.SpanParams(k=2)
    rng = np.random.default_rng(12)
    conf = np.round(rng.random((B, N)) * 8).astype(np.float32) / 8  # many ties
    masked = np.ones((B, N), dtype=np.uint8)
    masked[0] = 0                                  # sequence 0: nothing masked
    st = np.zeros((B, plk.SF_STATE_WORDS), dtype=np.int32)
    st[0, :4] = [1, 3, 9, 2]                       # left unchanged
    st[1, :4] = [7, 5, 6, -3]                      # invalid phase -> initial state
    st[2, :4] = [1, 10, 5, 1]                      # fast with an empty span -> cycle ends
    masked[2, :8] = 0
    st[3, :4] = [0, 0, 0, -1]                      # negative count -> initial state
    ostates = [po.SpanState(*st[b, :4], hist=()) for b in range(B)]
    m_dev, st_dev = torch.from_numpy(masked.copy()).cuda(), torch.from_numpy(st.copy()).cuda()
    un = torch.empty((B, N), dtype=torch.uint8, device="cuda")
    lk = torch.empty((B, N), dtype=torch.uint8, device="cuda")
    plk.slowfast_step(dm, params, torch.from_numpy(conf).cuda(), m_dev, st_dev, un, lk)
    m_or, u_or, l_or, ost = po.slowfast_step(conf, masked, ostates, op)
    torch.cuda.synchronize()
    assert np.array_equal(m_dev.cpu().numpy(), m_or)
    assert np.array_equal(un.cpu().numpy(), u_or)
    assert np.array_equal(lk.cpu().numpy(), l_or)
    got = st_dev.cpu().numpy()
    assert got[0, :4].tolist() == [1, 3, 9, 2] and l_or[0].all()
    for b in range(1, B):
        _check_state(got[b], ost[b], op.w_hist, b)
    assert u_or[2].sum() == 0 and ost[2].phase == po.SF_SLOW


def test_slowfast_lock_feeds_compaction():
    B, N, prompt = 2, 600, 40
    dm, params, op = _dims(B, N), plk.sf_params(k=2, k_max=2), po.SpanParams(k=2, k_max=2)
    m_dev = torch.from_numpy(synth.generation_mask(B, N, prompt)).cuda()
    st_dev = plk.sf_state(B)
    lk = torch.empty((B, N), dtype=torch.uint8, device="cuda")
    lk2 = torch.empty_like(lk)
    idx = torch.empty(B * N, dtype=torch.int32, device="cuda")
    seg = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    score = torch.zeros((B, N), dtype=torch.float32, device="cuda")
    seen_fast = False
    for t in range(6):
        conf = synth.span_confidences(B, N, t, seed=21, prompt=prompt)
        plk.slowfast_step(dm, params, torch.from_numpy(conf).cuda(), m_dev, st_dev, None, lk)
        plk.select_active(dm, score, lk, lk2, plk.SEL_THRESH_GT, float("inf"), 0, idx, seg)
        torch.cuda.synchronize()
        lock = lk.cpu().numpy()
        want_idx, want_seg = po.compact(lock)
        assert seg.cpu().numpy().tolist() == want_seg.tolist()
        assert idx[:int(want_seg[-1])].cpu().numpy().tolist() == want_idx.tolist()
        seen_fast |= bool(lock.any())
    assert seen_fast
