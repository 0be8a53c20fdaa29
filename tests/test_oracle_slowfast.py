"""Pins of the oracle's SlowFast span policy (the SlowFast Sampling page, part 2
"Methodology", the two-stage pipeline; part 4 "Ablation Studies").

The pages print no trajectory, so the oracle is pinned by
  - hand-worked trajectories: the expected unmasking, lock rows and state of
    every step were derived by hand from the stated rules, not by running code;
  - reductions: with the fast phase unreachable the policy is the plain
    "unmask the k most confident" sampler (checked against numpy's lexsort);
    with W_hist = 1 and tau_high = -inf every span is decoded in one fast step;
  - the exact variance against the standard library and the W = 2 closed form;
  - invariants on seeded random trajectories;
  - planted mistakes, each of which one of the above must catch.
"""
import inspect
import math
import statistics
import textwrap
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import plk_oracle as po

SLOW, FAST = po.SF_SLOW, po.SF_FAST
_ = 1.0  # confidence of a position whose value does not matter (already decoded)


def _run(fn, p, N, masked0, steps):
    """Runs hand-worked steps: (conf, unmasked positions, lock rows, (phase, s, e, nslow, hist))."""
    masked = np.array(masked0, dtype=np.uint8)
    st = po.SpanState()
    for t, (conf, want_unmask, want_lock, want_state) in enumerate(steps):
        conf = np.array(conf, dtype=np.float32)
        assert conf.shape == (N,)
        before = masked.copy()
        masked, unmask, lock, st = fn(conf, masked, st, p)
        got = sorted(int(i) for i in np.flatnonzero(unmask))
        assert got == sorted(want_unmask), (t, got, want_unmask)
        assert np.array_equal(masked, before & (1 - unmask)), t
        assert lock.tolist() == list(want_lock), (t, lock.tolist(), want_lock)
        assert (st.phase, st.s, st.e, st.nslow, st.hist) == want_state, (t, vars(st), want_state)


# Example A (N = 10, prompt = positions 0-1): slow steps, the switch on a small
# variance, in-span unmasking that ignores a confident position outside the
# span, the fallback, the end of the cycle, a variance exactly at the threshold
# (no switch: the comparison is strict), and the finished sequence.
P_A = po.SpanParams(k=1, tau_conv=0.5, tau_high=0.8, var_stable=1.0, w_hist=2, k_max=8)
MASK_A = [0, 0, 1, 1, 1, 1, 1, 1, 1, 1]
STEPS_A = [
    # s = 2; converged {2,3,4} -> e_t = 4; top-1 = 2
    ([1, 1, .9, .6, .7, .2, .1, .1, .1, .1], [2], [0] * 10, (SLOW, 2, 0, 1, [4])),
    # converged {3,4,5} -> e_t = 5; var(4,5) = 1/4 < 1 -> fast on [2,5]; top-1 = 4
    ([1, 1, _, .6, .7, .6, .1, .1, .1, .1], [4], [1, 1, 0, 0, 0, 0, 1, 1, 1, 1], (FAST, 2, 5, 2, [4, 5])),
    # in span {3,5}: only 3 is above 0.8 (6 is confident but outside the span)
    ([1, 1, _, .85, _, .5, .95, .1, .1, .1], [3], [1, 1, 0, 0, 0, 0, 1, 1, 1, 1], (FAST, 2, 5, 2, [4, 5])),
    # nothing above 0.8 in the span -> fallback top-1 = 5; span decoded -> cycle ends
    ([1, 1, _, _, _, .3, .95, .1, .1, .1], [5], [0] * 10, (SLOW, 0, 0, 0, [])),
    # new cycle s = 6; converged {8} -> e_t = 8; top-1 = 8
    ([1, 1, _, _, _, _, .3, .2, .9, .1], [8], [0] * 10, (SLOW, 6, 0, 1, [8])),
    # nothing converged -> e_t = s = 6; var(8,6) = 1, not < 1 -> stays slow; top-1 = 7
    ([1, 1, _, _, _, _, .1, .4, _, .2], [7], [0] * 10, (SLOW, 6, 0, 2, [8, 6])),
    # converged {6,9} -> e_t = 9; var(6,9) = 9/4 -> slow; top-1 = 6
    ([1, 1, _, _, _, _, .6, _, _, .55], [6], [0] * 10, (SLOW, 6, 0, 3, [8, 6, 9])),
    # e_t = 6; var(9,6) = 9/4; top-1 = 9; nothing left masked -> every row locked
    ([1, 1, _, _, _, _, _, _, _, .2], [9], [1] * 10, (SLOW, 6, 0, 4, [8, 6, 9, 6])),
    # nothing masked: nothing changes
    ([1] * 10, [], [1] * 10, (SLOW, 6, 0, 4, [8, 6, 9, 6])),
]

# Example B (N = 6, K_max = 2): the switch forced by K_max despite a large
# variance, and a span that is already decoded at the switch (the cycle ends at once).
P_B = po.SpanParams(k=1, tau_conv=0.5, tau_high=0.8, var_stable=1.0, w_hist=2, k_max=2)
MASK_B = [1] * 6
STEPS_B = [
    ([.9, .1, .1, .1, .1, .7], [0], [0] * 6, (SLOW, 0, 0, 1, [5])),
    # e_t = 2; var(5,2) = 9/4 but K_max = 2 slow steps -> fast on [0,2]
    ([_, .1, .6, .1, .1, .1], [2], [0, 0, 0, 1, 1, 1], (FAST, 0, 2, 2, [5, 2])),
    ([_, .81, _, .1, .1, .1], [1], [0] * 6, (SLOW, 0, 0, 0, [])),
    # s = 3; nothing converged -> e_t = 3; top-1 = 4
    ([_, _, _, .2, .3, .1], [4], [0] * 6, (SLOW, 3, 0, 1, [3])),
    # e_t = 3; var(3,3) = 0 -> fast on [3,3], but 3 was just unmasked -> cycle ends
    ([_, _, _, .2, _, .1], [3], [0] * 6, (SLOW, 0, 0, 0, [])),
    # s = 5, last position; nothing left -> every row locked
    ([_, _, _, _, _, 0.], [5], [1] * 6, (SLOW, 5, 0, 1, [5])),
]

# Example D (N = 5, W_hist = 1): both thresholds are strict, and equal
# confidences go to the lower index.
P_D = po.SpanParams(k=1, tau_conv=0.5, tau_high=0.75, var_stable=1.0, w_hist=1, k_max=8)
MASK_D = [1] * 5
STEPS_D = [
    # converged: only 3 (0.5 is not > 0.5) -> e_t = 3; one end point -> variance 0 -> fast on [0,3]
    ([.25, .5, .5, .625, .5], [3], [0, 0, 0, 0, 1], (FAST, 0, 3, 1, [3])),
    # 0.75 is not > 0.75 -> fallback top-1 among {0,1,2}: 1 and 2 tie -> 1
    ([.25, .75, .75, _, .9], [1], [0, 0, 0, 0, 1], (FAST, 0, 3, 1, [3])),
    ([.25, _, .875, _, .9], [2], [0, 0, 0, 0, 1], (FAST, 0, 3, 1, [3])),
    ([.5, _, _, _, .9], [0], [0] * 5, (SLOW, 0, 0, 0, [])),
    # s = 4, e_t = 4, fast on [4,4] at once decoded -> cycle ends; nothing left -> all locked
    ([_, _, _, _, .9], [4], [1] * 5, (SLOW, 0, 0, 0, [])),
]

# Example E (N = 12): the variance is taken over the LAST W_hist end points.
P_E = po.SpanParams(k=1, tau_conv=0.5, tau_high=0.8, var_stable=1.0, w_hist=2, k_max=8)
MASK_E = [1] * 12
STEPS_E = [
    ([.2] + [.1] * 9 + [.9, .1], [10], [0] * 12, (SLOW, 0, 0, 1, [10])),
    ([.3] + [.1] * 9 + [_, .1], [0], [0] * 12, (SLOW, 0, 0, 2, [10, 0])),
    # e_t = 1; var(0,1) = 1/4 -> fast on [0,1], already decoded -> cycle ends
    ([_, .6] + [.1] * 8 + [_, .1], [1], [0] * 12, (SLOW, 0, 0, 0, [])),
]

# Example F (N = 8, W_hist = 3): the variance is the population variance.
P_F = po.SpanParams(k=1, tau_conv=0.5, tau_high=0.8, var_stable=1.0, w_hist=3, k_max=8)
MASK_F = [1] * 8
STEPS_F = [
    # nothing converged -> e_t = s = 0
    ([.2, .1, .1, .1, .1, .1, .1, .1], [0], [0] * 8, (SLOW, 0, 0, 1, [0])),
    ([_, .6, .1, .1, .1, .1, .1, .1], [1], [0] * 8, (SLOW, 0, 0, 2, [0, 1])),
    # e_t = 2; variance of (0,1,2) = 2/3 < 1 (the sample variance would be 1) -> fast
    # on [0,2], already decoded -> cycle ends
    ([_, _, .6, .1, .1, .1, .1, .1], [2], [0] * 8, (SLOW, 0, 0, 0, [])),
]

EXAMPLES = [(P_A, MASK_A, STEPS_A), (P_B, MASK_B, STEPS_B), (P_D, MASK_D, STEPS_D), (P_E, MASK_E, STEPS_E),
            (P_F, MASK_F, STEPS_F)]


@pytest.mark.parametrize("case", range(len(EXAMPLES)))
def test_hand_worked_trajectories(case):
    p, m0, steps = EXAMPLES[case]
    _run(po.slowfast_step_seq, p, len(m0), m0, steps)


def _plain_topk_sampler(conf, masked, k):
    """Unmask the k most confident masked positions: larger first, NaN last, ties to the lower index."""
    pend = np.flatnonzero(masked)
    c = conf[pend].astype(np.float64)
    nan = np.isnan(c)
    order = np.lexsort((pend, np.where(nan, 0.0, -c), nan))
    out = np.zeros_like(masked)
    out[pend[order[:k]]] = 1
    return out


def _reduction_to_topk_holds(fn):
    """With var_stable < 0 and K_max beyond reach, every step is a slow step."""
    for seed, k in ((1, 1), (2, 3), (3, 7)):
        B, N, prompt = 2, 96, 16
        p = po.SpanParams(k=k, tau_conv=0.5, tau_high=0.9, var_stable=-1.0, w_hist=2, k_max=10 ** 9)
        masked = synth.generation_mask(B, N, prompt)
        states = [po.SpanState() for _ in range(B)]
        for t in range(200):
            conf = synth.span_confidences(B, N, t, seed=seed, prompt=prompt, rate=3.0)
            conf[:, ::17] = np.nan  # NaN is never preferred
            for b in range(B):
                want = _plain_topk_sampler(conf[b], masked[b], k)
                m2, unmask, lock, states[b] = fn(conf[b], masked[b], states[b], p)
                if not np.array_equal(unmask, want):
                    return False
                if lock.tolist() != ([1] * N if not m2.any() else [0] * N):
                    return False
                masked[b] = m2
            if not masked.any():
                break
        if masked.any():
            return False
    return True


def test_reduces_to_topk_sampler_when_fast_phase_unreachable():
    assert _reduction_to_topk_holds(po.slowfast_step_seq)


def _one_step_spans_hold(fn):
    """W_hist = 1 switches after every slow step; tau_high = -inf decodes the whole span at once."""
    N, prompt = 80, 8
    p = po.SpanParams(k=2, tau_conv=0.5, tau_high=-math.inf, var_stable=1.0, w_hist=1, k_max=8)
    masked = synth.generation_mask(1, N, prompt)[0]
    st = po.SpanState()
    for t in range(100):
        conf = synth.span_confidences(1, N, t, seed=4, prompt=prompt, rate=5.0)[0]
        pend = np.flatnonzero(masked)
        if pend.size == 0:
            return True
        if st.phase == FAST:
            want = [i for i in pend if st.s <= i <= st.e]  # every masked position of the span
            masked, unmask, lock, st = fn(conf, masked, st, p)
            if sorted(np.flatnonzero(unmask).tolist()) != want or st.phase != SLOW or st.nslow != 0:
                return False
        else:
            s = int(pend[0])
            conv = [i for i in pend if conf[i] > np.float32(0.5)]
            e_t = max(conv) if conv else s
            masked, unmask, lock, st = fn(conf, masked, st, p)
            left = [i for i in np.flatnonzero(masked) if s <= i <= e_t]
            if left:  # switched to fast on [s, e_t]
                if (st.phase, st.s, st.e) != (FAST, s, e_t) or lock[s:e_t + 1].any() or \
                        lock.sum() != N - (e_t - s + 1):
                    return False
            elif st.phase != SLOW or st.nslow not in (0, 1):
                return False
    return False


def test_unit_window_and_open_threshold_decode_each_span_in_one_step():
    assert _one_step_spans_hold(po.slowfast_step_seq)


def test_population_variance_exact():
    rng = np.random.default_rng(5)
    for n in range(1, 9):
        v = [int(x) for x in rng.integers(0, 5000, size=n)]
        assert po.population_variance(v) == statistics.pvariance([Fraction(x) for x in v])
    for a in range(20):
        for b in range(20):
            assert po.population_variance([a, b]) == Fraction(a - b, 2) ** 2  # W = 2 closed form
    assert po.population_variance([7]) == 0


def _invariants_hold(fn, seed, p, B=3, N=120, prompt=20):
    masked = synth.generation_mask(B, N, prompt)
    states = [po.SpanState() for _ in range(B)]
    for t in range(N + 1):
        conf = synth.span_confidences(B, N, t, seed=seed, prompt=prompt, rate=6.0)
        for b in range(B):
            st0, m0 = states[b], masked[b].copy()
            m1, unmask, lock, st1 = fn(conf[b], m0, st0, p)
            pend = m0.astype(bool)
            if (unmask.astype(bool) & ~pend).any() or not np.array_equal(m1, m0 & (1 - unmask)):
                return False
            if pend.any() and not unmask.any():  # progress on every step
                return False
            if st0.phase == FAST and unmask.any():
                pos = np.flatnonzero(unmask)
                if pos.min() < st0.s or pos.max() > st0.e:  # fast steps stay inside the span
                    return False
            if st0.phase == SLOW and pend.any():
                if unmask.sum() != min(p.k, pend.sum()):
                    return False
            if st1.phase == FAST:
                if not (st1.s <= st1.e and m1[st1.s:st1.e + 1].any()):
                    return False
                if lock.tolist() != [0 if st1.s <= i <= st1.e else 1 for i in range(N)]:
                    return False
            elif lock.tolist() != ([1] * N if not m1.any() else [0] * N):
                return False
            if st1.nslow > p.k_max:
                return False
            masked[b], states[b] = m1, st1
        if not masked.any():
            return True
    return False  # must finish within N steps


@pytest.mark.parametrize("seed,k,w,kmax,var", [(0, 1, 2, 8, 1.0), (1, 2, 2, 8, 1.0), (2, 3, 3, 4, 4.0),
                                                 (3, 1, 1, 1, 0.0), (4, 4, 2, 8, 100.0)])
def test_invariants_on_random_trajectories(seed, k, w, kmax, var):
    p = po.SpanParams(k=k, tau_conv=0.6, tau_high=0.85, var_stable=var, w_hist=w, k_max=kmax)
    assert _invariants_hold(po.slowfast_step_seq, seed, p)


def test_infinite_variance_threshold():
    # +inf: every window is stable, so W_hist = 1 switches after each slow step;
    # -inf: no window is, so only K_max ends the slow phase
    conf = np.array([.9, .2, .7, .1], dtype=np.float32)
    for var, k_max, want in ((np.inf, 8, po.SF_FAST), (-np.inf, 8, po.SF_SLOW), (-np.inf, 1, po.SF_FAST)):
        p = po.SpanParams(k=1, tau_conv=0.5, var_stable=var, w_hist=1, k_max=k_max)
        st = po.slowfast_step_seq(conf, np.ones(4, np.uint8), po.SpanState(), p)[3]
        assert st.phase == want and (st.e == 2 if want == po.SF_FAST else True)


def test_invalid_state_reads_as_initial_and_inputs_untouched():
    conf = np.array([.9, .2, .7, .1], dtype=np.float32)
    masked = np.ones(4, dtype=np.uint8)
    p = po.SpanParams()
    ref = po.slowfast_step_seq(conf, masked, po.SpanState(), p)
    bad = po.SpanState(phase=5, s=3, e=1, nslow=2, hist=[9, 9])
    got = po.slowfast_step_seq(conf, masked, bad, p)
    for a, b in zip(ref[:3], got[:3]):
        assert np.array_equal(a, b)
    assert vars(ref[3]) == vars(got[3])
    assert masked.tolist() == [1, 1, 1, 1] and bad.phase == 5


# ---------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one plausible error must fail a pin
# ---------------------------------------------------------------------------
_MUTANTS = [
    ("slowfast_step_seq", "float(conf[i]) > p.tau_high", "float(conf[i]) >= p.tau_high"),
    ("slowfast_step_seq", "float(conf[i]) > p.tau_conv", "float(conf[i]) >= p.tau_conv"),
    ("slowfast_step_seq", "max(converged)", "min(converged)"),
    ("_below", "v < Fraction(x)", "v <= Fraction(x)"),
    ("slowfast_step_seq", "st.hist[-p.w_hist:]", "st.hist[:p.w_hist]"),
    ("slowfast_step_seq", "chosen = hot if hot else _most_confident(conf, cand, p.k)", "chosen = hot"),
    ("slowfast_step_seq", "st = SpanState()  # the span is decoded", "pass  #"),
    ("slowfast_step_seq", "st.nslow >= p.k_max", "st.nslow > p.k_max"),
    ("slowfast_step_seq", "if st.nslow == 0:\n            st.s", "if True:\n            st.s"),
    ("slowfast_step_seq", "0 if st.s <= i <= st.e else 1", "1 if st.s <= i <= st.e else 0"),
    ("slowfast_step_seq", "else st.s\n", "else pending[-1]\n"),
    ("_most_confident", "(0, -v, i)", "(0, -v, -i)"),
    ("_most_confident", "(1, 0.0, i) if", "(-1, 0.0, i) if"),
    ("population_variance", "/ n", "/ max(n - 1, 1)"),
]


def _mutated_policy(fname, old, new):
    ns = dict(po.__dict__)
    src = textwrap.dedent(inspect.getsource(getattr(po, fname)))
    assert src.count(old) == 1, old
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    if fname != "slowfast_step_seq":  # rebind the policy to the mutated helper
        exec(compile(textwrap.dedent(inspect.getsource(po.slowfast_step_seq)), "<policy>", "exec"), ns)
    return ns["slowfast_step_seq"]


def _all_pins_hold(fn):
    for p, m0, steps in EXAMPLES:
        try:
            _run(fn, p, len(m0), m0, steps)
        except AssertionError:
            return False
    if not _reduction_to_topk_holds(fn) or not _one_step_spans_hold(fn):
        return False
    p = po.SpanParams(k=2, tau_conv=0.6, tau_high=0.85, var_stable=1.0, w_hist=2, k_max=8)
    return _invariants_hold(fn, 0, p)


def test_pins_hold_for_the_oracle():
    assert _all_pins_hold(po.slowfast_step_seq)


@pytest.mark.parametrize("fname,old,new", _MUTANTS)
def test_planted_mistakes_are_caught(fname, old, new):
    assert not _all_pins_hold(_mutated_policy(fname, old, new))
