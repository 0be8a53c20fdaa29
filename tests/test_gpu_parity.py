"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer results (lock, idx, seg_ptr) must match bit-exactly when both sides get
the same scores; floating-point results use the tolerances of parity_util.
Every input is seeded synthetic data from `synth`; the oracle never sees a value
produced by the GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import (Guarded, assert_bf16_close, assert_f32_close, check_guards, dev, guarded_workspace,
                               host, metrics, tdtype, weights_dev)

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(scope="module")
def plk():
    import partial_recompute_kv_b200 as m
    return m


def pdims(plk, D):
    return plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16 if D.dtype == "bf16" else plk.F32,
                    getattr(D, "rope_theta", 0.0), getattr(D, "Hkv", 0))


def int_dev(a, n):
    t = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    if len(a):
        t[: len(a)] = torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()
    return t


_SEL_GUARDS = {}


def sel_bufs(B, N):
    gi = Guarded((B * N,), torch.int32, fill=-1)
    gs = Guarded((B + 1,), torch.int32, fill=-7)
    _SEL_GUARDS[gi.t.data_ptr()] = gi
    _SEL_GUARDS[gs.t.data_ptr()] = gs
    return gi.t, gs.t


def check_compaction(idx, seg, ref_lock):
    ref_idx, ref_seg = oracle.compact(ref_lock)
    assert np.array_equal(host(seg), ref_seg)
    M = int(ref_seg[-1])
    hi = host(idx)
    assert np.array_equal(hi[:M], ref_idx)
    assert np.all(hi[M:] == -1), "nothing past M is written"
    for t, name in ((idx, "idx"), (seg, "seg_ptr")):  # and nothing outside the buffers
        g = _SEL_GUARDS.get(t.data_ptr())
        if g is not None:
            g.check(name)


# ---------------------------------------------------------------------------
# S2/S3 select + compaction: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,N", [(1, 1), (3, 1000), (2, 3000)])
@pytest.mark.parametrize("gt", [True, False])
@pytest.mark.parametrize("inplace", [False, True])
def test_select_threshold_bitexact(plk, B, N, gt, inplace):
    rng = np.random.default_rng(100 + N)
    s = rng.random((B, N)).astype(np.float32)
    s[rng.random((B, N)) < 0.02] = np.nan
    s[0, 0] = 0.5  # exactly tau: strict comparison never locks it
    lock = (rng.random((B, N)) < 0.3).astype(np.uint8)
    tau = np.float32(0.5)
    ref = oracle.lock_threshold(s.astype(np.float64), lock, float(tau), greater=gt)
    dm = plk.dims(B, N, 64, 4, 16, 64, dtype=plk.F32)
    score = dev(s, torch.float32)
    glin = Guarded((B, N), torch.uint8, init=lock)
    lin = glin.t
    glout = glin if inplace else Guarded((B, N), torch.uint8, fill=9)
    lout = glout.t
    idx, seg = sel_bufs(B, N)
    plk.select_active(dm, score, lin, lout, plk.SEL_THRESH_GT if gt else plk.SEL_THRESH_LT, float(tau), 0,
                      idx, seg)
    torch.cuda.synchronize()
    assert np.array_equal(host(lout), ref)
    check_compaction(idx, seg, ref)
    check_guards({"lock_in": glin, "lock_out": glout}, "threshold select")


# N <= 256: one CTA per sequence; larger N: a cluster of up to 8 CTAs per sequence (up to 4096 rows
# each; (1, 40000) is past that and goes back to one CTA)
@pytest.mark.parametrize("B,N", [(1, 5), (2, 777), (8, 4096), (1, 1024), (1, 8192), (1, 32000), (3, 40000)])
@pytest.mark.parametrize("kind", ["random", "ties", "nan"])
@pytest.mark.parametrize("largest", [True, False])
def test_select_topk_bitexact(plk, B, N, kind, largest):
    rng = np.random.default_rng(200 + N)
    if kind == "ties":
        s = rng.integers(-2, 3, (B, N)).astype(np.float32)
        z = s == 0
        s[z & (rng.random((B, N)) < 0.5)] = -0.0
    else:
        s = rng.standard_normal((B, N)).astype(np.float32)
        if kind == "nan":
            s[rng.random((B, N)) < 0.05] = np.nan
    lock = (rng.random((B, N)) < 0.2).astype(np.uint8)
    dm = plk.dims(B, N, 64, 4, 16, 64, dtype=plk.F32)
    score, lin = dev(s, torch.float32), dev(lock, torch.uint8)
    for k in sorted({0, 1, max(N // 10, 1), N // 2, N, N + 5}):
        ref = oracle.lock_topk(s.astype(np.float64), lock, k, largest)
        glout = Guarded((B, N), torch.uint8, fill=9)
        lout = glout.t
        idx, seg = sel_bufs(B, N)
        plk.select_active(dm, score, lin, lout, plk.SEL_TOPK_LARGEST if largest else plk.SEL_TOPK_SMALLEST,
                          0.0, k, idx, seg)
        torch.cuda.synchronize()
        assert np.array_equal(host(lout), ref), f"k={k}"
        check_compaction(idx, seg, ref)
        glout.check(f"top-k select k={k}: lock_out")


# ---------------------------------------------------------------------------
# S1 score_drift and S10 proxy commit
# ---------------------------------------------------------------------------
def _score_case(dtype):
    if dtype == "f32":
        return synth.Dims(B=2, N=100, d=64, H=4, hd=16, F=64, dtype="f32"), 8
    return synth.Dims(B=2, N=300, d=512, H=4, hd=128, F=512, dtype="bf16"), 128


@pytest.mark.parametrize("dtype,rank", [("f32", None), ("bf16", None), ("bf16", 16), ("bf16", 48), ("bf16", 256)])
@pytest.mark.parametrize("metric", ["cos", "l2"])
def test_score_drift(plk, dtype, rank, metric):
    """Ranks 16 and 48 (row blocks whose 16-byte chunk count is not a multiple of 8) run the
    K split over a cluster of 4 at d = 1024; rank 256 runs unsplit."""
    D, r = _score_case(dtype)
    if rank is not None:
        D, r = synth.Dims(B=2, N=300, d=1024, H=8, hd=128, F=512, dtype="bf16"), rank
    X = synth.hidden_states(D, seed=3)
    Ut = synth.proxy_basis(D.d, r, seed=3, dtype=dtype)
    p_exact = oracle.proxy_project(X.reshape(-1, D.d).astype(np.float64), Ut.astype(np.float64))
    rng = np.random.default_rng(3)
    moved = rng.random(D.B * D.N) < 0.3
    pc = p_exact + moved[:, None] * rng.standard_normal(p_exact.shape) * 0.5
    pc = pc.astype(np.float32).reshape(D.B, D.N, r)
    ref_s, ref_p = oracle.score_drift(X.astype(np.float64), Ut.astype(np.float64), pc, metric)
    dm = pdims(plk, D)
    gs = Guarded((D.B, D.N), torch.float32)
    gp = Guarded((D.B, D.N, r), torch.float32)
    score, pout = gs.t, gp.t
    plk.score_drift(dm, dev(X, tdtype(D)), dev(Ut, tdtype(D)), r, dev(pc, torch.float32),
                    plk.METRIC_COS if metric == "cos" else plk.METRIC_L2, score, proxy_out=pout)
    torch.cuda.synchronize()
    assert_f32_close(host(pout), ref_p, "proxy", tol=1e-5)
    assert_f32_close(host(score), ref_s, "score", tol=1e-4)
    check_guards({"score": gs, "proxy_out": gp}, "score_drift")


def test_score_drift_8b_shape_repeated(plk):
    """The scoring launch the benchmark times (1024 rows x 4096, rank 128, K split over a
    cluster of 8 CTAs), run several times on the same inputs: every run must match."""
    D = synth.Dims(B=1, N=1024, d=4096, H=32, hd=128, F=12288, dtype="bf16")
    r = 128
    X = synth.hidden_states(D, seed=5)
    Ut = synth.proxy_basis(D.d, r, seed=5, dtype="bf16")
    p_exact = oracle.proxy_project(X.reshape(-1, D.d).astype(np.float64), Ut.astype(np.float64))
    rng = np.random.default_rng(5)
    pc = (p_exact + (rng.random(D.N) < 0.25)[:, None] * rng.standard_normal(p_exact.shape) * 0.5)
    pc = pc.astype(np.float32).reshape(D.B, D.N, r)
    ref_s, ref_p = oracle.score_drift(X.astype(np.float64), Ut.astype(np.float64), pc, "l2")
    dm = pdims(plk, D)
    Xd, Ud, pcd = dev(X, torch.bfloat16), dev(Ut, torch.bfloat16), dev(pc, torch.float32)
    for run in range(6):
        score = torch.full((D.B, D.N), float("nan"), dtype=torch.float32, device="cuda")
        pout = torch.full((D.B, D.N, r), float("nan"), dtype=torch.float32, device="cuda")
        plk.score_drift(dm, Xd, Ud, r, pcd, plk.METRIC_L2, score, proxy_out=pout)
        torch.cuda.synchronize()
        assert_f32_close(host(pout), ref_p, f"proxy, run {run}", tol=1e-5)
        assert_f32_close(host(score), ref_s, f"score, run {run}", tol=1e-4)


@pytest.mark.parametrize("rank,metric", [(128, "l2"), (256, "cos"), (16, "cos")])
def test_score_drift_more_tiles_than_sms(plk, rank, metric):
    """21000 rows at d = 1024: 165 row tiles (the last one ragged) against 148 SMs, so the
    launch runs unsplit with two CTAs per SM and a shallower stage ring (3 stages at rank 128,
    2 at rank 256; rank 16 keeps its full ring).  Every row against the oracle."""
    D, r = synth.Dims(B=3, N=7000, d=1024, H=8, hd=128, F=512, dtype="bf16"), rank
    X = synth.hidden_states(D, seed=7)
    Ut = synth.proxy_basis(D.d, r, seed=7)
    p_exact = oracle.proxy_project(X.reshape(-1, D.d).astype(np.float64), Ut.astype(np.float64))
    rng = np.random.default_rng(7)
    pc = p_exact + (rng.random(D.B * D.N) < 0.3)[:, None] * rng.standard_normal(p_exact.shape) * 0.5
    pc = pc.astype(np.float32).reshape(D.B, D.N, r)
    ref_s, ref_p = oracle.score_drift(X.astype(np.float64), Ut.astype(np.float64), pc, metric)
    gs = Guarded((D.B, D.N), torch.float32)
    gp = Guarded((D.B, D.N, r), torch.float32)
    plk.score_drift(pdims(plk, D), dev(X, BF), dev(Ut, BF), r, dev(pc, torch.float32),
                    plk.METRIC_COS if metric == "cos" else plk.METRIC_L2, gs.t, proxy_out=gp.t)
    torch.cuda.synchronize()
    assert_f32_close(host(gp.t), ref_p, "proxy", tol=1e-5)
    assert_f32_close(host(gs.t), ref_s, "score", tol=1e-4)
    check_guards({"score": gs, "proxy_out": gp}, "score_drift")


def test_score_drift_scoring_shape_sampled(plk):
    """The scoring launch at its full size (8 sequences x 4096 rows x 4096, rank 128, L2 drift:
    256 row tiles, two CTAs per SM), checked against the oracle on 1024 sampled rows plus the
    first and last row of every sequence; every score finite.  Both outputs are fp32 and take the
    fp32 bound (1e-4): over 4096 bf16 products the tensor cores' fp32 accumulation reaches ~1.6e-5
    of the proxies' rms on some of these rows."""
    D, r = synth.SCORE_8B, synth.PROXY_RANK_8B
    X = synth.hidden_states(D, seed=6).reshape(-1, D.d)
    Ut = synth.proxy_basis(D.d, r, seed=6)
    rng = np.random.default_rng(6)
    pc = rng.standard_normal((D.B * D.N, r)).astype(np.float32)
    rows = np.unique(np.concatenate([rng.choice(D.B * D.N, 1024, replace=False),
                                     np.arange(0, D.B * D.N, D.N), np.arange(D.N - 1, D.B * D.N, D.N)]))
    ref_s, ref_p = oracle.score_drift(X[rows][None].astype(np.float64), Ut.astype(np.float64), pc[rows][None], "l2")
    score = torch.full((D.B, D.N), float("nan"), dtype=torch.float32, device="cuda")
    pout = torch.full((D.B, D.N, r), float("nan"), dtype=torch.float32, device="cuda")
    Xd = dev(X, BF)
    del X
    plk.score_drift(pdims(plk, D), Xd, dev(Ut, BF), r, dev(pc, torch.float32), plk.METRIC_L2, score, proxy_out=pout)
    torch.cuda.synchronize()
    s_all = host(score).reshape(-1)
    assert np.all(np.isfinite(s_all)), "score: non-finite values"
    assert_f32_close(s_all[rows], ref_s[0], "score (sampled rows)", tol=1e-4)
    assert_f32_close(host(pout).reshape(-1, r)[rows], ref_p[0], "proxy (sampled rows)")


def test_proxy_commit(plk):
    B, N, r = 3, 50, 16
    rng = np.random.default_rng(4)
    pc = rng.standard_normal((B, N, r)).astype(np.float32)
    pn = rng.standard_normal((B, N, r)).astype(np.float32)
    lock = (rng.random((B, N)) < 0.6).astype(np.uint8)
    idx, seg = oracle.compact(lock)
    ref = oracle.proxy_commit(pc, pn, idx)
    dm = plk.dims(B, N, 64, 4, 16, 64, dtype=plk.F32)
    gpc = Guarded((B, N, r), torch.float32, init=pc)
    plk.proxy_commit(dm, r, int_dev(idx, B * N), int_dev(seg, B + 1), dev(pn, torch.float32), gpc.t)
    torch.cuda.synchronize()
    assert np.array_equal(host(gpc.t), ref)
    gpc.check("proxy_commit: proxy_cache")


# ---------------------------------------------------------------------------
# S4..S10 layer steps, bf16
# ---------------------------------------------------------------------------
SMALL = synth.Dims(B=2, N=320, d=512, H=4, hd=128, F=1536, dtype="bf16")


def _run_layer_guarded(plk, D, Wd, X, idx, seg, st, dt=BF, what="layer step"):
    """plk_layer_step_partial with the caches, the active set and the workspace inside guard bands;
    returns the caches (host, float64) after checking that no guard byte changed."""
    dm = pdims(plk, D)
    g = {"K": Guarded(st.K.shape, dt, init=dev(st.K, dt)), "V": Guarded(st.V.shape, dt, init=dev(st.V, dt)),
         "Y": Guarded(st.Y.shape, dt, init=dev(st.Y, dt)),
         "idx": Guarded((D.B * D.N,), torch.int32, init=int_dev(idx, D.B * D.N)),
         "seg_ptr": Guarded((D.B + 1,), torch.int32, init=int_dev(seg, D.B + 1)),
         "workspace": guarded_workspace(plk, dm)}
    plk.layer_step_partial(dm, Wd, dev(X, dt), g["idx"].t, g["seg_ptr"].t, g["K"].t, g["V"].t, g["Y"].t,
                           g["workspace"].t)
    assert plk.get_status() == plk.OK
    check_guards(g, what)
    return host(g["K"].t), host(g["V"].t), host(g["Y"].t)


def _run_full_guarded(plk, D, Wd, X, dt=BF, what="full step"):
    dm = pdims(plk, D)
    g = {"K": Guarded((D.B, D.N, D.dkv), dt, fill=0), "V": Guarded((D.B, D.N, D.dkv), dt, fill=0),
         "Y": Guarded((D.B, D.N, D.d), dt, fill=0), "workspace": guarded_workspace(plk, dm)}
    plk.full_layer_step(dm, Wd, dev(X, dt), g["K"].t, g["V"].t, g["Y"].t, g["workspace"].t)
    assert plk.get_status() == plk.OK
    check_guards(g, what)
    return host(g["K"].t), host(g["V"].t), host(g["Y"].t)


def _run_partial(plk, D, W, X, idx, seg, st):
    return _run_layer_guarded(plk, D, weights_dev(W, D), X, idx, seg, st)


def test_full_layer_step_bf16(plk):
    D = SMALL
    W = synth.layer_weights(D, 0.02, seed=1)
    X = synth.hidden_states(D, seed=1)
    ref = oracle.full_layer_step(D, W, X, "bf16")
    K, V, Y = _run_full_guarded(plk, D, weights_dev(W, D), X)
    assert_bf16_close(K, ref.K, "K")
    assert_bf16_close(V, ref.V, "V")
    assert_bf16_close(Y, ref.Y, "Y")


@pytest.mark.parametrize("p_active", [0.05, 0.3, 1.0])
def test_partial_step_bf16(plk, p_active):
    D = SMALL
    W = synth.layer_weights(D, 0.02, seed=2)
    X = synth.hidden_states(D, seed=2)
    base = oracle.full_layer_step(D, W, X, "bf16")
    lock = synth.bernoulli_active(D.B, D.N, p_active, seed=7)
    if p_active == 1.0:
        lock[:] = 0
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=7), lock == 0, "bf16")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    K, V, Y = _run_partial(plk, D, W, X2, idx, seg, base)
    locked = lock.astype(bool)
    for g, o0, name in ((K, base.K, "K"), (V, base.V, "V"), (Y, base.Y, "Y")):
        assert np.array_equal(g[locked], o0[locked]), f"{name}: a locked row was written"
    act = ~locked
    assert_bf16_close(K[act], ref.K[act], "K active")
    assert_bf16_close(V[act], ref.V[act], "V active")
    assert_bf16_close(Y[act], ref.Y[act], "Y active")


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_layer_bf16(plk, theta):
    """RoPE variant: full step, then a partial step on perturbed active rows (positions up to
    N - 1 = 319 in each of two sequences)."""
    D = synth.Dims(**{**SMALL.__dict__, "rope_theta": theta})
    W = synth.layer_weights(D, 0.02, seed=8)
    X = synth.hidden_states(D, seed=8)
    base = oracle.full_layer_step(D, W, X, "bf16")
    dm = pdims(plk, D)
    K = torch.zeros((D.B, D.N, D.d), dtype=BF, device="cuda")
    V, Y = torch.zeros_like(K), torch.zeros_like(K)
    plk.full_layer_step(dm, weights_dev(W, D), dev(X, BF), K, V, Y, plk.alloc_workspace(dm))
    assert plk.get_status() == plk.OK
    assert_bf16_close(host(K), base.K, "K full")
    assert_bf16_close(host(Y), base.Y, "Y full")
    lock = synth.bernoulli_active(D.B, D.N, 0.3, seed=8)
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=8), lock == 0, "bf16")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    K, V, Y = _run_partial(plk, D, W, X2, idx, seg, base)
    locked = lock.astype(bool)
    assert np.array_equal(K[locked], base.K[locked]) and np.array_equal(Y[locked], base.Y[locked])
    act = ~locked
    assert_bf16_close(K[act], ref.K[act], "K active")
    assert_bf16_close(Y[act], ref.Y[act], "Y active")


def test_rope_layer_fp32(plk):
    D = synth.Dims(B=2, N=100, d=64, H=4, hd=16, F=64, eps=1e-6, dtype="f32", rope_theta=10000.0)
    W = synth.layer_weights(D, 1.0 / math.sqrt(D.d), seed=9)
    X = synth.hidden_states(D, seed=9)
    base = oracle.full_layer_step(D, W, X, "f64")
    lock = synth.bernoulli_active(D.B, D.N, 0.4, seed=9)
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=9), lock == 0, "f32")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "f64")
    dm = pdims(plk, D)
    K, V, Y = (dev(a, torch.float32) for a in (base.K, base.V, base.Y))
    plk.layer_step_partial(dm, weights_dev(W, D), dev(X2, torch.float32), int_dev(idx, D.B * D.N),
                           int_dev(seg, D.B + 1), K, V, Y, plk.alloc_workspace(dm))
    assert plk.get_status() == plk.OK
    act = lock == 0
    assert_f32_close(host(K)[act], ref.K[act], "K active")
    assert_f32_close(host(Y)[act], ref.Y[act], "Y active")


@pytest.mark.parametrize("shape", [dict(Hkv=1), dict(Hkv=2), dict(Hkv=2, rope_theta=10000.0),
                                   dict(B=1, N=640, d=1024, H=8, F=1024, Hkv=2)])
def test_gqa_layer_bf16(plk, shape):
    """Grouped-query variant (fewer K/V heads than query heads; K/V caches Hkv*hd wide): full
    step, then a partial step on perturbed active rows."""
    D = synth.Dims(**{**SMALL.__dict__, **shape})
    W = synth.layer_weights(D, 0.02, seed=12)
    X = synth.hidden_states(D, seed=12)
    base = oracle.full_layer_step(D, W, X, "bf16")
    dm = pdims(plk, D)
    K = torch.zeros((D.B, D.N, D.dkv), dtype=BF, device="cuda")
    V = torch.zeros_like(K)
    Y = torch.zeros((D.B, D.N, D.d), dtype=BF, device="cuda")
    plk.full_layer_step(dm, weights_dev(W, D), dev(X, BF), K, V, Y, plk.alloc_workspace(dm))
    assert plk.get_status() == plk.OK
    assert_bf16_close(host(K), base.K, "K full")
    assert_bf16_close(host(V), base.V, "V full")
    assert_bf16_close(host(Y), base.Y, "Y full")
    lock = synth.bernoulli_active(D.B, D.N, 0.3, seed=12)
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=12), lock == 0, "bf16")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    K, V, Y = _run_partial(plk, D, W, X2, idx, seg, base)
    locked = lock.astype(bool)
    for g, o0, name in ((K, base.K, "K"), (V, base.V, "V"), (Y, base.Y, "Y")):
        assert np.array_equal(g[locked], o0[locked]), f"{name}: a locked row was written"
    act = ~locked
    assert_bf16_close(K[act], ref.K[act], "K active")
    assert_bf16_close(V[act], ref.V[act], "V active")
    assert_bf16_close(Y[act], ref.Y[act], "Y active")


@pytest.mark.parametrize("Hkv,theta", [(1, 0.0), (2, 10000.0)])
def test_gqa_layer_fp32(plk, Hkv, theta):
    D = synth.Dims(B=2, N=100, d=64, H=4, hd=16, F=64, eps=1e-6, dtype="f32", rope_theta=theta, Hkv=Hkv)
    W = synth.layer_weights(D, 1.0 / math.sqrt(D.d), seed=13)
    X = synth.hidden_states(D, seed=13)
    base = oracle.full_layer_step(D, W, X, "f64")
    lock = synth.bernoulli_active(D.B, D.N, 0.4, seed=13)
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=13), lock == 0, "f32")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "f64")
    dm = pdims(plk, D)
    K, V, Y = (dev(a, torch.float32) for a in (base.K, base.V, base.Y))
    assert K.shape == (D.B, D.N, Hkv * D.hd)
    plk.layer_step_partial(dm, weights_dev(W, D), dev(X2, torch.float32), int_dev(idx, D.B * D.N),
                           int_dev(seg, D.B + 1), K, V, Y, plk.alloc_workspace(dm))
    assert plk.get_status() == plk.OK
    act = lock == 0
    assert np.array_equal(host(K)[~act], base.K.astype(np.float32)[~act])  # locked rows: the uploaded values
    assert_f32_close(host(K)[act], ref.K[act], "K active")
    assert_f32_close(host(V)[act], ref.V[act], "V active")
    assert_f32_close(host(Y)[act], ref.Y[act], "Y active")


def test_partial_step_m_zero_is_noop(plk):
    D = SMALL
    W = synth.layer_weights(D, 0.02, seed=3)
    X = synth.hidden_states(D, seed=3)
    rng = np.random.default_rng(3)
    st = oracle.LayerState(*(synth.round_bf16(rng.standard_normal((D.B, D.N, D.d)).astype(np.float32))
                             .astype(np.float64) for _ in range(3)))
    idx, seg = oracle.compact(np.ones((D.B, D.N), np.uint8))
    K, V, Y = _run_partial(plk, D, W, X, idx, seg, st)
    assert np.array_equal(K, st.K) and np.array_equal(V, st.V) and np.array_equal(Y, st.Y)


def test_workspace_too_small_is_rejected(plk):
    D = SMALL
    dm = pdims(plk, D)
    W = weights_dev(synth.layer_weights(D, 0.02), D)
    X = torch.zeros((D.B, D.N, D.d), dtype=BF, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(plk.PlkError) as e:
        plk.full_layer_step(dm, W, X, X.clone(), X.clone(), X.clone(), small)
    assert e.value.code == plk.ERR_WORKSPACE
    # large enough but not on a 256-byte boundary: refused as well, nothing enqueued
    n = plk.workspace_bytes(dm)
    raw = torch.empty(n + 256, dtype=torch.uint8, device="cuda")
    for off in (16, 128):
        with pytest.raises(plk.PlkError) as e:
            plk.full_layer_step(dm, W, X, X.clone(), X.clone(), X.clone(), raw[off:off + n])
        assert e.value.code == plk.ERR_WORKSPACE, off
    torch.cuda.synchronize()
    assert plk.get_status() == plk.OK


# ---------------------------------------------------------------------------
# the tiny fp32 workload: 20 denoising steps, every step checked
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("noise_var", [synth.TINY_NOISE_VAR, 0.1])
@pytest.mark.parametrize("entry", ["calls", "step", "steps"])
def test_tiny_fp32_driver(plk, noise_var, entry):
    """The tiny fp32 workload step by step.  With its own noise (variance 0.01) the active set
    empties within four steps; with variance 0.1 it shrinks from 13 rows to 1 over the 20 steps,
    so the fp32 layer runs on several rows at every step (decision margins >= 2e-4 from tau).
    entry "calls": the four API calls of a step; "step": one plk_denoise_step per step; "steps":
    all 20 steps in one plk_denoise_steps_host call from host buffers (the inputs built up front
    from the oracle's locks, which the other entries match bit for bit), every step's Y
    checked."""
    D = synth.TINY
    r = synth.TINY_RANK
    W = synth.layer_weights(D, 1.0 / math.sqrt(D.d))
    X0 = synth.hidden_states(D)
    Ut = synth.proxy_basis(D.d, r, dtype="f32")
    lock0 = synth.bernoulli_active(D.B, D.N, synth.TINY_P_ACTIVE)
    noises = [synth.step_noise((D.B, D.N, D.d), noise_var, step=t) for t in range(synth.TINY_STEPS)]
    perturb = lambda X, e, m: synth.perturb_rows(X, e, m, "f32")
    recs = oracle.tiny_run(D, W, X0, Ut.astype(np.float64), lock0, noises, synth.TINY_TAU, perturb)

    dm = pdims(plk, D)
    f32 = torch.float32
    Wd = weights_dev(W, D)
    Utd = dev(Ut, f32)
    K = torch.zeros((D.B, D.N, D.d), dtype=f32, device="cuda")
    V, Y = torch.zeros_like(K), torch.zeros_like(K)
    ws = plk.alloc_workspace(dm)
    plk.full_layer_step(dm, Wd, dev(X0, f32), K, V, Y, ws)
    score = torch.empty((D.B, D.N), dtype=f32, device="cuda")
    pnew = torch.empty((D.B, D.N, r), dtype=f32, device="cuda")
    pc = torch.zeros_like(pnew)
    plk.score_drift(dm, dev(X0, f32), Utd, r, pc, plk.METRIC_L2, score, proxy_out=pnew)
    pc.copy_(pnew)
    lock = dev(lock0, torch.uint8)
    idx, seg = sel_bufs(D.B, D.N)
    sws = plk.alloc_step_workspace(dm, r) if entry == "step" else None
    X = X0.copy()
    if entry == "steps":
        X_hosts, act = [], lock0 == 0
        for t, eps in enumerate(noises):
            X = perturb(X, eps, act)
            X_hosts.append(torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).pin_memory())
            act = recs[t]["lock"] == 0
        Y_hosts = [torch.full((D.B, D.N, D.d), float("nan"), dtype=f32).pin_memory() for _ in noises]
        gws = Guarded((plk.steps_workspace_bytes(dm, r),), torch.uint8)
        plk.denoise_steps_host(dm, Wd, Utd, r, plk.METRIC_COS, plk.SEL_THRESH_GT, synth.TINY_TAU, 0, pc, lock, K, V,
                               Y, X_hosts, Y_hosts, gws.t, torch.cuda.Stream(), torch.cuda.Stream())
        torch.cuda.current_stream().synchronize()
        assert plk.get_status() == plk.OK
        gws.check("denoise_steps_host: workspace")
        for t, rec in enumerate(recs):
            assert_f32_close(Y_hosts[t].numpy().astype(np.float64), rec["Y"], f"step {t}: Y_hosts")
        rec = recs[-1]
        assert np.array_equal(host(lock), rec["lock"]), "lock after the last step"
        for name, g in (("K", K), ("V", V), ("Y", Y), ("proxy", pc)):
            assert_f32_close(host(g), rec[name], f"last step: {name}")
        return
    for t, eps in enumerate(noises):
        X = perturb(X, eps, host(lock) == 0)
        Xd = dev(X, f32)
        if entry == "calls":
            plk.score_drift(dm, Xd, Utd, r, pc, plk.METRIC_COS, score, proxy_out=pnew)
            plk.select_active(dm, score, lock, lock, plk.SEL_THRESH_GT, synth.TINY_TAU, 0, idx, seg)
            plk.layer_step_partial(dm, Wd, Xd, idx, seg, K, V, Y, ws)
            plk.proxy_commit(dm, r, idx, seg, pnew, pc)
        else:
            plk.denoise_step(dm, Wd, Utd, r, plk.METRIC_COS, plk.SEL_THRESH_GT, synth.TINY_TAU, 0, pc, lock, K, V,
                             Y, Xd, sws)
        assert plk.get_status() == plk.OK
        rec = recs[t]
        assert np.array_equal(host(lock), rec["lock"]), f"step {t}: lock"
        if entry == "calls":
            M = int(rec["seg_ptr"][-1])
            assert np.array_equal(host(seg), rec["seg_ptr"]) and np.array_equal(host(idx)[:M], rec["idx"])
            assert_f32_close(host(score), rec["score"], f"step {t}: score")
        for name, g in (("K", K), ("V", V), ("Y", Y), ("proxy", pc)):
            assert_f32_close(host(g), rec[name], f"step {t}: {name}")


# ---------------------------------------------------------------------------
# the 8B-shape layer (d=4096, 32 x 128 heads, F=12288, N=1024) across the active
# fractions 1, 1/2, 1/4 (the benchmarked launch), 1/10, 1/20: every active row
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def layer_8b(plk):
    D = synth.LAYER_8B
    W = synth.layer_weights(D, synth.LAYER_8B_WSTD)
    X = synth.hidden_states(D)
    base = oracle.full_layer_step(D, W, X, "bf16")
    return dict(D=D, W=W, X=X, base=base, Wd=weights_dev(W, D))


def _check_layer_rows(K, V, Y, ref, base, lock, what):
    locked = lock.astype(bool)
    for g, o0, name in ((K, base.K, "K"), (V, base.V, "V"), (Y, base.Y, "Y")):
        assert np.array_equal(g[locked], o0[locked]), f"{what} {name}: a locked row was written"
    act = ~locked
    out = {}
    for g, o, name in ((K, ref.K, "K"), (V, ref.V, "V"), (Y, ref.Y, "Y")):
        out[name] = assert_bf16_close(g[act], o[act], f"{what} {name}")
    return out


def test_layer_8b_full_step(plk, layer_8b):
    """The full-recompute baseline at the 8B shape: every row of K, V and Y."""
    D, base = layer_8b["D"], layer_8b["base"]
    K, V, Y = _run_full_guarded(plk, D, layer_8b["Wd"], layer_8b["X"], what="8B full step")
    for g, o, name in ((K, base.K, "K"), (V, base.V, "V"), (Y, base.Y, "Y")):
        assert_bf16_close(g, o, f"8B full step {name}")


@pytest.mark.parametrize("frac", [0.25, 0.05])
def test_layer_8b_kv_are_deterministic(plk, layer_8b, frac):
    """The QKV projection lands the pieces of a split tile in a fixed order (at M = 256 its tiles
    split over 2-3 CTA pairs): identical calls give bit-identical K and V.  The O and down
    projections add their pieces into the residual stream in arrival order, so Y agrees up to the
    last bits."""
    D, base = layer_8b["D"], layer_8b["base"]
    pos = synth.layer_8b_positions(D.N, frac)
    lock = np.ones((1, D.N), np.uint8)
    lock[0, pos] = 0
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(layer_8b["X"], synth.step_noise((1, D.N, D.d), 0.01), lock == 0, "bf16")
    runs = [_run_layer_guarded(plk, D, layer_8b["Wd"], X2, idx, seg, base, what=f"8B M/N={frac} run {i}")
            for i in range(3)]
    for r in runs[1:]:
        for a, b, name in zip(runs[0][:2], r[:2], "KV"):
            assert np.array_equal(a, b), f"8B M/N={frac}: {name} differs between identical calls"
        assert_bf16_close(r[2], runs[0][2], f"8B M/N={frac}: Y of identical calls")


def test_layer_8b_reproducible_mode(plk, layer_8b):
    """plk_set_deterministic(1): the O and down projections land their split-tile pieces in a
    fixed order too, so identical calls give bit-identical K, V and Y; the outputs still meet the
    oracle."""
    D, W, base = layer_8b["D"], layer_8b["W"], layer_8b["base"]
    pos = synth.layer_8b_positions(D.N, 0.25)
    lock = np.ones((1, D.N), np.uint8)
    lock[0, pos] = 0
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(layer_8b["X"], synth.step_noise((1, D.N, D.d), 0.01), lock == 0, "bf16")
    plk.set_deterministic(True)
    try:
        runs = [_run_layer_guarded(plk, D, layer_8b["Wd"], X2, idx, seg, base, what=f"8B reproducible run {i}")
                for i in range(3)]
    finally:
        plk.set_deterministic(False)
    for r in runs[1:]:
        for a, b, name in zip(runs[0], r, "KVY"):
            assert np.array_equal(a, b), f"reproducible mode: {name} differs between identical calls"
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    _check_layer_rows(*runs[0], ref, base, lock, "8B reproducible mode")


@pytest.mark.parametrize("frac", synth.LAYER_8B_FRACTIONS)
def test_layer_8b_fraction(plk, layer_8b, frac, record_property):
    """Partial step from the full step's caches with the active rows perturbed: all M active rows of
    K, V and Y against the oracle (mean absolute error in the tensors' own units), locked rows
    bit-identical.  At M/N = 1/4 the distance to the oracle that rounds nothing is reported too."""
    D, W, base = layer_8b["D"], layer_8b["W"], layer_8b["base"]
    pos = synth.layer_8b_positions(D.N, frac)
    lock = np.ones((1, D.N), np.uint8)
    lock[0, pos] = 0
    idx, seg = oracle.compact(lock)
    assert idx.size == synth.active_count(D.N, frac)
    X2 = synth.perturb_rows(layer_8b["X"], synth.step_noise((1, D.N, D.d), 0.01), lock == 0, "bf16")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    K, V, Y = _run_layer_guarded(plk, D, layer_8b["Wd"], X2, idx, seg, base, what=f"8B M/N={frac}")
    res = _check_layer_rows(K, V, Y, ref, base, lock, f"8B M/N={frac}")
    for name, (mr, mae) in res.items():
        record_property(f"{name}_max_rel", mr)
        record_property(f"{name}_mae", mae)
    if frac == 0.25:
        # diagnostic: the same step with nothing rounded (outputs left in float64)
        f64 = oracle.layer_step_partial(D, W, X2, idx, seg, base, "f64")
        act = lock == 0
        for g, o, name in ((K, f64.K, "K"), (V, f64.V, "V"), (Y, f64.Y, "Y")):
            mr, mae, mrel = metrics(g[act], o[act])
            record_property(f"{name}_mae_vs_unrounded", mae)
            print(f"8B M/N=1/4 {name}: vs bf16-stored oracle mae {res[name][1]:.3e}; "
                  f"vs unrounded oracle mae {mae:.3e} (mae/rms {mrel:.3e}, max_rel {mr:.3e})")


# ---------------------------------------------------------------------------
# the 32-layer stack's last step (t = 255: 102 active rows in each of 4 sequences of
# 2048) and a long-context block (N = 8192, M = 76), both at the full 8B width
# ---------------------------------------------------------------------------
def _cache_state(shape, seed):
    rng = np.random.default_rng(seed)
    return oracle.LayerState(*(synth.round_bf16(rng.standard_normal(shape).astype(np.float32)).astype(np.float64)
                               for _ in range(3)))


def test_layer_8b_stack_last_step(plk):
    D = synth.STACK_8B
    W = synth.layer_weights(D, 0.02, seed=0, layer=3)
    X = synth.hidden_states(D, seed=31)
    st = _cache_state((D.B, D.N, D.d), 31)
    Mt = int(synth.linear_schedule(D.N)[255])
    assert Mt == 102
    lock = np.ones((D.B, D.N), np.uint8)
    rng = np.random.default_rng(31)
    for b in range(D.B):
        lock[b, rng.choice(D.N, Mt, replace=False)] = 0
    idx, seg = oracle.compact(lock)
    ref = oracle.layer_step_partial(D, W, X, idx, seg, st, "bf16")
    K, V, Y = _run_layer_guarded(plk, D, weights_dev(W, D), X, idx, seg, st, what="stack t=255")
    _check_layer_rows(K, V, Y, ref, st, lock, "stack t=255")


def test_layer_8b_long_context_block(plk):
    D = synth.LONG_8B
    W = synth.layer_weights(D, 0.02, seed=4)
    X = synth.hidden_states(D, seed=4)
    st = _cache_state((1, D.N, D.d), 32)
    M = int(synth.geometric_block_m(8)[0])
    assert M == 76
    b0 = 7936
    lock = np.ones((1, D.N), np.uint8)
    lock[0, b0:b0 + 32] = 0
    lock[0, synth.uniform_positions(0, b0, M - 32, tag=100)] = 0
    idx, seg = oracle.compact(lock)
    assert idx.size == M
    ref = oracle.layer_step_partial(D, W, X, idx, seg, st, "bf16")
    K, V, Y = _run_layer_guarded(plk, D, weights_dev(W, D), X, idx, seg, st, what="long-context block 0")
    _check_layer_rows(K, V, Y, ref, st, lock, "long-context block 0")


# ---------------------------------------------------------------------------
# reduced width with full-strength weights (std 1/sqrt(d)): attention, O and FFN
# change the rows by as much as the residual carries, so Y checks them directly;
# the block's change Y - X is compared as well
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("p_active", [0.1, 1.0])
def test_partial_step_bf16_unit_scale_weights(plk, p_active):
    D = SMALL
    W = synth.layer_weights(D, 1.0 / math.sqrt(D.d), seed=6)
    X = synth.hidden_states(D, seed=6)
    base = oracle.full_layer_step(D, W, X, "bf16")
    lock = synth.bernoulli_active(D.B, D.N, p_active, seed=6)
    idx, seg = oracle.compact(lock)
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.01, seed=6), lock == 0, "bf16")
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    K, V, Y = _run_partial(plk, D, W, X2, idx, seg, base)
    _check_layer_rows(K, V, Y, ref, base, lock, f"unit-scale p={p_active}")
    act = lock == 0
    dg, do = (Y - X2)[act], (ref.Y - X2)[act]
    assert np.sqrt(np.mean(do * do)) > 0.5 * np.sqrt(np.mean(X2[act].astype(np.float64) ** 2))  # a full-strength block
    _, mae, mrel = metrics(dg, do)
    assert mrel <= 2e-3, f"block change Y - X: mae {mae:.3e}, mae/rms {mrel:.3e}"


# ---------------------------------------------------------------------------
# long-context block decode (N = 8192, M from the seeded geometric draw), reduced width
# ---------------------------------------------------------------------------
def test_long_context_blocks_reduced_width(plk):
    D = synth.Dims(B=1, N=8192, d=256, H=2, hd=128, F=512, dtype="bf16")
    W = synth.layer_weights(D, 0.02, seed=4)
    X = synth.hidden_states(D, seed=4)
    rng = np.random.default_rng(4)
    st = oracle.LayerState(*(synth.round_bf16(rng.standard_normal((1, D.N, D.d)).astype(np.float32))
                             .astype(np.float64) for _ in range(3)))
    Ms = synth.geometric_block_m(8)
    prompt = 7936
    dm = pdims(plk, D)
    Wd = weights_dev(W, D)
    ws = plk.alloc_workspace(dm)
    K, V, Y = dev(st.K, BF), dev(st.V, BF), dev(st.Y, BF)
    for blk in (0, 7):
        M = int(Ms[blk])
        b0 = prompt + 32 * blk
        extra = synth.uniform_positions(0, b0, M - 32, tag=100 + blk)
        lock = np.ones((1, D.N), np.uint8)
        lock[0, np.arange(b0, b0 + 32)] = 0
        lock[0, extra] = 0
        idx, seg = oracle.compact(lock)
        assert idx.size == M
        ref = oracle.layer_step_partial(D, W, X, idx, seg, st, "bf16")
        before = [host(K), host(V), host(Y)]
        plk.layer_step_partial(dm, Wd, dev(X, BF), int_dev(idx, D.N), int_dev(seg, 2), K, V, Y, ws)
        assert plk.get_status() == plk.OK
        act = lock == 0
        for g, g0, o, name in ((K, before[0], ref.K, "K"), (V, before[1], ref.V, "V"), (Y, before[2], ref.Y, "Y")):
            gh = host(g)
            assert np.array_equal(gh[~act], g0[~act]), f"{name}: locked rows changed"
            assert_bf16_close(gh[act], o[act], f"block {blk} {name}")
        st = ref


# ---------------------------------------------------------------------------
# B = 4 multi-layer stack with the linear schedule, reduced width: score -> top-k
# among unlocked rows -> partial step, layer output feeding the next layer
# ---------------------------------------------------------------------------
def test_stack_b4_two_layers_reduced_width(plk):
    D = synth.Dims(B=4, N=2048, d=256, H=2, hd=128, F=512, dtype="bf16")
    r = 128
    sched = synth.linear_schedule(D.N)
    dm = pdims(plk, D)
    ws = plk.alloc_workspace(dm)
    layers = [synth.layer_weights(D, 0.02, seed=0, layer=l) for l in range(2)]
    Ut = synth.proxy_basis(D.d, r, seed=5)
    rng = np.random.default_rng(5)
    for t in (0, 128, 255):
        M_prev = int(sched[t - 1]) if t else D.N
        lock = np.ones((D.B, D.N), np.uint8)
        for b in range(D.B):
            lock[b, rng.choice(D.N, M_prev, replace=False)] = 0
        X = synth.hidden_states(D, seed=10 + t)
        for l, W in enumerate(layers):
            st = oracle.LayerState(*(synth.round_bf16(rng.standard_normal((D.B, D.N, D.d)).astype(np.float32))
                                     .astype(np.float64) for _ in range(3)))
            pc = rng.standard_normal((D.B, D.N, r)).astype(np.float32)
            ref_s, _ = oracle.score_drift(X.astype(np.float64), Ut.astype(np.float64), pc, "l2")
            score = torch.empty((D.B, D.N), dtype=torch.float32, device="cuda")
            plk.score_drift(dm, dev(X, BF), dev(Ut, BF), r, dev(pc, torch.float32), plk.METRIC_L2, score)
            assert_f32_close(host(score), ref_s, f"t{t} l{l} score")
            # top-k selection, both sides on the same (oracle's, fp32-rounded) scores
            s32 = ref_s.astype(np.float32)
            k = int(sched[t])
            ref_lock = oracle.lock_topk(s32.astype(np.float64), lock, k, True)
            lk_in, lk = dev(lock, torch.uint8), torch.empty((D.B, D.N), dtype=torch.uint8, device="cuda")
            idx_d, seg_d = sel_bufs(D.B, D.N)
            plk.select_active(dm, dev(s32, torch.float32), lk_in, lk, plk.SEL_TOPK_LARGEST, 0.0, k, idx_d, seg_d)
            torch.cuda.synchronize()
            assert np.array_equal(host(lk), ref_lock)
            check_compaction(idx_d, seg_d, ref_lock)
            idx, seg = oracle.compact(ref_lock)
            ref = oracle.layer_step_partial(D, W, X, idx, seg, st, "bf16")
            K, V, Y = dev(st.K, BF), dev(st.V, BF), dev(st.Y, BF)
            plk.layer_step_partial(dm, weights_dev(W, D), dev(X, BF), idx_d, seg_d, K, V, Y, ws)
            assert plk.get_status() == plk.OK
            act = ref_lock == 0
            for g, o, name in ((K, ref.K, "K"), (V, ref.V, "V"), (Y, ref.Y, "Y")):
                gh = host(g)
                assert np.array_equal(gh[~act], o[~act]), f"{name}: locked rows changed"
                assert_bf16_close(gh[act], o[act], f"t{t} l{l} {name}")
            lock = ref_lock
            X = ref.Y.astype(np.float32)  # next layer's input: this layer's output cache


# ---------------------------------------------------------------------------
# the device wait limit: a wait that nothing satisfies returns an error status
# ---------------------------------------------------------------------------
def test_wait_timeout_reports_status(plk):
    assert plk.get_status() == plk.OK
    plk.set_wait_limit(2_000_000)  # about a millisecond
    try:
        plk.selftest_wait_timeout()
        assert plk.get_status() == plk.ERR_TIMEOUT
        assert plk.get_status() == plk.OK  # cleared by the read
    finally:
        plk.set_wait_limit(4_000_000_000)
    x = torch.ones(4, device="cuda")
    assert float((x + 1).sum()) == 8.0  # the context is still usable


# ---------------------------------------------------------------------------
# the softmax's FMA-pipe exponential against exp2 (float64) and against CUDA's exp2f bound
# ---------------------------------------------------------------------------
def test_exp2_fma_error_bound(plk):
    """Every t the softmax can produce (-inf .. 8: the weights are kept below 2^8) on a dense
    grid plus the interval ends and the rounding ties of the range reduction; relative error
    <= 3e-6 (the polynomial's minimax error is 2.7e-6 in fp32), 0 below 2^-126."""
    t = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9) + 0.5, np.arange(-125, 9) - 0.5,
                        np.arange(-126, 9).astype(np.float64), [-126.0, -0.0, 0.0, 1e-30, -1e-30]]).astype(np.float32)
    below = np.array([-126.5, -127.0, -200.0, -1e30, -np.inf], np.float32)
    td = torch.from_numpy(np.concatenate([t, below])).cuda()
    out = torch.empty_like(td)
    plk.selftest_exp2(td, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    rel = np.abs(got[: t.size] - ref) / ref
    assert rel.max() <= 3e-6, rel.max()
    assert np.all(got[t.size:] == 0.0)


# ---------------------------------------------------------------------------
# the whole step from host memory (plk_denoise_step_host) against the oracle
# ---------------------------------------------------------------------------
def test_denoise_step_k_zero_is_noop(plk):
    """Top-k with k = 0 keeps no row: every row locks, and K, V, Y and the proxy cache are left
    as they were (the layer step and the folded proxy refresh see M = 0)."""
    D = synth.Dims(B=2, N=320, d=512, H=4, hd=128, F=1536, dtype="bf16")
    r = 64
    rng = np.random.default_rng(15)
    W = synth.layer_weights(D, 0.02, seed=15)
    X = synth.hidden_states(D, seed=15)
    caches = [synth.round_bf16(rng.standard_normal((D.B, D.N, D.d)).astype(np.float32)) for _ in range(3)]
    pc = rng.standard_normal((D.B, D.N, r)).astype(np.float32)
    dm = pdims(plk, D)
    g = {name: Guarded(c.shape, BF, init=dev(c, BF)) for name, c in zip("KVY", caches)}
    g["proxy"] = Guarded(pc.shape, torch.float32, init=pc)
    g["lock"] = Guarded((D.B, D.N), torch.uint8, fill=0)
    g["X"] = Guarded(X.shape, BF, init=dev(X, BF))
    g["workspace"] = Guarded((plk.step_workspace_bytes(dm, r),), torch.uint8)
    plk.denoise_step(dm, weights_dev(W, D), dev(synth.proxy_basis(D.d, r, seed=15), BF), r, plk.METRIC_L2,
                     plk.SEL_TOPK_LARGEST, 0.0, 0, g["proxy"].t, g["lock"].t, g["K"].t, g["V"].t, g["Y"].t, g["X"].t,
                     g["workspace"].t)
    assert plk.get_status() == plk.OK
    check_guards(g, "denoise_step k = 0")
    assert np.all(host(g["lock"].t) == 1)
    for name, ref in (("K", caches[0]), ("V", caches[1]), ("Y", caches[2])):
        assert np.array_equal(host(g[name].t), ref.astype(np.float64)), f"{name} changed"
    assert np.array_equal(host(g["proxy"].t), pc.astype(np.float64)), "proxy cache changed"


@pytest.mark.parametrize("entry", ["host", "device"])
def test_denoise_step_matches_oracle(plk, entry):
    """The whole step through plk_denoise_step_host (host X in, host Y out) or plk_denoise_step
    (device buffers); the proxy refresh runs inside the layer step's last kernel."""
    D = synth.Dims(B=2, N=320, d=512, H=4, hd=128, F=1536, dtype="bf16")
    r, k = 128, 96
    W = synth.layer_weights(D, 0.02, seed=14)
    X = synth.hidden_states(D, seed=14)
    Ut = synth.proxy_basis(D.d, r, seed=14)
    base = oracle.full_layer_step(D, W, X, "bf16")
    pc = oracle.to_f32(oracle.proxy_project(X.reshape(-1, D.d).astype(np.float64), Ut.astype(np.float64)))
    pc = pc.astype(np.float32).reshape(D.B, D.N, r)
    moved = np.zeros((D.B, D.N), bool)
    for b in range(D.B):
        moved[b, synth.uniform_positions(0, D.N, k, seed=14, tag=b)] = True
    X2 = synth.perturb_rows(X, synth.step_noise((D.B, D.N, D.d), 0.25, seed=14), moved, "bf16")
    # oracle: score -> top-k (the k moved rows of each sequence) -> layer step -> proxy refresh
    s, p = oracle.score_drift(X2.astype(np.float64), Ut.astype(np.float64), pc, "l2")
    ref_lock = oracle.lock_topk(s.astype(np.float32).astype(np.float64), np.zeros((D.B, D.N), np.uint8), k, True)
    assert np.array_equal(ref_lock == 0, moved)
    idx, seg = oracle.compact(ref_lock)
    ref = oracle.layer_step_partial(D, W, X2, idx, seg, base, "bf16")
    ref_pc = oracle.proxy_commit(pc, p, idx)

    dm = pdims(plk, D)
    g = {"K": Guarded(base.K.shape, BF, init=dev(base.K, BF)), "V": Guarded(base.V.shape, BF, init=dev(base.V, BF)),
         "Y": Guarded(base.Y.shape, BF, init=dev(base.Y, BF)), "proxy": Guarded(pc.shape, torch.float32, init=pc),
         "lock": Guarded((D.B, D.N), torch.uint8, fill=0)}
    n = plk.step_workspace_bytes(dm, r)
    assert n > plk.workspace_bytes(dm)
    g["workspace"] = Guarded((n,), torch.uint8)
    if entry == "host":
        X_host = torch.from_numpy(np.ascontiguousarray(X2)).to(BF).pin_memory()
        Y_host = torch.full(base.Y.shape, -3.0, dtype=BF).pin_memory()
        plk.denoise_step_host(dm, weights_dev(W, D), dev(Ut, BF), r, plk.METRIC_L2, plk.SEL_TOPK_LARGEST, 0.0, k,
                              g["proxy"].t, g["lock"].t, g["K"].t, g["V"].t, g["Y"].t, X_host, Y_host,
                              g["workspace"].t)
    else:
        g["X"] = Guarded(X2.shape, BF, init=dev(X2, BF))
        plk.denoise_step(dm, weights_dev(W, D), dev(Ut, BF), r, plk.METRIC_L2, plk.SEL_TOPK_LARGEST, 0.0, k,
                         g["proxy"].t, g["lock"].t, g["K"].t, g["V"].t, g["Y"].t, g["X"].t, g["workspace"].t)
    assert plk.get_status() == plk.OK
    check_guards(g, f"denoise_step ({entry})")
    assert np.array_equal(host(g["lock"].t), ref_lock)
    Yd = host(g["Y"].t)
    if entry == "host":
        assert np.array_equal(Y_host.to(torch.float64).numpy(), Yd), "Y_host is the device Y"
    _check_layer_rows(host(g["K"].t), host(g["V"].t), Yd, ref, base, ref_lock, f"{entry} step")
    assert_f32_close(host(g["proxy"].t), ref_pc, "proxy cache", tol=1e-5)


def _steps_case():
    """Four denoising steps at a small bf16 shape: step t moves a shrinking subset of the rows the
    previous step moved, so threshold locking (L2 drift below tau) shrinks the active set
    120 -> 80 -> 40 -> 8 rows per sequence."""
    D = synth.Dims(B=2, N=320, d=512, H=4, hd=128, F=1536, dtype="bf16")
    r, tau = 128, 0.05
    W = synth.layer_weights(D, 0.02, seed=15)
    X0 = synth.hidden_states(D, seed=15)
    Ut = synth.proxy_basis(D.d, r, seed=15)
    base = oracle.full_layer_step(D, W, X0, "bf16")
    pc0 = oracle.to_f32(oracle.proxy_project(X0.reshape(-1, D.d).astype(np.float64), Ut.astype(np.float64)))
    pc0 = pc0.astype(np.float32).reshape(D.B, D.N, r)
    Xs, moved, Xc = [], np.ones((D.B, D.N), bool), X0
    for t, cnt in enumerate((120, 80, 40, 8)):
        m = np.zeros((D.B, D.N), bool)
        for b in range(D.B):
            pool = np.flatnonzero(moved[b])
            m[b, pool[synth.uniform_positions(0, pool.size, cnt, seed=15 + t, tag=b)]] = True
        Xc = synth.perturb_rows(Xc, synth.step_noise((D.B, D.N, D.d), 0.25, seed=15, step=t), m, "bf16")
        Xs.append(Xc)
        moved = m
    return D, r, tau, W, Ut, base, pc0, Xs


@pytest.mark.parametrize("streams", ["separate", "same", "direct"])
def test_denoise_steps_host_pipelined(plk, streams):
    """plk_denoise_steps_host (each step's upload and download on their own streams beside the
    compute of the neighbouring steps) against the same steps as separate plk_denoise_step_host
    calls, bit for bit in reproducible mode, and against the oracle's chain of steps (threshold
    lock bit-exact, K, V and every step's Y within the bf16 bounds).  The call captures the step
    as CUDA graphs and launches those; "direct": a trace event is set, so the call launches the
    step's kernels directly instead.  "same": all three streams are one, and every step's Y goes
    to the same host buffer (it ends with the last step's Y)."""
    D, r, tau, W, Ut, base, pc0, Xs = _steps_case()
    T = len(Xs)
    # the oracle's chain: score -> lock (drift below tau) -> partial layer step -> proxy refresh
    state, pc, lock = base, pc0, np.zeros((D.B, D.N), np.uint8)
    ref_Y, ref_locks = [], []
    for X in Xs:
        s, p = oracle.score_drift(X.astype(np.float64), Ut.astype(np.float64), pc, "l2")
        lock = oracle.lock_threshold(s.astype(np.float32).astype(np.float64), lock, tau, greater=False)
        idx, seg = oracle.compact(lock)
        state = oracle.layer_step_partial(D, W, X, idx, seg, state, "bf16")
        pc = oracle.proxy_commit(pc, p, idx).astype(np.float32)
        ref_Y.append(state.Y)
        ref_locks.append(lock.copy())
    assert [int((l == 0).sum()) for l in ref_locks] == [240, 160, 80, 16]

    dm, Wd, Ud = pdims(plk, D), weights_dev(W, D), dev(Ut, BF)
    X_hosts = [torch.from_numpy(np.ascontiguousarray(X)).to(BF).pin_memory() for X in Xs]

    def fresh():
        return {"K": Guarded(base.K.shape, BF, init=dev(base.K, BF)), "V": Guarded(base.V.shape, BF, init=dev(base.V, BF)),
                "Y": Guarded(base.Y.shape, BF, init=dev(base.Y, BF)),
                "proxy": Guarded(pc0.shape, torch.float32, init=pc0),
                "lock": Guarded((D.B, D.N), torch.uint8, fill=0)}

    plk.set_deterministic(True)
    try:
        # the same steps as separate calls
        gs = fresh()
        sws = plk.alloc_step_workspace(dm, r)
        seq_Y = []
        for t in range(T):
            Yh = torch.full(base.Y.shape, -3.0, dtype=BF).pin_memory()
            plk.denoise_step_host(dm, Wd, Ud, r, plk.METRIC_L2, plk.SEL_THRESH_LT, tau, 0, gs["proxy"].t,
                                  gs["lock"].t, gs["K"].t, gs["V"].t, gs["Y"].t, X_hosts[t], Yh, sws)
            torch.cuda.synchronize()
            assert np.array_equal(host(gs["lock"].t), ref_locks[t]), f"separate calls: lock after step {t}"
            seq_Y.append(Yh.to(torch.float64).numpy())
        # pipelined
        g = fresh()
        n = plk.steps_workspace_bytes(dm, r)
        assert n > plk.step_workspace_bytes(dm, r)
        g["workspace"] = Guarded((n,), torch.uint8)
        if streams in ("separate", "direct"):
            up, down = torch.cuda.Stream(), torch.cuda.Stream()
            Y_hosts = [torch.full(base.Y.shape, -3.0, dtype=BF).pin_memory() for _ in range(T)]
        else:
            up = down = torch.cuda.current_stream()
            Y_hosts = [torch.full(base.Y.shape, -3.0, dtype=BF).pin_memory()] * T
        trace = [torch.cuda.Event(enable_timing=True)] if streams == "direct" else []
        plk.trace_events(trace)
        try:
            plk.denoise_steps_host(dm, Wd, Ud, r, plk.METRIC_L2, plk.SEL_THRESH_LT, tau, 0, g["proxy"].t,
                                   g["lock"].t, g["K"].t, g["V"].t, g["Y"].t, X_hosts, Y_hosts, g["workspace"].t, up,
                                   down)
        finally:
            plk.trace_events([])
        torch.cuda.current_stream().synchronize()  # the call's stream waits for the last download
        assert plk.get_status() == plk.OK
    finally:
        plk.set_deterministic(False)
    check_guards(g, f"denoise_steps_host ({streams})")
    assert np.array_equal(host(g["lock"].t), ref_locks[-1])
    for name in ("K", "V", "Y", "proxy"):
        assert np.array_equal(host(g[name].t), host(gs[name].t)), f"{name} differs from the separate calls"
    got = [y.to(torch.float64).numpy() for y in Y_hosts]
    steps = [T - 1] if streams == "same" else range(T)
    for t in steps:
        assert np.array_equal(got[t], seq_Y[t]), f"Y_hosts[{t}] differs from the separate call's Y"
        never = ref_locks[0].astype(bool)  # locked at step 0: Y keeps the base rows
        assert np.array_equal(got[t][never], base.Y[never]), f"step {t}: a row locked from the start was written"
        act = ~never
        assert_bf16_close(got[t][act], ref_Y[t][act], f"pipelined step {t} Y")
    K, V = host(g["K"].t), host(g["V"].t)
    act = ~ref_locks[0].astype(bool)
    assert_bf16_close(K[act], state.K[act], "pipelined K")
    assert_bf16_close(V[act], state.V[act], "pipelined V")
