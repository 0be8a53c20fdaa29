"""Pins of the CPU oracle against things other than itself.

Each test ties an oracle function to a library routine, a brute-force loop on a
tiny input, a closed form from the SureLock page ("Stopping Computation for
Converged Tokens in Masked Diffusion-LM Decoding", Sec. 2 "Algorithmic
Complexity"), or an invariant the pages state.  The mutation tests at the end
plant plausible mistakes in copies of the oracle and check that a pin fails.
"""
import hashlib
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle
import synth
from oracle import plk_oracle as po


def _dims(B=2, N=7, d=16, H=2, hd=8, F=24, dtype="f32", Hkv=0, rope_theta=0.0):
    return synth.Dims(B=B, N=N, d=d, H=H, hd=hd, F=F, eps=1e-6, dtype=dtype, Hkv=Hkv, rope_theta=rope_theta)


def _weights(dims, std=None, seed=0):
    return synth.layer_weights(dims, std if std is not None else 1.0 / math.sqrt(dims.d), seed=seed)


# ---------------------------------------------------------------------------
# rounding
# ---------------------------------------------------------------------------
def test_to_bf16_matches_torch_rounding():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, -3.3895314e38,
                  3.4e38, 1e-40, -1e-41, 2.0 ** -133, 2.0 ** -134], dtype=np.float32),
    ]).astype(np.float32)
    # exact ties: 1 + 2^-8 (rounds down to even) and 1 + 3*2^-8 (rounds up)
    got = oracle.to_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref)


def test_to_f32_is_numpy_cast():
    v = np.array([1.0 + 2.0 ** -30, 1e-50, 3.0], dtype=np.float64)
    np.testing.assert_array_equal(oracle.to_f32(v), v.astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# elementwise pieces against torch
# ---------------------------------------------------------------------------
def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 33))
    g = rng.standard_normal(33)
    ref = Fnn.rms_norm(torch.from_numpy(x), (33,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-14)


def test_silu_matches_torch():
    z = np.linspace(-50, 50, 1001)
    np.testing.assert_allclose(oracle.silu(z), Fnn.silu(torch.from_numpy(z)).numpy(),
                               rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------------------
# the full block against a composition of torch library routines
# ---------------------------------------------------------------------------
def torch_block(dims, W, X):
    B, N, d, H, hd, F = dims.B, dims.N, dims.d, dims.H, dims.hd, dims.F
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    x = t(X)
    xn = Fnn.rms_norm(x, (d,), t(W["g1"]), eps=dims.eps)
    Hkv = dims.Hkv or H
    qkv = Fnn.linear(xn, t(W["w_qkv"]))
    q, k, v = qkv.split([d, Hkv * hd, Hkv * hd], dim=-1)
    heads = lambda z, n: z.reshape(B, N, n, hd).transpose(1, 2)
    # grouped-query attention: torch repeats each K/V head for H / Hkv consecutive query heads
    a = Fnn.scaled_dot_product_attention(heads(q, H), heads(k, Hkv), heads(v, Hkv), is_causal=False,
                                         enable_gqa=Hkv != H)
    a = a.transpose(1, 2).reshape(B, N, d)
    h = x + Fnn.linear(a, t(W["w_o"]))
    hn = Fnn.rms_norm(h, (d,), t(W["g2"]), eps=dims.eps)
    g, u = Fnn.linear(hn, t(W["w_gu"])).split(F, dim=-1)
    y = h + Fnn.linear(Fnn.silu(g) * u, t(W["w_down"]))
    return k.numpy(), v.numpy(), y.numpy()


@pytest.mark.parametrize("shape", [dict(B=1, N=9, d=16, H=2, hd=8, F=24),
                                   dict(B=3, N=5, d=12, H=3, hd=4, F=8),
                                   dict(B=1, N=64, d=64, H=4, hd=16, F=256),
                                   dict(B=2, N=7, d=16, H=4, hd=4, F=24, Hkv=2),   # grouped-query
                                   dict(B=1, N=9, d=24, H=6, hd=4, F=8, Hkv=1),    # one K/V head
                                   dict(B=2, N=6, d=24, H=6, hd=4, F=8, Hkv=3)])
def test_full_step_matches_torch_composition(shape):
    dims = _dims(**shape)
    W = _weights(dims)
    X = synth.hidden_states(dims)
    st = oracle.full_layer_step(dims, W, X, "f64")
    k, v, y = torch_block(dims, W, X)
    np.testing.assert_allclose(st.K, k, rtol=0, atol=1e-12)
    np.testing.assert_allclose(st.V, v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(st.Y, y, rtol=0, atol=1e-11)


def test_attention_matches_sdpa_single_head():
    # textbook softmax(Q K^T / sqrt(hd)) V through the oracle's full step with
    # identity projections: d = hd, H = 1, w_qkv = [I; I; I], w_o = 0, FFN = 0
    N, d = 11, 6
    dims = _dims(B=1, N=N, d=d, H=1, hd=d, F=4)
    rng = np.random.default_rng(3)
    eye = np.eye(d)
    W = dict(w_qkv=np.concatenate([eye, 2 * eye, -eye]), w_o=np.eye(d), w_gu=np.zeros((8, d)),
             w_down=np.zeros((d, 4)), g1=np.ones(d), g2=np.ones(d))
    X = rng.standard_normal((1, N, d))
    st = oracle.full_layer_step(dims, W, X, "f64")
    xn = oracle.rmsnorm(X[0], np.ones(d), 1e-6)
    a = Fnn.scaled_dot_product_attention(torch.from_numpy(xn)[None], torch.from_numpy(2 * xn)[None],
                                         torch.from_numpy(-xn)[None]).numpy()[0]
    np.testing.assert_allclose(st.Y[0], X[0] + a, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# brute force: explicit scalar loops on a tiny input
# ---------------------------------------------------------------------------
def brute_block(dims, W, X, rows, store=None):
    """Scalar-loop block.  ``store`` (optional) maps a list of floats to the values a
    stored tensor holds: it is applied to the K and V rows (the cache) and to the
    output rows, and nowhere else."""
    B, N, d, H, hd, F = dims.B, dims.N, dims.d, dims.H, dims.hd, dims.F
    keep = store or (lambda vals: vals)
    Wq = W["w_qkv"]
    out = {}

    def norm(vec, g):
        ms = sum(z * z for z in vec) / len(vec)
        r = 1.0 / math.sqrt(ms + dims.eps)
        return [vec[i] * r * float(g[i]) for i in range(len(vec))]

    def lin(wm, vec):
        return [sum(float(wm[o][i]) * vec[i] for i in range(len(vec))) for o in range(len(wm))]

    xs = {(b, n): [float(X[b][n][c]) for c in range(d)] for b in range(B) for n in range(N)}
    kv = {}
    for (b, n), vec in xs.items():
        z = lin(Wq, norm(vec, W["g1"]))
        kv[(b, n)] = (z[:d], keep(z[d:2 * d]), keep(z[2 * d:]))
    for (b, n) in rows:
        q = kv[(b, n)][0]
        a = [0.0] * d
        for h in range(H):
            sc = []
            for m in range(N):
                kk = kv[(b, m)][1]
                sc.append(sum(q[h * hd + c] * kk[h * hd + c] for c in range(hd)) / math.sqrt(hd))
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            tot = sum(ex)
            for c in range(hd):
                a[h * hd + c] = sum(ex[m] / tot * kv[(b, m)][2][h * hd + c] for m in range(N))
        hres = [xs[(b, n)][c] + lin(W["w_o"], a)[c] for c in range(d)]
        hn = norm(hres, W["g2"])
        gu = lin(W["w_gu"], hn)
        act = [gu[f] / (1.0 + math.exp(-gu[f])) * gu[F + f] for f in range(F)]
        dn = lin(W["w_down"], act)
        out[(b, n)] = keep([hres[c] + dn[c] for c in range(d)])
    return kv, out


def test_full_and_partial_match_brute_force():
    dims = _dims(B=2, N=5, d=8, H=2, hd=4, F=12)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=4)
    rows = [(b, n) for b in range(2) for n in range(5)]
    kv, yb = brute_block(dims, W, X, rows)
    st = oracle.full_layer_step(dims, W, X, "f64")
    for (b, n) in rows:
        np.testing.assert_allclose(st.K[b, n], kv[(b, n)][1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(st.V[b, n], kv[(b, n)][2], rtol=0, atol=1e-12)
        np.testing.assert_allclose(st.Y[b, n], yb[(b, n)], rtol=0, atol=1e-12)
    lock = np.zeros((2, 5), np.uint8)
    idx, seg = oracle.compact(lock)
    zero = oracle.LayerState(np.zeros_like(st.K), np.zeros_like(st.V), np.zeros_like(st.Y))
    sp = oracle.layer_step_partial(dims, W, X, idx, seg, zero, "f64")
    for (b, n) in rows:
        np.testing.assert_allclose(sp.Y[b, n], yb[(b, n)], rtol=0, atol=1e-12)


def _torch_bf16(vals):
    """Round to bf16 with torch's conversion (an implementation independent of the oracle's)."""
    return torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).tolist()


def _bf16_case():
    dims = _dims(B=2, N=5, d=8, H=2, hd=4, F=12, dtype="bf16")
    W = synth.layer_weights(dims, 0.35, seed=3)
    X = synth.hidden_states(dims, seed=3)
    return dims, W, X


def _assert_within_one_ulp(a, b, what, frac=0.02):
    """Equal up to a bf16 rounding that lands on the other side of a tie: at most one
    bf16 step of the element, on a small fraction of the elements."""
    ulp = np.ldexp(1.0, np.frexp(np.abs(b) + 1e-300)[1] - 8)
    assert np.all(np.abs(a - b) <= ulp), what
    assert np.mean(a != b) <= frac, (what, np.mean(a != b))


def test_bf16_policy_rounds_exactly_the_stored_tensors():
    # brute force with torch's bf16 rounding applied to the K/V cache rows and the
    # output rows only: the oracle's bf16 policy must agree with it
    dims, W, X = _bf16_case()
    rows = [(b, n) for b in range(2) for n in range(5)]
    kv, yb = brute_block(dims, W, X, rows, store=_torch_bf16)
    st = oracle.full_layer_step(dims, W, X, "bf16")
    K = np.array([[kv[(b, n)][1] for n in range(5)] for b in range(2)])
    V = np.array([[kv[(b, n)][2] for n in range(5)] for b in range(2)])
    Y = np.array([[yb[(b, n)] for n in range(5)] for b in range(2)])
    _assert_within_one_ulp(st.K, K, "K")
    _assert_within_one_ulp(st.V, V, "V")
    _assert_within_one_ulp(st.Y, Y, "Y")
    # stored values are bf16 numbers; the f64 policy differs from them by at most half a step
    for a in (st.K, st.V, st.Y):
        np.testing.assert_array_equal(a, _torch_bf16_arr(a))
    f = oracle.full_layer_step(dims, W, X, "f64")
    assert np.max(np.abs(st.K - f.K) / np.ldexp(1.0, np.frexp(np.abs(f.K))[1] - 8)) <= 0.5 + 1e-9
    # the partial step with every row active agrees with the brute force too
    idx, seg = oracle.compact(np.zeros((2, 5), np.uint8))
    zero = oracle.LayerState(np.zeros_like(st.K), np.zeros_like(st.V), np.zeros_like(st.Y))
    part = oracle.layer_step_partial(dims, W, X, idx, seg, zero, "bf16")
    _assert_within_one_ulp(part.Y, Y, "partial Y")


def _torch_bf16_arr(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("old,new", [
    ("k = _store(k, policy)", "k = k"),                                          # cache rows not rounded
    ("y = _store(hres + _mm(act, _w(W, \"w_down\")), policy)",
     "y = hres + _mm(act, _w(W, \"w_down\"))"),                                 # output not rounded
    ("hres = x + _mm(a, ", "hres = x + _mm(to_bf16(a), "),                      # attention output rounded
    ("act = silu(gu[:, :F]) * gu[:, F:]", "act = to_bf16(silu(gu[:, :F]) * gu[:, F:])"),  # SwiGLU product rounded
    ("hn = rmsnorm(hres, W[\"g2\"], dims.eps)", "hn = to_bf16(rmsnorm(hres, W[\"g2\"], dims.eps))"),
])
def test_bf16_policy_mutants_are_caught(old, new):
    dims, W, X = _bf16_case()
    rows = [(b, n) for b in range(2) for n in range(5)]
    kv, yb = brute_block(dims, W, X, rows, store=_torch_bf16)
    K = np.array([[kv[(b, n)][1] for n in range(5)] for b in range(2)])
    Y = np.array([[yb[(b, n)] for n in range(5)] for b in range(2)])
    st = _mutant(po.full_layer_step, old, new)(dims, W, X, "bf16")
    with pytest.raises(AssertionError):
        _assert_within_one_ulp(st.K, K, "K")
        _assert_within_one_ulp(st.Y, Y, "Y")


# ---------------------------------------------------------------------------
# invariants stated by the SureLock page (Sec. 2)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("policy", ["f64", "bf16"])
def test_partial_with_all_rows_equals_full(policy):
    dims = _dims(B=2, N=12, d=32, H=2, hd=16, F=48, dtype="bf16" if policy == "bf16" else "f32")
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=5)
    full = oracle.full_layer_step(dims, W, X, policy)
    idx, seg = oracle.compact(np.zeros((2, 12), np.uint8))
    zero = oracle.LayerState(np.zeros_like(full.K), np.zeros_like(full.V), np.zeros_like(full.Y))
    part = oracle.layer_step_partial(dims, W, X, idx, seg, zero, policy)
    if policy == "f64":
        for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    else:
        # same values; a bf16 rounding may flip on a 1e-16 difference in the
        # two summation forms, so allow one bf16 ulp on a tiny fraction
        for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
            ulp = np.ldexp(1.0, np.frexp(np.abs(b) + 1e-30)[1] - 8)
            assert np.all(np.abs(a - b) <= ulp)
            assert np.mean(a != b) < 1e-2


def test_unchanged_inputs_partial_rows_equal_full_rows():
    dims = _dims(B=2, N=10, d=16, H=2, hd=8, F=32)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=6)
    full = oracle.full_layer_step(dims, W, X, "f64")
    lock = synth.bernoulli_active(2, 10, 0.4, seed=6)
    idx, seg = oracle.compact(lock)
    assert 0 < idx.size < 20
    part = oracle.layer_step_partial(dims, W, X, idx, seg, full, "f64")
    for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def _h(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def test_locked_rows_untouched():
    dims = _dims(B=2, N=10, d=16, H=2, hd=8, F=32)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=7)
    rng = np.random.default_rng(7)
    st = oracle.LayerState(rng.standard_normal((2, 10, 16)), rng.standard_normal((2, 10, 16)),
                           rng.standard_normal((2, 10, 16)))
    lock = synth.bernoulli_active(2, 10, 0.3, seed=8)
    idx, seg = oracle.compact(lock)
    out = oracle.layer_step_partial(dims, W, X, idx, seg, st, "f64")
    locked = lock.astype(bool)
    for new, old in ((out.K, st.K), (out.V, st.V), (out.Y, st.Y)):
        assert _h(new[locked]) == _h(old[locked])
        assert np.all(np.any(new[~locked] != old[~locked], axis=-1))


def test_attention_depends_on_locked_keys():
    # continued attention: an active row's output changes when a locked row's cached K changes
    dims = _dims(B=1, N=6, d=8, H=2, hd=4, F=8)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=9)
    st = oracle.full_layer_step(dims, W, X, "f64")
    lock = np.array([[1, 1, 0, 1, 1, 1]], np.uint8)
    idx, seg = oracle.compact(lock)
    a = oracle.layer_step_partial(dims, W, X, idx, seg, st, "f64")
    st2 = st.copy()
    st2.K[0, 4] += 1.0
    b = oracle.layer_step_partial(dims, W, X, idx, seg, st2, "f64")
    assert np.max(np.abs(a.Y[0, 2] - b.Y[0, 2])) > 1e-6


# ---------------------------------------------------------------------------
# the complexity closed form (SureLock Sec. 2 "Algorithmic Complexity")
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,N,d,H,hd,F,p", [(1, 16, 16, 2, 8, 24, 0.25), (3, 9, 12, 3, 4, 20, 0.5)])
def test_flop_count_closed_form(B, N, d, H, hd, F, p):
    dims = _dims(B=B, N=N, d=d, H=H, hd=hd, F=F)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=10)
    with oracle.count_flops() as cf:
        full = oracle.full_layer_step(dims, W, X, "f64")
    assert cf.flops == B * (N * (8 * d * d + 6 * d * F) + 4 * N * N * d)
    lock = synth.bernoulli_active(B, N, p, seed=10)
    idx, seg = oracle.compact(lock)
    M = idx.size
    with oracle.count_flops() as cp:
        oracle.layer_step_partial(dims, W, X, idx, seg, full, "f64")
    assert cp.flops == M * (8 * d * d + 6 * d * F) + 4 * M * N * d
    # the 8B-shape per-row figure
    assert 8 * 4096 ** 2 + 6 * 4096 * 12288 + 4 * 1024 * 4096 == 452_984_832


# ---------------------------------------------------------------------------
# S1 proxy and scores
# ---------------------------------------------------------------------------
def test_proxy_identity_basis_and_score_cases():
    rng = np.random.default_rng(11)
    d, r = 20, 5
    Ut = np.eye(d)[:r]
    X = rng.standard_normal((2, 4, d))
    s, p = oracle.score_drift(X, Ut, np.zeros((2, 4, r)), "l2")
    np.testing.assert_array_equal(p, X[..., :r])
    np.testing.assert_allclose(s, np.linalg.norm(X[..., :r], axis=-1), rtol=1e-15)
    s2, _ = oracle.score_drift(X, Ut, X[..., :r], "l2")
    np.testing.assert_array_equal(s2, 0.0)
    s3, _ = oracle.score_drift(X, Ut, X[..., :r], "cos")
    np.testing.assert_allclose(s3, 1.0, rtol=1e-15)
    s4, _ = oracle.score_drift(X, Ut, -3.0 * X[..., :r], "cos")
    np.testing.assert_allclose(s4, -1.0, rtol=1e-15)
    s5, _ = oracle.score_drift(X, Ut, np.zeros((2, 4, r)), "cos")
    np.testing.assert_array_equal(s5, 0.0)
    # orthonormal basis: |U^T x| <= |x|, and cosine against scipy's distance
    from scipy.spatial.distance import cosine as sp_cos
    U = synth.proxy_basis(d, r, dtype="f32").astype(np.float64)
    np.testing.assert_allclose(U @ U.T, np.eye(r), atol=1e-6)
    _, pu = oracle.score_drift(X, U, np.zeros((2, 4, r)), "l2")
    assert np.all(np.linalg.norm(pu, axis=-1) <= np.linalg.norm(X, axis=-1) * (1 + 1e-6))
    pc = rng.standard_normal((2, 4, r))
    sc, _ = oracle.score_drift(X, U, pc, "cos")
    for b in range(2):
        for n in range(4):
            assert abs(sc[b, n] - (1.0 - sp_cos(pu[b, n], pc[b, n]))) < 1e-13


# ---------------------------------------------------------------------------
# S10 proxy half: the refreshed rows take the fresh proxy as float32 (SPA-Cache part 1:
# the low-resolution snapshot is refreshed where the row was recomputed)
# ---------------------------------------------------------------------------
def _proxy_commit_case():
    rng = np.random.default_rng(18)
    B, N, r = 3, 11, 5
    cache = rng.standard_normal((B, N, r)).astype(np.float32).astype(np.float64)
    fresh = rng.standard_normal((B, N, r)) * 3.0  # float64 values, not float32-representable
    lock = (rng.random((B, N)) < 0.55).astype(np.uint8)
    idx, _ = oracle.compact(lock)
    assert 0 < idx.size < B * N
    return cache, fresh, lock, idx


def _proxy_commit_reference(cache, fresh, lock):
    """Row by row with Python scalars: active rows get struct-packed float32 values."""
    import struct
    out = cache.copy()
    B, N, r = cache.shape
    for b in range(B):
        for n in range(N):
            if lock[b, n] == 0:
                for c in range(r):
                    out[b, n, c] = struct.unpack("f", struct.pack("f", float(fresh[b, n, c])))[0]
    return out


def test_proxy_commit_refreshes_active_rows_as_float32():
    cache, fresh, lock, idx = _proxy_commit_case()
    got = oracle.proxy_commit(cache, fresh, idx)
    ref = _proxy_commit_reference(cache, fresh, lock)
    np.testing.assert_array_equal(got, ref)
    locked = lock.astype(bool)
    assert got[locked].tobytes() == cache[locked].tobytes()      # the other rows: byte-identical
    assert np.all(got[~locked] != fresh[~locked])                # fresh values were rounded ...
    assert np.max(np.abs(got[~locked] - fresh[~locked]) / np.abs(fresh[~locked])) <= 2.0 ** -24  # ... to float32
    assert np.array_equal(cache, _proxy_commit_case()[0])       # the input is not modified


@pytest.mark.parametrize("old,new", [
    ("flat[np.asarray(idx, dtype=np.int64)] = to_f32(", "_unused = ("),   # never writes the fresh proxy
    ("= to_f32(np.asarray(p)", "= (np.asarray(p)"),                     # writes the unrounded value
    ("[idx])", "[idx[::-1]])"),                                          # rows paired with the wrong fresh rows
])
def test_proxy_commit_mutants_are_caught(old, new):
    cache, fresh, lock, idx = _proxy_commit_case()
    got = _mutant(po.proxy_commit, old, new)(cache, fresh, idx)
    assert not np.array_equal(got, _proxy_commit_reference(cache, fresh, lock))


# ---------------------------------------------------------------------------
# S2/S3 integer semantics against numpy sorts
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("largest", [True, False])
def test_topk_against_lexsort(ties, largest):
    rng = np.random.default_rng(12)
    B, N = 3, 200
    s = rng.integers(0, 5, (B, N)).astype(np.float64) if ties else rng.standard_normal((B, N))
    lock = (rng.random((B, N)) < 0.3).astype(np.uint8)
    for k in (0, 1, 17, 140, 500):
        got = oracle.lock_topk(s, lock, k, largest)
        for b in range(B):
            cand = np.nonzero(lock[b] == 0)[0]
            key = -s[b, cand] if largest else s[b, cand]
            order = cand[np.lexsort((cand, key))]
            keep = np.zeros(N, bool)
            keep[order[:k]] = True
            np.testing.assert_array_equal(got[b], (~keep).astype(np.uint8))


def test_topk_nan_and_signed_zero():
    s = np.array([[np.nan, 0.0, -0.0, 1.0, np.nan, -1.0]])
    lock = np.zeros((1, 6), np.uint8)
    np.testing.assert_array_equal(oracle.lock_topk(s, lock, 3, True)[0], [1, 0, 0, 0, 1, 1])
    np.testing.assert_array_equal(oracle.lock_topk(s, lock, 2, False)[0], [1, 0, 1, 1, 1, 0])
    np.testing.assert_array_equal(oracle.lock_topk(s, lock, 6, True)[0], [0] * 6)


def test_threshold_monotone_and_strict():
    s = np.array([[0.99, 0.990001, np.nan, 1.0, -2.0]])
    lock = np.array([[0, 0, 0, 0, 1]], np.uint8)
    np.testing.assert_array_equal(oracle.lock_threshold(s, lock, 0.99, True), [[0, 1, 0, 1, 1]])
    np.testing.assert_array_equal(oracle.lock_threshold(s, lock, 0.99, False), [[0, 0, 0, 0, 1]])
    rng = np.random.default_rng(13)
    lk = np.zeros((2, 50), np.uint8)
    for _ in range(10):
        new = oracle.lock_threshold(rng.random((2, 50)), lk, 0.8, True)
        assert np.all(new >= lk)
        lk = new


def test_compact_against_nonzero():
    rng = np.random.default_rng(14)
    lock = (rng.random((4, 33)) < 0.6).astype(np.uint8)
    idx, seg = oracle.compact(lock)
    np.testing.assert_array_equal(idx, np.nonzero(lock.reshape(-1) == 0)[0])
    np.testing.assert_array_equal(seg, np.concatenate([[0], np.cumsum((lock == 0).sum(1))]))
    idx0, seg0 = oracle.compact(np.ones((2, 5), np.uint8))
    assert idx0.size == 0 and list(seg0) == [0, 0, 0]


# ---------------------------------------------------------------------------
# mutation tests: plant a plausible mistake in a copy of the oracle; a pin must fail
# ---------------------------------------------------------------------------
_FULL_MUTANTS = [
    ("hres = x + _mm(a", "hres = _mm(a"),                                  # dropped residual
    ("* scale          ", "* 1.0            "),                            # wrong softmax scale
    ("q, k = _qk(qkv, dims", "k, q = _qk(qkv, dims"),                     # q and k swapped
    ("_mm(a, _w(W, \"w_o\"))", "_mm(a, _w(W, \"w_o\").T)"),               # transposed operand
    ("silu(gu[:, :F]) * gu[:, F:]", "silu(gu[:, F:]) * gu[:, :F]"),       # gate/up swapped
    ("S = S - S.max(axis=1, keepdims=True)", "S = S - S.max(axis=0, keepdims=True)"),
    ("P = P / P.sum(axis=1, keepdims=True)", "P = P / P.sum(axis=0, keepdims=True)"),
    ("hn = rmsnorm(hres, W[\"g2\"]", "hn = rmsnorm(x, W[\"g2\"]"),
]


def _mutant(func, old, new):
    src = textwrap.dedent(inspect.getsource(func))
    assert old in src, old
    ns = dict(po.__dict__)
    exec(compile(src.replace(old, new, 1), "<mutant>", "exec"), ns)
    return ns[func.__name__]


@pytest.mark.parametrize("old,new", _FULL_MUTANTS)
def test_full_step_mutants_are_caught(old, new):
    dims = _dims(B=2, N=9, d=16, H=2, hd=8, F=24)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=15)
    W = dict(W, g2=np.linspace(0.5, 1.5, 16))
    mut = _mutant(po.full_layer_step, old, new)
    st = mut(dims, W, X, "f64")
    k, v, y = torch_block(dims, W, X)
    assert max(np.max(np.abs(st.K - k)), np.max(np.abs(st.V - v)), np.max(np.abs(st.Y - y))) > 1e-6


_PARTIAL_MUTANTS = [
    ("hres = x[rows] + _mm(a", "hres = _mm(a"),
    ("Kf[idx] = k", "Kf[idx] = v"),
    ("Vf[idx] = v", "pass"),
    ("s = s - s.max()", "s = s - s.min()"),  # harmless shift: must NOT be caught (control)
    ("* scale     # [N]", "           # [N]"),
    ("q[j:j + 1, cols]", "q[0:1, cols]"),
    ("Kb = Kf[b * N:(b + 1) * N]", "Kb = Kf[0:N]"),
    ("a[t, cols] = _mm(p[None, :], Vb[:, kv].T)[0]", "a[t, cols] = _mm(p[None, :], Kb[:, kv].T)[0]"),
    ("out.Y.reshape(B * N, d)[idx[rows]] = y", "out.Y.reshape(B * N, d)[idx[rows]] = hres"),
]


@pytest.mark.parametrize("old,new", _PARTIAL_MUTANTS)
def test_partial_step_mutants_are_caught(old, new):
    dims = _dims(B=2, N=8, d=16, H=2, hd=8, F=24)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=16)
    full = oracle.full_layer_step(dims, W, X, "f64")
    lock = synth.bernoulli_active(2, 8, 0.5, seed=16)
    idx, seg = oracle.compact(lock)
    assert idx.size > 2 and seg[1] > 0 and seg[2] > seg[1]
    mut = _mutant(po.layer_step_partial, old, new)
    # pin 1: unchanged inputs -> active rows equal full recompute
    part = mut(dims, W, X, idx, seg, full, "f64")
    err = max(np.max(np.abs(part.K - full.K)), np.max(np.abs(part.V - full.V)),
              np.max(np.abs(part.Y - full.Y)))
    # pin 2: from stale caches, active rows get exactly the fresh K/V of full recompute
    rng = np.random.default_rng(17)
    stale = oracle.LayerState(*(rng.standard_normal(full.K.shape) for _ in range(3)))
    part2 = mut(dims, W, X, idx, seg, stale, "f64")
    act = lock == 0
    err = max(err, np.max(np.abs(part2.K[act] - full.K[act])), np.max(np.abs(part2.V[act] - full.V[act])))
    if old == "s = s - s.max()":
        assert err < 1e-12  # subtracting any constant leaves softmax unchanged
    else:
        assert err > 1e-6


# ---------------------------------------------------------------------------
# KL lock rule (SureLock "Locking Condition": KL(p_t || p_{t-1}) <= eps, optional low-entropy gate)
# ---------------------------------------------------------------------------
def _sigmoid(a):
    return 1.0 / (1.0 + math.exp(-a))


def test_log_softmax_matches_torch():
    z = np.random.default_rng(30).standard_normal((5, 7, 33)) * 4.0
    ref = Fnn.log_softmax(torch.from_numpy(z), dim=-1).numpy()
    np.testing.assert_allclose(oracle.log_softmax(z), ref, rtol=0, atol=1e-12)


def test_kl_matches_torch_kl_div_in_the_stated_direction():
    rng = np.random.default_rng(31)
    zt, zp = rng.standard_normal((6, 40)) * 3, rng.standard_normal((6, 40)) * 3
    lt = torch.from_numpy(oracle.log_softmax(zt))
    lp = torch.from_numpy(oracle.log_softmax(zp))
    # torch: kl_div(input = log q, target = log p, log_target) = sum p (log p - log q) = KL(p || q)
    ref = Fnn.kl_div(lp, lt, reduction="none", log_target=True).sum(-1).numpy()
    np.testing.assert_allclose(oracle.kl_divergence(zt, zp), ref, rtol=1e-12, atol=1e-14)
    # the reverse direction differs: a swapped argument order would fail the line above
    assert np.max(np.abs(oracle.kl_divergence(zp, zt) - ref)) > 1e-3


@pytest.mark.parametrize("a,b", [(0.3, -1.2), (2.0, 2.5), (-4.0, 1.0)])
def test_kl_and_entropy_two_point_closed_form(a, b):
    p, q = _sigmoid(a), _sigmoid(b)
    kl = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
    h = -p * math.log(p) - (1 - p) * math.log(1 - p)
    assert abs(oracle.kl_divergence(np.array([a, 0.0]), np.array([b, 0.0])) - kl) < 1e-14
    assert abs(oracle.entropy(np.array([a, 0.0])) - h) < 1e-14


def test_kl_invariants():
    rng = np.random.default_rng(32)
    z = rng.standard_normal((50, 64)) * 2
    assert np.max(np.abs(oracle.kl_divergence(z, z))) < 1e-14
    assert np.max(np.abs(oracle.kl_divergence(z + 7.5, z))) < 1e-12  # softmax ignores a shift
    zp = z + rng.standard_normal(z.shape) * 0.3
    assert np.all(oracle.kl_divergence(z, zp) > 0)  # Gibbs' inequality
    np.testing.assert_allclose(oracle.entropy(np.zeros((3, 64))), math.log(64), rtol=1e-14)
    spike = np.zeros(64)
    spike[5] = 1000.0
    assert oracle.entropy(spike) < 1e-12


def test_kl_brute_force_tiny():
    rng = np.random.default_rng(33)
    zt, zp = rng.standard_normal(9), rng.standard_normal(9)
    et, ep = [math.exp(x) for x in zt], [math.exp(x) for x in zp]
    st, sp = sum(et), sum(ep)
    kl = sum((et[v] / st) * math.log((et[v] / st) / (ep[v] / sp)) for v in range(9))
    h = -sum((et[v] / st) * math.log(et[v] / st) for v in range(9))
    assert abs(oracle.kl_divergence(zt, zp) - kl) < 1e-14
    assert abs(oracle.entropy(zt) - h) < 1e-14


def test_kl_lock_semantics():
    rng = np.random.default_rng(34)
    B, N, V = 2, 6, 16
    zp = rng.standard_normal((B, N, V))
    zt = zp + rng.standard_normal((B, N, V)) * np.linspace(0.0, 0.5, N)[None, :, None]
    lock_in = np.zeros((B, N), np.uint8)
    lock_in[1, 2] = 1
    kl = oracle.kl_divergence(zt, zp)
    eps = float(np.median(kl))
    out, klo, ho = oracle.kl_lock(zt, zp, lock_in, eps)
    assert out[1, 2] == 1 and np.isnan(klo[1, 2]) and np.isnan(ho[1, 2])  # permanent, not examined
    act = lock_in == 0
    np.testing.assert_array_equal(out[act], (kl[act] <= eps).astype(np.uint8))
    # inclusive threshold: eps equal to a row's KL locks it
    j = np.argmax(np.where(act, kl, -1))
    out2, _, _ = oracle.kl_lock(zt, zp, lock_in, float(kl.flat[j]))
    assert out2.flat[j] == 1
    # the gate can only keep rows active; h_max = +inf is "off"
    h = oracle.entropy(zt)
    hm = float(np.median(h[act]))
    out3, _, _ = oracle.kl_lock(zt, zp, lock_in, eps, hm)
    np.testing.assert_array_equal(out3[act], ((kl[act] <= eps) & (h[act] <= hm)).astype(np.uint8))
    assert np.all(out3 <= out)


# ---------------------------------------------------------------------------
# RoPE layer variant (reading R8)
# ---------------------------------------------------------------------------
def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(40)
    H, hd, theta = 3, 16, 10000.0
    x = rng.standard_normal((5, H * hd))
    pos = np.array([0, 1, 7, 100, 4095])
    got = oracle.rope(x, pos, H, hd, theta).reshape(5, H, hd)
    z = x.reshape(5, H, hd)
    zc = z[..., : hd // 2] + 1j * z[..., hd // 2:]                      # pair (i, i + hd/2) as a + ib
    w = np.exp(1j * pos[:, None, None] * theta ** (-np.arange(hd // 2) * 2.0 / hd))
    ref = zc * w
    np.testing.assert_allclose(got[..., : hd // 2], ref.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[..., hd // 2:], ref.imag, rtol=0, atol=1e-12)


def test_rope_invariants():
    rng = np.random.default_rng(41)
    H, hd, theta = 2, 8, 500.0
    q, k = rng.standard_normal((1, H * hd)), rng.standard_normal((1, H * hd))
    np.testing.assert_array_equal(oracle.rope(q, [0], H, hd, theta), q)  # position 0: identity
    r = oracle.rope(q, [37], H, hd, theta)
    np.testing.assert_allclose(np.linalg.norm(r.reshape(H, hd), axis=1),
                               np.linalg.norm(q.reshape(H, hd), axis=1), rtol=1e-13)
    # scores depend on the relative position only
    def score(m, n):
        a = oracle.rope(q, [m], H, hd, theta).reshape(H, hd)
        b = oracle.rope(k, [n], H, hd, theta).reshape(H, hd)
        return np.sum(a * b, axis=1)
    np.testing.assert_allclose(score(9, 4), score(109, 104), rtol=0, atol=1e-12)
    assert np.max(np.abs(score(9, 4) - score(4, 9))) > 1e-3


def test_rope_partial_equals_full_and_keeps_locked_rows():
    dims = synth.Dims(B=2, N=7, d=16, H=2, hd=8, F=24, eps=1e-6, dtype="f32", rope_theta=100.0)
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=42)
    full = oracle.full_layer_step(dims, W, X, "f64")
    plain = oracle.full_layer_step(synth.Dims(**{**dims.__dict__, "rope_theta": 0.0}), W, X, "f64")
    assert np.max(np.abs(full.Y - plain.Y)) > 1e-3  # the rotation changes the layer
    np.testing.assert_array_equal(full.V, plain.V)   # and leaves V alone
    idx, seg = oracle.compact(np.zeros((2, 7), np.uint8))
    part = oracle.layer_step_partial(dims, W, X, idx, seg, oracle.LayerState(*(np.zeros_like(full.K),) * 3), "f64")
    for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
        assert np.max(np.abs(a - b)) < 1e-12
    lock = synth.bernoulli_active(2, 7, 0.5, seed=42)
    idx, seg = oracle.compact(lock)
    part = oracle.layer_step_partial(dims, W, X, idx, seg, full, "f64")  # unchanged inputs
    for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
        assert np.max(np.abs(a - b)) < 1e-12


# ---------------------------------------------------------------------------
# grouped-query attention (an optional layer variant): fewer K/V heads than query heads
# ---------------------------------------------------------------------------
def _replicated_mha(dims, W):
    """The MHA layer whose K and V weight rows repeat each K/V head for its group of query heads."""
    d, hd, H, Hkv = dims.d, dims.hd, dims.H, dims.Hkv
    g = H // Hkv
    wq = np.asarray(W["w_qkv"], dtype=np.float64)
    wk = wq[d:d + Hkv * hd].reshape(Hkv, hd, d)
    wv = wq[d + Hkv * hd:].reshape(Hkv, hd, d)
    rep = lambda w: np.repeat(w, g, axis=0).reshape(H * hd, d)
    mdims = _dims(B=dims.B, N=dims.N, d=d, H=H, hd=hd, F=dims.F, rope_theta=dims.rope_theta)
    return mdims, dict(W, w_qkv=np.concatenate([wq[:d], rep(wk), rep(wv)]))


@pytest.mark.parametrize("H,Hkv,theta", [(4, 2, 0.0), (6, 1, 0.0), (6, 3, 100.0), (4, 4, 0.0)])
def test_gqa_equals_mha_with_repeated_kv_heads(H, Hkv, theta):
    hd = 4
    dims = _dims(B=2, N=6, d=H * hd, H=H, hd=hd, F=12, Hkv=Hkv, rope_theta=theta)
    W = _weights(dims, seed=21)
    X = synth.hidden_states(dims, seed=21)
    st = oracle.full_layer_step(dims, W, X, "f64")
    mdims, mW = _replicated_mha(dims, W)
    ref = oracle.full_layer_step(mdims, mW, X, "f64")
    assert st.K.shape == (2, 6, Hkv * hd)
    np.testing.assert_allclose(st.Y, ref.Y, rtol=0, atol=1e-12)
    g = H // Hkv
    heads = lambda z, n: z.reshape(2, 6, n, hd)
    np.testing.assert_allclose(heads(st.K, Hkv), heads(ref.K, H)[:, :, ::g], rtol=0, atol=1e-12)
    np.testing.assert_allclose(heads(st.V, Hkv), heads(ref.V, H)[:, :, ::g], rtol=0, atol=1e-12)
    # the partial step from the full step's caches, a subset active
    lock = synth.bernoulli_active(2, 6, 0.5, seed=22)
    idx, seg = oracle.compact(lock)
    stale = oracle.LayerState(st.K * 0.5, st.V * 2.0, st.Y)
    part = oracle.layer_step_partial(dims, W, X, idx, seg, stale, "f64")
    mstale = oracle.LayerState(np.repeat(heads(stale.K, Hkv), g, axis=2).reshape(2, 6, H * hd),
                               np.repeat(heads(stale.V, Hkv), g, axis=2).reshape(2, 6, H * hd), stale.Y)
    mpart = oracle.layer_step_partial(mdims, mW, X, idx, seg, mstale, "f64")
    np.testing.assert_allclose(part.Y, mpart.Y, rtol=0, atol=1e-12)
    np.testing.assert_allclose(heads(part.K, Hkv), heads(mpart.K, H)[:, :, ::g], rtol=0, atol=1e-12)


def test_gqa_partial_with_all_rows_equals_full_and_keeps_locked_rows():
    dims = _dims(B=2, N=8, d=16, H=4, hd=4, F=12, Hkv=2, rope_theta=50.0)
    W = _weights(dims, seed=23)
    X = synth.hidden_states(dims, seed=23)
    full = oracle.full_layer_step(dims, W, X, "f64")
    idx, seg = oracle.compact(np.zeros((2, 8), np.uint8))
    zero = oracle.LayerState(np.zeros_like(full.K), np.zeros_like(full.V), np.zeros_like(full.Y))
    part = oracle.layer_step_partial(dims, W, X, idx, seg, zero, "f64")
    for a, b in ((part.K, full.K), (part.V, full.V), (part.Y, full.Y)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    lock = synth.bernoulli_active(2, 8, 0.4, seed=24)
    idx, seg = oracle.compact(lock)
    rng = np.random.default_rng(24)
    st = oracle.LayerState(*(rng.standard_normal(a.shape) for a in (full.K, full.V, full.Y)))
    out = oracle.layer_step_partial(dims, W, X, idx, seg, st, "f64")
    locked = lock.astype(bool)
    for new, old in ((out.K, st.K), (out.V, st.V), (out.Y, st.Y)):
        assert _h(new[locked]) == _h(old[locked])


@pytest.mark.parametrize("Hkv", [1, 2])
def test_gqa_flop_count_closed_form(Hkv):
    B, N, d, H, hd, F = 2, 8, 16, 4, 4, 12
    dims = _dims(B=B, N=N, d=d, H=H, hd=hd, F=F, Hkv=Hkv)
    dkv = Hkv * hd
    W = _weights(dims)
    X = synth.hidden_states(dims, seed=25)
    with oracle.count_flops() as cf:
        full = oracle.full_layer_step(dims, W, X, "f64")
    per_row = 2 * d * (d + 2 * dkv) + 2 * d * d + 6 * d * F
    assert cf.flops == B * (N * per_row + 4 * N * N * d)
    lock = synth.bernoulli_active(B, N, 0.5, seed=25)
    idx, seg = oracle.compact(lock)
    with oracle.count_flops() as cp:
        oracle.layer_step_partial(dims, W, X, idx, seg, full, "f64")
    assert cp.flops == idx.size * per_row + 4 * idx.size * N * d


@pytest.mark.parametrize("old,new", [
    ("g = h // (dims.H // kv_heads(dims))", "g = h % kv_heads(dims)"),        # heads dealt round-robin
    ("g = h // (dims.H // kv_heads(dims))", "g = h // kv_heads(dims)"),       # wrong group size
])
def test_gqa_head_mapping_mutants_are_caught(old, new):
    dims = _dims(B=1, N=6, d=24, H=6, hd=4, F=8, Hkv=3)
    W = _weights(dims, seed=26)
    X = synth.hidden_states(dims, seed=26)
    ns = dict(po.__dict__)
    src = textwrap.dedent(inspect.getsource(po._kv_cols))
    assert src.count(old) == 1
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    for f in (po.full_layer_step, po.layer_step_partial):
        exec(compile(textwrap.dedent(inspect.getsource(f)), "<oracle>", "exec"), ns)
    st = ns["full_layer_step"](dims, W, X, "f64")
    _, _, y = torch_block(dims, W, X)
    assert np.max(np.abs(st.Y - y)) > 1e-6
