"""The layer-step entry point that allocates nothing (plk_layer_step_partial_static).

It exists for callers that cannot call cudaMalloc -- e.g. code inside a
global-mode stream capture, real-time paths, or plugins whose host runtime owns
every device allocation -- and keeps its scratch in a device array inside the
library.  These tests call it through the C ABI twice in a row, on two
different inputs, and check each result against plk_layer_step_partial run with
a caller workspace on the same input.  The shared array keeps the previous
call's contents, so the second call also shows that nothing stale leaks in.
This file is collected last on purpose.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import assert_bf16_close, assert_f32_close, dev, host, weights_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plk():
    import partial_recompute_kv_b200 as m
    return m


CASES = [
    ("bf16", synth.Dims(B=1, N=256, d=512, H=4, hd=128, F=1536, dtype="bf16"), 0.02, 0.3),
    ("f32", synth.TINY, None, 0.25),
]


@pytest.mark.parametrize("name,D,std,p_active", CASES, ids=[c[0] for c in CASES])
def test_static_entry_matches_workspace_entry_twice(plk, name, D, std, p_active):
    dm = plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16 if D.dtype == "bf16" else plk.F32)
    assert 0 < plk.workspace_bytes(dm) <= plk.STATIC_WS_BYTES
    dt = torch.bfloat16 if D.dtype == "bf16" else torch.float32
    W = synth.layer_weights(D, std if std else 1.0 / math.sqrt(D.d), seed=21)
    Wd = weights_dev(W, D)
    rng = np.random.default_rng(21)
    caches = [rng.standard_normal((D.B, D.N, D.d)).astype(np.float32) for _ in range(3)]
    if D.dtype == "bf16":
        caches = [synth.round_bf16(c) for c in caches]
    lock = synth.bernoulli_active(D.B, D.N, p_active, seed=21)
    idx, seg = oracle.compact(lock)
    idx_d = torch.full((D.B * D.N,), -1, dtype=torch.int32, device="cuda")
    idx_d[: idx.size] = torch.from_numpy(idx.astype(np.int32)).cuda()
    seg_d = torch.from_numpy(seg.astype(np.int32)).cuda()
    inputs = [dev(synth.hidden_states(D, seed=s), dt) for s in (22, 23)]
    check = assert_bf16_close if D.dtype == "bf16" else assert_f32_close

    def run(static, X):
        K, V, Y = (dev(c, dt) for c in caches)
        if static:
            plk.layer_step_partial_static(dm, Wd, X, idx_d, seg_d, K, V, Y)
        else:
            plk.layer_step_partial(dm, Wd, X, idx_d, seg_d, K, V, Y, plk.alloc_workspace(dm))
        assert plk.get_status() == plk.OK
        return host(K), host(V), host(Y)

    refs = [run(False, X) for X in inputs]
    for call, X in enumerate(inputs):  # two calls in a row through the static entry point
        got = run(True, X)
        for g, r, what in zip(got, refs[call], "KVY"):
            check(g, r, f"static call {call + 1}: {what}")
            if D.dtype == "bf16" and what in "KV":  # the same kernels, QKV sums in a fixed order
                assert np.array_equal(g, r), f"static call {call + 1}: {what} differs bitwise"


def test_static_entry_rejects_dims_beyond_the_limit(plk):
    D = synth.LAYER_8B  # needs far more scratch than the array holds
    dm = plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16)
    assert plk.workspace_bytes(dm) > plk.STATIC_WS_BYTES
    t = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(8, dtype=torch.int32, device="cuda")
    w = {k: t for k in ("g1", "w_qkv", "w_o", "g2", "w_gu", "w_down")}
    with pytest.raises(plk.PlkError) as e:
        plk.layer_step_partial_static(dm, w, t, i, i, t, t, t)
    assert e.value.code == plk.ERR_WORKSPACE
    assert plk.get_status() == plk.OK
