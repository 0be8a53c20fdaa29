"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the oracle is float64; see the design notes for the derivation):
  * integer work (lock masks, active indices, segment pointers): bit-exact;
  * fp32 workloads: max_i |g_i - o_i| / max(|o_i|, rms(o)) <= 1e-4;
  * bf16 workloads: the same max relative error <= 2e-2, and the mean absolute
    error mean_i |g_i - o_i| <= 1e-3 in the tensor's own units (no rescaling).
    Both sides hold bf16 values here: the oracle's bf16 policy rounds exactly
    the tensors the layer stores in bf16 (the K/V cache rows and Y), so a
    difference is a whole number of bf16 steps of the element.
"""
import numpy as np
import torch

BF16_MAX_REL = 2e-2
BF16_MAE = 1e-3
F32_MAX_REL = 1e-4


def metrics(g, o):
    """(max relative error with the rms floor, mean absolute error, mean absolute error / rms(o))."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    if o.size == 0:
        return 0.0, 0.0, 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    floor = np.maximum(np.abs(o), rms if rms > 0 else 1.0)
    err = np.abs(g - o)
    max_rel = float(np.max(err / floor))
    mae = float(np.mean(err))
    return max_rel, mae, mae / (rms if rms > 0 else 1.0)


def assert_bf16_close(g, o, what):
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    mr, mae, mrel = metrics(g, o)
    assert mr <= BF16_MAX_REL and mae <= BF16_MAE, f"{what}: max_rel {mr:.3e} mae {mae:.3e} (mae/rms {mrel:.3e})"
    return mr, mae


def assert_f32_close(g, o, what, tol=F32_MAX_REL):
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    mr, _, _ = metrics(g, o)
    assert mr <= tol, f"{what}: max_rel {mr:.3e} > {tol}"
    return mr


def dev(a, dtype):
    """Upload a numpy array (exact values of `dtype`) to the GPU."""
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype).contiguous()


def host(t):
    return t.detach().to(torch.float64).cpu().numpy() if t.dtype.is_floating_point else t.cpu().numpy()


def tdtype(dims):
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


def weights_dev(W, dims):
    dt = tdtype(dims)
    return {k: dev(v, dt) for k, v in W.items()}
