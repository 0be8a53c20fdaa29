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


class Guarded:
    """A device tensor with guard bands of a known byte pattern on both sides.

    compute-sanitizer is not available to these tests, so a write past either end
    of a buffer would go unseen; the guard bands catch it: ``check()`` asserts
    that every guard byte still holds the pattern.  The tensor starts at a
    4096-byte offset into its allocation (alignment kept for TMA and vector
    accesses)."""

    PATTERN = 0xA5
    GUARD = 4096

    def __init__(self, shape, dtype, init=None, fill=None, device="cuda"):
        shape = tuple(int(s) for s in shape)
        n = int(np.prod(shape)) if shape else 1
        esize = torch.empty((), dtype=dtype).element_size()
        self.nbytes = n * esize
        body = (self.nbytes + 1023) // 1024 * 1024
        self.raw = torch.full((2 * self.GUARD + body,), self.PATTERN, dtype=torch.uint8, device=device)
        self.t = self.raw[self.GUARD:self.GUARD + self.nbytes].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init if isinstance(init, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(init)))
        elif fill is not None:
            self.t.fill_(fill)

    def check(self, what):
        if self.raw.is_cuda:
            torch.cuda.synchronize()
        head = self.raw[:self.GUARD]
        tail = self.raw[self.GUARD + self.nbytes:]
        bad_h = int((head != self.PATTERN).sum())
        bad_t = int((tail != self.PATTERN).sum())
        assert bad_h == 0 and bad_t == 0, f"{what}: {bad_h} guard bytes before and {bad_t} after the tensor changed"


def check_guards(guards, what):
    for name, g in guards.items():
        g.check(f"{what}: {name}")


def guarded_workspace(plk, dm):
    n = plk.workspace_bytes(dm)
    if n == 0:
        raise plk.PlkError(plk.ERR_SHAPE, "workspace_bytes")
    return Guarded((n,), torch.uint8)
