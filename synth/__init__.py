"""Seeded synthetic inputs for the partial-recompute denoising step.

This module only draws random numbers and rounds them to the storage type of
the workload (fp32 or bf16).  It holds none of the method's arithmetic: no
projection, no score, no lock rule, no layer math.  Both the CPU oracle and the
CUDA path consume what it produces, so both sides see bit-identical inputs.

Random streams: every array is drawn from ``numpy.random.default_rng`` (PCG64)
seeded with the pair ``(seed, stream)``; the stream ids are fixed below so that
adding a new array never shifts the draws of an existing one.

Distributions follow the workloads of the SureLock page (LLaDA-8B shape, one
bidirectional layer, section 4 "Experimental Results") as fixed by the shape
list that accompanies this library: N(mu, var) is read as mean and *variance*.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# stream ids for (seed, stream) seeding
S_WEIGHTS = 0
S_X = 1
S_U = 2
S_MASK = 3
S_NOISE = 4
S_POS = 5
S_PROXY = 6
S_LOGITS = 7
S_CONF = 8


def round_bf16(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even); returns float32 holding it.

    Used only to quantise *inputs* to the storage type of a bf16 workload.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(a)
    if nan.any():
        out[nan] = np.nan
    return out


def _rng(seed: int, stream: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), *[int(e) for e in extra]])


@dataclasses.dataclass(frozen=True)
class Dims:
    """Shape of one layer step: B sequences of N tokens, model dim d = H*hd, FFN dim F."""

    B: int
    N: int
    d: int
    H: int
    hd: int
    F: int
    eps: float = 1e-6
    dtype: str = "bf16"  # "bf16" or "f32"
    rope_theta: float = 0.0  # RoPE base for q and k; 0 = no rotary embedding
    Hkv: int = 0  # K/V heads (grouped-query attention); 0 = one per query head

    def __post_init__(self):
        assert self.d == self.H * self.hd, "d must equal H*hd"
        assert self.Hkv == 0 or (0 < self.Hkv <= self.H and self.H % self.Hkv == 0), "Hkv must divide H"

    @property
    def dkv(self) -> int:
        """Width of the K and V rows: (Hkv or H) * hd."""
        return (self.Hkv or self.H) * self.hd


def _normal(rng, shape, std, dtype):
    if dtype == "f32":
        a = rng.standard_normal(shape, dtype=np.float64) * std
        return a.astype(np.float32)
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return round_bf16(a)


def layer_weights(dims: Dims, std: float, seed: int = 0, layer: int = 0) -> dict:
    """Random-init weights of one layer, nn.Linear layout [out_features, in_features].

    w_qkv [d + 2 dkv, d] (rows 0..d-1 produce Q, then dkv rows K, then dkv rows V;
    dkv = d unless the layer has fewer K/V heads), w_o [d, d],
    w_gu [2F, d] (rows 0..F-1 gate, F..2F-1 up), w_down [d, F]; RMSNorm gains g1, g2
    are ones.  Values are exactly representable in the workload's dtype.
    """
    rng = _rng(seed, S_WEIGHTS, layer)
    d, F, dt = dims.d, dims.F, dims.dtype
    w = {
        "w_qkv": _normal(rng, (d + 2 * dims.dkv, d), std, dt),
        "w_o": _normal(rng, (d, d), std, dt),
        "w_gu": _normal(rng, (2 * F, d), std, dt),
        "w_down": _normal(rng, (d, F), std, dt),
        "g1": np.ones(d, dtype=np.float32),
        "g2": np.ones(d, dtype=np.float32),
    }
    return w


def hidden_states(dims: Dims, seed: int = 0, std: float = 1.0, layer: int = 0) -> np.ndarray:
    """X ~ N(0, std^2), shape [B, N, d], in the workload's dtype (float32 container)."""
    return _normal(_rng(seed, S_X, layer), (dims.B, dims.N, dims.d), std, dims.dtype)


def proxy_basis_draw(d: int, r: int, seed: int = 0) -> np.ndarray:
    """The seeded N(0,1) d x r matrix whose QR factor is the singular-proxy basis.

    Returned in float64; the orthonormalisation (numpy.linalg.qr) is done by
    ``proxy_basis`` below, a library routine applied to the draw.
    """
    return _rng(seed, S_U).standard_normal((d, r))


def proxy_basis(d: int, r: int, seed: int = 0, dtype: str = "bf16") -> np.ndarray:
    """U^T, shape [r, d]: r orthonormal directions (rows), rounded to the dtype.

    The draw is orthonormalised by numpy's QR (Householder); rows of the result
    are the columns of the Q factor.  bf16 rounding makes them orthonormal only
    to ~2^-9.
    """
    q, _ = np.linalg.qr(proxy_basis_draw(d, r, seed))
    ut = np.ascontiguousarray(q.T)
    return ut.astype(np.float32) if dtype == "f32" else round_bf16(ut.astype(np.float32))


def bernoulli_active(B: int, N: int, p_active: float, seed: int = 0) -> np.ndarray:
    """Initial lock mask (uint8, 1 = locked): each row is active with probability p_active."""
    u = _rng(seed, S_MASK).random((B, N))
    return (u >= p_active).astype(np.uint8)


def step_noise(shape, var: float, seed: int = 0, step: int = 0, dtype: str = "f32") -> np.ndarray:
    """Per-step perturbation eps ~ N(0, var) for all rows; the caller applies it to active rows."""
    rng = _rng(seed, S_NOISE, step)
    a = rng.standard_normal(shape, dtype=np.float64) * math.sqrt(var)
    return a.astype(np.float32)


def perturb_rows(X: np.ndarray, eps: np.ndarray, rows_mask: np.ndarray, dtype: str) -> np.ndarray:
    """Harness data prep: X + eps on the masked rows, stored back in the workload dtype."""
    out = X.copy()
    m = rows_mask.astype(bool)
    out[m] = (X[m].astype(np.float32) + eps[m].astype(np.float32)).astype(np.float32)
    if dtype == "bf16":
        out = round_bf16(out)
    return out


def uniform_positions(lo: int, hi: int, count: int, seed: int = 0, tag: int = 0) -> np.ndarray:
    """`count` distinct positions drawn uniformly from [lo, hi), sorted ascending."""
    rng = _rng(seed, S_POS, tag)
    return np.sort(rng.choice(np.arange(lo, hi), size=count, replace=False)).astype(np.int64)


def geometric_block_m(num_blocks: int, p: float = 1.0 / 64.0, lo: int = 32, cap: int = 480,
                      seed: int = 0) -> np.ndarray:
    """Long-context block decode: M = lo + min(G, cap), G ~ Geometric(p) on {0,1,...}."""
    rng = _rng(seed, S_POS, 4)
    g = rng.geometric(p, size=num_blocks) - 1  # numpy's geometric is on {1,2,...}
    return (lo + np.minimum(g, cap)).astype(np.int64)


def linear_schedule(N: int, steps: int = 256) -> np.ndarray:
    """Integer, vocabulary-free active-count schedule decaying linearly from N to floor(N/20)."""
    t = np.arange(steps, dtype=np.int64)
    return N - (t * (N - N // 20)) // (steps - 1)


# ---------------------------------------------------------------------------
# Named workloads (shapes and distributions of the pages' experiments)
# ---------------------------------------------------------------------------
def logits_pair(B: int, N: int, V: int, seed: int = 0, std: float = 2.0, drift=(0.0, 0.3),
                dtype: str = "f32"):
    """Two steps of vocabulary logits [B, N, V]: z_prev ~ N(0, std^2) per entry, and
    z_t = z_prev + N(0, s_i^2) with s_i spread uniformly over `drift` across rows, so that
    some rows barely move and others change a lot.  Rounded to bf16 for "bf16"."""
    rng = _rng(seed, S_LOGITS)
    zp = rng.standard_normal((B, N, V)).astype(np.float32) * np.float32(std)
    s = np.linspace(drift[0], drift[1], B * N, dtype=np.float32).reshape(B, N, 1)
    zt = zp + rng.standard_normal((B, N, V)).astype(np.float32) * s
    if dtype == "bf16":
        return round_bf16(zt), round_bf16(zp)
    return zt, zp


def span_confidences(B: int, N: int, step: int, seed: int = 0, prompt: int = 0, rate: float = 16.0,
                     width: float = 24.0, noise: float = 0.75, levels: int = 256) -> np.ndarray:
    """Per-position confidences [B, N] fp32 in [0, 1] at decoding step `step`.

    A confident region grows from the prompt end by about `rate` positions a
    step (each sequence with its own jitter): position i gets the logistic of
    (front - i) / width plus N(0, noise^2) per position, which leaves
    scattered confident positions ahead of the front and doubtful ones behind
    it.  Values are rounded to multiples of 1/levels so that equal confidences
    occur (ties).
    """
    rng = _rng(seed, S_CONF, step)
    i = np.arange(N, dtype=np.float64)
    front = prompt + rate * (step + 1) + rng.normal(0.0, 4.0, size=(B, 1))
    z = (front - i[None, :]) / width + rng.normal(0.0, noise, size=(B, N))
    c = 1.0 / (1.0 + np.exp(-z))
    return (np.round(c * levels) / levels).astype(np.float32)


def generation_mask(B: int, N: int, prompt: int) -> np.ndarray:
    """masked [B, N] u8: the prompt (first `prompt` positions) is given, the rest is masked."""
    m = np.ones((B, N), dtype=np.uint8)
    m[:, :prompt] = 0
    return m


# vocabulary size of the 8B model the pages name, for the KL-lock measurement
VOCAB_8B = 126464


TINY = Dims(B=1, N=64, d=64, H=4, hd=16, F=256, eps=1e-6, dtype="f32")
LAYER_8B = Dims(B=1, N=1024, d=4096, H=32, hd=128, F=12288, eps=1e-6, dtype="bf16")
STACK_8B = Dims(B=4, N=2048, d=4096, H=32, hd=128, F=12288, eps=1e-6, dtype="bf16")
LONG_8B = Dims(B=1, N=8192, d=4096, H=32, hd=128, F=12288, eps=1e-6, dtype="bf16")
SCORE_8B = Dims(B=8, N=4096, d=4096, H=32, hd=128, F=12288, eps=1e-6, dtype="bf16")

TINY_RANK = 8
TINY_TAU = 0.99
TINY_STEPS = 20
TINY_NOISE_VAR = 0.01
TINY_P_ACTIVE = 0.25
LAYER_8B_WSTD = 0.02
LAYER_8B_FRACTIONS = (1.0, 0.5, 0.25, 0.1, 0.05)
PROXY_RANK_8B = 128
SCORE_PCTS = (5, 10, 20)


def active_count(N: int, frac: float) -> int:
    """M = floor(frac * N) (1024 -> 1024/512/256/102/51)."""
    return int(math.floor(frac * N + 1e-9))


def layer_8b_positions(N: int, frac: float, seed: int = 0) -> np.ndarray:
    """Active positions of the single 8B-shape layer: all N at frac = 1, else uniform over the
    generated half [N/2, N)."""
    M = active_count(N, frac)
    if M >= N:
        return np.arange(N, dtype=np.int64)
    return uniform_positions(N // 2, N, M, seed=seed, tag=int(round(frac * 1000)))
