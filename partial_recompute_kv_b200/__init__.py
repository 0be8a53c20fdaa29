"""Python binding of the partial-recompute K/V library (libplk.so, sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (contiguous); calls are asynchronous on
torch's current stream unless ``stream`` is given.  There is no CPU fallback:
importing this module fails if the compiled library is missing.

The C contract of every call is documented in include/plk.h.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libplk.so")

OK, ERR_ARG, ERR_SHAPE, ERR_DTYPE, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5, -6
F32, BF16 = 0, 1
METRIC_COS, METRIC_L2 = 0, 1
SEL_THRESH_GT, SEL_THRESH_LT, SEL_TOPK_LARGEST, SEL_TOPK_SMALLEST = 0, 1, 2, 3

EXPORTED = (
    "plk_score_drift", "plk_select_active", "plk_layer_step_partial", "plk_full_layer_step",
    "plk_proxy_commit", "plk_layer_step_partial_static", "plk_kl_lock", "plk_slowfast_step", "plk_workspace_bytes",
    "plk_denoise_step", "plk_denoise_step_host", "plk_step_workspace_bytes", "plk_denoise_steps_host",
    "plk_steps_workspace_bytes",
    "plk_get_status",
    "plk_set_wait_limit", "plk_set_deterministic",
    "plk_selftest_wait_timeout", "plk_selftest_exp2", "plk_trace_events", "plk_error_string", "plk_version",
)


class PlkDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int), ("H", ctypes.c_int),
                ("hd", ctypes.c_int), ("F", ctypes.c_int), ("eps", ctypes.c_float), ("dtype", ctypes.c_int),
                ("rope_theta", ctypes.c_float), ("Hkv", ctypes.c_int)]


class PlkWeights(ctypes.Structure):
    _fields_ = [("g1", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p),
                ("g2", ctypes.c_void_p), ("w_gu", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


SF_HIST_MAX = 16
SF_STATE_WORDS = 4 + SF_HIST_MAX  # plk_sf_state: phase, s, e, nslow, hist[16] (int32)


class PlkSfParams(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int), ("w_hist", ctypes.c_int), ("k_max", ctypes.c_int),
                ("tau_conv", ctypes.c_float), ("tau_high", ctypes.c_float), ("var_stable", ctypes.c_float)]


class PlkError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {error_string(code)} ({code})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m partial_recompute_kv_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S, F, L, V = (ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_longlong,
                        ctypes.POINTER(PlkDims))
    W = ctypes.POINTER(PlkWeights)
    sig = {
        "plk_score_drift": (I, [V, P, P, I, P, I, P, P, P]),
        "plk_select_active": (I, [V, P, P, P, I, F, I, P, P, P]),
        "plk_layer_step_partial": (I, [V, W, P, P, P, P, P, P, P, S, P]),
        "plk_full_layer_step": (I, [V, W, P, P, P, P, P, S, P]),
        "plk_layer_step_partial_static": (I, [V, W, P, P, P, P, P, P, P]),
        "plk_proxy_commit": (I, [V, I, P, P, P, P, P]),
        "plk_kl_lock": (I, [V, I, P, P, P, P, F, F, P, P, P]),
        "plk_slowfast_step": (I, [V, ctypes.POINTER(PlkSfParams), P, P, P, P, P, P]),
        "plk_workspace_bytes": (S, [V]),
        "plk_denoise_step": (I, [V, W, P, I, I, I, F, I, P, P, P, P, P, P, P, S, P]),
        "plk_denoise_step_host": (I, [V, W, P, I, I, I, F, I, P, P, P, P, P, P, P, P, S, P]),
        "plk_step_workspace_bytes": (S, [V, I]),
        "plk_denoise_steps_host": (I, [V, W, P, I, I, I, F, I, P, P, P, P, P, I, ctypes.POINTER(P),
                                       ctypes.POINTER(P), P, S, P, P, P]),
        "plk_steps_workspace_bytes": (S, [V, I]),
        "plk_get_status": (I, [P]),
        "plk_set_wait_limit": (I, [L]),
        "plk_set_deterministic": (I, [I]),
        "plk_selftest_wait_timeout": (I, [P]),
        "plk_selftest_exp2": (I, [P, P, I, P]),
        "plk_trace_events": (I, [ctypes.POINTER(ctypes.c_void_p), I]),
        "plk_error_string": (ctypes.c_char_p, [I]),
        "plk_version": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _Lib:
    """The loaded libplk.so, opened on first use (so that the in-package build
    script can run before the library exists).  Raises ImportError if the
    library is missing: there is no fallback."""

    _cdll = None

    def __getattr__(self, name):
        if _Lib._cdll is None:
            _Lib._cdll = _load()
        return getattr(_Lib._cdll, name)


lib = _Lib()


def load():
    """Open the library now (raises ImportError if it is missing)."""
    return lib.plk_version()


def error_string(code: int) -> str:
    return lib.plk_error_string(int(code)).decode()


def version() -> int:
    return lib.plk_version()


def _check(code, where):
    if code != OK:
        raise PlkError(code, where)


def dims(B, N, d, H, hd, F, eps=1e-6, dtype=BF16, rope_theta=0.0, Hkv=0) -> PlkDims:
    """Layer shape; Hkv > 0 selects grouped-query attention with Hkv K/V heads (K/V rows Hkv*hd wide)."""
    return PlkDims(int(B), int(N), int(d), int(H), int(hd), int(F), float(eps), int(dtype), float(rope_theta),
                   int(Hkv))


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def weights(w: dict) -> PlkWeights:
    return PlkWeights(*(_ptr(w[k]) for k in ("g1", "w_qkv", "w_o", "g2", "w_gu", "w_down")))


def workspace_bytes(dm: PlkDims) -> int:
    return int(lib.plk_workspace_bytes(ctypes.byref(dm)))


def score_drift(dm, X, Ut, r, proxy_cache, metric, score_out, proxy_out=None, stream=None):
    _check(lib.plk_score_drift(ctypes.byref(dm), _ptr(X), _ptr(Ut), int(r), _ptr(proxy_cache), int(metric),
                               _ptr(proxy_out), _ptr(score_out), _stream(stream)), "score_drift")


def select_active(dm, score, lock_in, lock_out, mode, tau, k, idx_out, seg_ptr, stream=None):
    _check(lib.plk_select_active(ctypes.byref(dm), _ptr(score), _ptr(lock_in), _ptr(lock_out), int(mode),
                                 float(tau), int(k), _ptr(idx_out), _ptr(seg_ptr), _stream(stream)),
           "select_active")


def layer_step_partial(dm, w, X, idx, seg_ptr, K_cache, V_cache, Y, workspace, stream=None):
    pw = w if isinstance(w, PlkWeights) else weights(w)
    _check(lib.plk_layer_step_partial(ctypes.byref(dm), ctypes.byref(pw), _ptr(X), _ptr(idx), _ptr(seg_ptr),
                                      _ptr(K_cache), _ptr(V_cache), _ptr(Y), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "layer_step_partial")


STATIC_WS_BYTES = 32 << 20


def layer_step_partial_static(dm, w, X, idx, seg_ptr, K_cache, V_cache, Y, stream=None):
    """layer_step_partial with the library's own device-array scratch (no workspace,
    no allocation); see plk_layer_step_partial_static in include/plk.h."""
    pw = w if isinstance(w, PlkWeights) else weights(w)
    _check(lib.plk_layer_step_partial_static(ctypes.byref(dm), ctypes.byref(pw), _ptr(X), _ptr(idx),
                                             _ptr(seg_ptr), _ptr(K_cache), _ptr(V_cache), _ptr(Y),
                                             _stream(stream)), "layer_step_partial_static")


def _hptr(t):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise ValueError("host buffers must be contiguous CPU tensors (pinned for asynchronous copies)")
    return ctypes.c_void_p(t.data_ptr())


def step_workspace_bytes(dm, r) -> int:
    return int(lib.plk_step_workspace_bytes(ctypes.byref(dm), int(r)))


def alloc_step_workspace(dm, r, device="cuda"):
    n = step_workspace_bytes(dm, r)
    if n == 0:
        raise PlkError(ERR_SHAPE, "step_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def denoise_step(dm, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X, workspace,
                 stream=None):
    """The whole step on device buffers (see plk_denoise_step): score, select (lock in place),
    layer step with the proxy refresh folded in."""
    pw = w if isinstance(w, PlkWeights) else weights(w)
    _check(lib.plk_denoise_step(ctypes.byref(dm), ctypes.byref(pw), _ptr(Ut), int(r), int(metric), int(mode),
                                float(tau), int(k), _ptr(proxy_cache), _ptr(lock), _ptr(K_cache), _ptr(V_cache),
                                _ptr(Y), _ptr(X), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)), "denoise_step")


def denoise_step_host(dm, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X_host, Y_host,
                      workspace, stream=None):
    """The whole step from host memory (see plk_denoise_step_host): X_host -> device, score, select,
    layer step, proxy refresh, Y -> Y_host.  X_host / Y_host are CPU tensors (pinned)."""
    pw = w if isinstance(w, PlkWeights) else weights(w)
    _check(lib.plk_denoise_step_host(ctypes.byref(dm), ctypes.byref(pw), _ptr(Ut), int(r), int(metric), int(mode),
                                     float(tau), int(k), _ptr(proxy_cache), _ptr(lock), _ptr(K_cache),
                                     _ptr(V_cache), _ptr(Y), _hptr(X_host), _hptr(Y_host), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "denoise_step_host")


def steps_workspace_bytes(dm, r) -> int:
    return int(lib.plk_steps_workspace_bytes(ctypes.byref(dm), int(r)))


def alloc_steps_workspace(dm, r, device="cuda"):
    n = steps_workspace_bytes(dm, r)
    if n == 0:
        raise PlkError(ERR_SHAPE, "steps_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def denoise_steps_host(dm, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X_hosts,
                       Y_hosts, workspace, upload_stream, download_stream, stream=None):
    """len(X_hosts) consecutive whole steps from host memory (see plk_denoise_steps_host): step t
    reads X_hosts[t] and leaves Y after it in Y_hosts[t]; the uploads and downloads run on
    upload_stream / download_stream (torch.cuda.Stream) beside the compute on `stream`.  Host
    tensors are CPU tensors (pinned)."""
    if len(X_hosts) != len(Y_hosts):
        raise ValueError("X_hosts and Y_hosts differ in length")
    pw = w if isinstance(w, PlkWeights) else weights(w)
    T = len(X_hosts)
    xs = (ctypes.c_void_p * T)(*(_hptr(x) for x in X_hosts))
    ys = (ctypes.c_void_p * T)(*(_hptr(y) for y in Y_hosts))
    _check(lib.plk_denoise_steps_host(ctypes.byref(dm), ctypes.byref(pw), _ptr(Ut), int(r), int(metric), int(mode),
                                      float(tau), int(k), _ptr(proxy_cache), _ptr(lock), _ptr(K_cache),
                                      _ptr(V_cache), _ptr(Y), T, xs, ys, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream),
                                      _stream(upload_stream), _stream(download_stream)),
           "denoise_steps_host")


def full_layer_step(dm, w, X, K_cache, V_cache, Y, workspace, stream=None):
    pw = w if isinstance(w, PlkWeights) else weights(w)
    _check(lib.plk_full_layer_step(ctypes.byref(dm), ctypes.byref(pw), _ptr(X), _ptr(K_cache), _ptr(V_cache),
                                   _ptr(Y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "full_layer_step")


def proxy_commit(dm, r, idx, seg_ptr, proxy_new, proxy_cache, stream=None):
    _check(lib.plk_proxy_commit(ctypes.byref(dm), int(r), _ptr(idx), _ptr(seg_ptr), _ptr(proxy_new),
                                _ptr(proxy_cache), _stream(stream)), "proxy_commit")


def kl_lock(dm, V, logits_t, logits_prev, lock_in, lock_out, eps, h_max=math.inf, kl_out=None, h_out=None,
            stream=None):
    opt = lambda t: None if t is None else _ptr(t)
    _check(lib.plk_kl_lock(ctypes.byref(dm), int(V), _ptr(logits_t), _ptr(logits_prev), _ptr(lock_in),
                           _ptr(lock_out), float(eps), float(h_max), opt(kl_out), opt(h_out), _stream(stream)),
           "kl_lock")


def sf_params(k=1, w_hist=2, k_max=8, tau_conv=0.5, tau_high=0.9, var_stable=1.0) -> PlkSfParams:
    return PlkSfParams(int(k), int(w_hist), int(k_max), float(tau_conv), float(tau_high), float(var_stable))


def sf_state(B, device="cuda"):
    """Initial SlowFast state of B sequences: int32 [B, SF_STATE_WORDS] zeros (plk_sf_state rows)."""
    return torch.zeros((int(B), SF_STATE_WORDS), dtype=torch.int32, device=device)


def slowfast_step(dm, params, conf, masked, state, unmask_out=None, lock_out=None, stream=None):
    """One SlowFast decoding step: conf [B, N] fp32, masked [B, N] uint8 (in/out),
    state int32 [B, SF_STATE_WORDS] (in/out); unmask_out / lock_out [B, N] uint8 or None."""
    if state.dtype != torch.int32 or state.shape[-1] != SF_STATE_WORDS:
        raise ValueError("state must be int32 [B, %d]" % SF_STATE_WORDS)
    _check(lib.plk_slowfast_step(ctypes.byref(dm), ctypes.byref(params), _ptr(conf), _ptr(masked), _ptr(state),
                                 _ptr(unmask_out), _ptr(lock_out), _stream(stream)), "slowfast_step")


def get_status(stream=None) -> int:
    return int(lib.plk_get_status(_stream(stream)))


def set_wait_limit(cycles: int):
    _check(lib.plk_set_wait_limit(int(cycles)), "set_wait_limit")


def set_deterministic(on: bool):
    _check(lib.plk_set_deterministic(1 if on else 0), "set_deterministic")


def trace_events(events):
    """Register torch.cuda.Event objects (timing enabled) to be recorded between the
    layer step's kernels; an empty list unregisters.  Each event is recorded once
    first so that its CUDA handle exists."""
    handles = []
    for e in events:
        if e.cuda_event == 0:
            e.record()
        handles.append(e.cuda_event)
    arr = (ctypes.c_void_p * max(len(handles), 1))(*handles)
    _check(lib.plk_trace_events(arr, len(handles)), "trace_events")


def selftest_wait_timeout(stream=None):
    _check(lib.plk_selftest_wait_timeout(_stream(stream)), "selftest_wait_timeout")


def selftest_exp2(t, out, stream=None):
    """out = 2^t by the attention softmax's FMA-pipe exponential (fp32 tensors of equal size)."""
    if t.dtype != torch.float32 or out.dtype != torch.float32 or t.numel() != out.numel():
        raise ValueError("t and out must be float32 tensors of the same size")
    _check(lib.plk_selftest_exp2(_ptr(t), _ptr(out), int(t.numel()), _stream(stream)), "selftest_exp2")


def alloc_workspace(dm, device="cuda"):
    n = workspace_bytes(dm)
    if n == 0:
        raise PlkError(ERR_SHAPE, "workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)
