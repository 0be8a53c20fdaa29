"""The C-ABI library loads and exports every entry point declared in include/plk.h.

Runs without a GPU: only symbol lookup and host-side argument validation (which
returns before any CUDA call) are exercised.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "plk.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(plk_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def built():
    from partial_recompute_kv_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("plk_score_drift", "plk_select_active", "plk_layer_step_partial", "plk_full_layer_step"):
        assert required in names


def test_library_exports_every_declared_symbol(built):
    lib = ctypes.CDLL(built)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol(built):
    import partial_recompute_kv_b200 as plk
    assert sorted(plk.EXPORTED) == declared_functions()


def test_host_validation_without_gpu(built):
    import partial_recompute_kv_b200 as plk
    lib = plk.lib
    assert plk.version() == 100
    assert plk.error_string(plk.ERR_TIMEOUT) == "device wait exceeded its limit"
    # null dims / bad enums / bad shapes are rejected before any CUDA call
    assert lib.plk_score_drift(None, None, None, 8, None, 0, None, None, None) == plk.ERR_ARG
    bad_dtype = plk.dims(1, 8, 64, 4, 16, 64, dtype=7)
    assert lib.plk_score_drift(ctypes.byref(bad_dtype), None, None, 8, None, 0, None, None, None) == plk.ERR_DTYPE
    bad_hd = plk.dims(1, 8, 512, 8, 64, 256, dtype=plk.BF16)  # bf16 needs hd == 128
    assert lib.plk_full_layer_step(ctypes.byref(bad_hd), None, None, None, None, None, None, 0, None) == \
        plk.ERR_SHAPE
    bad_width = plk.dims(1, 8, 384, 3, 128, 256, dtype=plk.BF16)  # bf16 needs d % 256 == 0
    assert lib.plk_workspace_bytes(ctypes.byref(bad_width)) == 0
    bad_ffn = plk.dims(1, 8, 512, 4, 128, 320, dtype=plk.BF16)  # bf16 needs F % 128 == 0
    assert lib.plk_workspace_bytes(ctypes.byref(bad_ffn)) == 0
    bad_split = plk.dims(1, 8, 64, 3, 16, 64, dtype=plk.F32)  # d != H * hd
    assert lib.plk_workspace_bytes(ctypes.byref(bad_split)) == 0
    # grouped-query attention: 0 <= Hkv <= H and H % Hkv == 0 (checked before the null weights)
    for hkv, code in ((3, plk.ERR_SHAPE), (8, plk.ERR_SHAPE), (-1, plk.ERR_SHAPE), (2, plk.ERR_ARG),
                      (1, plk.ERR_ARG), (4, plk.ERR_ARG), (0, plk.ERR_ARG)):
        g = plk.dims(1, 8, 64, 4, 16, 64, dtype=plk.F32, Hkv=hkv)
        assert lib.plk_full_layer_step(ctypes.byref(g), None, None, None, None, None, None, 0, None) == code, hkv
    ok = plk.dims(2, 8, 64, 4, 16, 64, dtype=plk.F32)
    p = ctypes.c_void_p(16)
    assert lib.plk_select_active(ctypes.byref(ok), p, p, p, 9, 0.5, 1, p, p, None) == plk.ERR_ARG
    assert lib.plk_select_active(ctypes.byref(ok), p, p, p, plk.SEL_TOPK_LARGEST, 0.5, -1, p, p, None) == \
        plk.ERR_ARG
    assert lib.plk_score_drift(ctypes.byref(ok), p, p, 300, p, 0, None, p, None) == plk.ERR_ARG
    assert lib.plk_score_drift(ctypes.byref(ok), p, p, 8, p, 5, None, p, None) == plk.ERR_ARG
    assert lib.plk_score_drift(ctypes.byref(ok), p, p, 8, p, 0, p, p, None) == plk.ERR_ARG  # out aliases cache
    # base addresses the kernels read with 16-byte vectors or TMA must be 16-byte aligned
    odd, p48 = ctypes.c_void_p(24), ctypes.c_void_p(48)
    for args in ((odd, p, p, None), (p, odd, p, None), (p, p, odd, None), (p, p, p48, odd)):
        X, U, pc, po = args
        assert lib.plk_score_drift(ctypes.byref(ok), X, U, 8, pc, 0, po, p, None) == plk.ERR_ARG, args
    w_ok = plk.PlkWeights(*(16 * (i + 1) for i in range(6)))
    for i in range(6):
        w_bad = plk.PlkWeights(*(16 * (j + 1) + (8 if j == i else 0) for j in range(6)))
        assert lib.plk_full_layer_step(ctypes.byref(ok), ctypes.byref(w_bad), p, p, p, p, None, 0, None) == \
            plk.ERR_ARG, i
    for pos in range(4):  # X, K_cache, V_cache, Y
        a = [p, p, p, p]
        a[pos] = odd
        assert lib.plk_full_layer_step(ctypes.byref(ok), ctypes.byref(w_ok), *a, None, 0, None) == plk.ERR_ARG, pos
        assert lib.plk_layer_step_partial(ctypes.byref(ok), ctypes.byref(w_ok), a[0], p, p, *a[1:], None, 0,
                                          None) == plk.ERR_ARG, pos
    assert lib.plk_layer_step_partial(ctypes.byref(ok), ctypes.byref(w_ok), p, ctypes.c_void_p(18), p, p, p, p,
                                      None, 0, None) == plk.ERR_ARG  # idx on a 2-byte boundary
    # the pipelined steps: T >= 1 and a host buffer for every step's X and Y
    hs = (ctypes.c_void_p * 2)(16, 32)
    hole = (ctypes.c_void_p * 2)(16, None)
    steps = lib.plk_denoise_steps_host
    for T, xs, ys in ((0, hs, hs), (2, None, hs), (2, hs, None), (2, hole, hs), (2, hs, hole)):
        assert steps(ctypes.byref(ok), ctypes.byref(w_ok), p, 8, 0, plk.SEL_TOPK_LARGEST, 0.0, 1, p, p, p, p, p, T,
                     xs, ys, p, 1 << 30, None, None, None) == plk.ERR_ARG, (T, xs, ys)
    assert lib.plk_steps_workspace_bytes(ctypes.byref(bad_width), 8) == 0
    assert lib.plk_set_wait_limit(0) == plk.ERR_ARG
    assert lib.plk_set_deterministic(2) == plk.ERR_ARG
    assert lib.plk_set_deterministic(0) == plk.OK
    assert lib.plk_proxy_commit(ctypes.byref(ok), 0, p, p, p, p, None) == plk.ERR_ARG
    # SlowFast policy: bad params, shapes and aliasing are refused before any launch
    q = ctypes.c_void_p(32)
    sfp = plk.sf_params()
    assert lib.plk_slowfast_step(ctypes.byref(ok), None, p, p, p, None, None, None) == plk.ERR_ARG
    assert lib.plk_slowfast_step(ctypes.byref(ok), ctypes.byref(sfp), None, p, p, None, None, None) == plk.ERR_ARG
    for bad in (dict(k=0), dict(w_hist=0), dict(w_hist=plk.SF_HIST_MAX + 1), dict(k_max=0),
                dict(tau_conv=float("nan")), dict(tau_high=float("nan")), dict(var_stable=float("nan"))):
        bp = plk.sf_params(**bad)
        assert lib.plk_slowfast_step(ctypes.byref(ok), ctypes.byref(bp), p, q, p, None, None, None) == \
            plk.ERR_ARG, bad
    assert lib.plk_slowfast_step(ctypes.byref(ok), ctypes.byref(sfp), p, q, p, q, None, None) == plk.ERR_ARG
    assert lib.plk_slowfast_step(ctypes.byref(ok), ctypes.byref(sfp), p, q, p, None, q, None) == plk.ERR_ARG
    assert lib.plk_slowfast_step(ctypes.byref(ok), ctypes.byref(sfp), p, q, p, p, p, None) == plk.ERR_ARG
    long_seq = plk.dims(1, (1 << 20) + 1, 64, 4, 16, 64, dtype=plk.F32)
    assert lib.plk_slowfast_step(ctypes.byref(long_seq), ctypes.byref(sfp), p, q, p, None, None, None) == \
        plk.ERR_SHAPE


def test_slowfast_state_layout_matches_header():
    import partial_recompute_kv_b200 as plk
    src = open(HEADER).read()
    assert "#define PLK_SF_HIST_MAX %d" % plk.SF_HIST_MAX in src
    assert plk.SF_STATE_WORDS == 4 + plk.SF_HIST_MAX
    assert ctypes.sizeof(plk.PlkSfParams) == 24


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes structures of the binding have the C header's sizes and field offsets."""
    import shutil
    import subprocess

    import partial_recompute_kv_b200 as plk
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"plk_dims": plk.PlkDims, "plk_weights": plk.PlkWeights, "plk_sf_params": plk.PlkSfParams}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "plk.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append('  printf("plk_sf_state size %zu\\n", sizeof(plk_sf_state));')
    lines.append('  printf("PLK_STATIC_WS_BYTES %zu\\n", (size_t)PLK_STATIC_WS_BYTES);')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(((ln.rsplit(" ", 1)[0]), int(ln.rsplit(" ", 1)[1]))
               for ln in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
               if ln)
    for cname, py in structs.items():
        assert got[f"{cname} size"] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[f"{cname} {fname}"] == getattr(py, fname).offset, (cname, fname)
    assert got["plk_sf_state size"] == 4 * plk.SF_STATE_WORDS
    assert got["PLK_STATIC_WS_BYTES"] == plk.STATIC_WS_BYTES  # the binding's copy of the static array's size
