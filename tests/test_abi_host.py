"""The C-ABI library without a GPU: it loads, exports every symbol include/kvc.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_decode_attention_window_b200 as kvc
from sparse_decode_attention_window_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvc_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("kvc_score", "kvc_select", "kvc_compact", "kvc_decode_attn", "kvc_append"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = kvc.library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(_abi.EXPORTS)


def test_version():
    assert "sm_100a" in kvc.kvc_version()


def _shape(**kw):
    base = dict(n_slots=2, G=4, d=128, L=100, w=4, n_kv_heads=2, batch=1)
    base.update(kw)
    return kvc.KvcShape(base["n_slots"], base["G"], base["d"], base["L"], base["w"], base["n_kv_heads"],
                        base["batch"], kvc.KVC_BF16)


@pytest.mark.parametrize("kw,code", [
    (dict(n_slots=0), _abi.KVC_ERR_SHAPE),
    (dict(d=96), _abi.KVC_ERR_UNSUPPORTED),
    (dict(w=0), _abi.KVC_ERR_SHAPE),
    (dict(w=101), _abi.KVC_ERR_SHAPE),
    (dict(n_kv_heads=0), _abi.KVC_ERR_SHAPE),
])
def test_score_rejects_bad_shapes(kw, code):
    lib = kvc.library()
    sh = _shape(**kw)
    rc = lib.kvc_score(ctypes.byref(sh), None, None, None, 0, None, None, None, 0, None)
    assert rc == code
    assert lib.kvc_last_error()


def test_score_rejects_null_tensors():
    lib = kvc.library()
    rc = lib.kvc_score(ctypes.byref(_shape()), None, None, None, 0, None, None, None, 0, None)
    assert rc == _abi.KVC_ERR_INVALID_ARG


def test_alloc_budgets_validates_floor_avg_context():
    lib = kvc.library()
    p = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    assert lib.kvc_alloc_budgets(p, 4, 8, 100, 20, 30, p, None, None) == _abi.KVC_ERR_SHAPE   # floor > avg
    assert lib.kvc_alloc_budgets(p, 4, 8, 100, 200, 3, p, None, None) == _abi.KVC_ERR_SHAPE   # avg > L
    assert lib.kvc_alloc_budgets(p, 0, 8, 100, 20, 3, p, None, None) == _abi.KVC_ERR_SHAPE    # no layers
    assert lib.kvc_alloc_budgets(None, 4, 8, 100, 20, 3, p, None, None) == _abi.KVC_ERR_INVALID_ARG


def test_layout_and_append_validate():
    lib = kvc.library()
    p = ctypes.c_void_p(16)
    assert lib.kvc_layout(p, 0, 4, p, p, None) == _abi.KVC_ERR_SHAPE
    assert lib.kvc_layout(p, 4, -1, p, p, None) == _abi.KVC_ERR_SHAPE
    assert lib.kvc_append(ctypes.byref(_shape()), None, p, p, p, p, p, p, 64, None) == _abi.KVC_ERR_INVALID_ARG
    misaligned = ctypes.c_void_p(24)
    assert lib.kvc_append(ctypes.byref(_shape()), misaligned, p, p, p, p, p, p, 64, None) == _abi.KVC_ERR_INVALID_ARG


def test_layout_compact_validates():
    lib = kvc.library()
    p = ctypes.c_void_p(16)
    sh = ctypes.byref(_shape())
    f = lib.kvc_layout_compact
    assert f(sh, p, p, p, 64, p, 4, None, p, p, p, 1024, p, None) == _abi.KVC_ERR_INVALID_ARG   # no off
    assert f(sh, p, p, p, 64, p, 4, p, None, p, p, 1024, p, None) == _abi.KVC_ERR_INVALID_ARG   # no cap
    assert f(sh, p, p, p, 64, p, -1, p, p, p, p, 1024, p, None) == _abi.KVC_ERR_SHAPE           # reserve < 0
    assert f(sh, p, p, p, 0, p, 4, p, p, p, p, 1024, p, None) == _abi.KVC_ERR_SHAPE             # max_sel 0
    assert f(sh, p, ctypes.c_void_p(24), p, 64, p, 4, p, p, p, p, 1024, p, None) == _abi.KVC_ERR_INVALID_ARG
    assert b"kvc_layout_compact" in lib.kvc_last_error()


def test_select_validates_mass_and_chunks():
    lib = kvc.library()
    p = ctypes.c_void_p(16)
    sh = ctypes.byref(_shape())
    assert lib.kvc_select(sh, p, p, p, 0.0, None, None, 0, p, 10, p, None, 0, None) == _abi.KVC_ERR_INVALID_ARG
    assert lib.kvc_select(sh, p, p, p, 1.5, None, None, 0, p, 10, p, None, 0, None) == _abi.KVC_ERR_INVALID_ARG
    assert lib.kvc_select(sh, p, p, p, 0.9, None, p, 0, p, 10, p, None, 0, None) == _abi.KVC_ERR_SHAPE
    assert lib.kvc_select(sh, p, None, p, 0.9, None, None, 0, p, 10, p, None, 0, None) == _abi.KVC_ERR_INVALID_ARG


def test_workspace_sizes_are_positive_for_score_and_decode():
    sh = _shape(n_slots=32, L=8192, w=32, n_kv_heads=8, batch=4)
    assert kvc.kvc_workspace_size(kvc.KVC_WS_SCORE, sh) > 0
    assert kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh) > 0
    assert kvc.kvc_workspace_size(kvc.KVC_WS_SELECT, sh) == 0


def test_wait_limit_check_validates_its_limit():
    lib = kvc.library()
    for bad in (0, -5, 1000001):
        assert lib.kvc_check_wait_limit(bad, None) == _abi.KVC_ERR_INVALID_ARG
        assert b"limit_us" in lib.kvc_last_error()


def test_fused_decode_entries_validate():
    lib = kvc.library()
    p = ctypes.c_void_p(16)
    sh = ctypes.byref(_shape())
    # the chained form needs its promise array
    assert lib.kvc_append_decode_chain(sh, p, p, p, p, p, p, p, None, p, 64, p, p, 1 << 20, None) == \
        _abi.KVC_ERR_INVALID_ARG
    assert b"stable" in lib.kvc_last_error()
    assert lib.kvc_append_decode_chain(sh, None, p, p, p, p, p, p, p, p, 64, p, p, 1 << 20, None) == \
        _abi.KVC_ERR_INVALID_ARG
    assert lib.kvc_append_decode(sh, p, p, p, p, p, p, None, p, 64, p, p, 1 << 20, None) == _abi.KVC_ERR_INVALID_ARG
    bad = ctypes.byref(_shape(d=96))
    assert lib.kvc_append_decode_chain(bad, p, p, p, p, p, p, p, p, p, 64, p, p, 1 << 20, None) == \
        _abi.KVC_ERR_UNSUPPORTED


def test_diagnostic_path_knobs_set_get_and_reject():
    """Alternate kernel paths are chosen only through kvc_diag_set_path: every knob starts at
    auto, takes its documented choices, rejects unknown knobs and choices, and returns to auto."""
    lib = kvc.library()
    for knob, (k, choices) in _abi.KVC_DIAG.items():
        assert lib.kvc_diag_get_path(k) == 0, knob
        for name, c in choices.items():
            assert lib.kvc_diag_set_path(k, c) == _abi.KVC_OK
            assert kvc.kvc_diag_get_path(knob) == name
        assert lib.kvc_diag_set_path(k, len(choices)) == _abi.KVC_ERR_INVALID_ARG
        assert lib.kvc_diag_set_path(k, -1) == _abi.KVC_ERR_INVALID_ARG
        kvc.kvc_diag_set_path(knob, "auto")
        assert lib.kvc_diag_get_path(k) == 0
    assert lib.kvc_diag_set_path(len(_abi.KVC_DIAG), 0) == _abi.KVC_ERR_INVALID_ARG
    assert lib.kvc_diag_get_path(len(_abi.KVC_DIAG)) == -1


def test_environment_does_not_switch_kernel_paths():
    """No environment variable reaches the library's path choice: a process started with the
    old switch names set still reports every knob at auto."""
    import subprocess
    import sys
    env = dict(os.environ, KVC_SCORE_PATH="simt", KVC_SELECT_PATH="cta", KVC_COMPACT_PATH="grid",
               KVC_DECODE_PATH="tc", KVC_DECODE_SPLIT="tokens")
    code = ("import sys; sys.path.insert(0, %r); import sparse_decode_attention_window_b200 as k; "
            "print([k.library().kvc_diag_get_path(i) for i in range(5)])" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "[0, 0, 0, 0, 0]"
    src = open(os.path.join(ROOT, "sparse_decode_attention_window_b200", "csrc", "kvc.cu")).read()
    assert "getenv" not in src
