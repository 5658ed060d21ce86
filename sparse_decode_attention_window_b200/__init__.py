"""Attention-score-driven KV eviction and ragged decode attention for B200.

Python face of libkvc.so (include/kvc.h): the functions below carry the C ABI's
names and take torch CUDA tensors; they marshal pointers, sizes and the current
stream and call the library, nothing more. The library must be built
(`python -m sparse_decode_attention_window_b200.build`); without it every call
raises - there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import (KvcShape, KvcError, KVC_BF16, KVC_FP32, KVC_POL_TOPB, KVC_POL_MASS_COUNT, KVC_POL_LOCAL,
                   KVC_POL_SPECIAL, KVC_POL_FULL, KVC_POL_CHUNK, KVC_WS_SCORE, KVC_WS_SELECT, KVC_WS_DECODE)

__all__ = ["KvcShape", "KvcError", "make_shape", "kvc_score", "kvc_select", "kvc_alloc_budgets", "kvc_layout",
           "kvc_compact", "kvc_layout_compact", "kvc_append", "kvc_decode_attn", "kvc_workspace_size", "kvc_get_status", "kvc_version",
           "kvc_launch_count", "kvc_decode_attn_noalloc", "kvc_append_decode", "kvc_append_decode_chain", "kvc_select_chunks",
           "kvc_retained_mass", "kvc_profile_heads", "kvc_append_window", "kvc_check_wait_limit",
           "kvc_diag_set_path", "kvc_diag_get_path",
           "library", "KVC_BF16", "KVC_FP32", "KVC_POL_TOPB", "KVC_POL_MASS_COUNT", "KVC_POL_LOCAL",
           "KVC_POL_SPECIAL", "KVC_POL_FULL", "KVC_POL_CHUNK", "KVC_WS_SCORE", "KVC_WS_SELECT", "KVC_WS_DECODE"]


def library() -> ctypes.CDLL:
    return _abi.load()


def make_shape(n_slots, G, d, L, w=0, n_kv_heads=1, batch=1, dtype=torch.bfloat16) -> KvcShape:
    dt = KVC_FP32 if dtype == torch.float32 else KVC_BF16
    return KvcShape(int(n_slots), int(G), int(d), int(L), int(w), int(n_kv_heads), int(batch), dt)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("kvc: tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("kvc: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(name, rc):
    if rc != 0:
        raise KvcError(name, rc, library().kvc_last_error().decode())


def kvc_workspace_size(which: int, shape: KvcShape, C: int = 0) -> int:
    return int(library().kvc_workspace_size(which, ctypes.byref(shape), int(C)))


def kvc_score(shape, q_win, k, score, ws, chunk_end=None, C=0, row_lse=None, stream=None):
    _check("kvc_score", library().kvc_score(ctypes.byref(shape), _ptr(q_win), _ptr(k), _ptr(chunk_end), int(C),
                                            _ptr(row_lse), _ptr(score), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)))


def kvc_select(shape, score, policy, budget, idx, count, mass=0.9, special_mask=None, chunk_end=None, C=0,
               stream=None):
    max_sel = idx.shape[-1] if idx is not None else 0
    _check("kvc_select", library().kvc_select(ctypes.byref(shape), _ptr(score), _ptr(policy), _ptr(budget),
                                              float(mass), _ptr(special_mask), _ptr(chunk_end), int(C), _ptr(idx),
                                              int(max_sel), _ptr(count), None, 0, _stream(stream)))


def kvc_alloc_budgets(counts, n_layers, spl, L, avg_B, floor_B, budgets, slot_budgets=None, stream=None):
    _check("kvc_alloc_budgets", library().kvc_alloc_budgets(_ptr(counts), int(n_layers), int(spl), int(L),
                                                            int(avg_B), int(floor_B), _ptr(budgets),
                                                            _ptr(slot_budgets), _stream(stream)))


def kvc_layout(count, reserve, off, cap, stream=None):
    _check("kvc_layout", library().kvc_layout(_ptr(count), int(count.numel()), int(reserve), _ptr(off), _ptr(cap),
                                              _stream(stream)))


def kvc_compact(shape, k, v, idx, count, off, kp, vp, length, stream=None):
    _check("kvc_compact", library().kvc_compact(ctypes.byref(shape), _ptr(k), _ptr(v), _ptr(idx), int(idx.shape[-1]),
                                                _ptr(count), _ptr(off), _ptr(kp), _ptr(vp), int(kp.shape[0]),
                                                _ptr(length), _stream(stream)))


def kvc_layout_compact(shape, k, v, idx, count, reserve, off, cap, kp, vp, length, stream=None):
    """kvc_layout then kvc_compact, in one launch for up to 512 slots (see include/kvc.h)."""
    _check("kvc_layout_compact",
           library().kvc_layout_compact(ctypes.byref(shape), _ptr(k), _ptr(v), _ptr(idx), int(idx.shape[-1]),
                                        _ptr(count), int(reserve), _ptr(off), _ptr(cap), _ptr(kp), _ptr(vp),
                                        int(kp.shape[0]), _ptr(length), _stream(stream)))


def kvc_append_window(shape, k_new, v_new, off, cap, length, window, head, kp, vp, stream=None):
    """kvc_append with sliding-window eviction for the slots with window > 0 (see include/kvc.h)."""
    _check("kvc_append_window",
           library().kvc_append_window(ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(off), _ptr(cap),
                                       _ptr(length), _ptr(window), _ptr(head), _ptr(kp), _ptr(vp), int(kp.shape[0]),
                                       _stream(stream)))


def kvc_append(shape, k_new, v_new, off, cap, length, kp, vp, stream=None):
    _check("kvc_append", library().kvc_append(ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(off), _ptr(cap),
                                              _ptr(length), _ptr(kp), _ptr(vp), int(kp.shape[0]), _stream(stream)))


def kvc_decode_attn(shape, q, kp, vp, off, length, out, ws, stream=None):
    _check("kvc_decode_attn", library().kvc_decode_attn(ctypes.byref(shape), _ptr(q), _ptr(kp), _ptr(vp), _ptr(off),
                                                        _ptr(length), int(kp.shape[0]), _ptr(out), _ptr(ws),
                                                        ws.numel() * ws.element_size(), _stream(stream)))


def kvc_append_decode(shape, k_new, v_new, q, kp, vp, off, cap, length, out, ws, stream=None):
    _check("kvc_append_decode",
           library().kvc_append_decode(ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(kp), _ptr(vp),
                                       _ptr(off), _ptr(cap), _ptr(length), int(kp.shape[0]), _ptr(out), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)))


def kvc_append_decode_chain(shape, k_new, v_new, q, kp, vp, off, cap, stable, length, out, ws, stream=None):
    """kvc_append_decode for a decode-loop step after the first: `stable` holds per slot
    a row count that the previous kernel on the stream does not write (see include/kvc.h)."""
    _check("kvc_append_decode_chain",
           library().kvc_append_decode_chain(ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(kp),
                                             _ptr(vp), _ptr(off), _ptr(cap), _ptr(stable), _ptr(length),
                                             int(kp.shape[0]), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                             _stream(stream)))


def kvc_decode_attn_noalloc(shape, q, kp, vp, off, length, out, stream=None):
    """kvc_decode_attn without a workspace, for callers that cannot allocate device
    memory; its scratch is a fixed array inside the library (see include/kvc.h)."""
    _check("kvc_decode_attn_noalloc",
           library().kvc_decode_attn_noalloc(ctypes.byref(shape), _ptr(q), _ptr(kp), _ptr(vp), _ptr(off),
                                             _ptr(length), int(kp.shape[0]), _ptr(out), _stream(stream)))


def kvc_select_chunks(shape, chunk_score, chunk_end, target, idx, count, n_local=0, stream=None):
    _check("kvc_select_chunks",
           library().kvc_select_chunks(ctypes.byref(shape), _ptr(chunk_score), _ptr(chunk_end),
                                       int(chunk_end.numel()), _ptr(target), int(n_local), _ptr(idx),
                                       int(idx.shape[-1]), _ptr(count), _stream(stream)))


def kvc_retained_mass(shape, score, idx, count, retained, stream=None):
    _check("kvc_retained_mass",
           library().kvc_retained_mass(ctypes.byref(shape), _ptr(score), int(score.shape[-1]), _ptr(idx),
                                       int(idx.shape[-1]), _ptr(count), _ptr(retained), _stream(stream)))


def kvc_profile_heads(shape, score, policy, window, tau=0.95, special_mask=None, shares=None, stream=None):
    _check("kvc_profile_heads",
           library().kvc_profile_heads(ctypes.byref(shape), _ptr(score), _ptr(special_mask), int(window),
                                       float(tau), _ptr(policy), _ptr(shares), _stream(stream)))


def kvc_check_wait_limit(limit_us, stream=None):
    """Diagnostic: a kernel waits on a barrier nothing arrives on until limit_us, gives up and
    flags a wait timeout (see include/kvc.h)."""
    _check("kvc_check_wait_limit", library().kvc_check_wait_limit(int(limit_us), _stream(stream)))


def kvc_diag_set_path(knob: str, choice: str):
    """Diagnostic, cross-checks only: force an alternate kernel path for every later call
    in this process (knob, choice as in _abi.KVC_DIAG; "auto" restores the default)."""
    k, choices = _abi.KVC_DIAG[knob]
    _check("kvc_diag_set_path", library().kvc_diag_set_path(k, choices[choice]))


def kvc_diag_get_path(knob: str) -> str:
    k, choices = _abi.KVC_DIAG[knob]
    v = int(library().kvc_diag_get_path(k))
    return {c: n for n, c in choices.items()}[v]


def kvc_get_status(stream=None):
    _check("kvc_get_status", library().kvc_get_status(_stream(stream)))


def kvc_version() -> str:
    return library().kvc_version().decode()


def kvc_launch_count() -> int:
    return int(library().kvc_launch_count())
