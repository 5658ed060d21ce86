"""Comparison rules between the CUDA path and the fp64 oracle.

* scores: relative 2e-5 (bf16 inputs, fp32 accumulation) / 1e-5 (fp32), plus a tiny absolute floor.
* selected indices: bit-exact where the oracle's B-th / (B+1)-th score gap exceeds 1e-5
  relative; inside that band the GPU set must hold every token scoring above
  s_B (1 + 1e-5), only tokens scoring at least s_{B+1} (1 - 1e-5), and exactly B tokens.
* LMBA counts: exact unless the oracle's cum_{k-1} or cum_k lies within 1e-5 relative of
  0.9 * total, where k +- 1 is accepted.
* budgets: exact, computed by the oracle from the GPU's counts.
* layouts and packed rows: bit-exact.
* attention outputs: per output row, max |o - o_ref| / max |o_ref| <= 2e-3 (bf16) or 1e-5 (fp32).
"""
from __future__ import annotations

import numpy as np

GAP = 1e-5
OUT_TOL = {"bf16": 2e-3, "fp32": 1e-5}
SCORE_RTOL = {"bf16": 2e-5, "fp32": 1e-5}


def check_scores(gpu, ref, dtype, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    tol = SCORE_RTOL[dtype] * np.abs(ref) + 1e-9 * max(1.0, np.abs(ref).max())
    bad = np.abs(gpu - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} scores off, worst rel " \
        f"{(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-30)).max():.3e}"


def _desc(score):
    return np.lexsort((np.arange(score.shape[0]), -score))


def check_topb(gpu_idx, ref_score, B, what=""):
    """gpu_idx: the GPU's kept indices (ascending); ref_score: the oracle's fp64 scores."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    L = ref_score.shape[0]
    B = min(B, L)
    assert len(gpu_idx) == B, f"{what}: kept {len(gpu_idx)} tokens, want {B}"
    assert (np.diff(gpu_idx) > 0).all(), f"{what}: indices not strictly ascending"
    if B == L:
        np.testing.assert_array_equal(gpu_idx, np.arange(L))
        return
    if B == 0:
        return
    order = _desc(ref_score)
    sB, sB1 = ref_score[order[B - 1]], ref_score[order[B]]
    gap = (sB - sB1) / sB if sB > 0 else 0.0
    if gap > GAP:
        np.testing.assert_array_equal(gpu_idx, np.sort(order[:B]), err_msg=what)
    else:
        must = np.flatnonzero(ref_score > sB * (1 + GAP))
        assert np.isin(must, gpu_idx).all(), f"{what}: a clearly-above token is missing"
        assert (ref_score[gpu_idx] >= sB1 * (1 - GAP)).all(), f"{what}: a clearly-below token was kept"


def check_mass_count(gpu_k, ref_score, mass=0.9, what=""):
    order = _desc(ref_score)
    cum = np.cumsum(ref_score[order])
    target = mass * cum[-1]
    k = int(np.searchsorted(cum, target, side="left")) + 1
    if gpu_k == k:
        return
    near = lambda i: 0 <= i < len(cum) and abs(cum[i] - target) <= GAP * target
    assert abs(gpu_k - k) == 1 and (near(k - 1) or near(k - 2)), f"{what}: LMBA count {gpu_k} vs oracle {k}"


def check_chunks(gpu_tokens, ref_cscore, chunk_end, target, what=""):
    """GPU kept tokens vs the oracle's chunk scores, with the gap rule at the prefix cut."""
    gpu_tokens = np.asarray(gpu_tokens, dtype=np.int64)
    ends = np.asarray(chunk_end, dtype=np.int64)
    starts = np.concatenate([[0], ends[:-1] + 1])
    lens = ends - starts + 1
    assert (np.diff(gpu_tokens) > 0).all(), f"{what}: tokens not ascending"
    # chunks the GPU kept, whole
    cid = np.searchsorted(ends, gpu_tokens, side="left")
    kept = np.unique(cid)
    assert lens[kept].sum() == len(gpu_tokens), f"{what}: a chunk was kept partially"
    total = lens[kept].sum()
    assert total >= min(target, ends[-1] + 1), f"{what}: kept {total} < target {target}"
    order = _desc(ref_cscore)
    cum = np.cumsum(lens[order])
    n = int(np.searchsorted(cum, target, side="left")) + 1
    ref_kept = np.sort(order[:n])
    if np.array_equal(kept, ref_kept):
        return
    # tie band at the cut
    sN = ref_cscore[order[n - 1]]
    sN1 = ref_cscore[order[n]] if n < len(order) else -np.inf
    assert (sN - sN1) / sN <= GAP, f"{what}: chunk sets differ outside the tie band"
    must = np.flatnonzero(ref_cscore > sN * (1 + GAP))
    assert np.isin(must, kept).all(), f"{what}: a clearly-above chunk is missing"
    assert (ref_cscore[kept] >= sN1 * (1 - GAP)).all(), f"{what}: a clearly-below chunk was kept"
    # minimal: dropping the last kept chunk in score order falls short
    worst = kept[np.lexsort((-kept, ref_cscore[kept]))[0]]
    assert total - lens[worst] < target, f"{what}: chunk prefix not minimal"


def check_out(gpu, ref, dtype, what=""):
    gpu = np.asarray(gpu, dtype=np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    err = np.abs(gpu - ref).max(axis=1) / den
    assert (err <= OUT_TOL[dtype]).all(), f"{what}: worst row rel err {err.max():.3e} > {OUT_TOL[dtype]}"
    return float(err.max())
