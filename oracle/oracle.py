"""fp64 CPU oracle for the hot path: window scoring, per-head budget selection,
budget allocation, compaction, append and decode attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or runs
this module; only the tests, the smoke check and the benchmark's CPU-baseline
leg do. It shares no code with the CUDA library: it is written from the
definitions on the pages, in float64 numpy, one slot at a time, with no blocking,
fusion or reordering beyond what a definition states.

Sources (pages by title, with the equation or section each function follows):

* ZigZagKV: Dynamic KV Cache Compression for Long-context Modeling based on
  Layer Uncertainty (arXiv 2412.09036) - Eq. 7 (importance = attention of the
  last w tokens, summed), Eq. 3 (LMBA: smallest token set holding 90 % of the
  attention mass, averaged over heads), Eq. 4-6 (uncertainty and the bounded
  per-layer budget B_l = B_bound + (B - B_bound) * L * uncertainty_l).
* Model Tells You What to Discard: Adaptive KV Cache Compression for LLMs
  (FastGen, arXiv 2310.01801) - the three head policies of its abstract / Section 1:
  local heads keep the recent window, special-token heads keep special tokens,
  global heads keep the full cache.
* ChunkLLM: A Lightweight Pluggable Framework for Accelerating LLMs Inference
  (arXiv 2510.02361) - Section 2.2, Eq. 3: a chunk is represented by the key of
  its last (boundary) token; chunk attention is a softmax over query . chunk-key
  products; the top chunks are kept.

Parity pins: every function below is pinned by a CPU test against an invariant,
a closed form, brute force or an independent library routine, except the exact
integer semantics of the bounded allocation (rounding and cap), which the
ZigZagKV page does not fix (it never states B_bound): those readings are pinned
only by the properties Eq. 6 implies (sum, floor, cap, equal-uncertainty case) -
parity unpinned for the rounding rule itself.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def _f64(x) -> np.ndarray:
    """Exact widening of the caller's array (fp32 / bf16 torch tensor or numpy) to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# (a1) window scoring - ZigZagKV Eq. 7 (SnapKV-style observation window)
# ---------------------------------------------------------------------------
def window_scores(q_win, k, L: int, key_pos=None) -> np.ndarray:
    """Importance score of every cached key, per slot.

    q_win : [S*G, w, d] - the window queries; rows of slot s are q_win[s*G:(s+1)*G].
            Window row i sits at position L - w + i.
    k     : [S, N, d]   - keys; N = L for token keys, N = C for chunk keys.
    key_pos : None (key j is at position j) or int [N] positions of the keys
            (chunk keys: the position of the chunk's last token).

    For each slot, query head h of its group and window row i, the logits are
    q_{h,i} . k_j / sqrt(d) over the keys the row can see (key position <=
    L - w + i, the prompt's causal mask); each row is softmax-normalised and the
    score of key j is the sum of p_{h,i,j} over the group's heads and the w rows.
    Returns float64 [S, N].
    """
    q = _f64(q_win)
    kk = _f64(k)
    S, N, d = kk.shape
    SG, w, _ = q.shape
    G = SG // S
    pos = np.arange(N) if key_pos is None else np.asarray(key_pos, dtype=np.int64)
    row_pos = (L - w) + np.arange(w)                      # position of window row i
    visible = pos[None, :] <= row_pos[:, None]            # [w, N]
    visible = np.tile(visible, (G, 1))                    # rows ordered (h, i)
    out = np.zeros((S, N), dtype=np.float64)
    scale = 1.0 / np.sqrt(d)
    for s in range(S):
        qs = q[s * G:(s + 1) * G].reshape(G * w, d)
        logits = (qs @ kk[s].T) * scale                    # [G*w, N]
        logits = np.where(visible, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        p = e / e.sum(axis=1, keepdims=True)
        out[s] = p.sum(axis=0)
    return out


def chunk_keys(k, chunk_end) -> np.ndarray:
    """ChunkLLM Eq. 3: chunk c is represented by the key of its last token."""
    kk = _f64(k)
    return kk[:, np.asarray(chunk_end, dtype=np.int64), :]


def chunk_scores(q_win, k, L: int, chunk_end) -> np.ndarray:
    """Chunk-level window scores: the window scoring of a1 over the chunk keys,
    each visible to a window row once its last token is (ChunkLLM Section 2.2)."""
    return window_scores(q_win, chunk_keys(k, chunk_end), L, key_pos=chunk_end)


# ---------------------------------------------------------------------------
# (a2) selection
# ---------------------------------------------------------------------------
def _desc_order(score: np.ndarray) -> np.ndarray:
    """Indices sorted by score descending, equal scores by ascending index."""
    return np.lexsort((np.arange(score.shape[0]), -score))


def top_b(score, B: int) -> np.ndarray:
    """Per-head eviction keeps the B highest-scoring tokens (the per-head
    policy ZigZagKV reuses, Section 4.1). Returned in ascending position order."""
    sc = _f64(score)
    B = min(int(B), sc.shape[0])
    return np.sort(_desc_order(sc)[:B]).astype(np.int64)


def mass_count(score, mass: float = 0.9) -> int:
    """LMBA of one head (ZigZagKV Eq. 3): the size of the smallest set of tokens
    whose attention mass reaches `mass` of the head's total. The greedy prefix
    of the descending order is that smallest set; it is the first k with
    cum_k >= mass * total."""
    sc = _f64(score)
    cum = np.cumsum(sc[_desc_order(sc)])
    target = mass * cum[-1]
    return int(np.searchsorted(cum, target, side="left")) + 1


def local_indices(L: int, window: int) -> np.ndarray:
    """FastGen local heads: keep the most recent `window` tokens."""
    return np.arange(max(0, L - int(window)), L, dtype=np.int64)


def special_indices(special_mask_row) -> np.ndarray:
    """FastGen special-token heads: keep only the special tokens."""
    return np.flatnonzero(np.asarray(special_mask_row) != 0).astype(np.int64)


def full_indices(L: int) -> np.ndarray:
    """FastGen global heads: keep the whole cache."""
    return np.arange(L, dtype=np.int64)


def chunk_select(cscore, chunk_end, target_tokens: int):
    """ChunkLLM chunk selection: order chunks by chunk score (descending, ties by
    chunk index) and keep the shortest prefix of that order whose chunks hold at
    least `target_tokens` tokens. Returns (token indices ascending, chosen chunk ids ascending)."""
    sc = _f64(cscore)
    ends = np.asarray(chunk_end, dtype=np.int64)
    starts = np.concatenate([[0], ends[:-1] + 1])
    lens = ends - starts + 1
    order = _desc_order(sc)
    cum = np.cumsum(lens[order])
    n = int(np.searchsorted(cum, int(target_tokens), side="left")) + 1
    n = min(n, len(order))
    chosen = np.sort(order[:n])
    toks = np.concatenate([np.arange(starts[c], ends[c] + 1) for c in chosen]).astype(np.int64)
    return toks, chosen


# ---------------------------------------------------------------------------
# (a3) bounded per-layer allocation - ZigZagKV Eq. 4-6
# ---------------------------------------------------------------------------
def allocate_budgets(counts, L: int, avg_budget: int, floor_budget: int) -> np.ndarray:
    """Per-layer budgets from the per-head LMBA counts.

    counts : int [nL, H] - mass_count of every head (slot) of every layer.
    LMBA_l is the mean over a layer's heads (Eq. 3); uncertainty_l = LMBA_l /
    sum_l LMBA_l (Eq. 4); B_l = B_bound + (B - B_bound) * nL * uncertainty_l
    (Eq. 6), so sum_l B_l = nL * B and every B_l >= B_bound.

    Readings where the page is silent (it never states B_bound): budgets are
    integers - floor of the exact rational B_l, then one extra token to the
    layers with the largest remainders (ties to the lower layer) until the sum
    is nL * B; a layer cannot keep more than L tokens - layers whose B_l exceeds
    L are fixed at L and the rest is re-split over the other layers by the same
    formula (water-filling); if every count is zero the split is uniform.
    """
    c = np.asarray(counts, dtype=np.int64)
    nL = c.shape[0]
    C = [int(x) for x in c.sum(axis=1)]          # H * LMBA_l; the 1/H cancels in u_l
    T = nL * int(avg_budget)
    f = min(int(floor_budget), int(L))
    capped: set[int] = set()
    while True:
        U = [l for l in range(nL) if l not in capped]
        if not U:
            break
        R = T - len(capped) * L
        E = R - len(U) * f
        denom = sum(C[l] for l in U)
        w = {l: (C[l] if denom > 0 else 1) for l in U}
        den = denom if denom > 0 else len(U)
        ideal = {l: Fraction(f) + Fraction(E * w[l], den) for l in U}
        over = [l for l in U if ideal[l] > L]
        if not over:
            break
        capped.update(over)
    out = np.zeros(nL, dtype=np.int64)
    for l in capped:
        out[l] = L
    if U:
        num = {l: f * den + E * w[l] for l in U}
        base = {l: num[l] // den for l in U}
        rem = {l: num[l] % den for l in U}
        left = R - sum(base.values())
        by_rem = sorted(U, key=lambda l: (-rem[l], l))
        for i, l in enumerate(U):
            out[l] = base[l]
        for l in by_rem[:left]:
            out[l] += 1
    return out


# ---------------------------------------------------------------------------
# (a4) compaction into the packed per-head cache
# ---------------------------------------------------------------------------
def layout(counts, reserve: int, align: int = 16):
    """Packed layout: slot s owns rows [off_s, off_s + cap_s) with
    cap_s = round_up(count_s + reserve, align), slots back to back in slot order."""
    cnt = np.asarray(counts, dtype=np.int64)
    cap = ((cnt + int(reserve) + align - 1) // align) * align
    off = np.zeros(cnt.shape[0] + 1, dtype=np.int64)
    off[1:] = np.cumsum(cap)
    return off, cap


def compact(k, v, sel, off, total_rows=None):
    """Row r of slot s in the packed cache is K[s][sel[s][r]] (and V likewise),
    sel[s] ascending. Rows past each slot's count are left zero here."""
    kk, vv = _f64(k), _f64(v)
    d = kk.shape[2]
    rows = int(off[-1]) if total_rows is None else int(total_rows)
    kp = np.zeros((rows, d), dtype=np.float64)
    vp = np.zeros((rows, d), dtype=np.float64)
    for s, idx in enumerate(sel):
        o = int(off[s])
        kp[o:o + len(idx)] = kk[s][idx]
        vp[o:o + len(idx)] = vv[s][idx]
    return kp, vp


def append(kp, vp, off, length, k_new, v_new):
    """Append one new token per slot at row off_s + len_s; len_s += 1 (in place)."""
    kn, vn = _f64(k_new), _f64(v_new)
    for s in range(len(length)):
        r = int(off[s]) + int(length[s])
        kp[r] = kn[s]
        vp[r] = vn[s]
        length[s] += 1


# ---------------------------------------------------------------------------
# (a6) decode attention over the ragged packed cache
# ---------------------------------------------------------------------------
def decode_attention(q, kp, vp, off, length, G: int) -> np.ndarray:
    """o_h = sum_r softmax_r(q_h . Kp[off_s + r] / sqrt(d)) Vp[off_s + r] over the
    len_s rows of the slot s = h // G that query head h reads (GQA).
    q: [S*G, d]. Returns float64 [S*G, d]."""
    qq = _f64(q)
    kk, vv = _f64(kp), _f64(vp)
    SG, d = qq.shape
    out = np.zeros((SG, d), dtype=np.float64)
    scale = 1.0 / np.sqrt(d)
    for h in range(SG):
        s = h // G
        o, n = int(off[s]), int(length[s])
        if n == 0:
            continue
        ks, vs = kk[o:o + n], vv[o:o + n]
        logits = (ks @ qq[h]) * scale
        p = np.exp(logits - logits.max())
        p /= p.sum()
        out[h] = p @ vs
    return out


# ---------------------------------------------------------------------------
# next rows: attention loss (ZigZagKV Section 5.5, Table 3) and head profiling
# ---------------------------------------------------------------------------
def retained_mass(score, kept) -> float:
    """Share of a head's window-attention mass that the kept tokens hold:
    sum_{j in kept} score_j / sum_j score_j (0 for a head with no mass)."""
    sc = _f64(score)
    total = sc.sum()
    if total <= 0:
        return 0.0
    return float(sc[np.asarray(kept, dtype=np.int64)].sum() / total)


def attention_loss(retained, target: float = 0.9) -> float:
    """ZigZagKV's attention loss of one head: how far the retained mass falls short of
    the 0.9 the LMBA budget is defined by (0 when it reaches it). Reading: the page
    calls it the average deviation from achieving 0.9 attention; a head above 0.9
    deviates by nothing."""
    return max(0.0, float(target) - float(retained))


def profile_head(score, special_mask_row, window: int, tau: float) -> int:
    """FastGen-style head profiling from window attention (the pages give no
    criterion; this is the reading): among the policies local (keep the last
    `window` tokens), special (keep the special tokens) and full, pick the one that
    keeps the fewest tokens while retaining at least `tau` of the head's attention
    mass; ties in size go local, then special. Returns the policy code."""
    sc = _f64(score)
    L = sc.shape[0]
    cands = []
    loc = local_indices(L, window)
    cands.append((len(loc), 0, 2, loc))                  # LOCAL
    spc = special_indices(special_mask_row)
    cands.append((len(spc), 1, 3, spc))                  # SPECIAL
    for size, order, code, idx in sorted(cands, key=lambda c: (c[0], c[1])):
        if retained_mass(sc, idx) >= tau:
            return code
    return 4                                             # FULL


def chunk_select_local(cscore, chunk_end, target_tokens: int, n_local: int):
    """ChunkLLM chunk selection with always-kept local chunks (its Section 3.2 keeps
    the 15 or 16 most recent chunks): the last n_local chunks are kept, then the
    other chunks in score order (descending, ties by chunk index) until the kept
    chunks hold at least `target_tokens` tokens. Returns (tokens ascending, chunk ids ascending)."""
    sc = _f64(cscore)
    ends = np.asarray(chunk_end, dtype=np.int64)
    C = ends.shape[0]
    starts = np.concatenate([[0], ends[:-1] + 1])
    lens = ends - starts + 1
    n_local = max(0, min(int(n_local), C))
    forced = np.arange(C - n_local, C, dtype=np.int64)
    have = int(lens[forced].sum())
    rest = np.arange(0, C - n_local, dtype=np.int64)
    chosen = list(forced)
    if have < target_tokens and rest.size:
        order = rest[_desc_order(sc[rest])]
        cum = have + np.cumsum(lens[order])
        n = min(int(np.searchsorted(cum, int(target_tokens), side="left")) + 1, order.size)
        chosen += list(order[:n])
    chosen = np.sort(np.asarray(chosen, dtype=np.int64))
    toks = (np.concatenate([np.arange(starts[c], ends[c] + 1) for c in chosen]).astype(np.int64)
            if chosen.size else np.zeros(0, dtype=np.int64))
    return toks, chosen


# ---------------------------------------------------------------------------
# decode-time chunk re-selection - ChunkLLM ICAC
# ---------------------------------------------------------------------------
def icac_decode(q_win, k, v, chunk_end, q_dec, k_dec, v_dec, boundary_steps, keep_frac: float,
                n_local: int, G: int):
    """ChunkLLM decode with re-selection at chunk boundaries (its Section 2.3: chunk
    selection runs only when the current token closes a chunk - the Intra-Chunk
    Attention Consistency pattern - and the selection holds until the next boundary).

    One slot. The full cache (prompt plus every generated token) stays available;
    the attended cache is the selected chunks plus the tokens generated since the
    last selection. Step t appends token L + t to both, then attends over the
    attended cache with q_dec[t]. If step t is in `boundary_steps`, token L + t
    closes a chunk: the chunk list grows by it, every chunk is scored with the
    single query q_dec[t] (the chunk scoring of `chunk_scores` with a window of
    one), and the selection becomes `chunk_select_local` over all chunks with the
    target ceil(keep_frac * (L + t + 1)) tokens - for the steps after t.

    Returns (outputs [steps, G, d], selections: {step: token indices} at the start
    and after every boundary step, keyed -1 for the prompt selection).
    """
    kf = np.concatenate([_f64(k), _f64(k_dec)], axis=0)
    vf = np.concatenate([_f64(v), _f64(v_dec)], axis=0)
    L = _f64(k).shape[0]
    steps = _f64(q_dec).shape[0]
    ends = [int(e) for e in np.asarray(chunk_end, dtype=np.int64)]
    target = int(np.ceil(keep_frac * L))
    cs = chunk_scores(q_win, kf[None, :L], L, np.asarray(ends))[0]
    sel, _ = chunk_select_local(cs, np.asarray(ends), target, n_local)
    sels = {-1: sel.copy()}
    bset = set(int(b) for b in boundary_steps)
    outs = np.zeros((steps, G, kf.shape[1]))
    attended = list(sel)
    for t in range(steps):
        n = L + t + 1
        attended.append(L + t)
        idx = np.asarray(attended, dtype=np.int64)
        q = _f64(q_dec[t])
        outs[t] = decode_attention(q, kf[idx], vf[idx], [0, idx.size], [idx.size], G)
        if t in bset:
            ends.append(L + t)
            cs = chunk_scores(q[:, None, :], kf[None, :n], n, np.asarray(ends))[0]
            sel, _ = chunk_select_local(cs, np.asarray(ends), int(np.ceil(keep_frac * n)), n_local)
            sels[t] = sel.copy()
            attended = list(sel)
    return outs, sels


def sliding_local_indices(L: int, t: int, window: int) -> np.ndarray:
    """FastGen local heads with eviction while decoding: a local head attends to the most
    recent `window` tokens of the sequence, so at decode step t (token L + t appended) it
    keeps positions [L + t + 1 - window, L + t] (the local-window variant of the policy)."""
    n = int(L) + int(t) + 1
    return np.arange(max(0, n - int(window)), n, dtype=np.int64)
