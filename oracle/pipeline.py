"""The oracle run over one workload: scoring, selection, allocation and the
decode loop, slot by slot, in float64.

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline).

Slots are independent except for the ZigZagKV allocation, which needs the LMBA
counts of every slot; callers that check a sample of slots at full size can pass
the budgets to use (the allocation itself is then checked separately, exactly,
from the counts).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import oracle as O

# policy codes (same values the C-ABI uses; plain constants, no arithmetic)
TOPB, MASS_COUNT, LOCAL, SPECIAL, FULL, CHUNK = 0, 1, 2, 3, 4, 5


@dataclass
class OracleResult:
    scores: dict = field(default_factory=dict)      # slot -> float64 [L] (or [C] for chunks)
    sel: dict = field(default_factory=dict)         # slot -> int64 ascending token indices
    mass_counts: dict = field(default_factory=dict) # slot -> LMBA count (zigzag)
    budgets: np.ndarray | None = None               # per-layer budgets (zigzag)
    out: dict = field(default_factory=dict)         # (step, slot) -> float64 [G, d]


def slot_budget_topb(wl, s, budgets):
    if wl.policy == "topb":
        return wl.top_b
    layer = s // wl.slots_per_layer
    return int(budgets[layer])


def run_workload(inp, slots=None, steps=None, budgets=None, need_all_counts=True) -> OracleResult:
    """Run the oracle on `slots` (default: all) for `steps` decode steps (default: all).

    For "zigzag", the LMBA counts of all slots are computed (window scores of
    every slot) unless `budgets` is given.
    """
    wl = inp.wl
    S, G, L = wl.n_slots, wl.G, wl.L
    slots = list(range(S)) if slots is None else list(slots)
    steps = wl.steps if steps is None else int(steps)
    res = OracleResult()

    def score_of(s):
        if s not in res.scores:
            q = inp.q_win[s * G:(s + 1) * G]
            if wl.policy == "chunk":
                res.scores[s] = O.chunk_scores(q, inp.k[s:s + 1], L, inp.chunk_end.cpu().numpy())[0]
            else:
                res.scores[s] = O.window_scores(q, inp.k[s:s + 1], L)[0]
        return res.scores[s]

    if wl.policy == "zigzag":
        if budgets is None:
            counts = np.zeros((wl.n_layers, wl.slots_per_layer), dtype=np.int64)
            for s in range(S):
                c = O.mass_count(score_of(s), wl.mass)
                res.mass_counts[s] = c
                counts[s // wl.slots_per_layer, s % wl.slots_per_layer] = c
            budgets = O.allocate_budgets(counts, L, wl.avg_budget, wl.floor_budget)
        res.budgets = np.asarray(budgets)

    for s in slots:
        if wl.policy in ("topb", "zigzag"):
            res.sel[s] = O.top_b(score_of(s), slot_budget_topb(wl, s, res.budgets))
        elif wl.policy == "fastgen":
            pol = int(inp.policy[s])
            b = (s // wl.hkv) % wl.batch
            if pol == LOCAL:
                res.sel[s] = O.local_indices(L, wl.local_window)
            elif pol == SPECIAL:
                res.sel[s] = O.special_indices(inp.special_mask[b].cpu().numpy())
            else:
                res.sel[s] = O.full_indices(L)
        elif wl.policy == "chunk" and getattr(wl, "icac", False):
            # ChunkLLM decode-time re-selection: the prompt selection keeps n_local local
            # chunks; the decode loop below re-selects at the generated chunk boundaries
            toks, _ = O.chunk_select_local(score_of(s), inp.chunk_end.cpu().numpy(), wl.chunk_target, wl.n_local)
            res.sel[s] = toks
        elif wl.policy == "chunk":
            toks, _ = O.chunk_select(score_of(s), inp.chunk_end.cpu().numpy(), wl.chunk_target)
            res.sel[s] = toks
        else:  # pragma: no cover
            raise ValueError(wl.policy)

    if steps > 0 and wl.policy == "chunk" and getattr(wl, "icac", False):
        from workloads import decode_chunk_boundaries
        bnd = decode_chunk_boundaries(wl)
        ce = inp.chunk_end.cpu().numpy()
        for s in slots:
            outs, _ = O.icac_decode(inp.q_win[s * G:(s + 1) * G], inp.k[s], inp.v[s], ce,
                                    inp.q_dec[:steps, s * G:(s + 1) * G], inp.k_dec[:steps, s], inp.v_dec[:steps, s],
                                    [b for b in bnd if b < steps], wl.keep_frac, wl.n_local, G)
            for t in range(steps):
                res.out[(t, s)] = outs[t]
        return res

    if steps > 0 and wl.policy == "fastgen" and getattr(wl, "local_sliding", False):
        # local heads keep exactly their last local_window tokens while decoding
        for s in slots:
            kf = np.concatenate([O._f64(inp.k[s]), O._f64(inp.k_dec[:steps, s])], axis=0)
            vf = np.concatenate([O._f64(inp.v[s]), O._f64(inp.v_dec[:steps, s])], axis=0)
            local = int(inp.policy[s]) == LOCAL
            for t in range(steps):
                idx = (O.sliding_local_indices(L, t, wl.local_window) if local
                       else np.concatenate([res.sel[s], np.arange(L, L + t + 1)]))
                q = O._f64(inp.q_dec[t, s * G:(s + 1) * G])
                res.out[(t, s)] = O.decode_attention(q, kf[idx], vf[idx], [0, idx.size], [idx.size], G)
        return res

    if steps > 0:
        for s in slots:
            idx = res.sel[s]
            ks = O._f64(inp.k[s])[idx]
            vs = O._f64(inp.v[s])[idx]
            kn = O._f64(inp.k_dec[:steps, s])
            vn = O._f64(inp.v_dec[:steps, s])
            keys = np.concatenate([ks, kn], axis=0)
            vals = np.concatenate([vs, vn], axis=0)
            n0 = ks.shape[0]
            for t in range(steps):
                q = O._f64(inp.q_dec[t, s * G:(s + 1) * G])
                n = n0 + t + 1
                off = np.array([0, n], dtype=np.int64)
                ln = np.array([n], dtype=np.int64)
                res.out[(t, s)] = O.decode_attention(q, keys[:n], vals[:n], off, ln, G)
    return res
