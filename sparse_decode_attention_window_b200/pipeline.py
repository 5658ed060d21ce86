"""One workload through the C ABI: window scoring -> selection (-> ZigZagKV
allocation) -> layout -> compaction, then per decode step append -> decode.

With decode-time chunk re-selection (ChunkLLM's ICAC, Section 2.3) the full cache is
kept as well: every step appends to it, and a step whose token closes a chunk re-scores
all chunks with that step's query, re-selects them and re-compacts the attended cache
from the full one - the same calls as the prompt's, over the grown chunk list.

Host-side orchestration only: buffers are torch CUDA tensors allocated once,
every step is a libkvc call on one stream.
"""
from __future__ import annotations

import torch

import math

from . import (kvc_score, kvc_select, kvc_alloc_budgets, kvc_layout_compact, kvc_append, kvc_decode_attn,
               kvc_append_decode, kvc_append_decode_chain, kvc_select_chunks, kvc_append_window, KVC_POL_LOCAL,
               kvc_workspace_size, make_shape, KVC_WS_SCORE, KVC_WS_DECODE, KVC_POL_TOPB, KVC_POL_MASS_COUNT,
               KVC_POL_CHUNK)


def _round16(x: int) -> int:
    return (x + 15) // 16 * 16


class KvcPipeline:
    """Buffers and call sequence for one workload (see workloads.configs).

    `inp` is a workloads.Inputs whose tensors are on the target CUDA device.
    `decode_boundaries`: for a chunk workload with `icac`, the decode steps whose token
    closes a chunk (the chunk-boundary predictions the method receives).
    """

    def __init__(self, wl, inp, device=None, decode_boundaries=None):
        self.wl = wl
        self.inp = inp
        self._chained = False              # True while the last kernel issued was a decode step's
        dev = torch.device(device) if device is not None else inp.k.device
        self.dev = dev
        S, G, d, L = wl.n_slots, wl.G, wl.d, wl.L
        dt = inp.k.dtype
        self.shape = make_shape(S, G, d, L, wl.w, wl.hkv, wl.batch, dt)
        i32 = dict(dtype=torch.int32, device=dev)
        self.chunk_end = inp.chunk_end
        self.C = int(inp.chunk_end.numel()) if inp.chunk_end is not None else 0
        if wl.w > 0:
            N = self.C if wl.policy == "chunk" else L
            self.score = torch.empty((S, N), dtype=torch.float32, device=dev)
            self.ws_score = torch.zeros(kvc_workspace_size(KVC_WS_SCORE, self.shape, self.C), dtype=torch.uint8,
                                        device=dev)
        else:
            self.score = None
        self.max_sel = min(wl.top_b, L) if wl.policy == "topb" else L
        self.idx = torch.empty((S, self.max_sel), **i32)
        self.count = torch.empty((S,), **i32)
        self.budget = torch.empty((S,), **i32)
        self.policy = torch.empty((S,), dtype=torch.int8, device=dev)
        if wl.policy == "topb":
            self.policy.fill_(KVC_POL_TOPB)
            self.budget.fill_(wl.top_b)
        elif wl.policy == "zigzag":
            self.mass_count = torch.empty((S,), **i32)
            self.layer_budget = torch.empty((wl.n_layers,), **i32)
            self.pol_mass = torch.full((S,), KVC_POL_MASS_COUNT, dtype=torch.int8, device=dev)
            self.policy.fill_(KVC_POL_TOPB)
        elif wl.policy == "fastgen":
            self.policy.copy_(inp.policy)
            self.budget.fill_(wl.local_window)
        elif wl.policy == "chunk":
            self.policy.fill_(KVC_POL_CHUNK)
            self.budget.fill_(wl.chunk_target)
        self.off = torch.empty((S + 1,), dtype=torch.int64, device=dev)
        self.cap = torch.empty((S,), **i32)
        self.len = torch.empty((S,), **i32)
        self.kp_rows = S * _round16(self.max_sel + wl.reserve)
        self.kp = torch.empty((self.kp_rows, d), dtype=dt, device=dev)
        self.vp = torch.empty((self.kp_rows, d), dtype=dt, device=dev)
        self.out = torch.empty((S * G, d), dtype=torch.float32, device=dev)
        self.ws_decode = torch.zeros(kvc_workspace_size(KVC_WS_DECODE, self.shape), dtype=torch.uint8, device=dev)
        self.icac = bool(getattr(wl, "icac", False)) and wl.policy == "chunk"
        if self.icac:
            self._init_icac(decode_boundaries or [])
        # FastGen local heads that keep evicting while decoding: their rows form a ring
        self.sliding = bool(getattr(wl, "local_sliding", False)) and wl.policy == "fastgen"
        if self.sliding:
            self.window = torch.where(inp.policy.to(dev) == KVC_POL_LOCAL, wl.local_window, 0).to(torch.int32)
            self.head = torch.zeros((S,), **i32)

    def _init_icac(self, boundaries):
        wl, inp, dev = self.wl, self.inp, self.dev
        S, G, d, L = wl.n_slots, wl.G, wl.d, wl.L
        dt = inp.k.dtype
        i32 = dict(dtype=torch.int32, device=dev)
        self.boundaries = sorted(int(b) for b in boundaries if 0 <= int(b) < wl.steps)
        self.Lmax = _round16(L + wl.steps)
        # the full cache: prompt keys/values plus every generated token, a packed layout
        # with one Lmax-row region per slot
        self.kf = torch.zeros((S, self.Lmax, d), dtype=dt, device=dev)
        self.vf = torch.zeros((S, self.Lmax, d), dtype=dt, device=dev)
        self.kf[:, :L].copy_(inp.k)
        self.vf[:, :L].copy_(inp.v)
        self.off_f = torch.arange(0, (S + 1) * self.Lmax, self.Lmax, dtype=torch.int64, device=dev)
        self.cap_f = torch.full((S,), self.Lmax, **i32)
        self.len_f = torch.full((S,), L, **i32)
        # chunk list: the prompt's chunks, then one per boundary (token L + t closes it)
        ends = inp.chunk_end.to(torch.int64).cpu().tolist() + [L + t for t in self.boundaries]
        self.ends_all = torch.tensor(ends, **i32)
        self.C0 = self.C
        Cmax = len(ends)
        self.shape_full = make_shape(S, G, d, self.Lmax, 1, wl.hkv, wl.batch, dt)   # k stride Lmax, one query row
        self.score_f = torch.empty((S * Cmax,), dtype=torch.float32, device=dev)
        self.ws_score_f = torch.zeros(kvc_workspace_size(KVC_WS_SCORE, self.shape_full, Cmax), dtype=torch.uint8,
                                      device=dev)
        # per boundary: the token target ceil(keep_frac * current length)
        self.targets = torch.tensor([[math.ceil(wl.keep_frac * (L + t + 1))] * S for t in self.boundaries] or [[0] * S],
                                    **i32)
        self.prompt_target = torch.full((S,), wl.chunk_target, **i32)
        # the attended cache and the selection can now hold any token of the full cache
        self.max_sel = self.Lmax
        self.idx = torch.empty((S, self.max_sel), **i32)
        self.kp_rows = S * _round16(self.Lmax + wl.reserve)
        self.kp = torch.empty((self.kp_rows, d), dtype=dt, device=dev)
        self.vp = torch.empty((self.kp_rows, d), dtype=dt, device=dev)

    # ---- the hot path
    def score_step(self, stream=None):
        wl, inp = self.wl, self.inp
        if wl.policy == "chunk":
            kvc_score(self.shape, inp.q_win, inp.k, self.score, self.ws_score, chunk_end=self.chunk_end, C=self.C,
                      stream=stream)
        elif wl.w > 0:
            kvc_score(self.shape, inp.q_win, inp.k, self.score, self.ws_score, stream=stream)

    def select_step(self, stream=None):
        wl, inp = self.wl, self.inp
        if wl.policy == "zigzag":
            kvc_select(self.shape, self.score, self.pol_mass, self.budget, None, self.mass_count, mass=wl.mass,
                       stream=stream)
            kvc_alloc_budgets(self.mass_count, wl.n_layers, wl.slots_per_layer, wl.L, wl.avg_budget,
                              wl.floor_budget, self.layer_budget, self.budget, stream=stream)
            kvc_select(self.shape, self.score, self.policy, self.budget, self.idx, self.count, stream=stream)
        elif wl.policy == "fastgen":
            kvc_select(self.shape, None, self.policy, self.budget, self.idx, self.count,
                       special_mask=inp.special_mask, stream=stream)
        elif wl.policy == "chunk" and self.icac:
            kvc_select_chunks(self.shape, self.score, self.chunk_end, self.prompt_target, self.idx, self.count,
                              n_local=wl.n_local, stream=stream)
        elif wl.policy == "chunk":
            kvc_select(self.shape, self.score, self.policy, self.budget, self.idx, self.count,
                       chunk_end=self.chunk_end, C=self.C, stream=stream)
        else:
            kvc_select(self.shape, self.score, self.policy, self.budget, self.idx, self.count, stream=stream)

    def compact_step(self, stream=None):
        if self.icac:
            self.len_f.fill_(self.wl.L)    # the full cache restarts from the prompt
        if self.sliding:
            self.head.zero_()              # compaction stores a local head's window oldest first
        kvc_layout_compact(self.shape, self.inp.k, self.inp.v, self.idx, self.count, self.wl.reserve, self.off,
                           self.cap, self.kp, self.vp, self.len, stream=stream)
        self._chained = False              # the next decode follows a kernel that wrote the kept rows

    def compress(self, stream=None):
        self.score_step(stream)
        self.select_step(stream)
        self.compact_step(stream)

    def decode_step(self, t: int, q=None, k_new=None, v_new=None, out=None, fused=True, stream=None):
        """Append the step's new token to every slot, then decode. `fused` uses the
        one-launch kvc_append_decode; otherwise kvc_append then kvc_decode_attn."""
        inp = self.inp
        q = inp.q_dec[t] if q is None else q
        k_new = inp.k_dec[t] if k_new is None else k_new
        v_new = inp.v_dec[t] if v_new is None else v_new
        out = self.out if out is None else out
        if self.icac:
            kvc_append(self.shape, k_new, v_new, self.off_f, self.cap_f, self.len_f, self.kf.view(-1, self.wl.d),
                       self.vf.view(-1, self.wl.d), stream=stream)
        if self.sliding:
            # append (a full local window overwrites its oldest row), then decode
            kvc_append_window(self.shape, k_new, v_new, self.off, self.cap, self.len, self.window, self.head,
                              self.kp, self.vp, stream=stream)
            kvc_decode_attn(self.shape, q, self.kp, self.vp, self.off, self.len, out, self.ws_decode, stream=stream)
        elif fused and self._chained:
            # the previous step's launch wrote only its appended rows: the kept rows
            # [0, count) may be loaded before it ends
            kvc_append_decode_chain(self.shape, k_new, v_new, q, self.kp, self.vp, self.off, self.cap, self.count,
                                    self.len, out, self.ws_decode, stream=stream)
        elif fused:
            kvc_append_decode(self.shape, k_new, v_new, q, self.kp, self.vp, self.off, self.cap, self.len, out,
                              self.ws_decode, stream=stream)
            self._chained = True
        else:
            kvc_append(self.shape, k_new, v_new, self.off, self.cap, self.len, self.kp, self.vp, stream=stream)
            kvc_decode_attn(self.shape, q, self.kp, self.vp, self.off, self.len, out, self.ws_decode, stream=stream)
        if self.icac and t in self.boundaries:
            self.reselect_step(t, q, stream)
        return out

    def reselect_step(self, t: int, q, stream=None):
        """Token L + t closed a chunk: score every chunk with this step's query (a window
        of one row over the chunk keys of the full cache), re-select and re-compact the
        attended cache from the full cache, with room for the remaining steps."""
        wl = self.wl
        S, G, d = wl.n_slots, wl.G, wl.d
        i = self.boundaries.index(t)
        C = self.C0 + i + 1
        n = wl.L + t + 1
        ends = self.ends_all[:C]
        score = self.score_f[:S * C].view(S, C)
        kvc_score(self.shape_full, q.view(S * G, 1, d), self.kf, score, self.ws_score_f, chunk_end=ends, C=C,
                  stream=stream)
        shape_n = make_shape(S, G, d, n, 1, wl.hkv, wl.batch, self.kf.dtype)   # n tokens to choose from
        kvc_select_chunks(shape_n, score, ends, self.targets[i], self.idx, self.count, n_local=wl.n_local,
                          stream=stream)
        kvc_layout_compact(self.shape_full, self.kf, self.vf, self.idx, self.count, wl.steps - t - 1, self.off,
                           self.cap, self.kp, self.vp, self.len, stream=stream)
        self._chained = False

    def run(self, steps=None, record=False, stream=None):
        self.compress(stream)
        outs = []
        n = self.wl.steps if steps is None else steps
        for t in range(n):
            o = self.decode_step(t, stream=stream)
            if record:
                outs.append(o.clone())
        return outs
