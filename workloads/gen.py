"""Seeded synthetic inputs for the hot path.

This module is the only code shared by the CUDA path and the oracle. It draws
random numbers and shapes them into the workloads' structure (sinks, key
temperatures, policies, special-token sets, chunk boundaries); it computes no
part of the method (no attention, no selection, no compaction).

Draw order (fixed; every array comes from one torch.Generator seeded per workload):

  main generator (seed)          : q_win [nL,B,Hq,w,d], k [nL,B,Hkv,L,d], v [nL,B,Hkv,L,d],
                                   then the key temperature (U[lo,hi], one per KV head or per layer)
  decode generator (seed + 1000) : q_dec [steps, nL*B*Hq, d], k_dec, v_dec [steps, nL*B*Hkv, d]
  host generator  (seed + 2000)  : fastgen policy per slot, special positions per batch row
  host generator  (seed + 3000)  : chunk lengths ~ Geometric(1/mean) on {1, 2, ...}
  host generator  (seed + 4000)  : the same for the generated tokens (chunk_icac)

All draws are fp32 N(0, 1) (or U for temperatures); bf16 workloads round the final
fp32 values to the nearest bf16 (ties to even), so both sides read identical values.
Generation may run on the CPU or on the GPU; a given test or run uses one set of
arrays for both the CUDA path and the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from .configs import Workload

# policy codes shared by the binding and the oracle's callers
POL_TOPB, POL_MASS_COUNT, POL_LOCAL, POL_SPECIAL, POL_FULL, POL_CHUNK = 0, 1, 2, 3, 4, 5


@dataclass
class Inputs:
    wl: Workload
    q_win: torch.Tensor | None    # [S*G, w, d]  (slot-major: layer, batch, kv head, group member)
    k: torch.Tensor               # [S, L, d]
    v: torch.Tensor               # [S, L, d]
    q_dec: torch.Tensor           # [steps, S*G, d]
    k_dec: torch.Tensor           # [steps, S, d]
    v_dec: torch.Tensor           # [steps, S, d]
    policy: torch.Tensor | None   # int8 [S] (fastgen)
    special_mask: torch.Tensor | None  # uint8 [B, L] (fastgen)
    chunk_end: torch.Tensor | None     # int32 [C] (chunk)


def _torch_dtype(wl: Workload):
    return torch.float32 if wl.dtype == "fp32" else torch.bfloat16


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(wl: Workload, device="cpu") -> Inputs:
    device = torch.device(device)
    dt = _torch_dtype(wl)
    nL, B, Hq, Hkv, L, d, w, G = wl.n_layers, wl.batch, wl.hq, wl.hkv, wl.L, wl.d, wl.w, wl.G
    S = wl.n_slots
    g = _gen(wl.seed, device)

    q_win = None
    if w > 0:
        q_win = torch.randn((nL, B, Hq, w, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((nL, B, Hkv, L, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((nL, B, Hkv, L, d), generator=g, device=device, dtype=torch.float32)

    if wl.key_temp:
        lo, hi = wl.key_temp
        n = Hkv if wl.key_temp_per == "kv_head" else nL
        tau = lo + (hi - lo) * torch.rand((n,), generator=g, device=device, dtype=torch.float32)
        if wl.key_temp_per == "kv_head":
            k *= tau.view(1, 1, Hkv, 1, 1)
        else:
            k *= tau.view(nL, 1, 1, 1, 1)

    if wl.n_sinks > 0:
        # keys of tokens 0..n_sinks-1 point along the unit mean of the slot's
        # window queries, with length 4*sqrt(d): logits ~ 4 * q . u_hat
        qg = q_win.view(nL, B, Hkv, G * w, d)
        u = qg.mean(dim=3)
        u = u / u.norm(dim=-1, keepdim=True)
        k[:, :, :, : wl.n_sinks, :] = (4.0 * math.sqrt(d)) * u.unsqueeze(3)

    if q_win is not None:
        q_win = q_win.to(dt).reshape(S * G, w, d).contiguous()
    k = k.to(dt).reshape(S, L, d).contiguous()
    v = v.to(dt).reshape(S, L, d).contiguous()

    gd = _gen(wl.seed + 1000, device)
    q_dec = torch.randn((wl.steps, S * G, d), generator=gd, device=device).to(dt)
    k_dec = torch.randn((wl.steps, S, d), generator=gd, device=device).to(dt)
    v_dec = torch.randn((wl.steps, S, d), generator=gd, device=device).to(dt)

    policy = special_mask = chunk_end = None
    if wl.policy == "fastgen":
        policy, special_mask = fastgen_policies(wl)
        policy = policy.to(device)
        special_mask = special_mask.to(device)
    if wl.policy == "chunk":
        chunk_end = chunk_boundaries(wl).to(device)

    return Inputs(wl, q_win, k, v, q_dec, k_dec, v_dec, policy, special_mask, chunk_end)


def fastgen_policies(wl: Workload):
    """Per-slot head policy, uniform over {local, special, full}, and the special
    token set of each batch row: sinks 0..3 plus a seeded draw without replacement
    of round(special_frac * L) positions from [4, L)."""
    gh = _gen(wl.seed + 2000, "cpu")
    choices = torch.tensor([POL_LOCAL, POL_SPECIAL, POL_FULL], dtype=torch.int8)
    pick = torch.randint(0, 3, (wl.n_slots,), generator=gh)
    policy = choices[pick].contiguous()
    mask = torch.zeros((wl.batch, wl.L), dtype=torch.uint8)
    n_sinks = 4
    for b in range(wl.batch):
        mask[b, :n_sinks] = 1
        perm = torch.randperm(wl.L - n_sinks, generator=gh)[: wl.n_special] + n_sinks
        mask[b, perm] = 1
    return policy, mask


def chunk_boundaries(wl: Workload) -> torch.Tensor:
    """Chunk lengths ~ Geometric(p = 1/mean) on {1, 2, ...} by inverse CDF, drawn
    until they cover L; the last chunk is cut at L. Returns the last position of
    each chunk (int32, strictly increasing, ends at L-1)."""
    gh = _gen(wl.seed + 3000, "cpu")
    p = 1.0 / wl.chunk_mean
    ends = []
    pos = -1
    log1mp = math.log1p(-p)
    while pos < wl.L - 1:
        draw = torch.rand((4096,), generator=gh, dtype=torch.float64)
        u = 1.0 - draw                      # in (0, 1]
        lens = torch.floor(torch.log(u) / log1mp).to(torch.int64) + 1
        for ln in lens.tolist():
            pos = min(pos + int(ln), wl.L - 1)
            ends.append(pos)
            if pos >= wl.L - 1:
                break
    return torch.tensor(ends, dtype=torch.int32)


def decode_chunk_boundaries(wl: Workload) -> list:
    """Decode steps whose generated token closes a chunk: the chunk process of
    `chunk_boundaries` continued past the prompt (its last chunk ends at L - 1), with
    lengths ~ Geometric(p = 1/mean) from its own generator. Step t appends position L + t."""
    gh = _gen(wl.seed + 4000, "cpu")
    p = 1.0 / wl.chunk_mean
    log1mp = math.log1p(-p)
    steps = []
    pos = wl.L - 1
    while True:
        draw = torch.rand((256,), generator=gh, dtype=torch.float64)
        lens = torch.floor(torch.log(1.0 - draw) / log1mp).to(torch.int64) + 1
        for ln in lens.tolist():
            pos += int(ln)
            t = pos - wl.L
            if t >= wl.steps:
                return steps
            steps.append(t)
