"""kvc_decode_attn_noalloc: the decode entry point for callers that cannot allocate
device memory (for example an operator handed only its inputs and outputs by a
runtime that owns all device buffers, so it has no allocator and no workspace
handle). Its scratch is a fixed array inside the library instead of a caller
workspace.

Checked through the C ABI on two calls in a row - the second call must not see the
first call's leftovers - against kvc_decode_attn (the same kernel with a caller
workspace) and against the fp64 oracle, within the decode tolerance the parity tests
use; at a ragged shape and at the largest shape whose scratch still fits the fixed
array (one slot more is rejected). This file runs last; it must pass alone in a fresh
process as well as after the other tests."""
import numpy as np
import pytest
import torch

import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20    # the fixed array's size, as include/kvc.h states it


def _case(lens, G=4, d=128, seed=0):
    import sparse_decode_attention_window_b200 as kvc
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    S = len(lens)
    sh = kvc.make_shape(S, G, d, max(lens) + 16, 0, S, 1, torch.bfloat16)
    count = torch.tensor(lens, dtype=torch.int32, device="cuda")
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 0, off, cap)
    rows = max(int(off[-1]), 1)
    kp = torch.randn((rows, d), generator=g, device="cuda").to(torch.bfloat16)
    vp = torch.randn((rows, d), generator=g, device="cuda").to(torch.bfloat16)
    return kvc, sh, count, off, kp, vp


def _two_calls(kvc, sh, count, off, kp, vp, oracle_slots):
    S, G, d = sh.n_slots, sh.G, sh.d
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    offs, lens = off.cpu().numpy(), count.cpu().numpy()
    kh, vh = kp.cpu(), vp.cpu()
    for call in range(2):
        q = torch.randn((S * G, d), device="cuda").to(torch.bfloat16)
        ref = torch.empty((S * G, d), device="cuda")
        got = torch.full((S * G, d), float("nan"), device="cuda")
        kvc.kvc_decode_attn(sh, q, kp, vp, off, count, ref, ws)
        kvc.kvc_decode_attn_noalloc(sh, q, kp, vp, off, count, got)
        torch.cuda.synchronize()
        kvc.kvc_get_status()
        g_np = got.cpu().numpy()
        P.check_out(g_np, ref.cpu().numpy().astype(np.float64), "bf16", f"call {call} vs kvc_decode_attn")
        qh = q.cpu()
        for s in oracle_slots:
            n, o = int(lens[s]), int(offs[s])
            if n == 0:
                assert np.all(g_np[s * G:(s + 1) * G] == 0.0), f"call {call}: empty slot {s} not zero"
                continue
            want = O.decode_attention(qh[s * G:(s + 1) * G], kh[o:o + n], vh[o:o + n], [0, n], [n], G)
            P.check_out(g_np[s * G:(s + 1) * G], want, "bf16", f"call {call} slot {s} vs oracle")


def test_noalloc_decode_matches_workspace_decode_and_oracle_twice():
    # ragged lengths, long enough that several CTAs share each slot and merge partials
    kvc, sh, count, off, kp, vp = _case([9000, 17, 2500, 40000, 1, 700])
    _two_calls(kvc, sh, count, off, kp, vp, range(sh.n_slots))


def _largest_fitting_slot_count(kvc, G, d):
    def need(S):
        return kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, kvc.make_shape(S, G, d, 64, 0, S, 1, torch.bfloat16))
    lo, hi = 1, 4096               # need(lo) fits, need(hi) does not (4096 slots of G = 4, d = 128)
    assert need(lo) <= SCRATCH_BYTES < need(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if need(mid) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


def test_noalloc_at_the_largest_accepted_shape_and_one_slot_more():
    import sparse_decode_attention_window_b200 as kvc
    G, d = 4, 128
    S = _largest_fitting_slot_count(kvc, G, d)
    # short ragged lengths (empty slots included) so the whole scratch layout is in use
    lens = torch.randint(0, 40, (S,), generator=torch.Generator().manual_seed(S)).tolist()
    kvc, sh, count, off, kp, vp = _case(lens, G, d, seed=1)
    _two_calls(kvc, sh, count, off, kp, vp, list(range(0, S, 61)) + [S - 1])
    # one slot more needs more scratch than the fixed array holds: rejected before any launch
    sh1 = kvc.make_shape(S + 1, G, d, 64, 0, S + 1, 1, torch.bfloat16)
    t = torch.zeros((S + 1) * G * d, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(S + 2, dtype=torch.int64, device="cuda")
    ln = torch.zeros(S + 1, dtype=torch.int32, device="cuda")
    out = torch.zeros((S + 1) * G * d, dtype=torch.float32, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_decode_attn_noalloc(sh1, t, t.view(-1, d), t.view(-1, d), o, ln, out)
    assert e.value.status == 6 and "scratch" in str(e.value)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import sparse_decode_attention_window_b200 as kvc
    # 4096 slots of G = 4, d = 128 need more than the fixed 4 MiB of scratch
    sh = kvc.make_shape(4096, 4, 128, 64, 0, 4096, 1, torch.bfloat16)
    assert kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh) > SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(16, dtype=torch.int64, device="cuda")
    ln = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_decode_attn_noalloc(sh, t, t.view(1, 16), t.view(1, 16), o, ln, out)
    assert e.value.status == 6 and "scratch" in str(e.value)
