"""kvc_decode_attn_noalloc: the decode entry point for callers that cannot allocate
device memory (for example an operator handed only its inputs and outputs by a
runtime that owns all device buffers). Its scratch is a fixed array inside the
library instead of a caller workspace.

Checked through the C ABI against kvc_decode_attn (same kernel, caller workspace)
on two calls in a row - the second call must not see the first call's leftovers -
within the decode tolerance the parity tests use. This file runs last; it must
pass alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

from tests import parity as P

pytestmark = pytest.mark.gpu


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
    rows = int(off[-1])
    kp = torch.randn((rows, d), generator=g, device="cuda").to(torch.bfloat16)
    vp = torch.randn((rows, d), generator=g, device="cuda").to(torch.bfloat16)
    return kvc, sh, count, off, kp, vp


def test_noalloc_decode_matches_workspace_decode_twice():
    # ragged lengths, long enough that several CTAs share each slot and merge partials
    kvc, sh, count, off, kp, vp = _case([9000, 17, 2500, 40000, 1, 700])
    S, G, d = sh.n_slots, sh.G, sh.d
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    for call in range(2):
        q = torch.randn((S * G, d), device="cuda").to(torch.bfloat16)
        ref = torch.empty((S * G, d), device="cuda")
        got = torch.full((S * G, d), float("nan"), device="cuda")
        kvc.kvc_decode_attn(sh, q, kp, vp, off, count, ref, ws)
        kvc.kvc_decode_attn_noalloc(sh, q, kp, vp, off, count, got)
        torch.cuda.synchronize()
        kvc.kvc_get_status()
        P.check_out(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "bf16", f"call {call}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import sparse_decode_attention_window_b200 as kvc
    # 4096 slots of G = 4, d = 128 need more than the fixed 4 MiB of scratch
    sh = kvc.make_shape(4096, 4, 128, 64, 0, 4096, 1, torch.bfloat16)
    assert kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh) > (4 << 20)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(16, dtype=torch.int64, device="cuda")
    ln = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_decode_attn_noalloc(sh, t, t.view(1, 16), t.view(1, 16), o, ln, out)
    assert e.value.status == 6 and "scratch" in str(e.value)
