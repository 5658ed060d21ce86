"""CUDA path vs the fp64 oracle, through the C ABI, on the same seeded inputs.

Small workloads are checked on every slot and step; the full-size workloads run
in the same launch configuration the benchmark times and are checked on sampled
slots and steps (the oracle computes them one by one)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from workloads import get, make_inputs, POL_LOCAL, POL_SPECIAL
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_decode_attention_window_b200 as kvc
    kvc.library()
    yield


def _np(t):
    return t.detach().cpu().numpy()


def run_and_check(wl, slots=None, steps=None, gen_device="cpu", check_scores=True, fused=True):
    """Run the workload through the ABI and check it against the oracle.
    slots: slots to check (default all); steps: decode steps to check (default all)."""
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    import sparse_decode_attention_window_b200 as kvc

    if gen_device == "cpu":
        from dataclasses import replace
        inp_host = make_inputs(wl, "cpu")
        inp = replace(inp_host, **{f: (getattr(inp_host, f).cuda() if getattr(inp_host, f) is not None else None)
                                   for f in ("q_win", "k", "v", "q_dec", "k_dec", "v_dec", "policy",
                                             "special_mask", "chunk_end")})
    else:
        inp = inp_host = make_inputs(wl, "cuda")
    S, G, L, d = wl.n_slots, wl.G, wl.L, wl.d
    slots = list(range(S)) if slots is None else list(slots)
    steps = list(range(wl.steps)) if steps is None else list(steps)

    pipe = KvcPipeline(wl, inp)
    pipe.compress()
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    count = _np(pipe.count).astype(np.int64)
    idx = _np(pipe.idx)
    off, cap, ln = _np(pipe.off), _np(pipe.cap), _np(pipe.len)

    # layout: exact given the GPU counts
    ref_off, ref_cap = O.layout(count, wl.reserve)
    np.testing.assert_array_equal(off, ref_off)
    np.testing.assert_array_equal(cap, ref_cap)
    np.testing.assert_array_equal(ln, count)

    k_cpu = lambda s: inp.k[s].cpu()
    qw_cpu = lambda s: inp.q_win[s * G:(s + 1) * G].cpu()
    ce = _np(inp.chunk_end) if inp.chunk_end is not None else None
    sc_gpu = _np(pipe.score) if pipe.score is not None else None

    ref_scores = {}
    if wl.w > 0:
        for s in slots:
            if wl.policy == "chunk":
                ref_scores[s] = O.chunk_scores(qw_cpu(s), k_cpu(s)[None], L, ce)[0]
            else:
                ref_scores[s] = O.window_scores(qw_cpu(s), k_cpu(s)[None], L)[0]
            if check_scores:
                P.check_scores(sc_gpu[s], ref_scores[s], wl.dtype, f"score slot {s}")

    if wl.policy == "zigzag":
        mc = _np(pipe.mass_count).astype(np.int64)
        for s in slots:
            P.check_mass_count(int(mc[s]), ref_scores[s], wl.mass, f"LMBA slot {s}")
        ref_budget = O.allocate_budgets(mc.reshape(wl.n_layers, wl.slots_per_layer), L, wl.avg_budget,
                                        wl.floor_budget)
        np.testing.assert_array_equal(_np(pipe.layer_budget), ref_budget)
        np.testing.assert_array_equal(_np(pipe.budget), np.repeat(ref_budget, wl.slots_per_layer))

    for s in slots:
        got = idx[s, :count[s]].astype(np.int64)
        if wl.policy == "topb":
            P.check_topb(got, ref_scores[s], wl.top_b, f"top-B slot {s}")
        elif wl.policy == "zigzag":
            P.check_topb(got, ref_scores[s], int(_np(pipe.layer_budget)[s // wl.slots_per_layer]), f"slot {s}")
        elif wl.policy == "fastgen":
            pol = int(inp_host.policy[s])
            b = (s // wl.hkv) % wl.batch
            if pol == POL_LOCAL:
                want = O.local_indices(L, wl.local_window)
            elif pol == POL_SPECIAL:
                want = O.special_indices(_np(inp.special_mask[b]))
            else:
                want = O.full_indices(L)
            np.testing.assert_array_equal(got, want, err_msg=f"policy slot {s}")
        elif wl.policy == "chunk":
            P.check_chunks(got, ref_scores[s], ce, wl.chunk_target, f"chunks slot {s}")
        # packed rows are the kept rows, bit for bit
        o, n = int(off[s]), int(count[s])
        gi = torch.from_numpy(got).to(inp.k.device)
        assert torch.equal(pipe.kp[o:o + n], inp.k[s].index_select(0, gi)), f"packed K slot {s}"
        assert torch.equal(pipe.vp[o:o + n], inp.v[s].index_select(0, gi)), f"packed V slot {s}"

    # decode: the oracle attends over the GPU's (checked) selection plus the appended tokens
    worst = 0.0
    want_steps = set(steps)
    outs = {}
    for t in range(max(steps) + 1 if steps else 0):
        o_t = pipe.decode_step(t, fused=fused)
        if t in want_steps:
            outs[t] = _np(o_t).copy()
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    for s in slots:
        sel = idx[s, :count[s]].astype(np.int64)
        ks = O._f64(inp.k[s].cpu())[sel]
        vs = O._f64(inp.v[s].cpu())[sel]
        kn = O._f64(inp.k_dec[:, s].cpu())
        vn = O._f64(inp.v_dec[:, s].cpu())
        for t in sorted(want_steps):
            keys = np.concatenate([ks, kn[:t + 1]])
            vals = np.concatenate([vs, vn[:t + 1]])
            n = keys.shape[0]
            q = O._f64(inp.q_dec[t, s * G:(s + 1) * G].cpu())
            ref = O.decode_attention(q, keys, vals, [0, n], [n], G)
            worst = max(worst, P.check_out(outs[t][s * G:(s + 1) * G], ref, wl.dtype, f"decode slot {s} step {t}"))
    return pipe, worst


# ---------------------------------------------------------------- the workloads, small
def test_tiny_workload_all_slots_all_steps():
    run_and_check(get("tiny"))


@pytest.mark.parametrize("L,top_b", [(1024, 128), (1000, 64)])
def test_llama8b_shape_small_context(L, top_b):
    run_and_check(get("llama8b").scaled(batch=2, L=L, top_b=top_b, steps=6))


def test_zigzag_small():
    run_and_check(get("zigzag").scaled(n_layers=4, L=2048, steps=5))


def test_fastgen_small():
    run_and_check(get("fastgen").scaled(batch=2, L=3000, steps=7))


def test_chunk_small():
    run_and_check(get("chunk").scaled(L=6000, steps=5))


# ---------------------------------------------------------------- full sizes (benchmark launch configuration)
def test_llama8b_full_size():
    wl = get("llama8b")
    run_and_check(wl, slots=range(wl.n_slots), steps=[0, 31, 63], gen_device="cuda")


def test_zigzag_full_size_sampled():
    wl = get("zigzag")
    rng = np.random.default_rng(0)
    slots = sorted(rng.choice(wl.n_slots, size=12, replace=False).tolist())
    run_and_check(wl, slots=slots, steps=[0, 31], gen_device="cuda")


def test_fastgen_full_size_sampled():
    wl = get("fastgen")
    run_and_check(wl, slots=[0, 5, 17, 33, 50, 63], steps=[0, 127], gen_device="cuda")


def test_chunk_full_size_sampled():
    wl = get("chunk")
    run_and_check(wl, slots=[0, 3, 7], steps=[0, 255], gen_device="cuda")


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("L", [1, 7, 255, 256, 257, 4099])
def test_ragged_context_lengths(L):
    w = min(4, L)
    run_and_check(get("llama8b").scaled(batch=1, hq=8, hkv=2, L=L, w=w, top_b=max(1, L // 3), steps=2))


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (8, 2)])
def test_gqa_group_sizes(hq, hkv):
    run_and_check(get("llama8b").scaled(batch=1, hq=hq, hkv=hkv, L=600, w=8, top_b=100, steps=3))


@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (128, "fp32")])
def test_head_dims_and_dtypes(d, dtype):
    run_and_check(get("llama8b").scaled(batch=1, d=d, dtype=dtype, L=700, w=16, top_b=90, steps=3))


def test_window_of_one():
    run_and_check(get("llama8b").scaled(batch=1, L=513, w=1, top_b=50, steps=2))


@pytest.mark.parametrize("top_b", [1, 511, 512, 100000])
def test_budget_extremes(top_b):
    run_and_check(get("llama8b").scaled(batch=1, L=512, w=8, top_b=top_b, steps=2))


def test_mass_count_closed_forms_on_gpu():
    """Uniform scores keep ceil(0.9 L); a one-hot distribution keeps one token."""
    import sparse_decode_attention_window_b200 as kvc
    L = 1000
    sh = kvc.make_shape(3, 1, 64, L, 1, 3, 1, torch.bfloat16)
    sc = torch.zeros((3, L), dtype=torch.float32, device="cuda")
    sc[0] = 1.0
    sc[1, 123] = 5.0
    sc[2] = torch.linspace(1.0, 2.0, L, device="cuda")
    pol = torch.full((3,), kvc.KVC_POL_MASS_COUNT, dtype=torch.int8, device="cuda")
    bud = torch.zeros(3, dtype=torch.int32, device="cuda")
    cnt = torch.empty(3, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, sc, pol, bud, None, cnt, mass=0.9)
    c = cnt.cpu().numpy()
    assert c[0] == 900 and c[1] == 1
    P.check_mass_count(int(c[2]), _np(sc[2]).astype(np.float64))


# slot counts whose selection runs in clusters of 16, 8, 4 and 2 CTAs per slot, and at one CTA per slot
SELECT_SHAPES = [(1, 4096), (3, 2048), (9, 2048), (18, 1000), (37, 3000), (60, 777), (150, 300), (200, 777)]


@pytest.mark.parametrize("S,N", SELECT_SHAPES)
def test_selection_policies_over_slot_counts(S, N):
    """kvc_select on given fp32 scores with many ties: top-B (ragged budgets, 0 and >= N
    included) and the FastGen policies are exact against the oracle; LMBA counts agree
    within the tie band."""
    import sparse_decode_attention_window_b200 as kvc
    g = torch.Generator().manual_seed(7919 * S + N)
    sc = torch.exp((torch.randn((S, N), generator=g) * 8).round() / 4).float()   # positive, many ties
    kinds = [kvc.KVC_POL_TOPB, kvc.KVC_POL_MASS_COUNT, kvc.KVC_POL_TOPB, kvc.KVC_POL_LOCAL,
             kvc.KVC_POL_SPECIAL, kvc.KVC_POL_FULL, kvc.KVC_POL_MASS_COUNT]
    pol = torch.tensor([kinds[s % len(kinds)] for s in range(S)], dtype=torch.int8)
    bud = torch.randint(0, N + 4, (S,), generator=g, dtype=torch.int32)
    bud[0] = N // 3
    if S > 2:
        bud[2] = 0
    if S > 9:
        bud[9] = N
    special = (torch.rand((S, N), generator=g) < 0.05).to(torch.uint8)
    sh = kvc.make_shape(S, 1, 64, N, 1, 1, S, torch.bfloat16)
    idx = torch.full((S, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, sc.cuda(), pol.cuda(), bud.cuda(), idx, cnt, mass=0.9, special_mask=special.cuda())
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    idx, cnt = _np(idx), _np(cnt)
    sc64 = sc.double().numpy()
    for s in range(S):
        k = int(pol[s])
        got = idx[s, :cnt[s]].astype(np.int64)
        if k == kvc.KVC_POL_TOPB:
            want = O.top_b(sc64[s], max(int(bud[s]), 0))
        elif k == kvc.KVC_POL_MASS_COUNT:
            P.check_mass_count(int(cnt[s]), sc64[s], 0.9, f"slot {s}")
            continue
        elif k == kvc.KVC_POL_LOCAL:
            want = O.local_indices(N, int(bud[s]))
        elif k == kvc.KVC_POL_SPECIAL:
            want = O.special_indices(special[s].numpy())
        else:
            want = O.full_indices(N)
        np.testing.assert_array_equal(got, want, err_msg=f"slot {s} policy {k}")


@pytest.mark.parametrize("S,N,bound_holds", [(200, 4100, True), (200, 4100, False), (160, 777, True)])
def test_many_slot_mass_count_and_top_b(S, N, bound_holds):
    """More slots than SMs (two 512-thread CTAs per SM, keys re-read from L2 four at a time):
    LMBA counts within the tie band and top-B sets within the tie band of the oracle, for
    window-like scores (each slot's scores sum to G w, none above it) and for scores scaled far
    above that, on 16-byte-aligned and unaligned score rows (N = 777)."""
    import sparse_decode_attention_window_b200 as kvc
    G, w = 4, 8
    g = torch.Generator().manual_seed(S * 31 + N)
    raw = torch.softmax(torch.randn((S, N), generator=g) * 3, dim=1) * (G * w)   # sums to G w per slot
    sc = (raw if bound_holds else raw * 40).float()
    if bound_holds:
        assert float(sc.max()) <= G * w
    sh = kvc.make_shape(S, G, 64, N, w, 1, S, torch.bfloat16)
    pol = torch.tensor([kvc.KVC_POL_MASS_COUNT if s % 2 else kvc.KVC_POL_TOPB for s in range(S)], dtype=torch.int8)
    bud = torch.randint(1, N, (S,), generator=g, dtype=torch.int32)
    idx = torch.full((S, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, sc.cuda(), pol.cuda(), bud.cuda(), idx, cnt, mass=0.9)
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    idx, cnt = _np(idx), _np(cnt)
    sc64 = sc.double().numpy()
    for s in range(S):
        if s % 2:
            P.check_mass_count(int(cnt[s]), sc64[s], 0.9, f"slot {s}")
        else:
            P.check_topb(idx[s, :cnt[s]].astype(np.int64), sc64[s], int(bud[s]), f"slot {s}")


@pytest.mark.parametrize("S,C", [(1, 3000), (5, 1200), (9, 2048), (40, 700), (150, 200)])
@pytest.mark.parametrize("n_local", [0, 3])
def test_chunk_selection_over_slot_counts(S, C, n_local):
    """kvc_select_chunks on given fp32 chunk scores with ties and ragged chunk lengths is
    exact against the oracle for every slot count (cluster sizes 16 down to one CTA)."""
    import sparse_decode_attention_window_b200 as kvc
    g = torch.Generator().manual_seed(104729 * S + C + n_local)
    lens = torch.randint(1, 41, (C,), generator=g)
    ce = (torch.cumsum(lens, 0) - 1).to(torch.int32)
    L = int(ce[-1]) + 1
    sc = torch.exp((torch.randn((S, C), generator=g) * 8).round() / 4).float()
    tgt = torch.randint(1, L + 4, (S,), generator=g, dtype=torch.int32)
    tgt[0] = max(1, L // 2)
    sh = kvc.make_shape(S, 1, 64, L, 1, 1, S, torch.bfloat16)
    idx = torch.full((S, L), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    kvc.kvc_select_chunks(sh, sc.cuda(), ce.cuda(), tgt.cuda(), idx, cnt, n_local=n_local)
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    idx, cnt = _np(idx), _np(cnt)
    for s in range(S):
        want, _ = O.chunk_select_local(sc[s].double().numpy(), ce.numpy(), int(tgt[s]), n_local)
        np.testing.assert_array_equal(idx[s, :cnt[s]].astype(np.int64), want, err_msg=f"slot {s}")


@pytest.mark.parametrize("S", [4, 150])
def test_selection_flags_bad_policies_and_keeps_the_other_slots(S):
    """An unknown policy code, and SPECIAL without a special mask, keep nothing for that slot
    and set the index-range flag; the other slots of the launch (clusters of CTAs for few
    slots, one CTA per slot for many) are still exact."""
    import sparse_decode_attention_window_b200 as kvc
    N = 2048
    g = torch.Generator().manual_seed(S)
    sc = torch.rand((S, N), generator=g).float()
    pol = torch.full((S,), kvc.KVC_POL_TOPB, dtype=torch.int8)
    pol[1] = 9                                     # not a policy
    pol[2] = kvc.KVC_POL_SPECIAL                   # needs a special mask: none given
    bud = torch.full((S,), 100, dtype=torch.int32)
    sh = kvc.make_shape(S, 1, 64, N, 1, 1, S, torch.bfloat16)
    idx = torch.full((S, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, sc.cuda(), pol.cuda(), bud.cuda(), idx, cnt, mass=0.9)
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_get_status()
    assert "index-out-of-range" in str(e.value) and "wait-timeout" not in str(e.value)
    c, ix = _np(cnt), _np(idx)
    assert c[1] == 0 and c[2] == 0
    for s in [0] + list(range(3, S)):
        np.testing.assert_array_equal(ix[s, :c[s]].astype(np.int64), O.top_b(sc[s].double().numpy(), 100),
                                      err_msg=f"slot {s}")
    kvc.kvc_get_status()


def test_bounded_wait_gives_up_and_leaves_the_context_usable():
    """A wait on a barrier that nothing arrives on ends after its limit with the wait-timeout
    flag; the next status read is clean and the next library call is exact."""
    import sparse_decode_attention_window_b200 as kvc
    limit_us = 2000
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    kvc.kvc_check_wait_limit(limit_us)
    t1.record()
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_get_status()
    assert "wait-timeout" in str(e.value) and "index-out-of-range" not in str(e.value)
    assert limit_us * 1e-3 <= t0.elapsed_time(t1) < 1000.0
    kvc.kvc_get_status()
    S, N = 4, 4096
    sc = torch.rand((S, N), generator=torch.Generator().manual_seed(5)).float()
    sh = kvc.make_shape(S, 1, 64, N, 1, 1, S, torch.bfloat16)
    idx = torch.full((S, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, sc.cuda(), torch.full((S,), kvc.KVC_POL_TOPB, dtype=torch.int8, device="cuda"),
                   torch.full((S,), 300, dtype=torch.int32, device="cuda"), idx, cnt)
    kvc.kvc_get_status()
    for s in range(S):
        np.testing.assert_array_equal(_np(idx)[s, :300].astype(np.int64), O.top_b(sc[s].double().numpy(), 300))


def test_one_cta_per_slot_selection_on_workloads():
    """Selection at one CTA per slot (forced here; few slots take thread-block clusters by
    default) passes the same oracle checks."""
    import subprocess
    import sys
    forced = ['--kvc-path', 'select=cta']
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "selection_policies_over_slot_counts or chunk_selection_over_slot_counts or "
                              "llama8b_shape_small_context or zigzag_small or chunk_small or budget_extremes or "
                              "mass_count_closed_forms or chunk_selection_with_local_chunks"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_empty_slot_decodes_to_zero_and_append_overflow_is_reported():
    import sparse_decode_attention_window_b200 as kvc
    S, G, d = 3, 2, 64
    sh = kvc.make_shape(S, G, d, 16, 0, S, 1, torch.bfloat16)
    count = torch.tensor([0, 5, 0], dtype=torch.int32, device="cuda")
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 0, off, cap)
    assert cap.cpu().tolist() == [0, 16, 0]
    rows = int(off[-1])
    kp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    vp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    ln = count.clone()
    q = torch.randn(S * G, d, device="cuda").to(torch.bfloat16)
    out = torch.full((S * G, d), 7.0, device="cuda")
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    kvc.kvc_decode_attn(sh, q, kp, vp, off, ln, out, ws)
    o = _np(out)
    assert (o[0:2] == 0).all() and (o[4:6] == 0).all()
    ref = O.decode_attention(q[2:4].cpu(), kp[:5].cpu(), vp[:5].cpu(), [0, 5], [5], G)
    P.check_out(o[2:4], ref, "bf16")
    # slot 0 and 2 have capacity 0: appending overflows there (reported, not faulted)
    kn = torch.randn(S, d, device="cuda").to(torch.bfloat16)
    kvc.kvc_append(sh, kn, kn, off, cap, ln, kp, vp)
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_get_status()
    assert e.value.status == 7 and "append-overflow" in str(e.value)
    assert ln.cpu().tolist() == [0, 6, 0]
    kvc.kvc_get_status()   # the word was cleared


def test_special_policy_with_no_special_tokens():
    import sparse_decode_attention_window_b200 as kvc
    L = 300
    sh = kvc.make_shape(2, 1, 64, L, 0, 2, 1, torch.bfloat16)
    mask = torch.zeros((1, L), dtype=torch.uint8, device="cuda")
    pol = torch.full((2,), kvc.KVC_POL_SPECIAL, dtype=torch.int8, device="cuda")
    bud = torch.zeros(2, dtype=torch.int32, device="cuda")
    idx = torch.full((2, L), -1, dtype=torch.int32, device="cuda")
    cnt = torch.empty(2, dtype=torch.int32, device="cuda")
    kvc.kvc_select(sh, None, pol, bud, idx, cnt, special_mask=mask)
    assert cnt.cpu().tolist() == [0, 0]


def test_decode_is_independent_of_how_tokens_split_over_ctas():
    """The same slot decoded alone and next to other slots (different CTA ranges) agrees."""
    import sparse_decode_attention_window_b200 as kvc
    d, G = 128, 4
    torch.manual_seed(0)
    lens = [5000, 3, 777, 12000]
    S = len(lens)
    sh = kvc.make_shape(S, G, d, 16384, 0, S, 1, torch.bfloat16)
    count = torch.tensor(lens, dtype=torch.int32, device="cuda")
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 0, off, cap)
    rows = int(off[-1])
    kp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    vp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    q = torch.randn(S * G, d, device="cuda").to(torch.bfloat16)
    out = torch.empty((S * G, d), device="cuda")
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    kvc.kvc_decode_attn(sh, q, kp, vp, off, count, out, ws)
    sh1 = kvc.make_shape(1, G, d, 16384, 0, 1, 1, torch.bfloat16)
    for s in range(S):
        o1 = torch.empty((G, d), device="cuda")
        o_s = int(off[s])
        off1 = torch.tensor([0, int(cap[s])], dtype=torch.int64, device="cuda")
        kvc.kvc_decode_attn(sh1, q[s * G:(s + 1) * G].contiguous(), kp[o_s:].contiguous(), vp[o_s:].contiguous(),
                            off1, count[s:s + 1].clone(), o1, ws)
        P.check_out(_np(o1), _np(out[s * G:(s + 1) * G]).astype(np.float64), "bf16", f"slot {s}")
        ref = O.decode_attention(q[s * G:(s + 1) * G].cpu(), kp[o_s:o_s + lens[s]].cpu(), vp[o_s:o_s + lens[s]].cpu(),
                                 [0, lens[s]], [lens[s]], G)
        P.check_out(_np(out[s * G:(s + 1) * G]), ref, "bf16", f"slot {s} vs oracle")


@pytest.mark.parametrize("G,S,fused", [(4, 4096, True), (8, 2500, False), (2, 4096, False)])
def test_maximum_slot_counts(G, S, fused):
    """Large slot counts (up to the 4096 the decode takes): short ragged lengths including
    empty slots, sampled slots against the oracle."""
    import sparse_decode_attention_window_b200 as kvc
    d = 128
    g = torch.Generator().manual_seed(S + G)
    lens = torch.randint(0, 40, (S,), generator=g, dtype=torch.int32)
    sh = kvc.make_shape(S, G, d, 64, 0, S, 1, torch.bfloat16)
    count = lens.cuda()
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 1, off, cap)
    rows = int(off[-1])
    kp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    vp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    q = torch.randn(S * G, d, generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn(S, d, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(S, d, generator=g).to(torch.bfloat16).cuda()
    out = torch.empty((S * G, d), device="cuda")
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    ln = count.clone()
    if fused:
        kvc.kvc_append_decode(sh, kn, vn, q, kp, vp, off, cap, ln, out, ws)
    else:
        kvc.kvc_decode_attn(sh, q, kp, vp, off, ln, out, ws)
    kvc.kvc_get_status()
    o = _np(out)
    offs = _np(off)
    for s in list(range(0, S, 97)) + [S - 1]:
        n = int(lens[s])
        keys, vals = kp[offs[s]:offs[s] + n].cpu(), vp[offs[s]:offs[s] + n].cpu()
        if fused:
            keys, vals = torch.cat([keys, kn[s:s + 1].cpu()]), torch.cat([vals, vn[s:s + 1].cpu()])
            n += 1
        if n == 0:
            assert (o[s * G:(s + 1) * G] == 0).all()
            continue
        ref = O.decode_attention(q[s * G:(s + 1) * G].cpu(), keys, vals, [0, n], [n], G)
        P.check_out(o[s * G:(s + 1) * G], ref, "bf16", f"slot {s}")
    if fused:
        assert (_np(ln) == _np(count) + 1).all()


@pytest.mark.parametrize("name,kw", [("llama8b", {}), ("fastgen", dict(batch=2, L=6000, steps=24)),
                                     ("zigzag", dict(n_layers=6, L=8192, steps=12))])
def test_graph_replay_of_a_step_matches_eager(name, kw):
    """The step as the benchmark runs it - score, select, compact and the decode loop
    (chained steps, programmatic dependent launch) captured once in a CUDA graph and
    replayed twice - gives bit for bit the outputs of the same calls made eagerly."""
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    import sparse_decode_attention_window_b200 as kvc
    wl = get(name).scaled(**kw) if kw else get(name)
    inp = make_inputs(wl, "cuda")
    pipe = KvcPipeline(wl, inp)
    outs = torch.empty((wl.steps,) + tuple(pipe.out.shape), dtype=torch.float32, device="cuda")

    def step():
        pipe.compress()
        for t in range(wl.steps):
            pipe.decode_step(t, out=outs[t])

    step()
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    eager = outs.clone()
    idx_eager, cnt_eager = pipe.idx.clone(), pipe.count.clone()
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cs):
        step()
    torch.cuda.current_stream().wait_stream(cs)
    for _ in range(2):
        outs.zero_()
        g.replay()
        torch.cuda.synchronize()
        kvc.kvc_get_status()
        assert torch.equal(pipe.count, cnt_eager)
        assert torch.equal(pipe.idx, idx_eager)
        assert torch.equal(outs, eager), f"max diff {(outs - eager).abs().max().item():.3e}"
    del g


def test_wide_window_takes_cuda_core_scoring_path():
    """G*w = 256 rows exceeds the tensor-core tile: scoring runs on the CUDA-core kernels;
    decode with G = 8 query heads per KV head."""
    run_and_check(get("llama8b").scaled(batch=1, hq=16, hkv=2, L=900, w=32, top_b=100, steps=3))


def test_cuda_core_paths_on_bf16_workloads():
    """The CUDA-core scoring and decode kernels, forced for bf16, pass the same oracle checks."""
    import subprocess
    import sys
    forced = ['--kvc-path', 'score=simt', '--kvc-path', 'decode=simt']
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "llama8b_shape_small_context or zigzag_small or chunk_small or fastgen_small "
                              "or decode_is_independent"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.parametrize("name,kw", [("llama8b", dict(batch=2, L=1500, top_b=200, steps=4)),
                                     ("fastgen", dict(batch=2, L=2000, steps=4)),
                                     ("tiny", dict())])
def test_separate_append_then_decode_calls(name, kw):
    """kvc_append followed by kvc_decode_attn (two launches) gives the same results."""
    run_and_check(get(name).scaled(**kw), fused=False)


def test_fused_append_decode_overflow_keeps_old_rows():
    import sparse_decode_attention_window_b200 as kvc
    S, G, d = 3, 4, 128
    sh = kvc.make_shape(S, G, d, 64, 0, S, 1, torch.bfloat16)
    count = torch.tensor([16, 5, 0], dtype=torch.int32, device="cuda")
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 0, off, cap)          # caps 16, 16, 0: slot 0 full, slot 2 has no room
    rows = int(off[-1])
    kp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    vp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    kp0, vp0 = kp.clone(), vp.clone()
    ln = count.clone()
    q = torch.randn(S * G, d, device="cuda").to(torch.bfloat16)
    kn = torch.randn(S, d, device="cuda").to(torch.bfloat16)
    vn = torch.randn(S, d, device="cuda").to(torch.bfloat16)
    out = torch.empty((S * G, d), device="cuda")
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    kvc.kvc_append_decode(sh, kn, vn, q, kp, vp, off, cap, ln, out, ws)
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_get_status()
    assert "append-overflow" in str(e.value)
    assert ln.cpu().tolist() == [16, 6, 0]
    # slot 1 got its token at row off[1] + 5; slot 0's rows are untouched
    assert torch.equal(kp[16 + 5], kn[1]) and torch.equal(vp[16 + 5], vn[1])
    assert torch.equal(kp[:16], kp0[:16])
    o = _np(out)
    ref0 = O.decode_attention(q[0:G].cpu(), kp0[:16].cpu(), vp0[:16].cpu(), [0, 16], [16], G)
    keys1 = torch.cat([kp0[16:21], kn[1:2]]).cpu()
    vals1 = torch.cat([vp0[16:21], vn[1:2]]).cpu()
    ref1 = O.decode_attention(q[G:2 * G].cpu(), keys1, vals1, [0, 6], [6], G)
    P.check_out(o[0:G], ref0, "bf16", "full slot")
    P.check_out(o[G:2 * G], ref1, "bf16", "appended slot")
    assert (o[2 * G:] == 0).all()
    kvc.kvc_get_status()


@pytest.mark.parametrize("S,counts,G,d", [(32, None, 4, 128), (5, [1000, 3, 0, 64, 700], 4, 128),
                                          (70, None, 4, 128), (16, None, 8, 128), (12, None, 2, 64)])
def test_chained_append_decode_is_bit_identical(S, counts, G, d):
    """kvc_append_decode_chain (the kept rows may load before the previous launch ends)
    returns bit for bit what kvc_append_decode returns, step after step, on uniform,
    ragged and many-slot caches, for G = 2, 4, 8 and d = 64, 128; the results match the
    oracle."""
    import sparse_decode_attention_window_b200 as kvc
    steps = 12
    g = torch.Generator().manual_seed(S)
    cnt = (torch.full((S,), 1024, dtype=torch.int32) if counts is None and S == 32 else
           torch.randint(0, 900, (S,), generator=g, dtype=torch.int32) if counts is None else
           torch.tensor(counts, dtype=torch.int32))
    sh = kvc.make_shape(S, G, d, int(cnt.max()) + steps, 0, S, 1, torch.bfloat16)
    count = cnt.cuda()
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, steps, off, cap)
    rows = int(off[-1])
    kp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    vp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    kp0, vp0 = kp.clone(), vp.clone()
    q = torch.randn(steps, S * G, d, generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn(steps, S, d, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(steps, S, d, generator=g).to(torch.bfloat16).cuda()
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    outs = {}
    for chained in (False, True):
        kp.copy_(kp0)
        vp.copy_(vp0)
        ln = count.clone()
        o = torch.empty((steps, S * G, d), device="cuda")
        for t in range(steps):
            if chained and t > 0:
                kvc.kvc_append_decode_chain(sh, kn[t], vn[t], q[t], kp, vp, off, cap, count, ln, o[t], ws)
            else:
                kvc.kvc_append_decode(sh, kn[t], vn[t], q[t], kp, vp, off, cap, ln, o[t], ws)
        torch.cuda.synchronize()
        kvc.kvc_get_status()
        assert torch.equal(ln, count + steps)
        outs[chained] = _np(o)
    np.testing.assert_array_equal(outs[True], outs[False])
    offs = _np(off)
    for s in sorted({0, S // 2, S - 1}):
        c = int(cnt[s])
        keys = torch.cat([kp0[offs[s]:offs[s] + c], kn[:, s]]).cpu()
        vals = torch.cat([vp0[offs[s]:offs[s] + c], vn[:, s]]).cpu()
        for t in (0, steps - 1):
            n = c + t + 1
            ref = O.decode_attention(q[t, s * G:(s + 1) * G].cpu(), keys[:n], vals[:n], [0, n], [n], G)
            P.check_out(outs[True][t, s * G:(s + 1) * G], ref, "bf16", f"slot {s} step {t}")


def test_chained_append_decode_reports_a_broken_promise():
    """stable[s] above a slot's length is flagged; that slot gets no new token and the
    launch writes nothing outside the slots."""
    import sparse_decode_attention_window_b200 as kvc
    S, G, d = 4, 4, 128
    sh = kvc.make_shape(S, G, d, 512, 0, S, 1, torch.bfloat16)
    count = torch.tensor([300, 200, 64, 0], dtype=torch.int32, device="cuda")
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, 4, off, cap)
    rows = int(off[-1])
    kp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    vp = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    q = torch.randn(S * G, d, device="cuda").to(torch.bfloat16)
    kn = torch.randn(S, d, device="cuda").to(torch.bfloat16)
    out = torch.empty((S * G, d), device="cuda")
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    ln = count.clone()
    stable = count.clone()
    stable[1] = 260                    # above slot 1's length (and capacity)
    kvc.kvc_append_decode_chain(sh, kn, kn, q, kp, vp, off, cap, stable, ln, out, ws)
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_get_status()
    assert "index-out-of-range" in str(e.value) and "wait-timeout" not in str(e.value)
    assert ln.cpu().tolist() == [301, 200, 65, 1]   # the slot that broke the promise gets no token
    assert np.isfinite(_np(out)).all()
    kvc.kvc_get_status()


@pytest.mark.parametrize("S,d,dt", [(4, 128, torch.bfloat16), (37, 64, torch.bfloat16), (512, 128, torch.bfloat16),
                                    (600, 64, torch.bfloat16), (24, 128, torch.float32)])
def test_layout_compact_matches_the_two_calls(S, d, dt):
    """One launch of layout + compaction (or, above 512 slots, the two launches it falls back
    to) gives the same offsets, capacities, lengths and packed rows, byte for byte, as
    kvc_layout then kvc_compact; counts are ragged, with empty and negative slots and counts
    above max_sel."""
    import sparse_decode_attention_window_b200 as kvc
    L, max_sel, reserve = 300, 160, 5
    g = torch.Generator().manual_seed(S * 7 + d)
    count = torch.randint(0, max_sel + 1, (S,), generator=g, dtype=torch.int32)
    count[0] = 0
    count[min(1, S - 1)] = max_sel
    if S > 2:
        count[2] = -3
    if S > 3:
        count[3] = max_sel + 40                # more than idx holds: max_sel rows copied
    idx = torch.stack([torch.sort(torch.randperm(L, generator=g)[:max_sel])[0] for _ in range(S)]).to(torch.int32)
    k = torch.randn((S, L, d), generator=g).to(dt).cuda()
    v = torch.randn((S, L, d), generator=g).to(dt).cuda()
    sh = kvc.make_shape(S, 1, d, L, 0, S, 1, dt)
    rows = int(sum((max(int(c), 0) + reserve + 15) // 16 * 16 for c in count))
    cnt, ix = count.cuda(), idx.cuda()
    outs = []
    for fused in (True, False):
        off = torch.full((S + 1,), -7, dtype=torch.int64, device="cuda")
        cap = torch.full((S,), -7, dtype=torch.int32, device="cuda")
        ln = torch.full((S,), -7, dtype=torch.int32, device="cuda")
        kp = torch.zeros((rows, d), dtype=dt, device="cuda")
        vp = torch.zeros((rows, d), dtype=dt, device="cuda")
        if fused:
            kvc.kvc_layout_compact(sh, k, v, ix, cnt, reserve, off, cap, kp, vp, ln)
        else:
            kvc.kvc_layout(cnt, reserve, off, cap)
            kvc.kvc_compact(sh, k, v, ix, cnt, off, kp, vp, ln)
        kvc.kvc_get_status()
        outs.append([off.cpu(), cap.cpu(), ln.cpu(), kp.view(torch.uint8).cpu(), vp.view(torch.uint8).cpu()])
    for a, b, name in zip(outs[0], outs[1], ["off", "cap", "len", "kp", "vp"]):
        assert torch.equal(a, b), name
    # and the layout itself, by its definition
    caps = [(max(int(c), 0) + reserve + 15) // 16 * 16 for c in count]
    assert outs[0][1].tolist() == caps
    assert outs[0][0].tolist() == [0] + list(np.cumsum(caps))


def test_grid_stride_compaction_on_workloads():
    """The grid-stride compaction kernel (forced here; the one-wave kernel is the default)
    gives the same bit-exact packed caches."""
    import subprocess
    import sys
    forced = ['--kvc-path', 'compact=grid']
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "llama8b_shape_small_context or zigzag_small or fastgen_small or chunk_small"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.parametrize("forced", [["--kvc-path", "score=twopass"], ["--kvc-path", "score=cluster"],
                                    ["--kvc-path", "score_k=1"], ["--kvc-path", "score_k=3"],
                                    ["--kvc-path", "score_k=16"]],
                         ids=["two_launch", "cluster_128key_tiles", "one_cta_per_slot", "three_ctas_per_slot",
                              "sixteen_ctas_per_slot"])
def test_other_scoring_forms_on_workloads(forced):
    """Workloads whose scoring runs in 256-key slot clusters by default pass the same checks
    through the two-launch form (pass 1, merge, pass 2), the earlier slot-cluster form with
    128-key tiles, and the slot clusters at 1, 3 and 16 CTAs per slot, each forced here."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "llama8b_shape_small_context or chunk_small or llama8b_full_size or "
                              "ragged_context_lengths or gqa_group_sizes or head_dims_and_dtypes or window_of_one or "
                              "prefill_row_normalisers or chunk_full_size"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_token_split_decode_on_few_slot_workloads():
    """Workloads with few slots decode through thread-block clusters by default; the
    token-range split (forced here) passes the same oracle checks."""
    import subprocess
    import sys
    forced = ['--kvc-path', 'decode_split=tokens']
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "llama8b_shape_small_context or zigzag_small or chunk_small or fastgen_small "
                              "or decode_is_independent or separate_append or fused_append_decode_overflow "
                              "or ragged_context_lengths or gqa_group_sizes"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_tcgen05_decode_path_on_bf16_workloads():
    """The tcgen05 decode (opt-in cross-check path, d = 128) passes the same oracle checks,
    including full-size llama8b and the fused-append overflow case."""
    import subprocess
    import sys
    forced = ['--kvc-path', 'decode=tc']
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider", *forced,
                        "-k", "llama8b_shape_small_context or zigzag_small or chunk_small or fastgen_small "
                              "or llama8b_full_size or separate_append or fused_append_decode_overflow "
                              "or ragged_context_lengths or gqa_group_sizes"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


# ---------------------------------------------------------------- next rows
@pytest.mark.parametrize("dt,d,G,w,L", [("bf16", 128, 4, 32, 1000), ("bf16", 64, 2, 16, 777),
                                        ("fp32", 128, 4, 8, 600)])
def test_score_with_prefill_row_normalisers(dt, d, G, w, L):
    """kvc_score given each window row's softmax normaliser from prefill (natural log over the
    keys the row sees) skips its statistics pass; the scores still match the oracle's."""
    import sparse_decode_attention_window_b200 as kvc
    S = 6
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    g = torch.Generator().manual_seed(L + d)
    q = torch.randn((S * G, w, d), generator=g).to(tdt)
    k = torch.randn((S, L, d), generator=g).to(tdt)
    # the caller's normalisers, in fp64 from the same rounded inputs (row i sees keys <= L - w + i)
    qd, kd = q.double().numpy(), k.double().numpy()
    lse = np.empty((S * G, w))
    for s in range(S):
        z = np.einsum("jid,nd->jin", qd[s * G:(s + 1) * G], kd[s]) / math.sqrt(d)
        for i in range(w):
            zi = z[:, i, :L - w + i + 1]
            m = zi.max(axis=1)
            lse[s * G:(s + 1) * G, i] = m + np.log(np.exp(zi - m[:, None]).sum(axis=1))
    sh = kvc.make_shape(S, G, d, L, w, 1, S, tdt)
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_SCORE, sh), dtype=torch.uint8, device="cuda")
    score = torch.empty((S, L), device="cuda")
    kvc.kvc_score(sh, q.cuda(), k.cuda(), score, ws,
                  row_lse=torch.tensor(lse.reshape(-1), dtype=torch.float32, device="cuda"))
    kvc.kvc_get_status()
    ref = np.stack([O.window_scores(q[s * G:(s + 1) * G], k[s:s + 1], L)[0] for s in range(S)])
    P.check_scores(_np(score), ref, dt, f"row_lse {dt} d{d} G{G} w{w} L{L}")


def test_retained_mass_matches_oracle():
    """Attention retained by the selection (ZigZagKV's attention loss is 0.9 minus it)."""
    import sparse_decode_attention_window_b200 as kvc
    wl = get("zigzag").scaled(n_layers=2, L=2048, steps=0)
    pipe, _ = run_and_check(wl, steps=[])
    ret = torch.empty(wl.n_slots, dtype=torch.float32, device="cuda")
    kvc.kvc_retained_mass(pipe.shape, pipe.score, pipe.idx, pipe.count, ret)
    torch.cuda.synchronize()
    sc = _np(pipe.score).astype(np.float64)
    idx, cnt = _np(pipe.idx), _np(pipe.count)
    for s in range(wl.n_slots):
        want = O.retained_mass(sc[s], idx[s, :cnt[s]])
        assert abs(float(ret[s]) - want) <= 1e-6 * max(want, 1e-30) + 1e-7, (s, float(ret[s]), want)
        assert O.attention_loss(want) >= 0.0


def test_profile_heads_matches_oracle():
    """FastGen-style profiling of each head from its window scores."""
    import sparse_decode_attention_window_b200 as kvc
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    from workloads import fastgen_policies
    wl = get("llama8b").scaled(batch=2, L=3000, top_b=300, steps=0, n_sinks=4)
    inp = make_inputs(wl, "cuda")
    pipe = KvcPipeline(wl, inp)
    pipe.score_step()
    _, mask = fastgen_policies(wl.scaled(special_frac=0.04))
    mask = mask.cuda()
    pol = torch.empty(wl.n_slots, dtype=torch.int8, device="cuda")
    shares = torch.empty((wl.n_slots, 2), dtype=torch.float32, device="cuda")
    for tau in (0.05, 0.2, 0.5, 0.99):
        for W in (64, 256, 2000):
            kvc.kvc_profile_heads(pipe.shape, pipe.score, pol, W, tau=tau, special_mask=mask, shares=shares)
            torch.cuda.synchronize()
            sc = _np(pipe.score).astype(np.float64)
            got, sh = _np(pol), _np(shares)
            for s in range(wl.n_slots):
                b = (s // wl.hkv) % wl.batch
                want = O.profile_head(sc[s], _np(mask[b]), W, tau)
                fl = O.retained_mass(sc[s], O.local_indices(wl.L, W))
                fs = O.retained_mass(sc[s], O.special_indices(_np(mask[b])))
                assert abs(sh[s, 0] - fl) < 1e-6 and abs(sh[s, 1] - fs) < 1e-6
                near = min(abs(fl - tau), abs(fs - tau)) < 1e-5
                assert got[s] == want or near, (s, tau, W, got[s], want, fl, fs)


@pytest.mark.parametrize("n_local", [0, 15, 16, 5000])
def test_chunk_selection_with_local_chunks(n_local):
    """ChunkLLM selection keeping the most recent chunks, vs the oracle."""
    import sparse_decode_attention_window_b200 as kvc
    wl = get("chunk").scaled(L=8000, steps=0)
    inp = make_inputs(wl, "cpu")
    from dataclasses import replace
    dinp = replace(inp, **{f: getattr(inp, f).cuda() for f in ("q_win", "k", "v", "q_dec", "k_dec", "v_dec",
                                                                 "chunk_end")})
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    pipe = KvcPipeline(wl, dinp)
    pipe.score_step()
    idx = torch.empty((wl.n_slots, wl.L), dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.n_slots, dtype=torch.int32, device="cuda")
    target = torch.full((wl.n_slots,), wl.chunk_target, dtype=torch.int32, device="cuda")
    kvc.kvc_select_chunks(pipe.shape, pipe.score, dinp.chunk_end, target, idx, cnt, n_local=n_local)
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    ce = _np(dinp.chunk_end)
    C = len(ce)
    for s in range(wl.n_slots):
        ref_sc = O.chunk_scores(inp.q_win[s * wl.G:(s + 1) * wl.G], inp.k[s:s + 1], wl.L, ce)[0]
        got = _np(idx[s, :int(cnt[s])]).astype(np.int64)
        toks, chosen = O.chunk_select_local(ref_sc, ce, wl.chunk_target, n_local)
        if np.array_equal(got, toks):
            continue
        # outside exact agreement only the tie band at the cut may differ: the forced chunks and
        # the clearly-ranked ones must match
        nl = min(n_local, C)
        cid = np.unique(np.searchsorted(ce, got, side="left"))
        assert set(range(C - nl, C)) <= set(cid.tolist())
        free_sc = ref_sc[: C - nl]
        P.check_chunks(np.concatenate([np.arange(ce[c - 1] + 1 if c else 0, ce[c] + 1) for c in cid if c < C - nl])
                       if any(c < C - nl for c in cid) else np.zeros(0, np.int64),
                       free_sc, ce[: C - nl], wl.chunk_target - int((np.diff(np.concatenate([[-1], ce]))[C - nl:]).sum()),
                       f"slot {s}")


def _check_local_chunk_selection(got, ref_sc, ce, target, n_local, what):
    """GPU tokens of a selection with local chunks vs the oracle's rule (ties tolerated)."""
    C = len(ce)
    toks, _ = O.chunk_select_local(ref_sc, ce, target, n_local)
    if np.array_equal(got, toks):
        return
    nl = min(n_local, C)
    cid = np.unique(np.searchsorted(ce, got, side="left"))
    assert set(range(C - nl, C)) <= set(cid.tolist()), f"{what}: local chunks missing"
    starts = np.concatenate([[0], ce[:-1] + 1])
    lens = ce - starts + 1
    have = int(lens[C - nl:].sum())
    free = [c for c in cid if c < C - nl]
    free_toks = (np.concatenate([np.arange(starts[c], ce[c] + 1) for c in free]) if free
                 else np.zeros(0, np.int64))
    if have >= target:
        assert not free, f"{what}: local chunks reach the target, nothing else may be kept"
        return
    P.check_chunks(free_toks, ref_sc[: C - nl], ce[: C - nl], target - have, what)


@pytest.mark.parametrize("n_local", [0, 4])
def test_chunk_icac_reselection_matches_oracle(n_local):
    """ChunkLLM decode-time re-selection (NEXT-1): at every step whose token closes a chunk
    the chunks are re-scored with that step's query, re-selected and the attended cache is
    re-compacted from the full cache. Each GPU selection is checked against the oracle's
    rule on the oracle's chunk scores (ties tolerated); each step's output against fp64
    attention over the GPU's attended set; with no tie, the whole run equals icac_decode."""
    from workloads import decode_chunk_boundaries
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    import sparse_decode_attention_window_b200 as kvc
    from dataclasses import replace
    wl = get("chunk_icac").scaled(L=3000, steps=40, chunk_mean=8.0, n_local=n_local)
    inp = make_inputs(wl, "cpu")
    dinp = replace(inp, **{f: getattr(inp, f).cuda() for f in ("q_win", "k", "v", "q_dec", "k_dec", "v_dec",
                                                                 "chunk_end")})
    bnd = decode_chunk_boundaries(wl)
    assert len(bnd) >= 3
    pipe = KvcPipeline(wl, dinp, decode_boundaries=bnd)
    pipe.compress()
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    S, G, L = wl.n_slots, wl.G, wl.L
    ce0 = _np(dinp.chunk_end).astype(np.int64)
    kf = np.concatenate([O._f64(inp.k), O._f64(inp.k_dec).transpose(1, 0, 2)], axis=1)   # [S, L + steps, d]
    vf = np.concatenate([O._f64(inp.v), O._f64(inp.v_dec).transpose(1, 0, 2)], axis=1)
    sel = {}
    for s in range(S):
        got = _np(pipe.idx[s, :int(pipe.count[s])]).astype(np.int64)
        ref_sc = O.chunk_scores(inp.q_win[s * G:(s + 1) * G], inp.k[s:s + 1], L, ce0)[0]
        _check_local_chunk_selection(got, ref_sc, ce0, wl.chunk_target, n_local, f"prompt slot {s}")
        sel[s] = list(got)
    ends = list(ce0)
    exact = True
    gpu_out = []
    for t in range(wl.steps):
        out = _np(pipe.decode_step(t)).copy()
        gpu_out.append(out)
        torch.cuda.synchronize()
        kvc.kvc_get_status()
        for s in range(S):
            sel[s].append(L + t)
            idx = np.asarray(sel[s], dtype=np.int64)
            q = O._f64(inp.q_dec[t, s * G:(s + 1) * G])
            ref = O.decode_attention(q, kf[s][idx], vf[s][idx], [0, idx.size], [idx.size], G)
            P.check_out(out[s * G:(s + 1) * G], ref, "bf16", f"step {t} slot {s}")
        if t in bnd:
            ends.append(L + t)
            e = np.asarray(ends, dtype=np.int64)
            n = L + t + 1
            target = math.ceil(wl.keep_frac * n)
            for s in range(S):
                got = _np(pipe.idx[s, :int(pipe.count[s])]).astype(np.int64)
                q = O._f64(inp.q_dec[t, s * G:(s + 1) * G])
                ref_sc = O.chunk_scores(q[:, None, :], kf[s][None, :n], n, e)[0]
                _check_local_chunk_selection(got, ref_sc, e, target, n_local, f"boundary step {t} slot {s}")
                toks, _ = O.chunk_select_local(ref_sc, e, target, n_local)
                exact = exact and np.array_equal(got, toks)
                sel[s] = list(got)
                assert int(pipe.len[s]) == got.size
    if exact:
        for s in range(0, S, 3):
            outs, _ = O.icac_decode(inp.q_win[s * G:(s + 1) * G], inp.k[s], inp.v[s], ce0, inp.q_dec[:, s * G:(s + 1) * G],
                                    inp.k_dec[:, s], inp.v_dec[:, s], bnd, wl.keep_frac, n_local, G)
            for t in range(wl.steps):
                P.check_out(gpu_out[t][s * G:(s + 1) * G], outs[t], "bf16", f"icac_decode step {t} slot {s}")


def test_fastgen_sliding_local_window_matches_oracle():
    """NEXT-3: FastGen local heads keep exactly their most recent window while decoding
    (kvc_append_window overwrites the oldest row once the window is full); every other
    head keeps its selection plus all appended tokens. Enough steps to wrap the ring
    twice; every step of every slot against the oracle."""
    import sparse_decode_attention_window_b200 as kvc
    from sparse_decode_attention_window_b200.pipeline import KvcPipeline
    from oracle.pipeline import run_workload
    from dataclasses import replace
    wl = get("fastgen_sliding").scaled(batch=2, L=1500, local_window=48, steps=110)
    inp = make_inputs(wl, "cpu")
    dinp = replace(inp, **{f: (getattr(inp, f).cuda() if getattr(inp, f) is not None else None)
                           for f in ("q_win", "k", "v", "q_dec", "k_dec", "v_dec", "policy", "special_mask")})
    assert (inp.policy == POL_LOCAL).any()
    pipe = KvcPipeline(wl, dinp)
    pipe.compress()
    outs = []
    for t in range(wl.steps):
        outs.append(_np(pipe.decode_step(t)).copy())
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    ref = run_workload(inp)
    G = wl.G
    for s in range(wl.n_slots):
        if int(inp.policy[s]) == POL_LOCAL:
            assert int(pipe.len[s]) == wl.local_window
        for t in range(wl.steps):
            P.check_out(outs[t][s * G:(s + 1) * G], ref.out[(t, s)], "bf16", f"step {t} slot {s}")


@pytest.mark.parametrize("case", json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                                            "alloc_examples.json")))["cases"],
                         ids=lambda c: c["name"])
def test_allocation_worked_examples_on_gpu(case):
    """kvc_alloc_budgets on the hand-worked ZigZagKV Eq. 4-6 examples (exact, largest remainder,
    tied remainders to the lower layer, cap at the context, uniform, floor only)."""
    import sparse_decode_attention_window_b200 as kvc
    counts = np.array(case["counts"], dtype=np.int32)
    nL, spl = counts.shape
    budgets = torch.full((nL,), -1, dtype=torch.int32, device="cuda")
    slot_b = torch.full((nL * spl,), -1, dtype=torch.int32, device="cuda")
    kvc.kvc_alloc_budgets(torch.from_numpy(counts.reshape(-1)).cuda(), nL, spl, case["L"], case["avg"],
                          case["floor"], budgets, slot_b)
    kvc.kvc_get_status()
    assert budgets.cpu().tolist() == case["budgets"]
    assert slot_b.cpu().tolist() == [b for b in case["budgets"] for _ in range(spl)]


@pytest.mark.parametrize("S,counts,steps", [(40, "ragged", 96), (8, "uniform", 96), (6, [0, 1, 2, 3, 5, 7], 64)])
def test_chained_append_decode_every_step_matches_oracle(S, counts, steps):
    """Many chained append + decode launches back to back on one stream (each may start while
    the previous one drains): every step of every slot matches the oracle's attention over the
    cache grown by one token per step, and the lengths grow by exactly one per step. Ragged
    slots (the token split, ranges crossing slots), near-uniform slots (per-slot clusters) and
    a cache so small that most CTAs have no tokens (every CTA still takes its length ticket)."""
    import sparse_decode_attention_window_b200 as kvc
    G, d = 4, 128
    g = torch.Generator().manual_seed(1000 + S)
    if counts == "ragged":
        cnt = torch.randint(0, 600, (S,), generator=g, dtype=torch.int32)
        cnt[::7] = 0
    elif counts == "uniform":
        cnt = torch.randint(990, 1010, (S,), generator=g, dtype=torch.int32)
    else:
        cnt = torch.tensor(counts, dtype=torch.int32)
    sh = kvc.make_shape(S, G, d, int(cnt.max()) + steps, 0, S, 1, torch.bfloat16)
    count = cnt.cuda()
    off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    cap = torch.empty(S, dtype=torch.int32, device="cuda")
    kvc.kvc_layout(count, steps, off, cap)
    rows = int(off[-1])
    kp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    vp = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    kp0, vp0 = kp.cpu(), vp.cpu()
    q = torch.randn(steps, S * G, d, generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn(steps, S, d, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(steps, S, d, generator=g).to(torch.bfloat16).cuda()
    ws = torch.zeros(kvc.kvc_workspace_size(kvc.KVC_WS_DECODE, sh), dtype=torch.uint8, device="cuda")
    ln = count.clone()
    o = torch.empty((steps, S * G, d), device="cuda")
    for t in range(steps):
        if t > 0:
            kvc.kvc_append_decode_chain(sh, kn[t], vn[t], q[t], kp, vp, off, cap, count, ln, o[t], ws)
        else:
            kvc.kvc_append_decode(sh, kn[t], vn[t], q[t], kp, vp, off, cap, ln, o[t], ws)
    torch.cuda.synchronize()
    kvc.kvc_get_status()
    assert torch.equal(ln, count + steps)
    offs, oc = _np(off), _np(o)
    qc, knc, vnc = q.cpu(), kn.cpu(), vn.cpu()
    for s in range(S):
        c = int(cnt[s])
        keys = torch.cat([kp0[offs[s]:offs[s] + c], knc[:, s]])
        vals = torch.cat([vp0[offs[s]:offs[s] + c], vnc[:, s]])
        # the appended rows are in the cache, in order
        np.testing.assert_array_equal(_np(kp[offs[s]:offs[s] + c + steps].view(torch.int16)),
                                      keys.view(torch.int16).numpy())
        for t in range(steps):
            n = c + t + 1
            ref = O.decode_attention(qc[t, s * G:(s + 1) * G], keys[:n], vals[:n], [0, n], [n], G)
            P.check_out(oc[t, s * G:(s + 1) * G], ref, "bf16", f"slot {s} step {t}")
