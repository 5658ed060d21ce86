"""Pins for the fp64 oracle: each check ties it to something other than itself -
an invariant of the definition, a closed form, brute force, or an independent
library routine (torch fp64 softmax / topk / scaled_dot_product_attention)."""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- scoring
def test_score_rows_sum_to_group_times_window():
    r = _rng(0)
    S, G, w, L, d = 3, 2, 5, 40, 8
    q = r.standard_normal((S * G, w, d))
    k = r.standard_normal((S, L, d)) * 2.0
    sc = O.window_scores(q, k, L)
    assert sc.shape == (S, L)
    np.testing.assert_allclose(sc.sum(axis=1), G * w, rtol=0, atol=1e-12)
    assert (sc >= 0).all()


def test_score_single_row_is_library_softmax():
    r = _rng(1)
    L, d = 33, 16
    q = r.standard_normal((1, 1, d))
    k = r.standard_normal((1, L, d))
    sc = O.window_scores(q, k, L)[0]
    ref = torch.softmax(torch.from_numpy(k[0] @ q[0, 0] / math.sqrt(d)), dim=0).numpy()
    np.testing.assert_allclose(sc, ref, rtol=1e-13, atol=1e-15)


def test_score_two_keys_sigmoid():
    # d = 1, L = 2, one row: p_1 = sigmoid(q*(k1-k0)), p_0 = 1 - p_1
    q = np.array([[[1.7]]])
    k = np.array([[[0.3], [-1.1]]])
    sc = O.window_scores(q, k, 2)[0]
    p1 = 1.0 / (1.0 + math.exp(-(1.7 * (-1.1 - 0.3))))
    np.testing.assert_allclose(sc, [1.0 - p1, p1], rtol=1e-14)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "score_closed_forms.json")))["cases"],
                         ids=lambda c: c["name"])
def test_score_zero_keys_closed_form(case):
    L, w, G, d = case["L"], case["w"], case["G"], case["d"]
    r = _rng(2)
    q = r.standard_normal((G, w, d))
    k = np.zeros((1, L, d))
    sc = O.window_scores(q, k, L)[0]
    want = [n / dd for n, dd in zip(case["score_num"], case["score_den"])]
    np.testing.assert_allclose(sc, want, rtol=1e-14)


def test_score_causal_window_tail():
    # key L-1 is visible only to the last window row of each head
    r = _rng(3)
    G, w, L, d = 3, 4, 20, 8
    q = r.standard_normal((G, w, d))
    k = r.standard_normal((1, L, d))
    sc = O.window_scores(q, k, L)[0]
    last = 0.0
    for h in range(G):
        lg = k[0] @ q[h, w - 1] / math.sqrt(d)
        last += torch.softmax(torch.from_numpy(lg), 0).numpy()[L - 1]
    np.testing.assert_allclose(sc[L - 1], last, rtol=1e-13)


def test_score_group_is_sum_of_heads():
    r = _rng(4)
    G, w, L, d = 4, 3, 25, 8
    q = r.standard_normal((G, w, d))
    k = r.standard_normal((1, L, d))
    both = O.window_scores(q, k, L)[0]
    parts = sum(O.window_scores(q[h:h + 1], k, L)[0] for h in range(G))
    np.testing.assert_allclose(both, parts, rtol=1e-13)


def test_score_permutation_equivariance():
    r = _rng(5)
    G, w, L, d = 2, 4, 30, 8
    q = r.standard_normal((G, w, d))
    k = r.standard_normal((1, L, d))
    perm = np.arange(L)
    perm[: L - w + 1] = r.permutation(L - w + 1)   # keys every row sees
    a = O.window_scores(q, k, L)[0]
    b = O.window_scores(q, k[:, perm], L)[0]
    np.testing.assert_allclose(b, a[perm], rtol=1e-13)


def test_chunk_scores_single_token_chunks_equal_token_scores():
    r = _rng(6)
    G, w, L, d = 2, 4, 30, 8
    q = r.standard_normal((G, w, d))
    k = r.standard_normal((1, L, d))
    ends = np.arange(L)
    np.testing.assert_allclose(O.chunk_scores(q, k, L, ends)[0], O.window_scores(q, k, L)[0], rtol=1e-14)


def test_chunk_scores_visibility_and_sum():
    r = _rng(7)
    G, w, L, d = 2, 5, 40, 8
    q = r.standard_normal((G, w, d))
    k = r.standard_normal((1, L, d))
    ends = np.array([3, 9, 10, 20, 33, 36, 37, 39])
    cs = O.chunk_scores(q, k, L, ends)[0]
    np.testing.assert_allclose(cs.sum(), G * w, atol=1e-12)
    # chunk ending at 39 (= L-1) is visible only to the last row; at 36 to rows with L-w+i >= 36 -> i >= 1
    lg = lambda h, i: (k[0, ends] @ q[h, i]) / math.sqrt(d)
    last = 0.0
    for h in range(G):
        z = lg(h, w - 1)
        last += np.exp(z - z.max())[-1] / np.exp(z - z.max()).sum()
    np.testing.assert_allclose(cs[-1], last, rtol=1e-13)


# ---------------------------------------------------------------- top-B
def test_top_b_matches_library_topk():
    r = _rng(8)
    sc = r.random(500)
    for B in (1, 7, 64, 499, 500, 600):
        got = O.top_b(sc, B)
        ref = torch.topk(torch.from_numpy(sc), min(B, 500)).indices.numpy()
        np.testing.assert_array_equal(got, np.sort(ref))
        assert (np.diff(got) > 0).all()


def test_top_b_ties_take_lowest_index():
    sc = np.array([1.0, 2.0, 2.0, 2.0, 0.5, 2.0])
    np.testing.assert_array_equal(O.top_b(sc, 2), [1, 2])
    np.testing.assert_array_equal(O.top_b(sc, 5), [0, 1, 2, 3, 5])


# ---------------------------------------------------------------- LMBA mass count
def _brute_min_subset(sc, mass):
    total = sc.sum()
    n = len(sc)
    for size in range(1, n + 1):
        for comb in itertools.combinations(range(n), size):
            if sc[list(comb)].sum() >= mass * total - 1e-9 * total:
                return size
    return n


@pytest.mark.parametrize("seed", range(12))
def test_mass_count_is_smallest_subset_brute_force(seed):
    r = _rng(100 + seed)
    n = int(r.integers(1, 13))
    sc = r.integers(1, 1000, size=n).astype(np.float64)   # integer masses: exact sums
    total = sc.sum()
    if abs(0.9 * total - round(0.9 * total)) < 1e-6:      # keep the boundary away from exact ties
        sc[0] += 1
    assert O.mass_count(sc, 0.9) == _brute_min_subset(sc, 0.9)


def test_mass_count_closed_forms():
    assert O.mass_count(np.ones(20), 0.9) == 18              # uniform: ceil(0.9 L)
    assert O.mass_count(np.ones(7), 0.9) == 7                # ceil(6.3)
    oh = np.zeros(50); oh[17] = 3.0
    assert O.mass_count(oh, 0.9) == 1                        # one-hot
    geo = 0.5 ** np.arange(30)                               # 1 + 1/2 + 1/4 ... : 4 terms reach 0.9375 * 2
    assert O.mass_count(geo, 0.9) == 4


# ---------------------------------------------------------------- allocation
@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "alloc_examples.json")))["cases"],
                         ids=lambda c: c["name"])
def test_allocation_worked_examples(case):
    got = O.allocate_budgets(np.array(case["counts"]), case["L"], case["avg"], case["floor"])
    np.testing.assert_array_equal(got, case["budgets"])


@pytest.mark.parametrize("seed", range(20))
def test_allocation_properties(seed):
    r = _rng(200 + seed)
    nL = int(r.integers(1, 40))
    H = int(r.integers(1, 9))
    L = int(r.integers(16, 40000))
    avg = int(r.integers(1, L + 1))
    floor = int(r.integers(0, avg + 1))
    counts = r.integers(1, L + 1, size=(nL, H))
    if seed % 5 == 0:      # very skewed: forces the cap
        counts[:] = 1
        counts[0] = L
    b = O.allocate_budgets(counts, L, avg, floor)
    assert b.sum() == nL * avg
    assert (b >= min(floor, L)).all()
    assert (b <= L).all()
    # without a cap in play, each budget is within one token of Eq. 6
    if (b < L).all():
        C = counts.sum(axis=1)
        for l in range(nL):
            exact = Fraction(floor) + Fraction((avg - floor) * nL * int(C[l]), int(C.sum()))
            assert abs(Fraction(int(b[l])) - exact) < 1


# ---------------------------------------------------------------- policies
def test_policies_are_their_definitions():
    np.testing.assert_array_equal(O.local_indices(1000, 256), np.arange(744, 1000))
    np.testing.assert_array_equal(O.local_indices(100, 256), np.arange(100))
    np.testing.assert_array_equal(O.full_indices(9), np.arange(9))
    m = np.zeros(50, np.uint8); m[[0, 1, 2, 3, 17, 44]] = 1
    np.testing.assert_array_equal(O.special_indices(m), [0, 1, 2, 3, 17, 44])


# ---------------------------------------------------------------- chunks
def test_chunk_select_brute_force_prefix():
    r = _rng(9)
    for trial in range(30):
        L = int(r.integers(5, 60))
        cuts = np.sort(r.choice(np.arange(L - 1), size=int(r.integers(0, L - 1)), replace=False))
        ends = np.concatenate([cuts, [L - 1]])
        sc = r.random(len(ends))
        target = int(r.integers(1, L + 1))
        toks, chosen = O.chunk_select(sc, ends, target)
        lens = np.diff(np.concatenate([[-1], ends]))
        assert len(toks) == lens[chosen].sum() >= target
        # minimal: dropping the lowest-scoring chosen chunk falls short of the target
        worst = chosen[np.argmin(sc[chosen])]
        assert lens[chosen].sum() - lens[worst] < target
        # chosen chunks are exactly the top-|chosen| chunks by score
        np.testing.assert_array_equal(chosen, np.sort(np.argsort(-sc, kind="stable")[: len(chosen)]))
        assert (np.diff(toks) > 0).all()


def test_chunk_boundaries_partition_context():
    from workloads import get, chunk_boundaries
    wl = get("chunk").scaled(L=20000)
    ends = chunk_boundaries(wl).numpy().astype(np.int64)
    assert ends[-1] == wl.L - 1 and (np.diff(ends) >= 1).all() and ends[0] >= 0
    lens = np.diff(np.concatenate([[-1], ends]))
    assert abs(lens[:-1].mean() - 24.0) < 1.5          # Geometric(mean 24)


# ---------------------------------------------------------------- compaction
def test_layout_and_compaction_round_trip():
    r = _rng(10)
    S, L, d = 4, 50, 8
    k = r.standard_normal((S, L, d)); v = r.standard_normal((S, L, d))
    sel = [np.sort(r.choice(L, size=n, replace=False)) for n in (0, 1, 17, 50)]
    off, cap = O.layout([len(s) for s in sel], reserve=3)
    assert (cap % 16 == 0).all() and (cap >= np.array([len(s) for s in sel]) + 3).all()
    assert off[0] == 0 and (np.diff(off) == cap).all()
    kp, vp = O.compact(k, v, sel, off)
    for s in range(S):
        back = np.zeros((L, d)); back[sel[s]] = kp[off[s]:off[s] + len(sel[s])]
        np.testing.assert_array_equal(back[sel[s]], k[s][sel[s]])
        np.testing.assert_array_equal(vp[off[s]:off[s] + len(sel[s])], v[s][sel[s]])
    # budget = L keeps the cache as it is
    full = [np.arange(L)] * S
    off2, _ = O.layout([L] * S, reserve=0)
    kp2, _ = O.compact(k, v, full, off2)
    for s in range(S):
        np.testing.assert_array_equal(kp2[off2[s]:off2[s] + L], k[s])


# ---------------------------------------------------------------- decode
def test_decode_full_cache_equals_library_sdpa():
    r = _rng(11)
    S, G, n, d = 3, 4, 37, 16
    q = r.standard_normal((S * G, d))
    k = r.standard_normal((S, n, d)); v = r.standard_normal((S, n, d))
    off, _ = O.layout([n] * S, reserve=0)
    kp, vp = O.compact(k, v, [np.arange(n)] * S, off)
    out = O.decode_attention(q, kp, vp, off, [n] * S, G)
    tq = torch.from_numpy(q).view(S, G, 1, d)
    tk = torch.from_numpy(k).view(S, 1, n, d).expand(S, G, n, d)
    tv = torch.from_numpy(v).view(S, 1, n, d).expand(S, G, n, d)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).view(S * G, d).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_decode_single_token_returns_its_value():
    r = _rng(12)
    q = r.standard_normal((2, 8)); k = r.standard_normal((1, 8)); v = r.standard_normal((1, 8))
    out = O.decode_attention(q, k, v, [0, 1], [1], 2)
    np.testing.assert_array_equal(out, np.vstack([v, v]))


def test_append_then_decode_sees_new_token():
    r = _rng(13)
    d = 8
    k = r.standard_normal((1, 5, d)); v = r.standard_normal((1, 5, d))
    off, cap = O.layout([5], reserve=2)
    kp, vp = O.compact(k, v, [np.arange(5)], off)
    ln = np.array([5])
    kn = r.standard_normal((1, d)); vn = r.standard_normal((1, d))
    O.append(kp, vp, off, ln, kn, vn)
    assert ln[0] == 6
    np.testing.assert_array_equal(kp[5], kn[0])
    # a query aligned with the new key (large dot product) returns ~its value
    q = kn * 50.0
    out = O.decode_attention(q, kp, vp, off, ln, 1)
    np.testing.assert_allclose(out[0], vn[0], atol=1e-6)


# ---------------------------------------------------------------- whole workload
def test_tiny_workload_full_budget_is_dense_attention():
    """With B = L the compressed decode reproduces uncompressed attention (SDPA)."""
    from workloads import get, make_inputs
    from oracle.pipeline import run_workload
    wl = get("tiny").scaled(top_b=512)
    inp = make_inputs(wl, "cpu")
    res = run_workload(inp)
    S, G, d = wl.n_slots, wl.G, wl.d
    for t in range(wl.steps):
        k = torch.cat([inp.k.double(), inp.k_dec[: t + 1].double().transpose(0, 1)], dim=1)
        v = torch.cat([inp.v.double(), inp.v_dec[: t + 1].double().transpose(0, 1)], dim=1)
        n = k.shape[1]
        q = inp.q_dec[t].double().view(S, G, 1, d)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k.view(S, 1, n, d).expand(S, G, n, d), v.view(S, 1, n, d).expand(S, G, n, d)).view(S, G, d)
        for s in range(S):
            np.testing.assert_allclose(res.out[(t, s)], ref[s].numpy(), rtol=1e-11, atol=1e-12)


def test_tiny_workload_sinks_are_kept():
    """Sanity on the tiny workload's structure: the four sink keys rank in the top-64."""
    from workloads import get, make_inputs
    from oracle.pipeline import run_workload
    wl = get("tiny")
    res = run_workload(make_inputs(wl, "cpu"), steps=0)
    for s in range(wl.n_slots):
        assert {0, 1, 2, 3} <= set(res.sel[s].tolist())


# ---------------------------------------------------------------- next rows
def test_retained_mass_limits_and_lmba_consistency():
    r = _rng(300)
    sc = r.random(200) ** 4
    assert O.retained_mass(sc, np.arange(200)) == pytest.approx(1.0, abs=1e-15)
    assert O.retained_mass(sc, np.array([], dtype=np.int64)) == 0.0
    assert O.retained_mass(np.zeros(5), [0, 1]) == 0.0
    # the LMBA count is exactly where the top-k retained mass first reaches 0.9
    k = O.mass_count(sc, 0.9)
    assert O.retained_mass(sc, O.top_b(sc, k)) >= 0.9
    assert O.retained_mass(sc, O.top_b(sc, k - 1)) < 0.9
    assert O.attention_loss(O.retained_mass(sc, O.top_b(sc, k))) == 0.0
    assert O.attention_loss(0.5) == pytest.approx(0.4)


def test_top_b_retains_the_most_mass_brute_force():
    r = _rng(301)
    for _ in range(10):
        n = int(r.integers(3, 11))
        sc = r.random(n)
        for B in range(1, n + 1):
            best = max(O.retained_mass(sc, list(c)) for c in itertools.combinations(range(n), B))
            assert O.retained_mass(sc, O.top_b(sc, B)) == pytest.approx(best, rel=1e-12)


def test_profile_head_picks_the_cheapest_sufficient_policy():
    L, W = 100, 10
    mask = np.zeros(L, np.uint8); mask[[0, 1, 2, 3, 50]] = 1           # 5 special tokens
    local = np.zeros(L); local[90:] = 1.0                               # all mass in the window
    assert O.profile_head(local, mask, W, 0.95) == 2                    # LOCAL
    special = np.zeros(L); special[[0, 1, 2, 3, 50]] = 1.0
    assert O.profile_head(special, mask, W, 0.95) == 3                  # SPECIAL (5 tokens, cheaper than 10)
    both = np.zeros(L); both[[0, 1, 2, 3, 50]] = 1.0; both[95] = 1000.0   # most mass in the window
    assert O.profile_head(both, mask, W, 0.95) == 2
    flat = np.ones(L)
    assert O.profile_head(flat, mask, W, 0.95) == 4                     # FULL
    # with fewer special tokens than the window, special is tried first
    assert O.profile_head(special + local * 1e-9, mask, W, 0.95) == 3


def test_chunk_select_local_reduces_and_forces():
    r = _rng(302)
    for _ in range(30):
        L = int(r.integers(5, 80))
        cuts = np.sort(r.choice(np.arange(L - 1), size=int(r.integers(0, L - 1)), replace=False))
        ends = np.concatenate([cuts, [L - 1]])
        C = len(ends)
        sc = r.random(C)
        target = int(r.integers(1, L + 1))
        # no local chunks: the plain selection
        t0, c0 = O.chunk_select_local(sc, ends, target, 0)
        t1, c1 = O.chunk_select(sc, ends, target)
        np.testing.assert_array_equal(t0, t1)
        nl = int(r.integers(0, C + 1))
        toks, chosen = O.chunk_select_local(sc, ends, target, nl)
        lens = np.diff(np.concatenate([[-1], ends]))
        assert set(range(C - nl, C)) <= set(chosen.tolist())          # local chunks always kept
        assert len(toks) == lens[chosen].sum()
        assert len(toks) >= min(target, L) or len(chosen) == C
        free = [c for c in chosen if c < C - nl]
        if free:                                                         # minimal: the worst free chunk was needed
            worst = free[int(np.argmin(sc[free]))]
            assert lens[chosen].sum() - lens[worst] < target
            # the free chunks are the top chunks by score among the non-local ones
            others = np.arange(C - nl)
            top = np.sort(others[np.argsort(-sc[others], kind="stable")[: len(free)]])
            np.testing.assert_array_equal(np.sort(free), top)
    # every chunk local: everything kept
    ends = np.array([2, 5, 9])
    toks, chosen = O.chunk_select_local(np.array([0.1, 0.2, 0.3]), ends, 1, 3)
    np.testing.assert_array_equal(toks, np.arange(10))


# ---------------------------------------------------------------- ICAC re-selection (NEXT-1)
def _attend(q, keys, vals):
    """Plain softmax attention of each row of q over keys (numpy, fp64)."""
    lg = q @ keys.T / np.sqrt(q.shape[1])
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p @ vals


def _icac_case(seed, L=60, steps=8, d=8, G=2, w=3):
    r = _rng(seed)
    k = r.standard_normal((L, d)); v = r.standard_normal((L, d))
    qw = r.standard_normal((G, w, d))
    qd = r.standard_normal((steps, G, d)); kd = r.standard_normal((steps, d)); vd = r.standard_normal((steps, d))
    cuts = np.sort(r.choice(np.arange(L - 1), size=9, replace=False))
    ends = np.concatenate([cuts, [L - 1]])
    return k, v, qw, qd, kd, vd, ends


def test_icac_keep_everything_is_full_attention():
    """keep_frac = 1 keeps every chunk at every selection: each step is attention over
    the whole prompt plus the generated tokens, whatever the boundaries."""
    k, v, qw, qd, kd, vd, ends = _icac_case(401)
    out, sels = O.icac_decode(qw, k, v, ends, qd, kd, vd, [1, 2, 5], 1.0, 0, 2)
    for t in range(qd.shape[0]):
        keys = np.concatenate([k, kd[:t + 1]]); vals = np.concatenate([v, vd[:t + 1]])
        np.testing.assert_allclose(out[t], _attend(qd[t], keys, vals), rtol=1e-12, atol=1e-12)
    for t in (1, 2, 5):
        np.testing.assert_array_equal(sels[t], np.arange(k.shape[0] + t + 1))


def test_icac_selection_timing_and_attended_sets():
    """Brute force on explicit token sets: before any boundary the attended set is the
    prompt selection plus the generated tokens; a boundary step still attends over the old
    set, the next step over the new selection (which covers every token up to the boundary,
    the closed chunk among its candidates) plus the tokens generated after it."""
    k, v, qw, qd, kd, vd, ends = _icac_case(402)
    L, steps = k.shape[0], qd.shape[0]
    tb = 3
    out, sels = O.icac_decode(qw, k, v, ends, qd, kd, vd, [tb], 0.5, 1, 2)
    kf = np.concatenate([k, kd]); vf = np.concatenate([v, vd])
    s0 = sels[-1]
    for t in range(steps):
        att = np.concatenate([s0, np.arange(L, L + t + 1)]) if t <= tb else \
            np.concatenate([sels[tb], np.arange(L + tb + 1, L + t + 1)])
        np.testing.assert_allclose(out[t], _attend(qd[t], kf[att], vf[att]), rtol=1e-12, atol=1e-12)
    # the re-selection at tb: chunks are the prompt's plus [L, L + tb]; n_local = 1 keeps
    # that newest chunk; at least half of the L + tb + 1 tokens are kept
    new = sels[tb]
    assert set(range(L, L + tb + 1)) <= set(new.tolist())
    assert new.size >= math.ceil(0.5 * (L + tb + 1))
    # and it is the chunk selection of the boundary query over those chunks (scores by
    # direct softmax of q . chunk key over the visible chunks, summed over the group)
    e2 = np.concatenate([ends, [L + tb]])
    lg = qd[tb] @ kf[e2].T / np.sqrt(k.shape[1])
    p = np.exp(lg - lg.max(axis=1, keepdims=True)); p /= p.sum(axis=1, keepdims=True)
    toks, _ = O.chunk_select_local(p.sum(axis=0), e2, math.ceil(0.5 * (L + tb + 1)), 1)
    np.testing.assert_array_equal(new, toks)


def test_icac_query_picks_the_aligned_chunk():
    """Two prompt chunks; the boundary query points at the first chunk's key and away
    from the second's, so with room for one prompt chunk the re-selection keeps the first
    (plus the closed generated chunk, which n_local = 1 forces)."""
    d, G = 4, 1
    k = np.zeros((8, d)); v = np.arange(8 * d, dtype=float).reshape(8, d)
    k[3] = [5, 0, 0, 0]; k[7] = [-5, 0, 0, 0]           # chunk keys (last tokens of [0,3] and [4,7])
    ends = np.array([3, 7])
    qw = np.zeros((G, 1, d)); qw[0, 0] = [0, 1, 0, 0]     # prompt query: indifferent
    qd = np.zeros((2, G, d)); qd[0, 0] = [1, 0, 0, 0]     # step 0 query favours chunk 0
    kd = np.zeros((2, d)); vd = np.zeros((2, d))
    out, sels = O.icac_decode(qw, k, v, ends, qd, kd, vd, [0], 0.5, 1, G)
    # after step 0 (9 tokens, target 5): chunk [8] forced (1 token) + the best prompt chunk
    np.testing.assert_array_equal(sels[0], np.array([0, 1, 2, 3, 8]))


def test_sliding_local_indices_are_the_last_window():
    """The local head's attended set after step t: exactly the last `window` positions of
    the grown sequence (all of them while the sequence is shorter), brute-forced."""
    for L, W in ((10, 4), (3, 8), (100, 100), (50, 1)):
        for t in range(6):
            got = O.sliding_local_indices(L, t, W)
            seq = list(range(L + t + 1))
            np.testing.assert_array_equal(got, np.array(seq[-W:] if W <= len(seq) else seq))
