"""Pins for the oracle's split-KV plan (README core feature 2, plan stage).

The page names the plan/run split and its purpose (even out the load of
variable-length inputs) and lists stream-K among FlashInfer's influences,
but gives no algorithm.  So the pins are small cases worked by hand from the
adopted stream-K style specification plus the properties any correct work
list of that kind must have: every (request, kv head, token) covered exactly
once and in order, every CTA but the last given exactly the quota, partial
slots consistent with the merge offsets.
"""
import json
import os

import numpy as np
import pytest

import oracle
from serving_attention_paged_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "plan_small.json")


def test_plan_hand_worked_examples():
    for g in json.load(open(GOLDEN))["cases"]:
        q, items, cta_indptr, merge_indptr = oracle.plan(
            g["kv_indptr"], g["last_page_len"], page_size=g["page_size"],
            num_kv_heads=g["num_kv_heads"], num_sms=g["num_sms"], ctas_per_sm=g["ctas_per_sm"],
            min_chunk_tokens=g["min_chunk_tokens"], piece_cost=g.get("piece_cost_tokens", 0))
        assert q == g["quota"]
        assert cta_indptr.tolist() == g["cta_indptr"]
        assert merge_indptr.tolist() == g["merge_indptr"]
        assert items.tolist() == g["items"]


def check_plan_properties(indptr, last, P, hkv, W_, min_tokens, q, items, cta_indptr,
                          merge_indptr, c=0):
    indptr = np.asarray(indptr, np.int64)
    last = np.asarray(last, np.int64)
    B = len(last)
    n = np.diff(indptr)
    lens = np.where(n > 0, (n - 1) * P + last, 0)
    T = int(lens.sum())
    N = int((lens > 0).sum())
    groups = max(1, W_ // hkv)
    share = max(min_tokens, -(-(T + c * max(N - 1, 0)) // groups))
    assert q % 32 == 0 and share <= q < share + 32
    n_cta = len(cta_indptr) - 1
    n_groups = n_cta // hkv
    assert n_cta == n_groups * hkv and n_groups <= groups  # one wave: every CTA resident
    if c == 0:
        assert n_groups == (0 if B == 0 else max(1, -(-T // q)))
    assert cta_indptr[0] == 0 and cta_indptr[-1] == len(items)
    assert all(cta_indptr[i] <= cta_indptr[i + 1] for i in range(n_cta))
    cta = [items[cta_indptr[i]:cta_indptr[i + 1]] for i in range(n_cta)]
    for g in range(n_groups):
        ranges = None
        for h in range(hkv):
            mine = cta[g * hkv + h]
            assert np.all(mine[:, 1] == h)
            r = mine[:, [0, 3, 4]].tolist()
            ranges = r if ranges is None else ranges
            assert r == ranges  # the Hkv CTAs of a group read the same tokens
        tokens = sum(t1 - t0 for _, t0, t1 in ranges)
        used = tokens + c * max(sum(1 for _, t0, t1 in ranges if t1 > t0) - 1, 0)
        assert used <= q  # the budget holds
        if g < n_groups - 1:
            # balance: a group closes only when the next token would not fit
            assert used + c >= q and (c > 0 or tokens == q)
    # coverage: per (b, h) the pieces tile [0, L_b) in token order
    for b in range(B):
        for h in range(hkv):
            ps = [it for it in items.tolist() if it[0] == b and it[1] == h]
            assert len(ps) >= 1
            pos = 0
            for it in ps:
                assert it[2] == indptr[b] and it[3] == pos and it[4] >= it[3]
                pos = it[4]
            assert pos == lens[b]
            seg = b * hkv + h
            k = merge_indptr[seg + 1] - merge_indptr[seg]
            assert k == (len(ps) if len(ps) > 1 else 0)
            assert [it[5] for it in ps] == ([-1] if len(ps) == 1 else
                                            list(range(merge_indptr[seg], merge_indptr[seg + 1])))


@pytest.mark.parametrize("c", [0, 37, 160])
@pytest.mark.parametrize("seed", range(12))
def test_plan_properties_random(seed, c):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(0, 40))
    P = int(rng.choice([1, 2, 16, 64]))
    lens = rng.integers(0, 3000, size=B) * (rng.random(B) > 0.1)
    indptr, _, last = W.tables_from_lengths(lens, P)
    hkv = int(rng.choice([1, 2, 8]))
    sms, k = int(rng.integers(1, 200)), int(rng.integers(1, 4))
    mct = int(rng.choice([1, 64, 256, 1000]))
    q, items, ci, mi = oracle.plan(indptr, last, page_size=P, num_kv_heads=hkv, num_sms=sms,
                                   ctas_per_sm=k, min_chunk_tokens=mct, piece_cost=c)
    check_plan_properties(indptr, last, P, hkv, sms * k, mct, q, items, ci, mi, c)


def test_plan_empty_batch():
    q, items, ci, mi = oracle.plan(np.zeros(1, np.int32), np.zeros(0, np.int32), page_size=16,
                                   num_kv_heads=8, num_sms=148, ctas_per_sm=2)
    assert items.shape == (0, 6) and ci.tolist() == [0] and mi.tolist() == [0]
    assert q == 256


@pytest.mark.parametrize("c", [0, 160, 256])
def test_plan_benchmark_shapes(c):
    for n in (1, 2, 3):
        w = W.WORKLOADS[n]()
        q, items, ci, mi = oracle.plan(w.kv_indptr, w.last_page_len, page_size=w.page_size,
                                       num_kv_heads=w.num_kv_heads, num_sms=148, ctas_per_sm=4,
                                       piece_cost=c)
        check_plan_properties(w.kv_indptr, w.last_page_len, w.page_size, w.num_kv_heads, 592,
                              256, q, items, ci, mi, c)


def test_piece_cost_shifts_tokens_to_single_piece_groups():
    """With a piece cost c, a group of k pieces reads between q - c k and
    q - c (k - 1) tokens (it closes once the next piece would not fit), so a
    two-piece group reads about c fewer tokens than a one-piece group
    (uniform batch: 16 x 4096 tokens)."""
    w = W.WORKLOADS[2]()
    for c in (160, 256):
        q, items, ci, _ = oracle.plan(w.kv_indptr, w.last_page_len, page_size=16, num_kv_heads=8,
                                      num_sms=148, ctas_per_sm=3, piece_cost=c)
        groups = [items[ci[g * 8]:ci[g * 8 + 1]] for g in range((len(ci) - 1) // 8)]
        by_k = {}
        for pcs in groups[:-1]:
            k = len(pcs)
            tok = int((pcs[:, 4] - pcs[:, 3]).sum())
            assert q - c * k <= tok <= q - c * (k - 1)
            by_k.setdefault(k, []).append(tok)
        assert set(by_k) == {1, 2}
        assert np.mean(by_k[1]) - np.mean(by_k[2]) > c / 2


def sliced_work_list(lens, indptr, hkv, q):
    """The c = 0 rule stated a second way, without the walk: lay the requests'
    tokens end to end (request b at positions [s_b, s_b + L_b)); group g is
    the positions [g q, (g + 1) q) and holds, in request order, every request
    that overlaps it, cut to the overlap.  An empty request sits at s_b and
    belongs to the group of that position (the last group if s_b = T)."""
    lens = [int(x) for x in lens]
    T = sum(lens)
    n_groups = max(1, -(-T // q)) if lens else 0
    groups = [[] for _ in range(n_groups)]
    s = 0
    for b, L in enumerate(lens):
        if L == 0:
            groups[min(s // q, n_groups - 1)].append((b, 0, 0))
        for g in range(s // q, min(n_groups, -(-(s + L) // q))):
            lo, hi = max(s, g * q), min(s + L, (g + 1) * q)
            if hi > lo:
                groups[g].append((b, lo - s, hi - s))
        s += L
    return [[b, h, int(indptr[b]), t0, t1] for g in groups for h in range(hkv)
            for (b, t0, t1) in g]


@pytest.mark.parametrize("seed", range(20))
def test_plan_without_piece_cost_is_a_slicing_of_the_tokens(seed):
    """Pins the walk against its own definition written as arithmetic on
    token positions: an off-by-one in when a group closes, or in where an
    empty request lands, changes the sliced list."""
    rng = np.random.default_rng(500 + seed)
    B = int(rng.integers(1, 30))
    P = int(rng.choice([1, 4, 16]))
    lens = rng.integers(0, 700, size=B) * (rng.random(B) > 0.25)
    if seed % 4 == 0:  # requests ending exactly on group boundaries
        lens = np.where(lens > 0, 64 * (1 + lens // 200), 0)
    indptr, _, last = W.tables_from_lengths(lens, P)
    hkv = int(rng.choice([1, 2, 4]))
    sms = int(rng.integers(1, 40))
    q, items, ci, _ = oracle.plan(indptr, last, page_size=P, num_kv_heads=hkv, num_sms=sms,
                                  ctas_per_sm=1, min_chunk_tokens=32, piece_cost=0)
    assert items[:, :5].tolist() == sliced_work_list(lens, indptr, hkv, q)
