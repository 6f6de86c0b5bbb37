"""Pins for the oracle's split-KV plan (README core feature 2, plan stage).

The page names the plan/run split and its purpose (even out the load of
variable-length inputs) but gives no algorithm, so the pins are a worked
example done by hand from the adopted specification plus the properties
any correct work list must have: every (request, kv head, token) covered
exactly once, chunks page-aligned, the chunk size minimal under the budget.
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
        c, items, merge_indptr = oracle.plan(g["kv_indptr"], g["last_page_len"],
                                             page_size=g["page_size"],
                                             num_kv_heads=g["num_kv_heads"],
                                             num_sms=g["num_sms"], ctas_per_sm=g["ctas_per_sm"],
                                             min_chunk_tokens=g["min_chunk_tokens"])
        assert c == g["chunk_pages"]
        assert merge_indptr.tolist() == g["merge_indptr"]
        assert items.tolist() == g["items"]


def _work(n, c, hkv):
    return hkv * sum(max(1, -(-nb // c)) for nb in n)


def check_plan_properties(indptr, last, P, hkv, W_, c_min_tokens, c, items, merge_indptr):
    indptr = np.asarray(indptr, np.int64)
    last = np.asarray(last, np.int64)
    B = len(last)
    n = np.diff(indptr)
    lens = np.where(n > 0, (n - 1) * P + last, 0)
    c_min = max(1, -(-c_min_tokens // P))
    N = int(n.max()) if B else 0
    # chunk size minimal under the budget of k waves
    budget = max(1, -(-(hkv * B) // W_)) * W_
    if N <= c_min:
        assert c == max(N, 1)
    else:
        assert c_min <= c <= N
        assert _work(n, c, hkv) <= budget
        if c > c_min:
            assert _work(n, c - 1, hkv) > budget
    assert len(items) == _work(n, c, hkv)
    if B * hkv <= W_:
        assert len(items) <= W_
    # launch order: longest chunk first
    assert all(items[i, 4] >= items[i + 1, 4] for i in range(len(items) - 1))
    # coverage: per (b, h) the chunks tile [indptr[b], indptr[b+1]) in order
    cover = {}
    for (b, h, pb, pe, kl, slot) in sorted(items.tolist(), key=lambda x: (x[0], x[2], x[1])):
        assert 0 <= pe - pb <= c
        assert pb == indptr[b] or (pb - indptr[b]) % c == 0
        cover.setdefault((b, h), []).append((pb, pe, kl, slot))
    for b in range(B):
        nch = max(1, -(-int(n[b]) // c))
        assert merge_indptr[b + 1] - merge_indptr[b] == (nch if nch > 1 else 0)
        for h in range(hkv):
            ch = cover[(b, h)]
            assert len(ch) == nch
            pos = int(indptr[b])
            tot = 0
            for j, (pb, pe, kl, slot) in enumerate(ch):
                assert pb == pos
                pos = pe
                tot += kl
                assert slot == (-1 if nch == 1 else merge_indptr[b] + j)
            assert pos == indptr[b + 1]
            assert tot == lens[b]


@pytest.mark.parametrize("seed", range(12))
def test_plan_properties_random(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(0, 40))
    P = int(rng.choice([1, 2, 16, 64]))
    lens = rng.integers(0, 3000, size=B) * (rng.random(B) > 0.1)
    indptr, _, last = W.tables_from_lengths(lens, P)
    hkv = int(rng.choice([1, 2, 8]))
    sms, k = int(rng.integers(1, 200)), int(rng.integers(1, 4))
    mct = int(rng.choice([1, 64, 256, 1000]))
    c, items, mi = oracle.plan(indptr, last, page_size=P, num_kv_heads=hkv, num_sms=sms,
                               ctas_per_sm=k, min_chunk_tokens=mct)
    check_plan_properties(indptr, last, P, hkv, sms * k, mct, c, items, mi)


def test_plan_empty_batch():
    c, items, mi = oracle.plan(np.zeros(1, np.int32), np.zeros(0, np.int32), page_size=16,
                               num_kv_heads=8, num_sms=148, ctas_per_sm=2)
    assert c == 1 and items.shape == (0, 6) and mi.tolist() == [0]


def test_plan_benchmark_shapes():
    for n in (1, 2, 3):
        w = W.WORKLOADS[n]()
        c, items, mi = oracle.plan(w.kv_indptr, w.last_page_len, page_size=w.page_size,
                                   num_kv_heads=w.num_kv_heads, num_sms=148, ctas_per_sm=2)
        check_plan_properties(w.kv_indptr, w.last_page_len, w.page_size, w.num_kv_heads, 296,
                              256, c, items, mi)
