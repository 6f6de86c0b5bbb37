"""Pins for the oracle's prefill / append attention (README usage example:
prefill and append attention over a paged KV cache, causal).

The oracle evaluates each new query token as a decode over its request's
pages cut at the query's limit (its causal position, or all keys without
the mask).  The pins check that against what the definition fixes
independently: dense attention written out with a naive softmax on
contiguous tensors (causal and not), the first query of a fresh prefill
(one visible key: o = V_0, lse = s_0), and causality itself (a key's values
change only the queries that may see it).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from serving_attention_paged_b200 import workloads as W


def _widen(t, dtype):
    """16-bit tensor -> fp64 through the oracle's exact widening table."""
    bits = t.contiguous().view(torch.int16).view(-1).numpy().view(np.uint16).astype(np.int64)
    table = np.array([oracle.widen(b, dtype) for b in range(1 << 16)])
    return table[bits].reshape(tuple(t.shape))


def _dense(w, t, causal=True):
    """Attention on contiguous per-request K/V in the generator's logical token
    order (no pages), naive softmax in fp64; a query that sees no key gets
    o = 0, lse = -inf."""
    G, D = w.group, w.head_dim
    q = _widen(t["q"], w.dtype)
    lens, qo = w.kv_lens(), w.qo_indptr
    start = np.concatenate([[0], np.cumsum(lens)])
    o = np.zeros(q.shape)
    lse = np.zeros(q.shape[:2])
    for b in range(w.batch):
        K = _widen(w.logical_kv("k", int(start[b]), int(start[b + 1])), w.dtype)
        V = _widen(w.logical_kv("v", int(start[b]), int(start[b + 1])), w.dtype)
        Q = qo[b + 1] - qo[b]
        for i in range(Q):
            lim = int(lens[b]) - Q + i + 1 if causal else int(lens[b])
            if lim == 0:
                lse[qo[b] + i] = -np.inf
                continue
            for hq in range(w.num_qo_heads):
                s = w.sm_scale * (K[:lim, hq // G, :] @ q[qo[b] + i, hq])
                e = np.exp(s)  # tiny inputs: no max subtraction needed
                o[qo[b] + i, hq] = (e @ V[:lim, hq // G, :]) / e.sum()
                lse[qo[b] + i, hq] = math.log(e.sum())
    return o, lse


def _prefill(w, t, **kw):
    return oracle.paged_prefill(t["q"], t["k_pool"], t["v_pool"], w.qo_indptr, w.kv_indptr,
                                w.kv_indices, w.last_page_len, num_qo_heads=w.num_qo_heads,
                                num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                                page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, **kw)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_matches_dense_causal_brute_force(dtype):
    w = W.make_workload("pf_tiny", [7, 5, 9, 3], num_qo_heads=4, num_kv_heads=2, head_dim=16,
                        page_size=4, dtype=dtype, seed=31, qo_lens=[3, 5, 1, 0])
    t = w.materialize()
    o, lse = _prefill(w, t)
    o_ref, l_ref = _dense(w, t)
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse - l_ref).max() < 1e-12


def test_first_query_of_a_fresh_prefill_sees_one_key():
    """Q_b = L_b: query 0 of each request sees key 0 only: o = V_0 exactly and
    lse = s_0 = sm_scale <q, K_0>."""
    w = W.make_workload("pf_fresh", [6, 11], num_qo_heads=4, num_kv_heads=1, head_dim=16,
                        page_size=4, dtype="f16", seed=32, qo_lens=[6, 11])
    t = w.materialize()
    o, lse = _prefill(w, t)
    start = np.concatenate([[0], np.cumsum(w.kv_lens())])
    q = _widen(t["q"], "f16")
    for b in range(w.batch):
        K0 = _widen(w.logical_kv("k", int(start[b]), int(start[b]) + 1), "f16")[0, 0]
        V0 = _widen(w.logical_kv("v", int(start[b]), int(start[b]) + 1), "f16")[0, 0]
        row = w.qo_indptr[b]
        assert np.array_equal(o[row], np.broadcast_to(V0, o[row].shape))
        assert np.allclose(lse[row], w.sm_scale * (q[row] @ K0), rtol=0, atol=1e-12)


def test_causality_a_key_changes_only_the_queries_that_see_it():
    w = W.make_workload("pf_causal", [10, 8], num_qo_heads=2, num_kv_heads=1, head_dim=16,
                        page_size=4, dtype="bf16", seed=33, qo_lens=[4, 8])
    t = w.materialize()
    o1, l1 = _prefill(w, t)
    # key 8 of request 0 (of 10; its 4 queries see keys < 7, 8, 9, 10)
    rows = w.token_rows()
    t2 = dict(t)
    t2["k_pool"] = t["k_pool"].clone()
    t2["v_pool"] = t["v_pool"].clone()
    flat_k = t2["k_pool"].view(-1, w.num_kv_heads, w.head_dim)
    flat_v = t2["v_pool"].view(-1, w.num_kv_heads, w.head_dim)
    flat_k[int(rows[8])] += 1.0
    flat_v[int(rows[8])] -= 2.0
    o2, l2 = _prefill(w, t2)
    sees = np.array([False, False, True, True] + [False] * 8)  # queries of request 0, then 1
    for g in range(w.query_rows()):
        same = np.array_equal(o1[g], o2[g]) and np.array_equal(l1[g], l2[g])
        assert same != sees[g], g


def test_last_query_equals_decode_over_the_whole_request():
    w = W.make_workload("pf_last", [33, 20, 64], num_qo_heads=8, num_kv_heads=2, head_dim=16,
                        page_size=8, dtype="f16", seed=34, qo_lens=[5, 20, 1])
    t = w.materialize()
    last_rows = w.qo_indptr[1:] - 1
    o, lse = _prefill(w, t, queries=last_rows)
    od, ld = oracle.paged_decode(t["q"][last_rows], t["k_pool"], t["v_pool"], w.kv_indptr,
                                 w.kv_indices, w.last_page_len, num_qo_heads=8, num_kv_heads=2,
                                 head_dim=16, page_size=8, dtype="f16", sm_scale=w.sm_scale)
    assert np.array_equal(o, od) and np.array_equal(lse, ld)


def test_prefill_rejects_more_queries_than_keys():
    w = W.make_workload("pf_bad", [4], num_qo_heads=2, num_kv_heads=1, head_dim=16,
                        page_size=4, dtype="f16", seed=35, qo_lens=[5])
    t = w.materialize()
    with pytest.raises(ValueError):
        _prefill(w, t)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_without_mask_matches_dense_brute_force(dtype):
    """No causal mask: every query sees all of its request's keys; more
    queries than keys and a request without keys are allowed."""
    w = W.make_workload("pf_nomask", [7, 0, 9, 2], num_qo_heads=4, num_kv_heads=2, head_dim=16,
                        page_size=4, dtype=dtype, seed=36, qo_lens=[3, 2, 1, 5])
    t = w.materialize()
    o, lse = _prefill(w, t, causal=False)
    o_ref, l_ref = _dense(w, t, causal=False)
    empty = np.isneginf(l_ref)
    assert empty.sum() == 2 * w.num_qo_heads
    assert np.array_equal(np.isneginf(lse), empty) and np.all(o[empty] == 0)
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse[~empty] - l_ref[~empty]).max() < 1e-12
