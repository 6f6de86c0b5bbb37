"""Pins for the fp64 CPU oracle: closed forms, invariants, brute force.

The pages print no formula and no worked numeric example for paged decode
attention, so each pin comes from what the definition itself fixes (FlashInfer
README, core features 1-3 and the single-request decode example).  Together
they catch the plausible slips: a wrong page/offset split of the token index,
a wrong GQA head mapping, a dropped sm_scale, a log in the wrong base, a
wrong softmax normalisation, a mis-weighted merge.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from serving_attention_paged_b200 import workloads as W

D = 128


def _run(w, t, rows=None, tables=None):
    indptr, indices, last = tables if tables is not None else (w.kv_indptr, w.kv_indices,
                                                              w.last_page_len)
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], indptr, indices, last,
                               num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads,
                               head_dim=w.head_dim, page_size=w.page_size, dtype=w.dtype,
                               sm_scale=w.sm_scale, rows=rows)


def _f64(x):
    return x.detach().to(torch.float64).numpy()


# --------------------------------------------------------------------------
# widening of the 16-bit inputs
# --------------------------------------------------------------------------

def test_widen_fp16_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.widen(int(b), "f16") for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_widen_bf16_all_patterns():
    bits = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.widen(int(b) & 0xFFFF, "bf16") for b in bits.tolist()])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_token_gives_v_exactly(dtype):
    w = W.make_workload("one", [1, 1, 1], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype=dtype, seed=11, extra_pages=5)
    t = w.materialize()
    o, lse = _run(w, t)
    q = _f64(t["q"])
    for b in range(w.batch):
        row = w.kv_indices[w.kv_indptr[b]] * w.page_size
        for hq in range(w.num_qo_heads):
            h = hq // w.group
            k = _f64(t["k_pool"].view(-1, w.num_kv_heads, D)[row, h])
            v = _f64(t["v_pool"].view(-1, w.num_kv_heads, D)[row, h])
            assert np.array_equal(o[b, hq], v)
            s0 = w.sm_scale * math.fsum(q[b, hq] * k)
            assert abs(lse[b, hq] - s0) < 1e-12


def _identical_keys_case():
    w = W.make_workload("same_k", [37, 5, 64], num_qo_heads=4, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=12)
    t = w.materialize()
    kp = t["k_pool"].view(-1, w.num_kv_heads, D)
    rows = torch.from_numpy(w.token_rows())
    kp[rows] = kp[rows[0]].clone()  # every used key row equal to the first
    return w, t


def test_identical_keys_give_mean_of_v():
    w, t = _identical_keys_case()
    o, lse = _run(w, t)
    q = _f64(t["q"])
    k0 = _f64(t["k_pool"].view(-1, w.num_kv_heads, D)[int(w.token_rows()[0])])
    lens = w.kv_lens()
    start = 0
    for b in range(w.batch):
        L = int(lens[b])
        rows = w.token_rows()[start:start + L]
        start += L
        vp = _f64(t["v_pool"].view(-1, w.num_kv_heads, D)[torch.from_numpy(rows)])
        for hq in range(w.num_qo_heads):
            h = hq // w.group
            mean_v = vp[:, h].mean(axis=0)
            assert np.max(np.abs(o[b, hq] - mean_v)) < 1e-12
            s = w.sm_scale * math.fsum(q[b, hq] * k0[h])
            assert abs(lse[b, hq] - (s + math.log(L))) < 1e-12


def test_zero_scale_gives_mean_of_v_and_log_len():
    w = W.make_workload("zero_scale", [29, 1, 50], num_qo_heads=6, num_kv_heads=3, page_size=4,
                        dtype="bf16", seed=13)
    w.sm_scale = 0.0
    t = w.materialize()
    o, lse = _run(w, t)
    rows_all = w.token_rows()
    start = 0
    for b, L in enumerate(w.kv_lens()):
        rows = torch.from_numpy(rows_all[start:start + int(L)])
        start += int(L)
        vp = _f64(t["v_pool"].view(-1, w.num_kv_heads, D)[rows])
        for hq in range(w.num_qo_heads):
            assert np.max(np.abs(o[b, hq] - vp[:, hq // w.group].mean(axis=0))) < 1e-12
            assert abs(lse[b, hq] - math.log(L)) < 1e-12


def test_empty_request():
    w = W.make_workload("empty", [0, 3, 0], num_qo_heads=2, num_kv_heads=1, page_size=16,
                        dtype="f16", seed=14)
    t = w.materialize()
    o, lse = _run(w, t)
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert np.all(np.isneginf(lse[[0, 2]]))
    assert np.all(np.isfinite(lse[1]))


# --------------------------------------------------------------------------
# brute force on tiny inputs: contiguous tensors, naive softmax
# --------------------------------------------------------------------------

@pytest.mark.parametrize("P,dtype,hq,hkv", [(1, "f16", 4, 4), (4, "bf16", 6, 2), (16, "f16", 8, 1)])
def test_dense_brute_force(P, dtype, hq, hkv):
    lens = [1, 7, 40]
    w = W.make_workload("brute", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=P,
                        dtype=dtype, seed=15, extra_pages=3)
    t = w.materialize()
    o, lse = _run(w, t)
    q = _f64(t["q"])
    tok = 0
    for b, L in enumerate(lens):
        # logical K/V drawn straight from the generator: no page table involved
        K = _f64(w.logical_kv("k", tok, tok + L))
        V = _f64(w.logical_kv("v", tok, tok + L))
        tok += L
        for h in range(hq):
            kh, vh = K[:, h // (hq // hkv)], V[:, h // (hq // hkv)]
            s = (kh @ q[b, h]) * w.sm_scale
            e = np.exp(s)  # no max subtraction: safe at these sizes
            ref_o = (e[:, None] * vh).sum(0) / e.sum()
            ref_lse = np.log(e.sum())
            assert np.max(np.abs(o[b, h] - ref_o)) < 1e-12
            assert abs(lse[b, h] - ref_lse) < 1e-12


def test_dense_brute_force_small_head_dim_by_hand():
    """D = 4, two tokens, hand-sized numbers: o and lse follow from two exps."""
    q = np.array([[[1.0, 0.0, 0.5, -1.0]]], dtype=np.float16)          # [B=1, Hq=1, D=4]
    k = np.array([[[[0.5, 1.0, 0.0, 0.0]]], [[[1.0, 0.0, 2.0, 1.0]]]], dtype=np.float16)
    v = np.array([[[[1.0, 2.0, 3.0, 4.0]]], [[[-1.0, 0.0, 1.0, 0.5]]]], dtype=np.float16)
    # pool: 2 pages of 1 token; request reads page 1 then page 0
    o, lse = oracle.paged_decode(q, k, v, [0, 2], [1, 0], [1], num_qo_heads=1, num_kv_heads=1,
                                 head_dim=4, page_size=1, dtype="f16", sm_scale=0.5)
    s = [0.5 * (1.0 + 1.0 - 1.0), 0.5 * 0.5]  # token 0 = page 1 = k[1]; token 1 = k[0]
    z = math.exp(s[0]) + math.exp(s[1])
    ref = (math.exp(s[0]) * np.array([-1, 0, 1, 0.5]) + math.exp(s[1]) * np.array([1, 2, 3, 4])) / z
    assert np.max(np.abs(o[0, 0] - ref)) < 1e-15
    assert abs(lse[0, 0] - math.log(z)) < 1e-15


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_page_permutation_invariance_bitwise():
    lens = [33, 100, 16, 1]
    a = W.make_workload("perm_a", lens, num_qo_heads=8, num_kv_heads=4, page_size=16,
                        dtype="bf16", seed=21, shuffle=True, extra_pages=7)
    b = W.make_workload("perm_b", lens, num_qo_heads=8, num_kv_heads=4, page_size=16,
                        dtype="bf16", seed=21, shuffle=False, extra_pages=7)
    assert not np.array_equal(a.kv_indices, b.kv_indices)
    oa, la = _run(a, a.materialize())
    ob, lb = _run(b, b.materialize())
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_page_size_invariance_bitwise():
    lens = [65, 3, 128, 200]
    res = []
    for P in (1, 16, 64):
        w = W.make_workload("psize", lens, num_qo_heads=4, num_kv_heads=2, page_size=P,
                            dtype="f16", seed=22)
        res.append(_run(w, w.materialize()))
    for o, l in res[1:]:
        assert np.array_equal(o, res[0][0]) and np.array_equal(l, res[0][1])


def test_gqa_equals_duplicated_kv_heads():
    lens = [20, 45]
    g, hkv = 4, 2
    w = W.make_workload("gqa", lens, num_qo_heads=g * hkv, num_kv_heads=hkv, page_size=8,
                        dtype="f16", seed=23)
    t = w.materialize()
    o, lse = _run(w, t)
    # the same problem as plain multi-head attention: kv head h copied to q heads h*g..h*g+g-1
    kp = t["k_pool"].repeat_interleave(g, dim=2)
    vp = t["v_pool"].repeat_interleave(g, dim=2)
    o2, l2 = oracle.paged_decode(t["q"], kp, vp, w.kv_indptr, w.kv_indices, w.last_page_len,
                                 num_qo_heads=g * hkv, num_kv_heads=g * hkv, head_dim=D,
                                 page_size=8, dtype="f16", sm_scale=w.sm_scale)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_lse_merge_of_every_split_equals_whole():
    L = 23
    w = W.make_workload("split", [L], num_qo_heads=2, num_kv_heads=1, page_size=1,
                        dtype="bf16", seed=24)
    t = w.materialize()
    o_all, l_all = _run(w, t)
    idx = w.kv_indices
    for m in range(0, L + 1):
        # two "requests" reading tokens [0, m) and [m, L) of the same pool
        tables = (np.array([0, m, L], np.int32), idx, np.array([1 if m else 0, 1 if L - m else 0],
                                                               np.int32))
        q2 = t["q"].repeat(2, 1, 1)
        o2, l2 = oracle.paged_decode(q2, t["k_pool"], t["v_pool"], *tables, num_qo_heads=2,
                                     num_kv_heads=1, head_dim=D, page_size=1, dtype="bf16",
                                     sm_scale=w.sm_scale)
        om, lm = oracle.merge_state(o2[0], l2[0], o2[1], l2[1])
        assert np.max(np.abs(om - o_all[0])) < 1e-12
        assert np.max(np.abs(lm - l_all[0])) < 1e-12


def test_merge_state_special_cases():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((3, 5))
    l = rng.standard_normal(3)
    ninf = np.full(3, -np.inf)
    om, lm = oracle.merge_state(o, l, np.zeros((3, 5)), ninf)
    assert np.array_equal(om, o) and np.array_equal(lm, l)
    om, lm = oracle.merge_state(o, l, o, l)  # the same state twice: weights 1/2 each
    assert np.max(np.abs(om - o)) < 1e-15 and np.max(np.abs(lm - (l + math.log(2)))) < 1e-15
    om, lm = oracle.merge_state(o, ninf, o, ninf)
    assert np.all(om == 0) and np.all(np.isneginf(lm))
    # weights follow exp(lse): lse_b = lse_a + ln 3 gives o = (o_a + 3 o_b) / 4
    o2 = rng.standard_normal((3, 5))
    om, lm = oracle.merge_state(o, l, o2, l + math.log(3))
    assert np.max(np.abs(om - (o + 3 * o2) / 4)) < 1e-14
    assert np.max(np.abs(lm - (l + math.log(4)))) < 1e-14


def test_cascade_equals_attention_over_concatenation():
    w = W.make_workload("casc", [5, 0, 40, 17], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=25, prefix_len=64)
    t = w.materialize()
    oc, lc = oracle.cascade_decode(t["q"], t["k_pool"], t["v_pool"], w.prefix_indices,
                                   w.prefix_len, w.kv_indptr, w.kv_indices, w.last_page_len,
                                   num_qo_heads=8, num_kv_heads=2, head_dim=D, page_size=16,
                                   dtype="f16", sm_scale=w.sm_scale)
    of, lf = _run(w, t, tables=w.flat_tables())
    assert np.max(np.abs(oc - of)) < 1e-12
    assert np.max(np.abs(lc - lf)) < 1e-12


def test_row_subset_matches_full():
    w = W.make_workload("rows", [30, 70], num_qo_heads=4, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=26)
    t = w.materialize()
    o, lse = _run(w, t)
    rows = np.array([7, 0, 5])
    o2, l2 = _run(w, t, rows=rows)
    assert np.array_equal(o2, o.reshape(-1, D)[rows]) and np.array_equal(l2, lse.reshape(-1)[rows])
    o3, l3 = oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr, w.kv_indices,
                                 w.last_page_len, num_qo_heads=4, num_kv_heads=2, head_dim=D,
                                 page_size=16, dtype="f16", sm_scale=w.sm_scale, threads=4)
    assert np.array_equal(o3, o) and np.array_equal(l3, lse)


def test_request_subset_matches_full_bitwise():
    w = W.make_workload("subset", [30, 0, 70, 5], num_qo_heads=4, num_kv_heads=2, page_size=16,
                        dtype="bf16", seed=27, extra_pages=9)
    t = w.materialize()
    o, lse = _run(w, t)
    reqs = [2, 1, 3]
    o2, l2 = oracle.paged_decode_requests(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr,
                                          w.kv_indices, w.last_page_len, reqs, num_qo_heads=4,
                                          num_kv_heads=2, head_dim=D, page_size=16,
                                          dtype="bf16", sm_scale=w.sm_scale)
    assert np.array_equal(o2, o[reqs]) and np.array_equal(l2, lse[reqs])
