"""Pins for the oracle's rotary positions on the fly (README usage example:
decode with LLaMA-style RoPE, ``pos_encoding_mode="ROPE_LLAMA"``).

q is rotated to its position L_b - 1 and key t to position t; element pairs
(d, d + D/2) turn by pos * theta^(-2d/D); values are not rotated.  The pins
check that against properties the definition fixes independently of how
the oracle composes it: position 0 is the identity (a one-token request is
unchanged, bitwise); only relative positions matter (the same attention
written out densely with q left alone and each key turned by t - (L_b - 1));
positions are logical token indices, so the page layout cannot change the
result (bitwise); and a huge theta leaves every pair but the first still
(to fp64 rounding).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from serving_attention_paged_b200 import workloads as W

THETA = 10000.0


def _decode(w, t, **kw):
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr, w.kv_indices,
                               w.last_page_len, num_qo_heads=w.num_qo_heads,
                               num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                               page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, **kw)


def _turn(x, angles):
    """x [..., D] with pairs (d, d + D/2) turned by angles [..., D/2]."""
    h = x.shape[-1] // 2
    c, s = np.cos(angles), np.sin(angles)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def test_position_zero_is_the_identity():
    w = W.make_workload("rope1", [1, 1, 1], num_qo_heads=8, num_kv_heads=2, head_dim=32,
                        page_size=4, dtype="f16", seed=51)
    t = w.materialize()
    assert all(np.array_equal(a, b) for a, b in zip(_decode(w, t, rope_theta=THETA),
                                                     _decode(w, t)))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_only_relative_positions_matter(dtype):
    """RoPE(q, m) . RoPE(k, n) = q . RoPE(k, n - m): dense attention with q as
    it is and key t turned by t - (L_b - 1) must give the same result."""
    w = W.make_workload("rope_rel", [37, 5, 0, 64], num_qo_heads=8, num_kv_heads=2,
                        head_dim=32, page_size=8, dtype=dtype, seed=52)
    t = w.materialize()
    o, lse = _decode(w, t, rope_theta=THETA)
    q = t["q"].to(torch.float64).numpy()
    lens = w.kv_lens()
    start = np.concatenate([[0], np.cumsum(lens)])
    D, G = w.head_dim, w.group
    inv_freq = THETA ** (-2.0 * np.arange(D // 2) / D)
    for b in range(w.batch):
        L = int(lens[b])
        if L == 0:
            assert np.isneginf(lse[b]).all() and (o[b] == 0).all()
            continue
        K = w.logical_kv("k", int(start[b]), int(start[b + 1])).to(torch.float64).numpy()
        V = w.logical_kv("v", int(start[b]), int(start[b + 1])).to(torch.float64).numpy()
        rel = (np.arange(L) - (L - 1))[:, None] * inv_freq[None, :]  # [L, D/2]
        Kr = _turn(K, rel[:, None, :])
        for hq in range(w.num_qo_heads):
            s = w.sm_scale * (Kr[:, hq // G, :] @ q[b, hq])
            m = s.max()
            e = np.exp(s - m)
            assert abs(lse[b, hq] - (m + math.log(e.sum()))) < 1e-12
            assert np.abs(o[b, hq] - (e @ V[:, hq // G, :]) / e.sum()).max() < 1e-12


def test_positions_are_logical_token_indices():
    """The same logical requests laid out with 4 or 16 tokens per page, in
    another page order, give bitwise the same rotated attention."""
    lens = [23, 0, 50, 17]
    a = W.make_workload("rope_p", lens, num_qo_heads=4, num_kv_heads=4, head_dim=16,
                        page_size=4, dtype="f16", seed=53)
    b = W.make_workload("rope_p", lens, num_qo_heads=4, num_kv_heads=4, head_dim=16,
                        page_size=16, dtype="f16", seed=53, shuffle=False)
    oa, la = _decode(a, a.materialize(), rope_theta=THETA)
    ob, lb = _decode(b, b.materialize(), rope_theta=THETA)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_huge_theta_turns_only_the_first_pair():
    """With theta = 1e300, theta^(-2d/D) is below 1e-37 for every d > 0: those
    pairs turn by angles whose cosine is 1 and whose sine term vanishes under
    fp64 rounding, so only the pair (0, D/2) turns (by pos radians).  Zeroing
    both elements of that pair in q must then give the unrotated result."""
    w = W.make_workload("rope_big", [30, 7], num_qo_heads=2, num_kv_heads=1, head_dim=16,
                        page_size=4, dtype="f16", seed=54)
    t = w.materialize()
    q = t["q"].clone()
    q[..., 0] = 0
    q[..., 8] = 0
    t0 = dict(t, q=q)
    o_r, l_r = _decode(w, t0, rope_theta=1e300)
    o_n, l_n = _decode(w, t0)
    assert np.array_equal(o_r, o_n) and np.array_equal(l_r, l_n)
    # with the first pair present the rotation shows
    o_r2, _ = _decode(w, t, rope_theta=1e300)
    o_n2, _ = _decode(w, t)
    assert not np.array_equal(o_r2, o_n2)


def test_rope_needs_an_even_head_dim():
    w = W.make_workload("rope_odd", [3], num_qo_heads=1, num_kv_heads=1, head_dim=15,
                        page_size=4, dtype="f16", seed=55)
    with pytest.raises(ValueError):
        _decode(w, w.materialize(), rope_theta=THETA)
