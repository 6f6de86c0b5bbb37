"""Pins for the oracle's 8-bit KV cache (README core feature 3: efficient
kernels for low-precision attention for a compressed KV-Cache).

The cache holds FP8 codes (OCP E4M3 without infinities, or E5M2) with one
scale for K and one for V; a cached key is k_scale * code.  The pins check
the oracle's exact widening of every code against torch's own conversion, a
few values fixed by the formats' definitions, that an 8-bit cache gives the
same attention as a 16-bit cache holding the same values, that power-of-two
scales act exactly as the definition says (on sm_scale, on o), and dense
attention written out on tiny inputs with non-power-of-two scales.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from serving_attention_paged_b200 import workloads as W

FMTS = {"e4m3": torch.float8_e4m3fn, "e5m2": torch.float8_e5m2}


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_every_code_widens_like_torch(fmt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(FMTS[fmt]).to(torch.float64).numpy()
    got = np.array([oracle.widen8(c, fmt) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_values_fixed_by_the_formats():
    e4 = lambda c: oracle.widen8(c, "e4m3")  # noqa: E731
    e5 = lambda c: oracle.widen8(c, "e5m2")  # noqa: E731
    # E4M3: bias 7, 3 fraction bits, no infinities, max 448, NaN only at S.1111.111
    assert e4(0x38) == 1.0 and e4(0xB8) == -1.0
    assert e4(0x7E) == 448.0 and e4(0x08) == 2.0 ** -6 and e4(0x01) == 2.0 ** -9
    assert e4(0x7F) != e4(0x7F) and e4(0x78) == 256.0  # 0x78: exponent all ones is a number
    assert e4(0x00) == 0.0 and math.copysign(1.0, e4(0x80)) == -1.0
    # E5M2: bias 15, 2 fraction bits, IEEE infinities
    assert e5(0x3C) == 1.0 and e5(0x7B) == 57344.0 and e5(0x7C) == math.inf
    assert e5(0x04) == 2.0 ** -14 and e5(0x01) == 2.0 ** -16 and e5(0x7D) != e5(0x7D)


def _decode(w, t, **kw):
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr, w.kv_indices,
                               w.last_page_len, num_qo_heads=w.num_qo_heads,
                               num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                               page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, **kw)


def _fp8_workload(fmt, k_scale=1.0, v_scale=1.0, dtype="f16", seed=41):
    return W.make_workload("fp8", [9, 0, 33, 16], num_qo_heads=8, num_kv_heads=2, head_dim=32,
                           page_size=8, dtype=dtype, seed=seed, kv_dtype=fmt, k_scale=k_scale,
                           v_scale=v_scale)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_fp8_cache_equals_a_16bit_cache_of_the_same_values(fmt, dtype):
    """Every FP8 value is exact in fp16 and in bf16 (E4M3 spans 2^-9 .. 448 with
    3 fraction bits, E5M2 is the top byte of fp16), so with unit scales the
    attention must be bitwise the one over a 16-bit cache (in q's dtype)
    holding those values."""
    w = _fp8_workload(fmt, dtype=dtype)
    t = w.materialize()
    o8, l8 = _decode(w, t, kv_dtype=fmt)
    wide = W.DTYPES[dtype]
    t16 = dict(t, k_pool=t["k_pool"].to(wide), v_pool=t["v_pool"].to(wide))
    assert torch.equal(t16["k_pool"].to(torch.float64), t["k_pool"].to(torch.float64))
    o16, l16 = _decode(w, t16)
    assert np.array_equal(o8, o16) and np.array_equal(l8, l16)
    assert np.isneginf(l8[1]).all() and (o8[1] == 0).all()  # the empty request


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_power_of_two_scales_act_exactly(fmt):
    """k_scale = 2^j multiplies every score exactly like sm_scale * 2^j;
    v_scale = 2^j multiplies o exactly and leaves lse alone."""
    base = _fp8_workload(fmt, 1.0, 1.0, seed=42)
    t = base.materialize()
    o, l = _decode(base, t, kv_dtype=fmt)
    o_k, l_k = _decode(base, t, kv_dtype=fmt, k_scale=0.5)
    w2 = W.make_workload("fp8", [9, 0, 33, 16], num_qo_heads=8, num_kv_heads=2, head_dim=32,
                         page_size=8, dtype="f16", seed=42, kv_dtype=fmt,
                         sm_scale=base.sm_scale * 0.5)
    o_s, l_s = _decode(w2, t, kv_dtype=fmt)
    assert np.array_equal(o_k, o_s) and np.array_equal(l_k, l_s)
    o_v, l_v = _decode(base, t, kv_dtype=fmt, v_scale=4.0)
    assert np.array_equal(o_v, 4.0 * o) and np.array_equal(l_v, l)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_fp8_decode_matches_dense_brute_force(fmt, dtype):
    """Dense attention on the generator's logical token order, values widened
    by torch (not the oracle's table) and scaled, naive softmax in fp64."""
    ks, vs = 0.37, 1.9
    w = _fp8_workload(fmt, ks, vs, dtype=dtype, seed=43)
    t = w.materialize()
    o, lse = _decode(w, t, kv_dtype=fmt, k_scale=ks, v_scale=vs)
    q = t["q"].to(torch.float64).numpy()
    lens = w.kv_lens()
    start = np.concatenate([[0], np.cumsum(lens)])
    G = w.group
    for b in range(w.batch):
        if lens[b] == 0:
            assert np.isneginf(lse[b]).all() and (o[b] == 0).all()
            continue
        K = ks * w.logical_kv("k", int(start[b]), int(start[b + 1])).to(torch.float64).numpy()
        V = vs * w.logical_kv("v", int(start[b]), int(start[b + 1])).to(torch.float64).numpy()
        for hq in range(w.num_qo_heads):
            s = w.sm_scale * (K[:, hq // G, :] @ q[b, hq])
            e = np.exp(s)
            assert abs(lse[b, hq] - math.log(e.sum())) < 1e-12
            assert np.abs(o[b, hq] - (e @ V[:, hq // G, :]) / e.sum()).max() < 1e-12


def test_fp8_pool_bytes():
    w = _fp8_workload("e4m3")
    assert w.kv_bytes() == 2 * int(w.kv_lens().sum()) * w.num_kv_heads * w.head_dim
