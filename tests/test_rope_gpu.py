"""Rotary positions applied on the fly in decode, on the GPU, against the
fp64 oracle (README usage example: decode with pos_encoding_mode="ROPE_LLAMA").

The query is rotated to its position L_b - 1 and the key of token t to t
(rotate-half pairing of elements d and d + 64) before the dot product.  The
cases cover every GQA group (the pair partner is in the same lane for groups
1-4 and 8 lanes away for group 8), both q types, page sizes 1 and 16, two
bases, split plans (the query position must come from the whole request,
not from the piece), positions beyond 32 768, and an 8-bit cache with
rotation.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu

EDGE_LENS = [0, 1, 15, 16, 17, 33, 100, 257, 1000, 3000]


def _oracle(w, t, theta, threads=8):
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr, w.kv_indices,
                               w.last_page_len, num_qo_heads=w.num_qo_heads,
                               num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                               page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale,
                               kv_dtype=w.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale,
                               rope_theta=theta, threads=threads)


def _decode(w, dev, theta, **kw):
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                     num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                     sm_scale=w.sm_scale, num_pages=w.num_pages, kv_dtype=w.kv_dtype,
                     k_scale=w.k_scale, v_scale=w.v_scale, rope_theta=theta, **kw)
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    torch.cuda.synchronize()
    assert pd.check() == -1
    return pd, o, lse


@pytest.mark.parametrize("theta", [1e4, 5e5])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("P", [1, 16])
def test_rope_small_parity(theta, dtype, group, P):
    hkv = 2
    w = W.make_workload("rope_small", EDGE_LENS, num_qo_heads=hkv * group, num_kv_heads=hkv,
                        page_size=P, dtype=dtype, seed=400 + group + P, extra_pages=3)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t, theta)
    dev = {k: v.cuda() for k, v in t.items()}
    for kw in (dict(num_sms=10000, ctas_per_sm=1),
               dict(num_sms=3, ctas_per_sm=1, min_chunk_tokens=16)):
        pd, o, lse = _decode(w, dev, theta, **kw)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype,
                     f"rope theta={theta} G={group} P={P} {kw}")


@pytest.mark.parametrize("group", [2, 8])
def test_rope_positions_beyond_32k(group):
    """Angles of tens of thousands of radians: the reduction in turns keeps
    the rotation accurate at every position."""
    w = W.make_workload("rope_long", [33000, 40001], num_qo_heads=group, num_kv_heads=1,
                        page_size=16, dtype="bf16", seed=410 + group)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t, 1e4)
    dev = {k: v.cuda() for k, v in t.items()}
    for kw in (dict(num_sms=148, ctas_per_sm=2), dict(num_sms=1, ctas_per_sm=1)):
        pd, o, lse = _decode(w, dev, 1e4, **kw)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16", f"rope long G={group} {kw}")


@pytest.mark.parametrize("group", [4, 8])
def test_rope_with_fp8_cache(group):
    w = W.make_workload("rope_fp8", [700, 0, 129, 2500], num_qo_heads=2 * group, num_kv_heads=2,
                        page_size=16, dtype="f16", seed=420 + group, kv_dtype="e4m3",
                        k_scale=0.3, v_scale=0.7)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t, 1e4)
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o, lse = _decode(w, dev, 1e4, num_sms=9, ctas_per_sm=1, min_chunk_tokens=64)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "f16", f"rope fp8 G={group}")


def test_rope_changes_the_result_and_zero_theta_does_not():
    """Guards against a silently ignored rotation: with rope_theta > 0 the
    output differs from plain decode; with 0 it is plain decode, bitwise."""
    w = W.make_workload("rope_onoff", [500, 90], num_qo_heads=16, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=430)
    dev = {k: v.cuda() for k, v in w.materialize().items()}
    _, o_rope, _ = _decode(w, dev, 1e4, num_sms=148, ctas_per_sm=2)
    _, o_zero, l_zero = _decode(w, dev, 0.0, num_sms=148, ctas_per_sm=2)
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=16, num_kv_heads=2,
                     page_size=16, dtype="f16", sm_scale=w.sm_scale, num_pages=w.num_pages,
                     num_sms=148, ctas_per_sm=2)
    o_plain, l_plain = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    torch.cuda.synchronize()
    assert torch.equal(o_zero, o_plain) and torch.equal(l_zero, l_plain)
    assert (o_rope.float() - o_plain.float()).abs().max().item() > 0.05
