"""8-bit (FP8 E4M3 / E5M2) KV-cache decode on the GPU against the fp64 oracle.

README core feature 3: attention over a compressed KV-Cache.  The pools hold
8-bit codes with one scale for K and one for V; q and o stay fp16 / bf16.
Small cases span several tiles, ragged tails, empty requests, every GQA
group, page sizes 1 / 16 / 64, both q types and both formats, with
non-power-of-two scales, split and unsplit plans, on both decode kernels
(the tensor-core one widens K into TMEM and V into shared memory).  The
full-size uniform and ragged batches with E4M3 caches are checked on every
row.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu

EDGE_LENS = [0, 1, 15, 16, 17, 31, 32, 33, 100, 257, 1000]


def _oracle(w, t, threads=8):
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], w.kv_indptr, w.kv_indices,
                               w.last_page_len, num_qo_heads=w.num_qo_heads,
                               num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                               page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale,
                               kv_dtype=w.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale,
                               threads=threads)


def _decode(w, dev, **kw):
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                     num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                     sm_scale=w.sm_scale, num_pages=w.num_pages, kv_dtype=w.kv_dtype,
                     k_scale=w.k_scale, v_scale=w.v_scale, **kw)
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    torch.cuda.synchronize()
    assert pd.check() == -1
    return pd, o, lse


KERNELS = {"cuda_cores": 2, "tensor_cores": 4}  # PA_FLAG_CUDA_CORES / PA_FLAG_TENSOR_CORES


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("P", [1, 16, 64])
def test_fp8_small_parity(fmt, dtype, group, P, kernel):
    hkv = 2
    w = W.make_workload("fp8_small", EDGE_LENS, num_qo_heads=hkv * group, num_kv_heads=hkv,
                        page_size=P, dtype=dtype, seed=300 + group + P, extra_pages=3,
                        kv_dtype=fmt, k_scale=0.37, v_scale=1.3)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    from serving_attention_paged_b200 import pagedattn as C
    for kw in (dict(num_sms=10000, ctas_per_sm=1),
               dict(num_sms=3, ctas_per_sm=1, min_chunk_tokens=16)):
        pd, o, lse = _decode(w, dev, flags=KERNELS[kernel], **kw)
        assert C.pa_plan_uses_tensor_cores(pd.plan) == (kernel == "tensor_cores")
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype,
                     f"{kernel} {fmt} G={group} P={P} {kw}")


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("group", [4, 8])
def test_fp8_sharp_softmax(group, kernel):
    """Large score spread: the running maximum moves past the lazy slack."""
    w = W.make_workload("fp8_sharp", [2000, 700, 129, 5000, 1], num_qo_heads=2 * group,
                        num_kv_heads=2, page_size=16, dtype="bf16", seed=310 + group,
                        sm_scale=2.0, kv_dtype="e4m3", k_scale=0.5, v_scale=0.25)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o, lse = _decode(w, dev, num_sms=5, ctas_per_sm=1, min_chunk_tokens=300,
                         flags=KERNELS[kernel])
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16", f"fp8 sharp G={group} {kernel}")


def test_fp8_equals_16bit_cache_holding_the_same_values():
    """Every E4M3 value times a power-of-two scale is exact in fp16: a 16-bit
    cache holding those values must give the same result (to rounding)."""
    w8 = W.make_workload("fp8_same", [700, 33, 2000], num_qo_heads=16, num_kv_heads=2,
                         page_size=16, dtype="f16", seed=320, kv_dtype="e4m3", k_scale=0.25,
                         v_scale=0.5)
    t8 = w8.materialize()
    dev8 = {k: v.cuda() for k, v in t8.items()}
    _, o8, l8 = _decode(w8, dev8, num_sms=148, ctas_per_sm=2)
    k16 = (t8["k_pool"].to(torch.float32) * 0.25).to(torch.float16).cuda()
    v16 = (t8["v_pool"].to(torch.float32) * 0.5).to(torch.float16).cuda()
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w8.kv_indptr, w8.last_page_len, num_qo_heads=16, num_kv_heads=2,
                     page_size=16, dtype="f16", sm_scale=w8.sm_scale, num_pages=w8.num_pages,
                     num_sms=148, ctas_per_sm=2, flags=2)
    o16, l16 = pd.run(dev8["q"], k16, v16, dev8["kv_indices"])
    torch.cuda.synchronize()
    assert (o8.float() - o16.float()).abs().max().item() <= 2e-3
    assert (l8 - l16).abs().max().item() <= 1e-3


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_fp8_checked_indices_and_graph_replay(kernel):
    from serving_attention_paged_b200 import pagedattn as C
    w = W.make_workload("fp8_chk", [4000, 50, 9], num_qo_heads=32, num_kv_heads=8,
                        page_size=16, dtype="bf16", seed=330, kv_dtype="e5m2", k_scale=0.8,
                        v_scale=0.9)
    t = w.materialize()
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o_eager, l_eager = _decode(w, dev, num_sms=148, ctas_per_sm=2,
                                   flags=C.PA_FLAG_CHECK_INDICES | KERNELS[kernel])
    o_ref, l_ref = _oracle(w, t)
    assert_close(to_np(o_eager), to_np(l_eager), o_ref, l_ref, "bf16", "fp8 checked")
    bad = dev["kv_indices"].clone()
    bad[3] = w.num_pages + 1
    pd.run(dev["q"], dev["k_pool"], dev["v_pool"], bad)
    with pytest.raises(C.PagedAttnError) as e:
        pd.check()
    assert e.value.status == C.PA_ERR_DEVICE_CHECK and e.value.position == 3
    o = torch.zeros_like(o_eager)
    lse = torch.zeros_like(l_eager)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=s)
    for _ in range(2):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, l_eager)


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("n", ["2f8", "3f8"])
def test_fp8_full_size_every_row(n, kernel):
    w = W.WORKLOADS[n]()
    dev = w.materialize("cuda")
    pd, o, lse = _decode(w, dev, flags=KERNELS[kernel])
    indptr, indices, last = w.flat_tables()
    # 8-bit pools cross to the host as raw bytes
    o_ref, l_ref = oracle.paged_decode_requests(
        dev["q"], dev["k_pool"].view(torch.uint8), dev["v_pool"].view(torch.uint8), indptr,
        indices, last, list(range(w.batch)),
        num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
        page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale,
        threads=os.cpu_count() or 8, kv_dtype=w.kv_dtype, k_scale=w.k_scale,
        v_scale=w.v_scale)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, w.dtype, w.name)
    del dev
    torch.cuda.empty_cache()
