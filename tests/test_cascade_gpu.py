"""Cascade decode on the GPU against the fp64 oracle.

The oracle side is plain attention over each request's full token list
(shared prefix pages followed by its own pages); the GPU side runs the
tensor-core prefix level and the paged suffix level and merges them.
Cases cover several 128-key tiles with a ragged last tile, several
128-row query tiles, every GQA group, both dtypes, empty suffixes, a
prefix split over chunks, and the full-size shared-prefix workload.
"""
import os

import numpy as np
import pytest
import torch

from parity import assert_close, oracle_full, oracle_sampled, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(w, dev, **kw):
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                     num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                     sm_scale=w.sm_scale, num_pages=w.num_pages, prefix_len=w.prefix_len, **kw)
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"],
                    prefix_indices=dev["prefix_indices"])
    torch.cuda.synchronize()
    assert pd.check() == -1  # no bounded wait gave up
    return pd, o, lse


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_cascade_small(dtype, group):
    hkv = 2
    lens = [0, 5, 16, 100, 37]
    w = W.make_workload("casc", lens, num_qo_heads=hkv * group, num_kv_heads=hkv, page_size=16,
                        dtype=dtype, seed=60 + group, prefix_len=16 * 19)  # 304 keys: 3 tiles
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    for kw in (dict(num_sms=148, ctas_per_sm=2), dict(num_sms=1, ctas_per_sm=1)):
        pd, o, lse = _run(w, dev, **kw)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype, f"G={group} {kw}")


@pytest.mark.parametrize("P", [8, 32, 256])
def test_cascade_page_sizes(P):
    w = W.make_workload("casc_p", [3, 70, 0], num_qo_heads=8, num_kv_heads=2, page_size=P,
                        dtype="f16", seed=70 + P, prefix_len=P * (1024 // P if P < 1024 else 1))
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o, lse = _run(w, dev)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "f16", f"P={P}")


def test_cascade_many_query_tiles():
    """B * G = 300 query rows per kv head: three 128-row tiles, the last ragged."""
    lens = list(np.random.default_rng(1).integers(0, 60, size=75))
    w = W.make_workload("casc_rows", lens, num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="bf16", seed=81, prefix_len=512)
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o, lse = _run(w, dev)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16", "rows")


def test_cascade_equals_flat_decode():
    """The cascade result equals a plain paged decode over prefix ++ suffix pages."""
    w = W.make_workload("casc_flat", [40, 1, 300], num_qo_heads=32, num_kv_heads=8,
                        page_size=16, dtype="f16", seed=82, prefix_len=2048)
    t = w.materialize()
    dev = {k: v.cuda() for k, v in t.items()}
    _, oc, lc = _run(w, dev)
    indptr, indices, last = w.flat_tables()
    flat = W.PagedWorkload(name="flat", batch=w.batch, num_qo_heads=32, num_kv_heads=8,
                           head_dim=128, page_size=16, dtype="f16", seed=82,
                           num_pages=w.num_pages, kv_indptr=indptr, kv_indices=indices,
                           last_page_len=last)
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(flat.kv_indptr, flat.last_page_len, num_qo_heads=32, num_kv_heads=8,
                     page_size=16, dtype="f16", sm_scale=w.sm_scale, num_pages=w.num_pages)
    of, lf = pd.run(dev["q"], dev["k_pool"], dev["v_pool"],
                    torch.from_numpy(indices).cuda())
    torch.cuda.synchronize()
    assert (oc.float() - of.float()).abs().max().item() <= 2 * 2e-3
    assert (lc - lf).abs().max().item() <= 2e-3


def test_cascade_graph_replay():
    w = W.make_workload("casc_graph", [64, 700, 3], num_qo_heads=32, num_kv_heads=8,
                        page_size=16, dtype="f16", seed=83, prefix_len=1024)
    t = w.materialize()
    dev = {k: v.cuda() for k, v in t.items()}
    pd, o_eager, l_eager = _run(w, dev)
    o = torch.zeros_like(o_eager)
    lse = torch.zeros_like(l_eager)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse,
                   prefix_indices=dev["prefix_indices"], stream=s)
    for _ in range(3):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, l_eager)


def test_cascade_full_size_every_row():
    """Every row of the full-size shared-prefix workload against the oracle
    over each request's whole token list (prefix ++ suffix)."""
    w = W.WORKLOADS[5]()
    dev = w.materialize("cuda")
    pd, o, lse = _run(w, dev)
    o_ref, l_ref = oracle_sampled(w, dev, list(range(w.batch)), threads=os.cpu_count() or 8)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, w.dtype, w.name)
    del dev
    torch.cuda.empty_cache()
