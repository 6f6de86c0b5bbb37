"""Paged decode on the GPU against the fp64 oracle (element by element).

Small cases span several 32-token (CUDA-core) and 128-token (tensor-core)
tiles, ragged tails, empty requests, every supported GQA group, page sizes
1 / 16 / 64, both dtypes, forced split-KV and both decode kernels.  Full-size benchmark workloads run in the bench's launch
configuration and are checked on every row.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, oracle_full, oracle_sampled, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu

EDGE_LENS = [0, 1, 15, 16, 17, 31, 32, 33, 100, 257, 1000]


def _decode(w, dev, **kw):
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                     num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                     sm_scale=w.sm_scale, num_pages=w.num_pages, prefix_len=w.prefix_len, **kw)
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"],
                    prefix_indices=dev.get("prefix_indices"))
    torch.cuda.synchronize()
    assert pd.check() == -1  # no bounded wait gave up
    return pd, o, lse


KERNELS = {"auto": 0, "cuda_cores": 2, "tensor_cores": 4}  # PA_FLAG_CUDA_CORES / _TENSOR_CORES


def _to_dev(t):
    return {k: v.cuda() for k, v in t.items()}


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("P", [1, 16, 64])
def test_small_parity(dtype, group, P, kernel):
    hkv = 2
    w = W.make_workload("small", EDGE_LENS, num_qo_heads=hkv * group, num_kv_heads=hkv,
                        page_size=P, dtype=dtype, seed=40 + group + P, extra_pages=3)
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = _to_dev(t)
    # no split (large budget) and forced split (tiny budget, 16-token chunks)
    for kw in (dict(num_sms=10000, ctas_per_sm=1),
               dict(num_sms=3, ctas_per_sm=1, min_chunk_tokens=16)):
        pd, o, lse = _decode(w, dev, flags=KERNELS[kernel], **kw)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype,
                     f"G={group} P={P} {kernel} {kw}")


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [4, 8])
@pytest.mark.parametrize("sm_scale", [1.0, 3.0])
def test_sharp_softmax_moves_the_running_max(dtype, group, sm_scale, kernel):
    """Scores spread over tens of units in log2: the running maximum of a long
    piece moves many times past the lazy-rescale slack, so the rescale of the
    accumulated output (TMEM on the tensor-core path) runs."""
    w = W.make_workload("sharp", [2000, 700, 129, 5000, 1], num_qo_heads=2 * group,
                        num_kv_heads=2, page_size=16, dtype=dtype, seed=90 + group,
                        sm_scale=sm_scale)
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = _to_dev(t)
    for kw in (dict(num_sms=10000, ctas_per_sm=1),
               dict(num_sms=5, ctas_per_sm=1, min_chunk_tokens=300)):
        pd, o, lse = _decode(w, dev, flags=KERNELS[kernel], **kw)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype,
                     f"sharp G={group} scale={sm_scale} {kernel} {kw}")


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("cost", [-1, 1, 1000])
def test_piece_cost_plans(kernel, cost):
    """Plans with no piece cost, a tiny one and a huge one (many short
    pieces, many split segments) give the same attention."""
    w = W.make_workload("cost", [0, 3, 700, 5000, 1, 129, 2000], num_qo_heads=16,
                        num_kv_heads=2, page_size=16, dtype="bf16", seed=120)
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = _to_dev(t)
    pd, o, lse = _decode(w, dev, num_sms=7, ctas_per_sm=1, min_chunk_tokens=32,
                         flags=KERNELS[kernel], piece_cost_tokens=cost)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16", f"{kernel} cost={cost}")


@pytest.mark.parametrize("group", [4, 8])
def test_tensor_core_and_cuda_core_kernels_agree(group):
    """The two decode kernels on the same plan shape agree to rounding."""
    w = W.make_workload("agree", [4096, 3000, 17, 0, 1200], num_qo_heads=4 * group,
                        num_kv_heads=4, page_size=16, dtype="bf16", seed=95 + group)
    dev = _to_dev(w.materialize())
    _, o_tc, l_tc = _decode(w, dev, num_sms=148, ctas_per_sm=1, flags=KERNELS["tensor_cores"])
    _, o_cc, l_cc = _decode(w, dev, num_sms=148, ctas_per_sm=1, flags=KERNELS["cuda_cores"])
    assert (o_tc.float() - o_cc.float()).abs().max().item() <= 2 * 2e-3
    fin = torch.isfinite(l_cc)
    assert torch.equal(fin, torch.isfinite(l_tc))
    assert (l_tc[fin] - l_cc[fin]).abs().max().item() <= 2e-3


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_split_chunks_are_exercised(kernel):
    w = W.make_workload("split", [5000, 3, 700], num_qo_heads=32, num_kv_heads=8, page_size=16,
                        dtype="bf16", seed=5)
    t = w.materialize()
    o_ref, l_ref = oracle_full(w, t)
    dev = _to_dev(t)
    pd, o, lse = _decode(w, dev, num_sms=148, ctas_per_sm=2, flags=KERNELS[kernel])
    items = pd.work_items()
    assert (items[:, 5] >= 0).any()  # some requests really were split
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16", "split")
    # a second run reuses the self-reset arrival counters
    o2, lse2 = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_empty_batch_and_all_empty():
    for lens in ([], [0, 0, 0]):
        w = W.make_workload("empty", lens, num_qo_heads=8, num_kv_heads=2, page_size=16,
                            dtype="f16", seed=6, extra_pages=1)
        t = w.materialize()
        dev = _to_dev(t)
        pd, o, lse = _decode(w, dev)
        if lens:
            assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_single_token_gives_v():
    w = W.make_workload("one", [1] * 5, num_qo_heads=16, num_kv_heads=2, page_size=16,
                        dtype="bf16", seed=7, extra_pages=4)
    t = w.materialize()
    dev = _to_dev(t)
    pd, o, lse = _decode(w, dev)
    rows = torch.from_numpy(w.token_rows())
    v = t["v_pool"].view(-1, 2, 128)[rows]  # [5, Hkv, D]
    expect = v.repeat_interleave(8, dim=1)
    assert torch.equal(o.cpu(), expect)


def test_page_permutation_invariance_gpu():
    lens = [300, 77, 1024]
    ws = [W.make_workload("perm", lens, num_qo_heads=32, num_kv_heads=8, page_size=16,
                          dtype="f16", seed=8, shuffle=s) for s in (True, False)]
    outs = [_decode(w, _to_dev(w.materialize()), num_sms=148, ctas_per_sm=2)[1:] for w in ws]
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_cuda_graph_replay(kernel):
    w = W.make_workload("graph", [4000, 50, 2000, 9], num_qo_heads=32, num_kv_heads=8,
                        page_size=16, dtype="f16", seed=9)
    t = w.materialize()
    dev = _to_dev(t)
    pd, o_eager, l_eager = _decode(w, dev, num_sms=148, ctas_per_sm=2, flags=KERNELS[kernel])
    o = torch.zeros_like(o_eager)
    lse = torch.zeros_like(l_eager)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=s)
    for _ in range(3):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, l_eager)


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_bounds_checked_run_reports_bad_index(kernel):
    from serving_attention_paged_b200 import pagedattn as C
    w = W.make_workload("chk", [40, 40], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=10)
    t = w.materialize()
    dev = _to_dev(t)
    bad = dev["kv_indices"].clone()
    bad[4] = w.num_pages + 7  # out of range: the checked kernel skips it and records it
    from serving_attention_paged_b200.wrapper import PagedDecode
    pd = PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=8, num_kv_heads=2,
                     page_size=16, dtype="f16", sm_scale=w.sm_scale, num_pages=w.num_pages,
                     flags=C.PA_FLAG_CHECK_INDICES | KERNELS[kernel])
    pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    assert pd.check() == -1
    pd.run(dev["q"], dev["k_pool"], dev["v_pool"], bad)
    with pytest.raises(C.PagedAttnError) as e:
        pd.check()
    assert e.value.status == C.PA_ERR_DEVICE_CHECK and e.value.position == 4
    assert pd.check() == -1  # the word was cleared
    # request 0 (untouched pages) still matches the oracle
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], bad)
    o_ref, l_ref = oracle_full(w, t)
    assert_close(to_np(o)[:1], to_np(lse)[:1], o_ref[:1], l_ref[:1], "f16", "checked")
    with pytest.raises(C.PagedAttnError):
        pd.check()


@pytest.mark.parametrize("kind", ["decode", "cascade", "prefill"])
def test_timeout_word_is_reported_and_cleared(kind):
    """The reporting half of the bounded waits: a nonzero timeout word in the
    workspace (written here by a plain host-to-device copy, no kernel) makes
    pa_plan_check return PA_ERR_DEVICE_TIMEOUT, and the check clears it."""
    from serving_attention_paged_b200 import pagedattn as C
    from serving_attention_paged_b200.wrapper import PagedDecode, PagedPrefill
    w = W.make_workload("tmo", [40, 300], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=11, prefix_len=64 if kind == "cascade" else 0)
    common = dict(num_qo_heads=8, num_kv_heads=2, page_size=16, dtype="f16",
                  sm_scale=w.sm_scale, num_pages=w.num_pages)
    if kind == "prefill":
        pd = PagedPrefill(np.array([0, 8, 20], np.int32), w.kv_indptr, w.last_page_len,
                          **common)
    else:
        pd = PagedDecode(w.kv_indptr, w.last_page_len, prefix_len=w.prefix_len, **common)
    off = C.pa_plan_status_offset(pd.plan)
    assert pd.check() == -1
    word = torch.tensor([1, 0, 0, 0, 0, 0, 0, 0], dtype=torch.uint8)
    pd.workspace[off + 8:off + 16].copy_(word)
    torch.cuda.synchronize()
    with pytest.raises(C.PagedAttnError) as e:
        pd.check()
    assert e.value.status == C.PA_ERR_DEVICE_TIMEOUT
    assert pd.check() == -1  # cleared
    assert torch.all(pd.workspace[off + 8:off + 16] == 0)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_merge_state_parity(dtype):
    from serving_attention_paged_b200 import pagedattn as C
    rng = np.random.default_rng(3)
    rows, D = 300, 128
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[dtype]
    oa = torch.from_numpy(rng.standard_normal((rows, D))).to(tdt)
    ob = torch.from_numpy(rng.standard_normal((rows, D))).to(tdt)
    la = torch.from_numpy(rng.standard_normal(rows) * 5).float()
    lb = torch.from_numpy(rng.standard_normal(rows) * 5).float()
    la[:10] = -np.inf
    lb[5:15] = -np.inf
    o_ref, l_ref = oracle.merge_state(to_np(oa), to_np(la), to_np(ob), to_np(lb))
    o = torch.empty_like(oa).cuda()
    lse = torch.empty_like(la).cuda()
    ga, gb, gla, glb = oa.cuda(), ob.cuda(), la.cuda(), lb.cuda()
    C.pa_merge_state(ga, gla, gb, glb, o, lse, rows, D, dtype)
    torch.cuda.synchronize()
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, "bf16" if dtype == "bf16" else "f16",
                 "merge")
    # in place: outputs alias the first input
    C.pa_merge_state(ga, gla, gb, glb, ga, gla, rows, D, dtype)
    torch.cuda.synchronize()
    assert torch.equal(ga, o) and torch.equal(gla, lse)


# --------------------------------------------------------------------------
# full-size workloads, launch configuration of the benchmark, every row
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 2, 3, 4, "4c"])
def test_full_size_every_row(n):
    """Every (request, q head) row of the full-size workload, element by
    element against the oracle (run on all host cores over the pages each
    request reads: about 0.5 GB/s of K/V, so workload 4 takes ~10 s)."""
    w = W.WORKLOADS[n]()
    dev = w.materialize("cuda")
    pd, o, lse = _decode(w, dev)
    reqs = list(range(w.batch))
    o_ref, l_ref = oracle_sampled(w, dev, reqs, threads=os.cpu_count() or 8)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, w.dtype, w.name)
    del dev
    torch.cuda.empty_cache()


def test_vector_sparse_equals_contiguous_twin():
    """page_size 1 scattered and page_size 16 contiguous hold the same logical
    tokens: the two runs must agree to rounding."""
    a, b = W.WORKLOADS[4](), W.WORKLOADS["4c"]()
    da = a.materialize("cuda")
    _, oa, la = _decode(a, da)
    del da
    db = b.materialize("cuda")
    _, ob, lb = _decode(b, db)
    del db
    assert (oa.float() - ob.float()).abs().max().item() <= 2 * 2e-3
    assert (la - lb).abs().max().item() <= 1e-3
    torch.cuda.empty_cache()
