"""Prefill / append attention on the GPU against the fp64 oracle.

The oracle evaluates every new query token as plain attention over its
request's keys up to its limit; the GPU side runs the tensor-core prefill
kernel through the C ABI.  Cases cover every GQA group, both dtypes, the
causal rule and attention without the mask, page sizes 8 to 256, requests
with no new tokens, fresh prefills (Q_b = L_b), single-token appends, ragged
query tiles and 64-key tiles, stale NaN rows in partly used pages, few
persistent CTAs running long item lists, the index bounds check, graph
replay, and the full-size prefill workload on sampled query tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _oracle(w, t, causal=True, queries=None):
    return oracle.paged_prefill(t["q"], t["k_pool"], t["v_pool"], w.qo_indptr, w.kv_indptr,
                                w.kv_indices, w.last_page_len, num_qo_heads=w.num_qo_heads,
                                num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                                page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale,
                                causal=causal, queries=queries, threads=8)


def _prefill(w, causal=True, flags=0, num_sms=None):
    from serving_attention_paged_b200.wrapper import PagedPrefill
    return PagedPrefill(w.qo_indptr, w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                        num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                        sm_scale=w.sm_scale, num_pages=w.num_pages, causal=causal, flags=flags,
                        num_sms=num_sms)


def _run(w, dev, causal=True, flags=0, num_sms=None):
    pf = _prefill(w, causal, flags, num_sms)
    o, lse = pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])
    torch.cuda.synchronize()
    return pf, o, lse


def _check(w, dev, o_ref, l_ref, causal, what):
    pf, o, lse = _run(w, dev, causal)
    assert pf.check() == -1  # no bounded wait gave up, no bad index
    return assert_close(to_np(o), to_np(lse), o_ref, l_ref, w.dtype, what)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_prefill_small(dtype, group):
    """Fresh prefill, append, single-token append and an idle request; keys
    span several 64-key tiles with ragged ends; query tiles of 256 / G tokens
    (two halves of 128 / G) with ragged last ones, some without a second half."""
    hkv = 2
    kv = [200, 77, 1, 150, 64]
    qo = [200, 40, 1, 0, 33]
    w = W.make_workload("pf", kv, num_qo_heads=hkv * group, num_kv_heads=hkv, page_size=16,
                        dtype=dtype, seed=100 + group, qo_lens=qo)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    _check(w, dev, o_ref, l_ref, True, f"G={group} {dtype}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_without_mask(dtype):
    """No causal mask: every token sees all its request's keys; more tokens
    than keys, and a request without keys (o = 0, lse = -inf)."""
    w = W.make_workload("pf_nomask", [130, 0, 9, 300], num_qo_heads=8, num_kv_heads=2,
                        page_size=16, dtype=dtype, seed=110, qo_lens=[50, 3, 20, 1])
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t, causal=False)
    dev = {k: v.cuda() for k, v in t.items()}
    _check(w, dev, o_ref, l_ref, False, f"no mask {dtype}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("num_sms", [1, 3, 7])
def test_prefill_persistent_ctas_run_many_items(dtype, causal, num_sms):
    """Few persistent CTAs, so each runs a long list of items back to back:
    items with one or two halves, halves of different tile counts, items
    without keys and without tokens, across which the CTA carries its
    barriers, rings and TMEM.  Results equal the oracle's, and bit for bit
    those of one CTA per SM (every item's arithmetic is the same)."""
    kv = [200, 0, 77, 1, 150, 64, 300] if not causal else [200, 77, 1, 150, 64, 300]
    qo = [200, 3, 40, 1, 0, 33, 129] if not causal else [200, 40, 1, 0, 33, 129]
    w = W.make_workload("pf_persist", kv, num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype=dtype, seed=170 + num_sms, qo_lens=qo)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t, causal=causal)
    dev = {k: v.cuda() for k, v in t.items()}
    pf, o, lse = _run(w, dev, causal, num_sms=num_sms)
    assert pf.check() == -1
    assert len(pf.cta_indptr()) - 1 == min(num_sms, len(pf.tiles()) * w.num_kv_heads)
    assert_close(to_np(o), to_np(lse), o_ref, l_ref, dtype, f"{num_sms} CTAs {dtype}")
    _, o_all, lse_all = _run(w, dev, causal)
    assert torch.equal(o, o_all) and torch.equal(lse, lse_all)


@pytest.mark.parametrize("P", [8, 32, 64, 256])
def test_prefill_page_sizes(P):
    w = W.make_workload("pf_p", [333, 70, 129], num_qo_heads=8, num_kv_heads=2, page_size=P,
                        dtype="f16", seed=120 + P, qo_lens=[100, 70, 5])
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    _check(w, dev, o_ref, l_ref, True, f"P={P}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_stale_rows_of_partly_used_pages_do_not_leak(dtype):
    """Rows of a request's last page past its last key may hold anything: fill
    them (and every unused pool row) with NaN; the result must not change."""
    w = W.make_workload("pf_nan", [70, 45, 130], num_qo_heads=8, num_kv_heads=2, page_size=64,
                        dtype=dtype, seed=130, qo_lens=[70, 10, 3], extra_pages=2)
    t = w.materialize()
    o_ref, l_ref = _oracle(w, t)
    dev = {k: v.cuda() for k, v in t.items()}
    used = torch.zeros(w.num_pages * w.page_size, dtype=torch.bool)
    used[torch.from_numpy(w.token_rows())] = True
    for name in ("k_pool", "v_pool"):
        flat = dev[name].view(w.num_pages * w.page_size, -1)
        flat[(~used).cuda()] = float("nan")
    _check(w, dev, o_ref, l_ref, True, f"NaN stale rows {dtype}")


def test_prefill_many_tiles_per_request():
    """One long fresh prefill (1000 tokens, 16 tiles at G = 4) next to short
    appends: tiles of very different lengths in one launch."""
    w = W.make_workload("pf_long", [1000, 300, 2000], num_qo_heads=32, num_kv_heads=8,
                        page_size=16, dtype="bf16", seed=140, qo_lens=[1000, 17, 130])
    t = w.materialize()
    sample = np.r_[0:40, 960:1017, 1017:1147:7]
    o_ref, l_ref = _oracle(w, t, queries=sample)
    dev = {k: v.cuda() for k, v in t.items()}
    pf, o, lse = _run(w, dev)
    assert pf.check() == -1
    assert_close(to_np(o[sample]), to_np(lse[sample]), o_ref, l_ref, "bf16", "long prefill")


def test_prefill_index_check_reports_bad_page():
    from serving_attention_paged_b200 import pagedattn as C
    w = W.make_workload("pf_bad", [100, 60], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=150, qo_lens=[20, 60])
    t = w.materialize()
    bad = t["kv_indices"].clone()
    bad[5] = w.num_pages + 3  # request 0, tokens 80..95
    dev = {k: v.cuda() for k, v in t.items()}
    pf = _prefill(w, True, C.PA_FLAG_CHECK_INDICES)
    o, lse = pf.run(dev["q"], dev["k_pool"], dev["v_pool"], bad.cuda())
    torch.cuda.synchronize()
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_plan_check(pf.plan, pf.workspace)
    assert e.value.status == C.PA_ERR_DEVICE_CHECK and e.value.position == 5
    assert torch.isfinite(o.float()).all()
    # a clean run afterwards reports nothing
    pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse)
    torch.cuda.synchronize()
    assert pf.check() == -1


def test_prefill_graph_replay():
    """The run only enqueues work: captured once, replayed on new inputs."""
    w = W.make_workload("pf_graph", [300, 128], num_qo_heads=32, num_kv_heads=8, page_size=16,
                        dtype="f16", seed=160, qo_lens=[120, 128])
    t = w.materialize()
    dev = {k: v.cuda() for k, v in t.items()}
    pf = _prefill(w)
    o = torch.empty_like(dev["q"])
    lse = torch.empty(w.query_rows(), w.num_qo_heads, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=s)
    for scale in (1.0, -0.5):
        q2 = (t["q"].float() * scale).to(t["q"].dtype)
        dev["q"].copy_(q2.cuda())
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        t2 = dict(t, q=q2)
        o_ref, l_ref = _oracle(w, t2)
        assert_close(to_np(o), to_np(lse), o_ref, l_ref, "f16", f"replay {scale}")


def test_prefill_workload_full_size_sampled():
    """The prefill workload at full size (8 requests x 2048 keys, 1024 new
    tokens each, GQA 32/8, P 16, fp16) in the launch the bench times;
    sampled query tokens of every request against the oracle."""
    w = W.WORKLOADS[6]()
    dev = w.materialize("cuda")
    pf, o, lse = _run(w, dev)
    assert pf.check() == -1
    rng = np.random.default_rng(6)
    qo = w.qo_indptr
    sample = np.unique(np.concatenate(
        [qo[b] + np.r_[0, 31, 32, 1023, rng.integers(0, 1024, 4)] for b in range(w.batch)]))
    o_ref, l_ref = _oracle(w, dev, queries=sample)
    assert_close(to_np(o[sample]), to_np(lse[sample]), o_ref, l_ref, "f16", "prefill workload")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
