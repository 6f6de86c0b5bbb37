"""The C ABI on the host: exported symbols, plan parity with the oracle's
restatement (bit-exact), and argument validation.  No GPU needed: the plan
stage makes no CUDA call and run-stage argument checks happen before any."""
import os
import re

import numpy as np
import pytest

import oracle
from serving_attention_paged_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def C():
    from serving_attention_paged_b200 import build
    build.build()
    from serving_attention_paged_b200 import pagedattn
    return pagedattn


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(C):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(C.lib, n), n
    assert C.pa_abi_version() == 6


def _problem(C, w, num_sms=148, k=2, mct=0, flags=0):
    return C.make_problem(batch=w.batch, num_qo_heads=w.num_qo_heads,
                          num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                          sm_scale=w.sm_scale, num_sms=num_sms, ctas_per_sm=k,
                          min_chunk_tokens=mct, num_pages=w.num_pages, flags=flags)


def _compare_plan(C, indptr, last, P, hq, hkv, sms, k, mct, c=0):
    prob = C.make_problem(batch=len(last), num_qo_heads=hq, num_kv_heads=hkv, page_size=P,
                          dtype="f16", sm_scale=0.1, num_sms=sms, ctas_per_sm=k,
                          min_chunk_tokens=mct, num_pages=1 << 20,
                          piece_cost_tokens=c if c > 0 else -1)
    plan = C.pa_plan_create(prob, indptr, last)
    q, items, ci, mi = oracle.plan(indptr, last, page_size=P, num_kv_heads=hkv, num_sms=sms,
                                   ctas_per_sm=k, min_chunk_tokens=mct if mct else 256,
                                   piece_cost=c)
    assert C.pa_plan_quota_tokens(plan) == q
    assert np.array_equal(C.pa_plan_work_items(plan), items)
    assert np.array_equal(C.pa_plan_cta_indptr(plan), ci)
    assert np.array_equal(C.pa_plan_merge_indptr(plan, len(last) * hkv), mi)
    assert C.pa_plan_num_partials(plan) == mi[-1]
    return plan


@pytest.mark.parametrize("seed", range(25))
def test_plan_matches_oracle_bit_exact(C, seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(0, 70))
    P = int(rng.choice([1, 4, 16, 64]))
    lens = rng.integers(0, 5000, size=B) * (rng.random(B) > 0.15)
    indptr, _, last = W.tables_from_lengths(lens, P)
    hkv = int(rng.choice([1, 2, 4, 8]))
    g = int(rng.choice([1, 2, 4, 8]))
    _compare_plan(C, indptr, last, P, hkv * g, hkv, int(rng.integers(1, 300)),
                  int(rng.integers(1, 5)), int(rng.choice([0, 1, 100, 512])),
                  int(rng.choice([0, 1, 37, 160, 256, 1000])))


@pytest.mark.parametrize("c", [0, 160, 256])
@pytest.mark.parametrize("n", [1, 2, 3, 5, "4c"])
def test_plan_matches_oracle_on_benchmark_workloads(C, n, c):
    w = W.WORKLOADS[n]()
    _compare_plan(C, w.kv_indptr, w.last_page_len, w.page_size, w.num_qo_heads, w.num_kv_heads,
                  148, 3, 0, c)


def test_plan_matches_oracle_vector_sparse(C):
    w = W.WORKLOADS[4]()
    _compare_plan(C, w.kv_indptr, w.last_page_len, 1, 64, 8, 148, 1, 0, 256)


def test_plan_edge_cases(C):
    # empty batch, all-empty requests, one page, exactly full pages, B*Hkv above the budget
    for lens, P, sms in [([], 16, 148), ([0, 0], 16, 148), ([1], 16, 148), ([16, 32, 48], 16, 148),
                         ([100] * 50, 16, 2), ([3000, 1], 1, 1), ([0, 5000, 0], 16, 3)]:
        indptr, _, last = W.tables_from_lengths(lens, P)
        for c in (0, 160):
            _compare_plan(C, indptr, last, P, 8, 8, sms, 1, 0, c)


def test_plan_validation(C):
    w = W.make_workload("v", [20, 40], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=1)
    ok = _problem(C, w)
    C.pa_plan_create(ok, w.kv_indptr, w.last_page_len)

    def status(prob, indptr=w.kv_indptr, last=w.last_page_len):
        with pytest.raises(C.PagedAttnError) as e:
            C.pa_plan_create(prob, indptr, last)
        return e.value.status

    assert status(ok, indptr=np.array([1, 2, 4])) == C.PA_ERR_INVALID_ARG  # indptr[0] != 0
    assert status(ok, indptr=np.array([0, 3, 2])) == C.PA_ERR_INVALID_ARG  # decreasing
    assert status(ok, last=np.array([0, 8])) == C.PA_ERR_INVALID_ARG       # 0 with pages
    assert status(ok, last=np.array([17, 8])) == C.PA_ERR_INVALID_ARG      # > page_size
    bad = _problem(C, w); bad.num_qo_heads = 7
    assert status(bad) == C.PA_ERR_INVALID_ARG                             # Hq % Hkv
    bad = _problem(C, w); bad.head_dim = 64
    assert status(bad) == C.PA_ERR_UNSUPPORTED
    bad = _problem(C, w); bad.page_size = 12
    assert status(bad) == C.PA_ERR_UNSUPPORTED
    bad = _problem(C, w); bad.num_qo_heads = 32
    assert status(bad) == C.PA_ERR_UNSUPPORTED                             # group 16
    bad = _problem(C, w); bad.dtype = 7
    assert status(bad) == C.PA_ERR_INVALID_ARG
    bad = _problem(C, w); bad.num_sms = 0
    assert status(bad) == C.PA_ERR_INVALID_ARG
    bad = _problem(C, w); bad.num_pages = (1 << 32) // 16 + 1                # rows need 33 bits
    assert status(bad) == C.PA_ERR_UNSUPPORTED
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_cascade_plan_create(ok, 24, w.kv_indptr, w.last_page_len)  # not whole pages
    assert e.value.status == C.PA_ERR_INVALID_ARG
    small = _problem(C, w); small.page_size = 4                             # prefix boxes >= 8 rows
    indptr4, _, last4 = W.tables_from_lengths([20, 40], 4)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_cascade_plan_create(small, 16, indptr4, last4)
    assert e.value.status == C.PA_ERR_UNSUPPORTED


def test_run_argument_checks_before_any_launch(C):
    w = W.make_workload("v", [20, 40], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=1)
    plan = C.pa_plan_create(_problem(C, w), w.kv_indptr, w.last_page_len)
    nbytes = C.pa_plan_workspace_bytes(plan)
    assert nbytes % 256 == 0 and nbytes > 0
    fake = 1 << 40  # never dereferenced: every call below fails its host-side check
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run(plan, fake, fake, fake, fake, fake, None, fake, nbytes - 256, 0)
    assert e.value.status == C.PA_ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run(plan, None, fake, fake, fake, fake, None, fake, nbytes, 0)
    assert e.value.status == C.PA_ERR_INVALID_ARG
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run(plan, fake + 8, fake, fake, fake, fake, None, fake, nbytes, 0)  # misaligned q
    assert e.value.status == C.PA_ERR_INVALID_ARG
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_cascade_run(plan, fake, fake, fake, fake, fake, fake, None, fake, nbytes, 0)
    assert e.value.status == C.PA_ERR_INVALID_ARG  # not a cascade plan
    C.pa_merge_state(None, None, None, None, None, None, 0, 128, "f16", 0)  # nothing to do
    with pytest.raises(C.PagedAttnError):
        C.pa_merge_state(fake, fake, fake, fake, fake, fake, 4, 0, "f16", 0)


def test_cascade_plan_shape(C):
    w = W.WORKLOADS[5]()
    prob = _problem(C, w)
    plan = C.pa_cascade_plan_create(prob, w.prefix_len, w.kv_indptr, w.last_page_len)
    n, tok = C.pa_plan_prefix_chunks(plan)
    assert n >= 1 and tok % 128 == 0 and n * tok >= w.prefix_len > (n - 1) * tok
    q, items, ci, mi = oracle.plan(w.kv_indptr, w.last_page_len, page_size=16, num_kv_heads=8,
                                   num_sms=148, ctas_per_sm=2, piece_cost=300)
    assert np.array_equal(C.pa_plan_work_items(plan), items)
    assert np.array_equal(C.pa_plan_cta_indptr(plan), ci)


def test_decode_kernel_choice(C):
    """Default: tensor cores for GQA group 8, CUDA cores for 1, 2 and 4;
    PA_FLAG_CUDA_CORES / PA_FLAG_TENSOR_CORES override (CUDA cores win)."""
    w = W.make_workload("k", [20, 40], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=1)
    cases = [(1, 0, False), (2, 0, False), (4, 0, False), (8, 0, True),
             (4, C.PA_FLAG_TENSOR_CORES, True),
             (4, C.PA_FLAG_CUDA_CORES, False), (8, C.PA_FLAG_CUDA_CORES, False),
             (1, C.PA_FLAG_TENSOR_CORES, True), (2, C.PA_FLAG_TENSOR_CORES, True),
             (4, C.PA_FLAG_CUDA_CORES | C.PA_FLAG_TENSOR_CORES, False)]
    for group, flags, expect in cases:
        prob = C.make_problem(batch=w.batch, num_qo_heads=2 * group, num_kv_heads=2,
                              page_size=16, dtype="bf16", sm_scale=0.1, num_sms=148,
                              ctas_per_sm=1, num_pages=w.num_pages, flags=flags)
        plan = C.pa_plan_create(prob, w.kv_indptr, w.last_page_len)
        assert C.pa_plan_uses_tensor_cores(plan) is expect, (group, flags)


def test_default_piece_cost_follows_the_kernel(C):
    """piece_cost_tokens = 0 takes the default of the decode kernel the plan
    runs: 300 tokens for the CUDA-core kernel, 128 for the tensor-core one."""
    w = W.WORKLOADS[3]()
    for flags, c in ((0, 300), (C.PA_FLAG_TENSOR_CORES, 128)):
        base = dict(batch=w.batch, num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads,
                    page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, num_sms=148,
                    ctas_per_sm=2, num_pages=w.num_pages, flags=flags)
        default = C.pa_plan_create(C.make_problem(**base), w.kv_indptr, w.last_page_len)
        explicit = C.pa_plan_create(C.make_problem(piece_cost_tokens=c, **base), w.kv_indptr,
                                    w.last_page_len)
        assert np.array_equal(C.pa_plan_work_items(default), C.pa_plan_work_items(explicit))
        assert C.pa_plan_quota_tokens(default) == C.pa_plan_quota_tokens(explicit)


def test_plan_hand_worked_examples_library(C):
    """The library's work list against the hand-worked fixtures directly (not
    only through the oracle's restatement)."""
    import json
    path = os.path.join(ROOT, "tests", "golden", "plan_small.json")
    for g in json.load(open(path))["cases"]:
        hkv = g["num_kv_heads"]
        B = len(g["last_page_len"])
        prob = C.make_problem(batch=B, num_qo_heads=hkv, num_kv_heads=hkv,
                              page_size=g["page_size"], dtype="f16", sm_scale=0.1,
                              num_sms=g["num_sms"], ctas_per_sm=g["ctas_per_sm"],
                              min_chunk_tokens=g["min_chunk_tokens"], num_pages=1 << 20,
                              piece_cost_tokens=g.get("piece_cost_tokens", 0) or -1)
        plan = C.pa_plan_create(prob, np.array(g["kv_indptr"]), np.array(g["last_page_len"]))
        assert C.pa_plan_quota_tokens(plan) == g["quota"]
        assert C.pa_plan_work_items(plan).tolist() == g["items"]
        assert C.pa_plan_cta_indptr(plan).tolist() == g["cta_indptr"]
        assert C.pa_plan_merge_indptr(plan, B * hkv).tolist() == g["merge_indptr"]


def test_status_offset_lies_inside_the_workspace(C):
    for lens in ([], [5, 0, 3000], [100] * 40):
        indptr, _, last = W.tables_from_lengths(lens, 16)
        prob = C.make_problem(batch=len(lens), num_qo_heads=32, num_kv_heads=8, page_size=16,
                              dtype="bf16", sm_scale=0.1, num_sms=148, ctas_per_sm=1,
                              num_pages=1 << 16)
        plan = C.pa_plan_create(prob, indptr, last)
        off = C.pa_plan_status_offset(plan)
        assert off % 8 == 0 and off + 16 <= C.pa_plan_workspace_bytes(plan)


def test_kv8_and_rope_validation(C):
    """8-bit caches and rotary positions: bad scales, bad types and unbuilt
    combinations are refused before anything runs."""
    w = W.make_workload("v8", [20, 40], num_qo_heads=16, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=1)
    qo = np.array([0, 4, 6], np.int32)

    def prob(**kw):
        base = dict(batch=w.batch, num_qo_heads=16, num_kv_heads=2, page_size=16, dtype="f16",
                    sm_scale=0.1, num_sms=148, ctas_per_sm=2, num_pages=w.num_pages)
        base.update(kw)
        return C.make_problem(**base)

    def status(make):
        with pytest.raises(C.PagedAttnError) as e:
            make()
        return e.value.status

    def plan(p):
        return lambda: C.pa_plan_create(p, w.kv_indptr, w.last_page_len)

    ok8 = prob(kv_dtype="e4m3", k_scale=0.5, v_scale=2.0)
    p8 = C.pa_plan_create(ok8, w.kv_indptr, w.last_page_len)
    assert C.pa_plan_uses_tensor_cores(p8) is True  # 8-bit caches default to tensor cores
    p8c = C.pa_plan_create(prob(kv_dtype="e4m3", flags=C.PA_FLAG_CUDA_CORES), w.kv_indptr,
                           w.last_page_len)
    assert C.pa_plan_uses_tensor_cores(p8c) is False
    C.pa_plan_create(prob(kv_dtype="e5m2", k_scale=1.0, v_scale=1.0), w.kv_indptr,
                     w.last_page_len)
    okr = prob(rope_theta=1e4)
    assert C.pa_plan_uses_tensor_cores(C.pa_plan_create(okr, w.kv_indptr, w.last_page_len)) is False
    C.pa_plan_create(prob(kv_dtype="e4m3", rope_theta=5e5), w.kv_indptr, w.last_page_len)
    for bad in (dict(kv_dtype="e4m3", k_scale=0.0), dict(kv_dtype="e4m3", v_scale=-1.0),
                dict(kv_dtype="e5m2", k_scale=float("nan")), dict(kv_dtype="e4m3",
                                                                  v_scale=float("inf")),
                dict(kv_dtype="f32"), dict(rope_theta=-1.0), dict(rope_theta=float("nan"))):
        assert status(plan(prob(**bad))) == C.PA_ERR_INVALID_ARG, bad
    # not built: rotary positions on tensor cores, the cascade prefix level and
    # prefill with either
    C.pa_plan_create(prob(kv_dtype="e4m3", flags=C.PA_FLAG_TENSOR_CORES), w.kv_indptr,
                     w.last_page_len)
    assert status(plan(prob(rope_theta=1e4, flags=C.PA_FLAG_TENSOR_CORES))) == \
        C.PA_ERR_UNSUPPORTED
    C.pa_plan_create(prob(kv_dtype="e4m3", flags=C.PA_FLAG_TENSOR_CORES | C.PA_FLAG_CUDA_CORES),
                     w.kv_indptr, w.last_page_len)
    for kw in (dict(kv_dtype="e4m3"), dict(rope_theta=1e4)):
        assert status(lambda: C.pa_cascade_plan_create(prob(**kw), 32, w.kv_indptr,
                                                       w.last_page_len)) == C.PA_ERR_UNSUPPORTED
        assert status(lambda: C.pa_prefill_plan_create(prob(**kw), True, qo, w.kv_indptr,
                                                       w.last_page_len)) == C.PA_ERR_UNSUPPORTED
    # a cascade without a prefix is a plain decode: allowed
    C.pa_cascade_plan_create(prob(kv_dtype="e4m3"), 0, w.kv_indptr, w.last_page_len)
    # rotary positions are exact fp32 integers: requests beyond 2^24 tokens are refused
    indptr = np.array([0, (1 << 24) // 16 + 1], np.int32)
    big = C.make_problem(batch=1, num_qo_heads=16, num_kv_heads=2, page_size=16, dtype="f16",
                         sm_scale=0.1, num_sms=148, ctas_per_sm=2, num_pages=1 << 21,
                         rope_theta=1e4)
    assert status(lambda: C.pa_plan_create(big, indptr, np.array([1], np.int32))) == \
        C.PA_ERR_UNSUPPORTED
    big.rope_theta = 0.0
    C.pa_plan_create(big, indptr, np.array([1], np.int32))


def test_rope_plans_upload_each_request_length(C):
    """Rotary plans carry each request's length in the workspace (the query's
    position); others do not grow."""
    w = W.make_workload("rl", [20, 0, 40, 1000], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=1)
    args = dict(batch=w.batch, num_qo_heads=8, num_kv_heads=2, page_size=16, dtype="f16",
                sm_scale=0.1, num_sms=4, ctas_per_sm=1, num_pages=w.num_pages)
    plain = C.pa_plan_create(C.make_problem(**args), w.kv_indptr, w.last_page_len)
    rope = C.pa_plan_create(C.make_problem(rope_theta=1e4, **args), w.kv_indptr,
                            w.last_page_len)
    assert C.pa_plan_workspace_bytes(rope) >= C.pa_plan_workspace_bytes(plain)
    assert np.array_equal(C.pa_plan_work_items(rope), C.pa_plan_work_items(plain))
