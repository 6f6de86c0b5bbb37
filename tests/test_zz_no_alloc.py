"""pa_run_static_workspace: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: their memory pool already
owns all free GPU memory, or they do not control the process's allocator,
or they must avoid cudaMalloc's implicit synchronisation.  This entry point
runs the same kernel with a workspace compiled into the library (8 MiB per
GPU).  The test compares it with pa_run (caller workspace) on two calls in a
row, within the parity tolerance, and checks that a plan too large for the
fixed array is refused before anything runs.  It lives in its own file,
collected last, and passes alone in a fresh process as well.
"""
import pytest
import torch

from parity import assert_close, to_np
from serving_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _problem(C, w, num_sms=148, ctas_per_sm=3, flags=0):
    return C.make_problem(batch=w.batch, num_qo_heads=w.num_qo_heads,
                          num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                          sm_scale=w.sm_scale, num_sms=num_sms, ctas_per_sm=ctas_per_sm,
                          num_pages=w.num_pages, flags=flags)


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_static_workspace_matches_caller_workspace_twice(kernel):
    from serving_attention_paged_b200 import pagedattn as C
    lens = [3000, 0, 17, 900, 4096, 1]
    w = W.make_workload("static_ws", lens, num_qo_heads=32, num_kv_heads=8, page_size=16,
                        dtype="bf16", seed=91)
    dev = {k: v.cuda() for k, v in w.materialize().items()}
    flags = C.PA_FLAG_TENSOR_CORES if kernel == "tensor_cores" else C.PA_FLAG_CUDA_CORES
    plan = C.pa_plan_create(_problem(C, w, ctas_per_sm=1 if kernel == "tensor_cores" else 3,
                                     flags=flags), w.kv_indptr, w.last_page_len)
    assert C.pa_plan_uses_tensor_cores(plan) == (kernel == "tensor_cores")
    assert C.pa_plan_num_partials(plan) > 0  # the split path (partials, counters) is exercised
    nbytes = C.pa_plan_workspace_bytes(plan)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    C.pa_plan_upload(plan, ws, nbytes)
    o_ref = torch.empty_like(dev["q"])
    lse_ref = torch.empty(w.batch, w.num_qo_heads, device="cuda")
    C.pa_run(plan, dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o_ref, lse_ref,
             ws, nbytes)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full_like(dev["q"], float("nan"))
        lse = torch.full((w.batch, w.num_qo_heads), float("nan"), device="cuda")
        C.pa_run_static_workspace(plan, dev["q"], dev["k_pool"], dev["v_pool"],
                                  dev["kv_indices"], o, lse)
        torch.cuda.synchronize()
        assert_close(to_np(o), to_np(lse), to_np(o_ref), to_np(lse_ref), "bf16", "static ws")


def test_static_workspace_refuses_oversized_plans():
    from serving_attention_paged_b200 import pagedattn as C
    lens = [8192] * 64
    w = W.make_workload("static_ws_big", lens, num_qo_heads=64, num_kv_heads=8, page_size=16,
                        dtype="f16", seed=92)
    # a huge CTA budget cuts every request into many pieces: > 8 MiB of partial states
    plan = C.pa_plan_create(_problem(C, w, num_sms=4096, ctas_per_sm=8), w.kv_indptr,
                            w.last_page_len)
    assert C.pa_plan_workspace_bytes(plan) > (8 << 20)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run_static_workspace(plan, 1 << 40, 1 << 40, 1 << 40, 1 << 40, 1 << 40, None)
    assert e.value.status == C.PA_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("kernel", ["cuda_cores", "tensor_cores"])
def test_static_workspace_reports_bad_index(kernel):
    """With PA_FLAG_CHECK_INDICES a run on the fixed workspace records an
    out-of-range page index there; pa_static_workspace_check reports its
    position and clears it, as pa_plan_check does for a caller workspace."""
    from serving_attention_paged_b200 import pagedattn as C
    w = W.make_workload("static_chk", [40, 40], num_qo_heads=8, num_kv_heads=2, page_size=16,
                        dtype="f16", seed=93)
    dev = {k: v.cuda() for k, v in w.materialize().items()}
    flags = C.PA_FLAG_CHECK_INDICES | (C.PA_FLAG_TENSOR_CORES if kernel == "tensor_cores"
                                       else C.PA_FLAG_CUDA_CORES)
    plan = C.pa_plan_create(_problem(C, w, ctas_per_sm=1, flags=flags), w.kv_indptr,
                            w.last_page_len)
    o = torch.empty_like(dev["q"])
    lse = torch.empty(w.batch, w.num_qo_heads, device="cuda")
    C.pa_run_static_workspace(plan, dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"],
                              o, lse)
    assert C.pa_static_workspace_check(plan) == -1
    bad = dev["kv_indices"].clone()
    bad[4] = w.num_pages + 7  # skipped by the checked kernel and recorded
    C.pa_run_static_workspace(plan, dev["q"], dev["k_pool"], dev["v_pool"], bad, o, lse)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_static_workspace_check(plan)
    assert e.value.status == C.PA_ERR_DEVICE_CHECK and e.value.position == 4
    assert C.pa_static_workspace_check(plan) == -1  # the word was cleared
