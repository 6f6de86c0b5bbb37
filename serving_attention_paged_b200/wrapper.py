"""Convenience layer over the C ABI for PyTorch callers.

``PagedDecode`` holds a plan and its device workspace (allocated through
torch, the library itself never allocates) and calls ``pa_run`` /
``pa_cascade_run``; ``PagedPrefill`` does the same for ``pa_prefill_run``.
They only marshal arguments; all attention work is done by the library's
kernels.
"""
from __future__ import annotations

import torch

from . import pagedattn as C

_TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


class PagedDecode:
    """Plan once per decode step (host), run once per layer (device).

    ``prefix_len`` > 0 makes a cascade plan: every request first attends to a
    shared prefix of that many tokens (``prefix_indices`` at run time), then
    to its own pages.
    """

    def __init__(self, kv_indptr, last_page_len, *, num_qo_heads, num_kv_heads, page_size,
                 dtype, sm_scale, num_pages, head_dim=128, device=None, num_sms=None,
                 ctas_per_sm=None, min_chunk_tokens=0, prefix_len=0, flags=0,
                 piece_cost_tokens=0, kv_dtype=None, k_scale=1.0, v_scale=1.0,
                 rope_theta=0.0, stream=None):
        self.device = torch.device(device if device is not None else "cuda")
        dev_index = self.device.index if self.device.index is not None else torch.cuda.current_device()
        self.dtype = dtype
        self.batch = len(last_page_len)
        self.num_qo_heads, self.head_dim = num_qo_heads, head_dim
        self.prefix_len = prefix_len
        extra = dict(kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale, rope_theta=rope_theta)
        if num_sms is None or ctas_per_sm is None:
            shape = C.make_problem(batch=self.batch, num_qo_heads=num_qo_heads,
                                   num_kv_heads=num_kv_heads, head_dim=head_dim,
                                   page_size=page_size, dtype=dtype, sm_scale=sm_scale,
                                   num_sms=1, ctas_per_sm=1, flags=flags, **extra)
            sms, k = C.pa_problem_schedule(shape, dev_index)
            num_sms = sms if num_sms is None else num_sms
            ctas_per_sm = k if ctas_per_sm is None else ctas_per_sm
        self.problem = C.make_problem(batch=self.batch, num_qo_heads=num_qo_heads,
                                      num_kv_heads=num_kv_heads, head_dim=head_dim,
                                      page_size=page_size, dtype=dtype, sm_scale=sm_scale,
                                      num_sms=num_sms, ctas_per_sm=ctas_per_sm,
                                      min_chunk_tokens=min_chunk_tokens, num_pages=num_pages,
                                      flags=flags, piece_cost_tokens=piece_cost_tokens,
                                      **extra)
        if prefix_len:
            self.plan = C.pa_cascade_plan_create(self.problem, prefix_len, kv_indptr, last_page_len)
        else:
            self.plan = C.pa_plan_create(self.problem, kv_indptr, last_page_len)
        self.workspace_bytes = C.pa_plan_workspace_bytes(self.plan)
        self.workspace = torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8,
                                     device=self.device)
        C.pa_plan_upload(self.plan, self.workspace, self.workspace.numel(), stream)

    def work_items(self):
        return C.pa_plan_work_items(self.plan)

    def run(self, q, k_pool, v_pool, kv_indices, o=None, lse=None, prefix_indices=None,
            stream=None):
        if o is None:
            o = torch.empty(self.batch, self.num_qo_heads, self.head_dim,
                            dtype=_TORCH_DTYPES[self.dtype], device=self.device)
        if lse is None:
            lse = torch.empty(self.batch, self.num_qo_heads, dtype=torch.float32,
                              device=self.device)
        if self.prefix_len:
            C.pa_cascade_run(self.plan, q, k_pool, v_pool, prefix_indices, kv_indices, o, lse,
                             self.workspace, self.workspace.numel(), stream)
        else:
            C.pa_run(self.plan, q, k_pool, v_pool, kv_indices, o, lse, self.workspace,
                     self.workspace.numel(), stream)
        return o, lse

    def check(self, stream=None) -> int:
        return C.pa_plan_check(self.plan, self.workspace, stream)


class PagedPrefill:
    """Prefill / append attention: plan once per batch of new tokens (host),
    run once per layer (device).  ``qo_indptr`` gives each request's new query
    tokens (rows of q); with ``causal`` they are the last of its keys and
    each sees the keys up to its own position, else every token sees all of
    its request's keys."""

    def __init__(self, qo_indptr, kv_indptr, last_page_len, *, num_qo_heads, num_kv_heads,
                 page_size, dtype, sm_scale, num_pages, causal=True, head_dim=128, device=None,
                 num_sms=None, flags=0, stream=None):
        self.device = torch.device(device if device is not None else "cuda")
        self.dtype = dtype
        self.batch = len(last_page_len)
        self.total_q = int(qo_indptr[-1]) if self.batch else 0
        self.num_qo_heads, self.head_dim = num_qo_heads, head_dim
        # one persistent CTA per SM (ctas_per_sm does not apply to prefill plans)
        if num_sms is None:
            num_sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.problem = C.make_problem(batch=self.batch, num_qo_heads=num_qo_heads,
                                      num_kv_heads=num_kv_heads, head_dim=head_dim,
                                      page_size=page_size, dtype=dtype, sm_scale=sm_scale,
                                      num_sms=num_sms, ctas_per_sm=1, num_pages=num_pages,
                                      flags=flags)
        self.plan = C.pa_prefill_plan_create(self.problem, causal, qo_indptr, kv_indptr,
                                             last_page_len)
        self.workspace_bytes = C.pa_plan_workspace_bytes(self.plan)
        self.workspace = torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8,
                                     device=self.device)
        C.pa_plan_upload(self.plan, self.workspace, self.workspace.numel(), stream)

    def tiles(self):
        return C.pa_plan_prefill_tiles(self.plan)

    def cta_indptr(self):
        return C.pa_plan_cta_indptr(self.plan)

    def run(self, q, k_pool, v_pool, kv_indices, o=None, lse=None, stream=None):
        if o is None:
            o = torch.empty(self.total_q, self.num_qo_heads, self.head_dim,
                            dtype=_TORCH_DTYPES[self.dtype], device=self.device)
        if lse is None:
            lse = torch.empty(self.total_q, self.num_qo_heads, dtype=torch.float32,
                              device=self.device)
        C.pa_prefill_run(self.plan, q, k_pool, v_pool, kv_indices, o, lse, self.workspace,
                         self.workspace.numel(), stream)
        return o, lse

    def check(self, stream=None) -> int:
        return C.pa_plan_check(self.plan, self.workspace, stream)
