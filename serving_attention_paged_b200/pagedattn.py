"""ctypes binding of libpagedattn.so: the C ABI of ``include/pagedattn.h``.

Argument marshalling only.  Every step of the attention path runs in the
library's CUDA kernels; there is no Python or CPU fallback.  If the library
is missing the import fails loudly.  Functions keep the C names; device
buffers may be given as torch tensors (their ``data_ptr()`` is passed) or
as raw integer addresses, and streams as ``torch.cuda.Stream`` or raw
``cudaStream_t`` integers (default: torch's current stream).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m serving_attention_paged_b200.build` "
        "(there is no fallback implementation)")
lib = ctypes.CDLL(_LIB_PATH)

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE_TOO_SMALL = 0, 1, 2, 3
PA_ERR_CUDA, PA_ERR_DEVICE_CHECK, PA_ERR_NO_MEMORY, PA_ERR_DEVICE_TIMEOUT = 4, 5, 6, 7
PA_F16, PA_BF16, PA_F32, PA_E4M3, PA_E5M2 = 0, 1, 2, 3, 4
PA_FLAG_CHECK_INDICES = 1
PA_FLAG_CUDA_CORES = 2
PA_FLAG_TENSOR_CORES = 4
DTYPE_CODES = {"f16": PA_F16, "bf16": PA_BF16, "f32": PA_F32, "e4m3": PA_E4M3,
               "e5m2": PA_E5M2}


class pa_problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_qo_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("num_sms", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32), ("min_chunk_tokens", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("flags", ctypes.c_uint32),
                ("piece_cost_tokens", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("rope_theta", ctypes.c_float)]


class pa_work_item(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("request", "kv_head", "page_begin", "token_begin", "token_end", "partial_slot")]


class pa_prefill_tile(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("request", "q_begin", "n_q", "page_begin", "kv_base", "kv_end")]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_P = ctypes.POINTER
_SIGS = {
    "pa_plan_create": [_P(pa_problem), _vp, _vp, _P(_vp)],
    "pa_cascade_plan_create": [_P(pa_problem), _i32, _vp, _vp, _P(_vp)],
    "pa_prefill_plan_create": [_P(pa_problem), _i32, _vp, _vp, _vp, _P(_vp)],
    "pa_plan_prefill_tiles": [_vp, _P(_P(pa_prefill_tile)), _P(_i64)],
    "pa_prefill_run": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "pa_plan_quota_tokens": [_vp, _P(_i32)],
    "pa_plan_cta_indptr": [_vp, _P(_P(_i32)), _P(_i64)],
    "pa_plan_prefill_schedule": [_vp, _P(_P(_i32)), _P(_i64)],
    "pa_plan_work_items": [_vp, _P(_P(pa_work_item)), _P(_i64)],
    "pa_plan_merge_indptr": [_vp, _P(_P(_i32))],
    "pa_plan_num_partials": [_vp, _P(_i64)],
    "pa_plan_prefix_chunks": [_vp, _P(_i32), _P(_i32)],
    "pa_plan_workspace_bytes": [_vp, _P(_sz)],
    "pa_plan_status_offset": [_vp, _P(_sz)],
    "pa_plan_upload": [_vp, _vp, _sz, _vp],
    "pa_run": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "pa_cascade_run": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "pa_merge_state": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _vp],
    "pa_run_static_workspace": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "pa_plan_check": [_vp, _vp, _P(_i64), _vp],
    "pa_static_workspace_check": [_vp, _P(_i64), _vp],
    "pa_default_schedule": [_i32, _i32, _i32, _i32, ctypes.c_uint32, _P(_i32), _P(_i32)],
    "pa_problem_schedule": [_P(pa_problem), _i32, _P(_i32), _P(_i32)],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
lib.pa_plan_destroy.argtypes = [_vp]
lib.pa_plan_destroy.restype = None
lib.pa_status_string.argtypes = [ctypes.c_int]
lib.pa_status_string.restype = ctypes.c_char_p
lib.pa_abi_version.argtypes = []
lib.pa_abi_version.restype = ctypes.c_int32
lib.pa_plan_uses_tensor_cores.argtypes = [_vp]
lib.pa_plan_uses_tensor_cores.restype = ctypes.c_int32


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.pa_status_string(status).decode()} (status {status})")


def _check(status: int, where: str):
    if status != PA_OK:
        raise PagedAttnError(status, where)


def _ptr(x):
    """Device (or host) address of a tensor / integer / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _host_i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


class Plan:
    """Owns a ``pa_plan_t`` and the host arrays it was made from."""

    def __init__(self, handle: int):
        self.handle = handle
        self._destroy = lib.pa_plan_destroy  # still reachable during interpreter shutdown

    def __del__(self):
        if getattr(self, "handle", None):
            self._destroy(self.handle)
            self.handle = None


def make_problem(*, batch, num_qo_heads, num_kv_heads, head_dim=128, page_size, dtype,
                 sm_scale, num_sms, ctas_per_sm, min_chunk_tokens=0, num_pages=0,
                 flags=0, piece_cost_tokens=0, kv_dtype=None, k_scale=1.0, v_scale=1.0,
                 rope_theta=0.0) -> pa_problem:
    """``kv_dtype`` None: the pools hold ``dtype``; "e4m3" / "e5m2": 8-bit
    pools with ``k_scale`` / ``v_scale``.  ``rope_theta`` > 0: rotary
    positions applied on the fly."""
    if isinstance(dtype, str):
        dtype = DTYPE_CODES[dtype]
    if kv_dtype is None:
        kv_dtype = dtype
    elif isinstance(kv_dtype, str):
        kv_dtype = DTYPE_CODES[kv_dtype]
    return pa_problem(batch, num_qo_heads, num_kv_heads, head_dim, page_size, dtype, sm_scale,
                      num_sms, ctas_per_sm, min_chunk_tokens, num_pages, flags,
                      piece_cost_tokens, kv_dtype, k_scale, v_scale, rope_theta or 0.0)


def pa_plan_create(problem: pa_problem, kv_indptr_host, last_page_len_host) -> Plan:
    indptr, last = _host_i32(kv_indptr_host), _host_i32(last_page_len_host)
    h = _vp()
    _check(lib.pa_plan_create(ctypes.byref(problem), indptr.ctypes.data,
                              last.ctypes.data if last.size else None, ctypes.byref(h)),
           "pa_plan_create")
    return Plan(h.value)


def pa_cascade_plan_create(problem: pa_problem, prefix_len: int, kv_indptr_host,
                           last_page_len_host) -> Plan:
    indptr, last = _host_i32(kv_indptr_host), _host_i32(last_page_len_host)
    h = _vp()
    _check(lib.pa_cascade_plan_create(ctypes.byref(problem), prefix_len, indptr.ctypes.data,
                                      last.ctypes.data if last.size else None, ctypes.byref(h)),
           "pa_cascade_plan_create")
    return Plan(h.value)


def pa_prefill_plan_create(problem: pa_problem, causal: bool, qo_indptr_host, kv_indptr_host,
                           last_page_len_host) -> Plan:
    qo = _host_i32(qo_indptr_host)
    indptr, last = _host_i32(kv_indptr_host), _host_i32(last_page_len_host)
    h = _vp()
    _check(lib.pa_prefill_plan_create(ctypes.byref(problem), int(bool(causal)), qo.ctypes.data,
                                      indptr.ctypes.data, last.ctypes.data if last.size else None,
                                      ctypes.byref(h)),
           "pa_prefill_plan_create")
    return Plan(h.value)


def pa_plan_prefill_tiles(plan: Plan) -> np.ndarray:
    """The prefill tiles in launch order as an int32 array [n, 6] (a copy):
    request, q_begin, n_q, page_begin, kv_base, kv_end."""
    p, n = _P(pa_prefill_tile)(), _i64()
    _check(lib.pa_plan_prefill_tiles(plan.handle, ctypes.byref(p), ctypes.byref(n)),
           "pa_plan_prefill_tiles")
    if n.value == 0:
        return np.zeros((0, 6), dtype=np.int32)
    buf = ctypes.cast(p, _P(_i32 * (6 * n.value))).contents
    return np.frombuffer(buf, dtype=np.int32).reshape(n.value, 6).copy()


def pa_plan_quota_tokens(plan: Plan) -> int:
    c = _i32()
    _check(lib.pa_plan_quota_tokens(plan.handle, ctypes.byref(c)), "pa_plan_quota_tokens")
    return c.value


def pa_plan_cta_indptr(plan: Plan) -> np.ndarray:
    p, n = _P(_i32)(), _i64()
    _check(lib.pa_plan_cta_indptr(plan.handle, ctypes.byref(p), ctypes.byref(n)),
           "pa_plan_cta_indptr")
    return np.ctypeslib.as_array(p, shape=(n.value + 1,)).copy()


def pa_plan_prefill_schedule(plan: Plan) -> np.ndarray:
    """A prefill plan's items (tile * num_kv_heads + kv head) grouped by CTA,
    as an int32 array (a copy); pa_plan_cta_indptr delimits each CTA's list."""
    p, n = _P(_i32)(), _i64()
    _check(lib.pa_plan_prefill_schedule(plan.handle, ctypes.byref(p), ctypes.byref(n)),
           "pa_plan_prefill_schedule")
    if n.value == 0:
        return np.zeros(0, dtype=np.int32)
    return np.ctypeslib.as_array(p, shape=(n.value,)).copy()


def pa_plan_work_items(plan: Plan) -> np.ndarray:
    """The work list as an int32 array [n, 6] (a copy)."""
    p, n = _P(pa_work_item)(), _i64()
    _check(lib.pa_plan_work_items(plan.handle, ctypes.byref(p), ctypes.byref(n)),
           "pa_plan_work_items")
    if n.value == 0:
        return np.zeros((0, 6), dtype=np.int32)
    buf = ctypes.cast(p, _P(_i32 * (6 * n.value))).contents
    return np.frombuffer(buf, dtype=np.int32).reshape(n.value, 6).copy()


def pa_plan_num_partials(plan: Plan) -> int:
    n = _i64()
    _check(lib.pa_plan_num_partials(plan.handle, ctypes.byref(n)), "pa_plan_num_partials")
    return n.value


def pa_plan_merge_indptr(plan: Plan, n_segments: int) -> np.ndarray:
    """Partial-slot offsets per (request, kv head) segment: [B * Hkv + 1]."""
    p = _P(_i32)()
    _check(lib.pa_plan_merge_indptr(plan.handle, ctypes.byref(p)), "pa_plan_merge_indptr")
    return np.ctypeslib.as_array(p, shape=(n_segments + 1,)).copy()


def pa_plan_prefix_chunks(plan: Plan):
    n, t = _i32(), _i32()
    _check(lib.pa_plan_prefix_chunks(plan.handle, ctypes.byref(n), ctypes.byref(t)),
           "pa_plan_prefix_chunks")
    return n.value, t.value


def pa_plan_workspace_bytes(plan: Plan) -> int:
    n = _sz()
    _check(lib.pa_plan_workspace_bytes(plan.handle, ctypes.byref(n)), "pa_plan_workspace_bytes")
    return n.value


def pa_plan_status_offset(plan: Plan) -> int:
    n = _sz()
    _check(lib.pa_plan_status_offset(plan.handle, ctypes.byref(n)), "pa_plan_status_offset")
    return n.value


def pa_plan_upload(plan: Plan, workspace, workspace_bytes: int, stream=None):
    _check(lib.pa_plan_upload(plan.handle, _ptr(workspace), workspace_bytes, _stream(stream)),
           "pa_plan_upload")


def pa_run(plan: Plan, q, k_pool, v_pool, kv_indices, o, lse, workspace, workspace_bytes: int,
           stream=None):
    _check(lib.pa_run(plan.handle, _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(kv_indices),
                      _ptr(o), _ptr(lse), _ptr(workspace), workspace_bytes, _stream(stream)),
           "pa_run")


def pa_cascade_run(plan: Plan, q, k_pool, v_pool, prefix_indices, kv_indices, o, lse, workspace,
                   workspace_bytes: int, stream=None):
    _check(lib.pa_cascade_run(plan.handle, _ptr(q), _ptr(k_pool), _ptr(v_pool),
                              _ptr(prefix_indices), _ptr(kv_indices), _ptr(o), _ptr(lse),
                              _ptr(workspace), workspace_bytes, _stream(stream)),
           "pa_cascade_run")


def pa_prefill_run(plan: Plan, q, k_pool, v_pool, kv_indices, o, lse, workspace,
                   workspace_bytes: int, stream=None):
    _check(lib.pa_prefill_run(plan.handle, _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(kv_indices),
                              _ptr(o), _ptr(lse), _ptr(workspace), workspace_bytes,
                              _stream(stream)),
           "pa_prefill_run")


def pa_run_static_workspace(plan: Plan, q, k_pool, v_pool, kv_indices, o, lse, stream=None):
    """pa_run with the library's own fixed 8 MiB device workspace, for callers
    that cannot allocate device memory (see include/pagedattn.h)."""
    _check(lib.pa_run_static_workspace(plan.handle, _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                       _ptr(kv_indices), _ptr(o), _ptr(lse), _stream(stream)),
           "pa_run_static_workspace")


def pa_merge_state(o_a, lse_a, o_b, lse_b, o, lse, rows: int, head_dim: int, dtype,
                   stream=None):
    if isinstance(dtype, str):
        dtype = DTYPE_CODES[dtype]
    _check(lib.pa_merge_state(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o), _ptr(lse),
                              rows, head_dim, dtype, _stream(stream)), "pa_merge_state")


def pa_plan_check(plan: Plan, workspace, stream=None) -> int:
    """-1 when no bad page index was seen, else raises PagedAttnError(DEVICE_CHECK)
    with ``.position`` set to the first bad kv_indices position."""
    pos = _i64()
    st = lib.pa_plan_check(plan.handle, _ptr(workspace), ctypes.byref(pos), _stream(stream))
    if st == PA_ERR_DEVICE_CHECK:
        err = PagedAttnError(st, "pa_plan_check")
        err.position = pos.value
        raise err
    _check(st, "pa_plan_check")
    return pos.value


def pa_static_workspace_check(plan: Plan, stream=None) -> int:
    """pa_plan_check for the status words of the library's fixed workspace,
    as the last ``pa_run_static_workspace`` call left them."""
    pos = _i64()
    st = lib.pa_static_workspace_check(plan.handle, ctypes.byref(pos), _stream(stream))
    if st == PA_ERR_DEVICE_CHECK:
        err = PagedAttnError(st, "pa_static_workspace_check")
        err.position = pos.value
        raise err
    _check(st, "pa_static_workspace_check")
    return pos.value


def pa_default_schedule(device: int, num_qo_heads: int, num_kv_heads: int, dtype, flags: int = 0):
    if isinstance(dtype, str):
        dtype = DTYPE_CODES[dtype]
    sms, k = _i32(), _i32()
    _check(lib.pa_default_schedule(device, num_qo_heads, num_kv_heads, dtype, flags,
                                   ctypes.byref(sms), ctypes.byref(k)), "pa_default_schedule")
    return sms.value, k.value


def pa_problem_schedule(problem: pa_problem, device: int):
    """(SM count, resident CTAs per SM) of the decode kernel ``problem`` runs."""
    sms, k = _i32(), _i32()
    _check(lib.pa_problem_schedule(ctypes.byref(problem), device, ctypes.byref(sms),
                                   ctypes.byref(k)), "pa_problem_schedule")
    return sms.value, k.value


def pa_status_string(status: int) -> str:
    return lib.pa_status_string(status).decode()


def pa_plan_uses_tensor_cores(plan: Plan) -> bool:
    return lib.pa_plan_uses_tensor_cores(plan.handle) == 1


def pa_abi_version() -> int:
    return lib.pa_abi_version()
