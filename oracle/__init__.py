"""CPU oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA path (it
imports nothing from ``serving_attention_paged_b200``) and the CUDA path never
imports it.

Contents, each written from the FlashInfer README (core features 1-3, the
single-request decode usage example) and the flashinfer-cubin registry page
(paged-KV names ``kv_indptr`` / ``kv_indices`` / ``last_page_len``):

* ``paged_decode`` — the attention definition in fp64 (``paged_attention.c``),
  over 16-bit pools or 8-bit (FP8 E4M3 / E5M2) pools with a K and a V scale
  (README core feature 3: low-precision attention for a compressed KV-Cache),
  optionally with LLaMA-style rotary positions applied on the fly.
* ``merge_state`` / ``merge_states`` — combining attention states by their
  log-sum-exp (what split-KV and cascade attention rely on).
* ``cascade_decode`` — shared prefix merged with per-request suffix.
* ``paged_prefill`` — causal attention of new (appended) query tokens over
  the paged KV (README usage example: prefill / append attention).
* ``plan`` — the split-KV work-list specification restated with plain
  loops (the library's work list must agree with it exactly).

Parity status: every function here is pinned by ``tests/test_oracle.py``,
``tests/test_plan_oracle.py``, ``tests/test_prefill_oracle.py`` and
``tests/test_fp8_oracle.py`` (closed forms, invariants, brute force, and
torch's own FP8 conversion for the 8-bit widening).  The pages print no
worked numeric example, so nothing is pinned to a published output value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "paged_attention.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build_library(force: bool = False) -> str:
    """Compile the fp64 C oracle with gcc (plain -O2: no fast-math, no FMA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               _SRC, "-o", _LIB, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_library())
        i32, i64, dbl, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.oracle_paged_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                            dbl, vp, i64, vp, vp, i32]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_widen.argtypes = [ctypes.c_uint16, i32]
        lib.oracle_widen.restype = dbl
        lib.oracle_paged_decode_kv.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                               i32, i32, dbl, dbl, dbl, dbl, vp, i64, vp, vp,
                                               i32]
        lib.oracle_paged_decode_kv.restype = ctypes.c_int
        lib.oracle_widen8.argtypes = [ctypes.c_uint8, i32]
        lib.oracle_widen8.restype = dbl
        _lib = lib
    return _lib


DTYPE_CODE = {"f16": 0, "bf16": 1}


def _as_u16(x) -> np.ndarray:
    """fp16 / bf16 storage (torch tensor or numpy) as a contiguous uint16 array."""
    if hasattr(x, "detach"):  # torch tensor: reinterpret its 16-bit storage
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy()
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    return x.view(np.uint16)


def _as_u8(x) -> np.ndarray:
    """8-bit float storage (torch float8 tensor or uint8 numpy) as contiguous uint8."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu().contiguous().view(torch.uint8).numpy()
    return np.ascontiguousarray(x).view(np.uint8)


KV8_CODE = {"e4m3": 0, "e5m2": 1}


def _as_i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def widen(bits: int, dtype: str) -> float:
    """The oracle's exact fp16 / bf16 -> fp64 widening of one 16-bit pattern."""
    return _load().oracle_widen(bits, DTYPE_CODE[dtype])


def widen8(code: int, kv_dtype: str) -> float:
    """The oracle's exact FP8 (``e4m3``: OCP E4M3 without infinities, max 448;
    ``e5m2``: OCP E5M2) -> fp64 widening of one 8-bit pattern."""
    return _load().oracle_widen8(code, KV8_CODE[kv_dtype])


def paged_decode(q, k_pool, v_pool, kv_indptr, kv_indices, last_page_len, *, num_qo_heads,
                 num_kv_heads, head_dim, page_size, dtype, sm_scale, rows=None, threads=1,
                 kv_dtype=None, k_scale=1.0, v_scale=1.0, rope_theta=None):
    """fp64 attention of every (b, hq) row (or the listed ``rows`` = b*Hq+hq).

    ``dtype`` is q's (fp16 / bf16).  With ``kv_dtype=None`` the pools hold the
    same 16-bit type; with ``kv_dtype`` ``"e4m3"`` or ``"e5m2"`` they hold
    8-bit codes and each cached key is ``k_scale * code`` (values:
    ``v_scale * code``).

    ``rope_theta`` (README usage example: decode with LLaMA-style RoPE on the
    fly) rotates q to position L_b - 1 and key t to position t before the dot
    product: element pairs (d, d + D/2) turn by pos * rope_theta^(-2d/D).

    Returns ``(o, lse)``: o ``[n_rows, D]`` fp64 and lse ``[n_rows]`` fp64
    (natural log; -inf for an empty request).  With ``rows=None`` the result
    is reshaped to ``[B, Hq, D]`` / ``[B, Hq]``.
    """
    lib = _load()
    qa = _as_u16(q)
    if kv_dtype is None:
        ka, va, fmt = _as_u16(k_pool), _as_u16(v_pool), -1
    else:
        ka, va, fmt = _as_u8(k_pool), _as_u8(v_pool), KV8_CODE[kv_dtype]
    indptr, indices, last = _as_i32(kv_indptr), _as_i32(kv_indices), _as_i32(last_page_len)
    batch = len(last)
    if rows is None:
        n_rows = batch * num_qo_heads
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = len(rows_arr)
    o = np.zeros((n_rows, head_dim), dtype=np.float64)
    lse = np.zeros(n_rows, dtype=np.float64)
    if indices.size == 0:
        indices = np.zeros(1, dtype=np.int32)
    rc = lib.oracle_paged_decode_kv(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, indptr.ctypes.data, indices.ctypes.data,
        last.ctypes.data if last.size else None, batch, num_qo_heads, num_kv_heads, head_dim,
        page_size, DTYPE_CODE[dtype], fmt, float(sm_scale), float(k_scale), float(v_scale),
        float(rope_theta) if rope_theta else 0.0, rows_arr.ctypes.data if rows_arr is not None else None, n_rows, o.ctypes.data,
        lse.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("oracle_paged_decode rejected its arguments")
    if rows is None:
        return o.reshape(batch, num_qo_heads, head_dim), lse.reshape(batch, num_qo_heads)
    return o, lse


def paged_decode_requests(q, k_pool, v_pool, kv_indptr, kv_indices, last_page_len, requests, *,
                          num_qo_heads, num_kv_heads, head_dim, page_size, dtype, sm_scale,
                          threads=1, kv_dtype=None, k_scale=1.0, v_scale=1.0, rope_theta=None):
    """``paged_decode`` for every q head of the listed requests only.

    q and the pools may be large torch tensors on any device: only the pages
    those requests read are copied to the host, as a compact pool with the
    page table renumbered to match (the tokens each request reads, and their
    order, are unchanged).  Returns o ``[len(requests), Hq, D]`` and lse.
    """
    indptr, indices, last = _as_i32(kv_indptr), _as_i32(kv_indices), _as_i32(last_page_len)
    pages = [indices[indptr[b]:indptr[b + 1]] for b in requests]
    used = np.unique(np.concatenate(pages)) if pages else np.zeros(0, np.int64)
    remap = np.full(int(used.max()) + 1 if used.size else 1, -1, np.int64)
    remap[used] = np.arange(len(used))
    sub_indptr = np.zeros(len(requests) + 1, np.int32)
    sub_indptr[1:] = np.cumsum([len(p) for p in pages])
    sub_indices = (remap[np.concatenate(pages)] if pages else np.zeros(0)).astype(np.int32)
    sub_last = last[np.asarray(requests, dtype=np.int64)] if len(requests) else last[:0]
    if hasattr(k_pool, "detach"):
        import torch
        sel = torch.from_numpy(used.astype(np.int64)).to(k_pool.device)
        kp, vp = k_pool[sel].cpu(), v_pool[sel].cpu()
        qs = q[torch.as_tensor(list(requests), dtype=torch.int64, device=q.device)].cpu()
    else:
        kp, vp, qs = k_pool[used], v_pool[used], q[list(requests)]
    return paged_decode(qs, kp, vp, sub_indptr, sub_indices, sub_last,
                        num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads,
                        head_dim=head_dim, page_size=page_size, dtype=dtype,
                        sm_scale=sm_scale, threads=threads, kv_dtype=kv_dtype,
                        k_scale=k_scale, v_scale=v_scale, rope_theta=rope_theta)


def merge_state(o_a, lse_a, o_b, lse_b):
    """Combine two attention states over disjoint token sets (fp64).

    With M = max(lse_a, lse_b) and weights w = exp(lse - M):
    o = (w_a o_a + w_b o_b) / (w_a + w_b),  lse = M + ln(w_a + w_b).
    Both empty (lse = -inf) gives o = 0, lse = -inf.
    """
    return merge_states([(o_a, lse_a), (o_b, lse_b)])


def merge_states(states):
    """Combine any number of attention states ``(o [.., D], lse [..])`` (fp64)."""
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in states])
    os_ = np.stack([np.asarray(o, dtype=np.float64) for o, _ in states])
    M = lses.max(axis=0)
    empty = np.isneginf(M)
    Ms = np.where(empty, 0.0, M)
    w = np.exp(lses - Ms)  # exp(-inf) = 0 for empty states
    wsum = w.sum(axis=0)
    safe = np.where(empty, 1.0, wsum)
    o = (w[..., None] * os_).sum(axis=0) / safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, Ms + np.log(safe))
    return o, lse


def cascade_decode(q, k_pool, v_pool, prefix_indices, prefix_len, kv_indptr, kv_indices,
                   last_page_len, *, num_qo_heads, num_kv_heads, head_dim, page_size, dtype,
                   sm_scale, threads=1):
    """Two-level cascade: attention over the shared prefix, attention over each
    request's own pages, merged by log-sum-exp (FlashInfer README, core
    feature 3: cascade attention over a hierarchical KV cache)."""
    batch = len(_as_i32(last_page_len))
    npre = prefix_len // page_size
    pre_indptr = np.arange(batch + 1, dtype=np.int32) * npre
    pre_indices = np.tile(_as_i32(prefix_indices)[:npre], batch) if batch else np.zeros(0, np.int32)
    pre_last = np.full(batch, page_size if npre else 0, dtype=np.int32)
    kw = dict(num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
              page_size=page_size, dtype=dtype, sm_scale=sm_scale, threads=threads)
    o1, l1 = paged_decode(q, k_pool, v_pool, pre_indptr, pre_indices, pre_last, **kw)
    o2, l2 = paged_decode(q, k_pool, v_pool, kv_indptr, kv_indices, last_page_len, **kw)
    return merge_state(o1, l1, o2, l2)


def paged_prefill(q, k_pool, v_pool, qo_indptr, kv_indptr, kv_indices, last_page_len, *,
                  num_qo_heads, num_kv_heads, head_dim, page_size, dtype, sm_scale,
                  causal=True, queries=None, threads=1):
    """Prefill / append attention (README usage example: append attention
    with a causal mask, the new tokens being the last ones in the KV-Cache;
    prefill attention without the mask).

    Request b has L_b keys (its page table) and Q_b = qo_indptr[b + 1] -
    qo_indptr[b] new query tokens.  With ``causal`` those are its last Q_b
    keys (Q_b <= L_b) and query i (0-based) attends to keys
    t < L_b - Q_b + i + 1; without it every query attends to all L_b keys.
    Either way that is exactly a decode over the request's pages cut at the
    query's limit, so each query becomes one row of ``paged_decode`` with its
    own page list.

    q is ``[total_q, Hq, D]``.  Returns o ``[n, Hq, D]`` and lse ``[n, Hq]``
    for every query (``queries=None``) or the listed global query indices.
    """
    qo = [int(x) for x in _as_i32(qo_indptr)]
    indptr = [int(x) for x in _as_i32(kv_indptr)]
    indices = _as_i32(kv_indices)
    last = [int(x) for x in _as_i32(last_page_len)]
    B, P = len(last), page_size
    owner = []
    for b in range(B):
        n = indptr[b + 1] - indptr[b]
        L = (n - 1) * P + last[b] if n > 0 else 0
        Q = qo[b + 1] - qo[b]
        if causal and Q > L:
            raise ValueError(f"request {b}: {Q} queries but only {L} keys")
        owner += [(b, L, Q, i) for i in range(Q)]
    sel = list(range(len(owner))) if queries is None else [int(x) for x in queries]
    q_indptr, q_indices, q_last = [0], [], []
    for g in sel:
        b, L, Q, i = owner[g]
        lim = L - Q + i + 1 if causal else L
        n = -(-lim // P)
        q_indices.extend(indices[indptr[b]:indptr[b] + n].tolist())
        q_indptr.append(len(q_indices))
        q_last.append(lim - (n - 1) * P)
    if hasattr(q, "detach"):
        import torch
        qs = q[torch.as_tensor(sel, dtype=torch.int64, device=q.device)].cpu()
        kp, vp = k_pool.cpu(), v_pool.cpu()
    else:
        qs, kp, vp = np.asarray(q)[sel], k_pool, v_pool
    return paged_decode(qs, kp, vp, q_indptr, q_indices, q_last, num_qo_heads=num_qo_heads,
                        num_kv_heads=num_kv_heads, head_dim=head_dim, page_size=page_size,
                        dtype=dtype, sm_scale=sm_scale, threads=threads)


def plan(kv_indptr, last_page_len, *, page_size, num_kv_heads, num_sms, ctas_per_sm,
         min_chunk_tokens=256, piece_cost=0):
    """Split-KV work list (FlashInfer README core feature 2: variable-length
    inputs are scheduled in a plan stage to even out the load; the README
    also names stream-K among FlashInfer's inspirations).

    Specification (the reading adopted where the page is silent), restated
    here with plain loops; c = piece_cost is the budget a piece boundary
    costs, in tokens:
      L_b = 0 if n_b = 0 else (n_b - 1) * P + last_page_len[b]; T = sum_b L_b;
      N = number of non-empty requests; W = num_sms * ctas_per_sm;
      groups = max(1, floor(W / Hkv)).
      Walk for budget q: requests in order fill groups in order; a group's
      first piece costs its token count, each later piece c more; a group
      is full once it holds a piece and used + c >= q, and the next token
      then opens the next group (a request cut there goes on as that group's
      first piece).  An empty request is a zero-length, free piece of the
      group the next token goes to (the last group at the very end).
      q = 32 * ceil(max(min_chunk_tokens, ceil((T + c * max(N - 1, 0)) / groups)) / 32);
      n_groups = the groups the walk fills (0 for an empty batch), which is
      at most `groups`.  With c = 0, group g is token positions
      [g q, (g + 1) q) of the requests laid end to end.
      CTA g * Hkv + h runs the pieces of group g for kv head h.  A (request,
      head) segment cut into k > 1 pieces owns partial slots
      merge_indptr[b * Hkv + h] + 0 .. k - 1, in order.

    Returns ``(quota, items, cta_indptr, merge_indptr)``; items is int32
    ``[n, 6]``: request, kv_head, page_begin (= kv_indptr[b]), token_begin,
    token_end, partial_slot.
    """
    indptr = [int(x) for x in _as_i32(kv_indptr)]
    last = [int(x) for x in _as_i32(last_page_len)]
    B, P, Hkv, c = len(last), page_size, num_kv_heads, piece_cost
    L = []
    for b in range(B):
        n = indptr[b + 1] - indptr[b]
        L.append((n - 1) * P + last[b] if n > 0 else 0)
    T = sum(L)
    N = sum(1 for x in L if x > 0)
    groups = max(1, (num_sms * ctas_per_sm) // Hkv)

    def fill(q):
        """Pieces (b, t0, t1) per group for budget q."""
        out = [[]]
        load = 0          # budget used by the group being filled
        opened = False    # it holds a non-empty piece
        for b in range(B):
            if L[b] == 0:
                gi = len(out) - 1
                if opened and load + c >= q:
                    gi += 1
                    out.append([])
                    # the next token goes there: start it fresh
                    load, opened = 0, False
                out[gi].append((b, 0, 0))
                continue
            t = 0
            while t < L[b]:
                extra = c if opened else 0
                if opened and load + extra >= q:
                    out.append([])
                    load, opened = 0, False
                    continue
                n = min(L[b] - t, q - load - extra)
                out[-1].append((b, t, t + n))
                load += extra + n
                opened = True
                t += n
        # groups that received only empty requests after the last token
        while len(out) > 1 and all(t1 == t0 for (_, t0, t1) in out[-1]) and \
                not any(t1 > t0 for (_, t0, t1) in out[-1]):
            tail = out.pop()
            out[-1].extend(tail)
        return out

    q = 32 * (-(-max(min_chunk_tokens, -(-(T + c * max(N - 1, 0)) // groups)) // 32))
    group_pieces = fill(q) if B > 0 else []
    n_groups = len(group_pieces)
    assert n_groups <= groups

    items, cta_indptr = [], [0]
    for g in range(n_groups):
        for h in range(Hkv):
            for (b, t0, t1) in group_pieces[g]:
                items.append([b, h, indptr[b], t0, t1, -1])
            cta_indptr.append(len(items))

    count = [0] * (B * Hkv)
    for it in items:
        count[it[0] * Hkv + it[1]] += 1
    merge_indptr = [0] * (B * Hkv + 1)
    for seg in range(B * Hkv):
        merge_indptr[seg + 1] = merge_indptr[seg] + (count[seg] if count[seg] > 1 else 0)
    seen = [0] * (B * Hkv)
    for it in items:
        seg = it[0] * Hkv + it[1]
        if count[seg] > 1:
            it[5] = merge_indptr[seg] + seen[seg]
            seen[seg] += 1
    return (q, np.array(items, dtype=np.int32).reshape(-1, 6),
            np.array(cta_indptr, dtype=np.int32), np.array(merge_indptr, dtype=np.int32))


__all__ = ["build_library", "paged_decode", "paged_decode_requests", "merge_state", "merge_states", "cascade_decode",
           "paged_prefill", "plan", "widen", "widen8"]
