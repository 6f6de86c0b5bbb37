"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays them out as a paged KV cache.
It holds none of the attention arithmetic, so the CPU oracle (``oracle/``)
and the CUDA path can both be fed from it without sharing any method code.

Generator
---------
Every random value is a pure function of (seed, stream, counter): the
counter-based form of splitmix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): draw ``i`` of a stream with
key ``k`` is ``mix64(k + (i + 1) * 0x9E3779B97F4A7C15 mod 2**64)``.
Uniforms in (0, 1) take the top 53 bits plus one half.  Normal draws use
Box-Muller in fp64 (draws ``2p`` and ``2p+1`` give the pair ``p``; even
elements take the cosine branch, odd ones the sine branch), then round to
fp32 and then to the storage dtype, both with round-to-nearest-even.  The
same torch code runs on the CPU (small test cases, copied to the GPU) and
on the GPU (full-size pools that would be slow to draw on the host).

Workloads
---------
The shapes follow the FlashInfer README usage example ("single-request
decode", 32 heads, head_dim 128, kv_len 2048, fp16, randn inputs) and the
paged-KV names ``kv_indptr`` / ``kv_indices`` / ``last_page_len`` /
``kv_layout`` of the flashinfer-cubin registry page.  Keys and values are
drawn per *logical* token (request order, token order; for a cascade the
shared prefix comes first), then scattered to the pool rows the page table
assigns, so the same logical problem can be laid out in different page
orders or page sizes and must give the same attention result.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

# Stream identifiers: one independent splitmix64 stream per kind of draw.
STREAM_Q = 1
STREAM_K = 2
STREAM_V = 3
STREAM_LEN = 4
STREAM_PERM = 5

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
KV8_DTYPES = {"e4m3": torch.float8_e4m3fn, "e5m2": torch.float8_e5m2}
DTYPE_CODES = {"f16": 0, "bf16": 1}


def mix64(z: int) -> int:
    """splitmix64 finaliser on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def splitmix64_int(key: int, counter: int) -> int:
    """Draw ``counter`` of the stream with key ``key`` (Python ints)."""
    return mix64((key + (counter + 1) * GOLDEN) & MASK64)


def stream_key(seed: int, stream: int) -> int:
    return mix64((seed * GOLDEN + stream) & MASK64)


def _signed(x: int) -> int:
    x &= MASK64
    return x - (1 << 64) if x >> 63 else x


def _srl(x: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding uint64 bits."""
    return (x >> k) & ((1 << (64 - k)) - 1)


def splitmix64(key: int, counter: torch.Tensor) -> torch.Tensor:
    """Vectorised splitmix64 draws (int64 tensor holding uint64 bits).

    int64 multiplication wraps modulo 2**64 on both CPU and CUDA, which is
    exactly the uint64 arithmetic splitmix64 is defined with.
    """
    z = (counter + 1) * _signed(GOLDEN) + _signed(key)
    z = (z ^ _srl(z, 30)) * _signed(MIX1)
    z = (z ^ _srl(z, 27)) * _signed(MIX2)
    return z ^ _srl(z, 31)


def uniform(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """fp64 uniforms in the open interval (0, 1): (top 53 bits + 0.5) / 2**53."""
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return (_srl(splitmix64(key, i), 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def normal(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """fp64 N(0, 1) draws for element indices [start, start + count)."""
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    pair = i >> 1
    u1 = (_srl(splitmix64(key, 2 * pair), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    u2 = (_srl(splitmix64(key, 2 * pair + 1), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    r = torch.sqrt(-2.0 * torch.log(u1))
    th = (2.0 * math.pi) * u2
    return torch.where((i & 1) == 0, r * torch.cos(th), r * torch.sin(th))


def normal_as(key: int, start: int, count: int, dtype: str, device="cpu") -> torch.Tensor:
    """Normal draws rounded fp64 -> fp32 -> storage dtype (both RNE)."""
    return normal(key, start, count, device).to(torch.float32).to(DTYPES[dtype])


def uniform_np(key: int, count: int) -> np.ndarray:
    return uniform(key, 0, count).numpy()


def permutation(key: int, n: int) -> np.ndarray:
    """A uniformly random permutation of range(n): stable argsort of n draws."""
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    z = splitmix64(key, torch.arange(n, dtype=torch.int64)).numpy().view(np.uint64)
    return np.argsort(z, kind="stable").astype(np.int64)


@dataclass
class PagedWorkload:
    """One paged decode problem: shapes, page tables (host int32) and seeds.

    Pool layout is NHD: ``[num_pages, page_size, num_kv_heads, head_dim]``.
    ``kv_indptr`` / ``kv_indices`` / ``last_page_len`` describe the per-request
    page lists (for a cascade: the per-request *suffix*); ``prefix_indices``
    lists the shared prefix's pages (``prefix_len`` tokens, whole pages).
    """

    name: str
    batch: int
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    dtype: str
    seed: int
    num_pages: int
    kv_indptr: np.ndarray
    kv_indices: np.ndarray
    last_page_len: np.ndarray
    sm_scale: float = 0.0
    prefix_len: int = 0
    prefix_indices: Optional[np.ndarray] = None
    qo_lens: Optional[np.ndarray] = None  # prefill / append: new tokens per request
    # 8-bit KV cache: pools hold FP8 codes c, the cached key / value is scale * c
    kv_dtype: Optional[str] = None         # None (pools in `dtype`), "e4m3" or "e5m2"
    k_scale: float = 1.0
    v_scale: float = 1.0
    extra: dict = field(default_factory=dict)

    def __post_init__(self):
        if self.sm_scale == 0.0:
            self.sm_scale = 1.0 / math.sqrt(self.head_dim)
        self.kv_indptr = np.ascontiguousarray(self.kv_indptr, dtype=np.int32)
        self.kv_indices = np.ascontiguousarray(self.kv_indices, dtype=np.int32)
        self.last_page_len = np.ascontiguousarray(self.last_page_len, dtype=np.int32)
        if self.prefix_indices is not None:
            self.prefix_indices = np.ascontiguousarray(self.prefix_indices, dtype=np.int32)
        if self.qo_lens is not None:
            self.qo_lens = np.ascontiguousarray(self.qo_lens, dtype=np.int64)

    # -- derived sizes -------------------------------------------------------
    @property
    def group(self) -> int:
        return self.num_qo_heads // self.num_kv_heads

    def kv_lens(self) -> np.ndarray:
        """Suffix (or full, without a prefix) tokens per request."""
        n = np.diff(self.kv_indptr.astype(np.int64))
        return np.where(n > 0, (n - 1) * self.page_size + self.last_page_len, 0)

    def total_tokens(self) -> int:
        return int(self.prefix_len + self.kv_lens().sum())

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode step reads (prefix counted once)."""
        e = 1 if self.kv_dtype else 2
        return 2 * self.total_tokens() * self.num_kv_heads * self.head_dim * e

    def flat_tables(self):
        """Per-request page lists with the shared prefix's pages in front.

        Without a prefix this is just the suffix tables.  With one, request
        b's list is prefix pages ++ its own pages: the token sequence a
        non-cascaded decode of the same requests would read.
        """
        if not self.prefix_len:
            return self.kv_indptr, self.kv_indices, self.last_page_len
        npre = self.prefix_len // self.page_size
        n = np.diff(self.kv_indptr.astype(np.int64))
        indptr = np.zeros(self.batch + 1, dtype=np.int64)
        indptr[1:] = np.cumsum(n + npre)
        idx = np.concatenate(
            [np.concatenate([self.prefix_indices, self.kv_indices[self.kv_indptr[b]:self.kv_indptr[b + 1]]])
             for b in range(self.batch)]) if self.batch else np.zeros(0, np.int32)
        last = np.where(n > 0, self.last_page_len, self.page_size)
        return indptr.astype(np.int32), idx.astype(np.int32), last.astype(np.int32)

    def token_rows(self) -> np.ndarray:
        """Pool row of every logical token, in generation order (int64)."""
        P = self.page_size
        parts = []
        if self.prefix_len:
            t = np.arange(self.prefix_len, dtype=np.int64)
            parts.append(self.prefix_indices[t // P].astype(np.int64) * P + t % P)
        lens = self.kv_lens()
        for b in range(self.batch):
            L = int(lens[b])
            if L == 0:
                continue
            t = np.arange(L, dtype=np.int64)
            pages = self.kv_indices[self.kv_indptr[b]:self.kv_indptr[b + 1]].astype(np.int64)
            parts.append(pages[t // P] * P + t % P)
        return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)

    @property
    def qo_indptr(self) -> Optional[np.ndarray]:
        """Prefill / append: query-token offsets per request (int32 [B+1])."""
        if self.qo_lens is None:
            return None
        ind = np.zeros(self.batch + 1, dtype=np.int64)
        ind[1:] = np.cumsum(self.qo_lens)
        return ind.astype(np.int32)

    def query_rows(self) -> int:
        """q rows: one per request for decode, one per new token for prefill."""
        return self.batch if self.qo_lens is None else int(self.qo_lens.sum())

    def prefill_flops(self) -> int:
        """Causal attention flops of a prefill step (4 per query-key pair and element)."""
        lens = self.kv_lens()
        pairs = sum(int(Q) * int(L - Q) + int(Q) * (int(Q) + 1) // 2
                    for Q, L in zip(self.qo_lens, lens))
        return 4 * pairs * self.num_qo_heads * self.head_dim

    # -- tensors ---------------------------------------------------------------
    def make_q(self, device="cpu") -> torch.Tensor:
        rows = self.query_rows()
        n = rows * self.num_qo_heads * self.head_dim
        q = normal_as(stream_key(self.seed, STREAM_Q), 0, n, self.dtype, device)
        return q.view(rows, self.num_qo_heads, self.head_dim)

    def make_pool(self, which: str, device="cpu", chunk_tokens: int = 1 << 15,
                  rows: Optional[np.ndarray] = None) -> torch.Tensor:
        """K (``which='k'``) or V pool ``[num_pages, P, Hkv, D]``; unused rows are 0.

        An 8-bit pool holds each N(0, 1) draw (rounded to fp32) divided by the
        pool's scale and rounded to the FP8 format (torch's conversion, RNE)."""
        stream = STREAM_K if which == "k" else STREAM_V
        key = stream_key(self.seed, stream)
        w = self.num_kv_heads * self.head_dim
        pool_dtype = KV8_DTYPES[self.kv_dtype] if self.kv_dtype else DTYPES[self.dtype]
        pool = torch.zeros(self.num_pages * self.page_size, w,
                           dtype=torch.uint8 if self.kv_dtype else pool_dtype,
                           device=device).view(pool_dtype)  # 8-bit: byte 0 is +0.0
        if rows is None:
            rows = self.token_rows()
        rows_t = torch.from_numpy(rows).to(device)
        for j0 in range(0, len(rows), chunk_tokens):
            j1 = min(len(rows), j0 + chunk_tokens)
            if self.kv_dtype:
                scale = self.k_scale if which == "k" else self.v_scale
                x = normal(key, j0 * w, (j1 - j0) * w, device).to(torch.float32) / scale
                vals = x.to(pool_dtype).view(j1 - j0, w)
                # scatter the codes as bytes (indexing of 8-bit float tensors is not
                # available everywhere)
                pool.view(torch.uint8)[rows_t[j0:j1]] = vals.view(torch.uint8)
            else:
                vals = normal_as(key, j0 * w, (j1 - j0) * w, self.dtype, device).view(j1 - j0, w)
                pool[rows_t[j0:j1]] = vals
        return pool.view(self.num_pages, self.page_size, self.num_kv_heads, self.head_dim)

    def logical_kv(self, which: str, token_begin: int, token_end: int, device="cpu") -> torch.Tensor:
        """K or V of logical tokens [token_begin, token_end) as ``[n, Hkv, D]``
        (in the pool's storage type: FP8 codes for an 8-bit cache)."""
        stream = STREAM_K if which == "k" else STREAM_V
        w = self.num_kv_heads * self.head_dim
        n = (token_end - token_begin) * w
        if self.kv_dtype:
            scale = self.k_scale if which == "k" else self.v_scale
            x = normal(stream_key(self.seed, stream), token_begin * w, n, device).to(torch.float32)
            vals = (x / scale).to(KV8_DTYPES[self.kv_dtype])
        else:
            vals = normal_as(stream_key(self.seed, stream), token_begin * w, n, self.dtype, device)
        return vals.view(token_end - token_begin, self.num_kv_heads, self.head_dim)

    def materialize(self, device="cpu") -> dict:
        rows = self.token_rows()
        t = {
            "q": self.make_q(device),
            "k_pool": self.make_pool("k", device, rows=rows),
            "v_pool": self.make_pool("v", device, rows=rows),
            "kv_indptr": torch.from_numpy(self.kv_indptr).to(device),
            "kv_indices": torch.from_numpy(self.kv_indices).to(device),
            "last_page_len": torch.from_numpy(self.last_page_len).to(device),
        }
        if self.prefix_len:
            t["prefix_indices"] = torch.from_numpy(self.prefix_indices).to(device)
        return t


# ---------------------------------------------------------------------------
# Page-table builders
# ---------------------------------------------------------------------------

def tables_from_lengths(lens, page_size: int, page_order: Optional[np.ndarray] = None,
                        first_page: int = 0):
    """CSR page tables for requests of ``lens`` tokens.

    Request b gets ``ceil(L_b / P)`` consecutive entries of ``page_order``
    (default: pool pages ``first_page, first_page + 1, ...`` in order).
    ``last_page_len`` is ``L_b - P * (n_b - 1)`` (1..P) and 0 for an empty
    request.
    """
    lens = np.asarray(lens, dtype=np.int64)
    n = (lens + page_size - 1) // page_size
    indptr = np.zeros(len(lens) + 1, dtype=np.int64)
    indptr[1:] = np.cumsum(n)
    nnz = int(indptr[-1])
    if page_order is None:
        indices = np.arange(first_page, first_page + nnz, dtype=np.int64)
    else:
        indices = np.asarray(page_order[:nnz], dtype=np.int64)
    last = np.where(n > 0, lens - page_size * (n - 1), 0)
    return indptr.astype(np.int32), indices.astype(np.int32), last.astype(np.int32)


def make_workload(name, lens, *, num_qo_heads, num_kv_heads, head_dim=128, page_size=16,
                  dtype="f16", seed=0, shuffle=True, extra_pages=0, prefix_len=0,
                  sm_scale=0.0, qo_lens=None, kv_dtype=None, k_scale=1.0,
                  v_scale=1.0) -> PagedWorkload:
    """A paged problem whose pool holds exactly the pages used (+ ``extra_pages``).

    ``shuffle`` places every page at a random pool position (one permutation
    of the whole pool); otherwise pages are laid out in request order.  With
    ``prefix_len`` > 0 the shared prefix's pages come first in that order.
    """
    lens = np.asarray(lens, dtype=np.int64)
    if prefix_len % page_size:
        raise ValueError("the shared prefix must fill whole pages")
    npre = prefix_len // page_size
    nsuf = int(((lens + page_size - 1) // page_size).sum())
    num_pages = npre + nsuf + extra_pages
    order = (permutation(stream_key(seed, STREAM_PERM), num_pages) if shuffle
             else np.arange(num_pages, dtype=np.int64))
    prefix_indices = order[:npre].astype(np.int32) if prefix_len else None
    indptr, indices, last = tables_from_lengths(lens, page_size, order[npre:])
    return PagedWorkload(name=name, batch=len(lens), num_qo_heads=num_qo_heads,
                         num_kv_heads=num_kv_heads, head_dim=head_dim, page_size=page_size,
                         dtype=dtype, seed=seed, num_pages=num_pages, kv_indptr=indptr,
                         kv_indices=indices, last_page_len=last, prefix_len=prefix_len,
                         prefix_indices=prefix_indices, sm_scale=sm_scale, qo_lens=qo_lens,
                         kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale)


# ---------------------------------------------------------------------------
# The five benchmark workloads (seed = 1000 + workload number)
# ---------------------------------------------------------------------------

def single_request_decode(seed=1001) -> PagedWorkload:
    """B=1, 32/32 heads, D=128, kv_len 2048, P=16, fp16; 128 pages drawn from a
    shuffled 256-page pool (the README's single-request decode example, paged)."""
    w = make_workload("single_request_decode", [2048], num_qo_heads=32, num_kv_heads=32,
                      page_size=16, dtype="f16", seed=seed, extra_pages=128)
    return w


def batch_decode_uniform(seed=1002) -> PagedWorkload:
    """B=16, GQA 32/8, kv_len 4096 each, P=16, fp16, pool exactly the 4096 pages, shuffled."""
    return make_workload("batch_decode_uniform", [4096] * 16, num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="f16", seed=seed)


def ragged_lengths(seed=1003, batch=64, lo=128, hi=32768) -> np.ndarray:
    u = uniform_np(stream_key(seed, STREAM_LEN), batch)
    return np.floor(np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).astype(np.int64)


def batch_decode_ragged(seed=1003) -> PagedWorkload:
    """B=64, GQA 32/8, kv_len log-uniform in [128, 32768], P=16, bf16, shuffled exact pool."""
    return make_workload("batch_decode_ragged", ragged_lengths(seed), num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=seed)


def vector_sparse_lengths(seed=1004, batch=256, lo=512, hi=8192) -> np.ndarray:
    u = uniform_np(stream_key(seed, STREAM_LEN), batch)
    return lo + np.floor(u * (hi - lo + 1)).astype(np.int64)


def vector_sparse_decode(seed=1004, pool_tokens=1 << 21) -> PagedWorkload:
    """B=256, GQA 64/8, kv_len U[512, 8192], P=1, bf16; kv_indices are the first
    sum(L) entries of a random permutation of a 2M-token pool."""
    lens = vector_sparse_lengths(seed)
    order = permutation(stream_key(seed, STREAM_PERM), pool_tokens)
    indptr, indices, last = tables_from_lengths(lens, 1, order)
    return PagedWorkload(name="vector_sparse_decode", batch=len(lens), num_qo_heads=64,
                         num_kv_heads=8, head_dim=128, page_size=1, dtype="bf16", seed=seed,
                         num_pages=pool_tokens, kv_indptr=indptr, kv_indices=indices,
                         last_page_len=last)


def vector_sparse_small(seed=1004, batch=48, pool_tokens=1 << 19) -> PagedWorkload:
    """The first 48 requests of ``vector_sparse_decode`` (same length draws,
    GQA 64/8, P=1, bf16) in a 512K-token pool: small enough (2 x 1 GB pools)
    for a full counter capture of one launch."""
    lens = vector_sparse_lengths(seed, batch)
    order = permutation(stream_key(seed, STREAM_PERM), pool_tokens)
    indptr, indices, last = tables_from_lengths(lens, 1, order)
    return PagedWorkload(name="vector_sparse_small", batch=len(lens), num_qo_heads=64,
                         num_kv_heads=8, head_dim=128, page_size=1, dtype="bf16", seed=seed,
                         num_pages=pool_tokens, kv_indptr=indptr, kv_indices=indices,
                         last_page_len=last)


def vector_sparse_contiguous_twin(seed=1004) -> PagedWorkload:
    """The same requests and token values as ``vector_sparse_decode`` with
    P=16 and each request's pages contiguous and ascending in the pool."""
    lens = vector_sparse_lengths(seed)
    w = make_workload("vector_sparse_contiguous_twin", lens, num_qo_heads=64, num_kv_heads=8,
                      page_size=16, dtype="bf16", seed=seed, shuffle=False)
    return w


def cascade_lengths(seed=1005, batch=128, lo=64, hi=1024) -> np.ndarray:
    u = uniform_np(stream_key(seed, STREAM_LEN), batch)
    return lo + np.floor(u * (hi - lo + 1)).astype(np.int64)


def cascade_shared_prefix(seed=1005, prefix_len=16384) -> PagedWorkload:
    """B=128, GQA 32/8, a 16384-token shared prefix (1024 pages, own list) plus a
    per-request suffix U[64, 1024], P=16, fp16; all pages shuffled in one pool."""
    return make_workload("cascade_shared_prefix", cascade_lengths(seed), num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="f16", seed=seed,
                         prefix_len=prefix_len)


def prefill_append(seed=1006) -> PagedWorkload:
    """B=8 requests appending 1024 new tokens to 1024 cached ones (kv_len 2048,
    causal), GQA 32/8, P=16, fp16, shuffled exact pool."""
    return make_workload("prefill_append", [2048] * 8, num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="f16", seed=seed, qo_lens=[1024] * 8)


def batch_decode_uniform_fp8(seed=1002) -> PagedWorkload:
    """Workload 2 with an 8-bit E4M3 cache: the same draws stored as codes with
    per-tensor scales (K 0.02, V 0.02: the largest draw, ~6.5, maps below the
    format's 448)."""
    return make_workload("batch_decode_uniform_fp8", [4096] * 16, num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="f16", seed=seed, kv_dtype="e4m3",
                         k_scale=0.02, v_scale=0.02)


def batch_decode_ragged_fp8(seed=1003) -> PagedWorkload:
    """Workload 3 (bf16 q) with an 8-bit E4M3 cache, scales as for 2f8."""
    return make_workload("batch_decode_ragged_fp8", ragged_lengths(seed), num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=seed, kv_dtype="e4m3",
                         k_scale=0.02, v_scale=0.02)


WORKLOADS = {
    1: single_request_decode,
    2: batch_decode_uniform,
    3: batch_decode_ragged,
    4: vector_sparse_decode,
    5: cascade_shared_prefix,
    "4c": vector_sparse_contiguous_twin,
    "4s": vector_sparse_small,
    6: prefill_append,
    "2f8": batch_decode_uniform_fp8,
    "3f8": batch_decode_ragged_fp8,
}
