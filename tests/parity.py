"""Shared helpers for the GPU parity tests: run the library, run the oracle,
compare with the tolerance paged decode promises.

Tolerance (fp16 / bf16 inputs): max |o_gpu - o_oracle| <= 2e-3 and
max |lse_gpu - lse_oracle| <= 1e-3 against the fp64 oracle.  The output is
rounded once to the input dtype, which alone costs up to half an ulp: for
bf16 that exceeds 2e-3 once |o| >= 1 (fp16: |o| >= 8).  Where the dtype's
half-ulp at the reference value is itself >= 2e-3, the allowance is
2e-3 + that half-ulp.  An empty request must give exactly o = 0, lse = -inf.
"""
import numpy as np

import oracle

O_TOL = 2e-3
LSE_TOL = 1e-3
MANT_BITS = {"f16": 10, "bf16": 7}


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 1e-30)))
    if dtype == "f16":
        e = np.maximum(e, -14)
    return 0.5 * np.exp2(e - MANT_BITS[dtype])


def o_allowance(ref: np.ndarray, dtype: str) -> np.ndarray:
    hu = half_ulp(ref, dtype)
    return np.where(hu >= O_TOL, O_TOL + hu, O_TOL)


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    bad = err > o_allowance(o_ref, dtype)
    assert not bad.any(), (f"{what}: o mismatch at {np.argwhere(bad)[:5].tolist()}, "
                           f"max err {err.max():.3e}")
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{what}: -inf lse mismatch"
    if (~empty).any():
        lerr = np.abs(lse_gpu[~empty] - lse_ref[~empty])
        assert lerr.max() <= LSE_TOL, f"{what}: lse max err {lerr.max():.3e}"
    assert np.all(o_gpu[empty] == 0), f"{what}: empty request must give o = 0"
    return float(err.max()), float(np.abs(lse_gpu[~empty] - lse_ref[~empty]).max()
                                   if (~empty).any() else 0.0)


def oracle_full(w, t):
    """Oracle over all rows, inputs on the CPU (tables: prefix ++ own pages)."""
    indptr, indices, last = w.flat_tables()
    return oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], indptr, indices, last,
                               num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads,
                               head_dim=w.head_dim, page_size=w.page_size, dtype=w.dtype,
                               sm_scale=w.sm_scale, threads=8)


def oracle_sampled(w, dev, requests, threads=8):
    """Oracle for every q head of the listed requests of a device-resident
    problem (only those requests' pages are copied to the host)."""
    indptr, indices, last = w.flat_tables()
    return oracle.paged_decode_requests(
        dev["q"], dev["k_pool"], dev["v_pool"], indptr, indices, last, requests,
        num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
        page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, threads=threads)


def to_np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)
