"""The seeded input generator: splitmix64 bits, normal draws, page tables."""
import math

import numpy as np
import torch

from serving_attention_paged_b200 import workloads as W


def test_splitmix64_matches_integer_definition():
    for key in (0, 1, W.stream_key(1234, 2), (1 << 64) - 1):
        c = torch.tensor([0, 1, 2, 1000, (1 << 40) + 3], dtype=torch.int64)
        got = W.splitmix64(key, c).numpy().view(np.uint64)
        ref = [W.splitmix64_int(key, int(x)) for x in c]
        assert [int(x) for x in got] == ref


def test_splitmix64_known_sequence():
    # seed 0: the reference implementation's first outputs (Vigna's splitmix64.c)
    assert W.splitmix64_int(0, 0) == 0xE220A8397B1DCDAF
    assert W.splitmix64_int(0, 1) == 0x6E789E6AA1B965F4


def test_normal_moments_and_chunk_independence():
    key = W.stream_key(7, W.STREAM_K)
    z = W.normal(key, 0, 1 << 18)
    assert abs(z.mean().item()) < 0.01 and abs(z.std().item() - 1) < 0.01
    # a slice drawn on its own equals the same slice of a longer draw
    assert torch.equal(W.normal(key, 1001, 77), z[1001:1078])


def test_pool_chunking_and_placement():
    w = W.make_workload("t", [33, 0, 70], num_qo_heads=4, num_kv_heads=2, page_size=16,
                        dtype="bf16", seed=3, extra_pages=2)
    a = w.make_pool("k", chunk_tokens=7)
    b = w.make_pool("k", chunk_tokens=1 << 15)
    assert torch.equal(a, b)
    rows = w.token_rows()
    assert len(set(rows.tolist())) == len(rows)  # no two tokens share a pool row
    logical = w.logical_kv("k", 0, len(rows))
    assert torch.equal(a.view(-1, 2, 128)[torch.from_numpy(rows)], logical)


def test_permutation_and_tables():
    p = W.permutation(W.stream_key(1, W.STREAM_PERM), 1000)
    assert sorted(p.tolist()) == list(range(1000))
    indptr, idx, last = W.tables_from_lengths([0, 1, 16, 17], 16)
    assert indptr.tolist() == [0, 0, 1, 2, 4]
    assert last.tolist() == [0, 1, 16, 1]
    assert idx.tolist() == [0, 1, 2, 3]


def test_benchmark_workload_shapes():
    w1 = W.WORKLOADS[1]()
    assert w1.num_pages == 256 and w1.kv_lens().tolist() == [2048] and len(w1.kv_indices) == 128
    w2 = W.WORKLOADS[2]()
    assert w2.num_pages == 4096 and sorted(w2.kv_indices.tolist()) == list(range(4096))
    w3 = W.WORKLOADS[3]()
    L = w3.kv_lens()
    assert L.min() >= 128 and L.max() <= 32768 and w3.dtype == "bf16"
    assert sorted(w3.kv_indices.tolist()) == list(range(w3.num_pages))
    w5 = W.WORKLOADS[5]()
    assert w5.prefix_len == 16384 and len(w5.prefix_indices) == 1024
    assert 64 <= w5.kv_lens().min() and w5.kv_lens().max() <= 1024
    assert w2.kv_bytes() == 2 * 16 * 4096 * 8 * 128 * 2
    assert abs(w1.sm_scale - 1 / math.sqrt(128)) < 1e-15


def test_prefill_flop_accounting():
    """The bench's per-token flops (4 per visible key and element, all q heads)
    summed over every new token equal the workload's total, and a causal token
    sees L_b - Q_b + i + 1 keys: brute force on a small ragged batch."""
    import numpy as np

    import bench
    w = W.make_workload("pf_flops", [10, 7, 0, 33], num_qo_heads=4, num_kv_heads=2,
                        head_dim=16, page_size=4, dtype="f16", seed=9, qo_lens=[10, 3, 0, 5])
    allq = np.arange(w.query_rows())
    assert bench.prefill_query_flops(w, allq) == w.prefill_flops()
    lens, qo = w.kv_lens(), w.qo_indptr
    brute = 0
    for b in range(w.batch):
        Q = qo[b + 1] - qo[b]
        for i in range(Q):
            brute += 4 * (int(lens[b]) - Q + i + 1) * w.num_qo_heads * w.head_dim
    assert brute == w.prefill_flops()
    # one token alone: the last of request 3 sees all 33 keys
    assert bench.prefill_query_flops(w, np.array([w.query_rows() - 1])) == 4 * 33 * 4 * 16
    # workload 6: 8 * 32 * (1024 * 1024 + 1024 * 1025 / 2) pairs * 512
    assert W.WORKLOADS[6]().prefill_flops() == 8 * 32 * (1024 * 1024 + 1024 * 1025 // 2) * 512
