"""The prefill / append plan on the host (no GPU): its tiles cover every new
query token of every request exactly once, in runs of at most 256 / G
tokens of one request, with the key range of the causal rule (or all keys
without the mask), grouped by request with long tiles first; malformed
tables are rejected before anything runs."""
import numpy as np
import pytest

from serving_attention_paged_b200 import workloads as W


@pytest.fixture(scope="module")
def C():
    from serving_attention_paged_b200 import build
    build.build()
    from serving_attention_paged_b200 import pagedattn
    return pagedattn


def _problem(C, batch, hq=32, hkv=8, P=16, flags=0, num_sms=1):
    return C.make_problem(batch=batch, num_qo_heads=hq, num_kv_heads=hkv, page_size=P,
                          dtype="f16", sm_scale=0.088, num_sms=num_sms, ctas_per_sm=1,
                          num_pages=1 << 16, flags=flags)


def _item_load(tile, G):
    """The load the schedule counts for one item, from its tile: the 128-key
    tiles of its two 128-row halves plus 2."""
    _, _, n, _, base, end = (int(x) for x in tile)
    n0 = min(n, 128 // G)
    nt0 = -(-min(base + n0, end) // 128)
    nt1 = -(-end // 128) if n > n0 else 0
    return nt0 + nt1 + 2


def _list_schedule(loads, n_cta):
    """Greedy list scheduling written with an explicit scan (no heap): item w
    goes to the CTA with the least load so far, the lowest such CTA on ties."""
    lists, total = [[] for _ in range(n_cta)], [0] * n_cta
    for w, x in enumerate(loads):
        c = min(range(n_cta), key=lambda k: (total[k], k))
        lists[c].append(w)
        total[c] += x
    return lists, total


def _tables(kv_lens, P):
    n = [-(-L // P) for L in kv_lens]
    indptr = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    last = np.array([L - (k - 1) * P if k else 0 for L, k in zip(kv_lens, n)], np.int32)
    return indptr, last


def _expected_tiles(kv_lens, qo_lens, G, causal):
    """The tile rule written out: per request, runs of 256 / G new tokens."""
    per = 256 // G
    out, qo = [], 0
    indptr, _ = _tables(kv_lens, 16)
    for b, (L, Q) in enumerate(zip(kv_lens, qo_lens)):
        for t0 in range(0, Q, per):
            n = min(per, Q - t0)
            base, end = (L - Q + t0, L - Q + t0 + n) if causal else (L - 1, L)
            out.append((b, qo + t0, n, int(indptr[b]), base, end))
        qo += Q
    return out


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (32, 4), (16, 8)])
def test_tiles_cover_every_query_once_longest_first(C, causal, hq, hkv):
    rng = np.random.default_rng(5 + hq + hkv)
    kv_lens = [int(x) for x in rng.integers(1, 3000, 23)] + [0, 1, 64, 65]
    qo_lens = [int(rng.integers(0, L + 1)) for L in kv_lens]
    qo_lens[3] = kv_lens[3]  # a fresh prefill
    indptr, last = _tables(kv_lens, 16)
    qo_indptr = np.concatenate([[0], np.cumsum(qo_lens)]).astype(np.int32)
    plan = C.pa_prefill_plan_create(_problem(C, len(kv_lens), hq, hkv), causal, qo_indptr,
                                    indptr, last)
    tiles = C.pa_plan_prefill_tiles(plan)
    G = hq // hkv
    expected = _expected_tiles(kv_lens, qo_lens, G, causal)
    # the same set of tiles ...
    assert sorted(map(tuple, tiles.tolist())) == sorted(expected)
    # ... each request's tiles together, requests by decreasing longest tile
    # (ties by request), a request's tiles by decreasing ceil(kv_end / 128)
    # (ties in token order)
    keys = -(-tiles[:, 5] // 128)
    reqs = tiles[:, 0]
    starts = np.flatnonzero(np.r_[True, np.diff(reqs) != 0])
    assert len(starts) == len(np.unique(reqs))  # contiguous per request
    longest = [keys[reqs == r].max() for r in reqs[starts]]
    order = list(zip([-x for x in longest], reqs[starts].tolist()))
    assert order == sorted(order)
    for r in np.unique(reqs):
        mine = tiles[reqs == r]
        k = -(-mine[:, 5] // 128)
        assert np.all(np.diff(k) <= 0)
        for kk in np.unique(k):
            assert np.all(np.diff(mine[k == kk][:, 1]) > 0)
    # every new token of every request exactly once
    seen = np.zeros(qo_indptr[-1], np.int32)
    for r, q0, n, pb, base, end in tiles:
        assert 1 <= n <= 256 // G and pb == indptr[r]
        assert qo_indptr[r] <= q0 and q0 + n <= qo_indptr[r + 1]
        seen[q0:q0 + n] += 1
    assert np.all(seen == 1)
    assert C.pa_plan_workspace_bytes(plan) >= tiles.nbytes


def test_tiles_of_the_prefill_workload(C):
    w = W.WORKLOADS[6]()
    plan = C.pa_prefill_plan_create(_problem(C, w.batch, w.num_qo_heads, w.num_kv_heads,
                                             w.page_size), True, w.qo_indptr, w.kv_indptr,
                                    w.last_page_len)
    tiles = C.pa_plan_prefill_tiles(plan)
    G = w.num_qo_heads // w.num_kv_heads
    assert len(tiles) == w.batch * (1024 // (256 // G))
    # the last token of each request sees every key of it
    lens = w.kv_lens()
    for r in range(w.batch):
        mine = tiles[tiles[:, 0] == r]
        assert mine[:, 5].max() == lens[r] and mine[:, 4].min() == lens[r] - 1024


def test_prefill_plan_validation(C):
    indptr, last = _tables([40, 10], 16)
    ok = np.array([0, 40, 50], np.int32)
    C.pa_prefill_plan_create(_problem(C, 2), True, ok, indptr, last)
    for bad in ([0, 41, 51], [1, 40, 50], [0, 40, 39]):  # more queries than keys, bad start, decreasing
        with pytest.raises(C.PagedAttnError) as e:
            C.pa_prefill_plan_create(_problem(C, 2), True, np.array(bad, np.int32), indptr, last)
        assert e.value.status == C.PA_ERR_INVALID_ARG
    # without the mask more queries than keys are fine
    C.pa_prefill_plan_create(_problem(C, 2), False, np.array([0, 41, 51], np.int32), indptr, last)
    # pages must be whole tensor-memory-access boxes (>= 8 rows)
    i4, l4 = _tables([40, 10], 4)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_prefill_plan_create(_problem(C, 2, P=4), True, ok, i4, l4)
    assert e.value.status == C.PA_ERR_UNSUPPORTED


def test_plans_run_only_through_their_own_entry_point(C):
    indptr, last = _tables([40, 10], 16)
    pf = C.pa_prefill_plan_create(_problem(C, 2), True, np.array([0, 4, 6], np.int32), indptr,
                                  last)
    dec = C.pa_plan_create(_problem(C, 2), indptr, last)
    big = 1 << 40  # never dereferenced: the host check fails first
    ws_pf, ws_dec = C.pa_plan_workspace_bytes(pf), C.pa_plan_workspace_bytes(dec)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run(pf, big, big, big, big, big, None, big, ws_pf, 0)
    assert e.value.status == C.PA_ERR_INVALID_ARG
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_prefill_run(dec, big, big, big, big, big, None, big, ws_dec, 0)
    assert e.value.status == C.PA_ERR_INVALID_ARG
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_run_static_workspace(pf, big, big, big, big, big, None, 0)
    assert e.value.status == C.PA_ERR_INVALID_ARG
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_prefill_run(pf, big, big, big, big, big, None, big, ws_pf - 1, 0)
    assert e.value.status == C.PA_ERR_WORKSPACE_TOO_SMALL


def test_empty_prefill_plans_run_without_a_launch(C):
    """No requests, or requests without new tokens: no tiles, and the run
    returns at once (no CUDA call is made, so this runs on the host)."""
    empty = C.pa_prefill_plan_create(_problem(C, 0), True, np.zeros(1, np.int32),
                                     np.zeros(1, np.int32), np.zeros(0, np.int32))
    assert len(C.pa_plan_prefill_tiles(empty)) == 0
    nb = C.pa_plan_workspace_bytes(empty)
    C.pa_prefill_run(empty, None, None, None, None, None, None, 1 << 40, nb, 0)
    indptr, last = _tables([40, 10], 16)
    idle = C.pa_prefill_plan_create(_problem(C, 2), True, np.zeros(3, np.int32), indptr, last)
    assert len(C.pa_plan_prefill_tiles(idle)) == 0
    big = 1 << 40  # never dereferenced
    C.pa_prefill_run(idle, big, big, big, big, big, None, big, C.pa_plan_workspace_bytes(idle), 0)


def test_prefill_plans_report_tensor_cores(C):
    indptr, last = _tables([40, 10], 16)
    for flags in (0, C.PA_FLAG_CUDA_CORES):
        plan = C.pa_prefill_plan_create(_problem(C, 2, flags=flags), True,
                                        np.array([0, 4, 6], np.int32), indptr, last)
        assert C.pa_plan_uses_tensor_cores(plan) is True


def test_prefill_refuses_pools_beyond_signed_32bit_rows(C):
    """Page rows are TMA coordinates (signed 32-bit): a pool of 2^31 - 1 rows or
    more is refused before anything runs."""
    indptr, last = _tables([40, 10], 16)
    big = C.make_problem(batch=2, num_qo_heads=32, num_kv_heads=8, page_size=16, dtype="f16",
                         sm_scale=0.088, num_sms=1, ctas_per_sm=1, num_pages=(1 << 31) // 16)
    with pytest.raises(C.PagedAttnError) as e:
        C.pa_prefill_plan_create(big, True, np.array([0, 4, 6], np.int32), indptr, last)
    assert e.value.status == C.PA_ERR_UNSUPPORTED
    ok = C.make_problem(batch=2, num_qo_heads=32, num_kv_heads=8, page_size=16, dtype="f16",
                        sm_scale=0.088, num_sms=1, ctas_per_sm=1, num_pages=(1 << 26))
    C.pa_prefill_plan_create(ok, True, np.array([0, 4, 6], np.int32), indptr, last)


def test_prefill_pool_row_limit_at_its_edge(C):
    """The edge of the limit: with page size 8 (the smallest the prefill
    kernel moves), 2^28 - 1 pages (2^31 - 8 rows, the largest pool whose rows
    and the one-past-the-end fill row fit a signed 32-bit coordinate) are
    accepted and 2^28 pages (2^31 rows) refused; the same holds for cascade
    plans with a prefix."""
    indptr, last = _tables([40, 10], 8)

    def prob(num_pages):
        return C.make_problem(batch=2, num_qo_heads=32, num_kv_heads=8, page_size=8,
                              dtype="f16", sm_scale=0.088, num_sms=1, ctas_per_sm=1,
                              num_pages=num_pages)

    qo = np.array([0, 4, 6], np.int32)
    C.pa_prefill_plan_create(prob((1 << 28) - 1), True, qo, indptr, last)
    C.pa_cascade_plan_create(prob((1 << 28) - 1), 64, indptr, last)
    for make in (lambda p: C.pa_prefill_plan_create(p, True, qo, indptr, last),
                 lambda p: C.pa_cascade_plan_create(p, 64, indptr, last)):
        with pytest.raises(C.PagedAttnError) as e:
            make(prob(1 << 28))
        assert e.value.status == C.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("num_sms", [1, 5, 148, 1000])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 2)])
def test_persistent_schedule_deals_items_by_least_load(C, num_sms, hq, hkv):
    """min(num_sms, items) CTAs; every item (tile * Hkv + kv head) exactly once;
    the lists equal greedy list scheduling in item order by the estimated
    load; the CTAs' loads end within one item of each other."""
    rng = np.random.default_rng(num_sms + hq)
    kv_lens = [int(x) for x in rng.integers(1, 4000, 19)] + [1, 300]
    qo_lens = [int(rng.integers(0, L + 1)) for L in kv_lens]
    indptr, last = _tables(kv_lens, 16)
    qo_indptr = np.concatenate([[0], np.cumsum(qo_lens)]).astype(np.int32)
    plan = C.pa_prefill_plan_create(_problem(C, len(kv_lens), hq, hkv, num_sms=num_sms), True,
                                    qo_indptr, indptr, last)
    tiles = C.pa_plan_prefill_tiles(plan)
    sched = C.pa_plan_prefill_schedule(plan)
    ci = C.pa_plan_cta_indptr(plan)
    n_items = len(tiles) * hkv
    n_cta = min(num_sms, n_items)
    assert len(ci) == n_cta + 1 and ci[0] == 0 and ci[-1] == n_items
    assert np.all(np.diff(ci) >= 0)
    assert sorted(sched.tolist()) == list(range(n_items))
    loads = [_item_load(tiles[w // hkv], hq // hkv) for w in range(n_items)]
    lists, total = _list_schedule(loads, n_cta)
    assert [sched[ci[c]:ci[c + 1]].tolist() for c in range(n_cta)] == lists
    assert max(total) - min(total) <= max(loads)
    assert C.pa_plan_workspace_bytes(plan) >= tiles.nbytes + sched.nbytes


def test_item_load_of_a_hand_worked_tile():
    """G = 4 (32 tokens a half): a causal tile of 64 tokens at keys 1000..1063
    has half 0 seeing up to key 1032 (9 tiles of 128) and half 1 up to 1064
    (9 tiles); 20 with the fixed 2.  A 20-token tile has no second half."""
    assert _item_load((0, 0, 64, 0, 1000, 1064), 4) == 9 + 9 + 2
    assert _item_load((0, 0, 20, 0, 1000, 1020), 4) == 8 + 0 + 2
    assert _item_load((0, 0, 64, 0, 1023, 1087), 4) == 9 + 9 + 2
    assert _item_load((0, 0, 64, 0, 1000, 1024), 8) == 8 + 8 + 2


def test_empty_prefill_plan_has_no_ctas(C):
    indptr, last = _tables([40, 10], 16)
    plan = C.pa_prefill_plan_create(_problem(C, 2, num_sms=148), True, np.zeros(3, np.int32),
                                    indptr, last)
    assert len(C.pa_plan_prefill_schedule(plan)) == 0
    assert C.pa_plan_cta_indptr(plan).tolist() == [0]
