"""Pins for the oracle's paged KV write (page "test: add block-level
DeepSeek-V4 attention test", decode timeline: the paged KV write ahead of
the sparse attention core): a second formulation through numpy fancy
indexing over the flattened pools, untouched rows, faults."""
import numpy as np


def _case(seed=0, P=12, ps=16, d=64, B=3, cols=4, n=20):
    rng = np.random.default_rng(seed)
    pt = rng.permutation(P)[: B * cols].reshape(B, cols).astype(np.int32)
    k_pool = rng.integers(0, 1 << 16, size=(P, ps, d), dtype=np.uint16)
    v_pool = rng.integers(0, 1 << 16, size=(P, ps, d), dtype=np.uint16)
    # distinct (request, position) pairs
    flat = rng.choice(B * cols * ps, size=n, replace=False)
    req = (flat // (cols * ps)).astype(np.int32)
    pos = (flat % (cols * ps)).astype(np.int32)
    k_new = rng.integers(0, 1 << 16, size=(n, d), dtype=np.uint16)
    v_new = rng.integers(0, 1 << 16, size=(n, d), dtype=np.uint16)
    return k_new, v_new, req, pos, pt, k_pool, v_pool


def test_write_matches_fancy_indexing(oracle):
    k_new, v_new, req, pos, pt, k_pool, v_pool = _case()
    k_out, v_out, flags = oracle.paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool)
    assert flags == 0
    P, ps, d = k_pool.shape
    rows = pt[req, pos // ps].astype(np.int64) * ps + pos % ps
    k_ref = k_pool.reshape(P * ps, d).copy()
    v_ref = v_pool.reshape(P * ps, d).copy()
    k_ref[rows] = k_new
    v_ref[rows] = v_new
    assert np.array_equal(k_out.reshape(P * ps, d), k_ref)
    assert np.array_equal(v_out.reshape(P * ps, d), v_ref)
    # every other row is untouched
    other = np.setdiff1d(np.arange(P * ps), rows)
    assert np.array_equal(k_out.reshape(P * ps, d)[other], k_pool.reshape(P * ps, d)[other])


def test_read_back_through_the_page_table(oracle):
    k_new, v_new, req, pos, pt, k_pool, v_pool = _case(seed=1, d=128, ps=64, cols=2, n=50)
    k_out, v_out, _ = oracle.paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool)
    ps = k_pool.shape[1]
    for j in range(len(req)):
        page = pt[req[j], pos[j] // ps]
        assert np.array_equal(k_out[page, pos[j] % ps], k_new[j])
        assert np.array_equal(v_out[page, pos[j] % ps], v_new[j])


def test_faulty_tokens_are_skipped_and_flagged(oracle):
    k_new, v_new, req, pos, pt, k_pool, v_pool = _case(seed=2)
    req = req.copy()
    pos = pos.copy()
    pt = pt.copy()
    req[0] = 7                  # no such request
    pos[1] = 10 ** 6            # past the table
    pt[req[2], pos[2] // k_pool.shape[1]] = 999   # page outside the pool
    k_out, _, flags = oracle.paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool)
    assert flags == 3
    P, ps, d = k_pool.shape
    ok = np.arange(len(req)) >= 2
    ok[ok] = pt[req[ok], pos[ok] // ps] < P     # the bad page skips every token on it
    assert ok.sum() > 0 and not ok[2]
    rows = pt[req[ok], pos[ok] // ps].astype(np.int64) * ps + pos[ok] % ps
    assert np.array_equal(k_out.reshape(P * ps, d)[rows], k_new[ok])
    written = np.zeros(P * ps, dtype=bool)
    written[rows] = True
    assert np.array_equal(k_out.reshape(P * ps, d)[~written], k_pool.reshape(P * ps, d)[~written])
