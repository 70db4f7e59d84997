"""Pins for the oracle's per-token KV-set builder (CPU only).

The set of a query at position p (page "Roadmap item 24 - joint
compressed/window attention with sink", section "Contracts and lifetime";
page "test: add block-level DeepSeek-V4 attention test", opening section):
the complete recent window of raw tokens plus the complete compressed groups
(top-k picked for ratio 4, all of them for ratio 128, none for ratio 0), in
canonical (ascending key) order.
"""
import json
import os

import numpy as np
import pytest

TAG = 1 << 30
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_test_set_sizes.json")


def _split(keys):
    keys = np.asarray(keys, dtype=np.int64)
    win = keys[(keys & TAG) != 0] & (TAG - 1)
    cmp_ = keys[(keys & TAG) == 0]
    return cmp_, win


def test_block_test_printed_set_sizes(oracle):
    """kv/token max, prefix and extend of the page's three prefill layers."""
    g = json.load(open(GOLDEN))
    for case in g["prefill"]:
        S, W, r = case["seqlen"], case["W"], case["ratio"]
        pos = np.arange(S, dtype=np.int32)
        topk = None
        if r == 4:
            # index_topk (512) exceeds every count of complete groups here,
            # so every group id is listed: the builder keeps the complete ones
            K = case["index_topk"]
            topk = np.full((S, K), -1, dtype=np.int32)
            topk[:, : S // r] = np.arange(S // r, dtype=np.int32)
        indptr, indices = oracle.build_kv_sets(pos, W, r, topk)
        sizes = np.diff(indptr)
        assert sizes.max() == case["kv_per_token_max"], case
        prefix = max(len(_split(indices[indptr[i]:indptr[i + 1]])[0]) for i in range(S))
        extend = max(len(_split(indices[indptr[i]:indptr[i + 1]])[1]) for i in range(S))
        assert prefix == case["prefix"] and extend == case["extend"], case


def test_block_test_truncation_case(oracle):
    """ctx 2560 at ratio 4: 640 committed groups, truncated to top-k 512."""
    t = json.load(open(GOLDEN))["truncation"]
    p = t["ctx"] - 1
    rng = np.random.default_rng(0)
    committed = np.arange(t["ctx"] // t["ratio"] + 5)   # include incomplete ids too
    indptr_all, idx_all = oracle.build_kv_sets([p], t["W"], t["ratio"], None)
    cmp_all, win = _split(idx_all)
    assert len(cmp_all) == t["committed_groups"]
    topk = rng.choice(committed, t["index_topk"], replace=False).astype(np.int32)[None]
    indptr, idx = oracle.build_kv_sets([p], t["W"], t["ratio"], topk)
    cmp_, win = _split(idx)
    expect = np.unique(topk[topk < t["committed_groups"]])
    assert np.array_equal(cmp_, expect)
    assert len(win) == t["W"]
    # with every pick complete the set holds exactly 512 + 128 = 640 entries
    topk = rng.choice(t["committed_groups"], t["index_topk"], replace=False).astype(np.int32)[None]
    indptr, idx = oracle.build_kv_sets([p], t["W"], t["ratio"], topk)
    assert indptr[-1] == t["index_topk"] + t["W"] == 640


@pytest.mark.parametrize("W", [1, 3, 64, 128])
def test_dense_window_is_the_analytic_window(oracle, W):
    """check_dense_window: ratio 0 gathers exactly the causal window."""
    pos = np.array([0, 1, 2, W - 1, W, W + 1, 5 * W + 3, 1000], dtype=np.int32)
    indptr, indices = oracle.build_kv_sets(pos, W, 0, None)
    for i, p in enumerate(pos):
        expect = np.arange(max(0, p - W + 1), p + 1) | TAG
        assert np.array_equal(indices[indptr[i]:indptr[i + 1]], expect)


def test_closed_form_counts(oracle):
    """|set| = min(p+1, W) + min(K, nc) (ratio 4, distinct complete picks
    covering min(K, nc) groups), min(p+1, W) + nc (ratio 128), min(p+1, W)."""
    rng = np.random.default_rng(1)
    pos = rng.integers(0, 6000, size=300).astype(np.int32)
    W, K = 128, 512
    topk = np.full((pos.size, K), -1, dtype=np.int32)
    for i, p in enumerate(pos):
        nc = (p + 1) // 4
        take = min(K, nc)
        topk[i, :take] = rng.choice(nc, take, replace=False)
    ip, _ = oracle.build_kv_sets(pos, W, 4, topk)
    nc4 = (pos.astype(np.int64) + 1) // 4
    assert np.array_equal(np.diff(ip), np.minimum(pos + 1, W) + np.minimum(K, nc4))
    ip, _ = oracle.build_kv_sets(pos, W, 128, None)
    assert np.array_equal(np.diff(ip), np.minimum(pos + 1, W) + (pos.astype(np.int64) + 1) // 128)
    ip, _ = oracle.build_kv_sets(pos, W, 0, None)
    assert np.array_equal(np.diff(ip), np.minimum(pos + 1, W))


def test_group_boundaries(oracle):
    """Group g (tokens 4g..4g+3) enters at p = 4g+3 and not before; a
    ratio-128 group enters at p = 128g+127."""
    for r in (4, 128):
        for g in range(3):
            last = r * g + r - 1
            for p, inside in ((last - 1, False), (last, True)):
                if p < 0:
                    continue
                topk = np.array([[g]], dtype=np.int32) if r == 4 else None
                ip, idx = oracle.build_kv_sets([p], 8, r, topk)
                cmp_, _ = _split(idx)
                assert (g in cmp_) == inside, (r, g, p)


def test_invalid_and_repeated_topk_entries(oracle):
    """-1 padding, incomplete, negative and repeated ids are dropped; the
    rest appear once, ascending, before the window."""
    topk = np.array([[7, -1, 3, 3, 250, 7, 0, -5, 63, 64]], dtype=np.int32)
    ip, idx = oracle.build_kv_sets([255], 4, 4, topk)
    assert list(idx[:4]) == [0, 3, 7, 63]
    assert list(idx[4:]) == [TAG | t for t in range(252, 256)]


def _naive_sets(pos, W, ratio, topk):
    """A second route: a boolean mask over every possible key."""
    out = []
    for i, p in enumerate(pos):
        keys = []
        max_g = p + 2
        for g in range(max_g):
            complete = ratio > 0 and all(t <= p for t in range(ratio * g, ratio * g + ratio))
            picked = topk is None or g in set(topk[i].tolist())
            if complete and picked:
                keys.append(g)
        for t in range(p + 1):
            if p - t < W:
                keys.append(TAG | t)
        out.append(keys)
    return out


@pytest.mark.parametrize("ratio,use_topk", [(0, False), (4, True), (4, False), (128, False)])
def test_brute_force_tiny(oracle, ratio, use_topk):
    rng = np.random.default_rng(2 + ratio)
    pos = rng.integers(0, 300, size=40).astype(np.int32)
    pos[:3] = [0, 1, 299]
    W = 17
    topk = None
    if use_topk:
        topk = rng.integers(-1, 90, size=(pos.size, 12)).astype(np.int32)
    ip, idx = oracle.build_kv_sets(pos, W, ratio, topk)
    naive = _naive_sets(pos.tolist(), W, ratio, topk)
    for i in range(pos.size):
        assert list(idx[ip[i]:ip[i + 1]]) == naive[i]


def test_invariants(oracle):
    rng = np.random.default_rng(3)
    pos = rng.integers(0, 5000, size=500).astype(np.int32)
    topk = rng.integers(-1, 1300, size=(pos.size, 64)).astype(np.int32)
    ip, idx = oracle.build_kv_sets(pos, 100, 4, topk)
    assert ip[0] == 0 and np.all(np.diff(ip) >= 1) and ip[-1] == idx.size
    for i, p in enumerate(pos):
        row = idx[ip[i]:ip[i + 1]].astype(np.int64)
        assert np.all(np.diff(row) > 0)                      # strictly ascending
        cmp_, win = _split(row)
        assert np.all(4 * (cmp_ + 1) <= p + 1)                # complete groups only
        assert np.all((win <= p) & (win > p - 100))           # inside the window


def test_empty_batch_and_errors(oracle):
    ip, idx = oracle.build_kv_sets(np.zeros(0, dtype=np.int32), 8, 4, np.zeros((0, 4), dtype=np.int32))
    assert ip.tolist() == [0] and idx.size == 0
    with pytest.raises(oracle.OracleError):
        oracle.build_kv_sets([-1], 8, 0, None)
    with pytest.raises(oracle.OracleError):
        oracle.build_kv_sets([5], 8, 3, None)
