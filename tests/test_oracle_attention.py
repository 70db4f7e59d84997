"""Pins for the oracle's attention with sink, and for its exact merge.

What the method computes (page "Roadmap item 24 - joint compressed/window
attention with sink", section "Reuse and arithmetic"): compressed KV, the
recent window and a per-head sink share one softmax denominator; the sink
has no V; LSE is the natural log of that denominator. Each test below checks
the oracle against a route that does not run the oracle's own loop.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from tests._small import TAG, bits_to_f64, gather_rows, run_oracle, small_problem


def _sets(oracle, pr):
    return oracle.build_kv_sets(pr.pos, pr.W, pr.ratio, pr.topk if pr.ratio == 4 else None)


@pytest.mark.parametrize("ratio", [0, 4, 128])
def test_brute_force_dense_masked(oracle, ratio):
    """Full [keys + sink] logit matrix over every logical key of the
    request, -inf outside a mask built from positions, softmax by numpy."""
    pr = small_problem(seed=10 + ratio, ratio=ratio, S=300 if ratio == 128 else 40, ps=8 if ratio == 128 else 4)
    ip, idx = _sets(oracle, pr)
    O, L = run_oracle(oracle, pr, ip, idx)
    H, d = pr.q.shape[1], pr.q.shape[2]
    ps = pr.k_raw.shape[1]
    for i in range(pr.q.shape[0]):
        b, p = int(pr.req[i]), int(pr.pos[i])
        n_raw = pr.pt_raw.shape[1] * ps
        n_cmp = pr.pt_cmp.shape[1] * pr.k_cmp.shape[1]
        raw_keys = [TAG | t for t in range(n_raw)]
        cmp_keys = list(range(n_cmp))
        Kr, Vr = gather_rows(pr, b, raw_keys)
        Kc, Vc = gather_rows(pr, b, cmp_keys)
        mask_raw = np.array([(t <= p) and (p - t < pr.W) for t in range(n_raw)])
        picked = set(pr.topk[i].tolist()) if ratio == 4 else set(range(n_cmp))
        mask_cmp = np.array([ratio > 0 and (ratio * (g + 1) <= p + 1) and g in picked
                             for g in range(n_cmp)])
        Kall = np.concatenate([Kc, Kr])
        Vall = np.concatenate([Vc, Vr])
        mask = np.concatenate([mask_cmp, mask_raw])
        q = bits_to_f64(pr.q[i])                                   # [H, d]
        logits = pr.scale * q @ Kall.T                             # [H, all]
        logits[:, ~mask] = -np.inf
        full = np.concatenate([logits, pr.sink.astype(np.float64)[:, None]], axis=1)
        m = full.max(axis=1, keepdims=True)
        e = np.exp(full - m)
        P = e / e.sum(axis=1, keepdims=True)
        o_ref = P[:, :-1] @ Vall                                   # the sink column has no V
        lse_ref = (m[:, 0] + np.log(e.sum(axis=1)))
        np.testing.assert_allclose(O[i], o_ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(L[i], lse_ref, rtol=1e-12, atol=1e-12)


def _sdpa_with_sink(pr, i, keys, sink):
    """torch SDPA in float64: the set's keys plus one zero key whose value
    is zero; an additive mask puts sink_h on that key's logit (its scaled
    logit is exactly 0). LSE from torch.logsumexp over the same logits."""
    b = int(pr.req[i])
    K, V = gather_rows(pr, b, keys)
    H, d = pr.q.shape[1], pr.q.shape[2]
    q = torch.from_numpy(bits_to_f64(pr.q[i]))[:, None, :]                # [H,1,d]
    Kt = torch.from_numpy(np.concatenate([K, np.zeros((1, d))]))          # [n+1,d]
    Vt = torch.from_numpy(np.concatenate([V, np.zeros((1, d))]))
    mask = torch.zeros(H, 1, Kt.shape[0], dtype=torch.float64)
    mask[:, 0, -1] = torch.from_numpy(sink.astype(np.float64))
    o = F.scaled_dot_product_attention(q, Kt.expand(H, -1, -1), Vt.expand(H, -1, -1),
                                       attn_mask=mask, scale=pr.scale)
    logits = pr.scale * (q[:, 0, :] @ Kt.T) + mask[:, 0, :]
    return o[:, 0, :].numpy(), torch.logsumexp(logits, dim=1).numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_matches_sdpa_float64_with_sink_column(oracle, seed):
    pr = small_problem(seed=seed, H=8, d=64, S=48, W=16, K=6)
    ip, idx = _sets(oracle, pr)
    O, L = run_oracle(oracle, pr, ip, idx)
    for i in range(pr.q.shape[0]):
        o_ref, l_ref = _sdpa_with_sink(pr, i, idx[ip[i]:ip[i + 1]], pr.sink)
        np.testing.assert_allclose(O[i], o_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(L[i], l_ref, rtol=1e-12, atol=1e-12)


def test_sink_minus_inf_is_plain_softmax(oracle):
    pr = small_problem(seed=3, H=4, d=32)
    ip, idx = _sets(oracle, pr)
    sink = np.full(pr.q.shape[1], -np.inf, dtype=np.float32)
    O, L = run_oracle(oracle, pr, ip, idx, sink=sink)
    for i in range(pr.q.shape[0]):
        b = int(pr.req[i])
        K, V = gather_rows(pr, b, idx[ip[i]:ip[i + 1]])
        q = torch.from_numpy(bits_to_f64(pr.q[i]))[:, None, :]
        H = q.shape[0]
        o = F.scaled_dot_product_attention(q, torch.from_numpy(K).expand(H, -1, -1),
                                           torch.from_numpy(V).expand(H, -1, -1), scale=pr.scale)
        np.testing.assert_allclose(O[i], o[:, 0, :].numpy(), rtol=1e-10, atol=1e-12)
        lse = torch.logsumexp(pr.scale * q[:, 0, :] @ torch.from_numpy(K).T, dim=1).numpy()
        np.testing.assert_allclose(L[i], lse, rtol=1e-12, atol=1e-12)


def test_invariant_under_permuting_the_set(oracle):
    pr = small_problem(seed=4, H=4, d=32, S=60, W=20, K=8)
    ip, idx = _sets(oracle, pr)
    rng = np.random.default_rng(5)
    perm = idx.copy()
    for i in range(pr.q.shape[0]):
        perm[ip[i]:ip[i + 1]] = rng.permutation(idx[ip[i]:ip[i + 1]])
    O1, L1 = run_oracle(oracle, pr, ip, idx)
    O2, L2 = run_oracle(oracle, pr, ip, perm)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-12)


def test_closed_forms(oracle):
    """One key: O = v * sigmoid(s - sink), LSE = ln(e^s + e^sink).
    n identical keys: O = v * n e^s / (n e^s + e^sink)."""
    pr = small_problem(seed=6, B=1, S=8, H=3, d=8, W=1, ratio=0, ps=4)
    ip = np.array([0, 1], dtype=np.int32)
    i = 5
    rows = np.array([i], dtype=np.int32)
    for n in (1, 4):
        ipn = np.array([0] * (i + 1) + [n] * (pr.q.shape[0] - i), dtype=np.int32)
        idx = np.full(n, TAG | 2, dtype=np.int32)        # raw token 2, n times
        O, L = run_oracle(oracle, pr, ipn, idx, rows=rows)
        K, V = gather_rows(pr, 0, [TAG | 2])
        q = bits_to_f64(pr.q[i])
        s = pr.scale * q @ K[0]
        sink = pr.sink.astype(np.float64)
        w = n * np.exp(s) / (n * np.exp(s) + np.exp(sink))
        np.testing.assert_allclose(O[0], w[:, None] * V[0][None, :], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(L[0], np.log(n * np.exp(s) + np.exp(sink)), rtol=1e-13)
    del ip


def test_empty_set_gives_zero_output_and_sink_lse(oracle):
    pr = small_problem(seed=7, B=1, S=4, H=5, d=8, W=1, ratio=0)
    ip = np.zeros(pr.q.shape[0] + 1, dtype=np.int32)
    O, L = run_oracle(oracle, pr, ip, np.zeros(0, dtype=np.int32))
    assert np.all(O == 0)
    np.testing.assert_array_equal(L, np.broadcast_to(pr.sink.astype(np.float64), L.shape))


def _random_partition(rng, items, depth=0):
    """A random partition tree of `items` (a list of nested lists)."""
    if len(items) <= 1 or depth > 4 or rng.random() < 0.25:
        return items
    k = int(rng.integers(2, 4))
    cuts = np.sort(rng.choice(np.arange(1, len(items)), size=min(k - 1, len(items) - 1), replace=False))
    parts = np.split(np.asarray(items), cuts)
    return [_random_partition(rng, list(p), depth + 1) for p in parts]


def test_merge_lemma_over_random_partition_trees(oracle):
    """Merging LSE-weighted partials over any partition of the denominator
    equals the whole, to 1e-12 (docs: Block AttnRes model + ROCm-first plan,
    Summary; the sink is the part with O = 0 and LSE = sink)."""
    pr = small_problem(seed=8, H=3, d=16, S=64, W=24, K=10)
    ip, idx = _sets(oracle, pr)
    O, L = run_oracle(oracle, pr, ip, idx)
    rng = np.random.default_rng(9)
    N, H, d = pr.q.shape

    def partial(i, keys):
        ipn = np.zeros(N + 1, dtype=np.int32)
        ipn[i + 1:] = len(keys)
        o, l = run_oracle(oracle, pr, ipn, np.asarray(keys, dtype=np.int32),
                          rows=np.array([i], dtype=np.int32), include_sink=False)
        return o[0], l[0]

    def merge_tree(i, node, h):
        if node and not isinstance(node[0], list):       # a leaf: a set of keys
            o, l = partial(i, node)
            return o[h], l[h]
        parts = [merge_tree(i, c, h) for c in node]
        return oracle.lse_merge([p[1] for p in parts], np.stack([p[0] for p in parts]))

    for i in rng.choice(N, 12, replace=False):
        keys = list(idx[ip[i]:ip[i + 1]])
        tree = _random_partition(rng, keys)
        tree = tree if isinstance(tree[0], list) else [tree]
        for h in range(H):
            o_t, l_t = merge_tree(i, tree, h)
            o, l = oracle.lse_merge([l_t, float(pr.sink[h])], np.stack([o_t, np.zeros(d)]))
            np.testing.assert_allclose(o, O[i, h], rtol=0, atol=1e-12)
            assert abs(l - L[i, h]) <= 1e-12


def test_bad_page_and_bad_key_are_reported(oracle):
    pr = small_problem(seed=11)
    ip, idx = _sets(oracle, pr)
    bad = pr.pt_raw.copy()
    bad[0, 0] = 10 ** 6
    with pytest.raises(oracle.OracleError):
        oracle.sparse_sink_attn(pr.q, pr.k_raw, pr.v_raw, bad, pr.req, ip, idx, pr.sink, pr.scale,
                                k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp)
    idx2 = idx.copy()
    idx2[0] = -7
    with pytest.raises(oracle.OracleError):
        run_oracle(oracle, pr, ip, idx2)
