"""Pins for the oracle's backward of the attention with sink.

The backward is the follow-on item of page "Roadmap item 24 - joint
compressed/window attention with sink" (dQ, dK/dV scattered to pages,
d_sink, from the saved O and LSE). The oracle computes the gradients of
L = sum(dO * O) in FP64 from the chain rule; each test checks them by a
route that does not run that loop: torch autograd through a float64
softmax with a sink column, central finite differences of a numpy forward,
closed forms and invariants of the softmax.
"""
import numpy as np
import pytest
import torch

from tests._small import TAG, bf16_bits, bits_to_f64, small_problem


def _sets(oracle, pr):
    return oracle.build_kv_sets(pr.pos, pr.W, pr.ratio, pr.topk if pr.ratio == 4 else None)


def _dout(pr, seed):
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal(pr.q.shape))


def _bwd(oracle, pr, ip, idx, dout, sink=None, rows=None):
    return oracle.sparse_sink_attn_bwd(
        pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx,
        pr.sink if sink is None else sink, pr.scale, dout,
        k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, rows=rows, threads=2)


def _row_of(pr, b, key):
    """(is_raw, flat pool row) of one key of request b, by page table."""
    if key & TAG:
        t, pool, pt = key & (TAG - 1), pr.k_raw, pr.pt_raw
    else:
        t, pool, pt = key, pr.k_cmp, pr.pt_cmp
    ps = pool.shape[1]
    return bool(key & TAG), int(pt[b, t // ps]) * ps + t % ps


def _autograd(pr, ip, idx, dout, sink):
    """Gradients by torch autograd: per query, gather the set's rows from
    the flattened pools by index, softmax over [logits, sink] in float64,
    O = P[:, :-1] V, loss = sum(dO * O)."""
    H, d = pr.q.shape[1], pr.q.shape[2]
    q = torch.tensor(bits_to_f64(pr.q), requires_grad=True)
    pools = {name: torch.tensor(bits_to_f64(getattr(pr, name)).reshape(-1, d), requires_grad=True)
             for name in ("k_raw", "v_raw", "k_cmp", "v_cmp")}
    s = torch.tensor(sink.astype(np.float64), requires_grad=True)
    dO = torch.tensor(bits_to_f64(dout))
    loss = torch.zeros((), dtype=torch.float64)
    for i in range(pr.q.shape[0]):
        b = int(pr.req[i])
        keys = idx[ip[i]:ip[i + 1]]
        Ks, Vs = [], []
        for key in keys:
            raw, row = _row_of(pr, b, int(key))
            Ks.append(pools["k_raw" if raw else "k_cmp"][row])
            Vs.append(pools["v_raw" if raw else "v_cmp"][row])
        K = torch.stack(Ks) if Ks else torch.zeros((0, d), dtype=torch.float64)
        V = torch.stack(Vs) if Vs else torch.zeros((0, d), dtype=torch.float64)
        logits = torch.cat([pr.scale * q[i] @ K.T, s[:, None]], dim=1)     # [H, n+1]
        P = torch.softmax(logits, dim=1)
        O = P[:, :-1] @ V
        loss = loss + (dO[i] * O).sum()
    loss.backward()
    g = lambda t: np.zeros(tuple(t.shape)) if t.grad is None else t.grad.numpy()   # noqa: E731
    return (g(q), g(pools["k_raw"]), g(pools["v_raw"]), g(pools["k_cmp"]), g(pools["v_cmp"]), g(s))


@pytest.mark.parametrize("ratio,seed", [(4, 0), (128, 1), (0, 2)])
def test_matches_torch_autograd(oracle, ratio, seed):
    pr = small_problem(seed=20 + seed, ratio=ratio, S=300 if ratio == 128 else 40,
                       ps=8 if ratio == 128 else 4, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, seed)
    dq, dkr, dvr, dkc, dvc, ds = _bwd(oracle, pr, ip, idx, dout)
    r = _autograd(pr, ip, idx, dout, pr.sink)
    d = pr.q.shape[2]
    for got, ref in zip((dq, dkr.reshape(-1, d), dvr.reshape(-1, d), dkc.reshape(-1, d),
                         dvc.reshape(-1, d), ds), r):
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-11)


def _numpy_loss(pr, ip, idx, dout, q, k_raw, v_raw, k_cmp, v_cmp, sink):
    """sum(dO * O) by a dense numpy forward over the listed keys."""
    total = 0.0
    dO = bits_to_f64(dout)
    for i in range(q.shape[0]):
        b = int(pr.req[i])
        rows = [_row_of(pr, b, int(key)) for key in idx[ip[i]:ip[i + 1]]]
        d = q.shape[2]
        K = np.array([(k_raw if raw else k_cmp).reshape(-1, d)[row] for raw, row in rows]).reshape(-1, d)
        V = np.array([(v_raw if raw else v_cmp).reshape(-1, d)[row] for raw, row in rows]).reshape(-1, d)
        logits = np.concatenate([pr.scale * q[i] @ K.T, sink[:, None]], axis=1)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        P = e / e.sum(axis=1, keepdims=True)
        total += float((dO[i] * (P[:, :-1] @ V)).sum())
    return total


def test_central_differences(oracle):
    """A handful of entries of every gradient against central differences
    (step 1e-6) of a numpy forward at the BF16 inputs."""
    pr = small_problem(seed=31, S=24, H=3, d=8, W=6, K=3)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 5)
    dq, dkr, dvr, dkc, dvc, ds = _bwd(oracle, pr, ip, idx, dout)
    base = {"q": bits_to_f64(pr.q), "k_raw": bits_to_f64(pr.k_raw), "v_raw": bits_to_f64(pr.v_raw),
            "k_cmp": bits_to_f64(pr.k_cmp), "v_cmp": bits_to_f64(pr.v_cmp),
            "sink": pr.sink.astype(np.float64)}
    grads = {"q": dq, "k_raw": dkr, "v_raw": dvr, "k_cmp": dkc, "v_cmp": dvc, "sink": ds}
    rng = np.random.default_rng(7)
    eps = 1e-6
    for name, g in grads.items():
        flat = g.reshape(-1)
        # entries with a gradient (rows some set uses) and a couple of random ones
        nz = np.flatnonzero(np.abs(flat) > 1e-3)
        picks = list(rng.choice(nz, size=min(4, nz.size), replace=False)) + list(rng.integers(0, flat.size, 2))
        for e in picks:
            vals = []
            for sgn in (+1, -1):
                args = {k: v.copy() for k, v in base.items()}
                args[name].reshape(-1)[e] += sgn * eps
                vals.append(_numpy_loss(pr, ip, idx, dout, **args))
            fd = (vals[0] - vals[1]) / (2 * eps)
            assert abs(fd - flat[e]) <= 1e-6 * (1 + abs(fd)), (name, e, fd, flat[e])


def test_single_key_closed_form(oracle):
    """One key, no sink: P = 1, so dS = 0 (dq = dk = 0) and dv = sum_h dO_h."""
    pr = small_problem(seed=4, S=8, H=3, d=8, W=1, ratio=0)
    ip, idx = _sets(oracle, pr)
    assert np.all(np.diff(ip) == 1)
    dout = _dout(pr, 1)
    sink = np.full(pr.q.shape[1], -np.inf, dtype=np.float32)
    dq, dkr, dvr, dkc, dvc, ds = _bwd(oracle, pr, ip, idx, dout, sink=sink)
    assert np.all(dq == 0) and np.all(dkr == 0) and np.all(ds == 0)
    d = pr.q.shape[2]
    ref = np.zeros_like(dvr.reshape(-1, d))
    dO = bits_to_f64(dout)
    for i in range(pr.q.shape[0]):
        _, row = _row_of(pr, int(pr.req[i]), int(idx[ip[i]]))
        ref[row] += dO[i].sum(axis=0)
    np.testing.assert_allclose(dvr.reshape(-1, d), ref, rtol=1e-14, atol=1e-14)


def test_sum_of_dv_is_the_non_sink_mass(oracle):
    """sum over every pool row of dv = sum_{i,h} (1 - e^{sink_h - LSE_ih}) dO_ih,
    LSE from the forward oracle."""
    pr = small_problem(seed=8, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 2)
    _, _, dvr, _, dvc, _ = _bwd(oracle, pr, ip, idx, dout)
    _, lse = oracle.sparse_sink_attn(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink,
                                     pr.scale, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, threads=2)
    w = 1.0 - np.exp(pr.sink.astype(np.float64)[None, :] - lse)            # [N, H]
    ref = (w[:, :, None] * bits_to_f64(dout)).sum(axis=(0, 1))
    d = pr.q.shape[2]
    got = dvr.reshape(-1, d).sum(axis=0) + dvc.reshape(-1, d).sum(axis=0)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_key_shift_invariance_without_sink(oracle):
    """Without a sink, adding one vector to every K row leaves every softmax
    unchanged, so the dk of all rows sums to zero."""
    pr = small_problem(seed=9, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    sink = np.full(pr.q.shape[1], -np.inf, dtype=np.float32)
    _, dkr, _, dkc, _, ds = _bwd(oracle, pr, ip, idx, _dout(pr, 3), sink=sink)
    d = pr.q.shape[2]
    total = dkr.reshape(-1, d).sum(axis=0) + dkc.reshape(-1, d).sum(axis=0)
    scale_ref = np.abs(dkr).max()
    assert scale_ref > 1e-3
    np.testing.assert_allclose(total, 0.0, atol=1e-12 * max(1.0, scale_ref * 100))
    assert np.all(ds == 0)


def test_sink_gradient_balances_the_logit_gradients(oracle):
    """Adding one constant to every logit of a (query, head) and to its sink
    changes nothing, so d_sink_h = -sum_j dL/ds_j. With the keys the d unit
    vectors, s_j = scale * q_j, so dL/ds_j = dq_j / scale and the sum of a
    head's dq over its d entries is -scale * d_sink_h."""
    # one query, H heads, keys = the d unit vectors: then s_j = scale * q_j
    # and dL/dq_j = scale * dL/ds_j, so sum_j dq_j / scale = -d_sink
    rng = np.random.default_rng(12)
    H, d = 3, 8
    q = bf16_bits(rng.standard_normal((1, H, d)))
    k = np.zeros((1, d, d), dtype=np.float32)
    for j in range(d):
        k[0, j, j] = 1.0
    k_raw = bf16_bits(k)
    v_raw = bf16_bits(rng.standard_normal((1, d, d)))
    pt_raw = np.zeros((1, 1), dtype=np.int32)
    req = np.zeros(1, dtype=np.int32)
    indptr = np.array([0, d], dtype=np.int32)
    indices = np.array([TAG | t for t in range(d)], dtype=np.int32)
    sink = rng.standard_normal(H).astype(np.float32)
    dout = bf16_bits(rng.standard_normal((1, H, d)))
    scale = 0.37
    dq, _, _, _, _, ds = oracle.sparse_sink_attn_bwd(q, k_raw, v_raw, pt_raw, req, indptr, indices,
                                                     sink, scale, dout, threads=1)
    np.testing.assert_allclose(dq[0].sum(axis=1) / scale, -ds, rtol=1e-12, atol=1e-13)


def test_rows_partition_adds_up(oracle):
    """Gradients of a partition of the query tokens add up to the whole (dk,
    dv, dsink) and dq rows are the whole's rows."""
    pr = small_problem(seed=13, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 4)
    full = _bwd(oracle, pr, ip, idx, dout)
    N = pr.q.shape[0]
    perm = np.random.default_rng(0).permutation(N).astype(np.int32)
    a, b = perm[: N // 3], perm[N // 3:]
    pa = _bwd(oracle, pr, ip, idx, dout, rows=a)
    pb = _bwd(oracle, pr, ip, idx, dout, rows=b)
    np.testing.assert_allclose(pa[0], full[0][a], rtol=0, atol=0)
    for k in range(1, 6):
        np.testing.assert_allclose(pa[k] + pb[k], full[k], rtol=1e-12, atol=1e-12)


def test_empty_set_has_no_gradient(oracle):
    """A token whose set is empty: O = 0 and LSE = sink, so D = 0 and every
    gradient of that token is zero."""
    pr = small_problem(seed=14, S=12, H=2, d=8)
    ip, idx = _sets(oracle, pr)
    N = pr.q.shape[0]
    ip0 = np.zeros(N + 1, dtype=np.int32)
    dq, dkr, dvr, dkc, dvc, ds = _bwd(oracle, pr, ip0, idx[:0], _dout(pr, 6))
    assert np.all(dq == 0) and np.all(dkr == 0) and np.all(dvr == 0) and np.all(ds == 0)


def _fwd(oracle, pr, ip, idx, v_raw=None, v_cmp=None):
    return oracle.sparse_sink_attn(pr.q, pr.k_raw, pr.v_raw if v_raw is None else v_raw, pr.pt_raw, pr.req,
                                   ip, idx, pr.sink, pr.scale, k_cmp=pr.k_cmp,
                                   v_cmp=pr.v_cmp if v_cmp is None else v_cmp, pt_cmp=pr.pt_cmp, threads=2)


def test_saved_results_equal_to_the_exact_ones_change_nothing(oracle):
    pr = small_problem(seed=15, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 7)
    O, L = _fwd(oracle, pr, ip, idx)
    exact = _bwd(oracle, pr, ip, idx, dout)
    saved = oracle.sparse_sink_attn_bwd(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink, pr.scale,
                                        dout, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, threads=2,
                                        o_saved=O, lse_saved=L)
    for a, b in zip(exact, saved):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_saved_o_enters_only_through_d(oracle):
    """O_saved = O + delta moves D by dO . delta, so dq moves by
    -scale (dO . delta) sum_j p_j k_j (that sum is the forward with V := K),
    dsink by -sum_i p_sink (dO . delta), and dv not at all."""
    pr = small_problem(seed=16, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 8)
    O, L = _fwd(oracle, pr, ip, idx)
    delta = 1e-2 * np.random.default_rng(3).standard_normal(O.shape)
    base = oracle.sparse_sink_attn_bwd(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink, pr.scale,
                                       dout, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, threads=2,
                                       o_saved=O, lse_saved=L)
    moved = oracle.sparse_sink_attn_bwd(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink, pr.scale,
                                        dout, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, threads=2,
                                        o_saved=O + delta, lse_saved=L)
    dD = (bits_to_f64(dout) * delta).sum(axis=2)                                 # [N, H]
    PK, _ = _fwd(oracle, pr, ip, idx, v_raw=pr.k_raw, v_cmp=pr.k_cmp)             # sum_j p_j k_j
    np.testing.assert_allclose(moved[0] - base[0], -pr.scale * dD[:, :, None] * PK, rtol=1e-9, atol=1e-13)
    p_sink = np.exp(pr.sink.astype(np.float64)[None, :] - L)
    np.testing.assert_allclose(moved[5] - base[5], -(p_sink * dD).sum(axis=0), rtol=1e-9, atol=1e-13)
    # dv does not depend on O: identical sums (added in query order)
    np.testing.assert_array_equal(moved[2], base[2])
    np.testing.assert_array_equal(moved[4], base[4])


def test_saved_lse_scales_every_gradient(oracle):
    """With O_saved fixed, every gradient is linear in the probabilities, so
    LSE_saved = LSE + c multiplies all of them by e^-c."""
    pr = small_problem(seed=17, S=40, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 9)
    O, L = _fwd(oracle, pr, ip, idx)
    c = 0.3
    base, shifted = [oracle.sparse_sink_attn_bwd(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink,
                                                 pr.scale, dout, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp,
                                                 threads=2, o_saved=O, lse_saved=L + sh) for sh in (0.0, c)]
    for a, b in zip(base, shifted):
        np.testing.assert_allclose(b, np.exp(-c) * a, rtol=1e-12, atol=1e-14)


def test_sums_do_not_depend_on_the_thread_count(oracle):
    """The per-query contributions to the pool-shaped dk/dv and to dsink are
    added in query order, so one thread and several give identical sums."""
    pr = small_problem(seed=18, S=48, H=4, d=16)
    ip, idx = _sets(oracle, pr)
    dout = _dout(pr, 9)
    runs = [oracle.sparse_sink_attn_bwd(pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, ip, idx, pr.sink, pr.scale,
                                        dout, k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, threads=t)
            for t in (1, 3, 8)]
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            np.testing.assert_array_equal(a, b)
