"""GPU parity: the CUDA path against the FP64 oracle on identical seeded inputs.

Bar (stated by the method's tolerance for this path):
  * CSR key sets: bit-exact (indptr and indices);
  * FP8 page decode: bit-exact BF16;
  * O: |O - ref| <= 1e-2 * (1 + |ref|) for every element, zero failures;
  * LSE: |LSE - ref| <= 2e-3 for every (query, head).
The oracle builds its own key sets and decodes its own pages: nothing it
consumes comes from the CUDA path.
"""
import functools

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

O_RTOL = 1e-2
LSE_ATOL = 2e-3


@pytest.fixture(scope="module")
def spa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_paged_attention_build_b200 as m
    return m


@functools.lru_cache(maxsize=None)
def workload(name, shrink=1, fp8_format=0):
    from sparse_paged_attention_build_b200 import workloads
    return workloads.make(name, shrink=shrink, fp8_format=fp8_format)


@functools.lru_cache(maxsize=None)
def oracle_sets(name, shrink=1):
    import oracle
    w = workload(name, shrink)
    return oracle.build_kv_sets(w.pos, w.W, w.ratio, w.topk)


@functools.lru_cache(maxsize=None)
def oracle_cmp_pools(name, shrink=1, fp8_format=0):
    import oracle
    w = workload(name, shrink, fp8_format)
    if w.k_cmp_fp8 is None:
        return w.k_cmp, w.v_cmp
    k = oracle.dequant_fp8_pages(w.k_cmp_fp8, w.k_cmp_scale, w.cmp_page_ids, fmt=fp8_format)
    v = oracle.dequant_fp8_pages(w.v_cmp_fp8, w.v_cmp_scale, w.cmp_page_ids, fmt=fp8_format)
    return k, v


def oracle_attn(name, shrink, rows, fp8_format=0):
    import oracle
    w = workload(name, shrink, fp8_format)
    ip, idx = oracle_sets(name, shrink)
    k_cmp, v_cmp = oracle_cmp_pools(name, shrink, fp8_format)
    return oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, w.sink, w.scale,
                                   k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp,
                                   rows=None if rows is None else np.asarray(rows, dtype=np.int32))


def check_attn(out, lse, O_ref, L_ref, what):
    o = out.float().cpu().double().numpy()
    l_ = lse.cpu().double().numpy()
    err = np.abs(o - O_ref)
    bad = err > O_RTOL * (1.0 + np.abs(O_ref))
    assert not bad.any(), f"{what}: {bad.sum()} O elements out of tolerance, max err {err.max():.3g}"
    lerr = np.abs(l_ - L_ref)
    assert (lerr <= LSE_ATOL).all(), f"{what}: LSE max err {lerr.max():.3g}"
    return float(err.max()), float(lerr.max())


def batch(spa, name, shrink=1, num_splits=0):
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    return DeviceBatch(workload(name, shrink), num_splits=num_splits)


def sample_rows(w, n_random=48, seed=0):
    """Boundary rows of every request -- the window filling up (p = W-1, W),
    the first tile boundaries, the top-k starting to truncate (the complete
    groups outnumbering K: p = 4K-1 .. 4K+3 at ratio 4), the last tokens --
    plus n_random rows drawn uniformly."""
    rng = np.random.default_rng(seed)
    N = w.N
    rows = {0, 1, N - 1, N - 2}
    bounds = [w.W - 2, w.W - 1, w.W, w.W + 1, 63, 64, 127, 4 * 64 - 1, 2047, 2048, 2559]
    if w.ratio > 0 and w.K > 0:
        bounds += list(range(w.ratio * w.K - 2, w.ratio * w.K + w.ratio + 1))
    for p in bounds:
        hits = np.nonzero(w.pos == p)[0]
        rows.update(hits.tolist())   # every request
    rows.update(rng.choice(N, size=min(N, n_random), replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int32)


# ------------------------------------------------------------------ sets
@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_kv_sets_bit_exact_full_size(spa, name):
    b = batch(spa, name)
    b.build_sets()
    torch.cuda.synchronize()
    ip, idx = oracle_sets(name)
    got_ip = b.indptr.cpu().numpy()
    assert np.array_equal(got_ip, ip)
    assert np.array_equal(b.indices[: ip[-1]].cpu().numpy(), idx)
    assert b.status_word() == 0


def test_kv_sets_edge_cases(spa):
    import oracle
    rng = np.random.default_rng(5)
    # positions past 65535 have more than 16384 complete ratio-4 groups: the
    # builder's bitmap is too small for them and it sorts instead
    pos = np.concatenate([[0, 1, 2, 3, 4, 127, 128, 129, 4095, 65535, 65536, 65539],
                          rng.integers(0, 9000, 300), rng.integers(60000, 140000, 40)]).astype(np.int32)
    for K in (1, 5, 32, 33, 512, 2048):
        topk = rng.integers(-3, 2300, size=(pos.size, K)).astype(np.int32)
        far = pos >= 60000
        topk[far] = rng.integers(-3, 36000, size=(int(far.sum()), K))
        topk[:, : K // 2] = topk[:, :1]           # many repeats
        for ratio, W in ((4, 128), (4, 1), (128, 7), (0, 64)):
            t = torch.from_numpy(topk).cuda() if ratio == 4 else None
            st = spa.new_status()
            ip_g, idx_g = spa.build_kv_sets(torch.from_numpy(pos).cuda(), W, ratio, t,
                                            max_pos=int(pos.max()), dev_status=st)
            ip, idx = oracle.build_kv_sets(pos, W, ratio, topk if ratio == 4 else None)
            assert np.array_equal(ip_g.cpu().numpy(), ip), (K, ratio, W)
            assert np.array_equal(idx_g[: ip[-1]].cpu().numpy(), idx), (K, ratio, W)
            assert spa.read_status(st) == 0


def test_kv_sets_empty_and_faults(spa):
    ip, idx = spa.build_kv_sets(torch.zeros(0, dtype=torch.int32, device="cuda"), 8, 4, None, capacity=0)
    assert ip.cpu().tolist() == [0]
    # a negative position is reported and gets an empty set
    st = spa.new_status()
    pos = torch.tensor([5, -1, 7], dtype=torch.int32, device="cuda")
    ip, idx = spa.build_kv_sets(pos, 4, 0, None, capacity=100, dev_status=st)
    assert spa.read_status(st) & spa.DEV_BAD_INDEX
    assert ip.cpu().tolist() == [0, 4, 4, 8]
    # capacity overflow is reported, nothing is written past it
    st = spa.new_status()
    idx = torch.full((10,), -7, dtype=torch.int32, device="cuda")
    pos = torch.tensor([50, 60, 70], dtype=torch.int32, device="cuda")
    spa.build_kv_sets(pos, 8, 0, None, capacity=9, indices=idx, dev_status=st)
    assert spa.read_status(st) & spa.DEV_CAPACITY
    assert idx[9].item() == -7


# ------------------------------------------------------------------ dequant
@pytest.mark.parametrize("shrink", [16, 1])
def test_dequant_bit_exact(spa, shrink):
    b = batch(spa, "c5", shrink)
    b.dequant()
    torch.cuda.synchronize()
    k_ref, v_ref = oracle_cmp_pools("c5", shrink)
    got_k = b.k_cmp.view(torch.int16).cpu().numpy().view(np.uint16)
    got_v = b.v_cmp.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got_k, k_ref)
    assert np.array_equal(got_v, v_ref)
    assert b.status_word() == 0


def test_dequant_every_code_and_bad_page(spa):
    import oracle
    P, ps, d = 4, 16, 128
    src = np.arange(P * ps * d, dtype=np.int64).reshape(P, ps, d) % 256
    src = src.astype(np.uint8)
    rng = np.random.default_rng(2)
    scales = (rng.random((P, ps, d // 64)) * 4).astype(np.float32)
    scales[0, 0, 0] = 1e-40    # subnormal products
    scales[0, 0, 1] = 3e38     # overflow to inf
    ids = np.array([0, 2, 3], dtype=np.int32)
    ref = oracle.dequant_fp8_pages(src, scales, ids)
    dst = torch.zeros((P, ps, d), dtype=torch.bfloat16, device="cuda")
    st = spa.new_status()
    spa.dequant_fp8_pages(torch.from_numpy(src).cuda(), torch.from_numpy(scales).cuda(),
                          torch.from_numpy(ids).cuda(), dst, dev_status=st)
    got = dst.view(torch.int16).cpu().numpy().view(np.uint16)
    nan_ref = (ref & 0x7fff) > 0x7f80
    nan_got = (got & 0x7fff) > 0x7f80
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])
    assert spa.read_status(st) == 0
    bad = torch.tensor([1, 99], dtype=torch.int32, device="cuda")
    spa.dequant_fp8_pages(torch.from_numpy(src).cuda(), torch.from_numpy(scales).cuda(), bad, dst, dev_status=st)
    assert spa.read_status(st) & spa.DEV_BAD_PAGE


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("name,shrink", [("c1", 1), ("c2", 8), ("c3", 16), ("c4", 16), ("c5", 16)])
def test_attention_every_element_small(spa, name, shrink):
    b = batch(spa, name, shrink)
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    O, L = oracle_attn(name, shrink, None)
    check_attn(b.out, b.lse, O, L, f"{name}/{shrink}")


@pytest.mark.parametrize("name", ["c2", "c3", "c4", "c5"])
def test_attention_full_size_sampled(spa, name):
    """Full-size inputs in the launch configuration the benchmark times
    (automatic split count); sampled rows against the oracle."""
    b = batch(spa, name)
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    w = workload(name)
    # a few thousand prefill rows: the oracle runs at about 5e7 pairs/s
    rows = np.arange(w.N, dtype=np.int32) if w.kind == "decode" else sample_rows(w, n_random=2048)
    O, L = oracle_attn(name, 1, rows)
    check_attn(b.out[torch.from_numpy(rows).long().cuda()], b.lse[torch.from_numpy(rows).long().cuda()],
               O, L, name)


@pytest.mark.parametrize("splits", [1, 2, 3, 4, 5, 6, 7, 8, 9, 16])
def test_attention_split_counts(spa, splits):
    b = batch(spa, "c4", 8, num_splits=splits)
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    O, L = oracle_attn("c4", 8, None)
    check_attn(b.out, b.lse, O, L, f"splits={splits}")


def test_attention_no_sink_and_empty_sets(spa):
    import oracle
    w = workload("c1")
    b = batch(spa, "c1")
    b.build_sets()
    ip, idx = oracle_sets("c1")
    # empty every third set: indptr with repeated entries, keys dropped
    keep = np.ones(w.N, dtype=bool)
    keep[::3] = False
    sizes = np.diff(ip) * keep
    ip2 = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    idx2 = np.concatenate([idx[ip[i]:ip[i + 1]] for i in range(w.N) if keep[i]]).astype(np.int32)
    for sink in (w.sink, None):
        st = spa.new_status()
        out, lse = spa.sparse_sink_attn_fwd(
            b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, torch.from_numpy(ip2).cuda(),
            torch.from_numpy(idx2).cuda(), None if sink is None else b.sink, w.scale,
            k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp, dev_status=st)
        torch.cuda.synchronize()
        assert spa.read_status(st) == 0
        s = np.full(w.H, -np.inf, dtype=np.float32) if sink is None else w.sink
        O, L = oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip2, idx2, s, w.scale,
                                       k_cmp=w.k_cmp, v_cmp=w.v_cmp, pt_cmp=w.pt_cmp)
        o = out.float().cpu().double().numpy()
        l_ = lse.cpu().double().numpy()
        empty = ~keep
        assert np.all(o[empty] == 0)
        if sink is None:
            assert np.all(np.isneginf(l_[empty]))
            check_attn(out[torch.from_numpy(keep).cuda()], lse[torch.from_numpy(keep).cuda()],
                       O[keep], L[keep], "no sink")
        else:
            check_attn(out, lse, O, L, "empty sets")


def test_attention_bad_page_is_reported_not_trapped(spa):
    w = workload("c1")
    b = batch(spa, "c1")
    b.build_sets()
    pt = b.pt_raw.clone()
    pt[0, 0] = 10 ** 7
    st = spa.new_status()
    spa.sparse_sink_attn_fwd(b.q, b.k_raw, b.v_raw, pt, b.req, b.indptr, b.indices, b.sink, w.scale,
                             k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp, dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) & spa.DEV_BAD_PAGE
    # the context is still usable
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0


def test_pool_beyond_2GiB_uses_64bit_addressing(spa):
    """Rows placed past byte 2^31 of a >2 GiB pool are read correctly."""
    import oracle
    w = workload("c1")
    ps, d = w.k_raw.shape[1], w.k_raw.shape[2]
    page_bytes = ps * d * 2
    big_pages = (2 ** 31 + 2 ** 26) // page_bytes + w.k_raw.shape[0]
    shift = big_pages - w.k_raw.shape[0]
    k_big = torch.zeros((big_pages, ps, d), dtype=torch.bfloat16, device="cuda")
    v_big = torch.zeros_like(k_big)
    b = batch(spa, "c1")
    k_big[shift:] = b.k_raw
    v_big[shift:] = b.v_raw
    pt = (b.pt_raw + shift).contiguous()
    b.build_sets()
    st = spa.new_status()
    out, lse = spa.sparse_sink_attn_fwd(b.q, k_big, v_big, pt, b.req, b.indptr, b.indices, b.sink,
                                        w.scale, k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp,
                                        dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) == 0
    O, L = oracle_attn("c1", 1, None)
    check_attn(out, lse, O, L, ">2GiB pool")
    del k_big, v_big


# ------------------------------------------------------------------ fused FP8
def fp8_batches(name, shrink, num_splits=0):
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workload(name, shrink)
    return (w, DeviceBatch(w, num_splits=num_splits, fp8_path="decode"),
            DeviceBatch(w, num_splits=num_splits, fp8_path="fused"))


def assert_bit_identical(a_out, a_lse, b_out, b_lse, what):
    assert torch.equal(a_out.view(torch.int16), b_out.view(torch.int16)), f"{what}: O differs"
    assert torch.equal(a_lse.view(torch.int32), b_lse.view(torch.int32)), f"{what}: LSE differs"


@pytest.mark.parametrize("shrink,splits", [(32, 0), (8, 0), (8, 3)])
def test_fused_fp8_gather_bit_identical_to_page_decode(spa, shrink, splits):
    """Decoding the compressed rows inside the gather gives exactly the
    result of decoding the pages first (same BF16 operands, same kernel)."""
    w, dec, fus = fp8_batches("c5", shrink, splits)
    dec.step()
    fus.step()
    torch.cuda.synchronize()
    assert dec.status_word() == 0 and fus.status_word() == 0
    assert fus.kernels_per_step() == 2
    assert_bit_identical(dec.out, dec.lse, fus.out, fus.lse, f"c5/{shrink} splits={splits}")
    O, L = oracle_attn("c5", shrink, None)
    check_attn(fus.out, fus.lse, O, L, f"fused c5/{shrink}")


@pytest.mark.parametrize("fmt,splits", [(0, 0), (1, 2)])
def test_fused_fp8_gather_head_dim_64(spa, fmt, splits):
    """The FP8 gather at d = 64 (one 64-code piece group per row, one scale):
    bit-identical to decoding the pages first, and within tolerance of the
    oracle on every element."""
    import oracle
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workloads._decode("fp8-d64", 23, 16, np.full(16, 4096), 16, 64, 64, 4, 128, 64, fp8=True, fmt=fmt)
    dec = DeviceBatch(w, num_splits=splits, fp8_path="decode")
    fus = DeviceBatch(w, num_splits=splits, fp8_path="fused")
    dec.step()
    fus.step()
    torch.cuda.synchronize()
    assert dec.status_word() == 0 and fus.status_word() == 0
    assert_bit_identical(dec.out, dec.lse, fus.out, fus.lse, f"d64 FP8 format {fmt} splits={splits}")
    k = oracle.dequant_fp8_pages(w.k_cmp_fp8, w.k_cmp_scale, w.cmp_page_ids, fmt=fmt)
    v = oracle.dequant_fp8_pages(w.v_cmp_fp8, w.v_cmp_scale, w.cmp_page_ids, fmt=fmt)
    ip, idx = oracle.build_kv_sets(w.pos, w.W, w.ratio, w.topk)
    O, L = oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, w.sink, w.scale,
                                   k_cmp=k, v_cmp=v, pt_cmp=w.pt_cmp)
    check_attn(fus.out, fus.lse, O, L, f"fused d64 format {fmt}")


def test_fused_fp8_full_size_against_oracle(spa):
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workload("c5")
    b = DeviceBatch(w, fp8_path="fused")
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    O, L = oracle_attn("c5", 1, None)
    check_attn(b.out, b.lse, O, L, "fused c5 full size")


def test_fused_fp8_mixed_groups_and_faults(spa):
    """Sets whose four-row groups straddle the two pools (one compressed key
    dropped per query), and a faulty compressed page, on the fused path."""
    w, dec, fus = fp8_batches("c5", 16)
    dec.build_sets()
    dec.dequant()
    fus.build_sets()
    ip = dec.indptr.cpu().numpy()
    idx = dec.indices[: int(ip[-1])].cpu().numpy()
    keep = np.ones(idx.size, dtype=bool)
    keep[ip[:-1]] = False                     # drop each set's first (compressed) key
    idx2 = idx[keep].astype(np.int32)
    ip2 = (ip - np.arange(ip.size)).astype(np.int32)
    ip2_t, idx2_t = torch.from_numpy(ip2).cuda(), torch.from_numpy(idx2).cuda()
    st1, st2 = spa.new_status(), spa.new_status()
    o1, l1 = spa.sparse_sink_attn_fwd(dec.q, dec.k_raw, dec.v_raw, dec.pt_raw, dec.req, ip2_t, idx2_t,
                                      dec.sink, w.scale, k_cmp=dec.k_cmp, v_cmp=dec.v_cmp,
                                      pt_cmp=dec.pt_cmp, dev_status=st1)
    o2, l2 = spa.sparse_sink_attn_fwd_fp8(fus.q, fus.k_raw, fus.v_raw, fus.pt_raw, fus.req, ip2_t, idx2_t,
                                          fus.sink, w.scale, fus.k_cmp_fp8, fus.v_cmp_fp8, fus.k_cmp_scale,
                                          fus.v_cmp_scale, fus.pt_cmp, dev_status=st2)
    torch.cuda.synchronize()
    assert spa.read_status(st1) == 0 and spa.read_status(st2) == 0
    assert_bit_identical(o1, l1, o2, l2, "straddling groups")
    import oracle
    k_cmp, v_cmp = oracle_cmp_pools("c5", 16)
    O, L = oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip2, idx2, w.sink, w.scale,
                                   k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp)
    check_attn(o2, l2, O, L, "fused, straddling groups")
    # a compressed page id outside the pool: reported, skipped, no trap
    pt = fus.pt_cmp.clone()
    pt[0, 0] = 10 ** 7
    st = spa.new_status()
    spa.sparse_sink_attn_fwd_fp8(fus.q, fus.k_raw, fus.v_raw, fus.pt_raw, fus.req, fus.indptr, fus.indices,
                                 fus.sink, w.scale, fus.k_cmp_fp8, fus.v_cmp_fp8, fus.k_cmp_scale,
                                 fus.v_cmp_scale, pt, dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) & spa.DEV_BAD_PAGE
    fus.step()
    torch.cuda.synchronize()
    assert fus.status_word() == 0


def test_dequant_fnuz_every_code(spa):
    import oracle
    P, ps, d = 4, 16, 128
    src = (np.arange(P * ps * d, dtype=np.int64).reshape(P, ps, d) % 256).astype(np.uint8)
    rng = np.random.default_rng(5)
    scales = (rng.random((P, ps, d // 64)) * 4).astype(np.float32)
    ids = np.array([0, 1, 3], dtype=np.int32)
    ref = oracle.dequant_fp8_pages(src, scales, ids, fmt=1)
    dst = torch.zeros((P, ps, d), dtype=torch.bfloat16, device="cuda")
    st = spa.new_status()
    spa.dequant_fp8_pages(torch.from_numpy(src).cuda(), torch.from_numpy(scales).cuda(),
                          torch.from_numpy(ids).cuda(), dst, fp8_format=1, dev_status=st)
    got = dst.view(torch.int16).cpu().numpy().view(np.uint16)
    nan_ref = (ref & 0x7fff) > 0x7f80
    nan_got = (got & 0x7fff) > 0x7f80
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])
    assert spa.read_status(st) == 0


def test_fused_fp8_fnuz_bit_identical_and_against_oracle(spa):
    """The mixed cache encoded as E4M3 FNUZ: page decode and fused gather
    give identical results, within tolerance of the oracle."""
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workload("c5", 16, 1)
    assert w.fp8_format == 1
    dec = DeviceBatch(w, fp8_path="decode")
    fus = DeviceBatch(w, fp8_path="fused")
    dec.step()
    fus.step()
    torch.cuda.synchronize()
    assert dec.status_word() == 0 and fus.status_word() == 0
    k_ref, _ = oracle_cmp_pools("c5", 16, 1)
    got = dec.k_cmp.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, k_ref)
    assert_bit_identical(dec.out, dec.lse, fus.out, fus.lse, "FNUZ")
    O, L = oracle_attn("c5", 16, None, 1)
    check_attn(fus.out, fus.lse, O, L, "fused FNUZ")


# ------------------------------------------------------------------ paged KV write
def test_paged_kv_write_bit_exact_and_faults(spa):
    import oracle
    rng = np.random.default_rng(11)
    P, ps, d, B, cols = 40, 64, 128, 3, 8
    pt = rng.permutation(P)[: B * cols].reshape(B, cols).astype(np.int32)
    k_pool = rng.integers(0, 1 << 16, size=(P, ps, d), dtype=np.uint16)
    v_pool = rng.integers(0, 1 << 16, size=(P, ps, d), dtype=np.uint16)
    flat = rng.choice(B * cols * ps, size=500, replace=False)
    req = (flat // (cols * ps)).astype(np.int32)
    pos = (flat % (cols * ps)).astype(np.int32)
    req[0] = 9                                   # faulty request
    k_new = rng.integers(0, 1 << 16, size=(500, d), dtype=np.uint16)
    v_new = rng.integers(0, 1 << 16, size=(500, d), dtype=np.uint16)
    k_ref, v_ref, flags = oracle.paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool)
    assert flags == 2

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)

    kp, vp = dev_bf16(k_pool).clone(), dev_bf16(v_pool).clone()
    st = spa.new_status()
    spa.paged_kv_write(dev_bf16(k_new), dev_bf16(v_new), torch.from_numpy(req).cuda(),
                       torch.from_numpy(pos).cuda(), torch.from_numpy(pt).cuda(), kp, vp, dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) == spa.DEV_BAD_INDEX
    assert np.array_equal(kp.view(torch.int16).cpu().numpy().view(np.uint16), k_ref)
    assert np.array_equal(vp.view(torch.int16).cpu().numpy().view(np.uint16), v_ref)


def test_graph_capture_and_two_streams(spa):
    """The three calls capture into a CUDA graph; replays and a second
    stream give bit-identical results."""
    b = batch(spa, "c5", 16)
    b.step()
    torch.cuda.synchronize()
    ref_out, ref_lse = b.out.clone(), b.lse.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            b.step(stream=s)
    b.out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(b.out, ref_out) and torch.equal(b.lse, ref_lse)
    b2 = batch(spa, "c5", 16)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        b.step(stream=s1)
    with torch.cuda.stream(s2):
        b2.step(stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(b.out, ref_out) and torch.equal(b2.out, ref_out)
    assert torch.equal(b2.lse, ref_lse)


# ---------------------------------------------------------------- backward
# The backward reads the forward's saved O (BF16) and LSE (FP32). Parity
# feeds both sides the same saved values (the oracle's forward, O rounded to
# BF16 and LSE to FP32), so what is compared is the backward alone. Bar,
# from its arithmetic: P and dS enter the tensor-core products rounded to
# BF16 (relative 2^-9 per term) and every sum is FP32, so an element may be
# off by a small multiple of 2^-9 of its row's magnitude:
#   |g - ref| <= 2e-2 * rms(row of ref) + 1e-2 * |ref| + 1e-3 * rms(ref)
# (a row: the d entries of one dq (query, head), of one dk/dv pool row, or
# the H entries of dsink; the last term covers rows whose exact value
# cancels to zero while their FP32 terms are of the tensor's typical size). The chain check (the CUDA forward's own O and LSE
# into the backward) adds the forward's error to D; it is held to a
# relative Frobenius error of 2e-2 per gradient.
G_ROW = 2e-2
G_REL = 1e-2
G_FLOOR = 1e-3
G_CHAIN = 2e-2


def check_grad(g, ref, what):
    g = g.detach().double().cpu().numpy() if torch.is_tensor(g) else np.asarray(g, dtype=np.float64)
    g = g.reshape(ref.shape)
    r2 = ref.reshape(-1, ref.shape[-1]) if ref.ndim > 1 else ref.reshape(1, -1)
    g2 = g.reshape(r2.shape)
    rms_row = np.sqrt(np.mean(r2 * r2, axis=1, keepdims=True))
    rms_all = float(np.sqrt(np.mean(r2 * r2))) if r2.size else 0.0
    err = np.abs(g2 - r2)
    bad = err > G_ROW * rms_row + G_REL * np.abs(r2) + G_FLOOR * rms_all
    worst = float((err / np.maximum(rms_row, 1e-2 * rms_all + 1e-30)).max()) if r2.size else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {r2.size} out of tolerance, "
                           f"max err {err.max():.3g}, worst err / rms(row) {worst:.3g}")
    return worst


@functools.lru_cache(maxsize=None)
def dout_bits(name, shrink=1):
    from sparse_paged_attention_build_b200 import workloads
    return workloads.make_dout(workload(name, shrink))


def saved_from_oracle(O, L):
    """The oracle's forward as a forward would store it: O rounded to BF16
    (bits), LSE rounded to FP32; and the same values in FP64 for the oracle."""
    o_bf = torch.from_numpy(O).to(torch.float32).to(torch.bfloat16)
    l_f32 = torch.from_numpy(L).to(torch.float32)
    return o_bf, l_f32, o_bf.to(torch.float64).numpy(), l_f32.to(torch.float64).numpy()


def gpu_bwd(spa, b, name, shrink, out, lse, num_splits=0, indptr=None, indices=None, sink="w"):
    w = workload(name, shrink)
    dO = torch.from_numpy(dout_bits(name, shrink).view(np.int16)).cuda().view(torch.bfloat16)
    st = spa.new_status()
    ip = b.indptr if indptr is None else indptr
    ix = b.indices if indices is None else indices
    s = b.sink if isinstance(sink, str) else sink
    g = spa.sparse_sink_attn_bwd(b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, ip, ix, s, w.scale,
                                 out.cuda().contiguous(), lse.cuda().contiguous(), dO,
                                 k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp, num_splits=num_splits,
                                 dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) == 0
    return g


def oracle_bwd(name, shrink, rows=None, indptr=None, indices=None, sink="w", o_saved=None, lse_saved=None):
    import oracle
    w = workload(name, shrink)
    ip, idx = oracle_sets(name, shrink) if indptr is None else (indptr, indices)
    k_cmp, v_cmp = oracle_cmp_pools(name, shrink)
    return oracle.sparse_sink_attn_bwd(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx,
                                       w.sink if isinstance(sink, str) else sink, w.scale, dout_bits(name, shrink),
                                       k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp,
                                       rows=None if rows is None else np.asarray(rows, dtype=np.int32),
                                       o_saved=o_saved, lse_saved=lse_saved)


def oracle_fwd_sets(name, shrink, ip, idx, sink):
    import oracle
    w = workload(name, shrink)
    k_cmp, v_cmp = oracle_cmp_pools(name, shrink)
    return oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, sink, w.scale,
                                   k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp)


GRAD_NAMES = ("dq", "dk_raw", "dv_raw", "dk_cmp", "dv_cmp", "dsink")


def check_all_grads(g, r, what):
    worst = {}
    for n, a, ref in zip(GRAD_NAMES, g, r):
        if ref is None:
            assert a is None or float(a.abs().max()) == 0.0, n
            continue
        worst[n] = check_grad(a, ref, f"{what} {n}")
    return worst


def saved_case(spa, name, shrink, num_splits=0, ip=None, idx=None, sink="w"):
    """GPU backward and oracle backward on the same saved O/LSE."""
    w = workload(name, shrink)
    if ip is None:
        ip, idx = oracle_sets(name, shrink)
    s = w.sink if isinstance(sink, str) else np.full(w.H, -np.inf, dtype=np.float32)
    O, L = oracle_fwd_sets(name, shrink, ip, idx, s)
    o_bf, l_f32, o64, l64 = saved_from_oracle(O, L)
    b = batch(spa, name, shrink)
    g = gpu_bwd(spa, b, name, shrink, o_bf, l_f32, num_splits=num_splits,
                indptr=torch.from_numpy(ip).cuda(), indices=torch.from_numpy(idx).cuda(), sink=sink)
    r = oracle_bwd(name, shrink, indptr=ip, indices=idx, sink=s, o_saved=o64, lse_saved=l64)
    if sink is None:
        r = r[:5] + (None,)
    return g, r


@pytest.mark.parametrize("name,shrink", [("c1", 1), ("c2", 8), ("c3", 16), ("c4", 16)])
def test_bwd_every_element_small(spa, name, shrink):
    g, r = saved_case(spa, name, shrink)
    worst = check_all_grads(g, r, f"{name}/{shrink}")
    print(name, shrink, {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("splits", [1, 3, 16])
def test_bwd_split_counts(spa, splits):
    g, r = saved_case(spa, "c4", 8, num_splits=splits)
    check_all_grads(g, r, f"splits={splits}")


def test_bwd_no_sink_and_empty_sets(spa):
    w = workload("c1")
    ip, idx = oracle_sets("c1")
    keep = np.ones(w.N, dtype=bool)
    keep[::3] = False
    sizes = np.diff(ip) * keep
    ip2 = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    idx2 = np.concatenate([idx[ip[i]:ip[i + 1]] for i in range(w.N) if keep[i]]).astype(np.int32)
    for sink in ("w", None):
        g, r = saved_case(spa, "c1", 1, ip=ip2, idx=idx2, sink=sink)
        check_all_grads(g, r, f"empty sets, sink={sink}")
        assert float(g[0][torch.from_numpy(~keep).cuda()].abs().max()) == 0.0


def test_bwd_chain_from_the_cuda_forward(spa):
    """The CUDA forward's O and LSE into the CUDA backward, against the
    exact gradients: relative Frobenius error per gradient."""
    name, shrink = "c3", 16
    w = workload(name, shrink)
    b = batch(spa, name, shrink)
    b.step()
    torch.cuda.synchronize()
    g = gpu_bwd(spa, b, name, shrink, b.out, b.lse)
    r = oracle_bwd(name, shrink)
    for n, a, ref in zip(GRAD_NAMES, g, r):
        if ref is None:
            continue
        a = a.double().cpu().numpy().reshape(ref.shape)
        rel = np.linalg.norm(a - ref) / np.linalg.norm(ref)
        assert rel <= G_CHAIN, f"{n}: relative error {rel:.3g}"


def test_bwd_full_size_sampled_dq(spa):
    """c3 at full size in the benchmark's launch configuration (the CUDA
    forward's O/LSE for every token, the oracle's saved O/LSE for the
    sampled tokens): dq of the sampled tokens against the oracle (a token's
    dq depends only on its own saved O/LSE)."""
    import oracle
    name = "c3"
    w = workload(name)
    b = batch(spa, name)
    b.step()
    torch.cuda.synchronize()
    rows = sample_rows(w, n_random=24)
    O, L = oracle_attn(name, 1, rows)
    o_bf, l_f32, o64, l64 = saved_from_oracle(O, L)
    out, lse = b.out.clone(), b.lse.clone()
    ridx = torch.from_numpy(rows).long().cuda()
    out[ridx] = o_bf.cuda()
    lse[ridx] = l_f32.cuda()
    g = gpu_bwd(spa, b, name, 1, out, lse)
    o_full = np.zeros((w.N, w.H, w.d))
    l_full = np.zeros((w.N, w.H))
    o_full[rows] = o64
    l_full[rows] = l64
    r = oracle_bwd(name, 1, rows=rows, o_saved=o_full, lse_saved=l_full)
    check_grad(g[0][ridx], r[0], "c3 dq sampled")
    for t in g[1:5]:
        assert torch.isfinite(t).all()


# ---------------------------------------------------------------- packed D512 rows
@pytest.mark.parametrize("pages,ps", [(64, 64), (5, 1), (3, 128)])
def test_unpack_d512_bit_exact(spa, pages, ps):
    import oracle
    from sparse_paged_attention_build_b200 import workloads
    src = workloads.make_packed_d512(pages, ps, seed=pages + ps)
    ids = np.random.default_rng(ps).permutation(pages)[: max(1, pages - 2)].astype(np.int32)
    ref = oracle.unpack_d512_pages(src, ids)
    st = spa.new_status()
    dst = spa.unpack_d512_pages(torch.from_numpy(src).cuda(), torch.from_numpy(ids).cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert spa.read_status(st) == 0
    got = dst.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_unpack_d512_every_code_scale_and_bad_page(spa):
    """Every code under scale bytes 0 (a subnormal scale), 1, 120, 127, 140
    and 254, NaN codes and the NaN scale compared by position; a bad page id
    is reported and skipped."""
    import oracle
    src = np.zeros((2, 8, 584), dtype=np.uint8)
    codes = np.arange(256, dtype=np.uint8)
    src[:, :, :448] = np.concatenate([codes, codes[:192]])
    for r, sb in enumerate((0, 1, 120, 127, 140, 254, 255, 127)):
        src[:, r, 576:583] = sb
    src[:, :, 448:576] = np.arange(128, dtype=np.uint8)
    ids = np.array([0, 1], dtype=np.int32)
    ref = oracle.unpack_d512_pages(src, ids)
    st = spa.new_status()
    dst = spa.unpack_d512_pages(torch.from_numpy(src).cuda(), torch.from_numpy(ids).cuda(), dev_status=st)
    torch.cuda.synchronize()
    got = dst.view(torch.int16).cpu().numpy().view(np.uint16)
    nan_ref = (ref & 0x7F80 == 0x7F80) & (ref & 0x7F != 0)
    nan_got = (got & 0x7F80 == 0x7F80) & (got & 0x7F != 0)
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])
    bad = torch.tensor([0, 7], dtype=torch.int32, device="cuda")
    st2 = spa.new_status()
    spa.unpack_d512_pages(torch.from_numpy(src).cuda(), bad, dev_status=st2)
    torch.cuda.synchronize()
    assert spa.read_status(st2) & 1   # SPA_DEV_BAD_PAGE
