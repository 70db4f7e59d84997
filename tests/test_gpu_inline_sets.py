"""GPU: attention over sets built inside the kernel.

spa_sparse_sink_attn_fwd_inline_sets builds, per query, the set
spa_build_kv_sets builds from the same inputs (the complete groups -- all of
them, or those a top-k row picks, sorted, repeats removed -- then the
window) in its resolver. The keys and their order are the same, so its O
and LSE must be bit-identical to spa_build_kv_sets followed by
spa_sparse_sink_attn_fwd at the same split count -- including the status
word and the empty-set rows of faulty positions. Two cases are also checked
against the FP64 oracle directly, at the method's tolerance.
"""
import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_paged_attention_build_b200 as m
    return m


def _both(w, splits, fp8_path="decode"):
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    res = []
    for sets in ("csr", "inline"):
        b = DeviceBatch(w, num_splits=splits, sets=sets, fp8_path=fp8_path)
        b.step()
        torch.cuda.synchronize()
        res.append(b)
    return res


def _assert_identical(a, b, what):
    assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16)), f"{what}: O differs"
    assert torch.equal(a.lse.view(torch.int32), b.lse.view(torch.int32)), f"{what}: LSE differs"
    assert a.status_word() == b.status_word(), f"{what}: status {a.status_word()} vs {b.status_word()}"


def _no_topk(w, ratio=None):
    """The workload with its top-k list dropped (every complete group)."""
    return dataclasses.replace(w, topk=None, K=0, ratio=w.ratio if ratio is None else ratio)


@pytest.mark.parametrize("name,shrink,splits", [
    ("c4", 1, 0), ("c4", 1, 1), ("c4", 4, 2), ("c4", 8, 3), ("c4", 16, 12),   # ratio 128 (HCA)
    ("c2", 1, 0), ("c2", 8, 4),                                              # ratio 0 (window only)
])
def test_inline_sets_bit_identical_to_csr(spa, name, shrink, splits):
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make(name, shrink=shrink)
    csr, inl = _both(w, splits)
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"{name}/{shrink} splits={splits}")


@pytest.mark.parametrize("name,shrink,splits", [("c3", 16, 0), ("c1", 1, 1), ("c1", 1, 3), ("f2", 8, 0),
                                                ("f1", 8, 1)])
def test_inline_sets_every_complete_group(spa, name, shrink, splits):
    """Ratio-4 workloads (d = 64, 128 and 512) without their top-k lists:
    every complete group joins the set."""
    from sparse_paged_attention_build_b200 import workloads
    w = _no_topk(workloads.make(name, shrink=shrink))
    csr, inl = _both(w, splits)
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"{name}/{shrink} without top-k, splits={splits}")


@pytest.mark.parametrize("name,shrink,splits", [
    ("c1", 1, 0), ("c1", 1, 1), ("c1", 1, 3),       # top-k 16, d = 64
    ("c3", 16, 0), ("c3", 16, 2), ("c3", 1, 0),     # top-k 512, d = 128; the full prefill the bench times
    ("f1", 8, 0), ("f2", 8, 0), ("f2", 8, 3),       # top-k 512, d = 512
    ("c5", 8, 0), ("c5", 8, 4),                     # top-k 512, mixed cache decoded to BF16 first
])
def test_inline_sets_from_topk_rows(spa, name, shrink, splits):
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make(name, shrink=shrink)
    assert w.topk is not None
    csr, inl = _both(w, splits)
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"{name}/{shrink} splits={splits}")


@pytest.mark.parametrize("shrink,splits,fmt", [(8, 0, 0), (8, 4, 0), (1, 0, 0), (8, 2, 1)])
def test_inline_sets_fp8_gather(spa, shrink, splits, fmt):
    """The mixed cache with its FP8 pages decoded inside the gather
    (spa_sparse_sink_attn_fwd_fp8_inline_sets against build + the FP8 call),
    OCP E4M3 and E4M3 FNUZ codes."""
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make("c5", shrink=shrink, fp8_format=fmt)
    csr, inl = _both(w, splits, fp8_path="fused")
    assert csr.fused and inl.fused
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"c5/{shrink} fused, splits={splits}, format {fmt}")


def _planted_topk(w, width, seed):
    """Top-k rows of `width` entries with repeats, padding (-1, -7), groups
    that are not complete yet and values past 2^30 planted in them."""
    rng = np.random.default_rng(seed)
    n_groups = (w.pos.astype(np.int64) + 1) // w.ratio
    top = rng.integers(0, np.maximum(n_groups, 1)[:, None] + 40, size=(w.N, width)).astype(np.int64)
    kind = rng.integers(0, 10, size=top.shape)
    top[kind == 0] = -1
    top[kind == 1] = -7
    top[kind == 2] = (1 << 30) + 5
    rep = rng.integers(0, width, size=top.shape)
    top[kind == 3] = np.take_along_axis(top, rep, axis=1)[kind == 3]
    return np.ascontiguousarray(top.astype(np.int32))


@pytest.mark.parametrize("width", [1, 2, 31, 33, 300, 512])
def test_inline_sets_planted_topk_rows(spa, width):
    """Rows of any width up to 512 (not only powers of two), with repeats,
    padding, incomplete groups and huge values: each picks the same groups
    on both paths."""
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make("c3", shrink=16)
    w = dataclasses.replace(w, topk=_planted_topk(w, width, seed=width), K=width)
    csr, inl = _both(w, 2)
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"planted rows of width {width}")


@pytest.mark.parametrize("splits", [0, 3])
def test_inline_sets_past_one_bitmap_window(spa, splits):
    """Contexts whose complete groups outnumber one window of the resolver's
    bitmap (4096 groups) take several windows; one request stays below."""
    from sparse_paged_attention_build_b200 import workloads
    w = workloads._decode("long", 11, 4, np.array([70000, 65541, 100000, 16000]), 8, 64, 128, 4, 512, 64,
                          fp8=False)
    assert ((w.pos.astype(np.int64) + 1) // 4 > 4096).sum() == 3
    csr, inl = _both(w, splits)
    assert csr.status_word() == 0
    _assert_identical(csr, inl, f"long contexts, splits={splits}")


def test_inline_sets_faulty_positions(spa):
    """A position outside [0, 2^30) gives SPA_DEV_BAD_INDEX and an empty set
    (O = 0, LSE = the sink) on both paths."""
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make("c4", shrink=16)
    pos = w.pos.copy()
    pos[0], pos[-1] = -3, 1 << 30
    w = dataclasses.replace(w, pos=pos)
    csr, inl = _both(w, 2)
    assert inl.status_word() & spa.DEV_BAD_INDEX
    _assert_identical(csr, inl, "faulty positions")
    assert torch.count_nonzero(inl.out[0].float()) == 0
    np.testing.assert_allclose(inl.lse[0].cpu().numpy(), w.sink, rtol=0, atol=1e-6)


@pytest.mark.parametrize("name,shrink", [("c4", 16), ("c3", 16)])
def test_inline_sets_against_the_oracle(spa, name, shrink):
    import oracle
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workloads.make(name, shrink=shrink)
    b = DeviceBatch(w, sets="inline")
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    ip, idx = oracle.build_kv_sets(w.pos, w.W, w.ratio, w.topk)
    O, L = oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, w.sink, w.scale,
                                   k_cmp=w.k_cmp, v_cmp=w.v_cmp, pt_cmp=w.pt_cmp)
    o = b.out.float().cpu().double().numpy()
    err = np.abs(o - O)
    assert not (err > 1e-2 * (1.0 + np.abs(O))).any(), f"max err {err.max():.3g}"
    assert (np.abs(b.lse.cpu().double().numpy() - L) <= 2e-3).all()
