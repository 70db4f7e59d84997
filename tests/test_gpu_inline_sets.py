"""GPU: attention over sets built inside the kernel (no top-k list).

spa_sparse_sink_attn_fwd_all_groups builds, per query, the set
spa_build_kv_sets builds without a top-k list (every complete group, then
the window) in its resolver. The keys and their order are the same, so its
O and LSE must be bit-identical to spa_build_kv_sets followed by
spa_sparse_sink_attn_fwd at the same split count -- including the status
word and the empty-set rows of faulty positions. One case is also checked
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


def _both(w, splits):
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    res = []
    for sets in ("csr", "inline"):
        b = DeviceBatch(w, num_splits=splits, sets=sets)
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


def test_inline_sets_against_the_oracle(spa):
    import oracle
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workloads.make("c4", shrink=16)
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
