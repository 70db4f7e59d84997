"""The attention's bounded waits, driven to give up on purpose -- no fault.

Every wait between the warp roles of the attention forward has a time
limit; when one runs out the kernel sets SPA_DEV_TIMEOUT, the CTA unwinds
(waiting, with the fixed limit, for its own copies and tensor-core products
before it frees TMEM) and the call returns. The testing hook makes every
CTA wait on a barrier that nothing arrives at (a flag that nothing sets),
with a 2 ms limit: that wait always runs out, the others then give up on
the CTA's abort flag. The context must stay usable: the next normal call is
bit-identical to a clean run.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

STALL_LIMIT_NS = 2_000_000


@pytest.fixture(scope="module")
def spa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_paged_attention_build_b200 as m
    m.lib.spa_testing_stall_attention.argtypes = [ctypes.c_uint64]
    m.lib.spa_testing_stall_attention.restype = None
    return m


@pytest.mark.parametrize("name,shrink,splits", [("c1", 1, 1), ("c1", 1, 2), ("c4", 16, 12), ("f2", 8, 2)])
def test_stalled_wait_sets_timeout_and_next_call_is_clean(spa, name, shrink, splits):
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    w = workloads.make(name, shrink=shrink)
    b = DeviceBatch(w, num_splits=splits)
    b.step()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    ref_out = b.out.view(torch.int16).clone()
    ref_lse = b.lse.view(torch.int32).clone()

    st = spa.new_status()
    out = torch.full_like(b.out, float("nan"))
    lse = torch.full_like(b.lse, float("nan"))
    spa.lib.spa_testing_stall_attention(STALL_LIMIT_NS)
    try:
        spa.sparse_sink_attn_fwd(b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, b.indptr, b.indices, b.sink, w.scale,
                                 k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp, out=out, lse=lse,
                                 num_splits=splits, workspace=b.attn_ws, dev_status=st)
        torch.cuda.synchronize()    # the call returned and the context is usable
    finally:
        spa.lib.spa_testing_stall_attention(0)
    assert spa.read_status(st) & spa.DEV_TIMEOUT

    b.status.zero_()
    b.out.zero_()
    b.lse.zero_()
    b.attend()
    torch.cuda.synchronize()
    assert b.status_word() == 0
    assert torch.equal(b.out.view(torch.int16), ref_out)
    assert torch.equal(b.lse.view(torch.int32), ref_lse)
