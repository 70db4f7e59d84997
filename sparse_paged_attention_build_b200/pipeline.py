"""One pass of the hot path over a resident batch: KV-set build, FP8 page
decode (mixed cache only), sparse sink attention.

``DeviceBatch`` holds a workload's inputs in device memory plus every
output and workspace buffer, allocated once, so that a step launches only
the library's kernels (and the memsets they enqueue) and can be captured in
a CUDA graph.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (build_kv_sets, dequant_fp8_pages, kv_sets_capacity, sparse_sink_attn_fwd, sparse_sink_attn_fwd_fp8,
               sparse_sink_attn_fwd_inline_sets, sparse_sink_attn_fwd_fp8_inline_sets, attn_workspace_size,
               new_status, read_status)
from . import lib


def _dev(a, dtype=None, device="cuda"):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device)


INLINE_TOPK_MAX = 512   # widest top-k row the attention kernel sorts itself


def inline_sets_supported(w) -> bool:
    """Whether the attention kernel can build this workload's sets itself:
    top-k rows of at most INLINE_TOPK_MAX entries (or none)."""
    return w.topk is None or w.topk.shape[1] <= INLINE_TOPK_MAX


def splits_for(w, num_splits=0) -> int:
    """Slices per query the attention runs a workload with (0: the
    library's automatic choice)."""
    if num_splits > 0:
        return num_splits
    if w.d == 512:
        return int(lib.spa_sparse_sink_attn_choose_splits_d512(w.N, w.H))
    return int(lib.spa_sparse_sink_attn_choose_splits(w.N, w.H, 0))


class DeviceBatch:
    """A workload resident in device memory, with its outputs."""

    def __init__(self, w, device="cuda", num_splits=0, fp8_path="decode", sets="csr"):
        self.w = w
        # "csr": the sets are built by spa_build_kv_sets, then read by the
        # attention; "inline": the sets are built inside the attention kernel
        # (the *_inline_sets calls), from the same inputs
        if sets not in ("csr", "inline"):
            raise ValueError("sets is 'csr' or 'inline'")
        if fp8_path not in ("fused", "decode"):
            raise ValueError("fp8_path is 'fused' or 'decode'")
        if sets == "inline" and not inline_sets_supported(w):
            raise ValueError("sets built inside the kernel need top-k rows of at most 512 entries")
        self.inline_sets = sets == "inline"
        self.device = device
        bf16 = torch.bfloat16
        self.q = _dev(w.q.view(np.int16), bf16, device)
        self.pos = _dev(w.pos, None, device)
        self.req = _dev(w.req, None, device)
        self.topk = _dev(w.topk, None, device)
        self.k_raw = _dev(w.k_raw.view(np.int16), bf16, device)
        self.v_raw = _dev(w.v_raw.view(np.int16), bf16, device)
        self.pt_raw = _dev(w.pt_raw, None, device)
        self.pt_cmp = _dev(w.pt_cmp, None, device)
        self.sink = _dev(w.sink, None, device)
        self.fp8 = w.k_cmp_fp8 is not None
        # mixed cache: decode inside the attention gather ("fused"), or decode
        # the pages to a BF16 pool first ("decode")
        self.fused = self.fp8 and fp8_path == "fused"
        if self.fp8:
            self.k_cmp_fp8 = _dev(w.k_cmp_fp8, None, device)
            self.v_cmp_fp8 = _dev(w.v_cmp_fp8, None, device)
            self.k_cmp_scale = _dev(w.k_cmp_scale, None, device)
            self.v_cmp_scale = _dev(w.v_cmp_scale, None, device)
            self.cmp_page_ids = _dev(w.cmp_page_ids, None, device)
            if not self.fused:
                self.k_cmp = torch.zeros(w.k_cmp_fp8.shape, dtype=bf16, device=device)
                self.v_cmp = torch.zeros(w.v_cmp_fp8.shape, dtype=bf16, device=device)
        else:
            self.k_cmp = _dev(None if w.k_cmp is None else w.k_cmp.view(np.int16), bf16, device)
            self.v_cmp = _dev(None if w.v_cmp is None else w.v_cmp.view(np.int16), bf16, device)
        N = w.N
        self.max_pos = int(w.pos.max()) if N else 0
        self.capacity = kv_sets_capacity(N, w.W, w.ratio, w.K, w.topk is not None, self.max_pos)
        self.indptr = torch.empty(N + 1, dtype=torch.int32, device=device)
        self.indices = torch.empty(max(self.capacity, 1), dtype=torch.int32, device=device)
        self.sets_ws = torch.empty(max(int(lib.spa_build_kv_sets_workspace_size(N)), 16),
                                   dtype=torch.uint8, device=device)
        self.num_splits = num_splits
        ws = attn_workspace_size(N, w.H, w.d, num_splits)
        self.attn_ws = torch.empty(ws, dtype=torch.uint8, device=device) if ws else None
        self.out = torch.empty((N, w.H, w.d), dtype=bf16, device=device)
        self.lse = torch.empty((N, w.H), dtype=torch.float32, device=device)
        self.status = new_status(device)

    def build_sets(self, stream=None):
        w = self.w
        build_kv_sets(self.pos, w.W, w.ratio, self.topk, capacity=self.capacity, indptr=self.indptr,
                      indices=self.indices, workspace=self.sets_ws, dev_status=self.status,
                      stream=stream)

    def dequant(self, stream=None):
        if self.fp8 and not self.fused:
            dequant_fp8_pages(self.k_cmp_fp8, self.k_cmp_scale, self.cmp_page_ids, self.k_cmp,
                              fp8_format=self.w.fp8_format, dev_status=self.status, stream=stream)
            dequant_fp8_pages(self.v_cmp_fp8, self.v_cmp_scale, self.cmp_page_ids, self.v_cmp,
                              fp8_format=self.w.fp8_format, dev_status=self.status, stream=stream)

    def attend(self, stream=None):
        w = self.w
        if self.fused and self.inline_sets:
            sparse_sink_attn_fwd_fp8_inline_sets(self.q, self.k_raw, self.v_raw, self.pt_raw, self.req, self.pos,
                                                 self.topk, w.W, w.ratio, self.sink, w.scale, self.k_cmp_fp8,
                                                 self.v_cmp_fp8, self.k_cmp_scale, self.v_cmp_scale, self.pt_cmp,
                                                 out=self.out, lse=self.lse, num_splits=self.num_splits,
                                                 workspace=self.attn_ws, dev_status=self.status, stream=stream,
                                                 fp8_format=self.w.fp8_format)
            return
        if self.fused:
            sparse_sink_attn_fwd_fp8(self.q, self.k_raw, self.v_raw, self.pt_raw, self.req, self.indptr,
                                     self.indices, self.sink, w.scale, self.k_cmp_fp8, self.v_cmp_fp8,
                                     self.k_cmp_scale, self.v_cmp_scale, self.pt_cmp, out=self.out,
                                     lse=self.lse, num_splits=self.num_splits, workspace=self.attn_ws,
                                     dev_status=self.status, stream=stream, fp8_format=self.w.fp8_format)
            return
        if self.inline_sets:
            sparse_sink_attn_fwd_inline_sets(self.q, self.k_raw, self.v_raw, self.pt_raw, self.req, self.pos,
                                             self.topk, w.W, w.ratio, self.sink, w.scale, k_cmp=self.k_cmp,
                                             v_cmp=self.v_cmp, pt_cmp=self.pt_cmp, out=self.out, lse=self.lse,
                                             num_splits=self.num_splits, workspace=self.attn_ws,
                                             dev_status=self.status, stream=stream)
            return
        sparse_sink_attn_fwd(self.q, self.k_raw, self.v_raw, self.pt_raw, self.req, self.indptr,
                             self.indices, self.sink, w.scale, k_cmp=self.k_cmp, v_cmp=self.v_cmp,
                             pt_cmp=self.pt_cmp, out=self.out, lse=self.lse,
                             num_splits=self.num_splits, workspace=self.attn_ws,
                             dev_status=self.status, stream=stream)

    def step(self, stream=None):
        """The whole hot path: sets, decode (mixed cache), attention (the
        sets inside the attention kernel with sets="inline")."""
        if not self.inline_sets:
            self.build_sets(stream)
        self.dequant(stream)
        self.attend(stream)

    def splits_used(self) -> int:
        """Slices per query the attention runs with (0 resolves to the
        library's automatic choice)."""
        return splits_for(self.w, self.num_splits)

    def kernels_per_step(self) -> int:
        return (0 if self.inline_sets else 1) + (2 if self.fp8 and not self.fused else 0) + 1

    def nnz(self) -> int:
        """Keys in all sets (from the CSR arrays: run build_sets first)."""
        return int(self.indptr[-1].item())

    def status_word(self) -> int:
        return read_status(self.status)
