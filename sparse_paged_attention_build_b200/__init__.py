"""Sparse paged attention with an attention sink, forward, for B200.

A thin Python binding over ``libspa.so`` (C ABI in ``include/spa.h``). Every
function here only marshals arguments: it checks dtypes and devices, takes
raw pointers from torch tensors, allocates outputs and workspaces with torch
and calls the library on the current CUDA stream. All arithmetic of the path
runs in the library's CUDA kernels; there is no fallback of any kind: every
call raises ImportError when the built library is missing.

The three calls (same names as the C ABI, without the ``spa_`` prefix):

* :func:`build_kv_sets` -- per-token KV sets as CSR in canonical order.
* :func:`dequant_fp8_pages` -- OCP E4M3 pages with per-64 FP32 scales to BF16.
* :func:`sparse_sink_attn_fwd` -- attention over the sets with the sink in
  the denominator: BF16 O and FP32 natural-log LSE.
"""
from __future__ import annotations

import ctypes
import os

import torch

WINDOW_TAG = 1 << 30
DEV_BAD_PAGE, DEV_BAD_INDEX, DEV_CAPACITY, DEV_TIMEOUT, DEV_SCRATCH_RACE = 1, 2, 4, 8, 16
STATUS = {0: "SPA_OK", 1: "SPA_ERR_INVALID_ARG", 2: "SPA_ERR_UNSUPPORTED", 3: "SPA_ERR_CAPACITY",
          4: "SPA_ERR_WORKSPACE", 5: "SPA_ERR_ALIGNMENT", 6: "SPA_ERR_CUDA"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspa.so")


class SpaError(RuntimeError):
    def __init__(self, call, status, detail):
        super().__init__(f"{call}: {STATUS.get(status, status)} ({detail})")
        self.status = status
        self.detail = detail


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m sparse_paged_attention_build_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.spa_abi_version.restype = ctypes.c_int
    L.spa_status_string.argtypes = [ctypes.c_int]
    L.spa_status_string.restype = ctypes.c_char_p
    L.spa_last_error_detail.restype = ctypes.c_char_p
    L.spa_kv_sets_capacity.argtypes = [i32, i32, i32, i32, i32, i32]
    L.spa_kv_sets_capacity.restype = i64
    L.spa_build_kv_sets_workspace_size.argtypes = [i32]
    L.spa_build_kv_sets_workspace_size.restype = sz
    L.spa_build_kv_sets.argtypes = [P, i32, i32, i32, P, i32, P, P, i64, P, sz, P, P]
    L.spa_build_kv_sets.restype = ctypes.c_int
    L.spa_dequant_fp8_pages.argtypes = [P, P, i64, i32, i32, P, i32, i32, P, P, P]
    L.spa_dequant_fp8_pages.restype = ctypes.c_int
    L.spa_sparse_sink_attn_workspace_size.argtypes = [i32, i32, i32, i32]
    L.spa_sparse_sink_attn_workspace_size.restype = sz
    L.spa_sparse_sink_attn_choose_splits.argtypes = [i32, i32, i32]
    L.spa_sparse_sink_attn_choose_splits.restype = ctypes.c_int
    L.spa_sparse_sink_attn_choose_splits_d512.argtypes = [i32, i32]
    L.spa_sparse_sink_attn_choose_splits_d512.restype = ctypes.c_int
    L.spa_testing_stall_attention.argtypes = [ctypes.c_uint64]
    L.spa_testing_stall_attention.restype = None
    L.spa_sparse_sink_attn_fwd.argtypes = [
        P, i64, i64, i32, i32, i32,
        P, P, i64, i32, P, i32,
        P, P, i64, i32, P, i32,
        P, i32, P, P, P, ctypes.c_float, P, P, i32, P, sz, P, P]
    L.spa_sparse_sink_attn_fwd.restype = ctypes.c_int
    L.spa_sparse_sink_attn_fwd_inline_sets.argtypes = [
        P, i64, i64, i32, i32, i32,
        P, P, i64, i32, P, i32,
        P, P, i64, i32, P, i32,
        P, i32, P, P, i32, i32, i32, P, ctypes.c_float, P, P, i32, P, sz, P, P]
    L.spa_sparse_sink_attn_fwd_inline_sets.restype = ctypes.c_int
    L.spa_sparse_sink_attn_fwd_fp8.argtypes = [
        P, i64, i64, i32, i32, i32,
        P, P, i64, i32, P, i32,
        P, P, P, P, i64, i32, P, i32, i32,
        P, i32, P, P, P, ctypes.c_float, P, P, i32, P, sz, P, P]
    L.spa_sparse_sink_attn_fwd_fp8.restype = ctypes.c_int
    L.spa_sparse_sink_attn_fwd_fp8_inline_sets.argtypes = [
        P, i64, i64, i32, i32, i32,
        P, P, i64, i32, P, i32,
        P, P, P, P, i64, i32, P, i32, i32,
        P, i32, P, P, i32, i32, i32, P, ctypes.c_float, P, P, i32, P, sz, P, P]
    L.spa_sparse_sink_attn_fwd_fp8_inline_sets.restype = ctypes.c_int
    L.spa_paged_kv_write.argtypes = [P, P, i32, i32, P, P, P, i32, i32, i32, i64, P, P, P, P]
    L.spa_paged_kv_write.restype = ctypes.c_int
    L.spa_unpack_d512_pages.argtypes = [P, i64, i32, P, i32, P, P, P]
    L.spa_unpack_d512_pages.restype = ctypes.c_int
    L.spa_sparse_sink_attn_bwd.argtypes = [
        P, i64, i64, i32, i32, i32,
        P, P, i64, i32, P, i32,
        P, P, i64, i32, P, i32,
        P, i32, P, P, P, ctypes.c_float, P, P, P, P, P, P, P, P, P, i32, P, P]
    L.spa_sparse_sink_attn_bwd.restype = ctypes.c_int
    return L


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


class _LazyLib:
    def __getattr__(self, name):
        return getattr(_lib(), name)


lib = _LazyLib()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(call, status):
    if status != 0:
        raise SpaError(call, status, lib.spa_last_error_detail().decode())


def _need(t, name, dtype, device=True):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def new_status(device=None):
    """A zeroed device status word (int32 [1]) for the dev_status argument."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def read_status(dev_status) -> int:
    return int(dev_status.item()) & 0xffffffff


# --------------------------------------------------------------------------
def kv_sets_capacity(n_queries, window, ratio, topk_width, has_topk, max_pos) -> int:
    return int(lib.spa_kv_sets_capacity(n_queries, window, ratio, topk_width, int(has_topk), max_pos))


def build_kv_sets(pos, window, ratio, topk=None, capacity=None, max_pos=None, indptr=None,
                  indices=None, workspace=None, dev_status=None, stream=None):
    """CSR (indptr int32 [N+1], indices int32 [capacity]) of every query's
    key set; the keys of query i are indices[indptr[i]:indptr[i+1]]."""
    _need(pos, "pos", torch.int32)
    N = pos.shape[0]
    K = 0
    if topk is not None:
        _need(topk, "topk", torch.int32)
        topk = topk.contiguous()
        K = topk.shape[1] if topk.dim() == 2 else 0
    if capacity is None:
        if max_pos is None:
            raise ValueError("give capacity or max_pos (the largest position, known to the caller)")
        capacity = kv_sets_capacity(N, window, ratio, K, topk is not None, max_pos)
    dev = pos.device
    if indptr is None:
        indptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    if indices is None:
        indices = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
    ws_bytes = int(lib.spa_build_kv_sets_workspace_size(N))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _check("spa_build_kv_sets", lib.spa_build_kv_sets(
        _p(pos.contiguous()), N, window, ratio, _p(topk), K, _p(indptr), _p(indices), capacity,
        _p(workspace), workspace.numel(), _p(dev_status), _stream(stream)))
    return indptr, indices


def dequant_fp8_pages(src, scales, page_ids, dst, fp8_format=0, dev_status=None, stream=None):
    """dst[pg] = bf16(float(e4m3(src[pg])) * scale) for every listed page;
    fp8_format 0 = OCP E4M3, 1 = E4M3 FNUZ."""
    _need(src, "src", torch.uint8)
    _need(scales, "scales", torch.float32)
    _need(page_ids, "page_ids", torch.int32)
    _need(dst, "dst", torch.bfloat16)
    P, ps, d = src.shape
    assert src.is_contiguous() and scales.is_contiguous() and dst.is_contiguous()
    assert tuple(dst.shape) == (P, ps, d) and scales.numel() == P * ps * (d // 64)
    _check("spa_dequant_fp8_pages", lib.spa_dequant_fp8_pages(
        _p(src), _p(scales), P, ps, d, _p(page_ids.contiguous()), page_ids.numel(), fp8_format,
        _p(dst), _p(dev_status), _stream(stream)))
    return dst


def attn_workspace_size(n_queries, num_heads, head_dim, num_splits=0) -> int:
    return int(lib.spa_sparse_sink_attn_workspace_size(n_queries, num_heads, head_dim, num_splits))


def choose_splits(n_queries, num_heads, max_set_size=0) -> int:
    return int(lib.spa_sparse_sink_attn_choose_splits(n_queries, num_heads, max_set_size))


def sparse_sink_attn_fwd(q, k_raw, v_raw, pt_raw, req, indptr, indices, sink, scale,
                         k_cmp=None, v_cmp=None, pt_cmp=None, out=None, lse=None, num_splits=0,
                         workspace=None, dev_status=None, stream=None):
    """(O bf16 [N, H, d], LSE fp32 [N, H]) of sparse paged attention with sink.

    q: bf16 [N, H, d] (last dim contiguous); k_raw/v_raw (k_cmp/v_cmp): bf16
    [pages, page_size, d]; pt_raw/pt_cmp: int32 [B, cols]; req: int32 [N];
    indptr/indices: int32 CSR key sets; sink: fp32 [H] or None.
    """
    _need(q, "q", torch.bfloat16)
    for name, t in (("k_raw", k_raw), ("v_raw", v_raw)):
        _need(t, name, torch.bfloat16)
        assert t.is_contiguous(), name
    for name, t in (("pt_raw", pt_raw), ("req", req), ("indptr", indptr), ("indices", indices)):
        _need(t, name, torch.int32)
    N, H, d = q.shape
    if q.stride(2) != 1:
        raise ValueError("q's last dimension must be contiguous")
    if pt_cmp is not None:
        _need(pt_cmp, "pt_cmp", torch.int32)
        _need(k_cmp, "k_cmp", torch.bfloat16)
        _need(v_cmp, "v_cmp", torch.bfloat16)
        assert k_cmp.is_contiguous() and v_cmp.is_contiguous()
    if sink is not None:
        _need(sink, "sink", torch.float32)
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((N, H), dtype=torch.float32, device=q.device)
    ws_bytes = attn_workspace_size(N, H, d, num_splits)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    pt_raw = pt_raw.contiguous()
    _check("spa_sparse_sink_attn_fwd", lib.spa_sparse_sink_attn_fwd(
        _p(q), q.stride(0), q.stride(1), N, H, d,
        _p(k_raw), _p(v_raw), k_raw.shape[0], k_raw.shape[1], _p(pt_raw), pt_raw.shape[1],
        _p(k_cmp), _p(v_cmp), 0 if k_cmp is None else k_cmp.shape[0],
        1 if k_cmp is None else k_cmp.shape[1],
        _p(None if pt_cmp is None else pt_cmp.contiguous()), 0 if pt_cmp is None else pt_cmp.shape[1],
        _p(req.contiguous()), pt_raw.shape[0], _p(indptr.contiguous()), _p(indices.contiguous()),
        _p(None if sink is None else sink.contiguous()), float(scale), _p(out), _p(lse), num_splits,
        _p(workspace), 0 if workspace is None else workspace.numel(), _p(dev_status), _stream(stream)))
    return out, lse


def sparse_sink_attn_fwd_inline_sets(q, k_raw, v_raw, pt_raw, req, pos, topk, window, ratio, sink, scale,
                                     k_cmp=None, v_cmp=None, pt_cmp=None, out=None, lse=None, num_splits=0,
                                     workspace=None, dev_status=None, stream=None):
    """sparse_sink_attn_fwd over the sets spa_build_kv_sets builds from pos
    (int32 [N]), topk (int32 [N, K] with K <= 512, or None: every complete
    group), window and ratio, built inside the attention kernel."""
    _need(q, "q", torch.bfloat16)
    for name, t in (("k_raw", k_raw), ("v_raw", v_raw)):
        _need(t, name, torch.bfloat16)
        assert t.is_contiguous(), name
    for name, t in (("pt_raw", pt_raw), ("req", req), ("pos", pos)):
        _need(t, name, torch.int32)
    if topk is not None:
        _need(topk, "topk", torch.int32)
        topk = topk.contiguous()
    N, H, d = q.shape
    if q.stride(2) != 1:
        raise ValueError("q's last dimension must be contiguous")
    if pt_cmp is not None:
        _need(pt_cmp, "pt_cmp", torch.int32)
        _need(k_cmp, "k_cmp", torch.bfloat16)
        _need(v_cmp, "v_cmp", torch.bfloat16)
        assert k_cmp.is_contiguous() and v_cmp.is_contiguous()
    if sink is not None:
        _need(sink, "sink", torch.float32)
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((N, H), dtype=torch.float32, device=q.device)
    ws_bytes = attn_workspace_size(N, H, d, num_splits)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    pt_raw = pt_raw.contiguous()
    _check("spa_sparse_sink_attn_fwd_inline_sets", lib.spa_sparse_sink_attn_fwd_inline_sets(
        _p(q), q.stride(0), q.stride(1), N, H, d,
        _p(k_raw), _p(v_raw), k_raw.shape[0], k_raw.shape[1], _p(pt_raw), pt_raw.shape[1],
        _p(k_cmp), _p(v_cmp), 0 if k_cmp is None else k_cmp.shape[0],
        1 if k_cmp is None else k_cmp.shape[1],
        _p(None if pt_cmp is None else pt_cmp.contiguous()), 0 if pt_cmp is None else pt_cmp.shape[1],
        _p(req.contiguous()), pt_raw.shape[0], _p(pos.contiguous()), _p(topk),
        0 if topk is None else topk.shape[1], int(window), int(ratio),
        _p(None if sink is None else sink.contiguous()), float(scale), _p(out), _p(lse), num_splits,
        _p(workspace), 0 if workspace is None else workspace.numel(), _p(dev_status), _stream(stream)))
    return out, lse


def _fp8_attn_buffers(q, k_raw, v_raw, pt_raw, req, ints, sink, k_cmp_fp8, v_cmp_fp8, k_cmp_scale, v_cmp_scale,
                      pt_cmp, out, lse, num_splits, workspace):
    """Checks and output/workspace buffers shared by the two FP8 calls."""
    _need(q, "q", torch.bfloat16)
    for name, t in (("k_raw", k_raw), ("v_raw", v_raw)):
        _need(t, name, torch.bfloat16)
        assert t.is_contiguous(), name
    for name, t in (("pt_raw", pt_raw), ("req", req), ("pt_cmp", pt_cmp)) + tuple(ints):
        _need(t, name, torch.int32)
    for name, t in (("k_cmp_fp8", k_cmp_fp8), ("v_cmp_fp8", v_cmp_fp8)):
        _need(t, name, torch.uint8)
        assert t.is_contiguous(), name
    for name, t in (("k_cmp_scale", k_cmp_scale), ("v_cmp_scale", v_cmp_scale)):
        _need(t, name, torch.float32)
        assert t.is_contiguous(), name
    N, H, d = q.shape
    if q.stride(2) != 1:
        raise ValueError("q's last dimension must be contiguous")
    if sink is not None:
        _need(sink, "sink", torch.float32)
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((N, H), dtype=torch.float32, device=q.device)
    ws_bytes = attn_workspace_size(N, H, d, num_splits)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    return out, lse, workspace


def sparse_sink_attn_fwd_fp8(q, k_raw, v_raw, pt_raw, req, indptr, indices, sink, scale,
                             k_cmp_fp8, v_cmp_fp8, k_cmp_scale, v_cmp_scale, pt_cmp, out=None, lse=None,
                             num_splits=0, workspace=None, dev_status=None, stream=None, fp8_format=0):
    """Like sparse_sink_attn_fwd, with the compressed pool in FP8 (OCP E4M3
    codes uint8 [pages, page_size, d], FP32 scales [pages, page_size, d/64])
    decoded inside the attention gather; bit-identical to decoding the pages
    with dequant_fp8_pages first."""
    out, lse, workspace = _fp8_attn_buffers(q, k_raw, v_raw, pt_raw, req, (("indptr", indptr), ("indices", indices)),
                                            sink, k_cmp_fp8, v_cmp_fp8, k_cmp_scale, v_cmp_scale, pt_cmp, out, lse,
                                            num_splits, workspace)
    N, H, d = q.shape
    pt_raw = pt_raw.contiguous()
    _check("spa_sparse_sink_attn_fwd_fp8", lib.spa_sparse_sink_attn_fwd_fp8(
        _p(q), q.stride(0), q.stride(1), N, H, d,
        _p(k_raw), _p(v_raw), k_raw.shape[0], k_raw.shape[1], _p(pt_raw), pt_raw.shape[1],
        _p(k_cmp_fp8), _p(v_cmp_fp8), _p(k_cmp_scale), _p(v_cmp_scale), k_cmp_fp8.shape[0], k_cmp_fp8.shape[1],
        _p(pt_cmp.contiguous()), pt_cmp.shape[1], int(fp8_format),
        _p(req.contiguous()), pt_raw.shape[0], _p(indptr.contiguous()), _p(indices.contiguous()),
        _p(None if sink is None else sink.contiguous()), float(scale), _p(out), _p(lse), num_splits,
        _p(workspace), 0 if workspace is None else workspace.numel(), _p(dev_status), _stream(stream)))
    return out, lse


def sparse_sink_attn_fwd_fp8_inline_sets(q, k_raw, v_raw, pt_raw, req, pos, topk, window, ratio, sink, scale,
                                         k_cmp_fp8, v_cmp_fp8, k_cmp_scale, v_cmp_scale, pt_cmp, out=None,
                                         lse=None, num_splits=0, workspace=None, dev_status=None, stream=None,
                                         fp8_format=0):
    """sparse_sink_attn_fwd_fp8 over the sets built inside the kernel from
    pos, topk (int32 [N, K] with K <= 512, or None), window and ratio, as in
    sparse_sink_attn_fwd_inline_sets."""
    ints = (("pos", pos),) + ((("topk", topk),) if topk is not None else ())
    out, lse, workspace = _fp8_attn_buffers(q, k_raw, v_raw, pt_raw, req, ints, sink, k_cmp_fp8, v_cmp_fp8,
                                            k_cmp_scale, v_cmp_scale, pt_cmp, out, lse, num_splits, workspace)
    N, H, d = q.shape
    pt_raw = pt_raw.contiguous()
    topk = None if topk is None else topk.contiguous()
    _check("spa_sparse_sink_attn_fwd_fp8_inline_sets", lib.spa_sparse_sink_attn_fwd_fp8_inline_sets(
        _p(q), q.stride(0), q.stride(1), N, H, d,
        _p(k_raw), _p(v_raw), k_raw.shape[0], k_raw.shape[1], _p(pt_raw), pt_raw.shape[1],
        _p(k_cmp_fp8), _p(v_cmp_fp8), _p(k_cmp_scale), _p(v_cmp_scale), k_cmp_fp8.shape[0], k_cmp_fp8.shape[1],
        _p(pt_cmp.contiguous()), pt_cmp.shape[1], int(fp8_format),
        _p(req.contiguous()), pt_raw.shape[0], _p(pos.contiguous()), _p(topk),
        0 if topk is None else topk.shape[1], int(window), int(ratio),
        _p(None if sink is None else sink.contiguous()), float(scale), _p(out), _p(lse), num_splits,
        _p(workspace), 0 if workspace is None else workspace.numel(), _p(dev_status), _stream(stream)))
    return out, lse


def sparse_sink_attn_bwd(q, k_raw, v_raw, pt_raw, req, indptr, indices, sink, scale, out, lse, dout,
                         k_cmp=None, v_cmp=None, pt_cmp=None, dq=None, dk_raw=None, dv_raw=None,
                         dk_cmp=None, dv_cmp=None, dsink=None, num_splits=0, dev_status=None, stream=None):
    """Gradients of sum(dout * O) for the attention of sparse_sink_attn_fwd.

    out, lse: the forward's O (bf16 [N, H, d]) and LSE (fp32 [N, H]); dout:
    bf16 [N, H, d]. Returns (dq fp32 [N, H, d], dk_raw, dv_raw fp32 shaped
    like the raw pools, dk_cmp, dv_cmp (None without a compressed pool),
    dsink fp32 [H] (None without a sink)). Gradients passed in are added
    into; those not passed start from zeros.
    """
    _need(q, "q", torch.bfloat16)
    for name, t in (("k_raw", k_raw), ("v_raw", v_raw), ("out", out), ("dout", dout)):
        _need(t, name, torch.bfloat16)
        assert t.is_contiguous(), name
    for name, t in (("pt_raw", pt_raw), ("req", req), ("indptr", indptr), ("indices", indices)):
        _need(t, name, torch.int32)
    _need(lse, "lse", torch.float32)
    N, H, d = q.shape
    if q.stride(2) != 1:
        raise ValueError("q's last dimension must be contiguous")
    if pt_cmp is not None:
        _need(pt_cmp, "pt_cmp", torch.int32)
        _need(k_cmp, "k_cmp", torch.bfloat16)
        _need(v_cmp, "v_cmp", torch.bfloat16)
        assert k_cmp.is_contiguous() and v_cmp.is_contiguous()
    if sink is not None:
        _need(sink, "sink", torch.float32)

    def grad(t, like, name):
        if t is None:
            return torch.zeros(like.shape, dtype=torch.float32, device=like.device)
        _need(t, name, torch.float32)
        assert t.is_contiguous() and t.shape == like.shape, name
        return t

    dq = grad(dq, q, "dq")
    dk_raw, dv_raw = grad(dk_raw, k_raw, "dk_raw"), grad(dv_raw, v_raw, "dv_raw")
    if pt_cmp is not None:
        dk_cmp, dv_cmp = grad(dk_cmp, k_cmp, "dk_cmp"), grad(dv_cmp, v_cmp, "dv_cmp")
    else:
        dk_cmp = dv_cmp = None
    dsink = None if sink is None else grad(dsink, sink, "dsink")
    pt_raw = pt_raw.contiguous()
    _check("spa_sparse_sink_attn_bwd", lib.spa_sparse_sink_attn_bwd(
        _p(q), q.stride(0), q.stride(1), N, H, d,
        _p(k_raw), _p(v_raw), k_raw.shape[0], k_raw.shape[1], _p(pt_raw), pt_raw.shape[1],
        _p(k_cmp), _p(v_cmp), 0 if k_cmp is None else k_cmp.shape[0],
        1 if k_cmp is None else k_cmp.shape[1],
        _p(None if pt_cmp is None else pt_cmp.contiguous()), 0 if pt_cmp is None else pt_cmp.shape[1],
        _p(req.contiguous()), pt_raw.shape[0], _p(indptr.contiguous()), _p(indices.contiguous()),
        _p(None if sink is None else sink.contiguous()), float(scale), _p(out), _p(lse.contiguous()),
        _p(dout), _p(dq), _p(dk_raw), _p(dv_raw), _p(dk_cmp), _p(dv_cmp), _p(dsink), num_splits,
        _p(dev_status), _stream(stream)))
    return dq, dk_raw, dv_raw, dk_cmp, dv_cmp, dsink


def unpack_d512_pages(src, page_ids, dst=None, dev_status=None, stream=None):
    """BF16 [pages, page_size, 512] of the listed pages of a packed cache
    (uint8 [pages, page_size, 584]: 448 E4M3 codes, 64 BF16 values, 7 UE8M0
    scale bytes, 1 unused byte per token)."""
    _need(src, "src", torch.uint8)
    _need(page_ids, "page_ids", torch.int32)
    assert src.is_contiguous() and src.dim() == 3 and src.shape[2] == 584
    P, ps, _ = src.shape
    if dst is None:
        dst = torch.zeros((P, ps, 512), dtype=torch.bfloat16, device=src.device)
    _need(dst, "dst", torch.bfloat16)
    assert dst.is_contiguous() and tuple(dst.shape) == (P, ps, 512)
    page_ids = page_ids.contiguous()
    _check("spa_unpack_d512_pages", lib.spa_unpack_d512_pages(
        _p(src), P, ps, _p(page_ids), page_ids.numel(), _p(dst), _p(dev_status), _stream(stream)))
    return dst


def paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool, dev_status=None, stream=None):
    """Write token j's K and V rows (bf16 [n, d]) to row pt[req[j]][pos[j] //
    page_size] * page_size + pos[j] % page_size of the pools (bf16
    [pages, page_size, d])."""
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_pool", k_pool), ("v_pool", v_pool)):
        _need(t, name, torch.bfloat16)
        assert t.is_contiguous(), name
    for name, t in (("req", req), ("pos", pos), ("pt", pt)):
        _need(t, name, torch.int32)
    n, d = k_new.shape
    assert tuple(v_new.shape) == (n, d) and k_pool.shape == v_pool.shape and k_pool.shape[2] == d
    pt = pt.contiguous()
    _check("spa_paged_kv_write", lib.spa_paged_kv_write(
        _p(k_new), _p(v_new), n, d, _p(req.contiguous()), _p(pos.contiguous()), _p(pt), pt.shape[1], pt.shape[0],
        k_pool.shape[1], k_pool.shape[0], _p(k_pool), _p(v_pool), _p(dev_status), _stream(stream)))

