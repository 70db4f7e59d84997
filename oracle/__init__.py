"""FP64 CPU oracle for sparse paged attention with an attention sink.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does. It wraps ``spa_oracle.c`` (plain C, FP64, pthreads) through ctypes and
shares no code with the CUDA library.

What each function follows (page title, then section):

* :func:`build_kv_sets` -- "Roadmap item 24 - joint compressed/window
  attention with sink", "Contracts and lifetime" (logical request / position /
  kind keys, complete windows, C4/C128 group boundaries, canonical order) and
  "test: add block-level DeepSeek-V4 attention test", opening section and
  "Validation" (ratio 0 / 4 / 128 layers, top-k truncation).
* :func:`dequant_fp8_pages` -- "Roadmap item 24", "Reuse and arithmetic"
  (mixed FP8/BF16 cache decoded with an explicit OCP format).
* :func:`sparse_sink_attn` -- "Roadmap item 24", "Reuse and arithmetic"
  (one denominator for compressed KV, window and sink; the sink has no V;
  natural-log LSE) and "MI300X validation" (an FP64 O/LSE oracle).
* :func:`unpack_d512_pages` -- "Roadmap item 24", review notes on the packed
  joint KV gather (584 bytes per token for a 512-wide head, 576 of them
  data): 448 E4M3 codes with UE8M0 scales per 64, 64 BF16 values.
* :func:`sparse_sink_attn_bwd` -- "Roadmap item 24", the backward named as
  its follow-on item (dQ, dK/dV, d_sink): the chain rule through the forward
  above, with the sink's logit carrying no V.
* :func:`lse_merge` -- "[WS2] Add CP-aware Attention contract and dispatch
  metadata", "Summary" (deterministic (out, lse) merge) and "docs: Block
  AttnRes model + ROCm-first plan", "Summary" (attn-with-stats +
  softmax_merge, merge lemma).

Every function here is pinned by tests under ``tests/`` to values the pages
print, closed forms, library routines and brute force; none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

WINDOW_TAG = 1 << 30

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libspa_oracle.so")
_lib = None
_lock = threading.Lock()

_ERRORS = {1: "bad argument", 2: "bad index", 3: "bad page", 4: "capacity", 5: "no memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (no GPU involved)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["cc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_double.restype = dbl
            L.oracle_float_to_bf16_rne.argtypes = [ctypes.c_float]
            L.oracle_float_to_bf16_rne.restype = ctypes.c_uint16
            L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_to_double.restype = dbl
            L.oracle_build_kv_sets.argtypes = [P, i32, i32, i32, P, i32, P, P, i64]
            L.oracle_build_kv_sets.restype = ctypes.c_int
            L.oracle_dequant_fp8_pages.argtypes = [P, P, i64, i32, i32, P, i32, P]
            L.oracle_dequant_fp8_pages.restype = ctypes.c_int
            L.oracle_dequant_fp8_pages_fmt.argtypes = [P, P, i64, i32, i32, P, i32, i32, P]
            L.oracle_dequant_fp8_pages_fmt.restype = ctypes.c_int
            L.oracle_e4m3fnuz_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3fnuz_to_double.restype = dbl
            L.oracle_ue8m0_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_ue8m0_to_double.restype = dbl
            L.oracle_unpack_d512_pages.argtypes = [P, i64, i32, P, i32, P]
            L.oracle_unpack_d512_pages.restype = ctypes.c_int
            L.oracle_paged_kv_write.argtypes = [P, P, i32, i32, P, P, P, i32, i32, i32, i64, P, P]
            L.oracle_paged_kv_write.restype = ctypes.c_int
            L.oracle_sparse_sink_attn.argtypes = [
                P, i64, i64, i32, i32, i32,
                P, P, i64, i32, P, i32,
                P, P, i64, i32, P, i32,
                P, i32, P, P, P, dbl, i32, P, i32, P, P, i32]
            L.oracle_sparse_sink_attn.restype = ctypes.c_int
            L.oracle_sparse_sink_attn_bwd.argtypes = [
                P, i64, i64, i32, i32, i32,
                P, P, i64, i32, P, i32,
                P, P, i64, i32, P, i32,
                P, i32, P, P, P, dbl, P, P, P, P, i32, P, P, P, P, P, P, i32]
            L.oracle_sparse_sink_attn_bwd.restype = ctypes.c_int
            L.oracle_lse_merge.argtypes = [i32, P, P, i32, P, P]
            L.oracle_lse_merge.restype = None
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(status):
    if status != 0:
        raise OracleError(_ERRORS.get(status, f"status {status}"))


# --------------------------------------------------------------------------
# scalar conversions
# --------------------------------------------------------------------------

def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def float_to_bf16_rne(x: float) -> int:
    return lib().oracle_float_to_bf16_rne(float(x))


def e4m3_to_double(code: int) -> float:
    return lib().oracle_e4m3_to_double(int(code))


def e4m3_table() -> np.ndarray:
    """All 256 OCP E4M3 codes decoded to FP64."""
    return np.array([e4m3_to_double(c) for c in range(256)], dtype=np.float64)


def e4m3fnuz_to_double(code: int) -> float:
    return lib().oracle_e4m3fnuz_to_double(int(code))


def e4m3fnuz_table() -> np.ndarray:
    """All 256 E4M3 FNUZ codes decoded to FP64."""
    return np.array([e4m3fnuz_to_double(c) for c in range(256)], dtype=np.float64)


# --------------------------------------------------------------------------
# the three steps of the path
# --------------------------------------------------------------------------

def kv_sets_bound(pos, W, ratio, K, has_topk=True) -> int:
    pos = np.asarray(pos, dtype=np.int64)
    if pos.size == 0:
        return 0
    nc = (pos + 1) // ratio if ratio > 0 else np.zeros_like(pos)
    c = np.minimum(nc, K) if has_topk else nc
    return int((np.minimum(pos + 1, W) + c).sum())


def build_kv_sets(pos, W: int, ratio: int, topk=None, K: int | None = None):
    """CSR (indptr int32 [N+1], indices int32 [nnz]) of every query's key set."""
    pos = _c(pos, np.int32)
    N = pos.shape[0]
    if topk is not None:
        topk = _c(topk, np.int32)
        topk = topk.reshape(N, topk.shape[-1] if topk.ndim == 2 else -1)
        K = topk.shape[1]
    K = 0 if K is None else int(K)
    cap = kv_sets_bound(pos, W, ratio, K, topk is not None) + 1
    indptr = np.zeros(N + 1, dtype=np.int32)
    indices = np.zeros(cap, dtype=np.int32)
    _check(lib().oracle_build_kv_sets(_ptr(pos), N, W, ratio, _ptr(topk), K,
                                      _ptr(indptr), _ptr(indices), cap))
    return indptr, indices[: indptr[-1]].copy()


def dequant_fp8_pages(src, scales, page_ids, dst=None, fmt=0):
    """BF16 bits of the listed pages: bf16_rne(float(e4m3(byte)) * scale);
    fmt 0 = OCP E4M3, 1 = E4M3 FNUZ."""
    src = _c(src, np.uint8)
    P, ps, d = src.shape
    scales = _c(scales, np.float32).reshape(P, ps, d // 64)
    page_ids = _c(page_ids, np.int32)
    if dst is None:
        dst = np.zeros((P, ps, d), dtype=np.uint16)
    assert dst.dtype == np.uint16 and dst.flags.c_contiguous and dst.shape == (P, ps, d)
    _check(lib().oracle_dequant_fp8_pages_fmt(_ptr(src), _ptr(scales), P, ps, d, _ptr(page_ids),
                                              page_ids.shape[0], int(fmt), _ptr(dst)))
    return dst


def sparse_sink_attn(q, k_raw, v_raw, pt_raw, req, indptr, indices, sink, scale,
                     k_cmp=None, v_cmp=None, pt_cmp=None, rows=None, include_sink=True,
                     threads=None):
    """FP64 (O [n_rows, H, d], LSE [n_rows, H]) for the given query tokens.

    q: BF16 bits [N, H, d]; k_raw/v_raw (and k_cmp/v_cmp): BF16 bits
    [pages, page_size, d]; pt_raw/pt_cmp: int32 [B, cols]; req: int32 [N];
    indptr/indices: the CSR key sets; sink: float32 [H]; scale: float.
    """
    q = np.asarray(q)
    assert q.dtype == np.uint16 and q.ndim == 3 and q.strides[2] == 2
    N, H, d = q.shape
    k_raw, v_raw = _c(k_raw, np.uint16), _c(v_raw, np.uint16)
    pt_raw = _c(pt_raw, np.int32)
    if pt_cmp is not None:
        k_cmp, v_cmp, pt_cmp = _c(k_cmp, np.uint16), _c(v_cmp, np.uint16), _c(pt_cmp, np.int32)
    req, indptr, indices = _c(req, np.int32), _c(indptr, np.int32), _c(indices, np.int32)
    sink = _c(sink, np.float32)
    rows = None if rows is None else _c(rows, np.int32)
    n_rows = N if rows is None else rows.shape[0]
    out = np.zeros((n_rows, H, d), dtype=np.float64)
    lse = np.zeros((n_rows, H), dtype=np.float64)
    threads = threads or os.cpu_count() or 1
    _check(lib().oracle_sparse_sink_attn(
        _ptr(q), q.strides[0] // 2, q.strides[1] // 2, N, H, d,
        _ptr(k_raw), _ptr(v_raw), k_raw.shape[0], k_raw.shape[1], _ptr(pt_raw), pt_raw.shape[1],
        _ptr(k_cmp), _ptr(v_cmp), 0 if k_cmp is None else k_cmp.shape[0],
        1 if k_cmp is None else k_cmp.shape[1], _ptr(pt_cmp),
        0 if pt_cmp is None else pt_cmp.shape[1],
        _ptr(req), pt_raw.shape[0], _ptr(indptr), _ptr(indices), _ptr(sink), float(scale),
        1 if include_sink else 0, _ptr(rows), n_rows, _ptr(out), _ptr(lse), int(threads)))
    return out, lse


def sparse_sink_attn_bwd(q, k_raw, v_raw, pt_raw, req, indptr, indices, sink, scale, dout,
                         k_cmp=None, v_cmp=None, pt_cmp=None, rows=None, threads=None,
                         o_saved=None, lse_saved=None):
    """FP64 gradients of sum(dout * O) from the exact forward, or from saved
    forward results: o_saved [N, H, d] (for D = dO . O) and lse_saved [N, H]
    (for the probabilities), FP64 arrays, each optional.

    Returns (dq [n_rows, H, d], dk_raw, dv_raw, dk_cmp, dv_cmp, dsink [H]);
    dk/dv are shaped like their pools ([pages, page_size, d]) and hold the
    contributions of the given query tokens only (all of them when rows is
    None); dk_cmp/dv_cmp are None without a compressed pool and dsink is
    None without a sink. dout: BF16 bits [N, H, d].
    """
    q = np.asarray(q)
    assert q.dtype == np.uint16 and q.ndim == 3 and q.strides[2] == 2
    N, H, d = q.shape
    k_raw, v_raw = _c(k_raw, np.uint16), _c(v_raw, np.uint16)
    pt_raw = _c(pt_raw, np.int32)
    if pt_cmp is not None:
        k_cmp, v_cmp, pt_cmp = _c(k_cmp, np.uint16), _c(v_cmp, np.uint16), _c(pt_cmp, np.int32)
    req, indptr, indices = _c(req, np.int32), _c(indptr, np.int32), _c(indices, np.int32)
    sink = _c(sink, np.float32)
    dout = _c(dout, np.uint16)
    assert dout.shape == (N, H, d)
    o_saved = None if o_saved is None else _c(o_saved, np.float64).reshape(N, H, d)
    lse_saved = None if lse_saved is None else _c(lse_saved, np.float64).reshape(N, H)
    rows = None if rows is None else _c(rows, np.int32)
    n_rows = N if rows is None else rows.shape[0]
    dq = np.zeros((n_rows, H, d), dtype=np.float64)
    dk_raw = np.zeros(k_raw.shape, dtype=np.float64)
    dv_raw = np.zeros(v_raw.shape, dtype=np.float64)
    dk_cmp = None if k_cmp is None else np.zeros(k_cmp.shape, dtype=np.float64)
    dv_cmp = None if v_cmp is None else np.zeros(v_cmp.shape, dtype=np.float64)
    dsink = None if sink is None else np.zeros(H, dtype=np.float64)
    threads = threads or os.cpu_count() or 1
    _check(lib().oracle_sparse_sink_attn_bwd(
        _ptr(q), q.strides[0] // 2, q.strides[1] // 2, N, H, d,
        _ptr(k_raw), _ptr(v_raw), k_raw.shape[0], k_raw.shape[1], _ptr(pt_raw), pt_raw.shape[1],
        _ptr(k_cmp), _ptr(v_cmp), 0 if k_cmp is None else k_cmp.shape[0],
        1 if k_cmp is None else k_cmp.shape[1], _ptr(pt_cmp),
        0 if pt_cmp is None else pt_cmp.shape[1],
        _ptr(req), pt_raw.shape[0], _ptr(indptr), _ptr(indices), _ptr(sink), float(scale),
        _ptr(dout), _ptr(o_saved), _ptr(lse_saved), _ptr(rows), n_rows, _ptr(dq), _ptr(dk_raw), _ptr(dv_raw), _ptr(dk_cmp),
        _ptr(dv_cmp), _ptr(dsink), int(threads)))
    return dq, dk_raw, dv_raw, dk_cmp, dv_cmp, dsink


def lse_merge(lse_parts, o_parts):
    """Merge partials (LSE_s [S], O_s [S, d]) of one (query, head)."""
    lse_parts = _c(lse_parts, np.float64)
    o_parts = _c(o_parts, np.float64)
    S, d = o_parts.shape
    o = np.zeros(d, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib().oracle_lse_merge(S, _ptr(lse_parts), _ptr(o_parts), d, _ptr(o), _ptr(lse))
    return o, float(lse[0])


def ue8m0_to_double(code: int) -> float:
    return lib().oracle_ue8m0_to_double(int(code))


def unpack_d512_pages(src, page_ids, dst=None):
    """BF16 bits [pages, page_size, 512] of the listed pages of a packed
    cache (uint8 [pages, page_size, 584]: 448 E4M3 codes, 64 BF16, 7 UE8M0
    scale bytes, 1 unused byte per token)."""
    src = _c(src, np.uint8)
    P, ps, w = src.shape
    assert w == 584
    page_ids = _c(page_ids, np.int32)
    if dst is None:
        dst = np.zeros((P, ps, 512), dtype=np.uint16)
    assert dst.dtype == np.uint16 and dst.flags.c_contiguous and dst.shape == (P, ps, 512)
    _check(lib().oracle_unpack_d512_pages(_ptr(src), P, ps, _ptr(page_ids), page_ids.shape[0], _ptr(dst)))
    return dst


def paged_kv_write(k_new, v_new, req, pos, pt, k_pool, v_pool):
    """Copies of the pools (uint16 BF16 bits [pages, page_size, d]) with token
    j's rows written at pt[req[j]][pos[j] // ps] * ps + pos[j] % ps, and the
    fault flags (2: bad request/position, 1: bad page; 0: none)."""
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    req = _c(req, np.int32)
    pos = _c(pos, np.int32)
    pt = _c(pt, np.int32)
    k_out = np.array(k_pool, dtype=np.uint16, copy=True, order="C")
    v_out = np.array(v_pool, dtype=np.uint16, copy=True, order="C")
    P, ps, d = k_out.shape
    n = k_new.shape[0]
    flags = lib().oracle_paged_kv_write(_ptr(k_new), _ptr(v_new), n, d, _ptr(req), _ptr(pos), _ptr(pt),
                                        pt.shape[1], pt.shape[0], ps, P, _ptr(k_out), _ptr(v_out))
    return k_out, v_out, flags

