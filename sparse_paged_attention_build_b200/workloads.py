"""Seeded synthetic inputs shaped like the workloads of the pages.

This module only draws random inputs; it holds none of the method's
arithmetic (no key sets, no softmax, no decoding). Both the CUDA path and the
CPU oracle read the arrays it returns. BF16 values are returned as their
uint16 bit patterns (rounded to nearest even from FP32 normals by PyTorch);
FP8 caches are returned as OCP E4M3 bytes (encoded by PyTorch's
``float8_e4m3fn`` cast) with one FP32 scale per 64 elements of a row.

The five workloads:

``c1``  tiny ratio-4 prefill: 2 requests x 256 tokens, H=8, d=64, W=64,
        64 compressed entries per request, top-k 16, page size 16.
``c2``  dense sliding-window (ratio 0) prefill: 4 x 2560 tokens, H=128,
        d=128, W=128, page size 64, pool of 2x the needed pages.
``c3``  ratio-4 (CSA) prefill: 2 x 8192 tokens, H=128, d=128, W=128,
        seqlen/4 compressed entries, top-k 512, page size 64.
``c4``  ratio-128 (HCA) decode: 64 requests x 1 query, context lengths
        uniform in [16384, 65536], H=128, d=128, W=128, page size 64.
``c5``  mixed FP8/BF16 ratio-4 decode: 128 requests x 1 query, context
        32768, H=128, d=128, top-k 512 + W=128, FP8 compressed cache with
        per-64 FP32 scales, page size 128.

Two more at the DSV4-Flash attention shape (32 query heads, head width
512, the BF16 rows that the packed 584-byte cache decodes to):

``f1``  ratio-4 prefill: 1 request x 1024 tokens, H=32, d=512, W=128,
        top-k 512, page size 64.
``f2``  ratio-4 decode: 64 requests x 1 query, context 8192 (the input
        length of the pages' serving timeline), H=32, d=512, top-k 512 +
        W=128, page size 64.

``shrink`` keeps every per-token shape (H, d, W, K, page size) and reduces
only the number of requests and tokens, for parity cases the oracle finishes
in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BASE_SEED = 20261202
WINDOW_TAG = 1 << 30


@dataclass
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    N: int
    H: int
    d: int
    W: int
    ratio: int
    K: int                    # top-k width (0 when the layer has no top-k list)
    B: int
    q: np.ndarray             # uint16 [N, H, d]
    pos: np.ndarray           # int32 [N]
    req: np.ndarray           # int32 [N]
    topk: np.ndarray | None   # int32 [N, K], -1 padded
    k_raw: np.ndarray         # uint16 [P_raw, ps_raw, d]
    v_raw: np.ndarray
    pt_raw: np.ndarray        # int32 [B, cols_raw]
    k_cmp: np.ndarray | None  # uint16 [P_cmp, ps_cmp, d] (BF16 caches)
    v_cmp: np.ndarray | None
    pt_cmp: np.ndarray | None # int32 [B, cols_cmp]
    sink: np.ndarray          # float32 [H]
    scale: float
    # FP8 compressed cache (mixed workload only)
    k_cmp_fp8: np.ndarray | None = None   # uint8 [P_cmp, ps_cmp, d]
    v_cmp_fp8: np.ndarray | None = None
    k_cmp_scale: np.ndarray | None = None # float32 [P_cmp, ps_cmp, d/64]
    v_cmp_scale: np.ndarray | None = None
    cmp_page_ids: np.ndarray | None = None  # int32: pages holding compressed entries
    meta: dict = field(default_factory=dict)
    fp8_format: int = 0                       # 0 = OCP E4M3, 1 = E4M3 FNUZ

    @property
    def raw_page_size(self):
        return self.k_raw.shape[1]

    @property
    def cmp_page_size(self):
        if self.k_cmp is not None:
            return self.k_cmp.shape[1]
        if self.k_cmp_fp8 is not None:
            return self.k_cmp_fp8.shape[1]
        return 1


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return _bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _e4m3_with_scales(rng: np.random.Generator, shape, fmt: int = 0):
    """x ~ N(0,1); per 64-element group s = max|x| / fmax; byte = e4m3(x / s)
    with fmax = 448 for OCP E4M3 (fmt 0) or 240 for E4M3 FNUZ (fmt 1)."""
    P, ps, d = shape
    fmax, dtype = (448.0, torch.float8_e4m3fn) if fmt == 0 else (240.0, torch.float8_e4m3fnuz)
    x = rng.standard_normal((P, ps, d // 64, 64), dtype=np.float32)
    amax = np.abs(x).max(axis=-1, keepdims=True)
    s = np.where(amax > 0, amax / np.float32(fmax), np.float32(1.0)).astype(np.float32)
    y = np.clip(x / s, -fmax, fmax).astype(np.float32)
    codes = torch.from_numpy(y).to(dtype).view(torch.uint8).numpy()
    return codes.reshape(P, ps, d).copy(), s.reshape(P, ps, d // 64).copy()


def _page_table(rng: np.random.Generator, B: int, cols: int, pool_pages: int) -> np.ndarray:
    """Distinct random page ids for every (request, logical page)."""
    perm = rng.permutation(pool_pages)[: B * cols]
    return perm.reshape(B, cols).astype(np.int32)


def _draw_topk(rng: np.random.Generator, pos: np.ndarray, ratio: int, K: int) -> np.ndarray:
    """Per query, K group ids drawn uniformly without replacement among the
    groups whose ``ratio`` tokens all lie at or before the query (all of them
    when there are fewer), padded with -1."""
    out = np.full((pos.shape[0], K), -1, dtype=np.int32)
    for i, p in enumerate(pos.tolist()):
        avail = (p + 1) // ratio
        take = min(K, avail)
        if take:
            out[i, :take] = rng.choice(avail, take, replace=False)
    return out


def _prefill(name, seed, B, S, H, d, W, ratio, K, ps, pool_factor, cmp_per_req):
    ss = np.random.SeedSequence(seed)
    r_q, r_kv, r_cmp, r_sink, r_pt, r_topk = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]
    N = B * S
    pos = np.tile(np.arange(S, dtype=np.int32), B)
    req = np.repeat(np.arange(B, dtype=np.int32), S)
    q = _normal_bf16(r_q, (N, H, d))
    cols_raw = -(-S // ps)
    p_raw = pool_factor * B * cols_raw
    k_raw = _normal_bf16(r_kv, (p_raw, ps, d))
    v_raw = _normal_bf16(r_kv, (p_raw, ps, d))
    pt_raw = _page_table(r_pt, B, cols_raw, p_raw)
    k_cmp = v_cmp = pt_cmp = topk = None
    if ratio > 0:
        cols_cmp = -(-cmp_per_req // ps)
        p_cmp = pool_factor * B * cols_cmp
        k_cmp = _normal_bf16(r_cmp, (p_cmp, ps, d))
        v_cmp = _normal_bf16(r_cmp, (p_cmp, ps, d))
        pt_cmp = _page_table(r_pt, B, cols_cmp, p_cmp)
        if K > 0:
            topk = _draw_topk(r_topk, pos, ratio, K)
    sink = r_sink.standard_normal(H, dtype=np.float32)
    return Workload(name, "prefill", N, H, d, W, ratio, K if topk is not None else 0, B, q, pos, req,
                    topk, k_raw, v_raw, pt_raw, k_cmp, v_cmp, pt_cmp, sink, 1.0 / float(np.sqrt(d)))


def _zero_pool_with_pages(rng, P, ps, d, pages):
    """A pool of P pages where only ``pages`` hold N(0,1) BF16 rows; the rest
    is zero (never referenced)."""
    pool = np.zeros((P, ps, d), dtype=np.uint16)
    pages = np.asarray(sorted(set(int(x) for x in pages)), dtype=np.int64)
    if pages.size:
        pool[pages] = _normal_bf16(rng, (pages.size, ps, d))
    return pool


def _decode(name, seed, B, lengths, H, d, W, ratio, K, ps, fp8, fmt=0):
    ss = np.random.SeedSequence(seed)
    r_q, r_kv, r_cmp, r_sink, r_pt, r_topk = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]
    lengths = np.asarray(lengths, dtype=np.int64)
    N = B
    pos = (lengths - 1).astype(np.int32)
    req = np.arange(B, dtype=np.int32)
    q = _normal_bf16(r_q, (N, H, d))
    # raw cache: every request's pages cover its whole context
    cols_raw = int(-(-lengths.max() // ps))
    need_raw = [int(-(-L // ps)) for L in lengths]
    p_raw = int(sum(need_raw))
    perm = r_pt.permutation(p_raw).astype(np.int32)
    pt_raw = np.full((B, cols_raw), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need_raw):
        pt_raw[b, :n] = perm[off: off + n]
        off += n
    # only the pages under the last W tokens are ever read: fill those
    win_pages = []
    for b, L in enumerate(lengths.tolist()):
        for lp in range(max(0, L - W) // ps, (L - 1) // ps + 1):
            win_pages.append(pt_raw[b, lp])
    k_raw = _zero_pool_with_pages(r_kv, p_raw, ps, d, win_pages)
    v_raw = _zero_pool_with_pages(r_kv, p_raw, ps, d, win_pages)
    # compressed cache: one entry per complete group of the context
    groups = lengths // ratio
    cols_cmp = int(max(1, -(-groups.max() // ps)))
    need_cmp = [int(-(-g // ps)) for g in groups]
    p_cmp = int(max(1, sum(need_cmp)))
    perm = r_pt.permutation(p_cmp).astype(np.int32)
    pt_cmp = np.full((B, cols_cmp), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need_cmp):
        pt_cmp[b, :n] = perm[off: off + n]
        off += n
    cmp_page_ids = pt_cmp[pt_cmp >= 0].astype(np.int32)
    k_cmp = v_cmp = None
    kf8 = vf8 = ks = vs = None
    if fp8:
        kf8, ks = _e4m3_with_scales(r_cmp, (p_cmp, ps, d), fmt)
        vf8, vs = _e4m3_with_scales(r_cmp, (p_cmp, ps, d), fmt)
    else:
        k_cmp = _normal_bf16(r_cmp, (p_cmp, ps, d))
        v_cmp = _normal_bf16(r_cmp, (p_cmp, ps, d))
    topk = _draw_topk(r_topk, pos, ratio, K) if K > 0 else None
    sink = r_sink.standard_normal(H, dtype=np.float32)
    return Workload(name, "decode", N, H, d, W, ratio, K, B, q, pos, req, topk,
                    k_raw, v_raw, pt_raw, k_cmp, v_cmp, pt_cmp, sink, 1.0 / float(np.sqrt(d)),
                    kf8, vf8, ks, vs, cmp_page_ids, {"lengths": lengths}, fmt)


DESCRIPTIONS = {
    "c1": "tiny ratio-4 prefill: B=2 x 256 tokens, H=8, d=64, W=64, top-k 16, page 16",
    "c2": "dense sliding-window prefill: B=4 x 2560 tokens, H=128, d=128, W=128, page 64",
    "c3": "ratio-4 CSA prefill: B=2 x 8192 tokens, H=128, d=128, W=128, top-k 512, page 64",
    "c4": "ratio-128 HCA decode: 64 requests, context U[16384, 65536], H=128, d=128, W=128, page 64",
    "c5": "mixed FP8/BF16 ratio-4 decode: 128 requests, context 32768, H=128, d=128, top-k 512, W=128, page 128",
    "f1": "DSV4-Flash-shaped ratio-4 prefill: B=1 x 1024 tokens, H=32, d=512, W=128, top-k 512, page 64",
    "f2": "DSV4-Flash-shaped ratio-4 decode: 64 requests, context 8192, H=32, d=512, top-k 512, W=128, page 64",
}


def make(name: str, shrink: int = 1, seed_offset: int = 0, fp8_format: int = 0) -> Workload:
    """The named workload. ``shrink`` > 1 divides the number of requests and
    the tokens per request (prefill) or the context lengths (decode).
    ``fp8_format`` picks the encoding of the mixed cache (c5): 0 = OCP
    E4M3, 1 = E4M3 FNUZ."""
    idx = int(name[1:]) + (100 if name[0] == "f" else 0)
    seed = BASE_SEED + idx + 1000 * seed_offset
    if name == "c1":
        return _prefill(name, seed, 2, max(16, 256 // shrink), 8, 64, 64, 4, 16, 16, 2, max(4, 64 // shrink))
    if name == "c2":
        return _prefill(name, seed, max(1, 4 // shrink), max(64, 2560 // shrink), 128, 128, 128, 0, 0, 64, 2, 0)
    if name == "c3":
        S = max(64, 8192 // shrink)
        return _prefill(name, seed, max(1, 2 // shrink), S, 128, 128, 128, 4, 512, 64, 2, S // 4)
    if name == "c4":
        B = max(1, 64 // shrink)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed).spawn(7)[6]))
        lo, hi = max(129, 16384 // shrink), max(130, 65536 // shrink)
        lengths = rng.integers(lo, hi, size=B, endpoint=True)
        return _decode(name, seed, B, lengths, 128, 128, 128, 128, 0, 64, fp8=False)
    if name == "c5":
        B = max(1, 128 // shrink)
        L = max(1024, 32768 // shrink)
        return _decode(name, seed, B, np.full(B, L), 128, 128, 128, 4, 512, 128, fp8=True, fmt=fp8_format)
    if name == "f1":
        S = max(128, 1024 // shrink)
        return _prefill(name, seed, 1, S, 32, 512, 128, 4, 512, 64, 2, S // 4)
    if name == "f2":
        B = max(1, 64 // shrink)
        L = max(1024, 8192 // shrink)
        return _decode(name, seed, B, np.full(B, L), 32, 512, 128, 4, 512, 64, fp8=False)
    raise KeyError(name)


def make_dout(w: Workload, seed: int = 0) -> np.ndarray:
    """A seeded output gradient dO for a workload: BF16 bits [N, H, d], N(0,1)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([BASE_SEED, 77, seed])))
    return _normal_bf16(rng, (w.N, w.H, w.d))


PACKED_D512_BYTES = 584


def make_packed_d512(num_pages: int, page_size: int, seed: int = 0) -> np.ndarray:
    """A seeded packed cache of 512-wide rows, uint8 [num_pages, page_size,
    584]: per token 448 E4M3 codes (N(0,1) values divided by a power-of-two
    scale per 64, the smallest that keeps them within 448, encoded by
    PyTorch's float8_e4m3fn cast), 64 BF16 N(0,1) values, 7 UE8M0 scale
    bytes (127 + log2 of the scale) and one zero byte."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([BASE_SEED, 584, seed])))
    x = rng.standard_normal((num_pages, page_size, 7, 64)).astype(np.float32)
    amax = np.maximum(np.abs(x).max(axis=3), 1e-30)
    e = np.ceil(np.log2(amax / 448.0)).astype(np.int32)                   # 2^e >= amax / 448
    codes = torch.from_numpy(x / np.ldexp(1.0, e)[..., None].astype(np.float32)).to(torch.float8_e4m3fn)
    out = np.zeros((num_pages, page_size, PACKED_D512_BYTES), dtype=np.uint8)
    out[..., :448] = codes.view(torch.uint8).numpy().reshape(num_pages, page_size, 448)
    rope = _normal_bf16(rng, (num_pages, page_size, 64))
    out[..., 448:576] = rope.view(np.uint8).reshape(num_pages, page_size, 128)
    out[..., 576:583] = (127 + e).astype(np.uint8)
    return out
