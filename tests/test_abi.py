"""The C ABI without a GPU: the library loads, exports every symbol that
include/spa.h declares, sizes workspaces, and rejects each bad argument
with its own validation clause before touching the device (the guard
matrix asks that each fault hit a distinct clause: page "Roadmap item 24 -
joint compressed/window attention with sink", review of the ROCm guard
test)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spa.h")


@pytest.fixture(scope="module")
def L():
    from sparse_paged_attention_build_b200 import build
    build.build()
    import sparse_paged_attention_build_b200 as spa
    return spa.lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(spa_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10, names
    so = ctypes.CDLL(os.path.join(ROOT, "sparse_paged_attention_build_b200", "libspa.so"))
    for n in names:
        assert hasattr(so, n), n


def test_host_helpers(L):
    assert L.spa_abi_version() == 1
    assert L.spa_status_string(0) == b"ok"
    assert L.spa_status_string(4) == b"workspace missing or too small"
    # capacity bound: N * (min(W, p+1) + min(K, (p+1)/r))
    assert L.spa_kv_sets_capacity(16384, 128, 4, 512, 1, 8191) == 16384 * 640
    assert L.spa_kv_sets_capacity(64, 128, 128, 0, 0, 65535) == 64 * (128 + 512)
    assert L.spa_kv_sets_capacity(10, 128, 0, 0, 0, 5) == 60
    assert L.spa_build_kv_sets_workspace_size(17) == 3 * 8 + 16
    assert L.spa_sparse_sink_attn_workspace_size(100, 128, 128, 1) == 0
    # up to 8 slices merge inside a cluster: no workspace; more use FP32 partials
    for s in (2, 5, 8):
        assert L.spa_sparse_sink_attn_workspace_size(10, 128, 128, s) == 0
    w12 = L.spa_sparse_sink_attn_workspace_size(10, 128, 128, 12)
    assert w12 >= 10 * 12 * 128 * 128 * 4 + 10 * 12 * 128 * 8 + 10 * 4
    # (no GPU here: 148 SMs assumed, 296 persistent CTAs)
    assert L.spa_sparse_sink_attn_choose_splits(100000, 128, 0) == 1   # prefill fills the GPU
    assert L.spa_sparse_sink_attn_choose_splits(512, 128, 0) == 1
    assert L.spa_sparse_sink_attn_choose_splits(64, 128, 0) == 4       # decode: cluster slices
    assert L.spa_sparse_sink_attn_choose_splits(128, 128, 0) == 2
    assert L.spa_sparse_sink_attn_choose_splits(64, 128, 640) == 4
    assert L.spa_sparse_sink_attn_choose_splits(1, 128, 100) == 2      # no empty slices
    assert L.spa_sparse_sink_attn_choose_splits(1, 128, 65536) == 16   # long set, few queries
    assert 4 <= L.spa_sparse_sink_attn_choose_splits(64, 128, 8192) <= 8


FAKE = 0x10000  # a 16-byte aligned non-NULL address; never dereferenced on these paths


def sets_call(L, **kw):
    a = dict(pos=FAKE, n=8, W=128, ratio=4, topk=FAKE, K=16, indptr=FAKE, indices=FAKE, cap=1000,
             ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    return L.spa_build_kv_sets(a["pos"], a["n"], a["W"], a["ratio"], a["topk"], a["K"], a["indptr"],
                               a["indices"], a["cap"], a["ws"], a["ws_bytes"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(n=-1), 1, "n_queries < 0"),
    (dict(W=0), 1, "window < 1"),
    (dict(ratio=3), 1, "ratio must be"),
    (dict(K=-1), 1, "topk_width < 0"),
    (dict(cap=-1), 1, "capacity < 0"),
    (dict(indptr=None), 1, "indptr is NULL"),
    (dict(pos=None), 1, "pos is NULL"),
    (dict(indices=None), 1, "indices is NULL"),
    (dict(K=4096), 2, "topk_width >"),
    (dict(pos=FAKE + 2), 5, "int32 arrays"),
    (dict(ws=None), 4, "workspace needs"),
    (dict(ws_bytes=8), 4, "workspace needs"),
    (dict(ws=FAKE + 8), 5, "workspace must be 16-byte"),
])
def test_guard_matrix_build_kv_sets(L, kw, status, clause):
    assert sets_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def dq_call(L, **kw):
    a = dict(src=FAKE, scales=FAKE, P=4, ps=64, d=128, ids=FAKE, n=2, fmt=0, dst=FAKE)
    a.update(kw)
    return L.spa_dequant_fp8_pages(a["src"], a["scales"], a["P"], a["ps"], a["d"], a["ids"], a["n"],
                                   a["fmt"], a["dst"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(P=-1), 1, "num_pages < 0"),
    (dict(ps=0), 1, "page_size < 1"),
    (dict(d=0), 1, "head_dim < 1"),
    (dict(n=-1), 1, "n_page_ids < 0"),
    (dict(fmt=7), 1, "fp8_format must be 0"),
    (dict(d=96), 2, "multiple of 64"),
    (dict(src=None), 1, "must be non-NULL"),
    (dict(dst=FAKE + 4), 5, "src and dst must be 16-byte"),
    (dict(scales=FAKE + 1), 5, "scales/page_ids"),
])
def test_guard_matrix_dequant(L, kw, status, clause):
    assert dq_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def attn_call(L, **kw):
    a = dict(q=FAKE, sq=16384, sh=128, n=4, H=128, d=128, kr=FAKE, vr=FAKE, rp=10, rps=64, ptr=FAKE,
             ptrc=4, kc=FAKE, vc=FAKE, cp=10, cps=64, ptc=FAKE, ptcc=4, req=FAKE, B=1, ip=FAKE,
             idx=FAKE, sink=FAKE, scale=0.088, out=FAKE, lse=FAKE, splits=1, ws=None, wsb=0)
    a.update(kw)
    return L.spa_sparse_sink_attn_fwd(
        a["q"], a["sq"], a["sh"], a["n"], a["H"], a["d"], a["kr"], a["vr"], a["rp"], a["rps"], a["ptr"],
        a["ptrc"], a["kc"], a["vc"], a["cp"], a["cps"], a["ptc"], a["ptcc"], a["req"], a["B"], a["ip"],
        a["idx"], a["sink"], a["scale"], a["out"], a["lse"], a["splits"], a["ws"], a["wsb"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(n=-1), 1, "n_queries < 0"),
    (dict(H=0), 1, "num_heads < 1"),
    (dict(B=0), 1, "n_requests < 1"),
    (dict(d=96), 2, "head_dim must be 64, 128 or 512"),
    (dict(H=192), 2, "multiple of 128"),
    (dict(d=512, H=48), 2, "head_dim 512: num_heads above 32"),
    (dict(d=512, H=32, splits=9), 2, "head_dim 512: num_splits at most"),
    (dict(rp=-1), 1, "raw pool sizes"),
    (dict(rps=0), 1, "raw_page_size < 1"),
    (dict(rps=48), 2, "raw_page_size must be a power of two"),
    (dict(cp=-1), 1, "compressed pool sizes"),
    (dict(cps=0), 1, "cmp_page_size < 1"),
    (dict(cps=2048), 2, "cmp_page_size must be a power of two"),
    (dict(kc=None), 1, "k_cmp/v_cmp NULL"),
    (dict(scale=0.0), 1, "scale must be finite"),
    (dict(scale=float("inf")), 1, "scale must be finite"),
    (dict(splits=17), 1, "num_splits must be"),
    (dict(sq=-8), 1, "negative q stride"),
    (dict(q=None), 1, "q must be non-NULL"),
    (dict(out=None), 1, "q, out and lse"),
    (dict(vr=None), 1, "k_raw, v_raw and pt_raw"),
    (dict(idx=None), 1, "req, indptr and indices"),
    (dict(sh=129), 5, "q base and strides"),
    (dict(kr=FAKE + 8), 5, "K/V pools"),
    (dict(out=FAKE + 2), 5, "out must be"),
    (dict(lse=FAKE + 2), 5, "32-bit arrays"),
    (dict(splits=12), 4, "workspace needs"),
    (dict(splits=12, ws=FAKE + 16, wsb=1 << 30), 5, "workspace must be 256-byte"),
])
def test_guard_matrix_attention(L, kw, status, clause):
    assert attn_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_attention_zero_queries_is_a_no_op(L):
    assert attn_call(L, n=0, q=None, out=None, lse=None) == 0


def attn_inline_call(L, **kw):
    a = dict(q=FAKE, sq=16384, sh=128, n=4, H=128, d=128, kr=FAKE, vr=FAKE, rp=10, rps=64, ptr=FAKE,
             ptrc=4, kc=FAKE, vc=FAKE, cp=10, cps=64, ptc=FAKE, ptcc=4, req=FAKE, B=1, pos=FAKE, topk=None,
             K=0, W=128, ratio=128, sink=FAKE, scale=0.088, out=FAKE, lse=FAKE, splits=1, ws=None, wsb=0)
    a.update(kw)
    return L.spa_sparse_sink_attn_fwd_inline_sets(
        a["q"], a["sq"], a["sh"], a["n"], a["H"], a["d"], a["kr"], a["vr"], a["rp"], a["rps"], a["ptr"],
        a["ptrc"], a["kc"], a["vc"], a["cp"], a["cps"], a["ptc"], a["ptcc"], a["req"], a["B"], a["pos"],
        a["topk"], a["K"], a["W"], a["ratio"], a["sink"], a["scale"], a["out"], a["lse"], a["splits"], a["ws"],
        a["wsb"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(W=0), 1, "window must be >= 1"),
    (dict(ratio=3), 2, "ratio must be 0, 4 or 128"),
    (dict(K=-1), 1, "topk_width < 0"),
    (dict(ratio=4, topk=FAKE, K=513), 2, "topk_width > 512"),
    (dict(ratio=4, topk=FAKE + 2, K=16), 5, "32-bit arrays"),
    (dict(ptc=None), 1, "ratio > 0 needs the compressed pool"),
    (dict(kc=None), 1, "ratio > 0 needs the compressed pool"),
    (dict(ratio=0, ptc=FAKE, vc=None), 1, "k_cmp/v_cmp NULL"),
    (dict(pos=None), 1, "pos must be non-NULL"),
    (dict(pos=FAKE + 2), 5, "32-bit arrays"),
    (dict(req=None), 1, "req must be non-NULL"),
    (dict(n=-1), 1, "n_queries < 0"),
    (dict(d=96), 2, "head_dim must be 64, 128 or 512"),
    (dict(splits=12), 4, "workspace needs"),
])
def test_guard_matrix_attention_inline_sets(L, kw, status, clause):
    assert attn_inline_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_attention_inline_sets_window_only_needs_no_compressed_pool(L):
    # ratio 0: the window alone; only the zero-query call runs on the CPU
    assert attn_inline_call(L, ratio=0, ptc=None, kc=None, vc=None, n=0, q=None, out=None, lse=None) == 0


def attn8_inline_call(L, **kw):
    a = dict(q=FAKE, sq=16384, sh=128, n=4, H=128, d=128, kr=FAKE, vr=FAKE, rp=10, rps=64, ptr=FAKE,
             ptrc=4, k8=FAKE, v8=FAKE, ks=FAKE, vs=FAKE, cp=10, cps=128, ptc=FAKE, ptcc=4, fmt=0,
             req=FAKE, B=1, pos=FAKE, topk=FAKE, K=512, W=128, ratio=4, sink=FAKE, scale=0.088, out=FAKE,
             lse=FAKE, splits=1, ws=None, wsb=0)
    a.update(kw)
    return L.spa_sparse_sink_attn_fwd_fp8_inline_sets(
        a["q"], a["sq"], a["sh"], a["n"], a["H"], a["d"], a["kr"], a["vr"], a["rp"], a["rps"], a["ptr"],
        a["ptrc"], a["k8"], a["v8"], a["ks"], a["vs"], a["cp"], a["cps"], a["ptc"], a["ptcc"], a["fmt"],
        a["req"], a["B"], a["pos"], a["topk"], a["K"], a["W"], a["ratio"], a["sink"], a["scale"], a["out"],
        a["lse"], a["splits"], a["ws"], a["wsb"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(W=0), 1, "window must be >= 1"),
    (dict(ratio=5), 2, "ratio must be 0, 4 or 128"),
    (dict(K=513), 2, "topk_width > 512"),
    (dict(pos=None), 1, "pos must be non-NULL"),
    (dict(fmt=2), 1, "fp8_format must be 0"),
    (dict(ptc=None), 1, "pt_cmp must be non-NULL on the FP8 path"),
    (dict(ks=None), 1, "FP8 codes and scales must be non-NULL"),
    (dict(d=512), 2, "head_dim 512: the FP8 gather takes 64 or 128"),
    (dict(splits=12), 4, "workspace needs"),
])
def test_guard_matrix_attention_fp8_inline_sets(L, kw, status, clause):
    assert attn8_inline_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_attention_inline_sets_ignores_topk_width_at_ratio_0(L):
    # ratio 0 picks no group, so a row of any width is accepted (and unread)
    assert attn_inline_call(L, ratio=0, topk=FAKE, K=4096, ptc=None, kc=None, vc=None, n=0, q=None, out=None,
                            lse=None) == 0


def attn8_call(L, **kw):
    a = dict(q=FAKE, sq=16384, sh=128, n=4, H=128, d=128, kr=FAKE, vr=FAKE, rp=10, rps=64, ptr=FAKE,
             ptrc=4, k8=FAKE, v8=FAKE, ks=FAKE, vs=FAKE, cp=10, cps=128, ptc=FAKE, ptcc=4, fmt=0,
             req=FAKE, B=1, ip=FAKE, idx=FAKE, sink=FAKE, scale=0.088, out=FAKE, lse=FAKE, splits=1,
             ws=None, wsb=0)
    a.update(kw)
    return L.spa_sparse_sink_attn_fwd_fp8(
        a["q"], a["sq"], a["sh"], a["n"], a["H"], a["d"], a["kr"], a["vr"], a["rp"], a["rps"], a["ptr"],
        a["ptrc"], a["k8"], a["v8"], a["ks"], a["vs"], a["cp"], a["cps"], a["ptc"], a["ptcc"], a["fmt"],
        a["req"], a["B"], a["ip"], a["idx"], a["sink"], a["scale"], a["out"], a["lse"], a["splits"],
        a["ws"], a["wsb"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(fmt=3), 1, "fp8_format must be 0"),
    (dict(ptc=None), 1, "pt_cmp must be non-NULL"),
    (dict(ks=None), 1, "codes and scales"),
    (dict(v8=None), 1, "codes and scales"),
    (dict(n=-1), 1, "n_queries < 0"),
    (dict(cps=96), 2, "cmp_page_size must be a power of two"),
    (dict(k8=FAKE + 8), 5, "K/V pools"),
    (dict(vs=FAKE + 2), 5, "32-bit arrays"),
    (dict(splits=12), 4, "workspace needs"),
])
def test_guard_matrix_attention_fp8(L, kw, status, clause):
    assert attn8_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_attention_fp8_zero_queries_is_a_no_op(L):
    assert attn8_call(L, n=0, q=None, out=None, lse=None, k8=None, v8=None, ks=None, vs=None) == 0


def kvw_call(L, **kw):
    a = dict(kn=FAKE, vn=FAKE, n=4, d=128, req=FAKE, pos=FAKE, pt=FAKE, cols=4, B=2, ps=64, P=10,
             kp=FAKE, vp=FAKE)
    a.update(kw)
    return L.spa_paged_kv_write(a["kn"], a["vn"], a["n"], a["d"], a["req"], a["pos"], a["pt"], a["cols"], a["B"],
                                a["ps"], a["P"], a["kp"], a["vp"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(n=-1), 1, "n_tokens < 0"),
    (dict(d=12), 2, "multiple of 8"),
    (dict(B=0), 1, "n_requests and pt_cols"),
    (dict(P=-1), 1, "num_pages < 0"),
    (dict(ps=48), 2, "page_size must be a power of two"),
    (dict(pt=None), 1, "must be non-NULL"),
    (dict(kp=FAKE + 4), 5, "16-byte aligned"),
    (dict(pos=FAKE + 2), 5, "4-byte aligned"),
])
def test_guard_matrix_kv_write(L, kw, status, clause):
    assert kvw_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_kv_write_zero_tokens_is_a_no_op(L):
    assert kvw_call(L, n=0, kn=None, vn=None) == 0


def bwd_call(L, **kw):
    a = dict(q=FAKE, sq=16384, sh=128, n=4, H=128, d=128, kr=FAKE, vr=FAKE, rp=10, rps=64, ptr=FAKE,
             ptrc=4, kc=FAKE, vc=FAKE, cp=10, cps=64, ptc=FAKE, ptcc=4, req=FAKE, B=1, ip=FAKE,
             idx=FAKE, sink=FAKE, scale=0.088, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dkr=FAKE,
             dvr=FAKE, dkc=FAKE, dvc=FAKE, dsink=FAKE, splits=1)
    a.update(kw)
    return L.spa_sparse_sink_attn_bwd(
        a["q"], a["sq"], a["sh"], a["n"], a["H"], a["d"], a["kr"], a["vr"], a["rp"], a["rps"], a["ptr"],
        a["ptrc"], a["kc"], a["vc"], a["cp"], a["cps"], a["ptc"], a["ptcc"], a["req"], a["B"], a["ip"],
        a["idx"], a["sink"], a["scale"], a["out"], a["lse"], a["dout"], a["dq"], a["dkr"], a["dvr"],
        a["dkc"], a["dvc"], a["dsink"], a["splits"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(n=-1), 1, "n_queries < 0"),
    (dict(d=96), 2, "head_dim must be 64, 128 or 512"),
    (dict(d=512, H=32), 2, "the backward takes head_dim 64 or 128"),
    (dict(rps=48), 2, "raw_page_size must be a power of two"),
    (dict(kc=None), 1, "k_cmp/v_cmp NULL"),
    (dict(splits=17), 1, "num_splits must be"),
    (dict(q=None), 1, "q must be non-NULL"),
    (dict(dout=None), 1, "out, lse and dout"),
    (dict(lse=None), 1, "out, lse and dout"),
    (dict(dq=None), 1, "dq, dk_raw and dv_raw"),
    (dict(dvr=None), 1, "dq, dk_raw and dv_raw"),
    (dict(dkc=None), 1, "dk_cmp/dv_cmp NULL"),
    (dict(dq=FAKE + 4), 5, "out, dout, dq, dk and dv"),
    (dict(dout=FAKE + 2), 5, "out, dout, dq, dk and dv"),
    (dict(dkr=FAKE + 4), 5, "out, dout, dq, dk and dv"),
    (dict(lse=FAKE + 2), 5, "32-bit arrays"),
    (dict(dsink=FAKE + 1), 5, "32-bit arrays"),
])
def test_guard_matrix_attention_bwd(L, kw, status, clause):
    assert bwd_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_attention_bwd_zero_queries_is_a_no_op(L):
    assert bwd_call(L, n=0, q=None, out=None, lse=None, dout=None, dq=None, dkr=None, dvr=None) == 0


def unpack_call(L, **kw):
    a = dict(src=FAKE, P=10, ps=64, ids=FAKE, n=4, dst=FAKE)
    a.update(kw)
    return L.spa_unpack_d512_pages(a["src"], a["P"], a["ps"], a["ids"], a["n"], a["dst"], None, None)


@pytest.mark.parametrize("kw,status,clause", [
    (dict(P=-1), 1, "num_pages < 0"),
    (dict(ps=0), 1, "page_size < 1"),
    (dict(n=-1), 1, "n_page_ids < 0"),
    (dict(ps=8192), 2, "page_size above 4096"),
    (dict(src=None), 1, "src, page_ids and dst must be non-NULL"),
    (dict(ids=None), 1, "src, page_ids and dst must be non-NULL"),
    (dict(src=FAKE + 4), 5, "src must be 8-byte aligned"),
    (dict(dst=FAKE + 8), 5, "dst must be 16-byte aligned"),
    (dict(ids=FAKE + 2), 5, "page_ids misaligned"),
])
def test_guard_matrix_unpack_d512(L, kw, status, clause):
    assert unpack_call(L, **kw) == status
    assert clause in L.spa_last_error_detail().decode()


def test_unpack_d512_zero_pages_is_a_no_op(L):
    assert unpack_call(L, n=0, src=None, ids=None, dst=None) == 0
