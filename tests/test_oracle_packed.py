"""Pins for the oracle's decode of the packed 512-wide row (584 bytes per
token: 448 E4M3 codes, 64 BF16 values, 7 UE8M0 scale bytes, 1 unused byte),
the layout read from page "Roadmap item 24 - joint compressed/window
attention with sink", review notes on the packed joint KV gather (584 bytes
per token at head width 512, 576 of them data). Each test checks the oracle
against closed forms or PyTorch's own FP8 / BF16 conversions."""
import math

import numpy as np
import pytest
import torch

from sparse_paged_attention_build_b200 import workloads


def test_ue8m0_closed_forms(oracle):
    assert oracle.ue8m0_to_double(127) == 1.0
    assert oracle.ue8m0_to_double(128) == 2.0
    assert oracle.ue8m0_to_double(120) == 2.0 ** -7
    assert oracle.ue8m0_to_double(0) == 2.0 ** -127
    assert oracle.ue8m0_to_double(254) == 2.0 ** 127
    assert math.isnan(oracle.ue8m0_to_double(255))


def _torch_route(src):
    """The same decode by PyTorch: float8_e4m3fn -> float32, times the
    float32 power of two, rounded to BF16; the BF16 tail reinterpreted."""
    P, ps, _ = src.shape
    codes = torch.from_numpy(np.ascontiguousarray(src[..., :448])).view(torch.float8_e4m3fn).to(torch.float32)
    s = torch.from_numpy(src[..., 576:583].astype(np.int32) - 127)
    scale = torch.pow(torch.tensor(2.0, dtype=torch.float32), s.to(torch.float32))       # exact powers of two
    vals = (codes.view(P, ps, 7, 64) * scale[..., None]).view(P, ps, 448)
    head = vals.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    tail = np.ascontiguousarray(src[..., 448:576]).view(np.uint16).reshape(P, ps, 64)
    return np.concatenate([head, tail], axis=2)


def test_matches_pytorch_on_random_pages(oracle):
    src = workloads.make_packed_d512(6, 16, seed=1)
    got = oracle.unpack_d512_pages(src, np.arange(6, dtype=np.int32))
    ref = _torch_route(src)
    assert np.array_equal(got, ref)


def test_every_code_at_unit_and_shifted_scales(oracle):
    """All 256 codes (NaN codes compared as NaN) at scale bytes 127, 120,
    133: the value is the E4M3 table entry times 2^(s-127)."""
    table = oracle.e4m3_table()
    for sb in (127, 120, 133):
        src = np.zeros((1, 4, 584), dtype=np.uint8)
        codes = np.arange(256, dtype=np.uint8)
        src[0, :, :448] = np.concatenate([codes, codes[:192]]).reshape(1, 448)
        src[0, :, 576:583] = sb
        out = oracle.unpack_d512_pages(src, np.array([0], dtype=np.int32))
        f = torch.from_numpy(out[0, 0, :448].view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
        ref = np.concatenate([table, table[:192]]) * 2.0 ** (sb - 127)
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(f), nan)
        assert np.array_equal(f[~nan], ref[~nan])     # E4M3 x 2^k is exact in BF16


def test_tail_is_copied_and_pad_byte_ignored(oracle):
    src = workloads.make_packed_d512(2, 8, seed=2)
    a = oracle.unpack_d512_pages(src, np.array([0, 1], dtype=np.int32))
    src2 = src.copy()
    src2[..., 583] = 0xA5
    b = oracle.unpack_d512_pages(src2, np.array([0, 1], dtype=np.int32))
    assert np.array_equal(a, b)
    assert np.array_equal(a[..., 448:], np.ascontiguousarray(src[..., 448:576]).view(np.uint16))


def test_only_listed_pages_and_bad_page(oracle):
    src = workloads.make_packed_d512(3, 4, seed=3)
    dst = np.full((3, 4, 512), 0x1234, dtype=np.uint16)
    oracle.unpack_d512_pages(src, np.array([1], dtype=np.int32), dst)
    assert np.all(dst[0] == 0x1234) and np.all(dst[2] == 0x1234) and not np.all(dst[1] == 0x1234)
    with pytest.raises(oracle.OracleError):
        oracle.unpack_d512_pages(src, np.array([3], dtype=np.int32))
