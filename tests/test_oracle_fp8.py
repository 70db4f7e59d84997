"""Pins for the oracle's FP8 page decode and its BF16 rounding.

The mixed cache stores compressed KV as FP8 with an explicit OCP format
(page "Roadmap item 24 - joint compressed/window attention with sink",
section "Reuse and arithmetic"): OCP E4M3, one FP32 scale per 64 elements,
decoded to BF16.
"""
import math

import numpy as np
import torch


def test_e4m3_definition_points(oracle):
    assert oracle.e4m3_to_double(0x7E) == 448.0          # largest finite
    assert oracle.e4m3_to_double(0xFE) == -448.0
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_to_double(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert oracle.e4m3_to_double(0x38) == 1.0            # exponent field 7 = bias
    assert oracle.e4m3_to_double(0x78) == 256.0          # S.1111.000 is finite
    assert oracle.e4m3_to_double(0x00) == 0.0
    v = oracle.e4m3_to_double(0x80)
    assert v == 0.0 and math.copysign(1.0, v) < 0
    assert math.isnan(oracle.e4m3_to_double(0x7F))
    assert math.isnan(oracle.e4m3_to_double(0xFF))


def test_e4m3_all_codes_match_torch_float8(oracle):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = oracle.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(mine[~nan]))


def test_e4m3_encode_round_trip(oracle):
    """Every finite code survives encode(decode(code)) through torch."""
    table = oracle.e4m3_table()
    finite = np.where(~np.isnan(table))[0]
    back = torch.from_numpy(table[finite].astype(np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()
    # +0 and -0 both decode to zero; everything else maps back to itself
    assert np.array_equal(back.astype(np.int64), finite)


def test_bf16_rne_matches_torch(oracle):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(2000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 2000),
        # exact ties between two BF16 values, both parities of the kept LSB
        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38, 1e-40, np.inf, -np.inf], dtype=np.float32),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = np.array([oracle.float_to_bf16_rne(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(mine, ref)


def test_dequant_matches_torch_route(oracle):
    """bf16(float32(e4m3) * float32 scale) recomputed through torch's own
    float8 decode, float32 multiply and bfloat16 rounding."""
    rng = np.random.default_rng(1)
    P, ps, d = 6, 16, 128
    src = rng.integers(0, 256, size=(P, ps, d), dtype=np.uint8)
    src[src == 0x7F] = 0x7E
    src[src == 0xFF] = 0xFE
    scales = (rng.random((P, ps, d // 64)) * 3.0 + 1e-3).astype(np.float32)
    page_ids = np.array([4, 0, 2], dtype=np.int32)
    dst = oracle.dequant_fp8_pages(src, scales, page_ids)
    x = torch.from_numpy(src).view(torch.float8_e4m3fn).to(torch.float32)
    s = torch.from_numpy(scales).repeat_interleave(64, dim=2)
    ref = (x * s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for p in range(P):
        if p in page_ids:
            assert np.array_equal(dst[p], ref[p])
        else:
            assert np.all(dst[p] == 0)        # unlisted pages untouched


def test_dequant_generator_values_are_within_a_scale_of_n01():
    """The mixed workload's encoding: |x / s| <= 448 with s = amax / 448."""
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make("c5", shrink=64)
    codes = torch.from_numpy(w.k_cmp_fp8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.nanmax(np.abs(codes)) <= 448.0
    assert not np.isnan(codes).any()


# ---------------------------------------------------------------- E4M3 FNUZ
# The page also names the FNUZ flavour of E4M3 (bias 8, no negative zero,
# 0x80 the only NaN, largest magnitude 240).

def test_e4m3fnuz_definition_points(oracle):
    assert oracle.e4m3fnuz_to_double(0x7F) == 240.0        # largest finite: no NaN at S.1111.111
    assert oracle.e4m3fnuz_to_double(0xFF) == -240.0
    assert oracle.e4m3fnuz_to_double(0x08) == 2.0 ** -7    # smallest normal
    assert oracle.e4m3fnuz_to_double(0x01) == 2.0 ** -10   # smallest subnormal
    assert oracle.e4m3fnuz_to_double(0x40) == 1.0          # exponent field 8 = bias
    assert oracle.e4m3fnuz_to_double(0x00) == 0.0
    assert math.isnan(oracle.e4m3fnuz_to_double(0x80))     # no -0: the code is the NaN
    # the same code is worth half its OCP value wherever both are finite
    for c in range(256):
        if c in (0x7F, 0xFF, 0x80):
            continue
        assert oracle.e4m3fnuz_to_double(c) == 0.5 * oracle.e4m3_to_double(c)


def test_e4m3fnuz_all_codes_match_torch_float8(oracle):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fnuz).to(torch.float64).numpy()
    mine = oracle.e4m3fnuz_table()
    nan = np.isnan(ref)
    assert nan.sum() == 1
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])


def test_e4m3fnuz_encode_round_trip(oracle):
    table = oracle.e4m3fnuz_table()
    finite = np.where(~np.isnan(table))[0]
    back = torch.from_numpy(table[finite].astype(np.float32)).to(torch.float8_e4m3fnuz) \
        .view(torch.uint8).numpy()
    assert np.array_equal(back.astype(np.int64), finite)


def test_dequant_fnuz_matches_torch_route(oracle):
    rng = np.random.default_rng(3)
    P, ps, d = 4, 16, 128
    src = rng.integers(0, 256, size=(P, ps, d), dtype=np.uint8)
    src[src == 0x80] = 0x00
    scales = (rng.random((P, ps, d // 64)) * 3.0 + 1e-3).astype(np.float32)
    page_ids = np.array([3, 1], dtype=np.int32)
    dst = oracle.dequant_fp8_pages(src, scales, page_ids, fmt=1)
    x = torch.from_numpy(src).view(torch.float8_e4m3fnuz).to(torch.float32)
    s = torch.from_numpy(scales).repeat_interleave(64, dim=2)
    ref = (x * s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for p in page_ids:
        assert np.array_equal(dst[p], ref[p])
    # the two formats differ on the same bytes
    ocp = oracle.dequant_fp8_pages(src, scales, page_ids, fmt=0)
    assert not np.array_equal(ocp[3], dst[3])
