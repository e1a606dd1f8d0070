"""Pins of the oracle's MXFP4 quantiser (bf16 -> E2M1 codes + E8M0 scale per 32
elements, the indexer's operand format: m.youleyou.com/wenzhang/2906406.html
section 1).  The scale rule is the OCP MX conversion (a reading: the pages give
none): hand-worked blocks, a lossless round trip of MXFP4 values, nearest-value
rounding with ties to even, saturation, and the clamped indexer range."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_quantize.json")


def _bf16(values):
    return torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)


def _codes_of(packed):
    """[rows, n/2] bytes -> [rows, n] codes (element 2i = low nibble of byte i)."""
    p = np.asarray(packed)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def _dequant(codes, scales):
    mag = np.array([oracle.e2m1_value(c) for c in range(16)])
    c = _codes_of(codes)
    s = np.array([oracle.e8m0_value(b) for b in range(256)])[np.asarray(scales)]
    return mag[c] * np.repeat(s, 32, axis=-1)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_blocks(case):
    vals = case["values"] + [0.0] * (case["pad_zeros_to"] - len(case["values"]))
    x = _bf16(vals)
    assert np.array_equal(x.float().numpy()[: len(case["values"])].astype(np.float64),
                          np.array(case["values"], np.float64))  # the values are exact in bf16
    codes, scales = oracle.mxfp4_quantize(x.reshape(1, -1), mode=case["mode"])
    assert int(scales[0, 0]) == case["scale_byte"]
    got = _codes_of(codes)[0]
    n = len(case["codes"])
    assert got[:n].tolist() == case["codes"]
    assert all(int(c) in (0, 8) for c in got[len(case["values"]):])  # zero padding


def test_golden_magnitudes_are_the_e2m1_table():
    mags = json.load(open(GOLDEN))["e2m1_magnitudes"]
    for c, v in mags.items():
        assert oracle.e2m1_value(int(c)) == v


def test_round_trip_of_mxfp4_values_is_lossless():
    """Dequantised MXFP4 blocks whose largest magnitude code is 4 or 6 (the
    normalised blocks the rule produces) quantise back to the same codes and
    scale: a wrong exponent, rounding or nibble order breaks this."""
    rng = np.random.default_rng(7)
    rows = 256
    codes = rng.integers(0, 256, size=(rows, 64), dtype=np.uint8)
    c = _codes_of(codes)
    for r in range(rows):  # force the block maximum to code 6 (4.0) or 7 (6.0) in one element
        for b in range(4):
            blk = c[r, 32 * b:32 * b + 32]
            if (blk & 7).max() < 6:
                blk[rng.integers(32)] = rng.choice([6, 7, 14, 15])
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.integers(110, 140, size=(rows, 4), dtype=np.uint8)
    x = _dequant(codes, scales)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(xb.double().numpy(), x)  # exact in bf16
    c2, s2 = oracle.mxfp4_quantize(xb, mode=0)
    assert np.array_equal(s2, scales)
    # -0 and +0 both decode to 0: compare the decoded values
    assert np.array_equal(_dequant(c2, s2), x)


def test_nearest_value_with_ties_to_even():
    """Every element goes to an E2M1 value nearest to x / 2^X; on a tie the even
    code wins; beyond 6 it saturates."""
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.uniform(0, 6, 4000), np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])])
    y = torch.from_numpy(y).to(torch.bfloat16).double().numpy()  # exact bf16 inputs
    n = (len(y) // 31) * 31
    blocks = y[:n].reshape(-1, 31)
    x = np.concatenate([np.full((blocks.shape[0], 1), 6.0), blocks], axis=1)  # max 6: X = 0
    codes, scales = oracle.mxfp4_quantize(torch.from_numpy(x).to(torch.bfloat16), mode=0)
    assert np.all(scales == 127)
    got = _codes_of(codes)[:, 1:].reshape(-1)
    mags = np.array([oracle.e2m1_value(c) for c in range(8)])
    yy = blocks.reshape(-1)
    dist = np.abs(yy[:, None] - mags[None, :])
    best = dist.min(axis=1)
    assert np.allclose(dist[np.arange(len(yy)), got & 7], best, rtol=0, atol=0)
    tie = (dist == best[:, None]).sum(axis=1) > 1
    assert tie.sum() >= 7
    assert np.all((got[tie] & 1) == 0)


def test_saturation_sign_and_indexer_range():
    x = _bf16([100.0, -100.0, 13.0, -0.0001] + [0.0] * 28).reshape(1, -1)
    c, s = oracle.mxfp4_quantize(x, mode=1)
    assert int(s[0, 0]) == 128
    got = _codes_of(c)[0]
    assert got[:4].tolist() == [7, 15, 7, 8]  # +-6 saturated, 13/2 -> 6, tiny negative -> -0
    rng = np.random.default_rng(11)
    y = torch.from_numpy(rng.normal(0, 30, size=(64, 128))).to(torch.bfloat16)
    _, s1 = oracle.mxfp4_quantize(y, mode=1)
    assert s1.min() >= 125 and s1.max() <= 128


def test_non_finite_block_gets_a_nan_scale():
    x = _bf16([1.0, float("inf")] + [0.0] * 30 + [2.0] * 32).reshape(1, -1)
    c, s = oracle.mxfp4_quantize(x, mode=0)
    assert int(s[0, 0]) == 255 and int(s[0, 1]) == 126  # 2.0: floor(log2 2) - 2 = -1
    assert np.all(c[0, :16] == 0)


# ------------------------------------------------------------------ MXFP8 (E4M3) for the compressed cache

def test_e4m3_table_matches_torch_float8():
    """The oracle's E4M3 decoding (from the bit fields) equals torch's
    float8_e4m3fn for every finite code."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v)
        else:
            assert v == ref[c], c


def test_mxfp8_rounding_matches_torch_in_range():
    """Blocks whose maximum lies in [256, 448] have X = 0, so every code is the
    E4M3 rounding of the element itself; torch's float8_e4m3fn cast rounds to
    nearest even and must agree (no saturation in this range)."""
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.uniform(-448, 448, 31 * 300), rng.uniform(-2, 2, 31 * 300),
                           rng.uniform(-1e-2, 1e-2, 31 * 300)])
    x = torch.from_numpy(vals).to(torch.bfloat16).reshape(-1, 31)
    x = torch.cat([torch.full((x.shape[0], 1), 300.0, dtype=torch.bfloat16), x], dim=1)
    codes, scales = oracle.mxfp8_quantize(x)
    assert np.all(scales == 127)
    ref = x.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)


def test_mxfp8_hand_worked_block():
    """max |x| = 20 = 1.25 * 2^4: X = 4 - 8 = -4, byte 123; x * 16 = 320 = 1.25 * 2^8
    (exponent field 8+7 = 15, mantissa 010: 0x7A), 1 * 16 = 16 = 2^4 (field 11: 0x58),
    -0.1015625 * 16 = -1.625 (sign, field 7, mantissa 101: 0xBD), 0.0029296875 * 16 =
    0.046875 = 1.5 * 2^-5 (field 2, mantissa 100: 0x14); 2^-10 * 16 = 2^-6 is the
    smallest normal (0x08) and 2^-12 * 16 = 2^-8 the subnormal 2/8 * 2^-6 (0x02)."""
    x = torch.tensor([[20.0, 1.0, -0.1015625, 0.0029296875, 2.0 ** -10, 2.0 ** -12] + [0.0] * 26],
                     dtype=torch.bfloat16)
    codes, scales = oracle.mxfp8_quantize(x)
    assert int(scales[0, 0]) == 123
    assert codes[0, :6].tolist() == [0x7A, 0x58, 0xBD, 0x14, 0x08, 0x02]


def test_mxfp8_round_trip_is_lossless():
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 256, size=(200, 64), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10  # no NaN codes
    for r in range(200):
        for b in range(2):
            blk = codes[r, 32 * b:32 * b + 32]
            if ((blk & 0x7F) >> 3).max() < 15:  # the block maximum must reach the top binade (2^8)
                blk[rng.integers(32)] = rng.choice([0x78, 0x7E, 0xF9])
    scales = rng.integers(100, 140, size=(200, 2), dtype=np.uint8)
    x = oracle.mxfp8_dequantize(codes, scales)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(xb.double().numpy(), x)
    c2, s2 = oracle.mxfp8_quantize(xb)
    assert np.array_equal(s2, scales)
    np.testing.assert_array_equal(oracle.mxfp8_dequantize(c2, s2), x)


def test_mxfp8_saturates():
    x = torch.tensor([[1000.0, -1000.0, 480.0] + [500.0] * 29], dtype=torch.bfloat16)
    codes, scales = oracle.mxfp8_quantize(x)
    assert int(scales[0, 0]) == 127 + 1  # floor(log2 1000) = 9 -> X = 1
    # 1000 / 2 = 500 -> saturates to 448 (0x7E); 480 / 2 = 240 (0x77)
    assert codes[0, :3].tolist() == [0x7E, 0xFE, 0x77]
