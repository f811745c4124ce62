"""Pins of the oracle's number formats against library codecs and exhaustive checks."""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import ckv_oracle as O


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_matches_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = O.e4m3_decode(codes)
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_e2m1_decode_matches_ml_dtypes_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = O.e2m1_decode(codes)
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert O.E2M1_MAX == 6.0 and O.E4M3_MAX == 448.0


def _e4m3_midpoints():
    v = O.E4M3_TABLE[:0x7F]
    return ((v[1:] + v[:-1]) / 2).astype(np.float32)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.normal(size=20000).astype(np.float32) * 50,
        rng.uniform(-448, 448, 20000).astype(np.float32),
        rng.normal(size=5000).astype(np.float32) * 1e-2,     # subnormal range
        _e4m3_midpoints(), -_e4m3_midpoints(),               # exact ties
        O.E4M3_TABLE[:0x7F].astype(np.float32),              # exact grid values
        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, -(2.0 ** -10)], dtype=np.float32),
    ])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode_satfinite(x)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    x = np.array([449.0, 464.0, 480.0, 1e6, -500.0, -1e30], dtype=np.float32)
    got = O.e4m3_encode_satfinite(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_e4m3_encode_decode_identity_on_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(O.e4m3_encode_satfinite(vals), codes)


def test_e2m1_encode_matches_ml_dtypes():
    rng = np.random.default_rng(1)
    v = O.E2M1_TABLE[:8]
    mids = ((v[1:] + v[:-1]) / 2).astype(np.float32)
    x = np.concatenate([rng.normal(size=20000).astype(np.float32) * 3,
                        mids, -mids, v.astype(np.float32), -v.astype(np.float32),
                        np.array([7.0, 100.0, -9.0, 1e-30, -1e-30], dtype=np.float32)])
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = O.e2m1_encode_satfinite(x)
    assert np.array_equal(got, ref)


def test_e2m1_ties_go_to_even_code():
    # 0.25 -> 0 (code 0), 0.75 -> 1 (code 2), 1.25 -> 1 (code 2), 2.5 -> 2 (code 4), 5 -> 4 (code 6)
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    assert list(O.e2m1_encode_satfinite(x)) == [0, 2, 2, 4, 4, 6, 6]


def test_bf16_round_trip_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.normal(size=50000).astype(np.float32),
                        rng.normal(size=1000).astype(np.float32) * 1e-39,   # subnormals
                        rng.normal(size=1000).astype(np.float32) * 1e30,
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f32_to_bf16_bits(x)
    assert np.array_equal(got, ref)
    dec_ref = torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_bits_to_f64(got), dec_ref)


def _nearest_brute(xs, grid):
    """Brute force: the grid value of least distance, ties to the even index."""
    out = []
    for x in xs:
        a = abs(float(x))
        best = None
        for i, g in enumerate(grid):
            d = abs(a - g)
            if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
                best = (d, i)
        out.append(best[1])
    return np.array(out)


def test_round_to_grid_brute_force():
    rng = np.random.default_rng(3)
    grid = O.E2M1_TABLE[:8]
    x = rng.uniform(-7, 7, 3000).astype(np.float32)
    assert np.array_equal(O.e2m1_encode_satfinite(x) & 7, _nearest_brute(x, grid))


def test_fp8_token_quantizer_error_bound():
    rng = np.random.default_rng(4)
    for scale in [1e-3, 1.0, 300.0]:
        x = (rng.normal(size=512) * scale).astype(np.float32)
        codes, s = O.quantize_fp8_token(x)
        assert s == np.float32(np.max(np.abs(x)) / np.float32(448.0))
        y = O.dequant_fp8_token(codes, s)
        q = (x / s).astype(np.float64)
        # the stored code is the nearest e4m3 value to x/s: half of its local step at most
        grid = O.E4M3_TABLE[:0x7F]
        idx = np.clip(np.searchsorted(grid, np.abs(q)), 1, len(grid) - 1)
        step = grid[idx] - grid[idx - 1]
        assert np.all(np.abs(np.abs(q) - np.abs(y / s)) <= step / 2 + 1e-12)
        assert np.max(np.abs(y)) == pytest.approx(np.max(np.abs(x)), rel=1e-6)
    codes, s = O.quantize_fp8_token(np.zeros(16, dtype=np.float32))
    assert s == 1.0 and not np.any(codes & 0x7F)


def test_nvfp4_quantizer_error_bound_and_layout():
    rng = np.random.default_rng(5)
    x = rng.normal(size=512).astype(np.float32)
    packed, sc = O.quantize_nvfp4(x)
    assert packed.shape == (256,) and sc.shape == (32,)
    y = O.dequant_nvfp4(packed, sc)
    s = O.e4m3_decode(sc)
    # every element within half of the largest e2m1 step (2 -> 1.0) of its block scale
    assert np.all(np.abs(y - x).reshape(32, 16) <= s[:, None] * 1.0 + 1e-12)
    # element 2i is in the low nibble of byte i
    assert O.e2m1_decode(packed[0] & 0xF) * s[0] == y[0]
    assert O.e2m1_decode(packed[0] >> 4) * s[0] == y[1]
    # an all-zero block stores zero scale and zero codes
    packed, sc = O.quantize_nvfp4(np.zeros(32, dtype=np.float32))
    assert not np.any(packed) and not np.any(sc)


def test_nvfp4_entry_is_45_percent_smaller_than_fp8():
    # aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM…", § "Výkon nepřinesl jeden kernel": the NVFP4
    # compressed KV is about 45 % smaller than the FP8 one. At D=512: codes D/2 + one scale byte
    # per 16 elements, against D e4m3 bytes + one fp32 scale.
    d = 512
    nvfp4 = d // 2 + d // 16
    fp8 = d + 4
    assert abs((1 - nvfp4 / fp8) - 0.45) < 0.01


def _e4m3_code_of_power_of_two(k: int) -> int:
    """e4m3 code of 2^k from the format's fields (bias 7): normal for k >= -6 (exponent field
    k + 7, mantissa 0), subnormal below (mantissa 2^(k+9), exponent field 0)."""
    return (k + 7) << 3 if k >= -6 else 1 << (k + 9)


@pytest.mark.parametrize("k", [-9, -7, -6, -3, 0, 1, 5, 8])
def test_nvfp4_scale_is_the_block_max_over_six(k):
    """A block whose largest magnitude is 6 * 2^k has the exact scale 2^k: its scale code is the
    e4m3 code of 2^k and every element is an e2m1 value times 2^k, so each code is that value's
    own code (6 -> 7, the top finite magnitude). A divisor other than 6 (amax/4 gives the scale
    1.5 * 2^k and maps 6 * 2^k to the code of 4; amax/5 rounds the scale to 1.25 * 2^k and maps it
    to 4.8 -> the code of 4) fails both checks."""
    mags = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0, 6, 4, 3, 2, 1.5, 1, 0.5, 0], dtype=np.float64)
    signs = np.array([1, -1] * 8, dtype=np.float64)
    x = (mags * signs * 2.0 ** k).astype(np.float32)
    packed, sc = O.quantize_nvfp4(x)
    assert int(sc[0]) == _e4m3_code_of_power_of_two(k)
    mag_code = {6: 7, 4: 6, 3: 5, 2: 4, 1.5: 3, 1: 2, 0.5: 1, 0: 0}
    want = [mag_code[m] | (8 if s < 0 else 0) for m, s in zip(mags, signs)]
    got = []
    for byte in packed:
        got += [int(byte) & 0xF, int(byte) >> 4]
    # -0 keeps its sign bit (code 8); compare magnitudes there
    assert [g & 7 for g in got] == [w & 7 for w in want]
    assert all(g == w for g, w, m in zip(got, want, mags) if m != 0)


@pytest.mark.parametrize("k", [-20, -8, 0, 3, 11])
def test_fp8_token_scale_is_the_token_max_over_448(k):
    """A token whose largest magnitude is 448 * 2^k has the exact scale 2^k and its largest
    element the top finite e4m3 code 0x7E (0xFE negative); elements that are e4m3 values times
    2^k keep their own codes. A divisor of 240 or 256 maps the largest element to 240 or 256
    (codes 0x77, 0x78) and changes the scale, so both checks fail for it."""
    vals = np.array([448, -448, 1.0, 0.5, 3.0, -2.0, 0.0, 0.015625], dtype=np.float64)
    codes_want = [0x7E, 0xFE, 0x38, 0x30, 0x44, 0xC0, 0x00, 0x08]   # 0.015625 = 2^-6: exponent field 1
    x = (vals * 2.0 ** k).astype(np.float32)
    codes, s = O.quantize_fp8_token(x)
    assert s == np.float32(2.0 ** k)
    assert [int(c) for c in codes] == codes_want
