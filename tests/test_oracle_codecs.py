"""Pins for the E4M3 / E2M1 codecs and the read-copy quantisers."""
import os

import numpy as np
import pytest
import torch

from oracle import codecs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    return rows


def _same(a, b):
    return (np.isnan(a) and np.isnan(b)) or (a == b and np.signbit(a) == np.signbit(b))


def test_e4m3_spec_table():
    for code, value in _table("e4m3_codes.txt"):
        assert _same(float(codecs.e4m3_decode(code)), value), hex(code)
        if not np.isnan(value):
            assert int(codecs.e4m3_encode(value)) == code, hex(code)


def test_e2m1_spec_table():
    for code, value in _table("e2m1_codes.txt"):
        assert _same(float(codecs.e2m1_decode(code)), value), hex(code)
        assert int(codecs.e2m1_encode(value)) == code, hex(code)


def test_e4m3_matches_torch_cast():
    """Within the finite range the encoder agrees with torch's float8_e4m3fn cast (RNE)."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 150)])
    mids = (codecs.E4M3_VALUES[:-1] + codecs.E4M3_VALUES[1:]) / 2      # exact ties
    x = np.concatenate([x, mids, -mids, codecs.E4M3_VALUES]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ours = codecs.e4m3_decode(codecs.e4m3_encode(x))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_saturates_and_keeps_sign():
    assert int(codecs.e4m3_encode(1e6)) == 0x7E
    assert int(codecs.e4m3_encode(-500.0)) == 0xFE
    assert int(codecs.e4m3_encode(460.0)) == 0x7E
    assert int(codecs.e4m3_encode(-1e-30)) == 0x80
    assert int(codecs.e4m3_encode(2.0 ** -10)) == 0x00        # tie between 0 and 2^-9 -> even
    assert int(codecs.e4m3_encode(3 * 2.0 ** -10)) == 0x02    # tie between 1 and 2 (x 2^-9) -> even


def test_e2m1_ties_to_even_and_saturation():
    cases = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6,
             7.0: 0x7, 100.0: 0x7, 0.26: 0x1, 5.01: 0x7, -0.25: 0x8, -5.0: 0xE}
    for x, code in cases.items():
        assert int(codecs.e2m1_encode(x)) == code, x


def test_round_trip_every_finite_code():
    c8 = np.array([c for c in range(256) if c & 0x7F != 0x7F])
    np.testing.assert_array_equal(codecs.e4m3_encode(codecs.e4m3_decode(c8)), c8)
    c4 = np.arange(16)
    np.testing.assert_array_equal(codecs.e2m1_encode(codecs.e2m1_decode(c4)), c4)


def test_fp8_row_quantiser_error_bound():
    rng = np.random.default_rng(1)
    rows = (rng.standard_normal((64, 128)) * 0.1).astype(np.float32)
    rows[3] = 0.0
    codes, s = codecs.fp8_row_quantize(rows)
    assert s[3] == 0 and not codes[3].any()
    deq = codecs.fp8_row_dequantize(codes, s)
    q = rows.astype(np.float64) / np.where(s == 0, 1, s)[:, None]
    # half an E4M3 step at |q|: 2^-4 relative for normals, 2^-10 absolute below 2^-6
    step = np.where(np.abs(q) >= 2.0 ** -6, np.abs(q) * 2.0 ** -4, 2.0 ** -10)
    assert np.all(np.abs(deq - rows) <= (step * 1.0001 + 1e-7) * np.where(s == 0, 1, s)[:, None])
    amax_pos = np.argmax(np.abs(rows), axis=1)
    top = np.abs(codecs.e4m3_decode(codes[np.arange(64), amax_pos]))
    assert np.all(top[s > 0] >= 416)                       # the largest element uses the top of the range


def test_nvfp4_quantiser_error_bound():
    rng = np.random.default_rng(2)
    rows = (rng.standard_normal((32, 128)) * 0.1).astype(np.float32)
    rows[5, :16] = 1e-6                                     # scale underflows to 0 -> zero block
    codes, sc = codecs.nvfp4_quantize(rows)
    assert codes.shape == rows.shape and sc.shape == (32, 8)
    assert int(sc[5, 0]) == 0 and not codes[5, :16].any()
    deq = codecs.nvfp4_dequantize(codes, sc)
    sval = codecs.e4m3_decode(sc)
    q = rows.reshape(32, 8, 16) / np.where(sval == 0, 1, sval)[..., None]
    # E2M1 grid spacing: 0.5 below 2, 1 in [2, 4), 2 in [4, 6]; plus saturation above 6
    half = np.where(np.abs(q) < 2, 0.25, np.where(np.abs(q) < 4, 0.5, 1.0))
    over = np.maximum(np.abs(q) - 6, 0)
    bound = (half + over) * np.where(sval == 0, 0, sval)[..., None]
    err = np.abs(deq - rows).reshape(32, 8, 16)
    ok = np.where(sval[..., None] == 0, np.abs(rows.reshape(32, 8, 16)) < 1e-5, err <= bound * 1.0001)
    assert ok.all()



# ---- the scale rules themselves.  The bounds above hold for a range of
#      divisors; these pin the divisor: the block / row maximum must land on the
#      top code of the element format, within one rounding of the scale and
#      never saturating beyond it, and data that already sits on a scaled code
#      grid must come back exactly.

def _blocks_with_spread(rng, nrows, ncols):
    """Rows whose 16-element blocks have maxima spread over [0.1, 2000] (E4M3
    block scales amax/6 stay normal: >= 2^-6 and <= 448)."""
    rows = rng.standard_normal((nrows, ncols))
    blocks = rows.reshape(nrows, ncols // 16, 16)
    target = np.exp(rng.uniform(np.log(0.1), np.log(2000.0), size=blocks.shape[:2]))
    blocks *= (target / np.max(np.abs(blocks), axis=-1))[..., None]
    return blocks.reshape(nrows, ncols).astype(np.float32)


def test_nvfp4_block_max_takes_top_code_without_saturating():
    """s = E4M3(amax / 6): the block max divided by the decoded scale lies within
    one E4M3 rounding (2^-4 relative) of 6, i.e. in [6 / (1 + 2^-4), 6 / (1 - 2^-4)],
    so it encodes to magnitude code 7 (6.0) and nothing saturates by more than
    that rounding.  A divisor of 4 or 8 (or 5.5, 6.5) fails one of the bounds."""
    rng = np.random.default_rng(11)
    rows = _blocks_with_spread(rng, 256, 128)
    codes, sc = codecs.nvfp4_quantize(rows)
    sval = codecs.e4m3_decode(sc).astype(np.float32)
    blk = rows.reshape(256, 8, 16)
    q = (blk / sval[..., None]).astype(np.float32)                  # the quantiser's own fp32 division
    qmax = np.max(np.abs(q), axis=-1)
    assert np.all(qmax <= np.float32(6.0 / (1 - 2.0 ** -4)) * (1 + 2.0 ** -22))
    assert np.all(qmax >= np.float32(6.0 / (1 + 2.0 ** -4)) * (1 - 2.0 ** -22))
    arg = np.argmax(np.abs(blk), axis=-1)
    top = np.take_along_axis(codes.reshape(256, 8, 16), arg[..., None], axis=-1)[..., 0]
    assert np.all((top & 0x7) == 0x7)
    assert np.all(((top >> 3) & 1) == np.signbit(np.take_along_axis(blk, arg[..., None], -1)[..., 0]))


def test_nvfp4_exact_on_scaled_e2m1_grid():
    """Blocks of E2M1 values times 2^e whose max is 6 * 2^e have scale exactly 2^e
    (E4M3-representable for -6 <= e <= 8), so they quantise without error."""
    rng = np.random.default_rng(12)
    grid = np.concatenate([codecs.E2M1_VALUES, -codecs.E2M1_VALUES])
    for e in range(-6, 9):
        blocks = rng.choice(grid, size=(64, 16))
        blocks[np.arange(64), rng.integers(0, 16, 64)] = rng.choice([6.0, -6.0], 64)
        rows = (blocks * 2.0 ** e).reshape(8, 128).astype(np.float32)
        codes, sc = codecs.nvfp4_quantize(rows)
        np.testing.assert_array_equal(codecs.e4m3_decode(sc), 2.0 ** e)
        np.testing.assert_array_equal(codecs.nvfp4_dequantize(codes, sc), rows)


def test_fp8_row_max_takes_top_code_without_saturating():
    """s = amax / 448 (fp32): the row max divided by s is 448 up to fp32 rounding,
    so it encodes to 0x7E (0xFE when negative) and no element saturates beyond
    one rounding of the scale.  Divisors such as 430 or 470 fail."""
    rng = np.random.default_rng(13)
    rows = rng.standard_normal((512, 128)) * np.exp(rng.uniform(-12, 12, size=(512, 1)))
    rows = rows.astype(np.float32)
    codes, s = codecs.fp8_row_quantize(rows)
    q = (rows / s[:, None]).astype(np.float32)
    assert np.all(np.max(np.abs(q), axis=1) <= 448.0 * (1 + 2.0 ** -22))
    arg = np.argmax(np.abs(rows), axis=1)
    top = codes[np.arange(512), arg]
    assert np.all((top & 0x7F) == 0x7E)
    assert np.all(((top >> 7) & 1) == np.signbit(rows[np.arange(512), arg]))


def test_fp8_row_exact_on_scaled_e4m3_grid():
    """Rows of E4M3 values times 2^e whose max is 448 * 2^e have scale exactly 2^e,
    so they quantise without error."""
    rng = np.random.default_rng(14)
    grid = np.concatenate([codecs.E4M3_VALUES, -codecs.E4M3_VALUES])
    for e in range(-20, 21, 4):
        rows = rng.choice(grid, size=(32, 128))
        rows[np.arange(32), rng.integers(0, 128, 32)] = rng.choice([448.0, -448.0], 32)
        rows = (rows * 2.0 ** e).astype(np.float32)
        codes, s = codecs.fp8_row_quantize(rows)
        np.testing.assert_array_equal(s, np.float32(2.0 ** e))
        np.testing.assert_array_equal(codecs.fp8_row_dequantize(codes, s), rows)
