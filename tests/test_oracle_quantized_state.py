"""Pins of the quantised-state baseline oracle (oracle/quantized_state.py).

* A state whose values are exactly representable in the format (FP8 rows:
  E4M3 values times a power-of-two scale with the row maximum at 448 times
  that scale; NVFP4 blocks: E2M1 values times an E4M3 scale with the block
  maximum at 6 times it) is unchanged by a token that leaves the state as it
  is (Mamba-2 dt = 0; GDN alpha = 1, beta = 0): decoding and encoding are
  inverse on it, and the update is applied once.
* The output comes from the updated state before it is rounded again: it
  equals the fp64 recurrence's output and differs from the output of the
  rounded state.
* Rounding compounds: over many tokens of a slowly decaying GDN layer the
  baseline drifts from the exact state by far more than one rounding of that
  state (what a read copy of an exact checkpoint holds).
"""
import numpy as np
import pytest

from oracle import codecs as oc
from oracle import gdn as og
from oracle import mamba2 as om
from oracle import quantized_state as qs


def _representable(shape, fmt, rng):
    """Rows of exactly representable values in `fmt` (see the module docstring)."""
    n = shape[-1]
    if fmt == "fp8_e4m3_row":
        codes = rng.integers(0, 0x7F, size=shape).astype(np.uint8) | (rng.integers(0, 2, size=shape) << 7).astype(np.uint8)
        vals = oc.e4m3_decode(codes)
        vals[..., 0] = 448.0                                   # the row maximum
        scale = 2.0 ** rng.integers(-12, -4, size=shape[:-1])
        return vals * scale[..., None]
    codes = rng.integers(0, 16, size=shape).astype(np.uint8)
    vals = oc.e2m1_decode(codes).reshape(shape[:-1] + (n // 16, 16))
    vals[..., 0] = 6.0                                         # each block's maximum
    s_codes = rng.integers(8, 100, size=shape[:-1] + (n // 16,)).astype(np.uint8)
    return (vals * oc.e4m3_decode(s_codes)[..., None]).reshape(shape)


@pytest.mark.parametrize("fmt", qs.FMTS)
def test_representable_state_is_a_fixed_point(fmt):
    rng = np.random.default_rng(1)
    # Mamba-2: dt = 0 leaves h unchanged
    h = _representable((2, 4, 8, 32), fmt, rng)
    tok = {"x": rng.standard_normal((2, 4, 8)), "B": rng.standard_normal((2, 1, 32)),
           "C": rng.standard_normal((2, 1, 32)), "dt": np.zeros((2, 4))}
    A, D = -np.ones(4), rng.standard_normal(4)
    h2, y = qs.mamba2_step(h, tok, A, D, fmt)
    np.testing.assert_array_equal(h2, h)
    np.testing.assert_array_equal(y, om.step(h, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)[1])
    # GDN: alpha = 1, beta = 0 leaves S unchanged
    S = _representable((2, 3, 16, 32), fmt, rng)
    gt = {"q": rng.standard_normal((2, 3, 32)), "k": rng.standard_normal((2, 3, 32)),
          "v": rng.standard_normal((2, 3, 16)), "alpha": np.ones((2, 3)), "beta": np.zeros((2, 3))}
    S2, o = qs.gdn_step(S, gt, fmt)
    np.testing.assert_array_equal(S2, S)
    np.testing.assert_allclose(o, np.einsum("bhij,bhj->bhi", S, gt["q"]), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("fmt", qs.FMTS)
def test_output_comes_from_the_state_before_rounding(fmt):
    rng = np.random.default_rng(2)
    S = rng.standard_normal((2, 2, 16, 32)) * 0.1
    gt = {"q": rng.standard_normal((2, 2, 32)), "k": rng.standard_normal((2, 2, 32)),
          "v": rng.standard_normal((2, 2, 16)), "alpha": np.full((2, 2), 0.9), "beta": np.full((2, 2), 0.5)}
    S2, o = qs.gdn_step(S, gt, fmt)
    S_exact, o_exact = og.step(S, gt["q"], gt["k"], gt["v"], gt["alpha"], gt["beta"])
    np.testing.assert_array_equal(o, o_exact)
    o_rounded = np.einsum("bhij,bhj->bhi", S2, gt["q"])
    assert np.max(np.abs(o_rounded - o_exact)) > 1e-3 * np.max(np.abs(o_exact))
    np.testing.assert_array_equal(S2, qs.requantize(S_exact, fmt))


@pytest.mark.parametrize("fmt", qs.FMTS)
def test_rounding_compounds_over_tokens(fmt):
    rng = np.random.default_rng(3)
    B, H, dv, dk, T = 2, 2, 16, 32, 200
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.05
    exact, base = S0.copy(), qs.requantize(S0, fmt)
    for t in range(T):
        k = rng.standard_normal((B, H, dk))
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        tok = {"q": rng.standard_normal((B, H, dk)), "k": k, "v": rng.standard_normal((B, H, dv)),
               "alpha": np.full((B, H), 0.995), "beta": np.full((B, H), 0.3)}
        exact, _ = og.step(exact, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        base, _ = qs.gdn_step(base, tok, fmt)
    drift = np.sqrt(np.mean((base - exact) ** 2))
    one = np.sqrt(np.mean((qs.requantize(exact, fmt) - exact) ** 2))
    assert drift > 2.0 * one, f"{fmt}: drift {drift:.3e} vs one rounding {one:.3e}"
