"""Conventional decode with the state itself kept in low precision (oracle;
test infrastructure).

"ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding"
([summary ¶4]) contrasts a low-precision copy that serves only the reads --
the recurrence staying in high precision -- with a state that is stored in low
precision, whose rounding then compounds from token to token.  This module is
the latter design, the baseline of that comparison.  Per token and (batch,
head):

    S       = dequantise(codes)                    (exact)
    S', out = the conventional update of S in fp64 (``mamba2.step`` /
              ``gdn.step``); the output comes from the updated state before it
              is rounded again
    codes'  = quantise(S' rounded to fp32)         (``codecs``; every decision
              taken in fp32, the precision the kernel takes it in)

The carried state is the dequantised value of the codes (fp64), which is the
same information as the codes themselves.
"""
from __future__ import annotations

import numpy as np

from . import codecs, gdn, mamba2

FMTS = ("fp8_e4m3_row", "nvfp4")


def requantize(state, fmt):
    """fp64 state [..., n] -> the fp64 value of its quantised copy."""
    rows = np.asarray(state, dtype=np.float32)
    if fmt == "fp8_e4m3_row":
        codes, scales = codecs.fp8_row_quantize(rows)
        return codecs.fp8_row_dequantize(codes, scales)
    if fmt == "nvfp4":
        codes, scales = codecs.nvfp4_quantize(rows)
        return codecs.nvfp4_dequantize(codes, scales)
    raise ValueError(f"unknown format {fmt}")


def mamba2_step(state, tok, A, D, fmt):
    """One token on a quantised Mamba-2 state (the dequantised value, fp64);
    returns (new dequantised state, y)."""
    h, y = mamba2.step(state, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)
    return requantize(h, fmt), y


def gdn_step(state, tok, fmt, out_scale=1.0):
    """One token on a quantised GDN state (the dequantised value, fp64);
    returns (new dequantised state, o)."""
    S, o = gdn.step(state, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
    return requantize(S, fmt), o
