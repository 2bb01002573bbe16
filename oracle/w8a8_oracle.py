"""CPU oracle of the W8A8 output projection -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path never imports, calls or
links anything here, and this module imports nothing from the product package.

Method: "Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", gist.science technical summary,
section 4 "Experimental Results", item "Speedup": ISPA is run together with
post-training W8A8 quantisation (8-bit weights and 8-bit activations).  The
page names no number format, granularity or rounding.  Readings taken here:

  * the 8-bit format is e4m3: a sign bit, 4 exponent bits with bias 7 and 3
    mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; there is
    no infinity; S.1111.111 is NaN, so the largest finite value is 448;
  * activations A [n, D_in] carry one scale per token row and weights
    W [D_in, D_out] one scale per output channel (column):
    s = amax / 448, or 1 when the row / column is all zero;
  * a code is the e4m3 value nearest to x / s, with ties going to the even
    mantissa, and saturation at +-448;
  * amax / 448 and x / s are evaluated in fp32, correctly rounded.  This is the
    precision in which the GPU makes the same rounding decisions, so the codes
    and scales are compared bit for bit;
  * y[i, j] = s_a[i] * s_w[j] * sum_k dec(qa[i, k]) * dec(qw[k, j]).  The
    oracle evaluates this in fp64;
  * W is quantised after the absorb, that is, W_new = W + dW as the bf16
    projection uses it.

Pinned by tests/test_oracle_w8a8.py:
  * the decode table against torch's float8_e4m3fn;
  * the encoder against torch's float32 -> float8_e4m3fn conversion on every
    finite bf16 value in range, and against a brute-force nearest-code search;
  * saturation;
  * exactness when every scale is 1 and every value lies on the grid;
  * power-of-two equivariance of the row and column scales;
  * the error bound of a 3-bit mantissa.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of e4m3 codes, from the format's definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """Round-to-nearest-even e4m3 codes of fp32 values, saturating at +-448
    (NaN -> the NaN code with the input's sign)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)  # exact
    sign = np.signbit(x)
    nan = np.isnan(x)
    a = np.where(nan, 0.0, np.abs(x))
    a = np.minimum(a, E4M3_MAX)
    # binade of a (a = f * 2^ex with f in [0.5, 1)), floored at the smallest
    # normal binade 2^-6, below which the grid step stays 2^-9 (subnormals)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex.astype(np.int64) - 1, -6)
    step = np.exp2((e - 3).astype(np.float64))  # 3 mantissa bits
    q = np.rint(a / step).astype(np.int64)      # a / step is exact; rint ties to even
    carry = q >= 16                              # rounded up into the next binade
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 8, q)
    sub = q < 8                                  # only below 2^-6
    code = np.where(sub, q, ((e + 7) << 3) | (q - 8))
    code = np.where(nan, 0x7F, code)
    code = code | np.where(sign, 0x80, 0)
    return code.astype(np.uint8)


def _scales(amax: np.ndarray) -> np.ndarray:
    amax = amax.astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)  # fp32 division, correctly rounded
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows(x) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 codes [n, K] and fp32 scales [n] of x [n, K]."""
    x32 = np.asarray(x, dtype=np.float32)
    s = _scales(np.max(np.abs(x32), axis=1))
    return e4m3_encode((x32 / s[:, None]).astype(np.float32)), s


def quantize_cols(w) -> Tuple[np.ndarray, np.ndarray]:
    """Per-column e4m3 codes [K, N] and fp32 scales [N] of w [K, N]."""
    w32 = np.asarray(w, dtype=np.float32)
    s = _scales(np.max(np.abs(w32), axis=0))
    return e4m3_encode((w32 / s[None, :]).astype(np.float32)), s


def project_codes(qa, sa, qw, sw) -> np.ndarray:
    """y = diag(s_a) dec(qa) dec(qw) diag(s_w) in fp64 (qw is [K, N])."""
    acc = e4m3_decode(qa) @ e4m3_decode(qw)
    return np.asarray(sa, np.float64)[:, None] * acc * np.asarray(sw, np.float64)[None, :]


def project_w8a8(a, w) -> np.ndarray:
    """The W8A8 projection of activations a [n, K] by weights w [K, N]."""
    qa, sa = quantize_rows(a)
    qw, sw = quantize_cols(w)
    return project_codes(qa, sa, qw, sw)
