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
The block-scaled (MXFP8) variant at the end of this file is pinned there too:
  * its exponents against a brute-force search;
  * its codes against torch's conversion of the exactly scaled values;
  * exactness on the grid, per-block power-of-two equivariance, the error
    bound, and plain loops.
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


# ---------------------------------------------------------------------------
# Block-scaled variant (MXFP8): the planned layout for activation codes written
# by the attention epilogue.  A CTA there holds one head's 128 channels of a
# row, so it can scale blocks of 32 consecutive elements along K but not a
# whole row.  Readings:
#   * one power-of-two scale 2^e per block of MX_BLOCK = 32 consecutive
#     elements along K (a row of A, a column of W);
#   * e is the smallest integer with amax * 2^-e <= 448, so no element
#     saturates.  An all-zero block gets e = 0.  e is clamped to the ue8m0
#     range [-127, 127];
#   * the code is the e4m3 value nearest to x * 2^-e, with ties to even.  The
#     scaling is exact, so there is no rounding decision before the
#     conversion;
#   * y[i, j] = sum over blocks b of 2^(ea[i, b] + ew[b, j])
#     * sum over k in b of dec(qa[i, k]) * dec(qw[k, j]).
MX_BLOCK = 32


def mx_block_exponents(amax) -> np.ndarray:
    """Smallest e with amax * 2^-e <= 448 (0 for amax == 0), clamped to ue8m0."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    e0 = ex.astype(np.int64) - 1 - 8          # amax * 2^-e0 lies in [256, 512)
    e = np.where(np.ldexp(amax, -e0) <= E4M3_MAX, e0, e0 + 1)
    e = np.where(amax > 0, e, 0)
    return np.clip(e, -127, 127).astype(np.int64)


def _mx_blocks(x, axis):
    """View x with the K axis split into (blocks, MX_BLOCK); K % 32 == 0."""
    x = np.asarray(x, dtype=np.float32)
    if axis == 1:
        n, K = x.shape
        return x.reshape(n, K // MX_BLOCK, MX_BLOCK)
    K, N = x.shape
    return x.reshape(K // MX_BLOCK, MX_BLOCK, N)


def mx_quantize_rows(x) -> Tuple[np.ndarray, np.ndarray]:
    """Codes [n, K] and block exponents [n, K/32] of x [n, K] (blocks along rows)."""
    xb = _mx_blocks(x, 1).astype(np.float64)
    e = mx_block_exponents(np.max(np.abs(xb), axis=2))
    q = e4m3_encode(np.ldexp(xb, -e[:, :, None]).astype(np.float32))
    return q.reshape(np.shape(x)), e


def mx_quantize_cols(w) -> Tuple[np.ndarray, np.ndarray]:
    """Codes [K, N] and block exponents [K/32, N] of w [K, N] (blocks along columns)."""
    wb = _mx_blocks(w, 0).astype(np.float64)
    e = mx_block_exponents(np.max(np.abs(wb), axis=1))
    q = e4m3_encode(np.ldexp(wb, -e[:, None, :]).astype(np.float32))
    return q.reshape(np.shape(w)), e


def mx_project_codes(qa, ea, qw, ew) -> np.ndarray:
    """y from MX codes: one exactly scaled partial product per K block (fp64)."""
    n, K = qa.shape
    N = qw.shape[1]
    y = np.zeros((n, N))
    da, dw = e4m3_decode(qa), e4m3_decode(qw)
    for b in range(K // MX_BLOCK):
        ks = slice(b * MX_BLOCK, (b + 1) * MX_BLOCK)
        part = da[:, ks] @ dw[ks, :]
        y += np.ldexp(part, ea[:, b][:, None] + ew[b, :][None, :])
    return y


def project_mxfp8(a, w) -> np.ndarray:
    """The block-scaled W8A8 projection of a [n, K] by w [K, N]."""
    qa, ea = mx_quantize_rows(a)
    qw, ew = mx_quantize_cols(w)
    return mx_project_codes(qa, ea, qw, ew)


# ---------------------------------------------------------------------------
# MX activations against per-channel weights: the form the tensor-core
# product takes when the attention epilogue writes the codes.  Activation
# rows carry one power-of-two scale per 32-element block (mx_quantize_rows),
# the weights the per-output-channel fp32 scale of quantize_cols (one scale
# per column of a K-major weight code matrix, applied after the sum):
#   y[i, j] = s_w[j] * sum over blocks b of 2^ea[i, b]
#             * sum over k in b of dec(qa[i, k]) * dec(qw[k, j]).
# The block exponents are stored biased by 127 (the ue8m0 byte) by the GPU
# path; here they are plain integers.
def mx_rows_project_codes(qa, ea, qw, sw) -> np.ndarray:
    """y from MX activation codes and per-channel weight codes (fp64)."""
    n, K = qa.shape
    y = np.zeros((n, qw.shape[1]))
    da, dw = e4m3_decode(qa), e4m3_decode(qw)
    for b in range(K // MX_BLOCK):
        ks = slice(b * MX_BLOCK, (b + 1) * MX_BLOCK)
        y += np.ldexp(da[:, ks] @ dw[ks, :], np.asarray(ea)[:, b][:, None])
    return y * np.asarray(sw, dtype=np.float64)[None, :]


def project_mx_rows(a, w) -> np.ndarray:
    """The projection of a [n, K] by w [K, N] with MX activation rows and
    per-channel weight scales."""
    qa, ea = mx_quantize_rows(a)
    qw, sw = quantize_cols(w)
    return mx_rows_project_codes(qa, ea, qw, sw)
