"""Pins of the W8A8 oracle (oracle/w8a8_oracle.py) against things other than
itself: torch's float8_e4m3fn conversions (a library routine), a brute-force
nearest-code search written with plain loops, exact cases, invariances and
the error bound of a 3-bit mantissa.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import w8a8_oracle as w8


def _all_codes():
    return np.arange(256, dtype=np.uint8)


def test_decode_matches_torch_float8_e4m3fn():
    codes = _all_codes()
    ours = w8.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.isnan(ours).sum() == 2  # 0x7F and 0xFF
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_encode_matches_torch_on_every_bf16_value_in_range():
    x = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448.0)]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(w8.e4m3_encode(x), ref)


def test_encode_matches_torch_on_random_fp32():
    rng = np.random.default_rng(11)
    mag = np.exp2(rng.uniform(-14.0, np.log2(448.0), 200000)).astype(np.float32)
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(w8.e4m3_encode(x), ref)


def _brute_force_code(v: float) -> int:
    """Nearest finite e4m3 value by scanning all codes; ties go to the even
    mantissa; magnitudes beyond 448 saturate."""
    best, best_d = None, None
    for c in range(256):
        e, m = (c >> 3) & 0xF, c & 7
        if e == 15 and m == 7:
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        val = -mag if c & 0x80 else mag
        if (c & 0x80) != (0x80 if np.signbit(v) else 0):
            continue  # a zero result keeps the input's sign
        d = abs(val - v)
        if best is None or d < best_d or (d == best_d and (c & 1) == 0):
            best, best_d = c, d
    return best


def test_encode_matches_brute_force_nearest_search():
    rng = np.random.default_rng(12)
    # values around every binade, exact ties between grid points, the
    # subnormal range, zeros of both signs and saturation
    grid = w8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    ties = (grid[:-1] + grid[1:]) / 2
    vals = np.concatenate([rng.standard_normal(300) * 50, ties[::3], -ties[1::5],
                           rng.uniform(0, 2.0 ** -6, 40), [0.0, -0.0, 448.0, 449.0, 463.0, 464.0, 1e30, -1e30]])
    vals = vals.astype(np.float32)
    got = w8.e4m3_encode(vals)
    for v, g in zip(vals, got):
        assert int(g) == _brute_force_code(float(v)), (float(v), int(g))


def test_encode_saturates_and_keeps_nan():
    x = np.array([448.0, 460.0, 464.0, 1000.0, 3.4e38, -500.0, np.inf, -np.inf, np.nan], dtype=np.float32)
    c = w8.e4m3_encode(x)
    assert list(c[:5]) == [0x7E] * 5
    assert c[5] == 0xFE and c[6] == 0x7E and c[7] == 0xFE
    assert c[8] & 0x7F == 0x7F


def test_quantize_rows_scales_and_extremes():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((7, 40)) * rng.uniform(0.01, 100, (7, 1))).astype(np.float32)
    x[3] = 0.0
    q, s = w8.quantize_rows(x)
    assert s.dtype == np.float32 and s[3] == 1.0 and np.all(q[3] & 0x7F == 0)
    for i in range(7):
        if i == 3:
            continue
        assert s[i] == np.float32(np.max(np.abs(x[i])) / np.float32(448.0))
        # the element of largest magnitude lands on +-448
        j = int(np.argmax(np.abs(x[i])))
        assert q[i, j] & 0x7F == 0x7E
        assert np.all(np.abs(w8.e4m3_decode(q[i])) <= 448.0)


def test_projection_exact_on_grid_with_unit_scales():
    """Every value on the e4m3 grid and every row / column reaching 448: all
    scales are 1 and the W8A8 product is the exact product."""
    rng = np.random.default_rng(14)
    grid = w8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    a = rng.choice(grid, (9, 64)) * rng.choice([-1.0, 1.0], (9, 64))
    w = rng.choice(grid, (64, 24)) * rng.choice([-1.0, 1.0], (64, 24))
    a[:, 5] = 448.0
    w[7, :] = -448.0
    qa, sa = w8.quantize_rows(a)
    qw, sw = w8.quantize_cols(w)
    assert np.all(sa == 1.0) and np.all(sw == 1.0)
    assert np.array_equal(w8.e4m3_decode(qa), a) and np.array_equal(w8.e4m3_decode(qw), w)
    assert np.array_equal(w8.project_w8a8(a, w), a @ w)


def test_projection_power_of_two_equivariance():
    """Scaling one activation row (or one weight column) by 2^k leaves the
    codes unchanged and scales exactly that row (column) of y by 2^k; a
    transposed or misplaced scale breaks it."""
    rng = np.random.default_rng(15)
    a = rng.standard_normal((6, 48)).astype(np.float32)
    w = rng.standard_normal((48, 10)).astype(np.float32)
    y = w8.project_w8a8(a, w)
    a2 = a.copy()
    a2[2] *= 8.0
    y2 = w8.project_w8a8(a2, w)
    assert np.array_equal(y2[2], 8.0 * y[2]) and np.array_equal(np.delete(y2, 2, 0), np.delete(y, 2, 0))
    w2 = w.copy()
    w2[:, 4] *= 0.25
    y3 = w8.project_w8a8(a, w2)
    assert np.array_equal(y3[:, 4], 0.25 * y[:, 4]) and np.array_equal(np.delete(y3, 4, 1), np.delete(y, 4, 1))


def test_projection_error_bound_of_three_mantissa_bits():
    """Each code is within 2^-4 relative of its scaled input (half a unit of a
    3-bit mantissa) outside the subnormals, so the product is within a few
    percent of the exact one; it is lossy, not exact."""
    rng = np.random.default_rng(16)
    a = rng.standard_normal((64, 256)).astype(np.float32)
    w = (rng.standard_normal((256, 128)) / 16).astype(np.float32)
    qa, sa = w8.quantize_rows(a)
    rel = np.abs(w8.e4m3_decode(qa) * sa[:, None] - a) / np.abs(a)
    normal = np.abs(a) / sa[:, None] >= 2.0 ** -6
    assert rel[normal].max() <= 2.0 ** -4 * (1 + 1e-6)
    y = w8.project_w8a8(a, w)
    exact = a.astype(np.float64) @ w.astype(np.float64)
    err = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert 1e-3 < err < 0.05


def test_project_codes_brute_force_loops():
    rng = np.random.default_rng(17)
    qa = rng.integers(0, 0x7E, (3, 5)).astype(np.uint8) | rng.choice([0, 0x80], (3, 5)).astype(np.uint8)
    qw = rng.integers(0, 0x7E, (5, 4)).astype(np.uint8)
    sa = np.array([0.5, 2.0, 0.125], np.float32)
    sw = np.array([1.0, 0.25, 4.0, 3.0], np.float32)
    got = w8.project_codes(qa, sa, qw, sw)
    for i in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(5):
                acc += w8.e4m3_decode(qa[i, k]) * w8.e4m3_decode(qw[k, j])
            assert got[i, j] == pytest.approx(float(sa[i]) * float(sw[j]) * acc, rel=1e-15, abs=1e-300)


# ----------------------------------------------------------- block-scaled (MXFP8)
def _bf16_normal(rng, shape):
    """Normal draws rounded to bf16 (round to nearest even), as fp32."""
    x = rng.standard_normal(shape).astype(np.float32)
    u = x.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> 16) & 1)) & np.uint32(0xFFFF0000)).view(np.float32)


def test_mx_exponent_is_the_smallest_in_range_brute_force():
    rng = np.random.default_rng(30)
    amax = np.concatenate([np.exp2(rng.uniform(-30, 30, 500)),
                           448.0 * np.exp2(np.arange(-5, 6)),              # exactly on the boundary
                           np.nextafter(448.0 * np.exp2(np.arange(-5, 6)), np.inf)])  # just above it
    e = w8.mx_block_exponents(amax)
    for a, ei in zip(amax, e):
        ok = [k for k in range(-140, 140) if a * 2.0 ** -k <= 448.0]
        assert ei == min(ok), (a, ei)
    assert np.array_equal(w8.mx_block_exponents(448.0 * np.exp2(np.arange(-5, 6))), np.arange(-5, 6))
    assert w8.mx_block_exponents(np.array([0.0]))[0] == 0
    assert w8.mx_block_exponents(np.array([1e-45]))[0] == -127  # clamped to the ue8m0 range


def test_mx_codes_match_torch_on_exactly_scaled_blocks():
    rng = np.random.default_rng(31)
    x = _bf16_normal(rng, (37, 96)) * np.exp2(rng.integers(-12, 12, (37, 1))).astype(np.float32)
    q, e = w8.mx_quantize_rows(x)
    assert e.shape == (37, 3)
    scaled = (x.reshape(37, 3, 32) * np.exp2(-e[:, :, None])).reshape(37, 96).astype(np.float32)
    assert np.all(np.abs(scaled) <= 448.0)
    ref = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    qw, ew = w8.mx_quantize_cols(x.T.copy())
    assert np.array_equal(qw, q.T) and np.array_equal(ew, e.T)


def test_mx_projection_exact_on_grid():
    """Blocks whose values lie on the e4m3 grid and reach 448 have exponent 0
    and their codes are the values: the product is exact."""
    rng = np.random.default_rng(32)
    grid = w8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    a = rng.choice(grid, (5, 64)) * rng.choice([-1.0, 1.0], (5, 64))
    w = rng.choice(grid, (64, 7)) * rng.choice([-1.0, 1.0], (64, 7))
    a[:, [3, 40]] = 448.0
    w[[1, 33], :] = -448.0
    qa, ea = w8.mx_quantize_rows(a)
    qw, ew = w8.mx_quantize_cols(w)
    assert np.all(ea == 0) and np.all(ew == 0)
    assert np.array_equal(w8.project_mxfp8(a, w), a @ w)


def test_mx_per_block_power_of_two_equivariance():
    """Scaling one 32-element block of a row by 2^k moves only that block's
    exponent by k; the codes and every other output stay exactly the same."""
    rng = np.random.default_rng(33)
    a = rng.standard_normal((4, 96)).astype(np.float32)
    w = rng.standard_normal((96, 5)).astype(np.float32)
    qa, ea = w8.mx_quantize_rows(a)
    a2 = a.copy()
    a2[1, 32:64] *= 16.0
    qa2, ea2 = w8.mx_quantize_rows(a2)
    assert np.array_equal(qa2, qa)
    assert ea2[1, 1] == ea[1, 1] + 4 and np.array_equal(np.delete(ea2.ravel(), 4), np.delete(ea.ravel(), 4))
    y, y2 = w8.project_mxfp8(a, w), w8.project_mxfp8(a2, w)
    assert np.array_equal(np.delete(y2, 1, 0), np.delete(y, 1, 0))


def test_mx_error_bound_and_no_saturation():
    rng = np.random.default_rng(34)
    a = (rng.standard_normal((64, 256)) * np.exp2(rng.uniform(-8, 8, (64, 8))).repeat(32, 1)).astype(np.float32)
    qa, ea = w8.mx_quantize_rows(a)
    deq = (w8.e4m3_decode(qa).reshape(64, 8, 32) * np.exp2(ea[:, :, None])).reshape(64, 256)
    normal = np.abs(a) * np.exp2(-ea.repeat(32, 1)) >= 2.0 ** -6
    assert (np.abs(deq - a) / np.abs(a))[normal].max() <= 2.0 ** -4 * (1 + 1e-6)
    assert np.all(qa & 0x7F != 0x7F)  # nothing saturates into the NaN code
    w = (rng.standard_normal((256, 32)) / 16).astype(np.float32)
    exact = a.astype(np.float64) @ w.astype(np.float64)
    err = np.linalg.norm(w8.project_mxfp8(a, w) - exact) / np.linalg.norm(exact)
    assert 1e-3 < err < 0.05


def test_mx_project_codes_brute_force_loops():
    rng = np.random.default_rng(35)
    qa = rng.integers(0, 0x7E, (2, 64)).astype(np.uint8)
    qw = rng.integers(0, 0x7E, (64, 3)).astype(np.uint8) | rng.choice([0, 0x80], (64, 3)).astype(np.uint8)
    ea = rng.integers(-5, 5, (2, 2))
    ew = rng.integers(-5, 5, (2, 3))
    got = w8.mx_project_codes(qa, ea, qw, ew)
    for i in range(2):
        for j in range(3):
            acc = 0.0
            for k in range(64):
                b = k // 32
                acc += w8.e4m3_decode(qa[i, k]) * w8.e4m3_decode(qw[k, j]) * 2.0 ** (ea[i, b] + ew[b, j])
            assert got[i, j] == pytest.approx(acc, rel=1e-14, abs=1e-300)


def test_mx_rows_project_codes_brute_force_loops():
    rng = np.random.default_rng(36)
    qa = rng.integers(0, 0x7E, (3, 96)).astype(np.uint8) | rng.choice([0, 0x80], (3, 96)).astype(np.uint8)
    qw = rng.integers(0, 0x7E, (96, 4)).astype(np.uint8)
    ea = rng.integers(-9, 9, (3, 3))
    sw = rng.uniform(0.01, 2.0, 4)
    got = w8.mx_rows_project_codes(qa, ea, qw, sw)
    for i in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(96):
                acc += w8.e4m3_decode(qa[i, k]) * w8.e4m3_decode(qw[k, j]) * 2.0 ** ea[i, k // 32]
            assert got[i, j] == pytest.approx(acc * sw[j], rel=1e-14, abs=1e-300)


def test_mx_rows_with_zero_exponents_is_the_per_token_product_with_unit_scales():
    rng = np.random.default_rng(37)
    qa = rng.integers(0, 0x7E, (5, 64)).astype(np.uint8)
    qw = rng.integers(0, 0x7E, (64, 6)).astype(np.uint8) | rng.choice([0, 0x80], (64, 6)).astype(np.uint8)
    sw = rng.uniform(0.5, 1.5, 6)
    got = w8.mx_rows_project_codes(qa, np.zeros((5, 2), dtype=np.int64), qw, sw)
    assert np.array_equal(got, w8.project_codes(qa, np.ones(5), qw, sw))


def test_project_mx_rows_per_block_equivariance_and_accuracy():
    """Scaling a 32-element block of a row by 2^k changes nothing but that
    block's exponent, so the output is the same function of the unscaled
    block; and the result is as close to the exact product as 3-bit
    mantissas on both operands allow."""
    rng = np.random.default_rng(38)
    a = (rng.standard_normal((16, 128)) * np.exp2(rng.uniform(-6, 6, (16, 4))).repeat(32, 1)).astype(np.float32)
    w = (rng.standard_normal((128, 24)) / 11).astype(np.float32)
    qa, ea = w8.mx_quantize_rows(a)
    a2 = a.copy()
    a2[:, 64:96] *= 8.0
    qa2, ea2 = w8.mx_quantize_rows(a2)
    assert np.array_equal(qa2, qa) and np.array_equal(ea2[:, 2], ea[:, 2] + 3)
    y = w8.project_mx_rows(a, w)
    exact = a.astype(np.float64) @ w.astype(np.float64)
    err = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert 1e-3 < err < 0.05
