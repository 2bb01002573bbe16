"""GPU parity of the W8A8 output projection against the CPU oracle
(oracle/w8a8_oracle.py).  Source: "Instance-Specific Parametric Absorption",
gist.science technical summary, section 4 "Experimental Results", item
"Speedup" (ISPA with post-training W8A8 quantisation).

- The e4m3 codes and fp32 scales are integer-valued decisions taken in fp32
  on both sides, so they must match bit for bit.
- The projection from given codes is compared element by element.  The
  products of two e4m3 values are exact in fp32, so two things separate the
  GPU from the fp64 oracle:
  - the tensor core's summation.  For 8-bit inputs it may align partial sums
    to fewer bits than fp32 (the previous generation kept about 14), so it is
    bounded by 2^-11 of the sum of |terms|;
  - the final bf16 rounding, 2^-8 relative.
  The relative Frobenius error is bounded by 4e-3, which the bf16 rounding
  (about 2^-9 on average) dominates.
"""
import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from oracle import ispa_oracle as orc
from oracle import w8a8_oracle as w8
from helpers import CHAIN_W8A8_FRO, CHAIN_W8A8_MAX, REPORT, dev, fro_rel, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    ispa_build.build()


def _bf16(rng, shape, scale=1.0):
    return synth.round_bf16((rng.standard_normal(shape) * scale).astype(np.float32))


def _u8(t):
    return t.cpu().numpy()


def _f32(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("n,k,pad", [(4680, 1536, 0), (77, 128, 16), (1, 16, 0), (300, 5120, 0)])
def test_quantize_rows_bit_exact(n, k, pad):
    rng = np.random.default_rng(n + k)
    x = synth.round_bf16(_bf16(rng, (n, k)) * rng.uniform(1e-3, 1e2, (n, 1)).astype(np.float32))
    if n > 3:
        x[1] = 0.0                       # all-zero row: scale 1, zero codes
        x[2, : k // 2] *= np.float32(1e-4)  # subnormal codes next to the row maximum
        x[2] = synth.round_bf16(x[2])
        x[3, 5] = -0.0
    xd = torch.zeros(n, k + pad, dtype=torch.bfloat16, device="cuda")
    xd[:, :k] = dev(x, "bf16")
    codes, scales = ispa.quantize_e4m3_rows(xd[:, :k])
    torch.cuda.synchronize()
    qo, so = w8.quantize_rows(x)
    assert np.array_equal(_f32(scales), so)
    assert np.array_equal(_u8(codes), qo)


@pytest.mark.parametrize("d_in,d_out", [(1536, 1536), (128, 384), (5120, 256), (48, 16)])
def test_quantize_weight_bit_exact(d_in, d_out):
    rng = np.random.default_rng(d_in * 7 + d_out)
    w = _bf16(rng, (d_in, d_out), 1.0 / np.sqrt(d_in))
    w[:, 3] = 0.0
    w[:, 5] *= np.float32(1e3)
    w = synth.round_bf16(w)
    codes_t, scales = ispa.quantize_e4m3_weight(dev(w, "bf16"))
    torch.cuda.synchronize()
    qo, so = w8.quantize_cols(w)
    assert np.array_equal(_f32(scales), so)
    assert np.array_equal(_u8(codes_t), qo.T)


def _check_projection(y, qa, sa, qw, sw):
    ref = w8.project_codes(qa, sa, qw, sw)
    mag = w8.project_codes(qa & 0x7F, sa, qw & 0x7F, sw)  # sum of |terms| per element
    got = host(y)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -11 * mag + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    assert fro_rel(got, ref) <= 4e-3


@pytest.mark.parametrize("n,d_in,d_out", [(4680, 1536, 1536), (4680, 256, 1280), (300, 256, 384), (129, 128, 128),
                                          (1, 5120, 256), (517, 48, 128)])
def test_project_w8a8_matches_oracle(n, d_in, d_out):
    rng = np.random.default_rng(n + d_in + d_out)
    a = _bf16(rng, (n, d_in))
    w = _bf16(rng, (d_in, d_out), 1.0 / np.sqrt(d_in))
    qa, sa = w8.quantize_rows(a)
    qw, sw = w8.quantize_cols(w)
    y = ispa.project_w8a8(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                          torch.from_numpy(np.ascontiguousarray(qw.T)).cuda(), torch.from_numpy(sw).cuda())
    torch.cuda.synchronize()
    _check_projection(y, qa, sa, qw, sw)


def test_quantise_then_project_chain_matches_oracle():
    """The three device steps chained (weight codes, activation codes,
    projection) against the oracle's W8A8 projection of the same inputs."""
    rng = np.random.default_rng(21)
    a = _bf16(rng, (1000, 1536))
    w = _bf16(rng, (1536, 1536), 1.0 / np.sqrt(1536))
    qwt, sw = ispa.quantize_e4m3_weight(dev(w, "bf16"))
    qa, sa = ispa.quantize_e4m3_rows(dev(a, "bf16"))
    y = ispa.project_w8a8(qa, sa, qwt, sw)
    torch.cuda.synchronize()
    qa_o, sa_o = w8.quantize_rows(a)
    qw_o, sw_o = w8.quantize_cols(w)
    _check_projection(y, qa_o, sa_o, qw_o, sw_o)
    # W8A8 against the exact product: lossy, within the e4m3 error
    exact = a.astype(np.float64) @ w.astype(np.float64)
    assert 1e-3 < fro_rel(host(y), exact) < 0.05


def test_local_attention_project_w8a8_wan13b_sampled_rows():
    """L-layer of the Wan-1.3B shapes with the W8A8 projection: 4680 chunk
    queries over sink + current keys (6240).  The oracle's attention gives
    A_loc for 48 sampled rows (the last row included).  Its W8A8 projection
    with the weight quantised over all of W is the reference.

    Tolerance.  The GPU's bf16 A_loc differs from the oracle's by the
    attention error, so a few codes land one e4m3 step (2^-3 relative) away.
    Simulated in the oracle (2^-9 relative noise on A_loc before its bf16
    rounding, three draws): relative Frobenius error 1.4-1.6e-2, largest
    element error 1.6-1.9e-2 of max|y|.  The bounds are CHAIN_W8A8_FRO and
    CHAIN_W8A8_MAX (tests/helpers.py), about 2.5x the simulation of
    tests/chain_tolerances.py."""
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.single_layer_inputs(w, 1)
    W = synth.weight(w, 0)
    qwt, sw = ispa.quantize_e4m3_weight(dev(W, "bf16"))
    status = ispa.new_status()
    out = ispa.local_attention_project_w8a8(dev(x["q"], "bf16"),
                                            [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")),
                                             (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))],
                                            qwt, sw, w.n_heads, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "local_attention_project_w8a8")
    rows = np.sort(np.random.default_rng(5).choice(w.n_q, 48, replace=False))
    rows[-1] = w.n_q - 1
    a_ref, _ = orc.attention(x["q"][rows], np.concatenate([x["k_sink"], x["k_cur"]]),
                             np.concatenate([x["v_sink"], x["v_cur"]]), w.n_heads)
    # the pipeline stores A_loc in bf16 before quantising it
    y_ref = w8.project_w8a8(synth.round_bf16(a_ref.astype(np.float32)), W)
    y = host(out["y"])[rows]
    REPORT.append(("W8A8 L-layer chain: y (relative Frobenius)", fro_rel(y, y_ref), fro_rel(y, y_ref)))
    assert fro_rel(y, y_ref) <= CHAIN_W8A8_FRO
    assert np.max(np.abs(y - y_ref)) <= CHAIN_W8A8_MAX * np.max(np.abs(y_ref))
    # the quantised weight is the oracle's, bit for bit
    qw_o, sw_o = w8.quantize_cols(W)
    assert np.array_equal(_u8(qwt), qw_o.T) and np.array_equal(_f32(sw), sw_o)


# ---------------------------------------------------------------- MX form
def _mx_rows_input(rng, n, k):
    """bf16 rows whose 32-element blocks span many binades, with the edge
    cases of the exponent rule: an all-zero block, a block whose largest
    magnitude has mantissa exactly 1.75 (448 * 2^j: no carry), one just
    above, and one of bf16 subnormals."""
    x = _bf16(rng, (n, k)) * np.exp2(rng.integers(-20, 20, (n, k // 32))).repeat(32, 1).astype(np.float32)
    x = synth.round_bf16(x.astype(np.float32))
    if n > 4 and k >= 128:
        x[0, 0:32] = 0.0
        x[1, 32:64] = np.float32(0.5)
        x[1, 40] = np.float32(-448.0 * 2.0 ** -5)
        x[2, 64:96] = np.float32(0.25)
        x[2, 70] = synth.round_bf16(np.array([448.0 * 2.0 ** -3 * (1 + 2.0 ** -7)], np.float32))[0]
        x[3, 96:128] = np.float32(2.0 ** -130)
    return x


@pytest.mark.parametrize("n,k,pad", [(4680, 1536, 0), (300, 256, 32), (1, 32, 0), (77, 5120, 0)])
def test_mx_quantize_rows_bit_exact(n, k, pad):
    rng = np.random.default_rng(3 * n + k)
    x = _mx_rows_input(rng, n, k)
    xd = torch.zeros(n, k + pad, dtype=torch.bfloat16, device="cuda")
    xd[:, :k] = dev(x, "bf16")
    codes, exps = ispa.mx_quantize_e4m3_rows(xd[:, :k])
    torch.cuda.synchronize()
    qo, eo = w8.mx_quantize_rows(x)
    assert np.array_equal(_u8(exps).astype(np.int64) - 127, eo)
    assert np.array_equal(_u8(codes), qo)


def _check_mx_projection(y, qa, ea, qw, sw):
    ref = w8.mx_rows_project_codes(qa, ea, qw, sw)
    mag = w8.mx_rows_project_codes(qa & 0x7F, ea, qw & 0x7F, sw)
    got = host(y)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -11 * mag + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    assert fro_rel(got, ref) <= 4e-3


# (4680, 1536, 1536): the wan1.3b L-layer; (517, 1536, 1280): ragged rows and
# an overhanging last column tile; (1, 3584, 256): the longest K the tile's
# scales fit; (129, 128, 128): one K stage
@pytest.mark.parametrize("n,d_in,d_out", [(4680, 1536, 1536), (517, 1536, 1280), (1, 3584, 256), (129, 128, 128)])
def test_project_mx_matches_oracle(n, d_in, d_out):
    rng = np.random.default_rng(n + 3 * d_in + d_out)
    a = _mx_rows_input(rng, n, d_in)
    w = _bf16(rng, (d_in, d_out), 1.0 / np.sqrt(d_in))
    qa, ea = w8.mx_quantize_rows(a)
    qw, sw = w8.quantize_cols(w)
    y = ispa.project_mx(torch.from_numpy(qa).cuda(), torch.from_numpy((ea + 127).astype(np.uint8)).cuda(),
                        torch.from_numpy(np.ascontiguousarray(qw.T)).cuda(), torch.from_numpy(sw).cuda())
    torch.cuda.synchronize()
    _check_mx_projection(y, qa, ea, qw, sw)


def test_project_mx_rejects_long_k_before_launch():
    z = torch.zeros(16, 3712, dtype=torch.uint8, device="cuda")
    with pytest.raises(ispa.IspaError) as ei:
        ispa.project_mx(z, torch.zeros(16, 116, dtype=torch.uint8, device="cuda"),
                        torch.zeros(128, 3712, dtype=torch.uint8, device="cuda"),
                        torch.ones(128, device="cuda"))
    assert ei.value.code == 2


def test_local_attention_project_mx_wan13b():
    """The fused MX L-layer at the Wan-1.3B shapes (4680 chunk queries over
    sink + current keys).  The attention epilogue quantises its bf16 output:
    the plain single-pass attention of the same launch shape gives that bf16
    A_loc bit for bit (attention parity against the oracle is tested
    elsewhere), and the oracle's MX quantisation of it must equal the codes
    and exponents the epilogue wrote.  y is the oracle's block-scaled product
    of those codes with the oracle's weight codes, within the projection
    bound."""
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.single_layer_inputs(w, 1)
    W = synth.weight(w, 0)
    qwt, sw = ispa.quantize_e4m3_weight(dev(W, "bf16"))
    status = ispa.new_status()
    q = dev(x["q"], "bf16")
    local = [(dev(x["k_sink"], "bf16"), dev(x["v_sink"], "bf16")), (dev(x["k_cur"], "bf16"), dev(x["v_cur"], "bf16"))]
    out = ispa.local_attention_project_mx(q, local, qwt, sw, w.n_heads, status=status)
    plain = ispa.dual_attention(q, local, [], w.n_heads, dual=False, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "local_attention_project_mx")
    a_bf16 = host(plain["a_full"])
    qo, eo = w8.mx_quantize_rows(a_bf16)
    assert np.array_equal(_u8(out["a_exps"]).astype(np.int64) - 127, eo)
    assert np.array_equal(_u8(out["a_codes"]), qo)
    qw_o, sw_o = w8.quantize_cols(W)
    _check_mx_projection(out["y"], qo, eo, qw_o, sw_o)
    # MX against the bf16 projection of the same A_loc: lossy, within e4m3 error
    exact = a_bf16.astype(np.float64) @ W.astype(np.float64)
    err = fro_rel(host(out["y"]), exact)
    REPORT.append(("MX L-layer: y against the bf16 product (relative Frobenius)", err, err))
    assert 1e-3 < err < 0.05


def test_local_attention_project_mx_head_dim_64_ragged():
    """The MX epilogue with head_dim 64 (one 32-channel block per warpgroup
    and row), 4 heads, a ragged last query tile and ragged key segments:
    codes and exponents bit-exact against the oracle's MX quantisation of the
    plain pass's bf16 output, y within the projection bound."""
    H, d, n_q = 4, 64, 300
    c = synth.random_case(77, n_q, H, d, [100, 333])
    q = dev(c["q"], "bf16")
    local = [(dev(k, "bf16"), dev(v, "bf16")) for k, v in c["segments"]]
    rng = np.random.default_rng(78)
    W = _bf16(rng, (H * d, H * d), 1.0 / np.sqrt(H * d))
    qwt, sw = ispa.quantize_e4m3_weight(dev(W, "bf16"))
    status = ispa.new_status()
    out = ispa.local_attention_project_mx(q, local, qwt, sw, H, status=status)
    plain = ispa.dual_attention(q, local, [], H, dual=False, status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "local_attention_project_mx")
    qo, eo = w8.mx_quantize_rows(host(plain["a_full"]))
    assert np.array_equal(_u8(out["a_exps"]).astype(np.int64) - 127, eo)
    assert np.array_equal(_u8(out["a_codes"]), qo)
    qw_o, sw_o = w8.quantize_cols(W)
    _check_mx_projection(out["y"], qo, eo, qw_o, sw_o)

