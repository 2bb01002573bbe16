"""Guard bands around output buffers.  compute-sanitizer is closed on this
pool, so these tests catch writes past an output instead.

Each output is the interior of a larger buffer.  The bands before and after it
hold a canary pattern, and every band must be untouched after the call.  The
cases are ragged, so the last tile of each kernel lies partly outside the
matrix.  They cover:
- the TMA-store and TMA-reduce epilogues of the GEMMs;
- the attention outputs;
- the e4m3 quantisers and the W8A8 projection."""
import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from helpers import dev

pytestmark = pytest.mark.gpu

G_ROWS = 3  # guard rows before and after each matrix


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    ispa_build.build()


def _guarded(rows, cols, dtype):
    """A [rows + 2 G_ROWS, cols] buffer filled with a canary bit pattern, and
    its interior view [rows, cols] (contiguous: whole rows)."""
    n_bytes = (rows + 2 * G_ROWS) * cols * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((n_bytes,), 0xA5, dtype=torch.uint8, device="cuda")
    buf = raw.view(dtype).view(rows + 2 * G_ROWS, cols)
    return buf, buf[G_ROWS:G_ROWS + rows]


def _bands_intact(buf):
    b = buf.contiguous().view(torch.uint8).view(buf.shape[0], -1)
    return bool(torch.all(b[:G_ROWS] == 0xA5)) and bool(torch.all(b[-G_ROWS:] == 0xA5))


def _vec_guarded(n, dtype):
    raw = torch.full(((n + 2 * 16) * torch.tensor([], dtype=dtype).element_size(),), 0xA5, dtype=torch.uint8,
                     device="cuda")
    buf = raw.view(dtype)
    return buf, buf[16:16 + n]


def _vec_intact(buf):
    b = buf.view(torch.uint8).view(-1)
    eb = buf.element_size()
    return bool(torch.all(b[:16 * eb] == 0xA5)) and bool(torch.all(b[-16 * eb:] == 0xA5))


def test_projection_tma_store_stays_inside():
    rng = np.random.default_rng(1)
    n, d_in, d_out = 300, 256, 384  # 300 rows: the second 256-row tile is mostly outside
    a = dev(rng.standard_normal((n, d_in)).astype(np.float32), "bf16")
    w = dev((rng.standard_normal((d_in, d_out)) / 16).astype(np.float32), "bf16")
    buf, y = _guarded(n, d_out, torch.bfloat16)
    ispa.project(a, w, y)
    torch.cuda.synchronize()
    assert _bands_intact(buf)
    assert torch.isfinite(y.float()).all()


def test_statistics_tma_reduce_stays_inside():
    rng = np.random.default_rng(2)
    n, D = 257, 384  # 384 = 1.5 tiles of 256: the lower tile row is half outside
    A = dev(rng.standard_normal((n, D)).astype(np.float32), "bf16")
    Dl = dev(rng.standard_normal((n, D)).astype(np.float32), "bf16")
    gbuf, G = _guarded(D, D, torch.float32)
    rbuf, R = _guarded(D, D, torch.float32)
    ispa.gram_accumulate(A, Dl, G, R, zero_first=True)
    ebuf, E = _guarded(D, D, torch.float32)
    ispa.sym_gram_accumulate(Dl, E, zero_first=True)
    torch.cuda.synchronize()
    assert _bands_intact(gbuf) and _bands_intact(rbuf) and _bands_intact(ebuf)


def test_attention_outputs_stay_inside():
    n_q, H, d = 333, 2, 128
    case = synth.random_case(3, n_q, H, d, [100, 333, 500], dtype="bf16")
    (ks, vs), (kc, vc), (kh, vh) = case["segments"]
    D = H * d
    out, bufs = {}, []
    for k in ("a_loc", "a_full", "a_delta"):
        b, v = _guarded(n_q, D, torch.bfloat16)
        out[k] = v
        bufs.append(b)
    vbufs = []
    for k in ("lse_loc", "lse_full"):  # [H, n_q] fp32 inside a flat guarded vector (16-byte aligned start)
        b, v = _vec_guarded(H * n_q, torch.float32)
        out[k] = v.view(H, n_q)
        vbufs.append(b)
    status = ispa.new_status()
    t = lambda z: dev(z, "bf16")
    ispa.dual_attention(t(case["q"]), [(t(ks), t(vs)), (t(kc), t(vc))], [(t(kh), t(vh))], H, out=out,
                        status=status)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "dual_attention")
    assert all(_bands_intact(b) for b in bufs) and all(_vec_intact(b) for b in vbufs)


def test_w8a8_kernels_stay_inside():
    rng = np.random.default_rng(4)
    n, d_in, d_out = 300, 48, 128  # K shorter than one 128-element stage; ragged rows
    a = dev(rng.standard_normal((n, d_in)).astype(np.float32), "bf16")
    w = dev((rng.standard_normal((d_in, d_out)) / 8).astype(np.float32), "bf16")
    qbuf, qa = _guarded(n, d_in, torch.uint8)
    sbuf, sa = _vec_guarded(n, torch.float32)
    ispa.quantize_e4m3_rows(a, qa, sa)
    wbuf, qwt = _guarded(d_out, d_in, torch.uint8)
    swbuf, sw = _vec_guarded(d_out, torch.float32)
    ispa.quantize_e4m3_weight(w, qwt, sw)
    ybuf, y = _guarded(n, d_out, torch.bfloat16)
    ispa.project_w8a8(qa, sa, qwt, sw, y)
    torch.cuda.synchronize()
    assert _bands_intact(qbuf) and _bands_intact(wbuf) and _bands_intact(ybuf)
    assert _vec_intact(sbuf) and _vec_intact(swbuf)
    assert torch.isfinite(y.float()).all()
