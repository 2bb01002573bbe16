"""Python binding of libispa (ctypes), same names as the C ABI in include/ispa.h.

Argument marshalling only: tensors are passed as raw device pointers with their
sizes and strides, the caller's current CUDA stream is forwarded, and non-OK
status codes raise ``IspaError``.  Every step of the computation runs in the
CUDA kernels of libispa.so; there is no fallback of any kind -- importing the
functions works without a GPU, but calling a device entry point without the
built library or without a GPU raises.

Thin convenience wrappers (``dual_attention``, ``gram_accumulate``,
``absorb_solve``, ``local_attention_project``, ``project``, ``lse_merge``)
allocate the outputs with torch and call the C entry points.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libispa.so")

ISPA_OK = 0
STATUS_NAMES = {0: "ISPA_OK", 1: "ISPA_ERR_INVALID_ARG", 2: "ISPA_ERR_UNSUPPORTED", 3: "ISPA_ERR_CUDA",
                4: "ISPA_ERR_NOT_SPD", 5: "ISPA_ERR_TIMEOUT", 6: "ISPA_ERR_WORKSPACE"}
DT_BF16, DT_F32 = 0, 1
MAX_SEGMENTS = 8

# every symbol declared in include/ispa.h
EXPORTED = ("ispa_dual_attention", "ispa_lse_merge", "ispa_gram_accumulate", "ispa_sym_gram_accumulate",
            "ispa_layer_error_workspace_bytes", "ispa_layer_error", "ispa_select_layers", "ispa_absorb_workspace_bytes",
            "ispa_absorb_solve", "ispa_absorb_solve_noalloc", "ispa_project", "ispa_local_attention_project",
            "ispa_quantize_e4m3_rows", "ispa_quantize_e4m3_weight", "ispa_project_w8a8",
            "ispa_local_attention_project_w8a8", "ispa_mx_quantize_e4m3_rows", "ispa_project_mx",
            "ispa_local_attention_project_mx",
            "ispa_chunk_token_ranges", "ispa_kv_bytes", "ispa_selftest_wait_timeout", "ispa_status_string", "ispa_last_error",
            "ispa_version")


class IspaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}: {detail}")


class KVSegment(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n_tokens", ctypes.c_int64),
                ("row_stride", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libispa.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m ar_video_diffusion_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        i32, i64, f32, f64, vp, sz = c.c_int32, c.c_int64, c.c_float, c.c_double, c.c_void_p, c.c_size_t
        seg_p = c.POINTER(KVSegment)
        sig = {
            "ispa_dual_attention": (i32, [vp, i64, i64, i32, i32, i32, f32, seg_p, i32, seg_p, i32, vp, vp, vp, vp,
                                          vp, vp, vp]),
            "ispa_lse_merge": (i32, [vp, vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, vp]),
            "ispa_gram_accumulate": (i32, [vp, vp, i64, i64, i64, i32, vp, vp, i32, vp]),
            "ispa_sym_gram_accumulate": (i32, [vp, i64, i64, i64, i32, vp, i32, vp]),
            "ispa_layer_error_workspace_bytes": (sz, [i64]),
            "ispa_layer_error": (i32, [vp, vp, vp, vp, i32, vp, i64, vp, sz, vp, vp]),
            "ispa_select_layers": (i32, [c.POINTER(f64), i32, i32, c.POINTER(c.c_uint8)]),
            "ispa_absorb_workspace_bytes": (sz, [i64]),
            "ispa_absorb_solve": (i32, [vp, vp, vp, i32, i64, f64, f64, vp, vp, vp, sz, vp, vp]),
            "ispa_absorb_solve_noalloc": (i32, [vp, vp, vp, i32, i64, f64, f64, vp, vp, vp, vp]),
            "ispa_project": (i32, [vp, i64, i64, i64, i64, i32, vp, vp, vp]),
            "ispa_local_attention_project": (i32, [vp, i64, i64, i32, i32, i32, f32, seg_p, i32, vp, vp, vp, vp,
                                                   vp]),
            "ispa_quantize_e4m3_rows": (i32, [vp, i64, i64, i64, i32, vp, vp, vp]),
            "ispa_quantize_e4m3_weight": (i32, [vp, i64, i64, i32, vp, vp, vp]),
            "ispa_project_w8a8": (i32, [vp, vp, i64, i64, vp, vp, i64, vp, vp]),
            "ispa_local_attention_project_w8a8": (i32, [vp, i64, i64, i32, i32, i32, f32, seg_p, i32, vp, vp, vp,
                                                        vp, vp, vp, vp, vp]),
            "ispa_mx_quantize_e4m3_rows": (i32, [vp, i64, i64, i64, i32, vp, vp, vp]),
            "ispa_project_mx": (i32, [vp, vp, i64, i64, vp, vp, i64, vp, vp]),
            "ispa_local_attention_project_mx": (i32, [vp, i64, i64, i32, i32, i32, f32, seg_p, i32, vp, vp, vp,
                                                      vp, vp, vp, vp]),
            "ispa_chunk_token_ranges": (i32, [i64, i64, i64, i64, c.POINTER(i64)]),
            "ispa_kv_bytes": (i64, [i64, i32, c.c_uint64, i32, i64, i64, i64, i32, i64]),
            "ispa_selftest_wait_timeout": (i32, [c.c_uint32, vp, vp]),
            "ispa_status_string": (c.c_char_p, [i32]),
            "ispa_last_error": (c.c_char_p, []),
            "ispa_version": (i32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != ISPA_OK:
        raise IspaError(code, where, lib().ispa_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _row_stride(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D row-major matrix")
    return t.stride(0)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _segments(pairs: Sequence[Tuple[torch.Tensor, torch.Tensor]]):
    arr = (KVSegment * max(1, len(pairs)))()
    for i, (k, v) in enumerate(pairs):
        if k.shape != v.shape or k.stride() != v.stride():
            raise ValueError("k and v of a segment must have the same shape and strides")
        arr[i] = KVSegment(_dev(k, "k") if k.numel() else None, _dev(v, "v") if v.numel() else None,
                           k.shape[0], _row_stride(k, "k") if k.shape[0] else k.shape[1])
    return arr, len(pairs)


# ------------------------------------------------------------ raw C entry points
def ispa_dual_attention(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local, hist, n_hist,
                        a_loc, a_full, a_delta, lse_loc, lse_full, dev_status, stream):
    _check(lib().ispa_dual_attention(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local, hist,
                                     n_hist, a_loc, a_full, a_delta, lse_loc, lse_full, dev_status, stream),
           "ispa_dual_attention")


def ispa_lse_merge(o_loc, lse_loc, o_hist, lse_hist, n_q, n_heads, head_dim, dt, a_full, a_delta, lse_full, stream):
    _check(lib().ispa_lse_merge(o_loc, lse_loc, o_hist, lse_hist, n_q, n_heads, head_dim, dt, a_full, a_delta,
                                lse_full, stream), "ispa_lse_merge")


def ispa_gram_accumulate(a_loc, a_delta, n_rows, d_model, row_stride, dt, G, R, zero_first, stream):
    _check(lib().ispa_gram_accumulate(a_loc, a_delta, n_rows, d_model, row_stride, dt, G, R, zero_first, stream),
           "ispa_gram_accumulate")


def ispa_sym_gram_accumulate(x, n_rows, d_model, row_stride, dt, E, zero_first, stream):
    _check(lib().ispa_sym_gram_accumulate(x, n_rows, d_model, row_stride, dt, E, zero_first, stream),
           "ispa_sym_gram_accumulate")


def ispa_layer_error_workspace_bytes(d_model: int) -> int:
    return lib().ispa_layer_error_workspace_bytes(d_model)


def ispa_layer_error(G, R, E, W, w_dt, delta_w, d_model, workspace, workspace_bytes, num_den, stream):
    _check(lib().ispa_layer_error(G, R, E, W, w_dt, delta_w, d_model, workspace, workspace_bytes, num_den, stream),
           "ispa_layer_error")


def ispa_select_layers(eps, n_layers, k, selected):
    _check(lib().ispa_select_layers(eps, n_layers, k, selected), "ispa_select_layers")


def ispa_absorb_workspace_bytes(d_model: int) -> int:
    return lib().ispa_absorb_workspace_bytes(d_model)


def ispa_absorb_solve(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new, workspace, workspace_bytes,
                      dev_status, stream):
    _check(lib().ispa_absorb_solve(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new, workspace,
                                   workspace_bytes, dev_status, stream), "ispa_absorb_solve")


def ispa_absorb_solve_noalloc(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new, dev_status, stream):
    _check(lib().ispa_absorb_solve_noalloc(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new,
                                           dev_status, stream), "ispa_absorb_solve_noalloc")


def ispa_project(a, n_rows, d_in, d_out, a_stride, dt, w, y, stream):
    _check(lib().ispa_project(a, n_rows, d_in, d_out, a_stride, dt, w, y, stream), "ispa_project")


def ispa_local_attention_project(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local, w_new, y,
                                 a_loc_out, dev_status, stream):
    _check(lib().ispa_local_attention_project(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local,
                                              n_local, w_new, y, a_loc_out, dev_status, stream),
           "ispa_local_attention_project")


def ispa_quantize_e4m3_rows(x, n_rows, k, row_stride, dt, codes, scales, stream):
    _check(lib().ispa_quantize_e4m3_rows(x, n_rows, k, row_stride, dt, codes, scales, stream),
           "ispa_quantize_e4m3_rows")


def ispa_quantize_e4m3_weight(w, d_in, d_out, dt, codes_t, scales, stream):
    _check(lib().ispa_quantize_e4m3_weight(w, d_in, d_out, dt, codes_t, scales, stream), "ispa_quantize_e4m3_weight")


def ispa_project_w8a8(a_codes, a_scales, n_rows, d_in, w_codes_t, w_scales, d_out, y, stream):
    _check(lib().ispa_project_w8a8(a_codes, a_scales, n_rows, d_in, w_codes_t, w_scales, d_out, y, stream),
           "ispa_project_w8a8")


def ispa_local_attention_project_w8a8(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local,
                                      w_codes_t, w_scales, y, a_loc_out, a_codes, a_scales, dev_status, stream):
    _check(lib().ispa_local_attention_project_w8a8(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local,
                                                   n_local, w_codes_t, w_scales, y, a_loc_out, a_codes, a_scales,
                                                   dev_status, stream), "ispa_local_attention_project_w8a8")


def ispa_mx_quantize_e4m3_rows(x, n_rows, k, row_stride, dt, codes, exps, stream):
    _check(lib().ispa_mx_quantize_e4m3_rows(x, n_rows, k, row_stride, dt, codes, exps, stream),
           "ispa_mx_quantize_e4m3_rows")


def ispa_project_mx(a_codes, a_exps, n_rows, d_in, w_codes_t, w_scales, d_out, y, stream):
    _check(lib().ispa_project_mx(a_codes, a_exps, n_rows, d_in, w_codes_t, w_scales, d_out, y, stream),
           "ispa_project_mx")


def ispa_local_attention_project_mx(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local,
                                    w_codes_t, w_scales, y, a_codes, a_exps, dev_status, stream):
    _check(lib().ispa_local_attention_project_mx(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local,
                                                 n_local, w_codes_t, w_scales, y, a_codes, a_exps, dev_status,
                                                 stream), "ispa_local_attention_project_mx")


def ispa_chunk_token_ranges(chunk: int, frame_tokens: int, chunk_frames: int, sink_frames: int = 1):
    out = (ctypes.c_int64 * 6)()
    _check(lib().ispa_chunk_token_ranges(chunk, frame_tokens, chunk_frames, sink_frames, out),
           "ispa_chunk_token_ranges")
    return {"sink": (out[0], out[1]), "hist": (out[2], out[3]), "cur": (out[4], out[5])}


def ispa_kv_bytes(chunk, n_layers, l_layer_mask, transitioned, frame_tokens, chunk_frames, d_model, elem_bytes,
                  sink_frames=1) -> int:
    r = lib().ispa_kv_bytes(chunk, n_layers, l_layer_mask, int(bool(transitioned)), frame_tokens, chunk_frames,
                            d_model, elem_bytes, sink_frames)
    if r < 0:
        raise IspaError(1, "ispa_kv_bytes", "invalid arguments")
    return r


def ispa_selftest_wait_timeout(timeout_us, dev_status, stream):
    _check(lib().ispa_selftest_wait_timeout(timeout_us, dev_status, stream), "ispa_selftest_wait_timeout")


def ispa_status_string(code: int) -> str:
    return lib().ispa_status_string(code).decode()


def ispa_version() -> int:
    return lib().ispa_version()


# ------------------------------------------------------- torch-level wrappers
def new_status(device="cuda") -> torch.Tensor:
    """Zeroed two-int32 device status word (code, detail)."""
    return torch.zeros(2, dtype=torch.int32, device=device)


def raise_on_status(status: torch.Tensor, where: str):
    code, detail = (int(x) for x in status.cpu().tolist())
    if code != 0:
        raise IspaError(code, where, f"device status detail {detail}")


def dual_attention(q: torch.Tensor, local: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                   hist: Sequence[Tuple[torch.Tensor, torch.Tensor]], n_heads: int, softmax_scale: float = 0.0,
                   dual: bool = True, out: Optional[dict] = None, status: Optional[torch.Tensor] = None,
                   stream=None) -> dict:
    """Decomposable Attention of one chunk; returns a dict of output tensors.

    dual=True: a_loc, a_full, a_delta, lse_loc, lse_full.  dual=False: one
    pass over local + hist giving a_full and lse_full.
    """
    n_q, D = q.shape
    head_dim = D // n_heads
    dev = q.device
    if out is None:
        out = {"a_full": torch.empty(n_q, D, dtype=q.dtype, device=dev),
               "lse_full": torch.empty(n_heads, n_q, dtype=torch.float32, device=dev)}
        if dual:
            out["a_loc"] = torch.empty(n_q, D, dtype=q.dtype, device=dev)
            out["a_delta"] = torch.empty(n_q, D, dtype=q.dtype, device=dev)
            out["lse_loc"] = torch.empty(n_heads, n_q, dtype=torch.float32, device=dev)
    ls, nl = _segments(local)
    hs, nh = _segments(hist)
    ispa_dual_attention(_dev(q, "q"), n_q, _row_stride(q, "q"), n_heads, head_dim, _dtype_code(q), softmax_scale,
                        ls, nl, hs, nh, _dev(out.get("a_loc"), "a_loc"), _dev(out["a_full"], "a_full"),
                        _dev(out.get("a_delta"), "a_delta"), _dev(out.get("lse_loc"), "lse_loc"),
                        _dev(out.get("lse_full"), "lse_full"), _dev(status, "status"), _stream(stream))
    return out


def lse_merge(o_loc, lse_loc, o_hist, lse_hist, n_heads: int, out: Optional[dict] = None, stream=None) -> dict:
    n_q, D = o_loc.shape
    if out is None:
        out = {"a_full": torch.empty_like(o_loc), "a_delta": torch.empty_like(o_loc),
               "lse_full": torch.empty_like(lse_loc)}
    ispa_lse_merge(_dev(o_loc, "o_loc"), _dev(lse_loc, "lse_loc"), _dev(o_hist, "o_hist"), _dev(lse_hist, "lse_hist"),
                   n_q, n_heads, D // n_heads, _dtype_code(o_loc), _dev(out["a_full"], "a_full"),
                   _dev(out.get("a_delta"), "a_delta"), _dev(out.get("lse_full"), "lse_full"), _stream(stream))
    return out


def gram_accumulate(a_loc: torch.Tensor, a_delta: torch.Tensor, G: torch.Tensor, R: torch.Tensor,
                    zero_first: bool = False, stream=None):
    n, D = a_loc.shape
    ispa_gram_accumulate(_dev(a_loc, "a_loc"), _dev(a_delta, "a_delta"), n, D, _row_stride(a_loc, "a_loc"),
                         _dtype_code(a_loc), _dev(G, "G"), _dev(R, "R"), int(zero_first), _stream(stream))


def sym_gram_accumulate(x: torch.Tensor, E: torch.Tensor, zero_first: bool = False, stream=None):
    """E (+)= x^T x, lower triangle (x = A_full - A_loc for the layer selection)."""
    n, D = x.shape
    ispa_sym_gram_accumulate(_dev(x, "x"), n, D, _row_stride(x, "x"), _dtype_code(x), _dev(E, "E"), int(zero_first),
                             _stream(stream))


def layer_error(G: torch.Tensor, R: torch.Tensor, E: torch.Tensor, W: torch.Tensor, delta_w: torch.Tensor,
                workspace: Optional[torch.Tensor] = None, num_den: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Device float64 tensor [num, den]: the layer's reconstruction error is num / den."""
    D = G.shape[0]
    if workspace is None:
        workspace = torch.empty(ispa_layer_error_workspace_bytes(D), dtype=torch.uint8, device=G.device)
    if num_den is None:
        num_den = torch.empty(2, dtype=torch.float64, device=G.device)
    ispa_layer_error(_dev(G, "G"), _dev(R, "R"), _dev(E, "E"), _dev(W, "W"), _dtype_code(W), _dev(delta_w, "delta_w"),
                     D, _dev(workspace, "workspace"), workspace.numel(), _dev(num_den, "num_den"), _stream(stream))
    return num_den


def select_layers(eps: Sequence[float], k: int) -> List[int]:
    """Indices (increasing) of the k layers with the smallest error, ties to the lower index."""
    n = len(eps)
    arr = (ctypes.c_double * max(n, 1))(*[float(e) for e in eps])
    sel = (ctypes.c_uint8 * max(n, 1))()
    ispa_select_layers(arr, n, k, sel)
    return [l for l in range(n) if sel[l]]


def absorb_workspace(d_model: int, device="cuda") -> torch.Tensor:
    nbytes = ispa_absorb_workspace_bytes(d_model)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def absorb_solve(G: torch.Tensor, R: torch.Tensor, W: torch.Tensor, lambda_rel: float = 1e-2,
                 lambda_abs: float = 0.0, workspace: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None, delta_w: Optional[torch.Tensor] = None,
                 w_new: Optional[torch.Tensor] = None, stream=None):
    D = G.shape[0]
    if workspace is None:
        workspace = absorb_workspace(D, G.device)
    if delta_w is None:
        delta_w = torch.empty(D, D, dtype=torch.float32, device=G.device)
    if w_new is None:
        w_new = torch.empty_like(W)
    ispa_absorb_solve(_dev(G, "G"), _dev(R, "R"), _dev(W, "W"), _dtype_code(W), D, lambda_abs, lambda_rel,
                      _dev(delta_w, "delta_w"), _dev(w_new, "w_new"), _dev(workspace, "workspace"),
                      workspace.numel(), _dev(status, "status"), _stream(stream))
    return delta_w, w_new


def project(a: torch.Tensor, w: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    n, d_in = a.shape
    d_out = w.shape[1]
    if y is None:
        y = torch.empty(n, d_out, dtype=a.dtype, device=a.device)
    ispa_project(_dev(a, "a"), n, d_in, d_out, _row_stride(a, "a"), _dtype_code(a), _dev(w, "w"), _dev(y, "y"),
                 _stream(stream))
    return y


def local_attention_project(q: torch.Tensor, local: Sequence[Tuple[torch.Tensor, torch.Tensor]], w_new: torch.Tensor,
                            n_heads: int, softmax_scale: float = 0.0, y: Optional[torch.Tensor] = None,
                            a_loc: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                            stream=None):
    n_q, D = q.shape
    if y is None:
        y = torch.empty(n_q, D, dtype=q.dtype, device=q.device)
    if a_loc is None:
        a_loc = torch.empty(n_q, D, dtype=q.dtype, device=q.device)
    ls, nl = _segments(local)
    ispa_local_attention_project(_dev(q, "q"), n_q, _row_stride(q, "q"), n_heads, D // n_heads, _dtype_code(q),
                                 softmax_scale, ls, nl, _dev(w_new, "w_new"), _dev(y, "y"), _dev(a_loc, "a_loc"),
                                 _dev(status, "status"), _stream(stream))
    return y, a_loc


def quantize_e4m3_rows(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                       scales: Optional[torch.Tensor] = None, stream=None):
    """Per-row e4m3 codes (uint8 [n, k]) and fp32 scales [n] of bf16 x [n, k]."""
    n, k = x.shape
    if codes is None:
        codes = torch.empty(n, k, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(n, dtype=torch.float32, device=x.device)
    ispa_quantize_e4m3_rows(_dev(x, "x"), n, k, _row_stride(x, "x"), _dtype_code(x), _dev(codes, "codes"),
                            _dev(scales, "scales"), _stream(stream))
    return codes, scales


def quantize_e4m3_weight(w: torch.Tensor, codes_t: Optional[torch.Tensor] = None,
                         scales: Optional[torch.Tensor] = None, stream=None):
    """Per-output-channel e4m3 codes of bf16 w [d_in, d_out], returned
    TRANSPOSED (uint8 [d_out, d_in]), and fp32 scales [d_out]."""
    d_in, d_out = w.shape
    if codes_t is None:
        codes_t = torch.empty(d_out, d_in, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(d_out, dtype=torch.float32, device=w.device)
    ispa_quantize_e4m3_weight(_dev(w, "w"), d_in, d_out, _dtype_code(w), _dev(codes_t, "codes_t"),
                              _dev(scales, "scales"), _stream(stream))
    return codes_t, scales


def project_w8a8(a_codes: torch.Tensor, a_scales: torch.Tensor, w_codes_t: torch.Tensor, w_scales: torch.Tensor,
                 y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 y [n, d_out] of the W8A8 projection from the two sets of codes."""
    n, d_in = a_codes.shape
    d_out = w_codes_t.shape[0]
    if y is None:
        y = torch.empty(n, d_out, dtype=torch.bfloat16, device=a_codes.device)
    ispa_project_w8a8(_dev(a_codes, "a_codes"), _dev(a_scales, "a_scales"), n, d_in, _dev(w_codes_t, "w_codes_t"),
                      _dev(w_scales, "w_scales"), d_out, _dev(y, "y"), _stream(stream))
    return y


def local_attention_project_w8a8(q: torch.Tensor, local: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                                 w_codes_t: torch.Tensor, w_scales: torch.Tensor, n_heads: int,
                                 softmax_scale: float = 0.0, out: Optional[dict] = None,
                                 status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """L-layer with the W8A8 projection: local attention (bf16) -> A_loc ->
    e4m3 codes -> y.  Returns {"y", "a_loc", "a_codes", "a_scales"}."""
    n_q, D = q.shape
    if out is None:
        dev = q.device
        out = {"y": torch.empty(n_q, D, dtype=torch.bfloat16, device=dev),
               "a_loc": torch.empty(n_q, D, dtype=torch.bfloat16, device=dev),
               "a_codes": torch.empty(n_q, D, dtype=torch.uint8, device=dev),
               "a_scales": torch.empty(n_q, dtype=torch.float32, device=dev)}
    ls, nl = _segments(local)
    ispa_local_attention_project_w8a8(_dev(q, "q"), n_q, _row_stride(q, "q"), n_heads, D // n_heads,
                                      _dtype_code(q), softmax_scale, ls, nl, _dev(w_codes_t, "w_codes_t"),
                                      _dev(w_scales, "w_scales"), _dev(out["y"], "y"), _dev(out["a_loc"], "a_loc"),
                                      _dev(out["a_codes"], "a_codes"), _dev(out["a_scales"], "a_scales"),
                                      _dev(status, "status"), _stream(stream))
    return out


def mx_quantize_e4m3_rows(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                          exps: Optional[torch.Tensor] = None, stream=None):
    """MX e4m3 codes (uint8 [n, k]) and block exponent bytes (uint8
    [n, k / 32], ue8m0: e + 127) of bf16 x [n, k]."""
    n, k = x.shape
    if codes is None:
        codes = torch.empty(n, k, dtype=torch.uint8, device=x.device)
    if exps is None:
        exps = torch.empty(n, k // 32, dtype=torch.uint8, device=x.device)
    ispa_mx_quantize_e4m3_rows(_dev(x, "x"), n, k, _row_stride(x, "x"), _dtype_code(x), _dev(codes, "codes"),
                               _dev(exps, "exps"), _stream(stream))
    return codes, exps


def project_mx(a_codes: torch.Tensor, a_exps: torch.Tensor, w_codes_t: torch.Tensor, w_scales: torch.Tensor,
               y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 y [n, d_out] of the block-scaled projection of MX activation codes
    by per-channel weight codes."""
    n, d_in = a_codes.shape
    d_out = w_codes_t.shape[0]
    if y is None:
        y = torch.empty(n, d_out, dtype=torch.bfloat16, device=a_codes.device)
    ispa_project_mx(_dev(a_codes, "a_codes"), _dev(a_exps, "a_exps"), n, d_in, _dev(w_codes_t, "w_codes_t"),
                    _dev(w_scales, "w_scales"), d_out, _dev(y, "y"), _stream(stream))
    return y


def local_attention_project_mx(q: torch.Tensor, local: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                               w_codes_t: torch.Tensor, w_scales: torch.Tensor, n_heads: int,
                               softmax_scale: float = 0.0, out: Optional[dict] = None,
                               status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """L-layer with the MX projection: local attention whose epilogue writes
    MX codes of A_loc -> block-scaled product.  Returns {"y", "a_codes",
    "a_exps"}."""
    n_q, D = q.shape
    if out is None:
        dev = q.device
        out = {"y": torch.empty(n_q, D, dtype=torch.bfloat16, device=dev),
               "a_codes": torch.empty(n_q, D, dtype=torch.uint8, device=dev),
               "a_exps": torch.empty(n_q, D // 32, dtype=torch.uint8, device=dev)}
    ls, nl = _segments(local)
    ispa_local_attention_project_mx(_dev(q, "q"), n_q, _row_stride(q, "q"), n_heads, D // n_heads,
                                    _dtype_code(q), softmax_scale, ls, nl, _dev(w_codes_t, "w_codes_t"),
                                    _dev(w_scales, "w_scales"), _dev(out["y"], "y"), _dev(out["a_codes"], "a_codes"),
                                    _dev(out["a_exps"], "a_exps"), _dev(status, "status"), _stream(stream))
    return out
