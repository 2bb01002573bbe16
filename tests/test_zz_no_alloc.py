"""ispa_absorb_solve_noalloc: the absorb solve for callers that cannot
allocate device memory (host callbacks, allocator hooks, plugins handed
device pointers but no allocator, serving processes with memory fixed up
front).  Its working matrices come from a device array inside libispa, so the
caller passes only G, R, W and the outputs.

The tests call it through the C ABI, each case twice in a row -- every call
after the first finds an earlier call's leftovers in the shared array, among
them those of a larger call -- and compare each result with ispa_absorb_solve
given a caller-allocated workspace, within the dW tolerance of the other
absorb tests.  The cases cover each way the solve uses the array: bf16 W with
d_model a multiple of 128 (tensor-core S = R W), bf16 W with d_model = 576
(CUDA-core S = R W) and fp32 W.  The first case is also checked against the
oracle's dW from the same seeded activations.  This file is collected last so
that a run stopping at its first failure has already run every other test."""
import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from oracle import ispa_oracle as orc
from helpers import DW_REL_BF16, DW_REL_F32, fro_rel

pytestmark = pytest.mark.gpu


def _inputs(D, n, seed, w_dtype):
    """Seeded activations (bf16 values) and W; G, R formed on the host in fp64
    and handed to both solves as fp32."""
    g = np.random.default_rng(seed)
    A = synth.round_bf16((g.standard_normal((n, D)) * 0.2).astype(np.float32)).astype(np.float64)
    Dl = synth.round_bf16((g.standard_normal((n, D)) * 0.05).astype(np.float32)).astype(np.float64)
    W = (g.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32)
    if w_dtype == "bf16":
        W = synth.round_bf16(W)
    G, R = orc.gram(A, Dl)
    Wd = torch.from_numpy(W).cuda()
    Wd = Wd.to(torch.bfloat16) if w_dtype == "bf16" else Wd
    return (torch.from_numpy(G.astype(np.float32)).cuda(), torch.from_numpy(R.astype(np.float32)).cuda(), Wd,
            (G, R, W.astype(np.float64)))


def _noalloc(G, R, W):
    D = G.shape[0]
    dW = torch.empty(D, D, device="cuda")
    Wn = torch.empty_like(W)
    status = ispa.new_status()
    dt = ispa.DT_BF16 if W.dtype == torch.bfloat16 else ispa.DT_F32
    ispa.ispa_absorb_solve_noalloc(G.data_ptr(), R.data_ptr(), W.data_ptr(), dt, D, 0.0, 1e-2,
                                   dW.data_ptr(), Wn.data_ptr(), status.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "ispa_absorb_solve_noalloc")
    return dW, Wn


# (d_model, rows, seed, W dtype): largest first, so that the later, smaller
# calls run over a larger call's leftovers
CASES = [(1536, 4680, 1, "bf16"), (576, 2000, 3, "bf16"), (512, 2000, 2, "bf16"), (128, 600, 4, "f32")]


def test_noalloc_solve_matches_workspace_solve_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    ispa_build.build()
    for D, n, seed, wdt in CASES:
        G, R, W, (Gh, Rh, Wh) = _inputs(D, n, seed, wdt)
        tol = DW_REL_BF16 if wdt == "bf16" else DW_REL_F32
        ref_dW, ref_Wn = ispa.absorb_solve(G, R, W, lambda_rel=1e-2)
        torch.cuda.synchronize()
        ref = ref_dW.cpu().numpy().astype(np.float64)
        for _ in range(2):
            dW, Wn = _noalloc(G, R, W)
            assert fro_rel(dW.cpu().numpy().astype(np.float64), ref) <= tol, (D, wdt)
            assert fro_rel(Wn.float().cpu().numpy(), ref_Wn.float().cpu().numpy()) <= tol, (D, wdt)
        if D == 1536:
            # independent of the library's own solve: the oracle's dW from the same statistics
            dW_o = orc.absorb(Gh, Rh, Wh, orc.ridge_lambda(Gh))
            assert fro_rel(dW.cpu().numpy().astype(np.float64), dW_o) <= DW_REL_BF16


def test_noalloc_rejects_sizes_beyond_its_scratch():
    ispa_build.build()
    p = torch.empty(16, device="cuda") if torch.cuda.is_available() else None
    ptr = p.data_ptr() if p is not None else 256
    with pytest.raises(ispa.IspaError) as e:
        ispa.ispa_absorb_solve_noalloc(ptr, ptr, ptr, ispa.DT_BF16, 2112, 0.0, 1e-2, ptr, None, None, None)
    assert e.value.code == 2 and "2048" in str(e.value)
