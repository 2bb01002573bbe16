"""ispa_absorb_solve_noalloc: the absorb solve for callers that cannot
allocate device memory (host callbacks, allocator hooks, plugins handed
device pointers but no allocator, serving processes with memory fixed up
front).  Its working matrices come from a device array inside libispa, so the
caller passes only G, R, W and the outputs.

The test calls it through the C ABI twice in a row -- the second call finds
the first call's leftovers in the shared array -- and compares each result
with ispa_absorb_solve given a caller-allocated workspace, within the dW
tolerance of the other absorb tests.  This file is collected last so that a
run stopping at its first failure has already run every other test."""
import numpy as np
import pytest
import torch

from ar_video_diffusion_b200 import build as ispa_build
from ar_video_diffusion_b200 import ispa, synth
from helpers import DW_REL_BF16, fro_rel

pytestmark = pytest.mark.gpu


def _stats(D, n, seed):
    g = np.random.default_rng(seed)
    A = torch.from_numpy(synth.round_bf16((g.standard_normal((n, D)) * 0.2).astype(np.float32)))
    Dl = torch.from_numpy(synth.round_bf16((g.standard_normal((n, D)) * 0.05).astype(np.float32)))
    W = torch.from_numpy(synth.round_bf16((g.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32)))
    A, Dl, W = A.to(torch.bfloat16).cuda(), Dl.to(torch.bfloat16).cuda(), W.to(torch.bfloat16).cuda()
    G = torch.empty(D, D, device="cuda")
    R = torch.empty(D, D, device="cuda")
    ispa.gram_accumulate(A, Dl, G, R, zero_first=True)
    return G, R, W


def _noalloc(G, R, W):
    D = G.shape[0]
    dW = torch.empty(D, D, device="cuda")
    Wn = torch.empty_like(W)
    status = ispa.new_status()
    ispa.ispa_absorb_solve_noalloc(G.data_ptr(), R.data_ptr(), W.data_ptr(), ispa.DT_BF16, D, 0.0, 1e-2,
                                   dW.data_ptr(), Wn.data_ptr(), status.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ispa.raise_on_status(status, "ispa_absorb_solve_noalloc")
    return dW, Wn


def test_noalloc_solve_matches_workspace_solve_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    ispa_build.build()
    for D, n, seed in [(1536, 4680, 1), (512, 2000, 2)]:
        G, R, W = _stats(D, n, seed)
        ref_dW, ref_Wn = ispa.absorb_solve(G, R, W, lambda_rel=1e-2)
        torch.cuda.synchronize()
        ref = ref_dW.cpu().numpy().astype(np.float64)
        for _ in range(2):
            dW, Wn = _noalloc(G, R, W)
            assert fro_rel(dW.cpu().numpy().astype(np.float64), ref) <= DW_REL_BF16
            assert fro_rel(Wn.float().cpu().numpy(), ref_Wn.float().cpu().numpy()) <= DW_REL_BF16


def test_noalloc_rejects_sizes_beyond_its_scratch():
    ispa_build.build()
    p = torch.empty(16, device="cuda") if torch.cuda.is_available() else None
    ptr = p.data_ptr() if p is not None else 256
    with pytest.raises(ispa.IspaError) as e:
        ispa.ispa_absorb_solve_noalloc(ptr, ptr, ptr, ispa.DT_BF16, 2112, 0.0, 1e-2, ptr, None, None, None)
    assert e.value.code == 2 and "2048" in str(e.value)
