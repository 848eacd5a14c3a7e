"""fckl_fwd_noalloc: the forward loss for callers that cannot allocate device
memory (e.g. code inside a host framework whose allocator owns all device
memory).  It must agree with the workspace entry point fckl_fwd, call after
call, because every call reuses the library's one static scratch array.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import synth
from chunked_kl_loss_tcgen05_b200 import (FCKL_OK, FcklProblem, fckl_check, fckl_fwd,
                                          fckl_fwd_noalloc)
from chunked_kl_loss_tcgen05_b200.torch_api import alloc_workspace, arrays_to_device

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3


def _with_workspace(prob, d, stream):
    ws = alloc_workspace(prob, "cuda")
    loss = torch.empty(1, device="cuda")
    rl = torch.empty(prob.N, device="cuda")
    st = fckl_fwd(prob, d[0].data_ptr(), d[1].data_ptr(), d[2].data_ptr(), d[3].data_ptr(),
                  d[4].data_ptr(), loss.data_ptr(), rl.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert st == FCKL_OK
    assert fckl_check(ws.data_ptr(), stream) == FCKL_OK
    return loss.item(), rl.cpu().numpy()


@pytest.mark.parametrize("shape", [(3000, 512, 20000, 32, 0), (700, 256, 4096, 16, 256)])
def test_noalloc_forward_matches_workspace_forward(shape):
    N, H, V, K, chunk = shape
    inp = synth.make_custom(N, H, V, K, T=1.5, sigma=2.0, mask_frac=0.1, seed=2024, chunk=chunk)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    prob = FcklProblem(N, H, V, K, 1.5, chunk)
    stream = torch.cuda.current_stream().cuda_stream
    ref_loss, ref_rl = _with_workspace(prob, d, stream)
    m = inp.row_mask != 0
    for call in range(2):  # the second call runs on the scratch the first one left behind
        loss = torch.full((1,), float("nan"), device="cuda")
        rl = torch.full((N,), float("nan"), device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        st = fckl_fwd_noalloc(prob, d[0].data_ptr(), d[1].data_ptr(), d[2].data_ptr(),
                              d[3].data_ptr(), d[4].data_ptr(), loss.data_ptr(), rl.data_ptr(),
                              status.data_ptr(), stream)
        assert st == FCKL_OK, call
        torch.cuda.synchronize()
        assert status.item() == FCKL_OK, call
        assert abs(loss.item() - ref_loss) <= LOSS_RTOL * abs(ref_loss), (call, loss.item(), ref_loss)
        g = rl.cpu().numpy()
        np.testing.assert_allclose(g[m], ref_rl[m], rtol=LOSS_RTOL, atol=1e-4)
        assert (g[~m] == 0).all()
