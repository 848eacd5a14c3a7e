"""Bounded waits: a kernel whose accumulator-ready signal is withheld gives up
after its wait budget, records FCKL_ERR_TIMEOUT and exits; the CUDA context
stays usable and the next call is correct.  The failure is injected with the
library's own knob (FCKL_DEBUG_SKIP_ARRIVE: the MMA thread omits one commit in
the first forward launch), never with a trap, an assert or a bad address."""
import os

import numpy as np
import pytest
import torch

import synth
from chunked_kl_loss_tcgen05_b200 import FCKL_ERR_TIMEOUT, FCKL_OK, FcklProblem, fckl_check, fckl_fwd
from chunked_kl_loss_tcgen05_b200.torch_api import alloc_workspace, arrays_to_device

pytestmark = pytest.mark.gpu


def _fwd(prob, d, ws, stream):
    loss = torch.empty(1, device="cuda")
    st = fckl_fwd(prob, d[0].data_ptr(), d[1].data_ptr(), d[2].data_ptr(), d[3].data_ptr(),
                  None, loss.data_ptr(), None, ws.data_ptr(), ws.numel(), stream)
    assert st == FCKL_OK
    return fckl_check(ws.data_ptr(), stream), loss.item()


def test_withheld_signal_times_out_and_context_survives():
    inp = synth.make_custom(256, 256, 4096, 16, seed=9, chunk=64)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, None)
    prob = FcklProblem(256, 256, 4096, 16, 1.0, 64)
    ws = alloc_workspace(prob, "cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st0, ref = _fwd(prob, d, ws, stream)
    assert st0 == FCKL_OK
    os.environ["FCKL_DEBUG_SKIP_ARRIVE"] = "1"
    os.environ["FCKL_WAIT_TIMEOUT_MS"] = "200"
    try:
        st1, _ = _fwd(prob, d, ws, stream)
    finally:
        del os.environ["FCKL_DEBUG_SKIP_ARRIVE"]
        del os.environ["FCKL_WAIT_TIMEOUT_MS"]
    assert st1 == FCKL_ERR_TIMEOUT
    site = ws[:256].view(torch.int32)[2].item()
    assert site == 4  # the epilogue's wait for the withheld accumulator gave up first
    st2, again = _fwd(prob, d, ws, stream)
    assert st2 == FCKL_OK
    assert np.isfinite(again) and again == ref
