"""The host-input entry point (inputs streamed to the device chunk by chunk,
overlapped with the kernels) gives the results of the device-input entry point
on the same data."""
import numpy as np
import pytest
import torch

import synth
from chunked_kl_loss_tcgen05_b200.torch_api import (alloc_host_workspace, arrays_to_device,
                                                    fused_kl_fwd_bwd, fused_kl_fwd_bwd_host)

pytestmark = pytest.mark.gpu


def _host(inp, pinned):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    h = {"hidden": t(inp.hidden.view(np.int16)).view(torch.bfloat16), "topk_idx": t(inp.topk_idx),
         "topk_logit": t(inp.topk_logit), "row_mask": t(inp.row_mask)}
    return {k: (v.pin_memory() if pinned else v) for k, v in h.items()}


def _compare(inp, pinned, masked=True):
    cfg = inp.cfg
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit,
                         inp.row_mask if masked else None)
    ref_loss, _, ref_dH, ref_dW = fused_kl_fwd_bwd(*d, T=cfg.T, chunk=cfg.chunk)
    h = _host(inp, pinned)
    loss, dH, dW = fused_kl_fwd_bwd_host(h["hidden"], d[1], h["topk_idx"], h["topk_logit"],
                                         h["row_mask"] if masked else None, T=cfg.T,
                                         chunk=cfg.chunk)
    assert loss == ref_loss.item()
    assert torch.equal(dW, ref_dW)
    err = ((dH - ref_dH).norm() / ref_dH.norm().clamp_min(1e-30)).item()
    assert err < 1e-6, err  # dH's split-K reduce-adds land in any order


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("n_valid", [0, 37, 190, 300])
def test_masked_small(pinned, n_valid):
    inp = synth.make_custom(300, 64, 700, 9, T=1.2, sigma=2.0, seed=41, chunk=100)
    m = np.zeros(300, np.uint8)
    m[np.random.default_rng(n_valid).choice(300, size=n_valid, replace=False)] = 1
    inp.row_mask[:] = m
    _compare(inp, pinned)


@pytest.mark.parametrize("pinned", [True, False])
def test_unmasked_tiny_config(pinned):
    _compare(synth.make_inputs(0), pinned, masked=False)


def test_llama_8k_config():
    _compare(synth.make_inputs(1), pinned=True)


def test_back_to_back_calls_share_the_workspace():
    """Two calls enqueued without a host sync in between: the second call's
    copies must wait until the first call's kernels are done with the device
    copies of its inputs."""
    a = synth.make_custom(512, 128, 3000, 16, T=1.0, sigma=2.0, mask_frac=0.2, seed=5, chunk=128)
    b = synth.make_custom(512, 128, 3000, 16, T=1.0, sigma=2.0, mask_frac=0.1, seed=6, chunk=128)
    b.W[:] = a.W
    W = arrays_to_device(a.hidden, a.W, a.topk_idx, a.topk_logit, a.row_mask)[1]
    from chunked_kl_loss_tcgen05_b200 import FcklProblem, fckl_fwd_bwd_host
    prob = FcklProblem(512, 128, 3000, 16, 1.0, 128)
    ws = alloc_host_workspace(prob, W.device)
    outs = []
    hosts = [_host(a, True), _host(b, True)]
    stream = torch.cuda.current_stream()
    for h in hosts:
        dH = torch.empty(512, 128, device="cuda")
        dW = torch.empty(3000, 128, device="cuda")
        loss = torch.empty(1, pin_memory=True)
        st = fckl_fwd_bwd_host(prob, h["hidden"].data_ptr(), W.data_ptr(), h["topk_idx"].data_ptr(),
                               h["topk_logit"].data_ptr(), h["row_mask"].data_ptr(),
                               loss.data_ptr(), dH.data_ptr(), dW.data_ptr(), ws.data_ptr(),
                               ws.numel(), stream.cuda_stream)
        assert st == 0
        outs.append((loss, dH, dW))
    torch.cuda.synchronize()
    for inp, (loss, dH, dW) in zip((a, b), outs):
        d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
        rl, _, rdH, rdW = fused_kl_fwd_bwd(*d, T=1.0, chunk=128)
        assert loss[0].item() == rl.item()
        assert torch.equal(dW, rdW)
