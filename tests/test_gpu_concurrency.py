"""Calls from several host threads, each on its own stream and workspace, while
the library's second stream (the next chunk's row preparation) and its events
are shared: every call gives the result of the same call made alone."""
import threading

import pytest
import torch

import synth
from chunked_kl_loss_tcgen05_b200 import FcklProblem
from chunked_kl_loss_tcgen05_b200.torch_api import alloc_workspace, arrays_to_device, fused_kl_fwd_bwd

pytestmark = pytest.mark.gpu


def test_threads_on_their_own_streams():
    N, H, V, K, C = 900, 128, 3000, 16, 128
    cases = [synth.make_custom(N, H, V, K, T=1.2, sigma=2.0, mask_frac=m, seed=120 + i, chunk=C)
             for i, m in enumerate((0.0, 0.25, 0.5))]
    dev = [arrays_to_device(c.hidden, c.W, c.topk_idx, c.topk_logit,
                            c.row_mask if c.cfg.mask_frac else None) for c in cases]
    refs = []
    for d in dev:
        loss, _, dH, dW = fused_kl_fwd_bwd(*d, T=1.2, chunk=C)
        torch.cuda.synchronize()
        refs.append((loss.item(), dH.clone(), dW.clone()))
    results, errors = {}, []

    def worker(i):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            ws = alloc_workspace(FcklProblem(N, H, V, K, 1.2, C), "cuda")
            outs = []
            with torch.cuda.stream(s):
                for _ in range(4):
                    loss, _, dH, dW = fused_kl_fwd_bwd(*dev[i], T=1.2, chunk=C, workspace=ws,
                                                       check=False)
                    outs.append((loss, dH, dW))
            s.synchronize()
            results[i] = [(l.item(), h, w) for l, h, w in outs]
        except Exception as e:  # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    for i, (loss, dH, dW) in enumerate(refs):
        for l2, dH2, dW2 in results[i]:
            assert l2 == loss
            assert torch.equal(dW2, dW)
            assert ((dH2 - dH).norm() / dH.norm()).item() < 1e-6
