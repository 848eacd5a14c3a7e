"""Tensor-level argument checks of the PyTorch binding.  They run before any
CUDA call, so mismatched shapes, dtypes or placements never reach a kernel
(which would read past the end of a short buffer); none of these tests needs a
GPU."""
import types

import pytest
import torch

from chunked_kl_loss_tcgen05_b200 import torch_api as ta

N, H, V, K = 6, 16, 64, 4


def _inputs(**over):
    t = dict(hidden=torch.zeros(N, H, dtype=torch.bfloat16),
             W=torch.zeros(V, H, dtype=torch.bfloat16),
             topk_idx=torch.zeros(N, K, dtype=torch.int32),
             topk_logit=torch.zeros(N, K, dtype=torch.float32),
             row_mask=torch.ones(N, dtype=torch.uint8))
    t.update(over)
    return t


def _call(fn, t, **kw):
    return fn(t["hidden"], t["W"], t["topk_idx"], t["topk_logit"], t["row_mask"], **kw)


@pytest.mark.parametrize("over,exc", [
    (dict(W=torch.zeros(V, H + 8, dtype=torch.bfloat16)), ValueError),    # H differs
    (dict(hidden=torch.zeros(N * H, dtype=torch.bfloat16)), ValueError),  # not 2-D
    (dict(topk_logit=torch.zeros(N - 1, K)), ValueError),                 # fewer rows
    (dict(topk_logit=torch.zeros(N, K + 1)), ValueError),                 # K differs
    (dict(topk_idx=torch.zeros(N + 1, K, dtype=torch.int32),
          topk_logit=torch.zeros(N + 1, K)), ValueError),                 # N differs
    (dict(topk_idx=torch.zeros(N, K, dtype=torch.int64)), TypeError),
    (dict(topk_logit=torch.zeros(N, K, dtype=torch.float64)), TypeError),
    (dict(row_mask=torch.ones(N + 1, dtype=torch.uint8)), TypeError),
    (dict(row_mask=torch.ones(N, dtype=torch.bool)), TypeError),
    (dict(W=torch.zeros(V, H, dtype=torch.float32)), TypeError),          # not bf16
])
@pytest.mark.parametrize("fn", [ta.fused_kl_fwd_bwd, ta.fused_kl_fwd, ta.fused_kl_fwd_bwd_sliced])
def test_shape_and_dtype_mismatches_rejected(fn, over, exc):
    with pytest.raises(exc):
        _call(fn, _inputs(**over))


@pytest.mark.parametrize("fn", [ta.fused_kl_fwd_bwd, ta.fused_kl_fwd, ta.fused_kl_fwd_bwd_sliced])
def test_host_tensors_rejected_by_device_entry_points(fn):
    with pytest.raises(ValueError, match="CUDA"):
        _call(fn, _inputs())


def test_non_contiguous_rejected():
    t = _inputs(hidden=torch.zeros(H, N, dtype=torch.bfloat16).t())
    with pytest.raises(ValueError, match="contiguous"):
        _call(ta.fused_kl_fwd_bwd, t)


def test_host_input_entry_point_checks_shapes_then_placement():
    t = _inputs(topk_logit=torch.zeros(N - 1, K))
    with pytest.raises(ValueError):
        _call(ta.fused_kl_fwd_bwd_host, t)
    with pytest.raises(ValueError, match="W must be a contiguous CUDA tensor"):
        _call(ta.fused_kl_fwd_bwd_host, _inputs())   # inputs on the host, W too


def test_row_list_and_selection_checks():
    t = _inputs()
    with pytest.raises(TypeError, match="rows"):
        ta.fused_kl_rows(t["hidden"], t["W"], t["topk_idx"], t["topk_logit"],
                         torch.zeros(3, dtype=torch.int64))
    with pytest.raises(TypeError, match="score"):
        ta.select_top_rows(torch.zeros(N, dtype=torch.float64), 2)
    with pytest.raises(TypeError, match="row_mask"):
        ta.select_top_rows(torch.zeros(N), 2, torch.ones(N + 1, dtype=torch.uint8))
    with pytest.raises(TypeError, match="row_mask"):
        ta.student_entropy(t["hidden"], t["W"], torch.ones(N - 1, dtype=torch.uint8))


class _Fake:
    """Stand-in for a tensor on a given device (only what the checks read)."""

    def __init__(self, device, contiguous=True):
        self.is_cuda = device.startswith("cuda")
        self.device = torch.device(device)
        self._c = contiguous

    def is_contiguous(self):
        return self._c


def test_tensors_on_two_devices_rejected():
    with pytest.raises(ValueError, match="one device"):
        ta._check_placement(True, (("hidden", _Fake("cuda:0")), ("W", _Fake("cuda:1"))))
    ta._check_placement(True, (("hidden", _Fake("cuda:1")), ("W", _Fake("cuda:1")),
                               ("row_mask", None)))


def test_output_and_workspace_checks():
    prob = types.SimpleNamespace(N=N, H=H, V=V)
    cpu = torch.device("cpu")
    good = (torch.zeros(1), torch.zeros(N, H), torch.zeros(V, H))
    ta._check_out(good, prob, cpu)
    ta._check_out(good[1:], prob, cpu, with_loss=False)
    for bad in [(torch.zeros(0), good[1], good[2]),
                (good[0], torch.zeros(N + 1, H), good[2]),
                (good[0], good[1], torch.zeros(V, H, dtype=torch.float64)),
                (good[0], good[1], torch.zeros(H, V).t()),
                good[1:]]:
        with pytest.raises(ValueError):
            ta._check_out(bad, prob, cpu)
    ws = torch.zeros(256, dtype=torch.uint8)
    assert ta._workspace(ws, prob, cpu) is ws
    with pytest.raises(ValueError, match="workspace"):
        ta._workspace(torch.zeros(256, dtype=torch.int8), prob, cpu)
    with pytest.raises(ValueError, match="workspace"):
        ta._workspace(ws, prob, torch.device("cuda:0"))
