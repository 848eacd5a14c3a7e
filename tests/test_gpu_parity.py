"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances (stated for the method): loss within 1e-3 relative error; dH and dW
within 2e-2 relative Frobenius error (bf16 inputs, fp32 accumulation).  The
expected error is far smaller: logits are bf16 x bf16 products accumulated in
fp32 (~1e-6 relative), and the gradients carry one bf16 rounding of dlogits
(~2^-9 relative per element, averaging out in the products).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from chunked_kl_loss_tcgen05_b200 import FcklProblem, fckl_check, fckl_fwd_bwd, FCKL_OK
from chunked_kl_loss_tcgen05_b200 import FCKL_ERR_BAD_INDEX, FCKL_ERR_BAD_TEACHER
from chunked_kl_loss_tcgen05_b200.torch_api import (alloc_workspace, arrays_to_device,
                                                    fused_kl_fwd, fused_kl_fwd_bwd)

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
GRAD_RTOL = 2e-2


def rel_fro(a, b):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


def run_gpu(inp, chunk=None, T=None, fwd_only=False, row_loss=True, dw_rows=0):
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    T = inp.cfg.T if T is None else T
    chunk = inp.cfg.chunk if chunk is None else chunk
    if fwd_only:
        loss, rl = fused_kl_fwd(*d, T=T, chunk=chunk, want_row_loss=row_loss)
        torch.cuda.synchronize()
        return dict(loss=loss.item(), row_loss=rl.cpu().numpy())
    loss, rl, dH, dW = fused_kl_fwd_bwd(*d, T=T, chunk=chunk, want_row_loss=row_loss,
                                        dw_rows=dw_rows)
    torch.cuda.synchronize()
    return dict(loss=loss.item(), row_loss=rl.cpu().numpy(), dH=dH, dW=dW)


def check_full(inp, g, o):
    m = inp.row_mask != 0
    assert abs(g["loss"] - o["loss"]) <= LOSS_RTOL * abs(o["loss"]), (g["loss"], o["loss"])
    np.testing.assert_allclose(g["row_loss"][m], o["row_loss"][m], rtol=LOSS_RTOL, atol=1e-4)
    assert (g["row_loss"][~m] == 0).all()
    eh = rel_fro(g["dH"].cpu().numpy(), o["dH"])
    ew = rel_fro(g["dW"].cpu().numpy(), o["dW"])
    assert eh <= GRAD_RTOL and ew <= GRAD_RTOL, (eh, ew)
    return eh, ew


def test_tiny_config_full():
    inp = synth.make_inputs(0)
    o = oracle.oracle_from_inputs(inp)
    g = run_gpu(inp)
    eh, ew = check_full(inp, g, o)
    assert eh < 5e-3 and ew < 5e-3, (eh, ew)   # far inside the stated bound


@pytest.mark.parametrize("chunk,dw_rows", [(64, 0), (100, 0), (128, 0), (256, 0), (0, 0),
                                           (64, 256), (100, 200), (37, 4096)])
def test_tiny_config_chunk_invariance(chunk, dw_rows):
    """Chunking rows differently, and grouping chunks into one dW GEMM, gives
    the same loss and gradients."""
    inp = synth.make_inputs(0)
    ref = run_gpu(inp, chunk=256)
    g = run_gpu(inp, chunk=chunk, dw_rows=dw_rows)
    assert abs(g["loss"] - ref["loss"]) <= 1e-5 * abs(ref["loss"])
    np.testing.assert_allclose(g["row_loss"], ref["row_loss"], rtol=1e-5, atol=1e-6)
    assert rel_fro(g["dH"].cpu().numpy(), ref["dH"].cpu().numpy()) < 1e-5
    assert rel_fro(g["dW"].cpu().numpy(), ref["dW"].cpu().numpy()) < 1e-5


EDGE = [
    # name, N, H, V, K, T, mask_frac, chunk
    ("ragged_rows", 333, 128, 2048, 16, 1.0, 0.1, 128),
    ("vocab_tail", 200, 128, 1000, 8, 1.0, 0.0, 0),
    ("vocab_not_mult8", 130, 64, 1003, 5, 0.7, 0.0, 64),
    ("hidden_tail", 150, 200, 777, 12, 1.3, 0.2, 96),
    ("hidden_small", 64, 8, 300, 4, 1.0, 0.0, 0),
    ("k_one", 256, 256, 4096, 1, 1.0, 0.0, 0),
    ("k_max", 129, 64, 600, 256, 2.0, 0.0, 0),
    ("temperature_2", 256, 256, 4096, 16, 2.0, 0.25, 64),
    ("one_row", 1, 64, 512, 3, 1.0, 0.0, 0),
    ("many_chunks", 1000, 64, 513, 7, 1.0, 0.05, 37),
    ("k_equals_v", 64, 64, 200, 200, 1.0, 0.0, 0),       # the teacher covers the vocabulary
    ("temperature_small", 256, 128, 3000, 16, 0.25, 0.1, 0),
    ("temperature_large", 256, 128, 3000, 16, 8.0, 0.1, 0),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_shapes(case):
    name, N, H, V, K, T, mf, chunk = case
    seed = 100 + [c[0] for c in EDGE].index(name)
    inp = synth.make_custom(N, H, V, K, T=T, sigma=2.0, mask_frac=mf, seed=seed, chunk=chunk)
    o = oracle.oracle_from_inputs(inp)
    g = run_gpu(inp)
    check_full(inp, g, o)


def test_forward_only_matches():
    inp = synth.make_inputs(0)
    a = run_gpu(inp, fwd_only=True)
    b = run_gpu(inp)
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-6)
    np.testing.assert_allclose(a["row_loss"], b["row_loss"], rtol=1e-6, atol=1e-7)


def test_no_valid_rows():
    inp = synth.make_custom(100, 64, 512, 8, mask_frac=1.0, seed=3)
    g = run_gpu(inp)
    assert g["loss"] == 0.0
    assert not g["dH"].any().item() and not g["dW"].any().item()


def test_masked_rows_do_not_matter():
    inp = synth.make_custom(300, 128, 2000, 10, mask_frac=0.3, seed=4, chunk=128)
    g1 = run_gpu(inp)
    m = inp.row_mask == 0
    rng = np.random.default_rng(0)
    inp.hidden[m] = synth.f32_to_bf16_bits(rng.standard_normal((m.sum(), 128)).astype(np.float32) * 5)
    inp.topk_logit[m] = rng.standard_normal((m.sum(), 10)).astype(np.float32) * 7
    g2 = run_gpu(inp)
    assert g1["loss"] == g2["loss"]
    assert rel_fro(g2["dW"].cpu().numpy(), g1["dW"].cpu().numpy()) < 1e-6
    assert g2["dH"][torch.from_numpy(m).cuda()].abs().max().item() == 0.0


def _with_valid_count(inp, n_valid, seed):
    rng = np.random.default_rng(seed)
    m = np.zeros(inp.cfg.N, np.uint8)
    m[rng.choice(inp.cfg.N, size=n_valid, replace=False)] = 1
    inp.row_mask[:] = m
    return inp


@pytest.mark.parametrize("n_valid", [1, 63, 100, 150, 190, 299])
@pytest.mark.parametrize("fill", [0x00, 0xFF])
@pytest.mark.parametrize("dw_rows", [0, 300])
def test_compacted_rows_against_oracle(n_valid, fill, dw_rows):
    """Masked calls compact their valid rows on the device.  Chunk 100 (not a
    multiple of 64), alone or with three chunks per dW group (dw_rows = 300,
    which puts the partial 64-row block of the dW reduction across chunk slots
    for some counts); a workspace filled with 0xFF bytes (NaN in bf16 and fp32)
    shows that no stale value leaks in."""
    inp = _with_valid_count(synth.make_custom(300, 64, 700, 9, T=1.2, sigma=2.0, seed=21,
                                              chunk=100), n_valid, n_valid)
    o = oracle.oracle_from_inputs(inp)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    prob = FcklProblem(300, 64, 700, 9, 1.2, 100, dw_rows=dw_rows)
    ws = alloc_workspace(prob, d[0].device)
    ws.fill_(fill)
    loss, rl, dH, dW = fused_kl_fwd_bwd(*d, T=1.2, chunk=100, workspace=ws, want_row_loss=True,
                                        dw_rows=dw_rows)
    torch.cuda.synchronize()
    check_full(inp, dict(loss=loss.item(), row_loss=rl.cpu().numpy(), dH=dH, dW=dW), o)
    ws.fill_(fill)
    lf, rlf = fused_kl_fwd(*d, T=1.2, chunk=100, workspace=ws, want_row_loss=True)
    torch.cuda.synchronize()
    assert lf.item() == pytest.approx(loss.item(), rel=1e-6)
    np.testing.assert_allclose(rlf.cpu().numpy(), rl.cpu().numpy(), rtol=1e-6, atol=1e-7)


def test_llama_8k_config_full():
    inp = synth.make_inputs(1)
    g = run_gpu(inp)
    o = oracle.oracle_from_inputs(inp)
    check_full(inp, g, o)


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_large_config_sampled_rows(cfg):
    """Full-size configs.  The whole-batch call: per-row loss and dH on 64
    seeded valid rows against the oracle; the mean of the row losses, the zero
    column sums of dW and the zero dH of masked rows at full size.  Then the
    same 64 rows through the listed-row entry point, whose loss, dH rows and
    full [V, H] dW (the 64 rows' contribution, N_v = 64) the oracle gives
    exactly: at the workload's own chunk (one 64-row chunk) and in 16-row
    chunks grouped four to a dW GEMM (dw_rows = 64), so the full-width dW
    GEMM, the gpt-oss H = 2880 narrow last tile, T = 2 and a grouped dW
    reduction are all compared with the oracle at the real H and V."""
    inp = synth.make_inputs(cfg)
    rows = synth.sample_rows(inp, 64)
    g = run_gpu(inp)
    o = oracle.oracle_from_inputs(inp, rows=rows)
    np.testing.assert_array_equal(o["rows"], rows)
    np.testing.assert_allclose(g["row_loss"][rows], o["row_loss_rows"], rtol=LOSS_RTOL, atol=1e-4)
    dH_rows = g["dH"][torch.from_numpy(rows).cuda()].cpu().numpy()
    assert rel_fro(dH_rows, o["dH_rows"]) <= GRAD_RTOL
    m = inp.row_mask != 0
    mean = g["row_loss"][m].astype(np.float64).mean()
    assert abs(g["loss"] - mean) <= 1e-5 * abs(mean)
    if (~m).any():
        assert g["dH"][torch.from_numpy(~m).cuda()].abs().max().item() == 0.0
    dW = g["dW"]
    colsum = dW.double().sum(dim=0)
    scale = dW.double().abs().sum(dim=0)
    assert (colsum.abs() <= 2e-2 * scale + 1e-30).all().item()
    del g, dW
    torch.cuda.empty_cache()

    # listed rows: exact oracle targets for loss, dH and dW (N_v = 64)
    from chunked_kl_loss_tcgen05_b200.torch_api import fused_kl_rows
    o = oracle.fused_chunked_kl(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, None,
                                inp.cfg.T, rows=rows, n_valid=rows.size)
    o_loss = o["row_loss_rows"].sum() / rows.size
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, None)
    rows_d = torch.from_numpy(rows.astype(np.int32)).cuda()
    for chunk, dw_rows in ((inp.cfg.chunk, 0), (16, 64)):
        loss, rl, dH, dW = fused_kl_rows(d[0], d[1], d[2], d[3], rows_d, T=inp.cfg.T,
                                         chunk=chunk, dw_rows=dw_rows, want_row_loss=True)
        torch.cuda.synchronize()
        assert abs(loss.item() - o_loss) <= LOSS_RTOL * abs(o_loss), (chunk, loss.item(), o_loss)
        np.testing.assert_allclose(rl[rows_d].cpu().numpy(), o["row_loss_rows"], rtol=LOSS_RTOL,
                                   atol=1e-4)
        eh = rel_fro(dH[rows_d].cpu().numpy(), o["dH_rows"])
        ew = rel_fro(dW.cpu().numpy(), o["dW"])
        assert eh <= GRAD_RTOL and ew <= GRAD_RTOL, (chunk, eh, ew)
        del loss, rl, dH, dW
        torch.cuda.empty_cache()


def _raw_call(inp, ids=None, logits=None):
    d = list(arrays_to_device(inp.hidden, inp.W, inp.topk_idx if ids is None else ids,
                              inp.topk_logit if logits is None else logits, inp.row_mask))
    p = FcklProblem(inp.cfg.N, inp.cfg.H, inp.cfg.V, inp.cfg.K, inp.cfg.T, inp.cfg.chunk)
    ws = alloc_workspace(p, "cuda")
    loss = torch.empty(1, device="cuda")
    dH = torch.empty(inp.cfg.N, inp.cfg.H, device="cuda")
    dW = torch.empty(inp.cfg.V, inp.cfg.H, device="cuda")
    st = fckl_fwd_bwd(p, d[0].data_ptr(), d[1].data_ptr(), d[2].data_ptr(), d[3].data_ptr(),
                      None if d[4] is None else d[4].data_ptr(), loss.data_ptr(), None,
                      dH.data_ptr(), dW.data_ptr(), ws.data_ptr(), ws.numel(),
                      torch.cuda.current_stream().cuda_stream)
    assert st == FCKL_OK
    return fckl_check(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_out_of_range_id_is_reported():
    inp = synth.make_custom(64, 64, 512, 8, seed=5)
    assert _raw_call(inp) == FCKL_OK
    ids = inp.topk_idx.copy()
    ids[17, 3] = 512
    assert _raw_call(inp, ids=ids) == FCKL_ERR_BAD_INDEX
    ids = inp.topk_idx.copy()
    ids[5, 0] = -1
    assert _raw_call(inp, ids=ids) == FCKL_ERR_BAD_INDEX


def test_teacher_row_without_finite_logit_is_reported():
    inp = synth.make_custom(64, 64, 512, 8, seed=6)
    lg = inp.topk_logit.copy()
    lg[9, :] = -np.inf
    assert _raw_call(inp, logits=lg) == FCKL_ERR_BAD_TEACHER
    lg = inp.topk_logit.copy()
    lg[3, 2] = np.nan
    assert _raw_call(inp, logits=lg) == FCKL_ERR_BAD_TEACHER


def test_partly_minus_inf_teacher_logits():
    """-inf teacher logits are entries of probability 0 (a padded cache); rows
    keep at least one finite logit."""
    inp = synth.make_custom(300, 128, 2000, 16, T=1.0, sigma=2.0, mask_frac=0.1, seed=93,
                            chunk=128)
    rng = np.random.default_rng(93)
    pad = rng.random(inp.topk_logit.shape) < 0.3
    pad[:, 0] = False
    inp.topk_logit[pad] = -np.inf
    o = oracle.oracle_from_inputs(inp)
    check_full(inp, run_gpu(inp), o)


def test_masked_rows_with_invalid_teacher_data_are_ignored():
    """A masked row takes no part in the loss: its ids and logits are not even
    checked (the same call with clean masked rows gives the same result)."""
    inp = synth.make_custom(200, 64, 700, 8, mask_frac=0.3, seed=94, chunk=64)
    ref = run_gpu(inp)
    m = inp.row_mask == 0
    inp.topk_idx[m] = 700 + 5
    inp.topk_idx[np.nonzero(m)[0][:3]] = -3
    inp.topk_logit[m] = np.nan
    assert _raw_call(inp) == FCKL_OK
    g = run_gpu(inp)
    assert g["loss"] == ref["loss"]
    assert torch.equal(g["dW"], ref["dW"])


# ------------------------------------------------ sampled sparse targets (RS-KD)
@pytest.mark.parametrize("shape", [(300, 128, 2000, 24, 1.0, 128), (517, 64, 777, 64, 2.0, 0),
                                   (256, 256, 4096, 100, 1.0, 64),
                                   (1024, 3072, 128256, 100, 1.0, 0)])  # 8K Llama H, V, K
def test_sampled_target_teacher_full(shape):
    """Teacher given as sampled class weights (repeats allowed): p = w / sum w."""
    N, H, V, K, T, chunk = shape
    inp = synth.make_sampled_targets(N, H, V, K, T=T, mask_frac=0.1, seed=61 + N, chunk=chunk)
    s = np.sort(inp.topk_idx, axis=1)
    assert (s[:, 1:] == s[:, :-1]).any()          # the draws do repeat ids
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    loss, rl, dH, dW = fused_kl_fwd_bwd(*d, T=T, chunk=chunk, want_row_loss=True, teacher=1)
    torch.cuda.synchronize()
    o = oracle.oracle_from_inputs(inp, teacher="probs")
    check_full(inp, dict(loss=loss.item(), row_loss=rl.cpu().numpy(), dH=dH, dW=dW), o)


def test_repeated_ids_in_logit_cache():
    """Repeated ids in a top-K logit cache add into one teacher class."""
    inp = synth.make_custom(300, 128, 2000, 10, mask_frac=0.1, seed=71, chunk=128)
    inp.topk_idx[::3, 4] = inp.topk_idx[::3, 1]
    inp.topk_idx[::5, 9] = inp.topk_idx[::5, 2]
    o = oracle.oracle_from_inputs(inp)
    check_full(inp, run_gpu(inp), o)


def test_bad_sampled_weights_are_reported():
    inp = synth.make_sampled_targets(64, 64, 512, 8, seed=72)
    d = list(arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, None))
    from chunked_kl_loss_tcgen05_b200 import FcklError
    for bad in (-0.5, float("nan"), float("inf")):
        lg = inp.topk_logit.copy()
        lg[7, 3] = bad
        d[3] = torch.from_numpy(lg).cuda()
        with pytest.raises(FcklError) as ei:
            fused_kl_fwd_bwd(*d, teacher=1)
        assert ei.value.status == FCKL_ERR_BAD_TEACHER
    lg = inp.topk_logit.copy()
    lg[5, :] = 0.0                                 # a row with no mass
    d[3] = torch.from_numpy(lg).cuda()
    with pytest.raises(FcklError) as ei:
        fused_kl_fwd_bwd(*d, teacher=1)
    assert ei.value.status == FCKL_ERR_BAD_TEACHER


def test_global_valid_count_scales_loss_and_grads():
    """n_valid_total (the N_v of all data-parallel shards) replaces the local
    count in the mean and the gradient scale: doubling it halves everything."""
    inp = synth.make_custom(300, 128, 2000, 10, mask_frac=0.1, seed=81, chunk=128)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    l1, _, dH1, dW1 = fused_kl_fwd_bwd(*d, chunk=128)
    nv = int((inp.row_mask != 0).sum())
    l2, _, dH2, dW2 = fused_kl_fwd_bwd(*d, chunk=128, n_valid_total=2 * nv)
    torch.cuda.synchronize()
    assert l2.item() == pytest.approx(l1.item() / 2, rel=1e-6)
    assert rel_fro(dH2.cpu().numpy(), dH1.cpu().numpy() / 2) < 1e-6
    assert rel_fro(dW2.cpu().numpy(), dW1.cpu().numpy() / 2) < 1e-6
    o = oracle.oracle_from_inputs(inp)
    o2 = oracle.fused_chunked_kl(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask,
                                 inp.cfg.T, n_valid=2 * nv)
    assert abs(l2.item() - o2["row_loss"].sum() / (2 * nv)) <= LOSS_RTOL * abs(o["loss"] / 2)


@pytest.mark.parametrize("n_slices", [1, 3, 7, 40])
def test_sliced_dw_matches_plain_call(n_slices):
    """Splitting the last dW launch into vocabulary slices changes nothing but
    the launch pattern; the slices cover dW's rows in order and every event
    has fired once the stream is done.  V = 2000 has 8 tiles of 256, so 40
    slices leave 32 empty ones."""
    from chunked_kl_loss_tcgen05_b200.torch_api import fused_kl_fwd_bwd_sliced
    inp = synth.make_custom(600, 128, 2000, 10, mask_frac=0.1, seed=83, chunk=128)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    l1, _, dH1, dW1 = fused_kl_fwd_bwd(*d, chunk=128)
    l2, dH2, dW2, slices = fused_kl_fwd_bwd_sliced(*d, chunk=128, n_slices=n_slices)
    torch.cuda.synchronize()
    assert l2.item() == l1.item()
    assert torch.equal(dW2, dW1)
    assert rel_fro(dH2.cpu().numpy(), dH1.cpu().numpy()) < 1e-6
    bounds = [0] + [r1 for _, r1, _ in slices]
    assert [r0 for r0, _, _ in slices] == bounds[:-1] and bounds[-1] == 2000
    assert all(r0 % 256 == 0 for r0, r1, _ in slices if r1 > r0)
    assert sum(r1 > r0 for r0, r1, _ in slices) == min(n_slices, 8)
    assert all(ev.query() for _, _, ev in slices)


def test_dp_wrapper_single_rank_nccl():
    """The data-parallel wrapper on one NCCL rank (valid-count all-reduce, the
    last dW GEMM in vocabulary slices all-reduced as they finish, loss
    all-reduce) against the oracle and the plain call."""
    import torch.distributed as dist
    from chunked_kl_loss_tcgen05_b200.dp import fused_kl_fwd_bwd_dp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        inp = synth.make_custom(300, 128, 2000, 10, mask_frac=0.1, seed=82, chunk=128)
        d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
        l1, _, dH1, dW1 = fused_kl_fwd_bwd(*d, chunk=128)
        l2, dH2, dW2 = fused_kl_fwd_bwd_dp(*d, chunk=128, n_slices=5)
        torch.cuda.synchronize()
        assert l2.item() == pytest.approx(l1.item(), rel=1e-6)
        assert rel_fro(dW2.cpu().numpy(), dW1.cpu().numpy()) < 1e-6
        assert rel_fro(dH2.cpu().numpy(), dH1.cpu().numpy()) < 1e-6
        o = oracle.oracle_from_inputs(inp)
        check_full(inp, dict(loss=l2.item(), row_loss=o["row_loss"], dH=dH2, dW=dW2), o)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_shards", [2, 3])
def test_row_shards_with_global_count_match_oracle(n_shards):
    """The arithmetic of row-sharded data parallelism on one GPU: each shard of
    rows runs the sliced fused call with n_valid_total = the valid rows of ALL
    shards (about n_shards times its own count); the shards' losses and dW
    partials summed, and their dH rows side by side, equal the oracle on the
    whole batch (what the all-reduces of the multi-GPU wrapper produce)."""
    from chunked_kl_loss_tcgen05_b200.dp import shard_rows
    from chunked_kl_loss_tcgen05_b200.torch_api import fused_kl_fwd_bwd_sliced
    inp = synth.make_custom(700, 192, 3000, 12, T=1.3, mask_frac=0.15, seed=84, chunk=128)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    n_total = int((inp.row_mask != 0).sum())
    loss = 0.0
    dW = torch.zeros(inp.cfg.V, inp.cfg.H, device="cuda", dtype=torch.float64)
    dH = torch.empty(inp.cfg.N, inp.cfg.H, device="cuda")
    for r in range(n_shards):
        lo, hi = shard_rows(inp.cfg.N, r, n_shards)
        l, dHs, dWs, slices = fused_kl_fwd_bwd_sliced(
            d[0][lo:hi], d[1], d[2][lo:hi], d[3][lo:hi], d[4][lo:hi], T=1.3, chunk=128,
            n_slices=4, n_valid_total=n_total)
        torch.cuda.synchronize()
        assert all(ev.query() for _, _, ev in slices)
        loss += l.item()
        dW += dWs.double()
        dH[lo:hi] = dHs
    o = oracle.oracle_from_inputs(inp)
    assert abs(loss - o["loss"]) <= LOSS_RTOL * abs(o["loss"]), (loss, o["loss"])
    eh = rel_fro(dH.cpu().numpy(), o["dH"])
    ew = rel_fro(dW.cpu().numpy(), o["dW"])
    assert eh <= GRAD_RTOL and ew <= GRAD_RTOL, (eh, ew)
    assert eh < 5e-3 and ew < 5e-3, (eh, ew)   # far inside the stated bound


def test_autograd_wrapper_gradients():
    """loss = fused_chunked_kl_loss(...); (3 * loss).backward() gives hidden.grad
    and W.grad = 3 * (dH, dW) of the fused call, in the inputs' dtype, and the
    gradients match the oracle."""
    from chunked_kl_loss_tcgen05_b200.torch_api import fused_chunked_kl_loss
    inp = synth.make_custom(300, 128, 2000, 10, T=1.5, mask_frac=0.2, seed=91, chunk=128)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    h = d[0].view(torch.bfloat16).clone().requires_grad_(True)
    W = d[1].view(torch.bfloat16).clone().requires_grad_(True)
    loss = fused_chunked_kl_loss(h, W, d[2], d[3], d[4], T=1.5, chunk=128)
    (3.0 * loss).backward()
    l0, _, dH, dW = fused_kl_fwd_bwd(*d, T=1.5, chunk=128)
    assert loss.item() == l0.item()
    assert h.grad.dtype == torch.bfloat16 and W.grad.dtype == torch.bfloat16
    # dH's split-K reduce-adds land in any order: compare up to bf16 rounding
    ref = (3.0 * dH).to(torch.bfloat16).float()
    assert rel_fro(h.grad.float().cpu().numpy(), ref.cpu().numpy()) < 1e-2 * 2 ** -6
    assert torch.equal(W.grad, (3.0 * dW).to(torch.bfloat16))
    o = oracle.oracle_from_inputs(inp)
    assert rel_fro(h.grad.float().cpu().numpy(), 3.0 * o["dH"]) < GRAD_RTOL
    assert rel_fro(W.grad.float().cpu().numpy(), 3.0 * o["dW"]) < GRAD_RTOL


@pytest.mark.parametrize("env", [{"FCKL_NO_PDL": "1"}, {"FCKL_ONE_STREAM": "1"},
                                 {"FCKL_NO_PDL": "1", "FCKL_ONE_STREAM": "1"}])
def test_launch_modes_agree(env, monkeypatch):
    """Programmatic dependent launch and the second stream for the next chunk's
    gather and teacher prep change only when kernels start: the results equal
    those of plain stream order (dH up to the order of its fp32 split-K
    reduce-adds) for a masked call of many chunks, grouped and ungrouped."""
    inp = synth.make_custom(1500, 192, 3000, 12, T=1.3, sigma=2.0, mask_frac=0.2, seed=95,
                            chunk=128)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    for dw_rows in (0, 384):
        ref = fused_kl_fwd_bwd(*d, chunk=128, T=1.3, dw_rows=dw_rows, want_row_loss=True)
        torch.cuda.synchronize()
        with monkeypatch.context() as m:
            for k, v in env.items():
                m.setenv(k, v)
            g = fused_kl_fwd_bwd(*d, chunk=128, T=1.3, dw_rows=dw_rows, want_row_loss=True)
            torch.cuda.synchronize()
        assert g[0].item() == ref[0].item()
        assert torch.equal(g[1], ref[1])
        assert rel_fro(g[2].cpu().numpy(), ref[2].cpu().numpy()) < 1e-6
        assert torch.equal(g[3], ref[3])
