"""Row-sharded data parallelism, host logic on CPU: two or three gloo ranks each pass
their own row shard through fused_kl_fwd_bwd_dp (with the fp64 oracle as the
per-rank compute), and the all-reduced loss and dW plus the concatenated dH
shards must equal the unsharded result."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, out_q):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from chunked_kl_loss_tcgen05_b200.dp import fused_kl_fwd_bwd_dp, shard_rows

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_custom(**case)
        lo, hi = shard_rows(inp.cfg.N, rank, world)
        h = torch.from_numpy(oracle.widen_bf16(inp.hidden[lo:hi]))
        Wd = torch.from_numpy(oracle.widen_bf16(inp.W))

        def compute(hh, ww, ids, lg, mask, T, chunk, teacher, n_valid_total):
            o = oracle.fused_chunked_kl(hh.numpy(), ww.numpy(), ids.numpy(), lg.numpy(),
                                        mask.numpy(), T, n_valid=n_valid_total)
            loss = torch.tensor([o["row_loss"].sum() / n_valid_total if n_valid_total else 0.0],
                                dtype=torch.float64)
            V = ww.shape[0]
            cuts = [0, V // 3, V // 3, V]  # uneven slices, one of them empty
            slices = [(cuts[i], cuts[i + 1], None) for i in range(3)]
            return loss, torch.from_numpy(o["dH"]), torch.from_numpy(o["dW"]), slices

        loss, dH, dW = fused_kl_fwd_bwd_dp(
            h, Wd, torch.from_numpy(inp.topk_idx[lo:hi]), torch.from_numpy(inp.topk_logit[lo:hi]),
            torch.from_numpy(inp.row_mask[lo:hi]), T=inp.cfg.T, compute=compute)
        out_q.put((rank, float(loss.item()), dH.numpy(), dW.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", [dict(N=37, H=16, V=60, K=5, T=1.5, mask_frac=0.2, seed=3),
                                  dict(N=8, H=8, V=30, K=3, T=1.0, mask_frac=0.0, seed=4)])
def test_row_sharding_matches_unsharded(case, world):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, loss, dH, dW = q.get(timeout=120)
        res[rank] = (loss, dH, dW)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = oracle.oracle_from_inputs(synth.make_custom(**case))
    for r in range(world):
        np.testing.assert_allclose(res[r][0], full["loss"], rtol=1e-12)
        np.testing.assert_allclose(res[r][2], full["dW"], rtol=1e-10, atol=1e-16)
    np.testing.assert_allclose(np.concatenate([res[r][1] for r in range(world)]), full["dH"],
                               rtol=1e-10, atol=1e-16)


def _worker_leaves(rank, world, port, out_q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from chunked_kl_loss_tcgen05_b200.dp import fused_kl_fwd_bwd_dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:  # this rank leaves between steps, before its first collective
        out_q.put((rank, "left"))
        out_q.close()
        out_q.join_thread()
        os._exit(0)

    def compute(*a, **kw):
        raise AssertionError("never reached: the count all-reduce fails first")

    h = torch.zeros(4, 8)
    try:
        fused_kl_fwd_bwd_dp(h, torch.zeros(16, 8), torch.zeros(4, 2, dtype=torch.int32),
                            torch.zeros(4, 2), None, compute=compute)
        out_q.put((rank, "no error"))
    except Exception as e:  # the peer is gone: the collective must fail, not hang
        out_q.put((rank, "error: " + type(e).__name__))


def test_lost_rank_fails_the_collective_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    assert got[1] == "left"
    assert got[0].startswith("error"), got[0]
