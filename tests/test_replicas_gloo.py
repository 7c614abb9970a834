"""The multi-process host path on CPU: two gloo ranks exercise the helpers
that the benchmark's N-GPU run and a data-parallel trainer use (max over
ranks of a timing; global-batch load statistics summed over ranks, then the
load-balancing loss of the oracle) and must agree with one process that sees
the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_ref as R


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    rng = np.random.default_rng(11)
    T, E, k = 96, 8, 2
    L = rng.normal(size=(T, E))
    idx = R.topk_select(L, k)
    return L, idx, T, E, k


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from mixture_experts_layer_39_b200 import replicas
        assert replicas.world() == (world, rank, rank)
        slowest = replicas.max_over_ranks(1.5 + rank)
        L, idx, T, E, k = _batch()
        lo, hi = rank * T // world, (rank + 1) * T // world
        p = R.softmax(L[lo:hi])
        counts = np.bincount(idx[lo:hi].reshape(-1), minlength=E)
        stats = torch.tensor(R.router_load_stats(p, counts), dtype=torch.float64)
        replicas.sum_load_stats(stats)
        loss, dprob = R.router_aux_loss(stats.numpy(), T, k, 0.01)
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.concatenate([[slowest, loss], dprob, stats.numpy()]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_global_load_stats_and_max(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    L, idx, T, E, k = _batch()
    whole = R.router_load_stats(R.softmax(L), np.bincount(idx.reshape(-1), minlength=E))
    loss, dprob = R.router_aux_loss(whole, T, k, 0.01)
    for r in range(world):
        got = np.load(tmp_path / f"r{r}.npy")
        assert got[0] == 2.5                       # max over ranks of 1.5 + rank
        assert got[1] == pytest.approx(loss, rel=1e-12)
        np.testing.assert_allclose(got[2:2 + E], dprob, rtol=1e-12)
        np.testing.assert_allclose(got[2 + E:], whole, rtol=1e-12)
