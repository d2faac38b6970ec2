"""World-size-2 gloo run of the benchmark's multi-rank host logic on CPU: each
rank processes its own batch (no data-path collective), the timing is reduced
as the max over ranks, and the whole-job throughput counts every rank's tokens."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    # every rank: its own batch of the same layer (weights replicated)
    w = wl.Workload("dp", E=4, H=64, I=64, k=2, renorm=True, T=6, seed=100 + rank)
    x = wl.activations(w).float().numpy()
    gu, dn = wl.weights(wl.Workload("dp", E=4, H=64, I=64, k=2, renorm=True, T=6, seed=100))
    pg, ag = oracle.quantize(gu.numpy())
    pd, ad = oracle.quantize(dn.numpy())
    wgu = oracle.dequantize(pg, ag, gu.shape)
    wd = oracle.dequantize(pd, ad, dn.shape)
    idx, wts = oracle.route(wl.router_logits(w, wl.activations(w)).numpy(), w.k, w.renorm)
    y = oracle.forward(x, idx, wts, wgu, wd)
    fake_ms = 10.0 * (rank + 1)                       # rank 1 is the slow one
    total = bench.max_over_ranks(fake_ms)
    value = bench.job_throughput(w.T, world, total)
    out[rank] = (total, value, float(np.abs(y).sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 20.0             # max over ranks
    assert abs(out[0][1] - 2 * 6 / 0.020) < 1e-9      # all ranks' tokens / max time
    assert out[0][2] != out[1][2]                     # each rank computed its own batch
