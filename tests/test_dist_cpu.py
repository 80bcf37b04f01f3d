"""The multi-rank path of bench.py on CPU (gloo, world size 2): adapters are sharded
with no data exchange, the step time is the max over ranks, and the LoRAForge-S
allocation of a shard equals the allocation of the whole fleet restricted to it (the
budget is per adapter), which is why compression needs no collective."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import allocate as OA
from post_hoc_rank_b200 import synth

WORLD = 2
N_PER_RANK = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _sigma_rows(adapters, lay1):
    """Spectra of the given adapters' modules (σ_j = j^-1 e^{0.5 z}, seeded per adapter)."""
    rows = []
    for a in adapters:
        g = np.random.default_rng(synth.derive_seed(99, a))
        for _ in range(lay1.n):
            s = np.sort((1.0 / np.arange(1, 9)) * np.exp(0.5 * g.standard_normal(8)))[::-1]
            rows.append(s)
    return np.stack(rows)


def _worker(rank, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        base = bench.shard_adapter_base(rank, N_PER_RANK)
        adapters = list(range(base, base + N_PER_RANK))
        lay1 = synth.fleet_layout(1, shapes=[("a", 64, 48), ("b", 32, 80), ("c", 40, 40)], r=8, n_layers=1)
        sig = _sigma_rows(adapters, lay1)
        groups = np.repeat(np.arange(N_PER_RANK), lay1.n)
        ranks, _ = OA.spectral_ranks(sig, np.full(len(sig), 8), groups, 1, 4, 1)
        gathered = [torch.zeros(len(ranks), dtype=torch.int64) for _ in range(WORLD)]
        dist.all_gather(gathered, torch.as_tensor(np.asarray(ranks), dtype=torch.int64))
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        if rank == 0:
            out["ranks"] = torch.cat(gathered).numpy().tolist()
            out["max_ms"] = ms
            out["rate"] = bench.whole_job_rate(100, WORLD, ms)
            out["bases"] = [bench.shard_adapter_base(r, N_PER_RANK) for r in range(WORLD)]
    finally:
        dist.destroy_process_group()


def test_sharded_allocation_and_max_over_ranks():
    port = _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_worker, args=(port, out), nprocs=WORLD, start_method="spawn", join=True)
    # shards are disjoint and cover the fleet
    assert out["bases"] == [0, N_PER_RANK]
    # the slowest rank sets the time; the rate counts every rank's units
    assert out["max_ms"] == 15.0
    assert out["rate"] == pytest.approx(100 * WORLD / 15e-3)
    # the same allocation computed on the whole fleet in one process
    lay1 = synth.fleet_layout(1, shapes=[("a", 64, 48), ("b", 32, 80), ("c", 40, 40)], r=8, n_layers=1)
    sig = _sigma_rows(range(WORLD * N_PER_RANK), lay1)
    groups = np.repeat(np.arange(WORLD * N_PER_RANK), lay1.n)
    whole, _ = OA.spectral_ranks(sig, np.full(len(sig), 8), groups, 1, 4, 1)
    assert out["ranks"] == np.asarray(whole).tolist()
