"""Host logic of the N-sharded forward (int8_mixed_precision_column_b200.sharded).

The shard ranges, the peer-destination list and the column gather are checked
here without a GPU: gloo ranks on the CPU stand in for the GPUs, and the
oracle stands in for each rank's kernel (it computes that rank's shard of the
layer).  The assembled Y must equal the oracle's unsharded forward, and every
rank must find the same outlier columns.
"""

from __future__ import annotations

import datetime
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import sharded, workloads


@pytest.mark.parametrize("N,world", [(16, 1), (64, 2), (80, 3), (57344, 4), (57344, 8), (4096, 7), (272, 17)])
def test_shard_range_partitions_n(N, world):
    ranges = [sharded.shard_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
        assert hi == lo2
    sizes = [hi - lo for lo, hi in ranges]
    assert all(s >= 16 and s % 16 == 0 and lo % 16 == 0 for s, (lo, _) in zip(sizes, ranges))
    assert max(sizes) - min(sizes) <= 16


@pytest.mark.parametrize("N,world,rank", [(48, 4, 0), (40, 2, 0), (64, 2, 2), (64, 2, -1)])
def test_shard_range_rejects(N, world, rank):
    with pytest.raises(ValueError):
        sharded.shard_range(N, world, rank)


def test_peer_destinations_own_first_same_offset():
    bufs = [0x7000_0000, 0x9000_0000, 0xA000_0000, 0xB000_0000]
    d = sharded.peer_destinations(0x9000_0400, bufs, 1)
    assert d == [0x9000_0400, 0x7000_0400, 0xA000_0400, 0xB000_0400]
    assert sharded.peer_destinations(0x7000_0000, bufs[:1], 0) == [0x7000_0000]
    with pytest.raises(ValueError):
        sharded.peer_destinations(0x6000_0000, bufs, 0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(T, K, N):
    p = workloads.make_problem("shard", T, K, N, n_planted=5, bias_std=0.01, seed=7)
    CB, SCB = O.quantize_weight(p.W.numpy())
    return p.X.numpy(), CB, SCB, p.bias.numpy()


def _rank_main(rank: int, world: int, port: int, outdir: str, T: int, K: int, N: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        X, CB, SCB, bias = _problem(T, K, N)
        CBs, SCBs, bs, lo, hi = sharded.shard_layer(torch.from_numpy(CB), torch.from_numpy(SCB),
                                                    torch.from_numpy(bias), world, rank)
        r = O.linear_forward(X, CBs.numpy(), SCBs.numpy(), bs.numpy(), 6.0)   # this rank's "kernel"
        Y = sharded.gather_columns(torch.from_numpy(r["Y"]))
        idx_all = [None] * world
        dist.all_gather_object(idx_all, r["idx"].tolist())
        np.save(os.path.join(outdir, f"Y{rank}.npy"), Y.numpy())
        with open(os.path.join(outdir, f"r{rank}.json"), "w") as f:
            json.dump({"lo": lo, "hi": hi, "idx_all": idx_all}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world,N", [(2, 96), (3, 80)])
def test_gloo_ranks_assemble_the_unsharded_forward(tmp_path, world, N):
    T, K = 12, 64
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), T, K, N)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(180)
        assert pr.exitcode == 0
    X, CB, SCB, bias = _problem(T, K, N)
    full = O.linear_forward(X, CB, SCB, bias, 6.0)
    assert full["n_out"] >= 5
    los = []
    for r in range(world):
        meta = json.load(open(tmp_path / f"r{r}.json"))
        los.append((meta["lo"], meta["hi"]))
        assert all(i == full["idx"].tolist() for i in meta["idx_all"])   # same outlier columns everywhere
        Y = np.load(tmp_path / f"Y{r}.npy")
        assert Y.shape == (T, N)
        np.testing.assert_allclose(Y, full["Y"], rtol=1e-13, atol=1e-13)
    assert [sharded.shard_range(N, world, r) for r in range(world)] == los
