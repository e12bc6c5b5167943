"""Host-side logic of the multi-rank benchmark, run as 2 gloo ranks on CPU.

Under torchrun every rank runs an independent problem of the same shape
(weak scaling, no data-path collective); the step time is the max over ranks
and the value is the work of all ranks divided by it.
"""

from __future__ import annotations

import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from int8_mixed_precision_column_b200 import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        # local rank 0 builds the library if stale; every rank loads it after the barrier
        bench.ensure_library(world, lr)
        p = workloads.make_problem("rank", 8, 64, 32, n_planted=2, bias_std=0.01, seed=bench.rank_seed(rank))
        local_ms = 1.0 + 0.5 * rank          # rank 1 is the slow one
        bench.barrier(world)
        ms_max = bench.reduce_max(local_ms, world, "cpu")
        tops, tok = bench.whole_job(2.0 * 8 * 32 * 64, 8, world, ms_max)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "tops": tops, "tok": tok, "x_sum": float(p.X.float().sum()),
                       "shape": list(p.X.shape)}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_time_and_weak_scaling(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(120)
        assert pr.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert res[0]["ms_max"] == res[1]["ms_max"] == 1.5
    sec = 1.5e-3
    assert res[0]["tops"] == pytest.approx(2.0 * 8 * 32 * 64 * 2 / sec / 1e12)
    assert res[0]["tok"] == pytest.approx(8 * 2 / sec)
    # independent problems of one shape
    assert res[0]["shape"] == res[1]["shape"]
    assert res[0]["x_sum"] != res[1]["x_sum"]


def test_single_rank_defaults():
    assert bench.reduce_max(3.0, 1, "cpu") == 3.0
    bench.barrier(1)
    assert bench.rank_seed(0) != bench.rank_seed(1)


def test_clock_sampler_parses_nvidia_smi_rows(tmp_path):
    s = bench.ClockSampler("00000000:1B:00.0")
    s.path = str(tmp_path / "c.csv")
    rows = [
        "2026/12/02 10:00:00.100, 00000000:1B:00.0, 1965, 1965, 800.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.200, 00000000:1B:00.0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.300, 00000000:1B:00.0, 1700, 1965, 995.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.300, 00000000:2A:00.0, 300, 1965, 95.0, 0x0000000000000000, Active, Not Active, Not Active, Not Active",
    ]
    with open(s.path, "w") as f:
        f.write("\n".join(rows) + "\n")
    import time as _t

    t = _t.mktime(_t.strptime("2026/12/02 10:00:00", "%Y/%m/%d %H:%M:%S"))
    s.t0, s.t1 = t, t + 1

    class _Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc = _Done()
    out = s.stop()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]  # the other GPU's hw_slowdown is not ours
    assert out["samples"] == 3
