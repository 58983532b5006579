"""Host-side logic of the multi-GPU benchmark, on two gloo ranks on the CPU.

Each rank runs the whole workload on its own seeded inputs (weak scaling, no
data-path collective); the step time is the maximum over ranks and the job's
throughput is every rank's units over that time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.0 + rank                               # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms)
        value = bench.job_tokens_per_s(1000, world, ms_max)
        w = bench.rank_workload(WORKLOADS["tiny_gdn_fp32"].with_(T=16), rank)
        inp = make_inputs(w, "cpu")
        sums = torch.tensor([float(inp[n].double().sum()) for n in ("q", "k", "v", "g", "beta")],
                            dtype=torch.float64)
        gathered = [torch.zeros_like(sums) for _ in range(world)]
        dist.all_gather(gathered, sums)
        torch.save({"ms_max": ms_max, "value": value, "seed": w.seed, "sums": torch.stack(gathered)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_use_distinct_inputs(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r in res:
        assert r["ms_max"] == 2.0
        assert r["value"] == pytest.approx(world * 1000 / 2e-3)
    assert res[0]["seed"] != res[1]["seed"]
    sums = res[0]["sums"]
    assert torch.equal(sums, res[1]["sums"])          # both ranks saw the same gathered table
    assert not torch.equal(sums[0], sums[1])          # and their inputs differ


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_tokens_per_s(10, 1, 1.0) == pytest.approx(1e4)
