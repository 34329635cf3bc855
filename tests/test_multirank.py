"""The multi-GPU host logic of bench.py, run as two gloo ranks on the CPU.

Each rank draws its own batch of the workload (disjoint rows, no data-path
exchange); the job time is the maximum of the per-rank times; rank 0 alone
reports, and the reference arm does no work on the other ranks."""
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import types

    import bench
    import long_context_gsa_b200.workloads as W

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    cfg = W.scaled(W.LLAMA_8X, batch=1, hq=4, hkv=2, context=8 * 16)
    x = W.decode_inputs(cfg, device="cpu", seed=bench.rank_seed(cfg, rank))
    # per-rank timed totals differ; every rank must see the maximum
    step_ms, e2e_ms = 10.0 + rank, 30.0 - 5.0 * rank
    total, total_e2e = bench.max_over_ranks([step_ms, e2e_ms], world, "cpu")
    ref = bench.run_reference(types.SimpleNamespace(workload="pr1", steps=1, warmup=0), world, rank) if rank else None
    res = {"seed": bench.rank_seed(cfg, rank), "q_sum": float(x["q"].float().sum()), "total": total,
           "total_e2e": total_e2e, "rate": bench.job_rate(cfg.head_queries, world, 4, total),
           "ref_none": ref is None}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["q_sum"] != r[1]["q_sum"]                      # disjoint inputs per rank
    for i in range(world):
        assert r[i]["total"] == pytest.approx(11.0)           # max over ranks of 10, 11
        assert r[i]["total_e2e"] == pytest.approx(30.0)       # max over ranks of 30, 25
    # whole-job rate: units of both ranks over the slowest rank's time
    assert r[0]["rate"] == pytest.approx(1 * 4 * 2 * 4 / (11.0 / 1e3))
    assert r[1]["ref_none"]                                    # reference arm: rank 1 does no work
