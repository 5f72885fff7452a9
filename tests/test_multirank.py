"""Host-side logic of the multi-GPU run, on CPU with gloo (world size 2).

Blocks are independent, so ranks share no data: each rank solves its own
matrix (its own seed) and only the step time is reduced (max over ranks).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
        mx = bench.max_over_ranks(ms, torch.device("cpu"), world)
        w = synth.WORKLOADS["w4096x11008_bf16_t3_16of32"]
        q.put((rank, mx, bench.rank_seed(w, rank), bench.aggregate_gparams(w.params, world, mx)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_to_the_slowest_and_aggregate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    w = synth.WORKLOADS["w4096x11008_bf16_t3_16of32"]
    assert [r[1] for r in res] == [15.0, 15.0]               # both see the slowest rank
    assert res[0][2] != res[1][2]                            # distinct matrices per rank
    assert res[0][3] == pytest.approx(w.params * 2 / 15e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    assert bench.aggregate_gparams(10**9, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_on_other_ranks_does_nothing(capsys):
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
