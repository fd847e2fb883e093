"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks time and the sum of all ranks' work, and the reference arm's
rule that only rank 0 runs."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        t_ms = [0.125, 0.250][rank]
        flops = [1e9, 3e9][rank]
        mx, total = bench.reduce_max_sum(t_ms, flops, world, torch.device("cpu"))
        out[rank] = (mx, total)
    finally:
        dist.destroy_process_group()


def test_reduce_max_sum_two_ranks():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in (0, 1):
        mx, total = out[rank]
        assert mx == 0.25
        assert total == 4e9


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_sum(1.5, 7.0, 1, torch.device("cpu")) == (1.5, 7.0)


def test_reference_arm_other_ranks_exit(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""
