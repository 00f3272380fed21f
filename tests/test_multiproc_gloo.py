"""The multi-rank plumbing of bench.py on CPU: gloo, world size 2, 127.0.0.1 rendezvous."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks(1.5 + rank)           # per-rank times 1.5 and 2.5
    from synth.configs import BY_NAME
    cfg = bench.arm_config(BY_NAME["cla2_1p1b"], world)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, cfg["parallelism"]))


def test_max_over_ranks_and_replica_config():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]
    assert all(r[2] == "replicas x2" for r in res)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    bench.reference_arm(argparse.Namespace(config="cla2_1p1b", steps=1, warmup=3, gpus=2))
    assert capsys.readouterr().out == ""
