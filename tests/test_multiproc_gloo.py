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


def test_reference_arm_rank0_prints_one_contract_line(monkeypatch, capsys):
    import argparse
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.reference_arm(argparse.Namespace(config="cla2_1p1b", steps=1, warmup=3, gpus=1))
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tok/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["steps"] == 1 and d["warmup"] == 3 and d["config"]["workload"] == "cla2_1p1b"
    assert d["data"] == "synthetic (seeded Philox, q/k/v N(0,1)/8)"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
