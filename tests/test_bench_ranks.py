"""The benchmark's multi-rank logic on CPU: two gloo ranks reduce their step
times (max) and token counts (sum) as the GPU run does, replicas draw distinct
batches, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank: int, world: int, port: int, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        t_ms = [3.0, 5.0][rank]
        tokens = [256.0, 128.0][rank]
        mx = bench.reduce_over_ranks(t_ms, "max", world, "cpu")
        sm = bench.reduce_over_ranks(tokens, "sum", world, "cpu")
        q.put((rank, mx, sm, bench.replica_seed(0, rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_gpu_run():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [5.0, 5.0]          # time = max over ranks
    assert [g[2] for g in got] == [384.0, 384.0]      # tokens = whole-job sum
    assert got[0][3] != got[1][3]                     # each replica its own batch


def test_single_rank_reduction_is_identity():
    assert bench.reduce_over_ranks(1.5, "max", 1, "cpu") == 1.5


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.argparse.Namespace(workload="step3_decode", steps=1, warmup=0, cpu_seconds=1.0,
                                    reference_seconds=5.0, experts=0)
    assert bench.run_reference(args) is None


@pytest.mark.parametrize("name", ["step3_decode", "deepseek_decode", "dp_padded"])
def test_algorithmic_bytes_follow_touched_experts(name):
    import numpy as np
    import synth
    w = synth.WORKLOADS[name]
    valid = int(synth.workloads.valid_mask(w).sum())
    full = np.arange(w.E + 1) * (valid * w.k // w.E)
    a = bench.algorithmic(w, valid, full, w.k)
    assert a["touched_experts"] == w.E
    half = full.copy()
    half[1::2] = half[:-1:2]            # every other expert empty
    b = bench.algorithmic(w, valid, np.maximum.accumulate(half), w.k)
    assert b["touched_experts"] < a["touched_experts"]
    assert b["step_bytes"] < a["step_bytes"]


def test_reference_arm_line(capsys, monkeypatch):
    import json
    import oracle
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = bench.argparse.Namespace(workload="tiny", steps=2, warmup=1, cpu_seconds=0.2,
                                    reference_seconds=1.0, experts=0)
    res = bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line == json.loads(json.dumps(res))
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"]
    assert line["config"]["workload"] == "tiny" and line["n_gpus"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["warmup"] == 1
    assert line["cpu_baseline"]["cores"] == oracle.max_threads() >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("env,argv,want", [
    ({"WORLD_SIZE": "1"}, [], ("native", "step3_decode", False)),
    ({"WORLD_SIZE": "1"}, ["--workload", "fp8_prefill"], ("native", "fp8_prefill", True)),
    ({"WORLD_SIZE": "2"}, [], ("tp", "step3_decode", False)),       # the scaling command
    ({"WORLD_SIZE": "2"}, ["--replicas"], ("native", "step3_decode", False)),
    ({"WORLD_SIZE": "1"}, ["--tp"], ("tp", "dp_padded", False)),
    ({"WORLD_SIZE": "1"}, ["--impl", "reference"], ("reference", "step3_decode", False)),
])
def test_dispatch(monkeypatch, env, argv, want):
    for kk, v in env.items():
        monkeypatch.setenv(kk, v)
    seen = []
    for arm in ("native", "tp", "reference"):
        monkeypatch.setattr(bench, f"run_{arm}",
                            lambda a, arm=arm: seen.append((arm, a.workload, a.single)))
    bench.main(argv)
    assert seen == [want]
