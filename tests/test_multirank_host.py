"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The SS2D path shards by batch with no exchange step, so the only cross-rank work
is the barrier around the timed region and the reductions of its results: the
step time is the max over ranks and the work is the sum over ranks.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    import ss2d_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(10.0 + rank, world)
        units = bench.sum_over_ranks(100.0 * (rank + 1), world)
        w = ss2d_inputs.custom(1, 2, 3, 3, 2)
        x = ss2d_inputs.make_inputs(w, seed=bench.shard_seed(1, rank))["x"]
        q.put((rank, ms, units, x.sum().item()))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_distinct_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, units, _ in res:
        assert ms == 11.0        # max over ranks
        assert units == 300.0    # sum over ranks
    assert res[0][3] != res[1][3]  # each rank draws its own shard


def test_shard_seeds_are_distinct():
    import bench
    seeds = {bench.shard_seed(1, r) for r in range(8)}
    assert len(seeds) == 8


def test_reference_arm_runs_on_cpu(capsys):
    import json

    import bench
    # the tiny workload keeps this fast; the reference arm never touches a GPU
    rc = bench.main(["--impl", "reference", "--workload", "0", "--steps", "2", "--warmup", "3",
                     "--cpu-seconds", "2"])
    assert rc == 0
    line = capsys.readouterr().out.strip().splitlines()[-1]
    rec = json.loads(line)
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_algorithmic_bytes_match_the_stated_figure():
    import bench
    import ss2d_inputs
    w = ss2d_inputs.workload(1)
    # read u (308.3 MB), delta (1233.1 MB), B and C (102.8 MB each), write y (308.3 MB) in fp32
    assert abs(bench.fwd_algorithmic_bytes(w) / 1e6 - 2055.3) < 0.5
    assert w.updates == 4_932_501_504


def test_backward_and_producer_bytes():
    import bench
    import ss2d_inputs
    w = ss2d_inputs.workload(4)  # B=32 stage-1 shapes, fp32
    # forward 513.9 MB; backward reads x, delta, B, C, dy and writes dx, ddelta, dB, dC: 950.6 MB
    assert abs(bench.fwd_algorithmic_bytes(w) / 1e6 - 513.9) < 0.5
    assert abs(bench.bwd_algorithmic_bytes(w) / 1e6 - 950.6) < 0.5
    w1 = ss2d_inputs.workload(1)
    R = ss2d_inputs.dt_rank_of(w1.dim)
    # x read, y written (308.3 MB each), x_dbl (B, 4, R+2N, L) written, the small weights
    img = w1.batch * w1.dim * w1.L * 4
    xdbl = w1.batch * 4 * (R + 2 * w1.d_state) * w1.L * 4
    weights = 4 * (4 * (R + 2 * w1.d_state) * w1.dim + 4 * w1.dim * R + 4 * w1.dim * (w1.d_state + 2))
    assert bench.proj_algorithmic_bytes(w1, R) == 2 * img + xdbl + weights


def test_recorded_traffic_needs_the_captured_sources(monkeypatch):
    import bench
    rec = bench.recorded_traffic("vmamba_t_stage1_fp32")
    assert rec is None or rec > bench.fwd_algorithmic_bytes(__import__("ss2d_inputs").workload(1))
    # any change to the hashed kernel sources invalidates the record
    monkeypatch.setattr(bench, "source_hash", lambda files=None: "0" * 16)
    assert bench.recorded_traffic("vmamba_t_stage1_fp32") is None
    assert bench.recorded_traffic("no such workload") is None
