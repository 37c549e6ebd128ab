"""Host logic of the multi-GPU path on CPU ranks (world size 2, gloo): the
path shards batch x channels into independent problems with no exchange, so
what crosses ranks is only the timing: each rank's step time is reduced to
the maximum over ranks, and rank 0 reports the whole-job rate.  Also checks
that every rank draws its own shard and that the reference arm runs on rank
0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import torch.distributed as tdist
    import bench
    tdist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                             world_size=world)
    try:
        # rank r: step time 2 + r ms, launch time 1 - 0.5 r ms
        got = bench.max_over_ranks([2.0 + rank, 1.0 - 0.5 * rank], device="cpu")
        rate = bench.aggregate_rate(world, 1.0e6, got[0])
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "rate": rate}, f)
    finally:
        tdist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate_gloo(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == [3.0, 1.0]          # slowest rank's step, each value separately
        assert r["rate"] == pytest.approx(2 * 1.0e6 / 3.0e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], device="cpu") == [1.5, 2.5]


def test_shards_differ_per_rank():
    import bench
    import numpy as np
    import synthetic
    cfg = synthetic.CONFIGS[0]
    seeds = [bench.shard_seed(cfg, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == cfg["seed"]
    a = synthetic.make_config(0, seed=seeds[0])["u"]
    b = synthetic.make_config(0, seed=seeds[1])["u"]
    assert a.shape == b.shape and not np.array_equal(a, b)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "0",
                        "--steps", "2", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        line = json.loads(lines[0])
        assert line["impl"] == "reference" and line["n_gpus"] == 2
        assert line["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
