"""Host logic of bench.py that needs no GPU: the ``config`` object of each
JSON line is built by one function per operation and shared by the kernel
arm and the reference arm, so the two lines describe the same workload."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic  # noqa: E402

KEYS = {"workload", "batch", "d_inner", "d_state", "global_batch", "l2", "parallelism"}


@pytest.mark.parametrize("idx", sorted(synthetic.CONFIGS))
@pytest.mark.parametrize("world", [1, 4])
def test_scan_config_describes_the_workload(idx, world):
    cfg = synthetic.CONFIGS[idx]
    c = bench.scan_config(cfg, world)
    assert KEYS | {"seq_len", "seed"} <= set(c)
    assert c["workload"] == cfg["name"] and c["seq_len"] == cfg["L"]
    assert c["global_batch"] == cfg["batch"] * world
    assert c["parallelism"] == f"dp{world} (independent shards, no collective)"
    big = bench.algorithmic_bytes(cfg) > 126e6
    assert c["l2"].startswith("inputs larger" if big else "inputs smaller")


@pytest.mark.parametrize("idx", [i for i, c in synthetic.CONFIGS.items() if c["kind"] == "diag"])
def test_bwd_config_describes_the_workload(idx):
    cfg = synthetic.CONFIGS[idx]
    c = bench.bwd_config(cfg, 2)
    assert KEYS | {"seq_len"} <= set(c)
    assert c["workload"] == "backward of " + cfg["name"]
    assert c["global_batch"] == 2 * cfg["batch"]


@pytest.mark.parametrize("kind", ["diag", "scalarA"])
def test_step_config_describes_the_workload(kind):
    base = next(c for c in synthetic.CONFIGS.values() if c["kind"] == kind and c["L"] > 256)
    cfg = bench.step_workload(base, 64)
    c = bench.step_config(cfg, 1)
    assert KEYS <= set(c)
    assert c["batch"] == 64 and c["workload"] == bench.step_name(cfg)
    dim = cfg.get("dim") or cfg["nheads"] * cfg["headdim"]
    assert c["d_inner"] == dim
