"""Host logic of the multi-process benchmark (one process per GPU, weak scaling):
rank discovery from the launcher's environment, the max-over-ranks timing and
the whole-job aggregate, run as two `gloo` ranks on the CPU; and the oracle arm's
rule that ranks other than 0 do no work.  No GPU is touched."""
import contextlib
import io
import json
import os
import socket
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port() -> int:
    with contextlib.closing(socket.socket(socket.AF_INET, socket.SOCK_STREAM)) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str, step_ms: list):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import datetime

    import torch.distributed as dist

    import bench

    r, w, local = bench.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(step_ms[r], dist, "cpu")
        e2e = bench.max_over_ranks(10.0 * step_ms[r], dist, "cpu")    # a second collective, same order
        value = bench.whole_job_tflops(w, bench.GEMM_FLOPS, slowest)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    Path(out_dir, f"rank{r}.json").write_text(json.dumps(
        {"rank": r, "world": w, "local": local, "slowest": slowest, "e2e": e2e, "value": value}))


def test_two_gloo_ranks_take_the_slowest_step(tmp_path):
    step_ms = [0.50, 0.55]                  # rank 1 is the slower one
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path), step_ms), nprocs=2,
                       start_method="spawn", join=True)
    import bench
    got = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(2)]
    for r, g in enumerate(got):
        assert (g["rank"], g["world"], g["local"]) == (r, 2, r)
        assert g["slowest"] == pytest.approx(0.55)
        assert g["e2e"] == pytest.approx(5.5)
        # both ranks' FLOPs over the slowest rank's step time
        assert g["value"] == pytest.approx(2 * bench.GEMM_FLOPS / 0.55e-3 / 1e12)
    assert got[0]["value"] == got[1]["value"]


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(0.7, None, "cpu") == 0.7
    assert bench.whole_job_tflops(1, 2e12, 1.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        assert bench.run_reference(argparse.Namespace(steps=3, warmup=3)) is None
    assert out.getvalue() == ""
