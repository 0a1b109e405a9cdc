"""The N > 1 path of bench.py (independent replicas, one process per GPU) on the
CPU: two gloo ranks take the same collective steps, get the slowest rank's
time, draw distinct token streams, and only rank 0 prints."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    from quantized_routed_expert_04_b200 import synth
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    w, r, _ = bench.dist_env()
    # the two reductions of a bench run, in the same order on every rank
    step_ms = bench.max_over_ranks(1.0 + 0.5 * rank, w, "cpu")
    e2e_ms = bench.max_over_ranks(3.0 - rank, w, "cpu")
    cfg = synth.CONFIGS["tiny"]
    x = synth.make_x(cfg, 4, bench.replica_seed(0, r), step=0)
    dist.barrier()
    dist.destroy_process_group()
    res = {"world": w, "rank": r, "step_ms": step_ms, "e2e_ms": e2e_ms,
           "value": bench.whole_job_tokens_per_s(4, w, step_ms), "x": x.tolist()}
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump(res, f)


def test_two_gloo_replicas(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    for r, got in enumerate(res):
        assert got["world"] == world and got["rank"] == r
        assert got["step_ms"] == 1.5  # the slower rank's time, on both ranks
        assert got["e2e_ms"] == 3.0
        assert got["value"] == pytest.approx(4 * world / 1.5e-3)
    assert res[0]["x"] != res[1]["x"]  # each replica has its own tokens


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.whole_job_tokens_per_s(8, 1, 2.0) == pytest.approx(4000.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--config", "tiny",
                                      "--steps", "1", "--warmup", "3"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    assert buf.getvalue() == ""


def test_reference_arm_line(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--config", "tiny",
                                      "--steps", "2", "--warmup", "3"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    lines = buf.getvalue().strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert np.isfinite(line["ms_per_step"])
    # both arms describe the workload with the same config object
    from quantized_routed_expert_04_b200 import synth
    assert line["config"] == bench.config_desc(synth.CONFIGS["tiny"], 4, 1)
    assert line["cpu_baseline"]["host_cpu_count"] == os.cpu_count()
