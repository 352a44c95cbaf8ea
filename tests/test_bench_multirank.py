"""bench.py's multi-rank plumbing on CPU: two gloo ranks (the same code path torchrun drives on GPUs,
with NCCL there). Checks the max-over-ranks reduction and the whole-job unit conversion, and that
the reference arm runs on rank 0 only and prints one JSON line of the contract (the oracle itself
is replaced by a stub here: its timing is not what is tested).
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _StubRunner:
    def __init__(self, mats, xs):
        pass

    def token(self, t):
        pass


def _worker(rank, world, port, outdir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import io
    import contextlib
    import bench

    r, ws, _ = bench.dist_setup()
    assert (r, ws) == (rank, world)
    # every rank gets the slowest rank's time
    got = bench.max_over_ranks(1.5 + rank)
    bench.barrier()
    # whole-job unit: 64 tokens per rank over `world` ranks in 10 ms
    unit = bench.us_per_token_layer(10.0, 64, world)
    with open(os.path.join(outdir, f"helpers{rank}.json"), "w") as f:
        json.dump({"max": got, "unit": unit}, f)
    bench.OracleRunner = _StubRunner
    bench.host_workload = lambda: (None, None)
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "2",
                "--warmup", "3"]
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main()
    with open(os.path.join(outdir, f"out{rank}.txt"), "w") as f:
        f.write(buf.getvalue())
    assert rc == 0


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for rank in range(world):
        h = json.load(open(tmp_path / f"helpers{rank}.json"))
        assert h["max"] == pytest.approx(2.5)
        assert h["unit"] == pytest.approx(10.0 * 1000 / (64 * world))
    assert (tmp_path / "out1.txt").read_text() == ""  # other ranks print nothing
    lines = [ln for ln in (tmp_path / "out0.txt").read_text().splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    import bench
    assert line["metric"] == bench.METRIC
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["higher_is_better"] is False and line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"]
