"""The bench's multi-rank logic on CPU: two gloo ranks (world size 2) run the same
reductions bench.py uses under torchrun — the barrier, max over ranks of the timed
region, the sum of the units all ranks processed, and the whole-job rate built from
them — and the reference arm's rule that only rank 0 runs and prints."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import json, sys
sys.path.insert(0, {root!r})
import bench
world, rank, local, pg = bench.setup_dist(None)
assert pg is not None and pg.get_backend() == "gloo", pg
bench.barrier(pg)
units, ms = 100.0 * (rank + 1), 10.0 * (rank + 1)
out = {{"rank": rank, "world": world,
        "max": bench.max_over_ranks(pg, ms), "sum": bench.sum_over_ranks(pg, units),
        "rate": bench.whole_job_rate(pg, units, ms)}}
bench.barrier(pg)
pg.destroy_process_group()
print(json.dumps(out))
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(script: str, world: int, extra_env=None):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                   WORLD_SIZE=str(world), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, e[-2000:]
        outs.append(o)
    return outs


def test_two_gloo_ranks_aggregate_like_the_bench():
    outs = _launch(RANK_SCRIPT.format(root=ROOT), 2)
    res = sorted((json.loads(o.strip().splitlines()[-1]) for o in outs), key=lambda r: r["rank"])
    assert [r["rank"] for r in res] == [0, 1]
    for r in res:
        assert r["world"] == 2
        assert r["max"] == 20.0  # the slowest rank's time
        assert r["sum"] == 300.0  # units of all ranks
        units_all, ms_max, rate = r["rate"]
        assert (units_all, ms_max) == (300.0, 20.0)
        assert rate == pytest.approx(300.0 / 0.020)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun every rank but 0 exits 0 at once, printing nothing."""
    script = (f"import sys; sys.path.insert(0, {ROOT!r}); import bench; "
              "sys.argv = ['bench.py', '--impl', 'reference', '--gpus', '2']; "
              "sys.exit(bench.main())")
    port = _free_port()
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="1",
               WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, "-c", script], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=120)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
