"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, no GPU.

With N > 1 every rank runs its own replica of the workload; the only
collectives are the barriers around the timed region and the max over ranks of
its length.  These tests run that host logic as two real processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    n = bench.init_ranks("gloo", rank, timeout_s=60)
    bench.barrier()
    # each rank "timed" a different interval; all must agree on the slowest
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
    ms_again = bench.max_over_ranks(3.0 - rank, "cpu")
    value = bench.job_throughput(n, 1000, 4, ms)
    bench.finish_ranks()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"world": n, "ms": ms, "ms_again": ms_again, "value": value}, f)


def test_two_gloo_ranks_agree_on_the_slowest_rank(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["world"] == 2
        assert r["ms"] == 15.0 and r["ms_again"] == 3.0
        # whole-job throughput: both ranks' elements over the slowest rank's time
        assert r["value"] == pytest.approx(2 * 1000 * 4 / 15e-3 / 1e9)


def test_single_process_collectives_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, "cpu") == 7.5
    bench.barrier()
    assert bench.job_throughput(1, 10**9, 2, 1000.0) == pytest.approx(2.0)


def _run_bench(args, env_extra, timeout=300):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--workload", "tiny-f32"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    """The reference arm is the fp64 oracle on the host cores, on rank 0 only."""
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "tiny-f32"],
                   {"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "Gelem/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny-f32"
