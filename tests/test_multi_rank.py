"""Host logic of the N-GPU bench on CPU: two gloo ranks on 127.0.0.1.

Each rank runs independent work (replicas, no data-path collective); the only
cross-rank steps are barriers and the max over ranks of the step time.  The
reference arm runs on rank 0 alone, and the other ranks leave without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    r, w, local = bench.rank_info()
    times = [1.5, 2.25]                     # this rank's step time (ms); rank 1 is the slow one
    dist.barrier()
    worst = bench.max_over_ranks_of(times[r], w, "cpu")
    value = bench.weak_scaling_value(2.0e12, w, worst)
    dist.barrier()
    dist.destroy_process_group()
    with open(out_path, "w") as f:
        json.dump({"rank": r, "world": w, "local": local, "worst": worst, "value": value}, f)


def test_two_gloo_ranks_agree_on_the_slowest_rank(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, str(tmp_path / f"r{r}.json"))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r, j in enumerate(res):
        assert (j["rank"], j["world"], j["local"]) == (r, 2, r)
        assert j["worst"] == 2.25
        # two ranks x 2 TFLOP of work in the slowest rank's 2.25 ms
        assert abs(j["value"] - 2 * 2.0e12 / 2.25e-3 / 1e12) < 1e-9


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks_of(3.5, 1, "cpu") == 3.5
    assert abs(bench.weak_scaling_value(1e12, 1, 1.0) - 1000.0) < 1e-9   # 1 TFLOP in 1 ms


def test_reference_arm_line_on_rank_zero():
    """Rank 0 of `bench.py --impl reference` prints one JSON line with the contract's keys; the oracle
    is the reference arm, so its e2e moves no bytes and its cpu_baseline describes the same run."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                          "small_v3_bf16", "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("small_v3_bf16")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    """A non-zero rank of `bench.py --impl reference` exits 0 at once and prints nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""
