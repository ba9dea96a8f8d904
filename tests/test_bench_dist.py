"""Host logic of the multi-process benchmark on CPU, with two gloo ranks (world size 2).

`bench.py --gpus N` runs N independent replicas: each rank times its own steps on its GPU,
the job's time is the maximum over the ranks and the value is the units all ranks processed
per second of that time. These tests drive that reduction over a gloo process group, the
reference arm under torchrun (rank 0 alone runs the oracle sample and prints one line; the
other ranks exit 0 without work), and a replica that fails between steps: the surviving
rank's reduction ends with an error within the group's timeout instead of waiting. No GPU
is used.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = [2.0 + rank, 3.0 + 4 * rank]             # rank 1 is the slower replica
        t = bench.max_over_ranks(sum(step_ms), world, "cpu")
        v = bench.job_throughput(8192 * len(step_ms), world, t)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out, f"rank{rank}.json"), "w") as f:
        json.dump({"t": t, "v": v}, f)


def test_max_over_ranks_and_job_throughput_two_gloo_ranks(tmp_path):
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    assert r[0]["t"] == r[1]["t"] == 10.0                 # max(5, 10) ms on every rank
    assert r[0]["v"] == r[1]["v"] == 2 * 8192 * 2 / 0.010  # both ranks' tokens / 10 ms


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(8192, 1, 2.0) == 8192 / 0.002


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def _rank_dies(rank, world, port, out):
    """Rank 1 leaves before the reduction; rank 0 must get an error, not wait for ever."""
    import time
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)                                       # a replica that fails between steps
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0, world, "cpu")
        result = "no error"
    except Exception as e:                                # noqa: BLE001
        result = type(e).__name__
    with open(os.path.join(out, "rank0.json"), "w") as f:
        json.dump({"result": result, "seconds": time.monotonic() - t0}, f)
    os._exit(0)


def test_a_failed_rank_ends_the_reduction_with_an_error(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank was still waiting after 120 s"
    assert procs[1].exitcode == 3 and procs[0].exitcode == 0
    r = json.load(open(tmp_path / "rank0.json"))
    assert r["result"] != "no error" and r["seconds"] < 60
