"""The multi-rank host logic of bench.py on CPU: two processes with the gloo backend (the GPU job
runs the same functions over NCCL, one rank per GPU). Each rank decodes its own independently
seeded batch (weak scaling, no data-path collective); the job's time is the max over ranks and its
throughput counts every rank's units; the reference arm does no work on ranks other than 0; a rank
that leaves makes the other's next collective fail within the process-group timeout instead of
hanging."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, mode):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    import workloads
    res = {}
    bench.init_ranks("gloo", torch.device("cpu"), world, timeout_s=20 if mode == "normal" else 5)
    try:
        if mode == "normal":
            w = bench.rank_workload(workloads.WORKLOADS["gqa7_32k_decode_3p5pct"], rank, world)
            res["seed"] = w.seed
            res["shape"] = [w.B, w.Hq, w.Hkv, w.d]
            # a small seeded cache per rank: the ranks' data must differ
            small = bench.rank_workload(workloads.WORKLOADS["tiny_f32"], rank, world)
            k, _, _ = workloads.make_kv(small, "cpu")
            res["k_sum"] = float(k.double().sum())
            ms = 10.0 + 5.0 * rank                       # this rank's own duration
            res["max_ms"] = bench.max_over_ranks(ms, torch.device("cpu"), world)
            res["value"] = bench.job_throughput(896, world, 100, res["max_ms"])
            res["reference"] = bench.run_reference(None, rank) if rank != 0 else "rank0"
            bench.finish_ranks(world)
        else:   # rank 1 leaves before the collective; rank 0 must get an error, not hang
            if rank == 1:
                res["left"] = True
            else:
                try:
                    bench.max_over_ranks(1.0, torch.device("cpu"), world)
                    res["error"] = None
                except Exception as e:   # the collective fails once the peer is gone
                    res["error"] = type(e).__name__
    finally:
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    if mode != "normal":
        os._exit(0)   # skip the group's teardown with a dead peer


def _spawn(tmp_path, mode):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path), mode), nprocs=2, join=True,
                       start_method="spawn")
    return [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]


def test_two_ranks_max_over_ranks_and_job_throughput(tmp_path):
    r0, r1 = _spawn(tmp_path, "normal")
    assert r0["shape"] == r1["shape"] and r0["seed"] != r1["seed"]
    assert r0["k_sum"] != r1["k_sum"]                      # independent batches
    assert r0["max_ms"] == r1["max_ms"] == 15.0            # the slowest rank sets the time
    assert r0["value"] == r1["value"] == pytest.approx(896 * 2 * 100 / 0.015)
    assert r1["reference"] is None                         # the reference arm runs on rank 0 only


def test_rank_that_leaves_fails_the_next_collective(tmp_path):
    r0, r1 = _spawn(tmp_path, "leave")
    assert r1["left"] and r0["error"] is not None


def _bench_json(stdout: str):
    lines = [ln for ln in stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, stdout
    return json.loads(lines[0])


def test_bench_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun runs itself as two ranks (torch.distributed.run on
    127.0.0.1); the reference arm, which needs no GPU, prints one line from rank 0 with n_gpus 2
    and the same `config` object the GPU arm prints."""
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3", "--ref-seconds", "1"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    res = _bench_json(p.stdout)
    assert res["n_gpus"] == 2 and res["impl"] == "reference"
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    assert res["config"] == bench.bench_config(workloads.WORKLOADS[bench.WORKLOAD], 2)
    assert res["cpu_baseline"]["kind"] == "oracle" and res["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_refuses_a_rank_count_other_than_gpus():
    """Under a launcher whose WORLD_SIZE differs from --gpus the bench stops with an error naming
    the mismatch instead of timing a different number of GPUs."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3", "--ref-seconds", "1"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert p.returncode != 0 and "WORLD_SIZE=3" in (p.stderr + p.stdout)
