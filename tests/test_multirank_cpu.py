"""The multi-rank path of bench.py on the host: world-size-2 process groups on the gloo
backend (CPU).  The decode shards into independent (sequence, KV head) units, so ranks
exchange nothing but their timings: the job's step time is the maximum over the ranks, its
throughput the tokens of all ranks over that time, and every rank decodes its own sequences.
The reference arm under several ranks runs and prints on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_over_ranks([1.0 + rank, 5.0 - rank, 3.0 + 0.5 * rank])
        q.put((rank, got))
    finally:
        torch.distributed.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_step_time_is_the_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert results[rank] == [2.0, 5.0, 3.5]


def test_reduction_without_a_process_group_is_the_identity():
    import bench
    assert bench.reduce_over_ranks([0.25, 7.0]) == [0.25, 7.0]


def test_job_throughput_counts_every_rank():
    import bench
    # 16 sequences per rank, 8 ranks, 2 ms per step (the slowest rank's)
    assert bench.job_tokens_per_s(16, 8, 2.0) == pytest.approx(64000.0)
    assert bench.job_tokens_per_s(16, 1, 2.0) == pytest.approx(8000.0)


def test_ranks_decode_distinct_sequences():
    import bench
    seeds = [bench.rank_seed(1002, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == 1002
    assert seeds == [bench.rank_seed(1002, r) for r in range(8)]  # deterministic


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_0_only(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                          "--cpu-seconds", "0.5"], env=env, capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    else:
        assert lines == []


def test_gpus_flag_launches_the_ranks_itself():
    # no WORLD_SIZE in the environment: bench.py --gpus 2 starts two ranks (torch.distributed.run
    # on 127.0.0.1) and rank 0 prints the one line
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                          "--cpu-seconds", "0.5"], env=env, capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_world_size_must_match_the_gpus_flag():
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "3"], env=env,
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode != 0 and "WORLD_SIZE" in out.stderr


def test_reference_arm_config_is_the_gpu_arms():
    import argparse
    import bench
    import stief_inputs as si
    args = argparse.Namespace(int8=False, latent=False, joint=False, paged=False, unfused=False)
    c = bench.config_dict(si.WORKLOADS["llama3_8b_32k"], args, 1)
    assert c["workload"] == "llama3_8b_32k" and c["context"] == 32768 and c["ranks"] == [[64, 64]]
    assert "stief_append_decode" in c["step"] and "6 copies" in c["l2"]
