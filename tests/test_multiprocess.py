"""The N > 1 plumbing of bench.py on the CPU: two gloo ranks on 127.0.0.1.

The decode path does not shard (sequences are independent, each GPU runs its own
replica), so what runs across processes is the harness: the process group, the barrier
around the timed region and the max-over-ranks reduction of the device times.  These
tests run that code with the gloo backend (no GPU), and run the reference arm under
torch.distributed.run with two ranks: rank 0 alone does the work and prints one line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    bench.dist_barrier()
    # the slowest rank's device time is the step time of the whole job
    t = bench.dist_max(10.0 + 5.0 * rank)
    bench.dist_barrier()
    bench._finish()
    results[rank] = t


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_barrier_gloo(world):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert dict(results) == {r: 10.0 + 5.0 * (world - 1) for r in range(world)}


def test_reference_arm_two_ranks_prints_once(oracle_lib):
    """bench.py --impl reference launched the way the driver launches N > 1: rank 0 runs
    the oracle and prints the single JSON line, the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--config", "gqa_b1_h8_kv2_d64_t512"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    # the reference arm's config object is the one the GPU arm prints for the same workload
    import bench
    from mla_kv_cache_b200 import workloads as wl
    name = "gqa_b1_h8_kv2_d64_t512"
    cfg = wl.CONFIGS[name]
    lens = [cfg.max_seq_len] * cfg.batch
    assert rec["config"] == bench.config_fields(name, cfg, bench.step_bytes(cfg, lens), 2)
