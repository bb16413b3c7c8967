"""Multi-rank host logic of the benchmark on CPU: world size 2 over gloo.

The path shards over (batch, head) with no data-path collective, so what the
ranks share is the timing: every rank's step time is reduced to the slowest
one (all-reduce MAX) and the whole-job rate counts every rank's tokens.  The
reference arm under torch.distributed.run prints from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    import bench
    from lsh_attention_02_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    bench.init_ranks("gloo", timeout_s=60)
    mine = [1.0 + rank, 10.0 - 3 * rank]                     # rank 0: (1, 10), rank 1: (2, 7)
    got = bench.max_over_ranks(mine, world, "cpu")
    w = synth.WORKLOADS["long_64k"]
    rate = bench.whole_job_tokens_per_s(w, world, got[0])
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, got, rate))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from lsh_attention_02_b200 import synth
    tokens = synth.WORKLOADS["long_64k"].tokens
    for rank, got, rate in res:
        assert got == [2.0, 10.0], (rank, got)              # element-wise max over both ranks
        assert rate == pytest.approx(tokens * 2 / 2e-3)     # both ranks' tokens over the slowest step


def test_max_over_ranks_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.5], 1, "cpu") == [3.0, 4.5]


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks launched like the multi-GPU bench: rank 0 alone times the
    oracle and prints one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_f32",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env={**os.environ, "OMP_NUM_THREADS": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
