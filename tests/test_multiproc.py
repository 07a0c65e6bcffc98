"""Multi-process host logic on the CPU (gloo, world size 2).

With N GPUs the benchmark runs one independent replica per rank: tokens are
independent, so no collective touches the data path.  The host logic that
does span ranks - the max over ranks of the timed region and the whole-job
token count - is exercised here with gloo; so is the rule that only rank 0
prints, for the reference arm launched under torchrun."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    bench.init_dist(world, "gloo")
    # rank r "took" (r + 1) * 10 ms for 5 steps of 4096 tokens
    ms_step, tps = bench.throughput((rank + 1) * 10.0, 5, 4096, world)
    q.put((rank, ms_step, tps))
    dist.barrier()
    dist.destroy_process_group()


def test_timing_is_the_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_step, tps in res:
        assert ms_step == pytest.approx(20.0 / 5)             # slowest rank: 20 ms / 5 steps
        assert tps == pytest.approx(2 * 4096 / (4.0 / 1e3))   # every rank's tokens


def test_single_rank_throughput_is_local():
    sys.path.insert(0, ROOT)
    import bench
    ms_step, tps = bench.throughput(30.0, 10, 64, 1)
    assert ms_step == pytest.approx(3.0) and tps == pytest.approx(64 / 3e-3)


def test_reference_arm_prints_once_under_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
           "--workload", "silu_gated_t64_d64_f128_e8_k2_f32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["unit"] == "tokens/s"
    one = d["cpu_baseline"]["single_core"]           # a small float32 layer: one core too
    assert one["cores"] == 1 and one["value"] > 0


def test_oracle_rate_repeats_a_quick_batch():
    """On a batch far quicker than the budget, the sample is the batch
    repeated, and the rate is tokens over the summed time."""
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_ffn_09_b200 import synth
    w = synth.SILU_SMALL
    d = synth.make_inputs(w)
    rate, n, secs = bench.oracle_rate(w, d, 0.4)
    assert n > w.T and n % w.T == 0 and secs >= 0.1
    assert rate == pytest.approx(n / secs)
