"""The N > 1 path on CPU: two gloo ranks, no GPU.

Covers what bench.py does across ranks: per-rank seeds (independent batches),
the max over ranks of the timed region, the whole-job weak-scaling value, and
that the reference arm prints from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from gemm_epilogue_transformer_02_b200 import dist as D
    from gemm_epilogue_transformer_02_b200 import synth
    ws, r, _ = D.init(backend="gloo", timeout_s=60)
    # each rank draws its own batch
    inp = synth.block_inputs(16, 64, 64, 128, seed=D.rank_seed(1, r), w_std=0.02)
    local_time = 1.0 + r  # rank 1 is the slowest
    D.barrier()
    mx = D.max_over_ranks(local_time)
    val = D.weak_scaling_value(10.0, 4, mx, ws)
    out_q.put((r, float(inp.x.float().sum()), mx, val))
    D.shutdown()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, m0, v0), (r1, s1, m1, v1) = res
    assert (r0, r1) == (0, 1)
    assert s0 != s1                       # independent batches
    assert m0 == m1 == 2.0                # slowest rank's time, on every rank
    assert v0 == v1 == 2 * 10.0 * 4 / 2.0  # all ranks' work over the slowest time


def test_reference_arm_prints_from_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert p.returncode == 0
    assert p.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_line_on_rank0():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "1"], capture_output=True, text=True, env=env, timeout=600)
    assert p.returncode == 0
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    # the same metric and workload config as the GPU arm's line
    sys.path.insert(0, ROOT)
    import bench
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["config"] == bench.arm_config("flush", 1)
