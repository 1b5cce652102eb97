"""The N > 1 path on CPU: two gloo ranks, no GPU.

Covers what bench.py does across ranks: per-rank seeds (independent batches),
the max over ranks of the timed region, the whole-job weak-scaling value, and
that the reference arm prints from rank 0 only.  And the data-parallel
backward and cross-entropy of dist.py: each rank runs its half of the token
rows through the same call sequence, with the fp64 oracle standing in for the
library's kernels (the GPU runs them through the binding), and the gradients
summed over the two ranks must equal the oracle's full-batch backward.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
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


class _OracleOps:
    """The binding's call signatures, computed by the fp64 oracle on CPU tensors
    (test stand-in for the library's kernels on a machine without a GPU)."""

    def __init__(self, tile):
        from oracle import coda_oracle as O
        self.O, self.tile = O, tile

    @staticmethod
    def _t(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))

    def gemm_rowscale_bwd(self, dOut, hg, W2, r):
        d = self.O.gemm_rowscale_bwd(dOut.numpy(), hg.numpy(), W2.numpy(), r.numpy(), self.tile)
        return self._t(d["d_hg"]), self._t(d["dW2"]), self._t(d["pdr"])

    def rms_reduce_bwd(self, pdr, r, d_hg, h, gamma):
        d = self.O.rms_reduce_bwd(pdr.numpy(), r.numpy(), d_hg.numpy(), h.numpy(), gamma.numpy())
        return self._t(d["dh"]), self._t(d["dgamma"])

    def gemm_res_partialrms_bwd(self, dh, x, W1):
        d = self.O.gemm_res_partialrms_bwd(dh.numpy(), x.numpy(), W1.numpy())
        return self._t(d["dx"]), self._t(d["dW1"])

    def lmhead_ce(self, H, W, labels):
        d = self.O.lmhead_ce(H.numpy(), W.numpy(), labels.numpy())
        return self._t(d["loss"]), self._t(d["lse"]), self._t([d["mean"]])

    def loss_stats(self, loss):
        return self._t([float(loss.sum()), float(loss.numel())])

    def ce_global_finish(self, stats, M):
        s, c = float(stats[0]), float(stats[1])
        return self._t([s / c]), self._t(np.full(M, 1.0 / c))

    def lmhead_ce_bwd(self, H, W, labels, lse, d_loss=None):
        d = self.O.lmhead_ce_bwd(H.numpy(), W.numpy(), labels.numpy(), lse.numpy(), d_loss=d_loss.numpy(),
                                 chunk_cols=48)
        return self._t(d["dH"]), self._t(d["dW"])


def _dp_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from gemm_epilogue_transformer_02_b200 import dist as D
    from gemm_epilogue_transformer_02_b200 import synth
    from oracle import coda_oracle as O
    D.init(backend="gloo", timeout_s=60)
    ops = _OracleOps(tile=16)
    M, K, N, N2, V = 24 * world, 16, 40, 24, 100
    inp = synth.block_inputs(M, K, N, N2, seed=77, w_std=0.2)  # the same full batch on every rank
    f64 = lambda t: torch.from_numpy(O.bf16_to_f64(synth.bf16_bits(t)))
    x, res, W1, W2, gamma = (f64(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma))
    dOut = f64(synth.block_backward_dout(M, N2, seed=78, std=0.5))
    rows = slice(rank * M // world, (rank + 1) * M // world)
    # this rank's forward state (h, hg, r) for its rows
    fw = O.rmsnorm_block_reparam(x[rows].numpy(), res[rows].numpy(), W1.numpy(), W2.numpy(), gamma.numpy(), 1e-6,
                                 tile_cols=16)
    fwd = {k: torch.from_numpy(np.asarray(fw[k], dtype=np.float64)) for k in ("h", "hg", "r")}
    g = D.block_backward_dp(ops, dOut[rows], x[rows], W1, W2, gamma, fwd)
    # cross-entropy over the same split
    rng = np.random.default_rng(5)
    H = torch.from_numpy(rng.normal(size=(M, K)))
    Wv = torch.from_numpy(rng.normal(size=(K, V)) * 0.3)
    labels = torch.from_numpy(rng.integers(0, V, size=M))
    loss, lse, mean, d_loss = D.lmhead_ce_dp(ops, H[rows], Wv, labels[rows])
    dH, dWv = D.lmhead_ce_bwd_dp(ops, H[rows], Wv, labels[rows], lse, d_loss)
    out_q.put((rank, {k: g[k].numpy() for k in ("dW1", "dW2", "dgamma", "dx", "dres")}, float(mean[0]),
               dH.numpy(), dWv.numpy()))
    D.shutdown()


def test_two_gloo_ranks_data_parallel_backward_and_cross_entropy():
    from gemm_epilogue_transformer_02_b200 import synth
    from oracle import coda_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # full-batch oracle
    M, K, N, N2, V = 24 * world, 16, 40, 24, 100
    inp = synth.block_inputs(M, K, N, N2, seed=77, w_std=0.2)
    bits = [synth.bf16_bits(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    dOut = synth.bf16_bits(synth.block_backward_dout(M, N2, seed=78, std=0.5))
    ref = O.rmsnorm_block_backward_unfused(*bits, 1e-6, dOut)
    for rank, g, *_ in res:
        for k in ("dW1", "dW2", "dgamma"):   # summed over ranks: the full batch's
            np.testing.assert_allclose(g[k], ref[k], rtol=1e-10, atol=1e-12)
        rows = slice(rank * M // world, (rank + 1) * M // world)
        for k in ("dx", "dres"):              # per rank: its own rows
            np.testing.assert_allclose(g[k], ref[k][rows], rtol=1e-10, atol=1e-12)
    rng = np.random.default_rng(5)
    H = rng.normal(size=(M, K))
    Wv = rng.normal(size=(K, V)) * 0.3
    labels = rng.integers(0, V, size=M)
    cref = O.cross_entropy_unfused(H, Wv, labels)
    gref = O.cross_entropy_backward_unfused(H, Wv, labels)
    for rank, _, mean, dH, dWv in res:
        assert abs(mean - cref["loss"].mean()) <= 1e-12 * abs(cref["loss"].mean())
        rows = slice(rank * M // world, (rank + 1) * M // world)
        np.testing.assert_allclose(dH, gref["dH"][rows], rtol=1e-10, atol=1e-13)
        np.testing.assert_allclose(dWv, gref["dW"], rtol=1e-10, atol=1e-13)
