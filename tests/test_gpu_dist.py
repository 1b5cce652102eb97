"""The data-parallel calls of dist.py on one GPU, through NCCL.

A one-rank NCCL process group runs every collective of the data-parallel
backward and cross-entropy (each an identity on one rank), so the device
buffers, streams and call order of the multi-GPU path are exercised here; the
sums over ranks themselves are tested with two gloo ranks on CPU.  With one
rank the results must equal the single-GPU calls bit for bit.
"""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import dist as D
from gemm_epilogue_transformer_02_b200 import synth

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def group():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


def test_block_backward_dp_equals_single_gpu(group):
    inp = synth.block_inputs(300, 136, 520, 392, seed=24, w_std=0.05)
    d = [t.cuda() for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    dOut = synth.block_backward_dout(300, 392, seed=25, std=0.01).cuda()
    f = C.gemm_rmsnorm_gemm(*d, inp.eps)
    ref = C.block_backward(dOut, d[0], d[2], d[3], d[4], f)
    got = D.block_backward_dp(C, dOut, d[0], d[2], d[3], d[4], f)
    torch.cuda.synchronize()
    for k in ("dW2", "dgamma", "dres", "dx", "dW1"):
        assert torch.equal(got[k], ref[k]), k
    C.poll_status()


def test_cross_entropy_dp_equals_single_gpu(group):
    g = synth.make_gen(41)
    M, K, V = 300, 136, 1000
    H = synth.normal_bf16(g, (M, K)).cuda()
    W = synth.normal_bf16(g, (K, V), std=1.5 / K ** 0.5).cuda()
    labels = synth.labels_uniform(g, M, V).cuda()
    loss0, lse0, mean0 = C.lmhead_ce(H, W, labels)
    loss, lse, mean, d_loss = D.lmhead_ce_dp(C, H, W, labels)
    torch.cuda.synchronize()
    assert torch.equal(loss, loss0) and torch.equal(lse, lse0)
    assert torch.equal(mean, mean0)                      # the same fixed-order sum, divided by M
    assert torch.equal(d_loss, torch.full((M,), 1.0 / M, dtype=torch.float32, device="cuda"))
    stats = C.loss_stats(loss)
    torch.cuda.synchronize()
    assert float(stats[1]) == M
    dH0, dW0 = C.lmhead_ce_bwd(H, W, labels, lse)      # d_loss = 1/M inside the call
    dH, dW = D.lmhead_ce_bwd_dp(C, H, W, labels, lse, d_loss)
    torch.cuda.synchronize()
    assert torch.equal(dH, dH0) and torch.equal(dW, dW0)
    C.poll_status()
