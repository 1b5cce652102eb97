"""Parity of the QKV projection with RoPE in its epilogue against the fp64 oracle.

Source: KuCoin news flash "CODA: new research optimizes transformer training
with GEMM epilogue programming", section "CODA: the secret in the epilogue"
(RoPE takes the same re-parameterisation as RMSNorm and SwiGLU).  Workload of
the 1B model's attention input: 8192 tokens (batch 4 x sequence 2048), hidden
2048, 32 query heads and 8 key/value heads of dimension 64, theta 500000,
positions = token index within its sequence.
"""
import math

import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import b, check, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


@pytest.mark.parametrize("M,K,dh,nq,nkv", [(300, 136, 64, 5, 2), (257, 256, 128, 3, 1), (130, 64, 64, 4, 4)])
def test_qkv_rope_small(M, K, dh, nq, nkv):
    g = synth.make_gen(700 + M)
    N = (nq + 2 * nkv) * dh
    rope_cols = (nq + nkv) * dh
    x = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    pos = torch.randint(0, 8192, (M,), generator=g, dtype=torch.int32)
    out = C.gemm_qkv_rope(dev(x), dev(W), dev(pos), dh, rope_cols, theta=500000.0)
    ref = O.qkv_rope_unfused(b(x), b(W), pos.numpy(), dh, rope_cols, 500000.0)
    check("qkv", out, ref)
    check("v (unrotated)", out[:, rope_cols:], O.matmul(b(x), b(W))[:, rope_cols:])


def test_qkv_rope_llama1b_sampled_rows():
    M, K, dh, nq, nkv = 8192, 2048, 64, 32, 8
    N, rope_cols = (nq + 2 * nkv) * dh, (nq + nkv) * dh
    g = synth.make_gen(8)
    x = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, N), std=0.02)
    pos = (torch.arange(M, dtype=torch.int32) % 2048)
    out = C.gemm_qkv_rope(dev(x), dev(W), dev(pos), dh, rope_cols)
    C.poll_status()
    rows = np.sort(np.concatenate([[0, 2047, 2048, M - 1], np.random.default_rng(9).choice(M, 28, replace=False)]))
    ref = O.qkv_rope_unfused(b(x)[rows], b(W), pos.numpy()[rows], dh, rope_cols, 500000.0)
    check("qkv (sampled rows)", out[torch.as_tensor(rows, device="cuda")], ref)
