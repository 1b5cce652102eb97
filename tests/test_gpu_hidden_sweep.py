"""The fused block at larger model widths (sampled rows against the fp64 oracle).

The article's single-operator comparison of GEMM-RMSNorm-GEMM is made at the
hidden sizes of 1B, 7B and 70B models (KuCoin news flash "CODA: new research
optimizes transformer training with GEMM epilogue programming", section
"Experimental results"); it gives no dimensions, so LLaMA-3-style widths are
used: hidden 4096 with fused gate/up 28672, and hidden 8192 with 57344, on
8192 tokens, weights N(0, 0.02).
"""
import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import b, check, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,n2", [(4096, 28672), (8192, 57344)])
def test_block_at_larger_hidden_sizes(d, n2):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    M = 8192
    inp = synth.block_inputs(M, d, d, n2, seed=50 + d // 1024, w_std=0.02)
    dd = [dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    f = C.gemm_rmsnorm_gemm(*dd, inp.eps)
    C.poll_status()
    rows = np.sort(np.concatenate([[0, M - 1], np.random.default_rng(d).choice(np.arange(1, M - 1), 6,
                                                                                  replace=False)]))
    ref = O.rmsnorm_block_unfused(b(inp.x)[rows], b(inp.res)[rows], b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    ri = torch.as_tensor(rows, device="cuda")
    check("out", f["out"][ri], ref["out"])
    check("h", f["h"][ri], ref["h"])
