"""The one-launch GEMM-RMSNorm-GEMM block (coda_rmsnorm_block).

It must produce exactly what the two-launch path produces (the same
arithmetic: first-GEMM epilogue, then the second GEMM with the light
reduction in its epilogue) and match the fp64 oracle, on the tiny workload,
on ragged shapes (partial row blocks, a partial last column tile) and on the
1B block tail; calling it twice must give the same result (its completion
counters are reset on every call).
"""
import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import b, check, check_rel, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


def _both(inp):
    d = [dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    one = C.gemm_rmsnorm_gemm(*d, inp.eps, launches=1)
    one = {k: v.clone() for k, v in one.items()}
    two = C.gemm_rmsnorm_gemm(*d, inp.eps, launches=2)
    C.poll_status()
    return d, one, two


@pytest.mark.parametrize("shape", [(256, 512, 512, 1536), (333, 264, 776, 392), (1000, 512, 1024, 2048)])
def test_one_launch_block_equals_two_launch_and_oracle(shape):
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.block_inputs(M, K, N, N2, seed=40 + M, w_std=0.04)
    d, one, two = _both(inp)
    for k in ("out", "h", "hg", "partial", "r"):
        assert torch.equal(one[k], two[k]), k
    ref = O.rmsnorm_block_unfused(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    check("out", one["out"], ref["out"])
    check("h", one["h"], ref["h"])
    check_rel("r", one["r"], ref["r"], 1e-3)
    again = C.gemm_rmsnorm_gemm(*d, inp.eps, launches=1)
    assert torch.equal(again["out"], one["out"])


def test_one_launch_block_tail_full_size():
    inp = synth.llama1b_block_tail(with_down=False)
    d, one, two = _both(inp)
    for k in ("out", "h", "hg", "r"):
        assert torch.equal(one[k], two[k]), k
    rows = np.sort(np.concatenate([[0, 8191], np.random.default_rng(41).choice(8192, 22, replace=False)]))
    ref = O.rmsnorm_block_unfused(b(inp.x)[rows], b(inp.res)[rows], b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    check("out (sampled rows)", one["out"][torch.as_tensor(rows, device="cuda")], ref["out"])
