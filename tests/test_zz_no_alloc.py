"""The allocation-free RMSNorm backward entry point against the regular one.

coda_rms_reduce_bwd_noalloc serves callers that cannot allocate device memory
at call time (a fixed device-memory budget after start-up, or a framework that
owns all device memory and cannot hand out a workspace).  It keeps its scratch
in a static device array inside the library instead of a caller workspace.
These tests call both entry points through the C ABI on the same inputs, several
times in a row with sizes that shrink and grow, and require identical outputs.
(Sizes beyond the array are rejected before any launch; that is tested on the
host, without a device.)  The file is named so that pytest collects it last;
it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(M, N, seed):
    g = synth.make_gen(seed)
    T = C.partial_cols(N)
    pdr = (torch.randn(T, M, generator=g) * 5).cuda()
    r = (torch.rand(M, generator=g) + 0.5).cuda()
    d_hg = torch.randn(M, N, generator=g).cuda()
    h = synth.normal_bf16(g, (M, N)).cuda()
    gamma = synth.gamma_bf16(g, N).cuda()
    return pdr, r, d_hg, h, gamma


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(pdr, r, d_hg, h, gamma):
    lib = C.load_library()
    T, M = pdr.shape
    N = h.shape[1]
    dh = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dgamma = torch.empty(N, dtype=torch.float32, device="cuda")
    st = lib.coda_rms_reduce_bwd_noalloc(_p(pdr), _p(r), _p(d_hg), _p(h), _p(gamma), _p(dh), _p(dgamma), M, T, N,
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.coda_status_string(st).decode()
    return dh, dgamma


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row():
    """Large, small, large, small: each call leaves its partials in the shared
    array, and a later call over a smaller or differently shaped problem must
    not read any of them.  Both entry points run the same kernels on the same
    inputs, so their outputs must be identical bit for bit."""
    for M, N, seed in ((8192, 2048, 2), (300, 520, 1), (8192, 2048, 3), (1000, 776, 4)):
        args = _inputs(M, N, seed)
        dh_ref, dgamma_ref = C.rms_reduce_bwd(*args)      # caller-allocated workspace
        dh, dgamma = _noalloc(*args)                      # library's static scratch
        torch.cuda.synchronize()
        assert torch.equal(dh, dh_ref), (M, N)
        assert torch.equal(dgamma, dgamma_ref), (M, N)
    C.poll_status()
