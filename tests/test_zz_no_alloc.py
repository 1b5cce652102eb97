"""The allocation-free RMSNorm backward entry point against the regular one.

coda_rms_reduce_bwd_noalloc serves callers that cannot allocate device memory
at call time (a fixed device-memory budget after start-up, or a framework that
owns all device memory and cannot hand out a workspace).  It keeps its scratch
in a static device array inside the library instead of a caller workspace.
These tests call both entry points through the C ABI on the same inputs, twice
in a row with different sizes, and compare the outputs.  The file is named so
that pytest collects it last; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from tests._util import check

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 4


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


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    for M, N, seed in ((300, 520, 1), (8192, 2048, 2)):
        args = _inputs(M, N, seed)
        dh_ref, dgamma_ref = C.rms_reduce_bwd(*args)      # caller-allocated workspace
        dh, dgamma = _noalloc(*args)                      # library's static scratch
        torch.cuda.synchronize()
        check("noalloc dh", dh, dh_ref.double().cpu().numpy())
        check("noalloc dgamma", dgamma, dgamma_ref.double().cpu().numpy())
    C.poll_status()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = C.load_library()
    x = torch.zeros(16, dtype=torch.float32, device="cuda")
    # ceil(32768 / 32) * 2048 = 2^21 floats > 2^20
    st = lib.coda_rms_reduce_bwd_noalloc(_p(x), _p(x), _p(x), _p(x), _p(x), _p(x), _p(x), 32768, 8, 2048,
                                         ctypes.c_void_p(0))
    assert st == WORKSPACE_ERR
