"""Guard regions around every output and workspace of every C-ABI call.

A bounds check that stands in for a memory sanitizer: each output buffer (and
each workspace) is carved out of a larger allocation whose bytes before and
after it are filled with a known pattern; after the call, on ragged shapes
that leave partial tiles in every dimension, the pattern must be intact.  A
store past a tensor-map extent, a row kernel running one row too far, or a
workspace overrun shows up here as a changed guard byte.  The outputs
themselves are compared bit for bit with the same call made on plain buffers
through the binding, so the guarded calls compute the same thing.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 8192     # bytes of pattern on each side (a multiple of 256 keeps alignment)
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` with GUARD pattern bytes on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        self.nbytes = nbytes
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def ptr(self):
        return ctypes.c_void_p(self.t.data_ptr())

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        return bool((head == PATTERN).all().item()) and bool((tail == PATTERN).all().item())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ok(st):
    assert st == 0, C.load_library().coda_status_string(st).decode()


def _all_intact(**bufs):
    bad = [k for k, g in bufs.items() if not g.intact()]
    assert not bad, f"guard bytes changed next to: {bad}"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()
    yield
    C.poll_status()


BF, F32, U8 = torch.bfloat16, torch.float32, torch.uint8


@pytest.mark.parametrize("M,K,N", [(300, 200, 520), (1, 8, 8), (257, 136, 264), (600, 72, 2056)])
def test_first_gemm_reduction_and_second_gemm(M, K, N):
    lib = C.load_library()
    g = synth.make_gen(900 + M)
    x = synth.normal_bf16(g, (M, K)).cuda()
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K)).cuda()
    res = synth.normal_bf16(g, (M, N)).cuda()
    gamma = synth.gamma_bf16(g, N).cuda()
    T = C.partial_cols(N)
    h, hg, part = Guarded((M, N), BF), Guarded((M, N), BF), Guarded((T, M), F32)
    _ok(lib.coda_gemm_res_partialrms(_p(x), _p(W), _p(res), _p(gamma), h.ptr(), hg.ptr(), part.ptr(), M, N, K, _s()))
    _all_intact(h=h, hg=hg, partial=part)
    h0, hg0, p0 = C.gemm_res_partialrms(x, W, res, gamma)
    torch.cuda.synchronize()
    assert torch.equal(h.t, h0) and torch.equal(hg.t, hg0) and torch.equal(part.t, p0)

    r = Guarded((M,), F32)
    _ok(lib.coda_rms_reduce(part.ptr(), M, T, N, 1e-6, r.ptr(), _s()))
    _all_intact(r=r)
    N2 = N + 136
    W2 = synth.normal_bf16(g, (N, N2), std=1 / math.sqrt(N)).cuda()
    out, r2 = Guarded((M, N2), BF), Guarded((M,), F32)
    _ok(lib.coda_gemm_rowscale_partial(hg.ptr(), _p(W2), part.ptr(), T, N, 1e-6, r2.ptr(), out.ptr(), M, N2, N, _s()))
    _all_intact(out=out, r=r2)
    assert torch.equal(r.t, r2.t)
    out3 = Guarded((M, N2), BF)
    _ok(lib.coda_gemm_rowscale(hg.ptr(), _p(W2), r.ptr(), out3.ptr(), M, N2, N, _s()))
    _all_intact(out=out3)
    assert torch.equal(out.t, out3.t)
    C.poll_status()


def test_one_launch_block():
    lib = C.load_library()
    M, K, N, N2 = 300, 136, 520, 392
    inp = synth.block_inputs(M, K, N, N2, seed=901, w_std=0.05)
    x, res, W1, W2, gamma = (t.cuda() for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma))
    T = C.partial_cols(N)
    h, hg, part, r, out = (Guarded((M, N), BF), Guarded((M, N), BF), Guarded((T, M), F32), Guarded((M,), F32),
                           Guarded((M, N2), BF))
    nb = int(lib.coda_rmsnorm_block_workspace_size(M))
    ws = Guarded((max(nb, 16),), U8)
    _ok(lib.coda_rmsnorm_block(_p(x), _p(res), _p(W1), _p(W2), _p(gamma), inp.eps, h.ptr(), hg.ptr(), part.ptr(),
                               r.ptr(), out.ptr(), ws.ptr(), nb, M, K, N, N2, _s()))
    _all_intact(h=h, hg=hg, partial=part, r=r, out=out, ws=ws)
    f = C.gemm_rmsnorm_gemm(x, res, W1, W2, gamma, inp.eps)
    torch.cuda.synchronize()
    assert torch.equal(out.t, f["out"])
    C.poll_status()


def test_swiglu_and_its_backward():
    lib = C.load_library()
    M, K, F, N = 300, 136, 200, 72
    g = synth.make_gen(902)
    A = synth.normal_bf16(g, (M, K)).cuda()
    Wgu = synth.normal_bf16(g, (K, 2 * F), std=1 / math.sqrt(K)).cuda()
    r = (torch.rand(M, generator=g) + 0.5).cuda()
    act, gu = Guarded((M, F), BF), Guarded((M, 2 * F), BF)
    _ok(lib.coda_gemm_swiglu(_p(A), _p(Wgu), _p(r), act.ptr(), gu.ptr(), M, F, K, _s()))
    _all_intact(act=act, gateup=gu)
    act_only = Guarded((M, F), BF)  # the act-only kernel (no gate/up save)
    _ok(lib.coda_gemm_swiglu(_p(A), _p(Wgu), _p(r), act_only.ptr(), None, M, F, K, _s()))
    _all_intact(act_only=act_only)
    torch.cuda.synchronize()
    assert torch.equal(act_only.t, act.t)
    d_out = synth.normal_bf16(g, (M, N)).cuda()
    W_down = synth.normal_bf16(g, (F, N), std=1 / math.sqrt(N)).cuda()
    dgu = Guarded((M, 2 * F), BF)
    _ok(lib.coda_gemm_swiglu_bwd(_p(d_out), _p(W_down), gu.ptr(), dgu.ptr(), M, F, N, _s()))
    _all_intact(d_gateup=dgu)
    ref = C.gemm_swiglu_bwd(d_out, W_down, gu.t.clone())
    torch.cuda.synchronize()
    assert torch.equal(dgu.t, ref)
    C.poll_status()


def test_qkv_rope():
    lib = C.load_library()
    M, K, N, hd, rc = 130, 128, 320, 64, 192
    g = synth.make_gen(903)
    x = synth.normal_bf16(g, (M, K)).cuda()
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K)).cuda()
    pos = torch.randint(0, 4096, (M,), generator=g, dtype=torch.int32).cuda()
    out = Guarded((M, N), BF)
    _ok(lib.coda_gemm_qkv_rope(_p(x), _p(W), _p(pos), out.ptr(), M, N, K, hd, rc, 500000.0, _s()))
    _all_intact(out=out)
    C.poll_status()


def test_lmhead_ce_and_its_backward():
    lib = C.load_library()
    M, K, V = 129, 64, 4104
    g = synth.make_gen(904)
    H = synth.normal_bf16(g, (M, K)).cuda()
    W = synth.normal_bf16(g, (K, V), std=1.5 / math.sqrt(K)).cuda()
    labels = synth.labels_uniform(g, M, V).cuda()
    loss, lse, mean = Guarded((M,), F32), Guarded((M,), F32), Guarded((1,), F32)
    nb = int(lib.coda_lmhead_ce_workspace_size(M, V))
    ws = Guarded((nb,), U8)
    _ok(lib.coda_lmhead_ce(_p(H), _p(W), _p(labels), None, loss.ptr(), lse.ptr(), mean.ptr(), ws.ptr(), nb, M, V, K,
                           _s()))
    _all_intact(loss=loss, lse=lse, mean=mean, ws=ws)
    dH, dW = Guarded((M, K), F32), Guarded((K, V), F32)
    nb2 = int(lib.coda_lmhead_ce_bwd_workspace_size(M, V))
    ws2 = Guarded((nb2,), U8)
    _ok(lib.coda_lmhead_ce_bwd(_p(H), _p(W), _p(labels), lse.ptr(), None, None, dH.ptr(), dW.ptr(), ws2.ptr(), nb2,
                               M, V, K, _s()))
    _all_intact(dH=dH, dW=dW, ws=ws2)
    dH0, dW0 = C.lmhead_ce_bwd(H, W, labels, lse.t.clone())
    torch.cuda.synchronize()
    assert torch.equal(dH.t, dH0) and torch.equal(dW.t, dW0)
    C.poll_status()


def test_block_backward_calls():
    lib = C.load_library()
    M, N, N2, K = 300, 520, 392, 136
    g = synth.make_gen(905)
    dOut = synth.normal_bf16(g, (M, N2), std=0.5).cuda()
    hg = synth.normal_bf16(g, (M, N)).cuda()
    h = synth.normal_bf16(g, (M, N)).cuda()
    W2 = synth.normal_bf16(g, (N, N2), std=1 / math.sqrt(N)).cuda()
    gamma = synth.gamma_bf16(g, N).cuda()
    r = (torch.rand(M, generator=g) + 0.5).cuda()
    T = C.partial_cols(N)
    d_hg, dW2, pdr = Guarded((M, N), F32), Guarded((N, N2), F32), Guarded((T, M), F32)
    nb = int(lib.coda_gemm_rowscale_bwd_workspace_size(M, N))
    ws = Guarded((nb,), U8)
    _ok(lib.coda_gemm_rowscale_bwd(_p(dOut), _p(hg), _p(W2), _p(r), d_hg.ptr(), dW2.ptr(), pdr.ptr(), ws.ptr(), nb,
                                   M, N, N2, _s()))
    _all_intact(d_hg=d_hg, dW2=dW2, pdr=pdr, ws=ws)
    dh, dgamma = Guarded((M, N), BF), Guarded((N,), F32)
    nb2 = int(lib.coda_rms_reduce_bwd_workspace_size(M, N))
    ws2 = Guarded((nb2,), U8)
    _ok(lib.coda_rms_reduce_bwd(pdr.ptr(), _p(r), d_hg.ptr(), _p(h), _p(gamma), dh.ptr(), dgamma.ptr(), ws2.ptr(),
                                nb2, M, T, N, _s()))
    _all_intact(dh=dh, dgamma=dgamma, ws=ws2)
    x = synth.normal_bf16(g, (M, K)).cuda()
    W1 = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K)).cuda()
    dx, dW1 = Guarded((M, K), BF), Guarded((K, N), F32)
    _ok(lib.coda_gemm_res_partialrms_bwd(dh.ptr(), _p(x), _p(W1), dx.ptr(), dW1.ptr(), M, N, K, _s()))
    _all_intact(dx=dx, dW1=dW1)
    dx0, dW10 = C.gemm_res_partialrms_bwd(dh.t.clone(), x, W1)
    torch.cuda.synchronize()
    assert torch.equal(dx.t, dx0) and torch.equal(dW1.t, dW10)
    C.poll_status()


def test_backward_gemms_split_by_k():
    """The long-K backward GEMMs whose last wave splits by k-blocks zero part
    of their outputs with 2-D memsets before adding into them: the guard
    bytes around d_hg, pdr and dW1 stay intact, and the guarded call equals
    the plain one bit for bit."""
    lib = C.load_library()
    M, N, N2 = 300, 136, 4104
    g = synth.make_gen(907)
    dOut = synth.normal_bf16(g, (M, N2), std=0.5).cuda()
    hg = synth.normal_bf16(g, (M, N)).cuda()
    W2 = synth.normal_bf16(g, (N, N2), std=1 / math.sqrt(N)).cuda()
    r = (torch.rand(M, generator=g) + 0.5).cuda()
    T = C.partial_cols(N)
    d_hg, dW2, pdr = Guarded((M, N), F32), Guarded((N, N2), F32), Guarded((T, M), F32)
    nb = int(lib.coda_gemm_rowscale_bwd_workspace_size(M, N))
    ws = Guarded((nb,), U8)
    _ok(lib.coda_gemm_rowscale_bwd(_p(dOut), _p(hg), _p(W2), _p(r), d_hg.ptr(), dW2.ptr(), pdr.ptr(), ws.ptr(), nb,
                                   M, N, N2, _s()))
    _all_intact(d_hg=d_hg, dW2=dW2, pdr=pdr, ws=ws)
    d_hg0, dW20, pdr0 = C.gemm_rowscale_bwd(dOut, hg, W2, r)
    torch.cuda.synchronize()
    assert torch.equal(d_hg.t, d_hg0) and torch.equal(pdr.t, pdr0) and torch.equal(dW2.t, dW20)
    Mt, K, Nw = 4171, 64, 136
    dh = synth.normal_bf16(g, (Mt, Nw)).cuda()
    x = synth.normal_bf16(g, (Mt, K)).cuda()
    W1 = synth.normal_bf16(g, (K, Nw), std=1 / math.sqrt(K)).cuda()
    dW1 = Guarded((K, Nw), F32)
    _ok(lib.coda_gemm_res_partialrms_bwd(_p(dh), _p(x), _p(W1), None, dW1.ptr(), Mt, Nw, K, _s()))
    _all_intact(dW1=dW1)
    _, dW10 = C.gemm_res_partialrms_bwd(dh, x, W1, dx=False)
    torch.cuda.synchronize()
    assert torch.equal(dW1.t, dW10)
    C.poll_status()


def test_fp8_block_and_unfused_pieces():
    lib = C.load_library()
    M, K, N, N2 = 333, 272, 784, 400
    inp = synth.block_inputs(M, K, N, N2, seed=906, w_std=0.04)
    x, res, W1, W2, gamma = (t.cuda() for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma))
    x8, amax, sx = Guarded((M, K), U8), Guarded((1,), F32), Guarded((1,), F32)
    _ok(lib.coda_fp8_quantize(_p(x), M, K, 0, x8.ptr(), amax.ptr(), sx.ptr(), _s()))
    _all_intact(codes=x8, amax=amax, scale=sx)
    W1t8, a1, sw1 = Guarded((N, K), U8), Guarded((1,), F32), Guarded((1,), F32)
    _ok(lib.coda_fp8_quantize(_p(W1), K, N, 1, W1t8.ptr(), a1.ptr(), sw1.ptr(), _s()))
    _all_intact(codes_t=W1t8, amax=a1, scale=sw1)
    W2t8, _, sw2 = C.fp8_quantize(W2, transpose=True)
    s_hg = torch.ones(1, dtype=torch.float32, device="cuda")
    T = C.partial_cols(N)
    h, hg8, am, part = Guarded((M, N), BF), Guarded((M, N), U8), Guarded((1,), F32), Guarded((T, M), F32)
    _ok(lib.coda_gemm_res_partialrms_fp8(x8.ptr(), sx.ptr(), W1t8.ptr(), sw1.ptr(), _p(res), _p(gamma), _p(s_hg),
                                         h.ptr(), hg8.ptr(), am.ptr(), part.ptr(), M, N, K, _s()))
    _all_intact(h=h, hg8=hg8, amax=am, partial=part)
    out, r = Guarded((M, N2), BF), Guarded((M,), F32)
    _ok(lib.coda_gemm_rowscale_partial_fp8(hg8.ptr(), _p(s_hg), _p(W2t8), _p(sw2), part.ptr(), T, N, 1e-6, r.ptr(),
                                           out.ptr(), M, N2, N, _s()))
    _all_intact(out=out, r=r)
    t8 = Guarded((M, N), BF)
    _ok(lib.coda_gemm_fp8(x8.ptr(), sx.ptr(), W1t8.ptr(), sw1.ptr(), t8.ptr(), M, N, K, _s()))
    _all_intact(out=t8)
    s = Guarded((M, N), BF)
    _ok(lib.coda_unfused_add(_p(t8.t), _p(res), s.ptr(), M * N, _s()))
    _all_intact(sum=s)
    y, r3 = Guarded((M, N), BF), Guarded((M,), F32)
    _ok(lib.coda_unfused_rmsnorm(s.ptr(), _p(gamma), 1e-6, y.ptr(), r3.ptr(), M, N, _s()))
    _all_intact(y=y, r=r3)
    y8, am2, r4 = Guarded((M, N), U8), Guarded((1,), F32), Guarded((M,), F32)
    _ok(lib.coda_unfused_rmsnorm_fp8(s.ptr(), _p(gamma), 1e-6, _p(s_hg), y8.ptr(), am2.ptr(), r4.ptr(), M, N, _s()))
    _all_intact(y8=y8, amax=am2, r=r4)
    C.poll_status()
