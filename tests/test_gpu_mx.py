"""Parity of the MXFP8 (block-scaled e4m3) block and its quantiser with the
fp64 oracle.

The KuCoin news flash "CODA: new research optimizes transformer training with
GEMM epilogue programming" (section "The lazy cost of training large
models") names low-precision formats as the reason the non-GEMM share of
training time grows; the microscaled variant quantises hg block by block in
the first GEMM's epilogue.  What is compared:

* the quantiser bit for bit (codes and the tiled scale bytes, padding included);
* the block-scaled GEMM exactly on small-integer data, where every product
  and partial sum is exact in fp32, so that any misplaced scale shows as a
  factor of two; and at the usual bar on random data;
* the first GEMM's MXFP8 output exactly where its fp32 values are exact
  (small-integer operands), else scale by scale and code by code (a scale may
  differ by one where the fp32 and fp64 block maxima straddle a power of
  two, a code by one step at a rounding boundary);
* the block's floating-point outputs against the oracle at the usual bar,
  the second GEMM fed the GPU's own MXFP8 hg (the step) and the whole block
  against the oracle's composition (the chain).
"""
import ctypes

import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from oracle import coda_oracle_fp8 as F8
from oracle import coda_oracle_mx as MX
from tests._util import b, check, check_rel, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


def _exps(sf, R, K, operand=0):
    return MX.sf_untile(sf.cpu().numpy(), R, K, operand)


def _check_sf_bytes(sf, exps, R, operand):
    """The scale buffer byte for byte where the layout defines bytes
    (bytes of an A image that no scale maps to are never read)."""
    want, used = MX.sf_tile(exps, R, operand)
    got = sf.cpu().numpy()
    assert got.shape == want.shape
    np.testing.assert_array_equal(got[used], want[used])


def _same_sf(a, b, R, K, operand=0):
    """Two scale buffers equal where the layout defines bytes."""
    used = MX.sf_tile(np.zeros((R, K // 32), dtype=np.int64), R, operand)[1]
    return bool(np.array_equal(a.cpu().numpy()[used], b.cpu().numpy()[used]))


@pytest.mark.parametrize("rows,cols,operand", [(300, 384, 0), (300, 384, 1), (1, 128, 0), (1, 128, 1),
                                               (128, 256, 1), (257, 1152, 0), (257, 1024, 1)])
def test_mx_quantize_bit_exact(rows, cols, operand):
    g = synth.make_gen(1200 + rows + cols)
    t = synth.normal_bf16(g, (rows, cols), std=1.0).float()
    mag = torch.exp2(torch.randint(-24, 24, (rows, 1), generator=g).float())
    t = (t * mag).to(torch.bfloat16)
    t[0, :64] = 0.0                      # block 0 all zero: scale 1
    t[0, 32:35] = torch.tensor([448.0, -452.0, 1.0])  # block 1 just above a power-of-two boundary: 2^1
    if rows > 1:
        t[1, :32] = 0.0
        t[1, :2] = torch.tensor([448.0, -3.5])          # exactly at the boundary: scale 1
    q, sf = C.mx_quantize(dev(t), operand)
    C.poll_status()
    wq, we = MX.mx_quantize(O.bf16_to_f64(b(t)))
    np.testing.assert_array_equal(q.cpu().numpy(), wq)
    _check_sf_bytes(sf, we, rows, operand)
    assert int(we[0, 1]) == 1 and (rows == 1 or int(we[1, 0]) == 0)


def _small_int_mx(rng, R, K, vals, erange):
    codes = F8.e4m3_encode(rng.choice(vals, (R, K)))
    exps = rng.integers(erange[0], erange[1] + 1, (R, K // 32))
    return codes, exps


def _to_dev(codes, exps, R, operand):
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
            torch.from_numpy(MX.sf_tile(exps, R, operand)[0]).cuda())


@pytest.mark.parametrize("M,N,K", [(300, 384, 512), (256, 256, 128), (77, 640, 256)])
def test_mx_gemm_exact_small_integers(M, N, K):
    """Codes 0, +-0.5, +-1 and block exponents -2..2: every product is a
    multiple of 2^-6 below 2^4 in magnitude and every partial sum stays below
    2^15 of those units, so fp32 accumulation is exact whatever its order and
    the output is the exact sum rounded once to bf16.  A scale taken from the
    wrong row, block or operand changes values by factors of 2 to 16."""
    rng = np.random.default_rng(M + N + K)
    vals = [0.0, 0.5, 1.0, -0.5, -1.0]
    aq, ae = _small_int_mx(rng, M, K, vals, (-2, 2))
    bq, be = _small_int_mx(rng, N, K, vals, (-2, 2))
    A, Asf = _to_dev(aq, ae, M, 0)
    W, Wsf = _to_dev(bq, be, N, 1)
    out, r = C.gemm_rowscale_partial_mx(A, Asf, W, Wsf)
    C.poll_status()
    assert r is None
    exact = MX.gemm_rowscale_partial_mx(aq, ae, bq, be)["out"]
    np.testing.assert_array_equal(out.double().cpu().numpy(), F8.round_bf16(exact))


@pytest.mark.parametrize("M,N,K", [(300, 384, 512), (1, 256, 128), (520, 1152, 640)])
def test_mx_gemm_with_folded_row_scale(M, N, K):
    g = synth.make_gen(1300 + M)
    a = synth.normal_bf16(g, (M, K), std=2.0)
    w = synth.normal_bf16(g, (N, K), std=0.05)
    A, Asf = C.mx_quantize(dev(a), C.MX_A)
    W, Wsf = C.mx_quantize(dev(w), C.MX_B)
    T = 6
    partial = torch.rand((T, M), generator=g).mul(50.0).cuda()
    out, r = C.gemm_rowscale_partial_mx(A, Asf, W, Wsf, partial, 700, 1e-5)
    C.poll_status()
    ref = MX.gemm_rowscale_partial_mx(A.cpu().numpy(), _exps(Asf, M, K), W.cpu().numpy(), _exps(Wsf, N, K, 1),
                                      partial.double().cpu().numpy(), 700, 1e-5)
    check_rel("r", r, ref["r"], 1e-6)
    # random partials spread r over a decade, so the largest outputs sit far
    # out in the tail: held to the bar with the bf16 storage allowance
    check("out", out, ref["out"])


def _mx_inputs(inp):
    """Per-tensor e4m3 x and W1 (the FP8 block's quantiser), MXFP8 W2 (W2
    stored transposed); the GPU's and the oracle's quantisations asserted
    equal."""
    xd, W1d = dev(inp.x), dev(inp.W1)
    W2t = dev(inp.W2.t().contiguous())
    x8, _, sx = C.fp8_quantize(xd)
    W1t8, _, sw1 = C.fp8_quantize(W1d, transpose=True)
    W2q, W2sf = C.mx_quantize(W2t, C.MX_B)
    vx = O.bf16_to_f64(b(inp.x))
    vw1 = O.bf16_to_f64(b(inp.W1)).T
    osx, osw1 = F8.quant_scale(np.abs(vx).max()), F8.quant_scale(np.abs(vw1).max())
    ox8 = F8.quantize(vx.astype(np.float32), osx)
    oW1 = F8.quantize(vw1.astype(np.float32), osw1)
    oW2q, oW2e = MX.mx_quantize(O.bf16_to_f64(b(inp.W2)).T)
    np.testing.assert_array_equal(x8.cpu().numpy(), ox8)
    np.testing.assert_array_equal(W1t8.cpu().numpy(), oW1)
    np.testing.assert_array_equal(W2q.cpu().numpy(), oW2q)
    N2, N = W2q.shape
    np.testing.assert_array_equal(_exps(W2sf, N2, N, 1), oW2e)
    assert np.float32(sx.item()) == osx and np.float32(sw1.item()) == osw1
    gpu = dict(x8=x8, sx=sx, W1t8=W1t8, sw1=sw1, W2q=W2q, W2sf=W2sf)
    ora = dict(x8=ox8, sx=float(osx), W1t8=oW1, sw1=float(osw1), W2q=oW2q, W2e=oW2e)
    return gpu, ora


def _check_mx_output(name, hq, he, hg_ref, max_frac=2e-3):
    """The GPU's MXFP8 hg against the oracle's fp64 hg (computed from the
    same operands in another order): each block's scale is the oracle's,
    except where the block maximum lies within a hair of 448 * 2^e; each
    code equals the oracle's encoding of the value under the GPU's scale,
    or is one e4m3 step from it."""
    hq = np.asarray(hq)
    he = np.asarray(he)
    R, K = hq.shape
    amax = np.abs(hg_ref).reshape(R, K // 32, 32).max(axis=2)
    oe = MX.mx_exponent(amax)
    bad = he != oe
    assert bad.mean() <= max_frac, f"{name}: {bad.mean():.2e} of the scales differ"
    if bad.any():
        near = np.abs(amax[bad] / (448.0 * np.ldexp(1.0, np.minimum(he[bad], oe[bad]))) - 1.0)
        assert np.all(near < 1e-3), f"{name}: a scale differs away from a power-of-two boundary"
    want = F8.e4m3_encode(hg_ref * np.repeat(np.ldexp(1.0, -he.astype(np.int64)), 32, axis=1))
    diff = hq != want
    assert diff.mean() <= max_frac, f"{name}: {diff.mean():.2e} of the codes differ"
    if diff.any():
        dg, dw = F8.e4m3_decode(hq[diff]), F8.e4m3_decode(want[diff])
        step = 2.0 ** -3 * np.maximum(np.abs(dg), np.abs(dw)) + 2.0 ** -9
        assert np.all(np.abs(dg - dw) <= step), f"{name}: codes more than one step apart"


def test_mx_first_gemm_exact_small_integers():
    """x8 and W1t8 codes 0, +-1, +-2 with unit scales, res and gamma small
    powers of two: h and gamma * h are exact in fp32, so the epilogue's MXFP8
    hg must equal the oracle's bit for bit (scales and codes)."""
    M, N, K = 300, 384, 256
    rng = np.random.default_rng(12)
    x8 = F8.e4m3_encode(rng.choice([0.0, 1.0, -1.0, 2.0, -2.0], (M, K)))
    w8 = F8.e4m3_encode(rng.choice([0.0, 1.0, -1.0, 0.5], (N, K)))
    res = rng.choice([0.0, 0.25, -3.0, 64.0], (M, N))
    gamma = rng.choice([1.0, 0.5, 2.0, 0.125], N)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    bf = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).cuda()
    h, hq, hsf, part = C.gemm_res_partialrms_mx(torch.from_numpy(x8).cuda(), one, torch.from_numpy(w8).cuda(), one,
                                                bf(res), bf(gamma))
    C.poll_status()
    ref = MX.gemm_res_partialrms_mx(x8, 1.0, w8, 1.0, res, gamma, tile_cols=C.partial_tile_width())
    np.testing.assert_array_equal(hq.cpu().numpy(), ref["hq"])
    _check_sf_bytes(hsf, ref["he"], M, 0)
    check("h", h, ref["h"], strict=True)
    check("partial", part, ref["partial"], rel=1e-6)


@pytest.mark.parametrize("shape", [(256, 512, 512, 1536), (333, 272, 768, 384), (130, 1040, 256, 256)])
def test_mx_block_small(shape):
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.block_inputs(M, K, N, N2, seed=90 + M, w_std=0.04)
    gpu, ora = _mx_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    f = C.gemm_rmsnorm_gemm_mx(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                               gpu["W2q"], gpu["W2sf"], inp.eps)
    C.poll_status()
    ref = MX.rmsnorm_block_mx(ora["x8"], ora["sx"], ora["W1t8"], ora["sw1"], res, gamma, ora["W2q"], ora["W2e"],
                              inp.eps, tile_cols=C.partial_tile_width())
    check("h", f["h"], ref["h"])
    check("partial", f["partial"], ref["partial"], rel=1e-3)
    check_rel("r", f["r"], ref["r"], 1e-3)
    he = _exps(f["hsf"], M, N)
    _check_mx_output("hg (MXFP8)", f["hq"].cpu().numpy(), he, ref["hg"])
    # the second GEMM as a step: fed the GPU's own MXFP8 hg and partials
    step = MX.gemm_rowscale_partial_mx(f["hq"].cpu().numpy(), he, ora["W2q"], ora["W2e"],
                                       f["partial"].double().cpu().numpy(), N, inp.eps)
    check("out (step)", f["out"], step["out"], strict=True)
    # the whole block against the oracle's composition
    check("out (chain)", f["out"], ref["out"], strict=True)
    # and within the e4m3 error of the exact bf16 block
    exact = O.rmsnorm_block_unfused(b(inp.x), res, b(inp.W1), b(inp.W2), gamma, inp.eps)["out"]
    got = f["out"].double().cpu().numpy()
    rel_rms = float(np.sqrt(np.mean((got - exact) ** 2)) / np.sqrt(np.mean(exact ** 2)))
    assert rel_rms < 0.1, rel_rms
    # a repeated call is bitwise identical
    again = C.gemm_rmsnorm_gemm_mx(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                                   gpu["W2q"], gpu["W2sf"], inp.eps)
    for k in ("out", "h", "hq", "partial", "r"):
        assert torch.equal(f[k], again[k]), k
    assert _same_sf(f["hsf"], again["hsf"], M, N)


def test_mx_block_tail_full_size_sampled_rows():
    inp = synth.llama1b_block_tail(with_down=False)
    gpu, ora = _mx_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    f = C.gemm_rmsnorm_gemm_mx(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                               gpu["W2q"], gpu["W2sf"], inp.eps)
    C.poll_status()
    M, N = f["h"].shape
    rows = np.sort(np.concatenate([[0, M - 1], np.random.default_rng(78).choice(np.arange(1, M - 1), 22,
                                                                                 replace=False)]))
    g1 = MX.gemm_res_partialrms_mx(ora["x8"][rows], ora["sx"], ora["W1t8"], ora["sw1"], res[rows], gamma,
                                   tile_cols=C.partial_tile_width())
    ri = torch.as_tensor(rows, device="cuda")
    he_all = _exps(f["hsf"], M, N)
    check("h (sampled rows)", f["h"][ri], g1["h"])
    _check_mx_output("hg (MXFP8, sampled rows)", f["hq"][ri].cpu().numpy(), he_all[rows], g1["hg"])
    step = MX.gemm_rowscale_partial_mx(f["hq"][ri].cpu().numpy(), he_all[rows], ora["W2q"], ora["W2e"],
                                       f["partial"][:, ri].double().cpu().numpy(), N, inp.eps)
    check_rel("r (sampled rows)", f["r"][ri], step["r"], 1e-5)
    check("out (step, sampled rows)", f["out"][ri], step["out"], strict=True)
    chain = MX.gemm_rowscale_partial_mx(g1["hq"], g1["he"], ora["W2q"], ora["W2e"], g1["partial"], N, inp.eps)
    check("out (chain, sampled rows)", f["out"][ri], chain["out"], strict=True)


@pytest.mark.parametrize("shape", [(256, 512, 512, 1536), (333, 272, 768, 384)])
def test_mx_unfused_chain(shape):
    """The comparison chain of the MXFP8 block (FP8 GEMM, add, RMSNorm with a
    bf16 output, MXFP8 quantisation of y, block-scaled GEMM): the quantiser
    fed the chain's own y is bit-exact, the last GEMM fed the chain's own
    MXFP8 y is held to the bar (the step), and the whole chain against its
    oracle (which rounds t, h and y to bf16 as the chain stores them)."""
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.block_inputs(M, K, N, N2, seed=95 + M, w_std=0.04)
    gpu, ora = _mx_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    u = C.unfused_block_mx(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                           gpu["W2q"], gpu["W2sf"], inp.eps)
    C.poll_status()
    ref = MX.rmsnorm_block_mx_unfused(ora["x8"], ora["sx"], ora["W1t8"], ora["sw1"], res, gamma, ora["W2q"],
                                      ora["W2e"], inp.eps)
    check("t", u["t"], ref["t"])
    check("h", u["h"], ref["h"])
    check_rel("r", u["r"], ref["r"], 1e-3)
    check("y", u["y"], ref["y"])
    yq, ye = MX.mx_quantize(u["y"].double().cpu().numpy())
    np.testing.assert_array_equal(u["yq"].cpu().numpy(), yq)
    np.testing.assert_array_equal(_exps(u["ysf"], M, N), ye)
    step = MX.gemm_rowscale_partial_mx(yq, ye, ora["W2q"], ora["W2e"])
    check("out (step)", u["out"], step["out"], strict=True)
    check("out (chain)", u["out"], ref["out"])


# ---------------------------------------------------------------- guard regions

GUARD = 8192
PATTERN = 0xA5


class _Guarded:
    def __init__(self, n, dtype, shape=None):
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        self.nbytes = nbytes
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype)
        if shape is not None:
            self.t = self.t.view(shape)

    def ptr(self):
        return ctypes.c_void_p(self.t.data_ptr())

    def intact(self):
        torch.cuda.synchronize()
        return bool((self.raw[:GUARD] == PATTERN).all().item()) and \
            bool((self.raw[GUARD + self.nbytes:] == PATTERN).all().item())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_mx_calls_stay_inside_their_buffers():
    """Every output of the three MXFP8 calls carved out of a larger buffer
    whose guard bytes must stay intact, on ragged rows (333: a partial
    128-row scale block and a partial 256-row tile) and a column count with
    an odd number of 128-column blocks; outputs equal the unguarded calls'."""
    lib = C.load_library()
    M, K, N, N2 = 333, 272, 768, 384
    inp = synth.block_inputs(M, K, N, N2, seed=907, w_std=0.04)
    gpu, _ = _mx_inputs(inp)
    W2t = dev(inp.W2.t().contiguous())
    q = _Guarded(N2 * N, torch.uint8, (N2, N))
    sf = _Guarded(C.mx_sf_bytes(N2, N, C.MX_B), torch.uint8)
    assert lib.coda_mx_quantize(_p(W2t), N2, N, C.MX_B, q.ptr(), sf.ptr(), _s()) == 0
    assert q.intact() and sf.intact()
    assert torch.equal(q.t, gpu["W2q"]) and torch.equal(sf.t, gpu["W2sf"])
    T = C.partial_cols(N)
    h = _Guarded(M * N, torch.bfloat16, (M, N))
    hq = _Guarded(M * N, torch.uint8, (M, N))
    hsf = _Guarded(C.mx_sf_bytes(M, N, C.MX_A), torch.uint8)
    part = _Guarded(T * M, torch.float32, (T, M))
    res, gamma = dev(inp.res), dev(inp.gamma)
    assert lib.coda_gemm_res_partialrms_mx(_p(gpu["x8"]), _p(gpu["sx"]), _p(gpu["W1t8"]), _p(gpu["sw1"]), _p(res),
                                           _p(gamma), h.ptr(), hq.ptr(), hsf.ptr(), part.ptr(), M, N, K, _s()) == 0
    for nm, g in (("h", h), ("hq", hq), ("hsf", hsf), ("partial", part)):
        assert g.intact(), nm
    out = _Guarded(M * N2, torch.bfloat16, (M, N2))
    r = _Guarded(M, torch.float32)
    assert lib.coda_gemm_rowscale_partial_mx(hq.ptr(), hsf.ptr(), _p(gpu["W2q"]), _p(gpu["W2sf"]), part.ptr(), T, N,
                                             float(inp.eps), r.ptr(), out.ptr(), M, N2, N, _s()) == 0
    assert out.intact() and r.intact()
    ref = C.gemm_rmsnorm_gemm_mx(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], res, gamma, gpu["W2q"],
                                 gpu["W2sf"], inp.eps)
    for k, g in (("h", h), ("hq", hq), ("partial", part), ("out", out), ("r", r)):
        assert torch.equal(g.t, ref[k]), k
    assert _same_sf(hsf.t, ref["hsf"], M, N)
    C.poll_status()
