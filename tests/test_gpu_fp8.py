"""Parity of the FP8 (e4m3) block and its quantiser with the fp64 oracle.

The KuCoin news flash "CODA: new research optimizes transformer training with
GEMM epilogue programming" (section "The lazy cost of training large
models") names FP8 as the reason the non-GEMM share of training time grows.
The quantiser is compared bit for bit (byte work); the block's e4m3 output
hg8 code by code (a code may differ by one step where the fp32 and fp64
values of gamma * h straddle a rounding boundary); every floating-point
output against the fp64 oracle at the usual bar.  The GEMM operands of both
sides are quantised by each side's own quantiser, asserted equal.
"""
import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from oracle import coda_oracle_fp8 as F8
from tests._util import b, check, check_rel, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


def _oracle_quant(t_bits, transpose=False):
    """The oracle's own per-tensor quantisation of a bf16 tensor."""
    v = O.bf16_to_f64(t_bits)
    if transpose:
        v = v.T
    s = F8.quant_scale(np.abs(v).max())
    return F8.quantize(v.astype(np.float32), s), s


@pytest.mark.parametrize("rows,cols,transpose", [(100, 136, False), (136, 200, True), (64, 8, True),
                                                 (1, 8, False), (260, 64, True)])
def test_fp8_quantize_bit_exact(rows, cols, transpose):
    g = synth.make_gen(900 + rows + cols)
    t = synth.normal_bf16(g, (rows, cols), std=3.0)
    t[0, 0] = 1000.0  # a large element sets the scale; the rest sit well inside the range
    codes, amax, scale = C.fp8_quantize(dev(t), transpose=transpose)
    want, s = _oracle_quant(synth.bf16_bits(t), transpose)
    np.testing.assert_array_equal(codes.cpu().numpy(), want)
    assert float(amax.item()) == float(np.abs(O.bf16_to_f64(b(t))).max())
    assert np.float32(scale.item()) == s


def test_fp8_scale_from_amax():
    for a in (97.0, 0.0, 1e-30, 448.0, 3.0e38):
        amax = torch.tensor([a], dtype=torch.float32, device="cuda")
        got = C.fp8_scale_from_amax(amax)
        assert np.float32(got.item()) == F8.quant_scale(np.float32(a))


def _fp8_inputs(inp):
    """GPU and oracle quantisation of the block's inputs (codes asserted equal)."""
    xd, W1d, W2d = dev(inp.x), dev(inp.W1), dev(inp.W2)
    x8, _, sx = C.fp8_quantize(xd)
    W1t8, _, sw1 = C.fp8_quantize(W1d, transpose=True)
    W2t8, _, sw2 = C.fp8_quantize(W2d, transpose=True)
    ox8, osx = _oracle_quant(synth.bf16_bits(inp.x))
    oW1, osw1 = _oracle_quant(synth.bf16_bits(inp.W1), transpose=True)
    oW2, osw2 = _oracle_quant(synth.bf16_bits(inp.W2), transpose=True)
    for got, want in ((x8, ox8), (W1t8, oW1), (W2t8, oW2)):
        np.testing.assert_array_equal(got.cpu().numpy(), want)
    for got, want in ((sx, osx), (sw1, osw1), (sw2, osw2)):
        assert np.float32(got.item()) == want
    gpu = dict(x8=x8, sx=sx, W1t8=W1t8, sw1=sw1, W2t8=W2t8, sw2=sw2)
    ora = dict(x8=ox8, sx=float(osx), W1t8=oW1, sw1=float(osw1), W2t8=oW2, sw2=float(osw2))
    return gpu, ora


def _oracle_block(ora, res, gamma, s_hg, eps, rows=None):
    x8 = ora["x8"] if rows is None else ora["x8"][rows]
    res = res if rows is None else res[rows]
    return F8.rmsnorm_block_fp8(x8, ora["sx"], ora["W1t8"], ora["sw1"], res, gamma, s_hg, ora["W2t8"], ora["sw2"],
                                eps, tile_cols=C.partial_tile_width())


def _check_codes(name, got, want, max_frac):
    """e4m3 outputs: equal codes, except a few whose values are one e4m3 step
    apart (2^-3 of the magnitude in the normal range, 2^-9 among the
    subnormals; a value next to zero may change sign)."""
    g = got.cpu().numpy()
    w = np.asarray(want)
    diff = g != w
    frac = float(diff.mean()) if diff.size else 0.0
    assert frac <= max_frac, f"{name}: {frac:.2e} of the codes differ"
    if diff.any():
        dg, dw = F8.e4m3_decode(g[diff]), F8.e4m3_decode(w[diff])
        step = 2.0 ** -3 * np.maximum(np.abs(dg), np.abs(dw)) + 2.0 ** -9
        assert np.all(np.abs(dg - dw) <= step), f"{name}: codes more than one step apart"


def _run_gpu_block(gpu, inp, s_hg, eps):
    return C.gemm_rmsnorm_gemm_fp8(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                                   s_hg, gpu["W2t8"], gpu["sw2"], eps)


@pytest.mark.parametrize("shape", [(256, 512, 512, 1536), (333, 272, 784, 400), (130, 1040, 256, 272)])
def test_fp8_block_small(shape):
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.block_inputs(M, K, N, N2, seed=70 + M, w_std=0.04)
    gpu, ora = _fp8_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    s_hg = float(F8.quant_scale(_oracle_block(ora, res, gamma, 1.0, inp.eps)["amax"]))
    ref = _oracle_block(ora, res, gamma, s_hg, inp.eps)
    f = _run_gpu_block(gpu, inp, torch.tensor([s_hg], dtype=torch.float32, device="cuda"), inp.eps)
    C.poll_status()
    check("h", f["h"], ref["h"])
    check("partial", f["partial"], ref["partial"], rel=1e-3)
    check_rel("r", f["r"], ref["r"], 1e-3)
    check_rel("amax", f["amax"], np.array([ref["amax"]]), 1e-5)
    _check_codes("hg8", f["hg8"], ref["hg8"], 1e-3)
    check("out", f["out"], ref["out"])
    # the quantised block stays within e4m3's error of the exact bf16 block:
    # four operands each rounded to 3 mantissa bits (rms relative error about
    # 2^-4 / sqrt(3) each) give an rms error of a few percent
    exact = O.rmsnorm_block_unfused(b(inp.x), res, b(inp.W1), b(inp.W2), gamma, inp.eps)["out"]
    got = f["out"].double().cpu().numpy()
    rel_rms = float(np.sqrt(np.mean((got - exact) ** 2)) / np.sqrt(np.mean(exact ** 2)))
    assert rel_rms < 0.1, rel_rms


def test_fp8_block_delayed_scaling_and_repeat():
    """The second call quantises hg with the scale derived from the first
    call's amax: its codes then use the e4m3 range fully (the largest |code|
    is 448 = 0x7E, give or take one step), and a repeated call is bitwise
    identical."""
    inp = synth.block_inputs(333, 272, 784, 400, seed=403, w_std=0.04)
    gpu, _ = _fp8_inputs(inp)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    f1 = _run_gpu_block(gpu, inp, one, inp.eps)
    s_hg = C.fp8_scale_from_amax(f1["amax"])
    f2 = {k: v.clone() for k, v in _run_gpu_block(gpu, inp, s_hg, inp.eps).items()}
    f3 = _run_gpu_block(gpu, inp, s_hg, inp.eps)
    C.poll_status()
    top = int((f2["hg8"] & 0x7F).max().item())
    assert top in (0x7D, 0x7E)
    for k in ("out", "h", "hg8", "amax", "partial", "r"):
        assert torch.equal(f2[k], f3[k]), k


def test_fp8_block_tail_full_size_sampled_rows():
    inp = synth.llama1b_block_tail(with_down=False)
    gpu, ora = _fp8_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    # s_hg from the oracle's amax over every row (h alone decides it)
    h_all = F8.e4m3_decode(ora["x8"]) @ F8.e4m3_decode(ora["W1t8"]).T * (ora["sx"] * ora["sw1"]) + res
    amax = float(np.abs(gamma[None, :] * h_all).max())
    s_hg = float(F8.quant_scale(amax))
    f = _run_gpu_block(gpu, inp, torch.tensor([s_hg], dtype=torch.float32, device="cuda"), inp.eps)
    C.poll_status()
    check_rel("amax", f["amax"], np.array([amax]), 1e-5)
    rows = np.sort(np.concatenate([[0, 8191], np.random.default_rng(77).choice(np.arange(1, 8191), 22,
                                                                                 replace=False)]))
    ref = _oracle_block(ora, res, gamma, s_hg, inp.eps, rows=rows)
    ri = torch.as_tensor(rows, device="cuda")
    check("h (sampled rows)", f["h"][ri], ref["h"])
    check_rel("r (sampled rows)", f["r"][ri], ref["r"], 1e-3)
    _check_codes("hg8 (sampled rows)", f["hg8"][ri], ref["hg8"], 1e-3)
    check("out (sampled rows)", f["out"][ri], ref["out"])


@pytest.mark.parametrize("shape", [(256, 512, 512, 1536), (333, 272, 784, 400)])
def test_fp8_unfused_chain(shape):
    """The comparison chain of the FP8 block (FP8 GEMM, add, RMSNorm with an
    e4m3 output, FP8 GEMM) against its oracle, which stores t and h in bf16
    as the chain does."""
    M, K, N, N2 = shape
    inp = synth.tiny_block() if shape == (256, 512, 512, 1536) else \
        synth.block_inputs(M, K, N, N2, seed=80 + M, w_std=0.04)
    gpu, ora = _fp8_inputs(inp)
    res, gamma = O.bf16_to_f64(b(inp.res)), O.bf16_to_f64(b(inp.gamma))
    pre = F8.rmsnorm_block_fp8_unfused(ora["x8"], ora["sx"], ora["W1t8"], ora["sw1"], res, gamma, 1.0, ora["W2t8"],
                                       ora["sw2"], inp.eps)
    s_y = float(F8.quant_scale(pre["amax"]))
    ref = F8.rmsnorm_block_fp8_unfused(ora["x8"], ora["sx"], ora["W1t8"], ora["sw1"], res, gamma, s_y, ora["W2t8"],
                                       ora["sw2"], inp.eps)
    u = C.unfused_block_fp8(gpu["x8"], gpu["sx"], gpu["W1t8"], gpu["sw1"], dev(inp.res), dev(inp.gamma),
                            torch.tensor([s_y], dtype=torch.float32, device="cuda"), gpu["W2t8"], gpu["sw2"], inp.eps)
    C.poll_status()
    check("t", u["t"], ref["t"])
    check("h", u["h"], ref["h"])
    check_rel("r", u["r"], ref["r"], 1e-3)
    check_rel("amax", u["amax"], np.array([ref["amax"]]), 1e-3)
    # The oracle rounds t and h to bf16 as the chain stores them.  Where the
    # kernel's fp32 t and the oracle's fp64 t straddle a bf16 rounding
    # boundary, t (or h) moves by one bf16 ulp (2^-7 relative) between the two,
    # which moves y by |gamma| r 2^-7 (|t| + |h|) — several e4m3 steps where
    # t + res cancels.  So: few codes differ, and each differing one lies
    # within that shift plus half an e4m3 step of the oracle's y.
    g8, w8 = u["y8"].cpu().numpy(), ref["y8"]
    diff = g8 != w8
    assert diff.mean() <= 1e-2, diff.mean()
    shift = 1.1 * np.abs(gamma)[None, :] * ref["r"][:, None] * 2.0 ** -7 * (np.abs(ref["t"]) + np.abs(ref["h"]))
    bound = 2.0 ** -4 * (np.abs(ref["y"]) + shift) + 2.0 ** -10 * s_y + shift
    yq = F8.e4m3_decode(g8) * s_y
    assert np.all(np.abs(yq - ref["y"])[diff] <= bound[diff] * (1 + 1e-3))
    check("out", u["out"], ref["out"])
