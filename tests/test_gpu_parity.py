"""Parity of every library call with the fp64 oracle on small, ragged shapes.

Shapes span several 128 x 256 tiles with ragged tails in M, N and K (and in the
SwiGLU / vocabulary column tiles).  Inputs come from the seeded generators;
the oracle sees the same bf16 values.  Bar: max|err| <= 2e-2 * rms(oracle
output) per output tensor; cross-entropy losses within 1e-3 relative.
"""
import math

import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import CE_REL_TOL, b, check, check_rel, dev, host

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()
    C.set_wait_limit_ns(1_000_000_000)
    yield
    C.poll_status()


def gen(seed):
    return synth.make_gen(seed)


# ----------------------------------------------------------------- plain GEMM

@pytest.mark.parametrize("M,K,N", [(128, 64, 256), (300, 200, 520), (1, 8, 8), (257, 1096, 264), (640, 512, 768)])
def test_gemm_rowscale(M, K, N):
    g = gen(100 + M)
    A = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    r = torch.rand(M, generator=g) + 0.5
    out = C.gemm_rowscale(dev(A), dev(W), dev(r))
    check("out", out, O.gemm_rowscale(b(A), b(W), r.double().numpy()))
    plain = C.gemm_rowscale(dev(A), dev(W), None)
    check("plain", plain, O.matmul(b(A), b(W)))
    C.poll_status()


def test_gemm_rowscale_exact_small_integers():
    # small integers: every product and sum is exact in fp32 and bf16
    g = gen(7)
    M, K, N = 200, 72, 264
    A = torch.randint(-3, 4, (M, K), generator=g).to(torch.bfloat16)
    W = torch.randint(-3, 4, (K, N), generator=g).to(torch.bfloat16)
    out = C.gemm_rowscale(dev(A), dev(W), None)
    ref = A.double() @ W.double()
    assert torch.equal(out.cpu().double(), ref)


# ------------------------------------------------- first GEMM + partial RMS

@pytest.mark.parametrize("M,K,N", [(256, 512, 512), (300, 136, 520), (130, 64, 1032)])
def test_gemm_res_partialrms(M, K, N):
    g = gen(200 + N)
    x = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    res = synth.normal_bf16(g, (M, N))
    gamma = synth.gamma_bf16(g, N)
    h, hg, part = C.gemm_res_partialrms(dev(x), dev(W), dev(res), dev(gamma))
    ref = O.gemm_res_partialrms(b(x), b(W), b(res), b(gamma), C.partial_tile_width())
    check("h", h, ref["h"])
    check("hg", hg, ref["hg"])
    assert part.shape == (C.partial_cols(N), M)
    check_rel("partial", part, ref["partial"], 1e-4)
    # without residual, only partials requested
    _, _, p2 = C.gemm_res_partialrms(dev(x), dev(W), None, None, h=False, hg=False)
    check_rel("partial(no res)", p2, O.gemm_res_partialrms(b(x), b(W), None, None, C.partial_tile_width())["partial"], 1e-4)
    C.poll_status()


def test_gemm_rowscale_partial_folds_the_reduction():
    g = gen(4)
    M, K, N, Nn = 300, 200, 520, 776
    T = C.partial_cols(Nn)
    A = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    part = torch.rand(T, M, generator=g) * 300
    out, r = C.gemm_rowscale_partial(dev(A), dev(W), dev(part), Nn, 1e-6)
    r_ref = O.rms_reduce(part.double().numpy(), Nn, 1e-6)
    check("out", out, O.gemm_rowscale(b(A), b(W), r_ref))
    check_rel("r", r, r_ref, 1e-5)
    # the same reduction as the standalone kernel: identical r
    assert torch.equal(r, C.rms_reduce(dev(part), Nn, 1e-6))


def test_rms_reduce():
    g = gen(3)
    M, N = 1000, 2048
    T = C.partial_cols(N)
    part = torch.rand(T, M, generator=g) * 300
    r = C.rms_reduce(dev(part), N, 1e-6)
    check_rel("r", r, O.rms_reduce(part.double().numpy(), N, 1e-6), 1e-5)


# ----------------------------------------------------------- fused block

@pytest.mark.parametrize("fold", [True, False])
def test_tiny_block_matches_unfused_definition(fold):
    """The tiny GEMM-RMSNorm-GEMM workload (256 tokens, 512 -> 1536), with the
    light reduction folded into the second GEMM or run as its own kernel."""
    inp = synth.tiny_block()
    f = C.gemm_rmsnorm_gemm(dev(inp.x), dev(inp.res), dev(inp.W1), dev(inp.W2), dev(inp.gamma), inp.eps,
                            fold_reduce=fold)
    ref = O.rmsnorm_block_unfused(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    check("out", f["out"], ref["out"], strict=True)
    check("h", f["h"], ref["h"], strict=True)
    check_rel("r", f["r"], ref["r"], 1e-3)
    # the unfused comparison chain rounds t, h and y to bf16 as well: a looser bar
    u = C.unfused_block(dev(inp.x), dev(inp.res), dev(inp.W1), dev(inp.W2), dev(inp.gamma), inp.eps)
    check("unfused out", u["out"], ref["out"], rel=5e-2)
    C.poll_status()


def test_block_ragged_and_accuracy_claim():
    """Fused error is comparable to the unfused bf16 chain's error (both vs fp64)."""
    inp = synth.block_inputs(333, 264, 776, 392, seed=11, w_std=0.04)
    args = [dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    f = C.gemm_rmsnorm_gemm(*args, inp.eps)
    u = C.unfused_block(*args, inp.eps)
    ref = O.rmsnorm_block_unfused(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)["out"]
    ef = check("fused", f["out"], ref)
    eu = check("unfused", u["out"], ref, rel=5e-2)
    assert ef <= 1.25 * eu + 1e-3, (ef, eu)


def test_block_is_deterministic():
    inp = synth.block_inputs(300, 256, 512, 512, seed=12, w_std=0.05)
    args = [dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    a = C.gemm_rmsnorm_gemm(*args, inp.eps)["out"].clone()
    c = C.gemm_rmsnorm_gemm(*args, inp.eps)["out"]
    assert torch.equal(a, c)


def test_empty_batch_is_noop():
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    out = C.gemm_rowscale(x, W, None)
    assert out.shape == (0, 64)


# ------------------------------------------------------------------ SwiGLU

@pytest.mark.parametrize("M,K,F", [(300, 136, 200), (256, 512, 384)])
def test_gemm_swiglu(M, K, F):
    g = gen(300 + F)
    A = synth.normal_bf16(g, (M, K))
    Wgu = synth.normal_bf16(g, (K, 2 * F), std=1 / math.sqrt(K))
    r = torch.rand(M, generator=g) + 0.5
    act, gu = C.gemm_swiglu(dev(A), dev(Wgu), dev(r), save=True)
    ref = O.gemm_swiglu(b(A), b(Wgu), r.double().numpy())
    check("act", act, ref["act"])
    check("gate", gu[:, :F], ref["gate"])
    check("up", gu[:, F:], ref["up"])
    act2, _ = C.gemm_swiglu(dev(A), dev(Wgu), None)
    check("act(no r)", act2, O.gemm_swiglu(b(A), b(Wgu), None)["act"])
    # without the save the call runs its own kernel (no save buffers, one more
    # pipeline stage): the same arithmetic, so the same bits
    act3, gu3 = C.gemm_swiglu(dev(A), dev(Wgu), dev(r))
    assert gu3 is None and torch.equal(act3, act)


def test_swiglu_down_chain():
    inp = synth.block_inputs(260, 128, 256, 2 * 320, seed=13, w_std=0.06, with_down=True)
    f = C.gemm_rmsnorm_gemm(*[dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)], inp.eps)
    s = C.swiglu_down(f["hg"], f["r"], f["h"], dev(inp.W2), dev(inp.W_down))
    u = O.rmsnorm_block_unfused(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    d = O.swiglu_down_unfused(u["y"], b(inp.W2), b(inp.W_down), u["h"])
    # act is an intermediate computed from the bf16-stored hg: the rounding of
    # hg enters gate and up with an error ~2^-9 rms(gate) that the product
    # u * silu'(g) amplifies on the tail, so it gets a looser bar; the chain's
    # outputs (h2 and its partials) keep the bar.
    check("act", s["act"], d["a"], rel=5e-2, storage_rounding=2.0 ** -7)
    check("h2", s["h2"], d["h2"])
    p2 = O.gemm_res_partialrms(d["a"], b(inp.W_down), u["h"], None, C.partial_tile_width())["partial"]
    check("partial2", s["partial2"], p2)


# ----------------------------------------------------------- cross-entropy

@pytest.mark.parametrize("M,K,V", [(300, 136, 1000), (129, 64, 2056), (64, 256, 128256)])
def test_lmhead_ce(M, K, V):
    g = gen(400 + V)
    H = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, V), std=1.5 / math.sqrt(K))
    labels = synth.labels_uniform(g, M, V)
    labels[0], labels[-1] = 0, V - 1
    loss, lse, mean = C.lmhead_ce(dev(H), dev(W), dev(labels))
    ref = O.lmhead_ce(b(H), b(W), labels.numpy())
    check_rel("loss", loss, ref["loss"], CE_REL_TOL)
    check_rel("lse", lse, ref["lse"], CE_REL_TOL)
    assert abs(mean.item() - ref["mean"]) <= CE_REL_TOL * abs(ref["mean"])
    r = torch.rand(M, generator=g) + 0.5
    loss_r, _, _ = C.lmhead_ce(dev(H), dev(W), dev(labels), r=dev(r))
    check_rel("loss(r)", loss_r, O.lmhead_ce(b(H), b(W), labels.numpy(), r=r.double().numpy())["loss"], CE_REL_TOL)


def test_lmhead_ce_bad_labels_give_nan():
    g = gen(5)
    H = synth.normal_bf16(g, (40, 64))
    W = synth.normal_bf16(g, (64, 512), std=0.1)
    labels = torch.tensor([-1, 512, 7] + [3] * 37, dtype=torch.int64)
    loss, lse, _ = C.lmhead_ce(dev(H), dev(W), dev(labels))
    lo = loss.cpu()
    assert torch.isnan(lo[0]) and torch.isnan(lo[1]) and torch.isfinite(lo[2:]).all()
    assert torch.isfinite(lse.cpu()).all()


# ---------------------------------------------------------------- backward

def test_gemm_rowscale_bwd():
    g = gen(21)
    M, N, N2 = 300, 520, 392
    dOut = synth.normal_bf16(g, (M, N2), std=0.5)
    hg = synth.normal_bf16(g, (M, N))
    W2 = synth.normal_bf16(g, (N, N2), std=1 / math.sqrt(N))
    r = torch.rand(M, generator=g) + 0.5
    d_hg, dW2, pdr = C.gemm_rowscale_bwd(dev(dOut), dev(hg), dev(W2), dev(r))
    ref = O.gemm_rowscale_bwd(b(dOut), b(hg), b(W2), r.double().numpy(), C.partial_tile_width())
    check("d_hg", d_hg, ref["d_hg"])
    check("dW2", dW2, ref["dW2"])
    check("pdr", pdr, ref["pdr"])


def test_gemm_rowscale_bwd_last_wave_split_by_k():
    """P GEMM with K = 4104 (65 k-blocks): its tiles form a last partial wave,
    which runs as two halves of the k-blocks adding d_hg and pdr into zeroed
    outputs; the result is the oracle's and the same bits call after call."""
    g = gen(26)
    M, N, N2 = 300, 136, 4104
    dOut = synth.normal_bf16(g, (M, N2), std=0.5)
    hg = synth.normal_bf16(g, (M, N))
    W2 = synth.normal_bf16(g, (N, N2), std=1 / math.sqrt(N))
    r = torch.rand(M, generator=g) + 0.5
    d_hg, dW2, pdr = C.gemm_rowscale_bwd(dev(dOut), dev(hg), dev(W2), dev(r))
    d_hg2, dW22, pdr2 = C.gemm_rowscale_bwd(dev(dOut), dev(hg), dev(W2), dev(r))
    assert torch.equal(d_hg, d_hg2) and torch.equal(pdr, pdr2) and torch.equal(dW2, dW22)
    ref = O.gemm_rowscale_bwd(b(dOut), b(hg), b(W2), r.double().numpy(), C.partial_tile_width())
    check("d_hg", d_hg, ref["d_hg"])
    check("dW2", dW2, ref["dW2"])
    check("pdr", pdr, ref["pdr"])


@pytest.mark.parametrize("M,K,N", [(4171, 64, 136), (4136, 2048, 2560)])
def test_weight_gradient_last_wave_split_by_k(M, K, N):
    """dW1 = x^T dh over 4136-4171 tokens (65-66 k-blocks): the last partial
    wave (every tile of the 1-tile case; 6 of 80 tiles in the other, beside
    whole tiles) runs as halves of the k-blocks adding into zeroed rows of
    dW1.  Oracle parity and the same bits call after call."""
    g = gen(27 + K)
    dh = synth.normal_bf16(g, (M, N))
    x = synth.normal_bf16(g, (M, K))
    W1 = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    _, dW1 = C.gemm_res_partialrms_bwd(dev(dh), dev(x), dev(W1), dx=False)
    _, dW1b = C.gemm_res_partialrms_bwd(dev(dh), dev(x), dev(W1), dx=False)
    assert torch.equal(dW1, dW1b)
    check("dW1", dW1, O.matmul(b(x).T, b(dh)))


def test_rms_reduce_bwd():
    g = gen(22)
    M, N = 300, 520
    T = C.partial_cols(N)
    pdr = torch.randn(T, M, generator=g) * 5
    r = torch.rand(M, generator=g) + 0.5
    d_hg = torch.randn(M, N, generator=g)
    h = synth.normal_bf16(g, (M, N))
    gamma = synth.gamma_bf16(g, N)
    dh, dgamma = C.rms_reduce_bwd(dev(pdr), dev(r), dev(d_hg), dev(h), dev(gamma))
    ref = O.rms_reduce_bwd(pdr.double().numpy(), r.double().numpy(), d_hg.double().numpy(), b(h), b(gamma))
    check("dh", dh, ref["dh"])
    check("dgamma", dgamma, ref["dgamma"])


def test_gemm_res_partialrms_bwd():
    g = gen(23)
    M, N, K = 300, 520, 136
    dh = synth.normal_bf16(g, (M, N))
    x = synth.normal_bf16(g, (M, K))
    W1 = synth.normal_bf16(g, (K, N), std=1 / math.sqrt(K))
    dx, dW1 = C.gemm_res_partialrms_bwd(dev(dh), dev(x), dev(W1))
    ref = O.gemm_res_partialrms_bwd(b(dh), b(x), b(W1))
    check("dx", dx, ref["dx"])
    check("dW1", dW1, ref["dW1"])


def test_block_backward_chain():
    inp = synth.block_inputs(300, 136, 520, 392, seed=24, w_std=0.05)
    dOut = synth.block_backward_dout(300, 392, seed=25, std=0.01)
    d = [dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma)]
    f = C.gemm_rmsnorm_gemm(*d, inp.eps)
    g = C.block_backward(dev(dOut), d[0], d[2], d[3], d[4], f)
    ref = O.rmsnorm_block_backward_unfused(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps,
                                           b(dOut))
    for k in ("dW2", "dgamma", "dres", "dx", "dW1"):
        check(k, g[k], ref[k])
    C.poll_status()


# ------------------------------------------------------------ unfused chain

def test_unfused_pieces():
    g = gen(31)
    M, N = 77, 520
    a = synth.normal_bf16(g, (M, N))
    c = synth.normal_bf16(g, (M, N))
    s = C.unfused_add(dev(a), dev(c))
    check("add", s, O.as_f64(b(a)) + O.as_f64(b(c)))
    gamma = synth.gamma_bf16(g, N)
    y = C.unfused_rmsnorm(dev(a), dev(gamma), 1e-6)
    u = O.rmsnorm_block_unfused(np.zeros((M, 8)), b(a), np.zeros((8, N)), np.eye(N), b(gamma), 1e-6)
    check("rmsnorm", y, u["y"])


# ------------------------------------------------------------- bounded waits

def test_bounded_wait_gives_up_and_reports_timeout():
    assert C.selftest_bounded_wait(2_000_000) == 1     # 2 ms limit on a barrier nobody signals
    with pytest.raises(C.CodaError) as e:
        C.poll_status()
    assert e.value.status == 7
    C.poll_status()   # cleared
    # the context is still usable
    test_rms_reduce()


# ------------------------------------------------------------ SwiGLU backward

# (2600, 72, 2000): 88 tiles on 74 CTA pairs, so some pairs run two and load
# the second tile's first gate/up chunk during the first; ragged rows, a
# ragged last 64-column chunk and a K shorter than one k-block pair
@pytest.mark.parametrize("M,N,F", [(300, 136, 200), (256, 512, 384), (2600, 72, 2000)])
def test_gemm_swiglu_bwd(M, N, F):
    g = gen(500 + F)
    d_out = synth.normal_bf16(g, (M, N))
    W_down = synth.normal_bf16(g, (F, N), std=1 / math.sqrt(N))
    gu = synth.normal_bf16(g, (M, 2 * F), std=1.5)
    d_gu = C.gemm_swiglu_bwd(dev(d_out), dev(W_down), dev(gu))
    ref = O.gemm_swiglu_bwd(b(d_out), b(W_down), b(gu)[:, :F], b(gu)[:, F:])
    check("d_gate", d_gu[:, :F], ref["d_gate"])
    check("d_up", d_gu[:, F:], ref["d_up"])


def test_swiglu_mlp_backward_chain():
    g = gen(31)
    M, N, F = 260, 256, 320
    y = synth.normal_bf16(g, (M, N))
    W_gu = synth.normal_bf16(g, (N, 2 * F), std=1 / math.sqrt(N))
    W_down = synth.normal_bf16(g, (F, N), std=1 / math.sqrt(F))
    res = synth.normal_bf16(g, (M, N))
    d_h2 = synth.normal_bf16(g, (M, N), std=0.01)
    act, gu = C.gemm_swiglu(dev(y), dev(W_gu), None, save=True)
    bw = C.swiglu_mlp_backward(dev(d_h2), dev(y), dev(W_gu), dev(W_down), act, gu)
    C.poll_status()
    ref = O.swiglu_mlp_backward_unfused(b(y), b(W_gu), b(W_down), b(res), b(d_h2))
    # d_gate and d_up are intermediates built from the bf16-saved gate/up (a
    # product of three factors, like act): looser bar; the chain's outputs keep it
    check("d_gate", bw["d_gateup"][:, :F], ref["d_gate"], rel=5e-2, storage_rounding=2.0 ** -7)
    check("d_up", bw["d_gateup"][:, F:], ref["d_up"], rel=5e-2, storage_rounding=2.0 ** -7)
    check("d_y", bw["d_y"], ref["d_y"])
    check("dW_gu", bw["dW_gu"], ref["dW_gu"])
    check("dW_down", bw["dW_down"], ref["dW_down"])


def test_stream_order_holds_with_programmatic_launch():
    """Every pair GEMM is launched with programmatic stream serialisation and
    lets the next one start early; work placed between two GEMMs on the
    stream must still be seen.  Scaling the partials by 4 between the two
    GEMMs of the block halves r (eps = 0), so out must halve exactly."""
    inp = synth.tiny_block()
    x, res, W1, W2, g = (dev(t) for t in (inp.x, inp.res, inp.W1, inp.W2, inp.gamma))
    h, hg, part = C.gemm_res_partialrms(x, W1, res, g)
    out_ref, _ = C.gemm_rowscale_partial(hg, W2, part, 512, 0.0)
    for _ in range(3):  # the same sequence with an ordinary stream op in between
        h, hg, part = C.gemm_res_partialrms(x, W1, res, g)
        part.mul_(4.0)
        out, r = C.gemm_rowscale_partial(hg, W2, part, 512, 0.0)
        torch.cuda.synchronize()
        C.poll_status()
        assert torch.equal(out.float() * 2, out_ref.float())


def test_degenerate_rows_zero_hidden_state():
    """Rows whose h is exactly zero (x and res zero) have no RMS: their partials
    are 0, r = 1/sqrt(eps), and since hg is 0 their output row is exactly 0;
    the other rows are unaffected.  With eps = 0 the same rows give r = inf
    and a NaN output (0 * inf), as the definition does."""
    inp = synth.tiny_block()
    x, res = inp.x.clone(), inp.res.clone()
    zero_rows = [0, 5, 255]
    x[zero_rows] = 0
    res[zero_rows] = 0
    d = [dev(t) for t in (x, res, inp.W1, inp.W2, inp.gamma)]
    f = C.gemm_rmsnorm_gemm(*d, inp.eps)
    C.poll_status()
    ref = O.rmsnorm_block_unfused(b(x), b(res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    check("out", f["out"], ref["out"])
    zr = torch.as_tensor(zero_rows, device="cuda")
    assert torch.all(f["out"][zr] == 0)
    assert torch.all(f["partial"][:, zr] == 0)
    assert torch.allclose(f["r"][zr], torch.full((3,), 1.0 / math.sqrt(inp.eps), device="cuda"), rtol=1e-6)
    g0 = C.gemm_rmsnorm_gemm(*d, 0.0)
    C.poll_status()
    assert torch.isinf(g0["r"][zr]).all() and torch.isnan(g0["out"][zr].float()).all()
    keep = torch.as_tensor([i for i in range(256) if i not in zero_rows], device="cuda")
    assert torch.isfinite(g0["out"][keep].float()).all()


def test_fp8_quantize_all_zero_tensor():
    """An all-zero tensor has amax 0, scale 1 and all-zero codes."""
    t = torch.zeros(64, 32, dtype=torch.bfloat16, device="cuda")
    for tr in (False, True):
        codes, amax, scale = C.fp8_quantize(t, transpose=tr)
        torch.cuda.synchronize()
        assert float(amax.item()) == 0.0 and float(scale.item()) == 1.0
        assert int(codes.count_nonzero().item()) == 0
