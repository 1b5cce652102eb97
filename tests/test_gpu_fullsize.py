"""Full-size parity on the benchmark workloads, through the same calls bench.py times.

Workloads (seeded synthetic inputs, recipe in gemm_epilogue_transformer_02_b200/synth.py):
  * 1B block tail: 8192 tokens, hidden 2048, W1[2048,2048], W2[2048,16384];
  * SwiGLU + down projection continuing it: W_gu = W2, W_down[8192,2048];
  * LM-head cross-entropy: H[8192,2048], W_vocab[2048,128256];
  * backward of the block: dOut[8192,16384] (std 0.01).
The forward is row-independent, so the oracle evaluates sampled token rows;
cross-entropy is checked per sampled token (relative 1e-3) and the mean by its
definition over the GPU's own per-token losses; the backward evaluates every
gradient except dW2, which is checked on sampled columns.
"""
import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import CE_REL_TOL, b, check, check_rel, dev, host

pytestmark = pytest.mark.gpu

M, D, N2 = 8192, 2048, 16384


def sample_rows(n, total, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(np.arange(1, total - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, total - 1], rows]))


@pytest.fixture(scope="module")
def block():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    inp = synth.llama1b_block_tail(with_down=True)
    d = {k: dev(getattr(inp, k)) for k in ("x", "res", "W1", "W2", "gamma", "W_down")}
    f = C.gemm_rmsnorm_gemm(d["x"], d["res"], d["W1"], d["W2"], d["gamma"], inp.eps)
    C.poll_status()
    return inp, d, f


def test_block_tail_forward_sampled_rows(block):
    inp, d, f = block
    rows = sample_rows(48, M, 1)
    ref = O.rmsnorm_block_unfused(b(inp.x)[rows], b(inp.res)[rows], b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    out = f["out"][torch.as_tensor(rows, device="cuda")]
    check("out", out, ref["out"], strict=True)
    check("h", f["h"][torch.as_tensor(rows, device="cuda")], ref["h"], strict=True)
    check_rel("r", f["r"].cpu().numpy()[rows], ref["r"], 1e-3)
    # the unfused comparison chain computes the same block
    u = C.unfused_block(d["x"], d["res"], d["W1"], d["W2"], d["gamma"], inp.eps)
    check("unfused out", u["out"][torch.as_tensor(rows, device="cuda")], ref["out"], rel=5e-2)
    C.poll_status()


def test_swiglu_down_sampled_rows(block):
    inp, d, f = block
    s = C.swiglu_down(f["hg"], f["r"], f["h"], d["W2"], d["W_down"])
    C.poll_status()
    rows = sample_rows(24, M, 2)
    u = O.rmsnorm_block_unfused(b(inp.x)[rows], b(inp.res)[rows], b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    ref = O.swiglu_down_unfused(u["y"], b(inp.W2), b(inp.W_down), u["h"])
    ri = torch.as_tensor(rows, device="cuda")
    # the SwiGLU GEMM as a step: the oracle is fed the kernel's own inputs
    # (the bf16 hg and the fp32 r of the block), so only this GEMM's own
    # arithmetic and the bf16 storage of act are measured, at the full bar
    step = O.gemm_swiglu(b(f["hg"][ri]), b(d["W2"]), f["r"][ri].double().cpu().numpy())
    check("act (step, K=2048)", s["act"][ri], step["act"])
    # against the unfused chain, act also carries the rounding of hg to bf16
    # (an input of this step), amplified by the product silu(g) * u
    check("act (chain)", s["act"][ri], ref["a"], rel=5e-2, storage_rounding=2.0 ** -7)
    check("h2", s["h2"][ri], ref["h2"], strict=True)
    p2 = O.gemm_res_partialrms(ref["a"], b(inp.W_down), u["h"], None, C.partial_tile_width())["partial"]
    check("partial2", s["partial2"][:, ri], p2, strict=True)
    r2 = C.rms_reduce(s["partial2"], D, inp.eps)
    check_rel("r2", r2.cpu().numpy()[rows], O.rms_reduce(p2, D, inp.eps), 1e-3)


def test_lmhead_ce_sampled_tokens():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    H, W, labels = synth.lmhead_ce_inputs()
    loss, lse, mean = C.lmhead_ce(dev(H), dev(W), dev(labels))
    C.poll_status()
    rows = sample_rows(40, M, 3)
    ref = O.cross_entropy_unfused(b(H)[rows], b(W), labels.numpy()[rows])
    check_rel("loss", loss.cpu().numpy()[rows], ref["loss"], CE_REL_TOL)
    check_rel("lse", lse.cpu().numpy()[rows], ref["lse"], CE_REL_TOL)
    lo = loss.double().cpu().numpy()
    assert np.all(np.isfinite(lo))
    # mean = sum(loss) / M over all tokens; each sampled token is within 1e-3
    assert abs(mean.item() - lo.mean()) <= 1e-5 * abs(lo.mean())


def test_block_backward(block):
    inp, d, f = block
    dOut = synth.block_backward_dout()
    g = C.block_backward(dev(dOut), d["x"], d["W1"], d["W2"], d["gamma"], f)
    C.poll_status()
    cols = sample_rows(32, N2, 4)
    ref = O.rmsnorm_block_backward_cols(b(inp.x), b(inp.res), b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps,
                                        b(dOut), cols)
    check("dW2 (sampled columns)", g["dW2"][:, torch.as_tensor(cols, device="cuda")], ref["dW2_cols"], strict=True)
    check("dgamma", g["dgamma"], ref["dgamma"], strict=True)
    check("dres", g["dres"], ref["dres"], strict=True)
    check("dx", g["dx"], ref["dx"], strict=True)
    check("dW1", g["dW1"], ref["dW1"], strict=True)


def test_swiglu_backward_sampled_rows(block):
    """SwiGLU backward on the SwiGLU-chain workload: d_h2 std 0.01 (seed 5)."""
    inp, d, f = block
    s = C.swiglu_down(f["hg"], f["r"], f["h"], d["W2"], d["W_down"], save=True)
    d_h2 = synth.block_backward_dout(M, D, seed=5)
    y = f["hg"]  # the gate/up GEMM's operand (r is applied in its epilogue)
    d_gu = C.gemm_swiglu_bwd(dev(d_h2), d["W_down"], s["gateup"])
    C.poll_status()
    rows = sample_rows(24, M, 6)
    u = O.rmsnorm_block_unfused(b(inp.x)[rows], b(inp.res)[rows], b(inp.W1), b(inp.W2), b(inp.gamma), inp.eps)
    ref = O.swiglu_mlp_backward_unfused(u["y"], b(inp.W2), b(inp.W_down), u["h"], b(d_h2)[rows])
    ri = torch.as_tensor(rows, device="cuda")
    F = N2 // 2
    # the SwiGLU backward GEMM as a step (K = 2048): the oracle is fed the
    # kernel's own inputs, the saved bf16 gate/up of the forward, at the full bar
    gu = b(s["gateup"][ri])
    step = O.gemm_swiglu_bwd(b(d_h2)[rows], b(d["W_down"]), gu[:, :F], gu[:, F:])
    check("d_gate (step, K=2048)", d_gu[ri][:, :F], step["d_gate"])
    check("d_up (step, K=2048)", d_gu[ri][:, F:], step["d_up"])
    # against the unfused chain they also carry the rounding of hg and of the
    # saved gate/up (inputs of this step), as act does
    check("d_gate (chain)", d_gu[ri][:, :F], ref["d_gate"], rel=5e-2, storage_rounding=2.0 ** -7)
    check("d_up (chain)", d_gu[ri][:, F:], ref["d_up"], rel=5e-2, storage_rounding=2.0 ** -7)
    del y
