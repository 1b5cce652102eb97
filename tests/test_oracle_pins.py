"""Pins of the fp64 oracle against things other than itself (CPU only).

The oracle follows the KuCoin news flash "CODA: new research optimizes
transformer training with GEMM epilogue programming" (section "CODA: the
secret in the epilogue" for the GEMM-RMSNorm-GEMM pattern, the commuting row
scale r, the partial RMS and its light reduction; section "Five kinds of
building blocks" for chunk log-sum-exp and the online max / sum-exp state).

Every pin here is independent of the oracle's own code path: closed forms from
``tests/golden/closed_forms.txt`` (40-digit decimal), pure-Python brute force on
tiny shapes (no numpy matmul), invariants of the mathematics, and central
finite differences for the backward.  Each is chosen so that a plausible
mistake (dropped residual, eps outside the square root, mean over the wrong
axis, transposed operand, swapped gate/up, wrong label index, wrong sign in
the RMSNorm backward) fails at least one test.
"""
import math
import os

import numpy as np
import pytest

from oracle import coda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.txt")


def golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, val = line.split()[:2]
            out[name] = float(val)
    return out


# ----------------------------------------------------------------- brute force

def bf_matmul(A, B):
    A = [list(map(float, r)) for r in np.asarray(A, dtype=np.float64)]
    B = [list(map(float, r)) for r in np.asarray(B, dtype=np.float64)]
    n, k, m = len(A), len(B), len(B[0])
    return np.array([[math.fsum(A[i][t] * B[t][j] for t in range(k)) for j in range(m)]
                     for i in range(n)])


def bf_block(x, res, W1, W2, gamma, eps):
    h = bf_matmul(x, W1) + res
    M, N = h.shape
    y = np.zeros_like(h)
    for i in range(M):
        ms = math.fsum(float(v) * float(v) for v in h[i]) / N
        r = 1.0 / math.sqrt(ms + eps)
        for j in range(N):
            y[i, j] = gamma[j] * h[i, j] * r
    return h, y, bf_matmul(y, W2)


def bf_silu(v):
    return v / (1.0 + math.exp(-v))


def rng(seed=0):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------- widening

def test_bf16_widening_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x3EAB, 0x4049],
                    dtype=np.uint16)
    got = O.bf16_to_f64(bits)
    # 0x3EAB: sign 0, exponent 0x7D (2^-2), mantissa 0x2B/128 -> 0.25 * (1 + 43/128)
    want = [1.0, -2.0, 0.0, -0.0, math.inf, -math.inf, 2.0 ** -133, 0.25 * (1 + 43 / 128),
            2.0 * (1 + 0x49 / 128)]
    for g, w in zip(got, want):
        assert g == w
    assert math.copysign(1.0, got[3]) == -1.0


def test_bf16_widening_matches_torch_rounding():
    torch = pytest.importorskip("torch")
    v = torch.tensor([0.1, -3.3, 1e-3, 65504.0, 1.0 / 3.0])
    b = v.to(torch.bfloat16)
    bits = b.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.bf16_to_f64(bits), b.to(torch.float64).numpy())


# ------------------------------------------------------------ forward block

def test_block_matches_brute_force_with_ragged_shapes():
    r = rng(1)
    M, K, N, N2 = 5, 7, 6, 3
    x, res = r.normal(size=(M, K)), r.normal(size=(M, N))
    W1, W2 = r.normal(size=(K, N)), r.normal(size=(N, N2))
    gamma = 1 + 0.1 * r.normal(size=N)
    f = O.rmsnorm_block_unfused(x, res, W1, W2, gamma, 1e-6)
    h, y, out = bf_block(x, res, W1, W2, gamma, 1e-6)
    np.testing.assert_allclose(f["h"], h, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(f["y"], y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(f["out"], out, rtol=1e-12, atol=1e-12)


def test_identity_W1_gives_x_plus_res():
    r = rng(2)
    x, res = r.normal(size=(4, 8)), r.normal(size=(4, 8))
    f = O.rmsnorm_block_unfused(x, res, np.eye(8), np.eye(8), np.ones(8), 1e-6)
    np.testing.assert_array_equal(f["h"], x + res)


def test_constant_row_normalises_to_closed_form():
    g = golden()
    N = 16
    x = np.zeros((2, 4))
    res = np.stack([np.full(N, 1.0), np.full(N, -3.0)])
    W1 = rng(3).normal(size=(4, N))        # x = 0, so W1 must not matter
    f = O.rmsnorm_block_unfused(x, res, W1, np.eye(N), np.ones(N), 1e-6)
    assert np.allclose(f["y"][0], g["rms_const_row_c1"], rtol=0, atol=1e-15)
    assert np.allclose(f["y"][1], g["rms_const_row_cm3"], rtol=0, atol=1e-15)
    # gamma = 1 and W2 = I: out is y itself
    np.testing.assert_array_equal(f["out"], f["y"])


def test_rms_invariant_and_gamma_broadcast():
    r = rng(4)
    M, N = 6, 10
    h_in = r.normal(size=(M, N)) * 3
    gamma = 1 + 0.1 * r.normal(size=N)
    eps = 1e-3
    f = O.rmsnorm_block_unfused(np.zeros((M, 1)), h_in, np.zeros((1, N)), np.eye(N), gamma, eps)
    ms = np.array([math.fsum(v * v for v in row) / N for row in h_in])
    lhs = ((f["y"] / gamma[None, :]) ** 2).mean(axis=1)
    np.testing.assert_allclose(lhs, ms / (ms + eps), rtol=1e-13)


def test_partials_sum_to_row_sum_of_squares():
    r = rng(5)
    M, K, N = 5, 9, 37                     # 37 columns -> ragged last tile
    x, W, res = r.normal(size=(M, K)), r.normal(size=(K, N)), r.normal(size=(M, N))
    a = O.gemm_res_partialrms(x, W, res, np.ones(N), tile_cols=8)
    assert a["partial"].shape == (5, M)
    h = bf_matmul(x, W) + res
    for i in range(M):
        assert math.isclose(a["partial"][:, i].sum(), math.fsum(v * v for v in h[i]), rel_tol=1e-13)
        # tile 4 holds only the 5 columns 32..36
        assert math.isclose(a["partial"][4, i], math.fsum(v * v for v in h[i, 32:]), rel_tol=1e-13)


def test_reparameterised_block_equals_unfused():
    r = rng(6)
    M, K, N, N2 = 33, 40, 48, 24
    args = (r.normal(size=(M, K)), r.normal(size=(M, N)), r.normal(size=(K, N)) / 6,
            r.normal(size=(N, N2)) / 7, 1 + 0.1 * r.normal(size=N), 1e-6)
    u = O.rmsnorm_block_unfused(*args)
    for tile in (8, 16, 256):
        p = O.rmsnorm_block_reparam(*args, tile_cols=tile)
        np.testing.assert_allclose(p["out"], u["out"], rtol=1e-12, atol=1e-12 * np.abs(u["out"]).max())
        np.testing.assert_allclose(p["r"], u["r"], rtol=1e-12)


def test_rowscale_commutes_with_matmul():
    r = rng(7)
    A, W, s = r.normal(size=(4, 5)), r.normal(size=(5, 3)), r.uniform(0.5, 2, size=4)
    np.testing.assert_allclose(O.gemm_rowscale(A, W, s), bf_matmul(s[:, None] * A, W), rtol=1e-13)


# ------------------------------------------------------------------- SwiGLU

def test_silu_closed_forms():
    g = golden()
    v = O.silu(np.array([0.0, 1.0, -2.0, 800.0, -800.0]))
    assert v[0] == 0.0
    assert math.isclose(v[1], g["silu_1"], rel_tol=1e-15)
    assert math.isclose(v[2], g["silu_m2"], rel_tol=1e-15)
    assert v[3] == 800.0 and v[4] == 0.0
    z = np.linspace(-6, 6, 25)
    np.testing.assert_allclose(O.silu(-z), O.silu(z) - z, atol=1e-15)


def test_swiglu_gate_is_first_half_and_brute_force():
    r = rng(8)
    M, K, F = 3, 4, 5
    A, Wgu, s = r.normal(size=(M, K)), r.normal(size=(K, 2 * F)), r.uniform(0.5, 2, size=M)
    sw = O.gemm_swiglu(A, Wgu, s)
    acc = bf_matmul(A, Wgu)
    for i in range(M):
        for j in range(F):
            g, u = s[i] * acc[i, j], s[i] * acc[i, F + j]
            assert math.isclose(sw["act"][i, j], bf_silu(g) * u, rel_tol=1e-12, abs_tol=1e-14)
    # identity blocks: gate = up = y, so act = silu(y) * y
    y = r.normal(size=(2, F))
    d = O.swiglu_down_unfused(y, np.hstack([np.eye(F), np.eye(F)]), np.eye(F), np.zeros((2, F)))
    np.testing.assert_allclose(d["a"], O.silu(y) * y, rtol=1e-15)
    np.testing.assert_allclose(d["h2"], d["a"], rtol=1e-15)


def test_swiglu_chain_matches_steps():
    r = rng(9)
    M, K, N, F = 6, 8, 8, 5
    f = O.rmsnorm_block_reparam(r.normal(size=(M, K)), r.normal(size=(M, N)), r.normal(size=(K, N)),
                                r.normal(size=(N, 2 * F)), 1 + 0.1 * r.normal(size=N), 1e-6)
    Wgu, Wd = r.normal(size=(N, 2 * F)), r.normal(size=(F, N))
    y = f["r"][:, None] * f["hg"]
    d = O.swiglu_down_unfused(y, Wgu, Wd, f["h"])
    s = O.gemm_swiglu(f["hg"], Wgu, f["r"])
    np.testing.assert_allclose(s["act"], d["a"], rtol=1e-12, atol=1e-13)
    h2 = O.gemm_res_partialrms(s["act"], Wd, f["h"], None, 4)["h"]
    np.testing.assert_allclose(h2, d["h2"], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ cross-entropy

def test_ce_closed_forms():
    g = golden()
    M, K = 4, 3
    H = rng(10).normal(size=(M, K))
    for V, key in ((1000, "ce_uniform_V1000"), (128256, "ce_uniform_V128256")):
        if V == 128256:
            Hs, labels = H[:2], np.array([0, V - 1])
        else:
            Hs, labels = H, np.array([0, 7, 999, 500])
        c = O.lmhead_ce(Hs, np.zeros((K, V)), labels)
        np.testing.assert_allclose(c["loss"], g[key], rtol=1e-14)
        assert math.isclose(c["mean"], g[key], rel_tol=1e-14)
    # one logit L = 5 at the label: H = e_0, W row 0 = 5 at column 17
    W = np.zeros((K, 1000))
    W[0, 17] = 5.0
    c = O.lmhead_ce(np.array([[1.0, 0, 0]]), W, np.array([17]))
    assert math.isclose(c["loss"][0], g["ce_single_logit_L5_V1000"], rel_tol=1e-14)


def test_ce_online_chunks_match_brute_force_and_shift_invariance():
    r = rng(11)
    M, K, V = 4, 5, 23
    H, W = r.normal(size=(M, K)) * 3, r.normal(size=(K, V))
    labels = np.array([0, 22, 5, 11])
    z = bf_matmul(H, W)
    for chunk in (1, 3, 7, 256):
        c = O.lmhead_ce(H, W, labels, chunk_cols=chunk)
        for i in range(M):
            lse = math.log(math.fsum(math.exp(v) for v in z[i]))
            assert math.isclose(c["lse"][i], lse, rel_tol=1e-13)
            assert math.isclose(c["loss"][i], lse - z[i, labels[i]], rel_tol=1e-12)
    u = O.cross_entropy_unfused(H, W, labels)
    np.testing.assert_allclose(u["loss"], O.lmhead_ce(H, W, labels)["loss"], rtol=1e-13)
    # adding a constant to every logit of a row changes lse by that constant and loss not at all
    Hs = np.hstack([H, np.ones((M, 1))])
    Ws = np.vstack([W, np.full((1, V), 2.5)])
    cs = O.lmhead_ce(Hs, Ws, labels)
    np.testing.assert_allclose(cs["lse"], u["lse"] + 2.5, rtol=1e-13)
    np.testing.assert_allclose(cs["loss"], u["loss"], rtol=1e-12)


def test_ce_row_scale_and_bad_labels():
    r = rng(12)
    H, W, s = r.normal(size=(3, 4)), r.normal(size=(4, 9)), np.array([0.5, 1.0, 2.0])
    c = O.lmhead_ce(H, W, np.array([1, 2, 3]), r=s)
    u = O.cross_entropy_unfused(s[:, None] * H, W, np.array([1, 2, 3]))
    np.testing.assert_allclose(c["loss"], u["loss"], rtol=1e-13)
    bad = O.lmhead_ce(H, W, np.array([-1, 9, 3]))
    assert np.isnan(bad["loss"][0]) and np.isnan(bad["loss"][1]) and not np.isnan(bad["loss"][2])


# ----------------------------------------------------------------- backward

def _loss(x, res, W1, W2, gamma, eps, dOut):
    return float((O.rmsnorm_block_unfused(x, res, W1, W2, gamma, eps)["out"] * dOut).sum())


def test_backward_matches_central_finite_differences():
    r = rng(13)
    M, K, N, N2 = 4, 8, 8, 12
    x, res = r.normal(size=(M, K)), r.normal(size=(M, N))
    W1, W2 = r.normal(size=(K, N)) / 3, r.normal(size=(N, N2)) / 3
    gamma, eps = 1 + 0.1 * r.normal(size=N), 1e-6
    dOut = r.normal(size=(M, N2))
    b = O.rmsnorm_block_backward_unfused(x, res, W1, W2, gamma, eps, dOut)
    step = 1e-6
    named = {"x": (x, "dx"), "res": (res, "dres"), "W1": (W1, "dW1"), "W2": (W2, "dW2"),
             "gamma": (gamma, "dgamma")}
    for name, (arr, gname) in named.items():
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + step
            lp = _loss(x, res, W1, W2, gamma, eps, dOut)
            arr[idx] = old - step
            lm = _loss(x, res, W1, W2, gamma, eps, dOut)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * step)
        scale = np.abs(fd).max()
        assert np.abs(fd - b[gname]).max() <= 1e-6 * scale, name


def test_rmsnorm_backward_invariant_and_dres():
    r = rng(14)
    M, K, N, N2 = 5, 6, 12, 7
    x, res = r.normal(size=(M, K)), r.normal(size=(M, N))
    W1, W2 = r.normal(size=(K, N)), r.normal(size=(N, N2))
    gamma, eps = 1 + 0.1 * r.normal(size=N), 0.05
    b = O.rmsnorm_block_backward_unfused(x, res, W1, W2, gamma, eps, r.normal(size=(M, N2)))
    lhs = (b["h"] * b["dh"]).sum(axis=1)
    rhs = b["r"] * b["c"] * eps / (b["ms"] + eps)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(b["dres"], b["dh"])


def test_block_local_backward_equals_chain_rule():
    r = rng(15)
    M, K, N, N2 = 17, 24, 40, 32
    args = (r.normal(size=(M, K)), r.normal(size=(M, N)), r.normal(size=(K, N)) / 5,
            r.normal(size=(N, N2)) / 6, 1 + 0.1 * r.normal(size=N), 1e-6, r.normal(size=(M, N2)))
    u = O.rmsnorm_block_backward_unfused(*args)
    for tile in (8, 256):
        p = O.rmsnorm_block_backward_reparam(*args, tile_cols=tile)
        for k in ("dW2", "dgamma", "dh", "dres", "dx", "dW1"):
            ref = u[k]
            np.testing.assert_allclose(p[k], ref, rtol=0, atol=1e-12 * np.abs(ref).max(), err_msg=k)


def test_backward_brute_force_small():
    r = rng(16)
    M, K, N, N2 = 2, 3, 4, 3
    x, res = r.normal(size=(M, K)), r.normal(size=(M, N))
    W1, W2 = r.normal(size=(K, N)), r.normal(size=(N, N2))
    gamma, eps, dOut = 1 + 0.1 * r.normal(size=N), 1e-6, r.normal(size=(M, N2))
    b = O.rmsnorm_block_backward_unfused(x, res, W1, W2, gamma, eps, dOut)
    h, y, _ = bf_block(x, res, W1, W2, gamma, eps)
    dy = bf_matmul(dOut, W2.T)
    np.testing.assert_allclose(b["dW2"], bf_matmul(y.T, dOut), rtol=1e-12)
    np.testing.assert_allclose(b["dy"], dy, rtol=1e-12)
    np.testing.assert_allclose(b["dx"], bf_matmul(b["dh"], W1.T), rtol=1e-12)
    np.testing.assert_allclose(b["dW1"], bf_matmul(x.T, b["dh"]), rtol=1e-12)


def test_tolerance_helper():
    ok, err, rms = O.tolerance_ok(np.array([1.0, -1.0]), np.array([1.0, -1.0 + 0.019]))
    assert ok and math.isclose(rms, math.sqrt((1 + (1 - 0.019) ** 2) / 2))
    ok, _, _ = O.tolerance_ok(np.array([1.0, -1.0]), np.array([1.0, -1.0 + 0.03]))
    assert not ok


def test_column_sampled_backward_equals_full_definition():
    r = rng(17)
    M, K, N, N2 = 9, 12, 16, 20
    args = (r.normal(size=(M, K)), r.normal(size=(M, N)), r.normal(size=(K, N)), r.normal(size=(N, N2)),
            1 + 0.1 * r.normal(size=N), 1e-6, r.normal(size=(M, N2)))
    full = O.rmsnorm_block_backward_unfused(*args)
    cols = np.array([0, 3, 19, 7])
    part = O.rmsnorm_block_backward_cols(*args, cols)
    np.testing.assert_array_equal(part["dW2_cols"], full["dW2"][:, cols])
    for k in ("dgamma", "dh", "dres", "dx", "dW1"):
        np.testing.assert_array_equal(part[k], full[k])


# --------------------------------------------------------------- SwiGLU backward

def test_silu_grad_closed_form_and_numerical_derivative():
    g = golden()
    v = O.silu_grad(np.array([0.0, 2.0]))
    assert v[0] == 0.5
    assert math.isclose(v[1], g["silu_grad_2"], rel_tol=1e-15)
    z = np.linspace(-30, 30, 61)
    h = 1e-6
    num = (O.silu(z + h) - O.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_grad(z), num, rtol=1e-7, atol=1e-9)


def _swiglu_loss(y, Wgu, Wd, res, dh2):
    return float((O.swiglu_down_unfused(y, Wgu, Wd, res)["h2"] * dh2).sum())


def test_swiglu_mlp_backward_matches_finite_differences():
    r = rng(18)
    M, N, F = 3, 5, 4
    y, Wgu, Wd, res = r.normal(size=(M, N)), r.normal(size=(N, 2 * F)) / 2, r.normal(size=(F, N)) / 2, \
        r.normal(size=(M, N))
    dh2 = r.normal(size=(M, N))
    b = O.swiglu_mlp_backward_unfused(y, Wgu, Wd, res, dh2)
    step = 1e-6
    for arr, gname in ((y, "d_y"), (Wgu, "dW_gu"), (Wd, "dW_down"), (res, "d_res")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + step
            lp = _swiglu_loss(y, Wgu, Wd, res, dh2)
            arr[idx] = old - step
            lm = _swiglu_loss(y, Wgu, Wd, res, dh2)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * step)
        assert np.abs(fd - b[gname]).max() <= 1e-6 * np.abs(fd).max(), gname


def test_swiglu_bwd_step_equals_chain_rule_and_brute_force():
    r = rng(19)
    M, N, F = 4, 6, 5
    y, Wgu, Wd = r.normal(size=(M, N)), r.normal(size=(N, 2 * F)), r.normal(size=(F, N))
    dh2 = r.normal(size=(M, N))
    b = O.swiglu_mlp_backward_unfused(y, Wgu, Wd, np.zeros((M, N)), dh2)
    st = O.gemm_swiglu_bwd(dh2, Wd, b["gate"], b["up"])
    np.testing.assert_allclose(st["d_gate"], b["d_gate"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st["d_up"], b["d_up"], rtol=1e-13, atol=1e-14)
    d_act = bf_matmul(dh2, Wd.T)
    for i in range(M):
        for j in range(F):
            gv, uv = b["gate"][i, j], b["up"][i, j]
            s = 1 / (1 + math.exp(-gv))
            assert math.isclose(st["d_gate"][i, j], d_act[i, j] * uv * s * (1 + gv * (1 - s)), rel_tol=1e-11,
                                abs_tol=1e-13)
            assert math.isclose(st["d_up"][i, j], d_act[i, j] * gv * s, rel_tol=1e-11, abs_tol=1e-13)
