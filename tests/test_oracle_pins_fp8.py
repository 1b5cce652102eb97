"""Pins of the FP8 (e4m3) oracle (CPU only).

The e4m3 codec is pinned to closed-form values of the format, to ties and
saturation worked out by hand, and to torch's own float8_e4m3fn conversion
(a library routine); the FP8 block is pinned to pure-Python brute force on a
tiny ragged shape and to the exact block within e4m3's error bound.
"""
import math

import numpy as np
import pytest
import torch

from oracle import coda_oracle as O
from oracle import coda_oracle_fp8 as F8


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x3C, 1.5),
    (0x40, 2.0), (0x7E, 448.0), (0x77, 240.0), (0xB8, -1.0), (0xFE, -448.0), (0x80, -0.0)])
def test_e4m3_closed_forms(code, value):
    got = F8.e4m3_decode(np.array([code], dtype=np.uint8))[0]
    assert got == value and math.copysign(1.0, got) == math.copysign(1.0, value)


def test_e4m3_nan_codes_and_monotone_table():
    t = F8.e4m3_table()
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.isfinite(np.delete(t, [0x7F, 0xFF])).all()
    pos = t[:0x7F]
    assert (np.diff(pos) > 0).all() and len(pos) == 127


def test_e4m3_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(F8.e4m3_encode(F8.e4m3_decode(codes)), codes)


@pytest.mark.parametrize("v,code", [
    (1.0625, 0x38),            # halfway 1.0 (m=0) / 1.125 (m=1): even
    (1.1875, 0x3A),            # halfway 1.125 (m=1) / 1.25 (m=2): even
    (1.07, 0x39),              # nearer 1.125
    (2.0 ** -10, 0x00),        # halfway 0 / 2^-9: even (zero)
    (3 * 2.0 ** -10, 0x02),    # halfway 2^-9 (odd code) / 2^-8: even
    (15 * 2.0 ** -10, 0x08),   # halfway 7*2^-9 (0x07) / 2^-6 (0x08): even
    (448.0, 0x7E), (460.0, 0x7E), (464.0, 0x7E), (1e6, 0x7E), (-1e6, 0xFE),  # saturation
    (-2.0 ** -12, 0x80),       # rounds to zero, sign kept
])
def test_e4m3_ties_and_saturation(v, code):
    assert int(F8.e4m3_encode(np.array([v]))[0]) == code


def test_e4m3_encode_matches_torch_in_range():
    g = torch.Generator().manual_seed(5)
    v = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    v = v[v.abs() <= 448.0]
    want = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F8.e4m3_encode(v.double().numpy())
    np.testing.assert_array_equal(got, want)


def test_quantize_uses_fp32_scale_and_product():
    t = np.array([0.3, -1.7, 2.5e-3, 97.0], dtype=np.float32)
    s = F8.quant_scale(np.abs(t).max())
    assert s == np.float32(np.float32(97.0) / np.float32(448.0))
    q = F8.quantize(t, s)
    assert int(q[3]) == 0x7E  # the amax element maps to 448 exactly
    deq = F8.dequantize(q, s)
    # every element within half an e4m3 step (relative 2^-4) of its value, or below the subnormal step
    assert np.all(np.abs(deq - t) <= np.maximum(np.abs(t) * 2.0 ** -4, 2.0 ** -10 * float(s)) * (1 + 1e-6))
    assert F8.quant_scale(0.0) == np.float32(1.0)


def _brute_block(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, eps, tile):
    M, K = x8.shape
    N = W1t8.shape[0]
    N2 = W2t8.shape[0]
    d = F8.e4m3_table()
    h = [[sum(d[x8[i, k]] * d[W1t8[j, k]] for k in range(K)) * sx * sw1 + res[i, j] for j in range(N)]
         for i in range(M)]
    part = [[sum(h[i][j] ** 2 for j in range(t0, min(t0 + tile, N))) for i in range(M)]
            for t0 in range(0, N, tile)]
    r = [1.0 / math.sqrt(sum(part[t][i] for t in range(len(part))) / N + eps) for i in range(M)]
    hg8 = [[int(F8.e4m3_encode(np.array([gamma[j] * h[i][j] / s_hg]))[0]) for j in range(N)] for i in range(M)]
    out = [[r[i] * sum(d[hg8[i][k]] * d[W2t8[j, k]] for k in range(N)) * s_hg * sw2 for j in range(N2)]
           for i in range(M)]
    return np.array(h), np.array(part), np.array(r), np.array(hg8, dtype=np.uint8), np.array(out)


def _tiny_fp8_inputs(M, K, N, N2, seed):
    r = np.random.default_rng(seed)
    x8 = F8.e4m3_encode(r.normal(size=(M, K)) * 4)
    W1t8 = F8.e4m3_encode(r.normal(size=(N, K)) * 8)
    W2t8 = F8.e4m3_encode(r.normal(size=(N2, N)) * 8)
    res = r.normal(size=(M, N))
    gamma = 1 + 0.1 * r.normal(size=N)
    return x8, 0.25, W1t8, 1.0 / 64, res, gamma, W2t8, 1.0 / 128


def test_fp8_block_brute_force_tiny_ragged():
    x8, sx, W1t8, sw1, res, gamma, W2t8, sw2 = _tiny_fp8_inputs(3, 5, 7, 4, 11)
    s_hg = 0.01
    f = F8.rmsnorm_block_fp8(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, 1e-6, tile_cols=3)
    h, part, r, hg8, out = _brute_block(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, 1e-6, 3)
    np.testing.assert_allclose(f["h"], h, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(f["partial"], part, rtol=1e-13)
    np.testing.assert_allclose(f["r"], r, rtol=1e-13)
    np.testing.assert_array_equal(f["hg8"], hg8)
    np.testing.assert_allclose(f["out"], out, rtol=1e-12, atol=1e-12)
    assert f["amax"] == pytest.approx(np.abs(np.asarray(gamma)[None, :] * h).max(), rel=1e-15)


def test_fp8_block_within_e4m3_bound_of_exact_block():
    """With s_hg = amax/448 the only departure from the exact block evaluated on
    the dequantised GEMM operands is hg's rounding: |hg8 s - hg| <= 2^-4 |hg|
    (normal range) or half the subnormal step, so
    |out - out_exact| <= r sum_k (that bound) |W2|."""
    x8, sx, W1t8, sw1, res, gamma, W2t8, sw2 = _tiny_fp8_inputs(16, 32, 48, 24, 12)
    W1 = F8.dequantize(W1t8, sw1).T
    W2 = F8.dequantize(W2t8, sw2).T
    xe = F8.dequantize(x8, sx)
    exact = O.rmsnorm_block_unfused(xe, res, W1, W2, gamma, 1e-6)
    hg = np.asarray(gamma)[None, :] * exact["h"]
    s_hg = float(F8.quant_scale(np.abs(hg).max()))
    f = F8.rmsnorm_block_fp8(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, 1e-6)
    np.testing.assert_allclose(f["h"], exact["h"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f["r"], exact["r"], rtol=1e-12)
    step = np.maximum(np.abs(hg) * 2.0 ** -4, 2.0 ** -10 * s_hg)
    bound = exact["r"][:, None] * (step @ np.abs(W2))
    assert np.all(np.abs(f["out"] - exact["out"]) <= bound * (1 + 1e-9))
    assert np.abs(f["out"] - exact["out"]).max() > 0  # the quantisation is really there


def test_round_bf16_matches_torch_and_ties():
    g = torch.Generator().manual_seed(6)
    v = torch.randn(50000, generator=g, dtype=torch.float32) * 37.0
    want = v.to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(F8.round_bf16(v.double().numpy()), want)
    # halfway cases: 1 + 2^-8 lies between 1 and 1 + 2^-7 (odd last bit): even -> 1;
    # 1 + 3 * 2^-8 between 1 + 2^-7 (odd) and 1 + 2^-6 (even) -> 1 + 2^-6
    np.testing.assert_array_equal(F8.round_bf16([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)]),
                                  [1.0, 1 + 2.0 ** -6, -1.0])


def test_fp8_unfused_chain_brute_force_and_error_bound():
    """The unfused FP8 chain: pure-Python brute force on a tiny ragged shape,
    and with s_y = amax(y)/448 within e4m3's rounding of y of the exact block
    evaluated on the dequantised GEMM operands."""
    x8, sx, W1t8, sw1, res, gamma, W2t8, sw2 = _tiny_fp8_inputs(3, 5, 7, 4, 13)
    s_y = 0.002
    f = F8.rmsnorm_block_fp8_unfused(x8, sx, W1t8, sw1, res, gamma, s_y, W2t8, sw2, 1e-6)
    d = F8.e4m3_table()
    M, K, N, N2 = 3, 5, 7, 4
    def bf16(v):  # round to 8 significant bits, ties to even, written out for one value
        if v == 0:
            return 0.0
        e = math.floor(math.log2(abs(v))) - 7
        q = v / 2.0 ** e
        fl = math.floor(q)
        rq = fl + 1 if (q - fl > 0.5 or (q - fl == 0.5 and fl % 2 == 1)) else fl
        return rq * 2.0 ** e

    for i in range(M):
        t = [bf16(sum(d[x8[i, k]] * d[W1t8[j, k]] for k in range(K)) * sx * sw1) for j in range(N)]
        h = [bf16(t[j] + res[i, j]) for j in range(N)]
        r = 1.0 / math.sqrt(sum(v * v for v in h) / N + 1e-6)
        y8 = [int(F8.e4m3_encode(np.array([gamma[j] * h[j] * r / s_y]))[0]) for j in range(N)]
        assert list(f["y8"][i]) == y8
        for j in range(N2):
            want = sum(d[y8[k]] * d[W2t8[j, k]] for k in range(N)) * s_y * sw2
            assert f["out"][i, j] == pytest.approx(want, rel=1e-12, abs=1e-12)
    x8, sx, W1t8, sw1, res, gamma, W2t8, sw2 = _tiny_fp8_inputs(16, 32, 48, 24, 14)
    W2 = F8.dequantize(W2t8, sw2).T
    exact = O.rmsnorm_block_unfused(F8.dequantize(x8, sx), res, F8.dequantize(W1t8, sw1).T, W2, gamma, 1e-6)
    s_y = float(F8.quant_scale(np.abs(exact["y"]).max()))
    f = F8.rmsnorm_block_fp8_unfused(x8, sx, W1t8, sw1, res, gamma, s_y, W2t8, sw2, 1e-6)
    # e4m3's half step of y, and what the bf16 rounding of t and h (2^-8 each,
    # relative) carries into y (r moves by far less and is covered by 1.1)
    t_exact = F8.dequantize(x8, sx) @ F8.dequantize(W1t8, sw1).T
    carried = 1.1 * np.abs(gamma)[None, :] * exact["r"][:, None] * 2.0 ** -8 * (
        np.abs(t_exact) + np.abs(exact["h"]))
    step = 2.0 ** -4 * (np.abs(exact["y"]) + carried) + 2.0 ** -10 * s_y + carried
    assert np.all(np.abs(f["out"] - exact["out"]) <= (step @ np.abs(W2)) * (1 + 1e-9))
