"""Pins of the MXFP8 oracle against things fixed outside it: a block worked
by hand (tests/golden/mx_worked_example.txt), closed forms of the scale rule,
the rule's defining inequality, the e4m3 rounding bound, exact round trips,
hand-computed offsets of the tiled scale layout and brute-force products.
A plausible slip (an off-by-one exponent, floor instead of the
non-saturating scale, a transposed operand, a wrong layout stride) fails at
least one of them."""
import math
import os

import numpy as np
import pytest

from oracle import coda_oracle_fp8 as F8
from oracle import coda_oracle_mx as MX

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mx_worked_example.txt")


def _read_worked():
    blocks, elems = {}, {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("block "):
                _, b, e = line.split()[:3]
                blocks[int(b)] = int(e)
            elif line.startswith("elem "):
                _, c, v, q = line.split()[:4]
                elems[int(c)] = (float(v), int(q, 16))
    return blocks, elems


def test_worked_example_by_hand():
    blocks, elems = _read_worked()
    v = np.zeros((1, 128))
    want = np.zeros(128, dtype=np.uint8)
    for c, (val, q) in elems.items():
        v[0, c] = val
        want[c] = q
    codes, exps = MX.mx_quantize(v)
    assert [int(x) for x in exps[0]] == [blocks[b] for b in range(4)]
    assert [hex(int(x)) for x in codes[0]] == [hex(int(x)) for x in want]


@pytest.mark.parametrize("amax,e", [
    (448.0, 0), (449.0, 1), (448.0 * (1 + 2 ** -40), 1), (224.0, -1), (224.0 * (1 + 2 ** -40), 0),
    (1.0, -8), (1.75, -8), (1.75 * (1 + 2 ** -30), -7), (0.0, 0), (2.0 ** -140, -127),
    (3.0e38, 120), (1e-3, -18),
])
def test_exponent_closed_forms(amax, e):
    # 1e-3: 448 * 2^-19 = 8.5e-4 < 1e-3 <= 448 * 2^-18 = 1.7e-3
    assert int(MX.mx_exponent(np.array([amax]))[0]) == e


def test_exponent_is_the_smallest_non_saturating_one():
    rng = np.random.default_rng(5)
    a = np.exp(rng.uniform(-60, 60, 4000))
    e = MX.mx_exponent(a)
    for ai, ei in zip(a, e):
        ei = int(ei)
        assert ai <= 448.0 * 2.0 ** ei
        assert 448.0 * 2.0 ** (ei - 1) < ai


def test_exponent_bit_rule_on_fp32():
    """The exponent from the fp32 bits of amax (E its unbiased exponent, m its
    fraction): E - 8 when the fraction is at most 0.75 (1.75 = 448 / 2^8),
    else E - 7 -- the rule a kernel can evaluate exactly -- equals the
    definition on fp32 values, at the boundaries and at random."""
    rng = np.random.default_rng(6)
    vals = np.concatenate([
        np.exp(rng.uniform(-80, 80, 3000)).astype(np.float32),
        np.array([448, 449, 1.75, 1.0, 224, 3.0e38, 1.2e-38], dtype=np.float32),
        np.nextafter(np.float32(1.75), np.float32(2)) * np.float32(2.0) ** np.arange(-20, 20, dtype=np.float32),
    ])
    for v in vals:
        bits = int(np.float32(v).view(np.uint32))
        E = (bits >> 23) - 127
        frac = bits & 0x7FFFFF
        e = E - 8 if frac <= 0x600000 else E - 7
        e = max(e, -127)
        assert e == int(MX.mx_exponent(np.array([float(v)]))[0]), v


def test_rounding_bound_and_tight_scale():
    rng = np.random.default_rng(7)
    v = rng.standard_normal((16, 256)) * np.exp(rng.uniform(-8, 8, (16, 1)))
    v[3, 32:64] = 0.0  # an all-zero block
    codes, exps = MX.mx_quantize(v)
    d = MX.mx_dequantize(codes, exps)
    scale = np.repeat(np.ldexp(1.0, exps), 32, axis=1)
    # e4m3 keeps 3 fraction bits: half an ulp is 2^-4 of the binade's base,
    # and below the normal range half a subnormal step is 2^-10 of the scale
    assert np.all(np.abs(d - v) <= 2.0 ** -4 * np.abs(v) + 2.0 ** -10 * scale)
    q = np.abs(F8.e4m3_decode(codes)).reshape(16, 8, 32).max(axis=2)
    nz = np.abs(v).reshape(16, 8, 32).max(axis=2) > 0
    # the block's largest value lands in (224, 448] before rounding, so its
    # code is at least 224 (rounding may take 225 down to 224) and at most 448
    amax = np.abs(v).reshape(16, 8, 32).max(axis=2) * np.ldexp(1.0, -exps)
    assert np.all((amax[nz] > 224) & (amax[nz] <= 448))
    assert np.all((q[nz] >= 224) & (q[nz] <= 448))
    assert np.all(q[~nz] == 0) and np.all(exps[~nz] == 0)


def test_round_trip_of_representable_blocks():
    rng = np.random.default_rng(8)
    R, K = 6, 128
    codes = rng.integers(0, 0x7F, (R, K)).astype(np.uint8) | (rng.integers(0, 2, (R, K)) << 7).astype(np.uint8)
    codes[:, ::32] = 0x7A | (codes[:, ::32] & 0x80)  # one element of 320 per block: the scale is recovered
    exps = rng.integers(-20, 20, (R, K // 32))
    v = MX.mx_dequantize(codes, exps)
    c2, e2 = MX.mx_quantize(v)
    assert np.array_equal(e2, exps)
    # -0 and +0 both decode to 0; the encoder keeps the sign of the value
    assert np.array_equal(F8.e4m3_decode(c2), F8.e4m3_decode(codes))


def test_sf_layout_offsets_by_hand():
    # A layout, R = 300 (3 row blocks).  Row 33, block 5: k-block 1 (step 1),
    # row block 0, lane 1, column 1 -> (1 * 3 + 0) * 512 + 16 + 4 + 1
    assert MX.sf_offsets(33, 5, 300, 0) == [1536 + 21]
    # row 299 (row block 2, lane 11, column 1), block 0: 2 * 512 + 176 + 4
    assert MX.sf_offsets(299, 0, 300, 0) == [1204]
    # row 127 (lane 31, column 3), block 7: (1 * 3) * 512 + 496 + 12 + 3
    assert MX.sf_offsets(127, 7, 300, 0) == [1536 + 511]
    assert MX.sf_bytes(300, 256, 0) == 2 * 3 * 512
    # B layout, R = 384 (2 tiles of 256 rows), K = 256 (2 k-blocks).  Row 300,
    # block 6: k-block 1 (step 2), tile 1, atom 0 of the tile, lane 12, column
    # (300 // 32) % 4 = 1 -> (1 * 2 + 1) * 4096 + 12 * 16 + 4 + 2, and its three
    # copies 512 bytes apart
    assert MX.sf_offsets(300, 6, 384, 1) == [12486, 12998, 13510, 14022]
    # row 130, block 0: tile 0, atom 1 (rows 128-255), lane 2, column 0
    assert MX.sf_offsets(130, 0, 384, 1) == [2080, 2592, 3104, 3616]
    assert MX.sf_bytes(384, 256, 1) == 2 * 2 * 4096
    assert MX.sf_bytes(300, 256, 1) == 2 * 2 * 4096  # 300 rows: two tiles, the second part padding
    rng = np.random.default_rng(9)
    for operand, R, K in ((0, 300, 256), (0, 1, 384), (1, 300, 256), (1, 128, 512)):
        e = rng.integers(-30, 30, (R, K // 32))
        buf, used = MX.sf_tile(e, R, operand)
        assert np.array_equal(MX.sf_untile(buf, R, K, operand), e)
        seen = np.zeros(buf.size, dtype=int)
        for i in range(MX.sf_rows_padded(R, operand)):
            for j in range(K // 32):
                for o in MX.sf_offsets(i, j, R, operand):
                    seen[o] += 1
        assert seen.max() == 1  # no two scales (or copies) share a byte
        assert np.array_equal(seen == 1, used)
        pad = [o for i in range(R, MX.sf_rows_padded(R, operand)) for j in range(K // 32)
               for o in MX.sf_offsets(i, j, R, operand)]
        assert np.all(buf[pad] == 127)  # padding rows: scale 1
        assert used.all()  # every byte belongs to a scale or a padding row
        if operand == 1:  # four copies of each scale
            for i in range(R):
                for j in range(K // 32):
                    assert len({int(buf[o]) for o in MX.sf_offsets(i, j, R, 1)}) == 1


def _brute_gemm(aq, ae, bq, be):
    """Pure-Python sum over k of 2^ea decode(a) 2^eb decode(b)."""
    M, K = aq.shape
    N = bq.shape[0]
    tab = F8.e4m3_table()
    out = np.zeros((M, N))
    for i in range(M):
        for n in range(N):
            terms = [tab[aq[i, k]] * 2.0 ** int(ae[i, k // 32]) * tab[bq[n, k]] * 2.0 ** int(be[n, k // 32])
                     for k in range(K)]
            out[i, n] = math.fsum(terms)
    return out


def test_mx_gemm_brute_force_ragged():
    rng = np.random.default_rng(10)
    M, N, K = 5, 3, 96
    aq, ae = MX.mx_quantize(rng.standard_normal((M, K)) * 3)
    bq, be = MX.mx_quantize(rng.standard_normal((N, K)) * 0.05)
    ref = _brute_gemm(aq, ae, bq, be)
    got = MX.gemm_rowscale_partial_mx(aq, ae, bq, be)["out"]
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-300)
    # with partials: r = 1 / sqrt(sum_t partial / N + eps) scales each row
    partial = rng.uniform(0.5, 2.0, (3, M))
    r = [1.0 / math.sqrt(math.fsum(partial[:, i]) / 7 + 1e-5) for i in range(M)]
    got = MX.gemm_rowscale_partial_mx(aq, ae, bq, be, partial, 7, 1e-5)
    assert np.allclose(got["r"], r, rtol=1e-14)
    assert np.allclose(got["out"], np.array(r)[:, None] * ref, rtol=1e-13)


def test_mx_block_first_gemm_matches_fp8_block_and_quantises_hg():
    rng = np.random.default_rng(11)
    M, K, N = 9, 64, 256 + 128
    x8 = F8.e4m3_encode(rng.standard_normal((M, K)))
    w8 = F8.e4m3_encode(rng.standard_normal((N, K)) * 4)
    res = rng.standard_normal((M, N))
    gamma = rng.uniform(0.5, 1.5, N)
    g = MX.gemm_res_partialrms_mx(x8, 0.5, w8, 0.125, res, gamma)
    f = F8.rmsnorm_block_fp8(x8, 0.5, w8, 0.125, res, gamma, 1.0, np.zeros((1, N), np.uint8), 1.0, 1e-5)
    assert np.allclose(g["h"], f["h"], rtol=1e-14, atol=1e-14)
    assert np.allclose(g["partial"], f["partial"], rtol=1e-14)
    # hg quantised block by block: the codes of one block, worked from its own amax
    blk = g["hg"][4, 160:192]
    e = int(MX.mx_exponent(np.array([np.abs(blk).max()]))[0])
    assert int(g["he"][4, 5]) == e
    assert np.array_equal(g["hq"][4, 160:192], F8.e4m3_encode(blk * 2.0 ** -e))


def test_mx_unfused_chain_steps():
    """The unfused MXFP8 chain: t, h and r as the FP8 chain's (the same
    GEMM, add and norm), y rounded to bf16 (8 significant bits) from
    gamma h r, then quantised block by block from its own values."""
    rng = np.random.default_rng(13)
    M, K, N, N2 = 7, 64, 128, 96
    x8 = F8.e4m3_encode(rng.standard_normal((M, K)))
    w8 = F8.e4m3_encode(rng.standard_normal((N, K)) * 4)
    res = rng.standard_normal((M, N))
    gamma = rng.uniform(0.5, 1.5, N)
    w2q, w2e = MX.mx_quantize(rng.standard_normal((N2, N)) * 0.1)
    u = MX.rmsnorm_block_mx_unfused(x8, 0.5, w8, 0.125, res, gamma, w2q, w2e, 1e-5)
    f = F8.rmsnorm_block_fp8_unfused(x8, 0.5, w8, 0.125, res, gamma, 1.0, np.zeros((1, N), np.uint8), 1.0, 1e-5)
    assert np.array_equal(u["t"], f["t"]) and np.array_equal(u["h"], f["h"])
    assert np.allclose(u["r"], f["r"], rtol=1e-15)
    y = u["y"]
    m, _ = np.frexp(y)
    assert np.all(np.abs(m * 256 - np.round(m * 256)) == 0)  # 8 significant bits
    assert np.all(np.abs(y - f["y"]) <= 2.0 ** -8 * np.abs(f["y"]))
    q, e = MX.mx_quantize(y)
    assert np.array_equal(q, u["yq"]) and np.array_equal(e, u["ye"])
    ref = _brute_gemm(u["yq"], u["ye"], w2q, w2e)
    assert np.allclose(u["out"], ref, rtol=1e-12, atol=1e-300)
