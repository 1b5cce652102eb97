"""Pins of the oracle's RoPE in the QKV projection (CPU only).

Source: KuCoin news flash "CODA: new research optimizes transformer training
with GEMM epilogue programming", section "CODA: the secret in the epilogue"
(RoPE, rotary position encoding, takes the same re-parameterisation) and
section "Five kinds of building blocks" (RoPE as an elementwise transform).
The rotate-half form with angle pos * theta^(-2i/d) is the plain reading.
Pins: position 0 is the identity; every rotated pair keeps its norm; the
q.k product of two rotated vectors depends only on the position difference;
brute force with Python's math on a tiny case.  Those hold for any choice of
frequencies, so the frequencies themselves are pinned against values fixed by
the published source of RoPE, RoFormer (Su et al., 2021, section 3.2.2: pair i
of a d-wide head turns by pos * base^(-2(i-1)/d), i = 1..d/2), evaluated in
40-digit decimal arithmetic in tests/golden/closed_forms.txt.
"""
import math
import os

import numpy as np
import pytest

from oracle import coda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, val = line.split()[:2]
            out[name] = float(val)
    return out


# (base, head width d, 0-based pair index, position, golden key suffix)
@pytest.mark.parametrize("base,d,i,pos,key", [(10000.0, 64, 16, 100, "b10000_d64_i16_p100"),
                                              (500000.0, 128, 32, 707, "b500000_d128_i32_p707")])
def test_frequencies_match_roformer(base, d, i, pos, key):
    """A unit vector on the first column of pair i, and one on its partner,
    turned by one position: the outputs are the cosine and sine of the
    angle RoFormer's frequency gives.  A frequency exponent of -i/d instead of
    -2i/d, a pair of (i, i+1) instead of (i, i + d/2), or a swapped sign of
    the rotation fails here."""
    g = _golden()
    c, s = g["rope_cos_" + key], g["rope_sin_" + key]
    t = np.zeros((2, 2 * d))
    t[0, d + i] = 1.0          # second head, first column of pair i
    t[1, d + i + d // 2] = 1.0  # second head, partner column
    out = O.rope_rotate(t, [pos, pos], d, base)
    np.testing.assert_allclose([out[0, d + i], out[0, d + i + d // 2]], [c, s], rtol=0, atol=1e-13)
    np.testing.assert_allclose([out[1, d + i], out[1, d + i + d // 2]], [-s, c], rtol=0, atol=1e-13)
    rest = np.ones(2 * d, dtype=bool)
    rest[[d + i, d + i + d // 2]] = False
    assert not np.any(out[:, rest])


def test_position_zero_is_identity_and_pairs_keep_norm():
    r = np.random.default_rng(31)
    t = r.normal(size=(3, 16))
    np.testing.assert_allclose(O.rope_rotate(t, [0, 0, 0], 8, 10000.0), t, rtol=0, atol=0)
    pos = [5, 1000, 8191]
    out = O.rope_rotate(t, pos, 8, 500000.0)
    for h0 in (0, 8):
        n_in = t[:, h0:h0 + 4] ** 2 + t[:, h0 + 4:h0 + 8] ** 2
        n_out = out[:, h0:h0 + 4] ** 2 + out[:, h0 + 4:h0 + 8] ** 2
        np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def test_relative_position_property():
    r = np.random.default_rng(32)
    q, k = r.normal(size=(1, 8)), r.normal(size=(1, 8))
    dots = []
    for p in (3, 40, 1000):
        qr = O.rope_rotate(q, [p + 7], 8, 10000.0)
        kr = O.rope_rotate(k, [p], 8, 10000.0)
        dots.append(float((qr * kr).sum()))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


def test_brute_force_tiny():
    r = np.random.default_rng(33)
    d, theta = 4, 100.0
    t = r.normal(size=(2, 2 * d))
    pos = [3, 11]
    out = O.rope_rotate(t, pos, d, theta)
    for m in range(2):
        for h0 in (0, d):
            for i in range(d // 2):
                ang = pos[m] * theta ** (-2 * i / d)
                a, b = t[m, h0 + i], t[m, h0 + i + d // 2]
                assert math.isclose(out[m, h0 + i], a * math.cos(ang) - b * math.sin(ang), rel_tol=1e-12,
                                    abs_tol=1e-14)
                assert math.isclose(out[m, h0 + i + d // 2], b * math.cos(ang) + a * math.sin(ang),
                                    rel_tol=1e-12, abs_tol=1e-14)


def test_qkv_rope_leaves_v_columns():
    r = np.random.default_rng(34)
    x, W = r.normal(size=(4, 6)), r.normal(size=(6, 24))
    out = O.qkv_rope_unfused(x, W, [0, 1, 2, 3], 8, 16, 10000.0)
    qkv = x @ W
    np.testing.assert_allclose(out[:, 16:], qkv[:, 16:], rtol=1e-14)
    np.testing.assert_allclose(out[:, :16], O.rope_rotate(qkv[:, :16], [0, 1, 2, 3], 8, 10000.0), rtol=1e-14)


def test_rotations_compose_and_negative_positions_invert():
    """Rotations by positions add: rotating by p1 then p2 equals rotating by
    p1 + p2, and a negative position undoes the positive one (the kernel takes
    any int32 position)."""
    r = np.random.default_rng(35)
    t = r.normal(size=(3, 256))
    p1, p2 = [7, 2047, 123456], [5, -2047, 1_000_000]
    both = O.rope_rotate(O.rope_rotate(t, p1, 128, 500000.0), p2, 128, 500000.0)
    np.testing.assert_allclose(both, O.rope_rotate(t, np.add(p1, p2), 128, 500000.0), rtol=0, atol=1e-9)
    back = O.rope_rotate(O.rope_rotate(t, p1, 64, 500000.0), np.negative(p1), 64, 500000.0)
    np.testing.assert_allclose(back, t, rtol=0, atol=1e-9)
