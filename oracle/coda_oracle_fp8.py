"""fp64 CPU oracle for the FP8 (e4m3) variant of the GEMM-RMSNorm-GEMM block.

TEST INFRASTRUCTURE ONLY, like ``coda_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU legs) may use it.  It
shares no code with the CUDA library.

Source: KuCoin news flash "CODA: new research optimizes transformer training
with GEMM epilogue programming".  Section "The lazy cost of training large
models": low-precision formats such as FP8 speed up the matrix products
while the cost of moving tensors in and out does not shrink with them, so the
share of the non-GEMM work grows; the article names FP8 only as that
motivation and gives no FP8 recipe.  The readings taken here (each listed in
the design notes):

* The format is OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits; subnormals at exponent field 0; no infinities; the
  code S.1111.111 is NaN; the largest finite magnitude is 448.
* Encoding rounds to nearest, ties to the even code, and saturates finite
  values beyond 448 to +-448 (the "satfinite" conversion); the sign of a value
  that rounds to zero is kept.
* Scaling is per tensor: a tensor t is held as codes q with t ~ s * decode(q);
  s = amax(|t|) / 448 (s = 1 for an all-zero tensor), computed in fp32, and
  q = encode(fp32(t) * fp32(1 / s)).  For the block's second operand hg the
  scale is the one the caller passes in (delayed scaling: derived from an
  earlier call's amax), and the call reports this call's amax.
* Both GEMM operands are K-major: x8 [M, K], W1t8 [N, K], hg8 [M, N],
  W2t8 [N2, N] (the weights stored transposed).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """Value of every one of the 256 codes (fp64; NaN for the two NaN codes)."""
    vals = np.empty(256)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_TABLE = e4m3_table()
_POS = _TABLE[:0x7F]  # codes 0x00 .. 0x7E: the finite non-negative values, increasing


def e4m3_decode(codes) -> np.ndarray:
    """fp64 value of each e4m3 code (uint8 array)."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    """Round-to-nearest-even, saturating encoding of real values to e4m3 codes."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    # index of the largest representable value <= a (a >= 0)
    lo = np.clip(np.searchsorted(_POS, a, side="right") - 1, 0, 0x7E)
    hi = np.minimum(lo + 1, 0x7E)
    dlo = a - _POS[lo]
    dhi = _POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (lo % 2 == 1))
    mag = np.where(pick_hi, hi, lo).astype(np.uint8)
    mag = np.where(a >= E4M3_MAX, np.uint8(0x7E), mag)
    out = mag | np.where(np.signbit(v), np.uint8(0x80), np.uint8(0))
    return np.where(np.isnan(v), np.uint8(0x7F), out).astype(np.uint8)


def quant_scale(amax) -> np.float32:
    """Per-tensor scale s = amax / 448 in fp32 (1 for an all-zero tensor)."""
    a = np.float32(amax)
    return np.float32(1.0) if a == 0 else np.float32(a / np.float32(E4M3_MAX))


def quantize(t, s) -> np.ndarray:
    """Codes of t under scale s: encode(fp32(t) * fp32(1 / s)), products in fp32."""
    inv = np.float32(np.float32(1.0) / np.float32(s))
    prod = (np.asarray(t, dtype=np.float32) * inv).astype(np.float32)
    return e4m3_encode(prod.astype(np.float64))


def dequantize(q, s) -> np.ndarray:
    return e4m3_decode(q) * np.float64(s)


def rmsnorm_block_fp8(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, eps: float,
                      tile_cols: int = 256) -> dict:
    """The block with e4m3 GEMM operands (fp64 arithmetic otherwise):

    h = (decode(x8) decode(W1t8)^T) sx sw1 + res;  partial[t, i] = sum over
    column tile t of h^2;  r = 1 / sqrt(sum_t partial / N + eps);
    hg = gamma * h;  hg8 = encode(hg / s_hg);  amax = max |hg|;
    out = r * (decode(hg8) decode(W2t8)^T) s_hg sw2.

    The RMS statistics come from h before any quantisation, as in the bf16
    block; only the second GEMM's operand hg is quantised."""
    acc1 = e4m3_decode(x8) @ e4m3_decode(W1t8).T
    h = acc1 * (np.float64(sx) * np.float64(sw1)) + np.asarray(res, dtype=np.float64)
    M, N = h.shape
    T = -(-N // tile_cols)
    partial = np.zeros((T, M))
    for t in range(T):
        blk = h[:, t * tile_cols:(t + 1) * tile_cols]
        partial[t] = (blk * blk).sum(axis=1)
    r = 1.0 / np.sqrt(partial.sum(axis=0) / N + eps)
    hg = np.asarray(gamma, dtype=np.float64)[None, :] * h
    hg8 = e4m3_encode(hg / np.float64(s_hg))
    acc2 = e4m3_decode(hg8) @ e4m3_decode(W2t8).T
    out = r[:, None] * acc2 * (np.float64(s_hg) * np.float64(sw2))
    return {"h": h, "partial": partial, "r": r, "hg": hg, "hg8": hg8,
            "amax": float(np.abs(hg).max()) if hg.size else 0.0, "out": out}


def round_bf16(v) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits), ties to even."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)               # v = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0), e - 8)  # numpy rounds halves to even


def rmsnorm_block_fp8_unfused(x8, sx, W1t8, sw1, res, gamma, s_y, W2t8, sw2, eps: float) -> dict:
    """The FP8 block as separate operators, the comparison chain for the fused
    FP8 block, each intermediate stored in bf16 as the chain stores it:
    t = bf16((decode(x8) decode(W1t8)^T) sx sw1); h = bf16(t + res);
    r = 1 / sqrt(mean(h^2) + eps); y = gamma * h * r; y8 = encode(y / s_y);
    amax = max |y|; out = (decode(y8) decode(W2t8)^T) s_y sw2.  Here the
    normalised y is quantised (its scale s_y the caller's, as for hg8)."""
    t = round_bf16(e4m3_decode(x8) @ e4m3_decode(W1t8).T * (np.float64(sx) * np.float64(sw1)))
    h = round_bf16(t + np.asarray(res, dtype=np.float64))
    N = h.shape[1]
    r = 1.0 / np.sqrt((h * h).sum(axis=1) / N + eps)
    y = np.asarray(gamma, dtype=np.float64)[None, :] * h * r[:, None]
    y8 = e4m3_encode(y / np.float64(s_y))
    out = e4m3_decode(y8) @ e4m3_decode(W2t8).T * (np.float64(s_y) * np.float64(sw2))
    return {"t": t, "h": h, "r": r, "y": y, "y8": y8,
            "amax": float(np.abs(y).max()) if y.size else 0.0, "out": out}
