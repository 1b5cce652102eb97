"""fp64 CPU oracle for the block-scaled (MXFP8) variant of the block.

TEST INFRASTRUCTURE ONLY, like ``coda_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU legs) may use it.  It
shares no code with the CUDA library.

Source: KuCoin news flash "CODA: new research optimizes transformer training
with GEMM epilogue programming", section "The lazy cost of training large
models" (low precision speeds up the products while the data movement around
them stays, so the epilogue's share grows).  The article gives no low-precision
recipe; this module states the readings the MXFP8 variant takes (each listed in
the design notes):

* The microscaling format (the OCP "Microscaling Formats (MX)" specification,
  v1.0): a block of 32 consecutive elements along the reduction dimension K
  shares one power-of-two scale 2^e, stored as an E8M0 byte e + 127 (biased
  exponent, no sign or mantissa); the elements are e4m3 codes (the codec of
  ``coda_oracle_fp8``).  A block holds v ~ 2^e decode(q).
* The scale exponent is the smallest e with amax(|v|) <= 448 2^e, so that no
  element saturates; e is clamped to [-127, 127] and an all-zero block takes
  e = 0.  (The specification's own choice, floor(log2 amax) - 8, saturates
  elements between 448 and 512 times the scale; the smallest non-saturating
  exponent is the reading taken here.)
* Codes are encode(v 2^-e): round to nearest, ties to the even code.  v 2^-e
  is exact, so the only rounding is the e4m3 one.
* Both GEMM operands are K-major and block-scaled along K: A [M, K] with
  scales [M, K/32], B stored as Bt [N, K] with scales [N, K/32].
* The scales travel in one of two byte layouts (the library's header states
  them): operand 0, the GEMM's left operand A (rows i, nrb = ceil(R / 128)
  row blocks): one 512-byte atom per (k-block, row block), E(i, j) at
  ((j // 4) nrb + i // 128) 512 + (i % 32) 16 + ((i // 32) % 4) 4 + j % 4;
  operand 1, the right operand B (ntl = ceil(R / 256) tiles): one 4 KB image
  per (k-block, 256-row tile), E(i, j) four times at ((j // 4) ntl + i // 256)
  4096 + ((i // 128) % 2) 2048 + rep 512 + (i % 32) 16 + ((i // 32) % 4) 4 +
  j % 4, rep = 0..3.  Bytes of padding rows hold 127 (scale 1).
* The block: the first GEMM keeps the per-tensor e4m3 operands of the FP8
  block; its epilogue forms hg = gamma h in full precision and quantises it
  into MXFP8 itself, block by block, so hg's scales are those of the data
  being written (no scale carried over from an earlier call).  The second
  GEMM multiplies the block-scaled hg by a block-scaled W2 and applies the
  row scale r of the folded light reduction.
"""
from __future__ import annotations

import math

import numpy as np

from . import coda_oracle_fp8 as F8

MX_BLOCK = 32
E4M3_MAX = 448.0
E_MIN, E_MAX = -127, 127


def mx_exponent(amax) -> np.ndarray:
    """Scale exponent of each block: the smallest integer e with
    amax <= 448 * 2^e, clamped to [-127, 127]; 0 for amax == 0."""
    a = np.asarray(amax, dtype=np.float64)
    out = np.zeros(a.shape, dtype=np.int32)
    for idx in np.ndindex(a.shape):
        v = float(a[idx])
        if v == 0.0:
            continue
        # a first guess from frexp, then step until the definition holds
        _, ex = math.frexp(v / E4M3_MAX)
        e = ex
        while math.ldexp(E4M3_MAX, e) < v:
            e += 1
        while math.ldexp(E4M3_MAX, e - 1) >= v:
            e -= 1
        out[idx] = min(max(e, E_MIN), E_MAX)
    return out


def mx_quantize(v):
    """MXFP8 codes and scale exponents of v [R, K] (K a multiple of 32):
    returns (codes uint8 [R, K], exponents int32 [R, K / 32])."""
    v = np.asarray(v, dtype=np.float64)
    R, K = v.shape
    assert K % MX_BLOCK == 0
    blocks = v.reshape(R, K // MX_BLOCK, MX_BLOCK)
    e = mx_exponent(np.abs(blocks).max(axis=2) if K else np.zeros((R, 0)))
    scaled = blocks * np.ldexp(1.0, -e)[:, :, None]
    codes = F8.e4m3_encode(scaled).reshape(R, K)
    return codes, e


def mx_dequantize(codes, exps) -> np.ndarray:
    """fp64 values 2^e decode(q) of MXFP8 data."""
    codes = np.asarray(codes, dtype=np.uint8)
    exps = np.asarray(exps, dtype=np.int64)
    R, K = codes.shape
    vals = F8.e4m3_decode(codes).reshape(R, K // MX_BLOCK, MX_BLOCK)
    return (vals * np.ldexp(1.0, exps)[:, :, None]).reshape(R, K)


def sf_rows_padded(R: int, operand: int = 0) -> int:
    """Rows the layout holds: whole 128-row blocks (A) or 256-row tiles (B)."""
    unit = 128 if operand == 0 else 256
    return -(-R // unit) * unit


def sf_bytes(R: int, K: int, operand: int = 0) -> int:
    """Size of the scale buffer of an [R, K] operand."""
    nkb = K // 128
    if operand == 0:
        return nkb * (sf_rows_padded(R, 0) // 128) * 512
    return nkb * (sf_rows_padded(R, 1) // 256) * 4096


def sf_offsets(i: int, j: int, R: int, operand: int = 0) -> list:
    """Byte offsets of the scale of row i, 32-block j (one for A, four for B)."""
    kb, s = j // 4, j % 4
    within = (i % 32) * 16 + ((i // 32) % 4) * 4 + s
    if operand == 0:
        nrb = sf_rows_padded(R, 0) // 128
        return [(kb * nrb + i // 128) * 512 + within]
    ntl = sf_rows_padded(R, 1) // 256
    base = (kb * ntl + i // 256) * 4096 + ((i // 128) % 2) * 2048 + within
    return [base + rep * 512 for rep in range(4)]


def sf_tile(exps, R: int, operand: int = 0):
    """E8M0 bytes of exponents [R, K/32] in the layout, and the mask of the
    bytes it defines (all of them; padding rows hold 127)."""
    exps = np.asarray(exps, dtype=np.int64)
    nblk = exps.shape[1]
    assert nblk % 4 == 0
    size = sf_bytes(R, nblk * MX_BLOCK, operand)
    buf = np.full(size, 127, dtype=np.uint8)
    used = np.zeros(size, dtype=bool)
    for i in range(sf_rows_padded(R, operand)):
        for j in range(nblk):
            for o in sf_offsets(i, j, R, operand):
                buf[o] = exps[i, j] + 127 if i < R else 127
                used[o] = True
    return buf, used


def sf_untile(buf, R: int, K: int, operand: int = 0) -> np.ndarray:
    """Exponents [R, K/32] read back from the layout (the first copy)."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    out = np.empty((R, K // MX_BLOCK), dtype=np.int32)
    for i in range(R):
        for j in range(K // MX_BLOCK):
            out[i, j] = int(buf[sf_offsets(i, j, R, operand)[0]]) - 127
    return out


def gemm_res_partialrms_mx(x8, sx, W1t8, sw1, res, gamma, tile_cols: int = 256) -> dict:
    """First GEMM of the MXFP8 block (per-tensor e4m3 operands):
    h = (decode(x8) decode(W1t8)^T) sx sw1 + res;  partial[t, i] = sum over
    column tile t of h^2;  hg = gamma h;  (hq, he) = mx_quantize(hg)."""
    acc = F8.e4m3_decode(x8) @ F8.e4m3_decode(W1t8).T
    h = acc * (np.float64(sx) * np.float64(sw1)) + np.asarray(res, dtype=np.float64)
    M, N = h.shape
    T = -(-N // tile_cols)
    partial = np.zeros((T, M))
    for t in range(T):
        blk = h[:, t * tile_cols:(t + 1) * tile_cols]
        partial[t] = (blk * blk).sum(axis=1)
    hg = np.asarray(gamma, dtype=np.float64)[None, :] * h
    hq, he = mx_quantize(hg)
    return {"h": h, "partial": partial, "hg": hg, "hq": hq, "he": he}


def gemm_rowscale_partial_mx(aq, ae, bq, be, partial=None, n_norm: int = 0, eps: float = 0.0) -> dict:
    """Second GEMM of the MXFP8 block: out = r * (A Bt^T) with A, Bt the
    dequantised block-scaled operands and r = 1 / sqrt(sum_t partial / N + eps)
    (r = 1 without partials: a plain MXFP8 GEMM)."""
    A = mx_dequantize(aq, ae)
    B = mx_dequantize(bq, be)
    acc = A @ B.T
    if partial is None:
        return {"r": None, "out": acc}
    r = 1.0 / np.sqrt(np.asarray(partial, dtype=np.float64).sum(axis=0) / n_norm + eps)
    return {"r": r, "out": r[:, None] * acc}


def rmsnorm_block_mx(x8, sx, W1t8, sw1, res, gamma, W2q, W2e, eps: float, tile_cols: int = 256) -> dict:
    """The MXFP8 block: the two steps above composed."""
    g1 = gemm_res_partialrms_mx(x8, sx, W1t8, sw1, res, gamma, tile_cols)
    N = g1["h"].shape[1]
    g2 = gemm_rowscale_partial_mx(g1["hq"], g1["he"], W2q, W2e, g1["partial"], N, eps)
    return {**g1, "r": g2["r"], "out": g2["out"]}


def rmsnorm_block_mx_unfused(x8, sx, W1t8, sw1, res, gamma, W2q, W2e, eps: float) -> dict:
    """The MXFP8 block as separate operators, the comparison chain for the
    fused MXFP8 block, each intermediate stored in bf16 as the chain stores
    it: t = bf16((decode(x8) decode(W1t8)^T) sx sw1); h = bf16(t + res);
    r = 1 / sqrt(mean(h^2) + eps); y = bf16(gamma h r); (yq, ye) =
    mx_quantize(y); out = mx_dequantize(yq, ye) mx_dequantize(W2q, W2e)^T.
    Here the normalised y is quantised, block by block from its own values."""
    t = F8.round_bf16(F8.e4m3_decode(x8) @ F8.e4m3_decode(W1t8).T * (np.float64(sx) * np.float64(sw1)))
    h = F8.round_bf16(t + np.asarray(res, dtype=np.float64))
    N = h.shape[1]
    r = 1.0 / np.sqrt((h * h).sum(axis=1) / N + eps)
    y = F8.round_bf16(np.asarray(gamma, dtype=np.float64)[None, :] * h * r[:, None])
    yq, ye = mx_quantize(y)
    out = mx_dequantize(yq, ye) @ mx_dequantize(W2q, W2e).T
    return {"t": t, "h": h, "r": r, "y": y, "yq": yq, "ye": ye, "out": out}
