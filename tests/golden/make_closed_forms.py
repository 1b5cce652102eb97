"""Writes closed_forms.txt: closed-form values that pin the fp64 oracle.

Each value is evaluated from its formula with 40-digit decimal arithmetic;
nothing here comes from the CUDA library or from the oracle under test.
Formulas follow the definitions in the KuCoin news flash "CODA: new research
optimizes transformer training with GEMM epilogue programming"
(section "CODA: the secret in the epilogue": RMS normalisation of h = xW + res
with per-row scale r; SwiGLU; cross-entropy; RoPE).  The article names RoPE
without its formula; its frequencies are the ones RoFormer (Su et al., 2021,
"RoFormer: Enhanced Transformer with Rotary Position Embedding", section 3.2.2)
publishes: pair i of a d-wide head turns by pos * base^(-2(i-1)/d) for
i = 1..d/2 (base 10000 there; LLaMA 3 uses 500000).
"""
import os
from decimal import Decimal, getcontext

getcontext().prec = 40
EPS = Decimal("1e-6")


def _cos_sin(x):
    """cos x and sin x by their Taylor series in 40-digit decimal arithmetic."""
    c, s_, term, k = Decimal(0), Decimal(0), Decimal(1), 0
    while True:
        # term = x^k / k!
        if k % 4 == 0:
            c += term
        elif k % 4 == 1:
            s_ += term
        elif k % 4 == 2:
            c -= term
        else:
            s_ -= term
        k += 1
        term = term * x / k
        if abs(term) < Decimal("1e-45"):
            return c, s_


def rows():
    one = Decimal(1)
    yield ("rms_const_row_c1", one / (one + EPS).sqrt(),
           "RMSNorm of a constant row h_j = c with gamma = 1: y_j = c / sqrt(c^2 + eps), c = 1, eps = 1e-6")
    yield ("rms_const_row_cm3", Decimal(-3) / (Decimal(9) + EPS).sqrt(),
           "same with c = -3")
    yield ("silu_1", one / (one + (-one).exp()), "silu(1) = 1 / (1 + e^-1)")
    yield ("silu_m2", Decimal(-2) / (one + Decimal(2).exp()), "silu(-2) = -2 / (1 + e^2)")
    sig2 = one / (one + Decimal(-2).exp())
    yield ("silu_grad_2", sig2 * (one + 2 * (one - sig2)),
           "silu'(2) = s (1 + 2 (1 - s)), s = 1 / (1 + e^-2)")
    yield ("ce_uniform_V128256", Decimal(128256).ln(),
           "cross-entropy with all logits equal (W = 0), V = 128256: loss = ln V")
    yield ("ce_uniform_V1000", Decimal(1000).ln(), "same with V = 1000")
    L, V = Decimal(5), Decimal(1000)
    yield ("ce_single_logit_L5_V1000", (one + (V - 1) * (-L).exp()).ln(),
           "logit L = 5 at the label, 0 elsewhere, V = 1000: loss = ln(1 + (V-1) e^-L)")
    # RoPE (RoFormer's frequencies, 0-based pair index i: base^(-2i/d)).  Base
    # 10000, d = 64, pair i = 16: 10000^(-1/2) = 1/100, so position 100 turns by
    # exactly 1 radian.
    c1, s1 = _cos_sin(one)
    yield ("rope_cos_b10000_d64_i16_p100", c1, "RoPE pair i = 16 of a 64-wide head, base 10000, position 100: cos(100 * 10000^(-32/64)) = cos 1")
    yield ("rope_sin_b10000_d64_i16_p100", s1, "same pair: sin 1")
    # base 500000 (LLaMA 3), d = 128, pair i = 32: 500000^(-1/2); position 707
    ang = Decimal(707) / Decimal(500000).sqrt()
    c2, s2 = _cos_sin(ang)
    yield ("rope_cos_b500000_d128_i32_p707", c2, "RoPE pair i = 32 of a 128-wide head, base 500000, position 707: cos(707 / sqrt(500000))")
    yield ("rope_sin_b500000_d128_i32_p707", s2, "same pair: sin(707 / sqrt(500000))")


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.txt")
    with open(path, "w") as f:
        f.write("# name value formula (written by make_closed_forms.py; 40-digit decimal)\n")
        for name, val, formula in rows():
            f.write(f"{name} {val:.25e} {formula}\n")


if __name__ == "__main__":
    main()
