"""Writes closed_forms.txt: closed-form values that pin the fp64 oracle.

Each value is evaluated from its formula with 40-digit decimal arithmetic;
nothing here comes from the CUDA library or from the oracle under test.
Formulas follow the definitions in the KuCoin news flash "CODA: new research
optimizes transformer training with GEMM epilogue programming"
(section "CODA: the secret in the epilogue": RMS normalisation of h = xW + res
with per-row scale r; SwiGLU; cross-entropy).
"""
import os
from decimal import Decimal, getcontext

getcontext().prec = 40
EPS = Decimal("1e-6")


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


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.txt")
    with open(path, "w") as f:
        f.write("# name value formula (written by make_closed_forms.py; 40-digit decimal)\n")
        for name, val, formula in rows():
            f.write(f"{name} {val:.25e} {formula}\n")


if __name__ == "__main__":
    main()
