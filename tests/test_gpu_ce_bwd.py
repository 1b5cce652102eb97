"""Parity of the block-local LM-head cross-entropy backward with the fp64 oracle.

The backward recomputes each vocabulary chunk's logits from H and W and uses
the forward's saved log-sum-exp (section "CODA: the secret in the epilogue" of
the KuCoin news flash "CODA: new research optimizes transformer training with
GEMM epilogue programming": the backward inherits the block-local structure).
Small ragged shapes are compared in full; the full-size LM head (8192 tokens,
hidden 2048, vocabulary 128256) on sampled rows of dH and sampled columns of dW.
"""
import math

import numpy as np
import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding as C
from gemm_epilogue_transformer_02_b200 import synth
from oracle import coda_oracle as O
from tests._util import b, check, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


# V = 17000: two 8192-column chunks and a ragged third (the first two chunks'
# dH label corrections run inside the next chunk's gradient GEMM, the last
# one's in its own kernel)
@pytest.mark.parametrize("M,K,V,weighted", [(300, 136, 5000, False), (129, 64, 4104, True), (64, 256, 1000, False),
                                            (260, 64, 17000, True)])
def test_lmhead_ce_bwd_small(M, K, V, weighted):
    g = synth.make_gen(600 + V)
    H = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, V), std=1.5 / math.sqrt(K))
    labels = synth.labels_uniform(g, M, V)
    labels[0], labels[-1] = 0, V - 1
    d_loss = (torch.rand(M, generator=g) + 0.5) / M if weighted else None
    _, lse, _ = C.lmhead_ce(dev(H), dev(W), dev(labels))
    dH, dW = C.lmhead_ce_bwd(dev(H), dev(W), dev(labels), lse, d_loss=None if d_loss is None else dev(d_loss))
    C.poll_status()
    ref = O.cross_entropy_backward_unfused(b(H), b(W), labels.numpy(),
                                           None if d_loss is None else d_loss.double().numpy())
    check("dH", dH, ref["dH"])
    check("dW", dW, ref["dW"])


def test_lmhead_ce_bwd_fullsize_sampled():
    M, K, V = 8192, 2048, 128256
    H, W, labels = synth.lmhead_ce_inputs()
    Hd, Wd, Ld = dev(H), dev(W), dev(labels)
    _, lse, _ = C.lmhead_ce(Hd, Wd, Ld)
    dH, dW = C.lmhead_ce_bwd(Hd, Wd, Ld, lse)
    C.poll_status()
    Hb, Wb, lab = b(H), b(W), labels.numpy()
    # oracle lse of every token (row blocks keep the fp64 logits small)
    lse_ref = np.concatenate([O.cross_entropy_unfused(Hb[i:i + 512], Wb, lab[i:i + 512])["lse"]
                              for i in range(0, M, 512)])
    rng = np.random.default_rng(7)
    rows = np.sort(np.concatenate([[0, M - 1], rng.choice(np.arange(1, M - 1), 14, replace=False)]))
    ref_rows = O.cross_entropy_backward_unfused(Hb[rows], Wb, lab[rows], np.full(len(rows), 1.0 / M))
    check("dH (sampled rows)", dH[torch.as_tensor(rows, device="cuda")], ref_rows["dH"])
    cols = np.sort(np.concatenate([[0, V - 1], rng.choice(np.arange(1, V - 1), 30, replace=False)]))
    d = np.full(M, 1.0 / M)
    dW_ref = np.stack([O.matmul(Hb.T, O.lmhead_ce_grad_chunk(Hb, Wb[:, [v]], lab, lse_ref, int(v), d))[:, 0]
                       for v in cols], axis=1)
    check("dW (sampled columns)", dW[:, torch.as_tensor(cols, device="cuda")], dW_ref)


def test_lmhead_ce_bwd_repeated_labels_and_determinism():
    """Many tokens share a few labels, placed on both sides of 256-column
    bucket and 8192-column chunk boundaries; two tokens carry labels outside
    [0, V) (no onehot term).  Every dW label column sums its tokens' exact
    label entries in a fixed order, so two calls agree bit for bit."""
    M, K, V = 300, 136, 9000
    g = synth.make_gen(650)
    H = synth.normal_bf16(g, (M, K))
    W = synth.normal_bf16(g, (K, V), std=1.5 / math.sqrt(K))
    pool = torch.tensor([0, 1, 255, 256, 8191, 8192, 8999], dtype=torch.int64)
    labels = pool[torch.randint(0, len(pool), (M,), generator=g)]
    Hd, Wd, Ld = dev(H), dev(W), dev(labels)
    _, lse, _ = C.lmhead_ce(Hd, Wd, Ld)  # lse of every token (labels do not enter it)
    bad = labels.clone()
    bad[5], bad[200] = -1, V
    Bd = dev(bad)
    dH, dW = C.lmhead_ce_bwd(Hd, Wd, Bd, lse)
    dH2, dW2 = C.lmhead_ce_bwd(Hd, Wd, Bd, lse)
    C.poll_status()
    assert torch.equal(dH, dH2) and torch.equal(dW, dW2)
    ref = O.cross_entropy_backward_unfused(b(H), b(W), bad.numpy())
    check("dH", dH, ref["dH"])
    check("dW", dW, ref["dW"])
    check("dW label columns", dW[:, dev(pool)], ref["dW"][:, pool.numpy()])
