"""Pins of the oracle's LM-head cross-entropy backward (CPU only).

Source: KuCoin news flash "CODA: new research optimizes transformer training
with GEMM epilogue programming", section "CODA: the secret in the epilogue"
(cross-entropy and the backward pass take the same re-parameterisation; a
block-local forward epilogue gives a block-local backward).  The chain-rule
definition is pinned to central finite differences of the summed losses; the
chunked block-local form (logits recomputed per vocabulary chunk with the
saved log-sum-exp) is pinned to the definition.
"""
import numpy as np

from oracle import coda_oracle as O


def _loss(H, W, labels, d):
    return float((O.cross_entropy_unfused(H, W, labels)["loss"] * d).sum())


def test_ce_backward_matches_finite_differences():
    r = np.random.default_rng(21)
    M, K, V = 3, 4, 7
    H, W = r.normal(size=(M, K)), r.normal(size=(K, V))
    labels = np.array([0, 6, 3])
    d = r.uniform(0.5, 2.0, size=M)
    b = O.cross_entropy_backward_unfused(H, W, labels, d)
    step = 1e-6
    for arr, name in ((H, "dH"), (W, "dW")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + step
            lp = _loss(H, W, labels, d)
            arr[idx] = old - step
            lm = _loss(H, W, labels, d)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * step)
        assert np.abs(fd - b[name]).max() <= 1e-7 * max(1.0, np.abs(fd).max()), name


def test_ce_gradient_rows_sum_to_zero_and_mean_default():
    r = np.random.default_rng(22)
    M, K, V = 5, 6, 11
    H, W = r.normal(size=(M, K)), r.normal(size=(K, V))
    labels = r.integers(0, V, size=M)
    b = O.cross_entropy_backward_unfused(H, W, labels)
    np.testing.assert_allclose(b["G"].sum(axis=1), 0.0, atol=1e-15)
    # default weighting is the mean over tokens
    b1 = O.cross_entropy_backward_unfused(H, W, labels, np.full(M, 1.0 / M))
    np.testing.assert_array_equal(b["dW"], b1["dW"])


def test_chunked_block_local_backward_equals_definition():
    r = np.random.default_rng(23)
    M, K, V = 9, 8, 23
    H, W = r.normal(size=(M, K)), r.normal(size=(K, V))
    labels = np.array([0, 22, 5, 11, 7, 7, 19, 1, 3])
    d = r.uniform(0.1, 1.0, size=M)
    lse = O.cross_entropy_unfused(H, W, labels)["lse"]
    ref = O.cross_entropy_backward_unfused(H, W, labels, d)
    for chunk in (1, 3, 7, 4096):
        got = O.lmhead_ce_bwd(H, W, labels, lse, d, chunk_cols=chunk)
        np.testing.assert_allclose(got["dH"], ref["dH"], rtol=0, atol=1e-13 * np.abs(ref["dH"]).max())
        np.testing.assert_allclose(got["dW"], ref["dW"], rtol=0, atol=1e-13 * np.abs(ref["dW"]).max())


def test_out_of_range_label_has_no_onehot_term():
    """A token whose label lies outside [0, V) keeps only the softmax part of
    its gradient: its row of G sums to d_i (a valid row sums to 0), equals
    d_i softmax(z_i) computed directly, and the chunked backward agrees."""
    r = np.random.default_rng(24)
    M, K, V = 4, 5, 9
    H, W = r.normal(size=(M, K)), r.normal(size=(K, V))
    labels = np.array([3, -1, V, 0])
    d = np.array([0.25, 0.5, 0.75, 1.0])
    b = O.cross_entropy_backward_unfused(H, W, labels, d)
    np.testing.assert_allclose(b["G"].sum(axis=1), [0.0, 0.5, 0.75, 0.0], atol=1e-15)
    z = H @ W
    for i in (1, 2):
        e = np.exp(z[i] - z[i].max())
        np.testing.assert_allclose(b["G"][i], d[i] * e / e.sum(), rtol=1e-13)
    lse = np.log(np.exp(z).sum(axis=1))
    got = O.lmhead_ce_bwd(H, W, labels, lse, d, chunk_cols=4)
    np.testing.assert_allclose(got["dW"], b["dW"], rtol=0, atol=1e-13 * np.abs(b["dW"]).max())
    np.testing.assert_allclose(got["dH"], b["dH"], rtol=0, atol=1e-13 * np.abs(b["dH"]).max())
