"""Pins of the oracle's sparse-attention backward (fixed selected leaves):
against torch autograd in float64 on dense causal attention (when every leaf
is selected the sparse attention is the dense one), against central finite
differences on a small sparse case, and against autograd of the oracle's own
forward restated densely with a mask (a different computation path)."""
import numpy as np
import pytest
import torch

from oracle import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _dense_autograd(Q, K, V, dO, causal, mask=None):
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=True)  # [G, N, d]
    k = torch.tensor(K, dtype=torch.float64, requires_grad=True)  # [N, d]
    v = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    d = Q.shape[-1]
    s = torch.einsum("gnd,md->gnm", q, k) / np.sqrt(d)
    N = Q.shape[1]
    allow = torch.ones(N, N, dtype=torch.bool)
    if causal:
        allow &= torch.tril(torch.ones(N, N, dtype=torch.bool))
    if mask is not None:
        allow &= torch.tensor(mask)
    s = s.masked_fill(~allow, float("-inf"))
    o = torch.einsum("gnm,md->gnd", torch.softmax(s, dim=-1), v)
    o.backward(torch.tensor(dO, dtype=torch.float64))
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("G,causal", [(1, True), (3, True), (2, False)])
def test_all_leaves_selected_is_dense_attention(G, causal):
    N, C, d = 96, 16, 8
    M1 = N // C
    Q, K, V, dO = _rand((G, N, d), 1), _rand((N, d), 2), _rand((N, d), 3), _rand((G, N, d), 4)
    idx = np.tile(np.arange(M1, dtype=np.int32), (N, 1))
    got = oracle.attn_backward_rows(Q, K, V, idx, dO, C=C, causal=causal)
    want = _dense_autograd(Q, K, V, dO, causal)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=1e-10, atol=1e-12)


def test_sparse_selection_matches_a_masked_dense_autograd():
    N, C, d, K = 128, 16, 8, 3
    M1 = N // C
    rng = np.random.default_rng(5)
    idx = np.full((N, K), -1, np.int32)
    mask = np.zeros((N, N), bool)
    for t in range(N):
        c = t // C
        leaves = sorted(set([c] + list(rng.choice(c + 1, size=min(K - 1, c + 1), replace=False))))
        idx[t, :len(leaves)] = leaves
        for leaf in leaves:
            mask[t, leaf * C:(leaf + 1) * C] = True
    Q, Kk, V, dO = _rand((2, N, d), 6), _rand((N, d), 7), _rand((N, d), 8), _rand((2, N, d), 9)
    got = oracle.attn_backward_rows(Q, Kk, V, idx, dO, C=C, causal=True)
    want = _dense_autograd(Q, Kk, V, dO, True, mask)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=1e-10, atol=1e-12)


def test_central_differences_on_a_sparse_case():
    N, C, d, K = 48, 8, 4, 2
    rng = np.random.default_rng(10)
    idx = np.full((N, K), -1, np.int32)
    for t in range(N):
        c = t // C
        idx[t, 0] = c
        if c >= 2:
            idx[t, 1] = int(rng.integers(0, c))
        idx[t] = np.sort(np.where(idx[t] < 0, 10 ** 6, idx[t]))
        idx[t][idx[t] == 10 ** 6] = -1
    Q, Kk, V, W = _rand((1, N, d), 11), _rand((N, d), 12), _rand((N, d), 13), _rand((1, N, d), 14)

    def loss(Q_, K_, V_):  # <W, O>, so dO = W
        O = np.stack([oracle.attn_rows(Q_[0], np.arange(N), K_, V_, idx, C=C, causal=True)])
        return float((W * O).sum())

    dQ, dK, dV = oracle.attn_backward_rows(Q, Kk, V, idx, W, C=C, causal=True)
    eps = 1e-6
    for name, X, grad in (("Q", Q, dQ), ("K", Kk, dK), ("V", V, dV)):
        for flat in rng.choice(X.size, size=12, replace=False):
            Xp, Xm = X.copy(), X.copy()
            Xp.flat[flat] += eps
            Xm.flat[flat] -= eps
            args_p = {"Q": (Xp, Kk, V), "K": (Q, Xp, V), "V": (Q, Kk, Xp)}[name]
            args_m = {"Q": (Xm, Kk, V), "K": (Q, Xm, V), "V": (Q, Kk, Xm)}[name]
            num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert grad.flat[flat] == pytest.approx(num, rel=1e-6, abs=1e-8), name


@pytest.mark.parametrize("G,causal", [(1, True), (2, False)])
def test_sampled_backward_equals_the_full_backward(G, causal):
    # the sampled form (used at sizes where the full backward is too slow)
    # against the entries of the pinned full backward
    N, C, d, K = 300, 16, 8, 4
    rng = np.random.default_rng(31 + G)
    Q, Kh, Vh, dO = _rand((G, N, d), 32), _rand((N, d), 33), _rand((N, d), 34), _rand((G, N, d), 35)
    M1 = (N + C - 1) // C
    idx = np.full((N, K), -1, np.int64)
    for t in range(N):
        c = t // C
        pick = {0, c} | set(rng.choice(max(c, 1), size=min(K - 2, max(c, 1)), replace=False).tolist())
        pick = sorted(x for x in pick if x <= (c if causal else M1 - 1))[:K]
        idx[t, :len(pick)] = pick
    fQ, fK, fV = oracle.attn_backward_rows(Q, Kh, Vh, idx, dO, C=C, causal=causal)
    rows = [0, 17, 150, N - 1]
    leaves = [0, 5, M1 - 1]  # the last leaf is ragged (300 = 18 x 16 + 12)
    sQ, sK, sV = oracle.attn_backward_sampled(Q, Kh, Vh, idx, dO, C=C, causal=causal, rows=rows, leaves=leaves)
    np.testing.assert_allclose(sQ, fQ[:, rows], rtol=1e-12, atol=1e-12)
    for li, leaf in enumerate(leaves):
        n = min(C, N - leaf * C)
        np.testing.assert_allclose(sK[li, :n], fK[leaf * C:leaf * C + n], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sV[li, :n], fV[leaf * C:leaf * C + n], rtol=1e-12, atol=1e-12)
        assert not sK[li, n:].any() and not sV[li, n:].any()


@pytest.mark.parametrize("G,causal", [(1, True), (3, True), (2, False)])
def test_leaf_backward_equals_the_full_backward(G, causal):
    # the batched per-leaf form (normaliser and output from attn_rows, every
    # user of the leaf at once) against the rows of the pinned full backward,
    # on every leaf, the ragged last one included
    N, C, d, K = 300, 16, 8, 5
    rng = np.random.default_rng(41 + G)
    Q, Kh, Vh, dO = _rand((G, N, d), 42), _rand((N, d), 43), _rand((N, d), 44), _rand((G, N, d), 45)
    M1 = (N + C - 1) // C
    idx = np.full((N, K), -1, np.int64)
    for t in range(N):
        c = t // C
        pick = {0, c} | set(rng.choice(max(c, 1), size=min(K - 2, max(c, 1)), replace=False).tolist())
        pick = sorted(x for x in pick if x <= (c if causal else M1 - 1))[:K]
        idx[t, :len(pick)] = pick
    _, fK, fV = oracle.attn_backward_rows(Q, Kh, Vh, idx, dO, C=C, causal=causal)
    for leaf in range(M1):
        lK, lV = oracle.attn_backward_leaf(Q, Kh, Vh, idx, dO, leaf, C=C, causal=causal)
        n = min(C, N - leaf * C)
        np.testing.assert_allclose(lK[:n], fK[leaf * C:leaf * C + n], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lV[:n], fV[leaf * C:leaf * C + n], rtol=1e-10, atol=1e-12)
        assert not lK[n:].any() and not lV[n:].any()
