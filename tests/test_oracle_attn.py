"""Pins of the oracle's attention over selected blocks (close reading §02,
Eq.(2)) against dense softmax attention computed with numpy."""
import numpy as np
import pytest

from oracle import oracle


def _dense_attn(Q, K, V, causal):
    d = Q.shape[1]
    S = Q @ K.T / np.sqrt(d)
    if causal:
        S = np.where(np.tril(np.ones_like(S, dtype=bool)), S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=1, keepdims=True)
    return P @ V


@pytest.mark.parametrize("causal", [True, False])
def test_full_budget_is_dense_attention(causal):
    # K * C >= N: the walk keeps every eligible leaf and Eq.(2) becomes dense
    # (causal) softmax attention
    rng = np.random.default_rng(0)
    N, C, K, d = 64, 16, 4, 8
    Kh, Vh, Q = (rng.standard_normal((N, d)) for _ in range(3))
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    idx, _ = oracle.select_rows(Q, t, Kh, P, C=C, K=K, causal=causal, forced_mask=7 if causal else 0)
    O = oracle.attn_rows(Q, t, Kh, Vh, idx, C=C, causal=causal)
    np.testing.assert_allclose(O, _dense_attn(Q, Kh, Vh, causal), rtol=1e-12, atol=1e-12)


def test_single_block_is_attention_inside_that_block():
    rng = np.random.default_rng(1)
    N, C, d = 256, 32, 8
    Kh, Vh, Q = (rng.standard_normal((N, d)) for _ in range(3))
    t = np.full(8, N - 1, np.int64)
    idx = np.full((8, 3), -1, np.int32)
    idx[:, 0] = np.arange(8)
    O = oracle.attn_rows(Q[:8], t, Kh, Vh, idx, C=C, causal=True)
    for r in range(8):
        blk = slice(r * C, (r + 1) * C)
        ref = _dense_attn(Q[r:r + 1], Kh[blk], Vh[blk], False)
        np.testing.assert_allclose(O[r], ref[0], rtol=1e-12, atol=1e-12)


def test_causal_mask_inside_the_current_block():
    rng = np.random.default_rng(2)
    N, C, d = 64, 16, 4
    Kh, Vh, Q = (rng.standard_normal((N, d)) for _ in range(3))
    t = np.array([16, 20, 31], np.int64)
    idx = np.array([[1, -1], [1, -1], [1, -1]], np.int32)
    O, lse = oracle.attn_rows(Q[:3], t, Kh, Vh, idx, C=C, causal=True, want_lse=True)
    for r, tt in enumerate(t.tolist()):
        ks = slice(16, tt + 1)
        ref = _dense_attn(Q[r:r + 1], Kh[ks], Vh[ks], False)
        np.testing.assert_allclose(O[r], ref[0], rtol=1e-12, atol=1e-12)
        z = Kh[ks] @ Q[r] / np.sqrt(d)
        assert abs(lse[r] - (z.max() + np.log(np.exp(z - z.max()).sum()))) < 1e-12


def test_constant_values_give_that_value():
    N, C, d = 128, 16, 4
    rng = np.random.default_rng(3)
    Kh = rng.standard_normal((N, d))
    Vh = np.tile(np.array([1.5, -2.0, 0.25, 3.0]), (N, 1))
    t = np.arange(0, N, 5, dtype=np.int64)
    idx = np.tile(np.array([0, 2, 5, -1], np.int32), (len(t), 1))
    O = oracle.attn_rows(rng.standard_normal((len(t), d)), t, Kh, Vh, idx, C=C, causal=True)
    np.testing.assert_allclose(O, Vh[: len(t)], rtol=1e-13)


def test_no_visible_key_gives_zero():
    rng = np.random.default_rng(4)
    Kh, Vh = rng.standard_normal((64, 4)), rng.standard_normal((64, 4))
    O = oracle.attn_rows(rng.standard_normal((1, 4)), np.array([3]), Kh, Vh,
                         np.array([[2, -1]], np.int32), C=16, causal=True)
    assert np.all(O == 0.0)
