"""Pins of the oracle's pyramid geometry and pooling (close reading §04 4.1,
Eq.(3)-(4)) against closed forms and numpy block means."""
import numpy as np
import pytest

from oracle import oracle


@pytest.mark.parametrize("N,C,L", [
    (4096, 64, 7),        # close reading §5.2: L = log2(4096/64) + 1 = 7
    (16384, 64, 9),       # close reading §5.2: L = log2(16384/64) + 1 = 9
    (1024, 16, 7),        # 64 leaves
    (262144, 64, 13),     # 4096 leaves
    (64, 64, 1),          # a single leaf is the root
    (65, 64, 2),
])
def test_level_count(N, C, L):
    got, M, _ = oracle.geometry(N, C, 2)
    assert got == L
    assert M[1] == -(-N // C) and M[L] == 1


def test_level_sizes_ragged():
    # Eq.(3): M_{l+1} = ceil(M_l / 2) starting from ceil(N / C)
    L, M, off = oracle.geometry(1000, 16, 2)
    assert M[1:] == [63, 32, 16, 8, 4, 2, 1]
    assert off[1:] == [0, 63, 95, 111, 119, 123, 125]
    assert oracle.total_nodes(1000, 16, 2) == 126


def test_equal_groups_give_block_mean_of_raw_keys():
    # close reading §04 4.1: with equal group sizes the recursion equals the
    # mean of all raw keys inside the block
    rng = np.random.default_rng(0)
    N, C, d = 1024, 16, 8
    K = rng.standard_normal((N, d))
    P = oracle.build_pyramid(K, C)
    L, M, off = oracle.geometry(N, C)
    for lvl in range(1, L + 1):
        span = C * 2 ** (lvl - 1)
        ref = K.reshape(M[lvl], span, d).mean(axis=1)
        np.testing.assert_allclose(P[off[lvl]:off[lvl] + M[lvl]], ref, rtol=1e-12, atol=1e-13)


def test_ragged_tail_means_existing_children():
    # the last leaf holds 1000 - 62*16 = 8 keys; the last node of level 2 has
    # one child; level 3's last node averages a full node and that one-child node
    rng = np.random.default_rng(1)
    N, C, d = 1000, 16, 4
    K = rng.standard_normal((N, d))
    P = oracle.build_pyramid(K, C)
    _, M, off = oracle.geometry(N, C)
    leaf62 = K[992:1000].mean(0)
    np.testing.assert_allclose(P[off[1] + 62], leaf62, rtol=1e-12)
    np.testing.assert_allclose(P[off[2] + 31], leaf62, rtol=1e-12)
    node_2_30 = (K[960:976].mean(0) + K[976:992].mean(0)) / 2
    np.testing.assert_allclose(P[off[3] + 15], (node_2_30 + leaf62) / 2, rtol=1e-12)
    # a ragged node is NOT the mean of its raw keys (unequal children)
    assert not np.allclose(P[off[3] + 15], K[960:1000].mean(0))


def test_batched_heads_match_single_head():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((2, 3, 200, 4))
    P = oracle.build_pyramid(K, 16)
    for b in range(2):
        for h in range(3):
            np.testing.assert_array_equal(P[b, h], oracle.build_pyramid(K[b, h], 16))


@pytest.mark.parametrize("n0,steps,cap", [(0, 70, 200), (37, 100, 256), (128, 129, 300)])
def test_incremental_append_equals_rebuild(n0, steps, cap):
    # close reading §5.3 (decode cache): appending key n and refreshing its
    # leaf and ancestors gives the pyramid a full rebuild would give
    rng = np.random.default_rng(3)
    C, d = 16, 4
    K = rng.standard_normal((cap, d))
    P = oracle.build_pyramid(K, C, N=max(n0, 1), N_layout=cap) if n0 else \
        np.zeros((oracle.total_nodes(cap, C), d))
    for n in range(n0, n0 + steps):
        oracle.pyramid_append(P, K, n, C, 2, cap)
        R = oracle.build_pyramid(K, C, N=n + 1, N_layout=cap)
        L, M, off = oracle.geometry(cap, C)
        for lvl in range(1, L + 1):
            span = C * 2 ** (lvl - 1)
            live = -(-(n + 1) // span)
            np.testing.assert_allclose(P[off[lvl]:off[lvl] + live], R[off[lvl]:off[lvl] + live],
                                       rtol=1e-12, atol=1e-14)
