"""Pins of the oracle's PISA-1 / PISA-2 node scores (close reading §04 4.3,
Eq.(8)-(9): the Taylor view of the Eq.(7) LSE and its two ablations).

PISA-1 scores a node by the mean of its children's logits, PISA-2 by that mean
plus half their variance. The pins use facts other than those formulas:
linearity (the mean of the logits is the logit of the mean key, i.e. the
node's own summary), Jensen's inequality against the exact LSE, the cumulant
expansion's error orders as the children's spread shrinks (which fixes both
the 1/2 and the population variance), and a single scored level against a
brute-force ranking of the Eq.(1) flat scores.
"""
import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import oracle
from tests.test_oracle_select import _brute_flat, _rand

PISA1, PISA2 = oracle.VARIANTS["pisa1"], oracle.VARIANTS["pisa2"]


@pytest.mark.parametrize("G", [1, 3])
def test_pisa1_is_the_logit_of_the_nodes_own_summary(G):
    N, C, d = 1024, 16, 12
    Kh = _rand((N, d), 1)
    P = oracle.build_pyramid(Kh, C)
    L, M, off = oracle.geometry(N, C)
    q = _rand((G, d), 2)
    for level in range(1, L + 1):
        for node in (0, M[level] // 2, M[level] - 1):
            want = sum(q[h] @ P[off[level] + node] for h in range(G)) / np.sqrt(d)
            got = oracle.node_score(q, Kh, P, level, node, C, variant=PISA1)
            assert got == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_pisa1_lower_bounds_the_normalised_lse():
    N, C, d = 2048, 32, 16
    Kh = _rand((N, d), 3) * 2.0
    P = oracle.build_pyramid(Kh, C)
    L, M, off = oracle.geometry(N, C)
    rng = np.random.default_rng(4)
    for _ in range(40):
        q = rng.standard_normal((1, d)) * 2.0
        level = int(rng.integers(1, L + 1))
        node = int(rng.integers(0, M[level]))
        n = C if level == 1 else 2
        lse = oracle.node_score(q, Kh, P, level, node, C)
        p1 = oracle.node_score(q, Kh, P, level, node, C, variant=PISA1)
        assert p1 <= lse - np.log(n) + 1e-12


def test_pisa2_is_the_second_order_cumulant_expansion():
    # children logits z_r = mu + eps * delta_r: LSE - log n = mu + eps^2 var(delta)/2 + O(eps^3),
    # so PISA-2 errs by O(eps^3) and PISA-1 by Theta(eps^2); the ratio of the
    # errors across eps = 1e-1 and 1e-2 shows the orders (8 = 2^3, 4 = 2^2 per halving)
    C, d = 16, 8
    base = _rand((1, d), 5)
    delta = _rand((C, d), 6)
    q = _rand((1, d), 7)

    def errors(eps):
        Kh = base + eps * delta
        P = oracle.build_pyramid(Kh, C)
        exact = oracle.node_score(q, Kh, P, 1, 0, C) - np.log(C)
        e1 = abs(exact - oracle.node_score(q, Kh, P, 1, 0, C, variant=PISA1))
        e2 = abs(exact - oracle.node_score(q, Kh, P, 1, 0, C, variant=PISA2))
        return e1, e2

    e1a, e2a = errors(0.02)
    e1b, e2b = errors(0.01)
    assert e1a / e1b == pytest.approx(4.0, rel=0.05)   # Theta(eps^2)
    assert e2a / e2b == pytest.approx(8.0, rel=0.15)   # O(eps^3)
    assert e2a < 0.05 * e1a


@pytest.mark.parametrize("causal", [True, False])
def test_single_scored_level_pisa1_is_the_flat_eq1_ranking(causal):
    # M_2 <= K: only the leaf level is scored; PISA-1's leaf score is the mean
    # raw-key logit, i.e. q . (mean key) / sqrt(d) -- the Eq.(1) flat score
    N, C, K, d = 512, 16, 16, 8
    Kh = _rand((N, d), 8)
    P = oracle.build_pyramid(Kh, C)
    M1 = N // C
    means = Kh.reshape(M1, C, d).mean(axis=1)
    rng = np.random.default_rng(9)
    ts = rng.integers(0, N, size=24)
    Q = _rand((len(ts), 1, d), 10)
    idx, _ = oracle.select_rows(Q, ts, Kh, P, C=C, K=K, causal=causal, variant=PISA1)
    for r, t in enumerate(ts):
        want = _brute_flat(lambda i: float(Q[r, 0] @ means[i]), int(t), N, C, K, causal, 7)
        got = [int(x) for x in idx[r] if x >= 0]
        assert got == want


def test_variants_change_only_the_ranking_key():
    # same walk structure: per-level candidate and scored counts are equal for
    # the three scores (they depend on t only), while selections may differ
    N, C, K, d = 4096, 64, 8, 16
    Kh = _rand((N, d), 11)
    P = oracle.build_pyramid(Kh, C)
    ts = np.array([4095, 3000, 2048, 1500])
    Q = _rand((4, 1, d), 12)
    ref = oracle.select_rows(Q, ts, Kh, P, C=C, K=K, want_counts=True)
    diff = 0
    for v in (PISA1, PISA2):
        idx, _, counts = oracle.select_rows(Q, ts, Kh, P, C=C, K=K, want_counts=True, variant=v)
        np.testing.assert_array_equal(counts, ref[2])
        diff += int((idx != ref[0]).any(axis=1).sum())
    assert diff > 0  # the scores do rank differently on random data
