"""Pins of the oracle's pyramid walk, node scores and flat selections.

Each test checks the oracle against something other than itself: the page's
printed per-level walk-through, brute force with numpy/scipy, closed forms
(Jensen bounds, exact leaf LSE), constructed inputs with a known answer, and
degenerate cases that reduce to textbook routines.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "level_tables.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _eligible_leaves(t, N, C, causal):
    M1 = -(-N // C)
    return [i for i in range(M1) if (not causal) or i * C <= t]


def _forced(t, C, causal, mask):
    c = t // C
    f = set()
    if mask & 1:
        f.add(0)
    if mask & 2 and c >= 1:
        f.add(c - 1)
    if mask & 4 or causal:
        f.add(c)
    return f


def _brute_flat(score_fn, t, N, C, K, causal, mask):
    """Forced leaves + best others by (score desc, index asc), via a full sort."""
    elig = _eligible_leaves(t, N, C, causal)
    if len(elig) <= K:
        return sorted(elig)
    F = [i for i in elig if i in _forced(t, C, causal, mask)]
    rest = [i for i in elig if i not in F]
    order = sorted(rest, key=lambda i: (-score_fn(i), i))
    return sorted(F + order[:K - len(F)])


# ---------------------------------------------------------------- golden ----

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: f"N{c['N']}K{c['K']}")
def test_level_tables_from_the_page(case):
    N, C, K = case["N"], case["C"], case["K"]
    d = 8
    Kh = _rand((N, d), 10)
    P = oracle.build_pyramid(Kh, C)
    L, _, _ = oracle.geometry(N, C)
    assert L == case["L"]
    t = np.array([5, N // 3, N - 1], np.int64)
    Q = _rand((len(t), d), 11)
    idx, gap, counts = oracle.select_rows(Q, t, Kh, P, C=C, K=K, causal=False, forced_mask=0,
                                          want_counts=True)
    for row in range(len(t)):
        for lv in case["levels"]:
            l = lv["level"]
            assert counts[row, l - 1, 0] == lv["candidates"], (row, l)
            assert counts[row, l - 1, 1] == lv["scored"], (row, l)
            assert C * 2 ** (l - 1) == lv["tokens_per_node"]
        assert counts[row, 0, 1] * C == case["leaf_keys_scored"]
        assert (idx[row] >= 0).sum() == case["kept_leaves"]


# ------------------------------------------------------- Eq.(6) bounds ----

@pytest.mark.parametrize("causal,mask", [(True, 7), (False, 0), (True, 1)])
def test_eq6_bounds_and_output_shape(causal, mask):
    N, C, K, d = 1000, 8, 5, 8
    Kh = _rand((N, d), 20)
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    Q = _rand((N, d), 21)
    idx, gap, counts = oracle.select_rows(Q, t, Kh, P, C=C, K=K, causal=causal, forced_mask=mask,
                                          want_counts=True)
    assert (counts[:, :, 0] <= 2 * K).all()
    for r in range(N):
        row = idx[r]
        valid = row[row >= 0]
        assert np.all(np.diff(valid) > 0), "sorted ascending, no duplicates"
        assert np.all(row[len(valid):] == -1), "padding at the end"
        if causal:
            assert np.all(valid * C <= t[r]), "never a leaf wholly in the future"
            assert t[r] // C in valid, "current leaf kept"
        F = _forced(int(t[r]), C, causal, mask)
        assert F <= set(valid.tolist())
        n_elig = len(_eligible_leaves(int(t[r]), N, C, causal))
        assert len(valid) == min(K, n_elig)


# ------------------------------------------- single scored level == flat ----

@pytest.mark.parametrize("causal,mask,G", [(True, 7, 1), (False, 0, 1), (True, 3, 2), (False, 5, 4)])
def test_single_scored_level_is_exhaustive_lse_topk(causal, mask, G):
    # M_2 <= K: every coarse level keeps all candidates, so the walk reduces to
    # forced leaves + Top-K by exact LSE over each leaf's raw keys (Eq.7, l=1),
    # summed over the group (Eq.11): checked against scipy logsumexp + a sort.
    N, C, K, d = 100, 8, 7, 6   # M1 = 13, M2 = 7 <= K
    Kh = _rand((N, d), 30)
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    Q = _rand((N, G, d), 31)
    idx, _ = oracle.select_rows(Q, t, Kh, P, C=C, K=K, causal=causal, forced_mask=mask)
    idx_flat, _ = oracle.flat_rows("lse", Q, t, Kh, P, C=C, K=K, causal=causal, forced_mask=mask)
    np.testing.assert_array_equal(idx, idx_flat)
    for r in range(N):
        def score(i, r=r):
            keys = Kh[i * C:min(i * C + C, N)]
            return sum(logsumexp(keys @ Q[r, h] / np.sqrt(d)) for h in range(G))
        want = _brute_flat(score, r, N, C, K, causal, mask)
        got = idx[r][idx[r] >= 0].tolist()
        assert got == want, r


def test_bsa_is_flat_mean_summary_topk():
    # Eq.(1): score = q . kbar_i / sqrt(d) against every eligible leaf mean
    N, C, K, d = 300, 10, 6, 5
    Kh = _rand((N, d), 40)
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    Q = _rand((N, d), 41)
    idx, _ = oracle.flat_rows("bsa", Q, t, Kh, P, C=C, K=K)
    for r in range(0, N, 7):
        def score(i, r=r):
            return Kh[i * C:min(i * C + C, N)].mean(0) @ Q[r] / np.sqrt(d)
        assert idx[r][idx[r] >= 0].tolist() == _brute_flat(score, r, N, C, K, True, 7)


def test_bsa_with_unit_leaves_equals_exact_lse():
    # with C = 1 a leaf summary is its one raw key, so Eq.(1) and the exact
    # leaf LSE coincide
    N, K, d = 80, 9, 4
    Kh = _rand((N, d), 42)
    P = oracle.build_pyramid(Kh, 1)
    t = np.arange(N, dtype=np.int64)
    Q = _rand((N, d), 43)
    a, _ = oracle.flat_rows("bsa", Q, t, Kh, P, C=1, K=K)
    b, _ = oracle.flat_rows("lse", Q, t, Kh, P, C=1, K=K)
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------- node scores ----

def test_leaf_score_is_exact_lse_of_raw_keys():
    # close reading §04 4.3: at l = 1 Eq.(7) is the exact LSE over the raw
    # keys; minus log C it is the normalised true LSE F_q of the leaf
    N, C, d = 512, 16, 8
    Kh = _rand((N, d), 50)
    P = oracle.build_pyramid(Kh, C)
    q = _rand((1, d), 51)
    for i in range(0, N // C, 5):
        s = oracle.node_score(q, Kh, P, 1, i, C)
        z = Kh[i * C:(i + 1) * C] @ q[0] / np.sqrt(d)
        Fq = np.log(np.mean(np.exp(z)))
        assert abs((s - np.log(C)) - Fq) < 1e-12


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_jensen_sandwich_every_internal_node(seed):
    # close reading §04 4.3, Eq.(10): with equal children,
    #   mean_j m_j <= s - log g <= F_q(B)
    # m_j = q . (child mean) / sqrt d, F_q(B) = log mean_{k in B} exp(q . k / sqrt d)
    N, C, d, g = 2048, 16, 8, 2
    Kh = _rand((N, d), 60 + seed) * 1.5
    P = oracle.build_pyramid(Kh, C)
    L, M, _ = oracle.geometry(N, C)
    q = _rand((1, d), 70 + seed)
    for lvl in range(2, L + 1):
        span, cspan = C * 2 ** (lvl - 1), C * 2 ** (lvl - 2)
        for i in range(M[lvl]):
            s = oracle.node_score(q, Kh, P, lvl, i, C)
            m = [Kh[(2 * i + j) * cspan:(2 * i + j + 1) * cspan].mean(0) @ q[0] / np.sqrt(d)
                 for j in range(g)]
            Fq = np.log(np.mean(np.exp(Kh[i * span:(i + 1) * span] @ q[0] / np.sqrt(d))))
            mid = s - np.log(g)
            assert np.mean(m) <= mid + 1e-12
            assert mid <= Fq + 1e-12
            # and the middle term is exactly log mean exp of the child logits
            assert abs(mid - np.log(np.mean(np.exp(m)))) < 1e-12


def test_jensen_equality_when_children_are_constant():
    # equality at both ends when every key inside each child is the same
    N, C, d = 256, 8, 4
    base = _rand((N // C, d), 80)
    Kh = np.repeat(base, C, axis=0)
    P = oracle.build_pyramid(Kh, C)
    q = _rand((1, d), 81)
    s = oracle.node_score(q, Kh, P, 2, 3, C)
    z = Kh[3 * 2 * C:4 * 2 * C] @ q[0] / np.sqrt(d)
    assert abs((s - np.log(2)) - np.log(np.mean(np.exp(z)))) < 1e-12


def test_gqa_score_is_sum_over_heads():
    # Eq.(11): the group's node score is the sum of the heads' scores
    N, C, d = 512, 16, 8
    Kh = _rand((N, d), 90)
    P = oracle.build_pyramid(Kh, C)
    qg = _rand((4, d), 91)
    for lvl, i in [(1, 7), (2, 5), (3, 1), (5, 0)]:
        s = oracle.node_score(qg, Kh, P, lvl, i, C)
        parts = sum(oracle.node_score(qg[h:h + 1], Kh, P, lvl, i, C) for h in range(4))
        assert abs(s - parts) < 1e-11


# ------------------------------------------------ constructed answers ----

def test_planted_needles_are_found():
    # Leaves whose keys align with the query dominate the LSE of every
    # ancestor, so the greedy walk must reach all of them: the answer is the
    # forced leaves plus the needles, known by construction.
    rng = np.random.default_rng(100)
    N, C, K, d = 4096, 16, 8, 16      # 256 leaves, 9 levels
    Kh = rng.standard_normal((N, d)) * 0.1
    u = np.zeros(d)
    u[0] = 1.0
    needles = [17, 64, 130, 201, 240]  # K - 3 forced
    for leaf in needles:
        Kh[leaf * C:(leaf + 1) * C] += 6.0 * u
    P = oracle.build_pyramid(Kh, C)
    t = np.array([4095, 4000, 3900, 3880], np.int64)  # after every needle, c - 1 > 240
    Q = np.tile(6.0 * u, (len(t), 1)) + rng.standard_normal((len(t), d)) * 0.01
    idx, gap = oracle.select_rows(Q, t, Kh, P, C=C, K=K)
    for r in range(len(t)):
        c = int(t[r]) // C
        want = sorted(set(needles) | {0, c - 1, c})
        assert len(want) == K
        assert idx[r].tolist() == want


def test_all_equal_keys_ties_go_to_lower_index():
    # every eligible non-forced node ties exactly, so each level keeps the
    # forced path plus the lowest indices; the leaves kept are therefore the
    # forced ones plus the lowest-index other eligible leaves
    N, C, K, d = 1024, 16, 6, 8
    Kh = np.tile(_rand((1, d), 110), (N, 1))
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(0, N, 3, dtype=np.int64)
    Q = _rand((len(t), d), 111)
    idx, gap = oracle.select_rows(Q, t, Kh, P, C=C, K=K)
    for r, tt in enumerate(t.tolist()):
        F = _forced(tt, C, True, 7)
        elig = _eligible_leaves(tt, N, C, True)
        others = [i for i in elig if i not in F]
        want = sorted(F | set(others[:max(0, K - len(F))])) if len(elig) > K else elig
        assert idx[r][idx[r] >= 0].tolist() == want, tt
        if len(elig) > K:
            assert gap[r] == 0.0


def test_identical_group_heads_select_like_one_head():
    N, C, K, d = 1024, 16, 4, 8
    Kh = _rand((N, d), 120)
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    q1 = _rand((N, 1, d), 121)
    a, ga = oracle.select_rows(q1, t, Kh, P, C=C, K=K)
    b, gb = oracle.select_rows(np.repeat(q1, 4, axis=1), t, Kh, P, C=C, K=K)
    np.testing.assert_array_equal(a, b)
    fin = np.isfinite(ga)
    np.testing.assert_allclose(gb[fin], 4 * ga[fin], rtol=1e-9, atol=1e-12)


def test_budget_covering_everything_keeps_all_eligible():
    # K * C >= N: every eligible leaf is kept
    N, C, K, d = 64, 16, 4, 4
    Kh = _rand((N, d), 130)
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    idx, _ = oracle.select_rows(_rand((N, d), 131), t, Kh, P, C=C, K=K)
    for r in range(N):
        assert idx[r][idx[r] >= 0].tolist() == list(range(r // C + 1))


def test_decode_row_equals_prefill_row():
    # close reading §5.1/§5.3: the decode step selects for the newest token
    # against the pyramid of the prefix; the current path is forced, so the
    # future keys a prefill pyramid holds never change the answer
    rng = np.random.default_rng(140)
    N, cap, C, K, d = 700, 1024, 16, 5, 8
    Kh = rng.standard_normal((cap, d))
    Q = rng.standard_normal((N, d))
    Pfull = oracle.build_pyramid(Kh[:N], C)
    t = np.arange(N, dtype=np.int64)
    want, _ = oracle.select_rows(Q, t, Kh[:N], Pfull, C=C, K=K)
    P = np.zeros((oracle.total_nodes(cap, C), d))
    for n in range(N):
        oracle.pyramid_append(P, Kh, n, C, 2, cap)
        if n % 37 == 0 or n == N - 1:
            got, _ = oracle.select_rows(Q[n:n + 1], np.array([n]), Kh, P, C=C, K=K,
                                        N=n + 1, N_layout=cap)
            np.testing.assert_array_equal(got[0], want[n])
