"""Host logic of bench.py: the structural work model used for the roofline
(candidate/scored counts per level depend only on t for the causal walk) is
checked against the oracle's own per-level counts and selections."""
import numpy as np
import pytest

import bench
from oracle import oracle


@pytest.mark.parametrize("N,C,K,mask", [(4096, 16, 8, 7), (3000, 32, 6, 3), (2048, 64, 16, 7), (1000, 8, 5, 1)])
def test_walk_counts_match_oracle(N, C, K, mask):
    rng = np.random.default_rng(0)
    d = 8
    Kh = rng.standard_normal((N, d))
    P = oracle.build_pyramid(Kh, C)
    t = np.arange(N, dtype=np.int64)
    Q = rng.standard_normal((N, d))
    idx, _, counts = oracle.select_rows(Q, t, Kh, P, C=C, K=K, forced_mask=mask, want_counts=True)
    internal, leafkeys, attended = bench.walk_counts(N, C, K, mask)
    L = oracle.geometry(N, C)[0]
    want_internal = sum(counts[:, l - 1, 1] * 2 for l in range(2, L + 1))
    np.testing.assert_array_equal(internal, want_internal)
    np.testing.assert_array_equal(leafkeys, counts[:, 0, 1] * C)
    vis = np.array([sum(min(b * C + C, tt + 1) - b * C for b in row if b >= 0) for tt, row in zip(t, idx)])
    np.testing.assert_array_equal(attended, vis)
    forced = [{0} if mask & 1 else set() for _ in t]
    fvis = []
    for tt, row, f in zip(t.tolist(), idx, forced):
        c = tt // C
        if mask & 2 and c >= 1:
            f.add(c - 1)
        f.add(c)
        fvis.append(sum(min(b * C + C, tt + 1) - b * C for b in row if b in f))
    np.testing.assert_array_equal(bench.walk_counts.forced_keys, np.array(fvis))


def test_fp32_peak_formula():
    assert abs(bench.fp32_fma_peak_tflops(1965.0) - 74.45) < 0.01


def test_kernel_source_sections_resolve():
    # every kernel's measured-traffic key hashes existing files and section
    # markers (a renamed section would otherwise silently drop the record)
    for name, parts in bench.KERNEL_SOURCES.items():
        assert len(bench.source_sha(parts)) == 16, name


def test_measured_traffic_is_keyed_by_workload_and_source():
    assert bench.measured_traffic("stage1", "no_such_workload") is None
    rec = bench.measured_traffic("stage1", "mha8_n256k")
    assert rec is None or rec > 0
