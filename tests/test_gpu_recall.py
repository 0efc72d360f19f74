"""Planted-retrieval workload (16 heads, N = 65536, 8 needle leaves per head):
Recall@K of the block-major selection against the oracle's exhaustive
per-leaf LSE Top-K, and the share of eligible needle leaves each of them keeps.

Recall has no published value to meet (the pages quote recall only for a
trained model); the numbers are printed for the record and held to loose
floors: a selection that ignored the scores would keep about K of the ~500
eligible leaves of an average row, i.e. a Recall@K of a few percent.
Rows are sampled where more than K leaves are eligible (t >= 4 K C).
"""
import json

import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200.workloads import WORKLOADS, make_inputs
from oracle import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def test_needle_recall_against_exhaustive_lse():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    w = WORKLOADS["needle_mha16_n64k"]
    Q, K, V, meta = make_inputs(w)
    out = parity.gpu_prefill(w, Q, K, V, ws=True)
    idx = out["idx"].cpu().numpy()[0]  # [H, N, K]
    rng = np.random.default_rng(7)
    rows_per_head = 24
    lo_t = 4 * w.K * w.C
    inter, need_p, need_x, need_n = [], 0, 0, 0
    for h in range(w.Hkv):
        t = np.sort(rng.choice(np.arange(lo_t, w.N), size=rows_per_head, replace=False))
        Kh = oracle.to_f64(K[0, h])
        P = oracle.build_pyramid(Kh, w.C)
        ex, _ = oracle.flat_rows("lse", oracle.to_f64(Q[0, h, torch.from_numpy(t)]), t, Kh, P, C=w.C, K=w.K)
        needles = meta["needles"][0, h]
        for r, tr in enumerate(t):
            got = set(idx[h, tr][idx[h, tr] >= 0].tolist())
            want = set(ex[r][ex[r] >= 0].tolist())
            inter.append(len(got & want) / w.K)
            elig = [int(n) for n in needles if n * w.C <= tr]
            need_n += len(elig)
            need_p += sum(n in got for n in elig)
            need_x += sum(n in want for n in elig)
    rec = {"recall_at_K": float(np.mean(inter)), "needle_recall_pisa": need_p / max(need_n, 1),
           "needle_recall_exhaustive": need_x / max(need_n, 1), "rows": len(inter), "eligible_needles": need_n}
    print("needle recall:", json.dumps(rec))
    assert rec["recall_at_K"] > 0.3
    assert rec["needle_recall_pisa"] >= 0.5 * rec["needle_recall_exhaustive"]
