"""Comparison helpers for the GPU parity tests: run the CUDA path through the
C ABI and check it against the oracle element by element.

Acceptance rules:
  * pyramid: fp32 GPU summaries vs the fp64 oracle within |diff| <= 2e-6 + 1e-5 |x|;
  * indices: exactly equal to the oracle's, except rows whose smallest margin
    between the last kept and first dropped ranked score, over all levels,
    is below 1e-4 nats (a near-tie one fp32 rounding can flip); exempt rows
    must still be a valid selection (sorted, distinct, eligible, forced leaves
    present, min(K, eligible) entries);
  * outputs: the oracle's attention evaluated on the GPU's own indices, max
    abs error <= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

from hierarchical_block_sparse_b200 import pisa
from oracle import oracle

TIE_BAND = 1e-4
O_TOL = {"f32": 1e-4, "bf16": 2e-2}


def tdtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def gpu_prefill(w, Q, K, V, bsa: bool = False, ws: bool = False, variant: int = 0):
    """Run pisa_forward (or, with ws=True, the block-major pisa_forward_ws) and
    optionally pisa_bsa_select on cuda:0; returns GPU tensors. variant: the
    node score (0 Eq.7 LSE, 1 PISA-1, 2 PISA-2)."""
    dev = torch.device("cuda", 0)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    cfg = pisa.make_cfg(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=Q.shape[2], d=w.d, C=w.C, K=w.K, g=w.g, causal=w.causal,
                        forced_mask=w.forced_mask, dtype=Q.dtype, score_variant=variant)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    idx.fill_(-7)
    if ws:
        work = pisa.alloc_workspace(cfg, dev)
        work.fill_(0xAB)  # scratch must not need zeroing by the caller
        pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, work)
        assert pisa.pisa_workspace_status(cfg, work) == 0, "a tensor-core tile timed out"
    else:
        pisa.pisa_forward(cfg, Qd, Kd, Vd, pyr, idx, O)
    out = {"cfg": cfg, "pyr": pyr, "idx": idx, "O": O}
    if bsa:
        bidx = torch.full_like(idx, -7)
        pisa.pisa_bsa_select(cfg, Qd, pyr, bidx)
        out["bsa"] = bidx
    torch.cuda.synchronize()
    return out


def eligible(t, N, C, causal):
    M1 = -(-N // C)
    return min(M1, t // C + 1) if causal else M1


def forced(t, C, causal, mask):
    c = t // C
    f = set()
    if mask & 1:
        f.add(0)
    if mask & 2 and c >= 1:
        f.add(c - 1)
    if mask & 4 or causal:
        f.add(c)
    return f


def check_row_valid(row, t, N, C, K, causal, mask):
    row = np.asarray(row)
    v = row[row >= 0]
    assert np.all(row[len(v):] == -1), f"padding t={t}: {row}"
    assert np.all(np.diff(v) > 0), f"not sorted/distinct t={t}: {row}"
    n_el = eligible(t, N, C, causal)
    assert len(v) == min(K, n_el), f"count t={t}: {row}"
    assert np.all(v < n_el), f"ineligible leaf t={t}: {row}"
    assert forced(t, C, causal, mask) <= set(v.tolist()), f"forced missing t={t}: {row}"


def compare_indices(gpu_rows, ora_rows, gaps, t, w, N, what="select"):
    """Returns (n_rows, n_exempt, n_exempt_still_equal); asserts exact equality
    on non-exempt rows."""
    exempt = same = 0
    for r in range(len(t)):
        check_row_valid(gpu_rows[r], int(t[r]), N, w.C, w.K, w.causal, w.forced_mask)
        if gaps[r] < TIE_BAND:
            exempt += 1
            same += int(np.array_equal(gpu_rows[r], ora_rows[r]))
            continue
        assert np.array_equal(gpu_rows[r], ora_rows[r]), \
            f"{what} mismatch t={int(t[r])} gap={gaps[r]:.3g}\n gpu={gpu_rows[r]}\n ora={ora_rows[r]}"
    return len(t), exempt, same


def check_head(w, Q, K, V, res, b, kvh, rows, check_bsa=False, variant=0):
    """Check pyramid, selection and attention of one (b, kv-head) on query rows `rows`."""
    N = Q.shape[2]
    G = w.Hq // w.Hkv
    Kh = oracle.to_f64(K[b, kvh])
    Vh = oracle.to_f64(V[b, kvh])
    P = oracle.build_pyramid(Kh, w.C, w.g)
    gp = oracle.to_f64(res["pyr"][b, kvh])
    np.testing.assert_allclose(gp, P, rtol=1e-5, atol=2e-6)
    t = np.asarray(rows, np.int64)
    tt = torch.as_tensor(t)
    Qg = oracle.to_f64(Q[b, kvh * G:(kvh + 1) * G][:, tt]).transpose(1, 0, 2).copy()  # [n, G, d]
    idx_o, gap = oracle.select_rows(Qg, t, Kh, P, C=w.C, K=w.K, g=w.g, causal=w.causal,
                                    forced_mask=w.forced_mask, variant=variant)
    idx_g = res["idx"][b, kvh][tt.to(res["idx"].device)].cpu().numpy()
    n, ex, same = compare_indices(idx_g, idx_o, gap, t, w, N)
    # attention on the GPU's own indices, every head of the group
    worst = 0.0
    for h in range(G):
        O_o = oracle.attn_rows(Qg[:, h], t, Kh, Vh, idx_g, C=w.C, causal=w.causal)
        O_g = oracle.to_f64(res["O"][b, kvh * G + h][tt.to(res["O"].device)])
        worst = max(worst, float(np.max(np.abs(O_o - O_g))))
    assert worst <= O_TOL[w.dtype], f"attention max-abs error {worst} > {O_TOL[w.dtype]}"
    out = {"rows": n, "exempt": ex, "exempt_equal": same, "o_err": worst}
    if check_bsa:
        bidx_o, bgap = oracle.flat_rows("bsa", Qg, t, Kh, P, C=w.C, K=w.K, g=w.g, causal=w.causal,
                                        forced_mask=w.forced_mask)
        bidx_g = res["bsa"][b, kvh][tt.to(res["bsa"].device)].cpu().numpy()
        bn, bex, bsame = compare_indices(bidx_g, bidx_o, bgap, t, w, N, "bsa")
        out["bsa_exempt"] = bex
        out["bsa_exempt_equal"] = bsame
    return out


def sample_rows(N, C, n_random, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, C - 1, C, 2 * C + 5, N // 2, N - 2, N - 1]
    rnd = rng.integers(0, N, size=n_random).tolist()
    return sorted(set(r for r in fixed + rnd if 0 <= r < N))
