"""GPU parity of the backward with the selection fixed -- the CUDA-core call
(pisa_sparse_attn_backward) and the tensor-core calls
(pisa_sparse_attn_backward_ws, pisa_sparse_attn_backward_saved_ws) -- against
the oracle's fp64 backward, on the selection the GPU itself made; at the
bench's size on sampled rows and leaves."""
import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import oracle

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_f32": WORKLOADS["tiny_f32_n1k"],
    "mha_bf16": Workload("bwd_mha", 150, B=2, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8),
    "gqa4_d64": Workload("bwd_gqa4", 151, B=1, Hq=8, Hkv=2, N=800, d=64, C=32, K=8),
    "noncausal_g2": Workload("bwd_nc", 152, B=1, Hq=4, Hkv=2, N=700, d=128, C=64, K=6, causal=False,
                             forced_mask=1),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    pisa.load()


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    dt = Q.dtype
    dO = torch.from_numpy(np.random.default_rng(w.seed + 7).standard_normal(Q.shape).astype(np.float32)).to(dt)
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, dt)
    pisa.pisa_forward(cfg, Qd, Kd, Vd, pyr, idx, O)
    dQ = torch.full(Q.shape, float("nan"), dtype=torch.float32, device=dev)
    dK = torch.full(K.shape, float("nan"), dtype=torch.float32, device=dev)
    dV = torch.full(V.shape, float("nan"), dtype=torch.float32, device=dev)
    pisa.pisa_sparse_attn_backward(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    worst = 0.0
    for b in range(w.B):
        for h in range(w.Hkv):
            hs = slice(h * G, (h + 1) * G)
            rQ, rK, rV = oracle.attn_backward_rows(
                oracle.to_f64(Q[b, hs]), oracle.to_f64(K[b, h]), oracle.to_f64(V[b, h]),
                idx[b, h].cpu().numpy(), oracle.to_f64(dO[b, hs]), C=w.C, causal=w.causal)
            for got, ref in ((dQ[b, hs], rQ), (dK[b, h], rK), (dV[b, h], rV)):
                g = got.cpu().double().numpy()
                assert np.isfinite(g).all()
                err = float(np.abs(g - ref).max()) / max(1.0, float(np.abs(ref).max()))
                worst = max(worst, err)
    tol = 1e-4 if w.dtype == "f32" else 1e-3
    assert worst <= tol, worst


# block-major tensor-core backward (bf16, d = 128, C = 64)
BM_CASES = {
    "mha_ragged": Workload("bwdbm_mha", 160, B=2, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8),
    "gqa4": Workload("bwdbm_gqa4", 161, B=1, Hq=8, Hkv=2, N=800, d=128, C=64, K=8),
    "g16": Workload("bwdbm_g16", 162, B=1, Hq=16, Hkv=1, N=512, d=128, C=64, K=4),
    "noncausal_first_only": Workload("bwdbm_nc1", 163, B=1, Hq=4, Hkv=2, N=700, d=128, C=64, K=6, causal=False,
                                     forced_mask=1),
    "noncausal_previous_only": Workload("bwdbm_nc2", 164, B=1, Hq=2, Hkv=2, N=640, d=128, C=64, K=6, causal=False,
                                        forced_mask=2),
    "causal_mask0": Workload("bwdbm_m0", 165, B=1, Hq=2, Hkv=1, N=600, d=128, C=64, K=4, forced_mask=0),
    # leaf 0's bucket spans 32 tiles and several CTAs' ranges: their partial dK / dV meet in global memory
    "mha_4k_many_tiles": Workload("bwdbm_4k", 166, B=1, Hq=2, Hkv=2, N=4096, d=128, C=64, K=16),
}
# P and dS enter the tensor cores as bf16 (relative rounding 2^-9 per product);
# the bar is the bf16 output tolerance, relative to the largest reference entry
BM_TOL = 2e-2


def _bm_backward(w, drop_first_leaf=False):
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    dO = torch.from_numpy(np.random.default_rng(w.seed + 7).standard_normal(Q.shape).astype(np.float32)).to(Q.dtype)
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, pisa.alloc_workspace(cfg, dev))
    if drop_first_leaf:  # a caller selection that omits a forced leaf on some rows
        t = torch.arange(w.N, device=dev).view(1, 1, w.N, 1)
        idx = torch.where((idx == 0) & (t % 3 == 1), torch.full_like(idx, -1), idx).contiguous()
    ws = pisa.alloc_backward_workspace(cfg, dev)
    ws.random_(0, 256)  # scratch must not leak into the results
    grads = [torch.full(x.shape, float("nan"), dtype=torch.float32, device=dev) for x in (Q, K, V)]
    pisa.pisa_sparse_attn_backward_ws(cfg, Qd, Kd, Vd, idx, dOd, *grads, ws)
    assert pisa.pisa_workspace_status(cfg, ws) == 0
    return Q, K, V, dO, idx.cpu().numpy(), [g.cpu().double().numpy() for g in grads]


def _worst_vs_oracle(w, Q, K, V, dO, idx, grads):
    G = w.Hq // w.Hkv
    worst = 0.0
    for b in range(w.B):
        for h in range(w.Hkv):
            hs = slice(h * G, (h + 1) * G)
            ref = oracle.attn_backward_rows(
                oracle.to_f64(Q[b, hs]), oracle.to_f64(K[b, h]), oracle.to_f64(V[b, h]), idx[b, h],
                oracle.to_f64(dO[b, hs]), C=w.C, causal=w.causal)
            for got, r in zip((grads[0][b, hs], grads[1][b, h], grads[2][b, h]), ref):
                assert np.isfinite(got).all()
                worst = max(worst, float(np.abs(got - r).max()) / max(1.0, float(np.abs(r).max())))
    return worst


@pytest.mark.parametrize("name", list(BM_CASES))
def test_block_major_backward_matches_oracle(name):
    w = BM_CASES[name]
    Q, K, V, dO, idx, grads = _bm_backward(w)
    worst = _worst_vs_oracle(w, Q, K, V, dO, idx, grads)
    print(f"block-major backward {name}: worst error {worst:.2e} of max |ref|")
    assert worst <= BM_TOL, worst


def test_block_major_backward_with_unlisted_forced_leaves():
    w = BM_CASES["mha_ragged"]
    Q, K, V, dO, idx, grads = _bm_backward(w, drop_first_leaf=True)
    lists_first = (idx == 0).any(axis=-1)
    assert 0 < lists_first.sum() < lists_first.size  # some rows no longer list leaf 0
    worst = _worst_vs_oracle(w, Q, K, V, dO, idx, grads)
    print(f"block-major backward, unlisted forced leaves: worst error {worst:.2e}")
    assert worst <= BM_TOL, worst


@pytest.mark.parametrize("name", ["mha_ragged", "gqa4", "noncausal_first_only"])
def test_block_major_backward_from_saved_forward_state(name):
    # pisa_forward_ws leaves the normaliser, the fp32 output and the grouping in
    # its workspace; the saved-state backward starts from them
    w = BM_CASES[name]
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    dO = torch.from_numpy(np.random.default_rng(w.seed + 7).standard_normal(Q.shape).astype(np.float32)).to(Q.dtype)
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    ws = pisa.alloc_backward_workspace(cfg, dev)
    ws.random_(0, 256)
    pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, ws)
    grads = [torch.full(x.shape, float("nan"), dtype=torch.float32, device=dev) for x in (Q, K, V)]
    pisa.pisa_sparse_attn_backward_saved_ws(cfg, Qd, Kd, Vd, idx, dOd, *grads, ws)
    assert pisa.pisa_workspace_status(cfg, ws) == 0
    worst = _worst_vs_oracle(w, Q, K, V, dO, idx.cpu().numpy(), [g.cpu().double().numpy() for g in grads])
    print(f"block-major backward from saved state {name}: worst error {worst:.2e}")
    assert worst <= BM_TOL, worst


def test_block_major_backward_full_size_sampled():
    # the bench's workload and launch configuration (MHA-8, N = 262144): dQ of
    # sampled rows and dK, dV of sampled leaves (early, middle, last) against
    # the oracle's per-entry backward, on two KV heads
    w = WORKLOADS["mha8_n256k"]
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    dO = torch.from_numpy(np.random.default_rng(w.seed + 7).standard_normal(Q.shape).astype(np.float32)).to(Q.dtype)
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    ws = pisa.alloc_backward_workspace(cfg, dev)
    pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, ws)
    grads = [torch.empty(x.shape, dtype=torch.float32, device=dev) for x in (Q, K, V)]
    pisa.pisa_sparse_attn_backward_ws(cfg, Qd, Kd, Vd, idx, dOd, *grads, ws)
    assert pisa.pisa_workspace_status(cfg, ws) == 0
    del Qd, Kd, Vd, dOd, ws
    idx_h = idx.cpu().numpy()
    M1 = (w.N + w.C - 1) // w.C
    rng = np.random.default_rng(5)
    # rows: the first leaf's edges (C - 1, C, 2C) beside random ones; leaves:
    # the first (forced for every position: its bucket spans thousands of
    # tiles and many CTAs), the second, both sides of a scan-block boundary of
    # the bucket counts (1024 buckets), the middle and the last
    rows = sorted(set(rng.choice(w.N, size=14, replace=False).tolist()) | {0, w.C - 1, w.C, 2 * w.C, w.N - 1})
    leaves = [0, 1, 37, 1023, 1024, M1 // 2, M1 - 1]
    worst = 0.0
    for h in (0, 5):
        rQ, rK, rV = oracle.attn_backward_sampled(
            oracle.to_f64(Q[0, h:h + 1]), oracle.to_f64(K[0, h]), oracle.to_f64(V[0, h]), idx_h[0, h],
            oracle.to_f64(dO[0, h:h + 1]), C=w.C, causal=w.causal, rows=rows, leaves=leaves)
        gQ = grads[0][0, h, rows].cpu().double().numpy()
        gK = torch.stack([grads[1][0, h, l * w.C:(l + 1) * w.C] for l in leaves]).cpu().double().numpy()
        gV = torch.stack([grads[2][0, h, l * w.C:(l + 1) * w.C] for l in leaves]).cpu().double().numpy()
        for got, ref in ((gQ, rQ[0]), (gK, rK), (gV, rV)):
            assert np.isfinite(got).all()
            worst = max(worst, float(np.abs(got - ref).max()) / max(1.0, float(np.abs(ref).max())))
    print(f"block-major backward, 256K MHA-8 sampled: worst error {worst:.2e} of max |ref|")
    assert worst <= BM_TOL, worst
