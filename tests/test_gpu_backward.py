"""GPU parity of pisa_sparse_attn_backward (fixed selection) against the
oracle's fp64 backward, on the selection the GPU itself made."""
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
