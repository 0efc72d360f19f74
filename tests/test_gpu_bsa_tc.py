"""GPU parity of the tensor-core flat BSA selection (pisa_bsa_select_ws,
close reading §02 Eq.(1)) against the oracle's flat Eq.(1) selection: every
row of small shapes (ragged tails, GQA groups of 4 and 16, non-causal, the
smallest budget), exact ties, and the named workloads at full size on sampled
rows plus every row where it and the CUDA-core call (pisa_bsa_select)
disagree."""
import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import oracle
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = {
    "ragged": Workload("bsatc_ragged", 170, B=2, Hq=2, Hkv=2, N=3000, d=128, C=64, K=8),
    "gqa4_k16": Workload("bsatc_gqa4", 171, B=1, Hq=8, Hkv=2, N=9000, d=128, C=64, K=16),
    "noncausal": Workload("bsatc_nc", 172, B=1, Hq=2, Hkv=2, N=2000, d=128, C=64, K=6, causal=False, forced_mask=1),
    "gqa16": Workload("bsatc_g16", 173, B=1, Hq=32, Hkv=2, N=1500, d=128, C=64, K=8),
    "k3": Workload("bsatc_k3", 174, B=1, Hq=1, Hkv=1, N=4096, d=128, C=64, K=3),
    "one_leaf": Workload("bsatc_one", 175, B=1, Hq=2, Hkv=1, N=50, d=128, C=64, K=4),
    "mask0": Workload("bsatc_m0", 176, B=1, Hq=2, Hkv=2, N=2500, d=128, C=64, K=5, forced_mask=0),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    pisa.load()


def _bsa_both(w, Q, K):
    dev = torch.device("cuda", 0)
    Qd, Kd = Q.to(dev), K.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, _ = pisa.alloc_outputs(cfg, dev, Qd.dtype)
    pisa.pisa_build_pyramid(cfg, Kd, pyr)
    work = pisa.alloc_workspace(cfg, dev)
    work.fill_(0xCD)  # scratch must not need zeroing by the caller
    tc = torch.full_like(idx, -7)
    pisa.pisa_bsa_select_ws(cfg, Qd, pyr, tc, work)
    assert pisa.pisa_workspace_status(cfg, work) == 0, "a tensor-core tile timed out"
    cc = torch.full_like(idx, -7)
    pisa.pisa_bsa_select(cfg, Qd, pyr, cc)
    torch.cuda.synchronize()
    return pyr, tc, cc


def _check(w, Q, K, pyr, got, b, h, rows):
    G = w.Hq // w.Hkv
    N = Q.shape[2]
    Kh = oracle.to_f64(K[b, h])
    P = oracle.to_f64(pyr[b, h])  # the GPU pyramid is checked against the oracle's elsewhere
    P_o = oracle.build_pyramid(Kh, w.C, w.g)
    np.testing.assert_allclose(P, P_o, rtol=1e-5, atol=2e-6)
    t = np.asarray(rows, np.int64)
    tt = torch.as_tensor(t)
    Qg = oracle.to_f64(Q[b, h * G:(h + 1) * G][:, tt]).transpose(1, 0, 2).copy()
    want, gap = oracle.flat_rows("bsa", Qg, t, Kh, P_o, C=w.C, K=w.K, g=w.g, causal=w.causal,
                                 forced_mask=w.forced_mask)
    g = got[b, h][tt.to(got.device)].cpu().numpy()
    return parity.compare_indices(g, want, gap, t, w, N, "bsa_ws")


@pytest.mark.parametrize("name", list(SMALL))
def test_bsa_ws_small_every_row(name):
    w = SMALL[name]
    Q, K, _, _ = make_inputs(w)
    pyr, tc, _ = _bsa_both(w, Q, K)
    assert int((tc == -7).sum()) == 0
    n = ex = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            r = _check(w, Q, K, pyr, tc, b, h, list(range(w.N)))
            n += r[0]
            ex += r[1]
    print(f"[bsa_ws] {name}: rows {n}, inside the tie band {ex}")


def test_bsa_ws_exact_ties_go_to_lower_index():
    w = Workload("bsatc_ties", 177, B=1, Hq=2, Hkv=2, N=2048, d=128, C=64, K=6)
    Q, K, _, _ = make_inputs(w)
    K[:] = K[:, :, :1, :]
    pyr, tc, _ = _bsa_both(w, Q, K)
    for h in range(2):
        Kh = oracle.to_f64(K[0, h])
        P = oracle.build_pyramid(Kh, w.C)
        t = np.arange(w.N, dtype=np.int64)
        Qg = oracle.to_f64(Q[0, h])[:, None, :]
        want, _ = oracle.flat_rows("bsa", Qg, t, Kh, P, C=w.C, K=w.K)
        np.testing.assert_array_equal(tc[0, h].cpu().numpy(), want)


@pytest.mark.parametrize("name", ["mha16_n16k", "needle_mha16_n64k", "gqa32x8_n128k", "mha8_n256k"])
def test_bsa_ws_named_workload_full_size(name):
    w = WORKLOADS[name]
    Q, K, _, _ = make_inputs(w)
    pyr, tc, cc = _bsa_both(w, Q, K)
    assert int((tc == -7).sum()) == 0
    for h in range(w.Hkv):
        _check(w, Q, K, pyr, tc, 0, h, parity.sample_rows(w.N, w.C, 16, seed=300 + h))
    differ = (tc != cc).any(-1)
    nd = int(differ.sum())
    ex = 0
    for h in range(w.Hkv):
        rows = torch.nonzero(differ[0, h]).flatten().cpu().tolist()
        if rows:
            ex += _check(w, Q, K, pyr, tc, 0, h, rows)[1]
            _check(w, Q, K, pyr, cc, 0, h, rows)
    print(f"[bsa_ws] {name}: rows differing from the CUDA-core call {nd} of {differ.numel()}, "
          f"inside the tie band {ex}")
