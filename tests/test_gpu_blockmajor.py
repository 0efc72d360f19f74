"""GPU parity of the block-major tensor-core path (pisa_forward_ws,
pisa_select_ws, pisa_sparse_attn_ws) against the oracle, and its agreement
with the per-query path."""
import ctypes

import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import WORKLOADS, Workload, make_inputs
from tests import parity
from tests.test_gpu_parity import _report

pytestmark = pytest.mark.gpu

SMALL = {
    # ragged tail (3000 = 46*64 + 56), two sequences
    "bm_ragged": Workload("bm_ragged", 130, B=2, Hq=2, Hkv=2, N=3000, d=128, C=64, K=8),
    # GQA group of 4, K = 16: 32 candidates per level
    "bm_gqa4": Workload("bm_gqa4", 131, B=1, Hq=8, Hkv=2, N=5000, d=128, C=64, K=16),
    # non-causal, only the first leaf forced
    "bm_noncausal": Workload("bm_noncausal", 132, B=1, Hq=2, Hkv=2, N=2000, d=128, C=64, K=6, causal=False,
                             forced_mask=1),
    # GQA group of 16: 8 queries per tile
    "bm_gqa16": Workload("bm_gqa16", 133, B=1, Hq=32, Hkv=2, N=1500, d=128, C=64, K=8),
    # the smallest budget the forced leaves allow
    "bm_k3": Workload("bm_k3", 134, B=1, Hq=1, Hkv=1, N=4096, d=128, C=64, K=3),
    # a single leaf: the root is the leaf
    "bm_one_leaf": Workload("bm_one_leaf", 135, B=1, Hq=2, Hkv=1, N=50, d=128, C=64, K=4),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    pisa.load()


@pytest.mark.parametrize("name", list(SMALL))
def test_blockmajor_small_every_row(name):
    w = SMALL[name]
    Q, K, V, _ = make_inputs(w)
    res = parity.gpu_prefill(w, Q, K, V, ws=True)
    stats = [parity.check_head(w, Q, K, V, res, b, h, list(range(w.N)))
             for b in range(w.B) for h in range(w.Hkv)]
    _report("ws:" + name, stats)


# a group of 16 query heads per KV head (8 positions per tile) at a size where
# the tile walk hands its fine levels to the one-warp walk
LARGE = {"gqa32x2_n64k": Workload("gqa32x2_n64k", 136, B=1, Hq=32, Hkv=2, N=65536, d=128, C=64, K=16)}


@pytest.mark.parametrize("name", ["mha16_n16k", "needle_mha16_n64k", "gqa32x8_n128k", "mha8_n256k", "gqa32x2_n64k"])
def test_blockmajor_named_workload_full_size(name):
    w = WORKLOADS[name] if name in WORKLOADS else LARGE[name]
    Q, K, V, _ = make_inputs(w)
    res = parity.gpu_prefill(w, Q, K, V, ws=True)
    idx = res["idx"]
    assert int((idx == -7).sum()) == 0
    stats = [parity.check_head(w, Q, K, V, res, 0, h,
                               parity.sample_rows(w.N, w.C, 24, seed=100 + h)) for h in range(w.Hkv)]
    _report("ws:" + name, stats)
    t = torch.arange(w.N, device=idx.device)
    assert bool((idx.max(-1).values == t // w.C).all())
    # every row: the per-query path is an independent GPU implementation of
    # the same walk; each row where the two disagree goes to the oracle, and
    # the tensor-core row must equal the oracle's unless the oracle's margin
    # is inside the tie band (the per-query row is held to the same rule)
    ref = parity.gpu_prefill(w, Q, K, V, ws=False)
    differ = (ref["idx"] != idx).any(-1)  # [B, Hkv, N]
    n_diff = int(differ.sum())
    print(f"[blockmajor] {name}: rows differing from the per-query path: {n_diff} of {differ.numel()}")
    dstats = []
    for b in range(w.B):
        for h in range(w.Hkv):
            rows = torch.nonzero(differ[b, h]).flatten().cpu().tolist()
            if rows:
                dstats.append(parity.check_head(w, Q, K, V, res, b, h, rows))
                parity.check_head(w, Q, K, V, ref, b, h, rows)
    if dstats:
        ex = sum(s["exempt"] for s in dstats)
        print(f"[blockmajor] {name}: differing rows checked against the oracle: {n_diff}, "
              f"inside the tie band {ex}, tensor-core row equal to the oracle's there "
              f"{sum(s['exempt_equal'] for s in dstats)}, max|dO| {max(s['o_err'] for s in dstats):.3g}")
    agree = ~differ
    if bool(agree.any()):
        G = w.Hq // w.Hkv
        rows_ok = agree.repeat_interleave(G, dim=1)
        dO = (ref["O"].float() - res["O"].float()).abs().amax(-1)[rows_ok].max().item()
        assert dO <= 2 * parity.O_TOL["bf16"], dO


@pytest.mark.parametrize("name", ["bm_ragged", "bm_gqa4", "bm_noncausal"])
def test_select_ws_and_attn_ws_standalone(name):
    w = SMALL[name]
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Qd.dtype)
    work = pisa.alloc_workspace(cfg, dev)
    pisa.pisa_build_pyramid(cfg, Kd, pyr)
    pisa.pisa_select_ws(cfg, Qd, Kd, pyr, idx, work)
    # attention from indices alone (it derives its own normalisers)
    O2 = torch.empty_like(O)
    pisa.pisa_sparse_attn_ws(cfg, Qd, Kd, Vd, idx, O2, work)
    assert pisa.pisa_workspace_status(cfg, work) == 0
    res = {"cfg": cfg, "pyr": pyr, "idx": idx, "O": O2}
    stats = [parity.check_head(w, Q, K, V, res, b, h, list(range(0, w.N, 3)))
             for b in range(w.B) for h in range(w.Hkv)]
    _report("ws-standalone:" + name, stats)
    # the per-query attention on the same indices agrees
    pisa.pisa_sparse_attn(cfg, Qd, Kd, Vd, idx, O)
    torch.cuda.synchronize()
    assert (O.float() - O2.float()).abs().max().item() <= 2e-2


def test_workspace_errors():
    w = SMALL["bm_ragged"]
    cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8)
    need = pisa.pisa_workspace_bytes(cfg)
    dev = torch.device("cuda", 0)
    Q = torch.zeros(1, 2, 1000, 128, dtype=torch.bfloat16, device=dev)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev)
    small = torch.empty(need - 256, dtype=torch.uint8, device=dev)
    with pytest.raises(pisa.PisaError):
        pisa.pisa_select_ws(cfg, Q, Q, pyr, idx, small)
    bad = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=32, K=8)
    with pytest.raises(pisa.PisaError):
        pisa.pisa_workspace_bytes(bad)
    _ = w


def test_forward_host_equals_forward_ws():
    # pisa_forward_host: the same step from pinned host buffers, copies on the stream
    w = SMALL["bm_ragged"]
    Q, K, V, _ = make_inputs(w)
    res = parity.gpu_prefill(w, Q, K, V, ws=True)
    dev = torch.device("cuda", 0)
    cfg = res["cfg"]
    Qd, Kd, Vd = torch.empty_like(Q, device=dev), torch.empty_like(K, device=dev), torch.empty_like(V, device=dev)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    work = pisa.alloc_workspace(cfg, dev)
    Ih = torch.full(idx.shape, -7, dtype=idx.dtype).pin_memory()
    Oh = torch.zeros(O.shape, dtype=O.dtype).pin_memory()
    pisa.pisa_forward_host(cfg, Q.pin_memory(), K.pin_memory(), V.pin_memory(), Ih, Oh, Qd, Kd, Vd, pyr, idx, O,
                           work)
    torch.cuda.synchronize()
    assert torch.equal(Ih, res["idx"].cpu())
    # the attention tiles add fp32 partial outputs in an order that varies from
    # run to run, so O agrees to rounding, not bit for bit
    assert float((Oh.float() - res["O"].float().cpu()).abs().max()) <= parity.O_TOL[w.dtype]


def test_failed_forward_host_writes_nothing():
    # a call that fails validation enqueues no copy: the device buffers keep a sentinel
    w = SMALL["bm_ragged"]
    Q, K, V, _ = make_inputs(w)
    dev = torch.device("cuda", 0)
    cfg = pisa.make_cfg(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, C=w.C, K=w.K)
    Qd, Kd, Vd = (torch.full(x.shape, 3.0, dtype=x.dtype, device=dev) for x in (Q, K, V))
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Q.dtype)
    work = pisa.alloc_workspace(cfg, dev)
    Ih = torch.zeros(idx.shape, dtype=idx.dtype).pin_memory()
    Oh = torch.zeros(O.shape, dtype=O.dtype).pin_memory()
    lib = pisa.load()
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for bad_pyr, bad_bytes in ((None, work.numel()), (p(pyr), work.numel() - 256)):
        st = lib.pisa_forward_host(ctypes.byref(cfg), p(Q.pin_memory()), p(K.pin_memory()), p(V.pin_memory()),
                                   p(Ih), p(Oh), p(Qd), p(Kd), p(Vd), bad_pyr, p(idx), p(O), p(work), bad_bytes,
                                   stream)
        torch.cuda.synchronize()
        assert st == -1
        for x in (Qd, Kd, Vd):
            assert bool((x == 3.0).all()), "a failed call copied into the device buffers"
