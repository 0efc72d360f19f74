"""pisa_select_noalloc: the selection for callers that cannot allocate device
memory (a host application that owns the GPU memory pool, serving loops that
forbid allocations after start-up, C callers without an allocator). It uses
the library's fixed scratch array instead of a caller workspace, so it must
give what pisa_select_ws gives -- and keep doing so on the next call, which
finds the previous call's leftovers in the shared array. Its error word is
read with pisa_select_noalloc_status.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _select_both(lib, w, N, seed, dev, variant):
    Q, K, _, _ = make_inputs(w, N=N, seed=seed)
    Qd, Kd = Q.to(dev), K.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, score_variant=variant)
    pyr, idx_ref, _ = pisa.alloc_outputs(cfg, dev, Qd.dtype)
    pisa.pisa_build_pyramid(cfg, Kd, pyr)
    work = pisa.alloc_workspace(cfg, dev)
    pisa.pisa_select_ws(cfg, Qd, Kd, pyr, idx_ref, work)
    idx = torch.full_like(idx_ref, -7)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = lib.pisa_select_noalloc(ctypes.byref(cfg), _p(Qd), _p(Kd), _p(pyr), _p(idx), stream)
    torch.cuda.synchronize()
    word = lib.pisa_select_noalloc_status(ctypes.byref(cfg), stream)
    return status, word, idx, idx_ref


# group sizes 1 and 2 take the four-lanes-per-row stage-1 walker, 4 the
# 32-slot one; the PISA-1 score adds its own region to the scratch layout
@pytest.mark.parametrize("Hq,Hkv,variant", [(2, 2, 0), (4, 2, 0), (8, 2, 0), (4, 2, 1)])
def test_select_noalloc_matches_select_ws_on_two_calls_in_a_row(Hq, Hkv, variant):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    lib = pisa.load()
    dev = torch.device("cuda", 0)
    w = Workload("noalloc", 300, B=1, Hq=Hq, Hkv=Hkv, N=4096, d=128, C=64, K=8)
    # two calls in a row through the C ABI: different data and a ragged length
    # for the second, so stale scratch from the first cannot stand in for it
    for N, seed in ((4096, 301), (3000, 302)):
        status, word, idx, idx_ref = _select_both(lib, w, N, seed, dev, variant)
        assert status == 0, pisa.pisa_status_string(status)
        assert word == 0, "the no-alloc selection reported a timeout or a failed self-check"
        assert int((idx == -7).sum()) == 0, "every index slot written"
        # same kernels and per-row arithmetic as the workspace path: identical
        assert torch.equal(idx, idx_ref)


def test_select_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    lib = pisa.load()
    dev = torch.device("cuda", 0)
    buf = torch.zeros(1024, dtype=torch.bfloat16, device=dev)
    big = pisa.make_cfg(B=1, Hq=8, Hkv=8, N=262144, d=128, C=64, K=16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = lib.pisa_select_noalloc(ctypes.byref(big), _p(buf), _p(buf), _p(buf), _p(buf), stream)
    assert status == -6 and "scratch" in pisa.pisa_status_string(status)
