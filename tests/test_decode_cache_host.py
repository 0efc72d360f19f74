"""Host logic of pisa.DecodeCache (no GPU): when it grows, to what capacity
(the library's pisa_cache_capacity policy), and what it hands to
pisa_cache_grow. The grow call itself is replaced by a recorder here; on the
GPU it is covered by test_gpu_decode.py."""
import torch

from hierarchical_block_sparse_b200 import pisa


def _cache(N, monkeypatch, calls):
    cfg = pisa.make_cfg(B=2, Hq=4, Hkv=2, N=N, d=128, C=64, K=8)
    Kc = torch.zeros((2, 2, N, 128), dtype=torch.bfloat16)
    pyr = torch.zeros((2, 2, pisa.pisa_pyramid_rows(cfg) if N else 0, 128))
    monkeypatch.setattr(pisa, "pisa_cache_grow",
                        lambda co, k, v, p, cn, k2, v2, p2: calls.append((co.N, cn.N, k2.shape, p2.shape, k2.sum())))
    return pisa.DecodeCache(cfg, Kc, Kc.clone(), pyr)


def test_grows_only_past_the_capacity_and_by_doubling(monkeypatch):
    calls = []
    c = _cache(2048, monkeypatch, calls)
    c.reserve(100)
    c.reserve(2048)
    assert calls == [] and c.capacity == 2048
    c.reserve(2049)
    assert c.capacity == 4096 and len(calls) == 1
    old_n, new_n, kshape, pshape, _ = calls[0]
    assert (old_n, new_n) == (2048, 4096)
    assert tuple(kshape) == (2, 2, 4096, 128)
    assert tuple(pshape) == (2, 2, pisa.pisa_pyramid_rows(c.cfg), 128)
    assert c.Kc.shape[2] == 4096 and c.Vc.shape[2] == 4096
    c.reserve(9000)  # several doublings at once: the smallest C * 2^k that holds 9000
    assert c.capacity == 16384 and calls[-1][:2] == (4096, 16384)


def test_growing_an_empty_cache_starts_from_zeros(monkeypatch):
    calls = []
    c = _cache(0, monkeypatch, calls)
    c.reserve(1)
    assert c.capacity == 64
    assert calls[0][4] == 0  # the new buffers are zero-initialised
    assert not c.Kc.any() and not c.pyr.any()
