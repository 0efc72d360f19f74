"""GPU parity of the decode path (incremental pyramid append + the fused
single-stage step) against the oracle: the oracle rebuilds each sequence's
pyramid for the grown prefix and selects/attends for the newest query."""
import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import (WORKLOADS, Workload, decode_cache, decode_rows,
                                                      decode_step_inputs)
from oracle import oracle
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    pisa.load()


def _cfg(w, B, cap, variant=0):
    return pisa.make_cfg(B=B, Hq=w.Hq, Hkv=w.Hkv, N=cap, d=w.d, C=w.C, K=w.K, causal=True,
                         forced_mask=w.forced_mask, dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                         score_variant=variant)


def _check_seq(w, cap, Khost, Vhost, pyr_gpu, n, q, idx_g, o_g, check_pyr=True, variant=0):
    """One sequence after its token at position n was appended."""
    G = w.Hq // w.Hkv
    worst, exempt = 0.0, 0
    for h in range(w.Hkv):
        Kh = oracle.to_f64(Khost[h, : n + 1])
        Vh = oracle.to_f64(Vhost[h, : n + 1])
        P = oracle.build_pyramid(Kh, w.C, N=n + 1, N_layout=cap)
        if check_pyr:
            L, M, off = oracle.geometry(cap, w.C)
            gp = oracle.to_f64(pyr_gpu[h])
            for lvl in range(1, L + 1):
                live = -(-(n + 1) // (w.C * 2 ** (lvl - 1)))
                np.testing.assert_allclose(gp[off[lvl]:off[lvl] + live], P[off[lvl]:off[lvl] + live],
                                           rtol=1e-5, atol=2e-6)
        qg = oracle.to_f64(q[h * G:(h + 1) * G])[None]
        want, gap = oracle.select_rows(qg, np.array([n]), Kh, P, C=w.C, K=w.K, N=n + 1, N_layout=cap,
                                       forced_mask=w.forced_mask, variant=variant)
        got = idx_g[h].cpu().numpy()
        parity.check_row_valid(got, n, n + 1, w.C, w.K, True, w.forced_mask)
        if gap[0] >= parity.TIE_BAND:
            np.testing.assert_array_equal(got, want[0])
        else:
            exempt += 1
        for j in range(G):
            O_o = oracle.attn_rows(qg[:, j], np.array([n]), Kh, Vh, got[None], C=w.C, causal=True)
            worst = max(worst, float(np.abs(O_o[0] - oracle.to_f64(o_g[h * G + j])).max()))
    assert worst <= parity.O_TOL[w.dtype], worst
    return exempt


# (G, d, C, K, dtype, cap, prefixes): the decode kernel streams leaf blocks in
# tiles of 16 KB of rows, so these cover a leaf in one tile, a leaf in two
# scoring tiles (fp32 at d = 128; C = 128), several leaves' worth of rows per
# tile (d = 64, small C), and group sizes up to 8.
DECODE_SHAPES = [
    (1, 128, 64, 8, "bf16", 4096, [1000, 2048, 3071]),
    (2, 128, 64, 8, "bf16", 4096, [1000, 2048, 3071]),
    (1, 64, 16, 4, "f32", 1024, [100, 512, 990]),
    (1, 128, 64, 8, "f32", 4096, [700, 2048, 4000]),
    (4, 64, 32, 8, "bf16", 2048, [333, 1024, 2000]),
    (8, 128, 128, 4, "bf16", 4096, [1500, 2600, 4050]),
]


@pytest.mark.parametrize("fused", [False, True], ids=["append+decode", "decode_step"])
@pytest.mark.parametrize("G,d,C,K,dtype,cap,prefix", DECODE_SHAPES)
def test_decode_steps_small(G, d, C, K, dtype, cap, prefix, fused):
    w = Workload("dec_small", 120, B=1, Hq=2 * G, Hkv=2, N=0, d=d, C=C, K=K, decode_batch=3, dtype=dtype)
    dev = torch.device("cuda", 0)
    Kc, Vc, Kp, Vp = decode_cache(w, cap, max(prefix) + 29, dev)
    Khost = [decode_rows(Kp, s, max(prefix) + 29) for s in range(3)]
    Vhost = [decode_rows(Vp, s, max(prefix) + 29) for s in range(3)]
    for s in range(3):  # zero the rows past each sequence's prefix
        Kc[s, :, prefix[s]:] = 0
        Vc[s, :, prefix[s]:] = 0
        Khost[s] = torch.cat([Khost[s][:, : prefix[s]], torch.zeros_like(Khost[s][:, :1]).expand(-1, cap - prefix[s], -1)], 1)
        Vhost[s] = torch.cat([Vhost[s][:, : prefix[s]], torch.zeros_like(Vhost[s][:, :1]).expand(-1, cap - prefix[s], -1)], 1)
    cfg = _cfg(w, 3, cap)
    R = pisa.pisa_pyramid_rows(cfg)
    pyr = torch.zeros((3, w.Hkv, R, w.d), dtype=torch.float32, device=dev)
    lens = torch.tensor(prefix, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg, Kc, lens, pyr)
    pos = lens.clone()
    exempt = 0
    for step in range(6):
        q, k, v = decode_step_inputs(w, step, B=3)
        idx = torch.full((3, w.Hkv, w.K), -7, dtype=torch.int32, device=dev)
        o = torch.empty((3, w.Hq, w.d), dtype=q.dtype, device=dev)
        if fused:  # one launch: append, then select and attend
            pisa.pisa_decode_step(cfg, q.to(dev), k.to(dev), v.to(dev), Kc, Vc, pyr, pos, idx, o)
        else:
            pisa.pisa_pyramid_append(cfg, Kc, Vc, pyr, k.to(dev), v.to(dev), pos)
            pisa.pisa_decode(cfg, q.to(dev), Kc, Vc, pyr, pos, idx, o)
        torch.cuda.synchronize()
        for s in range(3):
            n = int(pos[s])
            Khost[s][:, n] = k[s]
            Vhost[s][:, n] = v[s]
            exempt += _check_seq(w, cap, Khost[s], Vhost[s], pyr[s], n, q[s], idx[s], o[s])
        # the caches now hold the new rows verbatim
        for s in range(3):
            n = int(pos[s])
            assert torch.equal(Kc[s, :, n].cpu(), k[s]) and torch.equal(Vc[s, :, n].cpu(), v[s])
        pos += 1
    assert exempt <= 2


def test_decode_out_of_range_positions():
    w = Workload("dec_bad", 121, B=1, Hq=2, Hkv=2, N=0, d=64, C=16, K=4, decode_batch=2, dtype="f32")
    cap = 256
    dev = torch.device("cuda", 0)
    cfg = _cfg(w, 2, cap)
    Kc = torch.randn(2, 2, cap, 64, device=dev)
    Vc = torch.randn(2, 2, cap, 64, device=dev)
    K0, V0 = Kc.clone(), Vc.clone()
    pyr = torch.zeros(2, 2, pisa.pisa_pyramid_rows(cfg), 64, device=dev)
    pos = torch.tensor([-1, cap], dtype=torch.int32, device=dev)
    q, k, v = decode_step_inputs(w, 0, B=2)
    idx = torch.full((2, 2, 4), 5, dtype=torch.int32, device=dev)
    o = torch.ones(2, 2, 64, device=dev)
    pisa.pisa_pyramid_append(cfg, Kc, Vc, pyr, k.to(dev), v.to(dev), pos)
    pisa.pisa_decode(cfg, q.to(dev), Kc, Vc, pyr, pos, idx, o)
    torch.cuda.synchronize()
    assert torch.equal(Kc, K0) and torch.equal(Vc, V0)
    assert bool((idx == -1).all()) and bool((o == 0).all()) and bool((pyr == 0).all())


def test_decode_full_size_sampled():
    # 64 sequences x 8 heads against 262144-key caches (the bench's fused step)
    w = WORKLOADS["mha8_n256k"]
    prefix = w.N
    cap = prefix + 64
    dev = torch.device("cuda", 0)
    Kc, Vc, Kp, Vp = decode_cache(w, cap, prefix, dev)
    B = w.decode_batch
    cfg = _cfg(w, B, cap)
    pyr = torch.empty((B, w.Hkv, pisa.pisa_pyramid_rows(cfg), w.d), dtype=torch.float32, device=dev)
    lens = torch.full((B,), prefix, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg, Kc, lens, pyr)
    q, k, v = decode_step_inputs(w, 0)
    idx = torch.full((B, w.Hkv, w.K), -7, dtype=torch.int32, device=dev)
    o = torch.empty((B, w.Hq, w.d), dtype=q.dtype, device=dev)
    pos = lens.clone()
    pisa.pisa_decode_step(cfg, q.to(dev), k.to(dev), v.to(dev), Kc, Vc, pyr, pos, idx, o)  # bench launch
    torch.cuda.synchronize()
    assert int((idx == -7).sum()) == 0
    for s in (0, 17, 63):
        Kh = torch.cat([decode_rows(Kp, s, prefix), k[s][:, None]], 1)
        Vh = torch.cat([decode_rows(Vp, s, prefix), v[s][:, None]], 1)
        _check_seq(w, cap, Kh, Vh, pyr[s], prefix, q[s], idx[s], o[s], check_pyr=(s == 0))


def test_pyramid_grow_then_decode_past_the_old_capacity():
    # the decode cache outgrows its capacity: the pyramid is re-laid out for
    # twice the capacity (pisa_pyramid_grow), the caller copies its K/V rows,
    # and decoding continues past the old capacity
    w = Workload("dec_grow", 122, B=1, Hq=2, Hkv=2, N=0, d=128, C=64, K=8, decode_batch=2)
    cap_old, cap_new = 2048, 4096
    lens = [1500, 2045]
    dev = torch.device("cuda", 0)
    Kc, Vc, Kp, Vp = decode_cache(w, cap_old, 2047, dev)
    Khost = [decode_rows(Kp, s, 2047) for s in range(2)]
    Vhost = [decode_rows(Vp, s, 2047) for s in range(2)]
    for s in range(2):
        Kc[s, :, lens[s]:] = 0
        Vc[s, :, lens[s]:] = 0
    cfg_old, cfg_new = _cfg(w, 2, cap_old), _cfg(w, 2, cap_new)
    pyr_old = torch.zeros((2, w.Hkv, pisa.pisa_pyramid_rows(cfg_old), w.d), dtype=torch.float32, device=dev)
    pos = torch.tensor(lens, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg_old, Kc, pos, pyr_old)
    pyr = torch.full((2, w.Hkv, pisa.pisa_pyramid_rows(cfg_new), w.d), float("nan"), dtype=torch.float32, device=dev)
    pisa.pisa_pyramid_grow(cfg_old, pyr_old, cfg_new, pyr)
    torch.cuda.synchronize()
    L, _, off = oracle.geometry(cap_new, w.C)
    for s in range(2):  # the grown layout holds the same summaries as a rebuild for cap_new
        for h in range(w.Hkv):
            Kh = oracle.to_f64(Khost[s][h, : lens[s]])
            P = oracle.build_pyramid(Kh, w.C, N=lens[s], N_layout=cap_new)
            gp = oracle.to_f64(pyr[s, h])
            for lvl in range(1, L + 1):
                live = -(-lens[s] // (w.C * 2 ** (lvl - 1)))
                np.testing.assert_allclose(gp[off[lvl]:off[lvl] + live], P[off[lvl]:off[lvl] + live],
                                           rtol=1e-5, atol=2e-6)
    Kc2 = torch.zeros((2, w.Hkv, cap_new, w.d), dtype=Kc.dtype, device=dev)
    Vc2 = torch.zeros_like(Kc2)
    Kc2[:, :, :cap_old] = Kc
    Vc2[:, :, :cap_old] = Vc
    for step in range(6):  # sequence 1 crosses position 2048
        q, k, v = decode_step_inputs(w, step, B=2)
        idx = torch.full((2, w.Hkv, w.K), -7, dtype=torch.int32, device=dev)
        o = torch.empty((2, w.Hq, w.d), dtype=q.dtype, device=dev)
        pisa.pisa_decode_step(cfg_new, q.to(dev), k.to(dev), v.to(dev), Kc2, Vc2, pyr, pos, idx, o)
        torch.cuda.synchronize()
        for s in range(2):
            n = int(pos[s])
            Kh = torch.cat([Khost[s][:, :n], k[s][:, None]], 1)
            Vh = torch.cat([Vhost[s][:, :n], v[s][:, None]], 1)
            Khost[s], Vhost[s] = Kh, Vh
            _check_seq(w, cap_new, Kh, Vh, pyr[s], n, q[s], idx[s], o[s])
        pos += 1
    assert int(pos[1]) > cap_old


def test_decode_cache_grows_geometrically_inside_the_library():
    # DecodeCache grows by the library's policy (pisa_cache_capacity) before a
    # step would write past the capacity; pisa_cache_grow moves K, V and the
    # pyramid in the library's kernels, and decoding continues past the old capacity
    w = Workload("dec_grow2", 123, B=1, Hq=4, Hkv=2, N=0, d=128, C=64, K=8, decode_batch=2)
    cap_old = 2048
    lens = [1800, 2046]
    dev = torch.device("cuda", 0)
    Kc, Vc, Kp, Vp = decode_cache(w, cap_old, 2047, dev)
    Khost = [decode_rows(Kp, s, 2047) for s in range(2)]
    Vhost = [decode_rows(Vp, s, 2047) for s in range(2)]
    for s in range(2):
        Kc[s, :, lens[s]:] = 0
        Vc[s, :, lens[s]:] = 0
    cfg = _cfg(w, 2, cap_old)
    pyr = torch.zeros((2, w.Hkv, pisa.pisa_pyramid_rows(cfg), w.d), dtype=torch.float32, device=dev)
    pos = torch.tensor(lens, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg, Kc, pos, pyr)
    cache = pisa.DecodeCache(cfg, Kc, Vc, pyr)
    caps = []
    for step in range(5):  # sequence 1 writes positions 2046..2050: the cache grows before position 2048
        q, k, v = decode_step_inputs(w, step, B=2)
        idx = torch.full((2, w.Hkv, w.K), -7, dtype=torch.int32, device=dev)
        o = torch.empty((2, w.Hq, w.d), dtype=q.dtype, device=dev)
        cache.step(q.to(dev), k.to(dev), v.to(dev), pos, idx, o, max_pos=max(lens) + step)
        torch.cuda.synchronize()
        caps.append(cache.capacity)
        for s in range(2):
            n = int(pos[s])
            Kh = torch.cat([Khost[s][:, :n], k[s][:, None]], 1)
            Vh = torch.cat([Vhost[s][:, :n], v[s][:, None]], 1)
            Khost[s], Vhost[s] = Kh, Vh
            _check_seq(w, cache.capacity, Kh, Vh, cache.pyr[s], n, q[s], idx[s], o[s])
            # the grown caches hold every row written so far, zeros past it
            assert torch.equal(cache.Kc[s, :, :n + 1].cpu(), Kh)
            assert torch.equal(cache.Vc[s, :, :n + 1].cpu(), Vh)
            assert not cache.Kc[s, :, n + 1:].any()
        pos += 1
    assert caps == [2048, 2048, 4096, 4096, 4096]


def test_failed_cache_grow_writes_nothing():
    # a null or aliased pyramid is rejected before the K and V copies are launched
    import ctypes
    dev = torch.device("cuda", 0)
    old = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=1024, d=128, C=64, K=8)
    new = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=2048, d=128, C=64, K=8)
    Kc, Vc = (torch.randn(2, 2, 1024, 128, device=dev).to(torch.bfloat16) for _ in range(2))
    Kn, Vn = (torch.full((2, 2, 2048, 128), 3.0, dtype=torch.bfloat16, device=dev) for _ in range(2))
    po = torch.zeros((2, 2, pisa.pisa_pyramid_rows(old), 128), dtype=torch.float32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = pisa.load()
    for pyr_old, pyr_new in ((None, p(po)), (p(po), p(po))):
        st = lib.pisa_cache_grow(ctypes.byref(old), p(Kc), p(Vc), pyr_old, ctypes.byref(new), p(Kn), p(Vn),
                                 pyr_new, stream)
        torch.cuda.synchronize()
        assert st == -1
        assert bool((Kn == 3.0).all()) and bool((Vn == 3.0).all()), "a failed call wrote the new caches"
