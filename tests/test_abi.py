"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function include/pisa.h declares, computes the pyramid geometry the oracle
computes, and rejects bad arguments before anything reaches a device."""
import ctypes

import pytest
import torch

from hierarchical_block_sparse_b200 import build as pisa_build
from hierarchical_block_sparse_b200 import pisa
from oracle import oracle


@pytest.fixture(scope="module")
def lib():
    pisa_build.build()
    return pisa.load()


def test_every_declared_symbol_is_exported(lib):
    names = pisa.exported_names()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    for required in ("pisa_build_pyramid", "pisa_select", "pisa_sparse_attn", "pisa_forward"):
        assert required in names


def test_version_and_status_strings(lib):
    assert "sm_100a" in pisa.pisa_version()
    for s in (0, -1, -2, -3, -4):
        assert pisa.pisa_status_string(s)
    assert pisa.pisa_status_string(-99) == "unknown status"


@pytest.mark.parametrize("N,C", [(1024, 16), (1000, 16), (16384, 64), (262144, 64), (262145, 64), (1, 64), (64, 64)])
def test_geometry_matches_oracle(lib, N, C):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=N, d=128, C=C, K=16)
    L, M, off = oracle.geometry(N, C, 2)
    assert pisa.pisa_num_levels(cfg) == L
    for lvl in range(1, L + 1):
        assert pisa.pisa_level_nodes(cfg, lvl) == M[lvl]
        assert pisa.pisa_level_offset(cfg, lvl) == off[lvl]
    assert pisa.pisa_pyramid_rows(cfg) == oracle.total_nodes(N, C, 2)


def test_geometry_general_branching(lib):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=5000, d=64, C=10, K=4, g=3)
    L, M, off = oracle.geometry(5000, 10, 3)
    assert pisa.pisa_num_levels(cfg) == L
    assert pisa.pisa_pyramid_rows(cfg) == oracle.total_nodes(5000, 10, 3)


def _call_select(lib, cfg, ptrs=(16, 16, 16, 16)):
    P = [ctypes.c_void_p(p) if p else None for p in ptrs]
    return lib.pisa_select(ctypes.byref(cfg), *P, None)


@pytest.mark.parametrize("field,value,status", [
    ("B", 0, -1), ("Hq", 3, -1), ("N", -5, -1), ("C", 0, -1), ("K", 0, -1),
    ("causal", 2, -1), ("forced_mask", 9, -1), ("dtype", 7, -1),
    ("K", 2, -1),            # three forced leaves need K >= 3
    ("g", 3, -2), ("d", 96, -2), ("K", 17, -2), ("C", 2048, -2),
])
def test_invalid_configs_are_rejected_before_launch(lib, field, value, status):
    cfg = pisa.make_cfg(B=1, Hq=4, Hkv=2, N=256, d=128, C=16, K=4)
    setattr(cfg, field, value)
    assert _call_select(lib, cfg) == status


def test_pyramid_grow_validates_before_launch(lib):
    old = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=2048, d=128, C=64, K=8)
    P = ctypes.c_void_p(4096)
    for field, value in (("N", 1024), ("C", 32), ("Hkv", 1), ("d", 64)):
        new = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=4096, d=128, C=64, K=8)
        setattr(new, field, value)
        assert lib.pisa_pyramid_grow(ctypes.byref(old), P, ctypes.byref(new), ctypes.c_void_p(8192), None) == -1
    new = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=4096, d=128, C=64, K=8)
    assert lib.pisa_pyramid_grow(ctypes.byref(old), P, ctypes.byref(new), P, None) == -1          # in place
    assert lib.pisa_pyramid_grow(ctypes.byref(old), None, ctypes.byref(new), P, None) == -1       # null
    assert lib.pisa_pyramid_grow(ctypes.byref(old), ctypes.c_void_p(4104), ctypes.byref(new), P, None) == -4


def test_score_variant_is_validated(lib):
    for v in (0, 1, 2):
        cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8, score_variant=v)
        assert lib.pisa_num_levels(ctypes.byref(cfg)) > 0
    for v in (-1, 3):
        cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8, score_variant=v)
        assert lib.pisa_num_levels(ctypes.byref(cfg)) == -1


def test_group_size_limits(lib):
    cfg = pisa.make_cfg(B=1, Hq=6, Hkv=2, N=256, d=128, C=16, K=4)   # G = 3
    assert _call_select(lib, cfg) == -2
    cfg = pisa.make_cfg(B=1, Hq=64, Hkv=2, N=256, d=128, C=16, K=4)  # G = 32
    assert _call_select(lib, cfg) == -2


def test_null_and_misaligned_pointers(lib):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=256, d=128, C=16, K=4)
    assert _call_select(lib, cfg, (16, 0, 16, 16)) == -1
    assert _call_select(lib, cfg, (16, 18, 16, 16)) == -4
    assert lib.pisa_build_pyramid(ctypes.byref(cfg), None, None, None) == -1
    assert lib.pisa_forward(None, None, None, None, None, None, None, None) == -1


def test_empty_sequence_is_a_noop(lib):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=0, d=128, C=16, K=4)
    assert pisa.pisa_num_levels(cfg) == 0
    assert pisa.pisa_pyramid_rows(cfg) == 0
    assert lib.pisa_forward(ctypes.byref(cfg), None, None, None, None, None, None, None) == 0


def test_decode_requires_causal(lib):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=256, d=128, C=16, K=4, causal=False, forced_mask=4)
    P = [ctypes.c_void_p(16)] * 7
    assert lib.pisa_decode(ctypes.byref(cfg), *P, None) == -1


def test_binding_refuses_cpu_tensors(lib):
    cfg = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=64, d=64, C=16, K=4, dtype=torch.float32)
    K = torch.zeros(1, 1, 64, 64)
    pyr = torch.zeros(1, 1, pisa.pisa_pyramid_rows(cfg), 64)
    with pytest.raises(ValueError):
        pisa.pisa_build_pyramid(cfg, K, pyr)


def test_workspace_bytes_and_limits(lib):
    cfg = pisa.make_cfg(B=1, Hq=8, Hkv=8, N=262144, d=128, C=64, K=16)
    n = pisa.pisa_workspace_bytes(cfg)
    # candidates + LSEs + grouping lists + the fp32 output accumulator dominate
    assert 1.0e9 < n < 3.0e9
    for field, value in (("C", 32), ("d", 64), ("dtype", 0)):
        bad = pisa.make_cfg(B=1, Hq=8, Hkv=8, N=262144, d=128, C=64, K=16)
        setattr(bad, field, value)
        assert lib.pisa_workspace_bytes(ctypes.byref(bad)) == -2
    zero = pisa.make_cfg(B=1, Hq=1, Hkv=1, N=0, d=128, C=64, K=4)
    assert pisa.pisa_workspace_bytes(zero) == 0


def test_workspace_calls_validate_before_launch(lib):
    cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8)
    need = pisa.pisa_workspace_bytes(cfg)
    P = [ctypes.c_void_p(4096)] * 4
    assert lib.pisa_select_ws(ctypes.byref(cfg), *P, None, need, None) == -1           # no workspace
    assert lib.pisa_select_ws(ctypes.byref(cfg), *P, ctypes.c_void_p(4096 + 16), need, None) == -4  # misaligned
    assert lib.pisa_select_ws(ctypes.byref(cfg), *P, ctypes.c_void_p(8192), need - 1, None) == -1   # too small
    # the block-major stage 1 reads pyramid rows with 256-bit loads: pyr needs 32 bytes
    P16 = [ctypes.c_void_p(4096), ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 16), ctypes.c_void_p(4096)]
    assert lib.pisa_select_ws(ctypes.byref(cfg), *P16, ctypes.c_void_p(8192), need, None) == -4
    assert lib.pisa_select_noalloc(ctypes.byref(cfg), *P16, None) == -4


def test_backward_workspace_validates_before_launch(lib):
    cfg = pisa.make_cfg(B=1, Hq=4, Hkv=2, N=1000, d=128, C=64, K=8)
    need = pisa.pisa_backward_workspace_bytes(cfg)
    # the forward's workspace plus D per (query, head), 256-byte rounded
    assert need == pisa.pisa_workspace_bytes(cfg) + ((2 * 1000 * 2 * 4 + 255) // 256) * 256
    P = [ctypes.c_void_p(4096)] * 8   # Q, K, V, idx, dO, dQ, dK, dV
    call = lib.pisa_sparse_attn_backward_ws
    assert call(ctypes.byref(cfg), *P, None, need, None) == -1                      # no workspace
    assert call(ctypes.byref(cfg), *P, ctypes.c_void_p(8192 + 16), need, None) == -4  # misaligned workspace
    assert call(ctypes.byref(cfg), *P, ctypes.c_void_p(8192), need - 1, None) == -1   # too small
    bad = list(P)
    bad[5] = ctypes.c_void_p(4096 + 4)                                              # misaligned dQ
    assert call(ctypes.byref(cfg), *bad, ctypes.c_void_p(8192), need, None) == -4
    bad[5] = None
    assert call(ctypes.byref(cfg), *bad, ctypes.c_void_p(8192), need, None) == -1
    saved = lib.pisa_sparse_attn_backward_saved_ws
    assert saved(ctypes.byref(cfg), *P, ctypes.c_void_p(8192), need - 1, None) == -1  # same checks
    assert saved(ctypes.byref(cfg), *bad, ctypes.c_void_p(8192), need, None) == -1
    for field, value in (("C", 32), ("d", 64), ("dtype", 0)):
        c2 = pisa.make_cfg(B=1, Hq=4, Hkv=2, N=1000, d=128, C=64, K=8)
        setattr(c2, field, value)
        assert lib.pisa_backward_workspace_bytes(ctypes.byref(c2)) == -2
        assert call(ctypes.byref(c2), *P, ctypes.c_void_p(8192), need, None) == -2


def test_cache_capacity_policy(lib):
    # the smallest C * 2^k holding n keys (geometric growth)
    assert [pisa.pisa_cache_capacity(n, 64) for n in (0, 1, 64, 65, 128, 129, 262144, 262145)] == \
        [64, 64, 64, 128, 128, 256, 262144, 524288]
    assert pisa.pisa_cache_capacity(1000, 48) == 48 * 32
    assert lib.pisa_cache_capacity(-1, 64) == -1
    assert lib.pisa_cache_capacity(10, 0) == -1


def test_cache_grow_validates_before_launch(lib):
    old = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=2048, d=128, C=64, K=8)
    new = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=4096, d=128, C=64, K=8)
    P = [ctypes.c_void_p(4096 * (i + 1)) for i in range(6)]  # Kc_old, Vc_old, pyr_old, Kc_new, Vc_new, pyr_new
    grow = lib.pisa_cache_grow

    def call(o, n, p):
        return grow(ctypes.byref(o), p[0], p[1], p[2], ctypes.byref(n), p[3], p[4], p[5], None)

    assert call(new, old, P) == -1                                  # smaller new capacity
    bad = pisa.make_cfg(B=2, Hq=2, Hkv=1, N=4096, d=128, C=64, K=8)
    assert call(old, bad, P) == -1                                  # other fields differ
    assert call(old, new, [P[0], P[1], P[2], P[0], P[4], P[5]]) == -1  # K in place
    assert call(old, new, [P[0], P[1], P[2], P[3], P[3], P[5]]) == -1  # K and V share a buffer
    assert call(old, new, [P[0], None, P[2], P[3], P[4], P[5]]) == -1
    assert call(old, new, [P[0], P[1], P[2], ctypes.c_void_p(8 + 4096 * 9), P[4], P[5]]) == -4
    empty = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=0, d=128, C=64, K=8)
    assert call(empty, new, P) == 0


def test_forward_host_validates_before_any_copy(lib):
    # every check of the device step runs before the first host-to-device copy:
    # a bad argument comes back as its own status (not as a failed copy)
    cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8)
    need = pisa.pisa_workspace_bytes(cfg)
    H = [ctypes.c_void_p(1 << 20)] * 5                       # Q, K, V, idx, O on the host
    D = [ctypes.c_void_p(4096 * (i + 1)) for i in range(6)]  # Q, K, V, pyr, idx, O on the device
    ws = ctypes.c_void_p(1 << 24)

    def call(dev, w=ws, n=need, host=H):
        return lib.pisa_forward_host(ctypes.byref(cfg), *host, *dev, w, n, None)

    assert call([D[0], D[1], D[2], None, D[4], D[5]]) == -1                     # no pyramid
    assert call([D[0], D[1], D[2], ctypes.c_void_p(4096 * 4 + 16), D[4], D[5]]) == -4  # pyramid 16- not 32-aligned
    assert call([D[0], D[1], D[2], D[3], None, D[5]]) == -1                     # no idx
    assert call(D, w=None) == -1                                                 # no workspace
    assert call(D, n=need - 1) == -1                                             # workspace too small
    assert call(D, w=ctypes.c_void_p((1 << 24) + 128)) == -4                     # workspace misaligned
    assert call(D, host=[H[0], None, H[2], H[3], H[4]]) == -1                   # no host K


def test_cache_grow_checks_the_pyramids_before_the_cache_copies(lib):
    old = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=2048, d=128, C=64, K=8)
    new = pisa.make_cfg(B=2, Hq=2, Hkv=2, N=4096, d=128, C=64, K=8)
    P = [ctypes.c_void_p(4096 * (i + 1)) for i in range(6)]  # Kc_old, Vc_old, pyr_old, Kc_new, Vc_new, pyr_new

    def call(p):
        return lib.pisa_cache_grow(ctypes.byref(old), p[0], p[1], p[2], ctypes.byref(new), p[3], p[4], p[5], None)

    assert call([P[0], P[1], None, P[3], P[4], P[5]]) == -1                     # no old pyramid
    assert call([P[0], P[1], P[2], P[3], P[4], P[2]]) == -1                     # pyramid grown in place
    assert call([P[0], P[1], P[2], P[3], P[4], ctypes.c_void_p(8 + 4096 * 6)]) == -4


def test_select_noalloc_status_validates(lib):
    big = pisa.make_cfg(B=1, Hq=8, Hkv=8, N=262144, d=128, C=64, K=16)
    assert lib.pisa_select_noalloc_status(ctypes.byref(big), None) == -6
    bad = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=32, K=8)
    assert lib.pisa_select_noalloc_status(ctypes.byref(bad), None) == -2
    empty = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=0, d=128, C=64, K=8)
    assert lib.pisa_select_noalloc_status(ctypes.byref(empty), None) == 0


def test_bsa_select_ws_and_fma_probe_validate_before_launch(lib):
    cfg = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=64, K=8)
    need = pisa.pisa_workspace_bytes(cfg)
    Q, pyr, idx = ctypes.c_void_p(4096), ctypes.c_void_p(8192), ctypes.c_void_p(12288)
    ws = ctypes.c_void_p(1 << 20)
    f = lib.pisa_bsa_select_ws
    assert f(ctypes.byref(cfg), Q, pyr, idx, None, need, None) == -1                     # no workspace
    assert f(ctypes.byref(cfg), Q, pyr, idx, ctypes.c_void_p((1 << 20) + 16), need, None) == -4  # misaligned
    assert f(ctypes.byref(cfg), Q, pyr, idx, ws, need - 1, None) == -1                    # too small
    assert f(ctypes.byref(cfg), None, pyr, idx, ws, need, None) == -1                     # no Q
    assert f(ctypes.byref(cfg), ctypes.c_void_p(4096 + 8), pyr, idx, ws, need, None) == -4  # Q misaligned
    bad = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=1000, d=128, C=32, K=8)
    assert f(ctypes.byref(bad), Q, pyr, idx, ws, need, None) == -2                        # C != 64
    empty = pisa.make_cfg(B=1, Hq=2, Hkv=2, N=0, d=128, C=64, K=8)
    assert f(ctypes.byref(empty), None, None, None, None, 0, None) == 0                   # nothing to do
    p = lib.pisa_fma_probe
    assert p(None, 148, 10, 0, None) == -1
    assert p(ctypes.c_void_p(4096), 0, 10, 0, None) == -1
    assert p(ctypes.c_void_p(4096), 148, 0, 1, None) == -1
