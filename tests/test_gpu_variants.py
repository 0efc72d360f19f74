"""GPU parity of the PISA-1 / PISA-2 node scores (close reading §04 4.3,
Eq.(8)-(9); pisa_cfg.score_variant) against the oracle's walk with the same
score: the per-query path, the block-major tensor-core path and the decode
step (as two calls and fused). Attention stays the exact softmax over the
selected leaves, checked by the oracle on the GPU's own indices."""
import numpy as np
import pytest
import torch

from hierarchical_block_sparse_b200 import pisa
from hierarchical_block_sparse_b200.workloads import WORKLOADS, Workload, decode_cache, decode_rows, \
    decode_step_inputs
from hierarchical_block_sparse_b200.workloads import make_inputs
from tests import parity
from tests.test_gpu_decode import _cfg, _check_seq
from tests.test_gpu_parity import _report

pytestmark = pytest.mark.gpu

VARIANTS = [pisa.PISA_SCORE_MEAN, pisa.PISA_SCORE_MEAN_VAR]
PER_QUERY = {
    "tiny_f32": WORKLOADS["tiny_f32_n1k"],
    "mha_bf16": Workload("v_mha", 140, B=1, Hq=2, Hkv=2, N=3000, d=128, C=64, K=8),
    "gqa4_d64": Workload("v_gqa4", 141, B=1, Hq=8, Hkv=2, N=2500, d=64, C=32, K=8),
}
BLOCK_MAJOR = {
    "mha_ragged": Workload("v_bm_mha", 142, B=2, Hq=2, Hkv=2, N=3000, d=128, C=64, K=8),
    "gqa2": Workload("v_bm_gqa2", 143, B=1, Hq=4, Hkv=2, N=4096, d=128, C=64, K=16),
    "gqa4": Workload("v_bm_gqa4", 144, B=1, Hq=8, Hkv=2, N=5000, d=128, C=64, K=16),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    pisa.load()


@pytest.mark.parametrize("variant", VARIANTS, ids=["pisa1", "pisa2"])
@pytest.mark.parametrize("name", list(PER_QUERY))
def test_per_query_path(name, variant):
    w = PER_QUERY[name]
    Q, K, V, _ = make_inputs(w)
    res = parity.gpu_prefill(w, Q, K, V, variant=variant)
    stats = [parity.check_head(w, Q, K, V, res, b, h, list(range(w.N)), variant=variant)
             for b in range(w.B) for h in range(w.Hkv)]
    _report(f"variant{variant}:" + name, stats)


@pytest.mark.parametrize("variant", VARIANTS, ids=["pisa1", "pisa2"])
@pytest.mark.parametrize("name", list(BLOCK_MAJOR))
def test_block_major_path(name, variant):
    w = BLOCK_MAJOR[name]
    Q, K, V, _ = make_inputs(w)
    res = parity.gpu_prefill(w, Q, K, V, ws=True, variant=variant)
    stats = [parity.check_head(w, Q, K, V, res, b, h, list(range(w.N)), variant=variant)
             for b in range(w.B) for h in range(w.Hkv)]
    _report(f"ws variant{variant}:" + name, stats)


@pytest.mark.parametrize("variant", VARIANTS, ids=["pisa1", "pisa2"])
@pytest.mark.parametrize("fused", [False, True], ids=["append+decode", "decode_step"])
def test_decode(variant, fused):
    w = Workload("v_dec", 145, B=1, Hq=4, Hkv=2, N=0, d=128, C=64, K=8, decode_batch=3)
    cap, prefix = 4096, [1000, 2048, 3071]
    dev = torch.device("cuda", 0)
    Kc, Vc, Kp, Vp = decode_cache(w, cap, 3100, dev)
    Khost = [decode_rows(Kp, s, 3100) for s in range(3)]
    Vhost = [decode_rows(Vp, s, 3100) for s in range(3)]
    for s in range(3):
        Kc[s, :, prefix[s]:] = 0
        Vc[s, :, prefix[s]:] = 0
    cfg = _cfg(w, 3, cap, variant)
    pyr = torch.zeros((3, w.Hkv, pisa.pisa_pyramid_rows(cfg), w.d), dtype=torch.float32, device=dev)
    pos = torch.tensor(prefix, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg, Kc, pos, pyr)
    exempt = 0
    for step in range(3):
        q, k, v = decode_step_inputs(w, step, B=3)
        idx = torch.full((3, w.Hkv, w.K), -7, dtype=torch.int32, device=dev)
        o = torch.empty((3, w.Hq, w.d), dtype=q.dtype, device=dev)
        if fused:
            pisa.pisa_decode_step(cfg, q.to(dev), k.to(dev), v.to(dev), Kc, Vc, pyr, pos, idx, o)
        else:
            pisa.pisa_pyramid_append(cfg, Kc, Vc, pyr, k.to(dev), v.to(dev), pos)
            pisa.pisa_decode(cfg, q.to(dev), Kc, Vc, pyr, pos, idx, o)
        torch.cuda.synchronize()
        for s in range(3):
            n = int(pos[s])
            Kh = torch.cat([Khost[s][:, :n], k[s][:, None]], 1)
            Vh = torch.cat([Vhost[s][:, :n], v[s][:, None]], 1)
            Khost[s] = torch.cat([Kh, Khost[s][:, n + 1:]], 1)
            Vhost[s] = torch.cat([Vh, Vhost[s][:, n + 1:]], 1)
            exempt += _check_seq(w, cap, Khost[s], Vhost[s], pyr[s], n, q[s], idx[s], o[s], check_pyr=False,
                                 variant=variant)
        pos += 1
    assert exempt <= 2
