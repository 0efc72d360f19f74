"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module holds only shapes and random numbers: none of the method's
arithmetic. Workloads follow the page "论文精读 · Block Sparse Attention with
Log-Linear Complexity (PISA)", §7.3 (random bf16 query/key tensors, fp32
accumulation, C=64, g=2) scaled to the five problem sizes below.

Recipe: numpy ``default_rng(42 + index)`` draws, in order, Q, K, V as i.i.d.
N(0, 1) float32 in [B, H, N, d] layout; the planted-retrieval workload then
draws a unit vector u and, per KV head, 8 distinct needle leaves; needle keys
become 4u + N(0, 0.1^2) noise and every query gets +2u. Values are rounded to
the workload dtype (round-to-nearest-even bf16) once, and that rounded tensor
is what both sides consume.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "decode_pool", "decode_offset",
           "decode_cache", "decode_rows", "decode_step_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    C: int
    K: int
    g: int = 2
    causal: bool = True
    forced_mask: int = 7
    dtype: str = "bf16"          # "bf16" or "f32" for Q, K, V and O
    needles: int = 0             # planted needle leaves per KV head
    decode_batch: int = 0        # sequences in the decode step (0: prefill only)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seed(self) -> int:
        return 42 + self.index

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # tiny fp32 case the oracle finishes in well under a second
    "tiny_f32_n1k": Workload("tiny_f32_n1k", 0, B=1, Hq=1, Hkv=1, N=1024, d=64, C=16, K=4, dtype="f32"),
    # short-context MHA prefill, 16 heads, 16K tokens
    "mha16_n16k": Workload("mha16_n16k", 1, B=1, Hq=16, Hkv=16, N=16384, d=128, C=64, K=16),
    # planted-retrieval MHA prefill, 16 heads, 64K tokens, 8 needle leaves per head
    "needle_mha16_n64k": Workload("needle_mha16_n64k", 2, B=1, Hq=16, Hkv=16, N=65536, d=128, C=64, K=16,
                                  needles=8),
    # GQA 32 query heads / 8 KV heads, 128K tokens
    "gqa32x8_n128k": Workload("gqa32x8_n128k", 3, B=1, Hq=32, Hkv=8, N=131072, d=128, C=64, K=16),
    # long MHA prefill, 8 heads, 256K tokens; decode with 64 sequences against 256K-key caches
    "mha8_n256k": Workload("mha8_n256k", 4, B=1, Hq=8, Hkv=8, N=262144, d=128, C=64, K=16, decode_batch=64),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _round(x: np.ndarray, dtype: str):
    """float32 ndarray -> torch tensor of the workload dtype (RNE for bf16)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def make_inputs(w: Workload, *, N: int | None = None, seed: int | None = None):
    """Q [B,Hq,N,d], K/V [B,Hkv,N,d] as CPU torch tensors of the workload dtype,
    plus meta {"u": unit vector or None, "needles": [B,Hkv,n] leaf ids or None}."""
    N = w.N if N is None else N
    rng = np.random.default_rng(w.seed if seed is None else seed)
    f32 = np.float32
    Q = rng.standard_normal((w.B, w.Hq, N, w.d), dtype=f32)
    K = rng.standard_normal((w.B, w.Hkv, N, w.d), dtype=f32)
    V = rng.standard_normal((w.B, w.Hkv, N, w.d), dtype=f32)
    meta = {"u": None, "needles": None}
    if w.needles:
        u = rng.standard_normal(w.d).astype(np.float64)
        u = (u / np.linalg.norm(u)).astype(f32)
        M1 = -(-N // w.C)
        needles = np.zeros((w.B, w.Hkv, w.needles), np.int64)
        for b in range(w.B):
            for h in range(w.Hkv):
                needles[b, h] = np.sort(rng.choice(M1, size=w.needles, replace=False))
                for leaf in needles[b, h]:
                    lo, hi = leaf * w.C, min(leaf * w.C + w.C, N)
                    noise = rng.standard_normal((hi - lo, w.d), dtype=f32) * f32(0.1)
                    K[b, h, lo:hi] = f32(4.0) * u[None, :] + noise
        Q += f32(2.0) * u
        meta = {"u": u, "needles": needles}
    return _round(Q, w.dtype), _round(K, w.dtype), _round(V, w.dtype), meta


def decode_pool(w: Workload, rows: int, *, seed: int | None = None):
    """Host pool of K and V rows [Hkv, rows, d] for decode caches.

    Sequence s of the decode batch holds pool rows starting at offset
    ``s * stride`` (mod rows) -- see ``decode_rows`` -- so a 64-sequence,
    256K-key cache (tens of GB) is filled from one seeded pool while every
    sequence still sees its own i.i.d. N(0,1) rows.
    """
    rng = np.random.default_rng((w.seed if seed is None else seed) + 1000)
    Kp = rng.standard_normal((w.Hkv, rows, w.d), dtype=np.float32)
    Vp = rng.standard_normal((w.Hkv, rows, w.d), dtype=np.float32)
    return _round(Kp, w.dtype), _round(Vp, w.dtype)


def decode_offset(seq: int, rows: int, stride: int = 7919) -> int:
    """Row of the pool where sequence ``seq``'s cache starts (wraps around)."""
    return (seq * stride) % rows


def decode_cache(w: Workload, cap: int, prefix: int, device, *, seed: int | None = None):
    """Device caches Kc, Vc [decode_batch, Hkv, cap, d] whose first ``prefix``
    rows hold each sequence's keys/values, drawn from one seeded host pool
    (see ``decode_pool``). Rows from ``prefix`` on are zero.
    Returns (Kc, Vc, Kpool, Vpool) with the pools on the host."""
    import torch
    Kp, Vp = decode_pool(w, prefix, seed=seed)
    B = w.decode_batch
    dt = Kp.dtype
    Kc = torch.zeros((B, w.Hkv, cap, w.d), dtype=dt, device=device)
    Vc = torch.zeros((B, w.Hkv, cap, w.d), dtype=dt, device=device)
    Kd, Vd = Kp.to(device), Vp.to(device)
    for s in range(B):
        off = decode_offset(s, prefix)
        for src, dst in ((Kd, Kc), (Vd, Vc)):
            dst[s, :, : prefix - off].copy_(src[:, off:])
            if off:
                dst[s, :, prefix - off: prefix].copy_(src[:, :off])
    return Kc, Vc, Kp, Vp


def decode_rows(pool, seq: int, prefix: int):
    """Host copy of sequence ``seq``'s first ``prefix`` cached rows [Hkv, prefix, d]."""
    import torch
    off = decode_offset(seq, prefix)
    return torch.cat([pool[:, off:prefix], pool[:, :off]], dim=1)


def decode_step_inputs(w: Workload, step: int, *, B: int | None = None, seed: int | None = None):
    """q_new [B, Hq, d], k_new and v_new [B, Hkv, d] for decode step ``step``."""
    B = w.decode_batch if B is None else B
    rng = np.random.default_rng([(w.seed if seed is None else seed), 2000 + step])
    q = rng.standard_normal((B, w.Hq, w.d), dtype=np.float32)
    k = rng.standard_normal((B, w.Hkv, w.d), dtype=np.float32)
    v = rng.standard_normal((B, w.Hkv, w.d), dtype=np.float32)
    return _round(q, w.dtype), _round(k, w.dtype), _round(v, w.dtype)
