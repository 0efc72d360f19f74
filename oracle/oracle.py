"""ctypes front end of the fp64 oracle (``pisa_oracle.c``).

TEST INFRASTRUCTURE ONLY. Imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product package.

Every function follows the page "论文精读 · Block Sparse Attention with
Log-Linear Complexity (PISA)" (qqtang-code.github.io); the C file's header
lists the equations (1)-(7), (11) and the §5.3 conventions it restates and
the readings taken where the page is silent. Inputs are converted to float64
exactly (bf16 and fp32 values are representable), so the oracle sees the
very values the GPU sees.

Pinned by tests/test_oracle_*.py (brute force, closed forms, the page's
worked level tables, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pisa_oracle.c")
_LIB = os.path.join(_HERE, "libpisa_oracle.so")
_lock = threading.Lock()
_lib = None

MAX_LEVELS = 64

__all__ = [
    "build_oracle", "geometry", "total_nodes", "build_pyramid", "pyramid_append",
    "select_rows", "flat_rows", "attn_rows", "attn_backward_rows", "node_score", "threads",
    "to_f64", "MAX_LEVELS",
]


def build_oracle(force: bool = False) -> str:
    """Compile pisa_oracle.c with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build_oracle())
        i64, i32, c_int = ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        P = ctypes.c_void_p
        lib.oracle_geometry.argtypes = [i64, c_int, c_int, P, P]
        lib.oracle_geometry.restype = c_int
        lib.oracle_total_nodes.argtypes = [i64, c_int, c_int]
        lib.oracle_total_nodes.restype = i64
        lib.oracle_build_pyramid.argtypes = [c_int, i64, i64, i64, c_int, c_int, c_int, P, P]
        lib.oracle_build_pyramid.restype = None
        lib.oracle_pyramid_append.argtypes = [i64, i64, c_int, c_int, c_int, P, P]
        lib.oracle_pyramid_append.restype = None
        lib.oracle_node_score.argtypes = [c_int, i64, i64, c_int, c_int, c_int, P, P, P, c_int, i64, c_int]
        lib.oracle_node_score.restype = ctypes.c_double
        lib.oracle_select_rows.argtypes = [c_int, i64, i64, c_int, c_int, c_int, c_int, c_int, c_int,
                                           P, P, i64, P, P, P, P, P, c_int]
        lib.oracle_select_rows.restype = None
        lib.oracle_flat_rows.argtypes = [c_int, c_int, i64, i64, c_int, c_int, c_int, c_int, c_int, c_int,
                                         P, P, i64, P, P, P, P]
        lib.oracle_flat_rows.restype = None
        lib.oracle_attn_rows.argtypes = [i64, c_int, c_int, c_int, c_int, P, P, i64, P, P, P, P, P]
        lib.oracle_attn_rows.restype = None
        _ = i32
        _lib = lib
        return lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def to_f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (any float dtype, any device) or array to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def threads() -> int:
    """Host threads OpenMP will use (OMP_NUM_THREADS or the process affinity)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0))


def geometry(N: int, C: int, g: int = 2):
    """Eq.(3): returns (L, M[1..L], off[1..L]) as python lists (index 0 unused)."""
    lib = _load()
    M = np.zeros(MAX_LEVELS + 1, np.int64)
    off = np.zeros(MAX_LEVELS + 1, np.int64)
    L = lib.oracle_geometry(int(N), int(C), int(g), _p(M), _p(off))
    if L < 0:
        raise ValueError("too many levels")
    return L, M[: L + 1].tolist(), off[: L + 1].tolist()


def total_nodes(N: int, C: int, g: int = 2) -> int:
    return int(_load().oracle_total_nodes(int(N), int(C), int(g)))


def build_pyramid(K: np.ndarray, C: int, g: int = 2, N: int | None = None,
                  N_layout: int | None = None) -> np.ndarray:
    """Eq.(3)-(4). K: [..., rows, d] float64. Returns P: [..., total_nodes(N_layout), d]."""
    K = np.ascontiguousarray(K, dtype=np.float64)
    lead, rows, d = K.shape[:-2], K.shape[-2], K.shape[-1]
    N = rows if N is None else int(N)
    N_layout = N if N_layout is None else int(N_layout)
    BH = int(np.prod(lead)) if lead else 1
    T = total_nodes(N_layout, C, g)
    P = np.zeros(lead + (T, d), np.float64)
    _load().oracle_build_pyramid(BH, N, N_layout, rows, d, C, g, _p(K), _p(P))
    return P


def pyramid_append(P: np.ndarray, Kh: np.ndarray, n: int, C: int, g: int, N_layout: int) -> None:
    """Decode upkeep for one head, in place: refresh the leaf of key n and its ancestors."""
    assert P.dtype == np.float64 and P.flags.c_contiguous
    Kh = np.ascontiguousarray(Kh, dtype=np.float64)
    _load().oracle_pyramid_append(int(n), int(N_layout), Kh.shape[-1], C, g, _p(Kh), _p(P))


VARIANTS = {"lse": 0, "pisa1": 1, "pisa2": 2}


def node_score(qg: np.ndarray, Kh: np.ndarray, P: np.ndarray, level: int, node: int, C: int,
               g: int = 2, N: int | None = None, N_layout: int | None = None, variant: int = 0) -> float:
    """Eq.(7) (+ Eq.11 sum over the G rows of qg [G, d]) for one node; variant
    1 / 2 scores by the PISA-1 / PISA-2 ablation (Eq.8-9) instead."""
    qg = np.ascontiguousarray(np.atleast_2d(qg), dtype=np.float64)
    Kh = np.ascontiguousarray(Kh, dtype=np.float64)
    N = Kh.shape[0] if N is None else N
    N_layout = N if N_layout is None else N_layout
    return float(_load().oracle_node_score(qg.shape[0], N, N_layout, qg.shape[1], C, g,
                                           _p(Kh), _p(np.ascontiguousarray(P)), _p(qg),
                                           int(level), int(node), int(variant)))


def select_rows(Qrows: np.ndarray, t: np.ndarray, Kh: np.ndarray, P: np.ndarray, *, C: int, K: int,
                g: int = 2, causal: bool = True, forced_mask: int = 7, N: int | None = None,
                N_layout: int | None = None, want_counts: bool = False, variant: int = 0):
    """Pyramid walk for query rows of one KV head (node score: variant 0 the
    Eq.7 LSE, 1 PISA-1, 2 PISA-2).

    Qrows: [n, G, d] (G query heads of the group), t: [n] positions.
    Returns (idx [n, K] int32, gap [n] float64[, counts [n, MAX_LEVELS, 2] int32]).
    """
    Qrows = np.ascontiguousarray(Qrows, dtype=np.float64)
    if Qrows.ndim == 2:
        Qrows = Qrows[:, None, :]
    n, G, d = Qrows.shape
    t = np.ascontiguousarray(t, dtype=np.int64)
    Kh = np.ascontiguousarray(Kh, dtype=np.float64)
    P = np.ascontiguousarray(P, dtype=np.float64)
    N = Kh.shape[0] if N is None else int(N)
    N_layout = N if N_layout is None else int(N_layout)
    idx = np.full((n, K), -7, np.int32)
    gap = np.zeros(n, np.float64)
    counts = np.zeros((n, MAX_LEVELS, 2), np.int32) if want_counts else None
    _load().oracle_select_rows(G, N, N_layout, d, C, K, g, int(causal), int(forced_mask),
                               _p(Kh), _p(P), n, _p(t), _p(Qrows), _p(idx), _p(gap), _p(counts), int(variant))
    return (idx, gap, counts) if want_counts else (idx, gap)


def flat_rows(kind: str, Qrows: np.ndarray, t: np.ndarray, Kh: np.ndarray, P: np.ndarray, *,
              C: int, K: int, g: int = 2, causal: bool = True, forced_mask: int = 7,
              N: int | None = None):
    """Flat selection over every eligible leaf.

    kind="bsa": Eq.(1) mean-summary dot (the quadratic BSA comparison);
    kind="lse": exact LSE over each leaf's raw keys (exhaustive reference).
    Returns (idx [n, K] int32, gap [n]).
    """
    k = {"bsa": 0, "lse": 1}[kind]
    Qrows = np.ascontiguousarray(Qrows, dtype=np.float64)
    if Qrows.ndim == 2:
        Qrows = Qrows[:, None, :]
    n, G, d = Qrows.shape
    t = np.ascontiguousarray(t, dtype=np.int64)
    Kh = np.ascontiguousarray(Kh, dtype=np.float64)
    P = np.ascontiguousarray(P, dtype=np.float64)
    N = Kh.shape[0] if N is None else int(N)
    idx = np.full((n, K), -7, np.int32)
    gap = np.zeros(n, np.float64)
    _load().oracle_flat_rows(k, G, N, N, d, C, K, g, int(causal), int(forced_mask),
                             _p(Kh), _p(P), n, _p(t), _p(Qrows), _p(idx), _p(gap))
    return idx, gap


def attn_rows(Qrows: np.ndarray, t: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, idx: np.ndarray, *,
              C: int, causal: bool = True, N: int | None = None, want_lse: bool = False):
    """Eq.(2) with the causal mask: Qrows [n, d], t [n], idx [n, K] -> O [n, d] (float64)."""
    Qrows = np.ascontiguousarray(Qrows, dtype=np.float64)
    n, d = Qrows.shape
    t = np.ascontiguousarray(t, dtype=np.int64)
    Kh = np.ascontiguousarray(Kh, dtype=np.float64)
    Vh = np.ascontiguousarray(Vh, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    K = idx.shape[1]
    N = Kh.shape[0] if N is None else int(N)
    O = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64) if want_lse else None
    _load().oracle_attn_rows(N, d, C, K, int(causal), _p(Kh), _p(Vh), n, _p(t), _p(Qrows),
                             _p(idx), _p(O), _p(lse))
    return (O, lse) if want_lse else O


def attn_backward_rows(Qg: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, idx: np.ndarray, dOg: np.ndarray, *,
                       C: int, causal: bool = True):
    """Backward of Eq.(2) over fixed selected leaves (close reading §5.3: the
    gradient flows only through the selected attention entries), for one KV
    head and its G query heads, every position 0..N-1.

    Qg, dOg: [G, N, d]; Kh, Vh: [N, d]; idx: [N, K] selected leaves (-1 pads).
    Per query row: s = q k_J / sqrt(d) over the keys J of its leaves (j <= t
    when causal), p = softmax(s), o = p V_J; then dV_J += p dO, dp = V_J dO,
    ds = p (dp - dO . o), dq = ds K_J / sqrt(d), dK_J += ds q / sqrt(d).
    Returns (dQ [G, N, d], dK [N, d], dV [N, d]) in float64 (plain numpy, a
    loop over rows: small cases only)."""
    Qg = np.asarray(Qg, np.float64)
    dOg = np.asarray(dOg, np.float64)
    Kh = np.asarray(Kh, np.float64)
    Vh = np.asarray(Vh, np.float64)
    G, N, d = Qg.shape
    inv = 1.0 / np.sqrt(d)
    dQ = np.zeros_like(Qg)
    dK = np.zeros_like(Kh)
    dV = np.zeros_like(Vh)
    for t in range(N):
        J = []
        for leaf in idx[t]:
            if leaf < 0:
                continue
            hi = min((int(leaf) + 1) * C, N)
            if causal:
                hi = min(hi, t + 1)
            J.extend(range(int(leaf) * C, hi))
        J = np.array(sorted(J), np.int64)
        if J.size == 0:
            continue
        KJ, VJ = Kh[J], Vh[J]
        for h in range(G):
            s = KJ @ Qg[h, t] * inv
            p = np.exp(s - s.max())
            p /= p.sum()
            o = p @ VJ
            do = dOg[h, t]
            dV[J] += np.outer(p, do)
            dp = VJ @ do
            ds = p * (dp - do @ o)
            dQ[h, t] = ds @ KJ * inv
            dK[J] += np.outer(ds, Qg[h, t]) * inv
    return dQ, dK, dV


def attn_backward_sampled(Qg: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, idx: np.ndarray, dOg: np.ndarray, *,
                          C: int, causal: bool = True, rows=(), leaves=()):
    """Selected entries of attn_backward_rows, for checks at sizes where the
    full backward is out of reach: dQ of the query positions `rows` (each needs
    its own row only) and dK, dV of the keys of the leaves `leaves` (each needs
    every position whose idx lists the leaf: its softmax over all of its
    selected keys, and its D = dO . o).

    Same arithmetic per row as attn_backward_rows. Returns (dQ [G, len(rows), d],
    dK [len(leaves), C, d], dV [len(leaves), C, d]) in float64; key rows past N
    stay zero."""
    G, N, d = Qg.shape
    inv = 1.0 / np.sqrt(d)

    def row_terms(t: int, h: int):
        J = []
        for leaf in idx[t]:
            if leaf < 0:
                continue
            hi = min((int(leaf) + 1) * C, N)
            if causal:
                hi = min(hi, t + 1)
            J.extend(range(int(leaf) * C, hi))
        J = np.array(sorted(J), np.int64)
        q = np.asarray(Qg[h, t], np.float64)
        do = np.asarray(dOg[h, t], np.float64)
        KJ = np.asarray(Kh[J], np.float64)
        VJ = np.asarray(Vh[J], np.float64)
        s = KJ @ q * inv
        p = np.exp(s - s.max())
        p /= p.sum()
        o = p @ VJ
        ds = p * (VJ @ do - do @ o)
        return J, p, ds, q, do, KJ

    dQ = np.zeros((G, len(rows), d))
    for i, t in enumerate(rows):
        for h in range(G):
            J, p, ds, q, do, KJ = row_terms(int(t), h)
            if J.size:
                dQ[h, i] = ds @ KJ * inv
    dK = np.zeros((len(leaves), C, d))
    dV = np.zeros((len(leaves), C, d))
    for li, leaf in enumerate(leaves):
        users = np.nonzero((np.asarray(idx) == leaf).any(axis=1))[0]
        if len(users) > 2048:  # many users (a forced first leaf): the same sums, batched over the users
            dK[li], dV[li] = attn_backward_leaf(Qg, Kh, Vh, idx, dOg, int(leaf), C=C, causal=causal)
            continue
        for t in users:
            for h in range(G):
                J, p, ds, q, do, KJ = row_terms(int(t), h)
                m = (J >= leaf * C) & (J < (leaf + 1) * C)
                if not m.any():
                    continue
                kl = J[m] - leaf * C
                dV[li, kl] += np.outer(p[m], do)
                dK[li, kl] += np.outer(ds[m], q) * inv
    return dQ, dK, dV


def attn_backward_leaf(Qg: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, idx: np.ndarray, dOg: np.ndarray,
                       leaf: int, *, C: int, causal: bool = True):
    """dK and dV of the keys of one leaf (the backward of Eq.(2) over fixed
    selected leaves, close reading §5.3), summed over every position whose idx
    lists the leaf, for leaves with many such positions (a forced first leaf
    has all N of them).

    Per user row t and head h: its softmax normaliser (the log-sum-exp over all
    of its selected keys, j <= t when causal) and its output o come from
    attn_rows; then for the leaf's keys j: p_j = exp(q.k_j / sqrt(d) - lse),
    dp_j = dO . v_j, ds_j = p_j (dp_j - dO . o); dV_j += p_j dO and
    dK_j += ds_j q / sqrt(d). The same terms as attn_backward_rows, taken for
    all users at once. Returns (dK [C, d], dV [C, d]) in float64; key rows
    past N stay zero."""
    G, N, d = Qg.shape
    inv = 1.0 / np.sqrt(d)
    idx = np.asarray(idx)
    users = np.nonzero((idx == leaf).any(axis=1))[0].astype(np.int64)
    dK = np.zeros((C, d))
    dV = np.zeros((C, d))
    lo, hi = leaf * C, min((leaf + 1) * C, N)
    if users.size == 0 or lo >= N:
        return dK, dV
    Kl = np.asarray(Kh[lo:hi], np.float64)
    Vl = np.asarray(Vh[lo:hi], np.float64)
    keys = np.arange(lo, hi)
    for h in range(G):
        q = np.asarray(Qg[h][users], np.float64)
        do = np.asarray(dOg[h][users], np.float64)
        o, lse = attn_rows(q, users, Kh, Vh, idx[users], C=C, causal=causal, N=N, want_lse=True)
        s = q @ Kl.T * inv
        p = np.exp(s - lse[:, None])
        if causal:
            p = np.where(keys[None, :] <= users[:, None], p, 0.0)
        ds = p * (do @ Vl.T - np.sum(do * o, axis=1)[:, None])
        dV[:hi - lo] += p.T @ do
        dK[:hi - lo] += ds.T @ q * inv
    return dK, dV
