"""Thin Python binding of ``libpisa.so`` (include/pisa.h), same names as the C ABI.

Argument marshalling only: torch tensors are passed as raw device pointers
together with torch's current CUDA stream; every step of the path runs in the
library's CUDA kernels. If the library is missing or a tensor is not on a CUDA
device, the call raises -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpisa.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "pisa.h")

PISA_DTYPE_F32, PISA_DTYPE_BF16 = 0, 1
STATUS = {0: "PISA_OK", -1: "PISA_E_INVALID", -2: "PISA_E_UNSUPPORTED", -3: "PISA_E_CUDA",
          -4: "PISA_E_ALIGNMENT", -5: "PISA_E_TIMEOUT", -6: "PISA_E_SCRATCH_LIMIT"}


class PisaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({msg})")
        self.status = status


class PisaCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "N", "d", "C", "K", "g", "causal", "forced_mask", "dtype", "score_variant")]


_lock = threading.Lock()
_lib = None


def exported_names() -> list[str]:
    """Function names declared in include/pisa.h."""
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z0-9_]+\s*\*?\s*(pisa_[a-z0-9_]+)\s*\(", src, re.M)))


def load(path: str | None = None):
    """Load libpisa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if path is None:
            from . import build as _build
            if not _build.up_to_date():  # sources newer than the library: rebuild, never run a stale one
                _build.build()
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m hierarchical_block_sparse_b200.build`")
        lib = ctypes.CDLL(p)
        P = ctypes.c_void_p
        cfgp = ctypes.POINTER(PisaCfg)
        sig = {
            "pisa_num_levels": (ctypes.c_int, [cfgp]),
            "pisa_level_nodes": (ctypes.c_int64, [cfgp, ctypes.c_int]),
            "pisa_level_offset": (ctypes.c_int64, [cfgp, ctypes.c_int]),
            "pisa_pyramid_rows": (ctypes.c_int64, [cfgp]),
            "pisa_build_pyramid": (ctypes.c_int, [cfgp, P, P, P]),
            "pisa_select": (ctypes.c_int, [cfgp, P, P, P, P, P]),
            "pisa_sparse_attn": (ctypes.c_int, [cfgp, P, P, P, P, P, P]),
            "pisa_forward": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P]),
            "pisa_bsa_select": (ctypes.c_int, [cfgp, P, P, P, P]),
            "pisa_bsa_select_ws": (ctypes.c_int, [cfgp, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_workspace_bytes": (ctypes.c_int64, [cfgp]),
            "pisa_workspace_status": (ctypes.c_int, [cfgp, P, P]),
            "pisa_select_ws": (ctypes.c_int, [cfgp, P, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_sparse_attn_ws": (ctypes.c_int, [cfgp, P, P, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_forward_ws": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_forward_host": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_forward_ws_events": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, ctypes.c_size_t,
                                                      ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, P]),
            "pisa_select_noalloc": (ctypes.c_int, [cfgp, P, P, P, P, P]),
            "pisa_select_noalloc_status": (ctypes.c_int, [cfgp, P]),
            "pisa_build_pyramid_prefix": (ctypes.c_int, [cfgp, P, P, P, P]),
            "pisa_pyramid_append": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P]),
            "pisa_pyramid_grow": (ctypes.c_int, [cfgp, P, cfgp, P, P]),
            "pisa_cache_capacity": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int]),
            "pisa_cache_grow": (ctypes.c_int, [cfgp, P, P, P, cfgp, P, P, P, P]),
            "pisa_sparse_attn_backward": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P]),
            "pisa_backward_workspace_bytes": (ctypes.c_int64, [cfgp]),
            "pisa_sparse_attn_backward_ws": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
            "pisa_sparse_attn_backward_saved_ws": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, ctypes.c_size_t,
                                                                  P]),
            "pisa_sparse_attn_backward_ws_events": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, ctypes.c_size_t,
                                                                   ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, P]),
            "pisa_decode": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P]),
            "pisa_decode_step": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, P, P]),
            "pisa_fma_probe": (ctypes.c_int, [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]),
            "pisa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "pisa_version": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        if path is None:
            _lib = lib
        return lib


PISA_SCORE_LSE, PISA_SCORE_MEAN, PISA_SCORE_MEAN_VAR = 0, 1, 2


def make_cfg(*, B: int, Hq: int, Hkv: int, N: int, d: int, C: int, K: int, g: int = 2, causal: bool = True,
             forced_mask: int = 7, dtype=torch.bfloat16, score_variant: int = PISA_SCORE_LSE) -> PisaCfg:
    dt = {torch.bfloat16: PISA_DTYPE_BF16, torch.float32: PISA_DTYPE_F32}.get(dtype, dtype)
    return PisaCfg(B, Hq, Hkv, N, d, C, K, g, int(causal), forced_mask, int(dt), int(score_variant))


def cfg_for(Q: torch.Tensor, K: torch.Tensor, *, C: int, K_: int, causal: bool = True, forced_mask: int = 7,
            g: int = 2, score_variant: int = PISA_SCORE_LSE) -> PisaCfg:
    B, Hq, N, d = Q.shape
    return make_cfg(B=B, Hq=Hq, Hkv=K.shape[1], N=N, d=d, C=C, K=K_, g=g, causal=causal,
                    forced_mask=forced_mask, dtype=Q.dtype, score_variant=score_variant)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("host buffers must live in host memory")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(name: str, status: int):
    if status != 0:
        raise PisaError(name, status, load().pisa_status_string(status).decode())


# ---- geometry -------------------------------------------------------------------

def pisa_num_levels(cfg: PisaCfg) -> int:
    return int(load().pisa_num_levels(ctypes.byref(cfg)))


def pisa_level_nodes(cfg: PisaCfg, level: int) -> int:
    return int(load().pisa_level_nodes(ctypes.byref(cfg), level))


def pisa_level_offset(cfg: PisaCfg, level: int) -> int:
    return int(load().pisa_level_offset(ctypes.byref(cfg), level))


def pisa_pyramid_rows(cfg: PisaCfg) -> int:
    r = int(load().pisa_pyramid_rows(ctypes.byref(cfg)))
    if r < 0:
        _check("pisa_pyramid_rows", r)
    return r


# ---- prefill ----------------------------------------------------------------------

def pisa_build_pyramid(cfg, K, pyr):
    _check("pisa_build_pyramid", load().pisa_build_pyramid(ctypes.byref(cfg), _ptr(K), _ptr(pyr), _stream()))


def pisa_select(cfg, Q, K, pyr, idx):
    _check("pisa_select", load().pisa_select(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(pyr), _ptr(idx), _stream()))


def pisa_sparse_attn(cfg, Q, K, V, idx, O):
    _check("pisa_sparse_attn", load().pisa_sparse_attn(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                                       _ptr(O), _stream()))


def pisa_forward(cfg, Q, K, V, pyr, idx, O):
    _check("pisa_forward", load().pisa_forward(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(pyr), _ptr(idx),
                                               _ptr(O), _stream()))


def pisa_bsa_select(cfg, Q, pyr, idx):
    _check("pisa_bsa_select", load().pisa_bsa_select(ctypes.byref(cfg), _ptr(Q), _ptr(pyr), _ptr(idx), _stream()))


def pisa_bsa_select_ws(cfg, Q, pyr, idx, ws):
    """Flat BSA selection (Eq.1) on the tensor cores, in the block-major workspace."""
    _check("pisa_bsa_select_ws", load().pisa_bsa_select_ws(ctypes.byref(cfg), _ptr(Q), _ptr(pyr), _ptr(idx),
                                                           _ptr(ws), ws.numel(), _stream()))


# ---- block-major tensor-core prefill (workspace) -----------------------------------

def pisa_workspace_bytes(cfg) -> int:
    r = int(load().pisa_workspace_bytes(ctypes.byref(cfg)))
    if r < 0:
        _check("pisa_workspace_bytes", r)
    return r


def alloc_workspace(cfg, device="cuda") -> torch.Tensor:
    """Caller-owned workspace for the *_ws calls (torch allocates; 256-byte aligned)."""
    return torch.empty(max(pisa_workspace_bytes(cfg), 256), dtype=torch.uint8, device=device)


def pisa_workspace_status(cfg, ws) -> int:
    """0, or -5 (PISA_E_TIMEOUT) when a tensor-core tile gave up a bounded wait (synchronises)."""
    return int(load().pisa_workspace_status(ctypes.byref(cfg), _ptr(ws), _stream()))


def pisa_select_ws(cfg, Q, K, pyr, idx, ws):
    _check("pisa_select_ws", load().pisa_select_ws(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(pyr), _ptr(idx),
                                                   _ptr(ws), ws.numel(), _stream()))


def pisa_sparse_attn_ws(cfg, Q, K, V, idx, O, ws):
    _check("pisa_sparse_attn_ws", load().pisa_sparse_attn_ws(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V),
                                                             _ptr(idx), _ptr(O), _ptr(ws), ws.numel(), _stream()))


def pisa_forward_ws(cfg, Q, K, V, pyr, idx, O, ws):
    _check("pisa_forward_ws", load().pisa_forward_ws(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(pyr),
                                                     _ptr(idx), _ptr(O), _ptr(ws), ws.numel(), _stream()))


def pisa_forward_host(cfg, Q_host, K_host, V_host, idx_host, O_host, Q, K, V, pyr, idx, O, ws):
    """pisa_forward_ws from host buffers (pinned for asynchronous copies) on the current stream."""
    _check("pisa_forward_host", load().pisa_forward_host(
        ctypes.byref(cfg), _host_ptr(Q_host), _host_ptr(K_host), _host_ptr(V_host), _host_ptr(idx_host),
        _host_ptr(O_host), _ptr(Q), _ptr(K), _ptr(V), _ptr(pyr), _ptr(idx), _ptr(O), _ptr(ws), ws.numel(),
        _stream()))


def pisa_select_noalloc(cfg, Q, K, pyr, idx):
    """pisa_select_ws without a workspace: for callers that cannot allocate device
    memory, the library's fixed 32 MiB scratch array is used instead (calls on a
    device share it, so they must not overlap on the GPU)."""
    _check("pisa_select_noalloc", load().pisa_select_noalloc(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(pyr),
                                                             _ptr(idx), _stream()))


def pisa_select_noalloc_status(cfg) -> int:
    """Error word of the last pisa_select_noalloc on this device: 0, or -5
    (PISA_E_TIMEOUT) when a tile gave up a bounded wait or a self-check failed
    (synchronises the current stream)."""
    return int(load().pisa_select_noalloc_status(ctypes.byref(cfg), _stream()))


def pisa_fma_probe(out, blocks: int, iters: int, packed: bool):
    """Launch the fp32 FMA throughput probe on the current stream (out: fp32, blocks * 256 elements)."""
    assert out.numel() >= blocks * 256 and out.dtype == torch.float32
    _check("pisa_fma_probe", load().pisa_fma_probe(_ptr(out), int(blocks), int(iters), int(bool(packed)),
                                                   _stream()))


PHASES = ["pyramid", "stage1", "group_candidates", "leaf_scores", "topk", "group_kept", "forced_tiles",
          "attn_tiles", "finalize"]


def pisa_forward_ws_events(cfg, Q, K, V, pyr, idx, O, ws, events):
    """pisa_forward_ws recording torch.cuda.Event objects (len(PHASES) + 1) at phase boundaries."""
    stream = torch.cuda.current_stream()
    for e in events:
        if e.cuda_event == 0:  # torch creates the underlying event on first record
            e.record(stream)
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("pisa_forward_ws_events", load().pisa_forward_ws_events(
        ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(pyr), _ptr(idx), _ptr(O), _ptr(ws), ws.numel(),
        arr, len(events), _stream()))


# ---- decode -------------------------------------------------------------------------

def pisa_build_pyramid_prefix(cfg, Kc, length, pyr):
    _check("pisa_build_pyramid_prefix", load().pisa_build_pyramid_prefix(ctypes.byref(cfg), _ptr(Kc), _ptr(length),
                                                                         _ptr(pyr), _stream()))


def pisa_pyramid_append(cfg, Kc, Vc, pyr, k_new, v_new, pos):
    _check("pisa_pyramid_append", load().pisa_pyramid_append(ctypes.byref(cfg), _ptr(Kc), _ptr(Vc), _ptr(pyr),
                                                             _ptr(k_new), _ptr(v_new), _ptr(pos), _stream()))


def pisa_sparse_attn_backward(cfg, Q, K, V, idx, dO, dQ, dK, dV):
    """dQ, dK, dV (fp32) of the sparse attention for the fixed selection idx."""
    _check("pisa_sparse_attn_backward", load().pisa_sparse_attn_backward(
        ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _stream()))


def pisa_backward_workspace_bytes(cfg) -> int:
    r = int(load().pisa_backward_workspace_bytes(ctypes.byref(cfg)))
    if r < 0:
        _check("pisa_backward_workspace_bytes", r)
    return r


def alloc_backward_workspace(cfg, device="cuda") -> torch.Tensor:
    """Caller-owned workspace for pisa_sparse_attn_backward_ws (256-byte aligned)."""
    return torch.empty(max(pisa_backward_workspace_bytes(cfg), 256), dtype=torch.uint8, device=device)


def pisa_sparse_attn_backward_ws(cfg, Q, K, V, idx, dO, dQ, dK, dV, ws):
    """pisa_sparse_attn_backward, block-major on the tensor cores (bf16, d = 128, C = 64)."""
    _check("pisa_sparse_attn_backward_ws", load().pisa_sparse_attn_backward_ws(
        ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(ws),
        ws.numel(), _stream()))


def pisa_sparse_attn_backward_saved_ws(cfg, Q, K, V, idx, dO, dQ, dK, dV, ws):
    """The backward reusing what pisa_forward_ws / pisa_sparse_attn_ws left in ws (same inputs)."""
    _check("pisa_sparse_attn_backward_saved_ws", load().pisa_sparse_attn_backward_saved_ws(
        ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(ws),
        ws.numel(), _stream()))


BWD_PHASES = ["statistics", "zeroing", "backward_tiles"]


def pisa_sparse_attn_backward_ws_events(cfg, Q, K, V, idx, dO, dQ, dK, dV, ws, events):
    """pisa_sparse_attn_backward_ws recording torch.cuda.Event objects (len(BWD_PHASES) + 1)."""
    stream = torch.cuda.current_stream()
    for e in events:
        if e.cuda_event == 0:
            e.record(stream)
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("pisa_sparse_attn_backward_ws_events", load().pisa_sparse_attn_backward_ws_events(
        ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(ws),
        ws.numel(), arr, len(events), _stream()))


def pisa_pyramid_grow(cfg_old, pyr_old, cfg_new, pyr_new):
    _check("pisa_pyramid_grow", load().pisa_pyramid_grow(ctypes.byref(cfg_old), _ptr(pyr_old), ctypes.byref(cfg_new),
                                                         _ptr(pyr_new), _stream()))


def pisa_cache_capacity(n: int, C: int) -> int:
    """The library's geometric capacity for n cached keys (smallest C * 2^k >= n)."""
    r = int(load().pisa_cache_capacity(int(n), int(C)))
    if r < 0:
        _check("pisa_cache_capacity", r)
    return r


def pisa_cache_grow(cfg_old, Kc_old, Vc_old, pyr_old, cfg_new, Kc_new, Vc_new, pyr_new):
    _check("pisa_cache_grow", load().pisa_cache_grow(ctypes.byref(cfg_old), _ptr(Kc_old), _ptr(Vc_old), _ptr(pyr_old),
                                                     ctypes.byref(cfg_new), _ptr(Kc_new), _ptr(Vc_new),
                                                     _ptr(pyr_new), _stream()))


class DecodeCache:
    """K and V caches [B, Hkv, capacity, d] and their pyramid, grown by the
    library's geometric policy: before a step would write at or past the
    capacity, buffers of pisa_cache_capacity(needed) rows are allocated (torch)
    and pisa_cache_grow moves the contents. cfg.N is the capacity. The
    per-sequence positions stay in the caller's pos tensor."""

    def __init__(self, cfg, Kc: torch.Tensor, Vc: torch.Tensor, pyr: torch.Tensor):
        self.cfg, self.Kc, self.Vc, self.pyr = cfg, Kc, Vc, pyr

    @property
    def capacity(self) -> int:
        return int(self.cfg.N)

    def reserve(self, n: int) -> None:
        """Make room for n keys per sequence (grows geometrically when needed)."""
        if n <= self.cfg.N:
            return
        c = self.cfg
        new = PisaCfg(c.B, c.Hq, c.Hkv, pisa_cache_capacity(n, c.C), c.d, c.C, c.K, c.g, c.causal, c.forced_mask,
                      c.dtype, c.score_variant)
        shape = (c.B, c.Hkv, new.N, c.d)
        # growing writes every row of the new buffers, except from an empty cache (nothing to move)
        alloc = torch.zeros if c.N == 0 else torch.empty
        Kc = alloc(shape, dtype=self.Kc.dtype, device=self.Kc.device)
        Vc = alloc(shape, dtype=self.Vc.dtype, device=self.Vc.device)
        pyr = alloc((c.B, c.Hkv, pisa_pyramid_rows(new), c.d), dtype=torch.float32, device=self.pyr.device)
        pisa_cache_grow(c, self.Kc, self.Vc, self.pyr, new, Kc, Vc, pyr)
        self.cfg, self.Kc, self.Vc, self.pyr = new, Kc, Vc, pyr

    def step(self, q_new, k_new, v_new, pos, idx, o, max_pos: int) -> None:
        """pisa_decode_step for every sequence, growing first if the largest
        position (max_pos, a host value: no device read) reaches the capacity."""
        self.reserve(max_pos + 1)
        pisa_decode_step(self.cfg, q_new, k_new, v_new, self.Kc, self.Vc, self.pyr, pos, idx, o)


def pisa_decode(cfg, q_new, Kc, Vc, pyr, pos, idx, o):
    _check("pisa_decode", load().pisa_decode(ctypes.byref(cfg), _ptr(q_new), _ptr(Kc), _ptr(Vc), _ptr(pyr),
                                             _ptr(pos), _ptr(idx), _ptr(o), _stream()))


def pisa_decode_step(cfg, q_new, k_new, v_new, Kc, Vc, pyr, pos, idx, o):
    _check("pisa_decode_step", load().pisa_decode_step(ctypes.byref(cfg), _ptr(q_new), _ptr(k_new), _ptr(v_new),
                                                       _ptr(Kc), _ptr(Vc), _ptr(pyr), _ptr(pos), _ptr(idx), _ptr(o),
                                                       _stream()))


def pisa_status_string(status: int) -> str:
    return load().pisa_status_string(status).decode()


def pisa_version() -> str:
    return load().pisa_version().decode()


# ---- allocation helpers (torch owns the memory) --------------------------------------

def alloc_outputs(cfg: PisaCfg, device="cuda", dtype=torch.bfloat16):
    """pyr (fp32), idx (int32) and O tensors sized for cfg."""
    R = pisa_pyramid_rows(cfg)
    pyr = torch.empty((cfg.B, cfg.Hkv, R, cfg.d), dtype=torch.float32, device=device)
    idx = torch.empty((cfg.B, cfg.Hkv, cfg.N, cfg.K), dtype=torch.int32, device=device)
    O = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=dtype, device=device)
    return pyr, idx, O


def forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, *, C: int, K_: int, causal: bool = True,
            forced_mask: int = 7):
    """Allocate outputs and run pisa_forward. Returns (O, idx, pyr)."""
    cfg = cfg_for(Q, K, C=C, K_=K_, causal=causal, forced_mask=forced_mask)
    pyr, idx, O = alloc_outputs(cfg, Q.device, Q.dtype)
    pisa_forward(cfg, Q, K, V, pyr, idx, O)
    return O, idx, pyr
