#!/usr/bin/env python
"""Prefill benchmark of the PISA path (pyramid pooling -> pyramid Top-K
selection -> sparse attention) on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pisa|reference]
                    [--workload mha8_n256k] [--seq N] [--no-decode] [--no-cpu-baseline]
                    [--no-bsa] [--no-sweep] [--no-per-config] [--no-backward]
                    [--no-variants] [--no-per-query] [--decode-only]

A step is one pisa_forward_ws over the whole workload (B*N tokens, all
heads) with inputs resident in HBM. Rank 0 prints one JSON line: the step,
its phases and the dominant phase's roofline, the end-to-end figure through
pisa_forward_host from pinned host buffers, the other prefill workloads,
flat BSA selection beside PISA's (and a sweep of both to 1M tokens), the
PISA-1 / PISA-2 scores, the backward with the selection fixed, the decode
step and the oracle's CPU baseline. Under torchrun every rank runs its own
seeded copy of the workload (weak scaling, no data-path collective); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FP32_LANES_PER_SM = 128
SM_COUNT = 148


def peaks():
    """Measured peaks (driver-written) or the recipe's fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "sm_max_mhz": d.get("sm_max_mhz", 1965.0),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def fp32_fma_peak_tflops(sm_mhz: float) -> float:
    """CUDA-core fp32 FMA peak: SMs x 128 lanes x 2 FLOP x clock."""
    return SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------- work model ----

def walk_counts(N: int, C: int, K: int, forced_mask: int):
    """Per query position t (causal): dots scored at internal levels, raw keys
    scored at the leaves, and keys attended. Exact for the causal walk: only
    WHICH non-forced nodes survive depends on the data; how many candidates each
    level has depends on t alone (non-forced survivors are wholly in the past
    and have both children; forced paths are fixed by t)."""
    t = np.arange(N, dtype=np.int64)
    c = t // C
    M1 = -(-N // C)
    L = 1
    m = M1
    while m > 1:
        m = -(-m // 2)
        L += 1
    n = np.ones(N, np.int64)            # candidates at the current level
    internal = np.zeros(N, np.int64)
    leafkeys = np.zeros(N, np.int64)
    attended = np.zeros(N, np.int64)
    forced_keys = np.zeros(N, np.int64)
    for lvl in range(L, 0, -1):
        s = lvl - 1
        cur = c >> s
        fs = [cur]
        if forced_mask & 1:
            fs.append(np.where(cur != 0, 0, -1))
        if forced_mask & 2:
            prev = np.where(c >= 1, (c - 1) >> s, -1)
            prev = np.where((prev == cur) | ((forced_mask & 1) & (prev == 0)), -1, prev)
            fs.append(prev)
        nf = sum((f >= 0).astype(np.int64) for f in fs)
        kept = np.minimum(n, K)
        scored = np.where((n > K) & (K - nf > 0), n - nf, 0)
        if lvl >= 2:
            internal += scored * 2
            span_child = C << (lvl - 2)
            nxt = 2 * (kept - nf)
            for f in fs:
                ok = f >= 0
                right_ok = (2 * f + 1) * span_child <= t
                nxt += np.where(ok, 1 + right_ok.astype(np.int64), 0)
            n = nxt
        else:
            leafkeys += scored * C
            fk = t - c * C + 1
            for f in fs[1:]:
                fk = fk + np.where(f >= 0, C, 0)
            attended += (kept - nf) * C + fk
            forced_keys += fk
    walk_counts.forced_keys = forced_keys
    return internal, leafkeys, attended


def algorithmic(w, N: int):
    """Per-launch algorithmic FLOPs and compulsory bytes of one prefill step."""
    internal, leafkeys, attended = walk_counts(N, w.C, w.K, w.forced_mask)
    G = w.Hq // w.Hkv
    units = w.B * w.Hkv
    e = 2 if w.dtype == "bf16" else 4
    d = w.d
    from hierarchical_block_sparse_b200.workloads import Workload  # noqa: F401
    M1 = -(-N // w.C)
    rows = 0
    m = M1
    while True:
        rows += m
        if m == 1:
            break
        m = -(-m // 2)
    q_b = w.B * w.Hq * N * d * e
    k_b = w.B * w.Hkv * N * d * e
    pyr_b = w.B * w.Hkv * rows * d * 4
    idx_b = w.B * w.Hkv * N * w.K * 4
    return {
        "internal_flops": float(units * G * internal.sum() * 2 * d),
        "leaf_flops": float(units * G * leafkeys.sum() * 2 * d),
        "select_flops": float(units * G * (internal.sum() + leafkeys.sum()) * 2 * d),
        "attn_flops": float(units * G * attended.sum() * 4 * d),
        "attn_forced_flops": float(units * G * walk_counts.forced_keys.sum() * 4 * d),
        "attn_free_flops": float(units * G * (attended.sum() - walk_counts.forced_keys.sum()) * 4 * d),
        "select_dots_per_query": float((internal.sum() + leafkeys.sum()) / N),
        "attended_keys_per_query": float(attended.sum() / N),
        "pool_bytes": float(k_b + pyr_b),
        "select_bytes": float(q_b + k_b + pyr_b + idx_b),
        "attn_bytes": float(q_b + 2 * k_b + idx_b + q_b),
        "prefill_bytes": float(q_b + 2 * k_b + q_b + pyr_b + idx_b),
        "selection_bytes": float(q_b + k_b + pyr_b + idx_b),
    }


def source_sha(parts):
    """Hash of a kernel's sources: whole files, or (file, section) pairs for the
    section of a file that starts at a "// ---- <section> ----" marker line and
    ends at the next marker."""
    h = hashlib.sha256()
    for part in parts:
        f, section = (part, None) if isinstance(part, str) else part
        text = open(os.path.join(ROOT, f), encoding="utf-8").read()
        if section is not None:
            lines = text.splitlines(keepends=True)
            marks = [i for i, ln in enumerate(lines) if ln.startswith("// ---") and ln.rstrip().endswith("----")]
            start = next(i for i in marks if section in lines[i])
            end = next((i for i in marks if i > start), len(lines))
            text = "".join(lines[start:end])
        h.update(text.encode())
    return h.hexdigest()[:16]


_CS = "hierarchical_block_sparse_b200/csrc/"
_BMF = _CS + "blockmajor.cu"
_TILE = [(_BMF, "tile plumbing"), _CS + "tc.cuh", _CS + "pisa_internal.h"]
KERNEL_SOURCES = {
    "stage1": [_CS + "walk_tc.cu", _CS + "tc.cuh", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "stage1_per_query": [(_BMF, "stage 1"), _CS + "pisa_stage1.cuh", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "bsa_tc": [_CS + "bsa_tc.cu", _CS + "tc.cuh", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "leaf_scores": [(_BMF, "stage 2: leaf LSEs")] + _TILE,
    "topk": [(_BMF, "final Top-K"), _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "attn_tiles": [(_BMF, "attention tiles")] + _TILE,
    "forced_tiles": [(_BMF, "forced leaves, dense")] + _TILE,
    "backward_tiles": [(_BMF, "backward tiles")] + _TILE,
    "pool": [_CS + "pool.cu", _CS + "pisa_device.cuh"],
    "select": [_CS + "select.cu", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "attn": [_CS + "attn.cu", _CS + "pisa_attn.cuh", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
    "decode": [_CS + "decode.cu", _CS + "tc.cuh", _CS + "pisa_walk.cuh", _CS + "pisa_device.cuh"],
}


def measured_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from profiles/ncu_traffic.json, if the
    kernel's sources are unchanged since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(kernel)
    except Exception:
        return None
    if not d or d.get("workload") != workload or d.get("source_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ cpu baseline ----

# ------------------------------------------------------------ replicas ----

def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank runs its own seeded copy of the workload (weak scaling)."""
    return base_seed + rank


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time is the slowest rank's: all-reduce MAX of a per-rank time
    (any backend: `device` is cuda for NCCL, cpu for gloo)."""
    if dist is None:
        return ms
    import torch
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the max-rank time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def oracle_prefill_sample(w, Q, K, V, rows_per_head: int, rng_seed: int = 0):
    """Time the oracle (fp64, OpenMP) on: the full pyramid of every KV head and
    selection + attention for `rows_per_head` sampled query rows of every head.
    Returns (seconds_pyramid, seconds_rows, rows_per_head)."""
    from oracle import oracle
    N = Q.shape[2]
    G = w.Hq // w.Hkv
    rng = np.random.default_rng(rng_seed)
    rows = np.sort(rng.choice(N, size=min(rows_per_head, N), replace=False)).astype(np.int64)
    tt = __import__("torch").as_tensor(rows)
    Kf = [[oracle.to_f64(K[b, h]) for h in range(w.Hkv)] for b in range(w.B)]
    Vf = [[oracle.to_f64(V[b, h]) for h in range(w.Hkv)] for b in range(w.B)]
    Qf = [[oracle.to_f64(Q[b, h * G:(h + 1) * G][:, tt]).transpose(1, 0, 2).copy() for h in range(w.Hkv)]
          for b in range(w.B)]
    t0 = time.perf_counter()
    P = [[oracle.build_pyramid(Kf[b][h], w.C) for h in range(w.Hkv)] for b in range(w.B)]
    t1 = time.perf_counter()
    for b in range(w.B):
        for h in range(w.Hkv):
            idx, _ = oracle.select_rows(Qf[b][h], rows, Kf[b][h], P[b][h], C=w.C, K=w.K, causal=w.causal,
                                        forced_mask=w.forced_mask)
            for j in range(G):
                oracle.attn_rows(Qf[b][h][:, j], rows, Kf[b][h], Vf[b][h], idx, C=w.C, causal=w.causal)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, len(rows)


def oracle_tokens_per_s(w, N, t_pyr, t_rows, nrows):
    """Extrapolate a sample to the whole workload: pyramid once + N rows."""
    per_row = t_rows / nrows
    total = t_pyr + N * per_row
    return w.B * N / total, total


def size_oracle_sample(w, Q, K, V, target_s: float):
    t_pyr, t_rows, n = oracle_prefill_sample(w, Q, K, V, 256)
    per_row = t_rows / n
    budget = max(target_s - t_pyr, 0.5)
    return int(min(max(8, budget / max(per_row, 1e-6)), Q.shape[2]))


# ------------------------------------------------------- measured FMA peak ----

def measure_fma_peak(dev, stream, blocks_per_sm: int = 8, iters: int = 20000, reps: int = 5):
    """fp32 FMA throughput of this GPU, measured with pisa_fma_probe (scalar and
    packed fp32x2 chains, full occupancy), CUDA events on the launch stream,
    with the SM clock sampled during the timed launches."""
    import torch
    from hierarchical_block_sparse_b200 import pisa
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = sms * blocks_per_sm
    out = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    res = {}
    with ClockSampler(dev.index) as clk:
        for packed in (False, True):
            for _ in range(2):
                pisa.pisa_fma_probe(out, blocks, iters, packed)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                pisa.pisa_fma_probe(out, blocks, iters, packed)
            e1.record(stream)
            torch.cuda.synchronize()
            flop = blocks * 256.0 * iters * 64 * (2 if packed else 1) * reps
            res["packed_tflops" if packed else "scalar_tflops"] = flop / (e0.elapsed_time(e1) / 1e3) / 1e12
    res["tflops"] = max(res["scalar_tflops"], res["packed_tflops"])
    res["clocks"] = clk.summary()
    res["how"] = (f"pisa_fma_probe: {blocks} blocks x 256 threads, 8 independent chains of {4 * iters} FMAs each, "
                  f"scalar and packed fp32x2, {reps} launches after 2 warm-up, CUDA events")
    return res


def dominant_roofline(w, phase_ms, alg, pk, fma_peak, fma_note, tc_peak):
    """Roofline entry for the phase that takes the most time."""
    dom = max(phase_ms, key=phase_ms.get)
    t_dom = phase_ms[dom] / 1e3
    tc_note = "bf16 dense, sustained (MEASURED_PEAKS.json)"
    if dom == "attn_tiles":
        roof = {"kernel": "attn_tile_kernel", "bound": "tensor", "achieved": alg["attn_free_flops"] / t_dom / 1e12,
                "peak": tc_peak, "unit": "TFLOP/s", "algorithmic_per_launch": alg["attn_free_flops"],
                "peak_note": tc_note}
    elif dom == "forced_tiles":
        roof = {"kernel": "forced_tile_kernel", "bound": "tensor",
                "achieved": alg["attn_forced_flops"] / t_dom / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
                "algorithmic_per_launch": alg["attn_forced_flops"], "peak_note": tc_note}
    elif dom == "leaf_scores":
        roof = {"kernel": "leaf_score_kernel", "bound": "tensor", "achieved": alg["leaf_flops"] / t_dom / 1e12,
                "peak": tc_peak, "unit": "TFLOP/s", "algorithmic_per_launch": alg["leaf_flops"],
                "peak_note": tc_note}
    elif dom == "stage1" and walk_on_tensor_cores(w):
        roof = {"kernel": "stage 1: walk_tc_kernel (coarse levels, tensor cores) + stage1_kernel (fine levels, "
                          "one warp per query)",
                "bound": "alu", "achieved": alg["internal_flops"] / t_dom / 1e12,
                "peak": fma_peak, "unit": "TFLOP/s", "algorithmic_per_launch": alg["internal_flops"],
                "peak_note": fma_note + "; the fine levels, which take most of the phase, run on the CUDA cores; "
                                        "achieved counts the walk's own child dots over the whole phase"}
    elif dom == "stage1":
        roof = {"kernel": "stage1_kernel", "bound": "alu", "achieved": alg["internal_flops"] / t_dom / 1e12,
                "peak": fma_peak, "unit": "TFLOP/s", "algorithmic_per_launch": alg["internal_flops"],
                "peak_note": fma_note}
    else:
        b = alg["pool_bytes"] if dom == "pyramid" else alg["selection_bytes"]
        roof = {"kernel": dom, "bound": "hbm", "achieved": b / t_dom / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "algorithmic_per_launch": b}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(dom, w.name)
    roof["launch_ms"] = phase_ms[dom]
    return roof


def walk_on_tensor_cores(w) -> bool:
    """The block-major selection walks on the tensor cores while the level
    above the finest ranked one has at most 8192 nodes (N <= 2M at C = 64)."""
    M1 = -(-w.N // w.C)
    M3 = -(-(-(-M1 // 2)) // 2)
    return M1 <= 2 or M3 <= 8192


SELECTION_PHASES = ("pyramid", "stage1", "group_candidates", "leaf_scores", "topk")


def time_bsa(cfg, Qd, Kd, pyr, idx, stream, work=None, reps: int = 3):
    """Flat BSA selection (pyramid + Eq.1 over every eligible leaf), ms: on the
    tensor cores (pisa_bsa_select_ws) when a workspace is given, else the
    per-query CUDA-core scan (pisa_bsa_select)."""
    import torch
    from hierarchical_block_sparse_b200 import pisa
    bidx = torch.empty_like(idx)

    def run():
        pisa.pisa_build_pyramid(cfg, Kd, pyr)
        if work is None:
            pisa.pisa_bsa_select(cfg, Qd, pyr, bidx)
        else:
            pisa.pisa_bsa_select_ws(cfg, Qd, pyr, bidx, work)

    run()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for _ in range(reps):
        run()
    b1.record(stream)
    torch.cuda.synchronize()
    if work is not None and pisa.pisa_workspace_status(cfg, work) != 0:
        raise RuntimeError("a tensor-core BSA tile timed out")
    return b0.elapsed_time(b1) / reps


def prefill_config_line(w, dev, stream, steps, warmup, pk, fma_peak, fma_note, tc_peak, bsa=True):
    """One workload's prefill measured like the headline step (pisa_forward_ws,
    phase events on the launch stream, inputs larger than L2): ms per step,
    tokens/s, selection ms, the dominant kernel's roofline, HBM fractions and
    the flat BSA selection beside it."""
    import torch
    from hierarchical_block_sparse_b200 import pisa
    from hierarchical_block_sparse_b200.workloads import make_inputs
    Q, K, V, _ = make_inputs(w)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    del Q, K, V
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Qd.dtype)
    work = pisa.alloc_workspace(cfg, dev)
    nph = len(pisa.PHASES)
    for _ in range(warmup):
        pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, work)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(steps)]
    for e in evs:
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    for e in evs:
        pisa.pisa_forward_ws_events(cfg, Qd, Kd, Vd, pyr, idx, O, work, e)
    torch.cuda.synchronize()
    if pisa.pisa_workspace_status(cfg, work) != 0:
        raise RuntimeError(f"a tensor-core tile timed out ({w.name})")
    ms = evs[0][0].elapsed_time(evs[-1][nph]) / steps
    phase_ms = {name: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs])) for i, name in enumerate(pisa.PHASES)}
    sel = sum(phase_ms[k] for k in SELECTION_PHASES)
    alg = algorithmic(w, w.N)
    hbm = pk["hbm_gbs"] * 1e9
    out = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "C": w.C, "K": w.K,
           "steps": steps, "ms_per_step": ms, "tokens_per_s": w.B * w.N / (ms / 1e3),
           "selection_ms": sel, "attention_ms": ms - sel, "phase_ms": phase_ms,
           "hbm_roofline_frac": {"prefill": alg["prefill_bytes"] / (ms / 1e3) / hbm,
                                 "selection": alg["selection_bytes"] / (sel / 1e3) / hbm,
                                 "pyramid": alg["pool_bytes"] / (phase_ms["pyramid"] / 1e3) / hbm},
           "roofline": dominant_roofline(w, phase_ms, alg, pk, fma_peak, fma_note, tc_peak),
           "work": {"internal_tflop": alg["internal_flops"] / 1e12, "leaf_tflop": alg["leaf_flops"] / 1e12,
                    "attn_tflop": alg["attn_flops"] / 1e12}}
    if bsa:
        out["bsa_selection_ms"] = time_bsa(cfg, Qd, Kd, pyr, idx, stream, work)
        out["bsa_cuda_core_ms"] = time_bsa(cfg, Qd, Kd, pyr, idx, stream, reps=1)
        out["pisa_vs_bsa_selection_speedup"] = out["bsa_selection_ms"] / sel
    del Qd, Kd, Vd, pyr, idx, O, work
    torch.cuda.empty_cache()
    return out


PER_CONFIG = ("mha16_n16k", "needle_mha16_n64k", "gqa32x8_n128k")
SWEEP_N = (262144, 524288, 1048576)


def selection_sweep(w, dev, stream, ns=SWEEP_N, reps: int = 3):
    """PISA's selection against flat BSA's on the headline workload's shape at
    growing N (both from the keys: the pyramid, then the selection; PISA
    through pisa_select_ws, BSA on the tensor cores), to locate where the
    log-linear walk overtakes the quadratic contraction on this GPU. Inputs
    are i.i.d. N(0, 1) in bf16, drawn on the device (seeded) to keep the
    sweep's host time short."""
    import torch
    from hierarchical_block_sparse_b200 import pisa
    out = {}
    gen = torch.Generator(device=dev)
    for n in ns:
        gen.manual_seed(1000 + n)
        Qd = torch.randn((w.B, w.Hq, n, w.d), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        Kd = torch.randn((w.B, w.Hkv, n, w.d), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
        pyr = torch.empty((w.B, w.Hkv, pisa.pisa_pyramid_rows(cfg), w.d), dtype=torch.float32, device=dev)
        idx = torch.empty((w.B, w.Hkv, n, w.K), dtype=torch.int32, device=dev)
        work = pisa.alloc_workspace(cfg, dev)

        def run():
            pisa.pisa_build_pyramid(cfg, Kd, pyr)
            pisa.pisa_select_ws(cfg, Qd, Kd, pyr, idx, work)

        run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
        if pisa.pisa_workspace_status(cfg, work) != 0:
            raise RuntimeError(f"a tensor-core tile timed out (selection sweep, N = {n})")
        p_ms = e0.elapsed_time(e1) / reps
        b_ms = time_bsa(cfg, Qd, Kd, pyr, idx, stream, work, reps=reps)
        out[str(n)] = {"pisa_selection_ms": p_ms, "bsa_selection_ms": b_ms, "pisa_vs_bsa_selection_speedup": b_ms / p_ms}
        del Qd, Kd, pyr, idx, work
        torch.cuda.empty_cache()
    return out


# -------------------------------------------------------------------- main ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="pisa", choices=["pisa", "reference"])
    ap.add_argument("--workload", default="mha8_n256k")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-bsa", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip timing the PISA-1 / PISA-2 scores")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the attention backward")
    ap.add_argument("--no-per-query", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the 16K / 64K / 128K workloads")
    ap.add_argument("--no-sweep", action="store_true", help="skip the PISA vs BSA selection sweep over N")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--decode-batch", type=int, default=0, help="override the decode batch (profiling)")
    ap.add_argument("--decode-cache", type=int, default=0, help="override the cached keys per sequence")
    ap.add_argument("--decode-only", action="store_true", help="skip the prefill measurement (profiling)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override the workload's sequence length (smaller cases for counter captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: --warmup raised to 3", file=sys.stderr)
        args.warmup = 3

    import torch
    from hierarchical_block_sparse_b200 import pisa
    from hierarchical_block_sparse_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS[args.workload]
    if args.seq:
        w = w.replace(N=args.seq, name=f"{w.name}_seq{args.seq}")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    config = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "C": w.C, "K": w.K,
              "g": w.g, "causal": w.causal, "forced_mask": w.forced_mask,
              "l2": "inputs larger than L2 (Q, K, V, O exceed 126 MB)",
              "parallelism": f"replicas{world}" if world > 1 else "single"}
    metric = "prefill tokens/s"
    unit = "tokens/s"

    if args.impl == "reference":
        if rank != 0:
            return 0
        return reference_arm(args, w, config, metric, unit)

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    pisa.load()
    if args.decode_only:
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        print(json.dumps({"decode": bench_decode(w, dev, torch.cuda.current_stream(), batch=args.decode_batch,
                                                 cache=args.decode_cache), "config": config}))
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    Q, K, V, meta = make_inputs(w, seed=replica_seed(w.seed, rank))
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    cfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask)
    pyr, idx, O = pisa.alloc_outputs(cfg, dev, Qd.dtype)
    work = pisa.alloc_workspace(cfg, dev)
    stream = torch.cuda.current_stream()
    nph = len(pisa.PHASES)
    pool_launches = 2 if pisa.pisa_num_levels(cfg) >= 6 else 1
    # our kernels per step: pyramid, stage 1 (pyramid split + tile walk, or the
    # one-warp walk), 3 grouping kernels, leaf scores, Top-K, 3 grouping
    # kernels, forced tiles, attention tiles, output conversion
    launches_per_step = pool_launches + (2 if walk_on_tensor_cores(w) else 1) + 3 + 1 + 1 + 3 + 1 + 1 + 1

    def step(ev=None):
        if ev is None:
            pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, work)
        else:
            pisa.pisa_forward_ws_events(cfg, Qd, Kd, Vd, pyr, idx, O, work, ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pisa.pisa_workspace_status(cfg, work) != 0:
        raise RuntimeError("a tensor-core tile timed out during warm-up")
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(args.steps)]
    for e in evs:  # create the underlying events before the timed region
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for s_ in range(args.steps):
            step(evs[s_])
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = evs[0][0].elapsed_time(evs[-1][nph])
    phase_ms = {name: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs]))
                for i, name in enumerate(pisa.PHASES)}
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / args.steps
    tokens = w.B * w.N * world
    value = job_tokens_per_s(w.B * w.N, world, ms_per_step)

    alg = algorithmic(w, w.N)
    pk = peaks()
    clocks = clk.summary()
    tc_peak = pk["bf16_tflops_sustained"] or pk["bf16_tflops"]
    fma = measure_fma_peak(dev, stream)
    fma_derived = fp32_fma_peak_tflops(pk["sm_max_mhz"])
    fma_peak = fma["tflops"]
    fma_note = ("fp32 FMA measured on this GPU with pisa_fma_probe (max of scalar and packed chains); "
                f"derived 148 SMs x 128 lanes x 2 FLOP x max clock = {fma_derived:.1f} TFLOP/s")
    roof = dominant_roofline(w, phase_ms, alg, pk, fma_peak, fma_note, tc_peak)
    if roof["bound"] == "alu":
        roof["peak_source"] = "measured"

    sel_total = sum(phase_ms[k] for k in SELECTION_PHASES)
    hbm = pk["hbm_gbs"] * 1e9
    out = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded i.i.d. N(0,1))",
        "config": config,
        "path": "block-major tensor-core (pisa_forward_ws)",
        "selection_ms": sel_total, "attention_ms": ms_per_step - sel_total, "phase_ms": phase_ms,
        "hbm_roofline_frac": {"prefill": alg["prefill_bytes"] / (ms_per_step / 1e3) / hbm,
                              "selection": alg["selection_bytes"] / (sel_total / 1e3) / hbm,
                              "pyramid": alg["pool_bytes"] / (phase_ms["pyramid"] / 1e3) / hbm},
        "work": {"select_dots_per_query": alg["select_dots_per_query"],
                 "attended_keys_per_query": alg["attended_keys_per_query"],
                 "internal_tflop": alg["internal_flops"] / 1e12, "leaf_tflop": alg["leaf_flops"] / 1e12,
                 "attn_tflop": alg["attn_flops"] / 1e12},
        "roofline": roof,
        "peaks_source": pk["source"],
        "fp32_fma_peak": {"measured_tflops": fma_peak, "scalar_tflops": fma["scalar_tflops"],
                          "packed_tflops": fma["packed_tflops"], "derived_tflops": fma_derived,
                          "clocks": fma["clocks"], "how": fma["how"]},
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    if pisa.pisa_workspace_status(cfg, work) != 0:
        raise RuntimeError("a tensor-core tile timed out in the timed region")

    # the per-query CUDA-core path (pisa_forward), for comparison
    if not args.no_per_query:
        pisa.pisa_forward(cfg, Qd, Kd, Vd, pyr, idx, O)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pisa.pisa_forward(cfg, Qd, Kd, Vd, pyr, idx, O)
        e1.record(stream)
        torch.cuda.synchronize()
        out["per_query_path_ms_per_step"] = e0.elapsed_time(e1)

    # ---- end to end through the C ABI with host buffers: pinned host -> device -> host ----
    # pisa_forward_host copies the step's Q, K, V in, runs the step and copies
    # idx and O out, all on one stream. Two sets of device buffers on two
    # streams take alternate steps, so one step's copies overlap the other's
    # kernels; every step's copies are inside the timed region.
    Qh, Kh, Vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    slots = []
    for i in range(2):
        if i == 0:
            sQ, sK, sV, spyr, sidx, sO, swork = Qd, Kd, Vd, pyr, idx, O, work
        else:
            sQ, sK, sV = torch.empty_like(Qd), torch.empty_like(Kd), torch.empty_like(Vd)
            spyr, sidx, sO = torch.empty_like(pyr), torch.empty_like(idx), torch.empty_like(O)
            swork = pisa.alloc_workspace(cfg, dev)
        slots.append({"dev": (sQ, sK, sV, spyr, sidx, sO, swork), "stream": torch.cuda.Stream(dev),
                      "Oh": torch.empty(O.shape, dtype=O.dtype, pin_memory=True),
                      "Ih": torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)})

    def e2e_step(i):
        sl = slots[i % 2]
        sQ, sK, sV, spyr, sidx, sO, swork = sl["dev"]
        with torch.cuda.stream(sl["stream"]):
            pisa.pisa_forward_host(cfg, Qh, Kh, Vh, sl["Ih"], sl["Oh"], sQ, sK, sV, spyr, sidx, sO, swork)

    def e2e_run(n):
        start = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for sl in slots:
            sl["stream"].wait_event(start)
        for i in range(n):
            e2e_step(i)
        for sl in slots:
            stream.wait_stream(sl["stream"])
        end = torch.cuda.Event(enable_timing=True)
        end.record(stream)
        return start, end

    e2e_run(2)
    torch.cuda.synchronize()
    n_e2e = max(4, min(args.steps, 6))
    e0, e1 = e2e_run(n_e2e)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    out["e2e"] = {"value": job_tokens_per_s(w.B * w.N, world, e2e_ms), "unit": unit,
                  "h2d_bytes_per_step": int(Qh.nbytes + Kh.nbytes + Vh.nbytes),
                  "d2h_bytes_per_step": int(O.nbytes + idx.nbytes), "ms_per_step": e2e_ms,
                  "call": "pisa_forward_host", "pipelining": "2 buffer sets on 2 streams, alternate steps"}
    del Qh, Kh, Vh, slots

    # ---- flat BSA selection, the quadratic comparison ----
    if not args.no_bsa:
        out["bsa_selection_ms"] = time_bsa(cfg, Qd, Kd, pyr, idx, stream, work)
        out["bsa_kernel"] = "tensor-core flat Eq.(1) contraction with a streaming Top-K (bsa_tc_kernel)"
        out["bsa_cuda_core_ms"] = time_bsa(cfg, Qd, Kd, pyr, idx, stream, reps=1)
        out["pisa_vs_bsa_selection_speedup"] = out["bsa_selection_ms"] / sel_total

    # ---- the same step ranking by the PISA-1 / PISA-2 scores (Eq.8-9 ablations) ----
    if not args.no_variants:
        vout = {}
        for vname, v in (("pisa1_mean", pisa.PISA_SCORE_MEAN), ("pisa2_mean_var", pisa.PISA_SCORE_MEAN_VAR)):
            vcfg = pisa.cfg_for(Qd, Kd, C=w.C, K_=w.K, causal=w.causal, forced_mask=w.forced_mask, score_variant=v)
            vwork = pisa.alloc_workspace(vcfg, dev)
            for _ in range(2):
                pisa.pisa_forward_ws(vcfg, Qd, Kd, Vd, pyr, idx, O, vwork)
            torch.cuda.synchronize()
            vev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(3)]
            for e in vev:
                for x in e:
                    x.record(stream)
            torch.cuda.synchronize()
            for e in vev:
                pisa.pisa_forward_ws_events(vcfg, Qd, Kd, Vd, pyr, idx, O, vwork, e)
            torch.cuda.synchronize()
            vms = max_over_ranks(vev[0][0].elapsed_time(vev[-1][nph]) / len(vev), dist, dev)
            vout[vname] = {"ms_per_step": vms, "tokens_per_s": job_tokens_per_s(w.B * w.N, world, vms),
                           "phase_ms": {name: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in vev]))
                                        for i, name in enumerate(pisa.PHASES)}}
            del vwork
        out["score_variants"] = vout

    # ---- backward of the attention with the selection fixed (dQ, dK, dV) ----
    # Block-major on the tensor cores (pisa_sparse_attn_backward_ws, phases
    # timed with events), and the per-query CUDA-core call for comparison.
    if not args.no_backward:
        gen = torch.Generator(device=dev).manual_seed(w.seed + 17)
        dOd = torch.randn(Qd.shape, generator=gen, device=dev, dtype=torch.float32).to(Qd.dtype)
        dQ = torch.empty(Qd.shape, dtype=torch.float32, device=dev)
        dK = torch.empty(Kd.shape, dtype=torch.float32, device=dev)
        dV = torch.empty(Vd.shape, dtype=torch.float32, device=dev)
        # per attended (query head, key): 4d FLOP to recompute the softmax and
        # the output, 10d for the logits again, dP, dQ, dK and dV
        bflops = alg["attn_flops"] * 14.0 / 4.0
        bws = pisa.alloc_backward_workspace(cfg, dev)
        nbp = len(pisa.BWD_PHASES)
        for _ in range(2):
            pisa.pisa_sparse_attn_backward_ws(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV, bws)
        torch.cuda.synchronize()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(nbp + 1)] for _ in range(3)]
        for e in bev:
            for x in e:
                x.record(stream)
        torch.cuda.synchronize()
        for e in bev:
            pisa.pisa_sparse_attn_backward_ws_events(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV, bws, e)
        torch.cuda.synchronize()
        bms = max_over_ranks(bev[0][0].elapsed_time(bev[-1][nbp]) / len(bev), dist, dev)
        # from the state the forward left in its workspace (training steps that keep it)
        pisa.pisa_forward_ws(cfg, Qd, Kd, Vd, pyr, idx, O, bws)
        pisa.pisa_sparse_attn_backward_saved_ws(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV, bws)
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(3):
            pisa.pisa_sparse_attn_backward_saved_ws(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV, bws)
        g1.record(stream)
        torch.cuda.synchronize()
        saved_ms = max_over_ranks(g0.elapsed_time(g1) / 3, dist, dev)
        del bws
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        pisa.pisa_sparse_attn_backward(cfg, Qd, Kd, Vd, idx, dOd, dQ, dK, dV)
        g1.record(stream)
        torch.cuda.synchronize()
        pq_ms = max_over_ranks(g0.elapsed_time(g1), dist, dev)
        # Training keeps the forward's workspace: the backward then starts from
        # the normaliser and fp32 output the forward left there (the headline
        # figure); the standalone call recomputes them from Q, K, V, dO and idx.
        sflops = alg["attn_flops"] * 10.0 / 4.0  # logits, dP, dQ, dK, dV: 10d per (query head, key)
        out["backward"] = {"ms": saved_ms, "tokens_per_s": job_tokens_per_s(w.B * w.N, world, saved_ms),
                           "call": "pisa_sparse_attn_backward_saved_ws (after pisa_forward_ws, whose workspace "
                                   "keeps the normaliser and the fp32 output)",
                           "kernel": "bwd_tile_kernel (key-major tcgen05 tiles; dK, dV in TMEM per leaf; dQ rows "
                                     "by bulk reductions)",
                           "algorithmic_tflop": sflops / 1e12, "achieved_tflops": sflops / (saved_ms / 1e3) / 1e12,
                           "bf16_tensor_peak_tflops": tc_peak,
                           "frac": sflops / (saved_ms / 1e3) / 1e12 / tc_peak,
                           "tiles_dram_bytes": measured_traffic("backward_tiles", w.name),
                           "standalone_ms": bms,
                           "standalone_call": "pisa_sparse_attn_backward_ws (statistics recomputed: bwd_stats_kernel, "
                                              "per-leaf LSE and P-weighted dP)",
                           "standalone_phase_ms": {name: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in bev]))
                                                   for i, name in enumerate(pisa.BWD_PHASES)},
                           "standalone_algorithmic_tflop": bflops / 1e12,
                           "standalone_frac": bflops / (bms / 1e3) / 1e12 / tc_peak,
                           "per_query_cuda_core_ms": pq_ms,
                           "per_query_cuda_core_frac_of_fp32_fma": bflops / (pq_ms / 1e3) / 1e12 / fma_peak}
        del dOd, dQ, dK, dV

    # ---- decode: 64 sequences, one new token each, against 256K-key caches ----
    if not args.no_decode and w.decode_batch:
        out["decode"] = bench_decode(w, dev, stream, batch=args.decode_batch, cache=args.decode_cache)

    del Qd, Kd, Vd, pyr, idx, O, work
    torch.cuda.empty_cache()

    # ---- the other prefill workloads (16K, 64K planted retrieval, 128K GQA 32/8) ----
    if not args.no_per_config:
        per = {}
        for name in PER_CONFIG:
            wc = WORKLOADS[name]
            line = prefill_config_line(wc, dev, stream, min(args.steps, 5), 3, pk, fma_peak, fma_note, tc_peak,
                                       bsa=not args.no_bsa)
            line["ms_per_step"] = max_over_ranks(line["ms_per_step"], dist, dev)
            line["tokens_per_s"] = job_tokens_per_s(wc.B * wc.N, world, line["ms_per_step"])
            per[name] = line
        out["per_config"] = per
        out["selection_ms_by_n"] = {str(v["N"]): v["selection_ms"] for v in per.values()}
        out["selection_ms_by_n"][str(w.N)] = sel_total

    # ---- PISA vs flat BSA selection beyond the headline N (the crossover) ----
    if not args.no_bsa and not args.no_sweep and world == 1 and w.name == "mha8_n256k":
        out["selection_sweep"] = {"workload": "mha8 shape (B 1, 8 heads, d 128, C 64, K 16), N varied",
                                  "by_n": selection_sweep(w, dev, stream)}

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = size_oracle_sample(w, Q, K, V, args.cpu_seconds)
        t_pyr, t_rows, nr = oracle_prefill_sample(w, Q, K, V, n, rng_seed=1)
        from oracle import oracle
        v, total = oracle_tokens_per_s(w, w.N, t_pyr, t_rows, nr)
        out["cpu_baseline"] = {"value": v, "unit": unit, "cores": oracle.threads(), "kind": "oracle",
                               "sample": f"full fp64 pyramid of all {w.B * w.Hkv} KV heads ({t_pyr:.2f} s) + "
                                         f"selection and attention for {nr} random query rows of every head "
                                         f"({t_rows:.2f} s), extrapolated to all {w.N} rows"}
    if rank == 0:
        print(json.dumps(out))
    return 0


def bench_decode(w, dev, stream, steps: int = 8, batch: int = 0, cache: int = 0):
    """Decode: every step appends one token per sequence and selects + attends
    for it (pisa_decode_step, one launch). Also times the same step as the two
    separate calls (pisa_pyramid_append, then pisa_decode)."""
    import torch
    from hierarchical_block_sparse_b200 import pisa
    from hierarchical_block_sparse_b200.workloads import decode_cache, decode_step_inputs
    if batch:
        w = w.replace(decode_batch=batch)
    prefix = cache or w.N
    cap = prefix + 64
    B = w.decode_batch
    Kc, Vc, _, _ = decode_cache(w, cap, prefix, dev)
    cfg = pisa.make_cfg(B=B, Hq=w.Hq, Hkv=w.Hkv, N=cap, d=w.d, C=w.C, K=w.K, causal=True,
                        forced_mask=w.forced_mask, dtype=Kc.dtype)
    pyr = torch.empty((B, w.Hkv, pisa.pisa_pyramid_rows(cfg), w.d), dtype=torch.float32, device=dev)
    pos = torch.full((B,), prefix, dtype=torch.int32, device=dev)
    pisa.pisa_build_pyramid_prefix(cfg, Kc, pos, pyr)
    ins = [tuple(x.to(dev) for x in decode_step_inputs(w, s)) for s in range(2 * steps + 3)]
    idx = torch.empty((B, w.Hkv, w.K), dtype=torch.int32, device=dev)
    o = torch.empty((B, w.Hq, w.d), dtype=Kc.dtype, device=dev)
    for s in range(3):
        q, k, v = ins[s]
        pisa.pisa_decode_step(cfg, q, k, v, Kc, Vc, pyr, pos, idx, o)
        pos += 1
    torch.cuda.synchronize()
    evf = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    # a short device-side wait first, so the host enqueues the steps while the
    # stream is busy and the events bracket the kernels, not the launch latency
    torch.cuda._sleep(10_000_000)
    for s in range(steps):
        q, k, v = ins[3 + s]
        evf[s][0].record(stream)
        pisa.pisa_decode_step(cfg, q, k, v, Kc, Vc, pyr, pos, idx, o)
        evf[s][1].record(stream)
        pos += 1
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda._sleep(10_000_000)
    for s in range(steps):
        q, k, v = ins[3 + steps + s]
        ev[s][0].record(stream)
        pisa.pisa_pyramid_append(cfg, Kc, Vc, pyr, k, v, pos)
        ev[s][1].record(stream)
        pisa.pisa_decode(cfg, q, Kc, Vc, pyr, pos, idx, o)
        ev[s][2].record(stream)
        pos += 1
    torch.cuda.synchronize()
    fused = float(np.mean([e[0].elapsed_time(e[1]) for e in evf])) * 1e3
    app = float(np.mean([e[0].elapsed_time(e[1]) for e in ev])) * 1e3
    dec = float(np.mean([e[1].elapsed_time(e[2]) for e in ev])) * 1e3
    # compulsory bytes per step (per sequence and KV head): the scored levels'
    # child summaries (fp32), the raw keys of every level-1 candidate (scored or
    # forced), the attended values, the new q/k/v rows and the updated leaf
    # and ancestor summaries. With one head per group and leaves of at most 64
    # keys the kernel keeps the scoring pass's logits and streams only the
    # attended values; otherwise it reads the attended keys a second time
    # (gathered bytes).
    internal, leafkeys, attended = walk_counts(prefix + 8, w.C, w.K, w.forced_mask)
    tlast = prefix + 4
    G = w.Hq // w.Hkv
    e = 2 if w.dtype == "bf16" else 4
    L = 1
    m = -(-cap // w.C)
    while m > 1:
        m = -(-m // 2)
        L += 1
    per_unit = internal[tlast] * w.d * 4 + (leafkeys[tlast] + walk_counts.forced_keys[tlast]) * w.d * e + \
        attended[tlast] * w.d * e + (G + 2) * w.d * e + L * w.d * 4
    step_bytes = per_unit * B * w.Hkv
    rereads_keys = not (G == 1 and w.C <= 64)
    gathered = step_bytes + (attended[tlast] * w.d * e * B * w.Hkv if rereads_keys else 0)
    pk = peaks()
    del Kc, Vc, pyr
    return {"batch": B, "cache_keys": prefix, "call": "pisa_decode_step", "us_per_step": fused,
            "tokens_per_s": B / (fused / 1e6), "compulsory_bytes_per_step": int(step_bytes),
            "gathered_bytes_per_step": int(gathered),
            "hbm_roofline_frac": step_bytes / (fused / 1e6) / (pk["hbm_gbs"] * 1e9),
            "split_calls_us": {"pisa_pyramid_append": app, "pisa_decode": dec, "total": app + dec}}


def reference_arm(args, w, config, metric, unit):
    """The oracle (fp64 CPU, the reference computation of this method), timed on
    the host cores on a bounded sample of the same workload per step."""
    from hierarchical_block_sparse_b200.workloads import make_inputs
    from oracle import oracle
    Q, K, V, _ = make_inputs(w)
    n = size_oracle_sample(w, Q, K, V, 4.0)
    for _ in range(args.warmup):
        oracle_prefill_sample(w, Q, K, V, max(8, n // 8), rng_seed=99)
    vals, secs = [], []
    for s in range(args.steps):
        t_pyr, t_rows, nr = oracle_prefill_sample(w, Q, K, V, n, rng_seed=s)
        v, _ = oracle_tokens_per_s(w, w.N, t_pyr, t_rows, nr)
        vals.append(v)
        secs.append(t_pyr + t_rows)
    value = float(np.mean(vals))
    sample = (f"per step: full fp64 pyramid of all {w.B * w.Hkv} KV heads + selection and attention for {n} "
              f"random query rows of every head, extrapolated to all {w.N} rows")
    out = {"metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": float(np.mean(secs)) * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded i.i.d. N(0,1))",
           "config": config, "impl": "reference",
           "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
