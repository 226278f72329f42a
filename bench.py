"""Benchmark of the TriAttention KV scoring-and-pruning pass on B200.

One step = one tri_prune call over the whole synthetic cache (every unit scored,
z-scored, selected and compacted in place). The prune overwrites slots [0, B) of each
unit, so between steps the overwritten rows (and lens) are restored from a pristine
device copy and L2 is flushed; that restore runs outside the CUDA-event-timed region,
which brackets exactly the prune launch on its stream.

Default workload: one-shot compression of a Qwen3-8B-shaped cache (36 layers x 8 KV
heads x GQA 4, head_dim 128, batch 4, 32768 -> 3072 keys per unit, ~19 GB of K/V).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu]

Prints ONE JSON line (rank 0).

    python bench.py --path calibrate [--steps K] [--warmup W]

measures instead the calibration-statistics estimator (tri_calibrate_estimate) on the pages'
calibration batch (about 10K tokens through a Qwen3-8B-shaped model: 36 layers, 32 query
heads, head_dim 128; 3 GB of bf16 pre-RoPE queries), one GPU.

    python bench.py --path decode [--steps K] [--warmup W]

measures the decode loop's cache maintenance in steady state on the periodic Qwen3-8B workload
(36 layers x 8 KV heads, batch 8, budget 3072, paged with 64-token pages): one cycle = 128
tri_append calls (one token for every sequence each) and one tri_prune (3200 -> 3072 keys per
unit), with the pages freed by the prune returned to a free list and handed out again.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "qwen3_8b_oneshot_32k_to_3072"
METRIC = "KV tokens scored+pruned/s (Qwen3-8B shape); achieved HBM GB/s as % of B200 peak"
UNIT = "keys/s"
PEAK_FALLBACK_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 datasheet HBM3e bandwidth (the HGX figure is 7.7 TB/s)
KERNEL_SOURCES = ["rope_aware_key_tri_b200/csrc/tri_kernel.cuh", "rope_aware_key_tri_b200/csrc/tri_api.cu"]
KERNEL_NAME = "tri_fused_kernel"


# ---------------------------------------------------------------------------------------
# host-side helpers (also exercised by the CPU multi-process tests)
# ---------------------------------------------------------------------------------------

def shard_sequences(global_batch: int, rank: int, world: int):
    """Contiguous block of sequences owned by ``rank`` (weak scaling: equal blocks)."""
    per = global_batch // world
    return list(range(rank * per, (rank + 1) * per))


def reduce_max(value: float, dist_mod=None) -> float:
    """Max over ranks of a host float (plumbing only: the data path has no collective)."""
    if dist_mod is None or not dist_mod.is_initialized() or dist_mod.get_world_size() == 1:
        return value
    import torch
    dev = "cuda" if dist_mod.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def algorithmic_bytes(lens, n_layers, n_kv, head_dim, budget) -> int:
    """Roofline bytes of one prune: read every key row, read+write every kept K and V row,
    read+write every kept position."""
    row = head_dim * 2
    tot = 0
    for n in lens:
        m = min(n, budget)
        tot += n * row + m * 4 * row + m * 8
    return tot * n_layers * n_kv


def _code_only(src: str) -> str:
    """C/C++/CUDA source without comments and whitespace runs (string literals kept), so that the
    hash below follows the code and not its comments."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"' or c == "'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the prune kernel's code (device code and its host-side launch planning)."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", f"{KERNEL_NAME}_{workload}.md")
    if not os.path.exists(path):
        return None
    src = None
    val = None
    for line in open(path):
        line = line.strip().lstrip("-* ")
        if line.startswith("source_sha256:"):
            src = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch:"):
            try:
                val = float(line.split(":", 1)[1].strip().split()[0])
            except ValueError:
                val = None
    if src != kernel_source_hash():
        return None
    return val


def roofline_hbm(algorithmic_bytes: float, ms: float, traffic=None) -> dict:
    """HBM roofline block: achieved algorithmic GB/s against the measured copy peak (the
    fraction the bandwidth targets refer to) and, for context, against the datasheet figure."""
    peak, kind = measured_peak()
    achieved = algorithmic_bytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic, "algorithmic_bytes": algorithmic_bytes, "peak_kind": f"{kind} (burst copy)",
            "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return PEAK_FALLBACK_GBS, "fallback"


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_spec(args):
    import tri_synth as ts
    spec = ts.WORKLOADS[args.workload]
    if args.layers:
        spec = ts.replace(spec, n_layers=args.layers)
    return spec


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def run_ours(args, rank, world, dist_mod):
    import torch

    import tri_synth as ts
    from rope_aware_key_tri_b200 import tri

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    spec = workload_spec(args)
    B = spec.budget
    cache = ts.make_cache(spec, seed=1000 + rank, device=dev)
    torch.cuda.synchronize()
    ctx = tri.TriContext(local)
    ctx.calibrate_load(spec.n_layers, spec.n_kv_heads, spec.group, spec.head_dim, spec.rope_base, spec.layout,
                       cache.q_mean, cache.q_norm_mean, cache.R, cache.offsets)
    if args.cluster_size or args.buffers:
        ctx.set_tuning(args.cluster_size, args.buffers)
    if args.combine != "mean":
        ctx.set_offset_combine(args.combine)
    if args.engine != "auto":
        ctx.set_score_engine(args.engine)
    tensor_engine = args.combine == "max" or args.engine == "tensor" or (args.engine == "auto" and spec.group >= 8)
    lens_host = cache.lens_host.tolist()
    lens0 = cache.lens.clone()
    paged = cache.paged

    # pristine copy of everything a prune can overwrite: slots [0, B) of every unit
    if not paged:
        Mmax = min(B, cache.cap)
        saveK = cache.K[:, :, :, :Mmax].clone()
        saveV = cache.V[:, :, :, :Mmax].clone()
        saveP = cache.pos[:, :, :, :Mmax].clone()

        def restore():
            cache.K[:, :, :, :Mmax].copy_(saveK)
            cache.V[:, :, :, :Mmax].copy_(saveV)
            cache.pos[:, :, :, :Mmax].copy_(saveP)
            cache.lens.copy_(lens0)
    else:
        ps = spec.page_size
        bt = cache.block_table_host
        pages = sorted({int(bt[b, j]) for b in range(spec.batch) for j in range((min(lens_host[b], B) + ps - 1) // ps)})
        pidx = torch.as_tensor(pages, device=dev, dtype=torch.long)
        saveK, saveV, saveP = cache.K[:, pidx].clone(), cache.V[:, pidx].clone(), cache.pos[:, pidx].clone()

        def restore():
            cache.K[:, pidx] = saveK
            cache.V[:, pidx] = saveV
            cache.pos[:, pidx] = saveP
            cache.lens.copy_(lens0)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one_prune():
        ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, B, block_table=cache.block_table,
                  stream=stream)

    for _ in range(args.warmup):
        restore()
        flush.zero_()
        one_prune()
    st, code, unit = ctx.get_error(stream)
    if st != tri.TRI_OK:
        raise RuntimeError(f"device reported a problem during warm-up: {st} {code} {unit}")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist_mod is not None and dist_mod.is_initialized():
        dist_mod.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            restore()
            flush.zero_()
            starts[i].record(stream)
            one_prune()
            ends[i].record(stream)
        torch.cuda.synchronize()
        wall1 = time.perf_counter()
    if dist_mod is not None and dist_mod.is_initialized():
        dist_mod.barrier()
    torch.cuda.synchronize()
    st, code, unit = ctx.get_error(stream)
    if st != tri.TRI_OK:
        raise RuntimeError(f"device reported a problem: {st} {code} {unit}")
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    mean_ms = sum(ms) / len(ms)
    mean_ms_max = reduce_max(mean_ms, dist_mod)
    keys_rank = sum(lens_host) * spec.n_layers * spec.n_kv_heads
    keys_total = keys_rank * world
    value = keys_total / (mean_ms_max / 1e3)
    # max mode: prefix + phase kernels, then per chunk of layers (scores under 1 GiB) the
    # coefficient images, the tensor-core scoring and the fused select/compaction (+ a memset)
    per_layer_scores = spec.batch * spec.n_kv_heads * cache.cap * spec.group * 4
    n_chunks = -(-spec.n_layers // max(1, min(spec.n_layers, (1 << 30) // per_layer_scores)))
    abytes = algorithmic_bytes(lens_host, spec.n_layers, spec.n_kv_heads, spec.head_dim, B)
    result = {
        "ms_per_step": mean_ms_max,
        "value": value,
        "ms_steps": {"min": min(ms), "median": statistics.median(ms), "max": max(ms)},
        "wall_ms_per_step_incl_restore": (wall1 - wall0) * 1e3 / args.steps,
        "roofline": roofline_hbm(abytes, mean_ms, None if tensor_engine else ncu_traffic(args.workload)),
        "clocks": clk.summary(),
        # fused engine: the validation kernel and the fused kernel; tensor-core engine (and the
        # max mode): validation, prefix and phase kernels, then per chunk of layers the
        # coefficient images, the tensor-core scoring and the fused select/compaction
        "gpu_launches": args.steps * (3 + 3 * n_chunks if tensor_engine else 2),
        "engine": "tensor cores + fused select" if tensor_engine else "fused (CUDA cores)",
        "keys_per_rank": keys_rank,
        "lens": lens_host,
    }

    # ---- end to end through the public API with host buffers ----------------------------
    if not args.no_e2e and world == 1:
        result["e2e"] = run_e2e(args, cache, ctx, spec, B, restore, stream, keys_rank)
    ctx.close()
    restore()  # hand back the unpruned cache (the CPU baseline samples it)
    torch.cuda.synchronize()
    return result, cache, spec


def run_e2e(args, cache, ctx, spec, B, restore, stream, keys_rank):
    """H2D of the step's inputs from pinned host memory, tri_prune, D2H of the kept rows
    and lengths, all inside CUDA events on the launching stream."""
    import torch
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    restore()
    torch.cuda.synchronize()
    need = 2 * cache.K.numel() * 2 + cache.pos.numel() * 4
    out_bytes_est = 2 * cache.K.numel() * 2 * min(1.0, B / max(1, cache.cap)) + cache.pos.numel() * 4
    if avail < 2.5 * (need + out_bytes_est):
        return {"value": None, "unit": UNIT, "skipped": f"host memory {avail / 1e9:.1f} GB too small"}
    hK = torch.empty(cache.K.shape, dtype=cache.K.dtype, pin_memory=True)
    hV = torch.empty(cache.V.shape, dtype=cache.V.dtype, pin_memory=True)
    hP = torch.empty(cache.pos.shape, dtype=cache.pos.dtype, pin_memory=True)
    hL = torch.empty(cache.lens.shape, dtype=torch.int32, pin_memory=True)
    hT = torch.empty(cache.t.shape, dtype=torch.int32, pin_memory=True)
    hK.copy_(cache.K); hV.copy_(cache.V); hP.copy_(cache.pos); hL.copy_(cache.lens); hT.copy_(cache.t)
    paged = cache.paged
    if not paged:
        Mmax = min(B, cache.cap)
        oK = torch.empty(cache.K[:, :, :, :Mmax].shape, dtype=cache.K.dtype, pin_memory=True)
        oV = torch.empty_like(oK, pin_memory=True)
        oP = torch.empty(cache.pos[:, :, :, :Mmax].shape, dtype=torch.int32, pin_memory=True)
    else:
        oK = torch.empty(cache.K.shape, dtype=cache.K.dtype, pin_memory=True)
        oV = torch.empty_like(oK, pin_memory=True)
        oP = torch.empty(cache.pos.shape, dtype=torch.int32, pin_memory=True)
    oL = torch.empty(cache.lens.shape, dtype=torch.int32, pin_memory=True)
    h2d = hK.numel() * 2 + hV.numel() * 2 + hP.numel() * 4 + hL.numel() * 4 + hT.numel() * 4
    d2h = oK.numel() * 2 + oV.numel() * 2 + oP.numel() * 4 + oL.numel() * 4
    n = max(1, args.e2e_steps)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n + 1)]
    for i in range(n + 1):  # first one is a warm-up
        torch.cuda.synchronize()
        ev[i][0].record(stream)
        cache.K.copy_(hK, non_blocking=True); cache.V.copy_(hV, non_blocking=True)
        cache.pos.copy_(hP, non_blocking=True); cache.lens.copy_(hL, non_blocking=True)
        cache.t.copy_(hT, non_blocking=True)
        ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, B, block_table=cache.block_table, stream=stream)
        if not paged:
            oK.copy_(cache.K[:, :, :, :Mmax], non_blocking=True)
            oV.copy_(cache.V[:, :, :, :Mmax], non_blocking=True)
            oP.copy_(cache.pos[:, :, :, :Mmax], non_blocking=True)
        else:
            oK.copy_(cache.K, non_blocking=True); oV.copy_(cache.V, non_blocking=True)
            oP.copy_(cache.pos, non_blocking=True)
        oL.copy_(cache.lens, non_blocking=True)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev[1:]]
    mean = sum(ms) / len(ms)
    del hK, hV, hP, oK, oV, oP
    return {"value": keys_rank / (mean / 1e3), "unit": UNIT, "ms_per_step": mean,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n}


# ---------------------------------------------------------------------------------------
# the oracle, timed on the host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------------------

def oracle_sample(cache, spec, n_units, trunc=None):
    """Host arrays for n_units evenly spread units (optionally their first ``trunc`` keys)."""
    import numpy as np
    U = cache.n_units
    ids = sorted(set(int(round(x)) for x in np.linspace(0, U - 1, n_units)))
    rows = [cache.unit_rows(u) for u in ids]
    n_keys = [len(r[2]) if trunc is None else min(trunc, len(r[2])) for r in rows]
    S = max(n_keys)
    d = spec.head_dim
    Kb = np.zeros((len(ids), S, d), np.uint16)
    Pb = np.zeros((len(ids), S), np.int32)
    for i, (r, n) in enumerate(zip(rows, n_keys)):
        Kb[i, :n] = r[0][:n]
        Pb[i, :n] = r[2][:n]
    qm = np.stack([cache.unit_stats(u)[0] for u in ids])
    qn = np.stack([cache.unit_stats(u)[1] for u in ids])
    RR = np.stack([cache.unit_stats(u)[2] for u in ids])
    tt = np.array([int(cache.t_host[cache.unit_index(u)[1]]) for u in ids], np.int64)
    return ids, Kb, Pb, np.array(n_keys, np.int32), tt, qm, qn, RR


def time_oracle(cache, spec, budget_s=10.0, cores=None, min_steps=1, combine="mean"):
    """Run the oracle on a bounded sample; returns (keys/s, cores, description)."""
    import numpy as np

    import oracle
    cores = cores or os.cpu_count() or 1
    # calibrate on one truncated unit
    ids, Kb, Pb, nk, tt, qm, qn, RR = oracle_sample(cache, spec, 1, trunc=1024)
    t0 = time.perf_counter()
    oracle.prune_batch(Kb, Pb, nk, tt, qm, qn, RR, cache.offsets, spec.rope_base,
                       max(1, spec.budget * 1024 // max(1, int(cache.lens_host.max()))), spec.layout, n_threads=1,
                       combine=combine)
    per_key = (time.perf_counter() - t0) / 1024.0
    N = int(cache.lens_host.max())
    unit_s = per_key * N
    n_units = max(1, int(budget_s * cores / max(unit_s, 1e-9)))
    trunc = None
    if n_units < cores:
        # a full unit per core would not fit the budget: take the first keys of each unit
        n_units = cores
        trunc = max(256, int(budget_s / per_key))
    n_units = min(n_units, cache.n_units)
    ids, Kb, Pb, nk, tt, qm, qn, RR = oracle_sample(cache, spec, n_units, trunc=trunc)
    Bs = spec.budget if trunc is None else max(1, spec.budget * trunc // N)
    t0 = time.perf_counter()
    oracle.prune_batch(Kb, Pb, nk, tt, qm, qn, RR, cache.offsets, spec.rope_base, Bs, spec.layout,
                       n_threads=cores, combine=combine)
    el = time.perf_counter() - t0
    keys = int(nk.sum())
    what = f"{len(ids)} of {cache.n_units} units" + (
        f", first {trunc} keys of each (budget scaled to {Bs})" if trunc else " in full") + \
        f"; {keys} keys in {el:.1f} s"
    return keys / el, cores, what


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, as it stands, on the host cores."""
    import torch

    import tri_synth as ts
    spec = workload_spec(args)
    # only the host copy of a bounded sample is needed: draw the cache on the GPU when one
    # is present (the full workload is ~19 GB), else draw it on the CPU
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    cache = ts.make_cache(spec, seed=1000, device=dev)
    per_step_budget = max(0.2, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    cores = os.cpu_count() or 1
    vals = []
    desc = None
    for i in range(args.warmup + args.steps):
        v, cores, desc = time_oracle(cache, spec, budget_s=per_step_budget, cores=cores, combine=args.combine)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "layers": spec.n_layers, "kv_heads": spec.n_kv_heads,
                   "group": spec.group, "head_dim": spec.head_dim, "batch": spec.batch,
                   "budget": spec.budget, "offsets_combine": args.combine},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------------------

CAL_METRIC = "calibration query rows reduced/s (Qwen3-8B shape: 36 layers x 32 heads x 128 dims per token)"
CAL_SHAPE = (36, 10240, 32, 128)  # layers, tokens, query heads, head_dim


def run_calibrate(args):
    """Time tri_calibrate_estimate: CUDA events around the call (its two launches) on the
    stream; a 256 MiB buffer is written between steps (3 GB of input exceeds L2 anyway)."""
    import torch
    import tri_synth as ts
    import oracle
    from rope_aware_key_tri_b200 import tri
    L, T, Hq, d = CAL_SHAPE
    if args.layers:
        L = args.layers
    q = ts.make_queries(L, T, Hq, d, seed=1, device="cuda")
    ctx = tri.TriContext(0)
    out = (torch.empty((L, Hq, d), device="cuda"), torch.empty((L, Hq, d // 2), device="cuda"),
           torch.empty((L, Hq, d // 2), device="cuda"))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        ctx.calibrate_estimate(q, tri.TRI_ROPE_HALF, out=out)
    torch.cuda.synchronize()
    times = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ctx.calibrate_estimate(q, tri.TRI_ROPE_HALF, out=out)
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    rows = L * T
    nbytes = q.numel() * 2 + sum(x.numel() * 4 for x in out)
    res = {"metric": CAL_METRIC, "value": rows / (ms * 1e-3), "unit": "rows/s", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 8-token partials, fp64 sums", "data": "synthetic",
           "config": {"workload": "qwen3_8b_calibration_10k", "layers": L, "tokens": T, "q_heads": Hq,
                      "head_dim": d, "layout": "half",
                      "timed": "CUDA events around tri_calibrate_estimate (partial sums + means)"},
           "roofline": roofline_hbm(nbytes, ms),
           "clocks": clk.summary(), "gpu_launches": 2 * args.steps,
           "ms_steps": {"min": min(times), "median": ms, "max": max(times)}}
    if args.no_e2e:
        ctx.close()
        return res
    # end to end: queries from pinned host memory, statistics back to the host
    qh = q.cpu().pin_memory()
    host = tuple(torch.empty(x.shape, dtype=torch.float32).pin_memory() for x in out)
    e2e = []
    for _ in range(2):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        q.copy_(qh, non_blocking=True)
        ctx.calibrate_estimate(q, tri.TRI_ROPE_HALF, out=out)
        for hx, dx in zip(host, out):
            hx.copy_(dx, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e.append(e0.elapsed_time(e1))
    res["e2e"] = {"value": rows / (statistics.median(e2e) * 1e-3), "unit": "rows/s",
                  "ms_per_step": statistics.median(e2e), "h2d_bytes_per_step": q.numel() * 2,
                  "d2h_bytes_per_step": sum(x.numel() * 4 for x in out), "steps": 2}
    if args.no_cpu:
        ctx.close()
        return res
    # the oracle on the host cores, on a bounded sample: whole layers until about 10 s
    import numpy as np
    dt, done = 0.0, 0
    while done < L and dt < 10.0:
        sub = qh[done:done + 1].contiguous().view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        oracle.calibrate(sub, oracle.HALF)
        dt += time.perf_counter() - t0
        done += 1
    res["cpu_baseline"] = {"value": done * T / dt, "unit": "rows/s", "cores": min(os.cpu_count() or 1, Hq),
                           "kind": "oracle", "sample": f"{done} of {L} layers, all {Hq} heads, {T} tokens, {dt:.1f} s"}
    ctx.close()
    return res


DEC_METRIC = "decode-loop cache maintenance: generated tokens/s (128 appends + 1 prune per 128 tokens, Qwen3-8B shape)"


def run_decode(args):
    """One timed step = one cadence cycle (128 appends, then the prune), CUDA events around the
    cycle on the stream; the block-table updates of the cycle (host writes, one copy to the
    device per page boundary) are inside it. The cache carries over from cycle to cycle: the
    prune brings every sequence back to B, the next 128 appends grow it to B + 128."""
    import numpy as np
    import torch
    import tri_synth as ts
    from rope_aware_key_tri_b200 import tri
    spec = ts.WORKLOADS["qwen3_8b_periodic_36l_3200"]
    L, Hkv, G, d, batch, B, cad = spec.n_layers, spec.n_kv_heads, spec.group, spec.head_dim, spec.batch, \
        spec.budget, 128
    if args.layers:
        L = args.layers
    ps = 64
    max_pages = (B + cad + ps - 1) // ps
    n_pages = batch * max_pages + batch
    g = torch.Generator(device="cuda").manual_seed(7)
    K = (torch.randn((L, n_pages, Hkv, ps, d), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    V = torch.randn((L, n_pages, Hkv, ps, d), generator=g, device="cuda").to(torch.bfloat16)
    P = torch.zeros((L, n_pages, Hkv, ps), dtype=torch.int32, device="cuda")
    # sequence s starts at B tokens (positions 0..B-1) in pages s*max_pages + j
    bt = np.full((batch, max_pages), -1, dtype=np.int32)
    free = list(range(n_pages))
    for s in range(batch):
        for j in range((B + ps - 1) // ps):
            bt[s, j] = free.pop(0)
    slot = torch.arange(ps, device="cuda", dtype=torch.int32)
    for s in range(batch):
        for j in range((B + ps - 1) // ps):
            P[:, int(bt[s, j]), :, :] = (j * ps + slot)[None, None, :]
    bt_dev = torch.from_numpy(bt).cuda()
    lens = torch.full((batch,), B, dtype=torch.int32, device="cuda")
    tpos = torch.full((batch,), B, dtype=torch.int32, device="cuda")
    qm, qn, R, offsets = ts.make_stats(ts.replace(spec, n_layers=L), 1)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(L, Hkv, G, d, spec.rope_base, spec.layout, qm, qn, R, offsets)
    new_k = (torch.randn((cad, L, batch, Hkv, d), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    new_v = torch.randn((cad, L, batch, Hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    host_len = B
    stream = torch.cuda.current_stream()

    def cycle():
        nonlocal host_len
        for i in range(cad):
            if host_len % ps == 0:  # every sequence needs its next page
                for s in range(batch):
                    bt[s, host_len // ps] = free.pop(0)
                bt_dev.copy_(torch.from_numpy(bt))  # from pageable memory: the host waits for it
            ctx.append(K, V, P, lens, bt_dev, new_k[i], new_v[i], tpos, advance=True)
            host_len += 1
        ctx.prune(K, V, P, lens, tpos, B, block_table=bt_dev)
        host_len = B
        for s in range(batch):  # pages past B go back to the free list
            for j in range((B + ps - 1) // ps, max_pages):
                if bt[s, j] >= 0:
                    free.append(int(bt[s, j]))
                    bt[s, j] = -1
        bt_dev.copy_(torch.from_numpy(bt))

    for _ in range(args.warmup):
        cycle()
    torch.cuda.synchronize()
    assert ctx.get_error()[0] == tri.TRI_OK

    def timed(fn):
        times = []
        for _ in range(args.steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return times

    # the same cycle with the appends of each page span (64 tokens) replayed from a CUDA graph
    # (the block-table updates and the prune stay outside): what the loop costs on the device
    # once the host no longer issues every append
    graphs, graph_note = [], None
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        for half in range(cad // ps):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=side, capture_error_mode="relaxed"):
                for i in range(half * ps, (half + 1) * ps):
                    ctx.append(K, V, P, lens, bt_dev, new_k[i], new_v[i], tpos, advance=True)
            graphs.append(gr)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        # capturing ran nothing: the state is still the one a cycle starts from
        assert ctx.get_error()[0] == tri.TRI_OK and torch.all(lens == B)
    except Exception as e:  # noqa: BLE001 -- reported in the JSON line, the host-driven number stands
        graphs, graph_note = [], f"unavailable: {type(e).__name__}: {str(e)[:120]}"

    # block-table copies from a rotation of pinned buffers, without a host wait (a copy from
    # pageable memory synchronises the stream first); a buffer is reused only after the
    # synchronised end of a cycle, never while its copy is pending
    pinned = [torch.empty((batch, max_pages), dtype=torch.int32).pin_memory() for _ in range(4)]
    pin_next = 0

    def table_to_device():
        nonlocal pin_next
        buf = pinned[pin_next % len(pinned)]
        pin_next += 1
        buf.numpy()[:] = bt
        bt_dev.copy_(buf, non_blocking=True)

    def cycle_graph():
        nonlocal host_len
        for gr in graphs:
            for s in range(batch):
                bt[s, host_len // ps] = free.pop(0)
            table_to_device()
            gr.replay()
            host_len += ps
        ctx.prune(K, V, P, lens, tpos, B, block_table=bt_dev)
        host_len = B
        for s in range(batch):
            for j in range((B + ps - 1) // ps, max_pages):
                if bt[s, j] >= 0:
                    free.append(int(bt[s, j]))
                    bt[s, j] = -1
        table_to_device()

    with ClockSampler(torch.cuda.current_device()) as clk:
        times_host = timed(cycle)
        times = timed(cycle_graph) if graphs else times_host
    st = ctx.get_error()
    assert st[0] == tri.TRI_OK, st
    assert torch.all(lens == B)
    ms = statistics.median(times)
    row = d * 2
    units = L * batch * Hkv
    nbytes = cad * units * (2 * row + 4) + algorithmic_bytes([B + cad] * batch, L, Hkv, d, B)
    ctx.close()
    return {"metric": DEC_METRIC, "value": batch * cad / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "qwen3_8b_periodic_36l_3200 (paged, 64-token pages)", "layers": L,
                       "kv_heads": Hkv, "group": G, "head_dim": d, "batch": batch, "budget": B, "cadence": cad,
                       "timed": "CUDA events around one cycle: 128 tri_append_advance (two CUDA-graph replays) + "
                                "block-table copies (pinned, asynchronous) + tri_prune"},
            "roofline": roofline_hbm(nbytes, ms),
            # 128 appends of one launch each, the prune's validation and fused kernels
            "clocks": clk.summary(), "gpu_launches": (cad + 2) * args.steps,
            "ms_steps": {"min": min(times), "median": ms, "max": max(times)},
            "appends": "graph replay per 64-token page span" if graphs else (graph_note or "host-driven"),
            "host_driven_ms_per_step": statistics.median(times_host)}


ATT_METRIC = "decode attention over the pruned cache: kept KV rows attended/s (Qwen3-8B shape)"


def run_attend(args):
    """One step = one decode step's attention over the whole pruned cache: every query head of
    every unit attends over its kept rows (tri_decode_attention), CUDA events around the call on
    its stream; a 256 MiB buffer is written between steps. The cache is the default workload
    (one-shot 32K -> 3072 compression of the Qwen3-8B-shaped cache) after one tri_prune."""
    import torch

    import tri_synth as ts
    from rope_aware_key_tri_b200 import tri
    spec = workload_spec(args)
    dev = torch.device("cuda", 0)
    cache = ts.make_cache(spec, seed=1000, device=dev)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(spec.n_layers, spec.n_kv_heads, spec.group, spec.head_dim, spec.rope_base, spec.layout,
                       cache.q_mean, cache.q_norm_mean, cache.R, cache.offsets)
    ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, spec.budget, block_table=cache.block_table)
    st = ctx.get_error()
    assert st[0] == tri.TRI_OK, st
    lens = cache.lens_host.tolist()
    gen = torch.Generator(device=dev).manual_seed(7)
    q = (2.0 * torch.randn((spec.n_layers, spec.batch, spec.n_q_heads, spec.head_dim), generator=gen,
                           device=dev)).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ctx.decode_attention(cache.K, cache.V, cache.lens, q, out=out, block_table=cache.block_table, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    times = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
    st = ctx.get_error()
    assert st[0] == tri.TRI_OK, st
    ms = sum(times) / len(times)
    units = spec.n_layers * spec.batch * spec.n_kv_heads
    rows = sum(lens) * spec.n_layers * spec.n_kv_heads
    nbytes = rows * 2 * spec.head_dim * 2 + q.numel() * 2 + out.numel() * 4
    # launches: validation, attention, and the chunk merge when units are split (three CTAs per
    # SM up to GQA 4, two at GQA 8)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cap_u = cache.cap
    per_sm = 3 if spec.group <= 4 else 2
    cpu = max(1, min(-(-4 * sms * per_sm // units), -(-cap_u // 256)))
    res = {"metric": ATT_METRIC, "value": rows / (ms * 1e-3), "unit": "rows/s", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
           "config": {"workload": f"{args.workload} after one prune", "layers": spec.n_layers,
                      "kv_heads": spec.n_kv_heads, "group": spec.group, "head_dim": spec.head_dim,
                      "batch": spec.batch, "kept_rows_per_unit": sorted(set(lens))[:4],
                      "l2": "256 MiB buffer written between steps; kept K+V %.2f GB" % (rows * 2 * spec.head_dim * 2 / 1e9),
                      "timed": "CUDA events around tri_decode_attention"},
           "roofline": roofline_hbm(nbytes, ms),
           "clocks": clk.summary(), "gpu_launches": (3 if cpu > 1 else 2) * args.steps,
           "ms_steps": {"min": min(times), "median": statistics.median(times), "max": max(times)}}
    if not args.no_e2e:
        # end to end: the step's queries from pinned host memory, the outputs back to the host
        qh = q.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        e2e = []
        for _ in range(3):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q.copy_(qh, non_blocking=True)
            step()
            oh.copy_(out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            e2e.append(e0.elapsed_time(e1))
        e = statistics.median(e2e[1:])
        res["e2e"] = {"value": rows / (e * 1e-3), "unit": "rows/s", "ms_per_step": e,
                      "h2d_bytes_per_step": q.numel() * 2, "d2h_bytes_per_step": out.numel() * 4, "steps": 2}
    if not args.no_cpu:
        res["cpu_baseline"] = time_oracle_attention(cache, spec, q)
    ctx.close()
    return res


def time_oracle_attention(cache, spec, q, budget_s=10.0):
    """The oracle's decode attention on whole units, threads over units (the C call releases the
    interpreter lock), until about budget_s seconds of wall time."""
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    cores = os.cpu_count() or 1
    qb = q.view(torch_int16()).cpu().numpy().view(np.uint16)
    G = spec.group
    order = list(range(cache.n_units))
    rows, done, t0 = 0, 0, time.perf_counter()

    def one(u):
        l, b, g = cache.unit_index(u)
        n = int(cache.lens_host[b])
        k, v, _ = cache.unit_rows(u)
        oracle.decode_attention(qb[l, b, g * G:(g + 1) * G], k[:n], v[:n])
        return n

    with ThreadPoolExecutor(max_workers=cores) as ex:
        while done < len(order) and time.perf_counter() - t0 < budget_s:
            batch = order[done:done + cores]
            rows += sum(ex.map(one, batch))
            done += len(batch)
    el = time.perf_counter() - t0
    return {"value": rows / el, "unit": "rows/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of {cache.n_units} units in full; {rows} rows in {el:.1f} s (incl. host copies)"}


def torch_int16():
    import torch
    return torch.int16


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (smaller cases for profiling)")
    ap.add_argument("--cluster-size", type=int, default=0)
    ap.add_argument("--combine", default="mean", choices=["mean", "max"],
                    help="how the future offsets combine in the score (max: the tensor-core variant)")
    ap.add_argument("--buffers", type=int, default=0)
    ap.add_argument("--engine", default="auto", choices=["auto", "cuda_cores", "tensor"],
                    help="kernels that score the mean mode (auto: tensor cores at group 8)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--path", default="prune", choices=["prune", "calibrate", "decode", "attend"],
                    help="prune: the scoring-and-pruning pass (default); calibrate: the statistics estimator; "
                         "decode: the decode loop's appends and prunes; attend: decode attention over the "
                         "pruned cache")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.path == "calibrate":
        print(json.dumps(run_calibrate(args)), flush=True)
        return
    if args.path == "decode":
        print(json.dumps(run_decode(args)), flush=True)
        return
    if args.path == "attend":
        print(json.dumps(run_attend(args)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist_mod = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist_mod = dist

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        if dist_mod is not None:
            dist_mod.destroy_process_group()
        return

    res, cache, spec = run_ours(args, rank, world, dist_mod)
    out = {
        "metric": METRIC,
        "value": res["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in, fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": args.workload, "layers": spec.n_layers, "kv_heads": spec.n_kv_heads,
                   "group": spec.group, "head_dim": spec.head_dim, "batch_per_gpu": spec.batch,
                   "keys_per_unit": sorted(set(int(x) for x in res["lens"]))[:4],
                   "budget": spec.budget, "parallelism": f"replicas x{world} (sequence shards, no collective)",
                   "l2": "256 MiB buffer written between steps (flushes L2); K+V inputs %.2f GB"
                         % ((cache.K.numel() + cache.V.numel()) * 2 / 1e9),
                   "offsets_combine": args.combine,
                   "timed": "CUDA events around the tri_prune call; row restore between steps untimed"},
        "roofline": res["roofline"],
        "clocks": res["clocks"],
        "gpu_launches": res["gpu_launches"],
        "engine": res["engine"],
        "ms_steps": res["ms_steps"],
        "wall_ms_per_step_incl_restore": res["wall_ms_per_step_incl_restore"],
    }
    if "e2e" in res:
        out["e2e"] = res["e2e"]
    if rank == 0 and world == 1 and not args.no_cpu:
        v, cores, what = time_oracle(cache, spec, budget_s=10.0, combine=args.combine)
        out["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": what}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist_mod is not None:
        dist_mod.barrier()
        dist_mod.destroy_process_group()


if __name__ == "__main__":
    main()
