#!/usr/bin/env python
"""Benchmark: single-token decode attention with ART on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--mode art|full|q8|q8_art] [--no-sweeps]

A step is one decode call over the whole batch of the workload (default: GQA
bf16, B=16, Hq=32, Hkv=8, d=128, per-sequence lengths uniform in [8192, 65536],
tile 64, 8 KV splits + combine -- the largest of the five long-context decode
shapes, 2.25 GiB of K/V): Q load, K/V tile stream, scores, online softmax, PV,
the ART probe and rule, the early-exit vote, the epilogue and the split
combine.  The KV cache is larger than L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  `value` is decoded query-heads per second over
all ranks, device-timed with CUDA events; `e2e` times the same call with the
step's query copied from pinned host memory and its result copied back; the
`roofline` object rates the decode kernel on the KV bytes it actually read
(device counters) against the measured HBM copy bandwidth.  `workloads` holds
the same measurements for all five workloads (full and ART modes, bytes read
and consumed, the thresholds-0 overhead and the thresholds-+inf scaling sweep),
`vskip` the q8 V-skip threshold sweep.  With N > 1 every rank decodes its own
batch of the same shape (weak scaling, no collective in the data path); timing
is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_early_split_b200 import inputs as I  # noqa: E402

METRIC = "decode attention query-heads/s and KV GB/s (fraction of HBM peak), full vs ART"
UNIT = "query-heads/s"
DEFAULT_WORKLOAD = "split_b16_h32x8_d128_Lvar"
# workload of the ablation, traversal-order, paged-cache and eviction sweeps
EXTRAS_WORKLOAD = "gqa_b4_h32x8_d128_L32k"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_traffic.txt")
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=I.WORKLOADS)
    ap.add_argument("--mode", default=None, choices=("art", "full", "q8", "q8_art"))
    ap.add_argument("--q8-path", default="auto", choices=("auto", "tensor_core", "two_pass", "cluster"),
                    help="q8 implementation of the timed mode (art_decode_attn_q8_skipv_path); default the library's")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="time the workload's two modes only (no other workloads, sweeps or extras)")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling: the workload's first N sequences only (bit-identical slabs); "
                         "implies --no-sweeps, and the line is no bench value (config.batch_of says so)")
    a = ap.parse_args(argv)
    if a.mode is None:
        a.mode = "q8_art" if a.workload.startswith("q8") else "art"
    if a.batch:
        a.no_sweeps = True
    return a


# ----------------------------------------------------------------------------- ranks
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def aggregate(elapsed_ms: float, units: float):
    """Max elapsed and summed units over ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return elapsed_ms, units
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers
def hbm_peak():
    try:
        v = json.load(open(PEAKS_FILE))["hbm_gbs"]
        return float(v), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources each timed kernel is compiled from, with the C-ABI file that sets its launch shape.
KERNEL_SOURCES = {
    "art_decode_tc_kernel": ("art_api.cu", "art_device.cuh", "art_kernels.cuh", "art_tc.cuh", "art_tc_pick.cuh",
                             "art_tc_gp1.cu", "art_tc_gp2.cu", "art_tc_gp4.cu", "art_tc_gp8.cu", "art_tc_q8.cu"),
    "art_decode_kernel": ("art_api.cu", "art_device.cuh", "art_kernels.cuh"),
    "q8_two_pass": ("art_api.cu", "art_device.cuh", "art_kernels.cuh", "art_q8_two.cuh"),
}


def kernel_family(kernel_name: str) -> str:
    return "q8_two_pass" if kernel_name.startswith("q8_") else kernel_name


def kernel_source_hash(family: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_early_split_b200", "csrc")
    for f in KERNEL_SOURCES[family]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(workload, mode, kernel_name):
    """DRAM bytes per call from a committed ncu summary, if it matches the kernel's current sources."""
    try:
        kv = dict(l.split(":", 1) for l in open(TRAFFIC_FILE).read().splitlines() if ":" in l)
        kv = {k.strip(): v.strip() for k, v in kv.items()}
        fam = kernel_family(kernel_name)
        if kv.get(f"source_sha256_16[{fam}]") != kernel_source_hash(fam):
            return None
        return float(kv[f"dram_bytes_per_launch[{workload}/{mode}]"])
    except Exception:
        return None


def launches_per_call(K, dp, w, mode, q8_path="auto") -> int:
    """Kernels one decode call launches: q8 over a two-pass workspace runs scores, weights + PV and
    combine (with ART: scores, probe pass, rule, limited pass, combine); every other call one
    kernel, plus the split combine with S > 1."""
    if (mode in ("q8", "q8_art") and q8_path in ("auto", "two_pass")
            and dp.ws_bytes >= K.capi.art_q8_workspace_bytes(dp.shape)):
        if mode == "q8":
            return 3
        if K.kernel_name(dp, mode) == "q8_pv_mma_kernel":
            return 5
    return 1 + (1 if w.num_splits > 1 else 0)


def kv_row_bytes(w):
    return w.d * {"f32": 4, "bf16": 2, "q8": 1}[w.kind] + (2 * (w.d // 32) if w.kind == "q8" else 0)


def bytes_read(w, tiles_read):
    """KV bytes fetched: per (b, kvh, split) `tiles_read` tiles of the split, K and V (+ q8 scales)."""
    rowb = kv_row_bytes(w)
    total = 0
    S = tiles_read.shape[2]
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // w.tile)
        for s in range(S):
            ta = (s * n) // S
            tb = ((s + 1) * n) // S
            split_rows = min(tb * w.tile, L) - ta * w.tile
            for h in range(w.Hkv):
                rows = min(int(tiles_read[b, h, s]) * w.tile, split_rows)
                total += 2 * rows * rowb
    return total


def bytes_consumed(w, used):
    """KV bytes the rule needed: per (b, kvh, split) the slowest head's tiles."""
    rowb = kv_row_bytes(w)
    G = w.G
    total = 0
    S = used.shape[2]
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // w.tile)
        for s in range(S):
            ta = (s * n) // S
            tb = ((s + 1) * n) // S
            split_rows = min(tb * w.tile, L) - ta * w.tile
            for h in range(w.Hkv):
                t = int(used[b, h * G:(h + 1) * G, s].max())
                total += 2 * min(t * w.tile, split_rows) * rowb
    return total


def oracle_batches(w, mode, nb, n_threads):
    """Run the oracle on the first `nb` sequences of the workload (all their query heads) in one call,
    OpenMP over (batch, query head); returns (#query heads, seconds)."""
    import oracle

    kind = {"f32": oracle.KV_F32, "bf16": oracle.KV_BF16, "q8": oracle.KV_Q8}[w.kind]
    t0 = time.perf_counter()
    oracle.decode(
        kind=kind, q=w.q[:nb], k=w.k[:nb], v=w.v[:nb],
        k_scale=None if w.k_scale is None else w.k_scale[:nb],
        v_scale=None if w.v_scale is None else w.v_scale[:nb],
        seq_lens=w.seq_lens[:nb], tile=w.tile, num_splits=w.num_splits,
        art=w.art if mode in ("art", "q8_art") else None, tau=w.tau if mode in ("q8", "q8_art") else 0.0,
        n_threads=n_threads)
    return nb * w.Hq, time.perf_counter() - t0


def oracle_threads(w):
    """Threads the oracle can use: one per (batch, query head) at most, capped by the host's cores."""
    return max(1, min(os.cpu_count() or 1, w.B * w.Hq))


def config_obj(w, mode, args, world):
    return {
        "workload": w.name, "mode": mode, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "L_max": w.L_max,
        "tile": w.tile, "num_splits": w.num_splits, "kv_storage": w.kind,
        "art": {k: w.art[k] for k in ("eps_scale", "eps_dir", "patience")} | {"n_probe": len(w.art["lanes"])},
        "tau": w.tau if mode.startswith("q8") else None,
        "l2": ("L2 flushed (512 MiB write) before every timed launch; step time = the launches' own time"
               if needs_flush(w) else "no flush: KV inputs larger than the 126 MB L2"),
        "parallelism": f"replicas x{world} (weak scaling)" if world > 1 else "single GPU",
    } | ({"batch_of": f"first {w.B} sequences of the workload (profiling case, not a bench value)"}
         if getattr(args, "batch", 0) else {})


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle as it stands, timed on the host cores: each step decodes the first `nb` sequences of
    the workload (all their query heads), nb chosen from one probe call so that a step takes ~2 s."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = I.workload(args.workload)
    cores = oracle_threads(w)
    h1, s1 = oracle_batches(w, args.mode, 1, cores)
    nb = int(max(1, min(w.B, 2.0 // max(s1, 1e-3))))
    for _ in range(args.warmup):
        oracle_batches(w, args.mode, nb, cores)
    tot_h = 0
    tot_s = 0.0
    for _ in range(args.steps):
        h, s = oracle_batches(w, args.mode, nb, cores)
        tot_h += h
        tot_s += s
    val = tot_h / tot_s
    sample = (f"first {nb} of {w.B} sequences of the workload per step = {nb * w.Hq} query heads "
              f"(the whole step is {w.B * w.Hq} query heads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_obj(w, args.mode, args, 1),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


ABLATION_GRID = {
    # criterion family -> (eps_scale, eps_dir) pairs, loosest last
    "both": [(1e-4, 1e-5), (1e-3, 1e-4), (1e-2, 1e-3), (1e-1, 1e-2)],
    "scale_only": [(1e-4, float("inf")), (1e-3, float("inf")), (1e-2, float("inf")), (1e-1, float("inf"))],
    "direction_only": [(float("inf"), 1e-5), (float("inf"), 1e-4), (float("inf"), 1e-3), (float("inf"), 1e-2)],
}


def art_ablation(K, dp, w, mode):
    """Premature-stop error against tiles saved for each criterion family and patience 1, 2, 4:
    per query head, ||O_ART - O_full|| / ||O_full|| (L2 over d), on the bench's own buffers."""
    import torch

    full_mode = "full" if mode == "art" else "q8"
    K.decode(dp, full_mode)
    o_full = dp.o.clone()
    nrm = torch.linalg.vector_norm(o_full, dim=-1).clamp_min(1e-30)
    n_tot = float((-(-w.seq_lens.astype(np.int64) // w.tile)).mean())
    rows = []
    for fam, pairs in ABLATION_GRID.items():
        for pat in (1, 2, 4):
            for es, ed in pairs:
                K.decode(dp, mode, art=dict(w.art, eps_scale=es, eps_dir=ed, patience=pat))
                rel = torch.linalg.vector_norm(dp.o - o_full, dim=-1) / nrm
                rows.append({"criterion": fam, "patience": pat,  # null threshold: criterion off (+inf)
                             "eps_scale": None if es == float("inf") else es,
                             "eps_dir": None if ed == float("inf") else ed,
                             "tiles_saved": 1.0 - float(dp.tiles.float().mean().item()) / n_tot,
                             "rel_err_mean": float(rel.mean().item()), "rel_err_max": float(rel.max().item())})
    torch.cuda.synchronize()
    return rows


def art_orders(K, dp, w, steps, stream):
    """ART with the configured thresholds along each traversal order (natural, recency first,
    importance first): time per call, tiles read, error against full attention, and the time to
    build the sequence on the GPU per step (importance: scoring and sort; the per-tile key summary
    is built once, as a cache would maintain it when keys are appended, and timed apart)."""
    import torch

    if w.kind not in ("f32", "bf16"):
        return None
    K.decode(dp, "full")
    o_full = dp.o.clone()
    nrm = torch.linalg.vector_norm(o_full, dim=-1).clamp_min(1e-30)
    n_tot = float((-(-w.seq_lens.astype(np.int64) // w.tile)).mean())
    out = {}
    summary = K.key_summary(dp, stream=stream.cuda_stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        summary = K.key_summary(dp, stream=stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    out["key_summary_ms"] = e0.elapsed_time(e1) / steps
    for kind in ("natural", "recency", "importance"):
        order = None
        build_ms = 0.0
        if kind != "natural":
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            order = K.tile_order(dp, kind, stream=stream.cuda_stream, summary=summary)
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(steps):
                order = K.tile_order(dp, kind, stream=stream.cuda_stream, summary=summary)
            e1.record(stream)
            torch.cuda.synchronize()
            build_ms = e0.elapsed_time(e1) / steps
        for _ in range(2):
            K.decode(dp, "art", order=order, stream=stream.cuda_stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            K.decode(dp, "art", order=order, stream=stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize()
        rel = torch.linalg.vector_norm(dp.o - o_full, dim=-1) / nrm
        out[kind] = {"ms": e0.elapsed_time(e1) / steps, "order_build_ms": build_ms,
                     "tiles_frac": float(dp.tiles.float().mean().item()) / n_tot,
                     "kv_bytes_read": bytes_read(w, dp.tiles_read().cpu().numpy()),
                     "rel_err_mean": float(rel.mean().item()), "rel_err_max": float(rel.max().item())}
    return out


def evict_sweep(K, dp, w, steps, stream):
    """Random eviction to a quarter of the cache (sink L/128, recent window L/32, the rest drawn
    uniformly), then full attention and ART on the packed cache: time of the selection, the packing
    and the decodes, KV bytes read, and error against full attention over the whole cache."""
    import torch

    L = int(w.L_max)
    budget, sink, recent = L // 4, L // 128, L // 32
    if budget < sink + recent + 1:
        return None
    full_mode, art_mode = ("q8", "q8_art") if w.kind == "q8" else ("full", "art")
    K.decode(dp, full_mode)
    o_full = dp.o.clone()
    nrm = torch.linalg.vector_norm(o_full, dim=-1).clamp_min(1e-30)
    gen = torch.Generator(device=dp.k.device).manual_seed(1234)
    keys = torch.randint(-2**31, 2**31 - 1, (w.B, w.Hkv, L), dtype=torch.int32, device=dp.k.device, generator=gen)
    dp2, kept = K.evict_random(dp, keys, sink, recent, budget, stream=stream.cuda_stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):  # selection + packing of K and V into the same buffers (no allocation)
        K.evict_random_into(dp, dp2, kept, keys, sink, recent, stream=stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    out = {"budget": budget, "n_sink": sink, "n_recent": recent, "select_and_pack_ms": e0.elapsed_time(e1) / steps}
    for m in (full_mode, art_mode):
        _, launch = time_mode(K, dp2, m, steps, 2, stream)
        rel = torch.linalg.vector_norm(dp2.o - o_full, dim=-1) / nrm
        out[m] = {"ms": launch, "kv_bytes_read": bytes_read(w, dp2.tiles_read().cpu().numpy()),
                  "rel_err_mean": float(rel.mean().item()), "rel_err_max": float(rel.max().item())}
    if K.device_status(dp2) != 0:
        raise RuntimeError("device status not OK after the eviction sweep")
    return out


def paged_sweep(K, w, steps, stream):
    """The same step over a paged copy of the cache (random page placement, block table per
    sequence), page sizes 64 and 256: ms per call in both modes, and KV bytes read."""
    import torch

    modes = ("q8", "q8_art") if w.kind == "q8" else ("full", "art")
    out = {}
    for page in (64, 256):
        if page % w.tile:
            continue
        pg = I.paginate(w, page, seed=1)
        dpp = K.upload(w, paged=pg)
        row = {"kernel": K.kernel_name(dpp, modes[1])}
        for m in modes:
            _, launch = time_mode(K, dpp, m, steps, 2, stream)
            row[m] = {"ms": launch, "kv_bytes_read": bytes_read(w, dpp.tiles_read().cpu().numpy())}
        if K.device_status(dpp) != 0:
            raise RuntimeError("device status not OK after the paged sweep")
        out[f"page_{page}"] = row
        del dpp
        torch.cuda.empty_cache()
    return out


def scaling_sweep(K, dp, w, mode, steps, stream, q8_path="auto"):
    """Thresholds +inf and patience k stop every (head, split) after exactly min(k, n) tiles, so the
    time per call against KV bytes read should be a line with a small intercept."""
    n = int(-(-int(w.seq_lens.max()) // w.tile)) // max(1, w.num_splits)
    ks = sorted({1, max(1, n // 8), max(1, n // 4), max(1, n // 2), max(1, n)})
    n_all = float((-(-w.seq_lens.astype(np.int64) // w.tile)).sum() * w.Hq)
    flush = needs_flush(w)
    pts = []
    for k in ks:
        art = dict(w.art, eps_scale=float("inf"), eps_dir=float("inf"), patience=k)
        _, launch = time_mode(K, dp, mode, steps, 2, stream, art=art, flush=flush, q8_path=q8_path)
        check_status(K, dp, w, f"{mode} patience {k}")
        rb = bytes_read(w, dp.tiles_read().cpu().numpy())
        cb = bytes_consumed(w, dp.split_tiles().cpu().numpy())
        pt = {"patience": k, "tiles_frac": float(dp.tiles.double().sum().item()) / n_all,
              "ms": launch, "kv_bytes_read": rb, "kv_bytes_consumed": cb, "read_over_consumed": rb / cb}
        # the same call with speculative reads bounded (art_params.max_spec_tiles = 1: a round is read
        # only if it starts at or before the safe point)
        _, launch_b = time_mode(K, dp, mode, steps, 2, stream, art=dict(art, max_spec_tiles=1), flush=flush,
                                q8_path=q8_path)
        check_status(K, dp, w, f"{mode} patience {k} bounded")
        rb_b = bytes_read(w, dp.tiles_read().cpu().numpy())
        pt["bounded"] = {"max_spec_tiles": 1, "ms": launch_b, "kv_bytes_read": rb_b, "read_over_consumed": rb_b / cb}
        pts.append(pt)
    x = np.array([p["kv_bytes_read"] for p in pts], dtype=np.float64)
    y = np.array([p["ms"] for p in pts], dtype=np.float64)
    slope, icpt = np.polyfit(x, y, 1) if len(pts) > 1 else (0.0, float(y[0]))
    return {"points": pts, "fit_ms": {"intercept": float(icpt), "per_gb": float(slope) * 1e9},
            "note": "eps = +inf, patience k: exactly min(k, n) tiles per (head, split); 'bounded': the same "
                    "call with speculative reads bounded to the round at the safe point"}


def check_status(K, dp, w, what):
    if K.device_status(dp) != 0:
        raise RuntimeError(f"device status not OK after {w.name} {what}")


def mode_row(K, dp, w, mode, steps, stream, peak, art=None, q8_path="auto"):
    """Time one mode on a workload's buffers; throughput, KV bytes read (device counters) and
    consumed (the slowest head of each kv head), and tile counts of the last call."""
    flush = needs_flush(w)
    _, launch = time_mode(K, dp, mode, steps, 2, stream, art=art, flush=flush, q8_path=q8_path)
    if K.device_status(dp) != 0:
        raise RuntimeError(f"device status not OK after {w.name} {mode}")
    n_full = -(-w.seq_lens.astype(np.int64) // w.tile)
    rb = bytes_read(w, dp.tiles_read().cpu().numpy())
    cb = bytes_consumed(w, dp.split_tiles().cpu().numpy())
    tiles = dp.tiles.cpu().numpy()
    gbs = rb / (launch / 1e3) / 1e9
    return {"ms": launch, "query_heads_per_s": w.B * w.Hq / (launch / 1e3), "kv_bytes_read": rb,
            "kv_bytes_consumed": cb, "kv_gbs_read": gbs, "frac_of_hbm": gbs / peak,
            "kv_gbs_consumed": cb / (launch / 1e3) / 1e9, "read_over_consumed": rb / cb,
            "mean_tiles_frac": float(tiles.mean() / n_full.mean())}


def measure_workload(K, w, dp, args, stream, peak, sweeps=True):
    """Full and ART modes of one workload: time per call, GB/s read and consumed, fraction of HBM;
    ART time per consumed KV byte against full attention's per byte; the thresholds-0 overhead and
    the thresholds-+inf scaling sweep."""
    full_mode, art_mode = ("q8", "q8_art") if w.kind == "q8" else ("full", "art")
    steps = max(3, min(args.steps, 10))
    out = {"kernel": {full_mode: K.kernel_name(dp, full_mode), art_mode: K.kernel_name(dp, art_mode)},
           "kv_cache_bytes": kv_cache_bytes(w),
           "l2": "flushed before every timed launch" if needs_flush(w) else "KV larger than L2, no flush"}
    out[full_mode] = mode_row(K, dp, w, full_mode, steps, stream, peak)
    out[art_mode] = mode_row(K, dp, w, art_mode, steps, stream, peak)
    f, a = out[full_mode], out[art_mode]
    out["art_over_full_time"] = a["ms"] / f["ms"]
    # time per consumed byte, ART over full (1.0: ART time follows what it consumed exactly)
    out["art_per_consumed_byte_over_full"] = (a["ms"] / a["kv_bytes_consumed"]) / (f["ms"] / f["kv_bytes_read"])
    # q8 with ART: the default (the rule over the two passes' probe records, which reads every K and
    # V tile once and the consumed V tiles again) and the tensor-core decode kernel (reads follow the
    # rule, a few rounds ahead), whose scaling sweep below shows time against bytes read
    scaling_path = "auto"
    if w.kind == "q8" and K.kernel_name(dp, art_mode) == "q8_pv_mma_kernel":
        out["q8_art_tensor_core"] = mode_row(K, dp, w, art_mode, steps, stream, peak, q8_path="tensor_core")
        scaling_path = "tensor_core"
    if sweeps:
        eps0 = dict(w.art, eps_scale=0.0, eps_dir=0.0)
        e = mode_row(K, dp, w, art_mode, steps, stream, peak, art=eps0)
        out["overhead_eps0"] = {"ms": e["ms"], "ratio_to_full": e["ms"] / f["ms"],
                                "note": "eps = 0: ART never stops and reads every tile"}
        out["scaling"] = scaling_sweep(K, dp, w, art_mode, steps, stream, q8_path=scaling_path)
        out["scaling"]["q8_path"] = scaling_path
    return out


def vskip_sweep(K, args, stream, device):
    """The q8 V-dequant skip threshold tau in {0, 1e-6, 1e-3, 1e-2} on the q8 workload (N(0,1) keys)
    and on its skewed variant (attention sink, Gumbel key offsets, log-normal V norms): ms per call
    with and without ART.  tau = 0 skips nothing, so the time differences are the skip's saving.
    For q8 without ART (the two-pass path) also the device's counts: V rows left out of every
    head's numerator and V tiles not read, as fractions, and the V bytes those tiles saved."""
    import torch

    steps = max(3, min(args.steps, 10))
    out = {"context": "pages: -22.8% decode time at 32K (turbo3 KV, Apple M5 Max), +5% with q8_0 KV "
                      "(M5 Max / M2 Pro); other hardware and formats, not a target"}
    for name in ("q8_b2_h32x8_d128_L32k", "q8_b2_h32x8_d128_L32k_skewed"):
        w = I.workload(name)
        dp = K.upload(w, device=device)
        rows = {}
        for tau in (0.0, 1e-6, 1e-3, 1e-2):
            row = {}
            for mode, path in (("q8", "auto"), ("q8_art", "auto"), ("q8_art_tensor_core", "tensor_core")):
                call = mode[:6] if mode.startswith("q8_art") else mode
                for _ in range(2):
                    K.decode(dp, call, tau=tau, stream=stream.cuda_stream, q8_path=path)
                torch.cuda.synchronize()
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
                for e0, e1 in ev:
                    l2_flush(stream)
                    e0.record(stream)
                    K.decode(dp, call, tau=tau, stream=stream.cuda_stream, q8_path=path)
                    e1.record(stream)
                torch.cuda.synchronize()
                row[mode] = {"ms": sum(a.elapsed_time(b) for a, b in ev) / steps,
                             "kv_bytes_read": bytes_read(w, dp.tiles_read().cpu().numpy()),
                             "mean_tiles_frac": float(dp.tiles.float().mean().item())
                             / float((-(-w.seq_lens.astype(np.int64) // w.tile)).mean())}
                if mode == "q8" and K.kernel_name(dp, mode).startswith("q8_pv"):
                    vs = dp.vskip_counts().cpu().numpy().astype(np.int64)
                    rows_all = float(w.seq_lens.astype(np.int64).sum() * w.Hkv)
                    tiles_all = float((-(-w.seq_lens.astype(np.int64) // w.tile)).sum() * w.Hkv)
                    v_row_bytes = w.d + 2 * (w.d // 32)  # codes + fp16 scales
                    row[mode]["v_rows_skipped_frac"] = float(vs[..., 0].sum()) / rows_all
                    row[mode]["v_tiles_not_read_frac"] = float(vs[..., 1].sum()) / tiles_all
                    row[mode]["v_bytes_not_read"] = int(vs[..., 1].sum()) * w.tile * v_row_bytes
            rows[f"tau_{tau:g}"] = row
        if K.device_status(dp) != 0:
            raise RuntimeError("device status not OK after the V-skip sweep")
        for mode in ("q8", "q8_art", "q8_art_tensor_core"):
            base = rows["tau_0"][mode]["ms"]
            for t in ("tau_1e-06", "tau_0.001", "tau_0.01"):
                rows[t][mode]["time_saved_vs_tau0"] = 1.0 - rows[t][mode]["ms"] / base
        out[name] = rows
        del dp
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- our arm
L2_BYTES = 126 * 1024 * 1024
_flush_buf = None


def needs_flush(w) -> bool:
    """KV caches under twice the L2 size are flushed from L2 between timed launches."""
    return kv_cache_bytes(w) < 2 * L2_BYTES


def kv_cache_bytes(w) -> int:
    rowb = kv_row_bytes(w)
    return int(2 * w.B * w.Hkv * w.L_max * rowb)


def l2_flush(stream):
    """Overwrite a buffer larger than L2 on `stream` (evicts the KV cache from L2)."""
    import torch

    global _flush_buf
    if _flush_buf is None:
        _flush_buf = torch.empty(4 * L2_BYTES, dtype=torch.uint8, device=torch.cuda.current_device())
    with torch.cuda.stream(stream):
        _flush_buf.fill_(1)


def time_mode(K, dp, mode, steps, warmup, stream, art=None, flush=False, q8_path="auto"):
    """Device time of `steps` calls: (total ms, mean per-launch ms from per-launch events).  With
    flush, L2 is overwritten before every launch and the total is the sum of the launches' own
    times (the flushes are not counted)."""
    import torch

    for _ in range(warmup):
        K.decode(dp, mode, art=art, stream=stream.cuda_stream, q8_path=q8_path)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        if flush:
            l2_flush(stream)
        ev[i][0].record(stream)
        K.decode(dp, mode, art=art, stream=stream.cuda_stream, q8_path=q8_path)
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in ev]
    total = sum(per) if flush else start.elapsed_time(end)
    return total, sum(per) / len(per)


def run_ours(args):
    import torch

    import kv_cache_early_split_b200 as K

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl")
    dev = torch.device("cuda", torch.cuda.current_device())
    w = I.workload(args.workload, keys_b=list(range(args.batch)) if args.batch else None)
    dp = K.upload(w, device=dev)
    stream = torch.cuda.Stream(device=dev)
    heads = w.B * w.Hq

    # main timed region (the method's mode), clocks sampled meanwhile
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(torch.cuda.current_device()))
    q8_path = args.q8_path if w.kind == "q8" else "auto"
    for _ in range(args.warmup):
        K.decode(dp, args.mode, stream=stream.cuda_stream, q8_path=q8_path)
    torch.cuda.synchronize()
    sampler.start()
    flush = needs_flush(w)
    total_ms, launch_ms = time_mode(K, dp, args.mode, args.steps, 0, stream, flush=flush, q8_path=q8_path)
    clocks = sampler.stop()
    if K.device_status(dp) != 0:
        raise RuntimeError("device status not OK after the timed region")
    tiles_read = dp.tiles_read().cpu().numpy()
    used = dp.split_tiles().cpu().numpy()
    tiles = dp.tiles.cpu().numpy()
    gpu_launches = args.steps * launches_per_call(K, dp, w, args.mode, q8_path)

    max_ms, all_heads = aggregate(total_ms, heads * args.steps)
    value = all_heads / (max_ms / 1e3)
    peak, peak_kind = hbm_peak()
    rb = bytes_read(w, tiles_read)
    cb = bytes_consumed(w, used)
    achieved = rb / (launch_ms / 1e3) / 1e9
    n_full = -(-w.seq_lens.astype(np.int64) // w.tile)

    # the other mode (full vs ART) on the same buffers
    other = {"art": "full", "full": "art", "q8": "q8_art", "q8_art": "q8"}[args.mode]
    o_total, o_launch = time_mode(K, dp, other, args.steps, args.warmup, stream, flush=flush)
    o_read = bytes_read(w, dp.tiles_read().cpu().numpy())
    o_cons = bytes_consumed(w, dp.split_tiles().cpu().numpy())
    o_max, _ = aggregate(o_total, 0)
    modes = {
        args.mode: {"query_heads_per_s": value, "ms_per_step": max_ms / args.steps,
                    "kv_gbs_read": achieved, "frac_of_hbm": achieved / peak,
                    "kv_bytes_read": rb, "kv_bytes_consumed": cb, "read_over_consumed": rb / cb,
                    "mean_tiles_frac": float(tiles.mean() / n_full.mean())},
        other: {"query_heads_per_s": heads * world * args.steps / (o_max / 1e3), "ms_per_step": o_max / args.steps,
                "kv_gbs_read": o_read / (o_launch / 1e3) / 1e9, "frac_of_hbm": o_read / (o_launch / 1e3) / 1e9 / peak,
                "kv_bytes_read": o_read, "kv_bytes_consumed": o_cons},
    }

    workloads = vskip = extras = None
    if not args.no_sweeps:
        # every workload, full and ART, with the overhead and scaling sweeps
        workloads = {}
        for name in I.WORKLOADS:
            if name == w.name:
                workloads[name] = measure_workload(K, w, dp, args, stream, peak)
                continue
            wl = I.workload(name)
            dpl = K.upload(wl, device=dev)
            workloads[name] = measure_workload(K, wl, dpl, args, stream, peak)
            del dpl, wl
            torch.cuda.empty_cache()
        vskip = vskip_sweep(K, args, stream, dev)
        # ablation, traversal orders, paged cache and eviction on the 32K GQA workload
        steps_x = max(3, min(args.steps, 10))
        we = w if w.name == EXTRAS_WORKLOAD else I.workload(EXTRAS_WORKLOAD)
        dpe = dp if we is w else K.upload(we, device=dev)
        extras = {"workload": we.name, "ablation": art_ablation(K, dpe, we, "art"),
                  "orders": art_orders(K, dpe, we, steps_x, stream),
                  "paged": paged_sweep(K, we, steps_x, stream),
                  "eviction": evict_sweep(K, dpe, we, steps_x, stream)}
        if dpe is not dp:
            del dpe
        del we
        torch.cuda.empty_cache()

    # end to end through the public call: the step's query in from pinned host memory, O and tiles back out
    q_host = dp.q.cpu().pin_memory()
    o_host = torch.empty_like(dp.o, device="cpu").pin_memory()
    t_host = torch.empty_like(dp.tiles, device="cpu").pin_memory()
    for _ in range(args.warmup):
        dp.q.copy_(q_host, non_blocking=True)
        K.decode(dp, args.mode, q8_path=q8_path)
        o_host.copy_(dp.o, non_blocking=True)
        t_host.copy_(dp.tiles, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for _ in range(args.steps):
        dp.q.copy_(q_host, non_blocking=True)
        K.decode(dp, args.mode, q8_path=q8_path)
        o_host.copy_(dp.o, non_blocking=True)
        t_host.copy_(dp.tiles, non_blocking=True)
    e1.record(cur)
    torch.cuda.synchronize()
    e2e_ms, e2e_heads = aggregate(e0.elapsed_time(e1), heads * args.steps)
    e2e = {"value": e2e_heads / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": int(q_host.numel() * q_host.element_size()),
           "d2h_bytes_per_step": int(o_host.numel() * 4 + t_host.numel() * 4),
           "note": "KV cache resident in HBM as in serving; per step the query goes in and O + tiles come out"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle over whole passes of the same workload, repeated until >= 10 s of CPU time
        cores = oracle_threads(w)
        h_done, secs, passes = 0, 0.0, 0
        while secs < 10.0:
            h, s_ = oracle_batches(w, args.mode, w.B, cores)
            h_done, secs, passes = h_done + h, secs + s_, passes + 1
        cpu = {"value": h_done / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{passes} whole passes of the workload ({h_done} query heads, {secs:.1f} s)"}

    kernel = K.kernel_name(dp, args.mode)
    if q8_path == "tensor_core":
        kernel = "art_decode_tc_kernel"
    elif q8_path == "cluster":
        kernel = "art_decode_kernel"
    # (the committed DRAM figures are for the library's default path of each mode)
    traffic = measured_traffic(w.name, args.mode, kernel) if q8_path == "auto" and not args.batch else None
    if launches_per_call(K, dp, w, args.mode, q8_path) == 3:
        mma = "_mma" if kernel == "q8_pv_mma_kernel" else ""
        kernel = f"q8_scores{mma}_kernel + q8_pv{mma}_kernel + q8_combine_kernel (timed as one call)"
    elif launches_per_call(K, dp, w, args.mode, q8_path) == 5:
        kernel = ("q8_scores_mma_kernel + q8_pv_mma_kernel (probe pass) + q8_rule_kernel + q8_pv_mma_kernel "
                  "(limited pass) + q8_combine_kernel (timed as one call)")
    elif w.num_splits > 1:
        kernel += " (timed with its split combine kernel)"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "storage": w.kind, "data": "synthetic",
        "config": config_obj(w, args.mode, args, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} hbm_gbs (copy)", "traffic": traffic,
                     "kernel": kernel, "bytes_per_launch": rb, "launch_ms": launch_ms},
        "modes": modes,
        "workloads": workloads,
        "vskip": vskip,
        "extras": extras,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
