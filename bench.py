"""Benchmark of the CalibAtt attention hot path on B200.

One step = one block-sparse self-attention call of the Wan-2.1-14B-shaped
720p layer (batch 1, 40 heads, head_dim 128, N = 21*45*80 = 75600 tokens,
128x128 blocks, per-head seeded calibrated masks at 32-38% block density).
Metric: effective TFLOP/s counted on retained blocks (4*B*B*D flop per
retained tile), with ms per call, as a fraction of the measured B200 dense
bf16 tensor peak, next to this library's own all-ones (dense) mask path.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torch.distributed.run; every rank runs an independent
720p layer (weak scaling, no collective on the data path).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

FLOP_PER_TILE = 4 * 128 * 128 * 128
REASON_BITS = {  # nvidia-smi clocks_event_reasons.active bitmask
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.mkdtemp(prefix="calibatt_clocks_"), f"clocks_rank{index}.csv")
        # nvidia-smi numbers GPUs physically, CUDA by CUDA_VISIBLE_DEVICES:
        # name the device by its UUID so that each rank samples its own GPU
        self.smi_id = str(index)
        try:
            import torch
            u = str(torch.cuda.get_device_properties(index).uuid)
            self.smi_id = u if u.startswith("GPU-") else f"GPU-{u}"
        except Exception:
            pass

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.smi_id}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                mask = int(parts[4], 16) if parts[4].startswith("0x") else int(parts[4])
            except ValueError:
                continue
            for bit, name in REASON_BITS.items():
                if mask & bit:
                    reasons.add(name)
        busy = [s for s in sm if s > 0]
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons - {"gpu_idle"}),
                "samples": len(sm)}


def measured_traffic(tiles, path=None):
    """DRAM bytes per launch of the sparse kernel from the committed ncu counters
    of the bench launch itself (profiles/tc_attn_sparse_720p_traffic.json), per
    retained tile times the tiles of this launch; None
    when a source the traffic depends on (the kernel file, the headers it
    includes, and the host file that builds the schedule) changed since the
    capture."""
    import hashlib
    path = path or os.path.join(ROOT, "profiles", "tc_attn_sparse_720p_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    for src, sha in t["kernel_sources_sha256"].items():
        with open(os.path.join(ROOT, src), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != sha:
                return None
    return t["dram_bytes_per_retained_tile"] * tiles


def rank_seed(base, rank):
    """Input seed of a rank: every rank times an independent layer (weak scaling)."""
    return base + 7919 * rank


def max_over_ranks(x, dist=None, device="cpu"):
    """Largest value of x over the ranks of the default process group (x itself
    when there is none); every rank must call it in the same order."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flop_per_rank, world, ms):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flop_per_rank / (ms * 1e-3) / 1e12


def head_partition(heads, rank, world):
    """Heads of one attention call that rank `rank` of `world` computes under
    --partition heads: heads[rank::world] (every head on exactly one rank;
    heads are independent, so no exchange follows)."""
    return list(range(heads))[rank::world]


# MUFU exp2 issue rate of one SM per clock (4 per SM sub-partition), the
# bound of the offline energy passes (16,384 exp2 per 128x128 tile against
# 512 tensor-core cycles for its one Q K^T)
EX2_PER_CLK_PER_SM = 16


def mufu_exp2_peak(sm_count, sm_mhz):
    """exp2 results per second of the whole GPU at a clock."""
    return EX2_PER_CLK_PER_SM * sm_count * sm_mhz * 1e6


DICT_FORMAT = "lists"  # --dict-format


def build_dict(C, masks, heads, nb, block, geometry=None, fmt=None):
    """One-layer dictionary (format `fmt`, default --dict-format); with
    geometry = (frames, rows, cols, anchors) the dual path of the layer runs
    as one launch."""
    fmt = fmt or DICT_FORMAT
    rp, ci, rep_arr = C.masks_to_layer_csr(masks, heads, nb)
    cap = C.count_intervals(rp, ci) if fmt == "intervals" else ci.size
    d = C.MaskDictionary(1, 1, heads, nb, nb, block, max(1, cap), bitmap=fmt == "bitmap",
                         intervals=fmt == "intervals")
    if geometry is not None:
        d.set_anchor_geometry(*geometry)
    d.set_layer(0, 0, rp, ci, rep_arr)
    return d


def time_calls(torch, fn, steps, warmup, stream):
    """Per-call device time (ms) with CUDA events on the launching stream."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def cpu_baseline(wl, masks, q, k, v, o=None, budget_s=12.0, seed=0):
    """The float64 oracle, as it stands, on a bounded seeded sample of query
    blocks.  With o (the library's output of the same call) the sampled rows
    are also compared: returns (baseline, parity)."""
    from oracle import calibatt_oracle as O

    rng = np.random.default_rng(seed)
    heads = sorted(masks)
    t_start = time.perf_counter()
    t_or = 0.0
    tiles = 0
    n_blocks = 0
    qn = kn = vn = on = None
    last_h = None
    err_max, err_sum, err_n = 0.0, 0.0, 0
    while time.perf_counter() - t_start < budget_s:
        h = int(rng.choice(heads))
        r = int(rng.integers(0, wl.num_blocks))
        if h != last_h:
            qn = q[0, :, h].float().cpu().numpy().astype(np.float64)
            kn = k[0, :, h].float().cpu().numpy().astype(np.float64)
            vn = v[0, :, h].float().cpu().numpy().astype(np.float64)
            on = o[0, :, h].float().cpu().numpy().astype(np.float64) if o is not None else None
            last_h = h
        rows = np.arange(r * wl.block, min(wl.seq_len, (r + 1) * wl.block))
        ts = time.perf_counter()
        ref, _ = O.block_sparse_attention(qn, kn, vn, masks[h], wl.block, rows=rows)
        t_or += time.perf_counter() - ts
        if on is not None:
            err = np.abs(on[rows] - ref)
            err_max, err_sum, err_n = max(err_max, float(err.max())), err_sum + float(err.sum()), err_n + err.size
        tiles += int(masks[h][r].sum())
        n_blocks += 1
    tflops = tiles * FLOP_PER_TILE / t_or / 1e12
    base = {"value": tflops, "unit": "TFLOP/s (effective, retained blocks)", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n_blocks} seeded (head, q-block) rows of the 720p layer, {tiles} retained tiles, "
                      f"{t_or:.1f} s of float64 NumPy; ms/call extrapolated to the full call = "
                      f"{t_or / max(tiles, 1) * sum(int(m.sum()) for m in masks.values()) * 1e3:.0f} ms"}
    if o is None:
        return base
    mean = err_sum / max(err_n, 1)
    parity = {"max_abs": err_max, "mean_abs": mean, "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3},
              "within_tolerance": err_max <= 2e-2 and mean <= 2e-3,
              "sample": f"the same {n_blocks} (head, q-block) rows of this run's block-sparse output "
                        f"against the float64 oracle"}
    return base, parity


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle on this workload, each step a bounded sample."""
    if rank != 0:
        return
    from oracle import calibatt_oracle as O
    import torch

    wl = W.WORKLOADS["720p"]
    masks, _ = W.workload_masks(wl)
    q, k, v = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cpu")
    rng = np.random.default_rng(5)
    per_step = []
    total_tiles = 0
    for step in range(args.warmup + args.steps):
        h = int(rng.integers(0, wl.heads))
        blocks = rng.choice(wl.num_blocks, 2, replace=False)
        qn = q[0, :, h].float().numpy().astype(np.float64)
        kn = k[0, :, h].float().numpy().astype(np.float64)
        vn = v[0, :, h].float().numpy().astype(np.float64)
        rows = np.concatenate([np.arange(r * 128, min(wl.seq_len, (r + 1) * 128)) for r in blocks])
        t0 = time.perf_counter()
        O.block_sparse_attention(qn, kn, vn, masks[h], wl.block, rows=rows)
        dt = time.perf_counter() - t0
        tiles = int(masks[h][blocks].sum())
        if step >= args.warmup:
            per_step.append((dt, tiles))
            total_tiles += tiles
    t = sum(d for d, _ in per_step)
    value = total_tiles * FLOP_PER_TILE / t / 1e12
    ms = t / len(per_step) * 1e3
    line = {"metric": "effective TFLOP/s (retained blocks) and ms/call, % of B200 BF16 tensor peak",
            "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "wan2.1-14b-720p self-attention, block-sparse path (2 query blocks per step)",
                       "batch": 1, "heads": wl.heads, "head_dim": wl.head_dim, "seq_len": wl.seq_len,
                       "block": wl.block},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": "each step: 2 seeded query blocks of one seeded head, float64 NumPy"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    del torch


def run_anchor_case(args, torch, C, pk):
    """The anchor path alone: the 12 repetitive heads of the dual-path 720p
    layer (anchor rows attend to all keys, the output is broadcast to every
    row), timed with CUDA events; a case of its own for profiling the anchor
    kernel.  Prints effective TFLOP/s (8.39 MFLOP per anchor tile x key block)."""
    import dataclasses
    wd = W.WORKLOADS["720p_dual"]
    _, rep_heads = W.workload_masks(wd)
    # --heads: the layer's first heads only (a smaller case for profiling)
    wd = dataclasses.replace(wd, heads=min(args.heads, wd.heads))
    rep_heads = tuple(h for h in rep_heads if h < wd.heads)
    q, k, v = W.make_qkv(wd.seed, 1, wd.seq_len, wd.heads, wd.head_dim, "bf16", wd.input_std, "cuda")
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    tiles = len(rep_heads) * -(-wd.frames * len(wd.anchors) * wd.cols // 128) * wd.num_blocks
    ws = anchor_workspace(torch, C, q, wd, len(rep_heads))
    per_call = time_calls(torch, lambda: C.calibatt_anchor_attn(q, k, v, o, wd.frames, wd.rows, wd.cols,
                                                                wd.anchors, list(rep_heads), workspace=ws,
                                                                stream=stream),
                          args.steps, args.warmup, stream)
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the anchor case")
    ms = statistics.mean(per_call)
    tf = tiles * FLOP_PER_TILE / (ms * 1e-3) / 1e12
    n_tiles = len(rep_heads) * -(-wd.frames * len(wd.anchors) * wd.cols // 128)
    first, parts = C.anchor_split_plan(n_tiles, C.device_sm_count(), wd.num_blocks)
    print(json.dumps({"anchor_case": {
        "heads": len(rep_heads), "anchor_tiles_x_key_blocks": tiles, "ms_per_call": ms,
        "effective_tflops": tf, "frac_of_burst_peak": tf / pk["bf16_tflops"],
        "split_tiles": n_tiles - first, "parts_per_split_tile": parts,
        "output_bytes": len(rep_heads) * wd.seq_len * wd.head_dim * 2}}), flush=True)


def anchor_workspace(torch, C, q, wd, n_heads):
    """The anchor call's workspace (its last partial wave of tiles split over
    key ranges), or None when the call would not split."""
    nbytes = C.calibatt_anchor_attn_workspace_size(q, wd.frames, wd.rows, wd.cols, len(wd.anchors), n_heads)
    return torch.empty(nbytes // 4, dtype=torch.float32, device="cuda") if nbytes else None


def run_energy_case(args, torch, C, pk):
    """The block energy alone on the 720p geometry with --heads heads (LSE
    pass, energy pass), timed with CUDA events; a case of its own for
    profiling the tensor-core energy modes."""
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["720p"], heads=args.heads)
    q, k, _ = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    e = torch.empty((1, wl.heads, wl.num_blocks, wl.num_blocks), device="cuda")
    ws = torch.empty(C.calibatt_block_energy_workspace_size(q) // 4, device="cuda")
    stream = torch.cuda.current_stream()
    per_call = time_calls(torch, lambda: C.calibatt_block_energy(q, k, e, ws, wl.block, stream=stream),
                          args.steps, args.warmup, stream)
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the energy case")
    ms = statistics.mean(per_call)
    exp2 = 2 * wl.seq_len ** 2 * wl.heads      # both passes exponentiate every score
    print(json.dumps({"energy_case": {
        "heads": wl.heads, "ms_per_call": ms, "exp2_per_call": exp2,
        "g_exp2_per_s": exp2 / (ms * 1e-3) / 1e9,
        "frac_of_mufu_peak_at_max_clock": exp2 / (ms * 1e-3) / mufu_exp2_peak(C.device_sm_count(), 1965.0)}}),
        flush=True)


def run_similarity_case(args, torch, C, pk):
    """The spatial-similarity pass alone on the 720p geometry with --heads
    heads (LSE pass, pass of per-query sums, row reduction), timed with CUDA
    events; a case of its own for profiling the tensor-core similarity mode."""
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["720p_dual"], heads=args.heads)
    q, k, _ = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    sim = torch.empty((1, wl.heads, wl.frames, wl.rows), device="cuda")
    ws = torch.empty(C.calibatt_spatial_similarity_workspace_size(q) // 4, device="cuda")
    stream = torch.cuda.current_stream()
    per_call = time_calls(torch, lambda: C.calibatt_spatial_similarity(q, k, sim, ws, wl.frames, wl.rows, wl.cols,
                                                                       wl.anchors, stream=stream),
                          args.steps, args.warmup, stream)
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the similarity case")
    ms = statistics.mean(per_call)
    exp2 = 3 * wl.seq_len ** 2 * wl.heads
    print(json.dumps({"similarity_case": {
        "heads": wl.heads, "ms_per_call": ms, "exp2_per_call": exp2,
        "g_exp2_per_s": exp2 / (ms * 1e-3) / 1e9,
        "frac_of_mufu_peak_at_max_clock": exp2 / (ms * 1e-3) / mufu_exp2_peak(C.device_sm_count(), 1965.0)}}),
        flush=True)


def run_dual_case(args, torch, C, pk):
    """The dual-path 720p layer alone (28 block-sparse heads and 12 anchor heads
    in ONE fused launch over the dictionary's joint schedule), timed with CUDA
    events; a case of its own for profiling the fused kernel."""
    import dataclasses
    wd = W.WORKLOADS["720p_dual"]
    dmasks, rep_heads = W.workload_masks(wd)
    # --heads: the layer's first heads only (a smaller case for profiling)
    wd = dataclasses.replace(wd, heads=min(args.heads, wd.heads))
    rep_heads = tuple(h for h in rep_heads if h < wd.heads)
    geom = (wd.frames, wd.rows, wd.cols, wd.anchors)
    q, k, v = W.make_qkv(wd.seed, 1, wd.seq_len, wd.heads, wd.head_dim, "bf16", wd.input_std, "cuda")
    o = torch.empty_like(q)
    # one launch over the joint schedule, or (--dual-launches 2) the block-sparse
    # and anchor launches of a dictionary without the anchor geometry
    d = build_dict(C, [dmasks[h] for h in range(wd.heads)], wd.heads, wd.num_blocks, wd.block,
                   geom if args.dual_launches == 1 else None)
    tiles = d.layer_info(0, 0)["retained_tiles"] + \
        len(rep_heads) * -(-wd.frames * len(wd.anchors) * wd.cols // 128) * wd.num_blocks
    stream = torch.cuda.current_stream()
    per_call = time_calls(torch, lambda: C.calibatt_dual_path_attn(q, k, v, o, d, 0, 0, wd.frames, wd.rows,
                                                                   wd.cols, wd.anchors, wd.block, stream=stream),
                          args.steps, args.warmup, stream)
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the dual-path case")
    d.close()
    ms = statistics.mean(per_call)
    tf = tiles * FLOP_PER_TILE / (ms * 1e-3) / 1e12
    print(json.dumps({"dual_case": {
        "sparse_heads": wd.heads - len(rep_heads), "anchor_heads": len(rep_heads),
        "launches_per_call": args.dual_launches,
        "tiles": tiles, "ms_per_call": ms, "effective_tflops": tf, "frac_of_burst_peak": tf / pk["bf16_tflops"]}}),
        flush=True)


def run_epilogue_probe(torch, B, C, fused=False):
    """Store rate of the anchor broadcast epilogue (the 12 repetitive heads of
    the dual-path 720p layer), in the anchor-only launch or (fused=True) in
    the fused dual-path launch.  The measurement build records, per CTA, the
    nanoseconds its epilogues spend issuing the output stores of anchor tiles;
    every output row of those heads is written once (N x D x 2 bytes per
    head), so the aggregate rate while in the epilogue is bytes / (mean
    per-CTA epilogue time)."""
    import ctypes
    lib = ctypes.CDLL(B.build(trace=True))
    for name, (res, argt) in C.SIGNATURES.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, argt
    lib.calibatt_epilogue_probe_read.restype = ctypes.c_int
    lib.calibatt_epilogue_probe_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    C.LIB = lib
    wd = W.WORKLOADS["720p_dual"]
    _, rep_heads = W.workload_masks(wd)
    q, k, v = W.make_qkv(wd.seed, 1, wd.seq_len, wd.heads, wd.head_dim, "bf16", wd.input_std, "cuda")
    o = torch.empty_like(q)

    dmasks, _ = W.workload_masks(wd)
    d = build_dict(C, [dmasks[h] for h in range(wd.heads)], wd.heads, wd.num_blocks, wd.block,
                   (wd.frames, wd.rows, wd.cols, wd.anchors)) if fused else None

    def call():
        if fused:
            C.calibatt_dual_path_attn(q, k, v, o, d, 0, 0, wd.frames, wd.rows, wd.cols, wd.anchors, wd.block)
        else:
            C.calibatt_anchor_attn(q, k, v, o, wd.frames, wd.rows, wd.cols, wd.anchors, list(rep_heads))

    call()
    torch.cuda.synchronize()
    lib.calibatt_trace_reset()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    call()
    b.record()
    torch.cuda.synchronize()
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out during the epilogue probe")
    ns = (ctypes.c_ulonglong * 1024)()
    items = (ctypes.c_ulonglong * 1024)()
    lib.calibatt_epilogue_probe_read(ns, items, 1024)
    used = [(ns[i], items[i]) for i in range(1024) if items[i] > 0]
    total_bytes = len(rep_heads) * wd.seq_len * wd.head_dim * 2
    mean_ns = sum(t for t, _ in used) / len(used)
    n_items = sum(n for _, n in used)
    if d is not None:
        d.close()
    print(json.dumps({"epilogue_probe": {
        "workload": "dual-path 720p layer, anchor tiles of its 12 repetitive heads, " +
                    ("fused launch" if fused else "anchor-only launch, whole tiles") + " (staged stores)",
        "anchor_tiles": n_items, "ctas": len(used), "output_bytes": total_bytes,
        "epilogue_ns_per_tile": sum(t for t, _ in used) / n_items,
        "bytes_per_tile": total_bytes / n_items,
        "aggregate_gbs_in_epilogue": total_bytes / mean_ns,
        "call_ms_measurement_build": a.elapsed_time(b),
        "epilogue_share_of_call": mean_ns / (a.elapsed_time(b) * 1e6),
        "call": "calibatt_dual_path_attn (one fused launch)" if fused else "calibatt_anchor_attn",
        "peak_hbm_gbs": peaks()["hbm_gbs"]}}), flush=True)


def softmax_phase_breakdown(recs, first=100, last=3900):
    """Per-block phases of the two softmax streams from trace records
    (event, key-block iteration, SM clock) of CTA 0: for each block a stream
    owns, the cycles from the end of its previous block to the scores being
    ready, the tensor-memory load, the row maximum, the spin on the other
    stream's reference, the publish, the wait for the P buffer, the
    exponential chain and the hand-off.  Event numbers follow the kernel's
    trace points (32/36 scores ready, 40/44 loaded, 12-17 reference, 56/60 P
    buffer free, 48/52 exponentials done, 20/24 P handed over)."""
    import collections
    ev = collections.defaultdict(dict)
    for e, i, t in recs:
        ev[e][i] = t
    names = ["wait_s_full", "tmem_ld", "row_max", "spin_ref", "publish", "wait_p_free", "exp_chain",
             "rescale_p_full"]
    out = {}
    for s in (0, 1):
        w = 4 * s
        seq = [(32 + w), (40 + w), (12 + s), (14 + s), (16 + s), (56 + w), (48 + w), (20 + w)]
        ph = collections.defaultdict(list)
        prev = None
        for g in sorted(ev[32 + w]):
            if first <= g < last and prev is not None and prev in ev[20 + w] and all(g in ev[e] for e in seq):
                t = [ev[20 + w][prev]] + [ev[e][g] for e in seq]
                for k, name in enumerate(names):
                    ph[name].append(t[k + 1] - t[k])
                ph["total"].append(t[-1] - t[0])
            prev = g
        tot = sum(ph["total"]) or 1
        out[f"stream{s}"] = {k: {"median_cycles": statistics.median(v), "share": round(sum(v) / tot, 4)}
                             for k, v in ph.items() if v}
        out[f"stream{s}"]["blocks"] = len(ph["total"])
    return out


def run_softmax_phases(args, torch, B, C):
    """The measurement build (-DCALIBATT_TRACE) on the 720p layer with
    --heads heads: one traced call after three warm-up calls, and the phase
    breakdown of CTA 0's two softmax streams."""
    import ctypes
    import dataclasses
    lib = ctypes.CDLL(B.build(trace=True))
    for name, (res, argt) in C.SIGNATURES.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, argt
    lib.calibatt_trace_read.restype = ctypes.c_int
    lib.calibatt_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_int]
    C.LIB = lib
    wl = dataclasses.replace(W.WORKLOADS["720p"], heads=args.heads)
    masks, _ = W.workload_masks(wl, seed_base=W.MASK_SEED_BASE["720p"])
    q, k, v = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    o = torch.empty_like(q)
    d = build_dict(C, [masks[h] for h in range(wl.heads)], wl.heads, wl.num_blocks, wl.block)
    for _ in range(3):
        C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block)
    torch.cuda.synchronize()
    lib.calibatt_trace_reset()
    C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block)
    torch.cuda.synchronize()
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the traced call")
    n_ev, n_it = 64, 4096
    buf = (ctypes.c_ulonglong * (n_ev * n_it))()
    n = lib.calibatt_trace_read(buf, n_ev * n_it)
    recs = [(i // n_it, i % n_it, buf[i]) for i in range(n) if buf[i] != 0]
    ms = statistics.mean(time_calls(torch, lambda: C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block),
                                    5, 1, torch.cuda.current_stream()))
    tiles = d.layer_info(0, 0)["retained_tiles"]
    d.close()
    print(json.dumps({"softmax_phases": {
        "workload": f"720p layer, {wl.heads} heads, measurement build, CTA 0",
        "ms_per_call_measurement_build": ms, "effective_tflops": tiles * FLOP_PER_TILE / (ms * 1e-3) / 1e12,
        **softmax_phase_breakdown(recs)}}), flush=True)


def run_sweep(args, C, torch, stream, pk):
    """Schedule sweep: a dictionary holding every (timestep, layer) record of
    the schedule, then one dual-path call per (t, l) on fresh seeded inputs,
    timed with CUDA events; the dense path is timed on a sample of the calls."""
    import time
    wl = W.WORKLOADS["720p_sweep"]
    T, L, H, nb = args.sweep_steps, args.sweep_layers, wl.heads, wl.num_blocks
    t_build = time.time()
    nnz = sum(W.sweep_record_blocks(wl, t, l, h, T) for t in range(T) for l in range(L) for h in range(H))
    if DICT_FORMAT == "intervals":
        raise SystemExit("the full sweep builds its dictionary as index lists or bitmaps")
    dct = C.MaskDictionary(T, L, H, nb, nb, wl.block, nnz, bitmap=DICT_FORMAT == "bitmap")
    dct.set_anchor_geometry(wl.frames, wl.rows, wl.cols, wl.anchors)
    for t in range(T):
        for l in range(L):
            masks, rep = W.sweep_layer_masks(wl, t, l, "cuda", T)
            rp, ci = W.layer_csr(masks)
            rep_arr = np.zeros(H, np.uint8)
            rep_arr[list(rep)] = 1
            dct.set_layer(t, l, rp, ci, rep_arr)
    build_s = time.time() - t_build
    info = dct.info()
    anchor_tiles_per_head = -(-wl.frames * len(wl.anchors) * wl.cols // 128) * nb
    tiles = 0
    for t in range(T):
        for l in range(L):
            li = dct.layer_info(t, l)
            tiles += li["retained_tiles"] + li["repetitive_heads"] * anchor_tiles_per_head
    o = None

    def call(q, k, v, o, t, l):
        C.calibatt_dual_path_attn(q, k, v, o, dct, t, l, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block,
                                  stream=stream)

    q, k, v = W.make_qkv(W.seed_for("sweep-qkv", 0, 0) % (1 << 62), 1, wl.seq_len, H, wl.head_dim, "bf16",
                         wl.input_std, "cuda")
    o = torch.empty_like(q)
    for _ in range(args.warmup):
        call(q, k, v, o, 0, 0)
    torch.cuda.synchronize()
    evs = []
    with ClockSampler(0) as clk:
        for t in range(T):
            for l in range(L):
                del q, k, v
                q, k, v = W.make_qkv(W.seed_for("sweep-qkv", t, l) % (1 << 62), 1, wl.seq_len, H, wl.head_dim,
                                     "bf16", wl.input_std, "cuda")
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                call(q, k, v, o, t, l)
                b.record(stream)
                evs.append((a, b))
        torch.cuda.synchronize()
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out during the sweep")
    per_call = [a.elapsed_time(b) for a, b in evs]
    sparse_s = sum(per_call) / 1e3
    # dense path: all-ones masks for every head, on the inputs of a sample of the calls
    ones = [np.ones((nb, nb), bool)] * H
    d_dense = build_dict(C, ones, H, nb, wl.block)
    dense_tiles = d_dense.layer_info(0, 0)["retained_tiles"]
    picks = [(i * T // max(1, args.dense_sample), (i * 7) % L) for i in range(min(args.dense_sample, T * L))]
    dense_ms = []
    for t, l in picks:
        q2, k2, v2 = W.make_qkv(W.seed_for("sweep-qkv", t, l) % (1 << 62), 1, wl.seq_len, H, wl.head_dim, "bf16",
                                wl.input_std, "cuda")
        dense_ms.append(statistics.mean(time_calls(
            torch, lambda: C.calibatt_block_sparse_attn(q2, k2, v2, o, d_dense, 0, 0, wl.block, stream=stream),
            1, 1, stream)))
        del q2, k2, v2
    d_dense.close()
    dense_s = statistics.mean(dense_ms) * T * L / 1e3
    value = tiles * FLOP_PER_TILE / sparse_s / 1e12
    line = {
        "metric": "effective TFLOP/s (retained blocks) and ms/call, % of B200 BF16 tensor peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": T * L, "warmup": args.warmup,
        "ms_per_step": sparse_s * 1e3 / (T * L), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "wan2.1-14b-720p schedule sweep, dual path (block-sparse + anchor heads)",
                   "timesteps": T, "layers": L, "heads": H, "repetitive_heads_per_call": W.SWEEP_REPETITIVE,
                   "anchors": list(wl.anchors), "density": "0.60 -> 0.20 over the timesteps",
                   "dictionary_format": DICT_FORMAT,
                   "inputs": "fresh seeded Q/K/V per call (2.32 GB > L2)", "parallelism": "replicas x1"},
        "pct_of_peak": value / pk["bf16_tflops"],
        "clocks": clk.summary(),
        "sweep": {"sparse_total_s": sparse_s, "dense_total_s": dense_s,
                  "dense_total_basis": f"mean of {len(dense_ms)} sampled calls x {T * L} calls",
                  "dense_ms_per_call": statistics.mean(dense_ms), "speedup_vs_dense": dense_s / sparse_s,
                  "effective_tiles": tiles, "dense_tiles_per_call": dense_tiles,
                  "dictionary_device_bytes": info["device_bytes"], "dictionary_blocks": info["nnz"],
                  "dictionary_build_s": build_s,
                  "min_ms_per_call": min(per_call), "max_ms_per_call": max(per_call)},
        "gpu_launches": T * L,
    }
    print(json.dumps(line), flush=True)
    dct.close()


def device_csr(C, torch, masks, heads, nb):
    """Device row_ptr / 16-bit col_idx / col_base of per-head bool masks and
    the host row_ptr (the direct-CSR call's inputs)."""
    rp, ci, _ = C.masks_to_layer_csr(masks, heads, nb)
    base = np.zeros(heads, np.int64)
    base[1:] = np.cumsum(rp[:, -1].astype(np.int64))[:-1]
    col = ci.astype(np.uint16).view(np.int16) if ci.size else np.zeros(1, np.int16)
    return (torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(), torch.from_numpy(base).cuda(), rp)


def run_format_ab(torch, C, stream, wl, masks, q, k, v, o, tiles, rounds=6, calls=2):
    """The headline call over the three dictionary formats of the same masks
    (index lists, bitmap, intervals), interleaved round by round so that the
    power-capped clock drifts alike for all three; median ms per format, the
    dictionary's device bytes, and whether the outputs are bitwise equal."""
    dicts = {f: build_dict(C, [masks[h] for h in range(wl.heads)], wl.heads, wl.num_blocks, wl.block, fmt=f)
             for f in ("lists", "bitmap", "intervals")}
    outs = {}
    for f, d in dicts.items():
        C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block, stream=stream)
        torch.cuda.synchronize()
        outs[f] = o.clone()
    same = all(torch.equal(outs["lists"], outs[f]) for f in outs)
    del outs
    ms = {f: [] for f in dicts}
    for _ in range(rounds):
        for f, d in dicts.items():
            ms[f] += time_calls(torch, lambda: C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block,
                                                                            stream=stream), calls, 1, stream)
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the dictionary-format comparison")
    res = {"interleaved": f"{rounds} rounds x {calls} calls per format", "outputs_bitwise_equal": same}
    for f, d in dicts.items():
        med = statistics.median(ms[f])
        res[f] = {"ms_per_call": med, "effective_tflops": tiles * FLOP_PER_TILE / (med * 1e-3) / 1e12,
                  "device_bytes": d.info()["device_bytes"]}
        d.close()
    return res


def run_480p_leg(args, torch, C, stream, pk):
    """The 480p block-sparse layer (21 x 30 x 52 = 32,760 tokens, 40 heads),
    timed like the headline call: ms per call, effective TFLOP/s and the
    fraction of the tensor peak."""
    wl = W.WORKLOADS["480p"]
    masks, _ = W.workload_masks(wl)
    q, k, v = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    o = torch.empty_like(q)
    d = build_dict(C, [masks[h] for h in range(wl.heads)], wl.heads, wl.num_blocks, wl.block)
    tiles = d.layer_info(0, 0)["retained_tiles"]
    per_call = time_calls(torch, lambda: C.calibatt_block_sparse_attn(q, k, v, o, d, 0, 0, wl.block, stream=stream),
                          max(5, args.steps), 3, stream)
    d.close()
    ms = statistics.mean(per_call)
    tf = tiles * FLOP_PER_TILE / (ms * 1e-3) / 1e12
    return {"workload": "wan2.1-14b-480p self-attention, block-sparse path", "seq_len": wl.seq_len,
            "heads": wl.heads, "retained_tiles": tiles, "density": round(tiles / (wl.heads * wl.num_blocks ** 2), 4),
            "ms_per_call": ms, "effective_tflops": tf, "frac_of_burst_peak": tf / pk["bf16_tflops"],
            "l2": "inputs 1.0 GB > 126 MB L2, no flush"}


def run_tiny_leg(torch, C):
    """The tiny configuration in full, on the GPU and on the oracle: head 0
    block-sparse, head 1 on the anchor path (anchors 0 and 4), float32, block
    64; then block energies of 4 seeded Q/K draws, selection at tau = 0.99 and
    their union.  Oracle wall time of the whole configuration, GPU device time
    of the same calls, and the largest output difference."""
    from oracle import calibatt_oracle as O

    wl = W.WORKLOADS["tiny"]
    masks, rep = W.workload_masks(wl)
    nb = wl.num_blocks
    q, k, v = W.make_qkv(wl.seed, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "fp32", wl.input_std, "cuda")
    draws = [W.make_qkv(s, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "fp32", wl.input_std, "cuda")[:2]
             for s in (10, 11, 12, 13)]
    o = torch.empty_like(q)
    d = build_dict(C, [masks[h] for h in range(wl.heads)], wl.heads, nb, wl.block)
    e = torch.empty((wl.batch, wl.heads, nb, nb), device="cuda")
    ws = torch.empty(C.calibatt_block_energy_workspace_size(q) // 4, device="cuda")
    sel = torch.empty((wl.batch * wl.heads * nb, nb), dtype=torch.uint8, device="cuda")
    cnt = torch.zeros((wl.batch * wl.heads * nb, nb), dtype=torch.int32, device="cuda")
    union = torch.empty_like(sel)

    def gpu_call():
        C.calibatt_dual_path_attn(q, k, v, o, d, 0, 0, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block)
        cnt.zero_()
        for dq, dk in draws:
            C.calibatt_block_energy(dq, dk, e, ws, wl.block)
            C.calibatt_select_blocks(e.view(-1, nb), 0.99, sel, cnt)
        C.calibatt_aggregate_masks(cnt, 4, 0.25, union)

    gpu_ms = statistics.median(time_calls(torch, gpu_call, 20, 3, torch.cuda.current_stream()))
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the tiny configuration")
    d.close()
    f64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)  # noqa: E731
    qn, kn, vn = f64(q), f64(k), f64(v)
    dn = [(f64(a), f64(b)) for a, b in draws]
    t0 = time.perf_counter()
    sparse_heads = [h for h in range(wl.heads) if masks[h] is not None]
    ref_s, _ = O.block_sparse_attention_bnhd(qn, kn, vn, masks, wl.block, heads=sparse_heads)
    ref_a = O.anchor_attention_bnhd(qn, kn, vn, wl.frames, wl.rows, wl.cols, wl.anchors, heads=list(rep))
    ref_sel = [O.select_blocks(O.block_energy_bnhd(a, b, wl.block).reshape(-1, nb), float(np.float32(0.99)))
               for a, b in dn]
    ref_union = O.aggregate_masks(np.stack(ref_sel), 4, 0.25)
    oracle_s = time.perf_counter() - t0
    out = f64(o)
    err = max(float(np.abs(out[:, :, sparse_heads] - ref_s).max()),
              float(np.abs(out[:, :, list(rep)] - ref_a).max()))
    return {"workload": "tiny: 2 frames x 8 rows x 16 cols, 2 heads (block-sparse + anchor), head_dim 64, "
                        "fp32, block 64; energy of 4 draws, tau 0.99, union",
            "gpu_ms": gpu_ms, "oracle_ms": oracle_s * 1e3, "oracle_cores": os.cpu_count(),
            "max_abs_err": err, "tolerance": 1e-4, "within_tolerance": err <= 1e-4,
            "union_equal": bool((union.cpu().numpy().astype(bool) == ref_union).all())}


SWEEP_SAMPLE_CALLS = 100
SWEEP_SAMPLE_DENSE = 10


def sweep_sample_picks(n_calls, steps=W.SWEEP_STEPS, layers=W.SWEEP_LAYERS):
    """(timestep, layer) calls of a sample of the schedule sweep: the same
    number of calls at every timestep (so the density ramp is sampled evenly),
    layers spread over the schedule."""
    per_t = max(1, n_calls // steps)
    return [(t, (7 * t + j * layers // per_t) % layers) for t in range(steps) for j in range(per_t)][:n_calls]


def run_sweep_sample(torch, C, stream, pk, n_calls=SWEEP_SAMPLE_CALLS, n_dense=SWEEP_SAMPLE_DENSE):
    """A sample of the schedule sweep (n_calls of its 2,000 dual-path 720p
    calls, fresh seeded Q/K/V per call, masks and repetitive heads exactly as
    the full sweep draws them), with the dense path timed on n_dense of the
    calls.  The aggregate ratio over the schedule is estimated as (mean dense
    ms) / (mean dual-path ms) of the sample."""
    wl = W.WORKLOADS["720p_sweep"]
    picks = sweep_sample_picks(n_calls)
    H, nb = wl.heads, wl.num_blocks
    nnz = sum(W.sweep_record_blocks(wl, t, l, h) for t, l in picks for h in range(H))
    dct = C.MaskDictionary(len(picks), 1, H, nb, nb, wl.block, nnz)
    dct.set_anchor_geometry(wl.frames, wl.rows, wl.cols, wl.anchors)
    for i, (t, l) in enumerate(picks):
        masks, rep = W.sweep_layer_masks(wl, t, l, "cuda")
        rp, ci = W.layer_csr(masks)
        rep_arr = np.zeros(H, np.uint8)
        rep_arr[list(rep)] = 1
        dct.set_layer(i, 0, rp, ci, rep_arr)
    anchor_tiles_per_head = -(-wl.frames * len(wl.anchors) * wl.cols // 128) * nb
    tiles = []
    for i in range(len(picks)):
        li = dct.layer_info(i, 0)
        tiles.append(li["retained_tiles"] + li["repetitive_heads"] * anchor_tiles_per_head)
    o = None
    per_call = []
    for i, (t, l) in enumerate(picks):
        q, k, v = W.make_qkv(W.seed_for("sweep-qkv", t, l) % (1 << 62), 1, wl.seq_len, H, wl.head_dim, "bf16",
                             wl.input_std, "cuda")
        if o is None:
            o = torch.empty_like(q)
            for _ in range(3):
                C.calibatt_dual_path_attn(q, k, v, o, dct, i, 0, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block,
                                          stream=stream)
        per_call.append(statistics.mean(time_calls(
            torch, lambda: C.calibatt_dual_path_attn(q, k, v, o, dct, i, 0, wl.frames, wl.rows, wl.cols, wl.anchors,
                                                     wl.block, stream=stream), 1, 0, stream)))
        del q, k, v
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out in the sweep sample")
    dct.close()
    ones = [np.ones((nb, nb), bool)] * H
    d_dense = build_dict(C, ones, H, nb, wl.block)
    dense_tiles = d_dense.layer_info(0, 0)["retained_tiles"]
    dense_ms = []
    for t, l in picks[::max(1, len(picks) // n_dense)][:n_dense]:
        q, k, v = W.make_qkv(W.seed_for("sweep-qkv", t, l) % (1 << 62), 1, wl.seq_len, H, wl.head_dim, "bf16",
                             wl.input_std, "cuda")
        dense_ms.append(statistics.mean(time_calls(
            torch, lambda: C.calibatt_block_sparse_attn(q, k, v, o, d_dense, 0, 0, wl.block, stream=stream),
            1, 1, stream)))
        del q, k, v
    d_dense.close()
    sparse_mean = statistics.mean(per_call)
    dense_mean = statistics.mean(dense_ms)
    calls = W.SWEEP_STEPS * W.SWEEP_LAYERS
    return {"workload": f"wan2.1-14b-720p schedule sweep, sample of {len(picks)} of its {calls} dual-path calls "
                        f"({len(picks) // W.SWEEP_STEPS} per timestep), dense path on {len(dense_ms)} of them",
            "ms_per_call": sparse_mean, "dense_ms_per_call": dense_mean,
            "speedup_vs_dense": dense_mean / sparse_mean,
            "estimated_total_s": sparse_mean * calls / 1e3, "estimated_dense_total_s": dense_mean * calls / 1e3,
            "effective_tflops": sum(tiles) * FLOP_PER_TILE / (sum(per_call) * 1e-3) / 1e12,
            "dense_tiles_per_call": dense_tiles,
            "min_ms_per_call": min(per_call), "max_ms_per_call": max(per_call)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the dense / dual-path / e2e legs")
    ap.add_argument("--heads", type=int, default=40,
                    help="heads of the 720p layer (fewer heads = smaller case for profiling); with --dual-case "
                         "and --anchor-case the dual-path layer's first heads")
    ap.add_argument("--workload", default="720p", choices=["720p", "sweep"],
                    help="sweep: the mask-dictionary schedule sweep (one dual-path 720p call per "
                         "timestep and layer), reported as aggregate time against the dense path")
    ap.add_argument("--dict-format", default="lists", choices=["lists", "bitmap", "intervals"],
                    help="mask dictionary storage: 2-byte index lists, one bit per block pair, or each "
                         "row's contiguous key-block intervals")
    ap.add_argument("--sweep-steps", type=int, default=W.SWEEP_STEPS)
    ap.add_argument("--sweep-layers", type=int, default=W.SWEEP_LAYERS)
    ap.add_argument("--epilogue-probe", action="store_true",
                    help="time the anchor broadcast epilogue with the library's measurement build "
                         "(-DCALIBATT_TRACE) and print its store rate")
    ap.add_argument("--epilogue-fused", action="store_true",
                    help="with --epilogue-probe: the anchor tiles of the fused dual-path launch")
    ap.add_argument("--softmax-phases", action="store_true",
                    help="trace the softmax streams of the block-sparse kernel with the library's measurement "
                         "build (-DCALIBATT_TRACE) and print their per-block phase breakdown")
    ap.add_argument("--similarity-case", action="store_true",
                    help="time the spatial-similarity pass alone (720p geometry, --heads heads)")
    ap.add_argument("--energy-case", action="store_true",
                    help="time the block energy alone (720p geometry, --heads heads)")
    ap.add_argument("--dual-case", action="store_true",
                    help="time the dual-path 720p layer alone (one fused launch of both paths)")
    ap.add_argument("--layout", default="bnhd", choices=["bnhd", "bhnd"],
                    help="storage of Q, K, V, O for the 720p call: token-major [B, N, H, D] (default) or "
                         "head-major [B, H, N, D] (the same logical tensors, other strides)")
    ap.add_argument("--dual-launches", type=int, default=1, choices=[1, 2],
                    help="--dual-case as one fused launch (1) or block-sparse + anchor launches (2)")
    ap.add_argument("--anchor-case", action="store_true",
                    help="time the anchor path alone (the 12 repetitive heads of the dual-path 720p layer)")
    ap.add_argument("--partition", default="replicas", choices=["replicas", "heads"],
                    help="with N > 1 ranks: every rank times its own 720p layer (replicas, weak scaling), or "
                         "the ranks split the 40 heads of ONE call, rank r taking heads r, r+N, ... (strong "
                         "scaling, each rank reading only its heads' Q/K/V)")
    ap.add_argument("--dense-sample", type=int, default=50,
                    help="sweep calls also timed on the dense path (its time does not depend on the masks)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    global DICT_FORMAT
    DICT_FORMAT = args.dict_format

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from calibrated_block_sparse_calibatt_b200 import build as B

    B.build()
    from calibrated_block_sparse_calibatt_b200 import calibatt as C

    pk = peaks()
    stream = torch.cuda.current_stream()
    if args.epilogue_probe:
        run_epilogue_probe(torch, B, C, fused=args.epilogue_fused)
        return
    if args.softmax_phases:
        run_softmax_phases(args, torch, B, C)
        return
    if args.anchor_case:
        run_anchor_case(args, torch, C, pk)
        return
    if args.dual_case:
        run_dual_case(args, torch, C, pk)
        return
    if args.similarity_case:
        run_similarity_case(args, torch, C, pk)
        return
    if args.energy_case:
        run_energy_case(args, torch, C, pk)
        return
    if args.workload == "sweep":
        if world > 1:
            raise SystemExit("the sweep workload runs on one GPU")
        run_sweep(args, C, torch, stream, pk)
        return
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["720p"], heads=args.heads)
    masks, _ = W.workload_masks(wl, seed_base=W.MASK_SEED_BASE["720p"])
    by_heads = args.partition == "heads"
    # under --partition heads every rank holds the same call's inputs and
    # computes only its heads of it
    q, k, v = W.make_qkv(wl.seed if by_heads else rank_seed(wl.seed, rank), 1, wl.seq_len, wl.heads, wl.head_dim,
                         "bf16", wl.input_std, "cuda")
    if args.layout == "bhnd":
        # the same [batch, N, heads, head_dim] tensors stored head-major: a head's
        # rows are contiguous (stride_n = head_dim) instead of heads*head_dim apart
        q, k, v = (t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3) for t in (q, k, v))
    o = torch.empty_like(q)
    d_sparse = build_dict(C, [masks[h] for h in range(wl.heads)], wl.heads, wl.num_blocks, wl.block)
    tiles = d_sparse.layer_info(0, 0)["retained_tiles"]
    flop = tiles * FLOP_PER_TILE
    density = tiles / (wl.heads * wl.num_blocks ** 2)

    def sparse_call():
        C.calibatt_block_sparse_attn(q, k, v, o, d_sparse, 0, 0, wl.block, stream=stream)

    my_heads = head_partition(wl.heads, rank, world) if by_heads else list(range(wl.heads))
    my_tiles = tiles
    if by_heads:
        # this rank's share of the call: the direct-CSR call over its heads
        # (device lists of every head, a schedule of its heads only)
        rp_d, col_d, base_d, rp_h = device_csr(C, torch, [masks[h] for h in range(wl.heads)], wl.heads,
                                               wl.num_blocks)
        items, cta_ptr = C.csr_schedule(rp_h, my_heads, C.device_sm_count())
        part_args = (rp_d, col_d, base_d, my_heads, torch.from_numpy(items.view(np.int32)).cuda(),
                     torch.from_numpy(cta_ptr).cuda(), cta_ptr.size - 1)
        my_tiles = int(sum(int(rp_h[h, -1]) for h in my_heads))

        def sparse_call():  # noqa: F811
            C.calibatt_block_sparse_attn_csr(q, k, v, o, *part_args, block=wl.block, stream=stream)

    # ---------------------------------------------------------------- timed region
    for _ in range(args.warmup):
        sparse_call()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        per_call = time_calls(torch, sparse_call, args.steps, 0, stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    if C.device_status() != 0:
        raise RuntimeError("device wait timed out during the benchmark")
    total_ms = max_over_ranks(sum(per_call), dist, "cuda")
    ms = total_ms / args.steps
    # replicas: every rank did a whole call; heads: the ranks together did one
    value = flop / (ms * 1e-3) / 1e12 if by_heads else aggregate_tflops(flop, world, ms)
    avg_launch_ms = statistics.mean(per_call)
    achieved = my_tiles * FLOP_PER_TILE / (avg_launch_ms * 1e-3) / 1e12

    extras = {}
    if by_heads:
        extras["head_partition"] = {"heads_this_rank": my_heads, "tiles_this_rank": my_tiles,
                                    "api": "calibatt_block_sparse_attn_csr with this rank's head_ids"}
    if not args.no_extras and not by_heads:
        # the anchor path alone: the dual-path layer's 12 repetitive heads on
        # the same inputs, with the workspace that splits its last wave of
        # tiles, timed like the headline call (steps calls back to back)
        wa = W.WORKLOADS["720p_dual"]
        _, a_heads = W.workload_masks(wa)
        a_ws = anchor_workspace(torch, C, q, wa, len(a_heads))
        a_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_anchor_attn(q, k, v, o, wa.frames, wa.rows, wa.cols, wa.anchors,
                                                  list(a_heads), workspace=a_ws, stream=stream),
            args.steps, args.warmup, stream)), dist, "cuda")
        a_tiles = len(a_heads) * -(-wa.frames * len(wa.anchors) * wa.cols // 128) * wa.num_blocks
        a_tf = a_tiles * FLOP_PER_TILE / (a_ms * 1e-3) / 1e12
        del a_ws
        extras["anchor_720p"] = {"heads": len(a_heads), "anchor_tiles_x_key_blocks": a_tiles, "ms_per_call": a_ms,
                                 "effective_tflops": a_tf, "frac_of_burst_peak": a_tf / pk["bf16_tflops"],
                                 "timing": f"{args.steps} calls back to back after {args.warmup} warm-up calls",
                                 "api": "calibatt_anchor_attn with its split workspace"}
        # dense path on the same inputs: all-ones skip lists held on the device,
        # through the direct-CSR call (no dictionary)
        nbk, hh = wl.num_blocks, wl.heads
        rp = np.tile((np.arange(nbk + 1) * nbk).astype(np.int32), (hh, 1))
        items, cta_ptr = C.csr_schedule(rp, list(range(hh)), C.device_sm_count())
        dense_args = (torch.from_numpy(rp).cuda(), torch.arange(nbk, dtype=torch.int16, device="cuda").repeat(hh * nbk),
                      torch.arange(hh, dtype=torch.int64, device="cuda") * nbk * nbk, list(range(hh)),
                      torch.from_numpy(items.view(np.int32)).cuda(), torch.from_numpy(cta_ptr).cuda(),
                      cta_ptr.size - 1)
        dense_tiles = q.shape[0] * hh * nbk * nbk
        dense_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_block_sparse_attn_csr(q, k, v, o, *dense_args, block=wl.block, stream=stream),
            max(3, args.steps // 4), 2, stream)), dist, "cuda")
        del dense_args
        extras["dense"] = {"ms_per_call": dense_ms,
                           "tflops": dense_tiles * FLOP_PER_TILE / (dense_ms * 1e-3) / 1e12,
                           "speedup_sparse_vs_dense": dense_ms / ms,
                           "api": "calibatt_block_sparse_attn_csr, all-ones lists"}
        # dual-path 720p layer: 12 anchor heads + 28 sparse heads
        wd = W.WORKLOADS["720p_dual"]
        dmasks, rep_heads = W.workload_masks(wd)
        geom = (wd.frames, wd.rows, wd.cols, wd.anchors)
        d_dual = build_dict(C, [dmasks[h] for h in range(wd.heads)], wd.heads, wd.num_blocks, wd.block, geom)
        d_two = build_dict(C, [dmasks[h] for h in range(wd.heads)], wd.heads, wd.num_blocks, wd.block)
        dual_tiles = d_dual.layer_info(0, 0)["retained_tiles"]
        anchor_tiles = len(rep_heads) * -(-wd.frames * len(wd.anchors) * wd.cols // 128) * wd.num_blocks
        dual_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_dual_path_attn(q, k, v, o, d_dual, 0, 0, wd.frames, wd.rows, wd.cols,
                                                     wd.anchors, wd.block, stream=stream),
            max(3, args.steps // 4), 2, stream)), dist, "cuda")
        two_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_dual_path_attn(q, k, v, o, d_two, 0, 0, wd.frames, wd.rows, wd.cols,
                                                     wd.anchors, wd.block, stream=stream),
            max(3, args.steps // 4), 2, stream)), dist, "cuda")
        d_two.close()
        # the anchor path alone, with the workspace that splits its last wave
        # of tiles and, for comparison, every tile whole: interleaved, the
        # order alternating round by round, so the power-capped clock drifts
        # alike for both
        a_ws = anchor_workspace(torch, C, q, wd, len(rep_heads))
        a_ms = {True: [], False: []}
        for rnd in range(6):
            for split in ((True, False) if rnd % 2 == 0 else (False, True)):
                a_ms[split] += time_calls(
                    torch, lambda: C.calibatt_anchor_attn(q, k, v, o, wd.frames, wd.rows, wd.cols, wd.anchors,
                                                          list(rep_heads), workspace=a_ws if split else None,
                                                          stream=stream),
                    2, 1, stream)
        anchor_ms = max_over_ranks(statistics.median(a_ms[True]), dist, "cuda")
        anchor_whole_ms = max_over_ranks(statistics.median(a_ms[False]), dist, "cuda")
        del a_ws
        d_dual.close()
        bcast_bytes = len(rep_heads) * wd.seq_len * wd.head_dim * 2
        anchor_tf = anchor_tiles * FLOP_PER_TILE / (anchor_ms * 1e-3) / 1e12
        extras["dual_path_720p"] = {
            "ms_per_call": dual_ms, "launches": 1, "two_launch_ms_per_call": two_ms,
            "effective_tflops": (dual_tiles + anchor_tiles) * FLOP_PER_TILE / (dual_ms * 1e-3) / 1e12,
            "anchor_heads": len(rep_heads), "anchor_ms": anchor_ms,
            "anchor_effective_tflops": anchor_tf, "anchor_frac_of_burst_peak": anchor_tf / pk["bf16_tflops"],
            "anchor_whole_tiles_ms": anchor_whole_ms, "anchor_output_bytes": bcast_bytes}
        # offline calibration: block energies of the dense attention (two Q K^T passes on the tensor cores)
        e_out = torch.empty((1, wl.heads, wl.num_blocks, wl.num_blocks), device="cuda")
        e_ws = torch.empty(C.calibatt_block_energy_workspace_size(q) // 4, device="cuda")
        energy_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_block_energy(q, k, e_out, e_ws, wl.block, stream=stream),
            3, 1, stream)), dist, "cuda")
        del e_out, e_ws
        exp2_per_call = 2 * wl.seq_len ** 2 * wl.heads      # both passes exponentiate every score
        sms = C.device_sm_count()
        ex2_peak = mufu_exp2_peak(sms, 1965.0)
        extras["block_energy_720p"] = {
            "ms_per_call": energy_ms, "heads": wl.heads,
            "tflops_two_qk_passes": 2 * 2.0 * wl.seq_len ** 2 * wl.head_dim * wl.heads / (energy_ms * 1e-3) / 1e12,
            "exp2_per_call": exp2_per_call,
            "roofline": {"bound": "mufu", "achieved": exp2_per_call / (energy_ms * 1e-3) / 1e9,
                         "peak": ex2_peak / 1e9, "unit": "G exp2/s",
                         "frac": exp2_per_call / (energy_ms * 1e-3) / ex2_peak,
                         "peak_basis": f"{EX2_PER_CLK_PER_SM} exp2/clk/SM x {sms} SMs x 1965 MHz (max SM clock); "
                                       "one exp2 pair in four runs on the FMA pipe and is counted all the same"}}
        # offline calibration: spatial-repetition scores of every (frame, row) of the 720p layer
        wd_ = W.WORKLOADS["720p_dual"]
        sim_out = torch.empty((1, wl.heads, wd_.frames, wd_.rows), device="cuda")
        sim_ws = torch.empty(C.calibatt_spatial_similarity_workspace_size(q) // 4, device="cuda")
        sim_ms = max_over_ranks(statistics.mean(time_calls(
            torch, lambda: C.calibatt_spatial_similarity(q, k, sim_out, sim_ws, wd_.frames, wd_.rows, wd_.cols,
                                                         wd_.anchors, stream=stream),
            3, 1, stream)), dist, "cuda")
        del sim_out, sim_ws
        # the LSE pass exponentiates every score once, the pass of sums twice
        # (each query's and its anchor-row partner's)
        sim_exp2 = 3 * wl.seq_len ** 2 * wl.heads
        extras["spatial_similarity_720p"] = {
            "ms_per_call": sim_ms, "heads": wl.heads, "frames_x_rows": wd_.frames * wd_.rows,
            "exp2_per_call": sim_exp2,
            "tflops_three_qk_passes": 3 * 2.0 * wl.seq_len ** 2 * wl.head_dim * wl.heads / (sim_ms * 1e-3) / 1e12,
            "roofline": {"bound": "mufu", "achieved": sim_exp2 / (sim_ms * 1e-3) / 1e9, "peak": ex2_peak / 1e9,
                         "unit": "G exp2/s", "frac": sim_exp2 / (sim_ms * 1e-3) / ex2_peak,
                         "peak_basis": f"{EX2_PER_CLK_PER_SM} exp2/clk/SM x {sms} SMs x 1965 MHz (max SM clock)"}}
        if C.device_status() != 0:
            raise RuntimeError("device wait timed out during the extra legs")
        if world == 1:
            extras["dictionary_formats"] = run_format_ab(torch, C, stream, wl, masks, q, k, v, o, tiles)
            extras["cfg_480p"] = run_480p_leg(args, torch, C, stream, pk)
            extras["cfg_tiny"] = run_tiny_leg(torch, C)
            extras["sweep_sample"] = run_sweep_sample(torch, C, stream, pk)

    # -------------------------------------------------------- end to end (host buffers)
    # Every step is one calibatt_block_sparse_attn_host call: its Q, K, V are
    # copied from pinned host memory into a device buffer set, the attention
    # runs, and O is copied back to pinned host memory, in stream order.
    # Consecutive steps rotate over three streams and three buffer sets, so
    # the copies of one step overlap the attention of the neighbouring ones
    # and the next step's input copy never queues behind an output copy
    # (2.3% faster than two sets; the link then carries ~64 GB/s both ways).
    e2e = None
    if not args.no_extras and not by_heads:
        n_sets = 3
        if args.layout == "bnhd":
            hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
            hos = [torch.empty_like(o, device="cpu").pin_memory() for _ in range(n_sets)]
        else:
            # pinned host tensors with the device tensors' strides (the host call
            # copies each tensor's byte extent as it lies)
            def pinned(t):
                return torch.empty_strided(t.size(), t.stride(), dtype=t.dtype, pin_memory=True)
            hq, hk, hv = (pinned(t).copy_(t) for t in (q, k, v))
            hos = [pinned(o) for _ in range(n_sets)]
        dsets = [[torch.empty_like(q) for _ in range(4)] for _ in range(n_sets)]
        streams = [torch.cuda.Stream() for _ in range(n_sets)]
        e2e_steps = max(6, args.steps // 2)

        def run_pipeline(n_steps):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(streams[0])
            for st in streams[1:]:
                st.wait_event(t0)
            for i in range(n_steps):
                b = i % n_sets
                dq, dk, dv, do = dsets[b]
                C.calibatt_block_sparse_attn_host(hq, hk, hv, hos[b], dq, dk, dv, do, d_sparse, 0, 0, wl.block,
                                                  stream=streams[b])
            for st in streams[1:]:
                end = torch.cuda.Event()
                end.record(st)
                streams[0].wait_event(end)
            t1.record(streams[0])
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        run_pipeline(n_sets + 1)                             # warm-up
        e2e_ms = max_over_ranks(run_pipeline(e2e_steps) / e2e_steps, dist, "cuda")
        nbytes = 3 * q.numel() * q.element_size()
        e2e = {"value": aggregate_tflops(flop, world, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": o.numel() * o.element_size(),
               "steps": e2e_steps, "api": "calibatt_block_sparse_attn_host, steps rotating over three streams and buffer sets"}
        if C.device_status() != 0:
            raise RuntimeError("device wait timed out during the end-to-end leg")
        del hq, hk, hv, hos, dsets

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not by_heads:
        # the block-sparse output of this run's inputs (the extra legs reused o)
        C.calibatt_block_sparse_attn(q, k, v, o, d_sparse, 0, 0, wl.block, stream=stream)
        torch.cuda.synchronize()
        cpu, parity = cpu_baseline(wl, masks, q, k, v, o)

    if rank == 0:
        line = {
            "metric": "effective TFLOP/s (retained blocks) and ms/call, % of B200 BF16 tensor peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "strong" if by_heads else "weak",
            "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "wan2.1-14b-720p self-attention, block-sparse path", "batch": 1,
                       "dictionary_format": DICT_FORMAT,
                       "heads": wl.heads, "head_dim": wl.head_dim, "seq_len": wl.seq_len, "block": wl.block,
                       "density": round(density, 4), "retained_tiles": tiles,
                       "l2": "inputs 2.32 GB > 126 MB L2, no flush",
                       "parallelism": f"heads split over {world} ranks" if by_heads else f"replicas x{world}",
                       "storage": "[batch, N, heads, head_dim]" if args.layout == "bnhd"
                       else "[batch, heads, N, head_dim] (head-major)"},
            "pct_of_peak": achieved / pk["bf16_tflops"],
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"],
                         # counters were taken on the default (token-major) storage
                         "traffic": measured_traffic(my_tiles) if args.layout == "bnhd" and not by_heads else None,
                         "traffic_unit": "bytes per launch (DRAM read + write)",
                         "algorithmic_bytes": 4 * q.numel() * q.element_size(),
                         "peak_source": f"{pk['source']} burst bf16",
                         # the timed calls run long enough for the power cap to lower the clock,
                         # the regime of the sustained figure: given alongside, not instead
                         "peak_sustained": pk["bf16_tflops_sustained"],
                         "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"]
                                               if pk["bf16_tflops_sustained"] else None)},
            "clocks": clk.summary(),
            "e2e": e2e,
            # the direct-CSR call of --partition heads also launches its list and schedule checks
            "gpu_launches": args.steps * (3 if by_heads else 1),
            "cpu_baseline": cpu,
            "parity": parity,
            **extras,
        }
        print(json.dumps(line), flush=True)
    d_sparse.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
