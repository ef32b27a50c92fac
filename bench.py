#!/usr/bin/env python
"""Benchmark of the Sparse VideoGen sparse-attention layer on B200.

One step = the whole hot path on one synthetic layer resident in HBM:
online profiling (+ its finalize kernel), block-mask construction for both
patterns, permutation of Q/K/V for temporal heads, block-sparse attention and
the inverse permutation of the temporal outputs.

Prints ONE JSON line (rank 0). `value` is TFLOP/s counted on computed blocks
(4*d per attended (query, key) pair, all heads, all ranks) divided by the
measured step time; `roofline` reports the attention kernel alone. The dense
baseline is the same attention kernel over the all-blocks mask.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import svg_inputs as SI  # noqa: E402

METRIC = "sparse-attn layer ms & TFLOPS (computed blocks) vs BF16 peak; speedup vs dense"
UNIT = "TFLOP/s (computed blocks)"
DEFAULT_WORKLOAD = SI.HUNYUAN.name
# the semantic-aware (SVG2) measurement: clusters of queries and keys, Lloyd
# iterations and the kept share of the centroid attention
SVG2_CQ, SVG2_CK, SVG2_ITERS, SVG2_TOP_P = 256, 256, 10, 0.9
SVG2_EAR_TAU = 0.01  # SVG-EAR: route skipped cluster pairs whose estimated error exceeds it


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return {"bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "hbm_gbs": pk["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "source": "fallback"}


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def _sources_digest(files) -> str:
    import hashlib
    paths = [os.path.join(ROOT, "video_dit_spatial_b200", "csrc", f) for f in files]
    return hashlib.sha256(b"".join(open(f, "rb").read() for f in paths)).hexdigest()[:16]


def _captured_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per full-size launch of `kernel` on `workload`
    from profiles/traffic.json (written from an ncu capture), or None when there
    is no entry or the kernel's sources changed since that capture."""
    try:
        entries = json.load(open(TRAFFIC_JSON))
    except (OSError, ValueError):
        return None
    e = entries.get(kernel)
    if not e or e.get("workload") != workload:
        return None
    try:
        if _sources_digest(e["sources"]) != e["sources_sha256_16"]:
            return None
    except OSError:
        return None
    return int(e["traffic_bytes_per_launch_full_size"])


def percentiles(ms_list):
    """p10 / p50 / p90 (linear interpolation) and the mean of a list of ms."""
    a = np.asarray(ms_list, dtype=np.float64)
    return {"p10": float(np.percentile(a, 10)), "p50": float(np.percentile(a, 50)),
            "p90": float(np.percentile(a, 90)), "mean": float(a.mean()), "n": int(a.size)}


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, dist, device) -> float:
    """The largest value over all ranks (every rank takes the same collective)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def computed_pairs(svg, g, kind) -> int:
    """(query, key) token pairs inside the computed blocks of one head."""
    from video_dit_spatial_b200.layer import BlockMaskCSR
    m = BlockMaskCSR(g, kind, "cuda")
    m.build(g)
    rp = m.row_ptr.cpu().numpy().astype(np.int64)
    ci = m.col_idx.cpu().numpy()[:m.nnz].astype(np.int64)
    N = g.N
    rows_in = np.minimum(g.block_q, N - np.arange(g.n_qblocks) * g.block_q)
    cols_in = np.minimum(g.block_k, N - np.arange(g.n_kblocks) * g.block_k)
    counts = np.diff(rp)
    return int(np.sum(np.repeat(rows_in, counts) * cols_in[ci]))


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", ident], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, flag in zip(names, parts[5:9]):
                    if flag.lower().startswith("active"):
                        reasons.add(n)
            os.unlink(self.path)
        except Exception:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline, and the --impl reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(wl, n_rows: int, heads, seed: int = 5):
    """Times the fp64 oracle's layer output on n_rows query rows of `heads`.

    Returns (seconds, flops) with flops = 4*d*attended keys of those rows.
    """
    import oracle as O
    kinds = SI.planted_head_kinds(wl)
    rng = np.random.default_rng(seed)
    flops = 0
    elapsed = 0.0
    for h in heads:
        q, k, v = (O.from_bf16_bits(t.view(torch.int16).numpy()) for t in SI.make_head(wl, 0, h))
        rows = np.sort(rng.choice(wl.N, size=n_rows, replace=False))
        kind = O.MASK_TEMPORAL if kinds[h] == 1 else O.MASK_SPATIAL
        t0 = time.perf_counter()
        pi = O.permutation(wl.T, wl.P, wl.n_text)
        lrows = pi[rows] if kind == O.MASK_TEMPORAL else rows
        qblocks = sorted(set((lrows // wl.block_q).tolist()))
        bm_rows = O.block_mask_rows(kind, qblocks, wl.T, wl.P, wl.n_text, wl.spatial_band,
                                    wl.temporal_width, wl.block_q, wl.block_k)
        bm = np.zeros(( -(-wl.N // wl.block_q), bm_rows.shape[1]), dtype=bool)
        bm[qblocks] = bm_rows
        O.layer_rows(q, k, v, kinds[h], wl.T, wl.P, wl.n_text, wl.spatial_band,
                     wl.temporal_width, wl.block_q, wl.block_k, wl.scale, rows=rows, bm=bm)
        elapsed += time.perf_counter() - t0
        cols_in = np.minimum(wl.block_k, wl.N - np.arange(bm.shape[1]) * wl.block_k)
        for r in lrows:
            flops += 4 * wl.d * int(np.sum(cols_in[bm[r // wl.block_q]]))
    return elapsed, flops


def oracle_components(wl, n_rows: int = 128, n_qblocks: int = 3):
    """Times the oracle's other steps on bounded samples of the workload, with
    a labelled extrapolation of each to the whole layer:
      profiling  the full and both masked attentions, MSEs and label of one head
                 on n_rows of its sampled rows (layer: n_samples rows x B*H heads);
      masks      brute-force block-mask rows (OR over token pairs) of n_qblocks
                 query blocks per pattern (layer: every query block, 2 patterns);
      permute    the layout transformation of one head's Q (layer: Q, K, V and
                 the inverse of O for every temporal head)."""
    import oracle as O
    kinds = SI.planted_head_kinds(wl)
    h = kinds.index(1) if 1 in kinds else 0
    q, k, v = (O.from_bf16_bits(t.view(torch.int16).numpy()) for t in SI.make_head(wl, 0, h))
    rows = SI.sample_rows(wl).numpy()
    sub = rows[np.linspace(0, rows.size - 1, min(n_rows, rows.size)).astype(np.int64)]
    t0 = time.perf_counter()
    O.profile_head(q, k, v, sub, wl.T, wl.P, wl.n_text, wl.spatial_band, wl.temporal_width,
                   wl.scale)
    t_prof = time.perf_counter() - t0
    nqb = -(-wl.N // wl.block_q)
    qbs = np.linspace(0, nqb - 1, n_qblocks).astype(np.int64)
    t0 = time.perf_counter()
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
        O.block_mask_rows(kind, qbs, wl.T, wl.P, wl.n_text, wl.spatial_band, wl.temporal_width,
                          wl.block_q, wl.block_k)
    t_mask = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.permute(q, wl.T, wl.P, wl.n_text)
    t_perm = time.perf_counter() - t0
    n_temporal = wl.B * sum(kinds)
    return {
        "profiling": {"seconds": t_prof, "sample": f"1 head x {sub.size} sampled rows",
                      "extrapolated_layer_s": t_prof * wl.n_samples / sub.size * wl.B * wl.H},
        "block_masks": {"seconds": t_mask,
                        "sample": f"{len(qbs)} query blocks x 2 patterns, brute force",
                        "extrapolated_layer_s": t_mask * nqb / len(qbs)},
        "permute": {"seconds": t_perm, "sample": "Q of 1 head",
                    "extrapolated_layer_s": t_perm * 4 * n_temporal},
    }


def cpu_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, wl):
    world, rank, _ = _dist_env()
    if rank != 0:
        return
    heads = [h for h, kd in enumerate(SI.planted_head_kinds(wl)) if kd == 0][:1] + \
            [h for h, kd in enumerate(SI.planted_head_kinds(wl)) if kd == 1][:1]
    n_rows = 24
    for _ in range(args.warmup):
        oracle_sample(wl, 4, heads[:1])
    times, flops = [], 0
    for s in range(args.steps):
        t, f = oracle_sample(wl, n_rows, heads, seed=100 + s)
        times.append(t)
        flops = f
    ms = 1e3 * statistics.mean(times)
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"fp64 oracle attention output of {n_rows} query rows x {len(heads)} heads "
              f"(one spatial, one temporal) of {wl.name} per step, with their block-mask rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# small-case driver for ncu captures
# ---------------------------------------------------------------------------
def run_capture(args, wl):
    """One kernel, three launches, on the workload cut to --heads heads (the
    planted head split kept at half spatial); inputs stay larger than L2."""
    import video_dit_spatial_b200 as svg
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    wl = wl.replace(H=args.heads, n_spatial=args.heads // 2)
    g = svg.Geom.from_workload(wl)
    q, k, v = (t.cuda() for t in SI.make_qkv(wl))
    rows = SI.sample_rows(wl).cuda()
    layers = {name: SparseVideoGenLayer(g, wl.n_samples, layout=name)
              for name in ("explicit", "fused", "gathered")}
    labels = torch.tensor(SI.planted_head_kinds(wl) * wl.B, dtype=torch.int8)
    for layer in layers.values():
        layer.build_masks()
        layer.labels.copy_(labels)
    ex, fu, ga = layers["explicit"], layers["fused"], layers["gathered"]
    o = torch.empty_like(q)
    svg.svg_permute_qkv(g, q, k, v, ex.qp, ex.kp, ex.vp, ex.labels)
    svg.svg_permute_qkv(g, None, k, v, None, fu.kp, fu.vp, fu.labels)

    def fused_attention(layer, kp, vp):
        m = layer.masks
        return lambda: svg.svg_sparse_attention_fused(
            g, q, k, v, kp, vp, layer.labels, m[0].row_ptr, m[0].col_idx, m[1].row_ptr,
            m[1].col_idx, o)
    fns = {
        # the attention kernel of the default (explicit) layout
        "attention": lambda: svg.svg_sparse_attention(
            g, q, k, v, ex.qp, ex.kp, ex.vp, ex.labels, ex.masks[0].row_ptr,
            ex.masks[0].col_idx, ex.masks[1].row_ptr, ex.masks[1].col_idx, o, ex.op),
        "attention_fused": fused_attention(fu, fu.kp, fu.vp),
        "attention_gathered": fused_attention(ga, None, None),
        "profile": lambda: fu.profile(q, k, v, rows),
        "permute": lambda: svg.svg_permute_qkv(g, q, k, v, ex.qp, ex.kp, ex.vp, ex.labels),
    }
    if args.capture in ("kmeans", "ear"):
        from video_dit_spatial_b200.layer import SemanticSparseLayer
        sl2 = SemanticSparseLayer(wl.B, wl.H, wl.N, wl.d, Cq=SVG2_CQ, Ck=SVG2_CK, iters=1,
                                  top_p=SVG2_TOP_P, block_k=wl.block_k,
                                  ear_tau=SVG2_EAR_TAU if args.capture == "ear" else None)
        sl2.plan(q, k, v)
        sl2.attend(q, k, v, o)
        BH = wl.B * wl.H
        if args.capture == "kmeans":
            # one assignment + sort + update round of the query clustering
            c_out = torch.empty_like(sl2.cq)
            fns["kmeans"] = lambda: svg.svg2_kmeans_step(
                BH, wl.N, wl.d, SVG2_CQ, q, sl2.cq, c_out, sl2.assign_q, sl2.order_q,
                sl2.offsets_q, sl2.workspace)
        else:
            fns["ear"] = lambda: svg.svg2_ear_compensate(
                BH, wl.N, wl.d, SVG2_CK, wl.block_k, wl.scale, sl2.qs, sl2.ck, sl2.vbar,
                sl2.offsets_k, sl2.row_ptr, sl2.col_idx, sl2.os, sl2.lse, sl2.ear_ws)
    if args.capture == "attention_fp8":
        v8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
        v_scale = torch.empty(wl.B * wl.H * wl.d, dtype=torch.float32, device="cuda")
        svg.svg_quantize_v_e4m3(g, v, ex.vp, ex.labels, v8, v_scale)
        fns["attention_fp8"] = lambda: svg.svg_sparse_attention_fp8pv(
            g, q, k, ex.qp, ex.kp, v8, v_scale, ex.labels, ex.masks[0].row_ptr,
            ex.masks[0].col_idx, ex.masks[1].row_ptr, ex.masks[1].col_idx, o, ex.op)
    fn = fns[args.capture]
    for it in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        print(f"{args.capture} {wl.name} H={wl.H} launch {it}: {e0.elapsed_time(e1):.3f} ms")
    st, bits = svg.svg_get_device_status()
    if st != svg.SVG_OK:
        raise RuntimeError(f"device status {st} bits {bits}")


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(SI.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-svg2", action="store_true")
    ap.add_argument("--capture", choices=["attention", "attention_fused", "attention_gathered",
                                          "attention_fp8", "profile", "permute", "kmeans",
                                          "ear"],
                    help="small case for an ncu capture: run one kernel 3 times on the "
                         "workload with --heads heads, print per-launch ms, no JSON line")
    ap.add_argument("--heads", type=int, default=4)
    args = ap.parse_args()
    wl = SI.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if args.capture:
        run_capture(args, wl)
        return
    if args.warmup < 3:
        args.warmup = 3

    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import video_dit_spatial_b200 as svg
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    svg.load()
    g = svg.Geom.from_workload(wl)
    dev = torch.device("cuda", local)

    # inputs: generated on the host (seeded per rank), pinned, copied once
    wl_r = wl.replace(seed=wl.seed + 7919 * rank) if rank else wl
    qh, kh, vh = (t.pin_memory() for t in SI.make_qkv(wl_r))
    rows_h = SI.sample_rows(wl).pin_memory()
    q, k, v = (t.to(dev, non_blocking=True) for t in (qh, kh, vh))
    rows = rows_h.to(dev)
    o = torch.empty_like(q)
    layer = SparseVideoGenLayer(g, wl.n_samples, dev)
    layout = layer.layout
    stream = torch.cuda.current_stream()

    def step():
        layer.forward(q, k, v, rows, o, rebuild_masks=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # algorithmic work of one step (computed-block pairs by each head's label)
    labels = layer.labels.cpu().numpy()
    pairs = {kind: computed_pairs(svg, g, kind) for kind in (0, 1)}
    attn_flops = sum(4 * wl.d * pairs[int(lb)] for lb in labels)
    dense_flops = 4 * wl.d * wl.N * wl.N * wl.B * wl.H

    clocks = ClockSampler(local) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    # one event before the first step and one after every step: the region's
    # time (the barrier-bracketed total) and each step's own time
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clock_info = clocks.stop() if clocks else None
    ms = max_over_ranks(evs[0].elapsed_time(evs[-1]) / args.steps, dist, dev)
    step_pct = percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)])
    # profile, finalize, 2 masks, attention, plus the layout passes: permute_qkv and
    # unpermute (explicit), permute of K and V (fused), none (gathered); plus the
    # profiling combine kernel when the key ranges are split (a workspace larger
    # than the per-tile sums)
    tiles = (wl.n_samples + 127) // 128
    split = svg.svg_profile_workspace_bytes(g, wl.n_samples) > wl.B * wl.H * 2 * tiles * 4
    gpu_launches = ({"explicit": 7, "fused": 6, "gathered": 5}[layout] + int(split)) * args.steps

    # per-kernel timing: an event pair around every launch on the launch stream,
    # after one untimed launch; p10 / p50 / p90 over the launches
    def time_fn(fn, reps):
        fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        ev[0].record(stream)
        for i in range(reps):
            fn()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        return percentiles([ev[i].elapsed_time(ev[i + 1]) for i in range(reps)])

    t_profile = time_fn(lambda: layer.profile(q, k, v, rows), 20)
    t_masks = time_fn(layer.build_masks, 20)
    # the attention kernel alone on the layer's layout (the roofline's kernel),
    # and each way of doing the layout transformation, for comparison
    m = layer.masks
    labels_d = layer.labels

    def attn_fused(kp, vp):
        return lambda: svg.svg_sparse_attention_fused(
            g, q, k, v, kp, vp, labels_d, m[0].row_ptr, m[0].col_idx, m[1].row_ptr,
            m[1].col_idx, o)
    kp, vp = (torch.empty_like(q) for _ in range(2))
    t_permute_kv = time_fn(lambda: svg.svg_permute_qkv(g, None, k, v, None, kp, vp, labels_d), 20)
    t_attn_fused = time_fn(attn_fused(kp, vp), max(5, args.steps // 2))
    t_attn_gathered = time_fn(attn_fused(None, None), 3)
    qp, op = (torch.empty_like(q) for _ in range(2))
    t_permute = time_fn(lambda: svg.svg_permute_qkv(g, q, k, v, qp, kp, vp, labels_d), 20)
    t_unpermute = time_fn(lambda: svg.svg_unpermute(g, op, o, labels_d), 20)

    def attn_explicit():
        svg.svg_sparse_attention(g, q, k, v, qp, kp, vp, labels_d, m[0].row_ptr, m[0].col_idx,
                                 m[1].row_ptr, m[1].col_idx, o, op)
    # The roofline's kernel is timed over a region of at least 2 s of back-to-back
    # launches, long enough for the clock to settle under the power cap, and is
    # held against the sustained bf16 peak (measured the same way); the burst
    # fraction is reported beside it.
    # the three layouts compared under the same conditions (the same short run)
    t_attn_explicit_short = time_fn(attn_explicit, max(5, args.steps // 2))
    first = t_attn_explicit_short["p50"]
    reps_attn = max(20, int(np.ceil(2000.0 / max(first, 1e-3))))
    attn_clocks = ClockSampler(local) if rank == 0 else None
    t_attn_explicit = time_fn(attn_explicit, reps_attn)
    attn_clock_info = attn_clocks.stop() if attn_clocks else None
    attn_region_s = t_attn_explicit["mean"] * reps_attn / 1e3
    # FP8 PV (e4m3 P and V, bf16 Q K^T): V quantised per (head, channel) from the
    # same permuted copies, then the FP8 attention kernel on the same CSR
    fp8 = None
    if wl.d == 128 and wl.block_q == 128 and not args.no_fp8:
        v8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
        v_scale = torch.empty(wl.B * wl.H * wl.d, dtype=torch.float32, device=dev)
        t_quant = time_fn(lambda: svg.svg_quantize_v_e4m3(g, v, vp, labels_d, v8, v_scale), 20)
        t_attn_fp8 = time_fn(lambda: svg.svg_sparse_attention_fp8pv(
            g, q, k, qp, kp, v8, v_scale, labels_d, m[0].row_ptr, m[0].col_idx, m[1].row_ptr,
            m[1].col_idx, o, op), max(10, args.steps))
        # half of the algorithmic work (QK^T) at the bf16 rate, half (PV) at twice it
        pk8 = _peaks()
        fp8 = {"pv": "e4m3 P x e4m3 V (per-channel scales), bf16 Q K^T",
               "quantize_v_ms": t_quant["p50"], "attention_ms": t_attn_fp8["p50"],
               "attention_ms_pct": t_attn_fp8,
               "attention_tflops": attn_flops / (t_attn_fp8["p50"] * 1e-3) / 1e12,
               "speedup_vs_bf16_attention": None,
               "mixed_peak_tflops_burst": 2.0 / (1.0 / pk8["bf16_tflops"] +
                                                 1.0 / (2.0 * pk8["bf16_tflops"])),
               "mixed_peak_note": "QK^T half at the measured bf16 burst peak, PV half at 2x "
                                  "it (nominal fp8/bf16 ratio)"}
        del v8, v_scale
    del kp, vp, qp, op
    torch.cuda.empty_cache()
    layouts = {
        "explicit": {"permute_qkv": t_permute, "attention": t_attn_explicit_short,
                     "unpermute": t_unpermute},
        "fused": {"permute_kv": t_permute_kv, "attention": t_attn_fused},
        "gathered": {"attention": t_attn_gathered},
    }
    layouts_ms = {name: dict({kk: t["p50"] for kk, t in parts.items()},
                             total=sum(t["p50"] for t in parts.values()))
                  for name, parts in layouts.items()}
    # the roofline's kernel: the layer's layout, from the long region when that is
    # the explicit layout (the default)
    if layout == "explicit":
        layouts[layout]["attention"] = t_attn_explicit
    else:
        attn_region_s = 0.0
    ms_attn = layouts[layout]["attention"]["p50"]
    ms_dense = None
    if not args.no_dense:
        od = torch.empty_like(q)
        ms_dense = time_fn(lambda: layer.dense(q, k, v, od), 3)["p50"]
        del od
    st, bits = svg.svg_get_device_status()
    if st != svg.SVG_OK:
        raise RuntimeError(f"device status {st} bits {bits}")

    # end to end through the public API: pinned host inputs -> device -> pinned
    # host output, every step, with the copies of neighbouring steps overlapped
    # with compute by the streamed executor (StreamedLayer)
    e2e = None
    if not args.no_e2e:
        from video_dit_spatial_b200.layer import StreamedLayer
        del layer, o
        torch.cuda.empty_cache()
        o_h = torch.empty((wl.B, wl.H, wl.N, wl.d), dtype=torch.bfloat16).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, rows_h))
        d2h = o_h.numel() * o_h.element_size()
        sl = StreamedLayer(g, wl.n_samples, dev)
        # the same K steps as the device timing (at least 4): the pipeline's fill
        # and drain (one step's compute and copy-back) are inside the region
        reps = max(4, args.steps)
        for i in range(2):
            sl.submit(i, qh, kh, vh, rows_h, o_h)
        sl.synchronize()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(sl.s_in)
        for i in range(2, 2 + reps):
            sl.submit(i, qh, kh, vh, rows_h, o_h)
        e1.record(sl.s_out)
        sl.synchronize()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / reps, dist, dev)
        e2e = {"value": job_throughput(attn_flops, world, e2e_ms), "unit": UNIT,
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # semantic-aware permutation (SVG2): k-means of Q and K, cluster selection,
    # tile CSR (the plan), then gather -> attention -> scatter, on the same layer
    svg2 = None
    if not args.no_svg2:
        from video_dit_spatial_b200.layer import SemanticSparseLayer
        sl2 = SemanticSparseLayer(wl.B, wl.H, wl.N, wl.d, Cq=SVG2_CQ, Ck=SVG2_CK,
                                  iters=SVG2_ITERS, top_p=SVG2_TOP_P, block_k=wl.block_k,
                                  device=dev)
        o2 = torch.empty_like(q)
        t_plan = time_fn(lambda: sl2.plan(q, k), 5)
        t_attend2 = time_fn(lambda: sl2.attend(q, k, v, o2), 5)
        t_attn2 = time_fn(lambda: svg.svg2_sparse_attention(
            wl.B * wl.H, wl.N, wl.d, wl.block_k, wl.scale, sl2.qs, sl2.ks, sl2.vs, sl2.row_ptr,
            sl2.col_idx, sl2.os), 10)
        rp2 = sl2.row_ptr.cpu().numpy().astype(np.int64)
        ci2 = sl2.col_idx.cpu().numpy()[:rp2[-1]].astype(np.int64)
        nqb2 = sl2.nqb
        rows_in = np.tile(np.minimum(128, wl.N - np.arange(nqb2) * 128), wl.B * wl.H)
        cols_in = np.minimum(wl.block_k, wl.N - np.arange(sl2.nkb) * wl.block_k)
        pairs2 = int(np.sum(np.repeat(rows_in, np.diff(rp2)) * cols_in[ci2]))
        flops2 = 4 * wl.d * pairs2
        svg2 = {"clusters_q": SVG2_CQ, "clusters_k": SVG2_CK, "kmeans_iters": SVG2_ITERS,
                "top_p": SVG2_TOP_P, "tile_density": float(rp2[-1]) / (wl.B * wl.H * nqb2 * sl2.nkb),
                "plan_ms": t_plan["p50"], "attend_ms": t_attend2["p50"],
                "attention_ms": t_attn2["p50"], "layer_ms": t_plan["p50"] + t_attend2["p50"],
                "attention_tflops": flops2 / (t_attn2["p50"] * 1e-3) / 1e12,
                "attention_frac_of_burst_peak": flops2 / (t_attn2["p50"] * 1e-3) / 1e12 /
                _peaks()["bf16_tflops"],
                "computed_block_tflop": flops2 / 1e12}
        del sl2
        torch.cuda.empty_cache()
        # SVG-EAR on the same layer: routing, then compensation of what is left out
        se = SemanticSparseLayer(wl.B, wl.H, wl.N, wl.d, Cq=SVG2_CQ, Ck=SVG2_CK,
                                 iters=SVG2_ITERS, top_p=SVG2_TOP_P, block_k=wl.block_k,
                                 ear_tau=SVG2_EAR_TAU, device=dev)
        t_plan_e = time_fn(lambda: se.plan(q, k, v), 5)
        t_attend_e = time_fn(lambda: se.attend(q, k, v, o2), 5)
        t_comp = time_fn(lambda: svg.svg2_ear_compensate(
            wl.B * wl.H, wl.N, wl.d, SVG2_CK, wl.block_k, wl.scale, se.qs, se.ck, se.vbar,
            se.offsets_k, se.row_ptr, se.col_idx, se.os, se.lse, se.ear_ws), 10)
        rpe = se.row_ptr.cpu().numpy().astype(np.int64)
        svg2["ear"] = {"tau": SVG2_EAR_TAU,
                       "tile_density": float(rpe[-1]) / (wl.B * wl.H * se.nqb * se.nkb),
                       "plan_ms": t_plan_e["p50"], "attend_ms": t_attend_e["p50"],
                       "compensate_ms": t_comp["p50"],
                       "layer_ms": t_plan_e["p50"] + t_attend_e["p50"]}
        del se, o2
        torch.cuda.empty_cache()
    if fp8 is not None:
        fp8["speedup_vs_bf16_attention"] = ms_attn / fp8["attention_ms"]
        fp8["frac_of_mixed_peak"] = fp8["attention_tflops"] / fp8["mixed_peak_tflops_burst"]
    pk = _peaks()
    achieved = attn_flops / (ms_attn * 1e-3) / 1e12
    sustained = attn_region_s >= 2.0
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    kernel_name = f"sparse_attention_pair_kernel<{wl.d},{wl.block_k}>"
    roofline = {"bound": "tensor", "kernel": kernel_name, "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": "bf16 dense, %s, %s (kernel timed over %.1f s of back-to-back "
                             "launches)" % ("sustained" if sustained else "burst", pk["source"],
                                            attn_region_s),
                "frac_of_burst_peak": achieved / pk["bf16_tflops"],
                "frac_of_sustained_peak": achieved / pk["bf16_tflops_sustained"],
                "clocks": attn_clock_info,
                "traffic": _captured_traffic(kernel_name, wl.name),
                "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of a 4-head "
                                "launch scaled by heads (profiles/traffic.json)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        kinds = SI.planted_head_kinds(wl)
        heads = [kinds.index(0), kinds.index(1)]
        secs, fl = oracle_sample(wl, 96, heads)
        comps = oracle_components(wl)
        attn_layer_s = attn_flops / (fl / secs)
        cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"fp64 oracle attention output of 96 query rows x 2 heads (one spatial, "
                         f"one temporal) of {wl.name}, with their block-mask rows; plus "
                         f"profiling, block masks and permutation on the samples in "
                         f"'components'",
               "seconds": secs + sum(c["seconds"] for c in comps.values()),
               "components": dict(comps, attention={
                   "seconds": secs, "sample": "96 query rows x 2 heads",
                   "extrapolated_layer_s": attn_layer_s}),
               # labelled extrapolation: each sample's rate over the whole layer
               "extrapolated_layer_hours": (attn_layer_s + sum(
                   c["extrapolated_layer_s"] for c in comps.values())) / 3600.0}

    if rank == 0:
        line = {
            "metric": METRIC, "value": job_throughput(attn_flops, world, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d,
                       "T": wl.T, "P": wl.P, "n_text": wl.n_text, "block": wl.block_q,
                       "spatial_band": wl.spatial_band, "temporal_width": wl.temporal_width,
                       "n_samples": wl.n_samples,
                       "l2": "inputs larger than L2 (Q,K,V %.2f GB)" % (3 * q.numel() * 2 / 1e9),
                       "parallelism": f"independent replicas x{world}" if world > 1 else "1 GPU"},
            "layer_ms": ms, "layer_ms_pct": step_pct,
            "attn_ms": ms_attn, "dense_ms": ms_dense,
            "speedup_vs_dense": (ms_dense / ms_attn) if ms_dense else None,
            "layer_speedup_vs_dense": (ms_dense / ms) if ms_dense else None,
            "attn_tflops": achieved,
            "dense_tflops": (dense_flops / (ms_dense * 1e-3) / 1e12) if ms_dense else None,
            "layout": layout,
            "kernel_ms": dict({"profile": t_profile["p50"], "block_masks": t_masks["p50"]},
                              **{k: t["p50"] for k, t in layouts[layout].items()}),
            "kernel_ms_pct": dict({"profile": t_profile, "block_masks": t_masks},
                                  **layouts[layout]),
            "layouts_ms": layouts_ms,
            "labels_temporal": int(np.sum(labels == 1)),
            "fp8_pv": fp8, "svg2_semantic": svg2,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": gpu_launches, "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
