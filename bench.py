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


def _captured_traffic():
    """DRAM bytes per full-size attention launch from the committed ncu summary,
    or None when the kernel sources changed since that capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "sparse_attention_pair_hunyuan_H4_d128.md")
    srcs = [os.path.join(ROOT, "video_dit_spatial_b200", "csrc", f)
            for f in ("attention.cu", "sm100.cuh")]
    try:
        text = open(path).read()
        digest = hashlib.sha256(b"".join(open(f, "rb").read() for f in srcs)).hexdigest()[:16]
    except OSError:
        return None
    fields = dict(line.strip().split(": ", 1) for line in text.splitlines()
                  if line.strip().startswith(("traffic_bytes", "kernel_sources")))
    if fields.get("kernel_sources_sha256_16") != digest:
        return None
    return int(fields["traffic_bytes_per_launch_full_size"])


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
    ap.add_argument("--capture", choices=["attention", "attention_fused", "attention_gathered",
                                          "profile", "permute"],
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
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clock_info = clocks.stop() if clocks else None
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
    # profile, finalize, 2 masks, attention, plus the layout passes: permute_qkv and
    # unpermute (explicit), permute of K and V (fused), none (gathered); plus the
    # profiling combine kernel when the key ranges are split (a workspace larger
    # than the per-tile sums)
    tiles = (wl.n_samples + 127) // 128
    split = svg.svg_profile_workspace_bytes(g, wl.n_samples) > wl.B * wl.H * 2 * tiles * 4
    gpu_launches = ({"explicit": 7, "fused": 6, "gathered": 5}[layout] + int(split)) * args.steps

    # per-kernel timing (events on the launch stream), then the dense baseline
    def time_fn(fn, reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms_profile = time_fn(lambda: layer.profile(q, k, v, rows), 5)
    ms_masks = time_fn(layer.build_masks, 5)
    # the attention kernel alone on the layer's layout (the roofline's kernel),
    # and each way of doing the layout transformation, for comparison
    m = layer.masks
    labels_d = layer.labels

    def attn_fused(kp, vp):
        return lambda: svg.svg_sparse_attention_fused(
            g, q, k, v, kp, vp, labels_d, m[0].row_ptr, m[0].col_idx, m[1].row_ptr,
            m[1].col_idx, o)
    kp, vp = (torch.empty_like(q) for _ in range(2))
    ms_permute_kv = time_fn(lambda: svg.svg_permute_qkv(g, None, k, v, None, kp, vp, labels_d),
                            5)
    ms_attn_fused = time_fn(attn_fused(kp, vp), max(3, args.steps))
    ms_attn_gathered = time_fn(attn_fused(None, None), 3)
    qp, op = (torch.empty_like(q) for _ in range(2))
    ms_permute = time_fn(lambda: svg.svg_permute_qkv(g, q, k, v, qp, kp, vp, labels_d), 5)
    ms_unpermute = time_fn(lambda: svg.svg_unpermute(g, op, o, labels_d), 5)
    ms_attn_explicit = time_fn(lambda: svg.svg_sparse_attention(
        g, q, k, v, qp, kp, vp, labels_d, m[0].row_ptr, m[0].col_idx, m[1].row_ptr,
        m[1].col_idx, o, op), max(3, args.steps // 2))
    del kp, vp, qp, op
    torch.cuda.empty_cache()
    layouts_ms = {
        "explicit": {"permute_qkv": ms_permute, "attention": ms_attn_explicit,
                     "unpermute": ms_unpermute,
                     "total": ms_permute + ms_attn_explicit + ms_unpermute},
        "fused": {"permute_kv": ms_permute_kv, "attention": ms_attn_fused,
                  "total": ms_permute_kv + ms_attn_fused},
        "gathered": {"attention": ms_attn_gathered, "total": ms_attn_gathered},
    }
    ms_attn = layouts_ms[layout]["attention"]
    ms_dense = None
    if not args.no_dense:
        od = torch.empty_like(q)
        ms_dense = time_fn(lambda: layer.dense(q, k, v, od), 2)
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
        reps = max(4, min(args.steps, 8))
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

    pk = _peaks()
    achieved = attn_flops / (ms_attn * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "sparse_attention_pair_kernel", "achieved": achieved,
                "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops_sustained"],
                "peak_kind": f"bf16 dense, sustained, {pk['source']}",
                "frac_of_burst_peak": achieved / pk["bf16_tflops"],
                "traffic": _captured_traffic() if wl.name == SI.HUNYUAN.name else None,
                "traffic_note": "ncu dram read+write of a 4-head launch, scaled by heads"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        kinds = SI.planted_head_kinds(wl)
        heads = [kinds.index(0), kinds.index(1)]
        secs, fl = oracle_sample(wl, 96, heads)
        cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"fp64 oracle attention output of 96 query rows x 2 heads (one spatial, "
                         f"one temporal) of {wl.name}, with their block-mask rows",
               "seconds": secs,
               # labelled extrapolation: the sample's rate over the layer's computed pairs
               "extrapolated_layer_hours": attn_flops / (fl / secs) / 3600.0}

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
            "layer_ms": ms,
            "attn_ms": ms_attn, "dense_ms": ms_dense,
            "speedup_vs_dense": (ms_dense / ms_attn) if ms_dense else None,
            "layer_speedup_vs_dense": (ms_dense / ms) if ms_dense else None,
            "attn_tflops": achieved,
            "dense_tflops": (dense_flops / (ms_dense * 1e-3) / 1e12) if ms_dense else None,
            "layout": layout,
            "kernel_ms": dict({"profile": ms_profile, "block_masks": ms_masks},
                              **{k: t for k, t in layouts_ms[layout].items() if k != "total"}),
            "layouts_ms": layouts_ms,
            "labels_temporal": int(np.sum(labels == 1)),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": gpu_launches, "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
