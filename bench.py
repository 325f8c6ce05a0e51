#!/usr/bin/env python
"""Benchmark of the rasterizer's hot path: one step = preprocess -> bin/sort
-> render forward -> render backward -> preprocess backward for one frame of
the 1M-Gaussian 1920x1080 synthetic scene (16x16 tiles), fp32.

Prints one JSON line.  ``value`` is Gaussian-pixel evaluations per second for
the whole job (all ranks).  A frame's evaluations are, per pixel, the list
entries the forward evaluated before the pixel stopped plus the entries of
its contributor prefix that the backward walks: sum(n_evaluated) +
sum(n_contrib), counted by the library's gs_render_stats.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Under torchrun each rank renders its own frame (replicas, no collective on
the data path); the timed region is the max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("rasterizer fwd+bwd ms/frame and Gaussian·pixel evals/s; bwd HBM GB/s vs B200 peak")
UNIT = "Gaussian·pixel evals/s"

# Algorithmic FP32 operations per blended term (each add, mul, min, div or
# exp counts one): forward = 15 to evaluate alpha + 9 to blend; backward = 15
# to re-evaluate alpha + 45 for the gradient formulas.  Only blended terms
# count: any other term provably contributes nothing and may be skipped.
OPS_FWD_EVAL = 24
OPS_BWD_EVAL = 60
# DRAM bytes per launch from the committed ncu capture of the render backward (k_render_bwd_warp)
# (dram__bytes_read.sum + dram__bytes_write.sum) and the SHA-1 of the render
# sources it was taken on; reported only while the sources are unchanged.
RECORDED_TRAFFIC = {"k_render_bwd": dict(bytes=172241664, sources_sha1="8243298a71f69c8b1810756cb1580be2c0fac093")}
# Algorithmic bytes: per (tile, Gaussian) pair visited, id + mean2d +
# conic/opacity + colour = 40 B read; the backward adds 36 B of gradient
# atomics per pair; per pixel the forward writes 20 B (image, T, n_contrib)
# and the backward reads 20 B (T, n_contrib, dL/dpixel).
BYTES_PAIR_READ = 40
BYTES_PAIR_ATOMIC = 36
BYTES_PIXEL = 20
SMS = 148
FP32_LANES_PER_SM = 128
# Algorithmic bytes of gs_bin_sort on its cell (4x4-tile super-tile) route:
# per Gaussian 156 B (key build 16, four depth-radix passes x 20, the
# rank-order scans 40, the first cell pass's per-rank reads 20), per
# (cell, Gaussian) pair 60 B (first pass write 8, second pass histogram +
# scatter 20, cell ranges 4, segment counting 22 incl. the rectangle gather,
# expansion reads 6), per (tile, Gaussian) pair the 4-byte id written.
BIN_BYTES_GAUSSIAN = 156
BIN_BYTES_CELL_PAIR = 60
BIN_BYTES_PAIR = 4
CELL = 4  # tiles per cell side


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return dict(hbm_gbs=float(d["hbm_gbs"]), sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), src="measured")
    return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0, src="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"gs_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
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
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=mx, reasons=sorted(reasons), samples=len(sm))


def _render_sources_sha1() -> str:
    import hashlib
    h = hashlib.sha1()
    for name in ("render.cu", "gs_internal.cuh", "pdl.cuh"):
        with open(os.path.join(ROOT, "differentiable_gaussian_splatting_preprocess_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _scene(cfg: int):
    from differentiable_gaussian_splatting_preprocess_b200 import scenes
    return scenes.preset(cfg)


def cpu_tile_stride(cfg: int) -> int:
    """Tile sample of the CPU oracle: every tile up to config 3, every 16th
    tile of the 1080p configs (the same sample in both arms)."""
    return 16 if cfg >= 4 else 1


def cpu_oracle_sample(sc, tile_stride: int):
    """Time the oracle on a bounded sample of the workload, forward and
    backward separately: forward = full preprocess and binning, then
    compositing (fp32 mirror) of every ``tile_stride``-th tile; backward =
    compositing backward (float64) of the same tiles, then the full
    preprocess backward.  Evaluations are counted like the GPU metric's:
    per sampled pixel, entries evaluated in the forward plus the contributor
    prefix walked by the backward."""
    import oracle
    cam = sc.cameras[0]
    t0 = time.perf_counter()
    pre = oracle.preprocess(cam, sc.means, sc.scales, sc.quats, sc.opacity, "f32")
    b = oracle.bin_pairs(cam, pre["depth"], pre["rect"], pre["tiles_touched"], "f32", want_keys=False)
    tiles = np.arange(0, cam.num_tiles, tile_stride, dtype=np.int32)
    r = oracle.render_fwd(cam, b["ranges"], b["ids"], pre["mean2d"], pre["conic_opacity"], sc.colors, "f32",
                          tiles=tiles)
    t1 = time.perf_counter()
    g = oracle.render_bwd(cam, sc.N, b["ranges"], b["ids"], pre["mean2d"], pre["conic_opacity"], sc.colors,
                          sc.dL_dimage[0], "f64", tiles=tiles)
    oracle.preprocess_bwd(cam, sc.means, sc.scales, sc.quats, pre["radius"], g["dL_dmean2d"],
                          g["dL_dconic_opacity"], g["dL_dcolor"], "f64")
    t2 = time.perf_counter()
    ev_f = int(r["n_eval"].astype(np.int64).sum())
    ev_b = int(r["n_contrib"].astype(np.int64).sum())
    sample = (f"full preprocess + binning of the {sc.name} scene, compositing fwd (fp32) + bwd (fp64) on every "
              f"{tile_stride}th tile ({tiles.size} of {cam.num_tiles})" if tile_stride > 1 else
              f"the whole {sc.name} frame: preprocess, binning, compositing fwd (fp32) + bwd (fp64), "
              f"preprocess bwd (fp64)")
    return dict(evals=ev_f + ev_b, evals_fwd=ev_f, evals_bwd=ev_b, seconds=t2 - t0, fwd_s=t1 - t0, bwd_s=t2 - t1,
                cores=oracle.num_threads(), sample=sample)


def cpu_baseline(sc, cfg: int, min_seconds: float = 10.0, single_thread_cfgs=(1, 2, 3)):
    """The oracle on the host cores: the bounded sample of ``cpu_oracle_sample``
    repeated until about ``min_seconds`` of host work, forward and backward
    reported separately; plus one-thread numbers for the small configs."""
    import oracle
    tot = dict(evals=0, evals_fwd=0, evals_bwd=0, seconds=0.0, fwd_s=0.0, bwd_s=0.0)
    reps = 0
    while tot["seconds"] < min_seconds and reps < 50:
        c = cpu_oracle_sample(sc, cpu_tile_stride(cfg))
        for k in tot:
            tot[k] += c[k]
        reps += 1
    out = dict(value=tot["evals"] / tot["seconds"], unit=UNIT, cores=c["cores"], kind="oracle",
               sample=f"{reps} x ({c['sample']}); {tot['seconds']:.1f} s in total",
               fwd=dict(value=tot["evals_fwd"] / tot["fwd_s"], unit=UNIT, ms_per_sample=1e3 * tot["fwd_s"] / reps),
               bwd=dict(value=tot["evals_bwd"] / tot["bwd_s"], unit=UNIT, ms_per_sample=1e3 * tot["bwd_s"] / reps))
    n0 = oracle.num_threads()
    st = {}
    try:
        oracle.set_threads(1)
        for k in single_thread_cfgs:
            c = cpu_oracle_sample(_scene(k), cpu_tile_stride(k))
            st[f"config{k}"] = dict(value=c["evals"] / c["seconds"], fwd_evals_per_s=c["evals_fwd"] / c["fwd_s"],
                                    bwd_evals_per_s=c["evals_bwd"] / c["bwd_s"], fwd_ms=1e3 * c["fwd_s"],
                                    bwd_ms=1e3 * c["bwd_s"], unit=UNIT, cores=1, sample=c["sample"])
    finally:
        oracle.set_threads(n0)
    out["single_thread"] = st
    return out


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    sc = _scene(args.config)
    stride = cpu_tile_stride(args.config)
    import oracle
    for _ in range(args.warmup):
        cpu_oracle_sample(sc, stride * 4)
    recs = [cpu_oracle_sample(sc, stride) for _ in range(args.steps)]
    secs = sum(r["seconds"] for r in recs)
    value = sum(r["evals"] for r in recs) / secs
    fwd = sum(r["evals_fwd"] for r in recs) / sum(r["fwd_s"] for r in recs)
    bwd = sum(r["evals_bwd"] for r in recs) / sum(r["bwd_s"] for r in recs)
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=ws, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * secs / len(recs), higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f32 fwd / f64 bwd", data="synthetic", impl="reference",
                config=dict(workload=f"{sc.name}: {sc.N} Gaussians, {sc.cameras[0].width}x{sc.cameras[0].height},"
                                     " 16x16 tiles (bounded tile sample per step)"),
                cpu_baseline=dict(kind="oracle", cores=oracle.num_threads(), value=value, unit=UNIT,
                                  sample=recs[-1]["sample"], fwd=dict(value=fwd, unit=UNIT),
                                  bwd=dict(value=bwd, unit=UNIT)),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    from differentiable_gaussian_splatting_preprocess_b200 import binding as B
    from differentiable_gaussian_splatting_preprocess_b200 import multiview as MV
    from differentiable_gaussian_splatting_preprocess_b200 import rasterizer as RZ

    world, rank, local = _dist()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    B.lib()

    sc = _scene(args.config)
    # Work of this rank.  Several views, or --split image: the fixed
    # workload is cut into (camera, band) units spread over the ranks
    # (multiview.assign_work: whole cameras when the ranks divide them,
    # tile-row bands otherwise) and the 3D gradients are summed with one
    # all-reduce.  One view without --split: every rank renders the whole
    # frame (replicas, no collective).
    split = len(sc.cameras) > 1 or args.split == "image"
    if split:
        units = MV.assign_work(sc.cameras, world, rank)
    else:
        units = [MV.WorkUnit(0, 0, sc.cameras[0].height, True)]
    cams = [MV.unit_view(sc.cameras, u) for u in units]
    mine = list(range(len(units)))
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    means, scales, quats, opacity, colors = (t(x) for x in (sc.means, sc.scales, sc.quats, sc.opacity, sc.colors))
    dl_rows = [np.ascontiguousarray(sc.dL_dimage[u.camera][:, u.y0:u.y1]) for u in units]
    dLs = {i: t(dl_rows[i]) for i in mine}
    rzs = {i: RZ.Rasterizer(cams[i], dev) for i in mine}
    caps = {}
    for i in mine:
        # size the pair buffers once (host read of P), then run in capacity mode
        fr = rzs[i].forward(means, scales, quats, opacity, colors)
        caps[i] = fr.capacity
        rzs[i].backward(fr, means, scales, quats, colors, dLs[i])  # allocates the 2D gradient buffers
    grads = RZ.zero_grads(sc.N, dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    sh_deg = args.sh_degree
    if sh_deg is not None:
        from differentiable_gaussian_splatting_preprocess_b200 import scenes as _scn
        shd = torch.from_numpy(_scn.random_sh(sc.N, sh_deg, seed=1)).to(dev)
        dsh = torch.zeros_like(shd)
        if args.sh_f16:
            shd = shd.half()  # binary16 storage, fp32 arithmetic (gs_sh_*_f16)
        colors = torch.empty((sc.N, 3), dtype=torch.float32, device=dev)
    exchange = split and world > 1
    adam = None
    if args.adam:
        # the optimiser stage: raw parameters (log scales, logit opacity) whose
        # activated values the step writes back into the rasterizer's inputs
        adam = dict(cfg=B.GsAdamConfig(1.6e-4, 5e-3, 1e-3, 5e-2, 2.5e-3, 0.9, 0.999, 1e-15, 3000), step=[0],
                    params=dict(means=means.clone(), log_scales=torch.log(scales), quats=quats.clone(),
                                logit_opacity=torch.logit(opacity), colors=colors.clone()))
        if sh_deg is not None:
            raise SystemExit("--adam covers RGB colours (no --sh-degree)")
        adam["m"] = torch.zeros((11 + 3) * sc.N, device=dev)
        adam["v"] = torch.zeros_like(adam["m"])
        # the optimiser updates its own copies and writes the activated
        # values to scratch buffers, so the timed scene (and its pair count)
        # stays that of the workload
        adam["scales"] = torch.empty_like(scales)
        adam["opacity"] = torch.empty_like(opacity)

    # several views: their projection and binning run ahead on a
    # high-priority stream while this stream composites the previous view
    # (multiview.render_views(overlap=True)); timed per stage (``rec``), the
    # stages run in sequence on one stream
    overlap = len(mine) > 1 and sh_deg is None and not args.no_overlap
    bin_st = MV.binning_stream(dev) if overlap else None

    def step(rec=None):
        """One step: every view of this rank through a1-a8 (gradients summed),
        then the gradient exchange when views are split over ranks.
        ``rec`` collects (stage, start event, end event)."""
        def timed(name, fn):
            if rec is None:
                fn()
                return
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            rec.append((name, e0, e1))

        if overlap and rec is None:
            cs = torch.cuda.current_stream(dev)  # the capture stream while a graph records
            bin_st.wait_stream(cs)
            for i in mine:
                cam, rz, cap, dL = cams[i], rzs[i], caps[i], dLs[i]
                b = rz._bufs
                rz.preprocess(means, scales, quats, opacity, bin_st)
                B.gs_bin_sort(cam, b["depth"], b["rect"], b["tiles_touched"], b["num_pairs"], cap, b["ids"],
                              b["ranges"], None, rz.workspace(sc.N, cap), bin_st)
                binned = torch.cuda.Event()
                binned.record(bin_st)
                cs.wait_event(binned)
                B.gs_render_fwd(cam, b["ranges"], b["ids"], b["mean2d"], b["conic_opacity"], colors, b["image"],
                                b["final_T"], b["n_contrib"], b["contrib_mask"])
                B.gs_render_bwd(cam, b["ranges"], b["ids"], b["mean2d"], b["conic_opacity"], colors, b["final_T"],
                                b["n_contrib"], dL, b["dL_dmean2d"], b["dL_dconic_opacity"], b["dL_dcolor"],
                                b["contrib_mask"])
                B.gs_preprocess_bwd(cam, means, scales, quats, b["radius"], b["conic_opacity"], b["dL_dmean2d"],
                                    b["dL_dconic_opacity"], b["dL_dcolor"], grads["dL_dmeans"], grads["dL_dscales"],
                                    grads["dL_dquats"], grads["dL_dopacity"], grads["dL_dcolors"])
            cs.wait_stream(bin_st)
        for i in (mine if not (overlap and rec is None) else []):
            cam, rz, cap, dL = cams[i], rzs[i], caps[i], dLs[i]
            b = rz._bufs
            if sh_deg is not None:
                timed("sh_fwd", lambda: B.gs_sh_fwd(cam, sh_deg, means, shd, colors, offset=0.5))
            timed("preprocess_fwd", lambda: rz.preprocess(means, scales, quats, opacity))
            timed("bin_sort", lambda: B.gs_bin_sort(cam, b["depth"], b["rect"], b["tiles_touched"], b["num_pairs"],
                                                   cap, b["ids"], b["ranges"], None, rz.workspace(sc.N, cap)))
            timed("render_fwd", lambda: B.gs_render_fwd(cam, b["ranges"], b["ids"], b["mean2d"], b["conic_opacity"],
                                                       colors, b["image"], b["final_T"], b["n_contrib"],
                                                       b["contrib_mask"]))
            timed("render_bwd", lambda: B.gs_render_bwd(cam, b["ranges"], b["ids"], b["mean2d"], b["conic_opacity"],
                                                       colors, b["final_T"], b["n_contrib"], dL, b["dL_dmean2d"],
                                                       b["dL_dconic_opacity"], b["dL_dcolor"], b["contrib_mask"]))
            timed("preprocess_bwd", lambda: B.gs_preprocess_bwd(
                cam, means, scales, quats, b["radius"], b["conic_opacity"], b["dL_dmean2d"], b["dL_dconic_opacity"],
                b["dL_dcolor"], grads["dL_dmeans"], grads["dL_dscales"], grads["dL_dquats"], grads["dL_dopacity"],
                grads["dL_dcolors"]))
            if sh_deg is not None:
                timed("sh_bwd", lambda: B.gs_sh_bwd(cam, sh_deg, means, shd, grads["dL_dcolors"], dsh,
                                                   grads["dL_dmeans"], offset=0.5))
        if exchange:
            timed("allreduce", lambda: MV.allreduce_grads(grads))
        if adam is not None:
            adam["step"][0] += 1
            timed("adam", lambda: B.gs_adam_step(adam["cfg"], adam["step"][0], adam["params"], grads, adam["m"],
                                                 adam["v"], adam["scales"], adam["opacity"]))

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    for i in mine:
        st = rzs[i].status()
        if st != 0:
            raise RuntimeError(f"device status {st}: {B.status_string(st)}")
    # work counts of this rank's views (outside the timed region)
    n_contrib = n_evaluated = n_blended = P = Ps = 0
    visited_fwd = visited_bwd = 0  # list entries a tile's walk reads: sum over tiles of the furthest pixel

    def visited(counts, cam):
        TX, TY = (cam.width + 15) // 16, (cam.height + 15) // 16
        full = torch.zeros((TY * 16, TX * 16), dtype=torch.int64, device=dev)
        full[:cam.height, :cam.width] = counts.view(torch.int32).to(torch.int64)
        return int(full.view(TY, 16, TX, 16).amax(dim=(1, 3)).sum().item())

    for i in mine:
        b, cam = rzs[i]._bufs, cams[i]
        rc = b["rect"].to(torch.int64)
        vis = b["tiles_touched"].view(torch.int32) > 0
        cells = (((rc[:, 2] - 1) // CELL - rc[:, 0] // CELL + 1) * ((rc[:, 3] - 1) // CELL - rc[:, 1] // CELL + 1))
        Ps += int(torch.where(vis, cells, torch.zeros_like(cells)).sum().item())
        ne = torch.empty((cam.height, cam.width), dtype=torch.uint32, device=dev)
        nb = torch.empty_like(ne)
        B.gs_render_stats(cam, b["ranges"], b["ids"], b["mean2d"], b["conic_opacity"], ne, nb)
        n_contrib += int(b["n_contrib"].view(torch.int32).to(torch.int64).sum().item())
        n_evaluated += int(ne.view(torch.int32).to(torch.int64).sum().item())
        n_blended += int(nb.view(torch.int32).to(torch.int64).sum().item())
        visited_fwd += visited(ne, cam)
        visited_bwd += visited(b["n_contrib"], cam)
        P += caps[i]
    evals_per_step = n_evaluated + n_contrib

    # the step recorded once into a CUDA graph (capacity mode: no host
    # round trip, so every call is capturable) and replayed: one launch per
    # step instead of ~35 launches per view through the Python binding
    graph, graph_launches = None, 0
    graph_spread = None
    if not args.no_graph and not exchange and adam is None:
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(dev)
        n0 = B.launch_count()
        with torch.cuda.graph(graph):
            step()
        graph_launches = B.launch_count() - n0  # kernels recorded per step
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(local)
    recs = [[] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    launches0 = B.launch_count()
    for k in range(args.steps):
        flush.zero_()  # L2 flush outside the timed intervals
        step(recs[k])
    launches = B.launch_count() - launches0  # this library's kernels in the timed steps
    graph_ms = []
    if graph is not None:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for k in range(args.steps):
            flush.zero_()
            ev[k][0].record(stream)
            graph.replay()
            ev[k][1].record(stream)
        launches = graph_launches * args.steps  # every recorded kernel runs once per replay
    torch.cuda.synchronize(dev)
    if graph is not None:
        graph_ms = [a.elapsed_time(b) for a, b in ev]
        srt = sorted(graph_ms)
        graph_spread = dict(min=srt[0], median=srt[len(srt) // 2], max=srt[-1])
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    clocks = sampler.stop()
    stage_ms = {}
    step_ms = []
    for rec in recs:
        for name, e0, e1 in rec:
            stage_ms.setdefault(name, []).append(e0.elapsed_time(e1))
        step_ms.append(rec[0][1].elapsed_time(rec[-1][2]))
    eager_ms = sum(step_ms)
    total_ms = sum(graph_ms) if graph is not None else eager_ms
    evals_all = evals_per_step
    if world > 1:
        tt = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_ms = float(tt.item())
        ev_t = torch.tensor([float(evals_per_step)], device=dev, dtype=torch.float64)
        dist.all_reduce(ev_t, op=dist.ReduceOp.SUM)
        evals_all = float(ev_t.item())
    value = evals_all * args.steps / (total_ms / 1e3)
    for i in mine:
        st = rzs[i].status()
        if st != 0:
            raise RuntimeError(f"device status {st}: {B.status_string(st)}")

    # roofline of the dominant kernel (render backward: FP32 issue bound)
    peaks = _peaks()
    # per-step time of each stage, summed over this rank's views (a rank
    # without a view has only the exchange; its stage times are 0)
    mean = {s: statistics.mean(v) * len(v) / args.steps for s, v in stage_ms.items()}
    for s_ in ("preprocess_fwd", "bin_sort", "render_fwd", "render_bwd", "preprocess_bwd"):
        mean.setdefault(s_, 0.0)
    dominant = max(mean, key=mean.get)
    nv = max(len(mine), 1)
    bwd_ops = n_blended * OPS_BWD_EVAL
    fwd_ops = n_blended * OPS_FWD_EVAL
    alu_peak = SMS * FP32_LANES_PER_SM * peaks["sm_max_mhz"] * 1e6 / 1e12  # T lane-ops/s
    per_s = lambda x, ms: x / (ms / 1e3) if ms > 0 else 0.0
    rb_ach = per_s(bwd_ops, mean["render_bwd"]) / 1e12
    rec_t = RECORDED_TRAFFIC["k_render_bwd"]
    traffic = rec_t["bytes"] if (rec_t["sources_sha1"] == _render_sources_sha1() and len(mine) == 1) else None
    roofline = dict(kernel="k_render_bwd_warp", bound="alu", achieved=rb_ach, peak=alu_peak, unit="Tops/s",
                    frac=rb_ach / alu_peak, traffic=traffic, ops_per_launch=bwd_ops // nv,
                    ops_basis=f"{OPS_BWD_EVAL} FP32 ops x {n_blended} blended terms",
                    peak_src=f"148 SMs x 128 FP32 lanes x {peaks['sm_max_mhz']:.0f} MHz (sm_max_mhz)")
    # HBM view of render fwd + bwd, as asked, per VISITED pair: the list
    # entries up to each tile's furthest evaluated (forward) or contributing
    # (backward) position; entries beyond are never read
    pix = sum(cams[i].width * cams[i].height for i in mine)
    fwd_bytes = visited_fwd * BYTES_PAIR_READ + pix * BYTES_PIXEL
    bwd_bytes = visited_bwd * (BYTES_PAIR_READ + BYTES_PAIR_ATOMIC) + pix * BYTES_PIXEL
    rfb_s = max((mean["render_fwd"] + mean["render_bwd"]) / 1e3, 1e-30)
    render_hbm = dict(achieved_gbs=(fwd_bytes + bwd_bytes) / rfb_s / 1e9, peak_gbs=peaks["hbm_gbs"],
                      frac=(fwd_bytes + bwd_bytes) / rfb_s / 1e9 / peaks["hbm_gbs"],
                      bytes_per_frame=fwd_bytes + bwd_bytes, peak_src=peaks["src"],
                      visited_pairs_fwd=visited_fwd, visited_pairs_bwd=visited_bwd,
                      basis=f"{BYTES_PAIR_READ} B per visited pair read by each pass, {BYTES_PAIR_ATOMIC} B of "
                            f"gradient atomics per pair visited by the backward, {BYTES_PIXEL} B per pixel per pass")
    fwd_alu = per_s(fwd_ops, mean["render_fwd"]) / 1e12
    # the metric's "bwd HBM GB/s": the render backward alone, algorithmic
    # bytes and, where the committed capture applies, measured DRAM bytes
    rb_s = max(mean["render_bwd"] / 1e3, 1e-30)
    bwd_hbm = dict(achieved_gbs=bwd_bytes / rb_s / 1e9, peak_gbs=peaks["hbm_gbs"],
                   frac=bwd_bytes / rb_s / 1e9 / peaks["hbm_gbs"], bytes_per_frame=bwd_bytes,
                   dram_gbs=(traffic / (rb_s / len(mine)) / 1e9) if traffic else None, peak_src=peaks["src"])
    # HBM view of the binning (the sort is the stage an HBM roofline fits)
    bin_bytes = len(mine) * sc.N * BIN_BYTES_GAUSSIAN + Ps * BIN_BYTES_CELL_PAIR + P * BIN_BYTES_PAIR
    bin_gbs = per_s(bin_bytes, mean["bin_sort"]) / 1e9
    bin_hbm = dict(achieved_gbs=bin_gbs, peak_gbs=peaks["hbm_gbs"], frac=bin_gbs / peaks["hbm_gbs"],
                   bytes_per_step=bin_bytes, cell_pairs=Ps, peak_src=peaks["src"],
                   basis=f"{BIN_BYTES_GAUSSIAN} B/Gaussian + {BIN_BYTES_CELL_PAIR} B/cell pair + "
                         f"{BIN_BYTES_PAIR} B/pair")

    # end to end through the public API: pinned host inputs -> device (on a
    # side stream, overlapped with the kernels that do not read them yet) ->
    # forward + backward of every view of this rank in capacity mode, the
    # gradient exchange, then the 3D gradients back to the host (third stream)
    e2e = None
    if not args.no_e2e:
        host_params = {k: torch.from_numpy(np.ascontiguousarray(x)).pin_memory()
                       for k, x in zip(("means", "scales", "quats", "opacity", "colors"),
                                       (sc.means, sc.scales, sc.quats, sc.opacity, sc.colors))}
        host_dl = [torch.from_numpy(dl_rows[i]).pin_memory() for i in mine]
        h2d = sum(x.numel() * x.element_size() for x in list(host_params.values()) + host_dl)
        rz_e2e, e2e_state = {}, {}
        host_out = {k: torch.empty(grads[k].shape, dtype=grads[k].dtype, pin_memory=True) for k in MV.GRAD_KEYS}
        def e2e_step():
            MV.render_views_from_host([cams[i] for i in mine], host_params, host_dl, rz_e2e,
                                      [caps[i] for i in mine], camera_ids=units, state=e2e_state,
                                      host_grads=host_out, reduce_fn=MV.allreduce_grads if exchange else None,
                                      device=dev, pipelined=True)

        # steps pipelined as a training loop runs them: step k+1's inputs are
        # copied in while step k computes and step k-1's gradients are copied
        # out; throughput = steps / wall time from the first copy to the last
        # gradient on the host
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            e2e_step()
        e2e_state["done"].synchronize()
        torch.cuda.synchronize(dev)
        e2e_times = [time.perf_counter() - t0]
        d2h = sum(o.numel() * o.element_size() for o in host_out.values())
        e2e_s = sum(e2e_times)
        if world > 1:
            tt = torch.tensor([e2e_s], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            e2e_s = float(tt.item())
        e2e = dict(value=evals_all * args.steps / e2e_s, unit=UNIT, h2d_bytes_per_step=h2d,
                   mode="pipelined steps: copy-in of step k+1, kernels of step k, copy-out of step k-1 overlap",
                   d2h_bytes_per_step=d2h, ms_per_step=1e3 * e2e_s / args.steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(sc, args.config)

    if rank == 0:
        cam0 = sc.cameras[0]
        if exchange:
            par = (f"image-space split x{world} (tile-row bands)" if len(sc.cameras) == 1 else
                   f"camera-parallel x{world} ((camera, band) units)")
        else:
            par = f"replicas x{world}" if world > 1 else "1 GPU"
        line = dict(
            metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
            ms_per_step=total_ms / args.steps, ms_per_step_eager=eager_ms / args.steps,
            launch_mode=("cuda graph replay" + (", views overlapped (projection and binning on a second stream)"
                                                 if overlap else "")) if graph is not None else "eager",
            replay_ms=graph_spread,
            higher_is_better=True, scaling="weak" if not exchange else "strong",
            vs_baseline=None, dtype="f32", data="synthetic",
            config=dict(workload=f"{sc.name}: {sc.N} Gaussians, {cam0.width}x{cam0.height}, {len(sc.cameras)} view(s), "
                                 f"16x16 tiles, fp32"
                                 + (f", SH degree {sh_deg} colours" if sh_deg is not None else "")
                                 + (" (binary16 coefficient storage)" if sh_deg is not None and args.sh_f16 else ""),
                        views_per_rank=len(mine), units_rank0=[(u.camera, u.y0, u.y1) for u in units],
                        num_pairs=P, evals_per_step=evals_per_step,
                        evaluated_fwd=n_evaluated, contributor_prefix_bwd=n_contrib, blended=n_blended,
                        l2="flushed between steps (256 MiB write)", parallelism=par),
            fwd_ms_per_frame=(mean["preprocess_fwd"] + mean["bin_sort"] + mean["render_fwd"]) / nv,
            bwd_ms_per_frame=(mean["render_bwd"] + mean["preprocess_bwd"]) / nv,
            stage_ms={s: round(v, 4) for s, v in mean.items()}, dominant_stage=dominant,
            roofline=roofline, render_fwd_alu=dict(achieved=fwd_alu, peak=alu_peak, unit="Tops/s",
                                                   frac=fwd_alu / alu_peak),
            render_hbm=render_hbm, render_bwd_hbm=bwd_hbm, bin_sort_hbm=bin_hbm, cpu_baseline=cpu, e2e=e2e, gpu_launches=launches,
            clocks=clocks)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--split", choices=["replica", "image"], default="replica",
                    help="one-view configs under torchrun: 'replica' (default) renders the whole frame on every "
                         "rank; 'image' cuts the frame into tile-row bands, one per rank, and sums the 3D "
                         "gradients with one all-reduce (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="several views: run every stage of every view in sequence on one stream (default: the "
                         "views' projection and binning run ahead on a second stream)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches only (default: the step is also captured in a CUDA graph and the "
                         "timed value comes from its replays; stage times always come from eager steps)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sh-degree", type=int, default=None,
                    help="colours from spherical harmonics of this degree (adds the SH stages to the step)")
    ap.add_argument("--adam", action="store_true",
                    help="add the fused optimiser step (gs_adam_step) to the step (eager timing only: the step "
                         "number changes every step)")
    ap.add_argument("--sh-f16", action="store_true",
                    help="with --sh-degree: store the SH coefficients in binary16 (the mixed-precision variant)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
