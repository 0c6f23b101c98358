"""Benchmark of the block-sparse 3D-tile attention path on B200.

One step = one pass of the whole hot path over one synthetic 720p video-DiT
layer (75,600 tokens, 40 heads, d = 128, top-p 0.95 / k_min 8 OR dual
windows, ~15% density), on raster Q, K, V: sta_build_mask_raster ->
sta_attn_fwd_raster (the tile gather of Q, K, V and the scatter of O back to
raster order happen inside the kernels' loads and stores).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --search-curve [--workload NAME]   (window search, recall vs density)
  python bench.py --sweep                              (every layer of the workload table)
  python bench.py --l2-probe                           (the attention's tile-load stream alone)
  python bench.py --mma-probe                          (cycles per tensor-core MMA by width)

Rank 0 prints one JSON line. Under torchrun every rank runs its own layer
(independent problems, no collective on the data path: weak scaling); the
time is the max over ranks of the device-timed region.
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_qkv, perturb_step, window_params, window_scale  # noqa: E402

METRIC = "kept-block attn TFLOP/s & % BF16 peak; ms/layer at 75,600 tokens, 15% density"
UNIT = "TFLOP/s"
HEADLINE = "dit720p"  # the 75,600-token 720p layer
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


NVTX = False  # --nvtx: name the calls of each step on the profiler timeline


class nvtx_range:
    """An NVTX range around one library call when --nvtx is given (for nsys /
    ncu timelines); nothing otherwise."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        if NVTX:
            torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        if NVTX:
            torch.cuda.nvtx.range_pop()
        return False


def flops_per_pair(d):
    return 4.0 * 64 * 64 * d


def max_over_ranks(x, device, world):
    """Largest value of x over all ranks (the job is as slow as its slowest rank)."""
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, device, world):
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_tflops(total_flops_per_step, steps, elapsed_ms):
    """Whole-job throughput: kept-pair flops of all ranks over the slowest rank's time."""
    return steps * total_flops_per_step / (elapsed_ms * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_source_hash():
    """Hash of the attention kernel's code (comments and blank space left
    out, so that editing a comment keeps a traffic capture valid)."""
    import re

    h = hashlib.sha256()
    d = os.path.join(ROOT, "block_sparse_attention_28_b200", "csrc")
    for name in ("sta_attn.cuh", "sta_tc.cuh", "sta_common.cuh"):
        with open(os.path.join(d, name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic():
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, or None when the summary is missing or the kernel changed."""
    p = os.path.join(ROOT, "profiles", "attn_fwd_720p_traffic.md")
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if line.startswith("traffic_bytes_per_launch:"):
            vals["t"] = float(line.split(":", 1)[1])
        if line.startswith("kernel_source_hash:"):
            vals["h"] = line.split(":", 1)[1].strip()
    if vals.get("h") != attn_source_hash():
        return None
    return vals.get("t")


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled every 10 ms
    through NVML (the library nvidia-smi reads) on a host thread; `stop`
    keeps the samples taken inside the timed region's host window. Falls back
    to `nvidia-smi -lms 100` when the NVML binding is missing. Read-only."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake", 0x80))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.device = device
        self.samples = []  # (host time, sm MHz, max MHz, reason names, watts)
        self.stop_flag = threading.Event()
        self.proc = None
        self.thread = None
        self.source = None
        self.limit_w = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.device).uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.source = "nvml"
            try:
                self.limit_w = nv.nvmlDeviceGetPowerManagementLimit(h) / 1000.0
            except Exception:
                self.limit_w = None

            def power_w():
                # instantaneous board power where the driver reports it, else
                # the (about 1 s) averaged figure
                try:
                    fv = nv.nvmlDeviceGetFieldValues(h, [nv.NVML_FI_DEV_POWER_INSTANT])[0]
                    if fv.nvmlReturn == 0:
                        return fv.value.uiVal / 1000.0
                except Exception:
                    pass
                return nv.nvmlDeviceGetPowerUsage(h) / 1000.0

            def run():
                while not self.stop_flag.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        watts = power_w()
                    except Exception:
                        break
                    names = [nm for nm, b in self.REASONS if bits & b]
                    self.samples.append((time.monotonic(), float(sm), float(smax), names, watts))
                    time.sleep(0.01)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id=GPU-{uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"

            def read():
                names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
                for ln in self.proc.stdout:
                    parts = [x.strip() for x in ln.split(",")]
                    try:
                        sm, smax, watts = float(parts[0]), float(parts[1]), float(parts[2])
                    except (ValueError, IndexError):
                        continue
                    act = [nm for nm, v in zip(names, parts[4:8]) if v.lower() == "active"]
                    self.samples.append((time.monotonic(), sm, smax, act, watts))

            self.thread = threading.Thread(target=read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t0=None, t1=None):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        win = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not win:
            win = self.samples
        reasons = sorted({nm for x in win for nm in x[3]})
        return {"sm_mhz": statistics.median(x[1] for x in win) if win else None,
                "sm_min_mhz": min(x[1] for x in win) if win else None,
                "sm_max_mhz": max(x[2] for x in win) if win else None,
                "power_w_median": statistics.median(x[4] for x in win) if win else None,
                "power_w_max": max(x[4] for x in win) if win else None,
                "power_limit_w": self.limit_w,
                "reasons": reasons, "samples": len(win), "source": self.source}


def count_step_launches(layer):
    """Kernels that one step launches, as CUPTI records them (torch.profiler)
    on an untimed step: (count, short kernel names), or (None, None) when the
    profiler cannot record kernels here."""
    try:
        from torch.profiler import ProfilerActivity, profile

        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CPU, ProfilerActivity.CUDA]) as prof:
            layer.step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    except Exception:  # no CUPTI: the caller falls back to the static count
        return None, None
    kernels = [n.split("(")[0].replace("void ", "") for n in names if "Memcpy" not in n and "Memset" not in n]
    return (len(kernels), kernels) if kernels else (None, None)


class Layer:
    """Device buffers and launches of one step of the path."""

    def __init__(self, sta, cfg, dev, seed_offset=0, workload=HEADLINE, density_index=0):
        from dataclasses import replace

        self.sta = sta
        self.cfg = replace(cfg, seed=cfg.seed + seed_offset)
        c = self.cfg
        self.B, self.Hh, self.d = c.B, c.heads, c.d
        self.g = sta.grid(c.T, c.H, c.W)
        self.nt = sta.sta_num_tiles(self.g)
        self.lpad = sta.sta_tiled_len(self.g)
        self.dev = dev
        self.q, self.k, self.v = make_qkv(c, device=dev)
        self._tiled = None  # tiled copies, made only for the reorder / tiled-call measurements
        self.o = torch.empty_like(self.q)
        if c.window_density:
            self.win = torch.from_numpy(window_params(cfg, window_scale(workload, density_index))).to(dev)
        else:
            self.win = None
        self.params = sta.mask_params(c.top_p, c.k_min, c.use_scores, 0.0, c.group_lo, self.win)
        self.bufs = sta.MaskBuffers(self.B, self.Hh, self.d, self.g, dev)
        self.qpairs = None  # the mask build's overlap pairing, when asked for
        # pool, tensor-core scores, select, scan, fill; attention (the tile
        # gather is the TMA box, so no reorder launch)
        self.launches_per_step = 5 + 1

    @property
    def qt(self):
        return self._tiled_bufs()[0]

    @property
    def kt(self):
        return self._tiled_bufs()[1]

    @property
    def vt(self):
        return self._tiled_bufs()[2]

    @property
    def ot(self):
        return self._tiled_bufs()[3]

    def _tiled_bufs(self):
        if self._tiled is None:
            shape_t = (self.B, self.Hh, self.lpad, self.d)
            self._tiled = tuple(torch.empty(shape_t, dtype=torch.bfloat16, device=self.dev) for _ in range(4))
        return self._tiled

    def reorder_in(self, q=None, k=None, v=None):
        s = self.sta
        q, k, v = (self.q if q is None else q), (self.k if k is None else k), (self.v if v is None else v)
        for src, dst in ((q, self.qt), (k, self.kt), (v, self.vt)):
            s.sta_reorder(src, dst, self.B, self.Hh, self.d, self.g)

    def build(self, q=None, k=None):
        """Mask from raster Q, K (sta_build_mask_raster)."""
        self.sta.build_mask(self.q if q is None else q, self.k if k is None else k, self.B, self.Hh, self.d,
                            self.g, self.params, self.bufs, raster=True)

    def attn(self, q=None, k=None, v=None, o=None):
        """Attention on raster Q, K, V into raster O (sta_attn_fwd_raster, or
        sta_attn_fwd_raster_paired with the build's overlap pairing)."""
        args = (self.q if q is None else q, self.k if k is None else k, self.v if v is None else v,
                self.o if o is None else o, None, self.bufs.row_ptr, self.bufs.col_idx)
        if self.qpairs is not None:
            self.sta.sta_attn_fwd_raster_paired(*args, self.qpairs, self.B, self.Hh, self.d, self.g)
        else:
            self.sta.sta_attn_fwd_raster(*args, self.B, self.Hh, self.d, self.g)

    def use_overlap_pairing(self, params_kw):
        """Mask recipe with the build's query-tile pairing by list overlap
        (sta_mask_params.query_pairs); attn() then runs the paired call."""
        if self.qpairs is None:
            self.qpairs = torch.empty((self.B * self.Hh, 2 * ((self.nt + 1) // 2)), dtype=torch.int32,
                                      device=self.dev)
        self.params = self.sta.mask_params(query_pairs=self.qpairs, **params_kw)

    def build_tiled(self):
        self.sta.build_mask(self.qt, self.kt, self.B, self.Hh, self.d, self.g, self.params, self.bufs)

    def attn_tiled(self):
        self.sta.sta_attn_fwd(self.qt, self.kt, self.vt, self.ot, None, self.bufs.row_ptr, self.bufs.col_idx,
                              self.B, self.Hh, self.d, self.g)

    def reorder_out(self, o=None):
        self.sta.sta_reorder(self.ot, self.o if o is None else o, self.B, self.Hh, self.d, self.g,
                             inverse=True)

    def run_e2e(self, hq, hk, hv, ho, steps):
        """End to end from pinned host memory: every step copies its Q, K, V to
        the device, runs the whole path and copies O back to the host. Two sets
        of raster device buffers, and copies on their own streams, let step i+1's
        host-to-device copy and step i-1's device-to-host copy overlap step i's
        kernels. Returns the mean milliseconds per step (CUDA events)."""
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ins = [(self.q, self.k, self.v), tuple(torch.empty_like(x) for x in (self.q, self.k, self.v))]
        outs = [self.o, torch.empty_like(self.o)]
        ev = lambda: torch.cuda.Event()
        in_ready, in_free = [ev(), ev()], [None, None]
        out_ready, out_free = [ev(), ev()], [None, None]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(comp)
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for i in range(steps):
            b = i % 2
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            with torch.cuda.stream(s_in):
                for dst, src in zip(ins[b], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
                in_ready[b].record(s_in)
            comp.wait_event(in_ready[b])
            self.build(ins[b][0], ins[b][1])
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            self.attn(*ins[b], outs[b])
            in_free[b] = ev()
            in_free[b].record(comp)
            out_ready[b].record(comp)
            s_out.wait_event(out_ready[b])
            with torch.cuda.stream(s_out):
                ho.copy_(outs[b], non_blocking=True)
                out_free[b] = ev()
                out_free[b].record(s_out)
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)
        t1.record(comp)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    def step(self, ev=None):
        """One pass of the path on raster Q, K, V: mask, then attention into
        raster O. The 1x8x8 tile gather and scatter happen in the TMA boxes and
        the epilogue, so no reorder pass runs (events 0-1 bracket nothing)."""
        if ev is not None:
            ev[0].record()
            ev[1].record()
        with nvtx_range("sta_build_mask_raster"):
            self.build()
        if ev is not None:
            ev[2].record()
        with nvtx_range("sta_attn_fwd_raster"):
            self.attn()
        if ev is not None:
            ev[3].record()
            ev[4].record()

    def dense_run(self, reps=2):
        """sta_attn_fwd on the same layer with every key tile listed (the dense
        mask): CUDA-event time per launch and TFLOP/s over all Nt^2 pairs."""
        R = self.B * self.Hh * self.nt
        dev = self.qt.device
        rp = (torch.arange(R + 1, device=dev, dtype=torch.int64) * self.nt).to(torch.int32)
        ci = torch.arange(self.nt, device=dev, dtype=torch.int32).repeat(R)
        self.sta.sta_attn_fwd_raster(self.q, self.k, self.v, self.o, None, rp, ci, self.B, self.Hh, self.d,
                                     self.g)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            self.sta.sta_attn_fwd_raster(self.q, self.k, self.v, self.o, None, rp, ci, self.B, self.Hh, self.d,
                                         self.g)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        pairs = R * self.nt
        del rp, ci
        return {"ms": ms, "pairs": pairs, "tflops": pairs * flops_per_pair(self.d) / (ms * 1e-3) / 1e12,
                "density": 1.0}

    def kept_pairs(self):
        return int(self.bufs.nnz.item())

    def query_pairs(self, bh=0, default=False):
        """The two query tiles of each 128-row CTA of head bh: the build's
        overlap pairing when in use (and not `default`), else the attention
        kernel's own: the same spatial tile in frames 2u and 2u+1, and
        right-hand neighbours within the last frame when the frame count is
        odd."""
        if self.qpairs is not None and not default:
            flat = self.qpairs[bh].cpu().numpy()
            return [(int(flat[2 * i]), int(flat[2 * i + 1]) if flat[2 * i + 1] >= 0 else None)
                    for i in range(flat.size // 2)]
        c = self.cfg
        nh, nw = -(-c.H // 8), -(-c.W // 8)
        tpf = nh * nw
        pairs = [(2 * u * tpf + r, (2 * u + 1) * tpf + r) for u in range(c.T // 2) for r in range(tpf)]
        if c.T % 2:
            base = (c.T - 1) * tpf
            pairs += [(base + i, base + i + 1 if i + 1 < tpf else None) for i in range(0, tpf, 2)]
        return pairs

    def pair_union_stats(self, default=False):
        """Pairing efficiency (|A|+|B|) / (2 |A u B|) of the 128-row CTAs."""
        rp = self.bufs.row_ptr.cpu().numpy()
        ci = self.bufs.col_idx[: int(rp[-1])].cpu().numpy()
        nt = self.nt
        tot_ab, tot_u = 0, 0
        for bh in range(self.B * self.Hh):
            for qa, qb in self.query_pairs(bh, default):
                ra = bh * nt + qa
                a = ci[rp[ra]:rp[ra + 1]]
                b = ci[rp[bh * nt + qb]:rp[bh * nt + qb + 1]] if qb is not None else np.zeros(0, np.int32)
                tot_ab += a.size + b.size
                tot_u += np.union1d(a, b).size
        return tot_ab / (2.0 * tot_u) if tot_u else 1.0, tot_u


def search_curve(sta, workload, dev, taus=(0.8, 0.9, 0.95, 0.99), lam=1.0):
    """Recall target against achieved density (Compact Attention Fig. 5(c)):
    exact block masses of the dense layer (dense list, exact LSE), the window
    search for every head at each target, then the window-only mask built from
    the searched windows and the attention on it, compared with the dense
    output (relative Frobenius error over the whole layer)."""
    cfg = CONFIGS[workload]
    layer = Layer(sta, cfg, dev, workload=workload)
    layer.reorder_in()
    B, Hh, d, g, nt = layer.B, layer.Hh, layer.d, layer.g, layer.nt
    R = B * Hh * nt
    rp = (torch.arange(R + 1, device=dev, dtype=torch.int64) * nt).to(torch.int32)
    ci = torch.arange(nt, device=dev, dtype=torch.int32).repeat(R)
    lse = torch.empty((B, Hh, layer.lpad), dtype=torch.float32, device=dev)
    sta.sta_attn_fwd(layer.qt, layer.kt, layer.vt, layer.ot, lse, rp, ci, B, Hh, d, g)
    o_dense = layer.ot.float()
    mass = torch.empty((B, Hh, nt, nt), dtype=torch.float32, device=dev)
    lse2 = torch.empty_like(lse)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sta.sta_attn_fwd_block_mass(layer.qt, layer.kt, layer.vt, layer.ot, lse2, rp, ci, lse, mass, B, Hh, d, g)
    e1.record()
    torch.cuda.synchronize()
    mass_ms = e0.elapsed_time(e1)
    del rp, ci
    G = len(cfg.group_lo)
    rows = []
    for tau in taus:
        win = torch.empty((B * Hh, G, 4), dtype=torch.int32, device=dev)
        stats = torch.empty((B * Hh, 2), dtype=torch.float32, device=dev)
        sta.sta_search_windows(mass, B, Hh, g, cfg.group_lo, tau, lam, win, stats)  # warm-up
        e0.record()
        sta.sta_search_windows(mass, B, Hh, g, cfg.group_lo, tau, lam, win, stats)
        e1.record()
        torch.cuda.synchronize()
        search_ms = e0.elapsed_time(e1)
        st = stats.cpu().numpy()
        params = sta.mask_params(0.0, 0, False, 0.0, cfg.group_lo, win[:Hh])
        sta.build_mask(layer.qt, layer.kt, B, Hh, d, g, params, layer.bufs)
        sta.sta_attn_fwd(layer.qt, layer.kt, layer.vt, layer.ot, None, layer.bufs.row_ptr,
                         layer.bufs.col_idx, B, Hh, d, g)
        torch.cuda.synchronize()
        rel = float(torch.linalg.vector_norm(layer.ot.float() - o_dense) / torch.linalg.vector_norm(o_dense))
        rows.append({"tau": tau, "lambda": lam, "recall_mean": float(st[:, 0].mean()),
                     "recall_min": float(st[:, 0].min()), "density": layer.kept_pairs() / (R * nt),
                     "density_min_head": float(st[:, 1].min()), "density_max_head": float(st[:, 1].max()),
                     "attn_rel_err_vs_dense": rel, "search_ms": search_ms})
    assert sta.sta_get_device_error() == sta.STA_OK
    return {"workload": cfg.name, "block_mass_ms": mass_ms, "curve": rows}


def real_tiled_rows(cfg):
    """Boolean [Lpad]: tiled rows that hold a real token (not grid padding)."""
    nh, nw = -(-cfg.H // 8), -(-cfg.W // 8)
    n = np.arange(cfg.T * nh * nw * 64)
    tile, r = n // 64, n % 64
    rem = tile % (nh * nw)
    y = (rem // nw) * 8 + r // 8
    x = (rem % nw) * 8 + r % 8
    return (y < cfg.H) & (x < cfg.W)


def _median_ms(fn, reps):
    """Median CUDA-event time of `reps` launches of fn (each timed alone)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def sweep(sta, dev, peak, reps=20):
    """Every timed row of the workload table, one JSON line each: the 480p
    window layer, the 720p layer, the 129-frame layer at four window
    densities, and the reuse layer (mask built once from step-0 inputs at
    fixed densities, attention timed on each of the perturbed steps).
    Inputs (Q, K, V tiled, >= 385 MB each) are larger than L2."""
    rows = []

    def attn_line(cfg_name, layer, extra):
        pairs = layer.kept_pairs()
        nt = layer.nt
        ms = _median_ms(layer.attn, reps)
        tf = pairs * flops_per_pair(layer.d) / (ms * 1e-3) / 1e12
        eff, _ = layer.pair_union_stats()
        line = {"workload": cfg_name, "density": pairs / (layer.B * layer.Hh * nt * nt), "kept_pairs": pairs,
                "attn_ms": ms, "attn_tflops": tf, "frac_of_sustained_peak": tf / peak,
                "pairing_efficiency": eff}
        line.update(extra)
        rows.append(line)
        print(json.dumps(line), flush=True)

    def build_extra(layer):
        build_ms = _median_ms(layer.build, reps)
        reo_ms = _median_ms(layer.reorder_in, reps) / 3.0
        c = layer.cfg
        raster = c.B * c.L * c.heads * c.d * 2
        tiled = c.B * c.heads * layer.lpad * c.d * 2
        nnz = layer.kept_pairs()
        build_bytes = (2 * raster if c.use_scores else 0) + 4 * nnz + 4 * (layer.B * layer.Hh * layer.nt + 1)
        return {"build_ms": build_ms, "build_gbs_algorithmic": build_bytes / (build_ms * 1e-3) / 1e9,
                "reorder_ms_per_tensor": reo_ms,
                "reorder_gbs": (raster + tiled) / (reo_ms * 1e-3) / 1e9}

    for wl, dens in (("dit480p", (0,)), (HEADLINE, (0,)), ("dit720p_129f", (0, 1, 2, 3))):
        for di in dens:
            layer = Layer(sta, CONFIGS[wl], dev, workload=wl, density_index=di)
            layer.build()
            extra = build_extra(layer)
            extra["density_target"] = CONFIGS[wl].window_density[di]
            attn_line(CONFIGS[wl].name, layer, extra)
            del layer
            torch.cuda.empty_cache()

    # rectified form on the 720p layer: time, and the error against dense
    # attention of the plain and of the rectified output on the same mask
    layer = Layer(sta, CONFIGS[HEADLINE], dev, workload=HEADLINE)
    layer.reorder_in()
    layer.build_tiled()
    B, Hh, d, g, nt = layer.B, layer.Hh, layer.d, layer.g, layer.nt
    ws_bytes = sta.sta_rectified_workspace(B, Hh, d, g)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    o_rect = torch.empty_like(layer.qt)

    def rect():
        sta.sta_attn_fwd_rectified(layer.qt, layer.kt, layer.vt, o_rect, None, layer.bufs.row_ptr,
                                   layer.bufs.col_idx, ws, ws_bytes, B, Hh, d, g)

    rect_ms = _median_ms(rect, reps)
    plain_ms = _median_ms(layer.attn_tiled, reps)
    o_plain = layer.ot.float()
    R = B * Hh * nt
    rp = (torch.arange(R + 1, device=dev, dtype=torch.int64) * nt).to(torch.int32)
    ci = torch.arange(nt, device=dev, dtype=torch.int32).repeat(R)
    sta.sta_attn_fwd(layer.qt, layer.kt, layer.vt, layer.ot, None, rp, ci, B, Hh, d, g)
    torch.cuda.synchronize()
    o_dense = layer.ot.float()
    real = torch.from_numpy(real_tiled_rows(layer.cfg)).to(dev)

    def rel(a):
        diff = (a - o_dense)[:, :, real]
        return float(torch.linalg.vector_norm(diff) / torch.linalg.vector_norm(o_dense[:, :, real]))

    line = {"workload": CONFIGS[HEADLINE].name + " (rectified form)", "density": layer.kept_pairs() / (R * nt),
            "kept_pairs": layer.kept_pairs(), "rectified_ms": rect_ms, "plain_ms_same_mask": plain_ms,
            "pooled_steps_per_cta": (nt + 63) // 64,
            "rel_err_vs_dense_plain": rel(o_plain), "rel_err_vs_dense_rectified": rel(o_rect.float())}
    rows.append(line)
    print(json.dumps(line), flush=True)
    del layer, o_rect, o_plain, o_dense, ws, rp, ci
    torch.cuda.empty_cache()

    # reuse layer: top_p = 0, k_min = round(rho * Nt), no windows; mask from step 0
    cfg = CONFIGS["reuse480p"]
    layer = Layer(sta, cfg, dev, workload="reuse480p")
    gen = torch.Generator(device=dev).manual_seed(1234)
    masters = [layer.q.float(), layer.k.float()]
    steps_inputs = []
    for _ in range(cfg.reuse_steps):
        qm, qb = perturb_step(masters[0], gen)
        km, kb = perturb_step(masters[1], gen)
        masters = [qm, km]
        steps_inputs.append((qb, kb))
    del masters
    for rho in cfg.fixed_densities:
        k_min = int(round(rho * layer.nt))
        # top-k lists of neighbouring frames overlap less at low density: the
        # build also pairs the query tiles by list overlap, once per reused mask
        layer.use_overlap_pairing(dict(top_p=0.0, k_min=k_min, use_scores=True, group_lo=cfg.group_lo))
        layer.build()
        extra = build_extra(layer)
        per_step = []
        for qb, kb in steps_inputs:
            per_step.append(_median_ms(lambda: layer.attn(qb, kb), max(3, reps // 4)))
        extra.update({"density_target": rho, "k_min": k_min, "reuse_steps": len(per_step),
                      "attn_ms_per_reuse_step": per_step, "pairing": "overlap (sta_mask_params.query_pairs)",
                      "pairing_efficiency_frames": layer.pair_union_stats(default=True)[0]})
        attn_line(cfg.name, layer, extra)
    del layer, steps_inputs
    torch.cuda.empty_cache()
    assert sta.sta_get_device_error() == sta.STA_OK
    return rows


def per_config(sta, dev, peaks, reps=10):
    """Compact record of every other timed layer of the workload table, for
    the default 1-GPU line: the 480p window layer, the 129-frame layer at its
    four window densities and the reuse layer at its five fixed densities
    (mask built once from step-0 inputs; attention over the ten perturbed
    steps). Per row: attention and build medians (CUDA events, each launch
    timed alone, inputs larger than L2), kept-pair TFLOP/s as a fraction of
    the measured burst and sustained bf16 peaks, the pairing efficiency of
    the 128-row CTAs, and the clocks sampled while that row ran."""
    burst = float(peaks.get("bf16_tflops", 1590.0))
    sust = float(peaks.get("bf16_tflops_sustained", burst))
    rows = []

    def record(name, layer, attn_fn, attn_reps, extra):
        clocks = ClockSampler(dev)
        clocks.start()
        h0 = time.monotonic()
        build_ms = _median_ms(layer.build, reps)
        ms = _median_ms(attn_fn, attn_reps)
        clk = clocks.stop(h0, time.monotonic())
        pairs = layer.kept_pairs()
        tf = pairs * flops_per_pair(layer.d) / (ms * 1e-3) / 1e12
        eff, _ = layer.pair_union_stats()
        row = {"workload": name, "density": pairs / (layer.B * layer.Hh * layer.nt ** 2), "kept_pairs": pairs,
               "attn_ms": ms, "attn_tflops": tf, "frac_burst": tf / burst, "frac_sustained": tf / sust,
               "pairing_efficiency": eff, "build_ms": build_ms,
               "clocks": {"sm_mhz": clk.get("sm_mhz"), "power_w_median": clk.get("power_w_median"),
                          "reasons": clk.get("reasons")}}
        row.update(extra)
        rows.append(row)

    for wl, dens in (("dit480p", (0,)), ("dit720p_129f", (0, 1, 2, 3))):
        for di in dens:
            layer = Layer(sta, CONFIGS[wl], dev, workload=wl, density_index=di)
            layer.build()
            record(CONFIGS[wl].name, layer, layer.attn, reps,
                   {"density_target": CONFIGS[wl].window_density[di]})
            del layer
            torch.cuda.empty_cache()

    cfg = CONFIGS["reuse480p"]
    layer = Layer(sta, cfg, dev, workload="reuse480p")
    gen = torch.Generator(device=dev).manual_seed(1234)
    masters = [layer.q.float(), layer.k.float()]
    steps_inputs = []
    for _ in range(cfg.reuse_steps):
        qm, qb = perturb_step(masters[0], gen)
        km, kb = perturb_step(masters[1], gen)
        masters = [qm, km]
        steps_inputs.append((qb, kb))
    del masters
    for rho in cfg.fixed_densities:
        k_min = int(round(rho * layer.nt))
        # top-k lists of neighbouring frames overlap less at low density: the
        # build also pairs the query tiles by list overlap, once per reused mask
        layer.use_overlap_pairing(dict(top_p=0.0, k_min=k_min, use_scores=True, group_lo=cfg.group_lo))
        layer.build()
        it = iter(range(10 ** 9))

        def attn_reuse():
            qb, kb = steps_inputs[next(it) % len(steps_inputs)]
            layer.attn(qb, kb)

        # one launch per perturbed step, in turn, over the mask of step 0
        record(cfg.name, layer, attn_reuse, 2 * len(steps_inputs),
               {"density_target": rho, "k_min": k_min, "reuse_steps": len(steps_inputs),
                "pairing": "overlap (sta_mask_params.query_pairs)",
                "pairing_efficiency_frames": layer.pair_union_stats(default=True)[0]})
    del layer, steps_inputs
    torch.cuda.empty_cache()
    assert sta.sta_get_device_error() == sta.STA_OK
    return rows


def blas_threads():
    """Threads of the BLAS library numpy uses (the oracle's matmuls)."""
    try:
        from threadpoolctl import threadpool_info

        return max((x.get("num_threads", 0) for x in threadpool_info() if x.get("user_api") == "blas"),
                   default=None)
    except Exception:
        return None


def l2_probe(sta, dev, iters=2000):
    """Rate of the attention kernel's load stream on its own (16 KB key-tile
    TMA loads at pseudo-random tiles), from an L2-resident 40 MB region and
    from a 4 GB region, at 1 and 2 CTAs per SM and 2 to 6 loads in flight."""
    from block_sparse_attention_28_b200 import probe

    props = torch.cuda.get_device_properties(dev)
    rows = []
    for label, nbytes in (("L2-resident 40 MB", 40 << 20), ("4 GB (DRAM)", 4 << 30)):
        buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        for cps in (1, 2):
            for slots in (2, 4, 6):
                if slots * 16384 * cps > 200 * 1024:
                    continue
                probe.sta_probe_tma_stream(buf, cps, slots, 50)
                ms = _median_ms(lambda: probe.sta_probe_tma_stream(buf, cps, slots, iters), 5)
                moved = props.multi_processor_count * cps * iters * 16384
                line = {"source": label, "ctas_per_sm": cps, "loads_in_flight_per_cta": slots, "ms": ms,
                        "tb_per_s": moved / (ms * 1e-3) / 1e12}
                rows.append(line)
                print(json.dumps(line), flush=True)
        del buf
        torch.cuda.empty_cache()
    assert probe.sta_probe_get_device_error() == sta.STA_OK
    return rows


def build_roofline(layer, build_ms, peaks):
    """The mask build against HBM: algorithmic bytes = the real rows of Q and
    K read (when scores are on) + the CSR written (col_idx and row_ptr), over
    the build's CUDA-event time, as a fraction of the measured copy
    bandwidth. The select pass is instruction-bound, so the fraction is low
    by design of the work, not by wasted traffic."""
    c = layer.cfg
    raster = c.B * c.L * c.heads * c.d * 2
    nbytes = (2 * raster if c.use_scores else 0) + 4 * layer.kept_pairs() + 4 * (layer.B * layer.Hh * layer.nt + 1)
    achieved = nbytes / (build_ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", 6650.0))
    return {"bound": "hbm", "algorithmic_bytes": nbytes, "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "kernels": "pool_tma, score_tc, select_rows, scan, fill"}


def mma_probe(sta, iters=4096):
    """Cost of one tcgen05.mma (bf16, M = 128, K = 16) of width N = 64, 128,
    256, with A from shared memory or from tensor memory: SM cycles per MMA
    (mean over the SMs, one CTA each) and multiply-adds per clock against the
    SM's dense peak of 4096."""
    from block_sparse_attention_28_b200 import probe

    rows = []
    for a_tmem in (False, True):
        for n in (64, 128, 256):
            probe.sta_probe_mma_rate(n, a_tmem, 64)  # warm-up
            cyc = probe.sta_probe_mma_rate(n, a_tmem, iters).double()
            per = float(cyc.mean()) / iters
            line = {"n": n, "a_operand": "tmem" if a_tmem else "smem", "cycles_per_mma": per,
                    "mac_per_clock": 128 * n * 16 / per, "of_peak": 128 * n * 16 / per / 4096}
            rows.append(line)
            print(json.dumps(line), flush=True)
    assert probe.sta_probe_get_device_error() == sta.STA_OK
    return rows


def cpu_oracle_sample(cfg, layer, budget_s, rows_per_head=8, max_heads=None):
    """Time the oracle (as it stands) on a bounded sample of the same layer:
    for sampled heads, its reorder, pooling, scores, selection and windows
    over the head, then masked attention for sampled query-tile rows.
    Returns (kept-pair flops / s, description, seconds, threads)."""
    import oracle as O

    T, H, W, d = cfg.T, cfg.H, cfg.W, cfg.d
    nt = layer.nt
    win = window_params(cfg, window_scale(HEADLINE, 0))
    rng = np.random.default_rng(123)
    heads = rng.permutation(cfg.heads)
    if max_heads:
        heads = heads[:max_heads]
    t0 = time.perf_counter()
    pairs, nrows, nheads = 0, 0, 0
    for h in heads:
        q = layer.q[:, :, h:h + 1].float().cpu().numpy()
        k = layer.k[:, :, h:h + 1].float().cpu().numpy()
        v = layer.v[:, :, h:h + 1].float().cpu().numpy()
        qt, kt, vt = (O.reorder_fwd(x.astype(np.float64), T, H, W) for x in (q, k, v))
        _, p = O.block_scores(O.pool(qt, T, H, W), O.pool(kt, T, H, W), 1.0 / math.sqrt(d))
        rows = rng.choice(nt, rows_per_head, replace=False)
        wm = O.window_mask(win[h:h + 1], cfg.group_lo, T, H, W)[0]
        mask = np.zeros((1, 1, nt, nt), dtype=bool)
        for r in rows:
            mask[0, 0, r] = O.select_row(p[0, 0, r], cfg.top_p, cfg.k_min) | wm[r]
        rp, ci = O.mask_to_csr(mask)
        O.attention_rows(qt, kt, vt, rp, ci, T, H, W, 1.0 / math.sqrt(d), rows)
        pairs += int(mask.sum())
        nrows += len(rows)
        nheads += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    threads = len(os.sched_getaffinity(0))
    desc = (f"{nheads} head(s) of the 75,600-token layer: full-head reorder, pooling, block scores and "
            f"windows, then selection and masked attention for {nrows} query-tile rows "
            f"({pairs} kept pairs)")
    return pairs * flops_per_pair(d) / dt / 1e12, desc, dt, threads


def run_reference(args, rank, world):
    """The CPU oracle timed as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    cfg = CONFIGS[HEADLINE]

    class _Stub:
        pass

    layer = _Stub()
    layer.q, layer.k, layer.v = make_qkv(cfg, device="cpu")
    from workloads import tile_counts

    layer.nt = tile_counts(cfg.T, cfg.H, cfg.W)[2]
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, layer, 1.0, rows_per_head=2, max_heads=1)
    vals, times = [], []
    desc = ""
    threads = 0
    for _ in range(args.steps):
        v, desc, dt, threads = cpu_oracle_sample(cfg, layer, 10.0, rows_per_head=4, max_heads=1)
        vals.append(v)
        times.append(dt)
    value = float(statistics.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded random-Fourier-feature Q/K, Gaussian V)",
        "config": {"workload": CONFIGS[HEADLINE].name, "tokens": cfg.L, "heads": cfg.heads, "d": cfg.d,
                   "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "blas_threads": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--no-launch-count", action="store_true",
                    help="skip the CUPTI count of one step's kernels (for runs under ncu); "
                         "gpu_launches is then the static count")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=16,
                    help="pipelined end-to-end steps (fill and drain are amortised over them)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-mask run of the same kernel")
    ap.add_argument("--nvtx", action="store_true", help="NVTX ranges around the calls of each step")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-config record of the other workload layers (1 GPU only)")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(CONFIGS),
                    help="workload (profiling of smaller layers); the headline is the 720p layer")
    ap.add_argument("--density-index", type=int, default=0)
    ap.add_argument("--heads", type=int, default=0,
                    help="use only this many heads of the workload (small cases for ncu captures)")
    ap.add_argument("--sweep", action="store_true",
                    help="time every layer of the workload table (one JSON line per row) and exit")
    ap.add_argument("--l2-probe", action="store_true",
                    help="rate of the attention's 16 KB TMA tile loads on their own, then exit")
    ap.add_argument("--mma-probe", action="store_true",
                    help="cycles per tensor-core MMA (bf16, M=128, K=16) for N = 64 / 128 / 256")
    ap.add_argument("--search-curve", action="store_true",
                    help="print the recall-target vs density curve of the window search and exit")
    args = ap.parse_args()
    global NVTX
    NVTX = args.nvtx

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import block_sparse_attention_28_b200 as sta

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.l2_probe:
        if rank == 0:
            l2_probe(sta, dev)
        return
    if args.mma_probe:
        if rank == 0:
            mma_probe(sta)
        return
    if args.sweep:
        if rank == 0:
            peaks, _ = load_peaks()
            sweep(sta, dev, float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))))
        return
    if args.search_curve:
        if rank == 0:
            print(json.dumps(search_curve(sta, args.workload, dev)), flush=True)
        return
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = CONFIGS[args.workload]
    if args.heads > 0:
        from dataclasses import replace

        cfg = replace(cfg, heads=args.heads)
    layer = Layer(sta, cfg, dev, seed_offset=rank, workload=args.workload,
                  density_index=args.density_index)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        layer.step()
    barrier()
    assert sta.sta_get_device_error() == sta.STA_OK
    n_launch, step_kernels = (None, None) if args.no_launch_count else count_step_launches(layer)
    launch_src = "cupti, one untimed step"
    if n_launch is None:
        n_launch, launch_src = layer.launches_per_step, "static count"
    barrier()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.1)
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    h0 = time.monotonic()
    t_start.record()
    for i in range(K):
        layer.step(evs[i])
    t_end.record()
    barrier()
    h1 = time.monotonic()
    clk = clocks.stop(h0, h1)
    elapsed_ms = t_start.elapsed_time(t_end)
    assert sta.sta_get_device_error() == sta.STA_OK

    build_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    elapsed_ms = max_over_ranks(elapsed_ms, dev, world)
    pairs = layer.kept_pairs()
    nt = layer.nt
    density = pairs / (layer.B * layer.Hh * nt * nt)
    flops = pairs * flops_per_pair(layer.d)
    total_flops = sum_over_ranks(flops, dev, world)
    value = whole_job_tflops(total_flops, K, elapsed_ms)
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12

    # end to end through the C ABI from pinned host buffers (H2D in, D2H out)
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv = (x.cpu().pin_memory() for x in (layer.q, layer.k, layer.v))
        ho = torch.empty(layer.o.shape, dtype=layer.o.dtype, pin_memory=True)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
        d2h = ho.numel() * ho.element_size()
        layer.run_e2e(hq, hk, hv, ho, 2)  # warm-up of the streams and second buffer set
        barrier()
        e2e_local = layer.run_e2e(hq, hk, hv, ho, args.e2e_steps)
        barrier()
        # every step read the same inputs: the host copy of O is the path's output
        assert torch.equal(ho.view(torch.int16), layer.o.cpu().view(torch.int16))
        e2e_ms = max_over_ranks(e2e_local, dev, world)
        e2e = {"value": whole_job_tflops(total_flops, 1, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    # the same kernel with every key tile listed (dense-mask run), outside the timed region
    dense = None
    if rank == 0 and not args.no_dense:
        dense = layer.dense_run(reps=2)

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    peak_burst = float(peaks.get("bf16_tflops", peak))
    eff, union_tiles = layer.pair_union_stats() if rank == 0 else (None, None)
    line = None
    per_cfg = None
    if rank == 0 and world == 1 and not args.no_per_config and args.workload == HEADLINE and args.heads == 0:
        per_cfg = per_config(sta, dev, peaks)
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline and args.workload == HEADLINE:
            v_cpu, desc, dt, threads = cpu_oracle_sample(cfg, layer, args.cpu_budget)
            cpu = {"value": v_cpu, "unit": UNIT, "cores": threads, "blas_threads": blas_threads(),
                   "kind": "oracle", "sample": f"{desc}; {dt:.1f} s"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-Fourier-feature Q/K, Gaussian V; no dataset)",
            "config": {
                "workload": cfg.name, "tokens": cfg.L, "padded_tokens": layer.lpad, "heads": cfg.heads,
                "d": cfg.d, "grid": [cfg.T, cfg.H, cfg.W], "top_p": cfg.top_p, "k_min": cfg.k_min,
                "density": density, "kept_pairs": pairs, "global_batch": world * cfg.B,
                "parallelism": f"independent layer per GPU x{world}",
                "l2": "inputs (Q,K,V 2.3 GB) larger than L2; no flush",
                "step": ("build_mask_raster (pool, scores, selection, windows, CSR) + attn_fwd_raster; "
                         "the 1x8x8 tile gather of Q/K/V and scatter of O are the attention kernel's "
                         "5D TMA boxes and epilogue stores, so no reorder pass runs"),
            },
            "ms_per_layer": build_ms + attn_ms,
            "ms_breakdown": {"build_mask": build_ms, "attn_fwd": attn_ms},
            "build_roofline": build_roofline(layer, build_ms, peaks),
            "attn_tflops": attn_tflops,
            "attn_frac_of_peak": attn_tflops / peak,
            "pairing_efficiency": eff,
            "dense_mask_run": dense,
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / peak, "frac_burst": attn_tflops / peak_burst,
                         "peak_burst": peak_burst, "traffic": load_traffic(),
                         "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
                         "kernel": "attn_fwd_kernel<128, MASS=false, RASTER=true>",
                         "algorithmic": f"{pairs} kept pairs x 4*64*64*{cfg.d} flop"},
            "cpu_baseline": cpu,
            "per_config": per_cfg,
            "e2e": e2e,
            "gpu_launches": K * n_launch,
            "gpu_launches_source": launch_src,
            "step_kernels": step_kernels,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
