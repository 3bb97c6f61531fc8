#!/usr/bin/env python
"""Render + analytic score replay throughput on B200.

One step = the whole path over one synthetic scene: preprocess (EWA projection, SH colour),
tile binning + depth sort, front-to-back compositing, score replay + token finalisation, for all
target views. Default workload: the DepthSplat-scale dense scene (5,898,240 Gaussians, SH degree
3, 4 target views 512x960). Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--impl ours|reference]
                  [--path score|backward|attributes] [--cpu-threads T]

--impl reference times the CPU oracle instead (one whole view per step, all host cores or T);
the default arm reports the same oracle timing once as its cpu_baseline, and (score path)
compares that view, element by element, with the CUDA path run on the same view alone
(parity_vs_oracle).

Timing: K timed steps with the library's per-kernel event pairs off give value, ms_per_step and
its median and minimum; K more with them on give the per-kernel times, the rooflines and
ms_per_step_with_kernel_events. Clocks are sampled during both.

--path backward times the renderer backward instead of the score replay (the gradient comparators:
raw, detached, support- and parameter-scale-normalised gradients, all four per step).
--path attributes times the attribute path instead: a 9-channel attribute render, the scatter of
a 9-channel per-pixel map back to the Gaussians, and the scalar attribution (coverage, error).

Multi-GPU: one process per GPU (torchrun); every rank renders and scores its own replica of the
workload (no data-path collective); value = all ranks' pixels / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "render+score-replay Mpix/s & Gaussian-pixel pairs/s; % of FP32/HBM roofline"
METRICS = {"score": METRIC,
           "backward": "render+backward Mpix/s & Gaussian-pixel pairs/s; % of FP32/HBM roofline",
           "attributes": "render+attributes Mpix/s & Gaussian-pixel pairs/s; % of FP32/HBM roofline"}
N_ATTR = 9  # attribute channels of the attributes path (learned feature channels beside RGB)
PATHS = {"score": "render+score_replay+tokens",
         "backward": "render+backward+gradients(raw,detached,support,pscale)",
         "attributes": "render+attribute_render(9ch)+scatter(9ch)+attribution"}
WORKLOADS = {
    1: "two_plane_occlusion_64x64_1v_256g",
    2: "three_layer_occlusion_128x128_4v_4096g",
    3: "resplat_pixel_aligned_256x448_8v_917504g_sh2",
    4: "atsplat_anchor_512x960_4v_311296g_sh2",
    5: "depthsplat_dense_512x960_4v_5898240g_sh3",
}


def make_scene(args):
    from synth import scenes
    return scenes.resplat_views(args.views) if args.views else scenes.make(args.config)


def workload_name(args, sc) -> str:
    if args.views:
        return f"resplat_pixel_aligned_256x448_{sc.V}v_{sc.G}g_sh2"
    return WORKLOADS[args.config]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--path", choices=["score", "backward", "attributes"], default="score")
    ap.add_argument("--shard", choices=["replicas", "views"], default="replicas",
                    help="views: each rank renders and replays its block of the views and one "
                         "reduce-scatter of the per-Gaussian partial sums gives every rank its "
                         "slice of tokens (strong scaling over views; score path only)")
    ap.add_argument("--deterministic", action="store_true",
                    help="fixed-point integer accumulation (bitwise reproducible sums)")
    ap.add_argument("--views", type=int, default=0,
                    help="view-count scaling: the ReSplat-scale layout with this many context and "
                         "target views at 256x448 (overrides --config)")
    ap.add_argument("--unfused", action="store_true",
                    help="score path: splat_render then splat_score_replay (two kernels) instead "
                         "of splat_render_score (one kernel)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="OpenMP threads of the CPU oracle (0 = all host cores)")
    return ap.parse_args()


# ----------------------------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    """nvidia-smi samples of the SM clock and the throttle reasons, kept only when they arrived
    inside the timed region (mark() .. stop())."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 100
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[tuple[float, str]] = []  # (arrival time, line)
        self.t0 = None
        self._first = threading.Event()

    def start(self, wait_s: float = 5.0):
        """Start sampling and wait (up to wait_s) for the first sample, so that sampling is live
        before the timed region begins."""
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", str(self.INTERVAL_MS)]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        self._first.wait(wait_s)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))
            self._first.set()

    def mark(self):
        """The timed region starts now."""
        self.t0 = time.monotonic()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t1 = time.monotonic()
        time.sleep(2 * self.INTERVAL_MS / 1e3)  # let a sample taken at the end arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0 = self.t0 if self.t0 is not None else 0.0
        return self.summarize(list(self.lines), t0, t1 + self.INTERVAL_MS / 1e3)

    @classmethod
    def summarize(cls, lines, t0: float, t1: float) -> dict:
        """Median SM clock, largest max clock and the throttle reasons seen in the samples that
        arrived in [t0, t1]. A region shorter than the sampling interval may hold none: then the
        first sample after t0 stands for it, and `window` says so."""
        parsed = []
        for t, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            act = {n for n, p in zip(cls.REASONS, parts[3:7]) if p.lower().startswith("active")}
            parsed.append((t, sm, smax, act))
        inside = [x for x in parsed if t0 <= x[0] <= t1]
        window = "timed region"
        if not inside:
            after = [x for x in parsed if x[0] >= t0]
            inside = after[:1]
            window = "first sample after the timed region began" if inside else "no sample"
        return {"sm_mhz": statistics.median(x[1] for x in inside) if inside else None,
                "sm_max_mhz": max(x[2] for x in inside) if inside else None,
                "reasons": sorted(set().union(*(x[3] for x in inside))) if inside else [],
                "samples": len(inside), "window": window,
                "interval_ms": cls.INTERVAL_MS}


def gpu_id_for(dev) -> str | None:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ----------------------------------------------------------------------------------------------
# roofline bookkeeping (algorithmic bytes / work per launch; see the design notes)

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def code_text(src: str) -> str:
    """C/C++/CUDA source with its comments removed (each replaced by one space, as the compiler
    does), trailing blanks cut and empty lines dropped: what remains is the code the compiler
    sees, so rewording a comment leaves it unchanged while any change to the code changes it.
    String and character literals are copied as they are."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == "/" and src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif c == "/" and src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c and src[j] != "\n":
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def code_digest(paths) -> str:
    """sha256 over the code (code_text) of the given repository files, in order."""
    import hashlib
    m = hashlib.sha256()
    for f in paths:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            m.update(code_text(fh.read()).encode())
        m.update(b"\0")
    return m.hexdigest()


def _current_record(fname: str, kernel: str, workload: str):
    """A kernel's entry of a committed ncu record under profiles/, only when it was captured on
    this workload and the code of the kernel's sources (comments aside) is still what was
    captured."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", fname)))["kernels"][kernel]
    except (OSError, KeyError, ValueError):
        return None
    if d.get("workload") != workload:
        return None
    try:
        if code_digest(d["sources"]) != d["code_sha256"]:
            return None
    except (OSError, KeyError, UnicodeDecodeError):
        return None
    return d


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture (profiles/dram_traffic.json)."""
    d = _current_record("dram_traffic.json", kernel, workload)
    return None if d is None else int(d["dram_read_bytes"]) + int(d["dram_write_bytes"])


def recorded_pipes(kernel: str, workload: str):
    """ncu pipe utilisation of the kernel (profiles/pipe_counters.json): FMA-pipe and ALU-pipe
    cycles active and issue slots used, in % of peak sustained, from one captured launch."""
    d = _current_record("pipe_counters.json", kernel, workload)
    if d is None:
        return None
    return {k: d[k] for k in ("fma_pipe_pct", "alu_pipe_pct", "issue_active_pct") if k in d}


def algorithmic_bytes(sc, n_inst: int, pairs: int, depth_passes: int = 3) -> dict:
    """Bytes each kernel group must move by its definition, per step; depth_passes = the number of
    depth-digit passes the binning ran. The projection and the finalisation use the per-unit
    figures of the path's scope table (projection: the parameters read once, 4 (11 + 3d) B per
    Gaussian, and ~52 B written per (view, Gaussian); finalisation: 28 + 16 B read per (view,
    Gaussian) and the (9 + 3d) x 4 B token written per Gaussian); the binning kernels, which
    replace the table's 43-bit instance sort, count their own unique inputs and outputs."""
    G, V, H, W, d = sc.G, sc.V, sc.H, sc.W, sc.d
    px = V * H * W
    TX, TY = (W + 15) // 16, (H + 15) // 16
    return {
        "project": G * 4 * (11 + 3 * d) + V * G * 52,

        # one depth-digit pass per launch over every (v, g): histogram reads the keys, the
        # scatter reads key + index and writes both
        "depth_hist": depth_passes * V * G * 4,
        # per pass keys and values in and out; the first reads no values (the index is implicit),
        # the last writes no keys
        "depth_scatter": max(depth_passes * 16 - 8, 0) * V * G,
        # rectangles (4 x 16 bit) gathered into depth order (order 4 B + rectangle 8 B in, 8 B +
        # count 4 B out), the counts scanned in place (4 B in, 4 B out), instances (tile, g)
        # emitted (rectangle, index, offset in; 8 B out)
        "emit": V * G * (12 + 12 + 8 + 16) + n_inst * 8,
        "tile_hist": n_inst * 4,
        "tile_scatter": n_inst * (4 + 4 + 4),
        # gather 36 B per list entry staged, write C_hat, T, n, last
        "render": n_inst * (4 + 36) + px * 24,
        # render and replay in one kernel: the list entries gathered by both phases, C_hat, T,
        # n, last written, C_obs read, 32 B of sums per (v, g)
        "render_replay": n_inst * 2 * (4 + 36) + px * (24 + 12) + V * G * 32,
        # gather 36 B per list entry, read C_hat, C_obs, the list bound and the contributor
        # count per pixel, add into 32 B of sums per (v, g)
        "replay": n_inst * (4 + 36) + px * (12 + 12 + 4 + 4) + V * G * 32,
        "finalize": V * G * (28 + 16) + G * 4 * (9 + 3 * d),
        # backward: list entries as the replay, per pixel C_hat, C_obs, T_final, last; ten fp64
        # sums per (v, g); the chain reads records (48 B) and sums (80 B) per (v, g), the
        # parameters, and writes four gradient rows
        "backward": n_inst * (4 + 36) + px * (12 + 12 + 4 + 4) + V * G * 80,
        "grad": V * G * (48 + 80) + G * (12 + 16 + 12 * d) + 4 * G * 4 * (11 + 3 * d),
        # attributes: list entries as the replay; per pixel the list bound and 9 channels out
        # (render) or in (scatter) or C_hat, C_obs in (attribution); 9 attributes read per
        # composited entry (from cache: per (v, g) counted once), 9 / 2 fp64 sums per Gaussian
        "features": n_inst * (4 + 36) + px * (4 + 4 * N_ATTR) + V * G * 4 * N_ATTR,
        "scatter": 2 * n_inst * (4 + 36) + px * (4 + 4 * N_ATTR + 4 + 24) + G * 8 * (N_ATTR + 2),
        "tiles": V * TX * TY,
    }


# Algorithmic fp32 work of the list-walking kernels, in lane operations (an fma is one; the
# exponential is the Cody-Waite one both sides use: x log2(e) and its rounding, two reduction fmas,
# a degree-7 Horner polynomial, the scale = 12), counted from the method's arithmetic by pair
# class. The render must decide every traversed (pixel, list entry) pair: the exponent of G and
# the skip decision (p - mu2D, the conic's quadratic form, the positive-exponent test and the
# comparison with the Gaussian's precomputed exponent cut that decides alpha < 1/255 without the
# exponential = 13). The later passes are handed the render's decisions (its per-pixel masks of
# composited entries) and walk only the composited pairs, except the map scatter and the
# attribution, which still visit every entry their warp's pixels composited. Each composited pair
# needs alpha = min(0.99, o exp(pw)) and the 1/255 test (15) and then its pass's own work:
#   render    T (1 - alpha), the stop test, w = alpha T, C += w c (unfused)                 = 10
#   replay    T (1 - alpha), w, w c, C_hat - P - w c (3 channels), the reciprocal of the
#             denominator, c - C+ (3 fmas), rho, both masks, w r, w rho, w rho d, P += w c  = 31
#   backward  1 / (1 - alpha), T, w, w r, <r, c> T - <r, S> / (1 - alpha), h = ga alpha,
#             h d, h d d^T (3), S += w c                                                    = 28
#   features  T (1 - alpha), w, 9 channels (mul, add)                                       = 21
#   scatter   two traversals: the 9-channel map (T, w, 9 products) and the attribution
#             (T, w, w, w |r|)                                                             = 12 + 5
# so a kernel's work per step = a x traversed pairs + b x composited pairs with (a, b) below.
ALU_OPS = {"render": (13, 25), "replay": (0, 46), "backward": (0, 43), "features": (0, 36),
           "scatter": (26, 47), "render_replay": (13, 25 + 46)}
# the backward visits its warps' union entries but, like the replay, is handed the render's
# decisions: its work is counted over the composited pairs; render_replay is the render and the
# replay in one kernel (splat_render_score)

def alu_ops(kernel: str, pairs: int, composited: int) -> int:
    a, b = ALU_OPS[kernel]
    return a * pairs + b * composited


# ----------------------------------------------------------------------------------------------
# CPU oracle baseline: one whole view of the workload, timed as it runs

def cpu_oracle_view(sc, obs_np, path="score", threads=0, keep_outputs=False):
    """The oracle (fp32 decision mode, OpenMP) over one complete view of the workload: projection
    and binning of every Gaussian into view 0, render and the pass of `path` over every tile of
    that view, and the per-Gaussian finalisation. Nothing is sampled or scaled: value = the
    view's pixels / the measured wall time. threads > 0 sets the oracle's OpenMP thread count.
    keep_outputs (score path): also return the view's image, final transmittance, contributor
    counts and tokens under "outputs", for the whole-view comparison with the CUDA path."""
    import numpy as np
    from oracle import oracle as O
    if threads > 0:
        O.lib().orc_set_threads(int(threads))
    one = _one_view(sc)
    t0 = time.perf_counter()
    p = O.project(one, "f")
    L = O.bin_lists(p, one.H, one.W)
    t_pb = time.perf_counter() - t0
    t1 = time.perf_counter()
    r = O.render(p, L, one.H, one.W, one.bg, "f")
    t_r = time.perf_counter() - t1
    if path == "backward":
        accb = O.backward(p, L, r, obs_np[:1], one.bg, one.H, one.W, "f")
    elif path == "attributes":
        rng2 = np.random.default_rng(1)
        f = rng2.uniform(0, 1, (one.G, N_ATTR)).astype(np.float32)
        m = rng2.uniform(0, 1, (1, one.H, one.W, N_ATTR)).astype(np.float32)
        O.render_features(p, L, r, f, one.H, one.W, "f")
        O.scatter(p, L, r, m, one.H, one.W, "f")
        O.attribution(p, L, r, obs_np[:1], one.H, one.W, "f")
    else:
        rp = O.replay(p, L, r, obs_np[:1], one.sh_degree, one.H, one.W, "f")
    t_rr = time.perf_counter() - t1
    t2 = time.perf_counter()
    tokens = None
    if path == "backward":
        O.gradients(p, accb, one, "f")
    elif path == "score":
        tokens = O.finalize(p, rp["acc"], one)
    t_fin = time.perf_counter() - t2
    second = {"backward": "backward", "attributes": "attribute render + scatters",
              "score": "replay"}[path]
    last = {"backward": "gradient chain", "attributes": "nothing further",
            "score": "finalisation"}[path]
    t_view = t_pb + t_rr + t_fin
    outputs = None
    if keep_outputs and path == "score":
        outputs = {"img": r["img"], "T": r["T"], "n_contrib": r["n_contrib"], "tokens": tokens}
    return {"value": one.H * one.W / t_view / 1e6, "unit": "Mpix/s",
            "cores": int(O.lib().orc_num_threads()), "kind": "oracle",
            "sample": (f"view 1 of {sc.V}, whole: projection + binning of all {sc.G} Gaussians "
                       f"({1e3 * t_pb:.1f} ms), render of all {one.H}x{one.W} pixels "
                       f"({1e3 * t_r:.1f} ms), {second} ({1e3 * (t_rr - t_r):.1f} ms), {last} "
                       f"({1e3 * t_fin:.1f} ms)"),
            "seconds": t_view, "outputs": outputs}


def _one_view(sc):
    import dataclasses
    return dataclasses.replace(sc, viewmats=sc.viewmats[:1], intrin=sc.intrin[:1])


def token_blocks(d: int) -> dict:
    """Column ranges of the token's blocks: [b (3), s^alpha, s^SH (3d), log q, eig (3), log tr]."""
    return {"b_mu": (0, 3), "s_alpha": (3, 4), "s_sh": (4, 4 + 3 * d),
            "log_q": (4 + 3 * d, 5 + 3 * d), "eig": (5 + 3 * d, 8 + 3 * d),
            "log_tr": (8 + 3 * d, 9 + 3 * d)}


COLOUR_ATOL, TOKEN_RTOL, NORM_FLOOR = 1e-5, 1e-4, 1e-3


def parity_report(g: dict, o: dict, d: int, chunk: int = 1 << 16) -> dict:
    """Element-by-element comparison of one whole view of the workload, CUDA path (g) against the
    oracle in fp32 decision mode (o); d = SH coefficients per channel ((degree + 1)^2): image,
    final transmittance, contributor counts and every Gaussian's token. The bars are the parity
    tests': colour within 1e-5 absolute, transmittance and counts exact, tokens within 1e-4
    relative L2 per Gaussian (floor 1e-3 x the median token norm); per token block the same ratio
    with the block's own floor (1e-3 x its median non-zero norm). Also the correctness metrics the
    experiment plan names for its score check ("Block 0": sign accuracy, blockwise cosine), over
    the Gaussians with q_g >= 1e-3: the fraction of token entries whose sign agrees (entries
    larger than 1e-4 of their token's norm) and each block's cosine between the two sides.
    Reported, not asserted: the tests assert."""
    import numpy as np
    img_err = float(np.abs(g["img"].astype(np.float64) - o["img"]).max(initial=0.0))
    t_mis = int((g["T"] != np.asarray(o["T"]).astype(np.float32)).sum())
    nc_mis = int((g["n_contrib"] != o["n_contrib"]).sum())
    zg, zo = g["tokens"], o["tokens"]
    G = zo.shape[0]
    if zg.shape != zo.shape or zo.shape[1] != 9 + 3 * d:
        raise ValueError(f"token arrays {zg.shape} / {zo.shape} for {d} SH coefficients")
    blocks = token_blocks(d)
    names = list(blocks)

    def block_norms(x):  # [n, K] -> [n, blocks] L2 norms of each block, and [n] of the row
        sq = np.stack([np.einsum("ij,ij->i", x[:, a:b], x[:, a:b]) for a, b in blocks.values()],
                      axis=1)
        return np.sqrt(sq), np.sqrt(sq.sum(axis=1))

    bn = np.empty((G, len(names)))
    norms = np.empty(G)
    for s in range(0, G, chunk):
        bn[s:s + chunk], norms[s:s + chunk] = block_norms(np.asarray(zo[s:s + chunk], np.float64))

    def floor_of(n):
        nz = n[n > 0]
        return NORM_FLOOR * (float(np.median(nz)) if nz.size else 0.0) or 1e-30

    floor = floor_of(norms)
    bfloor = np.array([floor_of(bn[:, i]) for i in range(len(names))])
    covered = np.exp(np.asarray(zo[:, 4 + 3 * d], np.float64)) >= 1e-3  # q_g >= 1e-3
    err = np.empty(G)
    be = np.empty((G, len(names)))
    cos = np.full((G, len(names)), np.nan, np.float32)
    n_sign = n_agree = 0
    for s in range(0, G, chunk):
        a64 = np.asarray(zg[s:s + chunk], np.float64)
        b64 = np.asarray(zo[s:s + chunk], np.float64)
        dbn, dn = block_norms(a64 - b64)
        err[s:s + chunk] = dn / np.maximum(norms[s:s + chunk], floor)
        be[s:s + chunk] = dbn / np.maximum(bn[s:s + chunk], bfloor)
        cov = covered[s:s + chunk]
        big = (np.abs(b64) > 1e-4 * norms[s:s + chunk, None]) & cov[:, None]
        n_sign += int(np.count_nonzero(big))
        n_agree += int(np.count_nonzero(big & (a64 * b64 > 0)))  # b != 0 where big
        gbn, _ = block_norms(a64)
        dots = np.stack([np.einsum("ij,ij->i", a64[:, a:b], b64[:, a:b])
                         for a, b in blocks.values()], axis=1)
        den = gbn * bn[s:s + chunk]
        with np.errstate(invalid="ignore", divide="ignore"):
            c = np.where(den > 0, dots / den, np.nan)
        c[~cov] = np.nan
        cos[s:s + chunk] = c
    berr = {k: be[:, i] for i, k in enumerate(names)}
    ok = err <= TOKEN_RTOL

    def cos_stat(i, f):
        v = cos[:, i]
        v = v[~np.isnan(v)]
        return float(f(v)) if v.size else None

    def q(a, p):
        return float(np.percentile(a, p)) if a.size else 0.0

    return {"pixels": int(np.asarray(o["n_contrib"]).size), "gaussians": int(G),
            "colour_max_abs_err": img_err, "colour_bar": COLOUR_ATOL,
            "T_final_mismatches": t_mis, "n_contrib_mismatches": nc_mis,
            "token_rel_err_max": float(err.max(initial=0.0)), "token_rel_err_p99": q(err, 99),
            "token_bar": TOKEN_RTOL,
            "token_block_rel_err_max": {k: float(v.max(initial=0.0)) for k, v in berr.items()},
            "token_block_rel_err_p99": {k: q(v, 99) for k, v in berr.items()},
            "gaussians_qg_ge_1e-3": int(covered.sum()),
            "frac_pass_qg_ge_1e-3": float(ok[covered].mean()) if covered.any() else None,
            "frac_pass_all": float(ok.mean()) if G else None,
            "sign_agreement_qg_ge_1e-3": n_agree / n_sign if n_sign else None,
            "block_cosine_min_qg_ge_1e-3": {k: cos_stat(i, np.min) for i, k in enumerate(names)},
            "block_cosine_median_qg_ge_1e-3": {k: cos_stat(i, np.median)
                                               for i, k in enumerate(names)}}


def gpu_view_outputs(sc, obs, fused: bool, deterministic: bool) -> dict:
    """The CUDA path over view 0 of the workload alone (its own workspace), as host arrays."""
    import torch
    from gaussian_splatting_raster_b200 import runner
    ds1 = runner.to_device(_one_view(sc))
    ws1 = runner.workspace_for(ds1)
    try:
        if deterministic:
            ws1.deterministic(True)
        out1 = runner.alloc_outputs(ds1)
        runner.render_and_score(ws1, ds1, obs[:1].contiguous(), out1, fused=fused)
        torch.cuda.synchronize()
        return {"img": out1.img.cpu().numpy(), "T": out1.T.cpu().numpy(),
                "n_contrib": out1.n_contrib.cpu().numpy(), "tokens": out1.tokens.cpu().numpy()}
    finally:
        ws1.close()


# ----------------------------------------------------------------------------------------------

def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


def pairs_sum_over_ranks(x: int, world: int) -> int:
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def max_over_ranks(x: float, world: int) -> float:
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args):
    """Reference arm: the CPU oracle, as it stands, one whole view of the same workload per step
    (every Gaussian projected and binned, every pixel rendered and replayed, every Gaussian
    finalised); ms_per_step is the mean measured time of those steps."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synth import scenes
    sc = make_scene(args)
    obs = scenes.smooth_observation(99, 1, sc.H, sc.W)
    times, samples = [], []
    for it in range(args.warmup + args.steps):
        s = cpu_oracle_view(sc, obs, path=args.path, threads=args.cpu_threads)
        if it >= args.warmup:
            times.append(s["seconds"])
            samples.append(s)
    # one step = one whole view, as it ran: steps x ms_per_step is the timed work
    ms = 1e3 * sum(times) / len(times)
    val = sc.H * sc.W * len(times) / sum(times) / 1e6
    line = {"metric": METRICS[args.path], "value": val, "unit": "Mpix/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(args, sc), "views_per_step": 1,
                       "path": PATHS[args.path], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": val, "unit": "Mpix/s", "cores": samples[0]["cores"],
                             "kind": "oracle", "sample": samples[0]["sample"]},
            "e2e": {"value": val, "unit": "Mpix/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    # Libraries (NCCL's version banner, for one) may write to stdout; the contract is one JSON
    # line there, so everything else goes to stderr and the line is written to the saved stdout.
    sys.stdout.flush()
    json_fd = os.dup(1)
    os.dup2(2, 1)
    import numpy as np
    import torch

    import gaussian_splatting_raster_b200 as P
    from gaussian_splatting_raster_b200 import runner
    from synth import scenes

    rank, world, local = dist_setup()
    dev = torch.device("cuda", torch.cuda.current_device())
    P.load_library()  # built in-tree by __graft_entry__.build(); fails loudly when missing
    sc = make_scene(args)
    ds = runner.to_device(sc)
    shard = args.shard == "views"
    if shard and args.path != "score":
        raise SystemExit("--shard views times the score path only")
    if shard and world == 1:
        import socket
        import torch.distributed as dist
        s_ = socket.socket()
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
        s_.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, device_id=dev)
    # observation: render of the perturbed scene (+ pixel noise), made by the same path, untimed
    obs_scene = runner.to_device(sc.observed_scene())
    obs_out = runner.alloc_outputs(obs_scene)
    ws_obs = runner.workspace_for(obs_scene)
    runner.render(ws_obs, obs_scene, obs_out)
    obs = obs_out.img.clone()
    if sc.obs_noise_sigma > 0:
        obs += torch.from_numpy(sc.pixel_noise()).to(dev)
    torch.cuda.synchronize()
    ws_obs.close()
    del obs_scene, obs_out, ws_obs
    if shard:
        from gaussian_splatting_raster_b200 import sharding
        vlo, vhi = sharding.view_ranges(sc.V, world)[rank]
        ws = P.Workspace(max(ds.G, 1), max(vhi - vlo, 1), ds.H, ds.W, ds.deg)
    else:
        ws = runner.workspace_for(ds)
    out = runner.alloc_outputs(ds)
    if args.deterministic:
        ws.deterministic(True)

    stream = torch.cuda.current_stream()
    l2_flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    K = P.grad_dim(ds.deg)

    def alloc_grads():
        return {k: torch.empty((ds.G, K), dtype=torch.float32, device=dev)
                for k in ("raw", "detached", "support", "pscale")}

    grads = alloc_grads() if args.path == "backward" else None
    if args.path == "attributes":
        gen = torch.Generator(device=dev).manual_seed(1)
        feats = torch.rand((ds.G, N_ATTR), generator=gen, device=dev)
        pmap = torch.rand((ds.V, ds.H, ds.W, N_ATTR), generator=gen, device=dev)

    def alloc_attr():
        return {"F": torch.empty((ds.V, ds.H, ds.W, N_ATTR), device=dev),
                "S": torch.empty((ds.G, N_ATTR), device=dev),
                "A": torch.empty((ds.G, 3), device=dev)}

    attr_out = alloc_attr() if args.path == "attributes" else None

    def run(ds_, obs_, out_, grads_, attr_):
        if args.path == "backward":
            return runner.render_and_backward(ws, ds_, obs_, out_, grads_)
        if args.path == "attributes":
            n = runner.render(ws, ds_, out_)
            ws.render_features(feats, attr_["F"])
            ws.scatter(pmap, attr_["S"])
            ws.attribution(obs_, attr_["A"])
            return n
        return runner.render_and_score(ws, ds_, obs_, out_, fused=not args.unfused)

    last_out = {}

    def step():
        if shard:
            r = sharding.sharded_tokens(ws, ds, obs, 1.0)
            last_out["o"] = r[2]
            return r[3]
        last_out["o"] = out
        return run(ds, obs, out, grads, attr_out)

    for _ in range(max(args.warmup, 3) if args.warmup > 0 else 0):
        n_inst = step()
    if args.warmup <= 0:
        n_inst = step()
    torch.cuda.synchronize()
    pairs = ws.pair_count()
    # composited pairs: sum over this rank's pixels of the entries that contributed (n_contrib)
    composited = int(last_out["o"].n_contrib.sum(dtype=torch.int64).item())
    pairs_rank, composited_rank = pairs, composited  # this rank's, for its kernels' rooflines
    n_total = int(sum(n_inst))

    # ---- timed region: device time per step (CUDA events), L2 flushed between steps ----------
    # Two passes of K steps: the first, as the library runs without its per-kernel event pairs,
    # gives value and ms_per_step; the second, with the library's event pair around every kernel
    # group (two event records each, which widen the gaps between launches), gives the per-kernel
    # times and the rooflines.
    sampler = ClockSampler(gpu_id_for(dev)) if rank == 0 else None

    def timed_steps():
        ms = []
        for _ in range(args.steps):
            l2_flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return ms

    ws.profile(False)
    if sampler:
        sampler.start()  # returns once sampling is live
    barrier(world)
    if sampler:
        sampler.mark()
    launches_before = ws.launch_count
    step_ms = timed_steps()
    launches = ws.launch_count - launches_before
    ws.profile(True)
    ws.profile_read(reset=True)
    barrier(world)
    prof_step_ms = timed_steps()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    # device memory in use after the timed steps (the workspace grows only during warm-up, so
    # this is the steady-state peak): library workspace + torch tensors + CUDA context
    free_b, total_b = torch.cuda.mem_get_info(dev)
    vram = {"device_used_gb": (total_b - free_b) / 1e9,
            "torch_reserved_gb": torch.cuda.memory_reserved(dev) / 1e9,
            "device_total_gb": total_b / 1e9}
    kern = ws.profile_read(reset=True)
    # The fused score path runs the render and the replay as one kernel, so the render's own
    # time -- the denominator of the replay's cost -- is taken from separate render-only steps
    # (projection, binning, render; same L2 flush), outside the timed region.
    fused = (args.path == "score" and not args.unfused and not shard
             and kern.get("render_replay", (0.0, 0))[1] > 0)  # (deterministic mode: two kernels)
    render_alone_ms = None
    if fused:
        for _ in range(args.steps):
            l2_flush.zero_()
            runner.render(ws, ds, out)
        torch.cuda.synchronize()
        render_alone_ms = ws.profile_read(reset=True)["render"][0] / args.steps
        runner.render_and_score(ws, ds, obs, out)  # leave the workspace as the timed steps did
        torch.cuda.synchronize()
    ws.profile(False)

    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    # every rank takes part in these reductions, in the same order
    median_ms = max_over_ranks(statistics.median(step_ms), world)
    min_ms = max_over_ranks(min(step_ms), world)
    prof_ms_per_step = max_over_ranks(sum(prof_step_ms), world) / args.steps
    px_step = sc.V * sc.H * sc.W
    # replicas: every rank does the whole workload; views: the ranks split one workload
    units = 1 if shard else world
    value = px_step * args.steps * units / (total_ms * 1e-3) / 1e6
    pairs_per_s = pairs * args.steps * (world if not shard else 1) / (total_ms * 1e-3)
    if shard:  # pairs of all ranks' views
        pairs_per_s = pairs_sum_over_ranks(pairs, world) * args.steps / (total_ms * 1e-3)
        composited = pairs_sum_over_ranks(composited, world)

    # ---- end to end through the public API with host buffers ----------------------------------
    # Every step copies its inputs from pinned host memory and its outputs (tokens, image, final
    # transmittance, contributor counts) back, all inside the timed region. The steps are
    # pipelined with double-buffered device inputs/outputs: step k+1's host->device copy and step
    # k-1's device->host copy run on two copy streams while step k computes. The stream is at least
    # 32 steps long: the first step's inputs and the last step's outputs cross the link without
    # compute beside them, and over a handful of steps that fill and drain would dominate the
    # per-step figure of what is a steady stream.
    e2e = None
    n_e2e = max(args.steps, 32)
    if not args.no_e2e and not shard:
        names = ("means", "log_scales", "quats", "opac", "sh", "viewmats", "intrin", "bg")
        host = {k: torch.from_numpy(np.ascontiguousarray(getattr(sc, k))).pin_memory()
                for k in names}
        host["obs"] = obs.cpu().pin_memory()
        dsets = [ds, runner.DeviceScene(*[getattr(ds, k).clone() for k in names], ds.H, ds.W)]
        dobs = [obs, obs.clone()]
        outs = [out, runner.alloc_outputs(ds)]
        dgrads = [grads, alloc_grads()] if args.path == "backward" else [None, None]
        dattr = [attr_out, alloc_attr()] if args.path == "attributes" else [None, None]

        def d_outputs(b):
            o = {"img": outs[b].img, "T": outs[b].T, "n_contrib": outs[b].n_contrib}
            if args.path == "backward":
                o.update(dgrads[b])
            elif args.path == "attributes":
                o.update(dattr[b])
            else:
                o["tokens"] = outs[b].tokens
            return o

        def h_outputs():
            return {k: torch.empty(t.shape, dtype=t.dtype).pin_memory()
                    for k, t in d_outputs(0).items()}
        h_out = [h_outputs(), h_outputs()]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        in_ready, comp_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def enqueue_h2d(b):
            with torch.cuda.stream(s_in):
                for k in names:
                    getattr(dsets[b], k).copy_(host[k], non_blocking=True)
                dobs[b].copy_(host["obs"], non_blocking=True)
                in_ready[b].record(s_in)

        barrier(world)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)
        s_out.wait_event(t0)
        enqueue_h2d(0)
        for k in range(n_e2e):
            b = k & 1
            if k + 1 < n_e2e:
                if k >= 1:
                    s_in.wait_event(comp_done[1 - b])  # step k-1 has read that input set
                enqueue_h2d(1 - b)
            stream.wait_event(in_ready[b])
            if k >= 2:
                stream.wait_event(out_free[b])  # step k-2's outputs have been copied out
            run(dsets[b], dobs[b], outs[b], dgrads[b], dattr[b])
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                for name, t in d_outputs(b).items():
                    h_out[b][name].copy_(t, non_blocking=True)
                out_free[b].record(s_out)
        t1.record(s_out)
        t1.synchronize()
        barrier(world)
        e2e_total = max_over_ranks(t0.elapsed_time(t1), world)
        e2e = {"value": px_step * n_e2e * world / (e2e_total * 1e-3) / 1e6,
               "unit": "Mpix/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_total / n_e2e, "steps": n_e2e, "pipelined": True}
        del dsets, dobs, outs, h_out, dgrads, dattr

    # ---- roofline of the dominant kernel ------------------------------------------------------
    peaks = load_peaks()
    per_kernel0 = {k: v for k, v in kern.items() if v[1] > 0}
    dp = per_kernel0.get("depth_scatter", (0.0, 0))[1] // max(args.steps, 1)
    ab = algorithmic_bytes(sc, n_total, pairs, dp)
    per_kernel = {k: {"ms_per_step": v[0] / args.steps, "launches": v[1]}
                  for k, v in kern.items() if v[1] > 0}
    dom = max(per_kernel, key=lambda k: per_kernel[k]["ms_per_step"])
    dom_ms = per_kernel[dom]["ms_per_step"]
    lanes = torch.cuda.get_device_properties(dev).multi_processor_count * 128
    if dom in ALU_OPS:
        ops = alu_ops(dom, pairs_rank, composited_rank)
        achieved = ops / (dom_ms * 1e-3) / 1e12
        peak = lanes * peaks["sm_max_mhz"] * 1e6 / 1e12
        roof = {"bound": "alu", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "Tops/s (fp32 pipe)", "frac": achieved / peak,
                "traffic": recorded_traffic(dom, workload_name(args, sc)),
                "ncu_pipes": recorded_pipes(dom, workload_name(args, sc)),
                "work": f"{ALU_OPS[dom][0]} ops x traversed pairs + {ALU_OPS[dom][1]} ops x "
                        f"composited pairs",
                "peak_source": f"{lanes} fp32 lanes x {peaks['sm_max_mhz']:.0f} MHz "
                               f"({peaks['source']} max clock)"}
    else:
        achieved = ab.get(dom, 0) / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": recorded_traffic(dom, workload_name(args, sc)),
                "peak_source": f"{peaks['source']} copy bandwidth"}
    for k, v in per_kernel.items():
        if k in ab:
            v["algorithmic_GBps"] = ab[k] / (v["ms_per_step"] * 1e-3) / 1e9
        if k in ALU_OPS:
            v["alu_frac"] = (alu_ops(k, pairs_rank, composited_rank) / (v["ms_per_step"] * 1e-3)
                             / (lanes * peaks["sm_max_mhz"] * 1e6))
    render_ms = sum(per_kernel.get(k, {}).get("ms_per_step", 0.0) for k in
                    ("project", "depth_hist", "depth_scatter", "emit", "tile_hist",
                     "hist_scan", "tile_scatter", "tile_ranges", "render", "other"))
    second = {"backward": ("backward", "grad"), "attributes": ("features", "scatter"),
              "score": ("replay", "finalize")}[args.path]
    replay_ms = sum(per_kernel.get(k, {}).get("ms_per_step", 0.0) for k in second)
    if fused:
        # render side: the render kernel timed alone; replay side: what the fused kernel takes
        # beyond it, plus the finalisation
        per_kernel["render_replay"]["render_alone_ms"] = render_alone_ms
        render_ms += render_alone_ms
        replay_ms += per_kernel["render_replay"]["ms_per_step"] - render_alone_ms

    # The oracle's view is also compared with the CUDA path over the same view, element by
    # element (score path, whole view: every pixel and every Gaussian's token).
    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        want = args.path == "score" and not shard
        cpu = cpu_oracle_view(sc, obs.cpu().numpy(), path=args.path, threads=args.cpu_threads,
                              keep_outputs=want)
        cpu.pop("seconds", None)
        ora = cpu.pop("outputs", None)
        if ora is not None:
            try:
                parity = {"view": f"1 of {sc.V}, whole",
                          **parity_report(gpu_view_outputs(sc, obs, not args.unfused,
                                                           args.deterministic), ora, sc.d)}
            except Exception as e:  # a report: its failure must not cost the line
                parity = {"error": f"{type(e).__name__}: {e}"[:300]}
        del ora

    if rank == 0:
        line = {
            "metric": METRICS[args.path], "value": value, "unit": "Mpix/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload_name(args, sc), "gaussians": sc.G, "views": sc.V,
                       "height": sc.H, "width": sc.W, "sh_degree": sc.sh_degree,
                       "path": PATHS[args.path],
                       "accumulation": "fixed-point (deterministic)" if args.deterministic
                       else "fp32 vector reductions",
                       "calls": ("splat_render_score (render and replay in one kernel)" if fused
                                 else "separate calls"),
                       "instances_per_step": n_total, "pairs_per_step": pairs,
                       "composited_pairs_per_step": composited,
                       "l2": "256 MiB buffer written between timed steps",
                       "parallelism": (f"views x{world} (reduce-scatter of per-Gaussian partials)"
                                       if shard else f"replicas x{world}")},
            "pairs_per_s": pairs_per_s,
            "ms_view": ms_per_step / sc.V,
            "render_ms_per_step": render_ms, f"{second[0]}_ms_per_step": replay_ms,
            "render_ms_per_view": render_ms / sc.V, f"{second[0]}_ms_per_view": replay_ms / sc.V,
            f"{second[0]}_over_render": replay_ms / render_ms if render_ms else None,
            "gpu_launches": int(launches), "per_kernel": per_kernel,
            "ms_per_step_with_kernel_events": prof_ms_per_step,
            "ms_per_step_median": median_ms, "ms_per_step_min": min_ms,
            "roofline": roof, "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu, "vram": vram,
            "parity_vs_oracle": parity,
        }
        os.write(json_fd, (json.dumps(line) + "\n").encode())
    ws.close()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
