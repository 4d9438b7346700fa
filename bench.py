#!/usr/bin/env python
"""Throughput of the fused low-bit dequant + matmul on B200.

Workload of the headline number: one Llama-3-8B-shaped decode step at batch 1,
the 7 projections (q, k, v, o, gate, up, down) of 32 layers, 224 distinct
asymmetric INT4 weights (group 32, fp16 scale + int8 zero point), fp16
activations. A step is the 224 GEMVs, replayed as one CUDA graph. The metric
is weight-GB/s: bytes of the format (nibbles + scales + zero points) streamed
per second, against the measured HBM copy bandwidth. The step's weights
(4.14 GB) are far larger than L2, so no flush is needed between steps.

Secondary numbers (same JSON line, key "secondary"): the single 4096x4096
GEMV, the K=8192 N=28672 batch sweep, the prefill GEMM, the LUT3 path, LUT3 x
MXFP8 with its activation quantiser, and the 1..8-bit affine GEMV.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lbq|reference]
Multi-GPU: one process per GPU under torchrun; each rank runs its own decode
step (replicas, weak scaling, no collective on the data path); the timing is
the max over ranks.
"""

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

METRIC = "decode GEMV weight-GB/s & % HBM peak; prefill GEMM TFLOP/s & % tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(FALLBACK_PEAKS)


def int4_bytes(K, N, group, mode):
    return K * N // 2 + (K // group) * N * (3 if mode == "asym" else 2)


def affine_bytes(K, N, group, bits):
    """Algorithmic bytes of a b-bit affine weight: K N b / 8 code bytes plus an
    FP16 scale and an int8 zero point per group of a column."""
    return K * N * bits // 8 + (K // group) * N * 3


def lut3_bytes(K, N):
    return K * N * 3 // 8 + (K // 64) * (N // 8) * 9


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "power_w_max": max(power),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed

def dist_setup(backend=None):
    """Rank / world from the torchrun environment; for world > 1 a process group
    with a short timeout (NCCL on GPUs; gloo when no GPU is visible, which is how
    the host logic is tested)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, value):
    """The largest of the ranks' values (every rank gets it)."""
    import torch
    if world == 1:
        return value
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v for v in vis.split(",") if v.strip()]
        if local < len(ids) and ids[local].strip().isdigit():
            return int(ids[local])
    return local


# ----------------------------------------------------------------------------- the decode step

class DecodeStep:
    """224 asym INT4 g32 GEMVs (32 layers x 7 projections), images resident in HBM.

    As in a decoder layer, q, k and v read one activation vector and gate and
    up another; with grouped=True each of those sets is one lbq_gemv_grouped
    launch (4 launches per layer), otherwise every projection is its own
    lbq_gemv call (7 per layer)."""

    # projection groups sharing X: (q, k, v), (o), (gate, up), (down)
    GROUPS = ((0, 1, 2), (3,), (4, 5), (6,))

    def __init__(self, torch, lbq, workloads, device, layers, grouped=True, w4a8=False):
        self.torch = torch
        self.lbq = lbq
        self.grouped = grouped
        self.w4a8 = w4a8  # W4A8: each shared X is quantised to INT8 once, then its GEMVs run on the codes
        self.bytes = 0
        self.calls = []  # per launch: list of (K, N, img, x, y, ws)
        proj = workloads.LLAMA3_8B_PROJ
        x_len = layers * sum(proj[g[0]][1] for g in self.GROUPS)
        y_len = layers * sum(N for (_, _, N) in proj)
        self.x_all = torch.empty(x_len, dtype=torch.float16, device=device)
        self.y_all = torch.empty(y_len, dtype=torch.float16, device=device)
        self.n_gemvs = layers * len(proj)
        xo = yo = 0
        # one workspace per (K, N): a workspace is reused only by calls of one
        # shape, whose tile counters sit at the same place every time
        self.ws = {}
        self.layers = []  # per layer: (first call, end call, X range, Y range) in calls / x_all / y_all
        for layer in range(layers):
            c0, x0, y0 = len(self.calls), xo, yo
            for grp in self.GROUPS:
                K = proj[grp[0]][1]
                x = self.x_all[xo:xo + K].view(1, K)
                x.copy_(workloads.activations_device(workloads.c2_seed(layer, grp[0]), 1, K, "f16", device))
                xo += K
                members = []
                for p in grp:
                    _, Kp, N = proj[p]
                    W = workloads.weights_device(workloads.c2_seed(layer, p), Kp, N, device)
                    img = lbq.pack(W, 32, "asym")
                    del W
                    y = self.y_all[yo:yo + N].view(1, N)
                    yo += N
                    if (Kp, N) not in self.ws:
                        self.ws[(Kp, N)] = torch.zeros(max(lbq.lbq_workspace_size(0, 1, Kp, N, 32, 1), 256),
                                                       dtype=torch.uint8, device=device)
                    members.append((Kp, N, img, x, y, self.ws[(Kp, N)]))
                    self.bytes += int4_bytes(Kp, N, 32, "asym")
                if w4a8:
                    xq = torch.empty((1, K), dtype=torch.int8, device=device)
                    sx = torch.empty((1, K // 32), dtype=torch.float32, device=device)
                    items = lbq.make_w4a8_items([(xq.data_ptr(), sx.data_ptr(), img.data_ptr(), y.data_ptr(), N)
                                                 for (_, N, img, x, y, _) in members])
                    self.calls.append(("w4a8", K, x, xq, sx, items, len(members), members))
                elif grouped and len(members) > 1:
                    items = lbq.make_gemv_items([(x.data_ptr(), img.data_ptr(), y.data_ptr(), N)
                                                 for (_, N, img, x, y, _) in members])
                    self.calls.append(("grouped", K, items, len(members), members))
                else:
                    for m in members:
                        self.calls.append(("single",) + m)
            self.layers.append((c0, len(self.calls), (x0, xo), (y0, yo)))
        torch.cuda.synchronize()

    def launch_all(self, calls=None):
        lbq = self.lbq
        stream = self.torch.cuda.current_stream().cuda_stream
        for c in (self.calls if calls is None else calls):
            if c[0] == "w4a8":
                _, K, x, xq, sx, items, n, _members = c
                lbq.lbq_quantize_int8(x.data_ptr(), 0, 1, K, xq.data_ptr(), sx.data_ptr(), stream)
                lbq.lbq_w4a8_gemv_grouped(items, n, K, 32, 1, 0, stream)
            elif c[0] == "grouped":
                _, K, items, n, _members = c
                lbq.lbq_gemv_grouped(items, n, K, 32, 1, 0, 0, stream)
            else:
                _, K, N, img, x, y, ws = c
                lbq.lbq_gemv(x.data_ptr(), 0, 1, K, N, 32, 1, img.data_ptr(), y.data_ptr(), 0,
                             ws.data_ptr(), ws.numel(), stream)

    def capture(self):
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.launch_all()  # warm the planner caches outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        before = self.lbq.lbq_launch_count()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch_all()
        self.launches_per_step = self.lbq.lbq_launch_count() - before
        torch.cuda.synchronize()
        return g


class E2EStep:
    """One decode step through the public C-ABI calls (no graph) with its
    inputs copied in from pinned host memory and its outputs copied back. The
    layers go in `chunks` groups, with one copy stream bringing X in and one
    taking Y out: a group's X for the next step is copied in as soon as this
    step's GEMVs of that group have read it, and a group's Y goes out as soon as
    its GEMVs are done, so the copies overlap the other groups' GEMVs (the
    step's X vectors are inputs of the step, as in the bench's graph). Every
    step's copies lie inside the timed region: the first step's inputs wait
    for the compute stream (reset()), and finish() makes the compute stream
    wait for the last outputs."""

    def __init__(self, torch, step, chunks=2):
        self.torch, self.step = torch, step
        n = len(step.layers)
        per = -(-n // chunks)
        self.groups = [step.layers[i:i + per] for i in range(0, n, per)]
        self.x_host = torch.empty_like(step.x_all, device="cpu").pin_memory()
        self.x_host.copy_(step.x_all.cpu())
        self.y_host = torch.empty_like(step.y_all, device="cpu").pin_memory()
        self.cs_in, self.cs_out = torch.cuda.Stream(), torch.cuda.Stream()
        self.ev_in = [torch.cuda.Event() for _ in self.groups]    # X of the group copied in
        self.ev_used = [torch.cuda.Event() for _ in self.groups]  # the group's GEMVs done
        self.ev_out = [torch.cuda.Event() for _ in self.groups]   # Y of the group copied out
        self.done = torch.cuda.Event()
        self.started = False

    def reset(self):
        """The next step's input copies wait for the compute stream's work so far."""
        self.started = False

    def run(self):
        torch, step = self.torch, self.step
        main = torch.cuda.current_stream()
        for i, g in enumerate(self.groups):
            (x0, _), (x1, _) = g[0][2], g[-1][2]
            with torch.cuda.stream(self.cs_in):
                if self.started:
                    self.cs_in.wait_event(self.ev_used[i])  # the previous step has read this X
                else:
                    self.cs_in.wait_stream(main)
                step.x_all[x0:x1].copy_(self.x_host[x0:x1], non_blocking=True)
                self.ev_in[i].record(self.cs_in)
        for i, g in enumerate(self.groups):
            main.wait_event(self.ev_in[i])
            if self.started:
                main.wait_event(self.ev_out[i])  # the previous step's Y of this group is out
            step.launch_all(step.calls[g[0][0]:g[-1][1]])
            self.ev_used[i].record(main)
            (y0, _), (y1, _) = g[0][3], g[-1][3]
            with torch.cuda.stream(self.cs_out):
                self.cs_out.wait_event(self.ev_used[i])
                self.y_host[y0:y1].copy_(step.y_all[y0:y1], non_blocking=True)
                self.ev_out[i].record(self.cs_out)
        self.done.record(self.cs_out)
        self.started = True

    def finish(self):
        """The compute stream waits for the last step's output copies."""
        self.torch.cuda.current_stream().wait_event(self.done)


def time_graph(torch, graph, steps, warmup, world):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)


def rotating_ms(torch, call, images, reps=5):
    """Per-launch time of call(image, stream) cycling through distinct weight
    copies (their total exceeds L2) inside one CUDA graph, CUDA events around
    `reps` replays on the capturing stream's successor (the current stream)."""
    def run():
        s = torch.cuda.current_stream().cuda_stream
        for img in images:
            call(img, s)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / (reps * len(images))


def rotating_gemv_ms(torch, lbq, images, X, N, group, mode, ws, reps=5):
    """INT4 lbq_gemm over rotating weight copies (M <= 16 takes the GEMV kernels)."""
    Y = torch.empty((X.shape[0], N), dtype=X.dtype, device=X.device)
    xdt = 0 if X.dtype == torch.float16 else 1
    m = {"sym": 0, "asym": 1}[mode]

    def call(img, s):
        lbq.lbq_gemm(X.data_ptr(), xdt, X.shape[0], X.shape[1], N, group, m, img.data_ptr(), Y.data_ptr(), xdt,
                     ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, s)

    return rotating_ms(torch, call, images, reps)


def rotating_lut3_ms(torch, lbq, images, X, N, ws, reps=5):
    Y = torch.empty((X.shape[0], N), dtype=X.dtype, device=X.device)

    def call(img, s):
        lbq.lbq_lut3_gemm(X.data_ptr(), 1, X.shape[0], X.shape[1], N, img.data_ptr(), Y.data_ptr(), 1,
                          ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, s)

    return rotating_ms(torch, call, images, reps)


# the MoE layer of the LUT-B write-up's latency table: 256 experts, top-8,
# hidden 2048, expert intermediate 512 (gate and up side by side: N = 1024)
MOE_LAYER = {"experts": 256, "top_k": 8, "hidden": 2048, "inter": 512}


def moe_expert_images(torch, lbq, workloads, device, seed, K, N, E):
    """E LUT3 expert images (seeded synthetic indices, codebooks, exponents) at one stride."""
    experts = [workloads.lut3_device(seed + e, K, N, device) for e in range(E)]
    images, stride = lbq.pack_lut3_experts(experts)
    del experts
    return images, stride


def moe_inputs(torch, lbq, workloads, device, T, top_k, E, K):
    """Seeded uniform routing (top_k distinct experts per token), its alignment
    on the device, and MXFP8 activations [T, K] drawn in the format."""
    import numpy as np
    rng = np.random.default_rng(7 + T)
    ids = torch.from_numpy(np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.int32))
    ids = ids.to(device)
    aligned = lbq.moe_align(ids, E)
    codes, scales = workloads.mx_activations_host(8 + T, T, K)
    return aligned, torch.from_numpy(codes).to(device), torch.from_numpy(scales).to(device), ids


def weight_copies(img0, l2_bytes, minimum=3):
    """img0 plus clones so that the copies together exceed 3x L2."""
    copies = max(minimum, (3 * l2_bytes) // img0.numel() + 1)
    return [img0] + [img0.clone() for _ in range(copies - 1)]


# the GEMV kernels the library does not pick by default, timed beside the default
GEMV_ALT_PATHS = (("tma_cudacore_m1_kernel", 1), ("direct_m1_kernel", 4), ("warp_mma_kernel", 2),
                  ("tcgen05_kernel", 3))


def secondary_measurements(torch, lbq, workloads, device, peaks, quick):
    # GEMVs are launched as in the step, with programmatic dependent launch
    # (the GEMMs never use it); weights rotate through copies larger than L2
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 1)
    try:
        return _secondary_measurements(torch, lbq, workloads, device, peaks, quick)
    finally:
        lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)


def _secondary_measurements(torch, lbq, workloads, device, peaks, quick):
    out = {}
    hbm = peaks["hbm_gbs"]
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    # c1: single 4096x4096 sym g32 GEMV, fp16
    K, N = 4096, 4096
    W = workloads.weights_device(0, K, N, device)
    img0 = lbq.pack(W, 32, "sym")
    del W
    copies = max(3, (3 * l2_bytes) // img0.numel() + 1)
    images = [img0] + [img0.clone() for _ in range(copies - 1)]
    X = workloads.activations_device(0, 1, K, "f16", device)
    ms = rotating_gemv_ms(torch, lbq, images, X, N, 32, "sym", lbq.workspace(0, 1, K, N, 32, "sym"))
    b = int4_bytes(K, N, 32, "sym")
    out["c1_gemv_4096x4096_sym_g32_m1"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm,
                                           "weight_copies": copies}
    for name, path in GEMV_ALT_PATHS:
        lbq.lbq_debug_gemv_path(path)
        ms = rotating_gemv_ms(torch, lbq, images, X, N, 32, "sym", lbq.workspace(0, 1, K, N, 32, "sym"))
        lbq.lbq_debug_gemv_path(0)
        out[f"c1_gemv_m1_{name}"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm}
    del images, img0
    if quick:
        return out
    # c3: K=8192 N=28672 sym g64/g128 with outliers, bf16, M in {1,2,4,8,16}
    K, N = 8192, 28672
    W = workloads.weights_device(3, K, N, device, outlier_frac=1e-3, outlier_mult=20.0)
    for group in (64, 128):
        img0 = lbq.pack(W, group, "sym")
        copies = max(2, (3 * l2_bytes) // img0.numel() + 1)
        images = [img0] + [img0.clone() for _ in range(copies - 1)]
        b = int4_bytes(K, N, group, "sym")
        for M in (1, 2, 4, 8, 16):
            X = workloads.activations_device(3, M, K, "bf16", device)
            ws = lbq.workspace(0, M, K, N, group, "sym")
            ms = rotating_gemv_ms(torch, lbq, images, X, N, group, "sym", ws, reps=3)
            out[f"c3_g{group}_m{M}"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm}
            if M in (1, 16):
                for name, path in GEMV_ALT_PATHS:
                    if path in (1, 2, 4) and M != 1:
                        continue
                    lbq.lbq_debug_gemv_path(path)
                    ws = lbq.workspace(0, M, K, N, group, "sym")
                    ms = rotating_gemv_ms(torch, lbq, images, X, N, group, "sym", ws, reps=3)
                    lbq.lbq_debug_gemv_path(0)
                    out[f"c3_g{group}_m{M}_{name}"] = {"us": ms * 1e3, "GBps": b / ms / 1e6,
                                                       "frac_hbm": b / ms / 1e6 / hbm}
        del images, img0
    del W
    # c4: prefill GEMM K=4096 N=14336 asym g128, bf16 X and Y, tcgen05
    tc_peak, tc_sus = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    K, N = 4096, 14336
    W = workloads.weights_device(4, K, N, device)
    images = weight_copies(lbq.pack(W, 128, "asym"), l2_bytes)
    del W
    for M in (512, 2048, 8192):
        X = workloads.activations_device(4, M, K, "bf16", device)
        ws = lbq.workspace(1, M, K, N, 128, "asym")
        ms = rotating_gemv_ms(torch, lbq, images, X, N, 128, "asym", ws, reps=3)
        tf = 2.0 * M * K * N / ms / 1e9
        out[f"c4_gemm_m{M}"] = {"us": ms * 1e3, "TFLOPs": tf, "frac_bf16_peak": tf / tc_peak,
                                "frac_bf16_sustained": tf / tc_sus, "weight_copies": len(images),
                                "stream_k": ws is not None}
        if ws is not None:  # the same launches with whole tiles only, for comparison
            lbq.lbq_debug_gemm_stream_k(0)
            try:
                ms_w = rotating_gemv_ms(torch, lbq, images, X, N, 128, "asym", ws, reps=3)
            finally:
                lbq.lbq_debug_gemm_stream_k(1)
            out[f"c4_gemm_m{M}"]["TFLOPs_whole_tiles"] = 2.0 * M * K * N / ms_w / 1e9
        del X
    del images
    # c5: LUT3 K=4096 N=14336, M=1 (GB/s of the format's bytes) and M=2048 (TFLOP/s)
    idx, cb, ex = workloads.lut3_device(5, K, N, device)
    images = weight_copies(lbq.pack_lut3(idx, cb, ex), l2_bytes)
    del idx, cb, ex
    b = lut3_bytes(K, N)
    for M in (1, 2048):
        X = workloads.activations_device(5, M, K, "bf16", device)
        ws = lbq.workspace(2, M, K, N, 0, "lut3")
        ms = rotating_lut3_ms(torch, lbq, images, X, N, ws, reps=3)
        if M == 1:
            out["c5_lut3_m1"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm,
                                 "image_bytes_read": images[0].numel(), "weight_copies": len(images),
                                 "kernel": "lut3_tmma_kernel"}
            # the register-pipelined direct kernel (the default for 8192 < K <= 16384), timed beside it
            lbq.lbq_debug_gemv_path(4)
            try:
                ms_d = rotating_lut3_ms(torch, lbq, images, X, N, ws, reps=3)
            finally:
                lbq.lbq_debug_gemv_path(0)
            out["c5_lut3_m1_direct_kernel"] = {"us": ms_d * 1e3, "GBps": b / ms_d / 1e6,
                                               "frac_hbm": b / ms_d / 1e6 / hbm}
            # batch 4 on the TMA-fed batch kernel, and on the skinny kernel beside it
            X4 = workloads.activations_device(5, 4, K, "bf16", device)
            ws4 = lbq.workspace(2, 4, K, N, 0, "lut3")
            ms4 = rotating_lut3_ms(torch, lbq, images, X4, N, ws4, reps=3)
            out["c5_lut3_m4"] = {"us": ms4 * 1e3, "GBps": b / ms4 / 1e6, "frac_hbm": b / ms4 / 1e6 / hbm,
                                 "kernel": "lut3_tmma_batch_kernel"}
            lbq.lbq_debug_lut3_batch_off(1)
            try:
                ms4s = rotating_lut3_ms(torch, lbq, images, X4, N, ws4, reps=3)
            finally:
                lbq.lbq_debug_lut3_batch_off(0)
            out["c5_lut3_m4_skinny_kernel"] = {"us": ms4s * 1e3, "GBps": b / ms4s / 1e6,
                                               "frac_hbm": b / ms4s / 1e6 / hbm}
            del X4, ws4
            # batch 16: two blocks of 8 rows on the batch kernel's columns
            X16 = workloads.activations_device(5, 16, K, "bf16", device)
            ws16 = lbq.workspace(2, 16, K, N, 0, "lut3")
            ms16 = rotating_lut3_ms(torch, lbq, images, X16, N, ws16, reps=3)
            out["c5_lut3_m16"] = {"us": ms16 * 1e3, "GBps": b / ms16 / 1e6, "frac_hbm": b / ms16 / 1e6 / hbm,
                                  "kernel": "lut3_tmma_batch_kernel"}
            lbq.lbq_debug_lut3_batch_off(1)
            try:
                ms16s = rotating_lut3_ms(torch, lbq, images, X16, N, ws16, reps=3)
            finally:
                lbq.lbq_debug_lut3_batch_off(0)
            out["c5_lut3_m16_skinny_kernel"] = {"us": ms16s * 1e3, "GBps": b / ms16s / 1e6,
                                                "frac_hbm": b / ms16s / 1e6 / hbm}
            del X16, ws16
        else:
            tf = 2.0 * M * K * N / ms / 1e9
            out[f"c5_lut3_m{M}"] = {"us": ms * 1e3, "TFLOPs": tf, "frac_bf16_peak": tf / tc_peak,
                                    "frac_bf16_sustained": tf / tc_sus, "stream_k": ws is not None}
            if ws is not None:  # whole tiles only, for comparison
                lbq.lbq_debug_gemm_stream_k(0)
                try:
                    ms_w = rotating_lut3_ms(torch, lbq, images, X, N, ws, reps=3)
                finally:
                    lbq.lbq_debug_gemm_stream_k(1)
                out[f"c5_lut3_m{M}"]["TFLOPs_whole_tiles"] = 2.0 * M * K * N / ms_w / 1e9
        del X
    del images
    # LUT3 x MXFP8 on the block-scaled FP8 tensor path, M=2048 (activations
    # already in MXFP8: codes + scales), against an FP8 peak of 2x the BF16 one
    # (the FP8 dense rate is twice the BF16 rate on this GPU; only BF16 is measured)
    idx, cb, ex = workloads.lut3_device(5, K, N, device)
    images = weight_copies(lbq.pack_lut3(idx, cb, ex), l2_bytes)
    del idx, cb, ex
    for M in (2048, 8192):
        codes_h, scales_h = workloads.mx_activations_host(60 + M, M, K)
        codes, scales = torch.from_numpy(codes_h).to(device), torch.from_numpy(scales_h).to(device)
        Ymx = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        wsmx = lbq.workspace(2, M, K, N, 0, "lut3")

        def mxcall(img, s):
            lbq.lbq_lut3_mx_gemm(codes.data_ptr(), scales.data_ptr(), M, K, N, img.data_ptr(), Ymx.data_ptr(), 1,
                                 wsmx.data_ptr() if wsmx is not None else None,
                                 wsmx.numel() if wsmx is not None else 0, s)

        ms = rotating_ms(torch, mxcall, images, reps=3)
        tf = 2.0 * M * K * N / ms / 1e9
        out[f"c5_lut3_mxfp8_m{M}"] = {"us": ms * 1e3, "TFLOPs": tf, "frac_fp8_peak": tf / (2 * tc_peak),
                                      "fp8_peak_tflops": 2 * tc_peak,
                                      "fp8_peak_source": "2 x the BF16 figure (%s)" % peaks["source"],
                                      "frac_bf16_peak": tf / tc_peak}
        del codes, scales, Ymx
    del images
    # MXFP8 activation quantiser (the activation side of the LUT3 x MXFP8
    # product): M=2048 K=4096 BF16, 2 bytes read and 1 + 1/32 written per value
    M, K = 2048, 4096
    xs = [workloads.activations_device(50 + i, M, K, "bf16", device)
          for i in range(max(3, 3 * l2_bytes // (M * K * 2) + 1))]
    codes = torch.empty((M, K), dtype=torch.uint8, device=device)
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device=device)

    def qcall(X, s):
        lbq.lbq_quantize_mxfp8(X.data_ptr(), 1, M, K, codes.data_ptr(), scales.data_ptr(), s)

    ms = rotating_ms(torch, qcall, xs, reps=3)
    b = M * K * 2 + M * K + M * K // 32
    out["mxfp8_quantize_m2048_k4096"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm,
                                         "bytes_per_launch": b, "input_copies": len(xs)}
    del xs
    # the decode step in W4A8 form: 32 layers, per shared activation vector one
    # INT8 quantisation and one grouped W4A8 launch (8 launches per layer), one
    # CUDA graph with programmatic dependent launch; GB/s of the INT4 weight bytes
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 1)
    wstep = DecodeStep(torch, lbq, workloads, device, 32, w4a8=True)
    g = wstep.capture()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(10):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 10
    out["c2_step_w4a8_32layers"] = {"us": ms * 1e3, "GBps": wstep.bytes / ms / 1e6,
                                     "frac_hbm": wstep.bytes / ms / 1e6 / hbm,
                                     "launches_per_step": wstep.launches_per_step,
                                     "weight_bytes_per_step": wstep.bytes,
                                     "activations": "INT8, one FP32 scale per 32 k (lbq_quantize_int8), once per "
                                                    "shared X"}
    del g, wstep
    # grouped MoE GEMM of LUT3 experts x MXFP8 activations at the write-up's
    # layer shape (E=256, top-8, H=2048, I=512): the gate/up GEMM (K=2048,
    # N=1024) and the down GEMM (K=512, N=2048, one row per pair), with the
    # device alignment, at 1, 16, 256 and 4096 tokens
    E, top_k, H, I = MOE_LAYER["experts"], MOE_LAYER["top_k"], MOE_LAYER["hidden"], MOE_LAYER["inter"]
    img1, st1 = moe_expert_images(torch, lbq, workloads, device, 1000, H, 2 * I, E)
    img2, st2 = moe_expert_images(torch, lbq, workloads, device, 5000, I, H, E)
    for T in (1, 16, 256, 4096):
        aligned, c1, s1, ids_dev = moe_inputs(torch, lbq, workloads, device, T, top_k, E, H)
        al2 = lbq.moe_align(ids_dev.view(-1, 1), E)  # the down GEMM: one row per pair
        c2h, s2h = workloads.mx_activations_host(9 + T, T * top_k, I)
        c2, s2 = torch.from_numpy(c2h).to(device), torch.from_numpy(s2h).to(device)
        Y1 = torch.empty((T * top_k, 2 * I), dtype=torch.bfloat16, device=device)
        Y2 = torch.empty((T * top_k, H), dtype=torch.bfloat16, device=device)

        def layer(_img, s):
            lbq.lbq_moe_align(ids_dev.data_ptr(), T * top_k, E, 128, None, aligned[0].data_ptr(),
                              aligned[1].data_ptr(), aligned[2].data_ptr(), aligned[0].numel(), s)
            lbq.lbq_moe_lut3_mx_gemm(c1.data_ptr(), s1.data_ptr(), T, top_k, H, 2 * I, aligned[0].data_ptr(),
                                     aligned[1].data_ptr(), aligned[2].data_ptr(), aligned[0].numel(),
                                     img1.data_ptr(), st1, E, Y1.data_ptr(), 1, s)
            lbq.lbq_moe_lut3_mx_gemm(c2.data_ptr(), s2.data_ptr(), T * top_k, 1, I, H, al2[0].data_ptr(),
                                     al2[1].data_ptr(), al2[2].data_ptr(), al2[0].numel(),
                                     img2.data_ptr(), st2, E, Y2.data_ptr(), 1, s)

        ms = rotating_ms(torch, layer, [None], reps=10)
        fl = 2.0 * T * top_k * (H * 2 * I + I * H)
        out[f"moe_lut3_mx_layer_t{T}"] = {"us": ms * 1e3, "TFLOPs": fl / ms / 1e9,
                                          "what": "align + gate/up GEMM + down GEMM (E=256, top-8, H=2048, I=512)"}
        del c1, s1, c2, s2, Y1, Y2, aligned, al2
    del img1, img2
    # generic b-bit affine GEMV, b = 1..8, at the gate/up shape K=4096 N=14336
    # g64, batch 1 (and batch 4 for 3 bits), FP16 X: GB/s of the format's bytes
    K, N, group = 4096, 14336, 64
    W = workloads.weights_device(8, K, N, device)
    for bits in range(1, 9):
        images = weight_copies(lbq.pack_affine(W, group, bits), l2_bytes)
        b = affine_bytes(K, N, group, bits)
        for M in ((1, 4) if bits == 3 else (1,)):
            X = workloads.activations_device(8, M, K, "f16", device)
            Ya = torch.empty((M, N), dtype=torch.float16, device=device)

            def acall(img, s):
                lbq.lbq_affine_gemv(X.data_ptr(), 0, M, K, N, group, bits, img.data_ptr(), Ya.data_ptr(), 0, s)

            ms = rotating_ms(torch, acall, images, reps=3)
            out[f"affine_b{bits}_g64_m{M}"] = {"us": ms * 1e3, "GBps": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm,
                                              "bytes_per_launch": b, "weight_copies": len(images)}
        del images
    del W
    return out


# ----------------------------------------------------------------------------- CPU baseline (oracle)

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def oracle_sample(seconds_target, layer=0, max_proj=7):
    """Time the oracle (dequant + FP64 matmul) on the first projections of one
    layer of the decode step, host-generated and quantised outside the timer."""
    import workloads
    from oracle import int4, matmul
    cores = _blas_threads()
    done_bytes, spent, names = 0, 0.0, []
    for p, (name, K, N) in enumerate(workloads.LLAMA3_8B_PROJ[:max_proj]):
        seed = workloads.c2_seed(layer, p)
        W = workloads.weights_host(seed, K, N)
        q, s, z = int4.quantize_asym(W, 32)
        X = workloads.activations_host(seed, 1, K, "f16")
        t0 = time.perf_counter()
        deq = int4.dequant(q, s, 32, z)
        matmul.matmul_f64(X, deq)
        spent += time.perf_counter() - t0
        done_bytes += int4_bytes(K, N, 32, "asym")
        names.append(name)
        if spent >= seconds_target:
            break
    return {"value": done_bytes / spent / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"layer {layer} projections {'+'.join(names)} of the decode step: exact dequant + FP64 "
                      f"matmul (numpy), {done_bytes} weight bytes in {spent:.2f} s"}


def oracle_per_config(column_budget=1024):
    """The oracle on a bounded sample of every other configuration: a K x
    min(N, column_budget) weight of the configuration's distribution and seed,
    dequant + FP64 matmul timed, reported as that configuration's metric
    (weight-GB/s of the sampled columns; GFLOP/s as well for the GEMMs)."""
    import workloads
    from oracle import int4, lut3, matmul
    out = {}

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def int4_case(name, seed, K, N, group, mode, Ms, xdt, **kw):
        n = min(N, column_budget)
        W = workloads.weights_host(seed, K, n, **kw)
        q, s, z = int4.quantize(W, group, mode)
        for M in Ms:
            X = workloads.activations_host(seed, M, K, xdt)
            dt = timed(lambda: matmul.matmul_f64(X, int4.dequant(q, s, group, z)))
            rec = {"columns": n, "seconds": dt, "GBps": int4_bytes(K, n, group, mode) / dt / 1e9}
            if M > 16:
                rec["GFLOPs"] = 2.0 * M * K * n / dt / 1e9
            out[f"{name}_m{M}"] = rec

    int4_case("c1_4096x4096_sym_g32", 0, 4096, 4096, 32, "sym", (1,), "f16")
    int4_case("c3_8192x28672_sym_g64", 3, 8192, 28672, 64, "sym", (1, 16), "bf16", outlier_frac=1e-3,
              outlier_mult=20.0)
    int4_case("c3_8192x28672_sym_g128", 3, 8192, 28672, 128, "sym", (1, 16), "bf16", outlier_frac=1e-3,
              outlier_mult=20.0)
    int4_case("c4_4096x14336_asym_g128", 4, 4096, 14336, 128, "asym", (512, 2048), "bf16")
    K, n = 4096, min(14336, column_budget)
    idx, cb, ex = workloads.lut3_host(5, K, n)
    for M in (1, 2048):
        X = workloads.activations_host(5, M, K, "bf16")
        dt = timed(lambda: matmul.matmul_f64(X, lut3.dequant(idx, cb, ex)))
        rec = {"columns": n, "seconds": dt, "GBps": lut3_bytes(K, n) / dt / 1e9}
        if M > 16:
            rec["GFLOPs"] = 2.0 * M * K * n / dt / 1e9
        out[f"c5_4096x14336_lut3_m{M}"] = rec
    return out


def oracle_one_core(seconds_target=4.0):
    """oracle_sample with the BLAS pool limited to one thread."""
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    with threadpool_limits(limits=1):
        r = oracle_sample(seconds_target, max_proj=7)
    r["cores"] = 1
    return r


def run_reference(args):
    """The reference arm: the oracle as it stands, on the host cores, same metric."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return 0
    import numpy as np
    import workloads
    from oracle import int4, matmul
    projs = list(enumerate(workloads.LLAMA3_8B_PROJ))
    prepared = []
    for p, (name, K, N) in projs:
        seed = workloads.c2_seed(0, p)
        W = workloads.weights_host(seed, K, N)
        q, s, z = int4.quantize_asym(W, 32)
        prepared.append((K, N, q, s, z, workloads.activations_host(seed, 1, K, "f16")))
    total_bytes, total_s = 0, 0.0
    for i in range(args.warmup + args.steps):
        K, N, q, s, z, X = prepared[i % len(prepared)]
        t0 = time.perf_counter()
        matmul.matmul_f64(X, int4.dequant(q, s, 32, z))
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            total_bytes += int4_bytes(K, N, 32, "asym")
            total_s += dt
    value = total_bytes / total_s / 1e9
    cores = _blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "Llama-3-8B-shaped decode step (layer 0 projections, one per step), asym INT4 "
                                   "g32, fp16 X, M=1", "l2": "n/a (host)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": "one projection of layer 0 per step, cycling q,k,v,o,gate,up,down: exact "
                                       "dequant + FP64 numpy matmul"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ncu cases

# name -> (K, N, group, mode, x dtype, M, GEMV path or None); the path is the
# test hook's kernel choice (1 TMA CUDA-core, 2 warp MMA, 3 tcgen05, 4 direct,
# 5 TMA-fed warp MMA). A tuple N is one grouped launch of GEMVs sharing X, as
# the decode step runs q/k/v and gate/up.
PROFILE_CASES = {
    "c1": (4096, 4096, 32, "sym", "f16", 1, None),
    "c2qkv": (4096, (4096, 1024, 1024), 32, "asym", "f16", 1, None),
    "c2o": (4096, 4096, 32, "asym", "f16", 1, None),
    "c2gateup": (4096, (14336, 14336), 32, "asym", "f16", 1, None),
    "c2gate": (4096, 14336, 32, "asym", "f16", 1, None),
    "c2down": (14336, 4096, 32, "asym", "f16", 1, None),
    "c2kv": (4096, 1024, 32, "asym", "f16", 1, None),
    "c2gate_mma": (4096, 14336, 32, "asym", "f16", 1, 2),
    "c2gate_direct": (4096, 14336, 32, "asym", "f16", 1, 4),
    "c2gate_tmma": (4096, 14336, 32, "asym", "f16", 1, 5),
    "c2o_tmma": (4096, 4096, 32, "asym", "f16", 1, 5),
    "c2down_tmma": (14336, 4096, 32, "asym", "f16", 1, 5),
    "c2gate_regs": (4096, 14336, 32, "asym", "f16", 1, 4, 0),  # batch-1 kernel variant: weights in registers
    "c3m1": (8192, 28672, 128, "sym", "bf16", 1, None),
    "c3m16": (8192, 28672, 128, "sym", "bf16", 16, None),
    "c4m512": (4096, 14336, 128, "asym", "bf16", 512, None),
    "c4m2048": (4096, 14336, 128, "asym", "bf16", 2048, None),
    "c5m1": (4096, 14336, 0, "lut3", "bf16", 1, None),
    "c5m16": (4096, 14336, 0, "lut3", "bf16", 16, None),
    "c5m2048": (4096, 14336, 0, "lut3", "bf16", 2048, None),
    "mxfp8q": (4096, 0, 0, "mxfp8", "bf16", 2048, None),
    "c5mx2048": (4096, 14336, 0, "lut3mx", "mxfp8", 2048, None),
    "affine2": (4096, 14336, 64, "affine2", "f16", 1, None),
    "w4a8gate": (4096, 14336, 32, "w4a8", "f16", 1, None),
    # grouped MoE GEMM (E=256, top-8, H=2048 -> 2 x I=1024), 256 tokens; N is the gate/up width
    "moe256": (2048, 1024, 0, "moe", "mxfp8", 256, None),
    "affine3": (4096, 14336, 64, "affine3", "f16", 1, None),
}


def run_profile_case(name):
    """A handful of launches of one shape, each on a distinct weight copy (the
    copies total more than L2), for an ncu capture; prints nothing to parse."""
    import torch
    import bit_weight_only_pack_b200 as lbq
    import workloads
    K, N, group, mode, xdt, M, path = PROFILE_CASES[name][:7]
    variant = PROFILE_CASES[name][7] if len(PROFILE_CASES[name]) > 7 else None
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    if mode == "mxfp8":
        # activation quantiser: copies of X larger than L2 in total
        xs = [workloads.activations_device(7 + i, M, K, xdt, device)
              for i in range(max(3, 3 * l2 // (M * K * 2) + 1))]
        for X in xs:
            lbq.quantize_mxfp8(X)
        torch.cuda.synchronize()
        lbq.device_status()
        print(f"profile case {name}: {len(xs)} launches of M={M} K={K}", flush=True)
        return 0
    if mode == "lut3mx":
        # LUT3 x MXFP8: activations drawn in the format, weight copies larger than L2
        idx, cb, ex = workloads.lut3_device(7, K, N, device)
        images = weight_copies(lbq.pack_lut3(idx, cb, ex), l2)
        del idx, cb, ex
        codes_h, scales_h = workloads.mx_activations_host(7, M, K)
        codes, scales = torch.from_numpy(codes_h).to(device), torch.from_numpy(scales_h).to(device)
        ws = lbq.workspace(2, M, K, N, 0, "lut3")
        for img in images:
            lbq.lut3_mx_gemm(codes, scales, img, N, ws=ws)
        torch.cuda.synchronize()
        lbq.device_status()
        print(f"profile case {name}: {len(images)} launches of K={K} N={N} M={M}", flush=True)
        return 0
    if mode == "moe":
        E, top_k, T = MOE_LAYER["experts"], MOE_LAYER["top_k"], M
        images, stride = moe_expert_images(torch, lbq, workloads, device, 1000, K, N, E)
        aligned, codes, scales, _ = moe_inputs(torch, lbq, workloads, device, T, top_k, E, K)
        for _ in range(3):
            lbq.moe_lut3_mx_gemm(codes, scales, top_k, aligned, images, stride, E, N)
        torch.cuda.synchronize()
        lbq.device_status()
        print(f"profile case {name}: 3 launches of T={T} top_k={top_k} E={E} K={K} N={N}", flush=True)
        return 0
    if mode == "w4a8":
        # W4A8 batch-1 GEMV on asym INT4 weights: X quantised once, weight copies larger than L2
        W = workloads.weights_device(7, K, N, device)
        images = weight_copies(lbq.pack(W, group, "asym"), l2)
        del W
        X = workloads.activations_device(7, M, K, xdt, device)
        xq, sx = lbq.quantize_int8(X)
        for img in images:
            lbq.w4a8_gemv(xq, sx, img, N, group, "asym")
        torch.cuda.synchronize()
        lbq.device_status()
        print(f"profile case {name}: {len(images)} launches of K={K} N={N} W4A8 M={M}", flush=True)
        return 0
    if mode.startswith("affine"):
        # b-bit affine GEMV: weight copies larger than L2
        bits = int(mode[len("affine"):])
        W = workloads.weights_device(7, K, N, device)
        images = weight_copies(lbq.pack_affine(W, group, bits), l2)
        del W
        X = workloads.activations_device(7, M, K, xdt, device)
        for img in images:
            lbq.affine_gemv(X, img, N, group, bits)
        torch.cuda.synchronize()
        lbq.device_status()
        print(f"profile case {name}: {len(images)} launches of K={K} N={N} bits={bits} M={M}", flush=True)
        return 0
    Ns = N if isinstance(N, tuple) else (N,)
    if mode == "lut3":
        idx, cb, ex = workloads.lut3_device(7, K, N, device)
        img0 = lbq.pack_lut3(idx, cb, ex)
        del idx, cb, ex
        img0s = [img0]
    else:
        img0s = []
        for i, n in enumerate(Ns):
            W = workloads.weights_device(7 + i, K, n, device)
            img0s.append(lbq.pack(W, group, mode))
            del W
    per_launch = sum(int(i.numel()) for i in img0s)
    copies = max(3, (3 * l2) // per_launch + 1)
    sets = [img0s] + [[i.clone() for i in img0s] for _ in range(copies - 1)]
    X = workloads.activations_device(7, M, K, xdt, device)
    if path is not None:
        lbq.lbq_debug_gemv_path(path)
    if variant is not None:
        lbq.lbq_debug_direct_variant(variant)
    if mode == "lut3":
        ws = lbq.workspace(2, M, K, N, 0, "lut3")
        for imgs in sets:
            lbq.lut3_gemm(X, imgs[0], N, ws=ws)
    elif len(Ns) > 1:
        for imgs in sets:
            lbq.gemv_grouped([(X, img, n) for img, n in zip(imgs, Ns)], group, mode)
    else:
        ws = lbq.workspace(1, M, K, N, group, mode)
        for imgs in sets:
            lbq.gemm(X, imgs[0], N, group, mode, ws=ws)
    torch.cuda.synchronize()
    lbq.lbq_debug_gemv_path(0)
    lbq.lbq_debug_direct_variant(-1)
    lbq.device_status()
    print(f"profile case {name}: {len(sets)} launches of K={K} N={N} {mode} M={M}", flush=True)
    return 0


# ----------------------------------------------------------------------------- main

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# decode step's four launch shapes (q/k/v grouped, o, gate/up grouped, down),
# each from a one-launch ncu capture of its profile case summarised under
# profiles/, with hashes of the kernel's sources and of its planner at capture
# time: shape -> (bytes, {source: sha256[:16]}, summary file). Each shape runs
# once per layer, so the step's traffic per launch is their mean.
STEP_KERNEL = ("gemv_tmma_kernel (gate/up) and gemv_direct_async_kernel (q/k/v, o, down)")
STEP_SOURCES = ("gemv_tmma.cuh", "gemv_direct.cuh", "gemv_m1.cuh", "w4a8.cuh", "tma.cuh", "common.cuh",
                "lbq.cu#tmma-plan", "lbq.cu#direct-plan")
STEP_CAPTURE_HASHES = {
    "gemv_tmma.cuh": "8cbbf88b681552a5",
    "gemv_direct.cuh": "370710b80822d44e",
    "gemv_m1.cuh": "a992f85dd1acbd76",
    "w4a8.cuh": "9b2ae43b5bafb58f",
    "tma.cuh": "5f428384c68b0ba7",
    "common.cuh": "6e369f75860e0aec",
    "lbq.cu#tmma-plan": "9cb96b64b3d66c78",
    "lbq.cu#direct-plan": "b62033ebadd8a276",
}
STEP_TRAFFIC = {
    "c2qkv": (14980608, STEP_CAPTURE_HASHES, "profiles/gemv_decode_step_shapes_4096x_asym_g32_m1.md"),
    "c2o": (9997056, STEP_CAPTURE_HASHES, "profiles/gemv_decode_step_shapes_4096x_asym_g32_m1.md"),
    "c2gateup": (70270976, STEP_CAPTURE_HASHES, "profiles/gemv_decode_step_shapes_4096x_asym_g32_m1.md"),
    "c2down": (34921728, STEP_CAPTURE_HASHES, "profiles/gemv_decode_step_shapes_4096x_asym_g32_m1.md"),
}
# the planner sections of lbq.cu (kernel choice, launch shape, K split, stages)
PLAN_MARKERS = {"tmma-plan": ("// M = 1: TMA-fed warp-MMA GEMV", "// Scratch of that kernel for one call"),
                "direct-plan": ("static lbq_status run_direct(", "// ----------------------------------------------------------------------------\n// M = 1: TMA-fed")}


def source_hash(name):
    """sha256[:16] of a kernel source, or of the marked planner section of lbq.cu."""
    import hashlib
    fname, _, section = name.partition("#")
    with open(os.path.join(ROOT, "bit_weight_only_pack_b200", "csrc", fname), "rb") as f:
        data = f.read()
    if section:
        a, b = (m.encode() for m in PLAN_MARKERS[section])
        i, j = data.find(a), data.find(b)
        if i < 0 or j < i:
            return None
        data = data[i:j]
    return hashlib.sha256(data).hexdigest()[:16]


def current_hashes():
    return {f: source_hash(f) for f in STEP_SOURCES}


def traffic_from_profiles():
    """Mean recorded DRAM bytes per launch of the step, or None when a shape has
    no record or a kernel source or the planner changed since its capture."""
    vals = []
    now = current_hashes()
    for nbytes, sources, _summary in STEP_TRAFFIC.values():
        if nbytes is None or sources != now:
            return None
        vals.append(nbytes)
    return sum(vals) / len(vals)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lbq", choices=["lbq", "reference"])
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--quick", action="store_true", help="skip the longer secondary measurements")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch the decode-step GEMVs without programmatic dependent launch")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--ungrouped", action="store_true",
                    help="one lbq_gemv launch per projection instead of grouped q/k/v and gate/up")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=2,
                    help="groups of layers whose host copies overlap the other groups' GEMVs in the e2e step")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run a small case for ncu (a few launches over weight copies larger than L2) and exit")
    args = ap.parse_args()
    if args.profile:
        return run_profile_case(args.profile)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import bit_weight_only_pack_b200 as lbq
    import workloads

    world, rank, local = dist_setup()
    device = torch.device("cuda", local)
    peaks = load_peaks()

    step = DecodeStep(torch, lbq, workloads, device, args.layers, grouped=not args.ungrouped)
    # the step's weights are written once and then only read, so the GEMVs may
    # overlap their weight streaming with the previous kernel's tail
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0 if args.no_pdl else 1)
    graph = step.capture()
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)
    sampler = ClockSampler(physical_gpu_index(local))
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    elapsed_ms = time_graph(torch, graph, args.steps, 0, world)
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(world, elapsed_ms)
    ms_per_step = elapsed_ms / args.steps
    value = world * step.bytes / (ms_per_step / 1e3) / 1e9

    # end to end through the public C-ABI call: every step copies its
    # activations in from pinned host memory, makes the step's C-ABI calls
    # (no graph) and copies the outputs back to pinned host memory
    e2e = E2EStep(torch, step, chunks=max(1, args.e2e_groups))
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0 if args.no_pdl else 1)
    for _ in range(args.warmup):
        e2e.run()
    e2e.finish()
    torch.cuda.synchronize()
    barrier(world)
    launches_before = lbq.lbq_launch_count()  # the timed steps' launches only
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    e2e.reset()
    for _ in range(args.steps):
        e2e.run()
    e2e.finish()
    e1.record()
    torch.cuda.synchronize()
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)
    e2e_launches = lbq.lbq_launch_count() - launches_before
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1)) / args.steps
    lbq.device_status()

    secondary = None
    if not args.no_secondary:
        sec_sampler = ClockSampler(physical_gpu_index(local))
        sec_sampler.start()
        time.sleep(0.25)
        secondary = secondary_measurements(torch, lbq, workloads, device, peaks, args.quick)
        secondary["clocks"] = sec_sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(10.0)
        cpu["one_core"] = oracle_one_core(4.0)
        cpu["per_config"] = oracle_per_config()

    hbm = peaks["hbm_gbs"]
    per_gpu = step.bytes / (ms_per_step / 1e3) / 1e9
    launches = step.launches_per_step
    # DRAM bytes per launch of the step from an ncu capture (see profiles/), for the default step only
    traffic = traffic_from_profiles() if (args.layers == 32 and not args.ungrouped) else None
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "Llama-3-8B-shaped decode step at M=1, 7 projections x %d layers, asymmetric "
                               "INT4 group 32 (fp16 scale + int8 zp), fp16 X, fp16 Y" % args.layers,
                   "weight_bytes_per_step": step.bytes, "gemvs_per_step": step.n_gemvs,
                   "launches_per_step": step.launches_per_step,
                   "grouping": "q/k/v and gate/up share X and run as one grouped launch each"
                               if step.grouped else "one launch per projection",
                   "l2": "inputs larger than L2 (%.2f GB of weights per step vs %d MB L2); no flush"
                         % (step.bytes / 1e9, torch.cuda.get_device_properties(device).L2_cache_size >> 20),
                   "timing": "CUDA events around K replays of one CUDA graph holding the step",
                   "pdl": not args.no_pdl,
                   "parallelism": "replicas" if world > 1 else "1 GPU"},
        "frac_hbm": per_gpu / hbm,
        "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": hbm, "unit": "GB/s", "frac": per_gpu / hbm,
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peaks["source"],
                     "traffic": traffic,
                     "kernel": STEP_KERNEL,
                     "per_launch": "algorithmic bytes per launch averaged over the step's %d launches (%.0f B) / "
                                   "average launch time (step time / launches); traffic = ncu DRAM read+write "
                                   "bytes per launch of the step's four launch shapes (one-launch captures), "
                                   "their mean; null if the kernel or its planner changed since the capture"
                                   % (launches, step.bytes / max(launches, 1)),
                     "algorithmic_bytes_per_step": step.bytes},
        "clocks": clocks,
        "e2e": {"value": world * step.bytes / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": step.x_all.numel() * 2, "d2h_bytes_per_step": step.y_all.numel() * 2,
                "ms_per_step": e2e_ms, "kernel_launches": e2e_launches,
                "how": "per step: pinned host X -> device, the step's lbq_gemv / lbq_gemv_grouped C-ABI calls "
                       "(no graph), device Y -> pinned host; in %d groups of layers, X in on one copy stream "
                       "(a group's next-step X as soon as this step's GEMVs of the group have read it), Y out on "
                       "another (as soon as the group's GEMVs are done), each group's GEMVs waiting only for its "
                       "own X and its previous Y copy; CUDA events on the launching stream, the first step's "
                       "copies after the start event and the end event after the last copy" % len(e2e.groups)},
        "gpu_launches": launches * args.steps,
        "cpu_baseline": cpu,
        "secondary": secondary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
