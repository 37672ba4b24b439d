"""Benchmark of the group-wise quantization hot path on B200.

One step = one pass of every hot-path row over the decode workload of the 4-bit GEMV
configuration (three weight matrices 4096x4096, 11008x4096, 4096x11008, drawn as
0.02 * Student-t(5) with 0.1% of entries x10):

    quantize (fp32 -> 4-bit codes, fp16 scales, u8 zeros)   -> pack into the 4-bit plane
    -> project a bf16 residual ~ N(0, (0.3 s)^2) into the cells -> requant-verify with it and
    without it (revocation), both in one pass -> dequant-GEMV at batch 1 (decode)
    -> dequant-GEMM at batch 64

The three matrices are one flat artifact (their buffers back to back), so quantize, pack,
project and the verify pair each run as one call over all of them; the GEMV and the GEMM run per
matrix.  K steps are captured as one CUDA graph and replayed for the timed region; per-row
durations come from a second K-step graph with an event pair around each row's calls, replayed
after it.
Printed: one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cq|reference]
       (N > 1: launch with torch.distributed.run, one process per GPU)
"""
import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

GROUP = 64
SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]       # rows (out) x cols (in)
N_LAYERS = 32
GEMM_M = 64
METRIC = "dequant-GEMV weight GB/s & tokens/s vs HBM peak; requant-verify weights/s"
WORKLOAD = "4-bit g=64 decode matrices 4096x4096, 11008x4096, 4096x11008 (0.02*t5, 0.1% outliers x10)"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# algorithmic bytes per weight of each step: what the method must move, counted from the formats
def kernel_bytes(n):
    G = n // GROUP
    meta = 3 * G                      # fp16 scale + u8 zero per group
    return {
        "quantize": 4 * n + n + meta,                 # read fp32 W, write u8 codes + meta
        "pack": n + n // 2,                           # read codes, write nibbles
        "project": 2 * n + 2 * n + 2 * G,             # read + write bf16 r, read scales
        # both checks (with r, and with r dropped) in one pass: codes + meta + bf16 r
        "verify_pair": n // 2 + meta + 2 * n,
        "gemv": n // 2 + meta,                        # weights (x, y negligible)
        "gemm": n // 2 + meta,
    }


KERNELS = ["quantize", "pack", "project", "verify_pair", "gemv", "gemm"]

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of
# the kernel's launch in a step of this workload (one launch over the three matrices' flat
# artifact; mean of two steps), taken with the kernel as it is now; a kernel changed since its
# capture gets no entry (traffic null).
MEASURED_TRAFFIC = {"quantize": 517.3e6}


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------------------
def count_kernel_nodes(graph):
    """Number of kernel nodes in a captured graph (all of them are libcq kernels)."""
    from cuda.bindings import driver as drv
    h = drv.CUgraph(graph.raw_cuda_graph())
    err, _, n = drv.cuGraphGetNodes(h, 0)
    if err != drv.CUresult.CUDA_SUCCESS:
        return None
    err, nodes, n = drv.cuGraphGetNodes(h, n)
    kinds = [drv.cuGraphNodeGetType(nd)[1] for nd in nodes]
    return sum(1 for k in kinds if k == drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL)


class Workload:
    """The three decode matrices as one flat artifact: their fp32 weights, codes, scales, zero
    points, 4-bit plane and bf16 residuals are allocated back to back, so the streaming rows
    (quantize, pack, project, both verify checks) each run as one call over all of them -- the
    format is a flat sequence of 64-weight groups, whatever the matrix shapes -- while the GEMV
    and the GEMM run per matrix on views of the same buffers."""

    def __init__(self, torch, cq, ops, synth, device, seed_base=1):
        self.torch, self.cq, self.ops = torch, cq, ops
        ns = [N * K for (N, K) in SHAPES]
        n_all = sum(ns)
        G_all = n_all // GROUP
        self.n_all = n_all
        w_parts, r_parts = [], []
        self.w = torch.empty(n_all, dtype=torch.float32, device=device)
        self.codes = torch.empty(n_all, dtype=torch.uint8, device=device)
        self.scale = torch.empty(G_all, dtype=torch.int16, device=device)
        self.zero = torch.empty(G_all, dtype=torch.uint8, device=device)
        self.plane = torch.empty(n_all // 2, dtype=torch.uint8, device=device)
        self.r = torch.empty(n_all, dtype=torch.bfloat16, device=device)
        for idx, (N, K) in enumerate(SHAPES):
            w_parts.append(synth.student_t_weights(N, K, seed=seed_base + 1000 * idx).ravel())
        self.w_host = torch.from_numpy(np.concatenate(w_parts)).pin_memory()
        self.w.copy_(self.w_host)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        cq.cq_quantize(self.w.view(1, n_all), None, self.codes, self.scale, self.zero, st)
        cq.cq_pack_varbits(self.codes, G_all, None, None, [None, None, self.plane, None])
        scale_np = self.scale.cpu().view(torch.int16).numpy().view(np.uint16)
        self.mats = []
        off = 0
        for idx, (N, K) in enumerate(SHAPES):
            n = N * K
            g0, g1 = off // GROUP, (off + n) // GROUP
            r_parts.append(synth.normal_residual_bf16(scale_np[g0:g1], seed=seed_base + 1000 * idx + 7,
                                                      rel_sigma=0.3).view(np.int16))
            x = synth.activations(1, K, seed=seed_base + 1000 * idx + 11, dtype="bf16")
            X = synth.activations(GEMM_M, K, seed=seed_base + 1000 * idx + 13, dtype="bf16")
            x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
            X_host = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
            qw = cq.QWeight(N, K, [None, None, self.plane[off // 2:(off + n) // 2], None], self.scale[g0:g1],
                            self.zero[g0:g1])
            m = dict(N=N, K=K, n=n, qw=qw, x_host=x_host, x=x_host.to(device), X_host=X_host, X=X_host.to(device),
                     y=torch.empty(1, N, device=device), Y=torch.empty(GEMM_M, N, device=device))
            need = cq.cq_gemm_workspace(N, K, GEMM_M)
            m["ws"] = torch.empty(max(need, 16), dtype=torch.uint8, device=device) if need else None
            self.mats.append(m)
            off += n
        self.r_host = torch.from_numpy(np.concatenate(r_parts)).view(torch.bfloat16).pin_memory()
        self.r.copy_(self.r_host)
        self.qw_all = cq.QWeight(1, n_all, [None, None, self.plane, None], self.scale, self.zero, residual=self.r)
        z = lambda dt: torch.zeros(1, dtype=dt, device=device)
        self.status, self.nclamp = z(torch.int32), z(torch.int64)
        self.mism, self.first, self.mism0, self.first0 = z(torch.int64), z(torch.int64), z(torch.int64), z(torch.int64)
        torch.cuda.synchronize()

    def step(self, stream, marks=None):
        """Enqueue one step: quantize, pack, project and both verify checks each as one call over
        the three matrices' flat artifact, then the GEMV and the GEMM per matrix. marks[kernel] =
        (start, end) external events around a row's calls: recorded inside a graph capture they
        become event nodes that time the row on replay (one pair per row keeps their own cost out
        of the launches they time)."""
        cq = self.cq

        def row(name, fn):
            if marks is not None:
                marks[name][0].record(stream)
            fn()
            if marks is not None:
                marks[name][1].record(stream)

        row("quantize", lambda: cq.cq_quantize(self.w.view(1, self.n_all), None, self.codes, self.scale, self.zero,
                                               self.status, stream))
        row("pack", lambda: cq.cq_pack_varbits(self.codes, self.n_all // GROUP, None, None,
                                               [None, None, self.plane, None], stream))
        row("project", lambda: cq.cq_project_residual(self.r, self.scale, self.nclamp, stream))
        row("verify_pair", lambda: cq.cq_requant_verify_pair(self.qw_all, 0, self.n_all, self.mism, self.first,
                                                             self.mism0, self.first0, None, stream))
        row("gemv", lambda: [cq.cq_dequant_gemv(m["qw"], m["x"], m["y"], stream) for m in self.mats])
        row("gemm", lambda: [cq.cq_dequant_gemm(m["qw"], m["X"], m["Y"], m["ws"], stream) for m in self.mats])

    def n_weights(self):
        return sum(m["n"] for m in self.mats)

    def step_bytes(self):
        tot = {k: 0 for k in KERNELS}
        for m in self.mats:
            for k, v in kernel_bytes(m["n"]).items():
                tot[k] += v
        return tot


def launches_of(kernel, wl):
    """Main-kernel launches of a row per step: the streaming rows run once over the flat artifact,
    the GEMV and the GEMM once per matrix."""
    return len(wl.mats) if kernel in ("gemv", "gemm") else 1


def max_over_ranks(value, dist, device):
    """The largest of the ranks' values, on every rank (identity without a process group):
    multi-GPU times are the slowest rank's."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(bytes_per_rank_step, world, ms_per_step):
    """Whole-job throughput in GB/s: every rank's bytes over the (max-over-ranks) step time."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


def time_graph(torch, graph, reps, stream):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(reps):
            graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def isolated_components(torch, cq, ops, device, peaks, stream):
    """Cold-L2 component rates: GEMV (rotating > 2x L2), the 32-layer decode proxy, verify."""
    torch.manual_seed(2026)              # every draw below (weights, activations) is seeded
    out = {}
    L2 = torch.cuda.get_device_properties(device).L2_cache_size
    # 32-layer 7B-shaped decode: distinct weights per layer (3.54 GB), one graph per token. Per
    # layer: q, k, v (4096x4096, one fused launch: they read the same x), o, gate and up
    # (11008x4096, one fused launch), down (4096x11008); the unfused variant launches all seven.
    base = []
    for (N, K) in SHAPES:
        w = torch.randn(N, K, device=device) * 0.02
        qw, _, _ = ops.quantize_and_pack(w)
        base.append(qw)
        del w

    def clone(q):
        return cq.QWeight(q.rows, q.cols, [None, None, q.planes[2].clone(), None], q.scale.clone(), q.zero.clone())

    stack = [{"qkv": [clone(base[0]) for _ in range(3)], "o": clone(base[0]),
              "gu": [clone(base[1]) for _ in range(2)], "down": clone(base[2])} for _ in range(N_LAYERS)]
    layers = [q for L in stack for q in L["qkv"] + [L["o"]] + L["gu"] + [L["down"]]]
    xs = {K: torch.randn(1, K, device=device).to(torch.bfloat16) for (_, K) in SHAPES}
    ys = {N: torch.empty(1, N, device=device) for (N, _) in SHAPES}
    y4 = [torch.empty(1, 4096, device=device) for _ in range(3)]
    y11 = [torch.empty(1, 11008, device=device) for _ in range(2)]
    token_bytes = sum(q.rows * q.cols // 2 + 3 * q.rows * q.cols // GROUP for q in layers)

    def token(fused):
        for L in stack:
            if fused:
                cq.cq_dequant_gemv_multi(L["qkv"], xs[4096], y4, stream)
                cq.cq_dequant_gemv(L["o"], xs[4096], y4[0], stream)
                cq.cq_dequant_gemv_multi(L["gu"], xs[4096], y11, stream)
                cq.cq_dequant_gemv(L["down"], xs[11008], y4[1], stream)
            else:
                for q in L["qkv"] + [L["o"]] + L["gu"] + [L["down"]]:
                    cq.cq_dequant_gemv(q, xs[q.cols], ys[q.rows], stream)

    for fused in (True, False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            token(fused)     # warm-up outside capture
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=stream):
                token(fused)
        for _ in range(3):
            g.replay()
        t_ms = time_graph(torch, g, 20, stream)
        key = "decode_32_layers" if fused else "decode_32_layers_unfused"
        out[key] = {"tokens_per_s": 1e3 / t_ms, "ms_per_token": t_ms, "weight_bytes_per_token": token_bytes,
                    "GBps": token_bytes / t_ms / 1e6, "frac_hbm": token_bytes / t_ms / 1e6 / peaks["hbm_gbs"],
                    "ceiling_tokens_per_s": peaks["hbm_gbs"] * 1e9 / token_bytes,
                    "launches_per_token": N_LAYERS * (4 if fused else 7)}
        del g
    # per shape, the same pool (rotation over 32 copies > 2 x L2)
    per = {}
    for si, (N, K) in enumerate(SHAPES):
        pool = [q for q in layers if q.rows == N and q.cols == K]
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g1, stream=stream):
                for q in pool:
                    cq.cq_dequant_gemv(q, xs[K], ys[N], stream)
        g1.replay()
        t = time_graph(torch, g1, 10, stream) / len(pool)
        b = N * K // 2 + 3 * N * K // GROUP
        per[f"{N}x{K}"] = {"us": t * 1e3, "GBps": b / t / 1e6, "frac_hbm": b / t / 1e6 / peaks["hbm_gbs"]}
        del g1
    out["gemv_m1_cold"] = per
    out["l2_bytes"] = L2
    del layers, stack
    torch.cuda.empty_cache()
    # fixed-4 pack of 8192x16384 codes from two alternating copies (268 MB > 2 x L2): every code
    # byte comes from HBM
    n = 8192 * 16384
    codes = [torch.randint(0, 16, (n,), dtype=torch.uint8, device=device) for _ in range(2)]
    plane = torch.empty(n // 2, dtype=torch.uint8, device=device)
    gp = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for c in codes:
            cq.cq_pack_varbits(c, n // GROUP, None, None, [None, None, plane, None], stream)
        torch.cuda.synchronize()
        with torch.cuda.graph(gp, stream=stream):
            for _ in range(5):
                for c in codes:
                    cq.cq_pack_varbits(c, n // GROUP, None, None, [None, None, plane, None], stream)
    gp.replay()
    t = time_graph(torch, gp, 3, stream) / 10
    b = n + n // 2
    out["pack_cold_8192x16384"] = {"us": t * 1e3, "GBps": b / t / 1e6, "frac_hbm": b / t / 1e6 / peaks["hbm_gbs"]}
    del gp, codes, plane
    torch.cuda.empty_cache()
    out["cellfill_stack"] = cellfill_stack_verify(torch, cq, ops, synth_module(), device, peaks, stream)
    out["rrq"] = rrq_components(torch, cq, ops, device, peaks, stream)
    out["vbq"] = vbq_components(torch, cq, ops, synth_module(), device, peaks, stream)
    out["scale_verify_2_4e10"] = scale_chunked_verify(torch, cq, ops, synth_module(), device, peaks, stream)
    out["requant"] = requant_components(torch, cq, ops, device, stream)
    return out


def vbq_components(torch, cq, ops, synth, device, peaks, stream):
    """Per-group widths on the 2048x8192 shape of the VBQ configuration (widths drawn from
    {1, 2, 4, 8} with probabilities .69/.15/.12/.04, mean 1.79 bits): quantize with the width map
    (4 B read + 1 B code + 3/64 B scale/zero + 1/64 B width per weight), the offset index (1 B
    read, 4 B written per group), pack (1 B code + 5/64 B index read, the planes written),
    unpack (the reverse), and the GEMV at m = 1 and m = 8 (planes + 3/64 B scale/zero + 5/64 B
    width/offset per weight). One matrix is 5.9 MB packed, far below L2, so every figure comes
    from a pool of copies run back to back in one graph (32 for the GEMV, 187 MB; 8 for the
    others), which also shows the grouped launch escaping launch latency."""
    N, K = 2048, 8192
    G = N * K // GROUP
    bits = torch.from_numpy(synth.vbq_bits(G, seed=2)).to(device)
    offset, pb = ops.varbits_index(bits, stream)
    plane_bytes = sum(pb)
    out = {"shape": f"{N}x{K}", "mean_bits": plane_bytes * 8 / (N * K), "plane_bytes": plane_bytes}

    def timed(fn, n_in_pool, bytes_one):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            fn()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=stream):
                fn()
        g.replay()
        t = time_graph(torch, g, 10, stream) / n_in_pool
        del g
        return {"us": t * 1e3, "GBps": bytes_one / t / 1e6, "frac_hbm": bytes_one / t / 1e6 / peaks["hbm_gbs"]}

    ws = [torch.randn(N, K, device=device) * 0.02 for _ in range(8)]
    qs = [ops.quantize_and_pack(w, bits, stream) for w in ws]
    codes_out = [torch.empty(N * K, dtype=torch.uint8, device=device) for _ in range(8)]
    sc = torch.empty(G, dtype=torch.int16, device=device)
    zr = torch.empty(G, dtype=torch.uint8, device=device)
    off2 = torch.empty(G, dtype=torch.int32, device=device)
    pb2 = torch.empty(4, dtype=torch.int64, device=device)
    out["quantize"] = timed(lambda: [cq.cq_quantize(w, bits, c, sc, zr, None, stream) for w, c in zip(ws, codes_out)],
                            8, N * K * 5 + G * 4)
    out["index"] = timed(lambda: [cq.cq_varbits_index(bits, off2, pb2, stream) for _ in range(8)], 8, G * 5)
    out["pack"] = timed(lambda: [cq.cq_pack_varbits(c, G, bits, offset, q.planes, stream)
                                 for (q, c, _), _ in zip(qs, range(8))], 8, N * K + G * 5 + plane_bytes)
    out["unpack"] = timed(lambda: [cq.cq_unpack_varbits(q, c, stream) for (q, _, _), c in zip(qs, codes_out)],
                          8, N * K + G * 5 + plane_bytes)
    del ws
    torch.cuda.empty_cache()
    # 32 packed copies for the GEMV pool
    pool = [q for q, _, _ in qs]
    while len(pool) < 32:
        q = pool[len(pool) % 8]
        pool.append(cq.QWeight(N, K, [p.clone() if p is not None else None for p in q.planes], q.scale.clone(),
                               q.zero.clone(), q.bits, q.offset))
    gemv_bytes = plane_bytes + G * 8
    for m in (1, 8):
        x = torch.randn(m, K, device=device).to(torch.bfloat16)
        y = torch.empty(m, N, device=device)
        out[f"gemv_m{m}"] = timed(lambda: [cq.cq_dequant_gemv(q, x, y, stream) for q in pool], len(pool), gemv_bytes)
    del pool, qs, codes_out
    torch.cuda.empty_cache()
    return out


def rrq_components(torch, cq, ops, device, peaks, stream):
    """Recurrent residual quantization on the config's 11008x4096 shape (4 two-bit stages =
    the 8-bit model): one stage (quantize the fp32 residual, write codes, scales, zero points
    and the new residual: 9 + 3/64 B per weight), and the stage-stack GEMV at m=1 over 1, 2
    and 4 stages (per stage 0.25 B codes + 3/64 B scale/zero; the stages share one 5/64 B width
    map and offset index), at m = 1 and m = 8, rotating over three stacks so the weights come
    from HBM."""
    N, K = 11008, 4096
    G = N * K // GROUP
    w = torch.randn(N, K, device=device) * 0.02
    stages, _, _ = ops.rrq_build(w, 4)
    r = w.clone()
    codes = torch.empty(N * K, dtype=torch.uint8, device=device)
    sc = torch.empty(G, dtype=torch.int16, device=device)
    zr = torch.empty(G, dtype=torch.uint8, device=device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        cq.cq_rrq_stage(r, 2, codes, sc, zr, None, stream)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            cq.cq_rrq_stage(r, 2, codes, sc, zr, None, stream)
    t = time_graph(torch, g, 10, stream)
    b = N * K * 9 + G * 3
    out = {"shape": f"{N}x{K}", "stage": {"us": t * 1e3, "GBps": b / t / 1e6, "frac_hbm": b / t / 1e6 / peaks["hbm_gbs"]}}
    # the stage-stack GEMV over a pool of stacks larger than L2 (3 x 4 stages x 17 MB)
    pool = [stages] + [ops.rrq_build(w * (1.0 + 0.01 * i), 4)[0] for i in (1, 2)]
    for m in (1, 8):
        x = torch.randn(m, K, device=device).to(torch.bfloat16)
        y = torch.empty(m, N, device=device)
        for n in (1, 2, 4):
            gs = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                for st in pool:
                    cq.cq_dequant_gemv_stages(st[:n], x, y, stream)
                torch.cuda.synchronize()
                with torch.cuda.graph(gs, stream=stream):
                    for st in pool:
                        cq.cq_dequant_gemv_stages(st[:n], x, y, stream)
            gs.replay()
            t = time_graph(torch, gs, 10, stream) / len(pool)
            b = n * (N * K // 4 + G * 3) + G * 5        # the stages share one width map and index
            out[f"gemv_m{m}_{n}_stages"] = {"us": t * 1e3, "GBps": b / t / 1e6,
                                            "frac_hbm": b / t / 1e6 / peaks["hbm_gbs"]}
            del gs
    del stages, pool, w, r, g
    torch.cuda.empty_cache()
    return out


def synth_module():
    from cell_updates_b200 import synth
    return synth


def cellfill_stack_verify(torch, cq, ops, synth, device, peaks, stream):
    """The CellFill configuration at its own size: a 28-layer 1.7B-shaped stack
    (1,526,726,656 weights, frozen 4-bit codes, bf16 residuals ~N(0,(0.3 s)^2)) built on the
    device by the counter-based generator; project, verify with the residual, verify without it
    (revocation), each over the whole stack in one call; then the bounded reparameterization
    (bf16 residual from an fp32 parameter theta ~ N(0, 2^2)) and its backward pass, whose
    residual is verified once more. Rates in weights/s and GB/s."""
    n = 28 * (4 * 2048 * 2048 + 2 * 2048 * 6144 + 6144 * 2048)
    G = n // GROUP
    plane = torch.empty(n // 2, dtype=torch.uint8, device=device)
    scale = torch.empty(G, dtype=torch.int16, device=device)
    zero = torch.empty(G, dtype=torch.uint8, device=device)
    r = torch.empty(n, dtype=torch.bfloat16, device=device)
    with torch.cuda.stream(stream):
        cq.cqs_code_words(plane.view(torch.int64), 3, 0, stream)
        cq.cqs_scales(scale, 3, 0, stream)
        cq.cqs_zeros(zero, 3, 0, stream)
        cq.cqs_residual_bf16(r, scale, 3, 0, float(synth.ih4_multiplier(0.3)), stream)
    torch.cuda.synchronize()
    ncl = torch.zeros(1, dtype=torch.int64, device=device)
    mism = torch.zeros(1, dtype=torch.int64, device=device)
    first = torch.zeros(1, dtype=torch.int64, device=device)
    mism0 = torch.zeros(1, dtype=torch.int64, device=device)
    first0 = torch.zeros(1, dtype=torch.int64, device=device)
    theta = torch.empty(n, dtype=torch.float32, device=device)
    grad = torch.empty(n, dtype=torch.float32, device=device)
    grad_theta = torch.empty(n, dtype=torch.float32, device=device)
    with torch.cuda.stream(stream):
        cq.cqs_normal_f32(theta, 3, 9, 0, float(synth.ih4_multiplier(2.0)), stream)
        cq.cqs_normal_f32(grad, 3, 10, 0, float(synth.ih4_multiplier(1.0)), stream)
    torch.cuda.synchronize()
    qw_r = cq.QWeight(1, n, [None, None, plane, None], scale, zero, residual=r)
    qw_0 = cq.QWeight(1, n, [None, None, plane, None], scale, zero)
    res = {"weights": n}
    calls = {"project": lambda: cq.cq_project_residual(r, scale, ncl, stream),
             "verify": lambda: cq.cq_requant_verify(qw_r, 0, n, mism, first, None, stream),
             "revoke_verify": lambda: cq.cq_requant_verify(qw_0, 0, n, mism, first, None, stream),
             "verify_pair": lambda: cq.cq_requant_verify_pair(qw_r, 0, n, mism, first, mism0, first0, None, stream),
             "reparam": lambda: cq.cq_reparam_residual(theta, scale, r, stream),
             "reparam_grad": lambda: cq.cq_reparam_residual_grad(theta, scale, grad, grad_theta, cq.CQ_BF16, stream)}
    # bytes per weight: read theta (4), write the bf16 residual (2) / read theta and dL/dr, write
    # dL/dtheta (12); plus the group's scale
    per_w = {"project": 4.0 + 2.0 / GROUP, "verify": 2.5 + 3.0 / GROUP, "revoke_verify": 0.5 + 3.0 / GROUP,
             "verify_pair": 2.5 + 3.0 / GROUP, "reparam": 6.0 + 2.0 / GROUP, "reparam_grad": 12.0 + 2.0 / GROUP}
    for name, fn in calls.items():
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                fn()
        g.replay()
        ms = time_graph(torch, g, 10, stream)
        if name in ("verify", "revoke_verify", "verify_pair"):
            assert int(mism.item()) == 0, f"{name}: {int(mism.item())} mismatches"
        if name == "verify_pair":
            assert int(mism0.item()) == 0, f"{name}: {int(mism0.item())} revocation mismatches"
        res[name] = {"ms": ms, "weights_per_s": n / (ms * 1e-3), "GBps": n * per_w[name] / (ms * 1e-3) / 1e9,
                     "frac_hbm": n * per_w[name] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        del g
    # the reparameterized residual re-quantizes to the codes, and dropping it revokes
    with torch.cuda.stream(stream):
        cq.cq_requant_verify_pair(qw_r, 0, n, mism, first, mism0, first0, None, stream)
    torch.cuda.synchronize()
    assert int(mism.item()) == 0 and int(mism0.item()) == 0, "reparameterized residual left its cell"
    res["decode_28_layers_served"] = cellfill_decode(torch, cq, plane, scale, zero, r, device, peaks, stream)
    del plane, scale, zero, r, qw_r, qw_0, theta, grad, grad_theta
    torch.cuda.empty_cache()
    return res


def cellfill_decode(torch, cq, plane, scale, zero, r, device, peaks, stream):
    """Decode over the CellFill stack as served (W = s (q - z) + r, bf16 residual): the 28
    layers' q, k, v, o (2048x2048), gate and up (6144x2048) and down (2048x6144) are consecutive
    slices of the stack's artifact; one token = 196 GEMVs at batch 1 in 112 launches (q/k/v and
    gate/up fused) in one graph, every weight's code, scale, zero point and residual read once
    (2.546875 B per weight, 3.89 GB per token)."""
    shapes = [(2048, 2048)] * 4 + [(6144, 2048)] * 2 + [(2048, 6144)]
    mats, off = [], 0
    for _ in range(28):
        for (N, K) in shapes:
            n = N * K
            mats.append(cq.QWeight(N, K, [None, None, plane[off // 2:(off + n) // 2], None],
                                   scale[off // GROUP:(off + n) // GROUP], zero[off // GROUP:(off + n) // GROUP],
                                   residual=r[off:off + n]))
            off += n
    assert off == plane.numel() * 2
    xs = {K: torch.randn(1, K, device=device).to(torch.bfloat16) for K in (2048, 6144)}
    ys = {N: torch.empty(1, N, device=device) for N in (2048, 6144)}
    token_bytes = off * (2.5 + 3.0 / GROUP)

    yq = [torch.empty(1, 2048, device=device) for _ in range(3)]
    yg = [torch.empty(1, 6144, device=device) for _ in range(2)]

    def token():
        # per layer: q, k, v in one launch (they read the same x), o, gate and up in one launch, down
        for L in range(28):
            q = mats[7 * L:7 * L + 7]
            cq.cq_dequant_gemv_multi(q[0:3], xs[2048], yq, stream)
            cq.cq_dequant_gemv(q[3], xs[2048], ys[2048], stream)
            cq.cq_dequant_gemv_multi(q[4:6], xs[2048], yg, stream)
            cq.cq_dequant_gemv(q[6], xs[6144], ys[2048], stream)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        token()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            token()
    for _ in range(3):
        g.replay()
    t_ms = time_graph(torch, g, 10, stream)
    out = {"tokens_per_s": 1e3 / t_ms, "ms_per_token": t_ms, "weight_bytes_per_token": token_bytes,
           "GBps": token_bytes / t_ms / 1e6, "frac_hbm": token_bytes / t_ms / 1e6 / peaks["hbm_gbs"],
           "ceiling_tokens_per_s": peaks["hbm_gbs"] * 1e9 / token_bytes, "launches_per_token": 4 * 28}
    # per shape over the 28 layers' copies (each shape's pool is larger than L2)
    per = {}
    for (N, K) in sorted(set(shapes)):
        pool = [q for q in mats if q.rows == N and q.cols == K]
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g1, stream=stream):
                for q in pool:
                    cq.cq_dequant_gemv(q, xs[K], ys[N], stream)
        g1.replay()
        t = time_graph(torch, g1, 5, stream) / len(pool)
        b = N * K * (2.5 + 3.0 / GROUP)
        per[f"{N}x{K}"] = {"us": t * 1e3, "GBps": b / t / 1e6, "frac_hbm": b / t / 1e6 / peaks["hbm_gbs"]}
        del g1
    out["gemv_m1_cold"] = per
    del g
    return out


def requant_components(torch, cq, ops, device, stream):
    """ReQuant on the decode configuration's 4096x4096 shape: round-to-nearest codes of weights
    ~0.02 t(5) (the same recipe), refined against H = X^T X from 1024 synthetic calibration rows
    (N(0, 1) with 1/32 of the input channels x10); the gradient pass, one sweep and the closing
    error pass, then four sweeps. Reports time, accepted moves and the output-error ratio."""
    from cell_updates_b200 import synth
    N, K = SHAPES[0]
    w = torch.from_numpy(synth.student_t_weights(N, K, seed=1)).to(device)
    codes, scale, zero, _ = ops.quantize(w)
    gen = torch.Generator(device=device)
    gen.manual_seed(2027)
    X = torch.randn(1024, K, device=device, dtype=torch.float64, generator=gen)
    X[:, torch.randperm(K, device=device, generator=gen)[:K // 32]] *= 10.0
    H = X.T @ X
    H = (H + H.T) * 0.5
    del X
    out = {"shape": f"{N}x{K}", "calibration_rows": 1024}
    for sweeps in (1, 4):
        q = codes.clone()
        eb = torch.empty(N, dtype=torch.float64, device=device)
        ea = torch.empty(N, dtype=torch.float64, device=device)
        mv = torch.empty(N, dtype=torch.int64, device=device)
        ws = torch.empty(cq.cq_requant_workspace(N, K), dtype=torch.uint8, device=device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            cq.cq_requant_refine(w, H, scale, zero, 4, q, sweeps, eb, ea, mv, ws, stream)
            b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        out[f"sweeps_{sweeps}"] = {"ms": ms, "weights_per_s": N * K * sweeps / (ms * 1e-3),
                                   "moves": int(mv.sum().item()),
                                   "error_ratio_mean": float((ea / eb).mean().item())}
    del H, w
    torch.cuda.empty_cache()
    return out


def scale_chunked_verify(torch, cq, ops, synth, device, peaks, stream):
    """The scale configuration's verify: 2.4e10 constrained 4-bit weights with bf16 residuals
    (~61 GB resident: 12 GB codes, 1.1 GB scales and zeros, 48 GB residuals), built on the
    device by the counter-based generator (seed 4), projected once, then both CellFill checks
    (with the residual and revoked) over the whole artifact in chunks of 2^31 weights, the
    chunks' calls captured in one graph. Rates in weights/s and GB/s (2.5 + 3/64 B per weight)."""
    n = 24_000_000_000
    chunk = 1 << 31
    G = n // GROUP
    torch.cuda.empty_cache()
    plane = torch.empty(n // 2, dtype=torch.uint8, device=device)
    scale = torch.empty(G, dtype=torch.int16, device=device)
    zero = torch.empty(G, dtype=torch.uint8, device=device)
    r = torch.empty(n, dtype=torch.bfloat16, device=device)
    with torch.cuda.stream(stream):
        cq.cqs_code_words(plane.view(torch.int64), 4, 0, stream)
        cq.cqs_scales(scale, 4, 0, stream)
        cq.cqs_zeros(zero, 4, 0, stream)
        cq.cqs_residual_bf16(r, scale, 4, 0, float(synth.ih4_multiplier(0.3)), stream)
        cq.cq_project_residual(r, scale, None, stream)
    torch.cuda.synchronize()
    qw = cq.QWeight(1, n, [None, None, plane, None], scale, zero, residual=r)
    starts = list(range(0, n, chunk))
    cnt = torch.zeros((len(starts), 4), dtype=torch.int64, device=device)

    def run():
        for i, c0 in enumerate(starts):
            nw = min(chunk, n - c0)
            cq.cq_requant_verify_pair(qw, c0, nw, cnt[i, 0:1], cnt[i, 1:2], cnt[i, 2:3], cnt[i, 3:4], None, stream)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            run()
    g.replay()
    ms = time_graph(torch, g, 5, stream)
    c = cnt.cpu()
    assert int(c[:, 0].sum()) == 0 and int(c[:, 2].sum()) == 0, "scale verify: mismatches after projection"
    per_w = 2.5 + 3.0 / GROUP
    res = {"weights": n, "chunks": len(starts), "ms": ms, "weights_per_s": n / (ms * 1e-3),
           "GBps": n * per_w / (ms * 1e-3) / 1e9, "frac_hbm": n * per_w / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del g, plane, scale, zero, r, qw
    torch.cuda.empty_cache()
    return res


def run_gpu(args, rank, world, local_rank):
    import torch
    from cell_updates_b200 import cq, ops, synth
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    peaks = load_peaks()
    cq.lib()
    wl = Workload(torch, cq, ops, synth, device, seed_base=1 + 100000 * rank)
    stream = torch.cuda.Stream(device)
    # eager run, then a one-step graph for the warm-up, a K-step graph for the timed region,
    # and a second K-step graph with an event pair around each row's three launches: it is
    # replayed after the timed region for the per-row breakdown only (event nodes add time of
    # their own, so they stay out of the headline)
    with torch.cuda.stream(stream):
        wl.step(stream)
    torch.cuda.synchronize()
    g1 = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g1, stream=stream):
            wl.step(stream)
    launches_per_step = count_kernel_nodes(g1)
    marks = [{k: (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
              for k in KERNELS} for _ in range(args.steps)]
    gK = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gK, stream=stream):
            for s_i in range(args.steps):
                wl.step(stream)
    gM = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gM, stream=stream):
            for s_i in range(args.steps):
                wl.step(stream, marks[s_i])
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g1.replay()
    # each K-step graph runs once untimed, so its first-launch set-up stays out of the timings
    gK.replay()
    gM.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    # the sampler (100 ms period) sees the clocks under the same load: the K-step graph replayed
    # for ~0.5 s right before the timed region (whose K steps alone last only milliseconds)
    t_load = time.time() + 0.5
    n_load = 0
    while time.time() < t_load:
        gK.replay()
        torch.cuda.synchronize()
        n_load += 1
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        gK.replay()
        end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    clk["window"] = f"the step graph replayed {n_load} x {args.steps} steps (~0.5 s) before and through the timed region"
    t_step = start.elapsed_time(end) / args.steps
    # the per-row breakdown: the same K steps with an event pair around each row
    with torch.cuda.stream(stream):
        start.record(stream)
        gM.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t_marked = start.elapsed_time(end) / args.steps
    # per-step spread: the one-step graph replayed with an event pair around each replay (its
    # graph-launch latency included), reported as median and p10/p90 beside the K-step headline
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    with torch.cuda.stream(stream):
        for a, b in pairs:
            a.record(stream)
            g1.replay()
            b.record(stream)
    torch.cuda.synchronize()
    one = np.array(sorted(a.elapsed_time(b) for a, b in pairs))
    spread = {"replays": len(pairs), "median_ms": float(np.median(one)), "p10_ms": float(np.percentile(one, 10)),
              "p90_ms": float(np.percentile(one, 90)), "graph": "one step per replay"}
    per_kernel = {k: 0.0 for k in KERNELS}           # ms summed over every launch
    for mk in marks:
        for k, (a, b) in mk.items():
            per_kernel[k] += a.elapsed_time(b)
    t_step = max_over_ranks(t_step, dist, device)
    checks = [int(wl.mism.item()), int(wl.mism0.item()), int(wl.status.item())]
    assert all(c == 0 for c in checks), f"hot-path results not clean: {checks}"

    bytes_step = wl.step_bytes()
    total_bytes = sum(bytes_step.values())
    n_w = wl.n_weights()
    value = job_value(total_bytes, world, t_step)            # GB/s over all ranks
    comps = {}
    for k in KERNELS:
        t_k = per_kernel[k] / args.steps                  # ms per step for this kernel
        comps[k] = {"us_per_step": t_k * 1e3, "GBps": bytes_step[k] / (t_k * 1e-3) / 1e9,
                    "frac_hbm": bytes_step[k] / (t_k * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "share": per_kernel[k] / max(sum(per_kernel.values()), 1e-12)}
    # the batch-64 GEMM is a dense contraction: its tensor-core rate against the sustained bf16 peak
    # (the kernel runs inside a long step) and the burst one
    t_gemm = per_kernel["gemm"] / args.steps * 1e-3
    gemm_flops = 2.0 * GEMM_M * wl.n_weights()
    comps["gemm"]["TFLOPs"] = gemm_flops / t_gemm / 1e12
    comps["gemm"]["frac_bf16_sustained"] = comps["gemm"]["TFLOPs"] / peaks["bf16_tflops_sustained"]
    comps["gemm"]["frac_bf16_burst"] = comps["gemm"]["TFLOPs"] / peaks["bf16_tflops"]
    dominant = max(KERNELS, key=lambda k: per_kernel[k])
    achieved = comps[dominant]["GBps"]
    roofline = {"kernel": dominant, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": MEASURED_TRAFFIC.get(dominant),
                "peak_source": peaks["source"],
                "algorithmic_bytes_per_launch": bytes_step[dominant] / launches_of(dominant, wl),
                "launches_timed": args.steps * launches_of(dominant, wl)}
    iso = isolated_components(torch, cq, ops, device, peaks, stream) if args.components else None

    # end to end: pinned host inputs -> device, the step, results -> host
    e2e = run_e2e(torch, wl, g1, stream, args.steps)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, device)
    e2e_value = job_value(total_bytes, world, e2e["ms_per_step"])

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step, "ms_per_step_with_event_nodes": t_marked,
            "step_spread": spread,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u4 codes / fp32 quantize / bf16 x, fp32 accumulate",
            "data": "synthetic (seeded Student-t weights, N(0,1) activations, N(0,(0.3s)^2) bf16 residuals)",
            "config": {"workload": WORKLOAD, "weights_per_step": n_w, "gemv_batch": 1, "gemm_batch": GEMM_M,
                       "residual": "bf16", "l2": "inputs larger than L2 (377 MB fp32 weights per step)",
                       "parallelism": f"replicas x{world}", "step": "+".join(KERNELS),
                       "value_is": "composite: the algorithmic bytes of all six rows of one step over the step "
                                   "time; the metric's own parts are the top-level dequant_gemv_*, tokens_per_s "
                                   "and requant_verify_* keys"},
            "roofline": roofline,
            # weights checked per second by the pass that checks both (with r, and revoked)
            "requant_verify_weights_per_s": n_w / (per_kernel["verify_pair"] / args.steps * 1e-3),
            "dequant_gemv_GBps_in_step": comps["gemv"]["GBps"],
            "components": comps,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                    "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["ms_per_step"]},
            "gpu_launches": launches_per_step * args.steps if launches_per_step is not None else None,
            "clocks": clk,
        }
        if iso:
            line["isolated"] = iso
            line["tokens_per_s"] = iso["decode_32_layers"]["tokens_per_s"]
            line["tokens_per_s_frac_of_ceiling"] = (iso["decode_32_layers"]["tokens_per_s"] /
                                                    iso["decode_32_layers"]["ceiling_tokens_per_s"])
            line["dequant_gemv_GBps_cold"] = {k: v["GBps"] for k, v in iso["gemv_m1_cold"].items()}
            served = iso["cellfill_stack"].get("decode_28_layers_served")
            if served:
                line["tokens_per_s_cellfill_served"] = served["tokens_per_s"]
            line["requant_verify_weights_per_s_cellfill_stack"] = iso["cellfill_stack"]["verify"]["weights_per_s"]
            line["requant_verify_weights_per_s_2_4e10"] = iso["scale_verify_2_4e10"]["weights_per_s"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_sample_rows)
    if dist:
        g1.reset()
        gK.reset()
        dist.barrier()
        dist.destroy_process_group()
    return line


def run_e2e(torch, wl, graph, stream, steps):
    """Same step with host buffers: H2D of W, r, x, X before and D2H of y, Y and the counters after."""
    h2d = wl.w_host.numel() * 4 + wl.r_host.numel() * 2
    d2h = 2 * 8 + 4
    for m in wl.mats:
        h2d += sum(t.numel() * t.element_size() for t in (m["x_host"], m["X_host"]))
        d2h += m["y"].numel() * 4 + m["Y"].numel() * 4
    outs = [{k: torch.empty_like(m[k], device="cpu").pin_memory() for k in ("y", "Y")} for m in wl.mats]
    counters = {k: torch.empty_like(getattr(wl, k), device="cpu").pin_memory() for k in ("mism", "mism0", "status")}
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(steps):
            wl.w.copy_(wl.w_host, non_blocking=True)
            wl.r.copy_(wl.r_host, non_blocking=True)
            for m in wl.mats:
                m["x"].copy_(m["x_host"], non_blocking=True)
                m["X"].copy_(m["X_host"], non_blocking=True)
            graph.replay()
            for m, o in zip(wl.mats, outs):
                for k in o:
                    o[k].copy_(m[k], non_blocking=True)
            for k, t in counters.items():
                t.copy_(getattr(wl, k), non_blocking=True)
        b.record(stream)
    torch.cuda.synchronize()
    return {"ms_per_step": a.elapsed_time(b) / steps, "h2d": h2d, "d2h": d2h}


# ---------------------------------------------------------------------------------------
# the CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------------------
_SAMPLE_CACHE = {}


def _sample_inputs(rows_per_matrix):
    """Inputs of the CPU sample (built once, not timed): the first rows of each matrix."""
    if rows_per_matrix in _SAMPLE_CACHE:
        return _SAMPLE_CACHE[rows_per_matrix]
    from cell_updates_b200 import synth
    from oracle import c_oracle as co
    out = []
    for idx, (N, K) in enumerate(SHAPES):
        rows = min(rows_per_matrix, N)
        w = np.ascontiguousarray(synth.student_t_weights(N, K, seed=1 + 1000 * idx)[:rows])
        _, scale, _, _ = co.quantize(w)
        r = synth.normal_residual_bf16(scale, seed=1 + 1000 * idx + 7, rel_sigma=0.3)
        x = synth.activations(1, K, seed=1 + 1000 * idx + 11, dtype="bf16")
        X = synth.activations(GEMM_M, K, seed=1 + 1000 * idx + 13, dtype="bf16")
        out.append((rows, K, w, r, x, X))
    _SAMPLE_CACHE[rows_per_matrix] = out
    return out


def cpu_sample(rows_per_matrix, threads=None):
    """The same step on a row sample of each matrix, on the host cores (all of them unless
    `threads` is given), with the oracle."""
    from oracle import c_oracle as co
    threads = threads or co.default_threads()
    inputs = _sample_inputs(rows_per_matrix)
    nbytes = n_w = 0
    t0 = time.perf_counter()
    for rows, K, w, r, x, X in inputs:
        codes, scale, zero, st = co.quantize(w, nthreads=threads)
        planes = co.pack(codes)
        rp, _ = co.project_bf16(r, scale)
        co.verify(planes, scale, zero, r=rp, r_dtype="bf16", nthreads=threads)
        co.verify(planes, scale, zero, nthreads=threads)
        co.dequant_matmul_f64(planes, scale, zero, rows, K, x, "bf16", nthreads=threads)
        co.dequant_matmul_f64(planes, scale, zero, rows, K, X, "bf16", nthreads=threads)
        n = rows * K
        n_w += n
        nbytes += sum(kernel_bytes(n).values())
    dt = time.perf_counter() - t0
    return nbytes, n_w, dt, threads


def cpu_baseline(rows, min_seconds=10.0):
    """The oracle as it stands, repeated on the row sample until ~min_seconds of CPU work."""
    nbytes = n_w = 0
    dt = 0.0
    reps = 0
    while dt < min_seconds:
        b, n, t, threads = cpu_sample(rows)
        nbytes, n_w, dt, reps = nbytes + b, n_w + n, dt + t, reps + 1
    # the same oracle on one thread, on a quarter of the row sample (one pass)
    rows1 = max(64, rows // 4)
    b1, n1, t1, _ = cpu_sample(rows1, threads=1)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {rows} rows of each of the 3 matrices ({n_w // reps} weights), the whole step, "
                      f"repeated {reps}x ({dt:.1f} s)",
            "seconds": dt,
            "single_thread": {"value": b1 / t1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"first {rows1} rows of each of the 3 matrices ({n1} weights), the whole "
                                        f"step, once ({t1:.1f} s)"}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    t_all = []
    warm = max(0, args.warmup)
    for i in range(warm + args.steps):
        nbytes, n_w, dt, threads = cpu_sample(args.cpu_sample_rows)
        if i >= warm:
            t_all.append(dt)
    ms = float(np.mean(t_all)) * 1e3
    value = nbytes / (ms * 1e-3) / 1e9
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp32 / fp64 (CPU oracle)", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_rows_per_matrix": args.cpu_sample_rows,
                       "weights_per_step": n_w, "step": "+".join(KERNELS)},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"first {args.cpu_sample_rows} rows of each matrix ({n_w} weights)"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_case(kernel, reps=3):
    """Run one libcq kernel `reps` times on an input larger than the L2 cache, for ncu captures
    (`ncu -k regex:<kernel name> -s <set-up launches + warm-up> -c 1 python bench.py --case
    <case>`). Cases: gemv (16384x16384, m=1), gemv8 (same, m=8), gemm (8192x28672, m=64),
    quantize, pack, project, verify (projected bf16 residual), revoke (no residual), pair (both
    checks), rrq (one 2-bit residual stage), stages / stages8 (the stage-stack GEMV over four
    2-bit stages, m=1 / m=8), vbq / vbq8 (the GEMV of a matrix of per-group widths drawn as in
    the VBQ configuration, m=1 / m=8), vpack / vunpack / vindex (pack, unpack and the offset
    index of the VBQ configuration's 2048x8192 width map), gemvr (the GEMV with a projected bf16
    residual, m=1), reparam / reparam_grad (the bounded reparameterization, bf16 residual, and its
    backward pass); the others on 8192x16384. Each is
    preceded by its set-up launches (random weights, quantize, pack)."""
    import torch
    from cell_updates_b200 import build, cq, ops, synth
    from types import SimpleNamespace
    a = SimpleNamespace(kernel=kernel, reps=reps)
    build.build()
    dev = torch.device("cuda")
    torch.manual_seed(0)
    N, K, m = {"gemv": (16384, 16384, 1), "gemv8": (16384, 16384, 8), "gemm": (8192, 28672, 64),
               "stages8": (8192, 16384, 8), "vbq8": (8192, 16384, 8), "vpack": (2048, 8192, 1),
               "vunpack": (2048, 8192, 1), "vindex": (2048, 8192, 1)}.get(a.kernel, (8192, 16384, 1))
    w = torch.randn(N, K, device=dev) * 0.02
    bits = None
    if a.kernel in ("vbq", "vbq8", "vpack", "vunpack", "vindex"):
        bits = torch.from_numpy(synth.vbq_bits(N * K // 64, seed=2)).to(dev)
    qw, codes, _ = ops.quantize_and_pack(w, bits)
    x = torch.randn(m, K, device=dev).to(torch.bfloat16)
    y = torch.empty(m, N, device=dev)
    ws = torch.empty(max(16, cq.cq_gemm_workspace(N, K, m)), dtype=torch.uint8, device=dev)
    r = (torch.randn(N * K, device=dev) * 1e-3).to(torch.bfloat16)
    mism = torch.empty(1, dtype=torch.int64, device=dev)
    first = torch.empty(1, dtype=torch.int64, device=dev)
    scale, zero = qw.scale, qw.zero
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if a.kernel in ("verify", "pair"):
        cq.cq_project_residual(r, scale, None)     # a residual inside its cells, as after an update
    stages = None
    if a.kernel in ("stages", "stages8"):
        stages, _, _ = ops.rrq_build(w, 4)
    if a.kernel == "rrq":
        rr = w.clone()
    if a.kernel in ("gemvr", "reparam", "reparam_grad"):
        r = (torch.randn(N * K, device=dev) * 1e-3).to(torch.bfloat16)
        cq.cq_project_residual(r, scale, None)     # served weights with a residual inside its cells
        theta = torch.randn(N * K, device=dev) * 2.0
        g_theta = torch.empty_like(theta) if a.kernel == "reparam_grad" else None
    if a.kernel in ("gemv", "gemv8", "gemm", "vbq", "vbq8", "gemvr"):
        del w                                      # keep the device footprint small under the profiler
        if a.kernel != "gemvr":
            del r
        torch.cuda.empty_cache()
    torch.cuda.synchronize()
    for _ in range(a.reps):
        if a.kernel in ("gemv", "gemv8", "vbq", "vbq8"):
            cq.cq_dequant_gemv(qw, x, y)
        elif a.kernel == "gemm":
            cq.cq_dequant_gemm(qw, x, y, ws)
        elif a.kernel == "quantize":
            cq.cq_quantize(w, None, codes, scale, zero, st)
        elif a.kernel == "pack":
            cq.cq_pack_varbits(codes, N * K // 64, None, None, qw.planes)
        elif a.kernel == "project":
            cq.cq_project_residual(r, scale, None)
        elif a.kernel == "verify":
            cq.cq_requant_verify(qw.with_residual(r), 0, N * K, mism, first)
        elif a.kernel == "revoke":
            cq.cq_requant_verify(qw, 0, N * K, mism, first)
        elif a.kernel == "pair":
            m0 = torch.empty(1, dtype=torch.int64, device=dev)
            f0 = torch.empty(1, dtype=torch.int64, device=dev)
            cq.cq_requant_verify_pair(qw.with_residual(r), 0, N * K, mism, first, m0, f0)
        elif a.kernel == "rrq":
            cq.cq_rrq_stage(rr, 2, codes, scale, zero, st)
        elif a.kernel == "vpack":
            cq.cq_pack_varbits(codes, N * K // 64, bits, qw.offset, qw.planes)
        elif a.kernel == "vunpack":
            cq.cq_unpack_varbits(qw, codes)
        elif a.kernel == "vindex":
            cq.cq_varbits_index(bits, qw.offset, torch.empty(4, dtype=torch.int64, device=dev))
        elif a.kernel in ("stages", "stages8"):
            cq.cq_dequant_gemv_stages(stages, x, y)
        elif a.kernel == "gemvr":
            cq.cq_dequant_gemv(qw.with_residual(r), x, y)
        elif a.kernel == "reparam":
            cq.cq_reparam_residual(theta, scale, r)
        elif a.kernel == "reparam_grad":
            cq.cq_reparam_residual_grad(theta, scale, theta, g_theta, cq.CQ_BF16)
        else:
            raise SystemExit(f"unknown kernel {a.kernel}")
    torch.cuda.synchronize()
    print("ok", a.kernel, N, K, m)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cq", choices=["cq", "reference"])
    ap.add_argument("--cpu-sample-rows", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-components", dest="components", action="store_false")
    ap.add_argument("--case", default=None, help="run one kernel for an ncu capture (see profile_case) and exit")
    ap.add_argument("--reps", type=int, default=3, help="launches of the --case kernel")
    args = ap.parse_args()
    if args.case:
        profile_case(args.case, args.reps)
        return
    args.warmup = max(args.warmup, 3) if args.impl == "cq" else args.warmup
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", args.gpus if args.gpus == 1 else 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_gpu(args, rank, world, local_rank)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
