"""Run one libcq kernel a few times on an input larger than the L2 cache, for ncu captures.

    python -m cell_updates_b200.profile_case <kernel> [--reps 3]

kernels: gemv (16384x16384, m=1), gemv8 (same, m=8), gemm (8192x28672, m=64), quantize,
pack, project, verify (projected bf16 residual), revoke (no residual), pair (both checks),
rrq (one 2-bit residual stage), stages / stages8 (the stage-stack GEMV over 4 two-bit stages,
m=1 / m=8), vbq / vbq8 (the GEMV of a matrix of per-group widths drawn as in the VBQ
configuration, m=1 / m=8), vpack / vunpack / vindex (pack, unpack and the offset index of the
VBQ configuration's 2048x8192 width map) -- all but the first three and the last three on
8192x16384.
Each is preceded by the set-up launches (random weights, quantize, pack); capture the
measured kernel with `ncu -k regex:<name> -s <set-up launches + warm-up> -c 1`.
"""
import argparse

import torch

from . import build, cq, ops, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel")
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
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
    if a.kernel in ("gemv", "gemv8", "gemm", "vbq", "vbq8"):
        del w, r                                   # keep the device footprint small under the profiler
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
        else:
            raise SystemExit(f"unknown kernel {a.kernel}")
    torch.cuda.synchronize()
    print("ok", a.kernel, N, K, m)


if __name__ == "__main__":
    main()
