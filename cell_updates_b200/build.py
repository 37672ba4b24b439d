"""Build the native libraries in-tree for sm_100a.

* ``libcq.so``       -- the quantizer's CUDA kernels behind the C ABI of include/cq.h;
* ``libcq_synth.so`` -- seeded device-side test inputs (include/cq_synth.h).

Each translation unit is compiled separately so the IEEE-exact kernels (quantize,
projection, verify) get ``-fmad=false`` on top of their explicit round-to-nearest
intrinsics, while the matmul kernels keep fused multiply-adds.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-prec-div=true", "-prec-sqrt=true", "-ftz=false", *ARCH]
EXACT = ["-fmad=false"]

LIBCQ_UNITS = {
    "cq_api.cu": [],
    "k_quantize.cu": EXACT,
    "k_pack.cu": EXACT,
    "k_project.cu": EXACT,
    "k_verify.cu": EXACT,
    "k_gemv.cu": [],
    "k_gemm.cu": [],
    "k_rrq.cu": [],
}
SYNTH_UNITS = {"synth.cu": EXACT}

LIBCQ = os.path.join(HERE, "libcq.so")
LIBSYNTH = os.path.join(HERE, "libcq_synth.so")
HEADERS = [os.path.join(CSRC, "cq_internal.cuh"), os.path.join(HERE, "..", "include", "cq.h"),
           os.path.join(HERE, "..", "include", "cq_synth.h")]


def _newer(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _compile(unit, extra, verbose):
    src = os.path.join(CSRC, unit)
    obj = os.path.join(BUILD, unit.replace(".cu", ".o"))
    if _newer(obj, [src, *HEADERS, __file__]):
        cmd = [NVCC, *COMMON, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
    return obj


def _link(objs, out, verbose):
    if _newer(out, objs):
        tmp = out + ".tmp"
        cmd = [NVCC, "-shared", *ARCH, "-o", tmp, *objs, "-lcudart_static", "-lrt", "-lpthread", "-ldl"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, out)


def build(verbose: bool = False) -> None:
    os.makedirs(BUILD, exist_ok=True)
    _link([_compile(u, f, verbose) for u, f in LIBCQ_UNITS.items()], LIBCQ, verbose)
    _link([_compile(u, f, verbose) for u, f in SYNTH_UNITS.items()], LIBSYNTH, verbose)


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
