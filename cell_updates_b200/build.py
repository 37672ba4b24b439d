"""Build the native libraries in-tree for sm_100a.

* ``libcq.so``       -- the quantizer's CUDA kernels behind the C ABI of include/cq.h;
* ``libcq_synth.so`` -- seeded device-side test inputs (include/cq_synth.h).

Each translation unit is compiled separately so the IEEE-exact kernels (quantize,
projection, verify, reparameterization) get ``-fmad=false`` on top of their explicit round-to-nearest
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
    "k_reparam.cu": EXACT,
    "k_requant.cu": EXACT,
}
SYNTH_UNITS = {"synth.cu": EXACT}

# test-only builds of libcq with a fault injected on the host side of a kernel's pipeline (a copy
# that is never requested, so a bounded wait runs out and the abort path runs); the tests load
# them by path, nothing else does
TEST_VARIANTS = {"drop_first_copy": {"k_quantize.cu": ["-DCQ_TEST_DROP_FIRST_COPY"],
                                      "k_gemm.cu": ["-DCQ_TEST_DROP_FIRST_COPY"]},
                 # every unit with its in-kernel index checks compiled in (cq_debug.cuh)
                 "debug": {u: ["-DCQ_DEBUG"] for u in LIBCQ_UNITS}}

LIBCQ = os.path.join(HERE, "libcq.so")
LIBSYNTH = os.path.join(HERE, "libcq_synth.so")
HEADERS = [*(os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cuh")),
           os.path.join(HERE, "..", "include", "cq.h"), os.path.join(HERE, "..", "include", "cq_synth.h")]


def _newer(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def test_variant_path(name):
    return os.path.join(BUILD, f"libcq_{name}.so")


def _compile(unit, extra, verbose, tag=""):
    src = os.path.join(CSRC, unit)
    obj = os.path.join(BUILD, unit.replace(".cu", f"{tag}.o"))
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
    for name, units in TEST_VARIANTS.items():
        objs = [_compile(u, f + units.get(u, []), verbose, tag=f"_{name}" if u in units else "")
                for u, f in LIBCQ_UNITS.items()]
        _link(objs, test_variant_path(name), verbose)


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
