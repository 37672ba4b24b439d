"""bench.py's byte accounting and CPU-baseline line, on the CPU.

Every GB/s figure and roofline fraction the bench prints divides the algorithmic bytes of a
kernel by its time. The per-weight figures follow from the formats alone (groups of 64, a fp16
scale and a u8 zero point per group, u8 codes before packing, 4-bit plane after it, bf16
residuals), so they are restated here from those sizes, independently of bench.py's table.
"""
import os
import sys

from fractions import Fraction

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

GROUP = 64
FP32, BF16, FP16, U8 = 4, 2, 2, 1
META = Fraction(FP16 + U8, GROUP)           # scale + zero point, per weight
NIBBLE = Fraction(1, 2)                     # one 4-bit code


def test_kernel_bytes_per_weight():
    n = 64 * 1000
    expected = {
        "quantize": FP32 + U8 + META,               # read fp32 w, write u8 code and metadata
        "pack": U8 + NIBBLE,                        # read u8 code, write a nibble
        "project": 2 * BF16 + Fraction(FP16, GROUP),  # read and write bf16 r, read the scale
        "verify_pair": NIBBLE + META + BF16,        # plane, metadata, bf16 r (revocation rides along)
        "gemv": NIBBLE + META,                      # the weights; x and y are negligible
        "gemm": NIBBLE + META,
    }
    got = bench.kernel_bytes(n)
    assert set(got) == set(expected) == set(bench.KERNELS)
    for k, per_w in expected.items():
        assert Fraction(got[k], n) == per_w, k


def test_roofline_traffic_is_plausible():
    # a recorded DRAM figure is per launch of the dominant kernel (one launch per step over the
    # three matrices' flat artifact): within its algorithmic bytes (outputs may still sit in L2,
    # so it can be lower, never far above)
    n_step = sum(r * c for r, c in bench.SHAPES)
    per_launch = bench.kernel_bytes(n_step)["quantize"]
    for k, t in bench.MEASURED_TRAFFIC.items():
        assert k in bench.KERNELS
        assert 0.5 * per_launch < t < 1.1 * per_launch, (k, t, per_launch)


def test_cpu_baseline_line():
    r = bench.cpu_baseline(64, min_seconds=0.2)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0 and r["cores"] >= 1
    st = r["single_thread"]
    assert st["cores"] == 1 and st["unit"] == "GB/s" and st["value"] > 0
