"""Recurrent residual quantization on the GPU against the oracle.

Bit-exact: every stage's codes, scales, zero points, status word and the residual it leaves
(fp32 bit patterns), over several stages, on shapes with ragged 32-group tiles and with a
planted non-finite group. Tolerance (benchmark spec: relative Frobenius error <= 2e-3,
per-element |err| <= 1e-2 rms(y)): the stage-stack GEMV against the fp64 sum of the oracle's
stages, for 1 to 4 two-bit stages and for a mixed list (fixed-4, 2-bit, per-group widths).
"""
import numpy as np
import pytest
import torch

from cell_updates_b200 import cq, ops, synth
from gpu_util import bf16_dev, check_matmul, dev, host
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from cell_updates_b200 import build
    build.build()
    cq.lib()


def _gpu_stage(r_d, bits=2):
    rows, cols = r_d.shape
    G = rows * cols // 64
    codes = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    scale = torch.empty(G, dtype=torch.int16, device="cuda")
    zero = torch.empty(G, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cq.cq_rrq_stage(r_d, bits, codes, scale, zero, status)
    return codes, scale, zero, status


@pytest.mark.parametrize("rows,cols", [(64, 512), (37, 64 * 9), (300, 64 * 21), (1000, 4096)])
def test_rrq_stages_bit_exact(rows, cols):
    w = synth.student_t_weights(rows, cols, seed=rows + cols)
    w[rows // 2, 70 % cols] = np.nan                     # a flagged group keeps its residual
    r_d = dev(w.copy())
    r_h = w.copy()
    for j in range(4):
        codes, scale, zero, status = _gpu_stage(r_d)
        oc, os_, oz, ost, r_h = co.rrq_stage(r_h, 2)
        torch.cuda.synchronize()
        assert np.array_equal(host(codes), oc), f"stage {j}: codes"
        assert np.array_equal(host(scale, np.uint16), os_), f"stage {j}: scales"
        assert np.array_equal(host(zero), oz), f"stage {j}: zeros"
        assert int(host(status)[0]) == ost == 1, f"stage {j}: status"
        assert np.array_equal(host(r_d).view(np.uint32), r_h.view(np.uint32)), f"stage {j}: residual bits"


@pytest.mark.parametrize("width", [1, 4, 8])
def test_rrq_stage_other_widths(width):
    w = synth.normal_weights(96, 64 * 12, seed=width)
    r_d = dev(w.copy())
    codes, scale, zero, status = _gpu_stage(r_d, width)
    oc, os_, oz, ost, r_h = co.rrq_stage(w, width)
    assert np.array_equal(host(codes), oc) and np.array_equal(host(scale, np.uint16), os_)
    assert np.array_equal(host(zero), oz) and int(host(status)[0]) == ost
    assert np.array_equal(host(r_d).view(np.uint32), r_h.view(np.uint32))


def _oracle_stack(w, n_stages):
    """the oracle's stages and the fp64 matmul of their sum, as a function of x"""
    stages, _ = co.rrq_build(w, n_stages, 2)
    G = w.size // 64
    bits = np.full(G, 2, np.uint8)
    off, pb = co.varbits_index(bits)
    packed = [(co.pack(c, bits, off, pb), s, z) for c, s, z, _ in stages]
    rows, cols = w.shape

    def matmul(x, x_dtype):
        return sum(co.dequant_matmul_f64(pl, s, z, rows, cols, x, x_dtype, bits, off) for pl, s, z in packed)
    return matmul


@pytest.mark.parametrize("rows,cols,n_stages", [(256, 512, 1), (333, 64 * 21, 2), (1000, 4096, 3), (512, 2048, 4),
                                                 (96, 1024, 6), (40, 64 * 200, 3)])
@pytest.mark.parametrize("m,x_dtype", [(1, "bf16"), (3, "f32"), (8, "bf16")])
def test_rrq_gemv_stages(rows, cols, n_stages, m, x_dtype):
    w = synth.normal_weights(rows, cols, seed=7 * rows + n_stages)
    stages, statuses, _ = ops.rrq_build(dev(w), n_stages)
    assert all(int(host(s)[0]) == 0 for s in statuses)
    matmul = _oracle_stack(w, n_stages)
    x = synth.activations(m, cols, seed=rows + m, dtype=x_dtype)
    x_d = bf16_dev(x) if x_dtype == "bf16" else dev(x)
    y = host(ops.gemv_stages(stages, x_d))
    check_matmul(y, matmul(x, x_dtype), f"rrq {rows}x{cols} stages={n_stages} m={m} {x_dtype}")


def test_rrq_gemv_stages_long_rows():
    """fp32 activations too long to stage in shared memory at batch 1 (read from L1 instead)."""
    rows, cols = 24, 64 * 640
    w = synth.normal_weights(rows, cols, seed=21)
    stages, _, _ = ops.rrq_build(dev(w), 2)
    matmul = _oracle_stack(w, 2)
    x = synth.activations(1, cols, seed=22, dtype="f32")
    check_matmul(host(ops.gemv_stages(stages, dev(x))), matmul(x, "f32"), "rrq long rows f32")


def test_rrq_more_stages_approach_the_weights():
    """The stack's product approaches the unquantized weights' product stage by stage
    (each 2-bit stage shrinks the residual about threefold)."""
    rows, cols, m = 512, 4096, 4
    w = synth.normal_weights(rows, cols, seed=5)
    x = synth.activations(m, cols, seed=6, dtype="f32")
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    stages, _, _ = ops.rrq_build(dev(w), 4)
    errs = []
    for n in range(1, 5):
        y = host(ops.gemv_stages(stages[:n], dev(x))).astype(np.float64)
        errs.append(np.linalg.norm(y - exact) / np.linalg.norm(exact))
    assert all(errs[i + 1] < errs[i] / 2 for i in range(3)), errs


def test_rrq_gemv_mixed_stage_formats():
    """A stack whose stages are a fixed 4-bit release, a 2-bit stage and per-group widths."""
    rows, cols, m = 200, 64 * 16, 2
    G = rows * cols // 64
    w = synth.normal_weights(rows, cols, seed=11)
    qw4, _, _ = ops.quantize_and_pack(dev(w))
    oc = co.quantize(w)
    planes4 = co.pack(oc[0])
    r = w - (synth.f16_bits_to_f32(oc[1])[:, None] *
             (oc[0].reshape(G, 64).astype(np.float32) - oc[2][:, None])).reshape(rows, cols)
    r = r.astype(np.float32)
    vb = synth.vbq_bits(G, seed=12)
    qv, _, _ = ops.quantize_and_pack(dev(r), dev(vb))
    ovc = co.quantize(r, vb)
    off, pb = co.varbits_index(vb)
    planes_v = co.pack(ovc[0], vb, off, pb)
    two, _, _ = ops.rrq_build(dev(r), 1)
    matmul2 = _oracle_stack(r, 1)
    x = synth.activations(m, cols, seed=13, dtype="bf16")
    ref = (co.dequant_matmul_f64(planes4, oc[1], oc[2], rows, cols, x, "bf16") +
           co.dequant_matmul_f64(planes_v, ovc[1], ovc[2], rows, cols, x, "bf16", vb, off) + matmul2(x, "bf16"))
    y = host(ops.gemv_stages([qw4, qv, two[0]], bf16_dev(x)))
    check_matmul(y, ref, "mixed stages")
