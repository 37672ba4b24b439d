"""Guard bands around every output of every entry point (compute-sanitizer is not available
here, so this stands in for its out-of-bounds-write check): each output buffer sits between
4 KiB of sentinel bytes, the calls run on ragged shapes (partial tiles, partial chunks, group
counts that are not multiples of the kernels' blocking), and the sentinels must be intact
afterwards. The values themselves are checked by the parity tests; here a few are compared
with the unguarded path to make sure the call did its work."""
import numpy as np
import pytest
import torch

from cell_updates_b200 import build, cq, ops, synth
from gpu_util import Guarded, bf16_dev, dev, host

pytestmark = pytest.mark.gpu

GROUP = 64


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    build.build()


def _weights(rows, cols, seed):
    return dev(synth.normal_weights(rows, cols, seed=seed))


@pytest.mark.parametrize("rows,cols", [(47, 64 * 9), (5, 64), (300, 64 * 21)])
def test_guards_quantize_pack_index_unpack(rows, cols):
    w = _weights(rows, cols, rows)
    G = rows * cols // GROUP
    codes = Guarded(rows * cols, torch.uint8)
    scale = Guarded(G, torch.int16)
    zero = Guarded(G, torch.uint8)
    st = Guarded(1, torch.int32)
    cq.cq_quantize(w, None, codes.t, scale.t, zero.t, st.t)
    for b, n in ((codes, "codes"), (scale, "scale"), (zero, "zero"), (st, "status")):
        b.check(f"quantize {n}")
    ref_codes, ref_scale, _, _ = ops.quantize(w)
    assert torch.equal(codes.t, ref_codes) and torch.equal(scale.t, ref_scale)
    # fixed 4-bit pack and unpack
    plane = Guarded(G * 32, torch.uint8)
    cq.cq_pack_varbits(codes.t, G, None, None, [None, None, plane.t, None])
    plane.check("pack fixed-4")
    back = Guarded(rows * cols, torch.uint8)
    cq.cq_unpack_varbits(cq.QWeight(rows, cols, [None, None, plane.t, None], scale.t, zero.t), back.t)
    back.check("unpack fixed-4")
    assert torch.equal(back.t, codes.t)
    # per-group widths: index, quantize, pack, unpack
    bits = torch.from_numpy(synth.vbq_bits(G, seed=rows + 1)).cuda()
    off = Guarded(G, torch.int32)
    pb = Guarded(4, torch.int64)
    cq.cq_varbits_index(bits, off.t, pb.t)
    off.check("index offsets")
    pb.check("index plane bytes")
    sizes = [int(v) for v in host(pb.t)]
    vcodes = Guarded(rows * cols, torch.uint8)
    cq.cq_quantize(w, bits, vcodes.t, scale.t, zero.t, st.t)
    vcodes.check("quantize widths")
    planes = [Guarded(max(16, n), torch.uint8) for n in sizes]
    cq.cq_pack_varbits(vcodes.t, G, bits, off.t, [p.t for p in planes])
    for i, p in enumerate(planes):
        p.check(f"pack plane {i}")
    vback = Guarded(rows * cols, torch.uint8)
    qv = cq.QWeight(rows, cols, [p.t for p in planes], scale.t, zero.t, bits, off.t)
    cq.cq_unpack_varbits(qv, vback.t)
    vback.check("unpack widths")
    assert torch.equal(vback.t, vcodes.t)


@pytest.mark.parametrize("rows,cols", [(47, 64 * 9), (300, 64 * 21)])
def test_guards_project_verify_reparam(rows, cols):
    qw, _, _ = ops.quantize_and_pack(_weights(rows, cols, 7))
    n = rows * cols
    G = n // GROUP
    scale = host(qw.scale, np.uint16)
    rb = synth.normal_residual_bf16(scale, seed=8, rel_sigma=0.6)
    r = Guarded(n, torch.bfloat16, fill=bf16_dev(rb))
    ncl = Guarded(1, torch.int64)
    cq.cq_project_residual(r.t, qw.scale, ncl.t)
    r.check("project r")
    ncl.check("project count")
    assert int(host(ncl.t)[0]) > 0
    outs = [Guarded(1, torch.int64) for _ in range(4)]
    flags = Guarded((G + 31) // 32, torch.int32)
    cq.cq_requant_verify(qw.with_residual(r.t), 0, n, outs[0].t, outs[1].t, flags.t)
    for o in outs[:2] + [flags]:
        o.check("verify")
    assert int(host(outs[0].t)[0]) == 0
    cq.cq_requant_verify_pair(qw.with_residual(r.t), 0, n, outs[0].t, outs[1].t, outs[2].t, outs[3].t, flags.t)
    for o in outs + [flags]:
        o.check("verify pair")
    theta = dev(np.random.default_rng(9).standard_normal(n).astype(np.float32) * 3)
    for dtype in (torch.bfloat16, torch.float32):
        rr = Guarded(n, dtype)
        cq.cq_reparam_residual(theta, qw.scale, rr.t)
        rr.check(f"reparam {dtype}")
        g = Guarded(n, torch.float32)
        cq.cq_reparam_residual_grad(theta, qw.scale, theta, g.t, cq.CQ_BF16 if dtype == torch.bfloat16 else cq.CQ_F32)
        g.check(f"reparam grad {dtype}")


@pytest.mark.parametrize("rows,cols,m", [(47, 64 * 9, 3), (300, 64 * 21, 8), (17, 64 * 4, 1)])
def test_guards_gemv(rows, cols, m):
    qw, _, _ = ops.quantize_and_pack(_weights(rows, cols, 11))
    x = bf16_dev(synth.activations(m, cols, seed=12, dtype="bf16"))
    y = Guarded(m * rows, torch.float32)
    cq.cq_dequant_gemv(qw, x, y.t)
    y.check("gemv")
    assert torch.allclose(y.t.view(m, rows), ops.gemv(qw, x))
    # with a bf16 residual (CellFill served weights)
    scale = host(qw.scale, np.uint16)
    r = bf16_dev(synth.normal_residual_bf16(scale, seed=13, rel_sigma=0.3))
    yr = Guarded(m * rows, torch.float32)
    cq.cq_dequant_gemv(qw.with_residual(r), x, yr.t)
    yr.check("gemv residual")
    # several matrices sharing x
    qw2, _, _ = ops.quantize_and_pack(_weights(rows + 5, cols, 14))
    ys = [Guarded(m * rows, torch.float32), Guarded(m * (rows + 5), torch.float32)]
    cq.cq_dequant_gemv_multi([qw, qw2], x, [g.t for g in ys])
    for g in ys:
        g.check("gemv multi")
    # per-group widths, and a stack of recurrent-residual stages
    G = rows * cols // GROUP
    bits = torch.from_numpy(synth.vbq_bits(G, seed=15)).cuda()
    qv, _, _ = ops.quantize_and_pack(_weights(rows, cols, 16), bits)
    yv = Guarded(m * rows, torch.float32)
    cq.cq_dequant_gemv(qv, x, yv.t)
    yv.check("gemv widths")
    stages, _, _ = ops.rrq_build(_weights(rows, cols, 17), 3)
    ysg = Guarded(m * rows, torch.float32)
    cq.cq_dequant_gemv_stages(stages, x, ysg.t)
    ysg.check("gemv stages")


@pytest.mark.parametrize("rows,cols,m", [(300, 64 * 24, 40), (129, 64 * 8, 16), (200, 64 * 7, 17)])
def test_guards_gemm_and_rrq(rows, cols, m):
    qw, _, _ = ops.quantize_and_pack(_weights(rows, cols, 21))
    x = bf16_dev(synth.activations(m, cols, seed=22, dtype="bf16"))
    y = Guarded(m * rows, torch.float32)
    need = cq.cq_gemm_workspace(rows, cols, m)
    ws = Guarded(max(need, 16), torch.uint8)
    cq.cq_dequant_gemm(qw, x, y.t, ws.t if need else None)
    y.check("gemm y")
    ws.check("gemm workspace")
    ys = Guarded(m * rows, torch.float32)
    st = Guarded(1, torch.int32)
    cq.cq_dequant_gemm_static(qw, x, ys.t, st.t)
    ys.check("gemm static y")
    st.check("gemm static status")
    r = Guarded(rows * cols, torch.float32, fill=_weights(rows, cols, 23))
    G = rows * cols // GROUP
    codes, scale, zero, status = (Guarded(rows * cols, torch.uint8), Guarded(G, torch.int16),
                                  Guarded(G, torch.uint8), Guarded(1, torch.int32))
    cq.cq_rrq_stage(r.t.view(rows, cols), 2, codes.t, scale.t, zero.t, status.t)
    for b, nme in ((r, "r"), (codes, "codes"), (scale, "scale"), (zero, "zero"), (status, "status")):
        b.check(f"rrq stage {nme}")
