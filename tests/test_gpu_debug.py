"""The debug build: in-kernel index checks that record a site number instead of trapping.

cell_updates_b200/_build/libcq_debug.so is libcq compiled with -DCQ_DEBUG (built by build.py,
loaded only here): the kernels check their derived indices (output rows and columns, shared-
and tensor-memory slots, the pipeline's group and tile cursors) and the indices they take from
data (a packed offset must sit on its 8 b grid, and its rank -- the count of earlier groups of
the same width -- cannot exceed the group's own index). A failed check skips the access it
guards and records its site, (unit << 8) | n, in a device word that cq_debug_word reads and
clears. These tests stand in for a memory checker:

* every entry point, on ragged shapes, through the debug build: no check fires, and the results
  are those of the release build (bit for bit; the GEMM, whose segments meet in fp32 atomics,
  to within rounding);
* a damaged offset map (one group's offset off its grid; one group's rank above its index,
  chosen so that even the unchecked address stays inside its plane) is reported by each kernel
  that reads it, with the site of that kernel, and the context stays usable;
* the self-test kernel's deliberate failure is reported and then cleared.
The release library has no checks and says so (CQ_ERR_UNSUPPORTED).
"""
import contextlib
import os

import numpy as np
import pytest
import torch

from cell_updates_b200 import build, cq, ops, synth
from gpu_util import bf16_dev, dev, host

pytestmark = pytest.mark.gpu

ROWS, COLS = 300, 64 * 21          # ragged 16-row tiles and 4-group chunks
GROWS, GCOLS = 384, 64 * 40        # a shape the tensor-core GEMM takes


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    build.build()


@contextlib.contextmanager
def debug_library():
    """cq's entry points (and so ops.*) bound to the debug build for the duration."""
    saved = (cq.LIBCQ_PATH, cq._lib)
    cq.LIBCQ_PATH, cq._lib = build.test_variant_path("debug"), None
    try:
        cq.lib()
        yield
    finally:
        torch.cuda.synchronize()
        cq.LIBCQ_PATH, cq._lib = saved


def _inputs():
    w = synth.normal_weights(ROWS, COLS, seed=5)
    bits = synth.vbq_bits(ROWS * COLS // 64, seed=6)
    wg = synth.normal_weights(GROWS, GCOLS, seed=7)
    return w, bits, wg


def _run_all(after=None):
    """Every entry point once; `after(name)` is called after each (the debug word check)."""
    after = after or (lambda name: None)
    w, bits, wg = _inputs()
    out = {}
    wd, bd = dev(w), dev(bits)
    q4, c4, st4 = ops.quantize_and_pack(wd)
    after("quantize/pack fixed-4")
    qv, cv, stv = ops.quantize_and_pack(wd, bd)
    after("quantize/index/pack per-group widths")
    out.update(codes4=host(c4), plane4=host(q4.planes[2]), scale4=host(q4.scale), zero4=host(q4.zero),
               st4=host(st4), codesv=host(cv), offsetv=host(qv.offset), stv=host(stv),
               planesv=[host(p) for p in qv.planes])
    out["unpack"] = host(ops.unpack(qv))
    after("unpack")
    x1 = bf16_dev(synth.activations(1, COLS, seed=8, dtype="bf16"))
    x3 = dev(synth.activations(3, COLS, seed=9, dtype="f32"))
    x8 = bf16_dev(synth.activations(8, COLS, seed=10, dtype="bf16"))
    for name, qw in (("gemv4", q4), ("gemvv", qv)):
        for xn, x in (("m1", x1), ("m3", x3), ("m8", x8)):
            out[f"{name}_{xn}"] = host(ops.gemv(qw, x))
            after(f"{name} {xn}")
    r = bf16_dev(synth.normal_residual_bf16(host(q4.scale, np.uint16), seed=11))
    n_clamped = ops.project(r, q4.scale)
    after("project")
    out["r_projected"], out["n_clamped"] = host(r.view(torch.int16)), host(n_clamped)
    q4r = q4.with_residual(r)
    out["gemv4r_m1"] = host(ops.gemv(q4r, x1))
    after("served-weight GEMV")
    out["verify"] = [host(t) for t in ops.verify(q4r, flags=True)]
    after("verify")
    rv = bf16_dev(synth.normal_residual_bf16(host(qv.scale, np.uint16), seed=17))
    ops.project(rv, qv.scale)
    out["verify_pair"] = [host(t) for t in ops.verify_pair(qv.with_residual(rv), flags=True)[:4]]
    after("project, verify pair (per-group widths)")
    stages, _, _ = ops.rrq_build(wd, 2)
    after("rrq stages")
    out["stages_m1"] = host(ops.gemv_stages(stages, x1))
    out["stages_m3"] = host(ops.gemv_stages(stages, x3))
    after("stage GEMV")
    theta = dev((np.random.default_rng(12).standard_normal(ROWS * COLS) * 2.0).astype(np.float32))
    out["reparam"] = host(ops.reparam(theta, q4.scale).view(torch.int16))
    gr = dev(np.random.default_rng(13).standard_normal(ROWS * COLS).astype(np.float32))
    out["reparam_grad"] = host(ops.reparam_grad(theta, q4.scale, gr))
    after("reparameterization")
    rng = np.random.default_rng(14)
    Xc = rng.standard_normal((128, 320))
    H = Xc.T @ Xc
    H = (H + H.T) * 0.5
    wr = synth.normal_weights(37, 320, seed=15)
    cr, sr, zr, _ = ops.quantize(dev(wr))
    rq = ops.requant_refine(dev(wr), dev(H), sr, zr, cr, sweeps=2)
    out["requant"] = [host(t) for t in rq]
    after("ReQuant")
    qg, _, _ = ops.quantize_and_pack(dev(wg))
    for m in (17, 64):
        xg = bf16_dev(synth.activations(m, GCOLS, seed=16 + m, dtype="bf16"))
        out[f"gemm_m{m}"] = host(ops.gemm(qg, xg))
        after(f"GEMM m={m}")
    return out


@pytest.mark.skipif(os.environ.get("CQ_TEST_DEBUG_LIB") == "1", reason="the whole suite runs on the debug build")
def test_release_build_has_no_checks():
    with pytest.raises(cq.CQError) as e:
        cq.cq_debug_word()
    assert e.value.status == 8                      # CQ_ERR_UNSUPPORTED
    with pytest.raises(cq.CQError):
        cq.cq_debug_selftest()


def test_selftest_is_reported_then_cleared():
    with debug_library():
        assert cq.cq_debug_word() == 0
        cq.cq_debug_selftest()
        assert cq.cq_debug_word() == 0x0F01
        assert cq.cq_debug_word() == 0


def test_every_entry_point_clean_and_equal_to_release():
    ref = _run_all()
    torch.cuda.synchronize()
    fired = []
    with debug_library():
        assert cq.cq_debug_word() == 0

        def after(name):
            word = cq.cq_debug_word()
            if word:
                fired.append((name, hex(word)))

        got = _run_all(after)
    assert not fired, fired
    for k, v in ref.items():
        if k.startswith("gemm_"):
            err = np.abs(got[k].astype(np.float64) - v)
            assert err.max() <= 1e-5 * max(np.abs(v).max(), 1e-30), k
        elif isinstance(v, list):
            for a, b in zip(v, got[k]):
                assert np.array_equal(a, b), k
        else:
            assert np.array_equal(v, got[k]), k


def _damaged(qv, g, new_offset):
    off = qv.offset.clone()
    off[g] = int(new_offset)
    return cq.QWeight(qv.rows, qv.cols, qv.planes, qv.scale, qv.zero, qv.bits, off)


def test_damaged_offsets_are_reported_by_every_reader():
    w, bits, _ = _inputs()
    KG = COLS // 64
    row0 = bits[:KG]
    g2 = int(np.flatnonzero(row0 == 2)[0])           # first 2-bit group of row 0
    g1 = int(np.flatnonzero(row0 == 1)[0])           # first 1-bit group of row 0
    x1 = bf16_dev(synth.activations(1, COLS, seed=8, dtype="bf16"))
    x3 = dev(synth.activations(3, COLS, seed=9, dtype="f32"))
    with debug_library():
        qv, codes, _ = ops.quantize_and_pack(dev(w), dev(bits))
        offs = host(qv.offset).view(np.uint32)
        pb = [int(p.numel()) for p in qv.planes]
        assert cq.cq_debug_word() == 0
        # (site for: pack, unpack, verify, batch-1 GEMV, batch-3 GEMV)
        cases = [
            # off its grid by one byte: the readers mask it back onto the grid (in bounds)
            (g2, int(offs[g2]) + 1, (0x0201, 0x0202, 0x0401, 0x0704, 0x0701)),
            # rank one above the group's own index
            (g1, 8 * (g1 + 1), (0x0201, 0x0202, 0x0401, 0x0705, 0x0702)),
        ]
        # even unchecked, both damaged groups' bytes would lie inside their planes
        assert int(offs[g2]) + 1 + 16 <= pb[1] and 8 * (g1 + 1) + 8 <= pb[0]
        for g, bad, sites in cases:
            dq = _damaged(qv, g, bad)
            ops.pack(codes, ROWS, COLS, dq.bits, dq.offset, pb)
            assert cq.cq_debug_word() == sites[0]
            ops.unpack(dq)
            assert cq.cq_debug_word() == sites[1]
            ops.verify(dq)
            assert cq.cq_debug_word() == sites[2]
            ops.gemv(dq, x1)
            assert cq.cq_debug_word() == sites[3]
            ops.gemv(dq, x3)
            assert cq.cq_debug_word() == sites[4]
        # the context is still usable and the undamaged artifact reads back exactly
        assert np.array_equal(host(ops.unpack(qv)), host(codes))
        assert cq.cq_debug_word() == 0
