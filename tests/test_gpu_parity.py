"""GPU (CUDA path through the C ABI) against the CPU oracle on the same seeded inputs.

Bit-exact: codes, scales, zeros, status, group offsets, plane bytes, unpacked codes,
projected residuals and clamp counts, verify counts / first index / group flags.
Tolerance (benchmark spec): the matmuls vs the fp64 oracle, relative Frobenius
error <= 2e-3 and per-element |err| <= 1e-2 * rms(y).
Sizes span several tiles plus ragged tails; the config-0 shape is included.
"""
import numpy as np
import pytest
import torch

from cell_updates_b200 import cq, ops, synth
from gpu_util import bf16_dev, check_matmul, dev, host, planes_host, u16_dev
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from cell_updates_b200 import build
    build.build()
    cq.lib()


def _oracle_qw(codes, scale, zero, bits):
    """the oracle's own packing of its own codes"""
    if bits is None:
        return co.pack(codes), None
    off, pb = co.varbits_index(bits)
    return co.pack(codes, bits, off, pb), off


def _quantize_both(w, bits=None):
    bits_d = dev(bits) if bits is not None else None
    qw, codes_d, st_d = ops.quantize_and_pack(dev(w), bits_d)
    torch.cuda.synchronize()
    oc = co.quantize(w, bits)
    return qw, codes_d, st_d, oc


def _assert_quant_equal(codes_d, qw, st_d, oc):
    codes, scale, zero, st = oc
    assert np.array_equal(host(codes_d), codes)
    assert np.array_equal(host(qw.scale, np.uint16), scale)
    assert np.array_equal(host(qw.zero), zero)
    assert int(host(st_d)[0]) == st


# ---- quantize ------------------------------------------------------------------------

@pytest.mark.parametrize("shape,seed", [((256, 512), 0), ((37, 64 * 13), 3), ((1, 64), 4)])
def test_quantize_fixed4_bit_exact(shape, seed):
    w = synth.normal_weights(*shape, seed=seed)
    qw, codes_d, st_d, oc = _quantize_both(w)
    _assert_quant_equal(codes_d, qw, st_d, oc)


def test_quantize_edge_groups_bit_exact():
    rng = np.random.default_rng(8)
    rows = []
    i = np.arange(64)
    rows.append((0.25 * (i % 16) - 2.0))                                  # exact grid
    t = np.full(64, 1.0); t[:10] = [0, 3.75, .625, .875, .125, .375, 3.625, 3.375, 1.125, 1.375]
    rows.append(t)                                                         # ties
    rows.append(np.full(64, 0.5)); rows.append(np.zeros(64)); rows.append(np.full(64, -0.5))
    rows.append(rng.uniform(1, 3, 64)); rows.append(-rng.uniform(1, 3, 64))
    r = np.zeros(64); r[3] = np.nan; rows.append(r)
    r = np.zeros(64); r[9] = -np.inf; rows.append(r)
    r = np.zeros(64); r[0], r[1] = -3e38, 3e38; rows.append(r)
    r = np.zeros(64); r[0], r[1] = 0.0, 1e6; rows.append(r)             # fp16 overflow of s
    rows.append(rng.standard_t(2, 64) * 1e-6)                              # sub-2^-14 scales
    rows.append(rng.standard_normal(64) * 1e4)
    w = np.stack([np.asarray(v, np.float32) for v in rows]).reshape(1, -1)
    w = np.repeat(w, 3, axis=0)
    G = w.size // 64
    bits = np.tile(np.array([1, 2, 4, 8], np.uint8), G // 4 + 1)[:G]
    bits[5] = 3                                                            # bad width
    for b in (None, bits):
        qw_codes = _quantize_both(w, b) if b is None else None
        if b is None:
            qw, codes_d, st_d, oc = qw_codes
            _assert_quant_equal(codes_d, qw, st_d, oc)
        else:
            codes_d, scale_d, zero_d, st_d = ops.quantize(dev(w), dev(b))
            torch.cuda.synchronize()
            oc = co.quantize(w, b)
            assert np.array_equal(host(codes_d), oc[0])
            assert np.array_equal(host(scale_d, np.uint16), oc[1])
            assert np.array_equal(host(zero_d), oc[2])
            assert int(host(st_d)[0]) == oc[3] == 7


def test_quantize_vbq_config2_bit_exact():
    # 2048 x 8192 ~ N(0, 0.02^2), widths drawn with the VBQ allocation statistics
    w = synth.normal_weights(2048, 8192, seed=2)
    bits = synth.vbq_bits(2048 * 8192 // 64, seed=2)
    qw, codes_d, st_d, oc = _quantize_both(w, bits)
    _assert_quant_equal(codes_d, qw, st_d, oc)
    off, pb = co.varbits_index(bits)
    assert np.array_equal(host(qw.offset, np.uint32), off)
    planes = co.pack(oc[0], bits, off, pb)
    for slot in range(4):
        assert np.array_equal(host(qw.planes[slot])[:pb[slot]], planes[slot][:pb[slot]])
    assert np.array_equal(host(ops.unpack(qw)), oc[0])


# ---- pack / index -------------------------------------------------------------------------

@pytest.mark.parametrize("G", [1, 3, 4095, 4096, 4097, 3 * 4096 + 5, 70000])
def test_varbits_index_and_pack_bit_exact(G):
    rng = np.random.default_rng(G)
    bits = synth.vbq_bits(G, seed=G)
    L = (1 << bits.astype(np.int64)) - 1
    codes = (rng.integers(0, 256, (G, 64)) & L[:, None]).astype(np.uint8).ravel()
    off, pb = co.varbits_index(bits)
    off_d, pb_d = ops.varbits_index(dev(bits))
    assert np.array_equal(host(off_d, np.uint32), off) and pb_d == pb
    planes_d = ops.pack(dev(codes), G, 64, dev(bits), off_d, pb_d)
    planes = co.pack(codes, bits, off, pb)
    for slot in range(4):
        assert np.array_equal(host(planes_d[slot])[:pb[slot]], planes[slot][:pb[slot]])
    qw = cq.QWeight(G, 64, planes_d, u16_dev(np.zeros(G, np.uint16)), dev(np.zeros(G, np.uint8)), dev(bits), off_d)
    assert np.array_equal(host(ops.unpack(qw)), codes)


@pytest.mark.parametrize("G", [262143, 262144, 262145, 600001, 1 << 20, (1 << 20) + 1, 1300001])
def test_varbits_index_large_unaligned_and_invalid(G):
    """The index's three chained passes over 64 to 318 tiles of 4096 groups (a ragged last tile
    on both sides of the power-of-two sizes); with the width map and the offsets off their
    16-byte boundaries; and with widths outside {1, 2, 4, 8}, which take no bytes and get offset
    0 while the valid groups keep the offsets of the valid subsequence."""
    bits = synth.vbq_bits(G, seed=G)
    off, pb = co.varbits_index(bits)
    off_d, pb_d = ops.varbits_index(dev(bits))
    assert np.array_equal(host(off_d, np.uint32), off) and pb_d == pb
    bbuf = torch.zeros(G + 16, dtype=torch.uint8, device="cuda")
    bbuf[1:G + 1] = dev(bits)
    obuf = torch.full((G + 4,), -1, dtype=torch.int32, device="cuda")
    pbt = torch.empty(4, dtype=torch.int64, device="cuda")
    cq.cq_varbits_index(bbuf[1:G + 1], obuf[1:G + 1], pbt)
    torch.cuda.synchronize()
    assert np.array_equal(host(obuf[1:G + 1], np.uint32), off) and [int(v) for v in pbt.cpu()] == pb
    assert int(obuf[0].item()) == -1 and int(obuf[G + 1].item()) == -1
    rng = np.random.default_rng(G)
    bad = bits.copy()
    idx = rng.choice(G, G // 97 + 1, replace=False)
    bad[idx] = rng.choice(np.array([0, 3, 5, 16, 255], np.uint8), idx.size)
    valid = np.ones(G, bool)
    valid[idx] = False
    off_v, pb_v = co.varbits_index(bits[valid])
    off_b, pb_b = ops.varbits_index(dev(bad))
    got = host(off_b, np.uint32)
    assert np.all(got[~valid] == 0) and np.array_equal(got[valid], off_v) and pb_b == pb_v


# ---- projection ---------------------------------------------------------------------------------

def _residual_cases(scale, seed):
    rng = np.random.default_rng(seed)
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float32)
    G = sf.size
    mult = rng.uniform(-0.8, 0.8, (G, 64)).astype(np.float32)
    mult[:, :6] = [0.5, -0.5, 0.5 - 2 ** -10, 0.5 + 2 ** -10, 1e30, -1e30]
    r = (mult * sf[:, None]).astype(np.float32)
    r[0, 7] = np.nan
    r[1, 8] = -0.0
    return r.ravel()


def test_project_f32_bit_exact():
    w = synth.normal_weights(256, 512, seed=0)
    _, scale, _, _ = co.quantize(w)
    r = _residual_cases(scale, 1)
    rp, n = co.project_f32(r, scale)
    r_d = dev(r)
    n_d = ops.project(r_d, u16_dev(scale))
    torch.cuda.synchronize()
    assert np.array_equal(host(r_d).view(np.uint32), rp.view(np.uint32))
    assert int(host(n_d)[0]) == n


def test_project_bf16_bit_exact():
    rng = np.random.default_rng(5)
    G = 3001
    scale = rng.integers(0x0001, 0x7C01, G).astype(np.uint16)        # incl. subnormal and +inf
    r = _residual_cases(scale, 2)
    rb = (r.view(np.uint32) >> 16).astype(np.uint16)
    rp, n = co.project_bf16(rb, scale)
    r_d = bf16_dev(rb)
    n_d = ops.project(r_d, u16_dev(scale))
    torch.cuda.synchronize()
    assert np.array_equal(host(r_d, np.uint16), rp)
    assert int(host(n_d)[0]) == n


# ---- requant verify --------------------------------------------------------------------------

def _verify_both(qw, planes, scale, zero, bits, off, r, r_dtype, first_w=0, n_w=None):
    total = qw.rows * qw.cols
    if n_w is None:
        n_w = total - first_w
    m_d, f_d, g_d = ops.verify(qw, first_w, n_w, flags=True)
    torch.cuda.synchronize()
    m, f, flags = co.verify(planes, scale, zero, bits, off, r, r_dtype, first_w, n_w, want_flags=True)
    assert int(host(m_d)[0]) == m
    assert int(host(f_d)[0]) == f
    assert np.array_equal(host(g_d, np.uint32)[:flags.size], flags)
    return m


@pytest.mark.parametrize("varbits", [False, True])
def test_verify_config0_and_controls(varbits):
    w = synth.normal_weights(256, 512, seed=0)
    G = 256 * 512 // 64
    bits = synth.vbq_bits(G, seed=9) if varbits else None
    codes, scale, zero, _ = co.quantize(w, bits)
    planes, off = _oracle_qw(codes, scale, zero, bits)
    qw, _, _, _ = _quantize_both(w, bits)
    # negative control: r ~ U(-0.6 s, 0.6 s) unprojected
    r = synth.uniform_residual_f32(scale, seed=10)
    m = _verify_both(qw.with_residual(dev(r)), planes, scale, zero, bits, off, r, "f32")
    assert m > 0
    # chunks of whole groups give the same answer piecewise
    for first, n in [(0, 64 * 100), (64 * 100, 64 * 37), (64 * 1000, w.size - 64 * 1000)]:
        _verify_both(qw.with_residual(dev(r)), planes, scale, zero, bits, off, r, "f32", first, n)
    # projected: bit-identical; dropped: revoked
    rp, _ = co.project_f32(r, scale)
    assert _verify_both(qw.with_residual(dev(rp)), planes, scale, zero, bits, off, rp, "f32") == 0
    assert _verify_both(qw, planes, scale, zero, bits, off, None, "f32") == 0
    # bf16 residual, projected and not
    rb = synth.normal_residual_bf16(scale, seed=11, rel_sigma=0.3)
    assert _verify_both(qw.with_residual(bf16_dev(rb)), planes, scale, zero, bits, off, rb, "bf16") > 0
    rbp, _ = co.project_bf16(rb, scale)
    assert _verify_both(qw.with_residual(bf16_dev(rbp)), planes, scale, zero, bits, off, rbp, "bf16") == 0


def test_verify_boundary_and_corrupt_scales():
    rng = np.random.default_rng(12)
    G = 4096 + 17
    codes = rng.integers(0, 16, G * 64).astype(np.uint8)
    zero = rng.integers(0, 16, G).astype(np.uint8)
    scale = rng.integers(0x0001, 0x7C00, G).astype(np.uint16)
    scale[:4] = [0x0000, 0x7C00, 0x7E00, 0xBC00]                        # 0, inf, NaN, -1
    planes = co.pack(codes)
    r = _residual_cases(scale, 13)
    qw = cq.QWeight(G, 64, [None, None, dev(planes[2]), None], u16_dev(scale), dev(zero))
    m = _verify_both(qw.with_residual(dev(r)), planes, scale, zero, None, None, r, "f32")
    assert m > 0


def _pair_both(qw_r, planes, scale, zero, bits, off, r, r_dtype, first_w=0, n_w=None):
    """cq_requant_verify_pair against the oracle's two checks (with r, and with r dropped)"""
    total = qw_r.rows * qw_r.cols
    if n_w is None:
        n_w = total - first_w
    m_d, f_d, m0_d, f0_d, g_d = ops.verify_pair(qw_r, first_w, n_w, flags=True)
    torch.cuda.synchronize()
    m, f, flags = co.verify(planes, scale, zero, bits, off, r, r_dtype, first_w, n_w, want_flags=True)
    m0, f0, _ = co.verify(planes, scale, zero, bits, off, None, "f32", first_w, n_w, want_flags=True)
    assert (int(host(m_d)[0]), int(host(f_d)[0])) == (m, f)
    assert (int(host(m0_d)[0]), int(host(f0_d)[0])) == (m0, f0)
    assert np.array_equal(host(g_d, np.uint32)[:flags.size], flags)
    return m, m0


@pytest.mark.parametrize("varbits", [False, True])
def test_verify_pair(varbits):
    """both CellFill checks in one call: with the residual and after dropping it"""
    rows, cols = 300, 64 * 21
    w = synth.normal_weights(rows, cols, seed=40)
    w[7, 100] = np.nan                                    # a flagged group: both checks mismatch there
    G = rows * cols // 64
    bits = synth.vbq_bits(G, seed=41) if varbits else None
    codes, scale, zero, _ = co.quantize(w, bits)
    planes, off = _oracle_qw(codes, scale, zero, bits)
    qw, _, _, _ = _quantize_both(w, bits)
    r = synth.uniform_residual_f32(scale, seed=42)
    m, m0 = _pair_both(qw.with_residual(dev(r)), planes, scale, zero, bits, off, r, "f32")
    assert m > 64 and m0 == 64
    rp, _ = co.project_f32(r, scale)
    m, m0 = _pair_both(qw.with_residual(dev(rp)), planes, scale, zero, bits, off, rp, "f32")
    assert m0 == 64                                       # only the flagged group fails revocation
    rb = synth.normal_residual_bf16(scale, seed=43, rel_sigma=0.3)
    _pair_both(qw.with_residual(bf16_dev(rb)), planes, scale, zero, bits, off, rb, "bf16")
    rbp, _ = co.project_bf16(rb, scale)
    for first, n in [(0, 64 * 100), (64 * 100, 64 * 37), (64 * 1000, w.size - 64 * 1000)]:
        _pair_both(qw.with_residual(bf16_dev(rbp)), planes, scale, zero, bits, off, rbp, "bf16", first, n)


def test_verify_pair_corrupt_scales():
    """zero, infinite, NaN and negative scales, residuals on and across the cell edges"""
    rng = np.random.default_rng(44)
    G = 4096 + 17
    codes = rng.integers(0, 16, G * 64).astype(np.uint8)
    zero = rng.integers(0, 16, G).astype(np.uint8)
    scale = rng.integers(0x0001, 0x7C00, G).astype(np.uint16)
    scale[:4] = [0x0000, 0x7C00, 0x7E00, 0xBC00]
    planes = co.pack(codes)
    r = _residual_cases(scale, 45)
    qw = cq.QWeight(G, 64, [None, None, dev(planes[2]), None], u16_dev(scale), dev(zero))
    m, m0 = _pair_both(qw.with_residual(dev(r)), planes, scale, zero, None, None, r, "f32")
    assert m > 0 and m0 > 0


# ---- matmuls ------------------------------------------------------------------------------------

def _matmul_case(rows, cols, m, x_dtype, bits=None, r=None, seed=0):
    w = synth.normal_weights(rows, cols, seed=seed)
    qw, _, _, oc = _quantize_both(w, bits)
    codes, scale, zero, _ = oc
    planes, off = _oracle_qw(codes, scale, zero, bits)
    x = synth.activations(m, cols, seed=seed + 1, dtype=x_dtype)
    x_d = bf16_dev(x) if x_dtype == "bf16" else dev(x)
    r_dtype = None
    if r is not None:
        r_dtype = "bf16" if r.dtype == np.uint16 else "f32"
        qw = qw.with_residual(bf16_dev(r) if r_dtype == "bf16" else dev(r))
    y_ref = co.dequant_matmul_f64(planes, scale, zero, rows, cols, x, x_dtype, bits, off, r, r_dtype or "f32")
    return qw, x_d, y_ref, scale


def test_gemv_config0_fp32_with_projected_residual():
    w = synth.normal_weights(256, 512, seed=0)
    _, scale, _, _ = co.quantize(w)
    rp, _ = co.project_f32(synth.uniform_residual_f32(scale, seed=10), scale)
    qw, x_d, y_ref, _ = _matmul_case(256, 512, 1, "f32", r=rp)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, "cfg0 r")
    qw0, x0, y0, _ = _matmul_case(256, 512, 1, "f32")
    check_matmul(host(ops.gemv(qw0, x0)), y0, "cfg0 revoked")


# shapes: whole and ragged 4-group chunks and 16-row tiles; more tiles than the persistent
# grid holds (5000 rows); activations too large to stage in shared memory (K = 16384, 12864)
@pytest.mark.parametrize("rows,cols", [(256, 512), (16, 64), (47, 64 * 9), (300, 64 * 21), (1000, 4096),
                                       (5000, 64 * 16), (48, 64 * 256), (40, 64 * 201)])
@pytest.mark.parametrize("m", [1, 3, 8])
def test_gemv_tensor_core_4bit(rows, cols, m):
    qw, x_d, y_ref, _ = _matmul_case(rows, cols, m, "bf16", seed=rows + m)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, f"{rows}x{cols} m={m}")


# several matrices sharing x in one launch: ragged tiles in every segment, more than four
# matrices (two launches), and a variable-width matrix in the list (single-matrix path)
@pytest.mark.parametrize("m", [1, 3, 8])
def test_gemv_multi_segments(m):
    cols = 64 * 21
    specs = [(300, None), (47, None), (64, "vbq"), (1000, None), (16, None), (129, None)]
    x = synth.activations(m, cols, seed=91 + m, dtype="bf16")
    qws, refs = [], []
    for i, (rows, kind) in enumerate(specs):
        w = synth.normal_weights(rows, cols, seed=70 + i)
        bits = synth.vbq_bits(rows * cols // 64, seed=80 + i) if kind else None
        qw, _, _, oc = _quantize_both(w, bits)
        planes, off = _oracle_qw(oc[0], oc[1], oc[2], bits)
        qws.append(qw)
        refs.append(co.dequant_matmul_f64(planes, oc[1], oc[2], rows, cols, x, "bf16", bits, off))
    ys = ops.gemv_multi(qws, bf16_dev(x))
    for i, (qw, y_ref) in enumerate(zip(qws, refs)):
        check_matmul(host(ys[i]), y_ref, f"multi[{i}] {qw.rows}x{qw.cols} m={m}")


@pytest.mark.parametrize("m", [1, 8])
def test_gemv_varbits(m):
    G = 512 * 1024 // 64
    bits = synth.vbq_bits(G, seed=3)
    qw, x_d, y_ref, _ = _matmul_case(512, 1024, m, "bf16", bits=bits, seed=5)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, f"vbq m={m}")


# the per-group-width kernels: ragged 16-row tiles, group runs that do not split evenly over the
# CTA's warps (fewer groups than warps, too), fp32 activations (two bf16 parts), width maps of one
# width only (8-bit groups take their own operand path), and at batch 1 long rows whose width
# runs take several passes of 64 (300, 257, 129, 128 groups)
@pytest.mark.parametrize("rows,cols,m,x_dtype,only", [(47, 64 * 9, 3, "f32", None), (300, 64 * 21, 8, "bf16", None),
                                                      (16, 64, 1, "bf16", None), (1000, 4096, 1, "f32", None),
                                                      (129, 64 * 37, 5, "bf16", 8), (64, 64 * 40, 8, "f32", 8),
                                                      (200, 64 * 16, 2, "bf16", 1), (33, 64 * 5, 7, "bf16", 2),
                                                      (70, 64 * 300, 1, "bf16", None), (50, 64 * 257, 1, "f32", 8),
                                                      (45, 64 * 129, 1, "bf16", 1), (9, 64 * 128, 1, "bf16", 2)])
def test_gemv_varbits_shapes(rows, cols, m, x_dtype, only):
    G = rows * cols // 64
    bits = np.full(G, only, np.uint8) if only else synth.vbq_bits(G, seed=rows + cols)
    qw, x_d, y_ref, _ = _matmul_case(rows, cols, m, x_dtype, bits=bits, seed=rows + m)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, f"vbq {rows}x{cols} m={m} {x_dtype} only={only}")


@pytest.mark.parametrize("rows,cols,m", [(70, 64 * 300, 1), (33, 64 * 40, 1), (33, 64 * 40, 3)])
def test_gemv_stages_fixed4_and_varbits(rows, cols, m):
    """A stack of a fixed-4 matrix and a per-group-width matrix of the same shape, multiplied with
    the same activations: the sum of the two products, the fixed-4 stage at batch 1 included."""
    bits = synth.vbq_bits(rows * cols // 64, seed=cols)
    q4, x_d, y4, _ = _matmul_case(rows, cols, m, "bf16", seed=41)
    qv, x_dv, yv, _ = _matmul_case(rows, cols, m, "bf16", bits=bits, seed=41)
    assert torch.equal(x_d, x_dv)
    check_matmul(host(ops.gemv_stages([q4, qv], x_d)), y4 + yv, f"fixed-4 + vbq stack {rows}x{cols} m={m}")
    check_matmul(host(ops.gemv_stages([qv, q4, qv], x_d)), y4 + 2 * yv, f"vbq + fixed-4 + vbq {rows}x{cols} m={m}")


def test_gemv_varbits_rows_too_long_to_stage():
    """Batch 1 with rows whose staged activations exceed the width-sorted kernel's shared
    memory (760 groups): the tensor-core kernel takes them."""
    rows, cols = 40, 64 * 760
    bits = synth.vbq_bits(rows * cols // 64, seed=23)
    for x_dtype in ("bf16", "f32"):
        qw, x_d, y_ref, _ = _matmul_case(rows, cols, 1, x_dtype, bits=bits, seed=29)
        check_matmul(host(ops.gemv(qw, x_d)), y_ref, f"vbq long rows m=1 {x_dtype}")


def test_gemv_fixed4_fp32_activations():
    qw, x_d, y_ref, _ = _matmul_case(300, 64 * 21, 6, "f32", seed=17)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, "fixed-4 f32 x")


@pytest.mark.parametrize("rows,cols,m", [(384, 64 * 40, 16), (384, 64 * 40, 64), (200, 64 * 7, 17),
                                         (1000, 4096, 33), (128, 64, 100), (2500, 2048, 256),
                                         (4096, 4096, 64)])
def test_gemm_tensor_core(rows, cols, m):
    qw, x_d, y_ref, _ = _matmul_case(rows, cols, m, "bf16", seed=rows + m)
    check_matmul(host(ops.gemm(qw, x_d)), y_ref, f"gemm {rows}x{cols} m={m}")


def test_gemm_slow_groups_and_activation_range():
    """Groups the fp16 tensor-core operand cannot hold (|s| > 4096, z > 15) are summed by the
    epilogue in fp32; batch rows of very small, very large and zero activations go through the
    per-row power of two. Checked per (batch row, row subset) so no scale hides another."""
    rows, cols, m = 300, 64 * 24, 40
    KG = cols // 64
    w = synth.normal_weights(rows, cols, seed=31)
    codes, scale, zero, _ = co.quantize(w)
    rng = np.random.default_rng(32)
    slow_rows = np.sort(rng.choice(rows, 37, replace=False))
    scale2, zero2 = scale.copy(), zero.copy()
    big = np.array([5000.0, 60000.0, 4100.0], np.float16).view(np.uint16)
    for n, r in enumerate(slow_rows):
        g = r * KG + rng.integers(0, KG)
        if n % 3 == 2:
            zero2[g] = 200                               # zero point beyond the 4-bit range
        else:
            scale2[g] = big[n % 3]
    planes = co.pack(codes)
    x = synth.activations(m, cols, seed=33, dtype="f32")
    x[0] *= 1e-30
    x[1] *= 1e30
    x[2] = 0.0
    x[3, ::7] *= 1e6                                     # a row with a few large outliers
    xb = synth.f32_to_bf16_bits(x).reshape(m, cols)
    y_ref = co.dequant_matmul_f64(planes, scale2, zero2, rows, cols, xb, "bf16")
    qw = cq.QWeight(rows, cols, [None, None, dev(planes[2]), None], u16_dev(scale2), dev(zero2))
    y = host(ops.gemm(qw, bf16_dev(xb)))
    assert np.array_equal(y[2], np.zeros(rows, np.float32))
    fast_rows = np.setdiff1d(np.arange(rows), slow_rows)
    for i in [0, 1, 3, 4, m - 1]:
        for sub, name in ((slow_rows, "slow"), (fast_rows, "fast")):
            check_matmul(y[i, sub], y_ref[i, sub], f"batch row {i}, {name} rows")


def test_gemm_small_batch_uses_gemv_slices():
    qw, x_d, y_ref, _ = _matmul_case(300, 64 * 21, 12, "bf16", seed=12)
    check_matmul(host(ops.gemm(qw, x_d)), y_ref, "gemm m=12")


def test_gemm_bf16_residual_uses_exact_formula():
    w = synth.normal_weights(128, 1024, seed=21)
    _, scale, _, _ = co.quantize(w)
    rb, _ = co.project_bf16(synth.normal_residual_bf16(scale, seed=22), scale)
    qw, x_d, y_ref, _ = _matmul_case(128, 1024, 20, "bf16", r=rb, seed=21)
    check_matmul(host(ops.gemm(qw, x_d)), y_ref, "gemm r bf16")


# the CellFill served weights W = s (q - z) + r with a bf16 residual, on tensor cores: ragged
# 16-row tiles, fewer groups than warps (K = 64, 320), groups that split unevenly over the warps,
# the decode and CellFill-stack shapes, projected and unprojected residuals
@pytest.mark.parametrize("rows,cols", [(16, 64), (47, 64 * 5), (300, 64 * 21), (1000, 4096), (2048, 2048),
                                       (6144, 2048), (2048, 6144), (100, 11008)])
@pytest.mark.parametrize("m", [1, 3, 8])
def test_gemv_bf16_residual_tensor_core(rows, cols, m):
    w = synth.normal_weights(rows, cols, seed=rows + cols)
    _, scale, _, _ = co.quantize(w)
    rb = synth.normal_residual_bf16(scale, seed=rows + 3, rel_sigma=0.3)
    if rows % 2:
        rb, _ = co.project_bf16(rb, scale)
    qw, x_d, y_ref, _ = _matmul_case(rows, cols, m, "bf16", r=rb, seed=rows + cols)
    check_matmul(host(ops.gemv(qw, x_d)), y_ref, f"gemv r bf16 {rows}x{cols} m={m}")


# the batch GEMM with a bf16 residual (CellFill served weights): every batch slice size, ragged
# row tiles, several K ranges per CTA
@pytest.mark.parametrize("rows,cols,m", [(384, 64 * 40, 64), (1000, 4096, 33), (200, 64 * 8, 16),
                                         (129, 64 * 24, 100)])
def test_gemm_bf16_residual_batches(rows, cols, m):
    w = synth.normal_weights(rows, cols, seed=rows + m)
    _, scale, _, _ = co.quantize(w)
    rb, _ = co.project_bf16(synth.normal_residual_bf16(scale, seed=rows + 1, rel_sigma=0.3), scale)
    qw, x_d, y_ref, _ = _matmul_case(rows, cols, m, "bf16", r=rb, seed=rows + m)
    check_matmul(host(ops.gemm(qw, x_d)), y_ref, f"gemm r bf16 {rows}x{cols} m={m}")


# several served-weight matrices (bf16 residual) that share x in one launch: ragged tiles in every
# segment, more than four matrices (two launches), and a matrix without a residual in the list
@pytest.mark.parametrize("m", [1, 5])
def test_gemv_multi_with_residuals(m):
    cols = 64 * 21
    specs = [(300, True), (47, True), (64, True), (129, True), (1000, True), (33, False), (16, True)]
    x = synth.activations(m, cols, seed=191 + m, dtype="bf16")
    qws, refs = [], []
    for i, (rows, with_r) in enumerate(specs):
        w = synth.normal_weights(rows, cols, seed=170 + i)
        qw, _, _, oc = _quantize_both(w, None)
        planes, off = _oracle_qw(oc[0], oc[1], oc[2], None)
        rb = None
        if with_r:
            rb, _ = co.project_bf16(synth.normal_residual_bf16(oc[1], seed=180 + i, rel_sigma=0.3), oc[1])
            qw = qw.with_residual(bf16_dev(rb))
        qws.append(qw)
        refs.append(co.dequant_matmul_f64(planes, oc[1], oc[2], rows, cols, x, "bf16", None, None, rb,
                                          "bf16" if with_r else "f32"))
    ys = ops.gemv_multi(qws, bf16_dev(x))
    for i, (qw, y_ref) in enumerate(zip(qws, refs)):
        check_matmul(host(ys[i]), y_ref, f"multi residual[{i}] {qw.rows}x{qw.cols} m={m}")
