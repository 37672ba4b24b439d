"""The C oracle and its NumPy twin agree bit for bit on the small workloads."""
import numpy as np
import pytest

from cell_updates_b200 import synth
from oracle import c_oracle as co
from oracle import np_oracle as no


@pytest.mark.parametrize("case", ["fixed4", "vbq"])
def test_quantize_pack_verify_agree(case):
    w = synth.normal_weights(256, 512, seed=0)
    w[3, 7] = np.nan
    G = 256 * 512 // 64
    bits = None if case == "fixed4" else synth.vbq_bits(G, seed=2)
    c = co.quantize(w, bits)
    n = no.quantize(w, bits)
    assert c[3] == n[3] == 1
    for a, b in zip(c[:3], n[:3]):
        assert np.array_equal(a, b)
    codes, scale, zero, _ = c
    if bits is None:
        pc, off = co.pack(codes), None
    else:
        off, pb = co.varbits_index(bits)
        pc = co.pack(codes, bits, off, pb)
    pn = no.pack(codes, bits)
    for a, b in zip(pc, pn):
        assert np.array_equal(a[:b.size], b)
    r = synth.uniform_residual_f32(scale, seed=10)
    mc, fc, flags = co.verify(pc, scale, zero, bits, off, r, want_flags=True)
    mn, fn, mask = no.verify(pn, scale, zero, bits, r)
    assert (mc, fc) == (mn, fn) and mc > 0
    cmask = ((flags[np.arange(G) // 32] >> (np.arange(G) % 32).astype(np.uint32)) & 1).astype(bool)
    assert np.array_equal(cmask, mask)
    rp_c, nc = co.project_f32(r, scale)
    rp_n, nn = no.project_f32(r, scale)
    assert nc == nn and np.array_equal(rp_c.view(np.uint32), rp_n.view(np.uint32))
    rb = synth.normal_residual_bf16(scale, seed=11, rel_sigma=0.3)
    pb_c, nbc = co.project_bf16(rb, scale)
    pb_n, nbn = no.project_bf16(rb, scale)
    assert nbc == nbn and np.array_equal(pb_c, pb_n)
    x = synth.activations(8, 512, seed=5, dtype="bf16")
    yc = co.dequant_matmul_f64(pc, scale, zero, 256, 512, x, "bf16", bits, off, rp_c)
    yn = no.dequant_matmul_f64(pn, scale, zero, 256, 512, x, "bf16", bits, rp_c)
    assert np.allclose(yc, yn, rtol=1e-12, atol=1e-12)


def test_chunked_verify_matches_whole():
    w = synth.normal_weights(64, 1024, seed=4)
    codes, scale, zero, _ = co.quantize(w)
    planes = co.pack(codes)
    r = synth.uniform_residual_f32(scale, seed=12)
    total, first, _ = co.verify(planes, scale, zero, r=r, nthreads=3)
    parts, firsts = 0, []
    for c0 in range(0, codes.size, 64 * 37):
        n = min(64 * 37, codes.size - c0)
        m, fb, _ = co.verify(planes, scale, zero, r=r, first_w=c0, n_w=n, nthreads=2)
        parts += m
        if fb >= 0:
            firsts.append(fb)
    assert parts == total and min(firsts) == first


def test_reparam_twins_agree():
    # the bounded reparameterization: C and NumPy give the same bits, forward and backward
    from oracle import np_oracle as no
    rng = np.random.default_rng(2027)
    G = 500
    scale = rng.integers(1, 0x7BFF, G).astype(np.uint16)
    theta = (rng.standard_normal(G * 64) * rng.choice([1e-3, 1.0, 30.0, 1e6], G * 64)).astype(np.float32)
    theta[:8] = [np.inf, -np.inf, np.nan, 0.0, -0.0, 1e-40, 2.0 ** 32, -3e38]
    g = rng.standard_normal(G * 64).astype(np.float32)
    for dt in ("f32", "bf16"):
        a, b = co.reparam(theta, scale, dt), no.reparam(theta, scale, dt)
        assert np.array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8)), dt
        ga, gb = co.reparam_grad(theta, scale, g, dt), no.reparam_grad(theta, scale, g, dt)
        assert np.array_equal(ga.view(np.uint32), gb.view(np.uint32)), dt


def test_requant_twins_agree():
    # ReQuant refinement: C and NumPy give the same codes, moves and errors, bit for bit
    rng = np.random.default_rng(2028)
    rows, cols = 5, 192
    w = synth.normal_weights(rows, cols, seed=12)
    codes, scale, zero, _ = co.quantize(w)
    X = rng.standard_normal((400, cols))
    X[:, 7] *= 10.0
    H = X.T @ X
    a = co.requant_refine(w, H, codes, scale, zero, 4, 2)
    b = no.requant_refine(w, H, codes, scale, zero, 4, 2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[3], b[3]) and a[3].sum() > 0
    assert np.array_equal(a[1].view(np.uint64), b[1].view(np.uint64))
    assert np.array_equal(a[2].view(np.uint64), b[2].view(np.uint64))
