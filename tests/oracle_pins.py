"""Pins for the oracle: checks against what the pages and the mathematics fix, not
against the oracle's own formulas.

Each ``pin_*(impl)`` raises ``AssertionError`` when ``impl`` is wrong.  The pins are:

* closed-form groups whose scale, zero and codes follow by hand (exact grids, exact
  half-way ties, clamped zero points, constant groups, each bit-width);
* brute force: for tiny random groups, enumeration of all 2^b reconstruction levels
  in exact rational arithmetic must give the same code as the RTN formula (the
  VBQ/CellFill codes are nearest-level codes);
* the invariants the CellFill abstract states: dequantize -> requantize returns the
  codes; a zero or projected residual leaves the artifact bit-identical; dropping the
  residual revokes exactly; drift stays within the cell;
* a negative control whose mismatch count is predicted in exact rational arithmetic;
* layout facts of packed storage (LSB-first codes, plain nibbles for 4-bit);
* the fp64 matmul against NumPy's BLAS and closed forms.
"""
from fractions import Fraction

import numpy as np

GROUP = 64


def _f16(bits):
    return float(np.uint16(bits).view(np.float16))


def _q1(impl, w, b):
    """quantize one 64-weight group of width b."""
    w = np.asarray(w, np.float32).reshape(1, GROUP)
    codes, scale, zero, st = impl.quantize(w, np.array([b], np.uint8))
    return codes, int(scale[0]), int(zero[0]), st


def _expect(impl, w, b, s16, z, q):
    codes, s, zz, st = _q1(impl, w, b)
    assert st == 0, f"status {st}"
    assert s == s16, f"scale {s:#06x} != {s16:#06x}"
    assert zz == z, f"zero {zz} != {z}"
    assert np.array_equal(codes, np.asarray(q, np.uint8)), f"codes {codes.tolist()} != {list(q)}"


def _fill(vals, rest):
    w = np.full(GROUP, rest, np.float32)
    w[:len(vals)] = vals
    return w


# ---- closed-form quantize cases ------------------------------------------------------------

def pin_quant_exact_grid(impl):
    # w_i = 0.25*(i mod 16) - 2: wmin=-2, wmax=1.75, range/15 = 0.25 exactly (fp16 0x3400),
    # z = rne(2/0.25) = 8, q_i = (i mod 16) - 8 + 8 = i mod 16.
    i = np.arange(GROUP)
    w = (0.25 * (i % 16) - 2.0).astype(np.float32)
    _expect(impl, w, 4, 0x3400, 8, i % 16)


def pin_quant_ties_half_even(impl):
    # wmin=0, wmax=3.75 -> s=0.25, z=0; w/s lands exactly on .5: 2.5->2, 3.5->4, 0.5->0,
    # 1.5->2, 14.5->14, 13.5->14, 4.5->4, 5.5->6; the filler 1.0 -> 4.
    w = _fill([0.0, 3.75, 0.625, 0.875, 0.125, 0.375, 3.625, 3.375, 1.125, 1.375], 1.0)
    q = [0, 15, 2, 4, 0, 2, 14, 14, 4, 6] + [4] * 54
    _expect(impl, w, 4, 0x3400, 0, q)


def pin_quant_zero_tie(impl):
    # wmin=-0.625, wmax=3.125 -> s=0.25; z = rne(2.5) = 2.  -2.5->-2 (q 0), -1.5->-2 (q 0),
    # -0.5->0 (q 2), 0.5->0 (q 2), 12.5->12 (q 14), 1.5->2 (q 4); filler 0 -> q 2.
    w = _fill([-0.625, 3.125, -0.375, -0.125, 0.125, 0.375], 0.0)
    q = [0, 14, 0, 2, 2, 4] + [2] * 58
    _expect(impl, w, 4, 0x3400, 2, q)


def pin_quant_clamped_zero(impl):
    # all positive: range 1.875 -> s=0.125 (0x3000); z = rne(-8) -> clamp 0;
    # 1->8, 2.875->23->15, 1.5->12, 2->16->15, filler 1.25->10.
    w = _fill([1.0, 2.875, 1.5, 2.0], 1.25)
    _expect(impl, w, 4, 0x3000, 0, [8, 15, 12, 15] + [10] * 60)
    # all negative: z = rne(23) -> clamp 15; -1->7, -2.875->-8->0, -1.5->3, -2->-1->0, -1.25->5.
    _expect(impl, -w, 4, 0x3000, 15, [7, 0, 3, 0] + [5] * 60)


def pin_quant_constant_groups(impl):
    # range 0 -> s floors at 2^-14 (0x0400).  0.5: z = rne(-8192) -> 0, q = 8192 -> 15.
    _expect(impl, np.full(GROUP, 0.5, np.float32), 4, 0x0400, 0, [15] * GROUP)
    _expect(impl, np.zeros(GROUP, np.float32), 4, 0x0400, 0, [0] * GROUP)
    _expect(impl, np.full(GROUP, -0.5, np.float32), 4, 0x0400, 15, [0] * GROUP)


def pin_quant_each_width(impl):
    # 1 bit: w in {-1, 3}: s = 4/1 = 4 (0x4400), z = rne(0.25) = 0, q(-1)=rne(-0.25)=0, q(3)=rne(0.75)=1
    w = np.tile(np.array([-1.0, 3.0], np.float32), 32)
    _expect(impl, w, 1, 0x4400, 0, np.tile([0, 1], 32))
    # 1 bit: w in {-1, 1}: s = 2 (0x4000), z = rne(0.5) = 0 (tie to even), q = rne(+-0.5) = 0
    _expect(impl, np.tile(np.array([-1.0, 1.0], np.float32), 32), 1, 0x4000, 0, [0] * GROUP)
    # 2 bits: {-0.75,-0.25,0.25,0.75}: s = 1.5/3 = 0.5 (0x3800), z = rne(1.5) = 2;
    # q = -2+2, 0+2, 0+2, 2+2->3
    w = np.tile(np.array([-0.75, -0.25, 0.25, 0.75], np.float32), 16)
    _expect(impl, w, 2, 0x3800, 2, np.tile([0, 2, 2, 3], 16))
    # 8 bits: w_j = v_j / 256 with v = 4j and v_63 = 255: s = (255/256)/255 = 2^-8 (0x1C00), z = 0,
    # q_j = v_j
    v = 4 * np.arange(GROUP)
    v[63] = 255
    _expect(impl, (v / 256.0).astype(np.float32), 8, 0x1C00, 0, v)


def pin_quant_fp16_scale_rounding(impl):
    # range 1: RN32(1/15) rounds to fp16 0x2C44 = 0.066650390625 (1/15*1024/0.0625... hand:
    # 1/15 = 0.0625 * 1.0666.., mantissa 0.0666..*1024 = 68.27 -> 68).  z = rne(0.5/s) =
    # rne(7.5018) = 8; q(0.5) = 8+8 -> 15, q(-0.5) = 0, q(0) = 8, q(0.1) = rne(1.50037)+8 = 10.
    w = _fill([-0.5, 0.5, 0.1], 0.0)
    _expect(impl, w, 4, 0x2C44, 8, [0, 15, 10] + [8] * 61)


def pin_quant_status(impl):
    w = np.zeros((4, GROUP), np.float32)
    w[0, 5] = np.nan
    w[1, 7] = np.inf
    w[2, 0], w[2, 1] = -3e38, 3e38            # range overflows binary32 -> scale overflow
    w[3] = np.linspace(-1, 1, GROUP)
    codes, scale, zero, st = impl.quantize(w.reshape(1, -1), np.array([4, 4, 4, 4], np.uint8))
    assert st == 1 | 2, st
    assert scale[:3].tolist() == [0, 0, 0] and zero[:3].tolist() == [0, 0, 0]
    assert not codes[:3 * GROUP].any() and scale[3] != 0
    codes, scale, zero, st = impl.quantize(w[3:].reshape(1, -1), np.array([3], np.uint8))
    assert st == 4 and scale[0] == 0


# ---- brute force against all 2^b levels (exact rationals) -----------------------------------

def _tiny_groups(rng, n):
    out = []
    for t in range(n):
        kind = t % 5
        if kind == 0:
            w = rng.standard_normal(GROUP) * 0.02
        elif kind == 1:
            w = rng.uniform(-1, 1, GROUP) * 10.0 ** rng.integers(-3, 3)
        elif kind == 2:
            w = rng.standard_t(3, GROUP) * 0.05
        elif kind == 3:
            w = rng.uniform(0.1, 0.3, GROUP)          # all positive
        else:
            w = np.round(rng.standard_normal(GROUP) * 8) / 32.0   # many duplicates
        out.append(w.astype(np.float32))
    return out


def pin_quant_bruteforce(impl, n_groups=60, seed=1234):
    rng = np.random.default_rng(seed)
    near_ties = 0
    for idx, w in enumerate(_tiny_groups(rng, n_groups)):
        b = (1, 2, 4, 8)[idx % 4]
        L = (1 << b) - 1
        codes, s16, z, st = _q1(impl, w, b)
        assert st == 0
        S = Fraction(_f16(s16))
        W = [Fraction(float(v)) for v in w]
        # scale: within half an fp16 ulp (plus one binary32 rounding) of range/L, floored at 2^-14
        exact = (max(W) - min(W)) / L
        if exact >= Fraction(1, 2 ** 14):
            e = Fraction(2) ** (int(np.floor(np.log2(float(exact)))) - 10)
            assert abs(S - exact) <= e / 2 + exact / 2 ** 23, (float(S), float(exact))
        else:
            assert S == Fraction(1, 2 ** 14) or abs(S - exact) <= Fraction(1, 2 ** 24)
        # zero point: nearest integer to -wmin/S, clamped
        zt = -min(W) / S
        zr = int(np.floor(float(zt) + 0.5))
        if abs(zt - Fraction(2 * int(np.floor(float(zt))) + 1, 2)) > Fraction(1, 2 ** 20):
            assert z == min(max(zr, 0), L), (z, float(zt))
        # codes: exhaustive nearest level among the 2^b levels S*(j - z)
        for i, wi in enumerate(W):
            dists = [abs(wi - S * (j - z)) for j in range(L + 1)]
            best = min(dists)
            arg = [j for j in range(L + 1) if dists[j] == best]
            t = wi / S
            half = Fraction(2 * int(np.floor(float(t))) + 1, 2)
            if abs(t - half) <= abs(t) / 2 ** 22 + Fraction(1, 2 ** 40):
                near_ties += 1
                assert int(codes[i]) in (min(max(int(np.floor(float(t))) + z, 0), L),
                                         min(max(int(np.floor(float(t))) + 1 + z, 0), L))
                continue
            assert int(codes[i]) in arg, (b, i, float(wi), float(S), z, int(codes[i]), arg)
    return near_ties


def pin_quant_min_maps_to_zero(impl, seed=7):
    # rne(a) + rne(-a) = 0, so the group minimum lands on code 0 whenever z is not clamped.
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((64, GROUP)) * 0.02).astype(np.float32)
    codes, scale, zero, _ = impl.quantize(w, np.full(64, 4, np.uint8))
    codes = codes.reshape(64, GROUP)
    for g in range(64):
        sf = Fraction(_f16(scale[g]))
        zt = -Fraction(float(w[g].min())) / sf
        if 0 < zt < 15:
            assert codes[g, int(np.argmin(w[g]))] == 0


def pin_quant_reconstruction_error(impl, seed=11):
    # |w - s(q - z)| <= s/2 (+ binary32 rounding) for every code that is not clamped.
    rng = np.random.default_rng(seed)
    w = (rng.standard_t(5, (128, GROUP)) * 0.02).astype(np.float32)
    codes, scale, zero, _ = impl.quantize(w, np.full(128, 4, np.uint8))
    s = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64)[:, None]
    q = codes.reshape(128, GROUP).astype(np.float64)
    err = np.abs(w.astype(np.float64) - s * (q - zero[:, None]))
    inner = (q > 0) & (q < 15)
    assert (err[inner] <= s.repeat(GROUP, 1)[inner] * (0.5 + 2 ** -20)).all()


# ---- packed storage ------------------------------------------------------------------------

def pin_pack_lsb_first(impl):
    # b=2: codes 1,2,3,0 -> byte 0 = 1 | 2<<2 | 3<<4 | 0<<6 = 0x39;  b=1: 0,1,0,1.. -> 0xAA;
    # b=8: bytes are the codes; b=4: low nibble first.
    codes = np.zeros((4, GROUP), np.uint8)
    codes[0] = np.tile([0, 1], 32)
    codes[1, :4] = [1, 2, 3, 0]
    codes[2, :2] = [0xA, 0x5]
    codes[3] = np.arange(GROUP) * 3
    bits = np.array([1, 2, 4, 8], np.uint8)
    planes = impl.pack(codes.ravel(), bits)
    assert planes[0][:8].tolist() == [0xAA] * 8
    assert planes[1][0] == 0x39 and not planes[1][1:16].any()
    assert planes[2][0] == 0x5A and not planes[2][1:32].any()
    assert planes[3][:64].tolist() == (np.arange(GROUP) * 3).tolist()


def pin_pack_fixed4_is_plain_nibbles(impl, seed=3):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, 8 * 256, dtype=np.uint8)
    planes = impl.pack(codes, None)
    expect = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    assert np.array_equal(planes[2][:expect.size], expect)
    assert np.array_equal(impl.unpack(planes, codes.size // GROUP, None), codes)


def pin_pack_roundtrip_and_totals(impl, seed=5):
    rng = np.random.default_rng(seed)
    G = 777
    bits = rng.choice(np.array([1, 2, 4, 8], np.uint8), G, p=[0.69, 0.15, 0.12, 0.04])
    codes = (rng.integers(0, 256, G * GROUP) & ((1 << bits.repeat(GROUP).astype(np.int64)) - 1)).astype(np.uint8)
    off, pbytes = impl.varbits_index(bits)
    for slot, b in enumerate((1, 2, 4, 8)):
        sel = bits == b
        assert pbytes[slot] == 8 * b * int(sel.sum())
        o = np.sort(np.asarray(off)[sel].astype(np.int64))
        assert np.array_equal(o, 8 * b * np.arange(sel.sum()))
    planes = impl.pack(codes, bits)
    assert np.array_equal(impl.unpack(planes, G, bits), codes)


def pin_index_hand_example(impl):
    # Widths 2,1,2,4,1,2 worked by hand from the layout (offset = 8b x the number of earlier
    # groups of the same width, in row-major order): the 2-bit groups 0, 2, 5 are ranks 0, 1, 2
    # -> 0, 16, 32; the 1-bit groups 1, 4 -> 0, 8; the 4-bit group 3 -> 0.  Plane sizes: two
    # 1-bit groups (16 B), three 2-bit (48 B), one 4-bit (32 B), none at 8 bits.  A reversed or
    # column-major rank, or offsets in bits or codes instead of bytes, changes these numbers.
    bits = np.array([2, 1, 2, 4, 1, 2], np.uint8)
    off, pbytes = impl.varbits_index(bits)
    assert np.asarray(off).astype(np.int64).tolist() == [0, 0, 16, 0, 8, 32]
    assert [int(v) for v in pbytes] == [16, 48, 32, 0]
    # and pack puts each group's bytes there: constant codes give constant bytes
    # (2-bit 1 -> 0x55, 2 -> 0xAA, 3 -> 0xFF; 1-bit 1 -> 0xFF, alternating 0,1 -> 0xAA;
    # 4-bit 7 -> 0x77)
    codes = np.zeros((6, GROUP), np.uint8)
    codes[0], codes[1], codes[2], codes[3], codes[5] = 1, 1, 2, 7, 3
    codes[4] = np.tile([0, 1], 32)
    planes = impl.pack(codes.ravel(), bits)
    assert planes[0][:16].tolist() == [0xFF] * 8 + [0xAA] * 8
    assert planes[1][:48].tolist() == [0x55] * 16 + [0xAA] * 16 + [0xFF] * 16
    assert planes[2][:32].tolist() == [0x77] * 32


# ---- the CellFill invariants -------------------------------------------------------------------

def _random_artifact(rng, G, bits=None, subnormal_scales=False):
    b = np.full(G, 4, np.int64) if bits is None else np.asarray(bits, np.int64)
    L = (1 << b) - 1
    codes = (rng.integers(0, 256, (G, GROUP)) % (L[:, None] + 1)).astype(np.uint8)
    zero = (rng.integers(0, 256, G) % (L + 1)).astype(np.uint8)
    if subnormal_scales:
        scale = rng.integers(1, 0x7BFF, G).astype(np.uint16)      # every positive finite fp16
    else:
        scale = np.asarray(rng.uniform(1e-3, 1e-1, G), np.float16).view(np.uint16)
    return codes.ravel(), scale.astype(np.uint16), zero


def pin_roundtrip_dequant_requant(impl, seed=21):
    # W = s(q - z) is exact, and (s k)/s = k exactly: requantizing returns every code.
    rng = np.random.default_rng(seed)
    for bits in (None, rng.choice(np.array([1, 2, 4, 8], np.uint8), 300)):
        G = 300
        codes, scale, zero = _random_artifact(rng, G, bits, subnormal_scales=True)
        planes = impl.pack(codes, bits)
        m, fb, mask = impl.verify(planes, scale, zero, bits)
        assert m == 0 and fb == -1 and not mask.any()
        m, fb, _ = impl.verify(planes, scale, zero, bits, r=np.zeros(G * GROUP, np.float32))
        assert m == 0 and fb == -1


def _boundary_residuals(rng, scale):
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float32)
    G = sf.size
    mult = rng.uniform(-3, 3, (G, GROUP)).astype(np.float32)
    mult[:, 0] = 0.5
    mult[:, 1] = -0.5
    mult[:, 2] = 0.5 - 2 ** -10
    mult[:, 3] = 0.5 + 2 ** -10
    mult[:, 4] = 1e30
    mult[:, 5] = -1e30
    return (mult * sf[:, None]).astype(np.float32).ravel()


def pin_projected_residual_f32(impl, seed=31):
    rng = np.random.default_rng(seed)
    G = 400
    codes, scale, zero = _random_artifact(rng, G)
    planes = impl.pack(codes, None)
    r = _boundary_residuals(rng, scale)
    rp, n = impl.project_f32(r, scale)
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64).repeat(GROUP)
    bound = (0.5 - 2 ** -10) * sf
    assert (np.abs(rp.astype(np.float64)) <= bound).all()                    # drift bounded
    inside = np.abs(r.astype(np.float64)) <= bound
    assert np.array_equal(rp[inside].view(np.uint32), r[inside].view(np.uint32))
    assert n == int((~inside).sum())
    m, fb, _ = impl.verify(planes, scale, zero, None, r=rp)
    assert m == 0 and fb == -1
    m, fb, _ = impl.verify(planes, scale, zero, None)                         # revoke
    assert m == 0 and fb == -1


def pin_projected_residual_bf16(impl, seed=41):
    rng = np.random.default_rng(seed)
    G = 2000
    codes, scale, zero = _random_artifact(rng, G, subnormal_scales=False)
    scale = rng.integers(0x0400, 0x7800, G).astype(np.uint16)   # wide spread of fp16 mantissas
    planes = impl.pack(codes, None)
    r = _boundary_residuals(rng, scale)
    rb = (r.view(np.uint32) >> 16).astype(np.uint16)           # any bf16 values
    rp, n = impl.project_bf16(rb, scale)
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64).repeat(GROUP)
    rv = (rp.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (np.abs(rv) <= (0.5 - 2 ** -10) * sf).all()
    assert (np.abs(rv).reshape(G, GROUP).max(axis=1) >= 0.4952 * sf[::GROUP]).all()
    m, fb, _ = impl.verify(planes, scale, zero, None, r=rp, r_dtype="bf16")
    assert m == 0 and fb == -1


def _expected_mismatch(codes, scale, zero, bits, r_f64):
    """Exact-rational prediction of the requant decision, away from rounding ties."""
    G = scale.size
    b = np.full(G, 4, np.int64) if bits is None else np.asarray(bits, np.int64)
    L = ((1 << b) - 1).repeat(GROUP)
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64).repeat(GROUP)
    z = np.asarray(zero, np.int64).repeat(GROUP)
    q = np.asarray(codes, np.int64)
    t = (q - z) + r_f64 / sf                          # exact to ~1e-16 in binary64
    frac = t - np.floor(t)
    tie = np.abs(frac - 0.5) < 2 ** -12
    qp = np.clip(np.floor(t + 0.5).astype(np.int64) + z, 0, L)
    return qp != q, tie


def pin_negative_control(impl, seed=51):
    # unprojected residuals: the predicted count (exact arithmetic, far from ties) must match
    rng = np.random.default_rng(seed)
    for bits in (None, rng.choice(np.array([1, 2, 4, 8], np.uint8), 500)):
        G = 500
        codes, scale, zero = _random_artifact(rng, G, bits)
        planes = impl.pack(codes, bits)
        sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float32)
        u = rng.uniform(-0.6, 0.6, (G, GROUP)).astype(np.float32)
        for lim in (0.5, -0.5):
            near = np.abs(u - lim) < 1e-3
            u[near] = 0.0
        r = (u * sf[:, None]).astype(np.float32).ravel()
        bad, tie = _expected_mismatch(codes, scale, zero, bits, r.astype(np.float64))
        assert not tie.any()
        m, fb, mask = impl.verify(planes, scale, zero, bits, r=r)
        assert m == int(bad.sum()) and m > 0
        assert fb == int(np.argmax(bad))
        assert np.array_equal(mask, bad.reshape(G, GROUP).any(axis=1))


def pin_bad_scale_flags(impl):
    codes = np.full(4 * GROUP, 3, np.uint8)
    scale = np.array([0x0000, 0x7C00, 0x7E00, 0x3C00], np.uint16)   # 0, inf, NaN, 1.0
    zero = np.array([1, 1, 1, 1], np.uint8)
    planes = impl.pack(codes, None)
    m, fb, mask = impl.verify(planes, scale, zero, None)
    assert m == 3 * GROUP and fb == 0 and mask.tolist() == [True, True, True, False]


# ---- fp64 dequantize-and-multiply ------------------------------------------------------------

def pin_matmul(impl, seed=61):
    rng = np.random.default_rng(seed)
    rows, cols = 24, 192
    G = rows * cols // GROUP
    bits = rng.choice(np.array([1, 2, 4, 8], np.uint8), G)
    codes, scale, zero = _random_artifact(rng, G, bits)
    planes = impl.pack(codes, bits)
    r = rng.standard_normal(rows * cols).astype(np.float32) * 1e-3
    x = rng.standard_normal((3, cols)).astype(np.float32)
    y = impl.dequant_matmul_f64(planes, scale, zero, rows, cols, x, "f32", bits, r)
    # independent dense construction + BLAS
    sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64)
    W = (sf[:, None] * (codes.reshape(G, GROUP).astype(np.float64) - zero[:, None])).reshape(rows, cols)
    W = W + r.reshape(rows, cols)
    ref = x.astype(np.float64) @ W.T
    assert y.shape == (3, rows)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # closed forms: x = e_k picks column k of W; codes == zero gives exactly r.x
    for k in (0, 63, 64, cols - 1):
        e = np.zeros((1, cols), np.float32)
        e[0, k] = 1.0
        yk = impl.dequant_matmul_f64(planes, scale, zero, rows, cols, e, "f32", bits, r)
        assert np.array_equal(yk[0], W[:, k])
    flat = np.asarray(zero).repeat(GROUP).astype(np.uint8)
    planes0 = impl.pack(flat, bits)
    y0 = impl.dequant_matmul_f64(planes0, scale, zero, rows, cols, x, "f32", bits, r)
    assert np.allclose(y0, x.astype(np.float64) @ r.reshape(rows, cols).astype(np.float64).T,
                       rtol=1e-12, atol=1e-15)


# ---- RRQ: recurrent residual quantization ---------------------------------------------
# [RRQ] page 2 listing, "Recurrent Residual Quantization" abstract: a 2-bit round-to-nearest
# base plus 2-bit round-to-nearest residual corrections, stacked to 4, 6 and 8 bits.

def _rrq_stages(impl, w, n):
    out, r = [], np.asarray(w, np.float32)
    for _ in range(n):
        codes, scale, zero, st, r_new = impl.rrq_stage(r, 2)
        out.append((r, codes, scale, zero, st, r_new))
        r = r_new
    return out


def pin_rrq_residual_inside_half_step(impl, seed=71):
    """Round-to-nearest leaves every weight within half a grid step of its level: for a
    group whose values straddle zero (so the zero point is not clamped),
    |r'| <= s/2 + L |range/L - s| <= s (1/2 + 3 * 2^-11) for the fp16-rounded s. Each
    stage must therefore shrink the residual to about s/2 of that stage."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_t(5, (32, 512)) * 0.02).astype(np.float32)
    for j, (r, codes, scale, zero, st, r_new) in enumerate(_rrq_stages(impl, w, 4)):
        assert st == 0
        R = r.reshape(-1, GROUP).astype(np.float64)
        Rn = r_new.reshape(-1, GROUP).astype(np.float64)
        sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64)
        straddle = (R.min(axis=1) <= 0) & (R.max(axis=1) >= 0)
        assert straddle.mean() > 0.9, f"stage {j}: test data should straddle zero"
        lim = sf * (0.5 + 3 * 2.0 ** -11) * (1 + 2.0 ** -20)
        worst = (np.abs(Rn).max(axis=1) / lim)[straddle].max()
        assert worst <= 1.0, f"stage {j}: residual {worst:.4f} of the half-step bound"


def pin_rrq_telescopes(impl, seed=73):
    """The stages' dequantized values plus the final residual give back the weights up to
    one binary32 rounding per stage: |w - sum_j s_j(q_j - z_j) - r_J| <= sum_j 2^-24 |r_j|
    elementwise (each stage's subtraction is rounded once; the product is exact)."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((16, 256)) * 0.05).astype(np.float32)
    stages = _rrq_stages(impl, w, 4)
    total = np.zeros(w.size, np.float64)
    bound = np.zeros(w.size, np.float64)
    for r, codes, scale, zero, st, r_new in stages:
        G = codes.size // GROUP
        sf = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64)
        total += (sf[:, None] * (codes.reshape(G, GROUP).astype(np.float64) -
                                 np.asarray(zero, np.float64)[:, None])).ravel()
        bound += 2.0 ** -24 * np.abs(r_new.astype(np.float64).ravel())
    r_last = stages[-1][5].astype(np.float64).ravel()
    err = np.abs(w.astype(np.float64).ravel() - total - r_last)
    assert (err <= bound * (1 + 1e-9) + 1e-300).all(), f"max excess {np.max(err - bound):.3e}"
    # and the package converges: four 2-bit stages at least 3^3 times finer than the base
    assert np.abs(r_last).max() * 27 <= np.abs(stages[0][5]).max()


def pin_rrq_on_grid_is_exact(impl):
    """Weights already on a 2-bit grid: the base reproduces them, the residual is exactly
    zero, and the next stage sees a constant group (floored scale 2^-14, zero 0, codes 0)."""
    s = np.float32(2.0 ** -4)
    levels = np.array([-1, 0, 1, 2], np.float32) * s        # z = 1: codes 0..3
    w = np.tile(levels, 16).reshape(1, GROUP).astype(np.float32)
    codes, scale, zero, st, r = impl.rrq_stage(w, 2)
    assert st == 0 and int(scale[0]) == 0x2C00 and int(zero[0]) == 1
    assert np.array_equal(codes, np.tile(np.array([0, 1, 2, 3], np.uint8), 16))
    assert np.array_equal(r, np.zeros_like(w))
    codes1, scale1, zero1, st1, r1 = impl.rrq_stage(r, 2)
    assert int(scale1[0]) == 0x0400 and int(zero1[0]) == 0 and not codes1.any()
    assert np.array_equal(r1, r)


def pin_rrq_base_is_the_2bit_quantizer(impl, seed=75):
    """The first stage is the group quantizer at 2 bits (pinned above), and a flagged group
    (a NaN) keeps its residual unchanged."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((4, 256)) * 0.03).astype(np.float32)
    w[2, 70] = np.nan
    codes, scale, zero, st, r = impl.rrq_stage(w, 2)
    qc, qs, qz, qst = impl.quantize(w, np.full(w.size // GROUP, 2, np.uint8))
    assert np.array_equal(codes, qc) and np.array_equal(scale, qs) and np.array_equal(zero, qz)
    assert st == qst == 1
    g = (2 * 256 + 70) // GROUP
    assert np.array_equal(r.reshape(-1, GROUP)[g].view(np.uint32), w.reshape(-1, GROUP)[g].view(np.uint32))



# ---- bounded reparameterization of the residual ([CF] Abstract) -------------------------------

def _rn32(fr):
    """The binary32 nearest to the rational fr (ties to even), by exact comparison."""
    x = np.float32(float(fr))
    best = None
    for cand in (np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - fr)
        key = (d, int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return float(best[1])


def pin_reparam_closed_forms(impl):
    # theta = a/b with b a power of two and 1 + theta^2 a rational square (Pythagorean triples
    # 3-4-5, 8-15-17, 16-63-65, 32-255-257): every step before the division is exact, so
    # phi = RN32(a / c) exactly.
    for a, b, c in ((3, 4, 5), (15, 8, 17), (63, 16, 65), (255, 32, 257)):
        theta = a / b
        assert impl.reparam_phi(theta) == _rn32(Fraction(a, c)), (a, b, c)
        assert impl.reparam_phi(-theta) == -_rn32(Fraction(a, c)), (a, b, c)
    assert impl.reparam_phi(0.0) == 0.0
    assert impl.reparam_phi(np.inf) == 1.0 and impl.reparam_phi(-np.inf) == -1.0
    assert impl.reparam_phi(3e38) == 1.0 and impl.reparam_phi(-3e38) == -1.0
    assert impl.reparam_phi(np.nan) == 0.0
    # theta^2 underflows for a subnormal theta: 1 + 0 = 1, sqrt(1) = 1, phi = theta exactly
    tiny = float(np.float32(1e-40))
    assert impl.reparam_phi(tiny) == tiny


def _theta_sweep(rng, G):
    t = rng.uniform(-6, 6, (G, GROUP)).astype(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 3e38, -3e38, 2.0 ** 32, -(2.0 ** 33), 1e-40,
                         -1e-40, 1e-3, 40.0, -4096.0], np.float32)
    t[:, :specials.size] = specials
    return t.ravel()


def pin_reparam_stays_in_cell(impl, seed=81):
    # whatever theta is, the residual is one the (pinned) projection leaves unchanged, and the
    # artifact re-quantizes to its codes: the invariance needs no projection step
    rng = np.random.default_rng(seed)
    G = 300
    codes, scale, zero = _random_artifact(rng, G, subnormal_scales=True)
    planes = impl.pack(codes, None)
    theta = _theta_sweep(rng, G)
    for dt in ("f32", "bf16"):
        r = impl.reparam(theta, scale, dt)
        rp, n = (impl.project_bf16 if dt == "bf16" else impl.project_f32)(r.copy(), scale)
        assert n == 0 and np.array_equal(np.asarray(rp).view(np.uint8), np.asarray(r).view(np.uint8)), dt
        m, fb, _ = impl.verify(planes, scale, zero, r=r, r_dtype=dt)
        assert m == 0 and fb == -1, (dt, m)
        # NaN parameters revoke their weight's update: r = +0 exactly
        bits = np.asarray(r).view(np.uint16 if dt == "bf16" else np.uint32)
        assert not bits[np.isnan(theta)].any()
        # the bound is reached at the infinities: r = +-c_dt, c_dt being what projecting a huge
        # residual gives
        big = np.full(G * GROUP, 1e30, np.float32)
        if dt == "bf16":
            big = (big.view(np.uint32) >> 16).astype(np.uint16)
            cb, _ = impl.project_bf16(big, scale)
            cf = (cb.astype(np.uint32) << 16).view(np.float32)
            rf = (bits.astype(np.uint32) << 16).view(np.float32)
        else:
            cf, _ = impl.project_f32(big, scale)
            rf = np.asarray(r, np.float32)
        assert np.array_equal(rf[theta == np.inf], cf[theta == np.inf])
        assert np.array_equal(rf[theta == -np.inf], -cf[theta == -np.inf])
        assert (np.abs(rf) <= cf).all()


def pin_reparam_zero_revokes(impl, seed=83):
    # theta = 0 gives r = +0 everywhere: the served weights are the release's exactly
    rng = np.random.default_rng(seed)
    G, rows = 64, 16
    codes, scale, zero = _random_artifact(rng, G)
    planes = impl.pack(codes, None)
    cols = G * GROUP // rows
    x = rng.standard_normal((2, cols)).astype(np.float32)
    for dt in ("f32", "bf16"):
        r = impl.reparam(np.zeros(G * GROUP, np.float32), scale, dt)
        assert not np.asarray(r).view(np.uint8).any()
        y0 = impl.dequant_matmul_f64(planes, scale, zero, rows, cols, x)
        y1 = impl.dequant_matmul_f64(planes, scale, zero, rows, cols, x, r=r, r_dtype=dt)
        assert np.array_equal(y0, y1)


def pin_reparam_monotone_odd(impl, seed=85):
    rng = np.random.default_rng(seed)
    G = 40
    scale = np.full(G, 0x2E66, np.uint16)               # one scale: compare across the sweep
    theta = np.sort(rng.uniform(-50, 50, G * GROUP).astype(np.float32))
    for dt in ("f32", "bf16"):
        r = impl.reparam(theta, scale, dt)
        rf = ((np.asarray(r).astype(np.uint32) << 16).view(np.float32) if dt == "bf16" else np.asarray(r))
        # increasing up to the rounding of the steps (the rounded square root can make two
        # neighbouring quotients differ by an ulp the wrong way)
        ulp = np.abs(rf[1:]).astype(np.float64) * 2.0 ** -22
        assert (np.diff(rf.astype(np.float64)) >= -ulp).all(), dt
        assert rf[0] < 0 < rf[-1]
        rn = impl.reparam(-theta, scale, dt)
        rnf = ((np.asarray(rn).astype(np.uint32) << 16).view(np.float32) if dt == "bf16" else np.asarray(rn))
        assert np.array_equal(rnf, -rf), dt


def pin_reparam_gradient(impl, seed=87):
    # the backward pass against a central finite difference of the fp64 map c * t / sqrt(1 + t^2)
    # (c = the bound the projection gives), not against the oracle's own derivative formula
    rng = np.random.default_rng(seed)
    G = 50
    scale = np.asarray(rng.uniform(1e-3, 1e-1, G), np.float16).view(np.uint16)
    theta = rng.uniform(-4, 4, G * GROUP).astype(np.float32)
    g = rng.standard_normal(G * GROUP).astype(np.float32)
    for dt in ("f32", "bf16"):
        big = np.full(G * GROUP, 1e30, np.float32)
        if dt == "bf16":
            cb, _ = impl.project_bf16((big.view(np.uint32) >> 16).astype(np.uint16), scale)
            c = (cb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        else:
            c = impl.project_f32(big, scale)[0].astype(np.float64)
        t = theta.astype(np.float64)
        h = 1e-4
        f = lambda u: u / np.sqrt(1.0 + u * u)
        expect = g.astype(np.float64) * c * (f(t + h) - f(t - h)) / (2 * h)
        got = impl.reparam_grad(theta, scale, g, dt).astype(np.float64)
        assert np.allclose(got, expect, rtol=1e-5, atol=1e-12 * np.abs(c).max()), dt
    # no gradient through a saturated or NaN parameter
    sat = np.array([np.inf, -np.inf, np.nan, 1e30] + [0.5] * 60, np.float32)
    gs = impl.reparam_grad(sat, scale[:1], np.ones(64, np.float32), "f32")
    assert not gs[:4].any() and (gs[4:] > 0).all()



# ---- ReQuant fixed-grid refinement (page 1, ReQuant abstract) ---------------------------------

def _calibration(rng, n, K):
    """Synthetic calibration activations: N(0, 1) with a few outlier input channels (x10)."""
    X = rng.standard_normal((n, K))
    X[:, rng.choice(K, max(1, K // 32), replace=False)] *= 10.0
    return X


def _out_error(X, w, codes, scale, zero):
    """||X (w - s (q - z))^T||^2 per row, straight from the definition (NumPy BLAS, fp64)."""
    rows, cols = w.shape
    S = np.asarray(scale, np.uint16).view(np.float16).astype(np.float64).reshape(rows, -1).repeat(GROUP, 1)
    Z = np.asarray(zero, np.float64).reshape(rows, -1).repeat(GROUP, 1)
    D = w.astype(np.float64) - S * (np.asarray(codes, np.float64).reshape(rows, cols) - Z)
    return ((X @ D.T) ** 2).sum(axis=0)


def pin_requant_weight_space_is_rtn(impl, seed=91):
    # With H = I the error is the weight-space one, which round-to-nearest already minimizes:
    # from the RTN start nothing moves, and from codes pushed one level off the refinement
    # returns every code to the exact nearest level (brute force over the 16 levels in exact
    # rational arithmetic; a level exactly half-way keeps its code: only strict gains move).
    rng = np.random.default_rng(seed)
    rows, cols = 3, 128
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    # a hand-made exact tie: group scale 0.25, zero 8, w = 0.125 lies half-way between 0 and 0.25
    w[0, :64] = (0.25 * (np.arange(64) % 16) - 2.0).astype(np.float32)
    w[0, 3] = np.float32(0.125)
    codes, scale, zero, _ = impl.quantize(w)
    H = np.eye(cols)
    q, eb, ea, mv = impl.requant_refine(w, H, codes, scale, zero, 4, 1)
    assert not mv.any() and np.array_equal(q, codes)
    S = np.asarray(scale, np.uint16).view(np.float16).astype(np.float32)
    pushed = np.array(codes, np.int64).reshape(rows, cols)
    for n in range(rows):
        for k in range(cols):
            if rng.random() < 0.3 and (n, k) != (0, 3):
                pushed[n, k] += 1 if pushed[n, k] < 15 else -1
    q, eb, ea, mv = impl.requant_refine(w, H, pushed.astype(np.uint8).ravel(), scale, zero, 4, 1)
    q = q.reshape(rows, cols)
    for n in range(rows):
        for k in range(cols):
            g = n * (cols // GROUP) + k // GROUP
            sf, zz, wf = Fraction(float(S[g])), int(zero[g]), Fraction(float(w[n, k]))
            errs = [abs(wf - sf * (lv - zz)) for lv in range(16)]
            best = min(errs)
            assert errs[int(q[n, k])] == best, (n, k, int(q[n, k]), errs.index(best))
    assert int(q[0, 3]) == int(codes[3])          # the tie stays where round-to-nearest put it


def pin_requant_strictly_lowers_output_error(impl, seed=93):
    rng = np.random.default_rng(seed)
    rows, cols = 8, 192
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    codes, scale, zero, _ = impl.quantize(w)
    X = _calibration(rng, 300, cols)
    H = X.T @ X
    e0 = _out_error(X, w, codes, scale, zero)
    q, eb, ea, mv = impl.requant_refine(w, H, codes, scale, zero, 4, 2)
    e1 = _out_error(X, w, q, scale, zero)
    assert q.max() <= 15                              # still codes of the same 4-bit grid
    assert mv.sum() > 0
    assert (e1[mv > 0] < e0[mv > 0]).all() and np.array_equal(e1[mv == 0], e0[mv == 0])
    assert np.allclose(eb, e0, rtol=1e-9) and np.allclose(ea, e1, rtol=1e-9)
    # each sweep lowers it further or leaves it
    q1 = impl.requant_refine(w, H, codes, scale, zero, 4, 1)[0]
    assert (_out_error(X, w, q1, scale, zero) >= e1 - 1e-12 * e0).all()


def pin_requant_local_optimum(impl, seed=95):
    # swept until a sweep moves nothing, no single move to a neighbouring level lowers the
    # output error (checked move by move from the definition)
    rng = np.random.default_rng(seed)
    rows, cols = 2, 128
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    codes, scale, zero, _ = impl.quantize(w)
    X = _calibration(rng, 200, cols)
    H = X.T @ X
    q = codes
    for _ in range(40):
        q, _, _, mv = impl.requant_refine(w, H, q, scale, zero, 4, 1)
        if not mv.any():
            break
    assert not mv.any()
    e = _out_error(X, w, q, scale, zero)
    qq = np.array(q, np.int64).reshape(rows, cols)
    for n in range(rows):
        for k in range(cols):
            for step in (-1, 1):
                if 0 <= qq[n, k] + step <= 15:
                    t = qq.copy()
                    t[n, k] += step
                    e2 = _out_error(X, w, t.ravel(), scale, zero)
                    assert e2[n] >= e[n] * (1 - 1e-12), (n, k, step)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
