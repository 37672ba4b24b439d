"""NumPy twin of the oracle, for small inputs.

TEST INFRASTRUCTURE -- see ``oracle/__init__.py``.  This is a second, independent
implementation of the definitions in ``cq_oracle.c``: vectorised binary32 arithmetic
(NumPy rounds every float32 ``+ - * /`` to nearest even and ``np.rint`` rounds half to
even), NumPy's own float16 conversion, and ``np.packbits(bitorder="little")`` for the
bit-plane layout.  It never calls the C oracle.

Sources (cited by page title and section):
  [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
        Without Changing the File They Ship", abstract: groups of 64 weights, per-group
        width from {1,2,4,8}, bit-packed storage, fused dequantize-and-multiply.
  [CF]  "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
        Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: frozen 4-bit codes
        and scales, residual confined to its rounding cell, exact re-quantization,
        revocation by dropping the residual, bounded drift.
  [SLQ] page 2 listing, SLQ abstract: asymmetric quantization.
  [RRQ] page 2 listing (thelatestinai.com/papers/2512.18934), "Recurrent Residual
        Quantization" abstract: a 2-bit round-to-nearest base and 2-bit round-to-nearest
        residual corrections stacked to 4, 6 and 8 bits.
"""
import numpy as np

GROUP = 64
ST_NONFINITE, ST_RANGE, ST_BADBITS = 1, 2, 4
WIDTHS = (1, 2, 4, 8)
CELL = np.float32(0.5 - 2.0 ** -10)   # [CF] inside the rounding cell with a 2^-10 margin
SMIN = np.float32(2.0 ** -14)         # smallest normal fp16: floor of the scale


def _f16_to_f32(s_bits):
    return np.asarray(s_bits, np.uint16).view(np.float16).astype(np.float32)


def _bf16_to_f32(b_bits):
    return (np.asarray(b_bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _clamp_code(v, L):
    """Integer clamp of a rounded value held as float32 (see the C oracle)."""
    return np.where(v < 0, np.float32(0), np.where(v > L, L, v))


# The individual steps of the definitions, named so that a reader can match each one to
# its reading, and so that the test suite can plant a single mistake in one of them.

def _rne(x):
    """round half to even (binary32 in, binary32 out)"""
    return np.rint(x)


def _scale_divisor(b):
    """s = range / (2^b - 1): the min-max grid spans the range with 2^b levels"""
    return ((1 << b) - 1).astype(np.float32)


def _zero_point(wmin, sf, L):
    return _clamp_code(_rne(-wmin / sf), L)


def _cell_halfwidth_f32(sf):
    """(0.5 - 2^-10) * s: the cell half-width less a 2^-10 margin"""
    return CELL * sf


def _bf16_bound(c):
    """bound of a bf16 residual: c rounded toward zero to bf16, so it never exceeds c"""
    return _bf16_to_f32((c.view(np.uint32) >> 16).astype(np.uint16))


def _served_weight(sf, k, r):
    """w' = RN32(RN32(s * k) + r); r is None after revocation"""
    wp = sf * k
    return wp if r is None else wp + r


def _dequant_f64(s, q, z):
    return s * (q - z)


_BIT_ORDER = "little"   # code j of a group in bits [j*b, (j+1)*b), least significant first


# ---- quantize ([SLQ] asymmetric min-max RTN, [CF] codes + scales, [VBQ] widths) ----

def quantize(w, bits=None):
    w = np.asarray(w, np.float32)
    rows, cols = w.shape
    G = rows * (cols // GROUP)
    W = w.reshape(G, GROUP)
    b = np.full(G, 4, np.int64) if bits is None else np.asarray(bits, np.int64)
    badbits = ~np.isin(b, WIDTHS)
    bb = np.where(badbits, 4, b)
    L = ((1 << bb) - 1).astype(np.float32)
    finite = np.isfinite(W).all(axis=1)
    with np.errstate(all="ignore"):
        Wf = np.where(finite[:, None], W, np.float32(0))
        wmin = Wf.min(axis=1)
        wmax = Wf.max(axis=1)
        s32 = (wmax - wmin) / _scale_divisor(bb)
        s16 = s32.astype(np.float16)
        sf = s16.astype(np.float32)
        overflow = np.isinf(sf)
        tiny = sf < SMIN
        s16 = np.where(tiny, np.float16(SMIN), s16)
        sf = np.where(tiny, SMIN, sf)
        z = _zero_point(wmin, sf, L)
        q = _clamp_code(_rne(Wf / sf[:, None]) + z[:, None], L[:, None])
    bad = badbits | ~finite | overflow
    status = 0
    if badbits.any():
        status |= ST_BADBITS
    if (~finite & ~badbits).any():
        status |= ST_NONFINITE
    if (overflow & finite & ~badbits).any():
        status |= ST_RANGE
    codes = np.where(bad[:, None], 0, q).astype(np.uint8).ravel()
    scale = np.where(bad, np.uint16(0), s16.view(np.uint16)).astype(np.uint16)
    zero = np.where(bad, 0, z).astype(np.uint8)
    return codes, scale, zero, status


def rrq_stage(r, b=2):
    """[RRQ] one stage: quantize the running residual at width b for every group, then
    r <- RN32(r - s*(q - z)) with the stored s, z, q (s*(q - z) is exact in binary32;
    a flagged group, s = +0, keeps its residual). Returns (codes, scale, zero, status, r')."""
    r = np.asarray(r, np.float32)
    rows, cols = r.shape
    G = rows * (cols // GROUP)
    codes, scale, zero, status = quantize(r, np.full(G, b, np.uint8))
    sf = _f16_to_f32(scale)
    deq = sf[:, None] * (codes.reshape(G, GROUP).astype(np.float32) - zero.astype(np.float32)[:, None])
    with np.errstate(invalid="ignore"):
        r_new = _rrq_residual(r.reshape(G, GROUP), deq).astype(np.float32).reshape(rows, cols)
    return codes, scale, zero, status, r_new


def _rrq_residual(r, deq):
    """what the stage does not represent: RN32(r - s*(q - z))"""
    return r - deq


# ---- packed storage ([VBQ]: per-group widths stored bit-packed) ----------------------

def _width_rank(sel):
    """Number of earlier groups (row-major group order) that have the same width."""
    return np.cumsum(sel) - sel


def varbits_index(bits):
    bits = np.asarray(bits, np.int64)
    off = np.zeros(bits.size, np.uint64)
    plane_bytes = []
    for b in WIDTHS:
        sel = bits == b
        rank = _width_rank(sel)
        off[sel] = (rank[sel] * 8 * b).astype(np.uint64)
        plane_bytes.append(int(sel.sum()) * 8 * b)
    return off.astype(np.uint32), plane_bytes


def _group_bits(codes_g, b):
    """(n, 64) codes -> (n, 8b) bytes, code j in bits [j*b, (j+1)*b), LSB first."""
    bitmat = ((codes_g[:, :, None].astype(np.uint16) >> np.arange(b)) & 1).astype(np.uint8)
    return np.packbits(bitmat.reshape(codes_g.shape[0], GROUP * b), axis=1, bitorder=_BIT_ORDER)


def _group_codes(bytes_g, b):
    bitmat = np.unpackbits(bytes_g, axis=1, bitorder=_BIT_ORDER).reshape(-1, GROUP, b)
    return (bitmat.astype(np.uint16) << np.arange(b)).sum(axis=2).astype(np.uint8)


def pack(codes, bits=None):
    codes = np.asarray(codes, np.uint8).reshape(-1, GROUP)
    if bits is None:
        return [np.zeros(1, np.uint8), np.zeros(1, np.uint8), _group_bits(codes, 4).ravel(),
                np.zeros(1, np.uint8)]
    bits = np.asarray(bits, np.int64)
    planes = []
    for b in WIDTHS:
        sel = bits == b
        p = _group_bits(codes[sel], b).ravel() if sel.any() else np.zeros(0, np.uint8)
        planes.append(p if p.size else np.zeros(1, np.uint8))
    return planes


def unpack(planes, G, bits=None):
    if bits is None:
        return _group_codes(np.asarray(planes[2][:32 * G], np.uint8).reshape(G, 32), 4).ravel()
    bits = np.asarray(bits, np.int64)
    codes = np.zeros((G, GROUP), np.uint8)
    for slot, b in enumerate(WIDTHS):
        sel = bits == b
        n = int(sel.sum())
        if n:
            codes[sel] = _group_codes(np.asarray(planes[slot][:n * 8 * b]).reshape(n, 8 * b), b)
    return codes.ravel()


def _codes_and_width(planes, G, bits):
    codes = unpack(planes, G, bits).reshape(G, GROUP)
    b = np.full(G, 4, np.int64) if bits is None else np.asarray(bits, np.int64)
    return codes, b


# ---- projection into the cell ([CF]) ---------------------------------------------------

def _halfwidth(scale):
    return _cell_halfwidth_f32(_f16_to_f32(scale))


def project_f32(r, scale):
    r = np.asarray(r, np.float32).reshape(-1, GROUP)
    c = _halfwidth(scale)[:, None]
    out = np.where(r > c, c, np.where(r < -c, -c, r)).astype(np.float32)
    changed = int((out.view(np.uint32) != r.view(np.uint32)).sum())
    return out.ravel(), changed


def project_bf16(r_bits, scale):
    rb = np.asarray(r_bits, np.uint16).reshape(-1, GROUP)
    c = _halfwidth(scale)
    cb = _bf16_bound(c)[:, None]
    r = _bf16_to_f32(rb)
    out = np.where(r > cb, cb, np.where(r < -cb, -cb, r)).astype(np.float32)
    ob = (out.view(np.uint32) >> 16).astype(np.uint16)
    return ob.ravel(), int((ob != rb).sum())


# ---- bounded reparameterization ([CF] Abstract: the bounded-reparameterization form) -----
# r = RN(c_dt * phi(theta)), phi(theta) = theta / sqrt(1 + theta^2) step by step in binary32
# (see the C oracle for the reading); NaN -> 0, |theta| > 2^32 -> sign(theta).
_SAT = np.float32(2.0 ** 32)


def _reparam_phi(theta):
    t = np.asarray(theta, np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        d = np.float32(1) + t * t
        phi = t / np.sqrt(d)
    phi = np.where(t > _SAT, np.float32(1), np.where(t < -_SAT, np.float32(-1), phi))
    return np.where(np.isnan(t), np.float32(0), phi).astype(np.float32)


def _reparam_dphi(theta):
    t = np.asarray(theta, np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        d = np.float32(1) + t * t
        dphi = (np.float32(1) / d) / np.sqrt(d)
    dead = np.isnan(t) | (np.abs(t) > _SAT)
    return np.where(dead, np.float32(0), dphi).astype(np.float32)


def _reparam_bound(scale, r_dtype):
    c = _halfwidth(scale)
    return _bf16_bound(c) if r_dtype == "bf16" else c


def _f32_to_bf16_rn(v):
    """Finite binary32 -> bf16 bits, round to nearest, ties to even."""
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def reparam(theta, scale, r_dtype="bf16"):
    t = np.asarray(theta, np.float32).reshape(-1, GROUP)
    c = _reparam_bound(scale, r_dtype)[:, None]
    v = (c * _reparam_phi(t)).astype(np.float32).ravel()
    return _f32_to_bf16_rn(v) if r_dtype == "bf16" else v


def reparam_grad(theta, scale, grad_r, r_dtype="bf16"):
    t = np.asarray(theta, np.float32).reshape(-1, GROUP)
    c = _reparam_bound(scale, r_dtype)[:, None]
    gc = np.asarray(grad_r, np.float32).reshape(-1, GROUP) * c
    return (gc * _reparam_dphi(t)).astype(np.float32).ravel()


# ---- ReQuant fixed-grid refinement (page 1, ReQuant abstract) --------------------------------
# Output reconstruction error E = sum_n d_n^T H d_n, H = X^T X; one sweep visits the row's codes
# in order and moves a code to a neighbouring level when that strictly lowers E (see the C
# oracle for the reading and the order of the binary64 operations).

def _rq_gradient(H, d):
    """g = H d with the sum over k in increasing order (vectorised over j, sequential over k)."""
    g = np.zeros(d.size, np.float64)
    for k in range(d.size):
        g = g + H[:, k] * d[k]
    return g


def _rq_error(d, g):
    e = np.float64(0.0)
    for k in range(d.size):
        e = e + d[k] * g[k]
    return float(e)


def _rq_changes(sk, hkk, gk):
    """The change of E for a move up (+s) and down (-s): (s s) H_kk -+ (2 s) g_k."""
    t2 = (sk * sk) * hkk
    t4 = (2.0 * sk) * gk
    return t2 - t4, t2 + t4


def _rq_update(g, delta, hk):
    """g <- g - delta * H[:, k] after a move of delta."""
    return g - delta * hk


def _rq_accept(up, down, q, L):
    """The move taken: +1, -1 or 0 (a strictly negative change only; up on a tie)."""
    step = 1 if (q < L and up < 0.0) else 0
    if q > 0 and down < 0.0 and (step == 0 or down < up):
        step = -1
    return step


def requant_refine(w, H, codes, scale, zero, b=4, sweeps=1):
    w = np.asarray(w, np.float32)
    rows, cols = w.shape
    H = np.asarray(H, np.float64)
    q = np.array(codes, np.uint8, copy=True).reshape(rows, cols)
    S = _f16_to_f32(scale).astype(np.float64).reshape(rows, -1).repeat(GROUP, axis=1)
    Z = np.asarray(zero, np.int64).reshape(rows, -1).repeat(GROUP, axis=1)
    L = (1 << b) - 1
    eb, ea, mv = np.zeros(rows), np.zeros(rows), np.zeros(rows, np.uint64)
    diag = np.diagonal(H).copy()
    for n in range(rows):
        d = w[n].astype(np.float64) - S[n] * (q[n].astype(np.int64) - Z[n]).astype(np.float64)
        g = _rq_gradient(H, d)
        eb[n] = _rq_error(d, g)
        for _ in range(sweeps):
            for k in range(cols):
                sk = S[n, k]
                up, down = _rq_changes(sk, diag[k], g[k])
                step = _rq_accept(up, down, int(q[n, k]), L)
                if step:
                    q[n, k] = int(q[n, k]) + step
                    g = _rq_update(g, sk if step > 0 else -sk, H[:, k])
                    mv[n] += 1
        d = w[n].astype(np.float64) - S[n] * (q[n].astype(np.int64) - Z[n]).astype(np.float64)
        ea[n] = _rq_error(d, _rq_gradient(H, d))
    return q.ravel(), eb, ea, mv


# ---- requant verify ([CF]: bit-identical re-quantization, exact revocation) -------------

def verify(planes, scale, zero, bits=None, r=None, r_dtype="f32"):
    """Whole-artifact check: returns (mismatches, first_bad, per-group mismatch mask)."""
    G = np.asarray(scale).size
    codes, b = _codes_and_width(planes, G, bits)
    L = ((1 << b) - 1).astype(np.float32)[:, None]
    sf = _f16_to_f32(scale)[:, None]
    z = np.asarray(zero).astype(np.float32)[:, None]
    k = codes.astype(np.float32) - z
    rf = None
    if r is not None:
        rf = _bf16_to_f32(r) if r_dtype == "bf16" else np.asarray(r, np.float32)
        rf = rf.reshape(G, GROUP)
    with np.errstate(all="ignore"):
        t = _served_weight(sf, k, rf) / sf
        qp = _clamp_code(_rne(t) + z, L)
    bad = np.isnan(t) | (qp != codes.astype(np.float32))
    flat = bad.ravel()
    first = int(np.argmax(flat)) if flat.any() else -1
    return int(flat.sum()), first, bad.any(axis=1)


# ---- fp64 dequantize-and-multiply ([VBQ] fused dequantize-and-multiply) -----------------

def dequantize_f64(planes, scale, zero, rows, cols, bits=None, r=None, r_dtype="f32"):
    G = rows * (cols // GROUP)
    codes, _ = _codes_and_width(planes, G, bits)
    s = _f16_to_f32(scale).astype(np.float64)[:, None]
    W = _dequant_f64(s, codes.astype(np.float64), np.asarray(zero, np.float64)[:, None])
    if r is not None:
        rf = _bf16_to_f32(r) if r_dtype == "bf16" else np.asarray(r, np.float32)
        W = W + rf.astype(np.float64).reshape(G, GROUP)
    return W.reshape(rows, cols)


def dequant_matmul_f64(planes, scale, zero, rows, cols, x, x_dtype="f32", bits=None, r=None,
                       r_dtype="f32"):
    W = dequantize_f64(planes, scale, zero, rows, cols, bits, r, r_dtype)
    xf = _bf16_to_f32(x) if x_dtype == "bf16" else np.asarray(x, np.float32)
    xf = xf.reshape(-1, cols).astype(np.float64)
    return xf @ W.T
