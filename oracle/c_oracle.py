"""ctypes binding of the C oracle ``cq_oracle.c`` (host arrays only).

TEST INFRASTRUCTURE -- see ``oracle/__init__.py``.  Every function takes and returns
NumPy arrays; nothing here touches a GPU.  The definitions, with their citations, are
in the C source.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p, i64, i32, u16 = C.c_void_p, C.c_int64, C.c_int, C.c_uint16
        L.oq_f32_to_f16.argtypes = [C.c_float]; L.oq_f32_to_f16.restype = u16
        L.oq_f16_to_f32.argtypes = [u16]; L.oq_f16_to_f32.restype = C.c_float
        L.oq_f32_to_bf16_rn.argtypes = [C.c_float]; L.oq_f32_to_bf16_rn.restype = u16
        L.oq_f32_to_bf16_rz.argtypes = [C.c_float]; L.oq_f32_to_bf16_rz.restype = u16
        for nm in ("oq_f32_to_f16_n", "oq_f16_to_f32_n", "oq_f32_to_bf16_rn_n", "oq_f32_to_bf16_rz_n"):
            getattr(L, nm).argtypes = [p, p, i64]
            getattr(L, nm).restype = None
        L.oq_quantize_group.argtypes = [p, i32, p, p, p]; L.oq_quantize_group.restype = C.c_uint32
        L.oq_quantize.argtypes = [p, i64, i64, p, p, p, p, p, i32]; L.oq_quantize.restype = i32
        L.oq_varbits_index.argtypes = [p, i64, p, p]; L.oq_varbits_index.restype = i32
        L.oq_rrq_stage.argtypes = [p, i64, i64, i32, p, p, p]; L.oq_rrq_stage.restype = C.c_uint32
        L.oq_pack.argtypes = [p, i64, p, p, p, p, p, p]; L.oq_pack.restype = i32
        L.oq_unpack.argtypes = [p, p, p, p, i64, p, p, p]; L.oq_unpack.restype = i32
        L.oq_project_f32.argtypes = [p, p, i64, p]; L.oq_project_f32.restype = i32
        L.oq_project_bf16.argtypes = [p, p, i64, p]; L.oq_project_bf16.restype = i32
        L.oq_verify.argtypes = [p, p, p, p, p, p, p, p, p, i32, i64, i64, p, p, p, i32]
        L.oq_verify.restype = i32
        L.oq_reparam_phi.argtypes = [C.c_float]; L.oq_reparam_phi.restype = C.c_float
        L.oq_reparam.argtypes = [p, p, i64, i32, p]; L.oq_reparam.restype = i32
        L.oq_reparam_grad.argtypes = [p, p, p, i64, i32, p]; L.oq_reparam_grad.restype = i32
        L.oq_requant_refine.argtypes = [p, i64, i64, p, p, p, i32, p, i32, p, p, p]
        L.oq_requant_refine.restype = i32
        L.oq_dequant_matmul_f64.argtypes = [p, p, p, p, p, p, p, p, p, i32, i64, i64, p, i32,
                                            i32, p, i32]
        L.oq_dequant_matmul_f64.restype = i32
        _lib = L
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: status {rc}")


# ---- number formats ---------------------------------------------------------------

def _conv(name, x, in_dtype, out_dtype):
    xs = np.ascontiguousarray(np.asarray(x, dtype=in_dtype).ravel())
    out = np.zeros(xs.size, out_dtype)
    getattr(lib(), name)(_ptr(xs), _ptr(out), xs.size)
    return out


def f32_to_f16_bits(x):
    return _conv("oq_f32_to_f16_n", x, np.float32, np.uint16)


def f16_bits_to_f32(h):
    return _conv("oq_f16_to_f32_n", h, np.uint16, np.float32)


def f32_to_bf16_rn_bits(x):
    return _conv("oq_f32_to_bf16_rn_n", x, np.float32, np.uint16)


def f32_to_bf16_rz_bits(x):
    return _conv("oq_f32_to_bf16_rz_n", x, np.float32, np.uint16)


# ---- quantize ---------------------------------------------------------------------

def quantize(w, bits=None, nthreads=None):
    """w: float32 [rows, cols] -> (codes u8 [rows*cols], scale fp16 bits u16 [G], zero u8 [G], status)."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    G = rows * (cols // 64)
    bits = _c(bits, np.uint8)
    codes = np.zeros(rows * cols, np.uint8)
    scale = np.zeros(G, np.uint16)
    zero = np.zeros(G, np.uint8)
    st = np.zeros(1, np.uint32)
    _check(lib().oq_quantize(_ptr(w), rows, cols, _ptr(bits), _ptr(codes), _ptr(scale), _ptr(zero),
                             _ptr(st), nthreads or default_threads()), "oq_quantize")
    return codes, scale, zero, int(st[0])


def rrq_stage(r, b=2):
    """One RRQ stage (see oq_rrq_stage): r float32 [rows, cols] -> (codes u8 [rows*cols],
    scale u16 [G], zero u8 [G], status, new residual float32 [rows, cols])."""
    r = np.array(r, dtype=np.float32, order="C", copy=True)
    rows, cols = r.shape
    G = rows * (cols // 64)
    codes = np.zeros(rows * cols, np.uint8)
    scale = np.zeros(G, np.uint16)
    zero = np.zeros(G, np.uint8)
    st = lib().oq_rrq_stage(_ptr(r), rows, cols, int(b), _ptr(codes), _ptr(scale), _ptr(zero))
    return codes, scale, zero, int(st), r


def rrq_build(w, stages, b=2):
    """The RRQ package: `stages` stages of width b from w -> list of (codes, scale, zero,
    status) and the final residual."""
    out = []
    r = np.asarray(w, np.float32)
    for _ in range(stages):
        codes, scale, zero, st, r = rrq_stage(r, b)
        out.append((codes, scale, zero, st))
    return out, r


def quantize_group(w64, b):
    w64 = _c(w64, np.float32)
    assert w64.size == 64
    q = np.zeros(64, np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint8)
    st = lib().oq_quantize_group(_ptr(w64), int(b), _ptr(q), _ptr(s), _ptr(z))
    return q, int(s[0]), int(z[0]), int(st)


# ---- packed storage ---------------------------------------------------------------

def varbits_index(bits):
    bits = _c(bits, np.uint8)
    G = bits.size
    off = np.zeros(G, np.uint32)
    pb = np.zeros(4, np.uint64)
    _check(lib().oq_varbits_index(_ptr(bits), G, _ptr(off), _ptr(pb)), "oq_varbits_index")
    return off, [int(v) for v in pb]


def _planes_alloc(bits, G, plane_bytes):
    if bits is None:
        return [np.zeros(1, np.uint8), np.zeros(1, np.uint8), np.zeros(32 * G, np.uint8),
                np.zeros(1, np.uint8)]
    return [np.zeros(max(1, n), np.uint8) for n in plane_bytes]


def pack(codes, bits=None, offset=None, plane_bytes=None):
    """codes u8 [G*64] -> list of 4 planes (b = 1, 2, 4, 8)."""
    codes = _c(codes, np.uint8)
    G = codes.size // 64
    bits = _c(bits, np.uint8)
    offset = _c(offset, np.uint32)
    planes = _planes_alloc(bits, G, plane_bytes)
    _check(lib().oq_pack(_ptr(codes), G, _ptr(bits), _ptr(offset), *[_ptr(p) for p in planes]),
           "oq_pack")
    return planes


def unpack(planes, G, bits=None, offset=None):
    bits = _c(bits, np.uint8)
    offset = _c(offset, np.uint32)
    planes = [_c(p, np.uint8) for p in planes]
    codes = np.zeros(G * 64, np.uint8)
    _check(lib().oq_unpack(*[_ptr(p) for p in planes], G, _ptr(bits), _ptr(offset), _ptr(codes)),
           "oq_unpack")
    return codes


# ---- residual projection ----------------------------------------------------------

def project_f32(r, scale):
    r = np.array(r, dtype=np.float32, copy=True).ravel()
    scale = _c(scale, np.uint16)
    n = np.zeros(1, np.uint64)
    _check(lib().oq_project_f32(_ptr(r), _ptr(scale), r.size, _ptr(n)), "oq_project_f32")
    return r, int(n[0])


def project_bf16(r_bits, scale):
    r = np.array(r_bits, dtype=np.uint16, copy=True).ravel()
    scale = _c(scale, np.uint16)
    n = np.zeros(1, np.uint64)
    _check(lib().oq_project_bf16(_ptr(r), _ptr(scale), r.size, _ptr(n)), "oq_project_bf16")
    return r, int(n[0])


# ---- bounded reparameterization of the residual ---------------------------------------

def reparam_phi(theta):
    """phi(theta) = theta / sqrt(1 + theta^2) in binary32, step by step (scalar)."""
    return float(np.float32(lib().oq_reparam_phi(float(np.float32(theta)))))


def reparam(theta, scale, r_dtype="bf16"):
    """theta f32 [n] -> r = RN(c_dt * phi(theta)): f32 [n], or bf16 bit patterns u16 [n]."""
    theta = _c(theta, np.float32)
    scale = _c(scale, np.uint16)
    assert theta.size == scale.size * 64
    rd = 1 if r_dtype == "bf16" else 0
    r = np.zeros(theta.size, np.uint16 if rd else np.float32)
    _check(lib().oq_reparam(_ptr(theta), _ptr(scale), theta.size, rd, _ptr(r)), "oq_reparam")
    return r


def reparam_grad(theta, scale, grad_r, r_dtype="bf16"):
    """dL/dtheta [n] f32 from dL/dr [n] f32 (straight through the final rounding)."""
    theta = _c(theta, np.float32)
    scale = _c(scale, np.uint16)
    grad_r = _c(grad_r, np.float32)
    rd = 1 if r_dtype == "bf16" else 0
    g = np.zeros(theta.size, np.float32)
    _check(lib().oq_reparam_grad(_ptr(theta), _ptr(scale), _ptr(grad_r), theta.size, rd, _ptr(g)),
           "oq_reparam_grad")
    return g


# ---- ReQuant fixed-grid refinement --------------------------------------------------------

def requant_refine(w, H, codes, scale, zero, b=4, sweeps=1):
    """Refine codes (u8 [rows*cols], not modified) on the frozen grid against H = X^T X (fp64
    [cols, cols]) -> (codes, err_before [rows], err_after [rows], moves [rows])."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    H = _c(H, np.float64)
    assert H.shape == (cols, cols)
    q = np.array(codes, np.uint8, copy=True).reshape(-1)
    scale = _c(scale, np.uint16)
    zero = _c(zero, np.uint8)
    eb = np.zeros(rows, np.float64)
    ea = np.zeros(rows, np.float64)
    mv = np.zeros(rows, np.uint64)
    _check(lib().oq_requant_refine(_ptr(w), rows, cols, _ptr(H), _ptr(scale), _ptr(zero), int(b), _ptr(q),
                                   int(sweeps), _ptr(eb), _ptr(ea), _ptr(mv)), "oq_requant_refine")
    return q, eb, ea, mv


# ---- requant verify -----------------------------------------------------------------

def verify(planes, scale, zero, bits=None, offset=None, r=None, r_dtype="f32", first_w=0,
           n_w=None, want_flags=False, nthreads=None):
    """Returns (mismatches, first_bad, group_flags or None)."""
    planes = [_c(p, np.uint8) for p in planes]
    scale = _c(scale, np.uint16)
    zero = _c(zero, np.uint8)
    bits = _c(bits, np.uint8)
    offset = _c(offset, np.uint32)
    if n_w is None:
        n_w = scale.size * 64 - first_w
    rd = 1 if r_dtype == "bf16" else 0
    if r is not None:
        r = _c(r, np.uint16 if rd == 1 else np.float32)
    ng = (n_w + 63) // 64
    flags = np.zeros(max(1, (ng + 31) // 32), np.uint32) if want_flags else None
    mism = np.zeros(1, np.uint64)
    fb = np.zeros(1, np.int64)
    _check(lib().oq_verify(_ptr(bits), _ptr(offset), *[_ptr(p) for p in planes], _ptr(scale),
                           _ptr(zero), _ptr(r), rd, first_w, n_w, _ptr(mism), _ptr(fb),
                           _ptr(flags), nthreads or default_threads()), "oq_verify")
    return int(mism[0]), int(fb[0]), flags


# ---- fp64 matmul reference --------------------------------------------------------------

def dequant_matmul_f64(planes, scale, zero, rows, cols, x, x_dtype="f32", bits=None, offset=None,
                       r=None, r_dtype="f32", nthreads=None):
    """y [m, rows] float64 = sum_k (s (q - z) + r) x.  x: [m, cols] f32, or u16 bf16 bits."""
    planes = [_c(p, np.uint8) for p in planes]
    scale = _c(scale, np.uint16)
    zero = _c(zero, np.uint8)
    bits = _c(bits, np.uint8)
    offset = _c(offset, np.uint32)
    xd = 1 if x_dtype == "bf16" else 0
    x = _c(x, np.uint16 if xd else np.float32)
    m = x.shape[0] if x.ndim == 2 else 1
    rd = 1 if r_dtype == "bf16" else 0
    if r is not None:
        r = _c(r, np.uint16 if rd else np.float32)
    y = np.zeros((m, rows), np.float64)
    _check(lib().oq_dequant_matmul_f64(_ptr(bits), _ptr(offset), *[_ptr(p) for p in planes],
                                       _ptr(scale), _ptr(zero), _ptr(r), rd, rows, cols, _ptr(x), xd,
                                       m, _ptr(y), nthreads or default_threads()),
           "oq_dequant_matmul_f64")
    return y
