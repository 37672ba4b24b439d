"""Python binding of libcq (include/cq.h): argument marshalling only.

Every function has the name of its C entry point and takes torch tensors that live on the
current CUDA device; outputs are caller-allocated, as in C.  The work is enqueued on the
current torch stream (or an explicit ``stream``).  Nothing here computes: if ``libcq.so``
is missing or a call returns a non-zero status, a ``CQError`` is raised -- there is no
fallback implementation.
"""
import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIBCQ_PATH = os.path.join(HERE, "libcq.so")
LIBSYNTH_PATH = os.path.join(HERE, "libcq_synth.so")

CQ_F32, CQ_BF16 = 0, 1
STATUS = ["CQ_OK", "CQ_ERR_ARG", "CQ_ERR_SHAPE", "CQ_ERR_BITS", "CQ_ERR_ALIGN", "CQ_ERR_NONFINITE",
          "CQ_ERR_RANGE", "CQ_ERR_CUDA", "CQ_ERR_UNSUPPORTED"]
QSTATUS_NONFINITE, QSTATUS_RANGE, QSTATUS_BADBITS, QSTATUS_TIMEOUT = 1, 2, 4, 8

# every symbol include/cq.h declares
EXPORTS = ["cq_quantize", "cq_varbits_index", "cq_pack_varbits", "cq_unpack_varbits",
           "cq_project_residual", "cq_requant_verify", "cq_dequant_gemv", "cq_dequant_gemv_multi", "cq_dequant_gemm",
           "cq_dequant_gemm_static", "cq_gemm_workspace", "cq_last_error", "cq_status_string", "cq_rrq_stage",
           "cq_dequant_gemv_stages", "cq_requant_verify_pair", "cq_reparam_residual", "cq_reparam_residual_grad", "cq_requant_refine",
           "cq_requant_workspace", "cq_debug_word", "cq_debug_selftest"]
SYNTH_EXPORTS = ["cqs_normal_f32", "cqs_code_words", "cqs_scales", "cqs_zeros", "cqs_residual_bf16"]


class CQError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS[status] if 0 <= status < len(STATUS) else status}: {msg}")
        self.status = status


class cq_qweight(C.Structure):
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64), ("bits", C.c_void_p), ("offset", C.c_void_p),
                ("plane", C.c_void_p * 4), ("scale", C.c_void_p), ("zero", C.c_void_p),
                ("residual", C.c_void_p), ("residual_dtype", C.c_int)]


_lib = None
_synth = None


def lib():
    """Load libcq.so (built in-tree by cell_updates_b200/build.py); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBCQ_PATH):
            raise CQError(8, f"{LIBCQ_PATH} is missing: run cell_updates_b200/build.py (no fallback exists)")
        L = C.CDLL(LIBCQ_PATH)
        p, i64, i32 = C.c_void_p, C.c_int64, C.c_int
        L.cq_quantize.argtypes = [p, i64, i64, p, p, p, p, p, p]
        L.cq_varbits_index.argtypes = [p, i64, p, p, p]
        L.cq_pack_varbits.argtypes = [p, i64, p, p, p, p]
        L.cq_unpack_varbits.argtypes = [p, p, p]
        L.cq_project_residual.argtypes = [p, i32, p, i64, p, p]
        L.cq_requant_verify.argtypes = [p, i64, i64, p, p, p, p]
        L.cq_dequant_gemv.argtypes = [p, p, i32, i32, p, p]
        L.cq_dequant_gemv_multi.argtypes = [p, i32, p, i32, i32, p, p]
        L.cq_dequant_gemm.argtypes = [p, p, i32, i32, p, p, C.c_size_t, p]
        L.cq_dequant_gemm_static.argtypes = [p, p, i32, i32, p, p, p]
        L.cq_rrq_stage.argtypes = [p, i64, i64, i32, p, p, p, p, p]
        L.cq_requant_verify_pair.argtypes = [p, i64, i64, p, p, p, p, p, p]
        L.cq_dequant_gemv_stages.argtypes = [p, i32, p, i32, i32, p, p]
        L.cq_reparam_residual.argtypes = [p, p, i64, p, i32, p]
        L.cq_reparam_residual_grad.argtypes = [p, p, p, i64, i32, p, p]
        L.cq_requant_refine.argtypes = [p, i64, i64, p, p, p, i32, p, i32, p, p, p, p, C.c_size_t, p]
        L.cq_requant_workspace.argtypes = [i64, i64]
        L.cq_requant_workspace.restype = C.c_size_t
        L.cq_debug_word.argtypes = [p]
        L.cq_debug_selftest.argtypes = [p]
        L.cq_gemm_workspace.argtypes = [i64, i64, i32]
        L.cq_gemm_workspace.restype = C.c_size_t
        L.cq_last_error.restype = C.c_char_p
        L.cq_status_string.argtypes = [i32]
        L.cq_status_string.restype = C.c_char_p
        for name in ("cq_quantize", "cq_varbits_index", "cq_pack_varbits", "cq_unpack_varbits",
                     "cq_project_residual", "cq_requant_verify", "cq_dequant_gemv", "cq_dequant_gemv_multi",
                     "cq_dequant_gemm", "cq_dequant_gemm_static", "cq_rrq_stage", "cq_dequant_gemv_stages",
                     "cq_requant_verify_pair", "cq_reparam_residual", "cq_reparam_residual_grad",
                     "cq_requant_refine", "cq_debug_word", "cq_debug_selftest"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def synth_lib():
    global _synth
    if _synth is None:
        if not os.path.exists(LIBSYNTH_PATH):
            raise CQError(8, f"{LIBSYNTH_PATH} is missing: run cell_updates_b200/build.py")
        S = C.CDLL(LIBSYNTH_PATH)
        p, i64, u64, u32 = C.c_void_p, C.c_int64, C.c_uint64, C.c_uint32
        S.cqs_normal_f32.argtypes = [p, i64, u64, u32, i64, C.c_float, p]
        S.cqs_code_words.argtypes = [p, i64, u64, i64, p]
        S.cqs_scales.argtypes = [p, i64, u64, i64, p]
        S.cqs_zeros.argtypes = [p, i64, u64, i64, p]
        S.cqs_residual_bf16.argtypes = [p, p, i64, u64, i64, C.c_float, p]
        for n in SYNTH_EXPORTS:
            getattr(S, n).restype = C.c_int
        _synth = S
    return _synth


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise CQError(1, "tensor is not on a CUDA device")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(rc, name):
    if rc != 0:
        raise CQError(rc, f"{name}: {lib().cq_last_error().decode()}")


def _dtype_code(t):
    if t.dtype == torch.float32:
        return CQ_F32
    if t.dtype == torch.bfloat16:
        return CQ_BF16
    raise CQError(1, f"unsupported dtype {t.dtype}")


class QWeight:
    """A quantized matrix in device memory (the fields of cq_qweight, as tensors).

    planes: list of 4 uint8 tensors or None (b = 1, 2, 4, 8); fixed 4-bit uses planes[2].
    scale: int16/uint16-sized tensor of fp16 bit patterns (any 2-byte dtype); zero: uint8.
    """

    def __init__(self, rows, cols, planes, scale, zero, bits=None, offset=None, residual=None):
        self.rows, self.cols = int(rows), int(cols)
        self.planes = list(planes)
        self.scale, self.zero, self.bits, self.offset = scale, zero, bits, offset
        self.residual = residual

    def struct(self):
        s = cq_qweight()
        s.rows, s.cols = self.rows, self.cols
        s.bits, s.offset = _ptr(self.bits), _ptr(self.offset)
        for i in range(4):
            s.plane[i] = _ptr(self.planes[i]) if self.planes[i] is not None else None
        s.scale, s.zero = _ptr(self.scale), _ptr(self.zero)
        s.residual = _ptr(self.residual)
        s.residual_dtype = _dtype_code(self.residual) if self.residual is not None else CQ_F32
        return s

    def with_residual(self, residual):
        return QWeight(self.rows, self.cols, self.planes, self.scale, self.zero, self.bits, self.offset, residual)


# ---- the entry points ------------------------------------------------------------------

def cq_quantize(w, bits, codes, scale, zero, status_word=None, stream=None):
    rows, cols = w.shape
    _check(lib().cq_quantize(_ptr(w), rows, cols, _ptr(bits), _ptr(codes), _ptr(scale), _ptr(zero),
                             _ptr(status_word), _stream(stream)), "cq_quantize")


def cq_varbits_index(bits, offset, plane_bytes, stream=None):
    _check(lib().cq_varbits_index(_ptr(bits), bits.numel(), _ptr(offset), _ptr(plane_bytes), _stream(stream)),
           "cq_varbits_index")


def cq_pack_varbits(codes, n_groups, bits, offset, planes, stream=None):
    arr = (C.c_void_p * 4)(*[_ptr(p) if p is not None else None for p in planes])
    _check(lib().cq_pack_varbits(_ptr(codes), n_groups, _ptr(bits), _ptr(offset), arr, _stream(stream)),
           "cq_pack_varbits")


def cq_unpack_varbits(qw, codes, stream=None):
    s = qw.struct()
    _check(lib().cq_unpack_varbits(C.byref(s), _ptr(codes), _stream(stream)), "cq_unpack_varbits")


def cq_project_residual(r, scale, n_clamped=None, stream=None):
    _check(lib().cq_project_residual(_ptr(r), _dtype_code(r), _ptr(scale), r.numel(), _ptr(n_clamped),
                                     _stream(stream)), "cq_project_residual")


def cq_requant_verify(qw, first_w, n_w, mismatches, first_bad, group_flags=None, stream=None):
    s = qw.struct()
    _check(lib().cq_requant_verify(C.byref(s), first_w, n_w, _ptr(mismatches), _ptr(first_bad),
                                   _ptr(group_flags), _stream(stream)), "cq_requant_verify")


def cq_dequant_gemv(qw, x, y, stream=None):
    s = qw.struct()
    m = x.shape[0] if x.dim() == 2 else 1
    _check(lib().cq_dequant_gemv(C.byref(s), _ptr(x), _dtype_code(x), m, _ptr(y), _stream(stream)),
           "cq_dequant_gemv")


def cq_dequant_gemv_multi(qws, x, ys, stream=None):
    """Several matrices with the same cols against one x (see include/cq.h)."""
    structs = [q.struct() for q in qws]
    arr = (C.POINTER(cq_qweight) * len(structs))(*[C.pointer(st) for st in structs])
    yarr = (C.c_void_p * len(ys))(*[_ptr(y) for y in ys])
    m = x.shape[0] if x.dim() == 2 else 1
    _check(lib().cq_dequant_gemv_multi(C.cast(arr, C.c_void_p), len(structs), _ptr(x), _dtype_code(x), m,
                                       C.cast(yarr, C.c_void_p), _stream(stream)), "cq_dequant_gemv_multi")


def cq_requant_verify_pair(qw, first_w, n_w, mism, first_bad, mism0, first0, group_flags=None, stream=None):
    """Verify with the residual and without it (revocation) in one pass (see include/cq.h)."""
    s = qw.struct()
    _check(lib().cq_requant_verify_pair(C.byref(s), first_w, n_w, _ptr(mism), _ptr(first_bad), _ptr(mism0),
                                        _ptr(first0), _ptr(group_flags), _stream(stream)), "cq_requant_verify_pair")


def cq_rrq_stage(r, bits, codes, scale, zero, status_word=None, stream=None):
    """One recurrent-residual stage: quantize r at one width, replace r by what it misses."""
    rows, cols = r.shape
    _check(lib().cq_rrq_stage(_ptr(r), rows, cols, int(bits), _ptr(codes), _ptr(scale), _ptr(zero),
                              _ptr(status_word), _stream(stream)), "cq_rrq_stage")


def cq_dequant_gemv_stages(stages, x, y, stream=None):
    """y = (sum of the stages' dequantized weights) x (see include/cq.h)."""
    structs = [q.struct() for q in stages]
    arr = (C.POINTER(cq_qweight) * len(structs))(*[C.pointer(st) for st in structs])
    m = x.shape[0] if x.dim() == 2 else 1
    _check(lib().cq_dequant_gemv_stages(C.cast(arr, C.c_void_p), len(structs), _ptr(x), _dtype_code(x), m, _ptr(y),
                                        _stream(stream)), "cq_dequant_gemv_stages")


def cq_reparam_residual(theta, scale, r, stream=None):
    """r = c * theta / sqrt(1 + theta^2), bounded into each weight's cell (see include/cq.h)."""
    _check(lib().cq_reparam_residual(_ptr(theta), _ptr(scale), theta.numel(), _ptr(r), _dtype_code(r),
                                     _stream(stream)), "cq_reparam_residual")


def cq_reparam_residual_grad(theta, scale, grad_r, grad_theta, r_dtype, stream=None):
    """dL/dtheta from dL/dr; r_dtype (CQ_F32 / CQ_BF16) picks the bound as in the forward pass."""
    _check(lib().cq_reparam_residual_grad(_ptr(theta), _ptr(scale), _ptr(grad_r), theta.numel(), int(r_dtype),
                                          _ptr(grad_theta), _stream(stream)), "cq_reparam_residual_grad")


def cq_requant_workspace(rows, cols):
    return int(lib().cq_requant_workspace(rows, cols))


def cq_requant_refine(w, H, scale, zero, bits, codes, sweeps, err_before=None, err_after=None, moves=None,
                      workspace=None, stream=None):
    """ReQuant refinement of codes (in place) on the frozen grid against H (see include/cq.h)."""
    rows, cols = w.shape
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().cq_requant_refine(_ptr(w), rows, cols, _ptr(H), _ptr(scale), _ptr(zero), int(bits), _ptr(codes),
                                   int(sweeps), _ptr(err_before), _ptr(err_after), _ptr(moves), _ptr(workspace),
                                   nbytes, _stream(stream)), "cq_requant_refine")


def cq_debug_word():
    """The first failed in-kernel index check since the last call (a debug build's site number),
    or 0; waits for the device. A release build raises CQError(CQ_ERR_UNSUPPORTED)."""
    w = C.c_uint32(0)
    _check(lib().cq_debug_word(C.byref(w)), "cq_debug_word")
    return int(w.value)


def cq_debug_selftest(stream=None):
    _check(lib().cq_debug_selftest(_stream(stream)), "cq_debug_selftest")


def cq_gemm_workspace(rows, cols, m):
    return int(lib().cq_gemm_workspace(rows, cols, m))


def cq_dequant_gemm(qw, x, y, workspace=None, stream=None):
    s = qw.struct()
    m = x.shape[0]
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().cq_dequant_gemm(C.byref(s), _ptr(x), _dtype_code(x), m, _ptr(y), _ptr(workspace), nbytes,
                                 _stream(stream)), "cq_dequant_gemm")


def cq_dequant_gemm_static(qw, x, y, status_word=None, stream=None):
    """cq_dequant_gemm without a workspace: the library's own static scratch (see include/cq.h)."""
    s = qw.struct()
    _check(lib().cq_dequant_gemm_static(C.byref(s), _ptr(x), _dtype_code(x), x.shape[0], _ptr(y),
                                        _ptr(status_word), _stream(stream)), "cq_dequant_gemm_static")


def cq_last_error():
    return lib().cq_last_error().decode()


# ---- device-side synthetic inputs (test data) ---------------------------------------

def _synth_check(rc, name):
    if rc != 0:
        raise CQError(rc, name)


def cqs_normal_f32(out, seed, stream_id, first, mult, stream=None):
    _synth_check(synth_lib().cqs_normal_f32(_ptr(out), out.numel(), seed, stream_id, first, mult, _stream(stream)),
                 "cqs_normal_f32")


def cqs_code_words(out_u64, seed, first_word, stream=None):
    _synth_check(synth_lib().cqs_code_words(_ptr(out_u64), out_u64.numel(), seed, first_word, _stream(stream)),
                 "cqs_code_words")


def cqs_scales(out, seed, first, stream=None):
    _synth_check(synth_lib().cqs_scales(_ptr(out), out.numel(), seed, first, _stream(stream)), "cqs_scales")


def cqs_zeros(out, seed, first, stream=None):
    _synth_check(synth_lib().cqs_zeros(_ptr(out), out.numel(), seed, first, _stream(stream)), "cqs_zeros")


def cqs_residual_bf16(out, scale, seed, first, mult, stream=None):
    _synth_check(synth_lib().cqs_residual_bf16(_ptr(out), _ptr(scale), out.numel(), seed, first, mult,
                                               _stream(stream)), "cqs_residual_bf16")
