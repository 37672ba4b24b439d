"""The C-ABI libraries load and export every symbol their headers declare, and reject bad
arguments on the host before touching a GPU (no compute call runs here)."""
import ctypes as C
import os
import re

import pytest

from cell_updates_b200 import build, cq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cqs?_[a-z0-9_]+)\s*\(", text)))


def test_libcq_exports_header_symbols():
    names = _declared("cq.h")
    assert names == sorted(cq.EXPORTS)
    lib = C.CDLL(cq.LIBCQ_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_test_builds_export_the_same_symbols():
    names = _declared("cq.h")
    for variant in build.TEST_VARIANTS:
        lib = C.CDLL(build.test_variant_path(variant))
        for n in names:
            assert hasattr(lib, n), (variant, n)


def test_debug_word_needs_a_debug_build():
    """Release: no checks compiled in, CQ_ERR_UNSUPPORTED with the word zeroed; both builds
    reject a NULL word on the host (no GPU is touched on either path)."""
    rel = C.CDLL(build.LIBCQ)
    rel.cq_debug_word.argtypes = [C.c_void_p]
    rel.cq_debug_selftest.argtypes = [C.c_void_p]
    w = C.c_uint32(0xDEAD)
    assert rel.cq_debug_word(C.byref(w)) == 8 and w.value == 0
    assert rel.cq_debug_word(None) == 1
    assert rel.cq_debug_selftest(None) == 8
    dbg = C.CDLL(build.test_variant_path("debug"))
    dbg.cq_debug_word.argtypes = [C.c_void_p]
    assert dbg.cq_debug_word(None) == 1


def test_libcq_synth_exports_header_symbols():
    names = _declared("cq_synth.h")
    assert names == sorted(cq.SYNTH_EXPORTS)
    lib = C.CDLL(cq.LIBSYNTH_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_host_validation_rejects_bad_arguments():
    L = cq.lib()
    p = C.c_void_p(16)   # never dereferenced: validation fails first
    assert L.cq_quantize(p, 4, 63, None, p, p, p, None, None) == 2          # cols % 64
    assert L.cq_quantize(p, -1, 64, None, p, p, p, None, None) == 2         # negative
    assert L.cq_quantize(C.c_void_p(8), 4, 64, None, p, p, p, None, None) == 4   # misaligned w
    assert L.cq_quantize(None, 4, 64, None, p, p, p, None, None) == 1       # NULL w
    assert L.cq_project_residual(p, 0, p, 100, None, None) == 2             # n % 64
    assert L.cq_project_residual(p, 5, p, 64, None, None) == 1              # bad dtype
    assert L.cq_varbits_index(p, (1 << 26) + 1, p, p, None) == 6            # 32-bit offsets
    qw = cq.cq_qweight()
    qw.rows, qw.cols = 4, 64
    qw.scale, qw.zero = 16, 16
    qw.plane[2] = 16
    assert L.cq_requant_verify(C.byref(qw), 32, 64, p, p, None, None) == 2  # not whole groups
    assert L.cq_requant_verify(C.byref(qw), 0, 512, p, p, None, None) == 2  # past the end
    assert L.cq_dequant_gemv(C.byref(qw), p, 1, 9, p, None) == 1            # m > 8
    qw.plane[2] = 8
    assert L.cq_dequant_gemv(C.byref(qw), p, 1, 1, p, None) == 4            # misaligned plane
    qw.plane[2] = 16
    qw.bits = 16                                                             # bits without offset
    assert L.cq_dequant_gemv(C.byref(qw), p, 1, 1, p, None) == 1
    assert "offset" in cq.cq_last_error()
    assert L.cq_gemm_workspace(8192, 28672, 8) == 0
    qw.bits = None
    other = cq.cq_qweight()
    other.rows, other.cols, other.scale, other.zero = 4, 128, 16, 16
    other.plane[2] = 16
    qws = (C.POINTER(cq.cq_qweight) * 2)(C.pointer(qw), C.pointer(other))
    ys = (C.c_void_p * 2)(16, 16)
    assert L.cq_dequant_gemv_multi(C.cast(qws, C.c_void_p), 2, p, 1, 1, C.cast(ys, C.c_void_p), None) == 2  # unequal cols
    assert L.cq_dequant_gemv_multi(None, 2, p, 1, 1, C.cast(ys, C.c_void_p), None) == 1                    # NULL list
    assert L.cq_dequant_gemv_multi(None, 0, p, 1, 1, None, None) == 0                                      # nothing to do
    assert L.cq_requant_verify_pair(C.byref(qw), 0, 256, p, p, p, p, None, None) == 1   # no residual
    qw.residual = 16
    assert L.cq_requant_verify_pair(C.byref(qw), 0, 256, p, p, None, p, None, None) == 1  # NULL result
    assert L.cq_requant_verify_pair(C.byref(qw), 32, 64, p, p, p, p, None, None) == 2    # not whole groups
    qw.residual = None
    # recurrent residual quantization
    assert L.cq_rrq_stage(p, 4, 64, 3, p, p, p, None, None) == 3             # width 3
    assert L.cq_rrq_stage(p, 4, 96, 2, p, p, p, None, None) == 2             # cols % 64
    assert L.cq_rrq_stage(C.c_void_p(8), 4, 64, 2, p, p, p, None, None) == 4  # misaligned r
    assert L.cq_rrq_stage(None, 4, 64, 2, p, p, p, None, None) == 1          # NULL r
    assert L.cq_dequant_gemv_stages(C.cast(qws, C.c_void_p), 0, p, 1, 1, p, None) == 1   # no stages
    assert L.cq_dequant_gemv_stages(C.cast(qws, C.c_void_p), 9, p, 1, 1, p, None) == 1   # too many
    assert L.cq_dequant_gemv_stages(C.cast(qws, C.c_void_p), 2, p, 1, 1, p, None) == 2   # unequal shapes
    qw.residual = 16
    one = (C.POINTER(cq.cq_qweight) * 1)(C.pointer(qw))
    assert L.cq_dequant_gemv_stages(C.cast(one, C.c_void_p), 1, p, 1, 1, p, None) == 8   # residual
    qw.residual = None


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(cq, "_lib", None)
    monkeypatch.setattr(cq, "LIBCQ_PATH", "/nonexistent/libcq.so")
    with pytest.raises(cq.CQError):
        cq.lib()
