"""A bounded device-side wait that runs out: the kernel gives up, says so, and the GPU stays usable.

The library never spins without a limit: every wait on a copy gives up after a bounded number
of hardware-suspended tries (about a second), raises the CTA's abort flag, lets the copies it
did issue land, and reports through its status word. This test makes one such wait run out on
purpose without any fault: a test-only build of the library
(cell_updates_b200/_build/libcq_drop_first_copy.so, built by build.py and loaded only here)
omits one warp's first tile request in the quantize kernel, so that warp's wait can never
complete. The call must return, the status word must carry CQ_QSTATUS_TIMEOUT, and afterwards
the regular library must still produce exact results on the same device.
"""
import ctypes as C
import time

import numpy as np
import pytest
import torch

from cell_updates_b200 import build, cq, ops, synth
from gpu_util import dev, host
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu


def test_quantize_wait_runs_out_and_reports_timeout(cuda_ok):
    build.build()
    L = C.CDLL(build.test_variant_path("drop_first_copy"))
    p, i64 = C.c_void_p, C.c_int64
    L.cq_quantize.argtypes = [p, i64, i64, p, p, p, p, p, p]
    L.cq_quantize.restype = C.c_int
    rows, cols = 1024, 4096
    w = synth.normal_weights(rows, cols, seed=0)
    wd = dev(w)
    G = rows * cols // 64
    codes = torch.zeros(rows * cols, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(G, dtype=torch.int16, device="cuda")
    zero = torch.zeros(G, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    rc = L.cq_quantize(wd.data_ptr(), rows, cols, None, codes.data_ptr(), scale.data_ptr(), zero.data_ptr(),
                       status.data_ptr(), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()                       # the kernel ends: the wait gave up
    elapsed = time.monotonic() - t0
    assert rc == 0
    assert int(host(status)[0]) & cq.QSTATUS_TIMEOUT, int(host(status)[0])
    assert elapsed < 30.0, elapsed
    # the groups of the tile that never arrived are left unwritten; every other group is exact
    oc, osc, oz, _ = co.quantize(w)
    got_scale = host(scale, np.uint16)
    assert not got_scale[:32].any()                # the dropped tile: 32 groups, untouched
    assert np.array_equal(got_scale[32:], osc[32:])
    # the context is still usable: the regular library quantizes the same weights exactly
    codes2, scale2, zero2, st2 = ops.quantize(wd)
    assert int(host(st2)[0]) == 0
    assert np.array_equal(host(codes2), oc)
    assert np.array_equal(host(scale2, np.uint16), osc)
    assert np.array_equal(host(zero2), oz)


def test_gemm_wait_runs_out_and_reports_status(cuda_ok):
    # the same test-only build omits CTA 0's first activation tiles in the tensor-core GEMM: the
    # MMA issuer's wait gives up, every role of that CTA takes the abort path (the issued copies
    # land, the issued MMAs drain, tensor memory is released), the status word in the workspace
    # is non-zero, and the regular library then computes the same product correctly
    build.build()
    L = C.CDLL(build.test_variant_path("drop_first_copy"))
    L.cq_dequant_gemm.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_size_t,
                                  C.c_void_p]
    L.cq_dequant_gemm.restype = C.c_int
    rows, cols, m = 512, 4096, 64
    w = synth.normal_weights(rows, cols, seed=3)
    qw, _, _ = ops.quantize_and_pack(dev(w))
    x = torch.from_numpy(synth.activations(m, cols, seed=4, dtype="bf16").view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.zeros((m, rows), device="cuda")
    need = cq.cq_gemm_workspace(rows, cols, m)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    s = qw.struct()
    torch.cuda.synchronize()
    t0 = time.monotonic()
    rc = L.cq_dequant_gemm(C.byref(s), x.data_ptr(), cq.CQ_BF16, m, y.data_ptr(), ws.data_ptr(), need,
                           C.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert rc == 0
    assert int(ws[:4].view(torch.int32).cpu()[0]) != 0
    assert elapsed < 30.0, elapsed
    ref = ops.gemm(qw, x)                          # regular library, same device: a correct product
    planes = [np.zeros(1, np.uint8)] * 2 + [host(qw.planes[2]), np.zeros(1, np.uint8)]
    from gpu_util import check_matmul
    y_ref = co.dequant_matmul_f64(planes, host(qw.scale, np.uint16), host(qw.zero), rows, cols,
                                  host(x.view(torch.int16)).view(np.uint16), "bf16")
    check_matmul(host(ref).astype(np.float64), y_ref, "gemm after an aborted call")
