"""cq_dequant_gemm_static: the GEMM entry point for callers that cannot allocate device
memory -- a plug-in handed its buffers by a host framework that owns all device memory, or a
serving loop with a fixed memory budget where an allocation could block or fail mid-request.
Its scratch is a static array inside the library, so the call itself allocates nothing.

Checked through the C ABI, on two calls in a row per case, against the oracle's fp64 product
(seeded NumPy inputs, the matmul tolerance of the other GPU tests) and against cq_dequant_gemm,
which takes a caller-allocated workspace:
  * m = 64, the tensor-core GEMM with one batch slice;
  * m = 80, two slices that reuse the static array one after the other in stream order;
  * m = 8, served by the GEMV kernels (no scratch used);
  * a shape whose scratch would exceed the static array, refused with CQ_ERR_RANGE;
  * a NULL weight descriptor, refused with CQ_ERR_ARG before any CUDA work.
Around each checked call, torch's allocator and the device's free memory stay unchanged, and
the status word the call hands back is 0.

The file name keeps it last in collection order, so a run that stops at the first failure has
already run every other test. It also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from cell_updates_b200 import build, cq, ops, synth
from gpu_util import bf16_dev, check_matmul, dev, host, u16_dev
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu


def _artifact(rows, cols, seed):
    """A 4-bit artifact quantized and packed by the oracle, and its device copy."""
    w = synth.normal_weights(rows, cols, seed=seed)
    codes, scale, zero, st = co.quantize(w)
    assert st == 0
    planes = co.pack(codes)
    qw = cq.QWeight(rows, cols, [None, None, dev(planes[2]), None], u16_dev(scale), dev(zero))
    return qw, planes, scale, zero


def _mem():
    torch.cuda.synchronize()
    return torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]


@pytest.mark.parametrize("m", [64, 80, 8])
def test_static_scratch_gemm_matches_oracle(cuda_ok, m):
    build.build()
    rows, cols = 1000, 64 * 40
    qw, planes, scale, zero = _artifact(rows, cols, seed=4321 + m)
    y = torch.empty((m, rows), device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    xs = [synth.activations(m, cols, seed=100 * m + call, dtype="bf16") for call in range(2)]
    x_devs = [bf16_dev(x) for x in xs]
    cq.cq_dequant_gemm_static(qw, x_devs[0], y, status)     # first call on the device: the set-up
    for call in range(2):
        y.fill_(float("nan"))
        status.fill_(-1)
        before = _mem()
        cq.cq_dequant_gemm_static(qw, x_devs[call], y, status)
        after = _mem()
        assert after == before, f"m={m} call {call}: memory changed {before} -> {after}"
        assert int(status.cpu()[0]) == 0
        got = host(y).astype(np.float64)
        assert np.isfinite(got).all()
        y_ref = co.dequant_matmul_f64(planes, scale, zero, rows, cols, xs[call], "bf16")
        check_matmul(got, y_ref, f"static scratch m={m} call {call} vs oracle")
        ref = ops.gemm(qw, x_devs[call])                   # the workspace-taking entry point
        check_matmul(got, host(ref).astype(np.float64), f"static scratch m={m} call {call} vs cq_dequant_gemm")


def test_static_scratch_refuses_what_does_not_fit(cuda_ok):
    build.build()
    # cols = 65792 (1028 groups, a multiple of four) needs 512 + 2 * 64 * 65792 bytes > 8 MiB
    rows, cols, m = 16, 65792, 64
    qw = cq.QWeight(rows, cols, [None, None, torch.zeros(rows * cols // 2, dtype=torch.uint8, device="cuda"), None],
                    torch.zeros(rows * cols // 64, dtype=torch.int16, device="cuda"),
                    torch.zeros(rows * cols // 64, dtype=torch.uint8, device="cuda"))
    x = torch.zeros((m, cols), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((m, rows), device="cuda")
    with pytest.raises(cq.CQError) as e:
        cq.cq_dequant_gemm_static(qw, x, y)
    assert e.value.status == 6 and "static buffer holds" in str(e.value)


def test_static_scratch_checks_arguments_first(cuda_ok):
    import ctypes as C
    L = cq.lib()
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((16, 4), device="cuda")
    rc = L.cq_dequant_gemm_static(None, C.c_void_p(x.data_ptr()), cq.CQ_BF16, 16, C.c_void_p(y.data_ptr()), None,
                                  None)
    assert rc == 1 and b"qweight is NULL" in L.cq_last_error()
