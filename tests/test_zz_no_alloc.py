"""cq_dequant_gemm_static: the GEMM entry point for callers that cannot allocate device
memory (its scratch is a static array inside the library). Checked through the C ABI against
cq_dequant_gemm, which takes a caller-allocated workspace, on two calls in a row.

The file name keeps it last in collection order, so a run that stops at the first failure has
already run every other test. It also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from cell_updates_b200 import build, cq, ops
from gpu_util import check_matmul, host

pytestmark = pytest.mark.gpu


def test_static_scratch_gemm_matches_workspace_gemm(cuda_ok):
    build.build()
    torch.manual_seed(1234)
    rows, cols, m = 1000, 64 * 40, 64
    w = torch.randn(rows, cols, device="cuda") * 0.02
    qw, _, _ = ops.quantize_and_pack(w)
    for call in range(2):
        x = (torch.randn(m, cols, device="cuda") * (1 + call)).to(torch.bfloat16)
        ref = ops.gemm(qw, x)                       # workspace-taking entry point
        y = torch.full((m, rows), float("nan"), device="cuda")
        cq.cq_dequant_gemm_static(qw, x, y)
        torch.cuda.synchronize()
        assert np.isfinite(host(y)).all()
        check_matmul(host(y), host(ref).astype(np.float64), f"static-scratch call {call}")
