"""ReQuant fixed-grid refinement on the GPU against the oracle: the refined codes, the number of
accepted moves and the per-row errors before and after are the same bit for bit (both sides run
the same binary64 operations in the same order). Page 1 (thelatestinai.com/papers/2608.20873),
ReQuant abstract: accepted updates strictly lower the reconstruction error and stay on the grid."""
import numpy as np
import pytest
import torch

from cell_updates_b200 import build, ops, synth
from gpu_util import dev, host, u16_dev
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    build.build()


def _case(rows, cols, n_cal, seed):
    rng = np.random.default_rng(seed)
    w = synth.normal_weights(rows, cols, seed=seed)
    codes, scale, zero, _ = co.quantize(w)
    X = rng.standard_normal((n_cal, cols))
    X[:, rng.choice(cols, max(1, cols // 32), replace=False)] *= 10.0     # outlier input channels
    H = X.T @ X
    H = (H + H.T) * 0.5                                                    # exactly symmetric
    return w, codes, scale, zero, H


@pytest.mark.parametrize("rows,cols,sweeps", [(5, 64, 1), (37, 320, 2), (130, 1024, 3), (64, 4096, 1)])
def test_requant_matches_oracle(rows, cols, sweeps):
    w, codes, scale, zero, H = _case(rows, cols, min(2 * cols, 1024), seed=rows + cols)
    q, eb, ea, mv = ops.requant_refine(dev(w), dev(H), u16_dev(scale), dev(zero), dev(codes), sweeps)
    oq, oeb, oea, omv = co.requant_refine(w, H, codes, scale, zero, 4, sweeps)
    assert np.array_equal(host(q), oq)
    assert np.array_equal(host(mv).astype(np.uint64), omv)
    assert np.array_equal(host(eb).view(np.uint64), oeb.view(np.uint64))
    assert np.array_equal(host(ea).view(np.uint64), oea.view(np.uint64))
    assert omv.sum() > 0 and (oea[omv > 0] < oeb[omv > 0]).all()
