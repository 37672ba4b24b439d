"""Full-size parity: every configuration at its own size, in the launch configuration bench.py
times, against the CPU oracle.

Where the oracle cannot redo the whole problem in seconds it checks sampled outputs it can
compute one by one (rows of a matmul, chunks of a verify), taking its inputs from the seeded
generators (never from the GPU), and the GPU run is checked on the whole problem through
properties that hold at any size (zero mismatches after projection and after revocation,
exactly the planted mismatches found, first index exact).

* config 1: the three decode matrices 4096x4096, 11008x4096, 4096x11008 (0.02 Student-t(5),
  0.1 % outliers x10, drawn as bench.py draws them): quantize bit-exact and GEMV at batch 1
  within tolerance on sampled rows.
* config 2: VBQ 2048x8192, GEMV at batch 1 and 8 over the whole matrix.
* config 3: CellFill stack of 28 layers (q, k, v, o 2048x2048; gate, up 2048x6144; down
  6144x2048) = 1,526,726,656 weights with bf16 residuals ~N(0, (0.3 s)^2), built on the device by
  the counter-based generator: project, verify, revoke, planted out-of-cell residuals; sampled
  chunks regenerated on the host by its NumPy twin.
* config 4: GEMM 8192x28672 and 28672x8192 at batch 1, 4, 16, 64 on sampled rows; chunked
  verify over 2.4e10 weights (61 GB resident).
"""
import numpy as np
import pytest
import torch

from cell_updates_b200 import cq, ops, synth
from gpu_util import bf16_dev, check_matmul, dev, host
from oracle import c_oracle as co

pytestmark = pytest.mark.gpu

GROUP = 64


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from cell_updates_b200 import build
    build.build()
    cq.lib()
    cq.synth_lib()
    yield
    torch.cuda.empty_cache()


def _sample_rows(N, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(k, N), replace=False).tolist()) | {0, N - 1, min(N - 1, 127), min(N - 1, 128)}
    return np.array(sorted(rows), dtype=np.int64)


def _oracle_rows(w, rows, x_bits):
    """The oracle's own quantization of the sampled rows, and its fp64 y on them."""
    wr = np.ascontiguousarray(w[rows])
    codes, scale, zero, st = co.quantize(wr)
    y = co.dequant_matmul_f64(co.pack(codes), scale, zero, len(rows), w.shape[1], x_bits, "bf16")
    return (codes, scale, zero, st), y


def _check_quant_rows(codes_d, qw, rows, oc):
    N, K = qw.rows, qw.cols
    codes, scale, zero, _ = oc
    KG = K // GROUP
    rows_t = torch.from_numpy(rows).cuda()
    g_codes = host(codes_d.view(N, K).index_select(0, rows_t)).ravel()
    g_scale = host(qw.scale.view(N, KG).index_select(0, rows_t), np.uint16).ravel()
    g_zero = host(qw.zero.view(N, KG).index_select(0, rows_t)).ravel()
    assert np.array_equal(g_codes, codes)
    assert np.array_equal(g_scale, scale)
    assert np.array_equal(g_zero, zero)


# ---- config 1: decode GEMV at full size ---------------------------------------------------

@pytest.mark.parametrize("idx,shape", list(enumerate([(4096, 4096), (11008, 4096), (4096, 11008)])))
def test_config1_gemv_full_size(idx, shape):
    N, K = shape
    w = synth.student_t_weights(N, K, seed=1 + 1000 * idx)
    qw, codes_d, st_d = ops.quantize_and_pack(dev(w))
    x = synth.activations(1, K, seed=1 + 1000 * idx + 11, dtype="bf16")
    y = host(ops.gemv(qw, bf16_dev(x)))
    assert int(host(st_d)[0]) == 0
    rows = _sample_rows(N, 192, seed=idx)
    oc, y_ref = _oracle_rows(w, rows, x)
    _check_quant_rows(codes_d, qw, rows, oc)
    check_matmul(y[:, rows], y_ref, f"cfg1 {N}x{K} m=1 (sampled rows)")


# ---- config 2: VBQ GEMV over the whole matrix -------------------------------------------------

@pytest.mark.parametrize("m", [1, 8])
def test_config2_vbq_gemv_full(m):
    N, K = 2048, 8192
    w = synth.normal_weights(N, K, seed=2)
    bits = synth.vbq_bits(N * K // GROUP, seed=2)
    qw, _, st_d = ops.quantize_and_pack(dev(w), dev(bits))
    x = synth.activations(m, K, seed=20 + m, dtype="bf16")
    y = host(ops.gemv(qw, bf16_dev(x)))
    codes, scale, zero, st = co.quantize(w, bits)
    off, pb = co.varbits_index(bits)
    y_ref = co.dequant_matmul_f64(co.pack(codes, bits, off, pb), scale, zero, N, K, x, "bf16", bits, off)
    assert int(host(st_d)[0]) == st == 0
    check_matmul(y, y_ref, f"cfg2 vbq m={m}")


# ---- synthetic 4-bit artifacts built on the device (configs 3 and 4) -----------------------

RESID_SIGMA = 0.3


def _device_artifact(n, seed):
    """plane (4-bit codes), fp16 scales, zeros and a bf16 residual ~N(0,(0.3 s)^2), on the GPU."""
    G = n // GROUP
    plane = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    scale = torch.empty(G, dtype=torch.int16, device="cuda")
    zero = torch.empty(G, dtype=torch.uint8, device="cuda")
    r = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    cq.cqs_code_words(plane.view(torch.int64), seed, 0)
    cq.cqs_scales(scale, seed, 0)
    cq.cqs_zeros(zero, seed, 0)
    cq.cqs_residual_bf16(r, scale, seed, 0, float(synth.ih4_multiplier(RESID_SIGMA)))
    return plane, scale, zero, r


def _host_chunk(seed, first, n):
    """The same artifact's weights [first, first + n) from the NumPy twin (first % 64 == 0)."""
    words = synth.hashed_code_words(seed, np.arange(first // 16, (first + n) // 16, dtype=np.int64))
    plane = words.astype("<u8").view(np.uint8)
    g = np.arange(first // GROUP, (first + n) // GROUP, dtype=np.int64)
    scale = synth.hashed_scales(seed, g)
    zero = synth.hashed_zeros(seed, g)
    r = synth.hashed_residual_bf16(seed, np.arange(first, first + n, dtype=np.int64),
                                   np.repeat(scale, GROUP), RESID_SIGMA)
    return plane, scale, zero, r


def _code_at(plane_host_chunk, i_rel):
    b = int(plane_host_chunk[i_rel >> 1])
    return (b >> 4) if (i_rel & 1) else (b & 0xF)


def _planted_bits(seed, i):
    """bf16 bits of +-0.6 s for weight i: outside its cell, pushing the code away from its clamp"""
    plane, scale, zero, _ = _host_chunk(seed, (i // GROUP) * GROUP, GROUP)
    q = _code_at(plane, i % GROUP)
    s = float(synth.f16_bits_to_f32(scale[0]))
    return int(synth.f32_to_bf16_bits(np.float32(0.6 * s if q < 15 else -0.6 * s)))


def _plant(r, seed, positions):
    """Write the planted residuals into the device residual; returns {index: bf16 bits}."""
    bits = {i: _planted_bits(seed, i) for i in positions}
    r16 = r.view(torch.int16)
    for i, b in bits.items():
        r16[i] = int(np.uint16(b).view(np.int16))
    return bits


def _chunk_checks(seed, plane, scale, zero, r_proj, first, n):
    """Sampled chunk: the GPU projection equals the oracle's bit for bit; the oracle and the GPU
    count the same mismatches for the unprojected residual (negative control), both 0 after
    projection."""
    hp, hs, hz, hr = _host_chunk(seed, first, n)
    # the device generator and its NumPy twin give the same artifact, bit for bit
    assert np.array_equal(host(plane[first // 2:(first + n) // 2]), hp)
    assert np.array_equal(host(scale[first // GROUP:(first + n) // GROUP], np.uint16), hs)
    assert np.array_equal(host(zero[first // GROUP:(first + n) // GROUP]), hz)
    rp_ref, _ = co.project_bf16(hr, hs)
    rp_gpu = host(r_proj[first:first + n].view(torch.int16)).view(np.uint16)
    assert np.array_equal(rp_gpu, rp_ref)
    m_ref, _, _ = co.verify([np.zeros(1, np.uint8)] * 2 + [hp, np.zeros(1, np.uint8)], hs, hz, r=hr, r_dtype="bf16")
    assert m_ref > 0
    # the same chunk on the GPU, with the unprojected residual uploaded from the host twin
    qw = cq.QWeight(1, n, [None, None, plane[first // 2:(first + n) // 2], None],
                    scale[first // GROUP:(first + n) // GROUP], zero[first // GROUP:(first + n) // GROUP],
                    residual=bf16_dev(hr))
    mism, fb, _ = ops.verify(qw)
    assert int(mism.item()) == m_ref
    m0, _, _ = co.verify([np.zeros(1, np.uint8)] * 2 + [hp, np.zeros(1, np.uint8)], hs, hz, r=rp_ref, r_dtype="bf16")
    assert m0 == 0


def _stack_weights():
    per_layer = 4 * 2048 * 2048 + 2 * 2048 * 6144 + 6144 * 2048
    return 28 * per_layer


def test_config3_cellfill_stack_full():
    seed = 3
    n = _stack_weights()
    assert n == 1_526_726_656
    plane, scale, zero, r = _device_artifact(n, seed)
    n_clamped = ops.project(r, scale)
    qw_r = cq.QWeight(1, n, [None, None, plane, None], scale, zero, residual=r)
    qw_0 = cq.QWeight(1, n, [None, None, plane, None], scale, zero)
    mism, fb, _ = ops.verify(qw_r)
    assert int(mism.item()) == 0 and int(fb.item()) == -1
    mism, fb, _ = ops.verify(qw_0)                       # revocation: the residual dropped
    assert int(mism.item()) == 0 and int(fb.item()) == -1
    frac = int(n_clamped.item()) / n
    assert 0.05 < frac < 0.15                            # ~9.6 % of N(0,(0.3s)^2) lies beyond 0.498 s
    rng = np.random.default_rng(33)
    for first in [0, (n // 2) // GROUP * GROUP, n - (1 << 20)] + [int(v) * GROUP for v in rng.integers(0, (n - (1 << 20)) // GROUP, 2)]:
        _chunk_checks(seed, plane, scale, zero, r, first, 1 << 20)
    planted = sorted(set(int(v) for v in rng.integers(0, n, 12)))
    _plant(r, seed, planted)
    mism, fb, _ = ops.verify(qw_r)
    assert int(mism.item()) == len(planted) and int(fb.item()) == planted[0]
    del plane, scale, zero, r, qw_r, qw_0
    torch.cuda.empty_cache()


def test_config4_chunked_verify_2_4e10():
    seed = 4
    n = 24_000_000_000
    plane, scale, zero, r = _device_artifact(n, seed)
    ops.project(r, scale)
    qw = cq.QWeight(1, n, [None, None, plane, None], scale, zero, residual=r)
    rng = np.random.default_rng(44)
    planted = sorted(set(int(v) for v in rng.integers(0, n, 16)) | {n - 1, (1 << 34) + 5})
    pbits = _plant(r, seed, planted)
    chunk = 1 << 31
    total, first_bad = 0, -1
    for c0 in range(0, n, chunk):
        nw = min(chunk, n - c0)
        mism, fb, _ = ops.verify(qw, c0, nw)
        k = int(mism.item())
        inside = [p for p in planted if c0 <= p < c0 + nw]
        assert k == len(inside)
        assert int(fb.item()) == (inside[0] if inside else -1)
        total += k
        if first_bad < 0 and k:
            first_bad = int(fb.item())
    assert total == len(planted) and first_bad == planted[0]
    for first in [0, ((1 << 34) // GROUP) * GROUP, n - (1 << 20)]:
        hp, hs, hz, hr = _host_chunk(seed, first, 1 << 20)
        rp_ref, _ = co.project_bf16(hr, hs)
        for p, b in pbits.items():                       # the planted values replace projected ones
            if first <= p < first + (1 << 20):
                rp_ref[p - first] = b
        assert np.array_equal(host(r[first:first + (1 << 20)].view(torch.int16)).view(np.uint16), rp_ref)
    del plane, scale, zero, r, qw
    torch.cuda.empty_cache()


# ---- config 4: GEMM at full size, sampled rows ------------------------------------------------

@pytest.mark.parametrize("idx,shape", list(enumerate([(8192, 28672), (28672, 8192)])))
def test_config4_gemm_full_size(idx, shape):
    N, K = shape
    w = synth.student_t_weights(N, K, seed=4 + 1000 * idx)
    qw, codes_d, st_d = ops.quantize_and_pack(dev(w))
    rows = _sample_rows(N, 96, seed=40 + idx)
    wr = np.ascontiguousarray(w[rows])
    del w
    oc = co.quantize(wr)
    _check_quant_rows(codes_d, qw, rows, oc)
    del codes_d
    planes = co.pack(oc[0])
    for m in (1, 4, 16, 64):
        x = synth.activations(m, K, seed=400 + m, dtype="bf16")
        y = host(ops.gemm(qw, bf16_dev(x)))
        y_ref = co.dequant_matmul_f64(planes, oc[1], oc[2], len(rows), K, x, "bf16")
        check_matmul(y[:, rows], y_ref, f"cfg4 {N}x{K} m={m} (sampled rows)")
