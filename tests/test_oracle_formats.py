"""The oracle's own fp16/bf16 converters (written from IEEE-754) against library
conversions: NumPy's float16 and PyTorch's bfloat16, which round to nearest even."""
import numpy as np
import torch

from oracle import c_oracle as co

LOW = np.array([0x0000, 0x0001, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x2000, 0x3000, 0x6000,
                0x7FFF, 0x8000, 0x8001, 0xE000, 0xFFFF], np.uint32)


def _sample_f32():
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    bits = (hi[:, None] | LOW[None, :]).ravel()
    x = bits.view(np.float32)
    return x[~np.isnan(x)]


def test_f32_to_f16_matches_numpy():
    x = _sample_f32()
    got = co.f32_to_f16_bits(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_f16_to_f32_exhaustive():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    h = h[~np.isnan(h.view(np.float16))]
    got = co.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_bf16_rn_matches_torch():
    x = _sample_f32()
    got = co.f32_to_bf16_rn_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rz_is_truncation_toward_zero():
    x = _sample_f32()
    x = x[np.isfinite(x)]
    got = (co.f32_to_bf16_rz_bits(x).astype(np.uint32) << 16).view(np.float32)
    ax, ag = np.abs(x.astype(np.float64)), np.abs(got.astype(np.float64))
    assert (ag <= ax).all() and (np.sign(got) * np.sign(x) >= 0).all()
    # the next bf16 away from zero is strictly above |x|
    nxt = ((co.f32_to_bf16_rz_bits(np.abs(x)).astype(np.uint32) + 1) << 16).view(np.float32)
    fin = np.isfinite(nxt)
    assert (nxt[fin].astype(np.float64) > ax[fin]).all()
