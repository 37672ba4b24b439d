"""Seeded synthetic inputs (host side).

This module only makes inputs: weights, activations, per-group bit-widths and residuals
with the shapes and distributions of the workloads the quantization pages describe.
It holds none of the quantizer's arithmetic, so the CUDA path and the CPU oracle can
both take their inputs from it.

Two families of generators:

* NumPy ``default_rng(seed)`` draws (normal, Student-t with outliers, categorical
  bit-widths, uniform residuals) for the matrices that fit in host memory;
* a counter-based generator, SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014; output function as in Vigna's public
  reference ``splitmix64.c``), used for inputs too large to build on the host.  The
  value at index ``i`` of stream ``(seed, stream)`` is the ``(i+1)``-th SplitMix64 output
  from the state ``key = mix(seed * GAMMA + stream)``.  Every value derived from it uses
  only integer operations and single IEEE binary32 multiplies, so the device generator
  in ``csrc/synth.cu`` (an independent implementation of the same definition) gives
  bit-identical values.
"""
import math

import numpy as np

GROUP = 64

# ---- SplitMix64 --------------------------------------------------------------------------

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream identifiers of the counter-based generator (shared numbering with csrc/synth.cu)
STREAM_WEIGHT = 1
STREAM_CODE = 2
STREAM_SCALE = 3
STREAM_ZERO = 4
STREAM_RESID = 5


def mix64(z):
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return mix64(np.uint64(seed) * GAMMA + np.uint64(stream))


def hash_u64(seed: int, stream: int, idx):
    """SplitMix64 output number idx+1 of the stream (idx: int64 array)."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(stream_key(seed, stream) + (idx + np.uint64(1)) * GAMMA)


# Irwin-Hall(4) approximation of a normal: the sum of the four 16-bit fields of one
# 64-bit output, centred.  Its standard deviation is sqrt(4 * (65536^2 - 1) / 12).
IH4_CENTER = 2 * 65535
IH4_STD = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)


def ih4_int(u):
    u = np.asarray(u, dtype=np.uint64)
    m = np.uint64(0xFFFF)
    s = (u & m) + ((u >> np.uint64(16)) & m) + ((u >> np.uint64(32)) & m) + (u >> np.uint64(48))
    return s.astype(np.int64) - IH4_CENTER


def ih4_multiplier(sigma: float) -> np.float32:
    """binary32 factor that maps the centred Irwin-Hall integer to standard deviation sigma."""
    return np.float32(sigma / IH4_STD)


def hashed_normal_f32(seed, stream, idx, sigma):
    """value_i = float32(d_i) * float32(sigma / IH4_STD): one binary32 multiply."""
    d = ih4_int(hash_u64(seed, stream, idx)).astype(np.float32)   # |d| < 2^18: exact
    return d * ih4_multiplier(sigma)


# Constrained synthetic 4-bit artifact (codes, scales, zeros) for the chunked
# re-quantization check at 2.4e10 weights, where a float matrix cannot be held.
def hashed_code_words(seed, word_idx):
    """64-bit words of row-major nibble codes: word j holds the codes of weights 16j..16j+15."""
    return hash_u64(seed, STREAM_CODE, word_idx)


def hashed_scales(seed, group_idx):
    """fp16 scale bits in [2^-8, 2^-7): exponent fixed, 10 mantissa bits from the hash."""
    return (np.uint64(0x1C00) | (hash_u64(seed, STREAM_SCALE, group_idx) & np.uint64(0x3FF))).astype(np.uint16)


def hashed_zeros(seed, group_idx):
    return ((hash_u64(seed, STREAM_ZERO, group_idx) >> np.uint64(20)) & np.uint64(0xF)).astype(np.uint8)


def f16_bits_to_f32(h):
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float32)


def hashed_residual_bf16(seed, idx, scale_bits_of_idx, rel_sigma):
    """bf16 bits of r_i = RN_bf16(float32(d_i) * RN32(s_f * k)), k = float32(rel_sigma/IH4_STD).

    The residual is a draw of N(0, (rel_sigma * s)^2) with s the weight's group scale.
    """
    k = ih4_multiplier(rel_sigma)
    d = ih4_int(hash_u64(seed, STREAM_RESID, idx)).astype(np.float32)
    mult = f16_bits_to_f32(scale_bits_of_idx) * k
    v = (d * mult).astype(np.float32)
    return f32_to_bf16_bits(v)


def f32_to_bf16_bits(v):
    """Round-to-nearest-even binary32 -> bfloat16 (bit patterns), finite inputs."""
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---- NumPy default_rng draws ---------------------------------------------------------------

def normal_weights(rows, cols, seed, sigma=0.02):
    """W ~ N(0, sigma^2), float32 [rows, cols]."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma)


def student_t_weights(rows, cols, seed, nu=5.0, scale=0.02, outlier_frac=1e-3, outlier_mult=10.0):
    """W = scale * t(nu), with a fraction of entries (chosen without replacement) x outlier_mult."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_t(nu, size=(rows, cols)) * scale).astype(np.float32)
    n_out = int(round(outlier_frac * rows * cols))
    if n_out:
        pos = rng.choice(rows * cols, size=n_out, replace=False)
        w.reshape(-1)[pos] *= np.float32(outlier_mult)
    return w


VBQ_WIDTHS = (1, 2, 4, 8)
VBQ_PROBS = (0.69, 0.15, 0.12, 0.04)   # the allocation statistics of the VBQ abstract


def vbq_bits(G, seed, probs=VBQ_PROBS):
    rng = np.random.default_rng(seed)
    return rng.choice(np.array(VBQ_WIDTHS, np.uint8), size=G, p=probs).astype(np.uint8)


def activations(m, K, seed, dtype="bf16"):
    """x ~ N(0, 1) [m, K]: float32 array, or bf16 bit patterns (uint16) when dtype == 'bf16'."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, K), dtype=np.float32)
    return f32_to_bf16_bits(x).reshape(m, K) if dtype == "bf16" else x


def uniform_residual_f32(scale_bits, seed, lo=-0.6, hi=0.6):
    """r ~ U(lo*s, hi*s) per weight (float32 [G*64]), s the weight's group scale."""
    rng = np.random.default_rng(seed)
    G = np.asarray(scale_bits).size
    u = rng.uniform(lo, hi, size=(G, GROUP)).astype(np.float32)
    return (u * f16_bits_to_f32(scale_bits)[:, None]).astype(np.float32).ravel()


def normal_residual_bf16(scale_bits, seed, rel_sigma=0.3):
    """r ~ N(0, (rel_sigma*s)^2) per weight, as bf16 bit patterns [G*64]."""
    rng = np.random.default_rng(seed)
    G = np.asarray(scale_bits).size
    u = rng.standard_normal((G, GROUP), dtype=np.float32) * np.float32(rel_sigma)
    return f32_to_bf16_bits(u * f16_bits_to_f32(scale_bits)[:, None]).ravel()
