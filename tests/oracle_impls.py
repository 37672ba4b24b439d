"""Uniform adapters over the two oracle implementations (C and NumPy twin).

Every pin in ``oracle_pins.py`` takes one of these objects, so the same pin checks the C
oracle, the NumPy twin, and deliberately broken copies of the twin (``mutants``).
"""
import numpy as np

from oracle import c_oracle as co
from oracle import np_oracle as no


class COracle:
    name = "c"

    def quantize(self, w, bits=None):
        return co.quantize(w, bits)

    def varbits_index(self, bits):
        return co.varbits_index(bits)

    def pack(self, codes, bits=None):
        if bits is None:
            return co.pack(codes)
        off, pb = co.varbits_index(bits)
        return co.pack(codes, bits, off, pb)

    def unpack(self, planes, G, bits=None):
        off = None if bits is None else co.varbits_index(bits)[0]
        return co.unpack(planes, G, bits, off)

    def project_f32(self, r, scale):
        return co.project_f32(r, scale)

    def project_bf16(self, r, scale):
        return co.project_bf16(r, scale)

    def verify(self, planes, scale, zero, bits=None, r=None, r_dtype="f32"):
        off = None if bits is None else co.varbits_index(bits)[0]
        m, fb, flags = co.verify(planes, scale, zero, bits, off, r, r_dtype, want_flags=True)
        G = np.asarray(scale).size
        mask = ((flags[np.arange(G) // 32] >> (np.arange(G) % 32).astype(np.uint32)) & 1).astype(bool)
        return m, fb, mask

    def rrq_stage(self, r, b=2):
        return co.rrq_stage(r, b)

    def reparam_phi(self, theta):
        return co.reparam_phi(theta)

    def reparam(self, theta, scale, r_dtype="bf16"):
        return co.reparam(theta, scale, r_dtype)

    def reparam_grad(self, theta, scale, grad_r, r_dtype="bf16"):
        return co.reparam_grad(theta, scale, grad_r, r_dtype)

    def requant_refine(self, w, H, codes, scale, zero, b=4, sweeps=1):
        return co.requant_refine(w, H, codes, scale, zero, b, sweeps)

    def dequant_matmul_f64(self, planes, scale, zero, rows, cols, x, x_dtype="f32", bits=None,
                           r=None, r_dtype="f32"):
        off = None if bits is None else co.varbits_index(bits)[0]
        return co.dequant_matmul_f64(planes, scale, zero, rows, cols, x, x_dtype, bits, off, r,
                                     r_dtype)


class NpOracle:
    name = "np"

    def quantize(self, w, bits=None):
        return no.quantize(w, bits)

    def varbits_index(self, bits):
        return no.varbits_index(bits)

    def pack(self, codes, bits=None):
        return no.pack(codes, bits)

    def unpack(self, planes, G, bits=None):
        return no.unpack(planes, G, bits)

    def project_f32(self, r, scale):
        return no.project_f32(r, scale)

    def project_bf16(self, r, scale):
        return no.project_bf16(r, scale)

    def verify(self, planes, scale, zero, bits=None, r=None, r_dtype="f32"):
        return no.verify(planes, scale, zero, bits, r, r_dtype)

    def rrq_stage(self, r, b=2):
        return no.rrq_stage(r, b)

    def reparam_phi(self, theta):
        return float(no._reparam_phi(np.float32(theta)))

    def reparam(self, theta, scale, r_dtype="bf16"):
        return no.reparam(theta, scale, r_dtype)

    def reparam_grad(self, theta, scale, grad_r, r_dtype="bf16"):
        return no.reparam_grad(theta, scale, grad_r, r_dtype)

    def requant_refine(self, w, H, codes, scale, zero, b=4, sweeps=1):
        return no.requant_refine(w, H, codes, scale, zero, b, sweeps)

    def dequant_matmul_f64(self, planes, scale, zero, rows, cols, x, x_dtype="f32", bits=None,
                           r=None, r_dtype="f32"):
        return no.dequant_matmul_f64(planes, scale, zero, rows, cols, x, x_dtype, bits, r, r_dtype)


IMPLS = {"c": COracle(), "np": NpOracle()}
