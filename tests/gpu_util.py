"""Helpers for the GPU parity tests: host<->device moves and the matmul tolerance of the
benchmark spec (relative Frobenius error <= 2e-3, per-element |err| <= 1e-2 rms(y))."""
import numpy as np
import torch

REL_FRO = 2e-3
MAX_OVER_RMS = 1e-2


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def host(t, np_dtype=None):
    a = t.detach().cpu()
    if np_dtype is not None:
        if a.dtype in (torch.int16, torch.bfloat16, torch.float16):
            a = a.view(torch.int16).numpy().view(np.uint16)
        elif a.dtype == torch.int32:
            a = a.numpy().view(np.uint32)
        else:
            a = a.numpy()
        return a.astype(np_dtype, copy=False)
    return a.numpy()


def bf16_dev(bits_u16):
    return dev(np.asarray(bits_u16, np.uint16).view(np.int16), None).view(torch.bfloat16)


def u16_dev(bits_u16):
    return dev(np.asarray(bits_u16, np.uint16).view(np.int16))


def planes_host(qw):
    return [host(p) if p is not None else np.zeros(1, np.uint8) for p in qw.planes]


def check_matmul(y_gpu, y_ref, what=""):
    y = np.asarray(y_gpu, np.float64)
    ref = np.asarray(y_ref, np.float64)
    err = y - ref
    fro = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref ** 2))
    mx = np.abs(err).max() / max(rms, 1e-300)
    assert fro <= REL_FRO and mx <= MAX_OVER_RMS, f"{what}: relF={fro:.3e} max/rms={mx:.3e}"
    return fro, mx


# ---- guard bands: a stand-in for a memory checker -------------------------------------------
GUARD_BYTES = 4096
SENTINEL = 0xA5


class Guarded:
    """A device buffer of `numel` elements of `dtype` with GUARD_BYTES of sentinel bytes on each
    side (the buffer itself keeps 16-byte alignment). After a call, check() asserts that no
    kernel wrote outside the buffer."""

    def __init__(self, numel, dtype, fill=None):
        esize = torch.empty(0, dtype=dtype).element_size()
        self.nbytes = int(numel) * esize
        self.raw = torch.full((self.nbytes + 2 * GUARD_BYTES,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype)
        if fill is not None:
            self.t.copy_(fill.reshape(-1).view(dtype) if torch.is_tensor(fill) else torch.as_tensor(fill))

    def check(self, what):
        torch.cuda.synchronize()
        pre = self.raw[:GUARD_BYTES]
        post = self.raw[GUARD_BYTES + self.nbytes:]
        bad_pre = int((pre != SENTINEL).sum())
        bad_post = int((post != SENTINEL).sum())
        assert bad_pre == 0 and bad_post == 0, f"{what}: {bad_pre} bytes written before, {bad_post} after the buffer"
