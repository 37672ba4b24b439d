"""Convenience wrappers over the C ABI: allocate the outputs with torch, then call libcq.

No arithmetic of the method happens here; every value is produced by a libcq kernel.
"""
import torch

from . import cq

GROUP = 64


def empty_u8(n, device):
    return torch.empty(int(n), dtype=torch.uint8, device=device)


def quantize(w, bits=None, stream=None):
    """fp32 [rows, cols] on the GPU -> (codes u8 [rows*cols], scale int16 [G] (fp16 bits), zero u8 [G], status)."""
    rows, cols = w.shape
    G = rows * cols // GROUP
    dev = w.device
    codes = empty_u8(rows * cols, dev)
    scale = torch.empty(G, dtype=torch.int16, device=dev)
    zero = empty_u8(G, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cq.cq_quantize(w, bits, codes, scale, zero, status, stream)
    return codes, scale, zero, status


def varbits_index(bits, stream=None):
    """-> (offset int32 [G], plane_bytes list of 4 ints).  Reads plane_bytes back (synchronizes)."""
    dev = bits.device
    offset = torch.empty(bits.numel(), dtype=torch.int32, device=dev)
    pb = torch.empty(4, dtype=torch.int64, device=dev)
    cq.cq_varbits_index(bits, offset, pb, stream)
    (stream if stream is not None else torch.cuda.current_stream()).synchronize()   # pb is read below
    return offset, [int(v) for v in pb.cpu()]


def pack(codes, rows, cols, bits=None, offset=None, plane_bytes=None, stream=None):
    """codes -> list of 4 planes (None where unused)."""
    G = rows * cols // GROUP
    dev = codes.device
    if bits is None:
        planes = [None, None, empty_u8(32 * G, dev), None]
    else:
        planes = [empty_u8(max(16, n), dev) for n in plane_bytes]
    cq.cq_pack_varbits(codes, G, bits, offset, planes, stream)
    return planes


def quantize_and_pack(w, bits=None, stream=None):
    """fp32 weights -> (QWeight, codes, status)."""
    rows, cols = w.shape
    codes, scale, zero, status = quantize(w, bits, stream)
    offset = pb = None
    if bits is not None:
        offset, pb = varbits_index(bits, stream)
    planes = pack(codes, rows, cols, bits, offset, pb, stream)
    return cq.QWeight(rows, cols, planes, scale, zero, bits, offset), codes, status


def unpack(qw, stream=None):
    codes = empty_u8(qw.rows * qw.cols, qw.scale.device)
    cq.cq_unpack_varbits(qw, codes, stream)
    return codes


def project(r, scale, stream=None):
    n = torch.zeros(1, dtype=torch.int64, device=r.device)
    cq.cq_project_residual(r, scale, n, stream)
    return n


def verify(qw, first_w=0, n_w=None, flags=False, stream=None):
    """-> (mismatches int64[1], first_bad int64[1], group_flags int32[...] or None), on the device."""
    dev = qw.scale.device
    if n_w is None:
        n_w = qw.rows * qw.cols - first_w
    mism = torch.empty(1, dtype=torch.int64, device=dev)
    first = torch.empty(1, dtype=torch.int64, device=dev)
    gf = None
    if flags:
        gf = torch.empty(max(1, (n_w // GROUP + 31) // 32), dtype=torch.int32, device=dev)
    cq.cq_requant_verify(qw, first_w, n_w, mism, first, gf, stream)
    return mism, first, gf


def verify_pair(qw, first_w=0, n_w=None, flags=False, stream=None):
    """-> (mismatches, first_bad, revoke_mismatches, revoke_first_bad, group_flags or None)."""
    dev = qw.scale.device
    if n_w is None:
        n_w = qw.rows * qw.cols - first_w
    out = [torch.empty(1, dtype=torch.int64, device=dev) for _ in range(4)]
    gf = None
    if flags:
        gf = torch.empty(max(1, (n_w // GROUP + 31) // 32), dtype=torch.int32, device=dev)
    cq.cq_requant_verify_pair(qw, first_w, n_w, out[0], out[1], out[2], out[3], gf, stream)
    return out[0], out[1], out[2], out[3], gf


def gemv(qw, x, stream=None):
    y = torch.empty((x.shape[0], qw.rows), dtype=torch.float32, device=x.device)
    cq.cq_dequant_gemv(qw, x, y, stream)
    return y


def gemv_multi(qws, x, stream=None):
    ys = [torch.empty((x.shape[0], q.rows), dtype=torch.float32, device=x.device) for q in qws]
    cq.cq_dequant_gemv_multi(qws, x, ys, stream)
    return ys


def gemm(qw, x, workspace=None, stream=None, check=True):
    """y = W x for a batch; with check, waits for the result and raises if the GEMM's status
    word (first 4 bytes of its workspace) says an internal wait gave up."""
    m = x.shape[0]
    y = torch.empty((m, qw.rows), dtype=torch.float32, device=x.device)
    need = cq.cq_gemm_workspace(qw.rows, qw.cols, m)
    if need and (workspace is None or workspace.numel() < need):
        # zero-filled: the word stays 0 when the call is served by the GEMV kernels instead
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    cq.cq_dequant_gemm(qw, x, y, workspace if need else None, stream)
    if check and need:
        word = int(workspace[:4].view(torch.int32).cpu()[0])   # synchronizes with the stream
        if word != 0:
            raise cq.CQError(7, f"cq_dequant_gemm: status word {word:#x} (an internal wait gave up)")
    return y


def rrq_build(w, n_stages, bits=2, stream=None):
    """Recurrent residual quantization of fp32 w [rows, cols] (left unchanged): n_stages
    stages of width `bits`, each packed -> (list of QWeight, statuses, final residual)."""
    rows, cols = w.shape
    G = rows * cols // GROUP
    dev = w.device
    r = w.clone()
    width = torch.full((G,), bits, dtype=torch.uint8, device=dev)
    offset, pb = varbits_index(width, stream)
    stages, statuses = [], []
    for _ in range(n_stages):
        codes = empty_u8(rows * cols, dev)
        scale = torch.empty(G, dtype=torch.int16, device=dev)
        zero = empty_u8(G, dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        cq.cq_rrq_stage(r, bits, codes, scale, zero, status, stream)
        planes = pack(codes, rows, cols, width, offset, pb, stream)
        stages.append(cq.QWeight(rows, cols, planes, scale, zero, width, offset))
        statuses.append(status)
    return stages, statuses, r


def gemv_stages(stages, x, stream=None):
    y = torch.empty((x.shape[0], stages[0].rows), dtype=torch.float32, device=x.device)
    cq.cq_dequant_gemv_stages(stages, x, y, stream)
    return y


def reparam(theta, scale, r_dtype=torch.bfloat16, stream=None):
    """Bounded reparameterization: theta (fp32 [n]) -> a residual of r_dtype inside every cell."""
    r = torch.empty(theta.numel(), dtype=r_dtype, device=theta.device)
    cq.cq_reparam_residual(theta, scale, r, stream)
    return r


def reparam_grad(theta, scale, grad_r, r_dtype=torch.bfloat16, stream=None):
    """dL/dtheta of reparam() from dL/dr (fp32 [n])."""
    g = torch.empty_like(theta)
    cq.cq_reparam_residual_grad(theta, scale, grad_r, g, cq.CQ_BF16 if r_dtype == torch.bfloat16 else cq.CQ_F32,
                                stream)
    return g


def requant_refine(w, H, scale, zero, codes, sweeps=1, bits=4, stream=None):
    """ReQuant on a copy of codes -> (codes, err_before, err_after, moves), all on the device."""
    rows = w.shape[0]
    q = codes.clone()
    eb = torch.empty(rows, dtype=torch.float64, device=w.device)
    ea = torch.empty(rows, dtype=torch.float64, device=w.device)
    mv = torch.empty(rows, dtype=torch.int64, device=w.device)
    ws = torch.empty(cq.cq_requant_workspace(*w.shape), dtype=torch.uint8, device=w.device)
    cq.cq_requant_refine(w, H, scale, zero, bits, q, sweeps, eb, ea, mv, ws, stream)
    return q, eb, ea, mv
