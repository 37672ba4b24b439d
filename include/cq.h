/*
 * cq.h -- C ABI of libcq: group-wise low-bit weight quantization for NVIDIA B200 (sm_100a).
 *
 * The method follows two abstracts (cited by page title and section):
 *   [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
 *         Without Changing the File They Ship" (thelatestinai.com/papers/2608.20873),
 *         abstract: every contiguous group of 64 weights has its own bit-width from
 *         {1,2,4,8}; the codes are kept bit-packed at their widths; fused
 *         dequantize-and-multiply kernels serve memory-bound decode.
 *   [CF]  "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
 *         Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: a 4-bit release
 *         whose integer codes and scales stay frozen; updates live in a per-weight
 *         residual confined to the rounding cell of each weight; rounding again gives the
 *         released codes exactly; removing the residual undoes the update; the change
 *         of every weight is limited.
 *   [SLQ] listing page thelatestinai.com/papers/2512.18934, SLQ abstract: asymmetric
 *         quantization (hence the zero point).
 *
 * Quantizer (the pages do not print it; this is the reading every entry point uses):
 * a group of 64 consecutive weights along a row has an fp16 scale s, a uint8 zero z
 * and a width b; L = 2^b - 1;
 *     s = RN_fp16(RN32(RN32(wmax - wmin) / L)), floored at 2^-14
 *     z = clamp(rne(RN32(-wmin / s)), 0, L)
 *     q = clamp(rne(RN32(w / s)) + z, 0, L)                 (rne: ties to even)
 * and the served weight is W = s * (q - z) + r, r an optional per-weight residual.
 *
 * Conventions for every call:
 *  - Every pointer is a DEVICE pointer owned by the caller, unless the comment says host.
 *  - Matrices are row-major [rows, cols]; groups run along cols (the input dimension), so
 *    there are G = rows * cols / 64 groups, group g = row * (cols/64) + col/64.
 *  - Arguments are validated on the host before anything is enqueued; a bad argument
 *    returns a non-zero cq_status, launches nothing and sets cq_last_error().
 *  - Work is enqueued asynchronously on `stream` (NULL = legacy default stream). The
 *    library never synchronizes and never allocates device memory; results that the
 *    device computes (counts, flags, status words) land in caller memory.
 *  - A launch failure returns CQ_ERR_CUDA with the CUDA error text in cq_last_error().
 *  - Calls on different streams that write the same buffers race, as usual in CUDA.
 */
#ifndef CQ_H
#define CQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t, without pulling in the CUDA headers. */
typedef struct CUstream_st *cq_stream_t;

typedef enum {
    CQ_OK = 0,
    CQ_ERR_ARG = 1,         /* NULL where a pointer is required, bad enum, m out of range */
    CQ_ERR_SHAPE = 2,       /* negative sizes, cols % 64 != 0, chunk not on group bounds */
    CQ_ERR_BITS = 3,        /* a host-visible bit-width outside {1,2,4,8}                 */
    CQ_ERR_ALIGN = 4,       /* a pointer that must be 16-byte aligned is not              */
    CQ_ERR_NONFINITE = 5,   /* reserved: non-finite input reported synchronously          */
    CQ_ERR_RANGE = 6,       /* a size beyond what the format or a workspace can address   */
    CQ_ERR_CUDA = 7,        /* a CUDA launch or memset failed                             */
    CQ_ERR_UNSUPPORTED = 8  /* a valid combination this build has no kernel for           */
} cq_status;

typedef enum { CQ_F32 = 0, CQ_BF16 = 1 } cq_dtype;

/* bits of the device status word written by cq_quantize */
#define CQ_QSTATUS_NONFINITE 1u /* a group held a NaN or infinity: written as s=+0, z=0, q=0 */
#define CQ_QSTATUS_RANGE 2u     /* a group's scale overflowed fp16: written as s=+0, z=0, q=0 */
#define CQ_QSTATUS_BADBITS 4u   /* bits[g] not in {1,2,4,8}: written as s=+0, z=0, q=0        */
#define CQ_QSTATUS_TIMEOUT 8u   /* an internal wait gave up (never expected): outputs incomplete */

/*
 * A quantized weight matrix ([VBQ] bit-packed per-group widths, [CF] frozen codes + scales).
 * Packed layout: one plane per width b in {1,2,4,8} (plane[0..3] for b = 1,2,4,8). Group g
 * of width b occupies 8*b bytes of plane b starting at byte offset[g]; code j of the group
 * is in bits [j*b, (j+1)*b) of that little-endian byte string, least significant bit first.
 * offset[g] = 8*b * (number of earlier groups, in row-major group order, of the same width).
 * Fixed 4-bit ([CF] 4-bit release): bits = offset = NULL, plane[2] holds plain row-major
 * nibbles (offset 32*g; even column in the low nibble); the other planes are unused.
 */
typedef struct {
    int64_t rows, cols;       /* N (outputs) x K (inputs); cols % 64 == 0                  */
    const uint8_t *bits;      /* [G] widths in {1,2,4,8}, or NULL for all-4                */
    const uint32_t *offset;   /* [G] byte offsets into plane[width], NULL when bits NULL   */
    const uint8_t *plane[4];  /* planes for b = 1, 2, 4, 8; 16-byte aligned when used      */
    const uint16_t *scale;    /* [G] fp16 bit patterns                                     */
    const uint8_t *zero;      /* [G]                                                       */
    const void *residual;     /* [rows*cols] of residual_dtype, or NULL (revoked / none)   */
    cq_dtype residual_dtype;
} cq_qweight;

/*
 * cq_quantize -- [VBQ] per-group widths, [CF] 4-bit codes and scales, [SLQ] asymmetry.
 * w: [rows, cols] fp32 (16-byte aligned). bits: [G] widths or NULL (= 4 for every group).
 * codes: [rows*cols] one code per byte (16-byte aligned); scale: [G] fp16 bits; zero: [G].
 * status_word: one uint32 (device) that receives the OR of CQ_QSTATUS_* over all groups;
 * it is cleared by the call; may be NULL. Groups with a non-finite weight, an fp16-overflowing
 * scale or a bad width are written as s=+0, z=0, q=0 and flagged; the call still returns CQ_OK.
 */
cq_status cq_quantize(const float *w, int64_t rows, int64_t cols, const uint8_t *bits,
                      uint8_t *codes, uint16_t *scale, uint8_t *zero, uint32_t *status_word,
                      cq_stream_t stream);

/*
 * cq_rrq_stage -- one stage of Recurrent Residual Quantization ([RRQ] the listing page
 * thelatestinai.com/papers/2512.18934, "Recurrent Residual Quantization" abstract: a 2-bit
 * round-to-nearest base plus 2-bit round-to-nearest residual corrections stacked to 4, 6 and
 * 8 bits, so one artifact holds several precisions). The running residual r ([rows, cols]
 * fp32, 16-byte aligned; the weights themselves for the first stage) is quantized exactly as
 * cq_quantize does with one width `bits` (1, 2, 4 or 8) for every group, then replaced in
 * place by what the stage does not represent: r <- RN32(r - s*(q - z)) with the stored s, z
 * and codes (the product is exact); a flagged group keeps its r. codes/scale/zero/status_word
 * as for cq_quantize. Calling it J+1 times (bits = 2) on the same buffer yields the stages of a
 * 2(J+1)-bit model; pack each stage with cq_pack_varbits (a width map of `bits`).
 * Errors: CQ_ERR_SHAPE (cols % 64), CQ_ERR_BITS (width), CQ_ERR_ARG (NULL), CQ_ERR_ALIGN.
 */
cq_status cq_rrq_stage(float *r, int64_t rows, int64_t cols, int bits, uint8_t *codes, uint16_t *scale,
                       uint8_t *zero, uint32_t *status_word, cq_stream_t stream);

/*
 * cq_dequant_gemv_stages -- the multiply over an RRQ stage stack ([RRQ] as above): y[m, rows]
 * (fp32, overwritten) = sum over k of (sum over stages j of s_j (q_j - z_j)) * x[m, k], for
 * 1 <= count <= 8 stages of the same shape, each fixed-4 or with a per-group width map, none
 * with a residual (CQ_ERR_UNSUPPORTED), 1 <= m <= 8, x fp32 or bf16 (16-byte aligned). Each
 * stage's group adds s_j * (sum over the group of (q_j - z_j) x), the group sum in fp32: at
 * m = 1 on CUDA cores (x rounded to fp32, exact for bf16), at m >= 2 on tensor cores with exact
 * products (as cq_dequant_gemv). fp32 accumulation either way.
 * Errors: CQ_ERR_ARG (count, NULL, m, dtype), CQ_ERR_SHAPE (unequal shapes), CQ_ERR_ALIGN.
 */
cq_status cq_dequant_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype x_dtype,
                                 int m, float *y, cq_stream_t stream);

/*
 * cq_varbits_index -- [VBQ] codes stored bit-packed at their group widths: builds offset[G] (byte
 * offsets as in cq_qweight) and plane_bytes[4] (device, uint64: bytes needed by each plane).
 * bits: [G]. Device-side, widths outside {1,2,4,8} count as width 0 (offset 0, no bytes);
 * pack and quantize flag them. n_groups <= 2^26 (byte offsets are 32-bit) else CQ_ERR_RANGE.
 * The offset array also serves as the call's temporary storage, so it must not alias bits.
 */
cq_status cq_varbits_index(const uint8_t *bits, int64_t n_groups, uint32_t *offset,
                           uint64_t *plane_bytes, cq_stream_t stream);

/*
 * cq_pack_varbits -- codes (one per byte, [n_groups*64]) -> planes, in the cq_qweight layout.
 * bits/offset NULL: fixed 4-bit into plane[2]. Only the low b bits of each code are stored.
 * plane[i] must hold plane_bytes[i] bytes and be 16-byte aligned when used; codes 16-byte aligned.
 */
cq_status cq_pack_varbits(const uint8_t *codes, int64_t n_groups, const uint8_t *bits,
                          const uint32_t *offset, uint8_t *const plane[4], cq_stream_t stream);

/* cq_unpack_varbits -- the inverse of cq_pack_varbits: qw's planes -> codes [rows*cols]. */
cq_status cq_unpack_varbits(const cq_qweight *qw, uint8_t *codes, cq_stream_t stream);

/*
 * cq_project_residual -- [CF] clamping the residual back into its rounding cell, in place:
 *     r <- c if r > c;  -c if r < -c;  r otherwise,   c = (0.5 - 2^-10) * s_group,
 * for fp32 r; for bf16 r the bound is c rounded toward zero to bf16 (never outward).
 * A NaN residual is left as it is (requant-verify then reports it). r: [n] (16-byte aligned),
 * n % 64 == 0, element i belongs to group i/64 of scale. n_clamped: one uint64 (device) that
 * receives the number of elements whose bits changed; cleared by the call; may be NULL.
 */
cq_status cq_project_residual(void *r, cq_dtype dtype, const uint16_t *scale, int64_t n,
                              uint64_t *n_clamped, cq_stream_t stream);

/*
 * cq_reparam_residual -- [CF] Abstract, CellFill as a bounded reparameterization: the update is
 * trained as an unconstrained parameter theta and served as a residual that lies in its
 * weight's cell whatever theta is, so the release re-quantizes to its codes with no projection
 * step. The map is not printed on the page; this library's reading:
 *     r_i = RN(c_dt * phi(theta_i)),   phi(t) = t / sqrt(1 + t^2)
 * c_dt: the bound cq_project_residual clamps to ((0.5 - 2^-10) * s for fp32 r; that value
 * rounded toward zero to bf16 for bf16 r); s the scale of weight i's group. phi is evaluated
 * as the binary32 steps u = RN(t*t), d = RN(1 + u), q = RN(sqrt(d)), phi = RN(t / q) (correctly
 * rounded, no contraction), then the fp32 product, then for bf16 r one round to nearest
 * bf16: the same bits on any IEEE-754 machine. |r| <= c_dt for every theta: +-inf gives +-c_dt,
 * |theta| > 2^32 gives phi = +-1, and a NaN theta gives r = +0 (that weight's update revoked).
 * theta: [n] fp32; r: [n] of r_dtype (overwritten); both 16-byte aligned; n % 64 == 0; element
 * i belongs to group i/64 of scale. Errors: CQ_ERR_SHAPE, CQ_ERR_ARG (NULL, dtype), CQ_ERR_ALIGN.
 */
cq_status cq_reparam_residual(const float *theta, const uint16_t *scale, int64_t n, void *r,
                              cq_dtype r_dtype, cq_stream_t stream);

/*
 * cq_reparam_residual_grad -- the backward pass of cq_reparam_residual for training theta,
 * straight through its final rounding: grad_theta_i = RN(RN(grad_r_i * c_dt) * phi'(theta_i)),
 * phi'(t) = (1 + t^2)^(-3/2) evaluated as RN(RN(1 / d) / q) with d and q as in the forward
 * pass; 0 for a NaN theta or |theta| > 2^32. grad_r: [n] fp32 (dL/dr); grad_theta: [n] fp32
 * (overwritten); r_dtype selects c_dt as in the forward pass. Alignment and errors as there.
 */
cq_status cq_reparam_residual_grad(const float *theta, const uint16_t *scale, const float *grad_r,
                                   int64_t n, cq_dtype r_dtype, float *grad_theta, cq_stream_t stream);

/*
 * cq_requant_refine -- ReQuant fixed-grid refinement (page 1, thelatestinai.com/papers/2608.20873,
 * ReQuant abstract: a backpropagation-free stage that revisits an existing quantized model's
 * integer assignments on its fixed grid, every accepted update strictly lowering the mean squared
 * reconstruction error; several sweeps over a round-to-nearest start). This library's reading:
 * the error is the layer's output error on calibration activations X,
 *     E(q) = sum_n d_n^T H d_n,   d_n = w_n - s (q_n - z),   H = X^T X,
 * the scales and zero points stay as they are, and an update moves one code to a neighbouring
 * level of the grid (q +- 1 within [0, 2^bits - 1]). Each of `sweeps` sweeps visits every row's
 * codes in order; a move is taken only if it lowers E strictly (of the two, the larger decrease;
 * up on a tie). Rows are refined independently. All arithmetic is binary64 in a fixed order
 * without fused multiply-adds, so the codes are the same on any IEEE-754 machine that keeps it.
 * w: [rows, cols] fp32 (the weights before quantization); H: [cols, cols] fp64, symmetric
 * (H[j, k] == H[k, j] bit for bit), 8-byte aligned; scale/zero: [G]; codes: [rows*cols], one code
 * per byte, refined in place (pack them with cq_pack_varbits). err_before / err_after: NULL or
 * [rows] fp64, E of each row before and after; moves: NULL or [rows] uint64, accepted updates.
 * workspace: at least cq_requant_workspace(rows, cols) bytes of device scratch (8-byte aligned).
 * One width `bits` for every group. cols may be at most 25600 (a row's state is kept on chip;
 * CQ_ERR_UNSUPPORTED beyond). Errors: CQ_ERR_SHAPE, CQ_ERR_BITS, CQ_ERR_ARG, CQ_ERR_RANGE
 * (workspace too small), CQ_ERR_ALIGN.
 */
cq_status cq_requant_refine(const float *w, int64_t rows, int64_t cols, const double *H,
                            const uint16_t *scale, const uint8_t *zero, int bits, uint8_t *codes,
                            int sweeps, double *err_before, double *err_after, uint64_t *moves,
                            void *workspace, size_t workspace_bytes, cq_stream_t stream);

/* Bytes of workspace cq_requant_refine needs (host function, no GPU work). */
size_t cq_requant_workspace(int64_t rows, int64_t cols);

/*
 * cq_requant_verify -- [CF] rounding the served weights again must give the released codes
 * exactly, and with the residual removed (qw->residual = NULL) the update is undone. For weight i in
 * [first_w, first_w + n_w) with code q, scale s, zero z, width b:
 *     w' = RN32(RN32(s*(q-z)) + r_i);  t = RN32(w'/s);  q' = clamp(rne(t) + z, 0, 2^b-1)
 * and a mismatch is q' != q (a NaN t is a mismatch). first_w and n_w are multiples of 64
 * and the range lies inside the matrix (chunks let a 2.4e10-weight check run piecewise).
 * mismatches: one uint64 (device) <- count; first_bad: one int64 (device) <- smallest
 * mismatching index or -1; group_flags: NULL or ceil(n_w/64/32) uint32 (device), bit j set
 * when group first_w/64 + j holds a mismatch. All three are cleared by the call. A mismatch
 * is a result, not an error. The residual must be 16-byte aligned.
 */
cq_status cq_requant_verify(const cq_qweight *qw, int64_t first_w, int64_t n_w,
                            uint64_t *mismatches, int64_t *first_bad, uint32_t *group_flags,
                            cq_stream_t stream);

/*
 * cq_requant_verify_pair -- both [CF] guarantees in one pass over a fixed-4 artifact with a
 * residual: the served weights s(q-z)+r re-quantize to the codes (mismatches, first_bad, and
 * group_flags if not NULL, exactly as cq_requant_verify with the residual), and dropping the
 * residual revokes the update (revoke_mismatches, revoke_first_bad, exactly as
 * cq_requant_verify with residual = NULL). The codes and metadata are read once. Per-group-width
 * artifacts are checked in two passes with the same results. qw->residual must be set
 * (CQ_ERR_ARG); other arguments and errors as for cq_requant_verify.
 */
cq_status cq_requant_verify_pair(const cq_qweight *qw, int64_t first_w, int64_t n_w, uint64_t *mismatches,
                                 int64_t *first_bad, uint64_t *revoke_mismatches, int64_t *revoke_first_bad,
                                 uint32_t *group_flags, cq_stream_t stream);

/*
 * cq_dequant_gemv -- [VBQ] fused dequantize-and-multiply for decode:
 *     y[i, n] = sum_k (s*(q-z) + r)[n, k] * x[i, k],   i < m, 1 <= m <= 8,
 * products accumulated in fp32. x: [m, cols] of x_dtype (16-byte aligned); y: [m, rows] fp32.
 * y is overwritten. Fixed-4 weights with bf16 x and no residual run on tensor cores (mma.sync,
 * exact products, fp32 accumulation; the zero point enters through the group sums of x). Per-
 * group widths, and fp32 x, without a residual: at m = 1 on CUDA cores, per group the fp32 sum of
 * (q - z) x (q - z exact) scaled by s; at m >= 2 on tensor cores with q - z as exact bf16
 * operands (fp32 x split into two bf16 parts, |x - hi - lo| <= 2^-17 |x|), the scale applied to
 * each group's fp32 sum. Weights that carry a residual run on an fp32 CUDA-core path.
 */
cq_status cq_dequant_gemv(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m,
                          float *y, cq_stream_t stream);

/*
 * cq_dequant_gemv_multi -- cq_dequant_gemv for several matrices that read the same x (the q, k
 * and v projections of a decoder layer, or its gate and up projections) in as few launches as
 * possible: consecutive runs of up to four fixed-4 matrices with bf16 x and no residual become
 * one tensor-core launch whose 16-row tiles cover all of them; any other matrix runs as in
 * cq_dequant_gemv. qws: count pointers to matrices that all have the same cols; x: [m, cols];
 * ys[i]: [m, qws[i]->rows] fp32, overwritten. Each output is the same contraction as
 * cq_dequant_gemv computes (same tolerance; the order of the fp32 partial sums can differ).
 * Validation is that of cq_dequant_gemv for every matrix, plus CQ_ERR_SHAPE for unequal cols.
 * The pages have no counterpart to the grouping: it serves decode, where one token runs many
 * small GEMVs and launch latency rivals the weight stream.
 */
cq_status cq_dequant_gemv_multi(const cq_qweight *const *qws, int count, const void *x, cq_dtype x_dtype,
                                int m, float *const *ys, cq_stream_t stream);

/*
 * cq_dequant_gemm -- the same contraction for a batch, 1 <= m <= 256. Fixed-4 weights with
 * bf16 x, no residual and m >= 16 run on the sm_100a tcgen05 tensor cores with accumulators
 * in tensor memory; m < 16 goes to the GEMV kernels, as do other formats (in slices of 8).
 * On the tensor cores each weight s * (q - z) is rounded once to fp16 (relative error below
 * 2^-11) and x is copied to fp16 with an exact power of two per row; groups with |s| > 4096,
 * a non-finite s or z > 15 are summed in fp32 instead (slowly). x must be 16-byte aligned
 * there (CQ_ERR_ALIGN otherwise).
 * workspace: caller-owned device scratch of at least cq_gemm_workspace(rows, cols, m) bytes
 * (may be NULL when that is 0), 16-byte aligned; it holds the fp16 copy of x and a status
 * word (first 4 bytes, non-zero if an internal wait gave up). y: [m, rows] fp32, overwritten.
 */
cq_status cq_dequant_gemm(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m,
                          float *y, void *workspace, size_t workspace_bytes, cq_stream_t stream);

/*
 * cq_dequant_gemm_static -- cq_dequant_gemm for callers that cannot allocate device memory:
 * no workspace argument, and no cudaMalloc, cudaFree or other allocating call inside. It is
 * meant for code that runs where allocation is not allowed or not wanted after start-up: a
 * plug-in that is handed device buffers by a host framework that owns all device memory, or a
 * serving loop with a fixed memory budget where an allocation could block on the device or
 * fail at the worst moment. The pages have no counterpart to this call.
 * Its scratch is an 8 MiB array inside the library that every GPU which loads the library
 * keeps until the process exits. A shape that would need more scratch than that is refused
 * with CQ_ERR_RANGE: the tensor-core GEMM needs 512 + 2 * min(m, 64) * cols bytes, so with
 * m >= 64 cols may be at most 65532. Arguments are checked first, so a bad call does no CUDA
 * work; the first valid call on a device then looks up the array's device address with that
 * device current (make that first call before any stream capture). All calls share the array
 * and the call clears what must start at zero, but calls that overlap on the GPU (other
 * streams, other threads) race on it.
 * status_word: NULL, or one uint32 (device) that receives, in stream order after the multiply,
 * the tensor-core GEMM's status word: 0, or non-zero if an internal wait gave up (y is then
 * incomplete). Shapes served by the GEMV kernels write 0 there (those mark an aborted output
 * with NaN instead).
 * Arguments, results and errors are otherwise those of cq_dequant_gemm.
 */
cq_status cq_dequant_gemm_static(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m,
                                 float *y, uint32_t *status_word, cq_stream_t stream);

/* Bytes of workspace cq_dequant_gemm needs for this shape (host function, no GPU work). */
size_t cq_gemm_workspace(int64_t rows, int64_t cols, int m);

/*
 * cq_debug_word -- the debug build's record of a failed in-kernel index check. A library built
 * with -DCQ_DEBUG checks the derived indices of its kernels (rows and columns of outputs,
 * shared-memory and tensor-memory slots, group indices, packed-offset alignment); a failing
 * check skips the access it guards and records its site, (unit << 8) | n, in a device word (the
 * first failure wins) instead of trapping. This call waits for the device to finish
 * (cudaDeviceSynchronize), stores in *word (host) the first non-zero site over all units, or 0,
 * and clears every unit's record. A release build (the default) has no checks: *word = 0 and
 * CQ_ERR_UNSUPPORTED. Errors: CQ_ERR_ARG (word NULL), CQ_ERR_CUDA.
 */
cq_status cq_debug_word(uint32_t *word);

/*
 * cq_debug_selftest -- debug build only: enqueues one kernel whose index check fails on purpose
 * (site 0x0F01, the access it guards skipped), so that a test can see cq_debug_word report it.
 * A release build returns CQ_ERR_UNSUPPORTED and enqueues nothing.
 */
cq_status cq_debug_selftest(cq_stream_t stream);

/* Text of the last non-OK status returned on the calling thread (thread-local, host). */
const char *cq_last_error(void);

/* Name of a status code (host). */
const char *cq_status_string(cq_status status);

#ifdef __cplusplus
}
#endif
#endif /* CQ_H */
