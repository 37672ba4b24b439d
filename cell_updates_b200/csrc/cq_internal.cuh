// cq_internal.cuh -- shared declarations of libcq (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/cq.h"
#include "cq_debug.cuh"

namespace cq {

constexpr int kGroup = 64;  // [VBQ] abstract: contiguous groups of 64 weights

// ---- host-side helpers ----------------------------------------------------------------
cq_status fail(cq_status st, const char *fmt, ...);   // records cq_last_error(), returns st
cq_status cuda_check(cudaError_t e, const char *what);  // CQ_OK or CQ_ERR_CUDA
cq_status launch_check(const char *what);               // cudaGetLastError() after a launch
int sm_count();                                          // cached per device, thread-safe

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned8(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// ---- kernel launchers (each file owns its kernels) ----------------------------------
cq_status launch_quantize(const float *w, int64_t G, const uint8_t *bits, uint8_t *codes,
                          uint16_t *scale, uint8_t *zero, uint32_t *status, cudaStream_t s);
cq_status launch_varbits_index(const uint8_t *bits, int64_t G, uint32_t *offset,
                               uint64_t *plane_bytes, cudaStream_t s);
cq_status launch_pack(const uint8_t *codes, int64_t G, const uint8_t *bits,
                      const uint32_t *offset, uint8_t *const plane[4], cudaStream_t s);
cq_status launch_unpack(const cq_qweight &qw, uint8_t *codes, cudaStream_t s);
cq_status launch_project(void *r, cq_dtype dt, const uint16_t *scale, int64_t n,
                         uint64_t *n_clamped, cudaStream_t s);
cq_status launch_verify(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism,
                        int64_t *first_bad, uint32_t *flags, cudaStream_t s);
cq_status launch_verify_pair(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism, int64_t *first_bad,
                             uint64_t *mism0, int64_t *first0, uint32_t *flags, cudaStream_t s);
cq_status launch_gemv(const cq_qweight &qw, const void *x, cq_dtype xdt, int m, float *y,
                      cudaStream_t s);
cq_status launch_gemv_multi(const cq_qweight *const *qws, int count, const void *x, cq_dtype xdt, int m,
                            float *const *ys, cudaStream_t s);
cq_status launch_gemm_tc(const cq_qweight &qw, const void *x, int m, float *y, void *ws,
                         size_t ws_bytes, cudaStream_t s);
size_t gemm_tc_workspace(int64_t rows, int64_t cols, int m);
cq_status launch_rrq_stage(float *r, int64_t G, int b, uint8_t *codes, uint16_t *scale, uint8_t *zero,
                           uint32_t *status, cudaStream_t s);
constexpr int kMaxRrqStages = 8;
cq_status launch_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype xdt, int m,
                             float *y, cudaStream_t s);
bool gemm_tc_eligible(const cq_qweight &qw, cq_dtype xdt, int m);
cq_status launch_requant(const float *w, int64_t N, int64_t K, const double *H, const uint16_t *scale,
                         const uint8_t *zero, int b, uint8_t *codes, int sweeps, double *err_before, double *err_after,
                         uint64_t *moves, double *g, cudaStream_t s);
size_t requant_workspace(int64_t rows, int64_t cols);
int64_t requant_max_cols();
cq_status launch_reparam(const float *theta, const uint16_t *scale, int64_t n, void *r, cq_dtype dt,
                         cudaStream_t s);
cq_status launch_reparam_grad(const float *theta, const uint16_t *scale, const float *grad_r, int64_t n, cq_dtype dt,
                              float *grad_theta, cudaStream_t s);
// the argument checks every matmul entry point shares (cq_api.cu)
cq_status check_matmul_args(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m, float *y, int max_m,
                            const char *fn);

// ---- device-side helpers -------------------------------------------------------------
__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// integer clamp of a value that rne() left in a float: same answer as exact integer
// arithmetic, since |v| >= 2^24 lies far outside [0, L] on the same side
__device__ __forceinline__ int clamp_code(float v, int L) {
  return v < 0.0f ? 0 : (v > static_cast<float>(L) ? L : static_cast<int>(v));
}

__device__ __forceinline__ int width_slot(int b) { return b == 1 ? 0 : b == 2 ? 1 : b == 4 ? 2 : 3; }
__device__ __forceinline__ bool width_ok(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }

}  // namespace cq

namespace cq {

// rne(RN32(x / s)) for a finite s > 0 with rc = RN32(1/s), without a division in the common
// case. qt = RN32(x * rc) is within |x/s| * (2^-23 + 2^-48) of x/s, and RN32(x/s) within
// |x/s| * 2^-24; for |qt| < 512 the two differ by less than 1e-4, so when qt lies within
// 0.4995 of its nearest integer (more than 5e-4 from a half-way point) that integer is also
// the nearest integer of RN32(x/s). Otherwise (near a tie, large or non-finite) the IEEE
// division decides. This is an
// error-bound filter with an exact fallback, in the manner of adaptive exact predicates.
__device__ __forceinline__ float rne_quotient(float x, float s, float rc) {
  const float qt = __fmul_rn(x, rc);
  const float tr = rintf(qt);
  if (fabsf(__fsub_rn(qt, tr)) < 0.4995f && fabsf(qt) < 512.0f) return tr;
  return rintf(__fdiv_rn(x, s));
}

}  // namespace cq
