// cq_api.cu -- the C ABI of libcq: argument validation and dispatch (see include/cq.h).
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "cq_internal.cuh"

namespace cq {

namespace {
thread_local char g_last_error[512] = "";

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
std::once_flag g_sm_once[kMaxDevices];
}  // namespace

cq_status fail(cq_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

cq_status cuda_check(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return CQ_OK;
  return fail(CQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

cq_status launch_check(const char *what) { return cuda_check(cudaGetLastError(), what); }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::call_once(g_sm_once[dev], [dev] {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  });
  return g_sm_count[dev];
}

namespace {

static bool width_ok_host(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }

cq_status check_shape(int64_t rows, int64_t cols, const char *fn) {
  if (rows < 0 || cols < 0) return fail(CQ_ERR_SHAPE, "%s: negative shape %lld x %lld", fn, (long long)rows, (long long)cols);
  if (cols % kGroup) return fail(CQ_ERR_SHAPE, "%s: cols=%lld is not a multiple of 64", fn, (long long)cols);
  if (cols && rows > INT64_MAX / cols) return fail(CQ_ERR_RANGE, "%s: rows*cols overflows", fn);
  return CQ_OK;
}

// the parts of a cq_qweight every consumer needs
cq_status check_qweight(const cq_qweight *qw, const char *fn, bool need_residual_align) {
  if (!qw) return fail(CQ_ERR_ARG, "%s: qweight is NULL", fn);
  cq_status st = check_shape(qw->rows, qw->cols, fn);
  if (st != CQ_OK) return st;
  const int64_t n = qw->rows * qw->cols;
  if (n == 0) return CQ_OK;
  if (!qw->scale || !qw->zero) return fail(CQ_ERR_ARG, "%s: scale/zero is NULL", fn);
  if ((qw->bits == nullptr) != (qw->offset == nullptr))
    return fail(CQ_ERR_ARG, "%s: bits and offset must both be set or both be NULL", fn);
  if (!qw->bits) {
    if (!qw->plane[2]) return fail(CQ_ERR_ARG, "%s: plane[2] (4-bit codes) is NULL", fn);
    if (!aligned16(qw->plane[2])) return fail(CQ_ERR_ALIGN, "%s: plane[2] is not 16-byte aligned", fn);
  } else {
    if (n / kGroup > (int64_t(1) << 26)) return fail(CQ_ERR_RANGE, "%s: too many groups for 32-bit offsets", fn);
    for (int i = 0; i < 4; ++i)
      if (qw->plane[i] && !aligned16(qw->plane[i])) return fail(CQ_ERR_ALIGN, "%s: plane[%d] is not 16-byte aligned", fn, i);
  }
  if (qw->residual) {
    if (qw->residual_dtype != CQ_F32 && qw->residual_dtype != CQ_BF16)
      return fail(CQ_ERR_ARG, "%s: bad residual dtype %d", fn, (int)qw->residual_dtype);
    if (need_residual_align && !aligned16(qw->residual))
      return fail(CQ_ERR_ALIGN, "%s: residual is not 16-byte aligned", fn);
  }
  return CQ_OK;
}

}  // namespace

cq_status check_matmul_args(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m, float *y, int max_m,
                            const char *fn) {
  cq_status st = check_qweight(qw, fn, false);
  if (st != CQ_OK) return st;
  if (m < 1 || m > max_m) return fail(CQ_ERR_ARG, "%s: m=%d outside [1, %d]", fn, m, max_m);
  if (x_dtype != CQ_F32 && x_dtype != CQ_BF16) return fail(CQ_ERR_ARG, "%s: bad x dtype %d", fn, (int)x_dtype);
  if (qw->rows && (!y || (qw->cols && !x))) return fail(CQ_ERR_ARG, "%s: NULL x or y", fn);
  if (x && !aligned16(x)) return fail(CQ_ERR_ALIGN, "%s: x is not 16-byte aligned", fn);
  return CQ_OK;
}

#ifdef CQ_DEBUG
// every unit's debug word, registered by its static initializer (cq_debug.cuh); the table is
// zero-initialized before any initializer runs
namespace {
constexpr int kMaxDebugUnits = 32;
uint32_t (*g_debug_takers[kMaxDebugUnits])();
int g_debug_units = 0;
std::mutex g_debug_mu;

__global__ void debug_selftest_kernel() {
  __shared__ uint32_t slot[1];
  if (threadIdx.x == 0) slot[0] = 0u;
  __syncthreads();
  const uint32_t i = threadIdx.x + 1;                 // one past the slot
  if (CQ_CHECK(i < 1, 0x0F01u)) slot[i] = 1u;
  __syncthreads();
  if (slot[0] != 0u) __threadfence();                 // keeps the slot live
}
}  // namespace

void register_debug_word(uint32_t (*take)()) {
  if (g_debug_units < kMaxDebugUnits) g_debug_takers[g_debug_units++] = take;
}
#endif

}  // namespace cq

using namespace cq;

extern "C" {

cq_status cq_debug_word(uint32_t *word) {
  if (!word) return fail(CQ_ERR_ARG, "cq_debug_word: NULL word");
  *word = 0;
#ifdef CQ_DEBUG
  std::lock_guard<std::mutex> lock(g_debug_mu);
  cq_status st = cuda_check(cudaDeviceSynchronize(), "cq_debug_word: synchronize");
  if (st != CQ_OK) return st;
  for (int u = 0; u < g_debug_units; ++u) {
    const uint32_t v = g_debug_takers[u]();
    if (v == 0xFFFFFFFFu) return fail(CQ_ERR_CUDA, "cq_debug_word: could not read a unit's word");
    if (!*word) *word = v;
  }
  return CQ_OK;
#else
  return fail(CQ_ERR_UNSUPPORTED, "cq_debug_word: a release build (no -DCQ_DEBUG) has no index checks");
#endif
}

cq_status cq_debug_selftest(cq_stream_t stream) {
#ifdef CQ_DEBUG
  debug_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return launch_check("cq_debug_selftest");
#else
  (void)stream;
  return fail(CQ_ERR_UNSUPPORTED, "cq_debug_selftest: a release build (no -DCQ_DEBUG) has no index checks");
#endif
}

const char *cq_last_error(void) { return g_last_error; }

const char *cq_status_string(cq_status s) {
  switch (s) {
    case CQ_OK: return "CQ_OK";
    case CQ_ERR_ARG: return "CQ_ERR_ARG";
    case CQ_ERR_SHAPE: return "CQ_ERR_SHAPE";
    case CQ_ERR_BITS: return "CQ_ERR_BITS";
    case CQ_ERR_ALIGN: return "CQ_ERR_ALIGN";
    case CQ_ERR_NONFINITE: return "CQ_ERR_NONFINITE";
    case CQ_ERR_RANGE: return "CQ_ERR_RANGE";
    case CQ_ERR_CUDA: return "CQ_ERR_CUDA";
    case CQ_ERR_UNSUPPORTED: return "CQ_ERR_UNSUPPORTED";
  }
  return "CQ_ERR_UNKNOWN";
}

cq_status cq_quantize(const float *w, int64_t rows, int64_t cols, const uint8_t *bits, uint8_t *codes,
                      uint16_t *scale, uint8_t *zero, uint32_t *status_word, cq_stream_t stream) {
  const char *fn = "cq_quantize";
  cq_status st = check_shape(rows, cols, fn);
  if (st != CQ_OK) return st;
  const int64_t G = rows * (cols / kGroup);
  if (G > 0) {
    if (!w || !codes || !scale || !zero) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
    if (!aligned16(w)) return fail(CQ_ERR_ALIGN, "%s: w is not 16-byte aligned", fn);
    if (!aligned16(codes)) return fail(CQ_ERR_ALIGN, "%s: codes is not 16-byte aligned", fn);
  }
  return launch_quantize(w, G, bits, codes, scale, zero, status_word, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_rrq_stage(float *r, int64_t rows, int64_t cols, int bits, uint8_t *codes, uint16_t *scale, uint8_t *zero,
                       uint32_t *status_word, cq_stream_t stream) {
  const char *fn = "cq_rrq_stage";
  cq_status st = check_shape(rows, cols, fn);
  if (st != CQ_OK) return st;
  if (!width_ok_host(bits)) return fail(CQ_ERR_BITS, "%s: width %d is not 1, 2, 4 or 8", fn, bits);
  const int64_t G = rows * (cols / kGroup);
  if (G > 0) {
    if (!r || !codes || !scale || !zero) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
    if (!aligned16(r)) return fail(CQ_ERR_ALIGN, "%s: r is not 16-byte aligned", fn);
    if (!aligned16(codes)) return fail(CQ_ERR_ALIGN, "%s: codes is not 16-byte aligned", fn);
  }
  return launch_rrq_stage(r, G, bits, codes, scale, zero, status_word, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_varbits_index(const uint8_t *bits, int64_t n_groups, uint32_t *offset, uint64_t *plane_bytes,
                           cq_stream_t stream) {
  const char *fn = "cq_varbits_index";
  if (n_groups < 0) return fail(CQ_ERR_SHAPE, "%s: negative n_groups", fn);
  if (n_groups > (int64_t(1) << 26)) return fail(CQ_ERR_RANGE, "%s: n_groups > 2^26 (32-bit byte offsets)", fn);
  if (!plane_bytes || (n_groups && (!bits || !offset))) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  return launch_varbits_index(bits, n_groups, offset, plane_bytes, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_pack_varbits(const uint8_t *codes, int64_t n_groups, const uint8_t *bits, const uint32_t *offset,
                          uint8_t *const plane[4], cq_stream_t stream) {
  const char *fn = "cq_pack_varbits";
  if (n_groups < 0) return fail(CQ_ERR_SHAPE, "%s: negative n_groups", fn);
  if (n_groups == 0) return CQ_OK;
  if (!codes || !plane) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  if (!aligned16(codes)) return fail(CQ_ERR_ALIGN, "%s: codes is not 16-byte aligned", fn);
  if ((bits == nullptr) != (offset == nullptr)) return fail(CQ_ERR_ARG, "%s: bits and offset must both be set or both NULL", fn);
  if (!bits) {
    if (!plane[2]) return fail(CQ_ERR_ARG, "%s: plane[2] is NULL", fn);
    if (!aligned16(plane[2])) return fail(CQ_ERR_ALIGN, "%s: plane[2] is not 16-byte aligned", fn);
  } else {
    if (n_groups > (int64_t(1) << 26)) return fail(CQ_ERR_RANGE, "%s: n_groups > 2^26", fn);
    for (int i = 0; i < 4; ++i)
      if (plane[i] && !aligned16(plane[i])) return fail(CQ_ERR_ALIGN, "%s: plane[%d] is not 16-byte aligned", fn, i);
  }
  return launch_pack(codes, n_groups, bits, offset, plane, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_unpack_varbits(const cq_qweight *qw, uint8_t *codes, cq_stream_t stream) {
  const char *fn = "cq_unpack_varbits";
  cq_status st = check_qweight(qw, fn, false);
  if (st != CQ_OK) return st;
  if (qw->rows * qw->cols == 0) return CQ_OK;
  if (!codes) return fail(CQ_ERR_ARG, "%s: codes is NULL", fn);
  if (!aligned16(codes)) return fail(CQ_ERR_ALIGN, "%s: codes is not 16-byte aligned", fn);
  return launch_unpack(*qw, codes, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_project_residual(void *r, cq_dtype dtype, const uint16_t *scale, int64_t n, uint64_t *n_clamped,
                              cq_stream_t stream) {
  const char *fn = "cq_project_residual";
  if (dtype != CQ_F32 && dtype != CQ_BF16) return fail(CQ_ERR_ARG, "%s: bad dtype %d", fn, (int)dtype);
  if (n < 0 || n % kGroup) return fail(CQ_ERR_SHAPE, "%s: n=%lld must be a non-negative multiple of 64", fn, (long long)n);
  if (n && (!r || !scale)) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  if (n && !aligned16(r)) return fail(CQ_ERR_ALIGN, "%s: r is not 16-byte aligned", fn);
  return launch_project(r, dtype, scale, n, n_clamped, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_reparam_residual(const float *theta, const uint16_t *scale, int64_t n, void *r, cq_dtype r_dtype,
                              cq_stream_t stream) {
  const char *fn = "cq_reparam_residual";
  if (r_dtype != CQ_F32 && r_dtype != CQ_BF16) return fail(CQ_ERR_ARG, "%s: bad residual dtype %d", fn, (int)r_dtype);
  if (n < 0 || n % kGroup) return fail(CQ_ERR_SHAPE, "%s: n=%lld must be a non-negative multiple of 64", fn, (long long)n);
  if (n && (!theta || !scale || !r)) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  if (n && (!aligned16(theta) || !aligned16(r))) return fail(CQ_ERR_ALIGN, "%s: theta and r must be 16-byte aligned", fn);
  return launch_reparam(theta, scale, n, r, r_dtype, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_reparam_residual_grad(const float *theta, const uint16_t *scale, const float *grad_r, int64_t n,
                                   cq_dtype r_dtype, float *grad_theta, cq_stream_t stream) {
  const char *fn = "cq_reparam_residual_grad";
  if (r_dtype != CQ_F32 && r_dtype != CQ_BF16) return fail(CQ_ERR_ARG, "%s: bad residual dtype %d", fn, (int)r_dtype);
  if (n < 0 || n % kGroup) return fail(CQ_ERR_SHAPE, "%s: n=%lld must be a non-negative multiple of 64", fn, (long long)n);
  if (n && (!theta || !scale || !grad_r || !grad_theta)) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  if (n && (!aligned16(theta) || !aligned16(grad_r) || !aligned16(grad_theta)))
    return fail(CQ_ERR_ALIGN, "%s: theta, grad_r and grad_theta must be 16-byte aligned", fn);
  return launch_reparam_grad(theta, scale, grad_r, n, r_dtype, grad_theta, reinterpret_cast<cudaStream_t>(stream));
}

size_t cq_requant_workspace(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return requant_workspace(rows, cols);
}

cq_status cq_requant_refine(const float *w, int64_t rows, int64_t cols, const double *H, const uint16_t *scale,
                            const uint8_t *zero, int bits, uint8_t *codes, int sweeps, double *err_before,
                            double *err_after, uint64_t *moves, void *workspace, size_t workspace_bytes,
                            cq_stream_t stream) {
  const char *fn = "cq_requant_refine";
  cq_status st = check_shape(rows, cols, fn);
  if (st != CQ_OK) return st;
  if (!width_ok_host(bits)) return fail(CQ_ERR_BITS, "%s: width %d is not 1, 2, 4 or 8", fn, bits);
  if (sweeps < 0) return fail(CQ_ERR_ARG, "%s: negative sweep count", fn);
  if (rows == 0 || cols == 0) return CQ_OK;
  if (cols > requant_max_cols())
    return fail(CQ_ERR_UNSUPPORTED, "%s: cols=%lld above the %lld a row's state can hold on chip", fn,
                (long long)cols, (long long)requant_max_cols());
  if (!w || !H || !scale || !zero || !codes) return fail(CQ_ERR_ARG, "%s: NULL buffer", fn);
  const size_t need = requant_workspace(rows, cols);
  if (!workspace || workspace_bytes < need)
    return fail(CQ_ERR_RANGE, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 7u) || (reinterpret_cast<uintptr_t>(H) & 7u))
    return fail(CQ_ERR_ALIGN, "%s: H and the workspace must be 8-byte aligned", fn);
  return launch_requant(w, rows, cols, H, scale, zero, bits, codes, sweeps, err_before, err_after, moves,
                        static_cast<double *>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_requant_verify(const cq_qweight *qw, int64_t first_w, int64_t n_w, uint64_t *mismatches,
                            int64_t *first_bad, uint32_t *group_flags, cq_stream_t stream) {
  const char *fn = "cq_requant_verify";
  cq_status st = check_qweight(qw, fn, true);
  if (st != CQ_OK) return st;
  if (!mismatches || !first_bad) return fail(CQ_ERR_ARG, "%s: mismatches/first_bad is NULL", fn);
  const int64_t total = qw->rows * qw->cols;
  if (first_w < 0 || n_w < 0 || first_w % kGroup || n_w % kGroup || first_w > total || n_w > total - first_w)
    return fail(CQ_ERR_SHAPE, "%s: chunk [%lld, +%lld) is not whole groups inside the %lld weights", fn,
                (long long)first_w, (long long)n_w, (long long)total);
  return launch_verify(*qw, first_w, n_w, mismatches, first_bad, group_flags, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_requant_verify_pair(const cq_qweight *qw, int64_t first_w, int64_t n_w, uint64_t *mismatches,
                                 int64_t *first_bad, uint64_t *revoke_mismatches, int64_t *revoke_first_bad,
                                 uint32_t *group_flags, cq_stream_t stream) {
  const char *fn = "cq_requant_verify_pair";
  cq_status st = check_qweight(qw, fn, true);
  if (st != CQ_OK) return st;
  if (!qw->residual && qw->rows > 0 && qw->cols > 0) return fail(CQ_ERR_ARG, "%s: the pair needs a residual", fn);
  if (!mismatches || !first_bad || !revoke_mismatches || !revoke_first_bad)
    return fail(CQ_ERR_ARG, "%s: a result pointer is NULL", fn);
  const int64_t total = qw->rows * qw->cols;
  if (first_w < 0 || n_w < 0 || first_w % kGroup || n_w % kGroup || first_w > total || n_w > total - first_w)
    return fail(CQ_ERR_SHAPE, "%s: chunk [%lld, +%lld) is not whole groups inside the %lld weights", fn,
                (long long)first_w, (long long)n_w, (long long)total);
  return launch_verify_pair(*qw, first_w, n_w, mismatches, first_bad, revoke_mismatches, revoke_first_bad, group_flags,
                            reinterpret_cast<cudaStream_t>(stream));
}


cq_status cq_dequant_gemv(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m, float *y,
                          cq_stream_t stream) {
  cq_status st = check_matmul_args(qw, x, x_dtype, m, y, 8, "cq_dequant_gemv");
  if (st != CQ_OK) return st;
  return launch_gemv(*qw, x, x_dtype, m, y, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_dequant_gemv_multi(const cq_qweight *const *qws, int count, const void *x, cq_dtype x_dtype, int m,
                                float *const *ys, cq_stream_t stream) {
  const char *fn = "cq_dequant_gemv_multi";
  if (count < 0) return fail(CQ_ERR_ARG, "%s: negative count", fn);
  if (count == 0) return CQ_OK;
  if (!qws || !ys) return fail(CQ_ERR_ARG, "%s: NULL matrix or output list", fn);
  for (int i = 0; i < count; ++i) {
    if (!qws[i]) return fail(CQ_ERR_ARG, "%s: matrix %d is NULL", fn, i);
    cq_status st = check_matmul_args(qws[i], x, x_dtype, m, ys[i], 8, fn);
    if (st != CQ_OK) return st;
    if (qws[i]->cols != qws[0]->cols)
      return fail(CQ_ERR_SHAPE, "%s: matrix %d has %lld cols, matrix 0 has %lld", fn, i,
                  (long long)qws[i]->cols, (long long)qws[0]->cols);
  }
  return launch_gemv_multi(qws, count, x, x_dtype, m, ys, reinterpret_cast<cudaStream_t>(stream));
}

cq_status cq_dequant_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype x_dtype, int m,
                                 float *y, cq_stream_t stream) {
  const char *fn = "cq_dequant_gemv_stages";
  if (count < 1 || count > kMaxRrqStages)
    return fail(CQ_ERR_ARG, "%s: %d stages, 1 to %d supported", fn, count, kMaxRrqStages);
  if (!stages) return fail(CQ_ERR_ARG, "%s: NULL stage list", fn);
  for (int j = 0; j < count; ++j) {
    if (!stages[j]) return fail(CQ_ERR_ARG, "%s: stage %d is NULL", fn, j);
    cq_status st = check_matmul_args(stages[j], x, x_dtype, m, y, 8, fn);
    if (st != CQ_OK) return st;
    if (stages[j]->rows != stages[0]->rows || stages[j]->cols != stages[0]->cols)
      return fail(CQ_ERR_SHAPE, "%s: stage %d is %lldx%lld, stage 0 is %lldx%lld", fn, j, (long long)stages[j]->rows,
                  (long long)stages[j]->cols, (long long)stages[0]->rows, (long long)stages[0]->cols);
    if (stages[j]->residual) return fail(CQ_ERR_UNSUPPORTED, "%s: stage %d has a residual", fn, j);
  }
  return launch_gemv_stages(stages, count, x, x_dtype, m, y, reinterpret_cast<cudaStream_t>(stream));
}

size_t cq_gemm_workspace(int64_t rows, int64_t cols, int m) {
  if (rows <= 0 || cols <= 0 || m < 16) return 0;
  return gemm_tc_workspace(rows, cols, m);
}

cq_status cq_dequant_gemm(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m, float *y, void *workspace,
                          size_t workspace_bytes, cq_stream_t stream) {
  const char *fn = "cq_dequant_gemm";
  cq_status st = check_matmul_args(qw, x, x_dtype, m, y, 256, fn);
  if (st != CQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (gemm_tc_eligible(*qw, x_dtype, m)) {
    const size_t need = gemm_tc_workspace(qw->rows, qw->cols, m);
    if (workspace_bytes < need)
      return fail(CQ_ERR_RANGE, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes, need);
    if (need && (!workspace || !aligned16(workspace)))
      return fail(CQ_ERR_ALIGN, "%s: workspace is NULL or not 16-byte aligned", fn);
    return launch_gemm_tc(*qw, x, m, y, workspace, workspace_bytes, s);
  }
  // small batches and the formats the tensor-core GEMM does not take: GEMV slices of 8
  const size_t xe = x_dtype == CQ_BF16 ? 2 : 4;
  for (int i0 = 0; i0 < m; i0 += 8) {
    const int mi = m - i0 < 8 ? m - i0 : 8;
    st = launch_gemv(*qw, static_cast<const char *>(x) + xe * i0 * qw->cols, x_dtype, mi, y + (int64_t)i0 * qw->rows, s);
    if (st != CQ_OK) return st;
  }
  return CQ_OK;
}

}  // extern "C"
