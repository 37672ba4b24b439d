// k_reparam.cu -- the bounded reparameterization of the CellFill residual, forward and backward.
//
// [CF] "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
// Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: besides projecting the
// residual back into its cell, CellFill can be trained as a bounded reparameterization, so
// that the residual stays inside the cell by construction for every value of the trained
// parameter. The bounded map is not printed; the reading is
//     r = RN(c_dt * phi(theta)),  phi(t) = t / sqrt(1 + t^2)
// with c_dt the projection's bound for the residual's format (c = (0.5 - 2^-10) s for fp32,
// c rounded toward zero to bf16 for bf16), every step one IEEE binary32 operation rounded to
// nearest in the order u = t*t, d = 1 + u, q = sqrt(d), phi = t / q (no contraction, no
// approximate square root or division), so the served residual is the same bit pattern on any
// IEEE machine. |phi| <= 1 since q >= |t| exactly and rounding is monotone, hence |r| <= c_dt.
// A NaN theta gives r = +0 (its update revoked) and |theta| > 2^32 gives phi = +-1, the value
// the formula rounds to there (theta^2 would overflow further out).
// Backward, straight through the final rounding: dL/dtheta = RN(RN(dL/dr * c_dt) * phi'),
// phi' = (1 + t^2)^(-3/2) = RN(RN(1 / d) / q), and 0 for a NaN or saturated theta.
//
// Layout: one lane per eight weights (32 bytes of theta); the eight lanes of a 64-weight group
// share its scale. Streaming. The backward pass keeps two such units in flight per lane at four
// CTAs of 256 threads per SM (more warps hide the long dependent sequences of the correctly
// rounded square root and divisions better than more units per lane: it went from 66 to 97 % of
// HBM); the forward pass, with one division fewer per weight, runs one unit per lane at six CTAs
// per SM (74.5 % of HBM against 72.5 % in the backward pass's shape, and 65 % at four CTAs).
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;          // backward: units in flight per lane, four CTAs per SM
constexpr int kFwdUnroll = 1;       // forward: one unit per lane, kFwdCtas CTAs per SM
constexpr int kFwdCtas = 6;          // and the grid's CTAs per SM
constexpr float kSat = 0x1p32f;

__device__ __forceinline__ float cell_bound(uint16_t s16, bool bf16) {
  const float c = __fmul_rn(0.5f - 0x1p-10f, f16_bits_to_f32(s16));
  return bf16 ? __uint_as_float(__float_as_uint(c) & 0xFFFF0000u) : c;   // toward zero (c >= 0 or NaN)
}

__device__ __forceinline__ float phi(float t) {
  if (t != t) return 0.0f;
  if (fabsf(t) > kSat) return t > 0.0f ? 1.0f : -1.0f;
  const float d = __fadd_rn(1.0f, __fmul_rn(t, t));
  return __fdiv_rn(t, __fsqrt_rn(d));
}

__device__ __forceinline__ float dphi(float t) {
  if (t != t || fabsf(t) > kSat) return 0.0f;
  const float d = __fadd_rn(1.0f, __fmul_rn(t, t));
  return __fdiv_rn(__fdiv_rn(1.0f, d), __fsqrt_rn(d));
}

__device__ __forceinline__ void load8(const float *p, int64_t u, float v[8]) {
  const float4 *q = reinterpret_cast<const float4 *>(p) + 2 * u;
  const float4 a = __ldcs(q), b = __ldcs(q + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(float *p, int64_t u, const float v[8]) {
  float4 *q = reinterpret_cast<float4 *>(p) + 2 * u;
  __stcs(q, make_float4(v[0], v[1], v[2], v[3]));
  __stcs(q + 1, make_float4(v[4], v[5], v[6], v[7]));
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, kFwdCtas)
reparam_kernel(const float *__restrict__ theta, const uint16_t *__restrict__ scale, int64_t n_units,
               void *__restrict__ r) {
  pdl_wait();
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u0 < n_units; u0 += kFwdUnroll * step) {
    float t[kFwdUnroll][8], c[kFwdUnroll];
#pragma unroll
    for (int k = 0; k < kFwdUnroll; ++k) {
      const int64_t u = u0 + k * step;
      if (u < n_units) {
        load8(theta, u, t[k]);
        c[k] = cell_bound(__ldg(scale + (u >> 3)), BF16);
      }
    }
#pragma unroll
    for (int k = 0; k < kFwdUnroll; ++k) {
      const int64_t u = u0 + k * step;
      if (u >= n_units) continue;
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(c[k], phi(t[k][j]));
      if (BF16) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
          o[j] = *reinterpret_cast<const uint32_t *>(&h);
        }
        __stcs(reinterpret_cast<uint4 *>(r) + u, make_uint4(o[0], o[1], o[2], o[3]));
      } else {
        store8(static_cast<float *>(r), u, v);
      }
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 4)
reparam_grad_kernel(const float *__restrict__ theta, const uint16_t *__restrict__ scale,
                    const float *__restrict__ grad_r, int64_t n_units, float *__restrict__ grad_theta) {
  pdl_wait();
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u0 < n_units; u0 += kUnroll * step) {
    float t[kUnroll][8], g[kUnroll][8], c[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t u = u0 + k * step;
      if (u < n_units) {
        load8(theta, u, t[k]);
        load8(grad_r, u, g[k]);
        c[k] = cell_bound(__ldg(scale + (u >> 3)), BF16);
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t u = u0 + k * step;
      if (u >= n_units) continue;
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(__fmul_rn(g[k][j], c[k]), dphi(t[k][j]));
      store8(grad_theta, u, v);
    }
  }
}

int grid_for(int64_t units, int unroll, int per_sm) {
  const int64_t need = (units + unroll * kThreads - 1) / (unroll * kThreads);
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  return static_cast<int>(need < cap ? need : cap);
}

}  // namespace

cq_status launch_reparam(const float *theta, const uint16_t *scale, int64_t n, void *r, cq_dtype dt,
                         cudaStream_t s) {
  if (n == 0) return CQ_OK;
  const int64_t units = n / 8;
  const dim3 grid(grid_for(units, kFwdUnroll, kFwdCtas));
  const cudaError_t e = dt == CQ_BF16 ? launch_pdl(reparam_kernel<true>, grid, dim3(kThreads), 0, s, theta, scale,
                                                   units, r)
                                      : launch_pdl(reparam_kernel<false>, grid, dim3(kThreads), 0, s, theta, scale,
                                                   units, r);
  cq_status st = cuda_check(e, "cq_reparam_residual");
  if (st != CQ_OK) return st;
  return launch_check("cq_reparam_residual");
}

cq_status launch_reparam_grad(const float *theta, const uint16_t *scale, const float *grad_r, int64_t n, cq_dtype dt,
                              float *grad_theta, cudaStream_t s) {
  if (n == 0) return CQ_OK;
  const int64_t units = n / 8;
  const dim3 grid(grid_for(units, kUnroll, 8));   // two waves of four resident CTAs per SM
  const cudaError_t e = dt == CQ_BF16 ? launch_pdl(reparam_grad_kernel<true>, grid, dim3(kThreads), 0, s, theta,
                                                   scale, grad_r, units, grad_theta)
                                      : launch_pdl(reparam_grad_kernel<false>, grid, dim3(kThreads), 0, s, theta,
                                                   scale, grad_r, units, grad_theta);
  cq_status st = cuda_check(e, "cq_reparam_residual_grad");
  if (st != CQ_OK) return st;
  return launch_check("cq_reparam_residual_grad");
}

}  // namespace cq
