// k_project.cu -- projection of the per-weight residual into its quantization cell.
//
// [CF] "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
// Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: an update is carried by a
// residual that may not leave the rounding cell of its weight; the constrained training path
// enforces this by clamping (projecting) the residual back into the cell.
// Reading: half-width c = (0.5 - 2^-10) * s (exact in binary32: 9 x 11 significant bits);
// a bf16 residual uses c rounded toward zero to bf16, so the clamp never rounds outward.
// The clamp is written with comparisons so that a NaN residual passes through unchanged.
//
// Layout: one lane per eight residuals (one 16-byte load for bf16, two for fp32); eight
// lanes share a group scale. Streaming, in place.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float cell_bound(uint16_t s16) {
  return __fmul_rn(0.5f - 0x1p-10f, f16_bits_to_f32(s16));
}

__device__ __forceinline__ float clamp_cell(float r, float c) {
  return r > c ? c : (r < -c ? -c : r);
}

constexpr int kUnroll = 4;    // units per lane and iteration: 64 bytes of bf16 in flight

__device__ __forceinline__ uint32_t project_pair(uint32_t w, float cb, uint32_t &changed) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  const uint32_t nlo = __float_as_uint(clamp_cell(lo, cb)) >> 16;
  const uint32_t nhi = __float_as_uint(clamp_cell(hi, cb)) & 0xFFFF0000u;
  const uint32_t nw = nlo | nhi;
  changed += ((nw ^ w) & 0xFFFFu) != 0;
  changed += ((nw ^ w) & 0xFFFF0000u) != 0;
  return nw;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
project_kernel(void *__restrict__ rv, const uint16_t *__restrict__ scale, int64_t n_units,
               unsigned long long *__restrict__ n_clamped) {
  pdl_wait();                     // r, the scales and the cleared count come from earlier work
  uint32_t changed = 0;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u0 < n_units; u0 += kUnroll * step) {
    if (BF16) {
      uint4 in[kUnroll];
      float cb[kUnroll];
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) {
        const int64_t u = u0 + t * step;
        if (u < n_units) {
          in[t] = __ldcs(reinterpret_cast<const uint4 *>(rv) + u);
          // c rounded toward zero to bf16: drop the low 16 bits (c >= 0 or NaN)
          cb[t] = __uint_as_float(__float_as_uint(cell_bound(__ldg(scale + (u >> 3)))) & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) {
        const int64_t u = u0 + t * step;
        if (u < n_units) {
          uint4 o;
          o.x = project_pair(in[t].x, cb[t], changed);
          o.y = project_pair(in[t].y, cb[t], changed);
          o.z = project_pair(in[t].z, cb[t], changed);
          o.w = project_pair(in[t].w, cb[t], changed);
          __stcs(reinterpret_cast<uint4 *>(rv) + u, o);
        }
      }
    } else {
      float4 in[kUnroll][2];
      float c[kUnroll];
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) {
        const int64_t u = u0 + t * step;
        if (u < n_units) {
          const float4 *p = reinterpret_cast<const float4 *>(rv) + 2 * u;
          in[t][0] = __ldcs(p);
          in[t][1] = __ldcs(p + 1);
          c[t] = cell_bound(__ldg(scale + (u >> 3)));
        }
      }
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) {
        const int64_t u = u0 + t * step;
        if (u < n_units) {
          float v[8] = {in[t][0].x, in[t][0].y, in[t][0].z, in[t][0].w, in[t][1].x, in[t][1].y, in[t][1].z, in[t][1].w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float o = clamp_cell(v[j], c[t]);
            changed += __float_as_uint(o) != __float_as_uint(v[j]);
            v[j] = o;
          }
          float4 *p = reinterpret_cast<float4 *>(rv) + 2 * u;
          __stcs(p, make_float4(v[0], v[1], v[2], v[3]));
          __stcs(p + 1, make_float4(v[4], v[5], v[6], v[7]));
        }
      }
    }
  }
  if (n_clamped) {
    changed = __reduce_add_sync(0xffffffffu, changed);   // every lane of the warp reaches this point
    if ((threadIdx.x & 31) == 0 && changed) atomicAdd(n_clamped, static_cast<unsigned long long>(changed));
  }
}

}  // namespace

cq_status launch_project(void *r, cq_dtype dt, const uint16_t *scale, int64_t n, uint64_t *n_clamped,
                         cudaStream_t s) {
  if (n_clamped) {
    cq_status st = cuda_check(launch_clear_results(nullptr, reinterpret_cast<unsigned long long *>(n_clamped), s),
                              "cq_project_residual: clear count");
    if (st != CQ_OK) return st;
    st = launch_check("cq_project_residual: clear count");
    if (st != CQ_OK) return st;
  }
  if (n == 0) return CQ_OK;
  const int64_t units = n / 8;
  const int64_t need = (units + kUnroll * kThreads - 1) / (kUnroll * kThreads);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  auto *cnt = reinterpret_cast<unsigned long long *>(n_clamped);
  const cudaError_t e = dt == CQ_BF16 ? launch_pdl(project_kernel<true>, dim3(blocks), dim3(kThreads), 0, s, r, scale,
                                                   units, cnt)
                                      : launch_pdl(project_kernel<false>, dim3(blocks), dim3(kThreads), 0, s, r, scale,
                                                   units, cnt);
  cq_status st = cuda_check(e, "cq_project_residual");
  if (st != CQ_OK) return st;
  return launch_check("cq_project_residual");
}

}  // namespace cq
