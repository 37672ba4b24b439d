// k_rrq.cu -- recurrent residual quantization: the multiply over a stack of stages.
//
// [RRQ] the listing page thelatestinai.com/papers/2512.18934, "Recurrent Residual
// Quantization" abstract: the weights are a low-bit base plus a sequence of quantized residual
// corrections (2-bit round-to-nearest stages stacked to 4, 6 and 8 bits), so one artifact
// serves several precisions; a model of 2(J+1) bits uses the first J+1 stages. The stages
// themselves come from cq_rrq_stage (the group quantizer with an in-place residual update,
// k_quantize.cu); here
//     y[i, n] = sum_k (sum_j s_j[n, g] * (q_j[n, k] - z_j[n, g])) * x[i, k]
// over any stage list of one shape, each stage fixed-4 or per-group width.
//
// Layout of the work: a warp per output row (grid-stride); lane l takes codes
// 16 (l % 4) .. 16 (l % 4) + 15 of group 8 p + l / 4 in pass p, so a warp covers eight groups
// per pass and reads each group's code bytes as one aligned 2, 4, 8 or 16-byte word per lane
// (8b bytes per group: the quarter of lane l starts at byte 2b (l % 4)). Per group the lane
// first sums its 16 weights over all stages in fp32 (s * (q - z), the product exact), then
// multiplies them with the batch rows of x, so x is read once per group and batch row
// whatever the number of stages. fp32 accumulation, a warp reduction per row.
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;

struct StageSet {
  const uint8_t *bits[kMaxRrqStages];
  const uint32_t *offset[kMaxRrqStages];
  const uint8_t *plane[kMaxRrqStages][4];
  const uint16_t *scale[kMaxRrqStages];
  const uint8_t *zero[kMaxRrqStages];
};

template <bool XBF16>
__device__ __forceinline__ void load_x16(const void *x, int64_t idx, float (&xv)[16]) {
  if (XBF16) {
    const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + idx);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = __ldg(p + h);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xv[8 * h + 2 * e] = __uint_as_float(w[e] << 16);
        xv[8 * h + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + idx);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 f = __ldg(p + h);
      xv[4 * h] = f.x;
      xv[4 * h + 1] = f.y;
      xv[4 * h + 2] = f.z;
      xv[4 * h + 3] = f.w;
    }
  }
}

// codes 16 c .. 16 c + 15 of one group of width b (LSB-first bit string at src) -> q[16]
__device__ __forceinline__ void load_codes16(const uint8_t *src, int b, int c, uint32_t (&q)[16]) {
  if (b == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(src + 4 * c);
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (w >> (2 * t)) & 3u;
  } else if (b == 4) {
    const uint2 w = *reinterpret_cast<const uint2 *>(src + 8 * c);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      q[t] = (w.x >> (4 * t)) & 15u;
      q[8 + t] = (w.y >> (4 * t)) & 15u;
    }
  } else if (b == 1) {
    const uint32_t w = *reinterpret_cast<const uint16_t *>(src + 2 * c);
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (w >> t) & 1u;
  } else {
    const uint4 w = *reinterpret_cast<const uint4 *>(src + 16 * c);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (ww[t >> 2] >> (8 * (t & 3))) & 255u;
  }
}

template <bool XBF16, int M>
__global__ void __launch_bounds__(kThreads)
gemv_stages_kernel(const __grid_constant__ StageSet ss, int count, const void *__restrict__ x, int m, int64_t N,
                   int64_t K, float *__restrict__ y) {
  const int lane = threadIdx.x & 31, c = lane & 3;
  const int64_t KG = K >> 6;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t n = blockIdx.x * static_cast<int64_t>(kThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    float acc[M];
#pragma unroll
    for (int i = 0; i < M; ++i) acc[i] = 0.0f;
    for (int64_t gk = lane >> 2; gk < KG; gk += 8) {
      const int64_t g = n * KG + gk;
      float wsum[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) wsum[t] = 0.0f;
      for (int j = 0; j < count; ++j) {
        int b = 4;
        const uint8_t *src;
        if (ss.bits[j]) {
          b = ss.bits[j][g];
          const int slot = b == 1 ? 0 : b == 2 ? 1 : b == 4 ? 2 : 3;
          src = ss.plane[j][slot] + ss.offset[j][g];
        } else {
          src = ss.plane[j][2] + g * 32;
        }
        if (!width_ok(b)) continue;                 // validated on the host for fixed widths
        const float s = f16_bits_to_f32(ss.scale[j][g]);
        const float z = static_cast<float>(ss.zero[j][g]);
        uint32_t q[16];
        load_codes16(src, b, c, q);
#pragma unroll
        for (int t = 0; t < 16; ++t) wsum[t] = fmaf(s, __fsub_rn(static_cast<float>(q[t]), z), wsum[t]);
      }
#pragma unroll
      for (int i = 0; i < M; ++i) {
        if (i < m) {
          float xv[16];
          load_x16<XBF16>(x, i * K + gk * 64 + 16 * c, xv);
#pragma unroll
          for (int t = 0; t < 16; ++t) acc[i] = fmaf(wsum[t], xv[t], acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < M; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && i < m) y[i * N + n] = v;
    }
  }
}

template <bool XBF16>
cq_status launch_m(const StageSet &ss, int count, const void *x, int m, int64_t N, int64_t K, float *y, int blocks,
                   cudaStream_t s) {
  if (m == 1) gemv_stages_kernel<XBF16, 1><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y);
  else if (m <= 4) gemv_stages_kernel<XBF16, 4><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y);
  else gemv_stages_kernel<XBF16, 8><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y);
  return launch_check("cq_dequant_gemv_stages");
}

}  // namespace

cq_status launch_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype xdt, int m,
                             float *y, cudaStream_t s) {
  const int64_t N = stages[0]->rows, K = stages[0]->cols;
  if (N == 0) return CQ_OK;
  if (K == 0) return cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * m * N, s), "cq_dequant_gemv_stages: zero y");
  StageSet ss = {};
  for (int j = 0; j < count; ++j) {
    ss.bits[j] = stages[j]->bits;
    ss.offset[j] = stages[j]->offset;
    for (int p = 0; p < 4; ++p) ss.plane[j][p] = stages[j]->plane[p];
    ss.scale[j] = stages[j]->scale;
    ss.zero[j] = stages[j]->zero;
  }
  const int64_t need = (N + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  return xdt == CQ_BF16 ? launch_m<true>(ss, count, x, m, N, K, y, blocks, s)
                        : launch_m<false>(ss, count, x, m, N, K, y, blocks, s);
}

}  // namespace cq
