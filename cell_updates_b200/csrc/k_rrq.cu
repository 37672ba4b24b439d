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
// Per 16 columns the stage sum of each weight is formed in fp32 first (s * (q - z), the
// product exact), then multiplied with the batch rows of x, so x is read once per column and
// batch row whatever the number of stages. fp32 accumulation, a warp reduction per row.
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;
constexpr int kPerLaunch = 4;         // stages per launch (their metadata lives in registers)

struct StageSet {
  const uint8_t *bits[kPerLaunch];
  const uint32_t *offset[kPerLaunch];
  const uint8_t *plane[kPerLaunch][4];
  const uint16_t *scale[kPerLaunch];
  const uint8_t *zero[kPerLaunch];
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

// codes 16 c .. 16 c + 15 of one group of width b (LSB-first bit string at src) -> q[16]; the
// chunk is 2b bytes at byte 2bc, aligned to its size
__device__ __forceinline__ void load_codes16(const uint8_t *src, int b, int c, uint32_t (&q)[16]) {
  if (b == 2) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(src + 4 * c));
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (w >> (2 * t)) & 3u;
  } else if (b == 4) {
    const uint2 w = __ldg(reinterpret_cast<const uint2 *>(src + 8 * c));
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      q[t] = (w.x >> (4 * t)) & 15u;
      q[8 + t] = (w.y >> (4 * t)) & 15u;
    }
  } else if (b == 1) {
    const uint32_t w = __ldg(reinterpret_cast<const uint16_t *>(src + 2 * c));
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (w >> t) & 1u;
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(src + 16 * c));
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 16; ++t) q[t] = (ww[t >> 2] >> (8 * (t & 3))) & 255u;
  }
}

// A warp per output row (grid-stride); lane l owns group 32 p + l in pass p, so the warp's
// code reads cover 32 consecutive groups. The lane reads each stage's width, offset, scale and
// zero point of its group once, then walks the group in four chunks of 16 columns: for each
// chunk it sums the 16 weights over the stages in fp32 and multiplies them with the chunk of
// every batch row of x (x stays in L1).
template <bool XBF16, int M>
__global__ void __launch_bounds__(kThreads)
gemv_stages_kernel(const __grid_constant__ StageSet ss, int count, const void *__restrict__ x, int m, int64_t N,
                   int64_t K, float *__restrict__ y, bool accumulate) {
  const int lane = threadIdx.x & 31;
  const int64_t KG = K >> 6;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t n = blockIdx.x * static_cast<int64_t>(kThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    float acc[M];
#pragma unroll
    for (int i = 0; i < M; ++i) acc[i] = 0.0f;
    for (int64_t gk = lane; gk < KG; gk += 32) {
      const int64_t g = n * KG + gk;
      const uint8_t *src[kPerLaunch];
      float sv[kPerLaunch], zv[kPerLaunch];
      int bv[kPerLaunch];
#pragma unroll
      for (int j = 0; j < kPerLaunch; ++j) {
        if (j < count) {
          int b = 4;
          if (ss.bits[j]) {
            b = __ldg(ss.bits[j] + g);
            const int slot = b == 1 ? 0 : b == 2 ? 1 : b == 4 ? 2 : 3;
            src[j] = ss.plane[j][slot] + __ldg(ss.offset[j] + g);
          } else {
            src[j] = ss.plane[j][2] + g * 32;
          }
          bv[j] = width_ok(b) ? b : 0;             // a bad width in a map contributes nothing
          sv[j] = f16_bits_to_f32(__ldg(ss.scale[j] + g));
          zv[j] = static_cast<float>(__ldg(ss.zero[j] + g));
        }
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float wsum[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) wsum[t] = 0.0f;
#pragma unroll
        for (int j = 0; j < kPerLaunch; ++j) {
          if (j < count && bv[j]) {
            uint32_t q[16];
            load_codes16(src[j], bv[j], c, q);
#pragma unroll
            for (int t = 0; t < 16; ++t) wsum[t] = fmaf(sv[j], __fsub_rn(static_cast<float>(q[t]), zv[j]), wsum[t]);
          }
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
    }
#pragma unroll
    for (int i = 0; i < M; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && i < m) y[i * N + n] = accumulate ? y[i * N + n] + v : v;
    }
  }
}

template <bool XBF16>
cq_status launch_m(const StageSet &ss, int count, const void *x, int m, int64_t N, int64_t K, float *y, bool acc,
                   int blocks, cudaStream_t s) {
  if (m == 1) gemv_stages_kernel<XBF16, 1><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y, acc);
  else if (m <= 4) gemv_stages_kernel<XBF16, 4><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y, acc);
  else gemv_stages_kernel<XBF16, 8><<<blocks, kThreads, 0, s>>>(ss, count, x, m, N, K, y, acc);
  return launch_check("cq_dequant_gemv_stages");
}

}  // namespace

cq_status launch_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype xdt, int m,
                             float *y, cudaStream_t s) {
  const int64_t N = stages[0]->rows, K = stages[0]->cols;
  if (N == 0) return CQ_OK;
  if (K == 0) return cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * m * N, s), "cq_dequant_gemv_stages: zero y");
  const int64_t need = (N + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  // up to kPerLaunch stages per launch; later launches add to y in stream order
  for (int j0 = 0; j0 < count; j0 += kPerLaunch) {
    const int cnt = count - j0 < kPerLaunch ? count - j0 : kPerLaunch;
    StageSet ss = {};
    for (int j = 0; j < cnt; ++j) {
      const cq_qweight &q = *stages[j0 + j];
      ss.bits[j] = q.bits;
      ss.offset[j] = q.offset;
      for (int p = 0; p < 4; ++p) ss.plane[j][p] = q.plane[p];
      ss.scale[j] = q.scale;
      ss.zero[j] = q.zero;
    }
    cq_status st = xdt == CQ_BF16 ? launch_m<true>(ss, cnt, x, m, N, K, y, j0 > 0, blocks, s)
                                  : launch_m<false>(ss, cnt, x, m, N, K, y, j0 > 0, blocks, s);
    if (st != CQ_OK) return st;
  }
  return CQ_OK;
}

}  // namespace cq
