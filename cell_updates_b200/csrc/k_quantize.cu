// k_quantize.cu -- per-group asymmetric min-max round-to-nearest quantization.
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: groups of 64 consecutive weights, each
// with its own width from {1,2,4,8}. [CF] "Nothing Changed but the Model: CellFill ...",
// Abstract: 4-bit integer codes and scales. [SLQ] abstract (page 2 listing): asymmetric
// grids. Reading of the formula: see include/cq.h.
//
// Every fp32 operation is an explicit round-to-nearest intrinsic, so nothing is contracted.
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;

// One thread owns one group of 64 weights: the group's scale and zero point (two IEEE
// divisions, a reciprocal) are paid once per 64 weights, the 256 bytes it loads are all in
// flight at once, and min/max need no shuffles. Loads go through L1 (ld.global.nc), so the
// second half of each 32-byte sector is an L1 hit for the next 16-byte load.
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const float *__restrict__ w, int64_t G, const uint8_t *__restrict__ bits,
                uint8_t *__restrict__ codes, uint16_t *__restrict__ scale,
                uint8_t *__restrict__ zero, uint32_t *__restrict__ status) {
  uint32_t flags = 0;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  // warp-uniform trip count (the exact path below votes across the warp)
  const int64_t warp_first = static_cast<int64_t>(blockIdx.x) * kThreads + (threadIdx.x & ~31);
  for (int64_t g0 = warp_first; g0 < G; g0 += step) {
    const int64_t g = g0 + (threadIdx.x & 31);
    const bool valid = g < G;
    float v[64];
    const float4 *p = reinterpret_cast<const float4 *>(w + (valid ? g : 0) * kGroup);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 t = __ldg(p + i);
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
    // NaN-propagating min/max: a NaN or an infinity shows up as a non-finite extreme
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int j = 1; j < 64; ++j) {
      asm("min.NaN.f32 %0, %0, %1;\n" : "+f"(lo) : "f"(v[j]));
      asm("max.NaN.f32 %0, %0, %1;\n" : "+f"(hi) : "f"(v[j]));
    }
    const bool finite = isfinite(lo) && isfinite(hi);
    const int b = (bits && valid) ? static_cast<int>(__ldg(bits + g)) : 4;
    const bool width_good = width_ok(b);
    const int L = width_good ? (1 << b) - 1 : 15;
    // s = RN_fp16(RN32(RN32(wmax - wmin) / L)), floored at the smallest normal fp16
    const float s32 = __fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(L));
    const __half hs = __float2half_rn(s32);
    uint16_t s16 = __half_as_ushort(hs);
    float sf = __half2float(hs);
    const bool overflow = isinf(sf);
    if (sf < 0x1p-14f) {
      s16 = 0x0400u;
      sf = 0x1p-14f;
    }
    const float rc = __frcp_rn(sf);
    const int z = clamp_code(rne_quotient(-lo, sf, rc), L);
    // t_j = rne(RN32(w_j / s)) through the division-free filter: with qt = RN32(w_j * rc),
    // |RN32(w_j / s) - qt| < |qt| * 2^-21, so |qt - rint(qt)| + |qt| * 2^-20 < 0.4999 decides
    // the rounding; the rest (near a half-way point, huge, non-finite) is redone with the
    // IEEE division in a branch of its own
    uint64_t need_exact = 0;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const float qt = __fmul_rn(v[j], rc);
      const float t = rintf(qt);
      need_exact |= static_cast<uint64_t>(!(__fmaf_rn(fabsf(qt), 0x1p-20f, fabsf(__fsub_rn(qt, t))) < 0.4999f)) << j;
      v[j] = t;                                 // v now holds the rounded quotients
    }
    if (__any_sync(0xffffffffu, need_exact != 0)) {
      // rare: re-read the weights and divide
#pragma unroll 1
      for (int j = 0; j < 64; ++j)
        if ((need_exact >> j) & 1u) v[j] = rintf(__fdiv_rn(__ldg(w + (valid ? g : 0) * kGroup + j), sf));
    }
    const bool bad = !width_good || !finite || overflow;
    if (valid) {
      if (bad) flags |= !width_good ? CQ_QSTATUS_BADBITS : (!finite ? CQ_QSTATUS_NONFINITE : CQ_QSTATUS_RANGE);
      const float zf = static_cast<float>(z), Lf = static_cast<float>(L);
      uint4 *dst = reinterpret_cast<uint4 *>(codes + g * kGroup);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t wd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float q = fminf(fmaxf(__fadd_rn(v[16 * c + 4 * k + e], zf), 0.0f), Lf);
            word |= static_cast<uint32_t>(static_cast<int>(q)) << (8 * e);
          }
          wd[k] = bad ? 0u : word;
        }
        __stcs(dst + c, make_uint4(wd[0], wd[1], wd[2], wd[3]));
      }
      scale[g] = bad ? 0 : s16;
      zero[g] = bad ? 0 : static_cast<uint8_t>(z);
    }
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if ((threadIdx.x & 31) == 0 && flags && status) atomicOr(status, flags);
}

}  // namespace

cq_status launch_quantize(const float *w, int64_t G, const uint8_t *bits, uint8_t *codes,
                          uint16_t *scale, uint8_t *zero, uint32_t *status, cudaStream_t s) {
  if (status) {
    cq_status st = cuda_check(cudaMemsetAsync(status, 0, sizeof(uint32_t), s), "cq_quantize: clear status");
    if (st != CQ_OK) return st;
  }
  if (G == 0) return CQ_OK;
  const int64_t need = (G + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  quantize_kernel<<<blocks, kThreads, 0, s>>>(w, G, bits, codes, scale, zero, status);
  return launch_check("cq_quantize");
}

}  // namespace cq
