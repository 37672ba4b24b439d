// k_quantize.cu -- per-group asymmetric min-max round-to-nearest quantization.
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: groups of 64 consecutive weights, each
// with its own width from {1,2,4,8}. [CF] "Nothing Changed but the Model: CellFill ...",
// Abstract: 4-bit integer codes and scales. [SLQ] abstract (page 2 listing): asymmetric
// grids. Reading of the formula: see include/cq.h.
//
// Layout: eight lanes own one group (8 fp32 each, two 16-byte loads), a warp covers four
// consecutive groups = 1 KiB of contiguous input; codes leave as one 8-byte store per lane.
// Every fp32 operation is an explicit round-to-nearest intrinsic, so nothing is contracted.
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;
constexpr int kGroupsPerBlock = kThreads / 8;

__global__ void __launch_bounds__(kThreads)
quantize_kernel(const float *__restrict__ w, int64_t G, const uint8_t *__restrict__ bits,
                uint8_t *__restrict__ codes, uint16_t *__restrict__ scale,
                uint8_t *__restrict__ zero, uint32_t *__restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  uint32_t flags = 0;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kGroupsPerBlock;
  // warp-uniform trip count: every lane takes part in the shuffles of every iteration
  const int64_t warp_first = static_cast<int64_t>(blockIdx.x) * kGroupsPerBlock + ((threadIdx.x >> 5) << 2);
  for (int64_t g0 = warp_first; g0 < G; g0 += step) {
    const int64_t g = g0 + (lane >> 3);
    const bool valid = g < G;
    float v[8];
    if (valid) {
      const float4 *p = reinterpret_cast<const float4 *>(w + g * kGroup + sub * 8);
      const float4 a = __ldcs(p), c = __ldcs(p + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    }
    bool finite = true;
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      finite = finite && isfinite(v[j]);
      lo = fminf(lo, v[j]);
      hi = fmaxf(hi, v[j]);
    }
#pragma unroll
    for (int o = 4; o; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      finite = __shfl_xor_sync(0xffffffffu, static_cast<int>(finite), o) && finite;
    }
    if (!valid) continue;
    const int b = bits ? static_cast<int>(__ldg(bits + g)) : 4;
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
    uint64_t packed = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float t = rne_quotient(v[j], sf, rc);
      const int q = clamp_code(__fadd_rn(t, static_cast<float>(z)), L);
      packed |= static_cast<uint64_t>(q) << (8 * j);
    }
    const bool bad = !width_good || !finite || overflow;
    if (bad) {
      flags |= !width_good ? CQ_QSTATUS_BADBITS : (!finite ? CQ_QSTATUS_NONFINITE : CQ_QSTATUS_RANGE);
      packed = 0;
      s16 = 0;
    }
    *reinterpret_cast<uint2 *>(codes + g * kGroup + sub * 8) =
        make_uint2(static_cast<uint32_t>(packed), static_cast<uint32_t>(packed >> 32));
    if (sub == 0) {
      scale[g] = s16;
      zero[g] = bad ? 0 : static_cast<uint8_t>(z);
    }
  }
  // the lanes that returned no flags still reach this point (no early exit above)
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0 && flags && status) atomicOr(status, flags);
}

}  // namespace

cq_status launch_quantize(const float *w, int64_t G, const uint8_t *bits, uint8_t *codes,
                          uint16_t *scale, uint8_t *zero, uint32_t *status, cudaStream_t s) {
  if (status) {
    cq_status st = cuda_check(cudaMemsetAsync(status, 0, sizeof(uint32_t), s), "cq_quantize: clear status");
    if (st != CQ_OK) return st;
  }
  if (G == 0) return CQ_OK;
  const int64_t need = (G + kGroupsPerBlock - 1) / kGroupsPerBlock;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  quantize_kernel<<<blocks, kThreads, 0, s>>>(w, G, bits, codes, scale, zero, status);
  return launch_check("cq_quantize");
}

}  // namespace cq
