// k_verify.cu -- bit-exact re-quantization check of a quantized release (+ residual).
//
// [CF] "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
// Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: rounding the served
// weights again with the frozen grid must reproduce the released codes exactly, which a
// program can check, and removing the residual must undo the update. For every weight:
//     k = q - z;  w' = RN32(RN32(s*k) + r);  t = RN32(w'/s);  q' = clamp(rne(t) + z, 0, L)
// and a mismatch is q' != q, a NaN t included.
//
// Exactness without a division per weight: s*k is exact in binary32 (11 + 8 significant
// bits), so fma(s, k, r) = RN32(RN32(s*k) + r). With rc = RN32(1/s), qt = RN32(w' * rc)
// lies within 3.1e-5 of w'/s whenever |qt| < 256, and RN32(w'/s) within 1.6e-5 of it. If
// |qt - k| < 0.5 - 2^-11 the rounded quotient is within 0.4996 of k, so rne gives k and
// q' = clamp(k + z) = q: no mismatch, decided exactly. Any other weight (a residual near
// or outside the cell edge, a NaN, a zero/infinite scale) takes the exact IEEE path.
//
// Layout: one lane per 8 consecutive weights: a 4-byte code word (fixed 4-bit) or the
// lane's b bytes of its group (per-group widths), plus 16 bytes of bf16 residual or 32
// of fp32. Mismatch counts are warp-aggregated; the smallest index and the per-group
// flags are only touched when a warp sees a mismatch.
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;

struct VerifyArgs {
  const uint8_t *bits;
  const uint32_t *offset;
  const uint8_t *plane[4];
  const uint16_t *scale;
  const uint8_t *zero;
  const void *r;
  int64_t first_w;
  int64_t n_units;    // n_w / 8
  unsigned long long *mism;
  unsigned long long *first_bad;   // int64 in the ABI; -1 is the all-ones pattern
  uint32_t *flags;
};

enum RKind { kNoR = 0, kF32 = 1, kBF16 = 2 };

template <int RK>
__device__ __forceinline__ void load_residual(const void *r, int64_t i0, float rv[8]) {
  if (RK == kBF16) {
    const uint4 t = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(r) + i0));
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      rv[2 * j] = __uint_as_float(w[j] << 16);
      rv[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else if (RK == kF32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(r) + i0);
    const float4 a = __ldcs(p), b = __ldcs(p + 1);
    rv[0] = a.x; rv[1] = a.y; rv[2] = a.z; rv[3] = a.w;
    rv[4] = b.x; rv[5] = b.y; rv[6] = b.z; rv[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) rv[j] = 0.0f;
  }
}

// the definition, evaluated with IEEE operations only
template <bool HAS_R>
__device__ __forceinline__ bool exact_match(int q, int z, int L, float sf, float r) {
  const float k = static_cast<float>(q - z);
  float wp = __fmul_rn(sf, k);
  if (HAS_R) wp = __fadd_rn(wp, r);
  const float t = __fdiv_rn(wp, sf);
  if (isnan(t)) return false;
  return clamp_code(__fadd_rn(rintf(t), static_cast<float>(z)), L) == q;
}

template <bool VAR, int RK>
__global__ void __launch_bounds__(kThreads) verify_kernel(VerifyArgs a) {
  const int lane = threadIdx.x & 31;
  uint32_t count = 0;
  int64_t first = INT64_MAX;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  // warp-uniform trip count (ballots below)
  const int64_t base_u = blockIdx.x * static_cast<int64_t>(kThreads) + (threadIdx.x & ~31);
  for (int64_t u0 = base_u; u0 < a.n_units; u0 += step) {
    const int64_t u = u0 + lane;
    const bool valid = u < a.n_units;
    const int64_t i0 = a.first_w + 8 * u;
    const int64_t g = i0 >> 6;
    uint32_t bad = 0;   // bit j: weight i0+j mismatches
    if (valid) {
      int b = 4;
      uint64_t word;
      if (VAR) {
        b = __ldg(a.bits + g);
        if (!width_ok(b)) b = 0;
        if (b) {
          const uint8_t *src = a.plane[width_slot(b)] + __ldg(a.offset + g) + ((i0 >> 3) & 7) * b;
          switch (b) {
            case 1: word = __ldg(src); break;
            case 2: word = __ldg(reinterpret_cast<const uint16_t *>(src)); break;
            case 4: word = __ldg(reinterpret_cast<const uint32_t *>(src)); break;
            default: {
              const uint2 t = __ldg(reinterpret_cast<const uint2 *>(src));
              word = static_cast<uint64_t>(t.x) | (static_cast<uint64_t>(t.y) << 32);
            }
          }
        } else {
          word = 0;
        }
      } else {
        word = __ldcs(reinterpret_cast<const uint32_t *>(a.plane[2]) + (i0 >> 3));
      }
      float rv[8];
      load_residual<RK>(a.r, i0, rv);
      const float sf = f16_bits_to_f32(__ldg(a.scale + g));
      const int z = __ldg(a.zero + g);
      const float rc = __frcp_rn(sf);
      const int L = b ? (1 << b) - 1 : 0;
      const uint64_t mask = b ? (1ull << b) - 1ull : 0ull;
      uint32_t slow = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = static_cast<int>((word >> (j * b)) & mask);
        const float k = static_cast<float>(q - z);
        const float wp = RK == kNoR ? __fmul_rn(sf, k) : __fmaf_rn(sf, k, rv[j]);
        const float d = __fsub_rn(__fmul_rn(wp, rc), k);
        slow |= static_cast<uint32_t>(!(fabsf(d) < 0.49951171875f)) << j;
      }
      if (VAR && b == 0) {
        bad = 0xFFu;   // a width outside {1,2,4,8}: no code of the group can be re-derived
      } else if (slow) {
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          if (!((slow >> j) & 1)) continue;
          const int q = static_cast<int>((word >> (j * b)) & mask);
          if (!exact_match<RK != kNoR>(q, z, L, sf, rv[j])) bad |= 1u << j;
        }
      }
    }
    const uint32_t any = __ballot_sync(0xffffffffu, bad != 0);
    if (any) {
      count += __popc(bad);
      if (bad) {
        const int64_t fi = i0 + (__ffs(bad) - 1);
        first = fi < first ? fi : first;
      }
      if (a.flags) {
        // units u0..u0+31 start on a multiple of 32, so the 8 units of a group are lanes
        // 8j..8j+7 of one warp; lane 8j publishes the group's flag
        const uint32_t gb = __ballot_sync(0xffffffffu, bad != 0);
        if (valid && (lane & 7) == 0 && ((gb >> lane) & 0xFFu)) {
          const int64_t gl = g - (a.first_w >> 6);
          atomicOr(a.flags + (gl >> 5), 1u << (gl & 31));
        }
      }
    }
  }
  count = __reduce_add_sync(0xffffffffu, count);
  if (lane == 0 && count) atomicAdd(a.mism, static_cast<unsigned long long>(count));
  if (first != INT64_MAX) atomicMin(a.first_bad, static_cast<unsigned long long>(first));
}

template <bool VAR>
void dispatch(int rk, VerifyArgs a, int blocks, cudaStream_t s) {
  switch (rk) {
    case kNoR: verify_kernel<VAR, kNoR><<<blocks, kThreads, 0, s>>>(a); break;
    case kF32: verify_kernel<VAR, kF32><<<blocks, kThreads, 0, s>>>(a); break;
    default: verify_kernel<VAR, kBF16><<<blocks, kThreads, 0, s>>>(a); break;
  }
}

}  // namespace

cq_status launch_verify(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism,
                        int64_t *first_bad, uint32_t *flags, cudaStream_t s) {
  cq_status st = cuda_check(cudaMemsetAsync(mism, 0, sizeof(uint64_t), s), "cq_requant_verify: clear count");
  if (st != CQ_OK) return st;
  st = cuda_check(cudaMemsetAsync(first_bad, 0xFF, sizeof(int64_t), s), "cq_requant_verify: clear first");
  if (st != CQ_OK) return st;
  const int64_t n_groups = n_w / kGroup;
  if (flags) {
    st = cuda_check(cudaMemsetAsync(flags, 0, static_cast<size_t>((n_groups + 31) / 32) * 4, s),
                    "cq_requant_verify: clear flags");
    if (st != CQ_OK) return st;
  }
  if (n_w == 0) return CQ_OK;
  VerifyArgs a;
  a.bits = qw.bits;
  a.offset = qw.offset;
  for (int i = 0; i < 4; ++i) a.plane[i] = qw.plane[i];
  a.scale = qw.scale;
  a.zero = qw.zero;
  a.r = qw.residual;
  a.first_w = first_w;
  a.n_units = n_w / 8;
  a.mism = reinterpret_cast<unsigned long long *>(mism);
  a.first_bad = reinterpret_cast<unsigned long long *>(first_bad);
  a.flags = flags;
  const int rk = qw.residual == nullptr ? kNoR : (qw.residual_dtype == CQ_BF16 ? kBF16 : kF32);
  const int64_t need = (a.n_units + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  if (qw.bits)
    dispatch<true>(rk, a, blocks, s);
  else
    dispatch<false>(rk, a, blocks, s);
  return launch_check("cq_requant_verify");
}

}  // namespace cq
