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
#include "cq_async.cuh"

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
  unsigned long long *mism0;       // pair mode: the same check without the residual (revocation)
  unsigned long long *first0;
};

// the results start at 0 mismatches and first index -1; one thread, then the verify grid
// (launched as its programmatic dependent) may start. Itself a programmatic dependent: it lets
// the verify grid start only after its own wait, when the kernel before it (which may have
// written the residual the verify grid reads) has finished.
__global__ void verify_clear_kernel(unsigned long long *mism, unsigned long long *first,
                                    unsigned long long *mism0, unsigned long long *first0) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    *mism = 0ull;
    *first = ~0ull;
    if (mism0) *mism0 = 0ull;
    if (first0) *first0 = ~0ull;
  }
}

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
  pdl_wait();                                    // inputs and cleared results from earlier work
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
          // select the plane without indexing the parameter array (keeps it out of local memory)
          const uint8_t *pl = b == 1 ? a.plane[0] : b == 2 ? a.plane[1] : b == 4 ? a.plane[2] : a.plane[3];
          const uint32_t o = __ldg(a.offset + g);
          // debug build: an offset off its grid or with a rank above the group's index is
          // recorded and read as rank 0
          const uint32_t oc = CQ_CHECK(o % (8u * b) == 0u && static_cast<int64_t>(o / (8u * b)) <= g, 0x0401u) ? o : 0u;
          const uint8_t *src = pl + oc + ((i0 >> 3) & 7) * b;
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
#pragma unroll
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

// ---- fixed 4-bit fast kernel ------------------------------------------------------------
// One lane per 32 consecutive weights (16 bytes of codes, 64 bytes of bf16 residual), so each
// lane keeps 80 bytes in flight; pairs of weights go through the packed fp32x2 pipe. The
// filter here is d = RN32(w' * rc - k) in one fused step: w' * rc is within |w'/s| * 2^-24 of
// w'/s, so |d| < 0.5 - 2^-11 again leaves RN32(w'/s) within 0.4996 of k. The per-weight test
// is folded into a NaN-propagating running maximum of |d|; a lane whose maximum reaches the
// threshold re-derives its 32 weights with the exact IEEE definition. Without a residual the
// bound needs no per-weight arithmetic: w' = s*k is exact, |d| <= |k| * |s*rc - 1| (1 + 2^-24),
// and |k| <= max(qor - z, z) with qor the bitwise OR of the lane's 32 codes bounds all 32.
__device__ __forceinline__ float max_nan_abs(float m, float d) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;\n" : "=f"(r) : "f"(m), "f"(fabsf(d)));
  return r;
}

// -(2^23 + q) as a float, for a nibble q already in the low bits
__device__ __forceinline__ float neg_magic_code(uint32_t bits) { return __uint_as_float(0xCB000000u | bits); }

// kPair: the same pass also checks the artifact without the residual (revocation) from the
// codes and metadata already in registers; its certificate is that of the no-residual case
template <int RK, bool kPair>
__global__ void __launch_bounds__(kThreads) verify4_kernel(VerifyArgs a) {
  pdl_wait();                                    // inputs and cleared results from earlier work
  const int lane = threadIdx.x & 31;
  uint32_t count = 0, count0 = 0;
  int64_t first = INT64_MAX, first0 = INT64_MAX;
  const int64_t n32 = a.n_units >> 2;            // units of 32 weights
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  const int64_t base_u = blockIdx.x * static_cast<int64_t>(kThreads) + (threadIdx.x & ~31);
  for (int64_t u0 = base_u; u0 < n32; u0 += step) {
    const int64_t u = u0 + lane;
    const bool valid = u < n32;
    uint32_t bad = 0, bad0 = 0;
    int64_t i0 = 0;
    int64_t g = 0;
    if (valid) {
      i0 = a.first_w + 32 * u;
      g = i0 >> 6;
      const uint4 cw = __ldcs(reinterpret_cast<const uint4 *>(a.plane[2] + (i0 >> 1)));
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
      uint32_t rw[16];
      if (RK == kBF16) {
        const uint4 *rp = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.r) + i0);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 t = __ldcs(rp + v);
          rw[4 * v] = t.x; rw[4 * v + 1] = t.y; rw[4 * v + 2] = t.z; rw[4 * v + 3] = t.w;
        }
      }
      float rf[32];
      if (RK == kF32) {
        const float4 *rp = reinterpret_cast<const float4 *>(static_cast<const float *>(a.r) + i0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 t = __ldcs(rp + v);
          rf[4 * v] = t.x; rf[4 * v + 1] = t.y; rf[4 * v + 2] = t.z; rf[4 * v + 3] = t.w;
        }
      }
      const float sf = f16_bits_to_f32(__ldg(a.scale + g));
      const int z = __ldg(a.zero + g);
      const float rc = __frcp_rn(sf);
      const float kb = 8388608.0f + static_cast<float>(z);     // 2^23 + z, exact
      const float2 kb2 = make_float2(kb, kb), ns2 = make_float2(-sf, -sf), rc2 = make_float2(rc, rc);
      float m = 0.0f;
      if (RK == kNoR) {
        // No residual: w' = s*k exactly, so |RN32(w' * rc - k)| <= |k| * |s * rc - 1| (1 + 2^-24).
        // |k| = |q - z| <= max(qor - z, z), qor = the OR of the lane's 32 codes (>= each code).
        uint32_t qor = words[0] | words[1] | words[2] | words[3];
        qor = (qor | (qor >> 4)) & 0x0F0F0F0Fu;
        qor |= qor >> 16;
        qor = (qor | (qor >> 8)) & 0xFu;
        const float kmax = static_cast<float>(max(static_cast<int>(qor) - z, z));
        const float eps = fabsf(__fmaf_rn(sf, rc, -1.0f));      // |s * rc - 1|, exact in one fma
        m = __fmul_rn(__fmul_rn(kmax, eps), 1.0f + 0x1p-22f);   // NaN when s is 0, inf or NaN
      } else {
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        const uint32_t w = words[wi];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int j = 8 * wi + 2 * p;                          // weights j, j+1
          // nk = z - q = -k exactly; w' = (-s) * nk + r = RN32(s*k + r); d = RN32(w' * rc - k)
          const float2 nk = __fadd2_rn(make_float2(neg_magic_code((w >> (8 * p)) & 0xFu),
                                                   neg_magic_code((w >> (8 * p + 4)) & 0xFu)), kb2);
          float2 wp;
          if (RK == kBF16) {
            const uint32_t r2 = rw[j >> 1];
            wp = __ffma2_rn(ns2, nk, make_float2(__uint_as_float(r2 << 16), __uint_as_float(r2 & 0xFFFF0000u)));
          } else if (RK == kF32) {
            wp = __ffma2_rn(ns2, nk, make_float2(rf[j], rf[j + 1]));
          } else {
            wp = __fmul2_rn(ns2, nk);
          }
          const float2 d = __ffma2_rn(wp, rc2, nk);
          m = max_nan_abs(m, d.x);
          m = max_nan_abs(m, d.y);
        }
      }
      }
      if (!(m < 0.49951171875f)) {
        // the exact definition, weight by weight, on inputs re-read from memory (rare path)
#pragma unroll 1
        for (int j = 0; j < 32; ++j) {
          const int64_t i = i0 + j;
          const int q = static_cast<int>((__ldg(a.plane[2] + (i >> 1)) >> (4 * (i & 1))) & 0xFu);
          float r = 0.0f;
          if (RK == kBF16) r = bf16_bits_to_f32(__ldg(static_cast<const uint16_t *>(a.r) + i));
          if (RK == kF32) r = __ldg(static_cast<const float *>(a.r) + i);
          if (!exact_match<RK != kNoR>(q, z, 15, sf, r)) bad |= 1u << j;
        }
      }
      if (kPair) {
        uint32_t qor = words[0] | words[1] | words[2] | words[3];
        qor = (qor | (qor >> 4)) & 0x0F0F0F0Fu;
        qor |= qor >> 16;
        qor = (qor | (qor >> 8)) & 0xFu;
        const float kmax = static_cast<float>(max(static_cast<int>(qor) - z, z));
        const float m0 = __fmul_rn(__fmul_rn(kmax, fabsf(__fmaf_rn(sf, rc, -1.0f))), 1.0f + 0x1p-22f);
        if (!(m0 < 0.49951171875f)) {
#pragma unroll 1
          for (int j = 0; j < 32; ++j) {
            const int64_t i = i0 + j;
            const int q = static_cast<int>((__ldg(a.plane[2] + (i >> 1)) >> (4 * (i & 1))) & 0xFu);
            if (!exact_match<false>(q, z, 15, sf, 0.0f)) bad0 |= 1u << j;
          }
        }
      }
    }
    if (kPair && __ballot_sync(0xffffffffu, bad0 != 0)) {
      count0 += __popc(bad0);
      if (bad0) {
        const int64_t fi = i0 + (__ffs(bad0) - 1);
        first0 = fi < first0 ? fi : first0;
      }
    }
    const uint32_t any = __ballot_sync(0xffffffffu, bad != 0);
    if (any) {
      count += __popc(bad);
      if (bad) {
        const int64_t fi = i0 + (__ffs(bad) - 1);
        first = fi < first ? fi : first;
      }
      if (a.flags && bad) {
        // the two lanes of a group may both publish; atomicOr makes that harmless
        const int64_t gl = g - (a.first_w >> 6);
        atomicOr(a.flags + (gl >> 5), 1u << (gl & 31));
      }
    }
  }
  count = __reduce_add_sync(0xffffffffu, count);
  if (lane == 0 && count) atomicAdd(a.mism, static_cast<unsigned long long>(count));
  if (first != INT64_MAX) atomicMin(a.first_bad, static_cast<unsigned long long>(first));
  if (kPair) {
    count0 = __reduce_add_sync(0xffffffffu, count0);
    if (lane == 0 && count0) atomicAdd(a.mism0, static_cast<unsigned long long>(count0));
    if (first0 != INT64_MAX) atomicMin(a.first0, static_cast<unsigned long long>(first0));
  }
}

// Revocation (no residual) of fixed-4 weights moves only 0.55 bytes per weight, so a lane
// keeps four 32-weight units in flight: a warp reads 4 x 512 contiguous bytes of codes (plus
// their scales and zeros) before it computes, which quadruples the bytes in flight per SM. The certificate is that of verify4_kernel without a residual.
constexpr int kRevokeUnroll = 4;

__global__ void __launch_bounds__(kThreads) revoke4_kernel(VerifyArgs a) {
  pdl_wait();                                    // inputs and cleared results from earlier work
  const int lane = threadIdx.x & 31;
  uint32_t count = 0;
  int64_t first = INT64_MAX;
  const int64_t n32 = a.n_units >> 2;            // units of 32 weights
  const int64_t warp_id = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  const int64_t step = static_cast<int64_t>(gridDim.x) * (kThreads / 32) * 32 * kRevokeUnroll;
  for (int64_t base = warp_id * 32 * kRevokeUnroll; base < n32; base += step) {
    uint4 cw[kRevokeUnroll];
    uint32_t sbits[kRevokeUnroll], zv[kRevokeUnroll];
#pragma unroll
    for (int k = 0; k < kRevokeUnroll; ++k) {
      const int64_t u = base + 32 * k + lane;
      cw[k] = make_uint4(0, 0, 0, 0);
      sbits[k] = 0x3C00u;                        // 1.0 for lanes past the end (never counted)
      zv[k] = 0;
      if (u < n32) {
        const int64_t i0 = a.first_w + 32 * u;
        cw[k] = __ldcs(reinterpret_cast<const uint4 *>(a.plane[2] + (i0 >> 1)));
        sbits[k] = __ldg(a.scale + (i0 >> 6));
        zv[k] = __ldg(a.zero + (i0 >> 6));
      }
    }
#pragma unroll
    for (int k = 0; k < kRevokeUnroll; ++k) {
      const int64_t u = base + 32 * k + lane;
      const bool valid = u < n32;
      const int64_t i0 = a.first_w + 32 * u;
      const int64_t g = i0 >> 6;
      const float sf = f16_bits_to_f32(static_cast<uint16_t>(sbits[k]));
      const int z = static_cast<int>(zv[k]);
      const float rc = __frcp_rn(sf);
      // |RN32(s*k * rc) - k| <= |k| * |s * rc - 1| (1 + 2^-24), |k| <= max(qor - z, z)
      uint32_t qor = cw[k].x | cw[k].y | cw[k].z | cw[k].w;
      qor = (qor | (qor >> 4)) & 0x0F0F0F0Fu;
      qor |= qor >> 16;
      qor = (qor | (qor >> 8)) & 0xFu;
      const float kmax = static_cast<float>(max(static_cast<int>(qor) - z, z));
      const float eps = fabsf(__fmaf_rn(sf, rc, -1.0f));
      const float m = __fmul_rn(__fmul_rn(kmax, eps), 1.0f + 0x1p-22f);   // NaN when s is 0, inf or NaN
      uint32_t bad = 0;
      if (valid && !(m < 0.49951171875f)) {
        // the exact definition, weight by weight (rare path)
#pragma unroll 1
        for (int j = 0; j < 32; ++j) {
          const int64_t i = i0 + j;
          const int q = static_cast<int>((__ldg(a.plane[2] + (i >> 1)) >> (4 * (i & 1))) & 0xFu);
          if (!exact_match<false>(q, z, 15, sf, 0.0f)) bad |= 1u << j;
        }
      }
      if (__ballot_sync(0xffffffffu, bad != 0)) {
        count += __popc(bad);
        if (bad) {
          const int64_t fi = i0 + (__ffs(bad) - 1);
          first = fi < first ? fi : first;
        }
        if (a.flags && bad) {
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

// the verify grids are programmatic dependents of the clearing kernel: their CTAs may be
// scheduled while it runs, and wait (griddepcontrol.wait) before touching memory
template <typename Kern>
cudaError_t launch_pdl(Kern kern, int blocks, const VerifyArgs &a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool VAR>
cudaError_t dispatch(int rk, const VerifyArgs &a, int blocks, cudaStream_t s) {
  switch (rk) {
    case kNoR: return launch_pdl(verify_kernel<VAR, kNoR>, blocks, a, s);
    case kF32: return launch_pdl(verify_kernel<VAR, kF32>, blocks, a, s);
    default: return launch_pdl(verify_kernel<VAR, kBF16>, blocks, a, s);
  }
}

cudaError_t dispatch4(int rk, bool pair, const VerifyArgs &a, int blocks, cudaStream_t s) {
  if (pair) return rk == kF32 ? launch_pdl(verify4_kernel<kF32, true>, blocks, a, s)
                              : launch_pdl(verify4_kernel<kBF16, true>, blocks, a, s);
  switch (rk) {
    case kNoR: return launch_pdl(revoke4_kernel, blocks, a, s);
    case kF32: return launch_pdl(verify4_kernel<kF32, false>, blocks, a, s);
    default: return launch_pdl(verify4_kernel<kBF16, false>, blocks, a, s);
  }
}

// clear the results (flags by memset, then the counters by one small kernel) and launch the
// verify grid; pair = fixed-4 with a residual, checked with it and without it in one pass
cq_status launch_verify_impl(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism, int64_t *first_bad,
                             uint64_t *mism0, int64_t *first0, uint32_t *flags, bool pair, cudaStream_t s,
                             const char *who) {
  const int64_t n_groups = n_w / kGroup;
  if (flags) {
    cq_status st = cuda_check(cudaMemsetAsync(flags, 0, static_cast<size_t>((n_groups + 31) / 32) * 4, s), who);
    if (st != CQ_OK) return st;
  }
  // the library-wide launcher (this file's launch_pdl above takes verify arguments)
  cq_status st = cuda_check(::cq::launch_pdl(verify_clear_kernel, dim3(1), dim3(32), 0, s,
                                             reinterpret_cast<unsigned long long *>(mism),
                                             reinterpret_cast<unsigned long long *>(first_bad),
                                             reinterpret_cast<unsigned long long *>(mism0),
                                             reinterpret_cast<unsigned long long *>(first0)),
                            who);
  if (st != CQ_OK) return st;
  st = launch_check(who);
  if (st != CQ_OK || n_w == 0) return st;
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
  a.mism0 = reinterpret_cast<unsigned long long *>(mism0);
  a.first0 = reinterpret_cast<unsigned long long *>(first0);
  const int rk = qw.residual == nullptr ? kNoR : (qw.residual_dtype == CQ_BF16 ? kBF16 : kF32);
  const int64_t need = (a.n_units + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  cudaError_t e;
  if (qw.bits) {
    e = dispatch<true>(rk, a, blocks, s);
  } else {
    // 32 weights per lane; n_w is a multiple of 64
    const int64_t need4 = (a.n_units / 4 + kThreads - 1) / kThreads;
    e = dispatch4(rk, pair, a, static_cast<int>(need4 < cap ? need4 : cap), s);
  }
  st = cuda_check(e, who);
  if (st != CQ_OK) return st;
  return launch_check(who);
}

}  // namespace

cq_status launch_verify(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism,
                        int64_t *first_bad, uint32_t *flags, cudaStream_t s) {
  return launch_verify_impl(qw, first_w, n_w, mism, first_bad, nullptr, nullptr, flags, false, s,
                            "cq_requant_verify");
}

cq_status launch_verify_pair(const cq_qweight &qw, int64_t first_w, int64_t n_w, uint64_t *mism, int64_t *first_bad,
                             uint64_t *mism0, int64_t *first0, uint32_t *flags, cudaStream_t s) {
  const char *who = "cq_requant_verify_pair";
  if (qw.bits == nullptr)
    return launch_verify_impl(qw, first_w, n_w, mism, first_bad, mism0, first0, flags, true, s, who);
  // per-group widths: the two checks as two passes
  cq_status st = launch_verify_impl(qw, first_w, n_w, mism, first_bad, nullptr, nullptr, flags, false, s, who);
  if (st != CQ_OK) return st;
  cq_qweight q0 = qw;
  q0.residual = nullptr;
  return launch_verify_impl(q0, first_w, n_w, mism0, first0, nullptr, nullptr, nullptr, false, s, who);
}

}  // namespace cq
