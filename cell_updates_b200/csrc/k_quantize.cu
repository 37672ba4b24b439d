// k_quantize.cu -- per-group asymmetric min-max round-to-nearest quantization.
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: groups of 64 consecutive weights, each
// with its own width from {1,2,4,8}. [CF] "Nothing Changed but the Model: CellFill ...",
// Abstract: 4-bit integer codes and scales. [SLQ] abstract (page 2 listing): asymmetric
// grids. Reading of the formula: see include/cq.h.
//
// Every fp32 operation is an explicit round-to-nearest intrinsic, so nothing is contracted.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 1;                       // the warp's tile buffer: refilled as soon as it is in registers
constexpr int kTileGroups = 32;                  // one tile: 32 groups, one per lane
constexpr int kBoxBytes = kTileGroups * 128;     // one box: 32 groups x 32 floats (128-byte rows)
constexpr int kTileBytes = 2 * kBoxBytes;        // 8 KiB of fp32 weights
constexpr int kSmem = 1024 + kWarps * kStages * kTileBytes + kWarps * kStages * 8 + 16;

// One thread owns one group of 64 weights: the group's scale and zero point (two IEEE
// divisions, a reciprocal) are paid once per 64 weights and min/max need no shuffles. The
// weights reach shared memory through TMA: each warp owns a buffer for one tile of 32 groups,
// two boxes of {32 floats, 32 groups} with the 128-byte swizzle, so a lane reads its own
// group's 16-byte chunks without bank conflicts (chunk c of row r sits at c ^ (r & 7)). Once
// the tile is in registers the warp requests its next tile, which streams in while it computes
// (16 warps per SM: measured faster than fewer warps with deeper rings).
//
// With kResid (one stage of recurrent residual quantization, [RRQ] the 2512.18934 listing
// page, "Recurrent Residual Quantization" abstract: 2-bit round-to-nearest residual
// corrections stacked on a 2-bit base) the warp keeps its tile buffer until the stage is done:
// each thread replaces its group's row in the buffer by what the stage does not represent,
// r <- RN32(r - s (q - z)) (the product exact; a flagged group keeps its values), and one lane
// writes the two boxes back in place with TMA stores; the buffer is refilled once the stores
// have read it. w is read and written through the tensor map only (tiles are disjoint), plus
// a thread's own rare exact-division re-read of its group before its row is stored, so it
// carries no __restrict__.
template <bool kResid>
__global__ void __launch_bounds__(kThreads, 1)
quantize_kernel(const __grid_constant__ CUtensorMap tm_w, float *w, int64_t G, const uint8_t *__restrict__ bits,
                int uniform_b, uint8_t *__restrict__ codes, uint16_t *__restrict__ scale,
                uint8_t *__restrict__ zero, uint32_t *__restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t *ring = smem + warp * kStages * kTileBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWarps * kStages * kTileBytes) + warp * kStages;
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + kWarps * kStages * kTileBytes +
                                                                        kWarps * kStages * 8);
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(bars + i, 1);
    mbar_init_fence();
  }
  if (threadIdx.x == 0) *abort_flag = 0u;
  __syncthreads();
  pdl_wait();                     // w, the cleared status word and the outputs' earlier readers

  uint32_t flags = 0;
  const int64_t n_tiles = (G + kTileGroups - 1) / kTileGroups;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t t_first = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  auto issue = [&](int slot, int64_t tile) {
#ifdef CQ_TEST_DROP_FIRST_COPY
    // test build only (never in libcq.so): CTA 0's warp 0 does not request its first tile, so
    // its first wait runs out after the bounded limit and the abort path runs
    if (blockIdx.x == 0 && warp == 0 && tile == t_first) return;
#endif
    uint64_t *bar = bars + slot;
    uint8_t *dst = ring + slot * kTileBytes;
    mbar_arrive_expect_tx(bar, kTileBytes);
    tma_load_2d(dst, &tm_w, 0, static_cast<int>(tile * kTileGroups), bar);
    tma_load_2d(dst + kBoxBytes, &tm_w, 32, static_cast<int>(tile * kTileGroups), bar);
  };
  int n_issued = 0, n_done = 0;
  if (lane == 0)
    for (int64_t t = t_first; n_issued < kStages && t < n_tiles; t += stride, ++n_issued) issue(n_issued, t);
  n_issued = __shfl_sync(0xffffffffu, n_issued, 0);
  int slot = 0;
  uint32_t phase = 0;
  for (int64_t tile = t_first; tile < n_tiles; tile += stride) {
    const bool got = mbar_wait(bars + slot, phase, abort_flag, nullptr);
    if (!__all_sync(0xffffffffu, got)) {
      flags |= CQ_QSTATUS_TIMEOUT;
      break;
    }
    const int64_t g = tile * kTileGroups + lane;
    const bool valid = g < G;
    float v[64];
    const uint8_t *row = ring + slot * kTileBytes + lane * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 t4 = *reinterpret_cast<const float4 *>(row + h * kBoxBytes + ((c ^ (lane & 7)) << 4));
        v[32 * h + 4 * c] = t4.x; v[32 * h + 4 * c + 1] = t4.y; v[32 * h + 4 * c + 2] = t4.z; v[32 * h + 4 * c + 3] = t4.w;
      }
    }
    // NaN-propagating min/max: a NaN or an infinity shows up as a non-finite extreme
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int j = 1; j < 64; ++j) {
      asm("min.NaN.f32 %0, %0, %1;\n" : "+f"(lo) : "f"(v[j]));
      asm("max.NaN.f32 %0, %0, %1;\n" : "+f"(hi) : "f"(v[j]));
    }
    // every lane's words of this slot are in registers (min/max consumed them): refill it (a
    // residual stage refills after writing the slot back); the proxy fence orders these generic
    // reads before the TMA write into the slot
    fence_proxy_async_smem();
    __syncwarp();
    ++n_done;
    const int cur = slot;
    const int64_t next = tile + static_cast<int64_t>(kStages) * stride;
    if (!kResid) {
      if (next < n_tiles) {
        if (lane == 0) issue(slot, next);
        ++n_issued;
      }
    }
    if (++slot == kStages) { slot = 0; phase ^= 1u; }
    const bool finite = isfinite(lo) && isfinite(hi);
    const int b = (bits && valid) ? static_cast<int>(__ldg(bits + g)) : uniform_b;
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
    // t_j = rne(RN32(w_j / s)) through a division-free certificate. With rc = RN(1/s) and
    // qt = RN32(w_j * rc): qt = (w/s)(1 + d1)(1 + d2) and RN32(w/s) = (w/s)(1 + d3), |d_i| <= 2^-24,
    // so |RN32(w_j / s) - qt| <= 1.5 * 2^-23 |w/s| < 2^-22 |qt|. If RN(|qt| 2^-22 + |qt - t|) is
    // below 0.5 - 2^-20 (t = rint(qt); qt - t is exact), RN32(w_j / s) is within 0.5 of t and
    // rounds to it. Otherwise (near a half-way point, huge, non-finite: ~1e-5 of the weights) the
    // thread redoes its whole group with the IEEE division.
    bool need_exact = false;
#pragma unroll
    for (int j = 0; j < 64; j += 2) {
      const float2 qt = __fmul2_rn(make_float2(v[j], v[j + 1]), make_float2(rc, rc));
      // t = rne(qt) for |qt| < 2^22 as (qt + 1.5 2^23) - 1.5 2^23 (two packed adds, no rounding
      // instruction); a larger or non-finite qt fails the certificate below (|qt| 2^-22 >= 1, or
      // NaN) and takes the exact path, which rounds with rintf
      const float2 t = __fadd2_rn(__fadd2_rn(qt, make_float2(12582912.0f, 12582912.0f)),
                                  make_float2(-12582912.0f, -12582912.0f));
      const float2 d = __fadd2_rn(qt, make_float2(-t.x, -t.y));
      const float2 m = __ffma2_rn(make_float2(fabsf(qt.x), fabsf(qt.y)), make_float2(0x1p-22f, 0x1p-22f),
                                  make_float2(fabsf(d.x), fabsf(d.y)));
      need_exact |= !(m.x < 0.5f - 0x1p-20f) || !(m.y < 0.5f - 0x1p-20f);
      v[j] = t.x;                               // v now holds the rounded quotients
      v[j + 1] = t.y;
    }
    if (__any_sync(0xffffffffu, need_exact)) {
      // rare: re-read the group and divide every weight
      if (need_exact) {
        const float *wg = w + (valid ? g : 0) * kGroup;
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = rintf(__fdiv_rn(wg[j], sf));   // unrolled: v stays in registers
      }
    }
    const bool bad = !width_good || !finite || overflow;
    if (valid) {
      if (bad) flags |= !width_good ? CQ_QSTATUS_BADBITS : (!finite ? CQ_QSTATUS_NONFINITE : CQ_QSTATUS_RANGE);
      // clamp(t + z, 0, L) in the float domain, offset by 2^23 so the integer sits in the low
      // mantissa bits: t + (2^23 + z) is exact whenever the clamp does not bind, and when it
      // does the rounded sum is still on the same side of the clamp interval
      const float kb = 8388608.0f + static_cast<float>(z), kl = 8388608.0f + static_cast<float>(L);
      uint4 *dst = reinterpret_cast<uint4 *>(codes + g * kGroup);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t wd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t e4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float cl = fminf(fmaxf(__fadd_rn(v[16 * c + 4 * k + e], kb), 8388608.0f), kl);
            e4[e] = __float_as_uint(cl);
            if (kResid) v[16 * c + 4 * k + e] = __fsub_rn(cl, kb);   // q - z, exact (both in [2^23, 2^24))
          }
          const uint32_t word = __byte_perm(__byte_perm(e4[0], e4[1], 0x0040), __byte_perm(e4[2], e4[3], 0x0040), 0x5410);
          wd[k] = bad ? 0u : word;
        }
        __stcs(dst + c, make_uint4(wd[0], wd[1], wd[2], wd[3]));
      }
      if (kResid && !bad) {
        // the new residual replaces the group's row of the tile buffer (same swizzled chunks)
        uint8_t *rrow = ring + cur * kTileBytes + lane * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float4 *p4 = reinterpret_cast<float4 *>(rrow + h * kBoxBytes + ((c ^ (lane & 7)) << 4));
            const float4 o = *p4;
            const int j = 32 * h + 4 * c;
            *p4 = make_float4(__fsub_rn(o.x, __fmul_rn(sf, v[j])), __fsub_rn(o.y, __fmul_rn(sf, v[j + 1])),
                              __fsub_rn(o.z, __fmul_rn(sf, v[j + 2])), __fsub_rn(o.w, __fmul_rn(sf, v[j + 3])));
          }
        }
      }
      scale[g] = bad ? 0 : s16;
      zero[g] = bad ? 0 : static_cast<uint8_t>(z);
    }
    if (kResid) {
      // write the tile back in place (rows past G are not written), then refill the buffer
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && CQ_CHECK(tile * kTileGroups < G, 0x0101u)) {
        const uint8_t *src = ring + cur * kTileBytes;
        tma_store_2d(&tm_w, src, 0, static_cast<int>(tile * kTileGroups));
        tma_store_2d(&tm_w, src + kBoxBytes, 32, static_cast<int>(tile * kTileGroups));
        bulk_commit();
        bulk_wait_read_all();
        if (next < n_tiles) issue(cur, next);
      }
      if (next < n_tiles) ++n_issued;
      __syncwarp();
    }
  }
  if (kResid && lane == 0) bulk_wait_all();
  // a warp that gave up lets the copies it issued land before the CTA exits
  for (; n_done < n_issued; ++n_done) {
    mbar_wait(bars + slot, phase, abort_flag, nullptr, false);
    if (++slot == kStages) { slot = 0; phase ^= 1u; }
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0 && flags && status) atomicOr(status, flags);
}

template <bool kResid>
cq_status launch_quantize_impl(float *w, int64_t G, const uint8_t *bits, int uniform_b, uint8_t *codes,
                               uint16_t *scale, uint8_t *zero, uint32_t *status, cudaStream_t s, const char *who) {
  if (status) {
    cq_status st = cuda_check(launch_clear_results(status, nullptr, s), who);
    if (st != CQ_OK) return st;
    st = launch_check(who);
    if (st != CQ_OK) return st;
  }
  if (G == 0) return CQ_OK;
  auto encode = encode_fn();
  if (!encode) return fail(CQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", who);
  if (G > (int64_t(1) << 31) - kTileGroups) return fail(CQ_ERR_RANGE, "%s: more than 2^31 groups", who);
  CUtensorMap tm;
  cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(G)};
  cuuint64_t strides[1] = {64 * sizeof(float)};
  cuuint32_t box[2] = {32, kTileGroups};
  cuuint32_t es[2] = {1, 1};
  CUresult r = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(w), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CQ_ERR_CUDA, "%s: weight tensor map (%d)", who, static_cast<int>(r));
  cq_status st = cuda_check(cudaFuncSetAttribute(quantize_kernel<kResid>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmem),
                            who);
  if (st != CQ_OK) return st;
  const int64_t tiles = (G + kTileGroups - 1) / kTileGroups;
  const int64_t need = (tiles + kWarps - 1) / kWarps;
  const int64_t cap = sm_count();
  const int blocks = static_cast<int>(need < cap ? need : cap);
  st = cuda_check(launch_pdl(quantize_kernel<kResid>, dim3(blocks), dim3(kThreads), kSmem, s, tm, w, G, bits, uniform_b,
                             codes, scale, zero, status),
                  who);
  if (st != CQ_OK) return st;
  return launch_check(who);
}

}  // namespace

cq_status launch_quantize(const float *w, int64_t G, const uint8_t *bits, uint8_t *codes,
                          uint16_t *scale, uint8_t *zero, uint32_t *status, cudaStream_t s) {
  // the plain quantizer only reads w
  return launch_quantize_impl<false>(const_cast<float *>(w), G, bits, 4, codes, scale, zero, status, s, "cq_quantize");
}

cq_status launch_rrq_stage(float *r, int64_t G, int b, uint8_t *codes, uint16_t *scale, uint8_t *zero,
                           uint32_t *status, cudaStream_t s) {
  return launch_quantize_impl<true>(r, G, nullptr, b, codes, scale, zero, status, s, "cq_rrq_stage");
}

}  // namespace cq
