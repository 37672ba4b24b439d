// k_gemv.cu -- fused dequantize-and-multiply for decode (batch m <= 8).
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: packed low-bit weights served by fused
// dequantize-and-multiply kernels; decode is memory-bandwidth bound. The served weight is
// W = s*(q - z) + r ([CF] "Nothing Changed but the Model: CellFill ...", Abstract).
//     y[i, n] = sum_k W[n, k] * x[i, k]      (fp32 accumulation)
//
// Two kernels:
//  * gemv4_mma: fixed 4-bit codes, bf16 x, no residual -- the decode hot path. Per group of
//    64 columns, sum_k W x = s * (sum_k (128 + q) x - (128 + z) * sum_k x). The operand
//    128 + q is built from a nibble with one LOP3 as the bf16 bit pattern 0x4300 | q (exact;
//    bf16 has 8 significant bits), x is bf16 already, so the tensor-core products are exact
//    and accumulate in fp32 (mma.sync m16n8k16). Scale and zero point are applied per group
//    in fp32; the per-group activation sums come from one more MMA with an all-ones A
//    operand, so the correction is exact for any zero point. The contraction over k is a
//    sum, so the kernel may pair any code with any activation as long as both operands
//    use the same order: each lane feeds the MMA with the 16 codes it loaded contiguously
//    (one 8-byte load per row and group) and permutes its 16 activations to match (PRMT).
//  * gemv_generic: any format (per-group widths), fp32 or bf16 x, with a residual; one warp
//    per row, fp32 CUDA-core math. Used for residual-carrying weights only: without a residual,
//    per-group widths and fp32 activations go to the tensor-core kernel of k_rrq.cu.
#include <cooperative_groups.h>

#include "cq_async.cuh"

namespace cq {
namespace {

// ------------------------------------------------------------------------------------
// tensor-core path
// ------------------------------------------------------------------------------------
// One CTA owns a 16-row tile and the whole K range; its warps split K and meet in shared
// memory at the end, so every output is written once (no atomics, no zero-fill, and the
// summation order is fixed). Weight and scale loads do not depend on earlier kernels, so
// they are issued before the programmatic-dependent-launch wait: back-to-back GEMVs in a
// stream overlap one kernel's weight streaming with the previous kernel's tail.
constexpr int kTileRows = 16;

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// the same with a zero accumulator in
__device__ __forceinline__ void mma_f16_16816_z(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// (w & mask) | magic in one LOP3
template <uint32_t kMask, uint32_t kMagic>
__device__ __forceinline__ uint32_t lop_or(uint32_t w) {
  uint32_t out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(w), "n"(kMask), "n"(kMagic));
  return out;
}

// nibbles i and i+4 of w (i = 0..3 after the shift) -> bf16 pair (128 + q_i, 128 + q_{i+4})
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) {
  uint32_t out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(w), "r"(0x000F000Fu), "r"(0x43004300u));
  return out;   // (w & 0x000F000F) | 0x43004300
}

// ---- the kernel -------------------------------------------------------------------------------
// Persistent CTAs of 16 warps, one per SM; CTA b owns the 16-row tiles b, b + G, b + 2G, ...
// Each tile is cut into chunks of 4 groups (16 rows x 128 bytes), and the CTA's chunks, tile
// after tile, are dealt to its warps round-robin, so every warp gets the same share (+-1)
// whatever the shape, and at any moment the CTA's loads cover a few KiB of each of 16 rows:
// long DRAM runs with few rows open. Every warp runs its own ring of kStages chunk buffers,
// filled by one TMA box per chunk (lane 0) plus per-lane cp.async copies of the chunk's scales
// and zero points; the same warp consumes them, so a buffer is refilled right after the warp
// has read it, without any cross-warp handshake. When a warp leaves a tile it stores its
// partial sums; the last of the tile's warps to arrive adds the partials in warp order and
// writes y (no atomics on y, no zero-fill, a fixed summation order, and no warp ever waits for
// another to finish a tile unless four tiles apart).
//
// Per group, sum_k W x = s * (sum_k (128 + q) x - (128 + z) sum_k x). The operand 128 + q is
// the bf16 bit pattern 0x4300 | q, made from a nibble pair with one LOP3; the activations are
// bf16 already, so the tensor-core products are exact and accumulate in fp32 (mma.sync
// m16n8k16). The correction enters the same accumulator through one more MMA: its A operand
// holds -(128 + z) (bit pattern 0xC300 | z, exact for z <= 127) and its B operand the group sum
// of x split into three bf16 parts (hi + mid + lo = the fp32 sum exactly), so the per-group
// result s * (...) needs only the scale multiply. When the activations are too large to
// stage, lanes read them from L1 and the group sums come from an MMA with an all-ones A.
// The contraction over k is a sum, so codes and activations may be paired in any order that
// both operands share: each lane feeds the 16 codes of one 8-byte word run and the staged
// activations are stored permuted to match.
constexpr int kWarps = 16;
constexpr int kGemvThreads = 32 * kWarps;
constexpr int kCG = 8;                                    // groups per chunk (two TMA boxes)
constexpr int kStages = 2;                                // chunk buffers per warp
constexpr int kBoxBytes = kTileRows * 4 * 32;             // one box: 16 rows x 4 groups
constexpr int kChunkBytes = 2 * kBoxBytes;
constexpr int kMetaBytes = 384;                           // [16][8] fp16 scales, then [16][8] zeros
constexpr int kRedSlots = 2;                              // tiles in reduction at once
constexpr int kRedFloats = kWarps * kTileRows * 8;        // one slot: every warp's 16 x 8 partials
// shared memory: [code rings | meta rings | barriers | reduction slots | counters | group sums |
//                 staged x]
constexpr int kOffMeta = kWarps * kStages * kChunkBytes;
constexpr int kOffBars = kOffMeta + kWarps * kStages * kMetaBytes;
constexpr int kOffRed = kOffBars + kWarps * kStages * 8;
constexpr int kOffCnt = kOffRed + kRedSlots * kRedFloats * 4;
constexpr int kOffSums = kOffCnt + 64;
constexpr int kSmemCap = 227 * 1024;
static_assert(kOffSums % 16 == 0 && kOffRed % 16 == 0, "shared-memory carve-up must keep 16-byte alignment");

// staged activations: m rows of K bf16 in fragment order, row pitch padded by 16 bytes so the
// rows a warp reads fall in different banks. Before them: per group the power-of-two factors
// of the 8 batch columns [KG][8] f32, then the group sums [m][KG] as three words (six fp16)
__host__ __device__ constexpr int64_t xstage_pitch(int64_t K) { return K * 2 + 16; }
__host__ __device__ constexpr int64_t sums_bytes(int m, int64_t K) {
  return (K / 64) * 32 + (((K / 64) * m * 12 + 15) & ~int64_t(15));
}
__host__ __device__ constexpr int64_t gemv_smem(int m, int64_t K, bool xs) {
  return 1024 + kOffSums + sums_bytes(m, K) + (xs ? m * xstage_pitch(K) : 0);
}

// 16 consecutive bf16 activations -> the 8 B-fragment registers in code-feeding order:
// pairs (0,4) (1,5) (2,6) (3,7) (8,12) (9,13) (10,14) (11,15)
__device__ __forceinline__ void permute16(const uint4 &lo, const uint4 &hi, uint32_t b[8]) {
  b[0] = __byte_perm(lo.x, lo.z, 0x5410); b[1] = __byte_perm(lo.x, lo.z, 0x7632);
  b[2] = __byte_perm(lo.y, lo.w, 0x5410); b[3] = __byte_perm(lo.y, lo.w, 0x7632);
  b[4] = __byte_perm(hi.x, hi.z, 0x5410); b[5] = __byte_perm(hi.x, hi.z, 0x7632);
  b[6] = __byte_perm(hi.y, hi.w, 0x5410); b[7] = __byte_perm(hi.y, hi.w, 0x7632);
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __low2float(*reinterpret_cast<const __half2 *>(&w)); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __high2float(*reinterpret_cast<const __half2 *>(&w)); }
__device__ __forceinline__ uint32_t word4(const uint4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// a warp's place in the CTA's chunk stream: local tile index, chunk within the tile
struct Cursor {
  int lt, c;
};
__device__ __forceinline__ void advance(Cursor &cu, int n_chunks) {
  cu.c += kWarps;
  while (cu.c >= n_chunks) {
    cu.c -= n_chunks;
    ++cu.lt;
  }
}

// Matrices that share the activations (q, k and v of a decoder layer; gate and up) run as
// one launch: their 16-row tiles are numbered one after the other (segment s owns the tiles
// tile0[s] .. tile0[s+1]-1) and every CTA deals with the concatenated sequence.
constexpr int kMaxSegs = 4;
struct GemvSegs {
  CUtensorMap tm[kMaxSegs];                 // the code plane of each matrix
  const uint16_t *scale[kMaxSegs];
  const uint8_t *zero[kMaxSegs];
  float *y[kMaxSegs];
  int64_t rows[kMaxSegs];
  int64_t tile0[kMaxSegs + 1];              // tile0[count] = all tiles; unused entries = INT64_MAX
};

__device__ __forceinline__ int seg_of(const GemvSegs &sg, int64_t tile) {
  return (tile >= sg.tile0[1]) + (tile >= sg.tile0[2]) + (tile >= sg.tile0[3]);
}
__device__ __forceinline__ const CUtensorMap *seg_map(const GemvSegs &sg, int s) {
  return s == 0 ? &sg.tm[0] : s == 1 ? &sg.tm[1] : s == 2 ? &sg.tm[2] : &sg.tm[3];
}
template <typename T, int kN>
__device__ __forceinline__ T seg_pick(const T (&a)[kN], int s) {
  return s == 0 ? a[0] : s == 1 ? a[1] : s == 2 ? a[2] : a[3];
}

template <bool FULL, bool XS>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv4_kernel(const __grid_constant__ GemvSegs segs, const __nv_bfloat16 *__restrict__ x, int m, int64_t K) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  pdl_launch_dependents();
  const int KG = static_cast<int>(K >> 6);
  const int n_chunks = (KG + kCG - 1) / kCG;
  const int64_t n_tiles = segs.tile0[kMaxSegs];
  const int n_local = static_cast<int>((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  // MMA row gid <-> tile row rho, MMA row gid + 8 <-> tile row rho + 8: with this order the
  // 8-byte code reads of a half-warp hit all 32 banks of the 128-byte swizzled box
  const int rho = 2 * (gid & 3) + (gid >> 2);
  uint8_t *ring = smem + warp * kStages * kChunkBytes;
  uint8_t *meta = smem + kOffMeta + warp * kStages * kMetaBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars) + warp * kStages;
  float *red = reinterpret_cast<float *>(smem + kOffRed);
  uint32_t *cnt = reinterpret_cast<uint32_t *>(smem + kOffCnt);            // [kRedSlots] arrivals
  volatile uint32_t *uses = reinterpret_cast<volatile uint32_t *>(smem + kOffCnt + 16);   // reductions done
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + kOffCnt + 32);
  float *fsc = reinterpret_cast<float *>(smem + kOffSums);                  // [KG][8] column factors
  uint32_t *sums = reinterpret_cast<uint32_t *>(smem + kOffSums + KG * 32); // [m][KG][3]
  uint8_t *xst = smem + kOffSums + sums_bytes(m, K);
  const int64_t xpitch = xstage_pitch(K);
  const int total = n_local * n_chunks;                                      // chunks of this CTA

  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(bars + i, FULL ? 33u : 1u);
    mbar_init_fence();
  }
  // the reduction slots need zeros only where a warp never writes: tiles with fewer chunks than warps
  if (n_chunks < kWarps)
    for (int i = threadIdx.x; i < kRedSlots * kRedFloats; i += kGemvThreads) red[i] = 0.0f;
  if (threadIdx.x < kRedSlots) { cnt[threadIdx.x] = 0u; uses[threadIdx.x] = 0u; }
  if (threadIdx.x == 0) *abort_flag = 0u;
  __syncthreads();

  // ---- producer side: the warp's own ring ----
  // lane l copies the scales (8 bytes) and zero points (4 bytes) of groups 4h..4h+3 of the
  // chunk for tile row l & 15, h = l >> 4; groups past the row's end are zero-filled
  const int prow = lane & 15, phalf = lane >> 4;
  Cursor prod = {0, warp};       // chunk number `warp` of the stream may lie beyond the first tile
  while (prod.c >= n_chunks) { prod.c -= n_chunks; ++prod.lt; }
  int prod_lt = -1, prod_y = 0;
  const uint16_t *ps = segs.scale[0];
  const uint8_t *pz = segs.zero[0];
  const CUtensorMap *ptm = &segs.tm[0];
  auto issue = [&](int slot) {
    if (prod.lt != prod_lt) {
      prod_lt = prod.lt;
      const int64_t tile = blockIdx.x + static_cast<int64_t>(prod_lt) * gridDim.x;
      const int sg = seg_of(segs, tile);
      const int64_t lrow0 = (tile - seg_pick(segs.tile0, sg)) * kTileRows, nrows = seg_pick(segs.rows, sg);
      int64_t row = lrow0 + prow;
      row = row < nrows ? row : nrows - 1;
      ps = seg_pick(segs.scale, sg) + row * KG + phalf * 4;
      pz = seg_pick(segs.zero, sg) + row * KG + phalf * 4;
      ptm = seg_map(segs, sg);
      prod_y = static_cast<int>(lrow0);
    }
    uint64_t *bar = bars + slot;
    const int g0 = prod.c * kCG;
    const bool second = g0 + 4 < KG;
    if (FULL) {
      const bool valid = g0 + phalf * 4 < KG;
      uint8_t *ms = meta + slot * kMetaBytes;
      cp_async_8z(ms + prow * 16 + phalf * 8, valid ? ps + g0 : ps, valid ? 8u : 0u);
      cp_async_4z(ms + 256 + prow * 8 + phalf * 4, valid ? pz + g0 : pz, valid ? 4u : 0u);
      cp_async_arrive_noinc(bar);
    }
    if (lane == 0) {
      uint8_t *dst = ring + slot * kChunkBytes;
      mbar_arrive_expect_tx(bar, second ? kChunkBytes : kBoxBytes);
      tma_load_2d(dst, ptm, prod.c * 256, prod_y, bar);
      if (second) tma_load_2d(dst + kBoxBytes, ptm, prod.c * 256 + 128, prod_y, bar);
    }
  };
  int n_issued = 0;
  for (int e = warp; n_issued < kStages && e < total; e += kWarps, ++n_issued) {
    issue(n_issued);
    advance(prod, n_chunks);
  }

  pdl_wait();   // x may be the output of the previous kernel in the stream; y is written below
  // Staged activations (XS): per group and batch row, x' = x * 2^-e in fp16 with e the power
  // of two that puts the group's max |x| in [256, 512): every bf16 value down to that max
  // times 2^-18 converts exactly, the fp16 group sums below stay finite, and the factor 2^e
  // (kept per group and column) multiplies the group's result. Thread t owns the 16-element
  // blocks t, t + 512, ... of the flattened [m][K/16]; the four lanes of a group agree on e
  // through two shuffles, so one pass and one barrier stage everything.
  if (XS) {
    const int bpr = KG * 4;                 // 16-element blocks per activation row
    const int nblk = m * bpr;
    for (int i = threadIdx.x; i < KG * 8; i += kGemvThreads)
      if ((i & 7) >= m) fsc[i] = 0.0f;      // MMA columns past the batch are never stored
    for (int b0 = 0; b0 < nblk; b0 += kGemvThreads * 4) {
      uint4 v[4][2];
      int nn[4], kk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u * kGemvThreads + threadIdx.x;
        int n = 0;
#pragma unroll
        for (int i = 1; i < 8; ++i) n += b >= i * bpr ? 1 : 0;      // m <= 8: no division
        nn[u] = n;
        kk[u] = b - n * bpr;
        v[u][0] = v[u][1] = make_uint4(0, 0, 0, 0);
        if (b < nblk) {
          const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(n) * K + kk[u] * 16);
          v[u][0] = __ldg(src);
          v[u][1] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u * kGemvThreads + threadIdx.x;
        const uint32_t w[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                               v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
        float se = 0.0f, so = 0.0f, amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
          se += lo;
          so += hi;
          amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        float sx = se + so;
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        so += __shfl_xor_sync(0xffffffffu, so, 1);
        so += __shfl_xor_sync(0xffffffffu, so, 2);
        int e = 0;
        if (amax > 0.0f && amax <= 3.0e38f) {
          e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
          e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float in_scale = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
        const float in_scale16 = in_scale * 0.0625f;
        if (b < nblk && CQ_CHECK(nn[u] < m && kk[u] < bpr &&
                                     (xst - smem) + nn[u] * xpitch + kk[u] * 32 + 32 <= dynamic_smem_bytes(), 0x0501u)) {
          uint32_t f[8];
          permute16(v[u][0], v[u][1], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            // words 1, 3, 5, 7 feed codes that carry a factor 16 (see below)
            const float sc = (i & 1) ? in_scale16 : in_scale;
            const __half2 h2 = __floats2half2_rn(__uint_as_float(f[i] << 16) * sc,
                                                 __uint_as_float(f[i] & 0xFFFF0000u) * sc);
            f[i] = *reinterpret_cast<const uint32_t *>(&h2);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(xst + nn[u] * xpitch + kk[u] * 32);
          dst[0] = make_uint4(f[0], f[1], f[2], f[3]);
          dst[1] = make_uint4(f[4], f[5], f[6], f[7]);
          if ((threadIdx.x & 3) == 0) {
            // exact three-way fp16 splits of the scaled sums: hi + mid + lo == value
            const int g = kk[u] >> 2;
            uint16_t hx[3], ho[3];
            float rx = sx * in_scale, ro = so * in_scale;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
              const __half a = __float2half_rn(rx), c = __float2half_rn(ro);
              hx[i] = __half_as_ushort(a);
              ho[i] = __half_as_ushort(c);
              rx -= __half2float(a);
              ro -= __half2float(c);
            }
            uint32_t *sw = sums + (nn[u] * KG + g) * 3;
            sw[0] = hx[0] | (static_cast<uint32_t>(hx[1]) << 16);
            sw[1] = hx[2] | (static_cast<uint32_t>(ho[0]) << 16);
            sw[2] = ho[1] | (static_cast<uint32_t>(ho[2]) << 16);
            fsc[g * 8 + nn[u]] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
          }
        }
      }
    }
  }
  __syncthreads();

  // per-lane constants. Lanes whose B column n = gid is past the batch read row 0's data: the
  // MMA columns they feed are never stored, so no predicates or zero buffers are needed.
  uint32_t off[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) off[j] = rho * 128 + ((((2 * j) + (tig >> 1)) ^ rho) << 4) + (tig & 1) * 8;
  const bool has_x = gid < m;
  const int xrow_s = has_x ? gid : 0;
  const uint8_t *xs_base = xst + xrow_s * xpitch + tig * 32;
  const uint32_t *sum_base = sums + xrow_s * KG * 3 + (tig < 2 ? tig : 2);
  const float *fsc_lane = fsc + 2 * tig;
  // correction operand per lane (k = 2 tig, 2 tig + 1), fp16 halves: tig 0 (Z, Z), tig 1
  // (Z, 960), tig 2 (960, 960), tig 3 (0, 0), Z = -(1024 + z) = 0xE400 | z (byte j of the
  // zero word); constant bytes 4..7 = E4 80 63 00
  const uint32_t csel_base = tig == 0 ? 0x4040u : (tig == 1 ? 0x6540u : (tig == 2 ? 0x6565u : 0x7777u));
  const uint32_t csel_mul = tig == 0 ? 0x0101u : (tig == 1 ? 0x0001u : 0u);
  const __nv_bfloat16 *xrow = x + static_cast<int64_t>(has_x ? gid : 0) * K + tig * 16;
  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};   // bf16 1.0
  const int arrivals = n_chunks < kWarps ? n_chunks : kWarps;

  // store this warp's partials of local tile lt; the last arrival reduces and writes y
  auto flush = [&](int lt, const float2 acc01, const float2 acc23) {
    const float acc[4] = {acc01.x, acc01.y, acc23.x, acc23.y};
    const int slot = lt % kRedSlots;
    const uint32_t use = static_cast<uint32_t>(lt / kRedSlots);
    // the slot's previous tile must be reduced (and its partials zeroed) first; lane 0 polls,
    // the warp follows its verdict
    uint32_t go = 1u;
    if (lane == 0) {
      for (uint32_t i = 0; uses[slot] != use; ++i) {
        if (*abort_flag) { go = 0u; break; }
        if (i > kSuspendLimit * 16u) { *abort_flag = 1u; go = 0u; break; }
        __nanosleep(32);
      }
      __threadfence_block();
    }
    if (!__shfl_sync(0xffffffffu, go, 0)) return;
    // partials of the m live columns only, column-major: [col][16 rows]
    float *rs = red + slot * kRedFloats;
    float *rw = rs + warp * (kTileRows * 8);
    if (2 * tig < m) {
      rw[(2 * tig) * 16 + rho] = acc[0];
      rw[(2 * tig) * 16 + rho + 8] = acc[2];
    }
    if (2 * tig + 1 < m) {
      rw[(2 * tig + 1) * 16 + rho] = acc[1];
      rw[(2 * tig + 1) * 16 + rho + 8] = acc[3];
    }
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) {
      __threadfence_block();
      old = atomicAdd(cnt + slot, 1u);
      __threadfence_block();
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    __syncwarp();
    if (old + 1 != static_cast<uint32_t>(arrivals)) return;
    // last arrival: lane l sums outputs l, l + 32, ... (col * 16 + row) over the warps, in warp order
    const int64_t tile = blockIdx.x + static_cast<int64_t>(lt) * gridDim.x;
    const int sg = seg_of(segs, tile);
    const int64_t lrow0 = (tile - seg_pick(segs.tile0, sg)) * kTileRows, N = seg_pick(segs.rows, sg);
    float *y = seg_pick(segs.y, sg);
    const bool bad = *abort_flag != 0u;
    const bool tile_ok = CQ_CHECK(sg >= 0 && sg < kMaxSegs && lrow0 >= 0 && lrow0 < N, 0x0502u);
    for (int idx = lane; idx < 16 * m; idx += 32) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        v += rs[w * (kTileRows * 8) + idx];
        rs[w * (kTileRows * 8) + idx] = 0.0f;
      }
      const int row = idx & 15, col = idx >> 4;
      const int64_t r = lrow0 + row;
      if (r < N && tile_ok) y[static_cast<int64_t>(col) * N + r] = bad ? __int_as_float(0x7fc00000) : v;
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) {
      cnt[slot] = 0u;
      __threadfence_block();
      uses[slot] = use + 1u;
    }
  };

  // ---- consumer side ----
  Cursor cons = {0, warp};
  while (cons.c >= n_chunks) { cons.c -= n_chunks; ++cons.lt; }
  float2 acc01 = make_float2(0.0f, 0.0f), acc23 = acc01;   // (row rho | rho + 8) x (col 2 tig, 2 tig + 1)
  int lt_cur = cons.lt;
  int slot = 0;
  uint32_t phase = 0;
  bool ok = true;
  int n_done = 0;
  for (int e = warp; e < total; e += kWarps) {
    if (cons.lt != lt_cur) {
      flush(lt_cur, acc01, acc23);
      acc01 = acc23 = make_float2(0.0f, 0.0f);
      lt_cur = cons.lt;
    }
    // every lane waits (the wait makes the TMA and cp.async data visible to it); the warp goes
    // on only if all of them saw the chunk arrive
    const bool got = mbar_wait_suspend(bars + slot, phase, abort_flag);
    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
    const uint8_t *box = ring + slot * kChunkBytes;
    const int g0 = cons.c * kCG;
    const int ng = KG - g0 < kCG ? KG - g0 : kCG;
    (void)CQ_CHECK(ng > 0, 0x0503u);
    const uint8_t *xb = xs_base + g0 * 128;
    const uint32_t *sb = sum_base + g0 * 3;
    const float *fb = fsc_lane + g0 * 8;
    uint4 sv0 = make_uint4(0, 0, 0, 0), sv1 = sv0;
    uint2 zv0 = make_uint2(0, 0), zv1 = zv0;
    int64_t r0 = 0, r1 = 0;
    const uint16_t *scale = segs.scale[0];
    const uint8_t *zero = segs.zero[0];
    if (FULL) {
      const uint8_t *ms = meta + slot * kMetaBytes;
      sv0 = *reinterpret_cast<const uint4 *>(ms + rho * 16);
      sv1 = *reinterpret_cast<const uint4 *>(ms + (rho + 8) * 16);
      zv0 = *reinterpret_cast<const uint2 *>(ms + 256 + rho * 8);
      zv1 = *reinterpret_cast<const uint2 *>(ms + 256 + (rho + 8) * 8);
    } else {
      const int64_t tile = blockIdx.x + static_cast<int64_t>(cons.lt) * gridDim.x;
      const int sg = seg_of(segs, tile);
      const int64_t N = seg_pick(segs.rows, sg);
      scale = seg_pick(segs.scale, sg);
      zero = seg_pick(segs.zero, sg);
      r0 = (tile - seg_pick(segs.tile0, sg)) * kTileRows + rho;
      r1 = r0 + 8;
      r0 = r0 < N ? r0 : N - 1;
      r1 = r1 < N ? r1 : N - 1;
    }
#pragma unroll
    for (int j = 0; j < kCG; ++j) {
      if (j < 4 || ng > 4) {
        if (!FULL && j >= ng) continue;
        float s0, s1;
        uint32_t zw0, zw1;
        if (FULL) {
          const uint32_t h0 = word4(sv0, j >> 1), h1 = word4(sv1, j >> 1);
          s0 = (j & 1) ? half_hi(h0) : half_lo(h0);
          s1 = (j & 1) ? half_hi(h1) : half_lo(h1);
          zw0 = j < 4 ? zv0.x : zv0.y;
          zw1 = j < 4 ? zv1.x : zv1.y;
        } else {
          const int g = g0 + j;
          s0 = f16_bits_to_f32(__ldg(scale + r0 * KG + g));
          s1 = f16_bits_to_f32(__ldg(scale + r1 * KG + g));
          zw0 = static_cast<uint32_t>(__ldg(zero + r0 * KG + g)) << (8 * (j & 3));
          zw1 = static_cast<uint32_t>(__ldg(zero + r1 * KG + g)) << (8 * (j & 3));
        }
        const uint8_t *cw = box + off[j & 3] + (j >> 2) * kBoxBytes;
        const uint2 w0 = *reinterpret_cast<const uint2 *>(cw);
        const uint2 w1 = *reinterpret_cast<const uint2 *>(cw + 1024);
        float p[4];
        if (XS) {
          // fp16 operands: for nibble pairs at bits 0-3 / 16-19 the pattern 0x6400 | q is
          // 1024 + q, at bits 4-7 / 20-23 it is 1024 + 16 q (the staged x carries 1/16 there)
          const uint4 *xp = reinterpret_cast<const uint4 *>(xb + j * 128);
          const uint4 xl = xp[0], xh = xp[1];
          const uint32_t bx[8] = {xl.x, xl.y, xl.z, xl.w, xh.x, xh.y, xh.z, xh.w};
          // correction: -(1024 + z) * sum x + 960 * sum of odd-position x, from the split sums
          const uint32_t bc = sb[j * 3];
          const uint32_t sel = csel_base + csel_mul * (j & 3);
          const uint32_t c0 = __byte_perm(zw0, 0x006380E4u, sel), c1 = __byte_perm(zw1, 0x006380E4u, sel);
          const uint32_t ac[4] = {c0, c1, c0, c1};
          mma_f16_16816_z(p, ac, bc, 0u);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t u0 = h ? w0.y : w0.x, u1 = h ? w1.y : w1.x;
            const uint32_t t0 = u0 >> 8, t1 = u1 >> 8;
            const uint32_t A0[4] = {lop_or<0x000F000Fu, 0x64006400u>(u0), lop_or<0x000F000Fu, 0x64006400u>(u1),
                                    lop_or<0x00F000F0u, 0x64006400u>(u0), lop_or<0x00F000F0u, 0x64006400u>(u1)};
            mma_f16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
            const uint32_t A1[4] = {lop_or<0x000F000Fu, 0x64006400u>(t0), lop_or<0x000F000Fu, 0x64006400u>(t1),
                                    lop_or<0x00F000F0u, 0x64006400u>(t0), lop_or<0x00F000F0u, 0x64006400u>(t1)};
            mma_f16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
          }
        } else {
          uint32_t bx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) bx[i] = 0u;
          if (has_x) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(xrow + (g0 + j) * 64);
            permute16(__ldg(xp), __ldg(xp + 1), bx);
          }
          float q[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          p[0] = p[1] = p[2] = p[3] = 0.0f;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t u0 = h ? w0.y : w0.x, u1 = h ? w1.y : w1.x;
            const uint32_t A0[4] = {nib_pair(u0), nib_pair(u1), nib_pair(u0 >> 4), nib_pair(u1 >> 4)};
            mma_bf16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
            mma_bf16_16816(q, ones, bx[4 * h + 0], bx[4 * h + 1]);
            const uint32_t A1[4] = {nib_pair(u0 >> 8), nib_pair(u1 >> 8), nib_pair(u0 >> 12), nib_pair(u1 >> 12)};
            mma_bf16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
            mma_bf16_16816(q, ones, bx[4 * h + 2], bx[4 * h + 3]);
          }
          const float zc0 = 128.0f + static_cast<float>(__byte_perm(zw0, 0u, 0x4440u + (j & 3)));
          const float zc1 = 128.0f + static_cast<float>(__byte_perm(zw1, 0u, 0x4440u + (j & 3)));
          p[0] = fmaf(-zc0, q[0], p[0]);
          p[1] = fmaf(-zc0, q[1], p[1]);
          p[2] = fmaf(-zc1, q[2], p[2]);
          p[3] = fmaf(-zc1, q[3], p[3]);
        }
        if (XS) {
          // scale times the activation factors of columns 2 tig, 2 tig + 1 of this group
          const float2 fc = *reinterpret_cast<const float2 *>(fb + j * 8);
          const float2 a01 = __fmul2_rn(make_float2(s0, s0), fc), a23 = __fmul2_rn(make_float2(s1, s1), fc);
          acc01 = __ffma2_rn(a01, make_float2(p[0], p[1]), acc01);
          acc23 = __ffma2_rn(a23, make_float2(p[2], p[3]), acc23);
        } else {
          acc01.x = fmaf(s0, p[0], acc01.x);
          acc01.y = fmaf(s0, p[1], acc01.y);
          acc23.x = fmaf(s1, p[2], acc23.x);
          acc23.y = fmaf(s1, p[3], acc23.y);
        }
      }
    }
    // every lane's reads of this slot have fed the MMAs above; refill it (the proxy fence orders
    // those generic reads before the TMA write into the slot)
    fence_proxy_async_smem();
    __syncwarp();
    ++n_done;
    if (e + kStages * kWarps < total) {
      issue(slot);
      advance(prod, n_chunks);
      ++n_issued;
    }
    advance(cons, n_chunks);
    if (++slot == kStages) { slot = 0; phase ^= 1u; }
  }
  if (ok && total > warp) flush(lt_cur, acc01, acc23);
  // a warp that gave up lets the copies it issued land before the CTA exits
  for (; n_done < n_issued; ++n_done) {
    mbar_wait_suspend(bars + slot, phase, abort_flag, false);
    if (++slot == kStages) { slot = 0; phase ^= 1u; }
  }
}

template <bool FULL, bool XS>
cq_status launch_gemv4(const GemvSegs &segs, const void *x, int m, int64_t K, cudaStream_t s) {
  const int smem = static_cast<int>(gemv_smem(m, K, XS));
  cq_status st = cuda_check(cudaFuncSetAttribute(gemv4_kernel<FULL, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem), "cq_dequant_gemv: shared memory attribute");
  if (st != CQ_OK) return st;
  const int64_t tiles = segs.tile0[kMaxSegs];
  const int64_t grid = tiles < sm_count() ? tiles : sm_count();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, gemv4_kernel<FULL, XS>, segs, static_cast<const __nv_bfloat16 *>(x), m, K),
                    "cq_dequant_gemv");
}

// the tensor-core path for up to kMaxSegs fixed-4 matrices with the same cols and bf16 x
cq_status launch_gemv4_segs(const cq_qweight *const *qws, int count, const void *x, int m, float *const *ys,
                            cudaStream_t s) {
  const int64_t K = qws[0]->cols, KG = K >> 6;
  GemvSegs segs;
  memset(&segs, 0, sizeof(segs));
  bool full = KG % 4 == 0;
  int64_t t = 0;
  for (int i = 0; i < kMaxSegs; ++i) {
    if (i < count) {
      const cq_qweight &qw = *qws[i];
      cq_status st = code_tensor_map(&segs.tm[i], qw.plane[2], qw.rows, qw.cols, kTileRows, "cq_dequant_gemv");
      if (st != CQ_OK) return st;
      segs.scale[i] = qw.scale;
      segs.zero[i] = qw.zero;
      segs.y[i] = ys[i];
      segs.rows[i] = qw.rows;
      segs.tile0[i] = t;
      t += (qw.rows + kTileRows - 1) / kTileRows;
      // the per-chunk scale (8-byte) and zero (4-byte) copies need aligned rows of whole 4-group runs
      full = full && aligned8(qw.scale) && (reinterpret_cast<uintptr_t>(qw.zero) & 3u) == 0;
    } else {
      segs.tile0[i] = INT64_MAX;
    }
  }
  segs.tile0[kMaxSegs] = t;
  if (count < kMaxSegs) segs.tile0[count] = t;
  // activations are staged once per CTA in shared memory when they fit
  const bool xs = gemv_smem(m, K, true) <= kSmemCap;
  if (gemv_smem(m, K, false) > kSmemCap) return fail(CQ_ERR_SHAPE, "cq_dequant_gemv: cols too large");
  if (full) return xs ? launch_gemv4<true, true>(segs, x, m, K, s) : launch_gemv4<true, false>(segs, x, m, K, s);
  return xs ? launch_gemv4<false, true>(segs, x, m, K, s) : launch_gemv4<false, false>(segs, x, m, K, s);
}

// ------------------------------------------------------------------------------------
// fixed 4-bit codes with a bf16 residual: the CellFill served weights W = s (q - z) + r
// ------------------------------------------------------------------------------------
// [CF] the served weight carries the residual, so decode streams 0.5 B of codes and 2 B of
// residual per weight. A CTA of 8 warps owns one 16-row tile (or, when the tiles do not fill
// the SMs, half of its groups, in a two-CTA cluster); warp w takes the w-th eighth of the CTA's
// groups, so each warp streams contiguous runs of codes and residual of 16 rows.
// Per group, on tensor cores (mma.sync m16n8k16, fp32 accumulation, exact products):
//   codes:    sum_k (128 + q) x  with 128 + q = bf16 0x4300 | q, minus (128 + z) sum_k x (the group
//             sum of x from an MMA with an all-ones A), times s;
//   residual: sum_k r x straight into the row accumulator (bf16 r and x: exact products).
// Both operands pair k the same way: lane (gid, tig) holds k = 16 tig .. 16 tig + 15 of the
// group for rows gid and gid + 8 (one 8-byte code load and two 16-byte residual loads per row),
// the codes in the nibble order (0,4) (1,5) (2,6) (3,7), the residual and x permuted to match.
// Each lane keeps the next group's loads in flight (two groups of loads per warp: ~80 B per
// lane); the first two groups' weight loads are issued before the wait for the previous kernel
// in the stream. The warps' partial sums meet in shared memory; y is written once per tile.
constexpr int kRWarps = 8;
constexpr int kRThreads = 32 * kRWarps;

struct RGroup {
  uint2 c0, c1;          // codes of rows gid, gid + 8 (16 nibbles each)
  uint4 r0l, r0h, r1l, r1h;   // residual of rows gid, gid + 8 (16 bf16 each)
  uint4 xl, xh;          // 16 bf16 activations of batch row gid (row 0 for gid >= m)
  uint32_t s0, s1, z0, z1;
};

// the weight side of a group (codes, residual, scale, zero point): independent of earlier kernels
__device__ __forceinline__ void rgroup_load_w(RGroup &b, const uint8_t *c0, const uint8_t *c1, const uint16_t *r0,
                                              const uint16_t *r1, const uint16_t *sc0, const uint16_t *sc1,
                                              const uint8_t *zp0, const uint8_t *zp1, int g) {
  b.c0 = __ldcs(reinterpret_cast<const uint2 *>(c0 + g * 32));
  b.c1 = __ldcs(reinterpret_cast<const uint2 *>(c1 + g * 32));
  const uint4 *p0 = reinterpret_cast<const uint4 *>(r0 + g * 64);
  const uint4 *p1 = reinterpret_cast<const uint4 *>(r1 + g * 64);
  b.r0l = __ldcs(p0);
  b.r0h = __ldcs(p0 + 1);
  b.r1l = __ldcs(p1);
  b.r1h = __ldcs(p1 + 1);
  b.s0 = __ldg(sc0 + g);
  b.s1 = __ldg(sc1 + g);
  b.z0 = __ldg(zp0 + g);
  b.z1 = __ldg(zp1 + g);
}
// the activation side: x may be the previous kernel's output
__device__ __forceinline__ void rgroup_load_x(RGroup &b, const __nv_bfloat16 *xr, int g) {
  const uint4 *xp = reinterpret_cast<const uint4 *>(xr + g * 64);
  b.xl = __ldg(xp);
  b.xh = __ldg(xp + 1);
}

__device__ __forceinline__ void rgroup_mma(const RGroup &b, float acc[4]) {
  uint32_t bx[8], ra[8], rb[8];
  permute16(b.xl, b.xh, bx);
  permute16(b.r0l, b.r0h, ra);
  permute16(b.r1l, b.r1h, rb);
  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};   // bf16 1.0
  float p[4] = {0.0f, 0.0f, 0.0f, 0.0f}, q[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t u0 = h ? b.c0.y : b.c0.x, u1 = h ? b.c1.y : b.c1.x;
    const uint32_t A0[4] = {nib_pair(u0), nib_pair(u1), nib_pair(u0 >> 4), nib_pair(u1 >> 4)};
    mma_bf16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
    mma_bf16_16816(q, ones, bx[4 * h + 0], bx[4 * h + 1]);
    const uint32_t A1[4] = {nib_pair(u0 >> 8), nib_pair(u1 >> 8), nib_pair(u0 >> 12), nib_pair(u1 >> 12)};
    mma_bf16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
    mma_bf16_16816(q, ones, bx[4 * h + 2], bx[4 * h + 3]);
  }
  const float s0 = f16_bits_to_f32(static_cast<uint16_t>(b.s0)), s1 = f16_bits_to_f32(static_cast<uint16_t>(b.s1));
  const float zc0 = 128.0f + static_cast<float>(b.z0), zc1 = 128.0f + static_cast<float>(b.z1);
  acc[0] = fmaf(s0, fmaf(-zc0, q[0], p[0]), acc[0]);
  acc[1] = fmaf(s0, fmaf(-zc0, q[1], p[1]), acc[1]);
  acc[2] = fmaf(s1, fmaf(-zc1, q[2], p[2]), acc[2]);
  acc[3] = fmaf(s1, fmaf(-zc1, q[3], p[3]), acc[3]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t A0[4] = {ra[4 * h + 0], rb[4 * h + 0], ra[4 * h + 1], rb[4 * h + 1]};
    mma_bf16_16816(acc, A0, bx[4 * h + 0], bx[4 * h + 1]);
    const uint32_t A1[4] = {ra[4 * h + 2], rb[4 * h + 2], ra[4 * h + 3], rb[4 * h + 3]};
    mma_bf16_16816(acc, A1, bx[4 * h + 2], bx[4 * h + 3]);
  }
}

// several matrices that read the same x in one launch: their 16-row tiles are numbered one after
// the other (segment s owns tiles tile0[s] .. tile0[s+1]-1)
struct RSegs {
  const uint8_t *plane[kMaxSegs];
  const uint16_t *scale[kMaxSegs];
  const uint8_t *zero[kMaxSegs];
  const uint16_t *res[kMaxSegs];
  float *y[kMaxSegs];
  int64_t rows[kMaxSegs];
  int64_t tile0[kMaxSegs + 1];              // tile0[count] = all tiles; unused entries = INT64_MAX
};

// SPLIT = 2 (matrices with no more tiles than SMs): a thread-block cluster of two CTAs owns a
// tile, each CTA taking half of the row's groups, so twice as many SMs stream the matrix and each
// CTA's run is half as long. The two CTAs' tile sums meet in the first CTA's hands through
// distributed shared memory between two cluster barriers (hardware barriers of co-scheduled
// CTAs, nothing polled), in a fixed order, so y stays deterministic.
template <int SPLIT>
__global__ void __launch_bounds__(kRThreads, 2)
gemv4r_kernel(const __grid_constant__ RSegs sg, const __nv_bfloat16 *__restrict__ x, int m, int64_t K) {
  __shared__ float red[kRWarps][kTileRows * 8];
  __shared__ float part[kTileRows * 8];          // SPLIT > 1: this CTA's tile sums
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int KG = static_cast<int>(K >> 6);
  const int rank = SPLIT > 1 ? static_cast<int>(cooperative_groups::this_cluster().block_rank()) : 0;
  const int64_t unit = blockIdx.x / SPLIT, n_units = gridDim.x / SPLIT;
  const int q0 = KG * rank / SPLIT, q1 = KG * (rank + 1) / SPLIT;     // this CTA's groups
  const int g0 = q0 + (q1 - q0) * warp / kRWarps, g1 = q0 + (q1 - q0) * (warp + 1) / kRWarps;
  const int64_t n_tiles = sg.tile0[kMaxSegs];
  for (int64_t tile = unit; tile < n_tiles; tile += n_units) {
    const int s = (tile >= sg.tile0[1]) + (tile >= sg.tile0[2]) + (tile >= sg.tile0[3]);
    const uint8_t *plane = seg_pick(sg.plane, s);
    const uint16_t *scale = seg_pick(sg.scale, s), *res = seg_pick(sg.res, s);
    const uint8_t *zero = seg_pick(sg.zero, s);
    const int64_t N = seg_pick(sg.rows, s), lrow0 = (tile - seg_pick(sg.tile0, s)) * kTileRows;
    (void)CQ_CHECK(s >= 0 && s < kMaxSegs && lrow0 >= 0 && lrow0 < N, 0x0504u);
    int64_t row0 = lrow0 + gid, row1 = row0 + 8;
    row0 = row0 < N ? row0 : N - 1;               // rows past the end: any valid row, never stored
    row1 = row1 < N ? row1 : N - 1;
    const uint8_t *c0 = plane + row0 * (K / 2) + tig * 8, *c1 = plane + row1 * (K / 2) + tig * 8;
    const uint16_t *r0 = res + row0 * K + tig * 16, *r1 = res + row1 * K + tig * 16;
    const uint16_t *sc0 = scale + row0 * KG, *sc1 = scale + row1 * KG;
    const uint8_t *zp0 = zero + row0 * KG, *zp1 = zero + row1 * KG;
    const __nv_bfloat16 *xr = x + static_cast<int64_t>(gid < m ? gid : 0) * K + tig * 16;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // the weights do not depend on earlier kernels, so the first two groups' weight loads are
    // issued before the wait for the previous kernel; x and y do depend on it
    RGroup a, b;
    if (g0 < g1) rgroup_load_w(a, c0, c1, r0, r1, sc0, sc1, zp0, zp1, g0);
    if (g0 + 1 < g1) rgroup_load_w(b, c0, c1, r0, r1, sc0, sc1, zp0, zp1, g0 + 1);
    if (tile == unit) pdl_wait();
    if (g0 < g1) rgroup_load_x(a, xr, g0);
    if (g0 + 1 < g1) rgroup_load_x(b, xr, g0 + 1);
    for (int g = g0; g < g1; g += 2) {
      rgroup_mma(a, acc);
      if (g + 2 < g1) {
        rgroup_load_w(a, c0, c1, r0, r1, sc0, sc1, zp0, zp1, g + 2);
        rgroup_load_x(a, xr, g + 2);
      }
      if (g + 1 >= g1) break;
      rgroup_mma(b, acc);
      if (g + 3 < g1) {
        rgroup_load_w(b, c0, c1, r0, r1, sc0, sc1, zp0, zp1, g + 3);
        rgroup_load_x(b, xr, g + 3);
      }
    }
    // partials of rows gid, gid + 8 and batch columns 2 tig, 2 tig + 1: [col][row]
    float *rw = red[warp];
    rw[(2 * tig) * 16 + gid] = acc[0];
    rw[(2 * tig + 1) * 16 + gid] = acc[1];
    rw[(2 * tig) * 16 + gid + 8] = acc[2];
    rw[(2 * tig + 1) * 16 + gid + 8] = acc[3];
    __syncthreads();
    float v = 0.0f;
    if (threadIdx.x < 16 * m) {
#pragma unroll
      for (int w = 0; w < kRWarps; ++w) v += red[w][threadIdx.x];
    }
    if (SPLIT > 1) {
      if (threadIdx.x < 16 * m) part[threadIdx.x] = v;
      cooperative_groups::this_cluster().sync();        // every CTA's sums are in place
      if (rank == 0 && threadIdx.x < 16 * m)
        for (int r = 1; r < SPLIT; ++r) v += cooperative_groups::this_cluster().map_shared_rank(part, r)[threadIdx.x];
      cooperative_groups::this_cluster().sync();        // read before any CTA rewrites its sums
    }
    if (rank == 0 && threadIdx.x < 16 * m) {
      const int row = threadIdx.x & 15, col = threadIdx.x >> 4;
      const int64_t rr = lrow0 + row;
      if (rr < N) seg_pick(sg.y, s)[static_cast<int64_t>(col) * N + rr] = v;
    }
    __syncthreads();
  }
}

// fixed 4-bit codes with a 16-byte aligned bf16 residual and bf16 x: the served-weight kernel
bool gemv_res_eligible(const cq_qweight &qw, cq_dtype xdt) {
  return qw.bits == nullptr && qw.residual != nullptr && qw.residual_dtype == CQ_BF16 && xdt == CQ_BF16 &&
         aligned16(qw.residual) && aligned8(qw.plane[2]) && qw.rows > 0 && qw.cols > 0;
}

// up to kMaxSegs served-weight matrices with the same cols in one launch
cq_status launch_gemv4r(const cq_qweight *const *qws, int count, const void *x, int m, float *const *ys,
                        cudaStream_t s) {
  RSegs sg;
  memset(&sg, 0, sizeof(sg));
  int64_t t = 0;
  for (int i = 0; i < kMaxSegs; ++i) {
    if (i < count) {
      const cq_qweight &qw = *qws[i];
      sg.plane[i] = static_cast<const uint8_t *>(qw.plane[2]);
      sg.scale[i] = qw.scale;
      sg.zero[i] = qw.zero;
      sg.res[i] = static_cast<const uint16_t *>(qw.residual);
      sg.y[i] = ys[i];
      sg.rows[i] = qw.rows;
      sg.tile0[i] = t;
      t += (qw.rows + kTileRows - 1) / kTileRows;
    } else {
      sg.tile0[i] = INT64_MAX;
    }
  }
  sg.tile0[kMaxSegs] = t;
  if (count < kMaxSegs) sg.tile0[count] = t;
  if (t <= sm_count()) {
    // a cluster of two CTAs per tile (see gemv4r_kernel), one tile per cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * t));
    cfg.blockDim = dim3(kRThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cuda_check(cudaLaunchKernelEx(&cfg, gemv4r_kernel<2>, sg, static_cast<const __nv_bfloat16 *>(x), m,
                                         qws[0]->cols),
                      "cq_dequant_gemv (residual, split)");
  }
  const int64_t cap = static_cast<int64_t>(sm_count()) * 2;
  const int64_t grid = t < cap ? t : cap;
  return cuda_check(launch_pdl(gemv4r_kernel<1>, dim3(static_cast<unsigned>(grid)), dim3(kRThreads), 0, s, sg,
                               static_cast<const __nv_bfloat16 *>(x), m, qws[0]->cols),
                    "cq_dequant_gemv (residual)");
}

// ------------------------------------------------------------------------------------
// generic fp32 path
// ------------------------------------------------------------------------------------
constexpr int kGenThreads = 256;

template <bool XBF16>
__device__ __forceinline__ float load_x(const void *x, int64_t i) {
  return XBF16 ? bf16_bits_to_f32(static_cast<const uint16_t *>(x)[i]) : static_cast<const float *>(x)[i];
}

template <bool XBF16, int RK, int M>
__global__ void __launch_bounds__(kGenThreads)
gemv_generic_kernel(const uint8_t *__restrict__ bits, const uint32_t *__restrict__ offset,
                    const uint8_t *__restrict__ p0, const uint8_t *__restrict__ p1,
                    const uint8_t *__restrict__ p2, const uint8_t *__restrict__ p3,
                    const uint16_t *__restrict__ scale, const uint8_t *__restrict__ zero,
                    const void *__restrict__ r, const void *__restrict__ x, int m, int64_t N,
                    int64_t K, float *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t KG = K >> 6;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kGenThreads / 32);
  for (int64_t n = blockIdx.x * static_cast<int64_t>(kGenThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    float acc[M];
#pragma unroll
    for (int i = 0; i < M; ++i) acc[i] = 0.0f;
    for (int64_t gk = lane; gk < KG; gk += 32) {
      const int64_t g = n * KG + gk;
      int b = 4;
      const uint8_t *src;
      if (bits) {
        b = bits[g];
        const uint8_t *pl = b == 1 ? p0 : b == 2 ? p1 : b == 4 ? p2 : p3;
        src = pl + offset[g];
      } else {
        src = p2 + g * 32;
      }
      if (!width_ok(b)) continue;
      if (bits && !CQ_CHECK(offset[g] % (8u * b) == 0u && offset[g] / (8u * b) <= g, 0x0505u)) continue;
      const float s = f16_bits_to_f32(scale[g]);
      const float z = static_cast<float>(zero[g]);
      for (int jb = 0; jb < 8; ++jb) {
        uint64_t word = 0;
        for (int t = 0; t < b; ++t) word |= static_cast<uint64_t>(src[jb * b + t]) << (8 * t);
        for (int j = 0; j < 8; ++j) {
          const int64_t k = gk * 64 + jb * 8 + j;
          const float q = static_cast<float>((word >> (j * b)) & ((1ull << b) - 1ull));
          float wv = s * (q - z);
          if (RK == 1) wv += static_cast<const float *>(r)[n * K + k];
          if (RK == 2) wv += bf16_bits_to_f32(static_cast<const uint16_t *>(r)[n * K + k]);
#pragma unroll
          for (int i = 0; i < M; ++i)
            if (i < m) acc[i] = fmaf(wv, load_x<XBF16>(x, i * K + k), acc[i]);
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

template <bool XBF16, int RK>
void launch_generic(const cq_qweight &qw, const void *x, int m, float *y, int blocks, cudaStream_t s) {
  gemv_generic_kernel<XBF16, RK, 8><<<blocks, kGenThreads, 0, s>>>(
      qw.bits, qw.offset, qw.plane[0], qw.plane[1], qw.plane[2], qw.plane[3], qw.scale, qw.zero,
      qw.residual, x, m, qw.rows, qw.cols, y);
}

}  // namespace

cq_status launch_gemv(const cq_qweight &qw, const void *x, cq_dtype xdt, int m, float *y, cudaStream_t s) {
  const int64_t N = qw.rows, K = qw.cols;
  if (N == 0) return CQ_OK;
  if (K == 0) return cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * m * N, s), "cq_dequant_gemv: zero y");
  const bool tc = qw.bits == nullptr && qw.residual == nullptr && xdt == CQ_BF16;
  if (tc) {
    const cq_qweight *one = &qw;
    return launch_gemv4_segs(&one, 1, x, m, &y, s);
  }
  // per-group widths, or fp32 activations, without a residual: the tensor-core kernel over a
  // list of one stage (k_rrq.cu)
  if (qw.residual == nullptr) {
    const cq_qweight *one = &qw;
    return launch_gemv_stages(&one, 1, x, xdt, m, y, s);
  }
  // the CellFill served weights: fixed 4-bit codes and a bf16 residual with bf16 x
  if (gemv_res_eligible(qw, xdt)) {
    const cq_qweight *one = &qw;
    return launch_gemv4r(&one, 1, x, m, &y, s);
  }
  const int64_t need = (N + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  const bool rf32 = qw.residual_dtype != CQ_BF16;
  if (xdt == CQ_BF16) {
    if (rf32) launch_generic<true, 1>(qw, x, m, y, blocks, s);
    else launch_generic<true, 2>(qw, x, m, y, blocks, s);
  } else {
    if (rf32) launch_generic<false, 1>(qw, x, m, y, blocks, s);
    else launch_generic<false, 2>(qw, x, m, y, blocks, s);
  }
  return launch_check("cq_dequant_gemv");
}

bool gemv_tc_eligible(const cq_qweight &qw, cq_dtype xdt) {
  return qw.bits == nullptr && qw.residual == nullptr && xdt == CQ_BF16 && qw.rows > 0 && qw.cols > 0;
}

cq_status launch_gemv_multi(const cq_qweight *const *qws, int count, const void *x, cq_dtype xdt, int m,
                            float *const *ys, cudaStream_t s) {
  // runs of up to kMaxSegs tensor-core-eligible matrices become one launch; anything else goes
  // through the single-matrix path
  // (the same for runs of matrices that carry a bf16 residual, on the served-weight kernel)
  int i = 0;
  while (i < count) {
    const bool tc = gemv_tc_eligible(*qws[i], xdt), res = gemv_res_eligible(*qws[i], xdt);
    if (!tc && !res) {
      cq_status st = launch_gemv(*qws[i], x, xdt, m, ys[i], s);
      if (st != CQ_OK) return st;
      ++i;
      continue;
    }
    int j = i + 1;
    while (j < count && j - i < kMaxSegs &&
           (tc ? gemv_tc_eligible(*qws[j], xdt) : gemv_res_eligible(*qws[j], xdt)))
      ++j;
    cq_status st = tc ? launch_gemv4_segs(qws + i, j - i, x, m, ys + i, s)
                      : launch_gemv4r(qws + i, j - i, x, m, ys + i, s);
    if (st != CQ_OK) return st;
    i = j;
  }
  return CQ_OK;
}

}  // namespace cq
