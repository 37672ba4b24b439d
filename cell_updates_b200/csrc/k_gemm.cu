// k_gemm.cu -- batched dequantize-and-multiply on the sm_100a tensor cores (tcgen05 + TMEM).
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: fused dequantize-and-multiply over packed
// low-bit weights. Here the batch is large enough (m >= 16) for a real dense contraction:
//     y[i, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) * x[i, k]
//
// Operands. Every weight is dequantized once, to fp16: A[n, k] = RN16(s * (q - z)). q - z is
// exact, and the exact product has at most 15 significant bits, so its one rounding is a
// relative error below 2^-11; |s| <= 4096 keeps |A| <= 61440 < 65504. The activations are
// copied to fp16 by a preparation kernel with one power of two per batch row,
// x16[i, k] = x[i, k] * 2^-e_i, chosen so that max_k |x16[i, k]| lies in [2^14, 2^15): a bf16
// value keeps all of its 8 significant bits, nothing overflows, and only values below 2^-28
// of the row's largest become fp16 subnormals. Products are exact in fp32 and the tensor
// cores accumulate a whole K range of a tile in fp32 in tensor memory; the epilogue writes
// y += acc * 2^e_i once per range. A group whose scale is above 4096 in magnitude (or not
// finite) or whose zero point is above 15 is left out of A (written as zeros) and added in
// fp32 by the epilogue warps, which are otherwise idle while a range accumulates.
//
// Structure (one CTA per SM, persistent; work = (128-row tile, step of four groups) items
// split evenly over the CTAs in row-major order, so a CTA covers a contiguous K range of one
// or a few tiles; a maximal run of one tile's steps in one CTA is a "segment"):
//   warps 2-9   dequantize: thread (row, part) loads 64 contiguous bytes of its row (two groups
//               of a step) plus their scales and zero points straight into registers, three
//               steps ahead, turns them into fp16 s * (q - z) and stores them to tensor memory
//               (its lane = its row). Codes never pass through shared memory: its bandwidth
//               (128 B per clock) goes to the activation tiles and the MMAs' operand reads.
//   warp 0      TMA producer: per step the fp16 activations (m rows x 64 per group, 128-byte
//               swizzled = the UMMA K-major layout)
//   warp 1      MMA issuer: per group four tcgen05.mma (M=128, N=NT, K=16), A from tensor
//               memory and B from shared memory, into the segment's accumulator (two
//               accumulators alternate between segments)
//   warps 10-13 epilogue: at a segment's end they tcgen05.ld their rows of the accumulator,
//               scale and add to y with atomics (segments of one tile in two CTAs combine
//               there), after adding the segment's slow groups in fp32
// Three steps are in flight in tensor memory (A slots: a_full when stored, step_free when their
// MMAs completed), so the dequantizers store steps i + 1 and i + 2 while the MMAs of step i run;
// the activation tiles have their own deeper ring (x_full / x_free, 5 stages at N = 64, 8 below).
// The preparation kernel also zeroes y and the status word. Every barrier wait is bounded: on
// timeout the CTA raises a status flag, drains what it issued, frees its tensor memory and
// returns.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kTileM = 128;
constexpr int kXWarp = 0;                          // TMA producer of the activation tiles
constexpr int kMmaWarp = 1;
constexpr int kDeqWarp0 = 2;
constexpr int kDeqWarps = 8;                       // two per TMEM lane quarter, two groups of a step each
constexpr int kEpiWarp0 = kDeqWarp0 + kDeqWarps;
constexpr int kEpiWarps = 4;                       // one per TMEM lane quarter
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kG = 4;                              // groups per pipeline step
constexpr int kSlots = 3;                          // steps in flight: A slots (tensor memory), activation stages
constexpr int kAccBufs = 2;                        // fp32 segment accumulators in tensor memory
constexpr int kFlagSlots = 8;                      // per-segment masks of rows with slow groups
constexpr uint32_t kACols = 32;                    // one group of A: 128 lanes x 64 fp16
constexpr uint32_t kMaxFastScale = 0x6C00u;        // 4096 in fp16 bits
constexpr uint32_t kMaxFastZero = 15u;
constexpr int kPrepThreads = 256;

template <int NT>
struct Cfg {
  static constexpr uint32_t kXBytes = NT * 128;                     // one group of activations
  static constexpr uint32_t kAccCols = kAccBufs * NT;
  static constexpr uint32_t kACol0 = kAccCols;                     // A slots follow the accumulators
  static constexpr uint32_t kCols = kAccCols + kSlots * kG * kACols;
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "tensor memory holds 512 columns");
  // activation stages: as many as fit in ~160 KB, so the TMA latency of the activation tiles
  // (from L2) is hidden behind several steps; at most 8
  static constexpr int kXStages = (160 * 1024) / (kG * kXBytes) < 8 ? (160 * 1024) / (kG * kXBytes) : 8;
  static_assert(kXStages >= kSlots, "activation stages");
  static constexpr int kBars = 2 * kSlots + 2 * kXStages + 2 * kAccBufs + kFlagSlots + 1;
  static constexpr uint32_t kSmem = 1024 + kXStages * kG * kXBytes + kBars * 8 + kFlagSlots * 16 + NT * 4 + 16;
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// one group's codes, residual and metadata for one dequantizer thread (residual variant)
struct ResBuf {
  uint4 c[2];
  uint4 r[8];
  uint32_t s, z;
};

__device__ __forceinline__ uint32_t word4c(const uint4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// one step's codes and metadata for one dequantizer thread: 64 bytes (two groups) of its row,
// the two groups' fp16 scales and zero points
struct CodeBuf {
  uint4 c[4];
  uint32_t s2, z2;
};

// UMMA shared-memory descriptor: K-major operand in the 128-byte swizzled canonical layout
// (8-row groups of 128-byte rows, 1024 bytes apart), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;              // leading byte offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;      // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;              // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;              // SWIZZLE_128B
  return d;
}

// instruction descriptor: D fp32, A and B fp16 (format 0), both K-major, M = 128, N = NT
template <int NT>
__device__ __forceinline__ constexpr uint32_t umma_idesc() {
  return (1u << 4) | (static_cast<uint32_t>(NT >> 3) << 17) | (static_cast<uint32_t>(kTileM >> 4) << 24);
}

// TS MMA (A from tensor memory: 128 lanes = rows, two fp16 per 32-bit column, K-major) with the
// B descriptor given as two 32-bit words and a compile-time accumulate flag: the issuing thread
// shares its scheduler with busy warps, so each MMA costs it as few instructions as possible
template <bool kAccum>
__device__ __forceinline__ void umma_ts_lean(uint32_t tmem_d, uint32_t tmem_a, uint32_t bdesc_lo, uint32_t bdesc_hi,
                                             uint32_t idesc) {
  if (kAccum)
    asm volatile(
        "{\n .reg .b64 bd;\n mov.b64 bd, {%2, %3};\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, 1;\n}\n" ::"r"(tmem_d),
        "r"(tmem_a), "r"(bdesc_lo), "r"(bdesc_hi), "r"(idesc));
  else
    asm volatile(
        "{\n .reg .b64 bd;\n mov.b64 bd, {%2, %3};\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, 0;\n}\n" ::"r"(tmem_d),
        "r"(tmem_a), "r"(bdesc_lo), "r"(bdesc_hi), "r"(idesc));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
[[maybe_unused]] __device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
[[maybe_unused]] __device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// a wait for a whole warp: every lane polls, and the warp leaves together and agrees on the
// outcome -- the tcgen05.ld / tcgen05.st that follow are .sync.aligned, which a warp whose
// lanes left the wait at different times would execute diverged
__device__ __forceinline__ bool warp_wait(uint64_t *b, uint32_t parity, volatile uint32_t *abort_flag,
                                          uint32_t *status) {
  const bool ok = mbar_wait(b, parity, abort_flag, status);
  return __all_sync(0xFFFFFFFFu, ok);
}

// named barrier of the epilogue warps only
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(32 * kEpiWarps) : "memory"); }

// ---- fp16 dequantization --------------------------------------------------------------------
// (w & mask) | 0x64006400: a nibble at bits 0-3 (16-19) gives the fp16 1024 + q, a nibble at
// bits 4-7 (20-23) gives 1024 + 16 q, in the low (high) half
__device__ __forceinline__ uint32_t nib_f16(uint32_t w, uint32_t mask) {
  uint32_t out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(w), "r"(mask), "r"(0x64006400u));
  return out;
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight codes of one row (K positions 8t .. 8t+7, the first in the low nibble) -> four 32-bit
// tensor-memory columns holding the fp16 pairs (0,4), (1,5), (2,6), (3,7) of s * (q - z); the
// preparation kernel stores the activations in the same order. zz1 = (1024 + z) in both
// halves, nzz16 = -(64 + z), s2 = s in both halves. The subtractions are exact: (1024 + q) -
// (1024 + z) directly, and (1024 + 16 q) / 16 - (64 + z) in one FMA whose product is exact.
__device__ __forceinline__ void deq_word(uint32_t wd, uint32_t zz1, uint32_t nzz16, uint32_t s2, uint32_t *out) {
  const uint32_t w8 = wd >> 8;
  out[0] = h2_mul(h2_sub(nib_f16(wd, 0x000F000Fu), zz1), s2);
  out[1] = h2_mul(h2_fma(nib_f16(wd, 0x00F000F0u), 0x2C002C00u, nzz16), s2);
  out[2] = h2_mul(h2_sub(nib_f16(w8, 0x000F000Fu), zz1), s2);
  out[3] = h2_mul(h2_fma(nib_f16(w8, 0x00F000F0u), 0x2C002C00u, nzz16), s2);
}

// groups the tensor cores take: |s| <= 4096 (finite) and z <= 15
__device__ __forceinline__ bool slow_group(uint32_t sbits, uint32_t z) {
  return (sbits & 0x7FFFu) > kMaxFastScale || z > kMaxFastZero;
}

// The work of one CTA: steps = (tile, kG groups) in row-major order; step p of a tile covers
// groups kG*p .. kG*p + kG - 1 (the tensor-core path takes K a multiple of 4 groups).
struct Walk {
  int64_t i;    // current step (tile * P + p)
  int tile, p;  // tile, step within the tile
};
__device__ __forceinline__ void walk_init(Walk &w, int64_t i, int P) {
  w.i = i;
  w.tile = static_cast<int>(i / P);
  w.p = static_cast<int>(i % P);
}
__device__ __forceinline__ void walk_next(Walk &w, int P) {
  ++w.i;
  if (++w.p == P) {
    w.p = 0;
    ++w.tile;
  }
}
// the step ends a segment: the tile's last step or the CTA's last
__device__ __forceinline__ bool walk_seg_end(const Walk &w, int P, int64_t it_end) {
  return w.p + 1 == P || w.i + 1 == it_end;
}

// ---- the activation preparation kernel --------------------------------------------------------
// grid (splits, m): every CTA of batch row i finds max_k |x[i, k]| (the row is read by each of
// the row's CTAs; the repeats hit L2), then converts its share of the row to fp16 scaled by
// 2^-e_i in the dequantizer's pair order, and zeroes its share of y[i, :]. xmul[i] = 2^e_i.
__global__ void __launch_bounds__(kPrepThreads)
gemm_prep_kernel(const uint16_t *__restrict__ x, int64_t K, uint16_t *__restrict__ x16, float *__restrict__ xmul,
                 float *__restrict__ y, int64_t N, uint32_t *__restrict__ status) {
  pdl_wait();                  // x, and the earlier readers of x16, xmul, y and the status word
  // the GEMM may set up (barriers, tensor memory, code loads) meanwhile: only after the wait, so
  // its early code loads never overtake the codes' producer
  pdl_launch_dependents();
  __shared__ uint32_t red[kPrepThreads / 32];
  const int64_t i = blockIdx.y;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + i * K);
  const int64_t n8 = K / 8;
  uint32_t mx = 0;             // non-negative bf16 values order like their bit patterns (NaN above inf)
  for (int64_t c = threadIdx.x; c < n8; c += kPrepThreads) {
    const uint4 v = __ldg(xr + c);
    const uint32_t a = v.x & 0x7FFF7FFFu, b = v.y & 0x7FFF7FFFu, d = v.z & 0x7FFF7FFFu, e = v.w & 0x7FFF7FFFu;
    mx = max(mx, max(max(a & 0xFFFFu, a >> 16), max(b & 0xFFFFu, b >> 16)));
    mx = max(mx, max(max(d & 0xFFFFu, d >> 16), max(e & 0xFFFFu, e >> 16)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int k = 1; k < kPrepThreads / 32; ++k) mx = max(mx, red[k]);
  // e_i: max * 2^-e_i in [2^14, 2^15); 0 for an all-zero or non-finite row
  int e = 0;
  if (mx != 0u && mx < 0x7F80u) {
    int fe;
    frexpf(bf16_bits_to_f32(static_cast<uint16_t>(mx)), &fe);   // max = f * 2^fe, f in [0.5, 1)
    e = fe - 15;
  }
  // 2^-e as two normal floats (|e| <= 147 does not fit one)
  const int ea = -e / 2, eb = -e - ea;
  const float fa = __int_as_float((ea + 127) << 23), fb = __int_as_float((eb + 127) << 23);
  if (blockIdx.x == 0 && threadIdx.x == 0) xmul[i] = ldexpf(1.0f, e);
  if (status && i == 0 && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
  // this CTA's share of the 8-element chunks
  const int64_t c0 = n8 * blockIdx.x / gridDim.x, c1 = n8 * (blockIdx.x + 1) / gridDim.x;
  uint4 *xo = reinterpret_cast<uint4 *>(x16 + i * K);
  for (int64_t c = c0 + threadIdx.x; c < c1; c += kPrepThreads) {
    const uint4 v = __ldg(xr + c);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = __fmul_rn(__fmul_rn(__uint_as_float(wv[j] << 16), fa), fb);
      f[2 * j + 1] = __fmul_rn(__fmul_rn(__uint_as_float(wv[j] & 0xFFFF0000u), fa), fb);
    }
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = __floats2half2_rn(f[j], f[j + 4]);      // pair (j, j + 4)
      o[j] = *reinterpret_cast<const uint32_t *>(&h);
    }
    xo[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  const int64_t n0 = N * blockIdx.x / gridDim.x, n1 = N * (blockIdx.x + 1) / gridDim.x;
  for (int64_t n = n0 + threadIdx.x; n < n1; n += kPrepThreads) y[i * N + n] = 0.0f;
}

// ---- the GEMM kernel ----------------------------------------------------------------------------
// One step = kG groups (256 columns) of one 128-row tile. A step's A operand occupies one of
// kSlots slots of tensor memory and its activations one of XS shared-memory stages; two MMA
// commits per step (step_free, x_free) release them. The dequantizers load their rows' codes straight
// into registers (three steps in flight per thread: 16-byte loads of 64 contiguous bytes per
// row and step), so codes never pass through shared memory, whose bandwidth the activation
// tiles and the MMAs' operand reads need.
template <int NT, bool RES>
__global__ void __launch_bounds__(kThreads, 1)
gemm4_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const uint8_t *__restrict__ plane,
                const uint16_t *__restrict__ scale, const uint8_t *__restrict__ zero,
                const uint16_t *__restrict__ res, const uint16_t *__restrict__ xb, const float *__restrict__ xmul,
                float *__restrict__ y, int m, int64_t N, int64_t K, int KG, int64_t n_items,
                uint32_t *__restrict__ status) {
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem;                                   // activation stages (1024-aligned, swizzled)
  constexpr int XS = C::kXStages;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sX + XS * kG * C::kXBytes);
  uint64_t *a_full = bars, *step_free = a_full + kSlots;   // A slots: stored / MMAs done
  uint64_t *x_full = step_free + kSlots, *x_free = x_full + XS;   // activation stages: landed / MMAs done
  uint64_t *acc_full = x_free + XS, *acc_empty = acc_full + kAccBufs;
  uint64_t *seg_done = acc_empty + kAccBufs;            // dequantizers finished a segment's masks
  uint64_t *drain = seg_done + kFlagSlots;
  uint32_t *seg_mask = reinterpret_cast<uint32_t *>(drain + 1);   // [kFlagSlots][4 lane quarters]
  float *s_xmul = reinterpret_cast<float *>(seg_mask + kFlagSlots * 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_xmul + NT);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t it_begin = static_cast<int64_t>(blockIdx.x) * n_items / gridDim.x;
  const int64_t it_end = static_cast<int64_t>(blockIdx.x + 1) * n_items / gridDim.x;
  const int n_local = static_cast<int>(it_end - it_begin);
  const int P = KG / kG;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(a_full + i, kDeqWarps);
      mbar_init(step_free + i, 1);
    }
    for (int i = 0; i < XS; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(x_free + i, 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, kEpiWarps);
    }
    for (int i = 0; i < kFlagSlots; ++i) mbar_init(seg_done + i, kDeqWarps);
    for (int i = 0; i < kFlagSlots * 4; ++i) seg_mask[i] = 0u;
    mbar_init(drain, 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kXWarp) {
    // ---------------- TMA producer: the step's activation tiles ----------------
    if (lane == 0) {
      pdl_wait();                 // the fp16 activations come from the preparation kernel
      Walk w;
      walk_init(w, it_begin, P);
      int x_issued = 0;
      bool dropped = false;
      for (int li = 0; li < n_local; ++li) {
        const int st = li % XS;
        if (!mbar_wait(x_free + st, ((li / XS) & 1) ^ 1, abort_flag, status)) break;
#ifdef CQ_TEST_DROP_FIRST_COPY
        // test build only (never in libcq.so): CTA 0 does not request its first activation
        // tiles, so the MMA issuer's wait runs out and every role takes the abort path
        if (blockIdx.x == 0 && li == 0) {
          dropped = true;
          x_issued = li + 1;
          walk_next(w, P);
          continue;
        }
#endif
        uint8_t *dst = sX + st * kG * C::kXBytes;
        (void)CQ_CHECK(static_cast<int64_t>(kG) * (w.p + 1) * 64 <= K, 0x0604u);
        mbar_arrive_expect_tx(x_full + st, kG * C::kXBytes);
        for (int jj = 0; jj < kG; ++jj) tma_load_2d(dst + jj * C::kXBytes, &tm_x, (kG * w.p + jj) * 64, 0, x_full + st);
        x_issued = li + 1;
        walk_next(w, P);
      }
      // every issued copy lands before the CTA exits
      for (int li = x_issued - XS > 0 ? x_issued - XS : 0; li < x_issued; ++li)
        if (!(dropped && li == 0)) mbar_wait(x_full + (li % XS), (li / XS) & 1, abort_flag, status, false);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc<NT>();
      // B descriptors differ only in the start-address field (bits 0-13, address >> 4), which
      // no offset here carries out of: adding to the low word is enough
      const uint64_t d0 = umma_desc_sw128(smem_u32(sX));
      const uint32_t dlo0 = static_cast<uint32_t>(d0), dhi = static_cast<uint32_t>(d0 >> 32);
      Walk w;
      walk_init(w, it_begin, P);
      int seg = 0;
      bool first = true;          // the next step opens a segment
      for (int li = 0; li < n_local; ++li) {
        const int st = li % kSlots, b = seg % kAccBufs, xst = li % XS;
        const uint32_t par = (li / kSlots) & 1;
        const bool seg_end = walk_seg_end(w, P, it_end);
        if (first && !mbar_wait(acc_empty + b, ((seg / kAccBufs) & 1) ^ 1, abort_flag, status)) break;
        if (!mbar_wait(x_full + xst, (li / XS) & 1, abort_flag, status)) break;
        if (!mbar_wait(a_full + st, par, abort_flag, status)) break;
        tc_fence_after();
        (void)CQ_CHECK(C::kACol0 + (st + 1) * kG * kACols <= C::kTmemCols && (b + 1) * NT <= C::kAccCols, 0x0603u);
        const uint32_t ta = tmem + C::kACol0 + st * kG * kACols;
        const uint32_t td = tmem + b * NT;
        const uint32_t blo = dlo0 + ((xst * kG * C::kXBytes) >> 4);
        if (first) umma_ts_lean<false>(td, ta, blo, dhi, idesc);
        else umma_ts_lean<true>(td, ta, blo, dhi, idesc);
        umma_ts_lean<true>(td, ta + 8, blo + 2, dhi, idesc);
        umma_ts_lean<true>(td, ta + 16, blo + 4, dhi, idesc);
        umma_ts_lean<true>(td, ta + 24, blo + 6, dhi, idesc);
#pragma unroll
        for (int jj = 1; jj < kG; ++jj) {
          const uint32_t taj = ta + jj * kACols, bj = blo + jj * (C::kXBytes >> 4);
          umma_ts_lean<true>(td, taj, bj, dhi, idesc);
          umma_ts_lean<true>(td, taj + 8, bj + 2, dhi, idesc);
          umma_ts_lean<true>(td, taj + 16, bj + 4, dhi, idesc);
          umma_ts_lean<true>(td, taj + 24, bj + 6, dhi, idesc);
        }
        umma_commit(step_free + st);
        umma_commit(x_free + xst);
        if (seg_end) {
          umma_commit(acc_full + b);
          ++seg;
        }
        first = seg_end;
        walk_next(w, P);
      }
      // all issued MMAs have completed before tensor memory is released
      umma_commit(drain);
      mbar_wait(drain, 0, abort_flag, status, false);
    }
  } else if (warp < kEpiWarp0) {
    // ---------------- dequantize: two groups of a row per thread, into tensor memory ----------------
    // a warp may only touch TMEM lanes 32 * (warp % 4) .. + 31, so rows follow the warp index
    const int quad = warp & 3;
    const int r = quad * 32 + lane;               // tile row = TMEM lane
    const int part = (warp - kDeqWarp0) >> 2;     // groups 2 part, 2 part + 1 of each step
    const uint32_t tlane = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t row_bytes = K / 2;
    Walk wl, wp;
    walk_init(wl, it_begin, P);
    walk_init(wp, it_begin, P);
    int seg = 0;
    bool slow = false;                            // this row has a slow group in the segment
    auto load = [&](CodeBuf &cb) {
      int64_t row = static_cast<int64_t>(wl.tile) * kTileM + r;
      row = row < N ? row : N - 1;                // rows past the end: any valid row, result unused
      const int g = kG * wl.p + 2 * part;
      if (CQ_CHECK(static_cast<int64_t>(wl.tile) * kTileM < N && g + 2 <= KG, 0x0601u)) {
        const uint4 *src = reinterpret_cast<const uint4 *>(plane + row * row_bytes + g * 32);
        cb.c[0] = __ldcs(src);
        cb.c[1] = __ldcs(src + 1);
        cb.c[2] = __ldcs(src + 2);
        cb.c[3] = __ldcs(src + 3);
        cb.s2 = __ldg(reinterpret_cast<const uint32_t *>(scale + row * KG + g));
        cb.z2 = __ldg(reinterpret_cast<const uint16_t *>(zero + row * KG + g));
      } else {
        cb = CodeBuf{};
      }
      walk_next(wl, P);
    };
    // dequantize a loaded step into its A slot; false when a wait gave up
    auto process = [&](const CodeBuf &cb, int li) -> bool {
      const int st = li % kSlots;
      uint32_t v[32];
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        const uint32_t z = (cb.z2 >> (8 * grp)) & 0xFFu;
        const uint32_t sbits = (cb.s2 >> (16 * grp)) & 0xFFFFu;
        const bool sl = slow_group(sbits, z);
        slow |= sl;
        const uint32_t zc = sl ? 0u : z;
        const uint32_t zz1 = 0x64006400u | zc | (zc << 16);
        const uint32_t nzz16 = 0xD400D400u | (zc << 4) | (zc << 20);
        const uint32_t s2 = sl ? 0u : (sbits | (sbits << 16));
        const uint4 lo = cb.c[2 * grp], hi = cb.c[2 * grp + 1];
        deq_word(lo.x, zz1, nzz16, s2, &v[0]);
        deq_word(lo.y, zz1, nzz16, s2, &v[4]);
        deq_word(lo.z, zz1, nzz16, s2, &v[8]);
        deq_word(lo.w, zz1, nzz16, s2, &v[12]);
        deq_word(hi.x, zz1, nzz16, s2, &v[16]);
        deq_word(hi.y, zz1, nzz16, s2, &v[20]);
        deq_word(hi.z, zz1, nzz16, s2, &v[24]);
        deq_word(hi.w, zz1, nzz16, s2, &v[28]);
        if (grp == 0) {
          // the slot is free once the MMAs of the step kSlots earlier have completed
          if (li >= kSlots && !warp_wait(step_free + st, ((li / kSlots) & 1) ^ 1, abort_flag, status)) return false;
          tc_fence_after();
        }
        tmem_st32(tmem + tlane + C::kACol0 + st * kG * kACols + (2 * part + grp) * kACols, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full + st);
      if (walk_seg_end(wp, P, it_end)) {
        // rows whose slow groups the epilogue adds; then the segment's mask is complete
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, slow);
        const int fs = seg % kFlagSlots;
        if (lane == 0) {
          if (bal) atomicOr(seg_mask + fs * 4 + quad, bal);
          mbar_arrive(seg_done + fs);
        }
        slow = false;
        ++seg;
      }
      walk_next(wp, P);
      return true;
    };
    if constexpr (!RES) {
      CodeBuf b0, b1, b2;
      if (n_local > 0) load(b0);
      if (n_local > 1) load(b1);
      if (n_local > 2) load(b2);
      for (int li = 0; li < n_local; li += 3) {
        if (!process(b0, li)) break;
        if (li + 3 < n_local) load(b0);
        if (li + 1 >= n_local || !process(b1, li + 1)) break;
        if (li + 4 < n_local) load(b1);
        if (li + 2 >= n_local || !process(b2, li + 2)) break;
        if (li + 5 < n_local) load(b2);
      }
    } else {
      // with a bf16 residual: A = RN16(fma(s, q - z, r)) (q - z exact in fp32, one fp32 rounding,
      // then one fp16 rounding), one group at a time with the next group's loads in flight (the
      // residual is four times the codes' bytes, so fewer groups fit in registers)
      const int n_grp = 2 * n_local;
      auto rload = [&](ResBuf &b, int t) {
        int64_t row = static_cast<int64_t>(wl.tile) * kTileM + r;
        row = row < N ? row : N - 1;
        const int g = kG * wl.p + 2 * part + (t & 1);
        const uint4 *src = reinterpret_cast<const uint4 *>(plane + row * row_bytes + g * 32);
        b.c[0] = __ldcs(src);
        b.c[1] = __ldcs(src + 1);
        const uint4 *rs = reinterpret_cast<const uint4 *>(res + row * K + g * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i) b.r[i] = __ldcs(rs + i);
        b.s = __ldg(scale + row * KG + g);
        b.z = __ldg(zero + row * KG + g);
        if (t & 1) walk_next(wl, P);
      };
      auto rprocess = [&](const ResBuf &b, int t) -> bool {
        const int li = t >> 1, grp = t & 1, st = li % kSlots;
        const bool sl = slow_group(b.s, b.z);
        slow |= sl;
        const float sf = sl ? 0.0f : f16_bits_to_f32(static_cast<uint16_t>(b.s));
        const float zb = 8388608.0f + static_cast<float>(sl ? 0u : b.z);
        uint32_t v[32];
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
          const uint32_t cw = wd < 4 ? word4c(b.c[0], wd) : word4c(b.c[1], wd - 4);
          const uint4 rr = b.r[wd];       // residuals of k = 8 wd .. 8 wd + 7
          const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // the pair (j, j + 4) of these eight: codes at nibbles j and j + 4
            const float qa = __fsub_rn(__uint_as_float(0x4B000000u | ((cw >> (4 * j)) & 15u)), zb);
            const float qb = __fsub_rn(__uint_as_float(0x4B000000u | ((cw >> (4 * j + 16)) & 15u)), zb);
            const uint32_t w0 = rw[j >> 1], w1 = rw[2 + (j >> 1)];
            const float ra = __uint_as_float((j & 1) ? (w0 & 0xFFFF0000u) : (w0 << 16));
            const float rb = __uint_as_float((j & 1) ? (w1 & 0xFFFF0000u) : (w1 << 16));
            const __half2 h = __floats2half2_rn(__fmaf_rn(sf, qa, ra), __fmaf_rn(sf, qb, rb));
            v[4 * wd + j] = *reinterpret_cast<const uint32_t *>(&h);
          }
        }
        if (grp == 0) {
          if (li >= kSlots && !warp_wait(step_free + st, ((li / kSlots) & 1) ^ 1, abort_flag, status)) return false;
          tc_fence_after();
        }
        tmem_st32(tmem + tlane + C::kACol0 + st * kG * kACols + (2 * part + grp) * kACols, v);
        if (grp == 1) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_full + st);
          if (walk_seg_end(wp, P, it_end)) {
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, slow);
            const int fs = seg % kFlagSlots;
            if (lane == 0) {
              if (bal) atomicOr(seg_mask + fs * 4 + quad, bal);
              mbar_arrive(seg_done + fs);
            }
            slow = false;
            ++seg;
          }
          walk_next(wp, P);
        }
        return true;
      };
      ResBuf a0, a1;
      if (n_grp > 0) rload(a0, 0);
      if (n_grp > 1) rload(a1, 1);
      for (int t = 0; t < n_grp; t += 2) {
        if (!rprocess(a0, t)) break;
        if (t + 2 < n_grp) rload(a0, t + 2);
        if (!rprocess(a1, t + 1)) break;
        if (t + 3 < n_grp) rload(a1, t + 3);
      }
    }
  } else {
    // ---------------- epilogue: one row per thread, all NT columns ----------------
    const int quad = warp & 3;                 // this warp may read TMEM lanes 32*quad .. +31
    const int r = quad * 32 + lane;
    const int et = threadIdx.x - 32 * kEpiWarp0;
    pdl_wait();                                // xmul and the zeroed y come from the preparation kernel
    if (et < NT) s_xmul[et] = et < m ? xmul[et] : 0.0f;
    epi_sync();
    Walk w;
    walk_init(w, it_begin, P);
    int seg = 0, ga = kG * w.p;
    bool open = true;                          // the next step opens a segment
    for (int li = 0; li < n_local; ++li) {
      if (open) ga = kG * w.p;
      const bool seg_end = walk_seg_end(w, P, it_end);
      open = seg_end;
      if (seg_end) {
        const int b = seg % kAccBufs, fs = seg % kFlagSlots;
        const int gb = kG * w.p + kG;
        const bool seg_ok = CQ_CHECK(gb <= KG && ga >= 0 && static_cast<int64_t>(w.tile) * kTileM < N, 0x0602u);
        const int64_t row = seg_ok ? static_cast<int64_t>(w.tile) * kTileM + r : N;
        if (!warp_wait(seg_done + fs, (seg / kFlagSlots) & 1, abort_flag, status)) break;
        const uint32_t mask = seg_mask[fs * 4 + quad];
        __syncwarp();
        if (lane == 0) seg_mask[fs * 4 + quad] = 0u;
        if (((mask >> lane) & 1u) && row < N) {
          // groups the tensor cores did not take: s * sum_k (q - z) x in fp32, straight to y
          for (int g = ga; g < gb; ++g) {
            const uint32_t sbits = scale[row * KG + g], z = zero[row * KG + g];
            if (!slow_group(sbits, z)) continue;
            const float sf = f16_bits_to_f32(static_cast<uint16_t>(sbits));
            const uint8_t *cp = plane + row * (K / 2) + g * 32;
            for (int i = 0; i < m; ++i) {
              const uint16_t *xg = xb + i * K + g * 64;
              float acc = 0.0f;
              for (int k = 0; k < 64; ++k) {
                const int q = (cp[k >> 1] >> ((k & 1) * 4)) & 15;
                acc = fmaf(static_cast<float>(q - static_cast<int>(z)), bf16_bits_to_f32(xg[k]), acc);
              }
              atomicAdd(y + static_cast<int64_t>(i) * N + row, __fmul_rn(acc, sf));
            }
          }
        }
        __syncwarp();
        if (!warp_wait(acc_full + b, (seg / kAccBufs) & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + b * NT;
        constexpr int kChunk = NT < 32 ? NT : 32;   // columns per load (registers are scarce)
#pragma unroll
        for (int c0 = 0; c0 < NT; c0 += kChunk) {
          uint32_t dv[kChunk];
#pragma unroll
          for (int c1 = 0; c1 < kChunk; c1 += 16) tmem_ld16(tbase + c0 + c1, dv + c1);
          tmem_wait_ld();
          if (row < N) {
#pragma unroll
            for (int c = 0; c < kChunk; ++c)
              if (c0 + c < m)
                atomicAdd(y + static_cast<int64_t>(c0 + c) * N + row, __fmul_rn(__uint_as_float(dv[c]), s_xmul[c0 + c]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + b);   // the accumulator has been read
        ++seg;
      }
      walk_next(w, P);
    }
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(C::kTmemCols));
  }
}

// ---- host side ---------------------------------------------------------------------------

// workspace: [0, 16) status word, [16, 16 + 4 * 64) xmul, [512, ...) fp16 activations of a
// batch slice of at most 64 rows
constexpr size_t kWsXmul = 16, kWsX16 = 512;
constexpr int kSliceRows = 64;

template <int NT, bool RES>
cq_status launch_nt(const cq_qweight &qw, const void *x, int m, float *y, uint8_t *ws, bool clear_status,
                    cudaStream_t s) {
  using C = Cfg<NT>;
  auto encode = encode_fn();
  if (!encode) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: cuTensorMapEncodeTiled unavailable");
  const int64_t N = qw.rows, K = qw.cols;
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  float *xmul = reinterpret_cast<float *>(ws + kWsXmul);
  uint16_t *x16 = reinterpret_cast<uint16_t *>(ws + kWsX16);
  CUtensorMap tm_x;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(m)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
    cuuint32_t box[2] = {64, NT};
    cuuint32_t es[2] = {1, 1};
    CUresult r = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: activation tensor map (%d)", (int)r);
  }
  // 1. the activation preparation (fp16 copy, y and status cleared)
  {
    const int64_t want = (2 * static_cast<int64_t>(sm_count()) + m - 1) / m;
    const int64_t splits = want < 1 ? 1 : want > 64 ? 64 : want;
    cq_status st = cuda_check(launch_pdl(gemm_prep_kernel, dim3(static_cast<unsigned>(splits), static_cast<unsigned>(m)),
                                         dim3(kPrepThreads), 0, s, static_cast<const uint16_t *>(x), K, x16, xmul, y, N,
                                         clear_status ? status : nullptr),
                              "cq_dequant_gemm: preparation");
    if (st != CQ_OK) return st;
    st = launch_check("cq_dequant_gemm: preparation");
    if (st != CQ_OK) return st;
  }
  // 2. the GEMM, allowed to start while the preparation runs (it waits for it where it must)
  const int KG = static_cast<int>(K / kGroup);
  const int64_t tiles = (N + kTileM - 1) / kTileM;
  const int64_t items = tiles * (KG / kG);                // steps of kG groups
  const int64_t grid = items < sm_count() ? items : sm_count();
  cq_status st = cuda_check(cudaFuncSetAttribute(gemm4_tc_kernel<NT, RES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(C::kSmem)),
                            "cq_dequant_gemm: shared memory attribute");
  if (st != CQ_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, gemm4_tc_kernel<NT, RES>, tm_x, static_cast<const uint8_t *>(qw.plane[2]),
                                       qw.scale, qw.zero, static_cast<const uint16_t *>(qw.residual),
                                       static_cast<const uint16_t *>(x), static_cast<const float *>(xmul), y, m, N, K,
                                       KG, items, status),
                    "cq_dequant_gemm");
}

}  // namespace

// fixed-4 weights, no residual or a bf16 one, bf16 x, m >= 16, K a multiple of 4 groups, and the
// alignments the per-thread loads need (16-byte codes and residual rows, 4-byte scale pairs,
// 2-byte zero pairs)
bool gemm_tc_eligible(const cq_qweight &qw, cq_dtype xdt, int m) {
  const bool res_ok = qw.residual == nullptr || (qw.residual_dtype == CQ_BF16 && aligned16(qw.residual));
  return qw.bits == nullptr && res_ok && xdt == CQ_BF16 && m >= 16 && qw.rows > 0 && qw.cols > 0 &&
         (qw.cols / kGroup) % kG == 0 && aligned16(qw.plane[2]) && (reinterpret_cast<uintptr_t>(qw.scale) & 3u) == 0 &&
         (reinterpret_cast<uintptr_t>(qw.zero) & 1u) == 0;
}

// the status word, the per-row powers of two and the fp16 activations of one batch slice
size_t gemm_tc_workspace(int64_t, int64_t cols, int m) {
  const int64_t rows = m < kSliceRows ? m : kSliceRows;
  return kWsX16 + static_cast<size_t>(rows) * static_cast<size_t>(cols) * 2;
}

cq_status launch_gemm_tc(const cq_qweight &qw, const void *x, int m, float *y, void *ws, size_t, cudaStream_t s) {
  const int64_t N = qw.rows;
  if (!aligned16(x)) return fail(CQ_ERR_ALIGN, "cq_dequant_gemm: x must be 16-byte aligned");
  // the batch in slices of at most 64 rows (the MMA's N); slices run in stream order, so each
  // preparation overwrites the previous slice's fp16 activations only after that GEMM ended
  for (int i0 = 0; i0 < m; i0 += kSliceRows) {
    const int mi = m - i0 < kSliceRows ? m - i0 : kSliceRows;
    const void *xi = static_cast<const uint16_t *>(x) + static_cast<int64_t>(i0) * qw.cols;
    float *yi = y + static_cast<int64_t>(i0) * N;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    cq_status st;
    if (qw.residual) {
      if (mi <= 16) st = launch_nt<16, true>(qw, xi, mi, yi, w8, i0 == 0, s);
      else if (mi <= 32) st = launch_nt<32, true>(qw, xi, mi, yi, w8, i0 == 0, s);
      else st = launch_nt<64, true>(qw, xi, mi, yi, w8, i0 == 0, s);
    } else {
      if (mi <= 16) st = launch_nt<16, false>(qw, xi, mi, yi, w8, i0 == 0, s);
      else if (mi <= 32) st = launch_nt<32, false>(qw, xi, mi, yi, w8, i0 == 0, s);
      else st = launch_nt<64, false>(qw, xi, mi, yi, w8, i0 == 0, s);
    }
    if (st != CQ_OK) return st;
  }
  return CQ_OK;
}

}  // namespace cq

// ---- entry point for callers that cannot allocate device memory --------------------------
//
// cq_dequant_gemm_static runs the same GEMM with its scratch in this file-scope device
// array instead of a caller-provided workspace. Each GPU that loads the library keeps the
// array until the process exits. In host code the array's name only stands in for it, so the
// device address is looked up once per device (cudaGetSymbolAddress, with that device
// current) and passed to the kernel.
namespace cq {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // the fp16 activations of a 64-row slice, K <= 65532
__device__ __align__(256) unsigned char g_gemm_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
void *g_scratch_ptr[kMaxScratchDevices];
cudaError_t g_scratch_err[kMaxScratchDevices];
std::once_flag g_scratch_once[kMaxScratchDevices];

cq_status static_scratch(void **out) {
  int dev = 0;
  cq_status st = cuda_check(cudaGetDevice(&dev), "cq_dequant_gemm_static: current device");
  if (st != CQ_OK) return st;
  if (dev < 0 || dev >= kMaxScratchDevices)
    return fail(CQ_ERR_RANGE, "cq_dequant_gemm_static: device %d beyond the %d supported", dev, kMaxScratchDevices);
  std::call_once(g_scratch_once[dev], [dev] {
    void *p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_gemm_scratch);
    g_scratch_ptr[dev] = g_scratch_err[dev] == cudaSuccess ? p : nullptr;
  });
  if (g_scratch_err[dev] != cudaSuccess || !g_scratch_ptr[dev])
    return fail(CQ_ERR_CUDA, "cq_dequant_gemm_static: scratch address on device %d: %s", dev,
                cudaGetErrorString(g_scratch_err[dev]));
  *out = g_scratch_ptr[dev];
  return CQ_OK;
}

}  // namespace
}  // namespace cq

extern "C" cq_status cq_dequant_gemm_static(const cq_qweight *qw, const void *x, cq_dtype x_dtype, int m, float *y,
                                            uint32_t *status_word, cq_stream_t stream) {
  using namespace cq;
  const char *fn = "cq_dequant_gemm_static";
  // the arguments first: a bad call does no CUDA work at all, not even the address look-up
  cq_status st = check_matmul_args(qw, x, x_dtype, m, y, 256, fn);
  if (st != CQ_OK) return st;
  const bool tc = gemm_tc_eligible(*qw, x_dtype, m);
  if (tc) {
    const size_t need = gemm_tc_workspace(qw->rows, qw->cols, m);
    if (need > kStaticScratchBytes)
      return fail(CQ_ERR_RANGE, "%s: this shape needs %zu bytes of scratch, the static buffer holds %zu", fn, need,
                  kStaticScratchBytes);
  }
  void *scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != CQ_OK) return st;
  // the regular entry point does the dispatch; the scratch is the static array
  st = cq_dequant_gemm(qw, x, x_dtype, m, y, scratch, kStaticScratchBytes, stream);
  if (st != CQ_OK || !status_word) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the tensor-core GEMM leaves its status word in the first 4 bytes of the scratch; the GEMV
  // kernels that serve the other cases have none (they mark an aborted output with NaN)
  if (tc && qw->rows > 0)
    return cuda_check(cudaMemcpyAsync(status_word, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s),
                      "cq_dequant_gemm_static: status word");
  return cuda_check(cudaMemsetAsync(status_word, 0, sizeof(uint32_t), s), "cq_dequant_gemm_static: status word");
}
