// k_gemm.cu -- batched dequantize-and-multiply on the sm_100a tensor cores (tcgen05 + TMEM).
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: fused dequantize-and-multiply over packed
// low-bit weights. Here the batch is large enough (m >= 16) for a real dense contraction:
//     y[i, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) * x[i, k]
//
// Exactness: q - z (|q - z| <= 15 for 4-bit codes) and x are exact bf16 operands, the tensor
// core forms exact products and accumulates one group (64 columns) in fp32 in tensor memory;
// the epilogue multiplies that group sum by the fp32 scale and accumulates in registers.
//
// Structure (one CTA per SM, persistent; work = (128-row tile, group) items split evenly
// over the CTAs in row-major order, so a CTA covers a contiguous K range of one or two tiles):
//   warp 0      TMA producer: code blocks of 8 groups (two adjacent 128-byte-wide boxes per
//               row, 128-byte swizzled: long DRAM runs and conflict-free shared reads)
//   warp 18     TMA producer: per group the activations (m rows x 64 bf16, swizzled = the
//               UMMA K-major layout); a separate warp, so code blocks are requested as soon as
//               a buffer frees up, however far the activation ring runs ahead
//   warp 1      MMA issuer: four tcgen05.mma (M=128, N=NT, K=16) per group into one of four
//               tensor-memory accumulators; commits release the A and x stages and publish
//   warps 2-9   dequantize: each thread turns half a row of the group's codes into bf16
//               (q - z) in the 128-byte swizzled K-major layout the MMA descriptor expects
//   warps 10-17 epilogue: tcgen05.ld the group's fp32 sums (one row and half the columns per
//               thread), acc += s * sum; at the end of a tile (or of the CTA's range) add to y
// y is zeroed first; tiles split between two CTAs are combined with fp32 atomics.
// Every barrier wait is bounded: on timeout the CTA raises a status flag, drains what it
// issued, frees its tensor memory and returns.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kTileM = 128;
constexpr int kDeqWarps = 8;                       // two per TMEM lane quarter: half a row each
constexpr int kEpiWarps = 8;                       // two per TMEM lane quarter: half the columns each
constexpr int kThreads = 32 * (3 + kDeqWarps + kEpiWarps);
constexpr int kXWarp = 2 + kDeqWarps + kEpiWarps;      // the last warp loads activations
constexpr int kBlockGroups = 8;                    // groups per code block (two 128-byte boxes per row)
constexpr uint32_t kCodeBox = kTileM * 128;        // one swizzled box: 128 rows x 4 groups
constexpr uint32_t kCodeStage = 2 * kCodeBox;      // 32 KiB
constexpr int kCodeStages = 4;                     // code blocks in flight
constexpr int kG = 4;                              // groups per pipeline step
constexpr int kSteps = 2;                          // A (tensor memory) and activation (shared) slots
constexpr int kAccBufs = 1;                        // fp32 step accumulator in tensor memory (released as soon as read)
constexpr uint32_t kACols = 32;                    // one group of A: 128 lanes x 64 bf16

template <int NT>
struct Cfg {
  static constexpr uint32_t kXBytes = NT * 128;                     // one group of activations
  static constexpr uint32_t kAccCols = kAccBufs * kG * NT;
  static constexpr uint32_t kACol0 = kAccCols;                     // A slots follow the accumulators
  static constexpr uint32_t kCols = kAccCols + kSteps * kG * kACols;
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "tensor memory holds 512 columns");
  static constexpr int kBars = 2 * kCodeStages + 3 * kSteps + 2 * kAccBufs + 1;
  static constexpr uint32_t kSmem = 1024 + kCodeStages * kCodeStage + kSteps * kG * kXBytes + kBars * 8 + 16;
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

// instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = NT
template <int NT>
__device__ __forceinline__ constexpr uint32_t umma_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(NT >> 3) << 17) |
         (static_cast<uint32_t>(kTileM >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// the same with A read from tensor memory (128 lanes = rows, two bf16 per 32-bit column, K-major)
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// TS MMA with the B descriptor given as two 32-bit words and a compile-time accumulate flag:
// the issuing thread shares its scheduler with busy warps, so each MMA costs it as few
// instructions as possible
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t *r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// (128 + q) pairs in natural column order from one word of 8 nibbles: pair j = columns 2j, 2j+1
__device__ __forceinline__ uint32_t nat_pair(uint32_t w, uint32_t w4, uint32_t sel) {
  uint32_t t = __byte_perm(w, w4, sel), out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(t), "r"(0x000F000Fu), "r"(0x43004300u));
  return out;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The work of one CTA: steps = (tile, pair of groups) in row-major order; a step covers
// groups g, g + 1 of a tile (only g when it is the tile's last, odd group). Code blocks of
// 8 groups = 4 steps; a block also ends at a tile end and at the end of the CTA's range.
struct ItemWalk {
  int64_t i;          // current step (tile * P + pair)
  int tile, p, g, ng; // tile, pair, first group, groups in this step (1 or 2)
  int block;          // index of the current code block
  int block_g0;       // first group of the current block
  bool block_start, block_end, tile_end;
};

__device__ __forceinline__ void walk_set_g(ItemWalk &w, int KG) {
  w.g = kG * w.p;
  w.ng = KG - w.g < kG ? KG - w.g : kG;
}
__device__ __forceinline__ int n_steps(int KG) { return (KG + kG - 1) / kG; }

__device__ __forceinline__ void walk_init(ItemWalk &w, int64_t it_begin, int KG) {
  const int P = n_steps(KG);
  w.i = it_begin;
  w.tile = static_cast<int>(it_begin / P);
  w.p = static_cast<int>(it_begin % P);
  walk_set_g(w, KG);
  w.block = 0;
  w.block_g0 = w.g;
  w.block_start = true;
}

// flags of the current step, given the CTA's end
__device__ __forceinline__ void walk_flags(ItemWalk &w, int64_t it_end, int KG) {
  const bool last = w.i + 1 >= it_end;
  w.tile_end = (w.g + w.ng == KG) || last;
  w.block_end = w.tile_end || (((w.g + kG) & (kBlockGroups - 1)) == 0);
}

// first (tile, group) of the block after the current one (valid when it exists)
__device__ __forceinline__ void walk_next_block(const ItemWalk &w, int KG, int &tile, int &g) {
  const int g_end = (w.block_g0 | (kBlockGroups - 1)) + 1;     // next multiple of 8
  if (g_end >= KG) {
    tile = w.tile + 1;
    g = 0;
  } else {
    tile = w.tile;
    g = g_end;
  }
}

// the (up to) 8 per-group bytes / halves of one row for the block starting at group g
__device__ __forceinline__ void load_block_zeros(const uint8_t *zero, int64_t row, int KG, int g, uint32_t &lo,
                                                 uint32_t &hi) {
  uint32_t v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = (g + j < KG && ((g + j) & ~7) == (g & ~7)) ? __ldg(zero + row * KG + g + j) : 0u;
  lo = v[0] | (v[1] << 8) | (v[2] << 16) | (v[3] << 24);
  hi = v[4] | (v[5] << 8) | (v[6] << 16) | (v[7] << 24);
}
__device__ __forceinline__ void load_block_scales(const uint16_t *scale, int64_t row, int KG, int g, uint32_t (&s)[4]) {
  uint32_t v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = (g + j < KG && ((g + j) & ~7) == (g & ~7)) ? __ldg(scale + row * KG + g + j) : 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) s[j] = v[2 * j] | (v[2 * j + 1] << 16);
}

__device__ __forceinline__ void walk_next(ItemWalk &w, int KG) {
  const bool new_block = w.block_end;
  ++w.i;
  if (++w.p == n_steps(KG)) {
    w.p = 0;
    ++w.tile;
  }
  walk_set_g(w, KG);
  w.block_start = new_block;
  if (new_block) {
    ++w.block;
    w.block_g0 = w.g;
  }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
gemm4_tc_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                const uint16_t *__restrict__ scale, const uint8_t *__restrict__ zero, float *__restrict__ y,
                int m, int64_t N, int KG, int64_t n_items, uint32_t *__restrict__ status) {
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sC = smem;                                   // code blocks (1024-aligned, swizzled)
  uint8_t *sX = sC + kCodeStages * kCodeStage;          // activation tiles (1024-aligned)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sX + kSteps * kG * C::kXBytes);
  uint64_t *c_full = bars, *c_empty = c_full + kCodeStages;
  // a step (kG groups) has an A slot in tensor memory and an activation slot in shared memory,
  // filled separately (a_full, x_full) and released together by one MMA commit (s_empty)
  uint64_t *a_full = c_empty + kCodeStages, *x_full = a_full + kSteps, *s_empty = x_full + kSteps;
  uint64_t *acc_full = s_empty + kSteps, *acc_empty = acc_full + kAccBufs;
  uint64_t *drain = acc_empty + kAccBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t it_begin = static_cast<int64_t>(blockIdx.x) * n_items / gridDim.x;
  const int64_t it_end = static_cast<int64_t>(blockIdx.x + 1) * n_items / gridDim.x;
  const int n_local = static_cast<int>(it_end - it_begin);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kCodeStages; ++i) {
      mbar_init(c_full + i, 1);
      mbar_init(c_empty + i, kDeqWarps);
    }
    for (int i = 0; i < kSteps; ++i) {
      mbar_init(a_full + i, kDeqWarps);
      mbar_init(x_full + i, 1);
      mbar_init(s_empty + i, 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer: code blocks ----------------
    if (lane == 0) {
      ItemWalk w;
      walk_init(w, it_begin, KG);
      int code_issued = 0;
      for (int li = 0; li < n_local; ++li) {
        walk_flags(w, it_end, KG);
        if (w.block_start) {
          const int cs = w.block % kCodeStages;
          if (!mbar_wait(c_empty + cs, ((w.block / kCodeStages) & 1) ^ 1, abort_flag, status)) break;
          mbar_arrive_expect_tx(c_full + cs, kCodeStage);
          uint8_t *dst = sC + cs * kCodeStage;
          tma_load_2d(dst, &tm_codes, w.block_g0 * 32, w.tile * kTileM, c_full + cs);
          tma_load_2d(dst + kCodeBox, &tm_codes, w.block_g0 * 32 + 128, w.tile * kTileM, c_full + cs);
          code_issued = w.block + 1;
        }
        walk_next(w, KG);
      }
      // every copy this thread started has landed before the CTA may exit
      for (int b = code_issued - kCodeStages > 0 ? code_issued - kCodeStages : 0; b < code_issued; ++b)
        mbar_wait(c_full + (b % kCodeStages), (b / kCodeStages) & 1, abort_flag, status, false);
    }
  } else if (warp == kXWarp) {
    // ---------------- TMA producer: the step's activation tiles ----------------
    if (lane == 0) {
      ItemWalk w;
      walk_init(w, it_begin, KG);
      int x_issued = 0;
      for (int li = 0; li < n_local; ++li) {
        const int st = li % kSteps;
        if (!mbar_wait(s_empty + st, ((li / kSteps) & 1) ^ 1, abort_flag, status)) break;
        uint8_t *dst = sX + st * kG * C::kXBytes;
        mbar_arrive_expect_tx(x_full + st, w.ng * C::kXBytes);
        for (int jj = 0; jj < w.ng; ++jj) tma_load_2d(dst + jj * C::kXBytes, &tm_x, (w.g + jj) * 64, 0, x_full + st);
        x_issued = li + 1;
        walk_flags(w, it_end, KG);
        walk_next(w, KG);
      }
      for (int li = x_issued - kSteps > 0 ? x_issued - kSteps : 0; li < x_issued; ++li)
        mbar_wait(x_full + (li % kSteps), (li / kSteps) & 1, abort_flag, status, false);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc<NT>();
      // B descriptors differ only in the start-address field (bits 0-13, address >> 4), which
      // no offset here carries out of: adding to the low word is enough
      const uint64_t d0 = umma_desc_sw128(smem_u32(sX));
      const uint32_t dlo0 = static_cast<uint32_t>(d0), dhi = static_cast<uint32_t>(d0 >> 32);
      const int P = n_steps(KG);
      int p = static_cast<int>(it_begin % P);
      for (int li = 0; li < n_local; ++li) {
        const int st = li % kSteps, b = li % kAccBufs;
        const int ng = KG - kG * p < kG ? KG - kG * p : kG;
        if (++p == P) p = 0;
        if (!mbar_wait(a_full + st, (li / kSteps) & 1, abort_flag, status)) break;
        if (!mbar_wait(x_full + st, (li / kSteps) & 1, abort_flag, status)) break;
        if (!mbar_wait(acc_empty + b, ((li / kAccBufs) & 1) ^ 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t ta = tmem + C::kACol0 + st * kG * kACols;
        const uint32_t td = tmem + b * kG * NT;
        const uint32_t blo = dlo0 + ((st * kG * C::kXBytes) >> 4);
#pragma unroll
        for (int jj = 0; jj < kG; ++jj) {
          if (jj < ng) {
            const uint32_t tdj = td + jj * NT, taj = ta + jj * kACols, bj = blo + jj * (C::kXBytes >> 4);
            umma_ts_lean<false>(tdj, taj, bj, dhi, idesc);
            umma_ts_lean<true>(tdj, taj + 8, bj + 2, dhi, idesc);
            umma_ts_lean<true>(tdj, taj + 16, bj + 4, dhi, idesc);
            umma_ts_lean<true>(tdj, taj + 24, bj + 6, dhi, idesc);
          }
        }
        umma_commit(s_empty + st);
        umma_commit(acc_full + b);
      }
      // all issued MMAs have completed before tensor memory is released
      umma_commit(drain);
      mbar_wait(drain, 0, abort_flag, status, false);
    }
  } else if (warp < 2 + kDeqWarps) {
    // ---------------- dequantize: half a row per thread, into tensor memory ----------------
    // a warp may only touch TMEM lanes 32 * (warp % 4) .. + 31, so rows follow the warp index
    const int quad = warp & 3;
    const int r = quad * 32 + lane;               // tile row = TMEM lane
    const int half = (warp - 2) >> 2;             // columns 32*half .. 32*half+31 of each group
    ItemWalk w;
    walk_init(w, it_begin, KG);
    auto clamp_row = [&](int tile) {
      const int64_t row = static_cast<int64_t>(tile) * kTileM + r;
      return row < N ? row : N - 1;
    };
    // zero points of the current block and, one block ahead, of the next one
    uint32_t zlo, zhi, nzlo = 0, nzhi = 0;
    load_block_zeros(zero, clamp_row(w.tile), KG, w.g, zlo, zhi);
    const uint32_t tlane = static_cast<uint32_t>(quad * 32) << 16;
    for (int li = 0; li < n_local; ++li) {
      walk_flags(w, it_end, KG);
      const int cs = w.block % kCodeStages;
      if (w.block_start) {
        if (li > 0) {
          zlo = nzlo;
          zhi = nzhi;
        }
        int nt, ng;
        walk_next_block(w, KG, nt, ng);
        if (li + 1 < n_local) load_block_zeros(zero, clamp_row(nt), KG, ng, nzlo, nzhi);   // rows clamp: in bounds
        if (!mbar_wait(c_full + cs, (w.block / kCodeStages) & 1, abort_flag, status)) break;
      }
      const int st = li % kSteps;
      // group j of the block sits in box j/4, 16-byte chunk (2*(j%4) + half) of the row, swizzled
      uint32_t v[kG][16];
#pragma unroll
      for (int jj = 0; jj < kG; ++jj) {
        const int j = w.g - w.block_g0 + jj;
        const uint32_t z = ((j < 4 ? zlo : zhi) >> (8 * (j & 3))) & 0xFFu;
        const uint32_t zz = 0x43004300u | z | (z << 16);      // (128 + z) in both halves
        const int chunk = ((j & 3) << 1) | half;
        const uint4 cw = *reinterpret_cast<const uint4 *>(sC + cs * kCodeStage + ((j >> 2) & 1) * kCodeBox +
                                                          r * 128 + ((chunk ^ (r & 7)) << 4));
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {       // columns 32*half + 8c .. +7, two per 32-bit TMEM column
          const uint32_t wd = words[c], w4 = wd >> 4;
          v[jj][4 * c + 0] = bf16x2_sub(nat_pair(wd, w4, 0x4400u), zz);
          v[jj][4 * c + 1] = bf16x2_sub(nat_pair(wd, w4, 0x5511u), zz);
          v[jj][4 * c + 2] = bf16x2_sub(nat_pair(wd, w4, 0x6622u), zz);
          v[jj][4 * c + 3] = bf16x2_sub(nat_pair(wd, w4, 0x7733u), zz);
        }
      }
      // the code words are in registers: the block's last step releases its buffer now
      __syncwarp();
      if (lane == 0 && w.block_end) mbar_arrive(c_empty + cs);
      if (!mbar_wait(s_empty + st, ((li / kSteps) & 1) ^ 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t ta = tmem + tlane + C::kACol0 + st * kG * kACols + half * 16;
#pragma unroll
      for (int jj = 0; jj < kG; ++jj)
        if (jj < w.ng) tmem_st16(ta + jj * kACols, v[jj]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full + st);
      walk_next(w, KG);
    }
  } else if (warp < 2 + kDeqWarps + kEpiWarps) {
    // ---------------- epilogue: row r = TMEM lane, half of the columns ----------------
    const int ew = warp - 2 - kDeqWarps;
    const int quad = warp & 3;                 // this warp may read TMEM lanes 32*quad .. +31
    const int chalf = ew >> 2;                 // columns chalf*NT/2 .. +NT/2
    constexpr int NH = NT / 2;
    const int r = quad * 32 + lane;
    float2 acc[NH / 2];                        // column pairs, updated with packed fp32x2 FMAs
#pragma unroll
    for (int c = 0; c < NH / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
    ItemWalk w;
    walk_init(w, it_begin, KG);
    auto clamp_row = [&](int tile) {
      const int64_t row = static_cast<int64_t>(tile) * kTileM + r;
      return row < N ? row : N - 1;
    };
    // scales of the current block and, one block ahead, of the next one
    uint32_t sc[4], nsc[4] = {0, 0, 0, 0};
    load_block_scales(scale, clamp_row(w.tile), KG, w.g, sc);
    for (int li = 0; li < n_local; ++li) {
      walk_flags(w, it_end, KG);
      const int b = li % kAccBufs;
      const int64_t row = static_cast<int64_t>(w.tile) * kTileM + r;
      if (w.block_start) {
        if (li > 0) {
#pragma unroll
          for (int j = 0; j < 4; ++j) sc[j] = nsc[j];
        }
        int nt, ng;
        walk_next_block(w, KG, nt, ng);
        if (li + 1 < n_local) load_block_scales(scale, clamp_row(nt), KG, ng, nsc);
      }
      // the step's scales: groups js .. js + kG - 1 of the block's scale vector (two per word)
      const int js = w.g - w.block_g0;
      float sfs[kG];
#pragma unroll
      for (int jj = 0; jj < kG; ++jj) {
        const int q = js + jj;
        const uint32_t sw = q < 2 ? sc[0] : q < 4 ? sc[1] : q < 6 ? sc[2] : sc[3];   // no local-memory indexing
        sfs[jj] = jj < w.ng ? f16_bits_to_f32(static_cast<uint16_t>((q & 1) ? (sw >> 16) : (sw & 0xFFFFu))) : 0.0f;
      }
      if (!mbar_wait(acc_full + b, (li / kAccBufs) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + b * kG * NT + chalf * NH;
#pragma unroll
      for (int jj = 0; jj < kG; ++jj) {
        if (jj < w.ng) {
          uint32_t d[NH];
          if constexpr (NH >= 16) {
#pragma unroll
            for (int c0 = 0; c0 < NH; c0 += 16)
              tmem_ld16(tbase + jj * NT + c0, *reinterpret_cast<uint32_t(*)[16]>(d + c0));
          } else {
            tmem_ld8(tbase + jj * NT, d);
          }
          tmem_wait_ld();
          const float sf = sfs[jj];
          const float2 s2 = make_float2(sf, sf);
#pragma unroll
          for (int c = 0; c < NH / 2; ++c)
            acc[c] = __ffma2_rn(s2, make_float2(__uint_as_float(d[2 * c]), __uint_as_float(d[2 * c + 1])), acc[c]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + b);
      if (w.tile_end) {
        if (row < N) {
#pragma unroll
          for (int c = 0; c < NH; ++c) {
            const int col = chalf * NH + c;
            if (col < m) atomicAdd(y + static_cast<int64_t>(col) * N + row, (c & 1) ? acc[c >> 1].y : acc[c >> 1].x);
          }
        }
#pragma unroll
        for (int c = 0; c < NH / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
      }
      walk_next(w, KG);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(C::kTmemCols));
  }
}

// ---- host side ---------------------------------------------------------------------------

template <int NT>
cq_status launch_nt(const cq_qweight &qw, const void *x, int m, float *y, uint32_t *status, cudaStream_t s) {
  using C = Cfg<NT>;
  auto encode = encode_fn();
  if (!encode) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: cuTensorMapEncodeTiled unavailable");
  const int64_t N = qw.rows, K = qw.cols;
  CUtensorMap tm_codes, tm_x;
  cq_status cs = code_tensor_map(&tm_codes, qw.plane[2], N, K, kTileM, "cq_dequant_gemm");
  if (cs != CQ_OK) return cs;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(m)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
    cuuint32_t box[2] = {64, NT};
    cuuint32_t es[2] = {1, 1};
    CUresult r = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: activation tensor map (%d)", (int)r);
  }
  const int KG = static_cast<int>(K / kGroup);
  const int64_t tiles = (N + kTileM - 1) / kTileM;
  const int64_t items = tiles * ((KG + kG - 1) / kG);     // steps of kG groups
  const int64_t grid = items < sm_count() ? items : sm_count();
  cq_status st = cuda_check(cudaFuncSetAttribute(gemm4_tc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(C::kSmem)),
                            "cq_dequant_gemm: shared memory attribute");
  if (st != CQ_OK) return st;
  gemm4_tc_kernel<NT><<<static_cast<unsigned>(grid), kThreads, C::kSmem, s>>>(tm_codes, tm_x, qw.scale, qw.zero, y,
                                                                              m, N, KG, items, status);
  return launch_check("cq_dequant_gemm");
}

}  // namespace

bool gemm_tc_eligible(const cq_qweight &qw, cq_dtype xdt, int m) {
  return qw.bits == nullptr && qw.residual == nullptr && xdt == CQ_BF16 && m >= 16 && qw.rows > 0 && qw.cols > 0;
}

// the workspace holds the kernel's status word (non-zero if a wait timed out)
size_t gemm_tc_workspace(int64_t, int64_t, int) { return 16; }

cq_status launch_gemm_tc(const cq_qweight &qw, const void *x, int m, float *y, void *ws, size_t, cudaStream_t s) {
  const int64_t N = qw.rows;
  uint32_t *status = static_cast<uint32_t *>(ws);
  cq_status st = cuda_check(cudaMemsetAsync(status, 0, sizeof(uint32_t), s), "cq_dequant_gemm: clear status");
  if (st != CQ_OK) return st;
  st = cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * static_cast<size_t>(m) * N, s), "cq_dequant_gemm: zero y");
  if (st != CQ_OK) return st;
  // the batch in slices of at most 64 columns (the epilogue keeps one fp32 sum per column
  // in registers; 64 of them fit without spilling)
  for (int i0 = 0; i0 < m; i0 += 64) {
    const int mi = m - i0 < 64 ? m - i0 : 64;
    const void *xi = static_cast<const uint16_t *>(x) + static_cast<int64_t>(i0) * qw.cols;
    float *yi = y + static_cast<int64_t>(i0) * N;
    if (mi <= 16) st = launch_nt<16>(qw, xi, mi, yi, status, s);
    else if (mi <= 32) st = launch_nt<32>(qw, xi, mi, yi, status, s);
    else st = launch_nt<64>(qw, xi, mi, yi, status, s);
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

constexpr size_t kStaticScratchBytes = 4096;
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
                                            cq_stream_t stream) {
  using namespace cq;
  const char *fn = "cq_dequant_gemm_static";
  void *scratch = nullptr;
  cq_status st = static_scratch(&scratch);
  if (st != CQ_OK) return st;
  if (qw && x_dtype == CQ_BF16 && m >= 16 && gemm_tc_eligible(*qw, x_dtype, m)) {
    const size_t need = gemm_tc_workspace(qw->rows, qw->cols, m);
    if (need > kStaticScratchBytes)
      return fail(CQ_ERR_RANGE, "%s: this shape needs %zu bytes of scratch, the static buffer holds %zu", fn, need,
                  kStaticScratchBytes);
  }
  // the regular entry point does the validation and dispatch; the scratch is the static array
  return cq_dequant_gemm(qw, x, x_dtype, m, y, scratch, kStaticScratchBytes, stream);
}
