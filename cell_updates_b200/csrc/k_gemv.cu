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
//    in fp32. The contraction over k is a sum, so the kernel may pair any code with any
//    activation as long as both operands use the same order: each lane feeds the MMA with
//    the 16 codes it loaded contiguously (one 8-byte load per row and group), and the
//    activations are staged once per CTA in shared memory in that same order, together
//    with their per-group sums.
//  * gemv_generic: any format (per-group widths), fp32 or bf16 x, optional residual; one
//    warp per row, fp32 CUDA-core math. Used for the small fp32-activation cases and for
//    residual-carrying weights.
#include "cq_internal.cuh"

namespace cq {
namespace {

// ------------------------------------------------------------------------------------
// tensor-core path
// ------------------------------------------------------------------------------------
constexpr int kMmaWarps = 4;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kKCH = 8;                       // groups per k-chunk (512 columns)
constexpr int kTilesPerWarp = 1;              // 16-row tiles per warp
constexpr int kTilesPerCta = kMmaWarps * kTilesPerWarp;
constexpr int kXRowBytes = kKCH * 64 * 2 + 16;   // padded: conflict-free 16-byte fragment loads

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// nibbles i and i+4 of w (i = 0..3 after the shift) -> bf16 pair (128 + q_i, 128 + q_{i+4})
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) {
  uint32_t out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(w), "r"(0x000F000Fu), "r"(0x43004300u));
  return out;   // (w & 0x000F000F) | 0x43004300
}

// position of column offset o (0..15 inside a lane's 16 columns) in fragment order:
// pairs (0,4) (1,5) (2,6) (3,7) (8,12) (9,13) (10,14) (11,15)
__device__ __forceinline__ int frag_pos(int o) { return (o & 8) + 2 * (o & 3) + ((o >> 2) & 1); }

__global__ void __launch_bounds__(kMmaThreads)
gemv4_mma_kernel(const uint8_t *__restrict__ plane4, const uint16_t *__restrict__ scale,
                 const uint8_t *__restrict__ zero, const __nv_bfloat16 *__restrict__ x, int m,
                 int64_t N, int64_t K, float *__restrict__ y) {
  __shared__ __align__(16) uint8_t xs[8 * kXRowBytes];   // [n][fragment-ordered columns]
  __shared__ __align__(16) float xsum[kKCH][8];            // per group, per batch column
  const int KG = static_cast<int>(K >> 6);
  const int kc = blockIdx.x;
  const int gk0 = kc * kKCH;
  const int ng = min(kKCH, KG - gk0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // ---- stage x[:, chunk] in fragment order, plus per-group sums -------------------------
  for (int p = warp; p < 8 * kKCH; p += kMmaWarps) {
    const int n = p / kKCH, gl = p % kKCH;
    float v0 = 0.0f, v1 = 0.0f;
    uint32_t raw = 0;
    if (n < m && gl < ng) {
      raw = __ldg(reinterpret_cast<const uint32_t *>(x + static_cast<int64_t>(n) * K + (gk0 + gl) * 64) + lane);
      v0 = __uint_as_float(raw << 16);
      v1 = __uint_as_float(raw & 0xFFFF0000u);
    }
    const int c0 = 2 * lane;                 // columns c0, c0+1 of this group
    const int blk = c0 >> 4, o0 = c0 & 15;
    uint16_t *row = reinterpret_cast<uint16_t *>(xs + n * kXRowBytes) + gl * 64 + blk * 16;
    row[frag_pos(o0)] = static_cast<uint16_t>(raw & 0xFFFFu);
    row[frag_pos(o0 + 1)] = static_cast<uint16_t>(raw >> 16);
    float sum = v0 + v1;
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) xsum[gl][n] = sum;
  }
  __syncthreads();

  const int gid = lane >> 2, tig = lane & 3;
  const int64_t half_k = K >> 1;
  for (int t = 0; t < kTilesPerWarp; ++t) {
    const int64_t tile = static_cast<int64_t>(blockIdx.y) * kTilesPerCta + warp * kTilesPerWarp + t;
    const int64_t r0 = tile * 16 + gid, r1 = r0 + 8;
    if (tile * 16 >= N) break;
    const int64_t lr0 = r0 < N ? r0 : N - 1, lr1 = r1 < N ? r1 : N - 1;
    // issue every weight load of the chunk first (16 bytes per row and group per lane)
    uint2 a0[kKCH], a1[kKCH];
    float s0[kKCH], s1[kKCH], zc0[kKCH], zc1[kKCH];
#pragma unroll
    for (int j = 0; j < kKCH; ++j) {
      if (j < ng) {
        const int64_t gk = gk0 + j;
        a0[j] = __ldcs(reinterpret_cast<const uint2 *>(plane4 + lr0 * half_k + gk * 32 + tig * 8));
        a1[j] = __ldcs(reinterpret_cast<const uint2 *>(plane4 + lr1 * half_k + gk * 32 + tig * 8));
        s0[j] = f16_bits_to_f32(__ldg(scale + lr0 * KG + gk));
        s1[j] = f16_bits_to_f32(__ldg(scale + lr1 * KG + gk));
        zc0[j] = 128.0f + static_cast<float>(__ldg(zero + lr0 * KG + gk));
        zc1[j] = 128.0f + static_cast<float>(__ldg(zero + lr1 * KG + gk));
      }
    }
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < kKCH; ++j) {
      if (j < ng) {
        const uint4 *bp = reinterpret_cast<const uint4 *>(xs + gid * kXRowBytes + (j * 64 + tig * 16) * 2);
        const uint4 bA = bp[0], bB = bp[1];
        const uint32_t bx[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
        float p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t w0[2] = {a0[j].x, a0[j].y}, w1[2] = {a1[j].x, a1[j].y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // codes k..k+7 of row r0 in w0[h], of row r1 in w1[h]; two MMAs per word
          const uint32_t A0[4] = {nib_pair(w0[h]), nib_pair(w1[h]), nib_pair(w0[h] >> 4), nib_pair(w1[h] >> 4)};
          mma_bf16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
          const uint32_t A1[4] = {nib_pair(w0[h] >> 8), nib_pair(w1[h] >> 8), nib_pair(w0[h] >> 12), nib_pair(w1[h] >> 12)};
          mma_bf16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
        }
        const float2 X = *reinterpret_cast<const float2 *>(&xsum[j][2 * tig]);
        acc[0] = fmaf(s0[j], fmaf(-zc0[j], X.x, p[0]), acc[0]);
        acc[1] = fmaf(s0[j], fmaf(-zc0[j], X.y, p[1]), acc[1]);
        acc[2] = fmaf(s1[j], fmaf(-zc1[j], X.x, p[2]), acc[2]);
        acc[3] = fmaf(s1[j], fmaf(-zc1[j], X.y, p[3]), acc[3]);
      }
    }
    const int c0 = 2 * tig, c1 = c0 + 1;
    if (r0 < N) {
      if (c0 < m) atomicAdd(y + static_cast<int64_t>(c0) * N + r0, acc[0]);
      if (c1 < m) atomicAdd(y + static_cast<int64_t>(c1) * N + r0, acc[1]);
    }
    if (r1 < N) {
      if (c0 < m) atomicAdd(y + static_cast<int64_t>(c0) * N + r1, acc[2]);
      if (c1 < m) atomicAdd(y + static_cast<int64_t>(c1) * N + r1, acc[3]);
    }
  }
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
    cq_status st = cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * m * N, s), "cq_dequant_gemv: zero y");
    if (st != CQ_OK) return st;
    const int64_t KG = K >> 6;
    dim3 grid(static_cast<unsigned>((KG + kKCH - 1) / kKCH),
              static_cast<unsigned>((N + 16 * kTilesPerCta - 1) / (16 * kTilesPerCta)));
    gemv4_mma_kernel<<<grid, kMmaThreads, 0, s>>>(qw.plane[2], qw.scale, qw.zero,
                                                  static_cast<const __nv_bfloat16 *>(x), m, N, K, y);
    return launch_check("cq_dequant_gemv");
  }
  const int64_t need = (N + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int blocks = static_cast<int>(need < cap ? need : cap);
  const int rk = qw.residual == nullptr ? 0 : (qw.residual_dtype == CQ_BF16 ? 2 : 1);
  if (xdt == CQ_BF16) {
    if (rk == 0) launch_generic<true, 0>(qw, x, m, y, blocks, s);
    else if (rk == 1) launch_generic<true, 1>(qw, x, m, y, blocks, s);
    else launch_generic<true, 2>(qw, x, m, y, blocks, s);
  } else {
    if (rk == 0) launch_generic<false, 0>(qw, x, m, y, blocks, s);
    else if (rk == 1) launch_generic<false, 1>(qw, x, m, y, blocks, s);
    else launch_generic<false, 2>(qw, x, m, y, blocks, s);
  }
  return launch_check("cq_dequant_gemv");
}

}  // namespace cq
