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
//  * gemv_generic: any format (per-group widths), fp32 or bf16 x, optional residual; one
//    warp per row, fp32 CUDA-core math. Used for the small fp32-activation cases and for
//    residual-carrying weights.
#include "cq_internal.cuh"

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
constexpr int kChunk = 8;                      // groups per register batch and warp

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

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::); }

// 16 consecutive bf16 activations (columns c..c+15) -> the 8 B-fragment registers in the
// order the codes are fed: pairs (0,4) (1,5) (2,6) (3,7) (8,12) (9,13) (10,14) (11,15)
__device__ __forceinline__ void x_fragments(const __nv_bfloat16 *p, uint32_t b[8]) {
  const uint4 lo = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint4 hi = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
  b[0] = __byte_perm(lo.x, lo.z, 0x5410); b[1] = __byte_perm(lo.x, lo.z, 0x7632);
  b[2] = __byte_perm(lo.y, lo.w, 0x5410); b[3] = __byte_perm(lo.y, lo.w, 0x7632);
  b[4] = __byte_perm(hi.x, hi.z, 0x5410); b[5] = __byte_perm(hi.x, hi.z, 0x7632);
  b[6] = __byte_perm(hi.y, hi.w, 0x5410); b[7] = __byte_perm(hi.y, hi.w, 0x7632);
}

template <int W>
__global__ void __launch_bounds__(W * 32)
gemv4_mma_kernel(const uint8_t *__restrict__ plane4, const uint16_t *__restrict__ scale,
                 const uint8_t *__restrict__ zero, const __nv_bfloat16 *__restrict__ x, int m,
                 int64_t N, int64_t K, float *__restrict__ y) {
  __shared__ float red[W][kTileRows][8];
  pdl_launch_dependents();
  const int KG = static_cast<int>(K >> 6);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t tile = blockIdx.x;
  const int64_t r0 = tile * kTileRows + gid, r1 = r0 + 8;
  const int64_t lr0 = r0 < N ? r0 : N - 1, lr1 = r1 < N ? r1 : N - 1;
  const int64_t half_k = K >> 1;
  const int per = (KG + W - 1) / W;
  const int g_begin = min(warp * per, KG), g_end = min(g_begin + per, KG);
  const uint8_t *row0 = plane4 + lr0 * half_k + tig * 8;
  const uint8_t *row1 = plane4 + lr1 * half_k + tig * 8;
  const uint16_t *srow0 = scale + lr0 * KG, *srow1 = scale + lr1 * KG;
  const uint8_t *zrow0 = zero + lr0 * KG, *zrow1 = zero + lr1 * KG;
  const bool has_x = gid < m;
  const __nv_bfloat16 *xrow = x + static_cast<int64_t>(has_x ? gid : 0) * K + tig * 16;
  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};   // bf16 1.0

  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  bool waited = false;
  for (int c0 = g_begin; c0 < g_end; c0 += kChunk) {
    const int nc = min(kChunk, g_end - c0);
    uint2 a0[kChunk], a1[kChunk];
    float s0[kChunk], s1[kChunk], zc0[kChunk], zc1[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      if (j < nc) {
        const int gk = c0 + j;
        a0[j] = __ldcs(reinterpret_cast<const uint2 *>(row0 + gk * 32));
        a1[j] = __ldcs(reinterpret_cast<const uint2 *>(row1 + gk * 32));
        s0[j] = f16_bits_to_f32(__ldg(srow0 + gk));
        s1[j] = f16_bits_to_f32(__ldg(srow1 + gk));
        zc0[j] = 128.0f + static_cast<float>(__ldg(zrow0 + gk));
        zc1[j] = 128.0f + static_cast<float>(__ldg(zrow1 + gk));
      }
    }
    if (!waited) {
      pdl_wait();        // x may be the output of the previous kernel in the stream
      waited = true;
    }
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      if (j < nc) {
        const int gk = c0 + j;
        uint32_t bx[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (has_x) x_fragments(xrow + gk * 64, bx);
        float p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float xs[4] = {0.0f, 0.0f, 0.0f, 0.0f};     // per-column sums of x over the group
        const uint32_t w0[2] = {a0[j].x, a0[j].y}, w1[2] = {a1[j].x, a1[j].y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t A0[4] = {nib_pair(w0[h]), nib_pair(w1[h]), nib_pair(w0[h] >> 4), nib_pair(w1[h] >> 4)};
          mma_bf16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
          mma_bf16_16816(xs, ones, bx[4 * h + 0], bx[4 * h + 1]);
          const uint32_t A1[4] = {nib_pair(w0[h] >> 8), nib_pair(w1[h] >> 8), nib_pair(w0[h] >> 12), nib_pair(w1[h] >> 12)};
          mma_bf16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
          mma_bf16_16816(xs, ones, bx[4 * h + 2], bx[4 * h + 3]);
        }
        // sum_k (q - z) x = sum_k (128 + q) x - (128 + z) sum_k x, in fp32
        acc[0] = fmaf(s0[j], fmaf(-zc0[j], xs[0], p[0]), acc[0]);
        acc[1] = fmaf(s0[j], fmaf(-zc0[j], xs[1], p[1]), acc[1]);
        acc[2] = fmaf(s1[j], fmaf(-zc1[j], xs[2], p[2]), acc[2]);
        acc[3] = fmaf(s1[j], fmaf(-zc1[j], xs[3], p[3]), acc[3]);
      }
    }
  }
  if (!waited) pdl_wait();
  red[warp][gid][2 * tig] = acc[0];
  red[warp][gid][2 * tig + 1] = acc[1];
  red[warp][gid + 8][2 * tig] = acc[2];
  red[warp][gid + 8][2 * tig + 1] = acc[3];
  __syncthreads();
  if (threadIdx.x < kTileRows * 8) {
    const int row = threadIdx.x & 15, col = threadIdx.x >> 4;
    const int64_t r = tile * kTileRows + row;
    if (col < m && r < N) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < W; ++w) v += red[w][row][col];
      y[static_cast<int64_t>(col) * N + r] = v;
    }
  }
}

template <int W>
cudaError_t launch_gemv4(const cq_qweight &qw, const void *x, int m, float *y, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((qw.rows + kTileRows - 1) / kTileRows));
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv4_mma_kernel<W>, qw.plane[2], qw.scale, qw.zero,
                            static_cast<const __nv_bfloat16 *>(x), m, qw.rows, qw.cols, y);
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
    // warps per tile: enough K-slices to keep ~8 groups (4 KiB of codes) per warp in flight
    const int64_t KG = K >> 6;
    (void)KG;
    const cudaError_t e = launch_gemv4<8>(qw, x, m, y, s);
    return cuda_check(e, "cq_dequant_gemv");
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
