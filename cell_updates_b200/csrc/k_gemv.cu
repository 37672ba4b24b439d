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
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

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

// ---- the kernel -------------------------------------------------------------------------------
// One CTA per 16-row tile and the whole K range, 8 warps. Chunks of 4 groups (128 bytes per
// row) are dealt to the warps round-robin, so at any moment a CTA's loads cover ~1 KiB of
// each of its 16 rows: long DRAM runs with few rows in flight (measured on this part: ~6 TB/s
// for 16-row tiles with >= 512-byte runs, against ~3 TB/s when every row of the matrix is in
// flight at once). Each warp double-buffers its codes, scales and zero points in registers:
// the next chunk's loads are issued before the current one is computed. The activations are
// staged once per CTA in shared memory, in the order the codes are fed to the MMA, together
// with their exact per-group sums; when they do not fit, each warp reads them from L1 and
// takes the sums from one more MMA with an all-ones operand. Warps meet in shared memory at
// the end, so every output is written once (no atomics, no zero-fill, fixed order). Codes
// and scales do not depend on earlier kernels and are requested before the programmatic-
// dependent-launch wait; activations are read, and y written, only after it.
constexpr int kWarps = 8;
constexpr int kGemvThreads = 32 * kWarps;
constexpr int kCG = 4;                                  // groups per chunk
constexpr int kXStageMax = 64 * 1024;                   // staged activations + sums, at most
constexpr int kRedBytes = kWarps * kTileRows * 8 * 4;

// staged activations: m rows of K bf16 in fragment order, row pitch padded by 16 bytes so the
// rows a warp reads fall in different banks, followed by fp32 sums [KG][8]
__host__ __device__ constexpr int64_t xstage_pitch(int64_t K) { return K * 2 + 16; }
__host__ __device__ constexpr int64_t xstage_bytes(int m, int64_t K) { return m * xstage_pitch(K) + (K / 64) * 32; }

struct Chunk {
  uint2 a0[kCG], a1[kCG];      // 8 code bytes per row and group for rows gid, gid+8
  uint2 s0, s1;                // 4 fp16 scales per row
  uint32_t z0, z1;             // 4 zero points per row
};

template <bool META4>
__device__ __forceinline__ void load_chunk(Chunk &ck, const uint8_t *row0, const uint8_t *row1, const uint16_t *srow0,
                                           const uint16_t *srow1, const uint8_t *zrow0, const uint8_t *zrow1, int g0,
                                           int ng) {
#pragma unroll
  for (int j = 0; j < kCG; ++j) {
    if (j < ng) {
      ck.a0[j] = __ldcs(reinterpret_cast<const uint2 *>(row0 + (g0 + j) * 32));
      ck.a1[j] = __ldcs(reinterpret_cast<const uint2 *>(row1 + (g0 + j) * 32));
    }
  }
  if (META4 && ng == kCG) {
    ck.s0 = __ldg(reinterpret_cast<const uint2 *>(srow0 + g0));
    ck.s1 = __ldg(reinterpret_cast<const uint2 *>(srow1 + g0));
    ck.z0 = __ldg(reinterpret_cast<const uint32_t *>(zrow0 + g0));
    ck.z1 = __ldg(reinterpret_cast<const uint32_t *>(zrow1 + g0));
  } else {
    uint32_t sv0[kCG], sv1[kCG], zv0[kCG], zv1[kCG];
#pragma unroll
    for (int j = 0; j < kCG; ++j) {
      sv0[j] = j < ng ? __ldg(srow0 + g0 + j) : 0u;
      sv1[j] = j < ng ? __ldg(srow1 + g0 + j) : 0u;
      zv0[j] = j < ng ? __ldg(zrow0 + g0 + j) : 0u;
      zv1[j] = j < ng ? __ldg(zrow1 + g0 + j) : 0u;
    }
    ck.s0 = make_uint2(sv0[0] | (sv0[1] << 16), sv0[2] | (sv0[3] << 16));
    ck.s1 = make_uint2(sv1[0] | (sv1[1] << 16), sv1[2] | (sv1[3] << 16));
    ck.z0 = zv0[0] | (zv0[1] << 8) | (zv0[2] << 16) | (zv0[3] << 24);
    ck.z1 = zv1[0] | (zv1[1] << 8) | (zv1[2] << 16) | (zv1[3] << 24);
  }
}

// 16 consecutive bf16 activations -> the 8 B-fragment registers in code-feeding order:
// pairs (0,4) (1,5) (2,6) (3,7) (8,12) (9,13) (10,14) (11,15)
__device__ __forceinline__ void permute16(const uint4 &lo, const uint4 &hi, uint32_t b[8]) {
  b[0] = __byte_perm(lo.x, lo.z, 0x5410); b[1] = __byte_perm(lo.x, lo.z, 0x7632);
  b[2] = __byte_perm(lo.y, lo.w, 0x5410); b[3] = __byte_perm(lo.y, lo.w, 0x7632);
  b[4] = __byte_perm(hi.x, hi.z, 0x5410); b[5] = __byte_perm(hi.x, hi.z, 0x7632);
  b[6] = __byte_perm(hi.y, hi.w, 0x5410); b[7] = __byte_perm(hi.y, hi.w, 0x7632);
}

template <bool META4, bool XS>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv4_kernel(const uint8_t *__restrict__ plane4, const uint16_t *__restrict__ scale,
             const uint8_t *__restrict__ zero, const __nv_bfloat16 *__restrict__ x, int m, int64_t N,
             int64_t K, float *__restrict__ y) {
  extern __shared__ __align__(16) uint8_t smem[];
  float (*red)[kTileRows][8] = reinterpret_cast<float (*)[kTileRows][8]>(smem);
  uint8_t *xst = smem + kRedBytes;
  pdl_launch_dependents();
  const int KG = static_cast<int>(K >> 6);
  const int n_chunks = (KG + kCG - 1) / kCG;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTileRows;
  const int64_t lr0 = row0 + gid < N ? row0 + gid : N - 1;
  const int64_t lr1 = row0 + gid + 8 < N ? row0 + gid + 8 : N - 1;
  const int64_t half_k = K >> 1;
  const uint8_t *crow0 = plane4 + lr0 * half_k + tig * 8, *crow1 = plane4 + lr1 * half_k + tig * 8;
  const uint16_t *srow0 = scale + lr0 * KG, *srow1 = scale + lr1 * KG;
  const uint8_t *zrow0 = zero + lr0 * KG, *zrow1 = zero + lr1 * KG;
  const int64_t xpitch = xstage_pitch(K);
  float *xsum = reinterpret_cast<float *>(xst + m * xpitch);          // [KG][8]
  auto chunk_range = [&](int c, int &g0, int &ng) {
    g0 = c * kCG;
    ng = KG - g0 < kCG ? KG - g0 : kCG;
  };

  // first chunk of this warp: codes and scales before the dependency wait
  Chunk cur, nxt;
  {
    int g0, ng;
    chunk_range(warp, g0, ng);
    if (warp < n_chunks) load_chunk<META4>(cur, crow0, crow1, srow0, srow1, zrow0, zrow1, g0, ng);
  }
  pdl_wait();                 // x may be the output of the previous kernel in the stream
  const bool has_x = gid < m;
  const __nv_bfloat16 *xrow = x + static_cast<int64_t>(has_x ? gid : 0) * K + tig * 16;
  if (XS) {
    // stage x: thread t owns 16-element blocks t, t + 256, ...; four lanes make one group
    const int nblk = m * (KG * 4);
    for (int b0 = 0; b0 < nblk; b0 += kGemvThreads * 4) {
      uint4 v[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u * kGemvThreads + threadIdx.x;
        if (b < nblk) {
          const int n = b / (KG * 4), kb = b - n * (KG * 4);
          const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(n) * K + kb * 16);
          v[u][0] = __ldg(src);
          v[u][1] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u * kGemvThreads + threadIdx.x;
        float sum = 0.0f;
        if (b < nblk) {
          const int n = b / (KG * 4), kb = b - n * (KG * 4);
          uint32_t f[8];
          permute16(v[u][0], v[u][1], f);
          uint4 *dst = reinterpret_cast<uint4 *>(xst + n * xpitch + kb * 32);
          dst[0] = make_uint4(f[0], f[1], f[2], f[3]);
          dst[1] = make_uint4(f[4], f[5], f[6], f[7]);
          const uint32_t w[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w, v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
        }
        // blocks 4j..4j+3 (one group) sit on lanes 4j..4j+3 of a warp (256 threads, group-aligned)
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (b < nblk && (threadIdx.x & 3) == 0) {
          const int n = b / (KG * 4), kb = b - n * (KG * 4);
          xsum[(kb >> 2) * 8 + n] = sum;
        }
      }
    }
    for (int p = threadIdx.x; p < KG * 8; p += kGemvThreads)
      if ((p & 7) >= m) xsum[p] = 0.0f;
    __syncthreads();
  }

  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};   // bf16 1.0
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int c = warp; c < n_chunks; c += kWarps) {
    int g0, ng;
    chunk_range(c, g0, ng);
    // the next chunk of this warp is requested before this one is computed
    const int cn = c + kWarps;
    if (cn < n_chunks) {
      int g0n, ngn;
      chunk_range(cn, g0n, ngn);
      load_chunk<META4>(nxt, crow0, crow1, srow0, srow1, zrow0, zrow1, g0n, ngn);
    }
#pragma unroll
    for (int j = 0; j < kCG; ++j) {
      if (j < ng) {
        const int g = g0 + j;
        uint32_t bx[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        float q[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (has_x) {
          if (XS) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(xst + gid * xpitch + (g * 64 + tig * 16) * 2);
            const uint4 lo = xp[0], hi = xp[1];
            bx[0] = lo.x; bx[1] = lo.y; bx[2] = lo.z; bx[3] = lo.w;
            bx[4] = hi.x; bx[5] = hi.y; bx[6] = hi.z; bx[7] = hi.w;
          } else {
            const uint4 *xp = reinterpret_cast<const uint4 *>(xrow + g * 64);
            permute16(__ldg(xp), __ldg(xp + 1), bx);
          }
        }
        float p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t w0[2] = {cur.a0[j].x, cur.a0[j].y}, w1[2] = {cur.a1[j].x, cur.a1[j].y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t A0[4] = {nib_pair(w0[h]), nib_pair(w1[h]), nib_pair(w0[h] >> 4), nib_pair(w1[h] >> 4)};
          mma_bf16_16816(p, A0, bx[4 * h + 0], bx[4 * h + 1]);
          if (!XS) mma_bf16_16816(q, ones, bx[4 * h + 0], bx[4 * h + 1]);
          const uint32_t A1[4] = {nib_pair(w0[h] >> 8), nib_pair(w1[h] >> 8), nib_pair(w0[h] >> 12),
                                  nib_pair(w1[h] >> 12)};
          mma_bf16_16816(p, A1, bx[4 * h + 2], bx[4 * h + 3]);
          if (!XS) mma_bf16_16816(q, ones, bx[4 * h + 2], bx[4 * h + 3]);
        }
        if (XS) {
          const float2 xs2 = *reinterpret_cast<const float2 *>(xsum + g * 8 + 2 * tig);
          q[0] = xs2.x; q[1] = xs2.y; q[2] = xs2.x; q[3] = xs2.y;
        }
        const uint32_t sw0 = (j < 2 ? cur.s0.x : cur.s0.y) >> (16 * (j & 1));
        const uint32_t sw1 = (j < 2 ? cur.s1.x : cur.s1.y) >> (16 * (j & 1));
        const float sc0 = f16_bits_to_f32(static_cast<uint16_t>(sw0));
        const float sc1 = f16_bits_to_f32(static_cast<uint16_t>(sw1));
        const float zc0 = 128.0f + static_cast<float>((cur.z0 >> (8 * j)) & 0xFFu);
        const float zc1 = 128.0f + static_cast<float>((cur.z1 >> (8 * j)) & 0xFFu);
        // sum_k (q - z) x = sum_k (128 + q) x - (128 + z) sum_k x, in fp32
        acc[0] = fmaf(sc0, fmaf(-zc0, q[0], p[0]), acc[0]);
        acc[1] = fmaf(sc0, fmaf(-zc0, q[1], p[1]), acc[1]);
        acc[2] = fmaf(sc1, fmaf(-zc1, q[2], p[2]), acc[2]);
        acc[3] = fmaf(sc1, fmaf(-zc1, q[3], p[3]), acc[3]);
      }
    }
    cur = nxt;
  }
  red[warp][gid][2 * tig] = acc[0];
  red[warp][gid][2 * tig + 1] = acc[1];
  red[warp][gid + 8][2 * tig] = acc[2];
  red[warp][gid + 8][2 * tig + 1] = acc[3];
  __syncthreads();
  if (threadIdx.x < kTileRows * 8) {
    const int row = threadIdx.x & 15, col = threadIdx.x >> 4;
    const int64_t r = row0 + row;
    if (col < m && r < N) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[w][row][col];
      y[static_cast<int64_t>(col) * N + r] = v;
    }
  }
}

template <bool META4, bool XS>
cq_status launch_gemv4(const cq_qweight &qw, const void *x, int m, float *y, cudaStream_t s) {
  const int smem = kRedBytes + (XS ? static_cast<int>(xstage_bytes(m, qw.cols)) : 0);
  cq_status st = cuda_check(cudaFuncSetAttribute(gemv4_kernel<META4, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem), "cq_dequant_gemv: shared memory attribute");
  if (st != CQ_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((qw.rows + kTileRows - 1) / kTileRows));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, gemv4_kernel<META4, XS>, qw.plane[2], qw.scale, qw.zero,
                                       static_cast<const __nv_bfloat16 *>(x), m, qw.rows, qw.cols, y),
                    "cq_dequant_gemv");
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
    // 16-byte scale and 8-byte zero vectors need a row pitch of a multiple of 8 groups
    const int64_t KG = K >> 6;
    // 8-byte scale and 4-byte zero vectors need a row pitch of a multiple of 4 groups
    const bool meta4 = (KG % 4 == 0) && aligned8(qw.scale) && (reinterpret_cast<uintptr_t>(qw.zero) & 3u) == 0;
    // small activation sets (decode) are staged once per CTA in shared memory
    const bool xs = xstage_bytes(m, K) <= kXStageMax;
    if (meta4) return xs ? launch_gemv4<true, true>(qw, x, m, y, s) : launch_gemv4<true, false>(qw, x, m, y, s);
    return xs ? launch_gemv4<false, true>(qw, x, m, y, s) : launch_gemv4<false, false>(qw, x, m, y, s);
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
