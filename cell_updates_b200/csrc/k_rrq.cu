// k_rrq.cu -- dequantize-and-multiply over per-group-width weights and over stacks of stages.
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence Without
// Changing the File They Ship", abstract: per-group bit-widths in bit-packed storage, served by a
// fused dequantize-and-multiply kernel for memory-bound decode. [RRQ] the listing page
// thelatestinai.com/papers/2512.18934, "Recurrent Residual Quantization" abstract: the weights
// are a low-bit base plus a sequence of quantized residual corrections (2-bit round-to-nearest
// stages stacked to 4, 6 and 8 bits), so one artifact serves several precisions; a model of
// 2(J+1) bits uses the first J+1 stages (made by cq_rrq_stage, k_quantize.cu). Two kernels serve
// both, for a list of stages of one shape, each fixed-4 or with a per-group width map:
//     y[i, n] = sum_j sum_g s_j[n, g] * sum_{k in g} (q_j[n, k] - z_j[n, g]) * x[i, k]
// (a single VBQ matrix is a list of one stage), chosen by batch size on measurement:
//
//  * batch 1, gemv_vbq1_kernel (CUDA cores): a warp per row lists the row's groups by width and
//    decodes one width per pass with constant masks (below, before the kernel).
//  * batch 2..8, gemv_vb_kernel (tensor cores, mma.sync m16n8k16, bf16 operands, fp32
//    accumulation): a warp takes 16 rows of one group at a time; A is the 16 x 64 block of
//    q - z, B the group's 64 activations of up to 8 batch rows. q - z is an integer in
//    [-255, 255], exact in bf16, so every product is exact; the group's four MMAs start from zero
//    and the group result is scaled by s (fp32) and added to the running sums, so the only
//    rounding is fp32 accumulation (fp32 activations enter as two bf16 parts, hi + lo, which
//    leaves |x - hi - lo| <= 2^-17 |x|). The contraction over k is a sum, so codes and
//    activations may be paired in any order both operands share: lane (gid, tig) feeds the 16
//    codes 16 tig .. 16 tig + 15 of rows gid and gid + 8, as the pairs (t, t + 8), and loads the
//    matching 16 activations of batch row gid. For widths 1, 2 and 4 the bf16 pair
//    (128 + q_t, 128 + q_{t+8}) comes from the packed bytes with one shift and one LOP3 whatever
//    the width (the width only sets the shift step and the mask), and one bf16x2 subtraction of
//    128 + z gives q - z; so rows of different widths in one warp run the same instructions.
//    8-bit groups (128 + q is not exact in bf16 past q = 127) go through fp32:
//    (2^23 + q) - (2^23 + z), exact, then packed to bf16.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kTileRows = 16;
constexpr int kPerLaunch = 4;         // stages per launch (their pointers live in the parameter space)

struct StageSet {
  const uint8_t *bits[kPerLaunch];
  const uint32_t *offset[kPerLaunch];
  const uint8_t *plane[kPerLaunch][4];
  const uint16_t *scale[kPerLaunch];
  const uint8_t *zero[kPerLaunch];
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<const uint32_t *>(&v); }

// (w & mask) | magic in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t w, uint32_t mask, uint32_t magic) {
  uint32_t out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(out) : "r"(w), "r"(mask), "r"(magic));
  return out;
}

// where a group's bytes are: width (0 for a width outside {1, 2, 4, 8}) and raw byte offset
struct RowMeta {
  int b;
  uint32_t off;
};
// what the MMA step needs of one row and group: the lane's packed code bytes, width, scale, zero
struct RowCodes {
  uint4 w;
  float s;
  uint32_t z;
  int b;
};

__device__ __forceinline__ RowMeta load_meta(const StageSet &ss, int j, int64_t gabs) {
  RowMeta m;
  if (ss.bits[j]) {
    const int b = __ldg(ss.bits[j] + gabs);
    m.b = width_ok(b) ? b : 0;
    m.off = __ldg(ss.offset[j] + gabs);
  } else {
    m.b = 4;
    m.off = static_cast<uint32_t>(gabs) * 32u;   // unused: the fixed-4 address is formed from gabs
  }
  return m;
}

// the lane's share of the group's packed bytes: for b <= 4 the aligned 8-byte word at byte
// (2 b tig) & ~7 of the group (in w.x, w.y), for b = 8 the 16 bytes at 16 tig
__device__ __forceinline__ RowCodes load_codes(const StageSet &ss, int j, int64_t gabs, const RowMeta &m, int tig) {
  RowCodes c;
  c.b = m.b;
  c.w = make_uint4(0u, 0u, 0u, 0u);
  // debug build: an offset off its 8 b grid, or a rank above the group's own index (a rank
  // counts earlier groups of the same width), is recorded (and the latter's load skipped)
  (void)CQ_CHECK(!ss.bits[j] || !m.b || (m.off & (8u * m.b - 1u)) == 0u, 0x0701u);
  if (m.b && CQ_CHECK(!ss.bits[j] || static_cast<int64_t>(m.off / (8u * m.b)) <= gabs, 0x0702u)) {
    const uint8_t *src;
    if (ss.bits[j]) {
      // offsets are multiples of 8 b by construction; the mask keeps a damaged map aligned
      src = ss.plane[j][width_slot(m.b)] + (m.off & ~static_cast<uint32_t>(8 * m.b - 1));
    } else {
      src = ss.plane[j][2] + gabs * 32;
    }
    if (m.b == 8) {
      c.w = __ldg(reinterpret_cast<const uint4 *>(src + 16 * tig));
    } else {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src + ((2 * m.b * tig) & ~7)));
      c.w.x = v.x;
      c.w.y = v.y;
    }
  }
  c.s = f16_bits_to_f32(__ldg(ss.scale[j] + gabs));
  c.z = __ldg(ss.zero[j] + gabs);
  return c;
}

// The A-operand share of one row: codes 16 tig .. 16 tig + 15 of the group, as eight bf16 pairs
// (q_t - z, q_{t+8} - z). Width 0 (outside {1, 2, 4, 8}) gives zeros.
__device__ __forceinline__ void row_operand(const RowCodes &c, int tig, uint32_t (&r)[8]) {
  const int b = c.b;
  if (b == 1 || b == 2 || b == 4) {
    uint32_t v0, v1;
    if (b == 4) {                       // codes 0-3 | 8-11 and 4-7 | 12-15 as 16-bit halves
      v0 = __byte_perm(c.w.x, c.w.y, 0x5410);
      v1 = __byte_perm(c.w.x, c.w.y, 0x7632);
    } else if (b == 2) {                // bytes 4 tig .. 4 tig + 3: codes 0-7 | 8-15
      v0 = v1 = (tig & 1) ? c.w.y : c.w.x;
    } else {                            // bytes 2 tig, 2 tig + 1 moved to bits 0-7 and 16-23
      const uint32_t u = (tig >> 1) ? c.w.y : c.w.x;
      const uint32_t o = 2u * (tig & 1);
      v0 = v1 = __byte_perm(u, 0u, 0x4040u | o | ((o + 1u) << 8));
    }
    const uint32_t mask = (b == 4 ? 0x000F000Fu : (b == 2 ? 0x00030003u : 0x00010001u));
    const uint32_t adj = b == 4 ? 16u : 0u;     // codes 4-7 of a 4-bit group restart at bit 0 of v1
    const uint32_t zz = (0x4300u | c.z) * 0x00010001u;   // bf16 (128 + z) twice
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t sh = t < 4 ? static_cast<uint32_t>(t * b) : static_cast<uint32_t>(t * b) - adj;
      const uint32_t p = and_or((t < 4 ? v0 : v1) >> sh, mask, 0x43004300u);   // 128 + q, exact
      r[t] = bf2_bits(__hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p),
                              *reinterpret_cast<const __nv_bfloat162 *>(&zz)));
    }
  } else if (b == 8) {
    const float zf = 8388608.0f + static_cast<float>(c.z);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t sel = 0x7440u | static_cast<uint32_t>(t & 3);   // [byte t & 3, 0, 0, 0x4B]
      const float f0 = __uint_as_float(__byte_perm(t < 4 ? c.w.x : c.w.y, 0x4B000000u, sel)) - zf;
      const float f1 = __uint_as_float(__byte_perm(t < 4 ? c.w.z : c.w.w, 0x4B000000u, sel)) - zf;
      r[t] = bf2_bits(__floats2bfloat162_rn(f0, f1));
    }
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) r[t] = 0u;
  }
}

// the same for a width B known to the whole warp: constant shifts and masks
template <int B>
__device__ __forceinline__ void row_operand_w(const RowCodes &c, int tig, uint32_t (&r)[8]) {
  uint32_t v0, v1;
  if (B == 4) {
    v0 = __byte_perm(c.w.x, c.w.y, 0x5410);
    v1 = __byte_perm(c.w.x, c.w.y, 0x7632);
  } else if (B == 2) {
    v0 = v1 = (tig & 1) ? c.w.y : c.w.x;
  } else {
    const uint32_t u = (tig >> 1) ? c.w.y : c.w.x;
    v0 = v1 = __byte_perm(u, 0u, (tig & 1) ? 0x4342u : 0x4140u);
  }
  constexpr uint32_t kMask = B == 4 ? 0x000F000Fu : (B == 2 ? 0x00030003u : 0x00010001u);
  const uint32_t zz = (0x4300u | c.z) * 0x00010001u;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int sh = B == 4 ? 4 * (t & 3) : t * B;
    const uint32_t p = and_or((t < 4 ? v0 : v1) >> sh, kMask, 0x43004300u);
    r[t] = bf2_bits(__hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p),
                            *reinterpret_cast<const __nv_bfloat162 *>(&zz)));
  }
}

// both rows' operands: one specialised path when every lane of the warp holds the same width
// in both rows (a stage of one width, or a uniform run of a width map), else the generic one
__device__ __forceinline__ void rows_operand(const RowCodes &cl, const RowCodes &ch, int tig, uint32_t (&alo)[8],
                                             uint32_t (&ahi)[8]) {
  const int b0 = __shfl_sync(0xffffffffu, cl.b, 0);
  const bool uni = __all_sync(0xffffffffu, cl.b == b0 && ch.b == b0);
  if (uni && b0 == 2) {
    row_operand_w<2>(cl, tig, alo);
    row_operand_w<2>(ch, tig, ahi);
  } else if (uni && b0 == 4) {
    row_operand_w<4>(cl, tig, alo);
    row_operand_w<4>(ch, tig, ahi);
  } else if (uni && b0 == 1) {
    row_operand_w<1>(cl, tig, alo);
    row_operand_w<1>(ch, tig, ahi);
  } else {
    row_operand(cl, tig, alo);
    row_operand(ch, tig, ahi);
  }
}

// batch row gid's activations 16 tig .. 16 tig + 15 of group g (zeros past the batch)
template <bool XF32>
struct XFrag {
  uint4 v[XF32 ? 4 : 2];
};
template <bool XF32>
__device__ __forceinline__ XFrag<XF32> load_x(const void *x, int64_t xi, bool has_x) {
  XFrag<XF32> f;
#pragma unroll
  for (int i = 0; i < (XF32 ? 4 : 2); ++i) f.v[i] = make_uint4(0u, 0u, 0u, 0u);
  if (has_x) {
    const uint4 *p = XF32 ? reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + xi)
                          : reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + xi);
#pragma unroll
    for (int i = 0; i < (XF32 ? 4 : 2); ++i) f.v[i] = __ldg(p + i);
  }
  return f;
}

// B operand from the fragment, as pairs (t, t + 8): register 2 c feeds MMA c's b0 (codes 2c,
// 2c + 8), register 2 c + 1 its b1 (codes 2c + 1, 2c + 9); fp32 activations as hi + lo parts
template <bool XF32>
__device__ __forceinline__ void b_operand(const XFrag<XF32> &f, uint32_t (&bh)[8], uint32_t (&bl)[8]) {
  if (XF32) {
    float xv[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xv[4 * i] = __uint_as_float(f.v[i].x);
      xv[4 * i + 1] = __uint_as_float(f.v[i].y);
      xv[4 * i + 2] = __uint_as_float(f.v[i].z);
      xv[4 * i + 3] = __uint_as_float(f.v[i].w);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float a = xv[2 * c + h], b = xv[2 * c + h + 8];
        const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
        bh[2 * c + h] = bf2_bits(hi);
        bl[2 * c + h] = bf2_bits(__floats2bfloat162_rn(a - __low2float(hi), b - __high2float(hi)));
      }
    }
  } else {
    const uint32_t lw[4] = {f.v[0].x, f.v[0].y, f.v[0].z, f.v[0].w};
    const uint32_t hw[4] = {f.v[1].x, f.v[1].y, f.v[1].z, f.v[1].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      bh[2 * c] = __byte_perm(lw[c], hw[c], 0x5410);
      bh[2 * c + 1] = __byte_perm(lw[c], hw[c], 0x7632);
      bl[2 * c] = bl[2 * c + 1] = 0u;
    }
  }
}

// CTA = one 16-row tile at a time (grid-stride); its warps split the tile's groups into
// contiguous runs and meet in shared memory, where the partial sums are added in warp order
// (deterministic, no atomics). A warp walks its (stage, group) items as a software pipeline:
// the widths and offsets of item i + 2 and the code bytes, scales, zero points and activations
// of item i + 1 are in flight while item i is multiplied, so the offset -> code dependence of
// the packed format costs no round trip of its own.
template <bool XF32>
__global__ void __launch_bounds__(kThreads, 1)
gemv_vb_kernel(const __grid_constant__ StageSet ss, int count, const void *__restrict__ x, int m, int64_t N,
               int64_t K, float *__restrict__ y, bool accumulate) {
  __shared__ float red[kWarps][kTileRows * 8];
  pdl_launch_dependents();   // the next kernel in the stream may be scheduled meanwhile
  pdl_wait();                // x and y may belong to the previous kernel
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t KG = K >> 6;
  const int64_t ga = KG * warp / kWarps;
  const int L = static_cast<int>(KG * (warp + 1) / kWarps - ga);
  const int n_items = L * count;
  const bool has_x = gid < m;
  const int64_t xrow = static_cast<int64_t>(has_x ? gid : 0) * K + 16 * tig;
  const int64_t n_tiles = (N + kTileRows - 1) / kTileRows;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t r0 = tile * kTileRows;
    const int64_t glo = (r0 + gid < N ? r0 + gid : N - 1) * KG + ga;
    const int64_t ghi = (r0 + gid + 8 < N ? r0 + gid + 8 : N - 1) * KG + ga;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};     // (row gid | gid + 8) x (batch 2 tig, 2 tig + 1)
    // item i = (stage j, group ga + g), g fastest; three cursors walk the sequence
    RowMeta ml1 = {}, mh1 = {}, ml2 = {}, mh2 = {};
    RowCodes cl = {}, ch = {};
    XFrag<XF32> xf = {};
    int j1 = 0, g1 = 0;        // item i + 1
    int j2 = 0, g2 = 0;        // item i + 2
    auto step = [&](int &j, int &g) {
      if (++g == L) { g = 0; ++j; }
    };
    if (n_items > 0) {
      ml1 = load_meta(ss, 0, glo);
      mh1 = load_meta(ss, 0, ghi);
      step(j1, g1);
      step(j2, g2);
      step(j2, g2);
      if (n_items > 1) {
        ml2 = load_meta(ss, j1, glo + g1);
        mh2 = load_meta(ss, j1, ghi + g1);
      }
      cl = load_codes(ss, 0, glo, ml1, tig);
      ch = load_codes(ss, 0, ghi, mh1, tig);
      xf = load_x<XF32>(x, xrow + ga * 64, has_x);
    }
#pragma unroll 2
    for (int i = 0; i < n_items; ++i) {
      // prefetch: widths/offsets of item i + 2, codes and activations of item i + 1
      RowMeta ml3 = ml2, mh3 = mh2;
      if (i + 2 < n_items) {
        ml3 = load_meta(ss, j2, glo + g2);
        mh3 = load_meta(ss, j2, ghi + g2);
      }
      RowCodes cl2 = cl, ch2 = ch;
      XFrag<XF32> xf2 = xf;
      if (i + 1 < n_items) {
        cl2 = load_codes(ss, j1, glo + g1, ml2, tig);
        ch2 = load_codes(ss, j1, ghi + g1, mh2, tig);
        xf2 = load_x<XF32>(x, xrow + (ga + g1) * 64, has_x);
      }
      step(j1, g1);
      step(j2, g2);
      // item i
      uint32_t bh[8], bl[8], alo[8], ahi[8];
      b_operand<XF32>(xf, bh, bl);
      rows_operand(cl, ch, tig, alo, ahi);
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t a[4] = {alo[2 * c], ahi[2 * c], alo[2 * c + 1], ahi[2 * c + 1]};
        mma_bf16(d, a, bh[2 * c], bh[2 * c + 1]);
        if (XF32) mma_bf16(d, a, bl[2 * c], bl[2 * c + 1]);
      }
      acc[0] = fmaf(cl.s, d[0], acc[0]);
      acc[1] = fmaf(cl.s, d[1], acc[1]);
      acc[2] = fmaf(ch.s, d[2], acc[2]);
      acc[3] = fmaf(ch.s, d[3], acc[3]);
      ml2 = ml3;
      mh2 = mh3;
      cl = cl2;
      ch = ch2;
      xf = xf2;
    }
    float *rw = red[warp];
    rw[gid * 8 + 2 * tig] = acc[0];
    rw[gid * 8 + 2 * tig + 1] = acc[1];
    rw[(gid + 8) * 8 + 2 * tig] = acc[2];
    rw[(gid + 8) * 8 + 2 * tig + 1] = acc[3];
    __syncthreads();
    if (threadIdx.x < kTileRows * 8) {
      const int row = threadIdx.x >> 3, col = threadIdx.x & 7;
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[w][threadIdx.x];
      if (col < m && r0 + row < N) {
        float *yp = y + static_cast<int64_t>(col) * N + r0 + row;
        *yp = accumulate ? *yp + v : v;
      }
    }
    __syncthreads();
  }
}

// ---- batch 1, one matrix of per-group widths: width-sorted passes --------------------------
// A warp per row. Within a row the groups of one width are consecutive in that width's plane,
// so the warp first lists the row's groups by width (one coalesced read of the width map per
// 32 groups, a ballot per width, ranks by popcount) in shared memory, then runs one pass per
// width in which lane i takes the i-th group of that width: the whole warp decodes one width
// with constant shifts (no divergence), and the code reads of a pass are contiguous in the
// plane. Per weight: the code as the bit pattern of 2^23 + q (shift, LOP3), minus 2^23 + z
// (exact), times x (fp32, staged once per CTA with the padded pitch of the lane kernel), summed
// per group in fp32 and scaled by s.
constexpr int kVbqWarps = 8;
constexpr int kVbqThreads = 32 * kVbqWarps;
constexpr int kVbqMaxGroups = 1024;        // per row (u16 list entries); longer rows use the tensor-core kernel
constexpr int kVbqPitch = 272;             // fp32 x: 256 bytes per group + 16

// staged x, then per warp a list of the row's group indices (u16), KG entries
__host__ __device__ constexpr int64_t vbq_smem(int64_t KG) {
  return KG * kVbqPitch + ((static_cast<int64_t>(kVbqWarps) * KG * 2 + 15) & ~int64_t(15));
}

// the 8 B bytes of one group of width B
template <int B>
struct GroupCodes {
  uint32_t w[2 * B];
};
template <int B>
__device__ __forceinline__ GroupCodes<B> load_group(const uint8_t *src) {
  GroupCodes<B> gc;
  if (B == 1) {
    const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
    gc.w[0] = v.x;
    gc.w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + i);
      gc.w[4 * i] = v.x; gc.w[4 * i + 1] = v.y; gc.w[4 * i + 2] = v.z; gc.w[4 * i + 3] = v.w;
    }
  }
  return gc;
}

// sum over the group of (q - z) * x, fp32. Widths 1, 2, 4: the codes are read in windows of 8
// (4 for width 4) that span at most 16 bits; code p of a window is masked in place, so its
// float bit pattern is 2^23 + q * 2^(p b) (no shift: one LOP3), minus 2^23 + z * 2^(p b) gives
// (q - z) * 2^(p b) exactly, and each window position has its own accumulator, scaled back by
// 2^(-p b) once per group (exact). Width 8: byte p of a word is placed into 2^23 + q by PRMT.
template <int B>
__device__ __forceinline__ float group_dot(const GroupCodes<B> &gc, uint32_t z, const uint8_t *xg) {
  // pairs of window positions go through the two-wide fp32 add and FMA (each half rounds as the
  // scalar operation would)
  if (B == 8) {
    const float zc = 8388608.0f + static_cast<float>(z);
    const float2 nz = make_float2(-zc, -zc);
    float2 d2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float4 f = *reinterpret_cast<const float4 *>(xg + 16 * c);
      const float2 q01 = make_float2(__uint_as_float(__byte_perm(gc.w[c], 0x4B000000u, 0x7440u)),
                                     __uint_as_float(__byte_perm(gc.w[c], 0x4B000000u, 0x7441u)));
      const float2 q23 = make_float2(__uint_as_float(__byte_perm(gc.w[c], 0x4B000000u, 0x7442u)),
                                     __uint_as_float(__byte_perm(gc.w[c], 0x4B000000u, 0x7443u)));
      d2[0] = __ffma2_rn(__fadd2_rn(q01, nz), make_float2(f.x, f.y), d2[0]);
      d2[1] = __ffma2_rn(__fadd2_rn(q23, nz), make_float2(f.z, f.w), d2[1]);
    }
    return (d2[0].x + d2[0].y) + (d2[1].x + d2[1].y);
  } else {
    constexpr int kWin = B == 4 ? 4 : 8;               // codes per window (8 or 16 bits)
    float2 nz[kWin / 2], dp[kWin / 2];
#pragma unroll
    for (int h = 0; h < kWin / 2; ++h) {
      nz[h] = make_float2(-fmaf(static_cast<float>(z), static_cast<float>(1u << (2 * h * B)), 8388608.0f),
                          -fmaf(static_cast<float>(z), static_cast<float>(1u << ((2 * h + 1) * B)), 8388608.0f));
      dp[h] = make_float2(0.0f, 0.0f);
    }
#pragma unroll
    for (int t0 = 0; t0 < 64; t0 += kWin) {
      const int bit0 = t0 * B;                         // first bit of the window in the group
      const uint32_t word = gc.w[bit0 / 32] >> (bit0 % 32);
      float xa[kWin];
#pragma unroll
      for (int h = 0; h < kWin / 4; ++h) {
        const float4 f = *reinterpret_cast<const float4 *>(xg + 4 * (t0 + 4 * h));
        xa[4 * h] = f.x; xa[4 * h + 1] = f.y; xa[4 * h + 2] = f.z; xa[4 * h + 3] = f.w;
      }
#pragma unroll
      for (int h = 0; h < kWin / 2; ++h) {
        const float2 q = make_float2(__uint_as_float(and_or(word, ((1u << B) - 1u) << (2 * h * B), 0x4B000000u)),
                                     __uint_as_float(and_or(word, ((1u << B) - 1u) << ((2 * h + 1) * B), 0x4B000000u)));
        dp[h] = __ffma2_rn(__fadd2_rn(q, nz[h]), make_float2(xa[2 * h], xa[2 * h + 1]), dp[h]);
      }
    }
    float d = 0.0f;
#pragma unroll
    for (int h = 0; h < kWin / 2; ++h) {
      d = fmaf(dp[h].x, __uint_as_float(static_cast<uint32_t>(127 - 2 * h * B) << 23), d);
      d = fmaf(dp[h].y, __uint_as_float(static_cast<uint32_t>(127 - (2 * h + 1) * B) << 23), d);
    }
    return d;
  }
}

// One width pass of a row: lane i takes list entries i, i + 32, ... (the row's groups of width
// B, or with list == nullptr every group of a fixed-4 stage) two at a time, both groups' loads
// issued before either product. The row's groups of one width are consecutive in the plane
// (offsets are ranks among same-width groups in row-major order, times 8 B), so the i-th one
// starts 8 B * i bytes after the first: one offset per pass, read by the caller, instead of one
// dependent offset load per group.
template <int B>
__device__ __forceinline__ float width_pass(const uint16_t *list, int cnt, int lane, int64_t g0, const uint8_t *pl,
                                           const uint16_t *scale, const uint8_t *zero, const uint8_t *xs) {
  float acc = 0.0f;
  for (int i = lane; i < cnt; i += 64) {
    const bool two = i + 32 < cnt;
    const int ib = two ? i + 32 : i;
    const int ga = list ? list[i] : i;
    const int gb = list ? list[ib] : ib;
    const uint8_t *sa = list ? pl + static_cast<int64_t>(i) * (8 * B) : pl + (g0 + ga) * 32;
    const uint8_t *sb = list ? pl + static_cast<int64_t>(ib) * (8 * B) : pl + (g0 + gb) * 32;
    const uint32_t za = __ldg(zero + g0 + ga), zb = __ldg(zero + g0 + gb);
    const float fa = f16_bits_to_f32(__ldg(scale + g0 + ga)), fb = f16_bits_to_f32(__ldg(scale + g0 + gb));
    const GroupCodes<B> ca = load_group<B>(sa);
    const GroupCodes<B> cb = load_group<B>(sb);
    acc = fmaf(fa, group_dot<B>(ca, za, xs + static_cast<int64_t>(ga) * kVbqPitch), acc);
    if (two) acc = fmaf(fb, group_dot<B>(cb, zb, xs + static_cast<int64_t>(gb) * kVbqPitch), acc);
  }
  return acc;
}

template <bool XBF16>
__global__ void __launch_bounds__(kVbqThreads, 3)
gemv_vbq1_kernel(const __grid_constant__ StageSet ss, int count, const void *__restrict__ x, int64_t N, int64_t K,
                 float *__restrict__ y, bool accumulate) {
  extern __shared__ __align__(16) uint8_t xs[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int KG = static_cast<int>(K >> 6);
  // stage x as fp32, one group per kVbqPitch bytes
  for (int64_t u = threadIdx.x; u < static_cast<int64_t>(KG) * 16; u += kVbqThreads) {
    float4 f;
    if (XBF16) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(x) + u);
      f = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                      __uint_as_float(v.y & 0xFFFF0000u));
    } else {
      f = __ldg(reinterpret_cast<const float4 *>(x) + u);
    }
    *reinterpret_cast<float4 *>(xs + (u >> 4) * kVbqPitch + (u & 15) * 16) = f;
  }
  __syncthreads();
  uint16_t *list = reinterpret_cast<uint16_t *>(xs + static_cast<int64_t>(KG) * kVbqPitch) + warp * KG;
  (void)CQ_CHECK(static_cast<int64_t>(KG) * kVbqPitch + (warp + 1) * KG * 2 <= dynamic_smem_bytes(), 0x0706u);
  const uint32_t lt = (1u << lane) - 1u;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * kVbqWarps;
  for (int64_t n = blockIdx.x * static_cast<int64_t>(kVbqWarps) + warp; n < N; n += warps) {
    const int64_t g0 = n * KG;
    float acc = 0.0f;
#pragma unroll 1
    for (int j = 0; j < count; ++j) {
      const uint8_t *bits = ss.bits[j];
      const uint16_t *scale = ss.scale[j];
      const uint8_t *zero = ss.zero[j];
      if (!bits) {                 // fixed 4-bit: every group, 32 bytes at 32 g of plane 4
        acc += width_pass<4>(nullptr, KG, lane, g0, ss.plane[j][2], scale, zero, xs);
        continue;
      }
      const uint32_t *offset = ss.offset[j];
      // list the row's groups by width: widths 1, 2, 4, 8 at list offsets base[0..3]
      int cnt[4] = {0, 0, 0, 0};
      for (int w0 = 0; w0 < KG; w0 += 32) {
        const int b = w0 + lane < KG ? __ldg(bits + g0 + w0 + lane) : 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) cnt[c] += __popc(__ballot_sync(0xffffffffu, b == (1 << c)));
      }
      int fill[4] = {0, cnt[0], cnt[0] + cnt[1], cnt[0] + cnt[1] + cnt[2]};
      const int base[4] = {fill[0], fill[1], fill[2], fill[3]};
      __syncwarp();     // the previous stage's passes have read the list
      for (int w0 = 0; w0 < KG; w0 += 32) {
        const int b = w0 + lane < KG ? __ldg(bits + g0 + w0 + lane) : 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t mk = __ballot_sync(0xffffffffu, b == (1 << c));
          if (b == (1 << c) && CQ_CHECK(fill[c] + __popc(mk & lt) < KG, 0x0703u))
            list[fill[c] + __popc(mk & lt)] = static_cast<uint16_t>(w0 + lane);
          fill[c] += __popc(mk);
        }
      }
      __syncwarp();
      // where each width's run of this row starts in its plane (the offset of its first group;
      // a multiple of 8 b by construction, the mask keeps a damaged map aligned)
      uint32_t first[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t o = cnt[c] ? __ldg(offset + g0 + list[base[c]]) : 0u;
        first[c] = o & ~((8u << c) - 1u);
        // debug build: the run must start on its 8 b grid, at a rank no higher than its first
        // group's index (else the pass is skipped)
        (void)CQ_CHECK((o & ((8u << c) - 1u)) == 0u, 0x0704u);
        if (cnt[c] && !CQ_CHECK(static_cast<int64_t>(o >> (3 + c)) <= g0 + list[base[c]], 0x0705u)) cnt[c] = 0;
      }
      acc += width_pass<1>(list + base[0], cnt[0], lane, g0, ss.plane[j][0] + first[0], scale, zero, xs);
      acc += width_pass<2>(list + base[1], cnt[1], lane, g0, ss.plane[j][1] + first[1], scale, zero, xs);
      acc += width_pass<4>(list + base[2], cnt[2], lane, g0, ss.plane[j][2] + first[2], scale, zero, xs);
      acc += width_pass<8>(list + base[3], cnt[3], lane, g0, ss.plane[j][3] + first[3], scale, zero, xs);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) y[n] = accumulate ? y[n] + acc : acc;
    __syncwarp();       // the list is rewritten for the next row
  }
}

template <bool XBF16>
cq_status launch_vbq1(const StageSet &ss, int count, const void *x, int64_t N, int64_t K, float *y, bool acc,
                      cudaStream_t s) {
  const int64_t smem = vbq_smem(K >> 6);
  cq_status st = cuda_check(cudaFuncSetAttribute(gemv_vbq1_kernel<XBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem)),
                            "cq_dequant_gemv: shared memory attribute");
  if (st != CQ_OK) return st;
  // one wave of resident CTAs (grid-stride over rows): as many per SM as registers and the
  // staged activations allow
  int per_sm = 1;
  st = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_vbq1_kernel<XBF16>, kVbqThreads,
                                                                static_cast<size_t>(smem)),
                  "cq_dequant_gemv: occupancy");
  if (st != CQ_OK) return st;
  const int64_t need = (N + kVbqWarps - 1) / kVbqWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int blocks = static_cast<int>(need < cap ? need : cap);
  // an ordinary launch: with programmatic dependent launch this latency-bound kernel measured
  // slower back to back (12.2 -> 14.4 us per 2048x8192 matrix)
  gemv_vbq1_kernel<XBF16><<<blocks, kVbqThreads, static_cast<size_t>(smem), s>>>(ss, count, x, N, K, y, acc);
  return launch_check("cq_dequant_gemv (batch 1, per-group widths / stages)");
}

}  // namespace

cq_status launch_gemv_stages(const cq_qweight *const *stages, int count, const void *x, cq_dtype xdt, int m,
                             float *y, cudaStream_t s) {
  const int64_t N = stages[0]->rows, K = stages[0]->cols;
  if (N == 0) return CQ_OK;
  if (K == 0) return cuda_check(cudaMemsetAsync(y, 0, sizeof(float) * m * N, s), "cq_dequant_gemv: zero y");
  const int64_t tiles = (N + kTileRows - 1) / kTileRows;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int blocks = static_cast<int>(tiles < cap ? tiles : cap);
  // up to kPerLaunch stages per launch; later launches add to y in stream order
  for (int j0 = 0; j0 < count; j0 += kPerLaunch) {
    const int cnt = count - j0 < kPerLaunch ? count - j0 : kPerLaunch;
    StageSet ss = {};
    for (int j = 0; j < cnt; ++j) {
      const cq_qweight &q = *stages[j0 + j];
      ss.bits[j] = q.bits;
      ss.offset[j] = q.offset;
      for (int p = 0; p < 4; ++p) ss.plane[j][p] = q.plane[p];
      ss.scale[j] = q.scale;
      ss.zero[j] = q.zero;
    }
    // batch 1 (measured faster there): width-sorted passes on CUDA cores; any other batch, or
    // rows too long to stage, tensor cores
    if (m == 1 && (K >> 6) <= kVbqMaxGroups && vbq_smem(K >> 6) <= 200 * 1024) {
      cq_status st = xdt == CQ_BF16 ? launch_vbq1<true>(ss, cnt, x, N, K, y, j0 > 0, s)
                                    : launch_vbq1<false>(ss, cnt, x, N, K, y, j0 > 0, s);
      if (st != CQ_OK) return st;
      continue;
    }
    const cudaError_t e = xdt == CQ_BF16
                              ? launch_pdl(gemv_vb_kernel<false>, dim3(blocks), dim3(kThreads), 0, s, ss, cnt, x, m,
                                           N, K, y, j0 > 0)
                              : launch_pdl(gemv_vb_kernel<true>, dim3(blocks), dim3(kThreads), 0, s, ss, cnt, x, m, N,
                                           K, y, j0 > 0);
    cq_status st = cuda_check(e, "cq_dequant_gemv (per-group widths / stages)");
    if (st != CQ_OK) return st;
    st = launch_check("cq_dequant_gemv (per-group widths / stages)");
    if (st != CQ_OK) return st;
  }
  return CQ_OK;
}

}  // namespace cq
