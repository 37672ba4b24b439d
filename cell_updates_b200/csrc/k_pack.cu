// k_pack.cu -- bit-packed planes for per-group widths.
//
// [VBQ] "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
// Without Changing the File They Ship", abstract: because widths are chosen per group, the
// codes can be stored densely packed at their own widths. The layout (one plane per width, row-major rank of the group
// among groups of its width, LSB-first codes) is defined in include/cq.h.
//
// Work unit: eight lanes per group, one lane per eight consecutive codes. Lane `sub` of a
// group of width b owns exactly b bytes of the plane (8 codes * b bits), so packing and
// unpacking are single stores/loads of 1, 2, 4 or 8 bytes with no read-modify-write.
#include "cq_async.cuh"

namespace cq {
namespace {

constexpr int kThreads = 256;

// 8 codes (one per byte of v, as the two words lo, hi) -> 8*b bits, code j at bits [j*b, (j+1)*b).
// Widths 1 and 2 gather four bytes' low bits with one multiply: with bytes c_i < 2^b at bit 8i,
// x * K (K = 0x10204080 for b = 1, 0x01041040 for b = 2) puts c_i at bit 32 - 4b + b i and every cross
// term at a distinct lower position (or past bit 31), so no carry reaches the top 4b bits.
__device__ __forceinline__ uint32_t gather4(uint32_t x, int b) {
  return b == 1 ? (x * 0x10204080u) >> 28 : (x * 0x01041040u) >> 24;
}
__device__ __forceinline__ uint64_t pack8(uint64_t v, int b) {
  const uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
  switch (b) {
    case 1: return gather4(lo & 0x01010101u, 1) | (gather4(hi & 0x01010101u, 1) << 4);
    case 2: return gather4(lo & 0x03030303u, 2) | (gather4(hi & 0x03030303u, 2) << 8);
    case 4: {
      // nibbles of four bytes -> 16 bits: (x | x >> 4) keeps pairs in each half word
      const uint32_t a = lo & 0x0F0F0F0Fu, c = hi & 0x0F0F0F0Fu;
      const uint32_t a2 = (a | (a >> 4)) & 0x00FF00FFu, c2 = (c | (c >> 4)) & 0x00FF00FFu;
      return static_cast<uint64_t>(__byte_perm(a2, c2, 0x6420));
    }
    default: return v;
  }
}

// 8*b bits -> 8 codes, one per byte (the inverse of pack8)
__device__ __forceinline__ uint32_t spread4(uint32_t x, int b) {
  // the low 4b bits of x -> four bytes of b bits each
  if (b == 1) {
    x &= 0xFu;
    x = (x | (x << 14)) & 0x00030003u;
    return (x | (x << 7)) & 0x01010101u;
  }
  x &= 0xFFu;
  x = (x | (x << 12)) & 0x000F000Fu;
  return (x | (x << 6)) & 0x03030303u;
}
__device__ __forceinline__ uint64_t unpack8(uint64_t p, int b) {
  const uint32_t w = static_cast<uint32_t>(p);
  switch (b) {
    case 1: return spread4(w, 1) | (static_cast<uint64_t>(spread4(w >> 4, 1)) << 32);
    case 2: return spread4(w, 2) | (static_cast<uint64_t>(spread4(w >> 8, 2)) << 32);
    case 4: {
      // 16 bits -> four bytes of one nibble each, per 32-bit half
      uint32_t a = w & 0xFFFFu, c = w >> 16;
      a = (a | (a << 8)) & 0x00FF00FFu;
      c = (c | (c << 8)) & 0x00FF00FFu;
      a = (a | (a << 4)) & 0x0F0F0F0Fu;
      c = (c | (c << 4)) & 0x0F0F0F0Fu;
      return a | (static_cast<uint64_t>(c) << 32);
    }
    default: return p;
  }
}

__device__ __forceinline__ void store_bytes(uint8_t *dst, uint64_t v, int b) {
  switch (b) {
    case 1: *dst = static_cast<uint8_t>(v); break;
    case 2: *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(v); break;
    case 4: *reinterpret_cast<uint32_t *>(dst) = static_cast<uint32_t>(v); break;
    default: *reinterpret_cast<uint2 *>(dst) = make_uint2(static_cast<uint32_t>(v), static_cast<uint32_t>(v >> 32)); break;
  }
}

__device__ __forceinline__ uint64_t load_bytes(const uint8_t *src, int b) {
  switch (b) {
    case 1: return __ldg(src);
    case 2: return __ldg(reinterpret_cast<const uint16_t *>(src));
    case 4: return __ldg(reinterpret_cast<const uint32_t *>(src));
    default: {
      const uint2 t = __ldg(reinterpret_cast<const uint2 *>(src));
      return static_cast<uint64_t>(t.x) | (static_cast<uint64_t>(t.y) << 32);
    }
  }
}

struct Planes {
  uint8_t *p[4];
  // select without indexing the parameter array (which would move it to local memory)
  __device__ __forceinline__ uint8_t *of(int b) const { return b == 1 ? p[0] : b == 2 ? p[1] : b == 4 ? p[2] : p[3]; }
};

__global__ void __launch_bounds__(kThreads)
pack_kernel(const uint8_t *__restrict__ codes, int64_t n_units, const uint8_t *__restrict__ bits,
            const uint32_t *__restrict__ offset, Planes planes) {
  for (int64_t u = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u < n_units;
       u += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t g = u >> 3;
    const int sub = static_cast<int>(u & 7);
    const uint2 c = __ldcs(reinterpret_cast<const uint2 *>(codes) + u);
    const uint64_t v = static_cast<uint64_t>(c.x) | (static_cast<uint64_t>(c.y) << 32);
    int b = 4;
    uint8_t *base;
    if (bits) {
      b = __ldg(bits + g);
      if (!width_ok(b)) continue;   // nothing to store; quantize reports the width
      const uint32_t o = __ldg(offset + g);
      // debug build: an offset off its 8 b grid, or a rank above the group's own index (a rank
      // counts earlier groups of the same width), is recorded and its group not stored
      if (!CQ_CHECK(o % (8u * b) == 0u && static_cast<int64_t>(o / (8u * b)) <= g, 0x0201u)) continue;
      base = planes.of(b) + o;
    } else {
      base = planes.p[2] + g * 32;
    }
    store_bytes(base + sub * b, pack8(v, b), b);
  }
}

// Unpack takes kPackUnroll units per lane and iteration and issues each phase's loads for all of
// them before using any (width and offset together, then the plane bytes, which depend on the
// offset), so a lane overlaps several dependent round trips: with one unit per iteration it ran
// at 1.6 TB/s on 2048x8192 (13.9 us; 12.4 us unrolled).
constexpr int kPackUnroll = 4;

__global__ void __launch_bounds__(kThreads)
unpack_kernel(uint8_t *__restrict__ codes, int64_t n_units, const uint8_t *__restrict__ bits,
              const uint32_t *__restrict__ offset, Planes planes) {
  pdl_wait();                     // the planes and the map come from earlier work; codes is written
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u0 < n_units;
       u0 += kPackUnroll * step) {
    int b[kPackUnroll];
    uint32_t o[kPackUnroll];
#pragma unroll
    for (int k = 0; k < kPackUnroll; ++k) {
      const int64_t u = u0 + k * step;
      b[k] = 4;
      o[k] = 0;
      if (bits && u < n_units) {
        b[k] = __ldg(bits + (u >> 3));
        o[k] = __ldg(offset + (u >> 3));
      }
    }
    uint64_t v[kPackUnroll];
#pragma unroll
    for (int k = 0; k < kPackUnroll; ++k) {
      const int64_t u = u0 + k * step;
      v[k] = 0;
      if (u >= n_units) continue;
      const int64_t g = u >> 3;
      const int sub = static_cast<int>(u & 7);
      if (bits) {
        if (width_ok(b[k]) &&
            CQ_CHECK(o[k] % (8u * b[k]) == 0u && static_cast<int64_t>(o[k] / (8u * b[k])) <= g, 0x0202u))
          v[k] = load_bytes(planes.of(b[k]) + o[k] + sub * b[k], b[k]);
        else
          b[k] = 0;                  // no group here: the codes are written as zeros
      } else {
        v[k] = load_bytes(planes.p[2] + g * 32 + sub * 4, 4);
      }
    }
#pragma unroll
    for (int k = 0; k < kPackUnroll; ++k) {
      const int64_t u = u0 + k * step;
      if (u >= n_units) break;
      const uint64_t c = b[k] ? unpack8(v[k], b[k]) : 0ull;
      reinterpret_cast<uint2 *>(codes)[u] = make_uint2(static_cast<uint32_t>(c), static_cast<uint32_t>(c >> 32));
    }
  }
}

// fixed 4-bit: one lane packs 32 codes (two 16-byte loads) into one 16-byte store, two such
// units per iteration so each lane keeps 64 bytes of loads in flight
__device__ __forceinline__ uint32_t nibbles_of4(uint32_t w) {
  // four codes (one per byte, low nibble used) -> 16 bits, code j at bits [4j, 4j+4)
  w &= 0x0F0F0F0Fu;
  w = (w | (w >> 4)) & 0x00FF00FFu;
  return (w | (w >> 8)) & 0x0000FFFFu;
}

__device__ __forceinline__ uint32_t pack8codes(uint32_t lo, uint32_t hi) {
  return nibbles_of4(lo) | (nibbles_of4(hi) << 16);
}

__global__ void __launch_bounds__(kThreads)
pack4_kernel(const uint8_t *__restrict__ codes, int64_t n32, uint8_t *__restrict__ plane) {
  pdl_wait();                     // the codes come from earlier work
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; u < n32; u += 2 * step) {
    const int64_t u2 = u + step;
    const uint4 *src = reinterpret_cast<const uint4 *>(codes);
    const uint4 a0 = __ldcs(src + 2 * u), a1 = __ldcs(src + 2 * u + 1);
    uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
    if (u2 < n32) {
      b0 = __ldcs(src + 2 * u2);
      b1 = __ldcs(src + 2 * u2 + 1);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(plane);
    __stcs(dst + u, make_uint4(pack8codes(a0.x, a0.y), pack8codes(a0.z, a0.w), pack8codes(a1.x, a1.y),
                               pack8codes(a1.z, a1.w)));
    if (u2 < n32)
      __stcs(dst + u2, make_uint4(pack8codes(b0.x, b0.y), pack8codes(b0.z, b0.w), pack8codes(b1.x, b1.y),
                                  pack8codes(b1.z, b1.w)));
  }
}

// ---- group -> byte offset index: three passes, no scratch beyond the offset array ------
//
// pass 1: every full tile but the last writes its four width counts into the first four
//         offset slots of its own range;
// pass 2: one block turns those counts into exclusive prefixes in place, counts the last
//         tile itself and writes the plane sizes;
// pass 3: every tile reads its four bases (before any thread overwrites them) and writes
//         the offsets of its groups. A tile only ever touches its own slots across passes.
constexpr int kIndexThreads = 512;
constexpr int kIndexPer = 8;
constexpr int64_t kTile = kIndexThreads * kIndexPer;  // 4096 groups

__device__ __forceinline__ uint64_t width_onehot16(int b) {
  // one 16-bit counter field per width slot
  return width_ok(b) ? (1ull << (16 * width_slot(b))) : 0ull;
}

// counts of the (up to) kIndexPer groups this thread owns in tile t, packed 4 x 16 bits
__device__ __forceinline__ uint64_t thread_counts(const uint8_t *bits, int64_t G, int64_t t,
                                                  int tid, int widths[kIndexPer]) {
  uint64_t c = 0;
  const int64_t g0 = t * kTile + static_cast<int64_t>(tid) * kIndexPer;
#pragma unroll
  for (int j = 0; j < kIndexPer; ++j) {
    const int64_t g = g0 + j;
    widths[j] = g < G ? static_cast<int>(__ldg(bits + g)) : 0;
    c += width_onehot16(widths[j]);
  }
  return c;
}

// exclusive scan of a packed 4x16-bit counter over the block; returns the block total too
__device__ __forceinline__ uint64_t block_exclusive_scan(uint64_t v, uint64_t *total) {
  __shared__ uint64_t warp_sums[kIndexThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint64_t s = lane < kIndexThreads / 32 ? warp_sums[lane] : 0;
    uint64_t si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    if (lane < kIndexThreads / 32) warp_sums[lane] = si - s;   // exclusive warp prefix
  }
  __syncthreads();
  const uint64_t excl = warp_sums[warp] + incl - v;
  // total = exclusive prefix of the last thread + its own value
  __shared__ uint64_t tot;
  if (threadIdx.x == kIndexThreads - 1) tot = excl + v;
  __syncthreads();
  *total = tot;
  __syncthreads();
  return excl;
}

__device__ __forceinline__ uint32_t field16(uint64_t v, int slot) {
  return static_cast<uint32_t>((v >> (16 * slot)) & 0xFFFFu);
}

__global__ void __launch_bounds__(kIndexThreads)
index_count_kernel(const uint8_t *__restrict__ bits, int64_t G, uint32_t *__restrict__ offset) {
  pdl_wait();                     // the widths and the offset slots' earlier readers
  pdl_launch_dependents();        // after the wait: a dependent may read the widths before its own
  const int64_t t = blockIdx.x;   // a full tile that is not the last one
  int widths[kIndexPer];
  uint64_t total;
  block_exclusive_scan(thread_counts(bits, G, t, threadIdx.x, widths), &total);
  if (threadIdx.x < 4) offset[t * kTile + threadIdx.x] = field16(total, threadIdx.x);
}

__global__ void __launch_bounds__(kIndexThreads)
index_scan_kernel(const uint8_t *__restrict__ bits, int64_t G, int64_t n_tiles,
                  uint32_t *__restrict__ offset, uint64_t *__restrict__ plane_bytes) {
  // the last tile's counts need only the widths, which the count pass's wait has made safe to
  // read (single launch: this kernel's own wait comes first)
  int widths[kIndexPer];
  uint64_t last;
  if (n_tiles == 1) pdl_wait();
  block_exclusive_scan(thread_counts(bits, G, n_tiles - 1, threadIdx.x, widths), &last);
  pdl_wait();                     // the count pass's slots
  pdl_launch_dependents();
  // prefix over the first n_tiles-1 tiles, 32-bit counts (G <= 2^26 keeps them exact)
  __shared__ uint32_t base[4];
  if (threadIdx.x < 4) base[threadIdx.x] = 0;
  __syncthreads();
  const int64_t full = n_tiles - 1;
  for (int64_t c0 = 0; c0 < full; c0 += kIndexThreads) {
    const int64_t t = c0 + threadIdx.x;
    uint32_t cnt[4] = {0, 0, 0, 0};
    if (t < full)
#pragma unroll
      for (int w = 0; w < 4; ++w) cnt[w] = offset[t * kTile + w];
    // two 64-bit scans with 32-bit fields (prefix <= 2^26)
    uint64_t lo = cnt[0] | (static_cast<uint64_t>(cnt[1]) << 32);
    uint64_t hi = cnt[2] | (static_cast<uint64_t>(cnt[3]) << 32);
    uint64_t tlo, thi;
    // reuse the 4x16 scan machinery on 2x32 fields: additions never carry between fields
    const uint64_t elo = block_exclusive_scan(lo, &tlo);
    const uint64_t ehi = block_exclusive_scan(hi, &thi);
    if (t < full) {
      offset[t * kTile + 0] = base[0] + static_cast<uint32_t>(elo);
      offset[t * kTile + 1] = base[1] + static_cast<uint32_t>(elo >> 32);
      offset[t * kTile + 2] = base[2] + static_cast<uint32_t>(ehi);
      offset[t * kTile + 3] = base[3] + static_cast<uint32_t>(ehi >> 32);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      base[0] += static_cast<uint32_t>(tlo);
      base[1] += static_cast<uint32_t>(tlo >> 32);
      base[2] += static_cast<uint32_t>(thi);
      base[3] += static_cast<uint32_t>(thi >> 32);
    }
    __syncthreads();
  }
  if (threadIdx.x < 4) {
    const int b = 1 << threadIdx.x;
    plane_bytes[threadIdx.x] = static_cast<uint64_t>(base[threadIdx.x] + field16(last, threadIdx.x)) * 8u * b;
  }
}

__global__ void __launch_bounds__(kIndexThreads)
index_write_kernel(const uint8_t *__restrict__ bits, int64_t G, int64_t n_tiles,
                   uint32_t *__restrict__ offset, const uint64_t *__restrict__ plane_bytes) {
  const int64_t t = blockIdx.x;
  int widths[kIndexPer];
  uint64_t total;
  // the widths were safe to read once the scan pass started (its predecessors had completed)
  const uint64_t excl = block_exclusive_scan(thread_counts(bits, G, t, threadIdx.x, widths), &total);
  pdl_wait();                     // the scan pass's bases and plane sizes
  pdl_launch_dependents();
  __shared__ uint32_t base[4];
  if (threadIdx.x < 4) {
    if (t < n_tiles - 1) {
      base[threadIdx.x] = offset[t * kTile + threadIdx.x];
    } else {
      const uint32_t per = 8u << threadIdx.x;   // bytes per group of width 2^slot
      base[threadIdx.x] = static_cast<uint32_t>(plane_bytes[threadIdx.x] / per) - field16(total, threadIdx.x);
    }
  }
  __syncthreads();   // every base is read before any slot of this tile is overwritten
  uint32_t run[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) run[w] = base[w] + field16(excl, w);
  const int64_t g0 = t * kTile + static_cast<int64_t>(threadIdx.x) * kIndexPer;
#pragma unroll
  for (int j = 0; j < kIndexPer; ++j) {
    const int64_t g = g0 + j;
    if (g >= G) break;
    const int b = widths[j];
    if (width_ok(b)) {
      const int sl = width_slot(b);
      offset[g] = run[sl] * 8u * static_cast<uint32_t>(b);
      run[sl] += 1;
    } else {
      offset[g] = 0;
    }
  }
}

int grid_for(int64_t units) {
  const int64_t need = (units + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(need < cap ? need : cap);
}

}  // namespace

cq_status launch_varbits_index(const uint8_t *bits, int64_t G, uint32_t *offset,
                               uint64_t *plane_bytes, cudaStream_t s) {
  if (G == 0) return cuda_check(cudaMemsetAsync(plane_bytes, 0, 4 * sizeof(uint64_t), s), "cq_varbits_index");
  const int64_t n_tiles = (G + kTile - 1) / kTile;
  // programmatic dependent launches: each pass is scheduled while the one before it finishes
  if (n_tiles > 1) {
    cq_status st = cuda_check(launch_pdl(index_count_kernel, dim3(static_cast<unsigned>(n_tiles - 1)),
                                         dim3(kIndexThreads), 0, s, bits, G, offset), "cq_varbits_index: count");
    if (st != CQ_OK) return st;
  }
  cq_status st = cuda_check(launch_pdl(index_scan_kernel, dim3(1), dim3(kIndexThreads), 0, s, bits, G, n_tiles,
                                       offset, plane_bytes), "cq_varbits_index: scan");
  if (st != CQ_OK) return st;
  st = cuda_check(launch_pdl(index_write_kernel, dim3(static_cast<unsigned>(n_tiles)), dim3(kIndexThreads), 0, s,
                             bits, G, n_tiles, offset, plane_bytes), "cq_varbits_index: write");
  if (st != CQ_OK) return st;
  return launch_check("cq_varbits_index");
}

cq_status launch_pack(const uint8_t *codes, int64_t G, const uint8_t *bits, const uint32_t *offset,
                      uint8_t *const plane[4], cudaStream_t s) {
  if (G == 0) return CQ_OK;
  if (!bits) {
    const int64_t n32 = G * 2;
    cq_status st = cuda_check(launch_pdl(pack4_kernel, dim3(grid_for((n32 + 1) / 2)), dim3(kThreads), 0, s, codes, n32,
                                         plane[2]),
                              "cq_pack_varbits");
    if (st != CQ_OK) return st;
    return launch_check("cq_pack_varbits");
  }
  Planes P{{plane[0], plane[1], plane[2], plane[3]}};
  // an ordinary launch, one unit per lane and iteration: unrolled like unpack and launched as a
  // programmatic dependent, pack measured slower (9.9 -> 11.6 us on 2048x8192)
  pack_kernel<<<grid_for(G * 8), kThreads, 0, s>>>(codes, G * 8, bits, offset, P);
  return launch_check("cq_pack_varbits");
}

cq_status launch_unpack(const cq_qweight &qw, uint8_t *codes, cudaStream_t s) {
  const int64_t G = qw.rows * (qw.cols / kGroup);
  if (G == 0) return CQ_OK;
  Planes P{{const_cast<uint8_t *>(qw.plane[0]), const_cast<uint8_t *>(qw.plane[1]),
            const_cast<uint8_t *>(qw.plane[2]), const_cast<uint8_t *>(qw.plane[3])}};
  cq_status st = cuda_check(launch_pdl(unpack_kernel, dim3(grid_for((G * 8 + kPackUnroll - 1) / kPackUnroll)),
                                       dim3(kThreads), 0, s, codes, G * 8, qw.bits, qw.offset, P),
                            "cq_unpack_varbits");
  if (st != CQ_OK) return st;
  return launch_check("cq_unpack_varbits");
}

}  // namespace cq
