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
//   warp 0     TMA producer: the tile's 4-bit codes (128 rows x 32 B) and the activations of
//              the group (m rows x 64 bf16, 128-byte swizzled = the UMMA K-major layout)
//   warp 1     MMA issuer: four tcgen05.mma (M=128, N=NT, K=16) per group into one of two
//              tensor-memory accumulators; commits release the stage and publish the group
//   warps 2-5  dequantize: thread r turns row r's 64 codes into bf16 (q - z) and writes them
//              in the 128-byte swizzled K-major layout the MMA descriptor expects
//   warps 6-9  epilogue: tcgen05.ld the group's 128 x NT fp32 sums (one row per thread),
//              acc += s * sum; at the end of a tile (or of the CTA's range) add to y
// y is zeroed first; tiles split between two CTAs are combined with fp32 atomics.
// Every barrier wait is bounded: on timeout the CTA raises a status flag, drains what it
// issued, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kTileM = 128;
constexpr int kThreads = 320;
constexpr uint32_t kCodeBytes = kTileM * 32;      // one group of 4-bit codes for 128 rows
constexpr uint32_t kABytes = kTileM * 128;         // bf16 A tile: 128 rows x 64 columns
constexpr uint32_t kSpinLimit = 1u << 22;          // try_wait rounds before giving up

template <int NT>
struct Cfg {
  static constexpr uint32_t kXBytes = NT * 128;
  static constexpr uint32_t kStageBytes = kABytes + kXBytes + kCodeBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
  static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
  static constexpr uint32_t kSmem = 1024 + kStages * kStageBytes + (4 * kStages + 8) * 8 + 16;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// bounded wait on the phase of the given parity; false on timeout or when another role gave up
__device__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile uint32_t *abort_flag, uint32_t *status,
                          bool honour_abort = true) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 63) == 63) {
      if (honour_abort && *abort_flag) return false;
      __nanosleep(64);
    }
  }
  *abort_flag = 1u;
  if (status) atomicOr(status, 1u);
  return false;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

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

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
gemm4_tc_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                const uint16_t *__restrict__ scale, const uint8_t *__restrict__ zero, float *__restrict__ y,
                int m, int64_t N, int KG, int64_t n_items, uint32_t *__restrict__ status) {
  using C = Cfg<NT>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;                               // S x 16 KiB, 1024-aligned
  uint8_t *sX = sA + S * kABytes;                   // S x NT*128 B, 1024-aligned
  uint8_t *sC = sX + S * C::kXBytes;                // S x 4 KiB
  uint64_t *bars = reinterpret_cast<uint64_t *>(sC + S * kCodeBytes);
  uint64_t *full = bars, *afull = bars + S, *empty = bars + 2 * S, *accf = bars + 3 * S, *acce = accf + 2;
  uint64_t *drain = acce + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t it_begin = static_cast<int64_t>(blockIdx.x) * n_items / gridDim.x;
  const int64_t it_end = static_cast<int64_t>(blockIdx.x + 1) * n_items / gridDim.x;
  const int n_local = static_cast<int>(it_end - it_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(afull + s, 4);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf + b, 1);
      mbar_init(acce + b, 4);
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
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int li = 0; li < n_local; ++li) {
        const int s = li % S;
        if (!mbar_wait(empty + s, ((li / S) & 1) ^ 1, abort_flag, status)) break;
        const int64_t i = it_begin + li;
        const int tile = static_cast<int>(i / KG), g = static_cast<int>(i % KG);
        mbar_arrive_expect_tx(full + s, kCodeBytes + C::kXBytes);
        tma_load_2d(sC + s * kCodeBytes, &tm_codes, g * 32, tile * kTileM, full + s);
        tma_load_2d(sX + s * C::kXBytes, &tm_x, g * 64, 0, full + s);
        issued = li + 1;
      }
      // every copy this thread started has landed before the CTA may exit
      for (int li = issued - S > 0 ? issued - S : 0; li < issued; ++li)
        mbar_wait(full + (li % S), (li / S) & 1, abort_flag, status, false);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc<NT>();
      int done = 0;
      for (int li = 0; li < n_local; ++li) {
        const int s = li % S, b = li & 1;
        if (!mbar_wait(afull + s, (li / S) & 1, abort_flag, status)) break;
        if (!mbar_wait(full + s, (li / S) & 1, abort_flag, status)) break;
        if (!mbar_wait(acce + b, ((li >> 1) & 1) ^ 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kABytes), b0 = smem_u32(sX + s * C::kXBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem + b * NT, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), idesc, kk > 0);
        umma_commit(empty + s);
        umma_commit(accf + b);
        done = li + 1;
      }
      // all issued MMAs have completed before tensor memory is released
      umma_commit(drain);
      mbar_wait(drain, 0, abort_flag, status, false);
      (void)done;
    }
  } else if (warp < 6) {
    // ---------------- dequantize: row r of every tile ----------------
    const int r = (warp - 2) * 32 + lane;
    for (int li = 0; li < n_local; ++li) {
      const int s = li % S;
      if (!mbar_wait(full + s, (li / S) & 1, abort_flag, status)) break;
      const int64_t i = it_begin + li;
      const int64_t tile = i / KG;
      const int g = static_cast<int>(i % KG);
      int64_t row = tile * kTileM + r;
      row = row < N ? row : N - 1;
      const uint32_t z = __ldg(zero + row * KG + g);
      const uint32_t zz = 0x43004300u | z | (z << 16);      // (128 + z) in both halves
      const uint4 *src = reinterpret_cast<const uint4 *>(sC + s * kCodeBytes + r * 32);
      const uint4 c0 = src[0], c1 = src[1];
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint8_t *dst_row = sA + s * kABytes + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {       // 16-byte chunk c = columns 8c .. 8c+7
        const uint32_t w = words[c], w4 = w >> 4;
        uint4 v;
        v.x = bf16x2_sub(nat_pair(w, w4, 0x4400u), zz);
        v.y = bf16x2_sub(nat_pair(w, w4, 0x5511u), zz);
        v.z = bf16x2_sub(nat_pair(w, w4, 0x6622u), zz);
        v.w = bf16x2_sub(nat_pair(w, w4, 0x7733u), zz);
        *reinterpret_cast<uint4 *>(dst_row + ((c ^ (r & 7)) << 4)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(afull + s);
    }
  } else {
    // ---------------- epilogue: row r = TMEM lane ----------------
    const int quad = warp & 3;                 // this warp may read TMEM lanes 32*quad .. +31
    const int r = quad * 32 + lane;
    float acc[NT];
#pragma unroll
    for (int c = 0; c < NT; ++c) acc[c] = 0.0f;
    for (int li = 0; li < n_local; ++li) {
      const int b = li & 1;
      const int64_t i = it_begin + li;
      const int64_t tile = i / KG;
      const int g = static_cast<int>(i % KG);
      int64_t row = tile * kTileM + r;
      const int64_t lrow = row < N ? row : N - 1;
      const float sf = f16_bits_to_f32(__ldg(scale + lrow * KG + g));
      if (!mbar_wait(accf + b, (li >> 1) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + b * NT;
#pragma unroll
      for (int c0 = 0; c0 < NT; c0 += 16) {
        uint32_t d[16];
        tmem_ld16(tbase + c0, d);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[c0 + j] = fmaf(sf, __uint_as_float(d[j]), acc[c0 + j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce + b);
      const bool last = (g == KG - 1) || (li == n_local - 1);
      if (last) {
        if (row < N) {
#pragma unroll
          for (int c = 0; c < NT; ++c)
            if (c < m) atomicAdd(y + static_cast<int64_t>(c) * N + row, acc[c]);
        }
#pragma unroll
        for (int c = 0; c < NT; ++c) acc[c] = 0.0f;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(C::kTmemCols));
  }
}

// ---- host side ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int NT>
cq_status launch_nt(const cq_qweight &qw, const void *x, int m, float *y, uint32_t *status, cudaStream_t s) {
  using C = Cfg<NT>;
  auto encode = encode_fn();
  if (!encode) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: cuTensorMapEncodeTiled unavailable");
  const int64_t N = qw.rows, K = qw.cols;
  CUtensorMap tm_codes, tm_x;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {32, kTileM};
    cuuint32_t es[2] = {1, 1};
    CUresult r = encode(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(qw.plane[2]), dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CQ_ERR_CUDA, "cq_dequant_gemm: code tensor map (%d)", (int)r);
  }
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
  const int64_t items = tiles * KG;
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
