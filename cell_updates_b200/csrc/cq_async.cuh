// cq_async.cuh -- asynchronous-copy building blocks shared by the matmul kernels: mbarrier
// waits with an iteration bound, TMA tiled loads, cp.async with mbarrier completion, and the
// driver's tensor-map encoder. Every wait gives up after kSuspendLimit tries: the caller raises
// its error flag, lets its own copies land and returns, so a lost arrival never hangs a GPU.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>

#include "cq_internal.cuh"

namespace cq {


__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
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

// try_wait that lets the hardware suspend the thread for up to hint_ns while the phase is open
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *b, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// bounded wait on the phase of the given parity; false on timeout or when another role gave
// up. A waiting thread is suspended in hardware (up to 1 us per try) instead of spinning, so
// waiting warps leave the issue slots to the warps that have work; after kSuspendLimit tries
// (about a second) the wait raises the abort flag and the status word.
constexpr uint32_t kSuspendLimit = 1u << 20;
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile uint32_t *abort_flag,
                                          uint32_t *status, bool honour_abort = true) {
  if (mbar_try_wait(b, parity)) return true;
  for (uint32_t i = 0; i < kSuspendLimit; ++i) {
    if (mbar_try_wait_hint(b, parity, 1000u)) return true;
    if (honour_abort && *abort_flag) return false;
  }
  *abort_flag = 1u;
  if (status) {
    // the status word may be cleared by the kernel this grid overlaps (programmatic dependent
    // launch): report only once that kernel has finished (no-op for an ordinary launch)
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    atomicOr(status, 1u);
  }
  return false;
}

// the same wait without a status word (the caller reports through its output)
__device__ __forceinline__ bool mbar_wait_suspend(uint64_t *b, uint32_t parity, volatile uint32_t *abort_flag,
                                                  bool honour_abort = true) {
  return mbar_wait(b, parity, abort_flag, nullptr, honour_abort);
}

// programmatic dependent launch: wait for the preceding grid's results / let the next grid start
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::); }

// launch `kern` as the programmatic dependent of the kernel before it in the stream: its CTAs
// may be scheduled while that kernel finishes; the kernel must execute pdl_wait() before it
// touches global memory that earlier work reads or writes
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// result words set to zero by one thread (either may be NULL) before the kernel that
// accumulates into them, which is launched as this kernel's programmatic dependent (one copy
// per translation unit). Itself launched as a programmatic dependent (launch_clear_results): it
// waits for the kernel before it, and only then lets its dependent start, so a dependent that
// reads its inputs before its own wait never sees them before their producer has finished.
static __global__ void clear_results_kernel(uint32_t *w32, unsigned long long *w64) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    if (w32) *w32 = 0u;
    if (w64) *w64 = 0ull;
  }
}

static inline cudaError_t launch_clear_results(uint32_t *w32, unsigned long long *w64, cudaStream_t s) {
  return launch_pdl(clear_results_kernel, dim3(1), dim3(32), 0, s, w32, w64);
}

// 2-D tiled TMA load into this CTA's shared memory, completing on an mbarrier (no multicast)
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled TMA store from this CTA's shared memory (bulk-group completion). The writing threads
// order their shared-memory stores before it with fence_proxy_async_smem() and a barrier;
// rows of the box past the tensor's extent are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];\n" ::"l"(map),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// the issuing thread's committed bulk stores have read their shared-memory source
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
// ... and have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// per-thread asynchronous copies of 4 or 8 bytes, L1-allocating
__device__ __forceinline__ void cp_async_4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_8(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// the same with a source size: src_bytes (0 or the full size) are read, the rest of the
// destination is zero-filled; with 0 nothing is read
__device__ __forceinline__ void cp_async_4z(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_8z(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// one arrival on the mbarrier once all of this thread's earlier cp.async copies have landed
// (the barrier's expected count includes it)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *b) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(b)) : "memory");
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// tensor map over a fixed-4 code plane viewed as [rows][cols/2] bytes, 128-byte swizzled boxes
// of 128 bytes (4 groups) by box_rows rows; out-of-range rows and columns read as zero
inline cq_status code_tensor_map(CUtensorMap *tm, const uint8_t *plane, int64_t rows, int64_t cols,
                                 uint32_t box_rows, const char *who) {
  auto encode = encode_fn();
  if (!encode) return fail(CQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", who);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols / 2)};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(plane), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CQ_ERR_CUDA, "%s: code tensor map (%d)", who, static_cast<int>(r));
  return CQ_OK;
}

}  // namespace cq
