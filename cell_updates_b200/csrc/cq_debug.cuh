// cq_debug.cuh -- in-kernel index checks, compiled in only under -DCQ_DEBUG.
//
// A check that fails records its site number in a device word (the first failure wins) and
// tells the caller to skip the access it guards; nothing traps, so a debug build run on a
// damaged input leaves the context usable and names where the first index went wrong. Release
// builds compile every check to `true` (no code). Sites are (unit << 8) | n with units
//   1 quantize, 2 pack/index, 3 project, 4 verify, 5 4-bit GEMV, 6 GEMM, 7 stage/VBQ GEMV,
//   8 reparameterization, 9 ReQuant, 15 self-test.
// Each translation unit owns one word; cq_debug_word (cq_api.cu) reads and clears them all.
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

namespace cq {
// bytes of dynamic shared memory this CTA was launched with
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t v;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;\n" : "=r"(v));
  return v;
}
}  // namespace cq

#ifdef CQ_DEBUG
namespace cq {
void register_debug_word(uint32_t (*take)());
namespace {
__device__ uint32_t g_debug_word;

__device__ __forceinline__ bool debug_check(bool ok, uint32_t site) {
  if (!ok) atomicCAS(&g_debug_word, 0u, site);
  return ok;
}

// the word of this unit, cleared (after the device has finished its work)
uint32_t take_debug_word() {
  uint32_t v = 0;
  const uint32_t z = 0;
  if (cudaMemcpyFromSymbol(&v, g_debug_word, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  if (cudaMemcpyToSymbol(g_debug_word, &z, sizeof z) != cudaSuccess) return 0xFFFFFFFFu;
  return v;
}

[[maybe_unused]] const bool g_debug_registered = (register_debug_word(&take_debug_word), true);
}  // namespace
}  // namespace cq
#define CQ_CHECK(ok, site) ::cq::debug_check(static_cast<bool>(ok), (site))
#else
#define CQ_CHECK(ok, site) (true)
#endif
