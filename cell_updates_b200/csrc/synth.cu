// synth.cu -- seeded device-side inputs (SplitMix64 counter generator), see include/cq_synth.h.
// Test-data synthesis only; it holds none of the quantizer's arithmetic.
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/cq_synth.h"

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t hash_at(uint64_t key, int64_t i) {
  return mix64(key + (static_cast<uint64_t>(i) + 1ull) * kGamma);
}

__device__ __forceinline__ float ih4(uint64_t u) {
  const int64_t s = static_cast<int64_t>(u & 0xFFFF) + static_cast<int64_t>((u >> 16) & 0xFFFF) +
                    static_cast<int64_t>((u >> 32) & 0xFFFF) + static_cast<int64_t>(u >> 48);
  return static_cast<float>(s - 2 * 65535);   // |value| < 2^18: exact
}

uint64_t key_of(uint64_t seed, uint32_t stream) { return mix64(seed * kGamma + stream); }

constexpr int kThreads = 256;

int grid(int64_t n) {
  const int64_t b = (n + kThreads - 1) / kThreads;
  return static_cast<int>(b < 148 * 16 ? b : 148 * 16);
}

#define GRID_STRIDE(i, n) \
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < (n); i += static_cast<int64_t>(gridDim.x) * kThreads)

__global__ void normal_kernel(float *out, int64_t n, uint64_t key, int64_t first, float mult) {
  GRID_STRIDE(i, n) out[i] = __fmul_rn(ih4(hash_at(key, first + i)), mult);
}

__global__ void words_kernel(uint64_t *out, int64_t n, uint64_t key, int64_t first) {
  GRID_STRIDE(i, n) out[i] = hash_at(key, first + i);
}

__global__ void scales_kernel(uint16_t *out, int64_t n, uint64_t key, int64_t first) {
  GRID_STRIDE(i, n) out[i] = static_cast<uint16_t>(0x1C00u | (hash_at(key, first + i) & 0x3FFu));
}

__global__ void zeros_kernel(uint8_t *out, int64_t n, uint64_t key, int64_t first) {
  GRID_STRIDE(i, n) out[i] = static_cast<uint8_t>((hash_at(key, first + i) >> 20) & 0xFu);
}

__global__ void resid_kernel(uint16_t *out, const uint16_t *scale, int64_t n, uint64_t key, int64_t first, float mult) {
  GRID_STRIDE(i, n) {
    const float sf = __half2float(__ushort_as_half(scale[i >> 6]));
    const float v = __fmul_rn(ih4(hash_at(key, first + i)), __fmul_rn(sf, mult));
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

int done() { return cudaGetLastError() == cudaSuccess ? 0 : 7; }

}  // namespace

extern "C" {

int cqs_normal_f32(float *out, int64_t n, uint64_t seed, uint32_t stream_id, int64_t first, float mult,
                   cq_stream_t stream) {
  if (n < 0 || first < 0 || (n && !out)) return 1;
  if (n) normal_kernel<<<grid(n), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, n, key_of(seed, stream_id), first, mult);
  return done();
}

int cqs_code_words(uint64_t *out, int64_t n, uint64_t seed, int64_t first, cq_stream_t stream) {
  if (n < 0 || first < 0 || (n && !out)) return 1;
  if (n) words_kernel<<<grid(n), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, n, key_of(seed, CQS_STREAM_CODE), first);
  return done();
}

int cqs_scales(uint16_t *out, int64_t n, uint64_t seed, int64_t first, cq_stream_t stream) {
  if (n < 0 || first < 0 || (n && !out)) return 1;
  if (n) scales_kernel<<<grid(n), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, n, key_of(seed, CQS_STREAM_SCALE), first);
  return done();
}

int cqs_zeros(uint8_t *out, int64_t n, uint64_t seed, int64_t first, cq_stream_t stream) {
  if (n < 0 || first < 0 || (n && !out)) return 1;
  if (n) zeros_kernel<<<grid(n), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, n, key_of(seed, CQS_STREAM_ZERO), first);
  return done();
}

int cqs_residual_bf16(uint16_t *out, const uint16_t *scale, int64_t n, uint64_t seed, int64_t first, float mult,
                      cq_stream_t stream) {
  if (n < 0 || first < 0 || first % 64 || n % 64 || (n && (!out || !scale))) return 1;
  if (n) resid_kernel<<<grid(n), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, scale, n, key_of(seed, CQS_STREAM_RESID), first, mult);
  return done();
}

}  // extern "C"
