// k_requant.cu -- ReQuant fixed-grid refinement of the codes.
//
// Page 1 (thelatestinai.com/papers/2608.20873), ReQuant abstract: after any initializer, a
// backpropagation-free stage revisits the integer assignments on the fixed grid; every accepted
// update strictly lowers the mean squared reconstruction error and stays on the grid; sweeps
// repeat over a round-to-nearest start. Reading (the abstract fixes neither the error's data nor
// the moves): the error is the layer's output error on calibration activations X,
//     E(q) = sum_n d_n^T H d_n,   d_n = w_n - s (q_n - z),   H = X^T X (binary64, symmetric)
// (in weight space round-to-nearest is already optimal); the grid (s, z) is frozen; a candidate
// update moves one code to a neighbouring level inside [0, L]. Rows are independent. A sweep of
// row n visits k = 0 .. K-1; with S the scale of k's group, t2 = (S*S)*H_kk, t4 = (2*S)*g_k, the
// moves change E by up = t2 - t4 (q_k < L) and down = t2 + t4 (q_k > 0); the smaller is taken when
// strictly negative (up on a tie), and then g_j <- g_j - delta*H_kj for every j, delta = +-S.
// Every operation is one binary64 operation rounded to nearest (this unit is compiled without
// contraction) and each g_j receives its updates in increasing k, so the codes equal the oracle's
// bit for bit.
//
// Two kernels:
//  * rq_gradient_kernel: g = D H for all rows, D[n, k] = (double)w - S (q - z) formed on the fly,
//    a 64 x 64 output tile per CTA, every output summed over k in increasing order (k tiles in
//    order, k in order within a tile), H read as rows k (H symmetric, so H[k, j] = H[j, k]);
//    rq_error_kernel then forms err[n] = sum_k d_k g_k in increasing k.
//  * rq_sweep_kernel: one warp per row, the row's g in shared memory; the warp decides each k
//    (all lanes compute the same decision from the broadcast g_k) and, on a move, updates its g
//    with the row k of H (lane-strided, coalesced).
#include "cq_internal.cuh"

namespace cq {
namespace {

constexpr int kRqTile = 64;          // gradient tile: 64 rows x 64 columns of g
constexpr int kRqK = 16;             // k per shared-memory stage
constexpr int kRqThreads = 256;      // 16 x 16 threads, 4 x 4 outputs each
constexpr int kSweepMaxWarps = 8;    // rows per sweep CTA when their g fit in shared memory
constexpr size_t kSweepSmem = 200 * 1024;

__device__ __forceinline__ double code_residual(const float *w, const uint16_t *scale, const uint8_t *zero,
                                                const uint8_t *codes, int64_t n, int64_t k, int64_t K) {
  const int64_t g = n * (K >> 6) + (k >> 6);
  const double S = static_cast<double>(f16_bits_to_f32(scale[g]));
  const int dq = static_cast<int>(codes[n * K + k]) - static_cast<int>(zero[g]);
  return __dsub_rn(static_cast<double>(w[n * K + k]), __dmul_rn(S, static_cast<double>(dq)));
}

// g[n, j] for a 64 x 64 tile; out of range rows / columns are neither read nor written
__global__ void __launch_bounds__(kRqThreads)
rq_gradient_kernel(const float *__restrict__ w, const double *__restrict__ H, const uint16_t *__restrict__ scale,
                   const uint8_t *__restrict__ zero, const uint8_t *__restrict__ codes, int64_t N, int64_t K,
                   double *__restrict__ g) {
  __shared__ double sD[kRqK][kRqTile + 1];
  __shared__ double sH[kRqK][kRqTile];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kRqTile, j0 = static_cast<int64_t>(blockIdx.x) * kRqTile;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  for (int64_t k0 = 0; k0 < K; k0 += kRqK) {
    // stage D[n0 .. +63][k0 .. +15] and H[k0 .. +15][j0 .. +63] (K is a multiple of 64)
    for (int i = threadIdx.x; i < kRqK * kRqTile; i += kRqThreads) {
      const int kk = i / kRqTile, c = i % kRqTile;
      const int64_t n = n0 + c, j = j0 + c;
      sD[kk][c] = n < N ? code_residual(w, scale, zero, codes, n, k0 + kk, K) : 0.0;
      sH[kk][c] = j < K ? H[(k0 + kk) * K + j] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRqK; ++kk) {
      double dv[4], hv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) dv[a] = sD[kk][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < 4; ++b) hv[b] = sH[kk][tx * 4 + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __dadd_rn(acc[a][b], __dmul_rn(hv[b], dv[a]));
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int64_t n = n0 + ty * 4 + a, j = j0 + tx * 4 + b;
      if (n < N && j < K) g[n * K + j] = acc[a][b];
    }
}

// err[n] = sum_k d_k g_k in increasing k (one warp per row: lane 0 sums, the other lanes fetch)
__global__ void rq_error_kernel(const float *__restrict__ w, const uint16_t *__restrict__ scale,
                                const uint8_t *__restrict__ zero, const uint8_t *__restrict__ codes,
                                const double *__restrict__ g, int64_t N, int64_t K, double *__restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (n >= N) return;
  double e = 0.0;
  for (int64_t k0 = 0; k0 < K; k0 += 32) {
    const double p = __dmul_rn(code_residual(w, scale, zero, codes, n, k0 + lane, K), g[n * K + k0 + lane]);
    for (int i = 0; i < 32; ++i) e = __dadd_rn(e, __shfl_sync(0xffffffffu, p, i));
  }
  if (lane == 0) err[n] = e;
}

// one warp per row: blockDim.x / 32 rows per CTA, each row's g (K doubles) in shared memory
__global__ void __launch_bounds__(32 * kSweepMaxWarps)
rq_sweep_kernel(const double *__restrict__ H, const uint16_t *__restrict__ scale, uint8_t *__restrict__ codes,
                double *__restrict__ g, int64_t N, int64_t K, int L, int sweeps,
                unsigned long long *__restrict__ moves) {
  extern __shared__ double sg[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
  if (n >= N) return;
  double *gr = sg + static_cast<int64_t>(warp) * K;
  if (!CQ_CHECK(static_cast<int64_t>(warp + 1) * K * 8 <= dynamic_smem_bytes(), 0x0901u)) return;
  for (int64_t j = lane; j < K; j += 32) gr[j] = g[n * K + j];
  __syncwarp();
  const int64_t KG = K >> 6;
  uint8_t *qn = codes + n * K;
  unsigned long long mv = 0;
  const int Ki = static_cast<int>(K);
  for (int sw = 0; sw < sweeps; ++sw) {
    for (int k0 = 0; k0 < Ki; k0 += 32) {
      // the lanes fetch 32 codes and the 32 diagonal entries of H at a time; every lane then
      // walks them in order
      int qv = qn[k0 + lane];
      const double hdiag = H[static_cast<int64_t>(k0 + lane) * (K + 1)];
      const double S = static_cast<double>(f16_bits_to_f32(scale[n * KG + (k0 >> 6)]));
      const double SS = __dmul_rn(S, S), S2 = __dmul_rn(2.0, S);
      for (int i = 0; i < 32; ++i) {
        const int k = k0 + i;
        const int q = __shfl_sync(0xffffffffu, qv, i);
        const double gk = gr[k];
        const double t2 = __dmul_rn(SS, __shfl_sync(0xffffffffu, hdiag, i));
        const double t4 = __dmul_rn(S2, gk);
        const double up = __dsub_rn(t2, t4), down = __dadd_rn(t2, t4);
        int step = (q < L && up < 0.0) ? 1 : 0;
        if (q > 0 && down < 0.0 && (step == 0 || down < up)) step = -1;
        (void)CQ_CHECK(q + step >= 0 && q + step <= L, 0x0902u);
        if (step) {                      // warp-uniform: every lane took the same decision
          const double delta = step > 0 ? S : -S;
          if (lane == i) qv = q + step;
          const double *hk = H + static_cast<int64_t>(k) * K;
          __syncwarp();
          // row k of H, lane-strided and coalesced (measured faster than explicitly batching
          // the loads, which the compiler does on its own); each g_j receives this one update
          for (int j = lane; j < Ki; j += 32) gr[j] = __dsub_rn(gr[j], __dmul_rn(delta, hk[j]));
          __syncwarp();
          ++mv;
        }
      }
      qn[k0 + lane] = static_cast<uint8_t>(qv);
    }
  }
  if (lane == 0 && moves) moves[n] = mv;
}

}  // namespace

// the longest row whose g fits a sweep CTA's shared memory
int64_t requant_max_cols() { return static_cast<int64_t>(kSweepSmem / sizeof(double)) / 64 * 64; }

size_t requant_workspace(int64_t rows, int64_t cols) {
  return static_cast<size_t>(rows) * static_cast<size_t>(cols) * sizeof(double);
}

cq_status launch_requant(const float *w, int64_t N, int64_t K, const double *H, const uint16_t *scale,
                         const uint8_t *zero, int b, uint8_t *codes, int sweeps, double *err_before, double *err_after,
                         uint64_t *moves, double *g, cudaStream_t s) {
  if (N == 0 || K == 0) return CQ_OK;
  const dim3 ggrid(static_cast<unsigned>((K + kRqTile - 1) / kRqTile), static_cast<unsigned>((N + kRqTile - 1) / kRqTile));
  const int err_warps = 8;
  const unsigned err_blocks = static_cast<unsigned>((N + err_warps - 1) / err_warps);
  rq_gradient_kernel<<<ggrid, kRqThreads, 0, s>>>(w, H, scale, zero, codes, N, K, g);
  cq_status st = launch_check("cq_requant_refine: gradient");
  if (st != CQ_OK) return st;
  if (err_before) {
    rq_error_kernel<<<err_blocks, 32 * err_warps, 0, s>>>(w, scale, zero, codes, g, N, K, err_before);
    st = launch_check("cq_requant_refine: error before");
    if (st != CQ_OK) return st;
  }
  const size_t row_bytes = static_cast<size_t>(K) * sizeof(double);
  int rows_per_cta = static_cast<int>(kSweepSmem / row_bytes);
  rows_per_cta = rows_per_cta > kSweepMaxWarps ? kSweepMaxWarps : rows_per_cta;
  const size_t smem = static_cast<size_t>(rows_per_cta) * row_bytes;
  st = cuda_check(cudaFuncSetAttribute(rq_sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)), "cq_requant_refine: shared memory attribute");
  if (st != CQ_OK) return st;
  rq_sweep_kernel<<<static_cast<unsigned>((N + rows_per_cta - 1) / rows_per_cta), 32 * rows_per_cta, smem, s>>>(
      H, scale, codes, g, N, K, (1 << b) - 1, sweeps, reinterpret_cast<unsigned long long *>(moves));
  st = launch_check("cq_requant_refine: sweep");
  if (st != CQ_OK) return st;
  if (err_after) {
    rq_gradient_kernel<<<ggrid, kRqThreads, 0, s>>>(w, H, scale, zero, codes, N, K, g);
    st = launch_check("cq_requant_refine: gradient after");
    if (st != CQ_OK) return st;
    rq_error_kernel<<<err_blocks, 32 * err_warps, 0, s>>>(w, scale, zero, codes, g, N, K, err_after);
    st = launch_check("cq_requant_refine: error after");
  }
  return st;
}

}  // namespace cq
