// K5 tail: fold the error GEMM's per-(row, token tile) partial sums into per-row losses and
// per-grid-point losses in a fixed order, then pick the grid point with the lowest loss.
//
// robotsatlas.com "AWQ", "How it works" and "Key mechanisms: Grid search over scales
// minimizing the layer output error". Ties go to the smallest grid index.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kReduceThreads = 256;

// Per-row losses: row r of grid point a adds its token-tile partials in tile order
// (partials are stored token-tile-major, so consecutive threads read consecutive rows).
__global__ void __launch_bounds__(kReduceThreads) search_row_loss_kernel(
    const double* __restrict__ row_part, int64_t N, int64_t N_pad, int n_alpha, int m_tiles,
    double* __restrict__ row_loss /*[n_alpha, N]*/) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(n_alpha) * N) return;
  const int64_t a = i / N, n = i % N;
  const int64_t rows_total = static_cast<int64_t>(n_alpha) * N_pad;
  const double* p = row_part + a * N_pad + n;
  double r = 0.0;
  for (int j = 0; j < m_tiles; ++j)
    if (AWQ_IN_BOUNDS(a * N_pad + n < rows_total)) r += p[static_cast<int64_t>(j) * rows_total];
  row_loss[i] = r;
}

// One CTA per grid point a: the N row losses are added by thread t in the order
// t, t+256, ... and the 256 thread sums by a fixed binary tree.
__global__ void __launch_bounds__(kReduceThreads) search_reduce_kernel(
    const double* __restrict__ row_loss, int64_t N, double* __restrict__ losses) {
  const int a = blockIdx.x;
  const int t = threadIdx.x;
  double acc = 0.0;
  for (int64_t n = t; n < N; n += kReduceThreads) acc += row_loss[static_cast<int64_t>(a) * N + n];
  __shared__ double red[kReduceThreads];
  red[t] = acc;
  __syncthreads();
#pragma unroll
  for (int w = kReduceThreads / 2; w > 0; w >>= 1) {
    if (t < w) red[t] += red[t + w];
    __syncthreads();
  }
  if (t == 0) losses[a] = red[0];
}

// Every CTA finds the first minimum itself (n_alpha is small) and copies its slice of the
// winning scale row (and, when asked, of its correctly rounded reciprocal); CTA 0 also writes
// the index.
__global__ void search_pick_kernel(const double* __restrict__ losses, int n_alpha,
                                   const float* __restrict__ s_table,
                                   const float* __restrict__ inv_table, int64_t K,
                                   int32_t* __restrict__ best_idx, float* __restrict__ best_s,
                                   float* __restrict__ best_inv_s) {
  int best = 0;
  double bl = losses[0];
  for (int a = 1; a < n_alpha; ++a) {
    const double l = losses[a];
    if (l < bl) { bl = l; best = a; }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) best_idx[0] = best;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k < K && AWQ_IN_BOUNDS(best >= 0 && best < n_alpha)) {
    best_s[k] = s_table[static_cast<int64_t>(best) * K + k];
    if (best_inv_s != nullptr) best_inv_s[k] = inv_table[static_cast<int64_t>(best) * K + k];
  }
}

}  // namespace awq
