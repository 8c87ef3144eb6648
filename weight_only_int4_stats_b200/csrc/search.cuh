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
  for (int j = 0; j < m_tiles; ++j) r += p[static_cast<int64_t>(j) * rows_total];
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
// winning scale row; CTA 0 also writes the index.
__global__ void search_pick_kernel(const double* __restrict__ losses, int n_alpha,
                                   const float* __restrict__ s_table, int64_t K,
                                   int32_t* __restrict__ best_idx, float* __restrict__ best_s) {
  int best = 0;
  double bl = losses[0];
  for (int a = 1; a < n_alpha; ++a) {
    const double l = losses[a];
    if (l < bl) { bl = l; best = a; }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) best_idx[0] = best;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k < K) best_s[k] = s_table[static_cast<int64_t>(best) * K + k];
}

// x'[m, k] = fp16(x[m, k] * inv_s[k]) for the tensor-core GEMM's activation operand.
__global__ void prescale_x_kernel(const __half* __restrict__ X, const float* __restrict__ inv_s,
                                  int64_t M, int64_t K, __half* __restrict__ Xs) {
  const int64_t i8 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i8 >= M * K) return;
  const int64_t k = i8 % K;
  uint4 v = *reinterpret_cast<const uint4*>(X + i8);
  const float4 s0 = *reinterpret_cast<const float4*>(inv_s + k);
  const float4 s1 = *reinterpret_cast<const float4*>(inv_s + k + 4);
  float2 f;
  f = __half22float2(u32_as_h2(v.x)); v.x = h2_as_u32(__floats2half2_rn(f.x * s0.x, f.y * s0.y));
  f = __half22float2(u32_as_h2(v.y)); v.y = h2_as_u32(__floats2half2_rn(f.x * s0.z, f.y * s0.w));
  f = __half22float2(u32_as_h2(v.z)); v.z = h2_as_u32(__floats2half2_rn(f.x * s1.x, f.y * s1.y));
  f = __half22float2(u32_as_h2(v.w)); v.w = h2_as_u32(__floats2half2_rn(f.x * s1.z, f.y * s1.w));
  *reinterpret_cast<uint4*>(Xs + i8) = v;
}

}  // namespace awq
