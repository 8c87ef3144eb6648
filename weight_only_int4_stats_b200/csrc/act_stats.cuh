// K1: per-input-channel activation magnitude s_x[k] = (1/M) sum_m |x[m, k]|.
//
// robotsatlas.com "AWQ", "How it works" and "Components: Activation saliency analysis":
// the calibration set is passed through the layer and the activation magnitude of every
// input channel is measured. The statistic is the mean absolute value over all tokens.
//
// HBM-bound column reduction. Pass 1: a CTA of 32 column lanes x 8 row lanes covers 256
// channels (one 16-byte load of 8 fp16 per lane and row) over a slice of the rows and
// accumulates |x| in fp64; the 8 row lanes are combined in a fixed order and the slice's
// partial sums go to the workspace. Pass 2 adds the slices in order and divides by M.
// fp64 accumulation of fp16 inputs is exact whenever the running sums span fewer than 53
// bits, so the result does not depend on the split.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kStatsCols = 256;   // channels per CTA (32 lanes x 8 fp16)
constexpr int kStatsRowLanes = 8;

__global__ void __launch_bounds__(256) act_stats_partial_kernel(const __half* __restrict__ X,
                                                                int64_t M, int64_t K,
                                                                int64_t rows_per_split,
                                                                double* __restrict__ part) {
  const int lane = threadIdx.x & 31;
  const int rl = threadIdx.x >> 5;                       // row lane 0..7
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kStatsCols + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(M, r0 + rows_per_split);
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  if (col0 < K) {
    const __half* p = X + col0;
    int64_t r = r0 + rl;
    // four independent 16-byte loads in flight per iteration
    for (; r + 3 * kStatsRowLanes < r1; r += 4 * kStatsRowLanes) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = AWQ_IN_BOUNDS(r + u * kStatsRowLanes < M && col0 + 8 <= K)
                   ? ldg_nc_v4(p + (r + u * kStatsRowLanes) * K)
                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __half2* h = reinterpret_cast<const __half2*>(&v[u]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 f = __half22float2(h[i]);
          acc[2 * i] += fabs(static_cast<double>(f.x));
          acc[2 * i + 1] += fabs(static_cast<double>(f.y));
        }
      }
    }
    for (; r < r1; r += kStatsRowLanes) {
      uint4 v = AWQ_IN_BOUNDS(r < M && col0 + 8 <= K) ? ldg_nc_v4(p + r * K)
                                                       : make_uint4(0u, 0u, 0u, 0u);
      const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        acc[2 * i] += fabs(static_cast<double>(f.x));
        acc[2 * i + 1] += fabs(static_cast<double>(f.y));
      }
    }
  }
  __shared__ double red[kStatsRowLanes][kStatsCols];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rl][lane * 8 + i] = acc[i];
  __syncthreads();
  // 256 threads: thread t finalises channel t of the tile, adding row lanes in order.
  const int t = threadIdx.x;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kStatsCols + t;
  if (c < K) {
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < kStatsRowLanes; ++j) s += red[j][t];
    if (AWQ_IN_BOUNDS(blockIdx.y < gridDim.y)) part[static_cast<int64_t>(blockIdx.y) * K + c] = s;
  }
}

__global__ void act_stats_finish_kernel(const double* __restrict__ part, int splits, int64_t M,
                                        int64_t K, float* __restrict__ s_x) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double s = 0.0;
  for (int j = 0; j < splits; ++j) s += part[static_cast<int64_t>(j) * K + k];
  s_x[k] = __double2float_rn(s / static_cast<double>(M));
}

// Split count so that the grid covers the GPU several times over.
inline int act_stats_splits(int64_t M, int64_t K, int num_sms) {
  const int64_t col_tiles = (K + kStatsCols - 1) / kStatsCols;
  int64_t want = (static_cast<int64_t>(num_sms) * 8 + col_tiles - 1) / col_tiles;
  int64_t by_rows = (M + 63) / 64;                       // at least 64 rows per slice
  int64_t s = want < by_rows ? want : by_rows;
  if (s < 1) s = 1;
  if (s > 65535) s = 65535;
  return static_cast<int>(s);
}

}  // namespace awq
