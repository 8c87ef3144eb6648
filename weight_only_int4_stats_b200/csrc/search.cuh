// K5 tail: fold the error GEMM's per-(row, token tile) partial sums into per-row losses and
// per-grid-point losses in a fixed order, then pick the grid point with the lowest loss.
//
// robotsatlas.com "AWQ", "How it works" and "Key mechanisms: Grid search over scales
// minimizing the layer output error". Ties go to the smallest grid index.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kReduceThreads = 256;

// Per-row losses: row r of grid point a adds its token-tile (or, for the Gram form,
// channel-tile) partials in tile order (partials are stored tile-major, so consecutive
// threads read consecutive rows), times `scale` (the Gram form's token count M, 1 otherwise).
__global__ void __launch_bounds__(kReduceThreads) search_row_loss_kernel(
    const double* __restrict__ row_part, int64_t N, int64_t N_pad, int n_alpha, int m_tiles,
    double scale, double* __restrict__ row_loss /*[n_alpha, N]*/) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(n_alpha) * N) return;
  const int64_t a = i / N, n = i % N;
  const int64_t rows_total = static_cast<int64_t>(n_alpha) * N_pad;
  const double* p = row_part + a * N_pad + n;
  double r = 0.0;
  for (int j = 0; j < m_tiles; ++j)
    if (AWQ_IN_BOUNDS(a * N_pad + n < rows_total)) r += p[static_cast<int64_t>(j) * rows_total];
  row_loss[i] = r * scale;
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

namespace awq {

// ---------------------------------------------------------------------------------------
// The Gram form of the search loss. For one row e of the error operand (e[k] = deq/s - w),
//   sum_m (sum_k e[k] x[m, k])^2 = e G e^T,   G = X^T X  (K x K, shared by every row and
// every grid point), which costs N K^2 per grid point instead of N K M. To keep both
// operands in fp16 range for any number of tokens, G is normalised to G'[i][j] =
// G[i][j] / (d_i d_j) with d_k = sqrt(G[k][k]) (a correlation matrix: unit diagonal, entries
// in [-1, 1]) and e is scaled to e'[k] = e[k] * r_k with r_k = d_k / sqrt(M) (the channel's
// root mean square), so that e G e^T = M * e' G' e'^T.
// ---------------------------------------------------------------------------------------

// XT[k][m] = X[m][k] for m < M, 0 for M <= m < M_pad (tokens contiguous per channel, the
// K-major layout of the contraction over tokens). 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) transpose_pad_kernel(const __half* __restrict__ X,
                                                            int64_t M, int64_t K, int64_t M_pad,
                                                            __half* __restrict__ XT) {
  __shared__ __half tile[32][33];
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * 32, k0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 8 * i, k = k0 + tx;
    tile[ty + 8 * i][tx] = (m < M && k < K) ? X[m * K + k] : __float2half(0.0f);
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + ty + 8 * i, m = m0 + tx;
    if (k < K && m < M_pad && AWQ_IN_BOUNDS(m < M_pad)) XT[k * M_pad + m] = tile[tx][ty + 8 * i];
  }
}

// rms[k] = sqrt(G[k][k] / M) (0 for a dead channel).
__global__ void gram_rms_kernel(const float* __restrict__ G, int64_t K, int64_t M,
                                float* __restrict__ rms) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k < K) rms[k] = sqrtf(G[k * K + k] / static_cast<float>(M));
}

// G2[i] = [hi | lo] of G'[i][j] = G[i][j] / (sqrt(G[i][i]) sqrt(G[j][j])) (0 when either
// channel is dead): hi = fp16(g'), lo = fp16((g' - hi) * 2^12), as for the error operand.
// Only the tiles of G on or above the diagonal are computed; G[i][j] is read as
// G[min(i,j)][max(i,j)], so G' is exactly symmetric.
__global__ void gram_normalize_kernel(const float* __restrict__ G, int64_t K,
                                      __half* __restrict__ G2) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t i = blockIdx.y;
  if (j >= K) return;
  const float gii = G[i * K + i], gjj = G[j * K + j];
  const int64_t lo = i < j ? i : j, hi_ = i < j ? j : i;
  float g = 0.0f;
  if (gii > 0.0f && gjj > 0.0f) g = G[lo * K + hi_] / (sqrtf(gii) * sqrtf(gjj));
  const __half hi = __float2half_rn(g);
  G2[i * 2 * K + j] = hi;
  G2[i * 2 * K + K + j] = __float2half_rn(__fmul_rn(__fsub_rn(g, __half2float(hi)), 4096.0f));
}

}  // namespace awq
