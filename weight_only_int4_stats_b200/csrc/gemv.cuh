// K3: W4A16 decode GEMM for M <= 16 tokens, Y[m, n] = sum_k x[m, k] * deq[n, k].
//
// builderai.tools "AWQ", "About" (kernels for 4-bit weights with 16-bit activations) and
// robotsatlas.com "AWQ", "Implementation pitfalls: Missing matched inference kernels"
// (dequantizing separately negates the speed-up, so dequantization happens in the kernel).
//
// HBM-bound: every packed weight is read once with 16-byte non-caching loads and never
// touches shared memory. A CTA of 8 warps owns 16 output rows; warp w takes groups
// w, w+8, ... of those rows and keeps several groups of loads in flight. Dequantization
// is register-only: a mask-and-or with 0x6400 turns two nibbles into the fp16 pair
// (1024+q_a, 1024+q_b) (the packed layout places consecutive k in the two halves), and one
// fp16 subtract (or a multiply-add for the nibbles stored 4 bits higher) leaves the exact
// integers q - z. Those feed mma.sync m16n8k16 (weights as the 16-row A operand, the
// activations as the 8-column B operand) into a per-group fp32 accumulator that is scaled
// once per group by the fp16 scale: y = sum_j s_j * sum_{k in j} x_k (q_k - z_j).
// The 8 warps' partial sums are added in a fixed order through shared memory.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16;
constexpr int kGemvPrefetch = 4;   // groups of loads in flight per warp

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four fp16 pairs (q-z) from one packed word: pairs (k0,k1), (k2,k3), (k4,k5), (k6,k7).
__device__ __forceinline__ void dequant_word_qz(uint32_t w, __half2 bias_lo, __half2 bias_hi,
                                                uint32_t (&out)[4]) {
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const uint32_t w8 = w >> 8;
  const uint32_t v0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  const uint32_t v1 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  const uint32_t v2 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
  const uint32_t v3 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
  out[0] = h2_as_u32(__hsub2(u32_as_h2(v0), bias_lo));
  out[1] = h2_as_u32(__hfma2(u32_as_h2(v1), sixteenth, bias_hi));
  out[2] = h2_as_u32(__hsub2(u32_as_h2(v2), bias_lo));
  out[3] = h2_as_u32(__hfma2(u32_as_h2(v3), sixteenth, bias_hi));
}

// x fragment for one MMA: two fp16 pairs, optionally multiplied by inv_s.
__device__ __forceinline__ uint4 load_x8(const __half* __restrict__ X, int64_t K, int m,
                                         int64_t k, bool valid, const float* __restrict__ inv_s) {
  if (!valid) return make_uint4(0u, 0u, 0u, 0u);
  uint4 v = *reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K + k);
  if (inv_s != nullptr) {
    const float4 s0 = *reinterpret_cast<const float4*>(inv_s + k);
    const float4 s1 = *reinterpret_cast<const float4*>(inv_s + k + 4);
    float2 f;
    f = __half22float2(u32_as_h2(v.x));
    v.x = h2_as_u32(__floats2half2_rn(f.x * s0.x, f.y * s0.y));
    f = __half22float2(u32_as_h2(v.y));
    v.y = h2_as_u32(__floats2half2_rn(f.x * s0.z, f.y * s0.w));
    f = __half22float2(u32_as_h2(v.z));
    v.z = h2_as_u32(__floats2half2_rn(f.x * s1.x, f.y * s1.y));
    f = __half22float2(u32_as_h2(v.w));
    v.w = h2_as_u32(__floats2half2_rn(f.x * s1.z, f.y * s1.w));
  }
  return v;
}

template <int kNTiles>   // 1: M <= 8, 2: M <= 16
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_w4a16_kernel(
    const __half* __restrict__ X, int M, const uint32_t* __restrict__ qweight,
    const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t N, int64_t K,
    const float* __restrict__ inv_s, __half* __restrict__ Y) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int r = lane >> 2;            // fragment row (and B column)
  const int c = lane & 3;             // quad position: owns k in [32c, 32c+32) of a group
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kGemvRows;
  const int64_t nA = n0 + r, nB = n0 + r + 8;
  const bool okA = nA < N, okB = nB < N;
  const int64_t G = K / kGroup;
  const int64_t wpr = K / 8;          // packed words per row

  float total[kNTiles][4];
#pragma unroll
  for (int t = 0; t < kNTiles; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) total[t][i] = 0.0f;

  // Ring of prefetched groups: two 16-byte weight loads (rows r and r+8), zeros, scales.
  uint4 wa[kGemvPrefetch], wb[kGemvPrefetch];
  uint8_t za[kGemvPrefetch], zb[kGemvPrefetch];
  __half sa[kGemvPrefetch], sb[kGemvPrefetch];
  auto issue = [&](int slot, int64_t g) {
    if (g < G) {
      const int64_t wo = g * 16 + c * 4;
      wa[slot] = okA ? ldg_nc_v4(qweight + nA * wpr + wo) : make_uint4(0u, 0u, 0u, 0u);
      wb[slot] = okB ? ldg_nc_v4(qweight + nB * wpr + wo) : make_uint4(0u, 0u, 0u, 0u);
      za[slot] = okA ? zeros[g * N + nA] : 0;
      zb[slot] = okB ? zeros[g * N + nB] : 0;
      sa[slot] = okA ? scales[g * N + nA] : __float2half(0.0f);
      sb[slot] = okB ? scales[g * N + nB] : __float2half(0.0f);
    }
  };
#pragma unroll
  for (int p = 0; p < kGemvPrefetch; ++p) issue(p, warp + static_cast<int64_t>(p) * kGemvWarps);

  for (int64_t gi = warp; gi < G; gi += kGemvWarps * kGemvPrefetch) {
#pragma unroll
    for (int p = 0; p < kGemvPrefetch; ++p) {
      const int64_t g = gi + static_cast<int64_t>(p) * kGemvWarps;
      if (g >= G) break;
      const uint4 wA = wa[p], wB = wb[p];
      const uint32_t zA = za[p], zB = zb[p];
      const float scA = __half2float(sa[p]), scB = __half2float(sb[p]);
      issue(p, g + static_cast<int64_t>(kGemvPrefetch) * kGemvWarps);
      // biases: 1024 + z and -(64 + z) as fp16 pairs, built from the bit patterns
      const __half2 loA = u32_as_h2((0x6400u | zA) * 0x00010001u);
      const __half2 hiA = __hneg2(u32_as_h2((0x5400u | (zA << 4)) * 0x00010001u));
      const __half2 loB = u32_as_h2((0x6400u | zB) * 0x00010001u);
      const __half2 hiB = __hneg2(u32_as_h2((0x5400u | (zB << 4)) * 0x00010001u));
      float acc[kNTiles][4];
#pragma unroll
      for (int t = 0; t < kNTiles; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;
      const uint32_t wordsA[4] = {wA.x, wA.y, wA.z, wA.w};
      const uint32_t wordsB[4] = {wB.x, wB.y, wB.z, wB.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t qa[4], qb[4];
        dequant_word_qz(wordsA[j], loA, hiA, qa);
        dequant_word_qz(wordsB[j], loB, hiB, qb);
        const int64_t kx = g * kGroup + 32 * c + 8 * j;
#pragma unroll
        for (int t = 0; t < kNTiles; ++t) {
          const int m = r + 8 * t;
          const uint4 xv = load_x8(X, K, m, kx, m < M, inv_s);
          // MMA for k-offsets 0..3 of the word, then 4..7
          const uint32_t a0[4] = {qa[0], qb[0], qa[1], qb[1]};
          mma_16816(acc[t], a0, xv.x, xv.y);
          const uint32_t a1[4] = {qa[2], qb[2], qa[3], qb[3]};
          mma_16816(acc[t], a1, xv.z, xv.w);
        }
      }
#pragma unroll
      for (int t = 0; t < kNTiles; ++t) {
        total[t][0] = fmaf(scA, acc[t][0], total[t][0]);
        total[t][1] = fmaf(scA, acc[t][1], total[t][1]);
        total[t][2] = fmaf(scB, acc[t][2], total[t][2]);
        total[t][3] = fmaf(scB, acc[t][3], total[t][3]);
      }
    }
  }

  // Fixed-order reduction over the 8 warps.
  __shared__ float red[kGemvWarps][kNTiles][4][32];
#pragma unroll
  for (int t = 0; t < kNTiles; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][t][i][lane] = total[t][i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int t = 0; t < kNTiles; ++t) {
      float v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) s += red[w][t][i][lane];
        v[i] = s;
      }
      // accumulator fragment: (row r, cols 2c, 2c+1) and (row r+8, cols 2c, 2c+1);
      // rows are output features n, columns are tokens m.
      const int m0 = 8 * t + 2 * c, m1 = m0 + 1;
      if (okA) {
        if (m0 < M) Y[static_cast<int64_t>(m0) * N + nA] = __float2half_rn(v[0]);
        if (m1 < M) Y[static_cast<int64_t>(m1) * N + nA] = __float2half_rn(v[1]);
      }
      if (okB) {
        if (m0 < M) Y[static_cast<int64_t>(m0) * N + nB] = __float2half_rn(v[2]);
        if (m1 < M) Y[static_cast<int64_t>(m1) * N + nB] = __float2half_rn(v[3]);
      }
    }
  }
}

}  // namespace awq
