// K2: group-wise asymmetric quantization of W diag(s), packed into this library's layout,
// and the search's error-operand builder that runs the same quantizer per grid point.
//
// robotsatlas.com "AWQ", "Components: Group-wise 4-bit quantization" (groups of 128, one
// scale per group) and "Hyperparameters" (4 or 3 bits); builderai.tools "AWQ", "About"
// (real INT4 weights are written). Per row n and group j, in IEEE fp32 with one rounding
// per operation and no contraction:
//   w' = w * s[k];  mx, mn = max, min of w' over the group;
//   scale = max((mx - mn) / qmax, 1e-5) rounded to fp16 -> sc;
//   z = clamp(rint(-mn / sc), 0, qmax);  q = clamp(rint(w' / sc) + z, 0, qmax).
//
// One warp owns one (row, group): lane l holds k = 128 j + 4 l .. 4 l + 3, the group's min
// and max come from five xor-shuffles each, and the packed words are assembled with
// xor-shuffle ORs between the lanes that share a word. A CTA of 8 warps covers 32 rows of
// one group so that the [G, N] scales and zeros leave as contiguous runs.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kQuantRowsPerCta = 32;

struct GroupQuant {
  float q[4];     // codes of this lane's 4 elements, as exact small integers
  float sc;       // fp16-rounded scale, widened
  float z;        // zero point
  __half sc_h;
};

template <int kBits>
__device__ __forceinline__ GroupQuant quantize_lane(const float (&w)[4]) {
  constexpr float qmax = static_cast<float>((1 << kBits) - 1);
  float mx = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
  float mn = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  GroupQuant g;
  float scale = __fdiv_rn(__fsub_rn(mx, mn), qmax);
  scale = fmaxf(scale, 1e-5f);
  g.sc_h = __float2half_rn(scale);
  g.sc = __half2float(g.sc_h);
  g.z = fminf(fmaxf(rintf(__fdiv_rn(-mn, g.sc)), 0.0f), qmax);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    g.q[i] = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[i], g.sc)), g.z), 0.0f), qmax);
  return g;
}

// Loads this lane's 4 weights of (row, group) and applies the per-channel scale.
__device__ __forceinline__ void load_scaled(const __half* __restrict__ W, int64_t K, int64_t n,
                                            int64_t k0, const float* __restrict__ s,
                                            float (&w)[4], float (&w_raw)[4]) {
  const uint2 raw = *reinterpret_cast<const uint2*>(W + n * K + k0);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  w_raw[0] = a.x; w_raw[1] = a.y; w_raw[2] = b.x; w_raw[3] = b.y;
  if (s != nullptr) {
    const float4 sv = *reinterpret_cast<const float4*>(s + k0);
    w[0] = __fmul_rn(w_raw[0], sv.x);
    w[1] = __fmul_rn(w_raw[1], sv.y);
    w[2] = __fmul_rn(w_raw[2], sv.z);
    w[3] = __fmul_rn(w_raw[3], sv.w);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = w_raw[i];
  }
}

// 4-bit: k-offset o of a word sits in nibble position o/2 + 4*(o%2).
__device__ __forceinline__ uint32_t nibble_pos(int o) { return (o >> 1) + 4 * (o & 1); }

template <int kBits>
__global__ void __launch_bounds__(256) quantize_pack_kernel(
    const __half* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ s,
    uint32_t* __restrict__ qweight, __half* __restrict__ scales, uint8_t* __restrict__ zeros) {
  __shared__ __half sh_scale[kQuantRowsPerCta];
  __shared__ uint8_t sh_zero[kQuantRowsPerCta];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t j = blockIdx.y;                          // group index
  const int64_t k0 = j * kGroup + 4 * lane;
  const int64_t words_per_row = (kBits == 4) ? K / 8 : 3 * K / 32;
#pragma unroll 1
  for (int rr = 0; rr < kQuantRowsPerCta / 8; ++rr) {
    const int lr = warp * (kQuantRowsPerCta / 8) + rr;  // local row 0..31
    const int64_t n = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta + lr;
    if (n >= N) break;                                   // warp-uniform
    float w[4], w_raw[4];
    load_scaled(W, K, n, k0, s, w, w_raw);
    const GroupQuant g = quantize_lane<kBits>(w);
    if (kBits == 4) {
      uint32_t part = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int o = 4 * (lane & 1) + i;
        part |= static_cast<uint32_t>(g.q[i]) << (4 * nibble_pos(o));
      }
      part |= __shfl_xor_sync(0xffffffffu, part, 1);
      if ((lane & 1) == 0) qweight[n * words_per_row + j * 16 + (lane >> 1)] = part;
    } else {
      uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int o = 4 * (lane & 7) + i;                // offset inside the 32-k block
        const uint32_t q = static_cast<uint32_t>(g.q[i]);
        const int oo = o & 15;
        const uint32_t lo = (q & 3u) << (2 * ((oo >> 1) + 8 * (oo & 1)));
        if (o < 16) p0 |= lo; else p1 |= lo;
        p2 |= ((q >> 2) & 1u) << ((o >> 1) + 16 * (o & 1));
      }
#pragma unroll
      for (int m = 1; m < 8; m <<= 1) {
        p0 |= __shfl_xor_sync(0xffffffffu, p0, m);
        p1 |= __shfl_xor_sync(0xffffffffu, p1, m);
        p2 |= __shfl_xor_sync(0xffffffffu, p2, m);
      }
      if ((lane & 7) == 0) {
        uint32_t* dst = qweight + n * words_per_row + (j * 4 + (lane >> 3)) * 3;
        dst[0] = p0; dst[1] = p1; dst[2] = p2;
      }
    }
    if (lane == 0) {
      sh_scale[lr] = g.sc_h;
      sh_zero[lr] = static_cast<uint8_t>(g.z);
    }
  }
  __syncthreads();
  const int t = threadIdx.x;
  const int64_t nb = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta;
  if (t < kQuantRowsPerCta && nb + t < N) scales[j * N + nb + t] = sh_scale[t];
  if (t >= 32 && t < 32 + kQuantRowsPerCta && nb + t - 32 < N)
    zeros[j * N + nb + t - 32] = sh_zero[t - 32];
}

// Search operand: for grid point a, E[a][n][k] = fp16(deq[n,k] * (1 / s_a[k]) - w[n,k]) with
// deq = (q - z) * sc from the quantizer above; rows N..N_pad-1 are written as zeros so that
// 128-row tiles never straddle two grid points.
template <int kBits>
__global__ void __launch_bounds__(256) search_build_error_kernel(
    const __half* __restrict__ W, int64_t N, int64_t K, int64_t N_pad,
    const float* __restrict__ s_table, __half* __restrict__ E) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t j = blockIdx.y;
  const int64_t a = blockIdx.z;
  const int64_t k0 = j * kGroup + 4 * lane;
  const float* s = s_table + a * K;
  __half* Ea = E + a * N_pad * K;
#pragma unroll 1
  for (int rr = 0; rr < kQuantRowsPerCta / 8; ++rr) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta +
                      warp * (kQuantRowsPerCta / 8) + rr;
    if (n >= N_pad) break;
    uint2 out = make_uint2(0u, 0u);
    if (n < N) {
      float w[4], w_raw[4];
      load_scaled(W, K, n, k0, s, w, w_raw);
      const GroupQuant g = quantize_lane<kBits>(w);
      const float4 sv = *reinterpret_cast<const float4*>(s + k0);
      const float sa[4] = {sv.x, sv.y, sv.z, sv.w};
      __half e[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float deq = __fmul_rn(__fsub_rn(g.q[i], g.z), g.sc);
        const float inv = __fdiv_rn(1.0f, sa[i]);
        e[i] = __float2half_rn(__fsub_rn(__fmul_rn(deq, inv), w_raw[i]));
      }
      out.x = h2_as_u32(__halves2half2(e[0], e[1]));
      out.y = h2_as_u32(__halves2half2(e[2], e[3]));
    }
    *reinterpret_cast<uint2*>(Ea + n * K + k0) = out;
  }
}

// s_table[a][k] = (float) pow((double) max(s_x[k], 1e-4f), (double) alphas[a]).
__global__ void scale_candidates_kernel(const float* __restrict__ s_x,
                                        const float* __restrict__ alphas, int n_alpha, int64_t K,
                                        float* __restrict__ s_table) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int a = blockIdx.y;
  if (k >= K || a >= n_alpha) return;
  const double base = static_cast<double>(fmaxf(s_x[k], 1e-4f));
  s_table[static_cast<int64_t>(a) * K + k] =
      __double2float_rn(pow(base, static_cast<double>(alphas[a])));
}

}  // namespace awq
