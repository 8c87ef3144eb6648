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
// Eight lanes own one (row, group): lane l holds 16 consecutive k, the group's min and max
// come from three xor-shuffles each, and each lane assembles its own packed words (4-bit:
// two whole words; 3-bit: one low-bit word, and the bit-2 word with one shuffle). A CTA of
// 8 warps covers 32 rows of one group so the [G, N] scales and zeros leave as contiguous runs.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kQuantRowsPerCta = 32;

// One (row, group) per 8 lanes: lane sub = lane % 8 holds k = 128 j + 16 sub .. + 15.
struct QuantGroup {
  float sc;       // fp16-rounded scale, widened
  float z;        // zero point
  float rcp;      // correctly rounded 1 / sc
  __half sc_h;
};

__device__ __forceinline__ void load16(const __half* __restrict__ W, int64_t K, int64_t n,
                                       int64_t k0, bool valid, const float* __restrict__ s,
                                       float (&w)[16], float (&w_raw)[16]) {
  uint4 u[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  if (valid) {
    const uint4* p = reinterpret_cast<const uint4*>(W + n * K + k0);
    u[0] = p[0];
    u[1] = p[1];
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t v[4] = {u[h].x, u[h].y, u[h].z, u[h].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(u32_as_h2(v[i]));
      w_raw[8 * h + 2 * i] = f.x;
      w_raw[8 * h + 2 * i + 1] = f.y;
    }
  }
  if (s != nullptr) {
    const float4* sp = reinterpret_cast<const float4*>(s + k0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 sv = sp[q];
      w[4 * q + 0] = __fmul_rn(w_raw[4 * q + 0], sv.x);
      w[4 * q + 1] = __fmul_rn(w_raw[4 * q + 1], sv.y);
      w[4 * q + 2] = __fmul_rn(w_raw[4 * q + 2], sv.z);
      w[4 * q + 3] = __fmul_rn(w_raw[4 * q + 3], sv.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = w_raw[i];
  }
}

// Group min/max over the 8 lanes of a (row, group) and the group's scale and zero point.
template <int kBits>
__device__ __forceinline__ QuantGroup group_params(const float (&w)[16]) {
  constexpr float qmax = static_cast<float>((1 << kBits) - 1);
  float mx = w[0], mn = w[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    mx = fmaxf(mx, w[i]);
    mn = fminf(mn, w[i]);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  QuantGroup g;
  float scale = __fdiv_rn(__fsub_rn(mx, mn), qmax);
  scale = fmaxf(scale, 1e-5f);
  g.sc_h = __float2half_rn(scale);
  g.sc = __half2float(g.sc_h);
  g.z = fminf(fmaxf(rintf(__fdiv_rn(-mn, g.sc)), 0.0f), qmax);
  g.rcp = __frcp_rn(g.sc);
  return g;
}

// q = clamp(rint(w' / sc) + z, 0, qmax) with the IEEE quotient. The product t = w' * rcp,
// rcp = 1/sc correctly rounded, is within 2^-23 |w'/sc| (two roundings) of the exact
// quotient, and rint of the correctly rounded quotient can only differ from rint(t) where
// the two straddle a half-integer. So for |t| <= 32 (absolute error <= 2^-18) rint(t) is the
// code unless t lies within 2^-17 of a half-integer; only then is the quotient formed with
// an IEEE division. For |t| > 32 the code clamps to 0 or qmax whatever the rounding, since
// 0 <= z <= 15.
template <int kBits>
__device__ __forceinline__ float code_of(float wp, const QuantGroup& g) {
  constexpr float qmax = static_cast<float>((1 << kBits) - 1);
  const float t = __fmul_rn(wp, g.rcp);
  float r = rintf(t);
  if (fabsf(__fsub_rn(t, r)) >= 0.5f - 0x1p-17f) r = rintf(__fdiv_rn(wp, g.sc));
  return fminf(fmaxf(__fadd_rn(r, g.z), 0.0f), qmax);
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
  const int sub = lane & 7;
  const int lr = 4 * warp + (lane >> 3);                 // local row 0..31
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta + lr;
  const bool valid = n < N;
  const int64_t j = blockIdx.y;                          // group index
  const int64_t k0 = j * kGroup + 16 * sub;
  float w[16], w_raw[16];
  load16(W, K, n, k0, valid, s, w, w_raw);
  const QuantGroup g = group_params<kBits>(w);
  uint32_t q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = static_cast<uint32_t>(code_of<kBits>(w[i], g));
  if (kBits == 4) {
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int o = 0; o < 8; ++o) {
      w0 |= q[o] << (4 * nibble_pos(o));
      w1 |= q[8 + o] << (4 * nibble_pos(o));
    }
    if (valid && AWQ_IN_BOUNDS(j * 16 + 2 * sub + 2 <= K / 8))
      *reinterpret_cast<uint2*>(qweight + n * (K / 8) + j * 16 + 2 * sub) = make_uint2(w0, w1);
  } else {
    // lanes sub = 2b + h hold offsets 16h..16h+15 of the group's 32-k block b
    const int h = sub & 1;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int o = 16 * h + e;                          // offset inside the 32-k block
      lo |= (q[e] & 3u) << (2 * ((e >> 1) + 8 * (e & 1)));
      hi |= ((q[e] >> 2) & 1u) << ((o >> 1) + 16 * (o & 1));
    }
    hi |= __shfl_xor_sync(0xffffffffu, hi, 1);
    if (valid && AWQ_IN_BOUNDS((j * 4 + (sub >> 1)) * 3 + 3 <= 3 * K / 32)) {
      uint32_t* dst = qweight + n * (3 * K / 32) + (j * 4 + (sub >> 1)) * 3;
      dst[h] = lo;
      if (h == 0) dst[2] = hi;
    }
  }
  if (sub == 0) {
    sh_scale[lr] = g.sc_h;
    sh_zero[lr] = static_cast<uint8_t>(g.z);
  }
  __syncthreads();
  const int t = threadIdx.x;
  const int64_t nb = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta;
  const bool in_g = AWQ_IN_BOUNDS(j < K / kGroup);
  if (t < kQuantRowsPerCta && nb + t < N && in_g) scales[j * N + nb + t] = sh_scale[t];
  if (t >= 32 && t < 32 + kQuantRowsPerCta && nb + t - 32 < N && in_g)
    zeros[j * N + nb + t - 32] = sh_zero[t - 32];
}

// Search operand: for grid point a, e = deq[n,k] * inv_a[k] - w[n,k] in fp32, with
// deq = (q - z) * sc from the quantizer above and inv_a = 1 / s_a (correctly rounded, from
// a table), stored in two fp16 parts, hi = fp16(e) and lo = fp16((e - hi) * 2^12) (e - hi
// is exact in fp32, the scaling by a power of 2 too): hi + 2^-12 lo represents e to about 22
// significant bits instead of fp16's 11. Row n of grid point a is row a * N_pad + n of a
// [rows, 2K] matrix holding hi in columns 0..K-1 and lo in K..2K-1; rows N..N_pad-1 are
// written as zeros so that 128-row tiles never straddle two grid points. With `rms` (the
// Gram form of the loss) e is first multiplied by the channel's root mean square rms[k].
template <int kBits>
__global__ void __launch_bounds__(256) search_build_error_kernel(
    const __half* __restrict__ W, int64_t N, int64_t K, int64_t N_pad,
    const float* __restrict__ s_table, const float* __restrict__ inv_table,
    const float* __restrict__ rms, __half* __restrict__ E) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int sub = lane & 7;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta + 4 * warp + (lane >> 3);
  const int64_t j = blockIdx.y;
  const int64_t a = blockIdx.z;
  const int64_t k0 = j * kGroup + 16 * sub;
  const float* s = s_table + a * K;
  const bool valid = n < N;
  float w[16], w_raw[16];
  load16(W, K, n, k0, valid, s, w, w_raw);
  const QuantGroup g = group_params<kBits>(w);
  if (n >= N_pad) return;
  uint4 out[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  uint4 out_lo[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  if (valid) {
    const float4* ip = reinterpret_cast<const float4*>(inv_table + a * K + k0);
    float inv[16];
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const float4 v = ip[qd];
      inv[4 * qd] = v.x; inv[4 * qd + 1] = v.y; inv[4 * qd + 2] = v.z; inv[4 * qd + 3] = v.w;
    }
    uint32_t e2[8], l2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float e[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int idx = 2 * i + u;
        const float q = code_of<kBits>(w[idx], g);
        const float deq = __fmul_rn(__fsub_rn(q, g.z), g.sc);
        e[u] = __fsub_rn(__fmul_rn(deq, inv[idx]), w_raw[idx]);
        if (rms != nullptr) e[u] = __fmul_rn(e[u], rms[k0 + idx]);
      }
      const __half2 hi = __floats2half2_rn(e[0], e[1]);
      const float2 hf = __half22float2(hi);
      e2[i] = h2_as_u32(hi);
      l2[i] = h2_as_u32(__floats2half2_rn(__fmul_rn(__fsub_rn(e[0], hf.x), 4096.0f),
                                          __fmul_rn(__fsub_rn(e[1], hf.y), 4096.0f)));
    }
    out[0] = make_uint4(e2[0], e2[1], e2[2], e2[3]);
    out[1] = make_uint4(e2[4], e2[5], e2[6], e2[7]);
    out_lo[0] = make_uint4(l2[0], l2[1], l2[2], l2[3]);
    out_lo[1] = make_uint4(l2[4], l2[5], l2[6], l2[7]);
  }
  if (!AWQ_IN_BOUNDS(a < gridDim.z && k0 + 16 <= K)) return;
  __half* row = E + (a * N_pad + n) * (2 * K);
  uint4* dst = reinterpret_cast<uint4*>(row + k0);
  dst[0] = out[0];
  dst[1] = out[1];
  uint4* dst_lo = reinterpret_cast<uint4*>(row + K + k0);
  dst_lo[0] = out_lo[0];
  dst_lo[1] = out_lo[1];
}

// inv_table[a][k] = 1 / s_table[a][k], correctly rounded.
__global__ void inv_table_kernel(const float* __restrict__ s_table, int64_t total,
                                 float* __restrict__ inv_table) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < total) inv_table[i] = __frcp_rn(s_table[i]);
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
