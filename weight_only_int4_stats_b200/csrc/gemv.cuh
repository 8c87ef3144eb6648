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

namespace awq {

// ---------------------------------------------------------------------------------------
// Streaming decode GEMM (the default decode path).
//
// Each CTA owns a contiguous range of whole 16-row tiles, so no output is split across CTAs
// and the result does not depend on the grid. One producer thread walks the CTA's
// (tile, 1024-k chunk) units and streams each unit's packed weights ([16 rows, 128 words]),
// fp16 scales and uint8 zeros ([8 groups, 16 rows] each) with TMA into an 8-slot shared
// memory ring. Under programmatic dependent launch the kernel starts while the previous
// kernel on the stream is still finishing: before griddepcontrol.wait it only issues L2
// prefetches of its weights, scales and zeros (coherent with any write of that kernel, so
// even a quantize-and-pack directly before it is safe), and every shared-memory load comes
// after the wait and hits L2. X ([M, K], small at decode) is bulk-copied into shared memory
// once, after the wait. Eight consumer warps
// each take one 128-wide group of every unit (the register-only dequant + mma.sync of the
// kernel above, fed from shared memory) and keep per-tile fp32 sums; at the end of a tile
// the eight warps' sums are added in a fixed order and written as fp16.
// ---------------------------------------------------------------------------------------
constexpr int kG2Warps = 8;                       // consumer warps = groups per unit
constexpr int kG2Threads = (kG2Warps + 1) * 32;   // + one producer warp
constexpr int kG2KC = kG2Warps * kGroup;          // k per unit (1024)
constexpr int kG2WBytes = kGemvRows * (kG2KC / 2);          // 8192: packed weights
constexpr int kG2SBytes = kG2Warps * kGemvRows * 2;         // 256: fp16 scales
constexpr int kG2ZBytes = kG2Warps * kGemvRows;             // 128: uint8 zeros
constexpr int kG2SlotBytes = kG2WBytes + kG2SBytes + kG2ZBytes;   // 8576 (multiple of 128)

struct G2Smem {
  int x_bytes;      // M * K * 2 rounded up to 128
  int slots;
  __host__ __device__ int slot_off() const { return x_bytes; }
  __host__ __device__ int bar_off() const { return x_bytes + slots * kG2SlotBytes; }
  template <int kNTiles>
  __host__ __device__ int red_off() const { return bar_off() + (2 * slots + 1) * 8 + 8; }
  template <int kNTiles>
  __host__ __device__ int total() const {
    return red_off<kNTiles>() + kG2Warps * kNTiles * 4 * 32 * 4;
  }
};

template <int kNTiles>
__global__ void __launch_bounds__(kG2Threads) gemv_stream_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
    const __grid_constant__ CUtensorMap tmap_z, const uint32_t* __restrict__ qweight,
    const __half* __restrict__ X, int M, int64_t N, int64_t K, const float* __restrict__ inv_s,
    __half* __restrict__ Y, G2Smem lay) {
  extern __shared__ __align__(128) uint8_t smem[];
  __half* xs = reinterpret_cast<__half*>(smem);
  uint8_t* slots = smem + lay.slot_off();
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar_off());
  uint64_t* empty = full + lay.slots;
  uint64_t* xfull = empty + lay.slots;
  float* red = reinterpret_cast<float*>(smem + lay.template red_off<kNTiles>());

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t T = (N + kGemvRows - 1) / kGemvRows;
  const int64_t P = gridDim.x;
  const int64_t t0 = blockIdx.x * T / P, t1 = (blockIdx.x + 1) * T / P;
  const int64_t C = (K + kG2KC - 1) / kG2KC;
  const int64_t units = (t1 - t0) * C;
  const int64_t G = K / kGroup;
  const int S = lay.slots;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kG2Warps);
    }
    mbar_init(xfull, 1);
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kG2Warps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      pdl_launch_dependents();
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_s);
      tma_prefetch_desc(&tmap_z);
      // HBM -> L2 for everything this CTA will read: its rows of packed weights are one
      // contiguous range; scales and zeros are fetched per unit through their tensor maps.
      {
        const int64_t row_bytes = K / 2;
        const int64_t r0 = t0 * kGemvRows, r1 = t1 * kGemvRows < N ? t1 * kGemvRows : N;
        const uint8_t* wrow = reinterpret_cast<const uint8_t*>(qweight) + r0 * row_bytes;
        const int64_t bytes = (r1 - r0) * row_bytes;
        for (int64_t off = 0; off < bytes; off += 65536)
          prefetch_l2_bulk(wrow + off, static_cast<uint32_t>(bytes - off < 65536 ? bytes - off : 65536));
      }
      for (int64_t u = 0; u < units; ++u) {
        const int64_t tile = t0 + u / C, chunk = u % C;
        prefetch_l2_tile_2d(&tmap_s, static_cast<int32_t>(tile * kGemvRows),
                            static_cast<int32_t>(chunk * kG2Warps));
        prefetch_l2_tile_2d(&tmap_z, static_cast<int32_t>(tile * kGemvRows),
                            static_cast<int32_t>(chunk * kG2Warps));
      }
      pdl_wait();
      mbar_arrive_expect_tx(xfull, static_cast<uint32_t>(M * K * 2));
      bulk_load_1d(xs, X, static_cast<uint32_t>(M * K * 2), xfull);
      for (int64_t u = 0; u < units; ++u) {
        const int slot = static_cast<int>(u % S);
        const uint32_t ph = static_cast<uint32_t>((u / S) & 1);
        if (!mbar_wait(&empty[slot], ph ^ 1)) break;
        const int64_t tile = t0 + u / C, chunk = u % C;
        uint8_t* sb = slots + slot * kG2SlotBytes;
        mbar_arrive_expect_tx(&full[slot], kG2SlotBytes);
        tma_load_2d(sb, &tmap_w, &full[slot], static_cast<int32_t>(chunk * (kG2KC / 8)),
                    static_cast<int32_t>(tile * kGemvRows));
        tma_load_2d(sb + kG2WBytes, &tmap_s, &full[slot], static_cast<int32_t>(tile * kGemvRows),
                    static_cast<int32_t>(chunk * kG2Warps));
        tma_load_2d(sb + kG2WBytes + kG2SBytes, &tmap_z, &full[slot],
                    static_cast<int32_t>(tile * kGemvRows), static_cast<int32_t>(chunk * kG2Warps));
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int r = lane >> 2, c = lane & 3;
  // A timed-out wait clears `ok`; the warp then skips all further waits and arithmetic but
  // still runs every named barrier, so the consumer warps can never deadlock each other.
  bool ok = __all_sync(0xffffffffu, mbar_wait(xfull, 0));
  if (inv_s != nullptr) {
    // x <- fp16(x * inv_s), in place, by the 256 consumer threads
    const int64_t n8 = static_cast<int64_t>(M) * K / 8;
    for (int64_t i = threadIdx.x; ok && i < n8; i += kG2Warps * 32) {
      const int64_t k = (i * 8) % K;
      uint4 v = reinterpret_cast<uint4*>(xs)[i];
      const float4 s0 = *reinterpret_cast<const float4*>(inv_s + k);
      const float4 s1 = *reinterpret_cast<const float4*>(inv_s + k + 4);
      float2 f;
      f = __half22float2(u32_as_h2(v.x)); v.x = h2_as_u32(__floats2half2_rn(f.x * s0.x, f.y * s0.y));
      f = __half22float2(u32_as_h2(v.y)); v.y = h2_as_u32(__floats2half2_rn(f.x * s0.z, f.y * s0.w));
      f = __half22float2(u32_as_h2(v.z)); v.z = h2_as_u32(__floats2half2_rn(f.x * s1.x, f.y * s1.y));
      f = __half22float2(u32_as_h2(v.w)); v.w = h2_as_u32(__floats2half2_rn(f.x * s1.z, f.y * s1.w));
      reinterpret_cast<uint4*>(xs)[i] = v;
    }
    named_bar_sync(1, kG2Warps * 32);
  }

  float total[kNTiles][4];
#pragma unroll
  for (int t = 0; t < kNTiles; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) total[t][i] = 0.0f;

  for (int64_t u = 0; u < units; ++u) {
    const int slot = static_cast<int>(u % S);
    const uint32_t ph = static_cast<uint32_t>((u / S) & 1);
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&full[slot], ph));
    const int64_t tile = t0 + u / C, chunk = u % C;
    const int64_t g = chunk * kG2Warps + warp;
    const uint8_t* sb = slots + slot * kG2SlotBytes;
    if (ok && g < G) {
      const uint4 wA = *reinterpret_cast<const uint4*>(sb + r * (kG2KC / 2) + (warp * 16 + 4 * c) * 4);
      const uint4 wB =
          *reinterpret_cast<const uint4*>(sb + (r + 8) * (kG2KC / 2) + (warp * 16 + 4 * c) * 4);
      const __half* ss = reinterpret_cast<const __half*>(sb + kG2WBytes) + warp * kGemvRows;
      const uint8_t* zz = sb + kG2WBytes + kG2SBytes + warp * kGemvRows;
      const uint32_t zA = zz[r], zB = zz[r + 8];
      const float scA = __half2float(ss[r]), scB = __half2float(ss[r + 8]);
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
      const int64_t kx = g * kGroup + 32 * c;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t qa[4], qb[4];
        dequant_word_qz(wordsA[j], loA, hiA, qa);
        dequant_word_qz(wordsB[j], loB, hiB, qb);
#pragma unroll
        for (int t = 0; t < kNTiles; ++t) {
          const int m = r + 8 * t;
          uint4 xv = make_uint4(0u, 0u, 0u, 0u);
          if (m < M) xv = *reinterpret_cast<const uint4*>(xs + m * K + kx + 8 * j);
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
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&empty[slot]);

    if (chunk == C - 1) {
      // tile complete: fixed-order sum over the eight consumer warps, fp16 store
#pragma unroll
      for (int t = 0; t < kNTiles; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          red[((warp * kNTiles + t) * 4 + i) * 32 + lane] = total[t][i];
          total[t][i] = 0.0f;
        }
      named_bar_sync(1, kG2Warps * 32);
      if (ok && warp < kNTiles) {
        const int t = warp;
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float s = 0.0f;
#pragma unroll
          for (int w = 0; w < kG2Warps; ++w) s += red[((w * kNTiles + t) * 4 + i) * 32 + lane];
          v[i] = s;
        }
        const int64_t nA = tile * kGemvRows + r, nB = nA + 8;
        const int m0 = 8 * t + 2 * c, m1 = m0 + 1;
        if (nA < N) {
          if (m0 < M) Y[static_cast<int64_t>(m0) * N + nA] = __float2half_rn(v[0]);
          if (m1 < M) Y[static_cast<int64_t>(m1) * N + nA] = __float2half_rn(v[1]);
        }
        if (nB < N) {
          if (m0 < M) Y[static_cast<int64_t>(m0) * N + nB] = __float2half_rn(v[2]);
          if (m1 < M) Y[static_cast<int64_t>(m1) * N + nB] = __float2half_rn(v[3]);
        }
      }
      named_bar_sync(1, kG2Warps * 32);
    }
  }
}

}  // namespace awq
