// K3: W4A16 decode GEMM for M <= 16 tokens, Y[m, n] = sum_k x[m, k] * deq[n, k].
// Two kernels: the register-streaming kernel below, which takes M <= 8 calls that the
// streaming kernel further down cannot (N % 16 != 0, or X larger than its shared memory),
// and the TMA-fed streaming kernel, the default.
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

template <bool kBf16 = false>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if constexpr (kBf16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
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
    if (g < G && AWQ_IN_BOUNDS(g * 16 + c * 4 + 4 <= wpr)) {
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
// Streaming decode GEMM (the decode path for M <= 16; N in whole 16-row tiles and X within
// one CTA's shared memory).
//
// Persistent: the grid is one or two CTAs per SM (as many as there are 16-row tiles, at
// most). Each CTA owns a contiguous range of whole 16-row tiles, floor(T/P) of them plus one
// for the first T mod P CTAs, so no output is split across CTAs and the result does not
// depend on the grid. (With boundaries at b*T/P instead, CTAs b and b + P/2, which a grid of
// two per SM usually places on one SM, got equal counts: at 688 tiles over 296 CTAs, 48 SMs
// ran six tiles while the rest ran four.) One producer thread walks
// the CTA's (tile, 2048-k chunk) units and streams each unit's packed weights (16 rows x
// 1 KB at 4 bits, 768 B at 3 bits), fp16 scales and uint8 zeros ([16 groups, 16 rows]) with
// TMA into a shared-memory ring. The packed weights arrive as 128-byte-wide boxes with the
// 128-byte swizzle (16-byte chunk c of row r of a box at chunk c ^ (r % 8)), so the consumers'
// 16-byte reads of eight rows at once hit eight different bank groups: without it the rows,
// 1 KB apart, all map to the same banks. A quarter-warp's eight 16-byte reads come from two
// rows and four chunks; lane row r reads weight row rho(r) = r/2 + 4(r%2) of the box (and
// rho(r) + 8), so the two rows of a quarter-warp differ in the swizzle's bit 2 and their
// chunks land in opposite halves of the 128-byte line: eight reads, eight bank groups, one
// wavefront. The MMA's row r is then weight row rho(r) of the tile.
//
// Back-to-back launches overlap (programmatic dependent launch). A CTA needs at most half of
// an SM's shared memory, so the next GEMM's CTAs become resident beside this one's as soon as
// every CTA of this grid has passed griddepcontrol.wait (where the next launch is allowed).
// Before the wait a CTA touches no output and no activation: it issues L2 prefetches of X
// and of inv_s (coherent with writes of the preceding kernel, so always safe) and, when the
// caller states that the weights are not written by the kernel launched just before
// (kGemvWeightsReady), TMA-loads the first ring slots. An L2 prefetch of the CTA's weight
// rows as well measured slower, with or without the early ring loads: it competes with them
// and with the preceding kernel's stream.
//
// After the wait the consumer warps stage X ([M, K], small at decode; each thread issues all
// its loads of a round at once) from global memory into shared memory in the order the MMA's
// B fragments read it -- [group][8-k chunk j][token][32-k
// quarter c] of 16 bytes -- so one fragment read is 64 contiguous bytes at M = 1. Eight
// consumer warps each take two of a unit's sixteen 128-wide groups, with register-only
// dequantization feeding mma.sync m16n8k16 (weights as the 16-row A operand, activations as
// the 8-column B operand). A warp copies its packed words, scales and zero points of the unit
// to registers and releases the ring slot before the arithmetic. Two dequantization forms:
//  * M = 1 (kOffset): a mask-and-or with 0x6400 turns the nibble pair (k0, k1) of a word
//    into the exact fp16 values (1024 + q0, 1024 + q1) and the pair (k2, k3), stored 4 bits
//    higher, into (1024 + 16 q2, 1024 + 16 q3) (the same after a shift by 8 for k4..k7);
//    these go to the MMA unchanged against X staged with columns k%8 in {2,3,6,7} divided by
//    16 (exact in fp16), so per group the MMA returns sum_k x_k q_k + C1 with
//    C1 = 1024 * sum_k xs_k; with C2 = sum_k x_k the group adds s * (mma - C1 - z C2).
//    Five integer operations per packed word; the fp32 cancellation of the 1024 offset keeps
//    about 13 significant bits of each group sum. (3-bit codes and bf16 have one raw pair
//    form, base 1024 or 128, so X is staged undivided and C1 = base * C2.)
//  * M > 1: one fp16 subtract (or multiply-add) per pair leaves the exact q - z first.
// Each group's eight MMAs run as four independent accumulator chains. At the end of a tile
// the consumer warps' partial sums are added in a fixed warp order and stored.
// ---------------------------------------------------------------------------------------
constexpr int kG4Groups = 16;                      // groups per unit
constexpr int kG4KC = kG4Groups * kGroup;          // k per unit (2048)
constexpr int kG4Warps = 8;                        // consumer warps (two groups each per unit)
constexpr int kG4Threads = (kG4Warps + 1) * 32;    // + one producer warp
constexpr int kG4WSlot = kGemvRows * kG4KC / 2;    // ring slot stride of the packed codes (16 KB)
constexpr int kG4SBytes = kG4Groups * kGemvRows * 2;           // 512
constexpr int kG4ZBytes = kG4Groups * kGemvRows;               // 256
constexpr int kG4Box = kGemvRows * 128;                        // one swizzled box: 16 rows x 128 B
constexpr int kGSMaxSlots = 6;
constexpr int kG4XRound = 4;                       // X chunks per thread per staging round

// Flag bits of the decode launch (awq_gemm_w4a16's flags).
constexpr unsigned kGemvWeightsReady = 1u;

// Shared memory, from a 1024-byte aligned base (the swizzle's period): the packed-code slots,
// then per slot its scales and zero points, the staged X, the per-(group, token) sums, the
// barriers and the tile-end reduction buffer.
struct G4Smem {
  int slots;     // ring depth
  int x_bytes;   // M * K * 2, rounded up to 128
  int c_bytes;   // C1/C2 per (group, token)
  __host__ __device__ int sz_off() const { return slots * kG4WSlot; }
  __host__ __device__ int x_off() const { return sz_off() + slots * (kG4SBytes + kG4ZBytes); }
  __host__ __device__ int c_off() const { return x_off() + x_bytes; }
  __host__ __device__ int bar_off() const { return c_off() + c_bytes; }
  __host__ __device__ int red_off() const { return bar_off() + (2 * kGSMaxSlots + 2) * 8; }
  // + 1024 bytes of slack for aligning the base
  __host__ __device__ int total(int n_tiles) const {
    return red_off() + kG4Warps * n_tiles * 4 * 32 * 4 + 1024;
  }
  __host__ __device__ static G4Smem make(int M, int64_t K, int n_tiles, int slots) {
    G4Smem l;
    l.slots = slots;
    l.x_bytes = static_cast<int>((static_cast<int64_t>(M) * K * 2 + 127) / 128 * 128);
    l.c_bytes = static_cast<int>(((K / kGroup) * 8 * n_tiles * 2 * 4 + 127) / 128 * 128);
    return l;
  }
};

// Byte offset of packed word w (0..kG4KC*bits/32 - 1 of a unit's row) of row r in a slot of
// swizzled 128-byte boxes.
__device__ __forceinline__ uint32_t g4_word_offset(int r, int w) {
  return static_cast<uint32_t>((w >> 5) * kG4Box + r * 128 + ((((w >> 2) & 7) ^ (r & 7)) << 4) +
                               (w & 3) * 4);
}

// One packed word -> the raw fp16 pairs (1024+q0,1024+q1), (1024+16q2,1024+16q3),
// (1024+q4,1024+q5), (1024+16q6,1024+16q7); with bf16 activations the raw bf16 pairs
// (128+q0,128+q1), (128+q2,128+q3), ... (bf16 keeps only 7 mantissa bits, so each nibble
// pair is shifted down first: 0x4300 is 128.0 and the low 4 mantissa bits hold q exactly).
template <bool kBf16 = false>
__device__ __forceinline__ void raw_word(uint32_t w, uint32_t (&v)[4]) {
  if constexpr (kBf16) {
    v[0] = lop3_and_or(w, 0x000F000Fu, 0x43004300u);
    v[1] = lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u);
    v[2] = lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u);
    v[3] = lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u);
  } else {
    const uint32_t w8 = w >> 8;
    v[0] = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
    v[1] = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
    v[2] = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
    v[3] = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
  }
}

// 3-bit: the raw pairs (base + q) of chunk i (k = 8i..8i+7) of a 32-k block whose low-bit words
// are w0 (offsets 0..15) / w1 (16..31) and whose bit-2 word is w2 (layout of the 3-bit packing:
// the pair's two crumbs at 2-bit field 4(i%2) + e of its low word, its two high bits at bits
// 4i + e and 4i + e + 16 of w2); base 1024 (fp16, 0x6400) or 128 (bf16, 0x4300).
template <bool kBf16>
__device__ __forceinline__ void raw3_chunk(uint32_t w0, uint32_t w1, uint32_t w2, int i,
                                           uint32_t (&v)[4]) {
  const uint32_t wlo = i < 2 ? w0 : w1;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int pp = 4 * (i & 1) + e, hb = 4 * i + e;
    const uint32_t lo = lop3_and_or(wlo >> (2 * pp), 0x00030003u, kBf16 ? 0x43004300u : 0x64006400u);
    const uint32_t hs = hb >= 2 ? (w2 >> (hb - 2)) : (w2 << (2 - hb));
    v[e] = lop3_and_or(hs, 0x00040004u, lo);
  }
}

// The exact pairs (q - z) in bf16: the raw pairs minus (128 + z).
__device__ __forceinline__ void dequant_word_qz_bf16(uint32_t w, uint32_t bias, uint32_t (&out)[4]) {
  raw_word<true>(w, out);
#pragma unroll
  for (int i = 0; i < 4; ++i) out[i] = b2_as_u32(__hsub2(u32_as_b2(out[i]), u32_as_b2(bias)));
}

template <int kNTiles, bool kOffset, bool kBf16 = false, int kBits = 4>
__global__ void __launch_bounds__(kG4Threads, 2) gemv_stream_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
    const __grid_constant__ CUtensorMap tmap_z,
    const act_t<kBf16>* __restrict__ X, int M, int64_t N, int64_t K,
    const float* __restrict__ inv_s, act_t<kBf16>* __restrict__ Y, G4Smem lay, unsigned flags) {
  static_assert(kBits == 4 || kBits == 3, "4- or 3-bit codes");
  constexpr int kTok = 8 * kNTiles;
  constexpr int kRowW = kG4KC * kBits / 32;            // packed words of one row in a unit
  constexpr int kBoxes = kRowW / 32;                   // 128-byte boxes per unit (8 or 6)
  constexpr uint32_t kTx = kGemvRows * kRowW * 4 + kG4SBytes + kG4ZBytes;
  // M = 1 with fp16 and 4 bits stages columns k%8 in {2,3,6,7} divided by 16 (the nibbles
  // stored 4 bits higher come out as 1024 + 16q); every other form has one raw pair form
  constexpr bool kDiv16 = !kBf16 && kBits == 4;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* wslots = smem;
  uint8_t* szslots = smem + lay.sz_off();
  act_t<kBf16>* xs = reinterpret_cast<act_t<kBf16>*>(smem + lay.x_off());   // [G][4][M][4] x 8
  float* cc = reinterpret_cast<float*>(smem + lay.c_off());
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar_off());
  uint64_t* empty = full + kGSMaxSlots;
  float* red = reinterpret_cast<float*>(smem + lay.red_off());
  const int S = lay.slots;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t T = (N + kGemvRows - 1) / kGemvRows;
  const int64_t P = gridDim.x;
  const int64_t bx = blockIdx.x, tq = T / P, tr = T % P;
  const int64_t t0 = bx * tq + (bx < tr ? bx : tr), t1 = t0 + tq + (bx < tr ? 1 : 0);
  const int Ki = static_cast<int>(K);
  const int G = Ki / kGroup;
  const int C = (Ki + kG4KC - 1) / kG4KC;
  const int64_t units = (t1 - t0) * C;

  // the trace build's record index of this CTA lives in the barrier area's spare word
  unsigned* trace_rec = reinterpret_cast<unsigned*>(empty + kGSMaxSlots);
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kG4Warps * 32);
    }
    fence_barrier_init();
#ifdef AWQ_TRACE
    *trace_rec = atomicAdd(&g_trace_ctas, 1u);
    AWQ_TRACE_AT(*trace_rec, kTrStart, globaltimer_ns());
    AWQ_TRACE_AT(*trace_rec, kTrN, N);
    AWQ_TRACE_AT(*trace_rec, kTrUnits, units);
    AWQ_TRACE_AT(*trace_rec, kTrBlock, blockIdx.x);
#endif
  }
  __syncthreads();
#ifdef AWQ_TRACE
  const unsigned rec = *trace_rec;
#else
  const unsigned rec = 0u;
  (void)trace_rec;
#endif
  (void)rec;

  if (warp == kG4Warps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_s);
      tma_prefetch_desc(&tmap_z);
      {   // X and inv_s first (the consumers stage X as soon as the dependency wait returns):
          // an L2 prefetch is coherent with the preceding kernel's writes (L2 is where they
          // land), so the staging loads after the wait hit L2
        const int64_t xb = static_cast<int64_t>(M) * K * 2;
        for (int64_t off = 0; off < xb; off += 65536)
          prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(X) + off,
                           static_cast<uint32_t>(xb - off < 65536 ? xb - off : 65536));
        if (inv_s != nullptr)
          for (int64_t off = 0; off < K * 4; off += 65536)
            prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(inv_s) + off,
                             static_cast<uint32_t>(K * 4 - off < 65536 ? K * 4 - off : 65536));
      }
      int slot = 0, chunk = 0;
      uint32_t ph = 0;
      int64_t tile = t0;
      auto issue = [&]() {
        if (!AWQ_IN_BOUNDS(slot < S && tile < t1 && chunk < C)) return;
        uint8_t* wb = wslots + slot * kG4WSlot;
        uint8_t* sz = szslots + slot * (kG4SBytes + kG4ZBytes);
        mbar_arrive_expect_tx(&full[slot], kTx);
        const int32_t row = static_cast<int32_t>(tile * kGemvRows);
#pragma unroll
        for (int b = 0; b < kBoxes; ++b)
          tma_load_2d(wb + b * kG4Box, &tmap_w, &full[slot], chunk * kRowW + b * 32, row);
        tma_load_2d(sz, &tmap_s, &full[slot], row, chunk * kG4Groups);
        tma_load_2d(sz + kG4SBytes, &tmap_z, &full[slot], row, chunk * kG4Groups);
        if (++slot == S) { slot = 0; ph ^= 1; }
        if (++chunk == C) { chunk = 0; ++tile; }
      };
      int64_t u = 0;
      if (flags & kGemvWeightsReady) {
        // the weights do not depend on the preceding kernel: fill the (empty) ring now
        const int64_t n_early = units < S ? units : S;
        for (; u < n_early; ++u) issue();
      }
      pdl_wait();
      AWQ_TRACE_AT(rec, kTrWaited, globaltimer_ns());
      // every kernel before this one has completed: the next grid may now be scheduled
      pdl_launch_dependents();
      for (; u < units; ++u) {
        if (!mbar_wait(&empty[slot], ph ^ 1)) break;
        issue();
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int r = lane >> 2, c = lane & 3;
  const int rw = (r >> 1) + 4 * (r & 1);   // weight row (of the tile) of the MMA's row r
  pdl_wait();   // X may be the preceding kernel's output
  // Stage X: x <- x * inv_s (kDiv16: columns k%8 in {2,3,6,7} / 16), in B-fragment order, and
  // for M = 1 per-(group, token) C1 / C2. Chunk i (8 values) of X is taken by consumer
  // thread i % 256 in round i / (256 kG4XRound), every load of a round issued before any is
  // used; the 16 chunks of one (token, group) are 16 consecutive lanes of one warp (four
  // xor-shuffles for the sums).
  {
    const int nch = M * Ki / 8;
    const int kpr = Ki / 8;   // chunks per token row
    const int tid = static_cast<int>(threadIdx.x);   // < kG4Warps * 32 (the producer returned)
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    for (int base = 0; base < nch; base += kG4Warps * 32 * kG4XRound) {
      uint4 v[kG4XRound];
      float4 s0[kG4XRound], s1[kG4XRound];
#pragma unroll
      for (int e = 0; e < kG4XRound; ++e) {
        if (base + e * kG4Warps * 32 >= nch) break;
        const int i = base + e * kG4Warps * 32 + tid;
        v[e] = i < nch ? *reinterpret_cast<const uint4*>(X + static_cast<int64_t>(i) * 8)
                       : make_uint4(0u, 0u, 0u, 0u);
        if (inv_s != nullptr && i < nch) {
          const int k = (M == 1 ? i : i % kpr) * 8;
          s0[e] = *reinterpret_cast<const float4*>(inv_s + k);
          s1[e] = *reinterpret_cast<const float4*>(inv_s + k + 4);
        }
      }
#pragma unroll
      for (int e = 0; e < kG4XRound; ++e) {
        if (base + e * kG4Warps * 32 >= nch) break;   // the same for every thread
        const int i = base + e * kG4Warps * 32 + tid;
        const bool live = i < nch;   // whole 16-lane blocks are live or not
        // (M = 1: one token row, no division)
        const int m = M == 1 ? 0 : i / kpr, rem = M == 1 ? i : i % kpr, g = rem >> 4, ch = rem & 15;
        if (inv_s != nullptr && live) v[e] = scale8<kBf16>(v[e], s0[e], s1[e]);
        if (kOffset && kDiv16) {
          v[e].y = h2_as_u32(__hmul2(u32_as_h2(v[e].y), sixteenth));
          v[e].w = h2_as_u32(__hmul2(u32_as_h2(v[e].w), sixteenth));
        }
        // chunk ch holds k = 8 ch .. 8 ch + 7 of the group: 32-k quarter ch / 4, 8-k chunk ch % 4
        const int dst = ((g * 4 + (ch & 3)) * M + m) * 4 + (ch >> 2);
        if (live && AWQ_IN_BOUNDS(dst < G * 16 * M)) reinterpret_cast<uint4*>(xs)[dst] = v[e];
        if (kOffset) {
          const float2 lx = act2_to_float2<kBf16>(v[e].x), hy = act2_to_float2<kBf16>(v[e].y);
          const float2 lz = act2_to_float2<kBf16>(v[e].z), hw = act2_to_float2<kBf16>(v[e].w);
          const float lo = (lx.x + lx.y) + (lz.x + lz.y), hi = (hy.x + hy.y) + (hw.x + hw.y);
          float c1 = lo + hi, c2 = kDiv16 ? lo + 16.0f * hi : lo + hi;
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) {
            c1 += __shfl_xor_sync(0xffffffffu, c1, o);
            c2 += __shfl_xor_sync(0xffffffffu, c2, o);
          }
          if (ch == 0 && live) {
            // C1 = base * sum of the staged values (c1 == c2 unless kDiv16)
            cc[(g * kTok + m) * 2] = kBf16 ? 128.0f * c2 : 1024.0f * c1;
            cc[(g * kTok + m) * 2 + 1] = c2;
          }
        }
      }
    }
    if (kOffset)
      for (int i = tid; i < G * kTok; i += kG4Warps * 32)
        if (i % kTok >= M) {
          cc[2 * i] = 0.0f;
          cc[2 * i + 1] = 0.0f;
        }
    named_bar_sync(1, kG4Warps * 32);
    if (threadIdx.x == 0) AWQ_TRACE_AT(rec, kTrXStaged, globaltimer_ns());
  }

  // A timed-out wait clears `ok`; the warp then skips further waits and arithmetic but still
  // runs every named barrier, so the consumer warps cannot deadlock one another.
  bool ok = true;
  float total[kNTiles][4];
#pragma unroll
  for (int t = 0; t < kNTiles; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) total[t][i] = 0.0f;

  int slot = 0, chunk = 0;
  uint32_t ph = 0;
  int64_t tile = t0;
  for (int64_t u = 0; u < units; ++u) {
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&full[slot], ph));
    if (threadIdx.x == 0 && u < kTrMaxUnits) AWQ_TRACE_AT(rec, kTrUnit0 + u, globaltimer_ns());
    // Copy this warp's operands of the unit (its two groups: packed codes of rows r and r + 8,
    // their scales and zero points) to registers and release the slot at once, so the
    // producer refills it while this unit is computed. Every lane arrives (release
    // semantics), which orders its own shared-memory reads first.
    const uint8_t* wb = wslots + slot * kG4WSlot;
    const uint8_t* sz = szslots + slot * (kG4SBytes + kG4ZBytes);
    uint4 wA[2], wB[2];   // 4-bit: words 4c..4c+3 of the group; 3-bit: .x .y .z = the lane's
                          // 32-k block (low words, bit-2 word)
    uint32_t zAi[2], zBi[2];
    float scA[2], scB[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int gl = 2 * warp + q;               // group inside the unit
      if constexpr (kBits == 4) {
        const int w0 = gl * 16 + 4 * c;          // one 16-byte chunk of a swizzled box
        wA[q] = *reinterpret_cast<const uint4*>(wb + g4_word_offset(rw, w0));
        wB[q] = *reinterpret_cast<const uint4*>(wb + g4_word_offset(rw + 8, w0));
      } else {
        const int w0 = gl * 12 + 3 * c;          // three words, possibly in two chunks
        wA[q] = make_uint4(*reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw, w0)),
                           *reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw, w0 + 1)),
                           *reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw, w0 + 2)), 0u);
        wB[q] = make_uint4(*reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw + 8, w0)),
                           *reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw + 8, w0 + 1)),
                           *reinterpret_cast<const uint32_t*>(wb + g4_word_offset(rw + 8, w0 + 2)),
                           0u);
      }
      const __half* ss = reinterpret_cast<const __half*>(sz) + gl * kGemvRows;
      const uint8_t* zz = sz + kG4SBytes + gl * kGemvRows;
      zAi[q] = zz[rw];
      zBi[q] = zz[rw + 8];
      scA[q] = __half2float(ss[rw]);
      scB[q] = __half2float(ss[rw + 8]);
    }
    if (ok) mbar_arrive(&empty[slot]);
    if (++slot == S) { slot = 0; ph ^= 1; }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int gl = 2 * warp + q;
      const int g = chunk * kG4Groups + gl;
      if (ok && g < G) {
        float acc[kNTiles][4][4];
#pragma unroll
        for (int t = 0; t < kNTiles; ++t)
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[t][j][i] = 0.0f;
        const uint32_t wordsA[4] = {wA[q].x, wA[q].y, wA[q].z, wA[q].w};
        const uint32_t wordsB[4] = {wB[q].x, wB[q].y, wB[q].z, wB[q].w};
        __half2 loA, hiA, loB, hiB;
        uint32_t bA = 0, bB = 0;   // bf16 bias pairs (128 + z)
        if (!kOffset) {
          if constexpr (kBf16) {
            bA = (0x4300u | zAi[q]) * 0x00010001u;
            bB = (0x4300u | zBi[q]) * 0x00010001u;
          } else {
            loA = u32_as_h2((0x6400u | zAi[q]) * 0x00010001u);
            hiA = u32_as_h2((0xD400u | (zAi[q] << 4)) * 0x00010001u);
            loB = u32_as_h2((0x6400u | zBi[q]) * 0x00010001u);
            hiB = u32_as_h2((0xD400u | (zBi[q] << 4)) * 0x00010001u);
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t va[4], vb[4];
          if constexpr (kBits == 3) {
            raw3_chunk<kBf16>(wA[q].x, wA[q].y, wA[q].z, j, va);
            raw3_chunk<kBf16>(wB[q].x, wB[q].y, wB[q].z, j, vb);
            if (!kOffset) {   // minus the bias pair (1024 + z) / (128 + z): the exact q - z
              const uint32_t ba = ((kBf16 ? 0x4300u : 0x6400u) | zAi[q]) * 0x00010001u;
              const uint32_t bb = ((kBf16 ? 0x4300u : 0x6400u) | zBi[q]) * 0x00010001u;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if constexpr (kBf16) {
                  va[i] = b2_as_u32(__hsub2(u32_as_b2(va[i]), u32_as_b2(ba)));
                  vb[i] = b2_as_u32(__hsub2(u32_as_b2(vb[i]), u32_as_b2(bb)));
                } else {
                  va[i] = h2_as_u32(__hsub2(u32_as_h2(va[i]), u32_as_h2(ba)));
                  vb[i] = h2_as_u32(__hsub2(u32_as_h2(vb[i]), u32_as_h2(bb)));
                }
              }
            }
          } else if (kOffset) {
            raw_word<kBf16>(wordsA[j], va);
            raw_word<kBf16>(wordsB[j], vb);
          } else if constexpr (kBf16) {
            dequant_word_qz_bf16(wordsA[j], bA, va);
            dequant_word_qz_bf16(wordsB[j], bB, vb);
          } else {
            dequant_word_qz(wordsA[j], loA, hiA, va);
            dequant_word_qz(wordsB[j], loB, hiB, vb);
          }
#pragma unroll
          for (int t = 0; t < kNTiles; ++t) {
            const int m = r + 8 * t;
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (m < M && AWQ_IN_BOUNDS(((g * 4 + j) * M + m) * 4 + c < G * 4 * M * 4))
              xv = reinterpret_cast<const uint4*>(xs)[((g * 4 + j) * M + m) * 4 + c];
            const uint32_t a0[4] = {va[0], vb[0], va[1], vb[1]};
            mma_16816<kBf16>(acc[t][j], a0, xv.x, xv.y);
            const uint32_t a1[4] = {va[2], vb[2], va[3], vb[3]};
            mma_16816<kBf16>(acc[t][j], a1, xv.z, xv.w);
          }
        }
#pragma unroll
        for (int t = 0; t < kNTiles; ++t) {
          float d[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) d[i] = (acc[t][0][i] + acc[t][1][i]) + (acc[t][2][i] + acc[t][3][i]);
          if (kOffset && AWQ_IN_BOUNDS((g * kTok + 8 * t + 2 * c) * 2 + 4 <= G * kTok * 2)) {
            const float zA = static_cast<float>(zAi[q]), zB = static_cast<float>(zBi[q]);
            const float4 cm = *reinterpret_cast<const float4*>(cc + (g * kTok + 8 * t + 2 * c) * 2);
            d[0] -= fmaf(zA, cm.y, cm.x);
            d[1] -= fmaf(zA, cm.w, cm.z);
            d[2] -= fmaf(zB, cm.y, cm.x);
            d[3] -= fmaf(zB, cm.w, cm.z);
          }
          total[t][0] = fmaf(scA[q], d[0], total[t][0]);
          total[t][1] = fmaf(scA[q], d[1], total[t][1]);
          total[t][2] = fmaf(scB[q], d[2], total[t][2]);
          total[t][3] = fmaf(scB[q], d[3], total[t][3]);
        }
      }
    }

    if (chunk == C - 1) {
      // tile complete: fixed-order sum over the consumer warps, store
#pragma unroll
      for (int t = 0; t < kNTiles; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          red[((warp * kNTiles + t) * 4 + i) * 32 + lane] = total[t][i];
          total[t][i] = 0.0f;
        }
      named_bar_sync(1, kG4Warps * 32);
      if (ok && warp < kNTiles) {
        const int t = warp;
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float sum = 0.0f;
#pragma unroll
          for (int w = 0; w < kG4Warps; ++w) sum += red[((w * kNTiles + t) * 4 + i) * 32 + lane];
          v[i] = sum;
        }
        const int64_t nA = tile * kGemvRows + rw, nB = nA + 8;
        const int m0 = 8 * t + 2 * c, m1 = m0 + 1;
        if (nA < N && AWQ_IN_BOUNDS(tile < t1)) {
          if (m0 < M) Y[static_cast<int64_t>(m0) * N + nA] = float_to_act<kBf16>(v[0]);
          if (m1 < M) Y[static_cast<int64_t>(m1) * N + nA] = float_to_act<kBf16>(v[1]);
        }
        if (nB < N && AWQ_IN_BOUNDS(tile < t1)) {
          if (m0 < M) Y[static_cast<int64_t>(m0) * N + nB] = float_to_act<kBf16>(v[2]);
          if (m1 < M) Y[static_cast<int64_t>(m1) * N + nB] = float_to_act<kBf16>(v[3]);
        }
      }
      named_bar_sync(1, kG4Warps * 32);
    }
    if (++chunk == C) { chunk = 0; ++tile; }
  }
  if (threadIdx.x == 0) AWQ_TRACE_AT(rec, kTrEnd, globaltimer_ns());
}

}  // namespace awq
