// K4: W4A16 GEMM on the 5th-generation tensor cores, and the error GEMM of the scale search.
//
// builderai.tools "AWQ", "About" (kernels for 4-bit weights with 16-bit activations);
// robotsatlas.com "AWQ", "Implementation pitfalls: Missing matched inference kernels"
// (dequantization must live inside the GEMM); robotsatlas.com "AWQ", "How it works" (the
// search scores each candidate scale by the layer's output error).
//
// Swap-AB formulation: the MMA's M side is 128 weight rows (output features n) and its N
// side is BN tokens, so D = W_tile * X_tile^T lands in TMEM as 128 lanes (one per output
// feature) x BN fp32 columns (one per token), and each dequantized weight is reused across
// BN tokens. Persistent: one CTA per SM walks the (tile, K slice) work units in a grouped
// order (see tile_of_block) with a shared-memory ring of K stages that runs on across tiles
// (a stage is one 64-k block, or for packed sources two: a whole 128-k group, so the MMA
// thread's per-stage waits and commit are paid once per eight MMAs), and two TMEM
// accumulators so a tile's epilogue overlaps the next tile's main loop:
//   warp 5       TMA producer: X slice (128-byte swizzle), and both parts of the A slice
//                (two-part fp16 source);
//   warp 1       TMEM allocator and single-thread tcgen05.mma issuer (kind::f16, fp32 acc);
//   warp 9       TMA producer of the packed source: kPG consecutive 128-k groups of packed
//                weights (with their scales and zero points) per slot of a ring as deep as
//                shared memory allows, running ahead of the stage ring. When few tokens share
//                each weight the kernel streams weights from DRAM, and TMA tiles of 128 rows
//                only reach full DRAM throughput with long rows (about 2.7 TB/s at 64 bytes
//                per row, 4.7 at 128, 5.5-5.9 at 256 on B200), so narrow token tiles take
//                four groups (256 bytes of 4-bit codes) per row per slot;
//   warps 0, 2, 3, 4, 6, 7, 8, 10
//                A builders (packed sources): 16-byte packed chunks from shared memory ->
//                fp16 (q - z) * scale in registers -> the canonical 128-byte swizzled
//                K-major layout, then fence.proxy.async so the tensor core sees the writes;
//   warps 12..15 epilogue: tcgen05.ld of their 32-lane quarter of the finished accumulator,
//                then fp16 Y, fp32 split-K partials, or (search) per-row sums of squares;
//   warp 11      idle.
// Warp w issues from sub-partition w % 4. The MMA issuer and both TMA producers share
// sub-partition 1 and no builder runs there: a builder warp placed beside the MMA issuer
// (or beside the X producer) was measured finishing its part of each stage 2000-3700
// cycles after the other builders, which held every MMA back by as much.
// Every mbarrier wait is bounded; a timeout sets the device status word and the roles
// leave their loops so the CTA still releases its TMEM and exits.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kTcBM = 128;      // weight rows per tile (MMA M)
constexpr int kTcBK = 64;       // K per stage: one 128-byte swizzle atom of fp16
constexpr int kTcBuilders = 8;  // A-builder warps
constexpr int kTcEpiWarps = 4;  // epilogue warps (one per TMEM lane quarter)
constexpr int kTcThreads = 16 * 32;
constexpr int kTcMmaWarp = 1;
constexpr int kTcXWarp = 5;
constexpr int kTcPackWarp = 9;
constexpr int kTcIdleWarp = 11;
constexpr int kTcEpiWarp0 = 12;   // warps 12..15: TMEM lane quarters 0..3 (warp % 4)
constexpr int kTcPkSlotsMax = 16;   // deepest packed ring
constexpr int kTcSmemMax = 232448;  // dynamic shared memory per CTA on sm_100

// kSplit16: the search's error operand in two fp16 parts, E = hi + 2^-12 lo, stored as one
// [rows, 2K] matrix (hi in columns 0..K-1, lo in K..2K-1); each part has its own accumulator
// and the epilogue combines them in fp32.
// kPair16: two fp16 weights of the same shape (a gated MLP's gate_proj and up_proj); the
// same rows of both are the two A parts, each with its own accumulator.
// kFp16x1: one plain fp16 matrix (the Gram matrix X^T X of the calibration tokens).
// kGram: the search's error operand (two parts, as kSplit16) against the normalised Gram
// matrix, itself in two fp16 parts [hi | lo] as the B operand: per 16-k step the MMAs
// A_hi B_hi -> accumulator 0 and A_hi B_lo, A_lo B_hi -> accumulator 1, recombined as
// D = D_0 + 2^-12 D_1 (the lo x lo product, 2^-24 relative, is left out).
enum class ASrc : int { kPacked4 = 0, kPacked3 = 1, kSplit16 = 2, kPair16 = 3, kFp16x1 = 4,
                        kGram = 5 };
// kStoreY: fp16 Y (or fp32 split-K partials); kRowSumSq: per-row sums of squares of the
// recombined two-part product; kSiluMul: fp16 H = silu(D_0) * D_1 of the two accumulators;
// kStoreF32: the fp32 product itself (the Gram matrix); kGramDot: per-row sums of
// D[n][j] * e'[n][j], the recombined product times the row's own error operand.
enum class Epi : int { kStoreY = 0, kRowSumSq = 1, kSiluMul = 2, kStoreF32 = 3, kGramDot = 4 };

template <int BN, ASrc kA, int kBlkT = 1>
struct TcLayout {
  static constexpr bool kPk = kA == ASrc::kPacked4 || kA == ASrc::kPacked3;
  static constexpr int kXParts = kA == ASrc::kGram ? 2 : 1;   // B tiles per stage
  static constexpr int kAParts = (kPk || kA == ASrc::kFp16x1) ? 1 : 2;   // A tiles (and
                                                                       // accumulators) per stage
  // packed sources with kBlkT = 2: two 64-k blocks (one 128-k group) per pipeline stage, so
  // the single MMA-issuing thread waits and commits once per eight MMAs instead of four
  static constexpr int kBlk = kPk ? kBlkT : 1;
  static constexpr int kXPartBytes = BN * kTcBK * 2;
  static constexpr int kXBlockBytes = kXParts * kXPartBytes;
  static constexpr int kXBytes = kBlk * kXBlockBytes;   // per stage
  static constexpr int kStages =
      kA == ASrc::kGram ? (BN >= 256 ? 2 : BN >= 128 ? 3 : 4)
      : kA == ASrc::kFp16x1 ? (BN >= 256 ? 4 : 6)
      : !kPk ? (BN >= 256 ? 3 : BN >= 128 ? 4 : BN >= 64 ? 5 : 6)
             : kBlk == 2 ? (BN >= 128 ? 2 : 3)   // packed, stages of two blocks
                         : (BN >= 256 ? 4 : BN >= 64 ? 5 : 6);
  static constexpr int kAPartBytes = kTcBM * kTcBK * 2;
  static constexpr int kABlockBytes = kAParts * kAPartBytes;
  static constexpr int kABytes = kBlk * kABlockBytes;   // per stage
  // packed source: kPG groups (2 kPG stages) per ring slot
  static constexpr int kPG = !kPk ? 1 : BN <= 64 ? 4 : BN <= 128 ? 2 : 1;
  static constexpr int kPGroupBytes = kA == ASrc::kPacked4 ? 64 : kA == ASrc::kPacked3 ? 48 : 0;
  static constexpr int kPRowBytes = kPG * kPGroupBytes;
  static constexpr int kPBytes = kTcBM * kPRowBytes;
  // the slot's fp16 scales [kPG][128] then its zero points [kPG][128]
  static constexpr int kSZBytes = kPG * (kTcBM * 2 + kTcBM);
  // the slot's inv_s [kPG][128] fp32 (packed sources with inv_s): the builders read it from
  // shared memory, broadcast across the tile's rows
  static constexpr int kInvBytes = kPk ? kPG * kGroup * 4 : 0;
  // as many packed slots as the shared memory left by the stages holds (1024 bytes of
  // alignment slack and 512 of barriers reserved)
  static constexpr int kPFit =
      (kTcSmemMax - 1024 - 512 - kStages * (kXBytes + kABytes)) /
      (kPBytes + kSZBytes + kInvBytes);
  static constexpr int kPSlots =
      !kPk ? 0 : (kPFit < kTcPkSlotsMax ? kPFit : kTcPkSlotsMax);
  static constexpr int kPBars = kPSlots > 0 ? kPSlots : 1;   // barrier pairs of the ring
  static constexpr int kXOff = 0;
  static constexpr int kAOff = kXOff + kStages * kXBytes;
  static constexpr int kPOff = kAOff + kStages * kABytes;
  static constexpr int kSZOff = kPOff + kPSlots * kPBytes;
  static constexpr int kIOff = kSZOff + kPSlots * kSZBytes;
  static constexpr int kBarOff = kIOff + kPSlots * kInvBytes;
  // full[S], empty[S], built[S], pfull[P], pempty[P], acc_full[2], acc_empty[2], tmem slot
  static constexpr int kBytes = kBarOff + (3 * kStages + 2 * kPBars + 4) * 8 + 16;
  static constexpr int kSmem = kBytes + 1024;   // slack for 1024-byte alignment
  static constexpr uint32_t kTxBytes = kXBytes + (kPk ? 0 : kABytes);
  // one accumulator per A part, double-buffered when TMEM's 512 columns allow (so a tile's
  // epilogue overlaps the next tile's main loop); a power of 2 of at least 32 columns
  static constexpr int kAccBufs = 2 * kAParts * BN <= 512 ? 2 : 1;
  static constexpr uint32_t kTmemCols = kAccBufs * kAParts * BN;
};

struct TcArgs {
  int64_t M;            // tokens
  int64_t N;            // valid weight rows (store epilogue) / rows per grid point (search)
  int64_t N_pad;        // rows per grid point including padding (search); N for the GEMM
  int64_t K;
  const __half* scales; // [K/128, N] (packed source)
  const uint8_t* zeros; // [K/128, N]
  void* Y;              // [M, N] fp16 (bf16 with bf16 activations): Y or the SiLU output H
  double* row_part;     // [m_tiles, rows_total] (search epilogue)
  int m_tiles;
  int row_tiles;        // 128-row tiles of the A matrix
  int64_t rows_total;   // rows of the A matrix (row_tiles * 128 for the search)
  int k_splits;         // > 1: each work unit covers a group-aligned slice of K (split-K)
  float* partial;       // [k_splits, M, N] fp32 partial sums (split-K store epilogue)
  int sz_tma;           // packed source: scales and zeros arrive by TMA with the packed group
                        // (needs N % 16 == 0); else the builders load them from global memory
  const float* inv_s;   // packed source: NULL, or [K] factors folded into the weights
  float* G;             // kStoreF32: [rows_total, M] fp32 output (the Gram matrix)
  int upper_only;       // kStoreF32: compute only the tiles that reach the diagonal or above it
                        // (G is symmetric; readers take G[min(i,j)][max(i,j)])
  const __half* E2;     // kGramDot: the error operand [rows_total, 2K] the epilogue reads
};

// Grouped tile order: consecutive work units sweep the token tiles of a group of
// kTcRasterRows weight-row tiles, so the units in flight at one time share a few A tiles and
// a few X tiles in L2 instead of each streaming its own X tile from HBM.
constexpr int kTcRasterRows = 16;

__device__ __forceinline__ void tile_of_block(int64_t bid, int row_tiles, int m_tiles,
                                              int& row_tile, int& m_tile) {
  const int64_t per_group = static_cast<int64_t>(kTcRasterRows) * m_tiles;
  const int64_t group = bid / per_group;
  const int64_t in_group = bid % per_group;
  const int first = static_cast<int>(group) * kTcRasterRows;
  const int rows_here = row_tiles - first < kTcRasterRows ? row_tiles - first : kTcRasterRows;
  row_tile = first + static_cast<int>(in_group % rows_here);
  m_tile = static_cast<int>(in_group / rows_here);
}

struct TcUnit {
  int row_tile, m_tile, ksplit, kb0, nkb;
};

__device__ __forceinline__ TcUnit unit_of(int64_t u, const TcArgs& a) {
  TcUnit t;
  const int64_t tiles = static_cast<int64_t>(a.row_tiles) * a.m_tiles;
  t.ksplit = static_cast<int>(u / tiles);
  tile_of_block(u % tiles, a.row_tiles, a.m_tiles, t.row_tile, t.m_tile);
  const int G = static_cast<int>(a.K / kGroup);
  const int kb0 = 2 * static_cast<int>(static_cast<int64_t>(t.ksplit) * G / a.k_splits);
  const int kb1 = 2 * static_cast<int>(static_cast<int64_t>(t.ksplit + 1) * G / a.k_splits);
  t.kb0 = kb0;
  t.nkb = kb1 - kb0;
  return t;
}

// Dequantize one 4-bit packed word (8 consecutive k) to four fp16 pairs (q - z) * c, with
// one scale pair per k pair: (k0,k1) by c.x, (k2,k3) by c.y, (k4,k5) by c.z, (k6,k7) by c.w
// (all four the group's scale, or the scale times the per-channel inv_s).
__device__ __forceinline__ uint4 dequant_word_scaled(uint32_t w, __half2 bias_lo,
                                                     __half2 bias_hi, uint4 c) {
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const uint32_t w8 = w >> 8;
  const uint32_t v0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  const uint32_t v1 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  const uint32_t v2 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
  const uint32_t v3 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
  uint4 o;
  o.x = h2_as_u32(__hmul2(__hsub2(u32_as_h2(v0), bias_lo), u32_as_h2(c.x)));
  o.y = h2_as_u32(__hmul2(__hfma2(u32_as_h2(v1), sixteenth, bias_hi), u32_as_h2(c.y)));
  o.z = h2_as_u32(__hmul2(__hsub2(u32_as_h2(v2), bias_lo), u32_as_h2(c.z)));
  o.w = h2_as_u32(__hmul2(__hfma2(u32_as_h2(v3), sixteenth, bias_hi), u32_as_h2(c.w)));
  return o;
}

// The four scale pairs of 8 consecutive k starting at k0: fp16(sc * inv_s[k]) pairs, or sc
// broadcast when inv_s is NULL (bf16 pairs for bf16 activations). inv_s points at the
// group's factors in the packed slot (shared memory) and k0 is relative to the group. Folding inv_s into the
// weights computes sum_k x[k] * (inv_s[k] * deq[k]) = sum_k (x[k] * inv_s[k]) * deq[k].
template <bool kBf16 = false>
__device__ __forceinline__ uint4 pair_scales(float sc, uint32_t sc2, const float* inv_s,
                                             int64_t k0) {
  if (inv_s == nullptr) return make_uint4(sc2, sc2, sc2, sc2);
  const float4 a = *reinterpret_cast<const float4*>(inv_s + k0);
  const float4 b = *reinterpret_cast<const float4*>(inv_s + k0 + 4);
  return make_uint4(float2_to_act2<kBf16>(sc * a.x, sc * a.y),
                    float2_to_act2<kBf16>(sc * a.z, sc * a.w),
                    float2_to_act2<kBf16>(sc * b.x, sc * b.y),
                    float2_to_act2<kBf16>(sc * b.z, sc * b.w));
}

// bf16 form of the 4-bit dequantization: the exact (q - z) pairs (raw 128 + q minus the bias
// pair 128 + z) times the scale pairs, one bf16 rounding of each product.
__device__ __forceinline__ uint4 dequant_word_scaled_bf16(uint32_t w, uint32_t bias, uint4 c) {
  const uint32_t v[4] = {lop3_and_or(w, 0x000F000Fu, 0x43004300u),
                         lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u),
                         lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u),
                         lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u)};
  const uint32_t cc[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = b2_as_u32(__hmul2(__hsub2(u32_as_b2(v[i]), u32_as_b2(bias)), u32_as_b2(cc[i])));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 3-bit: the fp16 pair (q - z) * sc for k-offsets (2e, 2e+1) of chunk i (k = 8i..8i+7) of a
// 32-k block whose low-bit words are w0 (offsets 0..15) / w1 (16..31) and whose bit-2 word
// is w2 (the pair's two bits sit at bits hb and hb + 16; both are moved to bit 2 of their
// 16-bit half by a single shift whose direction is fixed at compile time).
template <int kI, int kE, bool kBf16 = false>
__device__ __forceinline__ uint32_t dequant3_pair(uint32_t w0, uint32_t w1, uint32_t w2,
                                                  uint32_t bias_lo, uint32_t sc2u) {
  constexpr int pp = 4 * (kI & 1) + kE;     // 2-bit field of the pair inside its low word
  constexpr int hb = 4 * kI + kE;           // bit of the pair inside the bit-2 word
  const uint32_t wlo = (kI < 2) ? w0 : w1;
  // 1024 + q in fp16 (0x6400), 128 + q in bf16 (0x4300): q in the low mantissa bits
  const uint32_t lo = lop3_and_or(wlo >> (2 * pp), 0x00030003u, kBf16 ? 0x43004300u : 0x64006400u);
  const uint32_t hs = hb >= 2 ? (w2 >> (hb >= 2 ? hb - 2 : 0)) : (w2 << (hb < 2 ? 2 - hb : 0));
  uint32_t v;
  // (hs & 0x00040004) | lo
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(v) : "r"(hs), "r"(0x00040004u), "r"(lo));
  if constexpr (kBf16)
    return b2_as_u32(__hmul2(__hsub2(u32_as_b2(v), u32_as_b2(bias_lo)), u32_as_b2(sc2u)));
  else
    return h2_as_u32(__hmul2(__hsub2(u32_as_h2(v), u32_as_h2(bias_lo)), u32_as_h2(sc2u)));
}

// Byte offset of 16-byte chunk c (k = 8c..8c+7) of row r in a 64-wide fp16 tile stored in
// the 128-byte swizzled K-major layout (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

template <int BN, ASrc kA, Epi kEpi, bool kBf16 = false, int kBlkT = 1>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_s,
                   const __grid_constant__ CUtensorMap tmap_z, const TcArgs args) {
  using L = TcLayout<BN, kA, kBlkT>;
  constexpr int S = L::kStages;
  constexpr bool kPacked = L::kPk;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + S;
  uint64_t* built = empty + S;
  uint64_t* pfull = built + S;
  constexpr int P = L::kPBars;
  static_assert(!kPacked || L::kPSlots >= 2, "packed ring needs two slots");
  static_assert(kEpi != Epi::kRowSumSq || kA == ASrc::kSplit16,
                "the sum-of-squares epilogue recombines the two-part error operand");
  static_assert(kEpi != Epi::kStoreF32 || kA == ASrc::kFp16x1, "the Gram product");
  static_assert(kEpi != Epi::kGramDot || kA == ASrc::kGram, "the Gram-form loss");
  static_assert(kEpi != Epi::kSiluMul || kA == ASrc::kPair16,
                "the SiLU epilogue combines the gate and up accumulators");
  static_assert(kEpi != Epi::kStoreY || kPacked, "fp16 Y comes from the packed sources");
  static_assert(L::kSmem <= kTcSmemMax, "shared memory layout too large");
  uint64_t* pempty = pfull + P;
  uint64_t* acc_full = pempty + P;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t units =
      static_cast<int64_t>(args.row_tiles) * args.m_tiles * args.k_splits;
  if (kEpi == Epi::kStoreF32 && args.upper_only) {
    // One CTA per output tile: a tile whose rows all lie below its columns (every element
    // G[i][j] with i > j) is the transpose of a computed one, so its CTA has nothing to do.
    int row_tile, m_tile;
    tile_of_block(blockIdx.x % (static_cast<int64_t>(args.row_tiles) * args.m_tiles),
                  args.row_tiles, args.m_tiles, row_tile, m_tile);
    if (static_cast<int64_t>(row_tile) * kTcBM >= static_cast<int64_t>(m_tile + 1) * BN) return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&built[i], kTcBuilders * 32);
    }
    for (int i = 0; i < P; ++i) {
      mbar_init(&pfull[i], 1);
      mbar_init(&pempty[i], kTcBuilders * 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kTcEpiWarps * 32);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_a);
    if (kPacked && args.sz_tma) {
      tma_prefetch_desc(&tmap_s);
      tma_prefetch_desc(&tmap_z);
    }
    if (kA == ASrc::kPair16) tma_prefetch_desc(&tmap_s);
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Programmatic dependent launch: the setup above may overlap the previous kernel on the
  // stream; every thread waits for that kernel's completion (and memory) before its first
  // global access, and only then lets the next kernel launch (so a kernel that starts early
  // behind this one overlaps this kernel alone, never an earlier one).
  pdl_wait();
  pdl_launch_dependents();

  if (warp == kTcXWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;          // stage slot and phase, continuous across units
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const TcUnit t = unit_of(u, args);
        const int64_t m0 = static_cast<int64_t>(t.m_tile) * BN;
        const int64_t row0 = static_cast<int64_t>(t.row_tile) * kTcBM;
        for (int i = 0; i < t.nkb; i += L::kBlk) {
          const int kb = t.kb0 + i;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kTxBytes);
#pragma unroll
          for (int b = 0; b < L::kBlk; ++b)
            tma_load_2d(smem + L::kXOff + s * L::kXBytes + b * L::kXBlockBytes, &tmap_x,
                        &full[s], (kb + b) * kTcBK, static_cast<int32_t>(m0));
          if (kA == ASrc::kGram)   // the lo part of the normalised Gram matrix
            tma_load_2d(smem + L::kXOff + s * L::kXBytes + L::kXPartBytes, &tmap_x, &full[s],
                        static_cast<int32_t>(args.K) + kb * kTcBK, static_cast<int32_t>(m0));
          if (kA == ASrc::kFp16x1) {
            tma_load_2d(smem + L::kAOff + s * L::kABytes, &tmap_a, &full[s], kb * kTcBK,
                        static_cast<int32_t>(row0));
          } else if (kA == ASrc::kSplit16 || kA == ASrc::kGram) {
            uint8_t* a = smem + L::kAOff + s * L::kABytes;
            tma_load_2d(a, &tmap_a, &full[s], kb * kTcBK, static_cast<int32_t>(row0));
            tma_load_2d(a + L::kAPartBytes, &tmap_a, &full[s],
                        static_cast<int32_t>(args.K) + kb * kTcBK, static_cast<int32_t>(row0));
          } else if (kA == ASrc::kPair16) {   // gate rows, then the same rows of up
            uint8_t* a = smem + L::kAOff + s * L::kABytes;
            tma_load_2d(a, &tmap_a, &full[s], kb * kTcBK, static_cast<int32_t>(row0));
            tma_load_2d(a + L::kAPartBytes, &tmap_s, &full[s], kb * kTcBK,
                        static_cast<int32_t>(row0));
          }
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = f16_idesc(kTcBM, BN, kBf16);
      int s = 0;
      uint32_t ph = 0;
      int64_t lt = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x, ++lt) {
        const TcUnit t = unit_of(u, args);
        const int buf = static_cast<int>(lt % L::kAccBufs);
        const uint32_t acc_ph = static_cast<uint32_t>((lt / L::kAccBufs) & 1);
        if (!mbar_wait(&acc_empty[buf], acc_ph ^ 1)) break;   // epilogue released the buffer
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * L::kAParts * BN);
        for (int i = 0; i < t.nkb; i += L::kBlk) {
          ok = mbar_wait(&full[s], ph);
          if (ok && kPacked) ok = mbar_wait(&built[s], ph);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int b = 0; b < L::kBlk; ++b) {
          const uint32_t a_base = smem_u32(smem + L::kAOff + s * L::kABytes + b * L::kABlockBytes);
          const uint32_t x_base = smem_u32(smem + L::kXOff + s * L::kXBytes + b * L::kXBlockBytes);
#pragma unroll
          for (int kk = 0; kk < kTcBK / 16; ++kk) {
            const uint32_t acc = (i | b | kk) != 0 ? 1u : 0u;
            if (kA == ASrc::kGram) {
              // A_hi B_hi -> D_0; A_hi B_lo + A_lo B_hi -> D_1
              const uint64_t ah = sw128_kmajor_desc(a_base + kk * 32);
              const uint64_t al = sw128_kmajor_desc(a_base + L::kAPartBytes + kk * 32);
              const uint64_t bh = sw128_kmajor_desc(x_base + kk * 32);
              const uint64_t bl = sw128_kmajor_desc(x_base + L::kXPartBytes + kk * 32);
              tc_mma_f16(d_tmem, ah, bh, idesc, acc);
              tc_mma_f16(d_tmem + static_cast<uint32_t>(BN), ah, bl, idesc, acc);
              tc_mma_f16(d_tmem + static_cast<uint32_t>(BN), al, bh, idesc, 1u);
            } else {
#pragma unroll
              for (int part = 0; part < L::kAParts; ++part)   // part p: A tile p -> accumulator p
                tc_mma_f16(d_tmem + static_cast<uint32_t>(part * BN),
                           sw128_kmajor_desc(a_base + part * L::kAPartBytes + kk * 32),
                           sw128_kmajor_desc(x_base + kk * 32), idesc, acc);
            }
          }
          }
          tc_commit(&empty[s]);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        tc_commit(&acc_full[buf]);
      }
    }
  } else if (warp < kTcEpiWarp0 && warp != kTcPackWarp && warp != kTcIdleWarp) {
    // ------------------------------------------------------------------ A builders
    if (kPacked) {
      // builder index 0..7 of warps 0, 2, 3, 4, 6, 7, 8, 10 (skipping sub-partition 1)
      const int t = (warp - (warp + 3) / 4) * 32 + lane;   // 0..255
      const int r = t >> 1, h = t & 1;         // tile row, 32-k half of the 64-k stage
      const int64_t N = args.N;
      int s = 0, ps = 0;      // stage slot and packed slot, with their phases
      uint32_t ph = 0, pph = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const TcUnit tu = unit_of(u, args);
        const int64_t n = static_cast<int64_t>(tu.row_tile) * kTcBM + r;
        // one 128-k group per iteration: the stage's two 64-k blocks are built, then one proxy
        // fence and one arrival (K slices are whole groups, so nkb is even)
        for (int i = 0; i < tu.nkb; i += 2) {
          const int kb = tu.kb0 + i;
          uint32_t z = 0;
          __half sv = __float2half(0.0f);
          if (!args.sz_tma) {   // ragged N: this row's zero point and scale from global
            const int64_t g = kb >> 1;
            if (n < N && AWQ_IN_BOUNDS(g < args.K / kGroup)) {
              z = args.zeros[g * N + n];
              sv = args.scales[g * N + n];
            }
          }
          // the group's two 64-k blocks: one stage (kBlk = 2) or the two stages s and s1. A
          // stage is free once the MMAs that read it have completed; its X blocks are not
          // needed here, so building overlaps their loads
          const int s1 = L::kBlk == 2 ? s : (s + 1 == S ? 0 : s + 1);
          const uint32_t ph1 = L::kBlk == 2 ? ph : (s + 1 == S ? (ph ^ 1u) : ph);
          bool got = mbar_wait(&empty[s], ph ^ 1);
          if (L::kBlk == 1) got = got && mbar_wait(&empty[s1], ph1 ^ 1);
          if (got) got = mbar_wait(&pfull[ps], pph);
          ok = __all_sync(0xffffffffu, got);   // keep the warp converged for .aligned ops
          if (!ok) break;
          const int gi = (i >> 1) % L::kPG;          // group inside the slot
          if (!AWQ_IN_BOUNDS(ps < P && s < S && s1 < S && kb + 2 <= 2 * (args.K / kGroup))) {
            ok = false;
            break;
          }
          if (args.sz_tma) {   // rows past N were filled with zeros by the TMA unit
            const uint8_t* sz = smem + L::kSZOff + ps * L::kSZBytes;
            sv = reinterpret_cast<const __half*>(sz)[gi * kTcBM + r];
            z = sz[L::kPG * kTcBM * 2 + gi * kTcBM + r];
          }
          const __half2 lo = u32_as_h2((0x6400u | z) * 0x00010001u);
          const __half2 hi = u32_as_h2((0xD400u | (z << 4)) * 0x00010001u);
          const float scf = __half2float(sv);
          // the scale pair, and the bias pair 1024 + z (fp16) or 128 + z (bf16)
          const uint32_t sc = kBf16 ? float2_to_act2<true>(scf, scf) : h2_as_u32(__half2half2(sv));
          const uint32_t bias = kBf16 ? (0x4300u | z) * 0x00010001u : h2_as_u32(lo);
          const uint8_t* prow = smem + L::kPOff + ps * L::kPBytes + r * L::kPRowBytes;
          // this group's inv_s in the slot (k relative to the group), or NULL
          const float* inv_g =
              args.inv_s == nullptr
                  ? nullptr
                  : reinterpret_cast<const float*>(smem + L::kIOff + ps * L::kInvBytes) +
                        gi * kGroup;
#pragma unroll
          for (int e = 0; e < 2; ++e) {             // stage i + e of the group
            // block e: the second half of stage s (kBlk = 2), or stage s1
            uint8_t* atile = L::kBlk == 2 ? smem + L::kAOff + s * L::kABytes + e * L::kABlockBytes
                                          : smem + L::kAOff + (e ? s1 : s) * L::kABytes;
            if (kA == ASrc::kPacked4) {
              // row r of group gi: 64 bytes, this stage's 32 k at byte 32 * e + 16 * h
              const uint4 pw = *reinterpret_cast<const uint4*>(prow + gi * 64 + 32 * e + 16 * h);
              const uint32_t words[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int k0 = e * kTcBK + 32 * h + 8 * q;   // k inside the group
                const uint4 c4 = pair_scales<kBf16>(scf, sc, inv_g, k0);
                const uint4 o = kBf16 ? dequant_word_scaled_bf16(words[q], bias, c4)
                                      : dequant_word_scaled(words[q], lo, hi, c4);
                *reinterpret_cast<uint4*>(atile + sw128_offset(r, 4 * h + q)) = o;
              }
            } else {
              const uint32_t* pw =
                  reinterpret_cast<const uint32_t*>(prow + gi * 48 + 12 * (2 * e + h));
              const uint32_t w0 = pw[0], w1 = pw[1], w2 = pw[2];
              uint4 o, c4;
#define AWQ_DQ3_CHUNK(I)                                                                    \
  c4 = pair_scales<kBf16>(scf, sc, inv_g, e * kTcBK + 32 * h + 8 * (I));                  \
  o.x = dequant3_pair<I, 0, kBf16>(w0, w1, w2, bias, c4.x);                                \
  o.y = dequant3_pair<I, 1, kBf16>(w0, w1, w2, bias, c4.y);                                \
  o.z = dequant3_pair<I, 2, kBf16>(w0, w1, w2, bias, c4.z);                                \
  o.w = dequant3_pair<I, 3, kBf16>(w0, w1, w2, bias, c4.w);                                \
  *reinterpret_cast<uint4*>(atile + sw128_offset(r, 4 * h + I)) = o;
              AWQ_DQ3_CHUNK(0)
              AWQ_DQ3_CHUNK(1)
              AWQ_DQ3_CHUNK(2)
              AWQ_DQ3_CHUNK(3)
#undef AWQ_DQ3_CHUNK
            }
          }
          if (i % (2 * L::kPG) == 2 * L::kPG - 2 || i == tu.nkb - 2) {   // slot consumed
            mbar_arrive(&pempty[ps]);
            if (++ps == P) { ps = 0; pph ^= 1; }
          }
          fence_proxy_async_smem();
          mbar_arrive(&built[s]);
          if (L::kBlk == 1) mbar_arrive(&built[s1]);
          s = s1 + 1 == S ? 0 : s1 + 1;
          ph = s1 + 1 == S ? (ph1 ^ 1u) : ph1;
        }
      }
    }
  } else if (warp >= kTcEpiWarp0) {
    // ------------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quarter (w % 4), the only one it may access: 32 weight rows of
    // the finished accumulator, all BN token columns.
    const int wq = warp & 3;
    const int row = 32 * wq + lane;
    int64_t lt = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x, ++lt) {
      const TcUnit t = unit_of(u, args);
      const int buf = static_cast<int>(lt % L::kAccBufs);
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf],
                                             static_cast<uint32_t>((lt / L::kAccBufs) & 1)));
      if (!ok) break;
      tc_fence_after();
      const int64_t m0 = static_cast<int64_t>(t.m_tile) * BN;
      const int64_t arow = static_cast<int64_t>(t.row_tile) * kTcBM + row;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * wq) << 16) +
                             static_cast<uint32_t>(buf * L::kAParts * BN);
      const bool unit_ok =
          AWQ_IN_BOUNDS(t.row_tile < args.row_tiles && t.m_tile < args.m_tiles &&
                        t.ksplit < args.k_splits &&
                        (buf + 1) * L::kAParts * BN <= static_cast<int>(L::kTmemCols));
      double sumsq = 0.0;
#pragma unroll 1
      for (int col = 0; col < BN; col += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + col, v);
        tmem_ld_wait();
        if (kEpi == Epi::kStoreY) {
          if (arow < args.N && unit_ok) {
            if (args.k_splits == 1) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int64_t m = m0 + col + j;
                if (m < args.M)
                  static_cast<act_t<kBf16>*>(args.Y)[m * args.N + arow] =
                      float_to_act<kBf16>(__uint_as_float(v[j]));
              }
            } else {
              float* P = args.partial + static_cast<int64_t>(t.ksplit) * args.M * args.N;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int64_t m = m0 + col + j;
                if (m < args.M) P[m * args.N + arow] = __uint_as_float(v[j]);
              }
            }
          }
        } else if (kEpi == Epi::kStoreF32) {
          // Slices of the contraction (k_splits) of one output tile are the consecutive units of
          // one CTA (the grid is one CTA per tile), so slice s > 0 adds itself to the sum of
          // slices 0..s-1 with one rounded fp32 add, in order: short accumulation chains in
          // TMEM, a fixed summation order, no race.
          if (arow < args.rows_total && unit_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int64_t m = m0 + col + j;
              if (m < args.M) {
                float* gp = args.G + arow * args.M + m;
                *gp = t.ksplit == 0 ? __uint_as_float(v[j]) : __fadd_rn(*gp, __uint_as_float(v[j]));
              }
            }
          }
        } else if (kEpi == Epi::kGramDot) {
          // sum_j (D_0 + 2^-12 D_1)[n][j] * (hi + 2^-12 lo)[n][j] over the tile's 16 columns
          uint32_t vl[16];
          tmem_ld_32x32b_x16(taddr + BN + col, vl);
          tmem_ld_wait();
          if (arow < args.rows_total && unit_ok) {
            const __half* er = args.E2 + arow * 2 * args.K + m0 + col;
            const uint4* eh = reinterpret_cast<const uint4*>(er);
            const uint4* el = reinterpret_cast<const uint4*>(er + args.K);
            const uint4 h4[2] = {eh[0], eh[1]}, l4[2] = {el[0], el[1]};
            const uint32_t hw[8] = {h4[0].x, h4[0].y, h4[0].z, h4[0].w, h4[1].x, h4[1].y, h4[1].z, h4[1].w};
            const uint32_t lw[8] = {l4[0].x, l4[0].y, l4[0].z, l4[0].w, l4[1].x, l4[1].y, l4[1].z, l4[1].w};
            float part = 0.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 hf = __half22float2(u32_as_h2(hw[q])), lf = __half22float2(u32_as_h2(lw[q]));
              const float e0 = fmaf(lf.x, 0x1p-12f, hf.x), e1 = fmaf(lf.y, 0x1p-12f, hf.y);
              const float d0 = fmaf(__uint_as_float(vl[2 * q]), 0x1p-12f, __uint_as_float(v[2 * q]));
              const float d1 = fmaf(__uint_as_float(vl[2 * q + 1]), 0x1p-12f, __uint_as_float(v[2 * q + 1]));
              part = fmaf(d0, e0, part);
              part = fmaf(d1, e1, part);
            }
            sumsq += static_cast<double>(part);
          }
        } else if (kEpi == Epi::kSiluMul) {
          // h = silu(g) * u = g * u / (1 + exp(-g)), g and u the gate and up accumulators
          uint32_t vu[16];
          tmem_ld_32x32b_x16(taddr + BN + col, vu);
          tmem_ld_wait();
          if (arow < args.N && unit_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int64_t m = m0 + col + j;
              const float g = __uint_as_float(v[j]);
              const float h = __fdiv_rn(g * __uint_as_float(vu[j]), 1.0f + expf(-g));
              if (m < args.M) static_cast<__half*>(args.Y)[m * args.N + arow] = __float2half_rn(h);
            }
          }
        } else {
          // D = D_hi + 2^-12 D_lo, the error operand's two parts recombined in fp32
          uint32_t vl[16];
          tmem_ld_32x32b_x16(taddr + BN + col, vl);
          tmem_ld_wait();
          float part = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float f = fmaf(__uint_as_float(vl[j]), 0x1p-12f, __uint_as_float(v[j]));
            part = fmaf(f, f, part);
          }
          sumsq += static_cast<double>(part);
        }
      }
      if ((kEpi == Epi::kRowSumSq || kEpi == Epi::kGramDot) && unit_ok &&
          AWQ_IN_BOUNDS(arow < args.rows_total))
        args.row_part[static_cast<int64_t>(t.m_tile) * args.rows_total + arow] = sumsq;
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);            // the MMA may overwrite this accumulator
    }
  } else if (kPacked && warp == kTcPackWarp) {
    // ------------------------------------------------------------------ packed producer
    if (lane == 0) {
      int ps = 0;        // packed slot and phase, continuous across units
      uint32_t pph = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const TcUnit t = unit_of(u, args);
        const int32_t row0 = t.row_tile * kTcBM;
        // a last slot that runs past the unit's K slice loads groups it does not use (zero
        // filled past K); the transaction count is always the full box
        for (int i = 0; i < t.nkb; i += 2 * L::kPG) {
          const int g = (t.kb0 + i) >> 1;
          if (!mbar_wait(&pempty[ps], pph ^ 1)) {
            ok = false;
            break;
          }
          // inv_s of the slot's groups that lie inside K (a bulk copy stops at the array's end)
          const int64_t G = args.K / kGroup;
          const uint32_t inv_bytes =
              args.inv_s == nullptr ? 0u
                                    : static_cast<uint32_t>((G - g < L::kPG ? G - g : L::kPG) *
                                                            kGroup * 4);
          mbar_arrive_expect_tx(&pfull[ps],
                                L::kPBytes + (args.sz_tma ? L::kSZBytes : 0) + inv_bytes);
          tma_load_2d(smem + L::kPOff + ps * L::kPBytes, &tmap_a, &pfull[ps],
                      g * (L::kPGroupBytes / 4), row0);
          if (inv_bytes != 0 && AWQ_IN_BOUNDS(g < G && inv_bytes <= L::kInvBytes))
            bulk_load_1d(smem + L::kIOff + ps * L::kInvBytes, args.inv_s + g * kGroup, inv_bytes,
                         &pfull[ps]);
          if (args.sz_tma) {
            uint8_t* sz = smem + L::kSZOff + ps * L::kSZBytes;
            tma_load_2d(sz, &tmap_s, &pfull[ps], row0, g);
            tma_load_2d(sz + L::kPG * kTcBM * 2, &tmap_z, &pfull[ps], row0, g);
          }
          if (++ps == P) { ps = 0; pph ^= 1; }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// Y[m, n] = fp16 (bf16) of the sum over the K slices of the fp32 partial sums, slices added
// in order.
template <bool kBf16 = false>
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int k_splits,
                                     int64_t MN, act_t<kBf16>* __restrict__ Y) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= MN) return;
  if ((MN & 3) == 0) {   // every slice's start is 16-byte aligned
    float4 acc = *reinterpret_cast<const float4*>(partial + i);
    for (int s = 1; s < k_splits; ++s) {
      if (!AWQ_IN_BOUNDS(i + 4 <= MN)) break;
      const float4 v = *reinterpret_cast<const float4*>(partial + static_cast<int64_t>(s) * MN + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<uint32_t*>(Y + i) = float2_to_act2<kBf16>(acc.x, acc.y);
    *reinterpret_cast<uint32_t*>(Y + i + 2) = float2_to_act2<kBf16>(acc.z, acc.w);
  } else {   // this thread's four outputs, one at a time
    const int64_t end = i + 4 < MN ? i + 4 : MN;
    for (int64_t e = i; e < end; ++e) {
      float acc = partial[e];
      for (int s = 1; s < k_splits; ++s) acc += partial[static_cast<int64_t>(s) * MN + e];
      Y[e] = float_to_act<kBf16>(acc);
    }
  }
}

}  // namespace awq
