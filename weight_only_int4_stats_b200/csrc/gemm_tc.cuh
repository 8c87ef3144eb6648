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
// BN tokens. One CTA computes one 128 x BN tile with a 4-stage shared-memory ring of
// 64-wide K slices:
//   warp 0      TMA producer: X slice (128-byte swizzle) and the A source slice;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (kind::f16, fp32 acc);
//   warps 2..5  A builders (packed source only): 16-byte packed chunks from shared memory
//               -> fp16 (q - z) * scale in registers -> the canonical 128-byte swizzled
//               K-major layout, then fence.proxy.async so the tensor core sees the writes;
//               afterwards the same four warps run the epilogue (tcgen05.ld of their
//               32-lane quarter of TMEM).
// Epilogues: fp16 store of Y[m, n], or (search) each weight row's sum over the tile's
// tokens of the squared output, written as one fp64 partial per (row, token tile).
// Every mbarrier wait is bounded; a timeout sets the device status word and the roles
// leave their loops so the CTA still releases its TMEM and exits.
#pragma once
#include "common.cuh"

namespace awq {

constexpr int kTcBM = 128;      // weight rows per tile (MMA M)
constexpr int kTcBK = 64;       // K per stage: one 128-byte swizzle atom of fp16
constexpr int kTcStages = 4;
constexpr int kTcThreads = 192; // 6 warps

enum class ASrc : int { kPacked4 = 0, kFp16 = 1 };
enum class Epi : int { kStoreY = 0, kRowSumSq = 1 };

template <int BN, ASrc kA>
struct TcLayout {
  static constexpr int kXBytes = BN * kTcBK * 2;
  static constexpr int kABytes = kTcBM * kTcBK * 2;
  static constexpr int kPBytes = (kA == ASrc::kPacked4) ? kTcBM * kTcBK / 2 : 0;
  static constexpr int kXOff = 0;
  static constexpr int kAOff = kXOff + kTcStages * kXBytes;
  static constexpr int kPOff = kAOff + kTcStages * kABytes;
  static constexpr int kBarOff = kPOff + kTcStages * kPBytes;
  // full[S], empty[S], built[S], acc_full, tmem slot
  static constexpr int kBytes = kBarOff + (3 * kTcStages + 1) * 8 + 16;
  static constexpr int kSmem = kBytes + 1024;   // slack for 1024-byte alignment
  static constexpr uint32_t kTxBytes = kXBytes + (kA == ASrc::kFp16 ? kABytes : kPBytes);
  static constexpr uint32_t kTmemCols = BN;     // fp32 accumulator columns (power of 2)
};

struct TcArgs {
  int64_t M;            // tokens
  int64_t N;            // valid weight rows (store epilogue) / rows per grid point (search)
  int64_t N_pad;        // rows per grid point including padding (search); N for the GEMM
  int64_t K;
  const __half* scales; // [K/128, N] (packed source)
  const uint8_t* zeros; // [K/128, N]
  __half* Y;            // [M, N] (store epilogue)
  double* row_part;     // [rows_total, m_tiles] (search epilogue)
  int m_tiles;
};

// Dequantize one packed word (8 consecutive k) to four fp16 pairs (q - z) * sc.
__device__ __forceinline__ uint4 dequant_word_scaled(uint32_t w, __half2 bias_lo,
                                                     __half2 bias_hi, __half2 sc2) {
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const uint32_t w8 = w >> 8;
  const uint32_t v0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  const uint32_t v1 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  const uint32_t v2 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
  const uint32_t v3 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
  uint4 o;
  o.x = h2_as_u32(__hmul2(__hsub2(u32_as_h2(v0), bias_lo), sc2));
  o.y = h2_as_u32(__hmul2(__hfma2(u32_as_h2(v1), sixteenth, bias_hi), sc2));
  o.z = h2_as_u32(__hmul2(__hsub2(u32_as_h2(v2), bias_lo), sc2));
  o.w = h2_as_u32(__hmul2(__hfma2(u32_as_h2(v3), sixteenth, bias_hi), sc2));
  return o;
}

// Byte offset of 16-byte chunk c (k = 8c..8c+7) of row r in a 64-wide fp16 tile stored in
// the 128-byte swizzled K-major layout (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

template <int BN, ASrc kA, Epi kEpi>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ CUtensorMap tmap_a, const TcArgs args) {
  using L = TcLayout<BN, kA>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kTcStages;
  uint64_t* built = empty + kTcStages;
  uint64_t* acc_full = built + kTcStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int row_tile = blockIdx.y;
  const int64_t m0 = static_cast<int64_t>(m_tile) * BN;
  const int64_t row0 = static_cast<int64_t>(row_tile) * kTcBM;   // row in the A matrix
  const int nkb = static_cast<int>(args.K / kTcBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&built[s], 128);
    }
    mbar_init(acc_full, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (kb / kTcStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        mbar_arrive_expect_tx(&full[s], L::kTxBytes);
        tma_load_2d(smem + L::kXOff + s * L::kXBytes, &tmap_x, &full[s], kb * kTcBK,
                    static_cast<int32_t>(m0));
        if (kA == ASrc::kFp16)
          tma_load_2d(smem + L::kAOff + s * L::kABytes, &tmap_a, &full[s], kb * kTcBK,
                      static_cast<int32_t>(row0));
        else
          tma_load_2d(smem + L::kPOff + s * L::kPBytes, &tmap_a, &full[s], kb * (kTcBK / 8),
                      static_cast<int32_t>(row0));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = f16_idesc(kTcBM, BN);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (kb / kTcStages) & 1;
        ok = mbar_wait(&full[s], ph);
        if (ok && kA == ASrc::kPacked4) ok = mbar_wait(&built[s], ph);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + L::kAOff + s * L::kABytes);
        const uint32_t x_base = smem_u32(smem + L::kXOff + s * L::kXBytes);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 16; ++kk) {
          tc_mma_f16(tmem_d, sw128_kmajor_desc(a_base + kk * 32), sw128_kmajor_desc(x_base + kk * 32),
                     idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);
    }
  } else {
    // ------------------------------------------------------------------ A builders
    const int t = threadIdx.x - 64;   // 0..127
    bool ok = true;
    if (kA == ASrc::kPacked4) {
      const int64_t N = args.N;
      const int rA = t >> 1, rB = rA + 64;
      const int64_t nA = row0 + rA, nB = row0 + rB;
      __half2 loA, hiA, scA, loB, hiB, scB;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (kb / kTcStages) & 1;
        if ((kb & 1) == 0) {   // new group of 128: this thread's two rows' zero and scale
          const int64_t g = kb >> 1;
          const uint32_t zA = nA < N ? args.zeros[g * N + nA] : 0u;
          const uint32_t zB = nB < N ? args.zeros[g * N + nB] : 0u;
          const __half sA = nA < N ? args.scales[g * N + nA] : __float2half(0.0f);
          const __half sB = nB < N ? args.scales[g * N + nB] : __float2half(0.0f);
          loA = u32_as_h2((0x6400u | zA) * 0x00010001u);
          hiA = __hneg2(u32_as_h2((0x5400u | (zA << 4)) * 0x00010001u));
          loB = u32_as_h2((0x6400u | zB) * 0x00010001u);
          hiB = __hneg2(u32_as_h2((0x5400u | (zB << 4)) * 0x00010001u));
          scA = __half2half2(sA);
          scB = __half2half2(sB);
        }
        ok = mbar_wait(&full[s], ph) && mbar_wait(&empty[s], ph ^ 1);
        ok = __all_sync(0xffffffffu, ok);   // keep the warp converged for .aligned ops
        if (!ok) break;
        const uint8_t* ptile = smem + L::kPOff + s * L::kPBytes;
        uint8_t* atile = smem + L::kAOff + s * L::kABytes;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const int q = t + 128 * pass;          // 16-byte chunk of the packed tile
          const int r = q >> 1, h = q & 1;        // row, which 32-k half of the 64
          const uint4 pw = *reinterpret_cast<const uint4*>(ptile + q * 16);
          const __half2 lo = pass ? loB : loA, hi = pass ? hiB : hiA, sc = pass ? scB : scA;
          const uint32_t words[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 o = dequant_word_scaled(words[i], lo, hi, sc);
            *reinterpret_cast<uint4*>(atile + sw128_offset(r, 4 * h + i)) = o;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&built[s]);
      }
    }
    // ------------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait(acc_full, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int wq = warp & 3;                 // TMEM lane quarter this warp may access
      const int row = 32 * wq + lane;          // row inside the tile
      const int64_t arow = row0 + row;
      double sumsq = 0.0;
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(32 * wq) << 16) + cb * 32, v);
        tmem_ld_wait();
        if (kEpi == Epi::kStoreY) {
          if (arow < args.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int64_t m = m0 + cb * 32 + j;
              if (m < args.M) args.Y[m * args.N + arow] = __float2half_rn(__uint_as_float(v[j]));
            }
          }
        } else {
          float part = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float f = __uint_as_float(v[j]);
            part = fmaf(f, f, part);
          }
          sumsq += static_cast<double>(part);
        }
      }
      if (kEpi == Epi::kRowSumSq)
        args.row_part[arow * args.m_tiles + m_tile] = sumsq;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, L::kTmemCols);
  }
}

}  // namespace awq
