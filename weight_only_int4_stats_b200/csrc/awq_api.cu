// Host side of the C ABI declared in include/awq.h: argument checks, workspace carving,
// TMA descriptor encoding and kernel dispatch. All kernels live in the *.cuh files of this
// directory and are compiled into this one translation unit for sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "awq.h"
#include "act_stats.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "quantize.cuh"
#include "search.cuh"

namespace {

using awq::ASrc;
using awq::Epi;

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;
constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }
size_t align256(size_t v) { return (v + 255) & ~size_t{255}; }

awq_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// Per-device caches below are atomics: host threads may call the library concurrently, and
// a value computed twice is the same value, so a racing first call only repeats work.
int num_sms() {
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_acquire);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev].store(v, std::memory_order_release);
  }
  return v;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes per element; box [box_rows, box_cols].
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem,
                  int64_t rows, int64_t cols, int box_rows, int box_cols, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, ASrc kA, Epi kEpi, bool kBf16, int kBlkT>
awq_status launch_tc_blk(const void* Xop, int64_t M, const void* Aop, int64_t a_rows,
                         const awq::TcArgs& args, cudaStream_t st, const void* Aop2) {
  using L = awq::TcLayout<BN, kA, kBlkT>;
  static std::atomic<bool> attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AWQ_ERR_CUDA;
  auto kern = awq::tc_gemm_kernel<BN, kA, kEpi, kBf16, kBlkT>;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem) !=
        cudaSuccess)
      return AWQ_ERR_CUDA;
    attr_set[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tx, ta;
  // B operand rows M x (K, or 2K for the two-part normalised Gram matrix) columns
  if (!make_tmap_2d(&tx, Xop, kBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    2, M, kA == ASrc::kGram ? 2 * args.K : args.K, BN, awq::kTcBK, true))
    return AWQ_ERR_CUDA;
  if (kA == ASrc::kSplit16 || kA == ASrc::kGram) {   // [a_rows, 2K]: hi part, then lo part
    if (!make_tmap_2d(&ta, Aop, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a_rows, 2 * args.K,
                      awq::kTcBM, awq::kTcBK, true))
      return AWQ_ERR_CUDA;
  } else if (kA == ASrc::kPair16 || kA == ASrc::kFp16x1) {   // [a_rows, K] fp16 (kPair16:
                                                                  // the second map goes in ts)
    if (!make_tmap_2d(&ta, Aop, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a_rows, args.K, awq::kTcBM,
                      awq::kTcBK, true))
      return AWQ_ERR_CUDA;
  } else if (kA == ASrc::kPacked4) {   // kPG groups of 16 words (64 bytes) per row per load
    if (!make_tmap_2d(&ta, Aop, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a_rows, args.K / 8,
                      awq::kTcBM, L::kPRowBytes / 4, false))
      return AWQ_ERR_CUDA;
  } else {   // 3-bit: kPG groups of 12 words (48 bytes) per row per load
    if (!make_tmap_2d(&ta, Aop, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a_rows, 3 * args.K / 32,
                      awq::kTcBM, L::kPRowBytes / 4, false))
      return AWQ_ERR_CUDA;
  }
  // scales [G, N] fp16 and zeros [G, N] u8 as TMA tiles of kPG groups x 128 rows, when the
  // row stride of the zeros (N bytes) meets the 16-byte rule; otherwise the maps go unused
  CUtensorMap ts = ta, tz = ta;
  awq::TcArgs a = args;
  a.sz_tma = 0;
  if (kA == ASrc::kPair16 &&
      !make_tmap_2d(&ts, Aop2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a_rows, args.K, awq::kTcBM,
                    awq::kTcBK, true))
    return AWQ_ERR_CUDA;
  if ((kA == ASrc::kPacked4 || kA == ASrc::kPacked3) && args.N % 16 == 0) {
    const int64_t G = args.K / awq::kGroup;
    if (!make_tmap_2d(&ts, args.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, G, args.N, L::kPG,
                      awq::kTcBM, false) ||
        !make_tmap_2d(&tz, args.zeros, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, G, args.N, L::kPG,
                      awq::kTcBM, false))
      return AWQ_ERR_CUDA;
    a.sz_tma = 1;
  }
  a.m_tiles = static_cast<int>((M + BN - 1) / BN);
  a.row_tiles = static_cast<int>((a_rows + awq::kTcBM - 1) / awq::kTcBM);
  a.rows_total = a_rows;
  if (a.k_splits < 1) a.k_splits = 1;
  const int64_t units = static_cast<int64_t>(a.m_tiles) * a.row_tiles * a.k_splits;
  const int64_t sms = num_sms();
  // persistent, one CTA per SM; the fp32-store epilogue instead takes one CTA per output tile,
  // so that a tile's contraction slices are consecutive units of the same CTA
  const int64_t want = kEpi == Epi::kStoreF32 ? units / a.k_splits : sms;
  const unsigned grid = static_cast<unsigned>(units < want ? units : want);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(awq::kTcThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(L::kSmem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tx, ta, ts, tz, a) != cudaSuccess) return AWQ_ERR_CUDA;
  return launch_status();
}

// Packed sources take stages of two 64-k blocks where the builders or the single MMA-issuing
// thread set the pace: token tiles up to 128, and inv_s folded into the weights. Plain
// BN = 256 keeps four one-block stages (two two-block stages, all that fit, measured slower
// there: 1294 -> 1172 TFLOP/s on [28672, 8192] at M = 4096).
template <int BN, ASrc kA, Epi kEpi, bool kBf16 = false>
awq_status launch_tc(const void* Xop, int64_t M, const void* Aop, int64_t a_rows,
                     const awq::TcArgs& args, cudaStream_t st, const void* Aop2 = nullptr) {
  constexpr bool kPk = kA == ASrc::kPacked4 || kA == ASrc::kPacked3;
  if constexpr (kPk && BN == 256) {
    if (args.inv_s == nullptr)
      return launch_tc_blk<BN, kA, kEpi, kBf16, 1>(Xop, M, Aop, a_rows, args, st, Aop2);
    return launch_tc_blk<BN, kA, kEpi, kBf16, 2>(Xop, M, Aop, a_rows, args, st, Aop2);
  } else {
    return launch_tc_blk<BN, kA, kEpi, kBf16, kPk ? 2 : 1>(Xop, M, Aop, a_rows, args, st, Aop2);
  }
}

template <ASrc kA, Epi kEpi, bool kBf16 = false>
awq_status launch_tc_bn(const void* Xop, int64_t M, const void* Aop, int64_t a_rows,
                        const awq::TcArgs& args, cudaStream_t st, const void* Aop2 = nullptr) {
  if (M <= 32) return launch_tc<32, kA, kEpi, kBf16>(Xop, M, Aop, a_rows, args, st, Aop2);
  if (M <= 64) return launch_tc<64, kA, kEpi, kBf16>(Xop, M, Aop, a_rows, args, st, Aop2);
  if (M <= 128) return launch_tc<128, kA, kEpi, kBf16>(Xop, M, Aop, a_rows, args, st, Aop2);
  return launch_tc<256, kA, kEpi, kBf16>(Xop, M, Aop, a_rows, args, st, Aop2);
}

// Streaming decode GEMM (M <= 16), launched with programmatic dependent launch.
constexpr int kSmemLimit = 232448;   // 227 KB per CTA on sm_100
static_assert(awq::kGemvWeightsReady == AWQ_GEMM_WEIGHTS_READY, "flag values must agree");
static_assert((AWQ_GEMM_WEIGHTS_READY & AWQ_GEMM_BF16) == 0, "flags are distinct bits");

// Two CTAs of the streaming kernel fit on one SM when each takes at most half of its 228 KB
// (less 1 KB reserved per CTA): the next launch's CTAs then start beside this one's.
constexpr int kCoResidentSmem = (233472 - 2 * 1024) / 2;

// The streaming kernel's shared-memory plan for a shape: the deepest ring (6 down to 2 slots)
// that leaves room for a co-resident CTA, else the deepest that fits one CTA.
bool gemv_config(int64_t M, int64_t N, int64_t K, awq::G4Smem* out) {
  if (M < 1 || M > 16 || N % 16 != 0 || K / awq::kGroup > 65535) return false;
  const int nt = M <= 8 ? 1 : 2;
  for (int budget : {kCoResidentSmem, kSmemLimit})
    for (int slots = awq::kGSMaxSlots; slots >= 2; --slots) {
      const awq::G4Smem l = awq::G4Smem::make(static_cast<int>(M), K, nt, slots);
      if (l.total(nt) <= budget) {
        *out = l;
        return true;
      }
    }
  return false;
}

// Whether the streaming decode kernel takes this shape: N in whole 16-row tiles and X (plus the
// small sums, the reduction buffer and a two-slot ring) within one CTA's shared memory.
bool gemv_stream_fits(int64_t M, int64_t N, int64_t K) {
  awq::G4Smem l;
  return gemv_config(M, N, K, &l);
}

template <int kNTiles, bool kOffset, bool kBf16, int kBits>
awq_status launch_gemv_stream_t(const void* x, int64_t M, const uint32_t* qweight,
                                const __half* scales, const uint8_t* zeros, int64_t N, int64_t K,
                                const float* inv_s, unsigned flags, void* y, cudaStream_t st) {
  using A = awq::act_t<kBf16>;
  static std::atomic<bool> attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AWQ_ERR_CUDA;
  auto kern = awq::gemv_stream_kernel<kNTiles, kOffset, kBf16, kBits>;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
        cudaSuccess)
      return AWQ_ERR_CUDA;
    attr_set[dev].store(true, std::memory_order_release);
  }
  awq::G4Smem lay;
  if (!gemv_config(M, N, K, &lay)) return AWQ_ERR_UNSUPPORTED;
  // packed codes [N, K * bits / 32] words in boxes of 16 rows x 32 words (128 B, swizzled);
  // scales [G, N] fp16 and zero points [G, N] uint8 in boxes of 16 groups x 16 rows
  CUtensorMap tw, ts, tz;
  if (!make_tmap_2d(&tw, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, N, K * kBits / 32,
                    awq::kGemvRows, 32, true) ||
      !make_tmap_2d(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K / awq::kGroup, N,
                    awq::kG4Groups, awq::kGemvRows, false) ||
      !make_tmap_2d(&tz, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / awq::kGroup, N,
                    awq::kG4Groups, awq::kGemvRows, false))
    return AWQ_ERR_CUDA;
  const int64_t tiles = N / awq::kGemvRows;
  // Two CTAs per SM (each its own tile range and ring) when both fit, for M <= 8: a CTA's
  // per-unit chain is latency-bound and a second CTA runs a second chain (measured 21.5
  // against 23.3 us on the three decode shapes at M = 1). At M <= 16 (two token tiles) one
  // CTA per SM keeps the ring and X of the larger tiles (two were slower there).
  const int per_sm = kNTiles == 1 && lay.total(kNTiles) <= kCoResidentSmem ? 2 : 1;
  const int64_t ctas = static_cast<int64_t>(num_sms()) * per_sm;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < ctas ? tiles : ctas));
  cfg.blockDim = dim3(awq::kG4Threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(lay.total(kNTiles));
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tw, ts, tz, static_cast<const A*>(x),
                         static_cast<int>(M), N, K, inv_s, static_cast<A*>(y), lay,
                         flags) != cudaSuccess)
    return AWQ_ERR_CUDA;
  return launch_status();
}

template <bool kBf16, int kBits>
awq_status launch_gemv_stream_m(const void* x, int64_t M, const uint32_t* qweight,
                                const __half* scales, const uint8_t* zeros, int64_t N, int64_t K,
                                const float* inv_s, unsigned flags, void* y, cudaStream_t st) {
  if (M == 1)
    return launch_gemv_stream_t<1, true, kBf16, kBits>(x, M, qweight, scales, zeros, N, K, inv_s,
                                                       flags, y, st);
  if (M <= 8)
    return launch_gemv_stream_t<1, false, kBf16, kBits>(x, M, qweight, scales, zeros, N, K,
                                                        inv_s, flags, y, st);
  return launch_gemv_stream_t<2, false, kBf16, kBits>(x, M, qweight, scales, zeros, N, K, inv_s,
                                                      flags, y, st);
}

// Returns AWQ_ERR_UNSUPPORTED when the shape does not suit the streaming kernel; the caller
// then uses the register-streaming kernel (fp16, 4-bit, M <= 8) or the tensor-core path.
awq_status launch_gemv_stream(const void* x, int64_t M, const uint32_t* qweight,
                              const __half* scales, const uint8_t* zeros, int64_t N, int64_t K,
                              int bits, const float* inv_s, unsigned flags, void* y,
                              cudaStream_t st) {
  if (!gemv_stream_fits(M, N, K)) return AWQ_ERR_UNSUPPORTED;
  const bool bf16 = (flags & AWQ_GEMM_BF16) != 0;
  if (bits == 3)
    return bf16 ? launch_gemv_stream_m<true, 3>(x, M, qweight, scales, zeros, N, K, inv_s, flags,
                                                y, st)
                : launch_gemv_stream_m<false, 3>(x, M, qweight, scales, zeros, N, K, inv_s, flags,
                                                 y, st);
  return bf16 ? launch_gemv_stream_m<true, 4>(x, M, qweight, scales, zeros, N, K, inv_s, flags, y,
                                              st)
              : launch_gemv_stream_m<false, 4>(x, M, qweight, scales, zeros, N, K, inv_s, flags,
                                               y, st);
}

int tc_bn_for(int64_t M) { return M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

// Split-K for the tensor-core GEMM when the output has too few 128 x BN tiles to occupy the
// GPU (batched decode, small prefill). The persistent kernel runs one CTA per SM and hands
// out (tile, K slice) units round-robin, so the busiest SM does ceil(tiles * s / sms) units
// of K / s each: pick the split s that minimises that, i.e. ceil(tiles * s / sms) / s, with
// at least two 128-wide groups per slice and the partial traffic within about the packed
// weight bytes. A later s must win by more than 12% per extra slice: each slice adds a
// pipeline fill, an epilogue and 8 bytes of fp32 partial sums per output to reduce. On the
// batched shapes 12% measured best among 2, 6, 12, 40 and 60% (e.g. [14336, 4096] at M = 32
// runs unsplit, 26.6 -> 24.3 us; [4096, 14336] takes 4 slices instead of 9).
int splitk_for(int64_t M, int64_t N, int64_t K) {
  const int64_t bn = tc_bn_for(M);
  const int64_t tiles = ((N + awq::kTcBM - 1) / awq::kTcBM) * ((M + bn - 1) / bn);
  const int64_t sms = num_sms();
  if (tiles >= sms) return 1;
  int64_t s_max = (K / awq::kGroup) / 2;
  const int64_t by_traffic = K / (8 * M);
  if (s_max > by_traffic) s_max = by_traffic;
  if (s_max > 16) s_max = 16;
  int best = 1;
  double best_cost = 1.0;
  for (int64_t s = 2; s <= s_max; ++s) {
    const double cost =
        static_cast<double>((tiles * s + sms - 1) / sms) / static_cast<double>(s);
    if (cost * (1.0 + 0.12 * static_cast<double>(s - best)) < best_cost) {
      best = static_cast<int>(s);
      best_cost = cost;
    }
  }
  return best;
}

bool bad_dim(int64_t v) { return v < 0 || v > kMaxDim; }

}  // namespace

extern "C" {

const char* awq_status_string(awq_status status) {
  switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED";
    case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA";
    case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT";
    case AWQ_ERR_BOUNDS: return "AWQ_ERR_BOUNDS";
  }
  return "AWQ_ERR_UNKNOWN";
}

int awq_abi_version(void) { return 2; }

awq_status awq_check_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return AWQ_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, awq::g_status_word, sizeof(word)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(awq::g_status_word, &zero, sizeof(zero)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (word & awq::kDevErrBounds) return AWQ_ERR_BOUNDS;
  if (word & awq::kDevErrTimeout) return AWQ_ERR_TIMEOUT;
  return AWQ_OK;
}

awq_status awq_selftest_bounds(int* buf, void* stream) {
#ifdef AWQ_DEBUG_BOUNDS
  if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0) return AWQ_ERR_INVALID_ARG;
  awq::bounds_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(buf, 4);
  return launch_status();
#else
  (void)buf;
  (void)stream;
  return AWQ_ERR_UNSUPPORTED;   // the release build has no bounds checks
#endif
}

awq_status awq_trace_reset(void) {
#ifdef AWQ_TRACE
  static_assert(awq::kTraceWords == AWQ_TRACE_WORDS, "trace record size");
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(awq::g_trace_ctas, &zero, sizeof(zero)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  return AWQ_OK;
#else
  return AWQ_ERR_UNSUPPORTED;   // only the trace build records a timeline
#endif
}

awq_status awq_trace_read(unsigned long long* out, int64_t max_ctas, int64_t* n_ctas) {
#ifdef AWQ_TRACE
  if (out == nullptr || n_ctas == nullptr || max_ctas < 0) return AWQ_ERR_INVALID_ARG;
  unsigned count = 0;
  if (cudaMemcpyFromSymbol(&count, awq::g_trace_ctas, sizeof(count)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  int64_t n = count < static_cast<unsigned>(awq::kTraceCtas) ? count : awq::kTraceCtas;
  if (n > max_ctas) n = max_ctas;
  if (n > 0 &&
      cudaMemcpyFromSymbol(out, awq::g_trace,
                           static_cast<size_t>(n) * awq::kTraceWords * sizeof(unsigned long long)) !=
          cudaSuccess)
    return AWQ_ERR_CUDA;
  *n_ctas = count;
  return AWQ_OK;
#else
  (void)out;
  (void)max_ctas;
  (void)n_ctas;
  return AWQ_ERR_UNSUPPORTED;
#endif
}

awq_status awq_selftest_timeout(int* waited_out, void* stream) {
  if (waited_out == nullptr || (reinterpret_cast<uintptr_t>(waited_out) & 3u) != 0)
    return AWQ_ERR_INVALID_ARG;
  awq::timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      50ull * 1000 * 1000, waited_out);
  return launch_status();
}

// ------------------------------------------------------------------ act_stats
size_t awq_act_stats_workspace_size(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  const int splits = awq::act_stats_splits(M, K, num_sms());
  return static_cast<size_t>(splits) * static_cast<size_t>(K) * sizeof(double);
}

awq_status awq_act_stats(const awq_f16* X, int64_t M, int64_t K, float* s_x, void* workspace,
                         size_t ws_bytes, void* stream) {
  if (bad_dim(M) || bad_dim(K) || M == 0) return AWQ_ERR_INVALID_ARG;
  if (K == 0) return AWQ_OK;
  if (K % 8 != 0) return AWQ_ERR_INVALID_ARG;
  if (!X || !s_x || !aligned16(X) || !aligned16(s_x)) return AWQ_ERR_INVALID_ARG;
  const int splits = awq::act_stats_splits(M, K, num_sms());
  const size_t need = static_cast<size_t>(splits) * static_cast<size_t>(K) * sizeof(double);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return AWQ_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(workspace);
  const int64_t rows_per_split = (M + splits - 1) / splits;
  dim3 g1(static_cast<unsigned>((K + awq::kStatsCols - 1) / awq::kStatsCols),
          static_cast<unsigned>(splits));
  awq::act_stats_partial_kernel<<<g1, 256, 0, st>>>(reinterpret_cast<const __half*>(X), M, K,
                                                   rows_per_split, part);
  awq_status s = launch_status();
  if (s != AWQ_OK) return s;
  awq::act_stats_finish_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
      part, splits, M, K, s_x);
  return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------------ act_stats without allocation
// Scratch for awq_act_stats_noalloc: the fp64 partial sums live in this file-scope device
// array instead of a caller workspace. Every GPU that loads the library holds it until the
// process exits. In host code the name is only a stand-in for the symbol, so its device
// address is looked up once per device (with that device current) and cached.
namespace {
constexpr int64_t kNoAllocScratchDoubles = int64_t{1} << 17;   // 1 MiB
constexpr int64_t kNoAllocMaxK = 65536;                       // >= 2 row slices per call
static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchDoubles];

double* g_noalloc_ptr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

awq_status noalloc_scratch(double** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AWQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return AWQ_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<double*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return AWQ_OK;
}
}  // namespace

extern "C" {

awq_status awq_act_stats_noalloc(const awq_f16* X, int64_t M, int64_t K, float* s_x,
                                 void* stream) {
  if (bad_dim(M) || bad_dim(K) || M == 0) return AWQ_ERR_INVALID_ARG;
  if (K == 0) return AWQ_OK;
  if (K % 8 != 0 || K > kNoAllocMaxK) return AWQ_ERR_INVALID_ARG;
  if (!X || !s_x || !aligned16(X) || !aligned16(s_x)) return AWQ_ERR_INVALID_ARG;
  double* part = nullptr;
  awq_status s = noalloc_scratch(&part);
  if (s != AWQ_OK) return s;
  int splits = awq::act_stats_splits(M, K, num_sms());
  const int64_t cap = kNoAllocScratchDoubles / K;
  if (splits > cap) splits = static_cast<int>(cap);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Pass 1 writes every (slice, channel) partial it later reads, so nothing of an earlier
  // call's contents is used and the array needs no clearing.
  const int64_t rows_per_split = (M + splits - 1) / splits;
  dim3 g1(static_cast<unsigned>((K + awq::kStatsCols - 1) / awq::kStatsCols),
          static_cast<unsigned>(splits));
  awq::act_stats_partial_kernel<<<g1, 256, 0, st>>>(reinterpret_cast<const __half*>(X), M, K,
                                                   rows_per_split, part);
  if ((s = launch_status()) != AWQ_OK) return s;
  awq::act_stats_finish_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
      part, splits, M, K, s_x);
  return launch_status();
}

// ------------------------------------------------------------------ quantize_pack
awq_status awq_quantize_pack(const awq_f16* W, int64_t N, int64_t K, const float* s, int bits,
                             int group, uint32_t* qweight, awq_f16* scales, uint8_t* zeros,
                             void* stream) {
  if (bad_dim(N) || bad_dim(K) || K == 0) return AWQ_ERR_INVALID_ARG;
  if (group != awq::kGroup || K % awq::kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (bits != 4 && bits != 3) return AWQ_ERR_INVALID_ARG;
  if (N == 0) return AWQ_OK;
  if (!W || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      (s && !aligned16(s)))
    return AWQ_ERR_INVALID_ARG;
  if ((K / awq::kGroup) > 65535) return AWQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(static_cast<unsigned>((N + awq::kQuantRowsPerCta - 1) / awq::kQuantRowsPerCta),
            static_cast<unsigned>(K / awq::kGroup));
  const __half* w = reinterpret_cast<const __half*>(W);
  __half* sc = reinterpret_cast<__half*>(scales);
  if (bits == 4)
    awq::quantize_pack_kernel<4><<<grid, 256, 0, st>>>(w, N, K, s, qweight, sc, zeros);
  else
    awq::quantize_pack_kernel<3><<<grid, 256, 0, st>>>(w, N, K, s, qweight, sc, zeros);
  return launch_status();
}

// ------------------------------------------------------------------ search
namespace {
// The error operand E is built and reduced for a chunk of grid points at a time, so the
// workspace stays bounded whatever the layer: at most this many bytes of E per chunk (at
// least one grid point per chunk).
constexpr size_t kSearchChunkBytes = size_t{1} << 30;
// Column tile of the Gram-form loss GEMM (its N side is channels).
constexpr int kGramBN = 128;

// The loss is evaluated in its Gram form e G e^T (G = X^T X, N K^2 per grid point plus K^2 M
// once) when that is cheaper than the direct ||E X^T||^2 (N K M per grid point) with margin:
// the Gram MMAs cost 1.5 times the direct ones per product (three instead of two), so when
// M >= 2K.
bool search_uses_gram(int64_t M, int64_t K) { return M >= 2 * K; }

struct SearchWs {
  int chunk;   // grid points per chunk
  bool gram;
  int64_t M_pad;
  size_t table, inv, err, part, rows, xt, g, g2, rms, total;
};
SearchWs search_ws_layout(int64_t M, int64_t N, int64_t K, int n_alpha) {
  const int64_t N_pad = round_up(N, awq::kTcBM);
  SearchWs w;
  w.gram = search_uses_gram(M, K);
  w.M_pad = round_up(M, awq::kGroup);
  const int64_t m_tiles = w.gram ? K / kGramBN : (M + tc_bn_for(M) - 1) / tc_bn_for(M);
  const size_t per_point = static_cast<size_t>(N_pad) * 2 * K * sizeof(__half);   // hi, lo
  int64_t chunk = static_cast<int64_t>(kSearchChunkBytes / per_point);
  if (chunk < 1) chunk = 1;
  if (chunk > n_alpha) chunk = n_alpha;
  w.chunk = static_cast<int>(chunk);
  w.table = 0;
  w.inv = align256(static_cast<size_t>(n_alpha) * K * sizeof(float));
  w.err = w.inv + align256(static_cast<size_t>(n_alpha) * K * sizeof(float));
  w.part = w.err + align256(static_cast<size_t>(chunk) * per_point);
  w.rows = w.part + align256(static_cast<size_t>(chunk) * N_pad * m_tiles * sizeof(double));
  w.xt = w.rows + align256(static_cast<size_t>(n_alpha) * N * sizeof(double));
  size_t end = w.xt;
  if (w.gram) {   // X^T [K, M_pad] fp16, G [K, K] fp32, G' [K, 2K] fp16 parts, rms [K]
    w.g = w.xt + align256(static_cast<size_t>(K) * w.M_pad * sizeof(__half));
    w.g2 = w.g + align256(static_cast<size_t>(K) * K * sizeof(float));
    w.rms = w.g2 + align256(static_cast<size_t>(K) * 2 * K * sizeof(__half));
    end = w.rms + align256(static_cast<size_t>(K) * sizeof(float));
  }
  w.total = end;
  return w;
}
}  // namespace

size_t awq_search_scale_workspace_size(int64_t M, int64_t N, int64_t K, int n_alpha) {
  if (M <= 0 || N <= 0 || K <= 0 || n_alpha <= 0) return 0;
  return search_ws_layout(M, N, K, n_alpha).total;
}

awq_status awq_search_scale(const awq_f16* W, int64_t N, int64_t K, const awq_f16* X,
                            int64_t M, const float* s_x, const float* alphas, int n_alpha,
                            int bits, int group, const float* s_table, double* losses,
                            int32_t* best_idx, float* best_s, float* best_inv_s,
                            double* row_losses, void* workspace, size_t ws_bytes,
                            void* stream) {
  if (bad_dim(N) || bad_dim(K) || bad_dim(M) || N == 0 || K == 0 || M == 0)
    return AWQ_ERR_INVALID_ARG;
  if (group != awq::kGroup || K % awq::kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (bits != 4 && bits != 3) return AWQ_ERR_INVALID_ARG;
  if (n_alpha < 1 || n_alpha > 64) return AWQ_ERR_INVALID_ARG;
  if (!W || !X || !losses || !best_idx || !best_s) return AWQ_ERR_INVALID_ARG;
  if (!s_table && (!s_x || !alphas)) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(X) || !aligned16(losses) || !aligned16(best_idx) ||
      !aligned16(best_s) || (s_x && !aligned16(s_x)) || (alphas && !aligned16(alphas)) ||
      (s_table && !aligned16(s_table)) || (row_losses && !aligned16(row_losses)) ||
      (best_inv_s && !aligned16(best_inv_s)))
    return AWQ_ERR_INVALID_ARG;
  const int64_t N_pad = round_up(N, awq::kTcBM);
  if (N_pad / awq::kTcBM > 65535 || K / awq::kGroup > 65535) return AWQ_ERR_INVALID_ARG;
  const SearchWs lay = search_ws_layout(M, N, K, n_alpha);
  if (static_cast<int64_t>(lay.chunk) * N_pad / awq::kTcBM > 65535) return AWQ_ERR_INVALID_ARG;
  if (lay.gram && (K / 32 > 65535 || lay.M_pad / 32 > 2147483647LL)) return AWQ_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < lay.total || !aligned16(workspace)) return AWQ_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* table = reinterpret_cast<float*>(ws + lay.table);
  __half* E = reinterpret_cast<__half*>(ws + lay.err);
  double* part = reinterpret_cast<double*>(ws + lay.part);
  const __half* x = reinterpret_cast<const __half*>(X);
  awq_status s;

  const float* S = s_table;
  if (S == nullptr) {
    dim3 g(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>(n_alpha));
    awq::scale_candidates_kernel<<<g, 256, 0, st>>>(s_x, alphas, n_alpha, K, table);
    if ((s = launch_status()) != AWQ_OK) return s;
    S = table;
  }
  float* inv = reinterpret_cast<float*>(ws + lay.inv);
  {
    const int64_t total = static_cast<int64_t>(n_alpha) * K;
    awq::inv_table_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(S, total, inv);
    if ((s = launch_status()) != AWQ_OK) return s;
  }
  // Gram form: X^T (tokens contiguous, padded to whole groups), G = X^T X on the tensor
  // cores, the channels' root mean squares, and G normalised to two fp16 parts
  float* rms = nullptr;
  const __half* G2 = nullptr;
  if (lay.gram) {
    __half* XT = reinterpret_cast<__half*>(ws + lay.xt);
    float* G = reinterpret_cast<float*>(ws + lay.g);
    __half* G2w = reinterpret_cast<__half*>(ws + lay.g2);
    rms = reinterpret_cast<float*>(ws + lay.rms);
    dim3 gt(static_cast<unsigned>(lay.M_pad / 32), static_cast<unsigned>((K + 31) / 32));
    awq::transpose_pad_kernel<<<gt, 256, 0, st>>>(x, M, K, lay.M_pad, XT);
    if ((s = launch_status()) != AWQ_OK) return s;
    awq::TcArgs ga{};
    ga.M = K;            // B rows: channels j
    ga.N = K;
    ga.N_pad = K;
    ga.K = lay.M_pad;    // the contraction runs over tokens
    ga.G = G;
    ga.upper_only = 1;   // G is symmetric: the tiles at or above the diagonal suffice
    // the contraction over tokens in slices of about 2048 (128 accumulation steps each)
    ga.k_splits = static_cast<int>(lay.M_pad / 2048 > 1 ? lay.M_pad / 2048 : 1);
    s = launch_tc<256, ASrc::kFp16x1, Epi::kStoreF32>(XT, K, XT, K, ga, st);
    if (s != AWQ_OK) return s;
    awq::gram_rms_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(G, K, M, rms);
    if ((s = launch_status()) != AWQ_OK) return s;
    dim3 gn(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>(K));
    awq::gram_normalize_kernel<<<gn, 256, 0, st>>>(G, K, G2w);
    if ((s = launch_status()) != AWQ_OK) return s;
    G2 = G2w;
  }
  const int bn = lay.gram ? kGramBN : tc_bn_for(M);
  const int m_tiles = lay.gram ? static_cast<int>(K / kGramBN) : static_cast<int>((M + bn - 1) / bn);
  double* rl = row_losses != nullptr ? row_losses : reinterpret_cast<double*>(ws + lay.rows);
  const __half* w = reinterpret_cast<const __half*>(W);
  for (int a0 = 0; a0 < n_alpha; a0 += lay.chunk) {
    const int na = n_alpha - a0 < lay.chunk ? n_alpha - a0 : lay.chunk;
    const float* Sa = S + static_cast<int64_t>(a0) * K;
    const float* Ia = inv + static_cast<int64_t>(a0) * K;
    {
      dim3 g(static_cast<unsigned>(N_pad / awq::kQuantRowsPerCta),
             static_cast<unsigned>(K / awq::kGroup), static_cast<unsigned>(na));
      if (bits == 4)
        awq::search_build_error_kernel<4><<<g, 256, 0, st>>>(w, N, K, N_pad, Sa, Ia, rms, E);
      else
        awq::search_build_error_kernel<3><<<g, 256, 0, st>>>(w, N, K, N_pad, Sa, Ia, rms, E);
      if ((s = launch_status()) != AWQ_OK) return s;
    }
    {
      awq::TcArgs args{};
      args.M = lay.gram ? K : M;
      args.N = N;
      args.N_pad = N_pad;
      args.K = K;
      args.row_part = part;
      args.m_tiles = m_tiles;
      args.k_splits = 1;
      args.E2 = E;
      s = lay.gram ? launch_tc<kGramBN, ASrc::kGram, Epi::kGramDot>(G2, K, E, na * N_pad, args, st)
                   : launch_tc_bn<ASrc::kSplit16, Epi::kRowSumSq>(X, M, E, na * N_pad, args, st);
      if (s != AWQ_OK) return s;
    }
    {
      const int64_t n = static_cast<int64_t>(na) * N;
      awq::search_row_loss_kernel<<<static_cast<unsigned>((n + awq::kReduceThreads - 1) /
                                                          awq::kReduceThreads),
                                    awq::kReduceThreads, 0, st>>>(
          part, N, N_pad, na, m_tiles, lay.gram ? static_cast<double>(M) : 1.0,
          rl + static_cast<int64_t>(a0) * N);
      if ((s = launch_status()) != AWQ_OK) return s;
    }
  }
  awq::search_reduce_kernel<<<n_alpha, awq::kReduceThreads, 0, st>>>(rl, N, losses);
  if ((s = launch_status()) != AWQ_OK) return s;
  awq::search_pick_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
      losses, n_alpha, S, inv, K, best_idx, best_s, best_inv_s);
  return launch_status();
}

// ------------------------------------------------------------------ gated MLP input
awq_status awq_silu_mul_gemm(const awq_f16* X, int64_t M, const awq_f16* W_gate,
                             const awq_f16* W_up, int64_t I, int64_t K, awq_f16* H,
                             void* stream) {
  if (bad_dim(M) || bad_dim(I) || bad_dim(K) || K == 0) return AWQ_ERR_INVALID_ARG;
  if (K % awq::kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (M == 0 || I == 0) return AWQ_OK;
  if (!X || !W_gate || !W_up || !H) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(H))
    return AWQ_ERR_INVALID_ARG;
  if ((I + awq::kTcBM - 1) / awq::kTcBM > 65535) return AWQ_ERR_INVALID_ARG;
  awq::TcArgs args{};
  args.M = M;
  args.N = I;
  args.N_pad = I;
  args.K = K;
  args.Y = reinterpret_cast<__half*>(H);
  args.m_tiles = static_cast<int>((M + tc_bn_for(M) - 1) / tc_bn_for(M));
  args.k_splits = 1;
  return launch_tc_bn<ASrc::kPair16, Epi::kSiluMul>(X, M,
                                                    W_gate, I, args,
                                                    static_cast<cudaStream_t>(stream), W_up);
}

// ------------------------------------------------------------------ GEMM
size_t awq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int bits) {
  if (M <= 0 || K <= 0 || N <= 0) return 0;
  // the decode kernels need none; a call the streaming kernel cannot take (8 < M <= 16 with
  // an X too large for it, or 3 bits with N % 16 != 0) takes the tensor-core path below
  if (M <= 16 && (gemv_stream_fits(M, N, K) || (bits == 4 && M <= 8))) return 0;
  const int splits = splitk_for(M, N, K);
  return splits > 1 ? align256(static_cast<size_t>(splits) * M * N * sizeof(float)) : 0;
}

awq_status awq_gemm_w4a16(const awq_f16* X, int64_t M, const uint32_t* qweight,
                          const awq_f16* scales, const uint8_t* zeros, int64_t N, int64_t K,
                          int bits, int group, const float* inv_s, unsigned flags, awq_f16* Y,
                          void* workspace, size_t ws_bytes, void* stream) {
  if (bad_dim(M) || bad_dim(N) || bad_dim(K) || K == 0) return AWQ_ERR_INVALID_ARG;
  if (group != awq::kGroup || K % awq::kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (bits != 4 && bits != 3) return AWQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return AWQ_OK;
  if (!X || !qweight || !scales || !zeros || !Y) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      !aligned16(Y) || (inv_s && !aligned16(inv_s)))
    return AWQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<unsigned>(AWQ_GEMM_WEIGHTS_READY | AWQ_GEMM_BF16)) != 0)
    return AWQ_ERR_INVALID_ARG;
  const bool bf16 = (flags & AWQ_GEMM_BF16) != 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half* sc = reinterpret_cast<const __half*>(scales);

  if (M <= 16) {
    awq_status r = launch_gemv_stream(X, M, qweight, sc, zeros, N, K, bits, inv_s, flags, Y, st);
    if (r != AWQ_ERR_UNSUPPORTED) return r;
    // the streaming kernel cannot hold X (or N % 16 != 0): register streaming for fp16 4-bit
    // with M <= 8, the tensor-core path below otherwise
    if (M <= 8 && !bf16 && bits == 4) {
      const unsigned grid = static_cast<unsigned>((N + awq::kGemvRows - 1) / awq::kGemvRows);
      awq::gemv_w4a16_kernel<1><<<grid, awq::kGemvWarps * 32, 0, st>>>(
          reinterpret_cast<const __half*>(X), static_cast<int>(M), qweight, sc, zeros, N, K,
          inv_s, reinterpret_cast<__half*>(Y));
      return launch_status();
    }
  }
  if ((N + awq::kTcBM - 1) / awq::kTcBM > 65535) return AWQ_ERR_INVALID_ARG;
  const int splits = splitk_for(M, N, K);
  const size_t part_bytes =
      splits > 1 ? align256(static_cast<size_t>(splits) * M * N * sizeof(float)) : 0;
  if (part_bytes > 0 && (!workspace || ws_bytes < part_bytes || !aligned16(workspace)))
    return AWQ_ERR_WORKSPACE;
  float* partial = splits > 1 ? static_cast<float*>(workspace) : nullptr;
  awq::TcArgs args{};
  args.M = M;
  args.N = N;
  args.N_pad = N;
  args.K = K;
  args.scales = sc;
  args.zeros = zeros;
  args.Y = Y;
  args.m_tiles = static_cast<int>((M + tc_bn_for(M) - 1) / tc_bn_for(M));
  args.k_splits = splits;
  args.partial = partial;
  args.inv_s = inv_s;   // folded into the dequantized weights by the builders
  awq_status r;
  if (bf16)
    r = bits == 3 ? launch_tc_bn<ASrc::kPacked3, Epi::kStoreY, true>(X, M, qweight, N, args, st)
                  : launch_tc_bn<ASrc::kPacked4, Epi::kStoreY, true>(X, M, qweight, N, args, st);
  else
    r = bits == 3 ? launch_tc_bn<ASrc::kPacked3, Epi::kStoreY>(X, M, qweight, N, args, st)
                  : launch_tc_bn<ASrc::kPacked4, Epi::kStoreY>(X, M, qweight, N, args, st);
  if (r != AWQ_OK || splits == 1) return r;
  const int64_t MN = M * N;
  const unsigned rgrid = static_cast<unsigned>((MN / 4 + 1 + 255) / 256);
  if (bf16)
    awq::splitk_reduce_kernel<true><<<rgrid, 256, 0, st>>>(
        partial, splits, MN, reinterpret_cast<__nv_bfloat16*>(Y));
  else
    awq::splitk_reduce_kernel<false><<<rgrid, 256, 0, st>>>(partial, splits, MN,
                                                            reinterpret_cast<__half*>(Y));
  return launch_status();
}

}  // extern "C"
