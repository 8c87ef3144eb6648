// Shared device helpers for the AWQ B200 kernels: status word, bounded waits, mbarrier,
// TMA (cp.async.bulk.tensor, no multicast), tcgen05 (TMEM alloc, MMA, commit, loads).
// All inline PTX targets sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace awq {

constexpr int kGroup = 128;   // quantization group along K (the only size the kernels take)

// Device status word. Kernels OR error bits into it; awq_check_error() reads and clears it.
enum : unsigned {
  kDevErrTimeout = 1u,   // a bounded wait on an mbarrier ran out
  kDevErrBounds = 2u,    // a debug bounds check fired
};
__device__ unsigned int g_status_word;

// A wait gives up after this many nanoseconds of %globaltimer (about 2 s): every wait in
// these kernels normally completes in microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void flag_error(unsigned bits) { atomicOr(&g_status_word, bits); }

// Index checks of the debug build (compiled with AWQ_DEBUG_BOUNDS): AWQ_IN_BOUNDS(cond) is
// false, and records kDevErrBounds in the status word, when an index the kernel is about to
// use falls outside the extent the call's shapes give; the kernel then skips that access. In
// the release build it is the constant true and compiles away.
#ifdef AWQ_DEBUG_BOUNDS
__device__ __forceinline__ bool bounds_ok(bool cond) {
  if (!cond) flag_error(kDevErrBounds);
  return cond;
}
#define AWQ_IN_BOUNDS(cond) (::awq::bounds_ok(cond))
#else
#define AWQ_IN_BOUNDS(cond) (true)
#endif

// Timeline of the trace build (compiled with AWQ_TRACE): the streaming decode kernel records
// %globaltimer at fixed points of each CTA into g_trace, one record of kTraceWords words per
// CTA in the order the CTAs start (g_trace_ctas counts them; records past kTraceCtas are
// dropped). In the release and debug builds AWQ_TRACE_AT compiles away.
constexpr int kTraceWords = 32;
constexpr int kTraceCtas = 1 << 16;
// Record layout (word: content)
constexpr int kTrN = 0;          // N of the launch
constexpr int kTrUnits = 1;      // units of this CTA
constexpr int kTrStart = 2;      // CTA start
constexpr int kTrWaited = 3;     // the producer's griddepcontrol.wait returned
constexpr int kTrXStaged = 4;    // X staged in shared memory (consumers' barrier passed)
constexpr int kTrEnd = 5;        // the consumers' last unit done
constexpr int kTrBlock = 6;      // blockIdx.x
constexpr int kTrUnit0 = 8;      // 8 + u: consumer warp 0 saw unit u land (u < 24)
constexpr int kTrMaxUnits = kTraceWords - kTrUnit0;
#ifdef AWQ_TRACE
__device__ unsigned long long g_trace[static_cast<size_t>(kTraceCtas) * kTraceWords];
__device__ unsigned int g_trace_ctas;
#define AWQ_TRACE_AT(rec, word, value)                                                        \
  do {                                                                                       \
    if ((rec) < static_cast<unsigned>(::awq::kTraceCtas))                                    \
      ::awq::g_trace[static_cast<size_t>(rec) * ::awq::kTraceWords + (word)] =               \
          static_cast<unsigned long long>(value);                                            \
  } while (0)
#else
#define AWQ_TRACE_AT(rec, word, value) \
  do {                                 \
  } while (0)
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// The same test with a suspend-time hint: a thread whose phase is not complete is suspended
// until the phase completes or about `hint_ns` nanoseconds have passed, instead of spinning
// and taking issue slots from the warps that are working (a co-resident CTA of the next
// kernel waits here for the whole of the previous kernel).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kWaitSleepNs = 100000;   // longest single suspension (100 us)

// Waits for the phase with the given parity to complete. Returns false (and flags the
// status word) if it did not within `limit_ns` (default kWaitLimitNs); the caller then
// abandons its work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(a, parity, kWaitSleepNs)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      flag_error(kDevErrTimeout);
      return false;
    }
  }
}

// Self-test of the timeout path: one thread waits on an mbarrier that nothing ever arrives
// on, with a short limit, so the wait runs out, flags the status word and the kernel returns.
__global__ void timeout_selftest_kernel(unsigned long long limit_ns, int* waited_out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    const bool ok = mbar_wait(&bar, 0, limit_ns);
    *waited_out = ok ? 0 : 1;
  }
}

#ifdef AWQ_DEBUG_BOUNDS
// Self-test of the debug build's bounds checks: one thread walks one index past a buffer of
// n ints; the check stops the last store and records the violation.
__global__ void bounds_selftest_kernel(int* buf, int n) {
  if (threadIdx.x == 0)
    for (int i = 0; i <= n; ++i)
      if (AWQ_IN_BOUNDS(i < n)) buf[i] = i;
}
#endif

// ----------------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load into this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes),
      "r"(smem_u32(bar))
      : "memory");
}

// L2 prefetches (no shared-memory side effects; coherent with writes of earlier kernels).
__device__ __forceinline__ void prefetch_l2_bulk(const void* gsrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(gsrc)),
               "r"(bytes)
               : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's completion and memory
// flush (a no-op when launched without the attribute), and allow the next grid to launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier over a subset of the CTA's warps.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16 x fp16 -> fp32, one CTA.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored in the 128-byte
// swizzled canonical layout: rows of 64 fp16 (128 B), 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                       // leading offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride offset: 8-row atom
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: fp16 (format 0) or bf16 (format 1) A and B, both
// K-major, fp32 accumulator (D format 1), M x N tile.
__host__ __device__ constexpr uint32_t f16_idesc(int m, int n, bool bf16 = false) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// ----------------------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
  uint32_t r;
  // (a & mask) | orv
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
  return r;
}

// Load of data no kernel writes while this one runs (read-only path, no L1 allocation).
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}
__device__ __forceinline__ uint32_t b2_as_u32(__nv_bfloat162 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __nv_bfloat162 u32_as_b2(uint32_t u) {
  return *reinterpret_cast<__nv_bfloat162*>(&u);
}

// 16-bit activations: fp16, or bf16 when kBf16 (the weights' scales stay fp16 in storage).
template <bool kBf16>
using act_t = std::conditional_t<kBf16, __nv_bfloat16, __half>;

template <bool kBf16>
__device__ __forceinline__ float2 act2_to_float2(uint32_t v) {
  if constexpr (kBf16) return __bfloat1622float2(u32_as_b2(v));
  else return __half22float2(u32_as_h2(v));
}
template <bool kBf16>
__device__ __forceinline__ uint32_t float2_to_act2(float a, float b) {
  if constexpr (kBf16) return b2_as_u32(__floats2bfloat162_rn(a, b));
  else return h2_as_u32(__floats2half2_rn(a, b));
}
template <bool kBf16>
__device__ __forceinline__ act_t<kBf16> float_to_act(float a) {
  if constexpr (kBf16) return __float2bfloat16_rn(a);
  else return __float2half_rn(a);
}

// Eight activations (one 16-byte chunk) times eight fp32 factors, rounded back to 16 bits.
template <bool kBf16>
__device__ __forceinline__ uint4 scale8(uint4 v, float4 s0, float4 s1) {
  float2 f;
  f = act2_to_float2<kBf16>(v.x); v.x = float2_to_act2<kBf16>(f.x * s0.x, f.y * s0.y);
  f = act2_to_float2<kBf16>(v.y); v.y = float2_to_act2<kBf16>(f.x * s0.z, f.y * s0.w);
  f = act2_to_float2<kBf16>(v.z); v.z = float2_to_act2<kBf16>(f.x * s1.x, f.y * s1.y);
  f = act2_to_float2<kBf16>(v.w); v.w = float2_to_act2<kBf16>(f.x * s1.z, f.y * s1.w);
  return v;
}

}  // namespace awq
