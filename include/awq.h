/*
 * awq.h -- C ABI of the B200 (sm_100a) AWQ hot-path library (libawq_b200.so).
 *
 * AWQ, activation-aware weight quantization (MIT Han Lab; described on the robotsatlas.com
 * "AWQ" page, sections "How it works", "Key mechanisms", "Components" and
 * "Hyperparameters", and on the builderai.tools "AWQ" page, section "About"):
 *   1. measure each input channel's activation magnitude on a calibration set,
 *   2. scale salient weight channels up by s (and the activations down by s),
 *   3. pick s on a grid by minimising the layer's output error,
 *   4. quantize the scaled weights group-wise to 4 (or 3) bits with a per-group scale,
 *   5. run the layer with kernels that take the packed weights and fp16 activations.
 *
 * Conventions shared by every call
 *   - Tensors are row-major. W is [N, K] (N output features, K input channels); X is
 *     [M, K] (M tokens); Y = X W^T is [M, N]. fp16 means IEEE binary16 (awq_f16 below).
 *   - Every tensor pointer is a DEVICE pointer owned by the caller and must be 16-byte
 *     aligned. The library never allocates device memory: calls that need scratch space
 *     take a caller-owned workspace whose size the matching *_workspace_size query gives.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every
 *     call is asynchronous on it; outputs are valid once the stream reaches that point.
 *   - The group size must be 128 and K a multiple of 128; bits is 4 or 3.
 *   - Dimensions must be below 2^31.
 *   - Arguments are checked on the host before anything is launched: a call that returns
 *     an error other than AWQ_ERR_CUDA has launched nothing and written nothing.
 *   - Kernels bound every internal wait (about 2 s); a wait that runs out sets a device
 *     status word that awq_check_error() reports as AWQ_ERR_TIMEOUT.
 *   - Calls on one stream are ordered; calls that share a workspace must not overlap.
 *
 * Packed weight layout (this library's convention; the pages fix only "group-wise 4-bit
 * with a per-group scale, e.g. groups of 128"):
 *   - 4-bit: qweight is uint32 [N, K/8]; word j of row n holds k = 8j..8j+7, the code of
 *     k-offset i in nibble position i/2 + 4*(i%2) (positions 0..7 hold offsets
 *     0,2,4,6,1,3,5,7), so masks 0x000F000F / 0x00F000F0 on the word and on the word
 *     shifted right by 8 yield the consecutive pairs (k0,k1), (k2,k3), (k4,k5), (k6,k7).
 *   - 3-bit: qweight is uint32 [N, 3K/32]; per block of 32 consecutive k, word 0 holds the
 *     low two bits of offsets 0..15 and word 1 those of 16..31 (offset i mod 16 at 2-bit
 *     field i/2 + 8*(i%2)), word 2 holds bit 2 of offset i at bit i/2 + 16*(i%2).
 *   - scales: fp16 [K/128, N]; zeros: uint8 [K/128, N] (group-major).
 *   - Dequantized weight: (q - zero) * scale. Storage: 4.1875 bits per weight at 4 bits,
 *     3.1875 at 3 bits.
 */
#ifndef AWQ_B200_H_
#define AWQ_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t awq_f16; /* IEEE binary16 storage */

typedef enum {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad shape, unsupported bits/group */
  AWQ_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement */
  AWQ_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the size query's answer */
  AWQ_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (e.g. no GPU, launch) */
  AWQ_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out (see awq_check_error) */
  AWQ_ERR_BOUNDS = 6         /* debug build only: a kernel's index check failed */
} awq_status;

/* Human-readable name of a status code. Never NULL. */
AWQ_API const char* awq_status_string(awq_status status);

/* Version of this ABI (bumped on any signature or layout change). */
AWQ_API int awq_abi_version(void);

/* Synchronises `stream`, then reads and clears the device status word of the current
 * device. Returns AWQ_ERR_BOUNDS if (in the debug build) a kernel's index check failed,
 * else AWQ_ERR_TIMEOUT if a kernel reported a bounded-wait timeout since the last check,
 * AWQ_ERR_CUDA if the synchronisation failed, AWQ_OK otherwise. */
AWQ_API awq_status awq_check_error(void* stream);

/* Self-test of failure detection: launches one thread that waits on a barrier nothing ever
 * arrives on, with a 50 ms limit instead of the usual ~2 s, so the wait runs out the way a
 * stalled pipeline stage would. The kernel writes 1 to *waited_out (a device int) when its
 * wait ran out, sets the device status word, and returns; the next awq_check_error() on
 * the stream returns AWQ_ERR_TIMEOUT and the context stays usable. */
AWQ_API awq_status awq_selftest_timeout(int* waited_out, void* stream);

/* Self-test of the debug build's bounds checks (libawq_b200_debug.so, compiled with
 * AWQ_DEBUG_BOUNDS; in that build every kernel checks the indices of its global and shared
 * memory accesses against the extents the call's shapes give, skips an access that falls
 * outside, and records it in the device status word). Launches one thread that stores
 * buf[i] = i for i = 0..4 into a device buffer of 4 ints (16-byte aligned): the check stops
 * the fifth store, so buf holds 0..3 and the next awq_check_error() returns AWQ_ERR_BOUNDS.
 * The release build has no checks and returns AWQ_ERR_UNSUPPORTED without launching. */
AWQ_API awq_status awq_selftest_bounds(int* buf, void* stream);

/* Timeline of the trace build (libawq_b200_trace.so, compiled with AWQ_TRACE). In that build
 * the streaming decode kernel (awq_gemm_w4a16 with M <= 16 on its default path) records
 * %globaltimer nanoseconds at fixed points of every CTA: one record of AWQ_TRACE_WORDS
 * 64-bit words per CTA, in the order the CTAs start, for up to 65536 CTAs after the last
 * reset. Record words: 0 N of the launch; 1 units (tile, 2048-k chunk) of the CTA; 2 CTA
 * start; 3 the dependency wait returned (griddepcontrol.wait: the preceding kernel on the
 * stream has completed); 4 X staged in shared memory; 5 the CTA's last unit done;
 * 6 blockIdx.x; 8 + u (u < 24) unit u's packed weights have landed in shared memory and
 * the consumers start on it.
 * awq_trace_reset: synchronous; clears the record count.
 * awq_trace_read: synchronous; copies min(count, max_ctas) records to host memory `out`
 * (max_ctas * AWQ_TRACE_WORDS words, caller-owned) and the record count to *n_ctas.
 * The release and debug builds record nothing and return AWQ_ERR_UNSUPPORTED. */
#define AWQ_TRACE_WORDS 32
AWQ_API awq_status awq_trace_reset(void);
AWQ_API awq_status awq_trace_read(unsigned long long* out, int64_t max_ctas, int64_t* n_ctas);

/* ---------------------------------------------------------------- activation statistics
 * robotsatlas.com "AWQ", "How it works" / "Components: Activation saliency analysis":
 * the activation magnitude of every input channel on the calibration set,
 *     s_x[k] = (1/M) * sum_m |X[m, k]|      (fp64 accumulation, rounded once to fp32).
 * X: fp16 [M, K], M >= 1, K a multiple of 8. s_x: fp32 [K] (output).
 * workspace: at least awq_act_stats_workspace_size(M, K) bytes (fp64 partial sums). */
AWQ_API size_t awq_act_stats_workspace_size(int64_t M, int64_t K);
AWQ_API awq_status awq_act_stats(const awq_f16* X, int64_t M, int64_t K, float* s_x, void* workspace,
                         size_t ws_bytes, void* stream);

/* Same result as awq_act_stats, for callers that cannot allocate device memory. The AWQ
 * pages have no counterpart to this call; it exists because some callers have no way to
 * provide a workspace: a plugin inside another framework's engine that is handed only its
 * input and output pointers, or a latency-critical path that must not call cudaMalloc
 * (which can synchronize the whole device).
 * Instead of a workspace it uses one 1 MiB array of device memory that the library defines
 * at file scope; every GPU that loads the library holds that array until the process exits.
 * Limits: K <= 65536 (K a multiple of 8, M >= 1); a larger K returns AWQ_ERR_INVALID_ARG
 * before anything is launched. The row split is capped at 2^17 / K slices so the partial
 * sums fit the array (on a 148-SM B200 the cap binds for K = 4096 once M > 2048), which can
 * change the fp64 summation order relative to awq_act_stats (the results agree whenever
 * those sums are exact, as they are for fp16 inputs of moderate range).
 * The first call on each device looks up the array's device address (with that device
 * current) and caches it; make that first call before any stream capture.
 * Every call shares the one array: calls that may overlap on the GPU (different streams,
 * or different host threads on the same device) race on it and must be serialized by the
 * caller. Nothing in the array needs clearing between calls: each call overwrites every
 * partial sum it reads. No device memory is allocated or freed by this call. */
AWQ_API awq_status awq_act_stats_noalloc(const awq_f16* X, int64_t M, int64_t K, float* s_x,
                                         void* stream);

/* ---------------------------------------------------------------- quantize and pack
 * robotsatlas.com "AWQ", "Components: Group-wise 4-bit quantization" and "Hyperparameters";
 * builderai.tools "AWQ", "About" ("writes real INT4 weights"). Quantizes W diag(s) per
 * (row, group of 128) with an asymmetric code, in IEEE fp32 with one rounding per step:
 *     w' = w * s[k]; scale = max((max w' - min w') / qmax, 1e-5) rounded to fp16 (sc);
 *     z = clamp(rint(-min w' / sc), 0, qmax); q = clamp(rint(w' / sc) + z, 0, qmax),
 * qmax = 2^bits - 1, rint = round half to even.
 * W: fp16 [N, K]. s: fp32 [K], or NULL for s = 1 (plain round-to-nearest).
 * Outputs: qweight (layout above), scales fp16 [K/128, N], zeros uint8 [K/128, N].
 * N = 0 is a no-op. K % 128 == 0 (and K % 32 == 0 for 3 bits). No workspace. */
AWQ_API awq_status awq_quantize_pack(const awq_f16* W, int64_t N, int64_t K, const float* s, int bits,
                             int group, uint32_t* qweight, awq_f16* scales, uint8_t* zeros,
                             void* stream);

/* ---------------------------------------------------------------- scale search
 * robotsatlas.com "AWQ", "How it works" and "Key mechanisms": per-channel scale chosen by a
 * grid search that minimises the layer's output error. For every grid point a,
 *     s_a[k]  = max(s_x[k], 1e-4)^alphas[a]            (fp64 pow, rounded to fp32), or
 *               s_table[a][k] when s_table is not NULL,
 *     L[a]    = || (deq(Q(W diag(s_a))) diag(1/s_a)) X^T - W X^T ||_F^2,
 * with Q the quantizer of awq_quantize_pack. The error operand
 * E_a = fp16(deq * (1/s_a) - W) is formed per grid point and L[a] = ||E_a X^T||^2 is
 * evaluated on the tensor cores (fp16 operands, fp32 accumulation, fp64 reduction in a
 * fixed order). best_idx = the first index of the minimum; best_s = s_{best_idx}.
 * Searching q/k/v (or gate/up) jointly = passing their row-concatenated W.
 * W: fp16 [N, K]; X: fp16 [M, K] (calibration tokens); s_x: fp32 [K]; alphas: fp32 device
 * array [n_alpha] (1 <= n_alpha <= 64); s_table: NULL or fp32 [n_alpha, K].
 * Outputs (device): losses fp64 [n_alpha], best_idx int32 [1], best_s fp32 [K],
 * best_inv_s NULL or fp32 [K] (1 / best_s, correctly rounded: the inv_s that
 * awq_gemm_w4a16 takes for a layer packed with best_s), row_losses NULL or fp64
 * [n_alpha, N] (each row's share of L[a]).
 * workspace: at least awq_search_scale_workspace_size(M, N, K, n_alpha) bytes. */
AWQ_API size_t awq_search_scale_workspace_size(int64_t M, int64_t N, int64_t K, int n_alpha);
AWQ_API awq_status awq_search_scale(const awq_f16* W, int64_t N, int64_t K, const awq_f16* X,
                            int64_t M, const float* s_x, const float* alphas, int n_alpha,
                            int bits, int group, const float* s_table, double* losses,
                            int32_t* best_idx, float* best_s, float* best_inv_s,
                            double* row_losses, void* workspace, size_t ws_bytes,
                            void* stream);

/* ---------------------------------------------------------------- gated MLP calibration input
 * robotsatlas.com "AWQ", "How it works": the calibration set is passed through the model, so
 * each linear layer is calibrated on the activations that reach it. In a SiLU-gated MLP
 * (this library's reading of the decoder layer's MLP) down_proj sees
 *     H[m, i] = silu(g) * u,  g = sum_k X[m, k] W_gate[i, k],  u = sum_k X[m, k] W_up[i, k],
 * silu(g) = g / (1 + exp(-g)), from the full-precision (fp16) gate_proj and up_proj weights.
 * One tensor-core kernel computes both products of a 128-row tile (fp16 operands, fp32
 * accumulation) and writes fp16 H.
 * X: fp16 [M, K]; W_gate, W_up: fp16 [I, K]; H: fp16 [M, I] (output). K % 128 == 0.
 * M = 0 or I = 0 is a no-op. No workspace. */
AWQ_API awq_status awq_silu_mul_gemm(const awq_f16* X, int64_t M, const awq_f16* W_gate,
                                     const awq_f16* W_up, int64_t I, int64_t K, awq_f16* H,
                                     void* stream);

/* ---------------------------------------------------------------- W4A16 GEMM
 * builderai.tools "AWQ", "About" (kernels for 4-bit weights with 16-bit activations);
 * robotsatlas.com "AWQ", "Implementation pitfalls" (dequantization fused into the GEMM).
 *     Y[m, n] = sum_k X[m, k] * inv_s[k] * (q[n, k] - z[k/128, n]) * scale[k/128, n]
 * with inv_s[k] = 1 when inv_s is NULL (inv_s is the activation side of the per-channel
 * scaling: 1/s for a layer packed with W diag(s)). fp32 accumulation, fp16 output. The
 * decode kernels apply inv_s to the activations in fp32 (x' = fp16(x * inv_s)); the
 * tensor-core kernel folds it into the dequantized weights (fp16(scale * inv_s[k]) per k),
 * so no extra pass over X is made.
 * M <= 16 runs a decode kernel (HBM-bound GEMV, 4 or 3 bits; when N is a multiple of 16 and
 * X fits in one CTA's shared memory, or, for fp16 4-bit M <= 8, a register-streaming kernel);
 * other calls run the tensor-core kernel.
 * X: fp16 [M, K]; Y: fp16 [M, N]. M = 0 or N = 0 is a no-op.
 * flags: 0, or AWQ_GEMM_WEIGHTS_READY. The kernels are launched with programmatic dependent
 * launch, so a kernel of this call may start while the kernel launched just before it on
 * `stream` is still running; by default it reads nothing before that kernel has completed.
 * AWQ_GEMM_WEIGHTS_READY states that qweight, scales and zeros are NOT written by the kernel
 * launched immediately before this call on `stream` (they were written earlier, e.g. model
 * weights loaded once): the decode kernel then starts streaming them at once, overlapping
 * the preceding kernel. X is always read only after the preceding kernel has completed.
 * (This library's kernels let the next launch start only after their own predecessor has
 * completed, so with them the window is exactly one kernel.)
 * AWQ_GEMM_BF16: X and Y are bf16 instead of fp16 (sourcepulse.org "AWQ", "Maintenance &
 * Community": BF16 support); the packed weights, fp16 scales and zero points are the same.
 * The decode kernels dequantize to exact (q - z) bf16 pairs and scale each group's fp32 sum;
 * the tensor-core kernel feeds bf16 (q - z) * scale to the bf16 tensor cores. Other bits are
 * rejected.
 * workspace: at least awq_gemm_workspace_size(M, N, K, bits) bytes: 0 unless the
 * tensor-core kernel splits K across CTAs (few output tiles), then room for the fp32
 * partial sums; the size does not depend on inv_s or flags. */
#define AWQ_GEMM_WEIGHTS_READY 1u
#define AWQ_GEMM_BF16 2u
AWQ_API size_t awq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int bits);
AWQ_API awq_status awq_gemm_w4a16(const awq_f16* X, int64_t M, const uint32_t* qweight,
                          const awq_f16* scales, const uint8_t* zeros, int64_t N, int64_t K,
                          int bits, int group, const float* inv_s, unsigned flags, awq_f16* Y,
                          void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H_ */
