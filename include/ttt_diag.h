/*
 * ttt_diag.h -- diagnostics of libttt.so (not part of the TTT computation).
 *
 * ttt_selftest_umma checks the tensor-core plumbing the TTT kernels are built
 * on (shared-memory operand layouts, matrix and instruction descriptors,
 * tensor-memory accumulators) by computing one small product D = A * B on the
 * current device and writing it out, so a caller can compare it with any
 * reference matmul. ttt_diag_gelu exposes the MLP kernel's activation.
 */
#ifndef TTT_DIAG_H
#define TTT_DIAG_H

#include "ttt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Operand layouts in shared memory. */
#define TTT_DIAG_KMAJOR_SW128 0  /* rows of 64 K-elements, 128-byte swizzle */
#define TTT_DIAG_MNMAJOR_SW128 1 /* rows of 64 M/N-elements, 128-byte swizzle */
#define TTT_DIAG_KMAJOR_NONE 2   /* 8x8 core matrices, no swizzle */

/*
 * D[M][N] (fp32, row-major) = A[M][K] * B[K][N] (bf16, row-major), with A
 * and B staged in the given layouts and one 1-CTA tcgen05 MMA chain over K.
 * Supported: M in {64, 128}; N a multiple of 16 in [16, 256] (multiple of 8
 * for M = 64); K a multiple of 16 in [16, 256]. Device pointers; enqueued on
 * `stream`. Returns TTT_ERR_SHAPE / TTT_ERR_ARG for unsupported values.
 */
TTT_API ttt_status ttt_selftest_umma(int M, int N, int K, int a_layout, int b_layout,
                                     const void *A, const void *B, float *D, ttt_stream stream);

/*
 * GELU(h) and GELU'(h) as the TTT-MLP tensor-core kernel evaluates them
 * (exact-erf GELU; erf from Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7),
 * for n fp32 values h -> gelu, gelu_prime (device pointers, n >= 0, either
 * output may be NULL). Enqueued on `stream`. Lets a caller check the
 * kernel's activation against any reference.
 */
TTT_API ttt_status ttt_diag_gelu(const float *h, float *gelu, float *gelu_prime, int n,
                                 ttt_stream stream);

/*
 * Failure-path check: launches one small kernel whose on-chip wait (an
 * mbarrier that nothing ever arrives on) runs out after limit_us
 * microseconds (1 <= limit_us <= 1000000), the same bounded wait the TTT
 * kernels use. The kernel then records the timeout in the device status word
 * and exits normally, so the context stays usable; ttt_device_status() then
 * returns TTT_ERR_DEVICE_TIMEOUT once (and clears the word). Returns
 * TTT_ERR_ARG for a limit out of range.
 */
TTT_API ttt_status ttt_diag_wait_timeout(unsigned limit_us, ttt_stream stream);

/*
 * Per-kernel timing of the library's own launches. While enabled, every
 * entry point records a CUDA event on its stream before its first kernel and
 * after each kernel it launches (events are created on first use on the
 * current device; enabling costs nothing on the device beyond the event
 * records, and nothing synchronises). Up to 512 calls and 2048 events are kept;
 * ttt_diag_kernel_timing(enable) clears them. ttt_diag_kernel_times
 * synchronises on the last event and writes, for each kernel position in
 * launch order, the sum over the recorded calls of that kernel's duration (ms)
 * to ms[0..max); it returns how many kernels a call launched (0 when nothing
 * was recorded), TTT_ERR_ARG when the calls launched different numbers of
 * kernels, the record overflowed or the calls ran on another device, or
 * TTT_ERR_LAUNCH when an event query failed. Not thread-safe; meant for
 * benchmarks.
 */
TTT_API ttt_status ttt_diag_kernel_timing(int enable);
TTT_API int ttt_diag_kernel_times(float *ms, int max);

/*
 * The TTT-MLP forward of ttt_mlp_fwd ("How to Master Test-Time Training for
 * LLMs": the hidden state as a multi-layer perceptron; the mini-batch dual
 * form of "Test-Time Training: Linear Complexity Beyond Attention", Key
 * Architectural Mechanics part 4) computed by the alternative kernel that
 * runs every dense product as a tcgen05.mma issued by one thread (operands in
 * shared memory, fp32 accumulators in tensor memory), instead of the
 * warp-level MMA kernel ttt_mlp_fwd uses for these shapes. Same arguments,
 * results within the same tolerance; kept to measure one design against the
 * other. Supported: TTT_BF16, d = 64, dh = 256, b = 16 (TTT_ERR_SHAPE
 * otherwise).
 */
TTT_API ttt_status ttt_diag_mlp_fwd_tcgen05(const void *Q, const void *K, const void *V,
                                            const float *eta, const float *W1_0,
                                            const float *W2_0, const float *ln_gamma,
                                            const float *ln_beta, void *Z, float *W1_out,
                                            float *W2_out, int B, int H, int T, int d, int dh,
                                            int b, ttt_dtype dt, unsigned flags,
                                            ttt_stream stream);

/*
 * Cost of issuing tcgen05.mma from one thread: one block issues `count`
 * back-to-back M x N x 16 bf16 products (M in {64, 128}; N a multiple of 16
 * in [16, 256], of 8 for M = 64; 1 <= count <= 256) into `nacc` accumulators
 * in turn (1 <= nacc <= 4), twice, and writes the SM clock cycles of the
 * second round to cycles[0] (issuing the instructions) and cycles[1] (issue
 * until their commit's mbarrier completes). cycles: two device int64.
 * Operands are zero; the products themselves are discarded.
 */
TTT_API ttt_status ttt_diag_umma_issue_cycles(int M, int N, int count, int nacc,
                                              long long *cycles, ttt_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_DIAG_H */
