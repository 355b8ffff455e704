/*
 * ttt.h -- C ABI of libttt.so: the forward pass of a Test-Time-Training (TTT)
 * layer on one NVIDIA B200 (sm_100a), the backward passes of TTT-Linear and
 * large-chunk TTT, and the affine-map calls of a sequence-parallel
 * large-chunk forward.
 *
 * What the layer computes. The hidden state of a TTT layer is a fast weight W
 * per (batch, head) sequence: a linear map, or a small MLP. Tokens arrive as
 * query/key/value rows q_t, k_t, v_t (the outer model's projections, computed
 * elsewhere) with a per-token inner step size eta_t > 0. The fast weight is
 * trained while the sequence streams, by gradient descent on the
 * reconstruction loss l(W; t) = 1/2 || f(k_t; W) - v_t ||^2, and the layer
 * emits z_t = f(q_t; W_t). Sources, on the TTT pages:
 *   - "Test-Time Training: Linear Complexity Beyond Attention",
 *     "The Dual-Loop Structure" (the inner loop is online gradient descent);
 *     "Key Architectural Mechanics of TTT-Linear" part 1 (the loss), part 2
 *     (gradient and update), part 3 (read-out with the updated weight, then
 *     LayerNorm and a residual), part 4 "Mini-Batch Parallelism (Dual
 *     Formulation)" (mini-batches of b tokens; gradients inside a mini-batch
 *     at the weight it starts from; the change carried forward sequentially);
 *   - "How to Master Test-Time Training for LLMs": the fast weight may be a
 *     multi-layer perceptron;
 *   - "Test-Time Training Done Right" (abstract): large-chunk TTT.
 *
 * Conventions common to every entry point.
 *   - Row form: f(k; W) = k W with W[d_in][d_out] row-major (the pages write
 *     the same map in column form, W k).
 *   - Q, K, V, Z are [B][H][T][d], row-major and contiguous. eta is
 *     [B][H][T] fp32. LayerNorm gain and bias are [H][d] fp32, fixed per head
 *     (they belong to the outer model); LayerNorm uses eps = 1e-5 and the
 *     population variance.
 *   - A fast weight is shared by the batch ([H][...]) unless
 *     TTT_F_W0_PER_SEQ is set, in which case it is [B][H][...] (this is how a
 *     caller resumes a sequence: pass the previous call's W_out as W0).
 *   - Z is written in fp32. W_out (fp32, [B][H][...]) may be NULL.
 *   - Every pointer is a device pointer to memory the caller owns; the
 *     library keeps no pointer after the call returns. Inputs are never
 *     modified. W_out may alias W0 only when TTT_F_W0_PER_SEQ is set.
 *     Q, K, V, Z, W0 and W_out must be 16-byte aligned.
 *   - Calls enqueue work on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and return without synchronising. Arguments are
 *     checked on the host before anything is launched; a failed check
 *     returns its error code and launches nothing.
 *   - Kernels that wait on on-chip barriers bound every wait; if a wait runs
 *     out they record it in a device-side status word and return early, so
 *     the CUDA context stays usable. ttt_device_status() reports that word.
 *   - There is no CPU fallback: a device that is not sm_100 returns
 *     TTT_ERR_UNSUPPORTED_ARCH.
 */
#ifndef TTT_H
#define TTT_H

#include <stddef.h>

#if defined(__GNUC__)
#define TTT_API __attribute__((visibility("default")))
#else
#define TTT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TTT_OK = 0,
    TTT_ERR_ARG = -1,            /* bad flag bits or an inconsistent argument   */
    TTT_ERR_SHAPE = -2,          /* unsupported or inconsistent B,H,T,d,b       */
    TTT_ERR_DTYPE = -3,          /* dtype not supported for this shape          */
    TTT_ERR_ALIGN = -4,          /* a pointer is not 16-byte aligned            */
    TTT_ERR_PTR = -5,            /* a required pointer is NULL or not device memory */
    TTT_ERR_LAUNCH = -6,         /* the CUDA launch failed (see cudaGetLastError) */
    TTT_ERR_DEVICE_TIMEOUT = -7, /* a bounded on-chip wait ran out (device status) */
    TTT_ERR_UNSUPPORTED_ARCH = -8, /* current device is not sm_100              */
    TTT_ERR_WORKSPACE = -9,      /* workspace NULL, misaligned or too small     */
    TTT_ERR_SCRATCH_LIMIT = -10  /* needs more scratch than the library's static buffer */
} ttt_status;

typedef enum { TTT_BF16 = 0, TTT_FP32 = 1 } ttt_dtype; /* element type of Q, K, V */

typedef void *ttt_stream; /* a cudaStream_t */

#define TTT_F_LN 1u         /* f(k) = k + LN(k W) instead of f(k) = k W        */
#define TTT_F_W0_PER_SEQ 2u /* W0 is [B][H][...] instead of [H][...]           */
#define TTT_F_Z_BF16 4u     /* forward entry points: Z is stored as bf16,
                               rounded to nearest even, instead of fp32     */
#define TTT_F_L2_KEYS 8u    /* ttt_linear_fwd: keys scaled to unit length,
                               k / max(||k||_2, 1e-12), wherever the inner
                               loss and its gradient use them (the query is
                               used as given) */

#define TTT_ABI_VERSION 1

/* ABI version of the loaded library (TTT_ABI_VERSION at build time). */
TTT_API int ttt_abi_version(void);

/* Static, human-readable text for a status code; never NULL. */
TTT_API const char *ttt_status_string(int status);

/*
 * TTT-Linear forward, update-then-apply, mini-batch b.
 *   For mini-batch m (tokens mb .. mb+b-1) starting from weight W_m:
 *     G_s  = eta_s * dl/dx at x = k_s W_m        (one row per token s)
 *     z_t  = f(q_t; W_m - sum_{s<=t} k_s^T G_s)   (the token's own step included)
 *     W_{m+1} = W_m - K_m^T G
 *   which is the mini-batch dual form Zpre = Q W_m - tril(Q K^T) G,
 *   W_{m+1} = W_m - K^T G. Without TTT_F_LN, f(k) = k W and dl/dx = kW - v;
 *   with it, f(k) = k + LN(k W) and dl/dx is the LayerNorm backward of
 *   (f - v). ("Key Architectural Mechanics of TTT-Linear", parts 1-4.)
 * Arguments:
 *   Q, K, V   [B][H][T][d], dtype dt
 *   eta       [B][H][T] fp32
 *   W0        [H][d][d] (or [B][H][d][d] with TTT_F_W0_PER_SEQ) fp32
 *   ln_gamma, ln_beta  [H][d] fp32; required with TTT_F_LN, ignored without
 *   Z         [B][H][T][d] output: fp32, or bf16 with TTT_F_Z_BF16
 *   W_out     [B][H][d][d] fp32 output, the weight after the last token; may be NULL
 * Supported: any T >= 1 (when T is not a multiple of b, the last mini-batch
 *   holds the remaining T mod b tokens, every gradient again taken at its
 *   starting weight); d in {16, 32, 64} and 1 <= b <= 64 with b*d <= 4096
 *   for TTT_FP32 and TTT_BF16; TTT_BF16 with d = 64, b = 16 runs the
 *   tensor-core scan, every other case the fp32 CUDA-core kernel.
 * flags: TTT_F_LN, TTT_F_W0_PER_SEQ, TTT_F_Z_BF16, TTT_F_L2_KEYS. With
 *   TTT_F_L2_KEYS the key is normalised, as in the PyTorch listing on "Test-
 *   Time Training: Linear Complexity Beyond Attention"; with LayerNorm, the
 *   residual k of f(k) = k + LN(k W) is the normalised key too. The
 *   tensor-core scan keeps the raw bf16 keys in its products and applies
 *   the per-token scales 1 / ||k|| as row and column scalings in fp32; the
 *   other shapes scale the keys in the fp32 kernel.
 */
TTT_API ttt_status ttt_linear_fwd(const void *Q, const void *K, const void *V, const float *eta,
                          const float *W0, const float *ln_gamma, const float *ln_beta,
                          void *Z, float *W_out, int B, int H, int T, int d, int b,
                          ttt_dtype dt, unsigned flags, ttt_stream stream);

/*
 * One TTT-Linear token per sequence (online decode, b = 1), d = 64, with the
 * fast weight updated in place: for the token q, k, v [B][H][64] and step size
 * eta [B][H] of every sequence, and W [B][H][64][64] fp32 (the sequence's
 * state), computes x = k W, G = eta dl/dx, W <- W - k^T G and z = f(q; W)
 * after the update ("Key Architectural Mechanics of TTT-Linear", parts 1-3;
 * the listing's step()). The same result as ttt_linear_fwd with T = 1, b = 1
 * and TTT_F_W0_PER_SEQ with W_out == W0, from a kernel specialised for it:
 * one 128-thread block per sequence holding W in registers.
 * flags: TTT_F_LN (gamma, beta [H][64] required), TTT_F_Z_BF16, TTT_F_L2_KEYS.
 *   z [B][H][64].
 * Supported: d = 64 (TTT_ERR_SHAPE otherwise), TTT_BF16 or TTT_FP32 inputs.
 */
TTT_API ttt_status ttt_linear_decode(const void *q, const void *k, const void *v, const float *eta,
                                     float *W, const float *ln_gamma, const float *ln_beta,
                                     void *z, int B, int H, int d, ttt_dtype dt, unsigned flags,
                                     ttt_stream stream);

/*
 * One TTT-MLP token per sequence (online decode, b = 1), d = 64, dh = 256, both
 * layers updated in place: q, k, v [B][H][64], eta [B][H], W1 [B][H][64][256]
 * and W2 [B][H][256][64] fp32 (the sequence's state), gamma, beta [H][64],
 * z [B][H][64]. The same result as ttt_mlp_fwd with T = 1, b = 1 and
 * TTT_F_W0_PER_SEQ with the outputs aliasing the inputs, from a kernel
 * specialised for it: one 256-thread block per sequence, thread j holding
 * column j of W1 and row j of W2 in registers.
 * flags: TTT_F_LN (required), TTT_F_Z_BF16. Supported: d = 64, dh = 256
 * (TTT_ERR_SHAPE otherwise); TTT_BF16 or TTT_FP32 inputs; W1 and W2 distinct.
 */
TTT_API ttt_status ttt_mlp_decode(const void *q, const void *k, const void *v, const float *eta,
                                  float *W1, float *W2, const float *ln_gamma,
                                  const float *ln_beta, void *z, int B, int H, int d, int dh,
                                  ttt_dtype dt, unsigned flags, ttt_stream stream);

/*
 * Decode of n tokens per sequence in one call, the fast weight kept on chip
 * across them (the token loop of the listing's step() run inside one kernel,
 * "Test-Time Training: Linear Complexity Beyond Attention"): the tokens of
 * sequence s are q, k, v [B][H][n][64] and eta [B][H][n]; each takes its
 * update and reads out with the updated weight, exactly as n successive
 * ttt_linear_decode / ttt_mlp_decode calls would, and z is [B][H][n][64].
 * The weight lives in the registers of the sequence's block for the whole
 * call and is read and written once. Arguments, flags and errors as
 * ttt_linear_decode / ttt_mlp_decode, plus n >= 1 (TTT_ERR_SHAPE otherwise).
 */
TTT_API ttt_status ttt_linear_decode_tokens(const void *q, const void *k, const void *v,
                                            const float *eta, float *W, const float *ln_gamma,
                                            const float *ln_beta, void *z, int B, int H, int n,
                                            int d, ttt_dtype dt, unsigned flags,
                                            ttt_stream stream);
TTT_API ttt_status ttt_mlp_decode_tokens(const void *q, const void *k, const void *v,
                                         const float *eta, float *W1, float *W2,
                                         const float *ln_gamma, const float *ln_beta, void *z,
                                         int B, int H, int n, int d, int dh, ttt_dtype dt,
                                         unsigned flags, ttt_stream stream);

/*
 * TTT-Linear forward, online (b = 1), with n_steps gradient steps per token
 * ("How to Master Test-Time Training for LLMs", "How TTT Layers Actually
 * Work": the layer runs one or more steps of gradient descent per token).
 * At token t the weight takes n_steps steps W <- W - eta_t dl_t/dW, each
 * gradient at the weight the previous step left, then the token reads out
 * z_t = f(q_t; W). With n_steps = 1 this is ttt_linear_fwd with b = 1.
 * Arguments, flags (TTT_F_LN, TTT_F_W0_PER_SEQ, TTT_F_Z_BF16, TTT_F_L2_KEYS)
 * and errors as ttt_linear_fwd, without b; 1 <= n_steps <= 1024
 * (TTT_ERR_ARG otherwise); d in {16, 32, 64}. Runs the fp32 CUDA-core kernel.
 */
TTT_API ttt_status ttt_linear_fwd_steps(const void *Q, const void *K, const void *V,
                                        const float *eta, const float *W0, const float *ln_gamma,
                                        const float *ln_beta, void *Z, float *W_out, int B, int H,
                                        int T, int d, int n_steps, ttt_dtype dt, unsigned flags,
                                        ttt_stream stream);

/*
 * TTT-Linear backward: the outer gradients of the forward above ("Key
 * Architectural Mechanics of TTT-Linear", parts 1-4; the inner loop is
 * differentiated through, weight updates included). Given dZ = dL/dZ and,
 * optionally, dW_out = dL/dW_out, writes dL/d of every input:
 *   dQ, dK, dV  [B][H][T][d] fp32
 *   deta        [B][H][T] fp32
 *   dW0         [H][d][d] fp32, summed over the batch (or [B][H][d][d] with
 *               TTT_F_W0_PER_SEQ)
 *   dgamma, dbeta  [H][d] fp32, summed over the batch; required with
 *               TTT_F_LN, ignored (may be NULL) without
 * Inputs as ttt_linear_fwd, plus dZ [B][H][T][d] fp32 (required) and dW_out
 * [B][H][d][d] fp32 or NULL (taken as zero). The kernel first re-runs the
 * forward to checkpoint each mini-batch's starting weight, then walks the
 * mini-batches in reverse; the workspace (device memory, 256-byte aligned, at
 * least ttt_linear_bwd_workspace_bytes() bytes, owned by the caller and free
 * to reuse after the stream has passed the call) holds those checkpoints.
 * Outputs are overwritten, never accumulated into. fp32 CUDA cores for both
 * TTT_FP32 and TTT_BF16 inputs; deterministic (fixed summation order).
 * Supported: T % b == 0, d in {16, 32, 64}, 1 <= b with b*d <= 1024. Errors as
 * ttt_linear_fwd, plus TTT_ERR_WORKSPACE.
 */
TTT_API size_t ttt_linear_bwd_workspace_bytes(int B, int H, int T, int d, int b);
TTT_API ttt_status ttt_linear_bwd(const void *Q, const void *K, const void *V, const float *eta,
                                  const float *W0, const float *ln_gamma, const float *ln_beta,
                                  const float *dZ, const float *dW_out, float *dQ, float *dK,
                                  float *dV, float *deta, float *dW0, float *dgamma,
                                  float *dbeta, int B, int H, int T, int d, int b, ttt_dtype dt,
                                  unsigned flags, void *workspace, size_t workspace_bytes,
                                  ttt_stream stream);

/*
 * Large-chunk TTT backward: the outer gradients of ttt_chunk_fwd ("Test-Time
 * Training Done Right", abstract), differentiating through the per-chunk
 * weight updates. With Om_c = dL/dW_c, R_c = K_c W_c - V_c, P_c = K_c Om_{c+1}:
 *   Om_c = Om_{c+1} - A_c Om_{c+1} + Q_c^T dZ_c (A_c = K_c^T diag(eta) K_c),
 *   dQ_c = dZ_c W_c^T, dK_c = -diag(eta)(R_c Om_{c+1}^T + P_c W_c^T),
 *   dV_c = diag(eta) P_c, deta_t = -P_t . R_t, dW0 = Om_0.
 * Arguments as ttt_linear_bwd without LayerNorm: inputs Q, K, V (dtype dt),
 * eta, W0, dZ (fp32, required), dW_out (fp32 or NULL); outputs dQ, dK, dV
 * [B][H][T][d], deta [B][H][T], dW0 [H][d][d] summed over the batch (or
 * [B][H][d][d] with TTT_F_W0_PER_SEQ), all fp32, overwritten. workspace:
 * device memory of at least ttt_chunk_bwd_workspace_bytes() bytes, 256-byte
 * aligned, owned by the caller (per chunk: A_c, B_c, Q_c^T dZ_c, W_c and
 * Om_{c+1} in fp32, and dW0 per sequence). With bf16 inputs and
 * d = 128 the per-chunk products and (chunk % 128 == 0) the per-token
 * products run on the tensor cores, every fp32 operand as two bf16 terms,
 * dK as -diag(eta)(K_c S_c - V_c Om_{c+1}^T) with S_c = W_c Om_{c+1}^T +
 * Om_{c+1} W_c^T (the same quantity); the affine scans run on the tensor
 * cores too (A_c and the state as hi and lo terms), else on fp32 CUDA
 * cores. Deterministic.
 * Supported: d in {64, 128}, chunk % 32 == 0, T % chunk == 0; TTT_BF16 or
 * TTT_FP32. flags: only TTT_F_W0_PER_SEQ.
 */
TTT_API size_t ttt_chunk_bwd_workspace_bytes(int B, int H, int T, int d, int chunk);
TTT_API ttt_status ttt_chunk_bwd(const void *Q, const void *K, const void *V, const float *eta,
                                 const float *W0, const float *dZ, const float *dW_out, float *dQ,
                                 float *dK, float *dV, float *deta, float *dW0, int B, int H, int T,
                                 int d, int chunk, ttt_dtype dt, unsigned flags, void *workspace,
                                 size_t workspace_bytes, ttt_stream stream);

/*
 * TTT-MLP forward: f(k) = k + LN(GELU(k W1) W2) with W1 [d][dh], W2 [dh][d],
 * GELU the exact erf form; same mini-batch rule as ttt_linear_fwd, with both
 * layers updated ("How to Master Test-Time Training for LLMs": the hidden
 * state may be an MLP). In dual form, with A = GELU(K W1),
 * Gx_s = eta_s dl/dx_s and Gh = (Gx W2^T) * GELU'(K W1):
 *   Zpre = GELU(Q W1 - tril(Q K^T) Gh) W2 - tril(Aq A^T) Gx, z = q + LN(Zpre),
 *   W1 -= K^T Gh, W2 -= A^T Gx.
 * Arguments as ttt_linear_fwd, plus:
 *   W1_0  [H][d][dh] (or [B][H][d][dh]), W2_0 [H][dh][d] (or [B][H][dh][d]) fp32
 *   W1_out [B][H][d][dh], W2_out [B][H][dh][d] fp32 outputs, each may be NULL
 * flags must contain TTT_F_LN (the MLP form is defined with LayerNorm).
 * Supported: d in {16, 32, 64}, dh = 4 d, 1 <= b <= 16, T % b == 0,
 *   dtype TTT_BF16 or TTT_FP32.
 */
TTT_API ttt_status ttt_mlp_fwd(const void *Q, const void *K, const void *V, const float *eta,
                       const float *W1_0, const float *W2_0, const float *ln_gamma,
                       const float *ln_beta, void *Z, float *W1_out, float *W2_out, int B,
                       int H, int T, int d, int dh, int b, ttt_dtype dt, unsigned flags,
                       ttt_stream stream);

/*
 * TTT-MLP backward: the outer gradients of ttt_mlp_fwd (the inner loop is
 * differentiated through, weight updates included). Given dZ = dL/dZ and,
 * optionally, dW1_out = dL/dW1_out [B][H][d][dh] and dW2_out = dL/dW2_out
 * [B][H][dh][d] (NULL: taken as zero), writes dL/d of every input:
 *   dQ, dK, dV  [B][H][T][d] fp32;  deta [B][H][T] fp32
 *   dW1_0 [H][d][dh], dW2_0 [H][dh][d] fp32, summed over the batch (or
 *               [B][H][..] with TTT_F_W0_PER_SEQ)
 *   dgamma, dbeta [H][d] fp32, summed over the batch.
 * The kernel re-runs the forward to checkpoint each mini-batch's starting
 * weights in the workspace (2 d dh floats per mini-batch of every sequence),
 * then walks the mini-batches and their tokens in reverse; each token adds
 * the gradient through its own inner gradient (including the LayerNorm
 * backward's backward and GELU''). fp32 CUDA cores, one block per sequence;
 * outputs are overwritten, never accumulated into.
 * workspace: at least ttt_mlp_bwd_workspace_bytes(...) bytes, 256-byte aligned,
 *   owned by the caller, clobbered (0 for an unsupported shape).
 * Supported: TTT_F_LN set (TTT-MLP always has its LayerNorm), d in {16, 32, 64},
 *   dh = 4 d, 1 <= b <= 16, T % b == 0, TTT_BF16 or TTT_FP32 inputs.
 * flags: TTT_F_LN (required), TTT_F_W0_PER_SEQ.
 */
TTT_API size_t ttt_mlp_bwd_workspace_bytes(int B, int H, int T, int d, int dh, int b);
TTT_API ttt_status ttt_mlp_bwd(const void *Q, const void *K, const void *V, const float *eta,
                               const float *W1_0, const float *W2_0, const float *ln_gamma,
                               const float *ln_beta, const float *dZ, const float *dW1_out,
                               const float *dW2_out, float *dQ, float *dK, float *dV, float *deta,
                               float *dW1_0, float *dW2_0, float *dgamma, float *dbeta, int B,
                               int H, int T, int d, int dh, int b, ttt_dtype dt, unsigned flags,
                               void *workspace, size_t workspace_bytes, ttt_stream stream);

/*
 * Large-chunk TTT forward, apply-then-update ("Test-Time Training Done
 * Right"): the tokens of chunk c all read out with W_c, the weight left by
 * the chunks before it, then
 *   W_{c+1} = W_c - sum_{s in c} eta_s k_s^T (k_s W_c - v_s).
 * f(k) = k W (no LayerNorm). With eta_s = 1/chunk this is one step of
 * gradient descent on the chunk's mean loss.
 * Arguments as ttt_linear_fwd without LayerNorm; `chunk` is the chunk length.
 * workspace: device scratch of at least ttt_chunk_workspace_bytes(...) bytes
 *   (160 KiB per chunk of every sequence when d = 128, plus 8 bytes per chunk
 *   for its ready flag and read-out count and a ticket counter, rounded up to
 *   256 bytes; 0 for
 *   the shapes that need none, when workspace may be NULL), 256-byte aligned,
 *   owned by the caller; its contents on entry do not matter and are
 *   clobbered. Calls that share a workspace must not overlap on the GPU.
 * Supported: T % chunk == 0, chunk % 128 == 0; d = 128 with TTT_BF16 runs
 *   on the tensor cores (a memset of the flags and one launch whose blocks
 *   take three roles in start order: the per-chunk Gram products, the
 *   sequential affine scan over chunks, and the read-out of each chunk as
 *   soon as its weight is known), d in {64, 128}
 *   with TTT_FP32, and d = 64, run the fp32 CUDA-core kernel.
 * flags: TTT_F_W0_PER_SEQ, TTT_F_Z_BF16.
 */
TTT_API size_t ttt_chunk_workspace_bytes(int B, int H, int T, int d, int chunk);

TTT_API ttt_status ttt_chunk_fwd(const void *Q, const void *K, const void *V, const float *eta,
                         const float *W0, void *Z, float *W_out, int B, int H, int T, int d,
                         int chunk, ttt_dtype dt, unsigned flags, void *workspace,
                         size_t workspace_bytes, ttt_stream stream);

/*
 * Allocation-free ttt_chunk_fwd. The TTT pages have no counterpart to this
 * call; it exists for callers that cannot allocate device memory themselves,
 * for example a plugin running inside a host application whose own caching
 * allocator owns the whole GPU, or a serving loop that must not trigger the
 * implicit synchronisation of a device allocation. It computes exactly what
 * ttt_chunk_fwd computes (same kernels), but its scratch is a buffer of
 * TTT_CHUNK_NOALLOC_SCRATCH_BYTES that the library declares statically: every
 * GPU that loads libttt.so holds that buffer until the process exits, and no
 * call of this function allocates or frees anything.
 *   - Limit: problems whose ttt_chunk_workspace_bytes(...) exceeds
 *     TTT_CHUNK_NOALLOC_SCRATCH_BYTES (24 MiB + 4 KiB: 153 chunks of d = 128
 *     with their flags) return
 *     TTT_ERR_SCRATCH_LIMIT and launch nothing; use ttt_chunk_fwd with a
 *     caller-allocated workspace for them.
 *   - Every call looks up the buffer's device address on the current device
 *     (a lookup, not an allocation); the first call on a device also loads
 *     the module there, so make it before any stream capture on that device.
 *   - All calls share the one buffer. Its contents persist between calls and
 *     are fully overwritten before being read, so nothing needs clearing;
 *     but calls whose GPU work overlaps (different streams, or different host
 *     threads, on one device) race on it and must be serialised by the caller.
 * Arguments, supported shapes and errors are those of ttt_chunk_fwd, without
 * the workspace pair.
 */
#define TTT_CHUNK_NOALLOC_SCRATCH_BYTES ((24u << 20) + 4096u)
TTT_API ttt_status ttt_chunk_fwd_noalloc(const void *Q, const void *K, const void *V,
                                         const float *eta, const float *W0, void *Z,
                                         float *W_out, int B, int H, int T, int d, int chunk,
                                         ttt_dtype dt, unsigned flags, ttt_stream stream);

/*
 * Sequence-parallel large-chunk TTT. The weight step of every chunk is
 * affine in the weight (the gradient step of "Test-Time Training Done Right",
 * expanded):
 *   W_{c+1} = (I - A_c) W_c + B_c,  A_c = K_c^T diag(eta) K_c,  B_c = K_c^T diag(eta) V_c,
 * so a run of whole chunks (a segment) maps its starting weight to its final
 * weight by W -> M W + N. With every segment's (M, N) known, each segment's
 * starting weight follows from a short fold (ttt_affine_prefix), and the
 * segments then run their forwards independently: on separate ranks that each
 * hold one stretch of the sequence, or on one GPU as more, shorter sequences.
 *
 * ttt_chunk_map: (M, N) of every sequence of K, V, eta ([B][H][T][d],
 *   [B][H][T]), taken as one segment of T / chunk chunks. M and N are
 *   [B][H][d][d] fp32, 16-byte aligned, distinct, written in full.
 *   M = (I - A_{n-1}) ... (I - A_0); N is the weight the chunks end with from
 *   W = 0. Computed with the large-chunk forward's kernels: one forward from
 *   W = I with V = 0 (its final weight is M) and one from W = 0 (its final
 *   weight is N), their read-outs discarded.
 * workspace: at least ttt_chunk_map_workspace_bytes(...) bytes of device
 *   scratch, 256-byte aligned, owned by the caller, clobbered (a zero V, the
 *   discarded read-outs as bf16, the starting weights, and the forward's own
 *   workspace).
 * Supported shapes, dtypes and errors: those of ttt_chunk_fwd; the workspace
 *   size is 0 for an unsupported shape.
 */
TTT_API size_t ttt_chunk_map_workspace_bytes(int B, int H, int T, int d, int chunk, ttt_dtype dt);
TTT_API ttt_status ttt_chunk_map(const void *K, const void *V, const float *eta, float *M,
                                 float *N, int B, int H, int T, int d, int chunk, ttt_dtype dt,
                                 void *workspace, size_t workspace_bytes, ttt_stream stream);

/*
 * ttt_linear_map: the same map for TTT-Linear without LayerNorm, whose
 * mini-batch update ("Key Architectural Mechanics of TTT-Linear", part 4:
 * every gradient of mini-batch m at its starting weight W_m) is
 *   W_{m+1} = W_m - K_m^T diag(eta) (K_m W_m - V_m) = (I - A_m) W_m + B_m.
 * M, N [B][H][d][d] fp32 as for ttt_chunk_map; the segment is T tokens in
 * mini-batches of b (a last partial mini-batch is a step of its own, as in
 * ttt_linear_fwd). Computed with ttt_linear_fwd (no TTT_F_LN): from W = I with
 * V = 0, and from W = 0. workspace: at least ttt_linear_map_workspace_bytes(...)
 * bytes, 256-byte aligned, clobbered. Supported shapes and dtypes: those of
 * ttt_linear_fwd; the workspace size is 0 for an unsupported shape.
 */
TTT_API size_t ttt_linear_map_workspace_bytes(int B, int H, int T, int d, int b, ttt_dtype dt);
TTT_API ttt_status ttt_linear_map(const void *K, const void *V, const float *eta, float *M,
                                  float *N, int B, int H, int T, int d, int b, ttt_dtype dt,
                                  void *workspace, size_t workspace_bytes, ttt_stream stream);

/*
 * The fold of segment maps into starting weights, for S sequences of nseg
 * segments each:
 *   W_in[s][0] = W0[s],  W_in[s][j+1] = M[s][j] W_in[s][j] + N[s][j],
 *   W_end[s] = M[s][nseg-1] W_in[s][nseg-1] + N[s][nseg-1]  (if W_end != NULL).
 * Each (s, j) entry of M, N and W_in is a d x d fp32 row-major block starting
 * at float offset s * seq_stride + j * seg_stride. Two layouts are meant:
 * sequence-major (seq_stride = nseg d^2, seg_stride = d^2: the segments of one
 * sequence adjacent, as when one GPU splits [B][H][T][d] into
 * [B][H * nseg][T / nseg][d]) and segment-major (seq_stride = d^2,
 * seg_stride = S d^2: the maps gathered from nseg ranks, rank-major). The
 * strides must keep the blocks apart: seq_stride >= nseg * seg_stride with
 * seg_stride >= d^2, or seg_stride >= S * seq_stride with seq_stride >= d^2
 * (when nseg == 1 only seq_stride >= d^2 is needed); both multiples of 4.
 * W0 is [H][d][d] (sequence s uses head s % H; S a multiple of H) or, with
 * TTT_F_W0_PER_SEQ, [S][d][d]. W_end is [S][d][d] or NULL. W_in and W_end must
 * not overlap M, N or W0. All pointers 16-byte aligned. Supported: d = 64 and
 * 128, fp32 arithmetic (fused multiply-add, k ascending). One launch, one
 * block per sequence; nseg - 1 (or nseg, with W_end) dependent d^3 products.
 */
TTT_API ttt_status ttt_affine_prefix(const float *M, const float *N, const float *W0, float *W_in,
                                     float *W_end, int S, int H, int nseg, int d,
                                     long long seq_stride, long long seg_stride, unsigned flags,
                                     ttt_stream stream);

/*
 * Synchronises `stream`, then returns TTT_OK, TTT_ERR_DEVICE_TIMEOUT if a
 * kernel of this library ran out of a bounded wait since the last call
 * (the word is then cleared), or TTT_ERR_LAUNCH if the stream reports a CUDA
 * error.
 */
TTT_API ttt_status ttt_device_status(ttt_stream stream);

/*
 * Number of kernels this library has launched in this process so far (a
 * host-side counter, incremented once per successful kernel launch). Lets a
 * caller count the library's launches inside a timed region.
 */
TTT_API unsigned long long ttt_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H */
