// ttt_api.cu -- the extern "C" entry points of libttt.so (declared in
// include/ttt.h): host-side argument checks, then dispatch to a kernel
// launcher on the caller's stream. No allocation, no synchronisation (except
// in ttt_device_status).
#include <stdint.h>

#include <atomic>

#include <cuda.h>

#include "../../include/ttt.h"
#include "../../include/ttt_diag.h"
#include "ttt_common.cuh"

namespace ttt {

__device__ int g_device_status;  // set by a kernel whose bounded wait ran out

static std::atomic<unsigned long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// Optional per-kernel event timing (diagnostic, see ttt_diag.h). Marks of
// every call since timing was enabled are kept, so nothing synchronises until
// the durations are read.
namespace {
constexpr int kMaxMarks = 2048;
constexpr int kMaxCalls = 512;
bool g_timing = false;
bool g_timing_overflow = false;
int g_timing_dev = -1;
cudaEvent_t g_marks[kMaxMarks];
int g_nevents = 0;  // events created so far on g_timing_dev
int g_nmarks = 0;
int g_call_start[kMaxCalls];
int g_ncalls = 0;

bool record_mark(cudaStream_t s) {
    if (!g_timing) return false;
    if (g_nmarks >= kMaxMarks) {
        g_timing_overflow = true;
        return false;
    }
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != g_timing_dev) {
        if (g_timing_dev >= 0) {  // events belong to another device
            g_timing_overflow = true;
            return false;
        }
        g_timing_dev = dev;
    }
    if (g_nmarks == g_nevents) {
        if (cudaEventCreate(&g_marks[g_nevents]) != cudaSuccess) {
            g_timing_overflow = true;
            return false;
        }
        ++g_nevents;
    }
    cudaEventRecord(g_marks[g_nmarks++], s);
    return true;
}
}  // namespace

void timing_begin(cudaStream_t s) {
    if (!g_timing) return;
    if (g_ncalls >= kMaxCalls || g_nmarks >= kMaxMarks) {
        g_timing_overflow = true;
        return;
    }
    g_call_start[g_ncalls] = g_nmarks;
    if (record_mark(s)) ++g_ncalls;
}

void count_launch(cudaStream_t s) {
    count_launch(1);
    record_mark(s);
}

int *device_status_word() {
    int *p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_device_status) != cudaSuccess)
        return nullptr;
    return p;
}

// 2-D TMA descriptor over a row-major [rows][cols] bf16 (or fp32) tensor,
// box of box_rows x box_cols elements, 128-byte swizzle.
bool encode_tmap_2d(void *map, const void *base, bool f32, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows) {
    using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return false;
        fn = reinterpret_cast<EncodeFn>(p);
    }
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (f32 ? 4 : 2)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(static_cast<CUtensorMap *>(map),
              f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_bf16_2d(void *map, const void *base, uint64_t cols, uint64_t rows,
                         uint32_t box_cols, uint32_t box_rows) {
    return encode_tmap_2d(map, base, false, cols, rows, box_cols, box_rows);
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A pointer the GPU can dereference: device or managed memory.
bool is_device_ptr(const void *p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

// sm_100 check of the current device, cached per device ordinal.
ttt_status check_arch() {
    static int cached[64];  // 0 unknown, 1 ok, -1 not sm_100
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TTT_ERR_UNSUPPORTED_ARCH;
    }
    if (dev < 0 || dev >= 64) return TTT_ERR_UNSUPPORTED_ARCH;
    if (cached[dev] == 0) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cached[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return cached[dev] == 1 ? TTT_OK : TTT_ERR_UNSUPPORTED_ARCH;
}

bool supported_d(int d) { return d == 16 || d == 32 || d == 64; }

ttt_status check_device_ptrs(const void *const *ptrs, int n) {
    for (int i = 0; i < n; ++i)
        if (ptrs[i] && !is_device_ptr(ptrs[i])) return TTT_ERR_PTR;
    return TTT_OK;
}

ttt_status launched(cudaError_t e) { return e == cudaSuccess ? TTT_OK : TTT_ERR_LAUNCH; }

}  // namespace
}  // namespace ttt

namespace ttt {
// Large-chunk backward (ttt_chunk_bwd.cu).
bool chunk_bwd_supported(int d, int chunk);
size_t chunk_bwd_workspace_bytes(int B, int H, int T, int d, int chunk);
cudaError_t launch_chunk_bwd(const void *Q, const void *K, const void *V, const float *eta,
                             const float *W0, const float *dZ, const float *dW_out, float *dQ,
                             float *dK, float *dV, float *deta, float *dW0, int B, int H, int T,
                             int d, int chunk, bool bf16, bool w0_per_seq, void *workspace,
                             cudaStream_t s);
// TTT-Linear decode of n tokens per sequence, d = 64 (ttt_decode.cu).
cudaError_t launch_linear_decode(const void *q, const void *k, const void *v, const float *eta,
                                 const float *gamma, const float *beta, float *W, void *z, int B,
                                 int H, int n, bool bf16, bool ln, bool z_bf16, bool l2_keys,
                                 cudaStream_t s);
// TTT-MLP decode of n tokens per sequence, d = 64, hidden 256 (ttt_mlp_decode.cu).
cudaError_t launch_mlp_decode(const void *q, const void *k, const void *v, const float *eta,
                              const float *gamma, const float *beta, float *W1, float *W2,
                              void *z, int B, int H, int n, bool bf16, bool z_bf16,
                              cudaStream_t s);
// TTT-MLP backward (ttt_mlp_bwd.cu).
bool mlp_bwd_supported(int d, int dh, int b);
size_t mlp_bwd_workspace_bytes(int B, int H, int T, int d, int b);
cudaError_t launch_mlp_bwd(const void *Q, const void *K, const void *V, const float *eta,
                           const float *W1_0, const float *W2_0, const float *gamma,
                           const float *beta, const float *dZ, const float *dW1_out,
                           const float *dW2_out, float *dQ, float *dK, float *dV, float *deta,
                           float *dW1_0, float *dW2_0, float *dgamma, float *dbeta, int B, int H,
                           int T, int d, int b, bool bf16, bool w0_per_seq, void *workspace,
                           cudaStream_t s);
// TTT-Linear on the fp32 CUDA-core kernel with L2-normalised keys (ttt_simt.cu).
cudaError_t launch_linear_simt_keys(const LinearArgs &a, bool l2_keys, cudaStream_t s);
cudaError_t launch_linear_simt_opts(const LinearArgs &a, bool l2_keys, int n_steps,
                                   cudaStream_t s);
// Affine-map kernels of the sequence-parallel large-chunk forward (ttt_affine.cu).
cudaError_t launch_affine_eye(float *W, int S, int d, cudaStream_t s);
cudaError_t launch_affine_prefix(const float *M, const float *N, const float *W0, float *W_in,
                                 float *W_end, int S, int H, int nseg, int d, long long seq_stride,
                                 long long seg_stride, bool w0_per_seq, cudaStream_t s);
}  // namespace ttt

using namespace ttt;

namespace {
size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }
}  // namespace

extern "C" {

int ttt_abi_version(void) { return TTT_ABI_VERSION; }

const char *ttt_status_string(int status) {
    switch (status) {
        case TTT_OK: return "ok";
        case TTT_ERR_ARG: return "invalid argument or flag";
        case TTT_ERR_SHAPE: return "unsupported or inconsistent shape";
        case TTT_ERR_DTYPE: return "unsupported dtype";
        case TTT_ERR_ALIGN: return "pointer not 16-byte aligned";
        case TTT_ERR_PTR: return "required pointer is NULL or not device memory";
        case TTT_ERR_LAUNCH: return "CUDA launch failed";
        case TTT_ERR_DEVICE_TIMEOUT: return "a bounded on-chip wait ran out on the device";
        case TTT_ERR_UNSUPPORTED_ARCH: return "current device is not sm_100 (B200)";
        case TTT_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case TTT_ERR_SCRATCH_LIMIT:
            return "problem needs more scratch than the library's static buffer holds";
        default: return "unknown status";
    }
}

ttt_status ttt_linear_fwd(const void *Q, const void *K, const void *V, const float *eta,
                          const float *W0, const float *ln_gamma, const float *ln_beta,
                          void *Z, float *W_out, int B, int H, int T, int d, int b,
                          ttt_dtype dt, unsigned flags, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_W0_PER_SEQ | TTT_F_Z_BF16 | TTT_F_L2_KEYS)) return TTT_ERR_ARG;
    const bool ln = flags & TTT_F_LN;
    if (!Q || !K || !V || !eta || !W0 || !Z) return TTT_ERR_PTR;
    if (ln && (!ln_gamma || !ln_beta)) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || b > 64) return TTT_ERR_SHAPE;
    if (!supported_d(d) || b * d > 4096) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Z) || !aligned16(W0) ||
        (W_out && !aligned16(W_out)))
        return TTT_ERR_ALIGN;
    if (W_out && W_out == W0 && !(flags & TTT_F_W0_PER_SEQ)) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out};
    st = check_device_ptrs(ptrs, 9);
    if (st != TTT_OK) return st;

    LinearArgs a{Q, K, V, eta, W0, ln_gamma, ln_beta, static_cast<float *>(Z), W_out, B, H, T, d, b,
                 dt == TTT_BF16, ln, (flags & TTT_F_W0_PER_SEQ) != 0, (flags & TTT_F_Z_BF16) != 0};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    const bool l2 = flags & TTT_F_L2_KEYS;
    if (linear_tc_supported(d, b, dt == TTT_BF16)) return launched(launch_linear_tc(a, cs, l2));
    return launched(l2 ? launch_linear_simt_keys(a, true, cs) : launch_linear_simt(a, cs));
}

ttt_status ttt_linear_fwd_steps(const void *Q, const void *K, const void *V, const float *eta,
                                const float *W0, const float *ln_gamma, const float *ln_beta,
                                void *Z, float *W_out, int B, int H, int T, int d, int n_steps,
                                ttt_dtype dt, unsigned flags, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_W0_PER_SEQ | TTT_F_Z_BF16 | TTT_F_L2_KEYS)) return TTT_ERR_ARG;
    if (n_steps < 1 || n_steps > 1024) return TTT_ERR_ARG;
    const bool ln = flags & TTT_F_LN;
    if (!Q || !K || !V || !eta || !W0 || !Z) return TTT_ERR_PTR;
    if (ln && (!ln_gamma || !ln_beta)) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || !supported_d(d)) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Z) || !aligned16(W0) ||
        (W_out && !aligned16(W_out)))
        return TTT_ERR_ALIGN;
    if (W_out && W_out == W0 && !(flags & TTT_F_W0_PER_SEQ)) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out};
    st = check_device_ptrs(ptrs, 9);
    if (st != TTT_OK) return st;
    LinearArgs a{Q, K, V, eta, W0, ln_gamma, ln_beta, static_cast<float *>(Z), W_out, B, H, T, d, 1,
                 dt == TTT_BF16, ln, (flags & TTT_F_W0_PER_SEQ) != 0, (flags & TTT_F_Z_BF16) != 0};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_linear_simt_opts(a, (flags & TTT_F_L2_KEYS) != 0, n_steps, cs));
}

ttt_status ttt_linear_decode_tokens(const void *q, const void *k, const void *v,
                                    const float *eta, float *W, const float *ln_gamma,
                                    const float *ln_beta, void *z, int B, int H, int n, int d,
                                    ttt_dtype dt, unsigned flags, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_Z_BF16 | TTT_F_L2_KEYS)) return TTT_ERR_ARG;
    const bool ln = flags & TTT_F_LN;
    if (!q || !k || !v || !eta || !W || !z) return TTT_ERR_PTR;
    if (ln && (!ln_gamma || !ln_beta)) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || n <= 0 || (long long)B * H > (1LL << 30) || d != 64 ||
        (long long)B * H * n > (1LL << 34))
        return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(W) || !aligned16(z))
        return TTT_ERR_ALIGN;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {q, k, v, eta, W, ln ? ln_gamma : nullptr, ln ? ln_beta : nullptr, z};
    st = check_device_ptrs(ptrs, 8);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_linear_decode(q, k, v, eta, ln_gamma, ln_beta, W, z, B, H, n,
                                         dt == TTT_BF16, ln, (flags & TTT_F_Z_BF16) != 0,
                                         (flags & TTT_F_L2_KEYS) != 0, cs));
}

ttt_status ttt_linear_decode(const void *q, const void *k, const void *v, const float *eta,
                             float *W, const float *ln_gamma, const float *ln_beta, void *z, int B,
                             int H, int d, ttt_dtype dt, unsigned flags, ttt_stream stream) {
    return ttt_linear_decode_tokens(q, k, v, eta, W, ln_gamma, ln_beta, z, B, H, 1, d, dt, flags,
                                    stream);
}

ttt_status ttt_mlp_decode_tokens(const void *q, const void *k, const void *v, const float *eta,
                                 float *W1, float *W2, const float *ln_gamma,
                                 const float *ln_beta, void *z, int B, int H, int n, int d,
                                 int dh, ttt_dtype dt, unsigned flags, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_Z_BF16)) return TTT_ERR_ARG;
    if (!(flags & TTT_F_LN)) return TTT_ERR_ARG;  // TTT-MLP always has its LayerNorm
    if (!q || !k || !v || !eta || !W1 || !W2 || !ln_gamma || !ln_beta || !z) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || n <= 0 || (long long)B * H > (1LL << 30) || d != 64 || dh != 256 ||
        (long long)B * H * n > (1LL << 34))
        return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(W1) || !aligned16(W2) ||
        !aligned16(z))
        return TTT_ERR_ALIGN;
    if (W1 == W2) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {q, k, v, eta, W1, W2, ln_gamma, ln_beta, z};
    st = check_device_ptrs(ptrs, 9);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_mlp_decode(q, k, v, eta, ln_gamma, ln_beta, W1, W2, z, B, H, n,
                                      dt == TTT_BF16, (flags & TTT_F_Z_BF16) != 0, cs));
}

ttt_status ttt_mlp_decode(const void *q, const void *k, const void *v, const float *eta,
                          float *W1, float *W2, const float *ln_gamma, const float *ln_beta,
                          void *z, int B, int H, int d, int dh, ttt_dtype dt, unsigned flags,
                          ttt_stream stream) {
    return ttt_mlp_decode_tokens(q, k, v, eta, W1, W2, ln_gamma, ln_beta, z, B, H, 1, d, dh, dt,
                                 flags, stream);
}

size_t ttt_linear_bwd_workspace_bytes(int B, int H, int T, int d, int b) {
    return linear_bwd_workspace_bytes(B, H, T, d, b);
}

ttt_status ttt_linear_bwd(const void *Q, const void *K, const void *V, const float *eta,
                          const float *W0, const float *ln_gamma, const float *ln_beta,
                          const float *dZ, const float *dW_out, float *dQ, float *dK, float *dV,
                          float *deta, float *dW0, float *dgamma, float *dbeta, int B, int H,
                          int T, int d, int b, ttt_dtype dt, unsigned flags, void *workspace,
                          size_t workspace_bytes, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_W0_PER_SEQ)) return TTT_ERR_ARG;
    const bool ln = flags & TTT_F_LN;
    if (!Q || !K || !V || !eta || !W0 || !dZ || !dQ || !dK || !dV || !deta || !dW0)
        return TTT_ERR_PTR;
    if (ln && (!ln_gamma || !ln_beta || !dgamma || !dbeta)) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || T % b != 0 || !linear_bwd_supported(d, b))
        return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    const size_t need = linear_bwd_workspace_bytes(B, H, T, d, b);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TTT_ERR_WORKSPACE;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W0, ln ? ln_gamma : nullptr, ln ? ln_beta : nullptr, dZ,
                          dW_out, dQ, dK, dV, deta, dW0, ln ? dgamma : nullptr,
                          ln ? dbeta : nullptr, workspace};
    st = check_device_ptrs(ptrs, 17);
    if (st != TTT_OK) return st;
    LinearBwdArgs a{Q, K, V, eta, W0, ln_gamma, ln_beta, dZ, dW_out, dQ, dK, dV, deta, dW0,
                    dgamma, dbeta, B, H, T, d, b, dt == TTT_BF16, ln,
                    (flags & TTT_F_W0_PER_SEQ) != 0, workspace};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_linear_bwd(a, cs));
}

size_t ttt_chunk_bwd_workspace_bytes(int B, int H, int T, int d, int chunk) {
    return chunk_bwd_workspace_bytes(B, H, T, d, chunk);
}

ttt_status ttt_chunk_bwd(const void *Q, const void *K, const void *V, const float *eta,
                         const float *W0, const float *dZ, const float *dW_out, float *dQ, float *dK,
                         float *dV, float *deta, float *dW0, int B, int H, int T, int d, int chunk,
                         ttt_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                         ttt_stream stream) {
    if (flags & ~TTT_F_W0_PER_SEQ) return TTT_ERR_ARG;
    if (!Q || !K || !V || !eta || !W0 || !dZ || !dQ || !dK || !dV || !deta || !dW0) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk != 0 || !chunk_bwd_supported(d, chunk))
        return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(W0) || !aligned16(dZ) ||
        !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
        return TTT_ERR_ALIGN;
    const size_t need = chunk_bwd_workspace_bytes(B, H, T, d, chunk);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TTT_ERR_WORKSPACE;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV, deta, dW0, workspace};
    st = check_device_ptrs(ptrs, 13);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_chunk_bwd(Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV, deta, dW0, B, H, T, d,
                                     chunk, dt == TTT_BF16, (flags & TTT_F_W0_PER_SEQ) != 0,
                                     workspace, cs));
}

size_t ttt_mlp_bwd_workspace_bytes(int B, int H, int T, int d, int dh, int b) {
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || T % b || !mlp_bwd_supported(d, dh, b)) return 0;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return 0;
    return mlp_bwd_workspace_bytes(B, H, T, d, b);
}

ttt_status ttt_mlp_bwd(const void *Q, const void *K, const void *V, const float *eta,
                       const float *W1_0, const float *W2_0, const float *ln_gamma,
                       const float *ln_beta, const float *dZ, const float *dW1_out,
                       const float *dW2_out, float *dQ, float *dK, float *dV, float *deta,
                       float *dW1_0, float *dW2_0, float *dgamma, float *dbeta, int B, int H,
                       int T, int d, int dh, int b, ttt_dtype dt, unsigned flags, void *workspace,
                       size_t workspace_bytes, ttt_stream stream) {
    if (flags & ~(TTT_F_LN | TTT_F_W0_PER_SEQ)) return TTT_ERR_ARG;
    if (!(flags & TTT_F_LN)) return TTT_ERR_ARG;
    if (!Q || !K || !V || !eta || !W1_0 || !W2_0 || !ln_gamma || !ln_beta || !dZ || !dQ || !dK ||
        !dV || !deta || !dW1_0 || !dW2_0 || !dgamma || !dbeta)
        return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || T % b != 0 || !mlp_bwd_supported(d, dh, b))
        return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    const size_t need = mlp_bwd_workspace_bytes(B, H, T, d, b);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TTT_ERR_WORKSPACE;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ, dW1_out, dW2_out, dQ,
                          dK, dV, deta, dW1_0, dW2_0, dgamma, dbeta, workspace};
    st = check_device_ptrs(ptrs, 20);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_mlp_bwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ, dW1_out,
                                   dW2_out, dQ, dK, dV, deta, dW1_0, dW2_0, dgamma, dbeta, B, H, T,
                                   d, b, dt == TTT_BF16, (flags & TTT_F_W0_PER_SEQ) != 0,
                                   workspace, cs));
}

namespace {

// Validation shared by the TTT-MLP forward entry points; fills `a` on success.
ttt_status mlp_prepare(const void *Q, const void *K, const void *V, const float *eta,
                       const float *W1_0, const float *W2_0, const float *ln_gamma,
                       const float *ln_beta, void *Z, float *W1_out, float *W2_out, int B, int H,
                       int T, int d, int dh, int b, ttt_dtype dt, unsigned flags, ttt::MlpArgs &a) {
    if (flags & ~(TTT_F_LN | TTT_F_W0_PER_SEQ | TTT_F_Z_BF16)) return TTT_ERR_ARG;
    if (!(flags & TTT_F_LN)) return TTT_ERR_ARG;
    if (!Q || !K || !V || !eta || !W1_0 || !W2_0 || !ln_gamma || !ln_beta || !Z) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || b > 16 || T % b != 0) return TTT_ERR_SHAPE;
    if (!supported_d(d) || dh != 4 * d) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Z) || !aligned16(W1_0) ||
        !aligned16(W2_0) || (W1_out && !aligned16(W1_out)) || (W2_out && !aligned16(W2_out)))
        return TTT_ERR_ALIGN;
    const bool per_seq = flags & TTT_F_W0_PER_SEQ;
    if (!per_seq && ((W1_out && W1_out == W1_0) || (W2_out && W2_out == W2_0))) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1_out, W2_out};
    st = check_device_ptrs(ptrs, 11);
    if (st != TTT_OK) return st;
    a = ttt::MlpArgs{Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, static_cast<float *>(Z), W1_out,
                     W2_out, B, H, T, d, dh, b, dt == TTT_BF16, per_seq,
                     (flags & TTT_F_Z_BF16) != 0};
    return TTT_OK;
}

}  // namespace

ttt_status ttt_mlp_fwd(const void *Q, const void *K, const void *V, const float *eta,
                       const float *W1_0, const float *W2_0, const float *ln_gamma,
                       const float *ln_beta, void *Z, float *W1_out, float *W2_out, int B,
                       int H, int T, int d, int dh, int b, ttt_dtype dt, unsigned flags,
                       ttt_stream stream) {
    MlpArgs a;
    const ttt_status st = mlp_prepare(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1_out,
                                      W2_out, B, H, T, d, dh, b, dt, flags, a);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(mlp_tc_supported(d, dh, b, dt == TTT_BF16, (long long)B * H * T)
                        ? launch_mlp_tc(a, cs)
                        : launch_mlp_simt(a, cs));
}

ttt_status ttt_diag_mlp_fwd_tcgen05(const void *Q, const void *K, const void *V,
                                    const float *eta, const float *W1_0, const float *W2_0,
                                    const float *ln_gamma, const float *ln_beta, void *Z,
                                    float *W1_out, float *W2_out, int B, int H, int T, int d,
                                    int dh, int b, ttt_dtype dt, unsigned flags,
                                    ttt_stream stream) {
    MlpArgs a;
    const ttt_status st = mlp_prepare(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1_out,
                                      W2_out, B, H, T, d, dh, b, dt, flags, a);
    if (st != TTT_OK) return st;
    if (!mlp_tc_supported(d, dh, b, dt == TTT_BF16, (long long)B * H * T)) return TTT_ERR_SHAPE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_mlp_umma(a, cs));
}

size_t ttt_chunk_workspace_bytes(int B, int H, int T, int d, int chunk) {
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk) return 0;
    return chunk_tc_supported(d, chunk, true) ? chunk_tc_workspace_bytes(B, H, T, d, chunk) : 0;
}

ttt_status ttt_chunk_fwd(const void *Q, const void *K, const void *V, const float *eta,
                         const float *W0, void *Z, float *W_out, int B, int H, int T, int d,
                         int chunk, ttt_dtype dt, unsigned flags, void *workspace,
                         size_t workspace_bytes, ttt_stream stream) {
    if (flags & ~(TTT_F_W0_PER_SEQ | TTT_F_Z_BF16)) return TTT_ERR_ARG;
    if (!Q || !K || !V || !eta || !W0 || !Z) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk != 0 || chunk % 128 != 0)
        return TTT_ERR_SHAPE;
    if (d != 64 && d != 128) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Z) || !aligned16(W0) ||
        (W_out && !aligned16(W_out)))
        return TTT_ERR_ALIGN;
    const bool tc = chunk_tc_supported(d, chunk, dt == TTT_BF16);
    const size_t need = tc ? ttt_chunk_workspace_bytes(B, H, T, d, chunk) : 0;
    if (need && (!workspace || workspace_bytes < need ||
                 (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return TTT_ERR_WORKSPACE;
    if (W_out && W_out == W0 && !(flags & TTT_F_W0_PER_SEQ)) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {Q, K, V, eta, W0, Z, W_out, need ? workspace : nullptr};
    st = check_device_ptrs(ptrs, 8);
    if (st != TTT_OK) return st;

    ChunkArgs a{Q, K, V, eta, W0, static_cast<float *>(Z), W_out, B, H, T, d, chunk, dt == TTT_BF16,
                (flags & TTT_F_W0_PER_SEQ) != 0, (flags & TTT_F_Z_BF16) != 0, workspace, workspace_bytes};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(tc ? launch_chunk_tc(a, cs) : launch_chunk_simt(a, cs));
}

size_t ttt_chunk_map_workspace_bytes(int B, int H, int T, int d, int chunk, ttt_dtype dt) {
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk || chunk % 128) return 0;
    if ((d != 64 && d != 128) || (dt != TTT_BF16 && dt != TTT_FP32)) return 0;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return 0;
    // tensor-core shapes: one Gram pass and one scan of [M | N] (the forward's workspace)
    if (chunk_tc_supported(d, chunk, dt == TTT_BF16)) return ttt_chunk_workspace_bytes(B, H, T, d, chunk);
    // others: two forwards, from W = I with V = 0 and from W = 0
    const size_t n = (size_t)B * H * T * d, e = dt == TTT_BF16 ? 2 : 4;
    return round256(n * e) + round256(n * 2) + round256((size_t)B * H * d * d * sizeof(float));
}

ttt_status ttt_chunk_map(const void *K, const void *V, const float *eta, float *M, float *N, int B,
                         int H, int T, int d, int chunk, ttt_dtype dt, void *workspace,
                         size_t workspace_bytes, ttt_stream stream) {
    if (!K || !V || !eta || !M || !N) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk != 0 || chunk % 128 != 0)
        return TTT_ERR_SHAPE;
    if (d != 64 && d != 128) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(K) || !aligned16(V) || !aligned16(M) || !aligned16(N)) return TTT_ERR_ALIGN;
    if (M == N) return TTT_ERR_ARG;
    const size_t need = ttt_chunk_map_workspace_bytes(B, H, T, d, chunk, dt);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TTT_ERR_WORKSPACE;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {K, V, eta, M, N, workspace};
    st = check_device_ptrs(ptrs, 6);
    if (st != TTT_OK) return st;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    if (chunk_tc_supported(d, chunk, dt == TTT_BF16))
        return launched(launch_chunk_map_tc(K, V, eta, M, N, B, H, T, chunk, workspace, cs));
    const size_t S = (size_t)B * H, n = S * T * d, e = dt == TTT_BF16 ? 2 : 4;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    void *v_zero = ws;                                    // [B][H][T][d], V = 0
    void *z_scratch = ws + round256(n * e);               // discarded read-outs, bf16
    float *w_start = reinterpret_cast<float *>(ws + round256(n * e) + round256(n * 2));
    const unsigned f = TTT_F_W0_PER_SEQ | TTT_F_Z_BF16;
    // M: the forward from W = I with V = 0 (every B_c = 0)
    if (cudaMemsetAsync(v_zero, 0, n * e, cs) != cudaSuccess) return TTT_ERR_LAUNCH;
    if (launch_affine_eye(w_start, (int)S, d, cs) != cudaSuccess) return TTT_ERR_LAUNCH;
    st = ttt_chunk_fwd(K, K, v_zero, eta, w_start, z_scratch, M, B, H, T, d, chunk, dt, f, nullptr,
                       0, stream);
    if (st != TTT_OK) return st;
    // N: the forward from W = 0
    if (cudaMemsetAsync(w_start, 0, S * d * d * sizeof(float), cs) != cudaSuccess)
        return TTT_ERR_LAUNCH;
    return ttt_chunk_fwd(K, K, V, eta, w_start, z_scratch, N, B, H, T, d, chunk, dt, f, nullptr, 0,
                         stream);
}

size_t ttt_linear_map_workspace_bytes(int B, int H, int T, int d, int b, ttt_dtype dt) {
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || b > 64 || !supported_d(d) || b * d > 4096) return 0;
    if (dt != TTT_BF16 && dt != TTT_FP32) return 0;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return 0;
    const size_t n = (size_t)B * H * T * d, e = dt == TTT_BF16 ? 2 : 4;
    return round256(n * e) + round256(n * 2) + round256((size_t)B * H * d * d * sizeof(float));
}

ttt_status ttt_linear_map(const void *K, const void *V, const float *eta, float *M, float *N,
                          int B, int H, int T, int d, int b, ttt_dtype dt, void *workspace,
                          size_t workspace_bytes, ttt_stream stream) {
    if (!K || !V || !eta || !M || !N) return TTT_ERR_PTR;
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || b > 64) return TTT_ERR_SHAPE;
    if (!supported_d(d) || b * d > 4096) return TTT_ERR_SHAPE;
    if ((long long)B * H > (1LL << 30) || (long long)B * H * T * d > (1LL << 40)) return TTT_ERR_SHAPE;
    if (dt != TTT_BF16 && dt != TTT_FP32) return TTT_ERR_DTYPE;
    if (!aligned16(K) || !aligned16(V) || !aligned16(M) || !aligned16(N)) return TTT_ERR_ALIGN;
    if (M == N) return TTT_ERR_ARG;
    const size_t need = ttt_linear_map_workspace_bytes(B, H, T, d, b, dt);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TTT_ERR_WORKSPACE;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {K, V, eta, M, N, workspace};
    st = check_device_ptrs(ptrs, 6);
    if (st != TTT_OK) return st;

    const size_t S = (size_t)B * H, n = S * T * d, e = dt == TTT_BF16 ? 2 : 4;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    void *v_zero = ws;                                    // [B][H][T][d], V = 0
    void *z_scratch = ws + round256(n * e);               // discarded read-outs, bf16
    float *w_start = reinterpret_cast<float *>(ws + round256(n * e) + round256(n * 2));
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const unsigned f = TTT_F_W0_PER_SEQ | TTT_F_Z_BF16;  // f(k) = k W: no TTT_F_LN
    timing_begin(cs);
    // M: the forward from W = I with V = 0
    if (cudaMemsetAsync(v_zero, 0, n * e, cs) != cudaSuccess) return TTT_ERR_LAUNCH;
    if (launch_affine_eye(w_start, (int)S, d, cs) != cudaSuccess) return TTT_ERR_LAUNCH;
    st = ttt_linear_fwd(K, K, v_zero, eta, w_start, nullptr, nullptr, z_scratch, M, B, H, T, d, b,
                        dt, f, stream);
    if (st != TTT_OK) return st;
    // N: the forward from W = 0
    if (cudaMemsetAsync(w_start, 0, S * d * d * sizeof(float), cs) != cudaSuccess)
        return TTT_ERR_LAUNCH;
    return ttt_linear_fwd(K, K, V, eta, w_start, nullptr, nullptr, z_scratch, N, B, H, T, d, b, dt,
                          f, stream);
}

ttt_status ttt_affine_prefix(const float *M, const float *N, const float *W0, float *W_in,
                             float *W_end, int S, int H, int nseg, int d, long long seq_stride,
                             long long seg_stride, unsigned flags, ttt_stream stream) {
    if (flags & ~TTT_F_W0_PER_SEQ) return TTT_ERR_ARG;
    const bool per_seq = flags & TTT_F_W0_PER_SEQ;
    if (!M || !N || !W0 || !W_in) return TTT_ERR_PTR;
    if (S <= 0 || H <= 0 || nseg <= 0 || S > (1 << 30) || nseg > (1 << 16)) return TTT_ERR_SHAPE;
    if ((d != 64 && d != 128) || (!per_seq && S % H)) return TTT_ERR_SHAPE;
    const long long dd = (long long)d * d;
    if (seq_stride < 0 || seg_stride < 0 || seq_stride > (1LL << 40) || seg_stride > (1LL << 40))
        return TTT_ERR_ARG;
    const bool nested_seq = seg_stride >= dd && seq_stride >= (long long)nseg * seg_stride;
    const bool nested_seg = seq_stride >= dd && seg_stride >= (long long)S * seq_stride;
    const bool single = (nseg == 1 && seq_stride >= dd) || (S == 1 && seg_stride >= dd);
    if (!nested_seq && !nested_seg && !single) return TTT_ERR_ARG;
    if (seq_stride % 4 || seg_stride % 4) return TTT_ERR_ALIGN;
    if (!aligned16(M) || !aligned16(N) || !aligned16(W0) || !aligned16(W_in) ||
        (W_end && !aligned16(W_end)))
        return TTT_ERR_ALIGN;
    const float *outs[] = {W_in, W_end};
    for (const float *o : outs)
        if (o && (o == M || o == N || o == W0)) return TTT_ERR_ARG;
    ttt_status st = check_arch();
    if (st != TTT_OK) return st;
    const void *ptrs[] = {M, N, W0, W_in, W_end};
    st = check_device_ptrs(ptrs, 5);
    if (st != TTT_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    timing_begin(cs);
    return launched(launch_affine_prefix(M, N, W0, W_in, W_end, S, H, nseg, d, seq_stride,
                                         seg_stride, per_seq, cs));
}

ttt_status ttt_device_status(ttt_stream stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TTT_ERR_LAUNCH;
    int *w = device_status_word();
    if (!w) return TTT_ERR_LAUNCH;
    int v = 0;
    if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_LAUNCH;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice);
        return TTT_ERR_DEVICE_TIMEOUT;
    }
    return TTT_OK;
}

unsigned long long ttt_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

ttt_status ttt_diag_kernel_timing(int enable) {
    g_timing = enable != 0;
    g_timing_overflow = false;
    g_nmarks = 0;
    g_ncalls = 0;
    return TTT_OK;
}

int ttt_diag_kernel_times(float *ms, int max) {
    if (!g_timing || g_ncalls < 1) return 0;
    if (g_timing_overflow || !ms || max < 0) return TTT_ERR_ARG;
    if (cudaEventSynchronize(g_marks[g_nmarks - 1]) != cudaSuccess) return TTT_ERR_LAUNCH;
    // every call must have launched the same number of kernels
    const int n = (g_ncalls > 1 ? g_call_start[1] : g_nmarks) - 1;
    for (int c = 0; c < g_ncalls; ++c) {
        const int end = c + 1 < g_ncalls ? g_call_start[c + 1] : g_nmarks;
        if (end - g_call_start[c] - 1 != n) return TTT_ERR_ARG;
    }
    for (int i = 0; i < n && i < max; ++i) ms[i] = 0.f;
    for (int c = 0; c < g_ncalls; ++c)
        for (int i = 0; i < n && i < max; ++i) {
            float t = 0.f;
            const int m = g_call_start[c] + i;
            if (cudaEventElapsedTime(&t, g_marks[m], g_marks[m + 1]) != cudaSuccess)
                return TTT_ERR_LAUNCH;
            ms[i] += t;
        }
    return n;
}

}  // extern "C"
