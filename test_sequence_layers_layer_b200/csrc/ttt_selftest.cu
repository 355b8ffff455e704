// ttt_selftest.cu -- ttt_selftest_umma: one small tcgen05 product with
// operands staged in a chosen canonical shared-memory layout, to check the
// layouts and descriptors the TTT kernels use against a reference matmul.
#include "../../include/ttt_diag.h"
#include "sm100.cuh"
#include "ttt_common.cuh"
#include "ttt_gelu.cuh"

namespace ttt {
namespace {

using namespace sm100;

struct SelftestArgs {
    int M, N, K, a_layout, b_layout;
    const __nv_bfloat16 *A, *B;
    float *D;
    int *status;
};

// Bytes a (mn_rows x k_rows) operand occupies in `layout`: the 128-byte
// swizzle pads the contiguous dimension to whole 128-byte rows.
__host__ __device__ uint32_t operand_bytes(int layout, uint32_t mn_rows, uint32_t k_rows) {
    if (layout == TTT_DIAG_KMAJOR_SW128) return mn_rows * 128u * ((k_rows + 63) / 64);
    if (layout == TTT_DIAG_MNMAJOR_SW128) return k_rows * 128u * ((mn_rows + 63) / 64);
    return mn_rows * k_rows * 2u;
}

__device__ uint32_t operand_offset(int layout, uint32_t mn, uint32_t k, uint32_t mn_rows,
                                   uint32_t k_rows) {
    if (layout == TTT_DIAG_KMAJOR_SW128) return off_kmajor_sw128(mn, k, mn_rows);
    if (layout == TTT_DIAG_MNMAJOR_SW128) return off_mnmajor_sw128(k, mn, k_rows);
    return off_kmajor_none(mn, k, k_rows);
}

// Descriptor of K step s (16 elements) of an operand tile at `base`.
__device__ uint64_t operand_desc(int layout, uint32_t base, int s, uint32_t mn_rows,
                                 uint32_t k_rows) {
    const uint32_t k0 = 16u * s;
    if (layout == TTT_DIAG_KMAJOR_SW128)
        return make_sdesc(base + (k0 >> 6) * mn_rows * 128u + (k0 & 63) * 2, 16, 1024, kSw128);
    if (layout == TTT_DIAG_MNMAJOR_SW128)
        return make_sdesc(base + (k0 >> 3) * 1024u, k_rows * 128u, 1024, kSw128);
    return make_sdesc(base + (k0 >> 3) * 128u, 128, k_rows * 16u, kSwNone);
}

__global__ void __launch_bounds__(128) selftest_kernel(SelftestArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int M = a.M, N = a.N, K = a.K;
    uint8_t *sA = smem;
    uint8_t *sB = smem + ((operand_bytes(a.a_layout, M, K) + 1023) & ~1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ncols = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base, ncols);
    for (int e = threadIdx.x; e < M * K; e += blockDim.x) {
        const int m = e / K, k = e % K;
        *reinterpret_cast<__nv_bfloat16 *>(sA + operand_offset(a.a_layout, m, k, M, K)) = a.A[e];
    }
    for (int e = threadIdx.x; e < K * N; e += blockDim.x) {
        const int k = e / N, n = e % N;
        *reinterpret_cast<__nv_bfloat16 *>(sB + operand_offset(a.b_layout, n, k, N, K)) = a.B[e];
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;
    if (threadIdx.x == 0) {
        const uint32_t idesc = make_idesc_bf16(M, N, a.a_layout == TTT_DIAG_MNMAJOR_SW128,
                                               a.b_layout == TTT_DIAG_MNMAJOR_SW128);
        for (int s = 0; s < K / 16; ++s)
            mma_bf16(tbase, operand_desc(a.a_layout, smem_u32(sA), s, M, K),
                     operand_desc(a.b_layout, smem_u32(sB), s, N, K), idesc, s > 0);
        mma_commit(&bar);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, &abort_flag, a.status, 1));
    tc_fence_after();
    if (ok) {
        // M = 128: row r lives in lane r. M = 64: row 16w + i lives in lane 32w + i.
        const int row = (M == 128) ? 32 * warp + lane : 16 * warp + lane;
        const bool valid = (M == 128) || lane < 16;
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            tmem_ld16(taddr(tbase, 32 * warp, c0), v);
            tmem_ld_wait();
            if (valid)
                for (int i = 0; i < 16; ++i) a.D[(size_t)row * N + c0 + i] = v[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, ncols);
}

__global__ void gelu_kernel(const float *h, float *g, float *gp, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        float prime;
        const float v = gelu_and_prime(h[i], prime);
        if (g) g[i] = v;
        if (gp) gp[i] = prime;
    }
}

// Issue cost of tcgen05.mma: thread 0 issues `count` M x N x 16 products
// (zero operands, K-major, 128-byte swizzle) into `nacc` accumulators in
// turn, twice; the second round's cycles are written out.
constexpr int kIssueSmem = 1024 + 16384 + 32768;

__global__ void __launch_bounds__(128) umma_issue_kernel(int M, int N, int count, int nacc,
                                                         long long *cycles, int *status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) tmem_alloc(&tmem_base, 512);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;
    bool ok = true;
    for (int round = 0; round < 2 && ok; ++round) {
        if (threadIdx.x == 0) {
            const uint32_t idesc = make_idesc_bf16(M, N, false, false);
            const uint32_t a = smem_u32(smem), b = smem_u32(smem + 16384);
            const long long t0 = clock64();
            for (int i = 0; i < count; ++i)
                mma_bf16(tb + (uint32_t)((i % nacc) * N), make_sdesc(a + 32 * (i & 3), 16, 1024, kSw128),
                         make_sdesc(b + 32 * (i & 3), 16, 1024, kSw128), idesc, i >= nacc);
            const long long t1 = clock64();
            mma_commit(&bar);
            ok = mbar_wait(&bar, round & 1, &abort_flag, status, 91);
            const long long t2 = clock64();
            if (ok && round == 1) {
                cycles[0] = t1 - t0;
                cycles[1] = t2 - t0;
            }
        }
        ok = __syncthreads_or(!ok) == 0;
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tb, 512);
}

// One warp waits on an mbarrier nobody arrives on, with a short limit.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncwarp();
    sm100::mbar_wait(&bar, 0, &abort_flag, status, 90, limit_ns);
}

}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_diag_wait_timeout(unsigned limit_us, ttt_stream stream) {
    using namespace ttt;
    if (limit_us < 1 || limit_us > 1000000) return TTT_ERR_ARG;
    int *status = device_status_word();
    if (!status) return TTT_ERR_LAUNCH;
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us, status);
    if (cudaGetLastError() != cudaSuccess) return TTT_ERR_LAUNCH;
    count_launch(1);
    return TTT_OK;
}

extern "C" ttt_status ttt_diag_gelu(const float *h, float *gelu, float *gelu_prime, int n,
                                    ttt_stream stream) {
    using namespace ttt;
    if (n < 0) return TTT_ERR_SHAPE;
    if (n == 0) return TTT_OK;
    if (!h) return TTT_ERR_PTR;
    const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
    gelu_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(h, gelu, gelu_prime, n);
    if (cudaGetLastError() != cudaSuccess) return TTT_ERR_LAUNCH;
    count_launch(1);
    return TTT_OK;
}

extern "C" ttt_status ttt_selftest_umma(int M, int N, int K, int a_layout, int b_layout,
                                        const void *A, const void *B, float *D,
                                        ttt_stream stream) {
    using namespace ttt;
    if (M != 64 && M != 128) return TTT_ERR_SHAPE;
    if (N < 16 || N > 256 || N % (M == 64 ? 8 : 16) != 0 || N % 16 != 0) return TTT_ERR_SHAPE;
    if (K < 16 || K > 256 || K % 16 != 0) return TTT_ERR_SHAPE;
    if (a_layout < 0 || a_layout > 2 || b_layout < 0 || b_layout > 2) return TTT_ERR_ARG;
    if ((a_layout == TTT_DIAG_MNMAJOR_SW128 && M % 64) || (b_layout == TTT_DIAG_MNMAJOR_SW128 && N % 64))
        return TTT_ERR_SHAPE;
    if (!A || !B || !D) return TTT_ERR_PTR;
    SelftestArgs a{M, N, K, a_layout, b_layout, static_cast<const __nv_bfloat16 *>(A),
                   static_cast<const __nv_bfloat16 *>(B), D, device_status_word()};
    const size_t smem = 1024 + ((operand_bytes(a_layout, M, K) + 1023) & ~1023u) +
                        operand_bytes(b_layout, N, K);
    cudaError_t e = cudaFuncSetAttribute(selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return TTT_ERR_LAUNCH;
    selftest_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return TTT_ERR_LAUNCH;
    count_launch(1);
    return TTT_OK;
}

extern "C" ttt_status ttt_diag_umma_issue_cycles(int M, int N, int count, int nacc,
                                                 long long *cycles, ttt_stream stream) {
    using namespace ttt;
    if (M != 64 && M != 128) return TTT_ERR_SHAPE;
    if (N < 16 || N > 256 || N % (M == 64 ? 8 : 16) != 0) return TTT_ERR_SHAPE;
    if (count < 1 || count > 256 || nacc < 1 || nacc > 4 || nacc * N > 512) return TTT_ERR_SHAPE;
    if (!cycles) return TTT_ERR_PTR;
    if (cudaFuncSetAttribute(umma_issue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kIssueSmem) != cudaSuccess)
        return TTT_ERR_LAUNCH;
    umma_issue_kernel<<<1, 128, kIssueSmem, static_cast<cudaStream_t>(stream)>>>(
        M, N, count, nacc, cycles, device_status_word());
    if (cudaGetLastError() != cudaSuccess) return TTT_ERR_LAUNCH;
    count_launch(1);
    return TTT_OK;
}
