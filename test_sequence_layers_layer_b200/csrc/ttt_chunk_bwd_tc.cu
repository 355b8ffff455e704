// ttt_chunk_bwd_tc.cu -- the per-chunk Gram products of the large-chunk TTT
// backward on the tensor cores (d = 128, bf16 Q/K/V, fp32 dZ):
//   A_c = K_c^T diag(eta) K_c,   B_c = K_c^T diag(eta) V_c,   D_c = Q_c^T dZ_c
// ("Test-Time Training Done Right", abstract: the chunk's gradient step; the
// backward's recurrences use the same A_c, and D_c carries dZ into dL/dW_c),
// written in fp32 in the layout the backward's scan and token kernels read:
// per chunk [A_c | B_c | D_c], each row-major [d_in][d_out].
//
// One block per chunk, 32 tokens per pipeline stage. The products run on
// tcgen05 with M = d_in = 128 and the tokens as the reduction:
//   [A_c | B_c] (N = 256) = (eta K)^T [K | V]   -- with one eta over the chunk,
//       K^T [K | V] scaled by eta in fp32 (exact); otherwise eta K enters as
//       two bf16 terms hi + lo;
//   D_c (N = 256, the two halves added) = Q^T [dZ_hi | dZ_lo].
// Q, K, V enter exactly (bf16); dZ enters as hi + lo, so every product keeps
// ~16 significant bits per operand with fp32 accumulation.
#include "../../include/ttt.h"
#include "sm100.cuh"
#include "ttt_common.cuh"

namespace ttt {

bool encode_tmap_2d(void *map, const void *base, bool f32, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows);

namespace {

using namespace sm100;

constexpr int kD = 128, kRows = 32, kStages = 3;
constexpr int kThreads = 192;        // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: convert, epilogue
constexpr int kBox = kRows * 128;    // one 128-byte-wide box of a stage (4 KB)
// A stage: K (2 boxes) | V (2) | Q (2) | dZ fp32 (4) | [dZ hi | dZ lo] (4) | eta K hi (2) | lo (2)
constexpr int OFF_K = 0, OFF_Q = 4 * kBox, OFF_Z = 6 * kBox, OFF_ZB = 10 * kBox,
              OFF_EK = 14 * kBox;
constexpr int kStageBytes = 18 * kBox;                   // 72 KB
constexpr size_t kSmem = 1024 + kStages * kStageBytes;   // 217 KB
static_assert(kSmem <= 232448, "shared memory budget");

// 4 floats -> 4 bf16 hi terms and 4 bf16 lo terms (hi + lo ~ x).
__device__ __forceinline__ void split4(float a, float b, float c, float d, uint2 &hi, uint2 &lo) {
    split2(a, b, hi.x, lo.x);
    split2(c, d, hi.y, lo.y);
}

struct GramArgs {
    const float *eta;
    float *gram;  // [chunk][3][d][d]
    int chunk;
    int *status;
};

__global__ void __launch_bounds__(kThreads, 1)
    cb_gram_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmZ,
                      GramArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kStages], conv[kStages], empty[kStages], done, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;
    const long row0 = (long)g * a.chunk;  // first token row of the chunk in [B*H*T][d]
    const int nst = a.chunk / kRows;

    // one step size over the whole chunk?
    const float eta0 = a.eta[row0];
    bool differs = false;
    for (int i = threadIdx.x; i < a.chunk; i += kThreads)
        differs |= __float_as_uint(a.eta[row0 + i]) != __float_as_uint(eta0);
    const bool uniform = !__syncthreads_or(differs);

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;  // [A | B] in columns 0-255, [D_hi | D_lo] in 256-511
    int issued = 0;

    if (warp == 0 && lane == 0) {
        // TMA producer: K, V, Q as two 64-column bf16 boxes each, dZ as four
        // 32-column fp32 boxes, 32 token rows per stage.
        for (int r = 0; r < nst; ++r) {
            const int st = r % kStages;
            if (r >= kStages && !mbar_wait(&empty[st], ((r / kStages) - 1) & 1, &abort_flag, a.status, 91))
                break;
            uint8_t *sb = smem + st * kStageBytes;
            const int y = (int)(row0 + (long)r * kRows);
            mbar_arrive_expect_tx(&full[st], 10 * kBox);
            tma_load_2d(sb + OFF_K, &tmK, 0, y, &full[st]);
            tma_load_2d(sb + OFF_K + kBox, &tmK, 64, y, &full[st]);
            tma_load_2d(sb + OFF_K + 2 * kBox, &tmV, 0, y, &full[st]);
            tma_load_2d(sb + OFF_K + 3 * kBox, &tmV, 64, y, &full[st]);
            tma_load_2d(sb + OFF_Q, &tmQ, 0, y, &full[st]);
            tma_load_2d(sb + OFF_Q + kBox, &tmQ, 64, y, &full[st]);
#pragma unroll
            for (int b = 0; b < 4; ++b) tma_load_2d(sb + OFF_Z + b * kBox, &tmZ, 32 * b, y, &full[st]);
            issued = r + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer (MN-major operands: rows = tokens, 64 values per 128-byte row).
        const uint32_t idesc = make_idesc_bf16(128, 256, true, true);
        for (int r = 0; r < nst; ++r) {
            const int st = r % kStages;
            if (!mbar_wait(&conv[st], (r / kStages) & 1, &abort_flag, a.status, 92)) break;
            tc_fence_after();
            const uint32_t sb = smem_u32(smem + st * kStageBytes);
#pragma unroll
            for (int k = 0; k < kRows / 16; ++k) {
                const uint32_t ko = k * 2048;  // 16 token rows
                const uint64_t kv = make_sdesc(sb + OFF_K + ko, kBox, 1024, kSw128);
                const bool acc = (r | k) != 0;
                if (uniform) {
                    mma_bf16(tm, make_sdesc(sb + OFF_K + ko, kBox, 1024, kSw128), kv, idesc, acc);
                } else {
                    mma_bf16(tm, make_sdesc(sb + OFF_EK + ko, kBox, 1024, kSw128), kv, idesc, acc);
                    mma_bf16(tm, make_sdesc(sb + OFF_EK + 2 * kBox + ko, kBox, 1024, kSw128), kv, idesc,
                             true);
                }
                mma_bf16(tm + 256, make_sdesc(sb + OFF_Q + ko, kBox, 1024, kSw128),
                         make_sdesc(sb + OFF_ZB + ko, kBox, 1024, kSw128), idesc, acc);
            }
            mma_commit(&empty[st]);
        }
        mma_commit(&done);
    } else if (warp >= 2) {
        // Converters: dZ (fp32) -> [dZ hi | dZ lo] bf16 operand rows, and with
        // a varying eta, eta K -> hi and lo terms. A unit is 8 columns of one
        // token row; 128-byte rows, 16-byte chunk c of row r at c ^ (r & 7).
        const int t = threadIdx.x - 64;
        for (int r = 0; r < nst; ++r) {
            const int st = r % kStages;
            float ev[4];
            if (!uniform) {
#pragma unroll
                for (int k = 0; k < 4; ++k) ev[k] = a.eta[row0 + (long)r * kRows + ((t + 128 * k) >> 4)];
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (r / kStages) & 1, &abort_flag, a.status, 93)))
                break;
            uint8_t *sb = smem + st * kStageBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int u = t + 128 * k, row = u >> 4, col0 = 8 * (u & 15);
                const int sw = row & 7;
                // dZ: fp32 box col0 / 32, 16-byte chunks (col0 % 32) / 4 and + 1
                const uint8_t *zr = sb + OFF_Z + (col0 >> 5) * kBox + row * 128;
                const int c32 = (col0 & 31) >> 2;
                const float4 z0 = *reinterpret_cast<const float4 *>(zr + ((c32 ^ sw) << 4));
                const float4 z1 = *reinterpret_cast<const float4 *>(zr + (((c32 + 1) ^ sw) << 4));
                uint2 h0, l0, h1, l1;
                split4(z0.x, z0.y, z0.z, z0.w, h0, l0);
                split4(z1.x, z1.y, z1.z, z1.w, h1, l1);
                const int off = row * 128 + ((((col0 & 63) >> 3) ^ sw) << 4);
                *reinterpret_cast<uint4 *>(sb + OFF_ZB + (col0 >> 6) * kBox + off) =
                    make_uint4(h0.x, h0.y, h1.x, h1.y);
                *reinterpret_cast<uint4 *>(sb + OFF_ZB + (2 + (col0 >> 6)) * kBox + off) =
                    make_uint4(l0.x, l0.y, l1.x, l1.y);
                if (!uniform) {
                    const uint4 kq = *reinterpret_cast<const uint4 *>(sb + OFF_K + (col0 >> 6) * kBox + off);
                    const __nv_bfloat162 *kh = reinterpret_cast<const __nv_bfloat162 *>(&kq);
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v = __bfloat1622float2(kh[e]);
                        f[2 * e] = ev[k] * v.x;
                        f[2 * e + 1] = ev[k] * v.y;
                    }
                    uint2 eh0, el0, eh1, el1;
                    split4(f[0], f[1], f[2], f[3], eh0, el0);
                    split4(f[4], f[5], f[6], f[7], eh1, el1);
                    *reinterpret_cast<uint4 *>(sb + OFF_EK + (col0 >> 6) * kBox + off) =
                        make_uint4(eh0.x, eh0.y, eh1.x, eh1.y);
                    *reinterpret_cast<uint4 *>(sb + OFF_EK + (2 + (col0 >> 6)) * kBox + off) =
                        make_uint4(el0.x, el0.y, el1.x, el1.y);
                }
            }
            fence_async_smem();
            mbar_arrive(&conv[st]);
        }
        // Epilogue: lane = d_in row i of the accumulators.
        if (__all_sync(0xffffffffu, mbar_wait(&done, 0, &abort_flag, a.status, 94))) {
            tc_fence_after();
            const int sp = warp & 3, i = 32 * sp + lane;
            const float scale = uniform ? eta0 : 1.f;
            float *out = a.gram + (size_t)g * 3 * kD * kD + (size_t)i * kD;
#pragma unroll 1
            for (int q = 0; q < kD / 16; ++q) {
                float va[16], vb[16], dh[16], dl[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), va);
                tmem_ld16(taddr(tm, 32 * sp, 128 + 16 * q), vb);
                tmem_ld16(taddr(tm, 32 * sp, 256 + 16 * q), dh);
                tmem_ld16(taddr(tm, 32 * sp, 384 + 16 * q), dl);
                tmem_ld_wait();
                float4 *oa = reinterpret_cast<float4 *>(out + 16 * q);
                float4 *ob = reinterpret_cast<float4 *>(out + kD * kD + 16 * q);
                float4 *od = reinterpret_cast<float4 *>(out + 2 * kD * kD + 16 * q);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    oa[e] = make_float4(scale * va[4 * e], scale * va[4 * e + 1], scale * va[4 * e + 2],
                                        scale * va[4 * e + 3]);
                    ob[e] = make_float4(scale * vb[4 * e], scale * vb[4 * e + 1], scale * vb[4 * e + 2],
                                        scale * vb[4 * e + 3]);
                    od[e] = make_float4(dh[4 * e] + dl[4 * e], dh[4 * e + 1] + dl[4 * e + 1],
                                        dh[4 * e + 2] + dl[4 * e + 2], dh[4 * e + 3] + dl[4 * e + 3]);
                }
            }
        }
    }
    // Teardown: after an abort, let this block's own copies and MMAs land
    // before the shared memory and tensor memory are released.
    if (abort_flag) {
        if (warp == 0 && lane == 0)
            for (int r = issued - kStages < 0 ? 0 : issued - kStages; r < issued; ++r)
                mbar_drain(&full[r % kStages], (r / kStages) & 1);
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 512);
}

}  // namespace

bool chunk_bwd_gram_tc_supported(int d, int chunk, bool bf16) {
    return bf16 && d == kD && chunk >= kRows && chunk % kRows == 0;
}

// gram: [B*H*(T/chunk)][3][128][128] fp32, written in full.
cudaError_t launch_chunk_bwd_gram_tc(const void *Q, const void *K, const void *V, const float *eta,
                                     const float *dZ, int B, int H, int T, int chunk, float *gram,
                                     cudaStream_t s) {
    const uint64_t rows = (uint64_t)B * H * T;
    const int nch = B * H * (T / chunk);
    alignas(64) CUtensorMap tmK, tmV, tmQ, tmZ;
    if (!encode_tmap_2d(&tmK, K, false, kD, rows, 64, kRows) ||
        !encode_tmap_2d(&tmV, V, false, kD, rows, 64, kRows) ||
        !encode_tmap_2d(&tmQ, Q, false, kD, rows, 64, kRows) ||
        !encode_tmap_2d(&tmZ, dZ, true, kD, rows, 32, kRows))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(cb_gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmem);
    if (e != cudaSuccess) return e;
    cb_gram_tc_kernel<<<nch, kThreads, kSmem, s>>>(tmK, tmV, tmQ, tmZ,
                                                   GramArgs{eta, gram, chunk, device_status_word()});
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

}  // namespace ttt
