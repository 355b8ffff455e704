// ttt_chunk_tc.cu -- large-chunk TTT (apply-then-update) on the tensor cores.
//
// Method ("Test-Time Training Done Right", abstract: large chunks; the chunk
// rule itself is the TTT update of "Test-Time Training: Linear Complexity
// Beyond Attention", Key Architectural Mechanics part 2): every token of
// chunk c reads out with W_c, then
//   W_{c+1} = W_c - sum_{s in c} eta_s k_s^T (k_s W_c - v_s)
//           = W_c - A_c W_c + B_c,   A_c = K_c^T diag(eta) K_c,  B_c = K_c^T diag(eta) V_c.
// The update is affine in W, so the work splits into three launches:
//   1. gram:  A_c | B_c for every chunk of every sequence at once (the only
//             pass over K and V; tcgen05, M = d_in = 128, N = 256, K = tokens);
//   2. scan:  W_{c+1} = W_c - A_c W_c + B_c, 16 steps per sequence in fp32,
//             writing each W_c as the ready-made bf16 hi/lo operand image;
//   3. apply: Z_c = Q_c W_c for every chunk at once (the only pass over Q and
//             the only write of Z; tcgen05, M = 128 tokens, N = d_out, K = d_in;
//             W_c arrives by one bulk copy).
// Q/K/V tiles arrive by TMA with the 128-byte swizzle; accumulators live in
// tensor memory. W_c enters the apply products as two bf16 terms (hi + lo)
// so the read-out keeps ~16 significant bits of the fp32 state.
#include <mutex>

#include "../../include/ttt.h"
#include "sm100.cuh"
#include "ttt_common.cuh"

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: math/epilogue

// ---------------------------------------------------------------------------
// 1. gram: A_c | B_c = (diag(eta) K_c)^T [K_c | V_c]
constexpr int kGramRows = 32;                    // tokens per pipeline stage
constexpr int kGramStages = 4;
constexpr int kGramBox = kGramRows * 128;        // one 64-column box of a stage (4 KB)
constexpr int kGramStageBytes = 6 * kGramBox;    // K (2 boxes) | V (2) | eta*K (2)
constexpr size_t kGramSmem = 1024 + kGramStages * kGramStageBytes;  // 97 KB: two blocks per SM

struct GramArgs {
    const float *eta;
    float *AB;  // [chunks][128][256] fp32
    int chunk;
    int *status;
};

__global__ void __launch_bounds__(kThreads, 2)
    chunk_gram_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, GramArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kGramStages], conv[kGramStages], empty[kGramStages], done, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;
    const long row0 = (long)g * a.chunk;  // first token row of this chunk in [B*H*T][d]
    const int nst = a.chunk / kGramRows;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kGramStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    int issued = 0;

    if (warp == 0 && lane == 0) {
        // TMA producer: K rows and V rows of each stage, two 64-column boxes each.
        for (int r = 0; r < nst; ++r) {
            const int s = r % kGramStages;
            if (r >= kGramStages &&
                !mbar_wait(&empty[s], ((r / kGramStages) - 1) & 1, &abort_flag, a.status, 11))
                break;
            uint8_t *st = smem + s * kGramStageBytes;
            const int y = (int)(row0 + (long)r * kGramRows);
            mbar_arrive_expect_tx(&full[s], 4 * kGramBox);
            tma_load_2d(st, &tmK, 0, y, &full[s]);
            tma_load_2d(st + kGramBox, &tmK, 64, y, &full[s]);
            tma_load_2d(st + 2 * kGramBox, &tmV, 0, y, &full[s]);
            tma_load_2d(st + 3 * kGramBox, &tmV, 64, y, &full[s]);
            issued = r + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: D[d_in][0:128) += (eta K)^T K, D[d_in][128:256) += (eta K)^T V.
        const uint32_t idesc = make_idesc_bf16(128, 256, true, true);
        for (int r = 0; r < nst; ++r) {
            const int s = r % kGramStages;
            if (!mbar_wait(&conv[s], (r / kGramStages) & 1, &abort_flag, a.status, 12)) break;
            tc_fence_after();
            const uint32_t ab = smem_u32(smem + s * kGramStageBytes);
#pragma unroll
            for (int k = 0; k < kGramRows / 16; ++k) {
                const uint64_t ad = make_sdesc(ab + 4 * kGramBox + k * 2048, kGramBox, 1024, kSw128);
                const uint64_t bd = make_sdesc(ab + k * 2048, kGramBox, 1024, kSw128);
                mma_bf16(tm, ad, bd, idesc, (r | k) != 0);
            }
            mma_commit(&empty[s]);
        }
        mma_commit(&done);
    } else if (warp >= 2) {
        // Scale K's rows by eta into the A operand's buffer (K and V stay raw
        // as the B operand). Swizzling permutes 16-byte chunks inside a
        // 128-byte row only, so a chunk's row (token) is offset / 128.
        const int c = threadIdx.x - 64;
        constexpr int kChunks = 2 * kGramBox / 16;  // 16-byte chunks of K per stage
        for (int r = 0; r < nst; ++r) {
            const int s = r % kGramStages;
            // This thread's eta values for the stage, loaded before the wait.
            float ev[kChunks / 128];
#pragma unroll
            for (int i = 0; i < kChunks / 128; ++i) {
                const int o = (c + 128 * i) * 16;
                ev[i] = a.eta[row0 + (long)r * kGramRows + ((o % kGramBox) >> 7)];
            }
            if (!mbar_wait(&full[s], (r / kGramStages) & 1, &abort_flag, a.status, 13)) break;
            uint8_t *st = smem + s * kGramStageBytes;
#pragma unroll
            for (int i = 0; i < kChunks / 128; ++i) {
                const int o = (c + 128 * i) * 16;
                const float e = ev[i];
                const uint4 v = *reinterpret_cast<const uint4 *>(st + o);
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
                uint4 out;
                __nv_bfloat162 *ho = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h[i]);
                    ho[i] = __floats2bfloat162_rn(f.x * e, f.y * e);
                }
                *reinterpret_cast<uint4 *>(st + 4 * kGramBox + o) = out;
            }
            fence_async_smem();
            mbar_arrive(&conv[s]);
        }
        // Epilogue: lanes are d_in rows; write A_c | B_c rows (1 KB each).
        // (__all_sync reconverges the warp for the warp-collective TMEM loads.)
        if (__all_sync(0xffffffffu, mbar_wait(&done, 0, &abort_flag, a.status, 14))) {
            tc_fence_after();
            const int sp = warp & 3;
            const int row = 32 * sp + lane;
            float *dst = a.AB + ((size_t)g * kD + row) * 256;
            for (int q = 0; q < 16; ++q) {
                float v[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), v);
                tmem_ld_wait();
                float4 *d4 = reinterpret_cast<float4 *>(dst + 16 * q);
#pragma unroll
                for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
    // Teardown: after an abort, let this block's own copies and MMAs land
    // before the shared memory and tensor memory are released.
    if (abort_flag) {
        if (warp == 0 && lane == 0)
            for (int r = issued - kGramStages < 0 ? 0 : issued - kGramStages; r < issued; ++r)
                mbar_drain(&full[r % kGramStages], (r / kGramStages) & 1);
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 256);
}

// ---------------------------------------------------------------------------
// 2. scan: W_{c+1} = W_c - A_c W_c + B_c, one block per (sequence, 16 columns).
// A_c is staged in shared memory with coalesced loads each step; W_c is also
// written out as the apply kernel's bf16 hi/lo operand image.
constexpr int kScanPitch = kD + 4;  // padded A row (floats)
constexpr size_t kScanSmem = (size_t)kD * kScanPitch * 4 + kD * 16 * 4;

struct ScanArgs {
    const float *AB, *W0;
    uint8_t *Wimg;  // [chunks][hi 32 KB | lo 32 KB]: MN-major, 128-byte swizzle
    float *W_out;
    int H, chunks_per_seq;
    bool w0_per_seq;
};

__global__ void __launch_bounds__(256, 2) chunk_scan_kernel(ScanArgs a) {
    extern __shared__ __align__(16) float scan_smem[];
    float *sA = scan_smem;                 // [128][kScanPitch]
    float *sW = scan_smem + kD * kScanPitch;  // [128][16]
    const int seq = blockIdx.x, j0 = 16 * blockIdx.y;
    const int i = threadIdx.x >> 1, jh = 8 * (threadIdx.x & 1);
    const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : seq % a.H) * kD * kD;
#pragma unroll
    for (int j = 0; j < 8; ++j) sW[i * 16 + jh + j] = W0[i * kD + j0 + jh + j];
    for (int c = 0; c < a.chunks_per_seq; ++c) {
        const size_t g = (size_t)seq * a.chunks_per_seq + c;
        const float *AB = a.AB + g * kD * 256;
        // stage A_c (columns 0..127 of the 256-wide rows), coalesced
#pragma unroll 4
        for (int e = threadIdx.x; e < kD * kD / 4; e += 256) {
            const int r = e >> 5, c4 = e & 31;
            *reinterpret_cast<float4 *>(sA + r * kScanPitch + 4 * c4) =
                *reinterpret_cast<const float4 *>(AB + (size_t)r * 256 + 4 * c4);
        }
        const float4 b0 = *reinterpret_cast<const float4 *>(AB + (size_t)i * 256 + 128 + j0 + jh);
        const float4 b1 = *reinterpret_cast<const float4 *>(AB + (size_t)i * 256 + 128 + j0 + jh + 4);
        __syncthreads();
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = sW[i * 16 + jh + j];
        {  // W_c as the bf16 hi/lo operand image of the apply kernel
            uint4 hi, lo;
            __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(&hi);
            __nv_bfloat16 *l = reinterpret_cast<__nv_bfloat16 *>(&lo);
#pragma unroll
            for (int j = 0; j < 8; ++j) split_bf16(acc[j], h[j], l[j]);
            uint8_t *img = a.Wimg + g * 65536;
            const uint32_t off = off_mnmajor_sw128(i, j0 + jh, kD);
            *reinterpret_cast<uint4 *>(img + off) = hi;
            *reinterpret_cast<uint4 *>(img + 32768 + off) = lo;
        }
        acc[0] += b0.x; acc[1] += b0.y; acc[2] += b0.z; acc[3] += b0.w;
        acc[4] += b1.x; acc[5] += b1.y; acc[6] += b1.z; acc[7] += b1.w;
        const float *Ar = sA + i * kScanPitch;
#pragma unroll 8
        for (int k = 0; k < kD; k += 4) {
            const float4 av = *reinterpret_cast<const float4 *>(Ar + k);
            const float ak[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float4 w0 = *reinterpret_cast<const float4 *>(sW + (k + kk) * 16 + jh);
                const float4 w1 = *reinterpret_cast<const float4 *>(sW + (k + kk) * 16 + jh + 4);
                acc[0] = fmaf(-ak[kk], w0.x, acc[0]); acc[1] = fmaf(-ak[kk], w0.y, acc[1]);
                acc[2] = fmaf(-ak[kk], w0.z, acc[2]); acc[3] = fmaf(-ak[kk], w0.w, acc[3]);
                acc[4] = fmaf(-ak[kk], w1.x, acc[4]); acc[5] = fmaf(-ak[kk], w1.y, acc[5]);
                acc[6] = fmaf(-ak[kk], w1.z, acc[6]); acc[7] = fmaf(-ak[kk], w1.w, acc[7]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) sW[i * 16 + jh + j] = acc[j];
        __syncthreads();
    }
    if (a.W_out)
#pragma unroll
        for (int j = 0; j < 8; ++j) a.W_out[(size_t)seq * kD * kD + i * kD + j0 + jh + j] = sW[i * 16 + jh + j];
}

// ---------------------------------------------------------------------------
// 3. apply: Z_c = Q_c (W_c,hi + W_c,lo), one block per chunk, 128-token tiles.
constexpr int kApplyRows = 128;
constexpr int kApplyStages = 3;
constexpr int kApplyThreads = 320;  // warp 0: TMA, warp 1: MMA, warps 2-9: epilogue
constexpr int kApplyStageOff = 65536 + kApplyStages * 32768;  // epilogue staging, 8 KB per warp
constexpr size_t kApplySmem = 1024 + kApplyStageOff + 8 * 8192;

struct ApplyArgs {
    const uint8_t *Wimg;
    float *Z;
    int chunk;
    int *status;
};

__global__ void __launch_bounds__(kApplyThreads, 1)
    chunk_apply_kernel(const __grid_constant__ CUtensorMap tmQ, ApplyArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sW = smem;          // hi [0, 32K), lo [32K, 64K): MN-major, d_in rows
    uint8_t *sQ = smem + 65536;  // stages of 128 tokens x 128 d (two 64-column boxes)
    __shared__ uint64_t full[kApplyStages], empty[kApplyStages], tfull[2], tempty[2], wfull, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;
    const long row0 = (long)g * a.chunk;
    const int ntile = a.chunk / kApplyRows;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kApplyStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 256);
        }
        mbar_init(&wfull, 1);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    int issued = 0;
    bool w_issued = false;

    if (warp == 0 && lane == 0) {
        mbar_arrive_expect_tx(&wfull, 65536);
        bulk_load(sW, a.Wimg + (size_t)g * 65536, 32768, &wfull);
        bulk_load(sW + 32768, a.Wimg + (size_t)g * 65536 + 32768, 32768, &wfull);
        w_issued = true;
        for (int t = 0; t < ntile; ++t) {
            const int s = t % kApplyStages;
            if (t >= kApplyStages &&
                !mbar_wait(&empty[s], ((t / kApplyStages) - 1) & 1, &abort_flag, a.status, 21))
                break;
            uint8_t *st = sQ + s * 32768;
            const int y = (int)(row0 + (long)t * kApplyRows);
            mbar_arrive_expect_tx(&full[s], 32768);
            tma_load_2d(st, &tmQ, 0, y, &full[s]);
            tma_load_2d(st + 16384, &tmQ, 64, y, &full[s]);
            issued = t + 1;
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = make_idesc_bf16(128, 128, false, true);
        const uint32_t wb = smem_u32(sW);
        if (mbar_wait(&wfull, 0, &abort_flag, a.status, 22)) {
            for (int t = 0; t < ntile; ++t) {
                const int s = t % kApplyStages, acc = t & 1;
                if (!mbar_wait(&full[s], (t / kApplyStages) & 1, &abort_flag, a.status, 23)) break;
                if (t >= 2 && !mbar_wait(&tempty[acc], ((t >> 1) - 1) & 1, &abort_flag, a.status, 24))
                    break;
                tc_fence_after();
                const uint32_t qb = smem_u32(sQ + s * 32768);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const int k0 = 16 * k;
                    const uint64_t ad = make_sdesc(qb + (k0 >> 6) * 16384 + (k0 & 63) * 2, 16, 1024, kSw128);
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const uint64_t bd = make_sdesc(wb + p * 32768 + (k0 >> 3) * 1024, 16384, 1024, kSw128);
                        mma_bf16(tm + acc * 128, ad, bd, idesc, (k | p) != 0);
                    }
                }
                mma_commit(&empty[s]);
                mma_commit(&tfull[acc]);
            }
        }
    } else if (warp >= 2) {
        // Epilogue: lane = token row of the tile; each warp pair splits the
        // 128 fp32 columns of its subpartition's 32 rows. The warp's 32 x 64
        // block goes through shared memory (16-byte chunk c of row r at chunk
        // c ^ (r & 7): conflict-free both ways) so that every global store
        // writes two whole 256-byte half-rows of Z.
        const int sp = warp & 3, half = (warp - 2) >> 2;
        float *stage = reinterpret_cast<float *>(smem + kApplyStageOff) + (warp - 2) * 2048;
        for (int t = 0; t < ntile; ++t) {
            const int acc = t & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (t >> 1) & 1, &abort_flag, a.status, 25)))
                break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float v[16];
                tmem_ld16(taddr(tm, 32 * sp, acc * 128 + 64 * half + 16 * q), v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<float4 *>(stage + lane * 64 + (((4 * q + i) ^ (lane & 7)) << 2)) =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);  // the accumulator is read; the MMA may reuse it
            __syncwarp();
            float *zbase = a.Z + ((size_t)(row0 + (long)t * kApplyRows) + 32 * sp) * kD + 64 * half;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 2 * i + (lane >> 4), c = lane & 15;
                *reinterpret_cast<float4 *>(zbase + (size_t)r * kD + 4 * c) =
                    *reinterpret_cast<const float4 *>(stage + r * 64 + ((c ^ (r & 7)) << 2));
            }
            __syncwarp();
        }
    }
    if (abort_flag) {
        if (warp == 0 && lane == 0) {
            if (w_issued) mbar_drain(&wfull, 0);
            for (int t = issued - kApplyStages < 0 ? 0 : issued - kApplyStages; t < issued; ++t)
                mbar_drain(&full[t % kApplyStages], (t / kApplyStages) & 1);
        }
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 256);
}

}  // namespace

bool chunk_tc_supported(int d, int chunk, bool bf16) {
    return bf16 && d == kD && chunk >= kApplyRows && chunk % kApplyRows == 0;
}

size_t chunk_tc_workspace_bytes(int B, int H, int T, int d, int chunk) {
    if (d != kD || chunk <= 0 || T % chunk) return 0;
    const size_t n = (size_t)B * H * (T / chunk);
    return n * (kD * 256 + kD * kD) * sizeof(float);
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s) {
    const int cps = a.T / a.chunk;
    const int n = a.B * a.H * cps;
    float *AB = static_cast<float *>(a.workspace);
    uint8_t *Wimg = reinterpret_cast<uint8_t *>(AB + (size_t)n * kD * 256);
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmV, tmQ;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, 64, kGramRows) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, 64, kGramRows) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, 64, kApplyRows))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_gram_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kApplySmem);
    if (e != cudaSuccess) return e;
    int *status = device_status_word();
    chunk_gram_kernel<<<n, kThreads, kGramSmem, s>>>(tmK, tmV, GramArgs{a.eta, AB, a.chunk, status});
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    e = cudaFuncSetAttribute(chunk_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kScanSmem);
    if (e != cudaSuccess) return e;
    chunk_scan_kernel<<<dim3(a.B * a.H, kD / 16), 256, kScanSmem, s>>>(
        ScanArgs{AB, a.W0, Wimg, a.W_out, a.H, cps, a.w0_per_seq});
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    chunk_apply_kernel<<<n, kApplyThreads, kApplySmem, s>>>(tmQ, ApplyArgs{Wimg, a.Z, a.chunk, status});
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

}  // namespace ttt

// ---------------------------------------------------------------------------
// Allocation-free entry point: the same three kernels, with their scratch in a
// statically declared device buffer instead of a caller workspace.
namespace {

static __device__ __align__(256) unsigned char g_chunk_scratch[TTT_CHUNK_NOALLOC_SCRATCH_BYTES];

// Device address of g_chunk_scratch on the current device, looked up once per
// device with that device current. In host code the symbol is only a handle,
// never an address a kernel may be given.
void *chunk_scratch_on_current_device() {
    static std::mutex mu;
    static void *addr[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_chunk_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" ttt_status ttt_chunk_fwd_noalloc(const void *Q, const void *K, const void *V,
                                            const float *eta, const float *W0, float *Z,
                                            float *W_out, int B, int H, int T, int d, int chunk,
                                            ttt_dtype dt, unsigned flags, ttt_stream stream) {
    const size_t need = ttt_chunk_workspace_bytes(B, H, T, d, chunk);
    if (need == 0)  // shapes that run without scratch
        return ttt_chunk_fwd(Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, dt, flags, nullptr, 0,
                             stream);
    if (need > TTT_CHUNK_NOALLOC_SCRATCH_BYTES) return TTT_ERR_SCRATCH_LIMIT;
    void *scratch = chunk_scratch_on_current_device();
    if (!scratch) return TTT_ERR_LAUNCH;
    return ttt_chunk_fwd(Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, dt, flags, scratch,
                         TTT_CHUNK_NOALLOC_SCRATCH_BYTES, stream);
}
