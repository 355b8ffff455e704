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
//   2. scan:  W_{c+1} = W_c - A_c W_c + B_c, 16 steps per sequence (tcgen05,
//             M = N = K = 128, hi/lo operands; the state and the update in
//             fp32), writing each W_c as the ready-made bf16 hi/lo operand image;
//   3. apply: Z_c = Q_c W_c for every chunk at once (the only pass over Q and
//             the only write of Z; tcgen05, M = 128 tokens, N = d_out, K = d_in;
//             W_c arrives by one bulk copy).
// Q/K/V tiles arrive by TMA with the 128-byte swizzle; accumulators live in
// tensor memory. W_c enters the apply products as two bf16 terms (hi + lo)
// so the read-out keeps ~16 significant bits of the fp32 state.

#include "../../include/ttt.h"
#include "sm100.cuh"
#include "ttt_common.cuh"

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: math/epilogue

// Workspace per chunk: A_c as a bf16 hi | lo operand image (K-major, 32 KB
// each) and B_c in fp32 (64 KB; column quad q of row i at float4 q * 128 + i); after all chunks, each W_c as the
// apply kernel's bf16 hi | lo image (MN-major, 64 KB).
constexpr int kImgBytes = kD * kD * 2;            // one bf16 128 x 128 image
constexpr int kChunkWs = 2 * kImgBytes + kD * kD * 4;

// ---------------------------------------------------------------------------
// 1. gram: A_c | B_c = (diag(eta) K_c)^T [K_c | V_c]
constexpr int kGramRows = 32;                    // tokens per pipeline stage
constexpr int kGramStages = 4;
constexpr int kGramBox = kGramRows * 128;        // one 64-column box of a stage (4 KB)
constexpr int kGramStageBytes = 6 * kGramBox;    // K (2 boxes) | V (2) | eta*K (2)
constexpr size_t kGramSmem = 1024 + kGramStages * kGramStageBytes;  // 97 KB: two blocks per SM

struct GramArgs {
    const float *eta;
    float *AB;  // [chunks][kChunkWs bytes]: A_c hi | A_c lo | B_c
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
        // Epilogue: lanes are d_in rows i. A_c goes out as the scan's bf16
        // hi/lo operand image (K-major, 128-byte swizzle: row i = 128 bytes
        // per 64 columns j), B_c as fp32 rows. (__all_sync reconverges the
        // warp for the warp-collective TMEM loads.)
        if (__all_sync(0xffffffffu, mbar_wait(&done, 0, &abort_flag, a.status, 14))) {
            tc_fence_after();
            const int sp = warp & 3;
            const int row = 32 * sp + lane;
            uint8_t *blk = reinterpret_cast<uint8_t *>(a.AB) + (size_t)g * kChunkWs;
            float4 *bdst = reinterpret_cast<float4 *>(blk + 2 * kImgBytes);
            for (int q = 0; q < 16; ++q) {
                float v[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), v);
                tmem_ld_wait();
                if (q < 8) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint4 hi, lo;
                        __nv_bfloat16 *hb = reinterpret_cast<__nv_bfloat16 *>(&hi);
                        __nv_bfloat16 *lb = reinterpret_cast<__nv_bfloat16 *>(&lo);
#pragma unroll
                        for (int e = 0; e < 8; ++e) split_bf16(v[8 * h + e], hb[e], lb[e]);
                        const uint32_t off = off_kmajor_sw128(row, 16 * q + 8 * h, kD);
                        *reinterpret_cast<uint4 *>(blk + off) = hi;
                        *reinterpret_cast<uint4 *>(blk + kImgBytes + off) = lo;
                    }
                } else {  // B_c: column quad q4 of row i at float4 q4 * 128 + i
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        bdst[(4 * (q - 8) + i) * kD + row] =
                            make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
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
// 2. scan: W_{c+1} = W_c - A_c W_c + B_c, one block per sequence, on the
// tensor cores. The fp32 state W lives in the registers of 8 epilogue warps
// (row i = TMEM lane, 64 columns each); per chunk the MMA thread forms
// D = A_c W_c from the bf16 hi/lo images of A_c (written by the gram kernel,
// brought in by bulk copy, double-buffered) and of W_c (in shared memory):
// A_hi W_hi + A_hi W_lo + A_lo W_hi, M = N = 128, K = 128, fp32 in TMEM. The
// epilogue adds W_c + B_c - D in fp32 (B_c read from global ahead of time),
// rewrites the W image for the next chunk and bulk-stores it to global as the
// apply kernel's operand for that chunk.
constexpr int kScanThreads = 320;  // warp 0: A loads, warp 1: MMA + TMEM, warps 2-9: epilogue
constexpr size_t kScanSmem = 1024 + 2 * (size_t)kImgBytes /* W */ + 4 * (size_t)kImgBytes /* A x2 */;

struct ScanArgs {
    const uint8_t *AB;  // per chunk: A_c hi | lo image, B_c fp32
    const float *W0;
    uint8_t *Wimg;      // [chunks][hi 32 KB | lo 32 KB]: MN-major, 128-byte swizzle
    float *W_out;
    int H, chunks_per_seq;
    bool w0_per_seq;
    int *status;
};

__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_u32(ssrc)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kScanThreads, 1) chunk_scan_kernel(ScanArgs a) {
    extern __shared__ uint8_t scan_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(scan_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sW = smem;                  // W image: hi | lo (MN-major)
    uint8_t *sA = smem + 2 * kImgBytes;  // A images: [2 buffers][hi | lo] (K-major)
    __shared__ uint64_t aready[2], afree[2], dfull, wready, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.x, cps = a.chunks_per_seq;
    const size_t g0 = (size_t)seq * cps;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&aready[b], 1);
            mbar_init(&afree[b], 1);
        }
        mbar_init(&dfull, 1);
        mbar_init(&wready, 1);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    int issued = 0;

    if (warp == 0 && lane == 0) {
        // A_c images, two chunks ahead of nothing: buffer c & 1 is reused once
        // the MMAs of chunk c - 2 have completed.
        for (int c = 0; c < cps; ++c) {
            const int b = c & 1;
            if (c >= 2 && !mbar_wait(&afree[b], ((c >> 1) - 1) & 1, &abort_flag, a.status, 16)) break;
            mbar_arrive_expect_tx(&aready[b], 2 * kImgBytes);
            bulk_load(sA + b * 2 * kImgBytes, a.AB + (g0 + c) * kChunkWs, 2 * kImgBytes, &aready[b]);
            issued = c + 1;
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = make_idesc_bf16(128, 128, false, true);
        const uint32_t wb = smem_u32(sW);
        for (int c = 0; c < cps; ++c) {
            const int b = c & 1;
            if (!mbar_wait(&aready[b], (c >> 1) & 1, &abort_flag, a.status, 17)) break;
            if (!mbar_wait(&wready, c & 1, &abort_flag, a.status, 18)) break;
            tc_fence_after();
            const uint32_t ab = smem_u32(sA + b * 2 * kImgBytes);
            // (A, W) term pairs: hi hi, hi lo, lo hi
            const uint32_t aoff[3] = {0, 0, (uint32_t)kImgBytes}, woff[3] = {0, (uint32_t)kImgBytes, 0};
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const int k0 = 16 * k;
                    const uint64_t ad = make_sdesc(ab + aoff[p] + (k0 >> 6) * 16384 + (k0 & 63) * 2, 16, 1024, kSw128);
                    const uint64_t bd = make_sdesc(wb + woff[p] + (k0 >> 3) * 1024, 16384, 1024, kSw128);
                    mma_bf16(tm, ad, bd, idesc, (p | k) != 0);
                }
            mma_commit(&afree[b]);
            mma_commit(&dfull);
        }
    } else if (warp >= 2) {
        // Epilogue: row i = 32 (warp & 3) + lane, columns 64 half .. +63.
        const int sp = warp & 3, half = (warp - 2) >> 2;
        const int row = 32 * sp + lane, col0 = 64 * half;
        const bool leader = warp == 2 && lane == 0;
        const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : seq % a.H) * kD * kD;
        float w[64];
#pragma unroll
        for (int j4 = 0; j4 < 16; ++j4) {
            const float4 u = *reinterpret_cast<const float4 *>(W0 + (size_t)row * kD + col0 + 4 * j4);
            w[4 * j4] = u.x;
            w[4 * j4 + 1] = u.y;
            w[4 * j4 + 2] = u.z;
            w[4 * j4 + 3] = u.w;
        }
        // Write this thread's 64 values of W as its row of the MN-major image
        // (k = row, 64-column atom = half): 8 chunks of 8 bf16, hi and lo.
        auto emit = [&]() {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 hi, lo;
                __nv_bfloat16 *hb = reinterpret_cast<__nv_bfloat16 *>(&hi);
                __nv_bfloat16 *lb = reinterpret_cast<__nv_bfloat16 *>(&lo);
#pragma unroll
                for (int e = 0; e < 8; ++e) split_bf16(w[8 * ch + e], hb[e], lb[e]);
                const uint32_t off = off_mnmajor_sw128(row, col0 + 8 * ch, kD);
                *reinterpret_cast<uint4 *>(sW + off) = hi;
                *reinterpret_cast<uint4 *>(sW + kImgBytes + off) = lo;
            }
            fence_async_smem();
        };
        // image of W_c -> global (apply's operand for chunk c); W ready for the MMA
        auto publish = [&](int c) {
            if (leader) {
                bulk_store(a.Wimg + (g0 + c) * 65536, sW, 2 * kImgBytes);
                bulk_commit();
                mbar_arrive(&wready);
            }
        };
        emit();
        bool ok = !named_bar_or(1, 256, false);
        if (ok) publish(0);
        for (int c = 0; ok && c < cps; ++c) {
            // B_c row of this thread, read ahead of the product
            // (column quad q4 of row i at float4 q4 * 128 + i: a warp reads 512
            // contiguous bytes per load)
            const float4 *Bc = reinterpret_cast<const float4 *>(a.AB + (g0 + c) * kChunkWs + 2 * kImgBytes);
            float bv[64];
#pragma unroll
            for (int j4 = 0; j4 < 16; ++j4) {
                const float4 u = Bc[(col0 / 4 + j4) * kD + row];
                bv[4 * j4] = u.x;
                bv[4 * j4 + 1] = u.y;
                bv[4 * j4 + 2] = u.z;
                bv[4 * j4 + 3] = u.w;
            }
            bool got = mbar_wait(&dfull, c & 1, &abort_flag, a.status, 19);
            if (leader) bulk_wait_read();  // the image's last store has read it
            // every epilogue warp agrees before anyone moves on
            if (named_bar_or(1, 256, !__all_sync(0xffffffffu, got))) break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float v[16];
                tmem_ld16(taddr(tm, 32 * sp, col0 + 16 * q), v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) w[16 * q + e] = (w[16 * q + e] + bv[16 * q + e]) - v[e];
            }
            tc_fence_before();
            if (c + 1 < cps) emit();
            if (named_bar_or(1, 256, false)) break;
            if (c + 1 < cps) publish(c + 1);
        }
        if (leader) bulk_wait_all();
        if (ok && !abort_flag && a.W_out) {
            float *o = a.W_out + (size_t)seq * kD * kD + (size_t)row * kD + col0;
#pragma unroll
            for (int j4 = 0; j4 < 16; ++j4)
                *reinterpret_cast<float4 *>(o + 4 * j4) =
                    make_float4(w[4 * j4], w[4 * j4 + 1], w[4 * j4 + 2], w[4 * j4 + 3]);
        }
    }
    // Teardown: after an abort, let this block's own copies and MMAs land
    // before the shared memory and tensor memory are released.
    if (abort_flag) {
        if (warp == 0 && lane == 0)
            for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
                mbar_drain(&aready[c & 1], (c >> 1) & 1);
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 128);
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
    float *Z;  // bf16 instead when z_bf16
    int chunk;
    bool z_bf16;
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
            const size_t zbase = ((size_t)(row0 + (long)t * kApplyRows) + 32 * sp) * kD + 64 * half;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 2 * i + (lane >> 4), c = lane & 15;
                const float4 f = *reinterpret_cast<const float4 *>(stage + r * 64 + ((c ^ (r & 7)) << 2));
                store_z4(a.Z, a.z_bf16, zbase + (size_t)r * kD + 4 * c, f.x, f.y, f.z, f.w);
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
    chunk_scan_kernel<<<a.B * a.H, kScanThreads, kScanSmem, s>>>(
        ScanArgs{reinterpret_cast<const uint8_t *>(AB), a.W0, Wimg, a.W_out, a.H, cps, a.w0_per_seq, status});
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    chunk_apply_kernel<<<n, kApplyThreads, kApplySmem, s>>>(tmQ, ApplyArgs{Wimg, a.Z, a.chunk, a.z_bf16, status});
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

// Device address of g_chunk_scratch on the current device. In host code the
// symbol is only a handle, never an address a kernel may be given. The lookup
// allocates nothing and is repeated on every call, so an address is never
// carried over a device reset or a re-created context.
void *chunk_scratch_on_current_device() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_chunk_scratch) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return p;
}

}  // namespace

extern "C" ttt_status ttt_chunk_fwd_noalloc(const void *Q, const void *K, const void *V,
                                            const float *eta, const float *W0, void *Z,
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
