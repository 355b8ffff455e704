// ttt_chunk_bwd_tc.cu -- the large-chunk TTT backward on the tensor cores
// (d = 128, bf16 Q/K/V, fp32 dZ), three kernels in launch order:
//   cb_gram_tc_kernel   the per-chunk Gram products (below);
//   cb_scan_tc_kernel   the forward scan of W_c and the reverse scan of
//                       Om_{c+1} (further down);
//   cb_tok_tc_kernel<>  the per-token gradients in three passes (RP, DK, DQ).
//
// The per-chunk Gram products:
//   A_c = K_c^T diag(eta) K_c,   B_c = K_c^T diag(eta) V_c,   D_c = Q_c^T dZ_c
// ("Test-Time Training Done Right", abstract: the chunk's gradient step; the
// backward's recurrences use the same A_c, and D_c carries dZ into dL/dW_c),
// written per chunk into three d x d fp32 slots [A_c | B_c | D_c] in the
// layouts the tensor-core scan reads (A_c as bf16 hi and lo operand images,
// B_c and D_c as fp32 column quads; see the epilogue).
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
        // Epilogue: lane = d_in row i of the accumulators. The chunk's three
        // d x d slots take the scan's operand layouts: A_c as bf16 hi and lo
        // images (K-major, 128-byte swizzle, 32 KB each), B_c and D_c in fp32
        // with column quad q of row i at float4 q * 128 + i (so a 64-column
        // slice is 32 contiguous KB).
        if (__all_sync(0xffffffffu, mbar_wait(&done, 0, &abort_flag, a.status, 94))) {
            tc_fence_after();
            const int sp = warp & 3, i = 32 * sp + lane;
            const float scale = uniform ? eta0 : 1.f;
            float *slot = a.gram + (size_t)g * 3 * kD * kD;
            uint8_t *ahi = reinterpret_cast<uint8_t *>(slot), *alo = ahi + kD * kD * 2;
            float4 *ob = reinterpret_cast<float4 *>(slot + kD * kD);
            float4 *od = reinterpret_cast<float4 *>(slot + 2 * kD * kD);
#pragma unroll 1
            for (int q = 0; q < kD / 16; ++q) {
                float va[16], vb[16], dh[16], dl[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), va);
                tmem_ld16(taddr(tm, 32 * sp, 128 + 16 * q), vb);
                tmem_ld16(taddr(tm, 32 * sp, 256 + 16 * q), dh);
                tmem_ld16(taddr(tm, 32 * sp, 384 + 16 * q), dl);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float *x = va + 8 * h;
                    uint2 h0, l0, h1, l1;
                    split4(scale * x[0], scale * x[1], scale * x[2], scale * x[3], h0, l0);
                    split4(scale * x[4], scale * x[5], scale * x[6], scale * x[7], h1, l1);
                    const uint32_t o = off_kmajor_sw128(i, 16 * q + 8 * h, kD);
                    *reinterpret_cast<uint4 *>(ahi + o) = make_uint4(h0.x, h0.y, h1.x, h1.y);
                    *reinterpret_cast<uint4 *>(alo + o) = make_uint4(l0.x, l0.y, l1.x, l1.y);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ob[(4 * q + e) * kD + i] = make_float4(scale * vb[4 * e], scale * vb[4 * e + 1],
                                                           scale * vb[4 * e + 2], scale * vb[4 * e + 3]);
                    od[(4 * q + e) * kD + i] = make_float4(dh[4 * e] + dl[4 * e], dh[4 * e + 1] + dl[4 * e + 1],
                                                           dh[4 * e + 2] + dl[4 * e + 2],
                                                           dh[4 * e + 3] + dl[4 * e + 3]);
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

// ---------------------------------------------------------------------------
// The backward's two affine scans on the tensor cores (d = 128, slots in the
// layouts cb_gram_tc_kernel writes): per sequence
//   forward:  W_{c+1} = W_c - A_c W_c + B_c from W0, storing each W_c;
//   reverse:  Om_c = Om_{c+1} - A_c Om_{c+1} + D_c from dW_out (or 0),
//             storing each Om_{c+1}, and at the end dW0 = Om_0.
// A block per (sequence, direction, 64-column slice r): the columns of M
// evolve independently. One product per chunk, D = A_c [M_hi | M_lo] (M = 128
// rows i, N = 128: the slice's hi and lo terms side by side, K = 128), with
// A_c's hi and lo images as two instructions per K step, so each operand
// carries ~16 significant bits. The fp32 state is in the registers of four
// epilogue warps (row i = tensor-memory lane, 64 columns); they store it,
// form M - (D_hi + D_lo) + E_c and write the next slice image (K-major rows
// n: M_hi^T then M_lo^T). A_c's images and E_c's slice arrive by bulk copy,
// double-buffered, so a chunk's copies run while the previous product and
// update do.
constexpr int kScanThreads = 192;  // warp 0: copies, warp 1: MMA, warps 2-5: state
constexpr int kScanA = 2 * kD * kD * 2;            // A_c hi | lo images: 64 KB
constexpr int kScanE = kD * 64 * 4;                // E_c columns of the slice: 32 KB
constexpr int kScanImg = kD * kD * 2;              // slice image [M_hi^T | M_lo^T]: 32 KB
constexpr size_t kScanSmem = 1024 + 2 * kScanA + 2 * kScanE + kScanImg;  // 225 KB
static_assert(kScanSmem <= 232448, "shared memory budget");

struct ScanArgs {
    const float *W0, *dW_out, *gram;
    float *Wst, *Omst, *dW0_out;
    int H, NC;
    bool w0_per_seq;
    int *status;
};

__global__ void __launch_bounds__(kScanThreads, 1) cb_scan_tc_kernel(ScanArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem, *sE = smem + 2 * kScanA, *sW = sE + 2 * kScanE;
    __shared__ uint64_t aready[2], afree[2], eready[2], efree[2], dfull, wready, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.x, dir = blockIdx.y, j0 = 64 * blockIdx.z;
    const int NC = a.NC;
    const size_t dd = (size_t)kD * kD;
    auto chunk_of = [&](int st) { return (size_t)seq * NC + (dir == 0 ? st : NC - 1 - st); };
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&aready[b], 1);
            mbar_init(&afree[b], 1);
            mbar_init(&eready[b], 1);
            mbar_init(&efree[b], 4);  // one arrival per state warp
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
    int issued = 0;  // copy pairs issued

    if (warp == 0 && lane == 0) {
        for (int st = 0; st < NC; ++st) {
            const int b = st & 1;
            const float *slot = a.gram + chunk_of(st) * 3 * dd;
            if (st >= 2 && !mbar_wait(&afree[b], ((st >> 1) - 1) & 1, &abort_flag, a.status, 111)) break;
            mbar_arrive_expect_tx(&aready[b], kScanA);
            bulk_load(sA + b * kScanA, slot, kScanA, &aready[b]);
            if (st >= 2 && !mbar_wait(&efree[b], ((st >> 1) - 1) & 1, &abort_flag, a.status, 112)) {
                issued = 2 * st + 1;
                break;
            }
            mbar_arrive_expect_tx(&eready[b], kScanE);
            bulk_load(sE + b * kScanE, slot + (dir == 0 ? 1 : 2) * dd + (size_t)j0 * kD, kScanE, &eready[b]);
            issued = 2 * st + 2;
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = make_idesc_bf16(128, 128, false, false);
        const uint32_t wb = smem_u32(sW);
        for (int st = 0; st < NC; ++st) {
            const int b = st & 1;
            if (!mbar_wait(&aready[b], (st >> 1) & 1, &abort_flag, a.status, 113)) break;
            if (!mbar_wait(&wready, st & 1, &abort_flag, a.status, 114)) break;
            tc_fence_after();
            const uint32_t ab = smem_u32(sA + b * kScanA);
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
                const int k0 = 16 * k;
                const uint32_t o = (uint32_t)((k0 >> 6) * 16384 + (k0 & 63) * 2);
                const uint64_t bd = make_sdesc(wb + o, 16, 1024, kSw128);
                mma_bf16(tm, make_sdesc(ab + o, 16, 1024, kSw128), bd, idesc, k != 0);
                mma_bf16(tm, make_sdesc(ab + kScanA / 2 + o, 16, 1024, kSw128), bd, idesc, true);
            }
            mma_commit(&afree[b]);
            mma_commit(&dfull);
        }
    } else if (warp >= 2) {
        const int sp = warp & 3, row = 32 * sp + lane;
        float w[64];
        {
            const float *src = dir == 0 ? a.W0 + (size_t)(a.w0_per_seq ? seq : seq % a.H) * dd
                                        : (a.dW_out ? a.dW_out + (size_t)seq * dd : nullptr);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float4 u = src ? *reinterpret_cast<const float4 *>(src + (size_t)row * kD + j0 + 4 * q)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                w[4 * q] = u.x;
                w[4 * q + 1] = u.y;
                w[4 * q + 2] = u.z;
                w[4 * q + 3] = u.w;
            }
        }
        // this thread's column `row` of the slice image: K index row, rows n
        // (M_hi^T: n = jj, M_lo^T: n = 64 + jj)
        // (element (n, row) at off_kmajor_sw128(n, row, 128): a per-thread
        // base plus a per-n constant plus the swizzled 16-byte chunk)
        const uint32_t cb = (uint32_t)((row >> 6) * 16384 + (row & 7) * 2), rc = (uint32_t)((row & 63) >> 3);
        auto emit = [&]() {
#pragma unroll
            for (int jj = 0; jj < 64; ++jj) {
                __nv_bfloat16 hb, lb;
                split_bf16(w[jj], hb, lb);
                const uint32_t sw = (rc ^ (uint32_t)(jj & 7)) << 4;
                *reinterpret_cast<__nv_bfloat16 *>(sW + cb + (jj >> 3) * 1024 + (jj & 7) * 128 + sw) = hb;
                *reinterpret_cast<__nv_bfloat16 *>(sW + cb + 8192 + (jj >> 3) * 1024 + (jj & 7) * 128 + sw) = lb;
            }
            fence_async_smem();
        };
        emit();
        bool ok = !named_bar_or(1, 128, false);
        if (ok && warp == 2 && lane == 0) mbar_arrive(&wready);
        for (int st = 0; ok && st < NC; ++st) {
            const int b = st & 1;
            const size_t g = chunk_of(st);
            // the state entering the chunk: W_c (forward) or Om_{c+1} (reverse)
            float *o = (dir == 0 ? a.Wst : a.Omst) + g * dd + (size_t)row * kD + j0;
#pragma unroll
            for (int q = 0; q < 16; ++q)
                *reinterpret_cast<float4 *>(o + 4 * q) = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            bool got = mbar_wait(&eready[b], (st >> 1) & 1, &abort_flag, a.status, 115);
            got = got && mbar_wait(&dfull, st & 1, &abort_flag, a.status, 116);
            if (named_bar_or(1, 128, !__all_sync(0xffffffffu, got))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float4 *E = reinterpret_cast<const float4 *>(sE + b * kScanE);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float dh[16], dl[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), dh);
                tmem_ld16(taddr(tm, 32 * sp, 64 + 16 * q), dl);
                float ev[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 f = E[(4 * q + u) * kD + row];
                    ev[4 * u] = f.x;
                    ev[4 * u + 1] = f.y;
                    ev[4 * u + 2] = f.z;
                    ev[4 * u + 3] = f.w;
                }
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) w[16 * q + e] = w[16 * q + e] + ev[e] - (dh[e] + dl[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&efree[b]);  // this warp has read E_c
            if (st + 1 < NC) emit();                // the product of this chunk is done with the image
            if (named_bar_or(1, 128, false)) {
                ok = false;
                break;
            }
            if (st + 1 < NC && warp == 2 && lane == 0) mbar_arrive(&wready);
        }
        if (ok && !abort_flag && dir == 1) {
            float *o = a.dW0_out + (size_t)seq * dd + (size_t)row * kD + j0;
#pragma unroll
            for (int q = 0; q < 16; ++q)
                *reinterpret_cast<float4 *>(o + 4 * q) = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
    }
    // Teardown: after an abort, let this block's own copies and MMAs land
    // before the shared memory and tensor memory are released.
    if (abort_flag) {
        if (warp == 0 && lane == 0 && issued > 0) {
            // the copies of the last two chunks may both be in flight (one
            // per buffer): wait for each (a phase already complete returns)
            const int last = (issued - 1) / 2;  // the last chunk whose copies were issued
            for (int st = last > 0 ? last - 1 : 0; st <= last; ++st) {
                mbar_drain(&aready[st & 1], (st >> 1) & 1);
                if (st < last || issued % 2 == 0) mbar_drain(&eready[st & 1], (st >> 1) & 1);
            }
        }
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 128);
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
    GramArgs ga{eta, gram, chunk, device_status_word()};
    cb_gram_tc_kernel<<<nch, kThreads, kSmem, s>>>(tmK, tmV, tmQ, tmZ, ga);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

// The two scans of the backward on the tensor cores, after
// launch_chunk_bwd_gram_tc: W_c into Wst, Om_{c+1} into Omst (per chunk
// [d][d] fp32, row-major), dW0 = Om_0 of each sequence into dW0_out.
cudaError_t launch_chunk_bwd_scan_tc(const float *W0, const float *dW_out, const float *gram,
                                     float *Wst, float *Omst, float *dW0_out, int S, int H, int NC,
                                     bool w0_per_seq, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(cb_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kScanSmem);
    if (e != cudaSuccess) return e;
    ScanArgs sa{W0, dW_out, gram, Wst, Omst, dW0_out, H, NC, w0_per_seq, device_status_word()};
    cb_scan_tc_kernel<<<dim3((unsigned)S, 2, kD / 64), kScanThreads, kScanSmem, s>>>(sa);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}


// ---------------------------------------------------------------------------
// Per-token gradients of the large-chunk backward on the tensor cores (d =
// 128, bf16 inputs, chunk a multiple of 128), with W = W_c and Om = Om_{c+1}
// of each token's chunk:
//   R = K W - V,  P = K Om,  dV = diag(eta) P,  deta_t = -P_t . R_t,
//   dK = -diag(eta) (R Om^T + P W^T) = -diag(eta) (K S - V Om^T),
//       with S = W Om^T + Om W^T (one d x d matrix per chunk),
//   dQ = dZ W^T,
// as three passes of one kernel over 128-token tiles, a block per chunk:
//   RP: D = K [W | Om] (N = 256, K = d_in): A = K (exact), B = [W | Om]^T as
//       hi and lo terms; the epilogue forms R, dV and deta. Before its tiles
//       the block also forms S from the same two B images (S[i][j] = sum over
//       the 256 rows n of B[n][i] B[n +- 128][j]: both operands MN-major
//       views of the images, hi.hi + hi.lo + lo.hi) and stores it in fp32;
//   DK: D = [K | V] [S ; -Om^T] (K = 256, A exact); DQ: D = dZ_{hi,lo} W^T
//       (K = 128): B stacked as [hi rows | lo rows] (N = 256), so A x B gives
//       the hi and lo terms side by side (and, for DQ, A_lo x B_hi adds lo.hi
//       to the first half).
// So no per-token intermediate crosses HBM between the passes (dZ's bf16
// rows come from the Gram kernel, which splits dZ anyway). A tiles arrive by
// TMA one 64-wide K block at a time; B is built once per block in shared
// memory from fp32 (K-major, 128-byte swizzle); accumulators double-buffered
// in tensor memory.
namespace {

enum { kModeRP = 0, kModeDK = 1, kModeDQ = 2 };
constexpr int kTokTile = 128, kTokThreads = 192, kTokStages = 3;
constexpr int kTokStage = 2 * kTokTile * 128;            // A hi | lo for one 64-wide K block: 32 KB
constexpr int kTokBBytes = 4 * 2 * kD * 128;             // up to 4 K blocks x 256 rows: 128 KB
constexpr size_t kTokSmem = 1024 + kTokBBytes + kTokStages * kTokStage;  // 225 KB
static_assert(kTokSmem <= 232448, "shared memory budget");

struct TokArgs {
    const float *W, *Om;  // per chunk [d][d] fp32, row-major [i][j]
    const __nv_bfloat16 *V;
    const float *eta, *dZ;
    float *out;           // RP: dV; DK: dK; DQ: dQ   ([tokens][d] fp32)
    float *deta;          // RP only
    float *S;             // chunk g's S at S + g * s_stride (RP writes, DK reads)
    size_t s_stride;
    int chunk;
    int *status;
};

// Byte offset of element (n, k) in a K-major, 128-byte-swizzled image of
// `rows` rows per 64-wide K block.
__device__ __forceinline__ uint32_t kmajor_off(int n, int k, int rows) {
    return (uint32_t)((k >> 6) * rows * 128 + n * 128 + ((((k & 63) >> 3) ^ (n & 7)) << 4) + (k & 7) * 2);
}

// A warp's 32 token rows written through padded shared memory (16-byte
// accesses conflict-free) so that global memory sees whole row segments:
// lane l holds row l's NP consecutive 16-byte pieces.
constexpr int kStgWarp = 32 * (8 * 16 + 16);  // staging per warp: 32 rows of up to 128 bytes
template <int NP>
__device__ __forceinline__ void warp_rows_out(uint8_t *stg, const uint4 (&v)[NP], uint8_t *g0,
                                              size_t pitch, int lane) {
    constexpr int SP = NP * 16 + 16, RPI = 32 / NP;
#pragma unroll
    for (int i = 0; i < NP; ++i) *reinterpret_cast<uint4 *>(stg + lane * SP + 16 * i) = v[i];
    __syncwarp();
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int row = k * RPI + lane / NP, pc = lane % NP;
        *reinterpret_cast<uint4 *>(g0 + (size_t)row * pitch + 16 * pc) =
            *reinterpret_cast<const uint4 *>(stg + row * SP + 16 * pc);
    }
    __syncwarp();
}
__device__ __forceinline__ uint4 pack4f(float a, float b, float c, float d) {
    return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c), __float_as_uint(d));
}

// Threads of a token pass: DQ adds four warps that split dZ (fp32, by TMA)
// into the bf16 hi and lo operand images.
__host__ __device__ constexpr int tok_threads(int mode) { return mode == kModeDQ ? 320 : kTokThreads; }

template <int kMode>
__global__ void __launch_bounds__(tok_threads(kMode), 1)
    cb_tok_tc_kernel(const __grid_constant__ CUtensorMap tmA_hi, const __grid_constant__ CUtensorMap tmA_lo,
                     TokArgs a) {
    constexpr int KD = kMode == kModeDK ? 2 * kD : kD;  // reduction length
    constexpr int NKB = KD / 64;                         // 64-wide K blocks per tile
    constexpr bool kTwoA = kMode == kModeDQ;             // A as hi and lo terms
    // B image rows per K block: RP keeps hi and lo as two images of 256 rows
    // ([W | Om]^T); DK and DQ stack [hi rows | lo rows] of their 128 rows.
    constexpr int BR = 2 * kD;
    constexpr uint32_t kBLoOff = kMode == kModeRP ? (uint32_t)NKB * BR * 128 : 0u;
    // A ring: one term of a 64-wide K block per stage (DK: the K blocks of K,
    // then of V); DQ: dZ's fp32 K block (two 32-column boxes) per stage, and
    // two buffers for the bf16 hi and lo images, which the converter warps
    // fill once the product two K blocks before has read them.
    constexpr int STAGES = kMode == kModeDK ? 4 : kMode == kModeDQ ? 2 : 3;
    constexpr int SBYTES = kTwoA ? kTokStage : kTokStage / 2;
    constexpr int ABUF = kTwoA ? 2 * kTokStage : 0;  // DQ's bf16 images, after the ring
    constexpr int BBYTES = NKB * BR * 128 * (kMode == kModeRP ? 2 : 1);  // B images
    static_assert(BBYTES + STAGES * SBYTES + ABUF + 4 * kStgWarp + 1024 <= (int)kTokSmem, "smem plan");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = smem, *sA = smem + BBYTES;
    __shared__ uint64_t full[4], empty[4], bready, tfull[2], tempty[2], sfull, sfree, conv[2], aempty[2], drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;
    const long row0 = (long)g * a.chunk;
    const int ntile = a.chunk / kTokTile;
    const size_t dd = (size_t)kD * kD;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMode == kModeDQ ? 128 : 1);  // DQ: the converters free a stage
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&conv[b], 128);
            mbar_init(&aempty[b], 1);
        }
        mbar_init(&bready, 128);
        mbar_init(&sfull, 1);
        mbar_init(&sfree, 128);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 128);
        }
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    int issued = 0;

    if (warp == 0 && lane == 0) {
        // A tiles, one K block per stage
        for (int t = 0, u = 0; t < ntile; ++t) {
            for (int kb = 0; kb < NKB; ++kb, ++u) {
                const int st = u % STAGES;
                if (u >= STAGES &&
                    !mbar_wait(&empty[st], ((u / STAGES) - 1) & 1, &abort_flag, a.status, 101))
                    goto producer_done;
                uint8_t *sb = sA + st * SBYTES;
                const int y = (int)(row0 + (long)t * kTokTile);
                if (kMode == kModeDQ) {  // dZ fp32: two 32-column boxes
                    mbar_arrive_expect_tx(&full[st], SBYTES);
                    tma_load_2d(sb, &tmA_hi, 64 * kb, y, &full[st]);
                    tma_load_2d(sb + SBYTES / 2, &tmA_hi, 64 * kb + 32, y, &full[st]);
                } else {
                    mbar_arrive_expect_tx(&full[st], SBYTES);
                    if (kMode == kModeDK)  // [K | V]: K blocks 0-1 of K, 2-3 of V
                        tma_load_2d(sb, kb < 2 ? &tmA_hi : &tmA_lo, 64 * (kb & 1), y, &full[st]);
                    else
                        tma_load_2d(sb, &tmA_hi, 64 * kb, y, &full[st]);
                }
                issued = u + 1;
            }
        }
    producer_done:;
    } else if (warp == 1 && lane == 0) {
        const uint32_t id256 = make_idesc_bf16(128, 256, false, false);
        const uint32_t id128 = make_idesc_bf16(128, 128, false, false);
        const uint32_t bb = smem_u32(sB), ab = smem_u32(sA);
        if (mbar_wait(&bready, 0, &abort_flag, a.status, 102)) {
            if (kMode == kModeRP) {
                // S = W Om^T + Om W^T into columns 256-383 (the second
                // accumulator, free until tile 1): row n of the image
                // holds W[n][.] (n < 128) or Om[n - 128][.], so
                // S[i][j] = sum_n img[n][i] img[(n + 128) % 256][j]; both
                // operands are MN-major views (64-value blocks 32 KB apart,
                // 8-row groups 1 KB apart), 16 rows n per instruction.
                const uint32_t ids = make_idesc_bf16(128, 128, true, true);
                constexpr uint32_t kBlk = (uint32_t)BR * 128;
                for (int n0 = 0, first = 1; n0 < 2 * kD; n0 += 16) {
                    const uint32_t ra = (uint32_t)n0 * 128, rb = (uint32_t)((n0 + kD) % (2 * kD)) * 128;
                    const uint64_t ah = make_sdesc(bb + ra, kBlk, 1024, kSw128);
                    const uint64_t al = make_sdesc(bb + kBLoOff + ra, kBlk, 1024, kSw128);
                    const uint64_t bh = make_sdesc(bb + rb, kBlk, 1024, kSw128);
                    const uint64_t bl = make_sdesc(bb + kBLoOff + rb, kBlk, 1024, kSw128);
                    mma_bf16(tm + 256, ah, bh, ids, !first);
                    mma_bf16(tm + 256, ah, bl, ids, true);
                    mma_bf16(tm + 256, al, bh, ids, true);
                    first = 0;
                }
                mma_commit(&sfull);
            }
            for (int t = 0, u = 0; t < ntile; ++t) {
                const int acc = t & 1;
                if (t >= 2 && !mbar_wait(&tempty[acc], ((t >> 1) - 1) & 1, &abort_flag, a.status, 103))
                    break;
                if (kMode == kModeRP && t == 1 && !mbar_wait(&sfree, 0, &abort_flag, a.status, 106))
                    break;
                tc_fence_after();
                const uint32_t d = tm + 256 * acc;
                bool ok = true;
                for (int kb = 0; kb < NKB; ++kb, ++u) {
                    const int st = u % STAGES;
                    if (!mbar_wait(kMode == kModeDQ ? &conv[u & 1] : &full[st],
                                   kMode == kModeDQ ? ((u >> 1) & 1) : ((u / STAGES) & 1), &abort_flag,
                                   a.status, 104)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 =
                        kMode == kModeDQ ? ab + STAGES * SBYTES + (u & 1) * kTokStage : ab + st * SBYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t ko = (uint32_t)(16 * k * 2);
                        const uint64_t ahi = make_sdesc(a0 + ko, 16, 1024, kSw128);
                        const uint64_t bhi = make_sdesc(bb + kb * BR * 128 + ko, 16, 1024, kSw128);
                        const bool accum = (kb | k) != 0;
                        if (kMode == kModeRP) {
                            const uint64_t blo = make_sdesc(bb + kBLoOff + kb * BR * 128 + ko, 16, 1024, kSw128);
                            mma_bf16(d, ahi, bhi, id256, accum);
                            mma_bf16(d, ahi, blo, id256, true);
                        } else if (kTwoA) {
                            const uint64_t alo = make_sdesc(a0 + kTokStage / 2 + ko, 16, 1024, kSw128);
                            mma_bf16(d, ahi, bhi, id256, accum);  // hi.hi | hi.lo
                            mma_bf16(d, alo, bhi, id128, true);   // + lo.hi (first half)
                        } else {
                            mma_bf16(d, ahi, bhi, id256, accum);  // A.hi | A.lo
                        }
                    }
                    mma_commit(kMode == kModeDQ ? &aempty[u & 1] : &empty[st]);
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
            }
        }
    } else if (kMode == kModeDQ && warp >= 6) {
        // Converters: dZ (fp32 boxes of 32 columns, 128-byte swizzle) -> the
        // K block's bf16 hi and lo images (K-major, 128-byte swizzle). A unit
        // is 8 columns of one token row; 16-byte chunk c of row r at c ^ (r & 7).
        const int tc = threadIdx.x - 192;  // 0..127
        for (int t = 0, u = 0; t < ntile; ++t) {
            bool ok = true;
            for (int kb = 0; kb < NKB; ++kb, ++u) {
                const int st = u % STAGES;
                bool got = mbar_wait(&full[st], (u / STAGES) & 1, &abort_flag, a.status, 108);
                // image buffer u & 1: read by the product of K block u - 2
                got = got && (u < 2 || mbar_wait(&aempty[u & 1], ((u >> 1) - 1) & 1, &abort_flag, a.status, 109));
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t *sb = sA + st * SBYTES;
                uint4 hi[8], lo[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int un = tc + 128 * k, row = un >> 3, c8 = un & 7, sw = row & 7;
                    const uint8_t *zr = sb + (c8 >> 2) * (SBYTES / 2) + row * 128;
                    const int c32 = (c8 & 3) * 2;  // the unit's first 16-byte chunk in its box row
                    const float4 z0 = *reinterpret_cast<const float4 *>(zr + ((c32 ^ sw) << 4));
                    const float4 z1 = *reinterpret_cast<const float4 *>(zr + (((c32 + 1) ^ sw) << 4));
                    uint2 h0, l0, h1, l1;
                    split4(z0.x, z0.y, z0.z, z0.w, h0, l0);
                    split4(z1.x, z1.y, z1.z, z1.w, h1, l1);
                    hi[k] = make_uint4(h0.x, h0.y, h1.x, h1.y);
                    lo[k] = make_uint4(l0.x, l0.y, l1.x, l1.y);
                }
                mbar_arrive(&empty[st]);  // the fp32 stage is read: the producer may refill it
                uint8_t *abuf = sA + STAGES * SBYTES + (u & 1) * kTokStage;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int un = tc + 128 * k, row = un >> 3, c8 = un & 7;
                    const int off = row * 128 + ((c8 ^ (row & 7)) << 4);
                    *reinterpret_cast<uint4 *>(abuf + off) = hi[k];
                    *reinterpret_cast<uint4 *>(abuf + kTokStage / 2 + off) = lo[k];
                }
                fence_async_smem();
                mbar_arrive(&conv[u & 1]);
            }
            if (!ok) break;
        }
    } else if (warp >= 2) {
        const int tt = threadIdx.x - 64;  // 0..127
        // ---- B operand images from the fp32 W and Om of the chunk
        {
            const float *Wc = a.W + (size_t)g * dd, *Oc = a.Om + (size_t)g * dd;
            const float *Sc = a.S + (size_t)g * a.s_stride;
            // units: (row n, 8 consecutive k), NU per thread, loaded UB units
            // at a time before any is converted (so UB x 8 loads are in flight)
            constexpr int NROWS = kMode == kModeRP ? 2 * kD : kD;
            constexpr int NU = NROWS * (KD / 8) / 128, UB = 8;
            static_assert(NU % UB == 0, "whole batches");
            constexpr bool kColRead = kMode != kModeDQ;  // consecutive threads take consecutive n
            // Column reads (RP's W and Om, DK's S) go with consecutive threads
            // on consecutive n (one 128-byte row segment per warp load); row
            // reads with consecutive k
            auto unit_n = [&](int uidx) { return kColRead ? uidx % NROWS : uidx / (KD / 8); };
            auto unit_k0 = [&](int uidx) { return kColRead ? 8 * (uidx / NROWS) : 8 * (uidx % (KD / 8)); };
#pragma unroll 1
            for (int b0 = 0; b0 < NU; b0 += UB) {
                float f[UB][8];
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    const int uidx = tt + 128 * (b0 + j), n = unit_n(uidx), k0 = unit_k0(uidx);
                    if (kMode == kModeRP || (kMode == kModeDK && k0 < kD)) {
                        // RP: B[n][k] = W[k][n] (n < 128) or Om[k][n - 128] (K = d_in);
                        // DK, k < 128: B[n][k] = S[k][n]
                        const float *src = kMode == kModeDK ? Sc + n : (n < kD ? Wc + n : Oc + (n - kD));
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[j][e] = src[(size_t)(k0 + e) * kD];
                    } else {
                        // DK, k >= 128: B[n][k] = -Om[n][k - 128]; DQ: B[n][k] = W[n][k]
                        const float *src = (kMode == kModeDK ? Oc : Wc) + (size_t)n * kD + (k0 & (kD - 1));
                        const float sg = kMode == kModeDK ? -1.f : 1.f;
                        const float4 u0 = *reinterpret_cast<const float4 *>(src);
                        const float4 u1 = *reinterpret_cast<const float4 *>(src + 4);
                        f[j][0] = sg * u0.x; f[j][1] = sg * u0.y; f[j][2] = sg * u0.z; f[j][3] = sg * u0.w;
                        f[j][4] = sg * u1.x; f[j][5] = sg * u1.y; f[j][6] = sg * u1.z; f[j][7] = sg * u1.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    const int uidx = tt + 128 * (b0 + j), n = unit_n(uidx), k0 = unit_k0(uidx);
                    uint2 h0, l0, h1, l1;
                    split4(f[j][0], f[j][1], f[j][2], f[j][3], h0, l0);
                    split4(f[j][4], f[j][5], f[j][6], f[j][7], h1, l1);
                    if (kMode == kModeRP) {
                        const uint32_t o = kmajor_off(n, k0, BR);
                        *reinterpret_cast<uint4 *>(sB + o) = make_uint4(h0.x, h0.y, h1.x, h1.y);
                        *reinterpret_cast<uint4 *>(sB + kBLoOff + o) = make_uint4(l0.x, l0.y, l1.x, l1.y);
                    } else {
                        *reinterpret_cast<uint4 *>(sB + kmajor_off(n, k0, BR)) = make_uint4(h0.x, h0.y, h1.x, h1.y);
                        *reinterpret_cast<uint4 *>(sB + kmajor_off(kD + n, k0, BR)) =
                            make_uint4(l0.x, l0.y, l1.x, l1.y);
                    }
                }
            }
            fence_async_smem();
            mbar_arrive(&bready);
        }
        // ---- epilogue: lane = token row of the tile; every global row access
        // goes through the warp's staging rows (whole row segments)
        const int sp = warp & 3;
        uint8_t *stg = sA + STAGES * SBYTES + ABUF + (warp - 2) * kStgWarp;
        bool run = true;
        if (kMode == kModeRP) {
            // S: lane = row i, 128 fp32 columns from tensor memory
            run = __all_sync(0xffffffffu, mbar_wait(&sfull, 0, &abort_flag, a.status, 107));
            if (run) {
                tc_fence_after();
                uint8_t *s0 = reinterpret_cast<uint8_t *>(a.S + (size_t)g * a.s_stride + (size_t)32 * sp * kD);
#pragma unroll 1
                for (int q = 0; q < kD / 32; ++q) {
                    float x[32];
                    tmem_ld16(taddr(tm, 32 * sp, 256 + 32 * q), *reinterpret_cast<float(*)[16]>(&x[0]));
                    tmem_ld16(taddr(tm, 32 * sp, 256 + 32 * q + 16), *reinterpret_cast<float(*)[16]>(&x[16]));
                    tmem_ld_wait();
                    uint4 o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o8[e] = pack4f(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    warp_rows_out<8>(stg, o8, s0 + 128 * q, 4 * kD, lane);
                }
                tc_fence_before();
                mbar_arrive(&sfree);  // columns 256-383 are free for tile 1
            }
        }
        for (int t = 0; run && t < ntile; ++t) {
            const int acc = t & 1;
            const long tokw = row0 + (long)t * kTokTile + 32 * sp;  // the warp's first token
            const long tok = tokw + lane;
            const float et = a.eta[tok];
            // RP: the token's V row (256 B) loads while the tile's products run
            uint4 vr[kMode == kModeRP ? kD / 8 : 1];
            if (kMode == kModeRP) {
                const uint4 *vq = reinterpret_cast<const uint4 *>(a.V + tok * kD);
#pragma unroll
                for (int q = 0; q < kD / 8; ++q) vr[q] = vq[q];
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (t >> 1) & 1, &abort_flag, a.status, 105)))
                break;
            tc_fence_after();
            const uint32_t dcol = 256 * acc;
            if (kMode == kModeRP) {
                // A thread per token row; its output rows leave through the warp's
                // staging rows as whole segments (32 columns a round).
                float de = 0.f;
#pragma unroll
                for (int q = 0; q < kD / 32; ++q) {
                    float r[32], p[32];
                    tmem_ld16(taddr(tm, 32 * sp, dcol + 32 * q), *reinterpret_cast<float(*)[16]>(&r[0]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + 32 * q + 16), *reinterpret_cast<float(*)[16]>(&r[16]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + kD + 32 * q), *reinterpret_cast<float(*)[16]>(&p[0]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + kD + 32 * q + 16), *reinterpret_cast<float(*)[16]>(&p[16]));
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const __nv_bfloat162 *vh = reinterpret_cast<const __nv_bfloat162 *>(&vr[4 * q + c]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = __bfloat1622float2(vh[e]);
                            r[8 * c + 2 * e] -= x.x;
                            r[8 * c + 2 * e + 1] -= x.y;
                        }
                    }
                    uint4 o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        o8[e] = pack4f(et * p[4 * e], et * p[4 * e + 1], et * p[4 * e + 2], et * p[4 * e + 3]);
                        de = fmaf(p[4 * e], r[4 * e], de);
                        de = fmaf(p[4 * e + 1], r[4 * e + 1], de);
                        de = fmaf(p[4 * e + 2], r[4 * e + 2], de);
                        de = fmaf(p[4 * e + 3], r[4 * e + 3], de);
                    }
                    warp_rows_out<8>(stg, o8, reinterpret_cast<uint8_t *>(a.out + tokw * kD + 32 * q),
                                     4 * kD, lane);  // dV
                }
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
                a.deta[tok] = -de;
            } else {
                const float sc = kMode == kModeDK ? -et : 1.f;
#pragma unroll 1
                for (int q = 0; q < kD / 32; ++q) {
                    float x[32], y[32];
                    tmem_ld16(taddr(tm, 32 * sp, dcol + 32 * q), *reinterpret_cast<float(*)[16]>(&x[0]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + 32 * q + 16), *reinterpret_cast<float(*)[16]>(&x[16]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + kD + 32 * q), *reinterpret_cast<float(*)[16]>(&y[0]));
                    tmem_ld16(taddr(tm, 32 * sp, dcol + kD + 32 * q + 16), *reinterpret_cast<float(*)[16]>(&y[16]));
                    tmem_ld_wait();
                    if (q == kD / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(&tempty[acc]);  // the accumulator is read
                    }
                    uint4 o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o8[e] = pack4f(sc * (x[4 * e] + y[4 * e]), sc * (x[4 * e + 1] + y[4 * e + 1]),
                                       sc * (x[4 * e + 2] + y[4 * e + 2]), sc * (x[4 * e + 3] + y[4 * e + 3]));
                    warp_rows_out<8>(stg, o8, reinterpret_cast<uint8_t *>(a.out + tokw * kD + 32 * q),
                                     4 * kD, lane);
                }
            }
        }
    }
    if (abort_flag) {
        if (warp == 0 && lane == 0)
            for (int u = issued - STAGES < 0 ? 0 : issued - STAGES; u < issued; ++u)
                mbar_drain(&full[u % STAGES], (u / STAGES) & 1);
        if (warp == 1 && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 512);
}

template <int kMode>
cudaError_t launch_tok_mode(const CUtensorMap &hi, const CUtensorMap &lo, const TokArgs &a, int nch,
                            cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(cb_tok_tc_kernel<kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTokSmem);
    if (e != cudaSuccess) return e;
    cb_tok_tc_kernel<kMode><<<nch, tok_threads(kMode), kTokSmem, s>>>(hi, lo, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

}  // namespace

bool chunk_bwd_tok_tc_supported(int d, int chunk, bool bf16) {
    return bf16 && d == kD && chunk >= kTokTile && chunk % kTokTile == 0;
}

// S of chunk g goes to S + g * s_stride floats (the caller's d x d slot per
// chunk, free once the scans have run). The token passes need no other
// workspace: DQ splits dZ into its bf16 terms on chip.
cudaError_t launch_chunk_bwd_tok_tc(const void *K, const void *V, const float *eta, const float *dZ,
                                    const float *W, const float *Om, float *S, size_t s_stride,
                                    int B, int H, int T, int chunk, float *dQ, float *dK, float *dV,
                                    float *deta, cudaStream_t s) {
    const uint64_t rows = (uint64_t)B * H * T;
    const int nch = B * H * (T / chunk);
    int *status = device_status_word();
    alignas(64) CUtensorMap tmK, tmV, tmZ;
    if (!encode_tmap_2d(&tmK, K, false, kD, rows, 64, kTokTile) ||
        !encode_tmap_2d(&tmV, V, false, kD, rows, 64, kTokTile) ||
        !encode_tmap_2d(&tmZ, dZ, true, kD, rows, 32, kTokTile))
        return cudaErrorInvalidValue;
    TokArgs a{W, Om, static_cast<const __nv_bfloat16 *>(V), eta, dZ, dV, deta, S, s_stride,
              chunk, status};
    cudaError_t e = launch_tok_mode<kModeRP>(tmK, tmK, a, nch, s);
    if (e != cudaSuccess) return e;
    a.out = dK;
    if ((e = launch_tok_mode<kModeDK>(tmK, tmV, a, nch, s)) != cudaSuccess) return e;
    a.out = dQ;
    return launch_tok_mode<kModeDQ>(tmZ, tmZ, a, nch, s);
}

}  // namespace ttt
