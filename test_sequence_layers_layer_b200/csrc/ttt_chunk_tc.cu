// ttt_chunk_tc.cu -- large-chunk TTT (apply-then-update) on the tensor cores.
//
// Method ("Test-Time Training Done Right", abstract: large chunks; the chunk
// rule itself is the TTT update of "Test-Time Training: Linear Complexity
// Beyond Attention", Key Architectural Mechanics part 2): every token of
// chunk c reads out with W_c, then
//   W_{c+1} = W_c - sum_{s in c} eta_s k_s^T (k_s W_c - v_s)
//           = W_c - A_c W_c + B_c,   A_c = K_c^T diag(eta) K_c,  B_c = K_c^T diag(eta) V_c.
// The update is affine in W, so the work splits into three block roles of
// one launch, taken in start order (a ticket counter), each waiting only on
// blocks that started before it:
//   gram:     A_c | B_c for every chunk of every sequence (the only pass over
//             K and V; tcgen05, M = d_in = 128, N = 256, K = tokens), each
//             chunk published by a ready flag;
//   scan:     W_{c+1} = W_c - A_c W_c + B_c, one step per chunk, split by
//             64-column slices of W over 2 blocks per sequence (columns evolve
//             independently; tcgen05, M = 128, N = 128 = the slice's hi and lo
//             terms, K = 128; state and update in fp32), each step as soon as
//             its chunk is published, writing each W_c as the ready-made bf16
//             hi/lo operand image of the read-out;
//   read-out: Z_c = Q_c W_c once both slices of W_c are written (the only
//             pass over Q and the only write of Z), as Z_c^T = W_c^T Q_c^T on
//             tcgen05: M = d_out = 128 with W_c^T (hi and lo terms) as the A
//             operand in tensor memory, N = 128 tokens per tile, K = d_in.
//             Their HBM traffic overlaps the Gram's.
// Q/K/V tiles arrive by TMA with the 128-byte swizzle; accumulators live in
// tensor memory. W_c enters the read-out as two bf16 terms (hi + lo) so it
// keeps ~16 significant bits of the fp32 state.

#include <algorithm>

#include "../../include/ttt.h"
#include "sm100.cuh"
#include "ttt_common.cuh"

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: math/epilogue

// Workspace per chunk: A_c as a bf16 operand image (K-major, 32 KB; the scan
// takes A_c's rounded-to-nearest bf16 term only) and B_c in fp32 (64 KB;
// column quad q of row i at float4 q * 128 + i); after all chunks, each W_c
// as the read-out's bf16 hi | lo image (64 KB, layout at the read-out role);
// then the ticket counter, the chunks' ready flags and read-out counts.
constexpr int kImgBytes = kD * kD * 2;            // one bf16 128 x 128 image
constexpr int kChunkWs = kImgBytes + kD * kD * 4;

// ---------------------------------------------------------------------------
// One launch, three block roles by ticket (a counter in the workspace;
// tickets follow the order in which blocks start):
//   tickets [0, n): Gram of one chunk, chunk-major (chunk 0 of every sequence
//     first): A_c | B_c = (diag(eta) K_c)^T [K_c | V_c], then a ready flag;
//   next 2 per sequence (4 in map mode): scan of one 64-column slice of one
//     sequence's weight, W_{c+1}[:, j] = W_c[:, j] - A_c W_c[:, j] + B_c[:, j]
//     (columns of W evolve independently), waiting on each chunk's flag;
//   the rest (forward only): read-out of part of one chunk, waiting on the
//     count of scan slices that have stored W_c.
// Every wait is on blocks with smaller tickets, which have started and wait
// only on blocks before them, so the waits always end.
constexpr int kGramRows = 64;                    // tokens per pipeline stage
constexpr int kGramStages = 2;
constexpr int kGramBox = kGramRows * 128;        // one 64-column box of a stage (8 KB)
constexpr int kGramStageBytes = 6 * kGramBox;    // K (2 boxes) | V (2) | eta*K (2)
constexpr size_t kGramSmem = 1024 + kGramStages * kGramStageBytes;  // 97 KB: two blocks per SM
// With one step size for the whole chunk, K itself is the A operand (no eta*K
// copy, no conversion pass) and the accumulator is scaled by eta once: the
// same 96 KB then hold 3 stages of K | V.
constexpr int kGramStagesU = 3, kGramStageBytesU = 4 * kGramBox;
static_assert(kGramStagesU * kGramStageBytesU <= kGramStages * kGramStageBytes, "uniform-eta ring");
constexpr int kSlice = 64, kSlices = kD / kSlice;  // scan: output columns per block
constexpr int kSliceImg = 2 * kSlice * kD * 2;     // [W hi | W lo] slice image [128][128] bf16: 32 KB
static_assert(2 * kImgBytes / 2 + kSliceImg + 1024 <= (int)kGramSmem, "scan role fits the gram's smem");

// Ready flags and the ticket counter sit after the per-chunk workspace.
__host__ __device__ constexpr size_t sync_offset(size_t n) { return n * ((size_t)kChunkWs + 65536); }
// [0]: ticket counter, [1 + g]: chunk g's Gram published, [1 + n + g]: the
// number of scan blocks that have written their columns of W_g's read-out image.
__host__ __device__ constexpr size_t sync_bytes(size_t n) { return ((2 * n + 1) * 4 + 255) / 256 * 256; }

struct GramScanArgs {
    const float *eta;
    uint8_t *ws;        // per chunk: A_c hi | lo image, B_c fp32; then W_c images; then sync
    const float *W0;
    float *W_out;
    int chunk, H, nseq, cps;
    bool w0_per_seq;
    int *status;
    // Map mode: no read-out; the scan runs the map W -> M W + N of the whole
    // sequence instead of the forward: M from W = I without B_c, N from
    // W = 0 with B_c, 4 slices per sequence (M's two, then N's two).
    float *M = nullptr, *N = nullptr;
    // Forward: the read-out's output (bf16 instead when z_bf16) and the
    // number of read-out blocks per chunk (each takes chunk / parts tokens, a
    // multiple of 128); the last chunk of each sequence, read last, is split
    // over parts_last blocks.
    float *Z = nullptr;
    bool z_bf16 = false;
    int parts = 1, parts_last = 1;
};

// Read-out blocks per chunk, for n chunks: about 1024 read-out blocks in all
// (3.5 waves of the 296 resident blocks: enough to keep HBM busy while the
// last chunks wait for the scan, few enough that each block's W_c set-up is
// spread over several tiles), at least two 128-token tiles per block, and a
// divisor of the chunk's tiles.
int readout_parts(int chunk, int n) {
    int want = n >= 1024 ? 1 : 1024 / n;
    want = std::min(want, std::max(1, chunk / 256));
    for (int p = want; p > 1; --p)
        if ((chunk / 128) % p == 0) return p;
    return 1;
}

// The last chunk's read-outs are the kernel's tail, run while fewer and
// fewer blocks are left: up to 4x finer (one 128-token tile per block at
// most), again a divisor of the chunk's tiles.
int readout_parts_last(int chunk, int parts) {
    for (int p = std::min(chunk / 128, 4 * parts); p > parts; --p)
        if ((chunk / 128) % p == 0) return p;
    return parts;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Waits (bounded) until *flag != 0. On timeout sets *abort and the status.
__device__ bool wait_flag(const int *flag, volatile int *abort, int *status, int code) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        if (ld_acquire(flag)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicExch(status, code);
            return false;
        }
        __nanosleep(i < 16 ? 64 : 512);
    }
}

// Read-out role: Z_c^T = W_c^T Q_c^T per 128-token tile, with W_c^T (hi and
// lo bf16 terms, 64 + 64 columns) as the A operand in tensor memory and the Q
// tile as the K-major B operand, so that shared memory holds only a 3-stage
// Q ring (3 x 32 KB).
constexpr int kApplyTile = 128, kApplyTileBytes = kApplyTile * kD * 2;  // 32 KB
constexpr int kApplyStages = 3;
static_assert(kApplyStages * kApplyTileBytes <= kGramStages * kGramStageBytes,
              "read-out role fits the shared memory of the launch");

__device__ bool wait_count(const int *p, int want, volatile int *abort, int *status, int code) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        if (ld_acquire(p) >= want) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicExch(status, code);
            return false;
        }
        __nanosleep(i < 16 ? 64 : 512);
    }
}

__global__ void __launch_bounds__(kThreads, 2)
    chunk_fwd_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, GramScanArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bars[3 * kGramStagesU + 2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag, ticket;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = a.nseq * a.cps;
    int *sync = reinterpret_cast<int *>(a.ws + sync_offset(n));  // [0]: ticket counter, [1 + g]: flags
    if (threadIdx.x == 0) {
        ticket = atomicAdd(sync, 1);
        abort_flag = 0;
    }
    __syncthreads();
    const int tk = ticket;
    const bool gram = tk < n;
    const int nscan = a.nseq * (a.M ? 2 * kSlices : kSlices);
    const uint32_t ncols = 256;  // the gram and read-out roles' accumulator
    uint64_t *drain = &bars[3 * kGramStagesU + 1];

    if (tk >= n + nscan) {
        // ---- read-out of part `part` of chunk c of sequence s (chunk-major
        // ticket order): Z_c = Q_c W_c once both scan blocks of s have written
        // W_c's image. A chunk's tokens are split over a.parts blocks (the
        // last chunk's over a.parts_last), so that the last chunk's read-out,
        // which waits for the whole scan, is short. Q does not depend on the
        // scan: its first tiles load while the block waits for W_c.
        const int ai = tk - n - nscan, per_c = a.nseq * a.parts, head = (a.cps - 1) * per_c;
        const bool last = ai >= head;
        const int nparts = last ? a.parts_last : a.parts;
        const int c = last ? a.cps - 1 : ai / per_c;
        const int s = last ? (ai - head) / nparts : (ai % per_c) / nparts;
        const int part = last ? (ai - head) % nparts : ai % nparts;
        const int g = s * a.cps + c;
        const int ntile = a.chunk / nparts / kApplyTile;
        const long row0 = (long)g * a.chunk + (long)part * ntile * kApplyTile;
        uint64_t *qfull = bars, *qempty = bars + kApplyStages, *wfull = bars + 2 * kApplyStages,
                 *tfull = wfull + 1, *tempty = wfull + 2;
        if (threadIdx.x == 0) {
            for (int i = 0; i < kApplyStages; ++i) {
                mbar_init(&qfull[i], 1);
                mbar_init(&qempty[i], 1);
            }
            mbar_init(wfull, 128);
            mbar_init(tfull, 1);
            mbar_init(tempty, 128);
            mbar_init(drain, 1);
            fence_mbar_init();
        }
        if (warp == 1) tmem_alloc(&tmem_base, ncols);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // tensor memory: [0, 64) W^T hi, [64, 128) W^T lo (lane j = output
        // column j, column q = inputs 2q, 2q + 1), [128, 256) the accumulator
        // (lane j, column = token of the tile)
        const uint32_t tm = tmem_base, tA = tm, tD = tm + 128;
        int issued = 0;
        if (warp == 0 && lane == 0) {
            for (int t = 0; t < ntile; ++t) {
                const int st = t % kApplyStages;
                if (t >= kApplyStages &&
                    !mbar_wait(&qempty[st], ((t / kApplyStages) - 1) & 1, &abort_flag, a.status, 21))
                    break;
                uint8_t *sb = smem + st * kApplyTileBytes;
                const int y = (int)(row0 + (long)t * kApplyTile);
                mbar_arrive_expect_tx(&qfull[st], kApplyTileBytes);
                tma_load_2d(sb, &tmQ, 0, y, &qfull[st]);
                tma_load_2d(sb + kApplyTileBytes / 2, &tmQ, 64, y, &qfull[st]);
                issued = t + 1;
            }
        } else if (warp == 1 && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(128, kApplyTile, false, false);
            if (mbar_wait(wfull, 0, &abort_flag, a.status, 22)) {
                for (int t = 0; t < ntile; ++t) {
                    const int st = t % kApplyStages;
                    if (!mbar_wait(&qfull[st], (t / kApplyStages) & 1, &abort_flag, a.status, 23)) break;
                    if (t >= 1 && !mbar_wait(tempty, (t - 1) & 1, &abort_flag, a.status, 24)) break;
                    tc_fence_after();
                    const uint32_t qb = smem_u32(smem + st * kApplyTileBytes);
#pragma unroll
                    for (int k = 0; k < kD / 16; ++k) {
                        const int k0 = 16 * k;
                        const uint64_t bd = make_sdesc(qb + (k0 >> 6) * (kApplyTileBytes / 2) + (k0 & 63) * 2,
                                                       16, 1024, kSw128);
                        mma_bf16_tmem_a(tD, tA + 8 * k, bd, idesc, k != 0);
                        mma_bf16_tmem_a(tD, tA + 64 + 8 * k, bd, idesc, true);
                    }
                    mma_commit(&qempty[st]);
                    mma_commit(tfull);
                }
            }
        } else if (warp >= 2) {
            // Thread j = 32 (warp & 3) + lane: output column j. W_c^T row j
            // from the image (K-major rows n: hi j at n = 128 (j / 64) + j % 64,
            // lo 64 rows further; 16-byte chunk q of row n at q ^ (n & 7))
            // into tensor memory.
            const int j = 32 * (warp & 3) + lane;
            bool ok = true;
            if (warp == 2 && lane == 0) ok = wait_count(sync + 1 + n + g, kSlices, &abort_flag, a.status, 26);
            ok = !named_bar_or(1, 128, !ok);
            if (ok) {
                const uint8_t *img = a.ws + (size_t)n * kChunkWs + (size_t)g * 65536;
#pragma unroll
                for (int p = 0; p < 2; ++p) {  // hi, lo
                    const int nr = 128 * (j >> 6) + 64 * p + (j & 63);
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            img + kb * kImgBytes + (nr >> 3) * 1024 + (nr & 7) * 128);
                        float v[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 u = src[q ^ (nr & 7)];
                            v[4 * q] = __uint_as_float(u.x);
                            v[4 * q + 1] = __uint_as_float(u.y);
                            v[4 * q + 2] = __uint_as_float(u.z);
                            v[4 * q + 3] = __uint_as_float(u.w);
                        }
                        const uint32_t ta = taddr(tA, 32 * (warp & 3), 64 * p + 32 * kb);
                        tmem_st16(ta, *reinterpret_cast<float(*)[16]>(v));
                        tmem_st16(ta + 16, *reinterpret_cast<float(*)[16]>(v + 16));
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(wfull);
            }
            // Epilogue: thread j stores column j of each token row of the tile.
            // All of the tile's accumulator columns are loaded before the one
            // wait, so that the accumulator is released to the next tile's MMA
            // before any store.
            for (int t = 0; ok && t < ntile; ++t) {
                if (!__all_sync(0xffffffffu, mbar_wait(tfull, t & 1, &abort_flag, a.status, 25))) break;
                tc_fence_after();
                float v[kApplyTile / 16][16];
#pragma unroll
                for (int q = 0; q < kApplyTile / 16; ++q) tmem_ld16(taddr(tD, 32 * (warp & 3), 16 * q), v[q]);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(tempty);  // the accumulator is read; the next tile's MMA may start
                const size_t z0 = (size_t)(row0 + (long)t * kApplyTile) * kD + j;
#pragma unroll
                for (int q = 0; q < kApplyTile / 16; ++q)
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const size_t o = z0 + (size_t)(16 * q + e) * kD;
                        if (a.z_bf16)
                            reinterpret_cast<__nv_bfloat16 *>(a.Z)[o] = __float2bfloat16_rn(v[q][e]);
                        else
                            a.Z[o] = v[q][e];
                    }
            }
        }
        if (abort_flag) {
            if (warp == 0 && lane == 0)
                for (int t = issued - kApplyStages < 0 ? 0 : issued - kApplyStages; t < issued; ++t)
                    mbar_drain(&qfull[t % kApplyStages], (t / kApplyStages) & 1);
            if (warp == 1 && lane == 0) {
                mma_commit(drain);
                mbar_drain(drain, 0);
            }
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 1) tmem_dealloc(tm, ncols);
        return;
    }

    if (gram) {
        // ---- gram of chunk c of sequence s (chunk-major ticket order)
        const int c = tk / a.nseq, s = tk % a.nseq, g = s * a.cps + c;
        uint64_t *full = bars, *conv = bars + kGramStagesU, *empty = bars + 2 * kGramStagesU;
        uint64_t *done = &bars[3 * kGramStagesU];
        const long row0 = (long)g * a.chunk;  // first token row of this chunk in [B*H*T][d]
        const int nst = a.chunk / kGramRows;
        int issued = 0;
        // Barriers for either ring, and stage 0's K and V loads (at the same
        // place in both layouts) on their way before the step-size check.
        if (threadIdx.x == 0) {
            for (int i = 0; i < kGramStagesU; ++i) {
                mbar_init(&full[i], 1);
                mbar_init(&conv[i], 128);
                mbar_init(&empty[i], 1);
            }
            mbar_init(done, 1);
            mbar_init(drain, 1);
            fence_mbar_init();
            const int y = (int)row0;
            mbar_arrive_expect_tx(&full[0], 4 * kGramBox);
            tma_load_2d(smem, &tmK, 0, y, &full[0]);
            tma_load_2d(smem + kGramBox, &tmK, 64, y, &full[0]);
            tma_load_2d(smem + 2 * kGramBox, &tmV, 0, y, &full[0]);
            tma_load_2d(smem + 3 * kGramBox, &tmV, 64, y, &full[0]);
            issued = 1;
        }
        // one step size over the whole chunk?
        const float eta0 = a.eta[row0];
        bool differs = false;
        for (int i = threadIdx.x; i < a.chunk; i += kThreads)
            differs |= __float_as_uint(a.eta[row0 + i]) != __float_as_uint(eta0);
        const bool uniform = !__syncthreads_or(differs);
        const int stages = uniform ? kGramStagesU : kGramStages;
        const int stage_bytes = uniform ? kGramStageBytesU : kGramStageBytes;
        if (warp == 1) tmem_alloc(&tmem_base, ncols);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t tm = tmem_base;
        if (warp == 0 && lane == 0) {
            // TMA producer: K rows and V rows of each stage, two 64-column boxes each.
            for (int r = 1; r < nst; ++r) {
                const int st = r % stages;
                if (r >= stages &&
                    !mbar_wait(&empty[st], ((r / stages) - 1) & 1, &abort_flag, a.status, 11))
                    break;
                uint8_t *sb = smem + st * stage_bytes;
                const int y = (int)(row0 + (long)r * kGramRows);
                mbar_arrive_expect_tx(&full[st], 4 * kGramBox);
                tma_load_2d(sb, &tmK, 0, y, &full[st]);
                tma_load_2d(sb + kGramBox, &tmK, 64, y, &full[st]);
                tma_load_2d(sb + 2 * kGramBox, &tmV, 0, y, &full[st]);
                tma_load_2d(sb + 3 * kGramBox, &tmV, 64, y, &full[st]);
                issued = r + 1;
            }
        } else if (warp == 1 && lane == 0) {
            // MMA issuer: D[d_in][0:128) += (eta K)^T K, D[d_in][128:256) += (eta K)^T V
            // (uniform eta: K^T K | K^T V, scaled by eta in the epilogue).
            const uint32_t idesc = make_idesc_bf16(128, 256, true, true);
            const uint32_t aoff = uniform ? 0u : 4u * kGramBox;
            for (int r = 0; r < nst; ++r) {
                const int st = r % stages;
                if (!mbar_wait(uniform ? &full[st] : &conv[st], (r / stages) & 1, &abort_flag,
                               a.status, 12))
                    break;
                tc_fence_after();
                const uint32_t ab = smem_u32(smem + st * stage_bytes);
#pragma unroll
                for (int k = 0; k < kGramRows / 16; ++k) {
                    const uint64_t ad = make_sdesc(ab + aoff + k * 2048, kGramBox, 1024, kSw128);
                    const uint64_t bd = make_sdesc(ab + k * 2048, kGramBox, 1024, kSw128);
                    mma_bf16(tm, ad, bd, idesc, (r | k) != 0);
                }
                mma_commit(&empty[st]);
            }
            mma_commit(done);
        } else if (warp >= 2) {
            // Scale K's rows by eta into the A operand's buffer (K and V stay raw
            // as the B operand). Swizzling permutes 16-byte chunks inside a
            // 128-byte row only, so a chunk's row (token) is offset / 128.
            const int t = threadIdx.x - 64;
            constexpr int kChunks = 2 * kGramBox / 16;  // 16-byte chunks of K per stage
            for (int r = 0; r < nst && !uniform; ++r) {
                const int st = r % kGramStages;
                // This thread's eta values for the stage, loaded before the wait.
                float ev[kChunks / 128];
#pragma unroll
                for (int i = 0; i < kChunks / 128; ++i) {
                    const int o = (t + 128 * i) * 16;
                    ev[i] = a.eta[row0 + (long)r * kGramRows + ((o % kGramBox) >> 7)];
                }
                if (!mbar_wait(&full[st], (r / kGramStages) & 1, &abort_flag, a.status, 13)) break;
                uint8_t *sb = smem + st * kGramStageBytes;
#pragma unroll
                for (int i = 0; i < kChunks / 128; ++i) {
                    const int o = (t + 128 * i) * 16;
                    const float e = ev[i];
                    const uint4 v = *reinterpret_cast<const uint4 *>(sb + o);
                    const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&v);
                    uint4 out;
                    __nv_bfloat162 *ho = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __bfloat1622float2(hv[q]);
                        ho[q] = __floats2bfloat162_rn(f.x * e, f.y * e);
                    }
                    *reinterpret_cast<uint4 *>(sb + 4 * kGramBox + o) = out;
                }
                fence_async_smem();
                mbar_arrive(&conv[st]);
            }
            // Epilogue: lanes are d_in rows i. A_c goes out as the scan's bf16
            // operand image (K-major, 128-byte swizzle: row i = 128 bytes per
            // 64 columns j), B_c as fp32 rows; two accumulator loads per wait.
            // (__all_sync reconverges the warp for the warp-collective TMEM
            // loads.)
            if (__all_sync(0xffffffffu, mbar_wait(done, 0, &abort_flag, a.status, 14))) {
                tc_fence_after();
                const int sp = warp & 3;
                const int row = 32 * sp + lane;
                uint8_t *blk = a.ws + (size_t)g * kChunkWs;
                float4 *bdst = reinterpret_cast<float4 *>(blk + kImgBytes);
                const float scale = uniform ? eta0 : 1.f;
                auto emit16 = [&](int q, float (&v)[16]) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= scale;
                    if (q < 8) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint4 hi;
                            __nv_bfloat16 *hb = reinterpret_cast<__nv_bfloat16 *>(&hi);
#pragma unroll
                            for (int e = 0; e < 8; ++e) hb[e] = __float2bfloat16_rn(v[8 * h + e]);
                            *reinterpret_cast<uint4 *>(blk + off_kmajor_sw128(row, 16 * q + 8 * h, kD)) = hi;
                        }
                    } else {  // B_c: column quad q4 of row i at float4 q4 * 128 + i
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            bdst[(4 * (q - 8) + i) * kD + row] =
                                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                };
                for (int q = 0; q < 16; q += 2) {
                    float v0[16], v1[16];
                    tmem_ld16(taddr(tm, 32 * sp, 16 * q), v0);
                    tmem_ld16(taddr(tm, 32 * sp, 16 * q + 16), v1);
                    tmem_ld_wait();
                    emit16(q, v0);
                    emit16(q + 1, v1);
                }
                __threadfence();  // ordered before the chunk's ready flag
            }
        }
        // Teardown: after an abort, let this block's own copies and MMAs land
        // before the shared memory and tensor memory are released.
        if (abort_flag) {
            if (warp == 0 && lane == 0)
                for (int r = issued - stages < 0 ? 0 : issued - stages; r < issued; ++r)
                    mbar_drain(&full[r % stages], (r / stages) & 1);
            if (warp == 1 && lane == 0) {
                mma_commit(drain);
                mbar_drain(drain, 0);
            }
        }
        tc_fence_before();
        __syncthreads();
        // A_c and B_c are written: publish the chunk (release, device scope).
        if (threadIdx.x == 0 && !abort_flag) {
            __threadfence();
            atomicExch(sync + 1 + g, 1);
        }
        if (warp == 1) tmem_dealloc(tm, ncols);
        return;
    }

    // ---- scan of columns [64 r, 64 r + 64) of sequence s, on the tensor
    // cores. One product per chunk, D = A_c [W_c,hi | W_c,lo] (M = 128 rows
    // i, N = 128: the slice's hi and lo terms side by side, K = 128), from
    // the bf16 image of A_c (its hi term; A_c ~ I / chunk-scale, so its lo
    // term moves W by ~2^-9 of the ~1% step) and the slice's image in shared
    // memory (K-major: rows 0-63 W_hi^T, rows 64-127 W_lo^T). A_c and the
    // slice of B_c arrive by bulk copy as soon as the chunk is published and
    // their previous readers are done, so they land while the previous
    // chunk's epilogue or this chunk's product runs. The fp32 state is in
    // the registers of 4 epilogue warps (row i = TMEM lane, 64 columns); they
    // form W_c + B_c - (D_hi + D_lo) and write W_c's columns into the
    // read-out's operand image of chunk c in the workspace.
    const bool map = a.M != nullptr;
    const int per_seq = map ? 2 * kSlices : kSlices;
    const int si = tk - n, s = si / per_seq, r = si % per_seq, j0 = kSlice * (r % kSlices);
    const bool ident = map && r < kSlices;  // M: starts at I, takes no B_c
    float *out = map ? (ident ? a.M : a.N) : a.W_out;
    const int cps = a.cps;
    const size_t g0 = (size_t)s * cps;
    uint8_t *sA = smem;                   // A_c hi (K-major, 32 KB)
    uint8_t *sB = smem + kImgBytes;       // B_c columns j0.. (quad q of row i at float4 q * 128 + i)
    uint8_t *sWs = smem + 2 * kImgBytes;  // slice image: 2 column blocks of 16 KB
    uint64_t *aready = bars, *bready = bars + 1, *afree = bars + 2, *bfree = bars + 3,
             *dfull = bars + 4, *wready = bars + 5, *imgfree = bars + 6;
    uint8_t *Wimg = a.ws + (size_t)n * kChunkWs;
    if (threadIdx.x == 0) {
        mbar_init(aready, 1);
        mbar_init(bready, 1);
        mbar_init(afree, 1);
        mbar_init(bfree, 4);  // one arrival per epilogue warp
        mbar_init(dfull, 1);
        mbar_init(wready, 1);
        mbar_init(imgfree, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    int issued = 0;

    if (warp == 0 && lane == 0) {
        // A_c once chunk c's gram is published and the product of chunk
        // c - 1 is done with the buffer; B_c once the epilogue of c - 1 has
        // read the previous one.
        // Each chunk's A_c and B_c slice are also prefetched into L2 as soon
        // as the chunk is published (and the next chunk's too when it already
        // is), so that the copies into shared memory, which wait for the
        // previous step, hit L2 instead of waiting on HBM behind the streams.
        auto prefetch = [&](int c) {
            const uint8_t *blk = a.ws + (g0 + c) * kChunkWs;
            bulk_prefetch_l2(blk, kImgBytes);
            bulk_prefetch_l2(blk + kImgBytes + (size_t)j0 * kD * 4, kImgBytes);
        };
        int prefetched = 0;  // chunks [0, prefetched) are prefetched
        for (int c = 0; c < cps; ++c) {
            if (!wait_flag(sync + 1 + g0 + c, &abort_flag, a.status, 15)) break;
            asm volatile("fence.proxy.async.global;" ::: "memory");
            if (prefetched <= c) prefetch(c), prefetched = c + 1;
            if (c + 1 < cps && prefetched == c + 1 && ld_acquire(sync + 1 + g0 + c + 1)) {
                asm volatile("fence.proxy.async.global;" ::: "memory");
                prefetch(c + 1);
                prefetched = c + 2;
            }
            const uint8_t *blk = a.ws + (g0 + c) * kChunkWs;
            if (c >= 1 && !mbar_wait(afree, (c - 1) & 1, &abort_flag, a.status, 16)) break;
            mbar_arrive_expect_tx(aready, kImgBytes);
            bulk_load(sA, blk, kImgBytes, aready);
            issued = 2 * c + 1;
            if (c >= 1 && !mbar_wait(bfree, (c - 1) & 1, &abort_flag, a.status, 16)) break;
            mbar_arrive_expect_tx(bready, kImgBytes);
            bulk_load(sB, blk + kImgBytes + (size_t)j0 * kD * 4, kImgBytes, bready);
            issued = 2 * c + 2;
        }
    } else if (warp == 1 && lane == 0) {
        // The product of each chunk, and W_c's share of the read-out operand:
        // the slice image, read by the product, is also copied into chunk
        // c's image in the workspace (K block kb of slice r at
        // 32 KB kb + 16 KB r) by bulk store. The epilogue may rewrite the
        // slice image once the store has read it (imgfree); the chunk is
        // counted for the read-out once its store is complete, a step later.
        // The waits and the memory fence are on this thread, which next
        // waits for the epilogue, not on the epilogue's chain.
        const uint32_t idesc = make_idesc_bf16(128, 2 * kSlice, false, false);
        const uint32_t wb = smem_u32(sWs);
        const uint32_t ab = smem_u32(sA);
        int released = 0;  // chunks whose image share is counted
        auto release_upto = [&](int c_end) {
            if (released >= c_end) return;
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __threadfence();
            for (; released < c_end; ++released) atomicAdd(sync + 1 + n + g0 + released, 1);
        };
        int stored = 0;  // chunks whose image store is issued
        for (int c = 0; c < cps; ++c) {
            if (!mbar_wait(aready, c & 1, &abort_flag, a.status, 17)) break;
            if (!mbar_wait(wready, c & 1, &abort_flag, a.status, 18)) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
                const int k0 = 16 * k;
                const uint32_t o = (uint32_t)((k0 >> 6) * 16384 + (k0 & 63) * 2);
                mma_bf16(tm, make_sdesc(ab + o, 16, 1024, kSw128), make_sdesc(wb + o, 16, 1024, kSw128),
                         idesc, k != 0);
            }
            mma_commit(afree);
            mma_commit(dfull);
            if (!map) {
                uint8_t *img = Wimg + (g0 + c) * 65536 + (size_t)r * (kImgBytes / 2);
                bulk_store(img, sWs, kImgBytes / 2);
                bulk_store(img + kImgBytes, sWs + kImgBytes / 2, kImgBytes / 2);
                bulk_commit();
                stored = c + 1;
            }
            bulk_wait_read<0>();  // the slice image may be rewritten
            mbar_arrive(imgfree);
            if (!map) {
                bulk_wait<1>();  // images of chunks < c are stored
                release_upto(c);
            }
        }
        if (!map) {
            bulk_wait<0>();
            if (stored == cps && !abort_flag) release_upto(cps);
        }
    } else if (warp >= 2) {
        // Epilogue: row i = 32 (warp & 3) + lane, columns j0 .. j0 + 63.
        const int sp = warp & 3, row = 32 * sp + lane;
        float w[kSlice];
        if (map) {
#pragma unroll
            for (int q = 0; q < kSlice; ++q) w[q] = (ident && row == j0 + q) ? 1.f : 0.f;
        } else {
            const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? s : s % a.H) * kD * kD;
#pragma unroll
            for (int q = 0; q < kSlice / 4; ++q) {
                const float4 u = *reinterpret_cast<const float4 *>(W0 + (size_t)row * kD + j0 + 4 * q);
                w[4 * q] = u.x;
                w[4 * q + 1] = u.y;
                w[4 * q + 2] = u.z;
                w[4 * q + 3] = u.w;
            }
        }
        const float bscale = ident ? 0.f : 1.f;
        // This thread's column i of the slice image (rows n: W_hi^T then
        // W_lo^T; 128-byte swizzle, 16 KB per 64 values of i).
        auto emit = [&](int c) {
            const uint32_t cb = (uint32_t)((row >> 6) * 16384 + (row & 7) * 2);
#pragma unroll
            for (int jj = 0; jj < kSlice; ++jj) {
                __nv_bfloat16 hb, lb;
                split_bf16(w[jj], hb, lb);
                const int nh = jj, nl = kSlice + jj;
                *reinterpret_cast<__nv_bfloat16 *>(sWs + cb + (nh >> 3) * 1024 + (nh & 7) * 128 +
                                                   ((((row & 63) >> 3) ^ (nh & 7)) << 4)) = hb;
                *reinterpret_cast<__nv_bfloat16 *>(sWs + cb + (nl >> 3) * 1024 + (nl & 7) * 128 +
                                                   ((((row & 63) >> 3) ^ (nl & 7)) << 4)) = lb;
            }
            fence_async_smem();
        };
        emit(0);
        bool ok = !named_bar_or(1, 128, false);
        if (ok && warp == 2 && lane == 0) mbar_arrive(wready);
        for (int c = 0; ok && c < cps; ++c) {
            bool got = mbar_wait(bready, c & 1, &abort_flag, a.status, 19);
            got = got && mbar_wait(dfull, c & 1, &abort_flag, a.status, 20);
            if (named_bar_or(1, 128, !__all_sync(0xffffffffu, got))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float4 *Bc = reinterpret_cast<const float4 *>(sB);
#pragma unroll
            for (int q = 0; q < kSlice / 16; ++q) {
                float dh[16], dl[16];
                tmem_ld16(taddr(tm, 32 * sp, 16 * q), dh);
                tmem_ld16(taddr(tm, 32 * sp, kSlice + 16 * q), dl);
                float bv[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 f = Bc[(4 * q + u) * kD + row];
                    bv[4 * u] = f.x;
                    bv[4 * u + 1] = f.y;
                    bv[4 * u + 2] = f.z;
                    bv[4 * u + 3] = f.w;
                }
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[16 * q + e] = fmaf(bscale, bv[e], w[16 * q + e]) - (dh[e] + dl[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bfree);  // this warp has read B_c
            // the next slice image, once the store of this one has read it
            bool fr = true;
            if (c + 1 < cps) {
                fr = __all_sync(0xffffffffu, mbar_wait(imgfree, c & 1, &abort_flag, a.status, 27));
                if (fr) emit(c + 1);
            }
            if (named_bar_or(1, 128, !fr)) {
                ok = false;
                break;
            }
            if (c + 1 < cps && warp == 2 && lane == 0) mbar_arrive(wready);
        }
        if (ok && !abort_flag && out) {
            float *o = out + (size_t)s * kD * kD + (size_t)row * kD + j0;
#pragma unroll
            for (int q = 0; q < kSlice / 4; ++q)
                *reinterpret_cast<float4 *>(o + 4 * q) =
                    make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
    }
    // Teardown: after an abort, let this block's own copies and MMAs land
    // before the shared memory and tensor memory are released.
    if (abort_flag) {
        if (warp == 0 && lane == 0 && issued > 0) {
            const int c = (issued - 1) / 2;  // the last chunk whose copies were issued
            mbar_drain(aready, c & 1);
            if (issued % 2 == 0) mbar_drain(bready, c & 1);
        }
        if (warp == 1 && lane == 0) {
            mma_commit(drain);
            mbar_drain(drain, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 128);
}

}  // namespace

bool chunk_tc_supported(int d, int chunk, bool bf16) {
    return bf16 && d == kD && chunk >= 128 && chunk % 128 == 0;
}

size_t chunk_tc_workspace_bytes(int B, int H, int T, int d, int chunk) {
    if (d != kD || chunk <= 0 || T % chunk) return 0;
    const size_t n = (size_t)B * H * (T / chunk);
    return sync_offset(n) + sync_bytes(n);
}

// Map mode: the Gram products and the scan of [M | N] in one launch, no
// read-out (d = 128, bf16, chunk % 128 == 0; workspace as the forward's).
cudaError_t launch_chunk_map_tc(const void *K, const void *V, const float *eta, float *M, float *N,
                                int B, int H, int T, int chunk, void *workspace, cudaStream_t s) {
    const int cps = T / chunk;
    const int nseq = B * H, n = nseq * cps;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const uint64_t rows = (uint64_t)B * H * T;
    alignas(64) CUtensorMap tmK, tmV;
    if (!encode_tmap_bf16_2d(&tmK, K, kD, rows, 64, kGramRows) ||
        !encode_tmap_bf16_2d(&tmV, V, kD, rows, 64, kGramRows))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ws + sync_offset(n), 0, sync_bytes(n), s);
    if (e != cudaSuccess) return e;
    GramScanArgs g{eta, ws, nullptr, nullptr, chunk, H, nseq, cps, false, device_status_word()};
    g.M = M;
    g.N = N;
    // no read-out blocks: the Q map is never read (K's stands in)
    chunk_fwd_kernel<<<n + nseq * 2 * kSlices, kThreads, kGramSmem, s>>>(tmK, tmV, tmK, g);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s) {
    const int cps = a.T / a.chunk;
    const int nseq = a.B * a.H, n = nseq * cps;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmV, tmQ;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, 64, kGramRows) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, 64, kGramRows) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, 64, kApplyTile))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    // ticket counter, ready flags and read-out counts start at zero
    e = cudaMemsetAsync(ws + sync_offset(n), 0, sync_bytes(n), s);
    if (e != cudaSuccess) return e;
    GramScanArgs g{a.eta, ws, a.W0, a.W_out, a.chunk, a.H, nseq, cps, a.w0_per_seq, device_status_word()};
    g.Z = a.Z;
    g.z_bf16 = a.z_bf16;
    g.parts = readout_parts(a.chunk, n);
    g.parts_last = readout_parts_last(a.chunk, g.parts);
    // n Gram blocks, 2 scan blocks per sequence, parts read-out blocks per
    // chunk (parts_last for the last chunk of each sequence)
    const int nread = nseq * ((cps - 1) * g.parts + g.parts_last);
    chunk_fwd_kernel<<<n + nseq * kSlices + nread, kThreads, kGramSmem, s>>>(tmK, tmV, tmQ, g);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

}  // namespace ttt

// ---------------------------------------------------------------------------
// Allocation-free entry point: the same launch, with its scratch in a
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
