// ttt_linear_tc.cu -- TTT-Linear (d = 64, mini-batch b = 16, bf16 Q/K/V) on the
// tensor cores: one thread block per (batch, head) sequence scans all
// mini-batches with the fast weight resident on chip (fp32 in tensor memory).
//
// Method ("Test-Time Training: Linear Complexity Beyond Attention", Key
// Architectural Mechanics of TTT-Linear, parts 1-4). For mini-batch m with
// weight W_m:
//   X_m     = K_m W_m
//   G_m     = diag(eta) dl/dX_m     (LayerNorm backward of f - v, or X - V)
//   W_{m+1} = W_m - K_m^T G_m
//   Z_m     = epilogue( Q_m W_m - tril(Q_m K_m^T) G_m )
// Only G_m -> G_{m+1} is sequential. Because
//   X_{m+1} = K_{m+1} W_m - (K_{m+1} K_m^T) G_m = P_{m+1} - C_{m+1} G_m,
// the tensor cores form P_{m+1} = K_{m+1} W_m one mini-batch ahead; the
// critical chain per mini-batch is one 16x16 by 16x64 correction plus the
// LayerNorm backward, done in fp32 on CUDA cores by the scan warps.
//
// Per mini-batch the tensor core runs two MMA groups:
//   update:  W^T += (-G_j)^T K_j                                   (M=64, N=64, K=16)
//   product: [Q_{j+1}; K_{j+2}] x [W_{j+1}^T hi | W_{j+1}^T lo | K_{j+1}]^T  (M=128, N=144, K=64)
// The product's rows give Q_{j+1} W_{j+1} (read-out), Q_{j+1} K_{j+1}^T (causal
// term), K_{j+2} W_{j+1} (= P_{j+2}) and K_{j+2} K_{j+1}^T (= C_{j+2}) at once.
// The fp32 state is kept as W^T so that re-emitting it as the bf16 hi/lo
// operand writes whole 16-byte rows.
//
// Warp roles (16 warps):
//   0      TMA producer: K, Q, V in chunks of 64 tokens (4-slot ring)
//   1      MMA issuer (one thread) and tensor-memory owner
//   2      stages the product's A tile [Q_{j+1}; K_{j+2}] from the TMA tiles
//   3      copies the product (tensor-memory subpartition 3) out: P and C for
//          the scan, Q W and Q K^T into a 4-slot ring for the output warps
//   4-7    scan: X = P - C G_prev, LayerNorm backward, G (fp32 + bf16 hi/lo)
//   8-11   W re-emit: fp32 W^T from tensor memory -> bf16 hi/lo operand rows
//   12-15  output: Zpre = Q W - tril(Q K^T) G, LayerNorm + residual, store Z
// Precision: Q/K/V enter exactly (bf16); every other operand (W, G) enters
// the tensor cores as two bf16 terms hi + lo with fp32 accumulation, and the
// chain's corrections and all LayerNorm math are fp32.
#include "sm100.cuh"
#include "ttt_common.cuh"

// Optional pipeline trace: compiled in only when TTT_TRACE is defined (a
// profiling build). Block 0 records 32-bit SM clock stamps at each hand-off
// into shared memory (so tracing adds no global-memory traffic inside the
// pipeline) and copies them out when it exits.
constexpr int kTraceEvents = 32, kTraceSteps = 128;
#ifdef TTT_TRACE
__device__ unsigned g_ttt_trace[kTraceEvents * kTraceSteps];
#define TRACE(ev, i)                                                                  \
    do {                                                                              \
        if ((i) >= 0 && (i) < kTraceSteps) trace_smem[(ev) * kTraceSteps + (i)] = (unsigned)clock(); \
    } while (0)
#else
#define TRACE(ev, i) \
    do {             \
    } while (0)
#endif

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 64, kMB = 16;
constexpr int kChunkTok = 64, kMbPerChunk = kChunkTok / kMB, kSlots = 4;
constexpr int kTile = kChunkTok * kD * 2;  // 8 KB per tensor per chunk
constexpr int kThreads = 512;
constexpr int kBRows = 144;                // W^T hi (64) | W^T lo (64) | K_{j+1} (16)

// Shared memory map (offsets from a 1024-aligned base).
constexpr int OFF_K = 0;
constexpr int OFF_Q = OFF_K + kSlots * kTile;
constexpr int OFF_V = OFF_Q + kSlots * kTile;
constexpr int OFF_A = OFF_V + kSlots * kTile + 12288;  // 4 slots of 32 rows; the MMA window starts 96 rows earlier
constexpr int OFF_B = OFF_A + 4 * 4096;
constexpr int OFF_G = OFF_B + kBRows * 128;           // -G hi | lo (MN-major, 2 KB each), 2 buffers
constexpr int OFF_PF = OFF_G + 8192;                  // P fp32 [2][16][64], float4-swizzled
constexpr int kCStride = 20;                          // C rows padded to 16-byte multiples
constexpr int OFF_CF = OFF_PF + 2 * 16 * 64 * 4;      // C fp32 [2][16][kCStride]
constexpr int OFF_GF = OFF_CF + 2 * 16 * kCStride * 4;  // G fp32 [4][16][64]
constexpr int OFF_ZQ = OFF_GF + 4 * 16 * 64 * 4;      // Q W fp32 [4][16][64], float4-swizzled
constexpr int OFF_SF = OFF_ZQ + 4 * 16 * 64 * 4;      // Q K^T fp32 [4][16][kCStride]
constexpr int OFF_ETA = OFF_SF + 4 * 16 * kCStride * 4;  // eta fp32 [kSlots][64], one row per chunk
constexpr int OFF_KS = OFF_ETA + kSlots * kChunkTok * 4;  // 1 / |k| fp32 [kSlots][64] (L2 keys)
constexpr int OFF_TRACE = OFF_KS + kSlots * kChunkTok * 4;
#ifdef TTT_TRACE
constexpr int kTraceBytes = kTraceEvents * kTraceSteps * 4;
#else
constexpr int kTraceBytes = 0;
#endif
constexpr int kSmemBytes = OFF_TRACE + kTraceBytes + 1024;
static_assert(OFF_Q % 1024 == 0 && OFF_V % 1024 == 0 && OFF_A % 1024 == 0 && OFF_B % 1024 == 0 &&
                  OFF_G % 1024 == 0,
              "operand tiles need 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Tensor-memory columns (512 allocated). The M = 64 W^T accumulator keeps row
// r in lane 32 (r / 16) + r % 16; the M = 128 product keeps row r in lane r.
constexpr uint32_t TM_WT = 0, TM_B = 64;  // W^T (64 cols); product, 2 buffers of 144 cols
// Product rows 96-111 = Q_{j+1}, 112-127 = K_{j+2}: lanes 96-127 (subpartition 3).

struct Args {
    const float *eta, *W0, *gamma, *beta;
    float *Z, *W_out;
    int H, T;
    bool ln, w0_per_seq, z_bf16;
    int *status;
};

// Mean and 1/sigma of a 64-value row spread over 8 lanes (8 values each):
// local mean and sum of squared deviations, merged pairwise across lanes
// (the equal-count case of Chan et al.'s update), LayerNorm eps inside the root.
__device__ __forceinline__ void row_stats(const float (&x)[8], float &mu, float &rstd) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m += x[i];
    m *= 0.125f;
    float M2 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float d = x[i] - m;
        M2 = fmaf(d, d, M2);
    }
#pragma unroll
    for (int o = 1, n = 8; o < 8; o <<= 1, n <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float M2o = __shfl_xor_sync(0xffffffffu, M2, o);
        const float dl = mo - m;
        m = 0.5f * (m + mo);
        M2 = M2 + M2o + dl * dl * (0.5f * n);
    }
    mu = m;
    rstd = rsqrtf(M2 * (1.f / kD) + kLnEps);
}

// A thread (t, g) of the scan and output groups owns columns 4g..4g+3 and
// 32+4g..32+4g+3 of token row t ("two quads"), so eight threads of a row
// touch 128 contiguous bytes per access.

// The thread's 8 bf16 of row `row` of a 128-byte-swizzled [rows][64] tile.
__device__ __forceinline__ void load_quads_bf16(const uint8_t *tile, int row, int g,
                                                float (&v)[8]) {
    const uint8_t *r = tile + row * 128;
    const int sw = row & 7;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int chunk = 4 * h + (g >> 1);
        const uint2 u = *reinterpret_cast<const uint2 *>(r + ((chunk ^ sw) << 4) + (g & 1) * 8);
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        v[4 * h] = f0.x;
        v[4 * h + 1] = f0.y;
        v[4 * h + 2] = f1.x;
        v[4 * h + 3] = f1.y;
    }
}

// fp32 [16][64] staging rows written by tensor-memory readers (one row per
// lane) and read by (t, g) threads: float4 q of row t sits at q ^ (t & 7).
__device__ __forceinline__ int swz4(int row, int q) { return row * 16 + (q ^ (row & 7)); }

__device__ __forceinline__ void load_quads_f32_swz(const float *base, int row, int g,
                                                   float (&v)[8]) {
    const float4 *b = reinterpret_cast<const float4 *>(base);
    const float4 u0 = b[swz4(row, g)], u1 = b[swz4(row, 8 + g)];
    v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
    v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
}

// Packs 4 floats to 4 bf16 hi terms and 4 bf16 lo terms (hi + lo ~ x).
__device__ __forceinline__ void split4(float a, float b, float c, float d, uint2 &hi, uint2 &lo) {
    split2(a, b, hi.x, lo.x);
    split2(c, d, hi.y, lo.y);
}

template <bool kL2>  // L2-normalised keys: compiled as its own kernel
__global__ void __launch_bounds__(kThreads, 1)
    linear_ln_scan_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmV, Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + OFF_K, *sQ = smem + OFF_Q, *sV = smem + OFF_V;
    uint8_t *sA = smem + OFF_A, *sB = smem + OFF_B, *sG = smem + OFF_G;
    float *Pf = reinterpret_cast<float *>(smem + OFF_PF);
    float *Cf = reinterpret_cast<float *>(smem + OFF_CF);
    float *Gf = reinterpret_cast<float *>(smem + OFF_GF);
    float *Zqf = reinterpret_cast<float *>(smem + OFF_ZQ);
    float *Sf = reinterpret_cast<float *>(smem + OFF_SF);
    float *etas = reinterpret_cast<float *>(smem + OFF_ETA);
    // Key scales s_t = 1 / max(|k_t|, 1e-12) with L2-normalised keys, else 1.
    // The kernel keeps the raw bf16 keys in every product and applies s as
    // row / column scalings: P and C rows by the key token's s, C and Q K^T
    // columns by the source token's s, the key residual of the LayerNorm
    // backward and the G rows of the weight update by s.
    float *kscale = reinterpret_cast<float *>(smem + OFF_KS);
#ifdef TTT_TRACE
    volatile unsigned *trace_smem = reinterpret_cast<volatile unsigned *>(smem + OFF_TRACE);
    for (int e = threadIdx.x; e < kTraceEvents * kTraceSteps; e += blockDim.x) trace_smem[e] = 0;
#endif

    __shared__ uint64_t tfull[kSlots], tfree[kSlots], gready[4], efree[4], aready[4], afree[4],
        zready[4], zfree[4], pzdone[2], pcready[2], wdone, wsm, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.x, head = seq % a.H;
    // NM counts a partial last mini-batch: its rows past T get step size 0 (the
    // eta staging below), so their G rows are zero, and their Z is not stored.
    const int T = a.T, NM = (T + kMB - 1) / kMB, NC = (T + kChunkTok - 1) / kChunkTok;
    const long tok0 = (long)seq * T;  // first row of this sequence in [B*H*T][64]
    int *status = a.status;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tfree[s], 1 + 128);  // last update MMA of the chunk + output warps
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&gready[i], 128);
            mbar_init(&efree[i], 128);
            mbar_init(&aready[i], 32);
            mbar_init(&afree[i], 1);
            mbar_init(&zready[i], 32);
            mbar_init(&zfree[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pzdone[i], 1);
            mbar_init(&pcready[i], 32);
        }
        mbar_init(&wdone, 1);
        mbar_init(&wsm, 128);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    volatile int *abrt = &abort_flag;

    // Row r of mini-batch m in a K/Q/V ring (generic pointer to its 128 bytes).
    auto ring_row = [&](uint8_t *ring, int m, int r) -> uint8_t * {
        return ring + ((m / kMbPerChunk) % kSlots) * kTile + ((m % kMbPerChunk) * kMB + r) * 128;
    };
    // key scale of token t of mini-batch m (staged with the chunk's etas)
    auto kscale_of = [&](int m, int t) -> float {
        return kscale[((m / kMbPerChunk) % kSlots) * kChunkTok + (m % kMbPerChunk) * kMB + t];
    };
    auto chunk_wait = [&](int m, int code) -> bool {  // warp-uniform wait for m's chunk
        const int c = m / kMbPerChunk;
        return mbar_wait_warp(&tfull[c % kSlots], (c / kSlots) & 1, abrt, status, code);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int c = 0; c < NC; ++c) {
                const int s = c % kSlots;
                if (c >= kSlots && !mbar_wait(&tfree[s], ((c / kSlots) - 1) & 1, abrt, status, 31))
                    break;
                const int y = (int)(tok0 + (long)c * kChunkTok);
                mbar_arrive_expect_tx(&tfull[s], 3 * kTile);
                tma_load_2d(sK + s * kTile, &tmK, 0, y, &tfull[s]);
                tma_load_2d(sQ + s * kTile, &tmQ, 0, y, &tfull[s]);
                tma_load_2d(sV + s * kTile, &tmV, 0, y, &tfull[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t I_UPD = make_idesc_bf16(64, 64, true, true);
            const uint32_t I_PROD = make_idesc_bf16(128, kBRows, false, false);
            const uint32_t bb = smem_u32(sB), gb = smem_u32(sG);
            // Product i (i = -2 .. NM-2): A slot (i+2)%4, accumulator (i+2)%2.
            auto product = [&](int i) {
                const uint32_t arow = smem_u32(sA) + ((i + 2) & 3) * 4096 - 12288;  // 96 rows earlier
                const uint32_t d = tm + TM_B + ((i + 2) & 1) * kBRows;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(d, make_sdesc(arow + 32 * k, 16, 1024, kSw128),
                             make_sdesc(bb + 32 * k, 16, 1024, kSw128), I_PROD, k != 0);
                mma_commit(&pzdone[(i + 2) & 1]);
                mma_commit(&afree[(i + 2) & 3]);
            };
            bool ok = mbar_wait(&wsm, 0, abrt, status, 32) &&
                      mbar_wait(&aready[0], 0, abrt, status, 33) &&
                      mbar_wait(&aready[1], 0, abrt, status, 33);
            if (ok) {
                tc_fence_after();
                product(-2);  // P_0 = K_0 W_0
                product(-1);  // P_1, C_1, Q_0 W_0, Q_0 K_0^T
            }
            for (int j = 0; ok && j < NM; ++j) {
                if (!mbar_wait(&gready[j & 3], (j >> 2) & 1, abrt, status, 34)) break;
                TRACE(0, j);
                tc_fence_after();
                // W_{j+1}^T = W_j^T + (-G_j)^T K_j
                const uint32_t krow = smem_u32(ring_row(sK, j, 0));
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    mma_bf16(tm + TM_WT, make_sdesc(gb + (j & 1) * 4096 + p * 2048, 8192, 1024, kSw128),
                             make_sdesc(krow, 8192, 1024, kSw128), I_UPD, true);
                mma_commit(&wdone);
                TRACE(1, j);
                if (j % kMbPerChunk == kMbPerChunk - 1) mma_commit(&tfree[(j / kMbPerChunk) % kSlots]);
                if (j + 1 >= NM) break;
                const int i = j;
                if (!mbar_wait(&wsm, (j + 1) & 1, abrt, status, 35)) break;
                TRACE(2, j);
                if (!mbar_wait(&aready[(i + 2) & 3], ((i + 2) >> 2) & 1, abrt, status, 36)) break;
                TRACE(18, j);
                tc_fence_after();
                product(i);
                TRACE(3, j);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ A stager
        // A_i rows 0-15 = Q_{i+1}, rows 16-31 = K_{i+2} (copies of the TMA rows;
        // source and destination rows agree mod 8, so the swizzle carries over).
        for (int i = -2; i <= NM - 2; ++i) {
            const int s = (i + 2) & 3;
            if (i + 2 >= 4 && !mbar_wait_warp(&afree[s], (((i + 2) >> 2) - 1) & 1, abrt, status, 71)) break;
            if (i + 2 < NM && (i + 2) % kMbPerChunk == 0) {
                // First use of a new chunk: wait for it, and stage its eta row.
                if (!chunk_wait(i + 2, 72)) break;
                const int c = (i + 2) / kMbPerChunk;
                for (int e = lane; e < kChunkTok; e += 32) {
                    const long tok = (long)c * kChunkTok + e;
                    etas[(c % kSlots) * kChunkTok + e] = tok < T ? a.eta[tok0 + tok] : 0.f;
                    if constexpr (kL2) {  // the row's 16-byte chunks in any order: sum of squares
                        const uint8_t *kr = sK + (c % kSlots) * kTile + e * 128;
                        float ss = 0.f;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 u = *reinterpret_cast<const uint4 *>(kr + 16 * q);
                            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[h]));
                                ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                            }
                        }
                        kscale[(c % kSlots) * kChunkTok + e] = 1.f / fmaxf(sqrtf(ss), 1e-12f);
                    }
                }
            }
            uint8_t *dst = sA + s * 4096;
#pragma unroll
            for (int e = lane; e < 256; e += 32) {
                const int r = e >> 3, c = e & 7;
                const int m = r < 16 ? i + 1 : i + 2;
                if (m >= 0 && m < NM) {
                    const uint8_t *src = ring_row(r < 16 ? sQ : sK, m, r & 15);
                    *reinterpret_cast<uint4 *>(dst + r * 128 + c * 16) =
                        *reinterpret_cast<const uint4 *>(src + c * 16);
                }
            }
            fence_async_smem();
            mbar_arrive(&aready[s]);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ product copy-out
        // Product i (rows 96-127 = lanes 96-127): lanes 0-15 hold Q_{i+1} rows
        // (Q W, Q K^T -> output ring slot (i+1)%4), lanes 16-31 hold K_{i+2} rows
        // (P, C -> scan buffer (i+2)%2).
        const bool qrow = lane < 16;
        const int row = lane & 15;
        for (int i = -2; i <= NM - 2; ++i) {
            const int mz = i + 1, mp = i + 2;
            if (!mbar_wait_warp(&pzdone[(i + 2) & 1], ((i + 2) >> 1) & 1, abrt, status, 81)) break;
            if (mz >= 4 && !mbar_wait_warp(&zfree[mz & 3], ((mz >> 2) - 1) & 1, abrt, status, 82)) break;
            tc_fence_after();
            const uint32_t col = TM_B + ((i + 2) & 1) * kBRows;
            float *dst = qrow ? Zqf + (mz & 3) * 1024 : Pf + (mp & 1) * 1024;
            const bool live = qrow ? mz >= 0 : mp < NM;
            // key scales: this K row's (P and C rows), the source keys' (columns)
            const int msrc = i + 1;  // B rows 128-143 hold K_{i+1}
            const float rs = (kL2 && !qrow && live) ? kscale_of(mp, row) : 1.f;
            float v0[16], v1[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // hi + lo, 16 columns at a time
                tmem_ld16(taddr(tm, 96, col + 16 * c), v0);
                tmem_ld16(taddr(tm, 96, col + 64 + 16 * c), v1);
                tmem_ld_wait();
                if (live) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        d4[swz4(row, 4 * c + q)] =
                            kL2
                                ? make_float4(rs * (v0[4 * q] + v1[4 * q]), rs * (v0[4 * q + 1] + v1[4 * q + 1]),
                                              rs * (v0[4 * q + 2] + v1[4 * q + 2]),
                                              rs * (v0[4 * q + 3] + v1[4 * q + 3]))
                                : make_float4(v0[4 * q] + v1[4 * q], v0[4 * q + 1] + v1[4 * q + 1],
                                              v0[4 * q + 2] + v1[4 * q + 2], v0[4 * q + 3] + v1[4 * q + 3]);
                }
            }
            tmem_ld16(taddr(tm, 96, col + 128), v0);
            tmem_ld_wait();
            if (live) {
                float *g16 = qrow ? Sf + ((mz & 3) * 16 + row) * kCStride : Cf + ((mp & 1) * 16 + row) * kCStride;
                if (kL2 && msrc >= 0) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v0[e] *= rs * kscale_of(msrc, e);
                }
                float4 *c4 = reinterpret_cast<float4 *>(g16);
#pragma unroll
                for (int q = 0; q < 4; ++q) c4[q] = make_float4(v0[4 * q], v0[4 * q + 1], v0[4 * q + 2], v0[4 * q + 3]);
            }
            tc_fence_before();
            if (mp < NM) mbar_arrive(&pcready[mp & 1]);
            if (mz >= 0) mbar_arrive(&zready[mz & 3]);
            if (lane == 0) TRACE(4, mp);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ scan
        const int r = threadIdx.x - 128, t = r >> 3, g = r & 7;
        float gam[8], bet[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int col = (i < 4 ? 4 * g : 28 + 4 * g) + i;
            gam[i] = a.ln ? a.gamma[head * kD + col] : 1.f;
            bet[i] = a.ln ? a.beta[head * kD + col] : 0.f;
        }
        for (int j = 0; j < NM; ++j) {
            if (j % kMbPerChunk == 0 && !chunk_wait(j, 41)) break;
            if (!mbar_wait_warp(&pcready[j & 1], (j >> 1) & 1, abrt, status, 42)) break;
            if (threadIdx.x == 128) TRACE(5, j);
            float x[8];
            load_quads_f32_swz(Pf + (j & 1) * 1024, t, g, x);
            if (j > 0) {  // X_j = P_j - C_j G_{j-1}: coefficients in registers, two chains
                // G_{j-1} comes from all four scan warps: wait for all of it.
                if (!mbar_wait_warp(&gready[(j - 1) & 3], ((j - 1) >> 2) & 1, abrt, status, 44)) break;
                if (threadIdx.x == 128) TRACE(21, j);
                const float4 *c4 = reinterpret_cast<const float4 *>(Cf + ((j & 1) * 16 + t) * kCStride);
                float c[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 u = c4[q];
                    c[4 * q] = u.x; c[4 * q + 1] = u.y; c[4 * q + 2] = u.z; c[4 * q + 3] = u.w;
                }
                const float *gprev = Gf + ((j - 1) & 3) * 1024;
                float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < kMB; s += 2) {
                    const float4 u0 = *reinterpret_cast<const float4 *>(gprev + s * kD + 4 * g);
                    const float4 u1 = *reinterpret_cast<const float4 *>(gprev + s * kD + 32 + 4 * g);
                    const float4 w0 = *reinterpret_cast<const float4 *>(gprev + (s + 1) * kD + 4 * g);
                    const float4 w1 = *reinterpret_cast<const float4 *>(gprev + (s + 1) * kD + 32 + 4 * g);
                    x[0] = fmaf(-c[s], u0.x, x[0]); x[1] = fmaf(-c[s], u0.y, x[1]);
                    x[2] = fmaf(-c[s], u0.z, x[2]); x[3] = fmaf(-c[s], u0.w, x[3]);
                    x[4] = fmaf(-c[s], u1.x, x[4]); x[5] = fmaf(-c[s], u1.y, x[5]);
                    x[6] = fmaf(-c[s], u1.z, x[6]); x[7] = fmaf(-c[s], u1.w, x[7]);
                    y[0] = fmaf(-c[s + 1], w0.x, y[0]); y[1] = fmaf(-c[s + 1], w0.y, y[1]);
                    y[2] = fmaf(-c[s + 1], w0.z, y[2]); y[3] = fmaf(-c[s + 1], w0.w, y[3]);
                    y[4] = fmaf(-c[s + 1], w1.x, y[4]); y[5] = fmaf(-c[s + 1], w1.y, y[5]);
                    y[6] = fmaf(-c[s + 1], w1.z, y[6]); y[7] = fmaf(-c[s + 1], w1.w, y[7]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] += y[i];
            }
            if (threadIdx.x == 128) TRACE(6, j);
            // eta was staged (with the chunk) before the product that made P_j
            const float eta = etas[((j / kMbPerChunk) % kSlots) * kChunkTok + (j % kMbPerChunk) * kMB + t];
            float vv[8], G[8];
            load_quads_bf16(ring_row(sV, j, 0), t, g, vv);
            const float ksc = kL2 ? kscale_of(j, t) : 1.f;
            if (a.ln) {
                float kv[8];
                load_quads_bf16(ring_row(sK, j, 0), t, g, kv);
                if constexpr (kL2) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) kv[i] *= ksc;
                }
                float mu, rstd;
                row_stats(x, mu, rstd);
                if (threadIdx.x == 128) TRACE(24, j);
                float xh[8], gh[8], s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    xh[i] = (x[i] - mu) * rstd;
                    gh[i] = gam[i] * (kv[i] + gam[i] * xh[i] + bet[i] - vv[i]);
                    s1 += gh[i];
                    s2 = fmaf(gh[i], xh[i], s2);
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                }
                s1 *= 1.f / kD;
                s2 *= 1.f / kD;
                const float sc = eta * rstd;
#pragma unroll
                for (int i = 0; i < 8; ++i) G[i] = sc * (gh[i] - s1 - xh[i] * s2);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) G[i] = eta * (x[i] - vv[i]);
            }
            if (threadIdx.x == 128) TRACE(7, j);
            if (j >= 4 && !mbar_wait_warp(&efree[j & 3], ((j >> 2) - 1) & 1, abrt, status, 43)) break;
            float *gf = Gf + (j & 3) * 1024 + t * kD;
            *reinterpret_cast<float4 *>(gf + 4 * g) = make_float4(G[0], G[1], G[2], G[3]);
            *reinterpret_cast<float4 *>(gf + 32 + 4 * g) = make_float4(G[4], G[5], G[6], G[7]);
            if (threadIdx.x == 128) TRACE(25, j);
            // -G as bf16 hi + lo, MN-major (rows = tokens, 128-byte swizzle)
            uint8_t *gb = sG + (j & 1) * 4096;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint2 hi, lo;
                if constexpr (kL2)
                    split4(-ksc * G[4 * h], -ksc * G[4 * h + 1], -ksc * G[4 * h + 2],
                           -ksc * G[4 * h + 3], hi, lo);
                else
                    split4(-G[4 * h], -G[4 * h + 1], -G[4 * h + 2], -G[4 * h + 3], hi, lo);
                const uint32_t off = off_mnmajor_sw128(t, 32 * h + 4 * g, kMB);
                *reinterpret_cast<uint2 *>(gb + off) = hi;
                *reinterpret_cast<uint2 *>(gb + 2048 + off) = lo;
            }
            if (threadIdx.x == 128) TRACE(26, j);
            fence_async_smem();
            if (threadIdx.x == 128) TRACE(27, j);
            mbar_arrive(&gready[j & 3]);
            if (threadIdx.x == 128) TRACE(8, j);
        }
    } else if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------ W re-emit
        // Warp 8+q owns W^T rows 16q..16q+15 (tensor-memory subpartition q,
        // lanes 0-15): thread i < 16 handles d_in columns 0-31 of row 16q+i,
        // thread 16+i columns 32-63 of the same row.
        const int q = warp & 3;
        const int half = lane >> 4;          // d_in columns 32*half .. +31
        const int n = 16 * q + (lane & 15);  // W^T row = d_out index
        const int rt = threadIdx.x - 256;    // 0..127
        const uint32_t wl = taddr(tm, 32 * q, TM_WT);
        // Writes W^T row n, this half's columns, as hi (row n) and lo (row 64+n).
        auto emit = [&](const float (&w)[32]) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                uint2 h0, l0, h1, l1;
                split4(w[8 * c8], w[8 * c8 + 1], w[8 * c8 + 2], w[8 * c8 + 3], h0, l0);
                split4(w[8 * c8 + 4], w[8 * c8 + 5], w[8 * c8 + 6], w[8 * c8 + 7], h1, l1);
                const int chunk = 4 * half + c8;
                *reinterpret_cast<uint4 *>(sB + n * 128 + ((chunk ^ (n & 7)) << 4)) =
                    make_uint4(h0.x, h0.y, h1.x, h1.y);
                *reinterpret_cast<uint4 *>(sB + (64 + n) * 128 + ((chunk ^ (n & 7)) << 4)) =
                    make_uint4(l0.x, l0.y, l1.x, l1.y);
            }
        };
        // Rows 128-143 of the B tile: K_m (same swizzle phase: 128 = 0 mod 8).
        auto copy_k = [&](int m) {
            if (m < NM) {
                const int r = rt >> 3, c = rt & 7;
                *reinterpret_cast<uint4 *>(sB + (128 + r) * 128 + c * 16) =
                    *reinterpret_cast<const uint4 *>(ring_row(sK, m, r) + c * 16);
            }
        };
        bool ok = chunk_wait(0, 51);
        if (ok) {  // initial weight -> tensor memory (fp32, transposed) and the operand
            const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : head) * kD * kD;
            float w[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) w[k] = W0[(32 * half + k) * kD + n];
            // 32-lane stores: thread i < 16 writes all 64 columns of lane i
            // (columns 32-63 from thread 16+i); lanes 16-31 are not used by
            // the M = 64 accumulator and receive don't-care values.
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float mine = w[16 * (c & 1) + i];
                    const float up = __shfl_down_sync(0xffffffffu, mine, 16);
                    v[i] = c < 2 ? mine : up;
                }
                tmem_st16(wl + 16 * c, v);
            }
            tmem_st_wait();
            emit(w);
            copy_k(0);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&wsm);
        }
        for (int j = 0; ok && j < NM; ++j) {
            if (!mbar_wait_warp(&wdone, j & 1, abrt, status, 52)) break;
            if (lane == 0) TRACE(9 + q, j);
            tc_fence_after();
            float w[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float v[16];
                tmem_ld16_x2<32>(wl + 16 * c, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) w[16 * c + i] = v[i];
            }
            tmem_ld_wait();
            if (lane == 0 && q == 0) TRACE(19, j);
            if (j + 1 < NM) {
                if ((j + 1) % kMbPerChunk == 0 && !chunk_wait(j + 1, 53)) break;
                emit(w);
                copy_k(j + 1);
                if (lane == 0 && q == 0) TRACE(20, j);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&wsm);
                if (lane == 0) TRACE(13 + q, j);
            } else if (a.W_out) {
                float *dst = a.W_out + (size_t)seq * kD * kD + n;
#pragma unroll
                for (int k = 0; k < 32; ++k) dst[(32 * half + k) * kD] = w[k];
            }
        }
    } else {
        // ------------------------------------------------------------ output
        const int r = threadIdx.x - 384, t = r >> 3, g = r & 7;
        float gam[8], bet[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int col = (i < 4 ? 4 * g : 28 + 4 * g) + i;
            gam[i] = a.ln ? a.gamma[head * kD + col] : 1.f;
            bet[i] = a.ln ? a.beta[head * kD + col] : 0.f;
        }
        for (int m = 0; m < NM; ++m) {
            if (m % kMbPerChunk == 0 && !chunk_wait(m, 61)) break;
            if (!mbar_wait_warp(&zready[m & 3], (m >> 2) & 1, abrt, status, 62)) break;
            if (!mbar_wait_warp(&gready[m & 3], (m >> 2) & 1, abrt, status, 63)) break;
            float zp[8];
            load_quads_f32_swz(Zqf + (m & 3) * 1024, t, g, zp);
            const float *gm = Gf + (m & 3) * 1024;
            const float *srow = Sf + ((m & 3) * 16 + t) * kCStride;
            for (int s = 0; s <= t; ++s) {  // - tril(Q K^T) G, diagonal included
                const float c = srow[s];
                const float4 u0 = *reinterpret_cast<const float4 *>(gm + s * kD + 4 * g);
                const float4 u1 = *reinterpret_cast<const float4 *>(gm + s * kD + 32 + 4 * g);
                zp[0] = fmaf(-c, u0.x, zp[0]); zp[1] = fmaf(-c, u0.y, zp[1]);
                zp[2] = fmaf(-c, u0.z, zp[2]); zp[3] = fmaf(-c, u0.w, zp[3]);
                zp[4] = fmaf(-c, u1.x, zp[4]); zp[5] = fmaf(-c, u1.y, zp[5]);
                zp[6] = fmaf(-c, u1.z, zp[6]); zp[7] = fmaf(-c, u1.w, zp[7]);
            }
            float qv[8];
            if (a.ln) load_quads_bf16(ring_row(sQ, m, 0), t, g, qv);
            // G_m, Q W, Q K^T and the Q rows are read: release them before the
            // global stores, so the arrivals do not wait for the stores.
            mbar_arrive(&efree[m & 3]);
            mbar_arrive(&zfree[m & 3]);
            if (m % kMbPerChunk == kMbPerChunk - 1) mbar_arrive(&tfree[(m / kMbPerChunk) % kSlots]);
            float out[8];
            if (a.ln) {
                float mu, rstd;
                row_stats(zp, mu, rstd);
#pragma unroll
                for (int i = 0; i < 8; ++i) out[i] = qv[i] + gam[i] * ((zp[i] - mu) * rstd) + bet[i];
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) out[i] = zp[i];
            }
            if (m * kMB + t < T) {
                const size_t zo = (size_t)(tok0 + (long)m * kMB + t) * kD;
                store_z4(a.Z, a.z_bf16, zo + 4 * g, out[0], out[1], out[2], out[3]);
                store_z4(a.Z, a.z_bf16, zo + 32 + 4 * g, out[4], out[5], out[6], out[7]);
            }
            if (threadIdx.x == 384) TRACE(17, m);
        }
    }
    // ---------------------------------------------------------------- teardown
    if (*abrt && warp == 1 && lane == 0) {
        mma_commit(&drain);
        mbar_drain(&drain, 0);
    }
    if (*abrt && warp == 0 && lane == 0) {
        // let the last loads land: every slot's most recent phase
        for (int c = NC - kSlots < 0 ? 0 : NC - kSlots; c < NC; ++c)
            mbar_drain(&tfull[c % kSlots], (c / kSlots) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 512);
#ifdef TTT_TRACE
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e < kTraceEvents * kTraceSteps; e += blockDim.x)
            g_ttt_trace[e] = trace_smem[e];
#endif
}

}  // namespace

bool linear_tc_supported(int d, int b, bool bf16) { return bf16 && d == kD && b == kMB; }

cudaError_t launch_linear_tc(const LinearArgs &a, cudaStream_t s, bool l2_keys) {
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmQ, tmV;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, kD, kChunkTok) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, kD, kChunkTok) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, kD, kChunkTok))
        return cudaErrorInvalidValue;
    auto kernel = l2_keys ? linear_ln_scan_kernel<true> : linear_ln_scan_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    Args args{a.eta, a.W0, a.gamma, a.beta, a.Z, a.W_out, a.H, a.T, a.ln, a.w0_per_seq,
              a.z_bf16, device_status_word()};
    kernel<<<a.B * a.H, kThreads, kSmemBytes, s>>>(tmK, tmQ, tmV, args);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

}  // namespace ttt

#ifdef TTT_TRACE
extern "C" __attribute__((visibility("default"))) int ttt_trace_fetch(unsigned *host, int n) {
    const int cap = kTraceEvents * kTraceSteps;
    return cudaMemcpyFromSymbol(host, g_ttt_trace, sizeof(unsigned) * (n < cap ? n : cap)) ==
                   cudaSuccess
               ? 0
               : -1;
}
#endif
