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
// the tensor cores can form P_{m+1} = K_{m+1} W_m one mini-batch ahead; the
// critical chain per mini-batch is one 16x16 by 16x64 correction plus the
// LayerNorm backward, done in fp32 on CUDA cores by the scan warps.
//
// Warp roles (16 warps):
//   0      TMA producer: K, Q, V in chunks of 128 tokens (3-slot ring)
//   1      MMA issuer (one thread) and tensor-memory owner
//   4-7    scan: X = P - C G_prev, LayerNorm backward, G (fp32 + bf16 hi/lo)
//   8-11   W re-emit: fp32 W from tensor memory -> bf16 hi/lo operand in smem;
//          warp 8 also copies P and C out of tensor memory for the scan
//   12-15  output: Zpre = Q W - tril(S) G, LayerNorm + residual, store Z
// Precision: Q/K/V enter exactly (bf16); every other operand (W, G) enters
// the tensor cores as two bf16 terms hi + lo, accumulation is fp32, and the
// chain's corrections and all LayerNorm math are fp32.
#include "sm100.cuh"
#include "ttt_common.cuh"

// Optional pipeline trace: compiled in only when TTT_TRACE is defined (a
// profiling build); records SM clock stamps of block 0 at each hand-off.
#ifdef TTT_TRACE
__device__ long long g_ttt_trace[32 * 256];
#define TRACE(ev, i)                                                                   \
    do {                                                                               \
        if (blockIdx.x == 0 && (i) < 256) g_ttt_trace[(ev) * 256 + (i)] = clock64(); \
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
constexpr int kChunkTok = 128, kMbPerChunk = kChunkTok / kMB, kSlots = 3;
constexpr int kTile = kChunkTok * kD * 2;  // 16 KB per tensor per chunk
constexpr int kThreads = 512;

// Shared memory map (offsets from a 1024-aligned base).
constexpr int OFF_K = 0;                               // K ring + 48 rows of slack
constexpr int OFF_Q = OFF_K + kSlots * kTile + 6144;   // Q ring + slack
constexpr int OFF_V = OFF_Q + kSlots * kTile + 6144;   // V ring
constexpr int OFF_W = OFF_V + kSlots * kTile;          // W hi | lo (MN-major, 8 KB each)
constexpr int OFF_G = OFF_W + 16384;                   // -G hi | lo, 2 buffers (2 KB each)
constexpr int OFF_PF = OFF_G + 8192;                   // P fp32 [2][16][68]
constexpr int OFF_CF = OFF_PF + 2 * 16 * 68 * 4;       // C fp32 [2][16][17]
constexpr int OFF_GF = OFF_CF + 2 * 16 * 17 * 4;       // G fp32 [4][16][64]
constexpr int OFF_ZQ = OFF_GF + 4 * 16 * 64 * 4;       // Q W fp32 [16][68]
constexpr int OFF_SF = OFF_ZQ + 16 * 68 * 4;           // Q K^T fp32 [16][17]
constexpr int kSmemBytes = OFF_SF + 16 * 17 * 4 + 1024;
static_assert(OFF_Q % 1024 == 0 && OFF_V % 1024 == 0 && OFF_W % 1024 == 0 && OFF_G % 1024 == 0,
              "operand tiles need 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Tensor-memory columns (512 allocated; M = 64 accumulators use lanes 16w..).
constexpr uint32_t TM_W = 0, TM_P = 64, TM_Z = 192, TM_C = 320, TM_S = 352;

struct Args {
    const float *eta, *W0, *gamma, *beta;
    float *Z, *W_out;
    int H, T;
    bool ln, w0_per_seq;
    int *status;
};

__device__ __forceinline__ float sum8(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

// Mean and 1/sigma of a 64-value row spread over 8 lanes (8 values each):
// local mean and sum of squared deviations, merged pairwise across lanes
// (equal-count merge of Chan et al.), LayerNorm eps inside the root.
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

// 8 consecutive bf16 (columns 8g..8g+7) of row `row` of a 128-byte-swizzled
// [rows][64] tile, widened to fp32.
__device__ __forceinline__ void load_row8(const uint8_t *tile, int row, int g, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(tile + row * 128 + ((g ^ (row & 7)) << 4));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    linear_ln_scan_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmV, Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + OFF_K, *sQ = smem + OFF_Q, *sV = smem + OFF_V;
    uint8_t *sW = smem + OFF_W, *sG = smem + OFF_G;
    float *Pf = reinterpret_cast<float *>(smem + OFF_PF);
    float *Cf = reinterpret_cast<float *>(smem + OFF_CF);
    float *Gf = reinterpret_cast<float *>(smem + OFF_GF);
    float *Zqf = reinterpret_cast<float *>(smem + OFF_ZQ);
    float *Sf = reinterpret_cast<float *>(smem + OFF_SF);

    __shared__ uint64_t tfull[kSlots], tfree[kSlots], gready[4], efree[4], pcready[2], zsdone[2],
        zfree[2], wdone, wsm, pcdone, drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.x, head = seq % a.H;
    const int T = a.T, NM = T / kMB, NC = (T + kChunkTok - 1) / kChunkTok;
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
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pcready[i], 32);
            mbar_init(&zsdone[i], 1);
            mbar_init(&zfree[i], 32);
        }
        mbar_init(&wdone, 1);
        mbar_init(&wsm, 128);
        mbar_init(&pcdone, 1);
        mbar_init(&drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    volatile int *abrt = &abort_flag;

    // Address of mini-batch m's first row in a K or Q ring (16 rows = 2 KB).
    auto mb_row = [&](uint8_t *ring, int m) -> uint32_t {
        return smem_u32(ring) + ((m / kMbPerChunk) % kSlots) * kTile + (m % kMbPerChunk) * 2048;
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
            const uint32_t I_PW = make_idesc_bf16(64, 64, false, true);
            const uint32_t I_GRAM = make_idesc_bf16(64, 16, false, false);
            const uint32_t wb = smem_u32(sW), gb = smem_u32(sG);
            // D = A_window(64 rows from `arow`) * W   (W as hi + lo)
            auto issue_pw = [&](uint32_t d, uint32_t arow) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int p = 0; p < 2; ++p)
                        mma_bf16(d, make_sdesc(arow + 32 * k, 16, 1024, kSw128),
                                 make_sdesc(wb + p * 8192 + 2048 * k, 8192, 1024, kSw128), I_PW,
                                 (k | p) != 0);
            };
            // D = A_window(64 rows from `arow`) * (16 rows from `brow`)^T
            auto issue_gram = [&](uint32_t d, uint32_t arow, uint32_t brow) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(d, make_sdesc(arow + 32 * k, 16, 1024, kSw128),
                             make_sdesc(brow + 32 * k, 16, 1024, kSw128), I_GRAM, k != 0);
            };
            bool ok = mbar_wait(&tfull[0], 0, abrt, status, 32) && mbar_wait(&wsm, 0, abrt, status, 33);
            if (ok) {
                tc_fence_after();
                issue_pw(tm + TM_P, mb_row(sK, 0));                       // P_0 = K_0 W_0
                issue_pw(tm + TM_P + 64, mb_row(sK, 1));                  // P_1 = K_1 W_0
                issue_gram(tm + TM_C + 16, mb_row(sK, 1), mb_row(sK, 0));  // C_1 = K_1 K_0^T
                mma_commit(&pcdone);
                issue_pw(tm + TM_Z, mb_row(sQ, 0));                       // Q_0 W_0
                issue_gram(tm + TM_S, mb_row(sQ, 0), mb_row(sK, 0));      // Q_0 K_0^T
                mma_commit(&zsdone[0]);
            }
            for (int j = 0; ok && j < NM; ++j) {
                if (!mbar_wait(&gready[j & 3], (j >> 2) & 1, abrt, status, 34)) break;
                TRACE(0, j);
                tc_fence_after();
                // W_{j+1} = W_j + K_j^T (-G_j)
                const uint32_t krow = mb_row(sK, j);
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    mma_bf16(tm + TM_W, make_sdesc(krow, 8192, 1024, kSw128),
                             make_sdesc(gb + (j & 1) * 4096 + p * 2048, 2048, 1024, kSw128), I_UPD,
                             true);
                mma_commit(&wdone);
                TRACE(1, j);
                if (j % kMbPerChunk == kMbPerChunk - 1) mma_commit(&tfree[(j / kMbPerChunk) % kSlots]);
                if (j + 1 >= NM) break;
                if (!mbar_wait(&wsm, (j + 1) & 1, abrt, status, 35)) break;
                TRACE(2, j);
                tc_fence_after();
                if (j + 2 < NM) {
                    const int m = j + 2;
                    if (m % kMbPerChunk == 0) {
                        const int c = m / kMbPerChunk;
                        if (!mbar_wait(&tfull[c % kSlots], (c / kSlots) & 1, abrt, status, 36)) break;
                        tc_fence_after();
                    }
                    issue_pw(tm + TM_P + (m & 1) * 64, mb_row(sK, m));                    // P_{j+2}
                    issue_gram(tm + TM_C + (m & 1) * 16, mb_row(sK, m), mb_row(sK, m - 1));  // C_{j+2}
                    mma_commit(&pcdone);
                    TRACE(3, j);
                }
                const int m = j + 1;
                if (m >= 2 && !mbar_wait(&zfree[m & 1], ((m >> 1) - 1) & 1, abrt, status, 37)) break;
                tc_fence_after();
                issue_pw(tm + TM_Z + (m & 1) * 64, mb_row(sQ, m));                     // Q_m W_m
                issue_gram(tm + TM_S + (m & 1) * 16, mb_row(sQ, m), mb_row(sK, m));    // Q_m K_m^T
                mma_commit(&zsdone[m & 1]);
                TRACE(4, j);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ scan
        const int r = threadIdx.x - 128, t = r >> 3, g = r & 7;
        float gam[8], bet[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            gam[i] = a.ln ? a.gamma[head * kD + 8 * g + i] : 1.f;
            bet[i] = a.ln ? a.beta[head * kD + 8 * g + i] : 0.f;
        }
        float eta_next = a.eta[tok0 + t];
        for (int j = 0; j < NM; ++j) {
            const float eta = eta_next;
            if (j + 1 < NM) eta_next = a.eta[tok0 + (long)(j + 1) * kMB + t];
            if (j % kMbPerChunk == 0) {
                const int c = j / kMbPerChunk;
                if (!mbar_wait_warp(&tfull[c % kSlots], (c / kSlots) & 1, abrt, status, 41)) break;
            }
            if (!mbar_wait_warp(&pcready[j & 1], (j >> 1) & 1, abrt, status, 42)) break;
            if (threadIdx.x == 128) TRACE(5, j);
            float x[8];
            {
                const float4 *p4 = reinterpret_cast<const float4 *>(Pf + ((j & 1) * 16 + t) * 68 + 8 * g);
                const float4 u0 = p4[0], u1 = p4[1];
                x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w;
                x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
            }
            if (j > 0) {  // X_j = P_j - C_j G_{j-1}
                const float *crow = Cf + ((j & 1) * 16 + t) * 17;
                const float *gprev = Gf + ((j - 1) & 3) * 1024 + 8 * g;
#pragma unroll
                for (int s = 0; s < kMB; ++s) {
                    const float c = crow[s];
                    const float4 *g4 = reinterpret_cast<const float4 *>(gprev + s * kD);
                    const float4 u0 = g4[0], u1 = g4[1];
                    x[0] = fmaf(-c, u0.x, x[0]); x[1] = fmaf(-c, u0.y, x[1]);
                    x[2] = fmaf(-c, u0.z, x[2]); x[3] = fmaf(-c, u0.w, x[3]);
                    x[4] = fmaf(-c, u1.x, x[4]); x[5] = fmaf(-c, u1.y, x[5]);
                    x[6] = fmaf(-c, u1.z, x[6]); x[7] = fmaf(-c, u1.w, x[7]);
                }
            }
            const int row = (j % kMbPerChunk) * kMB + t;
            const int slot = (j / kMbPerChunk) % kSlots;
            float kv[8], vv[8], G[8];
            load_row8(sV + slot * kTile, row, g, vv);
            if (a.ln) {
                load_row8(sK + slot * kTile, row, g, kv);
                float mu, rstd;
                row_stats(x, mu, rstd);
                float xh[8], gh[8], s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    xh[i] = (x[i] - mu) * rstd;
                    gh[i] = gam[i] * (kv[i] + gam[i] * xh[i] + bet[i] - vv[i]);
                    s1 += gh[i];
                    s2 = fmaf(gh[i], xh[i], s2);
                }
                s1 = sum8(s1) * (1.f / kD);
                s2 = sum8(s2) * (1.f / kD);
                const float sc = eta * rstd;
#pragma unroll
                for (int i = 0; i < 8; ++i) G[i] = sc * (gh[i] - s1 - xh[i] * s2);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) G[i] = eta * (x[i] - vv[i]);
            }
            if (j >= 4 && !mbar_wait_warp(&efree[j & 3], ((j >> 2) - 1) & 1, abrt, status, 43)) break;
            float4 *gf4 = reinterpret_cast<float4 *>(Gf + (j & 3) * 1024 + t * kD + 8 * g);
            gf4[0] = make_float4(G[0], G[1], G[2], G[3]);
            gf4[1] = make_float4(G[4], G[5], G[6], G[7]);
            // -G as bf16 hi + lo, MN-major rows = tokens: one 16-byte chunk each.
            uint4 hi, lo;
            __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(&hi);
            __nv_bfloat16 *l = reinterpret_cast<__nv_bfloat16 *>(&lo);
#pragma unroll
            for (int i = 0; i < 8; ++i) split_bf16(-G[i], h[i], l[i]);
            const uint32_t off = off_mnmajor_sw128(t, 8 * g, kMB);
            *reinterpret_cast<uint4 *>(sG + (j & 1) * 4096 + off) = hi;
            *reinterpret_cast<uint4 *>(sG + (j & 1) * 4096 + 2048 + off) = lo;
            fence_async_smem();
            mbar_arrive(&gready[j & 3]);
            if (threadIdx.x == 128) TRACE(6, j);
        }
    } else if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------ W re-emit
        const int q = warp & 3;  // subpartition: W rows 16q..16q+15 in lanes 32q..32q+15
        const int row = 16 * q + (lane & 15);
        const bool live = lane < 16;
        const uint32_t wl = taddr(tm, 32 * q, TM_W);
        auto emit = [&](const float (&w)[64]) {
            if (live) {
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    uint4 hi, lo;
                    __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(&hi);
                    __nv_bfloat16 *l = reinterpret_cast<__nv_bfloat16 *>(&lo);
#pragma unroll
                    for (int i = 0; i < 8; ++i) split_bf16(w[8 * c8 + i], h[i], l[i]);
                    const uint32_t off = off_mnmajor_sw128(row, 8 * c8, kD);
                    *reinterpret_cast<uint4 *>(sW + off) = hi;
                    *reinterpret_cast<uint4 *>(sW + 8192 + off) = lo;
                }
            }
            fence_async_smem();
        };
        auto load_w = [&](float (&w)[64]) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[16];
                tmem_ld16(wl + 16 * c, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) w[16 * c + i] = v[i];
            }
            tmem_ld_wait();
        };
        // P_m and C_m (rows 0-15 of their accumulators, lanes 0-15) -> smem.
        auto copy_pc = [&](int m, bool with_c) {
            float v[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                tmem_ld16(taddr(tm, 0, TM_P + (m & 1) * 64 + 16 * c), v);
                tmem_ld_wait();
                if (lane < 16) {
                    float4 *d4 = reinterpret_cast<float4 *>(Pf + ((m & 1) * 16 + lane) * 68 + 16 * c);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
            if (with_c) {
                tmem_ld16(taddr(tm, 0, TM_C + (m & 1) * 16), v);
                tmem_ld_wait();
                if (lane < 16)
#pragma unroll
                    for (int i = 0; i < 16; ++i) Cf[((m & 1) * 16 + lane) * 17 + i] = v[i];
            }
            tc_fence_before();
            mbar_arrive(&pcready[m & 1]);
        };
        {  // initial weight -> tensor memory (fp32) and the bf16 operand
            const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : head) * kD * kD;
            float w[64];
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float4 u = live ? *reinterpret_cast<const float4 *>(W0 + row * kD + c)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                w[c] = u.x; w[c + 1] = u.y; w[c + 2] = u.z; w[c + 3] = u.w;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = w[16 * c + i];
                tmem_st16(wl + 16 * c, v);
            }
            tmem_st_wait();
            emit(w);
            tc_fence_before();
            mbar_arrive(&wsm);
        }
        bool ok = true;
        if (warp == 8) {
            ok = mbar_wait_warp(&pcdone, 0, abrt, status, 51);
            if (ok) {
                tc_fence_after();
                copy_pc(0, false);
                copy_pc(1, true);
            }
        }
        for (int j = 0; ok && j < NM; ++j) {
            if (!mbar_wait_warp(&wdone, j & 1, abrt, status, 52)) break;
            if (lane == 0) TRACE(7 + q, j);
            tc_fence_after();
            float w[64];
            load_w(w);
            if (j + 1 < NM) {
                emit(w);
                tc_fence_before();
                mbar_arrive(&wsm);
                if (lane == 0) TRACE(11 + q, j);
            } else if (a.W_out && live) {
                float *dst = a.W_out + (size_t)seq * kD * kD + row * kD;
#pragma unroll
                for (int c = 0; c < 64; c += 4)
                    *reinterpret_cast<float4 *>(dst + c) = make_float4(w[c], w[c + 1], w[c + 2], w[c + 3]);
            }
            if (warp == 8 && j + 2 < NM) {
                if (!mbar_wait_warp(&pcdone, (j + 1) & 1, abrt, status, 53)) break;
                if (lane == 0) TRACE(15, j);
                tc_fence_after();
                copy_pc(j + 2, true);
                if (lane == 0) TRACE(16, j);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------ output
        const int r = threadIdx.x - 384, t = r >> 3, g = r & 7;
        float gam[8], bet[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            gam[i] = a.ln ? a.gamma[head * kD + 8 * g + i] : 1.f;
            bet[i] = a.ln ? a.beta[head * kD + 8 * g + i] : 0.f;
        }
        for (int m = 0; m < NM; ++m) {
            // Every wait below is warp-uniform, and the group of four output
            // warps leaves the loop together (named_bar_or), so an abort can
            // never strand part of the group at a barrier.
            bool bad = false;
            if (m % kMbPerChunk == 0) {
                const int c = m / kMbPerChunk;
                bad = !mbar_wait_warp(&tfull[c % kSlots], (c / kSlots) & 1, abrt, status, 61);
            }
            if (warp == 12 && !bad) {  // Q_m W_m and Q_m K_m^T out of tensor memory (lanes 0-15)
                bad = !mbar_wait_warp(&zsdone[m & 1], (m >> 1) & 1, abrt, status, 62);
                if (!bad) {
                    tc_fence_after();
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        tmem_ld16(taddr(tm, 0, TM_Z + (m & 1) * 64 + 16 * c), v);
                        tmem_ld_wait();
                        if (lane < 16) {
                            float4 *d4 = reinterpret_cast<float4 *>(Zqf + lane * 68 + 16 * c);
#pragma unroll
                            for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        }
                    }
                    tmem_ld16(taddr(tm, 0, TM_S + (m & 1) * 16), v);
                    tmem_ld_wait();
                    if (lane < 16)
#pragma unroll
                        for (int i = 0; i < 16; ++i) Sf[lane * 17 + i] = v[i];
                    tc_fence_before();
                    mbar_arrive(&zfree[m & 1]);
                }
            }
            if (named_bar_or(1, 128, bad || *abrt != 0)) break;
            if (threadIdx.x == 384) TRACE(17, m);
            bad = !mbar_wait_warp(&gready[m & 3], (m >> 2) & 1, abrt, status, 63);
            if (threadIdx.x == 384) TRACE(18, m);
            if (!bad) {
                float zp[8];
                {
                    const float4 *z4 = reinterpret_cast<const float4 *>(Zqf + t * 68 + 8 * g);
                    const float4 u0 = z4[0], u1 = z4[1];
                    zp[0] = u0.x; zp[1] = u0.y; zp[2] = u0.z; zp[3] = u0.w;
                    zp[4] = u1.x; zp[5] = u1.y; zp[6] = u1.z; zp[7] = u1.w;
                }
                const float *gm = Gf + (m & 3) * 1024 + 8 * g;
                for (int s = 0; s <= t; ++s) {  // - tril(Q K^T) G, diagonal included
                    const float c = Sf[t * 17 + s];
                    const float4 *g4 = reinterpret_cast<const float4 *>(gm + s * kD);
                    const float4 u0 = g4[0], u1 = g4[1];
                    zp[0] = fmaf(-c, u0.x, zp[0]); zp[1] = fmaf(-c, u0.y, zp[1]);
                    zp[2] = fmaf(-c, u0.z, zp[2]); zp[3] = fmaf(-c, u0.w, zp[3]);
                    zp[4] = fmaf(-c, u1.x, zp[4]); zp[5] = fmaf(-c, u1.y, zp[5]);
                    zp[6] = fmaf(-c, u1.z, zp[6]); zp[7] = fmaf(-c, u1.w, zp[7]);
                }
                float out[8];
                if (a.ln) {
                    float qv[8];
                    load_row8(sQ + ((m / kMbPerChunk) % kSlots) * kTile, (m % kMbPerChunk) * kMB + t, g, qv);
                    float mu, rstd;
                    row_stats(zp, mu, rstd);
#pragma unroll
                    for (int i = 0; i < 8; ++i) out[i] = qv[i] + gam[i] * ((zp[i] - mu) * rstd) + bet[i];
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) out[i] = zp[i];
                }
                float4 *zo = reinterpret_cast<float4 *>(a.Z + (tok0 + (long)m * kMB + t) * kD + 8 * g);
                zo[0] = make_float4(out[0], out[1], out[2], out[3]);
                zo[1] = make_float4(out[4], out[5], out[6], out[7]);
                mbar_arrive(&efree[m & 3]);
                if (m % kMbPerChunk == kMbPerChunk - 1) mbar_arrive(&tfree[(m / kMbPerChunk) % kSlots]);
            }
            if (named_bar_or(1, 128, bad)) break;
            if (threadIdx.x == 384) TRACE(19, m);
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
}

}  // namespace

bool linear_tc_supported(int d, int b, bool bf16) { return bf16 && d == kD && b == kMB; }

cudaError_t launch_linear_tc(const LinearArgs &a, cudaStream_t s) {
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmQ, tmV;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, kD, kChunkTok) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, kD, kChunkTok) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, kD, kChunkTok))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(linear_ln_scan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Args args{a.eta, a.W0, a.gamma, a.beta, a.Z, a.W_out, a.H, a.T, a.ln, a.w0_per_seq,
              device_status_word()};
    linear_ln_scan_kernel<<<a.B * a.H, kThreads, kSmemBytes, s>>>(tmK, tmQ, tmV, args);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

}  // namespace ttt

#ifdef TTT_TRACE
extern "C" __attribute__((visibility("default"))) int ttt_trace_fetch(long long *host, int n) {
    return cudaMemcpyFromSymbol(host, g_ttt_trace, sizeof(long long) * (n < 32 * 256 ? n : 32 * 256)) ==
                   cudaSuccess
               ? 0
               : -1;
}
#endif
