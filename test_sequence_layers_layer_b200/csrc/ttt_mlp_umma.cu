// ttt_mlp_umma.cu -- TTT-MLP (d = 64, hidden 256, mini-batch b = 16, bf16 Q/K/V)
// on the fifth-generation tensor cores: one thread block per (batch, head)
// sequence scans all mini-batches; every dense product of the dual form is a
// tcgen05.mma issued by one thread, with operands in shared memory (fed by TMA
// for Q/K/V) and fp32 accumulators in tensor memory.
//
// Method ("Test-Time Training: Linear Complexity Beyond Attention", the dual
// form of "Key Architectural Mechanics of TTT-Linear", applied to the
// multi-layer-perceptron hidden state of "How to Master Test-Time Training for
// LLMs"). With f(x) = x + LN(GELU(x W1) W2) and the mini-batch's starting
// weights W1_m, W2_m:
//   H  = K W1_m,  A = GELU(H),  X = A W2_m
//   Gx = diag(eta) dl/dX          (LayerNorm backward of f(K) - V)
//   Gh = (Gx W2_m^T) * GELU'(H)
//   Hq = Q W1_m - tril(Q K^T) Gh,  Aq = GELU(Hq)
//   W1_{m+1} = W1_m - K^T Gh,  W2_{m+1} = W2_m - A^T Gx
//   Zpre = Aq W2_m - tril(Aq A^T) Gx,  Z = Q + LN(Zpre)      (tril keeps the diagonal)
// Since Aq W2_m = Aq W2_{m+1} + (Aq A^T) Gx, the read-out can use the NEXT
// weights: Zpre = Aq W2_{m+1} + striu(Aq A^T) Gx (strictly upper part, s > t).
// The scan uses that form: the read-out of mini-batch m - 1 shares one product
// with the key side of mini-batch m,
//   [X_m | Aq_{m-1} W2_m] = W2_m^T [A_m ; Aq_{m-1}]^T,
// so every product that sets the weights and the read-out's weight product
// run as one tensor-core group per mini-batch.
//
// Products per mini-batch (hidden units on the MMA's M side: 2 x M=128):
//   H^T | Hq0^T = W1^T [K_m ; Q_m]^T            M=256 N=32 K=64   (W1 hi, lo)
//   [X | Xq]^T  = W2^T [A_m ; Aq_{m-1}]^T       M=64  N=32 K=256  (3 hi/lo terms)
//   Gx W2^T     = W2 Gx^T                        M=256 N=16 K=64   (3 terms)
//   dW1^T       = Gh^T K_m                       M=256 N=64 K=16   (Gh hi, lo)
//   dW2         = A_m^T Gx                       M=256 N=64 K=16   (3 terms)
//   S2^T        = [A_m ; ..] Aq_m^T              M=64  N=16 K=256  (3 terms)
// The causal correction of Hq (16 x 16 by 16 x 256) is done on CUDA cores.
// Precision: Q/K/V enter the tensor cores exactly (bf16); every other operand
// (weights, activations, gradients) enters as two bf16 terms hi + lo (hi =
// truncation, lo = RN(x - hi)); accumulation is fp32. The fp32 master weights
// live in registers; each mini-batch's increments are accumulated from zero in
// tensor memory and added in fp32, then the weights are re-emitted as hi/lo
// operand images.
//
// Thread layout: 16 warps. Warp w reads tensor-memory subpartition w % 4; it
// owns hidden unit j = 128 ((w / 4) % 2) + 32 (w % 4) + lane and, of that
// unit's columns, half hh = w / 8 (tokens 8 hh .. 8 hh + 7, weight columns
// 32 hh .. 32 hh + 31). For token-wise LayerNorm work warp w owns token w.
// Thread 0 also issues the TMA loads and the MMAs; phases are separated by
// block barriers and by mbarriers the MMAs commit to.
#include "sm100.cuh"
#include "ttt_common.cuh"
#include "ttt_gelu.cuh"

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 64, kDH = 256, kMB = 16;
constexpr int kThreads = 512;
constexpr int kSlots = 3, kTile = kMB * kD * 2;  // one [16][64] bf16 tile: 2 KB
constexpr int kSlotBytes = 3 * kTile;            // K | Q | V

// Shared memory (offsets from a 1024-aligned base).
//   W1I, W2I: weight images, [j][i] bf16, 128-byte swizzle, rows of 128 bytes;
//     hi at +0, lo at +32 KB. As W1^T (M=j, K=i) and W2 (M=j, K=i) they are
//     K-major; as W2^T (M=i, K=j) the same bytes are MN-major.
//   ACT: activation image [n][j] bf16 (n: token rows 0-15 A_m, 16-31 Aq),
//     K-major 128-byte swizzle in four 64-column blocks of 4 KB; hi, lo.
//     Rows 0-15 read as A_m^T (M=j, K=t) are the same bytes MN-major.
//     The S2 product reads 64 rows from the block start (rows 32-63 land in
//     the next block or the next buffer and are never used).
//   GHI: Gh^T image [j][s] bf16, K-major without swizzle (8 x 8 core
//     matrices; 8-row groups 256 bytes apart, the two 8-column halves 128
//     bytes apart); hi, lo.
//   GXI: Gx image [t][i] bf16, 128-byte swizzle; K-major for Gx W2^T,
//     MN-major for A^T Gx; hi, lo.
//   TILES: TMA ring, 3 slots of K | Q | V ([16][64] bf16, 128-byte swizzle).
constexpr int OFF_W1I = 0;
constexpr int OFF_W2I = OFF_W1I + 65536;
constexpr int OFF_ACT = OFF_W2I + 65536;
constexpr int kActBytes = 16384;
constexpr int OFF_GHI = OFF_ACT + 2 * kActBytes;  // also the over-read tail of ACT lo
constexpr int kGhBytes = 8192;
constexpr int OFF_GXI = OFF_GHI + 2 * kGhBytes;
constexpr int OFF_TILES = OFF_GXI + 2 * kTile;
constexpr int OFF_XS = OFF_TILES + kSlots * kSlotBytes;  // X fp32 [16][64]
constexpr int OFF_XQS = OFF_XS + kMB * kD * 4;           // Aq W2 fp32 [16][64]
constexpr int OFF_GXF = OFF_XQS + kMB * kD * 4;          // Gx fp32 [2][16][64]
constexpr int OFF_S1F = OFF_GXF + 2 * kMB * kD * 4;      // tril(Q K^T) fp32 [16][16]
constexpr int OFF_S2F = OFF_S1F + kMB * kMB * 4;         // S2[t][s] = Aq_t . A_s fp32
constexpr int OFF_BAR = OFF_S2F + kMB * kMB * 4;
constexpr int kSmemBytes = OFF_BAR + 128 + 1024;
static_assert(OFF_W2I % 1024 == 0 && OFF_ACT % 1024 == 0 && OFF_GXI % 1024 == 0 &&
                  OFF_TILES % 1024 == 0 && kSlotBytes % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
// The S2 product reads 64 rows (8 KB) from the start of each 4 KB column
// block of ACT: 4 KB past the end of the lo image, inside GHI.
static_assert(OFF_TILES - (OFF_ACT + 2 * kActBytes) >= 4096, "S2 over-read stays in shared memory");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Tensor-memory columns (512 allocated). M=128 accumulators keep row r in
// lane r; the two 128-row halves of an M=256 product sit side by side. M=64
// accumulators keep row r in lane 32 (r / 16) + r % 16.
constexpr uint32_t TM_H = 0;      // H^T | Hq0^T: 2 x 32 columns
constexpr uint32_t TM_X = 64;     // [X | Xq]^T: 32 columns (M=64)
constexpr uint32_t TM_S = 96;     // S2^T: 16 columns (M=64)
constexpr uint32_t TM_G = 112;    // (W2 Gx^T): 2 x 16 columns
constexpr uint32_t TM_DW1 = 256;  // dW1^T: 2 x 64 columns
constexpr uint32_t TM_DW2 = 384;  // dW2: 2 x 64 columns

struct Args {
    const float *eta, *W1_0, *W2_0, *gamma, *beta;
    float *Z, *W1_out, *W2_out;
    int H, T;
    bool w0_per_seq, z_bf16;
    int *status;
};

// Byte offset of element (n, k) of the activation image (one of hi / lo).
__device__ __forceinline__ uint32_t act_off(int n, int k) {
    return (uint32_t)((k >> 6) * 4096 + (n >> 3) * 1024 + (n & 7) * 128 +
                      ((((k & 63) >> 3) ^ (n & 7)) << 4) + (k & 7) * 2);
}

// Byte offset of the bf16 pair (columns 2 l, 2 l + 1) of row t of a [16][64]
// 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t pair_off(int t, int l) {
    return (uint32_t)(t * 128 + (((l >> 2) ^ (t & 7)) << 4) + (l & 3) * 4);
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
}

__device__ __forceinline__ uint16_t bf16_bits(__nv_bfloat16 x) {
    return *reinterpret_cast<const uint16_t *>(&x);
}

// hi (truncation) and lo = RN(x - hi) of one value, as bf16 bit patterns.
__device__ __forceinline__ void split1(float x, uint16_t &hi, uint16_t &lo) {
    const uint32_t u = __float_as_uint(x) & 0xFFFF0000u;
    hi = (uint16_t)(u >> 16);
    lo = bf16_bits(__float2bfloat16_rn(x - __uint_as_float(u)));
}

// Writes 16 consecutive weight columns (chunks c0, c0 + 1 of 8 columns) of
// row j of a weight image pair (hi at img, lo at img + 32 KB).
__device__ __forceinline__ void emit16(uint8_t *img, int j, int c0, const float *w) {
    const int blk = j >> 7, jj = j & 127;
    uint8_t *row = img + blk * 16384 + (jj >> 3) * 1024 + (jj & 7) * 128;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint4 h, l;
        split2(w[8 * c + 0], w[8 * c + 1], h.x, l.x);
        split2(w[8 * c + 2], w[8 * c + 3], h.y, l.y);
        split2(w[8 * c + 4], w[8 * c + 5], h.z, l.z);
        split2(w[8 * c + 6], w[8 * c + 7], h.w, l.w);
        const uint32_t off = (uint32_t)(((c0 + c) ^ (jj & 7)) << 4);
        *reinterpret_cast<uint4 *>(row + off) = h;
        *reinterpret_cast<uint4 *>(row + 32768 + off) = l;
    }
}

// Mean and 1/sigma of a 64-value row held two values per lane (Chan et al.'s
// pairwise update over the butterfly), LayerNorm eps inside the root.
__device__ __forceinline__ void row_stats64(float x0, float x1, float &mu, float &rstd) {
    float m = 0.5f * (x0 + x1);
    float M2 = (x0 - m) * (x0 - m) + (x1 - m) * (x1 - m);
#pragma unroll
    for (int o = 1, n = 2; o < 32; o <<= 1, n <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float M2o = __shfl_xor_sync(0xffffffffu, M2, o);
        const float dl = mo - m;
        m = 0.5f * (m + mo);
        M2 = (M2 + M2o) + dl * dl * (0.5f * n);
    }
    mu = m;
    rstd = rsqrtf(M2 * (1.f / kD) + kLnEps);
}

__device__ __forceinline__ void warp_sum2(float &a, float &b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
}

// Shared-memory descriptors of the operand forms used here.
__device__ __forceinline__ uint64_t kdesc(uint32_t a) { return make_sdesc(a, 16, 1024, kSw128); }
__device__ __forceinline__ uint64_t mndesc(uint32_t a, uint32_t lbo) {
    return make_sdesc(a, lbo, 1024, kSw128);
}
__device__ __forceinline__ uint64_t nodesc(uint32_t a) { return make_sdesc(a, 128, 256, kSwNone); }

__global__ void __launch_bounds__(kThreads, 1)
    mlp_umma_scan_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmV, Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, blk = (warp >> 2) & 1, hh = warp >> 3;
    const int j = 128 * blk + 32 * sp + lane;
    const int seq = blockIdx.x, h = seq % a.H, T = a.T, NM = T / kMB;
    const size_t row0 = (size_t)seq * T;
    int *status = a.status;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *barH = full + kSlots, *barX = barH + 1, *barG = barH + 2, *barW = barH + 3,
             *barS = barH + 4;
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(barH + 5);
    volatile int *abrt = reinterpret_cast<volatile int *>(tmem_base_s + 1);

    if (tid == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(&full[s], 1);
        for (int b = 0; b < 5; ++b) mbar_init(barH + b, 1);
        *abrt = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_base_s, 512);

    // Activation image starts at zero (its query rows feed the first product).
    for (int e = tid; e < 2 * kActBytes / 16; e += kThreads)
        reinterpret_cast<uint4 *>(smem + OFF_ACT)[e] = make_uint4(0, 0, 0, 0);

    // Master weights: w1[c] = W1[32 hh + c][j] (= W1^T[j][..]), w2[c] = W2[j][32 hh + c].
    const int widx = a.w0_per_seq ? seq : h;
    const float *W1g = a.W1_0 + (size_t)widx * kD * kDH;
    const float *W2g = a.W2_0 + (size_t)widx * kDH * kD;
    float w1[32], w2[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) w1[c] = W1g[(size_t)(32 * hh + c) * kDH + j];
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
        const float4 u = *reinterpret_cast<const float4 *>(W2g + (size_t)j * kD + 32 * hh + c);
        w2[c] = u.x;
        w2[c + 1] = u.y;
        w2[c + 2] = u.z;
        w2[c + 3] = u.w;
    }
    emit16(smem + OFF_W1I, j, 4 * hh, w1);
    emit16(smem + OFF_W1I, j, 4 * hh + 2, w1 + 16);
    emit16(smem + OFF_W2I, j, 4 * hh, w2);
    emit16(smem + OFF_W2I, j, 4 * hh + 2, w2 + 16);
    const float2 gam = make_float2(a.gamma[(size_t)h * kD + 2 * lane], a.gamma[(size_t)h * kD + 2 * lane + 1]);
    const float2 bet = make_float2(a.beta[(size_t)h * kD + 2 * lane], a.beta[(size_t)h * kD + 2 * lane + 1]);
    // eta of this warp's token in mini-batches m and m + 1
    float eta_c = a.eta[row0 + warp];
    float eta_n = NM > 1 ? a.eta[row0 + kMB + warp] : 0.f;

    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_base_s;

    // TMA producer and MMA issuer: thread 0.
    int issued = 0, waited = -1;  // tiles issued / waited for by thread 0
    uint32_t commits[5] = {0, 0, 0, 0, 0};
    auto issue_tile = [&](int i) {
        const int s = i % kSlots;
        uint8_t *dst = smem + OFF_TILES + s * kSlotBytes;
        const int y = (int)(row0 + (size_t)i * kMB);
        fence_async_smem();
        mbar_arrive_expect_tx(&full[s], kSlotBytes);
        tma_load_2d(dst, &tmK, 0, y, &full[s]);
        tma_load_2d(dst + kTile, &tmQ, 0, y, &full[s]);
        tma_load_2d(dst + 2 * kTile, &tmV, 0, y, &full[s]);
        issued = i + 1;
    };
    auto commit = [&](int b) {
        mma_commit(barH + b);
        ++commits[b];
    };
    if (tid == 0)
        for (int i = 0; i < kSlots && i < NM; ++i) issue_tile(i);

    const uint32_t sW1 = smem_u32(smem + OFF_W1I), sW2 = smem_u32(smem + OFF_W2I);
    const uint32_t sACT = smem_u32(smem + OFF_ACT), sGH = smem_u32(smem + OFF_GHI);
    const uint32_t sGX = smem_u32(smem + OFF_GXI);
    constexpr uint32_t I_H = make_idesc_bf16(128, 32, false, false);
    constexpr uint32_t I_X = make_idesc_bf16(64, 32, true, false);
    constexpr uint32_t I_G = make_idesc_bf16(128, 16, false, false);
    constexpr uint32_t I_DW1 = make_idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_DW2 = make_idesc_bf16(128, 64, true, true);
    constexpr uint32_t I_S = make_idesc_bf16(64, 16, false, false);
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;

    // [X | Xq]^T = W2^T [act rows 0-31]^T, 3 terms, K = 256 in 16 steps.
    auto issue_x = [&]() {
        for (int s = 0; s < 16; ++s) {
            const uint32_t bo = (uint32_t)((s >> 2) * 4096 + (s & 3) * 32);
            const uint32_t ao = (uint32_t)(2048 * s);
            mma_bf16(tb + TM_X, mndesc(sW2 + ao, 32768), kdesc(sACT + bo), I_X, s != 0);
            mma_bf16(tb + TM_X, mndesc(sW2 + ao, 32768), kdesc(sACT + kActBytes + bo), I_X, true);
            mma_bf16(tb + TM_X, mndesc(sW2 + 32768 + ao, 32768), kdesc(sACT + bo), I_X, true);
        }
        commit(1);
    };

    // LayerNorm forward of mini-batch i for this warp's token t = warp:
    // Zpre = Aq W2_{i+1} + sum_{s > t} S2[t][s] Gx_i[s];  Z = Q + LN(Zpre).
    auto ln_forward = [&](int i) {
        const int t = warp;
        const float *XQ = reinterpret_cast<const float *>(smem + OFF_XQS);
        const float *Gxf = reinterpret_cast<const float *>(smem + OFF_GXF) + (i & 1) * kMB * kD;
        const float *S2 = reinterpret_cast<const float *>(smem + OFF_S2F);
        float2 z = *reinterpret_cast<const float2 *>(XQ + t * kD + 2 * lane);
        for (int s = t + 1; s < kMB; ++s) {
            const float c = S2[t * kMB + s];
            const float2 g = *reinterpret_cast<const float2 *>(Gxf + s * kD + 2 * lane);
            z.x = fmaf(c, g.x, z.x);
            z.y = fmaf(c, g.y, z.y);
        }
        float mu, rstd;
        row_stats64(z.x, z.y, mu, rstd);
        const uint8_t *tile = smem + OFF_TILES + (i % kSlots) * kSlotBytes;
        const float2 qv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + kTile + pair_off(t, lane)));
        store_z2(a.Z, a.z_bf16, (row0 + (size_t)i * kMB + t) * kD + 2 * lane,
                 qv.x + gam.x * (z.x - mu) * rstd + bet.x, qv.y + gam.y * (z.y - mu) * rstd + bet.y);
    };

    // Staging of the read-out sums: Xq rows (and X rows) from the M=64
    // accumulator into [t][i] fp32; S2 from its accumulator into S2[t][s].
    auto stage_x = [&](bool want_x) {
        if (warp < 4) {
            float v[16];
            tmem_ld16_x2<16>(tb + ((uint32_t)(32 * warp) << 16) + TM_X, v);
            tmem_ld_wait();
            const int i = 16 * warp + (lane & 15);
            float *dst = reinterpret_cast<float *>(smem + (lane < 16 ? OFF_XS : OFF_XQS));
            if (lane >= 16 || want_x) {
#pragma unroll
                for (int t = 0; t < kMB; ++t) dst[t * kD + i] = v[t];
            }
        }
    };
    auto stage_s2 = [&]() {
        if (warp == 0) {
            float v[16];
            tmem_ld16(tb + TM_S, v);
            tmem_ld_wait();
            if (lane < kMB) {
                float *S2 = reinterpret_cast<float *>(smem + OFF_S2F);
#pragma unroll
                for (int t = 0; t < kMB; ++t) S2[t * kMB + lane] = v[t];
            }
        }
    };

    bool ok = true;
    int m = 0;
    for (; m < NM; ++m) {
        const uint32_t par = m & 1;
        const int slot = m % kSlots;
        uint8_t *tile = smem + OFF_TILES + slot * kSlotBytes;
        const uint32_t sK = smem_u32(tile);

        // ---- A: H^T | Hq0^T = W1^T [K ; Q]^T
        if (tid == 0) {
            ok = mbar_wait(&full[slot], (m / kSlots) & 1, abrt, status, 71);
            if (ok) {
                waited = m;
                tc_fence_after();
                for (int b = 0; b < 2; ++b)
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t ao = (uint32_t)(b * 16384 + 32 * k);
                        mma_bf16(tb + TM_H + 32 * b, kdesc(sW1 + ao), kdesc(sK + 32 * k), I_H, k != 0);
                        mma_bf16(tb + TM_H + 32 * b, kdesc(sW1 + 32768 + ao), kdesc(sK + 32 * k), I_H, true);
                    }
                commit(0);
            }
        }
        ok = ok && mbar_wait(&full[slot], (m / kSlots) & 1, abrt, status, 71);
        ok = ok && mbar_wait(barH, par, abrt, status, 72);
        if (m > 0) ok = ok && mbar_wait(barS, (m - 1) & 1, abrt, status, 76);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();

        // ---- 1: A = GELU(H), GELU'(H) for tokens 8 hh ..; S2 of m - 1; S1 = tril(Q K^T)
        float gp[8];
        if (ok) {
            float hv[8];
            tmem_ld8(tb + lane_base + TM_H + 32 * blk + 8 * hh, hv);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float av = gelu_and_prime(hv[e], gp[e]);
                uint16_t hi, lo;
                split1(av, hi, lo);
                const uint32_t off = act_off(8 * hh + e, j);
                *reinterpret_cast<uint16_t *>(smem + OFF_ACT + off) = hi;
                *reinterpret_cast<uint16_t *>(smem + OFF_ACT + kActBytes + off) = lo;
            }
            if (m > 0) stage_s2();
            if (tid < kMB * kMB) {
                const int t = tid >> 4, s = tid & 15;
                float acc = 0.f;
                if (s <= t) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 qv = *reinterpret_cast<const uint4 *>(tile + kTile + t * 128 + ((c ^ (t & 7)) << 4));
                        const uint4 kv = *reinterpret_cast<const uint4 *>(tile + s * 128 + ((c ^ (s & 7)) << 4));
                        const uint32_t qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const float2 x = bf2_to_f2(qa[p]), y = bf2_to_f2(ka[p]);
                            acc = fmaf(x.x, y.x, acc);
                            acc = fmaf(x.y, y.y, acc);
                        }
                    }
                }
                reinterpret_cast<float *>(smem + OFF_S1F)[tid] = acc;
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) break;

        // ---- B: [X | Xq]^T
        if (tid == 0) {
            tc_fence_after();
            issue_x();
        }
        ok = __all_sync(0xffffffffu, mbar_wait(barX, par, abrt, status, 73));
        tc_fence_after();
        if (ok) stage_x(true);
        tc_fence_before();
        if (__syncthreads_or(!ok)) break;

        // ---- 2: LayerNorm backward of token t = warp -> Gx (fp32 and hi/lo)
        {
            const int t = warp;
            const float *XS = reinterpret_cast<const float *>(smem + OFF_XS);
            const float2 x = *reinterpret_cast<const float2 *>(XS + t * kD + 2 * lane);
            float mu, rstd;
            row_stats64(x.x, x.y, mu, rstd);
            const uint32_t po = pair_off(t, lane);
            const float2 kv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + po));
            const float2 vv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + 2 * kTile + po));
            const float xh0 = (x.x - mu) * rstd, xh1 = (x.y - mu) * rstd;
            const float g0 = gam.x * (kv.x + gam.x * xh0 + bet.x - vv.x);
            const float g1 = gam.y * (kv.y + gam.y * xh1 + bet.y - vv.y);
            float m1 = g0 + g1, m2 = g0 * xh0 + g1 * xh1;
            warp_sum2(m1, m2);
            const float sc = eta_c * rstd, a1 = m1 * (1.f / kD), a2 = m2 * (1.f / kD);
            const float G0 = sc * (g0 - a1 - xh0 * a2), G1 = sc * (g1 - a1 - xh1 * a2);
            *reinterpret_cast<float2 *>(smem + OFF_GXF + (par * kMB * kD + t * kD + 2 * lane) * 4) =
                make_float2(G0, G1);
            uint32_t hi, lo;
            split2(G0, G1, hi, lo);
            *reinterpret_cast<uint32_t *>(smem + OFF_GXI + po) = hi;
            *reinterpret_cast<uint32_t *>(smem + OFF_GXI + kTile + po) = lo;
        }
        eta_c = eta_n;
        eta_n = m + 2 < NM ? a.eta[row0 + (size_t)(m + 2) * kMB + warp] : 0.f;
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- C: W2 Gx^T (3 terms); meanwhile the read-out of m - 1
        if (tid == 0) {
            tc_fence_after();
            for (int b = 0; b < 2; ++b)
                for (int k = 0; k < 4; ++k) {
                    const uint32_t ao = (uint32_t)(b * 16384 + 32 * k);
                    const uint32_t d = tb + TM_G + 16 * b;
                    mma_bf16(d, kdesc(sW2 + ao), kdesc(sGX + 32 * k), I_G, k != 0);
                    mma_bf16(d, kdesc(sW2 + ao), kdesc(sGX + kTile + 32 * k), I_G, true);
                    mma_bf16(d, kdesc(sW2 + 32768 + ao), kdesc(sGX + 32 * k), I_G, true);
                }
            commit(2);
        }
        if (m > 0) ln_forward(m - 1);
        ok = __all_sync(0xffffffffu, mbar_wait(barG, par, abrt, status, 74));
        tc_fence_after();

        // ---- 3a: Gh = (W2 Gx^T) * GELU'(H) -> Gh^T image
        float ghv[8];
        if (ok) {
            tmem_ld8(tb + lane_base + TM_G + 16 * blk + 8 * hh, ghv);
            tmem_ld_wait();
            uint4 hv, lv;
            uint32_t *hp = &hv.x, *lp = &lv.x;
#pragma unroll
            for (int e = 0; e < 8; ++e) ghv[e] *= gp[e];
#pragma unroll
            for (int p = 0; p < 4; ++p) split2(ghv[2 * p], ghv[2 * p + 1], hp[p], lp[p]);
            const uint32_t off = (uint32_t)((j >> 3) * 256 + hh * 128 + (j & 7) * 16);
            *reinterpret_cast<uint4 *>(smem + OFF_GHI + off) = hv;
            *reinterpret_cast<uint4 *>(smem + OFF_GHI + kGhBytes + off) = lv;
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) break;

        // ---- D: dW1^T = Gh^T K (2 terms), dW2 = A^T Gx (3 terms); next tile
        if (tid == 0) {
            tc_fence_after();
            for (int b = 0; b < 2; ++b) {
                const uint32_t d1 = tb + TM_DW1 + 64 * b, d2 = tb + TM_DW2 + 64 * b;
                const uint32_t go = (uint32_t)(b * 4096), ao = (uint32_t)(b * 8192);
                mma_bf16(d1, nodesc(sGH + go), mndesc(sK, 2048), I_DW1, false);
                mma_bf16(d1, nodesc(sGH + kGhBytes + go), mndesc(sK, 2048), I_DW1, true);
                mma_bf16(d2, mndesc(sACT + ao, 4096), mndesc(sGX, 2048), I_DW2, false);
                mma_bf16(d2, mndesc(sACT + ao, 4096), mndesc(sGX + kTile, 2048), I_DW2, true);
                mma_bf16(d2, mndesc(sACT + kActBytes + ao, 4096), mndesc(sGX, 2048), I_DW2, true);
            }
            commit(3);
            if (m >= 1 && m + 2 < NM) issue_tile(m + 2);
        }

        // ---- 3b: Hq = Hq0 - tril(Q K^T) Gh, Aq = GELU(Hq) -> act rows 16..31
        {
            float hq[8], gall[kMB];
            tmem_ld8(tb + lane_base + TM_H + 32 * blk + 16 + 8 * hh, hq);
            if (hh) {
                const uint32_t off = (uint32_t)((j >> 3) * 256 + (j & 7) * 16);
                const uint4 hv = *reinterpret_cast<const uint4 *>(smem + OFF_GHI + off);
                const uint4 lv = *reinterpret_cast<const uint4 *>(smem + OFF_GHI + kGhBytes + off);
                const uint32_t hp[4] = {hv.x, hv.y, hv.z, hv.w}, lp[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 x = bf2_to_f2(hp[p]), y = bf2_to_f2(lp[p]);
                    gall[2 * p] = x.x + y.x;
                    gall[2 * p + 1] = x.y + y.y;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) gall[8 + e] = ghv[e];
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gall[e] = ghv[e];
#pragma unroll
                for (int e = 0; e < 8; ++e) gall[8 + e] = 0.f;
            }
            tmem_ld_wait();
            const float *S1 = reinterpret_cast<const float *>(smem + OFF_S1F);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int t = 8 * hh + e;
                float c = 0.f;
#pragma unroll
                for (int s = 0; s < kMB; ++s)
                    if (s <= t) c = fmaf(S1[t * kMB + s], gall[s], c);
                const float aq = gelu(hq[e] - c);
                uint16_t hi, lo;
                split1(aq, hi, lo);
                const uint32_t off = act_off(kMB + t, j);
                *reinterpret_cast<uint16_t *>(smem + OFF_ACT + off) = hi;
                *reinterpret_cast<uint16_t *>(smem + OFF_ACT + kActBytes + off) = lo;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S2^T = [A_m ; ..] Aq_m^T (3 terms), finished by the next mini-batch
        if (tid == 0) {
            tc_fence_after();
            for (int s = 0; s < 16; ++s) {
                const uint32_t o = (uint32_t)((s >> 2) * 4096 + (s & 3) * 32);
                mma_bf16(tb + TM_S, kdesc(sACT + o), kdesc(sACT + 2048 + o), I_S, s != 0);
                mma_bf16(tb + TM_S, kdesc(sACT + o), kdesc(sACT + kActBytes + 2048 + o), I_S, true);
                mma_bf16(tb + TM_S, kdesc(sACT + kActBytes + o), kdesc(sACT + 2048 + o), I_S, true);
            }
            commit(4);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(barW, par, abrt, status, 75));
        tc_fence_after();

        // ---- 4: W1 -= dW1, W2 -= dW2 (fp32); re-emit the hi/lo images
        if (ok) {
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                float d1[16], d2[16];
                tmem_ld16(tb + lane_base + TM_DW1 + 64 * blk + 32 * hh + 16 * hc, d1);
                tmem_ld16(tb + lane_base + TM_DW2 + 64 * blk + 32 * hh + 16 * hc, d2);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    w1[16 * hc + c] -= d1[c];
                    w2[16 * hc + c] -= d2[c];
                }
                emit16(smem + OFF_W1I, j, 4 * hh + 2 * hc, w1 + 16 * hc);
                emit16(smem + OFF_W2I, j, 4 * hh + 2 * hc, w2 + 16 * hc);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) break;
    }

    bool done = ok && m == NM;
    if (done && NM > 0) {
        // Read-out of the last mini-batch: Aq W2_NM from one more product.
        if (tid == 0) {
            tc_fence_after();
            issue_x();
        }
        bool w = mbar_wait(barS, (NM - 1) & 1, abrt, status, 76);
        w = w && mbar_wait(barX, NM & 1, abrt, status, 77);
        done = __all_sync(0xffffffffu, w);
        tc_fence_after();
        if (done) {
            stage_x(false);
            stage_s2();
        }
        tc_fence_before();
        done = !__syncthreads_or(!done);
        if (done) ln_forward(NM - 1);
    }
    if (!done && tid == 0) {
        // Aborted: let this block's own tile loads and tensor-core work land.
        for (int i = waited + 1; i < issued; ++i) mbar_drain(&full[i % kSlots], (i / kSlots) & 1);
        for (int b = 0; b < 5; ++b)
            if (commits[b]) mbar_drain(barH + b, (commits[b] - 1) & 1);
    }
    if (done && a.W1_out) {
        float *o = a.W1_out + (size_t)seq * kD * kDH;
#pragma unroll
        for (int c = 0; c < 32; ++c) o[(size_t)(32 * hh + c) * kDH + j] = w1[c];
    }
    if (done && a.W2_out) {
        float *o = a.W2_out + (size_t)seq * kDH * kD + (size_t)j * kD + 32 * hh;
#pragma unroll
        for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4 *>(o + c) = make_float4(w2[c], w2[c + 1], w2[c + 2], w2[c + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

}  // namespace

cudaError_t launch_mlp_umma(const MlpArgs &a, cudaStream_t s) {
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmQ, tmV;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, kD, kMB) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, kD, kMB) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, kD, kMB))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(mlp_umma_scan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Args args{a.eta, a.W1_0, a.W2_0, a.gamma, a.beta, a.Z, a.W1_out, a.W2_out, a.H, a.T,
              a.w0_per_seq, a.z_bf16, device_status_word()};
    mlp_umma_scan_kernel<<<a.B * a.H, kThreads, kSmemBytes, s>>>(tmK, tmQ, tmV, args);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

}  // namespace ttt
