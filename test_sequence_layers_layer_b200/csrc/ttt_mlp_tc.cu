// ttt_mlp_tc.cu -- TTT-MLP (d = 64, hidden 256, mini-batch b = 16, bf16 Q/K/V)
// on the tensor cores with warp-level MMA: each (batch, head) sequence is
// scanned by one thread-block cluster whose CTAs keep both fast-weight layers
// resident in registers (fp32) for all mini-batches.
//
// Method ("Test-Time Training: Linear Complexity Beyond Attention", TTT-MLP;
// the dual form of "Key Architectural Mechanics of TTT-Linear" applied to
// each layer). With f(x) = x + LN(GELU(x W1) W2) and the mini-batch's
// starting weights W1, W2:
//   H  = K W1,  A = GELU(H),  X = A W2
//   Gx = diag(eta) dl/dX        (LayerNorm backward of f(K) - V)
//   Gh = (Gx W2^T) * GELU'(H)
//   Hq = Q W1 - tril(Q K^T) Gh,  Aq = GELU(Hq)
//   Z  = Q + LN( Aq W2 - tril(Aq A^T) Gx )
//   W1 <- W1 - K^T Gh,  W2 <- W2 - A^T Gx
// tril keeps the diagonal.
//
// Why warp-level MMA: every product here is 16 tokens tall and the scan is
// sequential over the mini-batches, so a product is a handful of 16 x 8 x 16
// tiles. Issued by 16 warps at once they stay in registers end to end; a
// single-thread tcgen05 issuer would serialise ~2600 tile products per
// mini-batch behind one thread.
//
// Work split: the 16 warps of a cluster (kCL CTAs of 16/kCL warps) each own
// 16 hidden units j: rows j of W1^T and of W2 as fp32 MMA accumulator
// fragments (64 registers a thread). Products whose contraction runs over
// the hidden units (X = A W2, Aq W2, Aq A^T) are summed across the 16 warps
// through the cluster's distributed shared memory; products over d or over
// tokens stay inside the warp. Each warp also owns one token of the
// mini-batch for the LayerNorm work.
//
// Per mini-batch m, one exchange between the CTAs (distributed shared memory
// round trips cost ~1000 cycles here, so the scan makes one per mini-batch):
//   wait A(m)   (cluster: every CTA's X sums of m and Zpre / S2 sums of m - 1)
//   LayerNorm backward of all 16 tokens, in every CTA (identical results):
//               X = sum of the CTAs' sums -> Gx (fp32 and bf16 hi/lo); arrive B
//   LayerNorm forward of m - 1 for the warp's own token (overlaps B):
//               Zpre = sums - tril(S2) Gx,  Z = Q + LN(Zpre)
//   wait B(m)   (CTA: Gx of m)
//   Gh^T = W2 Gx^T * GELU'(H);  S1 = tril(Q K^T)
//   Hq^T = Hq0^T - Gh^T S1^T;  Aq = GELU(Hq);  partials of Aq A^T and Aq W2
//   W1^T -= Gh^T K,  W2 -= A^T Gx (own rows)
//   H^T = W1^T K^T and Hq0^T = W1^T Q^T of m + 1, A = GELU(H), GELU'(H),
//               partial X = A W2
//   wait L      (CTA: all partials written)
//   sums of this CTA's partials per token, pushed to the CTAs that need
//               them; arrive A(m + 1) in every CTA
// Precision: Q/K/V enter exactly (bf16); every other operand enters as two
// bf16 terms hi + lo (hi*hi + hi*lo + lo*hi, fp32 accumulation); sums
// across warps, the causal correction of Zpre and all LayerNorm math are fp32.
// Small increments (the weight updates, the causal correction of Hq) are
// accumulated from zero and then added to the large value in fp32: the tensor
// core aligns each product to the accumulator's exponent and truncates, so
// accumulating them into the weight directly would drop most of the lo
// terms, always toward zero.
#include "sm100.cuh"
#include "ttt_common.cuh"
#include "ttt_gelu.cuh"

// Optional phase trace, compiled in only when TTT_TRACE is defined (a
// profiling build): lane 0 of warps 0 and 7 of block 0 store the SM clock at
// each phase boundary of the first kMlpTraceSteps mini-batches.
#ifdef TTT_TRACE
constexpr int kMlpTraceEvents = 24, kMlpTraceSteps = 128;
__device__ unsigned g_ttt_mlp_trace[2 * kMlpTraceEvents * kMlpTraceSteps];
#define MTRACE_AT(ev, i)                                                                        \
    do {                                                                                        \
        if (blockIdx.x == 0 && lane == 0 && (warp == 0 || warp == 7) && (i) >= 0 &&             \
            (i) < kMlpTraceSteps)                                                               \
            g_ttt_mlp_trace[((warp == 7) * kMlpTraceEvents + (ev)) * kMlpTraceSteps + (i)] =   \
                (unsigned)clock();                                                              \
    } while (0)
#else
#define MTRACE_AT(ev, i) \
    do {                 \
    } while (0)
#endif
#define MTRACE(ev) MTRACE_AT(ev, m)

namespace ttt {
namespace {

using namespace sm100;

constexpr int kD = 64, kDH = 256, kMB = 16;
constexpr int kWarpsTotal = kDH / 16;                // 16 hidden units per warp
constexpr int kSlots = 4, kTileBytes = kMB * kD * 2;  // 2 KB: one [16][64] bf16 tile
constexpr int kSlotBytes = 3 * kTileBytes;           // K | Q | V
constexpr int kS2Pitch = 24;                         // padded row of a 16x16 partial
constexpr int kPart = kMB * kD;                      // floats in one [16][64] partial
constexpr int kS2Part = kMB * kS2Pitch;              // floats in one 16x16 partial

// Shared memory map of one CTA of a kCL-CTA cluster (offsets from a
// 1024-aligned base). Tiles of bf16 [16][64] use the 128-byte swizzle:
// 16-byte chunk c of row t sits at chunk c ^ (t & 7).
template <int kCL>
struct Layout {
    static constexpr int kWarps = kWarpsTotal / kCL, kThreads = kWarps * 32;
    static constexpr int TILES = 0;                             // [slot][K | Q | V]
    static constexpr int GXB = TILES + kSlots * kSlotBytes;     // Gx hi | Gx lo tiles
    static constexpr int GXF = GXB + 2 * kTileBytes;            // Gx fp32 [2][16][64]
    // This CTA's warps' partials (swizzled [16][64] / padded [16][24])
    static constexpr int XP = GXF + 2 * kPart * 4;              // X   [warp][16][64]
    static constexpr int ZP = XP + kWarps * kPart * 4;          // Zpre [warp][16][64]
    static constexpr int S2P = ZP + kWarps * kPart * 4;         // S2  [warp][16][24]
    // Per-CTA sums of those partials (index: mini-batch parity, source CTA),
    // at the same offsets in every CTA: the source CTA writes its own slot
    // and copies it into the others.
    static constexpr int XS = S2P + kWarps * kS2Part * 4;       // X    [2][kCL][warp][kCL][64]
    static constexpr int ZS = XS + 2 * kCL * kPart * 4;         // Zpre [2][kCL][16][64]
    static constexpr int SS = ZS + 2 * kCL * kPart * 4;         // S2   [2][kCL][16][16]
    static constexpr int BAR = SS + 2 * kCL * kMB * kMB * 4;
    static constexpr int kSmemBytes = BAR + 128 + 1024;         // barriers + alignment slack
};

struct Args {
    const float *eta, *W1_0, *W2_0, *gamma, *beta;
    float *Z, *W1_out, *W2_out;
    int H, T;
    bool w0_per_seq, z_bf16;
    int *status;
};

// Byte offset, inside a swizzled [16][64] tile, of the row this lane feeds
// to ldmatrix.x4 for k-step ks: matrices (tokens 0-7 | 8-15) x (columns
// 16ks..+7 | 16ks+8..+15), in the order b0, b1 of token tile 0 then of token
// tile 1 (equally: a0, a2, a1, a3 of the tile as a 16x16 A operand).
__device__ __forceinline__ uint32_t frag_off(int ks, int lane) {
    const int mi = lane >> 3, r = lane & 7;
    const int t = 8 * (mi >> 1) + r, chunk = 2 * ks + (mi & 1);
    return t * 128 + ((chunk ^ r) << 4);
}

// Same tile read transposed (ldmatrix .trans) as the B operand [token][col]
// of two column tiles 2np, 2np+1: matrices (tokens 0-7, tile 2np),
// (8-15, 2np), (0-7, 2np+1), (8-15, 2np+1).
__device__ __forceinline__ uint32_t frag_off_t(int np, int lane) {
    const int mi = lane >> 3, r = lane & 7;
    const int t = r + 8 * (mi & 1), chunk = 2 * np + (mi >> 1);
    return t * 128 + ((chunk ^ r) << 4);
}

// Byte offset of the bf16 pair (columns 2*lane, 2*lane+1) of row t.
__device__ __forceinline__ uint32_t pair_off(int t, int lane) {
    return t * 128 + (((lane >> 2) ^ (t & 7)) << 4) + (lane & 3) * 4;
}

// fp32 [16][64] partial: element (t, i) at word t*64 + ((i/8 ^ (t&7)) * 8) + i%8.
__device__ __forceinline__ int part_idx(int t, int i) {
    return t * 64 + ((((i >> 3) ^ (t & 7))) << 3) + (i & 7);
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
}

// Mean and 1/sigma of N 64-value rows held two values per lane: each lane's
// mean and sum of squared deviations, merged pairwise across the warp
// (equal-count case of Chan, Golub and LeVeque's update; the N rows'
// butterflies interleaved), LayerNorm eps inside the root. Every lane ends
// with the same bits.
template <int N>
__device__ __forceinline__ void row_stats64(const float (&x0)[N], const float (&x1)[N],
                                            float (&mu)[N], float (&rstd)[N]) {
    float m[N], M2[N];
#pragma unroll
    for (int r = 0; r < N; ++r) {
        m[r] = 0.5f * (x0[r] + x1[r]);
        M2[r] = (x0[r] - m[r]) * (x0[r] - m[r]) + (x1[r] - m[r]) * (x1[r] - m[r]);
    }
#pragma unroll
    for (int o = 1, n = 2; o < 32; o <<= 1, n <<= 1) {
        float mo[N], M2o[N];
#pragma unroll
        for (int r = 0; r < N; ++r) {
            mo[r] = __shfl_xor_sync(0xffffffffu, m[r], o);
            M2o[r] = __shfl_xor_sync(0xffffffffu, M2[r], o);
        }
#pragma unroll
        for (int r = 0; r < N; ++r) {
            const float dl = mo[r] - m[r];
            m[r] = 0.5f * (m[r] + mo[r]);
            M2[r] = (M2[r] + M2o[r]) + dl * dl * (0.5f * n);
        }
    }
#pragma unroll
    for (int r = 0; r < N; ++r) {
        mu[r] = m[r];
        rstd[r] = rsqrtf(M2[r] * (1.f / kD) + kLnEps);
    }
}

__device__ __forceinline__ void row_stats64(float x0, float x1, float &mu, float &rstd) {
    const float a0[1] = {x0}, a1[1] = {x1};
    float m[1], r[1];
    row_stats64<1>(a0, a1, m, r);
    mu = m[0];
    rstd = r[0];
}

// Warp sums of 2N values at once (interleaved butterflies).
template <int N>
__device__ __forceinline__ void warp_sum2(float (&a)[N], float (&b)[N]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ao[N], bo[N];
#pragma unroll
        for (int r = 0; r < N; ++r) {
            ao[r] = __shfl_xor_sync(0xffffffffu, a[r], o);
            bo[r] = __shfl_xor_sync(0xffffffffu, b[r], o);
        }
#pragma unroll
        for (int r = 0; r < N; ++r) {
            a[r] += ao[r];
            b[r] += bo[r];
        }
    }
}

// Packs a warp's 16x16 block held as two D tiles (rows = this warp's hidden
// units, columns = tokens) into its A fragment, split into hi and lo.
__device__ __forceinline__ void pack_split(const float (&x)[2][4], uint32_t (&hi)[4],
                                           uint32_t (&lo)[4]) {
    split2(x[0][0], x[0][1], hi[0], lo[0]);
    split2(x[0][2], x[0][3], hi[1], lo[1]);
    split2(x[1][0], x[1][1], hi[2], lo[2]);
    split2(x[1][2], x[1][3], hi[3], lo[3]);
}

// A fragment of the transpose of a 16x16 block given as an A fragment.
__device__ __forceinline__ void transpose_a(const uint32_t (&a)[4], uint32_t (&t)[4]) {
    t[0] = movt(a[0]);
    t[1] = movt(a[2]);
    t[2] = movt(a[1]);
    t[3] = movt(a[3]);
}

// A fragment (hi, lo) of k-step ks of a state block held as 8 D tiles
// (16 rows x 64 columns).
__device__ __forceinline__ void state_a(const float (&w)[8][4], int ks, uint32_t (&hi)[4],
                                        uint32_t (&lo)[4]) {
    split2(w[2 * ks][0], w[2 * ks][1], hi[0], lo[0]);
    split2(w[2 * ks][2], w[2 * ks][3], hi[1], lo[1]);
    split2(w[2 * ks + 1][0], w[2 * ks + 1][1], hi[2], lo[2]);
    split2(w[2 * ks + 1][2], w[2 * ks + 1][3], hi[3], lo[3]);
}

// Partial [16 tokens][64] = Act[t][j] W2[j][i] over this warp's 16 hidden
// units (act = A fragment of Act, hi/lo), written to the swizzled partial.
__device__ __forceinline__ void partial_times_w2(const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                                 const float (&w2)[8][4], float *part, int g,
                                                 int q) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float acc[4][4];
#pragma unroll
        for (int n4 = 0; n4 < 4; ++n4) {
            const int ni = 4 * half + n4;
            acc[n4][0] = acc[n4][1] = acc[n4][2] = acc[n4][3] = 0.f;
            uint32_t bh0, bl0, bh1, bl1;
            split2(w2[ni][0], w2[ni][1], bh0, bl0);
            split2(w2[ni][2], w2[ni][3], bh1, bl1);
            bh0 = movt(bh0);
            bl0 = movt(bl0);
            bh1 = movt(bh1);
            bl1 = movt(bl1);
            mma16816(acc[n4], ah, bh0, bh1);
            mma16816(acc[n4], ah, bl0, bl1);
            mma16816(acc[n4], al, bh0, bh1);
        }
#pragma unroll
        for (int n4 = 0; n4 < 4; ++n4) {
            const int ni = 4 * half + n4;
            *reinterpret_cast<float2 *>(part + part_idx(g, 8 * ni + 2 * q)) =
                make_float2(acc[n4][0], acc[n4][1]);
            *reinterpret_cast<float2 *>(part + part_idx(g + 8, 8 * ni + 2 * q)) =
                make_float2(acc[n4][2], acc[n4][3]);
        }
    }
}

template <int kCL>
__global__ void __launch_bounds__(Layout<kCL>::kThreads, 1)
    mlp_ln_scan_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmV, Args a) {
    using L = Layout<kCL>;
    constexpr int kWarps = L::kWarps;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int rank = kCL > 1 ? (int)cluster_rank() : 0;
    const int seq = blockIdx.x / kCL, h = seq % a.H, T = a.T, NM = T / kMB;
    const size_t row0 = (size_t)seq * T;
    const int gw = rank * kWarps + warp;  // warp index within the cluster

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR);
    // Barrier A (one per mini-batch parity) completes when this CTA's warps
    // have arrived and the other CTAs' sums have landed (as transaction
    // bytes of their bulk copies). Alternating objects keep a copy for
    // mini-batch m + 1 out of the phase of m: a CTA sends for m + 2 only
    // after its own barrier of m + 1 completed, i.e. after every CTA's
    // copies for m + 1, which each sent after its barrier of m completed.
    uint64_t *barA = full + kSlots, *barB = barA + 2, *barL = barA + 3;
    volatile int *abrt = reinterpret_cast<volatile int *>(barA + 4);
    volatile int *issued_s = abrt + 1;  // tiles issued so far (for the abort drain)
    int *status = a.status;
    const uint32_t sGxh = smem_u32(smem + L::GXB), sGxl = sGxh + kTileBytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(&full[s], 1);
        mbar_init(&barA[0], kWarps);  // this CTA's warps (+ the other CTAs' bytes)
        mbar_init(&barA[1], kWarps);
        mbar_init(barB, kWarps);       // this CTA's warps
        mbar_init(barL, kWarps);
        *abrt = 0;
        *issued_s = 0;
        fence_mbar_init();
    }
    if (kCL > 1) cluster_sync(); else __syncthreads();

    // Cluster address of this CTA's shared offset `off` in CTA c.
    auto cl = [&](int off, int c) { return kCL > 1 ? mapa(smem_u32(smem + off), c) : smem_u32(smem + off); };
    auto arrive_local = [&](uint64_t *bar) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    };
    auto wait_a = [&](int i) {
        return mbar_wait_warp(&barA[i & 1], (i >> 1) & 1, abrt, status, 62);
    };
    // TMA producer: mini-batch i into slot i % kSlots, issued by lane 0 of one
    // warp (warps take turns, so no warp carries it every mini-batch). Tiles 0
    // and 1 before the scan; tile m + 2 after barrier B of m, when the slot's
    // previous tile (m - 2) has had its last reader (the LayerNorm forward of
    // m - 2, done before every warp's arrival at B of m).
    int waited = -1;  // last tile this thread waited for
    auto issue = [&](int i) {
        const int s = i % kSlots;
        uint8_t *dst = smem + L::TILES + s * kSlotBytes;
        const int y = (int)(row0 + (size_t)i * kMB);
        mbar_arrive_expect_tx(&full[s], kSlotBytes);
        tma_load_2d(dst, &tmK, 0, y, &full[s]);
        tma_load_2d(dst + kTileBytes, &tmQ, 0, y, &full[s]);
        tma_load_2d(dst + 2 * kTileBytes, &tmV, 0, y, &full[s]);
        *issued_s = i + 1;
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < 2 && i < NM; ++i) issue(i);

    // State: hidden rows j0 = 16*gw + g and j0 + 8 of W1^T and W2, as 8 D
    // tiles over the 64 columns (tile n: columns 8n + 2q, 8n + 2q + 1).
    const int widx = a.w0_per_seq ? seq : h;
    const float *W1g = a.W1_0 + (size_t)widx * kD * kDH;
    const float *W2g = a.W2_0 + (size_t)widx * kDH * kD;
    const int j0 = 16 * gw + g;
    float w1[8][4], w2[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        const int i = 8 * n + 2 * q;
        w1[n][0] = W1g[(size_t)i * kDH + j0];
        w1[n][1] = W1g[(size_t)(i + 1) * kDH + j0];
        w1[n][2] = W1g[(size_t)i * kDH + j0 + 8];
        w1[n][3] = W1g[(size_t)(i + 1) * kDH + j0 + 8];
        const float2 u = *reinterpret_cast<const float2 *>(W2g + (size_t)j0 * kD + i);
        const float2 v = *reinterpret_cast<const float2 *>(W2g + (size_t)(j0 + 8) * kD + i);
        w2[n][0] = u.x;
        w2[n][1] = u.y;
        w2[n][2] = v.x;
        w2[n][3] = v.y;
    }
    // Token work of this warp: tokens warp + kWarps*c (c < kCL) for the
    // partial sums and the LayerNorm backward (every CTA computes Gx for all
    // 16 tokens, identically); token t_own = warp + kWarps*rank for the output.
    const int t_own = gw;
    const float2 gam = make_float2(a.gamma[(size_t)h * kD + 2 * lane], a.gamma[(size_t)h * kD + 2 * lane + 1]);
    const float2 bet = make_float2(a.beta[(size_t)h * kD + 2 * lane], a.beta[(size_t)h * kD + 2 * lane + 1]);

    // Front half of mini-batch i (all warps): H^T = W1^T K^T and
    // Hq0^T = W1^T Q^T (one split of W1), A = GELU(H), GELU'(H), partial
    // X = A W2 over this warp's hidden units.
    float gp[2][4], hq[2][4];
    uint32_t akT_h[4], akT_l[4];
    auto front = [&](int i) -> bool {
        if (!mbar_wait_warp(&full[i % kSlots], (i / kSlots) & 1, abrt, status, 61)) return false;
        waited = i;
        const uint32_t sK = smem_u32(smem + L::TILES + (i % kSlots) * kSlotBytes);
        const uint32_t sQ = sK + kTileBytes;
        float hk[2][4] = {};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) hq[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t ah[4], al[4], kb[4], qb[4];
            state_a(w1, ks, ah, al);
            ldsm_x4(kb, sK + frag_off(ks, lane));
            ldsm_x4(qb, sQ + frag_off(ks, lane));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                mma16816(hk[nt], ah, kb[2 * nt], kb[2 * nt + 1]);
                mma16816(hq[nt], ah, qb[2 * nt], qb[2 * nt + 1]);
                mma16816(hk[nt], al, kb[2 * nt], kb[2 * nt + 1]);
                mma16816(hq[nt], al, qb[2 * nt], qb[2 * nt + 1]);
            }
        }
        float ak[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) ak[nt][e] = gelu_and_prime(hk[nt][e], gp[nt][e]);
        pack_split(ak, akT_h, akT_l);
        uint32_t ah[4], al[4];
        transpose_a(akT_h, ah);
        transpose_a(akT_l, al);
        partial_times_w2(ah, al, w2, reinterpret_cast<float *>(smem + L::XP) + warp * kPart, g, q);
        return true;
    };

    // This CTA's sums over its warps' partials for this warp's tokens t_c:
    // X rows of mini-batch `ix` (ix < 0: none) for every CTA, Zpre and S2 rows
    // of mini-batch `iz` (iz < 0: none) for the CTA owning token t_c. Written
    // to this CTA's slot, copied to the other CTAs' same slot with bulk copies
    // that complete on their barrier A of mini-batch `ia`; then this warp
    // arrives on its own barrier A, expecting its twin warps' copies.
    auto reduce_push = [&](int ix, int iz, int ia) {
#pragma unroll
        for (int c = 0; c < kCL; ++c) {
            const int t = warp + kWarps * c;
            const int off = 4 * part_idx(t, 2 * lane);
            if (ix >= 0) {
                float2 r = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float2 u = *reinterpret_cast<const float2 *>(smem + L::XP + w * kPart * 4 + off);
                    r.x += u.x;
                    r.y += u.y;
                }
                *reinterpret_cast<float2 *>(
                    smem + L::XS + ((((ix & 1) * kCL + rank) * kWarps + warp) * kCL + c) * kD * 4 + 8 * lane) = r;
            }
            if (iz >= 0) {
                float2 r = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float2 u = *reinterpret_cast<const float2 *>(smem + L::ZP + w * kPart * 4 + off);
                    r.x += u.x;
                    r.y += u.y;
                }
                *reinterpret_cast<float2 *>(smem + L::ZS + (((iz & 1) * kCL + rank) * kMB + t) * kD * 4 + 8 * lane) = r;
                if ((lane >> 4) == c) {
                    float sv = 0.f;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w)
                        sv += *reinterpret_cast<const float *>(
                            smem + L::S2P + 4 * (w * kS2Part + t * kS2Pitch + (lane & 15)));
                    *reinterpret_cast<float *>(
                        smem + L::SS + 4 * ((((iz & 1) * kCL + rank) * kMB + t) * kMB + (lane & 15))) = sv;
                }
            }
        }
        uint32_t bytes = 0;  // from each other CTA's twin warp
        MTRACE_AT(17, ia - 1);
        if (kCL > 1) {
            fence_async_smem();
            __syncwarp();
            MTRACE_AT(18, ia - 1);
            if (lane == 0) {
                const int xs = L::XS + (((ix & 1) * kCL + rank) * kWarps + warp) * kCL * kD * 4;
#pragma unroll
                for (int k = 1; k < kCL; ++k) {
                    const int c = (rank + k) % kCL, t = warp + kWarps * c;
                    const uint32_t bar = mapa(smem_u32(&barA[ia & 1]), c);
                    if (ix >= 0) bulk_copy_to_cluster(cl(xs, c), smem_u32(smem + xs), kCL * kD * 4, bar);
                    if (iz >= 0) {
                        const int zs = L::ZS + (((iz & 1) * kCL + rank) * kMB + t) * kD * 4;
                        const int ss = L::SS + (((iz & 1) * kCL + rank) * kMB + t) * kMB * 4;
                        bulk_copy_to_cluster(cl(zs, c), smem_u32(smem + zs), kD * 4, bar);
                        bulk_copy_to_cluster(cl(ss, c), smem_u32(smem + ss), kMB * 4, bar);
                    }
                }
            }
            bytes = (kCL - 1) * ((ix >= 0 ? kCL * kD * 4 : 0) + (iz >= 0 ? (kD + kMB) * 4 : 0));
            MTRACE_AT(19, ia - 1);
        }
        __syncwarp();
        if (lane == 0) {
            if (bytes) mbar_arrive_expect_tx(&barA[ia & 1], bytes);
            else mbar_arrive(&barA[ia & 1]);
        }
    };

    // LayerNorm forward of mini-batch i for token t_own: Zpre = sum of the
    // Aq W2 partials - tril(S2) Gx with S2 = sum of the Aq A^T partials;
    // Z = Q + LN(Zpre).
    auto ln_forward = [&](int i) {
        const float *Gxf = reinterpret_cast<const float *>(smem + L::GXF) + (i & 1) * kPart;
        float z0 = 0.f, z1 = 0.f, sv = 0.f;
#pragma unroll
        for (int c = 0; c < kCL; ++c) {
            const int row = ((i & 1) * kCL + c) * kMB + t_own;
            const float2 u = *reinterpret_cast<const float2 *>(smem + L::ZS + row * kD * 4 + 8 * lane);
            z0 += u.x;
            z1 += u.y;
            sv += *reinterpret_cast<const float *>(smem + L::SS + 4 * (row * kMB + (lane & 15)));
        }
        float cs[kMB];
#pragma unroll
        for (int s = 0; s < kMB; ++s) cs[s] = __shfl_sync(0xffffffffu, sv, s);
        float y0 = 0.f, y1 = 0.f;  // second chain: odd s
#pragma unroll
        for (int s = 0; s < kMB; s += 2) {
            const float c0 = s <= t_own ? cs[s] : 0.f, c1 = s + 1 <= t_own ? cs[s + 1] : 0.f;
            const float2 g0 = *reinterpret_cast<const float2 *>(Gxf + s * kD + 2 * lane);
            const float2 g1 = *reinterpret_cast<const float2 *>(Gxf + (s + 1) * kD + 2 * lane);
            z0 = fmaf(-c0, g0.x, z0);
            z1 = fmaf(-c0, g0.y, z1);
            y0 = fmaf(-c1, g1.x, y0);
            y1 = fmaf(-c1, g1.y, y1);
        }
        z0 += y0;
        z1 += y1;
        float mu, rstd;
        row_stats64(z0, z1, mu, rstd);
        const uint8_t *tile = smem + L::TILES + (i % kSlots) * kSlotBytes;
        const float2 qv =
            bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + kTileBytes + pair_off(t_own, lane)));
        store_z2(a.Z, a.z_bf16, (row0 + (size_t)i * kMB + t_own) * kD + 2 * lane,
                 qv.x + gam.x * (z0 - mu) * rstd + bet.x, qv.y + gam.y * (z1 - mu) * rstd + bet.y);
    };

    int m = 0;
    bool ok = front(0);
    arrive_local(barL);
    ok = ok && mbar_wait_warp(barL, 0, abrt, status, 65);
    if (ok) reduce_push(0, -1, 0);
    // eta of this warp's tokens in mini-batches m and m + 1 (loaded two
    // mini-batches ahead, so its latency never stalls the scan)
    float eta_c[kCL], eta_n[kCL];
#pragma unroll
    for (int c = 0; c < kCL; ++c) {
        eta_c[c] = a.eta[row0 + warp + kWarps * c];
        eta_n[c] = NM > 1 ? a.eta[row0 + kMB + warp + kWarps * c] : 0.f;
    }

    // Scan. Barrier A of m (cluster): the X sums of m and the Zpre / S2 sums
    // of m - 1 are in place in every CTA; barrier B of m (CTA): Gx of m is in
    // place; barrier L (CTA): this CTA's partials are in place.
    for (; ok && m < NM; ++m) {
        const uint32_t par = m & 1;
        float eta_nn[kCL];
#pragma unroll
        for (int c = 0; c < kCL; ++c)
            eta_nn[c] = m + 2 < NM ? a.eta[row0 + (size_t)(m + 2) * kMB + warp + kWarps * c] : 0.f;
        MTRACE(3);
        if (!wait_a(m)) break;
        MTRACE(4);
        const uint8_t *tile = smem + L::TILES + (m % kSlots) * kSlotBytes;
        const uint32_t sK = smem_u32(tile), sQ = sK + kTileBytes;

        // ---- LayerNorm backward of this warp's tokens -> Gx (fp32 and hi/lo),
        // the kCL tokens' reductions interleaved
        {
            float x0[kCL], x1[kCL], mu[kCL], rstd[kCL];
#pragma unroll
            for (int c = 0; c < kCL; ++c) {
                x0[c] = x1[c] = 0.f;
#pragma unroll
                for (int src = 0; src < kCL; ++src) {
                    const float2 u = *reinterpret_cast<const float2 *>(
                        smem + L::XS + (((par * kCL + src) * kWarps + warp) * kCL + c) * kD * 4 + 8 * lane);
                    x0[c] += u.x;
                    x1[c] += u.y;
                }
            }
            row_stats64<kCL>(x0, x1, mu, rstd);
            float xh0[kCL], xh1[kCL], gh0[kCL], gh1[kCL], m1[kCL], m2[kCL];
#pragma unroll
            for (int c = 0; c < kCL; ++c) {
                const uint32_t po = pair_off(warp + kWarps * c, lane);
                const float2 kv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + po));
                const float2 vv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(tile + 2 * kTileBytes + po));
                xh0[c] = (x0[c] - mu[c]) * rstd[c];
                xh1[c] = (x1[c] - mu[c]) * rstd[c];
                gh0[c] = gam.x * (kv.x + gam.x * xh0[c] + bet.x - vv.x);
                gh1[c] = gam.y * (kv.y + gam.y * xh1[c] + bet.y - vv.y);
                m1[c] = gh0[c] + gh1[c];
                m2[c] = gh0[c] * xh0[c] + gh1[c] * xh1[c];
            }
            warp_sum2<kCL>(m1, m2);
#pragma unroll
            for (int c = 0; c < kCL; ++c) {
                const int t = warp + kWarps * c;
                const float sc = eta_c[c] * rstd[c], a1 = m1[c] * (1.f / kD), a2 = m2[c] * (1.f / kD);
                const float G0 = sc * (gh0[c] - a1 - xh0[c] * a2), G1 = sc * (gh1[c] - a1 - xh1[c] * a2);
                *reinterpret_cast<float2 *>(smem + L::GXF + (par * kPart + t * kD + 2 * lane) * 4) =
                    make_float2(G0, G1);
                uint32_t hi, lo;
                split2(G0, G1, hi, lo);
                const uint32_t po = pair_off(t, lane);
                *reinterpret_cast<uint32_t *>(smem + L::GXB + po) = hi;
                *reinterpret_cast<uint32_t *>(smem + L::GXB + kTileBytes + po) = lo;
            }
        }
        arrive_local(barB);
        MTRACE(5);
#pragma unroll
        for (int c = 0; c < kCL; ++c) {
            eta_c[c] = eta_n[c];
            eta_n[c] = eta_nn[c];
        }
        // ---- output of the previous mini-batch (overlaps the wait)
        if (m > 0) ln_forward(m - 1);
        MTRACE(14);
        if (!mbar_wait_warp(barB, par, abrt, status, 63)) break;
        MTRACE(6);
        if (lane == 0 && warp == m % kWarps && m + 2 < NM) issue(m + 2);

        // ---- Gh^T = (W2 Gx^T) * GELU'(H), negated
        float gh[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t ah[4], al[4], bh[4], bl[4];
            state_a(w2, ks, ah, al);
            ldsm_x4(bh, sGxh + frag_off(ks, lane));
            ldsm_x4(bl, sGxl + frag_off(ks, lane));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                mma16816(gh[nt], ah, bh[2 * nt], bh[2 * nt + 1]);
                mma16816(gh[nt], ah, bl[2 * nt], bl[2 * nt + 1]);
                mma16816(gh[nt], al, bh[2 * nt], bh[2 * nt + 1]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) gh[nt][e] = -gh[nt][e] * gp[nt][e];
        uint32_t ngh_h[4], ngh_l[4];  // -Gh^T (rows: hidden units, columns: tokens)
        pack_split(gh, ngh_h, ngh_l);
        MTRACE(7);

        // ---- S1 = tril(Q K^T)  (Hq0^T = W1^T Q^T came with the front half)
        float s1[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t kb[4], qb[4];
            ldsm_x4(kb, sK + frag_off(ks, lane));
            ldsm_x4(qb, sQ + frag_off(ks, lane));
            const uint32_t qa[4] = {qb[0], qb[2], qb[1], qb[3]};
#pragma unroll
            for (int ns = 0; ns < 2; ++ns) mma16816(s1[ns], qa, kb[2 * ns], kb[2 * ns + 1]);
        }
#pragma unroll
        for (int ns = 0; ns < 2; ++ns)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (8 * ns + 2 * q + (e & 1) > g + 8 * (e >> 1)) s1[ns][e] = 0.f;
        MTRACE(8);

        // ---- Hq^T = Hq0^T - Gh^T S1^T;  Aq = GELU(Hq)
        {
            uint32_t sbh[2][2], sbl[2][2];  // B[s][t] = S1[t][s], token tiles 0 and 1
            split2(s1[0][0], s1[0][1], sbh[0][0], sbl[0][0]);
            split2(s1[1][0], s1[1][1], sbh[0][1], sbl[0][1]);
            split2(s1[0][2], s1[0][3], sbh[1][0], sbl[1][0]);
            split2(s1[1][2], s1[1][3], sbh[1][1], sbl[1][1]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float c[4] = {};
                mma16816(c, ngh_h, sbh[nt][0], sbh[nt][1]);
                mma16816(c, ngh_h, sbl[nt][0], sbl[nt][1]);
                mma16816(c, ngh_l, sbh[nt][0], sbh[nt][1]);
#pragma unroll
                for (int e = 0; e < 4; ++e) hq[nt][e] += c[e];
            }
        }
        uint32_t aqA_h[4], aqA_l[4];  // Aq[t][j] as an A fragment
        {
            float aq[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) aq[nt][e] = gelu(hq[nt][e]);
            uint32_t th[4], tl[4];
            pack_split(aq, th, tl);
            transpose_a(th, aqA_h);
            transpose_a(tl, aqA_l);
        }
        MTRACE(9);
        // ---- partial S2 = Aq A^T over this warp's hidden units
        {
            uint32_t bh[4], bl[4];  // A[t][j] as an A fragment; B of A^T by token tiles
            transpose_a(akT_h, bh);
            transpose_a(akT_l, bl);
            float s2[2][4] = {};
#pragma unroll
            for (int ns = 0; ns < 2; ++ns) {
                mma16816(s2[ns], aqA_h, bh[ns], bh[ns + 2]);
                mma16816(s2[ns], aqA_h, bl[ns], bl[ns + 2]);
                mma16816(s2[ns], aqA_l, bh[ns], bh[ns + 2]);
            }
            float *S2p = reinterpret_cast<float *>(smem + L::S2P) + warp * kS2Part;
#pragma unroll
            for (int ns = 0; ns < 2; ++ns) {
                *reinterpret_cast<float2 *>(S2p + g * kS2Pitch + 8 * ns + 2 * q) =
                    make_float2(s2[ns][0], s2[ns][1]);
                *reinterpret_cast<float2 *>(S2p + (g + 8) * kS2Pitch + 8 * ns + 2 * q) =
                    make_float2(s2[ns][2], s2[ns][3]);
            }
        }
        MTRACE(10);
        // ---- partial Zpre = Aq W2 over this warp's hidden units
        partial_times_w2(aqA_h, aqA_l, w2, reinterpret_cast<float *>(smem + L::ZP) + warp * kPart, g, q);
        MTRACE(11);

        // ---- own state rows: W1^T -= Gh^T K,  W2 -= A^T Gx
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t kb[4];
            ldsm_x4_t(kb, sK + frag_off_t(np, lane));
            float u[2][4] = {};
            mma16816(u[0], ngh_h, kb[0], kb[1]);
            mma16816(u[0], ngh_l, kb[0], kb[1]);
            mma16816(u[1], ngh_h, kb[2], kb[3]);
            mma16816(u[1], ngh_l, kb[2], kb[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                w1[2 * np][e] += u[0][e];
                w1[2 * np + 1][e] += u[1][e];
            }
        }
        {
            uint32_t nah[4], nal[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                nah[r] = akT_h[r] ^ 0x80008000u;
                nal[r] = akT_l[r] ^ 0x80008000u;
            }
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bh[4], bl[4];
                ldsm_x4_t(bh, sGxh + frag_off_t(np, lane));
                ldsm_x4_t(bl, sGxl + frag_off_t(np, lane));
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float c[4] = {};
                    mma16816(c, nah, bh[2 * u], bh[2 * u + 1]);
                    mma16816(c, nah, bl[2 * u], bl[2 * u + 1]);
                    mma16816(c, nal, bh[2 * u], bh[2 * u + 1]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) w2[2 * np + u][e] += c[e];
                }
            }
        }
        MTRACE(12);
        // ---- front half of the next mini-batch; sums of this CTA's partials
        const bool more = m + 1 < NM;
        if (more && !front(m + 1)) break;
        MTRACE(0);
        arrive_local(barL);
        if (!mbar_wait_warp(barL, (m + 1) & 1, abrt, status, 65)) break;
        MTRACE(15);
        reduce_push(more ? m + 1 : -1, m, m + 1);
        MTRACE(16);
    }

    bool done = m == NM;
    if (done) {
        // Output of the last mini-batch once its sums are in place.
        if (wait_a(NM)) ln_forward(NM - 1);
        else done = false;
    }
    if (!done) {
        // Aborted: let this CTA's in-flight tile loads land before exiting
        // (every warp takes part in issuing, so every warp's lane 0 checks).
        __syncwarp();
        if (lane == 0) {
            const int n = *issued_s;
            for (int i = waited + 1; i < n; ++i) mbar_drain(&full[i % kSlots], (i / kSlots) & 1);
        }
    }
    __syncwarp();
    if (done && a.W1_out) {
        float *o = a.W1_out + (size_t)seq * kD * kDH;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int i = 8 * n + 2 * q;
            o[(size_t)i * kDH + j0] = w1[n][0];
            o[(size_t)(i + 1) * kDH + j0] = w1[n][1];
            o[(size_t)i * kDH + j0 + 8] = w1[n][2];
            o[(size_t)(i + 1) * kDH + j0 + 8] = w1[n][3];
        }
    }
    if (done && a.W2_out) {
        float *o = a.W2_out + (size_t)seq * kDH * kD;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int i = 8 * n + 2 * q;
            *reinterpret_cast<float2 *>(o + (size_t)j0 * kD + i) = make_float2(w2[n][0], w2[n][1]);
            *reinterpret_cast<float2 *>(o + (size_t)(j0 + 8) * kD + i) =
                make_float2(w2[n][2], w2[n][3]);
        }
    }
    // No CTA leaves while another may still copy into its shared memory: a
    // CTA's copies are waited for by their receiver before it gets here, and
    // on an aborted scan every sender waited out its own bounded wait after
    // its last copy. Every wait above is bounded, so every thread of the
    // cluster gets here.
    if (kCL > 1) cluster_sync();
}

}  // namespace

bool mlp_tc_supported(int d, int dh, int b, bool bf16, long long rows) {
    return bf16 && d == kD && dh == kDH && b == kMB && rows < (1LL << 31);
}

// Cluster size: 2 CTAs of 8 warps per sequence (255 registers a thread for
// the 64-register state plus the working set, two SMs per sequence).
constexpr int kCluster = 2;

cudaError_t launch_mlp_tc(const MlpArgs &a, cudaStream_t s) {
    using L = Layout<kCluster>;
    const uint64_t rows = (uint64_t)a.B * a.H * a.T;
    alignas(64) CUtensorMap tmK, tmQ, tmV;
    if (!encode_tmap_bf16_2d(&tmK, a.K, kD, rows, kD, kMB) ||
        !encode_tmap_bf16_2d(&tmQ, a.Q, kD, rows, kD, kMB) ||
        !encode_tmap_bf16_2d(&tmV, a.V, kD, rows, kD, kMB))
        return cudaErrorInvalidValue;
    auto kernel = mlp_ln_scan_kernel<kCluster>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kSmemBytes);
    if (e != cudaSuccess) return e;
    Args args{a.eta, a.W1_0, a.W2_0, a.gamma, a.beta, a.Z, a.W1_out, a.W2_out, a.H, a.T,
              a.w0_per_seq, a.z_bf16, device_status_word()};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.H * kCluster));
    cfg.blockDim = dim3(L::kThreads);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, tmK, tmQ, tmV, args);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

}  // namespace ttt

#ifdef TTT_TRACE
extern "C" __attribute__((visibility("default"))) int ttt_mlp_trace_fetch(unsigned *host, int n) {
    const int cap = 2 * kMlpTraceEvents * kMlpTraceSteps;
    return cudaMemcpyFromSymbol(host, g_ttt_mlp_trace, sizeof(unsigned) * (n < cap ? n : cap)) ==
                   cudaSuccess
               ? 0
               : -1;
}
#endif
