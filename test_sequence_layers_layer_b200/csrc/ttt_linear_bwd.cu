// ttt_linear_bwd.cu -- backward pass (outer gradients) of the TTT-Linear layer
// on CUDA cores in fp32: one block per (batch, head) sequence.
//
// Forward being differentiated ("Test-Time Training: Linear Complexity Beyond
// Attention", Key Architectural Mechanics of TTT-Linear, parts 1-4), row form
// x = k W, mini-batch m with starting weight W_m, tokens s, t of the batch:
//   x_s = k_s W_m;  with LN: xh_s = LN(x_s), gh_s = gamma (k_s + gamma xh_s + beta - v_s),
//        psi_s = (1/sigma_s)(gh_s - mean(gh_s) - xh_s mean(gh_s xh_s))   (= dl/dx_s);
//        without LN: psi_s = x_s - v_s
//   G_s = eta_s psi_s
//   zpre_t = q_t W_m - sum_{s<=t} (q_t . k_s) G_s
//   z_t = q_t + gamma LN(zpre_t) + beta (with LN), else z_t = zpre_t
//   W_{m+1} = W_m - sum_s k_s^T G_s
// Given dZ and dW_out, the mini-batches are walked in reverse carrying
// Om = dL/dW_{m+1}; each step below is the chain rule of one line above:
//   output LN:  dzpre = (1/sig_z)(dy - mean(dy) - y mean(dy y)), dy = gamma dz
//   read-out:   dq_t += dzpre_t W^T - sum_{s<=t} (dzpre_t . G_s) k_s
//               dk_s -= sum_{t>=s} (dzpre_t . G_s) q_t,  dG_s -= sum_{t>=s} (q_t . k_s) dzpre_t
//   update:     dk_s -= G_s Om^T,  dG_s -= k_s Om
//   step size:  deta_s = dG_s . psi_s,  dpsi_s = eta_s dG_s
//   inner LN:   dgh = (1/sig) P(dpsi) with P(u) = u - mean(u) - xh mean(u xh);
//               dxh = (1/sig)(-mean(gh xh) dpsi - gh mean(dpsi xh)) + gamma^2 dgh;
//               dsig = -(dpsi . psi)/sig;  dx = (1/sig) P(dxh) + dsig xh / d;
//               dk += gamma dgh, dv = -gamma dgh
//   key map:    dk_s += dx_s W^T
//   weight:     dW_m = Om + sum_t q_t^T dzpre_t + sum_s k_s^T dx_s
// The W_m are checkpointed by a forward pass over the sequence first (a
// workspace of one d x d fp32 matrix per mini-batch).
#include "../../include/ttt.h"
#include "ttt_common.cuh"

namespace ttt {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kWarps = kBwdThreads / 32;

struct BwdArgs {
    const void *Q, *K, *V;
    const float *eta, *W0, *gamma, *beta, *dZ, *dW_out;
    float *dQ, *dK, *dV, *deta;
    float *Wck;        // [seq][M][d][d]: W_m of every mini-batch
    float *dW0s;       // [seq][d][d]
    float *dgs, *dbs;  // [seq][d]
    int H, T, d, b;
    bool ln, w0_per_seq;
};

template <typename T>
__device__ __forceinline__ float ldx(const T *p, size_t i);
template <>
__device__ __forceinline__ float ldx<float>(const float *p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Shared-memory views of one block. Matrices with row stride d + 1 (W, Om)
// keep column walks free of bank conflicts.
struct Smem {
    float *W, *Om;                                  // d x (d+1)
    float *K, *Q, *V, *Xh, *Gh, *Psi, *G, *Y, *DZ;  // b x d
    float *DZP, *DQ, *DK, *DG, *DX, *DGh;           // b x d
    float *A, *Bm;                                  // b x b
    float *sig, *sigz, *eta;                        // b
    float *dgam, *dbet, *gam, *bet;                 // d
};

__device__ __forceinline__ Smem carve(float *p, int d, int b) {
    Smem s;
    const int dp = d * (d + 1), bd = b * d;
    s.W = p; p += dp;
    s.Om = p; p += dp;
    s.K = p; p += bd;
    s.Q = p; p += bd;
    s.V = p; p += bd;
    s.Xh = p; p += bd;
    s.Gh = p; p += bd;
    s.Psi = p; p += bd;
    s.G = p; p += bd;
    s.Y = p; p += bd;
    s.DZ = p; p += bd;
    s.DZP = p; p += bd;
    s.DQ = p; p += bd;
    s.DK = p; p += bd;
    s.DG = p; p += bd;
    s.DX = p; p += bd;
    s.DGh = p; p += bd;
    s.A = p; p += b * b;
    s.Bm = p; p += b * b;
    s.sig = p; p += b;
    s.sigz = p; p += b;
    s.eta = p; p += b;
    s.dgam = p; p += d;
    s.dbet = p; p += d;
    s.gam = p; p += d;
    s.bet = p; p += d;
    return s;
}

size_t bwd_smem_floats(int d, int b) {
    return 2 * (size_t)d * (d + 1) + 15 * (size_t)b * d + 2 * (size_t)b * b + 3 * (size_t)b + 4 * (size_t)d;
}

// Inner LayerNorm forward and its loss gradient for token s (one warp; lane
// handles columns lane and lane + 32). Leaves xh in Xh, gh in Gh, psi in Psi,
// G = eta psi in G and sigma in sig. Without LN, psi = x - v.
__device__ __forceinline__ void inner_token(const Smem &S, int s, int d, bool ln, int lane) {
    float x[2], k[2], v[2];
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        x[r] = j < d ? S.Xh[s * d + j] : 0.f;
        k[r] = j < d ? S.K[s * d + j] : 0.f;
        v[r] = j < d ? S.V[s * d + j] : 0.f;
        sum += x[r];
    }
    const float eta = S.eta[s];
    if (!ln) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int j = lane + 32 * r;
            if (j < d) {
                const float psi = x[r] - v[r];
                S.Psi[s * d + j] = psi;
                S.G[s * d + j] = eta * psi;
            }
        }
        return;
    }
    const float inv_d = 1.f / d;
    const float mu = warp_sum(sum) * inv_d;
    float sq = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        const float dv = j < d ? x[r] - mu : 0.f;
        sq += dv * dv;
    }
    const float sig = sqrtf(warp_sum(sq) * inv_d + kLnEps);
    float xh[2], gh[2], sg = 0.f, sgx = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        xh[r] = j < d ? (x[r] - mu) / sig : 0.f;
        const float g = j < d ? S.gam[j] : 0.f, be = j < d ? S.bet[j] : 0.f;
        gh[r] = j < d ? g * (k[r] + g * xh[r] + be - v[r]) : 0.f;
        sg += gh[r];
        sgx += gh[r] * xh[r];
    }
    const float mg = warp_sum(sg) * inv_d, c = warp_sum(sgx) * inv_d;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        if (j < d) {
            const float psi = (gh[r] - mg - xh[r] * c) / sig;
            S.Xh[s * d + j] = xh[r];
            S.Gh[s * d + j] = gh[r];
            S.Psi[s * d + j] = psi;
            S.G[s * d + j] = eta * psi;
        }
    }
    if (lane == 0) S.sig[s] = sig;
}

// Register-blocked products of the block (D = d, compile time). In a b x D
// product, thread (row group rg = tid / D, column c = tid % D) owns rows
// rg + RG k (k < 4) of column c and reads the row operand as float4
// broadcasts; in a D x D weight update it owns rows a0 .. a0 + WR - 1 of
// column c. Matrices W and Om have row stride D + 1.
template <int D>
struct Blk {
    static constexpr int RG = kBwdThreads / D;  // row groups: 16, 8, 4
    static constexpr int WR = D / RG;           // weight rows per thread: 1, 4, 16
    static constexpr int P = D + 1;
    int c, rg, b;

    __device__ __forceinline__ int row(int k) const { return rg + RG * k; }

    // acc[k] = sum_i A[r_k][i] B[i][c]          (B row stride D + 1)
    __device__ __forceinline__ void ab(const float *A, const float *B, float (&acc)[4]) const {
        for (int i = 0; i < D; i += 4) {
            const float b0 = B[i * P + c], b1 = B[(i + 1) * P + c], b2 = B[(i + 2) * P + c],
                        b3 = B[(i + 3) * P + c];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (row(k) < b) {
                    const float4 x = *reinterpret_cast<const float4 *>(A + row(k) * D + i);
                    acc[k] = fmaf(x.x, b0, fmaf(x.y, b1, fmaf(x.z, b2, fmaf(x.w, b3, acc[k]))));
                }
        }
    }
    // acc[k] = sum_j A[r_k][j] B[c][j]          (B row stride D + 1)
    __device__ __forceinline__ void abt(const float *A, const float *B, float (&acc)[4]) const {
        for (int j = 0; j < D; j += 4) {
            const float b0 = B[c * P + j], b1 = B[c * P + j + 1], b2 = B[c * P + j + 2],
                        b3 = B[c * P + j + 3];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (row(k) < b) {
                    const float4 x = *reinterpret_cast<const float4 *>(A + row(k) * D + j);
                    acc[k] = fmaf(x.x, b0, fmaf(x.y, b1, fmaf(x.z, b2, fmaf(x.w, b3, acc[k]))));
                }
        }
    }
    // M[a][c] += sum_s X[s][a] Y[s][c] (+ X2[s][a] Y2[s][c]) for a in a0 .. a0 + WR - 1
    __device__ __forceinline__ void outer(float *M, const float *X, const float *Y, const float *X2,
                                          const float *Y2) const {
        const int a0 = rg * WR;
        float acc[WR];
#pragma unroll
        for (int k = 0; k < WR; ++k) acc[k] = M[(a0 + k) * P + c];
        for (int s = 0; s < b; ++s) {
            const float y = Y[s * D + c], y2 = X2 ? Y2[s * D + c] : 0.f;
            if constexpr (WR >= 4) {
#pragma unroll
                for (int k = 0; k < WR; k += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(X + s * D + a0 + k);
                    acc[k] = fmaf(x.x, y, acc[k]);
                    acc[k + 1] = fmaf(x.y, y, acc[k + 1]);
                    acc[k + 2] = fmaf(x.z, y, acc[k + 2]);
                    acc[k + 3] = fmaf(x.w, y, acc[k + 3]);
                    if (X2) {
                        const float4 z = *reinterpret_cast<const float4 *>(X2 + s * D + a0 + k);
                        acc[k] = fmaf(z.x, y2, acc[k]);
                        acc[k + 1] = fmaf(z.y, y2, acc[k + 1]);
                        acc[k + 2] = fmaf(z.z, y2, acc[k + 2]);
                        acc[k + 3] = fmaf(z.w, y2, acc[k + 3]);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < WR; ++k) {
                    acc[k] = fmaf(X[s * D + a0 + k], y, acc[k]);
                    if (X2) acc[k] = fmaf(X2[s * D + a0 + k], y2, acc[k]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < WR; ++k) M[(a0 + k) * P + c] = acc[k];
    }
};

template <typename TIn, int D>
__global__ void __launch_bounds__(kBwdThreads) linear_bwd_kernel(BwdArgs a) {
    extern __shared__ float smem_f[];
    constexpr int dp1 = D + 1, d = D;
    const int b = a.b, bd = b * d;
    const Smem S = carve(smem_f, d, b);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seq = blockIdx.x, head = seq % a.H, M = a.T / b;
    const Blk<D> bk{tid % D, tid / D, b};
    const int c = bk.c;
    const size_t tok0 = (size_t)seq * a.T;
    const TIn *Qg = static_cast<const TIn *>(a.Q), *Kg = static_cast<const TIn *>(a.K),
              *Vg = static_cast<const TIn *>(a.V);
    const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : head) * d * d;
    float *Wck = a.Wck + (size_t)seq * M * d * d;

    for (int j = tid; j < d; j += kBwdThreads) {
        S.gam[j] = a.ln ? a.gamma[head * d + j] : 1.f;
        S.bet[j] = a.ln ? a.beta[head * d + j] : 0.f;
        S.dgam[j] = 0.f;
        S.dbet[j] = 0.f;
    }
    for (int e = tid; e < d * d; e += kBwdThreads) S.W[(e / d) * dp1 + e % d] = W0[e];
    __syncthreads();

    // ---- forward over the sequence: checkpoint W_m, then apply the update
    for (int m = 0; m < M; ++m) {
        const size_t r0 = tok0 + (size_t)m * b;
        for (int e = tid; e < d * d; e += kBwdThreads) Wck[(size_t)m * d * d + e] = S.W[(e / d) * dp1 + e % d];
        for (int e = tid; e < bd; e += kBwdThreads) {
            S.K[e] = ldx(Kg, r0 * d + e);
            S.V[e] = ldx(Vg, r0 * d + e);
        }
        for (int s = tid; s < b; s += kBwdThreads) S.eta[s] = a.eta[r0 + s];
        __syncthreads();
        {  // x = K W
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            bk.ab(S.K, S.W, acc);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (bk.row(k) < b) S.Xh[bk.row(k) * d + c] = acc[k];
        }
        __syncthreads();
        for (int s = warp; s < b; s += kWarps) inner_token(S, s, d, a.ln, lane);
        __syncthreads();
        // W -= K^T G  (as W += K^T (-G): negate G in place first)
        for (int e = tid; e < bd; e += kBwdThreads) S.G[e] = -S.G[e];
        __syncthreads();
        bk.outer(S.W, S.K, S.G, nullptr, nullptr);
        __syncthreads();
    }

    // ---- reverse walk: Om = dL/dW_{m+1}, starting from dW_out
    for (int e = tid; e < d * d; e += kBwdThreads)
        S.Om[(e / d) * dp1 + e % d] = a.dW_out ? a.dW_out[(size_t)seq * d * d + e] : 0.f;
    for (int m = M - 1; m >= 0; --m) {
        const size_t r0 = tok0 + (size_t)m * b;
        for (int e = tid; e < d * d; e += kBwdThreads) S.W[(e / d) * dp1 + e % d] = Wck[(size_t)m * d * d + e];
        for (int e = tid; e < bd; e += kBwdThreads) {
            S.K[e] = ldx(Kg, r0 * d + e);
            S.Q[e] = ldx(Qg, r0 * d + e);
            S.V[e] = ldx(Vg, r0 * d + e);
            S.DZ[e] = a.dZ[r0 * d + e];
        }
        for (int s = tid; s < b; s += kBwdThreads) S.eta[s] = a.eta[r0 + s];
        __syncthreads();
        {  // x = K W and q W
            float x[4] = {0.f, 0.f, 0.f, 0.f}, y[4] = {0.f, 0.f, 0.f, 0.f};
            bk.ab(S.K, S.W, x);
            bk.ab(S.Q, S.W, y);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (bk.row(k) < b) {
                    S.Xh[bk.row(k) * d + c] = x[k];
                    S.Y[bk.row(k) * d + c] = y[k];
                }
        }
        // A_ts = q_t . k_s (s <= t)
        for (int e = tid; e < b * b; e += kBwdThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int i = 0; i < d; i += 4) {
                    const float4 u = *reinterpret_cast<const float4 *>(S.Q + t * d + i);
                    const float4 v = *reinterpret_cast<const float4 *>(S.K + s * d + i);
                    acc = fmaf(u.x, v.x, fmaf(u.y, v.y, fmaf(u.z, v.z, fmaf(u.w, v.w, acc))));
                }
            S.A[e] = acc;
        }
        __syncthreads();
        for (int s = warp; s < b; s += kWarps) inner_token(S, s, d, a.ln, lane);
        __syncthreads();
        // zpre_t = q_t W - sum_{s<=t} A_ts G_s
        for (int e = tid; e < bd; e += kBwdThreads) {
            const int t = e / d, j = e % d;
            float acc = S.Y[e];
            for (int s = 0; s <= t; ++s) acc = fmaf(-S.A[t * b + s], S.G[s * d + j], acc);
            S.Y[e] = acc;
        }
        __syncthreads();
        // output LayerNorm backward -> dzpre; residual -> dq
        for (int t = warp; t < b; t += kWarps) {
            if (!a.ln) {
                for (int j = lane; j < d; j += 32) {
                    S.DZP[t * d + j] = S.DZ[t * d + j];
                    S.DQ[t * d + j] = 0.f;
                }
                continue;
            }
            float zp[2], dy[2], sum = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                zp[r] = j < d ? S.Y[t * d + j] : 0.f;
                sum += zp[r];
            }
            const float mu = warp_sum(sum) / d;
            float sq = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                const float dv = j < d ? zp[r] - mu : 0.f;
                sq += dv * dv;
            }
            const float sz = sqrtf(warp_sum(sq) / d + kLnEps);
            float y[2], sdy = 0.f, sdyy = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                y[r] = j < d ? (zp[r] - mu) / sz : 0.f;
                dy[r] = j < d ? S.gam[j] * S.DZ[t * d + j] : 0.f;
                sdy += dy[r];
                sdyy += dy[r] * y[r];
            }
            const float mdy = warp_sum(sdy) / d, mdyy = warp_sum(sdyy) / d;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                if (j < d) {
                    S.Y[t * d + j] = y[r];
                    S.DZP[t * d + j] = (dy[r] - mdy - y[r] * mdyy) / sz;
                    S.DQ[t * d + j] = S.DZ[t * d + j];
                }
            }
            if (lane == 0) S.sigz[t] = sz;
        }
        __syncthreads();
        // Bm_ts = dzpre_t . G_s (s <= t); output-LN parameter gradients
        for (int e = tid; e < b * b; e += kBwdThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int j = 0; j < d; j += 4) {
                    const float4 u = *reinterpret_cast<const float4 *>(S.DZP + t * d + j);
                    const float4 v = *reinterpret_cast<const float4 *>(S.G + s * d + j);
                    acc = fmaf(u.x, v.x, fmaf(u.y, v.y, fmaf(u.z, v.z, fmaf(u.w, v.w, acc))));
                }
            S.Bm[e] = acc;
        }
        if (a.ln)
            for (int j = tid; j < d; j += kBwdThreads) {
                float gb = 0.f, gg = 0.f;
                for (int t = 0; t < b; ++t) {
                    gb += S.DZ[t * d + j];
                    gg = fmaf(S.DZ[t * d + j], S.Y[t * d + j], gg);
                }
                S.dbet[j] += gb;
                S.dgam[j] += gg;
            }
        __syncthreads();
        {  // read-out and update terms: dq += dzpre W^T; dk = -G Om^T; dG = -k Om; causal sums
            float dq[4], dk[4] = {0.f, 0.f, 0.f, 0.f}, dg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 4; ++k) dq[k] = bk.row(k) < b ? S.DQ[bk.row(k) * d + c] : 0.f;
            bk.abt(S.DZP, S.W, dq);
            bk.abt(S.G, S.Om, dk);
            bk.ab(S.K, S.Om, dg);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = bk.row(k);
                if (r >= b) continue;
                float q = dq[k], kk = -dk[k], g = -dg[k];
                for (int s = 0; s <= r; ++s) q = fmaf(-S.Bm[r * b + s], S.K[s * d + c], q);
                for (int t = r; t < b; ++t) {
                    kk = fmaf(-S.Bm[t * b + r], S.Q[t * d + c], kk);
                    g = fmaf(-S.A[t * b + r], S.DZP[t * d + c], g);
                }
                S.DQ[r * d + c] = q;
                S.DK[r * d + c] = kk;
                S.DG[r * d + c] = g;
            }
        }
        __syncthreads();
        // step size and the inner loss gradient's own backward (per token)
        for (int s = warp; s < b; s += kWarps) {
            const float eta = S.eta[s];
            float dpsi[2], psi[2], sdp = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                const float dgv = j < d ? S.DG[s * d + j] : 0.f;
                psi[r] = j < d ? S.Psi[s * d + j] : 0.f;
                sdp += dgv * psi[r];
                dpsi[r] = eta * dgv;
            }
            const float de = warp_sum(sdp);
            if (lane == 0) a.deta[tok0 + (size_t)m * b + s] = de;
            if (!a.ln) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int j = lane + 32 * r;
                    if (j < d) {
                        S.DX[s * d + j] = dpsi[r];
                        a.dV[((size_t)m * b + s + tok0) * d + j] = -dpsi[r];
                    }
                }
                continue;
            }
            const float sig = S.sig[s];
            float xh[2], gh[2], s1 = 0.f, s2 = 0.f, s3 = 0.f, s4 = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                xh[r] = j < d ? S.Xh[s * d + j] : 0.f;
                gh[r] = j < d ? S.Gh[s * d + j] : 0.f;
                s1 += dpsi[r];
                s2 += dpsi[r] * xh[r];
                s3 += gh[r] * xh[r];
                s4 += dpsi[r] * psi[r];
            }
            const float inv_d = 1.f / d;
            const float mdp = warp_sum(s1) * inv_d, e_ = warp_sum(s2) * inv_d,
                        cc = warp_sum(s3) * inv_d, dsig = -warp_sum(s4) / sig;
            float dgh[2], dxh[2], t1 = 0.f, t2 = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                const float g = j < d ? S.gam[j] : 0.f;
                dgh[r] = j < d ? (dpsi[r] - mdp - xh[r] * e_) / sig : 0.f;
                dxh[r] = j < d ? (-cc * dpsi[r] - gh[r] * e_) / sig + g * g * dgh[r] : 0.f;
                t1 += dxh[r];
                t2 += dxh[r] * xh[r];
            }
            const float mdx = warp_sum(t1) * inv_d, mdxx = warp_sum(t2) * inv_d;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                if (j < d) {
                    const float g = S.gam[j];
                    S.DX[s * d + j] = (dxh[r] - mdx - xh[r] * mdxx) / sig + dsig * xh[r] * inv_d;
                    S.DGh[s * d + j] = dgh[r];
                    S.DK[s * d + j] += g * dgh[r];
                    a.dV[((size_t)m * b + s + tok0) * d + j] = -g * dgh[r];
                }
            }
        }
        __syncthreads();
        {  // key map: dk_s += dx_s W^T; store dq, dk
            float dk[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) dk[k] = bk.row(k) < b ? S.DK[bk.row(k) * d + c] : 0.f;
            bk.abt(S.DX, S.W, dk);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = bk.row(k);
                if (r < b) {
                    a.dK[(r0 + r) * d + c] = dk[k];
                    a.dQ[(r0 + r) * d + c] = S.DQ[r * d + c];
                }
            }
        }
        if (a.ln)  // inner-LN parameter gradients
            for (int j = tid; j < d; j += kBwdThreads) {
                const float g = S.gam[j], be = S.bet[j];
                float gb = 0.f, gg = 0.f;
                for (int s = 0; s < b; ++s) {
                    const float dgh = S.DGh[s * d + j];
                    gb += g * dgh;
                    gg += dgh * (S.K[s * d + j] + be - S.V[s * d + j]) + 2.f * g * S.Xh[s * d + j] * dgh;
                }
                S.dbet[j] += gb;
                S.dgam[j] += gg;
            }
        __syncthreads();
        // dW_m = Om + sum_t q_t^T dzpre_t + sum_s k_s^T dx_s
        bk.outer(S.Om, S.Q, S.DZP, S.K, S.DX);
        __syncthreads();
    }
    for (int e = tid; e < d * d; e += kBwdThreads) a.dW0s[(size_t)seq * d * d + e] = S.Om[(e / d) * dp1 + e % d];
    if (a.ln)
        for (int j = tid; j < d; j += kBwdThreads) {
            a.dgs[(size_t)seq * d + j] = S.dgam[j];
            a.dbs[(size_t)seq * d + j] = S.dbet[j];
        }
}

// Sums per-sequence gradients of per-head parameters over the batch, in a
// fixed order: out[h][e] = sum_b in[b * H + h][e] for e < n; a thread per
// element (grid: elements x H).
__global__ void sum_over_batch_kernel(const float *in, float *out, int B, int H, int n) {
    const int h = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    float acc = 0.f;
    for (int bb = 0; bb < B; ++bb) acc += in[((size_t)bb * H + h) * n + e];
    out[(size_t)h * n + e] = acc;
}

}  // namespace

bool linear_bwd_supported(int d, int b) {
    return (d == 16 || d == 32 || d == 64) && b >= 1 && b * d <= 1024;
}

size_t linear_bwd_workspace_bytes(int B, int H, int T, int d, int b) {
    if (B <= 0 || H <= 0 || T <= 0 || b <= 0 || T % b || !linear_bwd_supported(d, b)) return 0;
    const size_t S = (size_t)B * H;
    return 4 * (S * (size_t)(T / b) * d * d + S * d * d + 2 * S * d);
}

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
cudaError_t launch_linear_bwd(const LinearBwdArgs &a, cudaStream_t s) {
    const size_t S = (size_t)a.B * a.H, M = (size_t)(a.T / a.b), dd = (size_t)a.d * a.d;
    float *ws = static_cast<float *>(a.workspace);
    BwdArgs k{a.Q, a.K, a.V, a.eta, a.W0, a.gamma, a.beta, a.dZ, a.dW_out,
              a.dQ, a.dK, a.dV, a.deta,
              ws, a.w0_per_seq ? a.dW0 : ws + S * M * dd,
              ws + S * M * dd + S * dd, ws + S * M * dd + S * dd + S * a.d,
              a.H, a.T, a.d, a.b, a.ln, a.w0_per_seq};
    const size_t smem = bwd_smem_floats(a.d, a.b) * sizeof(float);
    cudaError_t e;
    auto go = [&](auto kernel) -> cudaError_t {
        cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (r != cudaSuccess) return r;
        kernel<<<(unsigned)S, kBwdThreads, smem, s>>>(k);
        return cudaSuccess;
    };
    if (a.bf16)
        e = a.d == 16 ? go(linear_bwd_kernel<__nv_bfloat16, 16>)
          : a.d == 32 ? go(linear_bwd_kernel<__nv_bfloat16, 32>) : go(linear_bwd_kernel<__nv_bfloat16, 64>);
    else
        e = a.d == 16 ? go(linear_bwd_kernel<float, 16>)
          : a.d == 32 ? go(linear_bwd_kernel<float, 32>) : go(linear_bwd_kernel<float, 64>);
    if (e != cudaSuccess) return e;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch(s);
    if (!a.w0_per_seq) {
        sum_over_batch_kernel<<<dim3(((int)dd + 255) / 256, a.H), 256, 0, s>>>(k.dW0s, a.dW0, a.B, a.H, (int)dd);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
    }
    if (a.ln) {
        sum_over_batch_kernel<<<dim3((a.d + 63) / 64, a.H), 64, 0, s>>>(k.dgs, a.dgamma, a.B, a.H, a.d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
        sum_over_batch_kernel<<<dim3((a.d + 63) / 64, a.H), 64, 0, s>>>(k.dbs, a.dbeta, a.B, a.H, a.d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
    }
    return cudaSuccess;
}

#endif  // TTT_HOST_RUN

}  // namespace ttt
