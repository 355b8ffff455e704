// ttt_chunk_bwd.cu -- backward pass (outer gradients) of large-chunk TTT on
// CUDA cores in fp32.
//
// Forward ("Test-Time Training Done Right", abstract), per sequence, chunk c
// of C tokens with starting weight W_c, f(k) = k W:
//   Z_c = Q_c W_c,   W_{c+1} = W_c - K_c^T diag(eta) (K_c W_c - V_c)
//       = W_c - A_c W_c + B_c,   A_c = K_c^T diag(eta) K_c,  B_c = K_c^T diag(eta) V_c.
// Given dZ and dW_out, with Om_c = dL/dW_c, R_c = K_c W_c - V_c and
// P_c = K_c Om_{c+1}, the chain rule of those two lines gives
//   Om_c  = Om_{c+1} - A_c Om_{c+1} + D_c,   D_c = Q_c^T dZ_c,   Om_NC = dW_out
//   dQ_c  = dZ_c W_c^T
//   dK_c  = -diag(eta) (R_c Om_{c+1}^T + P_c W_c^T)
//   dV_c  = diag(eta) P_c
//   deta_t = -P_t . R_t
//   dW0   = Om_0.
// Both recurrences are affine with the same A_c, so the work splits like the
// forward's: per-chunk Gram products (A_c, B_c, D_c) in parallel, one scan per
// sequence in each direction (W_c forward, Om_{c+1} backward), and the
// per-token gradients of every chunk in parallel from W_c and Om_{c+1}.
#include <type_traits>

#include "../../include/ttt.h"
#include "ttt_common.cuh"

namespace ttt {

// ttt_chunk_bwd_tc.cu
bool chunk_bwd_gram_tc_supported(int d, int chunk, bool bf16);
cudaError_t launch_chunk_bwd_gram_tc(const void *Q, const void *K, const void *V, const float *eta,
                                     const float *dZ, int B, int H, int T, int chunk, float *gram,
                                     cudaStream_t s);
cudaError_t launch_chunk_bwd_scan_tc(const float *W0, const float *dW_out, const float *gram,
                                     float *Wst, float *Omst, float *dW0_out, int S, int H, int NC,
                                     bool w0_per_seq, cudaStream_t s);
bool chunk_bwd_tok_tc_supported(int d, int chunk, bool bf16);
cudaError_t launch_chunk_bwd_tok_tc(const void *K, const void *V, const float *eta, const float *dZ,
                                    const float *W, const float *Om, float *S, size_t s_stride,
                                    int B, int H, int T, int chunk, float *dQ, float *dK, float *dV,
                                    float *deta, cudaStream_t s);

namespace {

constexpr int kT = 256;  // threads per block in every kernel here (CUDA-core path)

template <typename T>
__device__ __forceinline__ float ldv(const T *p, size_t i);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

// Workspace (fp32), per chunk g = seq * NC + c: [A_c | B_c | D_c] (3 d^2),
// then per chunk W_c (d^2), then per chunk Om_{c+1} (d^2), then per-sequence
// dW0 (d^2) when W0 is shared by the batch.
struct WsView {
    float *gram, *W, *Om, *dW0s;
};

__host__ __device__ inline WsView ws_view(float *ws, size_t nchunks, size_t S, int d) {
    const size_t dd = (size_t)d * d;
    WsView v;
    v.gram = ws;
    v.W = ws + 3 * nchunks * dd;
    v.Om = v.W + nchunks * dd;
    v.dW0s = v.Om + nchunks * dd;
    (void)S;
    return v;
}

// ---------------------------------------------------------------------------
// 1. Gram products of chunk g, one 64 x 64 output tile per block:
//    product 0: A = (eta K)^T K, 1: B = (eta K)^T V, 2: D = Q^T dZ.
template <typename TIn, int D>
__global__ void __launch_bounds__(kT) cb_gram_kernel(const TIn *Q, const TIn *K, const TIn *V,
                                                     const float *eta, const float *dZ, int T,
                                                     int C, float *gram) {
    __shared__ __align__(16) float Xs[32][64];
    __shared__ __align__(16) float Ys[32][64];
    const int g = blockIdx.x, p = blockIdx.y, tile = blockIdx.z;
    constexpr int NT = D / 64;
    const int i0 = 64 * (tile / NT), j0 = 64 * (tile % NT);
    const int NC = T / C, seq = g / NC, c = g % NC;
    const size_t row0 = (size_t)seq * T + (size_t)c * C;  // first token row of the chunk
    const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
    float acc[4][4] = {};
    for (int t0 = 0; t0 < C; t0 += 32) {
        for (int e = tid; e < 32 * 64; e += kT) {
            const int t = e / 64, i = e % 64;
            const size_t row = row0 + t0 + t;
            float x, y;
            if (p == 2) {
                x = ldv(Q, row * D + i0 + i);
                y = dZ[row * D + j0 + i];
            } else {
                x = eta[row] * ldv(K, row * D + i0 + i);
                y = p == 0 ? ldv(K, row * D + j0 + i) : ldv(V, row * D + j0 + i);
            }
            Xs[t][i] = x;
            Ys[t][i] = y;
        }
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < 32; ++t) {
            const float4 xv = *reinterpret_cast<const float4 *>(&Xs[t][4 * ti]);
            const float4 yv = *reinterpret_cast<const float4 *>(&Ys[t][4 * tj]);
            const float xs[4] = {xv.x, xv.y, xv.z, xv.w}, ys[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xs[a], ys[b], acc[a][b]);
        }
        __syncthreads();
    }
    float *out = gram + ((size_t)g * 3 + p) * D * D;
#pragma unroll
    for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4 *>(out + (size_t)(i0 + 4 * ti + a) * D + j0 + 4 * tj) =
            make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
}

// ---------------------------------------------------------------------------
// 2. The two affine scans of one sequence, M <- M - A_c M + E_c:
//    blockIdx.y = 0: M = W_c forward from W0, E = B_c, storing W_c;
//    blockIdx.y = 1: M = Om_{c+1} backward from dW_out, E = D_c, storing
//    Om_{c+1}, and at the end Om_0 = dW0 of the sequence.
// The columns of M evolve independently, so blockIdx.z picks a slice of
// scan_cols(D) columns (more blocks on the 16-step chains: 32 columns at
// d = 128). A thread owns a 4 x 4 block of the slice. A_c is symmetric
// (K^T diag(eta) K), so its row k stands for its column k. A_c sits in
// shared memory for the step's product; the next step's A_c and this step's
// E_c are loaded into registers while the product runs.
__host__ __device__ constexpr int scan_cols(int D) { return 16 * kT / D; }
template <int D>
__global__ void __launch_bounds__(kT) cb_scan_kernel(const float *W0, const float *dW_out,
                                                     int H, int NC, bool w0_per_seq, WsView w,
                                                     float *dW0_out) {
    constexpr int kScanCols = scan_cols(D);
    extern __shared__ __align__(16) float As[];  // A_c (D x D), then the slice of M (D x kScanCols)
    float *Ms = As + D * D;
    constexpr int RB = 4, CG = kScanCols / RB;   // CG column groups of 4
    static_assert(D / RB * CG == kT && D % kScanCols == 0, "a 4 x 4 block per thread");
    const int seq = blockIdx.x, dir = blockIdx.y, c0 = kScanCols * blockIdx.z, tid = threadIdx.x;
    const int i0 = RB * (tid / CG), j0 = RB * (tid % CG);  // within the slice
    const size_t dd = (size_t)D * D;
    const float *src0 = dir == 0 ? W0 + (size_t)(w0_per_seq ? seq : seq % H) * dd
                                 : (dW_out ? dW_out + (size_t)seq * dd : nullptr);
    for (int e = tid; e < D * kScanCols; e += kT) {
        const int i = e / kScanCols, j = e % kScanCols;
        Ms[e] = src0 ? src0[(size_t)i * D + c0 + j] : 0.f;
    }
    __syncthreads();
    // A_c of the first step into shared memory; each later step's A_c is
    // loaded into registers while the previous step's product runs
    constexpr int NPF = D * D / 4 / kT;  // float4 of A_c per thread
    auto chunk_of = [&](int st) { return (size_t)seq * NC + (dir == 0 ? st : NC - 1 - st); };
    {
        const float *Ag = w.gram + (chunk_of(0) * 3 + 0) * dd;
#pragma unroll
        for (int q = 0; q < NPF; ++q)
            *reinterpret_cast<float4 *>(As + 4 * (tid + q * kT)) =
                *reinterpret_cast<const float4 *>(Ag + 4 * (tid + q * kT));
    }
    for (int s = 0; s < NC; ++s) {
        const size_t g = chunk_of(s);
        float *store = (dir == 0 ? w.W : w.Om) + g * dd;
        for (int e = tid; e < D * kScanCols; e += kT) {
            const int i = e / kScanCols, j = e % kScanCols;
            store[(size_t)i * D + c0 + j] = Ms[e];
        }
        const float *E = w.gram + (g * 3 + (dir == 0 ? 1 : 2)) * dd;
        __syncthreads();  // A_c is in shared memory
        float4 pf[NPF];   // the next step's A
        if (s + 1 < NC) {
            const float *An = w.gram + (chunk_of(s + 1) * 3 + 0) * dd;
#pragma unroll
            for (int q = 0; q < NPF; ++q) pf[q] = *reinterpret_cast<const float4 *>(An + 4 * (tid + q * kT));
        }
        float4 ev[RB];  // this thread's 4 x 4 block of E
#pragma unroll
        for (int a = 0; a < RB; ++a)
            ev[a] = *reinterpret_cast<const float4 *>(E + (size_t)(i0 + a) * D + c0 + j0);
        float acc[RB][RB] = {};
        for (int k = 0; k < D; ++k) {
            const float4 u = *reinterpret_cast<const float4 *>(As + k * D + i0);
            const float4 v = *reinterpret_cast<const float4 *>(Ms + k * kScanCols + j0);
            const float av[RB] = {u.x, u.y, u.z, u.w}, mv[RB] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int a = 0; a < RB; ++a)
#pragma unroll
                for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(av[a], mv[b], acc[a][b]);
        }
        __syncthreads();  // every thread has read M and A_c
#pragma unroll
        for (int a = 0; a < RB; ++a) {
            float4 *m = reinterpret_cast<float4 *>(Ms + (i0 + a) * kScanCols + j0);
            const float4 o = *m;
            *m = make_float4(o.x - acc[a][0] + ev[a].x, o.y - acc[a][1] + ev[a].y,
                             o.z - acc[a][2] + ev[a].z, o.w - acc[a][3] + ev[a].w);
        }
        if (s + 1 < NC) {
#pragma unroll
            for (int q = 0; q < NPF; ++q) *reinterpret_cast<float4 *>(As + 4 * (tid + q * kT)) = pf[q];
        }
        __syncthreads();
    }
    if (dir == 1)
        for (int e = tid; e < D * kScanCols; e += kT) {
            const int i = e / kScanCols, j = e % kScanCols;
            dW0_out[(size_t)seq * dd + (size_t)i * D + c0 + j] = Ms[e];
        }
}

// ---------------------------------------------------------------------------
// 3. Per-token gradients of chunk g from W_c and Om_{c+1}, 32 tokens at a
// time. Thread (tr, tc): rows 4 tr .. 4 tr + 3 of the tile, columns
// tc + 32 a (a < D / 32), so that a warp reads 32 consecutive columns of a row
// and 32 different rows (row stride D + 1) of the same column without bank
// conflicts.
template <typename TIn, int D>
__global__ void __launch_bounds__(kT) cb_tok_kernel(const TIn *K, const TIn *V, const float *eta,
                                                    const float *dZ, int T, int C, WsView w,
                                                    float *dQ, float *dK, float *dV,
                                                    float *deta) {
    extern __shared__ __align__(16) float sm[];
    constexpr int P1 = D + 1, NA = D / 32, TT = 32;
    float *Wm = sm, *Om = Wm + D * P1;
    float *Ks = Om + D * P1, *Vs = Ks + TT * D, *Zs = Vs + TT * D, *Rs = Zs + TT * D,
          *Ps = Rs + TT * D;
    const int g = blockIdx.x, NC = T / C, seq = g / NC, c = g % NC;
    const size_t row0 = (size_t)seq * T + (size_t)c * C;
    const size_t dd = (size_t)D * D;
    const int tid = threadIdx.x, tr = tid / 32, tc = tid % 32;
    for (int e = tid; e < D * D; e += kT) {
        Wm[(e / D) * P1 + e % D] = w.W[g * dd + e];
        Om[(e / D) * P1 + e % D] = w.Om[g * dd + e];
    }
    for (int t0 = 0; t0 < C; t0 += TT) {
        __syncthreads();  // the previous tile's R, P and inputs are consumed
        for (int e = tid; e < TT * D; e += kT) {
            const size_t idx = (row0 + t0) * D + e;
            Ks[e] = ldv(K, idx);
            Vs[e] = ldv(V, idx);
            Zs[e] = dZ[idx];
        }
        __syncthreads();
        // R = K W - V and P = K Om
        float r[4][NA] = {}, pp[4][NA] = {};
        for (int k = 0; k < D; ++k) {
            float kv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) kv[a] = Ks[(4 * tr + a) * D + k];
#pragma unroll
            for (int b = 0; b < NA; ++b) {
                const float wv = Wm[k * P1 + tc + 32 * b], ov = Om[k * P1 + tc + 32 * b];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    r[a][b] = fmaf(kv[a], wv, r[a][b]);
                    pp[a][b] = fmaf(kv[a], ov, pp[a][b]);
                }
            }
        }
        float de[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int t = 4 * tr + a;
            const float et = eta[row0 + t0 + t];
#pragma unroll
            for (int b = 0; b < NA; ++b) {
                const int j = tc + 32 * b;
                r[a][b] -= Vs[t * D + j];
                Rs[t * D + j] = r[a][b];
                Ps[t * D + j] = pp[a][b];
                de[a] = fmaf(pp[a][b], r[a][b], de[a]);
                dV[(row0 + t0 + t) * D + j] = et * pp[a][b];
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {  // row sums over the warp's 32 column groups
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) de[a] += __shfl_xor_sync(0xffffffffu, de[a], o);
            if (tc == 0) deta[row0 + t0 + 4 * tr + a] = -de[a];
        }
        __syncthreads();
        // dQ = dZ W^T and dK = -eta (R Om^T + P W^T)
        float q[4][NA] = {}, kk[4][NA] = {};
        for (int j = 0; j < D; ++j) {
            float zv[4], rv[4], pv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                zv[a] = Zs[(4 * tr + a) * D + j];
                rv[a] = Rs[(4 * tr + a) * D + j];
                pv[a] = Ps[(4 * tr + a) * D + j];
            }
#pragma unroll
            for (int b = 0; b < NA; ++b) {
                const int i = tc + 32 * b;
                const float wv = Wm[i * P1 + j], ov = Om[i * P1 + j];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    q[a][b] = fmaf(zv[a], wv, q[a][b]);
                    kk[a][b] = fmaf(rv[a], ov, fmaf(pv[a], wv, kk[a][b]));
                }
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int t = 4 * tr + a;
            const float et = eta[row0 + t0 + t];
#pragma unroll
            for (int b = 0; b < NA; ++b) {
                const size_t o = (row0 + t0 + t) * D + tc + 32 * b;
                dQ[o] = q[a][b];
                dK[o] = -et * kk[a][b];
            }
        }
    }
}

size_t tok_smem_bytes(int D) { return (2 * (size_t)D * (D + 1) + 5 * 32 * (size_t)D) * sizeof(float); }

// out[h][e] = sum_b in[b * H + h][e], fixed order; a thread per element
// (grid: elements x H), so the B loads of all elements are in flight at once.
__global__ void cb_sum_over_batch_kernel(const float *in, float *out, int B, int H, int n) {
    const int h = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    float acc = 0.f;
    for (int bb = 0; bb < B; ++bb) acc += in[((size_t)bb * H + h) * n + e];
    out[(size_t)h * n + e] = acc;
}

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
template <typename TIn, int D>
cudaError_t launch_typed(const void *Q, const void *K, const void *V, const float *eta,
                         const float *W0, const float *dZ, const float *dW_out, float *dQ,
                         float *dK, float *dV, float *deta, float *dW0, int B, int H, int T,
                         int C, bool w0_per_seq, void *workspace, cudaStream_t s) {
    const int NC = T / C;
    const size_t S = (size_t)B * H, nch = S * NC;
    const WsView w = ws_view(static_cast<float *>(workspace), nch, S, D);
    const TIn *q = static_cast<const TIn *>(Q), *k = static_cast<const TIn *>(K),
              *v = static_cast<const TIn *>(V);
    cudaError_t e;
    // d = 128, bf16, chunk % 128 == 0: the per-token products on the tensor cores
    const bool tok_tc = std::is_same<TIn, __nv_bfloat16>::value && chunk_bwd_tok_tc_supported(D, C, true);
    float *dW0_seq = w0_per_seq ? dW0 : w.dW0s;
    if (std::is_same<TIn, __nv_bfloat16>::value && chunk_bwd_gram_tc_supported(D, C, true)) {
        // d = 128, bf16: the Gram products on the tensor cores, then the scans
        // on the tensor cores, which read the Gram's operand layouts
        if ((e = launch_chunk_bwd_gram_tc(Q, K, V, eta, dZ, B, H, T, C, w.gram, s)) != cudaSuccess)
            return e;
        if ((e = launch_chunk_bwd_scan_tc(W0, dW_out, w.gram, w.W, w.Om, dW0_seq, (int)S, H, NC,
                                          w0_per_seq, s)) != cudaSuccess)
            return e;
    } else {
        cb_gram_kernel<TIn, D><<<dim3((unsigned)nch, 3, (D / 64) * (D / 64)), kT, 0, s>>>(
            q, k, v, eta, dZ, T, C, w.gram);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
        const size_t scan_smem = ((size_t)D * D + (size_t)D * scan_cols(D)) * sizeof(float);  // A_c, M slice
        if ((e = cudaFuncSetAttribute(cb_scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)scan_smem)) != cudaSuccess)
            return e;
        cb_scan_kernel<D><<<dim3((unsigned)S, 2, D / scan_cols(D)), kT, scan_smem, s>>>(
            W0, dW_out, H, NC, w0_per_seq, w, dW0_seq);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
    }
    if (tok_tc) {
        // each chunk's S = W_c Om_{c+1}^T + Om_{c+1} W_c^T takes the place of
        // its A_c, which only the scans read
        if ((e = launch_chunk_bwd_tok_tc(K, V, eta, dZ, w.W, w.Om, w.gram, 3 * (size_t)D * D, B, H,
                                         T, C, dQ, dK, dV, deta, s)) != cudaSuccess)
            return e;
    } else {
        const size_t tsm = tok_smem_bytes(D);
        if ((e = cudaFuncSetAttribute(cb_tok_kernel<TIn, D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm)) !=
            cudaSuccess)
            return e;
        cb_tok_kernel<TIn, D><<<(unsigned)nch, kT, tsm, s>>>(k, v, eta, dZ, T, C, w, dQ, dK, dV,
                                                             deta);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
    }
    if (!w0_per_seq) {
        cb_sum_over_batch_kernel<<<dim3((D * D + 255) / 256, H), 256, 0, s>>>(w.dW0s, dW0, B, H, D * D);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch(s);
    }
    return cudaSuccess;
}
#endif  // TTT_HOST_RUN

}  // namespace

bool chunk_bwd_supported(int d, int chunk) {
    return (d == 64 || d == 128) && chunk >= 32 && chunk % 32 == 0;
}

size_t chunk_bwd_workspace_bytes(int B, int H, int T, int d, int chunk) {
    if (B <= 0 || H <= 0 || T <= 0 || chunk <= 0 || T % chunk || !chunk_bwd_supported(d, chunk))
        return 0;
    const size_t S = (size_t)B * H, nch = S * (T / chunk), dd = (size_t)d * d;
    return sizeof(float) * (5 * nch * dd + S * dd);
}

#ifndef TTT_HOST_RUN
cudaError_t launch_chunk_bwd(const void *Q, const void *K, const void *V, const float *eta,
                             const float *W0, const float *dZ, const float *dW_out, float *dQ,
                             float *dK, float *dV, float *deta, float *dW0, int B, int H, int T,
                             int d, int chunk, bool bf16, bool w0_per_seq, void *workspace,
                             cudaStream_t s) {
    if (bf16)
        return d == 64 ? launch_typed<__nv_bfloat16, 64>(Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV,
                                                         deta, dW0, B, H, T, chunk, w0_per_seq,
                                                         workspace, s)
                       : launch_typed<__nv_bfloat16, 128>(Q, K, V, eta, W0, dZ, dW_out, dQ, dK,
                                                          dV, deta, dW0, B, H, T, chunk,
                                                          w0_per_seq, workspace, s);
    return d == 64 ? launch_typed<float, 64>(Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV, deta, dW0,
                                             B, H, T, chunk, w0_per_seq, workspace, s)
                   : launch_typed<float, 128>(Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV, deta,
                                              dW0, B, H, T, chunk, w0_per_seq, workspace, s);
}

#endif  // TTT_HOST_RUN

}  // namespace ttt
