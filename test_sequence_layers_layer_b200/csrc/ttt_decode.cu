// ttt_decode.cu -- one TTT-Linear token per sequence (online decode, b = 1),
// d = 64, the fast weight updated in place.
//
// Method ("Test-Time Training: Linear Complexity Beyond Attention", Key
// Architectural Mechanics of TTT-Linear, parts 1-3, and the listing's step()):
// for the token (q, k, v) with step size eta and the sequence's weight W,
//   x = k W,  G = eta * dl/dx  (LayerNorm backward of f - v, or x - v),
//   W <- W - k^T G,  z = f-epilogue(q W)     (read out after the update).
// One block of 128 threads per sequence. Thread (column j, half h) keeps rows
// 32 h .. 32 h + 31 of column j of W in registers for the whole call, over
// all n tokens of the call: the k- and q-products are 32 FMAs per thread plus
// one shuffle with the partner thread of the other half; every row statistic
// (LayerNorm mean, variance, and the two means of its backward) is one block
// reduction through shared memory. Seven barriers per token (the next
// token's q, k, v are loaded while the current one is processed); W is read
// once and written once per call.
#include "../../include/ttt.h"
#include "ttt_common.cuh"

namespace ttt {
namespace {

constexpr int kDD = 64, kDecThreads = 128, kDecWarps = kDecThreads / 32;

struct DecodeArgs {
    const void *q, *k, *v;
    const float *eta, *gamma, *beta;
    float *W;  // [S][64][64], updated in place
    float *z;  // [S][n][64]; bf16 when z_bf16
    int H;
    bool bf16, ln, z_bf16, l2_keys;
    int n = 1;  // tokens per sequence in this call (q, k, v [S][n][64], eta [S][n])
};

__device__ __forceinline__ float dec_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over the block of a value held by the h == 0 thread of each column
// (the h == 1 partner holds the same value and contributes 0). `slot` is a
// 4-float area of shared memory used by this reduction only.
__device__ __forceinline__ float col_sum(float v, int h, float *slot) {
    const float w = dec_warp_sum(h == 0 ? v : 0.f);
    if ((threadIdx.x & 31) == 0) slot[threadIdx.x >> 5] = w;
    __syncthreads();
    return (slot[0] + slot[1]) + (slot[2] + slot[3]);
}

__global__ void __launch_bounds__(kDecThreads) linear_decode_kernel(DecodeArgs a) {
    extern __shared__ float dsm[];
    float *ks = dsm, *qs = ks + kDD, *vs = qs + kDD, *slots = vs + kDD;  // slots: 7 x 4 floats
    const int seq = blockIdx.x, tid = threadIdx.x, n = a.n;
    const int lane = tid & 31, warp = tid >> 5;
    const int j = warp * 16 + (lane >> 1), h = lane & 1;
    float *W = a.W + (size_t)seq * kDD * kDD;
    float Wr[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) Wr[r] = W[(32 * h + r) * kDD + j];
    const float g = a.ln ? a.gamma[(size_t)(seq % a.H) * kDD + j] : 1.f;
    const float be = a.ln ? a.beta[(size_t)(seq % a.H) * kDD + j] : 0.f;
    // token 0's q, k, v and eta; later tokens are loaded one token ahead
    float kn = 0.f, qn = 0.f, vn = 0.f;
    if (tid < kDD) {
        const size_t r0 = (size_t)seq * n * kDD + tid;
        kn = load_elem(a.k, r0, a.bf16);
        qn = load_elem(a.q, r0, a.bf16);
        vn = load_elem(a.v, r0, a.bf16);
    }
    float etan = a.eta[(size_t)seq * n];
    for (int t = 0; t < n; ++t) {
    const size_t row = ((size_t)seq * n + t) * kDD;
    if (t > 0) __syncthreads();  // every reader of the previous token's staging is done
    if (tid < kDD) {
        ks[tid] = kn;
        qs[tid] = qn;
        vs[tid] = vn;
    }
    const float eta = etan;
    if (t + 1 < n) {
        if (tid < kDD) {
            kn = load_elem(a.k, row + kDD + tid, a.bf16);
            qn = load_elem(a.q, row + kDD + tid, a.bf16);
            vn = load_elem(a.v, row + kDD + tid, a.bf16);
        }
        etan = a.eta[(size_t)seq * n + t + 1];
    }
    __syncthreads();  // k, q, v staged
    if (a.l2_keys) {  // k / max(||k||, 1e-12), as the listing normalises its key
        const float kk = ks[j];
        const float inv = 1.f / fmaxf(sqrtf(col_sum(kk * kk, h, slots + 24)), 1e-12f);
        if (h == 0) ks[j] = kk * inv;
        __syncthreads();
    }

    // x_j = sum_i k_i W[i][j]
    float x = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) x = fmaf(ks[32 * h + r], Wr[r], x);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    float G;
    if (a.ln) {
        const float mu = col_sum(x, h, slots) * (1.f / kDD);
        const float c = x - mu;
        const float var = col_sum(c * c, h, slots + 4) * (1.f / kDD);
        const float rs = rsqrtf(var + kLnEps);
        const float xh = c * rs;
        const float gh = g * (ks[j] + g * xh + be - vs[j]);
        const float m1 = col_sum(gh, h, slots + 8) * (1.f / kDD);
        const float m2 = col_sum(gh * xh, h, slots + 12) * (1.f / kDD);
        G = eta * (gh - m1 - xh * m2) * rs;
    } else {
        G = eta * (x - vs[j]);
    }
    // W <- W - k^T G ; then z_pre_j = sum_i q_i W[i][j]
    float zp = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        Wr[r] = fmaf(-ks[32 * h + r], G, Wr[r]);
        zp = fmaf(qs[32 * h + r], Wr[r], zp);
    }
    zp += __shfl_xor_sync(0xffffffffu, zp, 1);
    float z = zp;
    if (a.ln) {
        const float mu = col_sum(zp, h, slots + 16) * (1.f / kDD);
        const float c = zp - mu;
        const float var = col_sum(c * c, h, slots + 20) * (1.f / kDD);
        z = qs[j] + g * (c * rsqrtf(var + kLnEps)) + be;
    }
    if (h == 0) store_z1(a.z, a.z_bf16, row + j, z);
    }
#pragma unroll
    for (int r = 0; r < 32; ++r) W[(32 * h + r) * kDD + j] = Wr[r];
}

}  // namespace

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
cudaError_t launch_linear_decode(const void *q, const void *k, const void *v, const float *eta,
                                 const float *gamma, const float *beta, float *W, void *z, int B,
                                 int H, int n, bool bf16, bool ln, bool z_bf16, bool l2_keys,
                                 cudaStream_t s) {
    const DecodeArgs a{q, k, v, eta, gamma, beta, W, static_cast<float *>(z), H,
                       bf16, ln, z_bf16, l2_keys, n};
    const size_t smem = sizeof(float) * (3 * kDD + 7 * 4);
    linear_decode_kernel<<<(unsigned)(B * H), kDecThreads, smem, s>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}
#endif  // TTT_HOST_RUN

}  // namespace ttt
