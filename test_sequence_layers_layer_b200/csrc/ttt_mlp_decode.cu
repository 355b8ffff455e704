// ttt_mlp_decode.cu -- one TTT-MLP token per sequence (online decode, b = 1),
// d = 64, hidden 256, both layers updated in place.
//
// Method (TTT-MLP: "How to Master Test-Time Training for LLMs", the fast
// weight an MLP; update and read-out rules of "Key Architectural Mechanics of
// TTT-Linear", parts 1-3). For the token (q, k, v) with step size eta and the
// sequence's weights W1 [64][256], W2 [256][64]:
//   h = k W1, a = GELU(h), x = a W2, Gx = eta * LNbwd(x; gamma*(k + gamma*xhat + beta - v)),
//   Gh = (Gx W2^T) * GELU'(h),  W1 <- W1 - k^T Gh,  W2 <- W2 - a^T Gx,
//   z = q + gamma * LN(GELU(q W1) W2) + beta          (with the updated weights).
// One block of 256 threads per sequence; thread j owns hidden unit j: column
// j of W1 and row j of W2 in registers. Everything on layer 1 is then local
// to a thread; the two products over the hidden units (x = a W2 and the
// read-out's) are reduced across the block by a warp reduce-scatter (lane l
// ends with outputs 2l and 2l+1 of its warp's sum, 62 shuffles) and a sum of
// the 8 warps' partials through shared memory. The LayerNorm work runs on
// threads 0-63, one output each. The weights stay in registers over all n
// tokens of a call (the next token's q, k, v are loaded one token ahead) and
// are read once and written once per call.
#include "../../include/ttt.h"
#include "ttt_common.cuh"

namespace ttt {
namespace {

constexpr int kMD = 64, kMF = 256, kMThreads = 256, kMWarps = kMThreads / 32;

struct MlpDecodeArgs {
    const void *q, *k, *v;
    const float *eta, *gamma, *beta;
    float *W1, *W2;  // [S][64][256], [S][256][64], updated in place
    float *z;        // [S][n][64]; bf16 when z_bf16
    int H;
    bool bf16, z_bf16;
    int n = 1;  // tokens per sequence in this call (q, k, v [S][n][64], eta [S][n])
};

__device__ __forceinline__ float md_gelu(float h) {
    return h * 0.5f * (1.f + erff(h * 0.70710678118654752f));
}
__device__ __forceinline__ float md_gelu1(float h) {
    return 0.5f * (1.f + erff(h * 0.70710678118654752f)) +
           h * 0.39894228040143268f * expf(-0.5f * h * h);
}
__device__ __forceinline__ float md_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Warp reduce-scatter of the 64-vector v over the 32 lanes: afterwards lane l
// holds, in v[0] and v[1], elements 2l and 2l+1 of the sum over the warp.
// At each step a lane keeps the half its lane bit selects and adds the
// partner's copy of that half.
__device__ __forceinline__ void reduce_scatter64(float (&v)[kMD], int lane) {
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int o = 16 >> s, half = 32 >> s;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

// Sum over the block of a value held by threads 0..63 (others pass 0); all
// threads call it; `slot` is a 2-float area used by this reduction only.
__device__ __forceinline__ float sum64(float v, float *slot) {
    const float w = md_warp_sum(threadIdx.x < kMD ? v : 0.f);
    if (threadIdx.x == 0 || threadIdx.x == 32) slot[threadIdx.x >> 5] = w;
    __syncthreads();
    return slot[0] + slot[1];
}

__global__ void __launch_bounds__(kMThreads, 1) mlp_decode_kernel(MlpDecodeArgs a) {
    extern __shared__ float msm[];
    float *ks = msm, *qs = ks + kMD, *vs = qs + kMD, *xs = vs + kMD, *gx = xs + kMD;
    float *R = gx + kMD;                 // [8][64] warp partials
    float *slots = R + kMWarps * kMD;    // 8 reductions x 2 floats
    const int seq = blockIdx.x, j = threadIdx.x, lane = j & 31, warp = j >> 5, n = a.n;
    float *W1 = a.W1 + (size_t)seq * kMD * kMF, *W2 = a.W2 + (size_t)seq * kMF * kMD;
    float w1[kMD], w2[kMD];  // column j of W1, row j of W2
#pragma unroll
    for (int i = 0; i < kMD; ++i) w1[i] = W1[i * kMF + j];
#pragma unroll
    for (int c = 0; c < kMD; c += 4) {
        const float4 u = *reinterpret_cast<const float4 *>(W2 + (size_t)j * kMD + c);
        w2[c] = u.x;
        w2[c + 1] = u.y;
        w2[c + 2] = u.z;
        w2[c + 3] = u.w;
    }
    const int hh = seq % a.H;
    const float g = j < kMD ? a.gamma[(size_t)hh * kMD + j] : 0.f;
    const float be = j < kMD ? a.beta[(size_t)hh * kMD + j] : 0.f;
    // token 0's q, k, v and eta; later tokens are loaded one token ahead
    float kn = 0.f, qn = 0.f, vn = 0.f;
    if (j < kMD) {
        const size_t r0 = (size_t)seq * n * kMD + j;
        kn = load_elem(a.k, r0, a.bf16);
        qn = load_elem(a.q, r0, a.bf16);
        vn = load_elem(a.v, r0, a.bf16);
    }
    float etan = a.eta[(size_t)seq * n];
    for (int t = 0; t < n; ++t) {
    const size_t row = ((size_t)seq * n + t) * kMD;
    if (t > 0) __syncthreads();  // every reader of the previous token's staging is done
    if (j < kMD) {
        ks[j] = kn;
        qs[j] = qn;
        vs[j] = vn;
    }
    const float eta = etan;
    if (t + 1 < n) {
        if (j < kMD) {
            kn = load_elem(a.k, row + kMD + j, a.bf16);
            qn = load_elem(a.q, row + kMD + j, a.bf16);
            vn = load_elem(a.v, row + kMD + j, a.bf16);
        }
        etan = a.eta[(size_t)seq * n + t + 1];
    }
    __syncthreads();  // k, q, v staged

    // layer 1 (local): h_j = k . W1[:, j]
    float h = 0.f;
#pragma unroll
    for (int i = 0; i < kMD; ++i) h = fmaf(ks[i], w1[i], h);
    const float act = md_gelu(h), d1 = md_gelu1(h);
    // x = a W2: reduce-scatter of a_j * W2[j, :] over the block
    {
        float p[kMD];
#pragma unroll
        for (int c = 0; c < kMD; ++c) p[c] = act * w2[c];
        reduce_scatter64(p, lane);
        R[warp * kMD + 2 * lane] = p[0];
        R[warp * kMD + 2 * lane + 1] = p[1];
    }
    __syncthreads();
    float x = 0.f;
    if (j < kMD) {
#pragma unroll
        for (int w = 0; w < kMWarps; ++w) x += R[w * kMD + j];
    }
    // Gx = eta * LayerNorm backward of f - v (threads 0..63, one output each)
    const float mu = sum64(x, slots) * (1.f / kMD);
    const float cx = x - mu;
    const float rs = rsqrtf(sum64(cx * cx, slots + 2) * (1.f / kMD) + kLnEps);
    const float xh = cx * rs;
    const float gh = j < kMD ? g * (ks[j] + g * xh + be - vs[j]) : 0.f;
    const float m1 = sum64(gh, slots + 4) * (1.f / kMD);
    const float m2 = sum64(gh * xh, slots + 6) * (1.f / kMD);
    if (j < kMD) gx[j] = eta * (gh - m1 - xh * m2) * rs;
    __syncthreads();
    // Gh_j = (Gx . W2[j, :]) * GELU'(h_j); then both updates (local)
    float ga = 0.f;
#pragma unroll
    for (int c = 0; c < kMD; ++c) ga = fmaf(gx[c], w2[c], ga);
    const float Gh = ga * d1;
#pragma unroll
    for (int i = 0; i < kMD; ++i) w1[i] = fmaf(-ks[i], Gh, w1[i]);
#pragma unroll
    for (int c = 0; c < kMD; ++c) w2[c] = fmaf(-act, gx[c], w2[c]);
    // read-out with the updated weights
    float hq = 0.f;
#pragma unroll
    for (int i = 0; i < kMD; ++i) hq = fmaf(qs[i], w1[i], hq);
    const float aq = md_gelu(hq);
    {
        float p[kMD];
#pragma unroll
        for (int c = 0; c < kMD; ++c) p[c] = aq * w2[c];
        reduce_scatter64(p, lane);
        // R was last read before the Gx barrier above, so it can be rewritten
        R[warp * kMD + 2 * lane] = p[0];
        R[warp * kMD + 2 * lane + 1] = p[1];
    }
    __syncthreads();
    float xq = 0.f;
    if (j < kMD) {
#pragma unroll
        for (int w = 0; w < kMWarps; ++w) xq += R[w * kMD + j];
    }
    const float muq = sum64(xq, slots + 8) * (1.f / kMD);
    const float cq = xq - muq;
    const float rq = rsqrtf(sum64(cq * cq, slots + 10) * (1.f / kMD) + kLnEps);
    if (j < kMD) store_z1(a.z, a.z_bf16, row + j, qs[j] + g * (cq * rq) + be);
    }
#pragma unroll
    for (int i = 0; i < kMD; ++i) W1[i * kMF + j] = w1[i];
#pragma unroll
    for (int c = 0; c < kMD; c += 4)
        *reinterpret_cast<float4 *>(W2 + (size_t)j * kMD + c) =
            make_float4(w2[c], w2[c + 1], w2[c + 2], w2[c + 3]);
}

}  // namespace

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
cudaError_t launch_mlp_decode(const void *q, const void *k, const void *v, const float *eta,
                              const float *gamma, const float *beta, float *W1, float *W2,
                              void *z, int B, int H, int n, bool bf16, bool z_bf16,
                              cudaStream_t s) {
    const MlpDecodeArgs a{q, k, v, eta, gamma, beta, W1, W2, static_cast<float *>(z), H, bf16,
                          z_bf16, n};
    const size_t smem = sizeof(float) * (5 * kMD + kMWarps * kMD + 16);
    mlp_decode_kernel<<<(unsigned)(B * H), kMThreads, smem, s>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}
#endif  // TTT_HOST_RUN

}  // namespace ttt
