// ttt_simt.cu -- fp32 CUDA-core kernels of the TTT forward pass.
//
// One thread block per (batch, head) sequence; the fast weight lives in
// shared memory in fp32 for the whole scan and is written to HBM once at the
// end. These kernels cover every supported shape in plain fp32 FFMA
// arithmetic: they are the path for fp32 inputs and for shapes the tensor-core
// kernels do not take, and they carry the 1e-5 fp32 tolerance.
//
// Method (TTT pages, "Test-Time Training: Linear Complexity Beyond
// Attention", "Key Architectural Mechanics of TTT-Linear" parts 1-4): per
// mini-batch of b tokens starting from W_m,
//   G'  = diag(eta) * dl/dX  at X = K W_m,
//   Z   = f-epilogue( Q W_m - tril(Q K^T) G' ),   tril including the diagonal,
//   W_{m+1} = W_m - K^T G'.
#include "ttt_common.cuh"

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------
// LayerNorm helpers over one row of n values held in shared memory; one warp
// handles the row, its lanes striding over it.

// Returns (mean, 1/sigma) of row x[0..n).
__device__ __forceinline__ float2 row_stats(const float *x, int n) {
    float s = 0.f;
    for (int j = threadIdx.x & 31; j < n; j += 32) s += x[j];
    const float mu = warp_sum(s) / n;
    float v = 0.f;
    for (int j = threadIdx.x & 31; j < n; j += 32) {
        const float c = x[j] - mu;
        v += c * c;
    }
    const float var = warp_sum(v) / n;
    return make_float2(mu, rsqrtf(var + kLnEps));
}

// In place: x <- eta * dl/dx for l = 1/2||k + gamma*xhat + beta - v||^2,
// x = the pre-LayerNorm row. (LayerNorm backward: (ghat - mean(ghat) -
// xhat*mean(ghat*xhat)) / sigma with ghat = gamma * (f - v).)
__device__ __forceinline__ void ln_grad_row(float *x, const float *k, const float *v,
                                            const float *gamma, const float *beta, float eta,
                                            int n) {
    const float2 st = row_stats(x, n);
    float m1 = 0.f, m2 = 0.f;
    for (int j = threadIdx.x & 31; j < n; j += 32) {
        const float xh = (x[j] - st.x) * st.y;
        const float gh = gamma[j] * (k[j] + gamma[j] * xh + beta[j] - v[j]);
        m1 += gh;
        m2 += gh * xh;
    }
    m1 = warp_sum(m1) / n;
    m2 = warp_sum(m2) / n;
    __syncwarp();
    for (int j = threadIdx.x & 31; j < n; j += 32) {
        const float xh = (x[j] - st.x) * st.y;
        const float gh = gamma[j] * (k[j] + gamma[j] * xh + beta[j] - v[j]);
        x[j] = eta * (gh - m1 - xh * m2) * st.y;
    }
}

// Z[off + j] = q[j] + gamma[j] * LN(x)[j] + beta[j]   (fp32, or bf16 when zb)
__device__ __forceinline__ void ln_residual_store(const float *x, const float *q,
                                                  const float *gamma, const float *beta,
                                                  float *Z, bool zb, size_t off, int n) {
    const float2 st = row_stats(x, n);
    for (int j = threadIdx.x & 31; j < n; j += 32)
        store_z1(Z, zb, off + j, q[j] + gamma[j] * ((x[j] - st.x) * st.y) + beta[j]);
}

__device__ __forceinline__ float gelu(float h) {
    return h * 0.5f * (1.f + erff(h * 0.70710678118654752f));
}
__device__ __forceinline__ float gelu_prime(float h) {
    const float Phi = 0.5f * (1.f + erff(h * 0.70710678118654752f));
    return Phi + h * 0.39894228040143268f * expf(-0.5f * h * h);
}

__device__ __forceinline__ void load_tile(float *dst, const void *src, size_t base, int n,
                                          bool bf16) {
    for (int e = threadIdx.x; e < n; e += blockDim.x) dst[e] = load_elem(src, base + e, bf16);
}

// ---------------------------------------------------------------------------
// TTT-Linear, mini-batch dual form, fp32.
// Shared memory: W[d*d] | Qs Ks Vs Xs Zs [b*d] | S[b*b] | es[b].
// l2_keys: every key is scaled to unit length, k / max(||k||, 1e-12), before
// it enters the inner loss, its gradient and the update (the key
// normalisation of the PyTorch listing on "Test-Time Training: Linear
// Complexity Beyond Attention"); queries are used as given.
// n_steps > 1 (only with b = 1): the token takes n_steps gradient steps, each
// at the weight the previous one left, before it reads out ("How to Master
// Test-Time Training for LLMs", "How TTT Layers Actually Work": one or more
// gradient steps per token). With W' = W_m - k^T (G_1 + ... + G_n), the
// read-out q W' = q W_m - (q . k) (G_1 + ... + G_n); Gs holds that sum.
// Shared memory then also holds Gs[b*d] after es.
__global__ void __launch_bounds__(kThreads) linear_simt_kernel(LinearArgs a, bool l2_keys,
                                                               int n_steps) {
    extern __shared__ float sm[];
    const int d = a.d, b = a.b, T = a.T;
    const int seq = blockIdx.x, h = seq % a.H;
    float *W = sm, *Qs = W + d * d, *Ks = Qs + b * d, *Vs = Ks + b * d, *Xs = Vs + b * d,
          *Zs = Xs + b * d, *S = Zs + b * d, *es = S + b * b, *Gs = es + b;
    const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : h) * d * d;
    const float *gamma = a.ln ? a.gamma + (size_t)h * d : nullptr;
    const float *beta = a.ln ? a.beta + (size_t)h * d : nullptr;
    const int warp = threadIdx.x >> 5;

    for (int e = threadIdx.x; e < d * d; e += blockDim.x) W[e] = W0[e];
    for (int m0 = 0; m0 < T; m0 += b) {
        const size_t base = ((size_t)seq * T + m0) * d;
        // A partial last mini-batch holds nb < b tokens: the other rows are
        // zero with step size 0, so they change no weight and are not stored.
        const int nb = T - m0 < b ? T - m0 : b;
        load_tile(Qs, a.Q, base, nb * d, a.bf16);
        load_tile(Ks, a.K, base, nb * d, a.bf16);
        load_tile(Vs, a.V, base, nb * d, a.bf16);
        for (int e = nb * d + threadIdx.x; e < b * d; e += blockDim.x) Qs[e] = Ks[e] = Vs[e] = 0.f;
        for (int e = threadIdx.x; e < b; e += blockDim.x) es[e] = e < nb ? a.eta[(size_t)seq * T + m0 + e] : 0.f;
        __syncthreads();
        if (l2_keys) {  // one warp per key row; padding rows are zero and stay zero
            for (int t = warp; t < b; t += kWarps) {
                float *k = Ks + t * d;
                float ss = 0.f;
                for (int j = threadIdx.x & 31; j < d; j += 32) ss = fmaf(k[j], k[j], ss);
                const float inv = 1.f / fmaxf(sqrtf(warp_sum(ss)), 1e-12f);
                for (int j = threadIdx.x & 31; j < d; j += 32) k[j] *= inv;
            }
            __syncthreads();
        }
        // X = K W_m and Q W_m
        for (int e = threadIdx.x; e < b * d; e += blockDim.x) {
            const int t = e / d, j = e % d;
            float ax = 0.f, az = 0.f;
            for (int i = 0; i < d; ++i) {
                const float w = W[i * d + j];
                ax = fmaf(Ks[t * d + i], w, ax);
                az = fmaf(Qs[t * d + i], w, az);
            }
            Xs[e] = ax;
            Zs[e] = az;
        }
        // S = tril(Q K^T), diagonal included
        for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int i = 0; i < d; ++i) acc = fmaf(Qs[t * d + i], Ks[s * d + i], acc);
            S[e] = acc;
        }
        __syncthreads();
        // G' = diag(eta) dl/dX, one warp per row
        for (int t = warp; t < b; t += kWarps) {
            float *x = Xs + t * d;
            if (a.ln) {
                ln_grad_row(x, Ks + t * d, Vs + t * d, gamma, beta, es[t], d);
            } else {
                for (int j = threadIdx.x & 31; j < d; j += 32) x[j] = es[t] * (x[j] - Vs[t * d + j]);
            }
        }
        __syncthreads();
        // Further steps of the token (b = 1): apply G, sum it, take the next
        // gradient at the updated weight. The last G is applied below.
        for (int step = 1; step < n_steps; ++step) {
            for (int j = threadIdx.x; j < d; j += blockDim.x) Gs[j] = (step == 1 ? 0.f : Gs[j]) + Xs[j];
            for (int e = threadIdx.x; e < d * d; e += blockDim.x) W[e] -= Ks[e / d] * Xs[e % d];
            __syncthreads();
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float ax = 0.f;
                for (int i = 0; i < d; ++i) ax = fmaf(Ks[i], W[i * d + j], ax);
                Xs[j] = ax;
            }
            __syncthreads();
            if (warp == 0) {
                if (a.ln) {
                    ln_grad_row(Xs, Ks, Vs, gamma, beta, es[0], d);
                } else {
                    for (int j = threadIdx.x & 31; j < d; j += 32) Xs[j] = es[0] * (Xs[j] - Vs[j]);
                }
            }
            __syncthreads();
        }
        if (n_steps > 1) {
            for (int j = threadIdx.x; j < d; j += blockDim.x) Gs[j] += Xs[j];
            __syncthreads();
        }
        // Zpre = Q W_m - S G'  (with several steps: - S (G_1 + ... + G_n))
        const float *Gz = n_steps > 1 ? Gs : Xs;
        for (int e = threadIdx.x; e < b * d; e += blockDim.x) {
            const int t = e / d, j = e % d;
            float acc = Zs[e];
            for (int s = 0; s <= t; ++s) acc = fmaf(-S[t * b + s], Gz[s * d + j], acc);
            Zs[e] = acc;
        }
        // W_{m+1} = W_m - K^T G'
        for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
            const int i = e / d, j = e % d;
            float acc = 0.f;
            for (int s = 0; s < b; ++s) acc = fmaf(Ks[s * d + i], Xs[s * d + j], acc);
            W[e] -= acc;
        }
        __syncthreads();
        // output epilogue
        for (int t = warp; t < nb; t += kWarps) {
            const size_t out = base + (size_t)t * d;
            if (a.ln) {
                ln_residual_store(Zs + t * d, Qs + t * d, gamma, beta, a.Z, a.z_bf16, out, d);
            } else {
                for (int j = threadIdx.x & 31; j < d; j += 32) store_z1(a.Z, a.z_bf16, out + j, Zs[t * d + j]);
            }
        }
        __syncthreads();
    }
    if (a.W_out)
        for (int e = threadIdx.x; e < d * d; e += blockDim.x) a.W_out[(size_t)seq * d * d + e] = W[e];
}

// ---------------------------------------------------------------------------
// TTT-MLP, two-stage dual form, fp32.
// Shared memory: W1[d*dh] | W2[dh*d] | Qs Ks Vs Xs Zs [b*d] | Hk Ak Gh Hq [b*dh] | S[b*b] | es[b]
__global__ void __launch_bounds__(kThreads) mlp_simt_kernel(MlpArgs a) {
    extern __shared__ float sm[];
    const int d = a.d, dh = a.dh, b = a.b, T = a.T;
    const int seq = blockIdx.x, h = seq % a.H;
    float *W1 = sm, *W2 = W1 + d * dh, *Qs = W2 + dh * d, *Ks = Qs + b * d, *Vs = Ks + b * d,
          *Xs = Vs + b * d, *Zs = Xs + b * d, *Hk = Zs + b * d, *Ak = Hk + b * dh,
          *Gh = Ak + b * dh, *Hq = Gh + b * dh, *S = Hq + b * dh, *es = S + b * b;
    const int widx = a.w0_per_seq ? seq : h;
    const float *W1_0 = a.W1_0 + (size_t)widx * d * dh, *W2_0 = a.W2_0 + (size_t)widx * dh * d;
    const float *gamma = a.gamma + (size_t)h * d, *beta = a.beta + (size_t)h * d;
    const int warp = threadIdx.x >> 5;

    for (int e = threadIdx.x; e < d * dh; e += blockDim.x) {
        W1[e] = W1_0[e];
        W2[e] = W2_0[e];
    }
    for (int m0 = 0; m0 < T; m0 += b) {
        const size_t base = ((size_t)seq * T + m0) * d;
        load_tile(Qs, a.Q, base, b * d, a.bf16);
        load_tile(Ks, a.K, base, b * d, a.bf16);
        load_tile(Vs, a.V, base, b * d, a.bf16);
        for (int e = threadIdx.x; e < b; e += blockDim.x) es[e] = a.eta[(size_t)seq * T + m0 + e];
        __syncthreads();
        // Hk = K W1, Hq = Q W1 (the query side before its causal correction)
        for (int e = threadIdx.x; e < b * dh; e += blockDim.x) {
            const int t = e / dh, j = e % dh;
            float ak = 0.f, aq = 0.f;
            for (int i = 0; i < d; ++i) {
                const float w = W1[i * dh + j];
                ak = fmaf(Ks[t * d + i], w, ak);
                aq = fmaf(Qs[t * d + i], w, aq);
            }
            Hk[e] = ak;
            Ak[e] = gelu(ak);
            Hq[e] = aq;
        }
        for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int i = 0; i < d; ++i) acc = fmaf(Qs[t * d + i], Ks[s * d + i], acc);
            S[e] = acc;
        }
        __syncthreads();
        // X = A W2
        for (int e = threadIdx.x; e < b * d; e += blockDim.x) {
            const int t = e / d, j = e % d;
            float acc = 0.f;
            for (int i = 0; i < dh; ++i) acc = fmaf(Ak[t * dh + i], W2[i * d + j], acc);
            Xs[e] = acc;
        }
        __syncthreads();
        for (int t = warp; t < b; t += kWarps)
            ln_grad_row(Xs + t * d, Ks + t * d, Vs + t * d, gamma, beta, es[t], d);
        __syncthreads();
        // Gh' = (Gx' W2^T) * GELU'(Hk)
        for (int e = threadIdx.x; e < b * dh; e += blockDim.x) {
            const int t = e / dh, i = e % dh;
            float acc = 0.f;
            for (int j = 0; j < d; ++j) acc = fmaf(Xs[t * d + j], W2[i * d + j], acc);
            Gh[e] = acc * gelu_prime(Hk[e]);
        }
        __syncthreads();
        // Hq -= tril(Q K^T) Gh';  Aq = GELU(Hq) (in place)
        for (int e = threadIdx.x; e < b * dh; e += blockDim.x) {
            const int t = e / dh, i = e % dh;
            float acc = Hq[e];
            for (int s = 0; s <= t; ++s) acc = fmaf(-S[t * b + s], Gh[s * dh + i], acc);
            Hq[e] = gelu(acc);
        }
        __syncthreads();
        // S2 = tril(Aq Ak^T)
        for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int i = 0; i < dh; ++i) acc = fmaf(Hq[t * dh + i], Ak[s * dh + i], acc);
            S[e] = acc;
        }
        __syncthreads();
        // Zpre = Aq W2 - S2 Gx'
        for (int e = threadIdx.x; e < b * d; e += blockDim.x) {
            const int t = e / d, j = e % d;
            float acc = 0.f;
            for (int i = 0; i < dh; ++i) acc = fmaf(Hq[t * dh + i], W2[i * d + j], acc);
            for (int s = 0; s <= t; ++s) acc = fmaf(-S[t * b + s], Xs[s * d + j], acc);
            Zs[e] = acc;
        }
        __syncthreads();
        // W1 -= K^T Gh',  W2 -= Ak^T Gx'
        for (int e = threadIdx.x; e < d * dh; e += blockDim.x) {
            {
                const int i = e / dh, j = e % dh;
                float acc = 0.f;
                for (int s = 0; s < b; ++s) acc = fmaf(Ks[s * d + i], Gh[s * dh + j], acc);
                W1[e] -= acc;
            }
            {
                const int i = e / d, j = e % d;
                float acc = 0.f;
                for (int s = 0; s < b; ++s) acc = fmaf(Ak[s * dh + i], Xs[s * d + j], acc);
                W2[e] -= acc;
            }
        }
        for (int t = warp; t < b; t += kWarps)
            ln_residual_store(Zs + t * d, Qs + t * d, gamma, beta, a.Z, a.z_bf16, base + (size_t)t * d, d);
        __syncthreads();
    }
    if (a.W1_out)
        for (int e = threadIdx.x; e < d * dh; e += blockDim.x) a.W1_out[(size_t)seq * d * dh + e] = W1[e];
    if (a.W2_out)
        for (int e = threadIdx.x; e < d * dh; e += blockDim.x) a.W2_out[(size_t)seq * d * dh + e] = W2[e];
}

// ---------------------------------------------------------------------------
// Large-chunk TTT, apply-then-update, fp32. One block per sequence; the
// chunk's weight change accumulates in registers (d*d / 256 per thread).
constexpr int kChunkRows = 32;
constexpr int kMaxAccPerThread = 128 * 128 / kThreads;

__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkArgs a) {
    extern __shared__ float sm[];
    const int d = a.d, T = a.T, C = a.chunk;
    const int seq = blockIdx.x, h = seq % a.H;
    float *W = sm, *Qs = W + d * d, *Ks = Qs + kChunkRows * d, *Vs = Ks + kChunkRows * d,
          *Gs = Vs + kChunkRows * d, *es = Gs + kChunkRows * d;
    const float *W0 = a.W0 + (size_t)(a.w0_per_seq ? seq : h) * d * d;
    const int per = d * d / kThreads;  // d*d is a multiple of 256 for supported d
    float acc[kMaxAccPerThread];

    for (int e = threadIdx.x; e < d * d; e += blockDim.x) W[e] = W0[e];
    for (int c0 = 0; c0 < T; c0 += C) {
#pragma unroll
        for (int k = 0; k < kMaxAccPerThread; ++k) acc[k] = 0.f;
        for (int r0 = c0; r0 < c0 + C; r0 += kChunkRows) {
            const size_t base = ((size_t)seq * T + r0) * d;
            __syncthreads();
            load_tile(Qs, a.Q, base, kChunkRows * d, a.bf16);
            load_tile(Ks, a.K, base, kChunkRows * d, a.bf16);
            load_tile(Vs, a.V, base, kChunkRows * d, a.bf16);
            for (int e = threadIdx.x; e < kChunkRows; e += blockDim.x)
                es[e] = a.eta[(size_t)seq * T + r0 + e];
            __syncthreads();
            for (int e = threadIdx.x; e < kChunkRows * d; e += blockDim.x) {
                const int t = e / d, j = e % d;
                float az = 0.f, ax = 0.f;
                for (int i = 0; i < d; ++i) {
                    const float w = W[i * d + j];
                    az = fmaf(Qs[t * d + i], w, az);
                    ax = fmaf(Ks[t * d + i], w, ax);
                }
                store_z1(a.Z, a.z_bf16, base + e, az);
                Gs[e] = es[t] * (ax - Vs[e]);
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kMaxAccPerThread; ++k) {
                if (k < per) {
                    const int e = threadIdx.x + k * kThreads, i = e / d, j = e % d;
                    float s = acc[k];
                    for (int t = 0; t < kChunkRows; ++t) s = fmaf(Ks[t * d + i], Gs[t * d + j], s);
                    acc[k] = s;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kMaxAccPerThread; ++k)
            if (k < per) W[threadIdx.x + k * kThreads] -= acc[k];
    }
    __syncthreads();
    if (a.W_out)
        for (int e = threadIdx.x; e < d * d; e += blockDim.x) a.W_out[(size_t)seq * d * d + e] = W[e];
}

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
// Opt a kernel in to more than 48 KB of dynamic shared memory.
template <typename K>
cudaError_t set_smem(K kernel, size_t smem) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
#endif  // TTT_HOST_RUN

}  // namespace

#ifndef TTT_HOST_RUN
cudaError_t launch_linear_simt_opts(const LinearArgs &a, bool l2_keys, int n_steps,
                                   cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)a.d * a.d + 6 * (size_t)a.b * a.d +
                                         (size_t)a.b * a.b + a.b);
    cudaError_t e = set_smem(linear_simt_kernel, smem);
    if (e != cudaSuccess) return e;
    linear_simt_kernel<<<a.B * a.H, kThreads, smem, s>>>(a, l2_keys, n_steps);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

cudaError_t launch_linear_simt_keys(const LinearArgs &a, bool l2_keys, cudaStream_t s) {
    return launch_linear_simt_opts(a, l2_keys, 1, s);
}

cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t s) {
    return launch_linear_simt_opts(a, false, 1, s);
}

size_t mlp_simt_smem(int d, int dh, int b) {
    return sizeof(float) * (2 * (size_t)d * dh + 5 * (size_t)b * d + 4 * (size_t)b * dh +
                            (size_t)b * b + b);
}

cudaError_t launch_mlp_simt(const MlpArgs &a, cudaStream_t s) {
    const size_t smem = mlp_simt_smem(a.d, a.dh, a.b);
    cudaError_t e = set_smem(mlp_simt_kernel, smem);
    if (e != cudaSuccess) return e;
    mlp_simt_kernel<<<a.B * a.H, kThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)a.d * a.d + 4 * (size_t)kChunkRows * a.d + kChunkRows);
    cudaError_t e = set_smem(chunk_simt_kernel, smem);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<<<a.B * a.H, kThreads, smem, s>>>(a);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

#endif  // TTT_HOST_RUN

}  // namespace ttt
