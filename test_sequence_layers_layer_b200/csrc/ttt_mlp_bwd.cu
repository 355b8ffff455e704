// ttt_mlp_bwd.cu -- backward pass (outer gradients) of TTT-MLP on CUDA cores
// in fp32: one block of 256 threads per (batch, head) sequence. The kernel
// body, with its derivation, is ttt_mlp_bwd_body.inc; this file gives it a
// block context (threadIdx, __syncthreads, dynamic shared memory), sums the
// per-sequence weight and LayerNorm gradients over the batch, and launches.
#include <cstring>

#include "../../include/ttt.h"
#include "ttt_common.cuh"
#include "ttt_mlp_bwd_body.inc"

namespace ttt {
namespace {

constexpr int kBwdThreads = 256;

struct DevCtx {
    int tid, nt;
    float *sm;
    __device__ void sync() { __syncthreads(); }
    // sum over the 32 lanes of the calling warp; every lane must call it
    __device__ float warp_sum(float v) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        return v;
    }
};

__global__ void __launch_bounds__(kBwdThreads) mlp_bwd_kernel(mlp_bwd_body::Params p) {
    extern __shared__ float sm[];
    DevCtx cx{(int)threadIdx.x, (int)blockDim.x, sm};
    mlp_bwd_body::run_sequence(cx, p, (int)blockIdx.x);
}

// dgamma, dbeta [H][d] (and dW1_0, dW2_0 [H][..] when W0 is shared): sums of
// the sequences' own gradients over the batch, in batch order.
__global__ void mlp_bwd_sum_kernel(const float *ws, size_t ws_per_seq, int B, int H, int T,
                                   int d, int b, bool shared_w0, float *dW1_0, float *dW2_0,
                                   float *dgamma, float *dbeta) {
    const int h = blockIdx.x;
    const size_t dF = (size_t)d * 4 * d;
    for (size_t e = threadIdx.x; e < 2 * dF + 2 * (size_t)d; e += blockDim.x) {
        float acc = 0.f;
        for (int bb = 0; bb < B; ++bb) {
            const mlp_bwd_body::Ws w = mlp_bwd_body::ws_view(
                const_cast<float *>(ws) + (size_t)(bb * H + h) * ws_per_seq, T, d, b);
            acc += e < dF ? w.dW1[e] : e < 2 * dF ? w.dW2[e - dF]
                  : e < 2 * dF + d              ? w.dg[e - 2 * dF]
                                                : w.db[e - 2 * dF - d];
        }
        if (e < dF) {
            if (shared_w0) dW1_0[(size_t)h * dF + e] = acc;
        } else if (e < 2 * dF) {
            if (shared_w0) dW2_0[(size_t)h * dF + e - dF] = acc;
        } else if (e < 2 * dF + d) {
            dgamma[(size_t)h * d + e - 2 * dF] = acc;
        } else {
            dbeta[(size_t)h * d + e - 2 * dF - d] = acc;
        }
    }
}

}  // namespace

bool mlp_bwd_supported(int d, int dh, int b) {
    return (d == 16 || d == 32 || d == 64) && dh == 4 * d && b >= 1 && b <= mlp_bwd_body::kMlpBwdMaxB;
}

size_t mlp_bwd_workspace_bytes(int B, int H, int T, int d, int b) {
    return sizeof(float) * (size_t)B * H * mlp_bwd_body::ws_floats_per_seq(T, d, b);
}

cudaError_t launch_mlp_bwd(const void *Q, const void *K, const void *V, const float *eta,
                           const float *W1_0, const float *W2_0, const float *gamma,
                           const float *beta, const float *dZ, const float *dW1_out,
                           const float *dW2_out, float *dQ, float *dK, float *dV, float *deta,
                           float *dW1_0, float *dW2_0, float *dgamma, float *dbeta, int B, int H,
                           int T, int d, int b, bool bf16, bool w0_per_seq, void *workspace,
                           cudaStream_t s) {
    mlp_bwd_body::Params p{Q, K, V, eta, W1_0, W2_0, gamma, beta, dZ, dW1_out, dW2_out,
                          dQ, dK, dV, deta, dW1_0, dW2_0, static_cast<float *>(workspace),
                          H, T, d, b, bf16, w0_per_seq};
    const size_t smem = sizeof(float) * mlp_bwd_body::smem_floats(d, b);
    cudaError_t e = cudaFuncSetAttribute(mlp_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    mlp_bwd_kernel<<<(unsigned)(B * H), kBwdThreads, smem, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch(s);
    mlp_bwd_sum_kernel<<<(unsigned)H, 256, 0, s>>>(static_cast<const float *>(workspace),
                                                   mlp_bwd_body::ws_floats_per_seq(T, d, b), B, H,
                                                   T, d, b, !w0_per_seq, dW1_0, dW2_0, dgamma,
                                                   dbeta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}

}  // namespace ttt
