// ttt_common.cuh -- internal declarations shared by the CUDA sources of libttt.
// Not part of the public ABI (that is include/ttt.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ttt {

constexpr float kLnEps = 1e-5f;  // torch nn.LayerNorm default, as in the pages' listing

// Problem description handed from the ABI layer to a launcher. Pointers are
// device pointers already validated by the ABI layer.
struct LinearArgs {
    const void *Q, *K, *V;
    const float *eta, *W0, *gamma, *beta;
    float *Z, *W_out;  // Z is bf16 [..][d] instead when z_bf16
    int B, H, T, d, b;
    bool bf16, ln, w0_per_seq, z_bf16;
};

struct MlpArgs {
    const void *Q, *K, *V;
    const float *eta, *W1_0, *W2_0, *gamma, *beta;
    float *Z, *W1_out, *W2_out;  // Z is bf16 instead when z_bf16
    int B, H, T, d, dh, b;
    bool bf16, w0_per_seq, z_bf16;
};

struct ChunkArgs {
    const void *Q, *K, *V;
    const float *eta, *W0;
    float *Z, *W_out;  // Z is bf16 instead when z_bf16
    int B, H, T, d, chunk;
    bool bf16, w0_per_seq, z_bf16;
    void *workspace;
    size_t workspace_bytes;
};

// TTT-Linear backward (outer gradients), fp32 CUDA cores.
struct LinearBwdArgs {
    const void *Q, *K, *V;
    const float *eta, *W0, *gamma, *beta, *dZ, *dW_out;
    float *dQ, *dK, *dV, *deta, *dW0, *dgamma, *dbeta;
    int B, H, T, d, b;
    bool bf16, ln, w0_per_seq;
    void *workspace;
};
bool linear_bwd_supported(int d, int b);
size_t linear_bwd_workspace_bytes(int B, int H, int T, int d, int b);
cudaError_t launch_linear_bwd(const LinearBwdArgs &a, cudaStream_t s);

// Output stores: Z as fp32, or rounded to nearest-even bf16 (TTT_F_Z_BF16).
// off is the element offset of the first value; vector forms need off a
// multiple of their width.
__device__ __forceinline__ void store_z1(float *Z, bool bf16, size_t off, float v) {
    if (bf16) reinterpret_cast<__nv_bfloat16 *>(Z)[off] = __float2bfloat16_rn(v);
    else Z[off] = v;
}
__device__ __forceinline__ void store_z2(float *Z, bool bf16, size_t off, float a, float b) {
    if (bf16) reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(Z) + off)[0] =
        __floats2bfloat162_rn(a, b);
    else *reinterpret_cast<float2 *>(Z + off) = make_float2(a, b);
}
__device__ __forceinline__ void store_z4(float *Z, bool bf16, size_t off, float a, float b, float c,
                                         float d) {
    if (bf16) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&lo);
        u.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(Z) + off) = u;
    } else {
        *reinterpret_cast<float4 *>(Z + off) = make_float4(a, b, c, d);
    }
}

// Launchers return cudaSuccess or the launch error.
cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t s);
cudaError_t launch_mlp_simt(const MlpArgs &a, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s);

// TTT-Linear tensor-core scan (bf16, d = 64, b = 16).
bool linear_tc_supported(int d, int b, bool bf16);
cudaError_t launch_linear_tc(const LinearArgs &a, cudaStream_t s, bool l2_keys = false);

// TTT-MLP warp-MMA scan (bf16, d = 64, hidden 256, b = 16; rows = B*H*T).
bool mlp_tc_supported(int d, int dh, int b, bool bf16, long long rows);
cudaError_t launch_mlp_tc(const MlpArgs &a, cudaStream_t s);
cudaError_t launch_mlp_umma(const MlpArgs &a, cudaStream_t s);

// Large-chunk tensor-core path (bf16, d = 128, chunk % 128 == 0).
bool chunk_tc_supported(int d, int chunk, bool bf16);
size_t chunk_tc_workspace_bytes(int B, int H, int T, int d, int chunk);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s);
cudaError_t launch_chunk_map_tc(const void *K, const void *V, const float *eta, float *M, float *N,
                                int B, int H, int T, int chunk, void *workspace, cudaStream_t s);

// Encodes a 2-D bf16 TMA descriptor (CUtensorMap, 128 bytes) over a
// row-major [rows][cols] tensor with a box of box_rows x box_cols elements and
// the 128-byte swizzle. Returns false if the driver rejects it.
bool encode_tmap_bf16_2d(void *map, const void *base, uint64_t cols, uint64_t rows,
                         uint32_t box_cols, uint32_t box_rows);

// Host-side count of kernel launches (ttt_launch_count); launchers call
// count_launch() after each successful launch. With per-kernel timing
// enabled (ttt_diag_kernel_timing) it also records an event on `s` after the
// launch; entry points call timing_begin(s) before their first launch.
void count_launch(int n = 1);
void count_launch(cudaStream_t s);
void timing_begin(cudaStream_t s);

// Device-side status word (bounded waits that ran out set it). Defined in
// ttt_api.cu; kernels get its address as an argument.
int *device_status_word();

__device__ __forceinline__ float load_elem(const void *p, size_t i, bool bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace ttt
