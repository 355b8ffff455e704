// ttt_affine.cu -- the affine-map kernels of the sequence-parallel large-chunk
// forward.
//
// Large-chunk TTT ("Test-Time Training Done Right", abstract) updates the
// fast weight once per chunk by a gradient step on the chunk's eta-weighted
// reconstruction loss; expanded, that step is affine in the weight:
//   W_{c+1} = (I - A_c) W_c + B_c,  A_c = K_c^T diag(eta) K_c,  B_c = K_c^T diag(eta) V_c.
// A run of chunks (a segment of the sequence) therefore maps its starting
// weight to its final one by W -> M W + N. Given every segment's (M_j, N_j),
// the starting weight of segment j is the fold
//   W_in[0] = W0,  W_in[j+1] = M_j W_in[j] + N_j,
// after which the segments' forwards are independent of one another.
//
//   affine_eye_kernel     W[s] = I for every sequence (the starting weight from
//                         which a forward with V = 0 returns M)
//   affine_prefix_kernel  the fold, one block per sequence, the weight held in
//                         shared memory and M_j staged beside it; fp32 FMA
#include "../../include/ttt.h"
#include "ttt_common.cuh"

namespace ttt {
namespace {

constexpr int kPrefixThreads = 256;  // a 16 x 16 grid of threads

__global__ void affine_eye_kernel(float *W, size_t total, int d) {
    const size_t dd = (size_t)d * d;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i % dd;
        W[i] = (e / d == e % d) ? 1.f : 0.f;
    }
}

struct PrefixArgs {
    const float *M, *N, *W0;
    float *W_in, *W_end;
    int H, nseg;
    long long seq_stride, seg_stride;  // in floats, shared by M, N and W_in
    bool w0_per_seq;
};

constexpr size_t prefix_smem_bytes(int D) {
    return sizeof(float) * ((size_t)D * (D + 1) + (size_t)D * D);
}

// Thread (ty, tx) of the 16 x 16 grid owns rows ty + 16 i (i < D/16) and the
// column quads 4 tx + 64 q (q < D/64) of every D x D product. M_j sits in
// shared memory with row stride D + 1, so the two rows that a warp reads at
// one k fall in different banks; the weight keeps stride D and is read as
// float4 along a row (16 consecutive quads per half warp).
template <int D>
__global__ void __launch_bounds__(kPrefixThreads) affine_prefix_kernel(PrefixArgs a) {
    constexpr int TL = D / 16, NQ = TL / 4, MS = D + 1, DQ = D * D / 4;
    static_assert(D == 64 || D == 128, "D");
    extern __shared__ float smem[];
    float *Ms = smem;           // M_j, row stride D + 1
    float *Wc = smem + D * MS;  // the current weight W_in[j], row stride D
    const int s = blockIdx.x, tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const size_t off = (size_t)s * (size_t)a.seq_stride;
    const float4 *w0 =
        reinterpret_cast<const float4 *>(a.W0 + (size_t)(a.w0_per_seq ? s : s % a.H) * D * D);
    float4 *win0 = reinterpret_cast<float4 *>(a.W_in + off);
    for (int i = tid; i < DQ; i += kPrefixThreads) {
        const float4 v = w0[i];
        reinterpret_cast<float4 *>(Wc)[i] = v;
        win0[i] = v;
    }
    const int steps = a.W_end ? a.nseg : a.nseg - 1;
    for (int j = 0; j < steps; ++j) {
        const float4 *Mj = reinterpret_cast<const float4 *>(a.M + off + (size_t)j * a.seg_stride);
        const float *Nj = a.N + off + (size_t)j * a.seg_stride;
        for (int i = tid; i < DQ; i += kPrefixThreads) {
            const float4 v = Mj[i];
            float *p = Ms + (4 * i / D) * MS + (4 * i) % D;
            p[0] = v.x;
            p[1] = v.y;
            p[2] = v.z;
            p[3] = v.w;
        }
        __syncthreads();  // Ms staged; Wc holds W_in[j]
        float acc[TL][TL];
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int c = 0; c < TL; ++c) acc[i][c] = 0.f;
#pragma unroll 4
        for (int k = 0; k < D; ++k) {
            float x[TL];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float4 w = *reinterpret_cast<const float4 *>(Wc + k * D + 4 * tx + 64 * q);
                x[4 * q] = w.x;
                x[4 * q + 1] = w.y;
                x[4 * q + 2] = w.z;
                x[4 * q + 3] = w.w;
            }
#pragma unroll
            for (int i = 0; i < TL; ++i) {
                const float m = Ms[(ty + 16 * i) * MS + k];
#pragma unroll
                for (int c = 0; c < TL; ++c) acc[i][c] = fmaf(m, x[c], acc[i][c]);
            }
        }
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float4 n =
                    *reinterpret_cast<const float4 *>(Nj + (ty + 16 * i) * D + 4 * tx + 64 * q);
                acc[i][4 * q] += n.x;
                acc[i][4 * q + 1] += n.y;
                acc[i][4 * q + 2] += n.z;
                acc[i][4 * q + 3] += n.w;
            }
        __syncthreads();  // every read of Ms and Wc for this step is done
        float *out = j + 1 < a.nseg ? a.W_in + off + (size_t)(j + 1) * a.seg_stride
                                    : a.W_end + (size_t)s * D * D;
#pragma unroll
        for (int i = 0; i < TL; ++i)
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const int e = (ty + 16 * i) * D + 4 * tx + 64 * q;
                const float4 v = make_float4(acc[i][4 * q], acc[i][4 * q + 1], acc[i][4 * q + 2],
                                             acc[i][4 * q + 3]);
                *reinterpret_cast<float4 *>(Wc + e) = v;
                *reinterpret_cast<float4 *>(out + e) = v;
            }
        // the next step's staging writes only Ms; its barrier orders these
        // writes of Wc before the next reads
    }
}

#ifndef TTT_HOST_RUN  // launch code (a host build of the kernels for tests leaves it out)
template <int D>
cudaError_t launch_prefix(const PrefixArgs &a, int S, cudaStream_t s) {
    constexpr size_t smem = prefix_smem_bytes(D);
    cudaError_t e = cudaFuncSetAttribute(affine_prefix_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    affine_prefix_kernel<D><<<(unsigned)S, kPrefixThreads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch(s);
    return cudaSuccess;
}
#endif  // TTT_HOST_RUN

}  // namespace

#ifndef TTT_HOST_RUN
cudaError_t launch_affine_eye(float *W, int S, int d, cudaStream_t s) {
    const size_t total = (size_t)S * d * d;
    const size_t blocks = (total + 255) / 256;
    affine_eye_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, s>>>(W, total, d);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch(s);
    return e;
}

cudaError_t launch_affine_prefix(const float *M, const float *N, const float *W0, float *W_in,
                                 float *W_end, int S, int H, int nseg, int d, long long seq_stride,
                                 long long seg_stride, bool w0_per_seq, cudaStream_t s) {
    const PrefixArgs a{M, N, W0, W_in, W_end, H, nseg, seq_stride, seg_stride, w0_per_seq};
    return d == 64 ? launch_prefix<64>(a, S, s) : launch_prefix<128>(a, S, s);
}

#endif  // TTT_HOST_RUN

}  // namespace ttt
