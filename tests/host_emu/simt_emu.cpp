// Host run of the fp32 CUDA-core TTT-Linear kernel (ttt_simt.cu), for CPU
// tests of its arithmetic, indexing and synchronisation. The kernel source is
// compiled as C++ with the CUDA qualifiers emptied; each block runs as 256 OS
// threads (one per CUDA thread), __syncthreads() is a block-wide
// std::barrier, and the warp shuffles and __syncwarp() go through per-warp
// exchange buffers and barriers. TEST CODE ONLY: the library never calls it,
// and it is no fallback for the GPU kernels.
#include <barrier>
#include <math.h>
#include <memory>
#include <thread>
#include <vector>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#undef __global__
#undef __device__
#undef __shared__
#undef __forceinline__
#undef __launch_bounds__
#define __global__
#define __device__
#define __shared__
#define __forceinline__ inline
#define __launch_bounds__(...)

namespace emu {
constexpr int kMaxThreads = 256, kWarps = kMaxThreads / 32;
thread_local int tid = 0;
int nthreads = kMaxThreads;
std::unique_ptr<std::barrier<>> block_bar;
std::unique_ptr<std::barrier<>> warp_bar[kWarps];
float xbuf[kWarps][32];
}  // namespace emu

struct EmuIdx {
    unsigned x, y, z;
};
thread_local EmuIdx threadIdx;
EmuIdx blockIdx, blockDim, gridDim;

inline void __syncthreads() { emu::block_bar->arrive_and_wait(); }
inline void __syncwarp(unsigned = 0xffffffffu) { emu::warp_bar[emu::tid / 32]->arrive_and_wait(); }
inline float __shfl_xor_sync(unsigned, float v, int m) {
    const int w = emu::tid / 32, l = emu::tid % 32;
    emu::xbuf[w][l] = v;
    emu::warp_bar[w]->arrive_and_wait();
    const float r = emu::xbuf[w][l ^ m];
    emu::warp_bar[w]->arrive_and_wait();
    return r;
}
inline float rsqrtf(float x) { return 1.f / sqrtf(x); }

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_simt.cu"

// Dynamic shared memory of the one block that runs at a time (the kernels
// declare it with a block-scope extern in their own unnamed namespace).
namespace ttt {
namespace {
float sm[1 << 16];
}  // namespace
}  // namespace ttt

// Runs fn() as every thread of nblocks blocks of 256 threads, one block at a time.
template <class Fn>
static void run_blocks(int nblocks, Fn fn) {
    const int nt = emu::kMaxThreads;
    emu::nthreads = nt;
    blockDim = {(unsigned)nt, 1, 1};
    gridDim = {(unsigned)nblocks, 1, 1};
    emu::block_bar = std::make_unique<std::barrier<>>(nt);
    for (auto &w : emu::warp_bar) w = std::make_unique<std::barrier<>>(32);
    for (int blk = 0; blk < nblocks; ++blk) {
        blockIdx = {(unsigned)blk, 0, 0};
        std::vector<std::thread> th;
        for (int t = 0; t < nt; ++t)
            th.emplace_back([&, t] {
                emu::tid = t;
                threadIdx = {(unsigned)t, 0, 0};
                fn();
            });
        for (auto &x : th) x.join();
    }
}

extern "C" int ttt_mlp_simt_host_run(const void *Q, const void *K, const void *V, const float *eta,
                                     const float *W1, const float *W2, const float *gamma,
                                     const float *beta, float *Z, float *W1_out, float *W2_out,
                                     int B, int H, int T, int d, int dh, int b) {
    ttt::MlpArgs a{Q, K, V, eta, W1, W2, gamma, beta, Z, W1_out, W2_out, B, H, T, d, dh, b,
                   false, false, false};
    run_blocks(B * H, [&] { ttt::mlp_simt_kernel(a); });
    return 0;
}

extern "C" int ttt_chunk_simt_host_run(const void *Q, const void *K, const void *V,
                                       const float *eta, const float *W0, float *Z, float *W_out,
                                       int B, int H, int T, int d, int chunk) {
    ttt::ChunkArgs a{Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, false, false, false,
                     nullptr, 0};
    run_blocks(B * H, [&] { ttt::chunk_simt_kernel(a); });
    return 0;
}

extern "C" int ttt_linear_simt_host_run(const void *Q, const void *K, const void *V,
                                        const float *eta, const float *W0, const float *gamma,
                                        const float *beta, float *Z, float *W_out, int B, int H,
                                        int T, int d, int b, int bf16, int ln, int w0_per_seq,
                                        int z_bf16, int l2_keys, int n_steps) {
    ttt::LinearArgs a{Q, K, V, eta, W0, gamma, beta, Z, W_out, B, H, T, d, b, bf16 != 0,
                      ln != 0, w0_per_seq != 0, z_bf16 != 0};
    const int nt = emu::kMaxThreads;
    emu::nthreads = nt;
    blockDim = {(unsigned)nt, 1, 1};
    gridDim = {(unsigned)(B * H), 1, 1};
    emu::block_bar = std::make_unique<std::barrier<>>(nt);
    for (auto &w : emu::warp_bar) w = std::make_unique<std::barrier<>>(32);
    for (int seq = 0; seq < B * H; ++seq) {
        blockIdx = {(unsigned)seq, 0, 0};
        std::vector<std::thread> th;
        for (int t = 0; t < nt; ++t)
            th.emplace_back([&, t] {
                emu::tid = t;
                threadIdx = {(unsigned)t, 0, 0};
                ttt::linear_simt_kernel(a, l2_keys != 0, n_steps);
            });
        for (auto &x : th) x.join();
    }
    return 0;
}
