// Host stand-ins for the CUDA built-ins used by the library's fp32 kernels, so
// that their sources compile as C++ and run on the CPU in tests: each block
// runs as OS threads (one per CUDA thread), __syncthreads() is a block-wide
// std::barrier, and warp shuffles and __syncwarp() go through per-warp
// exchange buffers and barriers. TEST CODE ONLY.
//
// Limits: only `extern __shared__` (dynamic) shared memory works -- the
// including harness defines the array once, in the kernel's namespace; a
// static `__shared__` array inside a kernel would become a private array per
// OS thread, so kernels that declare one (the large-chunk backward's Gram
// kernel) are not run this way. Warp shuffles must be called by all 32 lanes.
#pragma once
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

// Runs fn() as every thread of an nx x ny x nz grid of blocks of nt threads
// (a multiple of 32, at most 256), one block at a time.
template <class Fn>
static void run_grid(int nx, int ny, Fn fn, int nt = emu::kMaxThreads, int nz = 1) {
    emu::nthreads = nt;
    blockDim = {(unsigned)nt, 1, 1};
    gridDim = {(unsigned)nx, (unsigned)ny, (unsigned)nz};
    emu::block_bar = std::make_unique<std::barrier<>>(nt);
    for (auto &w : emu::warp_bar) w = std::make_unique<std::barrier<>>(32);
    for (int bz = 0; bz < nz; ++bz)
        for (int by = 0; by < ny; ++by)
            for (int bx = 0; bx < nx; ++bx) {
                blockIdx = {(unsigned)bx, (unsigned)by, (unsigned)bz};
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

// Runs fn() as every thread of nblocks blocks (a one-dimensional grid).
template <class Fn>
static void run_blocks(int nblocks, Fn fn, int nt = emu::kMaxThreads) {
    run_grid(nblocks, 1, fn, nt);
}

