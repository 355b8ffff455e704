// Host run of the affine-map kernels of ttt_affine.cu (the identity fill and
// the fold of segment maps), for CPU tests, through the stand-ins of
// cuda_host_shim.h. TEST CODE ONLY: the library never calls it.
#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_affine.cu"

namespace ttt {
namespace {
float smem[1 << 16];  // the fold kernel's dynamic shared memory
}  // namespace
}  // namespace ttt

extern "C" int ttt_affine_prefix_host_run(const float *M, const float *N, const float *W0,
                                          float *W_in, float *W_end, int S, int H, int nseg,
                                          int d, long long seq_stride, long long seg_stride,
                                          int w0_per_seq) {
    const ttt::PrefixArgs a{M, N, W0, W_in, W_end, H, nseg, seq_stride, seg_stride,
                            w0_per_seq != 0};
    if (d == 64)
        run_blocks(S, [&] { ttt::affine_prefix_kernel<64>(a); });
    else if (d == 128)
        run_blocks(S, [&] { ttt::affine_prefix_kernel<128>(a); });
    else
        return -1;
    return 0;
}

extern "C" int ttt_affine_eye_host_run(float *W, int S, int d) {
    run_blocks(3, [&] { ttt::affine_eye_kernel(W, (size_t)S * d * d, d); });
    return 0;
}
