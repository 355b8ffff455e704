// Host run of the fp32 CUDA-core kernels of ttt_simt.cu (TTT-Linear, TTT-MLP,
// large chunk), for CPU tests of their arithmetic, indexing and
// synchronisation, through the stand-ins of cuda_host_shim.h. TEST CODE ONLY:
// the library never calls it, and it is no fallback for the GPU kernels.
#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_simt.cu"

// Dynamic shared memory of the one block that runs at a time (the kernels
// declare it with a block-scope extern in their own unnamed namespace).
namespace ttt {
namespace {
float sm[1 << 16];
}  // namespace
}  // namespace ttt

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
    run_blocks(B * H, [&] { ttt::linear_simt_kernel(a, l2_keys != 0, n_steps); });
    return 0;
}
