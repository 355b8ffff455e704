// Host run of the TTT-MLP decode kernel (ttt_mlp_decode.cu), for CPU tests,
// through the stand-ins of cuda_host_shim.h. TEST CODE ONLY.
#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_mlp_decode.cu"

namespace ttt {
namespace {
float msm[1024];  // the kernel's dynamic shared memory
}  // namespace
}  // namespace ttt

extern "C" int ttt_mlp_decode_host_run(const void *q, const void *k, const void *v,
                                       const float *eta, const float *gamma, const float *beta,
                                       float *W1, float *W2, float *z, int B, int H, int bf16) {
    const ttt::MlpDecodeArgs a{q, k, v, eta, gamma, beta, W1, W2, z, H, bf16 != 0, false};
    run_blocks(B * H, [&] { ttt::mlp_decode_kernel(a); }, ttt::kMThreads);
    return 0;
}

// n tokens per sequence in one call (q, k, v [S][n][64], eta [S][n], z [S][n][64]).
extern "C" int ttt_mlp_decode_tokens_host_run(const void *q, const void *k, const void *v,
                                              const float *eta, const float *gamma,
                                              const float *beta, float *W1, float *W2, float *z,
                                              int B, int H, int n, int bf16) {
    const ttt::MlpDecodeArgs a{q, k, v, eta, gamma, beta, W1, W2, z, H, bf16 != 0, false, n};
    run_blocks(B * H, [&] { ttt::mlp_decode_kernel(a); }, ttt::kMThreads);
    return 0;
}
