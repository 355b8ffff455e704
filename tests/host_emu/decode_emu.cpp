// Host run of the TTT-Linear decode kernel (ttt_decode.cu), for CPU tests,
// through the stand-ins of cuda_host_shim.h. TEST CODE ONLY.
#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_decode.cu"

namespace ttt {
namespace {
float dsm[1024];  // the decode kernel's dynamic shared memory
}  // namespace
}  // namespace ttt

extern "C" int ttt_linear_decode_host_run(const void *q, const void *k, const void *v,
                                          const float *eta, const float *gamma,
                                          const float *beta, float *W, float *z, int B, int H,
                                          int bf16, int ln, int l2_keys) {
    const ttt::DecodeArgs a{q, k, v, eta, gamma, beta, W, z, H, bf16 != 0, ln != 0, false,
                            l2_keys != 0};
    run_blocks(B * H, [&] { ttt::linear_decode_kernel(a); }, ttt::kDecThreads);
    return 0;
}

// n tokens per sequence in one call (q, k, v [S][n][64], eta [S][n], z [S][n][64]).
extern "C" int ttt_linear_decode_tokens_host_run(const void *q, const void *k, const void *v,
                                                 const float *eta, const float *gamma,
                                                 const float *beta, float *W, float *z, int B,
                                                 int H, int n, int bf16, int ln, int l2_keys) {
    const ttt::DecodeArgs a{q, k, v, eta, gamma, beta, W, z, H, bf16 != 0, ln != 0, false,
                            l2_keys != 0, n};
    run_blocks(B * H, [&] { ttt::linear_decode_kernel(a); }, ttt::kDecThreads);
    return 0;
}
