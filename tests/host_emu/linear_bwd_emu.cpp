// Host run of the TTT-Linear backward kernels of ttt_linear_bwd.cu (the
// per-sequence backward and the batch sums), for CPU tests, through the
// stand-ins of cuda_host_shim.h; the kernel arguments are set up as the
// library's launcher sets them up. TEST CODE ONLY: the library never calls it.
#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_linear_bwd.cu"

namespace ttt {
namespace {
float smem_f[1 << 16];  // the backward kernel's dynamic shared memory
}  // namespace
}  // namespace ttt

template <typename TIn>
static void run_kernel(const ttt::BwdArgs &k, int S, int d) {
    if (d == 16) run_blocks(S, [&] { ttt::linear_bwd_kernel<TIn, 16>(k); });
    else if (d == 32) run_blocks(S, [&] { ttt::linear_bwd_kernel<TIn, 32>(k); });
    else run_blocks(S, [&] { ttt::linear_bwd_kernel<TIn, 64>(k); });
}

extern "C" int ttt_linear_bwd_host_run(const void *Q, const void *K, const void *V,
                                       const float *eta, const float *W0, const float *gamma,
                                       const float *beta, const float *dZ, const float *dW_out,
                                       float *dQ, float *dK, float *dV, float *deta, float *dW0,
                                       float *dgamma, float *dbeta, int B, int H, int T, int d,
                                       int b, int bf16, int ln, int w0_per_seq) {
    if (!ttt::linear_bwd_supported(d, b) || T % b) return -1;
    if (ttt::bwd_smem_floats(d, b) > (size_t)(1 << 16)) return -1;
    const size_t S = (size_t)B * H, M = (size_t)(T / b), dd = (size_t)d * d;
    std::vector<float> ws(ttt::linear_bwd_workspace_bytes(B, H, T, d, b) / 4);
    float *w = ws.data();
    const ttt::BwdArgs k{Q, K, V, eta, W0, gamma, beta, dZ, dW_out, dQ, dK, dV, deta,
                         w, w0_per_seq ? dW0 : w + S * M * dd,
                         w + S * M * dd + S * dd, w + S * M * dd + S * dd + S * d,
                         H, T, d, b, ln != 0, w0_per_seq != 0};
    if (bf16) run_kernel<__nv_bfloat16>(k, (int)S, d);
    else run_kernel<float>(k, (int)S, d);
    // the batch sums: a thread per element, grid (elements, H), as launched
    if (!w0_per_seq)
        run_grid(((int)dd + 255) / 256, H, [&] { ttt::sum_over_batch_kernel(k.dW0s, dW0, B, H, (int)dd); }, 256);
    if (ln) {
        run_grid((d + 63) / 64, H, [&] { ttt::sum_over_batch_kernel(k.dgs, dgamma, B, H, d); }, 64);
        run_grid((d + 63) / 64, H, [&] { ttt::sum_over_batch_kernel(k.dbs, dbeta, B, H, d); }, 64);
    }
    return 0;
}
