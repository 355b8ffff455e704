// Host run of the large-chunk backward's fp32 scan and per-token kernels of
// ttt_chunk_bwd.cu (cb_scan_kernel, cb_tok_kernel, cb_sum_over_batch_kernel)
// for CPU tests, through the stand-ins of cuda_host_shim.h, from given
// per-chunk Gram products [A_c | B_c | D_c] (row-major fp32, as cb_gram_kernel
// writes them; that kernel declares static shared arrays, which the stand-ins
// do not support). The grids and arguments are those of the library's
// launcher. TEST CODE ONLY: the library never calls it.
#include <cstring>

#include "cuda_host_shim.h"

#define TTT_HOST_RUN
#include "../../test_sequence_layers_layer_b200/csrc/ttt_chunk_bwd.cu"

namespace ttt {
namespace {
float As[1 << 16];  // cb_scan_kernel's dynamic shared memory
float sm[1 << 16];  // cb_tok_kernel's
}  // namespace
}  // namespace ttt

template <typename TIn, int D>
static void run_typed(const void *K, const void *V, const float *eta, const float *dZ,
                      const float *W0, const float *dW_out, float *dQ, float *dK, float *dV,
                      float *deta, float *dW0, int B, int H, int T, int C, bool w0_per_seq,
                      const ttt::WsView &w) {
    const int NC = T / C, S = B * H, nch = S * NC;
    float *dW0_seq = w0_per_seq ? dW0 : w.dW0s;
    run_grid(S, 2, [&] { ttt::cb_scan_kernel<D>(W0, dW_out, H, NC, w0_per_seq, w, dW0_seq); },
             ttt::kT, D / ttt::scan_cols(D));
    run_blocks(nch, [&] {
        ttt::cb_tok_kernel<TIn, D>(static_cast<const TIn *>(K), static_cast<const TIn *>(V), eta,
                                   dZ, T, C, w, dQ, dK, dV, deta);
    }, ttt::kT);
    if (!w0_per_seq)
        run_grid((D * D + 255) / 256, H, [&] { ttt::cb_sum_over_batch_kernel(w.dW0s, dW0, B, H, D * D); },
                 256);
}

extern "C" int ttt_chunk_bwd_scan_tok_host_run(const void *K, const void *V, const float *eta,
                                               const float *dZ, const float *W0, const float *dW_out,
                                               const float *gram, float *dQ, float *dK, float *dV,
                                               float *deta, float *dW0, int B, int H, int T, int d,
                                               int chunk, int bf16, int w0_per_seq) {
    if (!ttt::chunk_bwd_supported(d, chunk) || T % chunk) return -1;
    if (ttt::tok_smem_bytes(d) > sizeof(ttt::sm)) return -1;
    const size_t S = (size_t)B * H, nch = S * (T / chunk), dd = (size_t)d * d;
    std::vector<float> ws(ttt::chunk_bwd_workspace_bytes(B, H, T, d, chunk) / 4);
    const ttt::WsView w = ttt::ws_view(ws.data(), nch, S, d);
    std::memcpy(w.gram, gram, sizeof(float) * 3 * nch * dd);
    const bool ps = w0_per_seq != 0;
    if (d == 64) {
        if (bf16) run_typed<__nv_bfloat16, 64>(K, V, eta, dZ, W0, dW_out, dQ, dK, dV, deta, dW0, B, H, T, chunk, ps, w);
        else run_typed<float, 64>(K, V, eta, dZ, W0, dW_out, dQ, dK, dV, deta, dW0, B, H, T, chunk, ps, w);
    } else {
        if (bf16) run_typed<__nv_bfloat16, 128>(K, V, eta, dZ, W0, dW_out, dQ, dK, dV, deta, dW0, B, H, T, chunk, ps, w);
        else run_typed<float, 128>(K, V, eta, dZ, W0, dW_out, dQ, dK, dV, deta, dW0, B, H, T, chunk, ps, w);
    }
    return 0;
}
