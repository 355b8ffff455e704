// Host run of the TTT-MLP backward kernel body (ttt_mlp_bwd_body.inc), for the
// CPU test of its arithmetic, indexing and barrier placement: each sequence
// runs as one "block" of nt OS threads, one per CUDA thread, with a
// std::barrier standing for every __syncthreads(). TEST CODE ONLY: the
// library never calls it, and it is no fallback for the GPU kernel.
#include <barrier>
#include <cstring>
#include <math.h>
#include <memory>
#include <thread>
#include <vector>

#define TTT_HD
#define TTT_HD_SIZES
#include "../../test_sequence_layers_layer_b200/csrc/ttt_mlp_bwd_body.inc"

namespace {

struct HostCtx {
    int tid, nt;
    float *sm;
    std::barrier<> *bar;
    std::unique_ptr<std::barrier<>> *warp_bar;  // one barrier of 32 per warp
    float *xbuf;               // [warps][32] exchange buffer
    void sync() { bar->arrive_and_wait(); }
    // sum over the 32 lanes of the calling warp (all lanes call it)
    float warp_sum(float v) {
        const int w = tid / 32, l = tid % 32;
        xbuf[w * 32 + l] = v;
        warp_bar[w]->arrive_and_wait();
        float s = 0.f;
        for (int k = 0; k < 32; ++k) s += xbuf[w * 32 + k];
        warp_bar[w]->arrive_and_wait();
        return s;
    }
};

}  // namespace

extern "C" int ttt_mlp_bwd_host_run(const void *Q, const void *K, const void *V, const float *eta,
                                    const float *W1_0, const float *W2_0, const float *gamma,
                                    const float *beta, const float *dZ, const float *dW1_out,
                                    const float *dW2_out, float *dQ, float *dK, float *dV,
                                    float *deta, float *dW1_0, float *dW2_0, float *dgamma,
                                    float *dbeta, int B, int H, int T, int d, int b, int bf16,
                                    int w0_per_seq, int nt) {
    if (T % b || nt < 1) return -1;
    const size_t per = mlp_bwd_body::ws_floats_per_seq(T, d, b);
    std::vector<float> ws(per * (size_t)B * H, 0.f);
    std::vector<float> sm(mlp_bwd_body::smem_floats(d, b), 0.f);
    mlp_bwd_body::Params p{Q, K, V, eta, W1_0, W2_0, gamma, beta, dZ, dW1_out, dW2_out,
                          dQ, dK, dV, deta, dW1_0, dW2_0, ws.data(), H, T, d, b, bf16 != 0,
                          w0_per_seq != 0};
    if (nt % 32) return -1;
    std::vector<float> xbuf(nt);
    for (int seq = 0; seq < B * H; ++seq) {
        std::barrier<> bar(nt);
        std::vector<std::unique_ptr<std::barrier<>>> wbars;
        for (int w = 0; w < nt / 32; ++w) wbars.push_back(std::make_unique<std::barrier<>>(32));
        std::vector<std::thread> th;
        for (int t = 0; t < nt; ++t)
            th.emplace_back([&, t] {
                HostCtx cx{t, nt, sm.data(), &bar, wbars.data(), xbuf.data()};
                mlp_bwd_body::run_sequence(cx, p, seq);
            });
        for (auto &x : th) x.join();
    }
    // the batch sums the GPU's second kernel makes
    const size_t dF = (size_t)d * 4 * d;
    for (int h = 0; h < H; ++h) {
        for (size_t e = 0; e < dF; ++e) {
            float a1 = 0.f, a2 = 0.f;
            for (int bb = 0; bb < B; ++bb) {
                auto w = mlp_bwd_body::ws_view(ws.data() + (size_t)(bb * H + h) * per, T, d, b);
                a1 += w.dW1[e];
                a2 += w.dW2[e];
            }
            if (!w0_per_seq) {
                dW1_0[(size_t)h * dF + e] = a1;
                dW2_0[(size_t)h * dF + e] = a2;
            }
        }
        for (int c = 0; c < d; ++c) {
            float g = 0.f, be = 0.f;
            for (int bb = 0; bb < B; ++bb) {
                auto w = mlp_bwd_body::ws_view(ws.data() + (size_t)(bb * H + h) * per, T, d, b);
                g += w.dg[c];
                be += w.db[c];
            }
            dgamma[(size_t)h * d + c] = g;
            dbeta[(size_t)h * d + c] = be;
        }
    }
    return 0;
}
