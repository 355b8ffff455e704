// ttt_gelu.cuh -- GELU and its derivative for the tensor-core MLP kernel.
//
// GELU(h) = h Phi(h) and GELU'(h) = Phi(h) + h phi(h), with Phi / phi the
// standard normal CDF / density (the exact, erf-based GELU of the TTT-MLP
// inner model). Both come from one exponential: with x = |h| / sqrt(2),
//   phi(h) = exp(-x^2) / sqrt(2 pi),
//   Phi(-|h|) = (1 - erf(x)) / 2,  erf from Abramowitz & Stegun, Handbook of
//   Mathematical Functions, formula 7.1.26 (Hastings' rational approximation:
//   1 - erf(x) = (a1 t + ... + a5 t^5) exp(-x^2), t = 1 / (1 + p x),
//   |error| <= 1.5e-7 for x >= 0),
// and Phi(|h|) = 1 - Phi(-|h|). The tail is formed directly, so Phi keeps its
// relative accuracy for negative h.
#pragma once

namespace ttt {

__device__ __forceinline__ float normal_cdf_and_pdf(float h, float &pdf) {
    constexpr float kRsqrt2 = 0.70710678118654752f, kInvSqrt2Pi = 0.39894228040143268f;
    constexpr float p = 0.3275911f, a1 = 0.254829592f, a2 = -0.284496736f, a3 = 1.421413741f,
                    a4 = -1.453152027f, a5 = 1.061405429f;
    const float x = fabsf(h) * kRsqrt2;
    const float t = __fdividef(1.f, fmaf(p, x, 1.f));
    const float e = __expf(-x * x);
    const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, a5, a4), a3), a2), a1);
    const float tail = 0.5f * poly * e;  // Phi(-|h|)
    pdf = e * kInvSqrt2Pi;
    return h >= 0.f ? 1.f - tail : tail;
}

__device__ __forceinline__ float gelu_and_prime(float h, float &prime) {
    float pdf;
    const float Phi = normal_cdf_and_pdf(h, pdf);
    prime = fmaf(h, pdf, Phi);
    return h * Phi;
}

__device__ __forceinline__ float gelu(float h) {
    float pdf;
    return h * normal_cdf_and_pdf(h, pdf);
}

}  // namespace ttt
