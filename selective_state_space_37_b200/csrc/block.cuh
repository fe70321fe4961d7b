// block.cuh -- the Mamba block's inner forward path around the scan (sm_100a).
//
// hidden → in_proj (x, z) → causal conv1d + SiLU (u) → selection projections
// (Δ's low-rank input, B, C) → Δ projection → selective scan (gate z) →
// out_proj.  The projections are plain dense GEMMs and go to cuBLAS (bf16 in
// and out, fp32 accumulation); this header holds the one kernel of the path
// that is not a GEMM or the scan: the standalone conv + SiLU that
// materialises u, which both the selection projections and the scan read.
#pragma once

#include "common.cuh"

namespace selscan {

constexpr int kConvThreads = 128;   // channels per block
constexpr int kConvSteps = 64;      // timesteps per thread

// u_t = silu(conv_b + Σ_{k=0}^{3} w[ch, k] x_{t-3+k}), x_{<0} = 0
// ("Understanding Mamba and Selective State Space Models (SSMs)" §3.3).
// One thread walks kConvSteps timesteps of one channel with the three
// previous inputs in registers, so every x is read once per window.
template <typename IO>
__global__ void __launch_bounds__(kConvThreads)
ss_conv_silu_kernel(const IO* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
                    IO* __restrict__ u, int64_t L, int64_t d) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int64_t ch = static_cast<int64_t>(blockIdx.x) * kConvThreads + threadIdx.x;
    if (ch >= d) return;
    const int64_t b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvSteps;
    if (t0 >= L) return;
    const int64_t t1 = (t0 + kConvSteps < L) ? t0 + kConvSteps : L;
    const float4 wv = *reinterpret_cast<const float4*>(w + ch * 4);
    const float cb = bias ? bias[ch] : 0.0f;
    const IO* xs = x + b * L * d + ch;
    IO* us = u + b * L * d + ch;
    float s0 = t0 >= 3 ? to_f32(xs[(t0 - 3) * d]) : 0.0f;
    float s1 = t0 >= 2 ? to_f32(xs[(t0 - 2) * d]) : 0.0f;
    float s2 = t0 >= 1 ? to_f32(xs[(t0 - 1) * d]) : 0.0f;
    for (int64_t t = t0; t < t1; ++t) {
        const float xv = to_f32(xs[t * d]);
        const float c = fmaf(wv.w, xv, fmaf(wv.z, s2, fmaf(wv.y, s1, fmaf(wv.x, s0, cb))));
        us[t * d] = from_f32<IO>(FAST ? silu_tanh(c) : silu_accurate(c));
        s0 = s1;
        s1 = s2;
        s2 = xv;
    }
}

}  // namespace selscan
