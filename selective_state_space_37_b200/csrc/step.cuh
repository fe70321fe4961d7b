// step.cuh -- single-token decode step (sm_100a).
//
// The streaming form of the selective SSM: each (batch, channel) state row of
// kN fp32 values is read, advanced by one token with the same equations as
// the forward scan ("Understanding Mamba and Selective State Space Models",
// §2.2 first cut, §3.1), and written back in place; y is produced for the
// token.  The kernel is bound by HBM traffic on the state (read + write), so
// the state moves in fully coalesced 16-byte accesses: four consecutive
// threads share one channel, each owning four consecutive states, and the
// readout Σ_n C_n h_n is finished with two butterfly shuffles.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace selscan {

constexpr int kStepThreads = 256;

struct StepParams {
    float* state;
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    void* y;
    const float* bias;
    int64_t channels;   // batch * d
    int d;
    int softplus;
};

template <typename IO>
__device__ __forceinline__ void load4(const IO* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xffff0000u);
}

template <typename IO>
__global__ void __launch_bounds__(kStepThreads) ss_step_kernel(const __grid_constant__ StepParams p) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * kStepThreads + threadIdx.x;
    const int64_t chan = gid >> 2;            // (b * d + ch)
    const int q = static_cast<int>(gid & 3);  // states 4q .. 4q+3
    const bool valid = chan < p.channels;
    const int64_t cs = valid ? chan : 0;
    const int64_t b = cs / p.d;
    const int ch = static_cast<int>(cs % p.d);

    float4* srow = reinterpret_cast<float4*>(p.state + cs * 16) + q;
    float4 h4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float Bv[4], Cv[4], Av[4];
    float uu = 0.f, xr = 0.f, zz = 0.f, Dv = 0.f, bv = 0.f;
    if (valid) {
        h4 = *srow;
        load4<IO>(static_cast<const IO*>(p.B) + b * 16 + 4 * q, Bv);
        load4<IO>(static_cast<const IO*>(p.C) + b * 16 + 4 * q, Cv);
        load4<float>(p.A + static_cast<int64_t>(ch) * 16 + 4 * q, Av);
        uu = to_f32(static_cast<const IO*>(p.u)[cs]);
        xr = to_f32(static_cast<const IO*>(p.delta)[cs]);
        if (p.z) zz = to_f32(static_cast<const IO*>(p.z)[cs]);
        if (p.D) Dv = __ldg(p.D + ch);
        if (p.bias) bv = __ldg(p.bias + ch);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) { Bv[k] = 0.f; Cv[k] = 0.f; Av[k] = -1.f; }
    }
    float dl = xr + bv;
    if (p.softplus) dl = FAST ? softplus_fast(dl) : softplus_accurate(dl);
    const float du = dl * uu;
    float hv[4] = {h4.x, h4.y, h4.z, h4.w};
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float a = FAST ? ex2_approx(dl * (Av[k] * kLog2e)) : expf(dl * Av[k]);
        hv[k] = fmaf(a, hv[k], du * Bv[k]);
        acc = fmaf(Cv[k], hv[k], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (!valid) return;
    *srow = make_float4(hv[0], hv[1], hv[2], hv[3]);
    if (q == 0) {
        float yv = fmaf(Dv, uu, acc);
        if (p.z) yv *= FAST ? silu_fast(zz) : silu_accurate(zz);
        static_cast<IO*>(p.y)[cs] = from_f32<IO>(yv);
    }
}

}  // namespace selscan
