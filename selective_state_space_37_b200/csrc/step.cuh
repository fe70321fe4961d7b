// step.cuh -- single-token decode step (sm_100a).
//
// The streaming form of the selective SSM: each (batch, channel) state row of
// kN fp32 values is read, advanced by one token with the same equations as
// the forward scan ("Understanding Mamba and Selective State Space Models",
// §2.2 first cut, §3.1), and written back in place; y is produced for the
// token.  The kernel is bound by HBM traffic on the state (read + write), so
// the state moves in fully coalesced 16-byte accesses: four consecutive
// threads share one channel, each owning four consecutive states, and the
// readout Σ_n C_n h_n is finished with two butterfly shuffles.  A block
// covers kStepChanPerBlock channels of one batch row, so a thread finds its
// (batch, channel) without integer division.
// With the conv prologue (CONV) the token's input is x and u = silu(cb +
// w0 s0 + w1 s1 + w2 s2 + w3 x) over the conv state s (the previous three x
// of the channel, fp32, oldest first), which then shifts in x ("Understanding
// Mamba and Selective State Space Models (SSMs)" §3.3, causal conv of width 4).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace selscan {

constexpr int kStepThreads = 256;
constexpr int kStepChanPerBlock = kStepThreads / 4;   // 64 channels, four threads each

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
    float* conv_state;     // [batch, d, 3] fp32, read and shifted (conv prologue only)
    const float* conv_w;   // [d, 4]
    const float* conv_b;   // [d] or null
    int64_t batch;
    int d;
    int softplus;
};

// x[b, L-3 .. L-1, ch] of a sequence as fp32 (zero before its start): the conv
// state a decode step continues from after a forward pass with the prologue.
template <typename IO>
__global__ void ss_conv_tail_kernel(const IO* __restrict__ x, float* __restrict__ conv_state, int64_t batch,
                                    int64_t L, int64_t d) {
    const int64_t n = batch * d;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = i / d, ch = i % d;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int64_t t = L - 3 + k;
            conv_state[i * 3 + k] = t >= 0 ? to_f32(x[(b * L + t) * d + ch]) : 0.0f;
        }
    }
}

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

// Grid: x over blocks of kStepChanPerBlock channels of one batch row,
// y over batch rows (strided when batch exceeds the grid's y extent).
template <typename IO, bool CONV>
__global__ void __launch_bounds__(kStepThreads) ss_step_kernel(const __grid_constant__ StepParams p) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int q = threadIdx.x & 3;   // states 4q .. 4q+3
    const int ch = blockIdx.x * kStepChanPerBlock + (threadIdx.x >> 2);
    const bool valid = ch < p.d;
    const int chs = valid ? ch : 0;
    float Av[4];
    load4<float>(p.A + static_cast<int64_t>(chs) * 16 + 4 * q, Av);
    const float Dv = (valid && p.D) ? __ldg(p.D + chs) : 0.f;
    const float bv = (valid && p.bias) ? __ldg(p.bias + chs) : 0.f;
    float cw[4] = {0.f, 0.f, 0.f, 0.f};
    float cb = 0.f;
    if (CONV) {
        load4<float>(p.conv_w + static_cast<int64_t>(chs) * 4, cw);
        cb = (valid && p.conv_b) ? __ldg(p.conv_b + chs) : 0.f;
    }
    // Two batch rows per iteration, all their loads issued before the math.
    constexpr int R = 2;
    for (int64_t b0 = blockIdx.y; b0 < p.batch; b0 += static_cast<int64_t>(R) * gridDim.y) {
        int64_t cs[R];
        bool ok[R];
        float4 h4[R];
        float uu[R], xr[R], zz[R], Bv[R][4], Cv[R][4], cs3[R][3];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t b = b0 + static_cast<int64_t>(r) * gridDim.y;
            ok[r] = valid && b < p.batch;
            const int64_t bs = b < p.batch ? b : 0;
            cs[r] = bs * p.d + chs;
            h4[r] = ok[r] ? *(reinterpret_cast<const float4*>(p.state + cs[r] * 16) + q)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            uu[r] = ok[r] ? to_f32(static_cast<const IO*>(p.u)[cs[r]]) : 0.f;
            xr[r] = ok[r] ? to_f32(static_cast<const IO*>(p.delta)[cs[r]]) : 0.f;
            zz[r] = (ok[r] && p.z) ? to_f32(static_cast<const IO*>(p.z)[cs[r]]) : 0.f;
            load4<IO>(static_cast<const IO*>(p.B) + bs * 16 + 4 * q, Bv[r]);
            load4<IO>(static_cast<const IO*>(p.C) + bs * 16 + 4 * q, Cv[r]);
            if (CONV) {
#pragma unroll
                for (int k = 0; k < 3; ++k) cs3[r][k] = ok[r] ? p.conv_state[cs[r] * 3 + k] : 0.f;
            }
        }
        if (CONV) __syncwarp();   // every lane of a channel has read its conv state before it shifts
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (CONV) {
                const float xv = uu[r];
                const float c = fmaf(cw[3], xv, fmaf(cw[2], cs3[r][2], fmaf(cw[1], cs3[r][1], fmaf(cw[0], cs3[r][0], cb))));
                uu[r] = FAST ? silu_tanh(c) : silu_accurate(c);
                if (ok[r] && q == 0) {
                    p.conv_state[cs[r] * 3 + 0] = cs3[r][1];
                    p.conv_state[cs[r] * 3 + 1] = cs3[r][2];
                    p.conv_state[cs[r] * 3 + 2] = xv;
                }
            }
            // λ = Δ / ln 2 on the fast path (decay 2^(λ A), Δ u = λ (ln 2 u)); Δ itself otherwise.
            float lam, dscale;
            if (FAST) {
                const float y2 = fmaf(xr[r], kLog2e, bv * kLog2e);
                lam = p.softplus ? softplus_log2_fast(y2) : y2;
                dscale = kLn2;
            } else {
                const float x = xr[r] + bv;
                lam = p.softplus ? softplus_accurate(x) : x;
                dscale = 1.0f;
            }
            const float du = lam * (dscale * uu[r]);
            float hv[4] = {h4[r].x, h4[r].y, h4[r].z, h4[r].w};
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float a = FAST ? ex2_approx(lam * Av[m]) : expf(lam * Av[m]);
                hv[m] = fmaf(a, hv[m], du * Bv[r][m]);
                acc = fmaf(Cv[r][m], hv[m], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (ok[r]) {
                *(reinterpret_cast<float4*>(p.state + cs[r] * 16) + q) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                if (q == 0) {
                    float yv = fmaf(Dv, uu[r], acc);
                    if (p.z) yv *= FAST ? silu_tanh(zz[r]) : silu_accurate(zz[r]);
                    static_cast<IO*>(p.y)[cs[r]] = from_f32<IO>(yv);
                }
            }
        }
    }
}

// The same step for problems the grid tiles exactly (d_inner a multiple of
// kStepChanPerBlock, batch = R x gridDim.y, batch x d_inner x kN < 2^31) and
// no conv prologue: every thread has a valid channel and R valid batch
// rows (all loads issued before the math), and every element offset fits in 32 bits, so the body carries no
// bounds predicates and no 64-bit index arithmetic (about half the
// instructions of the general kernel on the decode workload).
template <typename IO, int R>
__global__ void __launch_bounds__(kStepThreads) ss_step_full_kernel(const __grid_constant__ StepParams p) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int q = threadIdx.x & 3;   // states 4q .. 4q+3
    const int ch = blockIdx.x * kStepChanPerBlock + (threadIdx.x >> 2);
    const int d = p.d;
    float Av[4];
    load4<float>(p.A + ch * kN + 4 * q, Av);
    const float Dv = p.D ? __ldg(p.D + ch) : 0.f;
    const float bv = p.bias ? __ldg(p.bias + ch) : 0.f;
    const IO* u = static_cast<const IO*>(p.u);
    const IO* dl = static_cast<const IO*>(p.delta);
    const IO* zp = static_cast<const IO*>(p.z);
    const IO* Bp = static_cast<const IO*>(p.B);
    const IO* Cp = static_cast<const IO*>(p.C);
    IO* yp = static_cast<IO*>(p.y);
    int bb[R], cs[R];
    float4 h4[R];
    float uu[R], xr[R], zz[R], Bv[R][4], Cv[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        bb[r] = blockIdx.y + r * gridDim.y;
        cs[r] = bb[r] * d + ch;
        h4[r] = *(reinterpret_cast<const float4*>(p.state + cs[r] * kN) + q);
        uu[r] = to_f32(u[cs[r]]);
        xr[r] = to_f32(dl[cs[r]]);
        zz[r] = zp ? to_f32(zp[cs[r]]) : 0.f;
        load4<IO>(Bp + bb[r] * kN + 4 * q, Bv[r]);
        load4<IO>(Cp + bb[r] * kN + 4 * q, Cv[r]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float lam, dscale;
        if (FAST) {
            const float y2 = fmaf(xr[r], kLog2e, bv * kLog2e);
            lam = p.softplus ? softplus_log2_fast(y2) : y2;
            dscale = kLn2;
        } else {
            const float x = xr[r] + bv;
            lam = p.softplus ? softplus_accurate(x) : x;
            dscale = 1.0f;
        }
        const float du = lam * (dscale * uu[r]);
        float hv[4] = {h4[r].x, h4[r].y, h4[r].z, h4[r].w};
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float a = FAST ? ex2_approx(lam * Av[m]) : expf(lam * Av[m]);
            hv[m] = fmaf(a, hv[m], du * Bv[r][m]);
            acc = fmaf(Cv[r][m], hv[m], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        *(reinterpret_cast<float4*>(p.state + cs[r] * kN) + q) = make_float4(hv[0], hv[1], hv[2], hv[3]);
        if (q == 0) {
            float yv = fmaf(Dv, uu[r], acc);
            if (zp) yv *= FAST ? silu_tanh(zz[r]) : silu_accurate(zz[r]);
            yp[cs[r]] = from_f32<IO>(yv);
        }
    }
}

}  // namespace selscan
