// bwd.cuh -- backward of the selective scan for sm_100a.
//
// Gradients of a scalar J through the forward recurrence of "Understanding
// Mamba and Selective State Space Models (SSMs)" §2.2 (first cut), §3.1 and
// §2.1 (the same y = (Σ_n C h + D u) · z σ(z), Δ = softplus(Δraw + bias) as
// the forward kernel), given dy = ∂J/∂y and optionally ∂J/∂last_state.  The
// pages train these models ("Mamba 7.9.1" article §5.3-5.4, training loop
// and gradient checkpointing; model-architecture-mamba page, "Common
// issues": checkpointing for memory) but print no backward; the adjoint here
// is reverse-mode differentiation of the recurrence, run backwards in time
// with the adjoint state g_n = ∂J/∂h_t,n:
//   ds = dy · gate(z),  dz = dy · s · gate'(z),  g += ds · C,  dC += ds · h_t,
//   dB += g Δ u,  du = ds D + Σ g Δ B,  dΔ = Σ g (a A h_{t-1} + B u),
//   dA += g a Δ h_{t-1},  g ← a g,  dΔraw = dΔ · softplus'(x),  dbias += dΔraw.
//
// Work decomposition: one CTA = (batch b, block of kBwdCh channels), one
// thread per channel holding its 16 states (8 fp32x2 pairs), the whole
// sequence in one CTA (no time chunking).  The forward states the adjoint
// needs are recomputed (gradient checkpointing, two levels):
//   pass 0   -- forward over the whole sequence, writing the state entering
//               every kSeg-step segment to a global checkpoint buffer;
//   pass 1   -- segments last to first: from the segment's checkpoint, a
//               forward pass stores the state entering every kSub-step
//               sub-segment in shared memory; sub-segments last to first: a
//               forward pass stores h_t of its kSub steps in shared memory,
//               then the adjoint runs back over them.
// dB and dC (sums over channels) are reduced across each warp by a
// transposing butterfly (31 shuffles leave lane l with value l summed over
// the warp) and added to global memory with one atomic per lane per step;
// dA, dD, dbias accumulate per thread over time and are added at the end.
// The library zeroes the accumulated outputs before the launch.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "fwd.cuh"

namespace selscan {

constexpr int kBwdCh = 64;          // channels (threads) per CTA
constexpr int kSeg = 32;            // steps per global checkpoint segment
constexpr int kSub = 8;             // steps per shared-memory sub-segment
constexpr int kNSub = kSeg / kSub;
constexpr int kNP4 = kN / 4;        // float4 groups of a channel's 16 states

struct BwdParams {
    const void* u;
    const void* delta;
    const float* bias;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const void* dy;
    const float* dlast;
    void* du;
    void* ddelta;
    void* dz;
    float* dA;
    float* dB;
    float* dC;
    float* dD;
    float* dbias;
    float* ckpt;          // [batch][nseg][d][kN]
    int64_t L;
    int batch, d, nseg, nblk;
    int softplus;
};

template <typename IO>
struct BwdSmem {
    float4 hsub[kNSub][kNP4][kBwdCh];    // state entering each sub-segment
    float4 hstep[kSub][kNP4][kBwdCh];    // h_t of the current sub-segment
    float bc[kSeg][2 * kN];              // B then C of the segment, fp32
    IO tu[kSeg][kBwdCh];                 // the segment's u, Δraw, z, dy
    IO tdt[kSeg][kBwdCh];
    IO tz[kSeg][kBwdCh];
    IO tdy[kSeg][kBwdCh];
};

// Per-channel constants of the backward.
struct BwdChan {
    float Al[kN];      // A[ch, n] · log2 e (exp(Δ A) = 2^(Δ Al))
    float A[kN];
    float al;          // structured path: A[ch, n] = a (n + 1); al = a · log2 e
    float bias, Dv;
    bool valid;
};

// softplus(x) and σ(x) (its derivative) for one element.
template <bool FAST>
__device__ __forceinline__ void softplus_and_sigmoid(float x, float& sp, float& sig) {
    if (FAST) {
        const float e = ex2_approx(x * kLog2e);
        sp = (x > 20.0f) ? x : kLn2 * lg2_approx(1.0f + e);
        sig = (x > 20.0f) ? 1.0f : e * rcp_approx(1.0f + e);
    } else {
        sp = softplus_accurate(x);
        sig = (x > 20.0f) ? 1.0f : 1.0f / (1.0f + expf(-x));
    }
}

// exp(Δ A_n) for the 16 states.
template <bool FAST, bool STRUCT>
__device__ __forceinline__ void decays(float dt, const BwdChan& cp, float (&a)[kN]) {
    if (STRUCT) {
        const float r = ex2_approx(dt * cp.al);
        a[0] = r;
#pragma unroll
        for (int n = 1; n < kN; ++n) a[n] = a[n - 1] * r;
    } else {
#pragma unroll
        for (int n = 0; n < kN; ++n) a[n] = FAST ? ex2_approx(dt * cp.Al[n]) : expf(dt * cp.A[n]);
    }
}

// Sum over the warp of v[0..31] (each lane's own 32 values): on return lane
// l holds the warp's sum of v[l].  Each halving step keeps one half of the
// values, sends the other to the partner lane, and adds what comes back.
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = up ? v[i] : v[i + m];
            const float keep = up ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0];
}

// Loads the segment's tiles: B and C (fp32) of steps t0 .. t0+nt-1 and, for
// the block's channels, u and Δraw (and z, dy when `adjoint`).  Every load is
// independent, so their latencies overlap; rows >= nt are left unset.
template <typename IO>
__device__ __forceinline__ void load_seg(BwdSmem<IO>& S, const BwdParams& p, int b, int blk, int64_t t0, int nt,
                                         bool adjoint) {
    for (int i = threadIdx.x; i < nt * kN; i += kBwdCh) {
        const int r = i / kN, n = i % kN;
        const int64_t idx = (static_cast<int64_t>(b) * p.L + t0 + r) * kN + n;
        S.bc[r][n] = to_f32(static_cast<const IO*>(p.B)[idx]);
        S.bc[r][kN + n] = to_f32(static_cast<const IO*>(p.C)[idx]);
    }
    const int c = threadIdx.x;
    const int64_t ch = static_cast<int64_t>(blk) * kBwdCh + c;
    const bool ok = ch < p.d;
    const IO zero = from_f32<IO>(0.0f);
    for (int r = 0; r < nt; ++r) {
        const int64_t i = (static_cast<int64_t>(b) * p.L + t0 + r) * p.d + ch;
        S.tu[r][c] = ok ? static_cast<const IO*>(p.u)[i] : zero;
        S.tdt[r][c] = ok ? static_cast<const IO*>(p.delta)[i] : zero;
        if (adjoint) {
            S.tz[r][c] = (ok && p.z) ? static_cast<const IO*>(p.z)[i] : zero;
            S.tdy[r][c] = ok ? static_cast<const IO*>(p.dy)[i] : zero;
        }
    }
}

// One forward step (row r of the segment) of this thread's channel:
// h ← a h + Δ B u.
template <typename IO, bool FAST, bool STRUCT>
__device__ __forceinline__ void fwd_step(const BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int r,
                                         float (&h)[kN]) {
    const int c = threadIdx.x;
    const float x = to_f32(S.tdt[r][c]) + cp.bias;
    float dt, sig;
    if (p.softplus) softplus_and_sigmoid<FAST>(x, dt, sig);
    else dt = x;
    const float du = dt * to_f32(S.tu[r][c]);
    float a[kN];
    decays<FAST, STRUCT>(dt, cp, a);
#pragma unroll
    for (int n = 0; n < kN; n += 2) {
        const f32x2 hn = fma2(pk2(a[n], a[n + 1]), pk2(h[n], h[n + 1]),
                              mul2(pk2(du, du), pk2(S.bc[r][n], S.bc[r][n + 1])));
        h[n] = hn.x;
        h[n + 1] = hn.y;
    }
}

__device__ __forceinline__ void store_state(float4 (&dst)[kNP4][kBwdCh], int tid, const float (&h)[kN]) {
#pragma unroll
    for (int q = 0; q < kNP4; ++q) dst[q][tid] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
}
__device__ __forceinline__ void load_state(const float4 (&src)[kNP4][kBwdCh], int tid, float (&h)[kN]) {
#pragma unroll
    for (int q = 0; q < kNP4; ++q) {
        const float4 v = src[q][tid];
        h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
    }
}

template <typename IO, bool STRUCT>
__device__ __forceinline__ void bwd_item(BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                         int ch) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t d = p.d;
    const int64_t row0 = static_cast<int64_t>(b) * p.L;   // (b, t) row index base

    // ---------------------------------------------------------------- pass 0
    float h[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) h[n] = 0.0f;
    for (int seg = 0; seg < p.nseg; ++seg) {
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        const int nt = static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0));
        if (cp.valid) {
            float4* ck = reinterpret_cast<float4*>(p.ckpt + ((static_cast<int64_t>(b) * p.nseg + seg) * d + ch) * kN);
#pragma unroll
            for (int q = 0; q < kNP4; ++q) ck[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
        __syncthreads();
        load_seg<IO>(S, p, b, blk, t0, nt, false);
        __syncthreads();
        for (int r = 0; r < nt; ++r) fwd_step<IO, FAST, STRUCT>(S, p, cp, r, h);
    }

    // ---------------------------------------------------------------- pass 1
    float g[kN], dA_acc[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) {
        g[n] = (p.dlast && cp.valid) ? p.dlast[(static_cast<int64_t>(b) * d + ch) * kN + n] : 0.0f;
        dA_acc[n] = 0.0f;
    }
    float dD_acc = 0.0f, dbias_acc = 0.0f;
    for (int seg = p.nseg - 1; seg >= 0; --seg) {
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        const int nt = static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0));
        const int nsub = (nt + kSub - 1) / kSub;
        __syncthreads();
        load_seg<IO>(S, p, b, blk, t0, nt, true);
        __syncthreads();
        if (cp.valid) {
            const float4* ck =
                reinterpret_cast<const float4*>(p.ckpt + ((static_cast<int64_t>(b) * p.nseg + seg) * d + ch) * kN);
#pragma unroll
            for (int q = 0; q < kNP4; ++q) {
                const float4 v = ck[q];
                h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int n = 0; n < kN; ++n) h[n] = 0.0f;
        }
        // sub-checkpoints (each thread touches only its own column)
        for (int s = 0; s < nsub; ++s) {
            store_state(S.hsub[s], tid, h);
            const int ns = min(kSub, nt - s * kSub);
            for (int j = 0; j < ns; ++j) {
                fwd_step<IO, FAST, STRUCT>(S, p, cp, s * kSub + j, h);
            }
        }
        for (int s = nsub - 1; s >= 0; --s) {
            const int ns = min(kSub, nt - s * kSub);
            load_state(S.hsub[s], tid, h);
            for (int j = 0; j < ns; ++j) {
                fwd_step<IO, FAST, STRUCT>(S, p, cp, s * kSub + j, h);
                store_state(S.hstep[j], tid, h);
            }
            for (int j = ns - 1; j >= 0; --j) {
                const int r = s * kSub + j;
                const int64_t t = t0 + r;
                const int64_t i = (row0 + t) * d + ch;
                float hp[kN], hc[kN];
                load_state(S.hstep[j], tid, hc);
                if (j > 0) load_state(S.hstep[j - 1], tid, hp);
                else load_state(S.hsub[s], tid, hp);
                const float x = to_f32(S.tdt[r][tid]) + cp.bias;
                float dt, sig = 1.0f;
                if (p.softplus) softplus_and_sigmoid<FAST>(x, dt, sig);
                else dt = x;
                const float uv = to_f32(S.tu[r][tid]);
                const float dyv = to_f32(S.tdy[r][tid]);
                float a[kN];
                decays<FAST, STRUCT>(dt, cp, a);
                // s_t = Σ_n C h_t + D u, then the gate
                f32x2 acc = pk2(0.f, 0.f);
#pragma unroll
                for (int n = 0; n < kN; n += 2)
                    acc = fma2(pk2(S.bc[r][kN + n], S.bc[r][kN + n + 1]), pk2(hc[n], hc[n + 1]), acc);
                const float sv = acc.x + acc.y + cp.Dv * uv;
                float ds = dyv;
                if (p.z) {
                    const float zv = to_f32(S.tz[r][tid]);
                    const float sz = FAST ? rcp_approx(1.0f + ex2_approx(-zv * kLog2e)) : 1.0f / (1.0f + expf(-zv));
                    ds = dyv * zv * sz;
                    if (cp.valid)
                        static_cast<IO*>(p.dz)[i] = from_f32<IO>(dyv * sv * sz * (1.0f + zv * (1.0f - sz)));
                }
                dD_acc += ds * uv;
                float duv = ds * cp.Dv, dDelta = 0.0f;
                const float dtu = dt * uv;
                float red[32];
#pragma unroll
                for (int n = 0; n < kN; ++n) {
                    const float Bn = S.bc[r][n], Cn = S.bc[r][kN + n];
                    g[n] = fmaf(ds, Cn, g[n]);
                    red[kN + n] = ds * hc[n];                 // dC contribution
                    red[n] = g[n] * dtu;                      // dB contribution
                    duv = fmaf(g[n] * dt, Bn, duv);
                    const float ah = a[n] * hp[n];
                    dDelta = fmaf(g[n], fmaf(ah, cp.A[n], Bn * uv), dDelta);
                    dA_acc[n] = fmaf(g[n] * dt, ah, dA_acc[n]);
                    g[n] *= a[n];
                }
                const float dx = dDelta * sig;
                dbias_acc += dx;
                if (cp.valid) {
                    static_cast<IO*>(p.du)[i] = from_f32<IO>(duv);
                    static_cast<IO*>(p.ddelta)[i] = from_f32<IO>(dx);
                }
                const float tot = warp_transpose_sum(red, lane);
                float* dst = (lane < kN ? p.dB : p.dC) + (row0 + t) * kN + (lane & (kN - 1));
                atomicAdd(dst, tot);
            }
        }
    }
    if (cp.valid) {
#pragma unroll
        for (int n = 0; n < kN; ++n) atomicAdd(p.dA + static_cast<int64_t>(ch) * kN + n, dA_acc[n]);
        if (p.dD) atomicAdd(p.dD + ch, dD_acc);
        if (p.dbias) atomicAdd(p.dbias + ch, dbias_acc);
    }
}

template <typename IO>
__global__ void __launch_bounds__(kBwdCh) ss_bwd_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ __align__(16) unsigned char bwd_smem_raw[];
    auto& S = *reinterpret_cast<BwdSmem<IO>*>(bwd_smem_raw);
    const int g = blockIdx.x % p.nblk;
    const int b = blockIdx.x / p.nblk;
    const int ch = g * kBwdCh + threadIdx.x;
    BwdChan cp;
    cp.valid = ch < p.d;
    bool structured = true;
    const float* Arow = p.A + static_cast<int64_t>(cp.valid ? ch : 0) * kN;
    const float a0 = cp.valid ? Arow[0] : -1.0f;
#pragma unroll
    for (int n = 0; n < kN; ++n) {
        cp.A[n] = cp.valid ? Arow[n] : -static_cast<float>(n + 1);
        cp.Al[n] = cp.A[n] * kLog2e;
        structured = structured && (cp.A[n] == a0 * static_cast<float>(n + 1));
    }
    cp.al = a0 * kLog2e;
    cp.bias = (cp.valid && p.bias) ? p.bias[ch] : 0.0f;
    cp.Dv = (cp.valid && p.D) ? p.D[ch] : 0.0f;
    const int all_struct = __syncthreads_and(structured ? 1 : 0);
    if (std::is_same<IO, __nv_bfloat16>::value && all_struct)
        bwd_item<IO, true>(S, p, cp, b, g, ch);
    else
        bwd_item<IO, false>(S, p, cp, b, g, ch);
}

}  // namespace selscan
