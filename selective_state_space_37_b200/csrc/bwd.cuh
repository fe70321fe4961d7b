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
// Work decomposition: one CTA = (batch b, block of kBwdCh channels), the
// whole sequence in one CTA (no time chunking).  Two threads share a channel
// -- lanes l and l^16 of a warp, each with 8 of its 16 states -- so a warp
// serves 16 channels; the per-channel sums over states (readout, du, dΔ)
// take one shuffle each.  The forward states the adjoint
// needs are recomputed (gradient checkpointing, two levels):
//   pass 0   -- forward over the whole sequence, writing the state entering
//               every kSeg-step segment to a global checkpoint buffer;
//   pass 1   -- segments last to first: from the segment's checkpoint, a
//               forward pass stores the state entering every kSub-step
//               sub-segment in shared memory; sub-segments last to first: a
//               forward pass stores h_t of its kSub steps in shared memory,
//               then the adjoint runs back over them.
// dB and dC (sums over channels) are reduced across each half-warp by a
// transposing butterfly (15 shuffles leave lane j of the half with value j
// summed over its 16 channels) and added to global memory with one atomic
// per lane per step;
// dA, dD, dbias accumulate per thread over time and are added at the end.
// The library zeroes the accumulated outputs before the launch.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "fwd.cuh"

namespace selscan {

constexpr int kBwdCh = 64;          // channels per CTA
constexpr int kBwdThreads = 2 * kBwdCh;   // two threads per channel
constexpr int kBH = kN / 2;         // states per thread
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

// Per-thread constants of the backward: this thread's channel and half.
struct BwdChan {
    float A[kBH];      // A[ch, 8p + m]
    float Al[kBH];     // A[ch, 8p + m] · log2 e (exp(Δ A) = 2^(Δ Al))
    float al;          // structured path (A[ch, n] = a (n + 1)): a · log2 e
    float alb;         // a (8p + 1) · log2 e: exponent factor of the half's first decay
    float bias, Dv;
    int c;             // channel within the block
    int p;             // 0: states 0..7, 1: states 8..15
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

// exp(Δ A_n) for this thread's 8 states.
template <bool FAST, bool STRUCT>
__device__ __forceinline__ void decays(float dt, const BwdChan& cp, float (&a)[kBH]) {
    if (STRUCT) {
        const float r = ex2_approx(dt * cp.al);
        a[0] = ex2_approx(dt * cp.alb);   // r^(8p+1)
#pragma unroll
        for (int m = 1; m < kBH; ++m) a[m] = a[m - 1] * r;
    } else {
#pragma unroll
        for (int m = 0; m < kBH; ++m) a[m] = FAST ? ex2_approx(dt * cp.Al[m]) : expf(dt * cp.A[m]);
    }
}

// Loads the segment's tiles: B and C (fp32) of steps t0 .. t0+nt-1 and, for
// the block's channels, u and Δraw (and z, dy when `adjoint`).  Every load is
// independent, so their latencies overlap; rows >= nt are left unset.
template <typename IO>
__device__ __forceinline__ void load_seg(BwdSmem<IO>& S, const BwdParams& p, int b, int blk, int64_t t0, int nt,
                                         bool adjoint) {
    for (int i = threadIdx.x; i < nt * kN; i += kBwdThreads) {
        const int r = i / kN, n = i % kN;
        const int64_t idx = (static_cast<int64_t>(b) * p.L + t0 + r) * kN + n;
        S.bc[r][n] = to_f32(static_cast<const IO*>(p.B)[idx]);
        S.bc[r][kN + n] = to_f32(static_cast<const IO*>(p.C)[idx]);
    }
    const int c = threadIdx.x % kBwdCh;
    const int64_t ch = static_cast<int64_t>(blk) * kBwdCh + c;
    const bool ok = ch < p.d;
    const IO zero = from_f32<IO>(0.0f);
    for (int r = threadIdx.x / kBwdCh; r < nt; r += kBwdThreads / kBwdCh) {
        const int64_t i = (static_cast<int64_t>(b) * p.L + t0 + r) * p.d + ch;
        S.tu[r][c] = ok ? static_cast<const IO*>(p.u)[i] : zero;
        S.tdt[r][c] = ok ? static_cast<const IO*>(p.delta)[i] : zero;
        if (adjoint) {
            S.tz[r][c] = (ok && p.z) ? static_cast<const IO*>(p.z)[i] : zero;
            S.tdy[r][c] = ok ? static_cast<const IO*>(p.dy)[i] : zero;
        }
    }
}

// One forward step (row r of the segment) of this thread's half-channel:
// h ← a h + Δ B u.
template <typename IO, bool FAST, bool STRUCT, bool SP>
__device__ __forceinline__ void fwd_step(const BwdSmem<IO>& S, const BwdChan& cp, int r, float (&h)[kBH]) {
    const float x = to_f32(S.tdt[r][cp.c]) + cp.bias;
    float dt = x, sig;
    if (SP) softplus_and_sigmoid<FAST>(x, dt, sig);
    const float du = dt * to_f32(S.tu[r][cp.c]);
    float a[kBH];
    decays<FAST, STRUCT>(dt, cp, a);
    const float* Bh = &S.bc[r][kBH * cp.p];
#pragma unroll
    for (int m = 0; m < kBH; m += 2) {
        const f32x2 hn = fma2(pk2(a[m], a[m + 1]), pk2(h[m], h[m + 1]), mul2(pk2(du, du), pk2(Bh[m], Bh[m + 1])));
        h[m] = hn.x;
        h[m + 1] = hn.y;
    }
}

__device__ __forceinline__ void store_state(float4 (&dst)[kNP4][kBwdCh], const BwdChan& cp, const float (&h)[kBH]) {
    dst[2 * cp.p][cp.c] = make_float4(h[0], h[1], h[2], h[3]);
    dst[2 * cp.p + 1][cp.c] = make_float4(h[4], h[5], h[6], h[7]);
}
__device__ __forceinline__ void load_state(const float4 (&src)[kNP4][kBwdCh], const BwdChan& cp, float (&h)[kBH]) {
    const float4 v0 = src[2 * cp.p][cp.c], v1 = src[2 * cp.p + 1][cp.c];
    h[0] = v0.x; h[1] = v0.y; h[2] = v0.z; h[3] = v0.w;
    h[4] = v1.x; h[5] = v1.y; h[6] = v1.z; h[7] = v1.w;
}

template <typename IO, bool STRUCT, bool SP, bool HZ>
__device__ __forceinline__ void bwd_item(BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                         int ch) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int j16 = threadIdx.x & 15;                     // lane within the half-warp
    const int64_t d = p.d;
    const int64_t row0 = static_cast<int64_t>(b) * p.L;   // (b, t) row index base
    const int hp = kBH * cp.p;
    const bool writer = cp.valid && cp.p == 0;            // stores the per-channel outputs

    // ---------------------------------------------------------------- pass 0
    float h[kBH];
#pragma unroll
    for (int m = 0; m < kBH; ++m) h[m] = 0.0f;
    for (int seg = 0; seg < p.nseg; ++seg) {
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        const int nt = static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0));
        if (cp.valid) {
            float4* ck =
                reinterpret_cast<float4*>(p.ckpt + ((static_cast<int64_t>(b) * p.nseg + seg) * d + ch) * kN + hp);
            ck[0] = make_float4(h[0], h[1], h[2], h[3]);
            ck[1] = make_float4(h[4], h[5], h[6], h[7]);
        }
        __syncthreads();
        load_seg<IO>(S, p, b, blk, t0, nt, false);
        __syncthreads();
        if (nt == kSeg) {
#pragma unroll 8
            for (int r = 0; r < kSeg; ++r) fwd_step<IO, FAST, STRUCT, SP>(S, cp, r, h);
        } else {
            for (int r = 0; r < nt; ++r) fwd_step<IO, FAST, STRUCT, SP>(S, cp, r, h);
        }
    }

    // ---------------------------------------------------------------- pass 1
    float g[kBH], dA_acc[kBH];
#pragma unroll
    for (int m = 0; m < kBH; ++m) {
        g[m] = (p.dlast && cp.valid) ? p.dlast[(static_cast<int64_t>(b) * d + ch) * kN + hp + m] : 0.0f;
        dA_acc[m] = 0.0f;
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
            const float4* ck = reinterpret_cast<const float4*>(
                p.ckpt + ((static_cast<int64_t>(b) * p.nseg + seg) * d + ch) * kN + hp);
            const float4 v0 = ck[0], v1 = ck[1];
            h[0] = v0.x; h[1] = v0.y; h[2] = v0.z; h[3] = v0.w;
            h[4] = v1.x; h[5] = v1.y; h[6] = v1.z; h[7] = v1.w;
        } else {
#pragma unroll
            for (int m = 0; m < kBH; ++m) h[m] = 0.0f;
        }
        // sub-checkpoints (each thread touches only its own half-column); the
        // last sub-segment's steps are not needed for them
        for (int s = 0; s < nsub; ++s) {
            store_state(S.hsub[s], cp, h);
            if (s + 1 == nsub) break;
#pragma unroll
            for (int j = 0; j < kSub; ++j) fwd_step<IO, FAST, STRUCT, SP>(S, cp, s * kSub + j, h);
        }
        for (int s = nsub - 1; s >= 0; --s) {
            const int ns = min(kSub, nt - s * kSub);
            load_state(S.hsub[s], cp, h);
            if (ns == kSub) {
#pragma unroll
                for (int j = 0; j < kSub; ++j) {
                    fwd_step<IO, FAST, STRUCT, SP>(S, cp, s * kSub + j, h);
                    store_state(S.hstep[j], cp, h);
                }
            } else {
                for (int j = 0; j < ns; ++j) {
                    fwd_step<IO, FAST, STRUCT, SP>(S, cp, s * kSub + j, h);
                    store_state(S.hstep[j], cp, h);
                }
            }
            for (int j = ns - 1; j >= 0; --j) {
                const int r = s * kSub + j;
                const int64_t t = t0 + r;
                const int64_t i = (row0 + t) * d + ch;
                float hprev[kBH], hc[kBH];
                load_state(S.hstep[j], cp, hc);
                if (j > 0) load_state(S.hstep[j - 1], cp, hprev);
                else load_state(S.hsub[s], cp, hprev);
                const float x = to_f32(S.tdt[r][cp.c]) + cp.bias;
                float dt = x, sig = 1.0f;
                if (SP) softplus_and_sigmoid<FAST>(x, dt, sig);
                const float uv = to_f32(S.tu[r][cp.c]);
                const float dyv = to_f32(S.tdy[r][cp.c]);
                float a[kBH];
                decays<FAST, STRUCT>(dt, cp, a);
                const float* Bh = &S.bc[r][hp];
                const float* Ch = &S.bc[r][kN + hp];
                // s_t = Σ_n C h_t + D u (both halves), then the gate
                f32x2 acc = mul2(pk2(Ch[0], Ch[1]), pk2(hc[0], hc[1]));
#pragma unroll
                for (int m = 2; m < kBH; m += 2) acc = fma2(pk2(Ch[m], Ch[m + 1]), pk2(hc[m], hc[m + 1]), acc);
                const float sh = acc.x + acc.y;
                const float sv = sh + partner(sh) + cp.Dv * uv;
                float ds = dyv;
                if (HZ) {
                    const float zv = to_f32(S.tz[r][cp.c]);
                    const float sz = FAST ? rcp_approx(1.0f + ex2_approx(-zv * kLog2e)) : 1.0f / (1.0f + expf(-zv));
                    ds = dyv * zv * sz;
                    if (writer) static_cast<IO*>(p.dz)[i] = from_f32<IO>(dyv * sv * sz * (1.0f + zv * (1.0f - sz)));
                }
                dD_acc += ds * uv;
                float du_h = 0.0f, dD_h = 0.0f;
                const float dtu = dt * uv;
                float red[2 * kBH];
#pragma unroll
                for (int m = 0; m < kBH; ++m) {
                    g[m] = fmaf(ds, Ch[m], g[m]);
                    red[kBH + m] = ds * hc[m];                // dC contribution
                    red[m] = g[m] * dtu;                      // dB contribution
                    du_h = fmaf(g[m] * dt, Bh[m], du_h);
                    const float ah = a[m] * hprev[m];
                    dD_h = fmaf(g[m], fmaf(ah, cp.A[m], Bh[m] * uv), dD_h);
                    dA_acc[m] = fmaf(g[m] * dt, ah, dA_acc[m]);
                    g[m] *= a[m];
                }
                const float duv = fmaf(ds, cp.Dv, du_h + partner(du_h));
                const float dx = (dD_h + partner(dD_h)) * sig;
                dbias_acc += dx;
                if (writer) {
                    static_cast<IO*>(p.du)[i] = from_f32<IO>(duv);
                    static_cast<IO*>(p.ddelta)[i] = from_f32<IO>(dx);
                }
                // dB / dC summed over the half-warp's 16 channels: each halving
                // step keeps one half of the values, sends the other to the
                // partner lane and adds what comes back; lane j ends with value j.
#pragma unroll
                for (int mm = kBH; mm >= 1; mm >>= 1) {
                    const bool up = (j16 & mm) != 0;
#pragma unroll
                    for (int q = 0; q < mm; ++q) {
                        const float send = up ? red[q] : red[q + mm];
                        const float keep = up ? red[q + mm] : red[q];
                        red[q] = keep + __shfl_xor_sync(0xffffffffu, send, mm);
                    }
                }
                float* dst = (j16 < kBH ? p.dB : p.dC) + (row0 + t) * kN + hp + (j16 & (kBH - 1));
                atomicAdd(dst, red[0]);
            }
        }
    }
    if (cp.valid) {
#pragma unroll
        for (int m = 0; m < kBH; ++m) atomicAdd(p.dA + static_cast<int64_t>(ch) * kN + hp + m, dA_acc[m]);
        if (cp.p == 0) {
            if (p.dD) atomicAdd(p.dD + ch, dD_acc);
            if (p.dbias) atomicAdd(p.dbias + ch, dbias_acc);
        }
    }
}

// SP: Δ goes through softplus; HZ: the silu(z) gate is on.
template <typename IO, bool SP, bool HZ>
__global__ void __launch_bounds__(kBwdThreads) ss_bwd_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ __align__(16) unsigned char bwd_smem_raw[];
    auto& S = *reinterpret_cast<BwdSmem<IO>*>(bwd_smem_raw);
    const int blk = blockIdx.x % p.nblk;
    const int b = blockIdx.x / p.nblk;
    const int lane = threadIdx.x & 31;
    BwdChan cp;
    cp.c = (threadIdx.x >> 5) * 16 + (lane & 15);
    cp.p = lane >> 4;
    const int ch = blk * kBwdCh + cp.c;
    const int hp = kBH * cp.p;
    cp.valid = ch < p.d;
    bool structured = true;
    const float* Arow = p.A + static_cast<int64_t>(cp.valid ? ch : 0) * kN;
    const float a0 = cp.valid ? Arow[0] : -1.0f;
#pragma unroll
    for (int m = 0; m < kBH; ++m) {
        cp.A[m] = cp.valid ? Arow[hp + m] : -static_cast<float>(hp + m + 1);
        cp.Al[m] = cp.A[m] * kLog2e;
        structured = structured && (cp.A[m] == a0 * static_cast<float>(hp + m + 1));
    }
    cp.al = a0 * kLog2e;
    cp.alb = cp.al * static_cast<float>(hp + 1);
    cp.bias = (cp.valid && p.bias) ? p.bias[ch] : 0.0f;
    cp.Dv = (cp.valid && p.D) ? p.D[ch] : 0.0f;
    const int all_struct = __syncthreads_and(structured ? 1 : 0);
    if (std::is_same<IO, __nv_bfloat16>::value && all_struct)
        bwd_item<IO, true, SP, HZ>(S, p, cp, b, blk, ch);
    else
        bwd_item<IO, false, SP, HZ>(S, p, cp, b, blk, ch);
}

}  // namespace selscan
