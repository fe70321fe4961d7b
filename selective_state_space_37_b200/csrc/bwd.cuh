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
// Work decomposition: an item = (batch b, block of kBwdCh channels, time
// chunk k of cseg segments).  Two threads share a channel -- lanes l and
// l^16 of a warp, each with 8 of its 16 states -- so a warp serves 16
// channels; the per-channel sums over states (readout, du, dΔ) take one
// shuffle each.  Both recurrences are linear, so a chunk's entering state
// and adjoint follow from records of the other chunks (an exact carry, as in
// the forward's time chunks):
//   h_in(k) = Σ_{j<k} (Π_{j<i<k} P_i) h_loc(j),  G_in(k) = the same from the
//   other side over g_loc(j), j > k, starting from dlast_state,
// with P_j = exp(A Σ_{t in chunk j} Δ_t) (A is constant in time).
//   ss_bwd_chunk_kernel -- per item: a forward pass from zero over the chunk,
//               writing the state entering each kSeg-step segment (local
//               checkpoints, with Σ Δ since the chunk's start) and the
//               chunk's end state h_loc; then (chunks k > 0) the adjoint-only
//               recurrence g ← exp(Δ A)(g + ds C) from zero backwards over
//               the chunk, giving g_loc.  Its segment tiles arrive by
//               cp.async into a double-buffered raw area while the previous
//               segment's steps run (ChunkSmem).
//   ss_bwd_combine_kernel -- folds the records in chunk order into h_in(k)
//               and G_in(k) for every chunk (one thread per state).
//   ss_bwd_kernel -- per item: h_in and G_in from the folded records; then
//               segments last to first: the checkpoint made exact
//               (h_loc + exp(A Σ Δ) h_in), a forward pass that stores the
//               state entering every kSub-step sub-segment in shared memory;
//               sub-segments last to first: a forward pass keeps h_t of its
//               kSub steps in registers, then the adjoint runs back over them
//               and emits every gradient.
// Each segment's per-(step, channel) scalars -- Δ = softplus(Δraw + bias),
// its derivative σ(Δraw + bias), and for the structured A (A[d, n] = a (n+1))
// the decay bases r = exp(Δ a) and r^9 -- are computed once when the segment
// is staged, so the recomputed forward steps and the adjoint read them from
// shared memory instead of re-evaluating them per thread and per pass.
// dB and dC (sums over channels) go through a per-warp transpose in shared
// memory: every lane stores its 16 contributions, then lane j of half p sums
// value j over the half's 16 channels and adds it to global memory with one
// atomic per step.  dA, dD, dbias accumulate per thread over time and are
// added at the end.  The library zeroes the accumulated outputs before the
// launch.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "cp_async.cuh"
#include "fwd.cuh"

namespace selscan {

constexpr int kBwdCh = 64;          // channels per CTA
constexpr int kBwdThreads = 2 * kBwdCh;   // two threads per channel
constexpr int kBH = kN / 2;         // states per thread
constexpr int kSeg = 32;            // steps per global checkpoint segment
constexpr int kSub = 8;             // steps per shared-memory sub-segment
constexpr int kNSub = kSeg / kSub;
constexpr int kNP4 = kN / 4;        // float4 groups of a channel's 16 states
constexpr int kRedRow = 36;         // words per row of a warp's dB/dC transpose buffer:
                                    // 2 halves x 16 channels + 4 of padding (conflict-free float4 reads)

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
    float* ckpt;          // [batch][nseg][d][kN]: state entering each segment, from zero at its chunk's start
    float* sck;           // [batch][nseg][d]: Σ Δ from the chunk's start to the segment's start
    float* hloc;          // [batch][nchunk][d][kN]: state at the chunk's end, from zero at its start
    float* gloc;          // [batch][nchunk][d][kN]: adjoint at the chunk's start, from zero at its end
    float* send;          // [batch][nchunk][d]: Σ Δ over the chunk
    int64_t L;
    int batch, d, nseg, nblk;
    int nchunk, cseg;     // time chunks and segments per chunk
    int vec;              // rows of u, Δraw, z, dy start 16-byte aligned (d a multiple of 16 B / element)
    int softplus;
};

// Shared memory of the chunk pass: the raw tiles double-buffered, so one
// segment's copies (cp.async) overlap the previous segment's steps.
template <typename IO>
struct ChunkSmem {
    IO raw[2][3][kSeg][kBwdCh];   // [0] Δraw; forward: [1] u; adjoint-only: [1] z, [2] dy
    IO rbc[2][kSeg][kN];          // B (forward) or C (adjoint-only)
    float4 pre[kSeg][kBwdCh];     // forward {Δu, r, r^9, Δ}; adjoint-only {ds, r, r^9, Δ}
    float bc[kSeg][kN];           // B or C, fp32
};

template <typename IO>
struct BwdSmem {
    float4 hsub[kNSub][kNP4][kBwdCh];    // state entering each sub-segment
    float4 pre[kSeg][kBwdCh];            // {Δ, r, r^9, σ} per (step, channel) of the segment
    float bc[kSeg][2 * kN];              // B then C of the segment, fp32
    IO tu[kSeg][kBwdCh];                 // the segment's u, z, dy
    IO tz[kSeg][kBwdCh];
    IO tdy[kSeg][kBwdCh];
    float red[kBwdThreads / 32][2 * kBH][kRedRow];   // dB/dC transpose, one buffer per warp
};

// Per-thread constants of the backward: this thread's channel and half.
struct BwdChan {
    float A[kBH];      // A[ch, 8p + m]
    float Al[kBH];     // A[ch, 8p + m] · log2 e (exp(Δ A) = 2^(Δ Al))
    float bias, Dv;
    float al_s, bias_s;   // a · log2 e and the bias of the channel this thread stages (threadIdx.x % kBwdCh)
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

// exp(Δ A_n) for this thread's 8 states from the staged {Δ, r, r^9, σ}: on
// the structured path r^(8p+1) times powers of r (a product ladder over
// pairs), otherwise one exponential per state.
template <bool FAST, bool STRUCT>
__device__ __forceinline__ void decays(const float4 pr, const BwdChan& cp, float (&a)[kBH]) {
    if (STRUCT) {
        const float r = pr.y;
        const float r2 = r * r;
        a[0] = cp.p ? pr.z : r;
        a[1] = a[0] * r;
#pragma unroll
        for (int m = 2; m < kBH; m += 2) {
            const f32x2 v = mul2(pk2(a[m - 2], a[m - 1]), pk2(r2, r2));
            a[m] = v.x;
            a[m + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int m = 0; m < kBH; ++m) a[m] = FAST ? ex2_approx(pr.x * cp.Al[m]) : expf(pr.x * cp.A[m]);
    }
}

// Stages the segment: B and C (fp32) of steps t0 .. t0+nt-1 and, for the
// block's channels, u (and z, dy when `adjoint`) and the per-step scalars
// {Δ, r, r^9, σ}.  Every load is independent, so their latencies overlap;
// rows >= nt are left unset.
template <typename IO, bool FAST, bool STRUCT, bool SP>
__device__ __forceinline__ void load_seg(BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                         int64_t t0, int nt, bool adjoint) {
#pragma unroll 4
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
    const int64_t base = (static_cast<int64_t>(b) * p.L + t0) * p.d + ch;
    constexpr int kStride = kBwdThreads / kBwdCh;   // rows between a thread's rows
    constexpr int kRows = kSeg / kStride;           // rows per thread
    constexpr int kBatch = kRows / 2;               // rows whose loads are in flight together
    const int r0 = threadIdx.x / kBwdCh;
#pragma unroll 1
    for (int q0 = 0; q0 < kRows; q0 += kBatch) {
        // the batch's loads first, so one memory latency covers them
        IO lu[kBatch], ld[kBatch], lz[kBatch], ly[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int r = r0 + (q0 + q) * kStride;
            const int64_t i = base + static_cast<int64_t>(r) * p.d;
            const bool in = ok && r < nt;
            lu[q] = in ? static_cast<const IO*>(p.u)[i] : zero;
            ld[q] = in ? static_cast<const IO*>(p.delta)[i] : zero;
            if (adjoint) {
                lz[q] = (in && p.z) ? static_cast<const IO*>(p.z)[i] : zero;
                ly[q] = in ? static_cast<const IO*>(p.dy)[i] : zero;
            }
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int r = r0 + (q0 + q) * kStride;
            if (r >= nt) break;
            S.tu[r][c] = lu[q];
            const float x = to_f32(ld[q]) + cp.bias_s;
            float dt = x, sig = 1.0f;
            if (SP) softplus_and_sigmoid<FAST>(x, dt, sig);
            float rr = 0.0f, r9 = 0.0f;
            if (STRUCT) {
                rr = ex2_approx(dt * cp.al_s);
                const float r2 = rr * rr, r4 = r2 * r2;
                r9 = (r4 * r4) * rr;
            }
            S.pre[r][c] = make_float4(dt, rr, r9, sig);
            if (adjoint) {
                S.tz[r][c] = lz[q];
                S.tdy[r][c] = ly[q];
            }
        }
    }
}

// One forward step (row r of the segment) of this thread's half-channel:
// h ← a h + Δ B u.
template <typename IO, bool FAST, bool STRUCT>
__device__ __forceinline__ void fwd_step(const BwdSmem<IO>& S, const BwdChan& cp, int r, float (&h)[kBH]) {
    const float4 pr = S.pre[r][cp.c];
    const float du = pr.x * to_f32(S.tu[r][cp.c]);
    float a[kBH];
    decays<FAST, STRUCT>(pr, cp, a);
    const float4* Bq = reinterpret_cast<const float4*>(&S.bc[r][kBH * cp.p]);
    const float4 b0 = Bq[0], b1 = Bq[1];
    const float Bh[kBH] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
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

// One adjoint step (row r of the segment): given h_t (hc) and h_{t-1}
// (hprev), advances g from ∂J/∂h_t to ∂J/∂h_{t-1} and emits every gradient
// of step t.
// i is the step's (b, t, channel) element index; dst its dB or dC entry for
// this lane's value of the transpose.
template <typename IO, bool FAST, bool STRUCT, bool HZ>
__device__ __forceinline__ void adjoint_step(BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int r,
                                             int64_t i, float* dst, const float (&hc)[kBH],
                                             const float (&hprev)[kBH], float (&g)[kBH], float (&dA_acc)[kBH],
                                             float& dD_acc, float& dbias_acc) {
    const int lane = threadIdx.x & 31;
    const int hp = kBH * cp.p;
    // Both threads of a channel hold the same per-channel outputs (their sums
    // over the two halves commute exactly) and both store them: the same value
    // to the same address, without a divergent branch.
    const bool writer = cp.valid;
    const float4 pr = S.pre[r][cp.c];
    const float dt = pr.x, sig = pr.w;
    const float uv = to_f32(S.tu[r][cp.c]);
    const float dyv = to_f32(S.tdy[r][cp.c]);
    float a[kBH];
    decays<FAST, STRUCT>(pr, cp, a);
    const float4* Bq = reinterpret_cast<const float4*>(&S.bc[r][hp]);
    const float4* Cq = reinterpret_cast<const float4*>(&S.bc[r][kN + hp]);
    const float4 b0 = Bq[0], b1 = Bq[1], c0 = Cq[0], c1 = Cq[1];
    const float Bh[kBH] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    const float Ch[kBH] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};

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
    const float dtu = dt * uv;
    // Per state: g' = g + ds C; dC += ds h_t; dB += g' Δ u; du gets Δ Σ g' B;
    // dΔ gets Σ g' a h_{t-1} A + u Σ g' B; dA += Δ g' a h_{t-1}; g ← a g'.
    f32x2 gB = pk2(0.0f, 0.0f), gahA = pk2(0.0f, 0.0f);
    float red[2 * kBH];
#pragma unroll
    for (int m = 0; m < kBH; m += 2) {
        const f32x2 a2 = pk2(a[m], a[m + 1]);
        f32x2 g2 = fma2(pk2(ds, ds), pk2(Ch[m], Ch[m + 1]), pk2(g[m], g[m + 1]));
        const f32x2 rc = mul2(pk2(ds, ds), pk2(hc[m], hc[m + 1]));
        const f32x2 rb = mul2(g2, pk2(dtu, dtu));
        gB = fma2(g2, pk2(Bh[m], Bh[m + 1]), gB);
        const f32x2 gah = mul2(g2, mul2(a2, pk2(hprev[m], hprev[m + 1])));
        gahA = fma2(gah, pk2(cp.A[m], cp.A[m + 1]), gahA);
        const f32x2 da = fma2(pk2(dt, dt), gah, pk2(dA_acc[m], dA_acc[m + 1]));
        g2 = mul2(g2, a2);
        g[m] = g2.x; g[m + 1] = g2.y;
        dA_acc[m] = da.x; dA_acc[m + 1] = da.y;
        red[m] = rb.x; red[m + 1] = rb.y;
        red[kBH + m] = rc.x; red[kBH + m + 1] = rc.y;
    }
    const float gBs = gB.x + gB.y;
    const float du_h = dt * gBs;
    const float dD_h = fmaf(uv, gBs, gahA.x + gahA.y);
    const float duv = fmaf(ds, cp.Dv, du_h + partner(du_h));
    const float dx = (dD_h + partner(dD_h)) * sig;
    dbias_acc += dx;
    if (writer) {
        static_cast<IO*>(p.du)[i] = from_f32<IO>(duv);
        static_cast<IO*>(p.ddelta)[i] = from_f32<IO>(dx);
    }
    // dB / dC summed over the half-warp's 16 channels through the warp's
    // transpose buffer: row j holds value j of all 32 lanes; lane j of half p
    // then reads the 16 entries of its half in row j.
    float* R = &S.red[threadIdx.x >> 5][0][0];
    __syncwarp();
#pragma unroll
    for (int jv = 0; jv < 2 * kBH; ++jv) R[jv * kRedRow + lane] = red[jv];
    __syncwarp();
    const int j16 = lane & 15;
    const float4* q = reinterpret_cast<const float4*>(R + j16 * kRedRow + (lane >> 4) * 16);
    const float4 v0 = q[0], v1 = q[1], v2 = q[2], v3 = q[3];
    const f32x2 s01 = add2(add2(pk2(v0.x, v0.y), pk2(v0.z, v0.w)), add2(pk2(v1.x, v1.y), pk2(v1.z, v1.w)));
    const f32x2 s23 = add2(add2(pk2(v2.x, v2.y), pk2(v2.z, v2.w)), add2(pk2(v3.x, v3.y), pk2(v3.z, v3.w)));
    const f32x2 sum = add2(s01, s23);
    atomicAdd(dst, sum.x + sum.y);
}

// exp(A_n S) for this thread's 8 states (S a sum of Δ).
template <bool FAST>
__device__ __forceinline__ float decay_over(const BwdChan& cp, int m, float Ssum) {
    return FAST ? ex2_approx(Ssum * cp.Al[m]) : expf(Ssum * cp.A[m]);
}

// Starts the copies of segment (t0, nt) into raw buffer `buf`: Δraw and u
// (forward) or Δraw, z, dy (adjoint-only), and B or C.  Rows past nt and
// channels past d are zero-filled.  With unaligned rows (vec = 0) the
// channel tiles are loaded and stored synchronously instead.
template <typename IO, bool ADJ>
__device__ __forceinline__ void chunk_issue(ChunkSmem<IO>& S, int buf, const BwdParams& p, int b, int blk,
                                            int64_t t0, int nt) {
    constexpr int kPer = 16 / static_cast<int>(sizeof(IO));   // elements per 16-byte copy
    constexpr int kCpr = kBwdCh / kPer;                       // copies per tile row
    constexpr int kArr = ADJ ? 3 : 2;
    const int64_t c0 = static_cast<int64_t>(blk) * kBwdCh;
    const IO* src0 = static_cast<const IO*>(p.delta);
    const IO* src1 = ADJ ? static_cast<const IO*>(p.z) : static_cast<const IO*>(p.u);
    const IO* src2 = static_cast<const IO*>(p.dy);
    const int64_t row0 = static_cast<int64_t>(b) * p.L + t0;
    if (p.vec) {
        for (int i = threadIdx.x; i < kArr * kSeg * kCpr; i += kBwdThreads) {
            const int a = i / (kSeg * kCpr), rem = i % (kSeg * kCpr);
            const int r = rem / kCpr, j = rem % kCpr;
            const int64_t ch = c0 + static_cast<int64_t>(j) * kPer;
            const IO* base = a == 0 ? src0 : (a == 1 ? src1 : src2);
            const int64_t nval = p.d - ch;
            const uint32_t bytes = (r < nt && base && nval > 0)
                                       ? static_cast<uint32_t>(min(nval, static_cast<int64_t>(kPer)) * sizeof(IO))
                                       : 0u;
            const IO* g = bytes ? base + (row0 + r) * p.d + ch : static_cast<const IO*>(p.delta);
            cp_async16_n(&S.raw[buf][a][r][j * kPer], g, bytes);
        }
    } else {
        const IO zero = from_f32<IO>(0.0f);
        for (int i = threadIdx.x; i < kArr * kSeg * kBwdCh; i += kBwdThreads) {
            const int a = i / (kSeg * kBwdCh), rem = i % (kSeg * kBwdCh);
            const int r = rem / kBwdCh, c = rem % kBwdCh;
            const int64_t ch = c0 + c;
            const IO* base = a == 0 ? src0 : (a == 1 ? src1 : src2);
            S.raw[buf][a][r][c] = (r < nt && base && ch < p.d) ? base[(row0 + r) * p.d + ch] : zero;
        }
    }
    const IO* bsrc = ADJ ? static_cast<const IO*>(p.C) : static_cast<const IO*>(p.B);
    constexpr int kCb = kN / kPer;
    for (int i = threadIdx.x; i < kSeg * kCb; i += kBwdThreads) {
        const int r = i / kCb, j = i % kCb;
        const bool in = r < nt;
        const IO* g = in ? bsrc + (row0 + r) * kN + j * kPer : bsrc;
        cp_async16_n(&S.rbc[buf][r][j * kPer], g, in ? 16u : 0u);
    }
}

// Per-(step, channel) scalars of a staged segment: Δ, the decay bases, and
// Δu (forward) or ds = dy · gate(z) (adjoint-only); B or C widened to fp32.
template <typename IO, bool FAST, bool STRUCT, bool SP, bool HZ, bool ADJ>
__device__ __forceinline__ void chunk_prep(ChunkSmem<IO>& S, int buf, const BwdChan& cp, int nt) {
    const int c = threadIdx.x % kBwdCh;
#pragma unroll 4
    for (int r = threadIdx.x / kBwdCh; r < nt; r += kBwdThreads / kBwdCh) {
        const float x = to_f32(S.raw[buf][0][r][c]) + cp.bias_s;
        float dt = x, sig;
        if (SP) softplus_and_sigmoid<FAST>(x, dt, sig);
        float rr = 0.0f, r9 = 0.0f;
        if (STRUCT) {
            rr = ex2_approx(dt * cp.al_s);
            const float r2 = rr * rr, r4 = r2 * r2;
            r9 = (r4 * r4) * rr;
        }
        float v;
        if (!ADJ) {
            v = dt * to_f32(S.raw[buf][1][r][c]);
        } else {
            v = to_f32(S.raw[buf][2][r][c]);
            if (HZ) {
                const float zv = to_f32(S.raw[buf][1][r][c]);
                const float sz = FAST ? rcp_approx(1.0f + ex2_approx(-zv * kLog2e)) : 1.0f / (1.0f + expf(-zv));
                v *= zv * sz;
            }
        }
        S.pre[r][c] = make_float4(v, rr, r9, dt);
    }
    for (int i = threadIdx.x; i < nt * kN; i += kBwdThreads) S.bc[i / kN][i % kN] = to_f32(S.rbc[buf][i / kN][i % kN]);
}

// One pass of the chunk kernel over segments s0 .. s1-1: forward in time
// from v = h (writing the local checkpoints and their Σ Δ), or (ADJ)
// backward in time from v = g with g ← exp(Δ A)(g + ds C).
template <typename IO, bool FAST, bool STRUCT, bool SP, bool HZ, bool ADJ>
__device__ __forceinline__ void chunk_pass(ChunkSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                           int ch, int s0, int s1, float (&v)[kBH], float& Ssum) {
    const int hp = kBH * cp.p;
    const int n = s1 - s0;
    int buf = 0;
    {
        const int seg = ADJ ? s1 - 1 : s0;
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        chunk_issue<IO, ADJ>(S, 0, p, b, blk, t0, static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0)));
        cp_async_commit();
    }
    for (int i = 0; i < n; ++i, buf ^= 1) {
        const int seg = ADJ ? s1 - 1 - i : s0 + i;
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        const int nt = static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0));
        if (!ADJ && cp.valid) {
            const int64_t ci = (static_cast<int64_t>(b) * p.nseg + seg) * p.d + ch;
            float4* ck = reinterpret_cast<float4*>(p.ckpt + ci * kN + hp);
            ck[0] = make_float4(v[0], v[1], v[2], v[3]);
            ck[1] = make_float4(v[4], v[5], v[6], v[7]);
            if (cp.p == 0) p.sck[ci] = Ssum;
        }
        cp_async_wait_all();
        __syncthreads();   // the segment's tiles have landed; the previous steps are done with pre / bc
        chunk_prep<IO, FAST, STRUCT, SP, HZ, ADJ>(S, buf, cp, nt);
        if (i + 1 < n) {
            const int sn = ADJ ? seg - 1 : seg + 1;
            const int64_t tn = static_cast<int64_t>(sn) * kSeg;
            chunk_issue<IO, ADJ>(S, buf ^ 1, p, b, blk, tn, static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - tn)));
        }
        cp_async_commit();
        __syncthreads();   // pre / bc visible
        if (!ADJ) {
#pragma unroll 8
            for (int r = 0; r < nt; ++r) {
                const float4 pr = S.pre[r][cp.c];
                float a[kBH];
                decays<FAST, STRUCT>(make_float4(pr.w, pr.y, pr.z, 0.0f), cp, a);
                const float4* Bq = reinterpret_cast<const float4*>(&S.bc[r][hp]);
                const float4 b0 = Bq[0], b1 = Bq[1];
                const float Bh[kBH] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int m = 0; m < kBH; m += 2) {
                    const f32x2 hn = fma2(pk2(a[m], a[m + 1]), pk2(v[m], v[m + 1]),
                                          mul2(pk2(pr.x, pr.x), pk2(Bh[m], Bh[m + 1])));
                    v[m] = hn.x;
                    v[m + 1] = hn.y;
                }
                Ssum += pr.w;
            }
        } else {
#pragma unroll 8
            for (int r = nt - 1; r >= 0; --r) {
                const float4 pr = S.pre[r][cp.c];
                float a[kBH];
                decays<FAST, STRUCT>(make_float4(pr.w, pr.y, pr.z, 0.0f), cp, a);
                const float4* Cq = reinterpret_cast<const float4*>(&S.bc[r][hp]);
                const float4 c0 = Cq[0], c1 = Cq[1];
                const float Ch[kBH] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int m = 0; m < kBH; m += 2) {
                    const f32x2 gn = mul2(pk2(a[m], a[m + 1]),
                                          fma2(pk2(pr.x, pr.x), pk2(Ch[m], Ch[m + 1]), pk2(v[m], v[m + 1])));
                    v[m] = gn.x;
                    v[m + 1] = gn.y;
                }
            }
        }
    }
}

// The chunk pass of one item (see the file comment).
template <typename IO, bool STRUCT, bool SP, bool HZ>
__device__ __forceinline__ void chunk_item(ChunkSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                           int k, int ch) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int hp = kBH * cp.p;
    const int s0 = k * p.cseg, s1 = min(s0 + p.cseg, p.nseg);
    const int64_t rec = (static_cast<int64_t>(b) * p.nchunk + k) * p.d + ch;   // chunk record index
    float h[kBH];
#pragma unroll
    for (int m = 0; m < kBH; ++m) h[m] = 0.0f;
    float Ssum = 0.0f;
    chunk_pass<IO, FAST, STRUCT, SP, HZ, false>(S, p, cp, b, blk, ch, s0, s1, h, Ssum);
    if (cp.valid) {
        float4* hl = reinterpret_cast<float4*>(p.hloc + rec * kN + hp);
        hl[0] = make_float4(h[0], h[1], h[2], h[3]);
        hl[1] = make_float4(h[4], h[5], h[6], h[7]);
        if (cp.p == 0) p.send[rec] = Ssum;
    }
    if (k == 0) return;   // the first chunk's g_loc is never used
    float g[kBH];
#pragma unroll
    for (int m = 0; m < kBH; ++m) g[m] = 0.0f;
    float unused = 0.0f;
    chunk_pass<IO, FAST, STRUCT, SP, HZ, true>(S, p, cp, b, blk, ch, s0, s1, g, unused);
    if (cp.valid) {
        float4* gl = reinterpret_cast<float4*>(p.gloc + rec * kN + hp);
        gl[0] = make_float4(g[0], g[1], g[2], g[3]);
        gl[1] = make_float4(g[4], g[5], g[6], g[7]);
    }
}

// The gradient pass of one item (see the file comment).
template <typename IO, bool STRUCT, bool SP, bool HZ>
__device__ __forceinline__ void bwd_item(BwdSmem<IO>& S, const BwdParams& p, const BwdChan& cp, int b, int blk,
                                         int k, int ch) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    const int64_t d = p.d;
    const int64_t row0 = static_cast<int64_t>(b) * p.L;   // (b, t) row index base
    const int hp = kBH * cp.p;
    const int s0 = k * p.cseg, s1 = min(s0 + p.cseg, p.nseg);

    // entering state and adjoint of the chunk (the records after the fold)
    float hin[kBH], g[kBH], dA_acc[kBH];
    const int64_t rec = (static_cast<int64_t>(b) * p.nchunk + k) * d + ch;
#pragma unroll
    for (int m = 0; m < kBH; ++m) {
        hin[m] = cp.valid ? p.hloc[rec * kN + hp + m] : 0.0f;
        g[m] = cp.valid ? p.gloc[rec * kN + hp + m] : 0.0f;
        dA_acc[m] = 0.0f;
    }
    float h[kBH];
    float dD_acc = 0.0f, dbias_acc = 0.0f;
    for (int seg = s1 - 1; seg >= s0; --seg) {
        const int64_t t0 = static_cast<int64_t>(seg) * kSeg;
        const int nt = static_cast<int>(min(static_cast<int64_t>(kSeg), p.L - t0));
        const int nsub = (nt + kSub - 1) / kSub;
        __syncthreads();
        load_seg<IO, FAST, STRUCT, SP>(S, p, cp, b, blk, t0, nt, true);
        __syncthreads();
        if (cp.valid) {
            const int64_t ci = (static_cast<int64_t>(b) * p.nseg + seg) * d + ch;
            const float4* ck = reinterpret_cast<const float4*>(p.ckpt + ci * kN + hp);
            const float4 v0 = ck[0], v1 = ck[1];
            h[0] = v0.x; h[1] = v0.y; h[2] = v0.z; h[3] = v0.w;
            h[4] = v1.x; h[5] = v1.y; h[6] = v1.z; h[7] = v1.w;
            if (k > 0) {   // the local checkpoint plus the carried-in state decayed to it
                const float Ss = p.sck[ci];
#pragma unroll
                for (int m = 0; m < kBH; ++m) h[m] = fmaf(decay_over<FAST>(cp, m, Ss), hin[m], h[m]);
            }
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
            for (int j = 0; j < kSub; ++j) fwd_step<IO, FAST, STRUCT>(S, cp, s * kSub + j, h);
        }
        for (int s = nsub - 1; s >= 0; --s) {
            const int ns = min(kSub, nt - s * kSub);   // uniform over the CTA
            float hs[kSub][kBH];                        // h_t of the sub-segment's steps, in registers
            // element index and dB / dC entry of the sub-segment's first step
            const int64_t rs = row0 + t0 + s * kSub;
            const int64_t ib = rs * d + ch;
            float* dstb = ((threadIdx.x & 15) < kBH ? p.dB : p.dC) + rs * kN + kBH * ((threadIdx.x >> 4) & 1) +
                          (threadIdx.x & (kBH - 1));
            load_state(S.hsub[s], cp, h);
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                if (j < ns) fwd_step<IO, FAST, STRUCT>(S, cp, s * kSub + j, h);
#pragma unroll
                for (int m = 0; m < kBH; ++m) hs[j][m] = h[m];
            }
#pragma unroll
            for (int j = kSub - 1; j >= 0; --j) {
                if (j >= ns) continue;
                float hprev[kBH];
                if (j > 0) {
#pragma unroll
                    for (int m = 0; m < kBH; ++m) hprev[m] = hs[j - 1][m];
                } else {
                    load_state(S.hsub[s], cp, hprev);
                }
                adjoint_step<IO, FAST, STRUCT, HZ>(S, p, cp, s * kSub + j, ib + static_cast<int64_t>(j) * p.d,
                                                   dstb + j * kN, hs[j], hprev, g, dA_acc, dD_acc, dbias_acc);
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

// Between the two passes: one thread per (batch, channel, state) folds the
// chunk records in order, replacing h_loc(k) by the exact state entering
// chunk k and g_loc(k) by the exact adjoint at chunk k's end (dlast_state
// for the last chunk); P_k = exp(A Σ_{chunk k} Δ).
__global__ void __launch_bounds__(256) ss_bwd_combine_kernel(const __grid_constant__ BwdParams p) {
    const int64_t total = static_cast<int64_t>(p.batch) * p.d * kN;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(i % kN);
        const int64_t bc = i / kN;   // b * d + ch
        const int64_t b = bc / p.d, ch = bc % p.d;
        const float An = p.A[ch * kN + n];
        float h = 0.0f;
        for (int k = 0; k < p.nchunk; ++k) {
            const int64_t rec = (b * p.nchunk + k) * p.d + ch;
            const float hl = p.hloc[rec * kN + n];
            p.hloc[rec * kN + n] = h;
            h = k ? fmaf(expf(An * p.send[rec]), h, hl) : hl;
        }
        float g = p.dlast ? p.dlast[bc * kN + n] : 0.0f;
        for (int k = p.nchunk - 1; k >= 0; --k) {
            const int64_t rec = (b * p.nchunk + k) * p.d + ch;
            if (k == 0) {
                p.gloc[rec * kN + n] = g;
                break;
            }
            const float gl = p.gloc[rec * kN + n];
            p.gloc[rec * kN + n] = g;
            g = fmaf(expf(An * p.send[rec]), g, gl);
        }
    }
}

// Per-thread constants for channel blk * kBwdCh + cp.c; returns whether every
// channel of the block has the structured A (A[d, n] = a (n + 1)).
__device__ __forceinline__ bool init_chan(const BwdParams& p, int blk, BwdChan& cp, int& ch) {
    const int lane = threadIdx.x & 31;
    cp.c = (threadIdx.x >> 5) * 16 + (lane & 15);
    cp.p = lane >> 4;
    ch = blk * kBwdCh + cp.c;
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
    cp.bias = (cp.valid && p.bias) ? p.bias[ch] : 0.0f;
    {
        const int cs = blk * kBwdCh + static_cast<int>(threadIdx.x % kBwdCh);   // channel this thread stages
        const bool vs = cs < p.d;
        cp.al_s = (vs ? p.A[static_cast<int64_t>(cs) * kN] : -1.0f) * kLog2e;
        cp.bias_s = (vs && p.bias) ? p.bias[cs] : 0.0f;
    }
    cp.Dv = (cp.valid && p.D) ? p.D[ch] : 0.0f;
    return __syncthreads_and(structured ? 1 : 0) != 0;
}

// Grid of both kernels: one CTA per item, chunk-major
// (blockIdx.x = (k * batch + b) * nblk + blk).
// SP: Δ goes through softplus; HZ: the silu(z) gate is on.
template <typename IO, bool SP, bool HZ>
__global__ void __launch_bounds__(kBwdThreads, 3) ss_bwd_chunk_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ __align__(16) unsigned char bwd_smem_raw[];
    auto& S = *reinterpret_cast<ChunkSmem<IO>*>(bwd_smem_raw);
    const int blk = blockIdx.x % p.nblk;
    const int b = (blockIdx.x / p.nblk) % p.batch;
    const int k = blockIdx.x / (p.nblk * p.batch);
    BwdChan cp;
    int ch;
    const bool all_struct = init_chan(p, blk, cp, ch);
    if (std::is_same<IO, __nv_bfloat16>::value && all_struct)
        chunk_item<IO, true, SP, HZ>(S, p, cp, b, blk, k, ch);
    else
        chunk_item<IO, false, SP, HZ>(S, p, cp, b, blk, k, ch);
}

template <typename IO, bool SP, bool HZ>
__global__ void __launch_bounds__(kBwdThreads, 3) ss_bwd_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ __align__(16) unsigned char bwd_smem_raw[];
    auto& S = *reinterpret_cast<BwdSmem<IO>*>(bwd_smem_raw);
    const int blk = blockIdx.x % p.nblk;
    const int b = (blockIdx.x / p.nblk) % p.batch;
    const int k = blockIdx.x / (p.nblk * p.batch);
    BwdChan cp;
    int ch;
    const bool all_struct = init_chan(p, blk, cp, ch);
    if (std::is_same<IO, __nv_bfloat16>::value && all_struct)
        bwd_item<IO, true, SP, HZ>(S, p, cp, b, blk, k, ch);
    else
        bwd_item<IO, false, SP, HZ>(S, p, cp, b, blk, k, ch);
}

}  // namespace selscan
