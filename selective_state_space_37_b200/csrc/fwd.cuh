// fwd.cuh -- selective-scan forward kernel for sm_100a.
//
// Computes, per (batch b, channel ch), the selective recurrence of
// "Understanding Mamba and Selective State Space Models (SSMs)" §2.2 (first
// cut) with the readout of §3.1 and the skip term of §2.1:
//     Δ_t   = softplus(Δraw_t + bias)                         (§2.2 closing tip)
//     h_t,n = exp(Δ_t A_n) h_{t-1},n + Δ_t B_t,n u_t          (§2.2 first cut)
//     y_t   = (Σ_n C_t,n h_t,n + D u_t) · z_t σ(z_t)
// starting from h = 0 (§2.2 second cut), A diagonal (§4.3).
//
// Work decomposition
//   One CTA = one work item = (batch b, time chunk c, block of kCB channels).
//   Two threads share a channel: lanes l and l^16 of a warp, each keeping
//   kHalf of the kN fp32 states in registers (as packed fp32x2 pairs) for the
//   whole chunk, so one warp serves 16 channels.  Splitting the state gives
//   each scheduler two warps' worth of independent instructions for the same
//   number of channels, without cutting time into more chunks.
//   Tiles of kTT timesteps of u / Δraw / z ([kTT x kCB]) and of B / C
//   ([kTT x kN], shared by every channel) arrive in shared memory by TMA
//   (cp.async.bulk.tensor, no multicast) through a ring of STAGES buffers
//   completed on mbarriers; B and C are widened to fp32 once per tile.
//
// Per thread pair, timesteps go in groups of G: each thread computes the
//   per-step scalars (Δ, Δu, Du, gate) of half the group's steps, the pair
//   swaps Δ and Δu by shuffle, both threads advance their half-states through
//   all G steps in order, and each thread finishes the outputs of the steps
//   it prepared after one shuffle of the partial readouts.
//
// Time chunking (the recurrence is linear, so a chunk maps its entry state h0
//   to P ⊙ h0 + h_loc with P = Π exp(Δ A)):
//   Items take tickets from a global counter in chunk-major order.  An item
//   whose predecessor chunk has already published its inclusive end state
//   starts from it and is exact at once.  Otherwise it scans from zero
//   (writing provisional outputs), publishes its aggregate (P, h_loc), looks
//   back through its predecessors' aggregates to the nearest inclusive state
//   (decoupled look-back; every wait is bounded), publishes its own inclusive
//   state, then re-streams Δraw, z and its provisional y through the same TMA
//   ring and adds (Σ_n C_t,n P_t,n h0_n) · gate_t to each output.  Tickets are
//   taken in start order, so an item only ever waits on items that are
//   already running, and those publish before they wait.
//
// Units on the bf16 path: Δ is carried as λ = Δ / ln 2, so the decay is
//   2^(λ A), Δ·B·u = λ·(ln 2·B)·u (ln 2 folded into B once per tile), and the
//   softplus input is formed by one fused multiply-add.
//
// A = a_d (n+1) fast path (bf16 I/O): exp(Δ a_d (n+1)) = r^(n+1).  A thread
//   gets its first decay r^(8p+1) and r from the hardware exp and the rest of
//   its eight by a product ladder on pairs.  Detected per CTA with an exact
//   test on A.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace selscan {

constexpr int kN = 16;      // d_state
constexpr int kHalf = 8;    // states per thread
constexpr int kTT = 32;     // timesteps per tile
constexpr int kCB = 128;    // channels per CTA (two threads per channel)
constexpr int kNT = 2 * kCB;        // threads per CTA
constexpr int kRec = 48;    // floats per carry record: P[16], h_loc[16], inclusive[16]
constexpr int kConvW = 4;   // width of the causal conv1d prologue (d_conv)
constexpr int kHalo = kConvW - 1;   // rows of x the conv needs before a tile
static_assert(kNT == 2 * kCB, "two threads per channel");

enum : uint32_t { kStNone = 0, kStAgg = 1, kStIncl = 2, kStTimeout = 0xFFFFFFFFu };
enum : uint32_t {
    kPfSoftplus = 1u,
    kPfForceGeneral = 2u,
    kPfTestDrop = 4u,
    kPfHasZ = 8u,
    kPfHasBias = 16u,
    kPfHasD = 32u,
    kPfConv = 64u
};

struct FwdParams {
    const void* u;
    const void* delta;
    const float* bias;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    void* y;
    float* last_state;
    const float* h_init;   // [batch][d][kN] state entering the sequence, or null (zero)
    const float* conv_w;   // [d, kConvW] (conv prologue only)
    const float* conv_b;   // [d] or null
    int64_t L;
    int batch, d, chunk_len, nchunks, nblk;
    uint32_t pflags;
    uint32_t* hdr;       // [0]: error status (negative code as uint32), [1]: ticket counter,
                         // [2]: number of provisional items (diagnostic)
    uint32_t* status;    // [batch][nchunks][nblk] publication state of each item
    float* rec;          // [batch][nchunks][d][kRec] carry records
    uint64_t wait_ns;    // bound on one TMA completion wait
    uint32_t poll_limit; // bound on the polls of one carry wait
};

template <typename IO, int STAGES>
struct FwdSmem {
    // Rows kHalo.. hold u (scan pass) or the provisional y (fix-up pass); with
    // the conv prologue the scan pass fills rows 0.. with x from t0 - kHalo.
    IO a[STAGES][kHalo + kTT][kCB];
    IO dt[STAGES][kTT][kCB];
    IO z[STAGES][kTT][kCB];
    IO B[STAGES][kTT][kN];
    IO C[STAGES][kTT][kN];
    float bc[STAGES][kTT][2 * kN];   // per timestep: B (scaled to the λ units) then C, fp32
    uint64_t full[STAGES];
    int item;
    uint32_t st;
};

__device__ __forceinline__ void record_error(uint32_t* hdr, int code) {
    atomicCAS(&hdr[0], 0u, static_cast<uint32_t>(code));
}

// Value held by the other thread of this channel (lane ^ 16).
__device__ __forceinline__ float partner(float v) { return __shfl_xor_sync(0xffffffffu, v, 16); }

// λ for one element: Δ/ln 2 on the fast path (bias_s = bias·log2 e), Δ itself
// on the accurate path (bias_s = bias).  sp_mask selects the softplus.
template <bool FAST>
__device__ __forceinline__ float lam_of(float xraw, float bias_s, uint32_t sp_mask) {
    if (FAST) {
        const float y2 = fmaf(xraw, kLog2e, bias_s);
        return blend(sp_mask, softplus_log2_fast(y2), y2);
    }
    const float x = xraw + bias_s;
    return blend(sp_mask, softplus_accurate(x), x);
}

template <bool FAST>
__device__ __forceinline__ float gate_of(float zv) {
    return FAST ? silu_tanh(zv) : silu_accurate(zv);
}

// exp(Δ A) from λ and raw A.
template <bool FAST>
__device__ __forceinline__ float decay_of(float lam, float a) {
    return FAST ? ex2_approx(lam * a) : expf(lam * a);
}

struct ChanParams {
    float Av[kHalf];   // raw A of this thread's states 8p .. 8p+7
    float a;           // A[ch, 0]; on the structured path A[ch, n] = a (n + 1)
    float ab;          // a (8p + 1): exponent factor of this half's first decay
    float kq;          // 8p + 1: the power of r of this half's first decay
    float bias_s;      // bias in the softplus input's scale
    float Dv;
    uint32_t sp_mask;  // all ones: Δ goes through softplus
    uint32_t z_mask;   // all ones: the silu(z) gate is on
    uint32_t hi_mask;  // all ones on the thread holding the upper half (p = 1)
    int p;             // 0: states 0..7, 1: states 8..15
    bool valid;        // channel < d_inner
    float cw[kConvW];  // conv prologue weights (oldest tap first) and bias
    float cb;
};

// The scan's input u at tile row j.  xs points at row 0 of this channel's
// column of the tile.  Without the prologue u sits at row kHalo + j; with it,
// u = silu(cb + Σ_k cw[k] x_{t-3+k}) ("Understanding Mamba and Selective
// State Space Models (SSMs)" §3.3: causal conv of width 4 before the SSM)
// from rows j .. j+3, which hold x from t0 - 3 (zeros before the sequence).
template <typename IO, bool FAST, bool CONV>
__device__ __forceinline__ float u_at(const IO* __restrict__ xs, int j, const ChanParams& cp) {
    if (!CONV) return to_f32(xs[(j + kHalo) * kCB]);
    float c = cp.cb;
#pragma unroll
    for (int k = 0; k < kConvW; ++k) c = fmaf(cp.cw[k], to_f32(xs[(j + k) * kCB]), c);
    return FAST ? silu_tanh(c) : silu_accurate(c);
}

// Decays of this thread's eight states as pairs, for the structured path:
// (r^(8p+1), r^(8p+2)), ..., (r^(8p+7), r^(8p+8)) from base = r^(8p+1).
__device__ __forceinline__ void half_ladder(float base, float r, f32x2 (&Q)[4]) {
    const float r2 = r * r;
    const f32x2 R2 = pk2(r2, r2);
    Q[0] = pk2(base, base * r);
    Q[1] = mul2(Q[0], R2);
    Q[2] = mul2(Q[1], R2);
    Q[3] = mul2(Q[2], R2);
}

// Loads this thread's four B pairs and four C pairs of one timestep row.
__device__ __forceinline__ void load_bc(const float* __restrict__ bcrow, int p, f32x2 (&Bp)[4], f32x2 (&Cp)[4]) {
    const float4* q = reinterpret_cast<const float4*>(bcrow + kHalf * p);
    const float4 b0 = q[0], b1 = q[1];
    const float4 c0 = q[4], c1 = q[5];
    Bp[0] = pk2(b0.x, b0.y); Bp[1] = pk2(b0.z, b0.w); Bp[2] = pk2(b1.x, b1.y); Bp[3] = pk2(b1.z, b1.w);
    Cp[0] = pk2(c0.x, c0.y); Cp[1] = pk2(c0.z, c0.w); Cp[2] = pk2(c1.x, c1.y); Cp[3] = pk2(c1.z, c1.w);
}
__device__ __forceinline__ void load_c(const float* __restrict__ bcrow, int p, f32x2 (&Cp)[4]) {
    const float4* q = reinterpret_cast<const float4*>(bcrow + kN + kHalf * p);
    const float4 c0 = q[0], c1 = q[1];
    Cp[0] = pk2(c0.x, c0.y); Cp[1] = pk2(c0.z, c0.w); Cp[2] = pk2(c1.x, c1.y); Cp[3] = pk2(c1.z, c1.w);
}

// This thread's half of the readout Σ_n C_n h_n: one chain of packed
// products (even and odd states), then the two lanes' sum.
__device__ __forceinline__ float half_dot(const f32x2 (&Cp)[4], const f32x2 (&H)[4]) {
    f32x2 a = mul2(Cp[0], H[0]);
    a = fma2(Cp[1], H[1], a);
    a = fma2(Cp[2], H[2], a);
    a = fma2(Cp[3], H[3], a);
    float lo, hi;
    upk2(a, lo, hi);
    return lo + hi;
}

// One state update of this thread's half for one timestep.  Structured A:
// lam is λ a (r = 2^(λ a)); otherwise λ.
template <bool FAST, bool STRUCT, bool TRACK>
__device__ __forceinline__ void half_update(float lam, float du, const f32x2 (&Bp)[4], f32x2 (&H)[4],
                                            f32x2 (&PP)[4], float& R, const ChanParams& cp) {
    const f32x2 DU = pk2(du, du);
    if (STRUCT) {
        const float r = ex2_approx(lam);
        f32x2 Q[4];
        half_ladder(ex2_approx(lam * cp.kq), r, Q);
#pragma unroll
        for (int m = 0; m < 4; ++m) H[m] = fma2(Q[m], H[m], mul2(DU, Bp[m]));
        if (TRACK) R *= r;
    } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const f32x2 P = pk2(decay_of<FAST>(lam, cp.Av[2 * m]), decay_of<FAST>(lam, cp.Av[2 * m + 1]));
            H[m] = fma2(P, H[m], mul2(DU, Bp[m]));
            if (TRACK) PP[m] = mul2(PP[m], P);
        }
    }
}

// A group of NSTEP (even) timesteps of the scan, rows j0 .. j0+NSTEP-1.
// us/dts/zs point at this channel's column of the tile (row 0); yrow at this
// channel's output for row 0 of the tile.  FULL: softplus and gate both on
// (known at compile time).
template <typename IO, bool FAST, bool STRUCT, bool TRACK, int NSTEP, bool CONV, bool FULL>
__device__ __forceinline__ void scan_group(const IO* __restrict__ us, const IO* __restrict__ dts,
                                           const IO* __restrict__ zs, const float* __restrict__ bc, int j0,
                                           f32x2 (&H)[4], f32x2 (&PP)[4], float& R, const ChanParams& cp,
                                           IO* __restrict__ yrow, int64_t d) {
    constexpr int NH = NSTEP / 2;
    const uint32_t spm = FULL ? 0xffffffffu : cp.sp_mask;
    const uint32_t zm = FULL ? 0xffffffffu : cp.z_mask;
    // Phase A: this thread prepares steps j0 + 2i + p (λ a on the structured path).
    float lo[NH], dlo[NH], su[NH], g[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const int row = (j0 + 2 * i + cp.p) * kCB;
        const float uu = u_at<IO, FAST, CONV>(us, j0 + 2 * i + cp.p, cp);
        const float lam = lam_of<FAST>(to_f32(dts[row]), cp.bias_s, spm);
        lo[i] = STRUCT ? lam * cp.a : lam;
        dlo[i] = lam * uu;
        su[i] = cp.Dv * uu;
        g[i] = blend(zm, gate_of<FAST>(to_f32(zs[row])), 1.0f);
    }
    float lam[NSTEP], du[NSTEP];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const float lx = partner(lo[i]);
        const float dx = partner(dlo[i]);
        lam[2 * i] = blend(cp.hi_mask, lx, lo[i]);
        lam[2 * i + 1] = blend(cp.hi_mask, lo[i], lx);
        du[2 * i] = blend(cp.hi_mask, dx, dlo[i]);
        du[2 * i + 1] = blend(cp.hi_mask, dlo[i], dx);
    }
    // Phase B: the state updates, in time order.
    float part[NSTEP];
#pragma unroll
    for (int j = 0; j < NSTEP; ++j) {
        f32x2 Bp[4], Cp[4];
        load_bc(bc + (j0 + j) * 2 * kN, cp.p, Bp, Cp);
        half_update<FAST, STRUCT, TRACK>(lam[j], du[j], Bp, H, PP, R, cp);
        part[j] = half_dot(Cp, H);
    }
    // Finish the outputs of this thread's steps: y = (lower + upper + D u) gate.
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const float send = blend(cp.hi_mask, part[2 * i], part[2 * i + 1]);
        const float mine = blend(cp.hi_mask, part[2 * i + 1], part[2 * i]);
        const float yv = (mine + partner(send) + su[i]) * g[i];
        if (cp.valid) yrow[static_cast<int64_t>(j0 + 2 * i + cp.p) * d] = from_f32<IO>(yv);
    }
}

// One timestep of the scan (ragged tails); both threads prepare it.
template <typename IO, bool FAST, bool STRUCT, bool TRACK, bool CONV, bool FULL>
__device__ __forceinline__ void scan_one(const IO* __restrict__ us, const IO* __restrict__ dts,
                                         const IO* __restrict__ zs, const float* __restrict__ bc, int j,
                                         f32x2 (&H)[4], f32x2 (&PP)[4], float& R, const ChanParams& cp,
                                         IO* __restrict__ yrow, int64_t d) {
    const int row = j * kCB;
    const float uu = u_at<IO, FAST, CONV>(us, j, cp);
    const float lam = lam_of<FAST>(to_f32(dts[row]), cp.bias_s, FULL ? 0xffffffffu : cp.sp_mask);
    const float g = blend(FULL ? 0xffffffffu : cp.z_mask, gate_of<FAST>(to_f32(zs[row])), 1.0f);
    f32x2 Bp[4], Cp[4];
    load_bc(bc + j * 2 * kN, cp.p, Bp, Cp);
    half_update<FAST, STRUCT, TRACK>(STRUCT ? lam * cp.a : lam, lam * uu, Bp, H, PP, R, cp);
    const float part = half_dot(Cp, H);
    const float yv = (part + partner(part) + cp.Dv * uu) * g;
    if (cp.valid && cp.p == 0) yrow[static_cast<int64_t>(j) * d] = from_f32<IO>(yv);
}

// This thread's half of the entry-state correction Σ_n C_n P_t,n h0_n.
template <bool FAST, bool STRUCT>
__device__ __forceinline__ float half_corr(float lam, const f32x2 (&Cp)[4], const f32x2 (&H0)[4], f32x2 (&PQ)[4],
                                           float& Rq, const ChanParams& cp) {
    f32x2 CH[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) CH[m] = mul2(Cp[m], H0[m]);
    if (STRUCT) {
        Rq *= ex2_approx(lam * cp.a);
        // Σ_m c_m Rq^(8p+1+m) = Rq^(8p+1) · Σ_k (c_2k + c_2k+1 Rq) (Rq^2)^k
        const float R2 = Rq * Rq;
        const float R8 = (R2 * R2) * (R2 * R2);
        const float base = blend(cp.hi_mask, R8 * Rq, Rq);
        float s = 0.0f;
#pragma unroll
        for (int m = 3; m >= 0; --m) {
            float c0, c1;
            upk2(CH[m], c0, c1);
            s = fmaf(s, R2, fmaf(c1, Rq, c0));
        }
        return s * base;
    } else {
        f32x2 a0 = pk2(0.0f, 0.0f), a1 = pk2(0.0f, 0.0f);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            PQ[m] = mul2(PQ[m], pk2(decay_of<FAST>(lam, cp.Av[2 * m]), decay_of<FAST>(lam, cp.Av[2 * m + 1])));
            if (m & 1) a1 = fma2(CH[m], PQ[m], a1);
            else       a0 = fma2(CH[m], PQ[m], a0);
        }
        float lo, hi;
        upk2(add2(a0, a1), lo, hi);
        return lo + hi;
    }
}

// A group of NSTEP (even) timesteps of the fix-up pass.
template <typename IO, bool FAST, bool STRUCT, int NSTEP, bool FULL>
__device__ __forceinline__ void fix_group(const IO* __restrict__ ys, const IO* __restrict__ dts,
                                          const IO* __restrict__ zs, const float* __restrict__ bc, int j0,
                                          const f32x2 (&H0)[4], f32x2 (&PQ)[4], float& Rq, const ChanParams& cp,
                                          IO* __restrict__ yrow, int64_t d) {
    constexpr int NH = NSTEP / 2;
    float lo[NH], g[NH], yo[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const int row = (j0 + 2 * i + cp.p) * kCB;
        lo[i] = lam_of<FAST>(to_f32(dts[row]), cp.bias_s, FULL ? 0xffffffffu : cp.sp_mask);
        g[i] = blend(FULL ? 0xffffffffu : cp.z_mask, gate_of<FAST>(to_f32(zs[row])), 1.0f);
        yo[i] = to_f32(ys[row]);
    }
    float lam[NSTEP];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const float lx = partner(lo[i]);
        lam[2 * i] = blend(cp.hi_mask, lx, lo[i]);
        lam[2 * i + 1] = blend(cp.hi_mask, lo[i], lx);
    }
    float part[NSTEP];
#pragma unroll
    for (int j = 0; j < NSTEP; ++j) {
        f32x2 Cp[4];
        load_c(bc + (j0 + j) * 2 * kN, cp.p, Cp);
        part[j] = half_corr<FAST, STRUCT>(lam[j], Cp, H0, PQ, Rq, cp);
    }
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const float send = blend(cp.hi_mask, part[2 * i], part[2 * i + 1]);
        const float mine = blend(cp.hi_mask, part[2 * i + 1], part[2 * i]);
        const float yv = fmaf(mine + partner(send), g[i], yo[i]);
        if (cp.valid) yrow[static_cast<int64_t>(j0 + 2 * i + cp.p) * d] = from_f32<IO>(yv);
    }
}

template <typename IO, bool FAST, bool STRUCT, bool FULL>
__device__ __forceinline__ void fix_one(const IO* __restrict__ ys, const IO* __restrict__ dts,
                                        const IO* __restrict__ zs, const float* __restrict__ bc, int j,
                                        const f32x2 (&H0)[4], f32x2 (&PQ)[4], float& Rq, const ChanParams& cp,
                                        IO* __restrict__ yrow, int64_t d) {
    const int row = j * kCB;
    const float lam = lam_of<FAST>(to_f32(dts[row]), cp.bias_s, FULL ? 0xffffffffu : cp.sp_mask);
    const float g = blend(FULL ? 0xffffffffu : cp.z_mask, gate_of<FAST>(to_f32(zs[row])), 1.0f);
    f32x2 Cp[4];
    load_c(bc + j * 2 * kN, cp.p, Cp);
    const float part = half_corr<FAST, STRUCT>(lam, Cp, H0, PQ, Rq, cp);
    const float yv = fmaf(part + partner(part), g, to_f32(ys[row]));
    if (cp.valid && cp.p == 0) yrow[static_cast<int64_t>(j) * d] = from_f32<IO>(yv);
}

// Coordinates and tile-ring plumbing of one work item.
template <typename IO, bool USE_TMA, int STAGES>
struct ItemCtx {
    const FwdParams* p;
    FwdSmem<IO, STAGES>* S;
    const CUtensorMap *tm_u, *tm_dt, *tm_z, *tm_B, *tm_C, *tm_y;
    int tid, b, c, g, ntiles;
    int cc;             // this thread's channel within the block
    int64_t t_begin, t_end, d;
    bool has_z;
    bool conv;          // the scan pass streams x (with kHalo rows before the tile) for the conv prologue
    float bscale;
    uint32_t bytes_scan, bytes_fix;

    // pass 0: u, Δraw, z, B, C;  pass 1: provisional y, Δraw, z, C
    __device__ __forceinline__ void issue(int k, int s, int pass) const {
        const int t0 = static_cast<int>(t_begin + static_cast<int64_t>(k) * kTT);
        uint64_t* bar = &S->full[s];
        mbar_arrive_expect_tx(bar, pass == 0 ? bytes_scan : bytes_fix);
        if (pass == 0 && conv) tma_load_3d(&S->a[s][0][0], tm_u, g * kCB, t0 - kHalo, b, bar);
        else tma_load_3d(&S->a[s][kHalo][0], pass == 0 ? tm_u : tm_y, g * kCB, t0, b, bar);
        tma_load_3d(&S->dt[s][0][0], tm_dt, g * kCB, t0, b, bar);
        if (has_z) tma_load_3d(&S->z[s][0][0], tm_z, g * kCB, t0, b, bar);
        if (pass == 0) tma_load_3d(&S->B[s][0][0], tm_B, 0, t0, b, bar);
        tma_load_3d(&S->C[s][0][0], tm_C, 0, t0, b, bar);
    }

    __device__ __forceinline__ void fill_plain(int k, int pass) const {
        const int64_t t0 = t_begin + static_cast<int64_t>(k) * kTT;
        const IO* ga = static_cast<const IO*>(pass == 0 ? p->u : p->y);
        const IO* gd = static_cast<const IO*>(p->delta);
        const IO* gz = static_cast<const IO*>(p->z);
        for (int i = tid; i < kTT * kCB; i += kNT) {
            const int r = i / kCB, col = i % kCB;
            const int64_t t = t0 + r;
            const int ch = g * kCB + col;
            const bool ok = (t < p->L) && (ch < p->d);
            const int64_t idx = (static_cast<int64_t>(b) * p->L + t) * d + ch;
            S->a[0][kHalo + r][col] = ok ? ga[idx] : from_f32<IO>(0.f);
            S->dt[0][r][col] = ok ? gd[idx] : from_f32<IO>(0.f);
            if (has_z) S->z[0][r][col] = ok ? gz[idx] : from_f32<IO>(0.f);
        }
        if (pass == 0 && conv) {   // x rows t0 - kHalo .. t0 - 1 (zero before the sequence)
            for (int i = tid; i < kHalo * kCB; i += kNT) {
                const int r = i / kCB, col = i % kCB;
                const int64_t t = t0 - kHalo + r;
                const int ch = g * kCB + col;
                const bool ok = (t >= 0) && (t < p->L) && (ch < p->d);
                S->a[0][r][col] = ok ? ga[(static_cast<int64_t>(b) * p->L + t) * d + ch] : from_f32<IO>(0.f);
            }
        }
        const IO* gB = static_cast<const IO*>(p->B);
        const IO* gC = static_cast<const IO*>(p->C);
        for (int i = tid; i < kTT * kN; i += kNT) {
            const int r = i / kN, n = i % kN;
            const int64_t t = t0 + r;
            const bool ok = t < p->L;
            const int64_t idx = (static_cast<int64_t>(b) * p->L + t) * kN + n;
            if (pass == 0) S->B[0][r][n] = ok ? gB[idx] : from_f32<IO>(0.f);
            S->C[0][r][n] = ok ? gC[idx] : from_f32<IO>(0.f);
        }
    }

    // Waits for (or loads) tile k of this pass -- tile number kk of the CTA --
    // widens its B/C to fp32, and refills the stage the previous tile freed.
    __device__ __forceinline__ int acquire(int k, int kk, int pass) const {
        const int s = USE_TMA ? (kk % STAGES) : 0;
        if constexpr (USE_TMA) {
            if (!mbar_wait_bounded(&S->full[s], static_cast<uint32_t>((kk / STAGES) & 1), p->wait_ns))
                record_error(p->hdr, -4);
        } else {
            __syncthreads();
            fill_plain(k, pass);
            __syncthreads();
        }
        for (int i = tid; i < kTT * kN; i += kNT) {
            const int r = i / kN, n = i % kN;
            if (pass == 0) S->bc[s][r][n] = to_f32(S->B[s][r][n]) * bscale;
            S->bc[s][r][kN + n] = to_f32(S->C[s][r][n]);
        }
        __syncthreads();
        if constexpr (USE_TMA) {
            if (tid == 0 && k >= 1 && k + STAGES - 1 < ntiles) {
                fence_proxy_async_smem();
                issue(k + STAGES - 1, (kk - 1 + STAGES) % STAGES, pass);
            }
        }
        return s;
    }
};

// The scan (and, for a provisional chunk, look-back and fix-up) of one item,
// specialised on the decay form and on whether the entry state is known.
template <typename IO, bool USE_TMA, int STAGES, int G, bool UNROLL, bool STRUCT, bool EXACT, bool CONV, bool FULL>
__device__ __forceinline__ void run_item(const ItemCtx<IO, USE_TMA, STAGES>& it, const ChanParams& cp,
                                         f32x2 (&H)[4]) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    constexpr bool TRACK = !EXACT;
    const FwdParams& p = *it.p;
    auto& S = *it.S;
    const int tid = it.tid;
    const int64_t d = it.d;
    const int hp = kHalf * cp.p;   // first state index of this thread

    f32x2 PP[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) PP[m] = pk2(1.f, 1.f);
    float R = 1.f;
    int64_t t = it.t_begin;
    IO* ybase = static_cast<IO*>(p.y) + (static_cast<int64_t>(it.b) * p.L + it.t_begin) * d + (it.g * kCB + it.cc);
    int kk = 0;   // tiles consumed so far by this CTA (both passes)

    for (int k = 0; k < it.ntiles; ++k, ++kk) {
        const int s = it.acquire(k, kk, 0);
        const int nt = static_cast<int>((it.t_end - t) < kTT ? (it.t_end - t) : kTT);
        const IO* us = &S.a[s][0][it.cc];
        const IO* dts = &S.dt[s][0][it.cc];
        const IO* zs = &S.z[s][0][it.cc];
        const float* bc = &S.bc[s][0][0];
        IO* yrow = ybase + (t - it.t_begin) * d;
        if (UNROLL && nt == kTT) {
#pragma unroll
            for (int gi = 0; gi < kTT / G; ++gi)
                scan_group<IO, FAST, STRUCT, TRACK, G, CONV, FULL>(us, dts, zs, bc, gi * G, H, PP, R, cp, yrow, d);
        } else {
            int j0 = 0;
            for (; j0 + G <= nt; j0 += G)
                scan_group<IO, FAST, STRUCT, TRACK, G, CONV, FULL>(us, dts, zs, bc, j0, H, PP, R, cp, yrow, d);
            for (; j0 < nt; ++j0) scan_one<IO, FAST, STRUCT, TRACK, CONV, FULL>(us, dts, zs, bc, j0, H, PP, R, cp, yrow, d);
        }
        t += nt;
    }

    // ------------------------------------------------------------ epilogue
    const int b = it.b, c = it.c, g = it.g;
    const int ch = g * kCB + it.cc;
    const bool last = (c == p.nchunks - 1);
    const bool drop = (p.pflags & kPfTestDrop) && b == 0 && c == 0 && g == 0;
    uint32_t* st_me = p.status + (static_cast<int64_t>(b) * p.nchunks + c) * p.nblk + g;
    float* rec_me = p.rec + ((static_cast<int64_t>(b) * p.nchunks + c) * d + ch) * kRec + hp;
    float* ls = p.last_state ? p.last_state + (static_cast<int64_t>(b) * d + ch) * kN + hp : nullptr;

    float h[kHalf];
#pragma unroll
    for (int m = 0; m < 4; ++m) upk2(H[m], h[2 * m], h[2 * m + 1]);

    if constexpr (EXACT) {
        if (!last) {
            if (cp.valid) {
#pragma unroll
                for (int n = 0; n < kHalf; ++n) __stcg(rec_me + 32 + n, h[n]);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0 && !drop) st_release_gpu(st_me, kStIncl);
        } else if (cp.valid && ls) {
#pragma unroll
            for (int n = 0; n < kHalf; ++n) ls[n] = h[n];
        }
        return;
    } else {
        // Provisional chunk: make the provisional y visible to the TMA reads
        // of the fix-up pass, then publish the aggregate (P, h_loc).
        fence_proxy_async_global();
        float P[kHalf];
        if (STRUCT) {
            const float R2 = R * R;
            const float R8 = (R2 * R2) * (R2 * R2);
            f32x2 Q[4];
            half_ladder(blend(cp.hi_mask, R8 * R, R), R, Q);
#pragma unroll
            for (int m = 0; m < 4; ++m) upk2(Q[m], P[2 * m], P[2 * m + 1]);
        } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) upk2(PP[m], P[2 * m], P[2 * m + 1]);
        }
        if (cp.valid) {
#pragma unroll
            for (int n = 0; n < kHalf; ++n) {
                __stcg(rec_me + n, P[n]);
                __stcg(rec_me + 16 + n, h[n]);
            }
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release_gpu(st_me, kStAgg);

        // Start streaming the fix-up tiles while the look-back runs.
        if constexpr (USE_TMA) {
            if (tid == 0) {
                tma_prefetch_desc(it.tm_y);
                for (int s = 0; s < STAGES && s < it.ntiles; ++s) it.issue(s, (kk + s) % STAGES, 1);
            }
        }

        // Decoupled look-back: h0 = XP ⊙ I_j + Xh, walking j = c-1, c-2, ...
        float XP[kHalf], Xh[kHalf];
#pragma unroll
        for (int n = 0; n < kHalf; ++n) { XP[n] = 1.f; Xh[n] = 0.f; }
        for (int j = c - 1; j >= 0; --j) {
            if (tid == 0) {
                const uint32_t* sp = p.status + (static_cast<int64_t>(b) * p.nchunks + j) * p.nblk + g;
                uint32_t sv = ld_acquire_gpu(sp);
                uint32_t polls = 0;
                while (sv == kStNone) {
                    if (++polls > p.poll_limit) {
                        sv = kStTimeout;
                        record_error(p.hdr, -4);
                        break;
                    }
                    __nanosleep(128);
                    sv = ld_acquire_gpu(sp);
                }
                S.st = sv;
            }
            __syncthreads();
            const uint32_t sv = S.st;
            __syncthreads();
            if (sv == kStTimeout) break;
            if (cp.valid) {
                const float* rj = p.rec + ((static_cast<int64_t>(b) * p.nchunks + j) * d + ch) * kRec + hp;
                if (sv == kStIncl) {
#pragma unroll
                    for (int n = 0; n < kHalf; ++n) Xh[n] = fmaf(XP[n], __ldcg(rj + 32 + n), Xh[n]);
                } else {
#pragma unroll
                    for (int n = 0; n < kHalf; ++n) {
                        Xh[n] = fmaf(XP[n], __ldcg(rj + 16 + n), Xh[n]);
                        XP[n] *= __ldcg(rj + n);
                    }
                }
            }
            if (sv == kStIncl) break;
        }

        // Inclusive end state of this chunk: I = P ⊙ h0 + h_loc.
        if (!last) {
            if (cp.valid) {
#pragma unroll
                for (int n = 0; n < kHalf; ++n) __stcg(rec_me + 32 + n, fmaf(P[n], Xh[n], h[n]));
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release_gpu(st_me, kStIncl);
        } else if (cp.valid && ls) {
#pragma unroll
            for (int n = 0; n < kHalf; ++n) ls[n] = fmaf(P[n], Xh[n], h[n]);
        }

        // Fix-up pass over this chunk's outputs.
        f32x2 H0[4], PQ[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            H0[m] = pk2(Xh[2 * m], Xh[2 * m + 1]);
            PQ[m] = pk2(1.f, 1.f);
        }
        float Rq = 1.f;
        t = it.t_begin;
        for (int k = 0; k < it.ntiles; ++k, ++kk) {
            const int s = it.acquire(k, kk, 1);
            const int nt = static_cast<int>((it.t_end - t) < kTT ? (it.t_end - t) : kTT);
            const IO* ys = &S.a[s][kHalo][it.cc];
            const IO* dts = &S.dt[s][0][it.cc];
            const IO* zs = &S.z[s][0][it.cc];
            const float* bc = &S.bc[s][0][0];
            IO* yrow = ybase + (t - it.t_begin) * d;
            int j0 = 0;
            for (; j0 + G <= nt; j0 += G) fix_group<IO, FAST, STRUCT, G, FULL>(ys, dts, zs, bc, j0, H0, PQ, Rq, cp, yrow, d);
            for (; j0 < nt; ++j0)           fix_one<IO, FAST, STRUCT, FULL>(ys, dts, zs, bc, j0, H0, PQ, Rq, cp, yrow, d);
            t += nt;
        }
    }
}

// MINB resident CTAs per SM, groups of G steps, whole tiles unrolled or not;
// CONV: u comes from the causal conv1d + SiLU prologue over x; FULL: the
// softplus and the gate are both on (the host launches it only then).
template <typename IO, bool USE_TMA, int STAGES, int MINB, int G, bool UNROLL, bool CONV, bool FULL>
__global__ void __launch_bounds__(kNT, MINB)
ss_fwd_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_u,
              const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_z,
              const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
              const __grid_constant__ CUtensorMap tm_y) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    auto& S = *reinterpret_cast<FwdSmem<IO, STAGES>*>(smem_raw);
    const int tid = threadIdx.x;

    // ---------------------------------------------------------------- item
    if (tid == 0) S.item = (p.nchunks > 1) ? static_cast<int>(atomicAdd(&p.hdr[1], 1u))
                                           : static_cast<int>(blockIdx.x);
    __syncthreads();
    ItemCtx<IO, USE_TMA, STAGES> it;
    it.p = &p;
    it.S = &S;
    it.tm_u = &tm_u; it.tm_dt = &tm_dt; it.tm_z = &tm_z; it.tm_B = &tm_B; it.tm_C = &tm_C; it.tm_y = &tm_y;
    it.tid = tid;
    {
        const int item = S.item;
        it.g = item % p.nblk;
        const int rest = item / p.nblk;
        it.b = rest % p.batch;
        it.c = rest / p.batch;
    }
    const int lane = tid & 31;
    it.cc = (tid >> 5) * 16 + (lane & 15);
    it.t_begin = static_cast<int64_t>(it.c) * p.chunk_len;
    it.t_end = min(p.L, it.t_begin + p.chunk_len);
    it.ntiles = static_cast<int>((it.t_end - it.t_begin + kTT - 1) / kTT);
    it.d = p.d;
    it.has_z = (p.pflags & kPfHasZ) != 0;
    it.conv = CONV;
    it.bscale = FAST ? kLn2 : 1.0f;
    const int nact = it.has_z ? 3 : 2;   // per-channel tensors streamed per pass
    it.bytes_scan = static_cast<uint32_t>(((nact * kTT + (CONV ? kHalo : 0)) * kCB + 2 * kTT * kN) * sizeof(IO));
    it.bytes_fix = static_cast<uint32_t>((nact * kTT * kCB + kTT * kN) * sizeof(IO));
    const int ch = it.g * kCB + it.cc;

    // ------------------------------------------------- per-channel parameters
    ChanParams cp;
    cp.p = lane >> 4;
    cp.hi_mask = cp.p ? 0xffffffffu : 0u;
    cp.valid = ch < p.d;
    cp.z_mask = it.has_z ? 0xffffffffu : 0u;
    cp.sp_mask = (p.pflags & kPfSoftplus) ? 0xffffffffu : 0u;
    const int hp = kHalf * cp.p;
    bool structured = true;
    {
        const float* Arow = p.A + static_cast<int64_t>(cp.valid ? ch : 0) * kN;
        cp.a = cp.valid ? __ldg(Arow) : -1.0f;
#pragma unroll
        for (int n = 0; n < kHalf; ++n) {
            cp.Av[n] = cp.valid ? __ldg(Arow + hp + n) : -static_cast<float>(hp + n + 1);
            structured = structured && (cp.Av[n] == cp.a * static_cast<float>(hp + n + 1));
        }
    }
    const int all_struct = __syncthreads_and(structured ? 1 : 0);
    const bool use_struct = FAST && all_struct && !(p.pflags & kPfForceGeneral);
    cp.ab = cp.a * static_cast<float>(hp + 1);
    cp.kq = static_cast<float>(hp + 1);
    cp.Dv = (cp.valid && (p.pflags & kPfHasD)) ? __ldg(p.D + ch) : 0.f;
    const float biasv = (cp.valid && (p.pflags & kPfHasBias)) ? __ldg(p.bias + ch) : 0.f;
    cp.bias_s = FAST ? biasv * kLog2e : biasv;
#pragma unroll
    for (int k = 0; k < kConvW; ++k) cp.cw[k] = (CONV && cp.valid) ? __ldg(p.conv_w + static_cast<int64_t>(ch) * kConvW + k) : 0.f;
    cp.cb = (CONV && cp.valid && p.conv_b) ? __ldg(p.conv_b + ch) : 0.f;

    // ------------------------------------------------------- entry state
    f32x2 H[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) H[m] = pk2(0.f, 0.f);
    bool exact = true;
    if (it.c == 0 && p.h_init && cp.valid) {   // the sequence starts from a given state
        const float* r = p.h_init + (static_cast<int64_t>(it.b) * it.d + ch) * kN + hp;
#pragma unroll
        for (int m = 0; m < 4; ++m) H[m] = pk2(__ldg(r + 2 * m), __ldg(r + 2 * m + 1));
    }
    if (it.c > 0) {
        if (tid == 0)
            S.st = ld_acquire_gpu(p.status + (static_cast<int64_t>(it.b) * p.nchunks + (it.c - 1)) * p.nblk + it.g);
        __syncthreads();
        exact = (S.st == kStIncl);
        if (exact && cp.valid) {
            const float* r = p.rec + ((static_cast<int64_t>(it.b) * p.nchunks + (it.c - 1)) * it.d + ch) * kRec + 32 + hp;
#pragma unroll
            for (int m = 0; m < 4; ++m) H[m] = pk2(__ldcg(r + 2 * m), __ldcg(r + 2 * m + 1));
        }
    }
    if (!exact && tid == 0) atomicAdd(&p.hdr[2], 1u);

    if constexpr (USE_TMA) {
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < STAGES; ++s) mbar_init(&S.full[s], 1);
            fence_mbar_init();
            tma_prefetch_desc(&tm_u);
            tma_prefetch_desc(&tm_dt);
            if (it.has_z) tma_prefetch_desc(&tm_z);
            tma_prefetch_desc(&tm_B);
            tma_prefetch_desc(&tm_C);
        }
        __syncthreads();
        if (tid == 0)
            for (int s = 0; s < STAGES && s < it.ntiles; ++s) it.issue(s, s, 0);
    }

    static_assert(G % 2 == 0 && kTT % G == 0, "groups hold an even number of steps and tile a tile");
    if (use_struct) {
        if (exact) run_item<IO, USE_TMA, STAGES, G, UNROLL, true, true, CONV, FULL>(it, cp, H);
        else       run_item<IO, USE_TMA, STAGES, G, UNROLL, true, false, CONV, FULL>(it, cp, H);
    } else {
        if (exact) run_item<IO, USE_TMA, STAGES, G, UNROLL, false, true, CONV, FULL>(it, cp, H);
        else       run_item<IO, USE_TMA, STAGES, G, UNROLL, false, false, CONV, FULL>(it, cp, H);
    }
}

}  // namespace selscan
