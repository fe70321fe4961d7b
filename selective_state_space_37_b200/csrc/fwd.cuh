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
//   One CTA = one work item = (batch b, time chunk c, block of kCB channels);
//   one thread owns one channel and keeps its kN fp32 states in registers for
//   the whole chunk.  Tiles of kTT timesteps of u / Δraw / z ([kTT x kCB]) and
//   of B / C ([kTT x kN], shared by every channel) are brought into shared
//   memory by TMA (cp.async.bulk.tensor, no multicast) through a ring of
//   STAGES buffers completed on mbarriers; B and C are widened to fp32 once
//   per tile for all channels.
//
// Time chunking (the "hardware-aware parallel scan": the recurrence is linear,
// so a chunk maps its entry state h0 to P ⊙ h0 + h_loc with P = Π exp(Δ A)):
//   Items take tickets from a global counter in chunk-major order.  An item
//   whose predecessor chunk has already published its inclusive end state
//   starts from it and is exact at once.  Otherwise it scans from zero
//   (writing provisional outputs), publishes its aggregate (P, h_loc), looks
//   back through its predecessors' aggregates to the nearest inclusive state
//   (decoupled look-back; every wait is bounded), publishes its own inclusive
//   state and adds Σ_n C_t,n P_t,n h0_n · gate to each of its outputs.
//   Tickets are taken in start order, so an item only ever waits on items
//   that are already running, and those publish before they wait.
//
// A = a_d (n+1) fast path (bf16 I/O only): exp(Δ a_d (n+1)) = r^(n+1) with
//   r = exp(Δ a_d), one hardware exp per channel-timestep plus a product
//   ladder, instead of kN exps.  Detected per CTA with an exact test on A.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace selscan {

constexpr int kN = 16;      // d_state
constexpr int kTT = 32;     // timesteps per tile
constexpr int kNT = 128;    // threads per CTA
constexpr int kCB = kNT;    // channels per CTA (one per thread)
constexpr int kRec = 48;    // floats per carry record: P[16], h_loc[16], inclusive[16]

enum : uint32_t { kStNone = 0, kStAgg = 1, kStIncl = 2, kStTimeout = 0xFFFFFFFFu };
enum : uint32_t {
    kPfSoftplus = 1u,
    kPfForceGeneral = 2u,
    kPfTestDrop = 4u,
    kPfHasZ = 8u,
    kPfHasBias = 16u,
    kPfHasD = 32u
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
    int64_t L;
    int batch, d, chunk_len, nchunks, nblk;
    uint32_t pflags;
    uint32_t* hdr;       // [0]: error status (negative code as uint32), [1]: ticket counter
    uint32_t* status;    // [batch][nchunks][nblk] publication state of each item
    float* rec;          // [batch][nchunks][d][kRec] carry records
    uint64_t wait_ns;    // bound on one TMA completion wait
    uint32_t poll_limit; // bound on the polls of one carry wait
};

template <typename IO, int STAGES>
struct FwdSmem {
    IO u[STAGES][kTT][kCB];
    IO dt[STAGES][kTT][kCB];
    IO z[STAGES][kTT][kCB];
    IO B[STAGES][kTT][kN];
    IO C[STAGES][kTT][kN];
    float bc[STAGES][kTT][2 * kN];   // B (ln-free, fp32) then C, per timestep
    uint64_t full[STAGES];
    int item;
    uint32_t st;
};

__device__ __forceinline__ void record_error(uint32_t* hdr, int code) {
    atomicCAS(&hdr[0], 0u, static_cast<uint32_t>(code));
}

// r^1 .. r^16 by a balanced product ladder (depth 5).
__device__ __forceinline__ void power_ladder(float r, float (&pw)[kN]) {
    pw[0] = r;
    pw[1] = r * r;
    pw[2] = pw[1] * r;
    pw[3] = pw[1] * pw[1];
    pw[4] = pw[3] * r;
    pw[5] = pw[3] * pw[1];
    pw[6] = pw[3] * pw[2];
    pw[7] = pw[3] * pw[3];
#pragma unroll
    for (int j = 0; j < 8; ++j) pw[8 + j] = pw[7] * pw[j];
}

template <bool FAST>
__device__ __forceinline__ float delta_act(float x, bool softplus) {
    if (!softplus) return x;
    return FAST ? softplus_fast(x) : softplus_accurate(x);
}

template <bool FAST>
__device__ __forceinline__ float gate_of(float zv) {
    return FAST ? silu_fast(zv) : silu_accurate(zv);
}

// decay exp(Δ A_n); A2 holds A·log2(e) on the fast path and A itself otherwise.
template <bool FAST>
__device__ __forceinline__ float decay_of(float dl, float a2) {
    return FAST ? ex2_approx(dl * a2) : expf(dl * a2);
}

// One tile of nt timesteps for this thread's channel.
template <typename IO, bool FAST, bool STRUCT, bool TRACK>
__device__ __forceinline__ void scan_tile(const IO* __restrict__ us, const IO* __restrict__ dts,
                                          const IO* __restrict__ zs, const float* __restrict__ bc,
                                          int nt, float (&h)[kN], float (&P)[kN], float& R, float a2,
                                          const float (&A2)[kN], float biasv, float Dv, bool softplus,
                                          bool has_z, bool valid, IO* __restrict__ yrow, int64_t d) {
#pragma unroll 1
    for (int tt = 0; tt < nt; ++tt) {
        const float uu = to_f32(us[tt * kCB]);
        const float dl = delta_act<FAST>(to_f32(dts[tt * kCB]) + biasv, softplus);
        const float4* bq = reinterpret_cast<const float4*>(bc + tt * 2 * kN);
        float Bv[kN], Cv[kN];
#pragma unroll
        for (int q = 0; q < kN / 4; ++q) {
            const float4 b4 = bq[q];
            const float4 c4 = bq[kN / 4 + q];
            Bv[4 * q + 0] = b4.x; Bv[4 * q + 1] = b4.y; Bv[4 * q + 2] = b4.z; Bv[4 * q + 3] = b4.w;
            Cv[4 * q + 0] = c4.x; Cv[4 * q + 1] = c4.y; Cv[4 * q + 2] = c4.z; Cv[4 * q + 3] = c4.w;
        }
        const float du = dl * uu;
        if (STRUCT) {
            const float r = ex2_approx(dl * a2);
            float pw[kN];
            power_ladder(r, pw);
#pragma unroll
            for (int n = 0; n < kN; ++n) h[n] = fmaf(pw[n], h[n], du * Bv[n]);
            if (TRACK) R *= r;
        } else {
#pragma unroll
            for (int n = 0; n < kN; ++n) {
                const float a = decay_of<FAST>(dl, A2[n]);
                h[n] = fmaf(a, h[n], du * Bv[n]);
                if (TRACK) P[n] *= a;
            }
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int n = 0; n < kN; ++n) acc[n & 3] = fmaf(Cv[n], h[n], acc[n & 3]);
        float yv = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        yv = fmaf(Dv, uu, yv);
        if (has_z) yv *= gate_of<FAST>(to_f32(zs[tt * kCB]));
        if (valid) yrow[tt * d] = from_f32<IO>(yv);
    }
}

// Loads 16 consecutive IO elements (16-byte aligned) as fp32.
__device__ __forceinline__ void load16(const float* p, float (&v)[kN]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(q + i);
        v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[kN]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 w = __ldg(q + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
    }
}

template <typename IO, bool USE_TMA, int STAGES>
__global__ void __launch_bounds__(kNT)
ss_fwd_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_u,
              const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_z,
              const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C) {
    constexpr bool FAST = std::is_same<IO, __nv_bfloat16>::value;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    auto& S = *reinterpret_cast<FwdSmem<IO, STAGES>*>(smem_raw);
    const int tid = threadIdx.x;

    // ---------------------------------------------------------------- item
    if (tid == 0) S.item = (p.nchunks > 1) ? static_cast<int>(atomicAdd(&p.hdr[1], 1u))
                                           : static_cast<int>(blockIdx.x);
    __syncthreads();
    const int item = S.item;
    const int g = item % p.nblk;
    const int rest = item / p.nblk;
    const int b = rest % p.batch;
    const int c = rest / p.batch;
    const int ch = g * kCB + tid;
    const bool valid = ch < p.d;
    const int64_t t_begin = static_cast<int64_t>(c) * p.chunk_len;
    const int64_t t_end = min(p.L, t_begin + p.chunk_len);
    const int ntiles = static_cast<int>((t_end - t_begin + kTT - 1) / kTT);
    const bool has_z = (p.pflags & kPfHasZ) != 0;
    const bool softplus = (p.pflags & kPfSoftplus) != 0;
    const int64_t d = p.d;

    // ------------------------------------------------- per-channel parameters
    float A2[kN];
    bool structured = true;
    {
        float Arow[kN];
#pragma unroll
        for (int n = 0; n < kN; ++n) Arow[n] = valid ? __ldg(p.A + static_cast<int64_t>(ch) * kN + n)
                                                     : -static_cast<float>(n + 1);
#pragma unroll
        for (int n = 0; n < kN; ++n) {
            structured = structured && (Arow[n] == Arow[0] * static_cast<float>(n + 1));
            A2[n] = FAST ? Arow[n] * kLog2e : Arow[n];
        }
    }
    const int all_struct = __syncthreads_and(structured ? 1 : 0);
    const bool use_struct = FAST && all_struct && !(p.pflags & kPfForceGeneral);
    const float a2 = A2[0];
    const float Dv = (valid && (p.pflags & kPfHasD)) ? __ldg(p.D + ch) : 0.f;
    const float biasv = (valid && (p.pflags & kPfHasBias)) ? __ldg(p.bias + ch) : 0.f;

    // ------------------------------------------------------- entry state
    float h[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) h[n] = 0.f;
    bool exact = true;
    if (c > 0) {
        if (tid == 0)
            S.st = ld_acquire_gpu(p.status + (static_cast<int64_t>(b) * p.nchunks + (c - 1)) * p.nblk + g);
        __syncthreads();
        exact = (S.st == kStIncl);
        if (exact && valid) {
            const float* r = p.rec + ((static_cast<int64_t>(b) * p.nchunks + (c - 1)) * d + ch) * kRec + 32;
#pragma unroll
            for (int n = 0; n < kN; ++n) h[n] = __ldcg(r + n);
        }
    }

    // ------------------------------------------------------- tile pipeline
    const uint32_t tile_bytes = static_cast<uint32_t>(((has_z ? 3 : 2) * kTT * kCB + 2 * kTT * kN) * sizeof(IO));
    auto issue = [&](int k, int s) {
        const int t0 = static_cast<int>(t_begin + static_cast<int64_t>(k) * kTT);
        mbar_arrive_expect_tx(&S.full[s], tile_bytes);
        tma_load_3d(&S.u[s][0][0], &tm_u, g * kCB, t0, b, &S.full[s]);
        tma_load_3d(&S.dt[s][0][0], &tm_dt, g * kCB, t0, b, &S.full[s]);
        if (has_z) tma_load_3d(&S.z[s][0][0], &tm_z, g * kCB, t0, b, &S.full[s]);
        tma_load_3d(&S.B[s][0][0], &tm_B, 0, t0, b, &S.full[s]);
        tma_load_3d(&S.C[s][0][0], &tm_C, 0, t0, b, &S.full[s]);
    };
    auto fill_plain = [&](int k) {
        const int64_t t0 = t_begin + static_cast<int64_t>(k) * kTT;
        const IO* gu = static_cast<const IO*>(p.u);
        const IO* gd = static_cast<const IO*>(p.delta);
        const IO* gz = static_cast<const IO*>(p.z);
        for (int i = tid; i < kTT * kCB; i += kNT) {
            const int r = i / kCB, col = i % kCB;
            const int64_t t = t0 + r;
            const int cc = g * kCB + col;
            const bool ok = (t < p.L) && (cc < p.d);
            const int64_t idx = (static_cast<int64_t>(b) * p.L + t) * d + cc;
            S.u[0][r][col] = ok ? gu[idx] : from_f32<IO>(0.f);
            S.dt[0][r][col] = ok ? gd[idx] : from_f32<IO>(0.f);
            if (has_z) S.z[0][r][col] = ok ? gz[idx] : from_f32<IO>(0.f);
        }
        const IO* gB = static_cast<const IO*>(p.B);
        const IO* gC = static_cast<const IO*>(p.C);
        for (int i = tid; i < kTT * kN; i += kNT) {
            const int r = i / kN, n = i % kN;
            const int64_t t = t0 + r;
            const bool ok = t < p.L;
            const int64_t idx = (static_cast<int64_t>(b) * p.L + t) * kN + n;
            S.B[0][r][n] = ok ? gB[idx] : from_f32<IO>(0.f);
            S.C[0][r][n] = ok ? gC[idx] : from_f32<IO>(0.f);
        }
    };

    if constexpr (USE_TMA) {
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < STAGES; ++s) mbar_init(&S.full[s], 1);
            fence_mbar_init();
            tma_prefetch_desc(&tm_u);
            tma_prefetch_desc(&tm_dt);
            if (has_z) tma_prefetch_desc(&tm_z);
            tma_prefetch_desc(&tm_B);
            tma_prefetch_desc(&tm_C);
        }
        __syncthreads();
        if (tid == 0)
            for (int s = 0; s < STAGES && s < ntiles; ++s) issue(s, s);
    }

    float P[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) P[n] = 1.f;
    float R = 1.f;
    int64_t t = t_begin;
    IO* yrow = static_cast<IO*>(p.y) + (static_cast<int64_t>(b) * p.L + t_begin) * d + ch;

    for (int k = 0; k < ntiles; ++k) {
        const int s = USE_TMA ? (k % STAGES) : 0;
        if constexpr (USE_TMA) {
            if (!mbar_wait_bounded(&S.full[s], static_cast<uint32_t>((k / STAGES) & 1), p.wait_ns))
                record_error(p.hdr, -4);
        } else {
            __syncthreads();
            fill_plain(k);
            __syncthreads();
        }
        for (int i = tid; i < kTT * kN; i += kNT) {
            const int r = i / kN, n = i % kN;
            S.bc[s][r][n] = to_f32(S.B[s][r][n]);
            S.bc[s][r][kN + n] = to_f32(S.C[s][r][n]);
        }
        __syncthreads();
        if constexpr (USE_TMA) {
            if (tid == 0 && k >= 1 && k + STAGES - 1 < ntiles) {
                fence_proxy_async_smem();
                issue(k + STAGES - 1, (k - 1) % STAGES);
            }
        }
        const int nt = static_cast<int>((t_end - t) < kTT ? (t_end - t) : kTT);
        const IO* us = &S.u[s][0][tid];
        const IO* dts = &S.dt[s][0][tid];
        const IO* zs = &S.z[s][0][tid];
        const float* bc = &S.bc[s][0][0];
        if (use_struct) {
            if (exact) scan_tile<IO, FAST, true, false>(us, dts, zs, bc, nt, h, P, R, a2, A2, biasv, Dv, softplus, has_z, valid, yrow, d);
            else       scan_tile<IO, FAST, true, true >(us, dts, zs, bc, nt, h, P, R, a2, A2, biasv, Dv, softplus, has_z, valid, yrow, d);
        } else {
            if (exact) scan_tile<IO, FAST, false, false>(us, dts, zs, bc, nt, h, P, R, a2, A2, biasv, Dv, softplus, has_z, valid, yrow, d);
            else       scan_tile<IO, FAST, false, true >(us, dts, zs, bc, nt, h, P, R, a2, A2, biasv, Dv, softplus, has_z, valid, yrow, d);
        }
        t += nt;
        yrow += static_cast<int64_t>(nt) * d;
    }

    // ------------------------------------------------------------ epilogue
    const bool last = (c == p.nchunks - 1);
    const bool drop = (p.pflags & kPfTestDrop) && b == 0 && c == 0 && g == 0;
    uint32_t* st_me = p.status + (static_cast<int64_t>(b) * p.nchunks + c) * p.nblk + g;
    float* rec_me = p.rec + ((static_cast<int64_t>(b) * p.nchunks + c) * d + ch) * kRec;

    if (exact) {
        if (!last) {
            if (valid) {
#pragma unroll
                for (int n = 0; n < kN; ++n) __stcg(rec_me + 32 + n, h[n]);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0 && !drop) st_release_gpu(st_me, kStIncl);
        } else if (valid && p.last_state) {
            float* ls = p.last_state + (static_cast<int64_t>(b) * d + ch) * kN;
#pragma unroll
            for (int n = 0; n < kN; ++n) ls[n] = h[n];
        }
        return;
    }

    // Provisional chunk: publish the aggregate (P, h_loc) first.
    if (use_struct) power_ladder(R, P);
    if (valid) {
#pragma unroll
        for (int n = 0; n < kN; ++n) {
            __stcg(rec_me + n, P[n]);
            __stcg(rec_me + 16 + n, h[n]);
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_gpu(st_me, kStAgg);

    // Decoupled look-back: h0 = XP ⊙ I_j + Xh, walking j = c-1, c-2, ...
    float XP[kN], Xh[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) { XP[n] = 1.f; Xh[n] = 0.f; }
    for (int j = c - 1; j >= 0; --j) {
        if (tid == 0) {
            const uint32_t* sp = p.status + (static_cast<int64_t>(b) * p.nchunks + j) * p.nblk + g;
            uint32_t sv = ld_acquire_gpu(sp);
            uint32_t it = 0;
            while (sv == kStNone) {
                if (++it > p.poll_limit) {
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
        if (valid) {
            const float* rj = p.rec + ((static_cast<int64_t>(b) * p.nchunks + j) * d + ch) * kRec;
            if (sv == kStIncl) {
#pragma unroll
                for (int n = 0; n < kN; ++n) Xh[n] = fmaf(XP[n], __ldcg(rj + 32 + n), Xh[n]);
            } else {
#pragma unroll
                for (int n = 0; n < kN; ++n) {
                    Xh[n] = fmaf(XP[n], __ldcg(rj + 16 + n), Xh[n]);
                    XP[n] *= __ldcg(rj + n);
                }
            }
        }
        if (sv == kStIncl) break;
    }

    // Inclusive end state of this chunk: I = P ⊙ h0 + h_loc.
    if (!last) {
        if (valid) {
#pragma unroll
            for (int n = 0; n < kN; ++n) __stcg(rec_me + 32 + n, fmaf(P[n], Xh[n], h[n]));
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release_gpu(st_me, kStIncl);
    } else if (valid && p.last_state) {
        float* ls = p.last_state + (static_cast<int64_t>(b) * d + ch) * kN;
#pragma unroll
        for (int n = 0; n < kN; ++n) ls[n] = fmaf(P[n], Xh[n], h[n]);
    }

    // Fix-up: y_t += (Σ_n C_t,n · P_t,n · h0_n) · gate_t, P_t the in-chunk
    // prefix decay, recomputed exactly as during the scan.
    if (!valid) return;
    const IO* gd = static_cast<const IO*>(p.delta);
    const IO* gz = static_cast<const IO*>(p.z);
    const IO* gC = static_cast<const IO*>(p.C);
    IO* gy = static_cast<IO*>(p.y);
    float Rq = 1.f;
    float Pq[kN];
#pragma unroll
    for (int n = 0; n < kN; ++n) Pq[n] = 1.f;
#pragma unroll 1
    for (int64_t tq = t_begin; tq < t_end; ++tq) {
        const int64_t row = static_cast<int64_t>(b) * p.L + tq;
        const int64_t idx = row * d + ch;
        const float dl = delta_act<FAST>(to_f32(gd[idx]) + biasv, softplus);
        float Cv[kN];
        load16(gC + row * kN, Cv);
        float corr;
        if (use_struct) {
            Rq *= ex2_approx(dl * a2);
            float acc = Cv[kN - 1] * Xh[kN - 1];
#pragma unroll
            for (int n = kN - 2; n >= 0; --n) acc = fmaf(acc, Rq, Cv[n] * Xh[n]);
            corr = acc * Rq;
        } else {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int n = 0; n < kN; ++n) {
                Pq[n] *= decay_of<FAST>(dl, A2[n]);
                acc[n & 3] = fmaf(Cv[n] * Pq[n], Xh[n], acc[n & 3]);
            }
            corr = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
        if (has_z) corr *= gate_of<FAST>(to_f32(gz[idx]));
        gy[idx] = from_f32<IO>(to_f32(gy[idx]) + corr);
    }
}

}  // namespace selscan
