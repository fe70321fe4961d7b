// ssd.cuh -- multi-head scan with a scalar decay per head (the Mamba-2 / SSD
// model of the mamba README's Mamba-2 section; the model-architecture page's
// "Mamba-2 (multi-head, larger state)", headdim 64, d_state 64 or 128,
// ngroups 1), on the tensor cores (sm_100a).
//
// Per (batch b, head h), with the head's P = 64 channels sharing Δ, B, C:
//   Δ_t = softplus(dt_t + dt_bias),  H_t = exp(Δ_t A) H_{t-1} + Δ_t x_t B_tᵀ,
//   y_t = H_t C_t + D x_t           (H_t is P x N, x_t ∈ R^P, B_t, C_t ∈ R^N)
// The decay being one scalar per step makes the recurrence, over a chunk of
// Q = 64 steps with cum_t = Σ_{r<=t} Δ_r A, the matrix products
//   Y    = (C Bᵀ ∘ M) X  +  diag(e^{cum}) C G_inᵀ,   M[t,s] = e^{cum_t - cum_s} Δ_s (s <= t)
//   G_out = e^{cum_{Q-1}} G_in + Xᵀ diag(e^{cum_{Q-1} - cum_s} Δ_s) B
// so every step of a chunk is a dense contraction of bf16 tiles with fp32
// accumulation.  One CTA (4 warps) walks the chunks of one (b, h) in order
// and keeps G in the accumulators of its state product, so the carry between
// chunks never leaves the SM.  The products use the warp-level mma.sync
// m16n8k16 bf16 instructions with ldmatrix fragment loads from padded shared
// tiles; warp w owns rows 16w..16w+15 of S and Y (time) and of G (channel).
// Three CTAs share an SM (62 KB of shared memory and <= 168 registers each),
// so one CTA's tile copies (cp.async) and barriers overlap the others' products.
// When batch x heads leaves SMs idle, each sequence is cut into nseg segments
// of whole chunks and the carry between segments is made exact beforehand
// (the recurrence is linear with a scalar decay): a state pass (STATE) runs
// each segment but the last from G = 0 computing only G_out and Σ Δ A, a fold
// turns those into the state entering every segment, and the main pass runs
// each segment from its entering state.
#pragma once

#include "common.cuh"
#include "cp_async.cuh"

namespace selscan {

constexpr int kSsdQ = 64;          // chunk length
constexpr int kSsdP = 64;          // head dimension
constexpr int kSsdThreads = 128;   // 4 warps
constexpr int kSsdPad = 8;         // bf16 elements of row padding (ldmatrix without bank conflicts)

struct SsdParams {
    const __nv_bfloat16* x;    // [batch, L, H, P]
    const __nv_bfloat16* dt;   // [batch, L, H]
    const float* dt_bias;      // [H] or null
    const float* A;            // [H] (negative)
    const __nv_bfloat16* B;    // [batch, L, N]
    const __nv_bfloat16* C;    // [batch, L, N]
    const float* D;            // [H] or null
    __nv_bfloat16* y;          // [batch, L, H, P]
    float* final_state;        // [batch, H, P, N] or null
    float* rec;                // [batch, H, nseg - 1, P, N]: segment end states from zero, then (folded) the
                               // state entering the next segment
    float* esum;               // [batch, H, nseg]: Σ Δ A over each segment
    int64_t L;
    int batch, H;
    int nseg, cseg;            // time segments of the sequence and chunks per segment
    int softplus;
};

template <int N>
struct SsdTiles {
    __nv_bfloat16 X[kSsdQ][kSsdP + kSsdPad];    // x of the chunk [t][p]
    __nv_bfloat16 Bt[kSsdQ][N + kSsdPad];       // B [s][n]; then scaled by e^{cum_end - cum_s} Δ_s
    __nv_bfloat16 Ct[kSsdQ][N + kSsdPad];       // C [t][n]
};

template <int N>
struct SsdSmem {
    SsdTiles<N> tile[1];                        // this chunk's tiles
    __nv_bfloat16 G[kSsdP][N + kSsdPad];        // carried state, bf16 copy [p][n]
    float cum[kSsdQ];                           // inclusive prefix of Δ A
    float dlt[kSsdQ];                           // Δ_t
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
// D += A(16x16 bf16, row) · B(16x8 bf16, col), fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Grid: one CTA per (segment k, batch b, head h), blockIdx.x = (k * batch + b) * H + h;
// STATE runs segments 0 .. nseg - 2 only.
template <int N, bool STATE>
__global__ void __launch_bounds__(kSsdThreads, 3) ss_ssd_kernel(const __grid_constant__ SsdParams p) {
    constexpr int NT = N / 8;          // n8 tiles of the state width
    extern __shared__ __align__(16) unsigned char ssd_smem_raw[];
    auto& S = *reinterpret_cast<SsdSmem<N>*>(ssd_smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, c = lane & 3;           // fragment row / column group
    const int h = blockIdx.x % p.H;
    const int b = (blockIdx.x / p.H) % p.batch;
    const int sg = blockIdx.x / (p.H * p.batch);     // segment
    const int64_t bh = static_cast<int64_t>(b) * p.H + h;
    const float Ah = p.A[h];
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
    const float Dh = p.D ? p.D[h] : 0.0f;
    const int64_t seg_t0 = static_cast<int64_t>(sg) * p.cseg * kSsdQ;
    const int64_t seg_t1 = min(seg_t0 + static_cast<int64_t>(p.cseg) * kSsdQ, p.L);

    // G entering the segment: zero, or the folded record of the previous segment
    const float* gin = (!STATE && sg > 0) ? p.rec + (bh * (p.nseg - 1) + (sg - 1)) * kSsdP * N : nullptr;
    float accG[NT][4];                               // G rows 16w.. (channel p), all n
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        if (gin) {
            const int nc = 8 * j + 2 * c;
            const float2 lo = *reinterpret_cast<const float2*>(gin + (16 * w + g) * N + nc);
            const float2 hi = *reinterpret_cast<const float2*>(gin + (16 * w + g + 8) * N + nc);
            accG[j][0] = lo.x; accG[j][1] = lo.y; accG[j][2] = hi.x; accG[j][3] = hi.y;
            *reinterpret_cast<uint32_t*>(&S.G[16 * w + g][nc]) = pack_bf16(lo.x, lo.y);
            *reinterpret_cast<uint32_t*>(&S.G[16 * w + g + 8][nc]) = pack_bf16(hi.x, hi.y);
        } else {
            accG[j][0] = accG[j][1] = accG[j][2] = accG[j][3] = 0.0f;
        }
    }
    float esum = 0.0f;                               // Σ Δ A over the segment (STATE)

    // Copies of one chunk's x, B, C tiles (rows past the sequence read as zero).
    auto issue_tiles = [&](int64_t t0, SsdTiles<N>& T) {
        const int q = static_cast<int>(p.L - t0 < kSsdQ ? p.L - t0 : kSsdQ);
        for (int i = tid; i < kSsdQ * (kSsdP / 8); i += kSsdThreads) {
            const int r = i / (kSsdP / 8), k = (i % (kSsdP / 8)) * 8;
            const int rr = r < q ? r : 0;
            cp_async16(&T.X[r][k], p.x + ((static_cast<int64_t>(b) * p.L + t0 + rr) * p.H + h) * kSsdP + k, r < q);
        }
        for (int i = tid; i < kSsdQ * (N / 8); i += kSsdThreads) {
            const int r = i / (N / 8), k = (i % (N / 8)) * 8;
            const int rr = r < q ? r : 0;
            const int64_t off = (static_cast<int64_t>(b) * p.L + t0 + rr) * N + k;
            cp_async16(&T.Bt[r][k], p.B + off, r < q);
            if (!STATE) cp_async16(&T.Ct[r][k], p.C + off, r < q);
        }
    };
    // Warp 0 holds Δraw of the next chunk's steps 2·lane and 2·lane + 1.
    float dtn[2] = {0.0f, 0.0f};
    auto load_dt = [&](int64_t t0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t t = t0 + 2 * lane + e;
            dtn[e] = t < p.L ? __bfloat162float(p.dt[(static_cast<int64_t>(b) * p.L + t) * p.H + h]) : 0.0f;
        }
    };
    if (w == 0) load_dt(seg_t0);

    for (int64_t t0 = seg_t0; t0 < seg_t1; t0 += kSsdQ) {
        const int q = static_cast<int>(p.L - t0 < kSsdQ ? p.L - t0 : kSsdQ);
        __syncthreads();   // the previous chunk is done with every tile and with cum / dlt
        issue_tiles(t0, S.tile[0]);
        cp_async_commit();
        if (w == 0) {
            // Δ and the inclusive prefix of Δ A over the chunk: each lane takes two
            // consecutive steps, then one scan over the 32 pair sums.
            float dl[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float xr = dtn[e] + bias;
                dl[e] = (2 * lane + e < q) ? (p.softplus ? softplus_accurate(xr) : xr) : 0.0f;
            }
            const float a1 = dl[1] * Ah;
            float sc = fmaf(dl[0], Ah, a1);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, sc, o);
                if (lane >= o) sc += v;
            }
            S.cum[2 * lane + 1] = sc;
            S.cum[2 * lane] = sc - a1;
            S.dlt[2 * lane] = dl[0];
            S.dlt[2 * lane + 1] = dl[1];
            if (t0 + kSsdQ < seg_t1) load_dt(t0 + kSsdQ);
        }
        cp_async_wait_all();   // this thread's copies of the chunk have landed
        __syncthreads();
        auto& T = S.tile[0];
        const float cum_end = S.cum[kSsdQ - 1];
        if (STATE) {
            esum += cum_end;
            // G_out = e^{cum_end} G_in + Xᵀ (scaled B): scale B, then the state product
            for (int i = tid; i < kSsdQ * (N / 2); i += kSsdThreads) {
                const int r = i / (N / 2), kk = (i % (N / 2)) * 2;
                const float sc = __expf(cum_end - S.cum[r]) * S.dlt[r];
                __nv_bfloat162* v = reinterpret_cast<__nv_bfloat162*>(&T.Bt[r][kk]);
                const float2 f = __bfloat1622float2(*v);
                *v = __floats2bfloat162_rn(f.x * sc, f.y * sc);
            }
            __syncthreads();
            const float e_end = __expf(cum_end);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                accG[j][0] *= e_end; accG[j][1] *= e_end;
                accG[j][2] *= e_end; accG[j][3] *= e_end;
            }
#pragma unroll
            for (int ks = 0; ks < kSsdQ; ks += 16) {
                uint32_t af[4];
                ldsm_x4_t(af, &T.X[ks + (lane & 7) + (lane >> 4) * 8][16 * w + ((lane >> 3) & 1) * 8]);
#pragma unroll
                for (int j = 0; j < NT; j += 2) {
                    uint32_t bf[4];
                    ldsm_x4_t(bf, &T.Bt[ks + (lane & 7) + ((lane >> 3) & 1) * 8][8 * j + (lane >> 4) * 8]);
                    mma_bf16(accG[j], af, bf[0], bf[1]);
                    mma_bf16(accG[j + 1], af, bf[2], bf[3]);
                }
            }
            continue;
        }

        // ----------- S = C Bᵀ (causal tiles only) and C G_inᵀ, sharing C's fragments
        const int nS = 2 * (w + 1);                 // s-tiles 0 .. 16w+15
        const bool carry = t0 > seg_t0 || sg > 0;   // G_in is zero before the sequence's first chunk
        float accS[8][4], accY[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            accS[j][0] = accS[j][1] = accS[j][2] = accS[j][3] = 0.0f;
            accY[j][0] = accY[j][1] = accY[j][2] = accY[j][3] = 0.0f;
        }
#pragma unroll
        for (int k = 0; k < N; k += 16) {
            uint32_t af[4];
            ldsm_x4(af, &T.Ct[16 * w + (lane & 7) + ((lane >> 3) & 1) * 8][k + (lane >> 4) * 8]);
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                if (j < nS) {
                    uint32_t bf[4];
                    ldsm_x4(bf, &T.Bt[8 * j + (lane & 7) + (lane >> 4) * 8][k + ((lane >> 3) & 1) * 8]);
                    mma_bf16(accS[j], af, bf[0], bf[1]);
                    mma_bf16(accS[j + 1], af, bf[2], bf[3]);
                }
                if (carry) {
                    uint32_t gf[4];
                    ldsm_x4(gf, &S.G[8 * j + (lane & 7) + (lane >> 4) * 8][k + ((lane >> 3) & 1) * 8]);
                    mma_bf16(accY[j], af, gf[0], gf[1]);
                    mma_bf16(accY[j + 1], af, gf[2], gf[3]);
                }
            }
        }
        __syncthreads();   // every warp has read B: scale it in place for the state product
        for (int i = tid; i < kSsdQ * (N / 2); i += kSsdThreads) {
            const int r = i / (N / 2), k = (i % (N / 2)) * 2;
            const float sc = __expf(cum_end - S.cum[r]) * S.dlt[r];
            __nv_bfloat162* v = reinterpret_cast<__nv_bfloat162*>(&T.Bt[r][k]);
            const float2 f = __bfloat1622float2(*v);
            *v = __floats2bfloat162_rn(f.x * sc, f.y * sc);
        }

        // --------------------------------------- M = S ∘ decay ∘ Δ_s, as A fragments
        const int t_lo = 16 * w + g, t_hi = t_lo + 8;
        const float cum_lo = S.cum[t_lo], cum_hi = S.cum[t_hi];
        uint32_t mf[4][4];                          // k16 blocks of s (0 .. w)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int s0 = 8 * j + 2 * c;
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = s0 + (e & 1);
                const int t = (e < 2) ? t_lo : t_hi;
                const float ct = (e < 2) ? cum_lo : cum_hi;
                v[e] = (j < nS && s <= t) ? accS[j][e] * __expf(ct - S.cum[s]) * S.dlt[s] : 0.0f;
            }
            const int kb = j >> 1;
            if ((j & 1) == 0) {
                mf[kb][0] = pack_bf16(v[0], v[1]);
                mf[kb][1] = pack_bf16(v[2], v[3]);
            } else {
                mf[kb][2] = pack_bf16(v[0], v[1]);
                mf[kb][3] = pack_bf16(v[2], v[3]);
            }
        }

        // ---------------------------------------- Y = e^{cum} (C G_inᵀ) + M X
        if (carry) {
            const float e_lo = __expf(cum_lo), e_hi = __expf(cum_hi);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                accY[j][0] *= e_lo; accY[j][1] *= e_lo;
                accY[j][2] *= e_hi; accY[j][3] *= e_hi;
            }
        }
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            if (kb <= w) {
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    uint32_t bf[4];
                    ldsm_x4_t(bf, &T.X[16 * kb + (lane & 7) + ((lane >> 3) & 1) * 8][8 * j + (lane >> 4) * 8]);
                    mma_bf16(accY[j], mf[kb], bf[0], bf[1]);
                    mma_bf16(accY[j + 1], mf[kb], bf[2], bf[3]);
                }
            }
        }
        // + D x, then the outputs of rows t < q
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int pc = 8 * j + 2 * c;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = half ? t_hi : t_lo;
                const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&T.X[t][pc]));
                const float y0 = fmaf(Dh, xv.x, accY[j][2 * half]);
                const float y1 = fmaf(Dh, xv.y, accY[j][2 * half + 1]);
                if (t < q)
                    *reinterpret_cast<__nv_bfloat162*>(p.y + ((static_cast<int64_t>(b) * p.L + t0 + t) * p.H + h) *
                                                                 kSsdP + pc) = __floats2bfloat162_rn(y0, y1);
            }
        }

        // -------------------------- G_out = e^{cum_end} G_in + Xᵀ (scaled B)
        __syncthreads();   // scaled B complete; every warp is done reading the bf16 G copy
        const float e_end = __expf(cum_end);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            accG[j][0] *= e_end; accG[j][1] *= e_end;
            accG[j][2] *= e_end; accG[j][3] *= e_end;
        }
#pragma unroll
        for (int ks = 0; ks < kSsdQ; ks += 16) {
            uint32_t af[4];   // Xᵀ rows p = 16w.., k = s
            ldsm_x4_t(af, &T.X[ks + (lane & 7) + (lane >> 4) * 8][16 * w + ((lane >> 3) & 1) * 8]);
#pragma unroll
            for (int j = 0; j < NT; j += 2) {
                uint32_t bf[4];
                ldsm_x4_t(bf, &T.Bt[ks + (lane & 7) + ((lane >> 3) & 1) * 8][8 * j + (lane >> 4) * 8]);
                mma_bf16(accG[j], af, bf[0], bf[1]);
                mma_bf16(accG[j + 1], af, bf[2], bf[3]);
            }
        }
        // bf16 copy for the next chunk's C G_inᵀ (rows of this warp only)
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int nc = 8 * j + 2 * c;
            *reinterpret_cast<uint32_t*>(&S.G[16 * w + g][nc]) = pack_bf16(accG[j][0], accG[j][1]);
            *reinterpret_cast<uint32_t*>(&S.G[16 * w + g + 8][nc]) = pack_bf16(accG[j][2], accG[j][3]);
        }
    }
    if (STATE) {
        float* gout = p.rec + (bh * (p.nseg - 1) + sg) * kSsdP * N;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int nc = 8 * j + 2 * c;
            *reinterpret_cast<float2*>(gout + (16 * w + g) * N + nc) = make_float2(accG[j][0], accG[j][1]);
            *reinterpret_cast<float2*>(gout + (16 * w + g + 8) * N + nc) = make_float2(accG[j][2], accG[j][3]);
        }
        if (tid == 0) p.esum[bh * p.nseg + sg] = esum;
        return;
    }
    if (p.final_state && sg == p.nseg - 1) {
        float* fs = p.final_state + bh * kSsdP * N;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int nc = 8 * j + 2 * c;
            *reinterpret_cast<float2*>(fs + (16 * w + g) * N + nc) = make_float2(accG[j][0], accG[j][1]);
            *reinterpret_cast<float2*>(fs + (16 * w + g + 8) * N + nc) = make_float2(accG[j][2], accG[j][3]);
        }
    }
}

// Between the passes: one thread per (batch, head, p, n) folds the segment
// records in order, G_in(k + 1) = e^{Σ_k Δ A} G_in(k) + G_loc(k) from
// G_in(0) = 0, writing G_in(k + 1) over G_loc(k).
template <int N>
__global__ void __launch_bounds__(256) ss_ssd_fold_kernel(const __grid_constant__ SsdParams p) {
    const int64_t per = static_cast<int64_t>(kSsdP) * N;
    const int64_t total = static_cast<int64_t>(p.batch) * p.H * per;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t bh = i / per, e = i % per;
        float gv = 0.0f;
        for (int k = 0; k + 1 < p.nseg; ++k) {
            float* r = p.rec + (bh * (p.nseg - 1) + k) * per + e;
            gv = fmaf(expf(p.esum[bh * p.nseg + k]), gv, *r);
            *r = gv;
        }
    }
}

}  // namespace selscan
