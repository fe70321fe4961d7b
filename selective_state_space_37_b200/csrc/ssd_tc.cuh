// ssd_tc.cuh -- the multi-head scalar-decay scan (Mamba-2's SSD model) on the
// fifth-generation tensor cores of sm_100a: tcgen05.mma with its accumulators
// in tensor memory (TMEM), operand tiles staged by TMA in the 128-byte
// swizzled shared-memory layout the MMA descriptors read.
//
// Per (batch b, head h), with the head's P = 64 channels sharing Δ, B, C (the
// mamba README's Mamba-2 section; the model-architecture page's "Mamba-2
// (multi-head, larger state)", headdim 64, ngroups 1):
//   Δ_t = softplus(dt_t + dt_bias),  H_t = exp(Δ_t A) H_{t-1} + Δ_t x_t B_tᵀ,
//   y_t = H_t C_t + D x_t           (H_t is P x N, x_t ∈ R^P, B_t, C_t ∈ R^N).
// Over a chunk of Q = 128 steps with cum_t = Σ_{r<=t} Δ_r A (the recurrence
// has one scalar decay per step, so a chunk is a set of dense products):
//   Y = (C Bᵀ ∘ M) X + diag(e^{cum}) (C Gᵀ),   M[t,s] = e^{cum_t - cum_s} Δ_s (s <= t)
//   G ← e^{cum_end} G + (Bᵀ X̃)ᵀ,                X̃[s,:] = e^{cum_end - cum_s} Δ_s x_s
// with G the P x N state entering the chunk.
//
// One CTA walks the chunks of one (b, h) in order, its warps specialised:
//   warp 16 (producer, one thread): TMA loads of the x, B, C tiles and every
//     MMA (bf16 operands, fp32 accumulation, M = 128):
//       S   = C Bᵀ              128 x 128, K = N  -> TMEM columns [0, 128)
//       CG  = C G_hiᵀ + C G_loᵀ  128 x 64, K = N  -> TMEM columns [128, 192)
//       ΔGᵀ = Bᵀ X̃              128 x 64,  K = Q  -> TMEM columns [320, 384)
//       Y   = Mm X              128 x 64,  K = Q  -> TMEM columns [256, 320)
//   warp 17: Δ, the prefix of Δ A and the decay factors, a chunk ahead into
//     a double buffer;
//   warps 0..15 (compute): four threads per TMEM lane (one time step t, or
//     one state index n), each on a quarter of the lane's columns: X̃ from x,
//     the causal decay mask Mm from S, the state update, and the outputs
//     y = Y + e^{cum_t} CG + D x, staged in shared memory and written by a
//     bulk tensor store.
// The warps hand work over through mbarriers, so the tensor core runs the
// next chunk's C Bᵀ under this chunk's epilogue and Mm X under the state
// update, and B and C of the next chunk load as soon as their last MMA is
// done.  The carried state G stays fp32 in registers (the four threads of row
// n hold G[:, n]); the product with C reads it as two bf16 terms G_hi + G_lo,
// accumulated into one tile, so it is not rounded to bf16 before the readout.  Every wait is bounded: a
// wait that runs out records SS error -4 in the status word and the CTA
// winds down (copies in flight drained, MMAs completed, TMEM released).
//
// d_state 64 runs the same kernel with the second 64-column block of the B
// and C tiles held at zero, so the state rows n >= 64 stay zero.
//
// Time segments: sequences that would leave SMs idle -- those of the last,
// partly filled wave, or all of them when there are few -- are cut into
// segments of whole chunks with an exact carry (state pass from G = 0 keeping
// only G_out and Σ Δ A, the fold of ssd.cuh, then the main pass from each
// segment's entering state); the host chooses the plan.
#pragma once

#include "common.cuh"
#include "ssd.cuh"

namespace selscan {
namespace tc {

constexpr int kQ = 128;            // chunk length (MMA M for the time rows)
constexpr int kP = 64;             // head dimension
constexpr int kN = 128;            // state width handled here
constexpr int kRows = 128;         // TMEM lanes / tile rows
constexpr int kRT = 4;                // compute threads per tile row (warps w, w + 4, w + 8, w + 12
                                      // share TMEM lanes 32 (w % 4) ..)
constexpr int kComputeWarps = 4 * kRT;
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kPT = kP / kRT;         // a thread's columns of x, y and the state (16)
constexpr int kXC = kPT / 8;          // its 16-byte chunks of a 64-column row (2)
constexpr int kSB = (kQ / 32) / kRT;  // its 32-column blocks of the mask (1)
constexpr int kProducerWarp = kComputeWarps;       // one thread: TMA loads and MMAs
constexpr int kPrefixWarp = kComputeWarps + 1;     // the Δ prefix, a chunk ahead
constexpr int kThreads = kComputeThreads + 64;
static_assert(kComputeThreads == 512 && kSB == 1 && kXC == 2, "the barriers and splits below assume 4 threads per row");
constexpr uint32_t kTmemCols = 512;   // allocation (power of two >= the 384 columns used)
constexpr uint32_t kColS = 0, kColCG = 128, kColY = 256, kColG = 320;   // CG: 64 columns

// Instruction descriptors (kind::f16, bf16 x bf16 -> fp32, M = 128): bit 4 D
// format f32, bits 7/10 A/B format bf16, bit 15/16 A/B major (1: MN-major),
// bits 17.. N >> 3, bits 24.. M >> 4.
constexpr uint32_t kIdesc_128x128_KK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdesc_128x64_KMN = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((64u >> 3) << 17) |
                                       ((128u >> 4) << 24);
constexpr uint32_t kIdesc_128x64_MNMN = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                        ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdesc_128x128_KMN = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) |
                                        ((128u >> 4) << 24);

// Shared memory, byte offsets from a 1024-aligned base.  Every operand tile
// is a set of [rows][64 bf16] blocks of 128-byte rows in the 128-byte
// swizzle (16-byte chunk c of row r stored at chunk c ^ (r & 7)).
constexpr uint32_t kOffX0 = 0;            // x [t][p], two buffers
constexpr uint32_t kOffX1 = 16384;
constexpr uint32_t kOffXt = 32768;        // X̃ [s][p]
constexpr uint32_t kOffB = 49152;         // B [s][n]: blocks n 0..63, 64..127
constexpr uint32_t kOffC = 81920;         // C [t][n]: blocks n 0..63, 64..127
constexpr uint32_t kOffM = 114688;        // Mm [t][s]: blocks s 0..63, 64..127
constexpr uint32_t kOffGh = 147456;       // G_hi [n][p]  } one MN-major operand of
constexpr uint32_t kOffGl = 163840;       // G_lo [n][p]  } width 128: blocks 16 KB apart
constexpr uint32_t kOffY = 180224;        // y [t][p] staged for the bulk tensor store
constexpr uint32_t kOffCum = 196608;      // cum[2][128] f32 (by chunk parity)
constexpr uint32_t kOffCs = kOffCum + 1024;   // cum · log2 e, [2][128]
constexpr uint32_t kOffDlt = kOffCs + 1024;   // Δ, [2][128]
constexpr uint32_t kOffCf = kOffDlt + 1024;   // Δ_s e^{cum_r - cum_s}, r the last step of s's 32-block, [2][128]
constexpr uint32_t kOffWx = kOffCf + 1024;   // e^{cum_end - cum_s} Δ_s, the scale of X̃'s row s, [2][128]
constexpr uint32_t kOffBar = kOffWx + 1024;   // 16 mbarriers; TMEM base address at +128, x tiles waited at +132
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack

struct Params {
    const __nv_bfloat16* dt;   // [batch, L, H]
    const float* dt_bias;      // [H] or null
    const float* A;            // [H]
    const float* D;            // [H] or null
    __nv_bfloat16* y;          // [batch, L, H, P]
    float* final_state;        // [batch, H, P, N] or null
    float* rec;                // [batch, H, nseg - 1, P, N]
    float* esum;               // [batch, H, nseg]
    uint32_t* status;          // error word or null
    int64_t L;
    int batch, H;
    int n_whole;               // (batch, head) sequences 0 .. n_whole - 1 run whole, one CTA each; the
    int nseg, cseg;            // others are cut into nseg segments of cseg chunks of kQ steps
    int n;                     // d_state: 128, or 64 (B, C and the state padded to 128 with zeros)
    int softplus;
    int test_drop;             // test only: CTA 0 never signals its first C Bᵀ (a wait runs out)
    uint64_t wait_ns;          // bound on one hand-over wait
    uint64_t drain_ns;         // bound on the wind-down waits (copies in flight, the last MMAs)
};

// ------------------------------------------------------------ tcgen05 / TMA
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] · B[smem desc]; issued by one thread.
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}
// Arrive (once) on `bar` when every MMA this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32 (w % 4) ..).  The
// load and its wait are one asm statement: the registers are defined only once the data is in them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 16-column ranges of this thread's TMEM lane, one wait.
__device__ __forceinline__ void tmem_ld16x2(uint32_t a0, uint32_t a1, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31}, [%33];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(a0), "r"(a1)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: 128-byte swizzle, start / leading / stride
// byte offsets in 16-byte units, descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, int w,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}
// Tile of this CTA's shared memory -> global through the 4-D map (rows past the
// tensor's extent are not written); completion tracked by the bulk group.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* tm, uint32_t src, int x, int y, int z, int w) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed bulk store has finished reading shared memory / is complete
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_load_3d_u(uint32_t dst, const CUtensorMap* tm, int x, int y, int z,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// bf16 pair from two floats (round to nearest even), and back.
__device__ __forceinline__ uint32_t pk(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Address of logical 16-byte chunk c (0..7) of row r of a swizzled block.
__device__ __forceinline__ uint32_t chunk_addr(uint32_t block, int r, int c) {
    return block + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(c ^ (r & 7)) << 4);
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Barrier 1 over the 512 compute threads: true on every thread when `pred`
// holds on any of them.
__device__ __forceinline__ bool cw_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 512, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void cw_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// Grid: sequences are items i = b * H + h.  Main pass: CTAs 0 .. n_whole - 1 run items 0 .. n_whole - 1
// whole; CTA n_whole + j runs segment j % nseg of item n_whole + j / nseg.  STATE: CTA j runs segment
// j % (nseg - 1) of item n_whole + j / (nseg - 1) (segments 0 .. nseg - 2: G_out from zero, no outputs).
// Segment records are indexed by the split item's rank r = i - n_whole.
template <bool STATE>
__global__ void __launch_bounds__(kThreads, 1)
ss_ssd_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                 const __grid_constant__ CUtensorMap tm_y) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;   // 1024-aligned: the swizzle pattern is address based
    unsigned char* gbase = smem_raw + (base - raw);
    float* const cum2 = reinterpret_cast<float*>(gbase + kOffCum);
    float* const cs2 = reinterpret_cast<float*>(gbase + kOffCs);
    float* const dlt2 = reinterpret_cast<float*>(gbase + kOffDlt);
    float* const cf2 = reinterpret_cast<float*>(gbase + kOffCf);
    float* const wx2 = reinterpret_cast<float*>(gbase + kOffWx);
    uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kOffBar);
    uint64_t* x_full = bars;          // [2]: x tile of buffer 0 / 1 landed
    uint64_t* b_full = bars + 2;      // B tile landed
    uint64_t* c_full = bars + 3;      // C tile landed
    uint64_t* s_full = bars + 4;      // C Bᵀ in TMEM
    uint64_t* cg_done = bars + 5;     // C Bᵀ and C Gᵀ done: C free, G copies read
    uint64_t* dg_done = bars + 6;     // Bᵀ X̃ done: B and X̃ free
    uint64_t* y_done = bars + 7;      // Mm X done (and every MMA before it)
    uint64_t* xt_ready = bars + 8;    // X̃ written (one arrival per compute warp)
    uint64_t* mm_ready = bars + 9;    // Mm written and S read (one arrival per compute warp)
    uint64_t* ep_done = bars + 10;    // a chunk's epilogue done: G copies stored, TMEM columns and
                                      // its x buffer free
    uint64_t* pf_full = bars + 11;    // [2]: the Δ prefix of buffer 0 / 1 written
    uint64_t* pf_empty = bars + 13;   // [2]: the chunk reading prefix buffer 0 / 1 is done
    uint64_t* fin_bar = bars + 15;    // every MMA issued is done (wind-down)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + 128);
    int* xw_slot = reinterpret_cast<int*>(gbase + kOffBar + 132);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int item, sg, nseg_i;
    if (STATE) {
        item = p.n_whole + static_cast<int>(blockIdx.x) / (p.nseg - 1);
        sg = static_cast<int>(blockIdx.x) % (p.nseg - 1);
        nseg_i = p.nseg;
    } else if (static_cast<int>(blockIdx.x) < p.n_whole) {
        item = static_cast<int>(blockIdx.x);
        sg = 0;
        nseg_i = 1;
    } else {
        const int j = static_cast<int>(blockIdx.x) - p.n_whole;
        item = p.n_whole + j / p.nseg;
        sg = j % p.nseg;
        nseg_i = p.nseg;
    }
    const int64_t rk = item - p.n_whole;   // rank among the split items (records, Σ Δ A)
    const int h = item % p.H;
    const int b = item / p.H;
    const int64_t bh = static_cast<int64_t>(b) * p.H + h;
    const int64_t seg_t0 = nseg_i == 1 ? 0 : static_cast<int64_t>(sg) * p.cseg * kQ;
    const int64_t seg_t1 = nseg_i == 1 ? p.L : min(seg_t0 + static_cast<int64_t>(p.cseg) * kQ, p.L);
    const int nchunk = static_cast<int>((seg_t1 - seg_t0 + kQ - 1) / kQ);
    const uint64_t lim = p.wait_ns;

    if (tid == 0) {
        for (int i = 0; i < 16; ++i) mbar_init(bars + i, (i == 8 || i == 9) ? static_cast<uint32_t>(kComputeWarps) : 1u);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (p.n < kN) {   // d_state 64: B and C keep their second 64-column block at zero (TMA fills the first)
        for (int i = tid; i < 2 * 1024; i += kThreads) {
            const uint32_t blk = (i < 1024) ? kOffB + 16384u : kOffC + 16384u;
            sts128(base + blk + static_cast<uint32_t>(i & 1023) * 16u, make_uint4(0, 0, 0, 0));
        }
        fence_proxy_async_smem();   // before the MMAs read them (ordered by the barrier below)
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    auto record = [&]() {
        ok = false;
        if (p.status) atomicCAS(p.status, 0u, static_cast<uint32_t>(-4));
    };
    // tile copies issued / waited for, per tensor (producer's counts; x waits are the compute warps')
    int x_issued = 0, b_issued = 0, c_issued = 0, b_waited = 0, c_waited = 0;

    if (warp == kProducerWarp) {
        // =============================================================== producer (one thread)
        if (lane == 0) {
            auto chunk_t0 = [&](int ci) { return static_cast<int>(seg_t0 + static_cast<int64_t>(ci) * kQ); };
            auto issue_x = [&](int ci) {
                uint64_t* bar = x_full + (ci & 1);
                mbar_arrive_expect_tx(bar, kQ * kP * 2);
                tma_load_4d(base + ((ci & 1) ? kOffX1 : kOffX0), &tm_x, 0, h, chunk_t0(ci), b, bar);
            };
            const bool two = p.n == kN;   // B and C rows of 128 states: two 64-wide boxes
            auto issue_b = [&](int ci) {
                mbar_arrive_expect_tx(b_full, (two ? 2 : 1) * kQ * 64 * 2);
                tma_load_3d_u(base + kOffB, &tm_B, 0, chunk_t0(ci), b, b_full);
                if (two) tma_load_3d_u(base + kOffB + 16384, &tm_B, 64, chunk_t0(ci), b, b_full);
            };
            auto issue_c = [&](int ci) {
                mbar_arrive_expect_tx(c_full, (two ? 2 : 1) * kQ * 64 * 2);
                tma_load_3d_u(base + kOffC, &tm_C, 0, chunk_t0(ci), b, c_full);
                if (two) tma_load_3d_u(base + kOffC + 16384, &tm_C, 64, chunk_t0(ci), b, c_full);
            };
            auto pw_wait = [&](uint64_t* bar, uint32_t parity) {
                if (mbar_wait_bounded(bar, parity, lim)) return true;
                record();
                return false;
            };
            if (nchunk > 0) {
                tma_prefetch_desc(&tm_x);
                tma_prefetch_desc(&tm_B);
                if (!STATE) tma_prefetch_desc(&tm_C);
                issue_x(0);
                if (nchunk > 1) issue_x(1);
                issue_b(0);
                if (!STATE) issue_c(0);
                x_issued = nchunk > 1 ? 2 : 1;
                b_issued = 1;
                c_issued = STATE ? 0 : 1;
            }
            for (int ci = 0; ci < nchunk; ++ci) {
                const bool carry = !STATE && (ci > 0 || sg > 0);
                const bool more = ci + 1 < nchunk;
                const uint32_t par = static_cast<uint32_t>(ci & 1);
                if (!pw_wait(b_full, par)) break;
                ++b_waited;
                if (!STATE) {
                    if (!pw_wait(c_full, par)) break;
                    ++c_waited;
                    // S = C Bᵀ (its columns were last read by the previous chunk's mask)
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < kN / 16; ++k) {
                        const uint32_t off = (k >> 2) * 16384u + (k & 3) * 32u;
                        umma(tmem + kColS, sdesc(base + kOffC + off, 16, 1024), sdesc(base + kOffB + off, 16, 1024),
                             kIdesc_128x128_KK, k > 0);
                    }
                    if (!(p.test_drop && blockIdx.x == 0 && ci == 0)) umma_commit(s_full);
                }
                // the previous chunk's epilogue (for ci = 0, the compute warps' set-up)
                if (!pw_wait(ep_done, par)) break;
                if (ci >= 1 && more) {   // x buffer (ci + 1) & 1 was chunk ci - 1's
                    issue_x(ci + 1);
                    ++x_issued;
                }
                if (!STATE) {   // CG = C G_hiᵀ + C G_loᵀ, both accumulated into the same 64 columns
                    tc_fence_after();
                    if (carry) {
#pragma unroll
                        for (int k = 0; k < kN / 16; ++k) {
                            const uint32_t aoff = (k >> 2) * 16384u + (k & 3) * 32u;
                            const uint64_t ad = sdesc(base + kOffC + aoff, 16, 1024);
                            umma(tmem + kColCG, ad, sdesc(base + kOffGh + k * 2048u, 0, 1024), kIdesc_128x64_KMN, k > 0);
                            umma(tmem + kColCG, ad, sdesc(base + kOffGl + k * 2048u, 0, 1024), kIdesc_128x64_KMN, 1);
                        }
                    }
                    umma_commit(cg_done);
                }
                if (!pw_wait(xt_ready, par)) break;
                tc_fence_after();   // ΔGᵀ = Bᵀ X̃
#pragma unroll
                for (int k = 0; k < kQ / 16; ++k)
                    umma(tmem + kColG, sdesc(base + kOffB + k * 2048u, 16384, 1024),
                         sdesc(base + kOffXt + k * 2048u, 0, 1024), kIdesc_128x64_MNMN, k > 0);
                umma_commit(dg_done);
                if (!STATE && more) {
                    if (!pw_wait(cg_done, par)) break;
                    issue_c(ci + 1);
                    ++c_issued;
                }
                if (more) {
                    if (!pw_wait(dg_done, par)) break;
                    issue_b(ci + 1);
                    ++b_issued;
                }
                if (!STATE) {
                    if (!pw_wait(mm_ready, par)) break;
                    tc_fence_after();   // Y = Mm X
                    const uint32_t xbase = base + ((ci & 1) ? kOffX1 : kOffX0);
#pragma unroll
                    for (int k = 0; k < kQ / 16; ++k) {
                        const uint32_t aoff = (k >> 2) * 16384u + (k & 3) * 32u;
                        umma(tmem + kColY, sdesc(base + kOffM + aoff, 16, 1024), sdesc(xbase + k * 2048u, 0, 1024),
                             kIdesc_128x64_KMN, k > 0);
                    }
                    umma_commit(y_done);
                }
            }
        }
        __syncwarp();
    } else if (warp == kPrefixWarp) {
        // =============================================================== Δ prefix warp
        const float Ah = p.A[h];
        const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
        // Δraw of the chunk's steps 4·lane .. 4·lane + 3, kept as raw bf16 bits
        // (widened where used, so the load's latency stays off the chunk it is fetched in)
        uint32_t dtn[4] = {0u, 0u, 0u, 0u};
        auto load_dt = [&](int ci) {
            const int64_t t0 = seg_t0 + static_cast<int64_t>(ci) * kQ;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t t = t0 + 4 * lane + e;
                dtn[e] = t < p.L ? reinterpret_cast<const unsigned short*>(p.dt)[(static_cast<int64_t>(b) * p.L + t) *
                                                                                     p.H + h]
                                 : 0u;
            }
        };
        // Δ, the inclusive prefix of Δ A and the block factors of chunk ci into buffer ci & 1
        // (four steps per lane, one warp scan); then Δraw of chunk ci + 1.
        auto prefix = [&](int ci) {
            const int64_t t0 = seg_t0 + static_cast<int64_t>(ci) * kQ;
            const int q = static_cast<int>(p.L - t0 < kQ ? p.L - t0 : kQ);
            float dl[4], a[4], run = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // softplus through the hardware ex2 / lg2: log1p(e^x) = ln 2 · log2(1 + 2^(x log2 e)),
                // identity above x = 20 (well inside the bf16 outputs' precision)
                const float xr = __uint_as_float(dtn[e] << 16) + bias;
                const float spv = (xr > 20.0f) ? xr : kLn2 * lg2_approx(1.0f + ex2_approx(xr * kLog2e));
                dl[e] = (4 * lane + e < q) ? (p.softplus ? spv : xr) : 0.0f;
                run = fmaf(dl[e], Ah, run);
                a[e] = run;
            }
            float sc = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, sc, o);
                if (lane >= o) sc += v;
            }
            const float excl = sc - run;
            const int o = (ci & 1) * kQ + 4 * lane;
            float c2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) c2[e] = (excl + a[e]) * kLog2e;
            const float c2_end = __shfl_sync(0xffffffffu, c2[3], lane | 7);   // step 32·(lane / 8) + 31
            const float c2_tot = __shfl_sync(0xffffffffu, c2[3], 31);         // the chunk's last step
            *reinterpret_cast<float4*>(cum2 + o) = make_float4(excl + a[0], excl + a[1], excl + a[2], excl + a[3]);
            *reinterpret_cast<float4*>(cs2 + o) = make_float4(c2[0], c2[1], c2[2], c2[3]);
            *reinterpret_cast<float4*>(dlt2 + o) = make_float4(dl[0], dl[1], dl[2], dl[3]);
            *reinterpret_cast<float4*>(cf2 + o) =
                make_float4(ex2_approx(c2_end - c2[0]) * dl[0], ex2_approx(c2_end - c2[1]) * dl[1],
                            ex2_approx(c2_end - c2[2]) * dl[2], ex2_approx(c2_end - c2[3]) * dl[3]);
            *reinterpret_cast<float4*>(wx2 + o) =
                make_float4(ex2_approx(c2_tot - c2[0]) * dl[0], ex2_approx(c2_tot - c2[1]) * dl[1],
                            ex2_approx(c2_tot - c2[2]) * dl[2], ex2_approx(c2_tot - c2[3]) * dl[3]);
            if (ci + 1 < nchunk) load_dt(ci + 1);
            __syncwarp();
            if (lane == 0) mbar_arrive(pf_full + (ci & 1));   // release: the writes above precede it
        };
        if (nchunk > 0) load_dt(0);
        for (int ci = 0; ci < nchunk; ++ci) {
            if (ci >= 2) {   // buffer ci & 1 was chunk ci - 2's
                bool got = true;
                if (lane == 0) got = mbar_wait_bounded(pf_empty + (ci & 1), static_cast<uint32_t>(((ci >> 1) - 1) & 1), lim);
                got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    if (lane == 0) record();
                    break;
                }
            }
            prefix(ci);
        }
    } else {
        // =============================================================== compute warps
        const int row = tid & (kRows - 1);   // TMEM lane / tile row of this thread
        const int qc = tid >> 7;             // which quarter of the row's columns
        const int rb = warp & 3;             // this warp's 32-row block
        const uint32_t lane_base = static_cast<uint32_t>(rb * 32) << 16;   // this warp's TMEM lanes
        const float Dh = p.D ? p.D[h] : 0.0f;
        // Carried state: thread (n, qc) holds G[16 qc .. 16 qc + 15, n] (fp32).
        // Entering a segment > 0 of the main pass it is the folded record, else zero.
        // (d_state 64: rows n >= 64 stay zero -- their B and C columns are zero)
        float G[kPT];
        const int nn = p.n;
        const float* gin = (!STATE && sg > 0) ? p.rec + (rk * (p.nseg - 1) + (sg - 1)) * kP * nn : nullptr;
#pragma unroll
        for (int q = 0; q < kPT; ++q) G[q] = (gin && row < nn) ? gin[(kPT * qc + q) * nn + row] : 0.0f;
        auto store_g = [&]() {   // bf16 hi / lo copies of G: row n, chunks 2 qc, 2 qc + 1 of the [n][p] tiles
#pragma unroll
            for (int c = 0; c < kXC; ++c) {
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float g0 = G[8 * c + 2 * e], g1 = G[8 * c + 2 * e + 1];
                    hw[e] = pk(g0, g1);
                    lw[e] = pk(g0 - lo_f(hw[e]), g1 - hi_f(hw[e]));
                }
                sts128(chunk_addr(base + kOffGh, row, kXC * qc + c), make_uint4(hw[0], hw[1], hw[2], hw[3]));
                sts128(chunk_addr(base + kOffGl, row, kXC * qc + c), make_uint4(lw[0], lw[1], lw[2], lw[3]));
            }
        };
        if (gin) store_g();
        if (!STATE) {   // Mm right of the diagonal is zero in every chunk: written once
            const int rb0 = warp & 3;
#pragma unroll 1
            for (int g = kSB * qc; g < kSB * qc + kSB; ++g) {
                if (g <= rb0) continue;
                const uint32_t blk = base + kOffM + static_cast<uint32_t>(g >> 1) * 16384u;
#pragma unroll
                for (int c = 0; c < 4; ++c) sts128(chunk_addr(blk, row, (g & 1) * 4 + c), make_uint4(0, 0, 0, 0));
            }
        }
        fence_proxy_async_smem();   // G copies and the zero blocks (generic writes) before the MMAs read them
        cw_sync();
        if (tid == 0) mbar_arrive(ep_done);

        // every thread waits; one barrier over the compute warps makes the outcome uniform
        auto cw_wait2 = [&](uint64_t* bar0, uint32_t par0, uint64_t* bar1, uint32_t par1) {
            bool got = bar0 ? mbar_wait_bounded(bar0, par0, lim) : true;
            if (got && bar1) got = mbar_wait_bounded(bar1, par1, lim);
            const bool bad = cw_any(!got);
            if (bad) {
                ok = false;
                if (tid == 0) record();
            }
            return !bad;
        };
        float esum = 0.0f;
        int x_waited = 0;
        for (int ci = 0; ci < nchunk; ++ci) {
            const int64_t t0 = seg_t0 + static_cast<int64_t>(ci) * kQ;
            const int xb = ci & 1;
            const uint32_t par = static_cast<uint32_t>(xb);
            const uint32_t xbase = base + (xb ? kOffX1 : kOffX0);
            const bool carry = !STATE && (ci > 0 || sg > 0);
            const float* cum = cum2 + xb * kQ;
            const float* cs = cs2 + xb * kQ;
            const float* dlt = dlt2 + xb * kQ;
            const float* cf = cf2 + xb * kQ;
            if (!cw_wait2(x_full + xb, static_cast<uint32_t>((ci >> 1) & 1), pf_full + xb, static_cast<uint32_t>((ci >> 1) & 1)))
                break;
            ++x_waited;
            const float cum_end = cum[kQ - 1];
            if (STATE) esum += cum_end;

            {   // -------- X̃[s, :] = e^{cum_end - cum_s} Δ_s x_s (row s, chunks 2 qc, 2 qc + 1; a per-row
                // scale, so every 16-byte chunk keeps its place; addressed through the swizzle so that eight
                // consecutive rows hit eight bank groups).  X̃ was last read by the previous chunk's Bᵀ X̃,
                // waited for below.
                const int sr = row;
                const float w = wx2[xb * kQ + sr];
#pragma unroll
                for (int c = kXC * qc; c < kXC * qc + kXC; ++c) {
                    const uint4 v = lds128(chunk_addr(xbase, sr, c));
                    const uint4 o = make_uint4(pk(lo_f(v.x) * w, hi_f(v.x) * w), pk(lo_f(v.y) * w, hi_f(v.y) * w),
                                               pk(lo_f(v.z) * w, hi_f(v.z) * w), pk(lo_f(v.w) * w, hi_f(v.w) * w));
                    sts128(chunk_addr(base + kOffXt, sr, c), o);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(xt_ready);
            }
            if (!STATE) {
                // -------- Mm = S ∘ decay mask (row t, 32-column block qc).  Blocks right of the
                // diagonal are zero.  Strictly below it every s <= t, and the decay factors through the
                // block's last step r: e^{cum_t - cum_s} = e^{cum_t - cum_r} e^{cum_r - cum_s}, both factors
                // between the exact value and 1, so neither overflows nor loses the product.  The diagonal
                // block takes e^{cum_t - cum_s} per element.  Mm was last read by the previous chunk's Mm X.
                if (!cw_wait2(s_full, par, nullptr, 0)) break;
                tc_fence_after();
                const int t = row;
                const float ct = cs[t];
#pragma unroll 1
                for (int gi = 0; gi < kSB; ++gi) {
                    const int g = kSB * qc + gi;
                    const uint32_t blk = base + kOffM + static_cast<uint32_t>(g >> 1) * 16384u;
                    const int c0 = (g & 1) * 4;
                    if (g > rb) continue;   // zero, written before the first chunk
                    float sv[32];
                    tmem_ld32(tmem + lane_base + kColS + 32 * g, sv);
                    if (g < rb) {
                        const float rf = ex2_approx(ct - cs[32 * g + 31]);
                        const float2 rf2 = make_float2(rf, rf);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float4 fa = *reinterpret_cast<const float4*>(cf + 32 * g + 8 * c);
                            const float4 fb = *reinterpret_cast<const float4*>(cf + 32 * g + 8 * c + 4);
                            const float2 f2[4] = {make_float2(fa.x, fa.y), make_float2(fa.z, fa.w),
                                                  make_float2(fb.x, fb.y), make_float2(fb.z, fb.w)};
                            uint32_t wv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 m2 = __fmul2_rn(
                                    __fmul2_rn(make_float2(sv[8 * c + 2 * e], sv[8 * c + 2 * e + 1]), f2[e]), rf2);
                                wv[e] = pk(m2.x, m2.y);
                            }
                            sts128(chunk_addr(blk, t, c0 + c), make_uint4(wv[0], wv[1], wv[2], wv[3]));
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int s0 = 32 * g + 8 * c;
                            const float4 ca = *reinterpret_cast<const float4*>(cs + s0);
                            const float4 cb = *reinterpret_cast<const float4*>(cs + s0 + 4);
                            const float4 da = *reinterpret_cast<const float4*>(dlt + s0);
                            const float4 db = *reinterpret_cast<const float4*>(dlt + s0 + 4);
                            const float csv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                            const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
                            uint32_t wv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float m2[2];
#pragma unroll
                                for (int f = 0; f < 2; ++f) {
                                    const int i = 2 * e + f;
                                    m2[f] = (s0 + i <= t) ? sv[8 * c + i] * ex2_approx(ct - csv[i]) * dv[i] : 0.0f;
                                }
                                wv[e] = pk(m2[0], m2[1]);
                            }
                            sts128(chunk_addr(blk, t, c0 + c), make_uint4(wv[0], wv[1], wv[2], wv[3]));
                        }
                    }
                }
                fence_proxy_async_smem();   // Mm before the MMA reads it
                tc_fence_before();          // S read before its columns are written again
                __syncwarp();
                if (lane == 0) mbar_arrive(mm_ready);
            }
            // -------- G = e^{cum_end} G + ΔGᵀ[n, :] (row n, columns 16 qc .. 16 qc + 15), once Bᵀ X̃ is
            // done and C Gᵀ has read the previous copies of G
            if (!cw_wait2(STATE ? nullptr : cg_done, par, dg_done, par)) break;
            tc_fence_after();
            {
                const float e_end = __expf(cum_end);
                float dg[kPT];
                tmem_ld16(tmem + lane_base + kColG + kPT * qc, dg);
#pragma unroll
                for (int j = 0; j < kPT; ++j) G[j] = fmaf(e_end, G[j], dg[j]);
                if (!STATE) store_g();
            }
            if (!STATE) {
                // -------- y = Y + e^{cum_t} CG + D x (row t, columns 16 qc .. 16 qc + 15) into the staging tile
                if (tid == 0) bulk_wait_read0();   // the previous chunk's y tile has left shared memory
                if (!cw_wait2(y_done, par, nullptr, 0)) break;
                tc_fence_after();
                const int t = row;
                const float et = __expf(cum[t]);
                float acc[kPT];
                {   // Y and C Gᵀ in one TMEM round trip
                    float yg[2 * kPT];
                    tmem_ld16x2(tmem + lane_base + kColY + kPT * qc, tmem + lane_base + kColCG + kPT * qc, yg);
#pragma unroll
                    for (int j = 0; j < kPT; ++j) acc[j] = carry ? fmaf(et, yg[kPT + j], yg[j]) : yg[j];
                }
                uint4 xv[kXC];
#pragma unroll
                for (int c = 0; c < kXC; ++c) xv[c] = lds128(chunk_addr(xbase, t, kXC * qc + c));
#pragma unroll
                for (int c = 0; c < kXC; ++c) {
                    const uint32_t xw[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * c + 2 * e;
                        ow[e] = pk(fmaf(Dh, lo_f(xw[e]), acc[j]), fmaf(Dh, hi_f(xw[e]), acc[j + 1]));
                    }
                    sts128(chunk_addr(base + kOffY, t, kXC * qc + c), make_uint4(ow[0], ow[1], ow[2], ow[3]));
                }
            }
            fence_proxy_async_smem();   // G copies and the y tile before the async proxy reads them
            tc_fence_before();          // TMEM reads before the columns are written again
            cw_sync();
            if (tid == 0) {
                if (!STATE) {   // this chunk's y rows (rows past the sequence's end are clipped)
                    tma_store_4d(&tm_y, base + kOffY, 0, h, static_cast<int>(t0), b);
                    bulk_commit();
                }
                mbar_arrive(ep_done);
                mbar_arrive(pf_empty + xb);
            }
        }
        // outputs of the state: the segment's G_out (state pass) or the final state
        if (ok) {
            float* out = nullptr;
            if (STATE) out = p.rec + (rk * (p.nseg - 1) + sg) * kP * nn;
            else if (p.final_state && sg == nseg_i - 1) out = p.final_state + bh * kP * nn;
            if (out && row < nn) {
#pragma unroll
                for (int q2 = 0; q2 < kPT; ++q2) out[(kPT * qc + q2) * nn + row] = G[q2];
            }
            if (STATE && tid == 0) p.esum[rk * p.nseg + sg] = esum;
        }
        if (tid == 0) {
            if (!STATE) bulk_wait0();
            *xw_slot = x_waited;
        }
    }

    // Wind-down.  Copies still in flight land before the shared memory is
    // released, and every MMA issued completes before the TMEM columns are
    // (both bounded; a completed phase is recognised as well).
    __syncthreads();
    if (warp == kProducerWarp && lane == 0) {
        const uint64_t dlim = p.drain_ns;
        for (int cj = *xw_slot; cj < x_issued; ++cj)   // chunk cj's x: buffer cj & 1, phase cj >> 1
            mbar_wait_bounded(x_full + (cj & 1), static_cast<uint32_t>((cj >> 1) & 1), dlim);
        if (b_waited < b_issued) mbar_wait_bounded(b_full, static_cast<uint32_t>(b_waited & 1), dlim);
        if (c_waited < c_issued) mbar_wait_bounded(c_full, static_cast<uint32_t>(c_waited & 1), dlim);
        umma_commit(fin_bar);
        mbar_wait_bounded(fin_bar, 0, dlim);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tc
}  // namespace selscan
