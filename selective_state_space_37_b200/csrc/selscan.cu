// selscan.cu -- the C ABI of libselscan (declared in include/selscan.h):
// argument validation, work decomposition, workspace layout, TMA descriptor
// set-up and kernel launches.  No allocation happens here: every buffer,
// including the workspace, belongs to the caller.
#include <cublas_v2.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/selscan.h"
#include "block.cuh"
#include "bwd.cuh"
#include "fwd.cuh"
#include "ssd.cuh"
#include "ssd_tc.cuh"
#include "step.cuh"

using namespace selscan;

namespace {

constexpr int kVersion = 10000;             // 1.0.0
constexpr size_t kHeaderBytes = 256;        // error word, ticket counter, provisional-item count
constexpr uint32_t kDefaultPolls = 1u << 21;
constexpr uint64_t kTmaWaitNs = 2000000000ull;
constexpr int kMaxDevices = 64;
constexpr uint32_t kKnownFlags = SS_BF16 | SS_DELTA_SOFTPLUS | SS_SYNC_CHECK | SS_FORCE_GENERAL_A |
                                 SS_TEST_DROP_CARRY;

// Per-device caches below are atomics: host threads may make their first
// calls concurrently (they store the same values).
int sm_count_of_current_device() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < kMaxDevices) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Raises a kernel's dynamic shared-memory limit to `smem` once per device.
template <typename Kern>
int set_smem_limit(Kern kern, size_t smem, std::atomic<bool> (&done)[kMaxDevices], int dev) {
    const bool cached = dev >= 0 && dev < kMaxDevices;
    if (cached && done[dev].load(std::memory_order_acquire)) return SS_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
        return SS_ERR_CUDA;
    if (cached) done[dev].store(true, std::memory_order_release);
    return SS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Forward-kernel variants.  Wide: one resident CTA per SM (two warps per
// scheduler), a 2-stage tile ring, groups of 4 steps with whole tiles
// unrolled -- fastest when every SM can work on channels whose entry state is
// known.  Narrow: two resident CTAs per SM (four warps per scheduler, <= 128
// registers), a 3-stage ring, groups of 8 with the 32-step tile unrolled --
// better latency hiding when a problem has few channel blocks, so that almost
// every time chunk is provisional anyway.
enum Variant { kWide = 0, kNarrow = 1 };
constexpr int kCtasPerSm[2] = {1, 2};
// Items per resident CTA slot the automatic chunking aims for (load balance:
// the last wave is at most 1/kWaves of the work), and the shortest chunk.
constexpr int64_t kWaves = 8;
constexpr int64_t kMinChunk = 256;

// Variant and automatic number of time chunks for these sizes.
struct Choice {
    Variant v;
    int64_t nchunks;   // 1: no time chunking
};

Choice choose(const ss_dims* dims, uint32_t flags) {
    const int64_t L = dims->seqlen;
    const int64_t nblk = ceil_div(std::max<int64_t>(dims->d_inner, 1), kCB);
    const int64_t base = std::max<int64_t>(dims->batch * nblk, 1);
    const int64_t sms = sm_count_of_current_device();
    const bool bf16 = (flags & SS_BF16) != 0;
    Choice ch{kWide, 1};
    if (base >= sms || !bf16) {
        ch.nchunks = ceil_div(kWaves * sms * kCtasPerSm[kWide], base);
    } else if (2 * base >= sms) {
        // Between half and all of the SMs have a channel block: scanning each
        // sequence whole on those SMs beats chunking, whose extra chunks start
        // before their predecessors end and pay for a fix-up pass (measured on
        // the 130M-shaped layer, 96 blocks on 148 SMs: 0.186 ms unchunked,
        // 0.274 ms with two chunks).
        ch.nchunks = 1;
    } else {
        ch.v = kNarrow;
        ch.nchunks = ceil_div(kWaves * sms * kCtasPerSm[kNarrow], base);
    }
    const int64_t max_chunks = std::max<int64_t>(L / kMinChunk, 1);
    ch.nchunks = std::min(ch.nchunks, max_chunks);
    return ch;
}

// Library choice of chunk length; 0 = no time chunking.
int32_t auto_chunk_len(const ss_dims* dims, uint32_t flags) {
    const int64_t L = dims->seqlen;
    if (L <= kMinChunk) return 0;
    const Choice ch = choose(dims, flags);
    if (ch.nchunks <= 1) return 0;
    int64_t chunk = ceil_div(ceil_div(L, ch.nchunks), kTT) * kTT;
    if (chunk >= L) return 0;
    if (chunk > (1 << 30)) chunk = 1 << 30;
    return static_cast<int32_t>(chunk);
}

struct Plan {
    int64_t chunk_len;   // 0: unchunked
    int64_t nchunks;
    int64_t nblk;
    size_t status_off, status_bytes, rec_off, rec_bytes, total;
};

Plan make_plan(const ss_dims* dims, uint32_t flags, int32_t chunk_req) {
    Plan pl{};
    const int64_t L = dims->seqlen;
    pl.nblk = ceil_div(std::max<int64_t>(dims->d_inner, 1), kCB);
    int64_t chunk = chunk_req > 0 ? ceil_div(chunk_req, kTT) * kTT : auto_chunk_len(dims, flags);
    if (chunk <= 0 || chunk >= L) chunk = 0;
    pl.chunk_len = chunk;
    pl.nchunks = chunk > 0 ? ceil_div(L, chunk) : 1;
    pl.status_off = kHeaderBytes;
    if (pl.nchunks > 1) {
        pl.status_bytes = static_cast<size_t>(dims->batch * pl.nchunks * pl.nblk) * sizeof(uint32_t);
        pl.rec_off = (pl.status_off + pl.status_bytes + 255) / 256 * 256;
        pl.rec_bytes = static_cast<size_t>(dims->batch * pl.nchunks * dims->d_inner) * kRec * sizeof(float);
        pl.total = pl.rec_off + pl.rec_bytes;
    } else {
        pl.status_bytes = 0;
        pl.rec_off = kHeaderBytes;
        pl.rec_bytes = 0;
        pl.total = kHeaderBytes;
    }
    return pl;
}

// ------------------------------------------------------------ TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over a [batch, rows, inner] row-major tensor, box [1, box_rows, box_inner].
bool make_map(CUtensorMap* m, const void* base, bool bf16, uint64_t inner, uint64_t rows, uint64_t batch,
              uint32_t box_inner, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const uint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[3] = {inner, rows, batch};
    cuuint64_t strides[2] = {inner * es, rows * inner * es};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                           const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename IO, bool TMA, int STAGES, int MINB, int G, bool UNROLL, bool CONV, bool FULL = false>
int launch_fwd(const FwdParams& p, int64_t items, const CUtensorMap* maps, cudaStream_t stream) {
    auto kern = ss_fwd_kernel<IO, TMA, STAGES, MINB, G, UNROLL, CONV, FULL>;
    const size_t smem = sizeof(FwdSmem<IO, STAGES>);
    static std::atomic<bool> attr_set[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || set_smem_limit(kern, smem, attr_set, dev) != SS_OK) return SS_ERR_CUDA;
    kern<<<static_cast<unsigned>(items), kNT, smem, stream>>>(p, maps[0], maps[1], maps[2], maps[3], maps[4],
                                                              maps[5]);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// Forward-kernel instantiation for the variant, element type, TMA use, the
// conv prologue and (bf16) whether the softplus and the gate are both on.
template <bool CONV, bool FULL>
int launch_bf16(bool tma, Variant v, const FwdParams& p, int64_t items, const CUtensorMap* maps, cudaStream_t stream) {
    if (v == kNarrow)
        return tma ? launch_fwd<__nv_bfloat16, true, 3, 2, 8, true, CONV, FULL>(p, items, maps, stream)
                   : launch_fwd<__nv_bfloat16, false, 1, 2, 4, false, CONV, FULL>(p, items, maps, stream);
    return tma ? launch_fwd<__nv_bfloat16, true, 2, 1, 4, true, CONV, FULL>(p, items, maps, stream)
               : launch_fwd<__nv_bfloat16, false, 1, 1, 8, true, CONV, FULL>(p, items, maps, stream);
}

template <bool CONV>
int launch_variant(bool bf16, bool tma, Variant v, const FwdParams& p, int64_t items, const CUtensorMap* maps,
                   cudaStream_t stream) {
    if (bf16) {
        const bool full = (p.pflags & kPfSoftplus) && (p.pflags & kPfHasZ);
        return full ? launch_bf16<CONV, true>(tma, v, p, items, maps, stream)
                    : launch_bf16<CONV, false>(tma, v, p, items, maps, stream);
    }
    return tma ? launch_fwd<float, true, 2, 1, 8, false, CONV>(p, items, maps, stream)
               : launch_fwd<float, false, 1, 1, 8, false, CONV>(p, items, maps, stream);
}

// SSD workspace: a 256-byte header (word 0: the device status word), then,
// for up to kSsdMaxSeg time segments per sequence, the segment end-state
// records [batch, H, kmax - 1, P, N] fp32 and Σ Δ A per segment
// [batch, H, kmax]; each region 256-byte aligned.  kmax counts 64-step
// chunks, so it also covers the tensor-core kernel's 128-step chunks.
constexpr int64_t kSsdMaxSeg = 8;
struct SsdLayout {
    size_t rec, esum, total;
    int64_t nchunks, kmax;
};
SsdLayout ssd_layout(const ss_ssd_dims* d) {
    SsdLayout w{};
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    w.nchunks = ceil_div(std::max<int64_t>(d->seqlen, 1), kSsdQ);
    w.kmax = std::min(kSsdMaxSeg, w.nchunks);
    const int64_t bh = d->batch * d->nheads;
    w.rec = kHeaderBytes;
    w.esum = w.rec + al(static_cast<size_t>(bh * (w.kmax - 1) * kSsdP * d->d_state) * sizeof(float));
    w.total = w.esum + al(static_cast<size_t>(bh * w.kmax) * sizeof(float));
    return w;
}

// SELSCAN_SSD_MMA_SYNC=1 builds the SSD scan on the warp-level mma.sync
// kernel of ssd.cuh instead of the tcgen05 one (comparisons).
#ifndef SELSCAN_SSD_MMA_SYNC
#define SELSCAN_SSD_MMA_SYNC 0
#endif

// Tensor map of a row-major tensor of `rank` dimensions (innermost first,
// byte strides of dimensions 1..rank-1), bf16, 128-byte swizzle, box `box`.
bool make_map_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                    const cuuint32_t* box) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The tcgen05 scan (d_state 128): segments of whole 128-step chunks chosen
// like launch_ssd's (one resident CTA per SM; state pass charged half a
// chunk, splitting 10 %), then the state pass, the fold and the main pass.
int launch_ssd_tc(const tc::Params& base_p, const SsdParams& fold_p, const void* x, const void* B, const void* C,
                  int64_t items, const SsdLayout& w, int32_t chunk_len, bool have_ws, cudaStream_t stream) {
    tc::Params p = base_p;
    const int64_t L = p.L;
    const int64_t nchunks = ceil_div(std::max<int64_t>(L, 1), tc::kQ);
    const int64_t kmax = std::min<int64_t>(w.kmax, nchunks);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
    auto kmain = tc::ss_ssd_tc_kernel<false>;
    auto kstate = tc::ss_ssd_tc_kernel<true>;
    static std::atomic<bool> attr_main[kMaxDevices];
    static std::atomic<bool> attr_state[kMaxDevices];
    if (set_smem_limit(kmain, tc::kSmemBytes, attr_main, dev) != SS_OK ||
        set_smem_limit(kstate, tc::kSmemBytes, attr_state, dev) != SS_OK)
        return SS_ERR_CUDA;
    // Plan: items 0 .. n_whole - 1 run whole; the others are cut into nseg segments of cseg chunks
    // (a state pass over the first nseg - 1, a fold, then every segment from its exact entering state).
    int64_t n_whole = items, nseg = 1, cseg = nchunks;
    if (have_ws && nchunks > 1) {
        const int64_t slots = sm_count_of_current_device();
        if (chunk_len > 0) {   // forced segment length: every item is cut
            int64_t cs = std::max<int64_t>(1, ceil_div(chunk_len, tc::kQ));
            if (ceil_div(nchunks, cs) > kmax) cs = ceil_div(nchunks, kmax);
            cseg = cs;
            nseg = ceil_div(nchunks, cs);
            n_whole = nseg > 1 ? 0 : items;
        } else {
            // Cost in chunk-times of the busiest SM (one CTA per SM): every item whole; every item cut into
            // k segments; or only the items of the last, partly filled wave cut, so that their segments
            // fill that wave.  Cut items add a state pass over k - 1 segments (about half the work of a
            // chunk per chunk) and 10 % for the extra launches.
            const int64_t waves = items / slots, tail = items - waves * slots;
            auto cut_cost = [&](int64_t n, int64_t k, int64_t cs) {
                return 1.1 * static_cast<double>(ceil_div(n * k, slots) * cs +
                                                 ceil_div(n * (k - 1), slots) * cs / 2.0);
            };
            double best = static_cast<double>(ceil_div(items, slots) * nchunks);
            for (int64_t k = 2; k <= kmax; ++k) {
                const int64_t cs = ceil_div(nchunks, k);
                if (ceil_div(nchunks, cs) != k) continue;
                const double every = cut_cost(items, k, cs);
                if (every < best - 1e-9) {
                    best = every;
                    n_whole = 0;
                    nseg = k;
                    cseg = cs;
                }
                if (waves >= 1 && tail > 0) {
                    const double last = static_cast<double>(waves * nchunks) + cut_cost(tail, k, cs);
                    if (last < best - 1e-9) {
                        best = last;
                        n_whole = items - tail;
                        nseg = k;
                        cseg = cs;
                    }
                }
            }
        }
    }
    const int64_t n_cut = nseg > 1 ? items - n_whole : 0;
    if (nseg == 1) n_whole = items;
    const int64_t grid = n_whole + n_cut * nseg;
    if (grid >= (int64_t(1) << 31)) return SS_ERR_INVALID_ARG;
    p.n_whole = static_cast<int>(n_whole);
    p.nseg = static_cast<int>(nseg);
    p.cseg = static_cast<int>(cseg);
    const int64_t H = p.H, batch = p.batch;
    CUtensorMap mx, mb, mc, my;
    {
        const cuuint64_t dx[4] = {static_cast<cuuint64_t>(tc::kP), static_cast<cuuint64_t>(H),
                                  static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(batch)};
        const cuuint64_t sx[3] = {static_cast<cuuint64_t>(tc::kP * 2), static_cast<cuuint64_t>(H * tc::kP * 2),
                                  static_cast<cuuint64_t>(L * H * tc::kP * 2)};
        const cuuint32_t bx[4] = {64, 1, static_cast<cuuint32_t>(tc::kQ), 1};
        const int64_t N = p.n;   // 128, or 64 (one 64-wide box per row)
        const cuuint64_t db[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(L),
                                  static_cast<cuuint64_t>(batch)};
        const cuuint64_t sb[2] = {static_cast<cuuint64_t>(N * 2), static_cast<cuuint64_t>(L * N * 2)};
        const cuuint32_t bb[3] = {64, static_cast<cuuint32_t>(tc::kQ), 1};
        if (!make_map_sw128(&mx, x, 4, dx, sx, bx) || !make_map_sw128(&mb, B, 3, db, sb, bb) ||
            !make_map_sw128(&mc, C, 3, db, sb, bb) || !make_map_sw128(&my, p.y, 4, dx, sx, bx))
            return SS_ERR_CUDA;
    }
    if (n_cut > 0) {
        kstate<<<static_cast<unsigned>(n_cut * (nseg - 1)), tc::kThreads, tc::kSmemBytes, stream>>>(p, mx, mb, mc, my);
        SsdParams f = fold_p;   // the fold runs over the cut items' records (their ranks as one batch row)
        f.batch = 1;
        f.H = static_cast<int>(n_cut);
        f.nseg = static_cast<int>(nseg);
        const int64_t total = n_cut * kSsdP * p.n;
        const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), 4096);
        if (p.n == tc::kN) ss_ssd_fold_kernel<tc::kN><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(f);
        else ss_ssd_fold_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(f);
    }
    kmain<<<static_cast<unsigned>(grid), tc::kThreads, tc::kSmemBytes, stream>>>(p, mx, mb, mc, my);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// Segments for `items` (batch x heads) sequences of nchunks chunks on `slots`
// resident CTAs: the count with the smallest waves x chunks per segment, the
// state pass (about 0.3 of the main pass's work per chunk) added, and
// splitting charged 10 %.  chunk_len > 0 fixes the segment length instead.
void ssd_segments(int64_t items, int64_t nchunks, int64_t kmax, int64_t slots, int32_t chunk_len, int& nseg,
                  int& cseg) {
    slots = std::max<int64_t>(slots, 1);
    if (chunk_len > 0) {
        int64_t cs = std::max<int64_t>(1, ceil_div(chunk_len, kSsdQ));
        if (ceil_div(nchunks, cs) > kmax) cs = ceil_div(nchunks, kmax);
        cseg = static_cast<int>(cs);
        nseg = static_cast<int>(ceil_div(nchunks, cs));
        return;
    }
    double best = 0.0;
    nseg = 1;
    cseg = static_cast<int>(nchunks);
    for (int64_t k = 1; k <= kmax; ++k) {
        const int64_t cs = ceil_div(nchunks, k);
        if (ceil_div(nchunks, cs) != k) continue;
        double cost = static_cast<double>(ceil_div(items * k, slots) * cs);
        if (k > 1) cost = 1.1 * (cost + 0.3 * static_cast<double>(ceil_div(items * (k - 1), slots) * cs));
        if (k == 1 || cost < best - 1e-9) {
            best = cost;
            nseg = static_cast<int>(k);
            cseg = static_cast<int>(cs);
        }
    }
}

// Plans the segments (split only with a workspace) and launches the state
// pass, the fold and the main pass.
template <int N>
int launch_ssd(SsdParams& p, int64_t items, const SsdLayout& w, int32_t chunk_len, bool have_ws,
               cudaStream_t stream) {
    auto kmain = ss_ssd_kernel<N, false>;
    auto kstate = ss_ssd_kernel<N, true>;
    const size_t smem = sizeof(SsdSmem<N>);
    static std::atomic<bool> attr_main[kMaxDevices];
    static std::atomic<bool> attr_state[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
    if (set_smem_limit(kmain, smem, attr_main, dev) != SS_OK || set_smem_limit(kstate, smem, attr_state, dev) != SS_OK)
        return SS_ERR_CUDA;
    p.nseg = 1;
    p.cseg = static_cast<int>(w.nchunks);
    if (have_ws) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kmain, kSsdThreads, smem) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SS_ERR_CUDA;
        ssd_segments(items, w.nchunks, w.kmax, static_cast<int64_t>(per_sm) * sms, chunk_len, p.nseg, p.cseg);
    }
    if (items * p.nseg >= (int64_t(1) << 31)) return SS_ERR_INVALID_ARG;
    if (p.nseg > 1) {
        kstate<<<static_cast<unsigned>(items * (p.nseg - 1)), kSsdThreads, smem, stream>>>(p);
        const int64_t total = items * kSsdP * N;
        const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), 4096);
        ss_ssd_fold_kernel<N><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
    }
    kmain<<<static_cast<unsigned>(items * p.nseg), kSsdThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

int validate_dims(const ss_dims* dims, bool need_seqlen) {
    if (!dims) return SS_ERR_INVALID_ARG;
    if (dims->batch < 0 || dims->d_inner < 0 || dims->d_state <= 0) return SS_ERR_INVALID_ARG;
    if (need_seqlen && dims->seqlen < 0) return SS_ERR_INVALID_ARG;
    if (dims->d_state != kN) return SS_ERR_UNSUPPORTED;
    const int64_t lim = int64_t(1) << 31;
    if (dims->batch >= lim || dims->d_inner >= lim) return SS_ERR_INVALID_ARG;
    if (need_seqlen) {
        if (dims->seqlen >= lim) return SS_ERR_INVALID_ARG;
        // batch * seqlen * d_inner elements must stay far below 2^62
        const double elems = double(dims->batch) * double(dims->seqlen) * double(dims->d_inner);
        if (elems > 4.0e18) return SS_ERR_INVALID_ARG;
    }
    return SS_OK;
}

// Backward workspace: local checkpoints [batch][nseg][d][kN], their Σ Δ
// [batch][nseg][d], then chunk records for up to kBwdMaxChunks chunks:
// h_loc and g_loc [batch][kmax][d][kN], Σ Δ [batch][kmax][d]; each region
// 256-byte aligned.
constexpr int64_t kBwdMaxChunks = 16;
struct BwdLayout {
    size_t ckpt, sck, hloc, gloc, send, total;
    int64_t nseg, kmax;
};
BwdLayout bwd_layout(const ss_dims* dims) {
    BwdLayout w{};
    const int64_t b = dims->batch, d = dims->d_inner;
    w.nseg = ceil_div(std::max<int64_t>(dims->seqlen, 1), kSeg);
    w.kmax = std::min(kBwdMaxChunks, w.nseg);
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    size_t off = 0;
    w.ckpt = off; off += al(static_cast<size_t>(b * w.nseg * d) * kN * sizeof(float));
    w.sck = off;  off += al(static_cast<size_t>(b * w.nseg * d) * sizeof(float));
    w.hloc = off; off += al(static_cast<size_t>(b * w.kmax * d) * kN * sizeof(float));
    w.gloc = off; off += al(static_cast<size_t>(b * w.kmax * d) * kN * sizeof(float));
    w.send = off; off += al(static_cast<size_t>(b * w.kmax * d) * sizeof(float));
    w.total = off;
    return w;
}
size_t bwd_workspace(const ss_dims* dims) { return bwd_layout(dims).total; }

// Time chunks for `items` (batch, channel-block) items of nseg segments on
// `slots` resident CTAs: the count whose waves x (segments per chunk + a
// fixed cost of two segments per item: staging, records) is smallest,
// charging chunking 10 % for its extra pass (adjoint-only recurrence).  A
// positive chunk_len fixes the chunk length instead.
void bwd_chunks(int64_t items, int64_t nseg, int64_t kmax, int64_t slots, int32_t chunk_len, int& nchunk,
                int& cseg) {
    if (chunk_len > 0) {
        int64_t cs = std::max<int64_t>(1, ceil_div(chunk_len, kSeg));
        if (ceil_div(nseg, cs) > kmax) cs = ceil_div(nseg, kmax);
        cseg = static_cast<int>(cs);
        nchunk = static_cast<int>(ceil_div(nseg, cs));
        return;
    }
    double best = 0.0;
    nchunk = 1;
    cseg = static_cast<int>(nseg);
    for (int64_t k = 1; k <= kmax; ++k) {
        const int64_t cs = ceil_div(nseg, k);
        if (ceil_div(nseg, cs) != k) continue;
        const double waves = static_cast<double>(ceil_div(items * k, std::max<int64_t>(slots, 1)));
        const double cost = waves * static_cast<double>(cs + 2) * (k > 1 ? 1.1 : 1.0);
        if (k == 1 || cost < best - 1e-9) {
            best = cost;
            nchunk = static_cast<int>(k);
            cseg = static_cast<int>(cs);
        }
    }
}

// Plans the chunks (needs the kernels' occupancy) and launches the chunk pass
// then the gradient pass.
template <typename IO, bool SP, bool HZ>
int launch_bwd(BwdParams& p, int64_t items, int64_t kmax, int32_t chunk_len, cudaStream_t stream) {
    auto kchunk = ss_bwd_chunk_kernel<IO, SP, HZ>;
    auto kgrad = ss_bwd_kernel<IO, SP, HZ>;
    const size_t smem = sizeof(BwdSmem<IO>);
    static std::atomic<bool> attr_chunk[kMaxDevices];
    static std::atomic<bool> attr_grad[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
    const size_t smem_chunk = sizeof(ChunkSmem<IO>);
    if (set_smem_limit(kchunk, smem_chunk, attr_chunk, dev) != SS_OK ||
        set_smem_limit(kgrad, smem, attr_grad, dev) != SS_OK)
        return SS_ERR_CUDA;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kgrad, kBwdThreads, smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SS_ERR_CUDA;
    bwd_chunks(items, p.nseg, kmax, static_cast<int64_t>(per_sm) * sms, chunk_len, p.nchunk, p.cseg);
    const int64_t ctas = items * p.nchunk;
    if (ctas >= (int64_t(1) << 31)) return SS_ERR_INVALID_ARG;
    kchunk<<<static_cast<unsigned>(ctas), kBwdThreads, smem_chunk, stream>>>(p);
    const int64_t states = static_cast<int64_t>(p.batch) * p.d * kN;
    const int64_t cblocks = std::min<int64_t>(ceil_div(states, 256), int64_t(sms) * 16);
    ss_bwd_combine_kernel<<<static_cast<unsigned>(cblocks), 256, 0, stream>>>(p);
    kgrad<<<static_cast<unsigned>(ctas), kBwdThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

template <typename IO>
int launch_bwd_flags(BwdParams& p, int64_t items, int64_t kmax, int32_t chunk_len, cudaStream_t stream) {
    const bool hz = p.z != nullptr;
    if (p.softplus)
        return hz ? launch_bwd<IO, true, true>(p, items, kmax, chunk_len, stream)
                  : launch_bwd<IO, true, false>(p, items, kmax, chunk_len, stream);
    return hz ? launch_bwd<IO, false, true>(p, items, kmax, chunk_len, stream)
              : launch_bwd<IO, false, false>(p, items, kmax, chunk_len, stream);
}

// ------------------------------------------------------------- Mamba block
// One cuBLAS handle per (host thread, device): a handle binds one stream at a
// time, so threads never share one.
cublasHandle_t cublas_handle() {
    thread_local cublasHandle_t handles[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!handles[dev] && cublasCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
    return handles[dev];
}

// Row-major Y[M, N] = X[M, K] · W[N, K]ᵀ in bf16 with fp32 accumulation (a
// column-major cuBLAS call computing Yᵀ = W · Xᵀ).
bool gemm_bf16(cublasHandle_t h, const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K) {
    const float alpha = 1.0f, beta = 0.0f;
    return cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, static_cast<int>(N), static_cast<int>(M), static_cast<int>(K),
                        &alpha, W, CUDA_R_16BF, static_cast<int>(K), X, CUDA_R_16BF, static_cast<int>(K), &beta, Y,
                        CUDA_R_16BF, static_cast<int>(N), CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) ==
           CUBLAS_STATUS_SUCCESS;
}

constexpr size_t kCublasWorkspace = size_t(32) << 20;

// Scratch layout of ss_block_fwd: bf16 x, z, u, Δraw, y [M, d_inner], the
// Δ input [M, dt_rank], B, C [M, 16], then the scan's workspace and cuBLAS's.
struct BlockPlan {
    size_t x, z, u, delta, y, dtl, B, C, fwd_ws, fwd_ws_bytes, cublas_ws, total;
};

bool block_plan(const ss_block_weights* w, int64_t batch, int64_t seqlen, BlockPlan* pl) {
    if (!w || batch < 0 || seqlen < 0 || w->d_model <= 0 || w->d_inner <= 0 || w->dt_rank <= 0) return false;
    if (w->d_inner % 8 || w->d_model % 8 || w->dt_rank >= (int64_t(1) << 20)) return false;
    const int64_t M = batch * seqlen;
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || w->d_inner >= lim || w->d_model >= lim) return false;
    auto al = [](size_t v) { return (v + 255) / 256 * 256; };
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = al(off + bytes); return o; };
    const size_t act = static_cast<size_t>(M) * w->d_inner * 2;
    pl->x = take(act);
    pl->z = take(act);
    pl->u = take(act);
    pl->delta = take(act);
    pl->y = take(act);
    pl->dtl = take(static_cast<size_t>(M) * w->dt_rank * 2);
    pl->B = take(static_cast<size_t>(M) * kN * 2);
    pl->C = take(static_cast<size_t>(M) * kN * 2);
    ss_dims dims{batch, seqlen, w->d_inner, kN};
    pl->fwd_ws_bytes = make_plan(&dims, SS_BF16 | SS_DELTA_SOFTPLUS, 0).total;
    pl->fwd_ws = take(pl->fwd_ws_bytes);
    pl->cublas_ws = take(kCublasWorkspace);
    pl->total = off;
    return true;
}

// ------------------------------------------------ allocation-free entry point
// Workspace of ss_fwd_noalloc: one array in device memory per device that
// loads this library, kept until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SS_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in for it).
void* noalloc_scratch_address() {
    static void* addr[kMaxDevices] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

const char* ss_status_string(int status) {
    switch (status) {
        case SS_OK: return "SS_OK";
        case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG";
        case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED";
        case SS_ERR_CUDA: return "SS_ERR_CUDA";
        case SS_ERR_TIMEOUT: return "SS_ERR_TIMEOUT";
        case SS_ERR_WORKSPACE: return "SS_ERR_WORKSPACE";
        default: return "SS_ERR_UNKNOWN";
    }
}

int ss_version(void) { return kVersion; }

int32_t ss_fwd_chunk_len(const ss_dims* dims, uint32_t flags) {
    if (validate_dims(dims, true) != SS_OK) return 0;
    return static_cast<int32_t>(make_plan(dims, flags, 0).chunk_len);
}

size_t ss_fwd_workspace_bytes(const ss_dims* dims, uint32_t flags, int32_t chunk_len) {
    if (validate_dims(dims, true) != SS_OK) return 0;
    return make_plan(dims, flags, chunk_len).total;
}

int ss_check(const ss_launch* launch) {
    if (!launch) return SS_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return SS_ERR_CUDA;
    if (!launch->workspace || launch->workspace_bytes < sizeof(uint32_t)) return SS_OK;
    uint32_t word = 0;
    if (cudaMemcpy(&word, launch->workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SS_ERR_CUDA;
    return static_cast<int>(word);
}

// ss_fwd and ss_fwd_conv (conv_w non-null: u is computed from x = `u` by the
// causal conv1d + SiLU prologue).
// keep_status: leave the status word (header word 0) as it is, so that one
// word collects the failures of several calls (ss_fwd_host's slices).
static int fwd_impl(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                    const void* C, const float* D, const void* z, void* y, float* last_state, const float* conv_w,
                    const float* conv_b, uint32_t flags, const ss_dims* dims, const ss_launch* launch,
                    const float* h_init = nullptr, bool keep_status = false) {
    const bool conv = conv_w != nullptr;
    int rc = validate_dims(dims, true);
    if (rc != SS_OK) return rc;
    if (!launch || (flags & ~kKnownFlags)) return SS_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, d = dims->d_inner;
    if (batch == 0 || d == 0) return SS_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
    if (L == 0) {   // last_state = the entering state
        if ((last_state && !aligned16(last_state)) || (h_init && !aligned16(h_init))) return SS_ERR_INVALID_ARG;
        const size_t bytes = static_cast<size_t>(batch * d * kN) * sizeof(float);
        if (last_state && (h_init ? cudaMemcpyAsync(last_state, h_init, bytes, cudaMemcpyDeviceToDevice, stream)
                                  : cudaMemsetAsync(last_state, 0, bytes, stream)) != cudaSuccess)
            return SS_ERR_CUDA;
        return SS_OK;
    }
    if (!u || !delta || !A || !B || !C || !y) return SS_ERR_INVALID_ARG;
    const void* ptrs[] = {u, delta, delta_bias, A, B, C, D, z, y, last_state, conv_w, conv_b, h_init};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SS_ERR_INVALID_ARG;

    const bool bf16 = (flags & SS_BF16) != 0;
    const Plan pl = make_plan(dims, flags, launch->chunk_len);
    if (!launch->workspace || launch->workspace_bytes < pl.total || !aligned16(launch->workspace))
        return SS_ERR_WORKSPACE;
    const int64_t items = batch * pl.nchunks * pl.nblk;
    if (items >= (int64_t(1) << 31)) return SS_ERR_INVALID_ARG;

    unsigned char* ws = static_cast<unsigned char*>(launch->workspace);
    const size_t keep = keep_status ? sizeof(uint32_t) : 0;
    if (cudaMemsetAsync(ws + keep, 0, pl.status_off + pl.status_bytes - keep, stream) != cudaSuccess)
        return SS_ERR_CUDA;

    FwdParams p{};
    p.u = u; p.delta = delta; p.bias = delta_bias; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z;
    p.y = y; p.last_state = last_state; p.h_init = h_init;
    p.conv_w = conv_w; p.conv_b = conv_b;
    p.L = L; p.batch = static_cast<int>(batch); p.d = static_cast<int>(d);
    p.chunk_len = static_cast<int>(pl.chunk_len > 0 ? pl.chunk_len : L);
    p.nchunks = static_cast<int>(pl.nchunks); p.nblk = static_cast<int>(pl.nblk);
    p.pflags = ((flags & SS_DELTA_SOFTPLUS) ? kPfSoftplus : 0u) | ((flags & SS_FORCE_GENERAL_A) ? kPfForceGeneral : 0u) |
               ((flags & SS_TEST_DROP_CARRY) ? kPfTestDrop : 0u) | (z ? kPfHasZ : 0u) |
               (delta_bias ? kPfHasBias : 0u) | (D ? kPfHasD : 0u) | (conv ? kPfConv : 0u);
    p.hdr = reinterpret_cast<uint32_t*>(ws);
    p.status = reinterpret_cast<uint32_t*>(ws + pl.status_off);
    p.rec = reinterpret_cast<float*>(ws + pl.rec_off);
    p.wait_ns = kTmaWaitNs;
    p.poll_limit = launch->timeout_iters ? launch->timeout_iters : kDefaultPolls;

    // TMA needs 16-byte row strides: d * element size a multiple of 16.
    const bool tma = ((d * (bf16 ? 2 : 4)) % 16) == 0;
    CUtensorMap maps[6];
    std::memset(maps, 0, sizeof(maps));
    if (tma) {
        bool ok = make_map(&maps[0], u, bf16, d, L, batch, kCB, kTT + (conv ? kHalo : 0)) &&
                  make_map(&maps[1], delta, bf16, d, L, batch, kCB, kTT) &&
                  make_map(&maps[2], z ? z : u, bf16, d, L, batch, kCB, kTT) &&
                  make_map(&maps[3], B, bf16, kN, L, batch, kN, kTT) &&
                  make_map(&maps[4], C, bf16, kN, L, batch, kN, kTT) &&
                  make_map(&maps[5], y, bf16, d, L, batch, kCB, kTT);
        if (!ok) return SS_ERR_CUDA;
    }
    const Variant v = choose(dims, flags).v;
    rc = conv ? launch_variant<true>(bf16, tma, v, p, items, maps, stream)
              : launch_variant<false>(bf16, tma, v, p, items, maps, stream);
    if (rc != SS_OK) return rc;
    if (flags & SS_SYNC_CHECK) return ss_check(launch);
    return SS_OK;
}

int ss_fwd(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
           const void* C, const float* D, const void* z, void* y, float* last_state, uint32_t flags,
           const ss_dims* dims, const ss_launch* launch) {
    return fwd_impl(u, delta, delta_bias, A, B, C, D, z, y, last_state, nullptr, nullptr, flags, dims, launch);
}

// ------------------------------------------------------------- host-buffer forward
// Staging of ss_fwd_host: the forward workspace of one slice first (its
// header word 0 is the call's status word), then two slots, each holding one
// batch slice's u, Δraw, z, y [rows, L, d], B, C [rows, L, 16] and
// last_state [rows, d, 16]; every region 256-byte aligned.
struct HostPlan {
    size_t act, bc, st, slot, ws_off, ws, total;
    int64_t rows;
};
static HostPlan host_plan(const ss_dims* dims, uint32_t flags, int32_t rows_per_slice) {
    HostPlan h{};
    const size_t es = (flags & SS_BF16) ? 2 : 4;
    const int64_t L = dims->seqlen, d = dims->d_inner;
    h.rows = std::max<int64_t>(1, std::min<int64_t>(rows_per_slice > 0 ? rows_per_slice : 1, dims->batch));
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    h.act = al(static_cast<size_t>(h.rows * L * d) * es);
    h.bc = al(static_cast<size_t>(h.rows * L * kN) * es);
    h.st = al(static_cast<size_t>(h.rows * d * kN) * sizeof(float));
    h.slot = 4 * h.act + 2 * h.bc + h.st;
    ss_dims sd = *dims;
    sd.batch = h.rows;
    h.ws = al(ss_fwd_workspace_bytes(&sd, flags, 0));
    h.ws_off = h.ws;   // the slots follow the forward workspace
    h.total = h.ws + 2 * h.slot;
    return h;
}

// Copy streams and events of the host pipeline, one set per (host thread,
// device), created on first use and kept (like the cuBLAS handle).
struct HostPipe {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in_ready[2] = {}, done[2] = {}, out_free[2] = {};
    bool ok = false;
};
static HostPipe* host_pipe() {
    thread_local HostPipe pipes[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostPipe& h = pipes[dev];
    if (!h.ok) {
        bool ok = cudaStreamCreateWithFlags(&h.up, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&h.down, cudaStreamNonBlocking) == cudaSuccess;
        cudaEvent_t* evs[] = {&h.start, &h.end, &h.in_ready[0], &h.in_ready[1], &h.done[0], &h.done[1],
                              &h.out_free[0], &h.out_free[1]};
        for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return nullptr;
        h.ok = true;
    }
    return &h;
}

size_t ss_fwd_host_workspace_bytes(const ss_dims* dims, uint32_t flags, int32_t rows_per_slice) {
    if (validate_dims(dims, true) != SS_OK || (flags & ~kKnownFlags) || dims->batch == 0 || dims->d_inner == 0)
        return 0;
    return host_plan(dims, flags, rows_per_slice).total;
}

int ss_fwd_host(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                const void* C, const float* D, const void* z, void* y, float* last_state, uint32_t flags,
                const ss_dims* dims, const ss_launch* launch, int32_t rows_per_slice) {
    int rc = validate_dims(dims, true);
    if (rc != SS_OK) return rc;
    if (!launch || (flags & ~kKnownFlags)) return SS_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, d = dims->d_inner;
    if (batch == 0 || d == 0) return SS_OK;
    if (!A || (L > 0 && (!u || !delta || !B || !C || !y))) return SS_ERR_INVALID_ARG;
    const void* dev_ptrs[] = {A, D, delta_bias};
    for (const void* q : dev_ptrs)
        if (q && !aligned16(q)) return SS_ERR_INVALID_ARG;
    const HostPlan h = host_plan(dims, flags, rows_per_slice);
    if (!launch->workspace || launch->workspace_bytes < h.total || !aligned16(launch->workspace))
        return SS_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(launch->stream);
    if (L == 0) {   // last_state = h_{-1} = 0, nothing else to do
        if (last_state) {
            if (cudaStreamSynchronize(cs) != cudaSuccess) return SS_ERR_CUDA;
            std::memset(last_state, 0, static_cast<size_t>(batch * d * kN) * sizeof(float));
        }
        return SS_OK;
    }
    HostPipe* hp = host_pipe();
    if (!hp) return SS_ERR_CUDA;
    const size_t es = (flags & SS_BF16) ? 2 : 4;
    unsigned char* base = static_cast<unsigned char*>(launch->workspace);
    ss_launch sl = *launch;   // the slices' forward: workspace at the start, before the two slots
    sl.workspace = base;
    sl.workspace_bytes = h.ws;
    const uint32_t fflags = flags & ~static_cast<uint32_t>(SS_SYNC_CHECK);
    // one status word for the whole call: cleared once here, kept by every slice
    if (cudaMemsetAsync(base, 0, sizeof(uint32_t), cs) != cudaSuccess) return SS_ERR_CUDA;
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    // On an error after copies were queued, let them finish before returning:
    // they read and write the caller's host buffers.
    auto fail = [&](int code) {
        cudaStreamSynchronize(hp->up);
        cudaStreamSynchronize(hp->down);
        return code;
    };
    // the copy streams start after the work already queued on the caller's stream
    if (!ok(cudaEventRecord(hp->start, cs)) || !ok(cudaStreamWaitEvent(hp->up, hp->start, 0)) ||
        !ok(cudaStreamWaitEvent(hp->down, hp->start, 0)))
        return SS_ERR_CUDA;
    const int64_t nslices = ceil_div(batch, h.rows);
    for (int64_t s = 0; s < nslices; ++s) {
        const int slot = static_cast<int>(s & 1);
        const int64_t r0 = s * h.rows, nr = std::min(h.rows, batch - r0);
        unsigned char* sp = base + h.ws_off + slot * h.slot;
        void* su = sp;
        void* sd = sp + h.act;
        void* sz = sp + 2 * h.act;
        void* sy = sp + 3 * h.act;
        void* sB = sp + 4 * h.act;
        void* sC = sp + 4 * h.act + h.bc;
        float* sst = reinterpret_cast<float*>(sp + 4 * h.act + 2 * h.bc);
        const size_t act_bytes = static_cast<size_t>(nr * L * d) * es, act_off = static_cast<size_t>(r0 * L * d) * es;
        const size_t bc_bytes = static_cast<size_t>(nr * L * kN) * es, bc_off = static_cast<size_t>(r0 * L * kN) * es;
        // upload (after the forward of slice s - 2 has read this slot)
        if (s >= 2 && !ok(cudaStreamWaitEvent(hp->up, hp->done[slot], 0))) return fail(SS_ERR_CUDA);
        if (!ok(cudaMemcpyAsync(su, static_cast<const unsigned char*>(u) + act_off, act_bytes, cudaMemcpyHostToDevice,
                                hp->up)) ||
            !ok(cudaMemcpyAsync(sd, static_cast<const unsigned char*>(delta) + act_off, act_bytes,
                                cudaMemcpyHostToDevice, hp->up)) ||
            (z && !ok(cudaMemcpyAsync(sz, static_cast<const unsigned char*>(z) + act_off, act_bytes,
                                      cudaMemcpyHostToDevice, hp->up))) ||
            !ok(cudaMemcpyAsync(sB, static_cast<const unsigned char*>(B) + bc_off, bc_bytes, cudaMemcpyHostToDevice,
                                hp->up)) ||
            !ok(cudaMemcpyAsync(sC, static_cast<const unsigned char*>(C) + bc_off, bc_bytes, cudaMemcpyHostToDevice,
                                hp->up)) ||
            !ok(cudaEventRecord(hp->in_ready[slot], hp->up)))
            return fail(SS_ERR_CUDA);
        // forward of the slice (after its upload, and after slice s - 2's y left this slot)
        if (!ok(cudaStreamWaitEvent(cs, hp->in_ready[slot], 0)) ||
            (s >= 2 && !ok(cudaStreamWaitEvent(cs, hp->out_free[slot], 0))))
            return fail(SS_ERR_CUDA);
        ss_dims sdims = *dims;
        sdims.batch = nr;
        // the test-only dropped carry belongs to the caller's batch entry 0: the first slice
        const uint32_t sflags = s == 0 ? fflags : (fflags & ~static_cast<uint32_t>(SS_TEST_DROP_CARRY));
        rc = fwd_impl(su, sd, delta_bias, A, sB, sC, D, z ? sz : nullptr, sy, last_state ? sst : nullptr, nullptr,
                      nullptr, sflags, &sdims, &sl, nullptr, /*keep_status=*/true);
        if (rc != SS_OK) return fail(rc);
        if (!ok(cudaEventRecord(hp->done[slot], cs))) return fail(SS_ERR_CUDA);
        // download
        if (!ok(cudaStreamWaitEvent(hp->down, hp->done[slot], 0)) ||
            !ok(cudaMemcpyAsync(static_cast<unsigned char*>(y) + act_off, sy, act_bytes, cudaMemcpyDeviceToHost,
                                hp->down)) ||
            (last_state && !ok(cudaMemcpyAsync(last_state + r0 * d * kN, sst,
                                               static_cast<size_t>(nr * d * kN) * sizeof(float),
                                               cudaMemcpyDeviceToHost, hp->down))) ||
            !ok(cudaEventRecord(hp->out_free[slot], hp->down)))
            return fail(SS_ERR_CUDA);
    }
    // the caller's stream continues after the last download
    if (!ok(cudaEventRecord(hp->end, hp->down)) || !ok(cudaStreamWaitEvent(cs, hp->end, 0)))
        return fail(SS_ERR_CUDA);
    if (flags & SS_SYNC_CHECK) return ss_check(&sl);
    return SS_OK;
}

int ss_fwd_with_state(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* h_init, void* y, float* last_state,
                      uint32_t flags, const ss_dims* dims, const ss_launch* launch) {
    return fwd_impl(u, delta, delta_bias, A, B, C, D, z, y, last_state, nullptr, nullptr, flags, dims, launch, h_init);
}

int ss_fwd_conv(const void* x, const float* conv_w, const float* conv_b, const void* delta, const float* delta_bias,
                const float* A, const void* B, const void* C, const float* D, const void* z, void* y,
                float* last_state, float* conv_state, uint32_t flags, const ss_dims* dims, const ss_launch* launch) {
    if (!conv_w) return SS_ERR_INVALID_ARG;
    if (conv_state && !aligned16(conv_state)) return SS_ERR_INVALID_ARG;
    int rc = fwd_impl(x, delta, delta_bias, A, B, C, D, z, y, last_state, conv_w, conv_b,
                      flags & ~static_cast<uint32_t>(SS_SYNC_CHECK), dims, launch);
    if (rc != SS_OK) return rc;
    const int64_t n = dims->batch * dims->d_inner;
    if (conv_state && n > 0) {
        if (!x && dims->seqlen > 0) return SS_ERR_INVALID_ARG;
        cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
        const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 4096));
        if (flags & SS_BF16)
            ss_conv_tail_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
                static_cast<const __nv_bfloat16*>(x), conv_state, dims->batch, dims->seqlen, dims->d_inner);
        else
            ss_conv_tail_kernel<float><<<blocks, 256, 0, stream>>>(static_cast<const float*>(x), conv_state,
                                                                   dims->batch, dims->seqlen, dims->d_inner);
        if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    }
    if (flags & SS_SYNC_CHECK) return ss_check(launch);
    return SS_OK;
}

// ss_step and ss_step_conv (conv_w non-null: the token's input `u` is x, and
// u = silu(conv) over conv_state, which shifts in x).
static int step_impl(float* state, const void* u, const void* delta, const float* A, const void* B, const void* C,
                     const float* D, const void* z, void* y, const float* delta_bias, float* conv_state,
                     const float* conv_w, const float* conv_b, uint32_t flags, const ss_dims* dims,
                     const ss_launch* launch) {
    int rc = validate_dims(dims, false);
    if (rc != SS_OK) return rc;
    if (!launch || (flags & ~kKnownFlags)) return SS_ERR_INVALID_ARG;
    const bool conv = conv_w != nullptr;
    const int64_t batch = dims->batch, d = dims->d_inner;
    if (batch == 0 || d == 0) return SS_OK;
    if (!state || !u || !delta || !A || !B || !C || !y || (conv && !conv_state)) return SS_ERR_INVALID_ARG;
    const void* ptrs[] = {state, u, delta, A, B, C, D, z, y, delta_bias, conv_state, conv_w, conv_b};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SS_ERR_INVALID_ARG;
    const bool bf16 = (flags & SS_BF16) != 0;
    StepParams p{};
    p.state = state; p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z; p.y = y;
    p.bias = delta_bias; p.batch = batch; p.d = static_cast<int>(d);
    p.conv_state = conv_state; p.conv_w = conv_w; p.conv_b = conv_b;
    p.softplus = (flags & SS_DELTA_SOFTPLUS) ? 1 : 0;
    const dim3 grid(static_cast<unsigned>(ceil_div(d, kStepChanPerBlock)),
                    static_cast<unsigned>(std::min<int64_t>(ceil_div(batch, 2), 65535)));
    cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
    // exact tiling, 32-bit offsets: the predicate-free kernel
    constexpr int kFullRows = 1;   // batch rows per thread of the exact-tiling kernel (1, 2, 4 measured: 1 best)
    const bool full = !conv && d % kStepChanPerBlock == 0 && batch % kFullRows == 0 &&
                      batch / kFullRows <= 65535 && batch * d * kN < (int64_t(1) << 31);
    if (full) {
        const dim3 fgrid(static_cast<unsigned>(d / kStepChanPerBlock), static_cast<unsigned>(batch / kFullRows));
        if (bf16) ss_step_full_kernel<__nv_bfloat16, kFullRows><<<fgrid, kStepThreads, 0, stream>>>(p);
        else      ss_step_full_kernel<float, kFullRows><<<fgrid, kStepThreads, 0, stream>>>(p);
    } else if (bf16) {
        if (conv) ss_step_kernel<__nv_bfloat16, true><<<grid, kStepThreads, 0, stream>>>(p);
        else      ss_step_kernel<__nv_bfloat16, false><<<grid, kStepThreads, 0, stream>>>(p);
    } else {
        if (conv) ss_step_kernel<float, true><<<grid, kStepThreads, 0, stream>>>(p);
        else      ss_step_kernel<float, false><<<grid, kStepThreads, 0, stream>>>(p);
    }
    if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    if (flags & SS_SYNC_CHECK) {
        if (cudaStreamSynchronize(stream) != cudaSuccess) return SS_ERR_CUDA;
    }
    return SS_OK;
}

int ss_step(float* state, const void* u, const void* delta, const float* A, const void* B, const void* C,
            const float* D, const void* z, void* y, const float* delta_bias, uint32_t flags, const ss_dims* dims,
            const ss_launch* launch) {
    return step_impl(state, u, delta, A, B, C, D, z, y, delta_bias, nullptr, nullptr, nullptr, flags, dims, launch);
}

int ss_step_conv(float* state, float* conv_state, const void* x, const float* conv_w, const float* conv_b,
                 const void* delta, const float* A, const void* B, const void* C, const float* D, const void* z,
                 void* y, const float* delta_bias, uint32_t flags, const ss_dims* dims, const ss_launch* launch) {
    if (!conv_w) return SS_ERR_INVALID_ARG;
    return step_impl(state, x, delta, A, B, C, D, z, y, delta_bias, conv_state, conv_w, conv_b, flags, dims, launch);
}

size_t ss_bwd_workspace_bytes(const ss_dims* dims, uint32_t flags) {
    (void)flags;
    if (validate_dims(dims, true) != SS_OK) return 0;
    return bwd_workspace(dims);
}

int ss_bwd(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
           const void* C, const float* D, const void* z, const void* dy, const float* dlast_state,
           void* du, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
           float* ddelta_bias, uint32_t flags, const ss_dims* dims, const ss_launch* launch) {
    int rc = validate_dims(dims, true);
    if (rc != SS_OK) return rc;
    if (!launch || (flags & ~kKnownFlags)) return SS_ERR_INVALID_ARG;
    if ((z == nullptr) != (dz == nullptr)) return SS_ERR_INVALID_ARG;
    if ((dD && !D) || (ddelta_bias && !delta_bias)) return SS_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, d = dims->d_inner;
    if (batch == 0 || d == 0) return SS_OK;
    // Pointers to per-token tensors are not needed (and may be NULL) when L = 0.
    if (!A || !dA || (L > 0 && (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC)))
        return SS_ERR_INVALID_ARG;
    const void* ptrs[] = {u, delta, delta_bias, A, B, C, D, z, dy, dlast_state,
                          du, ddelta, dA, dB, dC, dD, dz, ddelta_bias};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SS_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
    // The summed gradients are accumulated: start them from zero.
    const size_t bytes_bc = static_cast<size_t>(batch * L) * kN * sizeof(float);
    if (cudaMemsetAsync(dA, 0, static_cast<size_t>(d) * kN * sizeof(float), stream) != cudaSuccess ||
        (bytes_bc && cudaMemsetAsync(dB, 0, bytes_bc, stream) != cudaSuccess) ||
        (bytes_bc && cudaMemsetAsync(dC, 0, bytes_bc, stream) != cudaSuccess) ||
        (dD && cudaMemsetAsync(dD, 0, static_cast<size_t>(d) * sizeof(float), stream) != cudaSuccess) ||
        (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, static_cast<size_t>(d) * sizeof(float), stream) != cudaSuccess))
        return SS_ERR_CUDA;
    // With no tokens, last_state = h_{-1} = 0 depends on nothing: every gradient is zero.
    if (L == 0) return (flags & SS_SYNC_CHECK) ? (cudaStreamSynchronize(stream) == cudaSuccess ? SS_OK : SS_ERR_CUDA)
                                              : SS_OK;
    const BwdLayout w = bwd_layout(dims);
    if (!launch->workspace || launch->workspace_bytes < w.total || !aligned16(launch->workspace))
        return SS_ERR_WORKSPACE;
    const int64_t nblk = ceil_div(d, kBwdCh);
    const int64_t items = batch * nblk;
    if (items >= (int64_t(1) << 31)) return SS_ERR_INVALID_ARG;

    BwdParams p{};
    p.u = u; p.delta = delta; p.bias = delta_bias; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z;
    p.dy = dy; p.dlast = dlast_state;
    p.du = du; p.ddelta = ddelta; p.dz = dz; p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.dbias = ddelta_bias;
    unsigned char* ws = static_cast<unsigned char*>(launch->workspace);
    p.ckpt = reinterpret_cast<float*>(ws + w.ckpt);
    p.sck = reinterpret_cast<float*>(ws + w.sck);
    p.hloc = reinterpret_cast<float*>(ws + w.hloc);
    p.gloc = reinterpret_cast<float*>(ws + w.gloc);
    p.send = reinterpret_cast<float*>(ws + w.send);
    p.L = L; p.batch = static_cast<int>(batch); p.d = static_cast<int>(d);
    p.nseg = static_cast<int>(w.nseg); p.nblk = static_cast<int>(nblk);
    p.softplus = (flags & SS_DELTA_SOFTPLUS) ? 1 : 0;
    p.vec = (d * static_cast<int64_t>((flags & SS_BF16) ? 2 : 4)) % 16 == 0 ? 1 : 0;
    rc = (flags & SS_BF16) ? launch_bwd_flags<__nv_bfloat16>(p, items, w.kmax, launch->chunk_len, stream)
                           : launch_bwd_flags<float>(p, items, w.kmax, launch->chunk_len, stream);
    if (rc != SS_OK) return rc;
    if (flags & SS_SYNC_CHECK) {
        if (cudaStreamSynchronize(stream) != cudaSuccess) return SS_ERR_CUDA;
    }
    return SS_OK;
}

size_t ss_ssd_fwd_workspace_bytes(const ss_ssd_dims* dims, uint32_t flags) {
    if (!dims || (flags & ~kKnownFlags) || dims->batch < 0 || dims->seqlen < 0 || dims->nheads < 0) return 0;
    if (dims->headdim != kSsdP || (dims->d_state != 64 && dims->d_state != 128)) return 0;
    return ssd_layout(dims).total;
}

int ss_ssd_fwd(const void* x, const void* dt, const float* dt_bias, const float* A, const void* B, const void* C,
               const float* D, void* y, float* final_state, uint32_t flags, const ss_ssd_dims* dims,
               const ss_launch* launch) {
    if (!dims || !launch || (flags & ~kKnownFlags)) return SS_ERR_INVALID_ARG;
    const int64_t batch = dims->batch, L = dims->seqlen, H = dims->nheads;
    if (batch < 0 || L < 0 || H < 0) return SS_ERR_INVALID_ARG;
    if (dims->headdim != kSsdP || (dims->d_state != 64 && dims->d_state != 128)) return SS_ERR_UNSUPPORTED;
    const int64_t lim = int64_t(1) << 31;
    if (batch * H >= lim || L >= lim || double(batch) * double(L) * double(H) * kSsdP > 4.0e18)
        return SS_ERR_INVALID_ARG;
    if (batch == 0 || H == 0) return SS_OK;
    if (!A || (L > 0 && (!x || !dt || !B || !C || !y))) return SS_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt, dt_bias, A, B, C, D, y, final_state};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SS_ERR_INVALID_ARG;
    const SsdLayout w = ssd_layout(dims);
    const bool have_ws = launch->workspace != nullptr;
    if (have_ws && (launch->workspace_bytes < w.total || !aligned16(launch->workspace))) return SS_ERR_WORKSPACE;
    cudaStream_t stream = static_cast<cudaStream_t>(launch->stream);
    if (have_ws && cudaMemsetAsync(launch->workspace, 0, sizeof(uint32_t), stream) != cudaSuccess)
        return SS_ERR_CUDA;
    SsdParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.dt = static_cast<const __nv_bfloat16*>(dt);
    p.dt_bias = dt_bias; p.A = A;
    p.B = static_cast<const __nv_bfloat16*>(B);
    p.C = static_cast<const __nv_bfloat16*>(C);
    p.D = D;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.final_state = final_state;
    if (have_ws) {
        unsigned char* ws = static_cast<unsigned char*>(launch->workspace);
        p.rec = reinterpret_cast<float*>(ws + w.rec);
        p.esum = reinterpret_cast<float*>(ws + w.esum);
    }
    p.L = L; p.batch = static_cast<int>(batch); p.H = static_cast<int>(H);
    p.softplus = (flags & SS_DELTA_SOFTPLUS) ? 1 : 0;
    const int64_t items = batch * H;
    int rc;
    if (!SELSCAN_SSD_MMA_SYNC) {
        if (L == 0) {   // no steps: the final state is zero
            if (final_state &&
                cudaMemsetAsync(final_state, 0, static_cast<size_t>(items * kSsdP * dims->d_state) * sizeof(float),
                                stream) != cudaSuccess)
                return SS_ERR_CUDA;
            rc = SS_OK;
        } else {
            tc::Params q{};
            q.dt = p.dt; q.dt_bias = p.dt_bias; q.A = p.A; q.D = p.D; q.y = p.y; q.final_state = p.final_state;
            q.rec = p.rec; q.esum = p.esum;
            q.status = have_ws ? static_cast<uint32_t*>(launch->workspace) : nullptr;
            q.L = L; q.batch = p.batch; q.H = p.H; q.softplus = p.softplus;
            q.n = static_cast<int>(dims->d_state);
            q.test_drop = (flags & SS_TEST_DROP_CARRY) ? 1 : 0;
            q.wait_ns = launch->timeout_iters ? static_cast<uint64_t>(launch->timeout_iters) * 1000ull : kTmaWaitNs;
            q.drain_ns = kTmaWaitNs;
            rc = launch_ssd_tc(q, p, x, B, C, items, w, launch->chunk_len, have_ws, stream);
        }
    } else {
        rc = dims->d_state == 128 ? launch_ssd<128>(p, items, w, launch->chunk_len, have_ws, stream)
                                  : launch_ssd<64>(p, items, w, launch->chunk_len, have_ws, stream);
    }
    if (rc != SS_OK) return rc;
    if (flags & SS_SYNC_CHECK) {
        if (have_ws) return ss_check(launch);
        if (cudaStreamSynchronize(stream) != cudaSuccess) return SS_ERR_CUDA;
    }
    return SS_OK;
}

size_t ss_block_scratch_bytes(const ss_block_weights* w, int64_t batch, int64_t seqlen) {
    BlockPlan pl{};
    return block_plan(w, batch, seqlen, &pl) ? pl.total : 0;
}

int ss_block_fwd(const void* hidden, void* out, const ss_block_weights* w, int64_t batch, int64_t seqlen,
                 void* scratch, size_t scratch_bytes, void* stream_v) {
    BlockPlan pl{};
    if (!block_plan(w, batch, seqlen, &pl)) return SS_ERR_INVALID_ARG;
    const int64_t M = batch * seqlen, di = w->d_inner, dm = w->d_model, rk = w->dt_rank;
    if (M == 0) return SS_OK;
    const void* need[] = {hidden, out, w->in_proj_x, w->in_proj_z, w->conv_w, w->x_proj_dt, w->x_proj_B,
                          w->x_proj_C, w->dt_proj, w->dt_bias, w->A, w->out_proj};
    for (const void* q : need)
        if (!q || !aligned16(q)) return SS_ERR_INVALID_ARG;
    if ((w->conv_b && !aligned16(w->conv_b)) || (w->D && !aligned16(w->D))) return SS_ERR_INVALID_ARG;
    if (!scratch || scratch_bytes < pl.total || !aligned16(scratch)) return SS_ERR_WORKSPACE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    cublasHandle_t h = cublas_handle();
    if (!h) return SS_ERR_CUDA;
    unsigned char* base = static_cast<unsigned char*>(scratch);
    if (cublasSetStream(h, stream) != CUBLAS_STATUS_SUCCESS ||
        cublasSetWorkspace(h, base + pl.cublas_ws, kCublasWorkspace) != CUBLAS_STATUS_SUCCESS)
        return SS_ERR_CUDA;
    void* x = base + pl.x;
    void* z = base + pl.z;
    void* u = base + pl.u;
    void* delta = base + pl.delta;
    void* y = base + pl.y;
    void* dtl = base + pl.dtl;
    void* Bm = base + pl.B;
    void* Cm = base + pl.C;
    // in_proj
    if (!gemm_bf16(h, hidden, w->in_proj_x, x, M, di, dm) || !gemm_bf16(h, hidden, w->in_proj_z, z, M, di, dm))
        return SS_ERR_CUDA;
    // causal conv1d + SiLU
    const dim3 grid(static_cast<unsigned>(ceil_div(di, kConvThreads)),
                    static_cast<unsigned>(ceil_div(seqlen, kConvSteps)), static_cast<unsigned>(batch));
    if (grid.y > 65535u || grid.z > 65535u) return SS_ERR_INVALID_ARG;
    ss_conv_silu_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), w->conv_w, w->conv_b, static_cast<__nv_bfloat16*>(u), seqlen, di);
    if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    // selection projections and Δ's projection
    if (!gemm_bf16(h, u, w->x_proj_dt, dtl, M, rk, di) || !gemm_bf16(h, u, w->x_proj_B, Bm, M, kN, di) ||
        !gemm_bf16(h, u, w->x_proj_C, Cm, M, kN, di) || !gemm_bf16(h, dtl, w->dt_proj, delta, M, di, rk))
        return SS_ERR_CUDA;
    // the selective scan, gated by z
    ss_dims dims{batch, seqlen, di, kN};
    ss_launch launch{};
    launch.stream = stream;
    launch.workspace = base + pl.fwd_ws;
    launch.workspace_bytes = pl.fwd_ws_bytes;
    int rc = ss_fwd(u, delta, w->dt_bias, w->A, Bm, Cm, w->D, z, y, nullptr, SS_BF16 | SS_DELTA_SOFTPLUS, &dims,
                    &launch);
    if (rc != SS_OK) return rc;
    // out_proj
    if (!gemm_bf16(h, y, w->out_proj, out, M, dm, di)) return SS_ERR_CUDA;
    return SS_OK;
}

int ss_fwd_noalloc(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                   const void* C, const float* D, const void* z, void* y, float* last_state, uint32_t flags,
                   const ss_dims* dims, void* stream) {
    // The same plan ss_fwd makes for these sizes decides the scratch need.
    const size_t need = ss_fwd_workspace_bytes(dims, flags, 0);
    if (need > SS_NOALLOC_SCRATCH_BYTES) return SS_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = noalloc_scratch_address();
        if (!scratch) return SS_ERR_CUDA;
    }
    ss_launch launch{};
    launch.stream = stream;
    launch.workspace = scratch;
    launch.workspace_bytes = scratch ? SS_NOALLOC_SCRATCH_BYTES : 0;
    return ss_fwd(u, delta, delta_bias, A, B, C, D, z, y, last_state, flags, dims, &launch);
}

}  // extern "C"
