/*
 * selscan.h -- C ABI of libselscan, the B200 (sm_100a) selective-scan library.
 *
 * The operations, all from the selective state-space model of Mamba:
 *
 *   ss_fwd   the forward scan over a whole sequence ("Algorithm 2" selective
 *            SSM of the mamba README, Usage > Selective SSM; equations of
 *            "Understanding Mamba and Selective State Space Models (SSMs)",
 *            §2.2 first and second cut, §3.1, §4.3):
 *              Δ_t   = softplus(Δraw_t + bias)                  (§2.2 closing tip)
 *              h_t,n = exp(Δ_t A_n) h_{t-1},n + Δ_t B_t,n u_t   (§2.2 first cut)
 *              y_t   = (Σ_n C_t,n h_t,n + D u_t) · z_t σ(z_t)    (§3.1, §2.1; gate optional)
 *            with h_{-1} = 0 (§2.2 second cut), per channel, A diagonal (§4.3).
 *   ss_step  one decode step on a carried state: the same body for a single
 *            token, reading and overwriting the state (the streaming "step"
 *            function of the Mamba tutorial, §"state management", and the
 *            "constant memory per token" property of the model-architecture
 *            page).
 *   ss_fwd_conv / ss_step_conv  the same with the causal conv1d + SiLU
 *            prologue of the Mamba block fused in ("Understanding Mamba and
 *            Selective State Space Models (SSMs)" §3.3).
 *   ss_block_fwd  the Mamba block's inner forward path around the scan
 *            (projections on cuBLAS, conv, scan, gate, output projection).
 *   ss_ssd_fwd  the multi-head scan with a scalar decay per head (Mamba-2's
 *            SSD model) on the tensor cores.
 *   ss_fwd_with_state  ss_fwd from a given entering state (continuation).
 *   ss_fwd_host  ss_fwd on activations in host memory, with uploads, scans
 *            and downloads of batch slices overlapped.
 *   ss_bwd   the gradients of ss_fwd's inputs from the gradient of its outputs
 *            (the models are trained and fine-tuned with gradient
 *            checkpointing: "Mamba 7.9.1" article §5.3-5.4; model-architecture
 *            page, "Common issues"); reverse-mode differentiation of the same
 *            recurrence, recomputing the forward states from checkpoints.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor pointer is a DEVICE pointer (cudaMalloc / torch CUDA
 *   memory) on the current device, contiguous row-major, 16-byte aligned.
 *   The caller owns all buffers; the library allocates nothing.
 * - Element type of u, delta, z, B, C and y: bf16 when SS_BF16 is set in
 *   `flags`, else fp32.  A, D, delta_bias and the states are always fp32.
 * - Layouts: u, delta, z, y [batch, seqlen, d_inner] (token-major, channels
 *   contiguous); B, C [batch, seqlen, d_state] (one group shared by all
 *   channels); A [d_inner, d_state]; D, delta_bias [d_inner];
 *   last_state / state [batch, d_inner, d_state].
 * - d_state must be 16 (SS_ERR_UNSUPPORTED otherwise).
 * - Calls are asynchronous on launch->stream.  A device-side failure (a
 *   cross-chunk wait that ran out) is recorded in the workspace and reported
 *   by ss_check(), or by the call itself when SS_SYNC_CHECK is set.
 * - Invalid arguments return SS_ERR_INVALID_ARG and launch nothing.
 *   Calls never trap or abort.
 */
#ifndef SELSCAN_H
#define SELSCAN_H

#include <stddef.h>
#include <stdint.h>

/* Exported symbols keep default visibility even when the library is built
 * with -fvisibility=hidden. */
#if defined(__GNUC__)
#define SS_API __attribute__((visibility("default")))
#else
#define SS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Problem sizes.  seqlen is ignored by ss_step. */
typedef struct ss_dims {
    int64_t batch;
    int64_t seqlen;
    int64_t d_inner;
    int64_t d_state;
} ss_dims;

/* Launch context.
 *   stream          cudaStream_t to launch on (NULL: the legacy default stream).
 *   workspace       device scratch of at least ss_fwd_workspace_bytes() bytes
 *                   (never less than 256: it always holds the device status
 *                   word), 16-byte aligned.  ss_fwd overwrites it on every
 *                   call; calls that overlap in time must not share one.
 *                   ss_step does not use it.
 *   workspace_bytes its size.
 *   timeout_iters   bound on the polls of one cross-chunk wait (0: library
 *                   default, about one second); for ss_ssd_fwd, the bound on
 *                   one wait in microseconds (0: two seconds).  When it runs out the call records
 *                   SS_ERR_TIMEOUT and finishes without hanging.
 *   chunk_len       timesteps per time chunk; 0 lets the library choose.  Any
 *                   positive value is accepted (it is rounded up to a multiple
 *                   of the 32-step tile); results agree up to rounding. */
typedef struct ss_launch {
    void*    stream;
    void*    workspace;
    size_t   workspace_bytes;
    uint32_t timeout_iters;
    int32_t  chunk_len;
} ss_launch;

/* Status codes. */
enum {
    SS_OK              = 0,
    SS_ERR_INVALID_ARG = -1,   /* NULL required pointer, negative size, misalignment, overflow */
    SS_ERR_UNSUPPORTED = -2,   /* d_state != 16 */
    SS_ERR_CUDA        = -3,   /* a CUDA runtime call or launch failed */
    SS_ERR_TIMEOUT     = -4,   /* a bounded cross-chunk wait ran out (results invalid) */
    SS_ERR_WORKSPACE   = -5    /* workspace missing or smaller than required */
};

/* Flags. */
enum {
    SS_BF16            = 1u << 0,  /* u, delta, z, B, C, y are bf16 (else fp32) */
    SS_DELTA_SOFTPLUS  = 1u << 1,  /* Δ = softplus(delta + delta_bias); else Δ = delta + delta_bias */
    SS_SYNC_CHECK      = 1u << 2,  /* synchronize the stream and return the device status */
    SS_FORCE_GENERAL_A = 1u << 3,  /* skip the A[d,n] = a_d (n+1) fast path even when A has that form */
    SS_TEST_DROP_CARRY = 1u << 30  /* TEST ONLY: the first chunk of batch 0, channel block 0 never
                                      publishes its carry, so its successor's bounded wait runs out
                                      (exercises SS_ERR_TIMEOUT without a hang); in ss_ssd_fwd
                                      the first CTA never signals its first C Bᵀ product, so its
                                      compute warps' wait runs out */
};

/* ss_fwd -- selective-scan forward pass over [batch, seqlen] tokens.
 *   u          [batch, seqlen, d_inner]  input sequence (x_n of §2.2)
 *   delta      [batch, seqlen, d_inner]  Δ before bias and softplus
 *   delta_bias [d_inner] fp32 or NULL    added to delta before softplus
 *   A          [d_inner, d_state] fp32   diagonal state matrix (negative reals)
 *   B, C       [batch, seqlen, d_state]  input / output projections per token
 *   D          [d_inner] fp32 or NULL    skip weight (NULL: no skip term)
 *   z          [batch, seqlen, d_inner] or NULL   gate input (NULL: no gate)
 *   y          [batch, seqlen, d_inner]  output, written in the I/O type
 *   last_state [batch, d_inner, d_state] fp32 or NULL   h after the last token
 * seqlen == 0 writes zeros to last_state; batch == 0 or d_inner == 0 is a no-op.
 * Returns SS_OK or an error code (see above). */
SS_API int ss_fwd(const void* u, const void* delta, const float* delta_bias, const float* A,
           const void* B, const void* C, const float* D, const void* z, void* y,
           float* last_state, uint32_t flags, const ss_dims* dims, const ss_launch* launch);

/* ss_step -- one decode step: for every (b, channel) the state row is
 * advanced by one token and y is produced, as ss_fwd would do for that token.
 *   state      [batch, d_inner, d_state] fp32, read and overwritten in place
 *   u, delta   [batch, d_inner]          this token's input and raw Δ
 *   A          [d_inner, d_state] fp32
 *   B, C       [batch, d_state]
 *   D          [d_inner] fp32 or NULL
 *   z          [batch, d_inner] or NULL
 *   y          [batch, d_inner]          output
 *   delta_bias [d_inner] fp32 or NULL
 * dims->seqlen is ignored; launch->workspace is not used.  Returns SS_OK or
 * an error code. */
SS_API int ss_step(float* state, const void* u, const void* delta, const float* A, const void* B,
            const void* C, const float* D, const void* z, void* y, const float* delta_bias,
            uint32_t flags, const ss_dims* dims, const ss_launch* launch);

/* ss_fwd_conv -- ss_fwd with the causal conv1d + SiLU prologue fused into the
 * scan: the input of the recurrence is
 *   u_t = silu(conv_b + Σ_{k=0}^{3} conv_w[ch, k] · x_{t-3+k}),  x_{<0} = 0,
 * the Conv1D layer of width d_conv = 4 in front of the SSM ("Understanding
 * Mamba and Selective State Space Models (SSMs)" §3.3: causal, each token
 * sees itself and the previous three; the SiLU after it is not on the
 * pages and is the Mamba block's reading).  u never touches memory.
 *   x          [batch, seqlen, d_inner] in the element type (takes u's place)
 *   conv_w     [d_inner, 4] fp32; tap 3 multiplies the current token
 *   conv_b     [d_inner] fp32, or NULL
 *   conv_state [batch, d_inner, 3] fp32, or NULL: receives x_{L-3} .. x_{L-1}
 *              (zero before the sequence), the state ss_step_conv continues from
 * Everything else, including y = (Σ_n C h + D u) · gate with this u, is as in
 * ss_fwd; errors as ss_fwd, and SS_ERR_INVALID_ARG for a NULL conv_w. */
SS_API int ss_fwd_conv(const void* x, const float* conv_w, const float* conv_b, const void* delta,
                       const float* delta_bias, const float* A, const void* B, const void* C, const float* D,
                       const void* z, void* y, float* last_state, float* conv_state, uint32_t flags,
                       const ss_dims* dims, const ss_launch* launch);

/* ss_step_conv -- ss_step with the same prologue for one token:
 *   conv_state [batch, d_inner, 3] fp32, read and overwritten: the previous
 *              three x of each channel, oldest first
 *   x          [batch, d_inner], this token's input (takes u's place)
 * u = silu(conv_b + w0 s0 + w1 s1 + w2 s2 + w3 x), then the SSM step of
 * ss_step on u, and the conv state becomes (s1, s2, x).  ss_fwd_conv over L
 * tokens equals L calls of ss_step_conv from zero states.  Errors as ss_step,
 * and SS_ERR_INVALID_ARG for a NULL conv_w or conv_state. */
SS_API int ss_step_conv(float* state, float* conv_state, const void* x, const float* conv_w, const float* conv_b,
                        const void* delta, const float* A, const void* B, const void* C, const float* D,
                        const void* z, void* y, const float* delta_bias, uint32_t flags, const ss_dims* dims,
                        const ss_launch* launch);

/* Weights of one Mamba block (bf16 matrices row-major [out, in]; fp32 vectors).
 * The block's interface is the README's Usage > Mamba (d_model, d_state = 16,
 * d_conv = 4, expand = 2 so d_inner = 2 d_model; output shaped like the input;
 * "roughly 3 · expand · d_model^2 parameters"); Δ comes from a linear
 * projection whose bias sets its range (README, Initialization). */
typedef struct ss_block_weights {
    const void* in_proj_x;   /* [d_inner, d_model] bf16: x = hidden · in_proj_xᵀ */
    const void* in_proj_z;   /* [d_inner, d_model] bf16: z = hidden · in_proj_zᵀ (the gate input) */
    const float* conv_w;     /* [d_inner, 4] causal conv1d taps, tap 3 on the current token */
    const float* conv_b;     /* [d_inner] or NULL */
    const void* x_proj_dt;   /* [dt_rank, d_inner] bf16: Δ's low-rank input = u · x_proj_dtᵀ */
    const void* x_proj_B;    /* [16, d_inner] bf16: B = u · x_proj_Bᵀ */
    const void* x_proj_C;    /* [16, d_inner] bf16: C = u · x_proj_Cᵀ */
    const void* dt_proj;     /* [d_inner, dt_rank] bf16: Δraw = (u · x_proj_dtᵀ) · dt_projᵀ */
    const float* dt_bias;    /* [d_inner] Δ's projection bias (added before the softplus) */
    const float* A;          /* [d_inner, 16] (negative; A = -exp(A_log)) */
    const float* D;          /* [d_inner] or NULL */
    const void* out_proj;    /* [d_model, d_inner] bf16: out = y · out_projᵀ */
    int64_t d_model, d_inner, dt_rank;
} ss_block_weights;

/* ss_block_fwd -- forward of one Mamba block's inner path, bf16 activations:
 *   x, z = hidden · in_proj_xᵀ, hidden · in_proj_zᵀ
 *   u    = silu(conv_b + causal_conv4(x))                  (deep-dive §3.3)
 *   Δraw = (u · x_proj_dtᵀ) · dt_projᵀ,  B = u · x_proj_Bᵀ,  C = u · x_proj_Cᵀ
 *   y    = ss_fwd(u, Δraw, A, B, C, D, z, dt_bias, softplus on)
 *   out  = y · out_projᵀ
 *   hidden, out  [batch, seqlen, d_model] bf16 (device)
 *   scratch      device buffer of at least ss_block_scratch_bytes() bytes,
 *                16-byte aligned: the bf16 intermediates, the scan's
 *                workspace and cuBLAS's workspace (nothing is allocated)
 *   stream       cudaStream_t
 * The projections run on cuBLAS (bf16 operands, fp32 accumulation); the conv
 * and the scan are this library's kernels.  Errors: SS_ERR_INVALID_ARG for
 * NULL/misaligned pointers or sizes (d_inner and d_model multiples of 8),
 * SS_ERR_WORKSPACE for a small scratch, SS_ERR_CUDA for a CUDA or cuBLAS
 * failure. */
SS_API int ss_block_fwd(const void* hidden, void* out, const ss_block_weights* w, int64_t batch, int64_t seqlen,
                        void* scratch, size_t scratch_bytes, void* stream);

/* Scratch bytes ss_block_fwd needs (0 for invalid sizes). */
SS_API size_t ss_block_scratch_bytes(const ss_block_weights* w, int64_t batch, int64_t seqlen);

/* Sizes of a multi-head scalar-decay scan (ss_ssd_fwd). */
typedef struct ss_ssd_dims {
    int64_t batch;
    int64_t seqlen;
    int64_t nheads;
    int64_t headdim;   /* must be 64 */
    int64_t d_state;   /* 64 or 128 */
} ss_ssd_dims;

/* ss_ssd_fwd -- the multi-head scan with one scalar decay per head and step
 * (the Mamba-2 / "State Space Dual" model of the mamba README's Mamba-2
 * section and the model-architecture page's "Mamba-2 (multi-head, larger
 * state)": headdim 64, d_state 64 or 128, ngroups 1 -- B and C shared by all
 * heads).  For each (b, head h), with the head's channels p sharing Δ, B, C:
 *   Δ_t = softplus(dt_t,h + dt_bias_h)   (dt + bias without SS_DELTA_SOFTPLUS)
 *   H_t[p, n] = exp(Δ_t A_h) H_{t-1}[p, n] + Δ_t B_t,n x_t,h,p,   H_{-1} = 0
 *   y_t,h,p = Σ_n C_t,n H_t[p, n] + D_h x_t,h,p
 *   x, y         [batch, seqlen, nheads, headdim] bf16
 *   dt           [batch, seqlen, nheads] bf16
 *   A            [nheads] fp32 (negative); dt_bias, D [nheads] fp32 or NULL
 *   B, C         [batch, seqlen, d_state] bf16
 *   final_state  [batch, nheads, headdim, d_state] fp32 or NULL
 *   flags        SS_DELTA_SOFTPLUS, SS_SYNC_CHECK (bf16 only; SS_BF16 ignored);
 *                SS_TEST_DROP_CARRY for tests
 *   launch       stream; workspace (optional, see below); chunk_len > 0
 *                fixes the segment length (rounded up to whole chunks),
 *                0 lets the library choose; timeout_iters the bound on one
 *                wait in microseconds, 0 for two seconds
 * Computed chunk by chunk (128 steps) as dense bf16 products with fp32
 * accumulation on the tensor cores -- tcgen05 MMAs, TMEM accumulators,
 * TMA-staged tiles -- the carried state fp32 on chip; d_state 64 runs the
 * same kernel with B, C and the state padded to 128 with zeros.  With a workspace of at least
 * ss_ssd_fwd_workspace_bytes(dims, flags) bytes (16-byte aligned; the call
 * owns it until its work on the stream is done) the library may also cut
 * each sequence into up to 8 segments run in parallel, when batch x heads
 * leaves SMs idle: a first pass computes each segment's end state from
 * zero, a fold makes every segment's entering state exact, and the main
 * pass runs the segments from those (results equal to the unsplit scan up
 * to rounding).  A NULL workspace never splits; a smaller one is
 * SS_ERR_WORKSPACE.  The workspace's first word is a status word the call
 * clears: the kernels bound every wait (2 s) and record
 * SS_ERR_TIMEOUT there if one runs out; with SS_SYNC_CHECK the call
 * synchronises the stream and returns that word.
 * Errors: SS_ERR_INVALID_ARG for NULL/misaligned pointers or sizes,
 * SS_ERR_UNSUPPORTED for headdim != 64 or d_state not 64 or 128,
 * SS_ERR_CUDA for a failed launch or (with SS_SYNC_CHECK) a stream error. */
SS_API int ss_ssd_fwd(const void* x, const void* dt, const float* dt_bias, const float* A, const void* B,
                      const void* C, const float* D, void* y, float* final_state, uint32_t flags,
                      const ss_ssd_dims* dims, const ss_launch* launch);

/* Workspace bytes that let ss_ssd_fwd split sequences into segments
 * (records for up to 8 segments); 0 for sizes it would reject. */
SS_API size_t ss_ssd_fwd_workspace_bytes(const ss_ssd_dims* dims, uint32_t flags);

/* ss_bwd -- backward of ss_fwd: given dy = dJ/dy and optionally
 * dlast_state = dJ/dlast_state for a scalar J, writes dJ/d(input) for every
 * input of ss_fwd with the same u, delta, delta_bias, A, B, C, D, z and flags
 * (SS_BF16, SS_DELTA_SOFTPLUS, SS_SYNC_CHECK).  With g_n = dJ/dh_t,n run
 * backwards in time from dlast_state:
 *   ds = dy gate(z),  dz = dy s gate'(z)  (s = Σ_n C h + D u, gate = z σ(z)),
 *   g += ds C,  dC += ds h_t,  dB += g Δ u,  du = ds D + Σ_n g Δ B,
 *   dΔ = Σ_n g (exp(Δ A) A h_{t-1} + B u),  dA += g exp(Δ A) Δ h_{t-1},
 *   g <- exp(Δ A) g,  ddelta = dΔ softplus'(Δraw + bias),  ddelta_bias += ddelta.
 * Inputs: as ss_fwd, plus
 *   dy           [batch, seqlen, d_inner], the element type of u
 *   dlast_state  [batch, d_inner, d_state] fp32, or NULL (zero)
 * Outputs (all written; the accumulated ones are zeroed by the call first):
 *   du, ddelta, dz  [batch, seqlen, d_inner], the element type of u
 *                   (ddelta is the gradient with respect to the raw Δ;
 *                   dz must be non-NULL exactly when z is)
 *   dA              [d_inner, d_state] fp32 (summed over batch and time)
 *   dB, dC          [batch, seqlen, d_state] fp32 (summed over channels)
 *   dD, ddelta_bias [d_inner] fp32 (summed over batch and time), or NULL to
 *                   skip; non-NULL dD needs D, non-NULL ddelta_bias needs
 *                   delta_bias
 * Workspace: launch->workspace of at least ss_bwd_workspace_bytes(dims)
 * bytes (forward-state checkpoints every 32 steps), 16-byte aligned, else
 * SS_ERR_WORKSPACE.  The sums over channels, batch and time use float
 * atomic adds, so the last bits of dA, dB, dC, dD and ddelta_bias depend on
 * the order the hardware applies them in.  The sequence is cut into time
 * chunks (launch->chunk_len > 0 fixes their length; 0 lets the library
 * choose), scanned in three launches: a chunk pass (each chunk's forward
 * from zero, with state checkpoints every 32 steps, and for every chunk but
 * the last the adjoint-only recurrence from zero), a fold of the chunk
 * records into each chunk's exact entering forward state and adjoint, and
 * the gradient pass over (batch, 64-channel block, chunk) items.
 * Errors: as ss_fwd (SS_ERR_INVALID_ARG for a NULL required pointer, a
 * misaligned pointer or dz/z mismatch). */
SS_API int ss_bwd(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                  const void* C, const float* D, const void* z, const void* dy, const float* dlast_state,
                  void* du, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
                  float* ddelta_bias, uint32_t flags, const ss_dims* dims, const ss_launch* launch);

/* ss_fwd_with_state -- ss_fwd from a given entering state instead of zero:
 * h_{-1} = h_init ([batch, d_inner, d_state] fp32, device, 16-byte aligned;
 * NULL is ss_fwd).  Continues a sequence after a previous call's last_state
 * (a prompt processed in pieces, or the tail of a sequence whose head was
 * scanned elsewhere): ss_fwd over [0, T) then ss_fwd_with_state over [T, L)
 * from its last_state gives ss_fwd over [0, L) up to rounding.  Only the
 * first time chunk reads h_init; the chunks' carry takes it to the rest.
 * With seqlen 0, last_state = h_init.  Other arguments, workspace and errors:
 * as ss_fwd.  (An engineering addition: the pages start every sequence from
 * h = 0.) */
SS_API int ss_fwd_with_state(const void* u, const void* delta, const float* delta_bias, const float* A,
                             const void* B, const void* C, const float* D, const void* z, const float* h_init,
                             void* y, float* last_state, uint32_t flags, const ss_dims* dims,
                             const ss_launch* launch);

/* ss_fwd_host -- ss_fwd on activations in HOST memory (an engineering
 * addition: the pages have no counterpart).  u, delta, z, B, C (inputs) and
 * y, last_state (outputs) are host pointers, same layouts and element types
 * as ss_fwd; page-locked (pinned) memory lets the copies run asynchronously,
 * pageable memory works but copies synchronously.  A, D and delta_bias are
 * DEVICE pointers (parameters stay resident).  The batch is cut into slices
 * of rows_per_slice rows (0 or less: 1); slice s is uploaded on a copy
 * stream, scanned on launch->stream and downloaded on a second copy stream,
 * through two device staging slots, so uploads, scans and downloads of
 * neighbouring slices overlap.  The results equal ss_fwd applied to each
 * slice.  launch->workspace is the staging: at least
 * ss_fwd_host_workspace_bytes(dims, flags, rows_per_slice) bytes, 16-byte
 * aligned, else SS_ERR_WORKSPACE; it must stay untouched until the call's
 * work on launch->stream completes.  The copy streams and their events are
 * created on the first call of each host thread on each device and kept.
 * The call is asynchronous on launch->stream: y and last_state are complete
 * once launch->stream has been synchronized (SS_SYNC_CHECK does it and
 * returns the device status).  The workspace starts with one status word
 * shared by all slices: a device-side failure in any slice stays recorded
 * there, so ss_check(launch) after the call (or SS_SYNC_CHECK) reports it.
 * SS_TEST_DROP_CARRY applies to the caller's batch entry 0 (the first
 * slice) only.  Errors: as ss_fwd. */
SS_API int ss_fwd_host(const void* u, const void* delta, const float* delta_bias, const float* A, const void* B,
                       const void* C, const float* D, const void* z, void* y, float* last_state, uint32_t flags,
                       const ss_dims* dims, const ss_launch* launch, int32_t rows_per_slice);

/* Staging bytes ss_fwd_host needs (two slices' activations and states plus
 * one slice's ss_fwd workspace); 0 for sizes it would reject. */
SS_API size_t ss_fwd_host_workspace_bytes(const ss_dims* dims, uint32_t flags, int32_t rows_per_slice);

/* Workspace bytes ss_bwd needs for these sizes (0 for invalid dims). */
SS_API size_t ss_bwd_workspace_bytes(const ss_dims* dims, uint32_t flags);

/* Workspace bytes ss_fwd needs for these sizes, flags and chunk length
 * (chunk_len 0: the library's own choice, the same one ss_fwd makes):
 * 256 bytes of header without time chunking, plus per-chunk carry records
 * (48 floats per (batch, chunk, channel)) and status words with it.
 * 0 for sizes ss_fwd would reject. */
SS_API size_t ss_fwd_workspace_bytes(const ss_dims* dims, uint32_t flags, int32_t chunk_len);

/* Chunk length ss_fwd uses for these sizes when launch->chunk_len is 0
 * (0 when the scan is not split in time). */
SS_API int32_t ss_fwd_chunk_len(const ss_dims* dims, uint32_t flags);

/* Synchronize launch->stream and return the device-side status recorded in
 * launch->workspace by the last ss_fwd on it (SS_OK when there is no
 * workspace), or SS_ERR_CUDA if the stream reports an error. */
SS_API int ss_check(const ss_launch* launch);

/* Human-readable name of a status code (static storage). */
SS_API const char* ss_status_string(int status);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
SS_API int ss_version(void);

/* Capacity of the scratch array behind ss_fwd_noalloc, in bytes. */
#define SS_NOALLOC_SCRATCH_BYTES (32u << 20)

/* ss_fwd_noalloc -- ss_fwd for callers that cannot allocate device memory.
 * (An engineering addition: the paper has no counterpart.)
 *
 * Some callers have no way to hand ss_fwd a workspace: runtimes that plan
 * every byte of device memory ahead of time and forbid allocation while
 * serving, plugin interfaces of host frameworks that pass an operator its
 * inputs and outputs but no allocator or scratch buffer, and latency-bound
 * paths that cannot afford cudaMalloc, which may synchronize the device.
 * This entry point takes the same arguments as ss_fwd except the launch
 * context (only a stream) and uses, as its workspace, one array of
 * SS_NOALLOC_SCRATCH_BYTES that the library reserves in device memory when
 * it is loaded (every GPU that loads the library holds it until the process
 * exits).  It calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * - The first call on each device looks up that array's device address for
 *   the current device (once; later calls reuse it).  Make that first call
 *   before any stream capture.
 * - Problems whose scratch need (ss_fwd_workspace_bytes with chunk_len 0)
 *   exceeds SS_NOALLOC_SCRATCH_BYTES are rejected with SS_ERR_WORKSPACE
 *   before anything is launched.
 * - Every call on a device shares the one array; each call resets the parts
 *   that must start at zero.  Calls whose work overlaps on the GPU (other
 *   streams, other host threads) race on it and give wrong results: order
 *   them on one stream.
 * - Pass SS_SYNC_CHECK in flags to synchronize and get the device status;
 *   ss_check cannot be used (the array is not exposed).  Without
 *   SS_SYNC_CHECK a device-side failure (a bounded cross-chunk wait that ran
 *   out: SS_ERR_TIMEOUT, its outputs invalid) is not reported to the caller
 *   at all, so callers that cannot afford the synchronization accept that.
 * Returns the same codes as ss_fwd. */
SS_API int ss_fwd_noalloc(const void* u, const void* delta, const float* delta_bias, const float* A,
                          const void* B, const void* C, const float* D, const void* z, void* y,
                          float* last_state, uint32_t flags, const ss_dims* dims, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SELSCAN_H */
