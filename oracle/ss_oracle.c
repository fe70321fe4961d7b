/*
 * ss_oracle.c -- plain CPU oracle of the Mamba selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this file.  The product path (the
 * CUDA library) never calls it and shares no code with it.
 *
 * What it computes follows the equations of "Understanding Mamba and Selective
 * State Space Models (SSMs)" (bqwf.cn deep-dive article):
 *   - §2.1   classic SSM, y_n = C h_n + D x_n (skip term D);
 *   - §2.2, first cut: the selective recurrence h_n = exp(Δ_n A) h_{n-1} + Δ_n B_n x_n;
 *   - §2.2, second cut: the recurrent scan, state starting at zero;
 *   - §2.2, closing tip: Δ goes through softplus, log(1 + exp(x));
 *   - §3.1 (end): the readout against C_n;
 *   - §4.3: A = -exp(A_log), a diagonal matrix, so every state index n
 *     evolves on its own.
 * The optional silu(z) output gate and the bias added to Δ before the softplus
 * are not on the pages; they follow the benchmark spec of the path
 * (y = (C_t·h_t + D u_t) * z σ(z), Δ = softplus(Δ_raw + bias)).
 *
 * Readings taken where the pages are garbled or silent (each is listed in the
 * design notes):
 *   - decay = exp(Δ·A) with A as given (negative); the pseudocode's
 *     "exp(-Δ·A)" assumes a positive magnitude for A;
 *   - the readout is the dot product Σ_n C_n h_n (the "⊙" of §3.1 would
 *     leave an N-vector per channel, contradicting y_n = C h_n of §2.1);
 *   - B̄ = Δ·B (as written), h_{-1} = 0;
 *   - D is one constant per channel;
 *   - softplus(x) = x for x > 20, else log1p(exp(x)).
 *
 * Layouts (row-major, no padding):
 *   u, delta, z, y : [batch, L, d]       (token-major, channels contiguous)
 *   B, C           : [batch, L, N]       (one group shared by all channels)
 *   A              : [d, N]
 *   D, delta_bias  : [d]
 *   last_state     : [batch, d, N]
 * Inputs come in as double; callers pass the exact values the GPU consumed
 * (bf16 or fp32 values widen to double without rounding).
 *
 * Two arithmetic modes:
 *   *_f64 : everything in double (the reference truth);
 *   *_f32 : state and all arithmetic in float, libm float functions.
 *
 * Nothing here is blocked, fused or reordered: each channel runs the
 * recurrence step by step in time order, exactly as the equations read.
 * The only parallelism is an OpenMP loop over independent (batch, channel)
 * pairs.
 *
 * Parity pins (tests/test_oracle_pins.py): closed form at L = 1, LTI
 * reduction to a direct convolution, linearity in u, chunked = sequential,
 * causality, channel independence, limiting cases, a hand-derived worked
 * example, and step-by-step decode equivalence.  The backward (adjoint) at
 * the end of this file is pinned by central finite differences of the
 * forward (tests/test_oracle_bwd_pins.py).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------------
 * Test-only planted mistakes.  0 (the default) is the oracle as specified;
 * a nonzero value switches on ONE deliberate error so that a test can show
 * that the pins catch it.  Never set outside tests.
 *   1: decay exp(-Δ·A) (the pseudocode's sign taken literally)
 *   2: skip term D dropped
 *   3: B and C swapped
 *   4: Δ bias ignored
 *   5: softplus skipped (Δ = Δ_raw + bias)
 *   6: readout taken before the state update (uses h_{t-1})
 *   7: gate σ(z) instead of z·σ(z)
 *   8: Δ missing from the input term (h = Ā h + B u)
 *   9: A read transposed (A[n*d + ch] instead of A[ch*N + n])
 * ------------------------------------------------------------------------- */
static int g_mutation = 0;
void ss_oracle_set_mutation(int m) { g_mutation = m; }
int ss_oracle_get_mutation(void) { return g_mutation; }

int ss_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void ss_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* softplus in double: log(1 + e^x), with the identity branch above 20
 * (there log1p(e^x) - x < 2.1e-9, below the precision either side keeps). */
static double softplus_d(double x)
{
    return x > 20.0 ? x : log1p(exp(x));
}

static float softplus_f(float x)
{
    return x > 20.0f ? x : log1pf(expf(x));
}

static double a_at_d(const double* A, int64_t ch, int64_t n, int64_t d, int64_t N)
{
    if (g_mutation == 9) return A[n * d + ch];
    return A[ch * N + n];
}

/* Δ for one element, double. */
static double delta_d(double raw, const double* bias, int64_t ch, int softplus)
{
    double x = raw;
    if (bias && g_mutation != 4) x += bias[ch];
    if (softplus && g_mutation != 5) return softplus_d(x);
    return x;
}

static float delta_f(float raw, const double* bias, int64_t ch, int softplus)
{
    float x = raw;
    if (bias && g_mutation != 4) x += (float)bias[ch];
    if (softplus && g_mutation != 5) return softplus_f(x);
    return x;
}

static double gate_d(double zv)
{
    double sig = 1.0 / (1.0 + exp(-zv));
    return g_mutation == 7 ? sig : zv * sig;
}

static float gate_f(float zv)
{
    float sig = 1.0f / (1.0f + expf(-zv));
    return g_mutation == 7 ? sig : zv * sig;
}

/* ---------------------------------------------------------------------------
 * Forward scan, double precision.
 * For every (b, ch): h = 0; for t in 0..L-1:
 *   Δ  = softplus(Δ_raw + bias)
 *   h_n = exp(Δ A_n) h_n + Δ B_n u          (n = 0..N-1)
 *   y  = (Σ_n C_n h_n + D u) · z σ(z)
 * and last_state = h after the final step.
 * The state lives in a stack array, so N <= 256 is required.
 * Returns 0, or -1 for unsupported sizes.
 * ------------------------------------------------------------------------- */
int ss_oracle_fwd_f64(const double* u, const double* delta, const double* delta_bias,
                      const double* A, const double* B, const double* C,
                      const double* D, const double* z, double* y, double* last_state,
                      int64_t batch, int64_t L, int64_t d, int64_t N, int softplus)
{
    if (N < 1 || N > 256 || batch < 0 || L < 0 || d < 0) return -1;
    const double* Bsel = (g_mutation == 3) ? C : B;
    const double* Csel = (g_mutation == 3) ? B : C;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            double h[256];
            for (int64_t n = 0; n < N; ++n) h[n] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = (b * L + t) * d + ch;      /* [b, t, ch] */
                const int64_t bc = (b * L + t) * N;          /* [b, t, 0]  */
                const double dt = delta_d(delta[i], delta_bias, ch, softplus);
                const double uv = u[i];
                double acc = 0.0;
                if (g_mutation == 6)
                    for (int64_t n = 0; n < N; ++n) acc += Csel[bc + n] * h[n];
                for (int64_t n = 0; n < N; ++n) {
                    const double an = a_at_d(A, ch, n, d, N);
                    const double decay = (g_mutation == 1) ? exp(-dt * an) : exp(dt * an);
                    const double input = (g_mutation == 8) ? Bsel[bc + n] * uv
                                                            : dt * Bsel[bc + n] * uv;
                    h[n] = decay * h[n] + input;
                }
                if (g_mutation != 6)
                    for (int64_t n = 0; n < N; ++n) acc += Csel[bc + n] * h[n];
                double yv = acc;
                if (D && g_mutation != 2) yv += D[ch] * uv;
                if (z) yv *= gate_d(z[i]);
                y[i] = yv;
            }
            if (last_state)
                for (int64_t n = 0; n < N; ++n) last_state[(b * d + ch) * N + n] = h[n];
        }
    }
    return 0;
}

/* Forward scan with the state and every operation in float (the fp32-state
 * oracle).  Same loop as ss_oracle_fwd_f64; outputs widened to double. */
int ss_oracle_fwd_f32(const double* u, const double* delta, const double* delta_bias,
                      const double* A, const double* B, const double* C,
                      const double* D, const double* z, double* y, double* last_state,
                      int64_t batch, int64_t L, int64_t d, int64_t N, int softplus)
{
    if (N < 1 || N > 256 || batch < 0 || L < 0 || d < 0) return -1;
    const double* Bsel = (g_mutation == 3) ? C : B;
    const double* Csel = (g_mutation == 3) ? B : C;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            float h[256];
            for (int64_t n = 0; n < N; ++n) h[n] = 0.0f;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = (b * L + t) * d + ch;
                const int64_t bc = (b * L + t) * N;
                const float dt = delta_f((float)delta[i], delta_bias, ch, softplus);
                const float uv = (float)u[i];
                float acc = 0.0f;
                if (g_mutation == 6)
                    for (int64_t n = 0; n < N; ++n) acc += (float)Csel[bc + n] * h[n];
                for (int64_t n = 0; n < N; ++n) {
                    const float an = (float)a_at_d(A, ch, n, d, N);
                    const float decay = (g_mutation == 1) ? expf(-dt * an) : expf(dt * an);
                    const float input = (g_mutation == 8) ? (float)Bsel[bc + n] * uv
                                                           : dt * (float)Bsel[bc + n] * uv;
                    h[n] = decay * h[n] + input;
                }
                if (g_mutation != 6)
                    for (int64_t n = 0; n < N; ++n) acc += (float)Csel[bc + n] * h[n];
                float yv = acc;
                if (D && g_mutation != 2) yv += (float)D[ch] * uv;
                if (z) yv *= gate_f((float)z[i]);
                y[i] = (double)yv;
            }
            if (last_state)
                for (int64_t n = 0; n < N; ++n)
                    last_state[(b * d + ch) * N + n] = (double)h[n];
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * One decode step (the streaming "step" of the tutorial pages: one token in,
 * state carried), double precision.  state [batch, d, N] is read and
 * overwritten; u, delta, z, y are [batch, d]; B, C are [batch, N].
 * The arithmetic is the body of the forward loop for a single t.
 * ------------------------------------------------------------------------- */
int ss_oracle_step_f64(double* state, const double* u, const double* delta,
                       const double* delta_bias, const double* A, const double* B,
                       const double* C, const double* D, const double* z, double* y,
                       int64_t batch, int64_t d, int64_t N, int softplus)
{
    if (N < 1 || batch < 0 || d < 0) return -1;
#pragma omp parallel for collapse(2)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            const int64_t i = b * d + ch;
            const double dt = delta_d(delta[i], delta_bias, ch, softplus);
            const double uv = u[i];
            double* h = state + i * N;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double an = a_at_d(A, ch, n, d, N);
                h[n] = exp(dt * an) * h[n] + dt * B[b * N + n] * uv;
                acc += C[b * N + n] * h[n];
            }
            double yv = acc;
            if (D) yv += D[ch] * uv;
            if (z) yv *= gate_d(z[i]);
            y[i] = yv;
        }
    }
    return 0;
}

/* Decode step with a float state and float arithmetic. */
int ss_oracle_step_f32(double* state, const double* u, const double* delta,
                       const double* delta_bias, const double* A, const double* B,
                       const double* C, const double* D, const double* z, double* y,
                       int64_t batch, int64_t d, int64_t N, int softplus)
{
    if (N < 1 || batch < 0 || d < 0) return -1;
#pragma omp parallel for collapse(2)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            const int64_t i = b * d + ch;
            const float dt = delta_f((float)delta[i], delta_bias, ch, softplus);
            const float uv = (float)u[i];
            double* h = state + i * N;
            float acc = 0.0f;
            for (int64_t n = 0; n < N; ++n) {
                const float an = (float)a_at_d(A, ch, n, d, N);
                const float hn = expf(dt * an) * (float)h[n] + dt * (float)B[b * N + n] * uv;
                h[n] = (double)hn;
                acc += (float)C[b * N + n] * hn;
            }
            float yv = acc;
            if (D) yv += (float)D[ch] * uv;
            if (z) yv *= gate_f((float)z[i]);
            y[i] = (double)yv;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Chunked forward scan, double precision: the time-parallel re-association
 * that a GPU uses, written out plainly so that "chunked = sequential" can be
 * checked on the CPU.
 *
 * The recurrence h_t = a_t ⊙ h_{t-1} + b_t is linear, so a chunk of steps acts
 * on its entry state as h_end = P ⊙ h_entry + h_loc, where P = Π a_t over the
 * chunk and h_loc is the chunk's end state when entered from zero.  Pairs
 * compose by (P, h) ∘ (P', h') = (P·P', P'·h + h').  The "hardware-aware
 * parallel algorithm" of the Mamba tutorial (discosf.com, §2.3) and the
 * single-launch scan of the deep-dive article (§2.2, second cut) rely on
 * exactly this associativity.
 *
 * Steps, per (b, ch):
 *   1. every chunk is scanned from a zero state, giving y_loc, P, h_loc;
 *   2. entry states are combined left to right: h0[0] = 0,
 *      h0[c+1] = P[c] ⊙ h0[c] + h_loc[c];
 *   3. each output gets the entry state's contribution:
 *      y_t = (y_loc,t + Σ_n C_t,n · Π_{s<=t in chunk} a_s,n · h0_n + D u_t) · gate.
 * The prefix product in step 3 is accumulated step by step.  The gate and
 * the D term are applied once, after the correction.
 * ------------------------------------------------------------------------- */
int ss_oracle_fwd_chunked_f64(const double* u, const double* delta, const double* delta_bias,
                              const double* A, const double* B, const double* C,
                              const double* D, const double* z, double* y, double* last_state,
                              int64_t batch, int64_t L, int64_t d, int64_t N, int softplus,
                              int64_t chunk)
{
    if (N < 1 || N > 256 || chunk < 1 || batch < 0 || L < 0 || d < 0) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            double h0[256];                      /* entry state of the current chunk */
            for (int64_t n = 0; n < N; ++n) h0[n] = 0.0;
            for (int64_t c0 = 0; c0 < L; c0 += chunk) {
                const int64_t c1 = (c0 + chunk < L) ? c0 + chunk : L;
                double hl[256], P[256];
                for (int64_t n = 0; n < N; ++n) { hl[n] = 0.0; P[n] = 1.0; }
                for (int64_t t = c0; t < c1; ++t) {
                    const int64_t i = (b * L + t) * d + ch;
                    const int64_t bc = (b * L + t) * N;
                    const double dt = delta_d(delta[i], delta_bias, ch, softplus);
                    const double uv = u[i];
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        const double a = exp(dt * a_at_d(A, ch, n, d, N));
                        hl[n] = a * hl[n] + dt * B[bc + n] * uv;  /* local state  */
                        P[n] *= a;                                /* prefix decay */
                        acc += C[bc + n] * (hl[n] + P[n] * h0[n]);
                    }
                    double yv = acc;
                    if (D) yv += D[ch] * uv;
                    if (z) yv *= gate_d(z[i]);
                    y[i] = yv;
                }
                /* combine: entry state of the next chunk */
                for (int64_t n = 0; n < N; ++n) h0[n] = P[n] * h0[n] + hl[n];
            }
            if (last_state)
                for (int64_t n = 0; n < N; ++n) last_state[(b * d + ch) * N + n] = h0[n];
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward of the forward scan, double precision (reverse mode by hand).
 *
 * Given the gradient dy = ∂J/∂y [batch, L, d] of a scalar J, and optionally
 * dlast = ∂J/∂last_state [batch, d, N], returns ∂J/∂ of every input:
 *   du, ddelta, dz : [batch, L, d]     (ddelta is with respect to Δ_raw)
 *   dB, dC         : [batch, L, N]     (summed over channels)
 *   dA             : [d, N]            (summed over batch and time)
 *   dD, dbias      : [d]               (summed over batch and time)
 * Outputs for absent optional inputs (D, z, bias) are left untouched and
 * may be NULL.
 *
 * For each (b, ch) the forward recurrence is run once, keeping x_t (the
 * softplus input), Δ_t, the states h_t and the pre-gate output s_t.  Then
 * time runs backwards with g_n = ∂J/∂h_t,n, starting from dlast:
 *   ds   = dy_t · gate(z_t)                         (y = s · gate)
 *   dz_t = dy_t · s_t · gate'(z_t),  gate'(z) = σ(z) (1 + z (1 - σ(z)))
 *   g_n += ds · C_t,n,      dC_t,n += ds · h_t,n    (s = Σ_n C h + D u)
 *   dD  += ds · u_t,        du_t    = ds · D
 *   with a_n = exp(Δ A_n) and the previous state h_{t-1}:
 *   dB_t,n += g_n Δ u_t,    du_t   += Σ_n g_n Δ B_t,n
 *   dΔ      = Σ_n g_n (a_n A_n h_{t-1},n + B_t,n u_t)
 *   dA_n   += g_n a_n Δ h_{t-1},n
 *   g_n     = a_n g_n                                (h_t = a h_{t-1} + ...)
 *   ddelta_t = dΔ · softplus'(x_t) (σ(x); 1 on the identity branch),
 *   dbias   += ddelta_t.
 * Channels run in parallel; the sums over channels (dB, dC) use atomic adds.
 * Test-only mutations 10..12 plant mistakes in this adjoint:
 *   10: softplus derivative dropped;  11: dA uses h_t instead of h_{t-1};
 *   12: the adjoint state is not decayed between steps.
 * Returns 0, or -1 for unsupported sizes / allocation failure.
 * ------------------------------------------------------------------------- */
int ss_oracle_bwd_f64(const double* u, const double* delta, const double* delta_bias,
                      const double* A, const double* B, const double* C,
                      const double* D, const double* z, const double* dy, const double* dlast,
                      double* du, double* ddelta, double* dA, double* dB, double* dC,
                      double* dD, double* dz, double* dbias,
                      int64_t batch, int64_t L, int64_t d, int64_t N, int softplus)
{
    if (N < 1 || N > 256 || batch < 0 || L < 0 || d < 0) return -1;
    for (int64_t i = 0; i < d * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < batch * L * N; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    if (D && dD) for (int64_t i = 0; i < d; ++i) dD[i] = 0.0;
    if (delta_bias && dbias) for (int64_t i = 0; i < d; ++i) dbias[i] = 0.0;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t ch = 0; ch < d; ++ch) {
        double* hs = (double*)malloc((size_t)(L + 1) * (size_t)N * sizeof(double));
        double* xs = (double*)malloc((size_t)(L + 1) * 3 * sizeof(double));
        if (!hs || !xs) {
            free(hs);
            free(xs);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        for (int64_t b = 0; b < batch; ++b) {
            /* forward, keeping h_t at hs[(t + 1) N .. ], h_{-1} = 0 at hs[0 .. N) */
            for (int64_t n = 0; n < N; ++n) hs[n] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = (b * L + t) * d + ch;
                const int64_t bc = (b * L + t) * N;
                const double x = delta[i] + (delta_bias ? delta_bias[ch] : 0.0);
                const double dt = softplus ? softplus_d(x) : x;
                const double* hp = hs + t * N;
                double* hn = hs + (t + 1) * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    hn[n] = exp(dt * A[ch * N + n]) * hp[n] + dt * B[bc + n] * u[i];
                    acc += C[bc + n] * hn[n];
                }
                xs[3 * t] = x;
                xs[3 * t + 1] = dt;
                xs[3 * t + 2] = acc + (D ? D[ch] * u[i] : 0.0);   /* s_t */
            }
            /* backward */
            double g[256];
            for (int64_t n = 0; n < N; ++n) g[n] = dlast ? dlast[(b * d + ch) * N + n] : 0.0;
            double dD_acc = 0.0, db_acc = 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const int64_t i = (b * L + t) * d + ch;
                const int64_t bc = (b * L + t) * N;
                const double x = xs[3 * t], dt = xs[3 * t + 1], s = xs[3 * t + 2];
                const double* hp = hs + t * N;         /* h_{t-1} */
                const double* hc = hs + (t + 1) * N;   /* h_t */
                double ds = dy[i];
                if (z) {
                    const double sig = 1.0 / (1.0 + exp(-z[i]));
                    ds = dy[i] * z[i] * sig;
                    dz[i] = dy[i] * s * sig * (1.0 + z[i] * (1.0 - sig));
                }
                double du_v = 0.0;
                if (D) {
                    dD_acc += ds * u[i];
                    du_v = ds * D[ch];
                }
                double dDelta = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double an = A[ch * N + n];
                    const double a = exp(dt * an);
                    g[n] += ds * C[bc + n];
#pragma omp atomic
                    dC[bc + n] += ds * hc[n];
#pragma omp atomic
                    dB[bc + n] += g[n] * dt * u[i];
                    du_v += g[n] * dt * B[bc + n];
                    dDelta += g[n] * (a * an * hp[n] + B[bc + n] * u[i]);
                    dA[ch * N + n] += g[n] * a * dt * (g_mutation == 11 ? hc[n] : hp[n]);
                    if (g_mutation != 12) g[n] *= a;
                }
                du[i] = du_v;
                double dx = dDelta;
                if (softplus && g_mutation != 10) dx = x > 20.0 ? dDelta : dDelta / (1.0 + exp(-x));
                ddelta[i] = dx;
                db_acc += dx;
            }
            if (D && dD) dD[ch] += dD_acc;
            if (delta_bias && dbias) dbias[ch] += db_acc;
        }
        free(hs);
        free(xs);
    }
    return failed ? -1 : 0;
}

/* ---------------------------------------------------------------------------
 * Causal depthwise conv1d of width W followed by SiLU, double precision: the
 * Conv1D embedding in front of the SSM ("Understanding Mamba and Selective
 * State Space Models (SSMs)" §3.3: d_conv = 4, each position sees itself
 * and the previous 3 tokens, causal), producing the scan's input u:
 *   c_t = bias[ch] + Σ_{k=0}^{W-1} w[ch, k] · x_{t-(W-1)+k}    (x_{<0} = 0)
 *   u_t = c_t σ(c_t)
 * x, u : [batch, L, d];  w : [d, W];  bias : [d] or NULL.
 * ------------------------------------------------------------------------- */
int ss_oracle_conv_silu_f64(const double* x, const double* w, const double* bias, double* u,
                            int64_t batch, int64_t L, int64_t d, int64_t W)
{
    if (W < 1 || batch < 0 || L < 0 || d < 0) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t ch = 0; ch < d; ++ch) {
            for (int64_t t = 0; t < L; ++t) {
                double c = bias ? bias[ch] : 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    const int64_t s = t - (W - 1) + k;
                    if (s >= 0) c += w[ch * W + k] * x[(b * L + s) * d + ch];
                }
                u[(b * L + t) * d + ch] = c / (1.0 + exp(-c));
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Multi-head scan with a scalar decay per head (the Mamba-2 / SSD model of
 * the mamba README's Mamba-2 section and the model-architecture page's
 * "Mamba-2 (multi-head, larger state)": headdim P, d_state N, ngroups = 1),
 * double precision, plain recurrence.  For each (b, head h), with the head's
 * P channels sharing Δ, B and C:
 *   Δ_t     = softplus(dt_t,h + dt_bias_h)        (or dt + bias without softplus)
 *   H_t[p,n] = exp(Δ_t A_h) H_{t-1}[p,n] + Δ_t B_t,n x_t,h,p
 *   y_t,h,p = Σ_n C_t,n H_t[p,n] + D_h x_t,h,p
 * starting from H = 0.  Layouts: x, y [batch, L, H, P]; dt [batch, L, H];
 * A, dt_bias, D [H]; B, C [batch, L, N]; final_state [batch, H, P, N].
 * ------------------------------------------------------------------------- */
int ss_oracle_ssd_f64(const double* x, const double* dt, const double* dt_bias, const double* A,
                      const double* B, const double* C, const double* D, double* y, double* final_state,
                      int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int softplus)
{
    if (batch < 0 || L < 0 || H < 0 || P < 1 || N < 1 || P * N > (1 << 20)) return -1;
    int failed = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            double* st = (double*)calloc((size_t)(P * N), sizeof(double));
            if (!st) {
#pragma omp atomic write
                failed = 1;
                continue;
            }
            for (int64_t t = 0; t < L; ++t) {
                const double xr = dt[(b * L + t) * H + h] + (dt_bias ? dt_bias[h] : 0.0);
                const double delta = softplus ? softplus_d(xr) : xr;
                const double a = exp(delta * A[h]);
                const double* Bt = B + (b * L + t) * N;
                const double* Ct = C + (b * L + t) * N;
                const double* xt = x + ((b * L + t) * H + h) * P;
                double* yt = y + ((b * L + t) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        st[p * N + n] = a * st[p * N + n] + delta * Bt[n] * xt[p];
                        acc += Ct[n] * st[p * N + n];
                    }
                    yt[p] = acc + (D ? D[h] * xt[p] : 0.0);
                }
            }
            if (final_state)
                for (int64_t i = 0; i < P * N; ++i) final_state[(b * H + h) * P * N + i] = st[i];
            free(st);
        }
    }
    return failed ? -1 : 0;
}
