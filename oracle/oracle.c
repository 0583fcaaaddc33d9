/*
 * CPU oracle for the Mamba selective-scan forward and the single-token state
 * update: plain, sequential, double precision.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU
 * baseline load this file's library. It shares no code, header, table or helper
 * with the CUDA path, and nothing in the CUDA path may call it.
 *
 * What it computes (each function cites the passage it follows):
 *  - The Mamba block "runs a short causal convolution, then feeds the result to
 *    the selective scan", with A derived as negative exponentials of A_log
 *    (pyshine.com "Mamba" tour, the detailed-map paragraph on the block).
 *  - The convolution is causal: output t depends only on inputs at positions <= t
 *    (qwerky.ai "Bringing ... SSMs to the Modular MAX Framework", "What We Built").
 *  - delta passes through softplus after adding the dt bias (pyshine.com tour,
 *    "Why You Need This": softplus of the bias sets each channel's time constant).
 *  - A is diagonal, so discretisation is a scalar exponential per state
 *    (paperlayer.ai summary of arXiv 2603.09555, §3 Method, "State-space duality").
 *  - The recurrence keeps a fixed-size hidden state, updated step by step
 *    (qwerky.ai, "Why State Space Models? Why Mamba?").
 *  - D (skip) and the z gate are optional (pyshine.com tour, the CUDA-core
 *    paragraph: dispatch on "whether D exists, whether z gating is present").
 *  - The step method applies the same math to one token, updating the conv and
 *    SSM states in place (pyshine.com tour, the block paragraph).
 *  - The bidirectional variant (kanishk-sama.me "ARM Selective-Scan Kernel",
 *    "What I built") is composed from the forward and reverse scans by the Python
 *    wrapper.
 *
 * Readings taken where the pages are silent (each is also listed with the design):
 *  - conv is a cross-correlation with W-1 zeros of history on the left:
 *    w[d][W-1] multiplies x[t], w[d][0] multiplies x[t-W+1]; bias before SiLU.
 *  - delta = softplus(dt + bias) when delta_softplus, else dt + bias.
 *  - y = sum_n C[n] h[n] + D u, then y *= silu(z): the skip term sits inside the gate.
 *  - reverse = the forward scan of the flipped sequence, flipped back; with a fused
 *    conv the convolution runs over the flipped x as well.
 *  - the reverse final state is the state after position 0 (its last step).
 *  - decode conv state holds the last W inputs, newest last; it shifts left by one
 *    and appends x_t before the convolution.
 *  - B and C are either input-dependent, (Bsz, N, L) and shared by all channels, or
 *    time-invariant, (D, N): one fixed row per channel, the same at every position
 *    (pyshine.com tour, the CUDA-core paragraph: the kernel dispatches on "whether B
 *    and C are variable or shared"; the time-invariant form is the classic LTI SSM).
 *  - a forward scan may continue a sequence processed earlier (a prompt taken in
 *    pieces, or a prefill after decode steps): it then starts from that sequence's
 *    state h0 and its conv reads the W-1 inputs that preceded position 0 (conv_hist,
 *    oldest first) where it would otherwise read zeros. The pages carry the conv and
 *    SSM states across calls in the step method and the inference cache (pyshine.com
 *    tour, the block paragraph; paperlayer.ai summary, §3 Method, "Autoregressive
 *    cache"); the same two states let a scan pick up where another call stopped.
 *
 * Parity pins: every function here is checked, on CPU, against closed forms,
 * brute-force products and invariants that do not call it twice the same way.
 */
#include <math.h>
#include <stddef.h>

static double softplus(double x) {
    /* softplus(x) = log(1 + e^x); for x > 700, e^x overflows and the value is x
     * to within 1e-300. */
    if (x > 700.0) return x;
    return log1p(exp(x));
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* Causal depthwise conv1d, optional SiLU.
 * x, out: (Bsz, D, L); w: (D, W); bias: (D) or NULL. */
void oracle_causal_conv1d(const double* x, const double* w, const double* bias, double* out,
                          long Bsz, long D, long L, int W, int apply_silu) {
    for (long b = 0; b < Bsz; ++b)
        for (long d = 0; d < D; ++d) {
            const double* xr = x + (b * D + d) * L;
            double* orow = out + (b * D + d) * L;
            for (long t = 0; t < L; ++t) {
                double acc = bias ? bias[d] : 0.0;
                for (int k = 0; k < W; ++k) {
                    long s = t - (W - 1) + k;
                    if (s >= 0) acc += w[d * W + k] * xr[s];
                }
                orow[t] = apply_silu ? silu(acc) : acc;
            }
        }
}

/* Selective-scan forward (one direction).
 * u, delta, z, out: (Bsz, D, L); Bm, Cm: (Bsz, N, L), or (D, N) when bc_shared
 * (time-invariant: channel d reads row d at every position); A: (D, N);
 * Dv, delta_bias, conv_b: (D) or NULL; conv_w: (D, W) or NULL (NULL: no conv);
 * h0: (Bsz, D, N) initial state or NULL (zeros); final_state: (Bsz, D, N) or NULL.
 * conv_hist: (Bsz, D, W-1) inputs at positions -(W-1) .. -1, oldest first, or NULL
 * (zeros); forward scans only.
 * reverse = 0 walks t = 0..L-1, reverse = 1 walks t = L-1..0. */
void oracle_selective_scan(const double* u, const double* delta, const double* A,
                           const double* Bm, const double* Cm, const double* Dv,
                           const double* z, const double* delta_bias, int delta_softplus,
                           int reverse, const double* conv_w, const double* conv_b,
                           int conv_width, const double* h0, const double* conv_hist,
                           double* out, double* final_state, long Bsz, long D, long L, long N,
                           int bc_shared) {
    double h[1024];
    if (N > 1024) return;
    for (long b = 0; b < Bsz; ++b)
        for (long d = 0; d < D; ++d) {
            const double* ur = u + (b * D + d) * L;
            const double* dr = delta + (b * D + d) * L;
            const double* zr = z ? z + (b * D + d) * L : NULL;
            /* B[n] at position t is Br[n * bn + t * bt] */
            const double* Br = bc_shared ? Bm + d * N : Bm + b * N * L;
            const double* Cr = bc_shared ? Cm + d * N : Cm + b * N * L;
            const long bn = bc_shared ? 1 : L, bt = bc_shared ? 0 : 1;
            double* yr = out + (b * D + d) * L;
            for (long n = 0; n < N; ++n) h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;
            for (long i = 0; i < L; ++i) {
                long t = reverse ? L - 1 - i : i;
                /* input to the scan: raw u, or SiLU of the causal conv of x */
                double ut;
                if (conv_w) {
                    double acc = conv_b ? conv_b[d] : 0.0;
                    for (int k = 0; k < conv_width; ++k) {
                        /* forward: x[t-W+1+k]; reverse (flipped sequence): x[t+W-1-k] */
                        long s = reverse ? t + (conv_width - 1) - k : t - (conv_width - 1) + k;
                        if (s >= 0 && s < L)
                            acc += conv_w[d * conv_width + k] * ur[s];
                        else if (s < 0 && !reverse && conv_hist)  /* s in [-(W-1), -1] */
                            acc += conv_w[d * conv_width + k] *
                                   conv_hist[(b * D + d) * (conv_width - 1) + (conv_width - 1) + s];
                    }
                    ut = silu(acc);
                } else {
                    ut = ur[t];
                }
                double dl = dr[t] + (delta_bias ? delta_bias[d] : 0.0);
                if (delta_softplus) dl = softplus(dl);
                double y = 0.0;
                for (long n = 0; n < N; ++n) {
                    double dA = exp(dl * A[d * N + n]);
                    double dBu = dl * Br[n * bn + t * bt] * ut;
                    h[n] = dA * h[n] + dBu;
                    y += Cr[n * bn + t * bt] * h[n];
                }
                if (Dv) y += Dv[d] * ut;
                if (zr) y *= silu(zr[t]);
                yr[t] = y;
            }
            if (final_state)
                for (long n = 0; n < N; ++n) final_state[(b * D + d) * N + n] = h[n];
        }
}

/* Single-token state update (decode), in place on state and conv_state.
 * state: (Bsz, D, N); conv_state: (Bsz, D, W) newest last, or unused if conv_w is NULL;
 * x, dt, z, out: (Bsz, D); Bt, Ct: (Bsz, N); A: (D, N); Dv, dt_bias, conv_b: (D) or NULL. */
void oracle_state_update(double* state, double* conv_state, const double* x, const double* dt,
                         const double* A, const double* Bt, const double* Ct, const double* Dv,
                         const double* z, const double* dt_bias, int dt_softplus,
                         const double* conv_w, const double* conv_b, int conv_width,
                         double* out, long Bsz, long D, long N) {
    for (long b = 0; b < Bsz; ++b)
        for (long d = 0; d < D; ++d) {
            long bd = b * D + d;
            double xt = x[bd];
            double xc;
            if (conv_w) {
                double* cs = conv_state + bd * conv_width;
                for (int k = 0; k < conv_width - 1; ++k) cs[k] = cs[k + 1];
                cs[conv_width - 1] = xt;
                double acc = conv_b ? conv_b[d] : 0.0;
                for (int k = 0; k < conv_width; ++k) acc += conv_w[d * conv_width + k] * cs[k];
                xc = silu(acc);
            } else {
                xc = xt;
            }
            double dl = dt[bd] + (dt_bias ? dt_bias[d] : 0.0);
            if (dt_softplus) dl = softplus(dl);
            double y = 0.0;
            for (long n = 0; n < N; ++n) {
                double dA = exp(dl * A[d * N + n]);
                state[bd * N + n] = dA * state[bd * N + n] + dl * Bt[b * N + n] * xc;
                y += Ct[b * N + n] * state[bd * N + n];
            }
            if (Dv) y += Dv[d] * xc;
            if (z) y *= silu(z[bd]);
            out[bd] = y;
        }
}
