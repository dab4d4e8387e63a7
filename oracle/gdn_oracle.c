/*
 * Float64 CPU oracle for the frame-wise Gated DeltaNet (GDN) forward pass.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference leg may load or run this file's library.  It shares
 * no code, header or constant with the CUDA library: it is the plain
 * token-by-token recurrence, written out so that it can be checked by eye.
 *
 * What it computes (one independent recurrence per batch entry b and head h):
 *
 *   SANA-WM's attention is "frame-wise Gated DeltaNet + softmax every 4 blocks
 *   (hybrid linear)" (sglang cookbook SANA-WM page, section 1, architecture
 *   table), carrying long causal history as a bounded state (same page,
 *   introduction; d9249 blog, key-idea section).  The pages do not print the
 *   recurrence; it is fixed here as the gated delta rule
 *
 *       S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t
 *
 *   with q_t, k_t L2-normalised per token (x / sqrt(sum x^2 + eps)),
 *   beta_t = sigmoid(beta_logit[t]) per token, and one gate per latent frame,
 *   a_f = exp(-softplus(gate_logit[f])), applied at every token of frame
 *   f = t / frame_len ("frame-wise").  S is d_k x d_v; row index = key dim.
 *   The decay multiplies the old state and the erase term; the new write
 *   beta k v^T is not decayed; the output reads the state after the update.
 *   gate_mode 1 takes the other reading of "frame-wise": a_f applies once, at
 *   the first token of frame f (t % frame_len == 0), and a_t = 1 elsewhere.
 *
 *   The dense checkpoint's "bidirectional" GDN (sglang cookbook SANA-WM page,
 *   dense-bidirectional section: full bidirectional attention over the whole
 *   clip) is not defined on the pages either.  It is fixed here as the sum of two
 *   scans from a zero state: the forward one above, and the same rule run from
 *   the last token to the first,
 *
 *       R_t = a_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T,  R_T = 0,
 *       o_t = S_t^T q_t + R_t^T q_t,
 *
 *   every token keeping its own q, k, v, beta and the gate of its own frame
 *   (applied at every token).
 *
 * Layouts (row-major): q,k [B,T,H,d_k]; v [B,T,H,d_v]; gate [B,ceil(T/frame_len),H];
 * beta [B,T,H]; state [B,H,d_k,d_v]; out [B,T,H,d_v].  Inputs are float32 (the
 * exact values the GPU side receives, bf16 values widened exactly); every
 * intermediate and every output is float64.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double softplus(double x)
{
    /* log(1 + e^x) without overflow */
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

static double sigmoid(double x)
{
    return 1.0 / (1.0 + exp(-x));
}

static void l2_normalise(const float* x, double* y, int n, double eps)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) y[i] = (double)x[i] * inv;
}

/* One (b, h) chain over T tokens, first to last (reverse = 0) or last to first
 * (reverse = 1).  S (d_k*d_v doubles) holds the state on entry and on exit.
 * With accumulate = 1 the outputs are added to what `out` holds. */
static void run_chain(const float* q, const float* k, const float* v,
                      const float* gate, const float* beta, double* S, double* out,
                      int b, int h, int H, int T, int dk, int dv, int frame_len,
                      double eps, int gate_mode, int reverse, int accumulate, double* work)
{
    const int F = (T + frame_len - 1) / frame_len;
    double* qn = work;
    double* kn = qn + dk;
    double* kS = kn + dk;
    for (int n = 0; n < T; ++n) {
        const int t = reverse ? T - 1 - n : n;
        const size_t row = ((size_t)b * T + t) * H + h;
        const int f = t / frame_len;
        const int gated = (gate_mode == 0) || (t % frame_len == 0);
        const double a = gated ? exp(-softplus((double)gate[((size_t)b * F + f) * H + h])) : 1.0;
        const double bt = sigmoid((double)beta[row]);
        l2_normalise(q + row * dk, qn, dk, eps);
        l2_normalise(k + row * dk, kn, dk, eps);
        const float* vt = v + row * dv;

        /* kS = k^T S_{t-1} */
        for (int j = 0; j < dv; ++j) kS[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) kS[j] += kn[i] * S[(size_t)i * dv + j];

        /* S_t = a (S_{t-1} - beta k (k^T S_{t-1})) + beta k v^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double s = S[(size_t)i * dv + j];
                s = a * (s - bt * kn[i] * kS[j]) + bt * kn[i] * (double)vt[j];
                S[(size_t)i * dv + j] = s;
            }

        /* o_t = S_t^T q */
        double* o = out + row * dv;
        if (!accumulate)
            for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * qn[i];
    }
}

/*
 * Run all B*H chains.  state_in may be NULL (zero initial state); state_out may
 * be NULL (final state not returned).  n_threads <= 0 lets OpenMP choose.
 * gate_mode 0: the frame's gate at every token; 1: once, at the frame's first token.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int gdn_oracle_forward(const float* q, const float* k, const float* v,
                       const float* gate_logit, const float* beta_logit,
                       const float* state_in, double* state_out, double* out,
                       int B, int H, int T, int d_k, int d_v, int frame_len,
                       double eps, int n_threads, int gate_mode)
{
    if (!q || !k || !v || !gate_logit || !beta_logit || !out) return -1;
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1 || frame_len < 1) return -1;
    if (gate_mode != 0 && gate_mode != 1) return -1;
    const int chains = B * H;
    int failed = 0;
#ifdef _OPENMP
    if (n_threads <= 0) n_threads = omp_get_max_threads();
    if (n_threads > chains) n_threads = chains;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(|:failed)
#endif
    for (int c = 0; c < chains; ++c) {
        const int b = c / H, h = c % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)d_k * d_v);
        double* work = (double*)malloc(sizeof(double) * (size_t)(2 * d_k + d_v));
        if (!S || !work) {
            free(S); free(work);
            failed |= 1;
            continue;
        }
        const size_t soff = ((size_t)b * H + h) * (size_t)d_k * d_v;
        for (size_t i = 0; i < (size_t)d_k * d_v; ++i)
            S[i] = state_in ? (double)state_in[soff + i] : 0.0;
        run_chain(q, k, v, gate_logit, beta_logit, S, out, b, h, H, T, d_k, d_v,
                  frame_len, eps, gate_mode, 0, 0, work);
        if (state_out)
            memcpy(state_out + soff, S, sizeof(double) * (size_t)d_k * d_v);
        free(S);
        free(work);
    }
    return failed ? -1 : 0;
}

/* Same recurrence with a float64 initial state (for carrying the oracle's own
 * state across streaming blocks without rounding it to float32). */
int gdn_oracle_forward_f64state(const float* q, const float* k, const float* v,
                                const float* gate_logit, const float* beta_logit,
                                const double* state_in, double* state_out, double* out,
                                int B, int H, int T, int d_k, int d_v, int frame_len,
                                double eps, int n_threads, int gate_mode)
{
    if (!q || !k || !v || !gate_logit || !beta_logit || !out) return -1;
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1 || frame_len < 1) return -1;
    if (gate_mode != 0 && gate_mode != 1) return -1;
    const int chains = B * H;
    int failed = 0;
#ifdef _OPENMP
    if (n_threads <= 0) n_threads = omp_get_max_threads();
    if (n_threads > chains) n_threads = chains;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(|:failed)
#endif
    for (int c = 0; c < chains; ++c) {
        const int b = c / H, h = c % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)d_k * d_v);
        double* work = (double*)malloc(sizeof(double) * (size_t)(2 * d_k + d_v));
        if (!S || !work) {
            free(S); free(work);
            failed |= 1;
            continue;
        }
        const size_t soff = ((size_t)b * H + h) * (size_t)d_k * d_v;
        for (size_t i = 0; i < (size_t)d_k * d_v; ++i)
            S[i] = state_in ? state_in[soff + i] : 0.0;
        run_chain(q, k, v, gate_logit, beta_logit, S, out, b, h, H, T, d_k, d_v,
                  frame_len, eps, gate_mode, 0, 0, work);
        if (state_out)
            memcpy(state_out + soff, S, sizeof(double) * (size_t)d_k * d_v);
        free(S);
        free(work);
    }
    return failed ? -1 : 0;
}

/*
 * Bidirectional form: out = forward scan + backward scan, both from a zero state,
 * the gate of each token's own frame at every token.  No state in or out.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int gdn_oracle_bidirectional(const float* q, const float* k, const float* v,
                             const float* gate_logit, const float* beta_logit, double* out,
                             int B, int H, int T, int d_k, int d_v, int frame_len,
                             double eps, int n_threads)
{
    if (!q || !k || !v || !gate_logit || !beta_logit || !out) return -1;
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1 || frame_len < 1) return -1;
    const int chains = B * H;
    int failed = 0;
#ifdef _OPENMP
    if (n_threads <= 0) n_threads = omp_get_max_threads();
    if (n_threads > chains) n_threads = chains;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(|:failed)
#endif
    for (int c = 0; c < chains; ++c) {
        const int b = c / H, h = c % H;
        double* S = (double*)calloc((size_t)d_k * d_v, sizeof(double));
        double* work = (double*)malloc(sizeof(double) * (size_t)(2 * d_k + d_v));
        if (!S || !work) {
            free(S); free(work);
            failed |= 1;
            continue;
        }
        run_chain(q, k, v, gate_logit, beta_logit, S, out, b, h, H, T, d_k, d_v,
                  frame_len, eps, 0, 0, 0, work);
        memset(S, 0, sizeof(double) * (size_t)d_k * d_v);
        run_chain(q, k, v, gate_logit, beta_logit, S, out, b, h, H, T, d_k, d_v,
                  frame_len, eps, 0, 1, 1, work);
        free(S);
        free(work);
    }
    return failed ? -1 : 0;
}

int gdn_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
