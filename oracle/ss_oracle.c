/*
 * ss_oracle.c -- plain float64 CPU reference for the Mamba-1 selective scan (S6)
 * forward pass and its single-token decode state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library under
 * selective_state_space_18_b200/csrc, and it never calls it.
 *
 * What it computes (nnterp docs, "selective_scan" component, SelectiveScan class
 * description; TransformerLens "ssm_mixer" module, compute_ssm_state):
 *
 *   dt_t   = softplus(dt_raw[b,c,t] + dt_bias[c])      (or no softplus when disabled)
 *   h_t[n] = exp(dt_t * A[c,n]) * h_{t-1}[n] + dt_t * B[b,n,t] * x[b,c,t]
 *   y_t    = sum_n C[b,n,t] * h_t[n] + D[c] * x[b,c,t]
 *   out_t  = y_t * silu(z[b,c,t])                        (only when z is given)
 *
 * with h_{-1} = h0[b,c,:] (zeros when h0 is NULL), and h_last = h_{L-1}.
 * Enforced boundary reset (the "s6_reset" blog draft, "Enforced Boundary Resetting";
 * the packed-sequence workload fixes the flag on each document's FIRST token):
 * at a flagged token the state is zeroed before that token's update, so
 * h_t = dt_t * B_t * x_t there.
 *
 * Layouts are channel-first as the nnterp page states for the kernel's tensors:
 * x, dt, z, y [batch, channels, seq]; B, C [batch, state_dim, seq];
 * A [channels, state_dim]; D, dt_bias [channels]; reset [batch, seq];
 * h0, h_last, decode state [batch, channels, state_dim].  Every array is
 * contiguous float64 except reset (uint8).
 *
 * The token loop can also return the state after every token (h_all) and the step
 * size of every token (betas [batch, channels, seq]: dt_t itself, which the nnterp
 * page exposes per token and channel; its log decay dt_t * A[c,n] is that times A).
 *
 * Two independent orderings of the same recurrence are provided:
 *   ss_oracle_scan      -- the token loop, in sequence order;
 *   ss_oracle_tree_scan -- an inclusive associative scan (recursive doubling) of
 *                          the affine maps h -> a*h + u with an explicit reset
 *                          flag ("s6_reset", "Associative Boundary Resetting").
 * ss_oracle_segment folds one segment's maps with the same operator into a single
 * composite (decay, end state), the unit a sequence cut into segments is joined by.
 * The test suite pins each against closed forms and against the other.
 *
 * Parallelism: OpenMP over independent (batch, channel) rows only, so that the
 * benchmark's CPU-baseline timing can use the host's cores.  Nothing else is
 * blocked, fused or reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_ERR_NULL = 1, ORC_ERR_SHAPE = 2, ORC_ERR_NOMEM = 3 };

/* softplus(r) = log(1 + e^r), evaluated without overflow for large r. */
static double orc_softplus(double r)
{
    if (r > 0.0)
        return r + log1p(exp(-r));
    return log1p(exp(r));
}

/* silu(v) = v * sigmoid(v) = v / (1 + e^{-v}). */
static double orc_silu(double v)
{
    return v / (1.0 + exp(-v));
}

/* Step size of token t of row (b,c): bias added before the softplus, per channel
 * (nnterp selective_scan: dt = softplus(dt_proj(x) + dt_bias)). */
static double orc_step(const double *dt, const double *dt_bias, int dt_softplus,
                       int64_t idx, int64_t c)
{
    double r = dt[idx] + (dt_bias ? dt_bias[c] : 0.0);
    return dt_softplus ? orc_softplus(r) : r;
}

int ss_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Token loop.  h_all (nullable) receives the state after every token,
 * [batch, channels, seq, state_dim] -- the "state after each token" the nnterp
 * page reads from the token loop.
 */
int ss_oracle_scan(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                   const double *x, const double *dt, const double *A, const double *B,
                   const double *C, const double *D, const double *z, const double *dt_bias,
                   const uint8_t *reset, const double *h0, int dt_softplus,
                   double *y, double *h_last, double *h_all, double *betas, int nthreads)
{
    if (!x || !dt || !A || !B || !C || !y)
        return ORC_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0 || seq <= 0)
        return ORC_ERR_SHAPE;
    if (nthreads <= 0)
        nthreads = 1;
    const int64_t rows = batch * channels;
    int status = ORC_OK;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / channels;
        const int64_t c = row % channels;
        double *h = (double *)malloc((size_t)state_dim * sizeof(double));
        if (!h) {
#pragma omp atomic write
            status = ORC_ERR_NOMEM;
            continue;
        }
        for (int64_t n = 0; n < state_dim; ++n)
            h[n] = h0 ? h0[row * state_dim + n] : 0.0;

        for (int64_t t = 0; t < seq; ++t) {
            const int64_t idx = row * seq + t;
            const double d = orc_step(dt, dt_bias, dt_softplus, idx, c);
            if (betas) /* the step size of this token (nnterp selective_scan, "betas") */
                betas[idx] = d;
            const double xv = x[idx];
            if (reset && reset[b * seq + t]) {
                /* state zeroed before this token's update */
                for (int64_t n = 0; n < state_dim; ++n)
                    h[n] = 0.0;
            }
            double acc = 0.0;
            for (int64_t n = 0; n < state_dim; ++n) {
                const double Bn = B[(b * state_dim + n) * seq + t];
                const double Cn = C[(b * state_dim + n) * seq + t];
                h[n] = exp(d * A[c * state_dim + n]) * h[n] + d * Bn * xv;
                acc += Cn * h[n];
            }
            double yv = acc + (D ? D[c] : 0.0) * xv;
            if (z)
                yv *= orc_silu(z[idx]);
            y[idx] = yv;
            if (h_all)
                for (int64_t n = 0; n < state_dim; ++n)
                    h_all[(row * seq + t) * state_dim + n] = h[n];
        }
        if (h_last)
            for (int64_t n = 0; n < state_dim; ++n)
                h_last[row * state_dim + n] = h[n];
        free(h);
    }
    return status;
}

/*
 * Element of the associative scan: the affine map h -> (r ? u : a*h + u).
 * Composition "left then right" ("s6_reset", Associative Boundary Resetting:
 * the binary operator (A_i, Bx_i) o (A_j, Bx_j) = (A_i A_j, A_j Bx_i + Bx_j),
 * extended by a flag that records whether the segment contains a reset; when
 * it does, the incoming state is discarded so the decay no longer matters).
 */
typedef struct {
    double a, u;
    int r;
} orc_elem;

static orc_elem orc_combine(orc_elem left, orc_elem right)
{
    orc_elem out;
    if (right.r) {
        out = right;
    } else if (left.r) {
        out.a = 1.0; /* unused: the segment discards its input state */
        out.u = right.a * left.u + right.u;
        out.r = 1;
    } else {
        out.a = left.a * right.a;
        out.u = right.a * left.u + right.u;
        out.r = 0;
    }
    return out;
}

/*
 * Associative-scan ordering of the same recurrence: for every (b, c, n) the
 * sequence of maps is reduced to inclusive prefixes by recursive doubling
 * (Hillis-Steele), then h_t = prefix_t applied to h0.
 */
int ss_oracle_tree_scan(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                        const double *x, const double *dt, const double *A, const double *B,
                        const double *C, const double *D, const double *z,
                        const double *dt_bias, const uint8_t *reset, const double *h0,
                        int dt_softplus, double *y, double *h_last, int nthreads)
{
    if (!x || !dt || !A || !B || !C || !y)
        return ORC_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0 || seq <= 0)
        return ORC_ERR_SHAPE;
    if (nthreads <= 0)
        nthreads = 1;
    const int64_t rows = batch * channels;
    int status = ORC_OK;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / channels;
        const int64_t c = row % channels;
        orc_elem *e = (orc_elem *)malloc((size_t)seq * sizeof(orc_elem));
        double *hs = (double *)malloc((size_t)(seq * state_dim) * sizeof(double));
        double *steps = (double *)malloc((size_t)seq * sizeof(double));
        if (!e || !hs || !steps) {
            free(e);
            free(hs);
            free(steps);
#pragma omp atomic write
            status = ORC_ERR_NOMEM;
            continue;
        }
        for (int64_t t = 0; t < seq; ++t)
            steps[t] = orc_step(dt, dt_bias, dt_softplus, row * seq + t, c);

        for (int64_t n = 0; n < state_dim; ++n) {
            const double An = A[c * state_dim + n];
            for (int64_t t = 0; t < seq; ++t) {
                e[t].a = exp(steps[t] * An);
                e[t].u = steps[t] * B[(b * state_dim + n) * seq + t] * x[row * seq + t];
                e[t].r = reset ? (reset[b * seq + t] != 0) : 0;
            }
            for (int64_t d = 1; d < seq; d *= 2) {
                /* descending t: element t - d still holds the previous round's value */
                for (int64_t t = seq - 1; t >= d; --t)
                    e[t] = orc_combine(e[t - d], e[t]);
            }
            const double hin = h0 ? h0[row * state_dim + n] : 0.0;
            for (int64_t t = 0; t < seq; ++t)
                hs[t * state_dim + n] = e[t].r ? e[t].u : e[t].a * hin + e[t].u;
        }

        for (int64_t t = 0; t < seq; ++t) {
            const int64_t idx = row * seq + t;
            double acc = 0.0;
            for (int64_t n = 0; n < state_dim; ++n)
                acc += C[(b * state_dim + n) * seq + t] * hs[t * state_dim + n];
            double yv = acc + (D ? D[c] : 0.0) * x[idx];
            if (z)
                yv *= orc_silu(z[idx]);
            y[idx] = yv;
        }
        if (h_last)
            for (int64_t n = 0; n < state_dim; ++n)
                h_last[row * state_dim + n] = hs[(seq - 1) * state_dim + n];
        free(e);
        free(hs);
        free(steps);
    }
    return status;
}

/*
 * Composite of one segment of the sequence (the affine map a whole segment applies
 * to the state that enters it): the segment's elements h -> (r ? u : a*h + u) folded
 * left to right with the operator above ("s6_reset", Associative Boundary
 * Resetting).  The result, per (b, c, n), is written as the map h -> decay*h + state:
 *
 *   decay[b,c,n] = product over the segment of exp(dt_t * A[c,n]), or 0 when the
 *                  segment holds a reset (the entering state is then discarded);
 *   state[b,c,n] = the segment's end state when it is entered with h = 0.
 *
 * Applying the composites of consecutive segments in order to h0 gives the state
 * at the end of their concatenation, which is what lets a sequence be cut into
 * segments that are scanned independently and then joined.
 */
int ss_oracle_segment(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                      const double *x, const double *dt, const double *A, const double *B,
                      const double *dt_bias, const uint8_t *reset, int dt_softplus,
                      double *decay, double *state, int nthreads)
{
    if (!x || !dt || !A || !B || !decay || !state)
        return ORC_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0 || seq <= 0)
        return ORC_ERR_SHAPE;
    if (nthreads <= 0)
        nthreads = 1;
    const int64_t rows = batch * channels;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / channels;
        const int64_t c = row % channels;
        for (int64_t n = 0; n < state_dim; ++n) {
            orc_elem acc = {1.0, 0.0, 0}; /* the identity map */
            for (int64_t t = 0; t < seq; ++t) {
                const double d = orc_step(dt, dt_bias, dt_softplus, row * seq + t, c);
                orc_elem e;
                e.a = exp(d * A[c * state_dim + n]);
                e.u = d * B[(b * state_dim + n) * seq + t] * x[row * seq + t];
                e.r = reset ? (reset[b * seq + t] != 0) : 0;
                acc = orc_combine(acc, e);
            }
            decay[row * state_dim + n] = acc.r ? 0.0 : acc.a;
            state[row * state_dim + n] = acc.u;
        }
    }
    return ORC_OK;
}

/*
 * Single-token decode update (nnterp selective_scan: mamba_selective_state_update
 * on a decode step; the state [batch, channels, state_dim] is updated in place and
 * is what the next step starts from).  x, dt, z, y are [batch, channels];
 * B, C are [batch, state_dim].  No reset on this path.
 */
int ss_oracle_update(int64_t batch, int64_t channels, int64_t state_dim, double *state,
                     const double *x, const double *dt, const double *A, const double *B,
                     const double *C, const double *D, const double *z,
                     const double *dt_bias, int dt_softplus, double *y, int nthreads)
{
    if (!state || !x || !dt || !A || !B || !C || !y)
        return ORC_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0)
        return ORC_ERR_SHAPE;
    if (nthreads <= 0)
        nthreads = 1;
    const int64_t rows = batch * channels;

#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / channels;
        const int64_t c = row % channels;
        const double d = orc_step(dt, dt_bias, dt_softplus, row, c);
        const double xv = x[row];
        double *h = state + row * state_dim;
        double acc = 0.0;
        for (int64_t n = 0; n < state_dim; ++n) {
            h[n] = exp(d * A[c * state_dim + n]) * h[n] + d * B[b * state_dim + n] * xv;
            acc += C[b * state_dim + n] * h[n];
        }
        double yv = acc + (D ? D[c] : 0.0) * xv;
        if (z)
            yv *= orc_silu(z[row]);
        y[row] = yv;
    }
    return ORC_OK;
}

/*
 * Mamba-2 gated state scan ("Mamba 2 Gated State Scan" exercise page): per batch item
 * b, with S_{-1} = h0[b] (zeros when h0 is NULL),
 *
 *   S_t = gamma[b,t] * S_{t-1} + k[b,t,:] v[b,t,:]^T      (Dk x Dv)
 *   y[b,t,:] = q[b,t,:]^T S_t                             (the updated state is read)
 *
 * and final_state[b] = S_{seq-1}.  Layouts: q, k [batch, seq, dk]; v, y
 * [batch, seq, dv]; gamma [batch, seq]; h0, final_state [batch, dk, dv].  The token
 * loop in sequence order, every sum in index order; OpenMP over batch items only.
 */
int ss_oracle_gated_scan(int64_t batch, int64_t seq, int64_t dk, int64_t dv, const double *q,
                         const double *k, const double *v, const double *gamma, const double *h0,
                         double *y, double *final_state, int nthreads)
{
    if (!q || !k || !v || !gamma || !y || !final_state)
        return ORC_ERR_NULL;
    if (batch <= 0 || seq <= 0 || dk <= 0 || dv <= 0)
        return ORC_ERR_SHAPE;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
#endif
    for (int64_t b = 0; b < batch; ++b) {
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
        if (!S) {
            failed = 1;
            continue;
        }
        for (int64_t i = 0; i < dk * dv; ++i)
            S[i] = h0 ? h0[b * dk * dv + i] : 0.0;
        for (int64_t t = 0; t < seq; ++t) {
            const double g = gamma[b * seq + t];
            const double *kt = k + (b * seq + t) * dk, *qt = q + (b * seq + t) * dk;
            const double *vt = v + (b * seq + t) * dv;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j)
                    S[i * dv + j] = g * S[i * dv + j] + kt[i] * vt[j];
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < dk; ++i)
                    acc += qt[i] * S[i * dv + j];
                y[(b * seq + t) * dv + j] = acc;
            }
        }
        for (int64_t i = 0; i < dk * dv; ++i)
            final_state[b * dk * dv + i] = S[i];
        free(S);
    }
    (void)nthreads;
    return failed ? ORC_ERR_NOMEM : ORC_OK;
}

/*
 * Causal depthwise convolution followed by SiLU, the step that produces the scan's x
 * (TransformerLens docs, ssm_mixer: "x is the post-conv SiLU input", SiLU(conv1d
 * output)).  Per row (b, c) with K taps w[c, 0..K-1] and bias cb[c]:
 *
 *   x[b,c,t] = silu( cb[c] + sum_{k<K} w[c,k] * u[b,c,t-K+1+k] )
 *
 * where u at t < 0 is taken from state_in[b,c,K-1+t] (the K-1 inputs that preceded
 * this call, oldest first; zeros when state_in is NULL).  state_out[b,c,:] receives
 * the last K-1 inputs of the concatenation state_in ++ u (oldest first).  Layouts:
 * u, x [batch, channels, seq]; w [channels, K]; cb [channels]; state_in, state_out
 * [batch, channels, K-1].  The sum runs over k in index order.
 */
int ss_oracle_conv_silu(int64_t batch, int64_t channels, int64_t seq, int64_t K, const double *u,
                        const double *w, const double *cb, const double *state_in, double *x,
                        double *state_out, int nthreads)
{
    if (!u || !w || !x)
        return ORC_ERR_NULL;
    if (batch <= 0 || channels <= 0 || seq <= 0 || K <= 0)
        return ORC_ERR_SHAPE;
    const int64_t rows = batch * channels, H = K - 1;
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(static)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t c = r % channels;
        const double *ur = u + r * seq;
        /* input at position t of the concatenation: t < 0 reads the state */
#define ORC_IN(t) ((t) >= 0 ? ur[(t)] : (state_in ? state_in[r * H + H + (t)] : 0.0))
        for (int64_t t = 0; t < seq; ++t) {
            double acc = cb ? cb[c] : 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += w[c * K + k] * ORC_IN(t - K + 1 + k);
            x[r * seq + t] = orc_silu(acc);
        }
        if (state_out)
            for (int64_t j = 0; j < H; ++j)
                state_out[r * H + j] = ORC_IN(seq - H + j);
#undef ORC_IN
    }
    (void)nthreads;
    return ORC_OK;
}
