/*
 * hyena_oracle.c -- plain, slow, fp64 CPU oracle for the gated Hyena cascade
 * operator.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg are the only callers.  The CUDA library never
 * links, loads or calls this file, and this file includes nothing from it.
 *
 * What is computed (per batch row b and channel c, every input widened
 * exactly to double):
 *
 *   v[t]    = x1[t] * x2[t]                               (pre-gate)
 *   conv[t] = (h_c * v)[t]                                 (causal, per channel)
 *   y[t]    = x3[t] * conv[t] + Dskip[c] * v[t]            (post-gate + skip)
 *
 * Sources for the pieces:
 *   - the three projections x1, x2, x3 and the gated filter output that
 *     feeds out_proj: evo2_flash README, hook table (rows
 *     "blocks.N.projections" and "blocks.N.filter");
 *   - the long filter is modal: an IIR parameterised by fp32 log-poles and
 *     residues, h_c[t] = sum_n R[c,n] exp(a[c,n] t): Evo2-7B-262K model card,
 *     §Architecture (training-dtype row) and §Implementation Notes
 *     (log_poles / residues kept in fp32; hcl evaluated as a modal-form IIR);
 *   - the explicit filters hcs (7 taps) and hcm (128 taps): Evo2-7B-262K
 *     model card, §Implementation Notes ("Block dispatch");
 *   - a carried per-channel modal state (hcl) and FIR window (hcm/hcs) so a
 *     long sequence can be fed in chunks, every position of every chunk being
 *     returned: Evo2-7B-262K model card §Implementation Notes ("Custom
 *     cache"), Evo1-1.5-7B-8K model card §Implementation Notes ("Cache
 *     subclass"), turboquant-evo2-int4 model card §"Important: a correctness
 *     fix comes with this" and §"Chunk size".
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): Dskip*v sits outside the x3 gate; the modal filter starts at t = 0
 * (h[0] = sum_n R_n) with no extra step size; modes are real; the modal
 * state is the R-free mode sum taken after the last token, layout
 * [B][D][N]; FIR taps are in lag order (taps[c][k] multiplies v[t-k]); the
 * FIR history holds the last K-1 values of v, layout [B][K-1][D], oldest
 * first.
 *
 * Two independent forms of the modal filter are provided so that each pins
 * the other: a direct O(L^2) convolution with the synthesised filter, and a
 * first-order recurrence per mode.
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* bf16 bit pattern -> double: a bf16 value is the upper half of an fp32. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int check_common(int B, int L, int D, int64_t ld_x, const void *x1,
                        const void *x2, const void *x3, const void *y)
{
    if (B < 1 || L < 0 || D < 1 || ld_x < D) return ORACLE_BAD_ARG;
    if (L > 0 && (!x1 || !x2 || !x3 || !y)) return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/*
 * Recurrence form.  For each mode n of channel c, with p = exp(a[c,n]):
 *     s_n[-1] = state_in[b,c,n]   (0 when state_in is NULL)
 *     s_n[t]  = p * s_n[t-1] + v[t]
 *     conv[t] = sum_n R[c,n] * s_n[t]
 * state_out[b,c,n] = s_n[L-1] (= state_in when L == 0).
 * y is dense [B][L][D] doubles.
 */
int hyena_oracle_modal_recurrence(int B, int L, int D, int N,
                                  const uint16_t *x1, const uint16_t *x2,
                                  const uint16_t *x3, int64_t ld_x,
                                  const float *log_poles, const float *residues,
                                  const float *Dskip, const double *state_in,
                                  double *y, double *state_out)
{
    /* The per-channel mode arrays below hold at most 256 modes. */
    if (check_common(B, L, D, ld_x, x1, x2, x3, y) || N < 1 || N > 256 || !log_poles ||
        !residues)
        return ORACLE_BAD_ARG;
    const long long BD = (long long)B * D;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bc = 0; bc < BD; ++bc) {
        const int b = (int)(bc / D), c = (int)(bc % D);
        double p[256], R[256], s[256];
        for (int n = 0; n < N; ++n) {
            p[n] = exp((double)log_poles[(size_t)c * N + n]);
            R[n] = (double)residues[(size_t)c * N + n];
            s[n] = state_in ? state_in[((size_t)b * D + c) * N + n] : 0.0;
        }
        const double dk = Dskip ? (double)Dskip[c] : 0.0;
        for (int t = 0; t < L; ++t) {
            const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
            const double v = bf16_bits_to_double(x1[ix]) * bf16_bits_to_double(x2[ix]);
            double conv = 0.0;
            for (int n = 0; n < N; ++n) {
                s[n] = p[n] * s[n] + v;
                conv += R[n] * s[n];
            }
            y[((size_t)b * L + t) * D + c] = bf16_bits_to_double(x3[ix]) * conv + dk * v;
        }
        if (state_out)
            for (int n = 0; n < N; ++n) state_out[((size_t)b * D + c) * N + n] = s[n];
    }
    return ORACLE_OK;
}

/*
 * Direct form.  The filter is synthesised from the modal parameters,
 *     h[k] = sum_n R[c,n] * exp(a[c,n] * k),   k = 0 .. L-1,
 * and applied as a plain causal convolution; a carried state enters through
 * its own closed-form decay,
 *     conv[t] = sum_{s<=t} h[t-s] v[s] + sum_n R[c,n] exp(a[c,n] (t+1)) S_in[n].
 * state_out[n] = exp(a L) S_in[n] + sum_{s<L} exp(a (L-1-s)) v[s].
 * O(L^2) per channel: use it on small L only.
 */
int hyena_oracle_modal_direct(int B, int L, int D, int N,
                              const uint16_t *x1, const uint16_t *x2,
                              const uint16_t *x3, int64_t ld_x,
                              const float *log_poles, const float *residues,
                              const float *Dskip, const double *state_in,
                              double *y, double *state_out,
                              double *scratch /* 2*L doubles per thread slot */,
                              int scratch_slots)
{
    if (check_common(B, L, D, ld_x, x1, x2, x3, y) || N < 1 || !log_poles ||
        !residues || (L > 0 && (!scratch || scratch_slots < 1)))
        return ORACLE_BAD_ARG;
    const long long BD = (long long)B * D;
    /* One thread per scratch slot so that slots are never shared. */
#pragma omp parallel for schedule(static, 1) num_threads(scratch_slots)
    for (int slot = 0; slot < scratch_slots; ++slot) {
        double *h = scratch + (size_t)slot * 2 * (size_t)L;
        double *v = h + L;
        for (long long bc = slot; bc < BD; bc += scratch_slots) {
            const int b = (int)(bc / D), c = (int)(bc % D);
            const float *ac = log_poles + (size_t)c * N;
            const float *rc = residues + (size_t)c * N;
            for (int k = 0; k < L; ++k) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) acc += (double)rc[n] * exp((double)ac[n] * k);
                h[k] = acc;
            }
            for (int t = 0; t < L; ++t) {
                const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
                v[t] = bf16_bits_to_double(x1[ix]) * bf16_bits_to_double(x2[ix]);
            }
            const double dk = Dskip ? (double)Dskip[c] : 0.0;
            for (int t = 0; t < L; ++t) {
                double conv = 0.0;
                for (int s = 0; s <= t; ++s) conv += h[t - s] * v[s];
                if (state_in)
                    for (int n = 0; n < N; ++n)
                        conv += (double)rc[n] * exp((double)ac[n] * (t + 1)) *
                                state_in[((size_t)b * D + c) * N + n];
                const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
                y[((size_t)b * L + t) * D + c] = bf16_bits_to_double(x3[ix]) * conv + dk * v[t];
            }
            if (state_out) {
                for (int n = 0; n < N; ++n) {
                    double acc = state_in ? exp((double)ac[n] * L) *
                                                state_in[((size_t)b * D + c) * N + n]
                                          : 0.0;
                    for (int s = 0; s < L; ++s) acc += exp((double)ac[n] * (L - 1 - s)) * v[s];
                    state_out[((size_t)b * D + c) * N + n] = acc;
                }
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Complex modes (Evo1-1.5-7B-8K model card, §Architecture: modal-form
 * "poles" / "residues" kept in fp32, Hyena state size 8).  Each mode n of
 * channel c has a complex pole p and a complex residue R, given as fp32
 * (real, imaginary) pairs, layout [D][N][2]; the filter is the real part of
 * the modal sum,
 *     h[k] = Re sum_n R[c,n] p[c,n]^k,   k >= 0,
 * so a conjugate pair (p, R), (conj p, conj R) is one mode with residue 2R.
 * The state is the complex R-free mode sum after the last token, layout
 * [B][D][N][2].
 *
 * Recurrence form, in complex arithmetic:
 *     s_n[-1] = state_in[b,c,n]  (0 when state_in is NULL)
 *     s_n[t]  = p s_n[t-1] + v[t]
 *     conv[t] = Re sum_n R_n s_n[t]
 */
int hyena_oracle_cmodal_recurrence(int B, int L, int D, int N,
                                   const uint16_t *x1, const uint16_t *x2,
                                   const uint16_t *x3, int64_t ld_x,
                                   const float *poles, const float *residues,
                                   const float *Dskip, const double *state_in,
                                   double *y, double *state_out)
{
    if (check_common(B, L, D, ld_x, x1, x2, x3, y) || N < 1 || N > 256 || !poles ||
        !residues)
        return ORACLE_BAD_ARG;
    const long long BD = (long long)B * D;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bc = 0; bc < BD; ++bc) {
        const int b = (int)(bc / D), c = (int)(bc % D);
        double complex p[256], R[256], s[256];
        for (int n = 0; n < N; ++n) {
            const size_t k = ((size_t)c * N + n) * 2;
            p[n] = (double)poles[k] + I * (double)poles[k + 1];
            R[n] = (double)residues[k] + I * (double)residues[k + 1];
            const size_t q = (((size_t)b * D + c) * N + n) * 2;
            s[n] = state_in ? state_in[q] + I * state_in[q + 1] : 0.0;
        }
        const double dk = Dskip ? (double)Dskip[c] : 0.0;
        for (int t = 0; t < L; ++t) {
            const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
            const double v = bf16_bits_to_double(x1[ix]) * bf16_bits_to_double(x2[ix]);
            double complex acc = 0.0;
            for (int n = 0; n < N; ++n) {
                s[n] = p[n] * s[n] + v;
                acc += R[n] * s[n];
            }
            y[((size_t)b * L + t) * D + c] = bf16_bits_to_double(x3[ix]) * creal(acc) + dk * v;
        }
        if (state_out)
            for (int n = 0; n < N; ++n) {
                const size_t q = (((size_t)b * D + c) * N + n) * 2;
                state_out[q] = creal(s[n]);
                state_out[q + 1] = cimag(s[n]);
            }
    }
    return ORACLE_OK;
}

/*
 * Direct form of the complex modes, from the polar form of each term (no
 * complex arithmetic): with p = rho e^{i theta}, R = m e^{i phi},
 *     Re(R p^k) = m rho^k cos(k theta + phi),
 *     h[k] = sum_n m_n rho_n^k cos(k theta_n + phi_n),
 * applied as a plain causal convolution; a carried state S = sigma e^{i psi}
 * adds Re(R p^(t+1) S) = m sigma rho^(t+1) cos((t+1) theta + phi + psi), and
 *     state_out = p^L S + sum_{s<L} p^(L-1-s) v[s]
 * (real and imaginary parts from rho^k (cos, sin)(k theta)).  O(L^2).
 */
int hyena_oracle_cmodal_direct(int B, int L, int D, int N,
                               const uint16_t *x1, const uint16_t *x2,
                               const uint16_t *x3, int64_t ld_x,
                               const float *poles, const float *residues,
                               const float *Dskip, const double *state_in,
                               double *y, double *state_out,
                               double *scratch /* 2*L doubles per thread slot */,
                               int scratch_slots)
{
    if (check_common(B, L, D, ld_x, x1, x2, x3, y) || N < 1 || !poles || !residues ||
        (L > 0 && (!scratch || scratch_slots < 1)))
        return ORACLE_BAD_ARG;
    const long long BD = (long long)B * D;
#pragma omp parallel for schedule(static, 1) num_threads(scratch_slots)
    for (int slot = 0; slot < scratch_slots; ++slot) {
        double *h = scratch + (size_t)slot * 2 * (size_t)L;
        double *v = h + L;
        for (long long bc = slot; bc < BD; bc += scratch_slots) {
            const int b = (int)(bc / D), c = (int)(bc % D);
            const float *pc = poles + (size_t)c * N * 2;
            const float *rc = residues + (size_t)c * N * 2;
            for (int k = 0; k < L; ++k) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    const double rho = hypot(pc[2 * n], pc[2 * n + 1]);
                    const double theta = atan2(pc[2 * n + 1], pc[2 * n]);
                    const double m = hypot(rc[2 * n], rc[2 * n + 1]);
                    const double phi = atan2(rc[2 * n + 1], rc[2 * n]);
                    acc += m * pow(rho, k) * cos(k * theta + phi);
                }
                h[k] = acc;
            }
            for (int t = 0; t < L; ++t) {
                const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
                v[t] = bf16_bits_to_double(x1[ix]) * bf16_bits_to_double(x2[ix]);
            }
            const double dk = Dskip ? (double)Dskip[c] : 0.0;
            for (int t = 0; t < L; ++t) {
                double conv = 0.0;
                for (int s = 0; s <= t; ++s) conv += h[t - s] * v[s];
                if (state_in)
                    for (int n = 0; n < N; ++n) {
                        const size_t q = (((size_t)b * D + c) * N + n) * 2;
                        const double rho = hypot(pc[2 * n], pc[2 * n + 1]);
                        const double theta = atan2(pc[2 * n + 1], pc[2 * n]);
                        const double m = hypot(rc[2 * n], rc[2 * n + 1]);
                        const double phi = atan2(rc[2 * n + 1], rc[2 * n]);
                        const double sigma = hypot(state_in[q], state_in[q + 1]);
                        const double psi = atan2(state_in[q + 1], state_in[q]);
                        conv += m * sigma * pow(rho, t + 1) * cos((t + 1) * theta + phi + psi);
                    }
                const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
                y[((size_t)b * L + t) * D + c] = bf16_bits_to_double(x3[ix]) * conv + dk * v[t];
            }
            if (state_out) {
                for (int n = 0; n < N; ++n) {
                    const size_t q = (((size_t)b * D + c) * N + n) * 2;
                    const double rho = hypot(pc[2 * n], pc[2 * n + 1]);
                    const double theta = atan2(pc[2 * n + 1], pc[2 * n]);
                    double re = 0.0, im = 0.0;
                    if (state_in) {
                        const double sigma = hypot(state_in[q], state_in[q + 1]);
                        const double psi = atan2(state_in[q + 1], state_in[q]);
                        re = sigma * pow(rho, L) * cos(L * theta + psi);
                        im = sigma * pow(rho, L) * sin(L * theta + psi);
                    }
                    for (int s = 0; s < L; ++s) {
                        const int k = L - 1 - s;
                        re += pow(rho, k) * cos(k * theta) * v[s];
                        im += pow(rho, k) * sin(k * theta) * v[s];
                    }
                    state_out[q] = re;
                    state_out[q + 1] = im;
                }
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Explicit causal FIR (hcs / hcm).  taps are bf16 bits, layout [D][K], lag
 * order.  For t-k < 0 the value comes from hist_in[b][K-1+(t-k)][c] (the
 * last K-1 values of v before this call, oldest first), or is 0 when
 * hist_in is NULL.
 *     conv[t] = sum_{k<K} taps[c,k] * v[t-k]
 *     y[t]    = x3[t] * conv[t] + Dskip[c] * v[t]
 * hist_out[b][j][c] = v[L-(K-1)+j] (history values when that index is < 0).
 */
int hyena_oracle_fir(int B, int L, int D, int K,
                     const uint16_t *x1, const uint16_t *x2, const uint16_t *x3,
                     int64_t ld_x, const uint16_t *taps, const float *Dskip,
                     const double *hist_in, double *y, double *hist_out)
{
    /* The history gather below holds at most 128 values (K <= 129). */
    if (check_common(B, L, D, ld_x, x1, x2, x3, y) || K < 1 || !taps ||
        (hist_out && K - 1 > 128))
        return ORACLE_BAD_ARG;
    const long long BD = (long long)B * D;
    const int H = K - 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bc = 0; bc < BD; ++bc) {
        const int b = (int)(bc / D), c = (int)(bc % D);
        const double dk = Dskip ? (double)Dskip[c] : 0.0;
        /* v at index t (t may be negative, down to -H). */
#define V_AT(tt)                                                                   \
    ((tt) >= 0 ? bf16_bits_to_double(x1[((size_t)b * L + (tt)) * (size_t)ld_x + c]) * \
                     bf16_bits_to_double(x2[((size_t)b * L + (tt)) * (size_t)ld_x + c]) \
               : (hist_in ? hist_in[((size_t)b * H + (size_t)(H + (tt))) * D + c] : 0.0))
        for (int t = 0; t < L; ++t) {
            double conv = 0.0;
            for (int k = 0; k < K; ++k) {
                const int s = t - k;
                if (s < -H) break;
                conv += bf16_bits_to_double(taps[(size_t)c * K + k]) * V_AT(s);
            }
            const size_t ix = ((size_t)b * L + t) * (size_t)ld_x + c;
            y[((size_t)b * L + t) * D + c] = bf16_bits_to_double(x3[ix]) * conv + dk * V_AT(t);
        }
        if (hist_out && H > 0) {
            /* Gather first, then write, so hist_out may alias hist_in. */
            double tmp[128];
            for (int j = 0; j < H; ++j) tmp[j] = V_AT(L - H + j);
            for (int j = 0; j < H; ++j) hist_out[((size_t)b * H + j) * D + c] = tmp[j];
        }
#undef V_AT
    }
    return ORACLE_OK;
}
