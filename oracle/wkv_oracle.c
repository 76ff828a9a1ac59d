/*
 * CPU oracle for the RWKV WKV operator: the float64 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. The product path (the CUDA library) never
 * links, loads or calls it, and this file shares no code with it.
 *
 * What it computes. "Linear attention without writing a CUDA kernel" (page 1),
 * section "The recurrence", defines wkv_t as a weighted mean of the values: the
 * current token enters with weight e^{u+k_t}, an earlier token i with weight
 * e^{-(t-1-i)w + k_i}. The same section gives the constant-cost form: a carried
 * state (numerator, denominator, max_exponent), where the max exponent is
 * subtracted before every exponential, as in a stable softmax. One step:
 *
 *   output  : e = max(m, k+u);  a = exp(m-e);  b = exp(k+u-e);
 *             out = (a*num + b*v) / (a*den + b)
 *   advance : e' = max(m-w, k); a' = exp(m-w-e'); b' = exp(k-e');
 *             num' = a'*num + b'*v;  den' = a'*den + b';  m' = e'
 *
 * This file runs that step in float64, in the order given there, one channel
 * at a time (channels are independent: w and u are per channel). The empty
 * state is (0, 0, -inf): the page leaves it open, and -inf makes exp(m-e) = 0,
 * so the first output is v_1 and the first state is (v_1, 1, k_1).
 *
 * Inputs are fp32 or bf16 codes (widened to float64 exactly); everything after
 * that is float64 with IEEE semantics (build without fast-math).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* element type codes of the k, v inputs */
#define ORACLE_F32 0
#define ORACLE_BF16 1

static double widen(const void *p, int dtype, size_t i)
{
    if (dtype == ORACLE_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* One token for one channel: writes the output and advances (num, den, m). */
static double wkv_token(double kt, double vt, double w, double u,
                        double *num, double *den, double *m)
{
    double kb = kt + u;                 /* exponent of the current token (with bonus) */
    double top = fmax(*m, kb);          /* the larger exponent is subtracted from both */
    double past = exp(*m - top);
    double cur = exp(kb - top);
    double out = (past * *num + cur * vt) / (past * *den + cur);

    double decayed = *m - w;            /* the carried exponent after one step of decay */
    double top2 = fmax(decayed, kt);
    double keep = exp(decayed - top2);
    double add = exp(kt - top2);
    *num = keep * *num + add * vt;
    *den = keep * *den + add;
    *m = top2;
    return out;
}

/*
 * Sequence forward over k, v laid out [B, T, C] (C fastest).
 *
 * state_in: three [B, C] float64 arrays (num, den, max_e), or all NULL for the
 * empty state. out: [B, T, C] float64. state_out: three [B, C] float64 arrays
 * (may be NULL). nthreads <= 0 uses the OpenMP default.
 */
void wkv_oracle_forward(int64_t B, int64_t T, int64_t C,
                        const void *k, const void *v, int kv_dtype,
                        const float *w, const float *u,
                        const double *num_in, const double *den_in, const double *max_in,
                        double *out,
                        double *num_out, double *den_out, double *max_out,
                        int nthreads)
{
    const int64_t CB = 16;                       /* channels per work item */
    const int64_t nblk = (C + CB - 1) / CB;
    const int64_t items = B * nblk;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        const int64_t b = it / nblk;
        const int64_t c0 = (it % nblk) * CB;
        const int64_t nc = (C - c0) < CB ? (C - c0) : CB;
        double num[16], den[16], m[16], wc[16], uc[16];
        for (int64_t j = 0; j < nc; ++j) {
            const int64_t s = b * C + c0 + j;
            wc[j] = (double)w[c0 + j];
            uc[j] = (double)u[c0 + j];
            if (num_in) {
                num[j] = num_in[s];
                den[j] = den_in[s];
                m[j] = max_in[s];
            } else {
                num[j] = 0.0;
                den[j] = 0.0;
                m[j] = -INFINITY;
            }
        }
        for (int64_t t = 0; t < T; ++t) {
            const size_t row = ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c0;
            for (int64_t j = 0; j < nc; ++j) {
                const double kt = widen(k, kv_dtype, row + (size_t)j);
                const double vt = widen(v, kv_dtype, row + (size_t)j);
                out[row + (size_t)j] = wkv_token(kt, vt, wc[j], uc[j], &num[j], &den[j], &m[j]);
            }
        }
        if (num_out) {
            for (int64_t j = 0; j < nc; ++j) {
                const int64_t s = b * C + c0 + j;
                num_out[s] = num[j];
                den_out[s] = den[j];
                max_out[s] = m[j];
            }
        }
    }
}

/*
 * One decode token for S independent streams: k, v [S, C] fp32; the state is
 * read from (num_in, den_in, max_in) and written to (num_out, den_out,
 * max_out), all float64 [S, C] (the two may be the same arrays).
 */
void wkv_oracle_step(int64_t S, int64_t C, const float *k, const float *v,
                     const float *w, const float *u,
                     const double *num_in, const double *den_in, const double *max_in,
                     double *out, double *num_out, double *den_out, double *max_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < S * C; ++i) {
        const int64_t c = i % C;
        double num = num_in[i], den = den_in[i], m = max_in[i];
        out[i] = wkv_token((double)k[i], (double)v[i], (double)w[c], (double)u[c], &num, &den, &m);
        num_out[i] = num;
        den_out[i] = den;
        max_out[i] = m;
    }
}

int wkv_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Two extensions of the same recurrence, from "RWKV-v6 Architecture:
 * Attention-Free Linear Transformers":
 *
 *   - section "2. Dynamic Data-Dependent Decay": the decay becomes a per-token
 *     vector w_t. Here w_t takes the place of w in the step above at token t
 *     (the state is multiplied by e^{-w_t} when token t is added), so an
 *     earlier token i reaches the output of token t with the exponent
 *     k_i - (w_{i+1} + ... + w_{t-1}).
 *   - section "3. Matrix-Valued Hidden State" (the readout) and the
 *     Time-Mixing description of "RWKV: Merging Transformer Training with RNN
 *     Speed": the output is gated by the receptance, y_t = sigmoid(r_t) * wkv_t.
 *
 * w_t: NULL (use w for every token) or [B, T, C] fp32. r: NULL (no gate) or
 * [B, T, C] of element type kv_dtype. Everything else as wkv_oracle_forward.
 */
void wkv_oracle_forward_ext(int64_t B, int64_t T, int64_t C,
                            const void *k, const void *v, int kv_dtype,
                            const float *w, const float *w_t, const float *u, const void *r,
                            const double *num_in, const double *den_in, const double *max_in,
                            double *out,
                            double *num_out, double *den_out, double *max_out,
                            int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t s = 0; s < B * C; ++s) {
        const int64_t b = s / C, c = s % C;
        double num = 0.0, den = 0.0, m = -INFINITY;
        if (num_in) {
            num = num_in[s];
            den = den_in[s];
            m = max_in[s];
        }
        const double uc = (double)u[c];
        for (int64_t t = 0; t < T; ++t) {
            const size_t i = ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c;
            const double kt = widen(k, kv_dtype, i);
            const double vt = widen(v, kv_dtype, i);
            const double wt = w_t ? (double)w_t[i] : (double)w[c];
            double y = wkv_token(kt, vt, wt, uc, &num, &den, &m);
            if (r) y = y / (1.0 + exp(-widen(r, kv_dtype, i)));
            out[i] = y;
        }
        if (num_out) {
            num_out[s] = num;
            den_out[s] = den;
            max_out[s] = m;
        }
    }
}

/*
 * One decode token for S streams with the same two extensions: w is [C]
 * (w_per_stream = 0) or [S, C] (the per-token decay of this step for every
 * stream); r is NULL or [S, C] fp32. Everything else as wkv_oracle_step.
 */
void wkv_oracle_step_ext(int64_t S, int64_t C, const float *k, const float *v,
                         const float *w, int w_per_stream, const float *u, const float *r,
                         const double *num_in, const double *den_in, const double *max_in,
                         double *out, double *num_out, double *den_out, double *max_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < S * C; ++i) {
        const int64_t c = i % C;
        double num = num_in[i], den = den_in[i], m = max_in[i];
        const double wi = (double)(w_per_stream ? w[i] : w[c]);
        double y = wkv_token((double)k[i], (double)v[i], wi, (double)u[c], &num, &den, &m);
        if (r) y = y / (1.0 + exp(-(double)r[i]));
        out[i] = y;
        num_out[i] = num;
        den_out[i] = den;
        max_out[i] = m;
    }
}

/*
 * Gradients of the forward for a loss whose gradient with respect to every
 * output is given (gout = dL/d wkv, [B, T, C]); no loss term on the final
 * state. This is the chain rule applied to the step function of "The
 * recurrence", backwards in time:
 *
 *   Write the state before token t as the pair (N_t, D_t) = (num, den) e^{m}
 *   and the output as wkv_t = A_t / Z_t with A_t = N_t + e^{u+k_t} v_t,
 *   Z_t = D_t + e^{u+k_t}. The state advances as N_{t+1} = e^{-w} N_t +
 *   e^{k_t} v_t (D likewise with v = 1). With dN_t = dL/dN_t (the total effect
 *   through every later output) and dD_t likewise:
 *     dN_t = g_t / Z_t + e^{-w} dN_{t+1},  dD_t = -g_t wkv_t / Z_t + e^{-w} dD_{t+1},
 *     dN_T = dD_T = 0,
 *     dv_t = g_t e^{u+k_t} / Z_t + e^{k_t} dN_{t+1},
 *     dk_t = g_t e^{u+k_t} (v_t - wkv_t) / Z_t + e^{k_t} (v_t dN_{t+1} + dD_{t+1}),
 *     du  += g_t e^{u+k_t} (v_t - wkv_t) / Z_t,
 *     dw  -= e^{-w} (N_t dN_{t+1} + D_t dD_{t+1}),
 *   and for the state passed in, (N_0, D_0) = (num0, den0) e^{m0}:
 *     dnum0 = e^{m0} dN_0, dden0 = e^{m0} dD_0, dm0 = num0 dnum0 + den0 dden0.
 *
 * Every exponential is taken relative to a running maximum, as in the forward:
 * Z_t relative to e_t = max(m_t, u + k_t), and (dN_t, dD_t) = (rn, rd) e^{Q_t}
 * with Q_t the largest exponent contributing to them.
 *
 * The s* outputs (optional, NULL to skip) are the same formulas with every
 * signed quantity replaced by the sum of the magnitudes of its own terms: g by
 * |g|, v by |v|, the state's numerator and wkv_t by the same sums taken over
 * |v| (for wkv_t that is sum_i p_i |v_i|, the scale the forward is measured
 * against), and the accumulators run on those. The result bounds the sum of
 * the magnitudes of every term that makes up each gradient: the scale against
 * which its rounding error is measured.
 *
 * dw and du are [C], summed over the batch rows; the state gradients are
 * [B, C] (NULL to skip).
 */
void wkv_oracle_backward(int64_t B, int64_t T, int64_t C,
                         const void *k, const void *v, int kv_dtype,
                         const float *w, const float *u,
                         const double *num_in, const double *den_in, const double *max_in,
                         const double *gout,
                         double *dk, double *dv, double *dw, double *du,
                         double *dnum, double *dden, double *dmax,
                         double *sk, double *sv, double *sw, double *su,
                         double *snum, double *sden, double *smax,
                         int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    /* per (b, c) partial sums of dw, du (and their scales), summed over b below */
    double *pw = (double *)calloc((size_t)(B * C) * 4, sizeof(double));

#pragma omp parallel
    {
        double *st = (double *)malloc(sizeof(double) * 4 * (size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t s = 0; s < B * C; ++s) {
            const int64_t b = s / C, c = s % C;
            const double wc = (double)w[c], uc = (double)u[c];
            double num = 0.0, den = 0.0, m = -INFINITY;
            if (num_in) {
                num = num_in[s];
                den = den_in[s];
                m = max_in[s];
            }
            const double num0 = num, den0 = den, m0 = m;
            /* the numerator over |v| (same exponents and denominator) */
            double numa = fabs(num), dena = den, ma = m;
            /* forward: the state before every token */
            for (int64_t t = 0; t < T; ++t) {
                const size_t i = ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c;
                st[4 * t] = num;
                st[4 * t + 1] = den;
                st[4 * t + 2] = m;
                st[4 * t + 3] = numa;
                const double kt = widen(k, kv_dtype, i), vt = widen(v, kv_dtype, i);
                (void)wkv_token(kt, vt, wc, uc, &num, &den, &m);
                (void)wkv_token(kt, fabs(vt), wc, uc, &numa, &dena, &ma);
            }
            /* backward */
            double rn = 0.0, rd = 0.0, an = 0.0, ad = 0.0, Q = -INFINITY;
            double gu = 0.0, gw = 0.0, au = 0.0, aw = 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                const size_t i = ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c;
                const double kt = widen(k, kv_dtype, i), vt = widen(v, kv_dtype, i), g = gout[i];
                const double nt = st[4 * t], dt = st[4 * t + 1], mt = st[4 * t + 2], nta = st[4 * t + 3];
                const double e = fmax(mt, kt + uc);
                const double a = exp(mt - e), bb = exp(kt + uc - e);
                const double z = a * dt + bb;
                const double out = (a * nt + bb * vt) / z;
                const double outa = (a * nta + bb * fabs(vt)) / z;  /* sum_i p_i |v_i| */
                const double p = g / z, q = -g * out / z;
                const double pa = fabs(g) / z, qa = fabs(g) * outa / z;
                const double E1 = exp(kt + Q);          /* e^{k_t} relative to dN_{t+1}'s exponent */
                const double E2 = exp(mt + Q - wc);     /* e^{m_t - w}, likewise */
                dv[i] = p * bb + rn * E1;
                dk[i] = p * bb * (vt - out) + E1 * (vt * rn + rd);
                gu += p * bb * (vt - out);
                gw -= E2 * (nt * rn + dt * rd);
                if (sv) {
                    sv[i] = pa * bb + an * E1;
                    sk[i] = pa * bb * (fabs(vt) + outa) + E1 * (fabs(vt) * an + ad);
                }
                au += pa * bb * (fabs(vt) + outa);
                aw += E2 * (nta * an + dt * ad);
                /* move the accumulators to position t: decay by w, add token t */
                const double Qn = fmax(Q - wc, -e);
                const double x1 = exp(Q - wc - Qn), x2 = exp(-e - Qn);
                rn = rn * x1 + p * x2;
                rd = rd * x1 + q * x2;
                an = an * x1 + pa * x2;
                ad = ad * x1 + qa * x2;
                Q = Qn;
            }
            pw[4 * s] = gw;
            pw[4 * s + 1] = gu;
            pw[4 * s + 2] = aw;
            pw[4 * s + 3] = au;
            if (dnum) {
                const double f = (m0 == -INFINITY || !(den0 > 0.0)) ? 0.0 : exp(m0 + Q);
                dnum[s] = rn * f;
                dden[s] = rd * f;
                dmax[s] = num0 * dnum[s] + den0 * dden[s];
                if (snum) {
                    snum[s] = an * f;
                    sden[s] = ad * f;
                    smax[s] = fabs(num0) * snum[s] + den0 * sden[s];
                }
            }
        }
        free(st);
    }
    for (int64_t c = 0; c < C; ++c) {
        double gw = 0.0, gu = 0.0, aw = 0.0, au = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            const int64_t s = b * C + c;
            gw += pw[4 * s];
            gu += pw[4 * s + 1];
            aw += pw[4 * s + 2];
            au += pw[4 * s + 3];
        }
        dw[c] = gw;
        du[c] = gu;
        if (sw) {
            sw[c] = aw;
            su[c] = au;
        }
    }
    free(pw);
}
