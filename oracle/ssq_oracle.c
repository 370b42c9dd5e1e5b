/*
 * ssq_oracle.c -- plain, slow CPU oracle for the quantized Mamba-2
 * recurrent-state update.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Scalar loops, no
 * blocking, no vectorisation, no reordering beyond what the definitions
 * state.  Build with -O2 -ffp-contract=off so that every fp32 operation below
 * is one correctly rounded IEEE operation in the order written.
 *
 * Citations use the page title and section; see ssq_oracle.h for the list
 * of sources and of the readings taken where the pages are silent.
 *
 * Parity pins (tests/test_oracle_*.py): the recurrence against its unrolled
 * closed form; the quantizer against brute-force code enumeration, the
 * |deq - v| <= Delta/2 bound, the grid-endpoint and dyadic-exactness
 * invariants, idempotence and scale equivariance; the readout against its
 * closed form at T=1.  The fp64 trajectory is pinned by the same closed
 * form.  Multi-step drift is reported, not pinned.
 */
#include "ssq_oracle.h"

#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

int oref_bits(int fmt)
{
    switch (fmt) {
    case OREF_I8_SYM: case OREF_I8_ASYM: return 8;
    case OREF_I4_SYM: case OREF_I4_ASYM: return 4;
    case OREF_BF16: return 16;
    default: return 32;
    }
}

int oref_is_quant(int fmt) { return fmt >= OREF_I8_SYM && fmt <= OREF_I4_ASYM; }
int oref_is_sym(int fmt) { return fmt == OREF_I8_SYM || fmt == OREF_I4_SYM; }

/* ssm-state-quantization README, Setup: heads outside the chosen lambda band
 * are not rounded ("mid band only" vs "all heads").  A head is quantized when
 * the format is an integer format and its mask entry is non-zero. */
int oref_row_is_quant(const oref_cfg* c, int h)
{
    if (!oref_is_quant(c->fmt)) return 0;
    if (c->head_mask == NULL) return 1;
    return c->head_mask[h] != 0;
}

/* ssm-state-quantization README, Setup: lambda = exp(dt * A).  dt*A is one
 * fp32 product; the exponential is taken in double and rounded once to
 * fp32. */
float oref_lambda(float dt, float A)
{
    float dA = dt * A;
    double e = exp((double)dA);
    return (float)e;
}

/* Round an fp32 value to the nearest bf16 value, ties to even, and return it
 * widened back to fp32 (bf16 keeps the top 16 bits of the fp32 pattern). */
float oref_bf16_round(float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) { /* inf / nan: truncate */
        u &= 0xffff0000u;
    } else {
        uint32_t lsb = (u >> 16) & 1u;
        u = u + 0x7fffu + lsb;
        u &= 0xffff0000u;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/* Largest code magnitude: qs = 2^(b-1)-1 on the symmetric grid, qa = 2^b-1 on
 * the asymmetric grid (ssm-state-quantization README, Setup). */
static float qmax_of(int fmt)
{
    int b = oref_bits(fmt);
    if (oref_is_sym(fmt)) return (float)((1 << (b - 1)) - 1);
    return (float)((1 << b) - 1);
}

/* Refit and round one row (ssm-state-quantization README, Setup: per-row
 * scale refit every step, symmetric or asymmetric grid; Findings 1: nearest
 * rounding).  Each value is rounded to the nearest integer multiple of the
 * step as v*inv with the product taken exactly (in double, where the product
 * of two floats is exact) and one rounding, ties to even; the zero point
 * likewise.  'pre' (optional) receives the pre-rounding value v*inv of each
 * entry, used by the tests to find entries on a rounding boundary. */
void oref_quantize_row_dbg(int fmt, int N, const float* v, int32_t* q,
                           float* delta_out, float* zero_out, float* pre)
{
    const float qm = qmax_of(fmt);
    const int sym = oref_is_sym(fmt);
    float delta, inv, z = 0.0f, lo = 0.0f;

    if (sym) {
        /* amax over the row; step amax / qs. */
        float amax = 0.0f;
        for (int n = 0; n < N; ++n) {
            float a = fabsf(v[n]);
            if (a > amax) amax = a;
        }
        delta = amax / qm;
    } else {
        /* [min, max] over the row; step (max - min) / qa. */
        float hi = v[0];
        lo = v[0];
        for (int n = 1; n < N; ++n) {
            if (v[n] < lo) lo = v[n];
            if (v[n] > hi) hi = v[n];
        }
        float range = hi - lo;
        delta = range / qm;
        /* Constant row: any positive step reproduces it; |lo| makes the
         * reconstruction exact (z = -/+1, code 0). */
        if (delta == 0.0f) delta = fabsf(lo);
    }
    /* A step below the smallest normal fp32 flushes the row to zero. */
    if (delta < FLT_MIN) delta = 0.0f;
    inv = (delta == 0.0f) ? 0.0f : 1.0f / delta;
    if (!sym) {
        /* Integer zero point: the code of lo is rint(lo*inv) + z = 0.
         * Adding +0 stores a negative zero as +0. */
        z = (float)rint(-(double)lo * (double)inv) + 0.0f;
    }

    for (int n = 0; n < N; ++n) {
        double p = (double)v[n] * (double)inv;   /* the exact product */
        float r = (float)rint(p);                 /* nearest, ties to even */
        if (pre) pre[n] = (float)p;
        float c;
        if (sym) {
            c = r;
            if (c > qm) c = qm;
            if (c < -qm) c = -qm;
        } else {
            c = r + z;                 /* exact: both are integers of equal
                                          sign or within a factor 2 */
            if (c > qm) c = qm;
        }
        q[n] = (int32_t)c;
    }
    *delta_out = delta;
    *zero_out = z;
}

void oref_quantize_row(int fmt, int N, const float* v, int32_t* q,
                       float* delta, float* zero)
{
    oref_quantize_row_dbg(fmt, N, v, q, delta, zero, NULL);
}

/* Dequantize a row: s = (q - z) * Delta on the asymmetric grid, q * Delta on
 * the symmetric grid.  q - z is exact in fp32 for the code and zero-point
 * ranges that occur; the product is one rounding. */
void oref_dequantize_row(int fmt, int N, const int32_t* q, float delta,
                         float zero, float* out)
{
    for (int n = 0; n < N; ++n) {
        if (oref_is_sym(fmt)) {
            out[n] = (float)q[n] * delta;
        } else {
            float d = (float)q[n] - zero;
            out[n] = d * delta;
        }
    }
}

/* Fill a logical state from an fp32 tensor S[H][P][N]: quantized rows go
 * through the row quantizer, fp rows are stored (bf16-rounded for bf16). */
void oref_state_from_f32(const oref_cfg* c, const float* S, oref_state* st)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state;
    for (int h = 0; h < H; ++h) {
        for (int p = 0; p < P; ++p) {
            const int r = h * P + p;
            const float* v = S + (size_t)r * N;
            if (oref_row_is_quant(c, h)) {
                oref_quantize_row(c->fmt, N, v, st->q + (size_t)r * N,
                                  st->delta + r, st->zero + r);
            } else {
                for (int n = 0; n < N; ++n) {
                    float s = v[n];
                    if (c->fmt == OREF_BF16) s = oref_bf16_round(s);
                    st->val[(size_t)r * N + n] = s;
                }
            }
        }
    }
}

/* Read a logical state back as fp32 S[H][P][N]. */
void oref_state_to_f32(const oref_cfg* c, const oref_state* st, float* S)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state;
    for (int h = 0; h < H; ++h) {
        for (int p = 0; p < P; ++p) {
            const int r = h * P + p;
            if (oref_row_is_quant(c, h)) {
                oref_dequantize_row(c->fmt, N, st->q + (size_t)r * N,
                                    st->delta[r], st->zero[r],
                                    S + (size_t)r * N);
            } else {
                memcpy(S + (size_t)r * N, st->val + (size_t)r * N,
                       sizeof(float) * (size_t)N);
            }
        }
    }
}

/* One decode step of one (layer, request).
 *
 * For every head h and row p:
 *   1. decode the stored row;
 *   2. lambda = exp(dt_h*A_h); dtx = dt_h*x_p; w_n = dtx*B_{g,n};
 *      s'_n = fma(lambda, s_n, w_n)          (the Mamba-2 recurrence
 *      S = exp(dt*A)*S + dt*B(x)x of "ssm-state-quantization", Setup, with
 *      the FP32 update of "Mamba state quantization for inference");
 *   3-5. refit, round and store the row (quantized heads), or store s'
 *      (fp heads; bf16-rounded for the bf16 format);
 *   6. y_p = sum_n C_{g,n} * stored_n + D_h*x_p, accumulated in double and
 *      read from the newly stored state ("ssm-state-quantization", Setup:
 *      the output is read from the quantized state).
 * x[H][P], B/C[G][N], dt/A/D[H], y[H][P].  'pre' (optional, [H*P*N])
 * receives s'*inv for quantized rows. */
void oref_step(const oref_cfg* c, oref_state* st, const float* x,
               const float* B, const float* C, const float* dt,
               const float* A, const float* D, float* y, float* pre)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int heads_per_group = H / G;
    float* s = (float*)malloc(sizeof(float) * (size_t)N);
    float* sn = (float*)malloc(sizeof(float) * (size_t)N);
    float* stored = (float*)malloc(sizeof(float) * (size_t)N);

    for (int h = 0; h < H; ++h) {
        const int g = h / heads_per_group;
        const float lam = oref_lambda(dt[h], A[h]);
        const float* Bg = B + (size_t)g * N;
        const float* Cg = C + (size_t)g * N;
        const int quant = oref_row_is_quant(c, h);
        for (int p = 0; p < P; ++p) {
            const int r = h * P + p;
            /* 1. decode */
            if (quant) {
                oref_dequantize_row(c->fmt, N, st->q + (size_t)r * N,
                                    st->delta[r], st->zero[r], s);
            } else {
                memcpy(s, st->val + (size_t)r * N, sizeof(float) * (size_t)N);
            }
            /* 2. decay and input */
            const float dtx = dt[h] * x[r];
            for (int n = 0; n < N; ++n) {
                float w = dtx * Bg[n];
                sn[n] = fmaf(lam, s[n], w);
            }
            /* 3-5. refit, round, store */
            if (quant) {
                int32_t* qr = st->q + (size_t)r * N;
                oref_quantize_row_dbg(c->fmt, N, sn, qr, st->delta + r,
                                      st->zero + r,
                                      pre ? pre + (size_t)r * N : NULL);
                oref_dequantize_row(c->fmt, N, qr, st->delta[r], st->zero[r],
                                    stored);
            } else {
                for (int n = 0; n < N; ++n) {
                    float v = sn[n];
                    if (c->fmt == OREF_BF16) v = oref_bf16_round(v);
                    st->val[(size_t)r * N + n] = v;
                    stored[n] = v;
                }
            }
            /* 6. readout from the stored state */
            double acc = 0.0;
            for (int n = 0; n < N; ++n)
                acc += (double)Cg[n] * (double)stored[n];
            acc += (double)D[h] * (double)x[r];
            y[r] = (float)acc;
        }
    }
    free(s);
    free(sn);
    free(stored);
}

/* Per-token scan ("ssm-state-quantization", Setup: a sequential scan that
 * rounds the state at every step): T applications of the decode step, token
 * t+1 reading the state stored at token t.
 * x[T][H][P], B/C[T][G][N], dt[T][H], A/D[H], y[T][H][P]. */
void oref_scan(const oref_cfg* c, oref_state* st, int T, const float* x,
               const float* B, const float* C, const float* dt,
               const float* A, const float* D, float* y)
{
    const size_t HP = (size_t)c->nheads * c->headdim;
    const size_t GN = (size_t)c->ngroups * c->d_state;
    for (int t = 0; t < T; ++t) {
        oref_step(c, st, x + t * HP, B + t * GN, C + t * GN,
                  dt + (size_t)t * c->nheads, A, D, y + t * HP, NULL);
    }
}

/* ---------------------------------------------------------------------------
 * Stochastic rounding ("ssm-state-quantization" README, Findings 9: SR of the
 * state keeps 8 bits within 0.4 ppl of the control).  Each entry rounds down
 * or up to a neighbouring grid level with probability given by its distance:
 * code = floor(v*inv + u) (+ z), u uniform in [0, 1) on a 2^-16 grid, the
 * product exact and the sum exact (both in double), then clamped to the
 * code range (the minimum can now round down one level, the maximum up one).
 * The grid (Delta, z) is refit as for nearest rounding.
 * Parity: the rounding rule is pinned by the tests (neighbours only, grid
 * points fixed, unbiased on average); the generator by statistics only.
 * ------------------------------------------------------------------------- */

/* Philox4x32-10 from its definition: ten rounds of two 32x32->64-bit
 * multiplications by fixed constants, the high halves XORed with the other
 * two counter words and the key, the key bumped by two Weyl constants after
 * each round. */
void oref_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

uint32_t oref_sr_u16(const oref_sr* r, int row, int n, int N)
{
    const uint32_t ctr[4] = {(uint32_t)row * (uint32_t)(N / 8) + (uint32_t)(n / 8),
                             r->layer, r->slot, r->step};
    const uint32_t key[2] = {(uint32_t)r->seed, (uint32_t)(r->seed >> 32)};
    uint32_t out[4];
    oref_philox4x32_10(ctr, key, out);
    return (out[(n % 8) / 2] >> (16 * (n % 2))) & 0xFFFFu;
}

void oref_quantize_row_sr(int fmt, int N, const float* v, const uint32_t* u16,
                          int32_t* q, float* delta_out, float* zero_out)
{
    /* the grid: as for nearest rounding */
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
    oref_quantize_row(fmt, N, v, tmp, delta_out, zero_out);
    free(tmp);
    const float delta = *delta_out, z = *zero_out;
    const float qm = qmax_of(fmt);
    const int sym = oref_is_sym(fmt);
    const float inv = (delta == 0.0f) ? 0.0f : 1.0f / delta;
    for (int n = 0; n < N; ++n) {
        const double p = (double)v[n] * (double)inv;       /* exact */
        const double k = floor(p + (double)u16[n] / 65536.0); /* exact sum */
        float c = (float)k;
        if (sym) {
            if (c > qm) c = qm;
            if (c < -qm) c = -qm;
        } else {
            c = c + z;
            if (c > qm) c = qm;
            if (c < 0.0f) c = 0.0f;
        }
        q[n] = (int32_t)c;
    }
}

/* One decode step with stochastic rounding of the quantized rows (steps 1,
 * 2 and 6 as oref_step). */
void oref_step_sr(const oref_cfg* c, oref_state* st, const oref_sr* r,
                  const float* x, const float* B, const float* C,
                  const float* dt, const float* A, const float* D, float* y)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int heads_per_group = H / G;
    float* s = (float*)malloc(sizeof(float) * (size_t)N);
    float* sn = (float*)malloc(sizeof(float) * (size_t)N);
    float* stored = (float*)malloc(sizeof(float) * (size_t)N);
    uint32_t* u = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)N);
    for (int h = 0; h < H; ++h) {
        const int g = h / heads_per_group;
        const float lam = oref_lambda(dt[h], A[h]);
        const float* Bg = B + (size_t)g * N;
        const float* Cg = C + (size_t)g * N;
        const int quant = oref_row_is_quant(c, h);
        for (int p = 0; p < P; ++p) {
            const int row = h * P + p;
            if (quant) {
                oref_dequantize_row(c->fmt, N, st->q + (size_t)row * N,
                                    st->delta[row], st->zero[row], s);
            } else {
                memcpy(s, st->val + (size_t)row * N, sizeof(float) * (size_t)N);
            }
            const float dtx = dt[h] * x[row];
            for (int n = 0; n < N; ++n) {
                float w = dtx * Bg[n];
                sn[n] = fmaf(lam, s[n], w);
            }
            if (quant) {
                for (int n = 0; n < N; ++n) u[n] = oref_sr_u16(r, row, n, N);
                int32_t* qr = st->q + (size_t)row * N;
                oref_quantize_row_sr(c->fmt, N, sn, u, qr, st->delta + row, st->zero + row);
                oref_dequantize_row(c->fmt, N, qr, st->delta[row], st->zero[row], stored);
            } else {
                for (int n = 0; n < N; ++n) {
                    float v = sn[n];
                    if (c->fmt == OREF_BF16) v = oref_bf16_round(v);
                    st->val[(size_t)row * N + n] = v;
                    stored[n] = v;
                }
            }
            double acc = 0.0;
            for (int n = 0; n < N; ++n)
                acc += (double)Cg[n] * (double)stored[n];
            acc += (double)D[h] * (double)x[row];
            y[row] = (float)acc;
        }
    }
    free(s);
    free(sn);
    free(stored);
    free(u);
}

/* T steps with stochastic rounding; token t draws with step r->step + t. */
void oref_scan_sr(const oref_cfg* c, oref_state* st, const oref_sr* r, int T,
                  const float* x, const float* B, const float* C,
                  const float* dt, const float* A, const float* D, float* y)
{
    const size_t HP = (size_t)c->nheads * c->headdim;
    const size_t GN = (size_t)c->ngroups * c->d_state;
    oref_sr rt = *r;
    for (int t = 0; t < T; ++t) {
        rt.step = r->step + (uint32_t)t;
        oref_step_sr(c, st, &rt, x + t * HP, B + t * GN, C + t * GN,
                     dt + (size_t)t * c->nheads, A, D, y + t * HP);
    }
}

/* Diagnostics of one decode step ("ssm-state-quantization" README, Findings
 * 4 and 5): for every row, without changing the state, the step that
 * oref_step would take is evaluated and
 *   diag[4r+0] = reversals: entries whose applied increment e + w opposes
 *                the new input w = fl(dt*x)*B_n (w != 0 and e + w of the
 *                other sign), e = fl(deq - s') the rounding error, e + w in
 *                fp32 (the decision is taken in fp32 on both sides);
 *   diag[4r+1] = sum over reversed entries of C_n * e_n (the reversal error
 *                seen by the readout);
 *   diag[4r+2] = sum over all entries of C_n * e_n (the readout-visible
 *                rounding error: y from the stored state minus y from s');
 *   diag[4r+3] = sum over all entries of C_n * s'_n (the readout signal).
 * Sums in double.  fp rows are not rounded: zeros but the signal. */
void oref_step_diag(const oref_cfg* c, const oref_state* st, const float* x,
                    const float* B, const float* C, const float* dt,
                    const float* A, const float* D, float* diag)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int heads_per_group = H / G;
    float* s = (float*)malloc(sizeof(float) * (size_t)N);
    float* sn = (float*)malloc(sizeof(float) * (size_t)N);
    float* w = (float*)malloc(sizeof(float) * (size_t)N);
    float* deq = (float*)malloc(sizeof(float) * (size_t)N);
    int32_t* q = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
    (void)D;
    for (int h = 0; h < H; ++h) {
        const int g = h / heads_per_group;
        const float lam = oref_lambda(dt[h], A[h]);
        const float* Bg = B + (size_t)g * N;
        const float* Cg = C + (size_t)g * N;
        const int quant = oref_row_is_quant(c, h);
        for (int p = 0; p < P; ++p) {
            const int r = h * P + p;
            if (quant) {
                oref_dequantize_row(c->fmt, N, st->q + (size_t)r * N, st->delta[r],
                                    st->zero[r], s);
            } else {
                memcpy(s, st->val + (size_t)r * N, sizeof(float) * (size_t)N);
            }
            const float dtx = dt[h] * x[r];
            for (int n = 0; n < N; ++n) {
                w[n] = dtx * Bg[n];
                sn[n] = fmaf(lam, s[n], w[n]);
            }
            double rev = 0.0, rev_err = 0.0, tot_err = 0.0, signal = 0.0;
            for (int n = 0; n < N; ++n) signal += (double)Cg[n] * (double)sn[n];
            if (quant) {
                float dl, z;
                oref_quantize_row(c->fmt, N, sn, q, &dl, &z);
                oref_dequantize_row(c->fmt, N, q, dl, z, deq);
                for (int n = 0; n < N; ++n) {
                    const float e = deq[n] - sn[n];
                    const float inc = e + w[n];
                    const int reversed = (w[n] > 0.0f && inc < 0.0f) || (w[n] < 0.0f && inc > 0.0f);
                    tot_err += (double)Cg[n] * (double)e;
                    if (reversed) {
                        rev += 1.0;
                        rev_err += (double)Cg[n] * (double)e;
                    }
                }
            }
            diag[4 * (size_t)r + 0] = (float)rev;
            diag[4 * (size_t)r + 1] = (float)rev_err;
            diag[4 * (size_t)r + 2] = (float)tot_err;
            diag[4 * (size_t)r + 3] = (float)signal;
        }
    }
    free(s);
    free(sn);
    free(w);
    free(deq);
    free(q);
}

/* Prefill hand-off ("Mamba state quantization for inference", "Mamba state
 * quantization needs phase-aware benchmarks": the prefill runs in fp32 and
 * only its last state is packed): from the stored state, T tokens of the fp32 recurrence
 * s'_n = fma(lambda, s_n, fl(dt*x) * B_n) with no rounding between tokens,
 * y_t read from the fp32 state (accumulated in double), and the state
 * quantized (or stored, bf16-rounded for the bf16 format) once after the
 * last token.  x[T][H][P], B/C[T][G][N], dt[T][H], A/D[H], y[T][H][P]. */
void oref_prefill(const oref_cfg* c, oref_state* st, int T, const float* x,
                  const float* B, const float* C, const float* dt,
                  const float* A, const float* D, float* y)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int hpg = H / G;
    const size_t HP = (size_t)H * P;
    const size_t GN = (size_t)G * N;
    float* s = (float*)malloc(sizeof(float) * (size_t)N);
    for (int h = 0; h < H; ++h) {
        const int g = h / hpg;
        const int quant = oref_row_is_quant(c, h);
        for (int p = 0; p < P; ++p) {
            const size_t r = (size_t)h * P + p;
            /* the stored state, decoded once */
            if (quant) {
                oref_dequantize_row(c->fmt, N, st->q + r * N, st->delta[r],
                                    st->zero[r], s);
            } else {
                memcpy(s, st->val + r * N, sizeof(float) * (size_t)N);
            }
            for (int t = 0; t < T; ++t) {
                const float lam = oref_lambda(dt[(size_t)t * H + h], A[h]);
                const float* Bg = B + t * GN + (size_t)g * N;
                const float* Cg = C + t * GN + (size_t)g * N;
                const float xv = x[t * HP + r];
                const float dtx = dt[(size_t)t * H + h] * xv;
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    float w = dtx * Bg[n];
                    s[n] = fmaf(lam, s[n], w);
                    acc += (double)Cg[n] * (double)s[n];
                }
                acc += (double)D[h] * (double)xv;
                y[t * HP + r] = (float)acc;
            }
            /* the hand-off: one refit and rounding of the final state */
            if (quant) {
                oref_quantize_row(c->fmt, N, s, st->q + r * N, st->delta + r,
                                  st->zero + r);
            } else {
                for (int n = 0; n < N; ++n) {
                    float v = s[n];
                    if (c->fmt == OREF_BF16) v = oref_bf16_round(v);
                    st->val[r * N + n] = v;
                }
            }
        }
    }
    free(s);
}

/* Unquantized trajectory in double, used only to report drift: the exact
 * recurrence S_t = A_t S_(t-1) + W_t of "Mamba state quantization for
 * inference" (no residual R_t), with lambda = exp(dt*A) and W = dt*B(x)x,
 * every operation in double.  S[H][P][N] in/out. */
void oref_scan_f64(const oref_cfg* c, double* S, int T, const float* x,
                   const float* B, const float* C, const float* dt,
                   const float* A, const float* D, double* y)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int hpg = H / G;
    const size_t HP = (size_t)H * P;
    const size_t GN = (size_t)G * N;
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            const double dtd = (double)dt[(size_t)t * H + h];
            const double lam = exp(dtd * (double)A[h]);
            const float* Bg = B + t * GN + (size_t)g * N;
            const float* Cg = C + t * GN + (size_t)g * N;
            for (int p = 0; p < P; ++p) {
                const size_t r = (size_t)h * P + p;
                const double xv = (double)x[t * HP + r];
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    double* sv = S + r * N + n;
                    *sv = lam * (*sv) + dtd * xv * (double)Bg[n];
                    acc += (double)Cg[n] * (*sv);
                }
                y[t * HP + r] = acc + (double)D[h] * xv;
            }
        }
    }
}

/* One decode step over nl layers and a batch of requests: the same step for
 * every (layer, request) pair.  states[l*batch + b];
 * x/y[nl][batch][H][P], B/C[nl][batch][G][N], dt[nl][batch][H], A/D[nl][H]. */
void oref_decode_batch(const oref_cfg* c, int nl, int batch,
                       oref_state* states, const float* x, const float* B,
                       const float* C, const float* dt, const float* A,
                       const float* D, float* y)
{
    const size_t HP = (size_t)c->nheads * c->headdim;
    const size_t GN = (size_t)c->ngroups * c->d_state;
    const size_t H = (size_t)c->nheads;
    for (int l = 0; l < nl; ++l) {
        for (int b = 0; b < batch; ++b) {
            const size_t lb = (size_t)l * batch + b;
            oref_step(c, &states[lb], x + lb * HP, B + lb * GN, C + lb * GN,
                      dt + lb * H, A + l * H, D + l * H, y + lb * HP, NULL);
        }
    }
}

/* ------------------------------------------------------------------------
 * DAMP mixed-tier state ("Mamba state quantization for inference", "Mixed
 * precision spends bits on persistent channels"): each key channel's vector
 * over head_dim is rotated by a Hadamard matrix; a chosen set of channels
 * stays in FP16, the rest is stored as 8-bit codes with a step and an
 * offset; the chosen channels come first; every token decodes the 8-bit
 * tier, updates in fp32, fits new steps and stores the packed state.
 *
 * Readings (listed in the design notes):
 *   - state S[h][p][n]: p the value dimension (head_dim), n the key channel
 *     (d_state).  Key channel n of head h is the vector S[h][.][n] of
 *     length P, rotated to t[k] = sum_p H[k][p] S[h][p][n] with H the +-1
 *     Sylvester-Hadamard matrix, H[k][p] = (-1)^popcount(k & p), P a power of
 *     two; the sums are formed by the fast Walsh-Hadamard transform in
 *     double (butterfly stages h = 1, 2, ..., P/2) and rounded once to fp32
 *     (the stage order fixes the order of the double additions, which
 *     matters only when a double sum is inexact).  The inverse is
 *     S[p] = (1/P) sum_k H[p][k] t[k], formed the same way.
 *   - chan[h][m]: position m -> key channel; positions 0..K-1 are the
 *     protected (FP16) tier, K..N-1 the INT8 tier.  The selection is an
 *     input (its calibration needs data).
 *   - INT8 tier: each position's P rotated values form one group with the
 *     asymmetric 8-bit grid of the row quantizer (fp32 step and zero point):
 *     8 + 64/P bits per value, 9 at P = 64.
 *   - FP16 tier: fp32 -> fp16 round to nearest even (overflow to inf).
 *   - The recurrence is linear, so it runs on the rotated state with the
 *     rotated input: t' = fma(lambda, t, fl(fl(dt * xr[k]) * B[n])), xr the
 *     rotation of x (as above).  y reads the stored state:
 *     y[p] = D x[p] + (1/P) sum_k H[p][k] sum_m C[chan[m]] t'_m[k], in
 *     double, rounded once.
 * ---------------------------------------------------------------------- */

static int hsign(int a, int b)
{
    return (__builtin_popcount((unsigned)(a & b)) & 1) ? -1 : 1;
}

/* In-place fast Walsh-Hadamard transform of a[0..P-1] in double (Fino and
 * Algazi, "Unified matrix treatment of the fast Walsh-Hadamard transform",
 * IEEE Trans. Computers 1976): stages h = 1, 2, 4, ..., P/2; at each stage
 * the pair (a[i], a[i+h]), bit h of i clear, becomes (a[i] + a[i+h],
 * a[i] - a[i+h]).  The result is sum_p H[k][p] a[p] in Sylvester order;
 * each output is one fixed sequence of double additions. */
static void fwht_double(int P, double* a)
{
    for (int h = 1; h < P; h *= 2)
        for (int i = 0; i < P; ++i)
            if ((i & h) == 0) {
                const double x = a[i], y = a[i + h];
                a[i] = x + y;
                a[i + h] = x - y;
            }
}

/* out[k] = fl32(sum_p H[k][p] v[p * stride]): the fast transform in double,
 * rounded once. */
void oref_hadamard(int P, const float* v, int stride, float* out)
{
    double* a = (double*)malloc(sizeof(double) * (size_t)P);
    for (int p = 0; p < P; ++p) a[p] = (double)v[(size_t)p * stride];
    fwht_double(P, a);
    for (int k = 0; k < P; ++k) out[k] = (float)a[k];
    free(a);
}

float oref_fp16_round(float v)
{
    return (float)(_Float16)v;
}

/* Tiers of one head from the rotated values t[m][k] (position-major). */
static void damp_store_head(const oref_damp_cfg* c, const float* t, float* hi, int32_t* q,
                            float* delta, float* zero)
{
    const int P = c->headdim, N = c->d_state, K = c->n_protected;
    for (int m = 0; m < K; ++m)
        for (int k = 0; k < P; ++k)
            hi[(size_t)m * P + k] = oref_fp16_round(t[(size_t)m * P + k]);
    for (int m = K; m < N; ++m) {
        const int i = m - K;
        oref_quantize_row(OREF_I8_ASYM, P, t + (size_t)m * P, q + (size_t)i * P, &delta[i],
                          &zero[i]);
    }
}

/* The stored (rotated) values of one head, position-major t[m][k]. */
static void damp_load_head(const oref_damp_cfg* c, const float* hi, const int32_t* q,
                           const float* delta, const float* zero, float* t)
{
    const int P = c->headdim, N = c->d_state, K = c->n_protected;
    for (int m = 0; m < K; ++m)
        for (int k = 0; k < P; ++k) t[(size_t)m * P + k] = hi[(size_t)m * P + k];
    for (int m = K; m < N; ++m) {
        const int i = m - K;
        oref_dequantize_row(OREF_I8_ASYM, P, q + (size_t)i * P, delta[i], zero[i],
                            t + (size_t)m * P);
    }
}

static void damp_head_ptrs(const oref_damp_cfg* c, const oref_damp_state* st, int h,
                           float** hi, int32_t** q, float** delta, float** zero)
{
    const int P = c->headdim, N = c->d_state, K = c->n_protected;
    *hi = st->hi + (size_t)h * K * P;
    *q = st->q + (size_t)h * (N - K) * P;
    *delta = st->delta + (size_t)h * (N - K);
    *zero = st->zero + (size_t)h * (N - K);
}

/* S[H][P][N] fp32 -> tiers: rotate every key channel, then store. */
void oref_damp_from_f32(const oref_damp_cfg* c, const float* S, oref_damp_state* st)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state;
    float* t = (float*)malloc(sizeof(float) * (size_t)N * P);
    for (int h = 0; h < H; ++h) {
        const int32_t* ch = c->chan + (size_t)h * N;
        for (int m = 0; m < N; ++m)
            oref_hadamard(P, S + (size_t)h * P * N + ch[m], N, t + (size_t)m * P);
        float *hi, *dl, *z;
        int32_t* q;
        damp_head_ptrs(c, st, h, &hi, &q, &dl, &z);
        damp_store_head(c, t, hi, q, dl, z);
    }
    free(t);
}

/* Tiers -> S[H][P][N] fp32: reconstruct, rotate back (the fast transform
 * in double, then the exact 1/P), round once. */
void oref_damp_to_f32(const oref_damp_cfg* c, const oref_damp_state* st, float* S)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state;
    float* t = (float*)malloc(sizeof(float) * (size_t)N * P);
    double* a = (double*)malloc(sizeof(double) * (size_t)P);
    for (int h = 0; h < H; ++h) {
        float *hi, *dl, *z;
        int32_t* q;
        damp_head_ptrs(c, st, h, &hi, &q, &dl, &z);
        damp_load_head(c, hi, q, dl, z, t);
        const int32_t* ch = c->chan + (size_t)h * N;
        for (int m = 0; m < N; ++m) {
            for (int k = 0; k < P; ++k) a[k] = (double)t[(size_t)m * P + k];
            fwht_double(P, a);       /* H is symmetric: H^-1 = H / P */
            for (int p = 0; p < P; ++p)
                S[(size_t)h * P * N + (size_t)p * N + ch[m]] = (float)(a[p] / (double)P);
        }
    }
    free(t);
    free(a);
}

/* One decode step of one (layer, request) on the tiered state.
 * x[H][P], B/C[G][N], dt/A/D[H], y[H][P]. */
void oref_damp_step(const oref_damp_cfg* c, oref_damp_state* st, const float* x,
                    const float* B, const float* C, const float* dt, const float* A,
                    const float* D, float* y)
{
    const int H = c->nheads, P = c->headdim, N = c->d_state, G = c->ngroups;
    const int heads_per_group = H / G;
    float* t = (float*)malloc(sizeof(float) * (size_t)N * P);
    float* xr = (float*)malloc(sizeof(float) * (size_t)P);
    double* yr = (double*)malloc(sizeof(double) * (size_t)P);
    for (int h = 0; h < H; ++h) {
        const int g = h / heads_per_group;
        const float lam = oref_lambda(dt[h], A[h]);
        const int32_t* ch = c->chan + (size_t)h * N;
        float *hi, *dl, *z;
        int32_t* q;
        damp_head_ptrs(c, st, h, &hi, &q, &dl, &z);
        /* reconstruct the low tier (and read the FP16 tier) */
        damp_load_head(c, hi, q, dl, z, t);
        /* the input, rotated like the state */
        oref_hadamard(P, x + (size_t)h * P, 1, xr);
        /* the recurrence in FP32 */
        for (int m = 0; m < N; ++m) {
            const float b = B[(size_t)g * N + ch[m]];
            for (int k = 0; k < P; ++k) {
                const float dtx = dt[h] * xr[k];
                const float w = dtx * b;
                t[(size_t)m * P + k] = fmaf(lam, t[(size_t)m * P + k], w);
            }
        }
        /* new quantization parameters, packed state written back */
        damp_store_head(c, t, hi, q, dl, z);
        /* readout from the stored state, rotated back */
        damp_load_head(c, hi, q, dl, z, t);
        for (int k = 0; k < P; ++k) {
            double acc = 0.0;
            for (int m = 0; m < N; ++m)
                acc += (double)C[(size_t)g * N + ch[m]] * (double)t[(size_t)m * P + k];
            yr[k] = acc;
        }
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int k = 0; k < P; ++k) acc += (double)hsign(p, k) * yr[k];
            acc /= (double)P;
            acc += (double)D[h] * (double)x[(size_t)h * P + p];
            y[(size_t)h * P + p] = (float)acc;
        }
    }
    free(t);
    free(xr);
    free(yr);
}
