/*
 * attn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of exact attention, used by tests/,
 * by __graft_entry__.smoke() and by bench.py's cpu_baseline / reference arm
 * to check and time the CUDA library.  It shares no code, header, table or
 * constant with the CUDA path under exact_attention_140_b200/csrc, and the
 * product path never loads it.
 *
 * What it computes (page "FlashAttention (SV)", section "Problematik med
 * standard-attention", the attention formula):
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V,   LSE_i = ln sum_j exp(s_ij)
 *
 * with the exact reading choices below (the pages leave them open):
 *   - scale is the caller's number (the formula's 1/sqrt(d_k) is the usual one);
 *   - causal mask is bottom-right aligned: query row i may see key j iff
 *     j <= i + (Nk - Nq); with Nq == Nk this is the ordinary j <= i;
 *   - grouped heads: query head h reads key/value head h / (Hq / Hkv);
 *   - a row with no allowed key returns O = 0 and LSE = -inf;
 *   - LSE is the natural-log log-sum-exp of the *scaled* scores.
 *
 * Layouts: Q, O are [B, Nq, Hq, d]; K, V are [B, Nk, Hkv, d]; LSE is
 * [B, Hq, Nq]; all row-major fp64.
 *
 * Functions:
 *   oracle_attn_fwd        two-pass softmax (max, then sum/weights), the
 *                          definition itself.
 *   oracle_attn_fwd_rows   the same for a list of (b, h, i) rows only.
 *   oracle_attn_online     the blockwise online-softmax recurrence of page
 *                          "FlashAttention (SV)", section "Online-beräkning av
 *                          Softmax" (running max and running sum of
 *                          exponentials, output rescaled when the max moves),
 *                          with an optional lazy threshold tau on the max
 *                          update (page "FlashAttention-4震撼发布", the new
 *                          online softmax that skips most output rescalings).
 *   oracle_attn_fwd_window the definition over the keys [k0, k1) only (the
 *                          mask rule unchanged, in absolute key indices): the
 *                          partial result of one key window of split-KV.
 *   oracle_combine         merge of partial results over disjoint key windows,
 *                          O = sum_s e^(LSE_s - LSE) O_s with LSE = ln sum_s
 *                          e^(LSE_s): the rescaling step of the online softmax
 *                          (page "FlashAttention (SV)", section "Online-beräkning
 *                          av Softmax") applied to whole windows.
 *   oracle_attn_bruteforce long-double, materialised S, p_j = 1/sum_k e^(s_k-s_j):
 *                          a different algebra, for tiny inputs.
 *   oracle_hadamard        M = diag(s) H_d / sqrt(d) (Sylvester H_d), the random
 *                          orthogonal matrix of page "FlashAttention-3 —
 *                          闪电注意力-3", section 3 (incoherent processing).
 *   oracle_e4m3_decode / oracle_e4m3_encode
 *                          OCP FP8 E4M3 ("fn": no infinities, max 448), encode to
 *                          the nearest value (bisection over the ordered code
 *                          list), ties to the even code, saturating to +-448.
 *   oracle_quant_e4m3_f32  per-tensor quantisation x * (448/amax) in fp32, then
 *                          E4M3 encode.
 *   oracle_gemm_add        D = A B + C in fp64 (the small-K A@B+C workload page
 *                          "FlashAttention-4震撼发布" names for Blackwell), rows
 *                          of A [M, K], B [K, N], C and D [M, N], row-major.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static int allowed(long long i, long long j, long long Nq, long long Nk, int causal)
{
    if (j < 0 || j >= Nk) return 0;
    if (!causal) return 1;
    return j <= i + (Nk - Nq);
}

/* One output row: query (b, h, i) over the keys [j_lo, j_hi) (the whole
 * range is [0, Nk)).  q_row points at Q[b,i,h,:]. */
static void attend_row(const double *q_row, const double *k, const double *v,
                       int b, int h, long long i, int Hq, int Hkv, int Nq, int Nk,
                       int d, int causal, double scale, long long j_lo, long long j_hi,
                       double *s, double *o_row, double *lse_out)
{
    const int kh = h / (Hq / Hkv);
    double m = -INFINITY;
    int any = 0;
    for (long long j = j_lo; j < j_hi; ++j) {
        if (!allowed(i, j, Nq, Nk, causal)) continue;
        const double *k_row = k + (((long long)b * Nk + j) * Hkv + kh) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q_row[c] * k_row[c];
        s[j] = scale * dot;
        if (!any || s[j] > m) m = s[j];
        any = 1;
    }
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    if (!any) { *lse_out = -INFINITY; return; }
    double l = 0.0;
    for (long long j = j_lo; j < j_hi; ++j) {
        if (!allowed(i, j, Nq, Nk, causal)) continue;
        const double w = exp(s[j] - m);
        const double *v_row = v + (((long long)b * Nk + j) * Hkv + kh) * d;
        l += w;
        for (int c = 0; c < d; ++c) o_row[c] += w * v_row[c];
    }
    for (int c = 0; c < d; ++c) o_row[c] /= l;
    *lse_out = m + log(l);
}

int oracle_attn_fwd(const double *q, const double *k, const double *v, double *o,
                    double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                    int causal, double scale)
{
    if (Hkv <= 0 || Hq % Hkv) return 1;
    const long long rows = (long long)B * Hq * Nq;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int b = (int)(r / ((long long)Hq * Nq));
                const int h = (int)((r / Nq) % Hq);
                const long long i = r % Nq;
                const long long qo = (((long long)b * Nq + i) * Hq + h) * d;
                attend_row(q + qo, k, v, b, h, i, Hq, Hkv, Nq, Nk, d, causal, scale, 0, Nk, s,
                           o + qo, lse + r);
            }
            free(s);
        }
    }
    return err;
}

/* The definition restricted to the keys [k0, k1) (clipped to [0, Nk)); the
 * causal rule keeps its absolute form j <= i + (Nk - Nq).  Rows with no
 * allowed key in the window get O = 0, LSE = -inf. */
int oracle_attn_fwd_window(const double *q, const double *k, const double *v, double *o,
                           double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           int causal, double scale, long long k0, long long k1)
{
    if (Hkv <= 0 || Hq % Hkv) return 1;
    if (k0 < 0) k0 = 0;
    if (k1 > Nk) k1 = Nk;
    const long long rows = (long long)B * Hq * Nq;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int b = (int)(r / ((long long)Hq * Nq));
                const int h = (int)((r / Nq) % Hq);
                const long long i = r % Nq;
                const long long qo = (((long long)b * Nq + i) * Hq + h) * d;
                attend_row(q + qo, k, v, b, h, i, Hq, Hkv, Nq, Nk, d, causal, scale, k0, k1, s,
                           o + qo, lse + r);
            }
            free(s);
        }
    }
    return err;
}

/* Merge S partial results of R rows: o_parts[s*R*d + r*d + c], lse_parts[s*R + r]
 * (natural log; -inf marks a window with no allowed key).  Writes o[r*d + c],
 * lse[r]: LSE = ln sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s, computed
 * with the largest LSE_s factored out; a row with every LSE_s = -inf gets
 * O = 0, LSE = -inf. */
int oracle_combine(const double *o_parts, const double *lse_parts, int S, long long R, int d,
                   double *o, double *lse)
{
    if (S < 1 || R < 0 || d < 1) return 1;
    for (long long r = 0; r < R; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_parts[(long long)s * R + r] > m) m = lse_parts[(long long)s * R + r];
        double *o_row = o + r * d;
        for (int c = 0; c < d; ++c) o_row[c] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double wsum = 0.0;
        for (int s = 0; s < S; ++s) {
            const double ls = lse_parts[(long long)s * R + r];
            if (ls == -INFINITY) continue;
            const double w = exp(ls - m);
            const double *src = o_parts + ((long long)s * R + r) * d;
            wsum += w;
            for (int c = 0; c < d; ++c) o_row[c] += w * src[c];
        }
        for (int c = 0; c < d; ++c) o_row[c] /= wsum;
        lse[r] = m + log(wsum);
    }
    return 0;
}

/* rows[n] = flattened (b*Hq + h)*Nq + i; outputs o[n*d + c], lse[n]. */
int oracle_attn_fwd_rows(const double *q, const double *k, const double *v, double *o,
                         double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         int causal, double scale, const long long *rows,
                         long long n_rows)
{
    if (Hkv <= 0 || Hq % Hkv) return 1;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long long n = 0; n < n_rows; ++n) {
                const long long r = rows[n];
                if (r < 0 || r >= (long long)B * Hq * Nq) {
#pragma omp atomic write
                    err = 3;
                    continue;
                }
                const int b = (int)(r / ((long long)Hq * Nq));
                const int h = (int)((r / Nq) % Hq);
                const long long i = r % Nq;
                const long long qo = (((long long)b * Nq + i) * Hq + h) * d;
                attend_row(q + qo, k, v, b, h, i, Hq, Hkv, Nq, Nk, d, causal, scale, 0, Nk, s,
                           o + n * d, lse + n);
            }
            free(s);
        }
    }
    return err;
}

/*
 * Online softmax over key blocks of size `block`.  Per row it keeps a
 * reference max m, a running sum l of exp(s - m) and an unnormalised output
 * acc.  When a block's max exceeds m by more than tau (natural-log units;
 * tau = 0 is the eager recurrence), m moves to the block max and l, acc are
 * multiplied by exp(m_old - m_new).  The final output is acc / l and the
 * LSE is m + ln l.
 */
int oracle_attn_online(const double *q, const double *k, const double *v, double *o,
                       double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       int causal, double scale, int block, double tau,
                       long long *n_rescales)
{
    if (Hkv <= 0 || Hq % Hkv || block <= 0) return 1;
    const long long rows = (long long)B * Hq * Nq;
    long long rescales = 0;
    int err = 0;
#pragma omp parallel reduction(+ : rescales)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)block);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s || !acc) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int b = (int)(r / ((long long)Hq * Nq));
                const int h = (int)((r / Nq) % Hq);
                const long long i = r % Nq;
                const int kh = h / (Hq / Hkv);
                const double *q_row = q + (((long long)b * Nq + i) * Hq + h) * d;
                double m = -INFINITY, l = 0.0;
                for (int c = 0; c < d; ++c) acc[c] = 0.0;
                for (long long j0 = 0; j0 < Nk; j0 += block) {
                    double m_blk = -INFINITY;
                    int any = 0;
                    for (int jj = 0; jj < block && j0 + jj < Nk; ++jj) {
                        const long long j = j0 + jj;
                        if (!allowed(i, j, Nq, Nk, causal)) continue;
                        const double *k_row = k + (((long long)b * Nk + j) * Hkv + kh) * d;
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c) dot += q_row[c] * k_row[c];
                        s[jj] = scale * dot;
                        if (!any || s[jj] > m_blk) m_blk = s[jj];
                        any = 1;
                    }
                    if (!any) continue;
                    if (m == -INFINITY || m_blk > m + tau) {
                        const double f = (m == -INFINITY) ? 0.0 : exp(m - m_blk);
                        l *= f;
                        for (int c = 0; c < d; ++c) acc[c] *= f;
                        if (m != -INFINITY) rescales += 1;
                        m = m_blk;
                    }
                    for (int jj = 0; jj < block && j0 + jj < Nk; ++jj) {
                        const long long j = j0 + jj;
                        if (!allowed(i, j, Nq, Nk, causal)) continue;
                        const double w = exp(s[jj] - m);
                        const double *v_row = v + (((long long)b * Nk + j) * Hkv + kh) * d;
                        l += w;
                        for (int c = 0; c < d; ++c) acc[c] += w * v_row[c];
                    }
                }
                double *o_row = o + (((long long)b * Nq + i) * Hq + h) * d;
                if (m == -INFINITY) {
                    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
                    lse[r] = -INFINITY;
                } else {
                    for (int c = 0; c < d; ++c) o_row[c] = acc[c] / l;
                    lse[r] = m + log(l);
                }
            }
        }
        free(s);
        free(acc);
    }
    if (n_rescales) *n_rescales = rescales;
    return err;
}

/*
 * Brute force for tiny inputs (Nk <= 64): long double, the full score
 * matrix materialised, and each weight formed as p_j = 1 / sum_k exp(s_k - s_j)
 * over allowed k (no max subtraction).  LSE = s_j0 + ln sum_k exp(s_k - s_j0)
 * with j0 the first allowed key.
 */
int oracle_attn_bruteforce(const double *q, const double *k, const double *v, double *o,
                           double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           int causal, double scale)
{
    if (Hkv <= 0 || Hq % Hkv || Nk > 64 || d > 512) return 1;
    long double S[64];
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int kh = h / (Hq / Hkv);
            for (int i = 0; i < Nq; ++i) {
                const double *q_row = q + (((long long)b * Nq + i) * Hq + h) * d;
                double *o_row = o + (((long long)b * Nq + i) * Hq + h) * d;
                int first = -1;
                for (int j = 0; j < Nk; ++j) {
                    const double *k_row = k + (((long long)b * Nk + j) * Hkv + kh) * d;
                    long double dot = 0.0L;
                    for (int c = 0; c < d; ++c) dot += (long double)q_row[c] * k_row[c];
                    S[j] = (long double)scale * dot;
                    if (first < 0 && allowed(i, j, Nq, Nk, causal)) first = j;
                }
                for (int c = 0; c < d; ++c) o_row[c] = 0.0;
                const long long lse_idx = ((long long)b * Hq + h) * Nq + i;
                if (first < 0) { lse[lse_idx] = -INFINITY; continue; }
                long double out[512];
                for (int c = 0; c < d; ++c) out[c] = 0.0L;
                for (int j = 0; j < Nk; ++j) {
                    if (!allowed(i, j, Nq, Nk, causal)) continue;
                    long double den = 0.0L;
                    for (int kk = 0; kk < Nk; ++kk)
                        if (allowed(i, kk, Nq, Nk, causal)) den += expl(S[kk] - S[j]);
                    const long double p = 1.0L / den;
                    const double *v_row = v + (((long long)b * Nk + j) * Hkv + kh) * d;
                    for (int c = 0; c < d; ++c) out[c] += p * v_row[c];
                }
                for (int c = 0; c < d; ++c) o_row[c] = (double)out[c];
                long double z = 0.0L;
                for (int kk = 0; kk < Nk; ++kk)
                    if (allowed(i, kk, Nq, Nk, causal)) z += expl(S[kk] - S[first]);
                lse[lse_idx] = (double)(S[first] + logl(z));
            }
        }
    return 0;
}

/* Elementwise causal/bounds mask as bytes: mask[i*Nk + j] = allowed(i, j). */
void oracle_mask(int Nq, int Nk, int causal, unsigned char *mask)
{
    for (long long i = 0; i < Nq; ++i)
        for (long long j = 0; j < Nk; ++j)
            mask[i * Nk + j] = (unsigned char)allowed(i, j, Nq, Nk, causal);
}

/*
 * M = diag(signs) * H_d / sqrt(d), with the Sylvester Hadamard matrix
 * H_d[r][c] = (-1)^popcount(r & c); d must be a power of two.  Row-major
 * d x d.  A row vector x is rotated as x M.
 */
int oracle_hadamard(int d, const double *signs, double *M)
{
    if (d <= 0 || (d & (d - 1))) return 1;
    const double inv = 1.0 / sqrt((double)d);
    for (int r = 0; r < d; ++r)
        for (int c = 0; c < d; ++c) {
            const int par = __builtin_popcount((unsigned)(r & c)) & 1;
            M[(long long)r * d + c] = signs[r] * (par ? -1.0 : 1.0) * inv;
        }
    return 0;
}

/* Rotate n rows of length d: Y = X M (plain triple loop). */
int oracle_rotate_rows(const double *X, long long n, int d, const double *M, double *Y)
{
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < n; ++r)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += X[r * d + t] * M[(long long)t * d + c];
            Y[r * d + c] = acc;
        }
    return 0;
}

/* OCP FP8 E4M3 (fn): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
 * Exponent field 0: subnormal m * 2^-9.  S.1111.111 is NaN; no infinities. */
double oracle_e4m3_decode(unsigned code)
{
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double val;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) val = ldexp((double)m, -9);
    else val = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -val : val;
}

/* Round to nearest E4M3 value, ties to the even code, saturating to +-448.
 * The non-negative finite codes 0x00..0x7E have increasing values, so the
 * code just below |x| is found by bisection over that ordered list; the
 * result is then the nearer of it and its successor (even code on a tie). */
unsigned oracle_e4m3_encode(double x)
{
    if (isnan(x)) return 0x7F;
    const unsigned sign = signbit(x) ? 0x80u : 0u;
    const double a = fabs(x);
    if (a >= 448.0) return sign | 0x7Eu;
    unsigned lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        const unsigned mid = (lo + hi) / 2;
        if (oracle_e4m3_decode(mid) <= a) lo = mid; else hi = mid;
    }
    const double vlo = oracle_e4m3_decode(lo), vhi = oracle_e4m3_decode(hi);
    if (vlo == a) return sign | lo;
    const double dlo = a - vlo, dhi = vhi - a;
    unsigned pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = (lo & 1u) ? hi : lo;
    return sign | pick;
}

/* Per-tensor FP8 quantisation as fp32 arithmetic: inv = 448 / amax and
 * y = x * inv, each one correctly rounded fp32 operation, then E4M3 encode.
 * (page "FlashAttention-3 — 闪电注意力-3", section 3: quantise after the
 * rotation; the per-tensor scale is descale = amax / 448.) */
void oracle_quant_e4m3_f32(const float *x, long long n, float amax, unsigned char *out)
{
    const float inv = 448.0f / amax;
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; ++i) {
        const float y = x[i] * inv;
        out[i] = (unsigned char)oracle_e4m3_encode((double)y);
    }
}

void oracle_e4m3_encode_array(const double *x, long long n, unsigned char *out)
{
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; ++i) out[i] = (unsigned char)oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const unsigned char *codes, long long n, double *out)
{
    for (long long i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(codes[i]);
}

/* D[m, n] = sum_k A[m, k] * B[k, n] + C[m, n] (C may be NULL: no addition).
 * Plain fp64 sums in increasing k. */
int oracle_gemm_add(const double *a, const double *b, const double *c, double *d,
                    long long M, long long N, long long K)
{
    if (M < 0 || N < 0 || K < 0) return 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long m = 0; m < M; ++m) {
        double *d_row = d + m * N;
        for (long long n = 0; n < N; ++n) d_row[n] = c ? c[m * N + n] : 0.0;
        for (long long k = 0; k < K; ++k) {
            const double x = a[m * K + k];
            const double *b_row = b + k * N;
            for (long long n = 0; n < N; ++n) d_row[n] += x * b_row[n];
        }
    }
    return 0;
}
