/*
 * CPU oracle for the Hybrid Linear Temporal Attention operator.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call this
 * file: only the tests, the package's smoke check and the benchmark's CPU-baseline leg
 * use it. It shares no code, header or constant with the CUDA library.
 *
 * What it computes, straight from the definitions and nothing cleverer:
 *
 *   Sliding-window attention (SWA) and dilated sliding-window attention (DSWA): the
 *   Kairos abstract (chatpaper.ai page, item (2)) and the zhichai.net blog (section 2.2,
 *   "Maintain the world") name the three branches: sliding windows capture local
 *   dynamics, dilated sliding windows mid-range dependencies. Here a query token in
 *   frame f attends with an explicit, max-subtracted softmax to every token of its key
 *   frames; SWA's key frames are max(0, f-w+1) .. f, DSWA's are f, f-r, ..., f-r(w-1)
 *   (taps below frame 0 are dropped). The softmax is the plain definition (llm-atlas
 *   long-context explainer, section 03 "Flash Attention": exact attention is softmax
 *   over all valid query-key pairs, whatever the tiling).
 *
 *   Gated delta rule (GDN): the persistent global memory of the same abstract. The
 *   related-papers analysis (zhaifeiyue.github.io, row A and the Kimi K2 paragraph)
 *   writes its decay term S_t = alpha_t S_{t-1} + ...; the long-context explainer
 *   (section 06 "Finite-state memory") describes the delta rule as "erase the old
 *   association aligned with the key, then write the true value", with a gate that
 *   forgets first. The full update used here is the Gated DeltaNet form
 *       S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,     o_t = S_t q_t,
 *   token by token in sequence order, S a d x d matrix (rows: value dimension, columns:
 *   key dimension), the output read after the update.
 *
 * Precision: inputs are float32 arrays (bf16 inputs are exactly representable); every
 * sum, product, exponential and state element is double precision.
 *
 * Parity status: every function here is pinned by tests that do not re-type its
 * formula (brute-force full attention, closed forms, contraction and retrieval
 * invariants; for the E4M3 codec and quantisers, PyTorch's float8_e4m3fn conversion,
 * the round-to-nearest reconstruction bound and lossless cases; for the rotary embedding,
 * the complex-exponential form, the relative-position (Toeplitz) property, norms and the
 * inverse); see tests/test_oracle_pins.py, tests/test_oracle_fp8_pins.py and
 * tests/test_oracle_rope_pins.py.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Key frames of a query in frame f, in increasing order. Returns the count. */
static int swa_key_frames(int f, int w, int *out)
{
    int lo = f - w + 1;
    if (lo < 0) lo = 0;
    int n = 0;
    for (int fk = lo; fk <= f; ++fk) out[n++] = fk;
    return n;
}

static int dswa_key_frames(int f, int w, int r, int *out)
{
    /* taps f - r*i, i = w-1 .. 0, kept only when >= 0; listed in increasing order */
    int n = 0;
    for (int i = w - 1; i >= 0; --i) {
        long fk = (long)f - (long)r * i;
        if (fk >= 0) out[n++] = (int)fk;
    }
    return n;
}

/* Explicit softmax attention of one query row over the tokens of the listed frames. */
static void softmax_row(const float *qrow, const float *K, const float *V, int N, int d,
                        const int *frames, int nf, double scale, double *z, double *out)
{
    int nk = nf * N;
    double m = -INFINITY;
    for (int i = 0; i < nf; ++i) {
        for (int n = 0; n < N; ++n) {
            const float *krow = K + ((long)frames[i] * N + n) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += (double)qrow[c] * (double)krow[c];
            s *= scale;
            z[(long)i * N + n] = s;
            if (s > m) m = s;
        }
    }
    double den = 0.0;
    for (int j = 0; j < nk; ++j) {
        z[j] = exp(z[j] - m);
        den += z[j];
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int i = 0; i < nf; ++i) {
        for (int n = 0; n < N; ++n) {
            const float *vrow = V + ((long)frames[i] * N + n) * d;
            double p = z[(long)i * N + n];
            for (int c = 0; c < d; ++c) out[c] += p * (double)vrow[c];
        }
    }
    for (int c = 0; c < d; ++c) out[c] /= den;
}

/*
 * Shared driver of the two windowed branches.
 * q, k, v: [BH][L][d] float32, L = T*N. Output o: double.
 * rows == NULL: every row, o is [BH][L][d].
 * rows != NULL: nrows flat indices bh*L + l, o is [nrows][d].
 */
static int window_attention(const float *q, const float *k, const float *v, double *o,
                            long BH, int T, int N, int d, int w, int r, int dilated,
                            double scale, const long *rows, long nrows)
{
    if (BH <= 0 || T <= 0 || N <= 0 || d <= 0 || w <= 0 || r <= 0) return 1;
    long L = (long)T * N;
    long total = rows ? nrows : BH * L;
    int err = 0;
#pragma omp parallel
    {
        int *frames = (int *)malloc(sizeof(int) * (size_t)w);
        double *z = (double *)malloc(sizeof(double) * (size_t)w * (size_t)N);
        if (!frames || !z) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long it = 0; it < total; ++it) {
                long flat = rows ? rows[it] : it;
                long bh = flat / L, l = flat % L;
                if (bh < 0 || bh >= BH) continue;
                int f = (int)(l / N);
                int nf = dilated ? dswa_key_frames(f, w, r, frames) : swa_key_frames(f, w, frames);
                const float *K = k + bh * L * d;
                const float *V = v + bh * L * d;
                softmax_row(q + flat * d, K, V, N, d, frames, nf, scale, z, o + it * d);
            }
        }
        free(frames);
        free(z);
    }
    return err;
}

int oracle_swa(const float *q, const float *k, const float *v, double *o,
               long BH, int T, int N, int d, int w, double scale,
               const long *rows, long nrows)
{
    return window_attention(q, k, v, o, BH, T, N, d, w, 1, 0, scale, rows, nrows);
}

int oracle_dswa(const float *q, const float *k, const float *v, double *o,
                long BH, int T, int N, int d, int w, int r, double scale,
                const long *rows, long nrows)
{
    return window_attention(q, k, v, o, BH, T, N, d, w, r, 1, scale, rows, nrows);
}

/*
 * Gated delta rule, token by token.
 * q, k, v: [BH][L][d] float32; a, b: [BH][L] float32 gates.
 * S0: [BH][d][d] double or NULL (zero state). o: [BH][L][d] double.
 * S_out: [BH][d][d] double or NULL. S_hist: [BH][L][d][d] double or NULL (every S_t,
 * for small invariant checks).
 */
int oracle_gdn(const float *q, const float *k, const float *v, const float *a,
               const float *b, const double *S0, double *o, double *S_out,
               double *S_hist, long BH, long L, int d)
{
    if (BH <= 0 || L < 0 || d <= 0) return 1;
    int err = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
        double *Sk = (double *)malloc(sizeof(double) * (size_t)d);
        if (!S || !Sk) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                if (S0) memcpy(S, S0 + bh * d * d, sizeof(double) * (size_t)d * d);
                else memset(S, 0, sizeof(double) * (size_t)d * d);
                for (long t = 0; t < L; ++t) {
                    const float *kt = k + (bh * L + t) * d;
                    const float *vt = v + (bh * L + t) * d;
                    const float *qt = q + (bh * L + t) * d;
                    double at = a[bh * L + t], bt = b[bh * L + t];
                    /* S k_t */
                    for (int i = 0; i < d; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += S[(long)i * d + j] * (double)kt[j];
                        Sk[i] = s;
                    }
                    /* S <- a S (I - b k k^T) + b v k^T = a (S - b (S k) k^T) + b v k^T */
                    for (int i = 0; i < d; ++i) {
                        for (int j = 0; j < d; ++j) {
                            double kj = (double)kt[j];
                            S[(long)i * d + j] = at * (S[(long)i * d + j] - bt * Sk[i] * kj)
                                                 + bt * (double)vt[i] * kj;
                        }
                    }
                    /* o_t = S_t q_t */
                    double *ot = o + (bh * L + t) * d;
                    for (int i = 0; i < d; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += S[(long)i * d + j] * (double)qt[j];
                        ot[i] = s;
                    }
                    if (S_hist)
                        memcpy(S_hist + (bh * L + t) * d * d, S, sizeof(double) * (size_t)d * d);
                }
                if (S_out) memcpy(S_out + bh * d * d, S, sizeof(double) * (size_t)d * d);
            }
        }
        free(S);
        free(Sk);
    }
    return err;
}

/*
 * GDN heads from raw inputs: the prologue upstream of the recurrence, then the recurrence.
 * The delta rule's erase step is a contraction only for unit keys (researchpapers.dev
 * summary, Theorem 2: ||I - b k k^T|| <= 1 needs ||k|| = 1 and b in [0, 1]), so the raw q and
 * k of a token are scaled to unit L2 norm (a zero vector stays zero); the gates are
 *     a_t = exp(-c * softplus(x_t)) in (0, 1],   b_t = sigmoid(y_t) in (0, 1),
 * softplus(x) = log(1 + e^x) evaluated without overflow. Everything in double precision;
 * the recurrence is the one of oracle_gdn, repeated here on the double inputs.
 */
int oracle_gdn_raw(const float *q, const float *k, const float *v, const float *x,
                   const float *y, double c, const double *S0, double *o, double *S_out,
                   long BH, long L, int d)
{
    if (BH <= 0 || L < 0 || d <= 0) return 1;
    int err = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
        double *Sk = (double *)malloc(sizeof(double) * (size_t)d);
        double *qn = (double *)malloc(sizeof(double) * (size_t)d);
        double *kn = (double *)malloc(sizeof(double) * (size_t)d);
        if (!S || !Sk || !qn || !kn) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                if (S0) memcpy(S, S0 + bh * d * d, sizeof(double) * (size_t)d * d);
                else memset(S, 0, sizeof(double) * (size_t)d * d);
                for (long t = 0; t < L; ++t) {
                    const float *kt = k + (bh * L + t) * d;
                    const float *vt = v + (bh * L + t) * d;
                    const float *qt = q + (bh * L + t) * d;
                    double qq = 0.0, kk = 0.0;
                    for (int j = 0; j < d; ++j) {
                        qq += (double)qt[j] * (double)qt[j];
                        kk += (double)kt[j] * (double)kt[j];
                    }
                    const double qs = qq > 0.0 ? 1.0 / sqrt(qq) : 0.0;
                    const double ks = kk > 0.0 ? 1.0 / sqrt(kk) : 0.0;
                    for (int j = 0; j < d; ++j) {
                        qn[j] = (double)qt[j] * qs;
                        kn[j] = (double)kt[j] * ks;
                    }
                    const double xt = x[bh * L + t], yt = y[bh * L + t];
                    const double sp = xt > 0.0 ? xt + log1p(exp(-xt)) : log1p(exp(xt));
                    const double at = exp(-c * sp);
                    const double bt = 1.0 / (1.0 + exp(-yt));
                    for (int i = 0; i < d; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += S[(long)i * d + j] * kn[j];
                        Sk[i] = s;
                    }
                    for (int i = 0; i < d; ++i)
                        for (int j = 0; j < d; ++j)
                            S[(long)i * d + j] = at * (S[(long)i * d + j] - bt * Sk[i] * kn[j])
                                                 + bt * (double)vt[i] * kn[j];
                    double *ot = o + (bh * L + t) * d;
                    for (int i = 0; i < d; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += S[(long)i * d + j] * qn[j];
                        ot[i] = s;
                    }
                }
                if (S_out) memcpy(S_out + bh * d * d, S, sizeof(double) * (size_t)d * d);
            }
        }
        free(S);
        free(Sk);
        free(qn);
        free(kn);
    }
    return err;
}

/*
 * FP8 attention inputs. The related-papers analysis (zhaifeiyue.github.io, row C1 and the
 * paragraphs on deployment quantisation) says the deployed model quantises attention to FP8
 * but gives no method. The format used here is the OCP 8-bit floating point E4M3 encoding
 * (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 * subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities; largest finite value 448).
 *
 * Quantisation with one fp32 scale per block of rows (or per channel): amax is the largest
 * magnitude in the block, every element x becomes the E4M3 code nearest to x * (448/amax)
 * (ties to the even code, magnitudes beyond 448 saturate to 448), and the stored scale is
 * amax/448, so that x ~ decode(code) * scale. The three fp32 operations (448/amax, the
 * product, amax/448) are single IEEE roundings, in this order, on both sides of a parity
 * test: the codes are then integers both sides must agree on bit for bit.
 */
double oracle_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* The non-negative finite E4M3 values, codes 0x00 .. 0x7E, increasing with the code. */
static void e4m3_table(double *tab)
{
    for (int c = 0; c < 0x7F; ++c) tab[c] = oracle_e4m3_decode(c);
}

/* Nearest code by exhaustive search over the 127 non-negative finite values; of two equally
 * near values (always neighbours) the even code wins; the sign bit is the sign of y. */
static int e4m3_encode_tab(const double *tab, float y)
{
    if (isnan(y)) return 0x7F;
    int sign = signbit(y) ? 0x80 : 0;
    if (isinf(y)) return sign | 0x7E;
    double a = fabs((double)y), bd = INFINITY;
    int best = 0;
    for (int c = 0; c < 0x7F; ++c) {
        double dd = fabs(tab[c] - a);
        if (dd < bd || (dd == bd && (c & 1) == 0)) {
            bd = dd;
            best = c;
        }
    }
    return sign | best;
}

int oracle_e4m3_encode(float y)
{
    double tab[0x7F];
    e4m3_table(tab);
    return e4m3_encode_tab(tab, y);
}

/* One block: rows r0 .. r0+nr-1 of a [L][d] head (optionally minus a per-channel shift),
 * columns c0 .. c0+nc-1 (a single channel when nc == 1 and the block runs down a column). */
static float quantize_block(const double *tab, const float *x, const float *shift, long r0,
                            long nr, int d, int c0, int nc, unsigned char *x8)
{
    float amax = 0.0f;
    for (long r = r0; r < r0 + nr; ++r)
        for (int c = c0; c < c0 + nc; ++c) {
            float v = x[r * d + c];
            if (shift) v = v - shift[c];
            float a = fabsf(v);
            if (a > amax) amax = a;
        }
    float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
    for (long r = r0; r < r0 + nr; ++r)
        for (int c = c0; c < c0 + nc; ++c) {
            float v = x[r * d + c];
            if (shift) v = v - shift[c];
            float y = v * inv;
            x8[r * d + c] = (unsigned char)e4m3_encode_tab(tab, y);
        }
    return amax / 448.0f;
}

/*
 * Row-block quantisation. x: [BH][L][d] float32; shift: [BH][d] or NULL (subtracted from
 * every row first, in fp32). Each head is cut into frames of frame_rows rows (the last frame
 * may be short) and each frame into runs of block_rows rows (the last run of a frame may be
 * short); a block never spans two frames. Output codes x8: [BH][L][d]; scales:
 * [BH][nframes][nb], nframes = ceil(L / frame_rows), nb = ceil(frame_rows / block_rows).
 */
int oracle_fp8_quantize_rows(const float *x, const float *shift, long BH, long L, int d,
                             long frame_rows, int block_rows, unsigned char *x8, float *scale)
{
    if (BH < 0 || L < 0 || d < 1 || frame_rows < 1 || block_rows < 1) return 1;
    double tab[0x7F];
    e4m3_table(tab);
    long nf = (L + frame_rows - 1) / frame_rows, nb = (frame_rows + block_rows - 1) / block_rows;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (long bh = 0; bh < BH; ++bh)
        for (long f = 0; f < nf; ++f) {
            long fr0 = f * frame_rows, fr1 = fr0 + frame_rows < L ? fr0 + frame_rows : L;
            for (long j = 0; j < nb; ++j) {
                long r0 = fr0 + j * block_rows;
                long nr = r0 >= fr1 ? 0 : (r0 + block_rows < fr1 ? block_rows : fr1 - r0);
                scale[(bh * nf + f) * nb + j] =
                    nr > 0 ? quantize_block(tab, x + bh * L * d, shift ? shift + bh * d : NULL,
                                            r0, nr, d, 0, d, x8 + bh * L * d)
                           : 0.0f;
            }
        }
    return 0;
}

/*
 * Per-channel quantisation: one scale per (head, channel) over all L rows of the head.
 * x: [BH][L][d] float32 -> x8: [BH][L][d] codes, scale: [BH][d].
 */
int oracle_fp8_quantize_channels(const float *x, long BH, long L, int d, unsigned char *x8,
                                 float *scale)
{
    if (BH < 0 || L < 0 || d < 1) return 1;
    double tab[0x7F];
    e4m3_table(tab);
#pragma omp parallel for collapse(2)
    for (long bh = 0; bh < BH; ++bh)
        for (int c = 0; c < d; ++c)
            scale[bh * d + c] = quantize_block(tab, x + bh * L * d, NULL, 0, L, d, c, 1, x8 + bh * L * d);
    return 0;
}

/*
 * Backward pass of the windowed attention (training: the backbone is trained from scratch,
 * related-papers analysis row E). Reverse-mode derivative of o_i = sum_j p_ij v_j,
 * p_ij = softmax_j(scale q_i . k_j) over the keys of row i's window frames, for a given
 * upstream gradient dO, written out per query row:
 *   dP_ij = dO_i . v_j,  D_i = sum_j p_ij dP_ij,  dS_ij = p_ij (dP_ij - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j += scale dS_ij q_i,  dv_j += p_ij dO_i.
 * q, k, v, dO: [BH][L][d] float32; dq, dk, dv: [BH][L][d] double (overwritten).
 * Heads run in parallel; the rows of a head run in order (dk, dv accumulate).
 */
static int window_backward(const float *q, const float *k, const float *v, const float *dO,
                           double *dq, double *dk, double *dv, long BH, int T, int N, int d,
                           int w, int r, int dilated, double scale)
{
    if (BH <= 0 || T <= 0 || N <= 0 || d <= 0 || w <= 0 || r <= 0) return 1;
    long L = (long)T * N;
    int err = 0;
    for (long i = 0; i < BH * L * d; ++i) dq[i] = dk[i] = dv[i] = 0.0;
#pragma omp parallel
    {
        int *frames = (int *)malloc(sizeof(int) * (size_t)w);
        double *pz = (double *)malloc(sizeof(double) * (size_t)w * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)w * (size_t)N);
        if (!frames || !pz || !dp) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                const float *Q = q + bh * L * d, *K = k + bh * L * d, *V = v + bh * L * d;
                const float *G = dO + bh * L * d;
                double *DQ = dq + bh * L * d, *DK = dk + bh * L * d, *DV = dv + bh * L * d;
                for (long l = 0; l < L; ++l) {
                    int f = (int)(l / N);
                    int nf = dilated ? dswa_key_frames(f, w, r, frames) : swa_key_frames(f, w, frames);
                    int nk = nf * N;
                    double m = -INFINITY;
                    for (int i = 0; i < nf; ++i)
                        for (int n = 0; n < N; ++n) {
                            long kr = (long)frames[i] * N + n;
                            double s = 0.0;
                            for (int c = 0; c < d; ++c) s += (double)Q[l * d + c] * (double)K[kr * d + c];
                            s *= scale;
                            pz[(long)i * N + n] = s;
                            if (s > m) m = s;
                        }
                    double den = 0.0;
                    for (int j = 0; j < nk; ++j) {
                        pz[j] = exp(pz[j] - m);
                        den += pz[j];
                    }
                    double Dsum = 0.0;
                    for (int i = 0; i < nf; ++i)
                        for (int n = 0; n < N; ++n) {
                            long j = (long)i * N + n, kr = (long)frames[i] * N + n;
                            pz[j] /= den;
                            double g = 0.0;
                            for (int c = 0; c < d; ++c) g += (double)G[l * d + c] * (double)V[kr * d + c];
                            dp[j] = g;
                            Dsum += pz[j] * g;
                        }
                    for (int i = 0; i < nf; ++i)
                        for (int n = 0; n < N; ++n) {
                            long j = (long)i * N + n, kr = (long)frames[i] * N + n;
                            double ds = pz[j] * (dp[j] - Dsum);
                            for (int c = 0; c < d; ++c) {
                                DQ[l * d + c] += scale * ds * (double)K[kr * d + c];
                                DK[kr * d + c] += scale * ds * (double)Q[l * d + c];
                                DV[kr * d + c] += pz[j] * (double)G[l * d + c];
                            }
                        }
                }
            }
        }
        free(frames);
        free(pz);
        free(dp);
    }
    return err;
}

int oracle_window_bwd(const float *q, const float *k, const float *v, const float *dO,
                      double *dq, double *dk, double *dv, long BH, int T, int N, int d, int w,
                      int r, double scale)
{
    return window_backward(q, k, v, dO, dq, dk, dv, BH, T, N, d, w, r, r > 1, scale);
}

/* Log-sum-exp of each query row's scaled scores over its window keys (natural log): the
 * softmax normaliser the backward pass reuses. q, k: [BH][L][d] float32; lse: [BH][L]. */
int oracle_window_lse(const float *q, const float *k, double *lse, long BH, int T, int N, int d,
                      int w, int r, double scale)
{
    if (BH <= 0 || T <= 0 || N <= 0 || d <= 0 || w <= 0 || r <= 0) return 1;
    long L = (long)T * N;
    int err = 0;
#pragma omp parallel
    {
        int *frames = (int *)malloc(sizeof(int) * (size_t)w);
        double *z = (double *)malloc(sizeof(double) * (size_t)w * (size_t)N);
        if (!frames || !z) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long it = 0; it < BH * L; ++it) {
                long bh = it / L, l = it % L;
                int f = (int)(l / N);
                int nf = r > 1 ? dswa_key_frames(f, w, r, frames) : swa_key_frames(f, w, frames);
                const float *K = k + bh * L * d;
                double m = -INFINITY;
                for (int i = 0; i < nf; ++i)
                    for (int n = 0; n < N; ++n) {
                        const float *krow = K + ((long)frames[i] * N + n) * d;
                        double s = 0.0;
                        for (int c = 0; c < d; ++c) s += (double)q[it * d + c] * (double)krow[c];
                        s *= scale;
                        z[(long)i * N + n] = s;
                        if (s > m) m = s;
                    }
                double den = 0.0;
                for (int j = 0; j < nf * N; ++j) den += exp(z[j] - m);
                lse[it] = m + log(den);
            }
        }
        free(frames);
        free(z);
    }
    return err;
}

/*
 * Backward pass of the gated delta rule: reverse-mode derivative of the token recurrence of
 * oracle_gdn (S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t) for the
 * upstream gradients dO (of every o_t) and dSL (of the final state, or NULL for zero). With
 * G the gradient of the current state, walking t = L-1 .. 0:
 *   G += dO_t q_t^T;  dq_t = S_t^T dO_t;  sk = S_{t-1} k_t;  gk = G k_t;
 *   dv_t = b_t gk;  db_t = gk . (v_t - a_t sk);  da_t = <G, S_{t-1}> - b_t gk . sk;
 *   dk_t = -a_t b_t (S_{t-1}^T gk + G^T sk) + b_t G^T v_t;  G <- a_t (G - b_t gk k_t^T)
 * and dS0 = G at the end. The forward states are recomputed and kept per head.
 * Inputs as oracle_gdn; dq, dk, dv: [BH][L][d], da, db: [BH][L], dS0: [BH][d][d] (or NULL).
 */
int oracle_gdn_bwd(const float *q, const float *k, const float *v, const float *a,
                   const float *b, const double *S0, const float *dO, const double *dSL,
                   double *dq, double *dk, double *dv, double *da, double *db, double *dS0,
                   long BH, long L, int d)
{
    if (BH <= 0 || L < 0 || d <= 0) return 1;
    int err = 0;
    const size_t dd = (size_t)d * d;
#pragma omp parallel
    {
        double *hist = (double *)malloc(sizeof(double) * dd * (size_t)(L + 1));
        double *G = (double *)malloc(sizeof(double) * dd);
        double *sk = (double *)malloc(sizeof(double) * (size_t)d);
        double *gk = (double *)malloc(sizeof(double) * (size_t)d);
        if (!hist || !G || !sk || !gk) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                /* forward: hist[t + 1] = S_t, hist[0] = S0 */
                if (S0) memcpy(hist, S0 + bh * dd, sizeof(double) * dd);
                else memset(hist, 0, sizeof(double) * dd);
                for (long t = 0; t < L; ++t) {
                    const float *kt = k + (bh * L + t) * d, *vt = v + (bh * L + t) * d;
                    double at = a[bh * L + t], bt = b[bh * L + t];
                    const double *Sp = hist + (size_t)t * dd;
                    double *Sn = hist + (size_t)(t + 1) * dd;
                    for (int i = 0; i < d; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += Sp[(long)i * d + j] * (double)kt[j];
                        for (int j = 0; j < d; ++j)
                            Sn[(long)i * d + j] = at * (Sp[(long)i * d + j] - bt * s * (double)kt[j])
                                                  + bt * (double)vt[i] * (double)kt[j];
                    }
                }
                /* backward */
                if (dSL) memcpy(G, dSL + bh * dd, sizeof(double) * dd);
                else memset(G, 0, sizeof(double) * dd);
                for (long t = L - 1; t >= 0; --t) {
                    const long tt = bh * L + t;
                    const float *kt = k + tt * d, *vt = v + tt * d, *qt = q + tt * d;
                    const float *gt = dO + tt * d;
                    double at = a[tt], bt = b[tt];
                    const double *Sp = hist + (size_t)t * dd, *St = hist + (size_t)(t + 1) * dd;
                    for (int i = 0; i < d; ++i)
                        for (int j = 0; j < d; ++j) G[(long)i * d + j] += (double)gt[i] * (double)qt[j];
                    for (int j = 0; j < d; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < d; ++i) s += St[(long)i * d + j] * (double)gt[i];
                        dq[tt * d + j] = s;
                    }
                    double gs = 0.0, gksk = 0.0, dbt = 0.0;
                    for (int i = 0; i < d; ++i) {
                        double s1 = 0.0, s2 = 0.0;
                        for (int j = 0; j < d; ++j) {
                            s1 += Sp[(long)i * d + j] * (double)kt[j];
                            s2 += G[(long)i * d + j] * (double)kt[j];
                            gs += G[(long)i * d + j] * Sp[(long)i * d + j];
                        }
                        sk[i] = s1;
                        gk[i] = s2;
                        gksk += s2 * s1;
                        dbt += s2 * ((double)vt[i] - at * s1);
                        dv[tt * d + i] = bt * s2;
                    }
                    db[tt] = dbt;
                    da[tt] = gs - bt * gksk;
                    for (int j = 0; j < d; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < d; ++i)
                            s += -at * bt * (Sp[(long)i * d + j] * gk[i] + G[(long)i * d + j] * sk[i])
                                 + bt * G[(long)i * d + j] * (double)vt[i];
                        dk[tt * d + j] = s;
                    }
                    for (int i = 0; i < d; ++i)
                        for (int j = 0; j < d; ++j)
                            G[(long)i * d + j] = at * (G[(long)i * d + j] - bt * gk[i] * (double)kt[j]);
                }
                if (dS0) memcpy(dS0 + bh * dd, G, sizeof(double) * dd);
            }
        }
        free(hist);
        free(G);
        free(sk);
        free(gk);
    }
    return err;
}

/*
 * Rotary position embedding (llm-atlas long-context explainer, the position-encoding section:
 * RoPE turns a position into a rotation of Q and K so that their dot product depends only on
 * the relative position). Kairos gives RoPE the local position and the linear path the global
 * one (the related-papers analysis, row B1). Reading used here: 1-D RoPE, the pair
 * (x_{2i}, x_{2i+1}) of a token at position p rotated by the angle p * base^(-2i/d);
 * p = l mod N (the token's index inside its frame) for pos_mode 0, p = l for pos_mode 1;
 * sign = -1 rotates back (the inverse rotation, which is also the map of the gradient).
 * x, y: [BH][L][d].
 */
int oracle_rope(const float *x, double *y, long BH, long L, int N, int d, double base,
                int pos_mode, int sign)
{
    if (d < 2 || d % 2 || (pos_mode == 0 && N < 1) || !(base > 1.0)) return 1;
    for (long bh = 0; bh < BH; ++bh)
        for (long l = 0; l < L; ++l) {
            const double p = pos_mode ? (double)l : (double)(l % N);
            const float *xr = x + (bh * L + l) * d;
            double *yr = y + (bh * L + l) * d;
            for (int i = 0; i < d / 2; ++i) {
                const double ang = sign * p * pow(base, -2.0 * i / d);
                const double c = cos(ang), s = sin(ang);
                const double x0 = xr[2 * i], x1 = xr[2 * i + 1];
                yr[2 * i] = x0 * c - x1 * s;
                yr[2 * i + 1] = x0 * s + x1 * c;
            }
        }
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
