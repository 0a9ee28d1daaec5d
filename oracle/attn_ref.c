/*
 * Plain fp64 CPU oracle for causal grouped-query attention (forward).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (the textbook scaled-dot-product attention that the Tessera
 * pages name as "a FlashAttention forward kernel with online softmax, causal
 * masking, grouped-query attention" -- hysenlabs.com Tessera review, section
 * "The kernel set and its torch fallback"; Tessera README, "What's in it" /
 * "Kernels"; the decoder it serves has "grouped-query attention", README
 * "What's in it" / "Training side"):
 *
 *   G = Hq / Hkv, query head h reads key/value head g = floor(h / G)
 *   J(i) = {0..i} when causal, {0..T-1} otherwise
 *   s_ij   = scale * sum_c Q[b,h,i,c] * K[b,g,j,c]          j in J(i)
 *   m_i    = max_j s_ij
 *   l_i    = sum_j exp(s_ij - m_i)
 *   O[b,h,i,:] = sum_j exp(s_ij - m_i) * V[b,g,j,:] / l_i
 *   LSE[b,h,i] = m_i + ln(l_i)                    (natural log, scaled logits)
 *
 * The FlashAttention tiling and online softmax reach exactly this result up to
 * rounding, so the oracle is the definition written out, one row at a time,
 * with no blocking, fusion or reordering.  Layouts are contiguous row-major:
 * Q, O [B,Hq,T,d]; K, V [B,Hkv,T,d]; LSE [B,Hq,T].
 *
 * The file also holds the backward (dQ, dK, dV given dO), below.
 *
 * Return codes: 0 ok, 1 invalid argument, 2 out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> fp64: a bf16 is the top 16 bits of an IEEE fp32, so widening is exact. */
static double bf16_bits_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One query row against the first n_keys rows of one key/value head.
 * q: [d]; kh, vh: [*, d] (row j at offset j*d); s: scratch of n_keys doubles.
 * Writes o[0..d) and *lse.
 */
static void attend_one_row(const double *q, const double *kh, const double *vh,
                           int64_t n_keys, int d, double scale, double *s,
                           double *o, double *lse)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += q[c] * kh[j * d + c];
        s[j] = scale * dot;
        if (s[j] > m)
            m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        s[j] = exp(s[j] - m); /* unnormalised probability */
        l += s[j];
    }
    for (int c = 0; c < d; ++c)
        o[c] = 0.0;
    for (int64_t j = 0; j < n_keys; ++j)
        for (int c = 0; c < d; ++c)
            o[c] += s[j] * vh[j * d + c];
    for (int c = 0; c < d; ++c)
        o[c] /= l;
    *lse = m + log(l);
}

static int check_shape(int B, int Hq, int Hkv, int T, int d)
{
    if (B < 0 || Hq < 1 || Hkv < 1 || T < 0 || d < 1)
        return 1;
    if (Hq % Hkv != 0)
        return 1;
    return 0;
}

/*
 * Full attention on fp64 inputs.  lse may be NULL.
 */
int oracle_attn_fwd_f64(const double *q, const double *k, const double *v,
                        double *o, double *lse, int B, int Hq, int Hkv, int T,
                        int d, int causal, double scale)
{
    if (check_shape(B, Hq, Hkv, T, d))
        return 1;
    if (B == 0 || T == 0)
        return 0;
    const int G = Hq / Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    if (!s)
        return 2;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            const double *kh = k + ((int64_t)b * Hkv + g) * T * d;
            const double *vh = v + ((int64_t)b * Hkv + g) * T * d;
            for (int i = 0; i < T; ++i) {
                const int64_t row = ((int64_t)b * Hq + h) * T + i;
                const int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)T;
                double lse_i;
                attend_one_row(q + row * d, kh, vh, n_keys, d, scale, s,
                               o + row * d, &lse_i);
                if (lse)
                    lse[row] = lse_i;
            }
        }
    }
    free(s);
    return 0;
}

/*
 * Selected rows of attention on bf16 inputs (raw bf16 bit patterns), widened
 * exactly to fp64 on read.  rows: n_rows triples (b, h, i).  Outputs:
 * o_rows [n_rows, d] and lse_rows [n_rows] in fp64.  Used to check outputs of
 * workloads too large to run through the oracle in full.
 */
int oracle_attn_rows_bf16(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int Hq, int Hkv, int T,
                          int d, int causal, double scale,
                          const int64_t *rows, int64_t n_rows, double *o_rows,
                          double *lse_rows)
{
    if (check_shape(B, Hq, Hkv, T, d))
        return 1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= T)
            return 1;
    }
    if (n_rows == 0)
        return 0;
    const int G = Hq / Hkv;
    double *kh = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *vh = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    if (!kh || !vh || !qi || !s) {
        free(kh); free(vh); free(qi); free(s);
        return 2;
    }
    int64_t cur_b = -1, cur_g = -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        const int64_t g = h / G;
        if (b != cur_b || g != cur_g) { /* widen this key/value head once */
            const int64_t base = (b * Hkv + g) * (int64_t)T * d;
            for (int64_t e = 0; e < (int64_t)T * d; ++e) {
                kh[e] = bf16_bits_to_f64(k[base + e]);
                vh[e] = bf16_bits_to_f64(v[base + e]);
            }
            cur_b = b;
            cur_g = g;
        }
        const int64_t qrow = (b * Hq + h) * (int64_t)T + i;
        for (int c = 0; c < d; ++c)
            qi[c] = bf16_bits_to_f64(q[qrow * d + c]);
        const int64_t n_keys = causal ? i + 1 : (int64_t)T;
        attend_one_row(qi, kh, vh, n_keys, d, scale, s, o_rows + r * d,
                       &lse_rows[r]);
    }
    free(kh); free(vh); free(qi); free(s);
    return 0;
}

/*
 * ------------------------------------------------------------------ backward
 * Gradient of the forward above with respect to Q, K and V, given dO (the
 * gradient of a loss with respect to O; LSE is treated as saved state, not as
 * an output that receives a gradient).  The pages list the attention backward
 * as not yet built; its plain reading is the exact derivative of the forward
 * definition, which the chain rule through the row softmax gives as
 *
 *   P_ij  = exp(s_ij - LSE_i)                  j in J(i)
 *   dV[b,g,j,:] += P_ij * dO[b,h,i,:]          over h in group g and i
 *   dP_ij = <dO[b,h,i,:], V[b,g,j,:]>
 *   D_i   = <dO[b,h,i,:], O[b,h,i,:]>          (= sum_j P_ij dP_ij)
 *   dS_ij = P_ij * (dP_ij - D_i)
 *   dQ[b,h,i,:]  = scale * sum_j dS_ij K[b,g,j,:]
 *   dK[b,g,j,:] += scale * dS_ij * Q[b,h,i,:]  over h in group g and i
 *
 * written out one query row at a time, with no blocking or reordering.
 */

/*
 * Backward of one query row: recomputes the row's scores, probabilities and
 * output, then adds its contributions to dk/dv (the key/value head's [T,d]
 * accumulators) and writes dq[0..d).  s, p: scratch of n_keys doubles;
 * o: scratch of d doubles.
 */
static void backward_one_row(const double *q, const double *dout, const double *kh,
                             const double *vh, int64_t n_keys, int d, double scale,
                             double *s, double *p, double *o, double *dq,
                             double *dkh, double *dvh)
{
    double lse;
    attend_one_row(q, kh, vh, n_keys, d, scale, s, o, &lse);
    /* attend_one_row leaves exp(s_ij - m) in s; recompute the scores */
    for (int64_t j = 0; j < n_keys; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += kh[j * d + c] * q[c];
        s[j] = dot * scale;
    }
    for (int64_t j = 0; j < n_keys; ++j)
        p[j] = exp(s[j] - lse);
    double D = 0.0;
    for (int c = 0; c < d; ++c)
        D += dout[c] * o[c];
    for (int c = 0; c < d; ++c)
        dq[c] = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        double dp = 0.0;
        for (int c = 0; c < d; ++c)
            dp += dout[c] * vh[j * d + c];
        const double ds = p[j] * (dp - D);
        for (int c = 0; c < d; ++c) {
            dvh[j * d + c] += p[j] * dout[c];
            dkh[j * d + c] += scale * ds * q[c];
            dq[c] += scale * ds * kh[j * d + c];
        }
    }
}

/*
 * Full backward on fp64 inputs: q, dout [B,Hq,T,d]; k, v [B,Hkv,T,d].
 * Writes dq [B,Hq,T,d], dk and dv [B,Hkv,T,d].
 */
int oracle_attn_bwd_f64(const double *q, const double *k, const double *v,
                        const double *dout, double *dq, double *dk, double *dv,
                        int B, int Hq, int Hkv, int T, int d, int causal,
                        double scale)
{
    if (check_shape(B, Hq, Hkv, T, d))
        return 1;
    const int64_t nkv = (int64_t)B * Hkv * T * d;
    for (int64_t e = 0; e < nkv; ++e) {
        dk[e] = 0.0;
        dv[e] = 0.0;
    }
    if (B == 0 || T == 0)
        return 0;
    const int G = Hq / Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !p || !o) {
        free(s); free(p); free(o);
        return 2;
    }
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int64_t kv = ((int64_t)b * Hkv + h / G) * T * d;
            for (int i = 0; i < T; ++i) {
                const int64_t row = ((int64_t)b * Hq + h) * T + i;
                const int64_t n_keys = causal ? i + 1 : T; /* keys j <= i */
                backward_one_row(q + row * d, dout + row * d, k + kv, v + kv, n_keys,
                                 d, scale, s, p, o, dq + row * d, dk + kv, dv + kv);
            }
        }
    }
    free(s); free(p); free(o);
    return 0;
}

/*
 * Selected rows of dQ on bf16 inputs (raw bit patterns, widened exactly).
 * rows: n_rows triples (b, h, i); dq_rows [n_rows, d].  A row of dQ needs only
 * its own query row and the key/value head, so workloads too large for the
 * full backward can still be checked row by row.
 */
int oracle_attn_bwd_dq_rows_bf16(const uint16_t *q, const uint16_t *k,
                                 const uint16_t *v, const uint16_t *dout, int B,
                                 int Hq, int Hkv, int T, int d, int causal,
                                 double scale, const int64_t *rows, int64_t n_rows,
                                 double *dq_rows)
{
    if (check_shape(B, Hq, Hkv, T, d))
        return 1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= T)
            return 1;
    }
    if (n_rows == 0)
        return 0;
    const int G = Hq / Hkv;
    const size_t td = (size_t)T * d;
    double *kh = (double *)malloc(sizeof(double) * td);
    double *vh = (double *)malloc(sizeof(double) * td);
    double *dkh = (double *)malloc(sizeof(double) * td); /* discarded */
    double *dvh = (double *)malloc(sizeof(double) * td); /* discarded */
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    double *gi = (double *)malloc(sizeof(double) * (size_t)d);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    if (!kh || !vh || !dkh || !dvh || !qi || !gi || !o || !s || !p) {
        free(kh); free(vh); free(dkh); free(dvh); free(qi); free(gi); free(o);
        free(s); free(p);
        return 2;
    }
    int64_t cur_b = -1, cur_g = -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        const int64_t g = h / G;
        if (b != cur_b || g != cur_g) {
            const int64_t base = (b * Hkv + g) * (int64_t)td;
            for (int64_t e = 0; e < (int64_t)td; ++e) {
                kh[e] = bf16_bits_to_f64(k[base + e]);
                vh[e] = bf16_bits_to_f64(v[base + e]);
            }
            cur_b = b;
            cur_g = g;
        }
        const int64_t qrow = (b * Hq + h) * (int64_t)T + i;
        for (int c = 0; c < d; ++c) {
            qi[c] = bf16_bits_to_f64(q[qrow * d + c]);
            gi[c] = bf16_bits_to_f64(dout[qrow * d + c]);
        }
        const int64_t n_keys = causal ? i + 1 : (int64_t)T;
        memset(dkh, 0, sizeof(double) * (size_t)n_keys * d);
        memset(dvh, 0, sizeof(double) * (size_t)n_keys * d);
        backward_one_row(qi, gi, kh, vh, n_keys, d, scale, s, p, o, dq_rows + r * d,
                         dkh, dvh);
    }
    free(kh); free(vh); free(dkh); free(dvh); free(qi); free(gi); free(o);
    free(s); free(p);
    return 0;
}

/*
 * ------------------------------------------------------------- paged decode
 * One decoding step of attention over a paged key/value cache (the serving
 * engine's "paged-KV" that the pages name; they give no layout, so this
 * library's reading is used): sequence b has seq_lens[b] cached tokens; its
 * token j lives in physical block block_table[b][j / bs] at row j % bs.
 *
 *   q        [B, Hq, d]                         one query row per head
 *   k_cache  [num_blocks, Hkv, bs, d]           v_cache likewise
 *   block_table [B, max_blocks] int32, seq_lens [B] int32
 *   o        [B, Hq, d],  lse [B, Hq]
 *
 * Query head h of sequence b attends to all seq_lens[b] tokens of key/value
 * head g = h / G (no further mask: the newest token is the query's own).
 * seq_lens[b] = 0 gives o = 0 and lse = -inf.  Written out by gathering the
 * sequence's keys and values into a contiguous buffer and applying the
 * forward's definition to the single query row.
 */
int oracle_paged_decode_f64(const double *q, const double *k_cache, const double *v_cache,
                            const int32_t *block_table, const int32_t *seq_lens, int B,
                            int Hq, int Hkv, int d, int bs, int max_blocks, int num_blocks,
                            double scale, double *o, double *lse)
{
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || d < 1 || bs < 1 || max_blocks < 0 ||
        num_blocks < 0)
        return 1;
    const int G = Hq / Hkv;
    int64_t max_len = 0;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || (int64_t)seq_lens[b] > (int64_t)max_blocks * bs)
            return 1;
        for (int64_t j = 0; j < seq_lens[b]; j += bs) {
            const int32_t blk = block_table[(int64_t)b * max_blocks + j / bs];
            if (blk < 0 || blk >= num_blocks)
                return 1;
        }
        if (seq_lens[b] > max_len)
            max_len = seq_lens[b];
    }
    double *kh = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * d);
    double *vh = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    if (!kh || !vh || !s) {
        free(kh); free(vh); free(s);
        return 2;
    }
    for (int b = 0; b < B; ++b) {
        const int64_t n = seq_lens[b];
        for (int g = 0; g < Hkv; ++g) {
            /* gather the sequence's keys and values of head g */
            for (int64_t j = 0; j < n; ++j) {
                const int32_t blk = block_table[(int64_t)b * max_blocks + j / bs];
                const int64_t src = (((int64_t)blk * Hkv + g) * bs + j % bs) * d;
                for (int c = 0; c < d; ++c) {
                    kh[j * d + c] = k_cache[src + c];
                    vh[j * d + c] = v_cache[src + c];
                }
            }
            for (int h = g * G; h < (g + 1) * G; ++h) {
                const int64_t row = (int64_t)b * Hq + h;
                if (n == 0) {
                    for (int c = 0; c < d; ++c)
                        o[row * d + c] = 0.0;
                    lse[row] = -INFINITY;
                    continue;
                }
                attend_one_row(q + row * d, kh, vh, n, d, scale, s, o + row * d, &lse[row]);
            }
        }
    }
    free(kh); free(vh); free(s);
    return 0;
}

/*
 * ----------------------------------------------------------------------------
 * Prologue of the attention block: RMSNorm, and the rotary embedding of the
 * projected queries and keys.
 *
 * The pages' decoder is a transformer with "RMSNorm, RoPE, grouped-query
 * attention and SwiGLU" (Tessera README, "What's in it" / "Training side"),
 * and its kernels include a fused RMSNorm (README "What's in it" / "Kernels";
 * hysenlabs.com review, "The kernel set and its torch fallback").  The pages
 * give no formula; the plain readings written out here are the usual ones:
 *
 *   RMSNorm over the last dimension with a learned weight w:
 *     y[r,c] = x[r,c] / sqrt( (1/dim) sum_c' x[r,c']^2 + eps ) * w[c]
 *
 *   Rotary position embedding of a head vector x (length d, even) at
 *   position p, pairing element i with element i + d/2 (i < d/2):
 *     theta_i = base^(-2i/d),   a = p * theta_i
 *     y[i]       = x[i] cos a - x[i + d/2] sin a
 *     y[i + d/2] = x[i] sin a + x[i + d/2] cos a
 *
 * The projection output is token-major: qkv [B, T, (Hq + 2 Hkv) d], per token
 * the Hq query heads, then the Hkv key heads, then the Hkv value heads, each d
 * wide.  The prologue writes the attention layout: q [B, Hq, T, d] and
 * k [B, Hkv, T, d] rotated, v [B, Hkv, T, d] copied.  positions [B, T] gives
 * each token's position (NULL: p = t).
 */
int oracle_rmsnorm_f64(const double *x, const double *w, int rows, int dim, double eps,
                       double *y)
{
    if (rows < 0 || dim < 1 || !(eps >= 0.0)) return 1;
    for (int r = 0; r < rows; ++r) {
        const double *xr = x + (int64_t)r * dim;
        double *yr = y + (int64_t)r * dim;
        double ss = 0.0;
        for (int c = 0; c < dim; ++c) ss += xr[c] * xr[c];
        const double inv = 1.0 / sqrt(ss / dim + eps);
        for (int c = 0; c < dim; ++c) yr[c] = xr[c] * inv * w[c];
    }
    return 0;
}

/* Rotate one head vector x (length d) at position p into y. */
static void rope_one_head(const double *x, double p, int d, double base, double *y)
{
    const int half = d / 2;
    for (int i = 0; i < half; ++i) {
        const double theta = pow(base, -2.0 * i / d);
        const double a = p * theta;
        const double c = cos(a), s = sin(a);
        y[i] = x[i] * c - x[i + half] * s;
        y[i + half] = x[i] * s + x[i + half] * c;
    }
}

int oracle_rope_qkv_f64(const double *qkv, const int32_t *positions, int B, int T, int Hq,
                        int Hkv, int d, double base, double *q, double *k, double *v)
{
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || d < 2 || d % 2 != 0 || !(base > 0.0)) return 1;
    const int H3 = Hq + 2 * Hkv;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            const double *tok = qkv + ((int64_t)b * T + t) * H3 * d;
            const double p = positions ? (double)positions[(int64_t)b * T + t] : (double)t;
            for (int h = 0; h < Hq; ++h)
                rope_one_head(tok + (int64_t)h * d, p, d, base,
                              q + (((int64_t)b * Hq + h) * T + t) * d);
            for (int h = 0; h < Hkv; ++h)
                rope_one_head(tok + (int64_t)(Hq + h) * d, p, d, base,
                              k + (((int64_t)b * Hkv + h) * T + t) * d);
            for (int h = 0; h < Hkv; ++h) {
                const double *src = tok + (int64_t)(Hq + Hkv + h) * d;
                double *dst = v + (((int64_t)b * Hkv + h) * T + t) * d;
                for (int c = 0; c < d; ++c) dst[c] = src[c];
            }
        }
    }
    return 0;
}
