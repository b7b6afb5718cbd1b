/*
 * Plain fp64 CPU oracle for the variable-length packed attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  The CUDA product path
 * never links, calls or includes anything from this directory, and this file
 * includes nothing from the product.
 *
 * What it computes (per query token t and query head h), following
 *   - boostr 0.2.0 varlen_attention.rs, VarLenAttentionOps docs,
 *     "Layout contract", "GQA key/value head mapping", "Cumulative sequence
 *     lengths": q [total_q, H, D], k/v [total_k, H_kv, D], sequence b owns
 *     query rows cu_q[b]..cu_q[b+1]-1 and key rows cu_k[b]..cu_k[b+1]-1;
 *     kv_head = h / (H / H_kv); output [total_q, H, D]; logsumexp [total_q, H];
 *   - realizar 0.8.4 attention.rs, IMP-111 standard_single_head_attention and
 *     standard_softmax: scores = q.k * (1/sqrt(D)), softmax(x) =
 *     exp(x - max) / sum exp(x - max), output = softmax(scores) @ V;
 *   - boostr flash.rs FlashAttentionOps docs, "Sliding window": with
 *     window_size W > 0 a query sees only the W most recent key positions;
 *     logsumexp is F32 and is what the backward pass consumes.
 *
 * Readings taken where the pages are silent (the varlen trait defines no
 * causal offset, window inclusivity, logsumexp base or empty-row result):
 *   - causal with L_q != L_k is bottom-right aligned: key j is visible to
 *     query i iff j <= i + (L_k - L_q);
 *   - the window holds exactly W keys ending at the diagonal:
 *     i + delta - W + 1 <= j <= i + delta, and W > 0 implies the upper bound
 *     even without the causal flag;
 *   - logsumexp is the natural log of sum_j exp(s_ij) over the visible keys
 *     of the SCALED scores s_ij = q_i.k_j / sqrt(D);
 *   - a query with no visible key gets output 0 and logsumexp -inf;
 *   - a key-value cache with a capacity stride (the kv_seq_len of flash.rs
 *     FlashAttentionOps: iterate over the first n positions while the
 *     tensor's size stays the memory stride), in the packed layout: when
 *     seqused_k is given, sequence b's key rows still start at cu_k[b] but
 *     only the first min(seqused_k[b], cu_k[b+1] - cu_k[b]) are its keys,
 *     and that count is the L_k of every rule above.
 *
 * Inputs are bf16 bit patterns; each is widened exactly to double.  All
 * arithmetic is double.  Rows are independent, so threads split the list of
 * requested (token, head) rows; nothing is blocked, fused or reordered
 * inside a row.
 *
 * FP8 inputs (boostr flash.rs, FlashAttentionOps::flash_attention_fwd_fp8:
 * per-tensor dequantization scales q_scale, k_scale, v_scale take FP8 to
 * FP32, o_scale is the scale the FP32 output is quantized with, accumulation
 * is FP32) are
 * decoded here from the E4M3 format definition and multiplied by their
 * scale, exactly, in double; the attention itself is the same definition.
 * Readings: the FP8 format is E4M3 (the pages do not name one); the output
 * code is O / o_scale (o_scale is the output's dequantization scale, as the
 * FP8 backward of the same trait uses it), with round-to-nearest-even and
 * saturation at +-448.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E4M3 (the "FN" variant of the OCP 8-bit floating-point formats): one sign
 * bit, four exponent bits with bias 7, three mantissa bits.  Exponent field 0
 * holds the subnormals (m / 8) * 2^-6; exponent 15 with mantissa 7 is NaN;
 * there are no infinities, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_to_double(uint8_t b) {
    const int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double x;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) x = ldexp((double)m, -9);
    else x = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -x : x;
}

/* Nearest E4M3 value of x, ties to the even mantissa; magnitudes of 448 and
 * more give 448 (saturation), NaN gives NaN.  Written as a search over the
 * non-negative finite codes 0x00..0x7E, whose values increase with the code. */
uint8_t oracle_double_to_e4m3(double x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0;
    for (int c = 1; c <= 0x7E; ++c)
        if (oracle_e4m3_to_double((uint8_t)c) <= a) lo = c;
    const double vl = oracle_e4m3_to_double((uint8_t)lo);
    const double vh = oracle_e4m3_to_double((uint8_t)(lo + 1));
    int pick;
    if (a - vl < vh - a) pick = lo;
    else if (a - vl > vh - a) pick = lo + 1;
    else pick = (lo & 1) ? lo + 1 : lo;
    return (uint8_t)(sign | pick);
}

/* element e of a packed tensor, widened to double and multiplied by its scale */
typedef double (*decode_fn)(const void* base, size_t e);
static double decode_bf16(const void* base, size_t e) {
    return bf16_bits_to_double(((const uint16_t*)base)[e]);
}
static double decode_e4m3(const void* base, size_t e) {
    return oracle_e4m3_to_double(((const uint8_t*)base)[e]);
}

/* Sequence b owning packed query token t: the b with cu_q[b] <= t < cu_q[b+1]. */
static int owning_sequence(const int32_t* cu_q, int batch, int64_t t) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if ((int64_t)cu_q[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* The visibility predicate, written out as stated above. */
static int key_visible(int64_t i, int64_t j, int64_t L_q, int64_t L_k,
                       int causal, int window) {
    int64_t delta = L_k - L_q;
    if (j < 0 || j >= L_k) return 0;
    if (causal && j > i + delta) return 0;
    if (window > 0) {
        if (j > i + delta) return 0;
        if (j < i + delta - window + 1) return 0;
    }
    return 1;
}

typedef struct {
    const void *q, *k, *v;
    decode_fn decode;
    double q_scale, k_scale, v_scale;
    double* err; /* optional [n_rows, D]: P-rounding error scale, see below */
    const int32_t *cu_q, *cu_k;
    const int32_t* seqused_k; /* NULL => every row of the sequence's range is a key */
    int batch, H, H_kv, D, causal, window;
    const int64_t* row_token; /* NULL => all rows r = t*H + h */
    const int32_t* row_head;
    int64_t row_begin, row_end;
    double* out; /* [n_rows, D] */
    double* lse; /* [n_rows] */
    int64_t max_lk;
} job_t;

/* One output row.  `decode` is passed as a constant by each caller below, so
 * the compiler specialises this function per input format. */
static inline __attribute__((always_inline)) void one_row(const job_t* jb, int64_t r, double* s,
                                                          decode_fn decode) {
    int64_t t;
    int h;
    if (jb->row_token) { t = jb->row_token[r]; h = jb->row_head[r]; }
    else { t = r / jb->H; h = (int)(r % jb->H); }
    const int D = jb->D;
    const int b = owning_sequence(jb->cu_q, jb->batch, t);
    const int64_t L_q = (int64_t)jb->cu_q[b + 1] - jb->cu_q[b];
    int64_t L_k = (int64_t)jb->cu_k[b + 1] - jb->cu_k[b];
    if (jb->seqused_k) {
        const int64_t used = jb->seqused_k[b] > 0 ? jb->seqused_k[b] : 0;
        if (used < L_k) L_k = used;
    }
    const int64_t i = t - jb->cu_q[b];
    const int group = jb->H / jb->H_kv;
    const int hk = h / group;
    const double scale = 1.0 / sqrt((double)D);
    const size_t qrow = ((size_t)t * jb->H + h) * D;
    double* o = jb->out + (size_t)r * D;
    double* err = jb->err ? jb->err + (size_t)r * D : NULL;

    /* scores of the visible keys; s[j] = -inf marks an invisible key */
    double m = -INFINITY;
    int64_t n_vis = 0;
    for (int64_t j = 0; j < L_k; ++j) {
        if (!key_visible(i, j, L_q, L_k, jb->causal, jb->window)) { s[j] = -INFINITY; continue; }
        const size_t krow = (((size_t)jb->cu_k[b] + j) * jb->H_kv + hk) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += (decode(jb->q, qrow + d) * jb->q_scale) * (decode(jb->k, krow + d) * jb->k_scale);
        s[j] = dot * scale;
        if (s[j] > m) m = s[j];
        ++n_vis;
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (err) for (int d = 0; d < D; ++d) err[d] = 0.0;
    if (n_vis == 0) { jb->lse[r] = -INFINITY; return; }

    double l = 0.0;
    for (int64_t j = 0; j < L_k; ++j) {
        if (s[j] == -INFINITY) continue;
        const double p = exp(s[j] - m);
        l += p;
        const size_t vrow = (((size_t)jb->cu_k[b] + j) * jb->H_kv + hk) * D;
        /* When P is rounded to E4M3 before it multiplies V, p (in units of the
         * row maximum, which is 1 here and at most 1 when the reference is an
         * earlier, smaller maximum) moves by at most e = max(2^-4 p, 2^-10):
         * half the spacing of E4M3 numbers relative to a normal value, or
         * absolute among the subnormals.  Modelling each rounding error as
         * uniform on [-e, e] and independent across keys, the output error has
         * variance sum_j (e_j^2 / 3) v_jd^2 / l^2; err accumulates that sum. */
        const double e = fmax(ldexp(p, -4), ldexp(1.0, -10));
        for (int d = 0; d < D; ++d) {
            const double vd = decode(jb->v, vrow + d) * jb->v_scale;
            o[d] += p * vd;
            if (err) err[d] += e * e / 3.0 * vd * vd;
        }
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    if (err) for (int d = 0; d < D; ++d) err[d] = sqrt(err[d]) / l;
    jb->lse[r] = m + log(l);
}

static void* run_job(void* arg) {
    const job_t* jb = (const job_t*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(jb->max_lk > 0 ? jb->max_lk : 1));
    if (!s) return (void*)1;
    if (jb->decode == decode_e4m3)
        for (int64_t r = jb->row_begin; r < jb->row_end; ++r) one_row(jb, r, s, decode_e4m3);
    else
        for (int64_t r = jb->row_begin; r < jb->row_end; ++r) one_row(jb, r, s, decode_bf16);
    free(s);
    return NULL;
}

/*
 * Compute output and logsumexp rows in fp64.
 *
 * q, k, v:     bf16 bit patterns, packed [total_q, H, D] and [total_k, H_kv, D].
 * cu_q, cu_k:  host int32 [batch + 1] cumulative lengths.
 * seqused_k:   optional host int32 [batch]: sequence b's keys are the first
 *              min(seqused_k[b], cu_k[b+1] - cu_k[b]) rows from cu_k[b]
 *              (NULL: all of them).
 * row_token, row_head: optional (token, head) pairs to compute (n_rows of
 *              them); when row_token is NULL every row is computed in the
 *              order r = token * H + head and n_rows must be total_q * H.
 * out:         [n_rows, D] doubles; lse: [n_rows] doubles.
 * Returns 0, or -1 on an argument error, -2 on an allocation failure.
 */
static int attention_rows(const void* q, const void* k, const void* v, decode_fn decode,
                          double q_scale, double k_scale, double v_scale,
                          const int32_t* cu_q, const int32_t* cu_k,
                          const int32_t* seqused_k, int batch,
                          int H, int H_kv, int D, int causal, int window,
                          const int64_t* row_token, const int32_t* row_head,
                          int64_t n_rows, double* out, double* lse, double* err, int nthreads) {
    if (batch < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || D < 1 || window < 0) return -1;
    if (n_rows < 0 || (n_rows > 0 && (!out || !lse))) return -1;
    if (!row_token && n_rows != (int64_t)cu_q[batch] * H) return -1;
    if (row_token && !row_head) return -1;
    int64_t max_lk = 0;
    for (int b = 0; b < batch; ++b) {
        int64_t lk = (int64_t)cu_k[b + 1] - cu_k[b];
        if (lk > max_lk) max_lk = lk;
    }
    if (nthreads < 1) nthreads = 1;
    if ((int64_t)nthreads > n_rows) nthreads = n_rows > 0 ? (int)n_rows : 1;

    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) { free(jobs); free(tids); return -2; }
    int rc = 0;
    for (int w = 0; w < nthreads; ++w) {
        job_t* jb = &jobs[w];
        jb->q = q; jb->k = k; jb->v = v; jb->cu_q = cu_q; jb->cu_k = cu_k;
        jb->decode = decode;
        jb->q_scale = q_scale; jb->k_scale = k_scale; jb->v_scale = v_scale;
        jb->err = err;
        jb->seqused_k = seqused_k;
        jb->batch = batch; jb->H = H; jb->H_kv = H_kv; jb->D = D;
        jb->causal = causal; jb->window = window;
        jb->row_token = row_token; jb->row_head = row_head;
        jb->row_begin = n_rows * w / nthreads;
        jb->row_end = n_rows * (w + 1) / nthreads;
        jb->out = out; jb->lse = lse; jb->max_lk = max_lk;
    }
    int started = 0;
    for (int w = 1; w < nthreads; ++w) {
        if (pthread_create(&tids[w], NULL, run_job, &jobs[w]) != 0) { rc = -2; break; }
        started = w;
    }
    if (run_job(&jobs[0]) != NULL) rc = -2;
    for (int w = 1; w <= started; ++w) {
        void* ret = NULL;
        pthread_join(tids[w], &ret);
        if (ret != NULL) rc = -2;
    }
    free(jobs);
    free(tids);
    return rc;
}

int oracle_varlen_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const int32_t* cu_q, const int32_t* cu_k,
                                 const int32_t* seqused_k, int batch,
                                 int H, int H_kv, int D, int causal, int window,
                                 const int64_t* row_token, const int32_t* row_head,
                                 int64_t n_rows, double* out, double* lse, int nthreads) {
    return attention_rows(q, k, v, decode_bf16, 1.0, 1.0, 1.0, cu_q, cu_k, seqused_k, batch, H,
                          H_kv, D, causal, window, row_token, row_head, n_rows, out, lse, NULL,
                          nthreads);
}

/*
 * The same rows for E4M3 inputs with per-tensor dequantization scales
 * (element value = decoded E4M3 * scale).  out is the exact output before it
 * is quantized (the caller divides by o_scale and applies oracle_double_to_e4m3);
 * err (optional, [n_rows, D]) receives the standard-deviation scale of the
 * error that rounding P to E4M3 may add, as described in one_row.
 */
int oracle_varlen_attention_rows_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v,
                                     double q_scale, double k_scale, double v_scale,
                                     const int32_t* cu_q, const int32_t* cu_k, int batch,
                                     int H, int H_kv, int D, int causal, int window,
                                     const int64_t* row_token, const int32_t* row_head,
                                     int64_t n_rows, double* out, double* lse, double* err,
                                     int nthreads) {
    return attention_rows(q, k, v, decode_e4m3, q_scale, k_scale, v_scale, cu_q, cu_k, NULL,
                          batch, H, H_kv, D, causal, window, row_token, row_head, n_rows, out,
                          lse, err, nthreads);
}

/* Element-wise E4M3 decoding / encoding of arrays (the definitions above). */
void oracle_e4m3_decode_array(const uint8_t* in, double* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_to_double(in[i]);
}

void oracle_e4m3_encode_array(const double* in, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_e4m3(in[i]);
}

/*
 * Backward pass (boostr 0.2.0 varlen_attention.rs, VarLenAttentionOps::
 * varlen_attention_bwd: dq [total_q, H, D], dk and dv [total_k, H_kv, D]
 * with full GQA support; boostr flash.rs, FlashAttentionOps docs, the
 * backward consumes the logsumexp of the forward).  Gradients of
 * L = sum_{t,h,d} dout[t,h,d] * out[t,h,d] with out the forward above,
 * written out from the definition for each query row i of head h:
 *   s_ij = q_i.k_j / sqrt(D) over the visible keys, P_ij = exp(s_ij - lse_i)
 *   (lse_i recomputed here exactly), O_i = sum_j P_ij v_j,
 *   dP_ij = dout_i.v_j, Delta_i = dout_i.O_i = sum_j P_ij dP_ij,
 *   dS_ij = P_ij (dP_ij - Delta_i),
 *   dq_i = sum_j dS_ij k_j / sqrt(D),
 *   dk_j += dS_ij q_i / sqrt(D), dv_j += P_ij dout_i
 * (dk and dv summed over the query heads of a KV head's group).  Rows with
 * no visible key contribute nothing.  Inputs are bf16 bit patterns, all
 * arithmetic double.  One thread per (sequence, KV head) pair; nothing is
 * blocked or reordered inside a row.
 */
typedef struct {
    const uint16_t *q, *k, *v, *dout;
    const int32_t *cu_q, *cu_k;
    int batch, H, H_kv, D, causal, window;
    double *dq, *dk, *dv;
    int64_t pair_begin, pair_end; /* (b, hk) pairs b * H_kv + hk */
    int64_t max_lk;
} bwd_job_t;

static void* run_bwd_job(void* arg) {
    const bwd_job_t* jb = (const bwd_job_t*)arg;
    const int D = jb->D, G = jb->H / jb->H_kv;
    const double scale = 1.0 / sqrt((double)D);
    const size_t n = (size_t)(jb->max_lk > 0 ? jb->max_lk : 1);
    double* s = (double*)malloc(sizeof(double) * n);
    double* dp = (double*)malloc(sizeof(double) * n);
    double* o = (double*)malloc(sizeof(double) * (size_t)D);
    if (!s || !dp || !o) { free(s); free(dp); free(o); return (void*)1; }
    for (int64_t pr = jb->pair_begin; pr < jb->pair_end; ++pr) {
        const int b = (int)(pr / jb->H_kv), hk = (int)(pr % jb->H_kv);
        const int64_t L_q = (int64_t)jb->cu_q[b + 1] - jb->cu_q[b];
        const int64_t L_k = (int64_t)jb->cu_k[b + 1] - jb->cu_k[b];
        for (int h = hk * G; h < (hk + 1) * G; ++h) {
            for (int64_t i = 0; i < L_q; ++i) {
                const size_t qrow = (((size_t)jb->cu_q[b] + i) * jb->H + h) * D;
                double m = -INFINITY;
                int64_t n_vis = 0;
                for (int64_t j = 0; j < L_k; ++j) {
                    if (!key_visible(i, j, L_q, L_k, jb->causal, jb->window)) { s[j] = -INFINITY; continue; }
                    const size_t krow = (((size_t)jb->cu_k[b] + j) * jb->H_kv + hk) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += bf16_bits_to_double(jb->q[qrow + d]) * bf16_bits_to_double(jb->k[krow + d]);
                    s[j] = dot * scale;
                    if (s[j] > m) m = s[j];
                    ++n_vis;
                }
                if (n_vis == 0) continue;
                double l = 0.0;
                for (int64_t j = 0; j < L_k; ++j)
                    if (s[j] != -INFINITY) l += exp(s[j] - m);
                const double lse = m + log(l);
                /* P_ij, O_i, dP_ij, Delta_i */
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t j = 0; j < L_k; ++j) {
                    if (s[j] == -INFINITY) continue;
                    const double p = exp(s[j] - lse);
                    const size_t vrow = (((size_t)jb->cu_k[b] + j) * jb->H_kv + hk) * D;
                    double dpj = 0.0;
                    for (int d = 0; d < D; ++d) {
                        const double vd = bf16_bits_to_double(jb->v[vrow + d]);
                        o[d] += p * vd;
                        dpj += bf16_bits_to_double(jb->dout[qrow + d]) * vd;
                    }
                    dp[j] = dpj;
                    s[j] = p; /* s now holds P */
                }
                double delta = 0.0;
                for (int d = 0; d < D; ++d) delta += bf16_bits_to_double(jb->dout[qrow + d]) * o[d];
                /* dS and the three gradients */
                double* dqi = jb->dq + qrow;
                for (int64_t j = 0; j < L_k; ++j) {
                    if (s[j] == -INFINITY) continue;
                    const double p = s[j];
                    const double ds = p * (dp[j] - delta);
                    const size_t krow = (((size_t)jb->cu_k[b] + j) * jb->H_kv + hk) * D;
                    for (int d = 0; d < D; ++d) {
                        dqi[d] += ds * bf16_bits_to_double(jb->k[krow + d]) * scale;
                        jb->dk[krow + d] += ds * bf16_bits_to_double(jb->q[qrow + d]) * scale;
                        jb->dv[krow + d] += p * bf16_bits_to_double(jb->dout[qrow + d]);
                    }
                }
            }
        }
    }
    free(s); free(dp); free(o);
    return NULL;
}

/*
 * dq [total_q, H, D], dk, dv [total_k, H_kv, D] doubles, zero-initialised
 * here.  Returns 0, -1 on an argument error, -2 on an allocation failure.
 */
int oracle_varlen_attention_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const uint16_t* dout, const int32_t* cu_q, const int32_t* cu_k,
                                int batch, int H, int H_kv, int D, int causal, int window,
                                double* dq, double* dk, double* dv, int nthreads) {
    if (batch < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || D < 1 || window < 0) return -1;
    const size_t nq = (size_t)cu_q[batch] * H * D, nk = (size_t)cu_k[batch] * H_kv * D;
    for (size_t x = 0; x < nq; ++x) dq[x] = 0.0;
    for (size_t x = 0; x < nk; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    int64_t max_lk = 0;
    for (int b = 0; b < batch; ++b) {
        int64_t lk = (int64_t)cu_k[b + 1] - cu_k[b];
        if (lk > max_lk) max_lk = lk;
    }
    const int64_t pairs = (int64_t)batch * H_kv;
    if (nthreads < 1) nthreads = 1;
    if ((int64_t)nthreads > pairs) nthreads = (int)pairs;
    bwd_job_t* jobs = (bwd_job_t*)calloc((size_t)nthreads, sizeof(bwd_job_t));
    pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) { free(jobs); free(tids); return -2; }
    int rc = 0;
    for (int w = 0; w < nthreads; ++w) {
        bwd_job_t* jb = &jobs[w];
        jb->q = q; jb->k = k; jb->v = v; jb->dout = dout; jb->cu_q = cu_q; jb->cu_k = cu_k;
        jb->batch = batch; jb->H = H; jb->H_kv = H_kv; jb->D = D;
        jb->causal = causal; jb->window = window;
        jb->dq = dq; jb->dk = dk; jb->dv = dv;
        jb->pair_begin = pairs * w / nthreads;
        jb->pair_end = pairs * (w + 1) / nthreads;
        jb->max_lk = max_lk;
    }
    int started = 0;
    for (int w = 1; w < nthreads; ++w) {
        if (pthread_create(&tids[w], NULL, run_bwd_job, &jobs[w]) != 0) { rc = -2; break; }
        started = w;
    }
    if (run_bwd_job(&jobs[0]) != NULL) rc = -2;
    for (int w = 1; w <= started; ++w) {
        void* ret = NULL;
        pthread_join(tids[w], &ret);
        if (ret != NULL) rc = -2;
    }
    free(jobs);
    free(tids);
    return rc;
}
