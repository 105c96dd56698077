/*
 * td_oracle.c -- plain fp64 CPU oracle for exact single-query (decode-step)
 * softmax attention and for the chunked max-rescaled merge of tree-attention
 * decoding.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no header, helper, table or constant with the
 * CUDA library: the element decoders, the ALiBi term and the merge below are
 * written out again here from their definitions.
 *
 * Sources followed (page title -- section):
 *   [GIST]  "Tree Attention Decoding" (gist tree_attn_decode.py) --
 *           function regular_decode (plain decode attention) and
 *           function tree_attn_decode (Algorithm 3: per-chunk local max,
 *           logsumexp, softmax*V, num/den; global max; renormalise; sum;
 *           divide).
 *   [ALIBI] "ALiBi with causal=True unexpected bias?" (llm-foundry issue
 *           #186) -- the broadcast bias row arange(1-N, 1) times the head
 *           slope, and the shift-invariance argument softmax(x)=softmax(x+c).
 *   [FA]    "Flash Aandacht: Revolutie in Transformer Efficientie" --
 *           section "De Wiskunde Achter Flash Aandacht", formula 1 (softmax
 *           decomposition with the max) and formula 2 (fusion of two parts;
 *           printed garbled, read as the rescaled num/den form of [GIST]).
 *
 * Everything is computed in IEEE binary64, sums in index order, no blocking,
 * no fusion, no reordering beyond what the definitions state.
 *
 * Readings of points the pages leave open (each also listed in the design
 * notes of the repository):
 *   - lse returned is the ABSOLUTE natural-log log-sum-exp of the scaled and
 *     biased scores, m + ln(l) (the gist's per-chunk lse is relative to the
 *     chunk max).
 *   - The ALiBi term is slope_h * (j - n + 1) for key j of a sequence of
 *     length n; it is added to the scaled score q.k * D^-1/2, unscaled.
 *   - An empty chunk contributes nothing to the merge; an empty sequence
 *     (n = 0) yields out = 0 and lse = -inf.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* element type codes of this oracle (its own numbering) */
#define OR_F32 0
#define OR_BF16 1
#define OR_F16 2
#define OR_F64 3 /* already-widened values (e.g. dequantised FP8 caches) */

/* ---------------------------------------------------------------- decoders */

/* bfloat16 is the upper 16 bits of an IEEE binary32: widen exactly. */
double or_decode_bf16(uint16_t h) {
    uint32_t w = (uint32_t)h << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double or_decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m/1024 * 2^-14 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/*
 * FP8 E4M3 (the "fn" variant of the OCP 8-bit floating point formats): 1 sign
 * bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 is subnormal
 * (m/8 * 2^-6); no infinities; S.1111.111 is NaN; the largest value is 448.
 */
double or_decode_e4m3(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xf;
    int m = b & 7;
    double v;
    if (e == 0)
        v = ldexp((double)m, -9); /* m/8 * 2^-6 */
    else if (e == 15 && m == 7)
        v = NAN;
    else
        v = ldexp((double)(m + 8), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* bytes per stored element of each input type */
static size_t elem_bytes(int dtype) {
    return dtype == OR_F64 ? 8 : dtype == OR_F32 ? 4 : 2;
}

static double load_elem(const void *base, int64_t idx, int dtype) {
    if (dtype == OR_F64) return ((const double *)base)[idx];
    if (dtype == OR_F32) return (double)((const float *)base)[idx];
    uint16_t h = ((const uint16_t *)base)[idx];
    return dtype == OR_BF16 ? or_decode_bf16(h) : or_decode_f16(h);
}

/* ALiBi broadcast-row term for key j of a length-n sequence: slope*(j-n+1). */
double or_alibi_bias(double slope, int64_t j, int64_t n) {
    return slope * (double)(j - n + 1);
}

/* ------------------------------------------------------- plain definition */

/*
 * Scores of one query against keys [j0, j1) of a length-n sequence:
 *   s_j = (q * D^-1/2) . k_j + slope*(j-n+1) + extra[j]   ([GIST] regular_decode;
 *   [ALIBI] bias row).  q points at D elements, k at row 0 of the sequence.
 */
static void scores(const void *q, int64_t q_off, const void *k, int64_t k_off,
                   int dtype, int D, int64_t n, int64_t j0, int64_t j1,
                   double slope, const double *extra, double *s) {
    double scale = 1.0 / sqrt((double)D);
    double *qs = (double *)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d) qs[d] = load_elem(q, q_off + d, dtype) * scale;
    for (int64_t j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += qs[d] * load_elem(k, k_off + j * (int64_t)D + d, dtype);
        acc += or_alibi_bias(slope, j, n);
        if (extra) acc += extra[j];
        s[j - j0] = acc;
    }
    free(qs);
}

/*
 * Full softmax attention of one query over a length-n sequence
 * ([GIST] regular_decode; [FA] standaard_aandacht for one query row):
 *   m = max_j s_j, l = sum_j e^(s_j - m), out = sum_j e^(s_j - m) v_j / l,
 *   lse = m + ln l.
 */
static int attend(const void *q, int64_t q_off, const void *k, const void *v,
                  int64_t kv_off, int dtype, int D, int64_t n, double slope,
                  const double *extra, double *out, double *lse) {
    if (n <= 0) {
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return 0;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double *o = (double *)calloc((size_t)D, sizeof(double));
    if (!s || !o) {
        free(s);
        free(o);
        return -2;
    }
    scores(q, q_off, k, kv_off, dtype, D, n, 0, n, slope, extra, s);
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double p = exp(s[j] - m);
        l += p;
        for (int d = 0; d < D; ++d)
            o[d] += p * load_elem(v, kv_off + j * (int64_t)D + d, dtype);
    }
    for (int d = 0; d < D; ++d) out[d] = o[d] / l;
    *lse = m + log(l);
    free(s);
    free(o);
    return 0;
}

/* single query over a single sequence, with an optional extra per-key term
 * (test hook used for the shift-invariance and the full S x S ALiBi checks) */
int or_attend_one(const void *q, const void *k, const void *v, int dtype,
                  int64_t n, int D, double slope, const double *extra_bias,
                  double *out, double *lse) {
    if (!q || (n > 0 && (!k || !v)) || !out || !lse || D <= 0 || n < 0) return -1;
    return attend(q, 0, k, v, 0, dtype, D, n, slope, extra_bias, out, lse);
}

/* ---------------------------------------------------- chunked (Algorithm 3) */

/*
 * Chunk boundaries of [0, n) into w chunks.
 *   mode 0: the gist's k.chunk(world_size) -- chunk size ceil(n/w), the last
 *           chunk shorter, and fewer than w non-empty chunks when n is small;
 *           missing chunks are empty (start == end == n).
 *   mode 1: balanced -- chunk i is [floor(i*n/w), floor((i+1)*n/w)).
 * starts receives w+1 entries; chunk i is [starts[i], starts[i+1]).
 */
int or_chunk_bounds(int64_t n, int w, int mode, int64_t *starts) {
    if (w <= 0 || n < 0 || !starts || (mode != 0 && mode != 1)) return -1;
    if (mode == 0) {
        int64_t cs = (n + w - 1) / w;
        for (int i = 0; i <= w; ++i) {
            int64_t st = (int64_t)i * cs;
            starts[i] = st < n ? st : n;
        }
    } else {
        for (int i = 0; i <= w; ++i) starts[i] = (int64_t)i * n / w;
    }
    return 0;
}

/*
 * One chunk's partial, in the gist's two-pass form (tree_attn_decode, "first
 * calculate local output"): over keys [j0, j1) of a length-n sequence,
 *   local_max = max s;  sim = s - local_max;  lse_c = ln sum e^sim;
 *   attn = softmax(sim);  out_c = attn . V;  den = e^lse_c;  num = out_c*den.
 * Returns (num[D], local_max, den).  Empty chunk: (0, -inf, 0).
 */
int or_chunk_partial(const void *q, const void *k, const void *v, int dtype,
                     int64_t n, int D, double slope, int64_t j0, int64_t j1,
                     double *num, double *m_out, double *den_out) {
    if (!q || !num || !m_out || !den_out || D <= 0 || j0 < 0 || j1 > n || j0 > j1)
        return -1;
    int64_t len = j1 - j0;
    if (len == 0) {
        for (int d = 0; d < D; ++d) num[d] = 0.0;
        *m_out = -INFINITY;
        *den_out = 0.0;
        return 0;
    }
    double *sim = (double *)malloc(sizeof(double) * (size_t)len);
    double *attn = (double *)malloc(sizeof(double) * (size_t)len);
    if (!sim || !attn) {
        free(sim);
        free(attn);
        return -2;
    }
    scores(q, 0, k, 0, dtype, D, n, j0, j1, slope, NULL, sim);
    double local_max = -INFINITY;
    for (int64_t t = 0; t < len; ++t)
        if (sim[t] > local_max) local_max = sim[t];
    for (int64_t t = 0; t < len; ++t) sim[t] -= local_max;
    /* logsumexp of the shifted scores (its max is 0, so a plain sum is safe) */
    double sum = 0.0;
    for (int64_t t = 0; t < len; ++t) sum += exp(sim[t]);
    double lse_c = log(sum);
    for (int64_t t = 0; t < len; ++t) attn[t] = exp(sim[t]) / sum;
    double den = exp(lse_c);
    for (int d = 0; d < D; ++d) {
        double o = 0.0;
        for (int64_t t = 0; t < len; ++t)
            o += attn[t] * load_elem(v, (j0 + t) * (int64_t)D + d, dtype);
        num[d] = o * den;
    }
    *m_out = local_max;
    *den_out = den;
    free(sim);
    free(attn);
    return 0;
}

/*
 * Merge of S partials (num_s[D], m_s, den_s) ([GIST] tree_attn_decode, the
 * all-reduce MAX / renormalise / two all-reduce SUMs / divide; [FA] formula 2
 * read as: rescale each part by e^(m_s - M) with M = max m_s, then add):
 *   M = max_s m_s;  r_s = e^(m_s - M);  den = sum r_s den_s;
 *   num = sum r_s num_s;  out = num / den;  lse = M + ln den.
 * Empty partials (m_s = -inf) contribute nothing; all empty -> out 0, lse -inf.
 */
int or_merge(const double *num, const double *m, const double *l, int64_t S, int D,
             double *out, double *lse) {
    if (!num || !m || !l || !out || !lse || S < 0 || D <= 0) return -1;
    double M = -INFINITY;
    for (int64_t s = 0; s < S; ++s)
        if (m[s] > M) M = m[s];
    if (M == -INFINITY) {
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return 0;
    }
    double den = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t s = 0; s < S; ++s) {
        if (m[s] == -INFINITY) continue;
        double r = exp(m[s] - M);
        den += r * l[s];
        for (int d = 0; d < D; ++d) out[d] += r * num[s * (int64_t)D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= den;
    *lse = M + log(den);
    return 0;
}

/* chunked decode of one sequence: partials per chunk, then the merge */
static int attend_chunked(const void *q, int64_t q_off, const void *k, const void *v,
                          int64_t kv_off, int dtype, int D, int64_t n, double slope,
                          int w, int mode, double *out, double *lse) {
    int64_t *starts = (int64_t *)malloc(sizeof(int64_t) * (size_t)(w + 1));
    double *num = (double *)malloc(sizeof(double) * (size_t)w * (size_t)D);
    double *mm = (double *)malloc(sizeof(double) * (size_t)w);
    double *dd = (double *)malloc(sizeof(double) * (size_t)w);
    int rc = -2;
    if (starts && num && mm && dd) {
        rc = or_chunk_bounds(n, w, mode, starts);
        const char *qb = (const char *)q;
        const char *kb = (const char *)k;
        const char *vb = (const char *)v;
        size_t es = elem_bytes(dtype);
        for (int c = 0; rc == 0 && c < w; ++c)
            rc = or_chunk_partial(qb + q_off * es, kb + kv_off * es, vb + kv_off * es,
                                  dtype, n, D, slope, starts[c], starts[c + 1],
                                  num + (size_t)c * D, mm + c, dd + c);
        if (rc == 0) rc = or_merge(num, mm, dd, w, D, out, lse);
    }
    free(starts);
    free(num);
    free(mm);
    free(dd);
    return rc;
}

/* ------------------------------------------------- batched, threaded driver */

typedef struct {
    const void *q, *k, *v;
    int dtype, B, H, D;
    int Hkv;                /* key/value heads; query head h reads kv head h / (H / Hkv) */
    int64_t Nmax;
    const int32_t *seqlens; /* host, [B], or NULL: every sequence has Nmax keys */
    const float *slopes;    /* host, [H], or NULL: no bias */
    const int64_t *bh;      /* host list of b*H+h, or NULL: all */
    int64_t n_bh;
    int chunks, mode;       /* chunks == 0: plain definition */
    double *out, *lse;
    int64_t next;           /* work counter */
    int rc;
} job_t;

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        int64_t i = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (i >= J->n_bh) break;
        int64_t bh = J->bh ? J->bh[i] : i;
        int64_t b = bh / J->H, h = bh % J->H;
        int64_t hkv = h / (J->H / J->Hkv);
        int64_t n = J->seqlens ? (int64_t)J->seqlens[b] : J->Nmax;
        double slope = J->slopes ? (double)J->slopes[h] : 0.0;
        int64_t q_off = bh * (int64_t)J->D;
        int64_t kv_off = (b * J->Hkv + hkv) * J->Nmax * (int64_t)J->D;
        int rc;
        if (J->chunks == 0)
            rc = attend(J->q, q_off, J->k, J->v, kv_off, J->dtype, J->D, n, slope, NULL,
                        J->out + i * (int64_t)J->D, J->lse + i);
        else
            rc = attend_chunked(J->q, q_off, J->k, J->v, kv_off, J->dtype, J->D, n, slope,
                                J->chunks, J->mode, J->out + i * (int64_t)J->D, J->lse + i);
        if (rc) __atomic_store_n(&J->rc, rc, __ATOMIC_RELAXED);
    }
    return NULL;
}

static int run(job_t *J, int threads) {
    if (!J->q || !J->k || !J->v || !J->out || !J->lse) return -1;
    if (J->dtype < OR_F32 || J->dtype > OR_F64 || J->B <= 0 || J->H <= 0 || J->D <= 0 ||
        J->Nmax < 0 || J->n_bh < 0 || J->Hkv <= 0 || J->H % J->Hkv != 0)
        return -1;
    if (J->seqlens)
        for (int b = 0; b < J->B; ++b)
            if (J->seqlens[b] < 0 || J->seqlens[b] > J->Nmax) return -1;
    if (J->bh)
        for (int64_t i = 0; i < J->n_bh; ++i)
            if (J->bh[i] < 0 || J->bh[i] >= (int64_t)J->B * J->H) return -1;
    if (threads <= 0) threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    J->next = 0;
    J->rc = 0;
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < threads; ++t)
        if (pthread_create(&tid[started], NULL, worker, J) == 0) ++started;
    worker(J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J->rc;
}

/*
 * Plain decode attention ([GIST] regular_decode with the [ALIBI] bias) for the
 * (b,h) pairs listed in bh (all B*H when bh is NULL).
 * Layout: q [B,H,1,D], k/v [B,H,Nmax,D] row-major in the given element type;
 * sequence b uses its first seqlens[b] keys (all Nmax when seqlens is NULL).
 * out [n_bh, D] and lse [n_bh] in fp64.  threads <= 0: all online cores.
 */
int or_full(const void *q, const void *k, const void *v, int dtype, int B, int H,
            int64_t Nmax, int D, const int32_t *seqlens, const float *slopes,
            const int64_t *bh, int64_t n_bh, double *out, double *lse, int threads) {
    job_t J = {q, k, v, dtype, B, H, D, H, Nmax, seqlens, slopes, bh,
               bh ? n_bh : (int64_t)B * H, 0, 0, out, lse, 0, 0};
    return run(&J, threads);
}

/*
 * Grouped-query form of the plain definition: H query heads share Hkv
 * key/value heads (H a multiple of Hkv), query head h attending to kv head
 * h / (H / Hkv).  Layout q [B,H,1,D], k/v [B,Hkv,Nmax,D]; slopes per query
 * head [H]; bh lists b*H+h over query heads.  Hkv = 1 is multi-query
 * attention, Hkv = H is or_full.
 */
int or_full_gqa(const void *q, const void *k, const void *v, int dtype, int B, int H, int Hkv,
                int64_t Nmax, int D, const int32_t *seqlens, const float *slopes,
                const int64_t *bh, int64_t n_bh, double *out, double *lse, int threads) {
    job_t J = {q, k, v, dtype, B, H, D, Hkv, Nmax, seqlens, slopes, bh,
               bh ? n_bh : (int64_t)B * H, 0, 0, out, lse, 0, 0};
    return run(&J, threads);
}

/* ---------------------------------------------------------------- prefill */

/*
 * Prefill attention of every query row of a sequence of S tokens: the plain
 * definition with the [ALIBI] bias row over the whole sequence and, when
 * causal, its causal mask ([ALIBI] causal=True; [FA] "Flash Aandacht"
 * computes the same rows blockwise):
 *   s_ij = (q_i D^-1/2) . k_j + slope_h (j - S + 1)   for j in J(i),
 *   J(i) = {0, .., i} if causal else {0, .., S-1},
 *   m_i = max_j s_ij, out_i = sum_j e^(s_ij - m_i) v_j / sum_j e^(s_ij - m_i),
 *   lse_i = m_i + ln sum_j e^(s_ij - m_i).
 * Layout q, k, v [B,H,S,D]; `rows` lists row indices (b*H + h)*S + i (all
 * B*H*S rows when NULL); out [n_rows, D], lse [n_rows] fp64.
 */
typedef struct {
    const void *q, *k, *v;
    int dtype, B, H, D, causal;
    int64_t S;
    const float *slopes;
    const int64_t *rows;
    int64_t n_rows;
    double *out, *lse;
    int64_t next;
    int rc;
} prefill_job_t;

static int prefill_row(const prefill_job_t *J, int64_t r, double *out, double *lse) {
    const int D = J->D;
    const int64_t S = J->S;
    const int64_t bh = r / S, i = r % S;
    const int64_t h = bh % J->H;
    const double slope = J->slopes ? (double)J->slopes[h] : 0.0;
    const int64_t nk = J->causal ? i + 1 : S;
    const int64_t kv_off = bh * S * (int64_t)D;
    double *s = (double *)malloc(sizeof(double) * (size_t)nk);
    double *o = (double *)calloc((size_t)D, sizeof(double));
    double *qs = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !o || !qs) {
        free(s);
        free(o);
        free(qs);
        return -2;
    }
    const double scale = 1.0 / sqrt((double)D);
    for (int d = 0; d < D; ++d) qs[d] = load_elem(J->q, r * (int64_t)D + d, J->dtype) * scale;
    double m = -INFINITY;
    for (int64_t j = 0; j < nk; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qs[d] * load_elem(J->k, kv_off + j * (int64_t)D + d, J->dtype);
        acc += or_alibi_bias(slope, j, S);
        s[j] = acc;
        if (acc > m) m = acc;
    }
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        const double p = exp(s[j] - m);
        l += p;
        for (int d = 0; d < D; ++d) o[d] += p * load_elem(J->v, kv_off + j * (int64_t)D + d, J->dtype);
    }
    for (int d = 0; d < D; ++d) out[d] = o[d] / l;
    *lse = m + log(l);
    free(s);
    free(o);
    free(qs);
    return 0;
}

static void *prefill_worker(void *arg) {
    prefill_job_t *J = (prefill_job_t *)arg;
    for (;;) {
        int64_t i = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (i >= J->n_rows) break;
        int64_t r = J->rows ? J->rows[i] : i;
        int rc = prefill_row(J, r, J->out + i * (int64_t)J->D, J->lse + i);
        if (rc) __atomic_store_n(&J->rc, rc, __ATOMIC_RELAXED);
    }
    return NULL;
}

int or_prefill(const void *q, const void *k, const void *v, int dtype, int B, int H, int64_t S,
               int D, int causal, const float *slopes, const int64_t *rows, int64_t n_rows,
               double *out, double *lse, int threads) {
    if (!q || !k || !v || !out || !lse || dtype < OR_F32 || dtype > OR_F64 || B <= 0 ||
        H <= 0 || S <= 0 || D <= 0 || n_rows < 0)
        return -1;
    prefill_job_t J = {q, k, v, dtype, B, H, D, causal ? 1 : 0, S, slopes, rows,
                       rows ? n_rows : (int64_t)B * H * S, out, lse, 0, 0};
    if (rows)
        for (int64_t i = 0; i < n_rows; ++i)
            if (rows[i] < 0 || rows[i] >= (int64_t)B * H * S) return -1;
    if (threads <= 0) threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < threads; ++t)
        if (pthread_create(&tid[started], NULL, prefill_worker, &J) == 0) ++started;
    prefill_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J.rc;
}

/* The same, through the chunked Algorithm-3 path with w chunks per (b,h). */
int or_chunked(const void *q, const void *k, const void *v, int dtype, int B, int H,
               int64_t Nmax, int D, const int32_t *seqlens, const float *slopes,
               const int64_t *bh, int64_t n_bh, int w, int mode, double *out,
               double *lse, int threads) {
    if (w <= 0 || (mode != 0 && mode != 1)) return -1;
    job_t J = {q, k, v, dtype, B, H, D, H, Nmax, seqlens, slopes, bh,
               bh ? n_bh : (int64_t)B * H, w, mode, out, lse, 0, 0};
    return run(&J, threads);
}
