/*
 * pa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what paged decode computes.  Only the
 * tests, the smoke check and the bench's CPU-baseline leg may load it.  It
 * shares no code, header, table or constant with the CUDA library: the two are
 * compared on the same seeded inputs and must agree.
 *
 * What it states (by page and section):
 *
 *   Storage decoding.  IEEE-754 binary32 / binary16, bfloat16 (the upper half
 *   of binary32), and OCP 8-bit floating point E4M3 ("FN": bias 7, no
 *   infinities, S.1111.111 is NaN, largest finite 448).  Each decoder reads the
 *   fields of the code and forms the value; nothing is looked up.
 *
 *   Cache append ("01. PagedAttention 详解" §4, decode step 2: the new token's k, v
 *   go into the next slot of the last block; the slot is block*block_size +
 *   offset, a negative slot is skipped).  Same dtype: the bytes are copied.
 *   fp8 cache (intelliparadigm PagedAttention article §4.3, kv_cache_dtype="fp8"): the
 *   value is divided by the per-tensor scale in binary32 and rounded to the
 *   nearest E4M3 value, ties to even, magnitudes at or above 448 saturating to
 *   448.  The rounding is done by exhaustive search over the 127 finite
 *   magnitudes, so it can be checked by eye.
 *
 *   Block copy (intelliparadigm PagedAttention article §3.3, copy_block inside
 *   maybe_copy_block; "PagedAttention 机制" §5.3.2, copy-on-write): a memcpy of
 *   whole blocks, K and V.  A pair list whose destination repeats, or names a
 *   block that is also a source, is rejected (the result would depend on
 *   order).
 *
 *   Decode attention ("PagedAttention 机制" §5.3.4 paged_attention: the key of
 *   logical token i sits at key_cache[block_tables[i // block_size],
 *   i % block_size]; intelliparadigm PagedAttention article §2.3: q.K per block then a
 *   softmax normalised over all blocks; "01. PagedAttention 详解" §4: per-block
 *   partials accumulated to the softmax over the whole context).  For each
 *   sequence s and query head h, with kv head g = h / (Hq / Hkv):
 *       K_s[i] = deq(key_cache[bt[s][i/bs], i%bs, g, :])   i < n_s
 *       z      = scale * K_s q
 *       w      = exp(z - max z) / sum exp(z - max z)
 *       out    = w^T V_s
 *   built by first gathering the logical, contiguous K_s and V_s, then doing
 *   textbook softmax attention over them in double.  n_s = 0 gives a zero row.
 *   deq multiplies the stored value by k_scale / v_scale (1 for non-fp8).
 *   The per-block, online or split form the kernels use is a reordering of
 *   this sum and is deliberately not reproduced here.
 *
 *   Prefill / chunked prefill ("01. PagedAttention 详解" §4, prefill: the N new
 *   tokens' K and V are first written into the blocks their table names, then
 *   ordinary attention runs over the cache).  Sequence s holds n_s tokens in
 *   the cache, the last L_s of which are this call's new tokens (rows
 *   query_start[s] .. query_start[s+1]-1 of q).  New token i sits at position
 *   p = n_s - L_s + i and, reading the attention as the usual causal one of a
 *   decoder, sees the keys at positions 0..p:
 *       out[row, h] = softmax(scale * K_s[0..p] q[row, h]) V_s[0..p]
 *   L_s = 1 is the decode step above; L_s = n_s is a prefill from an empty
 *   cache; anything between is a chunk of a chunked prefill.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_E4M3 = 3 };
enum { ORC_OK = 0, ORC_EARG = -1, ORC_EINDEX = -2, ORC_ENOMEM = -3 };

/* ---------------------------------------------------------------- decoding */

double orc_f32_value(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* binary16: sign, 5-bit exponent (bias 15), 10-bit fraction. */
double orc_f16_value(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);              /* 0.f * 2^-14 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);  /* 1.f * 2^(e-15) */
    return s ? -v : v;
}

/* bfloat16: sign, 8-bit exponent (bias 127), 7-bit fraction. */
double orc_bf16_value(uint16_t b) {
    int s = b >> 15, e = (b >> 7) & 255, f = b & 127;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);             /* 0.f * 2^-126 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);  /* 1.f * 2^(e-127) */
    return s ? -v : v;
}

/* OCP E4M3 (FN): sign, 4-bit exponent (bias 7), 3-bit mantissa; no infinities;
 * exponent 1111 with mantissa 111 is NaN, so the largest finite is 1.75*2^8. */
double orc_e4m3_value(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* 0.m * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);     /* 1.m * 2^(e-7) */
    return s ? -v : v;
}

static double value_at(const void* base, int dt, size_t i) {
    switch (dt) {
    case ORC_F32: return orc_f32_value(((const uint32_t*)base)[i]);
    case ORC_F16: return orc_f16_value(((const uint16_t*)base)[i]);
    case ORC_BF16: return orc_bf16_value(((const uint16_t*)base)[i]);
    case ORC_E4M3: return orc_e4m3_value(((const uint8_t*)base)[i]);
    }
    return NAN;
}

static size_t elem_size(int dt) {
    switch (dt) {
    case ORC_F32: return 4;
    case ORC_F16: case ORC_BF16: return 2;
    case ORC_E4M3: return 1;
    }
    return 0;
}

/* Nearest E4M3 code to x, ties to the even code, |x| >= 448 saturating. */
uint8_t orc_e4m3_encode(float x) {
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0)
        return sign | 0x7E;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(orc_e4m3_value((uint8_t)c) - a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return sign | (uint8_t)best;
}

/* array helpers for the Python side */
void orc_values(double* dst, const void* src, int dt, size_t n) {
    for (size_t i = 0; i < n; ++i) dst[i] = value_at(src, dt, i);
}

void orc_e4m3_encode_array(uint8_t* dst, const float* src, size_t n) {
    for (size_t i = 0; i < n; ++i) dst[i] = orc_e4m3_encode(src[i]);
}

/* ------------------------------------------------------------ cache append */

int orc_reshape_and_cache(const void* key, const void* value, int in_dt,
                          void* key_cache, void* value_cache, int cache_dt,
                          const int64_t* slot_mapping, int T, int Hkv, int D, int bs,
                          int64_t NB, float k_scale, float v_scale) {
    if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || NB <= 0) return ORC_EARG;
    if (in_dt != cache_dt && cache_dt != ORC_E4M3) return ORC_EARG;
    size_t ein = elem_size(in_dt), ec = elem_size(cache_dt);
    size_t row = (size_t)Hkv * D;
    for (int t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= NB * bs) return ORC_EINDEX;
        int64_t b = slot / bs, o = slot % bs;
        size_t dst0 = ((size_t)b * bs + (size_t)o) * row;
        size_t src0 = (size_t)t * row;
        for (int which = 0; which < 2; ++which) {
            const void* src = which ? value : key;
            void* dst = which ? value_cache : key_cache;
            float sc = which ? v_scale : k_scale;
            if (in_dt == cache_dt) {
                memcpy((char*)dst + dst0 * ec, (const char*)src + src0 * ein, row * ec);
            } else {
                for (size_t j = 0; j < row; ++j) {
                    float x = (float)value_at(src, in_dt, src0 + j); /* exact widening */
                    float y = x / sc;                                /* binary32 divide */
                    ((uint8_t*)dst)[dst0 + j] = orc_e4m3_encode(y);
                }
            }
        }
    }
    return ORC_OK;
}

/* -------------------------------------------------------------- block copy */

int orc_copy_blocks(void* key_cache, void* value_cache, size_t block_bytes, int64_t NB,
                    const int32_t* pairs, int n) {
    for (int i = 0; i < n; ++i) {
        int32_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= NB || d < 0 || d >= NB) return ORC_EINDEX;
        for (int j = 0; j < n; ++j) {
            if (j != i && pairs[2 * j + 1] == d) return ORC_EARG;  /* repeated destination */
            if (pairs[2 * j] == d) return ORC_EARG;                /* destination also a source */
        }
    }
    for (int i = 0; i < n; ++i) {
        size_t s = (size_t)pairs[2 * i], d = (size_t)pairs[2 * i + 1];
        memcpy((char*)key_cache + d * block_bytes, (char*)key_cache + s * block_bytes, block_bytes);
        memcpy((char*)value_cache + d * block_bytes, (char*)value_cache + s * block_bytes, block_bytes);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ decode */

typedef struct {
    double* out;              /* [nsel, Hq, D] */
    const void* q;            /* [S, Hq, D] */
    int q_dt;
    const void* kc;
    const void* vc;
    int kv_dt;
    const int32_t* bt;
    int MB;
    const int32_t* ctx;
    const int32_t* sel;       /* selected sequences (nsel of them) */
    int nsel, Hq, Hkv, D, bs;
    int64_t NB;
    double scale, k_scale, v_scale;
    int nthreads, tid;
    int status;
} decode_job;

/* Gather the logical K_s, V_s (n x D) of kv head g of sequence s. */
static int gather(const decode_job* j, int s, int g, int n, double* K, double* V) {
    for (int i = 0; i < n; ++i) {
        int32_t b = j->bt[(size_t)s * j->MB + i / j->bs];
        if (b < 0 || b >= j->NB) return ORC_EINDEX;
        size_t off = (((size_t)b * j->bs + (size_t)(i % j->bs)) * j->Hkv + g) * j->D;
        for (int d = 0; d < j->D; ++d) {
            K[(size_t)i * j->D + d] = value_at(j->kc, j->kv_dt, off + d) * j->k_scale;
            V[(size_t)i * j->D + d] = value_at(j->vc, j->kv_dt, off + d) * j->v_scale;
        }
    }
    return ORC_OK;
}

/* Textbook softmax attention of one query over n contiguous keys/values.
 * w (length n) receives the normalised weights. */
static void attend(const double* qv, const double* K, const double* V, int n, int D,
                   double scale, double* w, double* out) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (n == 0) return;
    double zmax = -INFINITY;
    for (int i = 0; i < n; ++i) {
        double z = 0.0;
        for (int d = 0; d < D; ++d) z += qv[d] * K[(size_t)i * D + d];
        w[i] = scale * z;
        if (w[i] > zmax) zmax = w[i];
    }
    double sum = 0.0;
    for (int i = 0; i < n; ++i) {
        w[i] = exp(w[i] - zmax);
        sum += w[i];
    }
    for (int i = 0; i < n; ++i) w[i] /= sum;
    for (int i = 0; i < n; ++i)
        for (int d = 0; d < D; ++d) out[d] += w[i] * V[(size_t)i * D + d];
}

static void* decode_worker(void* arg) {
    decode_job* j = (decode_job*)arg;
    int G = j->Hq / j->Hkv;
    double* K = NULL;
    double* V = NULL;
    double* w = NULL;
    double* qv = (double*)malloc(sizeof(double) * j->D);
    size_t cap = 0;
    int units = j->nsel * j->Hkv;
    for (int u = j->tid; u < units; u += j->nthreads) {
        int si = u / j->Hkv, g = u % j->Hkv;
        int s = j->sel ? j->sel[si] : si;
        int n = j->ctx[s];
        if ((size_t)n > cap) {
            cap = (size_t)n;
            free(K); free(V); free(w);
            K = (double*)malloc(sizeof(double) * cap * j->D);
            V = (double*)malloc(sizeof(double) * cap * j->D);
            w = (double*)malloc(sizeof(double) * cap);
            if (!K || !V || !w) { j->status = ORC_ENOMEM; break; }
        }
        int rc = gather(j, s, g, n, K, V);
        if (rc) { j->status = rc; break; }
        for (int hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            size_t qoff = ((size_t)s * j->Hq + h) * j->D;
            for (int d = 0; d < j->D; ++d) qv[d] = value_at(j->q, j->q_dt, qoff + d);
            attend(qv, K, V, n, j->D, j->scale, w, j->out + ((size_t)si * j->Hq + h) * j->D);
        }
    }
    free(K); free(V); free(w); free(qv);
    return NULL;
}

static int hw_threads(int want) {
    if (want > 0) return want;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* out: [nsel or S, Hq, D] double.  sel: NULL for all sequences, else nsel ids. */
int orc_paged_decode(double* out, const void* q, int q_dt, const void* key_cache,
                     const void* value_cache, int kv_dt, const int32_t* block_tables, int MB,
                     const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs,
                     int64_t NB, double scale, double k_scale, double v_scale,
                     const int32_t* sel, int nsel, int nthreads) {
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || MB < 0) return ORC_EARG;
    if (!sel) nsel = S;
    for (int i = 0; i < nsel; ++i) {
        int s = sel ? sel[i] : i;
        if (s < 0 || s >= S) return ORC_EARG;
        if (context_lens[s] < 0 || (int64_t)context_lens[s] > (int64_t)MB * bs) return ORC_EARG;
    }
    int nt = hw_threads(nthreads);
    decode_job* jobs = (decode_job*)calloc((size_t)nt, sizeof(decode_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nt, sizeof(pthread_t));
    for (int t = 0; t < nt; ++t) {
        decode_job j = {out, q, q_dt, key_cache, value_cache, kv_dt, block_tables, MB,
                        context_lens, sel, nsel, Hq, Hkv, D, bs, NB, scale, k_scale, v_scale,
                        nt, t, ORC_OK};
        jobs[t] = j;
        pthread_create(&th[t], NULL, decode_worker, &jobs[t]);
    }
    int status = ORC_OK;
    for (int t = 0; t < nt; ++t) {
        pthread_join(th[t], NULL);
        if (jobs[t].status && !status) status = jobs[t].status;
    }
    free(jobs);
    free(th);
    return status;
}

/* The normalised softmax weights of one (sequence, query head): w[0..n_s). */
int orc_decode_weights(double* w, const void* q, int q_dt, const void* key_cache, int kv_dt,
                       const int32_t* block_tables, int MB, const int32_t* context_lens,
                       int Hq, int Hkv, int D, int bs, int64_t NB, double scale, double k_scale,
                       int s, int h) {
    int n = context_lens[s];
    decode_job j = {NULL, q, q_dt, key_cache, key_cache, kv_dt, block_tables, MB, context_lens,
                    NULL, 0, Hq, Hkv, D, bs, NB, scale, k_scale, 1.0, 1, 0, ORC_OK};
    double* K = (double*)malloc(sizeof(double) * (size_t)(n ? n : 1) * D);
    double* V = (double*)malloc(sizeof(double) * (size_t)(n ? n : 1) * D);
    double* qv = (double*)malloc(sizeof(double) * D);
    double* o = (double*)malloc(sizeof(double) * D);
    int rc = gather(&j, s, h / (Hq / Hkv), n, K, V);
    if (!rc) {
        size_t qoff = ((size_t)s * Hq + h) * D;
        for (int d = 0; d < D; ++d) qv[d] = value_at(q, q_dt, qoff + d);
        attend(qv, K, V, n, D, scale, w, o);
    }
    free(K); free(V); free(qv); free(o);
    return rc;
}

/* ----------------------------------------------------------------- prefill */

typedef struct {
    decode_job base;          /* caches, tables, shapes, scales */
    double* out;              /* [nrow or T, Hq, D] */
    const int32_t* qstart;    /* [S+1] */
    const int32_t* rows;      /* NULL: every row; else nrow row ids */
    int nrow, S, T;
    int status;
} prefill_job;

/* Sequence owning q row t (query_start is non-decreasing). */
static int row_seq(const int32_t* qs, int S, int t) {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (qs[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

static void* prefill_worker(void* arg) {
    prefill_job* pj = (prefill_job*)arg;
    const decode_job* j = &pj->base;
    int G = j->Hq / j->Hkv;
    double* K = NULL;
    double* V = NULL;
    double* w = NULL;
    double* qv = (double*)malloc(sizeof(double) * j->D);
    size_t cap = 0;
    int nr = pj->rows ? pj->nrow : pj->T;
    /* one unit = (selected row, kv head): gather, then the G heads of the group */
    for (int u = j->tid; u < nr * j->Hkv; u += j->nthreads) {
        int ri = u / j->Hkv, g = u % j->Hkv;
        int t = pj->rows ? pj->rows[ri] : ri;
        int s = row_seq(pj->qstart, pj->S, t);
        int n = j->ctx[s];
        int L = pj->qstart[s + 1] - pj->qstart[s];
        int p = n - L + (t - pj->qstart[s]);      /* position of this token */
        int nk = p + 1;                           /* keys 0..p */
        if ((size_t)nk > cap) {
            cap = (size_t)nk;
            free(K); free(V); free(w);
            K = (double*)malloc(sizeof(double) * cap * j->D);
            V = (double*)malloc(sizeof(double) * cap * j->D);
            w = (double*)malloc(sizeof(double) * cap);
            if (!K || !V || !w) { pj->status = ORC_ENOMEM; break; }
        }
        int rc = gather(j, s, g, nk, K, V);
        if (rc) { pj->status = rc; break; }
        for (int hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            size_t qoff = ((size_t)t * j->Hq + h) * j->D;
            for (int d = 0; d < j->D; ++d) qv[d] = value_at(j->q, j->q_dt, qoff + d);
            attend(qv, K, V, nk, j->D, j->scale, w, pj->out + ((size_t)ri * j->Hq + h) * j->D);
        }
    }
    free(K); free(V); free(w); free(qv);
    return NULL;
}

/* out: [nrow or T, Hq, D] double.  q: [T, Hq, D].  query_start: [S+1] with
 * query_start[0] = 0, query_start[S] = T, and 0 <= L_s <= n_s.  rows: NULL for
 * every q row, else nrow row ids. */
int orc_paged_prefill(double* out, const void* q, int q_dt, const void* key_cache,
                      const void* value_cache, int kv_dt, const int32_t* block_tables, int MB,
                      const int32_t* context_lens, const int32_t* query_start, int S, int T,
                      int Hq, int Hkv, int D, int bs, int64_t NB, double scale, double k_scale,
                      double v_scale, const int32_t* rows, int nrow, int nthreads) {
    if (S < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || MB < 0)
        return ORC_EARG;
    if (query_start[0] != 0 || query_start[S] != T) return ORC_EARG;
    for (int s = 0; s < S; ++s) {
        int L = query_start[s + 1] - query_start[s];
        if (L < 0 || L > context_lens[s]) return ORC_EARG;
        if ((int64_t)context_lens[s] > (int64_t)MB * bs) return ORC_EARG;
    }
    if (rows)
        for (int i = 0; i < nrow; ++i)
            if (rows[i] < 0 || rows[i] >= T) return ORC_EARG;
    int nt = hw_threads(nthreads);
    prefill_job* jobs = (prefill_job*)calloc((size_t)nt, sizeof(prefill_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nt, sizeof(pthread_t));
    for (int t = 0; t < nt; ++t) {
        decode_job b = {NULL, q, q_dt, key_cache, value_cache, kv_dt, block_tables, MB,
                        context_lens, NULL, 0, Hq, Hkv, D, bs, NB, scale, k_scale, v_scale,
                        nt, t, ORC_OK};
        prefill_job pj = {b, out, query_start, rows, nrow, S, T, ORC_OK};
        jobs[t] = pj;
        pthread_create(&th[t], NULL, prefill_worker, &jobs[t]);
    }
    int status = ORC_OK;
    for (int t = 0; t < nt; ++t) {
        pthread_join(th[t], NULL);
        if (jobs[t].status && !status) status = jobs[t].status;
    }
    free(jobs);
    free(th);
    return status;
}
