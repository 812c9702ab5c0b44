/*
 * rfa_oracle.c -- plain, slow fp64 CPU oracle for rotary position embedding
 * (RoPE) fused into softmax attention, and for the DynamicNTK sin/cos table.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library, and it never calls it.
 *
 * Every function below is the plain definition, written out in fp64 with no
 * blocking, fusion or reordering:
 *   - inverse frequencies   invFreq_j = base^(-2j/D)       (page "RoPE fused
 *     into attention on Ascend", section 1.2, the freqs line of the snippet)
 *   - dynamic-NTK base      base' = base*((f*S/L)-(f-1))^(D/(D-2)) when S > L,
 *     no interpolation when S <= L (page "DynamicNTKOperation", function
 *     description; the closed form is the long-context workload's statement)
 *   - sin/cos table         freq = outer(positionIds_b, invFreq_b),
 *     emb = cat(freq, freq), sin(emb), cos(emb), batch by batch through the
 *     seqLens prefix sums (page "DynamicNTKOperation", computation process)
 *   - rotate-half RoPE      x' = x*cos(emb) + rotate_half(x)*sin(emb), i.e.
 *     x'[i] = x[i]c - x[i+D/2]s, x'[i+D/2] = x[i+D/2]c + x[i]s   (the rotation
 *     the pages elide; rotate-half is the pairing that cat(freq, freq) implies)
 *   - attention             out = softmax(Q'K'^T * scale) V, scale = 1/sqrt(D)
 *     by default (page "FlashAttention in ops-transformer", the attention
 *     formula), causal mask key > query within the sequence, GQA with
 *     contiguous groups kv_head = h / (Hq/Hkv) (page "RoPE, RMSNorm, GQA/MQA",
 *     section 12), softmax taken in two plain passes over the full score row.
 *
 * Build: gcc -O2 -std=c11 -shared -fPIC -pthread rfa_oracle.c -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_BF16 = 0, ORC_FP16 = 1 };
enum { ORC_BNSD = 0, ORC_TND = 1 };

/* Exact widening of a 16-bit float to double. */
static double widen16(uint16_t h, int dtype) {
    if (dtype == ORC_BF16) {
        uint32_t u = ((uint32_t)h) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

double oracle_widen16(uint16_t h, int dtype) { return widen16(h, dtype); }

/* invFreq_j = base^(-2j/D), j < D/2. */
void oracle_inv_freq(double base, int32_t D, double* out) {
    for (int32_t j = 0; j < D / 2; ++j) out[j] = pow(base, -2.0 * (double)j / (double)D);
}

/* Dynamic-NTK base: unchanged while S <= L, enlarged beyond it. */
double oracle_ntk_base(double base, int32_t D, int32_t S, int32_t L, double factor) {
    if (S <= L) return base;
    return base * pow(factor * (double)S / (double)L - (factor - 1.0), (double)D / (double)(D - 2));
}

/*
 * sin/cos table.  invFreq is [batch, headSize/2] (already widened to double),
 * seqLens [batch] must sum to ntokens.  Outputs are [ntokens, headSize].
 * Returns 0, or -1 if the lengths are not positive or do not sum to ntokens.
 */
int oracle_rope_sincos(const int32_t* positionIds, const double* invFreq, const int32_t* seqLens,
                       int32_t batch, int32_t ntokens, int32_t headSize, double* sinOut, double* cosOut) {
    int64_t total = 0;
    for (int32_t b = 0; b < batch; ++b) {
        if (seqLens[b] <= 0) return -1;
        total += seqLens[b];
    }
    if (total != ntokens) return -1;
    const int32_t half = headSize / 2;
    int64_t t = 0;
    for (int32_t b = 0; b < batch; ++b) {
        for (int32_t i = 0; i < seqLens[b]; ++i, ++t) {
            for (int32_t j = 0; j < headSize; ++j) {
                double a = (double)positionIds[t] * invFreq[(int64_t)b * half + (j % half)];
                sinOut[t * headSize + j] = sin(a);
                cosOut[t * headSize + j] = cos(a);
            }
        }
    }
    return 0;
}

/* Rotate-half RoPE of n rows of width D, row r at position pos[r]. */
void oracle_rope_rotate(const double* x, int64_t n, int32_t D, const int32_t* pos, const double* invFreq,
                        double* out) {
    const int32_t half = D / 2;
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t i = 0; i < half; ++i) {
            double a = (double)pos[r] * invFreq[i];
            double c = cos(a), s = sin(a);
            double x1 = x[r * D + i], x2 = x[r * D + i + half];
            out[r * D + i] = x1 * c - x2 * s;
            out[r * D + i + half] = x2 * c + x1 * s;
        }
    }
}

/* The Rope operator of page "DynamicNTKOperation" (operator context: q, k,
 * sin and cos go in, rotated q and k come out), for n rows of width D whose
 * row r uses table row trow[r] of sin/cos [*, D]:
 *   out[j] = x[j] * cos[j] + rot(x)[j] * sin[j]
 * rotate-half pairs (interleaved == 0): rot(x) = (-x[D/2..D), x[0..D/2));
 * adjacent pairs (interleaved != 0, the (x1,x2),(x3,x4),... blocks of page
 * "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 6): rot(x)[2i] = -x[2i+1],
 * rot(x)[2i+1] = x[2i]. */
void oracle_rope_apply(const double* x, int64_t n, int32_t D, const double* sin_t, const double* cos_t,
                       const int64_t* trow, int32_t interleaved, double* out) {
    const int32_t half = D / 2;
    for (int64_t r = 0; r < n; ++r) {
        const double* xr = x + r * D;
        const double* s = sin_t + trow[r] * D;
        const double* c = cos_t + trow[r] * D;
        for (int32_t j = 0; j < D; ++j) {
            double rx;
            if (interleaved)
                rx = (j & 1) ? xr[j - 1] : -xr[j + 1];
            else
                rx = (j < half) ? -xr[j + half] : xr[j - half];
            out[r * D + j] = xr[j] * c[j] + rx * s[j];
        }
    }
}

/* RMSNorm of n rows of width D (page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE",
 * sec. 8): out = gamma * x / sqrt(mean(x^2) + eps). */
void oracle_rms_norm(const double* x, int64_t n, int32_t D, const double* gamma, double eps, double* out) {
    for (int64_t r = 0; r < n; ++r) {
        double ss = 0.0;
        for (int32_t j = 0; j < D; ++j) ss += x[r * D + j] * x[r * D + j];
        const double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int32_t j = 0; j < D; ++j) out[r * D + j] = gamma[j] * (x[r * D + j] * inv);
    }
}

typedef struct {
    int32_t layout;  /* ORC_BNSD: q [B,Hq,S,D], k/v [B,Hkv,S,D], pos [B,S]
                        ORC_TND : q [T,Hq,D],   k/v [T,Hkv,D],   pos [T]   */
    int32_t dtype;   /* ORC_BF16 or ORC_FP16 for q, k, v */
    int32_t B;       /* batches (BNSD) or packed sequences (TND) */
    int32_t Hq, Hkv;
    int32_t S;       /* BNSD sequence length (ignored for TND) */
    int32_t D;
    int32_t causal;
    double scale;    /* multiplies q'.k' */
    int32_t nthreads;
    int32_t interleaved; /* 0: rotate-half pairs (i, i + D/2); 1: adjacent pairs (2i, 2i+1) */
} oracle_attn_desc;

/* RoPE of one row at position pos: rotate-half, or adjacent pairs (the
 * (x1,x2),(x3,x4),... blocks of page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE",
 * sec. 6), pair i turned by pos * invFreq[i]. */
static void rotate_row(const oracle_attn_desc* d, const double* x, int32_t pos, const double* invFreq, double* out) {
    if (!d->interleaved) {
        oracle_rope_rotate(x, 1, d->D, &pos, invFreq, out);
        return;
    }
    for (int32_t i = 0; i < d->D / 2; ++i) {
        double a = (double)pos * invFreq[i];
        double c = cos(a), s = sin(a);
        double x1 = x[2 * i], x2 = x[2 * i + 1];
        out[2 * i] = x1 * c - x2 * s;
        out[2 * i + 1] = x2 * c + x1 * s;
    }
}

typedef struct {
    const oracle_attn_desc* d;
    const uint16_t *q, *k, *v;
    const int32_t* pos;
    const double* invFreq; /* [B, D/2] */
    int64_t tok0;          /* first token of this sequence (TND) */
    int32_t b, kvh, len;
    double *Kr, *Vd;       /* [len, D] rotated keys, widened values */
    const int32_t* rows;   /* (b, h, i) triples */
    const int64_t* sel;    /* indices into rows that belong to this group */
    int64_t nsel;
    double* out;
    int32_t tid, nthreads;
} group_job;

static int64_t q_off(const oracle_attn_desc* d, int64_t tok0, int32_t b, int32_t h, int32_t i) {
    if (d->layout == ORC_BNSD) return (((int64_t)b * d->Hq + h) * d->S + i) * d->D;
    return ((tok0 + i) * d->Hq + h) * (int64_t)d->D;
}
static int64_t kv_off(const oracle_attn_desc* d, int64_t tok0, int32_t b, int32_t kh, int32_t j) {
    if (d->layout == ORC_BNSD) return (((int64_t)b * d->Hkv + kh) * d->S + j) * d->D;
    return ((tok0 + j) * d->Hkv + kh) * (int64_t)d->D;
}
static int32_t pos_at(const oracle_attn_desc* d, const int32_t* pos, int64_t tok0, int32_t b, int32_t i) {
    if (d->layout == ORC_BNSD) return pos[(int64_t)b * d->S + i];
    return pos[tok0 + i];
}

/* Phase 1: rotated K and widened V of one (sequence, kv head). */
static void* prep_kv(void* arg) {
    group_job* g = (group_job*)arg;
    const oracle_attn_desc* d = g->d;
    const int32_t D = d->D;
    double* xk = (double*)malloc(sizeof(double) * D);
    for (int32_t j = g->tid; j < g->len; j += g->nthreads) {
        int64_t o = kv_off(d, g->tok0, g->b, g->kvh, j);
        for (int32_t c = 0; c < D; ++c) {
            xk[c] = widen16(g->k[o + c], d->dtype);
            g->Vd[(int64_t)j * D + c] = widen16(g->v[o + c], d->dtype);
        }
        int32_t p = pos_at(d, g->pos, g->tok0, g->b, j);
        rotate_row(d, xk, p, g->invFreq + (int64_t)g->b * (D / 2), g->Kr + (int64_t)j * D);
    }
    free(xk);
    return NULL;
}

/* Phase 2: each selected query row, two-pass softmax over its full score row. */
static void* rows_job(void* arg) {
    group_job* g = (group_job*)arg;
    const oracle_attn_desc* d = g->d;
    const int32_t D = d->D;
    double* xq = (double*)malloc(sizeof(double) * D);
    double* qr = (double*)malloc(sizeof(double) * D);
    double* s = (double*)malloc(sizeof(double) * (g->len > 0 ? g->len : 1));
    for (int64_t n = g->tid; n < g->nsel; n += g->nthreads) {
        int64_t r = g->sel[n];
        int32_t h = g->rows[3 * r + 1], i = g->rows[3 * r + 2];
        double* o = g->out + r * D;
        int64_t qo = q_off(d, g->tok0, g->b, h, i);
        for (int32_t c = 0; c < D; ++c) xq[c] = widen16(g->q[qo + c], d->dtype);
        int32_t p = pos_at(d, g->pos, g->tok0, g->b, i);
        rotate_row(d, xq, p, g->invFreq + (int64_t)g->b * (D / 2), qr);
        int32_t jmax = d->causal ? i + 1 : g->len;
        /* pass 1: scores and their maximum */
        double m = -INFINITY;
        for (int32_t j = 0; j < jmax; ++j) {
            double acc = 0.0;
            const double* kr = g->Kr + (int64_t)j * D;
            for (int32_t c = 0; c < D; ++c) acc += qr[c] * kr[c];
            s[j] = acc * d->scale;
            if (s[j] > m) m = s[j];
        }
        /* pass 2: exponentials, their sum, and the weighted sum of values */
        for (int32_t c = 0; c < D; ++c) o[c] = 0.0;
        if (jmax <= 0) continue; /* no visible key: defined as a zero row */
        double z = 0.0;
        for (int32_t j = 0; j < jmax; ++j) {
            s[j] = exp(s[j] - m);
            z += s[j];
        }
        for (int32_t j = 0; j < jmax; ++j) {
            double w = s[j] / z;
            const double* vr = g->Vd + (int64_t)j * D;
            for (int32_t c = 0; c < D; ++c) o[c] += w * vr[c];
        }
    }
    free(xq);
    free(qr);
    free(s);
    return NULL;
}

static void run_threads(void* (*fn)(void*), group_job* base, int32_t nthreads) {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    group_job* jobs = (group_job*)malloc(sizeof(group_job) * nthreads);
    for (int32_t t = 0; t < nthreads; ++t) {
        jobs[t] = *base;
        jobs[t].tid = t;
        jobs[t].nthreads = nthreads;
        if (nthreads > 1)
            pthread_create(&th[t], NULL, fn, &jobs[t]);
        else
            fn(&jobs[t]);
    }
    if (nthreads > 1)
        for (int32_t t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(jobs);
}

/*
 * Attention output rows.  rows is [nrows, 3] of (b, h, i): sequence b, query
 * head h, query index i within the sequence.  out is [nrows, D].  seqLens
 * (TND only) gives the packed sequence lengths.  invFreq is [B, D/2] per
 * sequence.  Returns 0, or -1 on an invalid row or descriptor.
 */
int oracle_attention_rows(const oracle_attn_desc* d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* pos, const int32_t* seqLens, const double* invFreq,
                          const int32_t* rows, int64_t nrows, double* out) {
    if (d->D <= 0 || (d->D & 1) || d->Hkv <= 0 || d->Hq % d->Hkv != 0 || d->B <= 0) return -1;
    const int32_t G = d->Hq / d->Hkv;
    const int32_t D = d->D;
    int32_t nthreads = d->nthreads > 0 ? d->nthreads : 1;
    int64_t* tok0 = (int64_t*)malloc(sizeof(int64_t) * (d->B + 1));
    tok0[0] = 0;
    for (int32_t b = 0; b < d->B; ++b)
        tok0[b + 1] = tok0[b] + (d->layout == ORC_TND ? seqLens[b] : d->S);
    for (int64_t r = 0; r < nrows; ++r) {
        int32_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        int64_t len = tok0[b + 1] - tok0[b];
        if (b < 0 || b >= d->B || h < 0 || h >= d->Hq || i < 0 || i >= len) {
            free(tok0);
            return -1;
        }
    }
    int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (nrows > 0 ? nrows : 1));
    for (int32_t b = 0; b < d->B; ++b) {
        int32_t len = (int32_t)(tok0[b + 1] - tok0[b]);
        for (int32_t kvh = 0; kvh < d->Hkv; ++kvh) {
            int64_t nsel = 0;
            for (int64_t r = 0; r < nrows; ++r)
                if (rows[3 * r] == b && rows[3 * r + 1] / G == kvh) sel[nsel++] = r;
            if (nsel == 0) continue;
            group_job g;
            memset(&g, 0, sizeof g);
            g.d = d;
            g.q = q;
            g.k = k;
            g.v = v;
            g.pos = pos;
            g.invFreq = invFreq;
            g.tok0 = tok0[b];
            g.b = b;
            g.kvh = kvh;
            g.len = len;
            g.Kr = (double*)malloc(sizeof(double) * (size_t)len * D + 8);
            g.Vd = (double*)malloc(sizeof(double) * (size_t)len * D + 8);
            g.rows = rows;
            g.sel = sel;
            g.nsel = nsel;
            g.out = out;
            run_threads(prep_kv, &g, nthreads);
            run_threads(rows_job, &g, nthreads);
            free(g.Kr);
            free(g.Vd);
        }
    }
    free(sel);
    free(tok0);
    return 0;
}

/*
 * One full softmax row P[b, h, i, :] (length of sequence b), for checks on
 * the probabilities themselves.  Entries past the causal limit are zero.
 */
int oracle_attention_probs(const oracle_attn_desc* d, const uint16_t* q, const uint16_t* k, const int32_t* pos,
                           const int32_t* seqLens, const double* invFreq, int32_t b, int32_t h, int32_t i,
                           double* p) {
    if (d->Hkv <= 0 || d->Hq % d->Hkv != 0 || b < 0 || b >= d->B || h < 0 || h >= d->Hq) return -1;
    const int32_t D = d->D, G = d->Hq / d->Hkv, kvh = h / G;
    int64_t t0 = 0;
    int32_t len = d->S;
    if (d->layout == ORC_TND) {
        for (int32_t bb = 0; bb < b; ++bb) t0 += seqLens[bb];
        len = seqLens[b];
    }
    if (i < 0 || i >= len) return -1;
    double* x = (double*)malloc(sizeof(double) * D);
    double* qr = (double*)malloc(sizeof(double) * D);
    double* kr = (double*)malloc(sizeof(double) * D);
    int64_t qo = q_off(d, t0, b, h, i);
    for (int32_t c = 0; c < D; ++c) x[c] = widen16(q[qo + c], d->dtype);
    int32_t pq = pos_at(d, pos, t0, b, i);
    const double* inv = invFreq + (int64_t)b * (D / 2);
    rotate_row(d, x, pq, inv, qr);
    int32_t jmax = d->causal ? i + 1 : len;
    double m = -INFINITY;
    for (int32_t j = 0; j < len; ++j) {
        if (j >= jmax) {
            p[j] = 0.0;
            continue;
        }
        int64_t ko = kv_off(d, t0, b, kvh, j);
        for (int32_t c = 0; c < D; ++c) x[c] = widen16(k[ko + c], d->dtype);
        int32_t pk = pos_at(d, pos, t0, b, j);
        rotate_row(d, x, pk, inv, kr);
        double acc = 0.0;
        for (int32_t c = 0; c < D; ++c) acc += qr[c] * kr[c];
        p[j] = acc * d->scale;
        if (p[j] > m) m = p[j];
    }
    double z = 0.0;
    for (int32_t j = 0; j < jmax; ++j) {
        p[j] = exp(p[j] - m);
        z += p[j];
    }
    for (int32_t j = 0; j < jmax; ++j) p[j] /= z;
    free(x);
    free(qr);
    free(kr);
    return 0;
}
