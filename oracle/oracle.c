/*
 * oracle.c -- plain CPU reference of single-request (batch 1) autoregressive decode
 * of a dense decoder-only transformer, one token at a time.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA decode library never links,
 * calls or reads it, and the two share no source, header, table or constant generator.
 *
 * What it computes. The pages describe the decode path as one program that covers the
 * matrix products, attention, normalisation and sampling for one request, one token at a time
 * ("Breaking the memory wall: 3,000 tokens/s on standard GPUs", agentlenshq.com, section
 * "1. The Monokernel Runtime"; "3000 tokens per second: how to speed up LLMs on ordinary
 * GPUs", aikraft.ru, section 04 "Monokernel and optimized GPU code"), and they say the
 * engine keeps the model's output exact: no quantisation, speculative decoding, pruning or
 * KV-cache compression ("Kog inference engine: no precision cut, 3000 tokens/s per
 * request", zdabc.icu, opening section). So this oracle is the plain definition of the
 * pre-norm decoder step, written as scalar loops with no blocking, fusion or reordering:
 *
 *   x   = float(E[tok])
 *   per layer:  xn = rmsnorm(x, g_attn); q,k,v = Wq xn, Wk xn, Wv xn; rope(q,k, pos);
 *               Kc[pos] = bf16(k), Vc[pos] = bf16(v); o_h = softmax(q_h.Kc/sqrt(hd)) Vc;
 *               x += Wo o; xn = rmsnorm(x, g_ffn); x += Wd (silu(Wg xn) * (Wu xn))
 *   xn = rmsnorm(x, g_final); logits = W_lm xn; next = argmax(logits), lowest index on ties
 *
 * The pages never name the layer algebra (RoPE, GQA, SwiGLU, RMSNorm, untied head, greedy
 * argmax); it is fixed by the workload definitions this library is tested on. Where the
 * pages are silent the plainest reading is taken: rotate-half RoPE pairs (i, i+hd/2) with
 * frequency theta^(-2i/hd); contiguous GQA groups (q head h reads kv head h*Hkv/Hq); scale
 * 1/sqrt(hd); eps inside the square root, gain applied after normalising; no biases; the
 * KV cache stores bf16 rounded to nearest even, K after RoPE.
 *
 * Precision: fp32 arithmetic over bf16 weights (bf16 -> fp32 widening is exact). RoPE
 * angles are formed in fp64 and their cos/sin rounded to fp32. Every dot product is
 * summed in ascending index order by one thread, so the optional row-parallel mode
 * (n_threads > 1) is bit-identical to the single-threaded mode.
 *
 * Bytes model: the step counts the bytes it reads from the weights and the KV cache,
 * each distinct element once (a kv head serving several q heads is counted once). The
 * pages' light-speed bound divides bandwidth by exactly this quantity (aikraft.ru,
 * section 02 "The main enemy of speed: memory bandwidth, not FLOPS").
 *
 * Parity status of each function (what pins it, other than itself):
 *   orc_bf16_round   -- pinned: matches a library fp32->bf16 conversion on ties and edges.
 *   orc_rmsnorm      -- pinned: closed form for constant vectors; library rms_norm.
 *   orc_rope         -- pinned: identity at position 0, norm preservation, relative-position
 *                       invariance, library rotary embedding (rotate-half convention).
 *   orc_attend       -- pinned: one-entry cache returns V; equal keys give mean(V); library
 *                       scaled-dot-product attention.
 *   orc_silu         -- pinned: silu(0)=0, asymptotes, library silu.
 *   orc_argmax       -- pinned: brute force with planted ties.
 *   orc_matvec       -- pinned: library matmul in fp64 within the fp32 summation bound.
 *   orc_step         -- pinned: an independent fp64 full-sequence causal forward (matrices,
 *                       causal mask) reproduces every decode step; a library Llama-style
 *                       model in fp64 agrees within the bf16 KV-rounding bound; zero-weight
 *                       special cases; counted bytes equal the closed form.
 *   The conventions listed above (RoPE pairing, GQA grouping) are parity unpinned against
 *   the pages themselves, which print no worked example of the layer algebra.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

typedef struct {
    int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab;
    int32_t capacity;  /* KV positions the oracle can hold */
    int32_t n_threads; /* 1 = single-threaded; >1 = row-parallel, bit-identical */
    float rms_eps, rope_theta;
} orc_config;

/* bf16 tensors as raw 16-bit patterns, row-major [out][in], stacked over layers. */
typedef struct {
    const uint16_t *embed;      /* [vocab][d] */
    const uint16_t *attn_norm;  /* [L][d] */
    const uint16_t *wq;         /* [L][Hq*hd][d] */
    const uint16_t *wk;         /* [L][Hkv*hd][d] */
    const uint16_t *wv;         /* [L][Hkv*hd][d] */
    const uint16_t *wo;         /* [L][d][Hq*hd] */
    const uint16_t *ffn_norm;   /* [L][d] */
    const uint16_t *wg;         /* [L][F][d] */
    const uint16_t *wu;         /* [L][F][d] */
    const uint16_t *wd;         /* [L][d][F] */
    const uint16_t *final_norm; /* [d] */
    const uint16_t *lm_head;    /* [vocab][d] */
} orc_weights;

/* ---------------------------------------------------------------- scalar helpers */

ORC_API float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
ORC_API uint16_t orc_bf16_round(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

ORC_API float orc_silu(float z) { return z / (1.0f + expf(-z)); }

/* First index holding the maximum (strict >), i.e. the lowest index wins a tie. */
ORC_API int32_t orc_argmax(const float *v, int32_t n) {
    int32_t best = 0;
    for (int32_t i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* out[i] = x[i] / sqrt(mean(x^2) + eps) * g[i] */
ORC_API void orc_rmsnorm(const float *x, const uint16_t *g, int32_t n, float eps, float *out) {
    float ss = 0.0f;
    for (int32_t i = 0; i < n; ++i) ss += x[i] * x[i];
    float inv = 1.0f / sqrtf(ss / (float)n + eps);
    for (int32_t i = 0; i < n; ++i) out[i] = (x[i] * inv) * orc_bf16_to_f32(g[i]);
}

/* Rotate one head vector in place at absolute position pos (rotate-half pairing). */
ORC_API void orc_rope(float *v, int32_t hd, int32_t pos, float theta) {
    int32_t half = hd / 2;
    for (int32_t i = 0; i < half; ++i) {
        double freq = pow((double)theta, -2.0 * (double)i / (double)hd);
        double ang = (double)pos * freq;
        float c = (float)cos(ang), s = (float)sin(ang);
        float a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* y[r] = sum_k W[r][k] * x[k], ascending k, fp32 accumulation. */
static void matvec_rows(const uint16_t *W, const float *x, int32_t cols, float *y, int32_t r0,
                        int32_t r1) {
    for (int32_t r = r0; r < r1; ++r) {
        const uint16_t *w = W + (size_t)r * (size_t)cols;
        float acc = 0.0f;
        for (int32_t k = 0; k < cols; ++k) acc += orc_bf16_to_f32(w[k]) * x[k];
        y[r] = acc;
    }
}

ORC_API void orc_matvec(const uint16_t *W, const float *x, int32_t rows, int32_t cols, float *y) {
    matvec_rows(W, x, cols, y, 0, rows);
}

/* One q head over T cached positions: softmax(q.K_j * scale) weighted sum of V_j.
 * K, V are [T][hd] bf16. */
ORC_API void orc_attend(const float *q, const uint16_t *K, const uint16_t *V, int32_t T, int32_t hd,
                        float *out, float *scratch /* [T] */) {
    float scale = 1.0f / sqrtf((float)hd);
    float mx = -INFINITY;
    for (int32_t j = 0; j < T; ++j) {
        const uint16_t *k = K + (size_t)j * hd;
        float s = 0.0f;
        for (int32_t i = 0; i < hd; ++i) s += q[i] * orc_bf16_to_f32(k[i]);
        s *= scale;
        scratch[j] = s;
        if (s > mx) mx = s;
    }
    float sum = 0.0f;
    for (int32_t j = 0; j < T; ++j) {
        scratch[j] = expf(scratch[j] - mx);
        sum += scratch[j];
    }
    for (int32_t i = 0; i < hd; ++i) out[i] = 0.0f;
    for (int32_t j = 0; j < T; ++j) {
        float w = scratch[j] / sum;
        const uint16_t *v = V + (size_t)j * hd;
        for (int32_t i = 0; i < hd; ++i) out[i] += w * orc_bf16_to_f32(v[i]);
    }
}

/* ---------------------------------------------------------------- worker pool
 * Splits a row range into n_threads static blocks. Each row is computed entirely by one
 * thread in the same order as the single-threaded path, so results do not depend on the
 * thread count. */

typedef void (*row_fn)(void *arg, int32_t r0, int32_t r1);

typedef struct {
    int n;
    pthread_t *th;
    pthread_mutex_t mu;
    pthread_cond_t go, done;
    long gen;
    int remaining, stop;
    row_fn fn;
    void *arg;
    int32_t rows;
} pool;

typedef struct {
    pool *p;
    int id;
} pool_slot;

static void pool_block(pool *p, int id, int32_t *r0, int32_t *r1) {
    int64_t rows = p->rows;
    *r0 = (int32_t)(rows * id / p->n);
    *r1 = (int32_t)(rows * (id + 1) / p->n);
}

static void *pool_worker(void *vs) {
    pool_slot *s = (pool_slot *)vs;
    pool *p = s->p;
    long seen = 0;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        while (p->gen == seen && !p->stop) pthread_cond_wait(&p->go, &p->mu);
        if (p->stop) {
            pthread_mutex_unlock(&p->mu);
            break;
        }
        seen = p->gen;
        pthread_mutex_unlock(&p->mu);
        int32_t r0, r1;
        pool_block(p, s->id, &r0, &r1);
        if (r1 > r0) p->fn(p->arg, r0, r1);
        pthread_mutex_lock(&p->mu);
        if (--p->remaining == 0) pthread_cond_signal(&p->done);
        pthread_mutex_unlock(&p->mu);
    }
    free(s);
    return NULL;
}

static pool *pool_new(int n) {
    pool *p = (pool *)calloc(1, sizeof *p);
    p->n = n < 1 ? 1 : n;
    pthread_mutex_init(&p->mu, NULL);
    pthread_cond_init(&p->go, NULL);
    pthread_cond_init(&p->done, NULL);
    p->th = (pthread_t *)calloc((size_t)p->n, sizeof(pthread_t));
    for (int i = 1; i < p->n; ++i) {
        pool_slot *s = (pool_slot *)malloc(sizeof *s);
        s->p = p;
        s->id = i;
        pthread_create(&p->th[i], NULL, pool_worker, s);
    }
    return p;
}

static void pool_free(pool *p) {
    pthread_mutex_lock(&p->mu);
    p->stop = 1;
    pthread_cond_broadcast(&p->go);
    pthread_mutex_unlock(&p->mu);
    for (int i = 1; i < p->n; ++i) pthread_join(p->th[i], NULL);
    free(p->th);
    free(p);
}

static void pool_run(pool *p, int32_t rows, row_fn fn, void *arg) {
    if (p->n == 1) {
        fn(arg, 0, rows);
        return;
    }
    pthread_mutex_lock(&p->mu);
    p->fn = fn;
    p->arg = arg;
    p->rows = rows;
    p->remaining = p->n - 1;
    p->gen++;
    pthread_cond_broadcast(&p->go);
    pthread_mutex_unlock(&p->mu);
    int32_t r0, r1;
    pool_block(p, 0, &r0, &r1);
    if (r1 > r0) fn(arg, r0, r1);
    pthread_mutex_lock(&p->mu);
    while (p->remaining > 0) pthread_cond_wait(&p->done, &p->mu);
    pthread_mutex_unlock(&p->mu);
}

/* ---------------------------------------------------------------- decoder state */

typedef struct {
    orc_config c;
    orc_weights w;
    int has_weights;
    uint16_t *kc, *vc; /* [L][Hkv][capacity][hd] bf16 */
    float *x, *xn, *q, *k, *v, *o, *g, *u, *hdn, *tmp, *att;
    pool *pool;
} orc;

typedef struct {
    const uint16_t *W;
    const float *x;
    int32_t cols;
    float *y;
} mv_job;

static void mv_job_fn(void *a, int32_t r0, int32_t r1) {
    mv_job *j = (mv_job *)a;
    matvec_rows(j->W, j->x, j->cols, j->y, r0, r1);
}

static void matvec(orc *o, const uint16_t *W, const float *x, int32_t rows, int32_t cols, float *y,
                   double *bytes) {
    mv_job j = {W, x, cols, y};
    pool_run(o->pool, rows, mv_job_fn, &j);
    *bytes += 2.0 * (double)rows * (double)cols;
}

typedef struct {
    orc *o;
    int32_t layer, T;
} att_job;

static void att_job_fn(void *a, int32_t h0, int32_t h1) {
    att_job *j = (att_job *)a;
    orc *o = j->o;
    const orc_config *c = &o->c;
    int32_t hd = c->head_dim;
    for (int32_t h = h0; h < h1; ++h) {
        int32_t g = h * c->n_kv_heads / c->n_heads; /* contiguous GQA group */
        size_t base = (((size_t)j->layer * c->n_kv_heads + g) * c->capacity) * hd;
        orc_attend(o->q + (size_t)h * hd, o->kc + base, o->vc + base, j->T, hd, o->o + (size_t)h * hd,
                   o->att + (size_t)h * c->capacity);
    }
}

ORC_API orc *orc_new(const orc_config *c) {
    if (!c || c->n_layers < 0 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 ||
        c->n_heads % c->n_kv_heads || c->head_dim <= 0 || (c->head_dim & 1) || c->ffn_dim <= 0 ||
        c->vocab <= 0 || c->capacity <= 0)
        return NULL;
    orc *o = (orc *)calloc(1, sizeof *o);
    o->c = *c;
    size_t kv = (size_t)c->n_layers * c->n_kv_heads * c->capacity * c->head_dim;
    o->kc = (uint16_t *)calloc(kv ? kv : 1, sizeof(uint16_t));
    o->vc = (uint16_t *)calloc(kv ? kv : 1, sizeof(uint16_t));
    size_t qd = (size_t)c->n_heads * c->head_dim, kd = (size_t)c->n_kv_heads * c->head_dim;
    o->x = (float *)calloc(c->d_model, sizeof(float));
    o->xn = (float *)calloc(c->d_model, sizeof(float));
    o->tmp = (float *)calloc(c->d_model, sizeof(float));
    o->q = (float *)calloc(qd, sizeof(float));
    o->o = (float *)calloc(qd, sizeof(float));
    o->k = (float *)calloc(kd, sizeof(float));
    o->v = (float *)calloc(kd, sizeof(float));
    o->g = (float *)calloc(c->ffn_dim, sizeof(float));
    o->u = (float *)calloc(c->ffn_dim, sizeof(float));
    o->hdn = (float *)calloc(c->ffn_dim, sizeof(float));
    o->att = (float *)calloc((size_t)c->n_heads * c->capacity, sizeof(float));
    if (!o->kc || !o->vc || !o->x || !o->xn || !o->tmp || !o->q || !o->o || !o->k || !o->v || !o->g ||
        !o->u || !o->hdn || !o->att) {
        free(o->kc), free(o->vc), free(o->x), free(o->xn), free(o->tmp), free(o->q), free(o->o);
        free(o->k), free(o->v), free(o->g), free(o->u), free(o->hdn), free(o->att), free(o);
        return NULL;
    }
    o->pool = pool_new(c->n_threads);
    return o;
}

ORC_API void orc_free(orc *o) {
    if (!o) return;
    pool_free(o->pool);
    free(o->kc), free(o->vc), free(o->x), free(o->xn), free(o->tmp), free(o->q), free(o->o);
    free(o->k), free(o->v), free(o->g), free(o->u), free(o->hdn), free(o->att), free(o);
}

/* The weight arrays stay owned by the caller and must outlive every orc_step call. */
ORC_API int orc_set_weights(orc *o, const orc_weights *w) {
    if (!o || !w || !w->embed || !w->final_norm || !w->lm_head) return -1;
    if (o->c.n_layers > 0 && (!w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo || !w->ffn_norm ||
                              !w->wg || !w->wu || !w->wd))
        return -1;
    o->w = *w;
    o->has_weights = 1;
    return 0;
}

/* Fill KV positions [0, n) of one layer from src laid out [Hkv][n][hd] (bf16 patterns).
 * which: 0 = K (already rotated), 1 = V. */
ORC_API int orc_set_kv(orc *o, int32_t layer, int32_t which, const uint16_t *src, int32_t n) {
    const orc_config *c = &o->c;
    if (layer < 0 || layer >= c->n_layers || n < 0 || n > c->capacity || (which != 0 && which != 1))
        return -1;
    uint16_t *dst = which ? o->vc : o->kc;
    for (int32_t g = 0; g < c->n_kv_heads; ++g) {
        size_t db = (((size_t)layer * c->n_kv_heads + g) * c->capacity) * c->head_dim;
        size_t sb = (size_t)g * n * c->head_dim;
        memcpy(dst + db, src + sb, (size_t)n * c->head_dim * sizeof(uint16_t));
    }
    return 0;
}

/* Copy one layer's cached K or V rows [0, n) out, laid out [Hkv][n][hd]. */
ORC_API int orc_get_kv(const orc *o, int32_t layer, int32_t which, uint16_t *dst, int32_t n) {
    const orc_config *c = &o->c;
    if (layer < 0 || layer >= c->n_layers || n < 0 || n > c->capacity || (which != 0 && which != 1))
        return -1;
    const uint16_t *src = which ? o->vc : o->kc;
    for (int32_t g = 0; g < c->n_kv_heads; ++g) {
        size_t sb = (((size_t)layer * c->n_kv_heads + g) * c->capacity) * c->head_dim;
        memcpy(dst + (size_t)g * n * c->head_dim, src + sb, (size_t)n * c->head_dim * sizeof(uint16_t));
    }
    return 0;
}

/*
 * One decode step: feed `token` at absolute position `pos` (cache positions [0, pos) must
 * already hold K/V), append its K/V at `pos`, and, when logits or next is non-NULL, run
 * the final norm, the LM head and the greedy argmax. *bytes receives the bytes read from
 * weights and KV cache. Returns 0, or -1 on a bad argument.
 */
ORC_API int orc_step(orc *o, int32_t token, int32_t pos, float *logits, int32_t *next, double *bytes) {
    if (!o || !o->has_weights) return -1;
    const orc_config *c = &o->c;
    const orc_weights *w = &o->w;
    if (token < 0 || token >= c->vocab || pos < 0 || pos >= c->capacity) return -1;
    const int32_t d = c->d_model, hd = c->head_dim, Hq = c->n_heads, Hkv = c->n_kv_heads;
    const int32_t F = c->ffn_dim, qd = Hq * hd, kd = Hkv * hd, T = pos + 1;
    double nb = 0.0;

    const uint16_t *e = w->embed + (size_t)token * d;
    for (int32_t i = 0; i < d; ++i) o->x[i] = orc_bf16_to_f32(e[i]);
    nb += 2.0 * d;

    for (int32_t l = 0; l < c->n_layers; ++l) {
        /* attention block */
        orc_rmsnorm(o->x, w->attn_norm + (size_t)l * d, d, c->rms_eps, o->xn);
        nb += 2.0 * d;
        matvec(o, w->wq + (size_t)l * qd * d, o->xn, qd, d, o->q, &nb);
        matvec(o, w->wk + (size_t)l * kd * d, o->xn, kd, d, o->k, &nb);
        matvec(o, w->wv + (size_t)l * kd * d, o->xn, kd, d, o->v, &nb);
        for (int32_t h = 0; h < Hq; ++h) orc_rope(o->q + (size_t)h * hd, hd, pos, c->rope_theta);
        for (int32_t g = 0; g < Hkv; ++g) orc_rope(o->k + (size_t)g * hd, hd, pos, c->rope_theta);
        for (int32_t g = 0; g < Hkv; ++g) {
            size_t at = ((((size_t)l * Hkv + g) * c->capacity) + pos) * hd;
            for (int32_t i = 0; i < hd; ++i) {
                o->kc[at + i] = orc_bf16_round(o->k[(size_t)g * hd + i]);
                o->vc[at + i] = orc_bf16_round(o->v[(size_t)g * hd + i]);
            }
        }
        att_job aj = {o, l, T};
        pool_run(o->pool, Hq, att_job_fn, &aj);
        nb += 2.0 * 2.0 * (double)Hkv * T * hd; /* each kv head's K and V rows read once */
        matvec(o, w->wo + (size_t)l * d * qd, o->o, d, qd, o->tmp, &nb);
        for (int32_t i = 0; i < d; ++i) o->x[i] += o->tmp[i];

        /* feed-forward block */
        orc_rmsnorm(o->x, w->ffn_norm + (size_t)l * d, d, c->rms_eps, o->xn);
        nb += 2.0 * d;
        matvec(o, w->wg + (size_t)l * F * d, o->xn, F, d, o->g, &nb);
        matvec(o, w->wu + (size_t)l * F * d, o->xn, F, d, o->u, &nb);
        for (int32_t i = 0; i < F; ++i) o->hdn[i] = orc_silu(o->g[i]) * o->u[i];
        matvec(o, w->wd + (size_t)l * d * F, o->hdn, d, F, o->tmp, &nb);
        for (int32_t i = 0; i < d; ++i) o->x[i] += o->tmp[i];
    }

    if (logits || next) {
        float *lg = logits ? logits : (float *)malloc((size_t)c->vocab * sizeof(float));
        if (!lg) return -1;
        orc_rmsnorm(o->x, w->final_norm, d, c->rms_eps, o->xn);
        nb += 2.0 * d;
        matvec(o, w->lm_head, o->xn, c->vocab, d, lg, &nb);
        if (next) *next = orc_argmax(lg, c->vocab);
        if (!logits) free(lg);
    }
    if (bytes) *bytes = nb;
    return 0;
}
