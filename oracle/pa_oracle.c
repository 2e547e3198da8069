/*
 * pa_oracle.c -- fp64 CPU oracle for paged attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg call this code. It shares nothing with the CUDA library: no header, no
 * helper, no table. It is deliberately plain and slow.
 *
 * What it computes is the dense definition of attention from boostr's
 * `standard_attention_fwd` (flash_standard.rs): scores = Q.K^T * scale, an additive 0/-inf
 * mask, lse = logsumexp(scores) over the key axis, out = softmax(scores).V, with GQA query
 * head h reading KV head h / (Hq/Hkv) (`expand_kv`, repeat_interleave on the head axis).
 * The paged part follows ruDNN's `DevicePlan::attention` contract: K/V live in a paged cache
 * [pages, page_size, Hkv, D] reached through each sequence's block table; the oracle first
 * materialises each sequence's K/V contiguously (key t sits in page block_table[s][t / ps],
 * slot t % ps), then runs the dense definition on it.
 *
 * Readings where the pages leave a step open (each is listed in the design notes):
 *  - causal masking uses absolute, right-aligned positions: query j of a sequence with n
 *    queries and L keys (L includes the sequence's own new keys) sits at p = L - n + j
 *    (ruDNN "absolute positions ... including prefill chunks"; alice-llm "right-aligned
 *    causal mask"). Key t is masked when t > p.
 *  - the sliding window masks key t when t + window <= p (boostr `build_attention_mask`),
 *    window 0 meaning no window; it applies whether or not the mask is causal.
 *  - a row with no visible key gets out = 0 and lse = -inf.
 *  - lse is the natural-log logsumexp of the scaled, masked scores.
 * MLA (ruDNN `DevicePlan::mla`): score = scale * (q_lat . latent_t + q_rope . rope_t); the
 * latent is both key and value, so out has the latent width R.
 * Sparse top-K (alice-llm `llama3_sparse_attention`): proxy block scores from the first query
 * head of each group, top-K blocks per (query, kv head), attention over the selected blocks.
 * Readings: a sequence has ceil(L / block_size) blocks (the last may be partial), so that
 * "every block selected" is dense attention; the proxy score of a block is the largest scaled
 * score over the keys of the block the query can see (-inf if none); equal scores rank the
 * lower block index first.
 *
 * Inputs are the exact stored values (fp32, bf16 or fp16 bit patterns) widened to double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PAO_F32 0
#define PAO_BF16 1
#define PAO_F16 2

/* Exact widening of one stored element to double. */
static double pao_load(const void* base, int dtype, int64_t i) {
    if (dtype == PAO_F32) {
        return (double)((const float*)base)[i];
    }
    uint16_t h = ((const uint16_t*)base)[i];
    if (dtype == PAO_BF16) {
        uint32_t bits = (uint32_t)h << 16; /* bf16 is the top half of an IEEE binary32 */
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + frac), e - 25); /* (1 + frac/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

typedef struct {
    /* operands */
    const void* q;      /* [Nq, Hq, D]   (GQA)  or absorbed q [Nq, H, R]  (MLA) */
    const void* k;      /* [P, ps, Hkv, D]      or latent   [P, ps, 1, R] */
    const void* v;      /* [P, ps, Hkv, Dv]     or unused (MLA: V is the latent) */
    const void* qr;     /* MLA only: position q [Nq, H, Pr] */
    const void* kr;     /* MLA only: rope cache [P, ps, 1, Pr] */
    int dtype;
    int mla;
    /* schedule */
    const int32_t* seq_lens;
    const int32_t* query_offsets;
    int32_t num_seqs;
    const int32_t* block_tables;
    int32_t table_width, page_size, num_pages;
    /* geometry */
    int32_t hq, hkv, d, dv, pr;
    double scale;
    int causal;
    int32_t window;
    const int32_t* key_begin; /* optional [S]: keys t < key_begin[s] are dropped */
    const int32_t* key_end;   /* optional [S]: keys t >= key_end[s] are dropped */
    const uint8_t* want;      /* optional [Nq*Hq]: compute only rows with want != 0 */
    double* out;              /* [Nq, Hq, Dv] */
    double* lse;              /* [Nq, Hq] */
    /* sparse top-K block selection */
    int mode;                 /* 0: attention, 1: proxy block scores */
    int32_t block_size;       /* keys per sparse block */
    const int32_t* sel;       /* optional [Nq, Hkv, sel_width]: selected blocks, -1 = unused */
    int32_t sel_width;
    double* scores;           /* mode 1: [Nq, Hkv, max_blocks] */
    int32_t max_blocks;
    /* work distribution over (sequence, kv head) */
    int64_t next_item;
    pthread_mutex_t lock;
    int error;
} pao_job;

/* Is key t visible to a query at absolute position p? */
static int pao_visible(const pao_job* J, int32_t s, int64_t t, int64_t p) {
#ifdef PAO_MUTANT_CAUSAL_STRICT
    if (J->causal && t >= p) return 0;
#else
    if (J->causal && t > p) return 0;
#endif
#ifdef PAO_MUTANT_WINDOW_WIDE
    if (J->window > 0 && t + J->window < p) return 0;
#else
    if (J->window > 0 && t + J->window <= p) return 0;
#endif
    if (J->key_begin && t < J->key_begin[s]) return 0;
    if (J->key_end && t >= J->key_end[s]) return 0;
    return 1;
}

static void pao_run_item(pao_job* J, int32_t s, int32_t kvh, double* kbuf, double* vbuf,
                         double* krbuf, double* xbuf, double* qbuf, uint8_t* smask) {
    const int64_t L = J->seq_lens[s];
    const int64_t q0 = J->query_offsets[s];
    const int64_t n = J->query_offsets[s + 1] - q0;
    const int32_t ps = J->page_size;
    const int32_t G = J->hq / J->hkv;
    const int32_t kd = J->d;            /* width of the key rows */
    const int32_t vd = J->dv;           /* width of the value rows */
    const int32_t kheads = J->mla ? 1 : J->hkv;
    if (n == 0) return;
    if (J->want) { /* skip the gather when no row of this (sequence, kv head) is asked for */
        int any = 0;
        for (int32_t g = 0; g < G && !any; ++g)
            for (int64_t j = 0; j < n && !any; ++j)
                any = J->want[(q0 + j) * J->hq + (J->mla ? g : kvh * G + g)] != 0;
        if (!any) return;
    }

    /* 1. materialise this sequence's keys/values for this KV head contiguously */
    for (int64_t t = 0; t < L; ++t) {
#ifdef PAO_MUTANT_IDENTITY_TABLE
        int64_t page = t / ps; /* wrong: ignores the block table */
        int64_t slot = t % ps;
#else
        int64_t page = J->block_tables[(int64_t)s * J->table_width + t / ps];
        int64_t slot = t % ps;
#endif
        int64_t row = (page * ps + slot) * kheads + (J->mla ? 0 : kvh);
        for (int32_t c = 0; c < kd; ++c) kbuf[t * kd + c] = pao_load(J->k, J->dtype, row * kd + c);
        if (J->mla) {
            for (int32_t c = 0; c < J->pr; ++c)
                krbuf[t * J->pr + c] = pao_load(J->kr, J->dtype, (page * ps + slot) * J->pr + c);
        } else {
            for (int32_t c = 0; c < vd; ++c) vbuf[t * vd + c] = pao_load(J->v, J->dtype, row * vd + c);
        }
    }
    const double* V = J->mla ? kbuf : vbuf; /* MLA: the latent is both key and value */

    /* 2. dense masked softmax for every query head of the group and every query */
    for (int32_t g = 0; g < G; ++g) {
#ifdef PAO_MUTANT_GQA_MODULO
        const int32_t h = g * J->hkv + kvh; /* wrong map: h % Hkv == kvh */
#else
        const int32_t h = kvh * G + g;
#endif
        for (int64_t j = 0; j < n; ++j) {
            const int64_t qi = q0 + j;
            const int64_t r = qi * J->hq + h;
            if (J->want && !J->want[r]) continue;
#ifdef PAO_MUTANT_LEFT_ALIGNED
            const int64_t p = j;
#else
            const int64_t p = L - n + j;
#endif
            for (int32_t c = 0; c < kd; ++c) qbuf[c] = pao_load(J->q, J->dtype, r * kd + c);
            for (int32_t c = 0; c < J->pr; ++c) qbuf[kd + c] = pao_load(J->qr, J->dtype, r * J->pr + c);
            if (J->sel) { /* sparse: only the keys of the blocks selected for (query, kv head) */
                const int64_t nb = (L + J->block_size - 1) / J->block_size;
                const int32_t* row_sel = J->sel + (qi * J->hkv + kvh) * (int64_t)J->sel_width;
                for (int64_t b = 0; b < nb; ++b) smask[b] = 0;
                for (int32_t e = 0; e < J->sel_width; ++e)
                    if (row_sel[e] >= 0) smask[row_sel[e]] = 1;
            }
            double m = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                if (!pao_visible(J, s, t, p) || (J->sel && !smask[t / J->block_size])) {
                    xbuf[t] = -INFINITY;
                    continue;
                }
                double acc = 0.0;
                for (int32_t c = 0; c < kd; ++c) acc += qbuf[c] * kbuf[t * kd + c];
#ifndef PAO_MUTANT_DROP_ROPE
                if (J->mla)
                    for (int32_t c = 0; c < J->pr; ++c) acc += qbuf[kd + c] * krbuf[t * J->pr + c];
#endif
#ifdef PAO_MUTANT_SCALE_DROPPED
                xbuf[t] = acc;
#else
                xbuf[t] = J->scale * acc;
#endif
                if (xbuf[t] > m) m = xbuf[t];
            }
            double* o = J->out + r * vd;
            for (int32_t c = 0; c < vd; ++c) o[c] = 0.0;
            if (m == -INFINITY) { J->lse[r] = -INFINITY; continue; }
            double sum = 0.0;
            for (int64_t t = 0; t < L; ++t)
                if (xbuf[t] != -INFINITY) sum += exp(xbuf[t] - m);
#ifdef PAO_MUTANT_LSE_NO_MAX
            const double lse = log(sum);
#else
            const double lse = m + log(sum);
#endif
            J->lse[r] = lse;
            for (int64_t t = 0; t < L; ++t) {
                if (xbuf[t] == -INFINITY) continue;
#ifdef PAO_MUTANT_UNNORMALISED
                const double w = exp(xbuf[t] - m);
#else
                const double w = exp(xbuf[t] - lse);
#endif
                for (int32_t c = 0; c < vd; ++c) o[c] += w * V[t * vd + c];
            }
        }
    }
}

/* Number of sparse blocks of a sequence with L keys: the last block may be partial. */
static int64_t pao_num_blocks(int64_t L, int32_t block_size) {
#ifdef PAO_MUTANT_SPARSE_FLOOR
    return L / block_size; /* wrong: drops a partial last block */
#else
    return (L + block_size - 1) / block_size;
#endif
}

/*
 * Proxy block scores of one (sequence, kv head): for every query of the sequence, the proxy
 * query is the first query head of the KV head's group (alice-llm `llama3_sparse_attention`,
 * "cheap proxy"), and the score of block b is the largest scaled score q_proxy . k_t over the
 * keys t of the block the query can see; a block without a visible key scores -inf.
 */
static void pao_scores_item(pao_job* J, int32_t s, int32_t kvh, double* kbuf, double* qbuf) {
    const int64_t L = J->seq_lens[s];
    const int64_t q0 = J->query_offsets[s];
    const int64_t n = J->query_offsets[s + 1] - q0;
    const int32_t ps = J->page_size, kd = J->d, bs = J->block_size;
    const int32_t G = J->hq / J->hkv;
    if (n == 0) return;
    for (int64_t t = 0; t < L; ++t) {
        int64_t page = J->block_tables[(int64_t)s * J->table_width + t / ps];
        int64_t row = (page * ps + t % ps) * J->hkv + kvh;
        for (int32_t c = 0; c < kd; ++c) kbuf[t * kd + c] = pao_load(J->k, J->dtype, row * kd + c);
    }
    const int64_t nb = pao_num_blocks(L, bs);
#ifdef PAO_MUTANT_SPARSE_PROXY_LAST
    const int32_t h = kvh * G + G - 1; /* wrong proxy head */
#else
    const int32_t h = kvh * G;
#endif
    for (int64_t j = 0; j < n; ++j) {
        const int64_t qi = q0 + j;
        const int64_t p = L - n + j;
        for (int32_t c = 0; c < kd; ++c) qbuf[c] = pao_load(J->q, J->dtype, (qi * J->hq + h) * kd + c);
        double* out = J->scores + (qi * J->hkv + kvh) * (int64_t)J->max_blocks;
        for (int64_t b = 0; b < J->max_blocks; ++b) {
            double best = -INFINITY;
            if (b < nb) {
                const int64_t t1 = (b + 1) * bs < L ? (b + 1) * bs : L;
                for (int64_t t = b * bs; t < t1; ++t) {
#ifndef PAO_MUTANT_SPARSE_UNMASKED
                    if (!pao_visible(J, s, t, p)) continue;
#endif
                    double acc = 0.0;
                    for (int32_t c = 0; c < kd; ++c) acc += qbuf[c] * kbuf[t * kd + c];
                    acc *= J->scale;
                    if (acc > best) best = acc;
                }
            }
            out[b] = best;
        }
    }
}

static void* pao_worker(void* arg) {
    pao_job* J = (pao_job*)arg;
    int64_t maxL = 0;
    for (int32_t s = 0; s < J->num_seqs; ++s)
        if (J->seq_lens[s] > maxL) maxL = J->seq_lens[s];
    const int64_t rows = maxL > 0 ? maxL : 1;
    double* kbuf = (double*)malloc(sizeof(double) * rows * (size_t)J->d);
    double* vbuf = J->mla ? NULL : (double*)malloc(sizeof(double) * rows * (size_t)J->dv);
    double* krbuf = J->mla ? (double*)malloc(sizeof(double) * rows * (size_t)(J->pr > 0 ? J->pr : 1)) : NULL;
    double* xbuf = (double*)malloc(sizeof(double) * rows);
    double* qbuf = (double*)malloc(sizeof(double) * (size_t)(J->d + J->pr));
    uint8_t* smask = J->sel ? (uint8_t*)malloc((size_t)(rows / (J->block_size > 0 ? J->block_size : 1) + 2)) : NULL;
    if (!kbuf || (!J->mla && !vbuf) || (J->mla && !krbuf) || !xbuf || !qbuf || (J->sel && !smask)) {
        pthread_mutex_lock(&J->lock);
        J->error = 1;
        pthread_mutex_unlock(&J->lock);
    } else {
        const int32_t kheads = J->mla ? 1 : J->hkv;
        for (;;) {
            pthread_mutex_lock(&J->lock);
            int64_t it = J->next_item++;
            pthread_mutex_unlock(&J->lock);
            if (it >= (int64_t)J->num_seqs * kheads) break;
            if (J->mode == 1)
                pao_scores_item(J, (int32_t)(it / kheads), (int32_t)(it % kheads), kbuf, qbuf);
            else
                pao_run_item(J, (int32_t)(it / kheads), (int32_t)(it % kheads), kbuf, vbuf, krbuf, xbuf, qbuf,
                             smask);
        }
    }
    free(smask);
    free(kbuf);
    free(vbuf);
    free(krbuf);
    free(xbuf);
    free(qbuf);
    return NULL;
}

static int pao_check_schedule(const pao_job* J) {
    if (J->num_seqs < 0 || J->page_size <= 0 || J->table_width < 0) return -1;
    if (J->query_offsets[0] != 0) return -1;
    for (int32_t s = 0; s < J->num_seqs; ++s) {
        int64_t L = J->seq_lens[s];
        int64_t n = (int64_t)J->query_offsets[s + 1] - J->query_offsets[s];
        if (L < 0 || n < 0 || n > L) return -1;
        int64_t used = (L + J->page_size - 1) / J->page_size;
        if (used > J->table_width) return -1;
        for (int64_t b = 0; b < used; ++b) {
            int32_t page = J->block_tables[(int64_t)s * J->table_width + b];
            if (page < 0 || page >= J->num_pages) return -2;
        }
    }
    return 0;
}

static int pao_run(pao_job* J, int nthreads) {
    int rc = pao_check_schedule(J);
    if (rc) return rc;
    J->next_item = 0;
    J->error = 0;
    pthread_mutex_init(&J->lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, pao_worker, J) == 0) ++started;
        else break;
    }
    if (started == 0) pao_worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J->lock);
    return J->error ? -3 : 0;
}

/*
 * Paged GQA attention. Returns 0 on success, -1 on a malformed schedule, -2 on a block-table
 * entry outside the pool, -3 on an allocation failure.
 */
int pao_paged_attention(const void* q, const void* k_cache, const void* v_cache, int dtype,
                        const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                        const int32_t* block_tables, int32_t table_width, int32_t page_size,
                        int32_t num_pages, int32_t hq, int32_t hkv, int32_t d, int32_t dv,
                        double scale, int causal, int32_t window, const int32_t* key_begin,
                        const int32_t* key_end, const uint8_t* want_rows, double* out, double* lse,
                        int nthreads) {
    if (hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || dv <= 0 || window < 0) return -1;
    pao_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k_cache; J.v = v_cache; J.dtype = dtype; J.mla = 0;
    J.seq_lens = seq_lens; J.query_offsets = query_offsets; J.num_seqs = num_seqs;
    J.block_tables = block_tables; J.table_width = table_width; J.page_size = page_size;
    J.num_pages = num_pages; J.hq = hq; J.hkv = hkv; J.d = d; J.dv = dv; J.pr = 0;
    J.scale = scale; J.causal = causal; J.window = window;
    J.key_begin = key_begin; J.key_end = key_end; J.want = want_rows; J.out = out; J.lse = lse;
    return pao_run(&J, nthreads);
}

/* MLA absorbed-latent attention: one shared latent head; V is the latent itself. */
int pao_mla_attention(const void* q_latent, const void* q_rope, const void* latent_cache,
                      const void* rope_cache, int dtype, const int32_t* seq_lens,
                      const int32_t* query_offsets, int32_t num_seqs, const int32_t* block_tables,
                      int32_t table_width, int32_t page_size, int32_t num_pages, int32_t heads,
                      int32_t latent_dim, int32_t rope_dim, double scale, int causal,
                      int32_t window, const int32_t* key_begin, const int32_t* key_end,
                      const uint8_t* want_rows, double* out, double* lse, int nthreads) {
    if (heads <= 0 || latent_dim <= 0 || rope_dim < 0 || window < 0) return -1;
    pao_job J;
    memset(&J, 0, sizeof J);
    J.q = q_latent; J.k = latent_cache; J.v = NULL; J.qr = q_rope; J.kr = rope_cache;
    J.dtype = dtype; J.mla = 1;
    J.seq_lens = seq_lens; J.query_offsets = query_offsets; J.num_seqs = num_seqs;
    J.block_tables = block_tables; J.table_width = table_width; J.page_size = page_size;
    J.num_pages = num_pages; J.hq = heads; J.hkv = 1; J.d = latent_dim; J.dv = latent_dim;
    J.pr = rope_dim; J.scale = scale; J.causal = causal; J.window = window;
    J.key_begin = key_begin; J.key_end = key_end; J.want = want_rows; J.out = out; J.lse = lse;
    return pao_run(&J, nthreads);
}

/*
 * Merge of partial results over disjoint key subsets (ruDNN "merge FP32 statistics";
 * alice-llm `lse_combine`). Part i of row r holds the normalised output o_i and its
 * logsumexp lse_i over its keys. The merged logsumexp is the logsumexp of the lse_i, and the
 * merged output weights each o_i by exp(lse_i - lse). Parts with lse_i = -inf have no keys
 * and weight 0; a row whose parts are all empty gets out = 0, lse = -inf.
 * Layout: o_parts [nparts, rows, dv], lse_parts [nparts, rows].
 */
void pao_lse_combine(const double* o_parts, const double* lse_parts, int64_t nparts, int64_t rows,
                     int32_t dv, double* out, double* lse) {
    for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int64_t i = 0; i < nparts; ++i)
            if (lse_parts[i * rows + r] > m) m = lse_parts[i * rows + r];
        double* o = out + r * dv;
        for (int32_t c = 0; c < dv; ++c) o[c] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double sum = 0.0;
        for (int64_t i = 0; i < nparts; ++i) {
            double li = lse_parts[i * rows + r];
            if (li != -INFINITY) sum += exp(li - m);
        }
        const double total = m + log(sum);
        lse[r] = total;
        for (int64_t i = 0; i < nparts; ++i) {
            double li = lse_parts[i * rows + r];
            if (li == -INFINITY) continue;
            const double w = exp(li - total);
            for (int32_t c = 0; c < dv; ++c) o[c] += w * o_parts[(i * rows + r) * dv + c];
        }
    }
}

/*
 * Sparse top-K block attention (alice-llm `llama3_sparse_attention`: proxy block scores,
 * top-K block selection, attention over the selected blocks, merge of the partials). The keys
 * of sequence s are cut into ceil(L_s / block_size) blocks of block_size consecutive positions
 * (the last one may be partial); queries attend only to the keys of the blocks selected for
 * their (query, kv head), with the usual causal/window mask on top. All G query heads of a
 * group share their KV head's selection.
 */

/* Proxy block scores, [Nq, Hkv, max_blocks] (blocks past a sequence's count: -inf). */
int pao_sparse_block_scores(const void* q, const void* k_cache, int dtype, const int32_t* seq_lens,
                            const int32_t* query_offsets, int32_t num_seqs, const int32_t* block_tables,
                            int32_t table_width, int32_t page_size, int32_t num_pages, int32_t hq,
                            int32_t hkv, int32_t d, double scale, int causal, int32_t window,
                            int32_t block_size, int32_t max_blocks, double* scores, int nthreads) {
    if (hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || window < 0 || block_size <= 0 || max_blocks < 0)
        return -1;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (pao_num_blocks(seq_lens[s], block_size) > max_blocks) return -1;
    pao_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k_cache; J.v = NULL; J.dtype = dtype; J.mla = 0; J.mode = 1;
    J.seq_lens = seq_lens; J.query_offsets = query_offsets; J.num_seqs = num_seqs;
    J.block_tables = block_tables; J.table_width = table_width; J.page_size = page_size;
    J.num_pages = num_pages; J.hq = hq; J.hkv = hkv; J.d = d; J.dv = d; J.pr = 0;
    J.scale = scale; J.causal = causal; J.window = window;
    J.block_size = block_size; J.scores = scores; J.max_blocks = max_blocks;
    return pao_run(&J, nthreads);
}

/*
 * Top-K selection per (query, kv head) row from the proxy scores. A sequence with nb blocks
 * keeps k = nb blocks when topk is 0 or at least nb (the dense case), else k = topk: the k
 * highest scores, equal scores going to the lower block index. The selected indices are
 * written in ascending order into [Nq, Hkv, width], the rest of the row set to -1.
 * Returns -1 when width < k for some sequence.
 */
int pao_sparse_topk(const double* scores, const int32_t* seq_lens, const int32_t* query_offsets,
                    int32_t num_seqs, int32_t hkv, int32_t max_blocks, int32_t block_size, int32_t topk,
                    int32_t width, int32_t* sel) {
    if (hkv <= 0 || block_size <= 0 || topk < 0 || width < 0) return -1;
    uint8_t* picked = (uint8_t*)malloc((size_t)max_blocks + 1);
    if (!picked) return -3;
    for (int32_t s = 0; s < num_seqs; ++s) {
        const int64_t nb = pao_num_blocks(seq_lens[s], block_size);
        if (nb > max_blocks) { free(picked); return -1; }
        const int64_t k = (topk == 0 || topk >= nb) ? nb : topk;
        if (k > width) { free(picked); return -1; }
        for (int64_t qi = query_offsets[s]; qi < query_offsets[s + 1]; ++qi) {
            for (int32_t h = 0; h < hkv; ++h) {
                const double* sc = scores + (qi * hkv + h) * (int64_t)max_blocks;
                int32_t* out = sel + (qi * hkv + h) * (int64_t)width;
                for (int64_t b = 0; b < nb; ++b) picked[b] = 0;
                for (int64_t r = 0; r < k; ++r) { /* take the best block not taken yet */
                    int64_t best = -1;
                    for (int64_t b = 0; b < nb; ++b) {
                        if (picked[b]) continue;
#if defined(PAO_MUTANT_SPARSE_TIES_HIGH)
                        if (best < 0 || sc[b] >= sc[best]) best = b;
#elif defined(PAO_MUTANT_SPARSE_MIN)
                        if (best < 0 || sc[b] < sc[best]) best = b;
#else
                        if (best < 0 || sc[b] > sc[best]) best = b;
#endif
                    }
                    if (best < 0) break;
                    picked[best] = 1;
                }
                int32_t e = 0;
                for (int64_t b = 0; b < nb; ++b)
                    if (picked[b]) out[e++] = (int32_t)b;
                for (; e < width; ++e) out[e] = -1;
            }
        }
    }
    free(picked);
    return 0;
}

/*
 * Attention restricted to selected blocks. selection [Nq, Hkv, width]: block indices, -1 for
 * an unused entry. Returns -4 if an entry lies outside [0, nb) of its sequence or repeats a
 * block of its row; otherwise as pao_paged_attention.
 */
int pao_sparse_attention(const void* q, const void* k_cache, const void* v_cache, int dtype,
                         const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                         const int32_t* block_tables, int32_t table_width, int32_t page_size,
                         int32_t num_pages, int32_t hq, int32_t hkv, int32_t d, int32_t dv, double scale,
                         int causal, int32_t window, int32_t block_size, const int32_t* selection,
                         int32_t width, const uint8_t* want_rows, double* out, double* lse, int nthreads) {
    if (hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || dv <= 0 || window < 0 || block_size <= 0 || width < 0)
        return -1;
    for (int32_t s = 0; s < num_seqs; ++s) {
        const int64_t nb = pao_num_blocks(seq_lens[s], block_size);
        for (int64_t qi = query_offsets[s]; qi < query_offsets[s + 1]; ++qi)
            for (int32_t h = 0; h < hkv; ++h) {
                const int32_t* row = selection + (qi * hkv + h) * (int64_t)width;
                for (int32_t e = 0; e < width; ++e) {
                    if (row[e] == -1) continue;
                    if (row[e] < 0 || row[e] >= nb) return -4;
                    for (int32_t f = 0; f < e; ++f)
                        if (row[f] == row[e]) return -4;
                }
            }
    }
    pao_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k_cache; J.v = v_cache; J.dtype = dtype; J.mla = 0;
    J.seq_lens = seq_lens; J.query_offsets = query_offsets; J.num_seqs = num_seqs;
    J.block_tables = block_tables; J.table_width = table_width; J.page_size = page_size;
    J.num_pages = num_pages; J.hq = hq; J.hkv = hkv; J.d = d; J.dv = dv; J.pr = 0;
    J.scale = scale; J.causal = causal; J.window = window;
    J.want = want_rows; J.out = out; J.lse = lse;
    J.block_size = block_size; J.sel = selection; J.sel_width = width;
    return pao_run(&J, nthreads);
}

/*
 * Backward of paged GQA attention (boostr `standard_attention_bwd`, recomputing the weights from
 * Q and K): with P = softmax(scale * Q K^T + mask) per row, O = P V, and the upstream gradient
 * dO,
 *     dV_t += P_t dO,   dP_t = dO . V_t,   D = dO . O,   dS_t = P_t (dP_t - D),
 *     dQ = scale * sum_t dS_t K_t,   dK_t += scale * dS_t Q.
 * Query head h reads KV head h / G, so dK and dV sum over the G heads of a group (boostr
 * `sum_gqa_grads`), and over every query and sequence whose visible keys include the slot
 * (a page shared by several sequences receives all their contributions).
 * dq [Nq, Hq, D] is written; dk [P, ps, Hkv, D] and dv [P, ps, Hkv, Dv] are zeroed and then
 * accumulated. Same masking readings as the forward. Returns 0, or -1/-2/-3 as the forward.
 */
typedef struct {
    pao_job J;
    const void* dout;
    double* dq;
    double* dk;
    double* dv;
    pthread_mutex_t acc_lock;
} pao_bwd_job;

static void pao_bwd_item(pao_bwd_job* B, int32_t s, int32_t kvh, double* kbuf, double* vbuf, double* xbuf,
                         double* qbuf, double* dkl, double* dvl, double* obuf, double* gbuf) {
    pao_job* J = &B->J;
    const int64_t L = J->seq_lens[s];
    const int64_t q0 = J->query_offsets[s];
    const int64_t n = J->query_offsets[s + 1] - q0;
    const int32_t ps = J->page_size;
    const int32_t G = J->hq / J->hkv;
    const int32_t kd = J->d, vd = J->dv;
    if (n == 0) return;
    for (int64_t t = 0; t < L; ++t) {
        int64_t page = J->block_tables[(int64_t)s * J->table_width + t / ps];
        int64_t row = (page * ps + t % ps) * J->hkv + kvh;
        for (int32_t c = 0; c < kd; ++c) kbuf[t * kd + c] = pao_load(J->k, J->dtype, row * kd + c);
        for (int32_t c = 0; c < vd; ++c) vbuf[t * vd + c] = pao_load(J->v, J->dtype, row * vd + c);
        for (int32_t c = 0; c < kd; ++c) dkl[t * kd + c] = 0.0;
        for (int32_t c = 0; c < vd; ++c) dvl[t * vd + c] = 0.0;
    }
    for (int32_t g = 0; g < G; ++g) {
        const int32_t h = kvh * G + g;
        for (int64_t j = 0; j < n; ++j) {
            const int64_t r = (q0 + j) * J->hq + h;
            const int64_t p = L - n + j;
            for (int32_t c = 0; c < kd; ++c) qbuf[c] = pao_load(J->q, J->dtype, r * kd + c);
            for (int32_t c = 0; c < vd; ++c) gbuf[c] = pao_load(B->dout, J->dtype, r * vd + c);
            double m = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                if (!pao_visible(J, s, t, p)) { xbuf[t] = -INFINITY; continue; }
                double acc = 0.0;
                for (int32_t c = 0; c < kd; ++c) acc += qbuf[c] * kbuf[t * kd + c];
                xbuf[t] = J->scale * acc;
                if (xbuf[t] > m) m = xbuf[t];
            }
            double* dq = B->dq + r * kd;
            for (int32_t c = 0; c < kd; ++c) dq[c] = 0.0;
            if (m == -INFINITY) continue;
            double sum = 0.0;
            for (int64_t t = 0; t < L; ++t)
                if (xbuf[t] != -INFINITY) sum += exp(xbuf[t] - m);
            const double lse = m + log(sum);
            for (int32_t c = 0; c < vd; ++c) obuf[c] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                if (xbuf[t] == -INFINITY) continue;
                xbuf[t] = exp(xbuf[t] - lse); /* now P_t */
                for (int32_t c = 0; c < vd; ++c) obuf[c] += xbuf[t] * vbuf[t * vd + c];
            }
            double Dr = 0.0;
#ifndef PAO_MUTANT_BWD_NO_D
            for (int32_t c = 0; c < vd; ++c) Dr += gbuf[c] * obuf[c];
#endif
            for (int64_t t = 0; t < L; ++t) {
                if (xbuf[t] == -INFINITY) continue;
                const double P = xbuf[t];
                double dp = 0.0;
                for (int32_t c = 0; c < vd; ++c) dp += gbuf[c] * vbuf[t * vd + c];
                const double ds = P * (dp - Dr);
                for (int32_t c = 0; c < kd; ++c) dq[c] += J->scale * ds * kbuf[t * kd + c];
                for (int32_t c = 0; c < kd; ++c) dkl[t * kd + c] += J->scale * ds * qbuf[c];
                for (int32_t c = 0; c < vd; ++c) dvl[t * vd + c] += P * gbuf[c];
            }
        }
    }
    pthread_mutex_lock(&B->acc_lock);
    for (int64_t t = 0; t < L; ++t) {
        int64_t page = J->block_tables[(int64_t)s * J->table_width + t / ps];
        int64_t row = (page * ps + t % ps) * J->hkv + kvh;
        for (int32_t c = 0; c < kd; ++c) B->dk[row * kd + c] += dkl[t * kd + c];
        for (int32_t c = 0; c < vd; ++c) B->dv[row * vd + c] += dvl[t * vd + c];
    }
    pthread_mutex_unlock(&B->acc_lock);
}

static void* pao_bwd_worker(void* arg) {
    pao_bwd_job* B = (pao_bwd_job*)arg;
    pao_job* J = &B->J;
    int64_t maxL = 1;
    for (int32_t s = 0; s < J->num_seqs; ++s)
        if (J->seq_lens[s] > maxL) maxL = J->seq_lens[s];
    double* kbuf = (double*)malloc(sizeof(double) * maxL * J->d);
    double* vbuf = (double*)malloc(sizeof(double) * maxL * J->dv);
    double* dkl = (double*)malloc(sizeof(double) * maxL * J->d);
    double* dvl = (double*)malloc(sizeof(double) * maxL * J->dv);
    double* xbuf = (double*)malloc(sizeof(double) * maxL);
    double* qbuf = (double*)malloc(sizeof(double) * J->d);
    double* obuf = (double*)malloc(sizeof(double) * J->dv);
    double* gbuf = (double*)malloc(sizeof(double) * J->dv);
    if (!kbuf || !vbuf || !dkl || !dvl || !xbuf || !qbuf || !obuf || !gbuf) {
        pthread_mutex_lock(&J->lock);
        J->error = 1;
        pthread_mutex_unlock(&J->lock);
    } else {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            int64_t it = J->next_item++;
            pthread_mutex_unlock(&J->lock);
            if (it >= (int64_t)J->num_seqs * J->hkv) break;
            pao_bwd_item(B, (int32_t)(it / J->hkv), (int32_t)(it % J->hkv), kbuf, vbuf, xbuf, qbuf, dkl, dvl, obuf,
                         gbuf);
        }
    }
    free(kbuf); free(vbuf); free(dkl); free(dvl); free(xbuf); free(qbuf); free(obuf); free(gbuf);
    return NULL;
}

int pao_paged_attention_backward(const void* q, const void* k_cache, const void* v_cache, const void* d_out,
                                 int dtype, const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                                 const int32_t* block_tables, int32_t table_width, int32_t page_size,
                                 int32_t num_pages, int32_t hq, int32_t hkv, int32_t d, int32_t dv, double scale,
                                 int causal, int32_t window, double* dq, double* dk, double* dvout, int nthreads) {
    if (hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || dv <= 0 || window < 0) return -1;
    pao_bwd_job B;
    memset(&B, 0, sizeof B);
    pao_job* J = &B.J;
    J->q = q; J->k = k_cache; J->v = v_cache; J->dtype = dtype; J->mla = 0;
    J->seq_lens = seq_lens; J->query_offsets = query_offsets; J->num_seqs = num_seqs;
    J->block_tables = block_tables; J->table_width = table_width; J->page_size = page_size;
    J->num_pages = num_pages; J->hq = hq; J->hkv = hkv; J->d = d; J->dv = dv;
    J->scale = scale; J->causal = causal; J->window = window;
    int rc = pao_check_schedule(J);
    if (rc) return rc;
    B.dout = d_out; B.dq = dq; B.dk = dk; B.dv = dvout;
    memset(dk, 0, sizeof(double) * (size_t)num_pages * page_size * hkv * d);
    memset(dvout, 0, sizeof(double) * (size_t)num_pages * page_size * hkv * dv);
    pthread_mutex_init(&J->lock, NULL);
    pthread_mutex_init(&B.acc_lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, pao_bwd_worker, &B) == 0) ++started;
        else break;
    }
    if (started == 0) pao_bwd_worker(&B);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J->lock);
    pthread_mutex_destroy(&B.acc_lock);
    return J->error ? -3 : 0;
}
