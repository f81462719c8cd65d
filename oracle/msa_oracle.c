/*
 * msa_oracle.c -- plain, slow CPU definition of MiniMax Sparse Attention (MSA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness oracle that the CUDA
 * library is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (sources are the public write-ups of MiniMax M3's MSA):
 *   - "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
 *     (cloud.tencent.com article), section 二: a two-stage design.  The index
 *     branch takes ONE lightweight index query per GQA group, scores the KV
 *     blocks with it, max-pools the scores over each block ("Block Max Pool")
 *     and keeps the top-k blocks.  The sparse branch then runs full attention
 *     over the selected blocks only.
 *   - same article, section 六: every head of a GQA group shares that one
 *     block set.
 *   - "如何用MiniMax-M3的稀疏注意力技术解决大模型效率瓶颈" (mlqm.cn guide), the
 *     configuration-file passage: sparse_block_size 128, sparse_topk_blocks 16,
 *     sparse_index_dim 128.
 * The pages give no formula.  The readings used here (plain dot product with
 * no scale for the index score, causal masking inside the query's own block,
 * own block always kept, ties to the lower block id, 1/sqrt(d) on the sparse
 * branch) are listed in the design notes and restated at each step below.
 *
 * Index-branch variants (the guide's configuration sets
 * sparse_num_index_heads = 4, which one index head per GQA group cannot
 * match; the pages fix nothing more, so these are the plainest readings):
 *   - Hi index heads partition the GQA groups into contiguous sets of
 *     H_kv / Hi groups, and every group of a set uses its index head's
 *     selection (Hi = H_kv is one index head per group);
 *   - index keys are either one per (token, index head) or one per token,
 *     shared by every index head;
 *   - index keys are bf16, or FP8 E4M3 with one fp32 scale per key row: the
 *     score is scale * (q_idx . k), the dot over the exactly decoded values.
 *
 * Arithmetic: bf16 and e4m3 inputs are widened exactly to double; every sum,
 * max and exponential is in double.  Rows are independent, so they are spread over
 * POSIX threads; no row's arithmetic is split, reordered or fused.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -pthread -ffp-contract=off
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double, exact: a bf16 value is the top 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* FP8 E4M3 (the OCP 8-bit floating-point format, "E4M3FN": no infinities,
 * S.1111.111 is NaN) -> double, exact.  Exponent bias 7; exponent field 0 is
 * the subnormal range 2^-6 * m/8. */
static double e4m3_to_double(uint8_t x)
{
    const int sgn = x >> 7, e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

double oracle_e4m3_to_double(int x) { return e4m3_to_double((uint8_t)x); }

typedef struct {
    int B, Sq, H_q, H_kv, D, block, top_k;
    int KH;               /* index-key heads: 1 (shared) or H_kv (= index heads) */
    int key_fp8;          /* index keys are E4M3 bytes with per-row scales */
    int n_idx;            /* sparse branch: index heads whose selections the groups use */
    const uint8_t *k_idx8;
    const float *k_scale; /* [T, KH] */
    int64_t kv_capacity;
    const uint16_t *q_idx, *k_idx, *q, *k, *v;
    const int32_t *lens, *block_ids_in;
    const int64_t *kv_offsets, *rows;
    int64_t n_rows;
    double scale;
    /* outputs */
    int32_t *block_ids;
    float *block_scores;
    double *all_scores;   /* optional [n_rows, H_kv, nb_max] */
    double *boundary;     /* optional [n_rows, H_kv, 2] */
    int nb_max;
    double *out;          /* [n_rows, H_q, D] */
    double *wsum;         /* optional [n_rows, H_q] */
    int err;
} job_t;

typedef struct { job_t *job; int64_t first, stride; int kind; } slice_t;

/* Position of query row i of sequence b: the Sq query rows are the last Sq
 * tokens of the sequence, so p = L_b - Sq + i (decode: Sq = 1, p = L_b - 1,
 * the new token already sits in the cache and attends to itself). */
static int row_position(const job_t *J, int64_t r, int *b_out, int64_t *p_out)
{
    int b = (int)(r / J->Sq);
    int i = (int)(r % J->Sq);
    int64_t L = J->lens[b];
    if (L < J->Sq || J->kv_offsets[b] < 0 || J->kv_offsets[b] + L > J->kv_capacity)
        return -1;
    *b_out = b;
    *p_out = L - J->Sq + i;
    return 0;
}

typedef struct { double s; int j; } cand_t;

/* Ranking of candidate blocks: larger block score first; on equal scores the
 * lower block id first (the tie rule).  -0 and +0 compare equal. */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int int_cmp(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Index branch for one (query row, group). */
static void index_row(job_t *J, int64_t rr, int g)
{
    int64_t r = J->rows ? J->rows[rr] : rr;
    int b; int64_t p;
    const int K = J->top_k, blk = J->block, Di = J->D;
    int32_t *ids_out = J->block_ids + rr * J->H_kv * K;
    float *sc_out = J->block_scores + rr * J->H_kv * K;
    if (row_position(J, r, &b, &p)) { J->err = 1; return; }
    const int64_t off = J->kv_offsets[b];
    const int own = (int)(p / blk);       /* the query's own block */
    const int nvis = own + 1;             /* blocks 0..own are visible */
    double *S = (double *)malloc(sizeof(double) * nvis);
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (nvis > 0 ? nvis : 1));
    int *sel = (int *)malloc(sizeof(int) * (K + 1));
    {
        const uint16_t *qi = J->q_idx + (r * J->H_kv + g) * (int64_t)Di;
        const int kh = J->KH == 1 ? 0 : g;   /* shared keys: one row per token */
        /* Step 1+2: per-token index score (plain dot product of the index
         * head's query with the token's index key, no scale; FP8 keys: the
         * row's scale times the dot over the decoded values), then the block
         * max-pool over the visible tokens t <= p of each block. */
        for (int j = 0; j < nvis; ++j) {
            double best = -INFINITY;
            int64_t t_end = (int64_t)(j + 1) * blk;
            if (t_end > p + 1) t_end = p + 1;
            for (int64_t t = (int64_t)j * blk; t < t_end; ++t) {
                const int64_t krow = (off + t) * J->KH + kh;
                double s = 0.0;
                if (J->key_fp8) {
                    const uint8_t *ki = J->k_idx8 + krow * (int64_t)Di;
                    for (int d = 0; d < Di; ++d)
                        s += bf16_to_double(qi[d]) * e4m3_to_double(ki[d]);
                    s *= (double)J->k_scale[krow];
                } else {
                    const uint16_t *ki = J->k_idx + krow * (int64_t)Di;
                    for (int d = 0; d < Di; ++d)
                        s += bf16_to_double(qi[d]) * bf16_to_double(ki[d]);
                }
                if (s > best) best = s;
            }
            S[j] = best;
        }
        if (J->all_scores) {
            double *a = J->all_scores + (rr * J->H_kv + g) * (int64_t)J->nb_max;
            for (int j = 0; j < J->nb_max; ++j) a[j] = (j < nvis) ? S[j] : -INFINITY;
        }
        /* Step 3: top-k.  The own block is always kept; the other k-1 slots go
         * to the best blocks j < own under the ranking above.  With no more
         * than k visible blocks, every visible block is kept. */
        int nsel = 0;
        double last_in = INFINITY, first_out = NAN;
        if (nvis <= K) {
            for (int j = 0; j < nvis; ++j) sel[nsel++] = j;
        } else {
            for (int j = 0; j < own; ++j) { c[j].s = S[j] == 0.0 ? 0.0 : S[j]; c[j].j = j; }
            qsort(c, (size_t)own, sizeof(cand_t), cand_cmp);
            sel[nsel++] = own;
            for (int q = 0; q < K - 1; ++q) sel[nsel++] = c[q].j;
            if (K >= 2) last_in = c[K - 2].s;
            first_out = c[K - 1].s;
        }
        /* Step 4: ids ascending, each with its block score; pad with -1/-inf. */
        qsort(sel, (size_t)nsel, sizeof(int), int_cmp);
        for (int q = 0; q < K; ++q) {
            ids_out[g * K + q] = q < nsel ? sel[q] : -1;
            sc_out[g * K + q] = q < nsel ? (float)S[sel[q]] : -INFINITY;
        }
        if (J->boundary) {
            J->boundary[(rr * J->H_kv + g) * 2 + 0] = last_in;
            J->boundary[(rr * J->H_kv + g) * 2 + 1] = first_out;
        }
    }
    free(S); free(c); free(sel);
}

/* Sparse branch for one (query row, head): exact softmax attention over the
 * keys of the selected blocks (causal inside the own block); the block set is
 * the one of the head's group, shared by every head of the group. */
static void attn_row(job_t *J, int64_t rr, int h)
{
    int64_t r = J->rows ? J->rows[rr] : rr;
    int b; int64_t p;
    const int K = J->top_k, blk = J->block, D = J->D, G = J->H_q / J->H_kv;
    if (row_position(J, r, &b, &p)) { J->err = 1; return; }
    const int64_t off = J->kv_offsets[b];
    const int own = (int)(p / blk);
    int64_t max_keys = (int64_t)K * blk;
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * max_keys);
    double *z = (double *)malloc(sizeof(double) * max_keys);
    {
        const int g = h / G;                 /* contiguous head -> group map */
        /* contiguous group -> index-head map: H_kv / n_idx groups per index head */
        const int gi = g / (J->H_kv / J->n_idx);
        const int32_t *ids = J->block_ids_in + (r * J->n_idx + gi) * (int64_t)K;
        int64_t nk = 0;
        for (int q = 0; q < K; ++q) {
            int j = ids[q];
            if (j < 0) continue;
            if (j > own) { J->err = 2; continue; }
            int64_t t_end = (int64_t)(j + 1) * blk;
            if (t_end > p + 1) t_end = p + 1;
            for (int64_t t = (int64_t)j * blk; t < t_end; ++t) {
                if (nk == max_keys) { J->err = 3; break; }
                keys[nk++] = t;
            }
        }
        const uint16_t *qh = J->q + (r * J->H_q + h) * (int64_t)D;
        double m = -INFINITY;
        for (int64_t a = 0; a < nk; ++a) {
            const uint16_t *kt = J->k + ((off + keys[a]) * J->H_kv + g) * (int64_t)D;
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += bf16_to_double(qh[d]) * bf16_to_double(kt[d]);
            z[a] = s * J->scale;
            if (z[a] > m) m = z[a];
        }
        double *o = J->out + (rr * J->H_q + h) * (int64_t)D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        double l = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
            double w = exp(z[a] - m);
            z[a] = w;
            l += w;
            const uint16_t *vt = J->v + ((off + keys[a]) * J->H_kv + g) * (int64_t)D;
            for (int d = 0; d < D; ++d) o[d] += w * bf16_to_double(vt[d]);
        }
        for (int d = 0; d < D; ++d) o[d] /= l;
        if (J->wsum) {
            double ws = 0.0;
            for (int64_t a = 0; a < nk; ++a) ws += z[a] / l;
            J->wsum[rr * J->H_q + h] = ws;
        }
    }
    free(keys); free(z);
}

static void *worker(void *arg)
{
    slice_t *s = (slice_t *)arg;
    /* A job is one (row, group) of the index branch or one (row, head) of
     * the sparse branch; rows are independent, so jobs are too. */
    const int per = s->kind == 0 ? s->job->H_kv : s->job->H_q;
    const int64_t n_jobs = s->job->n_rows * per;
    for (int64_t jb = s->first; jb < n_jobs; jb += s->stride) {
        if (s->kind == 0) index_row(s->job, jb / per, (int)(jb % per));
        else attn_row(s->job, jb / per, (int)(jb % per));
    }
    return NULL;
}

static int run(job_t *J, int kind, int n_threads)
{
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 512) n_threads = 512;
    {
        int64_t n_jobs = J->n_rows * (kind == 0 ? J->H_kv : J->H_q);
        if (n_threads > n_jobs) n_threads = (int)(n_jobs > 0 ? n_jobs : 1);
    }
    pthread_t th[512];
    slice_t sl[512];
    /* Jobs are dealt round-robin so long and short rows spread evenly. */
    for (int t = 0; t < n_threads; ++t) {
        sl[t].job = J; sl[t].kind = kind;
        sl[t].first = t; sl[t].stride = n_threads;
        pthread_create(&th[t], NULL, worker, &sl[t]);
    }
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
    return J->err;
}

/* Index branch: block ids [n_rows, H_kv, top_k] (ascending, -1 padded), their
 * block scores (float of the double max, -inf padded), optionally every
 * visible block score and the ranking boundary (score of the last kept and of
 * the first dropped non-own block).  rows == NULL means all B*Sq rows.
 * Returns 0, or non-zero on an invalid input. */
/* Index branch with n_idx index heads (q_idx [B, Sq, n_idx, D_idx]), key_heads
 * index-key rows per token (1: shared; n_idx: one per index head), keys bf16
 * (k_idx) or E4M3 bytes (k_idx8, with k_scale [T, key_heads]).  Outputs as
 * oracle_index_topk, with n_idx in place of H_kv. */
int oracle_index_topk_ex(int B, int Sq, int n_idx, int key_heads, int D_idx, int block, int top_k,
                         const uint16_t *q_idx, const uint16_t *k_idx, const uint8_t *k_idx8,
                         const float *k_scale,
                         const int32_t *lens, const int64_t *kv_offsets, int64_t kv_capacity,
                         const int64_t *rows, int64_t n_rows,
                         int32_t *block_ids, float *block_scores,
                         double *all_scores, int nb_max, double *boundary, int n_threads)
{
    if (B < 1 || Sq < 1 || n_idx < 1 || D_idx < 1 || block < 1 || top_k < 1) return -1;
    if (key_heads != 1 && key_heads != n_idx) return -1;
    if ((k_idx8 == NULL) == (k_idx == NULL) || (k_idx8 != NULL && k_scale == NULL)) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Sq = Sq; J.H_kv = n_idx; J.D = D_idx; J.block = block; J.top_k = top_k;
    J.KH = key_heads; J.key_fp8 = k_idx8 != NULL; J.k_idx8 = k_idx8; J.k_scale = k_scale;
    J.q_idx = q_idx; J.k_idx = k_idx; J.lens = lens; J.kv_offsets = kv_offsets;
    J.kv_capacity = kv_capacity; J.rows = rows;
    J.n_rows = rows ? n_rows : (int64_t)B * Sq;
    J.block_ids = block_ids; J.block_scores = block_scores;
    J.all_scores = all_scores; J.nb_max = nb_max; J.boundary = boundary;
    return run(&J, 0, n_threads);
}

/* One index head per GQA group with its own bf16 keys (k_idx [T, H_kv, D]). */
int oracle_index_topk(int B, int Sq, int H_kv, int D_idx, int block, int top_k,
                      const uint16_t *q_idx, const uint16_t *k_idx,
                      const int32_t *lens, const int64_t *kv_offsets, int64_t kv_capacity,
                      const int64_t *rows, int64_t n_rows,
                      int32_t *block_ids, float *block_scores,
                      double *all_scores, int nb_max, double *boundary, int n_threads)
{
    return oracle_index_topk_ex(B, Sq, H_kv, H_kv, D_idx, block, top_k, q_idx, k_idx, NULL, NULL,
                                lens, kv_offsets, kv_capacity, rows, n_rows, block_ids,
                                block_scores, all_scores, nb_max, boundary, n_threads);
}

/* Sparse branch: out[n_rows, H_q, D] in double, given the block ids of each
 * (row, index head) [B*Sq, n_idx, top_k], group g using index head
 * g / (H_kv / n_idx); optionally the sum of each row's normalised weights. */
int oracle_sparse_attention_ex(int B, int Sq, int H_q, int H_kv, int n_idx, int D, int block,
                               int top_k, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               const int32_t *block_ids, const int32_t *lens,
                               const int64_t *kv_offsets, int64_t kv_capacity, double scale,
                               const int64_t *rows, int64_t n_rows,
                               double *out, double *wsum, int n_threads)
{
    if (B < 1 || Sq < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv || D < 1 || block < 1 || top_k < 1)
        return -1;
    if (n_idx < 1 || H_kv % n_idx) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Sq = Sq; J.H_q = H_q; J.H_kv = H_kv; J.D = D; J.block = block; J.top_k = top_k;
    J.n_idx = n_idx;
    J.q = q; J.k = k; J.v = v; J.block_ids_in = block_ids; J.lens = lens;
    J.kv_offsets = kv_offsets; J.kv_capacity = kv_capacity; J.scale = scale;
    J.rows = rows; J.n_rows = rows ? n_rows : (int64_t)B * Sq;
    J.out = out; J.wsum = wsum;
    return run(&J, 1, n_threads);
}

/* One index head per GQA group: block_ids [B*Sq, H_kv, top_k]. */
int oracle_sparse_attention(int B, int Sq, int H_q, int H_kv, int D, int block, int top_k,
                            const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *block_ids, const int32_t *lens,
                            const int64_t *kv_offsets, int64_t kv_capacity, double scale,
                            const int64_t *rows, int64_t n_rows,
                            double *out, double *wsum, int n_threads)
{
    return oracle_sparse_attention_ex(B, Sq, H_q, H_kv, H_kv, D, block, top_k, q, k, v, block_ids,
                                      lens, kv_offsets, kv_capacity, scale, rows, n_rows, out, wsum,
                                      n_threads);
}

/* ------------------------------------------------------------------ backward
 * Gradient of the sparse branch (the index branch's selection is piecewise
 * constant in its inputs and passes no gradient).  For one (row, head) with
 * kept keys K (t in a kept block, t <= p), z_t = scale * q.k_t,
 * P = softmax(z), O = sum_t P_t v_t, and an upstream gradient dO:
 *   dV_t += P_t dO                 dP_t = dO . v_t
 *   Delta = sum_t P_t dP_t (= dO . O)
 *   dZ_t = P_t (dP_t - Delta)
 *   dQ   = scale * sum_t dZ_t k_t  dK_t += scale * dZ_t q
 * dK and dV of a key sum over every (row, head) of its group that kept it.
 * A job is one (sequence, group): it owns the dK/dV rows of that sequence
 * and group, so jobs never write the same element. */
typedef struct {
    int B, Sq, H_q, H_kv, n_idx, D, block, top_k;
    int64_t kv_capacity;
    const uint16_t *q, *k, *v, *dout;
    const int32_t *lens, *block_ids;
    const int64_t *kv_offsets;
    double scale;
    double *dq;      /* [B*Sq, H_q, D] */
    double *dk, *dv; /* [kv_capacity, H_kv, D], zeroed by the caller */
    int err;
} bjob_t;

typedef struct { bjob_t *job; int first, stride; } bslice_t;

static void bwd_seq_group(bjob_t *J, int b, int g)
{
    const int K = J->top_k, blk = J->block, D = J->D, G = J->H_q / J->H_kv;
    const int64_t L = J->lens[b];
    if (L < J->Sq || J->kv_offsets[b] < 0 || J->kv_offsets[b] + L > J->kv_capacity) {
        J->err = 1;
        return;
    }
    const int64_t off = J->kv_offsets[b];
    const int gi = g / (J->H_kv / J->n_idx);
    int64_t max_keys = (int64_t)K * blk;
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * max_keys);
    double *z = (double *)malloc(sizeof(double) * max_keys);
    double *dp = (double *)malloc(sizeof(double) * max_keys);
    for (int i = 0; i < J->Sq; ++i) {
        const int64_t r = (int64_t)b * J->Sq + i;
        const int64_t p = L - J->Sq + i;
        const int own = (int)(p / blk);
        const int32_t *ids = J->block_ids + (r * J->n_idx + gi) * (int64_t)K;
        int64_t nk = 0;
        for (int q = 0; q < K; ++q) {
            int j = ids[q];
            if (j < 0) continue;
            if (j > own) { J->err = 2; continue; }
            int64_t t_end = (int64_t)(j + 1) * blk;
            if (t_end > p + 1) t_end = p + 1;
            for (int64_t t = (int64_t)j * blk; t < t_end && nk < max_keys; ++t) keys[nk++] = t;
        }
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            const uint16_t *qh = J->q + (r * J->H_q + h) * (int64_t)D;
            const uint16_t *doh = J->dout + (r * J->H_q + h) * (int64_t)D;
            /* forward: softmax weights */
            double m = -INFINITY;
            for (int64_t a = 0; a < nk; ++a) {
                const uint16_t *kt = J->k + ((off + keys[a]) * J->H_kv + g) * (int64_t)D;
                double s = 0.0;
                for (int d = 0; d < D; ++d) s += bf16_to_double(qh[d]) * bf16_to_double(kt[d]);
                z[a] = s * J->scale;
                if (z[a] > m) m = z[a];
            }
            double l = 0.0;
            for (int64_t a = 0; a < nk; ++a) { z[a] = exp(z[a] - m); l += z[a]; }
            for (int64_t a = 0; a < nk; ++a) z[a] /= l;          /* z now holds P */
            /* dP, Delta, dV */
            double delta = 0.0;
            for (int64_t a = 0; a < nk; ++a) {
                const int64_t kr = (off + keys[a]) * J->H_kv + g;
                const uint16_t *vt = J->v + kr * (int64_t)D;
                double s = 0.0;
                for (int d = 0; d < D; ++d) {
                    const double dod = bf16_to_double(doh[d]);
                    s += dod * bf16_to_double(vt[d]);
                    J->dv[kr * D + d] += z[a] * dod;
                }
                dp[a] = s;
                delta += z[a] * s;
            }
            /* dZ, dQ, dK */
            double *dqh = J->dq + (r * J->H_q + h) * (int64_t)D;
            for (int d = 0; d < D; ++d) dqh[d] = 0.0;
            for (int64_t a = 0; a < nk; ++a) {
                const double dz = z[a] * (dp[a] - delta);
                const int64_t kr = (off + keys[a]) * J->H_kv + g;
                const uint16_t *kt = J->k + kr * (int64_t)D;
                for (int d = 0; d < D; ++d) {
                    dqh[d] += J->scale * dz * bf16_to_double(kt[d]);
                    J->dk[kr * D + d] += J->scale * dz * bf16_to_double(qh[d]);
                }
            }
        }
    }
    free(keys); free(z); free(dp);
}

static void *bwd_worker(void *arg)
{
    bslice_t *s = (bslice_t *)arg;
    const int n = s->job->B * s->job->H_kv;
    for (int jb = s->first; jb < n; jb += s->stride) bwd_seq_group(s->job, jb / s->job->H_kv, jb % s->job->H_kv);
    return NULL;
}

/* Backward of the sparse branch for all B*Sq rows: dq [B*Sq, H_q, D] is
 * written; dk, dv [kv_capacity, H_kv, D] (double) are accumulated into and
 * must start at zero.  block_ids [B*Sq, n_idx, top_k] as for the forward. */
int oracle_sparse_attention_backward(int B, int Sq, int H_q, int H_kv, int n_idx, int D, int block,
                                     int top_k, const uint16_t *q, const uint16_t *k,
                                     const uint16_t *v, const uint16_t *dout,
                                     const int32_t *block_ids, const int32_t *lens,
                                     const int64_t *kv_offsets, int64_t kv_capacity, double scale,
                                     double *dq, double *dk, double *dv, int n_threads)
{
    if (B < 1 || Sq < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv || D < 1 || block < 1 || top_k < 1)
        return -1;
    if (n_idx < 1 || H_kv % n_idx) return -1;
    bjob_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Sq = Sq; J.H_q = H_q; J.H_kv = H_kv; J.n_idx = n_idx; J.D = D; J.block = block;
    J.top_k = top_k; J.kv_capacity = kv_capacity; J.q = q; J.k = k; J.v = v; J.dout = dout;
    J.lens = lens; J.block_ids = block_ids; J.kv_offsets = kv_offsets; J.scale = scale;
    J.dq = dq; J.dk = dk; J.dv = dv;
    int nt = n_threads < 1 ? 1 : (n_threads > 512 ? 512 : n_threads);
    if (nt > B * H_kv) nt = B * H_kv;
    pthread_t th[512];
    bslice_t sl[512];
    for (int t = 0; t < nt; ++t) {
        sl[t].job = &J; sl[t].first = t; sl[t].stride = nt;
        pthread_create(&th[t], NULL, bwd_worker, &sl[t]);
    }
    for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
    return J.err;
}
