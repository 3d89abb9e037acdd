/*
 * oracle.c -- plain, slow CPU restatement of the lightning indexer and its
 * per-query top-k: the dense full-prefix form, PIVOT's grouped form (Reuse
 * and Refine) and the MTP decode form.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link or call
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header or constant with the CUDA library.
 *
 * Every score is accumulated in double from inputs decoded exactly (bf16 or
 * fp32).  Every selection is a full sort.  No blocking, fusion or reordering
 * beyond what each definition states.
 *
 * Sources (pages are cited by title and by the part of the page):
 *  - "PIVOT: Efficient Query-Group Indexing for Token-Level Sparse Attention"
 *    (arXiv 2607.24593):
 *      Method, first paragraph: every query is scored against its whole
 *        prefix by the indexer score, Eq. (1), then keeps a top-k set.
 *        The text of Eq. (1) did not survive; the reading used here is the
 *        DSA lightning-indexer score
 *            I[t,s] = sum_j w[t,j] * max(0, q[t,j] . k[s]),   s <= t,
 *        which matches observation O3 of the same page (a per-head ReLU of
 *        q_{t,j} . k_s, summed over heads).
 *      Method, grouping paragraph: contiguous groups of a fixed size g that
 *        never cross a request boundary; the last group may be smaller.
 *      Experimental setup: the proxy is the mean of the group's queries;
 *        PIVOT-Reuse shares the proxy's top-k; k = 2048, c = 2k.
 *      Abstract: one shared full-prefix traversal yields a candidate set,
 *        then PIVOT-Refine re-scores it with each member's own indexer.
 *      Method, decode paragraph: the decode group is the current query plus
 *        the MTP draft queries of the same step.
 *      Results, indexer speed: PIVOT falls back to a dense scan for short
 *        groups, so it is never slower than the dense indexer.  The
 *        threshold is not given; here it is an argument, dense_below: a
 *        group whose shared scan would cover at most dense_below keys
 *        (t_last + 1 <= dense_below) is not grouped, every member scores its
 *        own prefix and takes its own top-k.  dense_below = 0 turns it off.
 *  - Block pre-filter (mode ORA_BLOCK), a candidate generator for Refine built
 *    from two other pages: "Not All Tokens Deserve Equal Resolution:
 *    Score-Adaptive Indexing for Sparse Attention in Long-Context LLMs"
 *    (abstract: coarse summaries of key chunks are scored first, then the
 *    tokens of the chosen chunks are refined exactly) and "Uncertainty-gated
 *    selection for block-sparse attention" (Sec. 3.1, step 1: a block is
 *    summarised by the mean of its keys, block size 64).  Readings: the
 *    block score is the indexer score of the group proxy against the block's
 *    mean key; only complete blocks inside the group's prefix are scored, so
 *    no key after the group's last member takes part; the partial block that
 *    holds the last member is always a candidate; the candidate budget c
 *    counts tokens (c / bn blocks, one of them the partial block if there
 *    is one); the mean key is rounded like the proxy (fp32 sum in key order,
 *    IEEE division, bf16 round-to-nearest-even).
 *  - Block pre-filter with the Quest bound (mode ORA_QUEST): the same
 *    candidate generator, but a block is summarised by the per-dimension
 *    minimum and maximum of its keys, and its score for a query is the
 *    coordinate-wise upper bound of q . k over the block ("Uncertainty-gated
 *    selection for block-sparse attention", Sec. 3.1, Eq. (2), after Quest):
 *    sum over dimensions of max(q_d * kmax_d, q_d * kmin_d).  Reading: the
 *    indexer scores each head's bound as it scores a dot product, so the
 *    block score is sum_j w_j * max(0, bound_j); everything else (complete
 *    blocks only, the partial block always a candidate, c / bn blocks) is
 *    as in ORA_BLOCK.  The minimum and maximum of bf16 keys are bf16 keys:
 *    no rounding step.
 *  - Token-sparse attention (ora_sparse_attn), the consumer of the selected
 *    sets: the PIVOT page's introduction says the selected set feeds sparse
 *    MLA attention.  The pages give no formula; the reading used here is
 *    softmax attention restricted to the selected positions, in the
 *    absorbed MLA form of the production models that page names: one
 *    latent row per key serves as the key (all Dqk dimensions) and its
 *    first Dv dimensions as the value, shared by every head.
 *  - Readings where the pages are silent (each also listed in the design
 *    notes): proxy of w = mean of w; proxy arithmetic = fp32 sum in member
 *    order, IEEE division, then round-to-nearest-even to bf16 for bf16
 *    queries; ties in the top-k go to the lower index; the output lists the
 *    selected positions in ascending order, padded with -1; Reuse member i
 *    takes the proxy ranking restricted to its own prefix s <= t_i; the
 *    shared scan of a group covers the prefix of its last member.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -pthread
 *        -o liboracle.so oracle.c      (see oracle/build.py)
 * -ffp-contract=off keeps every float operation of the proxy step separately
 * rounded, as its definition states.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORA_BF16 = 0, ORA_F32 = 1 };
enum { ORA_DENSE = 0, ORA_REUSE = 1, ORA_REFINE = 2, ORA_BLOCK = 3, ORA_QUEST = 4 };

/* ---------------------------------------------------------------- inputs */

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* element i of a bf16 (bit pattern) or fp32 array, exactly, as a double */
static double load_elem(const void *base, int dtype, size_t i) {
    if (dtype == ORA_BF16) return bf16_bits_to_double(((const uint16_t *)base)[i]);
    return (double)((const float *)base)[i];
}

/* round-to-nearest-even of a finite float to a bf16 bit pattern */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* --------------------------------------------------------------- Eq. (1) */

/* I[t,s] = sum_j w[t,j] * max(0, sum_i q[t,j,i] * k[s,i]).
 * q_row: element offset of q[t,0,0] in q; k_row: offset of k[s,0] in k. */
static double index_score(const void *q, size_t q_row, const void *k, size_t k_row,
                          const float *w_row, int H, int d, int dtype) {
    double total = 0.0;
    for (int j = 0; j < H; ++j) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i)
            dot += load_elem(q, dtype, q_row + (size_t)j * d + i) * load_elem(k, dtype, k_row + i);
        if (dot > 0.0) total += (double)w_row[j] * dot;
    }
    return total;
}

/* ------------------------------------------------------------- selection */

typedef struct {
    double score;
    int pos;
} cand_t;

/* higher score first; equal scores: lower position first */
static int by_score_desc_pos_asc(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos > y->pos) - (x->pos < y->pos);
}

static int int_asc(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* The first min(k, n) candidates in (score desc, pos asc) order, written as
 * ascending positions, then -1 up to k.  Sorts c in place. */
static void select_topk(cand_t *c, int n, int k, int *out) {
    qsort(c, (size_t)n, sizeof(cand_t), by_score_desc_pos_asc);
    int m = n < k ? n : k;
    for (int i = 0; i < m; ++i) out[i] = c[i].pos;
    qsort(out, (size_t)m, sizeof(int), int_asc);
    for (int i = m; i < k; ++i) out[i] = -1;
}

/* ------------------------------------------------------------ exported */

/* Scores of one query row against n consecutive keys starting at key row
 * key0: out[s] = I[q_row, key0 + s].  q_row indexes q [*, H, d] and w [*, H]. */
int ora_score_row(const void *q, const void *k, const float *w, int dtype, int H, int d,
                  long long q_row, long long key0, int n, double *out) {
    if (!q || !k || !w || !out || H <= 0 || d <= 0 || n < 0) return 1;
    for (int s = 0; s < n; ++s)
        out[s] = index_score(q, (size_t)q_row * H * d, k, (size_t)(key0 + s) * d,
                             w + (size_t)q_row * H, H, d, dtype);
    return 0;
}

/* The selection rule alone, applied to given scores (used to re-select on
 * scores exported by another implementation).  pos may be NULL (= 0..n-1). */
int ora_select(const double *scores, const int *pos, int n, int k, int *out) {
    if (n < 0 || k <= 0 || !out) return 1;
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    if (!c) return 2;
    for (int i = 0; i < n; ++i) {
        c[i].score = scores[i];
        c[i].pos = pos ? pos[i] : i;
    }
    select_topk(c, n, k, out);
    free(c);
    return 0;
}

/* Locate global row r among requests given by cu_seqlens. */
static int find_request(const int *cu, int num_seqs, long long r) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* Proxy of a group: per head and dimension the fp32 sum of the members'
 * queries in member order, divided by the group size (IEEE fp32), rounded
 * to bf16 for bf16 queries; w-proxy likewise in fp32.  Members are rows
 * m0, m0+1, ..., m0+cnt-1 of q [*, H, d] and w [*, H].
 * qbar receives H*d elements in dtype format, wbar H floats. */
static void group_proxy(const void *q, const float *w, int dtype, int H, int d,
                        long long m0, int cnt, void *qbar, float *wbar) {
    for (int j = 0; j < H; ++j) {
        for (int i = 0; i < d; ++i) {
            float sum = 0.0f;
            for (int m = 0; m < cnt; ++m)
                sum = sum + (float)load_elem(q, dtype, (size_t)(m0 + m) * H * d + (size_t)j * d + i);
            float mean = sum / (float)cnt;
            if (dtype == ORA_BF16) ((uint16_t *)qbar)[(size_t)j * d + i] = float_to_bf16_rne(mean);
            else ((float *)qbar)[(size_t)j * d + i] = mean;
        }
        float ws = 0.0f;
        for (int m = 0; m < cnt; ++m) ws = ws + w[(size_t)(m0 + m) * H + j];
        wbar[j] = ws / (float)cnt;
    }
}

/* Mean key of the bn keys at rows r0 .. r0+bn-1 of k [*, d]: per dimension
 * the fp32 sum in key order, divided by bn (IEEE fp32), rounded to bf16 for
 * bf16 keys.  kbar receives d elements in dtype format. */
static void block_mean(const void *k, int dtype, int d, long long r0, int bn, void *kbar) {
    for (int i = 0; i < d; ++i) {
        float sum = 0.0f;
        for (int r = 0; r < bn; ++r) sum = sum + (float)load_elem(k, dtype, (size_t)(r0 + r) * d + i);
        float mean = sum / (float)bn;
        if (dtype == ORA_BF16) ((uint16_t *)kbar)[i] = float_to_bf16_rne(mean);
        else ((float *)kbar)[i] = mean;
    }
}

/* Exported for tests of the block-mean step alone. */
/* Quest block score of the proxy (qbar [H, d], wbar [H]) for key rows
 * r0 .. r0+bn-1: per head the coordinate-wise upper bound of q . k over the
 * block, sum_d max(q_d * kmax_d, q_d * kmin_d), then the indexer's weighted
 * ReLU over the heads. */
static double quest_score(const void *qbar, const float *wbar, const void *k, int dtype, int H, int d,
                          long long r0, int bn) {
    double total = 0.0;
    for (int j = 0; j < H; ++j) {
        double bound = 0.0;
        for (int i = 0; i < d; ++i) {
            double lo = load_elem(k, dtype, (size_t)r0 * d + i), hi = lo;
            for (int r = 1; r < bn; ++r) {
                double v = load_elem(k, dtype, (size_t)(r0 + r) * d + i);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            double qd = load_elem(qbar, dtype, (size_t)j * d + i);
            double a = qd * hi, b = qd * lo;
            bound += a > b ? a : b;
        }
        if (bound > 0.0) total += (double)wbar[j] * bound;
    }
    return total;
}

int ora_block_mean(const void *k, int dtype, int d, long long r0, int bn, void *kbar) {
    if (!k || !kbar || bn <= 0 || d <= 0) return 1;
    block_mean(k, dtype, d, r0, bn, kbar);
    return 0;
}

/* Exported for tests of the proxy step alone. */
int ora_group_proxy(const void *q, const float *w, int dtype, int H, int d, long long m0, int cnt,
                    void *qbar, float *wbar) {
    if (!q || !w || !qbar || !wbar || cnt <= 0) return 1;
    group_proxy(q, w, dtype, H, d, m0, cnt, qbar, wbar);
    return 0;
}

/* One grouped selection.
 *   q, w: query rows; members are rows m0 .. m0+cnt-1; member t positions
 *         are pos0 .. pos0+cnt-1 (request-local); the group's last member
 *         sits at t_last = pos0+cnt-1.
 *   keys: key rows key0 + s for s = 0 .. t_last.
 *   mode: ORA_REUSE, ORA_REFINE, ORA_BLOCK or ORA_QUEST; c: candidate budget (Refine,
 *         Block); bn: block size (Block).
 *   member: which member (0..cnt-1) to produce; out: k entries. */
static int grouped_member_topk(const void *q, const void *k, const float *w, int dtype, int H, int d,
                               long long m0, int cnt, int pos0, long long key0, int topk, int c,
                               int mode, int bn, int member, int *out) {
    int t_last = pos0 + cnt - 1;
    int n = t_last + 1;
    size_t esz = dtype == ORA_BF16 ? 2 : 4;
    void *qbar = malloc(esz * (size_t)H * d);
    float *wbar = (float *)malloc(sizeof(float) * (size_t)H);
    cand_t *pc = (cand_t *)malloc(sizeof(cand_t) * (size_t)n);
    if (!qbar || !wbar || !pc) { free(qbar); free(wbar); free(pc); return 2; }
    group_proxy(q, w, dtype, H, d, m0, cnt, qbar, wbar);
    int t = pos0 + member;
    int rc = 0;
    if (mode == ORA_BLOCK || mode == ORA_QUEST) {
        /* complete blocks [j*bn, (j+1)*bn) inside the prefix, scored by the
         * proxy against their mean keys (ORA_BLOCK) or by the Quest bound
         * (ORA_QUEST); the partial block [part0, n) */
        int nfull = n / bn;
        int part0 = nfull * bn;
        int want = c / bn - (part0 < n ? 1 : 0);
        int take = want < nfull ? want : nfull;
        if (take < 0) take = 0;
        void *kbar = malloc(esz * (size_t)d);
        /* C holds distinct positions of the prefix: at most n entries */
        cand_t *mc = (cand_t *)malloc(sizeof(cand_t) * (size_t)n);
        if (!kbar || !mc) { free(kbar); free(mc); rc = 2; goto done; }
        for (int j = 0; j < nfull; ++j) {
            if (mode == ORA_QUEST) {
                pc[j].score = quest_score(qbar, wbar, k, dtype, H, d, key0 + (long long)j * bn, bn);
            } else {
                block_mean(k, dtype, d, key0 + (long long)j * bn, bn, kbar);
                pc[j].score = index_score(qbar, 0, kbar, 0, wbar, H, d, dtype);
            }
            pc[j].pos = j;
        }
        qsort(pc, (size_t)nfull, sizeof(cand_t), by_score_desc_pos_asc);
        /* C = tokens of the top `take` blocks and of the partial block; the
         * member re-scores those inside its own prefix */
        int m = 0;
        for (int i = 0; i < take; ++i)
            for (int r = 0; r < bn; ++r) {
                int s = pc[i].pos * bn + r;
                if (s > t) continue;
                mc[m].score = index_score(q, (size_t)(m0 + member) * H * d, k, (size_t)(key0 + s) * d,
                                          w + (size_t)(m0 + member) * H, H, d, dtype);
                mc[m].pos = s;
                ++m;
            }
        for (int s = part0; s < n && s <= t; ++s) {
            mc[m].score = index_score(q, (size_t)(m0 + member) * H * d, k, (size_t)(key0 + s) * d,
                                      w + (size_t)(m0 + member) * H, H, d, dtype);
            mc[m].pos = s;
            ++m;
        }
        select_topk(mc, m, topk, out);
        free(mc);
        free(kbar);
        goto done;
    }
    /* one shared scan of the group's full prefix with the proxy */
    for (int s = 0; s < n; ++s) {
        pc[s].score = index_score(qbar, 0, k, (size_t)(key0 + s) * d, wbar, H, d, dtype);
        pc[s].pos = s;
    }
    if (mode == ORA_REUSE) {
        /* the proxy ranking, restricted to the member's own prefix */
        select_topk(pc, t + 1, topk, out);
    } else {
        /* candidate set C: the proxy's top-min(c, n) over the whole prefix */
        qsort(pc, (size_t)n, sizeof(cand_t), by_score_desc_pos_asc);
        int nc = n < c ? n : c;
        cand_t *mc = (cand_t *)malloc(sizeof(cand_t) * (size_t)(nc > 0 ? nc : 1));
        if (!mc) { rc = 2; goto done; }
        int m = 0;
        for (int i = 0; i < nc; ++i) {
            int s = pc[i].pos;
            if (s > t) continue; /* the member's causal mask */
            mc[m].score = index_score(q, (size_t)(m0 + member) * H * d, k, (size_t)(key0 + s) * d,
                                      w + (size_t)(m0 + member) * H, H, d, dtype);
            mc[m].pos = s;
            ++m;
        }
        select_topk(mc, m, topk, out);
        free(mc);
    }
done:
    free(qbar);
    free(wbar);
    free(pc);
    return rc;
}

/* ------------------------------------------------------ threaded drivers */

typedef struct {
    int kind; /* 0 dense, 1 pivot, 2 decode */
    const void *q, *k;
    const float *w;
    int dtype, H, d, topk, g, c, mode, bn, dense_below;
    const int *cu;
    int num_seqs;
    const long long *rows;
    int nrows;
    /* decode */
    const int *kv_len;
    int G, n_max;
    int *out;
    int next;
    int rc;
    pthread_mutex_t lock;
} job_t;

static int take(job_t *J) {
    pthread_mutex_lock(&J->lock);
    int i = J->next++;
    pthread_mutex_unlock(&J->lock);
    return i;
}

static void set_rc(job_t *J, int rc) {
    if (!rc) return;
    pthread_mutex_lock(&J->lock);
    if (!J->rc) J->rc = rc;
    pthread_mutex_unlock(&J->lock);
}

static void run_dense_row(job_t *J, int i) {
    long long r = J->rows[i];
    int b = find_request(J->cu, J->num_seqs, r);
    int t = (int)(r - J->cu[b]);
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(t + 1));
    if (!c) { set_rc(J, 2); return; }
    for (int s = 0; s <= t; ++s) {
        c[s].score = index_score(J->q, (size_t)r * J->H * J->d, J->k, (size_t)(J->cu[b] + s) * J->d,
                                 J->w + (size_t)r * J->H, J->H, J->d, J->dtype);
        c[s].pos = s;
    }
    select_topk(c, t + 1, J->topk, J->out + (size_t)i * J->topk);
    free(c);
}

static void run_pivot_row(job_t *J, int i) {
    long long r = J->rows[i];
    int b = find_request(J->cu, J->num_seqs, r);
    int n = J->cu[b + 1] - J->cu[b];
    int t = (int)(r - J->cu[b]);
    int lo = (t / J->g) * J->g;
    int hi = lo + J->g < n ? lo + J->g : n;
    /* a short group (its last member's prefix holds at most dense_below
     * keys) falls back to the dense top-k of each member */
    if (J->dense_below > 0 && hi <= J->dense_below) {
        run_dense_row(J, i);
        return;
    }
    set_rc(J, grouped_member_topk(J->q, J->k, J->w, J->dtype, J->H, J->d, J->cu[b] + lo, hi - lo, lo,
                                  J->cu[b], J->topk, J->c, J->mode, J->bn, t - lo,
                                  J->out + (size_t)i * J->topk));
}

/* decode: rows[i] is a request b; writes G rows of topk. */
static void run_decode_req(job_t *J, int i) {
    int b = (int)J->rows[i];
    int n = J->kv_len[b];
    int G = J->G, H = J->H, d = J->d;
    int *out = J->out + (size_t)i * G * J->topk;
    long long key0 = (long long)b * J->n_max;
    long long m0 = (long long)b * G; /* query rows of q [B*G, H, d] */
    if (J->mode == ORA_DENSE) {
        for (int m = 0; m < G; ++m) {
            int t = n - G + m;
            cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(t + 1));
            if (!c) { set_rc(J, 2); return; }
            for (int s = 0; s <= t; ++s) {
                c[s].score = index_score(J->q, (size_t)(m0 + m) * H * d, J->k, (size_t)(key0 + s) * d,
                                         J->w + (size_t)(m0 + m) * H, H, d, J->dtype);
                c[s].pos = s;
            }
            select_topk(c, t + 1, J->topk, out + (size_t)m * J->topk);
            free(c);
        }
    } else {
        for (int m = 0; m < G; ++m)
            set_rc(J, grouped_member_topk(J->q, J->k, J->w, J->dtype, H, d, m0, G, n - G, key0,
                                          J->topk, J->c, J->mode, J->bn, m, out + (size_t)m * J->topk));
    }
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        int i = take(J);
        if (i >= J->nrows) break;
        if (J->kind == 0) run_dense_row(J, i);
        else if (J->kind == 1) run_pivot_row(J, i);
        else run_decode_req(J, i);
    }
    return NULL;
}

static int run_job(job_t *J, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    J->next = 0;
    J->rc = 0;
    pthread_mutex_init(&J->lock, NULL);
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (!started) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J->lock);
    return J->rc;
}

static int check_requests(const int *cu, int num_seqs) {
    if (!cu || num_seqs <= 0 || cu[0] != 0) return 1;
    for (int b = 0; b < num_seqs; ++b)
        if (cu[b + 1] < cu[b]) return 1;
    return 0;
}

/* Dense top-k for the given global query rows.
 * q [T,H,d], k [T,d] (bf16 bits or fp32), w [T,H] fp32; cu_seqlens host
 * [num_seqs+1]; out [nrows, topk] int32. */
int ora_dense_topk(const void *q, const void *k, const float *w, int dtype, const int *cu_seqlens,
                   int num_seqs, int H, int d, int topk, const long long *rows, int nrows, int *out,
                   int nthreads) {
    if (!q || !k || !w || !out || (nrows > 0 && !rows) || H <= 0 || d <= 0 || topk <= 0) return 1;
    if (check_requests(cu_seqlens, num_seqs)) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= cu_seqlens[num_seqs]) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 0; J.q = q; J.k = k; J.w = w; J.dtype = dtype; J.H = H; J.d = d; J.topk = topk;
    J.cu = cu_seqlens; J.num_seqs = num_seqs; J.rows = rows; J.nrows = nrows; J.out = out;
    return run_job(&J, nthreads);
}

/* PIVOT top-k (mode ORA_REUSE, ORA_REFINE, ORA_BLOCK or ORA_QUEST) for the given
 * global member rows; same layouts as ora_dense_topk; g >= 1; Refine and
 * Block / Quest need c >= topk and bn >= 1 (c / bn blocks).  Groups whose
 * last member's prefix holds at most dense_below keys (0 = none) take the
 * dense top-k instead. */
int ora_pivot_topk(const void *q, const void *k, const float *w, int dtype, const int *cu_seqlens,
                   int num_seqs, int H, int d, int topk, int g, int c, int mode, int bn, int dense_below,
                   const long long *rows, int nrows, int *out, int nthreads) {
    if (!q || !k || !w || !out || (nrows > 0 && !rows) || H <= 0 || d <= 0 || topk <= 0 || g <= 0 ||
        dense_below < 0)
        return 1;
    if (mode != ORA_REUSE && mode != ORA_REFINE && mode != ORA_BLOCK && mode != ORA_QUEST) return 1;
    if ((mode == ORA_REFINE || mode == ORA_BLOCK || mode == ORA_QUEST) && c < topk) return 1;
    if ((mode == ORA_BLOCK || mode == ORA_QUEST) && bn < 1) return 1;
    if (check_requests(cu_seqlens, num_seqs)) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= cu_seqlens[num_seqs]) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 1; J.q = q; J.k = k; J.w = w; J.dtype = dtype; J.H = H; J.d = d; J.topk = topk;
    J.g = g; J.c = c; J.mode = mode; J.bn = bn; J.dense_below = dense_below;
    J.cu = cu_seqlens; J.num_seqs = num_seqs; J.rows = rows;
    J.nrows = nrows; J.out = out;
    return run_job(&J, nthreads);
}

/* Decode top-k for the given requests.
 * q [B,G,H,d], kcache [B,n_max,d], w [B,G,H]; kv_len host [B] with
 * G <= kv_len[b] <= n_max; query m of request b sits at position
 * kv_len[b]-G+m and the cache already holds the keys of the group.
 * mode ORA_DENSE, ORA_REUSE, ORA_REFINE (c >= topk), ORA_BLOCK or ORA_QUEST
 * (c >= topk, bn >= 1); out [nreqs,G,topk]. */
int ora_decode_topk(const void *q, const void *kcache, const float *w, int dtype, const int *kv_len,
                    int B, int G, int n_max, int H, int d, int topk, int c, int mode, int bn,
                    const long long *reqs, int nreqs, int *out, int nthreads) {
    if (!q || !kcache || !w || !kv_len || !out || (nreqs > 0 && !reqs) || H <= 0 || d <= 0 ||
        topk <= 0 || G <= 0)
        return 1;
    if (mode != ORA_DENSE && mode != ORA_REUSE && mode != ORA_REFINE && mode != ORA_BLOCK && mode != ORA_QUEST)
        return 1;
    if ((mode == ORA_REFINE || mode == ORA_BLOCK || mode == ORA_QUEST) && c < topk) return 1;
    if ((mode == ORA_BLOCK || mode == ORA_QUEST) && bn < 1) return 1;
    for (int i = 0; i < nreqs; ++i) {
        if (reqs[i] < 0 || reqs[i] >= B) return 1;
        int n = kv_len[reqs[i]];
        if (n < G || n > n_max) return 1;
    }
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 2; J.q = q; J.k = kcache; J.w = w; J.dtype = dtype; J.H = H; J.d = d; J.topk = topk;
    J.c = c; J.mode = mode; J.bn = bn; J.kv_len = kv_len; J.G = G; J.n_max = n_max; J.rows = reqs;
    J.nrows = nreqs; J.out = out;
    return run_job(&J, nthreads);
}

/* ------------------------------------------------ token-sparse attention */

typedef struct {
    const void *q, *kv;
    int dtype, Ha, Dqk, Dv, topk;
    const int *idx, *cu_q, *cu_kv;
    int S;
    double scale;
    const long long *rows;
    int nrows;
    double *o, *lse;
    int next, rc;
    pthread_mutex_t lock;
} attn_job_t;

/* One query row r, every head:
 *   z_j = scale * sum_i q[r,h,i] * kv[row_j, i]   for the listed j (idx >= 0),
 *         row_j = cu_kv[b] + idx[r, j], b the request of r (cu_q);
 *   o[h, c] = sum_j exp(z_j - m) * kv[row_j, c] / sum_j exp(z_j - m), c < Dv,
 *   lse[h]  = m + log(sum_j exp(z_j - m)),  m = max_j z_j.
 * A row with no listed position gets o = 0 and lse = -inf.  Each listed
 * entry is one term (a position listed twice counts twice). */
static int attn_row(attn_job_t *J, int i) {
    long long r = J->rows[i];
    int b = find_request(J->cu_q, J->S, r);
    int nkv = J->cu_kv[b + 1] - J->cu_kv[b];
    const int *ix = J->idx + (size_t)r * J->topk;
    double *z = (double *)malloc(sizeof(double) * (size_t)(J->topk > 0 ? J->topk : 1));
    if (!z) return 2;
    for (int j = 0; j < J->topk; ++j)
        if (ix[j] >= nkv) { free(z); return 1; }
    for (int h = 0; h < J->Ha; ++h) {
        double *o = J->o + ((size_t)i * J->Ha + h) * J->Dv;
        for (int c = 0; c < J->Dv; ++c) o[c] = 0.0;
        double m = -INFINITY;
        for (int j = 0; j < J->topk; ++j) {
            if (ix[j] < 0) continue;
            size_t kr = (size_t)(J->cu_kv[b] + ix[j]) * J->Dqk;
            size_t qr = ((size_t)r * J->Ha + h) * J->Dqk;
            double dot = 0.0;
            for (int e = 0; e < J->Dqk; ++e)
                dot += load_elem(J->q, J->dtype, qr + e) * load_elem(J->kv, J->dtype, kr + e);
            z[j] = J->scale * dot;
            if (z[j] > m) m = z[j];
        }
        if (m == -INFINITY) {
            J->lse[(size_t)i * J->Ha + h] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int j = 0; j < J->topk; ++j) {
            if (ix[j] < 0) continue;
            double p = exp(z[j] - m);
            l += p;
            size_t kr = (size_t)(J->cu_kv[b] + ix[j]) * J->Dqk;
            for (int c = 0; c < J->Dv; ++c) o[c] += p * load_elem(J->kv, J->dtype, kr + c);
        }
        for (int c = 0; c < J->Dv; ++c) o[c] /= l;
        J->lse[(size_t)i * J->Ha + h] = m + log(l);
    }
    free(z);
    return 0;
}

static void *attn_worker(void *arg) {
    attn_job_t *J = (attn_job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= J->nrows) break;
        int rc = attn_row(J, i);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            if (!J->rc) J->rc = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/* Token-sparse attention for the given query rows.
 *   q [R, Ha, Dqk], kv [Nkv, Dqk] (bf16 bits or fp32); idx [R, topk] int32
 *   positions inside the row's request (-1 = no entry); cu_q, cu_kv host
 *   [S+1]: query rows cu_q[b] .. cu_q[b+1]-1 read kv rows cu_kv[b] + idx.
 *   o [nrows, Ha, Dv] and lse [nrows, Ha] in double. */
int ora_sparse_attn(const void *q, const void *kv, int dtype, const int *idx, const int *cu_q, const int *cu_kv,
                    int S, int Ha, int Dqk, int Dv, int topk, double scale, const long long *rows, int nrows,
                    double *o, double *lse, int nthreads) {
    if (!q || !kv || !idx || !o || !lse || (nrows > 0 && !rows) || Ha <= 0 || Dqk <= 0 || Dv <= 0 ||
        Dv > Dqk || topk <= 0)
        return 1;
    if (check_requests(cu_q, S) || check_requests(cu_kv, S)) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= cu_q[S]) return 1;
    attn_job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.kv = kv; J.dtype = dtype; J.Ha = Ha; J.Dqk = Dqk; J.Dv = Dv; J.topk = topk;
    J.idx = idx; J.cu_q = cu_q; J.cu_kv = cu_kv; J.S = S; J.scale = scale; J.rows = rows; J.nrows = nrows;
    J.o = o; J.lse = lse;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    pthread_mutex_init(&J.lock, NULL);
    int started = 0;
    for (int t = 0; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, attn_worker, &J) == 0) ++started;
    if (!started) attn_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J.lock);
    return J.rc;
}
