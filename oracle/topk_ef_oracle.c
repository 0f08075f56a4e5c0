/*
 * CPU oracle for Top-k sparsification with error feedback and the gTop-k
 * pairwise merge.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU library computes.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or helper with the CUDA library, and the library never
 * calls it: there is no CPU fallback.
 *
 * Sources (web pages, cited by title and section):
 *  - "Sparsified SGD with Memory" (EPFL, arxivdaily listing, abstract): send
 *    only the most important entries (top-k) and keep track of the accumulated
 *    error in memory (error compensation).
 *  - "The Convergence of Sparsified Gradient Methods" (IST Austria / ETH /
 *    KTH, arxivdaily listing, abstract): each node sorts its gradient by
 *    magnitude, transmits a subset and accumulates the remaining components
 *    locally.
 *  - "A Distributed Synchronous SGD Algorithm with Global Top-k Sparsification
 *    for Low Bandwidth Networks" (nubint review), ABSTRACT and the method
 *    section: the global top-k largest absolute values over P workers,
 *    sparse gradients carried with their irregular indices, identified by a
 *    tournament in O(log P) rounds.
 *
 * Where the pages are silent the following readings are used (each is one
 * line of the project design notes):
 *  - acc = fmaf(lr, grad, residual): lr times the gradient plus the memory,
 *    rounded once to fp32 (C99 fmaf is correctly rounded).
 *  - |x| order is the order of key(x) = bits(x) & 0x7FFFFFFF as an unsigned
 *    integer (equal to |x| order for all non-NaN values, -0 == +0); every NaN
 *    has key 0x7FFFFFFF (above +Inf, all NaNs equal, whatever the payload:
 *    NaN payloads and signs are implementation-defined in IEEE 754).
 *  - ties in |x| go to the lower index, so the selected set is unique.
 *  - output pairs (int32 index, fp32 signed value) in ascending index order.
 *  - the residual keeps acc at unselected slots and +0.0f at selected slots.
 *  - merge: worker i pairs with worker i + 2^r in round r; at a common index
 *    the two fp32 values are added once (round to nearest even); an index held
 *    by one side is copied; each round keeps the top min(k, |union|) entries;
 *    a worker with no partner in a round passes its set on unchanged; the
 *    result is the top-k of worker 0's final set.
 *
 * Precision: the pages fix none; the method's arithmetic is the single fp32
 * fused multiply-add of the memory update and the single fp32 add of the
 * merge, so the oracle performs exactly those two fp32 operations and nothing
 * else in floating point.  Build with -ffp-contract=off and without
 * -ffast-math.
 *
 * Selection is written as its definition: build the composite
 *     c(i) = ((0x7FFFFFFF - key(x_i)) << 32) | i
 * whose ascending order is (|x| descending, index ascending), sort all of
 * them (backend 0) or keep the k smallest in a bounded max-heap (backend 1,
 * for inputs too large to sort in host memory), then put the chosen indices
 * in ascending order.  The two backends are cross-checked by the tests.
 *
 * Mutants: compiling with -DORACLE_MUTANT=<n> plants one deliberate mistake;
 * the test suite uses these builds to show that its pins catch each kind of
 * mistake.  The default build (no macro) is the oracle.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

static uint32_t bits_of(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    return u;
}

/* |x| order key. */
static uint32_t key_of(float x)
{
#if ORACLE_MUTANT == 3
    /* mistake: signed order (largest values instead of largest magnitudes) */
    uint32_t u = bits_of(x);
    return (u & 0x80000000u) ? (0x7FFFFFFFu - (u & 0x7FFFFFFFu)) / 2u : 0x3FFFFFFFu + (u >> 1);
#else
    /* every NaN orders as one value above +Inf, whatever its payload */
    if (x != x) return 0x7FFFFFFFu;
    return bits_of(x) & 0x7FFFFFFFu;
#endif
}

/* Composite whose ascending order is (|x| descending, index ascending). */
static uint64_t composite(float x, uint32_t i)
{
#if ORACLE_MUTANT == 2
    /* mistake: ties go to the higher index */
    return ((uint64_t)(0x7FFFFFFFu - key_of(x)) << 32) | (uint64_t)(0xFFFFFFFFu - i);
#else
    return ((uint64_t)(0x7FFFFFFFu - key_of(x)) << 32) | (uint64_t)i;
#endif
}

static uint32_t composite_index(uint64_t c)
{
#if ORACLE_MUTANT == 2
    return 0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFu);
#else
    return (uint32_t)(c & 0xFFFFFFFFu);
#endif
}

static int cmp_u64(const void *a, const void *b)
{
    uint64_t x = *(const uint64_t *)a, y = *(const uint64_t *)b;
    return (x > y) - (x < y);
}

static int cmp_u32(const void *a, const void *b)
{
    uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Memory update of one step: acc = lr * grad + residual, one rounding.
 * ("Sparsified SGD with Memory", abstract: error compensation keeps the
 * accumulated error in memory; "The Convergence of Sparsified Gradient
 * Methods", abstract: the untransmitted components accumulate locally.)
 */
void oracle_accumulate(const float *grad, const float *residual, int64_t n,
                       float lr, float *acc)
{
    for (int64_t i = 0; i < n; ++i) {
#if ORACLE_MUTANT == 1
        /* mistake: memory term dropped */
        acc[i] = lr * grad[i];
#elif ORACLE_MUTANT == 4
        /* mistake: operands transposed */
        acc[i] = fmaf(grad[i], residual[i], lr);
#elif ORACLE_MUTANT == 9
        /* mistake: two roundings instead of one */
        {
            volatile float p = lr * grad[i];
            acc[i] = p + residual[i];
        }
#else
        acc[i] = fmaf(lr, grad[i], residual[i]);
#endif
    }
}

/* ---- bounded max-heap of composites (keeps the k smallest) ---- */
static void heap_sift_down(uint64_t *h, int64_t m, int64_t i)
{
    for (;;) {
        int64_t l = 2 * i + 1, r = l + 1, big = i;
        if (l < m && h[l] > h[big]) big = l;
        if (r < m && h[r] > h[big]) big = r;
        if (big == i) return;
        uint64_t t = h[i]; h[i] = h[big]; h[big] = t;
        i = big;
    }
}

static void heap_sift_up(uint64_t *h, int64_t i)
{
    while (i > 0) {
        int64_t p = (i - 1) / 2;
        if (h[p] >= h[i]) return;
        uint64_t t = h[i]; h[i] = h[p]; h[p] = t;
        i = p;
    }
}

/*
 * Top-k of x[0..m) by (|x| descending, index ascending), where element j
 * carries index ids[j] (or j itself when ids is NULL).  Writes the k chosen
 * indices to chosen[0..k) in ascending order.  backend 0: sort all
 * composites; backend 1: bounded heap.
 */
static int select_topk(const float *x, const int32_t *ids, int64_t m,
                       int64_t k, int backend, uint32_t *chosen)
{
    if (k <= 0) return ORACLE_OK;
    if (k > m) return ORACLE_EINVAL;
    if (backend == 0) {
        uint64_t *c = (uint64_t *)malloc((size_t)m * sizeof(uint64_t));
        if (!c) return ORACLE_ENOMEM;
        for (int64_t j = 0; j < m; ++j)
            c[j] = composite(x[j], ids ? (uint32_t)ids[j] : (uint32_t)j);
        qsort(c, (size_t)m, sizeof(uint64_t), cmp_u64);
        for (int64_t j = 0; j < k; ++j) chosen[j] = composite_index(c[j]);
        free(c);
    } else {
        uint64_t *h = (uint64_t *)malloc((size_t)k * sizeof(uint64_t));
        if (!h) return ORACLE_ENOMEM;
        int64_t hm = 0;
        for (int64_t j = 0; j < m; ++j) {
            uint64_t c = composite(x[j], ids ? (uint32_t)ids[j] : (uint32_t)j);
            if (hm < k) {
                h[hm] = c;
                heap_sift_up(h, hm);
                ++hm;
            } else if (c < h[0]) {
                h[0] = c;
                heap_sift_down(h, hm, 0);
            }
        }
        for (int64_t j = 0; j < k; ++j) chosen[j] = composite_index(h[j]);
        free(h);
    }
#if ORACLE_MUTANT != 8
    qsort(chosen, (size_t)k, sizeof(uint32_t), cmp_u32);
#endif
    return ORACLE_OK;
}

/*
 * Exported selection: chosen[0..k) = ascending indices of the top-k of x.
 */
int oracle_select(const float *x, int64_t m, int64_t k, int backend,
                  int32_t *chosen)
{
    if (m < 0 || k < 0 || k > m || !x || (k > 0 && !chosen)) return ORACLE_EINVAL;
    return select_topk(x, NULL, m, k, backend, (uint32_t *)chosen);
}

/*
 * One error-feedback step on one flat tensor.
 *   acc          = fmaf(lr, grad, residual)
 *   S            = top-k of acc by (|acc| desc, index asc)
 *   out          = (i, acc[i]) for i in S, ascending i
 *   residual[i]  = +0.0f for i in S, acc[i] otherwise
 * (The Convergence of Sparsified Gradient Methods, abstract: transmit a
 * subset, accumulate the rest locally; A Distributed Synchronous SGD
 * Algorithm with Global Top-k Sparsification, ABSTRACT: the k largest
 * absolute values, sent with their indices.)
 */
int oracle_compress(const float *grad, float *residual, int64_t n, float lr,
                    int64_t k, int backend, int32_t *out_idx, float *out_val)
{
    if (n < 0 || k < 0 || k > n || n > 2147483647LL) return ORACLE_EINVAL;
    if (n > 0 && (!grad || !residual)) return ORACLE_EINVAL;
    if (k > 0 && (!out_idx || !out_val)) return ORACLE_EINVAL;
    if (n == 0) return ORACLE_OK;

    float *acc = (float *)malloc((size_t)n * sizeof(float));
    uint32_t *chosen = (uint32_t *)malloc((size_t)(k > 0 ? k : 1) * sizeof(uint32_t));
    if (!acc || !chosen) { free(acc); free(chosen); return ORACLE_ENOMEM; }

    oracle_accumulate(grad, residual, n, lr, acc);
    int rc = select_topk(acc, NULL, n, k, backend, chosen);
    if (rc != ORACLE_OK) { free(acc); free(chosen); return rc; }

    for (int64_t i = 0; i < n; ++i) residual[i] = acc[i];
    for (int64_t j = 0; j < k; ++j) {
        uint32_t i = chosen[j];
        out_idx[j] = (int32_t)i;
        out_val[j] = acc[i];
#if ORACLE_MUTANT != 5
        /* mistake 5 leaves the sent value in memory */
        residual[i] = 0.0f;
#endif
    }
    free(acc);
    free(chosen);
    return ORACLE_OK;
}

/*
 * Batched form: tensor l is grad[offsets[l] .. offsets[l+1]) with its own
 * k[l]; indices are local to the tensor and the outputs of tensor l start at
 * sum_{j<l} k[j].  Each tensor is one independent call of oracle_compress.
 */
int oracle_compress_batched(const float *grad, float *residual,
                            const int64_t *offsets, const int64_t *k,
                            int32_t T, float lr, int backend,
                            int32_t *out_idx, float *out_val)
{
    if (T < 1 || !offsets || !k || offsets[0] != 0) return ORACLE_EINVAL;
    int64_t base = 0;
    for (int32_t l = 0; l < T; ++l) {
        int64_t nl = offsets[l + 1] - offsets[l];
        if (nl < 0 || k[l] < 0 || k[l] > nl) return ORACLE_EINVAL;
        int rc = oracle_compress(grad + offsets[l], residual + offsets[l], nl,
                                 lr, k[l], backend, out_idx + base,
                                 out_val + base);
        if (rc != ORACLE_OK) return rc;
        base += k[l];
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * gTop-k merge.
 * (A Distributed Synchronous SGD Algorithm with Global Top-k Sparsification,
 * ABSTRACT: the global top-k largest absolute values from P workers instead
 * of all local top-k; method section: a tournament over P workers in
 * O(log P) rounds.)
 *
 * Round r = 0, 1, ... while 2^r < P: for every i that is a multiple of
 * 2^(r+1) with i + 2^r < P,
 *     S_i <- top-min(k, |U|) of U = S_i (+) S_{i+2^r}
 * where (+) is the union of the two index sets with value a + b at a common
 * index and the single value elsewhere.  The union is formed on a dense
 * vector of length n with a presence flag per index.  The result is the top
 * min(k, |S_0|) of S_0 in ascending index order; the return value is its
 * length (or a negative error code).
 * ---------------------------------------------------------------------- */
typedef struct {
    int64_t size;
    int32_t *idx;
    float *val;
} oset_t;

static int64_t merge_union(const oset_t *a, const oset_t *b, float *dv,
                           uint8_t *pres, int32_t *ulist)
{
    int64_t u = 0;
    for (int64_t j = 0; j < a->size; ++j) {
        int32_t i = a->idx[j];
        dv[i] = a->val[j];
        pres[i] = 1;
        ulist[u++] = i;
    }
    for (int64_t j = 0; j < b->size; ++j) {
        int32_t i = b->idx[j];
        if (pres[i]) {
#if ORACLE_MUTANT == 6
            /* mistake: the partner's value at a common index is dropped */
            (void)0;
#else
            dv[i] = dv[i] + b->val[j];
#endif
        } else {
            dv[i] = b->val[j];
            pres[i] = 1;
            ulist[u++] = i;
        }
    }
    return u;
}

/* Replace s by the top-min(k, u) of the union list, ascending index. */
static int keep_topk(oset_t *s, const int32_t *ulist, int64_t u, int64_t k,
                     float *dv, uint8_t *pres, float *tmpv, uint32_t *chosen)
{
    int64_t m = k < u ? k : u;
    for (int64_t j = 0; j < u; ++j) tmpv[j] = dv[ulist[j]];
    int rc = select_topk(tmpv, ulist, u, m, 0, chosen);
    if (rc != ORACLE_OK) return rc;
    for (int64_t j = 0; j < m; ++j) {
        s->idx[j] = (int32_t)chosen[j];
        s->val[j] = dv[chosen[j]];
    }
    s->size = m;
    for (int64_t j = 0; j < u; ++j) pres[ulist[j]] = 0;
    return ORACLE_OK;
}

int64_t oracle_gtopk_merge(const int32_t *in_idx, const float *in_val,
                           int32_t P, int64_t k_in, int64_t k, int64_t n,
                           int32_t *out_idx, float *out_val)
{
    if (P < 1 || k_in < 0 || k < 0 || n < 0 || k_in > n || n > 2147483647LL)
        return ORACLE_EINVAL;
    if (k_in > 0 && (!in_idx || !in_val)) return ORACLE_EINVAL;
    if (k > 0 && (!out_idx || !out_val)) return ORACLE_EINVAL;
    for (int32_t p = 0; p < P; ++p)
        for (int64_t j = 0; j < k_in; ++j) {
            int32_t i = in_idx[(int64_t)p * k_in + j];
            if (i < 0 || (int64_t)i >= n) return ORACLE_EINVAL;
            if (j > 0 && in_idx[(int64_t)p * k_in + j - 1] >= i) return ORACLE_EINVAL;
        }

    int64_t cap = k_in > k ? k_in : k;
    int64_t ucap = 2 * cap + 1;
    oset_t *S = (oset_t *)calloc((size_t)P, sizeof(oset_t));
    float *dv = (float *)calloc((size_t)(n > 0 ? n : 1), sizeof(float));
    uint8_t *pres = (uint8_t *)calloc((size_t)(n > 0 ? n : 1), 1);
    int32_t *ulist = (int32_t *)malloc((size_t)ucap * sizeof(int32_t));
    float *tmpv = (float *)malloc((size_t)ucap * sizeof(float));
    uint32_t *chosen = (uint32_t *)malloc((size_t)ucap * sizeof(uint32_t));
    int64_t result = ORACLE_ENOMEM;
    if (!S || !dv || !pres || !ulist || !tmpv || !chosen) goto done;
    for (int32_t p = 0; p < P; ++p) {
        S[p].idx = (int32_t *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(int32_t));
        S[p].val = (float *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(float));
        if (!S[p].idx || !S[p].val) goto done;
        S[p].size = k_in;
        if (k_in > 0) {
            memcpy(S[p].idx, in_idx + (int64_t)p * k_in, (size_t)k_in * sizeof(int32_t));
            memcpy(S[p].val, in_val + (int64_t)p * k_in, (size_t)k_in * sizeof(float));
        }
    }

    for (int64_t step = 1; step < P; step *= 2) {
        for (int64_t i = 0; i + step < P; i += 2 * step) {
#if ORACLE_MUTANT == 7
            /* mistake: the partner index ignores the round */
            int64_t j = i + 1;
#else
            int64_t j = i + step;
#endif
            int64_t u = merge_union(&S[i], &S[j], dv, pres, ulist);
            int rc = keep_topk(&S[i], ulist, u, k, dv, pres, tmpv, chosen);
            if (rc != ORACLE_OK) { result = rc; goto done; }
        }
    }

    {
        /* result: top-min(k, |S_0|) of worker 0's set */
        oset_t empty = {0, NULL, NULL};
        int64_t u = merge_union(&S[0], &empty, dv, pres, ulist);
        int rc = keep_topk(&S[0], ulist, u, k, dv, pres, tmpv, chosen);
        if (rc != ORACLE_OK) { result = rc; goto done; }
        for (int64_t j = 0; j < S[0].size; ++j) {
            out_idx[j] = S[0].idx[j];
            out_val[j] = S[0].val[j];
        }
        result = S[0].size;
    }

done:
    if (S) {
        for (int32_t p = 0; p < P; ++p) { free(S[p].idx); free(S[p].val); }
        free(S);
    }
    free(dv);
    free(pres);
    free(ulist);
    free(tmpv);
    free(chosen);
    return result;
}

/* ------------------------------------------------------------------------
 * Hard-threshold sparsifier with error feedback.
 * ("Rethinking gradient sparsification as total error minimization",
 * abstract in the arxivdaily listing: the variant of Top-k in which k is set
 * by a constant hard threshold, used under error feedback.)
 *
 *   acc          = fmaf(lr, grad, residual)
 *   P            = { i : key(acc[i]) >= key(threshold) }   (|acc| at least |threshold|)
 *   S            = the first min(|P|, max_out) members of P, ascending index
 *   out          = (i, acc[i]) for i in S
 *   residual[i]  = +0.0f for i in S, acc[i] otherwise
 * Returns |P| (which may exceed max_out), or a negative error code.
 * ---------------------------------------------------------------------- */
int64_t oracle_threshold(const float *grad, float *residual, int64_t n,
                         float lr, float threshold, int64_t max_out,
                         int32_t *out_idx, float *out_val)
{
    if (n < 0 || max_out < 0 || n > 2147483647LL) return ORACLE_EINVAL;
    if (n > 0 && (!grad || !residual)) return ORACLE_EINVAL;
    if (max_out > 0 && (!out_idx || !out_val)) return ORACLE_EINVAL;
    if (n == 0) return 0;
    float *acc = (float *)malloc((size_t)n * sizeof(float));
    if (!acc) return ORACLE_ENOMEM;
    oracle_accumulate(grad, residual, n, lr, acc);
    const uint32_t t = key_of(threshold);
    int64_t passed = 0;
    for (int64_t i = 0; i < n; ++i) {
        residual[i] = acc[i];
#if ORACLE_MUTANT == 10
        /* mistake: strictly above the threshold */
        int in = key_of(acc[i]) > t;
#else
        int in = key_of(acc[i]) >= t;
#endif
        if (!in) continue;
        if (passed < max_out) {
            out_idx[passed] = (int32_t)i;
            out_val[passed] = acc[i];
            residual[i] = 0.0f;
        }
        ++passed;
    }
    free(acc);
    return passed;
}

/* ------------------------------------------------------------------------
 * gTop-k residual return.
 * (Error feedback, "Sparsified SGD with Memory" and "The Convergence of
 * Sparsified Gradient Methods", abstracts: what is not transmitted stays in
 * local memory; "A Distributed Synchronous SGD Algorithm with Global Top-k
 * Sparsification", ABSTRACT: only the global top-k of the P workers' values
 * updates the model.)  A value that worker p sent but whose index is not in
 * the global set was not transmitted in effect, so it goes back to p's
 * memory:
 *     for p, j:  i = sent_idx[p][j];  if i is not in global_idx[0..k_global):
 *                    residual[p][i] = residual[p][i] + sent_val[p][j]
 * (one fp32 add).  residual is [P][n].  Rows of sent_idx ascend strictly.
 * ---------------------------------------------------------------------- */
int oracle_residual_return(const int32_t *sent_idx, const float *sent_val,
                           int32_t P, int64_t k_sent,
                           const int32_t *global_idx, int64_t k_global,
                           float *residual, int64_t n)
{
    if (P < 1 || k_sent < 0 || k_global < 0 || n < 0 || n > 2147483647LL)
        return ORACLE_EINVAL;
    if ((k_sent > 0 && (!sent_idx || !sent_val)) || (k_global > 0 && !global_idx))
        return ORACLE_EINVAL;
    if (n > 0 && !residual) return ORACLE_EINVAL;
    uint8_t *in_global = (uint8_t *)calloc((size_t)(n > 0 ? n : 1), 1);
    if (!in_global) return ORACLE_ENOMEM;
    for (int64_t j = 0; j < k_global; ++j) {
        int32_t i = global_idx[j];
        if (i < 0 || (int64_t)i >= n) { free(in_global); return ORACLE_EINVAL; }
        in_global[i] = 1;
    }
    for (int32_t p = 0; p < P; ++p)
        for (int64_t j = 0; j < k_sent; ++j) {
            int32_t i = sent_idx[(int64_t)p * k_sent + j];
            if (i < 0 || (int64_t)i >= n) { free(in_global); return ORACLE_EINVAL; }
        }
    for (int32_t p = 0; p < P; ++p) {
        float *r = residual + (int64_t)p * n;
        for (int64_t j = 0; j < k_sent; ++j) {
            int32_t i = sent_idx[(int64_t)p * k_sent + j];
#if ORACLE_MUTANT == 11
            /* mistake: returns the values that did survive */
            if (!in_global[i]) continue;
#else
            if (in_global[i]) continue;
#endif
            r[i] = r[i] + sent_val[(int64_t)p * k_sent + j];
        }
    }
    free(in_global);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Top-k aggregation by AllGather (the O(kP) TopKAllReduce that the gTop-k
 * review compares against: "A Distributed Synchronous SGD Algorithm with
 * Global Top-k Sparsification", ABSTRACT: current methods use AllGather to
 * accumulate the sparse gradients).  Every worker receives all P local
 * top-k sets and sums them into a dense gradient, in rank order:
 *     out[i] = +0.0f for all i;  for p = 0..P-1, for each (i, v) in S_p:
 *         out[i] = out[i] + v            (one fp32 add each)
 * ---------------------------------------------------------------------- */
int oracle_allgather_sum(const int32_t *in_idx, const float *in_val,
                         int32_t P, int64_t k_in, int64_t n, float *out)
{
    if (P < 1 || k_in < 0 || n < 0 || k_in > n || n > 2147483647LL) return ORACLE_EINVAL;
    if (k_in > 0 && (!in_idx || !in_val)) return ORACLE_EINVAL;
    if (n > 0 && !out) return ORACLE_EINVAL;
    for (int32_t p = 0; p < P; ++p)
        for (int64_t j = 0; j < k_in; ++j) {
            int32_t i = in_idx[(int64_t)p * k_in + j];
            if (i < 0 || (int64_t)i >= n) return ORACLE_EINVAL;
            if (j > 0 && in_idx[(int64_t)p * k_in + j - 1] >= i) return ORACLE_EINVAL;
        }
    for (int64_t i = 0; i < n; ++i) out[i] = 0.0f;
#if ORACLE_MUTANT == 12
    /* mistake: reverse rank order */
    for (int32_t p = P - 1; p >= 0; --p)
#else
    for (int32_t p = 0; p < P; ++p)
#endif
        for (int64_t j = 0; j < k_in; ++j) {
            int32_t i = in_idx[(int64_t)p * k_in + j];
            out[i] = out[i] + in_val[(int64_t)p * k_in + j];
        }
    return ORACLE_OK;
}
