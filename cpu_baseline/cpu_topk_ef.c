/*
 * Multi-threaded CPU Top-k + error-feedback step: the host-core baseline the
 * GPU path is reported beside.  It computes what the library computes ("Sparsified
 * SGD with Memory", abstract: send the top-k entries and keep the rest in
 * memory; "A Distributed Synchronous SGD Algorithm with Global Top-k
 * Sparsification", ABSTRACT: the k largest absolute values):
 *     acc[i] = fmaf(lr, grad[i], residual[i])      one fp32 rounding
 *     the k indices of largest |acc| (ties to the lower index), ascending,
 *     with their acc; residual = acc with those slots +0.0f
 * but organised for speed on many cores: each OpenMP thread accumulates its
 * contiguous share and keeps the k best entries of that share in a bounded
 * max-heap of 64-bit rank words, (0x7FFFFFFF - key) << 32 | index, where a
 * smaller word ranks higher (key = |x| bits, every NaN 0x7FFFFFFF); the
 * threads' heaps are then merged by a quickselect of the k smallest words
 * and the winners sorted by index.
 *
 * Not the oracle and not test infrastructure: built with gcc -fopenmp,
 * timed by bench.py, and checked against the oracle by a CPU test.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline uint32_t mag_key(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    u &= 0x7FFFFFFFu;
    return u > 0x7F800000u ? 0x7FFFFFFFu : u;
}

static inline uint64_t rank_word(float a, uint32_t i)
{
    return ((uint64_t)(0x7FFFFFFFu - mag_key(a)) << 32) | i;
}

/* bounded max-heap of rank words */
static inline void sift_down(uint64_t *h, int64_t m, int64_t i)
{
    const uint64_t v = h[i];
    for (;;) {
        int64_t c = 2 * i + 1;
        if (c >= m) break;
        if (c + 1 < m && h[c + 1] > h[c]) ++c;
        if (h[c] <= v) break;
        h[i] = h[c];
        i = c;
    }
    h[i] = v;
}

static inline void sift_up(uint64_t *h, int64_t i)
{
    const uint64_t v = h[i];
    while (i > 0) {
        const int64_t p = (i - 1) / 2;
        if (h[p] >= v) break;
        h[i] = h[p];
        i = p;
    }
    h[i] = v;
}

/* move the k smallest of a[0..m) to a[0..k) (any order) */
static void select_smallest(uint64_t *a, int64_t m, int64_t k)
{
    int64_t lo = 0, hi = m - 1;
    uint64_t seed = 0x2545F4914F6CDD1Dull;
    while (lo < hi) {
        seed ^= seed << 13; seed ^= seed >> 7; seed ^= seed << 17;
        const uint64_t pv = a[lo + (int64_t)(seed % (uint64_t)(hi - lo + 1))];
        int64_t i = lo, j = hi;
        while (i <= j) {
            while (a[i] < pv) ++i;
            while (a[j] > pv) --j;
            if (i <= j) {
                const uint64_t t = a[i]; a[i] = a[j]; a[j] = t;
                ++i; --j;
            }
        }
        if (k - 1 <= j) hi = j;
        else if (k - 1 >= i) lo = i;
        else break;
    }
}

static int cmp_low32(const void *x, const void *y)
{
    const uint32_t a = (uint32_t)*(const uint64_t *)x, b = (uint32_t)*(const uint64_t *)y;
    return (a > b) - (a < b);
}

/* Returns 0, or -1 on bad arguments / allocation failure. */
int cpu_topk_ef(const float *grad, float *residual, int64_t n, float lr, int64_t k,
                int32_t *out_idx, float *out_val, int nthreads)
{
    if (n < 0 || k < 0 || k > n || n > 2147483647LL) return -1;
    const int T = nthreads > 0 ? nthreads : omp_get_max_threads();
    if (k == 0) {
#pragma omp parallel for num_threads(T) schedule(static)
        for (int64_t i = 0; i < n; ++i) residual[i] = fmaf(lr, grad[i], residual[i]);
        return 0;
    }
    uint64_t *heaps = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)T * (size_t)k);
    int64_t *fill = (int64_t *)calloc((size_t)T, sizeof(int64_t));
    if (!heaps || !fill) {
        free(heaps);
        free(fill);
        return -1;
    }
#pragma omp parallel num_threads(T)
    {
        const int t = omp_get_thread_num();
        const int nt = omp_get_num_threads();
        const int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
        uint64_t *h = heaps + (size_t)t * (size_t)k;
        int64_t m = 0;
        for (int64_t i = lo; i < hi; ++i) {
            const float a = fmaf(lr, grad[i], residual[i]);
            residual[i] = a;
            const uint64_t w = rank_word(a, (uint32_t)i);
            if (m < k) {
                h[m] = w;
                sift_up(h, m);
                ++m;
            } else if (w < h[0]) {
                h[0] = w;
                sift_down(h, m, 0);
            }
        }
        fill[t] = m;
    }
    /* gather the heaps, keep the k smallest words, order them by index */
    int64_t m = 0;
    for (int t = 0; t < T; ++t) {
        if (m != (int64_t)t * k)
            memmove(heaps + m, heaps + (size_t)t * (size_t)k, sizeof(uint64_t) * (size_t)fill[t]);
        m += fill[t];
    }
    select_smallest(heaps, m, k);
    qsort(heaps, (size_t)k, sizeof(uint64_t), cmp_low32);
#pragma omp parallel for num_threads(T) schedule(static)
    for (int64_t j = 0; j < k; ++j) {
        const uint32_t i = (uint32_t)heaps[j];
        out_idx[j] = (int32_t)i;
        out_val[j] = residual[i];
        residual[i] = 0.0f;
    }
    free(heaps);
    free(fill);
    return 0;
}
