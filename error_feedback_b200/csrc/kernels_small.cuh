// The whole error-feedback step of one small tensor in one kernel ("Sparsified
// SGD with Memory", abstract: send the top k, keep the rest in memory; "A
// Distributed Synchronous SGD Algorithm with Global Top-k Sparsification",
// ABSTRACT: the k largest absolute values, the lower index first among equal
// ones).
//
// For a tensor that one wave of blocks holds in shared memory (one block per
// SM, up to SK_MAX elements each) the prefilter, the candidate records and
// the separate select kernel cost more than they save: latency, not bytes,
// bounds the step.  Each block owns a contiguous slice:
//   1  acc = fmaf(lr, grad, residual) streamed once (written back to the
//      residual, kept in shared memory) and an 8,192-bin histogram of
//      key >> 18 of every element, added into a global histogram;
//   2  after a grid-wide exchange every block finds the bin b1 of the k-th
//      key, counts its elements above b1 and lists those in b1 (block << 18 |
//      low 18 key bits) in a grid-wide entry list;
//   3  after a second exchange every block reads the list and resolves the
//      k-th key T and the tie quota q from it (bits 17..9, then 8..0), and
//      its output offset from the earlier blocks' counts and entries;
//   4  it emits its selected elements in index order from shared memory.
// A bin b1 with more elements than the entry list takes two summed digit
// passes and an exact-count exchange instead (three more grid-wide steps).
// The histograms, the entry count and the barrier counter are cleared by the
// setup kernel launched before this one.
#pragma once

#include "common.cuh"
#include "kernels_compress.cuh"
#include "kernels_select.cuh"

namespace tke {

constexpr int SK_THREADS = 512;
constexpr int SK_MAX = 16384;            // elements per block
constexpr int SK_BINS = 8192;            // digit 1: key >> 18
constexpr int SK_LOW = 18;               // bits below digit 1
constexpr int SK_D2 = SK_LOW - 9;        // digit 2: bits 17..9 (512 bins); digit 3: bits 8..0
constexpr int SK_MIN_PER_BLOCK = 2048;   // fewer blocks for smaller tensors
constexpr int SK_VEC = 8;                // float4 of each input a thread loads at once

struct SmallShared {
    float acc[SK_MAX];
    uint32_t hist[SK_BINS];
    uint64_t scan[33];
    uint32_t red[33];
    FindResult fr;
    uint32_t pre;
    int flag;
};

struct SmallParams {
    const float* grad;
    float* resid;
    int64_t n;
    float lr;
    uint32_t k;
    int32_t* out_idx;      // the tensor's outputs (out_base applied)
    float* out_val;
    Ctrl* ctrl;
    uint32_t* hist;        // [SK_BINS] global digit-1 histogram (cleared)
    uint32_t* hist2;       // [512 + 512] crowded path's digit histograms (cleared)
    uint32_t* ent;         // [ENT_PER] entry list
    uint32_t* ent_cnt;     // its length (cleared)
    Slot* slots;           // [grid] per-block counts
};

// Sum over blocks j < c of word f of their slots (warp 0), every thread gets it.
__device__ __forceinline__ uint32_t sk_slots_before(const Slot* slots, int c, int f,
                                                    SmallShared& K) {
    if (threadIdx.x < 32) {
        uint32_t s = 0;
        for (int j0 = 0; j0 < c; j0 += 256) {
            uint32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 32 * u + (int)threadIdx.x;
                v[u] = j < c ? reinterpret_cast<const uint32_t*>(slots + j)[f] : 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        s = warp_sum(s);
        if (threadIdx.x == 0) K.pre = s;
    }
    __syncthreads();
    const uint32_t r = K.pre;
    __syncthreads();
    return r;
}

// Global histogram hg (nb bins, nb a multiple of the block size) into shared
// memory, then the bin of the rem-th largest (result in K.fr).
__device__ __forceinline__ void sk_find_global(const uint32_t* hg, int nb, uint32_t rem,
                                               SmallShared& K) {
    for (int i = threadIdx.x; i < nb; i += blockDim.x) K.hist[i] = hg[i];
    __syncthreads();
    block_find_bin(K.hist, nb, rem, K.red, &K.fr);
}

// Crowded k-th-key bin: digits 17..9 and 8..0 of the elements in bin b1 by
// summed global histograms, then exact counts of every block.  Writes T, the
// tie quota and this block's counts before it to out[0..3] (shared memory).
// Returns false if a wait gave up or the counts did not add up.  Out of line.
__device__ __noinline__ bool sk_crowded(const SmallParams& p, SmallShared& K, uint32_t epoch,
                                        uint32_t m, uint32_t b1, uint32_t rem, uint32_t* out) {
    const int tid = threadIdx.x, c = blockIdx.x;
    uint32_t* status = &p.ctrl->status;
    if (c == 0 && tid == 0) p.ctrl->r2_path = 1;
    // digit 2: bits 17..9 of the elements in b1
    for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        if ((key >> SK_LOW) == b1) atomicAdd(&K.hist[(key >> 9) & 511u], 1u);
    }
    __syncthreads();
    for (int i = tid; i < 512; i += SK_THREADS)
        if (K.hist[i]) atomicAdd(&p.hist2[i], K.hist[i]);
    if (!grid_barrier(&p.ctrl->bar, epoch, status, &K.flag)) return false;
    sk_find_global(p.hist2, 512, rem, K);
    if (!K.fr.ok) return false;
    const uint32_t t1 = K.fr.bin;
    const uint32_t rem2 = rem - K.fr.above;
    const uint32_t pre = (b1 << SK_D2) | t1;          // key >> 9 of the class
    __syncthreads();
    // digit 3: bits 8..0 of the elements in that class
    for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        if ((key >> 9) == pre) atomicAdd(&K.hist[key & 511u], 1u);
    }
    __syncthreads();
    for (int i = tid; i < 512; i += SK_THREADS)
        if (K.hist[i]) atomicAdd(&p.hist2[512 + i], K.hist[i]);
    if (!grid_barrier(&p.ctrl->bar, epoch, status, &K.flag)) return false;
    sk_find_global(p.hist2 + 512, 512, rem2, K);
    if (!K.fr.ok) return false;
    const uint32_t Tk = (pre << 9) | K.fr.bin;
    const uint32_t q = rem2 - K.fr.above;
    __syncthreads();
    uint32_t g = 0, e = 0;
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        g += key > Tk;
        e += key == Tk;
    }
    const uint64_t both = block_sum(((uint64_t)g << 32) | e, K.scan);
    if (tid == 0) {
        p.slots[c].gt_last = (uint32_t)(both >> 32);
        p.slots[c].eq_last = (uint32_t)both;
    }
    if (!grid_barrier(&p.ctrl->bar, epoch, status, &K.flag)) return false;
    const uint32_t bg = sk_slots_before(p.slots, c, 4, K);
    const uint32_t be = sk_slots_before(p.slots, c, 5, K);
    if (tid == 0) {
        out[0] = Tk;
        out[1] = q;
        out[2] = bg;
        out[3] = be;
    }
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(SK_THREADS, 1)
small_kernel(const __grid_constant__ SmallParams p) {
    extern __shared__ __align__(16) unsigned char sk_smem[];
    SmallShared& K = *reinterpret_cast<SmallShared*>(sk_smem);
    __shared__ uint32_t s_out[4];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    Ctrl* ctrl = p.ctrl;
    uint32_t* status = &ctrl->status;
    const int tid = threadIdx.x, c = blockIdx.x, G = gridDim.x;
    mark_phase(ctrl, 0);
    const BlockSpan block_span(ctrl);
    uint32_t epoch = 0;
    const uint32_t stall = ctrl->stall;
    const uint32_t k = p.k;
    // this block's slice [e0, e0 + m), a multiple of 4 elements long
    int64_t per = (p.n + G - 1) / G;
    per = (per + 3) & ~(int64_t)3;
    const int64_t e0 = min((int64_t)c * per, p.n);
    const uint32_t m = (uint32_t)(min(e0 + per, p.n) - e0);
    for (int i = tid; i < SK_BINS; i += SK_THREADS) K.hist[i] = 0;
    __syncthreads();

    // ---- 1: accumulate, keep, histogram
    const float* gp = p.grad + e0;
    float* rp = p.resid + e0;
    const float lr = p.lr;
    const bool vec = ((reinterpret_cast<uintptr_t>(gp) | reinterpret_cast<uintptr_t>(rp)) & 15u) == 0;
    if (vec) {
        // up to SK_VEC float4 of each input per thread in flight at once
        const uint32_t m4 = m >> 2;
        for (uint32_t b = 0; b < m4; b += SK_THREADS * SK_VEC) {
            float4 g[SK_VEC], r[SK_VEC];
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i < m4) {
                    g[u] = ld_stream(reinterpret_cast<const float4*>(gp) + i);
                    r[u] = ld_stream(reinterpret_cast<const float4*>(rp) + i);
                }
            }
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i >= m4) continue;
                float4 a;
                a.x = __fmaf_rn(lr, g[u].x, r[u].x);
                a.y = __fmaf_rn(lr, g[u].y, r[u].y);
                a.z = __fmaf_rn(lr, g[u].z, r[u].z);
                a.w = __fmaf_rn(lr, g[u].w, r[u].w);
                st_stream(reinterpret_cast<float4*>(rp) + i, a);
                reinterpret_cast<float4*>(K.acc)[i] = a;
                atomicAdd(&K.hist[key_of(a.x) >> SK_LOW], 1u);
                atomicAdd(&K.hist[key_of(a.y) >> SK_LOW], 1u);
                atomicAdd(&K.hist[key_of(a.z) >> SK_LOW], 1u);
                atomicAdd(&K.hist[key_of(a.w) >> SK_LOW], 1u);
            }
        }
        for (uint32_t i = 4 * m4 + tid; i < m; i += SK_THREADS) {
            const float a = __fmaf_rn(lr, __ldcs(gp + i), __ldcs(rp + i));
            __stcs(rp + i, a);
            K.acc[i] = a;
            atomicAdd(&K.hist[key_of(a) >> SK_LOW], 1u);
        }
    } else {
        for (uint32_t b = 0; b < m; b += SK_THREADS * SK_VEC) {
            float g[SK_VEC], r[SK_VEC];
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i < m) {
                    g[u] = __ldcs(gp + i);
                    r[u] = __ldcs(rp + i);
                }
            }
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i >= m) continue;
                const float a = __fmaf_rn(lr, g[u], r[u]);
                __stcs(rp + i, a);
                K.acc[i] = a;
                atomicAdd(&K.hist[key_of(a) >> SK_LOW], 1u);
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < SK_BINS; i += SK_THREADS)
        if (K.hist[i]) atomicAdd(&p.hist[i], K.hist[i]);
    mark_phase(ctrl, 1);
    if (!grid_barrier(&ctrl->bar, epoch, status, &K.flag, stall)) return;
    mark_phase(ctrl, 2);

    // ---- 2: the k-th key's bin; elements above it, the entry list
    {
        const uint4* h4 = reinterpret_cast<const uint4*>(p.hist);
        uint4* s4 = reinterpret_cast<uint4*>(K.hist);
        for (int i = tid; i < SK_BINS / 4; i += SK_THREADS) s4[i] = h4[i];
    }
    __syncthreads();
    block_find_bin(K.hist, SK_BINS, k, K.red, &K.fr);
    if (!K.fr.ok) {
        if (tid == 0) atomicOr(status, ST_INCONSISTENT);
        return;
    }
    const uint32_t b1 = K.fr.bin;
    const uint32_t rem = k - K.fr.above;
    if (c == 0 && tid == 0) {
        ctrl->mode = 0;
        ctrl->cand_total = (uint64_t)p.n;
    }
    // count first, reserve the block's entries with one atomic (its latency
    // overlapping the block sum of the counts above b1), then list them
    uint32_t gt_b = 0, in_t = 0;
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t d = key_of(K.acc[i]) >> SK_LOW;
        gt_b += d > b1;
        in_t += d == b1;
    }
    {
        uint64_t tot;
        const uint64_t ex = block_excl_scan(((uint64_t)gt_b << 32) | in_t, K.scan, &tot);
        const uint32_t in_b = (uint32_t)tot;
        if (tid == 0) {
            p.slots[c].gt_first = (uint32_t)(tot >> 32);
            K.pre = in_b ? atomicAdd(p.ent_cnt, in_b) : 0u;
        }
        __syncthreads();
        uint32_t at = (uint32_t)ex + K.pre;
        if (in_t) {
            for (uint32_t i = tid; i < m; i += SK_THREADS) {
                const uint32_t key = key_of(K.acc[i]);
                if ((key >> SK_LOW) == b1) {
                    if (at < ENT_PER) p.ent[at] = ((uint32_t)c << SK_LOW) | (key & ((1u << SK_LOW) - 1u));
                    ++at;
                }
            }
        }
    }
    if (!grid_barrier(&ctrl->bar, epoch, status, &K.flag)) return;
    mark_phase(ctrl, 4);

    // ---- 3: T, the tie quota and this block's output offset
    constexpr int EPT = (int)ENT_PER / SK_THREADS;
    uint32_t ev[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) ev[u] = p.ent[tid + u * SK_THREADS];
    const uint32_t E = *reinterpret_cast<const volatile uint32_t*>(p.ent_cnt);
    uint32_t Tk, q, before_gt, before_eq;
    if (E <= ENT_PER) {
        const uint32_t gts = sk_slots_before(p.slots, c, 2, K);
#pragma unroll
        for (int u = 0; u < EPT; ++u)
            if ((uint32_t)(tid + u * SK_THREADS) >= E) ev[u] = DEAD;
        // bits 17..9
        for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < EPT; ++u)
            if (ev[u] != DEAD) atomicAdd(&K.hist[(ev[u] >> 9) & 511u], 1u);
        __syncthreads();
        block_find_bin(K.hist, 512, rem, K.red, &K.fr);
        const bool ok1 = K.fr.ok;
        const uint32_t t1 = K.fr.bin;
        const uint32_t rem2 = rem - K.fr.above;
        __syncthreads();
        // bits 8..0 inside that class
        for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < EPT; ++u)
            if (ev[u] != DEAD && ((ev[u] >> 9) & 511u) == t1) atomicAdd(&K.hist[ev[u] & 511u], 1u);
        __syncthreads();
        block_find_bin(K.hist, 512, rem2, K.red, &K.fr);
        if (!ok1 || !K.fr.ok) {
            if (tid == 0) atomicOr(status, ST_INCONSISTENT);
            return;
        }
        const uint32_t low = (t1 << 9) | K.fr.bin;
        Tk = (b1 << SK_LOW) | low;
        q = rem2 - K.fr.above;
        uint32_t g = 0, e = 0;
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            if (ev[u] != DEAD && (int)(ev[u] >> SK_LOW) < c) {
                const uint32_t v = ev[u] & ((1u << SK_LOW) - 1u);
                g += v > low;
                e += v == low;
            }
        }
        const uint64_t both = block_sum(((uint64_t)g << 32) | e, K.scan);
        before_gt = gts + (uint32_t)(both >> 32);
        before_eq = (uint32_t)both;
    } else {
        if (!sk_crowded(p, K, epoch, m, b1, rem, s_out)) {
            if (tid == 0 && (*reinterpret_cast<volatile uint32_t*>(status) & ST_TIMEOUT) == 0)
                atomicOr(status, ST_INCONSISTENT);
            return;
        }
        Tk = s_out[0];
        q = s_out[1];
        before_gt = s_out[2];
        before_eq = s_out[3];
    }
    mark_phase(ctrl, 6);

    // ---- 4: emission in index order; thread t owns a contiguous run
    const uint32_t run = (m + SK_THREADS - 1) / SK_THREADS;
    const uint32_t i0 = min((uint32_t)tid * run, m), i1 = min(i0 + run, m);
    uint32_t g = 0, e = 0;
    for (uint32_t i = i0; i < i1; ++i) {
        const uint32_t key = key_of(K.acc[i]);
        g += key > Tk;
        e += key == Tk;
    }
    uint64_t tot;
    const uint64_t ex = block_excl_scan(((uint64_t)g << 32) | e, K.scan, &tot);
    uint32_t rg = before_gt + (uint32_t)(ex >> 32), re = before_eq + (uint32_t)ex;
    for (uint32_t i = i0; i < i1; ++i) {
        const float a = K.acc[i];
        const uint32_t key = key_of(a);
        uint32_t rank = 0xFFFFFFFFu;
        if (key > Tk) {
            rank = rg + (re < q ? re : q);
            ++rg;
        } else if (key == Tk) {
            if (re < q) rank = rg + re;
            ++re;
        }
        if (rank < k) {
            p.out_idx[rank] = (int32_t)(e0 + i);
            p.out_val[rank] = a;
            p.resid[e0 + i] = 0.0f;
        }
    }
    mark_phase(ctrl, 7);
}

}  // namespace tke
