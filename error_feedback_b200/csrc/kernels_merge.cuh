// gTop-k merge kernels ("A Distributed Synchronous SGD Algorithm with Global
// Top-k Sparsification for Low Bandwidth Networks", ABSTRACT and method
// section: the global top-k of P workers found by a tournament in O(log P)
// rounds).  In round r worker i (a multiple of 2^(r+1), with i + 2^r < P)
// absorbs worker i + 2^r: the two index-sorted lists are merged (merge path),
// values at a common index are added once in fp32, and the select kernel then
// keeps the top k of the merged list.  The P workers are P buffers on one
// GPU, so a round is a pair of kernels instead of a network exchange.
#pragma once

#include "common.cuh"

namespace tke {

constexpr int MG_THREADS = 512;
constexpr int MG_PER_THREAD = 4;
constexpr int MG_D = MG_THREADS * MG_PER_THREAD;   // merged positions per block
constexpr int MZ_THREADS = 512;
constexpr int MZ_LOADS = 12;                       // index loads in flight per thread

struct MergeSetupParams {
    const int32_t* in_idx;
    const float* in_val;
    int32_t P;
    int64_t k_in;
    int64_t n;
    Ctrl* ctrl;
    uint32_t kernels;
    uint4* zero_ptr;
    uint64_t zero_vec4;
    uint32_t* bad_words;    // [validate_blocks], one verdict per block
    uint32_t* sizes;        // [P]
    uint32_t* floors;       // [P] lower key bound of each set (0: none known)
    uint32_t* set_idx;      // [P][set_cap]
    float* set_val;
    int64_t set_cap;
    int32_t lonely;         // worker copied into the sets buffer (or -1)
    uint32_t validate_blocks;
};

// Blocks [0, validate_blocks) check the input rows (strictly ascending,
// inside [0, n)) and each write its verdict to its own word; the first select
// launch folds the verdicts into the status word.  The other blocks reset the
// control block, clear this call's counters and histograms, and copy the set
// of the worker that has no partner in round 0.
__global__ void __launch_bounds__(MZ_THREADS)
merge_setup_kernel(const MergeSetupParams p) {
    const int b = blockIdx.x, tid = threadIdx.x;
    // this grid waits for the kernel before it on the stream.  The first
    // round may be scheduled once every block of this grid has finished its
    // work (each triggers at its end), not from the start: scheduled while
    // these blocks still hold the SMs, its clusters are placed piecemeal
    // and no longer fit in one wave (measured on the 32-worker tournament:
    // 149 against 124 us per call)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if ((uint32_t)b < p.validate_blocks) {
        // a contiguous range of the P * k_in entries per block; each thread's
        // position inside its row is carried along (no division per entry),
        // and MZ_LOADS entries and their successors are loaded at once (one
        // round trip for the 32-worker tournament's 11 entries per thread)
        const int64_t tot = (int64_t)p.P * p.k_in;
        const int64_t per = (tot + p.validate_blocks - 1) / p.validate_blocks;
        const int64_t e0 = min((int64_t)b * per, tot), e1 = min(e0 + per, tot);
        bool bad = false;
        int64_t e = e0 + tid;
        int64_t j = e % p.k_in;                  // position of entry e in its row
        const int64_t step = (int64_t)blockDim.x;
        const int64_t jstep = step % p.k_in;
        while (e < e1) {
            int32_t v[MZ_LOADS], w[MZ_LOADS];
            bool last[MZ_LOADS];
            int64_t ee = e, jj = j;
#pragma unroll
            for (int u = 0; u < MZ_LOADS; ++u) {
                last[u] = jj + 1 >= p.k_in;      // no successor in the row
                v[u] = ee < e1 ? p.in_idx[ee] : 0;
                w[u] = (ee < e1 && !last[u]) ? p.in_idx[ee + 1] : 0;
                ee += step;
                jj += jstep;
                if (jj >= p.k_in) jj -= p.k_in;
            }
#pragma unroll
            for (int u = 0; u < MZ_LOADS; ++u) {
                if (e + u * step >= e1) break;
                if (v[u] < 0 || (int64_t)v[u] >= p.n) bad = true;
                if (!last[u] && w[u] <= v[u]) bad = true;
            }
            e = ee;
            j = jj;
        }
        const int any = __syncthreads_or(bad);
        if (tid == 0) p.bad_words[b] = any ? 1u : 0u;
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        return;
    }
    const int zb = b - (int)p.validate_blocks;
    const int nz = gridDim.x - (int)p.validate_blocks;
    if (zb == 0) {
        if (tid == 0) {
            Ctrl c;
            memset(&c, 0, sizeof(c));
            c.kernels = p.kernels;
            *p.ctrl = c;
        }
        for (int i = tid; i < p.P; i += blockDim.x) {
            p.sizes[i] = (uint32_t)p.k_in;
            p.floors[i] = 0;
        }
        if (p.lonely >= 0) {
            const int64_t src = (int64_t)p.lonely * p.k_in;
            const int64_t dst = (int64_t)p.lonely * p.set_cap;
            for (int64_t j = tid; j < p.k_in; j += blockDim.x) {
                p.set_idx[dst + j] = (uint32_t)p.in_idx[src + j];
                p.set_val[dst + j] = p.in_val[src + j];
            }
        }
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (uint64_t i = (uint64_t)zb * blockDim.x + tid; i < p.zero_vec4;
         i += (uint64_t)nz * blockDim.x)
        p.zero_ptr[i] = z;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

struct MergeRoundParams {
    const uint32_t* src_idx;    // sets of this round (row stride src_stride)
    const float* src_val;
    int64_t src_stride;
    const uint32_t* sizes;      // null: every set has size_const entries
    uint32_t size_const;
    int32_t np;                 // pairs
    int32_t step;               // 2^r
    int64_t mcap;               // merged positions per pair
    uint32_t* m_idx;            // [np][mcap]
    float* m_val;
    uint32_t* hist;             // pair p: digit-1 histogram at p * MHIST_WORDS
    uint32_t* live;             // [np]
};

// Number of A elements among the first d of the merge of A (a) and B (b),
// equal indices taking A first.  One full warp, 32 probes per step.
__device__ __forceinline__ int64_t warp_merge_path(const uint32_t* A, int64_t a,
                                                   const uint32_t* B, int64_t b, int64_t d) {
    const uint32_t lane = lane_id();
    int64_t lo = d - b > 0 ? d - b : 0;
    int64_t hi = d < a ? d : a;
    // f(i) = A[i-1] <= B[d-i] for i in (lo, hi]; true then false
    while (hi > lo) {
        const int64_t span = hi - lo;
        const int64_t stride = (span + 31) / 32;
        const int64_t i = lo + (int64_t)(lane + 1) * stride;
        bool f = false;
        if (i <= hi) f = A[i - 1] <= B[d - i];
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, f);
        const uint32_t cnt = (m == 0xFFFFFFFFu) ? 32u : (uint32_t)(__ffs(~m) - 1);
        const int64_t nlo = lo + (int64_t)cnt * stride;
        const int64_t nhi = lo + (int64_t)(cnt + 1) * stride - 1;
        lo = nlo;
        hi = nhi < hi ? nhi : hi;
        if (stride == 1) break;
    }
    return lo;
}

// Same search inside shared memory, by one thread.
__device__ __forceinline__ int local_merge_path(const uint32_t* A, int a, const uint32_t* B,
                                                int b, int d) {
    int lo = d - b > 0 ? d - b : 0;
    int hi = d < a ? d : a;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (A[mid - 1] <= B[d - mid]) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Round kernel: block (c, pair) writes merged positions [c*MG_D, (c+1)*MG_D)
// of its pair.  A common index appears once (A's slot holds a + b, B's slot
// is DEAD); slots past a + b are DEAD.  Also counts live entries and builds
// the digit-1 histogram of their keys.
__global__ void __launch_bounds__(MG_THREADS)
merge_round_kernel(const MergeRoundParams p) {
    __shared__ uint32_t sAi[MG_D + 1], sBi[MG_D + 1];
    __shared__ float sAv[MG_D + 1], sBv[MG_D + 1];
    __shared__ uint32_t s_h1[D1_BINS];
    __shared__ int64_t s_part[2];
    __shared__ uint32_t s_red[33];

    const int tid = threadIdx.x;
    const int pair = blockIdx.y;
    const int64_t c = blockIdx.x;
    const int64_t left = (int64_t)pair * 2 * p.step;
    const int64_t right = left + p.step;
    int64_t a = p.sizes ? p.sizes[left] : p.size_const;
    int64_t b = p.sizes ? p.sizes[right] : p.size_const;
    a = a < p.src_stride ? a : p.src_stride;
    b = b < p.src_stride ? b : p.src_stride;
    const uint32_t* Ai = p.src_idx + left * p.src_stride;
    const uint32_t* Bi = p.src_idx + right * p.src_stride;
    const float* Av = p.src_val + left * p.src_stride;
    const float* Bv = p.src_val + right * p.src_stride;
    uint32_t* Mi = p.m_idx + (int64_t)pair * p.mcap;
    float* Mv = p.m_val + (int64_t)pair * p.mcap;

    const int64_t d0 = c * MG_D;
    const int64_t dend = min(d0 + (int64_t)MG_D, p.mcap);
    const int64_t ab = min(a + b, p.mcap);
    if (d0 >= ab) {
        for (int64_t d = d0 + tid; d < dend; d += blockDim.x) {
            Mi[d] = DEAD;
            Mv[d] = 0.f;
        }
        return;
    }
    const int64_t d1 = min(d0 + (int64_t)MG_D, ab);
    if (tid < 64) {
        const int64_t dd = tid < 32 ? d0 : d1;
        const int64_t i = warp_merge_path(Ai, a, Bi, b, dd);
        if ((tid & 31) == 0) s_part[tid >> 5] = i;
    }
    for (int i = tid; i < D1_BINS; i += blockDim.x) s_h1[i] = 0;
    __syncthreads();
    const int64_t i0 = s_part[0], i1 = max(s_part[1], i0);
    const int64_t j0 = d0 - i0, j1 = max(d1 - s_part[1], j0);
    const int la = (int)min(i1 - i0, (int64_t)MG_D);
    const int lb = (int)min(j1 - j0, (int64_t)MG_D);
    // sA[x] = A[i0 - 1 + x] for x in [0, la]; sB[y] = B[j0 + y] for y in [0, lb]
    for (int x = tid; x <= la; x += blockDim.x) {
        const int64_t gi = i0 - 1 + x;
        const bool in = gi >= 0 && gi < a;
        sAi[x] = in ? Ai[gi] : DEAD;
        sAv[x] = in ? Av[gi] : 0.f;
    }
    for (int y = tid; y <= lb; y += blockDim.x) {
        const int64_t gj = j0 + y;
        const bool in = gj < b;
        sBi[y] = in ? Bi[gj] : DEAD;
        sBv[y] = in ? Bv[gj] : 0.f;
    }
    __syncthreads();

    const int span = (int)(d1 - d0);
    uint32_t live = 0;
    const int dl = tid * MG_PER_THREAD;
    // every lane runs the same MG_PER_THREAD steps (the histogram update is
    // aggregated across the warp); lanes past the span do nothing
    int ia = 0, ib = 0;
    if (dl < span) {
        ia = local_merge_path(sAi + 1, la, sBi, lb, dl);
        ib = dl - ia;
    }
#pragma unroll
    for (int u = 0; u < MG_PER_THREAD; ++u) {
        const int pos = dl + u;
        const bool valid = pos < span;
        uint32_t oi = DEAD;
        float ov = 0.f;
        if (valid) {
            const int64_t d = d0 + pos;
            const bool takeA = ia < la && (ib >= lb || sAi[1 + ia] <= sBi[ib]);
            if (takeA) {
                oi = sAi[1 + ia];
                ov = sAv[1 + ia];
                // partner: the next B element, B[d - i] with i = i0 + ia
                const int64_t jB = d - (i0 + ia);
                if (jB < b) {
                    const int64_t y = jB - j0;
                    if (y >= 0 && y <= lb && sBi[y] == oi) ov = __fadd_rn(ov, sBv[y]);
                }
                ++ia;
            } else {
                oi = ib < lb ? sBi[ib] : DEAD;
                ov = ib < lb ? sBv[ib] : 0.f;
                // the previous A element, A[iA - 1] with iA = d - j
                const int64_t iA = d - (j0 + ib);
                if (iA > 0) {
                    const int64_t x = iA - i0;   // sA[x] = A[iA - 1]
                    if (x >= 0 && x <= la && sAi[x] == oi) oi = DEAD;
                }
                ++ib;
            }
            Mi[d] = oi;
            Mv[d] = oi == DEAD ? 0.f : ov;
            if (oi != DEAD) ++live;
        }
        if (valid && oi != DEAD) atomicAdd(&s_h1[key_of(ov) >> 20], 1u);
    }
    // the block that ends the merged list clears the tail of the segment
    if (d1 == ab)
        for (int64_t d = d1 + tid; d < dend; d += blockDim.x) {
            Mi[d] = DEAD;
            Mv[d] = 0.f;
        }
    const uint32_t tl = block_sum(live, s_red);
    if (tid == 0 && tl) atomicAdd(&p.live[pair], tl);
    uint32_t* h = p.hist + (size_t)pair * MHIST_WORDS + MH_D1;
    for (int i = tid; i < D1_BINS; i += blockDim.x)
        if (s_h1[i]) atomicAdd(&h[i], s_h1[i]);
}

}  // namespace tke
