// Compress kernels: setup + threshold estimate, and the fused streaming pass.
//
// One error-feedback step ("Sparsified SGD with Memory" and "The Convergence
// of Sparsified Gradient Methods", abstracts in the arxivdaily listing; "A
// Distributed Synchronous SGD Algorithm with Global Top-k Sparsification",
// ABSTRACT) computes acc = fmaf(lr, grad, residual), keeps the k entries of
// largest |acc| and leaves the rest in memory.  The only pass over the full
// tensor is the streaming kernel below: it reads grad and residual once,
// writes acc back into residual, and appends every element whose key reaches
// a prefilter threshold T0 to a candidate list in index order.  The exact
// top-k is then found among the candidates (select kernel).  T0 comes from a
// strided sample; if it turns out too high (fewer than k candidates) or too
// low (candidate capacity exceeded) the select kernel rescans the residual
// instead, so the result never depends on the estimate.
#pragma once

#include "common.cuh"

namespace tke {

constexpr int TCAP_SMALL = 8;        // setup parameter block for T <= 8
constexpr int TCAP_LARGE = 256;      // tensors per group
constexpr int SAMPLE_M = 16384;      // samples per sampled tensor
constexpr int SAMPLE_THREADS = 1024;
constexpr int SAMPLE_PER_THREAD = SAMPLE_M / SAMPLE_THREADS;
constexpr int SAMPLE_BINS = 4096;    // key >> 19
constexpr int K1_THREADS = 512;
constexpr int K1_VECS = 4;           // float4 of each input per thread per tile
constexpr int TILE = K1_THREADS * K1_VECS * 4;   // 8192 elements
constexpr int ZERO_THREADS = 1024;

// Per-tensor metadata written by the setup kernel.
struct SegMeta {
    int64_t off;        // first element in the group's bucket
    int64_t n;          // elements
    int64_t out_base;   // first output slot
    uint32_t k;
    uint32_t T0;        // prefilter threshold key (NO_KEY when k == 0)
};
static_assert(sizeof(SegMeta) == 32, "SegMeta layout");

template <int TCAP>
struct SetupParams {
    const float* grad;
    const float* resid;
    float lr;
    int32_t T;
    int32_t n_sampled;
    uint32_t kernels;
    uint64_t cap;
    Ctrl* ctrl;
    SegMeta* meta;
    uint4* zero_ptr;        // region cleared for this call
    uint64_t zero_vec4;     // its size in 16-byte words
    int64_t off[TCAP + 1];
    int64_t out_base[TCAP];
    uint32_t k[TCAP];
    uint32_t m[TCAP];       // samples (0: no sampling)
    uint32_t r[TCAP];       // target rank among the samples
    uint16_t sampled[TCAP]; // tensor of sampling block i
};

// Blocks [0, n_sampled) each estimate T0 of one tensor from SAMPLE_M strided
// samples of acc; the remaining blocks clear the workspace state of this call
// and write the metadata of the tensors that are not sampled.
template <int TCAP>
__global__ void __launch_bounds__(SAMPLE_THREADS)
setup_kernel(const __grid_constant__ SetupParams<TCAP> p) {
    __shared__ uint32_t hist[SAMPLE_BINS];
    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    if (b < p.n_sampled) {
        const int l = p.sampled[b];
        const int64_t off = p.off[l];
        const int64_t n = p.off[l + 1] - off;
        const uint32_t m = p.m[l];
        for (int i = tid; i < SAMPLE_BINS; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        uint32_t key[SAMPLE_PER_THREAD];
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u) {
            const uint32_t s = (uint32_t)(u * SAMPLE_THREADS + tid);
            key[u] = NO_KEY;
            if (s < m) {
                const int64_t pos = off + ((int64_t)s * n) / (int64_t)m;
                const float a = __fmaf_rn(p.lr, __ldg(p.grad + pos), __ldg(p.resid + pos));
                key[u] = key_of(a);
            }
        }
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u)
            if (key[u] != NO_KEY) atomicAdd(&hist[key[u] >> 19], 1u);
        __syncthreads();
        if (tid < 32) {
            uint32_t bin, above, cnt;
            warp_find_bin(hist, SAMPLE_BINS, p.r[l], bin, above, cnt);
            if (tid == 0) {
                SegMeta sm;
                sm.off = off;
                sm.n = n;
                sm.out_base = p.out_base[l];
                sm.k = p.k[l];
                sm.T0 = bin << 19;
                p.meta[l] = sm;
            }
        }
        return;
    }
    const int zb = b - p.n_sampled;
    const int nz = gridDim.x - p.n_sampled;
    if (zb == 0) {
        if (tid == 0) {
            Ctrl c;
            memset(&c, 0, sizeof(c));
            c.cap = p.cap;
            c.kernels = p.kernels;
            *p.ctrl = c;
        }
        for (int l = tid; l < p.T; l += blockDim.x) {
            if (p.m[l] != 0) continue;
            SegMeta sm;
            sm.off = p.off[l];
            sm.n = p.off[l + 1] - p.off[l];
            sm.out_base = p.out_base[l];
            sm.k = p.k[l];
            sm.T0 = p.k[l] == 0 ? NO_KEY : 0u;
            p.meta[l] = sm;
        }
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (uint64_t i = (uint64_t)zb * blockDim.x + tid; i < p.zero_vec4;
         i += (uint64_t)nz * blockDim.x)
        p.zero_ptr[i] = z;
}

struct StreamParams {
    const float* grad;
    float* resid;
    float lr;
    int32_t T;
    int64_t N;
    uint32_t num_tiles;
    const SegMeta* meta;
    Ctrl* ctrl;
    uint64_t* tile_status;  // [num_tiles], cleared by the setup kernel
    uint32_t* cand_idx;     // [cap]
    float* cand_val;        // [cap]
    uint64_t cap;
    uint32_t* hist;         // [T][HIST_WORDS]; candidate D1 at offset 0
    int64_t* cand_start;    // [T+1]
};

constexpr uint64_t LB_AGG = 1ull << 62;
constexpr uint64_t LB_INC = 2ull << 62;
constexpr uint64_t LB_VAL = (1ull << 62) - 1;

// Decoupled look-back (run by one full warp): publishes this tile's count,
// returns the number of candidates in all earlier tiles.  Tiles are handed
// out in ticket order, so every earlier tile belongs to a running block and
// publishes without waiting; each wait is still bounded.
__device__ __forceinline__ uint64_t lookback(uint64_t* status, uint32_t t, uint32_t count,
                                             uint32_t* ctrl_status) {
    const uint32_t lane = lane_id();
    if (t == 0) {
        if (lane == 0) st_release_u64(&status[0], LB_INC | count);
        return 0;
    }
    if (lane == 0) st_release_u64(&status[t], LB_AGG | count);
    uint64_t excl = 0;
    int64_t top = (int64_t)t - 1;
    for (;;) {
        const int64_t i = top - (int64_t)lane;
        uint64_t s = LB_INC;  // before tile 0: inclusive zero
        if (i >= 0) {
            s = ld_acquire_u64(&status[i]);
            uint32_t it = 0;
            while ((s >> 62) == 0) {
                if (++it > SPIN_LIMIT) {
                    atomicOr(ctrl_status, ST_TIMEOUT);
                    s = LB_INC;
                    break;
                }
                __nanosleep(32);
                s = ld_acquire_u64(&status[i]);
            }
        }
        const uint32_t inc = __ballot_sync(0xFFFFFFFFu, (s >> 62) == 2);
        if (inc) {
            const uint32_t w = __ffs(inc) - 1;
            uint64_t v = lane <= w ? (s & LB_VAL) : 0;
            excl += warp_sum(v);
            break;
        }
        excl += warp_sum(s & LB_VAL);
        top -= 32;
    }
    if (lane == 0) st_release_u64(&status[t], LB_INC | (excl + count));
    return excl;
}

// Tensor l with off[l] <= e < off[l+1] (empty tensors are skipped).
__device__ __forceinline__ int seg_of(const int64_t* off, int T, int64_t e) {
    int lo = 0, hi = T;   // answer in [0, T)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= e) lo = mid; else hi = mid;
    }
    return lo;
}

// First l in [0, T] with off[l] >= e.
__device__ __forceinline__ int lower_bound_off(const int64_t* off, int T, int64_t e) {
    int lo = 0, hi = T + 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] < e) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// The fused streaming pass: acc = fmaf(lr, grad, residual) written to
// residual, candidates (key >= T0 of the element's tensor) appended in index
// order, their top-digit histogram per tensor, and each tensor's first
// candidate slot.  Persistent blocks take 8192-element tiles by ticket.
template <bool VEC>
__global__ void __launch_bounds__(K1_THREADS, 2)
stream_kernel(const StreamParams p) {
    __shared__ int64_t s_off[TCAP_LARGE + 1];
    __shared__ uint32_t s_T0[TCAP_LARGE];
    __shared__ uint32_t s_wcnt[K1_VECS * (K1_THREADS / 32)];
    __shared__ uint32_t s_red[33];
    __shared__ uint32_t s_tile;
    __shared__ uint64_t s_base;
    __shared__ uint32_t s_count;

    const int tid = threadIdx.x;
    const uint32_t lane = lane_id(), warp = warp_id();
    const int T = p.T;
    for (int l = tid; l < T; l += blockDim.x) {
        s_off[l] = p.meta[l].off;
        s_T0[l] = p.meta[l].T0;
    }
    if (tid == 0) s_off[T] = p.N;
    __syncthreads();

    for (;;) {
        if (tid == 0) s_tile = atomicAdd(&p.ctrl->tile_ticket, 1u);
        __syncthreads();
        const uint32_t t = s_tile;
        if (t >= p.num_tiles) break;
        const int64_t base = (int64_t)t * TILE;
        const int64_t tend = min(base + (int64_t)TILE, p.N);
        const int l_lo = seg_of(s_off, T, base);
        const int l_hi = seg_of(s_off, T, tend - 1);
        const bool uniform = (l_lo == l_hi);
        const uint32_t T0u = s_T0[l_lo];

        float g[K1_VECS][4], r[K1_VECS][4];
#pragma unroll
        for (int j = 0; j < K1_VECS; ++j) {
            const int64_t e = base + (int64_t)(j * K1_THREADS + tid) * 4;
            if (VEC && e + 3 < p.N) {
                const float4 gv = ld_stream(reinterpret_cast<const float4*>(p.grad + e));
                const float4 rv = ld_stream(reinterpret_cast<const float4*>(p.resid + e));
                g[j][0] = gv.x; g[j][1] = gv.y; g[j][2] = gv.z; g[j][3] = gv.w;
                r[j][0] = rv.x; r[j][1] = rv.y; r[j][2] = rv.z; r[j][3] = rv.w;
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    g[j][v] = 0.f;
                    r[j][v] = 0.f;
                    if (e + v < p.N) {
                        g[j][v] = __ldcs(p.grad + e + v);
                        r[j][v] = __ldcs(p.resid + e + v);
                    }
                }
            }
        }

        uint32_t flags = 0;
#pragma unroll
        for (int j = 0; j < K1_VECS; ++j) {
            const int64_t e = base + (int64_t)(j * K1_THREADS + tid) * 4;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float a = __fmaf_rn(p.lr, g[j][v], r[j][v]);
                r[j][v] = a;
                if (e + v < p.N) {
                    uint32_t T0 = T0u;
                    if (!uniform) {
                        int l = l_lo;
                        while (l < l_hi && s_off[l + 1] <= e + v) ++l;
                        T0 = s_T0[l];
                    }
                    if (key_of(a) >= T0) flags |= 1u << (j * 4 + v);
                }
            }
            if (VEC && e + 3 < p.N) {
                st_stream(reinterpret_cast<float4*>(p.resid + e),
                          make_float4(r[j][0], r[j][1], r[j][2], r[j][3]));
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    if (e + v < p.N) __stcs(p.resid + e + v, r[j][v]);
            }
        }

        // order-preserving positions: (vector j, thread, element v)
        uint32_t lane_excl[K1_VECS];
#pragma unroll
        for (int j = 0; j < K1_VECS; ++j) {
            const uint32_t c = __popc((flags >> (4 * j)) & 0xFu);
            const uint32_t incl = warp_incl_scan(c);
            lane_excl[j] = incl - c;
            if (lane == 31) s_wcnt[j * (K1_THREADS / 32) + warp] = incl;
        }
        __syncthreads();
        if (warp == 0) {
            constexpr int NE = K1_VECS * (K1_THREADS / 32);   // 64 entries
            static_assert(NE == 64, "two entries per lane");
            const uint32_t v0 = s_wcnt[2 * lane], v1 = s_wcnt[2 * lane + 1];
            const uint32_t sum = v0 + v1;
            const uint32_t incl = warp_incl_scan(sum);
            const uint32_t excl = incl - sum;
            s_wcnt[2 * lane] = excl;
            s_wcnt[2 * lane + 1] = excl + v0;
            const uint32_t tile_count = __shfl_sync(0xFFFFFFFFu, incl, 31);
            const uint64_t tb = lookback(p.tile_status, t, tile_count, &p.ctrl->status);
            if (lane == 0) {
                s_base = tb;
                s_count = tile_count;
            }
        }
        __syncthreads();
        const uint64_t tbase = s_base;

        if (flags) {
#pragma unroll
            for (int j = 0; j < K1_VECS; ++j) {
                const uint32_t fj = (flags >> (4 * j)) & 0xFu;
                if (!fj) continue;
                const int64_t e = base + (int64_t)(j * K1_THREADS + tid) * 4;
                uint64_t pos = tbase + s_wcnt[j * (K1_THREADS / 32) + warp] + lane_excl[j];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    if (!((fj >> v) & 1u)) continue;
                    if (pos < p.cap) {
                        int l = l_lo;
                        if (!uniform)
                            while (l < l_hi && s_off[l + 1] <= e + v) ++l;
                        p.cand_idx[pos] = (uint32_t)(e + v);
                        p.cand_val[pos] = r[j][v];
                        atomicAdd(&p.hist[(size_t)l * HIST_WORDS + (key_of(r[j][v]) >> 20)], 1u);
                    }
                    ++pos;
                }
            }
        }

        // first candidate slot of every tensor that starts inside this tile
        const int lb = max(1, lower_bound_off(s_off, T, base));
        const int ub = min(T, lower_bound_off(s_off, T, tend));
        for (int l = lb; l < ub; ++l) {
            const int64_t bound = s_off[l];
            uint32_t c = 0;
#pragma unroll
            for (int j = 0; j < K1_VECS; ++j) {
                const int64_t e = base + (int64_t)(j * K1_THREADS + tid) * 4;
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    c += ((flags >> (j * 4 + v)) & 1u) && (e + v < bound);
            }
            const uint32_t before = block_sum(c, s_red);
            if (tid == 0) p.cand_start[l] = (int64_t)(tbase + before);
        }
        if (t == p.num_tiles - 1 && tid == 0) {
            const uint64_t total = tbase + s_count;
            p.ctrl->cand_total = total;
            // tensors that start at the end of the bucket (empty ones), and T
            for (int l = lower_bound_off(s_off, T, p.N); l <= T; ++l)
                p.cand_start[l] = (int64_t)total;
        }
        __syncthreads();
    }
}

}  // namespace tke
