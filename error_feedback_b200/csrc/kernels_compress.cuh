// Compress kernels: setup + threshold estimate, and the fused streaming pass.
//
// One error-feedback step ("Sparsified SGD with Memory" and "The Convergence
// of Sparsified Gradient Methods", abstracts in the arxivdaily listing; "A
// Distributed Synchronous SGD Algorithm with Global Top-k Sparsification",
// ABSTRACT) computes acc = fmaf(lr, grad, residual), keeps the k entries of
// largest |acc| and leaves the rest in memory.  The only pass over the full
// tensor is the streaming kernel below: it reads grad and residual once,
// writes acc back into residual, and stages every element whose key reaches
// a prefilter threshold T0 as a candidate.  The exact top-k is then found
// among the candidates (select kernel).  T0 comes from a strided sample; if
// it turns out too high (fewer than k candidates) or too low (candidate
// capacity exceeded) the select kernel rescans the residual instead, so the
// result never depends on the estimate.
#pragma once

#include "common.cuh"

namespace tke {

constexpr int TCAP_SMALL = 8;        // setup parameter block for T <= 8
constexpr int TCAP_LARGE = 256;      // tensors per group
constexpr int SAMPLE_LOG2 = 14;
constexpr int SAMPLE_M = 1 << SAMPLE_LOG2;   // samples per sampled tensor
constexpr int SAMPLE_THREADS = 1024;
constexpr int SAMPLE_PER_THREAD = SAMPLE_M / SAMPLE_THREADS;
constexpr int SAMPLE_BINS = 4096;    // key >> 19
constexpr int K1_THREADS = 256;
constexpr int WT = 1024;             // elements per warp tile
constexpr int WT_VECS = WT / 128;    // float4 of each input per lane per warp tile
constexpr int WT_CAP = 16;           // candidates staged per warp tile
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

// Blocks [0, n_sampled) each estimate T0 of one tensor from SAMPLE_M samples
// of acc (256 evenly spread runs of 64 consecutive elements, so the loads
// coalesce); the remaining blocks clear the workspace state of this call
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
                // 256 chunks of 64 consecutive elements, evenly spread
                const int64_t pos = off + (((int64_t)(s >> 6) * n) >> 8) + (s & 63);
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
                // never above 0x7F800001: then "raw |x| bits >= T0" and "key >= T0"
                // agree for NaN too (lowering T0 only adds candidates)
                sm.T0 = min(bin << 19, 0x7F800001u);
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
    uint32_t num_wt;        // warp tiles of WT elements
    const SegMeta* meta;
    Ctrl* ctrl;
    uint32_t* wt_count;     // [num_wt] candidates of each warp tile (exact)
    uint32_t* st_idx;       // [num_wt][WT_CAP] staged candidates, index order
    float* st_val;
    uint32_t* hist;         // [T][HIST_WORDS]; candidate digit 1 at offset 0
    uint32_t* bound_before; // [T]: candidates of the warp tile holding off[l] below off[l]
};

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

// The fused streaming pass, the only full sweep of the step:
//   acc = fmaf(lr, grad, residual) written back to residual;
//   candidates (key >= T0 of the element's tensor) staged per warp tile in
//   index order (at most WT_CAP; the count is always exact);
//   digit-1 histogram of the candidates per tensor.
// Each warp owns whole 1,024-element warp tiles (grid-stride), so warps never
// wait for one another: the global order of the candidates is rebuilt by the
// select kernel from the per-warp-tile counts.
template <bool VEC>
__global__ void __launch_bounds__(K1_THREADS, 3)
stream_kernel(const StreamParams p) {
    __shared__ int64_t s_off[TCAP_LARGE + 1];
    __shared__ uint32_t s_T0[TCAP_LARGE];
    __shared__ uint32_t s_h1[D1_BINS];

    const int tid = threadIdx.x;
    const uint32_t lane = lane_id();
    const int T = p.T;
    const bool flat = (T == 1);
    for (int l = tid; l < T; l += blockDim.x) {
        s_off[l] = p.meta[l].off;
        s_T0[l] = p.meta[l].T0;
    }
    if (tid == 0) s_off[T] = p.N;
    if (flat)
        for (int i = tid; i < D1_BINS; i += blockDim.x) s_h1[i] = 0;
    __syncthreads();

    const uint32_t warps = blockDim.x >> 5;
    const uint32_t gw = blockIdx.x * warps + warp_id();
    const uint32_t GW = gridDim.x * warps;
    for (uint32_t w = gw; w < p.num_wt; w += GW) {
        const int64_t base = (int64_t)w * WT;
        const int64_t tend = min(base + (int64_t)WT, p.N);
        const int l_lo = flat ? 0 : seg_of(s_off, T, base);
        const int l_hi = flat ? 0 : seg_of(s_off, T, tend - 1);
        const bool uniform = (l_lo == l_hi);
        const uint32_t T0u = s_T0[l_lo];

        float r[WT_VECS][4];
        uint32_t flags = 0;
        if (VEC && uniform && tend - base == WT) {
            // full warp tile inside one tensor: 128-bit loads, no bounds checks
            const float4* g4 = reinterpret_cast<const float4*>(p.grad + base) + lane;
            float4* r4 = reinterpret_cast<float4*>(p.resid + base) + lane;
            float4 gv[WT_VECS], rv[WT_VECS];
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                gv[j] = ld_stream(g4 + 32 * j);
                rv[j] = ld_stream(r4 + 32 * j);
            }
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                float4 a;
                a.x = __fmaf_rn(p.lr, gv[j].x, rv[j].x);
                a.y = __fmaf_rn(p.lr, gv[j].y, rv[j].y);
                a.z = __fmaf_rn(p.lr, gv[j].z, rv[j].z);
                a.w = __fmaf_rn(p.lr, gv[j].w, rv[j].w);
                st_stream(r4 + 32 * j, a);
                r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                flags |= (uint32_t)((__float_as_uint(a.x) & KEY_MASK) >= T0u) << (4 * j);
                flags |= (uint32_t)((__float_as_uint(a.y) & KEY_MASK) >= T0u) << (4 * j + 1);
                flags |= (uint32_t)((__float_as_uint(a.z) & KEY_MASK) >= T0u) << (4 * j + 2);
                flags |= (uint32_t)((__float_as_uint(a.w) & KEY_MASK) >= T0u) << (4 * j + 3);
            }
        } else {
            float g[WT_VECS][4];
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                const int64_t e = base + j * 128 + lane * 4;
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
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                const int64_t e = base + j * 128 + lane * 4;
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
        }

        // candidates of the warp tile, in index order (vector j, lane, element v)
        const uint32_t any = __ballot_sync(0xFFFFFFFFu, flags != 0);
        const uint32_t cnt = any ? warp_sum((uint32_t)__popc(flags)) : 0u;
        if (lane == 0) p.wt_count[w] = cnt;
        if (cnt) {
            uint32_t before = 0;   // candidates of earlier vectors
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                const uint32_t fj = (flags >> (4 * j)) & 0xFu;
                if (!__any_sync(0xFFFFFFFFu, fj != 0)) continue;
                const uint32_t c = __popc(fj);
                const uint32_t incl = warp_incl_scan(c);
                uint32_t pos = before + incl - c;
                const int64_t e = base + j * 128 + lane * 4;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    if (!((fj >> v) & 1u)) continue;
                    if (cnt <= WT_CAP) {
                        p.st_idx[(size_t)w * WT_CAP + pos] = (uint32_t)(e + v);
                        p.st_val[(size_t)w * WT_CAP + pos] = r[j][v];
                    }
                    const uint32_t bin = key_of(r[j][v]) >> 20;
                    if (flat) {
                        atomicAdd(&s_h1[bin], 1u);
                    } else {
                        int l = l_lo;
                        if (!uniform)
                            while (l < l_hi && s_off[l + 1] <= e + v) ++l;
                        atomicAdd(&p.hist[(size_t)l * HIST_WORDS + bin], 1u);
                    }
                    ++pos;
                }
                before += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
        }

        // tensors that start inside this warp tile: candidates below the start
        if (!flat) {
            const int lb = max(1, lower_bound_off(s_off, T, base));
            const int ub = min(T, lower_bound_off(s_off, T, tend));
            for (int l = lb; l < ub; ++l) {
                const int64_t bound = s_off[l];
                uint32_t c = 0;
#pragma unroll
                for (int j = 0; j < WT_VECS; ++j) {
                    const int64_t e = base + j * 128 + lane * 4;
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        c += ((flags >> (j * 4 + v)) & 1u) && (e + v < bound);
                }
                c = warp_sum(c);
                if (lane == 0) p.bound_before[l] = c;
            }
        }
    }
    if (flat) {
        __syncthreads();
        for (int i = tid; i < D1_BINS; i += blockDim.x)
            if (s_h1[i]) atomicAdd(&p.hist[i], s_h1[i]);
    }
}

}  // namespace tke
