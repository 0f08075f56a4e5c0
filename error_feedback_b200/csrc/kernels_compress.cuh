// Compress kernels: setup + threshold estimate, and the fused streaming pass.
//
// One error-feedback step ("Sparsified SGD with Memory" and "The Convergence
// of Sparsified Gradient Methods", abstracts in the arxivdaily listing; "A
// Distributed Synchronous SGD Algorithm with Global Top-k Sparsification",
// ABSTRACT) computes acc = fmaf(lr, grad, residual), keeps the k entries of
// largest |acc| and leaves the rest in memory.  The only pass over the full
// tensor is the streaming kernel below: it reads grad and residual once,
// writes acc back into residual, and records where the elements whose key
// reaches a prefilter threshold T0 (the candidates) are.  The exact top-k is then found
// among the candidates (select kernel).  T0 comes from a strided sample; if
// it turns out too high (fewer than k candidates) or too low (candidate
// capacity exceeded) the select kernel rescans the residual instead, so the
// result never depends on the estimate.
#pragma once

#include "common.cuh"

namespace tke {

constexpr int TCAP_SMALL = 8;        // setup parameter block for T <= 8
constexpr int TCAP_LARGE = 256;      // tensors per group
constexpr int SAMPLE_LOG2 = 13;
constexpr int SAMPLE_M = 1 << SAMPLE_LOG2;   // samples per sampled tensor
constexpr int SAMPLE_THREADS = 1024;
constexpr int SAMPLE_PER_THREAD = SAMPLE_M / SAMPLE_THREADS;  // keys each thread holds
constexpr int SAMPLE_BINS = 4096;    // key >> 19
constexpr int K1_THREADS = 256;
constexpr int WT = 1024;             // elements per warp tile
constexpr int WT_VECS = WT / 128;    // float4 of each input per lane per warp tile
constexpr int WT_CAP = 16;           // candidate offsets staged per warp tile
constexpr uint32_t STREAM_PREFETCH = 3;   // warp tiles per warp pulled into L2 early
constexpr int ZERO_THREADS = 1024;

// Per-tensor metadata written by the setup kernel.
struct SegMeta {
    int64_t off;        // first element in the group's bucket
    int64_t n;          // elements
    int64_t out_base;   // first output slot
    uint32_t k;
    uint32_t T0;        // prefilter threshold key (NO_KEY when k == 0)
    uint32_t shift;     // relative digit: R1 = (key - T0) >> shift
    uint32_t t_ns[3];   // sampling block: ns from its start to the loaded samples,
                        // the first histogram level and the end (diagnostics)
};
static_assert(sizeof(SegMeta) == 48, "SegMeta layout");

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
    uint32_t m[TCAP];       // samples (0: no sampling; n: every element)
    uint32_t r[TCAP];       // target rank among the samples
    uint32_t r_hi[TCAP];    // rank of an upper estimate of the k-th key
    uint16_t sampled[TCAP]; // i-th sampled tensor (block i samples it)
    int32_t has_fixed_T0;   // hard threshold: every tensor uses fixed_T0
    uint32_t fixed_T0;
};

// Block i < n_sampled samples acc for the prefilter threshold T0 of the i-th
// sampled tensor: every element when the tensor has at most SAMPLE_M of them,
// otherwise SAMPLE_M samples in 128 evenly spread runs of 64 consecutive
// elements (the loads coalesce).  The keys stay in registers; T0 is the lower
// edge of the bin of the r-th largest in two histogram levels (key bits 30..19,
// then 18..7), so T0 <= that key.  The shift of the relative digits is
// chosen so that 4,095 bins of 2^shift keys above T0 reach twice past an
// upper estimate of the k-th key.  The remaining blocks clear the workspace
// state of this call and write the metadata of the tensors not sampled.
template <int TCAP>
__global__ void __launch_bounds__(SAMPLE_THREADS)
setup_kernel(const __grid_constant__ SetupParams<TCAP> p) {
    __shared__ uint32_t hist[SAMPLE_BINS];
    __shared__ uint32_t s_red[33];
    __shared__ FindResult s_fr;
    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    // the streaming kernel may be scheduled now (it waits for this grid);
    // this grid waits for the kernel before it on the stream
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (b < p.n_sampled) {
        const int l = p.sampled[b];
        const int64_t off = p.off[l];
        const int64_t n = p.off[l + 1] - off;
        const uint32_t m = p.m[l];
        const bool full = (int64_t)m == n;
        const uint64_t t_start = global_ns();
        for (int i2 = tid; i2 < SAMPLE_BINS; i2 += blockDim.x) hist[i2] = 0;
        // every element, or 128 runs of 64 consecutive elements; all loads
        // are issued before the first is used
        float gv[SAMPLE_PER_THREAD], rv[SAMPLE_PER_THREAD];
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u) {
            const uint32_t s = (uint32_t)(u * SAMPLE_THREADS + tid);
            const int64_t pos = full ? off + s : off + (((int64_t)(s >> 6) * n) >> 7) + (s & 63);
            gv[u] = s < m ? __ldg(p.grad + pos) : 0.f;
            rv[u] = s < m ? __ldg(p.resid + pos) : 0.f;
        }
        uint32_t key[SAMPLE_PER_THREAD];
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u) {
            const uint32_t s = (uint32_t)(u * SAMPLE_THREADS + tid);
            key[u] = s < m ? key_of(__fmaf_rn(p.lr, gv[u], rv[u])) : NO_KEY;
        }
        __syncthreads();
        const uint64_t t_loaded = global_ns();
        // level 1: key >> 19
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u)
            if (key[u] != NO_KEY) atomicAdd(&hist[key[u] >> 19], 1u);
        __syncthreads();
        block_find_bin(hist, SAMPLE_BINS, p.r[l], s_red, &s_fr);
        const uint32_t ok1 = s_fr.ok, b1 = s_fr.bin;
        const uint32_t rem = p.r[l] - s_fr.above;
        __syncthreads();
        block_find_bin(hist, SAMPLE_BINS, p.r_hi[l], s_red, &s_fr);
        const uint32_t bhi = s_fr.ok ? s_fr.bin : b1;
        const uint64_t t_level1 = global_ns();
        // level 2: bits 18..7 of the keys in bin b1
        __syncthreads();
        for (int i2 = tid; i2 < SAMPLE_BINS; i2 += blockDim.x) hist[i2] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u)
            if (key[u] != NO_KEY && (key[u] >> 19) == b1) atomicAdd(&hist[(key[u] >> 7) & 4095u], 1u);
        __syncthreads();
        block_find_bin(hist, SAMPLE_BINS, rem, s_red, &s_fr);
        const uint32_t ok2 = s_fr.ok, b2 = s_fr.bin;
        if (tid == 0) {
            uint32_t T0 = 0;
            if (ok1 && ok2) T0 = (b1 << 19) | (b2 << 7);
            // never above 0x7F800001: then "raw |x| bits >= T0" and "key >= T0"
            // agree for NaN too (lowering T0 only adds candidates)
            T0 = min(T0, 0x7F800001u);
            const uint64_t hi = ((uint64_t)(bhi + 1) << 19);
            const uint64_t d = hi > T0 ? hi - T0 : 0;
            uint32_t sh = 0;
            while (sh < (uint32_t)REL_MAX_SHIFT && ((uint64_t)(REL_BINS - 1) << sh) <= 2 * d) ++sh;
            SegMeta sm;
            memset(&sm, 0, sizeof(sm));
            sm.off = off;
            sm.n = n;
            sm.out_base = p.out_base[l];
            sm.k = p.k[l];
            sm.T0 = T0;
            sm.shift = sh;
            const uint64_t t_end = global_ns();
            sm.t_ns[0] = (uint32_t)(t_loaded - t_start);
            sm.t_ns[1] = (uint32_t)(t_level1 - t_start);
            sm.t_ns[2] = (uint32_t)(t_end - t_start);
            p.meta[l] = sm;
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
            memset(&sm, 0, sizeof(sm));
            sm.off = p.off[l];
            sm.n = p.off[l + 1] - p.off[l];
            sm.out_base = p.out_base[l];
            sm.k = p.k[l];
            sm.T0 = p.has_fixed_T0 ? p.fixed_T0 : (p.k[l] == 0 ? NO_KEY : 0u);
            sm.shift = REL_MAX_SHIFT;
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
    uint16_t* wt_off;       // [num_wt][WT_CAP]: their offsets in the tile, unordered
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

struct StreamShared {
    int64_t off[TCAP_LARGE + 1];
    uint32_t T0[TCAP_LARGE];
};

// General warp tile: a partial last tile, a tile that spans tensors, or
// unaligned inputs.  Computes acc, stores it, returns the candidate flags
// (bit 4j + v for element base + 128 j + 4 lane + v).
template <bool VEC>
__device__ __noinline__ uint32_t stream_tile_general(const StreamParams& p, const StreamShared& S,
                                                     int64_t base, int l_lo, int l_hi) {
    const uint32_t lane = lane_id();
    uint32_t flags = 0;
    for (int j = 0; j < WT_VECS; ++j) {
        const int64_t e = base + j * 128 + lane * 4;
        float a[4];
        if (VEC && e + 3 < p.N) {
            const float4 gv = ld_stream(reinterpret_cast<const float4*>(p.grad + e));
            const float4 rv = ld_stream(reinterpret_cast<const float4*>(p.resid + e));
            a[0] = __fmaf_rn(p.lr, gv.x, rv.x);
            a[1] = __fmaf_rn(p.lr, gv.y, rv.y);
            a[2] = __fmaf_rn(p.lr, gv.z, rv.z);
            a[3] = __fmaf_rn(p.lr, gv.w, rv.w);
            st_stream(reinterpret_cast<float4*>(p.resid + e), make_float4(a[0], a[1], a[2], a[3]));
        } else {
            for (int v = 0; v < 4; ++v) {
                a[v] = 0.f;
                if (e + v < p.N) {
                    a[v] = __fmaf_rn(p.lr, __ldcs(p.grad + e + v), __ldcs(p.resid + e + v));
                    __stcs(p.resid + e + v, a[v]);
                }
            }
        }
        for (int v = 0; v < 4; ++v) {
            if (e + v >= p.N) continue;
            int l = l_lo;
            while (l < l_hi && S.off[l + 1] <= e + v) ++l;
            if (key_of(a[v]) >= S.T0[l]) flags |= 1u << (j * 4 + v);
        }
    }
    return flags;
}

// Record the candidates of a warp tile: the exact count and, up to WT_CAP of
// them, their offsets in the tile (lane-major, so not in index order; the
// select kernel sorts each tile's few offsets and reads the values back from
// the residual, which now holds acc).  Bit 4j + v of a lane's flags is offset
// 128 j + 4 lane + v.
__device__ __forceinline__ void stream_tile_stage(const StreamParams& p, uint32_t w, uint32_t flags) {
    const uint32_t lane = lane_id();
    const uint32_t pc = (uint32_t)__popc(flags);
    const uint32_t incl = warp_incl_scan(pc);
    if (lane == 31) p.wt_count[w] = incl;
    uint32_t pos = incl - pc;
    uint16_t* dst = p.wt_off + (size_t)w * WT_CAP;
    while (flags && pos < (uint32_t)WT_CAP) {
        const uint32_t b = (uint32_t)(__ffs(flags) - 1);
        flags &= flags - 1;
        dst[pos++] = (uint16_t)(128u * (b >> 2) + 4u * lane + (b & 3u));
    }
}

__device__ __forceinline__ void stream_tile_record(const StreamParams& p, uint32_t w,
                                                   uint32_t flags) {
    if (__any_sync(0xFFFFFFFFu, flags != 0)) stream_tile_stage(p, w, flags);
    else if (lane_id() == 0) p.wt_count[w] = 0;
}

// The fused streaming pass, the only full sweep of the step:
//   acc = fmaf(lr, grad, residual) written back to residual;
//   candidates (key >= T0 of the element's tensor) recorded per warp tile of
//   1,024 elements: an exact count and the offsets of up to WT_CAP of them.
// Each warp owns whole warp tiles, so warps never wait for one another; the
// select kernel rebuilds the ordered candidate list from the records.  The loop
// over full tiles of one tensor is kept small; everything else is out of line.
template <bool VEC>
__global__ void __launch_bounds__(K1_THREADS, 3)
stream_kernel(const __grid_constant__ StreamParams p) {
    __shared__ StreamShared S;
    const int tid = threadIdx.x;
    {
        // While the setup kernel still runs (this grid is launched early),
        // pull this warp's first warp tiles into L2: the reads do not depend
        // on it, only the writes and the candidate test do.
        const uint32_t warps = blockDim.x >> 5;
        const uint32_t gw0 = blockIdx.x * warps + warp_id();
        const uint32_t GW0 = gridDim.x * warps;
        const uint32_t R0 = p.num_wt / GW0 >= 2 ? p.num_wt / GW0 - 1 : 0;
        if (VEC && lane_id() == 0) {
            for (uint32_t i = 0; i < STREAM_PREFETCH && i < R0; ++i) {
                const int64_t base = (int64_t)(gw0 + i * GW0) * WT;
                if (base + WT > p.N) break;
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.grad + base),
                             "r"((uint32_t)(WT * 4))
                             : "memory");
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.resid + base),
                             "r"((uint32_t)(WT * 4))
                             : "memory");
            }
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");   // setup_kernel's results
    const uint32_t lane = lane_id();
    const int T = p.T;
    const bool flat = (T == 1);
    for (int l = tid; l < T; l += blockDim.x) {
        S.off[l] = p.meta[l].off;
        S.T0[l] = p.meta[l].T0;
    }
    if (tid == 0) S.off[T] = p.N;
    __syncthreads();

    // Warp tiles are handed out statically for all but the last rounds, then
    // by ticket, so that no warp is left with a whole extra round at the end.
    const uint32_t warps = blockDim.x >> 5;
    const uint32_t gw = blockIdx.x * warps + warp_id();
    const uint32_t GW = gridDim.x * warps;
    const uint32_t R = p.num_wt / GW >= 2 ? p.num_wt / GW - 1 : 0;   // static rounds
    const float lr = p.lr;
    uint32_t w;
    if (R > 0) {
        w = gw;
    } else {
        uint32_t t = 0;
        if (lane == 0) t = atomicAdd(&p.ctrl->tile_ticket, 1u);
        w = R * GW + __shfl_sync(0xFFFFFFFFu, t, 0);
    }
    for (uint32_t round = 0; w < p.num_wt; ++round) {
        // next tile: static, or a ticket fetched now and read after this tile
        uint32_t ticket = 0;
        const bool stat_next = round + 1 < R;
        if (!stat_next && lane == 0) ticket = atomicAdd(&p.ctrl->tile_ticket, 1u);
        const int64_t base = (int64_t)w * WT;
        const int64_t tend = min(base + (int64_t)WT, p.N);
        const int l_lo = flat ? 0 : seg_of(S.off, T, base);
        const int l_hi = flat ? 0 : seg_of(S.off, T, tend - 1);
        if (VEC && l_lo == l_hi && tend - base == WT) {
            // full warp tile inside one tensor: 128-bit loads, no bounds checks
            const uint32_t T0 = S.T0[l_lo];
            const float4* g4 = reinterpret_cast<const float4*>(p.grad + base) + lane;
            float4* r4 = reinterpret_cast<float4*>(p.resid + base) + lane;
            float4 gv[WT_VECS], rv[WT_VECS];
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                gv[j] = ld_stream(g4 + 32 * j);
                rv[j] = ld_stream(r4 + 32 * j);
            }
            uint32_t flags = 0;
#pragma unroll
            for (int j = 0; j < WT_VECS; ++j) {
                float4 a;
                a.x = __fmaf_rn(lr, gv[j].x, rv[j].x);
                a.y = __fmaf_rn(lr, gv[j].y, rv[j].y);
                a.z = __fmaf_rn(lr, gv[j].z, rv[j].z);
                a.w = __fmaf_rn(lr, gv[j].w, rv[j].w);
                st_stream(r4 + 32 * j, a);
                flags |= (uint32_t)((__float_as_uint(a.x) & KEY_MASK) >= T0) << (4 * j);
                flags |= (uint32_t)((__float_as_uint(a.y) & KEY_MASK) >= T0) << (4 * j + 1);
                flags |= (uint32_t)((__float_as_uint(a.z) & KEY_MASK) >= T0) << (4 * j + 2);
                flags |= (uint32_t)((__float_as_uint(a.w) & KEY_MASK) >= T0) << (4 * j + 3);
            }
            stream_tile_record(p, w, flags);
        } else {
            stream_tile_record(p, w, stream_tile_general<VEC>(p, S, base, l_lo, l_hi));
        }
        w = stat_next ? w + GW : R * GW + __shfl_sync(0xFFFFFFFFu, ticket, 0);
    }
}

}  // namespace tke
