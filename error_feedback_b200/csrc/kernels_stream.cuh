// The fused streaming pass of the compress step ("Sparsified SGD with
// Memory" and "The Convergence of Sparsified Gradient Methods", abstracts in
// the arxivdaily listing): acc = fmaf(lr, grad, residual) written back to the
// residual, and the positions of the entries whose key reaches the
// prefilter threshold T0 recorded per warp tile.  The only full sweep of a
// step; everything it needs from the setup kernel is in SegMeta.
#pragma once

#include "common.cuh"
#include "kernels_compress.cuh"

namespace tke {

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
    uint32_t* r1;           // one tensor: its candidates' relative digit-1 histogram
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
    uint32_t r1[REL_BINS];      // one tensor: this block's share of p.r1
};

// Relative digit-1 bin of a candidate (key >= T0): min((key - T0) >> sh, 4095).
__device__ __forceinline__ uint32_t stream_rel_bin(float a, uint32_t T0, uint32_t sh) {
    return min((key_of(a) - T0) >> sh, (uint32_t)(REL_BINS - 1));
}

// General warp tile: a partial last tile, a tile that spans tensors, or
// unaligned inputs.  Computes acc, stores it, returns the candidate flags
// (bit 4j + v for element base + 128 j + 4 lane + v).
template <bool VEC>
__device__ __noinline__ uint32_t stream_tile_general(const StreamParams& p, StreamShared& S,
                                                     int64_t base, int l_lo, int l_hi,
                                                     uint32_t sh) {
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
            if (key_of(a[v]) >= S.T0[l]) {
                flags |= 1u << (j * 4 + v);
                if (p.r1) atomicAdd(&S.r1[stream_rel_bin(a[v], S.T0[l], sh)], 1u);
            }
        }
    }
    return flags;
}

// Record the candidates of a warp tile: the exact count and, up to WT_CAP of
// them, their offsets in the tile (lane-major, so not in index order; the
// select kernel sorts each tile's few offsets and reads the values back from
// the residual, which now holds acc).  Bit 4j + v of a lane's flags is offset
// 128 j + 4 lane + v.  With kRegs and hist, each candidate is also counted in
// the relative digit-1 histogram s_r1 (its acc in the caller's registers:
// element 128 j + 4 lane + v in rv[j]) in the same walk over the flags.
template <bool kRegs>
__device__ __forceinline__ void stream_tile_stage(const StreamParams& p, uint32_t w, uint32_t flags,
                                                  const float4* rv, bool hist, uint32_t* s_r1,
                                                  uint32_t T0, uint32_t sh) {
    const uint32_t lane = lane_id();
    const uint32_t pc = (uint32_t)__popc(flags);
    const uint32_t incl = warp_incl_scan(pc);
    if (lane == 31) p.wt_count[w] = incl;
    uint32_t pos = incl - pc;
    uint16_t* dst = p.wt_off + (size_t)w * WT_CAP;
    if (kRegs && hist) {
#pragma unroll
        for (int j = 0; j < WT_VECS; ++j) {
            const uint32_t f4 = (flags >> (4 * j)) & 0xFu;
            if (f4 == 0) continue;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                if ((f4 >> v) & 1u) {
                    if (pos < (uint32_t)WT_CAP) dst[pos] = (uint16_t)(128u * j + 4u * lane + v);
                    ++pos;
                    const float a = v == 0 ? rv[j].x : (v == 1 ? rv[j].y : (v == 2 ? rv[j].z : rv[j].w));
                    atomicAdd(&s_r1[stream_rel_bin(a, T0, sh)], 1u);
                }
            }
        }
    } else {
        while (flags && pos < (uint32_t)WT_CAP) {
            const uint32_t b = (uint32_t)(__ffs(flags) - 1);
            flags &= flags - 1;
            dst[pos++] = (uint16_t)(128u * (b >> 2) + 4u * lane + (b & 3u));
        }
    }
}

template <bool kRegs>
__device__ __forceinline__ void stream_tile_record(const StreamParams& p, uint32_t w,
                                                   uint32_t flags, const float4* rv,
                                                   bool hist = false, uint32_t* s_r1 = nullptr,
                                                   uint32_t T0 = 0, uint32_t sh = 0) {
    if (__any_sync(0xFFFFFFFFu, flags != 0))
        stream_tile_stage<kRegs>(p, w, flags, rv, hist, s_r1, T0, sh);
    else if (lane_id() == 0) p.wt_count[w] = 0;
}

// The fused streaming pass, the only full sweep of the step:
//   acc = fmaf(lr, grad, residual) written back to residual;
//   candidates (key >= T0 of the element's tensor) recorded per warp tile of
//   1,024 elements: an exact count and the offsets of up to WT_CAP of them.
// Each warp owns whole warp tiles, so warps never wait for one another; the
// select kernel rebuilds the ordered candidate list from the records.  The loop
// over full tiles of one tensor is kept small; everything else is out of line.
// MINB: resident blocks per SM the registers are sized for.  A single tensor
// with a short candidate list runs 4 per SM (64 registers): the step of the
// 25.6M-element workload at 0.1% and 0.01% density measured 1.2 to 2 us
// faster, although the kernel alone is slower.  Everything else runs 3 per
// SM (80 registers), which measured faster for a bucket (3.5 us on the
// VGG-16 bucket), for long candidate lists (2 us at 1% density; 90 us on
// 1.5e9 elements) and for the hard-threshold step (4 us).
template <bool VEC, int MINB>
__global__ void __launch_bounds__(K1_THREADS, MINB)
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
    // the select kernel may be scheduled now (it waits for this grid to end)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");   // setup_kernel's results
    if (tid == 0) span_first(p.ctrl, SPAN_STREAM_FIRST);
    const uint32_t lane = lane_id();
    const int T = p.T;
    const bool flat = (T == 1);
    for (int l = tid; l < T; l += blockDim.x) {
        S.off[l] = p.meta[l].off;
        S.T0[l] = p.meta[l].T0;
    }
    if (tid == 0) S.off[T] = p.N;
    // one tensor: the candidates' relative digit-1 histogram is built here
    const bool hist = flat && p.r1 != nullptr;
    const uint32_t sh = hist ? p.meta[0].shift : 0u;
    if (hist)
        for (int i = tid; i < REL_BINS; i += blockDim.x) S.r1[i] = 0;
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
                rv[j] = a;
            }
            stream_tile_record<true>(p, w, flags, rv, hist, S.r1, T0, sh);
        } else {
            stream_tile_record<false>(p, w, stream_tile_general<VEC>(p, S, base, l_lo, l_hi, sh),
                                      nullptr);
        }
        w = stat_next ? w + GW : R * GW + __shfl_sync(0xFFFFFFFFu, ticket, 0);
    }
    __syncthreads();
    if (hist)
        for (int i = tid; i < REL_BINS; i += blockDim.x)
            if (S.r1[i]) atomicAdd(&p.r1[i], S.r1[i]);
    if (tid == 0) span_last(p.ctrl, SPAN_STREAM_LAST);
}

}  // namespace tke
