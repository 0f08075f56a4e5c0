// Compress kernels: setup + threshold estimate (the fused streaming pass is
// in kernels_stream.cuh).
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
constexpr int WT_CAP = 32;           // candidate offsets staged per warp tile
constexpr int WT_THREAD = 16;        // staged candidates the select gathers per thread
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

// Prefilter threshold for the next call on the same flat tensor: written by
// the select kernel of a call that took the candidate path, used by the next
// call's setup kernel instead of sampling when the tag matches (same n, k,
// lr and residual).  The result never depends on it: a threshold that turns
// out too high or too low sends the call to the rescan of the residual, and
// that call clears the hint.
struct Hint {
    uint64_t tag;       // 0: none
    uint32_t T0;
    uint32_t shift;
    uint32_t pad[12];
};
static_assert(sizeof(Hint) == 64, "Hint layout");

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
    const Hint* hint;       // one sampled tensor: the previous call's threshold
    uint64_t hint_tag;      // ... used when its tag equals this (0: never)
    uint32_t stall;         // test hook: Ctrl::stall
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
        if (p.hint != nullptr && p.hint_tag != 0) {
            const Hint h = *p.hint;
            if (h.tag == p.hint_tag) {
                if (tid == 0) {
                    SegMeta sm;
                    memset(&sm, 0, sizeof(sm));
                    sm.off = off;
                    sm.n = n;
                    sm.out_base = p.out_base[l];
                    sm.k = p.k[l];
                    sm.T0 = h.T0;
                    sm.shift = h.shift;
                    p.meta[l] = sm;
                }
                return;
            }
        }
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
            c.stall = p.stall;
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

}  // namespace tke
