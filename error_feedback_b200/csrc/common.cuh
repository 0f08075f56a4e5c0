// Device helpers shared by the Top-k + error-feedback kernels.
//
// |x| order: key(x) = bits(x) & 0x7FFFFFFF compared as an unsigned integer,
// with every NaN mapped to 0x7FFFFFFF.  This equals the order of |x| for every
// non-NaN value (-0 == +0) and puts all NaNs, as one value, above +Inf, so "the k entries of largest absolute value" ("A
// Distributed Synchronous SGD Algorithm with Global Top-k Sparsification for
// Low Bandwidth Networks", ABSTRACT) is a total order once ties go to the
// lower index.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tke {

constexpr uint32_t KEY_MASK = 0x7FFFFFFFu;
constexpr uint32_t DEAD = 0xFFFFFFFFu;      // empty slot of a merged list
constexpr uint32_t NO_KEY = 0xFFFFFFFFu;    // threshold above every key

// Radix digits of the 31-bit key: 11 + 10 + 10 bits.
constexpr int D1_BITS = 11, D2_BITS = 10, D3_BITS = 10;
constexpr int D1_BINS = 1 << D1_BITS;       // key >> 20
constexpr int D2_BINS = 1 << D2_BITS;       // (key >> 10) & 1023
constexpr int D3_BINS = 1 << D3_BITS;       // key & 1023

// Relative digits of a prefiltered candidate (key >= T0 of its tensor):
//   rel = key - T0;  R1 = min(rel >> s, 4095);  R2 = rel & (2^s - 1)
// with a per-tensor shift s <= 12; R1 = 4095 collects everything above the
// covered range.
constexpr int REL_BINS = 4096;
constexpr int REL_MAX_SHIFT = 12;

// Per-tensor histogram words of the compress workspace.
constexpr int CH_R1 = 0;                        // candidates, relative digit 1
constexpr int CH_R2 = CH_R1 + REL_BINS;         // candidates in the k-th key's R1 bin, R2
constexpr int CH_D1 = CH_R2 + REL_BINS;         // residual rescan, digit 1
constexpr int CH_D2 = CH_D1 + D1_BINS;          // residual rescan, digit 2
constexpr int CH_D3 = CH_D2 + D2_BINS;          // residual rescan, digit 3
constexpr int CHIST_WORDS = CH_D3 + D3_BINS;    // 12,288
// Per-pair histogram words of the merge workspace.
constexpr int MH_D1 = 0, MH_D2 = D1_BINS, MH_D3 = D1_BINS + D2_BINS;
constexpr int MHIST_WORDS = D1_BINS + D2_BINS + D3_BINS;   // 4,096

// Device status bits (ctrl.status).
constexpr uint32_t ST_TIMEOUT = 1u;
constexpr uint32_t ST_BAD_INPUT = 2u;
constexpr uint32_t ST_INCONSISTENT = 4u;    // a count did not add up

// Bounded waits: iterations of ~64 ns sleeps before a wait gives up.
constexpr uint32_t SPIN_LIMIT = 1u << 22;
// ... and the time after which a grid barrier gives up, whichever comes first.
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;

// Control block at the start of every workspace.
struct Ctrl {
    uint32_t status;
    uint32_t mode;          // compress: 0 prefilter path, 1 rescan fallback
    uint32_t tile_ticket;   // dynamic tile counter of the streaming pass
    uint32_t bar;           // grid barrier counter of the select kernel
    uint64_t cand_total;    // candidates kept by the prefilter
    uint64_t cap;           // candidate capacity
    uint32_t kernels;       // kernels the call launched
    uint32_t r2_path;       // compress: a tensor's k-th bin was too full for its entry list
    uint32_t merge_bar[32]; // grid barrier counters, one per merge round
    uint32_t stall;         // test hook: extra arrivals the flat select's barrier waits for
    uint32_t path_small;    // SK_PATH_TAG: the last call was small_kernel's (status below)
    uint64_t sk_status;     // small_kernel: call tag (high half) and ST_* bits
    uint32_t sk_tag;        // small_kernel: the last call's tag (low half)
    uint32_t pad1;
    uint64_t t_phase[8];    // select kernel: globaltimer at each phase (block 0)
    uint64_t t_span[8];     // globaltimer over all blocks (diagnostics): the first
                            // block of a kernel stores ~t (atomicMax of the
                            // complement), the last one t; SPAN_* below
};
static_assert(sizeof(Ctrl) == 320, "Ctrl layout");

// Slots of Ctrl::t_span.
constexpr int SPAN_STREAM_FIRST = 0;   // streaming pass: first block past its wait on the setup
constexpr int SPAN_STREAM_LAST = 1;    // streaming pass: last block done
constexpr int SPAN_SELECT_FIRST = 2;   // select / threshold kernel: first block started
constexpr int SPAN_SELECT_LAST = 3;    // select / threshold kernel: last block done
constexpr int SPAN_GATHER_LAST = 4;    // its last block done gathering candidates
constexpr int SPAN_BAR2_LAST = 5;      // its last block at the barrier after the entry lists
constexpr int SPAN_OFFSET_LAST = 6;    // its last block with its output offset known
constexpr int SPAN_START_LAST = 7;     // its last block started

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void span_first(Ctrl* c, int i) {
    atomicMax(reinterpret_cast<unsigned long long*>(&c->t_span[i]), ~(unsigned long long)global_ns());
}
__device__ __forceinline__ void span_last(Ctrl* c, int i) {
    atomicMax(reinterpret_cast<unsigned long long*>(&c->t_span[i]), (unsigned long long)global_ns());
}

// Every NaN gets the largest key (NaN payloads are implementation-defined:
// an fma on the GPU returns the canonical NaN, other sources may not).
__device__ __forceinline__ uint32_t key_of(float x) {
    const uint32_t k = __float_as_uint(x) & KEY_MASK;
    return k > 0x7F800000u ? KEY_MASK : k;
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Streaming 128-bit loads/stores (the data is touched once).
__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4* p, float4 v) { __stcs(p, v); }

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v) {
    const uint32_t lane = lane_id();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= (uint32_t)o) v += t;
    }
    return v;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Block-wide exclusive scan.  s must hold 33 elements of shared memory.
// Returns the exclusive prefix of v; *total receives the block sum.  Ends
// with a __syncthreads so s may be reused right after.
template <typename T>
__device__ __forceinline__ T block_excl_scan(T v, T* s, T* total) {
    const uint32_t lane = lane_id(), warp = warp_id();
    const uint32_t nwarps = (blockDim.x + 31) >> 5;
    T incl = warp_incl_scan(v);
    if (lane == 31) s[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        T w = lane < nwarps ? s[lane] : T(0);
        T wi = warp_incl_scan(w);
        if (lane < nwarps) s[lane] = wi - w;
        if (lane == 31) s[32] = wi;
    }
    __syncthreads();
    T r = s[warp] + incl - v;
    *total = s[32];
    __syncthreads();
    return r;
}

template <typename T>
__device__ __forceinline__ T block_sum(T v, T* s) {
    T tot;
    block_excl_scan(v, s, &tot);
    return tot;
}

// Grid-wide barrier for a co-resident grid.  `counter` starts at 0 for the
// launch and only grows; `epoch` counts the barriers this block has passed.
// Gives up after SPIN_LIMIT waits or WAIT_LIMIT_NS, whichever comes first,
// records ST_TIMEOUT and returns false: every block then leaves the kernel.
// `extra` arrivals beyond the grid are waited for in addition (0; a test
// hook sets 1 so that the wait runs out).
__device__ __forceinline__ bool grid_barrier(uint32_t* counter, uint32_t& epoch,
                                             uint32_t* status, int* s_flag, uint32_t extra = 0) {
    __syncthreads();
    if (threadIdx.x == 0) {
        epoch += 1;
        const uint32_t target = epoch * gridDim.x + extra;
        // release: the block's writes (ordered before by the block barrier)
        // are visible to whoever acquires the count
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
        uint32_t it = 0;
        int ok = 1;
        uint64_t t0 = 0;
        while (ld_acquire_u32(counter) < target) {
            ++it;
            if (it == 33) t0 = global_ns();
            if (it > SPIN_LIMIT || (it > 33 && (it & 63u) == 0 && global_ns() - t0 > WAIT_LIMIT_NS)) {
                atomicOr(status, ST_TIMEOUT);
                ok = 0;
                break;
            }
            if (it > 32) __nanosleep(64);   // poll back to back at first
        }
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Find, in a histogram of nb bins (bin order = key order), the bin holding
// the rem-th largest element (1-based) counting from the top bin down.
// Executed by one full warp; every lane gets the result.
//   bin   : the bin
//   above : number of elements in bins above it
//   cnt   : elements in the bin
// Returns false when the histogram holds fewer than rem elements.
__device__ __forceinline__ bool warp_find_bin(const uint32_t* h, int nb, uint32_t rem,
                                              uint32_t& bin, uint32_t& above,
                                              uint32_t& cnt) {
    const uint32_t lane = lane_id();
    const int per = nb >> 5;                       // bins per lane (power of two)
    const int hi = nb - (int)lane * per;           // lane 0 owns the top bins
    const int lo = hi - per;
    uint32_t s = 0;
    // rotated walk: lanes start at different banks
    for (int i = 0; i < per; ++i) s += h[lo + ((i + (int)lane) & (per - 1))];
    uint32_t incl = warp_incl_scan(s);
    uint32_t excl = incl - s;
    uint32_t hit = __ballot_sync(0xFFFFFFFFu, incl >= rem);
    if (hit == 0) {
        bin = 0;
        above = __shfl_sync(0xFFFFFFFFu, incl, 31);
        cnt = 0;
        return false;
    }
    const uint32_t src = __ffs(hit) - 1;
    uint32_t rbin = 0, rabove = 0, rcnt = 0;
    if (lane == src) {
        uint32_t run = excl;
        for (int b = hi - 1; b >= lo; --b) {
            uint32_t c = h[b];
            if (run + c >= rem) {
                rbin = (uint32_t)b;
                rabove = run;
                rcnt = c;
                break;
            }
            run += c;
        }
    }
    bin = __shfl_sync(0xFFFFFFFFu, rbin, src);
    above = __shfl_sync(0xFFFFFFFFu, rabove, src);
    cnt = __shfl_sync(0xFFFFFFFFu, rcnt, src);
    return true;
}

struct FindResult {
    uint32_t bin, above, cnt, ok;
};

// Block-wide version of warp_find_bin over a shared-memory histogram of nb
// bins (nb a multiple of blockDim.x, both powers of two).  Every thread of
// the block must call it; the result is in *out after it returns.
__device__ __forceinline__ void block_find_bin(const uint32_t* h, int nb, uint32_t rem,
                                               uint32_t* s_red, FindResult* out) {
    const int t = threadIdx.x;
    const int per = nb / (int)blockDim.x;
    const int hi = nb - t * per;   // thread 0 owns the top bins
    const int lo = hi - per;
    uint32_t s = 0;
    for (int i = 0; i < per; ++i) s += h[lo + ((i + t) & (per - 1))];
    if (t == 0) out->ok = 0;
    uint32_t tot;
    const uint32_t ex = block_excl_scan(s, s_red, &tot);
    if (ex < rem && ex + s >= rem) {
        uint32_t run = ex;
        for (int b = hi - 1; b >= lo; --b) {
            const uint32_t c = h[b];
            if (run + c >= rem) {
                out->bin = (uint32_t)b;
                out->above = run;
                out->cnt = c;
                out->ok = 1;
                break;
            }
            run += c;
        }
    }
    if (tot < rem && t == 0) {
        out->bin = 0;
        out->above = tot;
        out->cnt = 0;
    }
    __syncthreads();
}

// One warp: the bin of the rem-th largest in an NB-bin shared-memory
// histogram (NB a multiple of 1024).  Lane l sums the W = NB / 32 bins
// [NB - W (l + 1), NB - W l) (rotated so that no two lanes hit one bank); a
// scan finds the lane whose bins hold it, then scans over that lane's bins,
// 32 at a time from the top, the bin.  Every lane gets the result; false
// when the histogram holds fewer than rem.  No block barrier.
template <int NB>
__device__ __forceinline__ bool warp_find(const uint32_t* h, uint32_t rem, uint32_t& bin,
                                          uint32_t& above) {
    constexpr int W = NB / 32;
    static_assert(W % 32 == 0, "whole bank rows per lane");
    const uint32_t lane = lane_id();
    const int lo = NB - W * ((int)lane + 1);
    uint32_t s = 0;
#pragma unroll 8
    for (int j = 0; j < W; ++j) s += h[lo + ((j + (int)lane) & (W - 1))];
    const uint32_t incl = warp_incl_scan(s);
    const uint32_t who = __ballot_sync(0xFFFFFFFFu, incl - s < rem && incl >= rem);
    if (!who) return false;
    const int src = __ffs(who) - 1;
    uint32_t run = __shfl_sync(0xFFFFFFFFu, incl - s, src);
    const int top = NB - W * src - 1;
    for (int c0 = 0; c0 < W; c0 += 32) {
        const uint32_t cnt = h[top - c0 - (int)lane];
        const uint32_t inc2 = run + warp_incl_scan(cnt);
        const uint32_t who2 = __ballot_sync(0xFFFFFFFFu, inc2 - cnt < rem && inc2 >= rem);
        if (who2) {
            const int src2 = __ffs(who2) - 1;
            bin = (uint32_t)(top - c0 - src2);
            above = __shfl_sync(0xFFFFFFFFu, inc2 - cnt, src2);
            return true;
        }
        run = __shfl_sync(0xFFFFFFFFu, inc2, 31);
    }
    return false;
}

// Shared-memory histogram increment, aggregated over the lanes of a warp
// that hit the same bin (the active lanes are given by `active`).
__device__ __forceinline__ void warp_agg_inc(uint32_t* h, uint32_t bin, bool active) {
    const uint32_t act = __ballot_sync(0xFFFFFFFFu, active);
    if (!active) return;
    const uint32_t peers = __match_any_sync(act, bin);
    if ((uint32_t)(__ffs(peers) - 1) == lane_id()) atomicAdd(&h[bin], (uint32_t)__popc(peers));
}

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) {
    return (a + b - 1) / b;
}

}  // namespace tke
