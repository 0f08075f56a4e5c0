// Segmented exact top-k selection and ordered emission.
//
// Input: a sequence of (index, value) positions split into segments (tensors
// of a bucket, or the merged lists of the merge's pairs), each with its own
// k.  For every segment the kernel finds the key T of its k-th element in the
// order (|value| desc, index asc) and the tie quota q = k - #{key > T}, and
// writes the selected entries in index order:
//     selected = {key > T} + the first q positions (in index order) with key == T
// ("A Distributed Synchronous SGD Algorithm with Global Top-k Sparsification",
// ABSTRACT: the k largest absolute values; lower index first among equal
// magnitudes makes the set unique.)
//
// T is found by radix digits of the 31-bit key.  Standard digits are 11 + 10
// + 10 bits (merge rounds, and the compress step's rescan of the residual).
// A prefiltered tensor of the compress step instead uses two digits of
// key - T0 (see common.cuh): the gather phase builds the first histogram
// while it copies the candidates into one list in index order; the few
// candidates in the k-th key's first-digit bin then go to a small per-tensor
// entry list from which every block reads T, the tie quota and its own
// output offset, so the candidate path needs three grid barriers in all.
//
// The grid is cooperative (all blocks resident): each block owns one
// contiguous range of positions, histograms are summed in global memory and
// separated by grid barriers, every block resolves the digits of the
// segments it touches, and the output offsets come from per-block counts
// exchanged through one more barrier.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "kernels_compress.cuh"
#include "kernels_stream.cuh"

namespace tke {

constexpr int SEL_THREADS = 512;
constexpr int SEG_MAX = 256;
constexpr int EMIT_PER_THREAD = 4;
constexpr int EMIT_TILE = SEL_THREADS * EMIT_PER_THREAD;
// Entry list of a prefiltered tensor: candidates in the bin of relative digit
// 1 that holds the k-th key, as (block << 12) | relative digit 2.
constexpr uint32_t ENT_PER = 4096;
// Tiles of more than WT_THREAD candidates a warp gathers at once.
constexpr int OVF_U = 4;
// Rescan queue of the hard-threshold step: 16-byte entries (tile + 1, 0,
// output position) in the per-tensor histogram words, which that step does
// not use.
constexpr uint32_t RQ_CAP = (uint32_t)CHIST_WORDS / 4;
// Its counters (slots reserved, slots handed out, blocks done queueing) in
// words of the control block that only merge calls use otherwise.
constexpr int RQ_RESERVE = 0, RQ_HEAD = 1, RQ_DONE = 2;

struct Slot {
    int32_t l_first, l_last;
    uint32_t gt_first, eq_first, gt_last, eq_last;
    uint32_t pad[2];
};

// Outcome of resolving some digits of one segment.
struct DigitState {
    uint32_t none;     // k == 0: nothing selected
    uint32_t prefix;   // decided high bits (standard) / T (final)
    uint32_t rem;      // rank still needed inside the prefix class / tie quota
    uint32_t ok;       // 0: the counts did not add up (or relative overflow)
};

// Relative digit 1 of a prefiltered tensor, resolved.
struct RelState {
    uint32_t b1;    // bin of the k-th key
    uint32_t rem;   // rank of the k-th key inside the bin
    uint32_t cnt;   // candidates in the bin
    uint32_t ok;    // 0: k == 0, or the counts did not add up
};

struct SelShared {
    int64_t seg[SEG_MAX + 1];
    __align__(16) uint32_t stage[REL_BINS];
    uint32_t h1[D1_BINS];
    uint64_t scan[33];
    uint32_t red[33];
    uint32_t T0[SEG_MAX];
    uint32_t shift[SEG_MAX];
    FindResult fr;
    RelState rs[2];            // first and last segment of the block's range
    RelState rs_early;         // one tensor, digit 1 built by the streaming pass
    uint32_t top_bin;          // its candidates in the top relative bin (overflow)
    DigitState ds;
    DigitState fin[2];         // final thresholds of the first and last segment
    int flag;
    uint32_t pre[4];
    uint64_t ovf_pos[SEL_THREADS];   // gather: output position of each overflow tile
    uint64_t before;                 // gather: output offset of the block
    uint64_t total;                  // gather (look-all): candidates of all blocks
};

// Block-wide copy of n words (n a multiple of 4, 16-byte aligned) into
// shared memory, zero-padded up to `pad` words.
__device__ __forceinline__ void stage_words(uint32_t* dst, const uint32_t* src, int n, int pad) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = threadIdx.x; i < n / 4; i += blockDim.x) d4[i] = s4[i];
    for (int i = n + threadIdx.x; i < pad; i += blockDim.x) dst[i] = 0;
}

// Standard digits 1..upto of a segment with histograms h1, h2, h3.
__device__ void resolve_std(const uint32_t* h1, const uint32_t* h2, const uint32_t* h3,
                            uint32_t k, int upto, SelShared& S, uint32_t* status) {
    __syncthreads();
    if (k == 0 || upto == 0) {
        if (threadIdx.x == 0) S.ds = DigitState{k == 0 ? 1u : 0u, 0u, k, 1u};
        __syncthreads();
        return;
    }
    uint32_t rem = k, prefix = 0, ok = 1;
    stage_words(S.stage, h1, D1_BINS, D1_BINS);
    __syncthreads();
    block_find_bin(S.stage, D1_BINS, rem, S.red, &S.fr);
    ok = S.fr.ok;
    rem -= S.fr.above;
    prefix = S.fr.bin;
    if (upto >= 2 && ok) {
        __syncthreads();
        stage_words(S.stage, h2, D2_BINS, D2_BINS);
        __syncthreads();
        block_find_bin(S.stage, D2_BINS, rem, S.red, &S.fr);
        ok = S.fr.ok;
        rem -= S.fr.above;
        prefix = (prefix << D2_BITS) | S.fr.bin;
    }
    if (upto >= 3 && ok) {
        __syncthreads();
        stage_words(S.stage, h3, D3_BINS, D3_BINS);
        __syncthreads();
        block_find_bin(S.stage, D3_BINS, rem, S.red, &S.fr);
        ok = S.fr.ok;
        rem -= S.fr.above;
        prefix = (prefix << D3_BITS) | S.fr.bin;
    }
    if (threadIdx.x == 0) {
        S.ds = DigitState{0u, prefix, rem, ok};
        if (!ok) atomicOr(status, ST_INCONSISTENT);
    }
    __syncthreads();
}

// Relative digit 1 of a prefiltered tensor from its global histogram r1.
// ... from the histogram already in S.stage.
__device__ RelState rel1_from_stage(uint32_t k, SelShared& S) {
    if (k == 0) return RelState{0u, 0u, 0u, 0u};
    block_find_bin(S.stage, REL_BINS, k, S.red, &S.fr);
    const RelState r{S.fr.bin, k - S.fr.above, S.fr.cnt,
                     (S.fr.ok && S.fr.bin != REL_BINS - 1) ? 1u : 0u};
    __syncthreads();
    return r;
}

__device__ RelState resolve_rel1(const uint32_t* r1, uint32_t k, SelShared& S) {
    __syncthreads();
    if (k == 0) return RelState{0u, 0u, 0u, 0u};
    stage_words(S.stage, r1, REL_BINS, REL_BINS);
    __syncthreads();
    return rel1_from_stage(k, S);
}

// T (prefix) and the tie quota (rem) from the relative digit-2 histogram h2
// (shared memory, REL_BINS words) of the k-th key's digit-1 bin.
__device__ DigitState finish_rel(const uint32_t* h2, const RelState& rs, uint32_t T0,
                                 uint32_t sh, SelShared& S) {
    block_find_bin(h2, REL_BINS, rs.rem, S.red, &S.fr);
    const DigitState d{0u, T0 + (rs.b1 << sh) + S.fr.bin, rs.rem - S.fr.above, S.fr.ok};
    __syncthreads();
    return d;
}

// ---------------------------------------------------------------- sources

// Compress: candidates of the streaming pass, or the whole residual.  The
// generic digit passes below run only for the rescan of the residual.
struct CompressSrc {
    float* resid;
    int64_t N;
    int32_t T;
    const SegMeta* meta;
    int64_t* cand_start;         // [T+1], built by the gather phase
    uint32_t* cand_idx;          // dense candidate list, index order
    float* cand_val;
    uint64_t cap;
    uint32_t* hist;              // [T][CHIST_WORDS]
    int32_t* out_idx;
    float* out_val;
    uint32_t num_wt;             // warp tiles of the streaming pass
    const uint32_t* wt_count;
    const uint16_t* wt_off;      // [num_wt][WT_CAP]
    uint32_t* ent;               // [T][ENT_PER] entry lists
    uint32_t* ent_cnt;           // [T] their lengths
    uint64_t* agg;               // [grid] each block's candidate count + 1 (0: not yet)
    int32_t r1_done;             // one tensor: the streaming pass built relative digit 1
    uint4* rq;                   // hard threshold: rescan queue [RQ_CAP] (null: none)
    int32_t force_dense;
    int32_t dense;               // decided inside the kernel

    __device__ int nseg() const { return T; }
    __device__ int64_t seg_bound(int l) const { return dense ? (l < T ? meta[l].off : N) : cand_start[l]; }
    __device__ uint32_t seg_k(int l) const { return meta[l].k; }
    __device__ uint32_t* h(int l, int part) const { return hist + (size_t)l * CHIST_WORDS + part; }
    __device__ bool uses_std(int) const { return true; }
    // the k-th key lies above the range of the relative digits
    __device__ bool rel_overflow(int l) const {
        const uint32_t k = meta[l].k;
        return k > 0 && h(l, CH_R1)[REL_BINS - 1] >= k;
    }
    __device__ uint32_t* d1(int l) const { return h(l, CH_D1); }
    __device__ uint32_t* d2(int l) const { return h(l, CH_D2); }
    __device__ uint32_t* d3(int l) const { return h(l, CH_D3); }
    __device__ void load(int64_t pos, uint32_t& idx, float& val) const {
        if (dense) { idx = (uint32_t)pos; val = resid[pos]; }
        else { idx = cand_idx[pos]; val = cand_val[pos]; }
    }
    __device__ void emit(int l, uint32_t rank, uint32_t idx, float val) const {
        const SegMeta& m = meta[l];
        out_idx[m.out_base + rank] = (int32_t)((int64_t)idx - m.off);
        out_val[m.out_base + rank] = val;
        resid[idx] = 0.0f;
    }
    __device__ void resolve_final(int l, SelShared& S, uint32_t* status) const {
        resolve_std(d1(l), d2(l), d3(l), seg_k(l), 3, S, status);
    }
};

// Merge round: merged lists of the pairs (DEAD marks empty slots).
struct MergeSrc {
    const uint32_t* m_idx;
    const float* m_val;
    int64_t mcap;                // positions per segment
    int32_t T;                   // segments (pairs)
    const uint32_t* live;        // [T] entries in each merged list (or null)
    uint32_t live_const;         // used when live is null
    uint32_t kmax;
    uint32_t* hist;              // [T][MHIST_WORDS]
    int32_t dense;               // always 0
    int32_t d1_done;             // the merge kernel already built digit 1
    int32_t final_out;
    int32_t* out_idx;            // final: the caller's arrays
    float* out_val;
    int32_t* out_count;
    int64_t out_k;
    uint32_t* set_idx;           // otherwise: the sets buffer
    float* set_val;
    int64_t set_cap;
    uint32_t* sizes;
    int32_t pair_stride;         // 2^(r+1)
    const uint32_t* bad_words;   // first select launch: input verdicts to fold
    int32_t n_bad;

    __device__ int nseg() const { return T; }
    __device__ int64_t seg_bound(int l) const { return (int64_t)l * mcap; }
    __device__ uint32_t seg_k(int l) const {
        const uint32_t lv = live ? live[l] : live_const;
        return lv < kmax ? lv : kmax;
    }
    __device__ bool uses_std(int) const { return true; }
    __device__ uint32_t* d1(int l) const { return hist + (size_t)l * MHIST_WORDS + MH_D1; }
    __device__ uint32_t* d2(int l) const { return hist + (size_t)l * MHIST_WORDS + MH_D2; }
    __device__ uint32_t* d3(int l) const { return hist + (size_t)l * MHIST_WORDS + MH_D3; }
    __device__ void load(int64_t pos, uint32_t& idx, float& val) const {
        idx = m_idx[pos];
        val = m_val[pos];
    }
    __device__ void emit(int l, uint32_t rank, uint32_t idx, float val) const {
        if (final_out) {
            out_idx[rank] = (int32_t)idx;
            out_val[rank] = val;
        } else {
            const int64_t s = (int64_t)l * pair_stride * set_cap + rank;
            set_idx[s] = idx;
            set_val[s] = val;
        }
    }
    __device__ void resolve_final(int l, SelShared& S, uint32_t* status) const {
        resolve_std(d1(l), d2(l), d3(l), seg_k(l), 3, S, status);
    }
    __device__ void fold_bad_input(Ctrl* ctrl) const {
        if (bad_words && blockIdx.x == 0 && threadIdx.x == 0) {
            uint32_t any = 0;
            for (int i = 0; i < n_bad; ++i) any |= bad_words[i];
            if (any) atomicOr(&ctrl->status, ST_BAD_INPUT);
        }
    }
    // Block 0: result lengths (and the padding of the caller's arrays).
    __device__ void finalize_block0() const {
        if (final_out) {
            const uint32_t k0 = seg_k(0);
            if (threadIdx.x == 0) *out_count = (int32_t)k0;
            for (int64_t i = (int64_t)k0 + threadIdx.x; i < out_k; i += blockDim.x) {
                out_idx[i] = -1;
                out_val[i] = 0.0f;
            }
        } else {
            for (int l = threadIdx.x; l < T; l += blockDim.x)
                sizes[(int64_t)l * pair_stride] = seg_k(l);
        }
    }
};

struct SelCommon {
    Ctrl* ctrl;
    uint32_t* bar;
    Slot* slots;
};

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ int seg_of_pos(const int64_t* s_seg, int T, int64_t p) {
    // largest l < T with s_seg[l] <= p
    int lo = 0, hi = T;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_seg[mid] <= p) lo = mid; else hi = mid;
    }
    return lo;
}

// digit d (1..3) of a key, and whether the key lies in the class decided by
// the first d-1 digits (prefix)
__device__ __forceinline__ uint32_t digit_of(uint32_t key, int d) {
    return d == 1 ? (key >> 20) : (d == 2 ? ((key >> 10) & (D2_BINS - 1)) : (key & (D3_BINS - 1)));
}
__device__ __forceinline__ bool in_class(uint32_t key, int d, uint32_t prefix) {
    return d == 1 ? true : (d == 2 ? ((key >> 20) == prefix) : ((key >> 10) == prefix));
}

// Phase timestamps (block 0 only) for the diagnostics call.
__device__ __forceinline__ void mark_phase(Ctrl* ctrl, int i) {
    if (blockIdx.x == 0 && threadIdx.x == 0) ctrl->t_phase[i] = global_ns();
}
// The same phase, latest over all blocks.
__device__ __forceinline__ void mark_last(Ctrl* ctrl, int slot) {
    if (threadIdx.x == 0) span_last(ctrl, slot);
}

// First start and last end over the blocks of a select-type kernel (thread 0
// of each block; its end is stamped on every return path).
struct BlockSpan {
    Ctrl* c;
    __device__ explicit BlockSpan(Ctrl* ctrl) : c(ctrl) {
        if (threadIdx.x == 0) {
            span_first(c, SPAN_SELECT_FIRST);
            span_last(c, SPAN_START_LAST);
        }
    }
    __device__ ~BlockSpan() {
        if (threadIdx.x == 0) span_last(c, SPAN_SELECT_LAST);
    }
};

// Output offset of a block inside segment l from the blocks before it: the
// (gt, eq) counts of the run of earlier blocks whose ranges continue l (their
// slots), summed by warp 0, which loads the slots of 128 blocks at a time.
// Result in S.pre[0..1].
__device__ void chain_prefix(const SelCommon& cm, int c, int l, SelShared& S) {
    constexpr int U = 4;
    if (threadIdx.x < 32) {
        const uint32_t lane = lane_id();
        uint32_t pg = 0, pe = 0;
        bool done = false;
        for (int c0 = c - 1; !done; c0 -= 32 * U) {
            int lf[U], ll[U];
            uint32_t g[U], e[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = c0 - 32 * u - (int)lane;
                lf[u] = ll[u] = -1;
                g[u] = e[u] = 0;
                if (j >= 0) {
                    const uint4* q = reinterpret_cast<const uint4*>(cm.slots + j);
                    const uint4 a = q[0], b = q[1];
                    lf[u] = (int)a.x;
                    ll[u] = (int)a.y;
                    g[u] = b.x;    // gt_last
                    e[u] = b.y;    // eq_last
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (done) continue;
                const bool match = ll[u] == l;
                const bool cont = match && lf[u] == l;
                const uint32_t contm = __ballot_sync(0xFFFFFFFFu, cont);
                const uint32_t matchm = __ballot_sync(0xFFFFFFFFu, match);
                const uint32_t run = (contm == 0xFFFFFFFFu) ? 32u : (uint32_t)(__ffs(~contm) - 1);
                const bool take = lane < run || (lane == run && ((matchm >> run) & 1u));
                pg += warp_sum(take ? g[u] : 0u);
                pe += warp_sum(take ? e[u] : 0u);
                if (run < 32) done = true;
            }
        }
        if (threadIdx.x == 0) {
            S.pre[0] = pg;
            S.pre[1] = pe;
        }
    }
    __syncthreads();
}

// Ordered emission of positions [a, b) of segment l: key > Tk always, key ==
// Tk while the tie quota q lasts; run_gt / run_eq are the counts of both
// classes at positions of l before a.
template <class Src>
__device__ void emit_range(const Src& src, int l, int64_t a, int64_t b, uint32_t Tk, uint32_t q,
                           uint32_t kseg, uint32_t run_gt, uint32_t run_eq, SelShared& S) {
    const int tid = threadIdx.x;
    for (int64_t base = a; base < b; base += EMIT_TILE) {
        uint32_t idx[EMIT_PER_THREAD];
        float val[EMIT_PER_THREAD];
        uint32_t cls = 0;   // bit u: gt, bit 4+u: eq
#pragma unroll
        for (int u = 0; u < EMIT_PER_THREAD; ++u) {
            const int64_t pos = base + (int64_t)tid * EMIT_PER_THREAD + u;
            idx[u] = DEAD;
            val[u] = 0.f;
            if (pos < b) src.load(pos, idx[u], val[u]);
            if (idx[u] != DEAD) {
                const uint32_t key = key_of(val[u]);
                if (key > Tk) cls |= 1u << u;
                else if (key == Tk) cls |= 1u << (4 + u);
            }
        }
        const uint64_t mine = ((uint64_t)__popc(cls & 0xFu) << 32) | (uint64_t)__popc(cls >> 4);
        uint64_t tot;
        const uint64_t ex = block_excl_scan(mine, S.scan, &tot);
        uint32_t g = run_gt + (uint32_t)(ex >> 32);
        uint32_t e = run_eq + (uint32_t)(ex & 0xFFFFFFFFu);
#pragma unroll
        for (int u = 0; u < EMIT_PER_THREAD; ++u) {
            if ((cls >> u) & 1u) {
                const uint32_t rank = g + (e < q ? e : q);
                if (rank < kseg) src.emit(l, rank, idx[u], val[u]);
                ++g;
            } else if ((cls >> (4 + u)) & 1u) {
                if (e < q) {
                    const uint32_t rank = g + e;
                    if (rank < kseg) src.emit(l, rank, idx[u], val[u]);
                }
                ++e;
            }
        }
        run_gt += (uint32_t)(tot >> 32);
        run_eq += (uint32_t)(tot & 0xFFFFFFFFu);
    }
}

// ------------------------------------------------ compress candidate path

// Relative digit-1 bin of a candidate of tensor l (key >= T0 of l).
__device__ __forceinline__ uint32_t rel_bin(uint32_t key, uint32_t T0, uint32_t sh) {
    return min((key - T0) >> sh, (uint32_t)(REL_BINS - 1));
}

__device__ __forceinline__ void r1_add(const CompressSrc& src, const SelShared& S, int l,
                                       float v, uint32_t* s_r1) {
    const uint32_t bin = rel_bin(key_of(v), S.T0[l], S.shift[l]);
    if (s_r1) atomicAdd(&s_r1[bin], 1u);
    else atomicAdd(src.h(l, CH_R1) + bin, 1u);
}

// Staged candidates of one warp tile, held by one thread: offsets (distinct,
// slots >= cnt hold 0xFFFF, above every offset) and the values read back
// from the residual (which holds acc).
struct TileCands {
    uint32_t o[WT_THREAD];
    float v[WT_THREAD];
};

// The offsets: their loads do not depend on the count (the slots past it
// hold stale data, masked by load_values), so they are issued together with
// the load of the count.
__device__ __forceinline__ void load_staged(const CompressSrc& src, uint32_t w, TileCands& t) {
    const uint4* p4 = reinterpret_cast<const uint4*>(src.wt_off + (size_t)w * WT_CAP);
    const uint4 a = p4[0], b = p4[1];
    t.o[0] = a.x & 0xFFFFu; t.o[1] = a.x >> 16; t.o[2] = a.y & 0xFFFFu; t.o[3] = a.y >> 16;
    t.o[4] = a.z & 0xFFFFu; t.o[5] = a.z >> 16; t.o[6] = a.w & 0xFFFFu; t.o[7] = a.w >> 16;
    t.o[8] = b.x & 0xFFFFu; t.o[9] = b.x >> 16; t.o[10] = b.y & 0xFFFFu; t.o[11] = b.y >> 16;
    t.o[12] = b.z & 0xFFFFu; t.o[13] = b.z >> 16; t.o[14] = b.w & 0xFFFFu; t.o[15] = b.w >> 16;
}

// The values of the first cnt slots (cnt <= WT_THREAD; none for a larger
// tile, which a warp gathers), and the masking of the other slots.
__device__ __forceinline__ void load_values(const CompressSrc& src, uint32_t w, uint32_t cnt,
                                            TileCands& t) {
    const int64_t base = (int64_t)w * WT;
    const uint32_t c = cnt <= (uint32_t)WT_THREAD ? cnt : 0u;
#pragma unroll
    for (int i = 0; i < WT_THREAD; ++i) {
        if ((uint32_t)i < c) {
            t.v[i] = src.resid[base + t.o[i]];
        } else {
            t.o[i] = 0xFFFFu;
            t.v[i] = 0.f;
        }
    }
}

// Write the staged candidates of warp tile w in index order (ranked by
// offset) from position pos of the dense list, and add each to the relative
// digit-1 histogram of its tensor: s_r1 (shared) when the caller's chunk
// lies in tensor lc, else the global one.  S.seg holds element offsets.
// In threshold mode (kThr) the dense list is the caller's output: a written
// candidate is sent, so its residual becomes +0.0f, and there is no
// histogram.
template <int C, bool kThr>
__device__ __forceinline__ void store_ranked(const CompressSrc& src, SelShared& S,
                                             uint32_t w, uint64_t pos, uint32_t cnt,
                                             const TileCands& t, uint32_t* s_r1, int lc) {
    const int64_t base = (int64_t)w * WT;
#pragma unroll
    for (int i = 0; i < C; ++i) {
        if ((uint32_t)i >= cnt) continue;
        uint32_t rank = 0;
#pragma unroll
        for (int j = 0; j < C; ++j) rank += t.o[j] < t.o[i];
        const int64_t e = base + t.o[i];
        const uint64_t q = pos + rank;
        if (q < src.cap) {
            src.cand_idx[q] = (uint32_t)e;
            src.cand_val[q] = t.v[i];
            if (kThr) src.resid[e] = 0.0f;
        }
        if (!kThr && !src.r1_done) r1_add(src, S, s_r1 ? lc : seg_of(S.seg, src.T, e), t.v[i], s_r1);
    }
}

// Published count (+1) of block j, waited for: every block publishes before
// any heavy work and all blocks are resident, so the wait is short; it is
// bounded all the same.
__device__ __forceinline__ uint64_t agg_wait(const uint64_t* agg, int j, uint64_t v,
                                             uint32_t* status) {
    uint32_t it = 0;
    while (v == 0) {
        if (++it > SPIN_LIMIT) {
            atomicOr(status, ST_TIMEOUT);
            break;
        }
        if (it > 32) __nanosleep(32);
        v = *reinterpret_cast<const volatile uint64_t*>(agg + j);
    }
    return v ? v - 1 : 0;
}

// Candidates of blocks [0, c) (S.before) and, with `all`, of every block
// (S.total), summed by warp 0 from the published counts.  The loads of a
// round of 8 per lane are issued together.
template <bool all>
__device__ void look_counts(const uint64_t* agg, int c, uint32_t* status, SelShared& S) {
    if (threadIdx.x < 32) {
        const int G = all ? (int)gridDim.x : c;
        uint64_t before = 0, total = 0;
        for (int j0 = 0; j0 < G; j0 += 32 * 8) {
            uint64_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 32 * u + (int)lane_id();
                v[u] = j < G ? *reinterpret_cast<const volatile uint64_t*>(agg + j) : 1u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 32 * u + (int)lane_id();
                if (j >= G) continue;
                const uint64_t cnt = agg_wait(agg, j, v[u], status);
                total += cnt;
                if (j < c) before += cnt;
            }
        }
        before = warp_sum(before);
        total = warp_sum(total);
        if (threadIdx.x == 0) {
            S.before = before;
            S.total = total;
        }
    }
    __syncthreads();
}

// Gather a warp tile with WT_THREAD < cnt <= WT_CAP staged candidates (one
// warp), its offset o and value v already loaded by lane i < cnt (staged
// slot i; 0xFFFF elsewhere): each lane ranks its offset among the others by
// shuffles and writes its candidate.
template <bool kThr>
__device__ __forceinline__ void store_warp_staged(const CompressSrc& src, SelShared& S,
                                                  uint32_t w, uint64_t pos, uint32_t cnt,
                                                  uint32_t o, float v, uint32_t* s_r1, int lc) {
    const uint32_t lane = lane_id();
    uint32_t rank = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) rank += __shfl_sync(0xFFFFFFFFu, o, i) < o;
    if (lane < cnt) {
        const int64_t e = (int64_t)w * WT + o;
        const uint64_t q = pos + rank;
        if (q < src.cap) {
            src.cand_idx[q] = (uint32_t)e;
            src.cand_val[q] = v;
            if (kThr) src.resid[e] = 0.0f;
        }
        if (!kThr && !src.r1_done) r1_add(src, S, s_r1 ? lc : seg_of(S.seg, src.T, e), v, s_r1);
    }
}

__device__ __forceinline__ float f4_get(const float4& v, int t) {
    return t == 0 ? v.x : (t == 1 ? v.y : (t == 2 ? v.z : v.w));
}

// Gather a warp tile with more than WT_CAP candidates (one warp): rescan it
// from the residual (which holds acc) with the streaming pass's test.  A
// full tile with a 16-byte aligned base is read as 8 float4 per lane (lane
// holds elements 128 j + 4 lane + t, so within each j the candidates are in
// index order lane by lane: one warp scan places them); any other tile as 32
// coalesced scalar loads (element 32 u + lane) with one ballot each.  All the
// loads of a tile are issued before the first is used.  Out of line: it runs
// for dense tiles only and keeps its registers to itself.
// What the rescan needs of CompressSrc, passed by value (a reference would
// make the caller keep a copy of the whole source in local memory).
struct RescanArgs {
    float* resid;
    int64_t N;
    uint32_t* cand_idx;
    float* cand_val;
    uint64_t cap;
    uint32_t* hist;
    int32_t T;
    int32_t r1_done;
    __device__ explicit RescanArgs(const CompressSrc& s)
        : resid(s.resid), N(s.N), cand_idx(s.cand_idx), cand_val(s.cand_val), cap(s.cap),
          hist(s.hist), T(s.T), r1_done(s.r1_done) {}
    __device__ void r1_add(const SelShared& S, int l, float v, uint32_t* s_r1) const {
        const uint32_t bin = rel_bin(key_of(v), S.T0[l], S.shift[l]);
        if (s_r1) atomicAdd(&s_r1[bin], 1u);
        else atomicAdd(hist + (size_t)l * CHIST_WORDS + CH_R1 + bin, 1u);
    }
};

template <bool kThr>
__device__ __noinline__ void gather_rescan(const RescanArgs src, SelShared& S, uint32_t w,
                                           uint64_t pos, uint32_t* s_r1, int lc) {
    const uint32_t lane = lane_id();
    const int T = src.T;
    const int64_t base = (int64_t)w * WT;
    const int64_t tend = min(base + (int64_t)WT, src.N);
    const float* tile = src.resid + base;
    if (tend - base == WT && (reinterpret_cast<uintptr_t>(tile) & 15u) == 0) {
        const float4* t4 = reinterpret_cast<const float4*>(tile) + lane;
        float4 v4[WT_VECS];
#pragma unroll
        for (int j = 0; j < WT_VECS; ++j) v4[j] = t4[32 * j];
        int l = lc;
        if (!s_r1) l = seg_of(S.seg, T, base + 4 * (int64_t)lane);
#pragma unroll
        for (int j = 0; j < WT_VECS; ++j) {
            const int64_t e0 = base + 128 * j + 4 * (int64_t)lane;
            const int lj = l;
            uint32_t f = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (!s_r1)
                    while (l < T - 1 && S.seg[l + 1] <= e0 + t) ++l;
                f |= (uint32_t)(key_of(f4_get(v4[j], t)) >= S.T0[l]) << t;
            }
            const uint32_t c = (uint32_t)__popc(f);
            const uint32_t incl = warp_incl_scan(c);
            uint64_t q = pos + incl - c;
            int l2 = lj;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (!s_r1)
                    while (l2 < T - 1 && S.seg[l2 + 1] <= e0 + t) ++l2;
                if ((f >> t) & 1u) {
                    const float a = f4_get(v4[j], t);
                    if (q < src.cap) {
                        src.cand_idx[q] = (uint32_t)(e0 + t);
                        src.cand_val[q] = a;
                        if (kThr) src.resid[e0 + t] = 0.0f;
                    }
                    if (!kThr && !src.r1_done) src.r1_add(S, l2, a, s_r1);
                    ++q;
                }
            }
            pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        return;
    }
    float v[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
        const int64_t e = base + 32 * u + lane;
        v[u] = e < tend ? src.resid[e] : 0.f;
    }
    // tensor of each element: walk forward from the lane's first element
    int l = lc;
    if (!s_r1 && base + (int64_t)lane < tend) l = seg_of(S.seg, T, base + lane);
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
        const int64_t e = base + 32 * u + lane;
        bool f = false;
        if (e < tend) {
            if (!s_r1)
                while (l < T - 1 && S.seg[l + 1] <= e) ++l;
            f = key_of(v[u]) >= S.T0[l];
        }
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, f);
        if (f) {
            const uint64_t q = pos + __popc(m & lt);
            if (q < src.cap) {
                src.cand_idx[q] = (uint32_t)e;
                src.cand_val[q] = v[u];
                if (kThr) src.resid[e] = 0.0f;
            }
            if (!kThr && !src.r1_done) src.r1_add(S, l, v[u], s_r1);
        }
        pos += __popc(m);
    }
}

// Hard threshold: queue tile w (output position pos) for rescanning by any
// warp (one warp, lane 0 writes).  False if the queue is full.
__device__ __forceinline__ bool rq_push(const CompressSrc& src, const SelCommon& cm, uint32_t w,
                                        uint64_t pos) {
    uint32_t slot = 0;
    if (lane_id() == 0) slot = atomicAdd(&cm.ctrl->merge_bar[RQ_RESERVE], 1u);
    slot = __shfl_sync(0xFFFFFFFFu, slot, 0);
    if (slot >= RQ_CAP) return false;
    if (lane_id() == 0) {
        uint32_t* e = reinterpret_cast<uint32_t*>(src.rq + slot);
        e[2] = (uint32_t)pos;
        e[3] = (uint32_t)(pos >> 32);
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(e), "r"(w + 1u) : "memory");
    }
    return true;
}

// Hard threshold: the warp takes queued tiles and rescans them while the
// queue holds untaken ones.  A ticket (atomic add) is taken only when one
// looked free; a ticket whose slot is not reserved yet is kept until its
// slot is filled or every block has finished queueing, so none is lost.  The
// block that queued a tile takes from the queue afterwards itself.
__device__ void rq_drain(const CompressSrc& src, const SelCommon& cm, SelShared& S) {
    uint32_t* head = &cm.ctrl->merge_bar[RQ_HEAD];
    const volatile uint32_t* resv = &cm.ctrl->merge_bar[RQ_RESERVE];
    const uint32_t* done = &cm.ctrl->merge_bar[RQ_DONE];
    for (;;) {
        uint32_t w1 = 0, plo = 0, phi = 0;
        if (lane_id() == 0) {
            const uint32_t r = min(*resv, RQ_CAP);
            const uint32_t h = *reinterpret_cast<volatile uint32_t*>(head);
            if (h < r) {
                const uint32_t t = atomicAdd(head, 1u);
                if (t < RQ_CAP) {
                    const uint32_t* e = reinterpret_cast<const uint32_t*>(src.rq + t);
                    uint32_t it = 0;
                    for (;;) {
                        if ((w1 = ld_acquire_u32(e)) != 0) break;
                        if (ld_acquire_u32(done) == gridDim.x && t >= *resv) break;
                        if (++it > SPIN_LIMIT) {
                            atomicOr(&cm.ctrl->status, ST_TIMEOUT);
                            break;
                        }
                        __nanosleep(32);
                    }
                    if (w1) {
                        plo = e[2];
                        phi = e[3];
                    }
                }
            }
        }
        w1 = __shfl_sync(0xFFFFFFFFu, w1, 0);
        if (w1 == 0) return;
        const uint64_t pos = ((uint64_t)__shfl_sync(0xFFFFFFFFu, phi, 0) << 32) |
                             __shfl_sync(0xFFFFFFFFu, plo, 0);
        gather_rescan<true>(RescanArgs(src), S, w1 - 1u, pos, nullptr, 0);
    }
}

// Candidates of warp tile w below element bound (one thread).
__device__ uint32_t tile_count_below(const CompressSrc& src, const SelShared& S, uint32_t w,
                                     uint32_t cnt, int64_t bound) {
    const int64_t base = (int64_t)w * WT;
    uint32_t c = 0;
    if (cnt <= (uint32_t)WT_CAP) {
        for (uint32_t i = 0; i < cnt; ++i)
            c += base + (int64_t)src.wt_off[(size_t)w * WT_CAP + i] < bound;
    } else {
        for (int64_t e = base; e < bound; ++e)
            c += key_of(src.resid[e]) >= S.T0[seg_of(S.seg, src.T, e)];
    }
    return c;
}

// Gather phase of the compress select.  Each block takes a contiguous chunk
// of warp tiles, publishes its candidate count at once and finds its output
// offset by looking back at the counts of the blocks before it (no grid
// barrier).  It copies its candidates, in index order, to [my0, my1) of the
// dense list (up to WT_THREAD staged ones per tile from registers loaded
// before the look-back; up to WT_CAP by a warp; more by a rescan of the
// tile), builds the relative
// digit-1 histograms (not in threshold mode) and records where each
// tensor's candidates start.
template <bool kThr>
__device__ void gather_phase(CompressSrc& src, const SelCommon& cm, SelShared& S, uint64_t& my0,
                             uint64_t& my1) {
    const int G = gridDim.x, c = blockIdx.x, tid = threadIdx.x;
    const uint32_t warp = warp_id(), nwarps = blockDim.x >> 5;
    const int T = src.T;
    uint32_t* status = &cm.ctrl->status;
    int64_t* s_off = S.seg;
    const uint32_t W = src.num_wt;
    const uint32_t per = (W + G - 1) / G;
    const uint32_t w0 = min((uint32_t)c * per, W), w1 = min(w0 + per, W);
    // the first round's tile of this thread, loaded before anything else
    uint32_t cnt = 0;
    TileCands tc;
    if (w0 + tid < w1) {
        cnt = src.wt_count[w0 + tid];
        load_staged(src, w0 + tid, tc);
    }
    // one tensor whose relative digit 1 the streaming pass built: that
    // histogram too (REL_BINS words, two 16-byte words per thread)
    static_assert(REL_BINS == 8 * SEL_THREADS, "digit-1 histogram load");
    const bool early = !kThr && src.r1_done;
    uint4 r1v[2];
    if (early) {
        const uint4* h4 = reinterpret_cast<const uint4*>(src.h(0, CH_R1));
        r1v[0] = h4[tid];
        r1v[1] = h4[tid + SEL_THREADS];
    }
    for (int l = tid; l < T; l += blockDim.x) {
        s_off[l] = src.meta[l].off;
        S.T0[l] = src.meta[l].T0;
        S.shift[l] = src.meta[l].shift;
    }
    if (tid == 0) s_off[T] = src.N;
    // one round: the block's count is the first scan's total, published
    // there; otherwise it is summed and published first
    const bool single = w1 - w0 <= blockDim.x;
    uint32_t mine = 0;
    if (!single) {
        mine = cnt;
        for (uint32_t w = w0 + tid + blockDim.x; w < w1; w += blockDim.x) mine += src.wt_count[w];
        mine = block_sum(mine, S.red);
        if (tid == 0) *reinterpret_cast<volatile uint64_t*>(src.agg + c) = (uint64_t)mine + 1;
    }

    // relative digit 1 in shared memory when the whole chunk is in one tensor
    const int64_t e0 = (int64_t)w0 * WT, e1 = min((int64_t)w1 * WT, src.N);
    __syncthreads();
    const int lc = w0 < w1 ? seg_of(s_off, T, e0) : 0;
    const bool one = !kThr && !src.r1_done && w0 < w1 && seg_of(s_off, T, e1 - 1) == lc;
    uint32_t* s_r1 = one ? S.stage : nullptr;
    if (one)
        for (int i = tid; i < REL_BINS; i += blockDim.x) S.stage[i] = 0;
    // tiles with more than WT_THREAD candidates of a piece: tile, count
    // (SEL_THREADS words further) and output position
    static_assert(2 * SEL_THREADS <= D1_BINS, "overflow tile list");
    uint32_t* s_ovf_w = S.h1;
    uint64_t before = 0, run = 0;
    bool have_before = false;
    for (uint32_t pw = w0; pw < w1 || !have_before; pw += blockDim.x) {
        const uint32_t w = pw + tid;
        if (tid == 0) S.flag = 0;
        uint32_t piece;
        const uint32_t ex = block_excl_scan(cnt, S.red, &piece);
        if (single) {
            mine = piece;
            if (tid == 0) *reinterpret_cast<volatile uint64_t*>(src.agg + c) = (uint64_t)mine + 1;
        }
        load_values(src, w, cnt, tc);
        if (!have_before) {
            // resolved while the other blocks publish their counts
            if (early) {
                uint4* s4 = reinterpret_cast<uint4*>(S.stage);
                s4[tid] = r1v[0];
                s4[tid + SEL_THREADS] = r1v[1];
                __syncthreads();
                const RelState r = rel1_from_stage(src.meta[0].k, S);
                if (tid == 0) {
                    S.rs_early = r;
                    S.top_bin = S.stage[REL_BINS - 1];
                }
            }
            if (src.r1_done) look_counts<true>(src.agg, c, status, S);
            else look_counts<false>(src.agg, c, status, S);
            before = S.before;
            have_before = true;
            mark_phase(cm.ctrl, 4);
            mark_last(cm.ctrl, SPAN_OFFSET_LAST);
        }
        const uint64_t pos = before + run + ex;
        if (w < w1 && T > 1) {
            const int64_t base = (int64_t)w * WT;
            const int64_t tend = min(base + (int64_t)WT, src.N);
            for (int l = max(1, lower_bound_off(s_off, T, base)); l < T && s_off[l] < tend; ++l)
                src.cand_start[l] = (int64_t)(pos + tile_count_below(src, S, w, cnt, s_off[l]));
        }
        if (pos >= src.cap) {
            // past the capacity: nothing of this tile is written (a compress
            // call then falls back to the rescan; the hard-threshold step
            // sends only the first cap)
        } else if (cnt > (uint32_t)WT_THREAD) {
            const uint32_t slot = atomicAdd(reinterpret_cast<uint32_t*>(&S.flag), 1u);
            s_ovf_w[slot] = w;
            s_ovf_w[SEL_THREADS + slot] = cnt;
            S.ovf_pos[slot] = pos;
        } else if (cnt > 4) {
            store_ranked<WT_THREAD, kThr>(src, S, w, pos, cnt, tc, s_r1, lc);
        } else if (cnt > 0) {
            store_ranked<4, kThr>(src, S, w, pos, cnt, tc, s_r1, lc);
        }
        // the next round's tile
        cnt = 0;
        if (w + blockDim.x < w1) {
            cnt = src.wt_count[w + blockDim.x];
            load_staged(src, w + blockDim.x, tc);
        }
        __syncthreads();
        // tiles of more than WT_THREAD candidates, a warp each; the loads of
        // OVF_U staged tiles of a warp are issued together
        const uint32_t novf = (uint32_t)S.flag;
        for (uint32_t i0 = warp; i0 < novf; i0 += nwarps * OVF_U) {
            uint32_t wo[OVF_U], cn[OVF_U], o[OVF_U];
            float v[OVF_U];
#pragma unroll
            for (int u = 0; u < OVF_U; ++u) {
                const uint32_t i = i0 + u * nwarps;
                wo[u] = i < novf ? s_ovf_w[i] : 0u;
                cn[u] = i < novf ? s_ovf_w[SEL_THREADS + i] : 0u;
                const bool st = cn[u] <= (uint32_t)WT_CAP && lane_id() < cn[u];
                o[u] = st ? (uint32_t)src.wt_off[(size_t)wo[u] * WT_CAP + lane_id()] : 0xFFFFu;
            }
#pragma unroll
            for (int u = 0; u < OVF_U; ++u) {
                const bool st = cn[u] <= (uint32_t)WT_CAP && lane_id() < cn[u];
                v[u] = st ? src.resid[(int64_t)wo[u] * WT + o[u]] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < OVF_U; ++u) {
                const uint32_t i = i0 + u * nwarps;
                if (i < novf && cn[u] <= (uint32_t)WT_CAP)
                    store_warp_staged<kThr>(src, S, wo[u], S.ovf_pos[i], cn[u], o[u], v[u], s_r1, lc);
            }
        }
        // more than WT_CAP: rescanned (hard threshold: queued for any warp of
        // the grid while the queue has room; dense tiles crowd into few blocks)
        for (uint32_t i = warp; i < novf; i += nwarps) {
            if (s_ovf_w[SEL_THREADS + i] <= (uint32_t)WT_CAP) continue;
            if (kThr && src.rq && rq_push(src, cm, s_ovf_w[i], S.ovf_pos[i])) continue;
            gather_rescan<kThr>(RescanArgs(src), S, s_ovf_w[i], S.ovf_pos[i], s_r1, lc);
        }
        __syncthreads();
        run += piece;
    }
    if (kThr && src.rq) {
        // this block has queued all its dense tiles
        __syncthreads();
        if (tid == 0)
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&cm.ctrl->merge_bar[RQ_DONE])
                         : "memory");
        rq_drain(src, cm, S);
    }
    my0 = before;
    my1 = before + mine;
    if (tid == 0) {
        if (c == 0) src.cand_start[0] = 0;
        if (c == G - 1)
            for (int l = 1; l <= T; ++l)
                if (s_off[l] >= src.N) src.cand_start[l] = (int64_t)my1;
    }
    if (one) {
        uint32_t* g = src.h(lc, CH_R1);
        for (int i = tid; i < REL_BINS; i += blockDim.x)
            if (S.stage[i]) atomicAdd(&g[i], S.stage[i]);
    }
    mark_phase(cm.ctrl, 5);
    mark_last(cm.ctrl, SPAN_GATHER_LAST);
}

// The gather phase, one grid barrier, and the decision every block takes
// alike: candidates only if the list fit and each tensor kept at least k of
// them with its k-th key inside the range of the relative digits.  Returns
// false if the barrier gave up.
__device__ bool compress_gather(CompressSrc& src, const SelCommon& cm, uint32_t& epoch,
                                SelShared& S, uint64_t& my0, uint64_t& my1) {
    gather_phase<false>(src, cm, S, my0, my1);
    const int T = src.T;
    const int tid = threadIdx.x;
    uint64_t total;
    uint32_t bad = 0;
    if (src.r1_done) {
        // one tensor, relative digit 1 built by the streaming pass and the
        // total known from the look-all: no barrier needed to decide
        total = S.total;
        const uint32_t k = src.meta[0].k;
        bad = (total < (uint64_t)k) || (k > 0 && S.top_bin >= k);
        mark_phase(cm.ctrl, 1);
    } else {
        if (!grid_barrier(cm.bar, epoch, &cm.ctrl->status, &S.flag)) return false;
        mark_phase(cm.ctrl, 1);
        total = (uint64_t)src.cand_start[T];
        for (int l = tid; l < T; l += blockDim.x)
            bad |= ((uint64_t)(src.cand_start[l + 1] - src.cand_start[l]) <
                    (uint64_t)src.meta[l].k) ||
                   src.rel_overflow(l);
        bad = block_sum(bad, S.red);
    }
    const bool fits = total <= src.cap;
    src.dense = (src.force_dense || !fits || bad) ? 1 : 0;
    if (blockIdx.x == 0 && tid == 0) {
        cm.ctrl->mode = src.dense;
        cm.ctrl->cand_total = total;
    }
    return true;
}

// Hard-threshold step ("Rethinking gradient sparsification as total error
// minimization", abstract: Top-k with k set by a constant hard threshold):
// the candidates of the streaming pass (key >= T0 = the threshold's key) are
// the passing entries; the gather phase writes the first cap of them, in
// index order, straight into the caller's output and zeroes their residual.
// The last block writes the number that passed.
__global__ void __launch_bounds__(SEL_THREADS)
threshold_kernel(CompressSrc src, SelCommon cm, int64_t* out_count) {
    __shared__ SelShared S;
    mark_phase(cm.ctrl, 0);
    const BlockSpan block_span(cm.ctrl);
    uint64_t my0, my1;
    gather_phase<true>(src, cm, S, my0, my1);
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
        *out_count = (int64_t)my1;
        cm.ctrl->cand_total = my1;
    }
    mark_phase(cm.ctrl, 7);
}

// One pass over positions [a, b) of prefiltered tensor l (block-wide) once
// its digit-1 bin rs.b1 is known: returns the candidates above that bin, and
// hands each candidate in the bin (its relative digit 2) to the entry list
// of l (to_entries) or to the shared-memory histogram S.stage.
__device__ uint32_t scan_rel_bin(const CompressSrc& src, int l, int64_t a, int64_t b,
                                 const RelState& rs, bool to_entries, SelShared& S) {
    const uint32_t T0 = S.T0[l], sh = S.shift[l];
    const uint32_t lmask = (1u << sh) - 1u;
    const uint32_t lane = lane_id();
    uint32_t above = 0;
    for (int64_t p0 = a; p0 < b; p0 += blockDim.x) {
        const int64_t p = p0 + threadIdx.x;
        bool hit = false;
        uint32_t low = 0;
        if (p < b) {
            const uint32_t rel = key_of(src.cand_val[p]) - T0;
            const uint32_t bin = min(rel >> sh, (uint32_t)(REL_BINS - 1));
            above += bin > rs.b1;
            hit = bin == rs.b1;
            low = rel & lmask;
        }
        if (to_entries) {
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, hit);
            if (m) {
                const uint32_t lead = (uint32_t)(__ffs(m) - 1);
                uint32_t at = 0;
                if (lane == lead) at = atomicAdd(src.ent_cnt + l, (uint32_t)__popc(m));
                at = __shfl_sync(0xFFFFFFFFu, at, lead);
                if (hit)
                    src.ent[(size_t)l * ENT_PER + at + __popc(m & ((1u << lane) - 1u))] =
                        ((uint32_t)blockIdx.x << 12) | low;
            }
        } else if (hit) {
            atomicAdd(&S.stage[low], 1u);
        }
    }
    return block_sum(above, S.red);
}

__device__ __forceinline__ void zero_stage(SelShared& S) {
    __syncthreads();
    for (int i = threadIdx.x; i < REL_BINS; i += blockDim.x) S.stage[i] = 0;
    __syncthreads();
}

// A tensor whose candidates [a, b) all lie in this block's range, at most
// EMIT_TILE of them: selected from registers alone (the candidates are read
// once; both relative digits are histogrammed locally) and emitted.  Returns
// false if the counts do not add up.
__device__ bool local_small(const CompressSrc& src, int l, int64_t a, int64_t b, SelShared& S) {
    const int tid = threadIdx.x;
    const uint32_t k = src.meta[l].k;
    const uint32_t T0 = S.T0[l], sh = S.shift[l];
    const uint32_t lmask = (1u << sh) - 1u;
    uint32_t idx[EMIT_PER_THREAD], key[EMIT_PER_THREAD], bin[EMIT_PER_THREAD];
    float val[EMIT_PER_THREAD];
#pragma unroll
    for (int u = 0; u < EMIT_PER_THREAD; ++u) {
        const int64_t pos = a + (int64_t)tid * EMIT_PER_THREAD + u;
        idx[u] = DEAD;
        val[u] = 0.f;
        if (pos < b) {
            idx[u] = src.cand_idx[pos];
            val[u] = src.cand_val[pos];
        }
        key[u] = key_of(val[u]);
        bin[u] = min((key[u] - T0) >> sh, (uint32_t)(REL_BINS - 1));
    }
    if (k == 0) return true;
    zero_stage(S);
#pragma unroll
    for (int u = 0; u < EMIT_PER_THREAD; ++u)
        if (idx[u] != DEAD) atomicAdd(&S.stage[bin[u]], 1u);
    __syncthreads();
    block_find_bin(S.stage, REL_BINS, k, S.red, &S.fr);
    if (!S.fr.ok) return false;
    const uint32_t b1 = S.fr.bin, rem = k - S.fr.above;
    zero_stage(S);
#pragma unroll
    for (int u = 0; u < EMIT_PER_THREAD; ++u)
        if (idx[u] != DEAD && bin[u] == b1) atomicAdd(&S.stage[(key[u] - T0) & lmask], 1u);
    __syncthreads();
    block_find_bin(S.stage, REL_BINS, rem, S.red, &S.fr);
    if (!S.fr.ok) return false;
    const uint32_t Tk = T0 + (b1 << sh) + S.fr.bin;
    const uint32_t q = rem - S.fr.above;
    uint32_t cls = 0;   // bit u: gt, bit 4+u: eq
#pragma unroll
    for (int u = 0; u < EMIT_PER_THREAD; ++u) {
        if (idx[u] == DEAD) continue;
        if (key[u] > Tk) cls |= 1u << u;
        else if (key[u] == Tk) cls |= 1u << (4 + u);
    }
    const uint64_t mine = ((uint64_t)__popc(cls & 0xFu) << 32) | (uint64_t)__popc(cls >> 4);
    uint64_t tot;
    const uint64_t ex = block_excl_scan(mine, S.scan, &tot);
    uint32_t g = (uint32_t)(ex >> 32), e = (uint32_t)(ex & 0xFFFFFFFFu);
#pragma unroll
    for (int u = 0; u < EMIT_PER_THREAD; ++u) {
        if ((cls >> u) & 1u) {
            const uint32_t rank = g + (e < q ? e : q);
            if (rank < k) src.emit(l, rank, idx[u], val[u]);
            ++g;
        } else if ((cls >> (4 + u)) & 1u) {
            if (e < q) src.emit(l, g + e, idx[u], val[u]);
            ++e;
        }
    }
    return true;
}

// Selection and emission on the dense candidate list.  The block's range
// [a0, a1) is what it gathered.  A small tensor (at most EMIT_TILE
// candidates) is selected from registers by one block after the barrier,
// block l mod G for tensor l, so that a range holding many of them does not
// hold up the grid.  A larger tensor that lies wholly inside the range is
// finished here alone.  For the (at most two) tensors that cross the
// range's ends: count the candidates above the k-th key's digit-1 bin (slot)
// and put the candidates in the bin on the tensor's entry list; after a
// barrier every block reads T, the tie quota and the entries of the blocks
// before it from that list.  A bin with more than ENT_PER candidates uses a
// global digit-2 histogram instead, and then all blocks exchange exact
// (gt, eq) counts through one more barrier.
__device__ void compress_candidates(const CompressSrc& src, const SelCommon& cm, uint32_t& epoch,
                                    SelShared& S, uint64_t a0, uint64_t a1) {
    const int c = blockIdx.x, tid = threadIdx.x;
    const int T = src.T;
    uint32_t* status = &cm.ctrl->status;
    __syncthreads();
    if (src.r1_done) {
        // one tensor: [0, total), the total from the look-all (cand_start[1]
        // is written by the last block and not yet ordered by a barrier)
        if (tid == 0) {
            S.seg[0] = 0;
            S.seg[1] = (int64_t)S.total;
        }
    } else {
        for (int l = tid; l <= T; l += blockDim.x) S.seg[l] = src.cand_start[l];
    }
    __syncthreads();
    const bool has = a1 > a0;
    // an empty range passes the tensor running through it on to the next block
    const int l_first = seg_of_pos(S.seg, T, (int64_t)a0);
    const int l_last = has ? seg_of_pos(S.seg, T, (int64_t)a1 - 1) : l_first;
    uint32_t A[2] = {0u, 0u};
    bool cross[2] = {false, false};
    for (int l = l_first; has && l <= l_last; ++l) {
        const int64_t a = max((int64_t)a0, S.seg[l]);
        const int64_t b = min((int64_t)a1, S.seg[l + 1]);
        if (a >= b) continue;
        const uint32_t k = src.meta[l].k;
        // a small tensor is selected by one block after the barrier
        if (S.seg[l + 1] - S.seg[l] <= (int64_t)EMIT_TILE) continue;
        const bool local = S.seg[l] >= (int64_t)a0 && S.seg[l + 1] <= (int64_t)a1;
        const RelState rs = src.r1_done ? S.rs_early : resolve_rel1(src.h(l, CH_R1), k, S);
        if (!rs.ok) {
            if (k && tid == 0) atomicOr(status, ST_INCONSISTENT);
            continue;
        }
        if (local) {
            zero_stage(S);
            scan_rel_bin(src, l, a, b, rs, false, S);
            __syncthreads();
            const DigitState d = finish_rel(S.stage, rs, S.T0[l], S.shift[l], S);
            if (!d.ok) {
                if (tid == 0) atomicOr(status, ST_INCONSISTENT);
                continue;
            }
            emit_range(src, l, a, b, d.prefix, d.rem, k, 0u, 0u, S);
            continue;
        }
        const bool fast = rs.cnt <= ENT_PER;
        if (!fast) zero_stage(S);
        const uint32_t above = scan_rel_bin(src, l, a, b, rs, fast, S);
        if (!fast) {
            __syncthreads();
            uint32_t* g = src.h(l, CH_R2);
            for (int i = tid; i < REL_BINS; i += blockDim.x)
                if (S.stage[i]) atomicAdd(&g[i], S.stage[i]);
            if (tid == 0) atomicOr(&cm.ctrl->r2_path, 1u);
        }
        if (l == l_first) {
            if (tid == 0) S.rs[0] = rs;
            A[0] = above;
            cross[0] = true;
        } else {
            if (tid == 0) S.rs[1] = rs;
            A[1] = above;
            cross[1] = true;
        }
    }
    if (tid == 0) {
        Slot sl;
        sl.l_first = l_first;
        sl.l_last = l_last;
        sl.gt_first = A[0];
        sl.eq_first = 0;
        sl.gt_last = l_first == l_last ? A[0] : A[1];
        sl.eq_last = 0;
        sl.pad[0] = sl.pad[1] = 0;
        cm.slots[c] = sl;
    }
    mark_last(cm.ctrl, SPAN_BAR2_LAST);
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return;
    mark_phase(cm.ctrl, 2);
    const bool r2p = *reinterpret_cast<volatile uint32_t*>(&cm.ctrl->r2_path) != 0;

    // T and the tie quota of the crossing tensors.  The entry words are
    // loaded together with their count (slots past it hold stale words and
    // are dropped); the first tensor's stay in registers for the count of
    // the entries of earlier blocks, whose slots warp 0 reads meanwhile.
    constexpr int EPT = (int)ENT_PER / SEL_THREADS;
    uint32_t ev0[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) ev0[u] = DEAD;
    const bool chain0 = cross[0] && max((int64_t)a0, S.seg[l_first]) > S.seg[l_first];
    DigitState fin[2];
#pragma unroll
    for (int side = 0; side < 2; ++side) {
        fin[side] = DigitState{1u, 0u, 0u, 0u};
        if (!cross[side]) continue;
        const int l = side == 0 ? l_first : l_last;
        const RelState rs = S.rs[side];
        if (rs.cnt <= ENT_PER) {
            const uint32_t* el = src.ent + (size_t)l * ENT_PER;
            uint32_t ev[EPT];
            const uint32_t E = min(*reinterpret_cast<volatile uint32_t*>(src.ent_cnt + l), ENT_PER);
#pragma unroll
            for (int u = 0; u < EPT; ++u) ev[u] = el[tid + u * SEL_THREADS];
#pragma unroll
            for (int u = 0; u < EPT; ++u)
                if ((uint32_t)(tid + u * SEL_THREADS) >= E) ev[u] = DEAD;
            if (side == 0) {
#pragma unroll
                for (int u = 0; u < EPT; ++u) ev0[u] = ev[u];
                if (chain0 && !r2p) chain_prefix(cm, c, l, S);
            }
            zero_stage(S);
#pragma unroll
            for (int u = 0; u < EPT; ++u)
                if (ev[u] != DEAD) atomicAdd(&S.stage[ev[u] & 4095u], 1u);
        } else {
            zero_stage(S);
            stage_words(S.stage, src.h(l, CH_R2), REL_BINS, REL_BINS);
        }
        __syncthreads();
        fin[side] = finish_rel(S.stage, rs, S.T0[l], S.shift[l], S);
        if (!fin[side].ok && tid == 0) atomicOr(status, ST_INCONSISTENT);
    }
    if (r2p) {
        // exact counts of both classes per block
        uint32_t gt[2] = {0u, 0u}, eq[2] = {0u, 0u};
#pragma unroll
        for (int side = 0; side < 2; ++side) {
            if (!cross[side] || !fin[side].ok) continue;
            const int l = side == 0 ? l_first : l_last;
            const int64_t a = max((int64_t)a0, S.seg[l]);
            const int64_t b = min((int64_t)a1, S.seg[l + 1]);
            const uint32_t Tk = fin[side].prefix;
            uint32_t g = 0, e = 0;
            for (int64_t p = a + tid; p < b; p += blockDim.x) {
                const uint32_t key = key_of(src.cand_val[p]);
                g += key > Tk;
                e += key == Tk;
            }
            gt[side] = block_sum(g, S.red);
            eq[side] = block_sum(e, S.red);
        }
        if (tid == 0) {
            Slot sl;
            sl.l_first = l_first;
            sl.l_last = l_last;
            sl.gt_first = gt[0];
            sl.eq_first = eq[0];
            sl.gt_last = l_first == l_last ? gt[0] : gt[1];
            sl.eq_last = l_first == l_last ? eq[0] : eq[1];
            sl.pad[0] = sl.pad[1] = 0;
            cm.slots[c] = sl;
        }
        if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return;
        mark_phase(cm.ctrl, 3);
    }
    mark_phase(cm.ctrl, 6);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

#pragma unroll
    for (int side = 0; side < 2; ++side) {
        if (!cross[side] || !fin[side].ok) continue;
        if (side == 1 && l_last == l_first) continue;
        const int l = side == 0 ? l_first : l_last;
        const int64_t a = max((int64_t)a0, S.seg[l]);
        const int64_t b = min((int64_t)a1, S.seg[l + 1]);
        uint32_t pg = 0, pe = 0;
        if (side == 0 && chain0) {
            if (r2p) chain_prefix(cm, c, l, S);   // the slots now hold exact counts
            pg = S.pre[0];
            pe = S.pre[1];
            __syncthreads();
            if (!r2p) {
                // candidates of the k-th key's bin held by earlier blocks
                const RelState rs = S.rs[0];
                const uint32_t t = fin[0].prefix - S.T0[l] - (rs.b1 << S.shift[l]);
                uint32_t g = 0, e = 0;
#pragma unroll
                for (int u = 0; u < EPT; ++u) {
                    const uint32_t v = ev0[u];
                    if (v != DEAD && (int)(v >> 12) < c) {
                        g += (v & 4095u) > t;
                        e += (v & 4095u) == t;
                    }
                }
                pg += block_sum(g, S.red);
                pe += block_sum(e, S.red);
            }
        }
        emit_range(src, l, a, b, fin[side].prefix, fin[side].rem, src.meta[l].k, pg, pe, S);
    }
    // small tensors (at most EMIT_TILE candidates), tensor l by block l mod G:
    // their candidates are all written, wherever they were gathered
    for (int l = c; l < T; l += (int)gridDim.x) {
        const int64_t a = S.seg[l], b = S.seg[l + 1];
        if (b > a && b - a <= (int64_t)EMIT_TILE && !local_small(src, l, a, b, S) && tid == 0)
            atomicOr(status, ST_INCONSISTENT);
    }
    mark_phase(cm.ctrl, 7);
}

// ---------------------------------------------------------------- kernel

// Standard-digit selection over the positions of src (the merge rounds, and
// the compress step's rescan of the residual): digit passes first_digit..3
// with a grid barrier after each, per-block (gt, eq) counts of the final key,
// one more barrier, and the ordered emission.  Every block of the grid calls
// it with the same epoch.
template <class Src>
__device__ void std_select(Src& src, const SelCommon& cm, uint32_t& epoch, SelShared& S,
                           int first_digit) {
    const int tid = threadIdx.x;
    const int c = blockIdx.x;
    const int G = gridDim.x;
    uint32_t* status = &cm.ctrl->status;
    const int T = src.nseg();
    __syncthreads();
    for (int l = tid; l <= T; l += blockDim.x) S.seg[l] = src.seg_bound(l);
    __syncthreads();
    const int64_t total = S.seg[T];

    // contiguous range of this block (multiple of 4 positions)
    int64_t span = ceil_div64(total, G);
    span = (span + 3) & ~(int64_t)3;
    const int64_t p0 = min((int64_t)c * span, total);
    const int64_t p1 = min(p0 + span, total);
    const bool has = p1 > p0;
    const int l_first = has ? seg_of_pos(S.seg, T, p0) : 0;
    const int l_last = has ? seg_of_pos(S.seg, T, p1 - 1) : -1;

    // ---- standard digit passes
    for (int d = first_digit; d <= 3; ++d) {
        for (int l = l_first; l <= l_last; ++l) {
            const int64_t a = max(p0, S.seg[l]);
            const int64_t b = min(p1, S.seg[l + 1]);
            if (a >= b || !src.uses_std(l)) continue;
            resolve_std(src.d1(l), src.d2(l), src.d3(l), src.seg_k(l), d - 1, S, status);
            if (S.ds.none || !S.ds.ok) continue;
            const uint32_t prefix = S.ds.prefix;
            uint32_t* hd = d == 1 ? src.d1(l) : (d == 2 ? src.d2(l) : src.d3(l));
            const bool use_smem = (d == 1) && (b - a) >= 4096;
            if (use_smem) {
                for (int i = tid; i < D1_BINS; i += blockDim.x) S.h1[i] = 0;
                __syncthreads();
            }
            for (int64_t pos = a + tid; pos < b; pos += blockDim.x) {
                uint32_t idx;
                float val;
                src.load(pos, idx, val);
                if (idx == DEAD) continue;
                const uint32_t key = key_of(val);
                if (!in_class(key, d, prefix)) continue;
                const uint32_t dg = digit_of(key, d);
                if (use_smem) atomicAdd(&S.h1[dg], 1u);
                else atomicAdd(&hd[dg], 1u);
            }
            if (use_smem) {
                __syncthreads();
                for (int i = tid; i < D1_BINS; i += blockDim.x)
                    if (S.h1[i]) atomicAdd(&hd[i], S.h1[i]);
                __syncthreads();
            }
        }
        if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return;
        mark_phase(cm.ctrl, 2 + d);
    }

    // ---- per-block counts of (key > T, key == T) in the first and last segment
    uint32_t gtF = 0, eqF = 0, gtL = 0, eqL = 0;
    for (int l = l_first; l <= l_last; ++l) {
        if (l != l_first && l != l_last) continue;
        const int64_t a = max(p0, S.seg[l]);
        const int64_t b = min(p1, S.seg[l + 1]);
        src.resolve_final(l, S, status);
        if (tid == 0) {
            if (l == l_first) S.fin[0] = S.ds;
            if (l == l_last) S.fin[1] = S.ds;
        }
        const uint32_t Tk = (S.ds.none || !S.ds.ok) ? NO_KEY : S.ds.prefix;
        uint32_t gt = 0, eq = 0;
        for (int64_t pos = a + tid; pos < b; pos += blockDim.x) {
            uint32_t idx;
            float val;
            src.load(pos, idx, val);
            if (idx == DEAD) continue;
            const uint32_t key = key_of(val);
            gt += key > Tk && Tk != NO_KEY;
            eq += key == Tk;
        }
        gt = block_sum(gt, S.red);
        eq = block_sum(eq, S.red);
        if (l == l_first) { gtF = gt; eqF = eq; }
        if (l == l_last) { gtL = gt; eqL = eq; }
    }
    if (tid == 0) {
        Slot sl;
        sl.l_first = has ? l_first : 0x7FFFFFFF;
        sl.l_last = has ? l_last : -1;
        sl.gt_first = gtF;
        sl.eq_first = eqF;
        sl.gt_last = gtL;
        sl.eq_last = eqL;
        sl.pad[0] = sl.pad[1] = 0;
        cm.slots[c] = sl;
    }
    if (c == 0) {
        if constexpr (std::is_same<Src, MergeSrc>::value) src.finalize_block0();
    }
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return;
    mark_phase(cm.ctrl, 6);
    // a kernel launched after this one with programmatic serialisation may be
    // scheduled now; it still waits for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- emission
    for (int l = l_first; l <= l_last; ++l) {
        const int64_t a = max(p0, S.seg[l]);
        const int64_t b = min(p1, S.seg[l + 1]);
        if (a >= b) continue;
        DigitState fs;
        if (l == l_first || l == l_last) {
            fs = l == l_first ? S.fin[0] : S.fin[1];
        } else {
            src.resolve_final(l, S, status);
            fs = S.ds;
        }
        if (fs.none || !fs.ok) continue;
        uint32_t pg = 0, pe = 0;
        if (l == l_first && a > S.seg[l]) {
            chain_prefix(cm, c, l, S);
            pg = S.pre[0];
            pe = S.pre[1];
            __syncthreads();
        }
        emit_range(src, l, a, b, fs.prefix, fs.rem, src.seg_k(l), pg, pe, S);
    }
    mark_phase(cm.ctrl, 7);
}

template <class Src>
__global__ void __launch_bounds__(SEL_THREADS)
select_kernel(Src src, SelCommon cm) {
    __shared__ SelShared S;
    uint32_t epoch = 0;
    mark_phase(cm.ctrl, 0);
    const BlockSpan block_span(cm.ctrl);

    int first_digit;
    if constexpr (std::is_same<Src, CompressSrc>::value) {
        uint64_t my0, my1;
        if (!compress_gather(src, cm, epoch, S, my0, my1)) return;
        if (!src.dense) {
            compress_candidates(src, cm, epoch, S, my0, my1);
            return;
        }
        first_digit = 1;
    } else {
        src.fold_bad_input(cm.ctrl);
        first_digit = src.d1_done ? 2 : 1;
    }
    std_select(src, cm, epoch, S, first_digit);
}

}  // namespace tke
