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
// + 10 bits; a prefiltered tensor of the compress step instead uses two
// digits of key - T0 (see common.cuh), whose first histogram the streaming
// pass already built and whose second is built while the candidates are
// gathered, so that path needs no digit pass of its own.
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

namespace tke {

constexpr int SEL_THREADS = 512;
constexpr int SEG_MAX = 256;
constexpr int EMIT_PER_THREAD = 4;
constexpr int EMIT_TILE = SEL_THREADS * EMIT_PER_THREAD;

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

struct SelShared {
    int64_t seg[SEG_MAX + 1];
    __align__(16) uint32_t stage[REL_BINS];
    uint32_t h1[D1_BINS];
    uint64_t scan[33];
    uint32_t red[33];
    uint32_t T0[SEG_MAX];
    uint32_t shift[SEG_MAX];
    uint32_t b1[SEG_MAX];      // relative digit 1 of the k-th key (gather phase)
    uint32_t a1[SEG_MAX];      // and the candidates above its bin
    FindResult fr;
    DigitState ds;
    DigitState fin[2];         // final thresholds of the first and last segment
    int flag;
    uint32_t pre[4];
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

// Relative digits of a prefiltered tensor.  With want_r2 false only digit 1
// is resolved (S.ds.prefix = its bin); otherwise S.ds.prefix = T and
// S.ds.rem = q.  ok = 0 when the k-th key lies above the covered range.
__device__ void resolve_rel(const uint32_t* r1, const uint32_t* r2, uint32_t k, uint32_t T0,
                            uint32_t shift, bool want_r2, SelShared& S,
                            uint32_t known_b1 = 0xFFFFFFFFu, uint32_t known_a1 = 0) {
    __syncthreads();
    if (k == 0) {
        if (threadIdx.x == 0) S.ds = DigitState{1u, 0u, 0u, 1u};
        __syncthreads();
        return;
    }
    uint32_t ok, b1, rem;
    if (known_b1 != 0xFFFFFFFFu) {
        ok = 1;
        b1 = known_b1;
        rem = k - known_a1;
    } else {
        stage_words(S.stage, r1, REL_BINS, REL_BINS);
        __syncthreads();
        block_find_bin(S.stage, REL_BINS, k, S.red, &S.fr);
        ok = (S.fr.ok && S.fr.bin != REL_BINS - 1) ? 1u : 0u;
        b1 = S.fr.bin;
        rem = k - S.fr.above;
    }
    uint32_t out = b1;
    if (want_r2 && ok) {
        __syncthreads();
        const int nlow = 1 << shift;
        if (nlow >= 4) {
            stage_words(S.stage, r2, nlow, REL_BINS);
        } else {
            for (int i = threadIdx.x; i < REL_BINS; i += blockDim.x)
                S.stage[i] = i < nlow ? r2[i] : 0u;
        }
        __syncthreads();
        block_find_bin(S.stage, REL_BINS, rem, S.red, &S.fr);
        ok = S.fr.ok;
        rem -= S.fr.above;
        out = T0 + (b1 << shift) + S.fr.bin;
    }
    if (threadIdx.x == 0) S.ds = DigitState{0u, out, rem, ok};
    __syncthreads();
}

// ---------------------------------------------------------------- sources

// Compress: candidates of the streaming pass, or the whole residual.
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
    const uint32_t* st_idx;      // [num_wt][WT_CAP]
    const float* st_val;
    const uint32_t* bound_before;
    int32_t force_dense;
    int32_t dense;               // decided inside the kernel

    __device__ int nseg() const { return T; }
    __device__ int64_t seg_bound(int l) const { return dense ? (l < T ? meta[l].off : N) : cand_start[l]; }
    __device__ uint32_t seg_k(int l) const { return meta[l].k; }
    __device__ uint32_t* h(int l, int part) const { return hist + (size_t)l * CHIST_WORDS + part; }
    // whether segment l is resolved by standard digits
    __device__ bool uses_std(int l) const {
        if (dense) return true;
        const uint32_t k = meta[l].k;
        return k > 0 && h(l, CH_R1)[REL_BINS - 1] >= k;
    }
    __device__ uint32_t* d1(int l) const { return h(l, dense ? CH_D1 : CH_C1); }
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
        if (uses_std(l)) {
            resolve_std(d1(l), d2(l), d3(l), seg_k(l), 3, S, status);
        } else {
            const SegMeta& m = meta[l];
            resolve_rel(h(l, CH_R1), h(l, CH_R2), m.k, m.T0, m.shift, true, S, S.b1[l], S.a1[l]);
            if (threadIdx.x == 0 && !S.ds.ok) atomicOr(status, ST_INCONSISTENT);
        }
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

// Gather-time bookkeeping of the second relative digit: a candidate of
// tensor l whose first relative digit is the k-th's bin counts in the
// tensor's digit-2 histogram.
__device__ __forceinline__ void rel2_add(const CompressSrc& src, const SelShared& S, int l,
                                         float v) {
    const uint32_t b1 = S.b1[l];
    if (b1 == 0xFFFFFFFFu) return;                 // tensor resolved otherwise
    const uint32_t rel = key_of(v) - S.T0[l];
    const uint32_t sh = S.shift[l];
    if ((rel >> sh) == b1) atomicAdd(src.h(l, CH_R2) + (rel & ((1u << sh) - 1u)), 1u);
}

// Gather phase of the compress select: rebuild the global candidate order
// from the streaming pass's per-warp-tile staging.  Each block takes a
// contiguous chunk of warp tiles; a grid barrier turns the chunk sums into
// offsets; every staged candidate is copied to its place in the dense list,
// and a warp tile that had more than WT_CAP candidates is rescanned from the
// residual (which holds acc) with the same predicate.  Also records where
// each tensor's candidates start, and builds the second relative digit of
// the tensors that use it.  Then decides the path for every block alike:
// candidates only if each tensor kept at least k of them and the list fit.
// Returns false if a barrier gave up.
__device__ bool compress_gather(CompressSrc& src, const SelCommon& cm, uint32_t& epoch,
                                SelShared& S) {
    const int G = gridDim.x, c = blockIdx.x, tid = threadIdx.x;
    const uint32_t lane = lane_id(), warp = warp_id(), nwarps = blockDim.x >> 5;
    const int T = src.T;
    uint32_t* status = &cm.ctrl->status;
    int64_t* s_off = S.seg;
    for (int l = tid; l < T; l += blockDim.x) {
        s_off[l] = src.meta[l].off;
        S.T0[l] = src.meta[l].T0;
        S.shift[l] = src.meta[l].shift;
        S.b1[l] = 0xFFFFFFFFu;
    }
    if (tid == 0) s_off[T] = src.N;
    __syncthreads();
    const uint32_t W = src.num_wt;
    const uint32_t per = (W + G - 1) / G;
    const uint32_t w0 = min((uint32_t)c * per, W), w1 = min(w0 + per, W);

    // relative digit 1 of the tensors of this chunk (the k-th key's bin)
    if (w0 < w1) {
        const int tl0 = seg_of(s_off, T, (int64_t)w0 * WT);
        const int tl1 = seg_of(s_off, T, min((int64_t)w1 * WT, src.N) - 1);
        for (int l = tl0; l <= tl1; ++l) {
            const SegMeta& m = src.meta[l];
            if (m.k == 0 || src.uses_std(l)) continue;
            resolve_rel(src.h(l, CH_R1), nullptr, m.k, m.T0, m.shift, false, S);
            if (tid == 0) {
                S.b1[l] = S.ds.ok ? S.ds.prefix : 0xFFFFFFFFu;
                S.a1[l] = S.ds.ok ? m.k - S.ds.rem : 0u;
            }
        }
    }

    uint32_t mine = 0;
    for (uint32_t w = w0 + tid; w < w1; w += blockDim.x) mine += src.wt_count[w];
    mine = block_sum(mine, S.red);
    if (tid == 0) cm.slots[c].gt_first = mine;
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return false;
    mark_phase(cm.ctrl, 1);

    uint64_t before = 0, total = 0;
    for (int i = tid; i < G; i += blockDim.x) {
        const uint64_t v = cm.slots[i].gt_first;
        total += v;
        if (i < c) before += v;
    }
    before = block_sum(before, S.scan);
    total = block_sum(total, S.scan);
    const bool fits = total <= src.cap;
    if (c == 0)
        for (int l = tid; l <= T; l += blockDim.x)
            if (l == 0) src.cand_start[0] = 0;
            else if (s_off[l] >= src.N) src.cand_start[l] = (int64_t)total;

    // overflow list in the stage buffer: pairs (warp tile, offset)
    uint32_t* s_ovf_w = S.stage;
    uint64_t* s_ovf_o = reinterpret_cast<uint64_t*>(S.stage + SEL_THREADS);
    uint32_t* s_ovf_n = S.stage + 3 * SEL_THREADS;
    uint64_t run = before;
    for (uint32_t pw = w0; pw < w1; pw += blockDim.x) {
        const uint32_t w = pw + tid;
        const uint32_t cnt = w < w1 ? src.wt_count[w] : 0u;
        if (tid == 0) *s_ovf_n = 0;
        uint32_t piece;
        const uint32_t ex = block_excl_scan(cnt, S.red, &piece);
        const uint64_t off = run + ex;
        if (w < w1) {
            const int64_t base = (int64_t)w * WT;
            const int64_t tend = min(base + (int64_t)WT, src.N);
            if (T > 1)
                for (int l = max(1, lower_bound_off(s_off, T, base)); l < T && s_off[l] < tend; ++l)
                    src.cand_start[l] = (int64_t)(off + src.bound_before[l]);
            if (fits && cnt) {
                if (cnt <= WT_CAP) {
                    int l = seg_of(s_off, T, base);
                    for (uint32_t i = 0; i < cnt; ++i) {
                        const uint32_t idx = src.st_idx[(size_t)w * WT_CAP + i];
                        const float v = src.st_val[(size_t)w * WT_CAP + i];
                        src.cand_idx[off + i] = idx;
                        src.cand_val[off + i] = v;
                        while (l < T - 1 && s_off[l + 1] <= (int64_t)idx) ++l;
                        rel2_add(src, S, l, v);
                    }
                } else {
                    const uint32_t slot = atomicAdd(s_ovf_n, 1u);
                    s_ovf_w[slot] = w;
                    s_ovf_o[slot] = off;
                }
            }
        }
        __syncthreads();
        const uint32_t novf = *s_ovf_n;
        for (uint32_t i = warp; i < novf; i += nwarps) {
            const uint32_t w2 = s_ovf_w[i];
            uint64_t pos = s_ovf_o[i];
            const int64_t base = (int64_t)w2 * WT;
            const int64_t tend = min(base + (int64_t)WT, src.N);
            int l = seg_of(s_off, T, base);
            for (int64_t e0 = base; e0 < tend; e0 += 32) {
                const int64_t e = e0 + lane;
                bool f = false;
                float v = 0.f;
                if (e < tend) {
                    while (l < T - 1 && s_off[l + 1] <= e) ++l;
                    v = src.resid[e];
                    f = key_of(v) >= S.T0[l];
                }
                const uint32_t m = __ballot_sync(0xFFFFFFFFu, f);
                if (f) {
                    const uint64_t q = pos + __popc(m & ((1u << lane) - 1u));
                    if (q < src.cap) {
                        src.cand_idx[q] = (uint32_t)e;
                        src.cand_val[q] = v;
                    }
                    rel2_add(src, S, l, v);
                }
                pos += __popc(m);
                // keep the lanes' tensor cursors in step
                l = __shfl_sync(0xFFFFFFFFu, l, 31);
            }
        }
        __syncthreads();
        run += piece;
    }
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return false;
    mark_phase(cm.ctrl, 2);

    uint32_t bad = 0;
    for (int l = tid; l < T; l += blockDim.x)
        bad |= (uint64_t)(src.cand_start[l + 1] - src.cand_start[l]) < (uint64_t)src.meta[l].k;
    bad = block_sum(bad, S.red);
    src.dense = (src.force_dense || !fits || bad) ? 1 : 0;
    if (c == 0 && tid == 0) {
        cm.ctrl->mode = src.dense;
        cm.ctrl->cand_total = total;
    }
    return true;
}

// ---------------------------------------------------------------- kernel

template <class Src>
__global__ void __launch_bounds__(SEL_THREADS)
select_kernel(Src src, SelCommon cm) {
    __shared__ SelShared S;
    const int tid = threadIdx.x;
    const int c = blockIdx.x;
    const int G = gridDim.x;
    uint32_t epoch = 0;
    uint32_t* status = &cm.ctrl->status;
    mark_phase(cm.ctrl, 0);

    int first_digit;
    if constexpr (std::is_same<Src, CompressSrc>::value) {
        if (!compress_gather(src, cm, epoch, S)) return;
        // digit passes: all three on the rescan path; on the candidate path
        // digits 2 and 3 only if some tensor uses standard digits
        uint32_t need = 0;
        if (!src.dense)
            for (int l = tid; l < src.T; l += blockDim.x) need |= src.uses_std(l) ? 1u : 0u;
        need = block_sum(need, S.red);
        first_digit = src.dense ? 1 : (need ? 2 : 4);
    } else {
        src.fold_bad_input(cm.ctrl);
        first_digit = src.d1_done ? 2 : 1;
    }
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
        const uint32_t Tk = fs.prefix;
        const uint32_t q = fs.rem;
        const uint32_t kseg = src.seg_k(l);
        // counts of earlier blocks in this segment
        if (tid < 32) {
            uint32_t pg = 0, pe = 0;
            if (l == l_first && a > S.seg[l]) {
                int cc = c - 1;
                for (;;) {
                    const int j = cc - (int)lane_id();
                    bool match = false, cont = false;
                    uint32_t g = 0, e = 0;
                    if (j >= 0) {
                        const Slot sl = cm.slots[j];
                        match = sl.l_last == l;
                        cont = match && sl.l_first == l;
                        g = sl.gt_last;
                        e = sl.eq_last;
                    }
                    const uint32_t contm = __ballot_sync(0xFFFFFFFFu, cont);
                    const uint32_t matchm = __ballot_sync(0xFFFFFFFFu, match);
                    const uint32_t run = (contm == 0xFFFFFFFFu) ? 32u : (uint32_t)(__ffs(~contm) - 1);
                    const bool take = lane_id() < run || (lane_id() == run && ((matchm >> run) & 1u));
                    pg += warp_sum(take ? g : 0u);
                    pe += warp_sum(take ? e : 0u);
                    if (run < 32) break;
                    cc -= 32;
                }
            }
            if (tid == 0) {
                S.pre[0] = pg;
                S.pre[1] = pe;
            }
        }
        __syncthreads();
        uint32_t run_gt = S.pre[0], run_eq = S.pre[1];
        __syncthreads();
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
    mark_phase(cm.ctrl, 7);
}

}  // namespace tke
