// Exact top-k selection and ordered emission for one flat tensor, after the
// streaming pass ("A Distributed Synchronous SGD Algorithm with Global Top-k
// Sparsification", ABSTRACT: the k largest absolute values; the lower index
// wins among equal magnitudes, which makes the set unique).
//
// The streaming pass left, per warp tile of 1,024 elements, the exact number
// of candidates (key >= T0) and the offsets of up to 32 of them, plus the
// relative digit-1 histogram R1 of all candidates.  R1 alone gives the bin b1
// of the k-th key, so every block knows from its first microseconds which of
// its candidates are in for sure (bin above b1), out (below) or undecided
// (in b1).  Each block of one wave (one per SM) owns a contiguous range of
// tiles:
//   A  stage its candidates in shared memory in index order (offsets ranked
//      inside each tile; tiles with more than 32 candidates rescanned from
//      the residual by a warp), count those above b1 and append those in b1
//      to a small grid-wide entry list (block << 12 | relative digit 2);
//   B  one grid-wide exchange; every block then reads the entry list, finds
//      the k-th key T and the tie quota q, and its output offset from the
//      earlier blocks' counts and entries;
//   C  emit its selected candidates from shared memory: (idx, acc) and
//      residual[idx] = +0.0f.
// A k-th-key bin holding more than 4,096 candidates takes a global digit-2
// histogram and an exact-count exchange (one more grid-wide step) instead.
// If the candidates cannot contain the answer (fewer than k, the k-th key
// above the relative digits' range) or are too many to stage in about one
// round per block (src.cap), every block switches, alike, to the
// standard-digit rescan of the residual, so the result never depends on the
// prefilter threshold.
#pragma once

#include "common.cuh"
#include "kernels_compress.cuh"
#include "kernels_select.cuh"

namespace tke {

constexpr int FS_THREADS = 512;
constexpr int FS_TILES = FS_THREADS;     // tiles per staging chunk, one per thread
constexpr int FS_CAND = 12288;           // candidates staged per round
constexpr int FS_WARPS = FS_THREADS / 32;
constexpr int FS_BATCH = 8;              // tiles whose candidate loads a warp keeps in flight
constexpr int FS_CBATCH = 4;             // candidate loads a thread keeps in flight
constexpr int FS_EMIT = 4;               // staged positions per thread per emission step

struct FlatShared {
    uint32_t hist[REL_BINS];             // R1, later the digit-2 histogram
    uint32_t cidx[FS_CAND];              // staged candidates of a round, index order
    float cval[FS_CAND];
    uint16_t off[FS_TILES * WT_CAP];     // staged offsets of the round's tiles
    uint32_t tstart[FS_TILES + 1];       // first staged position of each tile
    uint32_t tcnt[FS_TILES];
    uint16_t dense[FS_TILES];            // tiles of the round with more than WT_CAP candidates
    uint32_t wbm[FS_WARPS * 32];         // per warp: bitmap of a tile's candidate offsets
    uint64_t scan[33];
    uint32_t red[33];
    uint32_t ndense, nt, nc;
    int flag;
    FindResult fr1, fr2;
    uint32_t total;
    uint32_t pre[2];
    uint32_t crowd[4];                   // crowded path: T, tie quota, counts before the block
};

struct FlatParams {
    CompressSrc src;        // resid, meta, tile records, histograms, entry list, outputs
    SelCommon cm;
    Hint* hint;             // next call's prefilter threshold (null: none)
    uint64_t hint_tag;
};

// In one scan of a REL_BINS histogram (top bin first), the bins holding the
// r1-th and r2-th largest elements (1-based), and the total.  Every thread
// of the block must call it; results in *o1, *o2 and *total afterwards.
__device__ void fs_find2(const uint32_t* h, uint32_t r1, uint32_t r2, FlatShared& F) {
    const int t = threadIdx.x;
    constexpr int per = REL_BINS / FS_THREADS;
    const int hi = REL_BINS - t * per;
    const int lo = hi - per;
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) s += h[lo + ((i + t) & (per - 1))];
    if (t == 0) {
        F.fr1.ok = 0;
        F.fr2.ok = 0;
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan(s, F.red, &tot);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const uint32_t r = w == 0 ? r1 : r2;
        FindResult* o = w == 0 ? &F.fr1 : &F.fr2;
        if (ex < r && ex + s >= r) {
            uint32_t run = ex;
            for (int b = hi - 1; b >= lo; --b) {
                const uint32_t c = h[b];
                if (run + c >= r) {
                    o->bin = (uint32_t)b;
                    o->above = run;
                    o->cnt = c;
                    o->ok = 1;
                    break;
                }
                run += c;
            }
        }
    }
    if (t == 0) F.total = tot;
    __syncthreads();
}

// Sum over blocks j < c of field `f` of their slots (warp 0 loads them).
__device__ __forceinline__ uint32_t fs_slots_before(const Slot* slots, int c, int f, FlatShared& F) {
    if (threadIdx.x < 32) {
        uint32_t s = 0;
        for (int j = (int)lane_id(); j < c; j += 32) {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(slots + j);
            s += *reinterpret_cast<const volatile uint32_t*>(w + f);
        }
        s = warp_sum(s);
        if (threadIdx.x == 0) F.pre[0] = s;
    }
    __syncthreads();
    const uint32_t r = F.pre[0];
    __syncthreads();
    return r;
}

// One staging round: tiles [wr, wr + nt) with nt chosen here so that their
// candidates fit in FS_CAND.  Leaves the candidates in F.cidx / F.cval in
// index order, F.nc of them, and returns nt (0 when wr >= w1).  The counts
// and offsets of the chunk's tiles may be passed in already loaded.
struct ChunkRegs {
    uint32_t cnt;
    uint4 o[4];
};

__device__ __forceinline__ void fs_load_chunk(const CompressSrc& src, uint32_t w, uint32_t w1,
                                              ChunkRegs& r) {
    r.cnt = 0;
    if (w < w1) {
        r.cnt = src.wt_count[w];
        const uint4* p4 = reinterpret_cast<const uint4*>(src.wt_off + (size_t)w * WT_CAP);
#pragma unroll
        for (int i = 0; i < 4; ++i) r.o[i] = p4[i];
    }
}

// Candidates of a tile with more than WT_CAP of them, rescanned from the
// residual (which holds acc) by one warp, written in index order to
// positions [pos, pos + cnt) of the staging arrays.
__device__ __noinline__ void fs_stage_dense(const float* resid, int64_t N, uint32_t T0, uint32_t w,
                                            uint32_t pos, uint32_t cnt, uint32_t* cidx, float* cval,
                                            uint32_t* status) {
    const uint32_t lane = lane_id();
    const int64_t base = (int64_t)w * WT;
    const int64_t tend = min(base + (int64_t)WT, N);
    const uint32_t end = pos + cnt;
    const float* tile = resid + base;
    if (tend - base == WT && (reinterpret_cast<uintptr_t>(tile) & 15u) == 0) {
        const float4* t4 = reinterpret_cast<const float4*>(tile) + lane;
        float4 v4[WT_VECS];
#pragma unroll
        for (int j = 0; j < WT_VECS; ++j) v4[j] = t4[32 * j];
#pragma unroll
        for (int j = 0; j < WT_VECS; ++j) {
            uint32_t f = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) f |= (uint32_t)(key_of(f4_get(v4[j], t)) >= T0) << t;
            const uint32_t c = (uint32_t)__popc(f);
            const uint32_t incl = warp_incl_scan(c);
            uint32_t q = pos + incl - c;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if ((f >> t) & 1u) {
                    if (q < end) {
                        cidx[q] = (uint32_t)(base + 128 * j + 4 * lane + t);
                        cval[q] = f4_get(v4[j], t);
                    }
                    ++q;
                }
            }
            pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    } else {
        const uint32_t lt = (1u << lane) - 1u;
        for (int u = 0; u < 32; ++u) {
            const int64_t e = base + 32 * u + lane;
            const float v = e < tend ? resid[e] : 0.f;
            const bool f = e < tend && key_of(v) >= T0;
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, f);
            if (f) {
                const uint32_t q = pos + __popc(m & lt);
                if (q < end) {
                    cidx[q] = (uint32_t)e;
                    cval[q] = v;
                }
            }
            pos += __popc(m);
        }
    }
    if (lane == 0 && pos != end) atomicOr(status, ST_INCONSISTENT);
}

__device__ uint32_t fs_stage_round(const CompressSrc& src, FlatShared& F, uint32_t wr, uint32_t w1,
                                   ChunkRegs& r, uint32_t T0, uint32_t* status) {
    const int tid = threadIdx.x;
    if (wr >= w1) return 0;
    // the longest prefix of the chunk's tiles whose candidates fit
    uint32_t tot;
    const uint32_t ex = block_excl_scan(r.cnt, F.red, &tot);
    const bool mine = wr + tid < w1;
    const bool fits = mine && ex + r.cnt <= (uint32_t)FS_CAND;
    const uint32_t nt = (uint32_t)__syncthreads_count(fits);
    if (tid == 0) F.ndense = 0;
    __syncthreads();
    if ((uint32_t)tid < nt) {
        F.tstart[tid] = ex;
        F.tcnt[tid] = r.cnt;
        if (r.cnt > (uint32_t)WT_CAP) {
            F.dense[atomicAdd(&F.ndense, 1u)] = (uint16_t)tid;
        } else if (r.cnt > 0) {
            uint4* d = reinterpret_cast<uint4*>(F.off + tid * WT_CAP);
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = r.o[i];
        }
        if ((uint32_t)tid == nt - 1) {
            F.tstart[nt] = ex + r.cnt;
            F.nc = ex + r.cnt;
        }
    }
    __syncthreads();
    const uint32_t nc = F.nc;
    if (nc <= 4 * nt) {
        // sparse tiles, few candidates per tile on average: candidate-parallel (a
        // thread finds its tile by binary search and ranks its offset among the
        // tile's); a thread keeps FS_CBATCH value loads in flight
        for (uint32_t p0 = tid; p0 < nc; p0 += FS_THREADS * FS_CBATCH) {
            uint32_t e[FS_CBATCH], q[FS_CBATCH];
            float v[FS_CBATCH];
#pragma unroll
            for (int u = 0; u < FS_CBATCH; ++u) {
                const uint32_t p = p0 + (uint32_t)u * FS_THREADS;
                q[u] = 0xFFFFFFFFu;
                e[u] = 0;
                if (p < nc) {
                    // tile of position p: last t with tstart[t] <= p
                    uint32_t lo = 0, hi = nt;
                    while (hi - lo > 1) {
                        const uint32_t mid = (lo + hi) >> 1;
                        if (F.tstart[mid] <= p) lo = mid; else hi = mid;
                    }
                    const uint32_t c = F.tcnt[lo];
                    if (c <= (uint32_t)WT_CAP) {
                        const uint16_t* ot = F.off + lo * WT_CAP;
                        const uint32_t o = ot[p - F.tstart[lo]];
                        uint32_t rank = 0;
                        for (uint32_t j = 0; j < c; ++j) rank += ot[j] < o;
                        q[u] = F.tstart[lo] + rank;
                        e[u] = (wr + lo) * (uint32_t)WT + o;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < FS_CBATCH; ++u) v[u] = q[u] != 0xFFFFFFFFu ? src.resid[e[u]] : 0.f;
#pragma unroll
            for (int u = 0; u < FS_CBATCH; ++u) {
                if (q[u] != 0xFFFFFFFFu) {
                    F.cidx[q[u]] = e[u];
                    F.cval[q[u]] = v[u];
                }
            }
        }
    } else {
        // sparse tiles, many candidates per tile on average: a warp per tile, lane i holding
        // the tile's staged candidate i; its rank in index order comes from a
        // bitmap of the tile's offsets (one bit per element, 32 words) and one
        // warp scan of the words' popcounts.  A warp keeps the value loads of
        // FS_BATCH tiles in flight.
        {
            const uint32_t lane = lane_id(), warp = warp_id();
            uint32_t* bm = F.wbm + warp * 32;
            for (uint32_t t0 = warp; t0 < nt; t0 += FS_WARPS * FS_BATCH) {
                uint32_t o[FS_BATCH], cn[FS_BATCH];
                float v[FS_BATCH];
#pragma unroll
                for (int u = 0; u < FS_BATCH; ++u) {
                    const uint32_t t = t0 + (uint32_t)u * FS_WARPS;
                    cn[u] = t < nt ? F.tcnt[t] : 0u;
                    if (cn[u] > (uint32_t)WT_CAP) cn[u] = 0;            // dense: rescanned below
                    o[u] = lane < cn[u] ? (uint32_t)F.off[t * WT_CAP + lane] : 0xFFFFu;
                }
#pragma unroll
                for (int u = 0; u < FS_BATCH; ++u) {
                    const uint32_t t = t0 + (uint32_t)u * FS_WARPS;
                    v[u] = o[u] != 0xFFFFu ? src.resid[(size_t)(wr + t) * WT + o[u]] : 0.f;
                }
#pragma unroll
                for (int u = 0; u < FS_BATCH; ++u) {
                    if (cn[u] == 0) continue;                           // warp-uniform
                    const uint32_t t = t0 + (uint32_t)u * FS_WARPS;
                    const bool mine = o[u] != 0xFFFFu;
                    if (mine) atomicOr(&bm[o[u] >> 5], 1u << (o[u] & 31u));
                    __syncwarp();
                    const uint32_t w = bm[lane];
                    bm[lane] = 0u;
                    const uint32_t pc = (uint32_t)__popc(w);
                    const uint32_t ex = warp_incl_scan(pc) - pc;
                    const uint32_t wi = (o[u] >> 5) & 31u;
                    const uint32_t wx = __shfl_sync(0xFFFFFFFFu, ex, wi);
                    const uint32_t ww = __shfl_sync(0xFFFFFFFFu, w, wi);
                    if (mine) {
                        const uint32_t q = F.tstart[t] + wx + (uint32_t)__popc(ww & ((1u << (o[u] & 31u)) - 1u));
                        F.cidx[q] = (wr + t) * (uint32_t)WT + o[u];
                        F.cval[q] = v[u];
                    }
                    __syncwarp();
                }
            }
        }
    }
    // dense tiles: a warp each
    const uint32_t nd = F.ndense;
    for (uint32_t i = warp_id(); i < nd; i += FS_THREADS / 32) {
        const uint32_t t = F.dense[i];
        fs_stage_dense(src.resid, src.N, T0, wr + t, F.tstart[t], F.tcnt[t], F.cidx, F.cval, status);
    }
    __syncthreads();
    return nt;
}

// Emission of the staged candidates [0, nc): key > Tk always, key == Tk while
// the tie quota q lasts; (run_gt, run_eq) are the counts of both classes at
// lower indices.  Advances them past this round.
__device__ void fs_emit(const CompressSrc& src, FlatShared& F, uint32_t nc, uint32_t Tk, uint32_t q,
                        uint32_t k, int32_t* out_idx, float* out_val, int64_t idx_off,
                        uint32_t& run_gt, uint32_t& run_eq) {
    const int tid = threadIdx.x;
    for (uint32_t base = 0; base < nc; base += FS_THREADS * FS_EMIT) {
        uint32_t idx[FS_EMIT];
        float val[FS_EMIT];
        uint32_t cls = 0;   // bit u: gt, bit 4+u: eq
#pragma unroll
        for (int u = 0; u < FS_EMIT; ++u) {
            const uint32_t p = base + (uint32_t)tid * FS_EMIT + u;
            idx[u] = 0;
            val[u] = 0.f;
            if (p < nc) {
                idx[u] = F.cidx[p];
                val[u] = F.cval[p];
                const uint32_t key = key_of(val[u]);
                if (key > Tk) cls |= 1u << u;
                else if (key == Tk) cls |= 1u << (4 + u);
            }
        }
        const uint64_t mine = ((uint64_t)__popc(cls & 0xFu) << 32) | (uint64_t)__popc(cls >> 4);
        uint64_t tot;
        const uint64_t ex = block_excl_scan(mine, F.scan, &tot);
        uint32_t g = run_gt + (uint32_t)(ex >> 32);
        uint32_t e = run_eq + (uint32_t)(ex & 0xFFFFFFFFu);
#pragma unroll
        for (int u = 0; u < FS_EMIT; ++u) {
            bool take = false;
            uint32_t rank = 0;
            if ((cls >> u) & 1u) {
                rank = g + (e < q ? e : q);
                take = true;
                ++g;
            } else if ((cls >> (4 + u)) & 1u) {
                take = e < q;
                rank = g + e;
                ++e;
            }
            if (take && rank < k) {
                out_idx[rank] = (int32_t)((int64_t)idx[u] - idx_off);
                out_val[rank] = val[u];
                src.resid[idx[u]] = 0.0f;
            }
        }
        run_gt += (uint32_t)(tot >> 32);
        run_eq += (uint32_t)(tot & 0xFFFFFFFFu);
    }
}

// Exact counts of key > Tk and key == Tk among the staged candidates.
__device__ __forceinline__ void fs_count_exact(const FlatShared& F, uint32_t nc, uint32_t Tk,
                                               uint32_t& g, uint32_t& e) {
    for (uint32_t p = threadIdx.x; p < nc; p += FS_THREADS) {
        const uint32_t key = key_of(F.cval[p]);
        g += key > Tk;
        e += key == Tk;
    }
}

// The rescan of the residual when the candidates cannot hold the answer
// (out of line: it is rare, and the main path's straight-line code is what
// every block fetches).
__device__ __noinline__ void fs_fallback(const FlatParams& p, SelShared& S) {
    CompressSrc d = p.src;
    const SelCommon cm = p.cm;
    d.dense = 1;
    uint32_t epoch = 0;
    std_select(d, cm, epoch, S, 1);
}

// The k-th key's bin holds more candidates than the entry list (heavy ties
// or a crowded bin): a global digit-2 histogram of the bin, then exact
// counts of every block, two more grid-wide steps.  Out of line (rare).
// out: T, the tie quota, this block's counts above / equal to T before it.
// Returns false if a wait gave up or the counts did not add up.
__device__ __noinline__ bool fs_crowded(const FlatParams& p, FlatShared& F, SelShared& S,
                                        uint32_t epoch, uint32_t w0, uint32_t w1,
                                        uint32_t rounds, uint32_t nc_last, uint32_t T0,
                                        uint32_t sh, uint32_t b1, uint32_t rem) {
    const CompressSrc& src = p.src;
    const SelCommon& cm = p.cm;
    const int tid = threadIdx.x, c = blockIdx.x;
    uint32_t* status = &cm.ctrl->status;
    const uint32_t lmask = (1u << sh) - 1u;
    uint32_t Tk, q;
    ChunkRegs r;
    // the k-th key's bin holds more candidates than the entry list: a
    // global digit-2 histogram of the bin, then exact counts of every
    // block (two more grid-wide steps)
    if (c == 0 && tid == 0) cm.ctrl->r2_path = 1;
    for (int i = tid; i < REL_BINS; i += FS_THREADS) F.hist[i] = 0;
    __syncthreads();
    for (uint32_t wr = w0; wr < w1;) {
        uint32_t nt = 0, nc = nc_last;
        if (rounds > 1) {
            fs_load_chunk(src, wr + tid, w1, r);
            nt = fs_stage_round(src, F, wr, w1, r, T0, status);
            nc = F.nc;
        }
        for (uint32_t p0 = tid; p0 < nc; p0 += FS_THREADS) {
            const uint32_t rel = key_of(F.cval[p0]) - T0;
            if (min(rel >> sh, (uint32_t)(REL_BINS - 1)) == b1) atomicAdd(&F.hist[rel & lmask], 1u);
        }
        __syncthreads();
        if (rounds == 1) break;
        wr += nt;
    }
    {
        uint32_t* g2 = src.h(0, CH_R2);
        for (int i = tid; i < REL_BINS; i += FS_THREADS)
            if (F.hist[i]) atomicAdd(&g2[i], F.hist[i]);
    }
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return false;
    stage_words(F.hist, src.h(0, CH_R2), REL_BINS, REL_BINS);
    __syncthreads();
    fs_find2(F.hist, rem, rem, F);
    if (!F.fr1.ok) {
        if (tid == 0) atomicOr(status, ST_INCONSISTENT);
        return false;
    }
    Tk = T0 + (b1 << sh) + F.fr1.bin;
    q = rem - F.fr1.above;
    uint32_t g = 0, e = 0;
    if (rounds == 1) {
        fs_count_exact(F, nc_last, Tk, g, e);
    } else {
        for (uint32_t wr = w0; wr < w1;) {
            fs_load_chunk(src, wr + tid, w1, r);
            const uint32_t nt = fs_stage_round(src, F, wr, w1, r, T0, status);
            fs_count_exact(F, F.nc, Tk, g, e);
            __syncthreads();
            wr += nt;
        }
    }
    const uint64_t both = block_sum(((uint64_t)g << 32) | e, F.scan);
    if (tid == 0) {
        Slot sl = cm.slots[c];
        sl.gt_last = (uint32_t)(both >> 32);
        sl.eq_last = (uint32_t)both;
        cm.slots[c] = sl;
    }
    if (!grid_barrier(cm.bar, epoch, status, &S.flag)) return false;
    mark_phase(cm.ctrl, 3);
    const uint32_t bg = fs_slots_before(cm.slots, c, 4, F);
    const uint32_t be = fs_slots_before(cm.slots, c, 5, F);
    if (tid == 0) {
        F.crowd[0] = Tk;
        F.crowd[1] = q;
        F.crowd[2] = bg;
        F.crowd[3] = be;
    }
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(FS_THREADS, 1)
flat_select_kernel(const __grid_constant__ FlatParams p) {
    extern __shared__ __align__(16) unsigned char fs_smem[];
    FlatShared& F = *reinterpret_cast<FlatShared*>(fs_smem);
    __shared__ SelShared S;   // the rescan fallback's state
    // the next kernel on the stream may be scheduled now; it waits for this
    // grid to finish before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const CompressSrc& src = p.src;
    const SelCommon& cm = p.cm;
    Ctrl* ctrl = cm.ctrl;
    uint32_t* status = &ctrl->status;
    const int tid = threadIdx.x, c = blockIdx.x, G = gridDim.x;
    mark_phase(ctrl, 0);
    const BlockSpan block_span(ctrl);
    uint32_t epoch = 0;
    const uint32_t stall = ctrl->stall;

    const SegMeta m = src.meta[0];
    const uint32_t T0 = m.T0, sh = m.shift, k = m.k;
    const uint32_t W = src.num_wt;
    const uint32_t per = (W + G - 1) / G;
    const uint32_t w0 = min((uint32_t)c * per, W), w1 = min(w0 + per, W);

    // loads issued together: this block's first chunk of tile records and R1
    ChunkRegs r;
    fs_load_chunk(src, w0 + tid, w1, r);
    static_assert(REL_BINS == 8 * FS_THREADS, "R1 load");
    {
        const uint4* h4 = reinterpret_cast<const uint4*>(src.h(0, CH_R1));
        const uint4 a = h4[tid], b = h4[tid + FS_THREADS];
        uint4* s4 = reinterpret_cast<uint4*>(F.hist);
        s4[tid] = a;
        s4[tid + FS_THREADS] = b;
    }
    for (int i = tid; i < FS_WARPS * 32; i += FS_THREADS) F.wbm[i] = 0u;
    __syncthreads();
    // the k-th key's bin b1, and the (3k/2)-th key's bin for the next call's
    // hint
    fs_find2(F.hist, k, k + k / 2, F);
    mark_phase(ctrl, 1);
    const FindResult f1 = F.fr1;
    const uint32_t total = F.total;
    const bool cand_ok = !src.force_dense && k > 0 && f1.ok && f1.bin != (uint32_t)(REL_BINS - 1) &&
                         (uint64_t)total <= src.cap;
    if (c == 0 && tid == 0) {
        ctrl->mode = cand_ok ? 0u : 1u;
        ctrl->cand_total = total;
    }
    if (!cand_ok) {
        // every block takes the same decision: the standard-digit rescan;
        // the threshold that led here is not offered to the next call
        if (c == 0 && tid == 0 && p.hint) p.hint->tag = 0;
        fs_fallback(p, S);
        return;
    }
    const uint32_t b1 = f1.bin;
    const uint32_t rem = k - f1.above;
    const uint32_t lmask = (1u << sh) - 1u;
    uint32_t hint_T0 = 0;
    if (c == 0 && tid == 0 && p.hint) {
        // next call: the threshold where this call's (3k/2)-th key lies (or
        // this one's T0 if there were fewer candidates), with the widest
        // relative digits (4,095 bins of 2^12 keys: up to four times T0 in
        // value), so that a k-th key that grows from step to step stays in
        // range
        const uint32_t bt = F.fr2.ok ? F.fr2.bin : 0u;
        hint_T0 = min(T0 + (bt << sh), 0x7F800001u);
    }

    // ---- A: stage, classify, publish
    uint32_t gt_b = 0, in_b = 0;
    uint32_t rounds = 0, nc_last = 0;
    for (uint32_t wr = w0; wr < w1;) {
        if (wr != w0) fs_load_chunk(src, wr + tid, w1, r);
        const uint32_t nt = fs_stage_round(src, F, wr, w1, r, T0, status);
        if (rounds == 0) mark_phase(ctrl, 4);
        const uint32_t nc = F.nc;
        // count first, reserve this round's entries with one atomic, then
        // list them (no dependent global atomic per pass)
        uint32_t in_t = 0;
        for (uint32_t q = tid; q < nc; q += FS_THREADS) {
            const uint32_t bin = min((key_of(F.cval[q]) - T0) >> sh, (uint32_t)(REL_BINS - 1));
            gt_b += bin > b1;
            in_t += bin == b1;
        }
        uint32_t in_r;
        uint32_t at = block_excl_scan(in_t, F.red, &in_r);
        if (tid == 0) F.pre[1] = in_r ? atomicAdd(src.ent_cnt, in_r) : 0u;
        __syncthreads();
        at += F.pre[1];
        if (in_t) {
            for (uint32_t q = tid; q < nc; q += FS_THREADS) {
                const uint32_t rel = key_of(F.cval[q]) - T0;
                if (min(rel >> sh, (uint32_t)(REL_BINS - 1)) == b1) {
                    if (at < ENT_PER) src.ent[at] = ((uint32_t)c << 12) | (rel & lmask);
                    ++at;
                }
            }
        }
        in_b += in_r;
        ++rounds;
        nc_last = nc;
        wr += nt;
    }
    gt_b = block_sum(gt_b, F.red);
    if (tid == 0) {
        Slot sl;
        memset(&sl, 0, sizeof(sl));
        sl.gt_first = gt_b;
        sl.eq_first = in_b;
        cm.slots[c] = sl;
    }
    mark_phase(ctrl, 5);
    mark_last(ctrl, SPAN_GATHER_LAST);
    if (!grid_barrier(cm.bar, epoch, status, &S.flag, stall)) return;
    mark_phase(ctrl, 2);

    // ---- B: T, the tie quota and this block's output offset.  The entry
    // words, their count and the earlier blocks' counts are loaded together
    // (slots past the count hold stale words and are dropped).
    constexpr int EPT = (int)ENT_PER / FS_THREADS;
    uint32_t ev[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) ev[u] = src.ent[tid + u * FS_THREADS];
    const uint32_t E = *reinterpret_cast<const volatile uint32_t*>(src.ent_cnt);
    uint32_t gt_slots = 0;
    if (tid < 32) {
        // warp 0: the counts above b1 of blocks [0, c), 8 loads per lane in flight
        for (int j0 = 0; j0 < c; j0 += 256) {
            uint32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 32 * u + tid;
                v[u] = j < c ? cm.slots[j].gt_first : 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) gt_slots += v[u];
        }
        gt_slots = warp_sum(gt_slots);
    }
    uint32_t Tk, q, before_gt, before_eq;
    if (E <= ENT_PER) {
#pragma unroll
        for (int u = 0; u < EPT; ++u)
            if ((uint32_t)(tid + u * FS_THREADS) >= E) ev[u] = DEAD;
        for (int i = tid; i < REL_BINS; i += FS_THREADS) F.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < EPT; ++u)
            if (ev[u] != DEAD) atomicAdd(&F.hist[ev[u] & 4095u], 1u);
        __syncthreads();
        fs_find2(F.hist, rem, rem, F);
        if (!F.fr1.ok) {
            if (tid == 0) atomicOr(status, ST_INCONSISTENT);
            return;
        }
        const uint32_t t = F.fr1.bin;
        Tk = T0 + (b1 << sh) + t;
        q = rem - F.fr1.above;
        uint32_t g = tid == 0 ? gt_slots : 0u, e = 0;
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            if (ev[u] != DEAD && (int)(ev[u] >> 12) < c) {
                g += (ev[u] & 4095u) > t;
                e += (ev[u] & 4095u) == t;
            }
        }
        const uint64_t both = block_sum(((uint64_t)g << 32) | e, F.scan);
        before_gt = (uint32_t)(both >> 32);
        before_eq = (uint32_t)both;
    } else {
        if (!fs_crowded(p, F, S, epoch, w0, w1, rounds, nc_last, T0, sh, b1, rem)) return;
        Tk = F.crowd[0];
        q = F.crowd[1];
        before_gt = F.crowd[2];
        before_eq = F.crowd[3];
    }
    mark_last(ctrl, SPAN_OFFSET_LAST);
    mark_phase(ctrl, 6);

    // ---- C: emission in index order
    int32_t* out_idx = src.out_idx + m.out_base;
    float* out_val = src.out_val + m.out_base;
    uint32_t run_gt = before_gt, run_eq = before_eq;
    if (rounds == 1) {
        fs_emit(src, F, nc_last, Tk, q, k, out_idx, out_val, m.off, run_gt, run_eq);
    } else {
        for (uint32_t wr = w0; wr < w1;) {
            fs_load_chunk(src, wr + tid, w1, r);
            const uint32_t nt = fs_stage_round(src, F, wr, w1, r, T0, status);
            fs_emit(src, F, F.nc, Tk, q, k, out_idx, out_val, m.off, run_gt, run_eq);
            __syncthreads();
            wr += nt;
        }
    }
    if (c == 0 && tid == 0 && p.hint) {
        Hint h;
        memset(&h, 0, sizeof(h));
        h.tag = (*reinterpret_cast<volatile uint32_t*>(status) == 0) ? p.hint_tag : 0ull;
        h.T0 = hint_T0;
        h.shift = REL_MAX_SHIFT;
        *p.hint = h;
    }
    mark_phase(ctrl, 7);
}

}  // namespace tke
