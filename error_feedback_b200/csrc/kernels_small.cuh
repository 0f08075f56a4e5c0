// The whole error-feedback step of one small tensor in one launch
// ("Sparsified SGD with Memory", abstract: send the top k, keep the rest in
// memory; "A Distributed Synchronous SGD Algorithm with Global Top-k
// Sparsification", ABSTRACT: the k largest absolute values, the lower index
// first among equal ones).
//
// For a tensor that one wave of blocks holds in shared memory (one block per
// SM, up to SK_MAX elements each) latency, not bytes, bounds the step.  Each
// block owns a contiguous slice:
//   1  acc = fmaf(lr, grad, residual) streamed once (written back to the
//      residual, kept in shared memory); the elements whose key reaches the
//      previous call's threshold T0 (a hint kept in the workspace) are listed,
//      in index order, in the block's region of the candidate arrays;
//   2  every block announces its count in its own arrival word, tagged with
//      this call's tag (no counter to clear beforehand), and waits for every
//      block's word; all blocks then hold the same counts and take the same
//      decision:
//   3  the threshold decides (at least k and at most SK_CAP1 candidates):
//      every block loads the keys of all candidates (block order is index
//      order), resolves the k-th key T and the tie quota q by two (three)
//      histogram passes over bins relative to T0 whose width the hint also
//      carries, counts the candidates above / equal to T in the blocks before
//      it, and emits its own selected elements from shared memory; no second
//      exchange;
//   4  otherwise (no hint, too few or too many candidates, or the k-th key
//      beyond the bins' range) block 0 clears the exact path's counters and
//      releases the others through one tagged word, and every block runs it:
//      an 8,192-bin histogram of key >> 18 of every element, added into a
//      global histogram; after a grid-wide exchange every block finds the bin
//      b1 of the k-th key, counts its elements above b1 and lists those in b1
//      (block << 18 | low 18 key bits) in a grid-wide entry list; after a
//      second exchange every block reads the list and resolves T and q from
//      it (bits 17..9, then 8..0) and its output offset from the earlier
//      blocks' counts and entries; it emits its selected elements.  A bin b1
//      with more elements than the entry list takes two summed digit passes
//      and an exact-count exchange instead (three more grid-wide steps).
// Either way block 0 leaves the next call's threshold: the lower edge of the
// bin of the (3k/2)-th largest element, and a bin width that covers four
// times the distance from there to the k-th key.  The call's tag mixes a
// host-issued number with a counter in the workspace that block 0 advances
// every call, so that arrival words left by earlier calls (or by a replayed
// graph) never match it; errors are recorded with the tag as well.
#pragma once

#include "common.cuh"
#include "kernels_compress.cuh"
#include "kernels_select.cuh"

namespace tke {

constexpr int SK_THREADS = 512;
constexpr int SK_MAX = 16384;            // elements per block
constexpr int SK_BINS = 8192;            // exact path, digit 1: key >> 18
constexpr int SK_LOW = 18;               // bits below digit 1
constexpr int SK_D2 = SK_LOW - 9;        // digit 2: bits 17..9 (512 bins); digit 3: bits 8..0
constexpr int SK_MIN_PER_BLOCK = 2048;   // fewer blocks for smaller tensors
constexpr int SK_VEC = 8;                // float4 of each input a thread loads at once
constexpr int SK_GRID_MAX = 148;         // blocks: one per SM of a 148-SM part
constexpr int64_t SK_N_MAX = (int64_t)SK_GRID_MAX * SK_MAX;
constexpr uint32_t SK_CAP1 = 8192;       // candidates the threshold path takes
constexpr uint32_t SK_HINT_KMAX = SK_CAP1 / 4;   // larger k: no threshold hint
constexpr int SK_RBINS = 4096;           // threshold path: bins relative to T0
constexpr uint32_t SK_RSH_MAX = 12;      // their width: at most 2^12 keys (hinted)
constexpr uint32_t SK_RSH_ALL = 19;      // 4096 << 19 = 2^31: every key (T0 = 0)
constexpr uint32_t SK_PATH_TAG = 0x534B3031u;
static_assert(SK_GRID_MAX < SK_THREADS, "one arrival word per thread");
static_assert(SK_GRID_MAX < 256, "block numbers fit a byte");
static_assert(2 * SK_RBINS <= SK_BINS, "threshold path's two histograms");

// Arrival word of one block: this call's tag, written after the count.
struct SkFlag {
    uint64_t tag;
    uint32_t count;     // candidates the block listed
    uint32_t pad;
};

// Workspace words of the one-launch path.  The arrival words are never
// cleared (tags make them call-specific); the arrival counter of call s,
// arrive[s & 1], is cleared by call s - 1, which then marks it valid for call
// s in armed[s & 1] (a workspace that no call has prepared yet falls back to
// the arrival words).
struct SkSync {
    uint64_t seq;       // advanced by block 0 every call
    uint64_t go_tag;    // block 0's release word for the exact path
    uint64_t armed[2];  // sk_arm(s): arrive[s & 1] was cleared for call s
    uint32_t arrive[2];
    uint32_t pad[2];
    SkFlag flag[SK_GRID_MAX + 1];   // one past the grid: never written (test hook)
};

__device__ __forceinline__ uint64_t sk_arm(uint64_t seq) {
    return (seq * 0xD6E8FEB86659FD93ull) ^ 0x9E3779B97F4A7C15ull;
}

struct SmallShared {
    float acc[SK_MAX];          // this block's acc
    uint32_t own[SK_CAP1];      // threshold path: slice positions of its candidates
    uint32_t hist[SK_BINS];     // threshold path: pass 1 [0, 4096), pass 2 above
    uint32_t ckey[SK_CAP1];     // threshold path: every candidate's key, index order
    uint64_t scan[33];
    uint32_t red[33];
    FindResult fr, fr2;
    uint32_t pre;
    int flag;
    uint32_t pre_blk[SK_GRID_MAX + 1];  // candidates of the blocks before
    uint64_t tag, seq;
    uint32_t T0, sh, E, armed;
    uint32_t cnt[2];            // threshold path: earlier candidates above / at T
    uint32_t lkey[64], lpos[64];        // threshold path: the k-th key's bin, when short
    uint32_t lcnt, lsel[3];
};

struct SmallParams {
    const float* grad;
    float* resid;
    int64_t n;
    float lr;
    uint32_t k;
    int32_t* out_idx;      // the tensor's outputs (out_base applied)
    float* out_val;
    Ctrl* ctrl;
    uint32_t* hist;        // [SK_BINS] global digit-1 histogram (exact path)
    uint32_t* hist2;       // [512 + 512] crowded path's digit histograms
    uint32_t* ent;         // [ENT_PER] entry list
    uint32_t* ent_cnt;     // its length
    Slot* slots;           // [grid] per-block counts
    SkSync* sync;          // arrival and release words
    uint32_t* cand_idx;    // [n] candidate regions: block c's at its slice's start
    float* cand_val;
    Hint* hint;            // the threshold hint (read, then rewritten by block 0)
    uint64_t hint_tag;     // 0: no hint for this call
    uint64_t call_tag;     // host-issued, distinct per call
    uint32_t force_t0;     // test hook: threshold 0 (every element a candidate)
    uint32_t stall;        // test hook: every block also waits for a block past the grid
};

__device__ __forceinline__ uint64_t sk_mix(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return (x ^ (x >> 31)) | 1ull;      // never 0: zeroed memory matches no call
}

// Record error bits for this call: the status word holds the tag of the call
// whose errors it carries, so that no call has to clear it first.
__device__ __forceinline__ void sk_fail(Ctrl* ctrl, uint32_t tag32, uint32_t bits) {
    unsigned long long* w = reinterpret_cast<unsigned long long*>(&ctrl->sk_status);
    unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(w);
    for (;;) {
        const unsigned long long nv = (uint32_t)(old >> 32) == tag32
                                          ? (old | bits)
                                          : (((unsigned long long)tag32 << 32) | bits);
        const unsigned long long seen = atomicCAS(w, old, nv);
        if (seen == old) return;
        old = seen;
    }
}

// Wait until *w holds tag; false after SPIN_LIMIT polls or WAIT_LIMIT_NS.
__device__ __forceinline__ bool sk_wait_tag(const uint64_t* w, uint64_t tag) {
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (ld_acquire_u64(w) != tag) {
        ++it;
        if (it == 33) t0 = global_ns();
        if (it > SPIN_LIMIT || (it > 33 && (it & 63u) == 0 && global_ns() - t0 > WAIT_LIMIT_NS))
            return false;
        if (it > 32) __nanosleep(64);
    }
    return true;
}

// Wait until *w reaches target; false after SPIN_LIMIT polls or WAIT_LIMIT_NS.
__device__ __forceinline__ bool sk_wait_count(const uint32_t* w, uint32_t target) {
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (ld_acquire_u32(w) < target) {
        ++it;
        if (it == 33) t0 = global_ns();
        if (it > SPIN_LIMIT || (it > 33 && (it & 63u) == 0 && global_ns() - t0 > WAIT_LIMIT_NS))
            return false;
        if (it > 32) __nanosleep(64);
    }
    return true;
}

// Ordered passes over positions [0, cnt) of a shared-memory array: warp w
// owns a contiguous chunk and its lanes take consecutive positions, so that
// no two lanes of a warp hit one bank.

// The positions where pred holds, in index order: out(i, j) for each, j its
// rank among them.  Returns their number (every thread).  s_warp: 17 words.
template <class Pred, class Out>
__device__ __forceinline__ uint32_t sk_list_ordered(uint32_t cnt, uint32_t* s_warp, Pred pred,
                                                    Out out) {
    constexpr uint32_t NW = SK_THREADS / 32;
    const uint32_t w = warp_id(), lane = lane_id();
    const uint32_t C = ((cnt + NW - 1) / NW + 31) & ~31u;
    const uint32_t a0 = min(w * C, cnt), a1 = min(a0 + C, cnt);
    uint32_t n = 0;
    for (uint32_t b = a0; b < a1; b += 32)
        n += __popc(__ballot_sync(~0u, b + lane < a1 && pred(b + lane)));
    if (lane == 0) s_warp[w] = n;
    __syncthreads();
    if (w == 0) {
        const uint32_t v = lane < NW ? s_warp[lane] : 0u;
        const uint32_t inc = warp_incl_scan(v);
        if (lane < NW) s_warp[lane] = inc - v;
        if (lane == NW - 1) s_warp[NW] = inc;
    }
    __syncthreads();
    uint32_t r = s_warp[w];
    const uint32_t total = s_warp[NW];
    const uint32_t below = (1u << lane) - 1u;
    for (uint32_t b = a0; b < a1; b += 32) {
        const bool hit = b + lane < a1 && pred(b + lane);
        const uint32_t bal = __ballot_sync(~0u, hit);
        if (hit) out(b + lane, r + __popc(bal & below));
        r += __popc(bal);
    }
    __syncthreads();
    return total;
}

// Emission in index order: cls(i) is 2 for a key above T, 1 for a key equal
// to T, else 0; emit(i, rank) for every selected position, rank = the earlier
// positions above T plus min(the earlier positions equal to T, q), counting
// gt0 / eq0 before position 0.  s_warp: 16 words.
template <class Cls, class Emit>
__device__ __forceinline__ void sk_emit_ordered(uint32_t cnt, uint32_t gt0, uint32_t eq0,
                                                uint32_t q, uint32_t k, uint64_t* s_warp,
                                                Cls cls, Emit emit) {
    constexpr uint32_t NW = SK_THREADS / 32;
    const uint32_t w = warp_id(), lane = lane_id();
    const uint32_t C = ((cnt + NW - 1) / NW + 31) & ~31u;
    const uint32_t a0 = min(w * C, cnt), a1 = min(a0 + C, cnt);
    uint32_t g = 0, e = 0;
    for (uint32_t b = a0; b < a1; b += 32) {
        const uint32_t c = b + lane < a1 ? cls(b + lane) : 0u;
        g += __popc(__ballot_sync(~0u, c == 2u));
        e += __popc(__ballot_sync(~0u, c == 1u));
    }
    if (lane == 0) s_warp[w] = ((uint64_t)g << 32) | e;
    __syncthreads();
    if (w == 0) {
        const uint64_t v = lane < NW ? s_warp[lane] : 0ull;
        const uint64_t inc = warp_incl_scan(v);
        if (lane < NW) s_warp[lane] = inc - v;
    }
    __syncthreads();
    uint32_t rg = gt0 + (uint32_t)(s_warp[w] >> 32), re = eq0 + (uint32_t)s_warp[w];
    const uint32_t below = (1u << lane) - 1u;
    for (uint32_t b = a0; b < a1; b += 32) {
        const uint32_t c = b + lane < a1 ? cls(b + lane) : 0u;
        const uint32_t bg = __ballot_sync(~0u, c == 2u), be = __ballot_sync(~0u, c == 1u);
        const uint32_t mg = rg + __popc(bg & below), me = re + __popc(be & below);
        uint32_t rank = 0xFFFFFFFFu;
        if (c == 2u) rank = mg + min(me, q);
        else if (c == 1u && me < q) rank = mg + me;
        if (rank < k) emit(b + lane, rank);
        rg += __popc(bg);
        re += __popc(be);
    }
    __syncthreads();
}

// block_find_bin for two ranks with one scan (r1 -> *o1, r2 -> *o2).
__device__ __forceinline__ void sk_find_two(const uint32_t* h, int nb, uint32_t r1, uint32_t r2,
                                            uint32_t* s_red, FindResult* o1, FindResult* o2) {
    const int t = threadIdx.x;
    const int per = nb / (int)blockDim.x;
    const int hi = nb - t * per;   // thread 0 owns the top bins
    const int lo = hi - per;
    uint32_t sum = 0;
    for (int i = 0; i < per; ++i) sum += h[lo + ((i + t) & (per - 1))];
    if (t == 0) o1->ok = o2->ok = 0;
    uint32_t tot;
    const uint32_t ex = block_excl_scan(sum, s_red, &tot);
    for (int w = 0; w < 2; ++w) {
        const uint32_t rem = w == 0 ? r1 : r2;
        FindResult* out = w == 0 ? o1 : o2;
        if (ex < rem && ex + sum >= rem) {
            uint32_t run = ex;
            for (int b = hi - 1; b >= lo; --b) {
                const uint32_t cnt = h[b];
                if (run + cnt >= rem) {
                    out->bin = (uint32_t)b;
                    out->above = run;
                    out->cnt = cnt;
                    out->ok = 1;
                    break;
                }
                run += cnt;
            }
        }
    }
    __syncthreads();
}

// Rank of the element whose bin sets the next call's threshold: above the
// k-th, so that the next call's k-th key may be a little lower and still
// pass, and low enough that the growth of |acc| under error feedback keeps
// the next list short.
__device__ __forceinline__ uint32_t sk_hint_rank(uint32_t k) { return k + k / 2; }

// The next call's hint: threshold T0n, and the bin width 2^sh that makes the
// SK_RBINS bins cover four times the distance from T0n to the k-th key Tk
// (at least an eighth of an octave, at most SK_RSH_MAX).
__device__ __forceinline__ void sk_write_hint(const SmallParams& p, uint32_t T0n, uint32_t Tk) {
    const uint64_t d = Tk >= T0n ? (uint64_t)(Tk - T0n) : 0ull;
    const uint64_t need = max(4ull * d + 1ull, 1ull << 20);
    uint32_t sh = 0;
    while (sh < SK_RSH_MAX && ((uint64_t)SK_RBINS << sh) < need) ++sh;
    Hint h;
    memset(&h, 0, sizeof(h));
    h.tag = p.hint_tag;
    h.T0 = T0n;
    h.shift = sh;
    *p.hint = h;
}

// Sum over blocks j < c of word f of their slots (warp 0), every thread gets it.
__device__ __forceinline__ uint32_t sk_slots_before(const Slot* slots, int c, int f,
                                                    SmallShared& K) {
    if (threadIdx.x < 32) {
        uint32_t s = 0;
        for (int j0 = 0; j0 < c; j0 += 256) {
            uint32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 32 * u + (int)threadIdx.x;
                v[u] = j < c ? reinterpret_cast<const uint32_t*>(slots + j)[f] : 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        s = warp_sum(s);
        if (threadIdx.x == 0) K.pre = s;
    }
    __syncthreads();
    const uint32_t r = K.pre;
    __syncthreads();
    return r;
}

// Global histogram hg (nb bins, nb a multiple of the block size) into shared
// memory, then the bin of the rem-th largest (result in K.fr).
__device__ __forceinline__ void sk_find_global(const uint32_t* hg, int nb, uint32_t rem,
                                               SmallShared& K) {
    for (int i = threadIdx.x; i < nb; i += blockDim.x) K.hist[i] = hg[i];
    __syncthreads();
    block_find_bin(K.hist, nb, rem, K.red, &K.fr);
}

// Exact path, crowded k-th-key bin: digits 17..9 and 8..0 of the elements in
// bin b1 by summed global histograms, then exact counts of every block.
// Writes T, the tie quota and this block's counts before it to out[0..3]
// (shared memory).  Returns 0, or the ST_* bits of what failed.  Out of line.
__device__ __noinline__ uint32_t sk_crowded(const SmallParams& p, SmallShared& K, uint32_t epoch,
                                            uint32_t m, uint32_t b1, uint32_t rem, uint32_t* out) {
    const int tid = threadIdx.x, c = blockIdx.x;
    uint32_t* scratch = &p.ctrl->status;      // grid_barrier's own record; unused here
    if (c == 0 && tid == 0) p.ctrl->r2_path = 1;
    // digit 2: bits 17..9 of the elements in b1
    for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        if ((key >> SK_LOW) == b1) atomicAdd(&K.hist[(key >> 9) & 511u], 1u);
    }
    __syncthreads();
    for (int i = tid; i < 512; i += SK_THREADS)
        if (K.hist[i]) atomicAdd(&p.hist2[i], K.hist[i]);
    if (!grid_barrier(&p.ctrl->bar, epoch, scratch, &K.flag)) return ST_TIMEOUT;
    sk_find_global(p.hist2, 512, rem, K);
    if (!K.fr.ok) return ST_INCONSISTENT;
    const uint32_t t1 = K.fr.bin;
    const uint32_t rem2 = rem - K.fr.above;
    const uint32_t pre = (b1 << SK_D2) | t1;          // key >> 9 of the class
    __syncthreads();
    // digit 3: bits 8..0 of the elements in that class
    for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        if ((key >> 9) == pre) atomicAdd(&K.hist[key & 511u], 1u);
    }
    __syncthreads();
    for (int i = tid; i < 512; i += SK_THREADS)
        if (K.hist[i]) atomicAdd(&p.hist2[512 + i], K.hist[i]);
    if (!grid_barrier(&p.ctrl->bar, epoch, scratch, &K.flag)) return ST_TIMEOUT;
    sk_find_global(p.hist2 + 512, 512, rem2, K);
    if (!K.fr.ok) return ST_INCONSISTENT;
    const uint32_t Tk = (pre << 9) | K.fr.bin;
    const uint32_t q = rem2 - K.fr.above;
    __syncthreads();
    uint32_t g = 0, e = 0;
    for (uint32_t i = tid; i < m; i += SK_THREADS) {
        const uint32_t key = key_of(K.acc[i]);
        g += key > Tk;
        e += key == Tk;
    }
    const uint64_t both = block_sum(((uint64_t)g << 32) | e, K.scan);
    if (tid == 0) {
        p.slots[c].gt_last = (uint32_t)(both >> 32);
        p.slots[c].eq_last = (uint32_t)both;
    }
    if (!grid_barrier(&p.ctrl->bar, epoch, scratch, &K.flag)) return ST_TIMEOUT;
    const uint32_t bg = sk_slots_before(p.slots, c, 4, K);
    const uint32_t be = sk_slots_before(p.slots, c, 5, K);
    if (tid == 0) {
        out[0] = Tk;
        out[1] = q;
        out[2] = bg;
        out[3] = be;
    }
    __syncthreads();
    return 0;
}

// Threshold path, in every block: the E candidates of the G blocks' regions
// (every element with key >= T0) decide the top k.  Warp w gathers the keys
// of blocks w, w + 16, ... into shared memory in index order and counts them
// in SK_RBINS bins of (key - T0) >> sh, the top one open above; the k-th key
// T and the tie quota q follow from those bins and the sh bits below (in two
// steps above 12 bits).  Writes T, q and this block's counts of earlier
// candidates above / equal to T to out[0..3].  Returns false when the k-th
// key lies in the top bin (the exact path takes over).  The histogram words
// [0, 2 * SK_RBINS) and K.cnt must be zero on entry.  Block 0 also writes the
// next hint.
__device__ __forceinline__ bool sk_threshold_select(const SmallParams& p, SmallShared& K, int G,
                                                    int64_t per, uint32_t E, uint32_t T0,
                                                    uint32_t sh, uint32_t* out) {
    const int tid = threadIdx.x, c = blockIdx.x;
    const uint32_t k = p.k;
    const uint32_t lane = lane_id(), w = warp_id();
    constexpr int NW = SK_THREADS / 32;
    constexpr int R = (SK_GRID_MAX + NW - 1) / NW;      // blocks per warp at most
    uint32_t* h1 = K.hist;
    uint32_t* h2 = K.hist + SK_RBINS;
    // ---- keys in index order: warp w takes blocks w, w + 16, ...; the first
    // 64 candidates of each block all loaded at once, the rest after
    {
        float v[2][R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int j = (int)w + r * NW;
            if (j < G) {
                const uint32_t cnt = K.pre_blk[j + 1] - K.pre_blk[j];
                const float* src = p.cand_val + min((int64_t)j * per, p.n);   // other blocks'
                if (lane < cnt) v[0][r] = __ldcg(src + lane);
                if (32 + lane < cnt) v[1][r] = __ldcg(src + 32 + lane);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int j = (int)w + r * NW;
            if (j < G) {
                const uint32_t a = K.pre_blk[j], cnt = K.pre_blk[j + 1] - a;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (32u * h + lane < cnt) {
                        const uint32_t key = key_of(v[h][r]);
                        K.ckey[a + 32u * h + lane] = key;
                        atomicAdd(&h1[min((key - T0) >> sh, (uint32_t)(SK_RBINS - 1))], 1u);
                    }
                }
            }
        }
        for (int j = (int)w; j < G; j += NW) {
            const uint32_t a = K.pre_blk[j], cnt = K.pre_blk[j + 1] - a;
            const int64_t base = min((int64_t)j * per, p.n);
            for (uint32_t i = 64 + lane; i < cnt; i += 32) {
                const uint32_t key = key_of(__ldcg(p.cand_val + base + i));
                K.ckey[a + i] = key;
                atomicAdd(&h1[min((key - T0) >> sh, (uint32_t)(SK_RBINS - 1))], 1u);
            }
        }
    }
    __syncthreads();
    mark_phase(p.ctrl, 4);
    // ---- pass 1: the k-th key's bin (block 0: also the bin of the hint's rank)
    uint32_t hb = NO_KEY;
    const uint32_t rh = sk_hint_rank(k);
    if (c == 0 && p.hint_tag != 0 && rh <= E) {
        sk_find_two(h1, SK_RBINS, k, rh, K.red, &K.fr, &K.fr2);
        if (K.fr2.ok) hb = K.fr2.bin;
    } else {
        block_find_bin(h1, SK_RBINS, k, K.red, &K.fr);
    }
    const bool ok1 = K.fr.ok;
    const uint32_t b1 = K.fr.bin;
    const uint32_t rem = k - K.fr.above;
    if (!ok1 || b1 == (uint32_t)(SK_RBINS - 1)) return false;
    const uint32_t before = K.pre_blk[c];
    uint32_t Tk, rem2;
    if (K.fr.cnt <= 64u) {
        // ---- a short bin (the usual case): its entries into a list, with
        // the earlier blocks' candidates in higher bins counted on the way;
        // one warp then ranks the list
        uint32_t g = 0;
        for (uint32_t q = tid; q < E; q += SK_THREADS) {
            const uint32_t key = K.ckey[q];
            const uint32_t bin = min((key - T0) >> sh, (uint32_t)(SK_RBINS - 1));
            if (bin == b1) {
                const uint32_t at = atomicAdd(&K.lcnt, 1u);
                K.lkey[at] = key;
                K.lpos[at] = q;
            } else if (bin > b1 && q < before) {
                ++g;
            }
        }
        g = __reduce_add_sync(~0u, g);
        if (lane_id() == 0 && g) atomicAdd(&K.cnt[0], g);
        __syncthreads();
        mark_phase(p.ctrl, 5);
        if (tid < 32) {
            const uint32_t n1 = K.lcnt;
            // the rem-th largest key of the list: the key with fewer than rem
            // larger ones and at least rem at least as large
            uint32_t Tsel = 0;
            bool found = false;
            for (uint32_t j = tid; j < n1; j += 32) {
                const uint32_t kj = K.lkey[j];
                uint32_t gt = 0, ge = 0;
                for (uint32_t i = 0; i < n1; ++i) {
                    const uint32_t ki = K.lkey[i];
                    gt += ki > kj;
                    ge += ki >= kj;
                }
                if (gt < rem && rem <= ge) {
                    found = true;
                    Tsel = kj;
                }
            }
            const uint32_t who = __ballot_sync(~0u, found);
            const uint32_t T = who ? __shfl_sync(~0u, Tsel, __ffs(who) - 1) : 0u;
            uint32_t ga = 0, gb = 0, eb = 0;
            for (uint32_t j = tid; j < n1; j += 32) {
                const uint32_t kj = K.lkey[j];
                ga += kj > T;
                if (K.lpos[j] < before) {
                    gb += kj > T;
                    eb += kj == T;
                }
            }
            ga = warp_sum(ga);
            gb = warp_sum(gb);
            eb = warp_sum(eb);
            if (tid == 0) {
                K.lsel[0] = who ? 1u : 0u;
                K.lsel[1] = T;
                K.lsel[2] = rem - ga;
                K.cnt[0] += gb;
                K.cnt[1] = eb;
            }
        }
        __syncthreads();
        if (!K.lsel[0]) return false;
        Tk = K.lsel[1];
        rem2 = K.lsel[2];
    } else {
        // ---- pass 2: the bits below the bin (their top 12 when there are more)
        const uint32_t s2 = sh > 12u ? sh - 12u : 0u;          // bits left for pass 3
        const uint32_t nb2 = max(1u << (sh - s2), 512u);
        const uint32_t lmask = (1u << sh) - 1u;
        for (uint32_t q = tid; q < E; q += SK_THREADS) {
            const uint32_t r = K.ckey[q] - T0;
            if ((r >> sh) == b1) atomicAdd(&h2[(r & lmask) >> s2], 1u);
        }
        __syncthreads();
        mark_phase(p.ctrl, 5);
        block_find_bin(h2, (int)nb2, rem, K.red, &K.fr);
        const bool ok2 = K.fr.ok;
        const uint32_t t2 = K.fr.bin;
        rem2 = rem - K.fr.above;
        uint32_t low = t2 << s2;
        bool ok3 = true;
        if (s2 > 0) {
            // ---- pass 3 (threshold 0 only): the last s2 bits, in pass 1's words
            for (int i = tid; i < 512; i += SK_THREADS) h1[i] = 0;
            __syncthreads();
            const uint32_t pre3 = (b1 << (sh - s2)) | t2;
            for (uint32_t q = tid; q < E; q += SK_THREADS) {
                const uint32_t r = K.ckey[q] - T0;
                if ((r >> s2) == pre3) atomicAdd(&h1[r & ((1u << s2) - 1u)], 1u);
            }
            __syncthreads();
            block_find_bin(h1, 512, rem2, K.red, &K.fr);
            ok3 = K.fr.ok;
            low |= K.fr.bin;
            rem2 -= K.fr.above;
        }
        if (!ok2 || !ok3) return false;
        Tk = T0 + (b1 << sh) + low;
        // ---- earlier blocks' candidates above / equal to T: per warp, then
        // one shared-memory add per warp
        uint32_t g = 0, e = 0;
        for (uint32_t q = tid; q < before; q += SK_THREADS) {
            const uint32_t key = K.ckey[q];
            g += key > Tk;
            e += key == Tk;
        }
        g = __reduce_add_sync(~0u, g);
        e = __reduce_add_sync(~0u, e);
        if (lane_id() == 0 && (g | e)) {
            atomicAdd(&K.cnt[0], g);
            atomicAdd(&K.cnt[1], e);
        }
    }
    if (c == 0 && tid == 0 && p.hint_tag != 0) {
        if (hb != NO_KEY) {
            sk_write_hint(p, T0 + (hb << sh), Tk);
        } else {
            // fewer candidates than the hint's rank: an eighth of an octave lower
            sk_write_hint(p, T0 > (1u << 20) ? T0 - (1u << 20) : 0u, Tk);
        }
    }
    __syncthreads();
    if (tid == 0) {
        out[0] = Tk;
        out[1] = rem2;
        out[2] = K.cnt[0];
        out[3] = K.cnt[1];
    }
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(SK_THREADS, 1)
small_kernel(const __grid_constant__ SmallParams p) {
    extern __shared__ __align__(16) unsigned char sk_smem[];
    SmallShared& K = *reinterpret_cast<SmallShared*>(sk_smem);
    __shared__ uint32_t s_out[4];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    Ctrl* ctrl = p.ctrl;
    const int tid = threadIdx.x, c = blockIdx.x, G = gridDim.x;
    mark_phase(ctrl, 0);
    uint32_t epoch = 0;
    const uint32_t k = p.k;
    // this block's slice [e0, e0 + m), a multiple of 4 elements long
    int64_t per = (p.n + G - 1) / G;
    per = (per + 3) & ~(int64_t)3;
    const int64_t e0 = min((int64_t)c * per, p.n);
    const uint32_t m = (uint32_t)(min(e0 + per, p.n) - e0);
    // the call counter and the hint: read before this block arrives (block 0
    // rewrites them only after every block has arrived); the loads overlap
    // the streaming pass
    uint64_t seq = 0, htag = 0, armed = 0;
    uint32_t hT0 = 0, hsh = 0;
    if (tid == 0) {
        seq = *reinterpret_cast<volatile const uint64_t*>(&p.sync->seq);
        armed = *reinterpret_cast<volatile const uint64_t*>(&p.sync->armed[seq & 1]);
        htag = p.hint->tag;
        hT0 = p.hint->T0;
        hsh = p.hint->shift;
        if (c == 0) {
            // the next call's arrival counter (the call before this one, which
            // used it, is complete)
            p.sync->arrive[(seq + 1) & 1] = 0;
            p.sync->armed[(seq + 1) & 1] = sk_arm(seq + 1);
        }
    }

    // ---- 1: accumulate, keep
    const float* gp = p.grad + e0;
    float* rp = p.resid + e0;
    const float lr = p.lr;
    const bool vec = ((reinterpret_cast<uintptr_t>(gp) | reinterpret_cast<uintptr_t>(rp)) & 15u) == 0;
    if (vec) {
        // up to SK_VEC float4 of each input per thread in flight at once
        const uint32_t m4 = m >> 2;
        for (uint32_t b = 0; b < m4; b += SK_THREADS * SK_VEC) {
            float4 g[SK_VEC], r[SK_VEC];
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i < m4) {
                    g[u] = ld_stream(reinterpret_cast<const float4*>(gp) + i);
                    r[u] = ld_stream(reinterpret_cast<const float4*>(rp) + i);
                }
            }
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i >= m4) continue;
                float4 a;
                a.x = __fmaf_rn(lr, g[u].x, r[u].x);
                a.y = __fmaf_rn(lr, g[u].y, r[u].y);
                a.z = __fmaf_rn(lr, g[u].z, r[u].z);
                a.w = __fmaf_rn(lr, g[u].w, r[u].w);
                st_stream(reinterpret_cast<float4*>(rp) + i, a);
                reinterpret_cast<float4*>(K.acc)[i] = a;
            }
        }
        for (uint32_t i = 4 * m4 + tid; i < m; i += SK_THREADS) {
            const float a = __fmaf_rn(lr, __ldcs(gp + i), __ldcs(rp + i));
            __stcs(rp + i, a);
            K.acc[i] = a;
        }
    } else {
        for (uint32_t b = 0; b < m; b += SK_THREADS * SK_VEC) {
            float g[SK_VEC], r[SK_VEC];
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i < m) {
                    g[u] = __ldcs(gp + i);
                    r[u] = __ldcs(rp + i);
                }
            }
#pragma unroll
            for (int u = 0; u < SK_VEC; ++u) {
                const uint32_t i = b + (uint32_t)u * SK_THREADS + tid;
                if (i >= m) continue;
                const float a = __fmaf_rn(lr, g[u], r[u]);
                __stcs(rp + i, a);
                K.acc[i] = a;
            }
        }
    }
    if (tid == 0) {
        K.seq = seq;
        K.tag = sk_mix(p.call_tag ^ seq);
        uint32_t T0 = NO_KEY, sh = SK_RSH_MAX;
        if (p.hint_tag != 0 && htag == p.hint_tag) {
            T0 = hT0;
            sh = min(hsh, SK_RSH_MAX);
        }
        if (p.force_t0) {
            T0 = 0;
            sh = SK_RSH_ALL;
        }
        K.T0 = T0;
        K.sh = sh;
        K.armed = armed == sk_arm(seq) ? 1u : 0u;
        K.cnt[0] = K.cnt[1] = 0;
        K.lcnt = 0;
        if (c == 0) {
            ctrl->path_small = SK_PATH_TAG;
            ctrl->sk_tag = (uint32_t)K.tag;
        }
    }
    __syncthreads();
    const uint32_t T0 = K.T0, sh = K.sh;
    const uint64_t tag = K.tag;
    const uint32_t tag32 = (uint32_t)tag;

    // ---- candidates: key >= T0, in index order, into the block's region
    uint32_t E_b = 0;
    if (T0 != NO_KEY) {
        for (int i = tid; i < 2 * SK_RBINS; i += SK_THREADS) K.hist[i] = 0;
        E_b = sk_list_ordered(
            m, K.red, [&](uint32_t i) { return key_of(K.acc[i]) >= T0; },
            [&](uint32_t i, uint32_t j) {
                p.cand_idx[e0 + j] = (uint32_t)(e0 + i);
                p.cand_val[e0 + j] = K.acc[i];
                if (j < SK_CAP1) K.own[j] = i;
            });
    }
    mark_phase(ctrl, 1);
    // ---- 2: arrival; every block waits for every block (the test hook adds
    // one past the grid, which never arrives).  A prepared workspace counts
    // arrivals in one word; otherwise thread j watches block j's word.
    {
        const uint32_t nwait = (uint32_t)G + (p.stall ? 1u : 0u);
        uint32_t* arrive = &p.sync->arrive[K.seq & 1];
        bool ok = true;
        if (tid == 0) {
            // the release orders the block's candidate writes (made before the
            // block barrier) and the count before the arrival
            p.sync->flag[c].count = E_b;
            if (K.armed)
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
            else
                st_release_u64(&p.sync->flag[c].tag, tag);
            span_last(ctrl, SPAN_GATHER_LAST);   // diagnostics: the last arrival
        }
        if (K.armed) {
            if (tid == 0) ok = sk_wait_count(arrive, nwait);
        } else if ((uint32_t)tid < nwait) {
            ok = sk_wait_tag(&p.sync->flag[tid].tag, tag);
        }
        if (__syncthreads_and(ok) == 0) {
            if (tid == 0) sk_fail(ctrl, tag32, ST_TIMEOUT);
            return;
        }
        const uint32_t cnt =
            tid < G ? *reinterpret_cast<volatile const uint32_t*>(&p.sync->flag[tid].count) : 0u;
        uint32_t Et;
        const uint32_t pre = block_excl_scan(cnt, K.red, &Et);
        if (tid < G) K.pre_blk[tid] = pre;
        if (tid == 0) {
            K.pre_blk[G] = Et;
            K.E = Et;
        }
        __syncthreads();
    }
    const uint32_t E = K.E;
    mark_phase(ctrl, 2);
    if (c == 0 && tid == 0) {
        ctrl->cand_total = E;
        ctrl->cap = SK_CAP1;
        ctrl->kernels = 1;
        ctrl->r2_path = 0;
        p.sync->seq = K.seq + 1;     // every block has read it
    }

    // ---- 3: the threshold path
    uint32_t Tk = 0, q = 0, before_gt = 0, before_eq = 0;
    bool exact = true;
    if (T0 != NO_KEY && E >= k && E <= SK_CAP1) {
        exact = !sk_threshold_select(p, K, G, per, E, T0, sh, s_out);
        if (!exact) {
            Tk = s_out[0];
            q = s_out[1];
            before_gt = s_out[2];
            before_eq = s_out[3];
        }
    }
    if (c == 0 && tid == 0) ctrl->mode = exact ? 1u : 0u;
    mark_phase(ctrl, 3);

    // ---- 4: the exact path (same decision in every block)
    if (exact) {
        if (c == 0) {
            // its counters, cleared before anyone uses them, then the release
            for (int i = tid; i < SK_BINS; i += SK_THREADS) p.hist[i] = 0;
            for (int i = tid; i < 1024; i += SK_THREADS) p.hist2[i] = 0;
            if (tid == 0) {
                *p.ent_cnt = 0;
                ctrl->bar = 0;
            }
            __syncthreads();
            if (tid == 0) st_release_u64(&p.sync->go_tag, tag);
        } else {
            if (tid == 0) K.flag = sk_wait_tag(&p.sync->go_tag, tag) ? 1 : 0;
            __syncthreads();
            if (!K.flag) {
                if (tid == 0) sk_fail(ctrl, tag32, ST_TIMEOUT);
                return;
            }
        }
        // digit 1 of every element of the slice, into the global histogram
        for (int i = tid; i < SK_BINS; i += SK_THREADS) K.hist[i] = 0;
        __syncthreads();
        for (uint32_t i = tid; i < m; i += SK_THREADS) atomicAdd(&K.hist[key_of(K.acc[i]) >> SK_LOW], 1u);
        __syncthreads();
        for (int i = tid; i < SK_BINS; i += SK_THREADS)
            if (K.hist[i]) atomicAdd(&p.hist[i], K.hist[i]);
        if (!grid_barrier(&ctrl->bar, epoch, &ctrl->status, &K.flag)) {
            if (tid == 0) sk_fail(ctrl, tag32, ST_TIMEOUT);
            return;
        }
        mark_phase(ctrl, 4);

        // the k-th key's bin; elements above it, the entry list
        {
            const uint4* h4 = reinterpret_cast<const uint4*>(p.hist);
            uint4* s4 = reinterpret_cast<uint4*>(K.hist);
            for (int i = tid; i < SK_BINS / 4; i += SK_THREADS) s4[i] = h4[i];
        }
        __syncthreads();
        block_find_bin(K.hist, SK_BINS, k, K.red, &K.fr);
        if (!K.fr.ok) {
            if (tid == 0) sk_fail(ctrl, tag32, ST_INCONSISTENT);
            return;
        }
        const uint32_t b1 = K.fr.bin;
        const uint32_t rem = k - K.fr.above;
        if (c == 0 && p.hint_tag != 0) {
            // the next call's threshold: the bin of the (3k/2)-th largest
            const uint32_t rh = (uint32_t)min((int64_t)sk_hint_rank(k), p.n);
            block_find_bin(K.hist, SK_BINS, rh, K.red, &K.fr);
            if (tid == 0 && K.fr.ok) sk_write_hint(p, K.fr.bin << SK_LOW, (b1 + 1u) << SK_LOW);
        }
        // count first, reserve the block's entries with one atomic (its
        // latency overlapping the block sum of the counts above b1), then
        // list them
        uint32_t gt_b = 0, in_t = 0;
        for (uint32_t i = tid; i < m; i += SK_THREADS) {
            const uint32_t d = key_of(K.acc[i]) >> SK_LOW;
            gt_b += d > b1;
            in_t += d == b1;
        }
        {
            uint64_t tot;
            const uint64_t ex = block_excl_scan(((uint64_t)gt_b << 32) | in_t, K.scan, &tot);
            const uint32_t in_b = (uint32_t)tot;
            if (tid == 0) {
                p.slots[c].gt_first = (uint32_t)(tot >> 32);
                K.pre = in_b ? atomicAdd(p.ent_cnt, in_b) : 0u;
            }
            __syncthreads();
            uint32_t at = (uint32_t)ex + K.pre;
            if (in_t) {
                for (uint32_t i = tid; i < m; i += SK_THREADS) {
                    const uint32_t key = key_of(K.acc[i]);
                    if ((key >> SK_LOW) == b1) {
                        if (at < ENT_PER) p.ent[at] = ((uint32_t)c << SK_LOW) | (key & ((1u << SK_LOW) - 1u));
                        ++at;
                    }
                }
            }
        }
        if (!grid_barrier(&ctrl->bar, epoch, &ctrl->status, &K.flag)) {
            if (tid == 0) sk_fail(ctrl, tag32, ST_TIMEOUT);
            return;
        }
        mark_phase(ctrl, 5);

        // T, the tie quota and this block's output offset
        constexpr int EPT = (int)ENT_PER / SK_THREADS;
        uint32_t ev[EPT];
#pragma unroll
        for (int u = 0; u < EPT; ++u) ev[u] = p.ent[tid + u * SK_THREADS];
        const uint32_t En = *reinterpret_cast<const volatile uint32_t*>(p.ent_cnt);
        if (En <= ENT_PER) {
            const uint32_t gts = sk_slots_before(p.slots, c, 2, K);
#pragma unroll
            for (int u = 0; u < EPT; ++u)
                if ((uint32_t)(tid + u * SK_THREADS) >= En) ev[u] = DEAD;
            // bits 17..9
            for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int u = 0; u < EPT; ++u)
                if (ev[u] != DEAD) atomicAdd(&K.hist[(ev[u] >> 9) & 511u], 1u);
            __syncthreads();
            block_find_bin(K.hist, 512, rem, K.red, &K.fr);
            const bool ok1 = K.fr.ok;
            const uint32_t t1 = K.fr.bin;
            const uint32_t rem2 = rem - K.fr.above;
            __syncthreads();
            // bits 8..0 inside that class
            for (int i = tid; i < 512; i += SK_THREADS) K.hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int u = 0; u < EPT; ++u)
                if (ev[u] != DEAD && ((ev[u] >> 9) & 511u) == t1) atomicAdd(&K.hist[ev[u] & 511u], 1u);
            __syncthreads();
            block_find_bin(K.hist, 512, rem2, K.red, &K.fr);
            if (!ok1 || !K.fr.ok) {
                if (tid == 0) sk_fail(ctrl, tag32, ST_INCONSISTENT);
                return;
            }
            const uint32_t low = (t1 << 9) | K.fr.bin;
            Tk = (b1 << SK_LOW) | low;
            q = rem2 - K.fr.above;
            uint32_t g = 0, e = 0;
#pragma unroll
            for (int u = 0; u < EPT; ++u) {
                if (ev[u] != DEAD && (int)(ev[u] >> SK_LOW) < c) {
                    const uint32_t v = ev[u] & ((1u << SK_LOW) - 1u);
                    g += v > low;
                    e += v == low;
                }
            }
            const uint64_t both = block_sum(((uint64_t)g << 32) | e, K.scan);
            before_gt = gts + (uint32_t)(both >> 32);
            before_eq = (uint32_t)both;
        } else {
            const uint32_t err = sk_crowded(p, K, epoch, m, b1, rem, s_out);
            if (err) {
                if (tid == 0) sk_fail(ctrl, tag32, err);
                return;
            }
            Tk = s_out[0];
            q = s_out[1];
            before_gt = s_out[2];
            before_eq = s_out[3];
        }
    }

    // ---- 5: emission in index order from shared memory: the threshold path
    // only looks at the block's own candidates (one warp), the exact path at
    // the whole slice
    if (!exact) {
        if (tid < 32) {
            const uint32_t below = (1u << tid) - 1u;
            uint32_t rg = before_gt, re = before_eq;
            for (uint32_t b = 0; b < E_b; b += 32) {
                const uint32_t j = b + (uint32_t)tid;
                const uint32_t i = j < E_b ? K.own[j] : 0u;
                const uint32_t key = j < E_b ? key_of(K.acc[i]) : 0u;
                const uint32_t cl = j < E_b ? (key > Tk ? 2u : (key == Tk ? 1u : 0u)) : 0u;
                const uint32_t bg = __ballot_sync(~0u, cl == 2u), be = __ballot_sync(~0u, cl == 1u);
                const uint32_t mg = rg + __popc(bg & below), me = re + __popc(be & below);
                uint32_t rank = 0xFFFFFFFFu;
                if (cl == 2u) rank = mg + min(me, q);
                else if (cl == 1u && me < q) rank = mg + me;
                if (rank < k) {
                    p.out_idx[rank] = (int32_t)(e0 + i);
                    p.out_val[rank] = K.acc[i];
                    p.resid[e0 + i] = 0.0f;
                }
                rg += __popc(bg);
                re += __popc(be);
            }
        }
    } else {
        sk_emit_ordered(
            m, before_gt, before_eq, q, k, K.scan,
            [&](uint32_t i) {
                const uint32_t key = key_of(K.acc[i]);
                return key > Tk ? 2u : (key == Tk ? 1u : 0u);
            },
            [&](uint32_t i, uint32_t rank) {
                p.out_idx[rank] = (int32_t)(e0 + i);
                p.out_val[rank] = K.acc[i];
                p.resid[e0 + i] = 0.0f;
            });
    }
    mark_phase(ctrl, 7);
}

}  // namespace tke
