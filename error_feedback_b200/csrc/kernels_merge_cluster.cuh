// One gTop-k round in one kernel ("A Distributed Synchronous SGD Algorithm
// with Global Top-k Sparsification for Low Bandwidth Networks", ABSTRACT and
// method section: worker i absorbs worker i + 2^r and keeps the top k of the
// union, values at a common index added once).  Each pair of the round is
// one thread-block cluster of CL CTAs:
//   1. CTA c merges its share of the pair's merged list (merge path) into
//      registers and builds the histogram of the first radix digit (key
//      bits 30..20 in the first round; after it, bins of 2^13 keys above the
//      lower of the two sets' lowest keys);
//   2. the digit histograms are summed over the cluster through distributed
//      shared memory (each CTA sums a slice, then reads every slice), which
//      gives the bin b1 of the k-th key;
//   3. every CTA lists its entries in bin b1 (with its rank in the cluster)
//      and counts those above it; every CTA then gathers all the lists and
//      finds, locally, the k-th key T, the tie quota q and its own output
//      offset (the counts above b1 of the CTAs before it plus their listed
//      entries above / equal to T);
//   4. every CTA writes its share of the top k in index order.
// Four cluster barriers (the last keeps each CTA's shared memory alive for
// the others' reads), no grid barrier.  A bin b1 with more entries than
// the gather space resolves the remaining digits by two more summed
// histogram passes and exchanges exact counts instead.  Used when a round's
// merged lists fit (CL * QMAX positions per pair); larger rounds take the
// merge + select kernels.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels_merge.cuh"

namespace tke {

namespace cg = cooperative_groups;

constexpr int MC_THREADS = 512;
constexpr int64_t MC_PAIR_MAX = 65536;          // merged positions per pair

template <int CL>
struct McCfg {
    static constexpr int PT = (int)(MC_PAIR_MAX / CL / MC_THREADS);   // positions per thread
    static constexpr int QMAX = PT * MC_THREADS;                      // positions per CTA
    static constexpr int STAGE = 4 * (QMAX + 1);                      // staging words
    static constexpr int GCAP = STAGE - QMAX - 4;                     // gathered list capacity
    // digit-1 bins whose cluster sum one CTA owns (a multiple of 4; the last
    // CTA's slice ends at D1_BINS)
    static constexpr int SB = ((D1_BINS + CL - 1) / CL + 3) / 4 * 4;
    // first step of a binary search over the cluster ranks 0 .. CL - 1
    static constexpr int ST0 = CL > 8 ? 8 : CL > 4 ? 4 : CL > 2 ? 2 : 1;
};

// Merged positions of a pair that a cluster of CL CTAs holds.
template <int CL>
constexpr int64_t mc_pair_cap() {
    return (int64_t)CL * McCfg<CL>::QMAX;
}

// Relative digit 1 (rounds after the first): bin 0 holds the keys below the
// pair's floor L (sums at common indices can fall there), bins 1 .. 2046 the
// keys in [L + (b - 1) 2^13, L + b 2^13) (two octaves above L), bin 2047 the
// rest; the k-th key in bin 0 or 2047, or a bin too crowded to gather,
// repeats the digit with key >> 20.
constexpr int MC_RSH = 13;

__device__ __forceinline__ uint32_t mc_bin(uint32_t key, bool rel, uint32_t L) {
    if (!rel) return key >> 20;
    if (key < L) return 0u;
    return min(((key - L) >> MC_RSH) + 1u, (uint32_t)(D1_BINS - 1));
}
__device__ __forceinline__ uint32_t mc_low(uint32_t key, bool rel, uint32_t L) {
    return rel ? ((key - L) & ((1u << MC_RSH) - 1u)) : (key & 0xFFFFFu);
}

struct MergeClusterParams {
    const uint32_t* src_idx;     // sets of this round, row stride src_stride
    const float* src_val;
    int64_t src_stride;
    const uint32_t* sizes_in;    // null: every set has size_const entries
    uint32_t size_const;
    int32_t step;                // 2^r
    uint32_t kmax;
    uint32_t* dst_idx;           // sets buffer, row stride dst_stride
    float* dst_val;
    int64_t dst_stride;
    uint32_t* sizes_out;
    const uint32_t* floor_in;    // null (first round): digit 1 is key >> 20; else each set's
                                 // lowest key, and digit 1 is relative to the pair's lower one
    uint32_t* floor_out;         // the merged set's lowest key (its k-th)
    int32_t final_out;           // last round: the caller's arrays
    int32_t* out_idx;
    float* out_val;
    int32_t* out_count;
    int64_t out_k;
    const uint32_t* bad_words;   // first round: input verdicts to fold
    int32_t n_bad;
    Ctrl* ctrl;
};

// Fixed part of a CTA's shared memory; the staging words follow it.
struct McFixed {
    uint32_t h1[D1_BINS], h2[D2_BINS], h3[D3_BINS];   // this CTA's digit histograms
    uint32_t tot[D1_BINS];                            // cluster sums / local histograms
    uint64_t scan[33];
    uint32_t red[33];
    int64_t part[2];
    uint32_t live, above, nlist, gt, eq, pg, pe;
    uint32_t loff[17];                                // list offsets by cluster rank
    uint32_t lcnt[16];                                // list lengths by cluster rank
    __align__(16) uint32_t hslice[D1_BINS / 8];       // this CTA's slice of the summed h1
                                                      // (McCfg<CL>::SB <= D1_BINS / 8 bins)
    uint32_t live_tot;
    uint32_t E, pre_above;
    FindResult fr;
    uint32_t sel[8];                                  // the gathered select's results (local)
};

template <int CL>
constexpr size_t mc_smem_bytes() {
    return (sizeof(McFixed) + 15) / 16 * 16 + (size_t)McCfg<CL>::STAGE * 4;
}

// Sum of histogram `h` (nb bins) over the cluster into S.tot, then the bin of
// the rem-th largest; every CTA computes the same.
// All remote loads of a thread are issued before the first is summed (NB is
// a multiple of MC_THREADS).
template <int CL, int NB>
__device__ __forceinline__ void cluster_find(cg::cluster_group& cl, McFixed& S, uint32_t* h,
                                             uint32_t rem) {
    constexpr int PER = NB / MC_THREADS;
    uint32_t v[PER][CL];
#pragma unroll
    for (int j = 0; j < PER; ++j)
#pragma unroll
        for (int r = 0; r < CL; ++r) v[j][r] = *cl.map_shared_rank(h + threadIdx.x + j * MC_THREADS, r);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        uint32_t s = 0;
#pragma unroll
        for (int r = 0; r < CL; ++r) s += v[j][r];
        S.tot[threadIdx.x + j * MC_THREADS] = s;
    }
    __syncthreads();
    block_find_bin(S.tot, NB, rem, S.red, &S.fr);
}

template <int CL>
__global__ void __launch_bounds__(MC_THREADS, (CL >= 12 ? 2 : 1))
merge_cluster_kernel(const __grid_constant__ MergeClusterParams p) {
    using C = McCfg<CL>;
    static_assert(CL >= 8 && CL <= 16, "clusters of 8 to 16 CTAs");
    static_assert(C::SB * CL >= D1_BINS && C::SB <= D1_BINS / 8, "digit-1 slices");
    constexpr int PT = C::PT;
    constexpr int QMAX = C::QMAX;
    extern __shared__ __align__(16) unsigned char mc_smem[];
    McFixed& S = *reinterpret_cast<McFixed*>(mc_smem);
    uint32_t* stage = reinterpret_cast<uint32_t*>(mc_smem + (sizeof(McFixed) + 15) / 16 * 16);
    uint32_t* sAi = stage;
    uint32_t* sBi = stage + (QMAX + 1);
    float* sAv = reinterpret_cast<float*>(stage + 2 * (QMAX + 1));
    float* sBv = reinterpret_cast<float*>(stage + 3 * (QMAX + 1));
    cg::cluster_group cl = cg::this_cluster();
    const int tid = threadIdx.x;
    const int cr = (int)cl.block_rank();
    const int pair = blockIdx.x / CL;
    // the next round may be scheduled now; this one waits for the previous
    // round's sets and sizes (programmatic serialisation)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const bool stamp = blockIdx.x == 0 && tid == 0;     // diagnostics: CTA 0's phases
    if (stamp) p.ctrl->t_phase[0] = global_ns();
    if (p.bad_words && blockIdx.x == 0 && tid == 0) {
        uint32_t any = 0;
        for (int i = 0; i < p.n_bad; ++i) any |= p.bad_words[i];
        if (any) atomicOr(&p.ctrl->status, ST_BAD_INPUT);
    }
    const int64_t left = (int64_t)pair * 2 * p.step;
    const int64_t right = left + p.step;
    // digit 1 relative to the pair's lower floor when both are known
    uint32_t Lf = 0;
    bool rel = false;
    if (p.floor_in) {
        Lf = min(p.floor_in[left], p.floor_in[right]);
        rel = Lf != 0;
    }
    int64_t a = p.sizes_in ? p.sizes_in[left] : p.size_const;
    int64_t b = p.sizes_in ? p.sizes_in[right] : p.size_const;
    a = a < p.src_stride ? a : p.src_stride;
    b = b < p.src_stride ? b : p.src_stride;
    const uint32_t* Ai = p.src_idx + left * p.src_stride;
    const uint32_t* Bi = p.src_idx + right * p.src_stride;
    const float* Av = p.src_val + left * p.src_stride;
    const float* Bv = p.src_val + right * p.src_stride;
    const int64_t ab = a + b;
    const int64_t Q = (ab + CL - 1) / CL;                // <= QMAX (host check)
    const int64_t d0 = min((int64_t)cr * Q, ab);
    const int64_t d1 = min(d0 + Q, ab);
    if (tid < 64) {
        const int64_t dd = tid < 32 ? d0 : d1;
        const int64_t i = warp_merge_path(Ai, a, Bi, b, dd);
        if ((tid & 31) == 0) S.part[tid >> 5] = i;
    }
    for (int i = tid; i < D1_BINS; i += blockDim.x) S.h1[i] = 0;
    for (int i = tid; i < D2_BINS; i += blockDim.x) S.h2[i] = 0;
    for (int i = tid; i < D3_BINS; i += blockDim.x) S.h3[i] = 0;
    for (int i = tid; i < C::SB; i += blockDim.x) S.hslice[i] = 0;
    __syncthreads();
    if (stamp) p.ctrl->t_phase[1] = global_ns();
    const int64_t i0 = S.part[0], i1 = max(S.part[1], i0);
    const int64_t j0 = d0 - i0, j1 = max(d1 - S.part[1], j0);
    const int la = (int)min(i1 - i0, (int64_t)QMAX);
    const int lb = (int)min(j1 - j0, (int64_t)QMAX);
    // sA[x] = A[i0 - 1 + x] for x in [0, la]; sB[y] = B[j0 + y] for y in [0, lb];
    // all loads of a thread are issued before its stores
    {
        uint32_t ri[PT + 1];
        float rv[PT + 1];
#pragma unroll
        for (int u = 0; u <= PT; ++u) {
            const int x = tid + u * MC_THREADS;
            const int64_t gi = i0 - 1 + x;
            const bool in = x <= la && gi >= 0 && gi < a;
            ri[u] = in ? Ai[gi] : DEAD;
            rv[u] = in ? Av[gi] : 0.f;
        }
#pragma unroll
        for (int u = 0; u <= PT; ++u) {
            const int x = tid + u * MC_THREADS;
            if (x <= la) {
                sAi[x] = ri[u];
                sAv[x] = rv[u];
            }
        }
#pragma unroll
        for (int u = 0; u <= PT; ++u) {
            const int y = tid + u * MC_THREADS;
            const int64_t gj = j0 + y;
            const bool in = y <= lb && gj < b;
            ri[u] = in ? Bi[gj] : DEAD;
            rv[u] = in ? Bv[gj] : 0.f;
        }
#pragma unroll
        for (int u = 0; u <= PT; ++u) {
            const int y = tid + u * MC_THREADS;
            if (y <= lb) {
                sBi[y] = ri[u];
                sBv[y] = rv[u];
            }
        }
    }
    __syncthreads();
    if (stamp) p.ctrl->t_phase[2] = global_ns();

    // merge this thread's positions [dl, dl + pt) of the CTA's span
    const int span = (int)(d1 - d0);
    const int pt = (span + MC_THREADS - 1) / MC_THREADS;
    const int dl = tid * pt;
    uint32_t mi[PT];
    float mv[PT];
    uint32_t live = 0;
    {
        int ia = 0, ib = 0;
        if (dl < span) {
            ia = local_merge_path(sAi + 1, la, sBi, lb, dl);
            ib = dl - ia;
        }
#pragma unroll
        for (int u = 0; u < PT; ++u) {
            uint32_t oi = DEAD;
            float ov = 0.f;
            const int pos = dl + u;
            if (u < pt && pos < span) {
                const int64_t d = d0 + pos;
                const bool takeA = ia < la && (ib >= lb || sAi[1 + ia] <= sBi[ib]);
                if (takeA) {
                    oi = sAi[1 + ia];
                    ov = sAv[1 + ia];
                    // partner: the next B element, B[d - i] with i = i0 + ia
                    const int64_t y = d - (i0 + ia) - j0;
                    if (d - (i0 + ia) < b && y >= 0 && y <= lb && sBi[y] == oi)
                        ov = __fadd_rn(ov, sBv[y]);
                    ++ia;
                } else {
                    oi = ib < lb ? sBi[ib] : DEAD;
                    ov = ib < lb ? sBv[ib] : 0.f;
                    // the previous A element, A[iA - 1] with iA = d - j
                    const int64_t iA = d - (j0 + ib);
                    const int64_t x = iA - i0;           // sA[x] = A[iA - 1]
                    if (iA > 0 && x >= 0 && x <= la && sAi[x] == oi) oi = DEAD;
                    ++ib;
                }
            }
            mi[u] = oi;
            mv[u] = oi == DEAD ? 0.f : ov;
            if (oi != DEAD) {
                ++live;
                atomicAdd(&S.h1[mc_bin(key_of(mv[u]), rel, Lf)], 1u);
            }
        }
    }
    live = block_sum(live, S.red);
    if (tid == 0) S.live = live;
    if (stamp) p.ctrl->t_phase[3] = global_ns();
    uint32_t kp = 0, b1 = 0, rem = 0;
    bool ok = false;
    uint32_t* mylist = stage;                           // [QMAX]
    uint32_t* glist = stage + QMAX + 4;                 // [GCAP]
    constexpr uint32_t SENT = 0xFFFFFFFFu;              // padding entry of the lists
    for (int attempt = 0;; ++attempt) {
    if (attempt > 0) {
        // the relative digit did not decide: every CTA is past its reads of
        // the others' slices and lists; digit 1 again with key >> 20
        rel = false;
        cl.sync();
        for (int i = tid; i < D1_BINS; i += blockDim.x) S.h1[i] = 0;
        for (int i = tid; i < C::SB; i += blockDim.x) S.hslice[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < PT; ++u)
            if (mi[u] != DEAD) atomicAdd(&S.h1[key_of(mv[u]) >> 20], 1u);
    }
    cl.sync();                                           // [1] h1 and live of every CTA
    if (stamp) p.ctrl->t_phase[4] = global_ns();

    // live entries of the pair (warp 0, lane r reads rank r), and this CTA's
    // slice of the summed digit-1 histogram: bins [cr*SB, cr*SB + SB) (up to
    // D1_BINS) over all CTAs, one 16-byte remote load per thread
    constexpr int SB = C::SB;
    if (tid < 32) {
        const uint32_t lv = tid < CL ? *cl.map_shared_rank(&S.live, tid) : 0u;
        const uint32_t lt = warp_sum(lv);
        if (tid == 0) S.live_tot = lt;
    }
    for (int t = tid; t < (SB / 4) * CL; t += blockDim.x) {
        const int r = t / (SB / 4), j = t - r * (SB / 4);
        if (cr * SB + 4 * j >= D1_BINS) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(cl.map_shared_rank(S.h1 + cr * SB + 4 * j, r));
        atomicAdd(&S.hslice[4 * j + 0], v.x);
        atomicAdd(&S.hslice[4 * j + 1], v.y);
        atomicAdd(&S.hslice[4 * j + 2], v.z);
        atomicAdd(&S.hslice[4 * j + 3], v.w);
    }
    cl.sync();                                           // [1b] every slice summed
    const uint32_t live_tot = S.live_tot;
    kp = live_tot < p.kmax ? live_tot : p.kmax;
    b1 = 0;
    rem = kp;
    ok = kp > 0;
    if (kp > 0) {
        // the summed histogram from its CL owners, 16 bytes per thread
        for (int t = tid; t < D1_BINS / 4; t += blockDim.x) {
            const int r = (4 * t) / SB;
            const uint4 v = *reinterpret_cast<const uint4*>(
                cl.map_shared_rank(S.hslice + (4 * t - r * SB), r));
            reinterpret_cast<uint4*>(S.tot)[t] = v;
        }
        __syncthreads();
        if (tid < 32) {
            uint32_t bb = 0, ab = 0;
            const bool f = warp_find<D1_BINS>(S.tot, rem, bb, ab);
            if (tid == 0) {
                S.fr.ok = f ? 1u : 0u;
                S.fr.bin = bb;
                S.fr.above = ab;
            }
        }
        __syncthreads();
        ok = S.fr.ok;
        b1 = S.fr.bin;
        rem -= S.fr.above;
    }
    // this CTA's entries in bin b1 (low 20 key bits, in the staging space,
    // which the merge no longer needs) and its count above b1
    {
        uint32_t nin = 0, nab = 0;
#pragma unroll
        for (int u = 0; u < PT; ++u) {
            if (mi[u] == DEAD || kp == 0) continue;
            const uint32_t d = mc_bin(key_of(mv[u]), rel, Lf);
            nin += d == b1;
            nab += d > b1;
        }
        __syncthreads();                                 // staging reads are done
        uint32_t tin;
        uint32_t at = block_excl_scan(nin, S.red, &tin);
#pragma unroll
        for (int u = 0; u < PT; ++u) {
            if (mi[u] == DEAD || kp == 0) continue;
            const uint32_t key = key_of(mv[u]);
            if (mc_bin(key, rel, Lf) == b1) mylist[at++] = ((uint32_t)cr << 20) | mc_low(key, rel, Lf);
        }
        nab = block_sum(nab, S.red);
        if (tid == 0) {
            S.nlist = tin;
            S.above = nab;
        }
    }
    cl.sync();                                           // [2] every CTA's list and count
    if (stamp) p.ctrl->t_phase[5] = global_ns();

    // list lengths and counts above b1 of all CTAs (lane r reads rank r);
    // in the gathered list each CTA's entries start at a multiple of 4
    if (tid < 32) {
        const uint32_t lane = lane_id();
        uint32_t nr = 0, ar = 0;
        if (lane < (uint32_t)CL) {
            nr = *cl.map_shared_rank(&S.nlist, (int)lane);
            ar = *cl.map_shared_rank(&S.above, (int)lane);
        }
        const uint32_t np4 = (nr + 3u) & ~3u;
        const uint32_t incl = warp_incl_scan(np4);
        if (lane < (uint32_t)CL) {
            S.loff[lane] = incl - np4;
            S.lcnt[lane] = nr;
        }
        if (lane == (uint32_t)CL - 1) S.loff[CL] = incl;
        const uint32_t pa = warp_sum((int)lane < cr ? ar : 0u);
        const uint32_t all = __shfl_sync(0xFFFFFFFFu, incl, 31);
        if (lane == 0) {
            S.E = all;
            S.pre_above = pa;
        }
    }
    __syncthreads();
    // the relative digit decides unless the k-th key is in an open bin or
    // its bin is too crowded to gather (the same in every CTA)
    if (!rel || kp == 0 || (ok && b1 != 0 && b1 != (uint32_t)(D1_BINS - 1) &&
                            S.E <= (uint32_t)C::GCAP))
        break;
    }
    const uint32_t E = S.E, pre_above = S.pre_above;
    uint32_t T = NO_KEY, q = 0, pg = 0, pe = 0;
    const bool gathered = E <= (uint32_t)C::GCAP;       // the same in every CTA
    if (gathered) {
        // all lists, in cluster rank order, 16 bytes per remote load
        uint4* g4 = reinterpret_cast<uint4*>(glist);
        for (uint32_t u = tid; u < E / 4; u += blockDim.x) {
            int r = 0;
#pragma unroll
            for (int st = C::ST0; st >= 1; st >>= 1)
                if (r + st < CL && S.loff[r + st] <= 4 * u) r += st;
            const uint32_t i = 4 * u - S.loff[r];          // first entry of the load
            uint4 v = *reinterpret_cast<const uint4*>(cl.map_shared_rank(mylist + i, r));
            const uint32_t nr = S.lcnt[r];
            if (i + 0 >= nr) v.x = SENT;
            if (i + 1 >= nr) v.y = SENT;
            if (i + 2 >= nr) v.z = SENT;
            if (i + 3 >= nr) v.w = SENT;
            g4[u] = v;
        }
        __syncthreads();
        if (kp > 0 && ok) {
            // bits 19..10, then 9..0 of the k-th key inside bin b1: every
            // thread counts its share of the list into the (zeroed, here
            // unused) digit-2 and -3 histograms, warp 0 alone finds the bins
            // (a block-wide find costs four barriers, the warp's none)
            constexpr uint32_t SENT_ = 0xFFFFFFFFu;
            const uint32_t lsh = rel ? (uint32_t)MC_RSH - 10u : 10u;   // bits below pass A
            for (uint32_t i = tid; i < E; i += blockDim.x) {
                const uint32_t v = glist[i];
                if (v != SENT_) atomicAdd(&S.h2[((v & 0xFFFFFu) >> lsh) & 1023u], 1u);
            }
            if (tid == 0) S.sel[6] = S.sel[7] = 0;
            __syncthreads();
            if (tid < 32) {
                uint32_t bA = 0, aA = 0;
                const bool f = warp_find<D2_BINS>(S.h2, rem, bA, aA);
                if (tid == 0) {
                    S.sel[0] = f ? 1u : 0u;
                    S.sel[1] = bA;
                    S.sel[2] = aA;
                }
            }
            __syncthreads();
            const uint32_t bA = S.sel[1];
            const uint32_t remA = rem - S.sel[2];
            ok = S.sel[0] != 0;
            if (ok) {
                for (uint32_t i = tid; i < E; i += blockDim.x) {
                    const uint32_t v = glist[i];
                    if (v != SENT_ && (((v & 0xFFFFFu) >> lsh) & 1023u) == bA)
                        atomicAdd(&S.h3[v & ((1u << lsh) - 1u)], 1u);
                }
                __syncthreads();
                if (tid < 32) {
                    uint32_t bB = 0, aB = 0;
                    const bool f = warp_find<D3_BINS>(S.h3, remA, bB, aB);
                    if (tid == 0) {
                        S.sel[3] = f ? 1u : 0u;
                        S.sel[4] = bB;
                        S.sel[5] = aB;
                    }
                }
                __syncthreads();
                ok = S.sel[3] != 0;
                const uint32_t t = (bA << lsh) | S.sel[4];
                q = remA - S.sel[5];
                T = !ok ? NO_KEY : rel ? Lf + ((b1 - 1u) << MC_RSH) + t : (b1 << 20) | t;
                // entries of earlier CTAs in bin b1: above T, equal to T
                uint32_t g = 0, e = 0;
                for (uint32_t i = tid; i < E; i += blockDim.x) {
                    const uint32_t v = glist[i];
                    if (v != SENT_ && (int)(v >> 20) < cr) {
                        g += (v & 0xFFFFFu) > t;
                        e += (v & 0xFFFFFu) == t;
                    }
                }
                g = __reduce_add_sync(0xFFFFFFFFu, g);
                e = __reduce_add_sync(0xFFFFFFFFu, e);
                if (lane_id() == 0 && (g | e)) {
                    atomicAdd(&S.sel[6], g);
                    atomicAdd(&S.sel[7], e);
                }
                __syncthreads();
                pg = pre_above + S.sel[6];
                pe = S.sel[7];
            }
        }
    } else {
        // crowded bin: two more summed digit passes, then exact counts
        if (kp > 0) {
#pragma unroll
            for (int u = 0; u < PT; ++u)
                if (mi[u] != DEAD && (key_of(mv[u]) >> 20) == b1)
                    atomicAdd(&S.h2[(key_of(mv[u]) >> 10) & (D2_BINS - 1)], 1u);
        }
        cl.sync();
        uint32_t b2 = 0;
        if (kp > 0) {
            cluster_find<CL, D2_BINS>(cl, S, S.h2, rem);
            ok = ok && S.fr.ok;
            b2 = S.fr.bin;
            rem -= S.fr.above;
            const uint32_t pre = (b1 << D2_BITS) | b2;
#pragma unroll
            for (int u = 0; u < PT; ++u)
                if (mi[u] != DEAD && (key_of(mv[u]) >> 10) == pre)
                    atomicAdd(&S.h3[key_of(mv[u]) & (D3_BINS - 1)], 1u);
        }
        cl.sync();
        if (kp > 0) {
            cluster_find<CL, D3_BINS>(cl, S, S.h3, rem);
            ok = ok && S.fr.ok;
            q = rem - S.fr.above;
            T = ok ? (b1 << 20) | (b2 << 10) | S.fr.bin : NO_KEY;
        }
        uint32_t g = 0, e = 0;
#pragma unroll
        for (int u = 0; u < PT; ++u) {
            if (mi[u] == DEAD || T == NO_KEY) continue;
            const uint32_t key = key_of(mv[u]);
            g += key > T;
            e += key == T;
        }
        g = block_sum(g, S.red);
        e = block_sum(e, S.red);
        if (tid == 0) {
            S.gt = g;
            S.eq = e;
        }
        cl.sync();
        for (int r = 0; r < cr; ++r) {
            pg += *cl.map_shared_rank(&S.gt, r);
            pe += *cl.map_shared_rank(&S.eq, r);
        }
    }
    if (kp > 0 && T == NO_KEY && tid == 0) atomicOr(&p.ctrl->status, ST_INCONSISTENT);
    if (stamp) p.ctrl->t_phase[6] = global_ns();

    // emission in index order: rank = #gt + min(#eq, q) before the entry
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int u = 0; u < PT; ++u) {
        if (mi[u] == DEAD || T == NO_KEY) continue;
        const uint32_t key = key_of(mv[u]);
        g += key > T;
        e += key == T;
    }
    uint64_t tot_ge;
    const uint64_t ex = block_excl_scan(((uint64_t)g << 32) | e, S.scan, &tot_ge);
    if (T != NO_KEY) {
        uint32_t rg = pg + (uint32_t)(ex >> 32), re = pe + (uint32_t)(ex & 0xFFFFFFFFu);
        uint32_t* di = p.dst_idx + left * p.dst_stride;
        float* dv = p.dst_val + left * p.dst_stride;
#pragma unroll
        for (int u = 0; u < PT; ++u) {
            if (mi[u] == DEAD) continue;
            const uint32_t key = key_of(mv[u]);
            uint32_t rank = 0xFFFFFFFFu;
            if (key > T) {
                rank = rg + (re < q ? re : q);
                ++rg;
            } else if (key == T) {
                if (re < q) rank = rg + re;
                ++re;
            }
            if (rank < kp) {
                if (p.final_out) {
                    p.out_idx[rank] = (int32_t)mi[u];
                    p.out_val[rank] = mv[u];
                } else {
                    di[rank] = mi[u];
                    dv[rank] = mv[u];
                }
            }
        }
    }
    if (p.final_out) {
        // result length and the padding of the caller's arrays
        if (cr == 0 && tid == 0) *p.out_count = (int32_t)kp;
        for (int64_t i = (int64_t)kp + (int64_t)cr * blockDim.x + tid; i < p.out_k;
             i += (int64_t)CL * blockDim.x) {
            p.out_idx[i] = -1;
            p.out_val[i] = 0.0f;
        }
    } else if (cr == 0 && tid == 0) {
        p.sizes_out[left] = kp;
        if (p.floor_out) p.floor_out[left] = T == NO_KEY ? 0u : T;
    }
    if (stamp) p.ctrl->t_phase[7] = global_ns();
    // this CTA's shared memory stays valid until every CTA has read it
    cl.sync();
}

}  // namespace tke
