// One gTop-k round in one kernel ("A Distributed Synchronous SGD Algorithm
// with Global Top-k Sparsification for Low Bandwidth Networks", ABSTRACT and
// method section: worker i absorbs worker i + 2^r and keeps the top k of the
// union, values at a common index added once).  Each pair of the round is
// one thread-block cluster of MC_CL CTAs: CTA c of the cluster merges its
// share of the merged list (merge path) into registers, the radix digits of
// the k-th key are summed over the cluster through distributed shared memory
// (cluster barriers, no grid barrier), and every CTA writes its share of the
// top k in index order.  Used when a round's merged lists fit
// (MC_CL * MC_Q positions per pair); larger rounds take the merge + select
// kernels.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels_merge.cuh"

namespace tke {

namespace cg = cooperative_groups;

constexpr int MC_CL = 8;                        // CTAs per pair
constexpr int MC_THREADS = 512;
constexpr int MC_PT = 16;                       // merged positions per thread at most
constexpr int MC_Q = MC_THREADS * MC_PT;        // merged positions per CTA at most

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
    int32_t final_out;           // last round: the caller's arrays
    int32_t* out_idx;
    float* out_val;
    int32_t* out_count;
    int64_t out_k;
    const uint32_t* bad_words;   // first round: input verdicts to fold
    int32_t n_bad;
    Ctrl* ctrl;
};

// Shared memory of one CTA.
struct McShared {
    uint32_t h1[D1_BINS], h2[D2_BINS], h3[D3_BINS];   // this CTA's digit histograms
    uint32_t tot[D1_BINS];                            // cluster sums
    uint64_t scan[33];
    uint32_t red[33];
    int64_t part[2];
    uint32_t live, gt, eq;
    FindResult fr;
    uint32_t sAi[MC_Q + 1], sBi[MC_Q + 1];
    float sAv[MC_Q + 1], sBv[MC_Q + 1];
};

// Sum of histogram `h` (nb bins) over the cluster into S.tot, then the bin of
// the rem-th largest; every CTA computes the same.
__device__ __forceinline__ void cluster_find(cg::cluster_group& cl, McShared& S, uint32_t* h,
                                             int nb, uint32_t rem) {
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        uint32_t s = 0;
#pragma unroll
        for (int r = 0; r < MC_CL; ++r) s += *cl.map_shared_rank(h + i, r);
        S.tot[i] = s;
    }
    __syncthreads();
    block_find_bin(S.tot, nb, rem, S.red, &S.fr);
}

__global__ void __launch_bounds__(MC_THREADS, 1)
merge_cluster_kernel(const __grid_constant__ MergeClusterParams p) {
    extern __shared__ __align__(16) unsigned char mc_smem[];
    McShared& S = *reinterpret_cast<McShared*>(mc_smem);
    cg::cluster_group cl = cg::this_cluster();
    const int tid = threadIdx.x;
    const int cr = (int)cl.block_rank();
    const int pair = blockIdx.x / MC_CL;
    // the previous round's sets and sizes (programmatic serialisation)
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
    int64_t a = p.sizes_in ? p.sizes_in[left] : p.size_const;
    int64_t b = p.sizes_in ? p.sizes_in[right] : p.size_const;
    a = a < p.src_stride ? a : p.src_stride;
    b = b < p.src_stride ? b : p.src_stride;
    const uint32_t* Ai = p.src_idx + left * p.src_stride;
    const uint32_t* Bi = p.src_idx + right * p.src_stride;
    const float* Av = p.src_val + left * p.src_stride;
    const float* Bv = p.src_val + right * p.src_stride;
    const int64_t ab = a + b;
    const int64_t Q = (ab + MC_CL - 1) / MC_CL;          // <= MC_Q (host check)
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
    __syncthreads();
    if (stamp) p.ctrl->t_phase[1] = global_ns();
    const int64_t i0 = S.part[0], i1 = max(S.part[1], i0);
    const int64_t j0 = d0 - i0, j1 = max(d1 - S.part[1], j0);
    const int la = (int)min(i1 - i0, (int64_t)MC_Q);
    const int lb = (int)min(j1 - j0, (int64_t)MC_Q);
    // sA[x] = A[i0 - 1 + x] for x in [0, la]; sB[y] = B[j0 + y] for y in [0, lb]
    for (int x = tid; x <= la; x += blockDim.x) {
        const int64_t gi = i0 - 1 + x;
        const bool in = gi >= 0 && gi < a;
        S.sAi[x] = in ? Ai[gi] : DEAD;
        S.sAv[x] = in ? Av[gi] : 0.f;
    }
    for (int y = tid; y <= lb; y += blockDim.x) {
        const int64_t gj = j0 + y;
        const bool in = gj < b;
        S.sBi[y] = in ? Bi[gj] : DEAD;
        S.sBv[y] = in ? Bv[gj] : 0.f;
    }
    __syncthreads();
    if (stamp) p.ctrl->t_phase[2] = global_ns();

    // merge this thread's positions [dl, dl + MC_PT) of the CTA's span
    const int span = (int)(d1 - d0);
    const int pt = (span + MC_THREADS - 1) / MC_THREADS;  // positions per thread
    const int dl = tid * pt;
    uint32_t mi[MC_PT];
    float mv[MC_PT];
    uint32_t live = 0;
    {
        int ia = 0, ib = 0;
        if (dl < span) {
            ia = local_merge_path(S.sAi + 1, la, S.sBi, lb, dl);
            ib = dl - ia;
        }
#pragma unroll
        for (int u = 0; u < MC_PT; ++u) {
            uint32_t oi = DEAD;
            float ov = 0.f;
            const int pos = dl + u;
            if (u < pt && pos < span) {
                const int64_t d = d0 + pos;
                const bool takeA = ia < la && (ib >= lb || S.sAi[1 + ia] <= S.sBi[ib]);
                if (takeA) {
                    oi = S.sAi[1 + ia];
                    ov = S.sAv[1 + ia];
                    // partner: the next B element, B[d - i] with i = i0 + ia
                    const int64_t jB = d - (i0 + ia);
                    if (jB < b) {
                        const int64_t y = jB - j0;
                        if (y >= 0 && y <= lb && S.sBi[y] == oi) ov = __fadd_rn(ov, S.sBv[y]);
                    }
                    ++ia;
                } else {
                    oi = ib < lb ? S.sBi[ib] : DEAD;
                    ov = ib < lb ? S.sBv[ib] : 0.f;
                    // the previous A element, A[iA - 1] with iA = d - j
                    const int64_t iA = d - (j0 + ib);
                    if (iA > 0) {
                        const int64_t x = iA - i0;       // sA[x] = A[iA - 1]
                        if (x >= 0 && x <= la && S.sAi[x] == oi) oi = DEAD;
                    }
                    ++ib;
                }
            }
            mi[u] = oi;
            mv[u] = oi == DEAD ? 0.f : ov;
            if (oi != DEAD) {
                ++live;
                atomicAdd(&S.h1[key_of(mv[u]) >> 20], 1u);
            }
        }
    }
    live = block_sum(live, S.red);
    if (tid == 0) S.live = live;
    if (stamp) p.ctrl->t_phase[3] = global_ns();
    cl.sync();                                           // h1 and live of every CTA
    if (stamp) p.ctrl->t_phase[4] = global_ns();

    uint32_t live_tot = 0;
#pragma unroll
    for (int r = 0; r < MC_CL; ++r) live_tot += *cl.map_shared_rank(&S.live, r);
    const uint32_t kp = live_tot < p.kmax ? live_tot : p.kmax;
    uint32_t T = NO_KEY, q = 0;
    uint32_t rem = kp, b1 = 0, b2 = 0;
    bool ok = kp > 0;
    if (ok) {
        cluster_find(cl, S, S.h1, D1_BINS, rem);
        ok = S.fr.ok;
        b1 = S.fr.bin;
        rem -= S.fr.above;
#pragma unroll
        for (int u = 0; u < MC_PT; ++u)
            if (mi[u] != DEAD && (key_of(mv[u]) >> 20) == b1)
                atomicAdd(&S.h2[(key_of(mv[u]) >> 10) & (D2_BINS - 1)], 1u);
    }
    cl.sync();                                           // h2
    if (kp > 0) {
        cluster_find(cl, S, S.h2, D2_BINS, rem);
        ok = ok && S.fr.ok;
        b2 = S.fr.bin;
        rem -= S.fr.above;
        const uint32_t pre = (b1 << D2_BITS) | b2;
#pragma unroll
        for (int u = 0; u < MC_PT; ++u)
            if (mi[u] != DEAD && (key_of(mv[u]) >> 10) == pre)
                atomicAdd(&S.h3[key_of(mv[u]) & (D3_BINS - 1)], 1u);
    }
    cl.sync();                                           // h3
    if (kp > 0) {
        cluster_find(cl, S, S.h3, D3_BINS, rem);
        ok = ok && S.fr.ok;
        T = (b1 << 20) | (b2 << 10) | S.fr.bin;
        q = rem - S.fr.above;
        if (!ok) {
            if (tid == 0) atomicOr(&p.ctrl->status, ST_INCONSISTENT);
            T = NO_KEY;
            q = 0;
        }
    }
    if (stamp) p.ctrl->t_phase[5] = global_ns();
    // this thread's (key > T, key == T) counts, then the CTA's
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int u = 0; u < MC_PT; ++u) {
        if (mi[u] == DEAD || T == NO_KEY) continue;
        const uint32_t key = key_of(mv[u]);
        g += key > T;
        e += key == T;
    }
    uint64_t tot_ge;
    const uint64_t ex = block_excl_scan(((uint64_t)g << 32) | e, S.scan, &tot_ge);
    if (tid == 0) {
        S.gt = (uint32_t)(tot_ge >> 32);
        S.eq = (uint32_t)(tot_ge & 0xFFFFFFFFu);
    }
    cl.sync();                                           // every CTA's counts
    if (stamp) p.ctrl->t_phase[6] = global_ns();
    uint32_t pg = 0, pe = 0;
    for (int r = 0; r < cr; ++r) {
        pg += *cl.map_shared_rank(&S.gt, r);
        pe += *cl.map_shared_rank(&S.eq, r);
    }
    // emission in index order: rank = #gt + min(#eq, q) before the entry
    if (T != NO_KEY) {
        uint32_t rg = pg + (uint32_t)(ex >> 32), re = pe + (uint32_t)(ex & 0xFFFFFFFFu);
        uint32_t* di = p.dst_idx + left * p.dst_stride;
        float* dv = p.dst_val + left * p.dst_stride;
#pragma unroll
        for (int u = 0; u < MC_PT; ++u) {
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
             i += (int64_t)MC_CL * blockDim.x) {
            p.out_idx[i] = -1;
            p.out_val[i] = 0.0f;
        }
    } else if (cr == 0 && tid == 0) {
        p.sizes_out[left] = kp;
    }
    if (stamp) p.ctrl->t_phase[7] = global_ns();
    // this CTA's shared memory stays valid until every CTA has read it
    cl.sync();
}

}  // namespace tke
