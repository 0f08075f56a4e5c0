// Sparse-set steps around the gTop-k merge: the residual return of the
// values that did not survive, and the AllGather-style dense sum of all
// workers' sets (the comparator the gTop-k review measures against).
#pragma once

#include "common.cuh"

namespace tke {

// ------------------------------------------------------- residual return

constexpr int RET_THREADS = 256;
constexpr int RET_SAMPLE = 4096;     // entries of the global list kept in shared memory

struct ReturnParams {
    const int32_t* sent_idx;    // [P][k_sent], rows strictly ascending
    const float* sent_val;
    int64_t k_sent;
    int64_t total;              // P * k_sent
    const int32_t* gidx;        // [k_global], strictly ascending
    int64_t kg;
    float* residual;            // [P][n]
    int64_t n;
    Ctrl* ctrl;
};

// Whether global index list g[0..kg) holds i: the sample s[j] = g[j*kg/rs]
// (rs = min(kg, RET_SAMPLE) entries, in shared memory) narrows the search
// to one stretch of g between two samples.
__device__ __forceinline__ bool in_global(const int32_t* __restrict__ g, int64_t kg,
                                          const int32_t* s, int rs, int32_t i) {
    int lo = 0, hi = rs;                           // last sample <= i
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s[mid] <= i) lo = mid; else hi = mid;
    }
    if (s[lo] > i) return false;                   // below every entry
    int64_t a = ((int64_t)lo * kg) / rs;           // g[a] == s[lo] <= i
    int64_t b = lo + 1 < rs ? ((int64_t)(lo + 1) * kg) / rs : kg;   // g[b] > i (or end)
    while (b - a > 1) {
        const int64_t mid = (a + b) >> 1;
        if (__ldg(g + mid) <= i) a = mid; else b = mid;
    }
    return __ldg(g + a) == i;
}

// Scattered residual read: ask L2 for the 64-byte minimum from DRAM (the
// neighbouring values are not needed).
__device__ __forceinline__ float ld_scattered(const float* p) {
    float v;
    asm volatile("ld.global.L2::64B.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}

// For every worker p and sent entry (i, v) whose index i is not in the
// global list: residual[p][i] += v (one fp32 add).  Malformed input (an
// index outside [0, n), rows or global list not strictly ascending) sets
// ST_BAD_INPUT; an out-of-range index is never written.
__global__ void __launch_bounds__(RET_THREADS)
return_kernel(const __grid_constant__ ReturnParams p) {
    __shared__ int32_t s[RET_SAMPLE];
    const int rs = (int)(p.kg < RET_SAMPLE ? p.kg : RET_SAMPLE);
    for (int j = threadIdx.x; j < rs; j += blockDim.x) s[j] = p.gidx[((int64_t)j * p.kg) / rs];
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    bool bad = false;
    for (int64_t j = t0; j < p.kg; j += stride) {
        const int32_t i = p.gidx[j];
        bad |= i < 0 || (int64_t)i >= p.n || (j > 0 && p.gidx[j - 1] >= i);
    }
    for (int64_t t = t0; t < p.total; t += stride) {
        const int64_t row = t / p.k_sent, j = t - row * p.k_sent;
        const int32_t i = p.sent_idx[t];
        if (i < 0 || (int64_t)i >= p.n || (j > 0 && p.sent_idx[t - 1] >= i)) {
            bad = true;
            continue;
        }
        if (rs > 0 && in_global(p.gidx, p.kg, s, rs, i)) continue;
        float* r = p.residual + row * p.n + i;
        *r = __fadd_rn(ld_scattered(r), p.sent_val[t]);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane_id() == 0) atomicOr(&p.ctrl->status, ST_BAD_INPUT);
}

// ---------------------------------------------------------- AllGather sum

constexpr int AG_CHUNK = 1024;       // dense outputs per warp
constexpr int AG_THREADS = 256;
constexpr int AG_WARPS = AG_THREADS / 32;
constexpr int AG_MAX_P = 256;        // rows (workers) per call
constexpr int AG_WLIST = 256;        // entries of a chunk staged in shared memory

struct AllGatherParams {
    const int32_t* idx;         // [P][k_in], rows strictly ascending
    const float* val;
    int32_t P;
    int64_t k_in;
    int64_t n;
    int64_t nchunks;            // ceil(n / AG_CHUNK)
    uint32_t* bound;            // [nchunks + 1][P]: first j of row p at or after chunk c
    float* out;                 // [n]
    Ctrl* ctrl;
};

constexpr int64_t AG_GAP = 32;       // chunk bounds one entry writes at most
constexpr uint32_t AG_UNSET = 0xFFFFFFFFu;

// bound[p][c] = first position j in row p with idx[p][j] >= c * AG_CHUNK,
// c in [0, nchunks] (row-major; the table starts filled with AG_UNSET).
// Entry j of a row writes the bounds of the chunk boundaries between its
// predecessor's chunk and its own (and the last entry those after it), at
// most AG_GAP of them; the sum kernel finds the others by search.  Rows that
// are not strictly ascending, or indices outside [0, n), set ST_BAD_INPUT
// (the sum kernel never writes outside a chunk, whatever the bounds).
__global__ void __launch_bounds__(AG_THREADS)
ag_bounds_kernel(const __grid_constant__ AllGatherParams p) {
    const int64_t total = (int64_t)p.P * p.k_in;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t nb = p.nchunks + 1;
    bool bad = false;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
        const int64_t row = t / p.k_in, j = t - row * p.k_in;
        const int32_t i = p.idx[t];
        const int32_t prev = j > 0 ? p.idx[t - 1] : -1;
        if (i < 0 || (int64_t)i >= p.n || prev >= i) {
            bad = true;
            continue;
        }
        uint32_t* br = p.bound + row * nb;
        const int64_t c = i / AG_CHUNK;
        const int64_t cp = prev < 0 ? -1 : prev / AG_CHUNK;
        for (int64_t b = cp + 1; b <= c && b <= cp + AG_GAP; ++b) br[b] = (uint32_t)j;
        if (j == p.k_in - 1)
            for (int64_t b = c + 1; b <= p.nchunks && b <= c + AG_GAP; ++b) br[b] = (uint32_t)p.k_in;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane_id() == 0) atomicOr(&p.ctrl->status, ST_BAD_INPUT);
}

// Bound b of row r from the table's entry v, or (left unset) a binary search.
__device__ __forceinline__ uint32_t ag_bound(const AllGatherParams& p, int64_t r, int64_t b,
                                             uint32_t v) {
    if (v != AG_UNSET) return v < (uint32_t)p.k_in ? v : (uint32_t)p.k_in;
    const int32_t* row = p.idx + r * p.k_in;
    const int64_t key = b * AG_CHUNK;
    int64_t lo = 0, hi = p.k_in;               // first j with row[j] >= key
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if ((int64_t)row[mid] < key) lo = mid + 1; else hi = mid;
    }
    return (uint32_t)lo;
}

// Shared memory of one warp of the sum kernel (P rows).
__host__ __device__ constexpr size_t ag_warp_bytes(int P) {
    // rounded to 16 bytes: each warp's accumulator takes float4 accesses
    return ((size_t)AG_CHUNK * 4 + (size_t)AG_WLIST * 8 + 32 * 4 + ((size_t)2 * P + 2) * 4 + 15) /
           16 * 16;
}

// Dense rank-order sum.  Each warp owns one chunk of AG_CHUNK outputs at a
// time.  The chunk's entries of all rows, in rank order (row-major), are
// staged in shared memory and applied 32 at a time: lanes that hit the same
// index form a group (__match_any_sync), and its first lane adds the group's
// values to the accumulator one after another in rank order, so every output
// is +0 plus its values in rank order.  The chunk is written once.  A chunk
// with more entries than AG_WLIST reads them from global memory batch by
// batch instead.
__global__ void __launch_bounds__(AG_THREADS)
ag_sum_kernel(const __grid_constant__ AllGatherParams p) {
    extern __shared__ __align__(16) unsigned char ag_smem[];
    const int P = p.P;
    const uint32_t lane = lane_id();
    unsigned char* mine = ag_smem + (size_t)warp_id() * ag_warp_bytes(P);
    float* acc = reinterpret_cast<float*>(mine);
    int32_t* li = reinterpret_cast<int32_t*>(acc + AG_CHUNK);
    float* lv = reinterpret_cast<float*>(li + AG_WLIST);
    float* vs = lv + AG_WLIST;                  // [32] values of the current batch
    uint32_t* lo = reinterpret_cast<uint32_t*>(vs + 32);
    uint32_t* base = lo + P;                    // [P + 1]
    const int64_t nw = (int64_t)gridDim.x * AG_WARPS;
    // each lane scans the rows [per * lane, per * lane + per)
    constexpr int PER_MAX = AG_MAX_P / 32;
    const int per = (P + 31) / 32;
    const int64_t nb = p.nchunks + 1;
    // raw table bounds of this warp's next chunk, loaded one chunk ahead
    uint32_t ta[PER_MAX], tb[PER_MAX];
    auto fetch = [&](int64_t c) {
#pragma unroll
        for (int k = 0; k < PER_MAX; ++k) {
            const int r = per * (int)lane + k;
            ta[k] = tb[k] = AG_UNSET;
            if (k < per && r < P && c < p.nchunks) {
                ta[k] = p.bound[r * nb + c];
                tb[k] = p.bound[r * nb + c + 1];
            }
        }
    };
    int64_t c = (int64_t)blockIdx.x * AG_WARPS + warp_id();
    fetch(c);
    for (; c < p.nchunks; c += nw) {
        const int64_t c0 = c * AG_CHUNK;
        const int len = (int)(p.n - c0 < AG_CHUNK ? p.n - c0 : AG_CHUNK);
#pragma unroll
        for (int i = 0; i < AG_CHUNK / 128; ++i)
            reinterpret_cast<float4*>(acc)[lane + 32 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t run = 0;
#pragma unroll
        for (int k = 0; k < PER_MAX; ++k) {
            const int r = per * (int)lane + k;
            if (k >= per || r >= P) continue;
            const uint32_t a = ag_bound(p, r, c, ta[k]);
            uint32_t b = ag_bound(p, r, c + 1, tb[k]);
            if (b < a) b = a;
            lo[r] = a;
            base[r] = run;                          // local prefix, fixed below
            run += b - a;
        }
        fetch(c + nw);
        const uint32_t incl = warp_incl_scan(run);
        const uint32_t add = incl - run;
        for (int k = 0; k < per; ++k) {
            const int r = per * (int)lane + k;
            if (r >= P) break;
            base[r] += add;
        }
        const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
        if (lane == 0) base[P] = tot;
        __syncwarp();
        const bool staged = tot <= (uint32_t)AG_WLIST;
        if (staged) {
            for (uint32_t q = lane; q < tot; q += 32) {
                int r0 = 0, r1 = P;                 // row: last base <= q
                while (r1 - r0 > 1) {
                    const int mid = (r0 + r1) >> 1;
                    if (base[mid] <= q) r0 = mid; else r1 = mid;
                }
                const int64_t t = (int64_t)r0 * p.k_in + lo[r0] + (q - base[r0]);
                li[q] = (int32_t)((int64_t)p.idx[t] - c0);
                lv[q] = p.val[t];
            }
            __syncwarp();
        }
        for (uint32_t q0 = 0; q0 < tot; q0 += 32) {
            const uint32_t q = q0 + lane;
            int32_t x = -1;
            float v = 0.f;
            if (q < tot) {
                if (staged) {
                    x = li[q];
                    v = lv[q];
                } else {
                    int r0 = 0, r1 = P;
                    while (r1 - r0 > 1) {
                        const int mid = (r0 + r1) >> 1;
                        if (base[mid] <= q) r0 = mid; else r1 = mid;
                    }
                    const int64_t t = (int64_t)r0 * p.k_in + lo[r0] + (q - base[r0]);
                    x = (int32_t)((int64_t)p.idx[t] - c0);
                    v = p.val[t];
                }
                if (x < 0 || x >= len) x = -1;      // malformed input: dropped
            }
            // lanes with the same index, in rank order (lane order = q order)
            vs[lane] = v;
            const uint32_t grp = __match_any_sync(0xFFFFFFFFu, x);
            __syncwarp();
            if (x >= 0 && (uint32_t)(__ffs(grp) - 1) == lane) {
                float s = acc[x];
                for (uint32_t m = grp; m; m &= m - 1) s = __fadd_rn(s, vs[__ffs(m) - 1]);
                acc[x] = s;
            }
            __syncwarp();
        }
        if (len == AG_CHUNK && ((uintptr_t)p.out % 16) == 0) {
            float4* o4 = reinterpret_cast<float4*>(p.out + c0);
#pragma unroll
            for (int i = 0; i < AG_CHUNK / 128; ++i)
                __stcs(o4 + lane + 32 * i, reinterpret_cast<const float4*>(acc)[lane + 32 * i]);
        } else {
            for (int i = (int)lane; i < len; i += 32) p.out[c0 + i] = acc[i];
        }
        __syncwarp();
    }
}

}  // namespace tke
