// Host side of the C ABI declared in include/topk_ef.h: argument checks,
// workspace layout and the launch sequence of each call.
//
//   topk_ef_compress / _batched:  setup_kernel -> stream_kernel -> select kernel
//                                 (flat_select_kernel for a single tensor,
//                                 select_kernel<CompressSrc> for a bucket);
//                                 a single small tensor: small_kernel alone
//   gtopk_merge:                  merge_setup_kernel -> merge_cluster_kernel per
//                                 tournament round (one thread-block cluster per
//                                 pair), or (merge_round_kernel -> select_kernel)
//                                 per round when a pair's merged list exceeds
//                                 what a cluster holds
//   topk_ef_threshold:            setup_kernel -> stream_kernel -> threshold_kernel
//   gtopk_residual_return:        return_kernel
//   topk_allgather_sum:           ag_bounds_kernel -> ag_sum_kernel
//
// Every launch goes to the caller's stream; nothing is allocated and nothing
// is synchronised except by the two status read-back calls.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstring>
#include <mutex>
#include <random>
#include <string>
#include <vector>

#include "topk_ef.h"
#include "common.cuh"
#include "kernels_compress.cuh"
#include "kernels_stream.cuh"
#include "kernels_merge.cuh"
#include "kernels_select.cuh"
#include "kernels_sparse.cuh"
#include "kernels_merge_cluster.cuh"
#include "kernels_flat.cuh"
#include "kernels_small.cuh"

using namespace tke;

namespace {

thread_local int t_last_cuda_error = 0;
std::atomic<int> g_test_flags{0};

constexpr int64_t MAX_N = 2147483647LL;
constexpr int SLOT_MAX = 2048;         // select grid never exceeds this
constexpr size_t ALIGN = 256;
constexpr int MAX_MERGE_P = 2 * SEG_MAX;   // pairs per round <= SEG_MAX

size_t align_up(size_t x, size_t a = ALIGN) { return (x + a - 1) / a * a; }

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return TOPK_EF_ERR_CUDA;
}

// ------------------------------------------------------------------ tracing
// When enabled, every kernel launch (or only those of one kernel) is
// bracketed by two CUDA events on the call's stream; records accumulate until
// they are read back.

constexpr int TRACE_MAX = 4096;

struct Trace {
    int on = 0;
    int dev = -1;
    int n = 0;
    bool open = false;          // a launch is bracketed by its first event
    std::string only;           // trace only this kernel (empty: all)
    int every = 1;              // and of those only every every-th launch
    uint64_t seen = 0;          // launches that passed the name filter
    cudaEvent_t ev[2 * TRACE_MAX] = {};
    const char* name[TRACE_MAX] = {};
};
Trace g_trace;
std::mutex g_trace_mu;

void trace_before(cudaStream_t st, const char* name) {
    g_trace.open = false;
    if (!g_trace.on || g_trace.n >= TRACE_MAX) return;
    if (!g_trace.only.empty() && g_trace.only != name) return;
    if (g_trace.seen++ % (uint64_t)g_trace.every != 0) return;
    g_trace.name[g_trace.n] = name;
    cudaEventRecord(g_trace.ev[2 * g_trace.n], st);
    g_trace.open = true;
}

void trace_after(cudaStream_t st) {
    if (!g_trace.open) return;
    g_trace.open = false;
    cudaEventRecord(g_trace.ev[2 * g_trace.n + 1], st);
    ++g_trace.n;
}

// ------------------------------------------------------------ device facts

struct DevFacts {
    int sms = 0;
    int k1_blocks = 0;       // resident stream_kernel<.., 3> blocks per SM (a bucket)
    int k1_blocks1 = 0;      // resident stream_kernel<.., 4> blocks per SM (one tensor,
                             // short candidate list)
    int selc_blocks = 0;     // resident select_kernel<CompressSrc> blocks per SM
    int selm_blocks = 0;     // resident select_kernel<MergeSrc> blocks per SM
    int fs_blocks = 0;       // resident flat_select_kernel blocks per SM
    int sk_blocks = 0;       // resident small_kernel blocks per SM
};

std::mutex g_facts_mu;
DevFacts g_facts[64];
bool g_facts_ready[64];

int device_facts(DevFacts* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return TOPK_EF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_facts_mu);
    if (!g_facts_ready[dev]) {
        DevFacts f;
        if ((e = cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f.k1_blocks,
                                                               stream_kernel<true, 3>,
                                                               K1_THREADS, 0)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f.k1_blocks1,
                                                               stream_kernel<true, 4>,
                                                               K1_THREADS, 0)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                 &f.selc_blocks, select_kernel<CompressSrc>, SEL_THREADS, 0)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                 &f.selm_blocks, select_kernel<MergeSrc>, SEL_THREADS, 0)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaFuncSetAttribute(flat_select_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)sizeof(FlatShared))) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                 &f.fs_blocks, flat_select_kernel, FS_THREADS, sizeof(FlatShared))) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaFuncSetAttribute(small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)sizeof(SmallShared))) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                 &f.sk_blocks, small_kernel, SK_THREADS, sizeof(SmallShared))) != cudaSuccess)
            return cuda_fail(e);
        if (f.sms <= 0 || f.k1_blocks <= 0 || f.k1_blocks1 <= 0 || f.selc_blocks <= 0 ||
            f.selm_blocks <= 0)
            return TOPK_EF_ERR_CUDA;
        g_facts[dev] = f;
        g_facts_ready[dev] = true;
    }
    *out = g_facts[dev];
    return TOPK_EF_OK;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel on the stream is still running, and waits for it
// (griddepcontrol.wait) before touching anything that kernel produces.
template <typename Kern, typename Arg>
cudaError_t launch_pdl(Kern kernel, int grid, int block, cudaStream_t st, const Arg& arg) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, arg);
}

// ------------------------------------------------------- compress planning

// Per tensor: samples taken for the prefilter threshold, the rank of the
// threshold among them, and the candidate capacity reserved for it.
struct TensorPlan {
    int64_t off, n, out_base;
    uint32_t k, m, r, r_hi;
    int64_t cap;
};

TensorPlan plan_tensor(int64_t off, int64_t n, int64_t k, int64_t out_base) {
    TensorPlan t;
    t.off = off;
    t.n = n;
    t.out_base = out_base;
    t.k = (uint32_t)k;
    t.m = 0;
    t.r = 0;
    t.r_hi = 0;
    if (k == 0) {
        t.cap = 0;
    } else if (n <= SAMPLE_M) {
        // every element is sampled: T0 is the exact k-th key
        t.m = (uint32_t)n;
        t.r = (uint32_t)k;
        t.r_hi = (uint32_t)k;
        t.cap = n;
    } else {
        // Expected sample count above the k-th key: ks = k * m / n.  Put the
        // threshold at the sample of rank ks + 4 sqrt(ks) + 4, below the k-th
        // key unless the sample is far from typical (then the select kernel
        // rescans the residual); rank ks - 3 sqrt(ks) - 2 estimates the k-th
        // key from above.
        const double m = (double)SAMPLE_M;
        const double ks = (double)k * m / (double)n;
        const double r = std::ceil(ks + 4.0 * std::sqrt(ks) + 4.0);
        if (r >= m) {
            t.cap = n;
        } else {
            t.m = (uint32_t)SAMPLE_M;
            t.r = (uint32_t)r;
            t.r_hi = (uint32_t)std::max(1.0, std::floor(ks - 3.0 * std::sqrt(ks) - 2.0));
            const double e = 2.5 * r * (double)n / m + 4096.0;
            t.cap = std::min<int64_t>(n, (int64_t)std::ceil(e));
        }
    }
    return t;
}

// Workspace layout of one compress group (<= TCAP_LARGE tensors).
struct CLayout {
    size_t ctrl, meta, hint, zero_begin, cand_start, ent_cnt, agg, hist, zero_end, wt_count, wt_off,
        ent, slots, cand_idx, cand_val, sk_sync, sk_idx, sk_val, total;
    int64_t cap;
    uint32_t num_wt;
};

CLayout compress_layout(int64_t N, const std::vector<TensorPlan>& plans) {
    CLayout L;
    const size_t T = plans.size();
    int64_t cap = 0;
    for (const auto& p : plans) cap += p.cap;
    L.cap = cap;
    L.num_wt = (uint32_t)ceil_div64(N, WT);
    size_t o = 0;
    L.ctrl = o;
    o = align_up(o + sizeof(Ctrl));
    L.meta = o;
    o = align_up(o + T * sizeof(SegMeta));
    L.hint = o;
    o = align_up(o + sizeof(Hint));
    L.zero_begin = o;
    L.cand_start = o;
    o = align_up(o + (T + 1) * sizeof(int64_t));
    L.ent_cnt = o;
    o = align_up(o + T * sizeof(uint32_t));
    L.agg = o;
    o = align_up(o + SLOT_MAX * sizeof(uint64_t));
    L.hist = o;
    o = align_up(o + T * CHIST_WORDS * sizeof(uint32_t));
    L.zero_end = o;
    L.wt_count = o;
    o = align_up(o + (size_t)L.num_wt * sizeof(uint32_t));
    L.wt_off = o;
    o = align_up(o + (size_t)L.num_wt * WT_CAP * sizeof(uint16_t));
    L.ent = o;
    o = align_up(o + T * (size_t)ENT_PER * sizeof(uint32_t));
    L.slots = o;
    o = align_up(o + SLOT_MAX * sizeof(Slot));
    L.cand_idx = o;
    o = align_up(o + (size_t)cap * sizeof(uint32_t));
    L.cand_val = o;
    o = align_up(o + (size_t)cap * sizeof(float));
    // a single tensor small enough for small_kernel: its arrival words and
    // its candidate regions (one per block, at the block's slice)
    L.sk_sync = L.sk_idx = L.sk_val = 0;
    if (T == 1 && N > 0 && N <= SK_N_MAX) {
        L.sk_sync = o;
        o = align_up(o + sizeof(SkSync));
        L.sk_idx = o;
        o = align_up(o + (size_t)N * sizeof(uint32_t));
        L.sk_val = o;
        o = align_up(o + (size_t)N * sizeof(float));
    }
    L.total = o;
    return L;
}

// Validated per-group description of a (batched) compress call.
struct Group {
    int32_t t0, t1;                 // tensors [t0, t1)
    std::vector<TensorPlan> plans;  // offsets local to the group
    int64_t base;                   // first element of the group in the bucket
    int64_t N;                      // elements in the group
};

int make_groups(const int64_t* offsets, const int64_t* k, int32_t T, std::vector<Group>* out) {
    if (!offsets || !k || T < 1) return TOPK_EF_ERR_INVALID_ARG;
    if (offsets[0] != 0) return TOPK_EF_ERR_INVALID_ARG;
    for (int32_t l = 0; l < T; ++l) {
        const int64_t n = offsets[l + 1] - offsets[l];
        if (n < 0 || k[l] < 0 || k[l] > n) return TOPK_EF_ERR_INVALID_ARG;
    }
    if (offsets[T] > MAX_N) return TOPK_EF_ERR_INVALID_ARG;
    int64_t out_base = 0;
    for (int32_t g0 = 0; g0 < T; g0 += TCAP_LARGE) {
        Group g;
        g.t0 = g0;
        g.t1 = std::min<int32_t>(T, g0 + TCAP_LARGE);
        g.base = offsets[g0];
        g.N = offsets[g.t1] - g.base;
        for (int32_t l = g.t0; l < g.t1; ++l) {
            g.plans.push_back(plan_tensor(offsets[l] - g.base, offsets[l + 1] - offsets[l], k[l],
                                          out_base));
            out_base += k[l];
        }
        out->push_back(std::move(g));
    }
    return TOPK_EF_OK;
}

size_t groups_workspace(const std::vector<Group>& groups) {
    size_t mx = 0;
    for (const auto& g : groups) mx = std::max(mx, compress_layout(g.N, g.plans).total);
    return mx;
}

template <int TCAP>
cudaError_t launch_setup(const Group& g, const CLayout& L, char* ws, const float* grad,
                         const float* resid, float lr, bool force_t0_zero, uint32_t kernels,
                         cudaStream_t st, const uint32_t* fixed_T0 = nullptr,
                         uint64_t hint_tag = 0, uint32_t stall = 0) {
    SetupParams<TCAP> p;
    memset(&p, 0, sizeof(p));
    if (fixed_T0) {
        p.has_fixed_T0 = 1;
        p.fixed_T0 = *fixed_T0;
        force_t0_zero = true;          // no sampling
    }
    const int T = (int)g.plans.size();
    p.grad = grad;
    p.resid = resid;
    p.lr = lr;
    p.T = T;
    p.kernels = kernels;
    p.cap = (uint64_t)L.cap;
    p.ctrl = reinterpret_cast<Ctrl*>(ws + L.ctrl);
    p.meta = reinterpret_cast<SegMeta*>(ws + L.meta);
    p.zero_ptr = reinterpret_cast<uint4*>(ws + L.zero_begin);
    p.zero_vec4 = (L.zero_end - L.zero_begin) / 16;
    p.stall = stall;
    // a single tensor whose threshold comes from a true sample may take the
    // previous call's instead
    p.hint = reinterpret_cast<const Hint*>(ws + L.hint);
    p.hint_tag = (g.plans.size() == 1 && g.plans[0].m == (uint32_t)SAMPLE_M && !force_t0_zero)
                     ? hint_tag : 0;
    int ns = 0;
    for (int l = 0; l < T; ++l) {
        const TensorPlan& t = g.plans[l];
        p.off[l] = t.off;
        p.out_base[l] = t.out_base;
        p.k[l] = t.k;
        p.m[l] = force_t0_zero ? 0u : t.m;
        p.r[l] = t.r;
        p.r_hi[l] = t.r_hi;
        if (p.m[l]) p.sampled[ns++] = (uint16_t)l;
    }
    p.off[T] = g.N;
    p.n_sampled = ns;
    const uint64_t per_block = (uint64_t)ZERO_THREADS * 8;
    const int nz = (int)std::max<uint64_t>(1, std::min<uint64_t>(148, (p.zero_vec4 + per_block - 1) / per_block));
    return launch_pdl(setup_kernel<TCAP>, ns + nz, SAMPLE_THREADS, st, p);
}

// The streaming pass of one group (after its setup kernel, with
// programmatic serialisation); fills *sp for the select kernels.
cudaError_t launch_stream(const Group& g, const CLayout& L, char* ws, const float* gg, float* rg,
                          float lr, cudaStream_t st, const DevFacts& f, StreamParams* sp_out,
                          bool build_r1, bool four = false) {
    StreamParams sp;
    sp.grad = gg;
    sp.resid = rg;
    sp.lr = lr;
    sp.T = (int)g.plans.size();
    sp.N = g.N;
    sp.num_wt = L.num_wt;
    sp.meta = reinterpret_cast<const SegMeta*>(ws + L.meta);
    sp.ctrl = reinterpret_cast<Ctrl*>(ws + L.ctrl);
    sp.wt_count = reinterpret_cast<uint32_t*>(ws + L.wt_count);
    sp.wt_off = reinterpret_cast<uint16_t*>(ws + L.wt_off);
    // one tensor: the streaming pass builds the candidates' relative digit 1
    sp.r1 = build_r1 && g.plans.size() == 1
                ? reinterpret_cast<uint32_t*>(ws + L.hist) + CH_R1
                : nullptr;
    *sp_out = sp;
    const bool vec = ((uintptr_t)gg % 16 == 0) && ((uintptr_t)rg % 16 == 0);
    const bool one = four && g.plans.size() == 1;
    const int64_t warps_needed = L.num_wt;
    const int per_sm = one ? f.k1_blocks1 : f.k1_blocks;
    const int g1 = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div64(warps_needed, K1_THREADS / 32),
                                                               (int64_t)f.sms * per_sm));
    trace_before(st, "stream_kernel");
    cudaError_t e;
    if (one)
        e = vec ? launch_pdl(stream_kernel<true, 4>, g1, K1_THREADS, st, sp)
                : launch_pdl(stream_kernel<false, 4>, g1, K1_THREADS, st, sp);
    else
        e = vec ? launch_pdl(stream_kernel<true, 3>, g1, K1_THREADS, st, sp)
                : launch_pdl(stream_kernel<false, 3>, g1, K1_THREADS, st, sp);
    trace_after(st);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e;
}

// Select-kernel view of a group's workspace (the compress defaults).
CompressSrc make_src(const Group& g, const CLayout& L, char* ws, const StreamParams& sp,
                     float* rg) {
    CompressSrc src;
    memset(&src, 0, sizeof(src));
    src.resid = rg;
    src.N = g.N;
    src.T = (int)g.plans.size();
    src.meta = sp.meta;
    src.cand_start = reinterpret_cast<int64_t*>(ws + L.cand_start);
    src.cand_idx = reinterpret_cast<uint32_t*>(ws + L.cand_idx);
    src.cand_val = reinterpret_cast<float*>(ws + L.cand_val);
    src.cap = (uint64_t)L.cap;
    src.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
    src.num_wt = L.num_wt;
    src.wt_count = sp.wt_count;
    src.wt_off = sp.wt_off;
    src.ent = reinterpret_cast<uint32_t*>(ws + L.ent);
    src.ent_cnt = reinterpret_cast<uint32_t*>(ws + L.ent_cnt);
    src.agg = reinterpret_cast<uint64_t*>(ws + L.agg);
    return src;
}

// Tag of a flat compress call for the threshold hint: the next call may use
// this call's threshold only for the same residual, n, k and lr.
uint64_t hint_tag_of(const float* resid, int64_t n, uint32_t k, float lr) {
    auto mix = [](uint64_t x) {
        x += 0x9E3779B97F4A7C15ull;
        x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
        x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
        return x ^ (x >> 31);
    };
    uint32_t lb;
    memcpy(&lb, &lr, sizeof lb);
    uint64_t h = mix((uint64_t)(uintptr_t)resid);
    h = mix(h ^ (uint64_t)n);
    h = mix(h ^ ((uint64_t)k << 32 | lb));
    return h ? h : 1;
}

// A number distinct for every small_kernel launch of this process (a counter
// mixed with a per-process random start).  The kernel mixes it with the
// workspace's own call counter, so that a replayed graph differs too.
uint64_t next_call_tag() {
    static std::atomic<uint64_t> ctr{0};
    static const uint64_t start = [] {
        std::random_device rd;
        const uint64_t t = (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
        return ((uint64_t)rd() << 32) ^ (uint64_t)rd() ^ (t * 0x9E3779B97F4A7C15ull);
    }();
    return start + 0xD1B54A32D192ED03ull * (ctr.fetch_add(1) + 1);
}

int compress_group(const Group& g, const float* grad, float* resid, float lr, int32_t* out_idx,
                   float* out_val, char* ws, cudaStream_t st, const DevFacts& f, int flags) {
    const CLayout L = compress_layout(g.N, g.plans);
    const int T = (int)g.plans.size();
    const bool force_dense = (flags & 1) != 0;
    const bool force_t0 = (flags & 2) != 0;
    const uint32_t stall = (flags & 4) != 0 ? 1u : 0u;
    const float* gg = grad + g.base;
    float* rg = resid + g.base;
    // A single tensor takes flat_select_kernel, one block per SM, when its
    // candidate capacity is within what that grid stages in one round per
    // block; a bucket (or a huge tensor) takes the segmented select.
    const int G_flat = std::min(SLOT_MAX, f.sms);
    // A single tensor that one wave of blocks holds in shared memory takes
    // small_kernel alone: one launch, no setup
    const int sm_cap = std::min(SK_GRID_MAX, f.sms);
    const bool small = T == 1 && f.sk_blocks >= 1 && g.N > 0 && g.plans[0].k > 0 &&
                       !force_dense && L.sk_sync != 0 && g.N <= (int64_t)sm_cap * SK_MAX;
    if (small) {
        const int G = (int)std::max<int64_t>(1, std::min<int64_t>(sm_cap,
                                                   ceil_div64(g.N, SK_MIN_PER_BLOCK)));
        SmallParams kp;
        kp.grad = grad + g.base;
        kp.resid = resid + g.base;
        kp.n = g.N;
        kp.lr = lr;
        kp.k = g.plans[0].k;
        kp.out_idx = out_idx + g.plans[0].out_base;
        kp.out_val = out_val + g.plans[0].out_base;
        kp.ctrl = reinterpret_cast<Ctrl*>(ws + L.ctrl);
        static_assert(CH_R2 == CH_R1 + SK_BINS / 2 && CH_D1 == CH_R1 + SK_BINS &&
                      CHIST_WORDS - CH_D1 >= 1024, "small-kernel histograms in the tensor's words");
        kp.hist = reinterpret_cast<uint32_t*>(ws + L.hist) + CH_R1;
        kp.hist2 = reinterpret_cast<uint32_t*>(ws + L.hist) + CH_D1;
        kp.ent = reinterpret_cast<uint32_t*>(ws + L.ent);
        kp.ent_cnt = reinterpret_cast<uint32_t*>(ws + L.ent_cnt);
        kp.slots = reinterpret_cast<Slot*>(ws + L.slots);
        kp.sync = reinterpret_cast<SkSync*>(ws + L.sk_sync);
        kp.cand_idx = reinterpret_cast<uint32_t*>(ws + L.sk_idx);
        kp.cand_val = reinterpret_cast<float*>(ws + L.sk_val);
        kp.hint = reinterpret_cast<Hint*>(ws + L.hint);
        // the threshold hint: for a k that block 0 can select from alone, and
        // tagged apart from the flat path's hint
        kp.hint_tag = kp.k <= SK_HINT_KMAX && !force_t0
                          ? (hint_tag_of(rg, g.N, kp.k, lr) ^ 0x5A5A5A5A00000000ull) | 1ull : 0;
        kp.call_tag = next_call_tag();
        kp.force_t0 = force_t0 ? 1u : 0u;
        kp.stall = stall;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G);
        cfg.blockDim = dim3(SK_THREADS);
        cfg.dynamicSmemBytes = sizeof(SmallShared);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        trace_before(st, "small_kernel");
        const cudaError_t e = cudaLaunchKernelEx(&cfg, small_kernel, kp);
        trace_after(st);
        return e == cudaSuccess ? TOPK_EF_OK : cuda_fail(e);
    }
    const bool flat = T == 1 && f.fs_blocks >= 1 && L.cap <= (int64_t)G_flat * FS_CAND;
    const bool flat_skip = flat && g.plans[0].k == 0;   // nothing to select
    const uint32_t kernels = g.N > 0 ? (flat_skip ? 2u : 3u) : 1u;
    const uint64_t tag = flat && !force_t0 && !force_dense
                             ? hint_tag_of(rg, g.N, g.plans[0].k, lr) : 0;
    trace_before(st, "setup_kernel");
    cudaError_t e = T <= TCAP_SMALL
                        ? launch_setup<TCAP_SMALL>(g, L, ws, gg, rg, lr, force_t0, kernels, st,
                                                   nullptr, tag, stall)
                        : launch_setup<TCAP_LARGE>(g, L, ws, gg, rg, lr, force_t0, kernels, st);
    trace_after(st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (g.N == 0) return TOPK_EF_OK;

    // a single tensor: the streaming pass builds relative digit 1 (for the
    // segmented select only when the candidate list is short; long lists
    // would pay more in the streaming pass than the barrier it saves costs)
    const bool build_r1 = T == 1 && (flat || L.cap <= ((int64_t)1 << 19));
    StreamParams sp;
    // the flat select with a short candidate list: 4 streaming blocks per SM
    const bool four = flat && L.cap <= ((int64_t)1 << 19);
    if ((e = launch_stream(g, L, ws, gg, rg, lr, st, f, &sp, build_r1, four)) != cudaSuccess)
        return cuda_fail(e);
    if (flat_skip) return TOPK_EF_OK;
    Ctrl* ctrl = sp.ctrl;

    CompressSrc src = make_src(g, L, ws, sp, rg);
    src.out_idx = out_idx;
    src.out_val = out_val;
    src.r1_done = sp.r1 != nullptr ? 1 : 0;
    src.force_dense = force_dense ? 1 : 0;
    src.dense = 0;
    SelCommon cm;
    cm.ctrl = ctrl;
    cm.bar = &ctrl->bar;
    cm.slots = reinterpret_cast<Slot*>(ws + L.slots);
    if (flat) {
        // a normal launch chained to the streaming pass; its blocks exchange
        // counts once through global memory, which needs the whole grid (one
        // block per SM) resident: every wait in it is bounded
        FlatParams fp;
        fp.src = src;
        // no dense list here: the bound on the candidates is what the grid
        // stages in one round per block
        fp.src.cap = (uint64_t)G_flat * FS_CAND;
        fp.cm = cm;
        fp.hint = reinterpret_cast<Hint*>(ws + L.hint);
        fp.hint_tag = tag;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G_flat);
        cfg.blockDim = dim3(FS_THREADS);
        cfg.dynamicSmemBytes = sizeof(FlatShared);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        trace_before(st, "flat_select_kernel");
        e = cudaLaunchKernelEx(&cfg, flat_select_kernel, fp);
        trace_after(st);
        if (e != cudaSuccess) return cuda_fail(e);
        return TOPK_EF_OK;
    }
    // one block per SM: cheaper grid barriers, no less bandwidth for the
    // small candidate list (the rescan fallback is still memory bound)
    const int G = std::min(SLOT_MAX, f.sms * std::min(1, f.selc_blocks));
    void* args[] = {&src, &cm};
    trace_before(st, "select_kernel<CompressSrc>");
    e = cudaLaunchCooperativeKernel((const void*)select_kernel<CompressSrc>, dim3(G),
                                    dim3(SEL_THREADS), args, 0, st);
    trace_after(st);
    if (e != cudaSuccess) return cuda_fail(e);
    return TOPK_EF_OK;
}

// Hard-threshold step on one flat tensor: setup (fixed T0, no sampling),
// the streaming pass, and the threshold kernel writing the output.
int threshold_call(const float* grad, float* resid, int64_t n, float lr, uint32_t T0,
                   int64_t max_out, int32_t* out_idx, float* out_val, int64_t* out_count,
                   char* ws, cudaStream_t st, const DevFacts& f) {
    Group g;
    g.t0 = 0;
    g.t1 = 1;
    g.base = 0;
    g.N = n;
    TensorPlan t = plan_tensor(0, n, 0, 0);
    t.cap = 0;
    g.plans.push_back(t);
    const CLayout L = compress_layout(n, g.plans);
    const uint32_t kernels = n > 0 ? 3u : 1u;
    trace_before(st, "setup_kernel");
    cudaError_t e = launch_setup<TCAP_SMALL>(g, L, ws, grad, resid, lr, true, kernels, st, &T0);
    trace_after(st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) {
        e = cudaMemsetAsync(out_count, 0, sizeof(int64_t), st);
        return e == cudaSuccess ? TOPK_EF_OK : cuda_fail(e);
    }
    StreamParams sp;
    if ((e = launch_stream(g, L, ws, grad, resid, lr, st, f, &sp, false)) != cudaSuccess)
        return cuda_fail(e);
    CompressSrc src = make_src(g, L, ws, sp, resid);
    src.cand_idx = reinterpret_cast<uint32_t*>(out_idx);
    src.cand_val = out_val;
    src.cap = (uint64_t)std::min<int64_t>(max_out, n);
    src.rq = reinterpret_cast<uint4*>(ws + L.hist);   // cleared by the setup kernel
    SelCommon cm;
    cm.ctrl = sp.ctrl;
    cm.bar = &sp.ctrl->bar;
    cm.slots = reinterpret_cast<Slot*>(ws + L.slots);
    const int G = std::min(SLOT_MAX, f.sms * std::min(1, f.selc_blocks));
    void* args[] = {&src, &cm, &out_count};
    trace_before(st, "threshold_kernel");
    e = cudaLaunchCooperativeKernel((const void*)threshold_kernel, dim3(G), dim3(SEL_THREADS),
                                    args, 0, st);
    trace_after(st);
    return e == cudaSuccess ? TOPK_EF_OK : cuda_fail(e);
}

size_t threshold_workspace(int64_t n) {
    std::vector<TensorPlan> plans(1, plan_tensor(0, n, 0, 0));
    plans[0].cap = 0;
    return compress_layout(n, plans).total;
}

// The cluster merge kernel: one cluster of CL CTAs per pair, CL = 16, 14 or
// 12 at two CTAs per SM (sizes above 8 are non-portable) or 8 at one.  How
// many clusters of each size the device holds at once is found once per
// device.
constexpr int MC_SIZES[4] = {16, 14, 12, 8};
struct McFit {
    int active[4];              // resident clusters of MC_SIZES[i] CTAs (0: cannot run)
};
std::mutex g_mc_mu;
bool g_mc_probed[64];
McFit g_mc_fit[64];

template <int CL>
cudaError_t mc_config(int* active) {
    *active = 0;
    cudaError_t e = cudaFuncSetAttribute(merge_cluster_kernel<CL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)mc_smem_bytes<CL>());
    if (e == cudaSuccess && CL > 8)
        e = cudaFuncSetAttribute(merge_cluster_kernel<CL>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) {
        cudaGetLastError();            // not available on this device: try the next size
        return cudaSuccess;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL);
    cfg.blockDim = dim3(MC_THREADS);
    cfg.dynamicSmemBytes = mc_smem_bytes<CL>();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, merge_cluster_kernel<CL>, &cfg);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cudaSuccess;
    }
    *active = clusters > 0 ? clusters : 0;
    return cudaSuccess;
}

int merge_cluster_fit(McFit* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return TOPK_EF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mc_mu);
    if (!g_mc_probed[dev]) {
        McFit f;
        if ((e = mc_config<16>(&f.active[0])) != cudaSuccess) return cuda_fail(e);
        if ((e = mc_config<14>(&f.active[1])) != cudaSuccess) return cuda_fail(e);
        if ((e = mc_config<12>(&f.active[2])) != cudaSuccess) return cuda_fail(e);
        if ((e = mc_config<8>(&f.active[3])) != cudaSuccess) return cuda_fail(e);
        g_mc_fit[dev] = f;
        g_mc_probed[dev] = true;
    }
    *out = g_mc_fit[dev];
    return TOPK_EF_OK;
}

int64_t mc_cap(int i) {
    switch (i) {
        case 0: return mc_pair_cap<16>();
        case 1: return mc_pair_cap<14>();
        case 2: return mc_pair_cap<12>();
        default: return mc_pair_cap<8>();
    }
}

// Cluster size of a round of np pairs whose merged lists hold up to mcap
// positions (0: no size can run it).  16 CTAs per pair when the device holds
// all np such clusters at once.  Else the largest of 14 and 12 of which it
// does: fewer CTAs per pair, but one wave of clusters instead of two.  Else
// 16 in several waves (they still ran faster than one wave of 8-CTA clusters
// at one CTA per SM: 43.7 against 53.5 us for the first round of the
// 32-worker tournament), or 8 where the device holds no larger cluster.
// `forced` (a test flag: an index into MC_SIZES, or -1) picks a size
// wherever that size can run.
int round_cluster(const McFit& f, int32_t np, int64_t mcap, int forced) {
    auto fits = [&](int i) { return f.active[i] > 0 && mcap <= mc_cap(i); };
    if (forced >= 0 && forced < 4 && fits(forced)) return MC_SIZES[forced];
    if (fits(0) && np <= f.active[0]) return 16;
    for (int i = 1; i <= 2; ++i)
        if (fits(i) && np <= f.active[i]) return MC_SIZES[i];
    if (fits(0)) return 16;
    return fits(3) ? 8 : 0;
}

template <int CL>
cudaError_t launch_mc(int32_t np, cudaStream_t st, const MergeClusterParams& cp) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)np * CL);
    cfg.blockDim = dim3(MC_THREADS);
    cfg.dynamicSmemBytes = mc_smem_bytes<CL>();
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, merge_cluster_kernel<CL>, cp);
}

cudaError_t launch_merge_cluster(int cl, int32_t np, cudaStream_t st,
                                 const MergeClusterParams& cp) {
    switch (cl) {
        case 16: return launch_mc<16>(np, st, cp);
        case 14: return launch_mc<14>(np, st, cp);
        case 12: return launch_mc<12>(np, st, cp);
        default: return launch_mc<8>(np, st, cp);
    }
}

bool bad_fp32_ptr(const void* p) { return ((uintptr_t)p & 3u) != 0; }

// ------------------------------------------- compress without allocation
// Scratch for topk_ef_compress_static: one array in the module's global
// memory.  Each GPU that loads this library holds it until the process ends.
// In host code `g_static_scratch` is only a host-side stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress, taken once per
// device with that device current.
constexpr size_t STATIC_SCRATCH_BYTES = TOPK_EF_STATIC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_static_scratch[STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void* g_static_addr[64];

int static_scratch_addr(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return TOPK_EF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_static_addr[dev] = ptr;
    }
    *out = g_static_addr[dev];
    return TOPK_EF_OK;
}

// --------------------------------------------------------- merge planning

struct MLayout {
    size_t ctrl, sizes, floors, bad, zero_begin, hist, live, zero_end, slots, set_idx, set_val, m_idx,
        m_val, total;
    int64_t cap;
    int rounds;
    std::vector<int32_t> np;       // pairs per round
    std::vector<int64_t> mcap;     // merged positions per pair per round
    std::vector<int64_t> pbase;    // first pair-merge id of each round
    int64_t merges;                // total pair merges
    int64_t mmax;                  // merged positions buffer
    uint32_t vblocks;
};

MLayout merge_layout(int32_t P, int64_t k_in, int64_t k) {
    MLayout L;
    L.cap = std::max<int64_t>(1, std::max<int64_t>(k_in, std::min<int64_t>(k, (int64_t)P * k_in)));
    L.rounds = 0;
    while ((1LL << L.rounds) < P) ++L.rounds;
    L.merges = 0;
    L.mmax = 0;
    for (int r = 0; r < L.rounds; ++r) {
        const int64_t step = 1LL << r;
        const int32_t np = (int32_t)((P - step - 1) / (2 * step) + 1);
        const int64_t bound = std::min<int64_t>(L.cap, k_in << std::min(r, 40));
        const int64_t mc = 2 * std::max<int64_t>(bound, 1);
        L.np.push_back(np);
        L.mcap.push_back(mc);
        L.pbase.push_back(L.merges);
        L.merges += np;
        L.mmax = std::max<int64_t>(L.mmax, (int64_t)np * mc);
    }
    const int64_t hsegs = std::max<int64_t>(1, L.merges);
    const int64_t tot = (int64_t)P * k_in;
    L.vblocks = tot > 0 ? (uint32_t)std::min<int64_t>(148, ceil_div64(tot, MZ_THREADS * 8)) : 0u;
    size_t o = 0;
    L.ctrl = o;
    o = align_up(o + sizeof(Ctrl));
    L.sizes = o;
    o = align_up(o + (size_t)P * sizeof(uint32_t));
    L.floors = o;
    o = align_up(o + (size_t)P * sizeof(uint32_t));
    L.bad = o;
    o = align_up(o + 148 * sizeof(uint32_t));
    L.zero_begin = o;
    L.hist = o;
    o = align_up(o + (size_t)hsegs * MHIST_WORDS * sizeof(uint32_t));
    L.live = o;
    o = align_up(o + (size_t)hsegs * sizeof(uint32_t));
    L.zero_end = o;
    L.slots = o;
    o = align_up(o + SLOT_MAX * sizeof(Slot));
    L.set_idx = o;
    o = align_up(o + (size_t)P * L.cap * sizeof(uint32_t));
    L.set_val = o;
    o = align_up(o + (size_t)P * L.cap * sizeof(float));
    L.m_idx = o;
    o = align_up(o + (size_t)L.mmax * sizeof(uint32_t));
    L.m_val = o;
    o = align_up(o + (size_t)L.mmax * sizeof(float));
    L.total = o;
    return L;
}

int merge_args_ok(int32_t P, int64_t k_in, int64_t k, int64_t n) {
    if (P < 1 || P > MAX_MERGE_P || k_in < 0 || k < 0 || n < 0 || n > MAX_N || k_in > n)
        return TOPK_EF_ERR_INVALID_ARG;
    if (k > MAX_N || (int64_t)P * k_in > (int64_t)1 << 40) return TOPK_EF_ERR_INVALID_ARG;
    return TOPK_EF_OK;
}

}  // namespace

// ================================================================ C ABI

extern "C" {

size_t topk_ef_workspace_bytes(int64_t n, int64_t k) {
    if (n < 0 || k < 0 || k > n || n > MAX_N) return 0;
    const int64_t offsets[2] = {0, n};
    return topk_ef_batched_workspace_bytes(offsets, &k, 1);
}

size_t topk_ef_batched_workspace_bytes(const int64_t* offsets, const int64_t* k, int32_t T) {
    std::vector<Group> groups;
    if (make_groups(offsets, k, T, &groups) != TOPK_EF_OK) return 0;
    return groups_workspace(groups);
}

int topk_ef_compress_batched(const float* grad, float* residual, const int64_t* offsets,
                             const int64_t* k, int32_t T, float lr, int32_t* out_idx,
                             float* out_val, void* ws, size_t ws_bytes, void* stream) {
    std::vector<Group> groups;
    int rc = make_groups(offsets, k, T, &groups);
    if (rc != TOPK_EF_OK) return rc;
    const int64_t N = offsets[T];
    int64_t ktot = 0;
    for (int32_t l = 0; l < T; ++l) ktot += k[l];
    if (!ws) return TOPK_EF_ERR_INVALID_ARG;
    if (N > 0 && (!grad || !residual || bad_fp32_ptr(grad) || bad_fp32_ptr(residual)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (ktot > 0 && (!out_idx || !out_val || bad_fp32_ptr(out_val) || bad_fp32_ptr(out_idx)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (((uintptr_t)ws % ALIGN) != 0) return TOPK_EF_ERR_INVALID_ARG;
    if (ws_bytes < groups_workspace(groups)) return TOPK_EF_ERR_WORKSPACE;
    DevFacts f;
    if ((rc = device_facts(&f)) != TOPK_EF_OK) return rc;
    const int flags = g_test_flags.load();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (const auto& g : groups) {
        rc = compress_group(g, grad, residual, lr, out_idx, out_val, (char*)ws, st, f, flags);
        if (rc != TOPK_EF_OK) return rc;
    }
    return TOPK_EF_OK;
}

int topk_ef_compress(const float* grad, float* residual, int64_t n, float lr, int64_t k,
                     int32_t* out_idx, float* out_val, void* ws, size_t ws_bytes, void* stream) {
    if (n < 0 || k < 0 || k > n || n > MAX_N) return TOPK_EF_ERR_INVALID_ARG;
    const int64_t offsets[2] = {0, n};
    return topk_ef_compress_batched(grad, residual, offsets, &k, 1, lr, out_idx, out_val, ws,
                                    ws_bytes, stream);
}

int topk_ef_compress_static(const float* grad, float* residual, int64_t n, float lr, int64_t k,
                            int32_t* out_idx, float* out_val, void* stream) {
    if (n < 0 || k < 0 || k > n || n > MAX_N) return TOPK_EF_ERR_INVALID_ARG;
    const size_t need = topk_ef_workspace_bytes(n, k);
    if (need == 0) return TOPK_EF_ERR_INVALID_ARG;
    if (need > STATIC_SCRATCH_BYTES) return TOPK_EF_ERR_WORKSPACE;
    void* ws = nullptr;
    const int rc = static_scratch_addr(&ws);
    if (rc != TOPK_EF_OK) return rc;
    return topk_ef_compress(grad, residual, n, lr, k, out_idx, out_val, ws, STATIC_SCRATCH_BYTES,
                            stream);
}

int topk_ef_static_last_device_status(void* stream) {
    void* ws = nullptr;
    const int rc = static_scratch_addr(&ws);
    if (rc != TOPK_EF_OK) return rc;
    return topk_ef_last_device_status(ws, stream);
}

size_t topk_ef_threshold_workspace_bytes(int64_t n) {
    if (n < 0 || n > MAX_N) return 0;
    return threshold_workspace(n);
}

int topk_ef_threshold(const float* grad, float* residual, int64_t n, float lr, float threshold,
                      int64_t max_out, int32_t* out_idx, float* out_val, int64_t* out_count,
                      void* ws, size_t ws_bytes, void* stream) {
    if (n < 0 || n > MAX_N || max_out < 0 || !out_count || !ws) return TOPK_EF_ERR_INVALID_ARG;
    if (n > 0 && (!grad || !residual || bad_fp32_ptr(grad) || bad_fp32_ptr(residual)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (max_out > 0 && (!out_idx || !out_val || bad_fp32_ptr(out_idx) || bad_fp32_ptr(out_val)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (((uintptr_t)out_count % 8) != 0 || ((uintptr_t)ws % ALIGN) != 0)
        return TOPK_EF_ERR_INVALID_ARG;
    if (ws_bytes < threshold_workspace(n)) return TOPK_EF_ERR_WORKSPACE;
    DevFacts f;
    int rc = device_facts(&f);
    if (rc != TOPK_EF_OK) return rc;
    // key of the threshold; never above 0x7F800001, so that the streaming
    // pass's raw |bits| test and the key order agree (a NaN threshold passes
    // exactly the NaNs)
    uint32_t u;
    memcpy(&u, &threshold, sizeof u);
    uint32_t T0 = u & 0x7FFFFFFFu;
    if (T0 > 0x7F800001u) T0 = 0x7F800001u;
    return threshold_call(grad, residual, n, lr, T0, max_out, out_idx, out_val, out_count,
                          (char*)ws, reinterpret_cast<cudaStream_t>(stream), f);
}

size_t gtopk_residual_return_workspace_bytes(void) { return align_up(sizeof(Ctrl)); }

int gtopk_residual_return(const int32_t* sent_idx, const float* sent_val, int32_t P,
                          int64_t k_sent, const int32_t* global_idx, int64_t k_global,
                          float* residual, int64_t n, void* ws, size_t ws_bytes, void* stream) {
    if (P < 1 || k_sent < 0 || k_global < 0 || n < 0 || n > MAX_N || k_sent > n || k_global > n)
        return TOPK_EF_ERR_INVALID_ARG;
    if (!ws || ((uintptr_t)ws % ALIGN) != 0) return TOPK_EF_ERR_INVALID_ARG;
    if (k_sent > 0 && (!sent_idx || !sent_val || !residual || bad_fp32_ptr(sent_idx) ||
                       bad_fp32_ptr(sent_val) || bad_fp32_ptr(residual)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (k_global > 0 && (!global_idx || bad_fp32_ptr(global_idx))) return TOPK_EF_ERR_INVALID_ARG;
    if (ws_bytes < gtopk_residual_return_workspace_bytes()) return TOPK_EF_ERR_WORKSPACE;
    DevFacts f;
    int rc = device_facts(&f);
    if (rc != TOPK_EF_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(Ctrl), st);
    if (e != cudaSuccess) return cuda_fail(e);
    ReturnParams p;
    p.sent_idx = sent_idx;
    p.sent_val = sent_val;
    p.k_sent = k_sent;
    p.total = (int64_t)P * k_sent;
    p.gidx = global_idx;
    p.kg = k_global;
    p.residual = residual;
    p.n = n;
    p.ctrl = reinterpret_cast<Ctrl*>(ws);
    const int64_t work = std::max<int64_t>(p.total, k_global);
    if (work == 0) return TOPK_EF_OK;
    // one wave of resident blocks (grid-stride over the entries)
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, return_kernel, RET_THREADS,
                                                           0)) != cudaSuccess)
        return cuda_fail(e);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div64(work, RET_THREADS), (int64_t)f.sms * std::max(1, per_sm)));
    trace_before(st, "return_kernel");
    return_kernel<<<grid, RET_THREADS, 0, st>>>(p);
    trace_after(st);
    e = cudaGetLastError();
    return e == cudaSuccess ? TOPK_EF_OK : cuda_fail(e);
}

size_t topk_allgather_workspace_bytes(int32_t P, int64_t k_in, int64_t n) {
    if (P < 1 || P > AG_MAX_P || k_in < 0 || n < 0 || n > MAX_N || k_in > n) return 0;
    const int64_t nchunks = ceil_div64(n, AG_CHUNK);
    return align_up(sizeof(Ctrl)) + align_up((size_t)(nchunks + 1) * P * sizeof(uint32_t));
}

int topk_allgather_sum(const int32_t* in_idx, const float* in_val, int32_t P, int64_t k_in,
                       int64_t n, float* out, void* ws, size_t ws_bytes, void* stream) {
    const size_t need = topk_allgather_workspace_bytes(P, k_in, n);
    if (need == 0 || !ws || ((uintptr_t)ws % ALIGN) != 0) return TOPK_EF_ERR_INVALID_ARG;
    if (k_in > 0 && (!in_idx || !in_val || bad_fp32_ptr(in_idx) || bad_fp32_ptr(in_val)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (n > 0 && (!out || bad_fp32_ptr(out))) return TOPK_EF_ERR_INVALID_ARG;
    if (ws_bytes < need) return TOPK_EF_ERR_WORKSPACE;
    DevFacts f;
    int rc = device_facts(&f);
    if (rc != TOPK_EF_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    AllGatherParams p;
    p.idx = in_idx;
    p.val = in_val;
    p.P = P;
    p.k_in = k_in;
    p.n = n;
    p.nchunks = ceil_div64(n, AG_CHUNK);
    p.bound = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + align_up(sizeof(Ctrl)));
    p.out = out;
    p.ctrl = reinterpret_cast<Ctrl*>(ws);
    const size_t bound_bytes = (size_t)(p.nchunks + 1) * P * sizeof(uint32_t);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(Ctrl), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.bound, 0xFF, bound_bytes, st);   // AG_UNSET
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) return TOPK_EF_OK;
    const int64_t total = (int64_t)P * k_in;
    if (total > 0) {
        const int gb = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div64(total, AG_THREADS),
                                                                  (int64_t)f.sms * 8));
        trace_before(st, "ag_bounds_kernel");
        ag_bounds_kernel<<<gb, AG_THREADS, 0, st>>>(p);
        trace_after(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
    }
    const size_t smem = (size_t)AG_WARPS * ag_warp_bytes(P);
    if ((e = cudaFuncSetAttribute(ag_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return cuda_fail(e);
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ag_sum_kernel, AG_THREADS,
                                                           smem)) != cudaSuccess)
        return cuda_fail(e);
    const int64_t want = ceil_div64(p.nchunks, AG_WARPS);
    const int gs = (int)std::max<int64_t>(1, std::min<int64_t>(want,
                                                              (int64_t)f.sms * std::max(1, per_sm)));
    trace_before(st, "ag_sum_kernel");
    ag_sum_kernel<<<gs, AG_THREADS, smem, st>>>(p);
    trace_after(st);
    e = cudaGetLastError();
    return e == cudaSuccess ? TOPK_EF_OK : cuda_fail(e);
}

size_t gtopk_merge_workspace_bytes(int32_t P, int64_t k_in, int64_t k) {
    if (P < 1 || P > MAX_MERGE_P || k_in < 0 || k < 0) return 0;
    return merge_layout(P, k_in, k).total;
}

int gtopk_merge(const int32_t* in_idx, const float* in_val, int32_t P, int64_t k_in, int64_t k,
                int64_t n, int32_t* out_idx, float* out_val, int32_t* out_count, void* ws,
                size_t ws_bytes, void* stream) {
    int rc = merge_args_ok(P, k_in, k, n);
    if (rc != TOPK_EF_OK) return rc;
    if (k_in > 0 && (!in_idx || !in_val || bad_fp32_ptr(in_idx) || bad_fp32_ptr(in_val)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (k > 0 && (!out_idx || !out_val || bad_fp32_ptr(out_idx) || bad_fp32_ptr(out_val)))
        return TOPK_EF_ERR_INVALID_ARG;
    if (!out_count || !ws || ((uintptr_t)ws % ALIGN) != 0 || bad_fp32_ptr(out_count))
        return TOPK_EF_ERR_INVALID_ARG;
    const MLayout L = merge_layout(P, k_in, k);
    if (ws_bytes < L.total) return TOPK_EF_ERR_WORKSPACE;
    DevFacts f;
    if ((rc = device_facts(&f)) != TOPK_EF_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* w = (char*)ws;
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(w + L.ctrl);
    uint32_t* sizes = reinterpret_cast<uint32_t*>(w + L.sizes);
    uint32_t* floors = reinterpret_cast<uint32_t*>(w + L.floors);
    uint32_t* bad = reinterpret_cast<uint32_t*>(w + L.bad);
    uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.hist);
    uint32_t* live = reinterpret_cast<uint32_t*>(w + L.live);
    uint32_t* set_idx = reinterpret_cast<uint32_t*>(w + L.set_idx);
    float* set_val = reinterpret_cast<float*>(w + L.set_val);
    uint32_t* m_idx = reinterpret_cast<uint32_t*>(w + L.m_idx);
    float* m_val = reinterpret_cast<float*>(w + L.m_val);
    const bool single = (P == 1 || k_in == 0);
    // one cluster kernel per round when a cluster size holds every round
    bool cluster_path = !single;
    for (int r = 0; r < L.rounds; ++r)
        cluster_path = cluster_path && L.mcap[r] <= MC_PAIR_MAX;
    McFit fit;
    if (cluster_path && (rc = merge_cluster_fit(&fit)) != TOPK_EF_OK) return rc;
    const int forced_cl = ((g_test_flags.load() >> 3) & 7) - 1;
    std::vector<int> cls(L.rounds, 0);
    for (int r = 0; cluster_path && r < L.rounds; ++r) {
        cls[r] = round_cluster(fit, L.np[r], L.mcap[r], forced_cl);
        cluster_path = cls[r] != 0;
    }
    const uint32_t kernels =
        single ? 2u : (uint32_t)(cluster_path ? 1 + L.rounds : 1 + 2 * L.rounds);

    MergeSetupParams sp;
    memset(&sp, 0, sizeof(sp));
    sp.in_idx = in_idx;
    sp.in_val = in_val;
    sp.P = P;
    sp.k_in = k_in;
    sp.n = n;
    sp.ctrl = ctrl;
    sp.kernels = kernels;
    sp.zero_ptr = reinterpret_cast<uint4*>(w + L.zero_begin);
    // the per-pair histograms and live counts serve only the merge + select
    // kernels; the cluster kernel keeps its histograms in shared memory
    sp.zero_vec4 = cluster_path ? 0 : (L.zero_end - L.zero_begin) / 16;
    sp.bad_words = bad;
    sp.sizes = sizes;
    sp.floors = floors;
    sp.set_idx = set_idx;
    sp.set_val = set_val;
    sp.set_cap = L.cap;
    sp.lonely = (!single && (P % 2 == 1)) ? P - 1 : -1;
    sp.validate_blocks = L.vblocks;
    const int nz = (int)std::max<uint64_t>(
        1, std::min<uint64_t>(148, (sp.zero_vec4 + MZ_THREADS * 8 - 1) / (MZ_THREADS * 8)));
    trace_before(st, "merge_setup_kernel");
    cudaError_t e = launch_pdl(merge_setup_kernel, (int)(L.vblocks + nz), MZ_THREADS, st, sp);
    trace_after(st);
    if (e != cudaSuccess) return cuda_fail(e);

    const int G = std::min(SLOT_MAX, f.sms * f.selm_blocks);
    SelCommon cm;
    cm.ctrl = ctrl;
    cm.slots = reinterpret_cast<Slot*>(w + L.slots);

    MergeSrc ms;
    memset(&ms, 0, sizeof(ms));
    ms.kmax = (uint32_t)std::min<int64_t>(k, 0xFFFFFFFFLL);
    ms.out_idx = out_idx;
    ms.out_val = out_val;
    ms.out_count = out_count;
    ms.out_k = k;
    ms.set_idx = set_idx;
    ms.set_val = set_val;
    ms.set_cap = L.cap;
    ms.sizes = sizes;
    ms.bad_words = bad;
    ms.n_bad = (int32_t)L.vblocks;

    if (single) {
        ms.m_idx = reinterpret_cast<const uint32_t*>(in_idx);
        ms.m_val = in_val;
        ms.mcap = k_in;
        ms.T = 1;
        ms.live = nullptr;
        ms.live_const = (uint32_t)k_in;
        ms.hist = hist;
        ms.d1_done = 0;
        ms.final_out = 1;
        ms.pair_stride = 1;
        cm.bar = &ctrl->merge_bar[0];
        void* args[] = {&ms, &cm};
        const int G1 = (int)std::max<int64_t>(1, std::min<int64_t>(G, ceil_div64(k_in, 4096)));
        trace_before(st, "select_kernel<MergeSrc>");
        e = cudaLaunchCooperativeKernel((const void*)select_kernel<MergeSrc>, dim3(G1),
                                        dim3(SEL_THREADS), args, 0, st);
        trace_after(st);
        if (e != cudaSuccess) return cuda_fail(e);
        return TOPK_EF_OK;
    }

    if (cluster_path) {
        for (int r = 0; r < L.rounds; ++r) {
            MergeClusterParams cp;
            memset(&cp, 0, sizeof(cp));
            cp.src_idx = r == 0 ? reinterpret_cast<const uint32_t*>(in_idx) : set_idx;
            cp.src_val = r == 0 ? in_val : set_val;
            cp.src_stride = r == 0 ? k_in : L.cap;
            cp.sizes_in = r == 0 ? nullptr : sizes;
            cp.size_const = (uint32_t)k_in;
            cp.step = 1 << r;
            cp.kmax = ms.kmax;
            cp.dst_idx = set_idx;
            cp.dst_val = set_val;
            cp.dst_stride = L.cap;
            cp.sizes_out = sizes;
            // after round 0 every set's lower key bound is known: the
            // round's digit 1 can be relative to it
            cp.floor_in = r == 0 ? nullptr : floors;
            cp.floor_out = floors;
            cp.final_out = (r == L.rounds - 1) ? 1 : 0;
            cp.out_idx = out_idx;
            cp.out_val = out_val;
            cp.out_count = out_count;
            cp.out_k = k;
            cp.bad_words = r == 0 ? bad : nullptr;
            cp.n_bad = r == 0 ? (int32_t)L.vblocks : 0;
            cp.ctrl = ctrl;
            trace_before(st, "merge_cluster_kernel");
            e = launch_merge_cluster(cls[r], L.np[r], st, cp);
            trace_after(st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return TOPK_EF_OK;
    }

    for (int r = 0; r < L.rounds; ++r) {
        MergeRoundParams mp;
        mp.src_idx = r == 0 ? reinterpret_cast<const uint32_t*>(in_idx) : set_idx;
        mp.src_val = r == 0 ? in_val : set_val;
        mp.src_stride = r == 0 ? k_in : L.cap;
        mp.sizes = r == 0 ? nullptr : sizes;
        mp.size_const = (uint32_t)k_in;
        mp.np = L.np[r];
        mp.step = 1 << r;
        mp.mcap = L.mcap[r];
        mp.m_idx = m_idx;
        mp.m_val = m_val;
        mp.hist = hist + (size_t)L.pbase[r] * MHIST_WORDS;
        mp.live = live + L.pbase[r];
        dim3 grid((unsigned)ceil_div64(L.mcap[r], MG_D), (unsigned)L.np[r]);
        trace_before(st, "merge_round_kernel");
        merge_round_kernel<<<grid, MG_THREADS, 0, st>>>(mp);
        trace_after(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);

        ms.m_idx = m_idx;
        ms.m_val = m_val;
        ms.mcap = L.mcap[r];
        ms.T = L.np[r];
        ms.live = mp.live;
        ms.hist = mp.hist;
        ms.d1_done = 1;
        ms.final_out = (r == L.rounds - 1) ? 1 : 0;
        ms.pair_stride = 2 << r;
        if (r > 0) {
            ms.bad_words = nullptr;
            ms.n_bad = 0;
        }
        cm.bar = &ctrl->merge_bar[r];
        void* args[] = {&ms, &cm};
        // about 4,096 merged positions per block: small rounds use few blocks
        const int Gr = (int)std::max<int64_t>(
            1, std::min<int64_t>(G, ceil_div64((int64_t)L.np[r] * L.mcap[r], 4096)));
        trace_before(st, "select_kernel<MergeSrc>");
        e = cudaLaunchCooperativeKernel((const void*)select_kernel<MergeSrc>, dim3(Gr),
                                        dim3(SEL_THREADS), args, 0, st);
        trace_after(st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return TOPK_EF_OK;
}

int topk_ef_last_device_status(const void* ws, void* stream) {
    if (!ws) return TOPK_EF_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Ctrl c;
    cudaError_t e = cudaMemcpyAsync(&c, ws, sizeof(c), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    // small_kernel records its errors with the call's tag (nothing clears the
    // word before a call); every other path clears the control block first
    const uint32_t s = c.path_small == SK_PATH_TAG
                           ? ((uint32_t)(c.sk_status >> 32) == c.sk_tag ? (uint32_t)c.sk_status : 0u)
                           : c.status;
    if (s & ST_TIMEOUT) return TOPK_EF_ERR_DEVICE_TIMEOUT;
    if (s & ST_BAD_INPUT) return TOPK_EF_ERR_BAD_INPUT;
    if (s & ST_INCONSISTENT) return TOPK_EF_ERR_INTERNAL;
    return TOPK_EF_OK;
}

int topk_ef_path_info(const void* ws, void* stream, int64_t* info) {
    if (!ws || !info) return TOPK_EF_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Ctrl c;
    cudaError_t e = cudaMemcpyAsync(&c, ws, sizeof(c), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    info[0] = c.mode;
    info[1] = (int64_t)c.cand_total;
    info[2] = (int64_t)c.cap;
    info[3] = c.kernels;
    info[4] = c.r2_path ? 1 : 0;
    info[5] = 0;
    return TOPK_EF_OK;
}

int topk_ef_phase_times(const void* ws, void* stream, int64_t* ns) {
    if (!ws || !ns) return TOPK_EF_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Ctrl c;
    SegMeta m0;
    cudaError_t e = cudaMemcpyAsync(&c, ws, sizeof(c), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&m0, static_cast<const char*>(ws) + align_up(sizeof(Ctrl)), sizeof(m0),
                            cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    for (int i = 0; i < 8; ++i)
        ns[i] = c.t_phase[i] ? (int64_t)(c.t_phase[i] - c.t_phase[0]) : -1;
    for (int i = 0; i < 3; ++i) ns[8 + i] = m0.t_ns[2] ? (int64_t)m0.t_ns[i] : -1;
    // spans over all blocks, from the first streaming block past its wait
    const uint64_t s0 = c.t_span[SPAN_STREAM_FIRST] ? ~c.t_span[SPAN_STREAM_FIRST] : 0;
    const uint64_t sel0 = c.t_span[SPAN_SELECT_FIRST] ? ~c.t_span[SPAN_SELECT_FIRST] : 0;
    auto rel = [&](uint64_t t) { return (s0 && t) ? (int64_t)(t - s0) : (int64_t)-1; };
    ns[11] = rel(c.t_span[SPAN_STREAM_LAST]);
    ns[12] = rel(sel0);
    ns[13] = rel(c.t_phase[0]);
    ns[14] = rel(c.t_span[SPAN_SELECT_LAST]);
    ns[15] = rel(c.t_span[SPAN_START_LAST]);
    ns[16] = rel(c.t_span[SPAN_OFFSET_LAST]);
    ns[17] = rel(c.t_span[SPAN_GATHER_LAST]);
    ns[18] = rel(c.t_span[SPAN_BAR2_LAST]);
    ns[19] = -1;
    return TOPK_EF_OK;
}

int topk_ef_last_cuda_error(void) { return t_last_cuda_error; }

const char* topk_ef_status_string(int status) {
    switch (status) {
        case TOPK_EF_OK: return "ok";
        case TOPK_EF_ERR_INVALID_ARG: return "invalid argument";
        case TOPK_EF_ERR_WORKSPACE: return "workspace too small";
        case TOPK_EF_ERR_CUDA: return "CUDA error";
        case TOPK_EF_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case TOPK_EF_ERR_BAD_INPUT: return "malformed merge input";
        case TOPK_EF_ERR_INTERNAL: return "internal count mismatch";
        default: return "unknown status";
    }
}

int topk_ef_set_test_flags(int flags) { return g_test_flags.exchange(flags); }

int topk_ef_trace_enable(int on) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    int dev = 0;
    cudaError_t e;
    if (on) {
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e);
        if (g_trace.dev != dev) {
            if (g_trace.dev >= 0) {
                int cur = dev;
                cudaSetDevice(g_trace.dev);
                for (auto& ev : g_trace.ev) cudaEventDestroy(ev);
                cudaSetDevice(cur);
            }
            for (auto& ev : g_trace.ev)
                if ((e = cudaEventCreate(&ev)) != cudaSuccess) return cuda_fail(e);
            g_trace.dev = dev;
        }
    }
    g_trace.on = on ? 1 : 0;
    g_trace.n = 0;
    g_trace.open = false;
    g_trace.seen = 0;
    return TOPK_EF_OK;
}

int topk_ef_trace_only(const char* kernel_name, int every) {
    if (every < 1) return TOPK_EF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    g_trace.only = kernel_name ? kernel_name : "";
    g_trace.every = every;
    return TOPK_EF_OK;
}

int topk_ef_trace_read(float* ms, const char** names, int max_entries, int* count) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (!count || (max_entries > 0 && (!ms || !names))) return TOPK_EF_ERR_INVALID_ARG;
    const int n = std::min(g_trace.n, std::max(0, max_entries));
    *count = n;
    for (int i = 0; i < n; ++i) {
        cudaError_t e = cudaEventSynchronize(g_trace.ev[2 * i + 1]);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms[i], g_trace.ev[2 * i], g_trace.ev[2 * i + 1]);
        if (e != cudaSuccess) return cuda_fail(e);
        names[i] = g_trace.name[i];
    }
    g_trace.n = 0;
    return TOPK_EF_OK;
}

}  // extern "C"
