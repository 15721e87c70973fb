// race_attn.cu -- C ABI of the RACE Attention library: argument checks, work planning and
// kernel launches on the caller's stream.  Declarations and argument contracts are in
// include/race_attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <string>
#include <vector>

#include "race_attn.h"
#include "race_decode.cuh"
#include "race_generic.cuh"
#include "race_tc.cuh"
#include "race_tc_wide.cuh"

namespace {

// ---- opt-in kernel timing -------------------------------------------------------------
struct ProfEntry {
    std::string name;
    double ms;
    int64_t launches;
};
struct ProfPending {
    int entry;
    cudaEvent_t a, b;
};
bool g_prof_on = false;
bool g_tc_forward = true;   // tensor-core forward for the shapes it covers
bool g_tc_backward = true;  // tensor-core backward for the shapes it covers
std::vector<ProfEntry> g_prof;
std::vector<ProfPending> g_pending;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t prof_event()
{
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

int prof_entry(const char *name)
{
    for (size_t i = 0; i < g_prof.size(); ++i)
        if (g_prof[i].name == name) return (int)i;
    g_prof.push_back({name, 0.0, 0});
    return (int)g_prof.size() - 1;
}

// Run `fn` (which launches one kernel on st) between two recorded events when enabled.
template <typename Fn>
cudaError_t timed(const char *name, cudaStream_t st, Fn fn)
{
    if (!g_prof_on) return fn();
    ProfPending p{prof_entry(name), prof_event(), prof_event()};
    if (p.a) cudaEventRecord(p.a, st);
    cudaError_t e = fn();
    if (p.b) cudaEventRecord(p.b, st);
    if (p.a && p.b)
        g_pending.push_back(p);
    g_prof[p.entry].launches += 1;
    return e;
}

using race::generic::Args;
namespace gk = race::generic;

constexpr int64_t kSegAlign = 128;     // segment lengths are multiples of this many tokens
// so that only the last chunk of a head is ragged, where the TMA boxes read zeros past N
static_assert(kSegAlign % race::tc::T == 0, "segments hold whole chunks");
constexpr int64_t kMinSegTokens = 128;  // no segment shorter than this (unless N is)

struct Plan {
    int BH;
    int64_t N;
    int d, L, P, R, M, D, G;
    int64_t seg_len;
    int nseg;
    size_t state_elems;  // one [BH][nseg][M][D] fp32 state buffer
};

int device_sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // no device here: plan for a full B200
        return 148;
    }
    return n;
}

race_status_t check_sizes(int B, int H, int64_t N, int d, int L, int P)
{
    if (B < 1 || H < 1 || N < 0 || d < 1 || L < 1 || P < 1) return RACE_ERR_INVALID_ARG;
    if ((int64_t)B * H > 65535) return RACE_ERR_UNSUPPORTED;
    if (d % 8 != 0 || d > 128) return RACE_ERR_UNSUPPORTED;
    if (P > 5) return RACE_ERR_UNSUPPORTED;
    if ((int64_t)L << P > (int64_t)gk::MG * gk::MAXG) return RACE_ERR_UNSUPPORTED;
    return RACE_OK;
}

Plan make_plan(int B, int H, int64_t N, int d, int L, int P)
{
    Plan p;
    p.BH = B * H;
    p.N = N;
    p.d = d;
    p.L = L;
    p.P = P;
    p.R = 1 << P;
    p.M = L * p.R;
    p.D = d + 1;
    p.G = (p.M + gk::MG - 1) / gk::MG;
    // Segments per sequence.  One CTA walks one segment and holds its SM, so a pass takes
    // ceil(nseg * BH / SMs) waves, each as long as a segment's chunks plus a fixed cost per
    // CTA (TMEM, W and the start state: about two chunks).  The count that minimises this
    // is taken, with no segment shorter than kMinSegTokens (unless N is) and lengths a
    // multiple of kSegAlign; ties go to fewer segments (less scan work).
    const int64_t sms = device_sm_count();
    auto seg_len_for = [&](int64_t n) {
        int64_t len = (N + n - 1) / n;
        len = (len + kSegAlign - 1) / kSegAlign * kSegAlign;
        return len < kSegAlign ? kSegAlign : len;
    };
    int64_t maxseg = (N + kMinSegTokens - 1) / kMinSegTokens;
    if (maxseg > 4 * sms) maxseg = 4 * sms;
    int64_t best_len = seg_len_for(1), best_cost = -1;
    for (int64_t n = 1; n <= maxseg; ++n) {
        const int64_t len = seg_len_for(n), segs = (N + len - 1) / len;
        const int64_t waves = (segs * p.BH + sms - 1) / sms;
        const int64_t cost = waves * (len / kSegAlign + 2);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_len = len;
        }
    }
    p.seg_len = best_len;
    p.nseg = (int)((N + best_len - 1) / best_len);
    if (p.nseg < 1) p.nseg = 1;
    p.state_elems = (size_t)p.BH * p.nseg * p.M * p.D;
    return p;
}

bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }
// The tensor-core paths move rows in 32-byte accesses: they run only when every buffer they
// touch is 32-byte aligned (as every cudaMalloc or torch allocation is); otherwise the
// general path runs.
bool aligned32(std::initializer_list<const void *> ptrs)
{
    for (const void *p : ptrs)
        if (p && ((uintptr_t)p & 31u) != 0) return false;
    return true;
}

// Backward workspace: key- and query-side segment states, then the W image of the tensor-core
// path (16 KB), then c_i per token (fp32 [BH][N]).
constexpr size_t kWImageBytes = 16384;
size_t backward_workspace_bytes(const Plan &p)
{
    const size_t cbytes = ((size_t)p.BH * (size_t)p.N * sizeof(float) + 15) / 16 * 16;
    return 2 * p.state_elems * sizeof(float) + kWImageBytes + cbytes;
}

// ---- tensor maps of the TMA loads ---------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled()
{
    static const EncodeTiled fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (EncodeTiled) nullptr;
        }
        return (EncodeTiled)f;
    }();
    return fn;
}

// A [BH][N][64] bf16 tensor as a 3-D map (columns, rows, heads); boxes of 128 rows by
// box_cols columns: 64 with the 128-byte swizzle (a K128 tile) or 16 with the 32-byte swizzle
// (one value-tile atom).  Rows past N read as zero.
cudaError_t bf16_map(CUtensorMap *m, const void *ptr, const Plan &p, bool value_atom)
{
    const EncodeTiled fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    CUresult r;
    if (value_atom) {  // (16 columns, rows, 4 atoms, heads): one box fills a whole value tile
        const cuuint64_t dims[4] = {16, (cuuint64_t)p.N, 4, (cuuint64_t)p.BH};
        const cuuint64_t strides[3] = {128, 32, (cuuint64_t)p.N * 128};
        const cuuint32_t box[4] = {16, (cuuint32_t)race::tc::T, 4, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const cuuint64_t dims[3] = {64, (cuuint64_t)p.N, (cuuint64_t)p.BH};
        const cuuint64_t strides[2] = {128, (cuuint64_t)p.N * 128};
        const cuuint32_t box[3] = {64, (cuuint32_t)race::tc::T, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

Args base_args(const Plan &p, const float *W, float tau)
{
    Args a;
    std::memset(&a, 0, sizeof(a));
    a.W = W;
    a.N = p.N;
    a.d = p.d;
    a.L = p.L;
    a.P = p.P;
    a.M = p.M;
    a.G = p.G;
    a.hard = tau == 0.f;
    a.beta = a.hard ? 0.f : 1.f / tau;
    a.seg_len = p.seg_len;
    a.nseg = p.nseg;
    return a;
}

template <typename Kern>
cudaError_t launch(Kern kernel, dim3 grid, int cluster_x, size_t smem, cudaStream_t st,
                   const Args &a, int cluster_y = 1)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = dim3(gk::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = cluster_y;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_scan(float *buf, const Plan &p, int mode, cudaStream_t st, const float *init = nullptr,
                        float *total_out = nullptr)
{
    const int64_t MD = (int64_t)p.M * p.D;
    dim3 grid((unsigned)((MD + gk::NT - 1) / gk::NT), (unsigned)p.BH);
    return timed("segment_scan", st, [&] {
        gk::race_scan<<<grid, gk::NT, 0, st>>>(buf, p.nseg, MD, mode, init, total_out);
        return cudaGetLastError();
    });
}

// A pass split in two for a sequence sharded over several devices: BEGIN stops once the
// local statistics the other shards need are known (h_total: key side, forward; g_total:
// query side, backward), END continues from the other shards' statistics (h_init: the keys
// before this shard -- every other shard's when bidirectional -- and g_init: the queries
// after it).  ALL runs both halves with no other shards.
enum Stage { STAGE_ALL = 0, STAGE_BEGIN = 1, STAGE_END = 2 };
struct Shard {
    int stage = STAGE_ALL;
    const float *h_init = nullptr;
    float *h_total = nullptr;
    const float *g_init = nullptr;
    float *g_total = nullptr;
    void *dpq = nullptr, *dpk = nullptr;  // backward: dLoss/dp / |x| per row, for dW (optional)
};

// ---- the general path (every shape and dtype) ----------------------------------------

// Segment totals on the general path.  When the segments leave most SMs idle (short
// sequences), the chunks of each segment are split over a cluster of up to 8 CTAs along y
// (one CTA per SM); the partial sums are added in rank order, so the result does not depend
// on the timing.
template <typename Kern>
cudaError_t launch_agg(Kern kernel, const Plan &p, size_t smem, cudaStream_t st, Args a, int T)
{
    const int64_t chunks = (p.seg_len + T - 1) / T;
    const int64_t ctas = (int64_t)p.G * p.nseg * p.BH;
    int64_t split = std::min<int64_t>({8, chunks, device_sm_count() / std::max<int64_t>(1, ctas)});
    if (split < 2) split = 1;
    a.agg_split = (int)split;
    const dim3 grid((unsigned)p.G, (unsigned)(p.nseg * split), (unsigned)p.BH);
    return launch(kernel, grid, 1, smem, st, a, (int)split);
}

template <typename DT, int T>
cudaError_t generic_forward(const Plan &p, Args a, float *states, int causal, cudaStream_t st, const Shard &sh)
{
    const size_t smem = gk::Smem(T, p.d, p.P).total * sizeof(float);
    const dim3 grid((unsigned)p.G, (unsigned)p.nseg, (unsigned)p.BH);
    a.causal = causal;
    a.agg_out = states;
    cudaError_t e;
    if (sh.stage != STAGE_END) {
        e = timed("generic_agg_kv", st, [&] {
            return launch_agg(gk::race_agg<DT, T, gk::AGG_KV>, p, smem, st, a, T);
        });
        if (e != cudaSuccess) return e;
        if (sh.h_total && (e = launch_scan(states, p, gk::SCAN_TOTAL_ONLY, st, nullptr, sh.h_total)) != cudaSuccess)
            return e;
        if (sh.stage == STAGE_BEGIN) return cudaSuccess;
    }
    e = launch_scan(states, p, causal ? gk::SCAN_EXCL_PREFIX : gk::SCAN_TOTAL, st, sh.h_init);
    if (e != cudaSuccess) return e;
    a.state = states;
    a.state_seg_stride = causal ? (int64_t)p.M * p.D : 0;
    dim3 wgrid = grid;
    if (!causal) {  // the read-out needs no segments: split the rows over as many CTAs as fill the
                    // GPU once (one CTA per SM), whole T-token chunks each
        const int64_t chunks = (p.N + T - 1) / T;
        int64_t n = std::max<int64_t>(1, device_sm_count() / ((int64_t)p.G * p.BH));
        n = std::min(n, chunks);
        if (n > p.nseg) {
            a.ro_seg_len = (chunks + n - 1) / n * T;
            wgrid.y = (unsigned)((p.N + a.ro_seg_len - 1) / a.ro_seg_len);
        }
    }
    return timed("generic_fwd_walk", st,
                 [&] { return launch(gk::race_fwd_walk<DT, T>, wgrid, p.G, smem, st, a); });
}

template <typename DT, int T>
cudaError_t generic_backward(const Plan &p, Args a, const float *hstates, bool have_ctx,
                             float *hbuf, float *gbuf, int causal, cudaStream_t st, const Shard &sh)
{
    const size_t smem = gk::Smem(T, p.d, p.P).total * sizeof(float);
    const dim3 grid((unsigned)p.G, (unsigned)p.nseg, (unsigned)p.BH);
    const int64_t stride = causal ? (int64_t)p.M * p.D : 0;
    a.causal = causal;
    a.dpq = (float *)sh.dpq;
    a.dpk = (float *)sh.dpk;
    cudaError_t e;
    if (sh.stage != STAGE_END) {
        if (!have_ctx) {  // key-side prefix statistics, as the forward computes them
            a.agg_out = hbuf;
            e = timed("generic_agg_kv", st, [&] {
                return launch_agg(gk::race_agg<DT, T, gk::AGG_KV>, p, smem, st, a, T);
            });
            if (e != cudaSuccess) return e;
            e = launch_scan(hbuf, p, causal ? gk::SCAN_EXCL_PREFIX : gk::SCAN_TOTAL, st, sh.h_init);
            if (e != cudaSuccess) return e;
            hstates = hbuf;
        }
        a.state = hstates;
        a.state_seg_stride = stride;
        e = timed("generic_bwd_q_walk", st,
                  [&] { return launch(gk::race_bwd_q_walk<DT, T>, grid, p.G, smem, st, a); });
        if (e != cudaSuccess) return e;
        a.agg_out = gbuf;
        e = timed("generic_agg_qdy", st, [&] {
            return launch_agg(gk::race_agg<DT, T, gk::AGG_QDY>, p, smem, st, a, T);
        });
        if (e != cudaSuccess) return e;
        if (sh.g_total && (e = launch_scan(gbuf, p, gk::SCAN_TOTAL_ONLY, st, nullptr, sh.g_total)) != cudaSuccess)
            return e;
        if (sh.stage == STAGE_BEGIN) return cudaSuccess;
    }
    e = launch_scan(gbuf, p, causal ? gk::SCAN_EXCL_SUFFIX : gk::SCAN_TOTAL, st, sh.g_init);
    if (e != cudaSuccess) return e;
    a.state = gbuf;
    a.state_seg_stride = stride;
    return timed("generic_bwd_kv_walk", st,
                 [&] { return launch(gk::race_bwd_kv_walk<DT, T>, grid, p.G, smem, st, a); });
}

// ---- the tensor-core path (bf16, d = 64, L = 16, P = 4) --------------------------------

template <typename Kern>
cudaError_t tc_prepare(Kern kernel, size_t smem)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

// Segment totals of the key side: mode 0 = sum phi(k) [v, 1]^T, mode 1 = sum phi(q) dY^T.
cudaError_t tc_segment_totals(const Plan &p, race::tc::BwdArgs a, int mode, float *out, cudaStream_t st)
{
    namespace tc = race::tc;
    const dim3 grid((unsigned)p.nseg, (unsigned)p.BH);
    const size_t sm = tc::smem_bytes(tc::agg_smem::TOTAL);
    a.agg_out = out;
    cudaError_t e;
    if (mode == 0) {
        if ((e = tc_prepare(tc::tc_agg<0>, sm)) != cudaSuccess) return e;
        return timed("tc_agg_kv", st, [&] {
            tc::tc_agg<0><<<grid, tc::NTH, sm, st>>>(a);
            return cudaGetLastError();
        });
    }
    if ((e = tc_prepare(tc::tc_agg<1>, sm)) != cudaSuccess) return e;
    return timed("tc_agg_qdy", st, [&] {
        tc::tc_agg<1><<<grid, tc::NTH, sm, st>>>(a);
        return cudaGetLastError();
    });
}

cudaError_t tc_args(race::tc::BwdArgs &a, const Plan &p, const void *q, const void *k, const void *v,
                    const float *W, const void *out, const float *den, const void *dout, float tau, int causal)
{
    std::memset(&a, 0, sizeof(a));
    cudaError_t e;
    if ((e = bf16_map(&a.tm_q, q, p, false)) != cudaSuccess || (e = bf16_map(&a.tm_k, k, p, false)) != cudaSuccess ||
        (e = bf16_map(&a.tm_v_va, v, p, true)) != cudaSuccess)
        return e;
    if (out && (e = bf16_map(&a.tm_o, out, p, false)) != cudaSuccess) return e;
    if (dout && (e = bf16_map(&a.tm_do_va, dout, p, true)) != cudaSuccess) return e;
    a.q = (const __nv_bfloat16 *)q;
    a.k = (const __nv_bfloat16 *)k;
    a.v = (const __nv_bfloat16 *)v;
    a.o = (const __nv_bfloat16 *)out;
    a.dout = (const __nv_bfloat16 *)dout;
    a.den = den;
    a.W = W;
    a.N = p.N;
    a.seg_len = p.seg_len;
    a.nseg = p.nseg;
    a.beta = 1.f / tau;
    a.causal = causal;
    return cudaSuccess;
}

cudaError_t tc_forward(const Plan &p, const void *q, const void *k, const void *v, const float *W,
                       void *out, float *den, float *states, float tau, int causal, cudaStream_t st, const Shard &sh)
{
    namespace tc = race::tc;
    tc::BwdArgs ka;
    cudaError_t e = tc_args(ka, p, q, k, v, W, nullptr, nullptr, nullptr, tau, causal);
    if (e != cudaSuccess) return e;
    if (sh.stage != STAGE_END) {
        e = tc_segment_totals(p, ka, 0, states, st);
        if (e != cudaSuccess) return e;
        if (sh.h_total && (e = launch_scan(states, p, gk::SCAN_TOTAL_ONLY, st, nullptr, sh.h_total)) != cudaSuccess)
            return e;
        if (sh.stage == STAGE_BEGIN) return cudaSuccess;
    }
    e = launch_scan(states, p, causal ? gk::SCAN_EXCL_PREFIX : gk::SCAN_TOTAL, st, sh.h_init);
    if (e != cudaSuccess) return e;
    tc::Args a;
    std::memset(&a, 0, sizeof(a));
    a.tm_q = ka.tm_q;
    a.tm_k = ka.tm_k;
    a.tm_v_va = ka.tm_v_va;
    a.q = (const __nv_bfloat16 *)q;
    a.k = (const __nv_bfloat16 *)k;
    a.v = (const __nv_bfloat16 *)v;
    a.W = W;
    a.out = (__nv_bfloat16 *)out;
    a.den = den;
    a.N = p.N;
    a.seg_len = p.seg_len;
    a.nseg = p.nseg;
    a.beta = 1.f / tau;
    a.causal = causal;
    a.state = states;
    a.state_seg_stride = causal ? (int64_t)p.M * p.D : 0;
    const dim3 grid((unsigned)p.nseg, (unsigned)p.BH);
    if (!causal) {  // every chunk reads the total state: two chunks in flight per CTA
        const size_t sm_ro = tc::smem_bytes(tc::ro_smem::TOTAL);
        if ((e = tc_prepare(tc::tc_readout, sm_ro)) != cudaSuccess) return e;
        return timed("tc_readout", st, [&] {
            tc::tc_readout<<<grid, tc::NTH, sm_ro, st>>>(a);
            return cudaGetLastError();
        });
    }
    const size_t sm_walk = tc::smem_bytes(tc::fwd_smem::TOTAL);
    if ((e = tc_prepare(tc::tc_fwd_walk, sm_walk)) != cudaSuccess) return e;
    return timed("tc_fwd_walk", st, [&] {
        tc::tc_fwd_walk<<<grid, tc::NTH + 32, sm_walk, st>>>(a);
        return cudaGetLastError();
    });
}

cudaError_t tc_backward(const Plan &p, const void *q, const void *k, const void *v, const float *W,
                        const void *out, const float *den, const void *dout, const float *ctx, float *hbuf,
                        float *gbuf, uint8_t *wimg, float *cbuf, void *dq, void *dk, void *dv, float tau,
                        int causal, cudaStream_t st, const Shard &sh)
{
    namespace tc = race::tc;
    const dim3 grid((unsigned)p.nseg, (unsigned)p.BH);
    tc::BwdArgs a;
    cudaError_t e = tc_args(a, p, q, k, v, W, out, den, dout, tau, causal);
    if (e != cudaSuccess) return e;
    a.dq = (__nv_bfloat16 *)dq;
    a.dk = (__nv_bfloat16 *)dk;
    a.dv = (__nv_bfloat16 *)dv;
    a.wimg = wimg;
    a.cbuf = cbuf;
    a.dpq = (__nv_bfloat16 *)sh.dpq;
    a.dpk = (__nv_bfloat16 *)sh.dpk;
    e = timed("tc_w_image", st, [&] {
        tc::tc_w_image<<<1, tc::NTH, 0, st>>>(W, wimg);
        return cudaGetLastError();
    });
    if (e != cudaSuccess) return e;
    const int64_t stride = causal ? (int64_t)p.M * p.D : 0;
    const size_t sm_q = tc::smem_bytes(tc::bq_smem::TOTAL);
    const size_t sm_kv = tc::smem_bytes(tc::bkv_smem::TOTAL);
    if ((e = tc_prepare(tc::tc_bwd_q_walk, sm_q)) != cudaSuccess ||
        (e = tc_prepare(tc::tc_bwd_kv_walk, sm_kv)) != cudaSuccess)
        return e;
    if (sh.stage != STAGE_END) {
        const float *hstates = ctx;
        if (!hstates) {  // key-side prefix statistics, as the forward computes them
            if ((e = tc_segment_totals(p, a, 0, hbuf, st)) != cudaSuccess) return e;
            if ((e = launch_scan(hbuf, p, causal ? gk::SCAN_EXCL_PREFIX : gk::SCAN_TOTAL, st, sh.h_init)) !=
                cudaSuccess)
                return e;
            hstates = hbuf;
        }
        a.state = hstates;
        a.state_seg_stride = stride;
        e = timed("tc_bwd_q_walk", st, [&] {
            tc::tc_bwd_q_walk<<<grid, tc::NTH, sm_q, st>>>(a);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
        if ((e = tc_segment_totals(p, a, 1, gbuf, st)) != cudaSuccess) return e;
        if (sh.g_total && (e = launch_scan(gbuf, p, gk::SCAN_TOTAL_ONLY, st, nullptr, sh.g_total)) != cudaSuccess)
            return e;
        if (sh.stage == STAGE_BEGIN) return cudaSuccess;
    }
    if ((e = launch_scan(gbuf, p, causal ? gk::SCAN_EXCL_SUFFIX : gk::SCAN_TOTAL, st, sh.g_init)) != cudaSuccess)
        return e;
    a.state = gbuf;
    a.state_seg_stride = stride;
    return timed("tc_bwd_kv_walk", st, [&] {
        tc::tc_bwd_kv_walk<<<grid, tc::NTH, sm_kv, st>>>(a);
        return cudaGetLastError();
    });
}

// ---- the tensor-core path for d = 128, P = 5 (feature groups x value halves) -------------
namespace wd = race::tc::wide;

bool wide_ok(race_dtype_t dtype, int d, int L, int P, float tau, int causal, int64_t N)
{
    return dtype == RACE_BF16 && d == wd::WD && P == wd::WP && L % 8 == 0 && L >= 8 && L <= 32 && tau > 0.f &&
           causal && N < ((int64_t)1 << 31);
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// One head at a time: the segment plan is that of a single head, and the per-head arrays
// (projections, dLoss/dp^, fp32 sums over the groups) are reused for every head.
struct WidePlan {
    Plan p;
    int G, npw, npwp, ntile;
    size_t state_bytes;  // one head's segment states [2G][nseg][256][65] fp32
    size_t p_bytes;      // one side's projections [N][npwp] fp32
    size_t acc_bytes;    // [N][128] fp32 sums over the groups
    size_t dacc_bytes;   // [N] fp32
};

WidePlan wide_plan(int64_t N, int d, int L, int P)
{
    WidePlan w;
    w.p = make_plan(1, 1, N, d, L, P);
    w.G = L / 8;
    w.npw = L * P;
    w.npwp = (w.npw + 15) / 16 * 16;
    w.ntile = (int)((N + race::tc::T - 1) / race::tc::T);
    w.state_bytes = align256((size_t)2 * w.G * w.p.nseg * race::tc::MF * race::tc::DS * sizeof(float));
    w.p_bytes = align256((size_t)N * w.npwp * sizeof(float));
    w.acc_bytes = align256((size_t)N * wd::WD * sizeof(float));
    w.dacc_bytes = align256((size_t)N * sizeof(float));
    return w;
}

size_t wide_forward_bytes(const WidePlan &w) { return w.state_bytes + 2 * w.p_bytes + w.acc_bytes + w.dacc_bytes; }

// Context of the shapes this path can take (d = 128, P = 5, L a multiple of 8 up to 32,
// causal): room for either path's states, then a tag (kCtxTag when this path's forward left
// its scanned key-side states [BH][2G][nseg][256][65] there, 0 otherwise).
bool wide_shape(int d, int L, int P, int causal)
{
    return d == wd::WD && P == wd::WP && L % 8 == 0 && L >= 8 && L <= 32 && causal;
}
size_t wide_ctx_tag_offset(const Plan &p, const WidePlan &w)
{
    return align256(std::max(p.state_elems * sizeof(float), (size_t)p.BH * w.state_bytes));
}
// states of both sides, projections of both sides, dLoss/dp^ of one side at a time, the dv
// sums, c of the head
size_t wide_backward_bytes(const WidePlan &w)
{
    return 2 * w.state_bytes + 3 * w.p_bytes + w.acc_bytes + w.dacc_bytes;
}

cudaError_t map_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t cols, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_cols, CUtensorMapSwizzle sw)
{
    const EncodeTiled fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, (cuuint32_t)race::tc::T};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// One head's [N][128] bf16 as (16 columns, N rows, 8 atoms): a box of 4 atoms is one value half.
cudaError_t value_map_128(CUtensorMap *m, const void *ptr, int64_t N)
{
    const EncodeTiled fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {16, (cuuint64_t)N, 8};
    const cuuint64_t strides[2] = {256, 32};
    const cuuint32_t box[3] = {16, (cuuint32_t)race::tc::T, 4};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_scan_passes(float *buf, int npass, int nseg, int mode, cudaStream_t st,
                               const uint32_t *skip_if = nullptr)
{
    const int64_t MD = (int64_t)race::tc::MF * race::tc::DS;
    dim3 grid((unsigned)((MD + gk::NT - 1) / gk::NT), (unsigned)npass);
    return timed("segment_scan", st, [&] {
        gk::race_scan<<<grid, gk::NT, 0, st>>>(buf, nseg, MD, mode, nullptr, nullptr, skip_if, wd::kCtxTag);
        return cudaGetLastError();
    });
}

// p^ of the q and k rows of one head (bf16 [N][128] each) into pq, pk.
cudaError_t wide_projections(const WidePlan &w, const void *qh, const void *kh, const float *W, float *pq, float *pk,
                             cudaStream_t st)
{
    namespace tc = race::tc;
    wd::ProjArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    cudaError_t e;
    if ((e = map_2d(&pa.tm_x[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qh, wd::WD, (uint64_t)w.p.N, 256, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess ||
        (e = map_2d(&pa.tm_x[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kh, wd::WD, (uint64_t)w.p.N, 256, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
        return e;
    pa.W = W;
    pa.p[0] = pq;
    pa.p[1] = pk;
    pa.N = w.p.N;
    pa.ntile = w.ntile;
    pa.npw = w.npw;
    pa.npwp = w.npwp;
    const size_t sm = tc::smem_bytes(wd::proj_smem::TOTAL);
    if ((e = tc_prepare(wd::wide_proj, sm)) != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(2 * (int64_t)w.ntile, device_sm_count());
    return timed("wide_proj", st, [&] {
        wd::wide_proj<<<grid, tc::NTH, sm, st>>>(pa);
        return cudaGetLastError();
    });
}

cudaError_t wide_args(wd::WideArgs &a, const WidePlan &w, const float *pq, const float *pk, const void *vh,
                      const void *doh, float tau)
{
    std::memset(&a, 0, sizeof(a));
    cudaError_t e;
    const uint64_t N = (uint64_t)w.p.N, rb = (uint64_t)w.npwp * sizeof(float);
    if ((e = map_2d(&a.tm_pq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pq, (uint64_t)w.npwp, N, rb, wd::WPROJ,
                    CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess ||
        (e = map_2d(&a.tm_pk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pk, (uint64_t)w.npwp, N, rb, wd::WPROJ,
                    CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess ||
        (e = value_map_128(&a.tm_v, vh, w.p.N)) != cudaSuccess)
        return e;
    if (doh && (e = value_map_128(&a.tm_do, doh, w.p.N)) != cudaSuccess) return e;
    a.N = w.p.N;
    a.seg_len = w.p.seg_len;
    a.nseg = w.p.nseg;
    a.npwp = w.npwp;
    a.beta = 1.f / tau;
    return cudaSuccess;
}

// Segment totals of every (group, half) pass of one head (mode 0: key side, 1: query side).
cudaError_t wide_segment_totals(const WidePlan &w, wd::WideArgs a, int mode, float *out, cudaStream_t st)
{
    namespace tc = race::tc;
    const size_t sm = tc::smem_bytes(wd::wagg_smem::TOTAL);
    const dim3 grid((unsigned)(2 * w.G), (unsigned)w.p.nseg);
    a.agg_out = out;
    cudaError_t e;
    if (mode == 0) {
        if ((e = tc_prepare(wd::wide_agg<0>, sm)) != cudaSuccess) return e;
        return timed("wide_agg_kv", st, [&] {
            wd::wide_agg<0><<<grid, tc::NTH, sm, st>>>(a);
            return cudaGetLastError();
        });
    }
    if ((e = tc_prepare(wd::wide_agg<1>, sm)) != cudaSuccess) return e;
    return timed("wide_agg_qdy", st, [&] {
        wd::wide_agg<1><<<grid, tc::NTH, sm, st>>>(a);
        return cudaGetLastError();
    });
}

// ctx_tag: non-null when ctx (room for BH heads' states) receives them, with the tag set at the end.
cudaError_t wide_forward(int BH, int64_t N, int d, int L, int P, const void *q, const void *k, const void *v,
                         const float *W, void *out, float *den, float tau, void *workspace, float *ctx,
                         uint32_t *ctx_tag, cudaStream_t st)
{
    namespace tc = race::tc;
    const WidePlan w = wide_plan(N, d, L, P);
    uint8_t *ws = (uint8_t *)workspace;
    float *states = (float *)ws;
    float *pq = (float *)(ws + w.state_bytes);
    float *pk = (float *)(ws + w.state_bytes + w.p_bytes);
    float *acc = (float *)(ws + w.state_bytes + 2 * w.p_bytes);
    float *dacc = (float *)(ws + w.state_bytes + 2 * w.p_bytes + w.acc_bytes);
    const size_t sm_walk = tc::smem_bytes(wd::wfwd_smem::TOTAL);
    cudaError_t e;
    if ((e = tc_prepare(wd::wide_fwd_walk, sm_walk)) != cudaSuccess) return e;
    const size_t row_bytes = (size_t)N * wd::WD * sizeof(__nv_bfloat16);
    if (ctx_tag && (e = cudaMemsetAsync(ctx_tag, 0, 16, st)) != cudaSuccess) return e;
    for (int bh = 0; bh < BH; ++bh) {
        if (ctx_tag) states = (float *)((uint8_t *)ctx + bh * w.state_bytes);  // kept for the backward
        const uint8_t *qh = (const uint8_t *)q + bh * row_bytes, *kh = (const uint8_t *)k + bh * row_bytes;
        const uint8_t *vh = (const uint8_t *)v + bh * row_bytes;
        if ((e = wide_projections(w, qh, kh, W, pq, pk, st)) != cudaSuccess) return e;
        wd::WideArgs a;
        if ((e = wide_args(a, w, pq, pk, vh, nullptr, tau)) != cudaSuccess) return e;
        if ((e = wide_segment_totals(w, a, 0, states, st)) != cudaSuccess) return e;
        if ((e = launch_scan_passes(states, 2 * w.G, w.p.nseg, gk::SCAN_EXCL_PREFIX, st)) != cudaSuccess) return e;
        a.state = states;
        a.acc = acc;
        a.dacc = dacc;
        if ((e = map_2d(&a.tm_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, acc, wd::WD, (uint64_t)N, wd::WD * sizeof(float),
                        32, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
            return e;
        for (int g = 0; g < w.G; ++g) {
            a.g = g;
            a.first = g == 0;
            e = timed("wide_fwd_walk", st, [&] {
                wd::wide_fwd_walk<<<dim3(2, (unsigned)w.p.nseg), tc::NTH + 32, sm_walk, st>>>(a);
                return cudaGetLastError();
            });
            if (e != cudaSuccess) return e;
        }
        e = timed("wide_finish", st, [&] {
            wd::wide_finish<<<(unsigned)((N * 16 + 255) / 256), 256, 0, st>>>(
                acc, dacc, (__nv_bfloat16 *)((uint8_t *)out + bh * row_bytes), den ? den + (int64_t)bh * N : nullptr,
                N);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
    }
    if (ctx_tag && (e = cudaMemsetAsync(ctx_tag, 0x5A, 16, st)) != cudaSuccess) return e;
    return cudaSuccess;
}

// ctx_tag: non-null when ctx may hold the forward's key-side states (decided on the device).
cudaError_t wide_backward(int BH, int64_t N, int d, int L, int P, const void *q, const void *k, const void *v,
                          const float *W, const void *out, const float *den, const void *dout, void *dq, void *dk,
                          void *dv, float tau, void *workspace, const float *ctx, const uint32_t *ctx_tag,
                          cudaStream_t st)
{
    namespace tc = race::tc;
    const WidePlan w = wide_plan(N, d, L, P);
    uint8_t *ws = (uint8_t *)workspace;
    float *hstates = (float *)ws;
    float *gstates = (float *)(ws + w.state_bytes);
    uint8_t *arr = ws + 2 * w.state_bytes;
    float *pq = (float *)arr, *pk = (float *)(arr + w.p_bytes);
    float *dp = (float *)(arr + 2 * w.p_bytes);  // the q side's, then the k side's
    float *acc = (float *)(arr + 3 * w.p_bytes);
    float *cbuf = (float *)(arr + 3 * w.p_bytes + w.acc_bytes);
    const size_t sm_q = tc::smem_bytes(wd::wbq_smem::TOTAL), sm_kv = tc::smem_bytes(wd::wbkv_smem::TOTAL);
    const size_t sm_dx = tc::smem_bytes(wd::dx_smem::TOTAL);
    cudaError_t e;
    if ((e = tc_prepare(wd::wide_bwd_q_walk, sm_q)) != cudaSuccess ||
        (e = tc_prepare(wd::wide_bwd_kv_walk, sm_kv)) != cudaSuccess || (e = tc_prepare(wd::wide_dx, sm_dx)) != cudaSuccess)
        return e;
    const size_t row_bytes = (size_t)N * wd::WD * sizeof(__nv_bfloat16);
    const int dx_grid = (int)std::min<int64_t>(w.ntile, device_sm_count());
    auto launch_dx = [&](const void *xh, void *dxh) {  // dx of one side from dp
        wd::DxArgs xa;
        std::memset(&xa, 0, sizeof(xa));
        xa.x[0] = (const __nv_bfloat16 *)xh;
        xa.dp[0] = dp;
        xa.dx[0] = (__nv_bfloat16 *)dxh;
        xa.W = W;
        xa.N = N;
        xa.nsides = 1;
        xa.ntile = w.ntile;
        xa.npw = w.npw;
        xa.npwp = w.npwp;
        xa.kp = (w.npwp + 63) / 64 * 64;
        return timed("wide_dx", st, [&] {
            wd::wide_dx<<<dx_grid, tc::NTH, sm_dx, st>>>(xa);
            return cudaGetLastError();
        });
    };
    for (int bh = 0; bh < BH; ++bh) {
        const size_t off = bh * row_bytes;
        const uint8_t *qh = (const uint8_t *)q + off, *kh = (const uint8_t *)k + off, *vh = (const uint8_t *)v + off;
        const uint8_t *oh = (const uint8_t *)out + off, *doh = (const uint8_t *)dout + off;
        if ((e = wide_projections(w, qh, kh, W, pq, pk, st)) != cudaSuccess) return e;
        e = timed("wide_rowc", st, [&] {
            const int64_t threads = N * 16;
            wd::wide_rowc<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
                (const __nv_bfloat16 *)oh, (const __nv_bfloat16 *)doh, cbuf, N);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
        wd::WideArgs a;
        if ((e = wide_args(a, w, pq, pk, vh, doh, tau)) != cudaSuccess) return e;
        a.den = den + (int64_t)bh * N;
        a.cbuf = cbuf;
        a.ctx_tag = ctx_tag;
        a.ctx_states = ctx_tag ? (const float *)((const uint8_t *)ctx + bh * w.state_bytes) : nullptr;
        // query side: key-side prefix statistics (from the context when the forward left them
        // there), then the dq walks of every (group, half)
        if ((e = wide_segment_totals(w, a, 0, hstates, st)) != cudaSuccess) return e;
        if ((e = launch_scan_passes(hstates, 2 * w.G, w.p.nseg, gk::SCAN_EXCL_PREFIX, st, ctx_tag)) != cudaSuccess)
            return e;
        a.ctx_tag = nullptr;
        a.state = hstates;
        a.dp = dp;  // the walks add their shares of dLoss/dp^ onto zeros
        if ((e = cudaMemsetAsync(dp, 0, (size_t)N * w.npwp * sizeof(float), st)) != cudaSuccess) return e;
        e = timed("wide_bwd_q_walk", st, [&] {
            wd::wide_bwd_q_walk<<<dim3((unsigned)(2 * w.G), (unsigned)w.p.nseg), tc::NTH, sm_q, st>>>(a);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
        if ((e = launch_dx(qh, (uint8_t *)dq + off)) != cudaSuccess) return e;
        // key side: query-side suffix statistics, then the dk/dv walks, one group at a time
        if ((e = wide_segment_totals(w, a, 1, gstates, st)) != cudaSuccess) return e;
        if ((e = launch_scan_passes(gstates, 2 * w.G, w.p.nseg, gk::SCAN_EXCL_SUFFIX, st)) != cudaSuccess) return e;
        a.state = gstates;
        a.dp = dp;
        a.acc = acc;
        if ((e = map_2d(&a.tm_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, acc, wd::WD, (uint64_t)N, wd::WD * sizeof(float),
                        32, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
            return e;
        if ((e = cudaMemsetAsync(dp, 0, (size_t)N * w.npwp * sizeof(float), st)) != cudaSuccess) return e;
        for (int g = 0; g < w.G; ++g) {
            a.g = g;
            a.first = g == 0;
            e = timed("wide_bwd_kv_walk", st, [&] {
                wd::wide_bwd_kv_walk<<<dim3(2, (unsigned)w.p.nseg), tc::NTH, sm_kv, st>>>(a);
                return cudaGetLastError();
            });
            if (e != cudaSuccess) return e;
        }
        e = timed("wide_finish", st, [&] {
            wd::wide_finish<<<(unsigned)((N * 16 + 255) / 256), 256, 0, st>>>(
                acc, nullptr, (__nv_bfloat16 *)((uint8_t *)dv + off), nullptr, N);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
        if ((e = launch_dx(kh, (uint8_t *)dk + off)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename DT>
cudaError_t dispatch_forward(const Plan &p, const Args &a, float *states, int causal, cudaStream_t st,
                             const Shard &sh)
{
    if (p.d <= 64) return generic_forward<DT, 32>(p, a, states, causal, st, sh);
    return generic_forward<DT, 16>(p, a, states, causal, st, sh);
}

template <typename DT>
cudaError_t dispatch_backward(const Plan &p, const Args &a, const float *ctx, float *hbuf,
                              float *gbuf, int causal, cudaStream_t st, const Shard &sh)
{
    if (p.d <= 64) return generic_backward<DT, 32>(p, a, ctx, ctx != nullptr, hbuf, gbuf, causal, st, sh);
    return generic_backward<DT, 16>(p, a, ctx, ctx != nullptr, hbuf, gbuf, causal, st, sh);
}

// Bucket statistics of every key of each head (Algorithm 1's A and B): segment totals of the
// key side, summed over the segments into segment 0's slot of `tot`.
template <typename DT, int T>
cudaError_t generic_totals(const Plan &p, Args a, float *tot, cudaStream_t st)
{
    const size_t smem = gk::Smem(T, p.d, p.P).total * sizeof(float);
    a.causal = 0;
    a.agg_out = tot;
    return timed("generic_agg_kv", st, [&] { return launch_agg(gk::race_agg<DT, T, gk::AGG_KV>, p, smem, st, a, T); });
}

template <typename DT>
cudaError_t dispatch_totals(const Plan &p, const Args &a, float *tot, cudaStream_t st)
{
    if (p.d <= 64) return generic_totals<DT, 32>(p, a, tot, st);
    return generic_totals<DT, 16>(p, a, tot, st);
}

// Decode step: rows of each head's state split over nsplit CTAs (about two CTAs per SM over
// all heads, at least 32 rows per CTA).
struct DecodePlan {
    int nsplit, rows_per_split;
};
DecodePlan decode_plan(int BH, int M)
{
    const int target = 2 * device_sm_count();
    int nsplit = (target + BH - 1) / BH;
    const int maxsplit = (M + 31) / 32;
    if (nsplit > maxsplit) nsplit = maxsplit;
    if (nsplit < 1) nsplit = 1;
    DecodePlan dp;
    dp.rows_per_split = (M + nsplit - 1) / nsplit;
    dp.nsplit = (M + dp.rows_per_split - 1) / dp.rows_per_split;
    return dp;
}

}  // namespace

extern "C" {

const char *race_status_string(race_status_t s)
{
    switch (s) {
    case RACE_OK: return "RACE_OK";
    case RACE_ERR_INVALID_ARG: return "RACE_ERR_INVALID_ARG";
    case RACE_ERR_UNSUPPORTED: return "RACE_ERR_UNSUPPORTED";
    case RACE_ERR_WORKSPACE: return "RACE_ERR_WORKSPACE";
    case RACE_ERR_CUDA: return "RACE_ERR_CUDA";
    }
    return "RACE_ERR_UNKNOWN";
}

race_status_t race_attn_workspace_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                       int backward, race_dtype_t dtype, size_t *bytes)
{
    if (!bytes) return RACE_ERR_INVALID_ARG;
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    const Plan p = make_plan(B, H, N, d, L, P);
    *bytes = backward ? backward_workspace_bytes(p) : p.state_elems * sizeof(float);
    if (wide_ok(dtype, d, L, P, 1.f, causal, N)) {  // room for the feature-group path too
        const WidePlan w = wide_plan(N, d, L, P);
        *bytes = std::max(*bytes, backward ? wide_backward_bytes(w) : wide_forward_bytes(w));
    }
    return RACE_OK;
}

race_status_t race_attn_ctx_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                 size_t *bytes)
{
    if (!bytes) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    const Plan p = make_plan(B, H, N, d, L, P);
    *bytes = p.state_elems * sizeof(float);
    if (wide_shape(d, L, P, causal)) *bytes = wide_ctx_tag_offset(p, wide_plan(N, d, L, P)) + 256;
    return RACE_OK;
}

}  // extern "C"

namespace {

race_status_t forward_impl(const void *q, const void *k, const void *v, const float *W, void *out, float *den,
                           float *ctx, size_t ctx_bytes, int B, int H, int64_t N, int d, int L, int P, float tau,
                           int causal, race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                           race_stream_t stream, const Shard &sh)
{
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    if (!(tau >= 0.f) || !std::isfinite(tau)) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    if (N == 0) {  // an empty shard contributes zero statistics
        if (sh.h_total)
            return cudaMemsetAsync(sh.h_total, 0, (size_t)B * H * (L << P) * (d + 1) * sizeof(float),
                                   (cudaStream_t)stream) == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
        return RACE_OK;
    }
    const bool walk = sh.stage != STAGE_BEGIN;
    if (!k || !v || !W || !workspace || (walk && (!q || !out)) || (sh.stage == STAGE_BEGIN && !sh.h_total))
        return RACE_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(W) || !aligned16(workspace) || (q && !aligned16(q)) ||
        (out && !aligned16(out)) || (den && !aligned16(den)) || (ctx && !aligned16(ctx)) ||
        (sh.h_init && !aligned16(sh.h_init)) || (sh.h_total && !aligned16(sh.h_total)))
        return RACE_ERR_INVALID_ARG;
    const Plan p = make_plan(B, H, N, d, L, P);
    const size_t need = p.state_elems * sizeof(float);
    // d = 128, P = 5: the feature-group path when the workspace holds its arrays (it leaves
    // ctx untouched; the backward recomputes what it needs)
    const bool al32 = aligned32({q, k, v, out, workspace, ctx});
    const bool wide = sh.stage == STAGE_ALL && wide_ok(dtype, d, L, P, tau, causal, N) && al32 &&
                      workspace_bytes >= wide_forward_bytes(wide_plan(N, d, L, P));
    if (workspace_bytes < need && !wide) return RACE_ERR_WORKSPACE;
    if (ctx && ctx_bytes < need) return RACE_ERR_WORKSPACE;
    if (!q) q = k;  // the first half reads keys and values only
    Args a = base_args(p, W, tau);
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.den_out = den;
    float *states = ctx ? ctx : (float *)workspace;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    // for the shapes of the feature-group path, the tag after the states in ctx says whether
    // they are that path's (set by its forward) or not (cleared by every other forward)
    uint32_t *tag = nullptr;
    if (ctx && wide_shape(d, L, P, causal)) {
        const size_t off = wide_ctx_tag_offset(p, wide_plan(N, d, L, P));
        if (ctx_bytes >= off + 16) tag = (uint32_t *)((uint8_t *)ctx + off);
    }
    if (tag && !(wide && g_tc_forward) && cudaMemsetAsync(tag, 0, 16, st) != cudaSuccess) return RACE_ERR_CUDA;
    if (wide && g_tc_forward)
        e = wide_forward(B * H, N, d, L, P, q, k, v, W, out, den, tau, workspace, ctx, tag, st);
    else if (race::tc::fast_path_ok(dtype, d, L, P, tau, N) && al32 && g_tc_forward)
        e = tc_forward(p, q, k, v, W, out, den, states, tau, causal, st, sh);
    else if (dtype == RACE_F32)
        e = dispatch_forward<float>(p, a, states, causal, st, sh);
    else
        e = dispatch_forward<__nv_bfloat16>(p, a, states, causal, st, sh);
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

race_status_t backward_impl(const void *q, const void *k, const void *v, const float *W, const void *out,
                            const float *den, const void *dout, const float *ctx, size_t ctx_bytes, void *dq,
                            void *dk, void *dv, int B, int H, int64_t N, int d, int L, int P, float tau, int causal,
                            race_dtype_t dtype, void *workspace, size_t workspace_bytes, race_stream_t stream,
                            const Shard &sh)
{
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    if (!(tau >= 0.f) || !std::isfinite(tau)) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    if (tau == 0.f) return RACE_ERR_UNSUPPORTED;
    if (N == 0) {  // an empty shard contributes zero statistics
        if (sh.g_total)
            return cudaMemsetAsync(sh.g_total, 0, (size_t)B * H * (L << P) * (d + 1) * sizeof(float),
                                   (cudaStream_t)stream) == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
        return RACE_OK;
    }
    const bool first = sh.stage != STAGE_END, second = sh.stage != STAGE_BEGIN;
    if (!q || !k || !v || !W || !out || !den || !dout || !workspace || (first && !dq) || (second && (!dk || !dv)) ||
        (sh.stage == STAGE_BEGIN && !sh.g_total))
        return RACE_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, W, out, den, dout, workspace};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return RACE_ERR_INVALID_ARG;
    const void *opt[] = {ctx, dq, dk, dv, sh.h_init, sh.g_init, sh.g_total};
    for (const void *ptr : opt)
        if (ptr && !aligned16(ptr)) return RACE_ERR_INVALID_ARG;
    const Plan p = make_plan(B, H, N, d, L, P);
    const size_t one = p.state_elems * sizeof(float);
    const bool al32 = aligned32({q, k, v, out, dout, dq, dk, dv, workspace, ctx});
    const bool wide = sh.stage == STAGE_ALL && !sh.dpq && wide_ok(dtype, d, L, P, tau, causal, N) && al32 &&
                      workspace_bytes >= wide_backward_bytes(wide_plan(N, d, L, P));
    if (!wide && workspace_bytes < backward_workspace_bytes(p)) return RACE_ERR_WORKSPACE;
    if (ctx && ctx_bytes < one) return RACE_ERR_WORKSPACE;
    // for the shapes of the feature-group path the context may hold that path's states: only
    // that path reads it (after checking the tag on the device); the others recompute
    const float *wctx = nullptr;
    const uint32_t *tag = nullptr;
    if (ctx && wide_shape(d, L, P, causal)) {
        const size_t off = wide_ctx_tag_offset(p, wide_plan(N, d, L, P));
        if (ctx_bytes >= off + 16) {
            wctx = ctx;
            tag = (const uint32_t *)((const uint8_t *)ctx + off);
        }
        ctx = nullptr;
    }
    Args a = base_args(p, W, tau);
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = out;
    a.den_in = den;
    a.dout = dout;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    float *hbuf = (float *)workspace;
    float *gbuf = hbuf + p.state_elems;
    uint8_t *wimg = (uint8_t *)(gbuf + p.state_elems);
    float *cbuf = (float *)(wimg + kWImageBytes);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (wide && g_tc_backward)
        e = wide_backward(B * H, N, d, L, P, q, k, v, W, out, den, dout, dq, dk, dv, tau, workspace, wctx, tag, st);
    else if (race::tc::fast_path_ok(dtype, d, L, P, tau, N) && al32 && g_tc_backward)
        e = tc_backward(p, q, k, v, W, out, den, dout, ctx, hbuf, gbuf, wimg, cbuf, dq, dk, dv, tau, causal, st,
                        sh);
    else if (dtype == RACE_F32)
        e = dispatch_backward<float>(p, a, ctx, hbuf, gbuf, causal, st, sh);
    else
        e = dispatch_backward<__nv_bfloat16>(p, a, ctx, hbuf, gbuf, causal, st, sh);
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

// ---- gradient of W (the learnable-hyperplane variant) -----------------------------------
// Workspace after the backward's own: dLoss/dp / |x| for the q rows and the k rows (sized for
// the general path's fp32 [rows][L*P]; the tensor-core path uses bf16 [rows][64] of it), then
// the per-split partial sums of dW.
struct DwPlan {
    size_t dp_bytes;     // one side
    int tc_nblk;         // tensor-core reduction: CTAs
    int64_t tc_chunks_per_cta;
    int ksplit;          // general reduction: row splits
    int64_t rows_per_split;
    size_t partial_bytes;
};
DwPlan dw_plan(const Plan &p)
{
    DwPlan dp;
    const int64_t rows = (int64_t)p.BH * p.N;
    const int LP = p.L * p.P;
    dp.dp_bytes = ((size_t)rows * LP * sizeof(float) + 255) / 256 * 256;
    const int sms = device_sm_count();
    const int64_t cps = (int64_t)p.BH * ((p.N + race::tc::T - 1) / race::tc::T);
    dp.tc_nblk = (int)std::max<int64_t>(1, std::min<int64_t>(2 * sms, 2 * cps));
    dp.tc_chunks_per_cta = (2 * cps + dp.tc_nblk - 1) / dp.tc_nblk;
    const int tiles = ((LP + 63) / 64) * ((p.d + 63) / 64);
    dp.ksplit = (int)std::max<int64_t>(1, std::min<int64_t>((2 * sms + tiles - 1) / tiles, (2 * rows + 15) / 16));
    dp.rows_per_split = ((2 * rows + dp.ksplit - 1) / dp.ksplit + 15) / 16 * 16;
    const size_t tc_part = (size_t)dp.tc_nblk * 64 * 64 * sizeof(float);
    const size_t gen_part = (size_t)dp.ksplit * LP * p.d * sizeof(float);
    dp.partial_bytes = std::max(tc_part, gen_part);
    return dp;
}

cudaError_t tc_dw(const Plan &p, const DwPlan &dp, const void *q, const void *k, const void *dpq, const void *dpk,
                  float *partial, float *dW, cudaStream_t st)
{
    namespace tc = race::tc;
    tc::DwArgs a;
    std::memset(&a, 0, sizeof(a));
    cudaError_t e;
    if ((e = bf16_map(&a.tm_dp[0], dpq, p, false)) != cudaSuccess || (e = bf16_map(&a.tm_dp[1], dpk, p, false)) != cudaSuccess ||
        (e = bf16_map(&a.tm_x[0], q, p, false)) != cudaSuccess || (e = bf16_map(&a.tm_x[1], k, p, false)) != cudaSuccess)
        return e;
    a.chunks_per_head = (p.N + tc::T - 1) / tc::T;
    a.chunks_per_side = (int64_t)p.BH * a.chunks_per_head;
    a.chunks_per_cta = dp.tc_chunks_per_cta;
    a.partial = partial;
    const size_t sm = tc::smem_bytes(tc::dw_smem::TOTAL);
    if ((e = tc_prepare(tc::tc_dw, sm)) != cudaSuccess) return e;
    e = timed("tc_dw", st, [&] {
        tc::tc_dw<<<dp.tc_nblk, 128, sm, st>>>(a);
        return cudaGetLastError();
    });
    if (e != cudaSuccess) return e;
    return timed("dw_sum", st, [&] {
        tc::tc_dw_reduce<<<16, 256, 0, st>>>(partial, dp.tc_nblk, dW);
        return cudaGetLastError();
    });
}

template <typename DT>
cudaError_t generic_dw(const Plan &p, const DwPlan &dp, const void *q, const void *k, const float *dpq,
                       const float *dpk, float *partial, float *dW, cudaStream_t st)
{
    const int LP = p.L * p.P;
    const dim3 grid((unsigned)dp.ksplit, (unsigned)((LP + 63) / 64), (unsigned)((p.d + 63) / 64));
    cudaError_t e = timed("generic_dw", st, [&] {
        gk::race_dw_partial<DT><<<grid, gk::NT, 0, st>>>(dpq, dpk, (const DT *)q, (const DT *)k, (int64_t)p.BH * p.N,
                                                         LP, p.d, dp.rows_per_split, partial);
        return cudaGetLastError();
    });
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)LP * p.d;
    return timed("dw_sum", st, [&] {
        gk::race_dw_sum<<<(unsigned)((n + gk::NT - 1) / gk::NT), gk::NT, 0, st>>>(partial, dp.ksplit, n, dW);
        return cudaGetLastError();
    });
}

}  // namespace

extern "C" {

race_status_t race_attn_dw_workspace_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                          race_dtype_t dtype, size_t *bytes)
{
    (void)causal;
    if (!bytes) return RACE_ERR_INVALID_ARG;
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    const Plan p = make_plan(B, H, N, d, L, P);
    const DwPlan dp = dw_plan(p);
    *bytes = backward_workspace_bytes(p) + 2 * dp.dp_bytes + dp.partial_bytes;
    return RACE_OK;
}

race_status_t race_attn_backward_dw(const void *q, const void *k, const void *v, const float *W, const void *out,
                                    const float *den, const void *dout, const float *ctx, size_t ctx_bytes,
                                    void *dq, void *dk, void *dv, float *dW, int B, int H, int64_t N, int d, int L,
                                    int P, float tau, int causal, race_dtype_t dtype, void *workspace,
                                    size_t workspace_bytes, race_stream_t stream)
{
    if (!dW || !aligned16(dW)) return RACE_ERR_INVALID_ARG;
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    if (!(tau > 0.f) || !std::isfinite(tau)) return tau == 0.f ? RACE_ERR_UNSUPPORTED : RACE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (N == 0)
        return cudaMemsetAsync(dW, 0, (size_t)L * P * d * sizeof(float), st) == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
    const Plan p = make_plan(B, H, N, d, L, P);
    const DwPlan dp = dw_plan(p);
    const size_t bw = backward_workspace_bytes(p);
    if (!workspace) return RACE_ERR_INVALID_ARG;
    if (workspace_bytes < bw + 2 * dp.dp_bytes + dp.partial_bytes) return RACE_ERR_WORKSPACE;
    uint8_t *wsb = (uint8_t *)workspace;
    Shard sh;
    sh.dpq = wsb + bw;
    sh.dpk = wsb + bw + dp.dp_bytes;
    float *partial = (float *)(wsb + bw + 2 * dp.dp_bytes);
    s = backward_impl(q, k, v, W, out, den, dout, ctx, ctx_bytes, dq, dk, dv, B, H, N, d, L, P, tau, causal, dtype,
                      workspace, bw, stream, sh);
    if (s != RACE_OK) return s;
    cudaError_t e;
    // the same choice of path as the backward above made (it left dp in that path's format)
    if (race::tc::fast_path_ok(dtype, d, L, P, tau, N) && aligned32({q, k, v, out, dout, dq, dk, dv, workspace, ctx}) &&
        g_tc_backward)
        e = tc_dw(p, dp, q, k, sh.dpq, sh.dpk, partial, dW, st);
    else if (dtype == RACE_F32)
        e = generic_dw<float>(p, dp, q, k, (const float *)sh.dpq, (const float *)sh.dpk, partial, dW, st);
    else
        e = generic_dw<__nv_bfloat16>(p, dp, q, k, (const float *)sh.dpq, (const float *)sh.dpk, partial, dW, st);
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

race_status_t race_attn_forward(const void *q, const void *k, const void *v, const float *W,
                                void *out, float *den, float *ctx, size_t ctx_bytes, int B,
                                int H, int64_t N, int d, int L, int P, float tau, int causal,
                                race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                race_stream_t stream)
{
    return forward_impl(q, k, v, W, out, den, ctx, ctx_bytes, B, H, N, d, L, P, tau, causal, dtype, workspace,
                        workspace_bytes, stream, Shard());
}

race_status_t race_attn_backward(const void *q, const void *k, const void *v, const float *W,
                                 const void *out, const float *den, const void *dout,
                                 const float *ctx, size_t ctx_bytes, void *dq, void *dk,
                                 void *dv, int B, int H, int64_t N, int d, int L, int P,
                                 float tau, int causal, race_dtype_t dtype, void *workspace,
                                 size_t workspace_bytes, race_stream_t stream)
{
    return backward_impl(q, k, v, W, out, den, dout, ctx, ctx_bytes, dq, dk, dv, B, H, N, d, L, P, tau, causal,
                         dtype, workspace, workspace_bytes, stream, Shard());
}

race_status_t race_attn_forward_begin(const void *k, const void *v, const float *W, float *ctx, size_t ctx_bytes,
                                      float *h_total, int B, int H, int64_t N, int d, int L, int P, float tau,
                                      int causal, race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                      race_stream_t stream)
{
    Shard sh;
    sh.stage = STAGE_BEGIN;
    sh.h_total = h_total;
    return forward_impl(nullptr, k, v, W, nullptr, nullptr, ctx, ctx_bytes, B, H, N, d, L, P, tau, causal, dtype,
                        workspace, workspace_bytes, stream, sh);
}

race_status_t race_attn_forward_end(const void *q, const void *k, const void *v, const float *W,
                                    const float *h_init, void *out, float *den, float *ctx, size_t ctx_bytes, int B,
                                    int H, int64_t N, int d, int L, int P, float tau, int causal,
                                    race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                    race_stream_t stream)
{
    Shard sh;
    sh.stage = STAGE_END;
    sh.h_init = h_init;
    return forward_impl(q, k, v, W, out, den, ctx, ctx_bytes, B, H, N, d, L, P, tau, causal, dtype, workspace,
                        workspace_bytes, stream, sh);
}

race_status_t race_attn_backward_begin(const void *q, const void *k, const void *v, const float *W,
                                       const void *out, const float *den, const void *dout, const float *ctx,
                                       size_t ctx_bytes, const float *h_init, void *dq, float *g_total, int B,
                                       int H, int64_t N, int d, int L, int P, float tau, int causal,
                                       race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                       race_stream_t stream)
{
    Shard sh;
    sh.stage = STAGE_BEGIN;
    sh.h_init = h_init;
    sh.g_total = g_total;
    return backward_impl(q, k, v, W, out, den, dout, ctx, ctx_bytes, dq, nullptr, nullptr, B, H, N, d, L, P, tau,
                         causal, dtype, workspace, workspace_bytes, stream, sh);
}

race_status_t race_attn_backward_end(const void *q, const void *k, const void *v, const float *W,
                                     const void *out, const float *den, const void *dout, const float *g_init,
                                     void *dk, void *dv, int B, int H, int64_t N, int d, int L, int P, float tau,
                                     int causal, race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                     race_stream_t stream)
{
    Shard sh;
    sh.stage = STAGE_END;
    sh.g_init = g_init;
    return backward_impl(q, k, v, W, out, den, dout, nullptr, 0, nullptr, dk, dv, B, H, N, d, L, P, tau, causal,
                         dtype, workspace, workspace_bytes, stream, sh);
}

race_status_t race_attn_shard_combine(const float *gathered, int nshards, int shard, int which, int64_t elems,
                                      float *out, race_stream_t stream)
{
    if (!gathered || !out || nshards < 1 || shard < 0 || shard >= nshards || which < 0 || which > 2 || elems < 0)
        return RACE_ERR_INVALID_ARG;
    if (elems == 0) return RACE_OK;
    const unsigned blocks = (unsigned)((elems + gk::NT - 1) / gk::NT);
    cudaError_t e = timed("shard_combine", (cudaStream_t)stream, [&] {
        gk::race_shard_combine<<<blocks, gk::NT, 0, (cudaStream_t)stream>>>(gathered, nshards, shard, which, elems,
                                                                             out);
        return cudaGetLastError();
    });
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

race_status_t race_attn_hash_indices(const void *x, const float *W, int32_t *idx, int B, int H,
                                     int64_t N, int d, int L, int P, race_dtype_t dtype,
                                     race_stream_t stream)
{
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 0 || d < 1 || L < 1 || P < 1) return RACE_ERR_INVALID_ARG;
    if (d % 8 != 0 || d > 128 || P > 5) return RACE_ERR_UNSUPPORTED;
    if (N == 0) return RACE_OK;
    if (!x || !W || !idx) return RACE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W) || !aligned16(idx)) return RACE_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * H * N;
    const int64_t n = rows * L;
    const unsigned blocks = (unsigned)((n + gk::NT - 1) / gk::NT);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = timed("hash_indices", st, [&] {
        if (dtype == RACE_F32)
            gk::race_hash<float><<<blocks, gk::NT, 0, st>>>((const float *)x, W, idx, rows, d, L, P);
        else
            gk::race_hash<__nv_bfloat16>
                <<<blocks, gk::NT, 0, st>>>((const __nv_bfloat16 *)x, W, idx, rows, d, L, P);
        return cudaGetLastError();
    });
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

race_status_t race_attn_device_error(int *flag, race_stream_t stream)
{
    if (!flag) return RACE_ERR_INVALID_ARG;
    int v = 0;
    const int zero = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess ||
        cudaMemcpyFromSymbol(&v, race::tc::g_tc_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(race::tc::g_tc_error, &zero, sizeof(int)) != cudaSuccess)
        return RACE_ERR_CUDA;
    *flag = v;
    return RACE_OK;
}

race_status_t race_attn_selftest_wait_timeout(int64_t limit_ns, race_stream_t stream)
{
    if (limit_ns < 1 || limit_ns > 1000000000) return RACE_ERR_INVALID_ARG;
    race::tc::tc_wait_timeout_selftest<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_ns);
    return cudaGetLastError() == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

void race_attn_profile_enable(int on) { g_prof_on = on != 0; }

void race_attn_profile_reset(void)
{
    for (auto &p : g_pending) {
        cudaEventSynchronize(p.b);
        g_event_pool.push_back(p.a);
        g_event_pool.push_back(p.b);
    }
    g_pending.clear();
    g_prof.clear();
}

int race_attn_profile_read(char *names, float *ms, int64_t *launches, int max_kernels)
{
    int rc = 0;
    for (auto &p : g_pending) {
        float t = 0.f;
        if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&t, p.a, p.b) != cudaSuccess)
            rc = -1;
        g_prof[p.entry].ms += t;
        g_event_pool.push_back(p.a);
        g_event_pool.push_back(p.b);
    }
    g_pending.clear();
    if (rc) return rc;
    const int n = (int)g_prof.size();
    for (int i = 0; i < n && i < max_kernels; ++i) {
        if (names) {
            std::strncpy(names + 64 * i, g_prof[i].name.c_str(), 63);
            names[64 * i + 63] = 0;
        }
        if (ms) ms[i] = (float)g_prof[i].ms;
        if (launches) launches[i] = g_prof[i].launches;
    }
    return n;
}

}  // extern "C"

extern "C" {

race_status_t race_attn_state(const void *k, const void *v, const float *W, float *state, int B, int H,
                              int64_t N, int d, int L, int P, float tau, race_dtype_t dtype, void *workspace,
                              size_t workspace_bytes, race_stream_t stream)
{
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    if (!(tau >= 0.f) || !std::isfinite(tau)) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, N, d, L, P);
    if (s != RACE_OK) return s;
    if (!state || !W || !aligned16(state) || !aligned16(W)) return RACE_ERR_INVALID_ARG;
    const Plan p = make_plan(B, H, N, d, L, P);
    const size_t md = (size_t)p.M * p.D;
    cudaStream_t st = (cudaStream_t)stream;
    if (N == 0)
        return cudaMemsetAsync(state, 0, (size_t)p.BH * md * sizeof(float), st) == cudaSuccess ? RACE_OK
                                                                                             : RACE_ERR_CUDA;
    if (!k || !v || !workspace || !aligned16(k) || !aligned16(v) || !aligned16(workspace))
        return RACE_ERR_INVALID_ARG;
    if (workspace_bytes < p.state_elems * sizeof(float)) return RACE_ERR_WORKSPACE;
    float *tot = (float *)workspace;
    cudaError_t e;
    if (race::tc::fast_path_ok(dtype, d, L, P, tau, N) && g_tc_forward) {
        race::tc::BwdArgs ka;
        e = tc_args(ka, p, k, k, v, W, nullptr, nullptr, nullptr, tau, 0);
        if (e == cudaSuccess) e = tc_segment_totals(p, ka, 0, tot, st);
    } else {
        Args a = base_args(p, W, tau);
        a.q = k;
        a.k = k;
        a.v = v;
        e = dtype == RACE_F32 ? dispatch_totals<float>(p, a, tot, st) : dispatch_totals<__nv_bfloat16>(p, a, tot, st);
    }
    if (e == cudaSuccess) e = launch_scan(tot, p, gk::SCAN_TOTAL, st);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(state, md * sizeof(float), tot, (size_t)p.nseg * md * sizeof(float), md * sizeof(float),
                              (size_t)p.BH, cudaMemcpyDeviceToDevice, st);
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

race_status_t race_attn_decode_workspace_size(int B, int H, int d, int L, int P, size_t *bytes)
{
    if (!bytes) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, 1, d, L, P);
    if (s != RACE_OK) return s;
    const int M = L << P;
    const DecodePlan dp = decode_plan(B * H, M);
    *bytes = (size_t)B * H * dp.nsplit * (size_t)(d + 1) * sizeof(float);
    return RACE_OK;
}

race_status_t race_attn_decode_step(const void *q, const void *k, const void *v, const float *W, float *state,
                                    void *out, float *den, int B, int H, int d, int L, int P, float tau,
                                    race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                    race_stream_t stream)
{
    if (dtype != RACE_F32 && dtype != RACE_BF16) return RACE_ERR_INVALID_ARG;
    if (!(tau >= 0.f) || !std::isfinite(tau)) return RACE_ERR_INVALID_ARG;
    race_status_t s = check_sizes(B, H, 1, d, L, P);
    if (s != RACE_OK) return s;
    const void *ptrs[] = {q, k, v, W, state, out, workspace};
    for (const void *ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return RACE_ERR_INVALID_ARG;
    if (den && !aligned16(den)) return RACE_ERR_INVALID_ARG;
    namespace dk = race::decode;
    dk::Args a;
    std::memset(&a, 0, sizeof(a));
    const int BH = B * H;
    a.q = q;
    a.k = k;
    a.v = v;
    a.W = W;
    a.state = state;
    a.part = (float *)workspace;
    a.out = out;
    a.den = den;
    a.d = d;
    a.L = L;
    a.P = P;
    a.M = L << P;
    a.D = d + 1;
    const DecodePlan dp = decode_plan(BH, a.M);
    a.nsplit = dp.nsplit;
    a.rows_per_split = dp.rows_per_split;
    a.hard = tau == 0.f;
    a.beta = a.hard ? 0.f : 1.f / tau;
    if (workspace_bytes < (size_t)BH * dp.nsplit * (size_t)a.D * sizeof(float)) return RACE_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t smem = (size_t)dk::update_smem_floats(d, a.D, dp.rows_per_split, P) * sizeof(float);
    const dim3 grid((unsigned)dp.nsplit, (unsigned)BH);
    cudaError_t e = timed("decode_update", st, [&] {
        const bool narrow = d <= 64;  // two column slots of 32 cover d (else four: d <= 128)
        if (dtype == RACE_F32) {
            if (narrow)
                dk::race_decode_update<float, 2><<<grid, dk::NT, smem, st>>>(a);
            else
                dk::race_decode_update<float, 4><<<grid, dk::NT, smem, st>>>(a);
        } else {
            if (narrow)
                dk::race_decode_update<__nv_bfloat16, 2><<<grid, dk::NT, smem, st>>>(a);
            else
                dk::race_decode_update<__nv_bfloat16, 4><<<grid, dk::NT, smem, st>>>(a);
        }
        return cudaGetLastError();
    });
    if (e == cudaSuccess && dp.nsplit > 1)  // one split per head writes out_t itself
        e = timed("decode_readout", st, [&] {
            if (dtype == RACE_F32)
                dk::race_decode_readout<float><<<BH, dk::NT, 0, st>>>(a);
            else
                dk::race_decode_readout<__nv_bfloat16><<<BH, dk::NT, 0, st>>>(a);
            return cudaGetLastError();
        });
    return e == cudaSuccess ? RACE_OK : RACE_ERR_CUDA;
}

}  // extern "C"
