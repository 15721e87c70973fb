// race_tc.cuh -- tcgen05 (5th-generation tensor core) path of RACE Attention for the shape
// bf16 inputs, d = 64, L = 16 tables of P = 4 hyperplanes (L * 2^P = 256 features).
//
// Method ("RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training"):
// soft bucket assignment per token (zh §2.2), bucket statistics A, B (zh §2.2), the global
// read-out sum_l phi_l(q)^T B_l / sum_l phi_l(q)^T A_l (Algorithm 1) and its causal form
// with cumulative statistics (Algorithm 2, zh §2.3), evaluated chunk by chunk:
//
//   per chunk of T = 128 tokens, with V~ = [V | 1] (80 columns, 15 of them zero):
//     proj   = X W^T                        (X = raw q or k rows; W split as bf16 hi + lo)
//     Phi    = soft hash of proj / |x|      (CUDA cores: tanh, sigmoid products)
//     S      = Phi_Q Phi_K^T                (causal only; masked to j <= i)
//     Y      = Phi_Q H_prev  (+ S V~)       (H_prev: state before the chunk, staged as bf16)
//     H     += Phi_K^T V~                   (causal; fp32 master copy stays in TMEM)
//     out    = Y[:, :64] / Y[:, 64],  den = Y[:, 64]
//
// Every GEMM above is a tcgen05.mma with operands in shared memory (SW128 / SW32 swizzled
// tiles) and the accumulator in tensor memory; one thread issues them, completion is
// signalled through an mbarrier that the other threads wait on with a bounded poll.
// One CTA of 256 threads walks one segment of one (b, h) sequence; thread t owns token
// row t % 128 and the tables of half t / 128 (tables 0-7 or 8-15).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "race_attn.h"
#include "race_common.cuh"
#include "race_tc_util.cuh"

namespace race {
namespace tc {

constexpr int T = 128;      // tokens per chunk (MMA M)
constexpr int NTH = 256;    // threads per CTA
constexpr int DH = 64;      // head dimension
constexpr int NPROJ = 64;   // L * P projections
constexpr int MF = 256;     // L * 2^P features
constexpr int NV = 80;      // value columns: 64 of V, the ones column, 15 zero
constexpr int DS = 65;      // state row length in global memory (64 + ones column)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far above any chunk's MMA time

constexpr uint32_t TILE = 16384;  // one [128][64] bf16 SW128 tile

// error word shared by all launches of this path (1 = an MMA completion wait timed out)
__device__ int g_tc_error;

struct Args {
    const __nv_bfloat16 *q, *k, *v;
    const float *W;
    __nv_bfloat16 *out;
    float *den;
    const float *state;        // walk start states [BH][nseg][256][65]
    int64_t state_seg_stride;  // floats between segments' states (0 = one shared state)
    float *agg_out;            // aggregate output [BH][nseg][256][65]
    int64_t N, seg_len;
    int nseg;
    float beta;
    int causal;
};

// ---- shared memory maps (byte offsets from a 1024-aligned base) -------------------------
namespace fwd_smem {
constexpr uint32_t PHQ = 0;                 // Phi_Q [128][256]: 4 SW128 tiles
constexpr uint32_t XQ = PHQ;                // q rows during the projection
constexpr uint32_t XK = PHQ + TILE;         // k rows during the projection
constexpr uint32_t SB = PHQ;                // masked S as bf16 [128][128]: 2 tiles
constexpr uint32_t PHK = PHQ + 4 * TILE;    // Phi_K [128][256]
constexpr uint32_t HS128 = PHK + 4 * TILE;  // staged H[:, 0:64] as [256][64] SW128 (2 tiles)
constexpr uint32_t HS32 = HS128 + 2 * TILE; // staged H[:, 64:80] as [256][16] SW32 (8 KB)
constexpr uint32_t V = HS32 + 8192;         // v rows [128][64]
constexpr uint32_t ONES = V + TILE;         // ones column block [128][16] SW32 (4 KB)
constexpr uint32_t WHI = ONES + 4096;       // W hi [64][64]
constexpr uint32_t WLO = WHI + 8192;        // W lo [64][64]
constexpr uint32_t BAR = WLO + 8192;        // mbarrier, TMEM address, abort flag
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace fwd_smem

namespace agg_smem {
constexpr uint32_t PHK = 0;                 // Phi_K, also k rows during the projection
constexpr uint32_t XK = PHK;
constexpr uint32_t V = PHK + 4 * TILE;
constexpr uint32_t ONES = V + TILE;
constexpr uint32_t WHI = ONES + 4096;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t BAR = WLO + 8192;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace agg_smem

// TMEM columns
namespace fwd_tmem {
constexpr uint32_t PROJ = 0;    // [128][64] q projections, [128][64] k projections at +64
constexpr uint32_t S = 0;       // [128][128] (reuses PROJ once the features are formed)
constexpr uint32_t Y = 128;     // [128][80]
constexpr uint32_t HTOP = 256;  // H rows 0..127   [128][80]
constexpr uint32_t HBOT = 336;  // H rows 128..255 [128][80]
constexpr uint32_t NCOLS = 512;
}  // namespace fwd_tmem
namespace agg_tmem {
constexpr uint32_t PROJ = 0;
constexpr uint32_t HTOP = 64;
constexpr uint32_t HBOT = 144;
constexpr uint32_t NCOLS = 256;
}  // namespace agg_tmem

struct Ctl {
    uint64_t bar;
    uint32_t tmem;
    uint32_t abort;
};

__device__ __forceinline__ uint8_t *aligned_base(uint8_t *raw)
{
    const uint32_t a = smem_u32(raw);
    return raw + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ uint32_t lane_base() { return (uint32_t)((threadIdx.x >> 5) & 3) * 32u; }

// W [64][64] fp32 -> two SW128 tiles of bf16 (hi = round(W), lo = round(W - hi)).
__device__ void load_w_split(const float *W, uint8_t *whi, uint8_t *wlo)
{
    for (int e = threadIdx.x; e < NPROJ * DH; e += NTH) {
        const int n = e >> 6, c = e & 63;
        const float w = W[e];
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
        const uint32_t off = sw128_off(n, c >> 3) + (c & 7) * 2;
        *reinterpret_cast<__nv_bfloat16 *>(whi + off) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(wlo + off) = lo;
    }
}

// Ones column block: row j holds 1 in column 0 when j < nvalid, zeros elsewhere.
__device__ void write_ones(uint8_t *ones, int nvalid)
{
    if (threadIdx.x < T) {
        const int j = threadIdx.x;
        const uint32_t one = j < nvalid ? 0x3F80u : 0u;  // bf16 1.0 in the low half
        const uint32_t a = smem_u32(ones);
        st_shared_v4(a + sw32_off(j, 0), one, 0u, 0u, 0u);
        st_shared_v4(a + sw32_off(j, 1), 0u, 0u, 0u, 0u);
    }
}

// Wait for the MMAs committed to ctl->bar; one thread polls (bounded), all learn the outcome.
__device__ __forceinline__ bool wait_mma(Ctl *ctl, uint32_t &phase)
{
    if (threadIdx.x == 0) {
        if (!mbar_wait(&ctl->bar, phase & 1u, WAIT_LIMIT_NS)) {
            ctl->abort = 1u;
            atomicExch(&g_tc_error, 1);
        }
    }
    ++phase;
    __syncthreads();
    fence_after_sync();
    return *(volatile uint32_t *)&ctl->abort == 0u;
}

// Hand the shared-memory tiles written so far to the tensor core and sync the CTA.
__device__ __forceinline__ void publish_smem()
{
    fence_smem_async();
    fence_before_sync();
    __syncthreads();
}

// Squared L2 norm of row r of a [128][64] SW128 tile.
__device__ __forceinline__ float row_sqnorm(const uint8_t *tile, int r)
{
    const uint32_t a = smem_u32(tile);
    float s = 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint4 w = ld_shared_v4(a + sw128_off(r, ch));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x0 = bf16_lo(ws[i]), x1 = bf16_hi(ws[i]);
            s = fmaf(x0, x0, s);
            s = fmaf(x1, x1, s);
        }
    }
    return s;
}

// Soft bucket assignment of the 8 tables of half h for token row r, from the 32
// projections in TMEM (columns col0 + 32h ..), written as bf16 into the Phi tile
// [128][256].  phi_l[r] = prod_p sigmoid(2 beta c_rp u_p) with u = tanh(proj / |x|): the
// corner softmax of zh §2.2 in factorised form; sigmoid(2z) = (1 + tanh z) / 2.
__device__ __forceinline__ void features_half(uint32_t tmem, uint32_t col0, int r, int h, float inv_norm,
                                              float beta, bool valid, uint8_t *phi)
{
    float pr[32];
    {
        float a[16], b[16];
        const uint32_t t = tmem + (lane_base() << 16) + col0 + 32u * h;
        tmem_ld16(t, a);
        tmem_ld16(t + 16, b);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            pr[i] = a[i];
            pr[16 + i] = b[i];
        }
    }
    const uint32_t base = smem_u32(phi);
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        float f[16];
        f[0] = 1.f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float u = tanh_fast(pr[4 * l + p] * inv_norm);
            const float t = tanh_fast(beta * u);
            const float s1 = 0.5f + 0.5f * t, s0 = 0.5f - 0.5f * t;
            const int hh = 1 << p;
#pragma unroll
            for (int c = 0; c < hh; ++c) {
                f[c + hh] = f[c] * s1;
                f[c] *= s0;
            }
        }
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = valid ? pack_bf16x2(f[2 * i], f[2 * i + 1]) : 0u;
        const int tl = 8 * h + l;            // table 0..15 -> features 16 tl .. 16 tl + 15
        const uint32_t blk = base + (uint32_t)(tl >> 2) * TILE;
        const int ch = (tl & 3) * 2;
        st_shared_v4(blk + sw128_off(r, ch), w[0], w[1], w[2], w[3]);
        st_shared_v4(blk + sw128_off(r, ch + 1), w[4], w[5], w[6], w[7]);
    }
}

// proj[128][64] (+)= X[128][64] (W_hi + W_lo)^T
__device__ __forceinline__ void issue_proj(uint32_t d, uint32_t x, uint32_t whi, uint32_t wlo)
{
    constexpr uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sdesc(x + kk * 32, 16, 1024, LAYOUT_SW128);
        mma_bf16(d, a, sdesc(whi + kk * 32, 16, 1024, LAYOUT_SW128), id, kk > 0);
        mma_bf16(d, a, sdesc(wlo + kk * 32, 16, 1024, LAYOUT_SW128), id, 1);
    }
}

// D[128][80] (+)= A * [V | 1] with A given per K-step (16 tokens) by a_at(kk); B from the
// V tile (MN-major SW128) and the ones block (MN-major SW32).
template <typename AF>
__device__ __forceinline__ void issue_times_vt(uint32_t d, AF a_at, int a_mn, uint32_t vt, uint32_t ones,
                                               bool acc_first)
{
    const uint32_t i64 = idesc_bf16(128, 64, a_mn, 1), i16 = idesc_bf16(128, 16, a_mn, 1);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint64_t a = a_at(kk);
        const uint32_t acc = (kk > 0 || acc_first) ? 1u : 0u;
        mma_bf16(d, a, sdesc(vt + kk * 2048, TILE, 1024, LAYOUT_SW128), i64, acc);
        mma_bf16(d + 64, a, sdesc(ones + kk * 512, 4096, 256, LAYOUT_SW32), i16, acc);
    }
}

// H (both halves) += Phi_K^T [V | 1]
__device__ __forceinline__ void issue_state_update(uint32_t tm, uint32_t htop, uint32_t hbot, uint32_t phk,
                                                   uint32_t vt, uint32_t ones)
{
    issue_times_vt(tm + htop, [&](int kk) { return sdesc(phk + kk * 2048, TILE, 1024, LAYOUT_SW128); }, 1,
                   vt, ones, true);
    issue_times_vt(tm + hbot,
                   [&](int kk) { return sdesc(phk + 2 * TILE + kk * 2048, TILE, 1024, LAYOUT_SW128); }, 1,
                   vt, ones, true);
}

// Row of the state (lane r of the H half h: feature m = 128h + r), 80 columns -> regs.
__device__ __forceinline__ void read_state_row(uint32_t tmem, uint32_t col, float (&hv)[80])
{
    const uint32_t t = tmem + (lane_base() << 16) + col;
#pragma unroll
    for (int c = 0; c < 5; ++c) {
        float x[16];
        tmem_ld16(t + 16 * c, x);
#pragma unroll
        for (int i = 0; i < 16; ++i) hv[16 * c + i] = x[i];
    }
    tmem_wait_ld();
}

// Stage one state row (feature m) as bf16 into the [256][64] SW128 + [256][16] SW32 tiles.
__device__ __forceinline__ void stage_state_row(const float (&hv)[80], int m, uint8_t *hs128, uint8_t *hs32)
{
    const uint32_t b128 = smem_u32(hs128) + (uint32_t)(m >> 7) * TILE;
    const int rr = m & 127;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
        st_shared_v4(b128 + sw128_off(rr, ch), pack_bf16x2(hv[8 * ch], hv[8 * ch + 1]),
                     pack_bf16x2(hv[8 * ch + 2], hv[8 * ch + 3]), pack_bf16x2(hv[8 * ch + 4], hv[8 * ch + 5]),
                     pack_bf16x2(hv[8 * ch + 6], hv[8 * ch + 7]));
    const uint32_t b32 = smem_u32(hs32);
#pragma unroll
    for (int ch = 0; ch < 2; ++ch)
        st_shared_v4(b32 + sw32_off(m, ch), pack_bf16x2(hv[64 + 8 * ch], hv[65 + 8 * ch]),
                     pack_bf16x2(hv[66 + 8 * ch], hv[67 + 8 * ch]), pack_bf16x2(hv[68 + 8 * ch], hv[69 + 8 * ch]),
                     pack_bf16x2(hv[70 + 8 * ch], hv[71 + 8 * ch]));
}

__device__ __forceinline__ void seg_bounds(const Args &a, int seg, int64_t &t0, int64_t &t1)
{
    t0 = (int64_t)seg * a.seg_len;
    t1 = t0 + a.seg_len;
    if (t1 > a.N) t1 = a.N;
}

// ------------------------------------------------------------------------------------------
// Segment totals: H_seg = sum_{j in segment} phi(k_j) [v_j, 1]^T   (grid: nseg x BH)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 2) tc_agg_kv(Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace agg_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        ctl->abort = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, agg_tmem::NCOLS);
    load_w_split(a.W, sm + WHI, sm + WLO);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = ctl->tmem;
    {  // zero state
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
        const uint32_t t = tm + (lane_base() << 16) + (h ? agg_tmem::HBOT : agg_tmem::HTOP);
#pragma unroll
        for (int c = 0; c < 5; ++c) tmem_st16(t + 16 * c, z);
        tmem_wait_st();
    }
    int64_t t0, t1;
    seg_bounds(a, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        load_tile_async<NTH>(sm + XK, a.k + (base + c0) * DH, nv);
        load_tile_async<NTH>(sm + V, a.v + (base + c0) * DH, nv);
        cp_async_commit();
        write_ones(sm + ONES, nv);
        cp_async_wait_all();
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_proj(tm + agg_tmem::PROJ, sb + XK, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        const float inv = 1.f / fmaxf(sqrtf(row_sqnorm(sm + XK, r)), kNormEps);
        if (!(ok = wait_mma(ctl, phase))) break;
        features_half(tm, agg_tmem::PROJ, r, h, inv, a.beta, r < nv, sm + PHK);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_state_update(tm, agg_tmem::HTOP, agg_tmem::HBOT, sb + PHK, sb + V, sb + ONES);
            mma_commit(&ctl->bar);
        }
        ok = wait_mma(ctl, phase);
    }
    if (ok) {
        float hv[80];
        read_state_row(tm, h ? agg_tmem::HBOT : agg_tmem::HTOP, hv);
        const int m = 128 * h + r;
        float *dst = a.agg_out + (((int64_t)bh * a.nseg + seg) * MF + m) * DS;
#pragma unroll
        for (int c = 0; c < DS; ++c) dst[c] = hv[c];
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, agg_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// Walk: causal (Algorithm 2) or bidirectional read-out (Algorithm 1).  grid: nseg x BH
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 1) tc_fwd_walk(Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace fwd_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const bool causal = a.causal != 0;
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        ctl->abort = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, fwd_tmem::NCOLS);
    load_w_split(a.W, sm + WHI, sm + WLO);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = ctl->tmem;
    {  // start state: fp32 master into TMEM, bf16 copy into the staging tiles
        const int m = 128 * h + r;
        const float *src = a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride + (int64_t)m * DS;
        float hv[80];
#pragma unroll
        for (int c = 0; c < 80; ++c) hv[c] = c < DS ? src[c] : 0.f;
        const uint32_t t = tm + (lane_base() << 16) + (h ? fwd_tmem::HBOT : fwd_tmem::HTOP);
#pragma unroll
        for (int c = 0; c < 5; ++c) {
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = hv[16 * c + i];
            tmem_st16(t + 16 * c, x);
        }
        tmem_wait_st();
        stage_state_row(hv, m, sm + HS128, sm + HS32);
    }
    int64_t t0, t1;
    seg_bounds(a, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        load_tile_async<NTH>(sm + XQ, a.q + (base + c0) * DH, nv);
        if (causal) {
            load_tile_async<NTH>(sm + XK, a.k + (base + c0) * DH, nv);
            load_tile_async<NTH>(sm + V, a.v + (base + c0) * DH, nv);
        }
        cp_async_commit();
        if (causal) write_ones(sm + ONES, nv);
        cp_async_wait_all();
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_proj(tm + fwd_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
            if (causal) issue_proj(tm + fwd_tmem::PROJ + 64, sb + XK, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        const float inv_q = 1.f / fmaxf(sqrtf(row_sqnorm(sm + XQ, r)), kNormEps);
        const float inv_k = causal ? 1.f / fmaxf(sqrtf(row_sqnorm(sm + XK, r)), kNormEps) : 0.f;
        if (!(ok = wait_mma(ctl, phase))) break;
        features_half(tm, fwd_tmem::PROJ, r, h, inv_q, a.beta, r < nv, sm + PHQ);
        if (causal) features_half(tm, fwd_tmem::PROJ + 64, r, h, inv_k, a.beta, r < nv, sm + PHK);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            if (causal) {  // S = Phi_Q Phi_K^T
                constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint32_t off = (kk >> 2) * TILE + (kk & 3) * 32;
                    mma_bf16(tm + fwd_tmem::S, sdesc(sb + PHQ + off, 16, 1024, LAYOUT_SW128),
                             sdesc(sb + PHK + off, 16, 1024, LAYOUT_SW128), id, kk > 0);
                }
            }
            {  // Y = Phi_Q H_prev
                constexpr uint32_t i64 = idesc_bf16(128, 64, 0, 1), i16 = idesc_bf16(128, 16, 0, 1);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint64_t aq = sdesc(sb + PHQ + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024, LAYOUT_SW128);
                    mma_bf16(tm + fwd_tmem::Y, aq, sdesc(sb + HS128 + kk * 2048, TILE, 1024, LAYOUT_SW128), i64,
                             kk > 0);
                    mma_bf16(tm + fwd_tmem::Y + 64, aq, sdesc(sb + HS32 + kk * 512, 8192, 256, LAYOUT_SW32), i16,
                             kk > 0);
                }
            }
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        if (causal) {
            // masked S (j <= i) as bf16: row r, columns 64h .. 64h+63
            const uint32_t t = tm + (lane_base() << 16) + fwd_tmem::S + 64u * h;
            const uint32_t blk = sb + SB + (uint32_t)h * TILE;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x[16];
                tmem_ld16(t + 16 * c, x);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (64 * h + 16 * c + i > r) x[i] = 0.f;
                st_shared_v4(blk + sw128_off(r, 2 * c), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                             pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
                st_shared_v4(blk + sw128_off(r, 2 * c + 1), pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]),
                             pack_bf16x2(x[12], x[13]), pack_bf16x2(x[14], x[15]));
            }
            publish_smem();
            if (threadIdx.x == 0) {
                fence_after_sync();
                // Y += S [V | 1]
                issue_times_vt(tm + fwd_tmem::Y,
                               [&](int kk) {
                                   return sdesc(sb + SB + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024,
                                                LAYOUT_SW128);
                               },
                               0, sb + V, sb + ONES, true);
                // H += Phi_K^T [V | 1]
                issue_state_update(tm, fwd_tmem::HTOP, fwd_tmem::HBOT, sb + PHK, sb + V, sb + ONES);
                mma_commit(&ctl->bar);
            }
            if (!(ok = wait_mma(ctl, phase))) break;
        }
        {  // out = Y[:, :64] / Y[:, 64]: this thread writes columns 32h .. 32h+31 of row r
            float y[32], dn[16];
            const uint32_t t = tm + (lane_base() << 16) + fwd_tmem::Y;
            float y0[16], y1[16];
            tmem_ld16(t + 32u * h, y0);
            tmem_ld16(t + 32u * h + 16, y1);
            tmem_ld16(t + 64, dn);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                y[i] = y0[i];
                y[16 + i] = y1[i];
            }
            if (r < nv) {
                const float d = dn[0];
                const float inv = d != 0.f ? 1.f / d : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + (base + c0 + r) * DH + 32 * h);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(pack_bf16x2(y[8 * v4] * inv, y[8 * v4 + 1] * inv),
                                         pack_bf16x2(y[8 * v4 + 2] * inv, y[8 * v4 + 3] * inv),
                                         pack_bf16x2(y[8 * v4 + 4] * inv, y[8 * v4 + 5] * inv),
                                         pack_bf16x2(y[8 * v4 + 6] * inv, y[8 * v4 + 7] * inv));
                if (h == 0 && a.den) a.den[base + c0 + r] = d;
            }
        }
        if (causal) {  // stage the updated state for the next chunk's read-out
            float hv[80];
            read_state_row(tm, h ? fwd_tmem::HBOT : fwd_tmem::HTOP, hv);
            stage_state_row(hv, 128 * h + r, sm + HS128, sm + HS32);
        }
        publish_smem();
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, fwd_tmem::NCOLS);
}

// ==========================================================================================
// Backward.  With c_i = -(dO_i . o_i) and dY_i = [dO_i, c_i] / den_i (the gradient of
// out_i = Y_i[:64] / Y_i[64] with respect to Y_i):
//   dq side (prefix state H, chunks in order):
//     dPhi_Q[i] = (dO_i H_prev[:, :64]^T + c_i H_prev[:, 64] + sum_{j<=i} (v_j.dO_i + c_i) Phi_K[j]) / den_i
//     H += Phi_K^T [V | 1]
//   dk/dv side (suffix state G = sum_i Phi_Q[i] dY_i^T, chunks walked backwards), with
//   Phi_Q' = Phi_Q / den (row-scaled):
//     dV[j]     = Phi_K[j] G_next[:, :64] + sum_{i>=j} (Phi_K[j].Phi_Q'[i]) dO_i
//     dPhi_K[j] = [v_j, 1] G_next^T + sum_{i>=j} (v_j.dO_i + c_i) Phi_Q'[i]
//     G += Phi_Q'^T [dO | c]
//   feature-map VJP per table (CUDA cores): dz = phi (dphi - phi.dphi),
//   du_p = beta sum_r c_rp dz_r, dp~ = du (1 - u^2); then dX^ = dP~ W (tcgen05) and
//   dx = (dX^ - x^ (x^ . dX^)) / |x|.
// The terms v_j.dO_i and c_i nearly cancel when o_i is close to v_j (short prefixes), so
// they are formed in fp32 from exact bf16 inputs (dO, v), with c_i added in fp32, and the
// dq side reads the state as a bf16 hi + lo pair.
// ==========================================================================================

struct BwdArgs {
    const __nv_bfloat16 *q, *k, *v, *o, *dout;
    const float *den, *W;
    __nv_bfloat16 *dq, *dk, *dv;
    const float *state;
    int64_t state_seg_stride;
    float *agg_out;
    int64_t N, seg_len;
    int nseg;
    float beta;
    int causal;
};

// Per-row scalars of a chunk: rowc[r] = c_r = -(dO_r . o_r), rowinv[r] = 1/den_r (0 beyond
// nvalid); dO read from its SW128 tile, o from global.  Optionally the SW32 block dc32
// gets c_r (bf16) in column 0.  Threads 0..127, one row each.
__device__ __forceinline__ void row_scalars(const uint8_t *do_tile, const __nv_bfloat16 *o, const float *den,
                                            int nvalid, float *rowc, float *rowinv, uint8_t *dc32)
{
    if (threadIdx.x >= T) return;
    const int r = threadIdx.x;
    float c = 0.f, inv = 0.f;
    if (r < nvalid) {
        const uint32_t a = smem_u32(do_tile);
        const uint4 *o4 = reinterpret_cast<const uint4 *>(o + (int64_t)r * DH);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 g = ld_shared_v4(a + sw128_off(r, ch)), ov = o4[ch];
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, ow[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                c = fmaf(bf16_lo(gw[i]), bf16_lo(ow[i]), c);
                c = fmaf(bf16_hi(gw[i]), bf16_hi(ow[i]), c);
            }
        }
        c = -c;
        const float dn = den[r];
        inv = dn != 0.f ? 1.f / dn : 0.f;
    }
    rowc[r] = c;
    rowinv[r] = inv;
    if (dc32) {
        const uint32_t b = smem_u32(dc32);
        st_shared_v4(b + sw32_off(r, 0), pack_bf16x2(c, 0.f), 0u, 0u, 0u);
        st_shared_v4(b + sw32_off(r, 1), 0u, 0u, 0u, 0u);
    }
}

// u = tanh(proj / |x|) and t = tanh(beta u) of the 32 projections of half h (8 tables),
// kept in registers for the feature-map VJP.
__device__ __forceinline__ void proj_keep(uint32_t tmem, uint32_t col0, int h, float inv_norm, float beta,
                                          float (&u)[32], float (&t)[32])
{
    float a[16], b[16];
    const uint32_t ta = tmem + (lane_base() << 16) + col0 + 32u * h;
    tmem_ld16(ta, a);
    tmem_ld16(ta + 16, b);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        u[i] = tanh_fast(a[i] * inv_norm);
        u[16 + i] = tanh_fast(b[i] * inv_norm);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] = tanh_fast(beta * u[i]);
}

// Features of the 8 tables of half h from t = tanh(beta u), times `scale`, as bf16 into row r
// of the Phi tile [128][256].
__device__ __forceinline__ void write_features(const float (&t)[32], int r, int h, float scale, uint8_t *phi)
{
    const uint32_t base = smem_u32(phi);
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        float f[16];
        f[0] = scale;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float s1 = 0.5f + 0.5f * t[4 * l + p], s0 = 0.5f - 0.5f * t[4 * l + p];
            const int hh = 1 << p;
#pragma unroll
            for (int c = 0; c < hh; ++c) {
                f[c + hh] = f[c] * s1;
                f[c] *= s0;
            }
        }
        const int tl = 8 * h + l;
        const uint32_t blk = base + (uint32_t)(tl >> 2) * TILE;
        const int ch = (tl & 3) * 2;
        st_shared_v4(blk + sw128_off(r, ch), pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        st_shared_v4(blk + sw128_off(r, ch + 1), pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                     pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
    }
}

// Feature-map VJP for the 8 tables of half h.  dphi[m] = (D[m] + add_scale * add_vec[m]) * mul
// with D read from TMEM columns col0 + 128h .. (16 per table) and add_vec (features, fp32,
// shared memory) optional; writes dp~ (32 values) as bf16 into row r of the DP tile
// ([128][64] SW128, projections 32h .. 32h+31).
__device__ __forceinline__ void features_vjp_half(uint32_t tmem, uint32_t col0, int r, int h, float beta,
                                                  bool valid, const float (&u)[32], const float (&t)[32],
                                                  const float *add_vec, float add_scale, float mul,
                                                  uint8_t *dp_tile)
{
    float dp[32];
    const uint32_t ta = tmem + (lane_base() << 16) + col0 + 128u * h;
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        float g[16];
        tmem_ld16(ta + 16 * l, g);
        tmem_wait_ld();
        if (add_vec) {
            const float *av = add_vec + 128 * h + 16 * l;
#pragma unroll
            for (int c = 0; c < 16; ++c) g[c] = fmaf(add_scale, av[c], g[c]) * mul;
        }
        float f[16];
        f[0] = 1.f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float s1 = 0.5f + 0.5f * t[4 * l + p], s0 = 0.5f - 0.5f * t[4 * l + p];
            const int hh = 1 << p;
#pragma unroll
            for (int c = 0; c < hh; ++c) {
                f[c + hh] = f[c] * s1;
                f[c] *= s0;
            }
        }
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) dot = fmaf(f[c], g[c], dot);
        float du[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float dz = f[c] * (g[c] - dot);
#pragma unroll
            for (int p = 0; p < 4; ++p) du[p] += ((c >> p) & 1) ? dz : -dz;
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float uu = u[4 * l + p];
            dp[4 * l + p] = valid ? beta * du[p] * (1.f - uu * uu) : 0.f;
        }
    }
    const uint32_t b = smem_u32(dp_tile);
#pragma unroll
    for (int ch = 0; ch < 4; ++ch)
        st_shared_v4(b + sw128_off(r, 4 * h + ch), pack_bf16x2(dp[8 * ch], dp[8 * ch + 1]),
                     pack_bf16x2(dp[8 * ch + 2], dp[8 * ch + 3]), pack_bf16x2(dp[8 * ch + 4], dp[8 * ch + 5]),
                     pack_bf16x2(dp[8 * ch + 6], dp[8 * ch + 7]));
}

// D[128][64] = DP[128][64] (W_hi + W_lo): W as MN-major B (rows = projections, cols = d).
__device__ __forceinline__ void issue_dxhat(uint32_t d, uint32_t dp, uint32_t whi, uint32_t wlo)
{
    constexpr uint32_t id = idesc_bf16(128, 64, 0, 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sdesc(dp + kk * 32, 16, 1024, LAYOUT_SW128);
        mma_bf16(d, a, sdesc(whi + kk * 2048, TILE, 1024, LAYOUT_SW128), id, kk > 0);
        mma_bf16(d, a, sdesc(wlo + kk * 2048, TILE, 1024, LAYOUT_SW128), id, 1);
    }
}

// D[128][N] (+)= A[128][64] B[N][64]^T, both K-major SW128.
__device__ __forceinline__ void issue_k64(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool acc_first)
{
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
        mma_bf16(d, sdesc(a + kk * 32, 16, 1024, LAYOUT_SW128), sdesc(b + kk * 32, 16, 1024, LAYOUT_SW128), idesc,
                 (kk > 0 || acc_first) ? 1u : 0u);
}

// D[128][N] (+)= A[128][80] B[N][80]^T, both K-major, K split as 64 (SW128) + 16 (SW32).
__device__ __forceinline__ void issue_k80(uint32_t d, uint32_t a128, uint32_t a32, uint32_t b128, uint32_t b32,
                                          uint32_t idesc, bool acc_first)
{
    issue_k64(d, a128, b128, idesc, acc_first);
    mma_bf16(d, sdesc(a32, 16, 256, LAYOUT_SW32), sdesc(b32, 16, 256, LAYOUT_SW32), idesc, 1u);
}

// D[128][N] (+)= A[128][128] B where A = K-major bf16 [128][128] (2 tiles) and B is
// MN-major [K=128 rows][N] spanning N/64 tiles (LBO = TILE).
__device__ __forceinline__ void issue_tt_times(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool acc_first)
{
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_bf16(d, sdesc(a + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024, LAYOUT_SW128),
                 sdesc(b + kk * 2048, TILE, 1024, LAYOUT_SW128), idesc, (kk > 0 || acc_first) ? 1u : 0u);
}

// Masked T x T block from TMEM (row r, columns col0 + 64h ..) to bf16 K-major tile h of dst.
// Adds add_row to every element of the row and add_col[col] per column (either optional)
// before masking; keep_upper keeps column >= row (else column <= row).
__device__ __forceinline__ void mask_block_to_smem(uint32_t tmem, uint32_t col0, int r, int h, bool keep_upper,
                                                   float add_row, const float *add_col, uint8_t *dst)
{
    const uint32_t t = tmem + (lane_base() << 16) + col0 + 64u * h;
    const uint32_t blk = smem_u32(dst) + (uint32_t)h * TILE;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float x[16];
        tmem_ld16(t + 16 * c, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int col = 64 * h + 16 * c + i;
            float y = x[i] + add_row;
            if (add_col) y += add_col[col];
            x[i] = (keep_upper ? (col < r) : (col > r)) ? 0.f : y;
        }
        st_shared_v4(blk + sw128_off(r, 2 * c), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                     pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
        st_shared_v4(blk + sw128_off(r, 2 * c + 1), pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]),
                     pack_bf16x2(x[12], x[13]), pack_bf16x2(x[14], x[15]));
    }
}

// dx = (dX^ - x^ (x^ . dX^)) / max(|x|, eps) for row r, columns 32h .. 32h+31; dX^ from TMEM
// column col0; x re-read from global; the two halves exchange partial dots through xch.
__device__ __forceinline__ void write_dx(uint32_t tmem, uint32_t col0, int r, int h, bool valid, float rawn,
                                         const __nv_bfloat16 *xrow, __nv_bfloat16 *dst, float *xch)
{
    float g[32];
    {
        float a[16], b[16];
        const uint32_t ta = tmem + (lane_base() << 16) + col0 + 32u * h;
        tmem_ld16(ta, a);
        tmem_ld16(ta + 16, b);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            g[i] = a[i];
            g[16 + i] = b[i];
        }
    }
    float x[32];
    float dot = 0.f;
    if (valid) {
        const uint4 *x4 = reinterpret_cast<const uint4 *>(xrow + 32 * h);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const uint4 w = x4[ch];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[8 * ch + 2 * i] = bf16_lo(ws[i]);
                x[8 * ch + 2 * i + 1] = bf16_hi(ws[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) dot = fmaf(x[i], g[i], dot);
    }
    xch[threadIdx.x] = dot;
    __syncthreads();
    dot += xch[threadIdx.x ^ 128];
    if (!valid) return;
    const float n = fmaxf(rawn, kNormEps), inv = 1.f / n;
    const float proj = rawn > kNormEps ? dot * inv * inv : 0.f;  // x^ . dX^ / |x|
    uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * h);
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = (g[8 * ch + i] - x[8 * ch + i] * proj) * inv;
        d4[ch] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                            pack_bf16x2(y[6], y[7]));
    }
}

__device__ __forceinline__ void bseg_bounds(const BwdArgs &a, int seg, int64_t &t0, int64_t &t1)
{
    t0 = (int64_t)seg * a.seg_len;
    t1 = t0 + a.seg_len;
    if (t1 > a.N) t1 = a.N;
}

// Stage one state row (feature m) as a bf16 hi + lo pair of [256][64] SW128 tiles plus its
// ones column in fp32.
__device__ __forceinline__ void stage_state_hilo(const float (&hv)[80], int m, uint8_t *hi, uint8_t *lo, float *col64)
{
    const uint32_t bh_ = smem_u32(hi) + (uint32_t)(m >> 7) * TILE, bl = smem_u32(lo) + (uint32_t)(m >> 7) * TILE;
    const int rr = m & 127;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x0 = hv[8 * ch + 2 * i], x1 = hv[8 * ch + 2 * i + 1];
            wh[i] = pack_bf16x2(x0, x1);
            wl[i] = pack_bf16x2(x0 - bf16_lo(wh[i]), x1 - bf16_hi(wh[i]));
        }
        st_shared_v4(bh_ + sw128_off(rr, ch), wh[0], wh[1], wh[2], wh[3]);
        st_shared_v4(bl + sw128_off(rr, ch), wl[0], wl[1], wl[2], wl[3]);
    }
    col64[m] = hv[64];
}

// A walk's start state row (global fp32 [256][65]) for feature m = 128h + r -> registers,
// then into TMEM (the half's columns).
__device__ __forceinline__ void load_start_row(const float *src_all, int h, int r, uint32_t tm, uint32_t htop,
                                               uint32_t hbot, float (&hv)[80])
{
    const float *src = src_all + (int64_t)(128 * h + r) * DS;
#pragma unroll
    for (int c = 0; c < 80; ++c) hv[c] = c < DS ? src[c] : 0.f;
    const uint32_t t = tm + (lane_base() << 16) + (h ? hbot : htop);
#pragma unroll
    for (int c = 0; c < 5; ++c) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = hv[16 * c + i];
        tmem_st16(t + 16 * c, x);
    }
    tmem_wait_st();
}

// ------------------------------------------------------------------------------------------
// Segment totals of the backward's key side: G_seg = sum_{i in segment} phi(q_i) dY_i^T,
// formed as Phi_Q'^T [dO | c] with Phi_Q' = Phi_Q / den.
// ------------------------------------------------------------------------------------------
namespace aggq_smem {
constexpr uint32_t PHQ = 0;
constexpr uint32_t XQ = PHQ;
constexpr uint32_t DO = PHQ + 4 * TILE;
constexpr uint32_t DC32 = DO + TILE;
constexpr uint32_t WHI = DC32 + 4096;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t ROWC = WLO + 8192;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t BAR = ROWINV + 512;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace aggq_smem

__global__ void __launch_bounds__(NTH, 2) tc_agg_qdy(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace aggq_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        ctl->abort = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, agg_tmem::NCOLS);
    load_w_split(a.W, sm + WHI, sm + WLO);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = ctl->tmem;
    {
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
        const uint32_t t = tm + (lane_base() << 16) + (h ? agg_tmem::HBOT : agg_tmem::HTOP);
#pragma unroll
        for (int c = 0; c < 5; ++c) tmem_st16(t + 16 * c, z);
        tmem_wait_st();
    }
    int64_t t0, t1;
    bseg_bounds(a, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        load_tile_async<NTH>(sm + XQ, a.q + (base + c0) * DH, nv);
        load_tile_async<NTH>(sm + DO, a.dout + (base + c0) * DH, nv);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        row_scalars(sm + DO, a.o + (base + c0) * DH, a.den + base + c0, nv, rowc, rowinv, sm + DC32);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_proj(tm + agg_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        const float inv = 1.f / fmaxf(sqrtf(row_sqnorm(sm + XQ, r)), kNormEps);
        if (!(ok = wait_mma(ctl, phase))) break;
        {
            float u[32], t[32];
            proj_keep(tm, agg_tmem::PROJ, h, inv, a.beta, u, t);
            write_features(t, r, h, r < nv ? rowinv[r] : 0.f, sm + PHQ);
        }
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_state_update(tm, agg_tmem::HTOP, agg_tmem::HBOT, sb + PHQ, sb + DO, sb + DC32);
            mma_commit(&ctl->bar);
        }
        ok = wait_mma(ctl, phase);
    }
    if (ok) {
        float hv[80];
        read_state_row(tm, h ? agg_tmem::HBOT : agg_tmem::HTOP, hv);
        const int m = 128 * h + r;
        float *dst = a.agg_out + (((int64_t)bh * a.nseg + seg) * MF + m) * DS;
#pragma unroll
        for (int c = 0; c < DS; ++c) dst[c] = hv[c];
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, agg_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// dq walk (chunks in order, prefix state H)
// ------------------------------------------------------------------------------------------
namespace bq_smem {
constexpr uint32_t RA = 0;               // k rows at load; Phi_K [128][256] after the features
constexpr uint32_t XK = RA;
constexpr uint32_t PHK = RA;
constexpr uint32_t RB = 4 * TILE;        // q rows + W at load; masked P''; dP~ + W at the end
constexpr uint32_t XQ = RB;
constexpr uint32_t PB = RB;
constexpr uint32_t DP = RB;
constexpr uint32_t WHI = RB + TILE;
constexpr uint32_t WLO = RB + TILE + 8192;
constexpr uint32_t V = RB + 2 * TILE;
constexpr uint32_t ONES = V + TILE;
constexpr uint32_t DO = ONES + 4096;     // dO rows [128][64]
constexpr uint32_t HSHI = DO + TILE;     // staged H[:, :64], bf16 hi  [256][64]
constexpr uint32_t HSLO = HSHI + 2 * TILE;  // and lo
constexpr uint32_t HDEN = HSLO + 2 * TILE;  // H[:, 64] fp32 [256]
constexpr uint32_t ROWC = HDEN + 1024;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t XCH = ROWINV + 512;
constexpr uint32_t BAR = XCH + 1024;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace bq_smem
namespace bq_tmem {
constexpr uint32_t PROJ = 0;   // q 0..63, k 64..127
constexpr uint32_t P = 0;      // [128][128]
constexpr uint32_t DPHI = 0;   // [128][256]
constexpr uint32_t DX = 0;     // [128][64]
constexpr uint32_t HTOP = 256;
constexpr uint32_t HBOT = 336;
constexpr uint32_t NCOLS = 512;
}  // namespace bq_tmem

__global__ void __launch_bounds__(NTH, 1) tc_bwd_q_walk(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace bq_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *xch = reinterpret_cast<float *>(sm + XCH), *hden = reinterpret_cast<float *>(sm + HDEN);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const bool causal = a.causal != 0;
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        ctl->abort = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, bq_tmem::NCOLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = ctl->tmem;
    {
        float hv[80];
        load_start_row(a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride, h, r, tm,
                       bq_tmem::HTOP, bq_tmem::HBOT, hv);
        stage_state_hilo(hv, 128 * h + r, sm + HSHI, sm + HSLO, hden);
    }
    int64_t t0, t1;
    bseg_bounds(a, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        load_tile_async<NTH>(sm + XQ, a.q + (base + c0) * DH, nv);
        load_tile_async<NTH>(sm + DO, a.dout + (base + c0) * DH, nv);
        if (causal) {
            load_tile_async<NTH>(sm + XK, a.k + (base + c0) * DH, nv);
            load_tile_async<NTH>(sm + V, a.v + (base + c0) * DH, nv);
        }
        cp_async_commit();
        load_w_split(a.W, sm + WHI, sm + WLO);
        if (causal) write_ones(sm + ONES, nv);
        cp_async_wait_all();
        __syncthreads();
        row_scalars(sm + DO, a.o + (base + c0) * DH, a.den + base + c0, nv, rowc, rowinv, nullptr);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_proj(tm + bq_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
            if (causal) issue_proj(tm + bq_tmem::PROJ + 64, sb + XK, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        const float raw_q = sqrtf(row_sqnorm(sm + XQ, r));
        const float inv_q = 1.f / fmaxf(raw_q, kNormEps);
        const float inv_k = causal ? 1.f / fmaxf(sqrtf(row_sqnorm(sm + XK, r)), kNormEps) : 0.f;
        const float c_r = rowc[r], invden_r = rowinv[r];
        if (!(ok = wait_mma(ctl, phase))) break;
        float u[32], t[32];
        proj_keep(tm, bq_tmem::PROJ, h, inv_q, a.beta, u, t);
        if (causal) features_half(tm, bq_tmem::PROJ + 64, r, h, inv_k, a.beta, valid, sm + PHK);
        publish_smem();
        if (causal) {
            if (threadIdx.x == 0) {  // P'' = dO V^T
                fence_after_sync();
                issue_k64(tm + bq_tmem::P, sb + DO, sb + V, idesc_bf16(128, 128, 0, 0), false);
                mma_commit(&ctl->bar);
            }
            if (!(ok = wait_mma(ctl, phase))) break;
            mask_block_to_smem(tm, bq_tmem::P, r, h, false, c_r, nullptr, sm + PB);  // v_j.dO_i + c_i, j <= i
            publish_smem();
        }
        if (threadIdx.x == 0) {
            fence_after_sync();
            // D = dO H_prev[:, :64]^T (+ tril(P'') Phi_K)
            issue_k64(tm + bq_tmem::DPHI, sb + DO, sb + HSHI, idesc_bf16(128, 256, 0, 0), false);
            issue_k64(tm + bq_tmem::DPHI, sb + DO, sb + HSLO, idesc_bf16(128, 256, 0, 0), true);
            if (causal) {
                issue_tt_times(tm + bq_tmem::DPHI, sb + PB, sb + PHK, idesc_bf16(128, 256, 0, 1), true);
                issue_state_update(tm, bq_tmem::HTOP, bq_tmem::HBOT, sb + PHK, sb + V, sb + ONES);
            }
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        // dphi = (D + c_i H_prev[:, 64]) / den_i
        features_vjp_half(tm, bq_tmem::DPHI, r, h, a.beta, valid, u, t, hden, c_r, invden_r, sm + DP);
        load_w_split(a.W, sm + WHI, sm + WLO);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_dxhat(tm + bq_tmem::DX, sb + DP, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        write_dx(tm, bq_tmem::DX, r, h, valid, raw_q, a.q + (base + c0 + r) * DH, a.dq + (base + c0 + r) * DH, xch);
        if (causal) {
            float hv[80];
            read_state_row(tm, h ? bq_tmem::HBOT : bq_tmem::HTOP, hv);
            stage_state_hilo(hv, 128 * h + r, sm + HSHI, sm + HSLO, hden);
        }
        publish_smem();
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, bq_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// dk/dv walk (chunks in reverse, suffix state G)
// ------------------------------------------------------------------------------------------
namespace bkv_smem {
constexpr uint32_t PHQ = 0;              // q rows + W at load; Phi_Q'; dP~ + W at the end
constexpr uint32_t XQ = PHQ;
constexpr uint32_t WHI0 = PHQ + 2 * TILE;
constexpr uint32_t WLO0 = WHI0 + 8192;
constexpr uint32_t DP = PHQ;
constexpr uint32_t WHI1 = PHQ + TILE;
constexpr uint32_t WLO1 = WHI1 + 8192;
constexpr uint32_t PHK = PHQ + 4 * TILE; // k rows at load; Phi_K; then masked S'^T and P'
constexpr uint32_t XK = PHK;
constexpr uint32_t STB = PHK;            // tiles 0-1
constexpr uint32_t PPB = PHK + 2 * TILE; // tiles 2-3
constexpr uint32_t V = PHK + 4 * TILE;
constexpr uint32_t ONES = V + TILE;
constexpr uint32_t DO = ONES + 4096;     // dO rows [128][64]
constexpr uint32_t DC32 = DO + TILE;     // c in column 0, [128][16] SW32
constexpr uint32_t GS128 = DC32 + 4096;
constexpr uint32_t GS32 = GS128 + 2 * TILE;
constexpr uint32_t ROWC = GS32 + 8192;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t XCH = ROWINV + 512;
constexpr uint32_t BAR = XCH + 1024;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace bkv_smem
namespace bkv_tmem {
constexpr uint32_t PROJ = 0;    // q 0..63, k 64..127
constexpr uint32_t ST = 0;      // S'^T [128][128]
constexpr uint32_t PP = 128;    // V dO^T [128][128]
constexpr uint32_t DPHI = 0;    // [128][256]
constexpr uint32_t DX = 0;      // [128][64]
constexpr uint32_t GTOP = 256;
constexpr uint32_t GBOT = 336;
constexpr uint32_t DVT = 416;   // dV [128][64]
constexpr uint32_t NCOLS = 512;
}  // namespace bkv_tmem

__global__ void __launch_bounds__(NTH, 1) tc_bwd_kv_walk(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace bkv_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *xch = reinterpret_cast<float *>(sm + XCH);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const bool causal = a.causal != 0;
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        ctl->abort = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, bkv_tmem::NCOLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = ctl->tmem;
    {
        float hv[80];
        load_start_row(a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride, h, r, tm,
                       bkv_tmem::GTOP, bkv_tmem::GBOT, hv);
        stage_state_row(hv, 128 * h + r, sm + GS128, sm + GS32);
    }
    int64_t t0, t1;
    bseg_bounds(a, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    const int64_t nchunks = (t1 - t0 + T - 1) / T;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t ci = nchunks - 1; ci >= 0 && ok; --ci) {
        const int64_t c0 = t0 + ci * T;
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        load_tile_async<NTH>(sm + XK, a.k + (base + c0) * DH, nv);
        load_tile_async<NTH>(sm + V, a.v + (base + c0) * DH, nv);
        if (causal) {
            load_tile_async<NTH>(sm + XQ, a.q + (base + c0) * DH, nv);
            load_tile_async<NTH>(sm + DO, a.dout + (base + c0) * DH, nv);
        }
        cp_async_commit();
        load_w_split(a.W, sm + WHI0, sm + WLO0);
        write_ones(sm + ONES, nv);
        cp_async_wait_all();
        __syncthreads();
        if (causal) row_scalars(sm + DO, a.o + (base + c0) * DH, a.den + base + c0, nv, rowc, rowinv, sm + DC32);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_proj(tm + bkv_tmem::PROJ + 64, sb + XK, sb + WHI0, sb + WLO0);
            if (causal) issue_proj(tm + bkv_tmem::PROJ, sb + XQ, sb + WHI0, sb + WLO0);
            mma_commit(&ctl->bar);
        }
        const float raw_k = sqrtf(row_sqnorm(sm + XK, r));
        const float inv_k = 1.f / fmaxf(raw_k, kNormEps);
        const float inv_q = causal ? 1.f / fmaxf(sqrtf(row_sqnorm(sm + XQ, r)), kNormEps) : 0.f;
        const float invden_r = causal ? rowinv[r] : 0.f;
        if (!(ok = wait_mma(ctl, phase))) break;
        float u[32], t[32];
        proj_keep(tm, bkv_tmem::PROJ + 64, h, inv_k, a.beta, u, t);
        write_features(t, r, h, valid ? 1.f : 0.f, sm + PHK);
        if (causal) {  // Phi_Q' = Phi_Q / den
            float uq[32], tq[32];
            proj_keep(tm, bkv_tmem::PROJ, h, inv_q, a.beta, uq, tq);
            write_features(tq, r, h, invden_r, sm + PHQ);
        }
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            // dV = Phi_K G_next[:, :64]
            {
                constexpr uint32_t id = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    mma_bf16(tm + bkv_tmem::DVT, sdesc(sb + PHK + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024, LAYOUT_SW128),
                             sdesc(sb + GS128 + kk * 2048, TILE, 1024, LAYOUT_SW128), id, kk > 0);
            }
            if (causal) {
                // S'^T = Phi_K Phi_Q'^T ; V dO^T
                constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint32_t off = (kk >> 2) * TILE + (kk & 3) * 32;
                    mma_bf16(tm + bkv_tmem::ST, sdesc(sb + PHK + off, 16, 1024, LAYOUT_SW128),
                             sdesc(sb + PHQ + off, 16, 1024, LAYOUT_SW128), id, kk > 0);
                }
                issue_k64(tm + bkv_tmem::PP, sb + V, sb + DO, id, false);
            }
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        if (causal) {
            mask_block_to_smem(tm, bkv_tmem::ST, r, h, true, 0.f, nullptr, sm + STB);
            mask_block_to_smem(tm, bkv_tmem::PP, r, h, true, 0.f, rowc, sm + PPB);  // v_j.dO_i + c_i, i >= j
        }
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            if (causal)  // dV += triu(S'^T) dO
                issue_tt_times(tm + bkv_tmem::DVT, sb + STB, sb + DO, idesc_bf16(128, 64, 0, 1), true);
            // dPhi_K = [V | 1] G_next^T (+ triu(P') Phi_Q')
            issue_k80(tm + bkv_tmem::DPHI, sb + V, sb + ONES, sb + GS128, sb + GS32, idesc_bf16(128, 256, 0, 0),
                      false);
            if (causal) {
                issue_tt_times(tm + bkv_tmem::DPHI, sb + PPB, sb + PHQ, idesc_bf16(128, 256, 0, 1), true);
                issue_state_update(tm, bkv_tmem::GTOP, bkv_tmem::GBOT, sb + PHQ, sb + DO, sb + DC32);
            }
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        {  // dv, columns 32h .. 32h+31 of row r (TMEM loads are warp-collective: every lane
           // loads, only valid rows store)
            float a0[16], a1[16];
            const uint32_t ta = tm + (lane_base() << 16) + bkv_tmem::DVT + 32u * h;
            tmem_ld16(ta, a0);
            tmem_ld16(ta + 16, a1);
            tmem_wait_ld();
            if (valid) {
                uint4 *d4 = reinterpret_cast<uint4 *>(a.dv + (base + c0 + r) * DH + 32 * h);
                d4[0] = make_uint4(pack_bf16x2(a0[0], a0[1]), pack_bf16x2(a0[2], a0[3]), pack_bf16x2(a0[4], a0[5]),
                                   pack_bf16x2(a0[6], a0[7]));
                d4[1] = make_uint4(pack_bf16x2(a0[8], a0[9]), pack_bf16x2(a0[10], a0[11]),
                                   pack_bf16x2(a0[12], a0[13]), pack_bf16x2(a0[14], a0[15]));
                d4[2] = make_uint4(pack_bf16x2(a1[0], a1[1]), pack_bf16x2(a1[2], a1[3]), pack_bf16x2(a1[4], a1[5]),
                                   pack_bf16x2(a1[6], a1[7]));
                d4[3] = make_uint4(pack_bf16x2(a1[8], a1[9]), pack_bf16x2(a1[10], a1[11]),
                                   pack_bf16x2(a1[12], a1[13]), pack_bf16x2(a1[14], a1[15]));
            }
        }
        features_vjp_half(tm, bkv_tmem::DPHI, r, h, a.beta, valid, u, t, nullptr, 0.f, 1.f, sm + DP);
        load_w_split(a.W, sm + WHI1, sm + WLO1);
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_dxhat(tm + bkv_tmem::DX, sb + DP, sb + WHI1, sb + WLO1);
            mma_commit(&ctl->bar);
        }
        if (!(ok = wait_mma(ctl, phase))) break;
        write_dx(tm, bkv_tmem::DX, r, h, valid, raw_k, a.k + (base + c0 + r) * DH, a.dk + (base + c0 + r) * DH, xch);
        if (causal) {
            float hv[80];
            read_state_row(tm, h ? bkv_tmem::GBOT : bkv_tmem::GTOP, hv);
            stage_state_row(hv, 128 * h + r, sm + GS128, sm + GS32);
        }
        publish_smem();
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, bkv_tmem::NCOLS);
}

// ---- host side ---------------------------------------------------------------------------

inline bool fast_path_ok(race_dtype_t dtype, int d, int L, int P, float tau)
{
    return dtype == RACE_BF16 && d == 64 && L == 16 && P == 4 && tau > 0.f;
}

inline size_t smem_bytes(uint32_t total) { return total + 1024; }

}  // namespace tc
}  // namespace race
