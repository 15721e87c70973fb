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
// Every GEMM above is a tcgen05.mma with operands in shared memory and the accumulator in
// tensor memory; one thread issues them and completion is signalled through an mbarrier,
// polled with a time limit (by one thread before a CTA barrier where other threads' shared
// data is read next, else by every thread).  One CTA of 512 threads walks one segment of
// one (b, h) sequence; the segment aggregates and the bidirectional read-out split the CTA
// into two 256-thread groups that take alternate chunks.  Thread t owns token row r = t % 128 (its TMEM lane) and quarter
// qd = t / 128 of every per-row job: tables 4qd .. 4qd+3 (feature block qd), a quarter of
// the output columns, a quarter of the state rows.
//
// Shared-memory tile formats (bf16):
//   K128 tile: [128 rows][64 cols], 128-byte rows, 16-byte chunks XOR-swizzled by row % 8.
//   Value tile: [rows][16 * natoms] as natoms SW32 atoms of [rows][16] (32-byte rows); the
//     value dimension of V~ = [V | 1], [dO | c] and of the staged states, so that one MMA
//     covers all 80 (or 64) value columns, as the N side (MN-major) or the K side (K-major).
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
constexpr int NTH = 512;    // threads per CTA
constexpr int DH = 64;      // head dimension
constexpr int NPROJ = 64;   // L * P projections
constexpr int MF = 256;     // L * 2^P features
constexpr int DS = 65;      // state row length in global memory (64 + ones column)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far above any chunk's MMA time

constexpr uint32_t TILE = 16384;   // one K128 tile
constexpr uint32_t VA128 = 4096;   // one SW32 atom of 128 rows
constexpr uint32_t VA256 = 8192;   // one SW32 atom of 256 rows

// error word shared by all launches of this path (1 = an MMA or load completion wait timed out)
__device__ int g_tc_error;

// Tensor maps: every [B*H][N][64] bf16 tensor is described as a 3-D tensor (64 columns, N
// rows, B*H heads) so that rows past a head's end read as zero; "k128" boxes are 128 rows x
// 64 columns with the 128-byte swizzle (a K128 tile), "va" boxes 128 rows x 16 columns with
// the 32-byte swizzle (one value-tile atom).
struct Args {
    CUtensorMap tm_q, tm_k, tm_v_va;
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

struct BwdArgs {
    CUtensorMap tm_q, tm_k, tm_o, tm_v_va, tm_do_va;
    const __nv_bfloat16 *q, *k, *v, *o, *dout;
    const float *den, *W;
    const uint8_t *wimg;       // W as the two bf16 K128 tiles (hi, lo) of load_w_split, 16 KB
    float *cbuf;               // c_i = -(dO_i . o_i) per token [BH][N], written by the dq walk
    __nv_bfloat16 *dpq, *dpk;  // optional: dLoss/dp / |x| per q (k) row [BH*N][64], for dW
    __nv_bfloat16 *dq, *dk, *dv;
    const float *state;
    int64_t state_seg_stride;
    float *agg_out;
    int64_t N, seg_len;
    int nseg;
    float beta;
    int causal;
};

struct Ctl {
    uint64_t bar;    // MMA completion
    uint64_t bar_b;  // MMA completion of the second thread group (segment aggregates)
    uint64_t ld[4];  // TMA / bulk load completion, one per buffer set
    uint32_t tmem;
    uint32_t abort;
    uint32_t abort_b;  // the second thread group's (segment aggregates)
};

// ---- small helpers ---------------------------------------------------------------------

__device__ __forceinline__ uint8_t *aligned_base(uint8_t *raw)
{
    const uint32_t a = smem_u32(raw);
    return raw + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ uint32_t lane_base() { return (uint32_t)((threadIdx.x >> 5) & 3) * 32u; }
__device__ __forceinline__ uint32_t tlane(uint32_t tm, uint32_t col) { return tm + (lane_base() << 16) + col; }

// byte offset of 8-element chunk c8 of row `row` in a value tile with `rows` rows
__device__ __forceinline__ uint32_t va_off(int row, int c8, uint32_t rows)
{
    return (uint32_t)(c8 >> 1) * rows * 32u + sw32_off(row, c8 & 1);
}

__device__ __forceinline__ void seg_bounds(int64_t seg_len, int64_t N, int seg, int64_t &t0, int64_t &t1)
{
    t0 = (int64_t)seg * seg_len;
    t1 = t0 + seg_len;
    if (t1 > N) t1 = N;
}

// W [64][64] fp32 -> two K128-format tiles [64][64] of bf16 (hi = round(W), lo = round(W - hi)).
__device__ void load_w_split(const float *W, uint8_t *whi, uint8_t *wlo)
{
    for (int e = threadIdx.x; e < NPROJ * DH / 2; e += NTH) {
        const float2 w = reinterpret_cast<const float2 *>(W)[e];
        const int n = (2 * e) >> 6, c = (2 * e) & 63;
        const uint32_t hi = pack_bf16x2(w.x, w.y);
        const uint32_t lo = pack_bf16x2(w.x - bf16_lo(hi), w.y - bf16_hi(hi));
        const uint32_t off = sw128_off(n, c >> 3) + (c & 7) * 2;
        *reinterpret_cast<uint32_t *>(whi + off) = hi;
        *reinterpret_cast<uint32_t *>(wlo + off) = lo;
    }
}

// ---- asynchronous loads -----------------------------------------------------------------
// Thread 0 issues every TMA / bulk load.  Barrier ctl->ld[b] has at most one load group in
// flight; every thread keeps the same two bit masks, so the parity of the group in flight is
// known everywhere (bit masks rather than counters: b is often a runtime value).
struct Loads {
    uint32_t odd;   // bit b: an odd number of groups has been issued on barrier b
    uint32_t pend;  // bit b: the last group on barrier b has not been waited for
};
__device__ __forceinline__ uint32_t load_parity(const Loads &ld, int b) { return ((ld.odd >> b) & 1u) ^ 1u; }

// Arm barrier b for `bytes` of traffic (by the issuing thread, thread 0 unless given) and
// count the group; the TMA copies that follow, issued by the same thread, complete it.
__device__ __forceinline__ uint64_t *arm_load(Ctl *ctl, Loads &ld, int b, uint32_t bytes,
                                              bool issuer = threadIdx.x == 0)
{
    if (issuer) mbar_expect_tx(&ctl->ld[b], bytes);
    ld.odd ^= 1u << b;
    ld.pend |= 1u << b;
    return &ctl->ld[b];
}

// Rows [row0, row0 + 128) of head bh into a K128 tile (rows past the head's end read as 0).
__device__ __forceinline__ void tma_k128(uint32_t dst, const CUtensorMap *m, int64_t row0, int bh, uint64_t *bar)
{
    tma_load3(dst, m, 0, (int)row0, bh, bar);
}

// Columns 0..63 of rows [row0, row0 + 128) of head bh into atoms 0..3 of a 128-row value tile:
// one box of a 4-D map (16 columns, rows, 4 atoms of 16 columns, heads) whose shared-memory
// image is the four atoms one after another.
__device__ __forceinline__ void tma_va(uint32_t dst, const CUtensorMap *m, int64_t row0, int bh, uint64_t *bar)
{
    tma_load4(dst, m, 0, (int)row0, 0, bh, bar);
}

// Every thread waits (bounded) for the groups in flight on the barriers in `mask`, then the
// CTA syncs; false once the CTA has given up.
__device__ __forceinline__ bool wait_loads(Ctl *ctl, Loads &ld, uint32_t mask)
{
    bool fail = false;
    uint32_t todo = mask & ld.pend;
    while (todo) {
        const int b = __ffs(todo) - 1;
        todo &= todo - 1u;
        if (mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS))
            ld.pend &= ~(1u << b);
        else
            fail = true;
    }
    if (fail) {
        ctl->abort = 1u;
        atomicExch(&g_tc_error, 1);
    }
    __syncthreads();
    return *(volatile uint32_t *)&ctl->abort == 0u;
}

// Every thread waits (bounded) for the groups in flight on the barriers in `mask`, without a
// barrier: each thread observes the completion itself.  A timeout marks the CTA as given up,
// which the next synchronised wait reports.
__device__ __forceinline__ void wait_loads_nosync(Ctl *ctl, Loads &ld, uint32_t mask)
{
    uint32_t todo = mask & ld.pend;
    while (todo) {
        const int b = __ffs(todo) - 1;
        todo &= todo - 1u;
        if (mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS)) {
            ld.pend &= ~(1u << b);
        } else {
            ctl->abort = 1u;
            atomicExch(&g_tc_error, 1);
        }
    }
}

// Thread 0 alone waits for barrier b (data read by the tensor core only); false on timeout,
// after marking the CTA as given up.
__device__ __forceinline__ bool wait_load_t0(Ctl *ctl, Loads &ld, int b)
{
    if (!((ld.pend >> b) & 1u)) return true;
    if (mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS)) {
        ld.pend &= ~(1u << b);
        return true;
    }
    ctl->abort = 1u;
    atomicExch(&g_tc_error, 1);
    return false;
}

// Before exit: thread 0 waits (bounded) for every load group still in flight.
__device__ __forceinline__ void drain_loads(Ctl *ctl, const Loads &ld)
{
    if (threadIdx.x != 0) return;
    for (int b = 0; b < 4; ++b)
        if ((ld.pend >> b) & 1u) mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS);
}

// Atom 4 of a 128-row value tile: column 64 = x (1 for the ones column), zeros elsewhere.
__device__ __forceinline__ void write_col64(uint8_t *tile, int r, float x)
{
    const uint32_t b = smem_u32(tile) + 4 * VA128;
    st_shared_v4(b + sw32_off(r, 0), pack_bf16x2(x, 0.f), 0u, 0u, 0u);
    st_shared_v4(b + sw32_off(r, 1), 0u, 0u, 0u, 0u);
}

// Wait for the MMAs committed to ctl->bar; one thread (`poller`) polls (bounded), all learn the
// outcome.
__device__ __forceinline__ bool wait_mma(Ctl *ctl, uint32_t &phase, unsigned poller = 0)
{
    if (threadIdx.x == poller && ctl->abort == 0u) {
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

// Every thread waits (bounded) for the MMAs committed to ctl->bar itself, with no CTA
// barrier, so no warp waits for another.  Used where what follows reads no shared memory
// that other threads wrote since the last barrier.  A timeout marks the CTA as given up,
// which the next synchronised wait reports (the control flow does not depend on it).
__device__ __forceinline__ void wait_mma_each(Ctl *ctl, uint32_t &phase)
{
    if (*(volatile uint32_t *)&ctl->abort == 0u && !mbar_wait(&ctl->bar, phase & 1u, WAIT_LIMIT_NS)) {
        ctl->abort = 1u;
        atomicExch(&g_tc_error, 1);
    }
    ++phase;
    fence_after_sync();
}

// Hand the shared-memory tiles written so far to the tensor core and sync the CTA.
__device__ __forceinline__ void publish_smem()
{
    fence_smem_async();
    fence_before_sync();
    __syncthreads();
}

// Raw L2 norm of row r of a K128 tile.
__device__ __forceinline__ float row_norm(const uint8_t *tile, int r)
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
    return sqrtf(s);
}

// Per-row scalars of a chunk from the dO rows (value tile) and o rows (K128 tile):
// rowc[r] = c_r = -(dO_r . o_r), rowinv[r] = 1/den_r (0 beyond nvalid); optionally c_r
// into column 64 of the value tile.  One thread per row.
__device__ __forceinline__ void row_scalars(int r, const uint8_t *doc, const uint8_t *o_tile, const float *den,
                                            int nvalid, float *rowc, float *rowinv, uint8_t *doc_col64)
{
    float c = 0.f, inv = 0.f;
    if (r < nvalid) {
        const uint32_t a = smem_u32(doc), ao = smem_u32(o_tile);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 g = ld_shared_v4(a + va_off(r, ch, T)), ov = ld_shared_v4(ao + sw128_off(r, ch));
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
    if (doc_col64) write_col64(doc_col64, r, c);
}

// Per-row scalars of a chunk from the c_i the dq walk stored and den: rowc[r] = c_r,
// rowinv[r] = 1/den_r (both 0 beyond the valid rows); c_r also into column 64 of the value
// tile doc.  One thread per row.
__device__ __forceinline__ void load_row_scalars(int r, bool valid, const float *c_row, const float *den_row,
                                                 float *rowc, float *rowinv, uint8_t *doc)
{
    float c = 0.f, inv = 0.f;
    if (valid) {
        c = *c_row;
        const float dn = *den_row;
        inv = dn != 0.f ? 1.f / dn : 0.f;
    }
    rowc[r] = c;
    rowinv[r] = inv;
    write_col64(doc, r, c);
}

// u = tanh(proj / |x|) and t = tanh(beta u) of this thread's 16 projections (tables
// 4qd .. 4qd+3), read from TMEM columns col0 + 16qd.
__device__ __forceinline__ void proj_tanh(uint32_t tm, uint32_t col0, int qd, float inv_norm, float beta,
                                          float (&u)[16], float (&t)[16])
{
    uint32_t w[16];
    tmem_ld16_nowait(tlane(tm, col0 + 16u * qd), w);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) u[i] = tanh_fast(__uint_as_float(w[i]) * inv_norm);
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = tanh_fast(beta * u[i]);
}

// Corner weights of table l from t: phi_r = prod_p sigmoid(2 beta c_rp u_p) with
// sigmoid(2z) = (1 + tanh z) / 2 -- the softmax over hypercube corners of zh §2.2 in its
// factorised form.  Times `scale`.
__device__ __forceinline__ void corner_weights(const float (&t)[16], int l, float scale, float (&f)[16])
{
    float a[4], b[4];
    {
        const float s1a = 0.5f + 0.5f * t[4 * l], s0a = 0.5f - 0.5f * t[4 * l];
        const float s1b = (0.5f + 0.5f * t[4 * l + 1]) * scale, s0b = (0.5f - 0.5f * t[4 * l + 1]) * scale;
        a[0] = s0a * s0b;
        a[1] = s1a * s0b;
        a[2] = s0a * s1b;
        a[3] = s1a * s1b;
    }
    {
        const float s1c = 0.5f + 0.5f * t[4 * l + 2], s0c = 0.5f - 0.5f * t[4 * l + 2];
        const float s1d = 0.5f + 0.5f * t[4 * l + 3], s0d = 0.5f - 0.5f * t[4 * l + 3];
        b[0] = s0c * s0d;
        b[1] = s1c * s0d;
        b[2] = s0c * s1d;
        b[3] = s1c * s1d;
    }
#pragma unroll
    for (int hi = 0; hi < 4; ++hi)
#pragma unroll
        for (int lo = 0; lo < 4; ++lo) f[4 * hi + lo] = a[lo] * b[hi];
}

// This thread's 64 features (feature block qd) of row r, times `scale`, into the Phi tile.
__device__ __forceinline__ void write_features(const float (&t)[16], int r, int qd, float scale, uint8_t *phi)
{
    const uint32_t blk = smem_u32(phi) + (uint32_t)qd * TILE;
#pragma unroll
    for (int l = 0; l < 4; ++l) {
        float f[16];
        corner_weights(t, l, scale, f);
        st_shared_v4(blk + sw128_off(r, 2 * l), pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        st_shared_v4(blk + sw128_off(r, 2 * l + 1), pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                     pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
    }
}

// This thread's 64 features of row r (feature block qd), times `scale`, as bf16 pairs into
// its TMEM lane at columns col0 + 32qd .. +31 (feature f of the row at column col0 + f/2,
// lower half for even f): the A operand layout of a tensor-memory MMA.
__device__ __forceinline__ void write_features_tmem(const float (&t)[16], int qd, float scale, uint32_t tm,
                                                    uint32_t col0)
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // tables 2h, 2h+1: 16 columns
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float f[16];
            corner_weights(t, 2 * h + e, scale, f);
#pragma unroll
            for (int c = 0; c < 8; ++c) w[8 * e + c] = pack_bf16x2(f[2 * c], f[2 * c + 1]);
        }
        tmem_st16u(tlane(tm, col0 + 32u * qd + 16u * h), w);
    }
}

// Feature-map VJP for this thread's 4 tables: dphi[m] = (D[m] + add_scale * add_vec[m]) * mul
// with D from TMEM columns col0 + 64qd (16 per table) and add_vec (fp32, shared memory,
// indexed by feature) optional; dz = phi (dphi - phi.dphi), du_p = beta sum_r c_rp dz_r,
// dp~ = du (1 - u^2) -> 16 values as bf16 into row r of the DP tile (projections 16qd ..).
__device__ __forceinline__ void features_vjp(uint32_t tm, uint32_t col0, int r, int qd, float beta, bool valid,
                                             const float (&u)[16], const float (&t)[16], const float *add_vec,
                                             float add_scale, float mul, uint8_t *dp_tile,
                                             __nv_bfloat16 *dp_row = nullptr, float dp_scale = 0.f)
{
    uint32_t g[4][16];
#pragma unroll
    for (int l = 0; l < 4; ++l) tmem_ld16_nowait(tlane(tm, col0 + 64u * qd + 16u * l), g[l]);
    tmem_wait_ld();
    float dp[16];
#pragma unroll
    for (int l = 0; l < 4; ++l) {
        float gg[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) gg[c] = __uint_as_float(g[l][c]);
        if (add_vec) {  // 16-byte loads (the vector is read by every thread of a quarter)
            const float4 *av4 = reinterpret_cast<const float4 *>(add_vec + 64 * qd + 16 * l);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 av = av4[c4];
                gg[4 * c4] = fmaf(add_scale, av.x, gg[4 * c4]) * mul;
                gg[4 * c4 + 1] = fmaf(add_scale, av.y, gg[4 * c4 + 1]) * mul;
                gg[4 * c4 + 2] = fmaf(add_scale, av.z, gg[4 * c4 + 2]) * mul;
                gg[4 * c4 + 3] = fmaf(add_scale, av.w, gg[4 * c4 + 3]) * mul;
            }
        }
        // Under phi the sign c_p has mean t_p = tanh(beta u_p), so
        // du_p = beta sum_c c_cp phi_c (g_c - phi.g) = beta (2 A_p - (1 + t_p) phi.g),
        // A_p = sum over the corners with bit p set of phi_c g_c.
        float f[16];
        corner_weights(t, l, 1.f, f);
        float fg[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) fg[c] = f[c] * gg[c];
        float s1[8], s2[4];
#pragma unroll
        for (int c = 0; c < 8; ++c) s1[c] = fg[2 * c] + fg[2 * c + 1];     // pairs over bit 0
#pragma unroll
        for (int c = 0; c < 4; ++c) s2[c] = s1[2 * c] + s1[2 * c + 1];     // quads over bits 0-1
        const float dot = (s2[0] + s2[1]) + (s2[2] + s2[3]);
        float ap[4];
        ap[0] = ((fg[1] + fg[3]) + (fg[5] + fg[7])) + ((fg[9] + fg[11]) + (fg[13] + fg[15]));
        ap[1] = ((s1[1] + s1[3]) + (s1[5] + s1[7]));
        ap[2] = s2[1] + s2[3];
        ap[3] = s2[2] + s2[3];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float uu = u[4 * l + p];
            const float du = beta * (2.f * ap[p] - (1.f + t[4 * l + p]) * dot);
            dp[4 * l + p] = valid ? du * (1.f - uu * uu) : 0.f;
        }
    }
    const uint32_t b = smem_u32(dp_tile);
#pragma unroll
    for (int ch = 0; ch < 2; ++ch)
        st_shared_v4(b + sw128_off(r, 2 * qd + ch), pack_bf16x2(dp[8 * ch], dp[8 * ch + 1]),
                     pack_bf16x2(dp[8 * ch + 2], dp[8 * ch + 3]), pack_bf16x2(dp[8 * ch + 4], dp[8 * ch + 5]),
                     pack_bf16x2(dp[8 * ch + 6], dp[8 * ch + 7]));
    if (dp_row && valid) {  // dLoss/dp / |x| of this row's 16 projections, for the gradient of W
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(dp[2 * k] * dp_scale, dp[2 * k + 1] * dp_scale);
        st_global_v8(dp_row + 16 * qd, pk);
    }
}

// Masked T x T block from TMEM (row r, columns col0 + 32qd ..) to bf16 K128 tile (qd >> 1)
// of dst.  Adds add_row to every element (ADD_ROW) and add_col[col] per column (ADD_COL)
// before masking; UPPER keeps column >= row (else column <= row).  A warp's 32 rows and
// 32 columns lie wholly on one side of the diagonal unless its row block is the quarter's
// own, so only those warps compare element by element; the warps wholly outside the
// kept triangle store zeros without reading TMEM.
template <bool UPPER, bool ADD_ROW, bool ADD_COL>
__device__ __forceinline__ void mask_block(uint32_t tm, uint32_t col0, int r, int qd, float add_row,
                                           const float *add_col, uint8_t *dst)
{
    const uint32_t blk = smem_u32(dst) + (uint32_t)(qd >> 1) * TILE;
    const int rb = (int)((threadIdx.x >> 5) & 3);  // this warp's 32-row block
    const bool all_zero = UPPER ? rb > qd : rb < qd, diag = rb == qd;
    if (all_zero) {
#pragma unroll
        for (int c = 0; c < 4; ++c) st_shared_v4(blk + sw128_off(r, 4 * (qd & 1) + c), 0u, 0u, 0u, 0u);
        return;
    }
    uint32_t w[2][16];
    tmem_ld16_nowait(tlane(tm, col0 + 32u * qd), w[0]);
    tmem_ld16_nowait(tlane(tm, col0 + 32u * qd + 16u), w[1]);
    tmem_wait_ld();
    const int lim = r - 32 * qd;  // column offset of the diagonal within this warp's 32 columns
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float x[8], ac[8];
        if (ADD_COL) {  // 16-byte loads of the per-column terms
            const float4 a0 = reinterpret_cast<const float4 *>(add_col + 32 * qd + 8 * c)[0];
            const float4 a1 = reinterpret_cast<const float4 *>(add_col + 32 * qd + 8 * c)[1];
            ac[0] = a0.x; ac[1] = a0.y; ac[2] = a0.z; ac[3] = a0.w;
            ac[4] = a1.x; ac[5] = a1.y; ac[6] = a1.z; ac[7] = a1.w;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float y = __uint_as_float(w[c >> 1][8 * (c & 1) + i]);
            if (ADD_ROW) y += add_row;
            if (ADD_COL) y += ac[i];
            x[i] = (diag && (UPPER ? (8 * c + i < lim) : (8 * c + i > lim))) ? 0.f : y;
        }
        st_shared_v4(blk + sw128_off(r, 4 * (qd & 1) + c), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                     pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    }
}

// This thread's 40 state columns (row m = 128 (qd & 1) + r of the state, columns
// 40 (qd >> 1) .. +39) from TMEM (state halves at col_top / col_bot).
__device__ __forceinline__ void read_state40(uint32_t tm, uint32_t col_top, uint32_t col_bot, int qd, float (&hv)[40])
{
    const uint32_t base = ((qd & 1) ? col_bot : col_top) + 40u * (qd >> 1);
    uint32_t a[16], b[16], c[8];
    tmem_ld16_nowait(tlane(tm, base), a);
    tmem_ld16_nowait(tlane(tm, base + 16), b);
    tmem_ld8_nowait(tlane(tm, base + 32), c);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        hv[i] = __uint_as_float(a[i]);
        hv[16 + i] = __uint_as_float(b[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) hv[32 + i] = __uint_as_float(c[i]);
}

// Stage those 40 columns as bf16 into a 256-row, 5-atom value tile.
__device__ __forceinline__ void stage40(const float (&hv)[40], int m, int qd, uint8_t *va)
{
    const uint32_t b = smem_u32(va);
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int c8 = 5 * (qd >> 1) + k;
        st_shared_v4(b + va_off(m, c8, 256), pack_bf16x2(hv[8 * k], hv[8 * k + 1]),
                     pack_bf16x2(hv[8 * k + 2], hv[8 * k + 3]), pack_bf16x2(hv[8 * k + 4], hv[8 * k + 5]),
                     pack_bf16x2(hv[8 * k + 6], hv[8 * k + 7]));
    }
}

// Stage as a bf16 hi + lo pair of 4-atom value tiles (columns 0..63) plus column 64 in fp32.
__device__ __forceinline__ void stage40_hilo(const float (&hv)[40], int m, int qd, uint8_t *hi, uint8_t *lo,
                                             float *col64)
{
    const uint32_t bh_ = smem_u32(hi), bl = smem_u32(lo);
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int c8 = 5 * (qd >> 1) + k;
        if (c8 >= 8) break;
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x0 = hv[8 * k + 2 * i], x1 = hv[8 * k + 2 * i + 1];
            wh[i] = pack_bf16x2(x0, x1);
            wl[i] = pack_bf16x2(x0 - bf16_lo(wh[i]), x1 - bf16_hi(wh[i]));
        }
        st_shared_v4(bh_ + va_off(m, c8, 256), wh[0], wh[1], wh[2], wh[3]);
        st_shared_v4(bl + va_off(m, c8, 256), wl[0], wl[1], wl[2], wl[3]);
    }
    if (qd >> 1) col64[m] = hv[24];
}

// Start state: this thread's 40 columns of row m from global fp32 [256][65] into TMEM.
__device__ __forceinline__ void load_state40(const float *src_all, int m, int qd, uint32_t tm, uint32_t col_top,
                                             uint32_t col_bot, float (&hv)[40])
{
    const float *src = src_all + (int64_t)m * DS;
    const int c0 = 40 * (qd >> 1);
#pragma unroll
    for (int i = 0; i < 40; ++i) hv[i] = (c0 + i < DS) ? src[c0 + i] : 0.f;
    const uint32_t base = ((qd & 1) ? col_bot : col_top) + (uint32_t)c0;
    float a[16], b[16], c[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = hv[i];
        b[i] = hv[16 + i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = hv[32 + i];
    tmem_st16(tlane(tm, base), a);
    tmem_st16(tlane(tm, base + 16), b);
    tmem_st8(tlane(tm, base + 32), c);
    tmem_wait_st();
}

__device__ __forceinline__ void zero_state40(uint32_t tm, uint32_t col_top, uint32_t col_bot, int qd)
{
    const uint32_t base = ((qd & 1) ? col_bot : col_top) + 40u * (qd >> 1);
    float z16[16], z8[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) z8[i] = 0.f;
    tmem_st16(tlane(tm, base), z16);
    tmem_st16(tlane(tm, base + 16), z16);
    tmem_st8(tlane(tm, base + 32), z8);
    tmem_wait_st();
}

// This thread's 40 state columns of row m to global fp32 [256][65].
__device__ __forceinline__ void store_state40(const float (&hv)[40], float *dst_all, int m, int qd)
{
    float *dst = dst_all + (int64_t)m * DS;
    const int c0 = 40 * (qd >> 1);
#pragma unroll
    for (int i = 0; i < 40; ++i)
        if (c0 + i < DS) dst[c0 + i] = hv[i];
}

// dx = (dX^ - x^ (x^ . dX^)) / max(|x|, eps) for row r, columns 16qd .. 16qd+15; dX^ from
// TMEM column col0; x from a K128 tile in shared memory if xtile, else the two 16-byte
// words xpre the caller loaded;
// the four quarters exchange partial dots (named barriers 1..4, one per 32-row block).
__device__ __forceinline__ void write_dx(uint32_t tm, uint32_t col0, int r, int qd, bool valid, float rawn,
                                         const uint8_t *xtile, const uint4 *xpre, __nv_bfloat16 *dst, float *xch)
{
    uint32_t w[16];
    tmem_ld16_nowait(tlane(tm, col0 + 16u * qd), w);
    float x[16];
    if (valid) {
        uint4 v4[2];
        if (xtile) {
            v4[0] = ld_shared_v4(smem_u32(xtile) + sw128_off(r, 2 * qd));
            v4[1] = ld_shared_v4(smem_u32(xtile) + sw128_off(r, 2 * qd + 1));
        } else {
            v4[0] = xpre[0];
            v4[1] = xpre[1];
        }
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            const uint32_t ws[4] = {v4[ch].x, v4[ch].y, v4[ch].z, v4[ch].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[8 * ch + 2 * i] = bf16_lo(ws[i]);
                x[8 * ch + 2 * i + 1] = bf16_hi(ws[i]);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
    }
    tmem_wait_ld();
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) dot = fmaf(x[i], __uint_as_float(w[i]), dot);
    xch[threadIdx.x] = dot;
    // the four quarters of this thread's 32 rows are the warps w, w+4, w+8, w+12: they alone meet
    asm volatile("bar.sync %0, 128;" ::"r"(1 + (int)((threadIdx.x >> 5) & 3)) : "memory");
    dot = xch[r] + xch[128 + r] + xch[256 + r] + xch[384 + r];
    if (!valid) return;
    const float n = fmaxf(rawn, kNormEps), inv = 1.f / n;
    const float pj = rawn > kNormEps ? dot * inv * inv : 0.f;  // x^ . dX^ / |x|
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = (__uint_as_float(w[i]) - x[i] * pj) * inv;
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(y[2 * k], y[2 * k + 1]);
    st_global_v8(dst + 16 * qd, pk);
}

// 16 consecutive TMEM columns of row r (col0 + 16qd) as bf16 to global (16 values), scaled.
__device__ __forceinline__ void store_row16(uint32_t tm, uint32_t col0, int qd, bool valid, float scale,
                                            __nv_bfloat16 *dst)
{
    uint32_t w[16];
    tmem_ld16_nowait(tlane(tm, col0 + 16u * qd), w);
    tmem_wait_ld();
    if (!valid) return;
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(__uint_as_float(w[2 * k]) * scale, __uint_as_float(w[2 * k + 1]) * scale);
    st_global_v8(dst + 16 * qd, pk);
}

// out = Y[:, 16 qq ..] / Y[:, 64] for the quarters qq of `qds` (n of them) of row r, with Y at
// TMEM column ycol: the quarters' columns and column 64 come in with one TMEM round trip.
// Returns den = Y[r, 64].
template <int NQ>
__device__ __forceinline__ float store_out_quarters(uint32_t tm, uint32_t ycol, const int (&qds)[NQ], bool valid,
                                                   __nv_bfloat16 *dst)
{
    uint32_t w[NQ][16], dn[8];
#pragma unroll
    for (int i = 0; i < NQ; ++i) tmem_ld16_nowait(tlane(tm, ycol + 16u * qds[i]), w[i]);
    tmem_ld8_nowait(tlane(tm, ycol + 64u), dn);
    tmem_wait_ld();
    const float d = __uint_as_float(dn[0]);
    if (valid) {
        const float2 sc = dup2(d != 0.f ? 1.f / d : 0.f);
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float2 y = mul2(make_float2(__uint_as_float(w[i][2 * k]), __uint_as_float(w[i][2 * k + 1])), sc);
                pk[k] = pack_bf16x2(y.x, y.y);
            }
            st_global_v8(dst + 16 * qds[i], pk);
        }
    }
    return d;
}

// ---- MMA issue helpers (one thread) ------------------------------------------------------
// Descriptors are built once and advanced by adding (byte offset >> 4) to the start field.

// proj[128][64] = X[128][64] (W_hi + W_lo)^T       (X, W: K128 tiles, K-major)
__device__ __forceinline__ void issue_proj(uint32_t d, uint32_t x, uint32_t whi, uint32_t wlo)
{
    constexpr uint32_t id = idesc_bf16(128, 64, 0, 0);
    const uint64_t ax = sdesc(x, 16, 1024, LAYOUT_SW128), bh = sdesc(whi, 16, 1024, LAYOUT_SW128),
                   bl = sdesc(wlo, 16, 1024, LAYOUT_SW128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        mma_bf16(d, ax + 2 * kk, bh + 2 * kk, id, kk > 0);
        mma_bf16(d, ax + 2 * kk, bl + 2 * kk, id, 1);
    }
}

// D[128][N] (+)= A[128][K=256] B^T, A K-major (4 K128 tiles), B K-major rows = N (4 tiles).
__device__ __forceinline__ void issue_k256_kk(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool acc_first)
{
    const uint64_t da = sdesc(a, 16, 1024, LAYOUT_SW128), db = sdesc(b, 16, 1024, LAYOUT_SW128);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
        const uint32_t off = ((kk >> 2) * TILE + (kk & 3) * 32) >> 4;
        mma_bf16(d, da + off, db + off, idesc, (kk > 0 || acc_first) ? 1u : 0u);
    }
}

// D[128][N] (+)= A[128][K=256] B, A K-major (4 K128 tiles), B = value tile MN-major with
// 256 K-rows (atom stride VA256, N = 16 * natoms).
__device__ __forceinline__ void issue_k256_va(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool acc_first)
{
    const uint64_t da = sdesc(a, 16, 1024, LAYOUT_SW128), db = sdesc(b, VA256, 256, LAYOUT_SW32);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
        const uint32_t off = ((kk >> 2) * TILE + (kk & 3) * 32) >> 4;
        mma_bf16(d, da + off, db + kk * (512 >> 4), idesc, (kk > 0 || acc_first) ? 1u : 0u);
    }
}

// D[128][N] (+)= A[128][K=256] B^T with A in TMEM (128 columns of bf16 pairs from a_tmem) and
// B K-major rows = N (4 K128 tiles).
__device__ __forceinline__ void issue_k256_tkk(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc)
{
    const uint64_t db = sdesc(b, 16, 1024, LAYOUT_SW128);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
        const uint32_t off = ((kk >> 2) * TILE + (kk & 3) * 32) >> 4;
        mma_bf16_ts(d, a_tmem + 8u * kk, db + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// D[128][N] (+)= A[128][K=256] B with A in TMEM and B a value tile MN-major with 256 K-rows
// (atom stride VA256, N = 16 * natoms).
__device__ __forceinline__ void issue_k256_tva(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc)
{
    const uint64_t db = sdesc(b, VA256, 256, LAYOUT_SW32);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) mma_bf16_ts(d, a_tmem + 8u * kk, db + kk * (512 >> 4), idesc, kk > 0 ? 1u : 0u);
}

// D[128][N] (+)= A[128][K=128] B with A K-major (2 K128 tiles, a_mn = 0) or MN-major
// (M spans tiles at LBO = TILE, a_mn = 1), B = 128-row value tile MN-major (N = 16 natoms).
__device__ __forceinline__ void issue_k128_va(uint32_t d, uint32_t a, int a_mn, uint32_t b, uint32_t idesc,
                                              bool acc_first)
{
    const uint64_t da = a_mn ? sdesc(a, TILE, 1024, LAYOUT_SW128) : sdesc(a, 16, 1024, LAYOUT_SW128);
    const uint64_t db = sdesc(b, VA128, 256, LAYOUT_SW32);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = a_mn ? (kk * 2048) >> 4 : ((kk >> 2) * TILE + (kk & 3) * 32) >> 4;
        mma_bf16(d, da + aoff, db + kk * (512 >> 4), idesc, (kk > 0 || acc_first) ? 1u : 0u);
    }
}

// D[128][N] (+)= A[128][K=128] B, A K-major (2 K128 tiles), B MN-major K128 tiles spanning
// N / 64 tiles (LBO = TILE), K-rows = 128.
__device__ __forceinline__ void issue_k128_k128mn(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc,
                                                  bool acc_first)
{
    const uint64_t da = sdesc(a, 16, 1024, LAYOUT_SW128), db = sdesc(b, TILE, 1024, LAYOUT_SW128);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = ((kk >> 2) * TILE + (kk & 3) * 32) >> 4;
        mma_bf16(d, da + aoff, db + kk * (2048 >> 4), idesc, (kk > 0 || acc_first) ? 1u : 0u);
    }
}

// D[128][N] (+)= A B^T with A = value tile K-major (rows 128, atom stride arows*32), B = value
// tile K-major (rows = N, atom stride brows*32), K = 16 * natoms.
__device__ __forceinline__ void issue_va_va(uint32_t d, uint32_t a, uint32_t arows, uint32_t b, uint32_t brows,
                                            int natoms, uint32_t idesc, bool acc_first)
{
    const uint64_t da = sdesc(a, 16, 256, LAYOUT_SW32), db = sdesc(b, 16, 256, LAYOUT_SW32);
    for (int kk = 0; kk < natoms; ++kk)
        mma_bf16(d, da + kk * ((arows * 32) >> 4), db + kk * ((brows * 32) >> 4), idesc,
                 (kk > 0 || acc_first) ? 1u : 0u);
}

// state (two halves of 128 rows) += Phi^T [B], Phi = [128 tokens][256] K128 tiles read
// MN-major, B = 128-row value tile (N = 80) MN-major.
__device__ __forceinline__ void issue_state_update(uint32_t tm, uint32_t htop, uint32_t hbot, uint32_t phi,
                                                   uint32_t va)
{
    constexpr uint32_t id = idesc_bf16(128, 80, 1, 1);
    issue_k128_va(tm + htop, phi, 1, va, id, true);
    issue_k128_va(tm + hbot, phi + 2 * TILE, 1, va, id, true);
}

// ==========================================================================================
// Forward
// ==========================================================================================

namespace agg_smem {  // two thread groups, each with its own rows, features and value tile
constexpr uint32_t X = 0;                    // k or q rows [128][64]
constexpr uint32_t PHI = TILE;               // Phi [128][256]
constexpr uint32_t VA = 5 * TILE;            // value tile [128][80] (5 atoms)
constexpr uint32_t GROUP = VA + 5 * VA128;   // bytes per group (a multiple of 1024)
constexpr uint32_t WHI = 2 * GROUP;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t RN = WLO + 8192;          // row norms [2][128]
constexpr uint32_t ROWC = RN + 1024;         // c_i [2][128]
constexpr uint32_t ROWINV = ROWC + 1024;     // 1 / den_i [2][128]
constexpr uint32_t BAR = ROWINV + 1024;
constexpr uint32_t VBAR = BAR + 64;          // per group: its state update is done (value tile free)
constexpr uint32_t TOTAL = VBAR + 64;
constexpr uint32_t RED = GROUP;              // at the end: group 1's state, fp32 [256][80]
static_assert(256 * 80 * 4 <= GROUP, "reduction buffer");
}  // namespace agg_smem
namespace agg_tmem {  // per group, at 256 * group
constexpr uint32_t PROJ = 0;
constexpr uint32_t HTOP = 64;
constexpr uint32_t HBOT = 144;
constexpr uint32_t NCOLS = 512;
}  // namespace agg_tmem

namespace fwd_smem {
constexpr uint32_t PHK = 0;                  // Phi_K [128][256]
constexpr uint32_t SB = 4 * TILE;            // masked S as bf16 [128][128]: 2 tiles
constexpr uint32_t XQ = SB + 2 * TILE;       // q rows of the next chunk (loaded a chunk ahead)
constexpr uint32_t XK = XQ + TILE;           // k rows likewise
constexpr uint32_t VA0 = XK + TILE;          // [V | 1] [128][80], two buffers (chunk parity)
constexpr uint32_t VA1 = VA0 + 5 * VA128;
constexpr uint32_t HS = VA1 + 5 * VA128;     // staged H [256][80] value tile (5 atoms)
constexpr uint32_t WHI = HS + 5 * VA256;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t RN = WLO + 8192;          // q norms [128], k norms [128]
constexpr uint32_t BAR = RN + 1024;
constexpr uint32_t FB = BAR + 64;            // the walk's own mbarriers (FwdBars)
constexpr uint32_t TOTAL = FB + 128;
}  // namespace fwd_smem
namespace fwd_tmem {
constexpr uint32_t PROJ = 0;    // [128][64] q projections, [128][64] k projections at +64
constexpr uint32_t S = 0;       // [128][128] (reuses PROJ once the features are formed)
constexpr uint32_t Y = 128;     // [128][80]
constexpr uint32_t HTOP = 208;  // H rows 0..127   [128][80]
constexpr uint32_t HBOT = 288;  // H rows 128..255 [128][80]
constexpr uint32_t PHQ = 368;   // Phi_Q [128][256] as bf16 pairs (128 columns): the A operand
constexpr uint32_t NCOLS = 512;
}  // namespace fwd_tmem

// Common prologue: barrier, TMEM allocation, W tiles.
__device__ __forceinline__ uint32_t kernel_setup(Ctl *ctl, uint32_t ncols, const float *W, uint8_t *whi,
                                                 uint8_t *wlo)
{
    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar, 1);
        mbar_init(&ctl->bar_b, 1);
        for (int b = 0; b < 4; ++b) mbar_init(&ctl->ld[b], 1);
        ctl->abort = 0;
        ctl->abort_b = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&ctl->tmem, ncols);
    if (whi) load_w_split(W, whi, wlo);
    fence_smem_async();  // W is read by the tensor core
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    return ctl->tmem;
}

__device__ __forceinline__ void kernel_teardown(uint32_t tm, uint32_t ncols)
{
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, ncols);
}

// Barrier of one 256-thread group (named barrier 1 + g).
__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// ------------------------------------------------------------------------------------------
// Segment totals.  MODE 0: H_seg = sum_j phi(k_j) [v_j, 1]^T (the bucket statistics A, B of
// zh §2.2 over the segment).  MODE 1: G_seg = sum_i phi(q_i) dY_i^T = Phi_Q'^T [dO | c] with
// Phi_Q' = Phi_Q / den (the backward's key-side statistics).   grid: nseg x BH
// The CTA's two groups of 256 threads take the segment's chunks alternately, each with its
// own tiles, TMEM accumulator and barriers, so that one group's MMA and load waits overlap
// the other group's feature math; the two partial sums are added at the end.  A group's
// state update is not committed on its own: the next chunk's projection commit reports it
// too, since MMAs complete in issue order.  Thread (r, h) of a group owns token row r and
// quarters 2h, 2h+1 of the per-row work.
// ------------------------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(NTH, 1) tc_agg(const __grid_constant__ BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace agg_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int g = threadIdx.x >> 8, gt = threadIdx.x & 255;
    const int r = gt & 127, h = gt >> 7;
    const bool leader = gt == 0;
    float *rn = reinterpret_cast<float *>(sm + RN) + 128 * g;
    float *rowc = reinterpret_cast<float *>(sm + ROWC) + 128 * g;
    float *rowinv = reinterpret_cast<float *>(sm + ROWINV) + 128 * g;
    const uint32_t sb = smem_u32(sm), gb = sb + (uint32_t)g * GROUP;
    uint8_t *xg = sm + g * GROUP + X, *vag = sm + g * GROUP + VA;
    uint64_t *mbar = g ? &ctl->bar_b : &ctl->bar;
    // each group decides on its own flag, read only after its own barrier, so that all its
    // threads leave the loop together; the CTA checks both flags after the loops
    volatile uint32_t *gabort = g ? &ctl->abort_b : &ctl->abort;
    const CUtensorMap *xmap = MODE == 0 ? &a.tm_k : &a.tm_q;
    const CUtensorMap *vmap = MODE == 0 ? &a.tm_v_va : &a.tm_do_va;
    uint64_t *vbar = reinterpret_cast<uint64_t *>(sm + VBAR) + g;
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t *>(sm + VBAR), 1);
        mbar_init(reinterpret_cast<uint64_t *>(sm + VBAR) + 1, 1);
    }
    const uint32_t tm = kernel_setup(ctl, agg_tmem::NCOLS, a.W, sm + WHI, sm + WLO);
    const uint32_t tg = tm + 256u * g;  // this group's TMEM columns
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) zero_state40(tg, agg_tmem::HTOP, agg_tmem::HBOT, 2 * h + qq);
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};  // barriers 2g (rows) and 2g + 1 (values) of this group
    auto load_x = [&](int64_t c) {
        uint64_t *bar = arm_load(ctl, ld, 2 * g, TILE, leader);
        if (leader) tma_k128(gb + X, xmap, c, bh, bar);
    };
    auto load_v = [&](int64_t c) {
        uint64_t *bar = arm_load(ctl, ld, 2 * g + 1, TILE, leader);
        if (leader) tma_va(gb + VA, vmap, c, bh, bar);
    };
    // bounded wait on this group's MMA barrier, then the group syncs
    auto wait_group_mma = [&]() {
        if (leader && *gabort == 0u && !mbar_wait(mbar, phase & 1u, WAIT_LIMIT_NS)) {
            *gabort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        ++phase;
        group_sync(g);
        fence_after_sync();
        return *gabort == 0u;
    };
    auto wait_group_load = [&](int b) {
        bool fail = false;
        if ((ld.pend >> b) & 1u) {
            if (mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS))
                ld.pend &= ~(1u << b);
            else
                fail = true;
        }
        if (fail) {
            *gabort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        group_sync(g);
        return *gabort == 0u;
    };
    auto publish_group = [&]() {
        fence_smem_async();
        fence_before_sync();
        group_sync(g);
    };
    int64_t c0 = t0 + (int64_t)g * T;  // this group's chunks: every other one of the segment
    if (c0 < t1) {
        load_x(c0);
        load_v(c0);
    }
    bool pending = false;  // a state update of this group is in flight
    uint32_t vphase = 0;   // phase of vbar (waited on by the leader)
    for (; c0 < t1 && ok; c0 += 2 * T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const int64_t cn = c0 + 2 * T;  // this group's next chunk
        if (pending) {  // the value tile comes in as soon as the last state update has read it
            if (leader && *gabort == 0u && !mbar_wait(vbar, vphase & 1u, WAIT_LIMIT_NS)) {
                *gabort = 1u;
                atomicExch(&g_tc_error, 1);
            }
            ++vphase;
            load_v(c0);
        }
        if (!(ok = wait_group_load(2 * g))) break;
        if (leader) {  // the projection runs while the row norms are formed
            fence_after_sync();
            issue_proj(tg + agg_tmem::PROJ, gb + X, sb + WHI, sb + WLO);
            mma_commit(mbar);
        }
        if (h == 0) rn[r] = row_norm(xg, r);
        if (MODE == 1 && h == 1) {  // c_i and 1/den_i (0 beyond the valid rows)
            float c = 0.f, inv = 0.f;
            if (r < nv) {
                c = a.cbuf[base + c0 + r];
                const float dn = a.den[base + c0 + r];
                inv = dn != 0.f ? 1.f / dn : 0.f;
            }
            rowc[r] = c;
            rowinv[r] = inv;
        }
        if (!(ok = wait_group_mma())) break;
        pending = false;
        if (cn < t1) load_x(cn);  // the rows are consumed: the next chunk's rows come in during the features
        if (h == 1) write_col64(vag, r, MODE == 0 ? (r < nv ? 1.f : 0.f) : rowc[r]);  // [v | 1] or [dO | c]
        {
            const float inv = 1.f / fmaxf(rn[r], kNormEps);
            const float sc = r < nv ? (MODE == 0 ? 1.f : rowinv[r]) : 0.f;
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                float u[16], t[16];
                proj_tanh(tg, agg_tmem::PROJ, 2 * h + qq, inv, a.beta, u, t);
                write_features(t, r, 2 * h + qq, sc, sm + g * GROUP + PHI);
            }
        }
        if (!(ok = wait_group_load(2 * g + 1))) break;  // this chunk's values (group-synced)
        publish_group();
        if (leader) {
            fence_after_sync();
            issue_state_update(tg, agg_tmem::HTOP, agg_tmem::HBOT, gb + PHI, gb + VA);
            mma_commit(vbar);
        }
        pending = true;
    }
    if (pending && ok) {  // the group's last state update
        if (leader && *gabort == 0u && !mbar_wait(vbar, vphase & 1u, WAIT_LIMIT_NS)) {
            *gabort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        group_sync(g);
        fence_after_sync();
        ok = *gabort == 0u;
    }
    drain_loads(ctl, ld);  // thread 0 only; group 1's loads are drained by its own leader
    if (g == 1 && leader)
        for (int b = 2; b < 4; ++b)
            if ((ld.pend >> b) & 1u) mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS);
    __syncthreads();
    if (ctl->abort == 0u && ctl->abort_b == 0u) {  // H = group 0's sum + group 1's sum
        float *red = reinterpret_cast<float *>(sm + RED);
        if (g == 1) {
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int qd = 2 * h + qq;
                float hv[40];
                read_state40(tg, agg_tmem::HTOP, agg_tmem::HBOT, qd, hv);
                float *dst = red + (128 * (qd & 1) + r) * 80 + 40 * (qd >> 1);
#pragma unroll
                for (int i = 0; i < 40; ++i) dst[i] = hv[i];
            }
        }
        __syncthreads();
        if (g == 0) {
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int qd = 2 * h + qq;
                float hv[40];
                read_state40(tg, agg_tmem::HTOP, agg_tmem::HBOT, qd, hv);
                const float *src = red + (128 * (qd & 1) + r) * 80 + 40 * (qd >> 1);
#pragma unroll
                for (int i = 0; i < 40; ++i) hv[i] += src[i];
                store_state40(hv, a.agg_out + ((int64_t)bh * a.nseg + seg) * MF * DS, 128 * (qd & 1) + r, qd);
            }
        }
    }
    kernel_teardown(tm, agg_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// Causal walk (Algorithm 2, zh §2.3).  grid: nseg x BH, NTH + 32 threads.
// Phi_Q lives in tensor memory as the A operand of S = Phi_Q Phi_K^T and Y = Phi_Q H_prev, so
// shared memory holds dedicated q / k row tiles and two [V | 1] tiles: every load of the
// next chunk is issued a whole chunk ahead.  Threads 0..NTH-1 compute; one lane of the last
// warp issues every TMA load and MMA (an issuing thread is held until the tensor core's queue
// takes its last MMA, so no computing warp issues).  The two sides hand over through
// mbarriers: the computing warps arrive (one lane per warp) when a tile is ready, the issuer
// commits MMAs to barriers the computing threads poll.  The next chunk's projections are
// issued as soon as the mask has read S (they share its tensor-memory columns), so they run
// under this chunk's S V~ product and read-out.
// ------------------------------------------------------------------------------------------
struct FwdBars {
    uint64_t rows, v[2];                     // TMA: q and k rows; value tile p
    uint64_t proj, s, sv;                    // MMA commits
    uint64_t norm, phiq, phik, sbar, done;   // the computing warps' hand-overs (16 arrivals)
};
static_assert(sizeof(FwdBars) <= 128, "walk barriers");

__global__ void __launch_bounds__(NTH + 32, 1) tc_fwd_walk(const __grid_constant__ Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace fwd_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    FwdBars *fb = reinterpret_cast<FwdBars *>(sm + FB);
    float *rn = reinterpret_cast<float *>(sm + RN);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const bool issuer_warp = threadIdx.x >= NTH;
    const int r = threadIdx.x & 127, qd = (threadIdx.x >> 7) & 3;
    const uint32_t sb = smem_u32(sm);
    if (threadIdx.x == 0) {
        mbar_init(&fb->rows, 1);
        mbar_init(&fb->v[0], 1);
        mbar_init(&fb->v[1], 1);
        mbar_init(&fb->proj, 1);
        mbar_init(&fb->s, 1);
        mbar_init(&fb->sv, 1);
        mbar_init(&fb->norm, NTH / 32);
        mbar_init(&fb->phiq, NTH / 32);
        mbar_init(&fb->phik, NTH / 32);
        mbar_init(&fb->sbar, NTH / 32);
        mbar_init(&fb->done, NTH / 32);
    }
    const uint32_t tm = kernel_setup(ctl, fwd_tmem::NCOLS, a.W, sm + WHI, sm + WLO);
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    volatile uint32_t *abort_flag = &ctl->abort;
    // bounded wait on a barrier phase; a timeout marks the CTA as given up (every later wait
    // then returns at once) and the walk loops below leave
    auto wait = [&](uint64_t *bar, uint32_t &ph) {
        bool good = *abort_flag == 0u && mbar_wait(bar, ph & 1u, WAIT_LIMIT_NS);
        ++ph;
        if (!good && *abort_flag == 0u) {
            *abort_flag = 1u;
            atomicExch(&g_tc_error, 1);
        }
        return *abort_flag == 0u;
    };
    if (issuer_warp) {
        if (threadIdx.x == NTH) {  // the issuing lane
            // phases and pending flags as scalars: arrays indexed by the chunk parity would live in
            // local memory
            uint32_t ph_rows = 0, ph_v0 = 0, ph_v1 = 0, ph_proj = 0, ph_norm = 0, ph_phiq = 0, ph_phik = 0,
                     ph_sb = 0, ph_done = 0;
            auto issue_rows = [&](int64_t c) {
                mbar_expect_tx(&fb->rows, 2u * TILE);
                tma_k128(sb + XQ, &a.tm_q, c, bh, &fb->rows);
                tma_k128(sb + XK, &a.tm_k, c, bh, &fb->rows);
            };
            auto issue_v = [&](int64_t c, int p) {
                mbar_expect_tx(&fb->v[p], TILE);
                tma_va(sb + (p ? VA1 : VA0), &a.tm_v_va, c, bh, &fb->v[p]);
            };
            auto issue_proj_of = [&](int p) {  // the rows and value tile p of the chunk have landed
                if (!wait(&fb->rows, ph_rows) || !(p ? wait(&fb->v[1], ph_v1) : wait(&fb->v[0], ph_v0))) return false;
                fence_after_sync();
                issue_proj(tm + fwd_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
                issue_proj(tm + fwd_tmem::PROJ + 64, sb + XK, sb + WHI, sb + WLO);
                mma_commit(&fb->proj);
                return true;
            };
            int rows_pending = 0, v_pend0 = 0, v_pend1 = 0;  // TMA groups issued, not yet waited for
            bool ok = true;
            if (t0 < t1) {
                issue_rows(t0);
                issue_v(t0, 0);
                rows_pending = 1;
                v_pend0 = 1;
                ok = issue_proj_of(0);
                rows_pending = v_pend0 = 0;
            }
            int par = 0;
            for (int64_t c0 = t0; c0 < t1 && ok; c0 += T, par ^= 1) {
                const bool more = c0 + T < t1;
                // the q / k rows are read by the projections and the row norms
                if (!(ok = wait(&fb->norm, ph_norm) && wait(&fb->proj, ph_proj))) break;
                if (more) {
                    issue_rows(c0 + T);
                    issue_v(c0 + T, par ^ 1);  // last read by the previous chunk's MMAs
                    rows_pending = 1;
                    if (par) v_pend0 = 1;
                    else v_pend1 = 1;
                }
                if (!(ok = wait(&fb->phiq, ph_phiq))) break;
                fence_after_sync();  // Y = Phi_Q H_prev
                issue_k256_tva(tm + fwd_tmem::Y, tm + fwd_tmem::PHQ, sb + HS, idesc_bf16(128, 80, 0, 1));
                if (!(ok = wait(&fb->phik, ph_phik))) break;
                fence_after_sync();  // S = Phi_Q Phi_K^T, then H += Phi_K^T V~
                issue_k256_tkk(tm + fwd_tmem::S, tm + fwd_tmem::PHQ, sb + PHK, idesc_bf16(128, 128, 0, 0));
                mma_commit(&fb->s);
                issue_state_update(tm, fwd_tmem::HTOP, fwd_tmem::HBOT, sb + PHK, sb + (par ? VA1 : VA0));
                if (!(ok = wait(&fb->sbar, ph_sb))) break;
                fence_after_sync();  // Y += tril(S) V~
                issue_k128_va(tm + fwd_tmem::Y, sb + SB, 0, sb + (par ? VA1 : VA0), idesc_bf16(128, 80, 0, 1), true);
                mma_commit(&fb->sv);
                if (more) {  // the next chunk's projections: S has been read, the rows are (being) loaded
                    ok = issue_proj_of(par ^ 1);
                    rows_pending = 0;
                    if (par) v_pend0 = 0;
                    else v_pend1 = 0;
                    if (!ok) break;
                }
                if (!(ok = wait(&fb->done, ph_done))) break;
            }
            // leave nothing in flight: every MMA issued has been committed; wait (bounded) for
            // the last commit and for any load group not yet waited for
            mma_commit(&fb->proj);
            mbar_wait(&fb->proj, ph_proj & 1u, WAIT_LIMIT_NS);
            if (rows_pending) mbar_wait(&fb->rows, ph_rows & 1u, WAIT_LIMIT_NS);
            if (v_pend0) mbar_wait(&fb->v[0], ph_v0 & 1u, WAIT_LIMIT_NS);
            if (v_pend1) mbar_wait(&fb->v[1], ph_v1 & 1u, WAIT_LIMIT_NS);
        }
    } else {
        {  // start state: fp32 master into TMEM, bf16 copy into the staging tile
            float hv[40];
            load_state40(a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride, 128 * (qd & 1) + r,
                         qd, tm, fwd_tmem::HTOP, fwd_tmem::HBOT, hv);
            stage40(hv, 128 * (qd & 1) + r, qd, sm + HS);
        }
        fence_smem_async();
        fence_before_sync();
        asm volatile("bar.sync 1, %0;" ::"n"(NTH) : "memory");  // the staged state before the first Y
        uint32_t ph_rows = 0, ph_proj = 0, ph_s = 0, ph_sv = 0;
        const bool elect = (threadIdx.x & 31) == 0;
        auto hand_over = [&](uint64_t *bar) {  // this warp's writes are complete: one arrival
            __syncwarp();
            if (elect) mbar_arrive(bar);
        };
        int par = 0;
        bool ok = true;
        for (int64_t c0 = t0; c0 < t1 && ok; c0 += T, par ^= 1) {
            const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
            const bool valid = r < nv;
            if (!(ok = wait(&fb->rows, ph_rows))) break;
            if (qd == 0) rn[r] = row_norm(sm + XQ, r);
            if (qd == 1) rn[128 + r] = row_norm(sm + XK, r);
            if (qd == 2) write_col64(sm + (par ? VA1 : VA0), r, valid ? 1.f : 0.f);
            fence_smem_async();
            hand_over(&fb->norm);
            if (!(ok = wait(&fb->proj, ph_proj))) break;
            asm volatile("bar.sync 1, %0;" ::"n"(NTH) : "memory");  // the row norms
            {  // Phi_Q into tensor memory
                float u[16], t[16];
                proj_tanh(tm, fwd_tmem::PROJ, qd, 1.f / fmaxf(rn[r], kNormEps), a.beta, u, t);
                write_features_tmem(t, qd, valid ? 1.f : 0.f, tm, fwd_tmem::PHQ);
            }
            tmem_wait_st();
            fence_before_sync();
            hand_over(&fb->phiq);
            {
                float u[16], t[16];
                proj_tanh(tm, fwd_tmem::PROJ + 64, qd, 1.f / fmaxf(rn[128 + r], kNormEps), a.beta, u, t);
                write_features(t, r, qd, valid ? 1.f : 0.f, sm + PHK);
            }
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->phik);
            if (!(ok = wait(&fb->s, ph_s))) break;
            fence_after_sync();
            mask_block<false, false, false>(tm, fwd_tmem::S, r, qd, 0.f, nullptr, sm + SB);  // j <= i
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->sbar);
            if (!(ok = wait(&fb->sv, ph_sv))) break;
            fence_after_sync();
            {  // out = Y[:, :64] / Y[:, 64]: columns 16qd .. 16qd+15 of row r
                const int qds[1] = {qd};
                const float d = store_out_quarters<1>(tm, fwd_tmem::Y, qds, valid, a.out + (base + c0 + r) * DH);
                if (qd == 0 && valid && a.den) a.den[base + c0 + r] = d;
            }
            {  // stage the updated state for the next chunk's read-out
                float hv[40];
                read_state40(tm, fwd_tmem::HTOP, fwd_tmem::HBOT, qd, hv);
                stage40(hv, 128 * (qd & 1) + r, qd, sm + HS);
            }
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->done);
        }
    }
    kernel_teardown(tm, fwd_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// Bidirectional read-out (Algorithm 1, zh §2.2): Y_i = Phi(q_i)^T H with the head's total
// state H, out_i = Y_i[:64] / Y_i[64].  No chunk depends on another, so the CTA's two
// 256-thread groups take alternate chunks of the segment, as the segment aggregates do:
// while one group waits for its MMA or its rows, the other forms features.  Both read one
// bf16 copy of H staged at the start.   grid: nseg x BH
// ------------------------------------------------------------------------------------------
namespace ro_smem {
constexpr uint32_t X = 0;             // q rows [128][64] (per group)
constexpr uint32_t PHI = TILE;        // Phi_Q [128][256] (per group)
constexpr uint32_t GROUP = 5 * TILE;  // bytes per group
constexpr uint32_t HS = 2 * GROUP;    // H as a bf16 value tile [256][80] (5 atoms)
constexpr uint32_t WHI = HS + 5 * VA256;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t RN = WLO + 8192;   // row norms [2][128]
constexpr uint32_t BAR = RN + 1024;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace ro_smem
namespace ro_tmem {  // per group, at 256 * group
constexpr uint32_t PROJ = 0;  // [128][64]
constexpr uint32_t Y = 64;    // [128][80]
constexpr uint32_t NCOLS = 512;
}  // namespace ro_tmem

__global__ void __launch_bounds__(NTH, 1) tc_readout(const __grid_constant__ Args a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace ro_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int g = threadIdx.x >> 8, gt = threadIdx.x & 255;
    const int r = gt & 127, h = gt >> 7;
    const bool leader = gt == 0;
    float *rn = reinterpret_cast<float *>(sm + RN) + 128 * g;
    const uint32_t sb = smem_u32(sm), gb = sb + (uint32_t)g * GROUP;
    uint8_t *xg = sm + g * GROUP + X, *phig = sm + g * GROUP + PHI;
    uint64_t *mbar = g ? &ctl->bar_b : &ctl->bar;
    volatile uint32_t *gabort = g ? &ctl->abort_b : &ctl->abort;  // as in the segment aggregates
    const uint32_t tm = kernel_setup(ctl, ro_tmem::NCOLS, a.W, sm + WHI, sm + WLO);
    const uint32_t tg = tm + 256u * g;  // this group's TMEM columns
    {  // H into the value tile: quarter qd = 2g + h takes 40 columns of state row 128 (qd & 1) + r
        const int qd = 2 * g + h, m = 128 * (qd & 1) + r, c0 = 40 * (qd >> 1);
        const float *src = a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride + (int64_t)m * DS;
        float hv[40];
#pragma unroll
        for (int i = 0; i < 40; ++i) hv[i] = (c0 + i < DS) ? src[c0 + i] : 0.f;
        stage40(hv, m, qd, sm + HS);
    }
    publish_smem();
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};  // barrier g: this group's rows
    auto load_x = [&](int64_t c) {
        uint64_t *bar = arm_load(ctl, ld, g, TILE, leader);
        if (leader) tma_k128(gb + X, &a.tm_q, c, bh, bar);
    };
    auto wait_group_mma = [&]() {  // bounded, then the group syncs
        if (leader && *gabort == 0u && !mbar_wait(mbar, phase & 1u, WAIT_LIMIT_NS)) {
            *gabort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        ++phase;
        group_sync(g);
        fence_after_sync();
        return *gabort == 0u;
    };
    auto wait_group_load = [&]() {
        if ((ld.pend >> g) & 1u) {
            if (mbar_wait(&ctl->ld[g], load_parity(ld, g), WAIT_LIMIT_NS)) {
                ld.pend &= ~(1u << g);
            } else {
                *gabort = 1u;
                atomicExch(&g_tc_error, 1);
            }
        }
        group_sync(g);
        return *gabort == 0u;
    };
    int64_t c0 = t0 + (int64_t)g * T;  // this group's chunks: every other one of the segment
    if (c0 < t1) load_x(c0);
    for (; c0 < t1 && ok; c0 += 2 * T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        const int64_t cn = c0 + 2 * T;
        if (!(ok = wait_group_load())) break;
        if (leader) {  // the projection runs while the row norms are formed
            fence_after_sync();
            issue_proj(tg + ro_tmem::PROJ, gb + X, sb + WHI, sb + WLO);
            mma_commit(mbar);
        }
        if (h == 0) rn[r] = row_norm(xg, r);
        if (!(ok = wait_group_mma())) break;
        if (cn < t1) load_x(cn);  // the rows are consumed: the next ones come in meanwhile
        {
            const float inv = 1.f / fmaxf(rn[r], kNormEps);
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                float u[16], t[16];
                proj_tanh(tg, ro_tmem::PROJ, 2 * h + qq, inv, a.beta, u, t);
                write_features(t, r, 2 * h + qq, valid ? 1.f : 0.f, phig);
            }
        }
        fence_smem_async();
        fence_before_sync();
        group_sync(g);
        if (leader) {  // Y = Phi_Q H
            fence_after_sync();
            issue_k256_va(tg + ro_tmem::Y, gb + PHI, sb + HS, idesc_bf16(128, 80, 0, 1), false);
            mma_commit(mbar);
        }
        if (!(ok = wait_group_mma())) break;
        {  // out = Y[:, :64] / Y[:, 64]: columns 16 (2h + qq) .. of row r
            const int qds[2] = {2 * h, 2 * h + 1};
            const float dd = store_out_quarters<2>(tg, ro_tmem::Y, qds, valid, a.out + (base + c0 + r) * DH);
            if (h == 0 && valid && a.den) a.den[base + c0 + r] = dd;
        }
        fence_before_sync();  // the read-out of Y precedes the next chunk's MMAs
    }
    if (leader && ((ld.pend >> g) & 1u)) mbar_wait(&ctl->ld[g], load_parity(ld, g), WAIT_LIMIT_NS);
    kernel_teardown(tm, ro_tmem::NCOLS);
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

// D[128][64] = DP[128][64] (W_hi + W_lo): W as MN-major B (rows = projections, cols = d).
__device__ __forceinline__ void issue_dxhat(uint32_t d, uint32_t dp, uint32_t whi, uint32_t wlo)
{
    constexpr uint32_t id = idesc_bf16(128, 64, 0, 1);
    const uint64_t da = sdesc(dp, 16, 1024, LAYOUT_SW128), bh = sdesc(whi, TILE, 1024, LAYOUT_SW128),
                   bl = sdesc(wlo, TILE, 1024, LAYOUT_SW128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        mma_bf16(d, da + 2 * kk, bh + kk * (2048 >> 4), id, kk > 0);
        mma_bf16(d, da + 2 * kk, bl + kk * (2048 >> 4), id, 1);
    }
}

namespace bq_smem {
constexpr uint32_t RA = 0;                 // k, o, q rows at load; Phi_K [128][256] after the features
constexpr uint32_t XK = RA;
constexpr uint32_t OT = RA + TILE;
constexpr uint32_t XQ = RA + 2 * TILE;
constexpr uint32_t PHK = RA;
constexpr uint32_t RB = 4 * TILE;          // W at load; masked P''; dP~ + W at the end
constexpr uint32_t PB = RB;
constexpr uint32_t DP = RB;
constexpr uint32_t WHI = RB + TILE;
constexpr uint32_t WLO = RB + TILE + 8192;
constexpr uint32_t VA = RB + 2 * TILE;     // [V | 1] [128][80]
constexpr uint32_t DOV = VA + 5 * VA128;   // dO [128][64] (4 atoms)
constexpr uint32_t HSHI = DOV + 4 * VA128; // staged H[:, :64], bf16 hi  [256][64] (4 atoms)
constexpr uint32_t HSLO = HSHI + 4 * VA256;  // and lo
constexpr uint32_t HDEN = HSLO + 4 * VA256;  // H[:, 64] fp32 [256]
constexpr uint32_t ROWC = HDEN + 1024;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t RN = ROWINV + 512;
constexpr uint32_t XCH = RN + 1024;
constexpr uint32_t BAR = XCH + 2048;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace bq_smem
namespace bq_tmem {
constexpr uint32_t PROJ = 0;   // q 0..63, k 64..127
constexpr uint32_t P = 128;    // [128][128]
constexpr uint32_t DPHI = 0;   // [128][256]
constexpr uint32_t DX = 0;     // [128][64]
constexpr uint32_t HTOP = 256;
constexpr uint32_t HBOT = 336;
constexpr uint32_t NCOLS = 512;
}  // namespace bq_tmem

// ------------------------------------------------------------------------------------------
// dq walk (chunks in order, prefix state H)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 1) tc_bwd_q_walk(const __grid_constant__ BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace bq_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *xch = reinterpret_cast<float *>(sm + XCH), *hden = reinterpret_cast<float *>(sm + HDEN);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    float *rn = reinterpret_cast<float *>(sm + RN);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const bool causal = a.causal != 0;
    const uint32_t tm = kernel_setup(ctl, bq_tmem::NCOLS, a.W, sm + WHI, sm + WLO);
    {
        float hv[40];
        load_state40(a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride, 128 * (qd & 1) + r, qd,
                     tm, bq_tmem::HTOP, bq_tmem::HBOT, hv);
        stage40_hilo(hv, 128 * (qd & 1) + r, qd, sm + HSHI, sm + HSLO, hden);
    }
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};
    auto issue_kv_do = [&](int64_t c) {  // q, k, v, dO, o rows of chunk c
        uint64_t *bar = arm_load(ctl, ld, 0, (causal ? 5u : 3u) * TILE);
        if (threadIdx.x == 0) {
            tma_va(sb + DOV, &a.tm_do_va, c, bh, bar);
            tma_k128(sb + OT, &a.tm_o, c, bh, bar);
            tma_k128(sb + XQ, &a.tm_q, c, bh, bar);
            if (causal) {
                tma_k128(sb + XK, &a.tm_k, c, bh, bar);
                tma_va(sb + VA, &a.tm_v_va, c, bh, bar);
            }
        }
    };
    auto reload_w = [&]() {  // W tiles (hi, lo) back over the masked block
        uint64_t *bar = arm_load(ctl, ld, 3, 2u * 8192u);
        if (threadIdx.x == 0) bulk_load(sb + WHI, a.wimg, 2u * 8192u, bar);
    };
    if (t0 < t1) {
        issue_kv_do(t0);
    }
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        if (!(ok = wait_loads(ctl, ld, 1u))) break;
        if (threadIdx.x == 3 * 128) {  // the projections and P'' run while quarters 0-2 form the row norms
                                       // and scalars (a thread issuing MMAs is held until the tensor
                                       // core's queue takes the last one)
            fence_after_sync();
            issue_proj(tm + bq_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
            if (causal) {
                issue_proj(tm + bq_tmem::PROJ + 64, sb + XK, sb + WHI, sb + WLO);
                // P'' = dO V^T (needs no features)
                issue_va_va(tm + bq_tmem::P, sb + DOV, T, sb + VA, T, 4, idesc_bf16(128, 128, 0, 0), false);
            }
            mma_commit(&ctl->bar);
        }
        if (qd == 0) rn[r] = row_norm(sm + XQ, r);
        if (causal && qd == 1) rn[128 + r] = row_norm(sm + XK, r);
        if (qd == 2) {
            row_scalars(r, sm + DOV, sm + OT, a.den + base + c0, nv, rowc, rowinv, nullptr);
            if (valid) a.cbuf[base + c0 + r] = rowc[r];  // for the key-side passes
        }
        if (causal && qd == 3) write_col64(sm + VA, r, valid ? 1.f : 0.f);
        fence_smem_async();
        if (!(ok = wait_mma(ctl, phase, 3 * 128))) break;
        const float raw_q = rn[r];
        const float c_r = rowc[r], invden_r = rowinv[r];
        float u[16], t[16];
        proj_tanh(tm, bq_tmem::PROJ, qd, 1.f / fmaxf(raw_q, kNormEps), a.beta, u, t);
        if (causal) {
            float uk[16], tk[16];
            proj_tanh(tm, bq_tmem::PROJ + 64, qd, 1.f / fmaxf(rn[128 + r], kNormEps), a.beta, uk, tk);
            write_features(tk, r, qd, valid ? 1.f : 0.f, sm + PHK);
            mask_block<false, true, false>(tm, bq_tmem::P, r, qd, c_r, nullptr, sm + PB);  // v_j.dO_i + c_i, j <= i
        }
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            // D = dO H_prev[:, :64]^T (+ tril(P'') Phi_K)
            issue_va_va(tm + bq_tmem::DPHI, sb + DOV, T, sb + HSHI, 256, 4, idesc_bf16(128, 256, 0, 0), false);
            issue_va_va(tm + bq_tmem::DPHI, sb + DOV, T, sb + HSLO, 256, 4, idesc_bf16(128, 256, 0, 0), true);
            if (causal) {
                issue_k128_k128mn(tm + bq_tmem::DPHI, sb + PB, sb + PHK, idesc_bf16(128, 256, 0, 1), true);
                issue_state_update(tm, bq_tmem::HTOP, bq_tmem::HBOT, sb + PHK, sb + VA);
            }
            mma_commit(&ctl->bar);
        }
        wait_mma_each(ctl, phase);
        if (c0 + T < t1) issue_kv_do(c0 + T);  // Phi_K (where the q, k, o rows go), V~ and dO are free now
        reload_w();
        // dphi = (D + c_i H_prev[:, 64]) / den_i
        features_vjp(tm, bq_tmem::DPHI, r, qd, a.beta, valid, u, t, hden, c_r, invden_r, sm + DP,
                     a.dpq ? a.dpq + (base + c0 + r) * DH : nullptr, 1.f / fmaxf(raw_q, kNormEps));
        publish_smem();
        if (threadIdx.x == 0 && wait_load_t0(ctl, ld, 3)) {
            fence_after_sync();
            issue_dxhat(tm + bq_tmem::DX, sb + DP, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        uint4 xq4[2];  // this row's q values, fetched while dX^ runs
        if (valid) {
            uint32_t w8[8];
            ld_global_v8(a.q + (base + c0 + r) * DH + 16 * qd, w8);
            xq4[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            xq4[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
        }
        wait_mma_each(ctl, phase);
        write_dx(tm, bq_tmem::DX, r, qd, valid, raw_q, nullptr, xq4, a.dq + (base + c0 + r) * DH, xch);
        if (causal) {
            float hv[40];
            read_state40(tm, bq_tmem::HTOP, bq_tmem::HBOT, qd, hv);
            stage40_hilo(hv, 128 * (qd & 1) + r, qd, sm + HSHI, sm + HSLO, hden);
        }
        // the staged state and the TMEM reads are handed over by the next chunk's first barrier
        fence_smem_async();
        fence_before_sync();
    }
    drain_loads(ctl, ld);
    kernel_teardown(tm, bq_tmem::NCOLS);
}

namespace bkv_smem {
constexpr uint32_t PHQ = 0;                // W (tile 1) at load; Phi_Q'; dP~ + W at the end
constexpr uint32_t DP = PHQ;
constexpr uint32_t WHI = PHQ + TILE;
constexpr uint32_t WLO = WHI + 8192;
constexpr uint32_t PHK = PHQ + 4 * TILE;   // k rows (tile 0), q rows (tile 1) at load; Phi_K; then masked S'^T and P'
constexpr uint32_t XK = PHK;
constexpr uint32_t XQ = PHK + TILE;
constexpr uint32_t STB = PHK;              // tiles 0-1
constexpr uint32_t PPB = PHK + 2 * TILE;   // tiles 2-3
constexpr uint32_t VA = PHK + 4 * TILE;    // [V | 1] [128][80]
constexpr uint32_t DOC = VA + 5 * VA128;   // [dO | c] [128][80]
constexpr uint32_t GS = DOC + 5 * VA128;   // staged G [256][80]
constexpr uint32_t ROWC = GS + 5 * VA256;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t RN = ROWINV + 512;
constexpr uint32_t XCH = RN + 1024;
constexpr uint32_t BAR = XCH + 2048;
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

// ------------------------------------------------------------------------------------------
// dk/dv walk (chunks in reverse, suffix state G)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 1) tc_bwd_kv_walk(const __grid_constant__ BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace bkv_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *xch = reinterpret_cast<float *>(sm + XCH), *rn = reinterpret_cast<float *>(sm + RN);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const bool causal = a.causal != 0;
    const uint32_t tm = kernel_setup(ctl, bkv_tmem::NCOLS, a.W, sm + WHI, sm + WLO);
    {
        float hv[40];
        load_state40(a.state + (int64_t)bh * a.nseg * MF * DS + seg * a.state_seg_stride, 128 * (qd & 1) + r, qd,
                     tm, bkv_tmem::GTOP, bkv_tmem::GBOT, hv);
        stage40(hv, 128 * (qd & 1) + r, qd, sm + GS);
    }
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t base = (int64_t)bh * a.N;
    const int64_t nchunks = (t1 - t0 + T - 1) / T;
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};
    auto issue_kv_do = [&](int64_t c) {  // k, v, dO (and q) rows of chunk c
        uint64_t *bar = arm_load(ctl, ld, 0, (causal ? 4u : 2u) * TILE);
        if (threadIdx.x == 0) {
            tma_k128(sb + XK, &a.tm_k, c, bh, bar);
            tma_va(sb + VA, &a.tm_v_va, c, bh, bar);
            if (causal) {
                tma_va(sb + DOC, &a.tm_do_va, c, bh, bar);
                tma_k128(sb + XQ, &a.tm_q, c, bh, bar);
            }
        }
    };
    auto reload_w = [&]() {  // W tiles (hi, lo) back over Phi_Q'
        uint64_t *bar = arm_load(ctl, ld, 3, 2u * 8192u);
        if (threadIdx.x == 0) bulk_load(sb + WHI, a.wimg, 2u * 8192u, bar);
    };
    if (nchunks > 0) issue_kv_do(t0 + (nchunks - 1) * T);
    for (int64_t ci = nchunks - 1; ci >= 0 && ok; --ci) {
        const int64_t c0 = t0 + ci * T;
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        if (!(ok = wait_loads(ctl, ld, 1u))) break;
        if (threadIdx.x == 3 * 128) {  // projections and V dO^T run while quarters 0-2 form the row norms
                                       // and scalars (a thread issuing MMAs is held until the tensor
                                       // core's queue takes the last one)
            fence_after_sync();
            issue_proj(tm + bkv_tmem::PROJ + 64, sb + XK, sb + WHI, sb + WLO);
            if (causal) {
                issue_va_va(tm + bkv_tmem::PP, sb + VA, T, sb + DOC, T, 4, idesc_bf16(128, 128, 0, 0), false);
                issue_proj(tm + bkv_tmem::PROJ, sb + XQ, sb + WHI, sb + WLO);
            }
            mma_commit(&ctl->bar);
        }
        if (qd == 0) rn[128 + r] = row_norm(sm + XK, r);
        if (causal && qd == 1) rn[r] = row_norm(sm + XQ, r);
        if (causal && qd == 2)
            load_row_scalars(r, valid, a.cbuf + base + c0 + r, a.den + base + c0 + r, rowc, rowinv, sm + DOC);
        if (qd == 2) write_col64(sm + VA, r, valid ? 1.f : 0.f);
        fence_smem_async();
        if (!(ok = wait_mma(ctl, phase, 3 * 128))) break;
        const float raw_k = rn[128 + r];
        float u[16], t[16];
        proj_tanh(tm, bkv_tmem::PROJ + 64, qd, 1.f / fmaxf(raw_k, kNormEps), a.beta, u, t);
        write_features(t, r, qd, valid ? 1.f : 0.f, sm + PHK);
        float uq[16], tq[16];
        if (causal) proj_tanh(tm, bkv_tmem::PROJ, qd, 1.f / fmaxf(rn[r], kNormEps), a.beta, uq, tq);
        publish_smem();
        if (threadIdx.x == 0) {  // dV = Phi_K G_next[:, :64], while Phi_Q' is formed
            fence_after_sync();
            issue_k256_va(tm + bkv_tmem::DVT, sb + PHK, sb + GS, idesc_bf16(128, 64, 0, 1), false);
        }
        if (causal) {
            write_features(tq, r, qd, rowinv[r], sm + PHQ);  // Phi_Q' = Phi_Q / den
            publish_smem();
            if (threadIdx.x == 0) {
                fence_after_sync();
                issue_k256_kk(tm + bkv_tmem::ST, sb + PHK, sb + PHQ, idesc_bf16(128, 128, 0, 0), false);  // S'^T
            }
        }
        // the commit reports dV too: it is complete before the masks overwrite Phi_K
        if (threadIdx.x == 0) mma_commit(&ctl->bar);
        wait_mma_each(ctl, phase);
        if (causal) {
            mask_block<true, false, false>(tm, bkv_tmem::ST, r, qd, 0.f, nullptr, sm + STB);
            mask_block<true, false, true>(tm, bkv_tmem::PP, r, qd, 0.f, rowc, sm + PPB);  // v_j.dO_i + c_i, i >= j
        }
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            if (causal)  // dV += triu(S'^T) dO
                issue_k128_va(tm + bkv_tmem::DVT, sb + STB, 0, sb + DOC, idesc_bf16(128, 64, 0, 1), true);
            // dPhi_K = [V | 1] G_next^T (+ triu(P') Phi_Q')
            issue_va_va(tm + bkv_tmem::DPHI, sb + VA, T, sb + GS, 256, 5, idesc_bf16(128, 256, 0, 0), false);
            if (causal) {
                issue_k128_k128mn(tm + bkv_tmem::DPHI, sb + PPB, sb + PHQ, idesc_bf16(128, 256, 0, 1), true);
                issue_state_update(tm, bkv_tmem::GTOP, bkv_tmem::GBOT, sb + PHQ, sb + DOC);
            }
            mma_commit(&ctl->bar);
        }
        wait_mma_each(ctl, phase);
        if (ci > 0) issue_kv_do(c0 - T);  // Phi_K / masks, V~ and [dO | c] are free now
        if (causal && ci > 0 && qd == 2) {  // the next chunk's c_i and den_i into L2
            prefetch_l2(a.cbuf + base + c0 - T + r);
            prefetch_l2(a.den + base + c0 - T + r);
        }
        reload_w();
        store_row16(tm, bkv_tmem::DVT, qd, valid, 1.f, a.dv + (base + c0 + r) * DH);
        features_vjp(tm, bkv_tmem::DPHI, r, qd, a.beta, valid, u, t, nullptr, 0.f, 1.f, sm + DP,
                     a.dpk ? a.dpk + (base + c0 + r) * DH : nullptr, 1.f / fmaxf(raw_k, kNormEps));
        publish_smem();
        if (threadIdx.x == 0 && wait_load_t0(ctl, ld, 3)) {
            fence_after_sync();
            issue_dxhat(tm + bkv_tmem::DX, sb + DP, sb + WHI, sb + WLO);
            mma_commit(&ctl->bar);
        }
        uint4 xk4[2];  // this row's k values (its tile is being reloaded), fetched while dX^ runs
        if (valid) {
            uint32_t w8[8];
            ld_global_v8(a.k + (base + c0 + r) * DH + 16 * qd, w8);
            xk4[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            xk4[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
        }
        if (causal) {  // the updated state is staged while dX^ runs
            float hv[40];
            read_state40(tm, bkv_tmem::GTOP, bkv_tmem::GBOT, qd, hv);
            stage40(hv, 128 * (qd & 1) + r, qd, sm + GS);
        }
        wait_mma_each(ctl, phase);
        write_dx(tm, bkv_tmem::DX, r, qd, valid, raw_k, nullptr, xk4, a.dk + (base + c0 + r) * DH, xch);
        // the staged state and the TMEM reads are handed over by the next chunk's first barrier
        fence_smem_async();
        fence_before_sync();
    }
    drain_loads(ctl, ld);
    kernel_teardown(tm, bkv_tmem::NCOLS);
}

// ------------------------------------------------------------------------------------------
// Gradient of W (the learnable-hyperplane variant): p = W_l x^ for every q and k row, so
// dW = sum over rows of (dLoss/dp / |x|) x^T with the raw rows x.  The walks leave
// dLoss/dp / |x| per row ([rows][64] bf16); here each CTA sums a range of 128-row chunks of
// the q side then the k side on the tensor core, D[64 projections][64] += dp^T x, and
// writes its partial; tc_dw_reduce adds the partials in CTA order.  The MMA's M is 128:
// rows 64..127 of the accumulator come from the x tile placed after the dp tile and are
// not read.   grid: nblk, 128 threads
// ------------------------------------------------------------------------------------------
struct DwArgs {
    CUtensorMap tm_dp[2], tm_x[2];  // [BH][N][64] bf16 as 3-D maps, K128 boxes (q side, k side)
    int64_t chunks_per_head;        // ceil(N / 128)
    int64_t chunks_per_side;        // BH * chunks_per_head
    int64_t chunks_per_cta;
    float *partial;                 // [nblk][64][64]
};

namespace dw_smem {
constexpr uint32_t STAGE = 2 * TILE;  // dp tile, then x tile
constexpr uint32_t BAR = 2 * STAGE;   // 2 stages
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace dw_smem

__global__ void __launch_bounds__(128, 1) tc_dw(const __grid_constant__ DwArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + dw_smem::BAR);  // tma[2], mma[2]
    __shared__ uint32_t tmem_slot;
    __shared__ uint32_t failed;
    const uint32_t sb = smem_u32(sm);
    const int64_t c_begin = (int64_t)blockIdx.x * a.chunks_per_cta;
    int64_t c_end = c_begin + a.chunks_per_cta;
    if (c_end > 2 * a.chunks_per_side) c_end = 2 * a.chunks_per_side;
    const int n = c_end > c_begin ? (int)(c_end - c_begin) : 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        failed = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(&tmem_slot, 64);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = tmem_slot;
    if (threadIdx.x == 0 && n > 0) {
        constexpr uint32_t id = idesc_bf16(128, 64, 1, 1);
        auto load = [&](int i) {
            const int64_t c = c_begin + i;
            const int side = c >= a.chunks_per_side ? 1 : 0;
            const int64_t hc = c - side * a.chunks_per_side;
            const int head = (int)(hc / a.chunks_per_head), row = (int)((hc % a.chunks_per_head) * T);
            const uint32_t st = sb + (uint32_t)(i & 1) * dw_smem::STAGE;
            mbar_expect_tx(&bars[i & 1], 2 * TILE);
            tma_load3(st, &a.tm_dp[side], 0, row, head, &bars[i & 1]);
            tma_load3(st + TILE, &a.tm_x[side], 0, row, head, &bars[i & 1]);
        };
        bool ok = true;
        load(0);
        for (int i = 0; i < n && ok; ++i) {
            if (i + 1 < n) {
                if (i >= 1 && !mbar_wait(&bars[2 + ((i + 1) & 1)], ((i - 1) >> 1) & 1, WAIT_LIMIT_NS)) {
                    ok = false;  // the stage's previous MMAs never completed
                    break;
                }
                load(i + 1);
            }
            if (!mbar_wait(&bars[i & 1], (i >> 1) & 1, WAIT_LIMIT_NS)) {
                ok = false;
                break;
            }
            fence_after_sync();
            const uint32_t st = sb + (uint32_t)(i & 1) * dw_smem::STAGE;
            const uint64_t da = sdesc(st, TILE, 1024, LAYOUT_SW128), db = sdesc(st + TILE, TILE, 1024, LAYOUT_SW128);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tm, da + kk * (2048 >> 4), db + kk * (2048 >> 4), id, (i > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars[2 + (i & 1)]);
        }
        // the last commit covers every MMA issued before it; then every load in flight
        if (ok && !mbar_wait(&bars[2 + ((n - 1) & 1)], ((n - 1) >> 1) & 1, WAIT_LIMIT_NS)) ok = false;
        if (!ok) {
            failed = 1;
            atomicExch(&g_tc_error, 1);
            for (int s = 0; s < 2; ++s) mbar_wait(&bars[s], 0, WAIT_LIMIT_NS);  // bounded drain
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    float *dst = a.partial + (int64_t)blockIdx.x * 64 * 64;
    if (threadIdx.x < 64) {  // rows 0..63 of the accumulator: warps 0 and 1
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 16) {
            uint32_t w[16];
            tmem_ld16_nowait(tlane(tm, (uint32_t)c0), w);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                dst[threadIdx.x * 64 + c0 + i] = (n > 0 && !failed) ? __uint_as_float(w[i]) : 0.f;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(tm, 64);
}

// dW[e] = sum over the CTAs of partial[b][e], in CTA order.
__global__ void tc_dw_reduce(const float *partial, int nblk, float *dW)
{
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= 64 * 64) return;
    float s = 0.f;
    for (int b = 0; b < nblk; ++b) s += partial[(int64_t)b * 64 * 64 + e];
    dW[e] = s;
}

// W [64][64] fp32 -> its two bf16 K128 tiles (hi, lo) in global memory, byte for byte as
// load_w_split lays them out in shared memory, so that the walks reload them with one bulk
// copy.  One CTA of NTH threads.
__global__ void __launch_bounds__(NTH, 1) tc_w_image(const float *W, uint8_t *img)
{
    load_w_split(W, img, img + 8192);
}

// Waits on a barrier that nothing arrives on, for at most limit_ns, and reports the timeout
// the way the kernels above do.  One CTA of one warp.
__global__ void tc_wait_timeout_selftest(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        if (!mbar_wait(&bar, 0u, limit_ns)) atomicExch(&g_tc_error, 1);
    }
    __syncwarp();
}

// ---- host side ---------------------------------------------------------------------------

// Token coordinates of the TMA loads are 32-bit.
inline bool fast_path_ok(race_dtype_t dtype, int d, int L, int P, float tau, int64_t N)
{
    return dtype == RACE_BF16 && d == 64 && L == 16 && P == 4 && tau > 0.f && N < ((int64_t)1 << 31);
}

inline size_t smem_bytes(uint32_t total) { return total + 1024; }

// TMA destinations: K128 tiles 1024-byte aligned (128-byte swizzle), value tiles 256-byte
// aligned (32-byte swizzle); bulk copies 16-byte aligned.
static_assert(agg_smem::X % 1024 == 0 && agg_smem::PHI % 1024 == 0 && agg_smem::VA % 1024 == 0 &&
                  agg_smem::GROUP % 1024 == 0,
              "agg tiles");
static_assert(sizeof(Ctl) <= 64, "control block");
static_assert(fwd_smem::XQ % 1024 == 0 && fwd_smem::XK % 1024 == 0 && fwd_smem::VA0 % 1024 == 0 &&
                  fwd_smem::VA1 % 1024 == 0 && fwd_smem::HS % 1024 == 0 && fwd_smem::SB % 1024 == 0,
              "fwd tiles");
static_assert(bq_smem::XQ % 1024 == 0 && bq_smem::XK % 1024 == 0 && bq_smem::OT % 1024 == 0 &&
                  bq_smem::VA % 1024 == 0 && bq_smem::DOV % 1024 == 0 &&
                  bq_smem::WHI % 16 == 0,
              "dq walk tiles");
static_assert(bkv_smem::XQ % 1024 == 0 && bkv_smem::XK % 1024 == 0 && bkv_smem::VA % 1024 == 0 &&
                  bkv_smem::DOC % 1024 == 0 && bkv_smem::WHI % 16 == 0,
              "dk/dv walk tiles");
static_assert(ro_smem::X % 1024 == 0 && ro_smem::PHI % 1024 == 0 && ro_smem::GROUP % 1024 == 0 &&
                  ro_smem::HS % 1024 == 0 && ro_smem::WHI % 1024 == 0,
              "read-out tiles");
static_assert(agg_smem::TOTAL + 1024 <= 232448 && fwd_smem::TOTAL + 1024 <= 232448 &&
                  bq_smem::TOTAL + 1024 <= 232448 && bkv_smem::TOTAL + 1024 <= 232448 &&
                  ro_smem::TOTAL + 1024 <= 232448,
              "shared memory per CTA");

}  // namespace tc
}  // namespace race
