// race_tc_wide.cuh -- tcgen05 path of RACE Attention for bf16 inputs with d = 128 and tables
// of P = 5 hyperplanes (R = 32 corners), L a multiple of 8 up to 32 (L * 2^P up to 1,024
// features), causal.
//
// The read-out of Algorithm 2 (zh §2.3) is a sum over features and over value columns:
//   num_i = sum_f Phi_Q[i, f] (sum_{j<=i} Phi_K[j, f] v_j),  den_i = sum_f Phi_Q[i, f] (sum_{j<=i} Phi_K[j, f])
// and every feature belongs to exactly one table.  So the features are cut into groups of
// 8 tables (256 features, 40 projections) and the value columns into two halves of 64; each
// (group, half) pass is the causal walk of the d = 64, 256-feature kernels (race_tc.cuh),
// with the same TMEM and shared-memory shapes, and the passes' partial sums are added in a
// fixed order (group 0 first), so results do not depend on scheduling.  The backward is
// linear in dPhi, so it splits the same way: each pass leaves its share of dLoss/dp^ for its
// group's projections and of dv for its half.
//
//   wide_proj     p^ = W x / |x| for every q and k row of a head: one tcgen05 GEMM per
//                 128-row tile (x bf16 exact, W as bf16 hi + lo), fp32 [N][npwp]
//   wide_agg<0>   per (group, half) segment totals sum_j phi_g(k_j) [v_j,h | 1]^T
//   wide_agg<1>   per (group, half) sum_i phi_g(q_i) / den_i [dO_i,h | c_i]^T (c only in half 0)
//   wide_fwd_walk one group's causal walk for both halves: partial numerator and den, summed
//                 over the groups in fp32 in memory
//   wide_finish   out = numerator / den (forward) or dv (backward) from the fp32 sums
//   wide_rowc     c_i = -(dO_i . o_i) over all 128 columns
//   wide_bwd_q_walk / wide_bwd_kv_walk: the dq / dk,dv walks of the (group, half) passes
//   wide_dx       dx = (dX^ - x^ (x^ . dX^)) / |x| with dX^ = dp^ W on the tensor core
//
// Projections of the group come from shared memory (a [128][40] fp32 tile per chunk and
// side, loaded by TMA from the p^ array), so the walks hold neither x nor W; their shared
// memory stays within the per-CTA limit with the 128-wide rows.
#pragma once

#include "race_tc.cuh"

namespace race {
namespace tc {
namespace wide {

constexpr int WD = 128;                            // head dimension
constexpr int WP = 5;                              // hyperplanes per table
constexpr int WPROJ = 40;                          // projections of a feature group (8 tables)
constexpr uint32_t PTILE = 128u * WPROJ * 4u;      // one chunk's projections of a group, fp32 [128][40]
constexpr uint32_t WTILE_MAX = 160u * 128u;        // one K-half of W as K-major bf16 rows [npwp <= 160][64]
constexpr uint32_t kCtxTag = 0x5A5A5A5Au;          // a context holds this path's key-side states

// Per head.  Tensor maps: p^ as 2-D fp32 (npwp columns, N rows), boxes of 40 columns x 128
// rows (no swizzle); v and dO as 3-D bf16 (16 columns, N rows, 8 atoms of 16 columns), boxes
// of 4 atoms with the 32-byte swizzle (one value half); rows past N read as zero.
struct WideArgs {
    CUtensorMap tm_pq, tm_pk, tm_v, tm_do;
    CUtensorMap tm_acc;      // acc as 2-D fp32 (128 columns, N rows), boxes 32 x 128, 128-byte swizzle
    const float *den;        // [N] (backward)
    const float *cbuf;       // [N] c_i (backward)
    float *acc;              // [N][128] fp32: numerator (forward) or dv (backward) over the groups so far
    float *dacc;             // [N] fp32: den over the groups so far (forward)
    float *dp;               // [N][npwp] dLoss/dp^ of the walk's side (backward; zero before the walk)
    const float *state;      // walk start states [2 * groups][nseg][256][65]
    float *agg_out;          // segment totals [2 * groups][nseg][256][65]
    const float *ctx_states; // a saved context's scanned key-side states of the head, laid out as state
    const uint32_t *ctx_tag; // == kCtxTag when ctx_states holds them (written by this path's forward)
    int64_t N, seg_len;
    int nseg, npwp;
    int g;                   // the launch's feature group (walks launched once per group)
    int first;               // the launch is the first of its group sum (stores instead of adding)
    float beta;
};

struct ProjArgs {
    CUtensorMap tm_x[2];     // q, k rows of one head: 2-D bf16 (128 columns, N rows), 64 x 128 boxes, 128-byte swizzle
    const float *W;          // [npw][128] fp32
    float *p[2];             // [N][npwp] fp32 (q side, k side)
    int64_t N;
    int ntile;               // ceil(N / 128)
    int npw, npwp;
};

__device__ __forceinline__ void tma_load2(uint32_t dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ const float *state_of(const WideArgs &a, int pass, int seg)
{
    return a.state + ((int64_t)pass * a.nseg + seg) * MF * DS;
}

// ---- the soft hash with 5 hyperplanes per table ---------------------------------------------
// Thread (r, qd) of a 512-thread CTA owns tables 2qd, 2qd+1 of the group, i.e. projections
// 10qd .. 10qd+9 and features 64qd .. 64qd+63 (feature 32e + c of table 2qd+e, corner c).

// u = tanh(p^) and t = tanh(beta u) of this thread's 10 projections, from row r of a [128][40]
// fp32 tile.  The 40 bytes start 16-byte aligned for even qd and 8 bytes past for odd qd: two
// 16-byte loads and one 8-byte load.
__device__ __forceinline__ void proj_tanh10(const uint8_t *ptile, int r, int qd, float beta, float (&u)[10],
                                            float (&t)[10])
{
    const uint32_t a = smem_u32(ptile) + (uint32_t)(r * WPROJ + 10 * qd) * 4u;
    float p[10];
    if ((qd & 1) == 0) {
        const uint4 x0 = ld_shared_v4(a), x1 = ld_shared_v4(a + 16);
        const float2 x2 = *reinterpret_cast<const float2 *>(ptile + (uint32_t)(r * WPROJ + 10 * qd + 8) * 4u);
        p[0] = __uint_as_float(x0.x); p[1] = __uint_as_float(x0.y); p[2] = __uint_as_float(x0.z);
        p[3] = __uint_as_float(x0.w); p[4] = __uint_as_float(x1.x); p[5] = __uint_as_float(x1.y);
        p[6] = __uint_as_float(x1.z); p[7] = __uint_as_float(x1.w); p[8] = x2.x; p[9] = x2.y;
    } else {
        const float2 x0 = *reinterpret_cast<const float2 *>(ptile + (uint32_t)(r * WPROJ + 10 * qd) * 4u);
        const uint4 x1 = ld_shared_v4(a + 8), x2 = ld_shared_v4(a + 24);
        p[0] = x0.x; p[1] = x0.y;
        p[2] = __uint_as_float(x1.x); p[3] = __uint_as_float(x1.y); p[4] = __uint_as_float(x1.z);
        p[5] = __uint_as_float(x1.w); p[6] = __uint_as_float(x2.x); p[7] = __uint_as_float(x2.y);
        p[8] = __uint_as_float(x2.z); p[9] = __uint_as_float(x2.w);
    }
#pragma unroll
    for (int i = 0; i < 10; ++i) u[i] = tanh_fast(p[i]);
#pragma unroll
    for (int i = 0; i < 10; ++i) t[i] = tanh_fast(beta * u[i]);
}

// Corner weights of table e (0/1) of the thread: phi_c = prod_p (1 + s_cp t_p) / 2 with
// s_cp = +1 where bit p of c is set (sigmoid(2z) = (1 + tanh z) / 2: the softmax over the
// hypercube corners of zh §2.2, factorised).  Times `scale`.
__device__ __forceinline__ void corner_weights32(const float (&t)[10], int e, float scale, float (&f)[32])
{
    const float *tt = t + 5 * e;
    float s0[5], s1[5];
#pragma unroll
    for (int p = 0; p < 5; ++p) {
        s1[p] = 0.5f + 0.5f * tt[p];
        s0[p] = 0.5f - 0.5f * tt[p];
    }
    float a[4], b[8], d[4];
    a[0] = s0[0] * s0[1] * scale;
    a[1] = s1[0] * s0[1] * scale;
    a[2] = s0[0] * s1[1] * scale;
    a[3] = s1[0] * s1[1] * scale;
    d[0] = s0[3] * s0[4];
    d[1] = s1[3] * s0[4];
    d[2] = s0[3] * s1[4];
    d[3] = s1[3] * s1[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) b[k] = ((k & 1) ? s1[2] : s0[2]) * d[k >> 1];  // bits 2, 3, 4
#pragma unroll
    for (int hi = 0; hi < 8; ++hi)
#pragma unroll
        for (int lo = 0; lo < 4; ++lo) f[4 * hi + lo] = a[lo] * b[hi];
}

// The thread's 64 features of row r, times `scale`, into K128 tile qd of a Phi tile.
__device__ __forceinline__ void write_features64(const float (&t)[10], int r, int qd, float scale, uint8_t *phi)
{
    const uint32_t blk = smem_u32(phi) + (uint32_t)qd * TILE;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float f[32];
        corner_weights32(t, e, scale, f);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            st_shared_v4(blk + sw128_off(r, 4 * e + c), pack_bf16x2(f[8 * c], f[8 * c + 1]),
                         pack_bf16x2(f[8 * c + 2], f[8 * c + 3]), pack_bf16x2(f[8 * c + 4], f[8 * c + 5]),
                         pack_bf16x2(f[8 * c + 6], f[8 * c + 7]));
    }
}

// The same 64 features as bf16 pairs into the thread's TMEM lane, columns col0 + 32qd .. +31:
// the A-operand layout of a tensor-memory MMA (feature f at column col0 + f/2).
__device__ __forceinline__ void write_features64_tmem(const float (&t)[10], int qd, float scale, uint32_t tm,
                                                      uint32_t col0)
{
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float f[32];
        corner_weights32(t, e, scale, f);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = pack_bf16x2(f[2 * c], f[2 * c + 1]);
        tmem_st16u(tlane(tm, col0 + 32u * qd + 16u * e), w);
    }
}

// Feature-map VJP of the thread's two tables: dphi = (D + add_scale * add_vec) * mul with D
// from TMEM columns col0 + 64qd .. +63 and add_vec (fp32 per feature, shared memory) optional;
// du_p = beta sum_c s_cp phi_c (dphi_c - phi.dphi) = beta (2 A_p - (1 + t_p) phi.dphi), A_p the
// sum of phi_c dphi_c over the corners with bit p set; dp^ = du (1 - u^2) (0 for invalid rows).
__device__ __forceinline__ void features_vjp10(uint32_t tm, uint32_t col0, int qd, float beta, bool valid,
                                               const float (&u)[10], const float (&t)[10], const float *add_vec,
                                               float add_scale, float mul, float (&dp)[10])
{
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        uint32_t g[2][16];
        tmem_ld16_nowait(tlane(tm, col0 + 64u * qd + 32u * e), g[0]);
        tmem_ld16_nowait(tlane(tm, col0 + 64u * qd + 32u * e + 16u), g[1]);
        tmem_wait_ld();
        float f[32];
        corner_weights32(t, e, 1.f, f);
        float fg[32];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
            float av[4] = {0.f, 0.f, 0.f, 0.f};
            if (add_vec) {  // 16-byte loads (the vector is read by every thread of a quarter)
                const float4 a4 = reinterpret_cast<const float4 *>(add_vec + 64 * qd + 32 * e)[c4];
                av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c = 4 * c4 + k;
                float gg = __uint_as_float(g[c >> 4][c & 15]);
                if (add_vec) gg = fmaf(add_scale, av[k], gg) * mul;
                fg[c] = f[c] * gg;
            }
        }
        float s1[16], s2[8], s3[4];
#pragma unroll
        for (int k = 0; k < 16; ++k) s1[k] = fg[2 * k] + fg[2 * k + 1];  // corners with equal bits 1..4
#pragma unroll
        for (int k = 0; k < 8; ++k) s2[k] = s1[2 * k] + s1[2 * k + 1];   // equal bits 2..4
#pragma unroll
        for (int k = 0; k < 4; ++k) s3[k] = s2[2 * k] + s2[2 * k + 1];   // equal bits 3..4
        const float s40 = s3[0] + s3[1], s41 = s3[2] + s3[3];           // bit 4 clear / set
        const float dot = s40 + s41;
        float ap[5];
        ap[0] = 0.f;
#pragma unroll
        for (int c = 1; c < 32; c += 2) ap[0] += fg[c];
        ap[1] = 0.f;
#pragma unroll
        for (int k = 1; k < 16; k += 2) ap[1] += s1[k];
        ap[2] = (s2[1] + s2[3]) + (s2[5] + s2[7]);
        ap[3] = s3[1] + s3[3];
        ap[4] = s41;
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            const float uu = u[5 * e + p];
            const float du = beta * (2.f * ap[p] - (1.f + t[5 * e + p]) * dot);
            dp[5 * e + p] = valid ? du * (1.f - uu * uu) : 0.f;
        }
    }
}

// Partial sums to global memory without reading it back: stored (the first contribution)
// or added there by the memory system (red.global.add, no value returned), so no thread
// waits on the round trip.  Each element receives one contribution per launch, or two that
// commute exactly (a + b onto zero), so the sums do not depend on scheduling.
__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void red_add_v2(float *p, float a, float b)
{
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_add_f32(float *p, float a)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

// ---- bulk stores and reductions from shared memory (TMA, no multicast) ---------------------
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void tma_add_2d(const CUtensorMap *map, int x, int y, uint32_t src)
{
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     map),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of the committed bulk groups may be overwritten
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// the committed bulk groups are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16 fp32 values of row r, value columns 16qd .. 16qd+15 of a half, into a [128][64] fp32
// staging tile laid out as the TMA image of two boxes of [128][32] with the 128-byte swizzle.
__device__ __forceinline__ void stage_row16(uint32_t stage, int r, int qd, const float (&y)[16])
{
    const uint32_t box = stage + (uint32_t)(qd >> 1) * TILE;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        st_shared_v4(box + sw128_off(r, 4 * (qd & 1) + i), __float_as_uint(y[4 * i]), __float_as_uint(y[4 * i + 1]),
                     __float_as_uint(y[4 * i + 2]), __float_as_uint(y[4 * i + 3]));
}

// The staged tile into columns 64h .. 64h+63 of rows row0 .. row0+127 of an fp32 [N][128]
// array, stored or added (one writer per element per launch; rows past N are left out), as
// one committed bulk group.  Issued by one thread after the staging is published.
__device__ __forceinline__ void put_tile64(const CUtensorMap *map, uint32_t stage, int h, int row0, bool add)
{
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        if (add)
            tma_add_2d(map, 64 * h + 32 * b, row0, stage + (uint32_t)b * TILE);
        else
            tma_store_2d(map, 64 * h + 32 * b, row0, stage + (uint32_t)b * TILE);
    }
    bulk_commit();
}

// 10 fp32 values added in memory at dst, 16-byte aligned for even qd and 8 bytes past a
// 16-byte boundary for odd qd (dst = row base + 40 bytes x qd): two 16-byte and one 8-byte
// reduction.
__device__ __forceinline__ void add10(float *dst, const float (&v)[10], int qd)
{
    if ((qd & 1) == 0) {
        red_add_v4(dst, v[0], v[1], v[2], v[3]);
        red_add_v4(dst + 4, v[4], v[5], v[6], v[7]);
        red_add_v2(dst + 8, v[8], v[9]);
    } else {
        red_add_v2(dst, v[0], v[1]);
        red_add_v4(dst + 2, v[2], v[3], v[4], v[5]);
        red_add_v4(dst + 6, v[6], v[7], v[8], v[9]);
    }
}


// Bounded wait on one TMA barrier by the calling thread alone; false on timeout (after
// marking the CTA, or the thread group behind `flag`, as given up).
__device__ __forceinline__ bool wait_one_load(Ctl *ctl, Loads &ld, int b, volatile uint32_t *flag)
{
    if (!((ld.pend >> b) & 1u)) return true;
    if (mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS)) {
        ld.pend &= ~(1u << b);
        return true;
    }
    *flag = 1u;
    atomicExch(&g_tc_error, 1);
    return false;
}

// ------------------------------------------------------------------------------------------
// Projections p^ = W x / max(|x|, eps) of every q and k row of one head: the normalised
// projections of the soft hash (zh §2.2) before the squash.  Persistent: CTA b takes the
// 128-row tiles b, b + gridDim.x, ... of the q rows, then of the k rows; while one tile is
// read out, the next tile's projection runs into the other accumulator and the rows of the
// tile after it load into the other row buffer.   grid: min(tiles, SMs), 512 threads
// ------------------------------------------------------------------------------------------
namespace proj_smem {
constexpr uint32_t X0 = 0;                     // a tile's rows: 2 K128 tiles (columns 0-63, 64-127)
constexpr uint32_t X1 = 2 * TILE;
constexpr uint32_t WHI = 4 * TILE;             // W as K-major bf16 hi: 2 K-halves of [npwp][64]
constexpr uint32_t WLO = WHI + 2 * WTILE_MAX;  // and lo
constexpr uint32_t RN = WLO + 2 * WTILE_MAX;   // partial squared norms [2 buffers][4 quarters][128]
constexpr uint32_t BAR = RN + 4096;
constexpr uint32_t MB = BAR + 64;              // MMA completion, one per accumulator
constexpr uint32_t TOTAL = MB + 64;
}  // namespace proj_smem

__global__ void __launch_bounds__(NTH, 1) wide_proj(const __grid_constant__ ProjArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace proj_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    uint64_t *mb = reinterpret_cast<uint64_t *>(sm + MB);
    float *rn = reinterpret_cast<float *>(sm + RN);
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    if (threadIdx.x == 0) {
        mbar_init(&mb[0], 1);
        mbar_init(&mb[1], 1);
    }
    // W [npw][128] fp32 -> bf16 hi + lo, K-major (row n of K-half kh at kh * WTILE_MAX); rows
    // npw .. npwp-1 are zero
    for (int e = threadIdx.x; e < a.npwp * 64; e += NTH) {
        const int n = e >> 6, c = 2 * (e & 63);
        float2 w = make_float2(0.f, 0.f);
        if (n < a.npw) w = *reinterpret_cast<const float2 *>(a.W + (int64_t)n * WD + c);
        const uint32_t hi = pack_bf16x2(w.x, w.y);
        const uint32_t lo = pack_bf16x2(w.x - bf16_lo(hi), w.y - bf16_hi(hi));
        const uint32_t off = (uint32_t)(c >> 6) * WTILE_MAX + sw128_off(n, (c & 63) >> 3) + (c & 7) * 2;
        *reinterpret_cast<uint32_t *>(sm + WHI + off) = hi;
        *reinterpret_cast<uint32_t *>(sm + WLO + off) = lo;
    }
    const uint32_t tm = kernel_setup(ctl, 512, nullptr, nullptr, nullptr);
    const int ntiles = 2 * a.ntile, npw8 = a.npwp >> 3;
    const uint32_t idesc = idesc_bf16(128, a.npwp, 0, 0);
    Loads ld = {};
    auto tile_of = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };
    auto issue_load = [&](int j) {  // called by every thread (load bookkeeping); thread 0 issues
        const int i = tile_of(j), side = i >= a.ntile ? 1 : 0, b = j & 1;
        const int row0 = (i - side * a.ntile) * T;
        uint64_t *bar = arm_load(ctl, ld, b, 2u * TILE);
        if (threadIdx.x == 0) {
            const uint32_t dst = sb + (b ? X1 : X0);
            tma_load2(dst, &a.tm_x[side], 0, row0, bar);
            tma_load2(dst + TILE, &a.tm_x[side], 64, row0, bar);
        }
    };
    // thread 0: once tile j's rows are in, issue its projection into accumulator j & 1
    auto issue_mma = [&](int j) {
        const int b = j & 1;
        if (*(volatile uint32_t *)&ctl->abort != 0u || !wait_one_load(ctl, ld, b, &ctl->abort)) return;
        fence_after_sync();
        const uint32_t xs = sb + (b ? X1 : X0), d = tm + (uint32_t)b * 256u;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            const uint64_t ax = sdesc(xs + kh * TILE, 16, 1024, LAYOUT_SW128);
            const uint64_t bh = sdesc(sb + WHI + kh * WTILE_MAX, 16, 1024, LAYOUT_SW128);
            const uint64_t bl = sdesc(sb + WLO + kh * WTILE_MAX, 16, 1024, LAYOUT_SW128);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(d, ax + 2 * kk, bh + 2 * kk, idesc, (kh | kk) != 0 ? 1u : 0u);
                mma_bf16(d, ax + 2 * kk, bl + 2 * kk, idesc, 1u);
            }
        }
        mma_commit(&mb[b]);
    };
    if (tile_of(0) < ntiles) issue_load(0);
    if (tile_of(1) < ntiles) issue_load(1);
    if (threadIdx.x == 0 && tile_of(0) < ntiles) issue_mma(0);
    for (int j = 0; tile_of(j) < ntiles; ++j) {
        const int i = tile_of(j), side = i >= a.ntile ? 1 : 0, b = j & 1;
        const int64_t row0 = (int64_t)(i - side * a.ntile) * T;
        const uint32_t xs = sb + (b ? X1 : X0);
        wait_loads_nosync(ctl, ld, 1u << b);
        {  // this thread's quarter of the row's squared norm (columns 32qd .. 32qd+31)
            const uint32_t xt = xs + (uint32_t)(qd >> 1) * TILE;
            float s = 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const uint4 v = ld_shared_v4(xt + sw128_off(r, 4 * (qd & 1) + ch));
                const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float x0 = bf16_lo(ws[k]), x1 = bf16_hi(ws[k]);
                    s = fmaf(x0, x0, s);
                    s = fmaf(x1, x1, s);
                }
            }
            rn[(b * 4 + qd) * 128 + r] = s;
        }
        if (*(volatile uint32_t *)&ctl->abort == 0u && !mbar_wait(&mb[b], (uint32_t)(j >> 1) & 1u, WAIT_LIMIT_NS)) {
            ctl->abort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        fence_after_sync();
        // the norms are complete, tile j's MMA has read its rows buffer, and every thread has
        // read accumulator (j + 1) & 1 for tile j - 1
        __syncthreads();
        if (*(volatile uint32_t *)&ctl->abort != 0u) break;
        if (tile_of(j + 2) < ntiles) issue_load(j + 2);
        if (threadIdx.x == 0 && tile_of(j + 1) < ntiles) issue_mma(j + 1);  // runs under this tile's read-out
        const float n2 = (rn[b * 512 + r] + rn[b * 512 + 128 + r]) + (rn[b * 512 + 256 + r] + rn[b * 512 + 384 + r]);
        const float inv = 1.f / fmaxf(sqrtf(n2), kNormEps);
        uint32_t w[5][8];
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            const int c8 = qd + 4 * k;
            if (c8 < npw8) tmem_ld8_nowait(tlane(tm + (uint32_t)b * 256u, 8u * c8), w[k]);
        }
        tmem_wait_ld();
        fence_before_sync();
        if (row0 + r < a.N) {
            float *dst = a.p[side] + (row0 + r) * a.npwp;
#pragma unroll
            for (int k = 0; k < 5; ++k) {
                const int c8 = qd + 4 * k;
                if (c8 >= npw8) break;
                uint32_t o[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) o[m] = __float_as_uint(__uint_as_float(w[k][m]) * inv);
                st_global_v8(dst + 8 * c8, o);
            }
        }
    }
    drain_loads(ctl, ld);
    kernel_teardown(tm, 512);
}

// ------------------------------------------------------------------------------------------
// Segment totals of one (group, half) pass.  MODE 0: H_seg = sum_j phi_g(k_j) [v_j,h | 1]^T
// (the bucket statistics A, B of zh §2.2 over the segment, for the group's tables and the
// half's value columns).  MODE 1: G_seg = sum_i phi_g(q_i) / den_i [dO_i,h | c_i]^T, with c
// in half 0 only (the backward's query-side statistics).   grid: (2 * groups) x nseg: the
// passes of a segment side by side, so that they read the segment's rows from L2 together.
// As in the 256-feature kernels, the CTA's two groups of 256 threads take alternate chunks,
// each with its own tiles, TMEM accumulator and barriers, and the two sums are added at the
// end.  Thread (r, hh) of a thread group owns row r and quarters 2hh, 2hh+1 of the features.
// ------------------------------------------------------------------------------------------
namespace wagg_smem {
constexpr uint32_t PT = 0;                  // projections of the group's rows [128][40] fp32
constexpr uint32_t PHI = PTILE;             // Phi [128][256]
constexpr uint32_t VA = PHI + 4 * TILE;     // value tile [128][80] (5 atoms)
constexpr uint32_t GROUP = VA + 5 * VA128;  // bytes per thread group
constexpr uint32_t BAR = 2 * GROUP;
constexpr uint32_t VBAR = BAR + 64;         // per thread group: its state update is done
constexpr uint32_t TOTAL = VBAR + 64;
constexpr uint32_t RED = GROUP;             // at the end: thread group 1's state, fp32 [256][80]
static_assert(256 * 80 * 4 <= GROUP, "reduction buffer");
}  // namespace wagg_smem

template <int MODE>
__global__ void __launch_bounds__(NTH, 1) wide_agg(const __grid_constant__ WideArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace wagg_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    const int seg = blockIdx.y, pass = blockIdx.x, g = pass >> 1, hv = pass & 1;
    if (MODE == 0 && a.ctx_tag && *a.ctx_tag == kCtxTag) {  // the forward saved them (already scanned)
        const int64_t off = ((int64_t)pass * a.nseg + seg) * MF * DS;
        for (int i = threadIdx.x; i < MF * DS; i += NTH) a.agg_out[off + i] = a.ctx_states[off + i];
        return;
    }
    const int gi = threadIdx.x >> 8, gt = threadIdx.x & 255;
    const int r = gt & 127, hh = gt >> 7;
    const bool leader = gt == 0;
    const uint32_t sb = smem_u32(sm), gb = sb + (uint32_t)gi * GROUP;
    uint8_t *pg = sm + gi * GROUP + PT, *phig = sm + gi * GROUP + PHI, *vag = sm + gi * GROUP + VA;
    uint64_t *vbar = reinterpret_cast<uint64_t *>(sm + VBAR) + gi;
    volatile uint32_t *gabort = gi ? &ctl->abort_b : &ctl->abort;
    const CUtensorMap *pmap = MODE == 0 ? &a.tm_pk : &a.tm_pq;
    const CUtensorMap *vmap = MODE == 0 ? &a.tm_v : &a.tm_do;
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t *>(sm + VBAR), 1);
        mbar_init(reinterpret_cast<uint64_t *>(sm + VBAR) + 1, 1);
    }
    const uint32_t tm = kernel_setup(ctl, 512, nullptr, nullptr, nullptr);
    const uint32_t tg = tm + 256u * gi;  // this thread group's state: rows 0-127 at +0, 128-255 at +80
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) zero_state40(tg, 0, 80, 2 * hh + qq);
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    bool ok = true;
    Loads ld = {};  // barriers 2gi (projections) and 2gi + 1 (values) of this thread group
    auto load_p = [&](int64_t c) {
        uint64_t *bar = arm_load(ctl, ld, 2 * gi, PTILE, leader);
        if (leader) tma_load2(gb + PT, pmap, WPROJ * g, (int)c, bar);
    };
    auto load_v = [&](int64_t c) {
        uint64_t *bar = arm_load(ctl, ld, 2 * gi + 1, TILE, leader);
        if (leader) tma_load3(gb + VA, vmap, 0, (int)c, 4 * hv, bar);
    };
    auto wait_group_load = [&](int b) {  // every thread of the group waits, then the group syncs
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
        group_sync(gi);
        return *gabort == 0u;
    };
    int64_t c0 = t0 + (int64_t)gi * T;  // this thread group's chunks: every other one of the segment
    if (c0 < t1) {
        load_p(c0);
        load_v(c0);
    }
    bool pending = false;  // a state update of this thread group is in flight
    uint32_t vphase = 0;
    for (; c0 < t1 && ok; c0 += 2 * T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        const int64_t cn = c0 + 2 * T;
        if (pending) {  // the last state update has read Phi and the value tile
            if (leader && *gabort == 0u && !mbar_wait(vbar, vphase & 1u, WAIT_LIMIT_NS)) {
                *gabort = 1u;
                atomicExch(&g_tc_error, 1);
            }
            ++vphase;
            group_sync(gi);
            fence_after_sync();
            load_v(c0);
        }
        if (!(ok = wait_group_load(2 * gi))) break;
        float sc = valid ? 1.f : 0.f, col = sc;
        if (MODE == 1) {  // Phi_Q / den_i and column 64 = c_i (half 0) or 0
            float c = 0.f, inv = 0.f;
            if (valid) {
                c = a.cbuf[c0 + r];
                const float dn = a.den[c0 + r];
                inv = dn != 0.f ? 1.f / dn : 0.f;
            }
            sc = inv;
            col = hv == 0 ? c : 0.f;
        }
#pragma unroll 1
        for (int qq = 0; qq < 2; ++qq) {
            float u[10], t[10];
            proj_tanh10(pg, r, 2 * hh + qq, a.beta, u, t);
            write_features64(t, r, 2 * hh + qq, sc, phig);
        }
        if (hh == 1) write_col64(vag, r, col);
        fence_smem_async();
        fence_before_sync();
        group_sync(gi);  // Phi and column 64 are written; the projections tile has been read
        if (cn < t1) load_p(cn);
        if (leader) {
            if (wait_one_load(ctl, ld, 2 * gi + 1, gabort)) {
                fence_after_sync();
                issue_state_update(tg, 0, 80, gb + PHI, gb + VA);
                mma_commit(vbar);
            }
        }
        pending = true;
    }
    if (pending && ok) {  // the thread group's last state update
        if (leader && *gabort == 0u && !mbar_wait(vbar, vphase & 1u, WAIT_LIMIT_NS)) {
            *gabort = 1u;
            atomicExch(&g_tc_error, 1);
        }
        group_sync(gi);
        fence_after_sync();
    }
    drain_loads(ctl, ld);  // thread 0: thread group 0's loads
    if (gi == 1 && leader)
        for (int b = 2; b < 4; ++b)
            if ((ld.pend >> b) & 1u) mbar_wait(&ctl->ld[b], load_parity(ld, b), WAIT_LIMIT_NS);
    __syncthreads();
    if (ctl->abort == 0u && ctl->abort_b == 0u) {  // H = group 0's sum + group 1's sum
        float *red = reinterpret_cast<float *>(sm + RED);
        if (gi == 1) {
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int qd = 2 * hh + qq;
                float hvv[40];
                read_state40(tg, 0, 80, qd, hvv);
                float *dst = red + (128 * (qd & 1) + r) * 80 + 40 * (qd >> 1);
#pragma unroll
                for (int i = 0; i < 40; ++i) dst[i] = hvv[i];
            }
        }
        __syncthreads();
        if (gi == 0) {
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int qd = 2 * hh + qq;
                float hvv[40];
                read_state40(tg, 0, 80, qd, hvv);
                const float *src = red + (128 * (qd & 1) + r) * 80 + 40 * (qd >> 1);
#pragma unroll
                for (int i = 0; i < 40; ++i) hvv[i] += src[i];
                store_state40(hvv, a.agg_out + ((int64_t)pass * a.nseg + seg) * MF * DS, 128 * (qd & 1) + r, qd);
            }
        }
    }
    kernel_teardown(tm, 512);
}

// ------------------------------------------------------------------------------------------
// Causal walk of one (group, half) pass (Algorithm 2, zh §2.3).   grid: 2 (value halves) x
// nseg, NTH + 32 threads; launched once per group, group 0 first.
// The structure is that of the 256-feature walk: Phi_Q in tensor memory, one lane of the last
// warp issuing every TMA load and MMA, hand-overs through mbarriers.  The chunk's projections
// come as two [128][40] fp32 tiles (q, k), loaded a chunk ahead once the features of the
// current chunk have been formed.  Each pass adds its partial numerator Y[:, :64] and den
// Y[:, 64] to fp32 sums over the groups (group 0 stores); wide_finish divides.
// ------------------------------------------------------------------------------------------
namespace wfwd_smem {
constexpr uint32_t PHK = 0;                // Phi_K [128][256]
constexpr uint32_t SB = 4 * TILE;          // masked S as bf16 [128][128]
constexpr uint32_t PQ = SB + 2 * TILE;     // the chunk's q projections of the group [128][40] fp32
constexpr uint32_t PK = PQ + PTILE;        // and k projections
constexpr uint32_t VA0 = PK + PTILE;       // [V_h | 1] [128][80], two buffers (chunk parity)
constexpr uint32_t VA1 = VA0 + 5 * VA128;
constexpr uint32_t HS = VA1 + 5 * VA128;   // staged H [256][80]
constexpr uint32_t BAR = HS + 5 * VA256;
constexpr uint32_t FB = BAR + 64;
constexpr uint32_t TOTAL = FB + 128;
}  // namespace wfwd_smem
namespace wfwd_tmem {
constexpr uint32_t S = 0;       // [128][128]
constexpr uint32_t Y = 128;     // [128][80]
constexpr uint32_t HTOP = 208;  // H rows 0..127
constexpr uint32_t HBOT = 288;  // H rows 128..255
constexpr uint32_t PHQ = 368;   // Phi_Q as bf16 pairs (128 columns)
}  // namespace wfwd_tmem

struct WFwdBars {
    uint64_t rows, v[2];            // TMA: projection tiles; value tile p
    uint64_t s, sv, fin;            // MMA commits
    uint64_t phiq, phik, sbar, done;  // the computing warps' hand-overs (16 arrivals)
};
static_assert(sizeof(WFwdBars) <= 128, "walk barriers");

__global__ void __launch_bounds__(NTH + 32, 1) wide_fwd_walk(const __grid_constant__ WideArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace wfwd_smem;
    namespace tmc = wfwd_tmem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    WFwdBars *fb = reinterpret_cast<WFwdBars *>(sm + FB);
    const int seg = blockIdx.y, h = blockIdx.x, g = a.g;
    const bool issuer_warp = threadIdx.x >= NTH;
    const int r = threadIdx.x & 127, qd = (threadIdx.x >> 7) & 3;
    const uint32_t sb = smem_u32(sm);
    if (threadIdx.x == 0) {
        mbar_init(&fb->rows, 1);
        mbar_init(&fb->v[0], 1);
        mbar_init(&fb->v[1], 1);
        mbar_init(&fb->s, 1);
        mbar_init(&fb->sv, 1);
        mbar_init(&fb->fin, 1);
        mbar_init(&fb->phiq, NTH / 32);
        mbar_init(&fb->phik, NTH / 32);
        mbar_init(&fb->sbar, NTH / 32);
        mbar_init(&fb->done, NTH / 32);
    }
    const uint32_t tm = kernel_setup(ctl, 512, nullptr, nullptr, nullptr);
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    volatile uint32_t *abort_flag = &ctl->abort;
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
            // scalars, not arrays indexed by the chunk parity (those would live in local memory)
            uint32_t ph_v0 = 0, ph_v1 = 0, ph_phiq = 0, ph_phik = 0, ph_sb = 0, ph_done = 0;
            uint32_t n_rows = 0, n_v0 = 0, n_v1 = 0;  // loads issued per barrier
            auto issue_rows = [&](int64_t c) {
                mbar_expect_tx(&fb->rows, 2u * PTILE);
                tma_load2(sb + PQ, &a.tm_pq, WPROJ * g, (int)c, &fb->rows);
                tma_load2(sb + PK, &a.tm_pk, WPROJ * g, (int)c, &fb->rows);
                ++n_rows;
            };
            auto issue_v = [&](int64_t c, int p) {
                mbar_expect_tx(&fb->v[p], TILE);
                tma_load3(sb + (p ? VA1 : VA0), &a.tm_v, 0, (int)c, 4 * h, &fb->v[p]);
                if (p) ++n_v1;
                else ++n_v0;
            };
            if (t0 < t1) {
                issue_rows(t0);
                issue_v(t0, 0);
            }
            bool ok = true, staged = false;  // staged: a Y tile is being written out from SB
            int par = 0;
            for (int64_t c0 = t0; c0 < t1 && ok; c0 += T, par ^= 1) {
                const bool more = c0 + T < t1;
                if (more) issue_v(c0 + T, par ^ 1);  // its buffer was last read by the previous chunk's MMAs
                if (!(ok = wait(&fb->phiq, ph_phiq))) break;
                fence_after_sync();  // Y = Phi_Q H_prev
                issue_k256_tva(tm + tmc::Y, tm + tmc::PHQ, sb + HS, idesc_bf16(128, 80, 0, 1));
                if (!(ok = wait(&fb->phik, ph_phik))) break;
                if (more) issue_rows(c0 + T);  // both projection tiles have been read
                if (!(ok = par ? wait(&fb->v[1], ph_v1) : wait(&fb->v[0], ph_v0))) break;
                if (staged) {  // the mask after this S overwrites SB: the last Y tile has left it
                    bulk_wait_read();
                    staged = false;
                }
                fence_after_sync();  // S = Phi_Q Phi_K^T, then H += Phi_K^T V~
                issue_k256_tkk(tm + tmc::S, tm + tmc::PHQ, sb + PHK, idesc_bf16(128, 128, 0, 0));
                mma_commit(&fb->s);
                issue_state_update(tm, tmc::HTOP, tmc::HBOT, sb + PHK, sb + (par ? VA1 : VA0));
                if (!(ok = wait(&fb->sbar, ph_sb))) break;
                fence_after_sync();  // Y += tril(S) V~
                issue_k128_va(tm + tmc::Y, sb + SB, 0, sb + (par ? VA1 : VA0), idesc_bf16(128, 80, 0, 1), true);
                mma_commit(&fb->sv);
                if (!(ok = wait(&fb->done, ph_done))) break;
                put_tile64(&a.tm_acc, sb + SB, h, (int)c0, !a.first);  // Y[:, :64], staged in SB
                staged = true;
            }
            bulk_wait_all();
            // leave nothing in flight: the last commit covers every MMA issued; then every load
            // group issued has completed (a wait on the parity of the last phase returns at once
            // when that phase is over)
            mma_commit(&fb->fin);
            mbar_wait(&fb->fin, 0u, WAIT_LIMIT_NS);
            if (n_rows) mbar_wait(&fb->rows, (n_rows - 1u) & 1u, WAIT_LIMIT_NS);
            if (n_v0) mbar_wait(&fb->v[0], (n_v0 - 1u) & 1u, WAIT_LIMIT_NS);
            if (n_v1) mbar_wait(&fb->v[1], (n_v1 - 1u) & 1u, WAIT_LIMIT_NS);
        }
    } else {
        {  // start state: fp32 master into TMEM, bf16 copy into the staging tile
            float hv[40];
            load_state40(state_of(a, 2 * g + h, seg), 128 * (qd & 1) + r, qd, tm, tmc::HTOP, tmc::HBOT, hv);
            stage40(hv, 128 * (qd & 1) + r, qd, sm + HS);
        }
        fence_smem_async();
        fence_before_sync();
        asm volatile("bar.sync 1, %0;" ::"n"(NTH) : "memory");  // the staged state before the first Y
        uint32_t ph_rows = 0, ph_s = 0, ph_sv = 0;
        const bool elect = (threadIdx.x & 31) == 0;
        auto hand_over = [&](uint64_t *bar) {
            __syncwarp();
            if (elect) mbar_arrive(bar);
        };
        int par = 0;
        bool ok = true;
        for (int64_t c0 = t0; c0 < t1 && ok; c0 += T, par ^= 1) {
            const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
            const bool valid = r < nv;
            if (!(ok = wait(&fb->rows, ph_rows))) break;
            if (qd == 2) write_col64(sm + (par ? VA1 : VA0), r, valid ? 1.f : 0.f);
            {  // Phi_Q into tensor memory
                float u[10], t[10];
                proj_tanh10(sm + PQ, r, qd, a.beta, u, t);
                write_features64_tmem(t, qd, valid ? 1.f : 0.f, tm, tmc::PHQ);
            }
            tmem_wait_st();
            fence_before_sync();
            hand_over(&fb->phiq);
            {
                float u[10], t[10];
                proj_tanh10(sm + PK, r, qd, a.beta, u, t);
                write_features64(t, r, qd, valid ? 1.f : 0.f, sm + PHK);
            }
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->phik);
            if (!(ok = wait(&fb->s, ph_s))) break;
            fence_after_sync();
            mask_block<false, false, false>(tm, tmc::S, r, qd, 0.f, nullptr, sm + SB);  // j <= i
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->sbar);
            if (!(ok = wait(&fb->sv, ph_sv))) break;
            fence_after_sync();
            {  // this pass's Y[:, 16qd ..] and Y[:, 64] into the sums over the groups
                uint32_t w[16], dn8[8];
                tmem_ld16_nowait(tlane(tm, tmc::Y + 16u * qd), w);
                tmem_ld8_nowait(tlane(tm, tmc::Y + 64u), dn8);
                tmem_wait_ld();
                float y[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) y[i] = __uint_as_float(w[i]);
                stage_row16(sb + SB, r, qd, y);  // the issuer writes the tile out (SB is free: S V~ is done)
                if (valid && h == 0 && qd == 0) {
                    const float dn = __uint_as_float(dn8[0]);
                    if (a.first)
                        a.dacc[c0 + r] = dn;
                    else
                        red_add_f32(a.dacc + c0 + r, dn);
                }
            }
            {  // stage the updated state for the next chunk's read-out
                float hv[40];
                read_state40(tm, tmc::HTOP, tmc::HBOT, qd, hv);
                stage40(hv, 128 * (qd & 1) + r, qd, sm + HS);
            }
            fence_smem_async();
            fence_before_sync();
            hand_over(&fb->done);
        }
    }
    kernel_teardown(tm, 512);
}

// ==========================================================================================
// Backward of one (group, half) pass.  With c_i = -(dO_i . o_i) over all 128 columns and
// dY_i = [dO_i, c_i] / den_i, the pass's share (value half h, features of group g) is that of
// the 256-feature walks with dO, v restricted to the half's 64 columns and the c terms kept
// in half 0 only (c multiplies the ones column, which both halves carry):
//   dq walk:    dPhi_Q[i] = (dO_i,h H_prev[:, :64]^T + c'_i H_prev[:, 64]
//                             + sum_{j<=i} (v_j,h . dO_i,h + c'_i) Phi_K[j]) / den_i
//   dk/dv walk: dV[j]_h   = Phi_K[j] G_next[:, :64] + sum_{i>=j} (Phi_K[j] . Phi_Q'[i]) dO_i,h
//               dPhi_K[j] = [v_j,h, 1] G_next^T + sum_{i>=j} (v_j,h . dO_i,h + c'_i) Phi_Q'[i]
// with c' = c in half 0 and 0 in half 1.  The feature-map VJP turns dPhi into dLoss/dp^ for
// the group's 40 projections; the halves' shares are added in dp (half 0 stores, half 1 adds),
// and wide_dx finishes dq and dk.  dv is summed over the groups like the forward's numerator.
// ==========================================================================================

// c_i = -(dO_i . o_i) for `rows` rows of 128 bf16 columns: 16 threads per row.
__global__ void __launch_bounds__(256) wide_rowc(const __nv_bfloat16 *o, const __nv_bfloat16 *dout, float *c,
                                                 int64_t rows)
{
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = t >> 4;
    const int part = (int)(t & 15);
    float s = 0.f;
    if (row < rows) {
        const uint4 a = reinterpret_cast<const uint4 *>(o + row * WD)[part];
        const uint4 b = reinterpret_cast<const uint4 *>(dout + row * WD)[part];
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s = fmaf(bf16_lo(aw[i]), bf16_lo(bw[i]), s);
            s = fmaf(bf16_hi(aw[i]), bf16_hi(bw[i]), s);
        }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (row < rows && part == 0) c[row] = -s;
}

namespace wbq_smem {
constexpr uint32_t RA = 0;                  // q, k projection tiles at load; Phi_K [128][256] after the features
constexpr uint32_t PQ = RA;
constexpr uint32_t PK = RA + PTILE;
constexpr uint32_t PHK = RA;
constexpr uint32_t PB = 4 * TILE;           // masked P'' bf16 [128][128]
constexpr uint32_t VA = PB + 2 * TILE;      // [V_h | 1] [128][80]
constexpr uint32_t DOV = VA + 5 * VA128;    // dO_h [128][64]
constexpr uint32_t HSHI = DOV + 4 * VA128;  // staged H[:, :64] bf16 hi [256][64]
constexpr uint32_t HSLO = HSHI + 4 * VA256; // and lo
constexpr uint32_t HDEN = HSLO + 4 * VA256; // H[:, 64] fp32 [2 buffers][256]
constexpr uint32_t ROWC = HDEN + 2048;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t BAR = ROWINV + 512;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace wbq_smem
namespace wbq_tmem {
constexpr uint32_t P = 128;    // [128][128]
constexpr uint32_t DPHI = 0;   // [128][256]
constexpr uint32_t HTOP = 256;
constexpr uint32_t HBOT = 336;
}  // namespace wbq_tmem

// ------------------------------------------------------------------------------------------
// dq walk of every (group, half) pass (chunks in order, prefix state H).   grid: (2 * groups)
// x nseg.  The two halves' shares of dLoss/dp^ are added in memory onto zeros.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 1) wide_bwd_q_walk(const __grid_constant__ WideArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace wbq_smem;
    namespace tmc = wbq_tmem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *hden = reinterpret_cast<float *>(sm + HDEN);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.y, g = blockIdx.x >> 1, h = blockIdx.x & 1;
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const uint32_t tm = kernel_setup(ctl, 512, nullptr, nullptr, nullptr);
    {
        float hv[40];
        load_state40(state_of(a, 2 * g + h, seg), 128 * (qd & 1) + r, qd, tm, tmc::HTOP, tmc::HBOT, hv);
        stage40_hilo(hv, 128 * (qd & 1) + r, qd, sm + HSHI, sm + HSLO, hden);
    }
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};
    auto issue_loads = [&](int64_t c) {  // the chunk's projections of both sides, dO_h and v_h
        uint64_t *bar = arm_load(ctl, ld, 0, 2u * PTILE + 2u * TILE);
        if (threadIdx.x == 0) {
            tma_load2(sb + PQ, &a.tm_pq, WPROJ * g, (int)c, bar);
            tma_load2(sb + PK, &a.tm_pk, WPROJ * g, (int)c, bar);
            tma_load3(sb + DOV, &a.tm_do, 0, (int)c, 4 * h, bar);
            tma_load3(sb + VA, &a.tm_v, 0, (int)c, 4 * h, bar);
        }
    };
    if (t0 < t1) issue_loads(t0);
    int par = 0;
    for (int64_t c0 = t0; c0 < t1 && ok; c0 += T, par ^= 1) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        if (!(ok = wait_loads(ctl, ld, 1u))) break;
        if (threadIdx.x == 3 * 128) {  // P'' = dO V^T (needs no features) while the features are formed
            fence_after_sync();
            issue_va_va(tm + tmc::P, sb + DOV, T, sb + VA, T, 4, idesc_bf16(128, 128, 0, 0), false);
            mma_commit(&ctl->bar);
        }
        if (qd == 2) {
            float c = 0.f, inv = 0.f;
            if (valid) {
                c = a.cbuf[c0 + r];
                const float dn = a.den[c0 + r];
                inv = dn != 0.f ? 1.f / dn : 0.f;
            }
            rowc[r] = h == 0 ? c : 0.f;
            rowinv[r] = inv;
        }
        if (qd == 3) write_col64(sm + VA, r, valid ? 1.f : 0.f);
        float u[10], t[10], uk[10], tk[10];
        proj_tanh10(sm + PQ, r, qd, a.beta, u, t);
        proj_tanh10(sm + PK, r, qd, a.beta, uk, tk);
        fence_smem_async();
        if (!(ok = wait_mma(ctl, phase, 3 * 128))) break;  // every thread has read the projection tiles
        const float c_r = rowc[r], invden_r = rowinv[r];
        write_features64(tk, r, qd, valid ? 1.f : 0.f, sm + PHK);
        mask_block<false, true, false>(tm, tmc::P, r, qd, c_r, nullptr, sm + PB);  // v_j.dO_i + c'_i, j <= i
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            // D = dO H_prev[:, :64]^T (hi + lo) + tril(P'') Phi_K, then H += Phi_K^T V~
            issue_va_va(tm + tmc::DPHI, sb + DOV, T, sb + HSHI, 256, 4, idesc_bf16(128, 256, 0, 0), false);
            issue_va_va(tm + tmc::DPHI, sb + DOV, T, sb + HSLO, 256, 4, idesc_bf16(128, 256, 0, 0), true);
            issue_k128_k128mn(tm + tmc::DPHI, sb + PB, sb + PHK, idesc_bf16(128, 256, 0, 1), true);
            issue_state_update(tm, tmc::HTOP, tmc::HBOT, sb + PHK, sb + VA);
            mma_commit(&ctl->bar);
        }
        wait_mma_each(ctl, phase);
        if (c0 + T < t1) issue_loads(c0 + T);  // Phi_K, P'', V~ and dO have been read
        {  // dphi = (D + c'_i H_prev[:, 64]) / den_i -> dLoss/dp^ of the group's projections
            float dp[10];
            features_vjp10(tm, tmc::DPHI, qd, a.beta, valid, u, t, hden + 256 * par, c_r, invden_r, dp);
            if (valid) add10(a.dp + (c0 + r) * a.npwp + WPROJ * g + 10 * qd, dp, qd);
        }
        {  // the updated state, staged for the next chunk (its den column into the other buffer)
            float hv[40];
            read_state40(tm, tmc::HTOP, tmc::HBOT, qd, hv);
            stage40_hilo(hv, 128 * (qd & 1) + r, qd, sm + HSHI, sm + HSLO, hden + 256 * (par ^ 1));
        }
        // the staged state and the TMEM reads are handed over by the next chunk's first barrier
        fence_smem_async();
        fence_before_sync();
    }
    drain_loads(ctl, ld);
    kernel_teardown(tm, 512);
}

namespace wbkv_smem {
constexpr uint32_t PHQ = 0;                // Phi_Q' [128][256]
constexpr uint32_t PHK = 4 * TILE;         // k, q projection tiles at load; Phi_K; then masked S'^T and P'
constexpr uint32_t PK = PHK;
constexpr uint32_t PQ = PHK + PTILE;
constexpr uint32_t STB = PHK;              // tiles 0-1
constexpr uint32_t PPB = PHK + 2 * TILE;   // tiles 2-3
constexpr uint32_t VA = PHK + 4 * TILE;    // [V_h | 1] [128][80]
constexpr uint32_t DOC = VA + 5 * VA128;   // [dO_h | c'] [128][80]
constexpr uint32_t GS = DOC + 5 * VA128;   // staged G [256][80]
constexpr uint32_t ROWC = GS + 5 * VA256;
constexpr uint32_t ROWINV = ROWC + 512;
constexpr uint32_t BAR = ROWINV + 512;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace wbkv_smem
namespace wbkv_tmem {
constexpr uint32_t ST = 0;      // S'^T [128][128]
constexpr uint32_t PP = 128;    // V dO^T [128][128]
constexpr uint32_t DPHI = 0;    // [128][256]
constexpr uint32_t GTOP = 256;
constexpr uint32_t GBOT = 336;
constexpr uint32_t DVT = 416;   // dV_h [128][64]
}  // namespace wbkv_tmem

// ------------------------------------------------------------------------------------------
// dk/dv walk of one group for both halves (chunks in reverse, suffix state G).   grid: 2
// (value halves) x nseg; launched once per group, group 0 first.  dv is summed over the
// groups (group 0 stores) by TMA from a staged tile, dLoss/dp^ over the halves (added onto
// zeros).
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NTH, 1) wide_bwd_kv_walk(const __grid_constant__ WideArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace wbkv_smem;
    namespace tmc = wbkv_tmem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *rowc = reinterpret_cast<float *>(sm + ROWC), *rowinv = reinterpret_cast<float *>(sm + ROWINV);
    const int seg = blockIdx.y, g = a.g, h = blockIdx.x;
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const uint32_t tm = kernel_setup(ctl, 512, nullptr, nullptr, nullptr);
    {
        float hv[40];
        load_state40(state_of(a, 2 * g + h, seg), 128 * (qd & 1) + r, qd, tm, tmc::GTOP, tmc::GBOT, hv);
        stage40(hv, 128 * (qd & 1) + r, qd, sm + GS);
    }
    int64_t t0, t1;
    seg_bounds(a.seg_len, a.N, seg, t0, t1);
    const int64_t nchunks = (t1 - t0 + T - 1) / T;
    uint32_t phase = 0;
    bool ok = true;
    Loads ld = {};
    auto issue_loads = [&](int64_t c) {  // the chunk's projections of both sides, v_h and dO_h
        uint64_t *bar = arm_load(ctl, ld, 0, 2u * PTILE + 2u * TILE);
        if (threadIdx.x == 0) {
            tma_load2(sb + PK, &a.tm_pk, WPROJ * g, (int)c, bar);
            tma_load2(sb + PQ, &a.tm_pq, WPROJ * g, (int)c, bar);
            tma_load3(sb + VA, &a.tm_v, 0, (int)c, 4 * h, bar);
            tma_load3(sb + DOC, &a.tm_do, 0, (int)c, 4 * h, bar);
        }
    };
    if (nchunks > 0) issue_loads(t0 + (nchunks - 1) * T);
    int64_t staged_row0 = -1;  // the previous chunk's dV tile, staged in PHQ, not yet written out
    for (int64_t ci = nchunks - 1; ci >= 0 && ok; --ci) {
        const int64_t c0 = t0 + ci * T;
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : T);
        const bool valid = r < nv;
        if (!(ok = wait_loads(ctl, ld, 1u))) break;
        if (threadIdx.x == 0 && staged_row0 >= 0)  // the barrier above published it
            put_tile64(&a.tm_acc, sb + PHQ, h, (int)staged_row0, !a.first);
        if (threadIdx.x == 3 * 128) {  // P' = V dO^T while the features are formed
            fence_after_sync();
            issue_va_va(tm + tmc::PP, sb + VA, T, sb + DOC, T, 4, idesc_bf16(128, 128, 0, 0), false);
            mma_commit(&ctl->bar);
        }
        if (qd == 2) {  // c'_i and 1/den_i (0 beyond the valid rows); c' into column 64 of [dO | c']
            float c = 0.f, inv = 0.f;
            if (valid) {
                c = a.cbuf[c0 + r];
                const float dn = a.den[c0 + r];
                inv = dn != 0.f ? 1.f / dn : 0.f;
            }
            rowc[r] = h == 0 ? c : 0.f;
            rowinv[r] = inv;
            write_col64(sm + DOC, r, rowc[r]);
        }
        if (qd == 3) write_col64(sm + VA, r, valid ? 1.f : 0.f);
        float u[10], t[10], uq[10], tq[10];
        proj_tanh10(sm + PK, r, qd, a.beta, u, t);
        proj_tanh10(sm + PQ, r, qd, a.beta, uq, tq);
        fence_smem_async();
        if (!(ok = wait_mma(ctl, phase, 3 * 128))) break;  // every thread has read the projection tiles
        write_features64(t, r, qd, valid ? 1.f : 0.f, sm + PHK);
        if (threadIdx.x == 0 && staged_row0 >= 0) bulk_wait_read();  // PHQ is rewritten next
        staged_row0 = -1;
        publish_smem();
        if (threadIdx.x == 0) {  // dV = Phi_K G_next[:, :64], while Phi_Q' is formed
            fence_after_sync();
            issue_k256_va(tm + tmc::DVT, sb + PHK, sb + GS, idesc_bf16(128, 64, 0, 1), false);
        }
        write_features64(tq, r, qd, rowinv[r], sm + PHQ);  // Phi_Q' = Phi_Q / den
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            issue_k256_kk(tm + tmc::ST, sb + PHK, sb + PHQ, idesc_bf16(128, 128, 0, 0), false);  // S'^T
            mma_commit(&ctl->bar);  // also reports dV: it is complete before the masks overwrite Phi_K
        }
        wait_mma_each(ctl, phase);
        mask_block<true, false, false>(tm, tmc::ST, r, qd, 0.f, nullptr, sm + STB);
        mask_block<true, false, true>(tm, tmc::PP, r, qd, 0.f, rowc, sm + PPB);  // v_j.dO_i + c'_i, i >= j
        publish_smem();
        if (threadIdx.x == 0) {
            fence_after_sync();
            // dV += triu(S'^T) dO; dPhi_K = [V | 1] G_next^T + triu(P') Phi_Q'; G += Phi_Q'^T [dO | c']
            issue_k128_va(tm + tmc::DVT, sb + STB, 0, sb + DOC, idesc_bf16(128, 64, 0, 1), true);
            issue_va_va(tm + tmc::DPHI, sb + VA, T, sb + GS, 256, 5, idesc_bf16(128, 256, 0, 0), false);
            issue_k128_k128mn(tm + tmc::DPHI, sb + PPB, sb + PHQ, idesc_bf16(128, 256, 0, 1), true);
            issue_state_update(tm, tmc::GTOP, tmc::GBOT, sb + PHQ, sb + DOC);
            mma_commit(&ctl->bar);
        }
        wait_mma_each(ctl, phase);
        if (ci > 0) issue_loads(c0 - T);  // Phi_K / masks, V~ and [dO | c'] have been read
        if (ci > 0 && qd == 2) {  // the next chunk's c_i and den_i into L2
            prefetch_l2(a.cbuf + c0 - T + r);
            prefetch_l2(a.den + c0 - T + r);
        }
        {  // this pass's dV[:, 16qd ..], staged for the sum over the groups (wide_finish writes dv)
            uint32_t w[16];
            tmem_ld16_nowait(tlane(tm, tmc::DVT + 16u * qd), w);
            tmem_wait_ld();
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = __uint_as_float(w[i]);
            stage_row16(sb + PHQ, r, qd, y);  // Phi_Q' has been read; written out at the next barrier
            staged_row0 = c0;
        }
        {
            float dp[10];
            features_vjp10(tm, tmc::DPHI, qd, a.beta, valid, u, t, nullptr, 0.f, 1.f, dp);
            if (valid) add10(a.dp + (c0 + r) * a.npwp + WPROJ * g + 10 * qd, dp, qd);
        }
        {
            float hv[40];
            read_state40(tm, tmc::GTOP, tmc::GBOT, qd, hv);
            stage40(hv, 128 * (qd & 1) + r, qd, sm + GS);
        }
        // the staged state and the TMEM reads are handed over by the next chunk's first barrier
        fence_smem_async();
        fence_before_sync();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (ok && staged_row0 >= 0) put_tile64(&a.tm_acc, sb + PHQ, h, (int)staged_row0, !a.first);
        bulk_wait_all();
    }
    drain_loads(ctl, ld);
    kernel_teardown(tm, 512);
}

// ------------------------------------------------------------------------------------------
// From the fp32 sums over the feature groups of one head: out = num / den in bf16 and den
// (den_out, may be null) when den is given, else dv = the sum in bf16.  16 threads per row.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) wide_finish(const float *acc, const float *den, __nv_bfloat16 *dst,
                                                   float *den_out, int64_t rows)
{
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = t >> 4;
    const int part = (int)(t & 15);
    if (row >= rows) return;
    uint32_t w8[8];
    ld_global_v8(acc + row * WD + 8 * part, w8);
    const float4 x0 = make_float4(__uint_as_float(w8[0]), __uint_as_float(w8[1]), __uint_as_float(w8[2]),
                                  __uint_as_float(w8[3]));
    const float4 x1 = make_float4(__uint_as_float(w8[4]), __uint_as_float(w8[5]), __uint_as_float(w8[6]),
                                  __uint_as_float(w8[7]));
    float sc = 1.f;
    if (den) {
        const float dn = den[row];
        sc = dn != 0.f ? 1.f / dn : 0.f;
        if (den_out && part == 0) den_out[row] = dn;
    }
    reinterpret_cast<uint4 *>(dst + row * WD)[part] =
        make_uint4(pack_bf16x2(x0.x * sc, x0.y * sc), pack_bf16x2(x0.z * sc, x0.w * sc),
                   pack_bf16x2(x1.x * sc, x1.y * sc), pack_bf16x2(x1.z * sc, x1.w * sc));
}

// ------------------------------------------------------------------------------------------
// dx of the rows of one head (one or two sides: q, k) from dLoss/dp^ (p^ = W x^,
// x^ = x / max(|x|, eps)): dX^ = dp^ W on the tensor core (dp^ and W each as bf16 hi + lo;
// the lo x lo product is left out), then dx = (dX^ - x^ (x^ . dX^)) / |x|.  Persistent over
// the 128-row tiles of side 0, then side 1.
// grid: min(tiles, SMs), 512 threads
// ------------------------------------------------------------------------------------------
struct DxArgs {
    const __nv_bfloat16 *x[2];  // rows of the head [N][128] per side
    const float *dp[2];         // [N][npwp] dLoss/dp^ per side
    const float *W;             // [npw][128]
    __nv_bfloat16 *dx[2];       // gradient of the rows [N][128] per side
    int64_t N;
    int nsides, ntile, npw, npwp, kp;  // kp = npwp rounded up to 64: the MMA's K
};

constexpr uint32_t BT_MAX = 192u * 128u;  // one N-half of W as MN-major rows [kp <= 192][64]
namespace dx_smem {
constexpr uint32_t AHI = 0;                  // dp^ hi, K-major [128][kp] (kp / 64 K128 tiles)
constexpr uint32_t ALO = 3 * TILE;           // and lo
constexpr uint32_t BHI = 6 * TILE;           // W hi, MN-major: N-half nh at nh * kp * 128
constexpr uint32_t BLO = BHI + 2 * BT_MAX;   // and lo
constexpr uint32_t XCH = BLO + 2 * BT_MAX;   // partial sums [2][512]
constexpr uint32_t BAR = XCH + 4096;
constexpr uint32_t TOTAL = BAR + 64;
}  // namespace dx_smem

__global__ void __launch_bounds__(NTH, 1) wide_dx(const __grid_constant__ DxArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_base(smem_raw);
    using namespace dx_smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(sm + BAR);
    float *xch = reinterpret_cast<float *>(sm + XCH);
    const int r = threadIdx.x & 127, qd = threadIdx.x >> 7;
    const uint32_t sb = smem_u32(sm);
    const uint32_t bt = (uint32_t)a.kp * 128u;  // bytes of one N-half of W
    // W [npw][128] fp32 -> bf16 hi + lo, MN-major: element (k, n) of N-half n / 64 at row k
    for (int e = threadIdx.x; e < a.kp * 64; e += NTH) {
        const int kk = e >> 6, n = 2 * (e & 63);
        float2 w = make_float2(0.f, 0.f);
        if (kk < a.npw) w = *reinterpret_cast<const float2 *>(a.W + (int64_t)kk * WD + n);
        const uint32_t hi = pack_bf16x2(w.x, w.y);
        const uint32_t lo = pack_bf16x2(w.x - bf16_lo(hi), w.y - bf16_hi(hi));
        const uint32_t off = (uint32_t)(n >> 6) * bt + sw128_off(kk, (n & 63) >> 3) + (n & 7) * 2;
        *reinterpret_cast<uint32_t *>(sm + BHI + off) = hi;
        *reinterpret_cast<uint32_t *>(sm + BLO + off) = lo;
    }
    const uint32_t tm = kernel_setup(ctl, 128, nullptr, nullptr, nullptr);
    const int ntiles = a.nsides * a.ntile, kp8 = a.kp >> 3, np8 = a.npwp >> 3;
    const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
    uint32_t phase = 0;
    for (int i = blockIdx.x; i < ntiles; i += gridDim.x) {
        const int side = i >= a.ntile ? 1 : 0;
        const int64_t row = (int64_t)(i - side * a.ntile) * T + r;
        const bool valid = row < a.N;
        {  // this CTA's next tile: its dp^ and x rows into L2 while this one is worked on
            const int in = i + (int)gridDim.x;
            const int sn = in >= a.ntile ? 1 : 0;
            const int64_t rn = (int64_t)(in - sn * a.ntile) * T + r;
            if (in < ntiles && rn < a.N) {
                const char *pd = reinterpret_cast<const char *>(a.dp[sn] + rn * a.npwp);
                const int bytes = 4 * a.npwp;
                for (int off = 128 * qd; off < bytes; off += 512) prefetch_l2(pd + off);
                if (qd == 3) prefetch_l2(pd + bytes - 4);  // the row's last line, if it starts mid-line
                if (qd < 2) prefetch_l2(a.x[sn] + rn * WD + 64 * qd);
            }
        }
        // this thread's 8-column chunks qd, qd + 4, ... (at most 6) of the row's dp^ as hi + lo
        float4 v[6][2];
#pragma unroll
        for (int k = 0; k < 6; ++k) {
            const int c8 = qd + 4 * k;
            if (valid && c8 < np8) {
                uint32_t w8[8];
                ld_global_v8(a.dp[side] + row * a.npwp + 8 * c8, w8);
                v[k][0] = make_float4(__uint_as_float(w8[0]), __uint_as_float(w8[1]), __uint_as_float(w8[2]),
                                      __uint_as_float(w8[3]));
                v[k][1] = make_float4(__uint_as_float(w8[4]), __uint_as_float(w8[5]), __uint_as_float(w8[6]),
                                      __uint_as_float(w8[7]));
            } else {
                v[k][0] = v[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int k = 0; k < 6; ++k) {
            const int c8 = qd + 4 * k;
            if (c8 >= kp8) break;
            const float x[8] = {v[k][0].x, v[k][0].y, v[k][0].z, v[k][0].w, v[k][1].x, v[k][1].y, v[k][1].z, v[k][1].w};
            uint32_t wh[4], wl[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                wh[m] = pack_bf16x2(x[2 * m], x[2 * m + 1]);
                wl[m] = pack_bf16x2(x[2 * m] - bf16_lo(wh[m]), x[2 * m + 1] - bf16_hi(wh[m]));
            }
            const uint32_t off = (uint32_t)(c8 >> 3) * TILE + sw128_off(r, c8 & 7);
            st_shared_v4(sb + AHI + off, wh[0], wh[1], wh[2], wh[3]);
            st_shared_v4(sb + ALO + off, wl[0], wl[1], wl[2], wl[3]);
        }
        publish_smem();
        if (threadIdx.x == 0 && ctl->abort == 0u) {
            fence_after_sync();
            const uint64_t ah = sdesc(sb + AHI, 16, 1024, LAYOUT_SW128), al = sdesc(sb + ALO, 16, 1024, LAYOUT_SW128);
            const uint64_t bh = sdesc(sb + BHI, bt, 1024, LAYOUT_SW128), bl = sdesc(sb + BLO, bt, 1024, LAYOUT_SW128);
            for (int kk = 0; kk < a.kp / 16; ++kk) {
                const uint32_t ao = ((kk >> 2) * TILE + (kk & 3) * 32) >> 4, bo = kk * (2048 >> 4);
                mma_bf16(tm, ah + ao, bh + bo, idesc, kk > 0 ? 1u : 0u);
                mma_bf16(tm, ah + ao, bl + bo, idesc, 1u);
                mma_bf16(tm, al + ao, bh + bo, idesc, 1u);
            }
            mma_commit(&ctl->bar);
        }
        wait_mma_each(ctl, phase);
        uint32_t w[2][16];
        tmem_ld16_nowait(tlane(tm, 32u * qd), w[0]);
        tmem_ld16_nowait(tlane(tm, 32u * qd + 16u), w[1]);
        float x[32];
        if (valid) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.x[side] + row * WD + 32 * qd);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 v = src[k];
                const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    x[8 * k + 2 * m] = bf16_lo(ws[m]);
                    x[8 * k + 2 * m + 1] = bf16_hi(ws[m]);
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) x[k] = 0.f;
        }
        tmem_wait_ld();
        fence_before_sync();
        float ss = 0.f, dd = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            ss = fmaf(x[k], x[k], ss);
            dd = fmaf(x[k], __uint_as_float(w[k >> 4][k & 15]), dd);
        }
        xch[threadIdx.x] = ss;
        xch[512 + threadIdx.x] = dd;
        // the four quarters of this thread's 32 rows are the warps w, w+4, w+8, w+12: they alone meet
        asm volatile("bar.sync %0, 128;" ::"r"(1 + (int)((threadIdx.x >> 5) & 3)) : "memory");
        if (valid) {
            const float n2 = (xch[r] + xch[128 + r]) + (xch[256 + r] + xch[384 + r]);
            const float dot = (xch[512 + r] + xch[640 + r]) + (xch[768 + r] + xch[896 + r]);
            const float rawn = sqrtf(n2), inv = 1.f / fmaxf(rawn, kNormEps);
            const float pj = rawn > kNormEps ? dot * inv * inv : 0.f;  // x^ . dX^ / |x|
            float y[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) y[k] = (__uint_as_float(w[k >> 4][k & 15]) - x[k] * pj) * inv;
            __nv_bfloat16 *dst = a.dx[side] + row * WD + 32 * qd;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint32_t pk[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) pk[m] = pack_bf16x2(y[16 * k + 2 * m], y[16 * k + 2 * m + 1]);
                st_global_v8(dst + 16 * k, pk);
            }
        }
    }
    kernel_teardown(tm, 128);
}

// TMA destinations 1024-byte aligned; every CTA within the shared-memory limit.
static_assert(wagg_smem::PHI % 1024 == 0 && wagg_smem::VA % 1024 == 0 && wagg_smem::GROUP % 1024 == 0,
              "aggregate tiles");
static_assert(wfwd_smem::PQ % 1024 == 0 && wfwd_smem::PK % 1024 == 0 && wfwd_smem::VA0 % 1024 == 0 &&
                  wfwd_smem::VA1 % 1024 == 0 && wfwd_smem::HS % 1024 == 0 && wfwd_smem::SB % 1024 == 0,
              "walk tiles");
static_assert(proj_smem::WHI % 1024 == 0 && proj_smem::WLO % 1024 == 0 && WTILE_MAX % 1024 == 0,
              "projection tiles");
static_assert(wbq_smem::PK % 1024 == 0 && wbq_smem::PB % 1024 == 0 && wbq_smem::VA % 1024 == 0 &&
                  wbq_smem::DOV % 1024 == 0 && wbq_smem::HSHI % 1024 == 0 && wbq_smem::HSLO % 1024 == 0,
              "dq walk tiles");
static_assert(wbkv_smem::PHK % 1024 == 0 && wbkv_smem::PQ % 1024 == 0 && wbkv_smem::VA % 1024 == 0 &&
                  wbkv_smem::DOC % 1024 == 0 && wbkv_smem::GS % 1024 == 0,
              "dk/dv walk tiles");
static_assert(dx_smem::ALO % 1024 == 0 && dx_smem::BHI % 1024 == 0 && dx_smem::BLO % 1024 == 0 &&
                  (BT_MAX / 3) % 1024 == 0,
              "dx tiles");
static_assert(dx_smem::TOTAL + 1024 <= 232448 && proj_smem::TOTAL + 1024 <= 232448 && wagg_smem::TOTAL + 1024 <= 232448 &&
                  wfwd_smem::TOTAL + 1024 <= 232448 && wbq_smem::TOTAL + 1024 <= 232448 &&
                  wbkv_smem::TOTAL + 1024 <= 232448,
              "shared memory per CTA");

}  // namespace wide
}  // namespace tc
}  // namespace race
