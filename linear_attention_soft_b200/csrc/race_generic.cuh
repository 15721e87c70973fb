// race_generic.cuh -- general-shape RACE Attention kernels (fp32 CUDA-core arithmetic).
//
// Method: "RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training",
// zh §2.2 (soft bucketization, bucket statistics, global read-out = Algorithm 1) and zh §2.3
// (causal streaming statistics = Algorithm 2).  The backward pass is the chain rule
// through those steps.
//
// This path serves every supported shape and dtype (fp32 inputs need fp32 arithmetic to
// hold a 1e-4 relative error).  Work layout:
//
//   * A (b, h) sequence is cut into segments; a segment is walked in chunks of T tokens.
//     Per chunk the scan does the intra-chunk masked block plus the inter-chunk read-out
//     of the carried state, then folds the chunk into the state.  Segment start states
//     come from three steps: per-segment totals (race_agg), a prefix/suffix over segments
//     (race_scan), then the walk.
//   * The L*R features are split in groups of MG = 128 (whole tables per group).  The G
//     groups of one segment run as the G CTAs of one thread-block cluster: each CTA keeps
//     its group's state [MG][d+1] in shared memory for the whole walk, computes its
//     tables' share of every output row, and the cluster sums the shares through
//     distributed shared memory, one cluster barrier per chunk.  The sum over tables is
//     exact in the method (the read-out adds the tables' numerators and denominators), so
//     splitting by table changes only the fp32 summation order.
//
// Thread tiles (256 threads, ty = warp, tx = lane), all conflict-free in shared memory
// because row strides are odd (d+1, MG+1, T+1) or the access is a broadcast:
//   TD tile  (T x D outputs): rows ty*RPT.., columns tx + 32 s
//   TT tile  (T x T):         element e = tid + 256 a -> (e / T, e % T)
//   TM tile  (T x MG):        rows ty*RPT.., features tx + 32 s
//   MD tile  (MG x D):        features ty*16.., columns tx + 32 s
#pragma once

#include <cooperative_groups.h>

#include "race_common.cuh"

namespace race {
namespace generic {

namespace cg = cooperative_groups;

constexpr int NT = 256;   // threads per CTA
constexpr int MG = 128;   // features per group = per CTA of a cluster
constexpr int MAXG = 8;   // groups per cluster (portable cluster size)
constexpr int CSLOT = 5;  // column slots of 32: D = d + 1 <= 160

enum AggMode { AGG_KV = 0, AGG_QDY = 1 };
enum ScanMode { SCAN_EXCL_PREFIX = 0, SCAN_EXCL_SUFFIX = 1, SCAN_TOTAL = 2, SCAN_TOTAL_ONLY = 3 };

struct Args {
    const void *q, *k, *v, *o, *dout;
    const float *den_in;
    void *out, *dq, *dk, *dv;
    float *den_out;
    const float *W;
    const float *state;       // walk start states: [BH][nseg][M][D] (or [BH][1][M][D])
    int64_t state_seg_stride;  // elements between consecutive segments' states (0 = shared)
    float *agg_out;           // race_agg output: [BH][nseg][M][D]
    int64_t N;
    int d, L, P, M, G;
    float beta;
    int hard, causal;
    int64_t seg_len;
    int nseg;
    float *dpq, *dpk;  // optional: dLoss/dp / |x| per q (k) row [BH*N][L*P] fp32, for dW
    int64_t ro_seg_len;  // bidirectional read-out only: tokens per CTA (0: the segments)
    int agg_split;       // race_agg: CTAs per segment, a cluster along y (0 or 1: one)
};

// Shared-memory carve-up, in floats.  Identical on host and device.
struct Smem {
    int xq, xk, nq, nk, vt, dy, wg, phq, phk, hs, s1, s2, dph, ub, dpb, red1, red2, total;
    __host__ __device__ Smem(int T, int d, int P)
    {
        const int D = d + 1, tgP = (MG >> P) * P;
        int o = 0;
        auto take = [&](int n) { int r = o; o += (n + 3) & ~3; return r; };
        xq = take(T * D);  // raw rows, stride d+1
        xk = take(T * D);
        nq = take(T);
        nk = take(T);
        vt = take(T * D);
        dy = take(T * D);
        wg = take(tgP * d);
        phq = take(T * (MG + 1));
        phk = take(T * (MG + 1));
        hs = take(MG * D);
        s1 = take(T * (T + 1));
        s2 = take(T * (T + 1));
        dph = take(T * (MG + 1));
        ub = take(T * tgP);
        dpb = take(T * tgP);
        red1 = take(2 * T * D);
        red2 = take(2 * T * d);
        total = o;
    }
};

// ------------------------------------------------------------------------------------
// small cooperative helpers
// ------------------------------------------------------------------------------------

// rows [0, nvalid) of a [.., d] tensor into dst[T][d+1] as fp32, zero rows beyond.
template <typename DT, int T>
__device__ void load_rows(const DT *src, int nvalid, int d, float *dst)
{
    const int D = d + 1;
    for (int e = threadIdx.x; e < T * d; e += NT) {
        const int i = e / d, c = e - i * d;
        dst[i * D + c] = i < nvalid ? to_f32(src[(int64_t)i * d + c]) : 0.f;
    }
}

// v~ = [v, 1] rows (zero rows beyond nvalid, ones column included).
template <typename DT, int T>
__device__ void load_vt(const DT *src, int nvalid, int d, float *dst)
{
    const int D = d + 1;
    for (int e = threadIdx.x; e < T * D; e += NT) {
        const int i = e / D, c = e - i * D;
        float x = 0.f;
        if (i < nvalid) x = c < d ? to_f32(src[(int64_t)i * d + c]) : 1.f;
        dst[e] = x;
    }
}

// Row norms (raw, unfloored) of x[T][d+1], one warp per row.
template <int T>
__device__ void row_norms(const float *x, int d, float *nrm)
{
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = w; i < T; i += NT / 32) {
        float s = 0.f;
        for (int c = lane; c < d; c += 32) s = fmaf(x[i * (d + 1) + c], x[i * (d + 1) + c], s);
        s = warp_sum(s);
        if (lane == 0) nrm[i] = sqrtf(s);
    }
}

// dY_i = [dO_i / den_i, -(dO_i . o_i) / den_i], zero beyond nvalid; one warp per row.
template <typename DT, int T>
__device__ void load_dy(const DT *dout, const DT *o, const float *den, int nvalid, int d,
                        float *dy)
{
    const int D = d + 1, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = w; i < T; i += NT / 32) {
        if (i >= nvalid) {
            for (int c = lane; c < D; c += 32) dy[i * D + c] = 0.f;
            continue;
        }
        const float dn = den[i];
        const float inv = dn != 0.f ? 1.f / dn : 0.f;
        float s = 0.f;
        for (int c = lane; c < d; c += 32) {
            const float g = to_f32(dout[(int64_t)i * d + c]);
            s = fmaf(g, to_f32(o[(int64_t)i * d + c]), s);
            dy[i * D + c] = g * inv;
        }
        s = warp_sum(s);
        if (lane == 0) dy[i * D + d] = -s * inv;
    }
}

// W rows of the tables of group g -> wg[tg][P][d].
__device__ inline void load_w_group(const float *W, int g, int P, int d, int tg, float *wg)
{
    const int t0 = g * (MG >> P);
    const int n = tg * P * d;
    const float *src = W + (int64_t)t0 * P * d;
    for (int e = threadIdx.x; e < n; e += NT) wg[e] = src[e];
}

// Soft bucket assignment of rows x[T][d+1] for the tg tables held in wg (zh §2.2):
// x^ = x/|x|, u = tanh(W_l x^), phi_l[r] = softmax_r(beta c_r . u).  The softmax is
// evaluated in its factorised form prod_p sigmoid(2 beta c_rp u_p), which is the same
// function because the logit is linear in the corner's signs.  hard: one-hot sign hash.
template <int T>
__device__ void group_features(const float *x, const float *rawn, int nvalid, const float *wg,
                               int tg, int P, int d, float beta, int hard, float *phi, float *u)
{
    const int R = 1 << P, D = d + 1;
    for (int item = threadIdx.x; item < T * tg; item += NT) {
        const int i = item % T, l = item / T;
        float *out = phi + i * (MG + 1) + l * R;
        if (i >= nvalid) {
            for (int r = 0; r < R; ++r) out[r] = 0.f;
            if (u)
                for (int p = 0; p < P; ++p) u[i * (tg * P) + l * P + p] = 0.f;
            continue;
        }
        const float *xr = x + i * D;
        const float inv = 1.f / fmaxf(rawn[i], kNormEps);
        // the plane loop is unrolled to its maximum (P <= 5) so that every index into f is a
        // compile-time constant and f stays in registers
        float f[32];
        f[0] = 1.f;
        int rs = 0;
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            if (p >= P) break;
            const float *w = wg + (l * P + p) * d;
            float s = 0.f;
            for (int c = 0; c < d; ++c) s = fmaf(w[c], xr[c], s);
            const float pr = s * inv;
            if (hard) {
                if (pr > 0.f) rs |= 1 << p;
            } else {
                const float up = tanhf(pr);
                if (u) u[i * (tg * P) + l * P + p] = up;
                const float e = expf(-2.f * beta * fabsf(up));
                const float big = 1.f / (1.f + e), small = e * big;
                const float s1 = up >= 0.f ? big : small, s0 = up >= 0.f ? small : big;
#pragma unroll
                for (int r = 0; r < (1 << p); ++r) {
                    f[r + (1 << p)] = f[r] * s1;
                    f[r] *= s0;
                }
            }
        }
        if (hard) {
            for (int r = 0; r < R; ++r) out[r] = r == rs ? 1.f : 0.f;
        } else {
#pragma unroll
            for (int r = 0; r < 32; ++r)
                if (r < R) out[r] = f[r];
        }
    }
}

// Feature-map backward inside a table: dz = phi (dphi - phi.dphi), du_p = beta sum_r c_rp dz_r,
// dp = du (1 - u^2).  Writes dp[T][tg*P].
template <int T>
__device__ void group_features_bwd(const float *phi, const float *dphi, const float *u,
                                   int nvalid, int tg, int P, float beta, float *dp)
{
    const int R = 1 << P;
    for (int item = threadIdx.x; item < T * tg; item += NT) {
        const int i = item % T, l = item / T;
        float *o = dp + i * (tg * P) + l * P;
        if (i >= nvalid) {
            for (int p = 0; p < P; ++p) o[p] = 0.f;
            continue;
        }
        const float *f = phi + i * (MG + 1) + l * R;
        const float *g = dphi + i * (MG + 1) + l * R;
        float dot = 0.f;
        for (int r = 0; r < R; ++r) dot = fmaf(f[r], g[r], dot);
        float du[5] = {0.f, 0.f, 0.f, 0.f, 0.f};  // unrolled to P <= 5: kept in registers
        for (int r = 0; r < R; ++r) {
            const float dz = f[r] * (g[r] - dot);
#pragma unroll
            for (int p = 0; p < 5; ++p)
                if (p < P) du[p] += ((r >> p) & 1) ? dz : -dz;
        }
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            if (p >= P) break;
            const float up = u[i * (tg * P) + l * P + p];
            o[p] = beta * du[p] * (1.f - up * up);
        }
    }
}

// dp[T][tg*P] of this group's tables, divided by |x| of each row, into rows [0, nvalid) of a
// [rows][LP] buffer at the group's first projection (for the gradient of W).
template <int T>
__device__ void store_dp(const float *dp, const float *rawn, int nvalid, int tg, int P, int g, int LP, float *dst)
{
    const int n = tg * P, lp0 = g * (MG >> P) * P;
    for (int e = threadIdx.x; e < nvalid * n; e += NT) {
        const int i = e / n, j = e - i * n;
        dst[(int64_t)i * LP + lp0 + j] = dp[i * n + j] / fmaxf(rawn[i], kNormEps);
    }
}

// dxh[T][d] = sum_{l,p} W[l,p,:] dp[:, l*P+p]   (this group's share of dL/dx^)
template <int T>
__device__ void group_dxhat(const float *wg, const float *dp, int tg, int P, int d, float *dxh)
{
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31, n = tg * P;
    float acc[RPT][4];
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int s = 0; s < 4; ++s) acc[a][s] = 0.f;
    for (int lp = 0; lp < n; ++lp) {
        float w[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int c = tx + 32 * s;
            w[s] = c < d ? wg[lp * d + c] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float g = dp[(ty * RPT + a) * n + lp];
#pragma unroll
            for (int s = 0; s < 4; ++s) acc[a][s] = fmaf(w[s], g, acc[a][s]);
        }
    }
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int c = tx + 32 * s;
            if (c < d) dxh[(ty * RPT + a) * d + c] = acc[a][s];
        }
}

// acc[a][s] (+)= sum_m A[i][m] B[m][c], A = [T][MG+1] features, B = [MG][D] state (TD tile)
template <int T>
__device__ __forceinline__ void td_feat_state(const float *A, const float *Bm, int Mg, int D,
                                              float (&acc)[T / 8][CSLOT])
{
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    for (int m = 0; m < Mg; ++m) {
        float b[CSLOT];
#pragma unroll
        for (int s = 0; s < CSLOT; ++s) {
            const int c = tx + 32 * s;
            b[s] = c < D ? Bm[m * D + c] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float x = A[(ty * RPT + a) * (MG + 1) + m];
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) acc[a][s] = fmaf(x, b[s], acc[a][s]);
        }
    }
}

// acc[a][s] += sum_j S[i][j] V[j][c], S = [T][T+1], V = [T][D] (TD tile)
template <int T>
__device__ __forceinline__ void td_tt_rows(const float *S, const float *V, int D,
                                           float (&acc)[T / 8][CSLOT])
{
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    for (int j = 0; j < T; ++j) {
        float b[CSLOT];
#pragma unroll
        for (int s = 0; s < CSLOT; ++s) {
            const int c = tx + 32 * s;
            b[s] = c < D ? V[j * D + c] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float x = S[(ty * RPT + a) * (T + 1) + j];
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) acc[a][s] = fmaf(x, b[s], acc[a][s]);
        }
    }
}

// S[i][j] = sum_k A[i][k] B[j][k] over k < K, rows of stride `as`, masked to
// (i, j) in mask: mode 0 = none, 1 = j <= i, 2 = j >= i; also zero beyond nvalid.
template <int T>
__device__ void tt_dot(const float *A, const float *B, int stride, int K, int mode, int nvalid,
                       float *S)
{
    constexpr int PER = T * T / NT;
#pragma unroll
    for (int a = 0; a < PER; ++a) {
        const int e = threadIdx.x + NT * a;
        const int i = e / T, j = e % T;
        float s = 0.f;
        for (int kk = 0; kk < K; ++kk) s = fmaf(A[i * stride + kk], B[j * stride + kk], s);
        bool keep = i < nvalid && j < nvalid;
        if (mode == 1) keep = keep && j <= i;
        if (mode == 2) keep = keep && j >= i;
        S[i * (T + 1) + j] = keep ? s : 0.f;
    }
}

// state[m][c] += sum_j F[j][m] V[j][c]   (MD tile; F = [T][MG+1], V = [T][D])
template <int T>
__device__ void md_update(float *St, const float *F, const float *V, int Mg, int D)
{
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    constexpr int RB = 8;
    for (int r0 = 0; r0 < MG / 8; r0 += RB) {
        float acc[RB][CSLOT];
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) acc[r][s] = 0.f;
        for (int j = 0; j < T; ++j) {
            float b[CSLOT];
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) {
                const int c = tx + 32 * s;
                b[s] = c < D ? V[j * D + c] : 0.f;
            }
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const float f = F[j * (MG + 1) + ty * (MG / 8) + r0 + r];
#pragma unroll
                for (int s = 0; s < CSLOT; ++s) acc[r][s] = fmaf(f, b[s], acc[r][s]);
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int m = ty * (MG / 8) + r0 + r;
            if (m >= Mg) continue;
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) {
                const int c = tx + 32 * s;
                if (c < D) St[m * D + c] += acc[r][s];
            }
        }
    }
}

// dph[i][m] = sum_c X[i][c] St[m][c] + (P2 ? sum_j P2[i][j] F[j][m] : 0)   (TM tile)
template <int T>
__device__ void tm_grad(const float *X, const float *St, const float *P2, const float *F, int Mg,
                        int D, float *dph)
{
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    float acc[RPT][MG / 32];
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int s = 0; s < MG / 32; ++s) acc[a][s] = 0.f;
    for (int c = 0; c < D; ++c) {
        float b[MG / 32];
#pragma unroll
        for (int s = 0; s < MG / 32; ++s) {
            const int m = tx + 32 * s;
            b[s] = m < Mg ? St[m * D + c] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float x = X[(ty * RPT + a) * D + c];
#pragma unroll
            for (int s = 0; s < MG / 32; ++s) acc[a][s] = fmaf(x, b[s], acc[a][s]);
        }
    }
    if (P2) {
        for (int j = 0; j < T; ++j) {
            float b[MG / 32];
#pragma unroll
            for (int s = 0; s < MG / 32; ++s) b[s] = F[j * (MG + 1) + tx + 32 * s];
#pragma unroll
            for (int a = 0; a < RPT; ++a) {
                const float x = P2[(ty * RPT + a) * (T + 1) + j];
#pragma unroll
                for (int s = 0; s < MG / 32; ++s) acc[a][s] = fmaf(x, b[s], acc[a][s]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int s = 0; s < MG / 32; ++s) dph[(ty * RPT + a) * (MG + 1) + tx + 32 * s] = acc[a][s];
}

// dx = (dx^ - x^ (x^ . dx^)) / max(|x|, eps) for the rows a cluster rank owns, with dx^
// summed over the cluster's groups (`parts` = rank-local buffer of [T][d]).
template <typename DT, int T>
__device__ void reduce_dx(cg::cluster_group &cl, int G, int rank, const float *parts,
                          const float *x, const float *rawn, int nvalid, int d, DT *dst)
{
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = rank + G * w; i < nvalid; i += G * (NT / 32)) {
        float g[4], xh[4];
        const float rn = rawn[i], n = fmaxf(rn, kNormEps), inv = 1.f / n;
        float dot = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int c = lane + 32 * s;
            g[s] = 0.f;
            xh[s] = 0.f;
            if (c < d) {
                for (int r = 0; r < G; ++r) g[s] += cl.map_shared_rank(parts, r)[i * d + c];
                xh[s] = x[i * (d + 1) + c] * inv;
                dot = fmaf(xh[s], g[s], dot);
            }
        }
        dot = warp_sum(dot);
        if (rn <= kNormEps) dot = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int c = lane + 32 * s;
            if (c < d) store_as(dst + (int64_t)i * d + c, (g[s] - xh[s] * dot) * inv);
        }
    }
}

__device__ inline void seg_range(const Args &a, int seg, int64_t &t0, int64_t &t1)
{
    t0 = (int64_t)seg * a.seg_len;
    t1 = t0 + a.seg_len;
    if (t1 > a.N) t1 = a.N;
}

// ------------------------------------------------------------------------------------
// race_agg: per-segment bucket statistics of one group (no cluster).
//   AGG_KV : sum_j phi(k_j) [v_j, 1]^T                (A, B of zh §2.2 over the segment)
//   AGG_QDY: sum_i phi(q_i) dY_i^T                    (the backward's key-side statistics)
// grid (G, nseg, BH)
// ------------------------------------------------------------------------------------
template <typename DT, int T, int MODE>
__global__ void __launch_bounds__(NT) race_agg(Args a)
{
    extern __shared__ float sm[];
    const Smem L(T, a.d, a.P);
    // with S = agg_split > 1 the S CTAs of a cluster along y share a segment: CTA `sub` takes
    // its chunks sub, sub + S, ... and rank 0 adds the S partial states in rank order
    const int S = a.agg_split > 1 ? a.agg_split : 1;
    const int g = blockIdx.x, seg = blockIdx.y / S, sub = blockIdx.y % S, bh = blockIdx.z;
    const int d = a.d, D = d + 1, R = 1 << a.P;
    const int Mg = min(MG, a.M - g * MG), tg = Mg / R;
    const int64_t base = (int64_t)bh * a.N * d;
    float *x = sm + L.xq, *nr = sm + L.nq, *val = sm + L.vt, *wg = sm + L.wg, *ph = sm + L.phq,
          *st = sm + L.hs;
    load_w_group(a.W, g, a.P, d, tg, wg);
    for (int e = threadIdx.x; e < MG * D; e += NT) st[e] = 0.f;
    int64_t t0, t1;
    seg_range(a, seg, t0, t1);
    for (int64_t c0 = t0 + (int64_t)sub * T; c0 < t1; c0 += (int64_t)S * T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : (int64_t)T);
        __syncthreads();
        if (MODE == AGG_KV) {
            load_rows<DT, T>((const DT *)a.k + base + c0 * d, nv, d, x);
            load_vt<DT, T>((const DT *)a.v + base + c0 * d, nv, d, val);
        } else {
            load_rows<DT, T>((const DT *)a.q + base + c0 * d, nv, d, x);
            load_dy<DT, T>((const DT *)a.dout + base + c0 * d, (const DT *)a.o + base + c0 * d,
                           a.den_in + (int64_t)bh * a.N + c0, nv, d, val);
        }
        __syncthreads();
        row_norms<T>(x, d, nr);
        __syncthreads();
        group_features<T>(x, nr, nv, wg, tg, a.P, d, a.beta, a.hard, ph, nullptr);
        __syncthreads();
        md_update<T>(st, ph, val, Mg, D);
    }
    __syncthreads();
    float *dst = a.agg_out + (((int64_t)bh * a.nseg + seg) * a.M + (int64_t)g * MG) * D;
    if (S == 1) {
        for (int e = threadIdx.x; e < Mg * D; e += NT) dst[e] = st[e];
        return;
    }
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();  // every partial state is complete
    if (cl.block_rank() == 0)
        for (int e = threadIdx.x; e < Mg * D; e += NT) {
            float acc = st[e];
            for (int q = 1; q < S; ++q) acc += cl.map_shared_rank(st, q)[e];
            dst[e] = acc;
        }
    cl.sync();  // no CTA leaves while rank 0 still reads its shared memory
}

// ------------------------------------------------------------------------------------
// race_scan: over the segments of each (b, h), element-wise on the [M][D] states.
//   SCAN_EXCL_PREFIX / SUFFIX: each segment's slot becomes the sum of the segments before
//     (after) it, starting from init (statistics of tokens held elsewhere, e.g. earlier or
//     later shards of the sequence; null = zero);
//   SCAN_TOTAL: slot 0 becomes init + the sum of all segments;
//   SCAN_TOTAL_ONLY: the buffer is left as it is.
// total_out (optional) receives the sum of all segments (plus init, except TOTAL_ONLY).
// skip_if (optional): the scan does nothing when *skip_if == skip_tag (the buffer already
// holds the scanned states, decided on the device).
// grid (ceil(M*D / NT), BH)
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT) race_scan(float *buf, int nseg, int64_t MD, int mode, const float *init,
                                                float *total_out, const uint32_t *skip_if = nullptr,
                                                uint32_t skip_tag = 0)
{
    const int64_t e = (int64_t)blockIdx.x * NT + threadIdx.x;
    if (e >= MD || (skip_if && *skip_if == skip_tag)) return;
    float *b = buf + (int64_t)blockIdx.y * nseg * MD + e;
    const int64_t oe = (int64_t)blockIdx.y * MD + e;
    constexpr int K = 8;  // segments loaded together: independent loads in flight
    float run = (init && mode != SCAN_TOTAL_ONLY) ? init[oe] : 0.f;
    if (mode == SCAN_TOTAL || mode == SCAN_TOTAL_ONLY) {
        for (int s = 0; s < nseg; ++s) run += b[(int64_t)s * MD];
        if (mode == SCAN_TOTAL) b[0] = run;
        if (total_out) total_out[oe] = run;
        return;
    }
    const bool rev = mode == SCAN_EXCL_SUFFIX;
    for (int s0 = 0; s0 < nseg; s0 += K) {
        float v[K];
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const int s = rev ? nseg - 1 - (s0 + i) : s0 + i;
            v[i] = (s0 + i < nseg) ? b[(int64_t)s * MD] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const int s = rev ? nseg - 1 - (s0 + i) : s0 + i;
            if (s0 + i < nseg) {
                b[(int64_t)s * MD] = run;
                run += v[i];
            }
        }
    }
    if (total_out) total_out[oe] = run;
}

// ------------------------------------------------------------------------------------
// Gradient of W: dW[lp][c] = sum over rows of dp[row][lp] x[row][c] (dp = dLoss/dp / |x|),
// over the q rows then the k rows.  CTA (ks, i, j) sums its share of the rows into the
// 64 x 64 output tile (i, j); race_dw_sum adds the shares in ks order.  16 x 16 threads,
// each a 4 x 4 block of the tile, rows staged 16 at a time.
// grid (ksplit, ceil(LP / 64), ceil(d / 64))
// ------------------------------------------------------------------------------------
template <typename DT>
__global__ void __launch_bounds__(NT) race_dw_partial(const float *dpq, const float *dpk, const DT *q, const DT *k,
                                                      int64_t rows, int LP, int d, int64_t rows_per_split,
                                                      float *partial)
{
    __shared__ float As[16][64], Bs[16][64];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int lp0 = blockIdx.y * 64, c0 = blockIdx.z * 64;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    int64_t r0 = (int64_t)blockIdx.x * rows_per_split, r1 = r0 + rows_per_split;
    if (r1 > 2 * rows) r1 = 2 * rows;
    for (int64_t rb = r0; rb < r1; rb += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += NT) {
            const int rr = e >> 6, cc = e & 63;
            const int64_t row = rb + rr;
            float av = 0.f, bv = 0.f;
            if (row < r1) {
                const bool kside = row >= rows;
                const int64_t rw = kside ? row - rows : row;
                if (lp0 + cc < LP) av = (kside ? dpk : dpq)[rw * LP + lp0 + cc];
                if (c0 + cc < d) bv = to_f32((kside ? k : q)[rw * d + c0 + cc]);
            }
            As[rr][cc] = av;
            Bs[rr][cc] = bv;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[kk][ty * 4 + i];
                bv[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float *dst = partial + (int64_t)blockIdx.x * LP * d;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int lp = lp0 + ty * 4 + i, c = c0 + tx * 4 + j;
            if (lp < LP && c < d) dst[(int64_t)lp * d + c] = acc[i][j];
        }
}

// dW[e] = sum over the splits of partial[s][e], in split order.
__global__ void __launch_bounds__(NT) race_dw_sum(const float *partial, int nsplit, int64_t n, float *dW)
{
    const int64_t e = (int64_t)blockIdx.x * NT + threadIdx.x;
    if (e >= n) return;
    float s = 0.f;
    for (int k = 0; k < nsplit; ++k) s += partial[(int64_t)k * n + e];
    dW[e] = s;
}

// ------------------------------------------------------------------------------------
// race_shard_combine: out = sum of the selected shards' statistics, in shard order:
// which = 0 the shards before `shard`, 1 those after it, 2 every other shard.
// gathered is [nshards][elems].  grid ceil(elems / NT)
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT) race_shard_combine(const float *gathered, int nshards, int shard, int which,
                                                         int64_t elems, float *out)
{
    const int64_t e = (int64_t)blockIdx.x * NT + threadIdx.x;
    if (e >= elems) return;
    float run = 0.f;
    for (int s = 0; s < nshards; ++s) {
        const bool take = which == 0 ? s < shard : which == 1 ? s > shard : s != shard;
        if (take) run += gathered[(int64_t)s * elems + e];
    }
    out[e] = run;
}

__device__ inline void load_state(const Args &a, int g, int seg, int bh, int Mg, float *st)
{
    const int D = a.d + 1;
    const float *src = a.state + (int64_t)bh * a.nseg * a.M * D + seg * a.state_seg_stride +
                       (int64_t)g * MG * D;
    for (int e = threadIdx.x; e < MG * D; e += NT) st[e] = e < Mg * D ? src[e] : 0.f;
}

// ------------------------------------------------------------------------------------
// race_fwd_walk: Y_i = phi(q_i)^T H_prev + sum_{j<=i in chunk} (phi(q_i).phi(k_j)) v~_j,
// then H += Phi_K^T V~ (causal); bidirectional: Y_i = phi(q_i)^T H_total.
// grid (G, nseg, BH), cluster (G, 1, 1)
// ------------------------------------------------------------------------------------
template <typename DT, int T>
__global__ void __launch_bounds__(NT) race_fwd_walk(Args a)
{
    extern __shared__ float sm[];
    cg::cluster_group cl = cg::this_cluster();
    const Smem L(T, a.d, a.P);
    const int g = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z, G = a.G;
    const int rank = (int)cl.block_rank();
    const int d = a.d, D = d + 1, R = 1 << a.P;
    const int Mg = min(MG, a.M - g * MG), tg = Mg / R;
    const int64_t base = (int64_t)bh * a.N * d;
    float *xq = sm + L.xq, *xk = sm + L.xk, *nq = sm + L.nq, *nk = sm + L.nk, *vt = sm + L.vt,
          *wg = sm + L.wg, *phq = sm + L.phq, *phk = sm + L.phk, *st = sm + L.hs, *S = sm + L.s1,
          *red = sm + L.red1;
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    load_w_group(a.W, g, a.P, d, tg, wg);
    load_state(a, g, seg, bh, Mg, st);
    int64_t t0, t1;
    if (!a.causal && a.ro_seg_len > 0) {  // every row reads the same total state: any split works
        t0 = (int64_t)seg * a.ro_seg_len;
        t1 = t0 + a.ro_seg_len < a.N ? t0 + a.ro_seg_len : a.N;
    } else {
        seg_range(a, seg, t0, t1);
    }
    int buf = 0;
    for (int64_t c0 = t0; c0 < t1; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : (int64_t)T);
        __syncthreads();
        load_rows<DT, T>((const DT *)a.q + base + c0 * d, nv, d, xq);
        if (a.causal) {
            load_rows<DT, T>((const DT *)a.k + base + c0 * d, nv, d, xk);
            load_vt<DT, T>((const DT *)a.v + base + c0 * d, nv, d, vt);
        }
        __syncthreads();
        row_norms<T>(xq, d, nq);
        if (a.causal) row_norms<T>(xk, d, nk);
        __syncthreads();
        group_features<T>(xq, nq, nv, wg, tg, a.P, d, a.beta, a.hard, phq, nullptr);
        if (a.causal) group_features<T>(xk, nk, nv, wg, tg, a.P, d, a.beta, a.hard, phk, nullptr);
        __syncthreads();
        float acc[RPT][CSLOT];
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) acc[r][s] = 0.f;
        td_feat_state<T>(phq, st, Mg, D, acc);  // inter-chunk read-out of the carried state
        if (a.causal) {
            tt_dot<T>(phq, phk, MG + 1, Mg, 1, nv, S);  // intra-chunk block, j <= i
            __syncthreads();
            td_tt_rows<T>(S, vt, D, acc);
            md_update<T>(st, phk, vt, Mg, D);  // fold the chunk into the statistics
        }
        float *part = red + buf * T * D;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) {
                const int c = tx + 32 * s;
                if (c < D) part[(ty * RPT + r) * D + c] = acc[r][s];
            }
        cl.sync();
        // sum the groups' shares of the rows this rank owns; O = numerator / denominator
        for (int e = threadIdx.x; e < T * D; e += NT) {
            const int i = e / D, c = e - i * D;
            if (i >= nv || (i % G) != rank) continue;
            float y = 0.f, dn = 0.f;
            for (int r = 0; r < G; ++r) {
                const float *p = cl.map_shared_rank(part, r);
                y += p[i * D + c];
                dn += p[i * D + d];
            }
            if (c < d)
                store_as((DT *)a.out + base + (c0 + i) * d + c, dn != 0.f ? y / dn : 0.f);
            else if (a.den_out)
                a.den_out[(int64_t)bh * a.N + c0 + i] = dn;
        }
        buf ^= 1;
    }
    cl.sync();
}

// ------------------------------------------------------------------------------------
// race_bwd_q_walk: dphi(q_i) = H_i dY_i, split as dY H_prev^T + tril(dY V~^T) Phi_K,
// then H += Phi_K^T V~ (causal); dq through the feature-map VJP.
// grid (G, nseg, BH), cluster (G, 1, 1)
// ------------------------------------------------------------------------------------
template <typename DT, int T>
__global__ void __launch_bounds__(NT) race_bwd_q_walk(Args a)
{
    extern __shared__ float sm[];
    cg::cluster_group cl = cg::this_cluster();
    const Smem L(T, a.d, a.P);
    const int g = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z, G = a.G;
    const int rank = (int)cl.block_rank();
    const int d = a.d, D = d + 1, R = 1 << a.P;
    const int Mg = min(MG, a.M - g * MG), tg = Mg / R;
    const int64_t base = (int64_t)bh * a.N * d;
    float *xq = sm + L.xq, *xk = sm + L.xk, *nq = sm + L.nq, *nk = sm + L.nk, *vt = sm + L.vt,
          *dy = sm + L.dy, *wg = sm + L.wg, *phq = sm + L.phq, *phk = sm + L.phk, *st = sm + L.hs,
          *Pm = sm + L.s1, *dph = sm + L.dph, *ub = sm + L.ub, *dpb = sm + L.dpb,
          *red = sm + L.red2;
    load_w_group(a.W, g, a.P, d, tg, wg);
    load_state(a, g, seg, bh, Mg, st);
    int64_t t0, t1;
    seg_range(a, seg, t0, t1);
    int buf = 0;
    for (int64_t c0 = t0; c0 < t1; c0 += T) {
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : (int64_t)T);
        __syncthreads();
        load_rows<DT, T>((const DT *)a.q + base + c0 * d, nv, d, xq);
        load_dy<DT, T>((const DT *)a.dout + base + c0 * d, (const DT *)a.o + base + c0 * d,
                       a.den_in + (int64_t)bh * a.N + c0, nv, d, dy);
        if (a.causal) {
            load_rows<DT, T>((const DT *)a.k + base + c0 * d, nv, d, xk);
            load_vt<DT, T>((const DT *)a.v + base + c0 * d, nv, d, vt);
        }
        __syncthreads();
        row_norms<T>(xq, d, nq);
        if (a.causal) row_norms<T>(xk, d, nk);
        __syncthreads();
        group_features<T>(xq, nq, nv, wg, tg, a.P, d, a.beta, 0, phq, ub);
        if (a.causal) {
            group_features<T>(xk, nk, nv, wg, tg, a.P, d, a.beta, 0, phk, nullptr);
            tt_dot<T>(dy, vt, D, D, 1, nv, Pm);  // P[i][j] = dY_i . v~_j, j <= i
        }
        __syncthreads();
        tm_grad<T>(dy, st, a.causal ? Pm : nullptr, phk, Mg, D, dph);
        __syncthreads();
        if (a.causal) md_update<T>(st, phk, vt, Mg, D);
        group_features_bwd<T>(phq, dph, ub, nv, tg, a.P, a.beta, dpb);
        __syncthreads();
        if (a.dpq) store_dp<T>(dpb, nq, nv, tg, a.P, g, a.L * a.P, a.dpq + ((int64_t)bh * a.N + c0) * (a.L * a.P));
        float *part = red + buf * T * d;
        group_dxhat<T>(wg, dpb, tg, a.P, d, part);
        cl.sync();
        reduce_dx<DT, T>(cl, G, rank, part, xq, nq, nv, d, (DT *)a.dq + base + c0 * d);
        buf ^= 1;
    }
    cl.sync();
}

// ------------------------------------------------------------------------------------
// race_bwd_kv_walk (reverse chunk order): with G_j = sum_{i >= j} phi(q_i) dY_i^T,
//   dphi(k_j) = G_j v~_j = V~ G_next^T + triu(V~ dY^T) Phi_Q,
//   dv~_j     = G_j^T phi(k_j) = Phi_K G_next + triu(Phi_K Phi_Q^T) dY,
// then G += Phi_Q^T dY (causal); dk through the feature-map VJP.
// grid (G, nseg, BH), cluster (G, 1, 1)
// ------------------------------------------------------------------------------------
template <typename DT, int T>
__global__ void __launch_bounds__(NT) race_bwd_kv_walk(Args a)
{
    extern __shared__ float sm[];
    cg::cluster_group cl = cg::this_cluster();
    const Smem L(T, a.d, a.P);
    const int g = blockIdx.x, seg = blockIdx.y, bh = blockIdx.z, G = a.G;
    const int rank = (int)cl.block_rank();
    const int d = a.d, D = d + 1, R = 1 << a.P;
    const int Mg = min(MG, a.M - g * MG), tg = Mg / R;
    const int64_t base = (int64_t)bh * a.N * d;
    float *xq = sm + L.xq, *xk = sm + L.xk, *nq = sm + L.nq, *nk = sm + L.nk, *vt = sm + L.vt,
          *dy = sm + L.dy, *wg = sm + L.wg, *phq = sm + L.phq, *phk = sm + L.phk, *st = sm + L.hs,
          *Pm = sm + L.s1, *ST = sm + L.s2, *dph = sm + L.dph, *ub = sm + L.ub, *dpb = sm + L.dpb,
          *redv = sm + L.red1, *redx = sm + L.red2;
    constexpr int RPT = T / 8;
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    load_w_group(a.W, g, a.P, d, tg, wg);
    load_state(a, g, seg, bh, Mg, st);
    int64_t t0, t1;
    seg_range(a, seg, t0, t1);
    const int64_t nchunks = (t1 - t0 + T - 1) / T;
    int buf = 0;
    for (int64_t ci = nchunks - 1; ci >= 0; --ci) {
        const int64_t c0 = t0 + ci * T;
        const int nv = (int)(t1 - c0 < T ? t1 - c0 : (int64_t)T);
        __syncthreads();
        load_rows<DT, T>((const DT *)a.k + base + c0 * d, nv, d, xk);
        load_vt<DT, T>((const DT *)a.v + base + c0 * d, nv, d, vt);
        if (a.causal) {
            load_rows<DT, T>((const DT *)a.q + base + c0 * d, nv, d, xq);
            load_dy<DT, T>((const DT *)a.dout + base + c0 * d, (const DT *)a.o + base + c0 * d,
                           a.den_in + (int64_t)bh * a.N + c0, nv, d, dy);
        }
        __syncthreads();
        row_norms<T>(xk, d, nk);
        if (a.causal) row_norms<T>(xq, d, nq);
        __syncthreads();
        group_features<T>(xk, nk, nv, wg, tg, a.P, d, a.beta, 0, phk, ub);
        if (a.causal) {
            group_features<T>(xq, nq, nv, wg, tg, a.P, d, a.beta, 0, phq, nullptr);
            tt_dot<T>(vt, dy, D, D, 2, nv, Pm);  // P'[j][i] = v~_j . dY_i, i >= j
        }
        __syncthreads();
        if (a.causal) tt_dot<T>(phk, phq, MG + 1, Mg, 2, nv, ST);  // S^T[j][i], i >= j
        tm_grad<T>(vt, st, a.causal ? Pm : nullptr, phq, Mg, D, dph);
        float acc[RPT][CSLOT];
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) acc[r][s] = 0.f;
        td_feat_state<T>(phk, st, Mg, D, acc);
        __syncthreads();
        if (a.causal) {
            td_tt_rows<T>(ST, dy, D, acc);
            md_update<T>(st, phq, dy, Mg, D);
        }
        group_features_bwd<T>(phk, dph, ub, nv, tg, a.P, a.beta, dpb);
        float *pv = redv + buf * T * D;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int s = 0; s < CSLOT; ++s) {
                const int c = tx + 32 * s;
                if (c < D) pv[(ty * RPT + r) * D + c] = acc[r][s];
            }
        __syncthreads();
        if (a.dpk) store_dp<T>(dpb, nk, nv, tg, a.P, g, a.L * a.P, a.dpk + ((int64_t)bh * a.N + c0) * (a.L * a.P));
        float *px = redx + buf * T * d;
        group_dxhat<T>(wg, dpb, tg, a.P, d, px);
        cl.sync();
        for (int e = threadIdx.x; e < T * d; e += NT) {
            const int i = e / d, c = e - i * d;
            if (i >= nv || (i % G) != rank) continue;
            float y = 0.f;
            for (int r = 0; r < G; ++r) y += cl.map_shared_rank(pv, r)[i * D + c];
            store_as((DT *)a.dv + base + (c0 + i) * d + c, y);
        }
        reduce_dx<DT, T>(cl, G, rank, px, xk, nk, nv, d, (DT *)a.dk + base + c0 * d);
        buf ^= 1;
    }
    cl.sync();
}

// ------------------------------------------------------------------------------------
// race_hash: idx[row][l] = sum_p [W_lp . x_row > 0] 2^p.   grid over rows*L
// ------------------------------------------------------------------------------------
template <typename DT>
__global__ void __launch_bounds__(NT) race_hash(const DT *x, const float *W, int32_t *idx,
                                                int64_t rows, int d, int L, int P)
{
    const int64_t e = (int64_t)blockIdx.x * NT + threadIdx.x;
    if (e >= rows * L) return;
    const int64_t row = e / L;
    const int l = (int)(e - row * L);
    const DT *xr = x + row * d;
    int r = 0;
    for (int p = 0; p < P; ++p) {
        const float *w = W + ((int64_t)l * P + p) * d;
        float s = 0.f;
        for (int c = 0; c < d; ++c) s = fmaf(w[c], to_f32(xr[c]), s);
        if (s > 0.f) r |= 1 << p;
    }
    idx[e] = r;
}

}  // namespace generic
}  // namespace race
