// race_decode.cuh -- streaming (decode-time) step of RACE Attention.
//
// Method ("RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training"):
// the causal form keeps cumulative bucket statistics A, B per table (Algorithm 2, zh §2.3),
// so a new token t needs only the statistics of the tokens before it:
//   H += phi(k_t) [v_t, 1]^T                 (H = [B | A], [L*2^P][d+1] fp32 per head)
//   Y  = phi(q_t)^T H,   out_t = Y[:d] / Y[d],   den_t = Y[d]
// with the soft bucket assignment of zh §2.2 (or the sign hash when tau = 0), exactly as
// the forward pass computes it.
//
// The step is bound by reading and writing H (2 * L*2^P * (d+1) * 4 bytes per head).  The
// rows of H are split over `nsplit` CTAs per head (grid nsplit x B*H) so that a few heads
// still fill the GPU; each CTA forms the features of its rows for q_t and k_t, updates its
// rows and writes its share of Y; a second kernel sums the shares in a fixed order.  With
// one CTA per head (many heads) the CTA writes out_t itself and the second kernel is not
// launched.
//
// Features: every warp takes whole rows W_lp (coalesced), dotted with q_t and k_t at once;
// lane pairs of the butterfly sums then apply the nonlinearity of one projection each, and
// every thread multiplies out the corner weights of its rows.  So no thread runs a long
// dependent chain of loads before the first row of H is read.
#pragma once

#include "race_common.cuh"

namespace race {
namespace decode {

constexpr int NT = 256;    // threads per CTA
constexpr int NW = NT / 32;
constexpr int CS = 5;      // column slots of 32: d + 1 <= 160
constexpr int PB = 4;      // projections a warp forms together

struct Args {
    const void *q, *k, *v;  // [BH][d]
    const float *W;         // [L][P][d]
    float *state;           // [BH][M][D]
    float *part;            // [BH][nsplit][D] shares of Y (unused when nsplit = 1)
    void *out;              // [BH][d]
    float *den;             // [BH] or null
    int d, L, P, M, D;
    int nsplit, rows_per_split;
    float beta;
    int hard;
};

// Tables that the rows [m0, m0 + rows_per_split) of one split can touch.
__host__ __device__ inline int split_tables(int rows_per_split, int P) { return rows_per_split / (1 << P) + 2; }

// Shared memory of race_decode_update, in floats.
__host__ __device__ inline int update_smem_floats(int d, int D, int rows_per_split, int P)
{
    return 2 * d + D + 2 + 2 * rows_per_split + NW * D + D + 4 * P * split_tables(rows_per_split, P);
}

// sigmoid(2 beta c u) for the two signs c = -1, +1 of one projection pr = W_lp . x^, with
// u = tanh(pr) (zh §2.2); the sign hash (0 / 1 by the sign of pr) when hard.
__device__ inline float2 corner_pair(float pr, float beta, int hard)
{
    if (hard) {
        const float s1 = pr > 0.f ? 1.f : 0.f;
        return make_float2(1.f - s1, s1);
    }
    const float up = tanhf(pr);
    const float e = expf(-2.f * beta * fabsf(up));
    const float big = 1.f / (1.f + e), small = e * big;
    return up >= 0.f ? make_float2(small, big) : make_float2(big, small);
}

// grid (nsplit, BH): rows [m0, m1) of head bh's state.  NS column slots of 32 cover d.
template <typename DT, int NS>
__global__ void __launch_bounds__(NT, NS <= 2 ? 4 : 2) race_decode_update(Args a)
{
    extern __shared__ float sm[];
    const int split = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = a.d, D = a.D, P = a.P, R = 1 << P;
    const int m0 = split * a.rows_per_split;
    const int m1 = min(a.M, m0 + a.rows_per_split);
    const int l0 = m0 / R, nl = m0 < m1 ? (m1 - 1) / R - l0 + 1 : 0;
    float *xq = sm, *xk = xq + d, *vt = xk + d, *nrm = vt + D, *phq = nrm + 2, *phk = phq + a.rows_per_split,
          *red = phk + a.rows_per_split, *ysm = red + NW * D, *sg = ysm + D;  // sg: [2][nl][P] pairs
    const DT *q = reinterpret_cast<const DT *>(a.q) + (int64_t)bh * d;
    const DT *k = reinterpret_cast<const DT *>(a.k) + (int64_t)bh * d;
    const DT *v = reinterpret_cast<const DT *>(a.v) + (int64_t)bh * d;
    for (int c = tid; c < d; c += NT) {
        xq[c] = to_f32(q[c]);
        xk[c] = to_f32(k[c]);
        vt[c] = to_f32(v[c]);
    }
    if (tid == 0) vt[d] = 1.f;
    __syncthreads();
    if (warp < 2) {  // |q| (warp 0), |k| (warp 1)
        const float *x = warp ? xk : xq;
        float s = 0.f;
        for (int c = lane; c < d; c += 32) s = fmaf(x[c], x[c], s);
        s = warp_sum(s);
        if (lane == 0) nrm[warp] = sqrtf(s);
    }
    __syncthreads();
    // projections W_lp . q^ and W_lp . k^ of this CTA's tables: warp w takes PB rows of W at
    // a time (rows j = w, w + NW, ...), every lane its columns c = lane + 32i
    const int nproj = nl * P;
    const float *Wc = a.W + (int64_t)l0 * P * d;
    const float invq = 1.f / fmaxf(nrm[0], kNormEps), invk = 1.f / fmaxf(nrm[1], kNormEps);
    for (int j0 = warp; j0 < nproj; j0 += NW * PB) {
        float s[2 * PB];
#pragma unroll
        for (int b = 0; b < 2 * PB; ++b) s[b] = 0.f;
        for (int c = lane; c < d; c += 32) {
            const float xqc = xq[c], xkc = xk[c];
#pragma unroll
            for (int b = 0; b < PB; ++b) {
                const int j = j0 + b * NW;
                const float w = j < nproj ? Wc[(int64_t)j * d + c] : 0.f;
                s[b] = fmaf(w, xqc, s[b]);
                s[PB + b] = fmaf(w, xkc, s[PB + b]);
            }
        }
#pragma unroll
        for (int b = 0; b < 2 * PB; ++b) s[b] = warp_sum(s[b]);
        // lane i < 2 PB: sum i (q for i < PB, k above) of row j0 + (i % PB) NW
        if (lane < 2 * PB) {
            float x = s[0];
#pragma unroll
            for (int b = 1; b < 2 * PB; ++b) x = lane == b ? s[b] : x;
            const int which = lane >= PB, j = j0 + (lane % PB) * NW;
            if (j < nproj) {
                const float2 c2 = corner_pair(x * (which ? invk : invq), a.beta, a.hard);
                reinterpret_cast<float2 *>(sg)[which * nproj + j] = c2;
            }
        }
    }
    __syncthreads();
    // corner weights of this CTA's rows: phi_r = prod_p sigmoid(2 beta c_rp u_p), c_rp the
    // sign of bit p of r (one-hot when hard)
    const int nrows = m1 > m0 ? m1 - m0 : 0;
    for (int i = tid; i < 2 * nrows; i += NT) {
        const int which = i >= nrows, mi = which ? i - nrows : i;
        const int m = m0 + mi, rr = m & (R - 1);
        const float2 *sp = reinterpret_cast<const float2 *>(sg) + which * nproj + (m / R - l0) * P;
        float f = 1.f;
        for (int p = 0; p < P; ++p) {
            const float2 c2 = sp[p];
            f *= (rr >> p) & 1 ? c2.y : c2.x;
        }
        (which ? phk : phq)[mi] = f;
    }
    __syncthreads();
    // H[m] += phi_k[m] v~ and this CTA's share of Y = sum_m phi_q[m] H[m]; warp w takes rows
    // m0 + w, m0 + w + NW, ..., RB of them loaded before any is written back.  Columns
    // c = lane + 32 s (< d) sit in slots; column d (the A statistic) of the batch's row b sits
    // in lane b.
    constexpr int RB = NS <= 2 ? 16 : 8;
    float y[NS], ydn = 0.f;
#pragma unroll
    for (int s = 0; s < NS; ++s) y[s] = 0.f;
    float *H = a.state + ((int64_t)bh * a.M + m0) * D;
    for (int i0 = warp; i0 < nrows; i0 += NW * RB) {
        float h[RB][NS];
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int i = i0 + b * NW;
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                const int c = lane + 32 * s;
                h[b][s] = (i < nrows && c < d) ? H[(int64_t)i * D + c] : 0.f;
            }
        }
        const int id = i0 + lane * NW;  // this lane's row for column d
        const bool has_d = lane < RB && id < nrows;
        const float hd = has_d ? H[(int64_t)id * D + d] : 0.f;
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int i = i0 + b * NW;
            if (i >= nrows) break;
            const float fk = phk[i], fq = phq[i];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                const int c = lane + 32 * s;
                if (c < d) {
                    const float hn = fmaf(fk, vt[c], h[b][s]);
                    H[(int64_t)i * D + c] = hn;
                    y[s] = fmaf(fq, hn, y[s]);
                }
            }
        }
        if (has_d) {
            const float hn = fmaf(phk[id], vt[d], hd);
            H[(int64_t)id * D + d] = hn;
            ydn = fmaf(phq[id], hn, ydn);
        }
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const int c = lane + 32 * s;
        if (c < d) red[warp * D + c] = y[s];
    }
    ydn = warp_sum(ydn);
    if (lane == 0) red[warp * D + d] = ydn;
    __syncthreads();
    for (int c = tid; c < D; c += NT) {
        float t = 0.f;
        for (int w = 0; w < NW; ++w) t += red[w * D + c];
        if (a.nsplit == 1)
            ysm[c] = t;
        else
            a.part[((int64_t)bh * a.nsplit + split) * D + c] = t;
    }
    if (a.nsplit != 1) return;
    __syncthreads();  // one split: out = Y[:d] / Y[d] here (0 where Y[d] = 0)
    const float dn = ysm[d];
    DT *out = reinterpret_cast<DT *>(a.out) + (int64_t)bh * d;
    for (int c = tid; c < d; c += NT) store_as(out + c, dn != 0.f ? ysm[c] / dn : 0.f);
    if (tid == 0 && a.den) a.den[bh] = dn;
}

// grid BH: Y = sum of the shares (split order), out = Y[:d] / Y[d] (0 where Y[d] = 0).
template <typename DT>
__global__ void __launch_bounds__(NT) race_decode_readout(Args a)
{
    __shared__ float ysm[CS * 32];
    const int bh = blockIdx.x, D = a.D, d = a.d;
    for (int c = threadIdx.x; c < D; c += NT) {
        float t = 0.f;
        for (int s = 0; s < a.nsplit; ++s) t += a.part[((int64_t)bh * a.nsplit + s) * D + c];
        ysm[c] = t;
    }
    __syncthreads();
    const float dn = ysm[d];
    DT *out = reinterpret_cast<DT *>(a.out) + (int64_t)bh * d;
    for (int c = threadIdx.x; c < d; c += NT) store_as(out + c, dn != 0.f ? ysm[c] / dn : 0.f);
    if (threadIdx.x == 0 && a.den) a.den[bh] = dn;
}

}  // namespace decode
}  // namespace race
