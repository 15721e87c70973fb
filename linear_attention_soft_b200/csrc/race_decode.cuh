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
// rows and writes its share of Y; a second kernel sums the shares in a fixed order.
#pragma once

#include "race_common.cuh"

namespace race {
namespace decode {

constexpr int NT = 256;    // threads per CTA
constexpr int NW = NT / 32;
constexpr int CS = 5;      // column slots of 32: d + 1 <= 160
constexpr int RB = 8;      // state rows a warp loads before it updates them

struct Args {
    const void *q, *k, *v;  // [BH][d]
    const float *W;         // [L][P][d]
    float *state;           // [BH][M][D]
    float *part;            // [BH][nsplit][D] shares of Y
    void *out;              // [BH][d]
    float *den;             // [BH] or null
    int d, L, P, M, D;
    int nsplit, rows_per_split;
    float beta;
    int hard;
};

// Shared memory of race_decode_update, in floats.
__host__ __device__ inline int update_smem_floats(int d, int D, int rows_per_split)
{
    return 2 * d + D + 2 + 2 * rows_per_split + NW * D;
}

// The 2^P corner weights of table l for the normalised row x^ = x / |x| (x in shared
// memory, rawn = |x|): prod_p sigmoid(2 beta c_rp tanh(W_lp . x^)), or the one-hot sign
// hash when hard.
__device__ inline void table_features(const float *x, float rawn, const float *Wl, int P, int d, float beta,
                                      int hard, float (&f)[32])
{
    const float inv = 1.f / fmaxf(rawn, kNormEps);
    const int R = 1 << P;
    f[0] = 1.f;
    int rs = 0;
    for (int p = 0; p < P; ++p) {
        const float *w = Wl + p * d;
        float s = 0.f;
        for (int c = 0; c < d; ++c) s = fmaf(w[c], x[c], s);
        const float pr = s * inv;
        if (hard) {
            if (pr > 0.f) rs |= 1 << p;
            continue;
        }
        const float up = tanhf(pr);
        const float e = expf(-2.f * beta * fabsf(up));
        const float big = 1.f / (1.f + e), small = e * big;
        const float s1 = up >= 0.f ? big : small, s0 = up >= 0.f ? small : big;
        const int h = 1 << p;
        for (int r = 0; r < h; ++r) {
            f[r + h] = f[r] * s1;
            f[r] *= s0;
        }
    }
    if (hard)
        for (int r = 0; r < R; ++r) f[r] = r == rs ? 1.f : 0.f;
}

// grid (nsplit, BH): rows [m0, m1) of head bh's state.  NS column slots of 32 cover d + 1.
template <typename DT, int NS>
__global__ void __launch_bounds__(NT) race_decode_update(Args a)
{
    extern __shared__ float sm[];
    const int split = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = a.d, D = a.D, P = a.P, R = 1 << P;
    const int m0 = split * a.rows_per_split;
    const int m1 = min(a.M, m0 + a.rows_per_split);
    float *xq = sm, *xk = xq + d, *vt = xk + d, *nrm = vt + D, *phq = nrm + 2, *phk = phq + a.rows_per_split,
          *red = phk + a.rows_per_split;
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
    // features of this CTA's rows: one (table, q|k) item per thread
    if (m0 < m1) {
        const int l0 = m0 / R, l1 = (m1 - 1) / R;
        for (int item = tid; item < 2 * (l1 - l0 + 1); item += NT) {
            const int which = item & 1, l = l0 + (item >> 1);
            float f[32];
            table_features(which ? xk : xq, nrm[which], a.W + (int64_t)l * P * d, P, d, a.beta, a.hard, f);
            float *dst = which ? phk : phq;
            for (int r = 0; r < R; ++r) {
                const int m = l * R + r;
                if (m >= m0 && m < m1) dst[m - m0] = f[r];
            }
        }
    }
    __syncthreads();
    // H[m] += phi_k[m] v~ and this CTA's share of Y = sum_m phi_q[m] H[m]; warp w takes rows
    // m0 + w, m0 + w + NW, ..., RB of them loaded before any is written back
    float y[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) y[s] = 0.f;
    float *H = a.state + (int64_t)bh * a.M * D;
    for (int i0 = warp; i0 < m1 - m0; i0 += NW * RB) {
        float h[RB][NS];
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int i = i0 + b * NW;
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                const int c = lane + 32 * s;
                h[b][s] = (i < m1 - m0 && c < D) ? H[(int64_t)(m0 + i) * D + c] : 0.f;
            }
        }
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const int i = i0 + b * NW;
            if (i >= m1 - m0) break;
            const float fk = phk[i], fq = phq[i];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                const int c = lane + 32 * s;
                if (c < D) {
                    const float hn = fmaf(fk, vt[c], h[b][s]);
                    H[(int64_t)(m0 + i) * D + c] = hn;
                    y[s] = fmaf(fq, hn, y[s]);
                }
            }
        }
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const int c = lane + 32 * s;
        if (c < D) red[warp * D + c] = y[s];
    }
    __syncthreads();
    for (int c = tid; c < D; c += NT) {
        float t = 0.f;
        for (int w = 0; w < NW; ++w) t += red[w * D + c];
        a.part[((int64_t)bh * a.nsplit + split) * D + c] = t;
    }
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
