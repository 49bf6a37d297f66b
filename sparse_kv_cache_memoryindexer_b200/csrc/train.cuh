// One training step of the memory indexer against frozen keys (hyper.ai summary, "Method"; blog
// review, section 3): forward as the index score, focal / binary cross-entropy loss against the
// window's golden labels, gradients of W^DQ, W^IUQ and W^w (the rounding of c and q to their
// storage type is passed straight through).
//
//   k_train_entries   one CTA per (128-entry tile of one sequence, layer): the tile's keys and the
//                     sequence's queries in shared memory (fp32); two threads per entry compute the
//                     64 head dot products a_h (32 each), x = sum_h w_h ReLU(a_h), the loss and
//                     g = dl/dx / N; then dw_h += g ReLU(a_h) and dq_h += (g w_h 1[a_h > 0] scale) K_s
//                     (a 64 x 128 x 128 product per tile, two threads per key dimension), added to the
//                     sequence's gradients with atomics.
//   k_train_dc        dc = dq W^IUQ (one thread per (layer, sequence, j)).
//   k_outer           g_W[l][m][n] = sum_b U[l][b][m] V[l][b][n]: the three weight gradients.
#pragma once
#include "common.cuh"

namespace lsa {

namespace train {

constexpr int TT = 128;       // entries per tile
constexpr int THREADS = 256;  // two per entry
constexpr int NHMAX = 64;
constexpr int DMAX = 128;

template <int QDT, int KDT>
__global__ void __launch_bounds__(THREADS) k_train_entries(const void *__restrict__ q, const float *__restrict__ w,
                                                           const void *__restrict__ K, const float *__restrict__ ksc,
                                                           const uint8_t *__restrict__ labels,
                                                           const int64_t *__restrict__ offs,
                                                           const int *__restrict__ tile_start, int B, int64_t T,
                                                           int n_h, int d_I, float gamma, float alpha, double invN,
                                                           float *__restrict__ dq, float *__restrict__ dw,
                                                           double *__restrict__ loss)
{
    extern __shared__ float sm[];
    float *qs = sm;                                  // [n_h][d_I]
    float *ks = qs + NHMAX * DMAX;                   // [TT][d_I + 1]
    float *gs = ks + TT * (DMAX + 1);                // [TT][n_h + 1]
    __shared__ float wsm[NHMAX], dwsm[NHMAX];
    __shared__ double lred[THREADS / 32];
    const int l = blockIdx.y;
    const int t = blockIdx.x;
    const int NT = tile_start[B];
    if (t >= NT) return;
    int lo = 0, hi = B - 1;  // the sequence of tile t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    const int64_t s0 = (int64_t)(t - tile_start[b]) * TT;
    const int nrow = (int)min((int64_t)TT, S - s0);
    const int KP = d_I + 1, GP = n_h + 1;
    // stage the queries, head weights and keys (fp32)
    const int64_t qb = ((int64_t)l * B + b) * n_h * d_I;
    for (int i = threadIdx.x; i < n_h * d_I; i += THREADS) qs[i] = load_elem<QDT>(q, qb + i);
    for (int i = threadIdx.x; i < n_h; i += THREADS) {
        wsm[i] = w[((int64_t)l * B + b) * n_h + i];
        dwsm[i] = 0.f;
    }
    for (int i = threadIdx.x; i < TT * d_I; i += THREADS) {
        const int rr = i / d_I, e = i % d_I;
        ks[rr * KP + e] = rr < nrow ? load_elem<KDT>(K, ((int64_t)l * T + off + s0 + rr) * d_I + e) : 0.f;
    }
    __syncthreads();
    // forward: thread (entry rr, half hf) takes heads hf*32 .. hf*32+31
    const int rr = threadIdx.x >> 1, hf = threadIdx.x & 1;
    const bool valid = rr < nrow;
    const float scale = (KDT == DT_FP8 && valid) ? ksc[(int64_t)l * T + off + s0 + rr] : 1.f;
    float a[32];
#pragma unroll
    for (int k = 0; k < 32; k++) a[k] = 0.f;
    const int h0 = hf * 32;
    for (int e = 0; e < d_I; e++) {
        const float kv = ks[rr * KP + e];
#pragma unroll
        for (int k = 0; k < 32; k++)
            if (h0 + k < n_h) a[k] = fmaf(qs[(h0 + k) * d_I + e], kv, a[k]);
    }
    float xp = 0.f;
#pragma unroll
    for (int k = 0; k < 32; k++) {
        a[k] *= scale;
        if (h0 + k < n_h) xp = fmaf(wsm[h0 + k], fmaxf(a[k], 0.f), xp);
    }
    const float x = xp + __shfl_xor_sync(0xffffffffu, xp, 1);  // the two halves of the entry
    double lsum = 0.0;
    float g = 0.f;
    if (valid) {
        const int y = labels[off + s0 + rr] != 0;
        const float p = 1.f / (1.f + expf(-x));
        const float pt = y ? p : 1.f - p;
        const float at = alpha < 0.f ? 1.f : (y ? alpha : 1.f - alpha);
        const float lpt = y ? -log1pf(expf(-x)) : -log1pf(expf(x));
        const float q1 = 1.f - pt;
        float dl;
        if (gamma == 0.f) {
            dl = at * (y ? p - 1.f : p);
            if (hf == 0) lsum = -(double)at * lpt;
        } else {
            dl = at * (gamma * powf(q1, gamma - 1.f) * lpt * pt * q1 - powf(q1, gamma) * q1) * (y ? 1.f : -1.f);
            if (hf == 0) lsum = -(double)at * powf(q1, gamma) * lpt;
        }
        g = (float)(dl * invN);
    }
    // G[rr][h] = g w_h 1[a_h > 0] scale;  dw_h += g ReLU(a_h)
#pragma unroll
    for (int k = 0; k < 32; k++) {
        const bool head = h0 + k < n_h;
        if (head) gs[rr * GP + h0 + k] = (valid && a[k] > 0.f) ? g * wsm[h0 + k] * scale : 0.f;
        float c = (valid && head) ? g * fmaxf(a[k], 0.f) : 0.f;
#pragma unroll
        for (int o = 16; o >= 2; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);  // lanes of the same half
        if ((threadIdx.x & 31) < 2 && head) atomicAdd(&dwsm[h0 + k], c);
    }
    // loss
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if ((threadIdx.x & 31) == 0) lred[threadIdx.x >> 5] = lsum;
    __syncthreads();
    // dq[h][e] += sum_rr G[rr][h] K[rr][e]: thread (e, half) takes heads half*32 .. +31
    {
        const int e = threadIdx.x >> 1, hh0 = (threadIdx.x & 1) * 32;
        if (e < d_I) {
            float acc[32];
#pragma unroll
            for (int k = 0; k < 32; k++) acc[k] = 0.f;
            for (int r2 = 0; r2 < nrow; r2++) {
                const float kv = ks[r2 * KP + e];
#pragma unroll
                for (int k = 0; k < 32; k++)
                    if (hh0 + k < n_h) acc[k] = fmaf(gs[r2 * GP + hh0 + k], kv, acc[k]);
            }
            float *dqb = dq + ((int64_t)l * B + b) * n_h * d_I;
#pragma unroll
            for (int k = 0; k < 32; k++)
                if (hh0 + k < n_h && acc[k] != 0.f) atomicAdd(dqb + (hh0 + k) * d_I + e, acc[k]);
        }
    }
    if (threadIdx.x < n_h) atomicAdd(dw + ((int64_t)l * B + b) * n_h + threadIdx.x, dwsm[threadIdx.x]);
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int i = 0; i < THREADS / 32; i++) s += lred[i];
        atomicAdd(loss, s * invN);
    }
}

// dc[l][b][j] = sum_o dq[l][b][o] W_iuq[l][o][j]
template <int DT>
__global__ void __launch_bounds__(256) k_train_dc(const float *__restrict__ dq, const void *__restrict__ W_iuq, int L,
                                                  int B, int nq, int r, float *__restrict__ dc)
{
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (idx >= (int64_t)L * B * r) return;
    const int j = (int)(idx % r);
    const int64_t lb = idx / r;
    const int l = (int)(lb / B);
    const float *dqb = dq + lb * nq;
    float acc = 0.f;
    for (int o = 0; o < nq; o++) acc = fmaf(dqb[o], load_elem<DT>(W_iuq, ((int64_t)l * nq + o) * r + j), acc);
    dc[idx] = acc;
}

// out[l][m][n] = sum_b U[l][b][m] V[l][b][n]; U fp32, V of type VDT
template <int VDT>
__global__ void __launch_bounds__(256) k_outer(const float *__restrict__ U, const void *__restrict__ V, int L, int B,
                                               int M, int N, float *__restrict__ out)
{
    const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (idx >= (int64_t)L * M * N) return;
    const int n = (int)(idx % N);
    const int64_t lm = idx / N;
    const int m = (int)(lm % M), l = (int)(lm / M);
    float acc = 0.f;
    for (int b = 0; b < B; b++)
        acc = fmaf(U[((int64_t)l * B + b) * M + m], load_elem<VDT>(V, ((int64_t)l * B + b) * N + n), acc);
    out[idx] = acc;
}

inline size_t entries_smem(void) { return sizeof(float) * ((size_t)NHMAX * DMAX + (size_t)TT * (DMAX + 1) + (size_t)TT * (NHMAX + 1)); }

}  // namespace train

}  // namespace lsa
