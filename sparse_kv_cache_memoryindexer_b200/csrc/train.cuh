// One training step of the memory indexer against frozen keys (hyper.ai summary, "Method"; blog
// review, section 3): forward as the index score, focal / binary cross-entropy loss against the
// window's golden labels, gradients of W^DQ, W^IUQ and W^w (the rounding of c and q to their
// storage type is passed straight through).
//
//   k_train_entries   TPC consecutive 128-entry tiles (global tile order) of one layer per CTA: the
//                     tile's keys and the sequence's queries in shared memory (fp32); per entry the
//                     64 head dot products a_h, x = sum_h w_h ReLU(a_h), the loss and g = dl/dx / N;
//                     then dw_h += g ReLU(a_h) and dq_h += (g w_h 1[a_h > 0] scale) K_s (a 64 x 128 x
//                     128 product per tile), added to the sequence's gradients with atomics.
//   k_train_dc        dc = dq W^IUQ (split over rows of W^IUQ, partial sums added with atomics).
//   k_outer           g_W[l][m][n] = sum_b U[l][b][m] V[l][b][n]: the three weight gradients.
#pragma once
#include "common.cuh"

namespace lsa {

namespace train {

constexpr int TT = 128;       // entries per tile
constexpr int THREADS = 256;  // two per entry
constexpr int NHMAX = 64;
constexpr int DMAX = 128;

// Register-tiled SIMT: in the forward, warp hg takes heads 8 hg .. 8 hg + 7 and lane takes entries
// lane + 32 i (i < 4), so each thread holds 4 x 8 products; in the dq product warp hq takes heads
// 8 hq .. + 7 and lane takes key dimensions lane + 32 j (j < 4).  Keys sit in shared memory as rows
// of d_I + 1 floats (odd stride: the column reads of both phases are free of bank conflicts), the
// queries transposed [d_I][64] and G [TT][68] (16-byte rows), so the per-head operands are float4
// broadcasts.  A CTA walks TPC consecutive tiles and adds its dq / dw to the sequence's gradients
// only when the sequence changes or at its end.
constexpr int TPC = 8;
constexpr int GP = NHMAX + 4;

template <int QDT, int KDT>
__global__ void __launch_bounds__(THREADS, 1) k_train_entries(const void *__restrict__ q, const float *__restrict__ w,
                                                              const void *__restrict__ K, const float *__restrict__ ksc,
                                                              const uint8_t *__restrict__ labels,
                                                              const int64_t *__restrict__ offs,
                                                              const int *__restrict__ tile_start, int B, int64_t T,
                                                              int n_h, int d_I, float gamma, float alpha, double invN,
                                                              float *__restrict__ dq, float *__restrict__ dw,
                                                              double *__restrict__ loss)
{
    extern __shared__ __align__(16) float sm[];
    float *qT = sm;                                  // [DMAX][NHMAX]
    float *gs = qT + DMAX * NHMAX;                   // [TT][GP]
    float *ks = gs + TT * GP;                        // [TT][d_I + 1]
    __shared__ float wsm[NHMAX], xpart[THREADS / 32][TT], gsm[TT], scsm[TT];
    __shared__ double lred[THREADS / 32];
    const int l = blockIdx.y;
    const int NT = tile_start[B];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int KP = d_I + 1;
    const int hg0 = warp * 8;                        // this warp's 8 heads (both phases)
    float dqa[8][4], dwa[8];
    double lsum = 0.0;
    int cur_b = -1;
    auto flush = [&](int bb) {
        float *dqb = dq + ((int64_t)l * B + bb) * n_h * d_I;
#pragma unroll
        for (int k = 0; k < 8; k++)
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = lane + 32 * j;
                if (hg0 + k < n_h && e < d_I && dqa[k][j] != 0.f) atomicAdd(dqb + (hg0 + k) * d_I + e, dqa[k][j]);
            }
        if (lane == 0)
#pragma unroll
            for (int k = 0; k < 8; k++)
                if (hg0 + k < n_h && dwa[k] != 0.f) atomicAdd(dw + ((int64_t)l * B + bb) * n_h + hg0 + k, dwa[k]);
    };
    for (int tt = 0; tt < TPC; tt++) {
        const int t = blockIdx.x * TPC + tt;
        if (t >= NT) break;
        int lo = 0, hi = B - 1;  // the sequence of tile t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_start[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        const int b = lo;
        if (b != cur_b) {
            if (cur_b >= 0) flush(cur_b);
#pragma unroll
            for (int k = 0; k < 8; k++) {
                dwa[k] = 0.f;
#pragma unroll
                for (int j = 0; j < 4; j++) dqa[k][j] = 0.f;
            }
            __syncthreads();  // the previous tile's readers of qT are done
            const int64_t qb = ((int64_t)l * B + b) * n_h * d_I;
            for (int i = threadIdx.x; i < DMAX * NHMAX; i += THREADS) qT[i] = 0.f;
            __syncthreads();
            {
                // the queries [n_h][d_I], 16-byte vector loads issued together, stored transposed
                constexpr int QB = QDT == DT_F32 ? 4 : 2;
                constexpr int QPV = 16 / QB;
                constexpr int NQV = (NHMAX * DMAX / QPV + THREADS - 1) / THREADS;
                const int vpr = d_I / QPV;
                const uint8_t *qp = (const uint8_t *)q + qb * QB;
                uint4 buf[NQV];
#pragma unroll
                for (int v = 0; v < NQV; v++) {
                    const int idx = threadIdx.x + v * THREADS;
                    buf[v] = idx < n_h * vpr ? __ldg((const uint4 *)(qp + (int64_t)idx * 16)) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int v = 0; v < NQV; v++) {
                    const int idx = threadIdx.x + v * THREADS;
                    if (idx < n_h * vpr) {
                        const int hh = idx / vpr, e0 = (idx % vpr) * QPV;
                        const uint32_t wv[4] = {buf[v].x, buf[v].y, buf[v].z, buf[v].w};
#pragma unroll
                        for (int j = 0; j < QPV; j++)
                            qT[(e0 + j) * NHMAX + hh] = QDT == DT_F32 ? __uint_as_float(wv[j])
                                                                     : bf16_bits_to_float((unsigned short)(wv[j >> 1] >> (16 * (j & 1))));
                    }
                }
            }
            for (int i = threadIdx.x; i < NHMAX; i += THREADS) wsm[i] = i < n_h ? w[((int64_t)l * B + b) * n_h + i] : 0.f;
            cur_b = b;
        }
        const int64_t off = offs[b], S = offs[b + 1] - off;
        const int64_t s0 = (int64_t)(t - tile_start[b]) * TT;
        const int nrow = (int)min((int64_t)TT, S - s0);
        __syncthreads();  // qT / wsm ready; the previous tile's readers of ks / gs are done
        {
            // 16-byte vector loads, all issued before any conversion (d_I is a multiple of EPV)
            constexpr int EB = KDT == DT_F32 ? 4 : (KDT == DT_BF16 ? 2 : 1);
            constexpr int EPV = 16 / EB;
            constexpr int NV = (TT * DMAX / EPV + THREADS - 1) / THREADS;
            const int vpr = d_I / EPV;
            const uint8_t *kb = (const uint8_t *)K + ((int64_t)l * T + off + s0) * d_I * EB;
            uint4 buf[NV];
#pragma unroll
            for (int v = 0; v < NV; v++) {
                const int idx = threadIdx.x + v * THREADS;
                const int rr = idx / vpr;
                buf[v] = make_uint4(0u, 0u, 0u, 0u);
                if (idx < TT * vpr && rr < nrow) buf[v] = __ldg((const uint4 *)(kb + (int64_t)idx * 16));
            }
#pragma unroll
            for (int v = 0; v < NV; v++) {
                const int idx = threadIdx.x + v * THREADS;
                if (idx < TT * vpr) {
                    const int rr = idx / vpr, e0 = (idx % vpr) * EPV;
                    const uint32_t wv[4] = {buf[v].x, buf[v].y, buf[v].z, buf[v].w};
                    float *dst = ks + rr * KP + e0;
#pragma unroll
                    for (int j = 0; j < EPV; j++) {
                        float f;
                        if (KDT == DT_F32) f = __uint_as_float(wv[j]);
                        else if (KDT == DT_BF16) f = bf16_bits_to_float((unsigned short)(wv[j >> 1] >> (16 * (j & 1))));
                        else f = e4m3_to_float((unsigned char)(wv[j >> 2] >> (8 * (j & 3))));
                        dst[j] = f;
                    }
                }
            }
        }
        if (threadIdx.x < TT)
            scsm[threadIdx.x] = (KDT == DT_FP8 && (int)threadIdx.x < nrow) ? ksc[(int64_t)l * T + off + s0 + threadIdx.x] : 1.f;
        __syncthreads();
        // forward: a[i][k] = scale (q_{hg0+k} . K_{lane+32i})
        float a[4][8];
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int k = 0; k < 8; k++) a[i][k] = 0.f;
        for (int e = 0; e < d_I; e++) {
            const float4 q0 = *(const float4 *)(qT + e * NHMAX + hg0), q1 = *(const float4 *)(qT + e * NHMAX + hg0 + 4);
            const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float kv = ks[(lane + 32 * i) * KP + e];
#pragma unroll
                for (int k = 0; k < 8; k++) a[i][k] = fmaf(qv[k], kv, a[i][k]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float sc = scsm[lane + 32 * i];
            float xp = 0.f;
#pragma unroll
            for (int k = 0; k < 8; k++) {
                a[i][k] *= sc;
                xp = fmaf(wsm[hg0 + k], fmaxf(a[i][k], 0.f), xp);
            }
            xpart[warp][lane + 32 * i] = xp;
        }
        __syncthreads();
        // per entry: x, loss, g = dl/dx / N
        if (threadIdx.x < TT) {
            const int rr = threadIdx.x;
            float g = 0.f;
            if (rr < nrow) {
                float x = 0.f;
#pragma unroll
                for (int wv = 0; wv < THREADS / 32; wv++) x += xpart[wv][rr];
                const int y = labels[off + s0 + rr] != 0;
                const float p = 1.f / (1.f + expf(-x));
                const float pt = y ? p : 1.f - p;
                const float at = alpha < 0.f ? 1.f : (y ? alpha : 1.f - alpha);
                const float lpt = y ? -log1pf(expf(-x)) : -log1pf(expf(x));
                const float q1 = 1.f - pt;
                float dl;
                if (gamma == 0.f) {
                    dl = at * (y ? p - 1.f : p);
                    lsum -= (double)at * lpt;
                } else {
                    dl = at * (gamma * powf(q1, gamma - 1.f) * lpt * pt * q1 - powf(q1, gamma) * q1) * (y ? 1.f : -1.f);
                    lsum -= (double)at * powf(q1, gamma) * lpt;
                }
                g = (float)(dl * invN);
            }
            gsm[rr] = g;
        }
        __syncthreads();
        // G[r][h] = g w_h 1[a > 0] scale_r;  dw_h += g ReLU(a)
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int rr = lane + 32 * i;
            const float g = gsm[rr], sc = scsm[rr];
#pragma unroll
            for (int k = 0; k < 8; k++) {
                gs[rr * GP + hg0 + k] = a[i][k] > 0.f ? g * wsm[hg0 + k] * sc : 0.f;
                float c = g * fmaxf(a[i][k], 0.f);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
                dwa[k] += c;  // every lane holds the warp's sum; lane 0 adds it at the flush
            }
        }
        __syncthreads();
        // dq[h][e] += sum_r G[r][h] K[r][e]
        for (int rr = 0; rr < nrow; rr++) {
            const float4 g0 = *(const float4 *)(gs + rr * GP + hg0), g1 = *(const float4 *)(gs + rr * GP + hg0 + 4);
            const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = lane + 32 * j;
                const float kv = e < d_I ? ks[rr * KP + e] : 0.f;
#pragma unroll
                for (int k = 0; k < 8; k++) dqa[k][j] = fmaf(gv[k], kv, dqa[k][j]);
            }
        }
    }
    if (cur_b >= 0) flush(cur_b);
    // loss
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if (lane == 0) lred[warp] = lsum;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s2 = 0.0;
        for (int i = 0; i < THREADS / 32; i++) s2 += lred[i];
        if (s2 != 0.0) atomicAdd(loss, s2 * invN);
    }
}

// dc[l][b][j] = sum_o dq[l][b][o] W_iuq[l][o][j] (W^IUQ read once, memory-bound): one CTA per
// (layer, DC_COLS columns, DC_OCH rows o); thread t takes 4 consecutive columns (one 8- or 16-byte
// load of W per row, coalesced, 16 rows in flight) and keeps BM sequences' sums (BM = B rounded up
// to 8 or 16, so no FMA is predicated off); the CTA's dq rows sit in shared memory as [o][BM]
// (read as float4 broadcasts), and the partial sums over the CTA's rows are added to dc (zeroed
// before) with atomics.
constexpr int DC_BMAX = 16;
constexpr int DC_OCH = 128;
constexpr int DC_COLS = 1024;

template <int DT, int BM>
__global__ void __launch_bounds__(256) k_train_dc(const float *__restrict__ dq, const void *__restrict__ W_iuq, int L,
                                                  int B, int nq, int r, float *__restrict__ dc)
{
    __shared__ float4 sdq4[DC_OCH][BM / 4];
    float *sdq = (float *)sdq4;
    const int l = blockIdx.z;
    const int o0 = blockIdx.y * DC_OCH;
    const int j = blockIdx.x * DC_COLS + 4 * threadIdx.x;
    const int on = min(DC_OCH, nq - o0);
    for (int i = threadIdx.x; i < BM * DC_OCH; i += 256) {  // coalesced over o
        const int bb = i / DC_OCH, o = i % DC_OCH;
        sdq[o * BM + bb] = (o < on && bb < B) ? __ldg(dq + ((int64_t)l * B + bb) * nq + o0 + o) : 0.f;
    }
    __syncthreads();
    if (j >= r) return;  // r is a multiple of 4
    float acc[BM][4];
#pragma unroll
    for (int bb = 0; bb < BM; bb++) acc[bb][0] = acc[bb][1] = acc[bb][2] = acc[bb][3] = 0.f;
    const int64_t wrow = (int64_t)l * nq + o0;
#pragma unroll 16
    for (int o = 0; o < on; o++) {
        float w[4];
        if (DT == DT_F32) {
            const float4 v = __ldg((const float4 *)((const float *)W_iuq + (wrow + o) * r + j));
            w[0] = v.x;
            w[1] = v.y;
            w[2] = v.z;
            w[3] = v.w;
        } else {
            const uint2 v = __ldg((const uint2 *)((const unsigned short *)W_iuq + (wrow + o) * r + j));
            w[0] = __uint_as_float(v.x << 16);
            w[1] = __uint_as_float(v.x & 0xffff0000u);
            w[2] = __uint_as_float(v.y << 16);
            w[3] = __uint_as_float(v.y & 0xffff0000u);
        }
#pragma unroll
        for (int bq = 0; bq < BM / 4; bq++) {
            const float4 d = sdq4[o][bq];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                acc[4 * bq + 0][c] = fmaf(d.x, w[c], acc[4 * bq + 0][c]);
                acc[4 * bq + 1][c] = fmaf(d.y, w[c], acc[4 * bq + 1][c]);
                acc[4 * bq + 2][c] = fmaf(d.z, w[c], acc[4 * bq + 2][c]);
                acc[4 * bq + 3][c] = fmaf(d.w, w[c], acc[4 * bq + 3][c]);
            }
        }
    }
#pragma unroll
    for (int bb = 0; bb < BM; bb++) {
        if (bb < B) {
            float *dst = dc + ((int64_t)l * B + bb) * r + j;
#pragma unroll
            for (int c = 0; c < 4; c++)
                if (acc[bb][c] != 0.f) atomicAdd(dst + c, acc[bb][c]);
        }
    }
}

// out[l][m][n] = sum_b U[l][b][m] V[l][b][n] (U fp32, V of type VDT), written once (store-bound):
// thread t of block (x, y, l) takes 4 consecutive n (one 16-byte store per row) and OUT_MR rows m,
// with V[l][0..B)[n..n+3] kept in registers.  N is a multiple of 4, B at most DC_BMAX.
constexpr int OUT_MR = 8;

template <int VDT, int BM>  // BM: B rounded up to 8 or DC_BMAX (registers for V)
__global__ void __launch_bounds__(256) k_outer(const float *__restrict__ U, const void *__restrict__ V, int L, int B,
                                               int M, int N, float *__restrict__ out)
{
    __shared__ float su[BM][OUT_MR];
    const int l = blockIdx.z;
    const int n = (blockIdx.x * 256 + threadIdx.x) * 4;
    const int m0 = blockIdx.y * OUT_MR;
    if (threadIdx.x < BM * OUT_MR) {  // the CTA's rows of U for every sequence
        const int bb = threadIdx.x / OUT_MR, mi = threadIdx.x % OUT_MR;
        su[bb][mi] = (bb < B && m0 + mi < M) ? __ldg(U + ((int64_t)l * B + bb) * M + m0 + mi) : 0.f;
    }
    __syncthreads();
    if (n >= N) return;
    float4 vb[BM];
#pragma unroll
    for (int bb = 0; bb < BM; bb++) {
        vb[bb] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (bb < B) {
            const int64_t at = ((int64_t)l * B + bb) * N + n;
            vb[bb] = make_float4(load_elem<VDT>(V, at), load_elem<VDT>(V, at + 1), load_elem<VDT>(V, at + 2),
                                 load_elem<VDT>(V, at + 3));
        }
    }
#pragma unroll 2
    for (int mi = 0; mi < OUT_MR; mi++) {
        const int m = m0 + mi;
        if (m >= M) break;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int bb = 0; bb < BM; bb++) {
            if (bb < B) {
                const float u = su[bb][mi];
                acc.x = fmaf(u, vb[bb].x, acc.x);
                acc.y = fmaf(u, vb[bb].y, acc.y);
                acc.z = fmaf(u, vb[bb].z, acc.z);
                acc.w = fmaf(u, vb[bb].w, acc.w);
            }
        }
        *(float4 *)(out + ((int64_t)l * M + m) * N + n) = acc;
    }
}

inline size_t entries_smem(void) { return sizeof(float) * ((size_t)DMAX * NHMAX + (size_t)TT * GP + (size_t)TT * (DMAX + 1)); }

}  // namespace train

}  // namespace lsa
