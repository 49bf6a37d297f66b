// Stage 5: native Lightning-Indexer score over the fetched entries and per-query Top-k
// (blog review "FlashMemory-DeepSeek-V4", sections 2.2 and 3.2).
//
// Scores of sequence b, query i, fetched slot j live at Y[tau*off_b + i*S_b + j] (fp32).
// Selection: per query, a radix select on order-preserving 32-bit keys (4 passes of 8 bits)
// finds the k-th largest score; the survivors (all larger keys, plus the first equal keys in
// slot order, i.e. smallest entry index) are sorted by (score desc, entry asc) with a bitonic
// sort in shared memory.
#pragma once
#include "common.cuh"

namespace lsa {

// SIMT score: one thread per fetched slot, all tau queries of its sequence.
template <int D, int KDT, int QDT>
__global__ void __launch_bounds__(TILE) k_li_score_simt(const void *__restrict__ qd, const float *__restrict__ wd,
                                                         const void *__restrict__ hotK,
                                                         const float *__restrict__ hotsc,
                                                         const int32_t *__restrict__ count,
                                                         const int64_t *__restrict__ offs, int tau, int n_h,
                                                         float *__restrict__ Y)
{
    extern __shared__ float smem[];
    float *sq = smem;
    float *sw = smem + n_h * D;
    const int b = blockIdx.y;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    for (int64_t j0 = (int64_t)blockIdx.x * TILE; j0 < F; j0 += (int64_t)gridDim.x * TILE) {
        const int64_t j = j0 + threadIdx.x;
        const bool valid = j < F;
        float kr[D];
        float scale = 1.f;
        if (valid) {
#pragma unroll
            for (int e = 0; e < D; e++) kr[e] = load_elem<KDT>(hotK, (off + j) * D + e);
            if (hotsc) {
                scale = hotsc[off + j];
                if (!(scale >= 0.f)) flag(ERRF_SCALE);
            }
        }
        for (int i = 0; i < tau; i++) {
            __syncthreads();
            const int64_t q0 = (((int64_t)b * tau + i) * n_h) * D;
            for (int t = threadIdx.x; t < n_h * D; t += blockDim.x) sq[t] = load_elem<QDT>(qd, q0 + t);
            for (int t = threadIdx.x; t < n_h; t += blockDim.x) sw[t] = wd[((int64_t)b * tau + i) * n_h + t];
            __syncthreads();
            if (!valid) continue;
            float y = 0.f;
            for (int h = 0; h < n_h; h++) {
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < D; e++) dot = fmaf(sq[h * D + e], kr[e], dot);
                y = fmaf(sw[h], fmaxf(dot * scale, 0.f), y);
            }
            Y[(int64_t)tau * off + (int64_t)i * S + j] = y;
        }
    }
}

constexpr int SEL_THREADS = 512;

// Block-wide exclusive scan of one int per thread (SEL_THREADS threads); returns the
// exclusive prefix and writes the block total to *total.  Ends with a barrier.
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int inc = warp_incl_scan(v);
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int t = lane < SEL_THREADS / 32 ? warp_tot[lane] : 0;
        int ti = warp_incl_scan(t);
        if (lane < SEL_THREADS / 32) warp_tot[lane] = ti - t;
        if (lane == 31) *total = ti;
    }
    __syncthreads();
    const int r = warp_tot[warp] + inc - v;
    __syncthreads();
    return r;
}

// One block per (sequence, query).  kpow2 = next power of two >= k (shared: kpow2 x 8 bytes).
// TAIL: after the F fetched slots of sequence b come tail_count[b] (at most W) more candidates,
// the entries compressed during the window (scores tail[b*W + j], entry numbers S_b + j); the Y rows
// then have tau_y queries per sequence of which block (b, i) reads query i.
template <bool TAIL>
__global__ void __launch_bounds__(SEL_THREADS) k_topk_select(const float *__restrict__ Y,
                                                             const int32_t *__restrict__ idx,
                                                             const int32_t *__restrict__ count,
                                                             const int64_t *__restrict__ offs, int tau, int k,
                                                             int kpow2, int32_t *__restrict__ topk_idx,
                                                             float *__restrict__ topk_score,
                                                             const float *__restrict__ tail = nullptr,
                                                             const int32_t *__restrict__ tail_count = nullptr,
                                                             int W = 0, int tau_y = 0)
{
    extern __shared__ unsigned long long sel[];  // (key << 32) | ~slot
    __shared__ unsigned int hist[256];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, tot_b;
    __shared__ unsigned int s_prefix, s_remaining;

    const int b = blockIdx.x / tau, i = blockIdx.x % tau;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F0 = count[b];
    F0 = F0 < 0 ? 0 : (F0 > S ? (int)S : F0);
    const float *row = Y + (int64_t)(TAIL ? tau_y : tau) * off + (int64_t)i * S;
    int nt = 0;
    if (TAIL && tail_count) {
        nt = tail_count[b];
        nt = nt < 0 ? 0 : (nt > W ? W : nt);
    }
    const float *trow = TAIL ? tail + (int64_t)b * W : nullptr;
    const int F = F0 + nt;  // candidates
    auto cand = [&](int j) { return (!TAIL || j < F0) ? row[j] : trow[j - F0]; };

    for (int t = threadIdx.x; t < kpow2; t += SEL_THREADS) sel[t] = 0ull;
    __syncthreads();

    if (F <= k) {
        for (int j = threadIdx.x; j < F; j += SEL_THREADS)
            sel[j] = ((unsigned long long)float_to_ordered(cand(j)) << 32) | (uint32_t)(~(uint32_t)j);
    } else {
        uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
        for (int pass = 0; pass < 4; pass++) {
            const int shift = 24 - 8 * pass;
            for (int t = threadIdx.x; t < 256; t += SEL_THREADS) hist[t] = 0;
            __syncthreads();
            for (int j = threadIdx.x; j < F; j += SEL_THREADS) {
                const uint32_t u = float_to_ordered(cand(j));
                if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                uint32_t cum = 0, chosen = 0;
                for (int d = 255; d >= 0; d--) {
                    if (cum + hist[d] >= remaining) {
                        chosen = (uint32_t)d;
                        break;
                    }
                    cum += hist[d];
                }
                s_remaining = remaining - cum;
                s_prefix = prefix | (chosen << shift);
            }
            __syncthreads();
            prefix = s_prefix;
            remaining = s_remaining;
            pmask |= 255u << shift;
            __syncthreads();
        }
        // prefix is now the k-th largest key; take every larger key and the first `remaining`
        // equal keys in slot order.
        int carry_gt = 0, carry_eq = 0;
        const int n_gt_total = k - (int)remaining;
        for (int base = 0; base < F; base += SEL_THREADS) {
            const int j = base + threadIdx.x;
            uint32_t u = 0;
            int gt = 0, eq = 0;
            if (j < F) {
                u = float_to_ordered(cand(j));
                gt = u > prefix;
                eq = u == prefix;
            }
            const int pg = block_excl_scan(gt, warp_tot, &tot_a) + carry_gt;
            const int pe = block_excl_scan(eq, warp_tot, &tot_b) + carry_eq;
            if (gt) sel[pg] = ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j);
            if (eq && pe < (int)remaining)
                sel[n_gt_total + pe] = ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j);
            carry_gt += tot_a;
            carry_eq += tot_b;
            __syncthreads();
        }
    }
    __syncthreads();
    // bitonic sort, descending
    for (int size = 2; size <= kpow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < kpow2 / 2; t += SEL_THREADS) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool desc = ((lo & size) == 0);
                const unsigned long long a = sel[lo], c = sel[hi];
                if ((a < c) == desc) {
                    sel[lo] = c;
                    sel[hi] = a;
                }
            }
            __syncthreads();
        }
    }
    const int nsel = F < k ? F : k;
    const int64_t o0 = ((int64_t)b * tau + i) * k;
    for (int r = threadIdx.x; r < k; r += SEL_THREADS) {
        if (r < nsel) {
            const unsigned long long v = sel[r];
            const int j = (int)~(uint32_t)(v & 0xffffffffull);  // candidate slot (always below F)
            topk_idx[o0 + r] = (j >= 0 && j < F0) ? __ldg(idx + off + j)
                                                  : ((j >= F0 && j < F) ? (int32_t)(S + (j - F0)) : -1);
            if (topk_score) topk_score[o0 + r] = ordered_to_float((uint32_t)(v >> 32));
        } else {
            topk_idx[o0 + r] = -1;
            if (topk_score) topk_score[o0 + r] = -INFINITY;
        }
    }
}

// ------------------------------------------------------------------ one decode step
// Stage 5 for one decode step: each sequence's query of the step is copied into TQ query slots
// (slot 0; the others are zero, as are their weights) so that the scorers built for groups of
// queries serve the step unchanged.  qs / ws are the step's queries and weights with a batch
// stride (elements) between sequences.
__global__ void __launch_bounds__(256) k_step_prep(const void *__restrict__ qs, int64_t q_bstride,
                                                   const float *__restrict__ ws, int64_t w_bstride, int dt, int B,
                                                   int TQ, int n_h, int d_I, void *__restrict__ q_out,
                                                   float *__restrict__ w_out)
{
    const int64_t rows = (int64_t)B * TQ * n_h;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int h = (int)(r % n_h);
    const int qi = (int)((r / n_h) % TQ);
    const int b = (int)(r / ((int64_t)n_h * TQ));
    const size_t es = dt == DT_F32 ? 4 : 2;
    uint8_t *dst = (uint8_t *)q_out + (size_t)r * d_I * es;
    const uint8_t *src = (const uint8_t *)qs + ((size_t)b * q_bstride + (size_t)h * d_I) * es;
    for (int e = lane; e < d_I; e += 32) {
        if (es == 4) ((float *)dst)[e] = qi == 0 ? ((const float *)src)[e] : 0.f;
        else ((uint16_t *)dst)[e] = qi == 0 ? ((const uint16_t *)src)[e] : (uint16_t)0;
    }
    if (lane == 0) w_out[r] = qi == 0 ? ws[(size_t)b * w_bstride + h] : 0.f;
}

// Scores of the entries compressed during the window: one warp per (sequence, entry j < W);
// y = sum_h w_h ReLU(scale_j q_h . k_j).  Keys [B][W][d_I] in the hot-key type, scales nullable.
__global__ void __launch_bounds__(256) k_li_window(const void *__restrict__ q, const float *__restrict__ w,
                                                   int TQ, int dt, const void *__restrict__ winK,
                                                   const float *__restrict__ winsc,
                                                   const int32_t *__restrict__ win_count, int B, int W, int n_h,
                                                   int d_I, float *__restrict__ tail)
{
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= (int64_t)B * W) return;
    const int b = (int)(gw / W), j = (int)(gw % W);
    int n = win_count[b];
    if (n < 0 || n > W) {
        if (lane == 0 && j == 0) flag(ERRF_COUNT);
        n = n < 0 ? 0 : W;
    }
    if (j >= n) return;
    const float sc = winsc ? winsc[(int64_t)b * W + j] : 1.f;
    if (winsc && lane == 0 && !(sc >= 0.f)) flag(ERRF_SCALE);
    const size_t es = dt == DT_F32 ? 4 : 2;
    const uint8_t *kr = (const uint8_t *)winK + ((size_t)b * W + j) * d_I * es;
    float y = 0.f;
    for (int h = lane; h < n_h; h += 32) {
        const uint8_t *qr = (const uint8_t *)q + ((size_t)b * TQ * n_h + h) * d_I * es;  // query slot 0
        float d = 0.f;
        for (int e = 0; e < d_I; e++) {
            const float qv = es == 4 ? ((const float *)qr)[e] : __bfloat162float(((const __nv_bfloat16 *)qr)[e]);
            const float kv = es == 4 ? ((const float *)kr)[e] : __bfloat162float(((const __nv_bfloat16 *)kr)[e]);
            d = fmaf(qv, kv, d);
        }
        y = fmaf(w[(size_t)b * TQ * n_h + h], fmaxf(sc * d, 0.f), y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
    if (lane == 0) tail[(int64_t)b * W + j] = y;
}

}  // namespace lsa
