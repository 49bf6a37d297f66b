// Stage 5: native Lightning-Indexer score over the fetched entries and per-query Top-k
// (blog review "FlashMemory-DeepSeek-V4", sections 2.2 and 3.2).
//
// Scores of sequence b, query i, fetched slot j live at Y[tau*off_b + i*S_b + j] (fp32).
// Selection: per query, a radix select on order-preserving 32-bit keys finds the k-th largest
// score (12 + 10 + 10 bits, two reads of the scores); the survivors (all larger keys, plus the
// first equal keys in slot order, i.e. smallest entry index) are sorted by (score desc, entry asc)
// with a bitonic sort in shared memory.
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

// Order-preserving keys of a query's candidates are split as 12 + 10 + 10 bits.  SEL_CAP keys of the
// k-th key's 12-bit bucket are staged in shared memory, so that the two finer passes read shared
// memory instead of the scores again.
constexpr int SEL_BINS = 4096;
constexpr int SEL_CAP = 4096;

// The bin holding the `want`-th largest key of a histogram of NB bins (thread t owns NB / SEL_THREADS
// consecutive bins, highest first): *bin_out, and *above_out = keys in higher bins.  want >= 1 and
// at most the histogram's total.  Ends with a barrier.
template <int NB>
__device__ __forceinline__ void sel_find_bin(const unsigned int *hist, int want, int *warp_tot, int *tot, int *bin_out,
                                             int *above_out)
{
    constexpr int PER = NB / SEL_THREADS;
    const int hi = NB - PER * (int)threadIdx.x;  // bins [hi - PER, hi)
    int cnt = 0;
#pragma unroll
    for (int q = 1; q <= PER; q++) cnt += (int)hist[hi - q];
    int above = block_excl_scan(cnt, warp_tot, tot);
    if (above < want && above + cnt >= want) {
#pragma unroll
        for (int q = 1; q <= PER; q++) {
            const int c = (int)hist[hi - q];
            if (above + c >= want) {
                *bin_out = hi - q;
                *above_out = above;
                break;
            }
            above += c;
        }
    }
    __syncthreads();
}

// One block per (sequence, query).  kpow2 = next power of two >= k; dynamic shared memory:
// kpow2 + SEL_CAP 8-byte keys.  When the candidates exceed k: a 12-bit histogram of the keys
// (one read of the scores) gives the bucket of the k-th largest key; a second read writes every key
// of a higher bucket to the selection in slot order and stages the bucket's own keys (slot order)
// in shared memory; two 10-bit passes over those find the k-th key K, and the staged keys above K,
// then the first keys equal to K in slot order (smallest entry index), complete the selection.  A
// bucket of more than SEL_CAP keys takes three 8-bit passes over the scores instead.  The k keys
// are sorted by (score desc, slot asc) with a bitonic sort in shared memory.
__global__ void __launch_bounds__(SEL_THREADS) k_topk_select(const float *__restrict__ Y,
                                                             const int32_t *__restrict__ idx,
                                                             const int32_t *__restrict__ count,
                                                             const int64_t *__restrict__ offs, int tau, int k,
                                                             int kpow2, int32_t *__restrict__ topk_idx,
                                                             float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sel[];  // [kpow2] (key << 32) | ~slot, then [SEL_CAP] staged keys
    unsigned long long *stage = sel + kpow2;
    __shared__ unsigned int hist[SEL_BINS];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, tot_b, s_bin, s_above;

    const int b = blockIdx.x / tau, i = blockIdx.x % tau;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    const float *row = Y + (int64_t)tau * off + (int64_t)i * S;
    const int lane = threadIdx.x & 31;
    auto key64 = [](uint32_t u, int j) { return ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j); };

    for (int t = threadIdx.x; t < kpow2; t += SEL_THREADS) sel[t] = 0ull;
    __syncthreads();

    if (F <= k) {
        for (int j = threadIdx.x; j < F; j += SEL_THREADS) sel[j] = key64(float_to_ordered(__ldg(row + j)), j);
    } else {
        // read 1: 12-bit histogram (lanes with the same bucket add once)
        for (int t = threadIdx.x; t < SEL_BINS; t += SEL_THREADS) hist[t] = 0;
        __syncthreads();
        for (int base = 0; base < F; base += SEL_THREADS) {
            const int j = base + threadIdx.x;
            const uint32_t bk = j < F ? float_to_ordered(__ldg(row + j)) >> 20 : 0xFFFFFFFFu;
            const unsigned peers = __match_any_sync(0xffffffffu, bk);
            if (bk != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[bk], (unsigned)__popc(peers));
        }
        __syncthreads();
        sel_find_bin<SEL_BINS>(hist, k, warp_tot, &tot_a, &s_bin, &s_above);
        const uint32_t beta = (uint32_t)s_bin;
        const int above = s_above;              // keys of higher buckets: all selected
        const int nbeta = (int)hist[beta];
        const bool staged = nbeta <= SEL_CAP;
        __syncthreads();
        // read 2: higher buckets to the selection, the k-th key's bucket to the stage (slot order)
        int carry_gt = 0, carry_eq = 0;
        for (int base = 0; base < F; base += SEL_THREADS) {
            const int j = base + threadIdx.x;
            uint32_t u = 0;
            int gt = 0, eq = 0;
            if (j < F) {
                u = float_to_ordered(__ldg(row + j));
                gt = (u >> 20) > beta;
                eq = (u >> 20) == beta;
            }
            const int pg = block_excl_scan(gt, warp_tot, &tot_a) + carry_gt;
            const int pe = block_excl_scan(eq, warp_tot, &tot_b) + carry_eq;
            if (gt) sel[pg] = key64(u, j);
            if (eq && staged) stage[pe] = key64(u, j);
            carry_gt += tot_a;
            carry_eq += tot_b;
            __syncthreads();
        }
        const int want = k - above;             // keys still to take from bucket beta (>= 1)
        if (staged) {
            // two 10-bit passes over the staged keys
            uint32_t prefix = beta << 20, pmask = 0xFFF00000u;
            int remaining = want;
#pragma unroll 1
            for (int pass = 0; pass < 2; pass++) {
                const int shift = 10 - 10 * pass;
                for (int t = threadIdx.x; t < 1024; t += SEL_THREADS) hist[t] = 0;
                __syncthreads();
                for (int q = threadIdx.x; q < nbeta; q += SEL_THREADS) {
                    const uint32_t u = (uint32_t)(stage[q] >> 32);
                    if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 1023u], 1u);
                }
                __syncthreads();
                sel_find_bin<1024>(hist, remaining, warp_tot, &tot_a, &s_bin, &s_above);
                prefix |= (uint32_t)s_bin << shift;
                remaining -= s_above;
                pmask |= 1023u << shift;
                __syncthreads();
            }
            // prefix is the k-th largest key; take the staged keys above it, then the first
            // `remaining` equal to it in slot order
            int cg = 0, ce = 0;
            for (int base = 0; base < nbeta; base += SEL_THREADS) {
                const int q = base + threadIdx.x;
                unsigned long long v = 0ull;
                int gt = 0, eq = 0;
                if (q < nbeta) {
                    v = stage[q];
                    const uint32_t u = (uint32_t)(v >> 32);
                    gt = u > prefix;
                    eq = u == prefix;
                }
                const int pg = block_excl_scan(gt, warp_tot, &tot_a) + cg;
                const int pe = block_excl_scan(eq, warp_tot, &tot_b) + ce;
                if (gt) sel[above + pg] = v;
                if (eq && pe < remaining) sel[k - remaining + pe] = v;
                cg += tot_a;
                ce += tot_b;
                __syncthreads();
            }
        } else {
            // a crowded bucket: three 8-bit passes over the scores for the low 20 bits
            uint32_t prefix = beta << 20, pmask = 0xFFF00000u;
            int remaining = want;
#pragma unroll 1
            for (int pass = 0; pass < 3; pass++) {
                const int shift = pass < 2 ? 12 - 8 * pass : 0;
                const uint32_t bins = pass < 2 ? 255u : 15u;
                for (int t = threadIdx.x; t < 1024; t += SEL_THREADS) hist[t] = 0;
                __syncthreads();
                for (int j = threadIdx.x; j < F; j += SEL_THREADS) {
                    const uint32_t u = float_to_ordered(__ldg(row + j));
                    if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & bins], 1u);
                }
                __syncthreads();
                sel_find_bin<1024>(hist, remaining, warp_tot, &tot_a, &s_bin, &s_above);
                prefix |= (uint32_t)s_bin << shift;
                remaining -= s_above;
                pmask |= bins << shift;
                __syncthreads();
            }
            int cg = 0, ce = 0;
            for (int base = 0; base < F; base += SEL_THREADS) {
                const int j = base + threadIdx.x;
                uint32_t u = 0;
                int gt = 0, eq = 0;
                if (j < F) {
                    u = float_to_ordered(__ldg(row + j));
                    gt = (u >> 20) == beta && u > prefix;
                    eq = u == prefix;
                }
                const int pg = block_excl_scan(gt, warp_tot, &tot_a) + cg;
                const int pe = block_excl_scan(eq, warp_tot, &tot_b) + ce;
                if (gt) sel[above + pg] = key64(u, j);
                if (eq && pe < remaining) sel[k - remaining + pe] = key64(u, j);
                cg += tot_a;
                ce += tot_b;
                __syncthreads();
            }
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
            topk_idx[o0 + r] = (j >= 0 && j < F) ? __ldg(idx + off + j) : -1;
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
// Lane l holds key elements l * E .. l * E + E - 1 (E = d_I / 32); per head the lanes read their
// part of the query row (one coalesced row per head) and a warp sum gives the dot product.
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
    const int E = d_I >> 5;  // 1, 2 or 4
    const bool f32 = dt == DT_F32;
    const int64_t kb = ((int64_t)b * W + j) * d_I + (int64_t)lane * E;
    float kv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 4; e++)
        if (e < E) kv[e] = f32 ? __ldg((const float *)winK + kb + e) : bf16_bits_to_float(__ldg((const unsigned short *)winK + kb + e));
    const int64_t qb = (int64_t)b * TQ * n_h * d_I + (int64_t)lane * E;  // query slot 0
    const float *wr = w + (int64_t)b * TQ * n_h;
    float y = 0.f;
    for (int h = 0; h < n_h; h++) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 4; e++) {
            if (e < E) {
                const int64_t at = qb + (int64_t)h * d_I + e;
                const float qv = f32 ? __ldg((const float *)q + at) : bf16_bits_to_float(__ldg((const unsigned short *)q + at));
                d = fmaf(qv, kv[e], d);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        y = fmaf(__ldg(wr + h), fmaxf(sc * d, 0.f), y);
    }
    if (lane == 0) tail[(int64_t)b * W + j] = y;
}

}  // namespace lsa
