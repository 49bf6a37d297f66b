// Stage 5: native Lightning-Indexer score over the fetched entries and per-query Top-k
// (blog review "FlashMemory-DeepSeek-V4", sections 2.2 and 3.2).
//
// Scores of sequence b, query i, fetched slot j live at Y[tau*off_b + i*S_b + j] (fp32).
// Selection: per query, the k-th largest score is found on order-preserving keys held in shared
// memory (a 12-bit bucket histogram, then the bucket's keys); the survivors are sorted by (score
// desc, entry asc) with a bitonic sort in shared memory (k_topk_select).
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

constexpr int SEL_THREADS = 1024;

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

// The k-th largest key of a query is found from a 12-bit histogram of the order-preserving score
// keys (its bucket beta) and then inside the bucket; a candidate's 64-bit key (score key << 32) |
// ~slot orders by score and then by smaller slot, and no two are equal.
constexpr int SEL_BINS = 4096;
constexpr int SEL_CAP = 4096;      // bucket keys sorted in shared memory

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

// Shared memory of k_topk_select for kpow2 and a key capacity fcap (dynamic part).
__host__ __device__ inline size_t topk_select_smem(int kpow2, int fcap)
{
    return sizeof(unsigned long long) * ((size_t)kpow2 + SEL_CAP) + sizeof(uint32_t) * (size_t)fcap;
}

// One block per (sequence, query).  kpow2 = next power of two >= max(k, 64).  Dynamic shared memory:
// kpow2 selection keys, SEL_CAP staged keys, then the query's score keys when it has at most fcap
// candidates (read from the scores once, eight independent loads in flight per thread; a larger
// query reads its scores from global memory at every pass).  With more than k candidates: a 12-bit
// histogram gives the bucket beta of the k-th largest key; the keys of higher buckets are appended
// to the selection and the bucket's keys to the stage (any order: the keys carry their slots); the
// stage sorted by key gives the bucket's largest keys.  A bucket of more than SEL_CAP keys is
// resolved by three more radix passes (8/8/4 bits) and an ordered pass (the first keys equal to
// the k-th in slot order).  The k keys are sorted by (score desc, slot asc).
__global__ void __launch_bounds__(SEL_THREADS) k_topk_select(const float *__restrict__ Y,
                                                             const int32_t *__restrict__ idx,
                                                             const int32_t *__restrict__ count,
                                                             const int64_t *__restrict__ offs, int tau, int k,
                                                             int kpow2, int fcap, int32_t *__restrict__ topk_idx,
                                                             float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sel[];  // [kpow2] selection, [SEL_CAP] stage, then keys
    unsigned long long *stage = sel + kpow2;
    uint32_t *keys = (uint32_t *)(stage + SEL_CAP);
    __shared__ unsigned int hist[SEL_BINS];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, tot_b, s_bin, s_above, s_ngt, s_nst;

    const int b = blockIdx.x / tau, i = blockIdx.x % tau;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    const float *row = Y + (int64_t)tau * off + (int64_t)i * S;
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    const bool resident = F <= fcap;
    auto key64 = [](uint32_t u, int j) { return ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j); };
    auto key_at = [&](int j) -> uint32_t { return resident ? keys[j] : float_to_ordered(__ldg(row + j)); };

    if (resident) {
        for (int base = 0; base < F; base += 8 * SEL_THREADS) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; q++) {
                const int j = base + q * SEL_THREADS + threadIdx.x;
                v[q] = j < F ? __ldg(row + j) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; q++) {
                const int j = base + q * SEL_THREADS + threadIdx.x;
                if (j < F) keys[j] = float_to_ordered(v[q]);
            }
        }
    }
    for (int t = threadIdx.x; t < kpow2; t += SEL_THREADS) sel[t] = 0ull;
    __syncthreads();

    if (F <= k) {
        for (int j = threadIdx.x; j < F; j += SEL_THREADS) sel[j] = key64(key_at(j), j);
    } else {
        for (int t = threadIdx.x; t < SEL_BINS; t += SEL_THREADS) hist[t] = 0;
        if (threadIdx.x == 0) s_ngt = s_nst = 0;
        __syncthreads();
        for (int j = threadIdx.x; j < F; j += SEL_THREADS) atomicAdd(&hist[key_at(j) >> 20], 1u);
        __syncthreads();
        sel_find_bin<SEL_BINS>(hist, k, warp_tot, &tot_a, &s_bin, &s_above);
        const uint32_t beta = (uint32_t)s_bin;
        const int above = s_above;              // keys of higher buckets: all selected
        const int nbeta = (int)hist[beta];
        const bool staged = nbeta <= SEL_CAP;
        const int want = k - above;             // keys still to take from bucket beta (>= 1)
        // higher buckets to the selection, bucket beta to the stage (appends in any order)
        for (int base = 0; base < F; base += SEL_THREADS) {
            const int j = base + threadIdx.x;
            uint32_t u = 0;
            bool gt = false, eq = false;
            if (j < F) {
                u = key_at(j);
                gt = (u >> 20) > beta;
                eq = staged && (u >> 20) == beta;
            }
            const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
            int pg = 0, pe = 0;
            if (lane == 0) {
                if (bg) pg = atomicAdd(&s_ngt, __popc(bg));
                if (be) pe = atomicAdd(&s_nst, __popc(be));
            }
            pg = __shfl_sync(0xffffffffu, pg, 0);
            pe = __shfl_sync(0xffffffffu, pe, 0);
            if (gt) sel[pg + __popc(bg & lt)] = key64(u, j);
            if (eq) stage[pe + __popc(be & lt)] = key64(u, j);
        }
        __syncthreads();
        if (staged) {
            int np = 64;
            while (np < nbeta) np <<= 1;
            for (int t = nbeta + threadIdx.x; t < np; t += SEL_THREADS) stage[t] = 0ull;
            block_sort_desc_u64(stage, np);
            for (int t = threadIdx.x; t < want; t += SEL_THREADS) sel[above + t] = stage[t];
        } else {
            // a crowded bucket: three radix passes (8/8/4 bits) for the k-th key K, then the
            // bucket's keys above K and the first keys equal to K in slot order
            uint32_t prefix = beta << 20, pmask = 0xFFF00000u;
            int remaining = want;
#pragma unroll 1
            for (int pass = 0; pass < 3; pass++) {
                const int shift = pass < 2 ? 12 - 8 * pass : 0;
                const uint32_t bins = pass < 2 ? 255u : 15u;
                for (int t = threadIdx.x; t < 1024; t += SEL_THREADS) hist[t] = 0;
                __syncthreads();
                for (int j = threadIdx.x; j < F; j += SEL_THREADS) {
                    const uint32_t u = key_at(j);
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
                    u = key_at(j);
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
    block_sort_desc_u64(sel, kpow2);
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
// Lane l holds key elements l E .. l E + E - 1 (E = d_I / 32).  Heads go in groups of 16: the
// lanes' query parts of the 16 heads are loaded first (one coalesced row per head), then the 16
// partial dot products are summed over the warp by a reduce-scatter (16 shuffles: after it, lanes
// l and l ^ 1 hold the whole dot product of one head of the group).
template <int E, bool F32>
__global__ void __launch_bounds__(256) k_li_window(const void *__restrict__ q, const float *__restrict__ w, int TQ,
                                                   const void *__restrict__ winK, const float *__restrict__ winsc,
                                                   const int32_t *__restrict__ win_count, int B, int W, int n_h,
                                                   float *__restrict__ tail)
{
    constexpr int D = 32 * E;
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
    auto ld = [&](const void *base, int64_t at) {
        return F32 ? __ldg((const float *)base + at) : bf16_bits_to_float(__ldg((const unsigned short *)base + at));
    };
    float kv[E];
#pragma unroll
    for (int e = 0; e < E; e++) kv[e] = ld(winK, ((int64_t)b * W + j) * D + lane * E + e);
    const int64_t qb = (int64_t)b * TQ * n_h * D + (int64_t)lane * E;  // query slot 0
    const float *wr = w + (int64_t)b * TQ * n_h;
    // the head of the group whose dot product this lane holds after the reduce-scatter
    const int hl = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    float y = 0.f;
    for (int h0 = 0; h0 < n_h; h0 += 16) {
        float qv[16][E];
#pragma unroll
        for (int g = 0; g < 16; g++)
#pragma unroll
            for (int e = 0; e < E; e++) qv[g][e] = h0 + g < n_h ? ld(q, qb + (int64_t)(h0 + g) * D + e) : 0.f;
        float v[16];
#pragma unroll
        for (int g = 0; g < 16; g++) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < E; e++) d = fmaf(qv[g][e], kv[e], d);
            v[g] = d;
        }
        // reduce-scatter: 16 -> 8 -> 4 -> 2 -> 1 values per lane, then the lane pair
#pragma unroll
        for (int half = 8, m = 16; half >= 1; half >>= 1, m >>= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < half; i++) {
                const float send = upper ? v[i] : v[half + i];
                const float keep = upper ? v[half + i] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        const float dot = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
        const int h = h0 + hl;
        float c = ((lane & 1) == 0 && h < n_h) ? __ldg(wr + h) * fmaxf(sc * dot, 0.f) : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        y += c;
    }
    if (lane == 0) tail[(int64_t)b * W + j] = y;
}

}  // namespace lsa
