// Stage 5: native Lightning-Indexer score over the fetched entries and per-query Top-k
// (blog review "FlashMemory-DeepSeek-V4", sections 2.2 and 3.2).
//
// Scores of sequence b, query i, fetched slot j live at Y[tau*off_b + i*S_b + j] (fp32).
// Selection: per query, the k-th largest score is found on order-preserving keys held in shared
// memory (a histogram of 4096 buckets spread over the query's own key range, then the bucket's
// keys); the survivors are sorted by (score desc, entry asc) with a bitonic sort in shared memory
// (k_topk_select).
#pragma once
#include "select_common.cuh"

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

// The k-th largest key of a query is found from a histogram of the order-preserving score keys
// over SEL_NB buckets of the query's key range (its bucket beta) and then inside the bucket; a
// candidate's 64-bit key (score key << 32) | ~slot orders by score and then by smaller slot, and
// no two are equal.
constexpr int SEL_BINS = SEL_NB;
constexpr int SEL_CAP = 4096;      // bucket keys sorted in shared memory
constexpr int SEL_RANK_SEG = 64;   // largest bucket above beta whose keys are ranked by counting

// The bin holding the `want`-th largest key of a histogram of NB bins (thread t owns NB / SEL_THREADS
// consecutive bins, highest first): *bin_out, and *above_out = keys in higher bins.  want >= 1 and
// at most the histogram's total.  Returns the keys in bins above this thread's.  Ends with a barrier.
template <int NB>
__device__ __forceinline__ int sel_find_bin(const unsigned int *hist, int want, int *warp_tot, int *tot, int *bin_out,
                                            int *above_out)
{
    constexpr int PER = NB / SEL_THREADS;
    const int hi = NB - PER * (int)threadIdx.x;  // bins [hi - PER, hi)
    int cnt = 0;
#pragma unroll
    for (int q = 1; q <= PER; q++) cnt += (int)hist[hi - q];
    const int above0 = block_excl_scan(cnt, warp_tot, tot);
    int above = above0;
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
    return above0;
}

// Shared memory of k_topk_select for kpow2 (dynamic part): the selection and the stage.
__host__ __device__ inline size_t topk_select_smem(int kpow2)
{
    return sizeof(unsigned long long) * ((size_t)kpow2 + SEL_CAP);
}

// A query's scores in 16-byte vectors from their first 16-byte boundary; the at most three scores
// before it and the at most three after the last whole vector belong to threads 0..5 (lone()).
struct ScoreRow {
    const float *row;
    const float4 *vec;
    int F, head, nvec, tail0;
    __device__ ScoreRow(const float *r, int f) : row(r), F(f)
    {
        head = min((int)((4 - (((uintptr_t)r >> 2) & 3)) & 3), f);
        nvec = (f - head) >> 2;
        tail0 = head + 4 * nvec;
        vec = (const float4 *)(r + head);
    }
    __device__ int lone() const
    {
        const int t = (int)threadIdx.x;
        return t < head ? t : (t < head + (F - tail0) ? tail0 + (t - head) : -1);
    }
};

// One block per (sequence, query).  kpow2 = next power of two >= max(k, 64).  Dynamic shared memory:
// kpow2 selection keys and SEL_CAP staged keys; the query's scores are read from global memory at
// every pass (as 16-byte vectors, four in flight per thread; after the first pass they come from
// L2), so two blocks fit on an SM.  With more than k candidates: the range of the query's scores,
// then a histogram over 4096 buckets of that range gives the bucket beta of the k-th largest key.
// Each bucket above beta gets a segment of the selection (higher buckets first) and its keys are
// scattered into it; the bucket's keys go to the stage (any order: the keys carry their slots), and
// the stage sorted by key gives the bucket's largest keys.  When no bucket above beta holds more
// than SEL_RANK_SEG keys, a key's output position is its segment's start plus the keys of its
// segment above it (no sort of the selection); otherwise the k keys are sorted.  A bucket beta of
// more than SEL_CAP keys is resolved by four radix passes over its keys and an ordered pass (the
// first keys equal to the k-th in slot order).  The output is ordered by (score desc, slot asc).
__global__ void __launch_bounds__(SEL_THREADS, 2) k_topk_select(const float *__restrict__ Y,
                                                                const int32_t *__restrict__ idx,
                                                                const int32_t *__restrict__ count,
                                                                const int64_t *__restrict__ offs, int tau, int k,
                                                                int kpow2, int32_t *__restrict__ topk_idx,
                                                                float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sel[];  // [kpow2] selection, [SEL_CAP] stage
    unsigned long long *stage = sel + kpow2;
    __shared__ unsigned int hist[SEL_BINS];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, tot_b, s_bin, s_above, s_ngt, s_nst, s_maxseg;
    __shared__ float s_fmin[32], s_fmax[32];

    const int b = blockIdx.x / tau, i = blockIdx.x % tau;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    const float *row = Y + (int64_t)tau * off + (int64_t)i * S;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = (1u << lane) - 1u;
    auto key64 = [](uint32_t u, int j) { return ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j); };
    auto key_at = [&](int j) -> uint32_t { return float_to_ordered(__ldg(row + j)); };
    const ScoreRow sr(row, F);
    const int lone = sr.lone();
    const float4 NONE = make_float4(NAN, NAN, NAN, NAN);
    // fn(y, j) for every score of the query, four vector loads in flight per thread
    auto each = [&](auto fn) {
        for (int v0 = 0; v0 < sr.nvec; v0 += 4 * SEL_THREADS) {
            float4 x[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int v = v0 + q * SEL_THREADS + (int)threadIdx.x;
                x[q] = v < sr.nvec ? __ldg(sr.vec + v) : NONE;
            }
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int v = v0 + q * SEL_THREADS + (int)threadIdx.x;
                if (v < sr.nvec) {
                    const int j = sr.head + 4 * v;
                    fn(x[q].x, j);
                    fn(x[q].y, j + 1);
                    fn(x[q].z, j + 2);
                    fn(x[q].w, j + 3);
                }
            }
        }
        if (lone >= 0) fn(__ldg(row + lone), lone);
    };

    for (int t = threadIdx.x; t < kpow2; t += SEL_THREADS) sel[t] = 0ull;
    if (F <= k) {
        __syncthreads();
        for (int j = threadIdx.x; j < F; j += SEL_THREADS) sel[j] = key64(key_at(j), j);
    } else {
        // the range of the query's scores (NaN aside), then the histogram
        float fmn = INFINITY, fmx = -INFINITY;
        each([&](float y, int) {
            fmn = fminf(fmn, y);
            fmx = fmaxf(fmx, y);
        });
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            fmn = fminf(fmn, __shfl_xor_sync(0xffffffffu, fmn, o));
            fmx = fmaxf(fmx, __shfl_xor_sync(0xffffffffu, fmx, o));
        }
        if (lane == 0) {
            s_fmin[warp] = fmn;
            s_fmax[warp] = fmx;
        }
        for (int t = threadIdx.x; t < SEL_BINS; t += SEL_THREADS) hist[t] = 0;
        if (threadIdx.x == 0) {
            s_ngt = s_nst = 0;
            s_maxseg = 0;
        }
        __syncthreads();
        fmn = INFINITY;
        fmx = -INFINITY;
        for (int w = 0; w < SEL_THREADS / 32; w++) {
            fmn = fminf(fmn, s_fmin[w]);
            fmx = fmaxf(fmx, s_fmax[w]);
        }
        const SelRange rg = sel_range_f(fmn, fmx);
        each([&](float y, int) { atomicAdd(&hist[sel_bucket_f(rg, y)], 1u); });
        __syncthreads();
        const int my_above = sel_find_bin<SEL_BINS>(hist, k, warp_tot, &tot_a, &s_bin, &s_above);
        const uint32_t beta = (uint32_t)s_bin;
        const int above = s_above;              // keys of higher buckets: all selected
        const int nbeta = (int)hist[beta];
        const bool staged = nbeta <= SEL_CAP;
        const int want = k - above;             // keys still to take from bucket beta (>= 1)
        {
            // every bucket above beta becomes the start of its segment of the selection (higher
            // buckets first); the largest such bucket decides how the selection is ordered
            constexpr int PER = SEL_BINS / SEL_THREADS;
            const int hi = SEL_BINS - PER * (int)threadIdx.x;
            int run = my_above, mx = 0;
#pragma unroll
            for (int q = 1; q <= PER; q++) {
                const int bin = hi - q;
                if (bin > (int)beta) {
                    const int c = (int)hist[bin];
                    hist[bin] = (unsigned int)run;
                    run += c;
                    mx = max(mx, c);
                }
            }
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) atomicMax(&s_maxseg, mx);
        }
        __syncthreads();
        // higher buckets scattered to their segments, bucket beta to the stage (any order); the
        // loop runs the same trips in every lane (the stage appends are warp-aggregated)
        auto scatter = [&](bool in, float y, int j) {
            const uint32_t bk = in ? sel_bucket_f(rg, y) : 0u;
            if (in && bk > beta) sel[atomicAdd(&hist[bk], 1u)] = key64(float_to_ordered(y), j);
            const bool eq = in && staged && bk == beta;
            const unsigned be = __ballot_sync(0xffffffffu, eq);
            if (be) {
                int pe = 0;
                if (lane == 0) pe = atomicAdd(&s_nst, __popc(be));
                pe = __shfl_sync(0xffffffffu, pe, 0);
                if (eq) stage[pe + __popc(be & lt)] = key64(float_to_ordered(y), j);
            }
        };
        for (int v0 = 0; v0 < sr.nvec; v0 += 2 * SEL_THREADS) {
            float4 x[2];
#pragma unroll
            for (int q = 0; q < 2; q++) {
                const int v = v0 + q * SEL_THREADS + (int)threadIdx.x;
                x[q] = v < sr.nvec ? __ldg(sr.vec + v) : NONE;
            }
#pragma unroll
            for (int q = 0; q < 2; q++) {
                const int v = v0 + q * SEL_THREADS + (int)threadIdx.x;
                const bool in = v < sr.nvec;
                const int j = sr.head + 4 * v;
                scatter(in, x[q].x, j);
                scatter(in, x[q].y, j + 1);
                scatter(in, x[q].z, j + 2);
                scatter(in, x[q].w, j + 3);
            }
        }
        scatter(lone >= 0, lone >= 0 ? __ldg(row + lone) : 0.f, lone);
        __syncthreads();
        const bool ranked = staged && s_maxseg <= SEL_RANK_SEG;
        if (staged) {
            int np = 64;
            while (np < nbeta) np <<= 1;
            for (int t = nbeta + threadIdx.x; t < np; t += SEL_THREADS) stage[t] = 0ull;
            block_sort_desc_u64(stage, np);
            if (ranked) {
                // output position of a selected key = its segment's start + the keys of the segment
                // above it; the stage's largest keys follow in order
                const int64_t o0 = ((int64_t)b * tau + i) * k;
                for (int t = threadIdx.x; t < above; t += SEL_THREADS) {
                    const unsigned long long v = sel[t];
                    const uint32_t bk = sel_bucket(rg, (uint32_t)(v >> 32));
                    const int lo = bk + 1 < (uint32_t)SEL_BINS ? (int)hist[bk + 1] : 0, hi = (int)hist[bk];
                    int r = lo;
                    for (int q = lo; q < hi; q++) r += sel[q] > v;
                    const int jj = (int)~(uint32_t)(v & 0xffffffffull);
                    topk_idx[o0 + r] = __ldg(idx + off + jj);
                    if (topk_score) topk_score[o0 + r] = ordered_to_float((uint32_t)(v >> 32));
                }
                for (int t = threadIdx.x; t < want; t += SEL_THREADS) {
                    const unsigned long long v = stage[t];
                    const int jj = (int)~(uint32_t)(v & 0xffffffffull);
                    topk_idx[o0 + above + t] = __ldg(idx + off + jj);
                    if (topk_score) topk_score[o0 + above + t] = ordered_to_float((uint32_t)(v >> 32));
                }
                return;
            }
            for (int t = threadIdx.x; t < want; t += SEL_THREADS) sel[above + t] = stage[t];
        } else {
            // a crowded bucket: four radix passes of 8 bits over the keys of bucket beta give the
            // k-th key K; then the bucket's keys above K and the first keys equal to K in slot order
            uint32_t prefix = 0u, pmask = 0u;
            int remaining = want;
#pragma unroll 1
            for (int pass = 0; pass < 4; pass++) {
                const int sh = 24 - 8 * pass;
                for (int t = threadIdx.x; t < 1024; t += SEL_THREADS) hist[t] = 0;
                __syncthreads();
                for (int j = threadIdx.x; j < F; j += SEL_THREADS) {
                    const uint32_t u = key_at(j);
                    if ((u & pmask) == prefix && sel_bucket(rg, u) == beta) atomicAdd(&hist[(u >> sh) & 255u], 1u);
                }
                __syncthreads();
                sel_find_bin<1024>(hist, remaining, warp_tot, &tot_a, &s_bin, &s_above);
                prefix |= (uint32_t)s_bin << sh;
                remaining -= s_above;
                pmask |= 255u << sh;
                __syncthreads();
            }
            int cg = 0, ce = 0;
            for (int base = 0; base < F; base += SEL_THREADS) {
                const int j = base + threadIdx.x;
                uint32_t u = 0;
                int gt = 0, eq = 0;
                if (j < F) {
                    u = key_at(j);
                    gt = sel_bucket(rg, u) == beta && u > prefix;
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
// Device part of one decode step's Top-k (the first launch of the step, k_step_front, runs it).

// Score of window entry j of sequence b (one warp): y = sum_h w_h ReLU(scale_j q_h . k_j) for the
// entries compressed during the window.  Keys [B][W][d_I] in the hot-key type, scales nullable;
// q [n_h][d_I] and w [n_h] are the sequence's query and weights (any memory space).  Lane l holds
// key elements l E .. l E + E - 1 (E = d_I / 32).  Heads go in groups of 16: the lanes' query
// parts of the 16 heads are loaded first (one coalesced row per head), then the 16 partial dot
// products are summed over the warp by a reduce-scatter (16 shuffles: after it, lanes l and l ^ 1
// hold the whole dot product of one head of the group).  Every lane returns y.
template <int E, bool F32>
__device__ __forceinline__ float li_window_entry(int b, int j, int lane, const void *q, const float *w,
                                                 const void *__restrict__ winK, const float *__restrict__ winsc,
                                                 int W, int n_h)
{
    constexpr int D = 32 * E;
    const float sc = winsc ? winsc[(int64_t)b * W + j] : 1.f;
    if (winsc && lane == 0 && !(sc >= 0.f)) flag(ERRF_SCALE);
    float kv[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int64_t at = ((int64_t)b * W + j) * D + lane * E + e;
        kv[e] = F32 ? __ldg((const float *)winK + at) : bf16_bits_to_float(__ldg((const unsigned short *)winK + at));
    }
    auto ldq = [&](int at) {
        return F32 ? ((const float *)q)[at] : bf16_bits_to_float(((const unsigned short *)q)[at]);
    };
    // the head of the group whose dot product this lane holds after the reduce-scatter
    const int hl = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    float y = 0.f;
    for (int h0 = 0; h0 < n_h; h0 += 16) {
        float qv[16][E];
#pragma unroll
        for (int g = 0; g < 16; g++)
#pragma unroll
            for (int e = 0; e < E; e++) qv[g][e] = h0 + g < n_h ? ldq((h0 + g) * D + lane * E + e) : 0.f;
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
        float c = ((lane & 1) == 0 && h < n_h) ? w[h] * fmaxf(sc * dot, 0.f) : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        y += c;
    }
    return y;
}

}  // namespace lsa
