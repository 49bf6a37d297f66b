// Top-k of one decode step (three launches).  A step has one query per sequence; its candidates
// are the F fetched slots, then the window entries as candidates F .. F + n - 1 (reported as
// entries S_b + j).  A candidate's 64-bit key is (order-preserving score key << 32) | ~slot: larger
// score first, then smaller slot, and no two keys are equal.
//   k_step_front   one grid, CTA roles that do not wait for one another: the scorer's work items
//                  and their table; the cleared score histograms; per sequence the step's query
//                  and weights copied to the scorer's dense layout and the window entries' scores
//   k_li_tc<1>     (li_tc.cuh) the fetched entries' scores, and their histogram: the top 14 bits
//                  of the score key (HIST_BINS bins, li_tc.cuh) counted per sequence
//   k_ss_select    one CTA per query: the histogram (plus the window entries) gives the bin beta of
//                  the k-th largest key; one pass over the candidates scatters the keys of higher
//                  bins into their bins' segments of the selection and stages bin beta's keys; the
//                  stage sorted gives its largest keys, and when no bin above beta is large a key's
//                  output position is its segment's start plus the keys of its segment above it
//                  (otherwise the k keys are sorted).  A bin beta of more than SCAP keys is
//                  resolved by four radix passes over its keys and an ordered pass (the first keys
//                  equal to the k-th in slot order).  A query with at most k candidates takes them
//                  all.  The output is as the batched select writes it.
#pragma once
#include "select_common.cuh"
#include "li_tc.cuh"
#include "topk.cuh"

namespace lsa {

namespace stepsel {

constexpr int HB = li::HIST_BINS;  // histogram bins per query
constexpr int SEL_TH = SEL_THREADS;
constexpr int SCAP = 4096;         // staged keys sorted in shared memory
constexpr int RANK_SEG = 64;       // largest bin above beta whose keys are ranked by counting

__device__ __forceinline__ uint32_t bin_of(uint32_t u) { return u >> li::HIST_SHIFT; }

struct Query {
    const float *row;   // fetched scores (query slot 0 of the Y layout)
    const float *trow;  // window-entry scores
    int F0, nt;
    int64_t off, S;
};

__device__ __forceinline__ Query query(int b, const float *Y, const int32_t *count, const int64_t *offs,
                                       const float *tail, const int32_t *tail_count, int W)
{
    Query q;
    q.off = offs[b];
    q.S = offs[b + 1] - q.off;
    int F = count[b];
    q.F0 = F < 0 ? 0 : (F > q.S ? (int)q.S : F);
    int nt = tail_count ? tail_count[b] : 0;
    q.nt = nt < 0 ? 0 : (nt > W ? W : nt);
    q.row = Y + q.off;
    q.trow = tail + (int64_t)b * (W > 0 ? W : 0);
    return q;
}

__device__ __forceinline__ uint32_t key_of(const Query &q, int j)
{
    return float_to_ordered(j < q.F0 ? q.row[j] : q.trow[j - q.F0]);
}

// The step's first launch: three CTA roles in one grid, none waiting on another.
//   CTA 0           the prefix over the sequences of the scorer's work items (ceil(ceil(F_b/128)/ch)
//                   per sequence, claim counter zeroed) and the item table, a warp per sequence
//   nclear CTAs     zero the histograms, 4096 words each
//   B CTAs          one per sequence: its query and weights copied to the scorer's dense layout
//                   (and to shared memory) and the window entries' scores (a warp an entry)
struct FrontParams {
    const int32_t *count;      // [B] fetched entries
    const int64_t *offs;       // [B+1]
    const int32_t *win_count;  // [B] window entries, or null (no window entries)
    int W, B, n_h, d_I, dt;
    int ch;                    // key tiles per scorer work item
    int *item_start;           // [B+1]
    int *item_counter;
    ItemInfo *items;           // the scorer's item table
    int *ghist;                // [B][HB]
    const void *qs;            // the step's queries [B][n_h][d_I], batch stride q_bstride elements
    int64_t q_bstride;
    const float *ws;           // the step's weights [B][n_h], batch stride w_bstride
    int64_t w_bstride;
    void *q_out;               // dense copy [B][n_h][d_I]
    float *w_out;              // [B][n_h]
    const void *winK;          // [B][W][d_I] window keys (hot-key type)
    const float *winsc;        // [B][W] or null
    float *tail;               // [B][W] window-entry scores
    int nclear;                // CTAs of the second role
};

constexpr int FRONT_TH = 512;

// HB is a multiple of 4096, so every clearing CTA takes a whole block of 4096 words
__host__ __device__ inline int front_clear_ctas(int B) { return (int)((int64_t)B * HB / 4096); }
// dynamic shared memory of k_step_front: one sequence's query and weights
__host__ __device__ inline size_t front_smem(int n_h, int d_I, int dt)
{
    return (size_t)n_h * d_I * (dt == DT_F32 ? 4 : 2) + sizeof(float) * (size_t)n_h;
}

template <int E, bool F32>
__global__ void __launch_bounds__(FRONT_TH) k_step_front(FrontParams p)
{
    extern __shared__ float4 front_sm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = FRONT_TH / 32;
    const int role_cta = (int)blockIdx.x - 1;
    if (role_cta >= 0 && role_cta < p.nclear) {
        int4 *dst = (int4 *)(p.ghist + (int64_t)role_cta * 4096);
        for (int i = threadIdx.x; i < 1024; i += FRONT_TH) dst[i] = make_int4(0, 0, 0, 0);
        return;
    }
    if (role_cta >= p.nclear) {
        // ---- one sequence: dense query copy, window entries
        const int b = role_cta - p.nclear;
        const int nq = p.n_h * p.d_I;
        void *sq = (void *)front_sm;
        float *sw = (float *)((uint8_t *)front_sm + (size_t)nq * (F32 ? 4 : 2));
        constexpr int es = F32 ? 4 : 2;
        const uint8_t *src = (const uint8_t *)p.qs + (int64_t)b * p.q_bstride * es;
        uint8_t *dst = (uint8_t *)p.q_out + (int64_t)b * nq * es;  // 16-byte aligned: nq * es is a multiple of 64
        const int nv = nq * es / 16;
        if (((uintptr_t)src & 15) == 0) {
            for (int t = threadIdx.x; t < nv; t += FRONT_TH) {
                const uint4 v = __ldg((const uint4 *)src + t);
                ((uint4 *)sq)[t] = v;
                ((uint4 *)dst)[t] = v;
            }
        } else {  // a query row off 16-byte alignment: element by element, eight loads in flight
            for (int t0 = threadIdx.x; t0 < nq; t0 += 8 * FRONT_TH) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    const int t = t0 + u * FRONT_TH;
                    v[u] = 0.f;
                    if (t < nq) v[u] = F32 ? __ldg((const float *)src + t)
                                          : __uint_as_float((uint32_t)__ldg((const uint16_t *)src + t));
                }
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    const int t = t0 + u * FRONT_TH;
                    if (t >= nq) continue;
                    if (F32) {
                        ((float *)sq)[t] = v[u];
                        ((float *)dst)[t] = v[u];
                    } else {
                        const uint16_t h = (uint16_t)__float_as_uint(v[u]);
                        ((uint16_t *)sq)[t] = h;
                        ((uint16_t *)dst)[t] = h;
                    }
                }
            }
        }
        for (int t = threadIdx.x; t < p.n_h; t += FRONT_TH) {
            const float v = p.ws[(int64_t)b * p.w_bstride + t];
            sw[t] = v;
            p.w_out[(int64_t)b * p.n_h + t] = v;
        }
        __syncthreads();
        int n = p.win_count ? p.win_count[b] : 0;
        if (n < 0 || n > p.W) {
            if (threadIdx.x == 0) flag(ERRF_COUNT);
            n = n < 0 ? 0 : p.W;
        }
        for (int j = warp; j < n; j += NW) {
            const float y = li_window_entry<E, F32>(b, j, lane, sq, sw, p.winK, p.winsc, p.W, p.n_h);
            if (lane == 0) p.tail[(int64_t)b * p.W + j] = y;
        }
        return;
    }
    // ---- CTA 0: the scorer's items
    __shared__ int wt_items[NW];
    __shared__ int carry_items;
    if (threadIdx.x == 0) {
        carry_items = 0;
        p.item_start[0] = 0;
        *p.item_counter = 0;
    }
    __syncthreads();
    for (int base = 0; base < p.B; base += FRONT_TH) {
        const int b = base + threadIdx.x;
        int ni = 0;
        if (b < p.B) {
            const int64_t S = p.offs[b + 1] - p.offs[b];
            int F = p.count[b];
            if (F < 0 || F > S) flag(ERRF_COUNT);
            F = F < 0 ? 0 : (F > S ? (int)S : F);
            const int tiles = (F + TILE - 1) / TILE;
            ni = (tiles + p.ch - 1) / p.ch;
        }
        const int ii = warp_incl_scan(ni);
        if (lane == 31) wt_items[warp] = ii;
        __syncthreads();
        if (warp == 0) {
            const int vi = lane < NW ? wt_items[lane] : 0;
            const int si = warp_incl_scan(vi) - vi;
            if (lane < NW) wt_items[lane] = si;
        }
        __syncthreads();
        const int pi = carry_items + wt_items[warp] + ii;
        if (b < p.B) p.item_start[b + 1] = pi;
        __syncthreads();
        if (threadIdx.x == FRONT_TH - 1) carry_items = pi;
        __syncthreads();
    }
    // the item table, a warp per sequence (item_start was written by this block: visible after the
    // barrier)
    for (int b = warp; b < p.B; b += NW) {
        const int64_t off = p.offs[b], S = p.offs[b + 1] - off;
        int F = p.count[b];
        F = F < 0 ? 0 : (F > S ? (int)S : F);
        li::write_items(p.items, p.item_start[b], b, F, (int)S, off, 1, p.ch, lane);
    }
}

// The histogram of the fetched entries' scores, for a scorer that does not count it (the SIMT
// scorer): grid (x, B), the x CTAs of a sequence striding over its fetched slots.
__global__ void __launch_bounds__(256) k_step_hist(const float *__restrict__ Y, const int32_t *__restrict__ count,
                                                   const int64_t *__restrict__ offs, int *__restrict__ ghist)
{
    const int b = blockIdx.y;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    int *h = ghist + (int64_t)b * HB;
    for (int j = blockIdx.x * 256 + threadIdx.x; j < F; j += gridDim.x * 256)
        atomicAdd(h + bin_of(float_to_ordered(Y[off + j])), 1);
}

// Dynamic shared memory of k_ss_select: kpow2 selection keys, SCAP staged keys, HB bin counters.
__host__ __device__ inline size_t select_smem(int kpow2)
{
    return sizeof(unsigned long long) * ((size_t)kpow2 + SCAP) + sizeof(int) * (size_t)HB;
}

__global__ void __launch_bounds__(SEL_TH, 1) k_ss_select(const float *__restrict__ Y, const int32_t *__restrict__ count,
                                                         const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                         const int32_t *__restrict__ tail_count, int W,
                                                         const int *__restrict__ ghist, const int32_t *__restrict__ idx,
                                                         int k, int kpow2, int32_t *__restrict__ topk_idx,
                                                         float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sk[];  // [kpow2] selection, [SCAP] stage, then HB ints
    unsigned long long *stage = sk + kpow2;
    int *hs = (int *)(stage + SCAP);
    __shared__ int warp_tot[32];
    __shared__ int tot_a, tot_b, s_bin, s_above, s_nst, s_maxseg;
    const int b = blockIdx.x;
    const Query q = query(b, Y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    auto key64 = [](uint32_t u, int j) { return ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j); };
    auto emit = [&](int r, unsigned long long v) {
        const int64_t o = (int64_t)b * k + r;
        const int j = (int)~(uint32_t)(v & 0xffffffffull);  // candidate slot
        topk_idx[o] = (j >= 0 && j < q.F0) ? __ldg(idx + q.off + j)
                                           : ((j >= q.F0 && j < nc) ? (int32_t)(q.S + (j - q.F0)) : -1);
        if (topk_score) topk_score[o] = ordered_to_float((uint32_t)(v >> 32));
    };
    for (int t = threadIdx.x; t < kpow2; t += SEL_TH) sk[t] = 0ull;
    if (nc <= k) {
        __syncthreads();
        for (int j = threadIdx.x; j < nc; j += SEL_TH) sk[j] = key64(key_of(q, j), j);
    } else {
        // the histogram: the fetched entries' (from the scorer) and the window entries'
        const int4 *g4 = (const int4 *)(ghist + (int64_t)b * HB);
        for (int t = threadIdx.x; t < HB / 4; t += SEL_TH) ((int4 *)hs)[t] = __ldg(g4 + t);
        if (threadIdx.x == 0) {
            s_nst = 0;
            s_maxseg = 0;
        }
        __syncthreads();
        for (int j = q.F0 + threadIdx.x; j < nc; j += SEL_TH) atomicAdd(&hs[bin_of(key_of(q, j))], 1);
        __syncthreads();
        const int my_above = sel_find_bin<HB>((const unsigned int *)hs, k, warp_tot, &tot_a, &s_bin, &s_above);
        const uint32_t beta = (uint32_t)s_bin;
        const int above = s_above;              // keys of higher bins: all selected
        const int nbeta = hs[beta];
        const bool staged = nbeta <= SCAP;
        const int want = k - above;             // keys still to take from bin beta (>= 1)
        __syncthreads();                        // every thread has read hs[beta] before the bins change
        {
            // every bin above beta becomes the start of its segment of the selection
            constexpr int PER = HB / SEL_TH;
            const int hi = HB - PER * (int)threadIdx.x;
            int run = my_above, mx = 0;
#pragma unroll
            for (int i = 1; i <= PER; i++) {
                const int bin = hi - i;
                if (bin > (int)beta) {
                    const int c = hs[bin];
                    hs[bin] = run;
                    run += c;
                    mx = max(mx, c);
                }
            }
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) atomicMax(&s_maxseg, mx);
        }
        __syncthreads();
        // higher bins scattered to their segments, bin beta to the stage (any order)
        for (int base = 0; base < nc; base += SEL_TH) {
            const int j = base + threadIdx.x;
            uint32_t u = 0;
            bool eq = false;
            if (j < nc) {
                u = key_of(q, j);
                const uint32_t bn = bin_of(u);
                if (bn > beta) sk[atomicAdd(&hs[bn], 1)] = key64(u, j);
                eq = staged && bn == beta;
            }
            const unsigned be = __ballot_sync(0xffffffffu, eq);
            int pe = 0;
            if (lane == 0 && be) pe = atomicAdd(&s_nst, __popc(be));
            pe = __shfl_sync(0xffffffffu, pe, 0);
            if (eq) stage[pe + __popc(be & lt)] = key64(u, j);
        }
        __syncthreads();
        if (staged) {
            int np = 64;
            while (np < nbeta) np <<= 1;
            for (int t = nbeta + threadIdx.x; t < np; t += SEL_TH) stage[t] = 0ull;
            block_sort_desc_u64(stage, np);
            if (s_maxseg <= RANK_SEG) {
                // output position of a selected key = its segment's start + the keys of its segment
                // above it; the stage's largest keys follow in order
                for (int t = threadIdx.x; t < above; t += SEL_TH) {
                    const unsigned long long v = sk[t];
                    const uint32_t bn = bin_of((uint32_t)(v >> 32));
                    const int lo = bn + 1 < (uint32_t)HB ? hs[bn + 1] : 0, hi = hs[bn];
                    int r = lo;
                    for (int i = lo; i < hi; i++) r += sk[i] > v;
                    emit(r, v);
                }
                for (int t = threadIdx.x; t < want; t += SEL_TH) emit(above + t, stage[t]);
                return;
            }
            for (int t = threadIdx.x; t < want; t += SEL_TH) sk[above + t] = stage[t];
        } else {
            // a crowded bin: four radix passes of 8 bits over its keys give the k-th key K; then the
            // bin's keys above K and the first keys equal to K in slot order
            unsigned int *h256 = (unsigned int *)stage;  // the stage is free here
            uint32_t prefix = 0u, pmask = 0u;
            int remaining = want;
#pragma unroll 1
            for (int pass = 0; pass < 4; pass++) {
                const int sh = 24 - 8 * pass;
                for (int t = threadIdx.x; t < 1024; t += SEL_TH) h256[t] = 0;
                __syncthreads();
                for (int j = threadIdx.x; j < nc; j += SEL_TH) {
                    const uint32_t u = key_of(q, j);
                    if ((u & pmask) == prefix && bin_of(u) == beta) atomicAdd(&h256[(u >> sh) & 255u], 1u);
                }
                __syncthreads();
                sel_find_bin<1024>(h256, remaining, warp_tot, &tot_a, &s_bin, &s_above);
                prefix |= (uint32_t)s_bin << sh;
                remaining -= s_above;
                pmask |= 255u << sh;
                __syncthreads();
            }
            int cg = 0, ce = 0;
            for (int base = 0; base < nc; base += SEL_TH) {
                const int j = base + threadIdx.x;
                uint32_t u = 0;
                int gt = 0, eq = 0;
                if (j < nc) {
                    u = key_of(q, j);
                    gt = bin_of(u) == beta && u > prefix;
                    eq = u == prefix;
                }
                const int pg = block_excl_scan(gt, warp_tot, &tot_a) + cg;
                const int pe = block_excl_scan(eq, warp_tot, &tot_b) + ce;
                if (gt) sk[above + pg] = key64(u, j);
                if (eq && pe < remaining) sk[k - remaining + pe] = key64(u, j);
                cg += tot_a;
                ce += tot_b;
                __syncthreads();
            }
        }
    }
    block_sort_desc_u64(sk, kpow2);
    const int nsel = nc < k ? nc : k;
    for (int r = threadIdx.x; r < k; r += SEL_TH) {
        if (r < nsel) {
            emit(r, sk[r]);
        } else {
            const int64_t o = (int64_t)b * k + r;
            topk_idx[o] = -1;
            if (topk_score) topk_score[o] = -INFINITY;
        }
    }
}

}  // namespace stepsel

}  // namespace lsa
