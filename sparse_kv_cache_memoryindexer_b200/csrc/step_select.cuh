// Top-k select of one decode step, spread over many CTAs.  A step has one query per sequence, so
// the one-CTA-per-query select of the batched call would leave all but B SMs idle; here the
// candidates of a query (its F fetched slots, then its window entries as candidates F .. F + n - 1,
// reported as entries S_b + j) are cut into chunks of CH with one CTA per chunk.  A candidate's
// 64-bit key is (order-preserving score key << 32) | ~slot: larger score first, then smaller slot,
// and no two keys are equal.
//   k_step_front per query: candidates, chunk ranges (a prefix over the sequences), state; other
//                CTAs of the same launch clear the histograms, copy the step's queries for the
//                scorer and score the window entries
//   k_ss_hist12  per chunk: histogram of the top 12 bits of the score keys, added to the query's
//                histogram in global memory; the query's last chunk to finish picks the bucket
//                beta holding the k-th largest key (the keys above beta are all selected)
//   k_ss_write   per chunk: keys of higher buckets appended to the query's selection, keys of
//                bucket beta appended to the query's stage (order does not matter: the keys carry
//                their slots); the query's last chunk to finish then takes the `want` largest staged
//                keys (a sort in shared memory, or a radix select over the stage for a crowded
//                bucket), sorts the k keys (bitonic) and writes the output as the one-CTA select
//                writes it.
// A query with at most k candidates takes them all.  CTAs of one launch do not wait for one
// another: the per-query step after the histogram runs in whichever chunk CTA of the query finishes
// last (a counter per query, reset by that CTA), and kernel boundaries order the rest.
#pragma once
#include "select_common.cuh"
#include "li_tc.cuh"
#include "topk.cuh"

namespace lsa {

namespace stepsel {

constexpr int CH = 4096;   // candidates per chunk
constexpr int TH = 256;    // threads per chunk CTA
constexpr int SORT_TH = 1024;
constexpr int NB = SEL_NB; // buckets of the histogram (over the query's key range)
constexpr int SCAP = 8192; // staged keys a final CTA sorts in shared memory
constexpr int NS = 12;     // state words per query
constexpr int RANK_SEG = 64; // largest bucket above beta whose keys the final step ranks by counting

struct Query {
    const float *row;   // fetched scores (query slot 0 of the Y layout)
    const float *trow;  // window-entry scores
    int F0, nt;
    int64_t off, S;
};

__device__ __forceinline__ Query query(int b, const float *Y, int tau_y, const int32_t *count, const int64_t *offs,
                                       const float *tail, const int32_t *tail_count, int W)
{
    Query q;
    q.off = offs[b];
    q.S = offs[b + 1] - q.off;
    int F = count[b];
    q.F0 = F < 0 ? 0 : (F > q.S ? (int)q.S : F);
    int nt = tail_count ? tail_count[b] : 0;
    q.nt = nt < 0 ? 0 : (nt > W ? W : nt);
    q.row = Y + (int64_t)tau_y * q.off;
    q.trow = tail + (int64_t)b * (W > 0 ? W : 0);
    return q;
}

__device__ __forceinline__ uint32_t key_of(const Query &q, int j)
{
    return float_to_ordered(j < q.F0 ? q.row[j] : q.trow[j - q.F0]);
}

// state per query (NS words): [0] bucket beta, [1] keys wanted from bucket beta (0: the query takes
// every candidate), [2] keys of higher buckets, [3] candidates, [4] keys appended to the selection,
// [5] keys appended to the stage, [6] finish counter of the write step, [7] keys of the largest
// bucket above beta, [8] smallest and [9]
// largest score key of the query (the window entries' from the first launch, the fetched entries'
// added by the scorer).  ghist: [B][NB] bucket histograms, then the finish counters [B].
__device__ __forceinline__ SelRange query_range(const uint32_t *st) { return sel_range(st[8], st[9]); }

// The step's first launch: three CTA roles in one grid, none waiting on another.
//   CTA 0           two prefixes over the sequences: the scorer's work items (ceil(ceil(F_b/128)/ch)
//                   per sequence, claim counter zeroed) and the select's chunks; the select state
//   nclear CTAs     zero the bucket histograms and finish counters, 4096 words each
//   B CTAs          one per sequence: its query and weights copied to the scorer's dense layout
//                   (and to shared memory), the window entries' scores (a warp an entry) and the
//                   range of their keys
struct FrontParams {
    const int32_t *count;      // [B] fetched entries
    const int64_t *offs;       // [B+1]
    const int32_t *win_count;  // [B] window entries, or null (no window entries)
    int W, B, k, n_h, d_I, dt;
    int ch;                    // key tiles per scorer work item
    int *item_start;           // [B+1]
    int *item_counter;
    ItemInfo *items;           // the scorer's item table
    int *chunk_start;          // [B+1]
    int *chunk_query;          // [chunks] the query of each chunk
    uint32_t *state;           // [B][NS]
    int *ghist;                // [B][NB], then [B] finish counters
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

__host__ __device__ inline int front_clear_ctas(int B) { return (int)(((int64_t)B * (NB + 1) + 4095) / 4096); }
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
        const int64_t i0 = (int64_t)role_cta * 4096, n = (int64_t)p.B * (NB + 1);
        for (int64_t i = i0 + threadIdx.x; i < n && i < i0 + 4096; i += FRONT_TH) p.ghist[i] = 0;
        return;
    }
    if (role_cta >= p.nclear) {
        // ---- one sequence: dense query copy, window entries, their key range
        const int b = role_cta - p.nclear;
        __shared__ uint32_t s_min, s_max;
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
        if (threadIdx.x == 0) {
            s_min = 0xFFFFFFFFu;
            s_max = 0u;
        }
        __syncthreads();
        int n = p.win_count ? p.win_count[b] : 0;
        if (n < 0 || n > p.W) {
            if (threadIdx.x == 0) flag(ERRF_COUNT);
            n = n < 0 ? 0 : p.W;
        }
        uint32_t tmin = 0xFFFFFFFFu, tmax = 0u;
        for (int j = warp; j < n; j += NW) {
            const float y = li_window_entry<E, F32>(b, j, lane, sq, sw, p.winK, p.winsc, p.W, p.n_h);
            if (lane == 0) p.tail[(int64_t)b * p.W + j] = y;
            const uint32_t u = float_to_ordered(y);
            tmin = min(tmin, u);
            tmax = max(tmax, u);
        }
        if (lane == 0 && tmin <= tmax) {
            atomicMin(&s_min, tmin);
            atomicMax(&s_max, tmax);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            p.state[NS * b + 8] = s_min;
            p.state[NS * b + 9] = s_max;
        }
        return;
    }
    // ---- CTA 0: the two prefixes
    __shared__ int wt_items[NW], wt_chunks[NW];
    __shared__ int carry_items, carry_chunks;
    if (threadIdx.x == 0) {
        carry_items = 0;
        carry_chunks = 0;
        p.item_start[0] = 0;
        *p.item_counter = 0;
        p.chunk_start[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < p.B; base += FRONT_TH) {
        const int b = base + threadIdx.x;
        int ni = 0, nchunk = 0;
        if (b < p.B) {
            const int64_t S = p.offs[b + 1] - p.offs[b];
            int F = p.count[b];
            if (F < 0 || F > S) flag(ERRF_COUNT);
            F = F < 0 ? 0 : (F > S ? (int)S : F);
            int nt = p.win_count ? p.win_count[b] : 0;
            nt = nt < 0 ? 0 : (nt > p.W ? p.W : nt);
            const int tiles = (F + TILE - 1) / TILE;
            ni = (tiles + p.ch - 1) / p.ch;
            const int nc = F + nt;
            nchunk = nc > 0 ? (nc + CH - 1) / CH : 1;  // a query without candidates still writes its row
            uint32_t *st = p.state + NS * b;
            st[0] = 0u;
            st[1] = nc > p.k ? (uint32_t)p.k : 0u;
            st[2] = 0u;
            st[3] = (uint32_t)nc;
            st[4] = 0u;
            st[5] = 0u;
            st[6] = 0u;
            st[7] = 0u;
        }
        const int ii = warp_incl_scan(ni), ic = warp_incl_scan(nchunk);
        if (lane == 31) {
            wt_items[warp] = ii;
            wt_chunks[warp] = ic;
        }
        __syncthreads();
        if (warp == 0) {
            const int vi = lane < NW ? wt_items[lane] : 0, vc = lane < NW ? wt_chunks[lane] : 0;
            const int si = warp_incl_scan(vi) - vi, sc = warp_incl_scan(vc) - vc;
            if (lane < NW) {
                wt_items[lane] = si;
                wt_chunks[lane] = sc;
            }
        }
        __syncthreads();
        const int pi = carry_items + wt_items[warp] + ii, pc = carry_chunks + wt_chunks[warp] + ic;
        if (b < p.B) {
            p.item_start[b + 1] = pi;
            p.chunk_start[b + 1] = pc;
        }
        __syncthreads();
        if (threadIdx.x == FRONT_TH - 1) {
            carry_items = pi;
            carry_chunks = pc;
        }
        __syncthreads();
    }
    // the query of every chunk and the scorer's item table, a warp per sequence (chunk_start and
    // item_start were written by this block: visible after the barrier)
    for (int b = warp; b < p.B; b += NW) {
        for (int c = p.chunk_start[b] + lane; c < p.chunk_start[b + 1]; c += 32) p.chunk_query[c] = b;
        const int64_t off = p.offs[b], S = p.offs[b + 1] - off;
        int F = p.count[b];
        F = F < 0 ? 0 : (F > S ? (int)S : F);
        li::write_items(p.items, p.item_start[b], b, F, (int)S, off, 1, p.ch, lane);
    }
}

// Range of the fetched entries' score keys, added to the query's state words 8 and 9, for a scorer
// that does not report it (the SIMT scorer): one thread per candidate chunk slot.
__global__ void __launch_bounds__(TH) k_ss_range(const float *__restrict__ Y, int tau_y,
                                                 const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                 int B, const int *__restrict__ chunk_start, const int *__restrict__ chunk_query, uint32_t *state)
{
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = chunk_query[c];
    const int64_t off = offs[b], S = offs[b + 1] - off;
    int F = count[b];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    const float *row = Y + (int64_t)tau_y * off;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(F, j0 + CH);
    uint32_t tmin = 0xFFFFFFFFu, tmax = 0u;
    for (int j = j0 + threadIdx.x; j < j1; j += TH) {
        const uint32_t u = float_to_ordered(row[j]);
        tmin = min(tmin, u);
        tmax = max(tmax, u);
    }
    tmin = __reduce_min_sync(0xffffffffu, tmin);
    tmax = __reduce_max_sync(0xffffffffu, tmax);
    if ((threadIdx.x & 31) == 0 && tmin <= tmax) {
        atomicMin(state + NS * b + 8, tmin);
        atomicMax(state + NS * b + 9, tmax);
    }
}

// Called by every thread of the chunk CTA after its part of a per-query sum is in global memory:
// true in the CTA that finishes the query's chunks last (which then also resets the counter).
__device__ __forceinline__ bool last_chunk_of_query(int *done, int b, int nch)
{
    __shared__ int is_last;
    __threadfence();  // this CTA's global writes before its count
    __syncthreads();
    if (threadIdx.x == 0) {
        is_last = atomicAdd(done + b, 1) == nch - 1;
        if (is_last) done[b] = 0;  // nobody else counts on this query in this launch
    }
    __syncthreads();
    if (!is_last) return false;
    __threadfence();  // the other chunks' writes, counted before ours, are read after this
    return true;
}

// Block-wide exclusive scans of two counts (TH threads): positions and totals.
__device__ __forceinline__ void block_excl_scan2(int a, int b, int &pa, int &pb, int &ta, int &tb)
{
    __shared__ int wa[TH / 32], wb[TH / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ia = warp_incl_scan(a), ib = warp_incl_scan(b);
    if (lane == 31) {
        wa[warp] = ia;
        wb[warp] = ib;
    }
    __syncthreads();
    int ba = 0, bb = 0, sa = 0, sb = 0;
#pragma unroll
    for (int w = 0; w < TH / 32; w++) {
        ba += w < warp ? wa[w] : 0;
        bb += w < warp ? wb[w] : 0;
        sa += wa[w];
        sb += wb[w];
    }
    pa = ba + ia - a;
    pb = bb + ib - b;
    ta = sa;
    tb = sb;
    __syncthreads();  // wa, wb free for the next call
}

__global__ void __launch_bounds__(TH) k_ss_hist12(const float *__restrict__ Y, int tau_y,
                                                  const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                  const float *__restrict__ tail, const int32_t *__restrict__ tail_count,
                                                  int W, int B, const int *__restrict__ chunk_start, const int *__restrict__ chunk_query, uint32_t *state,
                                                  int *ghist)
{
    __shared__ int hist[NB];
    __shared__ int s_beta, s_above;
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = chunk_query[c];
    uint32_t *st = state + NS * b;
    const int want = (int)st[1];
    if (want == 0) return;  // takes all its candidates (the same for every chunk of b)
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    for (int t = threadIdx.x; t < NB; t += TH) hist[t] = 0;
    __syncthreads();
    const SelRange rg = query_range(st);
    for (int j = j0 + threadIdx.x; j < j1; j += TH) atomicAdd(&hist[sel_bucket(rg, key_of(q, j))], 1);
    __syncthreads();
    int *gh = ghist + (int64_t)b * NB;
    for (int t = threadIdx.x; t < NB; t += TH)
        if (hist[t]) atomicAdd(gh + t, hist[t]);
    int *done = ghist + (int64_t)B * NB;
    if (!last_chunk_of_query(done, b, chunk_start[b + 1] - chunk_start[b])) return;
    // the bucket of the want-th largest key: thread t owns buckets NB - 16 (t + 1) .. NB - 16 t - 1
    constexpr int PER = NB / TH;
    __shared__ int s_maxseg;
    if (threadIdx.x == 0) s_maxseg = 0;
    const int hi = NB - PER * (int)threadIdx.x;
    int h[PER], cnt = 0;
#pragma unroll
    for (int i = 1; i <= PER; i++) {
        h[i - 1] = __ldcg(gh + hi - i);
        cnt += h[i - 1];
    }
    int above0, unused_p, total, unused_t;
    block_excl_scan2(cnt, 0, above0, unused_p, total, unused_t);
    int above = above0;
    if (above < want && above + cnt >= want) {
        for (int i = 1; i <= PER; i++) {
            if (above + h[i - 1] >= want) {
                s_beta = hi - i;
                s_above = above;
                break;
            }
            above += h[i - 1];
        }
    }
    __syncthreads();
    // every bucket above beta becomes the start of its segment of the selection (higher buckets
    // first); the largest such bucket decides how the final step orders the selection
    int run = above0, mx = 0;
#pragma unroll
    for (int i = 1; i <= PER; i++) {
        if (hi - i > s_beta) {
            gh[hi - i] = run;
            run += h[i - 1];
            mx = max(mx, h[i - 1]);
        }
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    if ((threadIdx.x & 31) == 0) atomicMax(&s_maxseg, mx);
    __syncthreads();
    if (threadIdx.x == 0) {
        st[0] = (uint32_t)s_beta;
        st[2] = (uint32_t)s_above;
        st[1] = (uint32_t)(want - s_above);
        st[7] = (uint32_t)s_maxseg;
    }
}

// Per query, by the whole block: the selection's keys of higher buckets plus the want largest keys
// of bucket beta, sorted by key descending (score descending, slot ascending), then the output.
// sk: kpow2 + SCAP keys of shared memory.  The selection and the stage were written by other CTAs
// of the same launch: they are read through L2.
__device__ __forceinline__ void final_of_query(int b, unsigned long long *sk, const unsigned long long *sel, int kcap,
                                               const unsigned long long *stage, const uint32_t *state,
                                               const int *gh, int W,
                                               const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                               const int64_t *__restrict__ offs, int k, int kpow2,
                                               int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    unsigned long long *ss = sk + kpow2;
    __shared__ int hist[256];
    __shared__ int s_dig, s_above, s_n;
    const int nth = blockDim.x;
    const uint32_t *st = state + NS * b;
    const int nc = (int)__ldcg(st + 3);
    const int want = (int)__ldcg(st + 1);
    const int above = (int)__ldcg(st + 2);
    const int nsel = nc < k ? nc : k;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    int F0 = count[b];
    F0 = F0 < 0 ? 0 : (F0 > S ? (int)S : F0);
    const unsigned long long *mine = sel + (int64_t)b * kcap;
    const int nfirst = want == 0 ? nsel : above;  // keys already in the selection
    for (int t = threadIdx.x; t < kpow2; t += nth) sk[t] = t < nfirst ? __ldcg(mine + t) : 0ull;
    auto emit = [&](int r, unsigned long long v) {
        const int64_t o = (int64_t)b * k + r;
        const int j = (int)~(uint32_t)(v & 0xffffffffull);  // candidate slot
        topk_idx[o] = (j >= 0 && j < F0) ? __ldg(idx + off + j) : ((j >= F0 && j < nc) ? (int32_t)(S + (j - F0)) : -1);
        if (topk_score) topk_score[o] = ordered_to_float((uint32_t)(v >> 32));
    };
    if (want > 0) {
        const unsigned long long *stg = stage + off + (int64_t)b * W;
        const int ns = (int)__ldcg(st + 5);  // the keys of bucket beta (at least want)
        if (ns <= SCAP) {
            int np = 64;
            while (np < ns) np <<= 1;
            for (int t = threadIdx.x; t < np; t += nth) ss[t] = t < ns ? __ldcg(stg + t) : 0ull;
            block_sort_desc_u64(ss, np);
            if (__ldcg(st + 7) <= (uint32_t)RANK_SEG) {
                // the selection lies in segments by bucket (higher buckets first): a key's output
                // position is its segment's start plus the keys of its segment above it; the
                // stage's largest keys follow in order
                const SelRange rg = sel_range(__ldcg(st + 8), __ldcg(st + 9));
                for (int t = threadIdx.x; t < above; t += nth) {
                    const unsigned long long v = sk[t];
                    const uint32_t bk = sel_bucket(rg, (uint32_t)(v >> 32));
                    const int lo = bk + 1 < (uint32_t)NB ? __ldcg(gh + bk + 1) : 0, hi = __ldcg(gh + bk);
                    int r = lo;
                    for (int q = lo; q < hi; q++) r += sk[q] > v;
                    emit(r, v);
                }
                for (int t = threadIdx.x; t < want; t += nth) emit(above + t, ss[t]);
                return;
            }
            for (int t = threadIdx.x; t < want; t += nth) sk[above + t] = ss[t];
        } else {
            // a crowded bucket: radix select of the want-th largest key over the stage, 8 bits at a
            // time from the top, until the digit's keys are exactly the ones still wanted
            unsigned long long prefix = 0ull, pmask = 0ull;
            int remaining = want;
            for (int pos = 64; pos > 0;) {
                const int wb = pos >= 8 ? 8 : pos, sh = pos - wb;
                const unsigned long long dm = (1ull << wb) - 1ull;
                for (int t = threadIdx.x; t < 256; t += nth) hist[t] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < ns; i += nth) {
                    const unsigned long long v = __ldcg(stg + i);
                    if ((v & pmask) == prefix) atomicAdd(&hist[(int)((v >> sh) & dm)], 1);
                }
                __syncthreads();
                if (threadIdx.x < 32) {  // the digit holding the remaining-th largest key, from the top
                    const int lane = threadIdx.x;
                    int c[8], sum = 0;
#pragma unroll
                    for (int q = 0; q < 8; q++) {
                        c[q] = hist[255 - 8 * lane - q];
                        sum += c[q];
                    }
                    int ab = warp_incl_scan(sum) - sum;
                    if (ab < remaining && ab + sum >= remaining) {
#pragma unroll
                        for (int q = 0; q < 8; q++) {
                            if (ab + c[q] >= remaining) {
                                s_dig = 255 - 8 * lane - q;
                                s_above = ab;
                                s_n = c[q];
                                break;
                            }
                            ab += c[q];
                        }
                    }
                }
                __syncthreads();
                prefix |= (unsigned long long)s_dig << sh;
                pmask |= dm << sh;
                remaining -= s_above;
                pos = sh;
                const bool whole = s_n == remaining;  // every key of the digit is wanted
                __syncthreads();
                if (whole) break;
            }
            // the wanted keys are exactly those >= prefix (its bits below the last pass are zero)
            if (threadIdx.x == 0) s_n = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < ns; i += nth) {
                const unsigned long long v = __ldcg(stg + i);
                if (v >= prefix) {
                    const int pos = atomicAdd(&s_n, 1);
                    if (pos < want) sk[above + pos] = v;
                }
            }
        }
    }
    block_sort_desc_u64(sk, kpow2);
    for (int r = threadIdx.x; r < k; r += nth) {
        if (r < nsel) {
            emit(r, sk[r]);
        } else {
            const int64_t o = (int64_t)b * k + r;
            topk_idx[o] = -1;
            if (topk_score) topk_score[o] = -INFINITY;
        }
    }
}

// Per chunk (SORT_TH threads): keys of higher buckets appended to the query's selection, keys of
// bucket beta to its stage; the query's last chunk to finish completes the query (final_of_query).
// Dynamic shared memory: kpow2 + SCAP keys.
__global__ void __launch_bounds__(SORT_TH, 1) k_ss_write(const float *__restrict__ Y, int tau_y,
                                                      const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                      const float *__restrict__ tail,
                                                      const int32_t *__restrict__ tail_count, int W, int B,
                                                      const int *__restrict__ chunk_start, const int *__restrict__ chunk_query, uint32_t *state, int kcap,
                                                      int *ghist, unsigned long long *sel, unsigned long long *stage,
                                                      const int32_t *__restrict__ idx, int k, int kpow2,
                                                      int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sk[];
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = chunk_query[c];
    uint32_t *st = state + NS * b;
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const bool every = st[1] == 0u;  // at most k candidates: every one, whatever its key
    const uint32_t beta = st[0];
    const SelRange rg = query_range(st);
    unsigned long long *out = sel + (int64_t)b * kcap;
    unsigned long long *stg = stage + q.off + (int64_t)b * W;  // capacity S_b + W
    int *gh = ghist + (int64_t)b * NB;                          // segment starts of the buckets above beta
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = j0; base < j1; base += SORT_TH) {
        const int j = base + threadIdx.x;
        uint32_t u = 0;
        bool gt = false, eq = false;
        if (j < j1) {
            u = key_of(q, j);
            const uint32_t bk = sel_bucket(rg, u);
            gt = every || bk > beta;
            eq = !every && bk == beta;
        }
        const unsigned long long key64 = ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j);
        // with more than k candidates a key of a higher bucket goes to its bucket's segment;
        // otherwise every candidate is appended
        if (gt && !every) out[atomicAdd(gh + sel_bucket(rg, u), 1)] = key64;
        const unsigned bg = __ballot_sync(0xffffffffu, gt && every), be = __ballot_sync(0xffffffffu, eq);
        int pg = 0, pe = 0;
        if (lane == 0) {
            if (bg) pg = (int)atomicAdd(st + 4, (uint32_t)__popc(bg));
            if (be) pe = (int)atomicAdd(st + 5, (uint32_t)__popc(be));
        }
        pg = __shfl_sync(0xffffffffu, pg, 0);
        pe = __shfl_sync(0xffffffffu, pe, 0);
        if (gt && every) out[pg + __popc(bg & lt)] = key64;
        if (eq) stg[pe + __popc(be & lt)] = key64;
    }
    // the finish counter of the query: state word 6 (zeroed by the front launch)
    if (!last_chunk_of_query((int *)(st + 6), 0, chunk_start[b + 1] - chunk_start[b])) return;
    final_of_query(b, sk, sel, kcap, stage, state, ghist + (int64_t)b * NB, W, idx, count, offs, k, kpow2, topk_idx,
                   topk_score);
}

}  // namespace stepsel

}  // namespace lsa
