// Top-k of one decode step (four launches).  A step has one query per sequence; its candidates
// are the F fetched slots, then the window entries as candidates F .. F + n - 1 (reported as
// entries S_b + j).  A candidate's 64-bit key is (order-preserving score key << 32) | ~slot: larger
// score first, then smaller slot, and no two keys are equal.
//   k_step_front   one grid, CTA roles that do not wait for one another: the scorer's work items
//                  and their table, the select's chunks (CH candidates each) and state; the cleared
//                  score histograms; per sequence the step's query and weights copied to the
//                  scorer's dense layout and the window entries' scores
//   k_li_tc<1>     (li_tc.cuh) the fetched entries' scores, and their histogram: the top 14 bits
//                  of the score key (HIST_BINS bins, li_tc.cuh) counted per sequence
//   k_ss_beta      one CTA per query: the histogram plus the window entries give the bin beta of
//                  the k-th largest key
//   k_ss_write     per chunk (one CTA per SM walks the chunks): the chunk's keys of higher bins are
//                  appended to the query's selection and bin beta's to its stage
//                  (any order: the keys carry their slots).  The query's last chunk to finish then
//                  orders the selection and the stage together (order_desc: buckets over their own
//                  score range, counting within a bucket) and writes the first k (a crowded stage
//                  is cut to its want largest keys by a radix select first).  A query with at most k candidates takes
//                  them all.  The output is as the batched select writes it.
#pragma once
#include "select_common.cuh"
#include "li_tc.cuh"
#include "topk.cuh"

namespace lsa {

namespace stepsel {

constexpr int HB = li::HIST_BINS;  // histogram bins per query
constexpr int SEL_TH = SEL_THREADS;
constexpr int CH = 4096;           // candidates per chunk
constexpr int SCAP = 4096;         // staged keys sorted in shared memory
constexpr int RANK_SEG = 32;       // largest bucket of the final order whose keys are ranked by counting
constexpr int NS = 8;              // state words per query

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
//   CTA 0           two prefixes over the sequences: the scorer's work items (ceil(ceil(F_b/128)/ch)
//                   per sequence, claim counter zeroed) and the select's chunks; the select state;
//                   then, a warp per sequence, the item table and the query of every chunk
//   nclear CTAs     zero the histograms, 4096 words each
//   B CTAs          one per sequence: its query and weights copied to the scorer's dense layout
//                   (and to shared memory) and the window entries' scores (a warp an entry)
struct FrontParams {
    const int32_t *count;      // [B] fetched entries
    const int64_t *offs;       // [B+1]
    const int32_t *win_count;  // [B] window entries, or null (no window entries)
    int W, B, k, n_h, d_I, dt;
    int ch;                    // key tiles per scorer work item
    int *chunk_start;          // [B+1]
    int *chunk_query;          // [chunks] the query of each chunk
    uint32_t *state;           // [B][NS]: [1] k if the query has more than k candidates, else 0;
                               // [3] candidates; [4] keys in the selection; [5] keys staged;
                               // [6] the write step's finish counter
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
    // ---- CTA 0: the scorer's items and the select's chunks
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
    // the item table and the query of every chunk, a warp per sequence (item_start and chunk_start
    // were written by this block: visible after the barrier)
    for (int b = warp; b < p.B; b += NW) {
        for (int c = p.chunk_start[b] + lane; c < p.chunk_start[b + 1]; c += 32) p.chunk_query[c] = b;
        const int64_t off = p.offs[b], S = p.offs[b + 1] - off;
        int F = p.count[b];
        F = F < 0 ? 0 : (F > S ? (int)S : F);
        li::write_items(p.items, p.item_start[b], b, F, (int)S, off, 1, p.ch, lane, 32);
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

// Per query with more than k candidates (one CTA of SEL_TH threads each): the bin beta of the k-th
// largest key from the scorer's histogram plus the window entries, into state words 0 (beta) and 2
// (keys of higher bins).  Dynamic shared memory: HB ints.
__global__ void __launch_bounds__(SEL_TH, 1) k_ss_beta(const float *__restrict__ Y, const int32_t *__restrict__ count,
                                                       const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                       const int32_t *__restrict__ tail_count, int W,
                                                       uint32_t *state, const int *__restrict__ ghist, int k)
{
    extern __shared__ int hs[];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, s_bin, s_above;
    const int b = blockIdx.x;
    uint32_t *st = state + NS * b;
    if (st[1] == 0u) return;  // at most k candidates: no bin needed
    const Query q = query(b, Y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int4 *g4 = (const int4 *)(ghist + (int64_t)b * HB);
    for (int t = threadIdx.x; t < HB / 4; t += SEL_TH) ((int4 *)hs)[t] = __ldg(g4 + t);
    __syncthreads();
    for (int j = q.F0 + threadIdx.x; j < nc; j += SEL_TH) atomicAdd(&hs[bin_of(key_of(q, j))], 1);
    __syncthreads();
    sel_find_bin<HB>((const unsigned int *)hs, k, warp_tot, &tot_a, &s_bin, &s_above);
    if (threadIdx.x == 0) {
        st[0] = (uint32_t)s_bin;
        st[2] = (uint32_t)s_above;
    }
}

// Called by every thread of the chunk CTA after its appends are in global memory: true in the CTA
// that finishes the query's chunks last.
__device__ __forceinline__ bool last_chunk_of_query(int *done, int nch)
{
    __shared__ int is_last;
    __threadfence();  // this CTA's global writes before its count
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(done, 1) == nch - 1;
    __syncthreads();
    if (!is_last) return false;
    __threadfence();  // the other chunks' writes, counted before ours, are read after this
    return true;
}

// Dynamic shared memory of k_ss_write (the query's last chunk): order_cap keys to order, as many of
// scratch, and SEL_NB bucket counters.
// Keys the final step may order: kpow2 + SCAP rounded up to a power of two (room for the bitonic
// fallback's padding).
__host__ __device__ inline int order_cap(int kpow2)
{
    int c = 64;
    while (c < kpow2 + SCAP) c <<= 1;
    return c;
}

__host__ __device__ inline size_t write_smem(int kpow2)
{
    return sizeof(unsigned long long) * 2 * (size_t)order_cap(kpow2) + sizeof(int) * (size_t)SEL_NB;
}

// One chunk of k_ss_write (and, in the query's last chunk to finish, the query's final step).
__device__ __forceinline__ void write_chunk(int c, unsigned long long *dsm, int *warp_tot, int &tot_a, int &s_bin,
                                            int &s_above, int &s_dig, int &s_dabove, int &s_dn, int &s_n,
                                            const float *__restrict__ Y, const int32_t *__restrict__ count,
                                            const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                            const int32_t *__restrict__ tail_count, int W, int B,
                                            const int *__restrict__ chunk_start, const int *__restrict__ chunk_query,
                                            uint32_t *state, const int *__restrict__ ghist, int kcap,
                                            unsigned long long *sel, unsigned long long *stage,
                                            const int32_t *__restrict__ idx, int k, int kpow2,
                                            int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    const int b = chunk_query[c];
    uint32_t *st = state + NS * b;
    const Query q = query(b, Y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const bool every = st[1] == 0u;  // at most k candidates: every one, whatever its key
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    auto key64 = [](uint32_t u, int j) { return ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j); };
    const uint32_t beta = st[0];      // the bin of the k-th largest key (k_ss_beta)
    const int above = (int)st[2];     // keys of higher bins
    // this chunk's appends: keys of higher bins to the selection, bin beta's to the stage
    unsigned long long *out = sel + (int64_t)b * kcap;
    unsigned long long *stg = stage + q.off + (int64_t)b * W;  // capacity S_b + W
    for (int base = j0; base < j1; base += SEL_TH) {
        const int j = base + threadIdx.x;
        uint32_t u = 0;
        bool gt = false, eq = false;
        if (j < j1) {
            u = key_of(q, j);
            const uint32_t bn = bin_of(u);
            gt = every || bn > beta;
            eq = !every && bn == beta;
        }
        const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        int pg = 0, pe = 0;
        if (lane == 0) {
            if (bg) pg = (int)atomicAdd(st + 4, (uint32_t)__popc(bg));
            if (be) pe = (int)atomicAdd(st + 5, (uint32_t)__popc(be));
        }
        pg = __shfl_sync(0xffffffffu, pg, 0);
        pe = __shfl_sync(0xffffffffu, pe, 0);
        if (gt) out[pg + __popc(bg & lt)] = key64(u, j);
        if (eq) stg[pe + __popc(be & lt)] = key64(u, j);
    }
    if (!last_chunk_of_query((int *)(st + 6), chunk_start[b + 1] - chunk_start[b])) return;

    // ---- the query's final step.  With at most SCAP staged keys, the selection and the whole stage
    // are ordered together (order_desc) and the first k positions written; otherwise a radix select
    // over the stage picks its want largest keys first.
    const int ocap = order_cap(kpow2);
    unsigned long long *sk = dsm;                   // ocap
    unsigned long long *tmp = sk + ocap;            // ocap
    int *cnt = (int *)(tmp + ocap);                 // SEL_NB
    int *h256 = cnt;                                // (the radix select's digits, before the order)
    const int nsel = nc < k ? nc : k;
    const int nfirst = every ? nsel : above;  // keys already in the selection
    int nord = nfirst;                        // keys to order
    for (int t = threadIdx.x; t < nfirst; t += SEL_TH) sk[t] = __ldcg(out + t);
    if (!every) {
        const int want = k - above;
        const int ns = (int)__ldcg(st + 5);  // the keys of bin beta
        if (ns <= SCAP) {
            for (int t = threadIdx.x; t < ns; t += SEL_TH) sk[above + t] = __ldcg(stg + t);
            nord = above + ns;
        } else {
            nord = k;
            // a crowded bin: radix select of the want-th largest key over the stage, 8 bits at a
            // time from the top, until the digit's keys are exactly the ones still wanted
            unsigned long long prefix = 0ull, pmask = 0ull;
            int remaining = want;
            for (int pos = 64; pos > 0;) {
                const int wb = pos >= 8 ? 8 : pos, sh = pos - wb;
                const unsigned long long dm = (1ull << wb) - 1ull;
                for (int t = threadIdx.x; t < 256; t += SEL_TH) h256[t] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < ns; i += SEL_TH) {
                    const unsigned long long v = __ldcg(stg + i);
                    if ((v & pmask) == prefix) atomicAdd(&h256[(int)((v >> sh) & dm)], 1);
                }
                __syncthreads();
                if (threadIdx.x < 32) {  // the digit holding the remaining-th largest key, from the top
                    int cc[8], sum = 0;
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        cc[i] = h256[255 - 8 * lane - i];
                        sum += cc[i];
                    }
                    int ab = warp_incl_scan(sum) - sum;
                    if (ab < remaining && ab + sum >= remaining) {
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            if (ab + cc[i] >= remaining) {
                                s_dig = 255 - 8 * lane - i;
                                s_dabove = ab;
                                s_dn = cc[i];
                                break;
                            }
                            ab += cc[i];
                        }
                    }
                }
                __syncthreads();
                prefix |= (unsigned long long)s_dig << sh;
                pmask |= dm << sh;
                remaining -= s_dabove;
                pos = sh;
                const bool whole = s_dn == remaining;  // every key of the digit is wanted
                __syncthreads();
                if (whole) break;
            }
            // the wanted keys are exactly those >= prefix (its bits below the last pass are zero)
            if (threadIdx.x == 0) s_n = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < ns; i += SEL_TH) {
                const unsigned long long v = __ldcg(stg + i);
                if (v >= prefix) {
                    const int pos = atomicAdd(&s_n, 1);
                    if (pos < want) sk[above + pos] = v;
                }
            }
        }
    }
    __syncthreads();
    int npow2 = 64;
    while (npow2 < nord) npow2 <<= 1;
    order_desc(sk, nord, npow2, tmp, cnt, RANK_SEG, [&](int r, unsigned long long v) {
        if (r >= k) return;  // a staged key below the k-th
        const int64_t o = (int64_t)b * k + r;
        const int j = (int)~(uint32_t)(v & 0xffffffffull);  // candidate slot
        topk_idx[o] = (j >= 0 && j < q.F0) ? __ldg(idx + q.off + j)
                                           : ((j >= q.F0 && j < nc) ? (int32_t)(q.S + (j - q.F0)) : -1);
        if (topk_score) topk_score[o] = ordered_to_float((uint32_t)(v >> 32));
    });
    for (int r = nsel + threadIdx.x; r < k; r += SEL_TH) {
        const int64_t o = (int64_t)b * k + r;
        topk_idx[o] = -1;
        if (topk_score) topk_score[o] = -INFINITY;
    }
}

__global__ void __launch_bounds__(SEL_TH, 1) k_ss_write(const float *__restrict__ Y, const int32_t *__restrict__ count,
                                                        const int64_t *__restrict__ offs,
                                                        const float *__restrict__ tail,
                                                        const int32_t *__restrict__ tail_count, int W, int B,
                                                        const int *__restrict__ chunk_start,
                                                        const int *__restrict__ chunk_query, uint32_t *state,
                                                        const int *__restrict__ ghist, int kcap,
                                                        unsigned long long *sel, unsigned long long *stage,
                                                        const int32_t *__restrict__ idx, int k, int kpow2,
                                                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long dsm[];
    __shared__ int warp_tot[32];
    __shared__ int tot_a, s_bin, s_above, s_dig, s_dabove, s_dn, s_n;
    const int nchunks = chunk_start[B];
    for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
        __syncthreads();  // shared memory of the previous chunk done with
        write_chunk(c, dsm, warp_tot, tot_a, s_bin, s_above, s_dig, s_dabove, s_dn, s_n, Y, count, offs, tail,
                    tail_count, W, B, chunk_start, chunk_query, state, ghist, kcap, sel, stage, idx, k, kpow2,
                    topk_idx, topk_score);
    }
}

}  // namespace stepsel

}  // namespace lsa
