// Top-k select of one decode step, spread over many CTAs.  A step has one query per sequence, so
// the one-CTA-per-query select of the batched call would leave all but B SMs idle; here the
// candidates of a query (its F fetched slots, then its window entries as candidates F .. F + n - 1,
// reported as entries S_b + j) are cut into chunks of CH with one CTA per chunk.  A candidate's
// 64-bit key is (order-preserving score key << 32) | ~slot: larger score first, then smaller slot,
// and no two keys are equal.
//   k_ss_setup   per query: candidates, chunk ranges (a prefix over the sequences), state; its other
//                CTAs clear the histograms
//   k_ss_hist12  per chunk: histogram of the top 12 bits of the score keys, added to the query's
//                histogram in global memory; the query's last chunk to finish picks the bucket
//                beta holding the k-th largest key (the keys above beta are all selected)
//   k_ss_write   per chunk: keys of higher buckets appended to the query's selection, keys of
//                bucket beta appended to the query's stage (order does not matter: the keys carry
//                their slots)
//   k_ss_final   per query: the `want` largest staged keys (a sort in shared memory, or a radix
//                select over the stage for a crowded bucket) complete the selection; bitonic sort
//                of the k keys and the output, as the one-CTA select writes it.
// A query with at most k candidates takes them all.  CTAs of one launch do not wait for one
// another: the per-query step after the histogram runs in whichever chunk CTA of the query finishes
// last (a counter per query, reset by that CTA), and kernel boundaries order the rest.
#pragma once
#include "common.cuh"

namespace lsa {

namespace stepsel {

constexpr int CH = 2048;   // candidates per chunk
constexpr int TH = 256;    // threads per chunk CTA
constexpr int SORT_TH = 1024;
constexpr int NB = 4096;   // buckets of the first pass (top 12 bits of the score key)
constexpr int SCAP = 8192; // staged keys a final CTA sorts in shared memory
constexpr int NS = 8;      // state words per query

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
// [5] keys appended to the stage.  ghist: [B][NB] bucket histograms, then the finish counters [B].
__global__ void __launch_bounds__(1024) k_ss_setup(const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                   const int32_t *__restrict__ tail_count, int W, int B, int k,
                                                   int *__restrict__ chunk_start, uint32_t *__restrict__ state,
                                                   int *__restrict__ ghist)
{
    if (blockIdx.x > 0) {  // CTAs 1.. clear the histograms and finish counters, 4096 words each
        const int64_t i0 = (int64_t)(blockIdx.x - 1) * 4096, n = (int64_t)B * (NB + 1);
        for (int64_t i = i0 + threadIdx.x; i < n && i < i0 + 4096; i += blockDim.x) ghist[i] = 0;
        return;
    }
    __shared__ int wt[32];
    __shared__ int carry;
    if (threadIdx.x == 0) {
        carry = 0;
        chunk_start[0] = 0;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < B; base += blockDim.x) {
        const int b = base + threadIdx.x;
        int n = 0;
        if (b < B) {
            const int64_t S = offs[b + 1] - offs[b];
            int F = count[b];
            F = F < 0 ? 0 : (F > S ? (int)S : F);
            int nt = tail_count ? tail_count[b] : 0;
            nt = nt < 0 ? 0 : (nt > W ? W : nt);
            const int nc = F + nt;
            n = (nc + CH - 1) / CH;
            uint32_t *st = state + NS * b;
            st[0] = 0u;
            st[1] = nc > k ? (uint32_t)k : 0u;
            st[2] = 0u;
            st[3] = (uint32_t)nc;
            st[4] = 0u;
            st[5] = 0u;
            st[6] = 0u;
            st[7] = 0u;
        }
        const int inc = warp_incl_scan(n);
        if (lane == 31) wt[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            const int v = lane < (int)(blockDim.x >> 5) ? wt[lane] : 0;
            wt[lane] = warp_incl_scan(v) - v;
        }
        __syncthreads();
        const int pos = carry + wt[warp] + inc;
        if (b < B) chunk_start[b + 1] = pos;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = pos;
        __syncthreads();
    }
}

__device__ __forceinline__ int query_of_chunk(const int *chunk_start, int B, int c)
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_start[mid] <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
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
                                                  int W, int B, const int *__restrict__ chunk_start, uint32_t *state,
                                                  int *ghist)
{
    __shared__ int hist[NB];
    __shared__ int s_beta, s_above;
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = query_of_chunk(chunk_start, B, c);
    uint32_t *st = state + NS * b;
    const int want = (int)st[1];
    if (want == 0) return;  // takes all its candidates (the same for every chunk of b)
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    for (int t = threadIdx.x; t < NB; t += TH) hist[t] = 0;
    __syncthreads();
    for (int j = j0 + threadIdx.x; j < j1; j += TH) atomicAdd(&hist[key_of(q, j) >> 20], 1);
    __syncthreads();
    int *gh = ghist + (int64_t)b * NB;
    for (int t = threadIdx.x; t < NB; t += TH)
        if (hist[t]) atomicAdd(gh + t, hist[t]);
    int *done = ghist + (int64_t)B * NB;
    if (!last_chunk_of_query(done, b, chunk_start[b + 1] - chunk_start[b])) return;
    // the bucket of the want-th largest key: thread t owns buckets NB - 16 (t + 1) .. NB - 16 t - 1
    constexpr int PER = NB / TH;
    const int hi = NB - PER * (int)threadIdx.x;
    int cnt = 0;
#pragma unroll
    for (int i = 1; i <= PER; i++) cnt += __ldcg(gh + hi - i);
    int above, unused_p, total, unused_t;
    block_excl_scan2(cnt, 0, above, unused_p, total, unused_t);
    if (above < want && above + cnt >= want) {
        for (int i = 1; i <= PER; i++) {
            const int h = __ldcg(gh + hi - i);
            if (above + h >= want) {
                s_beta = hi - i;
                s_above = above;
                break;
            }
            above += h;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        st[0] = (uint32_t)s_beta;
        st[2] = (uint32_t)s_above;
        st[1] = (uint32_t)(want - s_above);
    }
}

__global__ void __launch_bounds__(TH) k_ss_write(const float *__restrict__ Y, int tau_y, const int32_t *__restrict__ count,
                                                 const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                 const int32_t *__restrict__ tail_count, int W, int B,
                                                 const int *__restrict__ chunk_start, uint32_t *state, int kcap,
                                                 unsigned long long *__restrict__ sel,
                                                 unsigned long long *__restrict__ stage)
{
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = query_of_chunk(chunk_start, B, c);
    uint32_t *st = state + NS * b;
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const bool all = st[1] == 0u;  // at most k candidates: every one, whatever its key
    const uint32_t beta = st[0];
    unsigned long long *out = sel + (int64_t)b * kcap;
    unsigned long long *stg = stage + q.off + (int64_t)b * W;  // capacity S_b + W
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = j0; base < j1; base += TH) {
        const int j = base + threadIdx.x;
        uint32_t u = 0;
        bool gt = false, eq = false;
        if (j < j1) {
            u = key_of(q, j);
            gt = all || (u >> 20) > beta;
            eq = !all && (u >> 20) == beta;
        }
        const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        int pg = 0, pe = 0;
        if (lane == 0) {
            if (bg) pg = (int)atomicAdd(st + 4, (uint32_t)__popc(bg));
            if (be) pe = (int)atomicAdd(st + 5, (uint32_t)__popc(be));
        }
        pg = __shfl_sync(0xffffffffu, pg, 0);
        pe = __shfl_sync(0xffffffffu, pe, 0);
        const unsigned long long key64 = ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j);
        if (gt) out[pg + __popc(bg & lt)] = key64;
        if (eq) stg[pe + __popc(be & lt)] = key64;
    }
}

// Per query (SORT_TH threads): the selection's keys of higher buckets plus the want largest keys of
// bucket beta, sorted by key descending (score descending, slot ascending), then the output.
// Dynamic shared memory: kpow2 + SCAP keys.
__global__ void __launch_bounds__(SORT_TH) k_ss_final(const unsigned long long *__restrict__ sel, int kcap,
                                                      const unsigned long long *__restrict__ stage,
                                                      const uint32_t *__restrict__ state, int W,
                                                      const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                                      const int64_t *__restrict__ offs, int k, int kpow2,
                                                      int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sk[];
    unsigned long long *ss = sk + kpow2;
    __shared__ int hist[256];
    __shared__ int s_dig, s_above, s_n;
    const int b = blockIdx.x;
    const uint32_t *st = state + NS * b;
    const int nc = (int)st[3];
    const int want = (int)st[1];
    const int above = (int)st[2];
    const int nsel = nc < k ? nc : k;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    int F0 = count[b];
    F0 = F0 < 0 ? 0 : (F0 > S ? (int)S : F0);
    const unsigned long long *mine = sel + (int64_t)b * kcap;
    const int nfirst = want == 0 ? nsel : above;  // keys already in the selection
    for (int t = threadIdx.x; t < kpow2; t += SORT_TH) sk[t] = t < nfirst ? mine[t] : 0ull;
    if (want > 0) {
        const unsigned long long *stg = stage + off + (int64_t)b * W;
        const int ns = (int)st[5];  // the keys of bucket beta (at least want)
        if (ns <= SCAP) {
            int np = 64;
            while (np < ns) np <<= 1;
            for (int t = threadIdx.x; t < np; t += SORT_TH) ss[t] = t < ns ? stg[t] : 0ull;
            block_sort_desc_u64(ss, np);
            for (int t = threadIdx.x; t < want; t += SORT_TH) sk[above + t] = ss[t];
        } else {
            // a crowded bucket: radix select of the want-th largest key over the stage (the top 12
            // bits are beta in every staged key; 52 bits remain: 8-bit digits, the last one 4 bits)
            unsigned long long prefix = (unsigned long long)st[0] << 52, pmask = 0xFFFull << 52;
            int remaining = want;
            for (int pass = 0; pass < 7; pass++) {
                const int shift = pass < 6 ? 44 - 8 * pass : 0;
                const unsigned long long dmask = pass < 6 ? 255ull : 15ull;
                for (int t = threadIdx.x; t < 256; t += SORT_TH) hist[t] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < ns; i += SORT_TH) {
                    const unsigned long long v = stg[i];
                    if ((v & pmask) == prefix) atomicAdd(&hist[(int)((v >> shift) & dmask)], 1);
                }
                __syncthreads();
                if (threadIdx.x == 0) {
                    int cum = 0, dg = 0;
                    for (int d = 255; d >= 0; d--) {
                        if (cum + hist[d] >= remaining) {
                            dg = d;
                            break;
                        }
                        cum += hist[d];
                    }
                    s_dig = dg;
                    s_above = cum;
                }
                __syncthreads();
                prefix |= (unsigned long long)s_dig << shift;
                pmask |= dmask << shift;
                remaining -= s_above;
                __syncthreads();
            }
            // prefix is the want-th largest staged key: take every staged key at or above it
            if (threadIdx.x == 0) s_n = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < ns; i += SORT_TH) {
                const unsigned long long v = stg[i];
                if (v >= prefix) {
                    const int pos = atomicAdd(&s_n, 1);
                    if (pos < want) sk[above + pos] = v;
                }
            }
        }
    }
    block_sort_desc_u64(sk, kpow2);
    for (int r = threadIdx.x; r < k; r += SORT_TH) {
        const int64_t o = (int64_t)b * k + r;
        if (r < nsel) {
            const unsigned long long v = sk[r];
            const int j = (int)~(uint32_t)(v & 0xffffffffull);  // candidate slot
            topk_idx[o] = (j >= 0 && j < F0) ? __ldg(idx + off + j)
                                             : ((j >= F0 && j < nc) ? (int32_t)(S + (j - F0)) : -1);
            if (topk_score) topk_score[o] = ordered_to_float((uint32_t)(v >> 32));
        } else {
            topk_idx[o] = -1;
            if (topk_score) topk_score[o] = -INFINITY;
        }
    }
}

}  // namespace stepsel

}  // namespace lsa
