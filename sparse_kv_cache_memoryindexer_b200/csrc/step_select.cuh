// Top-k select of one decode step, spread over many CTAs.  A step has one query per sequence, so
// the one-CTA-per-query select of the batched call would leave all but B SMs idle; here the
// candidates of a query (its F fetched slots, then its window entries as candidates F .. F + n - 1,
// reported as entries S_b + j) are cut into chunks of CH, and the most-significant-digit-first
// radix search on the order-preserving keys runs with one CTA per chunk:
//   k_ss_setup   per query: candidates, chunk ranges (a prefix over the sequences), search state
//   k_ss_hist    per chunk: histogram of the next 8-bit digit of the keys that match the prefix so
//                far, added to the query's histogram in global memory; the query's last chunk to
//                finish then picks the digit where the count from the top reaches the keys still
//                wanted (4 passes: the k-th largest key K*)
//   k_ss_count   per chunk: keys above K* and keys equal to it; the query's last chunk turns the
//                chunk counts into chunk offsets (slot order)
//   k_ss_write   per chunk: every key above K*, and the first equal keys in slot order, to the
//                query's selection
//   k_ss_sort    per query: bitonic sort of the selection (key descending, slot ascending) and the
//                output, as the one-CTA select writes it.
// CTAs of one launch do not wait for one another: the per-query step after a launch's chunks runs
// in whichever chunk CTA of the query finishes last (a counter per query, reset by that CTA), and
// kernel boundaries order the rest.
#pragma once
#include "common.cuh"

namespace lsa {

namespace stepsel {

constexpr int CH = 2048;   // candidates per chunk
constexpr int TH = 256;    // threads per chunk CTA
constexpr int SORT_TH = 512;

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

// state per query: [0] prefix (the key bits fixed so far), [1] keys still wanted at the prefix,
// [2] keys above the final K*, [3] candidates.  ghist: [B][256] digit histograms, then the
// per-query finish counters of k_ss_hist [B] and of k_ss_count [B].
__global__ void __launch_bounds__(1024) k_ss_setup(const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                   const int32_t *__restrict__ tail_count, int W, int B, int k,
                                                   int *__restrict__ chunk_start, uint32_t *__restrict__ state,
                                                   int *__restrict__ ghist)
{
    __shared__ int wt[32];
    __shared__ int carry;
    if (threadIdx.x == 0) {
        carry = 0;
        chunk_start[0] = 0;
    }
    for (int i = threadIdx.x; i < B * 258; i += blockDim.x) ghist[i] = 0;
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
            // a query with at most k candidates takes them all: prefix 0 is below every key
            state[4 * b + 0] = 0u;
            state[4 * b + 1] = nc > k ? (uint32_t)k : 0u;
            state[4 * b + 2] = nc > k ? 0u : (uint32_t)nc;
            state[4 * b + 3] = (uint32_t)nc;
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

__global__ void __launch_bounds__(TH) k_ss_hist(const float *__restrict__ Y, int tau_y, const int32_t *__restrict__ count,
                                                const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                const int32_t *__restrict__ tail_count, int W, int B,
                                                const int *__restrict__ chunk_start, uint32_t *state, int pass,
                                                int *ghist, int *done)
{
    static_assert(TH == 256, "one digit bin per thread in the digit step");
    __shared__ int hist[256];
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = query_of_chunk(chunk_start, B, c);
    const uint32_t remaining = state[4 * b + 1];
    if (remaining == 0u) return;  // takes all its candidates (the same for every chunk of b)
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const int shift = 24 - 8 * pass;
    const uint32_t pmask = pass == 0 ? 0u : ~((1u << (32 - 8 * pass)) - 1u);
    const uint32_t prefix = state[4 * b + 0];
    for (int t = threadIdx.x; t < 256; t += TH) hist[t] = 0;
    __syncthreads();
    for (int j = j0 + threadIdx.x; j < j1; j += TH) {
        const uint32_t u = key_of(q, j);
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < 256; t += TH)
        if (hist[t]) atomicAdd(ghist + b * 256 + t, hist[t]);
    if (!last_chunk_of_query(done, b, chunk_start[b + 1] - chunk_start[b])) return;
    // the digit: thread t holds bin 255 - t, so an inclusive scan over the threads counts the keys
    // at or above each digit; exactly one bin has above < remaining <= at or above
    const int dg = 255 - (int)threadIdx.x;
    const int h = atomicExch(ghist + b * 256 + dg, 0);  // read, and clear for the next pass
    int pos, unused_p, total, unused_t;
    block_excl_scan2(h, 0, pos, unused_p, total, unused_t);
    const uint32_t above = (uint32_t)pos, upto = (uint32_t)(pos + h);
    const bool chosen = h > 0 && above < remaining && upto >= remaining;
    // fewer matching keys than wanted cannot happen (every pass counts the same keys); digit 0 then
    const bool none = threadIdx.x == TH - 1 && (uint32_t)total < remaining;
    if (chosen || none) {
        const uint32_t cum = none ? (uint32_t)total : above;
        state[4 * b + 0] = prefix | ((uint32_t)(none ? 0 : dg) << shift);
        state[4 * b + 1] = remaining - cum;
        state[4 * b + 2] += cum;
    }
}

__global__ void __launch_bounds__(TH) k_ss_count(const float *__restrict__ Y, int tau_y, const int32_t *__restrict__ count,
                                                 const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                 const int32_t *__restrict__ tail_count, int W, int B,
                                                 const int *__restrict__ chunk_start,
                                                 const uint32_t *__restrict__ state, int *gtc, int *eqc, int *done)
{
    __shared__ int sgt, seq;
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = query_of_chunk(chunk_start, B, c);
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const uint32_t K = state[4 * b + 0];
    const bool all = state[4 * b + 1] == 0u;  // at most k candidates: every one, whatever its key
    if (threadIdx.x == 0) sgt = seq = 0;
    __syncthreads();
    int ng = 0, ne = 0;
    for (int j = j0 + threadIdx.x; j < j1; j += TH) {
        const uint32_t u = key_of(q, j);
        ng += (all || u > K) ? 1 : 0;
        ne += (!all && u == K) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ng += __shfl_xor_sync(0xffffffffu, ng, o);
        ne += __shfl_xor_sync(0xffffffffu, ne, o);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&sgt, ng);
        atomicAdd(&seq, ne);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        gtc[c] = sgt;
        eqc[c] = seq;
    }
    const int c0 = chunk_start[b], c1 = chunk_start[b + 1];
    if (!last_chunk_of_query(done, b, c1 - c0)) return;
    // exclusive offsets of the query's chunk counts, in chunk (slot) order
    int carry_g = 0, carry_e = 0;
    for (int base = c0; base < c1; base += TH) {
        const int cc = base + threadIdx.x;
        const int g = cc < c1 ? __ldcg(gtc + cc) : 0, e = cc < c1 ? __ldcg(eqc + cc) : 0;
        int pg, pe, tg, te;
        block_excl_scan2(g, e, pg, pe, tg, te);
        if (cc < c1) {
            gtc[cc] = carry_g + pg;
            eqc[cc] = carry_e + pe;
        }
        carry_g += tg;
        carry_e += te;
    }
}

__global__ void __launch_bounds__(TH) k_ss_write(const float *__restrict__ Y, int tau_y, const int32_t *__restrict__ count,
                                                 const int64_t *__restrict__ offs, const float *__restrict__ tail,
                                                 const int32_t *__restrict__ tail_count, int W, int B,
                                                 const int *__restrict__ chunk_start,
                                                 const uint32_t *__restrict__ state, const int *__restrict__ gtb,
                                                 const int *__restrict__ eqb, int kcap,
                                                 unsigned long long *__restrict__ sel)
{
    __shared__ int warp_tot[32];
    const int c = blockIdx.x;
    if (c >= chunk_start[B]) return;
    const int b = query_of_chunk(chunk_start, B, c);
    const Query q = query(b, Y, tau_y, count, offs, tail, tail_count, W);
    const int nc = q.F0 + q.nt;
    const int j0 = (c - chunk_start[b]) * CH, j1 = min(nc, j0 + CH);
    const uint32_t K = state[4 * b + 0];
    const int want_eq = (int)state[4 * b + 1], n_gt = (int)state[4 * b + 2];
    const bool all = want_eq == 0;  // at most k candidates: every one, whatever its key
    unsigned long long *out = sel + (int64_t)b * kcap;
    int carry_gt = gtb[c], carry_eq = eqb[c];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = j0; base < j1; base += TH) {
        const int j = base + threadIdx.x;
        uint32_t u = 0;
        int gt = 0, eq = 0;
        if (j < j1) {
            u = key_of(q, j);
            gt = (all || u > K) ? 1 : 0;
            eq = (!all && u == K) ? 1 : 0;
        }
        // block exclusive scans of gt and eq
        int pos[2];
        int tot[2];
#pragma unroll
        for (int k2 = 0; k2 < 2; k2++) {
            const int v = k2 == 0 ? gt : eq;
            const int inc = warp_incl_scan(v);
            if (lane == 31) warp_tot[warp] = inc;
            __syncthreads();
            int before = 0, total = 0;
            for (int w = 0; w < TH / 32; w++) {
                before += w < warp ? warp_tot[w] : 0;
                total += warp_tot[w];
            }
            pos[k2] = before + inc - v;
            tot[k2] = total;
            __syncthreads();
        }
        const unsigned long long key64 = ((unsigned long long)u << 32) | (uint32_t)(~(uint32_t)j);
        if (gt) out[carry_gt + pos[0]] = key64;
        if (eq && carry_eq + pos[1] < want_eq) out[n_gt + carry_eq + pos[1]] = key64;
        carry_gt += tot[0];
        carry_eq += tot[1];
    }
}

__global__ void __launch_bounds__(SORT_TH) k_ss_sort(const unsigned long long *__restrict__ sel, int kcap,
                                                      const uint32_t *__restrict__ state,
                                                      const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                                      const int64_t *__restrict__ offs, int k, int kpow2,
                                                      int32_t *__restrict__ topk_idx, float *__restrict__ topk_score)
{
    extern __shared__ unsigned long long sk[];
    const int b = blockIdx.x;
    const int nc = (int)state[4 * b + 3];
    const int nsel = nc < k ? nc : k;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    int F0 = count[b];
    F0 = F0 < 0 ? 0 : (F0 > S ? (int)S : F0);
    for (int t = threadIdx.x; t < kpow2; t += SORT_TH) sk[t] = t < nsel ? sel[(int64_t)b * kcap + t] : 0ull;
    __syncthreads();
    for (int size = 2; size <= kpow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < kpow2 / 2; t += SORT_TH) {
                const int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = sk[lo], c = sk[hi];
                if ((a < c) == desc) {
                    sk[lo] = c;
                    sk[hi] = a;
                }
            }
            __syncthreads();
        }
    }
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
