// Golden labels of one future window (blog review "FlashMemory-DeepSeek-V4", section 4.1;
// hyper.ai summary, "Dataset"; gist.science summary, section 2.2): for every token i of the window
// and every CSA layer l, softmax over the raw indexer logits of the sequence's entries and keep the
// top-p nucleus (entries by probability descending, ties to the smaller entry, until the kept mass
// reaches p of the total); an entry is golden for token i if at least theta layers keep it; the
// window's label set is the union over its tokens.
//
// k_golden_nucleus   one CTA per (sequence, token, layer) row.  The kept set is {key > K*} plus the
//                    first n of {key == K*} in entry order, where key is the order-preserving
//                    integer image of the logit: the first n_p entries of the row sorted by
//                    (logit desc, entry asc), n_p the first count whose mass sum e reaches p Z
//                    (e = exp(z - max z), Z = sum of all e).
//                    Fast path (two reads of the row): the maximum; then Z in fp32 exp with an
//                    error bound of its own, while the entries within 4 of the maximum are
//                    gathered in shared memory.  Their mass (in double) tells whether they hold
//                    the nucleus (the kept set is a prefix of the sorted row, so any such prefix
//                    of candidates gives the same crossing); they are sorted and scanned in double
//                    for the crossing against both ends of the target's interval
//                    p [Z - err, Z + err].  When both ends give the
//                    same position it is the one an fp64 Z gives; otherwise Z is recomputed in
//                    double and the scan repeated.  The kept entries' bits are set from the
//                    sorted candidates.
//                    General path (more than CAND entries within 4, or less than the target's
//                    mass there): Z in double and, for a few depths D, the mass and count of the
//                    entries within D of the maximum; the smallest such set whose mass reaches
//                    p Z and that has at most CAND entries is sorted and scanned in double;
//                    otherwise (flat rows) K* and n come from a most-significant-digit-first
//                    radix search on the key driven by the masses, and a pass over the row sets
//                    the bits.
//                    Bits go to a [tau][Lc][ceil(T/32)] bit plane by atomicOr (words can
//                    straddle two sequences).
// k_golden_vote      32 words per CTA: bit-sliced vote counts over the Lc layers per token, theta
//                    test, OR over the tokens, one label byte per entry.
#pragma once
#include "select_common.cuh"

namespace lsa {

namespace golden {

constexpr int THREADS = 256;
constexpr int CAND = 4096;       // candidates sorted in shared memory
constexpr int ND = 6;            // depths below the maximum tried for the candidate set
__device__ __forceinline__ float depth(int k) { return k == 0 ? 4.f : (k == 1 ? 8.f : (k == 2 ? 12.f : (k == 3 ? 16.f : (k == 4 ? 24.f : 40.f)))); }

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = -INFINITY;
    for (int w = 0; w < THREADS / 32; w++) r = fmaxf(r, red[w]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ double block_sum(double v, double *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double r = 0.0;
    for (int w = 0; w < THREADS / 32; w++) r += red[w];
    __syncthreads();
    return r;
}

// Appends v to cand when `take` (at most CAND entries; *counter counts every append, so a count
// above CAND tells that some did not fit): one shared atomic per warp.  Every lane of the warp calls.
__device__ __forceinline__ void warp_append(bool take, unsigned long long v, int *counter, unsigned long long *cand)
{
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (!m) return;
    const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(counter, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    const int at = base + __popc(m & ((1u << lane) - 1u));
    if (take && at < CAND) cand[at] = v;
}

// Block-wide inclusive scan of one double per thread: returns this thread's inclusive prefix and
// the block total in *total.  red: THREADS / 32 doubles.  Starts and ends with a barrier.
__device__ __forceinline__ double block_incl_scan_d(double v, double *red, double *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) red[warp] = v;
    __syncthreads();
    double before = 0.0, t = 0.0;
    for (int w = 0; w < THREADS / 32; w++) {
        before += w < warp ? red[w] : 0.0;
        t += red[w];
    }
    *total = t;
    __syncthreads();
    return before + v;
}

// Crossing of the sorted candidates cand[0..nc): the first position r whose cumulative mass
// sum_{r' <= r} exp(z_r' - m) reaches target_lo (*cross_lo) and target_hi (*cross_hi); INT_MAX
// when not reached.  Masses in double, summed in blocks of THREADS in candidate order.
__device__ __forceinline__ void scan_crossing(const unsigned long long *cand, int nc, float m, double target_lo,
                                              double target_hi, double *red, int *s_lo, int *s_hi)
{
    if (threadIdx.x == 0) {
        *s_lo = INT_MAX;
        *s_hi = INT_MAX;
    }
    double carry = 0.0;
    for (int base = 0; base < nc; base += THREADS) {
        const int r0 = base + threadIdx.x;
        const double e = r0 < nc ? exp((double)ordered_to_float((uint32_t)(cand[r0] >> 32)) - (double)m) : 0.0;
        double total;
        const double inc = carry + block_incl_scan_d(e, red, &total);
        if (r0 < nc && inc >= target_lo) atomicMin(s_lo, r0);
        if (r0 < nc && inc >= target_hi) atomicMin(s_hi, r0);
        carry += total;
        __syncthreads();
        if (*s_hi < INT_MAX) break;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(THREADS) k_golden_nucleus(const float *__restrict__ z, const int64_t *__restrict__ offs,
                                                            int64_t T, int B, int tau, int Lc, double p,
                                                            uint32_t *__restrict__ bits, int64_t W32,
                                                            int32_t *__restrict__ nsize)
{
    __shared__ double hmass[256];
    __shared__ int hcnt[256];
    __shared__ unsigned long long cand[CAND];  // (key << 32) | ~entry
    __shared__ double dmass[ND][THREADS / 32];
    __shared__ int dcnt[ND][THREADS / 32];
    __shared__ int s_nc, s_depth, s_cross, s_cross_hi;
    __shared__ float fred[THREADS / 32];
    __shared__ double dred[THREADS / 32];
    __shared__ uint32_t s_prefix;
    __shared__ double s_need;
    __shared__ int s_taken_above, s_last_eq;
    __shared__ int warp_tot[32];
    const int r = blockIdx.x;
    const int b = r / (tau * Lc), i = (r / Lc) % tau, l = r % Lc;
    const int64_t off = offs[b], S = offs[b + 1] - off;
    if (S <= 0) {
        if (threadIdx.x == 0 && nsize) nsize[r] = 0;
        return;
    }
    const float *row = z + ((int64_t)i * Lc + l) * T + off;
    uint32_t *plane = bits + ((int64_t)i * Lc + l) * W32;
    // the row in 16-byte vectors from its first 16-byte boundary; the at most three entries before
    // it and the at most three after the last whole vector go to threads 0..5 one by one
    const int head = (int)min((int64_t)((4 - (((uintptr_t)row >> 2) & 3)) & 3), S);
    const int64_t nvec = (S - head) >> 2;
    const int64_t tail0 = head + 4 * nvec;
    const float4 *vrow = (const float4 *)(row + head);
    const int64_t lone = threadIdx.x < head ? (int64_t)threadIdx.x
                         : (threadIdx.x < head + (S - tail0) ? tail0 + (threadIdx.x - head) : (int64_t)-1);
    float m = -INFINITY;
    {
        float4 mv[4];
#pragma unroll
        for (int q = 0; q < 4; q++) mv[q] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        for (int64_t base = 0; base < nvec; base += 4 * THREADS) {  // four vector loads in flight
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int64_t v = base + q * THREADS + threadIdx.x;
                if (v < nvec) {
                    const float4 x = __ldg(vrow + v);
                    mv[q] = make_float4(fmaxf(mv[q].x, x.x), fmaxf(mv[q].y, x.y), fmaxf(mv[q].z, x.z), fmaxf(mv[q].w, x.w));
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 4; q++) m = fmaxf(m, fmaxf(fmaxf(mv[q].x, mv[q].y), fmaxf(mv[q].z, mv[q].w)));
        if (lone >= 0) m = fmaxf(m, __ldg(row + lone));
    }
    m = block_max(m, fred);

    // ---------------------------------------------------------------- fast path
    if (m > -INFINITY && m < INFINITY) {
        if (threadIdx.x == 0) s_nc = 0;
        __syncthreads();
        // Z in fp32 and the bound of its error: e^x = 2^(x log2 e) with x = z - m rounded once, the
        // product and log2 e rounded once each (an error of 3 * 2^-24 |x| in the exponent, |x| < 104
        // wherever the result is normal); exp2f is within 2 ulp (2^-22 relative); each thread's
        // fp32 sum of its at most S / THREADS + 5 terms rounds by at most that many ulps; a result
        // below the smallest normal is off by at most 2^-126 absolute.  An entry within 4 of the
        // maximum is appended to the candidates by its own thread (they are few).
        constexpr float LOG2E = 1.4426950408889634f;
        float zf = 0.f;
        auto take = [&](float x, int s) {  // (s: the entry, only formed for an appended one)
            zf += exp2f((x - m) * LOG2E);
            if (m - x < 4.f) {
                const int at = atomicAdd(&s_nc, 1);
                if (at < CAND) cand[at] = ((unsigned long long)float_to_ordered(x) << 32) | (uint32_t)(~(uint32_t)s);
            }
        };
        const int nv = (int)nvec;  // (S < 2^31 entries)
        for (int base = 0; base < nv; base += 4 * THREADS) {
            float4 x[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {  // four vector loads in flight
                const int v = base + q * THREADS + (int)threadIdx.x;
                x[q] = v < nv ? __ldg(vrow + v) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int s = head + 4 * (base + q * THREADS + (int)threadIdx.x);
                take(x[q].x, s);
                take(x[q].y, s + 1);
                take(x[q].z, s + 2);
                take(x[q].w, s + 3);
            }
        }
        if (lone >= 0) take(__ldg(row + lone), (int)lone);
        __syncthreads();
        const double Z32 = block_sum((double)zf, dred);
        // (plus the rounding of sums in double, here and in an fp64 Z: terms per thread + 64 ulps)
        const double err = 1.01 * Z32 * (0x1p-22 + 3.0 * 104.0 * 0x1p-24 + ((double)S / THREADS + 5.0) * 0x1p-24) +
                           (double)S * 0x1p-126 + 2.0 * Z32 * ((double)S / THREADS + 64.0) * 0x1p-53;
        const int nc = s_nc;
        if (nc <= CAND) {
            // the exact mass of the entries within 4 of the maximum
            double m4 = 0.0;
            for (int t = threadIdx.x; t < nc; t += THREADS)
                m4 += exp((double)ordered_to_float((uint32_t)(cand[t] >> 32)) - (double)m);
            m4 = block_sum(m4, dred);
            const double t_hi = p * (Z32 + err) * (1.0 + 0x1p-50);
            const double t_lo = p * (Z32 - err) * (1.0 - 0x1p-50);
            if (m4 >= t_hi) {  // the entries within 4 hold the nucleus
                int np2 = 64;
                while (np2 < nc) np2 <<= 1;
                for (int t = nc + threadIdx.x; t < np2; t += THREADS) cand[t] = 0ull;
                block_sort_desc_u64(cand, np2);
                scan_crossing(cand, nc, m, t_lo, t_hi, dred, &s_cross, &s_cross_hi);
                int cross = s_cross;
                if (cross != s_cross_hi) {
                    // the target's interval holds a crossing: Z in double decides
                    double zd = 0.0;
                    for (int64_t s = threadIdx.x; s < S; s += THREADS) zd += exp((double)__ldg(row + s) - (double)m);
                    const double Zd = block_sum(zd, dred);
                    scan_crossing(cand, nc, m, p * Zd, p * Zd, dred, &s_cross, &s_cross_hi);
                    cross = s_cross;
                }
                if (cross >= nc) cross = nc - 1;  // rounding left the target above the candidates' mass
                for (int t = threadIdx.x; t <= cross; t += THREADS) {
                    const int64_t g = off + (int64_t)(int)(~(uint32_t)(cand[t] & 0xffffffffull));
                    atomicOr(plane + (g >> 5), 1u << (g & 31));
                }
                if (threadIdx.x == 0 && nsize) nsize[r] = cross + 1;
                return;
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- general path
    double tot = 0.0, dm[ND];
    int dc[ND];
#pragma unroll
    for (int k = 0; k < ND; k++) {
        dm[k] = 0.0;
        dc[k] = 0;
    }
    for (int64_t s = threadIdx.x; s < S; s += THREADS) {
        const float zs = __ldg(row + s);
        const double e = exp((double)zs - (double)m);
        tot += e;
#pragma unroll
        for (int k = 0; k < ND; k++)
            if (m - zs < depth(k)) {
                dm[k] += e;
                dc[k]++;
            }
    }
    {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
        for (int k = 0; k < ND; k++) {
            double v = dm[k];
            int c = dc[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                v += __shfl_xor_sync(0xffffffffu, v, o);
                c += __shfl_xor_sync(0xffffffffu, c, o);
            }
            if (lane == 0) {
                dmass[k][warp] = v;
                dcnt[k][warp] = c;
            }
        }
    }
    tot = block_sum(tot, dred);  // (its barriers also publish dmass / dcnt)
    const double target = p * tot;
    if (threadIdx.x == 0) {
        s_depth = -1;
        for (int k = 0; k < ND; k++) {
            double v = 0.0;
            int c = 0;
            for (int w = 0; w < THREADS / 32; w++) {
                v += dmass[k][w];
                c += dcnt[k][w];
            }
            if (v >= target && c <= CAND) {
                s_depth = k;
                break;
            }
        }
        s_nc = 0;
        s_cross = INT_MAX;
    }
    __syncthreads();
    if (s_depth >= 0) {
        // ---- candidate path: the entries within depth(k) of the maximum, sorted
        const float D = depth(s_depth);
        for (int64_t base = 0; base < S; base += THREADS) {
            const int64_t s = base + threadIdx.x;
            const float zs = s < S ? row[s] : -INFINITY;
            warp_append(s < S && m - zs < D,
                        ((unsigned long long)float_to_ordered(zs) << 32) | (uint32_t)(~(uint32_t)s), &s_nc, cand);
        }
        __syncthreads();
        const int nc = s_nc < CAND ? s_nc : CAND;
        int np2 = 64;
        while (np2 < nc) np2 <<= 1;
        for (int t = nc + threadIdx.x; t < np2; t += THREADS) cand[t] = 0ull;
        block_sort_desc_u64(cand, np2);  // descending
        // cumulative mass in sorted order; the first position where it reaches the target
        double carry = 0.0;
        for (int base = 0; base < nc; base += THREADS) {
            const int r0 = base + threadIdx.x;
            const double e = r0 < nc ? exp((double)ordered_to_float((uint32_t)(cand[r0] >> 32)) - (double)m) : 0.0;
            // block inclusive scan of e (warp scan + warp totals)
            const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
            double v = e;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (lane == 31) dred[warp] = v;
            __syncthreads();
            double before = 0.0, total = 0.0;
            for (int w = 0; w < THREADS / 32; w++) {
                before += w < warp ? dred[w] : 0.0;
                total += dred[w];
            }
            const double inc = carry + before + v;
            if (r0 < nc && inc >= target) atomicMin(&s_cross, r0);  // the first position reaching it
            carry += total;
            __syncthreads();
            if (s_cross < INT_MAX) break;
        }
        __syncthreads();
        const int cross = s_cross < INT_MAX ? s_cross : nc - 1;
        if (threadIdx.x == 0) {
            s_prefix = (uint32_t)(cand[cross] >> 32);
            s_last_eq = (int)(~(uint32_t)(cand[cross] & 0xffffffffull));
            if (nsize) nsize[r] = cross + 1;
        }
        __syncthreads();
    } else {

    // radix search: all keys above the prefix are kept; `need` is the mass still to be taken
    uint32_t prefix = 0, pmask = 0;
    double need = target;
    int above = 0;
    for (int pass = 0; pass < 4; pass++) {
        const int shift = 24 - 8 * pass;
        for (int t = threadIdx.x; t < 256; t += THREADS) {
            hmass[t] = 0.0;
            hcnt[t] = 0;
        }
        __syncthreads();
        for (int64_t s = threadIdx.x; s < S; s += THREADS) {
            const uint32_t u = float_to_ordered(row[s]);
            if ((u & pmask) == prefix) {
                const int d = (int)((u >> shift) & 255u);
                atomicAdd(&hmass[d], exp((double)row[s] - (double)m));
                atomicAdd(&hcnt[d], 1);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double cum = 0.0;
            int chosen = -1, last = -1, cabove = 0;
            for (int d = 255; d >= 0; d--) {
                if (hcnt[d] == 0) continue;
                last = d;
                if (cum + hmass[d] >= need) {
                    chosen = d;
                    break;
                }
                cum += hmass[d];
                cabove += hcnt[d];
            }
            if (chosen < 0) {  // rounding left `need` above the remaining mass: keep everything down to the last key
                chosen = last;
                cum -= hmass[last];
                cabove -= hcnt[last];
            }
            s_need = need - cum;
            s_prefix = prefix | ((uint32_t)chosen << shift);
            s_taken_above = cabove;
        }
        __syncthreads();
        prefix = s_prefix;
        need = s_need;
        above += s_taken_above;
        pmask |= 255u << shift;
        __syncthreads();
    }
    // keys equal to the prefix: the first n_eq in entry order
    const uint32_t K = prefix;
    const int cnt_eq = hcnt[(K & 255u)];
    const double eK = exp((double)ordered_to_float(K) - (double)m);
    int n_eq = (int)ceil(need / eK);
    n_eq = n_eq < 1 ? 1 : (n_eq > cnt_eq ? cnt_eq : n_eq);
    // the entry index of the n_eq-th equal key (a scan in entry order; only when keys tie)
    if (threadIdx.x == 0) s_last_eq = (int)S;
    __syncthreads();
    if (n_eq < cnt_eq) {
        int carry = 0;
        for (int64_t base = 0; base < S; base += THREADS) {
            const int64_t s = base + threadIdx.x;
            const int eq = (s < S) && float_to_ordered(row[s]) == K;
            const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
            const int inc = warp_incl_scan(eq);
            if (lane == 31) warp_tot[warp] = inc;
            __syncthreads();
            int before = 0, tot_eq = 0;
            for (int w = 0; w < THREADS / 32; w++) {
                before += w < warp ? warp_tot[w] : 0;
                tot_eq += warp_tot[w];
            }
            if (eq && carry + before + inc == n_eq) s_last_eq = (int)s;
            carry += tot_eq;
            __syncthreads();
            if (carry >= n_eq) break;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s_prefix = K;
        if (nsize) nsize[r] = above + n_eq;
    }
    __syncthreads();
    }  // radix path
    const uint32_t K = s_prefix;
    const int64_t last_eq = s_last_eq;
    // kept bits, one atomicOr per 32-entry word of the global entry numbering
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t g0 = ((off >> 5) + warp) << 5; g0 < off + S; g0 += (int64_t)THREADS) {
        const int64_t g = g0 + lane, s = g - off;
        bool keep = false;
        if (g >= off && s < S) {
            const uint32_t u = float_to_ordered(row[s]);
            keep = u > K || (u == K && s <= last_eq);
        }
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0 && bal) atomicOr(plane + (g0 >> 5), bal);
    }
}

// One CTA per 32 consecutive 32-entry words: lane = word, warp = a group of tokens.  A thread adds
// the Lc layer words of each of its tokens into a bit-sliced counter (slice k holds bit k of every
// entry's vote count), compares the counts with theta slice by slice, and ORs the result over its
// tokens; the warps' results are ORed in shared memory and written as one byte per entry.
constexpr int VOTE_THREADS = 1024;
constexpr int VOTE_SLICES = 8;  // vote counts up to 255 layers

__global__ void __launch_bounds__(VOTE_THREADS, 2) k_golden_vote(const uint32_t *__restrict__ bits, int64_t W32, int64_t T,
                                                              int tau, int Lc, int theta, uint8_t *__restrict__ label)
{
    __shared__ uint32_t s_any[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * 32 + lane;
    if (threadIdx.x < 32) s_any[threadIdx.x] = 0u;
    __syncthreads();
    int ns = 0;
    while (ns < VOTE_SLICES && (Lc >> ns) != 0) ns++;  // slices holding counts up to Lc
    uint32_t any = 0u;
    if (w < W32 && theta <= Lc) {
        for (int i = warp; i < tau; i += VOTE_THREADS / 32) {
            const uint32_t *col = bits + (int64_t)i * Lc * W32 + w;
            uint32_t c[VOTE_SLICES];
#pragma unroll
            for (int k = 0; k < VOTE_SLICES; k++) c[k] = 0u;
            for (int l0 = 0; l0 < Lc; l0 += 4) {
                uint32_t x[4];
#pragma unroll
                for (int u = 0; u < 4; u++) x[u] = l0 + u < Lc ? __ldg(col + (int64_t)(l0 + u) * W32) : 0u;
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    uint32_t carry = x[u];
#pragma unroll
                    for (int k = 0; k < VOTE_SLICES; k++) {
                        const uint32_t t = c[k] & carry;
                        c[k] ^= carry;
                        carry = t;
                    }
                }
            }
            // count >= theta, from the most significant slice down
            uint32_t gt = 0u, eq = 0xffffffffu;
#pragma unroll
            for (int k = VOTE_SLICES - 1; k >= 0; k--) {
                if (k >= ns) continue;
                if ((theta >> k) & 1) {
                    eq &= c[k];
                } else {
                    gt |= eq & c[k];
                    eq &= ~c[k];
                }
            }
            any |= gt | eq;
        }
    }
    if (any) atomicOr(&s_any[lane], any);
    __syncthreads();
    for (int t = threadIdx.x; t < 32 * 32; t += VOTE_THREADS) {
        const int64_t g = (int64_t)blockIdx.x * 1024 + t;
        if (g < T) label[g] = (uint8_t)((s_any[t >> 5] >> (t & 31)) & 1u);
    }
}

}  // namespace golden

}  // namespace lsa
