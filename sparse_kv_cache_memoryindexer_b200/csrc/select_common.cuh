// Device helpers shared by the Top-k selects and the golden-label nucleus: the select's score
// buckets and a block-wide bitonic sort of 64-bit keys.
#pragma once
#include "common.cuh"

namespace lsa {

// Buckets of a Top-k select.  The order-preserving score keys of one query lie in [umin, umax],
// scores [ymin, ymax]; bucket(u) = floor((y - ymin) * SEL_NB / (ymax - ymin)) clamped to
// [0, SEL_NB), linear in the score so that the buckets follow the spread of the query's own scores
// (a split on the bits of the key would put the scores of one binade into eight buckets).  It is
// non-decreasing in the key (fp32 subtraction and multiplication are monotone), and degenerate
// ranges (a single value, an infinite span) put every finite score into bucket 0.  A NaN goes to
// the end its key sorts to.
constexpr int SEL_NB = 4096;
struct SelRange {
    float ymin, scale;
};
__device__ __forceinline__ SelRange sel_range(uint32_t umin, uint32_t umax)
{
    SelRange r;
    r.ymin = ordered_to_float(umin);
    const float span = ordered_to_float(umax) - r.ymin;
    r.scale = span > 0.f ? (float)SEL_NB / span : 0.f;
    return r;
}
__device__ __forceinline__ uint32_t sel_bucket(const SelRange &r, uint32_t u)
{
    const float y = ordered_to_float(u);
    if (y != y) return (u & 0x80000000u) ? (uint32_t)(SEL_NB - 1) : 0u;
    const float t = (y - r.ymin) * r.scale;
    return t >= (float)(SEL_NB - 1) ? (uint32_t)(SEL_NB - 1) : (t > 0.f ? (uint32_t)t : 0u);
}
// The same bucket from the score itself: sel_bucket(r, float_to_ordered(y)) (a NaN's key sorts to
// the top when its sign bit is clear, to the bottom otherwise).
__device__ __forceinline__ uint32_t sel_bucket_f(const SelRange &r, float y)
{
    if (y != y) return signbit(y) ? 0u : (uint32_t)(SEL_NB - 1);
    const float t = (y - r.ymin) * r.scale;
    return t >= (float)(SEL_NB - 1) ? (uint32_t)(SEL_NB - 1) : (t > 0.f ? (uint32_t)t : 0u);
}
// The range from the smallest and largest scores that are not NaN (none: every score in bucket 0
// or at its NaN end).
__device__ __forceinline__ SelRange sel_range_f(float ymin, float ymax)
{
    SelRange r;
    r.ymin = ymin;
    const float span = ymax - ymin;
    r.scale = span > 0.f ? (float)SEL_NB / span : 0.f;
    return r;
}

// Descending bitonic sort of n 64-bit keys in shared memory by the whole block (n a power of two,
// at least 64; blockDim.x a multiple of 32).  Strides of 64 and more exchange through shared memory
// with a barrier each; for the strides below 64 every warp takes 64 consecutive keys into registers
// (two per lane) and finishes them with shuffles, so a sort of 2,048 keys needs 26 barriers instead
// of 66.  Starts and ends with a barrier.
__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m)
{
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ void block_sort_desc_u64(unsigned long long *v, int n)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride >= 64; stride >>= 1) {
            for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
                const int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = v[lo], c = v[hi];
                if ((a < c) == desc) {
                    v[lo] = c;
                    v[hi] = a;
                }
            }
            __syncthreads();
        }
        for (int blk = warp; blk < n / 64; blk += nw) {
            const int e0 = blk * 64 + 2 * lane;  // this lane's keys e0, e0 + 1
            unsigned long long a = v[e0], b = v[e0 + 1];
            const bool desc = (e0 & size) == 0;  // the same for e0 + 1 and every partner below 64
            for (int stride = (size >> 1) < 32 ? (size >> 1) : 32; stride >= 2; stride >>= 1) {
                const int m = stride >> 1;               // partner lane (keys e0 ^ stride)
                const bool low = (e0 & stride) == 0;     // this lane holds the lower index of the pair
                const unsigned long long pa = shfl_xor_u64(a, m), pb = shfl_xor_u64(b, m);
                const bool keep_max = low == desc;
                a = keep_max ? (a > pa ? a : pa) : (a < pa ? a : pa);
                b = keep_max ? (b > pb ? b : pb) : (b < pb ? b : pb);
            }
            if ((a < b) == desc) {  // stride 1: the lane's own pair
                const unsigned long long x = a;
                a = b;
                b = x;
            }
            v[e0] = a;
            v[e0 + 1] = b;
        }
        __syncthreads();
    }
}


// Block-wide minimum and maximum of one key per thread (threads without a key pass 0xFFFFFFFF and
// 0); *lo / *hi: shared words, written by this call.  Starts and ends with a barrier.
__device__ __forceinline__ void block_min_max(uint32_t vmin, uint32_t vmax, uint32_t *lo, uint32_t *hi)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        *lo = 0xFFFFFFFFu;
        *hi = 0u;
    }
    __syncthreads();
    vmin = __reduce_min_sync(0xffffffffu, vmin);
    vmax = __reduce_max_sync(0xffffffffu, vmax);
    if ((threadIdx.x & 31) == 0) {
        atomicMin(lo, vmin);
        atomicMax(hi, vmax);
    }
    __syncthreads();
}

// The n distinct 64-bit keys of v (any order; blockDim.x = 1024) put in descending order without a
// sort of all of them: SEL_NB buckets linear in the score (key >> 32) over the keys' own range, the
// keys scattered into their buckets' segments (higher buckets first), and a key's position = its
// segment's start + the keys of its segment above it.  When a bucket holds more than max_seg keys,
// the keys are sorted instead (bitonic, v padded to npow2 >= n with zeros; npow2 a power of two
// >= 64).  emit(position, key) is called once per key.  tmp: n keys of shared memory; cnt: SEL_NB
// ints of shared memory.  Ends with a barrier.
template <typename Emit>
__device__ __forceinline__ void order_desc(unsigned long long *v, int n, int npow2, unsigned long long *tmp, int *cnt,
                                           int max_seg, Emit emit)
{
    __shared__ uint32_t s_lo, s_hi;
    __shared__ int s_mx;
    __shared__ int s_wt[32];
    constexpr int PER = SEL_NB / 1024;
    uint32_t tmin = 0xFFFFFFFFu, tmax = 0u;
    for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const uint32_t u = (uint32_t)(v[t] >> 32);
        tmin = min(tmin, u);
        tmax = max(tmax, u);
    }
    for (int t = threadIdx.x; t < SEL_NB; t += blockDim.x) cnt[t] = 0;
    if (threadIdx.x == 0) s_mx = 0;
    block_min_max(tmin, tmax, &s_lo, &s_hi);
    const SelRange rg = sel_range(s_lo, s_hi);
    for (int t = threadIdx.x; t < n; t += blockDim.x) atomicAdd(&cnt[sel_bucket(rg, (uint32_t)(v[t] >> 32))], 1);
    __syncthreads();
    {
        // exclusive counts from the top: thread t owns buckets SEL_NB - PER (t + 1) .. SEL_NB - PER t - 1
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        const int hi = SEL_NB - PER * (int)threadIdx.x;
        int c[PER], sum = 0, mx = 0;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            c[i] = cnt[hi - 1 - i];
            sum += c[i];
            mx = max(mx, c[i]);
        }
        const int inc = warp_incl_scan(sum);
        if (lane == 31) s_wt[warp] = inc;
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) atomicMax(&s_mx, mx);
        __syncthreads();
        if (warp == 0) {
            const int x = lane < (int)(blockDim.x >> 5) ? s_wt[lane] : 0;
            s_wt[lane] = warp_incl_scan(x) - x;
        }
        __syncthreads();
        int run = s_wt[warp] + inc - sum;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            cnt[hi - 1 - i] = run;
            run += c[i];
        }
    }
    __syncthreads();
    if (s_mx <= max_seg) {
        for (int t = threadIdx.x; t < n; t += blockDim.x) {
            const unsigned long long x = v[t];
            tmp[atomicAdd(&cnt[sel_bucket(rg, (uint32_t)(x >> 32))], 1)] = x;
        }
        __syncthreads();
        // cnt[b] is now the end of bucket b's segment, and the end of bucket b + 1's is b's start
        for (int t = threadIdx.x; t < n; t += blockDim.x) {
            const unsigned long long x = tmp[t];
            const uint32_t b = sel_bucket(rg, (uint32_t)(x >> 32));
            const int lo = b + 1 < (uint32_t)SEL_NB ? cnt[b + 1] : 0, hi = cnt[b];
            int r = lo;
            for (int i = lo; i < hi; i++) r += tmp[i] > x;
            emit(r, x);
        }
    } else {
        for (int t = n + threadIdx.x; t < npow2; t += blockDim.x) v[t] = 0ull;
        block_sort_desc_u64(v, npow2);
        for (int t = threadIdx.x; t < n; t += blockDim.x) emit(t, v[t]);
    }
    __syncthreads();
}

}  // namespace lsa
