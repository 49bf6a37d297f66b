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

}  // namespace lsa
