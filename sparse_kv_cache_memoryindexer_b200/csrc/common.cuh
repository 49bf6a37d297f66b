// Shared device helpers of the LSA indexer library (one translation unit: lsa.cu includes
// every kernel header, so the device error word below needs no relocatable device code).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

enum : int { DT_F32 = 0, DT_BF16 = 1, DT_FP8 = 2 };

// Entries per score tile: one TMEM lane / one thread per entry.
constexpr int TILE = 128;
constexpr int COMPACT_TILES = 256;  // tiles per CTA of the compaction (one per thread)

// Bits of the device error word (read and cleared by lsa_check_device).
enum : unsigned {
    ERRF_OFFSETS = 1u,  // seq_offsets not a non-decreasing prefix ending at total_S
    ERRF_INDEX = 2u,    // a fetched entry index outside its sequence
    ERRF_COUNT = 4u,    // a fetched count outside [0, S_b]
    ERRF_SCALE = 8u,    // a key scale that is negative or NaN
    ERRF_TIMEOUT = 16u, // a bounded wait inside a pipelined kernel gave up
};

// One word per device (per loaded copy of this library).
static __device__ unsigned int g_err_word;

__device__ __forceinline__ void flag(unsigned bits) { atomicOr(&g_err_word, bits); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }

__device__ __forceinline__ float e4m3_to_float(uint8_t c)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

template <int DT>
__device__ __forceinline__ float load_elem(const void *base, int64_t i)
{
    if constexpr (DT == DT_F32) return __ldg((const float *)base + i);
    else if constexpr (DT == DT_BF16) return bf16_bits_to_float(__ldg((const unsigned short *)base + i));
    else return e4m3_to_float(__ldg((const unsigned char *)base + i));
}

template <int DT>
__device__ __forceinline__ void store_elem(void *base, int64_t i, float v)
{
    if constexpr (DT == DT_F32) ((float *)base)[i] = v;
    else ((__nv_bfloat16 *)base)[i] = __float2bfloat16_rn(v);
}

// Order-preserving map fp32 -> uint32 (larger float <=> larger key) and back.
__device__ __forceinline__ uint32_t float_to_ordered(float f)
{
    uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(uint32_t u)
{
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

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

// Sequence owning global tile t: largest b with tile_start[b] <= t (tile_start has B+1 entries).
__device__ __forceinline__ int seq_of_tile(const int *tile_start, int B, int t)
{
    int lo = 0, hi = B;  // invariant: tile_start[lo] <= t < tile_start[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(tile_start + mid) <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

// 16-byte read that does not allocate in L1 (streamed data, including mapped host memory).
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ int warp_incl_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
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
