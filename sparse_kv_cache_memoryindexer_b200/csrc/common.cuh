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

}  // namespace lsa
