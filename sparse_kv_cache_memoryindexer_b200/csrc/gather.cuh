// Stage 4b: fetch of C^MemComp from the CPU cold pool into the GPU hot buffer (hyper.ai
// summary, "Method"; blog review section 3), plus the device-side gather of the matching
// index keys of one layer for the decode-step Lightning Indexer.
//
// The pool is mapped page-locked host memory: the kernel reads it directly over the host link
// (zero-copy), one warp per row, 16 bytes per lane, several rows in flight per warp so that
// enough read requests are outstanding to cover the link latency.  E4M3 keys are decoded
// exactly to bf16 on the way into the hot key buffer (their scales are copied unchanged), so
// the decode-step tensor-core kernel reads bf16 operands directly.
#pragma once
#include "common.cuh"

namespace lsa {

constexpr int GATHER_ROWS_PER_WARP = 4;
constexpr int GATHER_MAX_CHUNKS = 4;  // row_bytes <= 4 * 32 * 16 = 2048 per in-flight row

// 16 E4M3 codes -> 16 bf16 values (exact: every E4M3 value is a bf16 value).
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 v, uint4 &lo, uint4 &hi)
{
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; k++) {
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            const uint16_t two = (uint16_t)(in[k] >> (16 * hh));
            __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
            const float2 f = __half22float2(__half2(h));
            __nv_bfloat162 b = __float22bfloat162_rn(f);
            o[2 * k + hh] = *reinterpret_cast<uint32_t *>(&b);
        }
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// krow16: 16-byte chunks of one source key row; kconv: source rows are E4M3, destination rows bf16.
__global__ void __launch_bounds__(256) k_gather(const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                                const int64_t *__restrict__ offs,
                                                const uint8_t *__restrict__ pool, int row16,
                                                uint8_t *__restrict__ hot_kv,
                                                const uint8_t *__restrict__ Ksel, const float *__restrict__ ksc,
                                                int krow16, bool kconv, uint8_t *__restrict__ hotK,
                                                float *__restrict__ hotsc)
{
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    int F = count[b];
    if (F < 0 || F > S) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(ERRF_COUNT);
        F = F < 0 ? 0 : (int)S;
    }
    const int warps = blockDim.x >> 5;
    const int64_t wid = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5);
    const int64_t wstride = (int64_t)gridDim.x * warps;
    const int64_t rb = (int64_t)row16 * 16, kb = (int64_t)krow16 * 16, kbo = kconv ? 2 * kb : kb;
    for (int64_t j0 = wid * GATHER_ROWS_PER_WARP; j0 < F; j0 += wstride * GATHER_ROWS_PER_WARP) {
        int64_t src[GATHER_ROWS_PER_WARP];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++) {
            src[r] = -1;
            const int64_t j = j0 + r;
            if (j < F) {
                const int s = __ldg(idx + off + j);
                if (s >= 0 && s < S) src[r] = off + s;
                else if (lane == 0) flag(ERRF_INDEX);
            }
        }
        uint4 v[GATHER_ROWS_PER_WARP][GATHER_MAX_CHUNKS];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < GATHER_MAX_CHUNKS; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) v[r][c] = ld_stream16(pool + src[r] * rb + (int64_t)ch * 16);
            }
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < GATHER_MAX_CHUNKS; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16)
                    *(uint4 *)(hot_kv + (off + j0 + r) * rb + (int64_t)ch * 16) = v[r][c];
            }
        if (Ksel) {
#pragma unroll
            for (int r = 0; r < GATHER_ROWS_PER_WARP; r++) {
                if (src[r] < 0) continue;
                for (int ch = lane; ch < krow16; ch += 32) {
                    const uint4 v = __ldg((const uint4 *)(Ksel + src[r] * kb + (int64_t)ch * 16));
                    if (kconv) {
                        uint4 lo, hi;
                        e4m3x16_to_bf16(v, lo, hi);
                        uint4 *d = (uint4 *)(hotK + (off + j0 + r) * kbo + (int64_t)ch * 32);
                        d[0] = lo;
                        d[1] = hi;
                    } else {
                        *(uint4 *)(hotK + (off + j0 + r) * kbo + (int64_t)ch * 16) = v;
                    }
                }
                if (ksc && lane == 0) hotsc[off + j0 + r] = __ldg(ksc + src[r]);
            }
        }
    }
}

}  // namespace lsa
