// Stage 1: Memory-Indexer projections c^Q = h W^DQ, q = c^Q W^IUQ, w = h W^w
// (blog review "FlashMemory-DeepSeek-V4", section 3.1).
//
// The weights are stored transposed (row = one output, the layout of a linear layer), so every
// output is a dot product of an input row with one contiguous weight row.  The weight stream
// dominates (B <= 64 inputs against d x r weights), so one warp owns one output row and streams
// it once per group of 16 inputs with 16-byte loads; the inputs stay in L1/L2.
#pragma once
#include "common.cuh"

namespace lsa {

constexpr int PROJ_BGROUP = 16;

template <int DT>
__device__ __forceinline__ void load8(const void *base, int64_t i, float (&v)[8])
{
    if constexpr (DT == DT_F32) {
        const float4 *p = (const float4 *)((const float *)base + i);
        float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        uint4 u = __ldg((const uint4 *)((const unsigned short *)base + i));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            v[2 * k] = __uint_as_float(w[k] << 16);
            v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
}

// out[l][b][o] = sum_i x[l][b][i] * W[l][o][i], stored in ODT (rounded to nearest even).
// IN must be a multiple of 8; x and W 16-byte aligned.
template <int DT, int ODT>
__global__ void __launch_bounds__(256) k_rowdot(const void *__restrict__ x, const void *__restrict__ W,
                                                void *__restrict__ out, int B, int IN, int OUT)
{
    const int lane = threadIdx.x & 31;
    const int o = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int l = blockIdx.y;
    if (o >= OUT) return;
    const int64_t wrow = ((int64_t)l * OUT + o) * IN;
    for (int b0 = 0; b0 < B; b0 += PROJ_BGROUP) {
        float acc[PROJ_BGROUP];
#pragma unroll
        for (int k = 0; k < PROJ_BGROUP; k++) acc[k] = 0.f;
        for (int i = lane * 8; i < IN; i += 256) {
            float wv[8];
            load8<DT>(W, wrow + i, wv);
#pragma unroll
            for (int k = 0; k < PROJ_BGROUP; k++) {
                if (b0 + k < B) {
                    float xv[8];
                    load8<DT>(x, ((int64_t)l * B + b0 + k) * IN + i, xv);
#pragma unroll
                    for (int e = 0; e < 8; e++) acc[k] = fmaf(xv[e], wv[e], acc[k]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < PROJ_BGROUP; k++) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
        }
        if (lane < PROJ_BGROUP && b0 + lane < B) {
            float v = acc[0];
#pragma unroll
            for (int k = 1; k < PROJ_BGROUP; k++)
                if (lane == k) v = acc[k];
            store_elem<ODT>(out, ((int64_t)l * B + b0 + lane) * OUT + o, v);
        }
    }
}

}  // namespace lsa
