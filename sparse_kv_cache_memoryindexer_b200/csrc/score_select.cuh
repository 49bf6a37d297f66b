// Stages 2-4a: Memory-Indexer index score, threshold, OR over the indexer layers, and the
// compaction of the fetched set (blog review "FlashMemory-DeepSeek-V4", sections 3.1 and 4.2;
// hyper.ai summary, "Method").
//
// Work unit: a tile of TILE = 128 consecutive entries of one sequence, for all L layers, so the
// OR over layers stays in registers.  A tile writes four 32-bit fetch words (one per warp);
// the compaction kernel turns them into the ascending index list of each sequence.
#pragma once
#include "common.cuh"

namespace lsa {

// tile_start[b] = sum_{b' < b} ceil(S_b' / TILE), b = 0..B.  One block; also validates offsets.
__global__ void __launch_bounds__(1024) k_tile_setup(const int64_t *__restrict__ offs, int B, int64_t T,
                                                     int *__restrict__ tile_start)
{
    __shared__ int warp_tot[32];
    __shared__ int carry;
    if (threadIdx.x == 0) {
        carry = 0;
        tile_start[0] = 0;
        if (offs[0] != 0 || offs[B] != T) flag(ERRF_OFFSETS);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < B; base += blockDim.x) {
        const int b = base + threadIdx.x;
        int n = 0;
        if (b < B) {
            int64_t S = offs[b + 1] - offs[b];
            if (S < 0) {
                flag(ERRF_OFFSETS);
                S = 0;
            }
            n = (int)((S + TILE - 1) / TILE);
        }
        int inc = warp_incl_scan(n);
        if (lane == 31) warp_tot[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int v = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            warp_tot[lane] = warp_incl_scan(v) - v;  // exclusive prefix of warp totals
        }
        __syncthreads();
        const int pos = carry + warp_tot[warp] + inc;  // inclusive position
        if (b < B) tile_start[b + 1] = pos;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = pos;
        __syncthreads();
    }
}

// SIMT index score (any dtype, d_I = D in {32, 64, 128}, n_h <= 128).  One thread per entry.
// Shared memory: q of the current layer and sequence (n_h x D fp32) and w (n_h fp32).
template <int D, int KDT, int QDT>
__global__ void __launch_bounds__(TILE) k_score_simt(const void *__restrict__ q, const float *__restrict__ w,
                                                      const void *__restrict__ K, const float *__restrict__ kscale,
                                                      const int64_t *__restrict__ offs,
                                                      const int *__restrict__ tile_start, int B, int64_t T, int L,
                                                      int n_h, float thr_logit, float *__restrict__ scores_out,
                                                      uint32_t *__restrict__ tile_mask)
{
    extern __shared__ float smem[];
    float *sq = smem;
    float *sw = smem + n_h * D;
    const int tile = blockIdx.x;
    if (tile >= tile_start[B]) return;
    const int b = seq_of_tile(tile_start, B, tile);
    const int64_t S = offs[b + 1] - offs[b];
    const int64_t s = (int64_t)(tile - tile_start[b]) * TILE + threadIdx.x;
    const bool valid = s < S;
    const int64_t row = offs[b] + s;
    bool fetched = false;
    for (int l = 0; l < L; l++) {
        __syncthreads();
        const int64_t q0 = ((int64_t)l * B + b) * n_h * D;
        for (int i = threadIdx.x; i < n_h * D; i += blockDim.x) sq[i] = load_elem<QDT>(q, q0 + i);
        for (int i = threadIdx.x; i < n_h; i += blockDim.x) sw[i] = w[((int64_t)l * B + b) * n_h + i];
        __syncthreads();
        if (!valid) continue;
        float kr[D];
        const int64_t k0 = ((int64_t)l * T + row) * D;
#pragma unroll
        for (int e = 0; e < D; e++) kr[e] = load_elem<KDT>(K, k0 + e);
        float scale = 1.f;
        if (kscale) {
            scale = kscale[(int64_t)l * T + row];
            if (!(scale >= 0.f)) flag(ERRF_SCALE);
        }
        float x = 0.f;
        for (int h = 0; h < n_h; h++) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < D; e++) dot = fmaf(sq[h * D + e], kr[e], dot);
            x = fmaf(sw[h], fmaxf(dot * scale, 0.f), x);
        }
        if (scores_out) scores_out[(int64_t)l * T + row] = 1.f / (1.f + expf(-x));
        fetched |= (x >= thr_logit);
    }
    const unsigned m = __ballot_sync(0xffffffffu, valid && fetched);
    if ((threadIdx.x & 31) == 0) tile_mask[(int64_t)tile * 4 + (threadIdx.x >> 5)] = m;
}

// Compaction (stage 4a): one block per sequence scans its tiles' fetch words in order and writes
// the ascending list of fetched entries, the count, and optionally a byte mask.
__global__ void __launch_bounds__(1024) k_compact(const uint32_t *__restrict__ tile_mask,
                                                  const int *__restrict__ tile_start,
                                                  const int64_t *__restrict__ offs, int B,
                                                  int32_t *__restrict__ idx_out, int32_t *__restrict__ count_out,
                                                  uint8_t *__restrict__ mask_out)
{
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int b = blockIdx.x;
    const int t0 = tile_start[b], t1 = tile_start[b + 1];
    const int64_t off = offs[b], S = offs[b + 1] - offs[b];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = t0; base < t1; base += blockDim.x) {
        const int t = base + threadIdx.x;
        uint4 m = make_uint4(0, 0, 0, 0);
        if (t < t1) m = *(const uint4 *)(tile_mask + (int64_t)t * 4);
        const int c = __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
        const int inc = warp_incl_scan(c);
        if (lane == 31) warp_tot[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int v = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            warp_tot[lane] = warp_incl_scan(v) - v;
        }
        __syncthreads();
        int pos = carry + warp_tot[warp] + inc - c;
        if (t < t1) {
            const int64_t s0 = (int64_t)(t - t0) * TILE;
            const uint32_t words[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int k = 0; k < 4; k++) {
                uint32_t bits = words[k];
                while (bits) {
                    const int bit = __ffs(bits) - 1;
                    bits &= bits - 1;
                    idx_out[off + pos++] = (int32_t)(s0 + 32 * k + bit);
                }
            }
            if (mask_out) {
                for (int e = 0; e < TILE && s0 + e < S; e++)
                    mask_out[off + s0 + e] = (uint8_t)((words[e >> 5] >> (e & 31)) & 1u);
            }
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = pos;  // last thread's running end = block total
        __syncthreads();
    }
    if (threadIdx.x == 0) count_out[b] = carry;
}

}  // namespace lsa
