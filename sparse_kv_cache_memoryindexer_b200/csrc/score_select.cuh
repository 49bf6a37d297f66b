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
// Run by every thread of one block (any size that is a multiple of 32).
__device__ __forceinline__ void tile_setup_body(const int64_t *__restrict__ offs, int B, int64_t T,
                                                int *__restrict__ tile_start, int *__restrict__ chunk_start,
                                                int32_t *__restrict__ count_out)
{
    __shared__ int warp_tot[32];
    __shared__ int carry;
    if (threadIdx.x == 0) {
        carry = 0;
        tile_start[0] = 0;
        if (offs[0] != 0 || offs[B] != T) flag(ERRF_OFFSETS);
    }
    __syncthreads();
    // chunk_start: exclusive prefix of ceil(tiles_b / COMPACT_TILES), the compaction's CTAs per
    // sequence; an empty sequence has none, so its count is written here.
    {
        __shared__ int wt[32];
        __shared__ int ccarry;
        if (threadIdx.x == 0) {
            ccarry = 0;
            chunk_start[0] = 0;
        }
        __syncthreads();
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        for (int base = 0; base < B; base += blockDim.x) {
            const int b = base + threadIdx.x;
            int n = 0;
            if (b < B) {
                int64_t S = offs[b + 1] - offs[b];
                if (S < 0) S = 0;
                if (S == 0) count_out[b] = 0;
                const int64_t tiles = (S + TILE - 1) / TILE;
                n = (int)((tiles + COMPACT_TILES - 1) / COMPACT_TILES);
            }
            int inc = warp_incl_scan(n);
            if (lane == 31) wt[warp] = inc;
            __syncthreads();
            if (warp == 0) {
                int v = lane < (int)(blockDim.x >> 5) ? wt[lane] : 0;
                wt[lane] = warp_incl_scan(v) - v;
            }
            __syncthreads();
            const int pos = ccarry + wt[warp] + inc;
            if (b < B) chunk_start[b + 1] = pos;
            __syncthreads();
            if (threadIdx.x == blockDim.x - 1) ccarry = pos;
            __syncthreads();
        }
    }
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

__global__ void __launch_bounds__(1024) k_tile_setup(const int64_t *__restrict__ offs, int B, int64_t T,
                                                     int *__restrict__ tile_start, int *__restrict__ chunk_start,
                                                     int32_t *__restrict__ count_out)
{
    tile_setup_body(offs, B, T, tile_start, chunk_start, count_out);
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

// Compaction (stage 4a): the ascending list of fetched entries of each sequence from the fetch
// words, the count, and optionally a byte mask.  One CTA per chunk of COMPACT_TILES tiles of one
// sequence: its sequence-local start is the number of fetched entries in the sequence's earlier
// tiles (summed from their fetch words, a few KB read from L2), its tiles' starts come from a block
// scan, and each of its 32 warps writes the entries of 8 tiles with consecutive lanes on
// consecutive list positions.
constexpr int COMPACT_SMEM_B = 1024;  // sequences whose chunk starts k_compact keeps in shared memory
__device__ __forceinline__ int popc4(uint4 m) { return __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w); }

constexpr int COMPACT_THREADS = 4 * COMPACT_TILES;  // the chunk's tiles counted by the first COMPACT_TILES
                                                    // threads, written by all warps (8 tiles each)

__global__ void __launch_bounds__(COMPACT_THREADS, 2) k_compact(const uint32_t *__restrict__ tile_mask,
                                                            const int *__restrict__ tile_start,
                                                            const int *__restrict__ chunk_start,
                                                            const int64_t *__restrict__ offs, int B,
                                                            int32_t *__restrict__ idx_out, int32_t *__restrict__ count_out,
                                                            uint8_t *__restrict__ mask_out)
{
    constexpr int NW = COMPACT_THREADS / 32, TPW = COMPACT_TILES / NW;  // warps, tiles written per warp
    __shared__ int red[NW];
    __shared__ int scan[COMPACT_TILES / 32];
    __shared__ int s_cs[COMPACT_SMEM_B + 1];
    __shared__ uint4 s_mask[COMPACT_TILES];
    __shared__ int s_pos[COMPACT_TILES];
    const int c = blockIdx.x;
    // the sequence of chunk c: largest b with chunk_start[b] <= c (the chunk starts read in one
    // coalesced pass into shared memory when there are few sequences, not one load per search step)
    const bool in_smem = B <= COMPACT_SMEM_B;
    if (in_smem) {
        for (int t = threadIdx.x; t <= B; t += COMPACT_THREADS) s_cs[t] = chunk_start[t];
        __syncthreads();
    }
    const int *cs = in_smem ? s_cs : chunk_start;
    if (c >= cs[B]) return;
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cs[mid] <= c) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = tile_start[b], t1 = tile_start[b + 1];
    const int ci = c - chunk_start[b];
    const int ct0 = t0 + ci * COMPACT_TILES, ct1 = min(t1, ct0 + COMPACT_TILES);
    const int64_t off = offs[b], S = offs[b + 1] - off;
    // fetched entries before this chunk
    int part = 0;
    for (int t = t0 + threadIdx.x; t < ct0; t += COMPACT_THREADS) part += popc4(*(const uint4 *)(tile_mask + (int64_t)t * 4));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[warp] = part;
    // this chunk: one tile per thread of the first COMPACT_TILES
    const int t = ct0 + threadIdx.x;
    uint4 m = make_uint4(0, 0, 0, 0);
    if (threadIdx.x < COMPACT_TILES && t < ct1) m = *(const uint4 *)(tile_mask + (int64_t)t * 4);
    const int cnt = popc4(m);
    const int inc = warp_incl_scan(cnt);
    if (lane == 31 && warp < COMPACT_TILES / 32) scan[warp] = inc;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < NW; w++) base += red[w];
    if (threadIdx.x < COMPACT_TILES) {
        int before = 0;
#pragma unroll
        for (int w = 0; w < COMPACT_TILES / 32; w++) {
            before += w < warp ? scan[w] : 0;
            total += scan[w];
        }
        s_mask[threadIdx.x] = m;
        s_pos[threadIdx.x] = base + before + inc - cnt;  // list position of this tile's first entry
        if (ct1 == t1 && threadIdx.x == 0) count_out[b] = base + total;
    }
    __syncthreads();
    // coalesced writes: warp w walks tiles w TPW .. w TPW + TPW - 1 of the chunk; the mask goes out as
    // 4 bytes per lane when the sequence's bytes start on a 4-byte boundary
    const bool mask_words = mask_out && (((uintptr_t)(mask_out + off)) & 3u) == 0;
    const int nj = max(0, min(TPW, ct1 - (ct0 + warp * TPW)));  // this warp's tiles
#pragma unroll 2
    for (int j = 0; j < nj; j++) {
        const int jt = warp * TPW + j;  // tile within the chunk
        const uint4 mw = s_mask[jt];
        int p = s_pos[jt];
        const int64_t s0 = (int64_t)(ct0 + jt - t0) * TILE;
        const uint32_t below = (1u << lane) - 1u;
        const uint32_t words[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const uint32_t wk = words[k];
            if ((wk >> lane) & 1u) idx_out[off + p + __popc(wk & below)] = (int32_t)(s0 + 32 * k + lane);
            p += __popc(wk);
            if (mask_out && !mask_words && s0 + 32 * k + lane < S)
                mask_out[off + s0 + 32 * k + lane] = (uint8_t)((wk >> lane) & 1u);
        }
        if (mask_words) {
            // lane: entries 4 lane .. 4 lane + 3 of the tile (bits 4 (lane % 8) .. of word lane / 8)
            const uint32_t wl = lane < 8 ? mw.x : (lane < 16 ? mw.y : (lane < 24 ? mw.z : mw.w));
            const uint32_t nib = (wl >> (4 * (lane & 7))) & 0xFu;
            const uint32_t bytes = (nib & 1u) | ((nib & 2u) << 7) | ((nib & 4u) << 14) | ((nib & 8u) << 21);
            const int64_t e = s0 + 4 * lane;
            if (e + 3 < S) {
                *(uint32_t *)(mask_out + off + e) = bytes;
            } else {
#pragma unroll
                for (int q = 0; q < 4; q++)
                    if (e + q < S) mask_out[off + e + q] = (uint8_t)((bytes >> (8 * q)) & 1u);
            }
        }
    }
}

}  // namespace lsa
