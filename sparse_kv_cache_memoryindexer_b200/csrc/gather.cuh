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
// The launches that read the host pool (k_gather_rows, k_incr_fetch) run beside the Lightning Top-k:
// a few SMs with many reads in flight each.  A warp keeps GATHER_ROWS_PER_WARP rows in flight, so
// 16 CTAs of 1024 threads hold 2 MB of 1 KB rows in flight, enough for the host link, on 16 SMs;
// a CTA-per-SM spread of the same reads slowed the Top-k beside it several times over (the host
// reads in flight hold every SM's load path).
constexpr int GATHER_LINK_CTAS = 16;
template <int CH>
constexpr int link_threads() { return CH <= 2 ? 1024 : 512; }  // 64 or 128 registers a thread
constexpr int GATHER_ROWS_MAX_B = 8192; // sequences of the rows-only launch (shared prefix of B + 1 ints)

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

// Shared-memory exclusive prefix pre[0..B] of the counts (clamped to [0, S_b], a bad count flagged),
// built by one CTA of any size up to 1024 threads (warp_sum: 32 ints of shared memory); returns the
// total.  Every thread calls it.
__device__ __forceinline__ int block_count_prefix(const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                  int B, int *pre, int *warp_sum)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nt = blockDim.x, nw = nt >> 5;
    auto clamped = [&](int b) {
        const int64_t S = offs[b + 1] - offs[b];
        int F = count[b];
        if (F < 0 || F > S) {
            if (blockIdx.x == 0) flag(ERRF_COUNT);
            F = F < 0 ? 0 : (int)S;
        }
        return F;
    };
    const int per = (B + nt - 1) / nt;
    const int lo = min(B, (int)threadIdx.x * per), hi = min(B, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; b++) sum += clamped(b);
    const int inc = warp_incl_scan(sum);
    if (lane == 31) warp_sum[warp] = inc;
    __syncthreads();
    int base = 0, total = 0;
    for (int k = 0; k < nw; k++) {
        base += k < warp ? warp_sum[k] : 0;
        total += warp_sum[k];
    }
    int run = base + inc - sum;
    for (int b = lo; b < hi; b++) {
        pre[b] = run;
        run += clamped(b);
    }
    if (threadIdx.x == 0) pre[B] = total;
    __syncthreads();
    return total;
}

// The sequence of fetched-row number g (g < pre[B]): the largest b with pre[b] <= g, which is never
// an empty sequence.
__device__ __forceinline__ int sequence_of_row(const int *pre, int B, int64_t g)
{
    int a = 0, z = B - 1;
    while (a < z) {
        const int mid = (a + z + 1) >> 1;
        if (pre[mid] <= g) a = mid;
        else z = mid - 1;
    }
    return a;
}

// Keys only (device to device): every 16-byte chunk of every fetched key row is one work unit, all
// rows of all sequences numbered in one range (prefix of the counts in shared memory, as in
// k_gather_rows), so the launch is balanced and every load is a full coalesced chunk.  E4M3 chunks
// are decoded to 32 bytes of bf16; chunk 0 of a row also copies the row's scale.
__global__ void __launch_bounds__(128) k_gather_keys(const int32_t *__restrict__ idx,
                                                     const int32_t *__restrict__ count,
                                                     const int64_t *__restrict__ offs, int B,
                                                     const uint8_t *__restrict__ Ksel, const float *__restrict__ ksc,
                                                     int krow16, bool kconv, uint8_t *__restrict__ hotK,
                                                     float *__restrict__ hotsc)
{
    extern __shared__ int pre[];
    __shared__ int warp_sum[32];
    const int total = block_count_prefix(count, offs, B, pre, warp_sum);
    const int64_t kb = (int64_t)krow16 * 16, kbo = kconv ? 2 * kb : kb;
    const int64_t units = (int64_t)total * krow16;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = u / krow16;
        const int ch = (int)(u - g * krow16);
        const int b = sequence_of_row(pre, B, g);
        const int64_t off = offs[b], S = offs[b + 1] - off;
        const int64_t j = g - pre[b];
        const int s = __ldg(idx + off + j);
        if (s < 0 || s >= S) {
            if (ch == 0) flag(ERRF_INDEX);
            continue;
        }
        const int64_t src = off + s, dst = off + j;
        const uint4 v = __ldg((const uint4 *)(Ksel + src * kb + (int64_t)ch * 16));
        if (kconv) {
            uint4 lo, hi;
            e4m3x16_to_bf16(v, lo, hi);
            uint4 *d = (uint4 *)(hotK + dst * kbo + (int64_t)ch * 32);
            d[0] = lo;
            d[1] = hi;
        } else {
            *(uint4 *)(hotK + dst * kbo + (int64_t)ch * 16) = v;
        }
        if (ksc && ch == 0) hotsc[dst] = __ldg(ksc + src);
    }
}

// Rows only, for a launch that runs beside other kernels: GATHER_LINK_CTAS fat CTAs, every fetched
// row of every sequence numbered in one range so that ragged counts cannot leave most warps idle.
// Each CTA first builds the exclusive prefix pre[0..B] of the counts in shared memory ((B + 1)
// ints), then warp w of the W warps of the launch takes rows g = 4 (w + i W) .. + 3 and finds the
// sequence of g by binary search in pre.
template <int CH>  // 16-byte chunks per lane and row (row_bytes <= CH * 512)
__global__ void __launch_bounds__(link_threads<CH>()) k_gather_rows(const int32_t *__restrict__ idx,
                                                     const int32_t *__restrict__ count,
                                                     const int64_t *__restrict__ offs, int B,
                                                     const uint8_t *__restrict__ pool, int row16,
                                                     uint8_t *__restrict__ hot_kv)
{
    extern __shared__ int pre[];
    __shared__ int warp_sum[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int total = block_count_prefix(count, offs, B, pre, warp_sum);

    const int64_t rb = (int64_t)row16 * 16;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t g0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + warp) * GATHER_ROWS_PER_WARP; g0 < total;
         g0 += wstride * GATHER_ROWS_PER_WARP) {
        int64_t src[GATHER_ROWS_PER_WARP], dst[GATHER_ROWS_PER_WARP];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++) {
            src[r] = -1;
            dst[r] = 0;
            const int64_t g = g0 + r;
            if (g < total) {
                const int a = sequence_of_row(pre, B, g);
                const int64_t off = offs[a], S = offs[a + 1] - off;
                const int64_t j = g - pre[a];
                const int s = __ldg(idx + off + j);
                if (s >= 0 && s < S) {
                    src[r] = off + s;
                    dst[r] = off + j;
                } else if (lane == 0) {
                    flag(ERRF_INDEX);
                }
            }
        }
        uint4 v[GATHER_ROWS_PER_WARP][CH];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) v[r][c] = ld_stream16(pool + src[r] * rb + (int64_t)ch * 16);
            }
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) *(uint4 *)(hot_kv + dst[r] * rb + (int64_t)ch * 16) = v[r][c];
            }
    }
}

// ------------------------------------------------------------------ incremental fetch
// The hot buffer of the previous window (rows of C_{t-tau}, at that window's offsets) stays
// resident; the new window's buffer gets the rows of C_t: rows in both sets by a device copy, only
// C_t \ C_{t-tau} over the host link.  Sequences keep their entry numbering between windows (they
// may grow).  Three launches, all over the new fetched rows numbered in one range:
//   k_incr_map    one thread per row: look the entry up in the previous (ascending) list of its
//                 sequence; map[slot] = previous slot, or -1 and the row number appended to miss[]
//   k_incr_copy   one warp per row with a previous slot (device copy), several rows in flight
//   k_incr_fetch  the link launch over miss[0 .. *nmiss): as k_gather_rows
// A previous list that is not ascending only costs host reads (a missed lookup fetches the row).

__device__ __forceinline__ int prev_count_clamped(const int32_t *pcount, const int64_t *poffs, int b)
{
    const int64_t pS = poffs[b + 1] - poffs[b];
    int F = pcount[b];
    if (F < 0 || F > pS) {
        flag(ERRF_COUNT);
        F = F < 0 ? 0 : (int)pS;
    }
    return F;
}

__global__ void __launch_bounds__(128) k_incr_map(const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                                  const int64_t *__restrict__ offs, int B,
                                                  const int32_t *__restrict__ pidx, const int32_t *__restrict__ pcount,
                                                  const int64_t *__restrict__ poffs, int32_t *__restrict__ map,
                                                  int32_t *__restrict__ miss, int *__restrict__ nmiss)
{
    extern __shared__ int pre[];
    __shared__ int warp_sum[32];
    const int total = block_count_prefix(count, offs, B, pre, warp_sum);
    const int lane = threadIdx.x & 31;
    // every thread of a warp runs the same number of iterations (the ballot below needs them all)
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); g0 < total; g0 += stride) {
        const int64_t g = g0 + lane;
        bool missed = false;
        if (g < total) {
            const int b = sequence_of_row(pre, B, g);
            const int64_t off = offs[b], S = offs[b + 1] - off, j = g - pre[b];
            const int s = __ldg(idx + off + j);
            int slot = -1;
            if (s < 0 || s >= S) {
                flag(ERRF_INDEX);
            } else {
                const int64_t poff = poffs[b];
                int lo = 0, hi = prev_count_clamped(pcount, poffs, b);  // lower bound of s in the previous list
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (__ldg(pidx + poff + mid) < s) lo = mid + 1;
                    else hi = mid;
                }
                const int pc = prev_count_clamped(pcount, poffs, b);
                if (lo < pc && __ldg(pidx + poff + lo) == s) slot = lo;
                else missed = true;
            }
            map[off + j] = slot;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, missed);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(nmiss, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (missed) miss[base + __popc(bal & ((1u << lane) - 1))] = (int32_t)g;
    }
}

template <int CH>  // 16-byte chunks per lane and row (row_bytes <= CH * 512)
__global__ void __launch_bounds__(256) k_incr_copy(const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                   int B, const int64_t *__restrict__ poffs,
                                                   const int32_t *__restrict__ map, const uint8_t *__restrict__ prev_hot,
                                                   int row16, uint8_t *__restrict__ hot)
{
    extern __shared__ int pre[];
    __shared__ int warp_sum[32];
    const int total = block_count_prefix(count, offs, B, pre, warp_sum);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t rb = (int64_t)row16 * 16;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
    // one warp per row, GATHER_ROWS_PER_WARP rows in flight per warp
    for (int64_t g0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + warp) * GATHER_ROWS_PER_WARP; g0 < total;
         g0 += wstride * GATHER_ROWS_PER_WARP) {
        int64_t src[GATHER_ROWS_PER_WARP], dst[GATHER_ROWS_PER_WARP];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++) {
            src[r] = -1;
            dst[r] = 0;
            const int64_t g = g0 + r;
            if (g < total) {
                const int b = sequence_of_row(pre, B, g);
                const int64_t slot = offs[b] + (g - pre[b]);
                const int m = map[slot];
                if (m >= 0) {
                    src[r] = poffs[b] + m;
                    dst[r] = slot;
                }
            }
        }
        uint4 v[GATHER_ROWS_PER_WARP][CH];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) v[r][c] = __ldg((const uint4 *)(prev_hot + src[r] * rb + (int64_t)ch * 16));
            }
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) *(uint4 *)(hot + dst[r] * rb + (int64_t)ch * 16) = v[r][c];
            }
    }
}

template <int CH>
__global__ void __launch_bounds__(link_threads<CH>()) k_incr_fetch(const int32_t *__restrict__ idx, const int32_t *__restrict__ count,
                                                    const int64_t *__restrict__ offs, int B,
                                                    const int32_t *__restrict__ miss, const int *__restrict__ nmiss,
                                                    const uint8_t *__restrict__ pool, int row16, uint8_t *__restrict__ hot,
                                                    int32_t *__restrict__ host_rows)
{
    extern __shared__ int pre[];
    __shared__ int warp_sum[32];
    const int total = block_count_prefix(count, offs, B, pre, warp_sum);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int n = *nmiss;
    n = n < 0 ? 0 : (n > total ? total : n);
    if (host_rows && blockIdx.x == 0 && threadIdx.x == 0) *host_rows = n;
    const int64_t rb = (int64_t)row16 * 16;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t i0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + warp) * GATHER_ROWS_PER_WARP; i0 < n;
         i0 += wstride * GATHER_ROWS_PER_WARP) {
        int64_t src[GATHER_ROWS_PER_WARP], dst[GATHER_ROWS_PER_WARP];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++) {
            src[r] = -1;
            dst[r] = 0;
            if (i0 + r < n) {
                const int64_t g = miss[i0 + r];
                if (g >= 0 && g < total) {
                    const int b = sequence_of_row(pre, B, g);
                    const int64_t off = offs[b], S = offs[b + 1] - off, j = g - pre[b];
                    const int s = __ldg(idx + off + j);
                    if (s >= 0 && s < S) {
                        src[r] = off + s;
                        dst[r] = off + j;
                    }
                }
            }
        }
        uint4 v[GATHER_ROWS_PER_WARP][CH];
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) v[r][c] = ld_stream16(pool + src[r] * rb + (int64_t)ch * 16);
            }
#pragma unroll
        for (int r = 0; r < GATHER_ROWS_PER_WARP; r++)
#pragma unroll
            for (int c = 0; c < CH; c++) {
                const int ch = lane + 32 * c;
                if (src[r] >= 0 && ch < row16) *(uint4 *)(hot + dst[r] * rb + (int64_t)ch * 16) = v[r][c];
            }
    }
}

}  // namespace lsa
