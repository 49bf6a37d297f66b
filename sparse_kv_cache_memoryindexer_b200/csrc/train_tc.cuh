// One training step of the memory indexer on the tensor cores (bf16 weights and queries, bf16 or
// E4M3 keys, 64 heads x 128): the two per-entry contractions of k_train_entries (train.cuh) as
// tcgen05 MMAs (hyper.ai summary, "Method"; blog review, sections 3.1 and 4).
//
// Per 128-entry tile of one layer (a CTA walks TPC consecutive tiles):
//   forward   a = K_tile q^T: keys as the A operand (M = 128 entries, K-major), the sequence's
//             queries as B (N = 64 heads, K-major), fp32 accumulator in TMEM (64 columns).  The
//             bf16 products are exact; E4M3 keys are decoded exactly to bf16 in shared memory.
//   epilogue  one thread per entry (its TMEM lane): x = sum_h w_h ReLU(scale a_h), the loss and
//             g = dl/dx / N as in train.cuh; dw_h += g ReLU(scale a_h) in registers; the rows of
//             G = g w_h scale 1[scale a_h > 0] split into bf16 parts G = hi + lo (+ at most 2^-18 |G|).
//   backward  dq^T += K^T hi + K^T lo: the same key tile read as an MN-major A operand (M = 128 key
//             dimensions, K = 128 entries) and G as an MN-major B operand (N = 64 heads); the
//             accumulator (64 columns) stays in TMEM over the CTA's tiles of one sequence and is
//             added to the sequence's dq with atomics when the sequence changes (dw likewise).
// Shared-memory tiles use the 128-byte swizzle: rows of 128 bytes, 16-byte chunk c of row r at
// chunk position c ^ (r % 8).  A bf16 key tile is two such [128][64] boxes 16 KB apart, the
// queries two [64][64] boxes 8 KB apart, each G part one [128][64] box.
// Every mbarrier wait is bounded (about 2 s) and its result is handed to the whole block; on time-out
// the CTA flags ERRF_TIMEOUT, stops, waits (bounded) for the MMAs it issued, frees its TMEM and returns.
#pragma once
#include "gather.cuh"
#include "tc_common.cuh"

namespace lsa {

namespace train_tc {

constexpr int TT = 128;
constexpr int NH = 64;
constexpr int DI = 128;
constexpr int THREADS = 128;
constexpr int TPC = 8;
constexpr uint32_t IDESC_FWD = tc::idesc_bf16(128, NH);
// bf16 A and B, both MN-major (bits 15 and 16), fp32 accumulator, M = 128, N = 64
constexpr uint32_t IDESC_BWD = tc::idesc_bf16(128, NH) | (1u << 15) | (1u << 16);

// shared-memory plan (from a 1024-byte aligned base)
constexpr uint32_t OFF_K = 0;          // keys [2][128][64] bf16
constexpr uint32_t OFF_Q = 32768;      // queries [2][64][64] bf16
constexpr uint32_t OFF_GHI = 49152;    // G hi [128][64] bf16
constexpr uint32_t OFF_GLO = 65536;    // G lo
constexpr uint32_t OFF_W = 81920;      // w [64] fp32
constexpr uint32_t OFF_SC = 82176;     // scales [128] fp32
constexpr uint32_t OFF_DW = 82688;     // dw partial sums [4][64] fp32
constexpr uint32_t OFF_L = 83712;      // loss partial sums [4] double
constexpr uint32_t OFF_BAR = 83744;    // 2 mbarriers
constexpr uint32_t OFF_MISC = 83760;   // TMEM address, abort flag, wait result
constexpr uint32_t SMEM_BYTES = 83776 + 1024;

__device__ __forceinline__ uint32_t sw128(int row, int chunk)
{
    return (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: lbo = bytes between
// 64-element blocks along M or N, sbo = bytes between 8-row groups along K.
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int KDT>
__global__ void __launch_bounds__(THREADS) k_train_entries_tc(const __nv_bfloat16 *__restrict__ q,
                                                              const float *__restrict__ w,
                                                              const uint8_t *__restrict__ K,
                                                              const float *__restrict__ ksc,
                                                              const uint8_t *__restrict__ labels,
                                                              const int64_t *__restrict__ offs,
                                                              const int *__restrict__ tile_start, int B, int64_t T,
                                                              float gamma, float alpha, double invN,
                                                              float *__restrict__ dq, float *__restrict__ dw,
                                                              double *__restrict__ loss)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(base);
    float *wsm = (float *)(base + OFF_W);
    float *scs = (float *)(base + OFF_SC);
    float *dwr = (float *)(base + OFF_DW);
    double *lred = (double *)(base + OFF_L);
    const uint32_t bar_f = sb + OFF_BAR, bar_b = sb + OFF_BAR + 8;
    uint32_t *tmem_holder = (uint32_t *)(base + OFF_MISC);
    volatile int *abort_flag = (volatile int *)(base + OFF_MISC + 4);
    volatile int *wait_ok = (volatile int *)(base + OFF_MISC + 8);

    const int l = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NT = __ldg(tile_start + B);
    const int t0 = blockIdx.x * TPC;
    if (t0 >= NT) return;

    if (tid == 0) {
        mbar_init(bar_f, 1);
        mbar_init(bar_b, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(128));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t d_fwd = tmem, d_bwd = tmem + NH;           // columns 0..63 and 64..127
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    float dwacc[NH];
#pragma unroll
    for (int h = 0; h < NH; h++) dwacc[h] = 0.f;
    double lsum = 0.0;
    int cur_b = -1;
    bool dq_has = false;
    uint32_t ph_f = 0, ph_b = 0;
    bool pend_f = false, pend_b = false;   // MMAs issued whose completion this CTA has not observed
    bool ok = true;

    // Completion of the MMAs committed to `bar`: thread 0 waits (bounded) and a barrier hands the
    // answer to the block, so every thread takes the same branch afterwards.
    auto wait_mma = [&](uint32_t bar, uint32_t phase) -> bool {
        if (tid == 0) *wait_ok = mbar_wait(bar, phase, abort_flag) ? 1 : 0;
        __syncthreads();
        const bool r = *wait_ok != 0;
        tc_fence_after();
        return r;
    };

    auto flush = [&](int bb) {
        // dq^T of this CTA's tiles of sequence bb: TMEM lane = key dimension e, column = head
        if (dq_has) {
            float v[32];
            float *dqb = dq + ((int64_t)l * B + bb) * NH * DI;
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
                tmem_ld32(d_bwd + lane_off + 32 * hh, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i++)
                    if (v[i] != 0.f) atomicAdd(dqb + (32 * hh + i) * DI + tid, v[i]);
            }
        }
        // dw: reduce the per-entry partial sums over the block
#pragma unroll
        for (int h = 0; h < NH; h++) {
            float c = dwacc[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            if (lane == 0) dwr[warp * NH + h] = c;
            dwacc[h] = 0.f;
        }
        __syncthreads();
        if (tid < NH) {
            const float s = dwr[tid] + dwr[NH + tid] + dwr[2 * NH + tid] + dwr[3 * NH + tid];
            if (s != 0.f) atomicAdd(dw + ((int64_t)l * B + bb) * NH + tid, s);
        }
        dq_has = false;
    };

    for (int tt = 0; tt < TPC && ok; tt++) {
        const int t = t0 + tt;
        if (t >= NT) break;
        int lo = 0, hi = B - 1;  // the sequence of tile t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(tile_start + mid) <= t) lo = mid;
            else hi = mid - 1;
        }
        const int b = lo;
        const int64_t off = offs[b], S = offs[b + 1] - off;
        const int64_t s0 = (int64_t)(t - __ldg(tile_start + b)) * TT;
        const int nrow = (int)min((int64_t)TT, S - s0);
        if (b != cur_b) {
            if (cur_b >= 0) flush(cur_b);
            // the sequence's queries (two swizzled boxes) and head weights
            const uint8_t *qs = (const uint8_t *)(q + ((int64_t)l * B + b) * NH * DI);
            uint4 qv[8];
#pragma unroll
            for (int i = 0; i < 8; i++) qv[i] = __ldg((const uint4 *)(qs + (int64_t)(tid + THREADS * i) * 16));
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int ci = tid + THREADS * i, row = ci >> 4, c16 = ci & 15;
                *(uint4 *)(base + OFF_Q + (uint32_t)(c16 >> 3) * 8192u + sw128(row, c16 & 7)) = qv[i];
            }
            if (tid < NH) wsm[tid] = __ldg(w + ((int64_t)l * B + b) * NH + tid);
            cur_b = b;
        }
        // the key tile as bf16 in two swizzled boxes (rows past the sequence are zero)
        const int64_t row0 = (int64_t)l * T + off + s0;
        if (KDT == DT_BF16) {
            const uint8_t *kb = K + row0 * (DI * 2);
            uint4 kv[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int ci = tid + THREADS * i, row = ci >> 4;
                kv[i] = row < nrow ? __ldg((const uint4 *)(kb + (int64_t)ci * 16)) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int ci = tid + THREADS * i, row = ci >> 4, c16 = ci & 15;
                *(uint4 *)(base + OFF_K + (uint32_t)(c16 >> 3) * 16384u + sw128(row, c16 & 7)) = kv[i];
            }
        } else {
            const uint8_t *kb = K + row0 * DI;
            uint4 kv[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int ci = tid + THREADS * i, row = ci >> 3;
                kv[i] = row < nrow ? __ldg((const uint4 *)(kb + (int64_t)ci * 16)) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int ci = tid + THREADS * i, row = ci >> 3, c8 = ci & 7;   // codes 16 c8 .. 16 c8 + 15
                uint4 lo4, hi4;
                e4m3x16_to_bf16(kv[i], lo4, hi4);                             // bf16 chunks 2 c8, 2 c8 + 1
                const uint32_t box = OFF_K + (uint32_t)(c8 >> 2) * 16384u;
                *(uint4 *)(base + box + sw128(row, (2 * c8) & 7)) = lo4;
                *(uint4 *)(base + box + sw128(row, (2 * c8 + 1) & 7)) = hi4;
            }
        }
        scs[tid] = (KDT == DT_FP8 && tid < nrow) ? __ldg(ksc + row0 + tid) : 1.f;
        // generic-proxy writes of the tiles -> visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < DI / 16; kk++) {
                    const uint32_t aoff = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
                    const uint32_t boff = (uint32_t)(kk >> 2) * 8192u + (uint32_t)(kk & 3) * 32u;
                    mma_bf16(d_fwd, sdesc(sb + OFF_K + aoff), sdesc(sb + OFF_Q + boff), IDESC_FWD, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar_f);
            }
            __syncwarp();
        }
        pend_f = true;
        if (!wait_mma(bar_f, ph_f)) { ok = false; break; }
        ph_f ^= 1;
        pend_f = false;
        // epilogue: thread tid = entry tid of the tile (its TMEM lane); two passes over the
        // accumulator (the logit first, then G and dw), 32 heads at a time
        const bool valid = tid < nrow;
        const float sc = scs[tid];
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            float v[32];
            tmem_ld32(d_fwd + lane_off + 32 * hh, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                x0 = fmaf(wsm[32 * hh + i], fmaxf(v[i] * sc, 0.f), x0);
                x1 = fmaf(wsm[32 * hh + i + 1], fmaxf(v[i + 1] * sc, 0.f), x1);
            }
        }
        float g = 0.f;
        if (valid) {
            const float x = x0 + x1;
            const int y = labels[off + s0 + tid] != 0;
            const float p = 1.f / (1.f + expf(-x));
            const float pt = y ? p : 1.f - p;
            const float at = alpha < 0.f ? 1.f : (y ? alpha : 1.f - alpha);
            const float lpt = y ? -log1pf(expf(-x)) : -log1pf(expf(x));
            const float q1 = 1.f - pt;
            float dl;
            if (gamma == 0.f) {
                dl = at * (y ? p - 1.f : p);
                lsum -= (double)at * lpt;
            } else {
                dl = at * (gamma * powf(q1, gamma - 1.f) * lpt * pt * q1 - powf(q1, gamma) * q1) * (y ? 1.f : -1.f);
                lsum -= (double)at * powf(q1, gamma) * lpt;
            }
            g = (float)(dl * invN);
        }
        // G = g w_h scale 1[a_h > 0] as bf16 hi + lo, rows of 64 heads; dw partial sums
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            float v[32];
            tmem_ld32(d_fwd + lane_off + 32 * hh, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; c++) {
                uint32_t ph[4], pl[4];
#pragma unroll
                for (int k2 = 0; k2 < 4; k2++) {
                    const int i = 8 * c + 2 * k2, h = 32 * hh + i;
                    const float a0 = v[i] * sc, a1 = v[i + 1] * sc;
                    const float G0 = a0 > 0.f ? g * wsm[h] * sc : 0.f;
                    const float G1 = a1 > 0.f ? g * wsm[h + 1] * sc : 0.f;
                    const float h0 = __bfloat162float(__float2bfloat16_rn(G0));
                    const float h1 = __bfloat162float(__float2bfloat16_rn(G1));
                    ph[k2] = pack_bf16x2(h0, h1);
                    pl[k2] = pack_bf16x2(G0 - h0, G1 - h1);
                    dwacc[h] = fmaf(g, fmaxf(a0, 0.f), dwacc[h]);
                    dwacc[h + 1] = fmaf(g, fmaxf(a1, 0.f), dwacc[h + 1]);
                }
                *(uint4 *)(base + OFF_GHI + sw128(tid, 4 * hh + c)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                *(uint4 *)(base + OFF_GLO + sw128(tid, 4 * hh + c)) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            if (elect_one()) {
#pragma unroll
                for (int part = 0; part < 2; part++) {
                    const uint32_t gb = sb + (part == 0 ? OFF_GHI : OFF_GLO);
#pragma unroll
                    for (int kk = 0; kk < TT / 16; kk++)
                        mma_bf16(d_bwd, sdesc_mn(sb + OFF_K + 2048u * kk, 16384u, 1024u),
                                 sdesc_mn(gb + 2048u * kk, 16384u, 1024u), IDESC_BWD,
                                 (dq_has || part > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar_b);
            }
            __syncwarp();
        }
        dq_has = true;
        pend_b = true;
        // the next tile overwrites the key and G tiles, and the flush reads the accumulator
        if (!wait_mma(bar_b, ph_b)) { ok = false; break; }
        ph_b ^= 1;
        pend_b = false;
    }
    if (ok) {
        if (cur_b >= 0) flush(cur_b);
    } else if (tid == 0) {
        // let the MMAs this CTA issued finish before its TMEM is released
        volatile int never = 0;
        if (pend_f) mbar_wait(bar_f, ph_f, &never);
        if (pend_b) mbar_wait(bar_b, ph_b, &never);
    }
    // loss
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if (lane == 0) lred[warp] = lsum;
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        const double s2 = lred[0] + lred[1] + lred[2] + lred[3];
        if (s2 != 0.0) atomicAdd(loss, s2 * invN);
    }
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128));
    }
}

inline bool supported(int dt, int kdt, int n_h, int d_I)
{
    return dt == DT_BF16 && (kdt == DT_BF16 || kdt == DT_FP8) && n_h == NH && d_I == DI && tc_available();
}

}  // namespace train_tc

}  // namespace lsa
