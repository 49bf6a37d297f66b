// Tensor-core (tcgen05 + TMEM + TMA) Memory-Indexer index score for n_h = 64, d_I = 128
// (blog review "FlashMemory-DeepSeek-V4", section 3.1; OR rule: section 4.2):
//     x_{l,s} = sum_h w_{l,h} ReLU(scale_s * (q_{l,h} . K_{l,s})),   fetched if x >= logit(thr) in any l.
//
// MMA orientation: one tile = 128 entries of one sequence.  For each layer the tile's keys are
// the A operand (M = 128 rows = TMEM lanes, K = d_I = 128) and the 64 head queries are the B
// operand (N = 64), so the accumulator row of entry s holds its 64 head dot products and the
// ReLU-weighted head sum runs inside one thread (one TMEM lane per entry).  The 0.5 threshold,
// the OR over layers and the ballot into fetch words are fused in the epilogue.
//
// Warp roles (persistent CTA per SM, contiguous range of tiles):
//   warp 0        TMA producer: key tiles (one per (tile, layer)) and the queries of each sequence
//   warp 1        TMEM allocator + MMA issuer (one elected thread)
//   warps 2..5    epilogue: tcgen05.ld of the accumulator, score, threshold, OR, ballot
//   warps 6..13   (E4M3 keys only) converters: E4M3 tile (shared memory) -> f16 A tile written
//                 straight into tensor memory (tcgen05.st), so the MMA reads A from TMEM and only
//                 the queries from shared memory.  Two warps per TMEM lane quarter, each converting
//                 half of every row, so that two independent chains share each sub-partition.
// E4M3 keys run the MMA in f16: a bit-level decode gives each code's value times 2^-8 exactly
// (e4m3x4_to_f16_scaled, K positions permuted (0,2,1,3) within groups of four); k_q_to_f16
// converts the queries to f16 with the same permutation and a per-head power-of-two scale 2^e_h
// (largest element in [2^14, 2^15)), and multiplies w_h by 2^(8 - e_h), so that
// w_h ReLU(q_h . K) is unchanged.  Exact except for query elements more than 2^28 times smaller
// than their head's largest, whose products lie below the fp32 rounding of the dot product.
// Every wait is bounded (about 2 s of global time): on time-out the CTA flags ERRF_TIMEOUT,
// stops issuing work, waits (bounded) for its own copies in flight, frees TMEM and returns.
#pragma once
#include "tc_common.cuh"

namespace lsa {

namespace tc {

constexpr int NH = 64;           // heads (MMA N)
constexpr int NACC = 8;          // TMEM accumulator slots of 64 columns (bf16 keys: all 512 columns)
constexpr int NACC_FP8 = 4;      // E4M3 keys: 4 accumulator slots (columns 0..255) ...
constexpr int ASLOTS = 4;        // ... and 4 A-operand slots of 64 columns (columns 256..511)
constexpr int MAX_STAGES = 8;
constexpr int MAX_L_TC = 3;      // indexer layers handled by one launch
constexpr uint32_t IDESC = idesc_bf16(128, NH);
constexpr uint32_t IDESC_F16 = idesc_f16(128, NH);

// Queries to f16 with a per-head power-of-two scale and the (0,2,1,3) permutation of each group of
// four K positions (see the header comment); one warp per head, four consecutive elements per lane.
// q [R][128] bf16, w [R] fp32 -> qh [R][128] f16, wh [R] fp32, R = L * B * 64.
__global__ void __launch_bounds__(256) k_q_to_f16(const __nv_bfloat16 *__restrict__ q, const float *__restrict__ w,
                                                  __half *__restrict__ qh, float *__restrict__ wh, int R)
{
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= R) return;
    float v[4];
    float mx = 0.f;
    const int perm[4] = {0, 2, 1, 3};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        v[k] = __bfloat162float(q[(int64_t)row * DI + 4 * lane + perm[k]]);
        mx = fmaxf(mx, fabsf(v[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    if (mx > 0.f) {
        const int E = (int)((__float_as_uint(mx) >> 23) & 0xff) - 127;  // bf16 values are fp32-normal
        e = 14 - E;
        e = e < -100 ? -100 : (e > 100 ? 100 : e);
    }
    const float up = __uint_as_float((uint32_t)(127 + e) << 23);        // 2^e, exact
    const float down = __uint_as_float((uint32_t)(127 + 8 - e) << 23);  // 2^(8-e): the keys carry 2^-8
#pragma unroll
    for (int k = 0; k < 4; k++) qh[(int64_t)row * DI + 4 * lane + k] = __float2half_rn(v[k] * up);
    if (lane == 0) wh[row] = w[row] * down;
}

struct Params {
    const float *w;          // [L][B][64]
    const float *kscale;     // [L][T] or null
    const int64_t *offs;     // [B+1]
    const int *tile_start;   // [B+1]
    float *scores_out;       // [L][T] or null
    uint32_t *tile_mask;     // [tiles][4]
    int64_t T;
    int B, L, stages, astages, qslots;
    float thr;
};

struct SeqTracker {
    // Sequence b owning tile t, found by walking forward from the previous answer.
    int b;
    __device__ __forceinline__ int of(const int *tile_start, int B, int t)
    {
        while (b + 1 <= B && __ldg(tile_start + b + 1) <= t) b++;
        return b;
    }
};

// Shared-memory plan (offsets from a 1024-byte aligned base).
struct Smem {
    uint32_t kraw, abuf, qbuf, sw, bars, misc, total;
    __host__ __device__ static Smem plan(bool fp8, int L, int stages, int astages, int qslots)
    {
        Smem s;
        const uint32_t kstage = fp8 ? 128 * 128 : 128 * 256;
        s.kraw = 0;
        s.abuf = s.kraw + kstage * stages;  // (unused: the E4M3 A operand lives in TMEM)
        s.qbuf = s.abuf;
        s.sw = s.qbuf + qslots * L * NH * DI * 2;
        s.bars = s.sw + 4 * L * NH * 4;
        s.misc = s.bars + 8 * (4 * MAX_STAGES + 4 + 2 * NACC);
        s.total = s.misc + 64 + 1024;  // + alignment slack
        return s;
    }
};

constexpr int CONV_WARPS = 8;

template <bool FP8>
__global__ void __launch_bounds__(FP8 ? 192 + 32 * CONV_WARPS : 192, 1)
    k_score_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Smem sp = Smem::plan(FP8, p.L, p.stages, p.astages, p.qslots);
    const uint32_t sbase = smem_u32(base);
    const uint32_t kraw = sbase + sp.kraw, abuf = sbase + sp.abuf, qbuf = sbase + sp.qbuf;
    float *sw = (float *)(base + sp.sw);
    const uint32_t bars = sbase + sp.bars;
    // barrier addresses
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    auto afull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + i); };
    auto aempty = [&](int i) { return bars + 8u * (3 * MAX_STAGES + i); };
    auto qfull = [&](int i) { return bars + 8u * (4 * MAX_STAGES + i); };
    auto qempty = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 2 + i); };
    auto tfull = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 4 + i); };
    auto tempty = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 4 + NACC + i); };
    uint32_t *tmem_holder = (uint32_t *)(base + sp.misc);
    volatile int *abort_flag = (volatile int *)(base + sp.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = p.L, B = p.B;
    const int64_t T = p.T;
    constexpr int nacc = FP8 ? NACC_FP8 : NACC;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; i++) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), FP8 ? CONV_WARPS : 1);
        }
        for (int i = 0; i < p.astages; i++) {
            mbar_init(afull(i), CONV_WARPS);
            mbar_init(aempty(i), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(qfull(i), 1);
            mbar_init(qempty(i), 1);
        }
        for (int i = 0; i < nacc; i++) {
            mbar_init(tfull(i), 1);
            mbar_init(tempty(i), 4);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int NT = __ldg(p.tile_start + B);
    const int G = gridDim.x;
    const int t_begin = (int)((int64_t)blockIdx.x * NT / G);
    const int t_end = (int)((int64_t)(blockIdx.x + 1) * NT / G);

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&kmap) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&qmap) : "memory");
            SeqTracker tr{0};
            int stage = 0;
            uint32_t phase = 0;
            int qslot = -1, prev_b = -1;
            uint32_t quse[2] = {0, 0};
            uint32_t last_phase[MAX_STAGES];
            bool issued[MAX_STAGES];
            for (int i = 0; i < MAX_STAGES; i++) issued[i] = false;
            const uint32_t kbytes = FP8 ? 128 * 128 : 128 * 256;
            const uint32_t kstage = kbytes;
            bool ok = true;
            for (int t = t_begin; t < t_end && ok; t++) {
                const int b = tr.of(p.tile_start, B, t);
                if (b != prev_b) {
                    qslot = (qslot + 1) % p.qslots;
                    if (!mbar_wait(qempty(qslot), (quse[qslot] & 1) ^ 1, abort_flag)) { ok = false; break; }
                    quse[qslot]++;
                    mbar_expect_tx(qfull(qslot), (uint32_t)L * NH * DI * 2);
                    for (int l = 0; l < L; l++) {
                        const uint32_t qd = qbuf + (uint32_t)(qslot * L + l) * NH * DI * 2;
                        const int row = (l * B + b) * NH;
                        tma_load_2d(qd, &qmap, 0, row, qfull(qslot));
                        tma_load_2d(qd + NH * 128, &qmap, 64, row, qfull(qslot));
                    }
                    prev_b = b;
                }
                const int64_t row0 = __ldg(p.offs + b) + (int64_t)(t - __ldg(p.tile_start + b)) * TILE;
                for (int l = 0; l < L; l++) {
                    if (!mbar_wait(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(full(stage), kbytes);
                    const uint32_t dst = kraw + (uint32_t)stage * kstage;
                    const int y = (int)(l * T + row0);
                    if (FP8) {
                        tma_load_2d(dst, &kmap, 0, y, full(stage));
                    } else {
                        tma_load_2d(dst, &kmap, 0, y, full(stage));
                        tma_load_2d(dst + 128 * 128, &kmap, 64, y, full(stage));
                    }
                    issued[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort_flag) {
                // let the copies this thread started land before the CTA exits
                volatile int never = 0;
                for (int i = 0; i < p.stages; i++)
                    if (issued[i]) mbar_wait(full(i), last_phase[i], &never);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            SeqTracker tr{0};
            int stage = 0, as = 0, acc = 0;
            uint32_t phase = 0, aphase = 0, accphase = 0;
            int qslot = -1, prev_b = -1;
            uint32_t quse[2] = {0, 0};
            bool ok = true;
            for (int t = t_begin; t < t_end && ok; t++) {
                const int b = tr.of(p.tile_start, B, t);
                if (b != prev_b) {
                    qslot = (qslot + 1) % p.qslots;
                    if (!mbar_wait(qfull(qslot), quse[qslot] & 1, abort_flag)) { ok = false; break; }
                    quse[qslot]++;
                    prev_b = b;
                }
                const bool last_of_seq = (t + 1 == t_end) || (__ldg(p.tile_start + b + 1) <= t + 1);
                for (int l = 0; l < L; l++) {
                    uint32_t a_base;
                    if (FP8) {
                        if (!mbar_wait(afull(as), aphase, abort_flag)) { ok = false; break; }
                        a_base = tmem + (uint32_t)(NACC_FP8 * NH + as * 64);  // TMEM columns of A slot `as`
                    } else {
                        if (!mbar_wait(full(stage), phase, abort_flag)) { ok = false; break; }
                        a_base = kraw + (uint32_t)stage * 128 * 256;
                    }
                    if (!mbar_wait(tempty(acc), accphase ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b_base = qbuf + (uint32_t)(qslot * L + l) * NH * DI * 2;
                    const uint32_t d = tmem + (uint32_t)acc * NH;
#pragma unroll
                    for (int kk = 0; kk < DI / 16; kk++) {
                        const uint32_t kb = b_base + (uint32_t)(kk >> 2) * (NH * 128) + (uint32_t)(kk & 3) * 32;
                        if (FP8) {
                            mma_f16_tmem_a(d, a_base + (uint32_t)kk * 8, sdesc(kb), IDESC_F16, kk > 0 ? 1u : 0u);
                        } else {
                            const uint32_t ka = a_base + (uint32_t)(kk >> 2) * (128 * 128) + (uint32_t)(kk & 3) * 32;
                            mma_bf16(d, sdesc(ka), sdesc(kb), IDESC, kk > 0 ? 1u : 0u);
                        }
                    }
                    if (FP8) {
                        mma_commit(aempty(as));
                        if (++as == p.astages) { as = 0; aphase ^= 1; }
                    } else {
                        mma_commit(empty(stage));
                        if (++stage == p.stages) { stage = 0; phase ^= 1; }
                    }
                    mma_commit(tfull(acc));
                    if (l == L - 1 && last_of_seq) mma_commit(qempty(qslot));
                    if (++acc == nacc) { acc = 0; accphase ^= 1; }
                }
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------- epilogue
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        float *myw = sw + (size_t)quarter * L * NH;
        SeqTracker tr{0}, trn{0};
        int acc = 0;
        uint32_t accphase = 0;
        int prev_b = -1;
        bool ok = true;
        // E4M3 scales are per entry and layer: load them one tile ahead so that the global-load
        // latency overlaps the previous tile instead of stalling every layer-tile.
        float sc_cur[MAX_L_TC] = {1.f, 1.f, 1.f}, sc_nxt[MAX_L_TC] = {1.f, 1.f, 1.f};
        auto load_scales = [&](int tt, float (&out)[MAX_L_TC]) {
            const int bb = trn.of(p.tile_start, B, tt);
            const int64_t SS = __ldg(p.offs + bb + 1) - __ldg(p.offs + bb);
            const int64_t ss = (int64_t)(tt - __ldg(p.tile_start + bb)) * TILE + quarter * 32 + lane;
            const int64_t rr = __ldg(p.offs + bb) + ss;
#pragma unroll
            for (int l = 0; l < MAX_L_TC; l++) out[l] = (l < L && ss < SS) ? __ldg(p.kscale + (int64_t)l * T + rr) : 1.f;
        };
        if (FP8 && t_begin < t_end) load_scales(t_begin, sc_nxt);
        for (int t = t_begin; t < t_end && ok; t++) {
            const int b = tr.of(p.tile_start, B, t);
            if (b != prev_b) {
                __syncwarp();
                for (int i = lane; i < L * NH; i += 32) {
                    const int l = i / NH, h = i % NH;
                    myw[i] = __ldg(p.w + ((int64_t)l * B + b) * NH + h);
                }
                __syncwarp();
                prev_b = b;
            }
            if (FP8) {
#pragma unroll
                for (int l = 0; l < MAX_L_TC; l++) sc_cur[l] = sc_nxt[l];
                if (t + 1 < t_end) load_scales(t + 1, sc_nxt);
            }
            const int64_t S = __ldg(p.offs + b + 1) - __ldg(p.offs + b);
            const int64_t s = (int64_t)(t - __ldg(p.tile_start + b)) * TILE + quarter * 32 + lane;
            const bool valid = s < S;
            const int64_t row = __ldg(p.offs + b) + s;
            bool fetched = false;
#pragma unroll
            for (int l = 0; l < MAX_L_TC; l++) {
                if (l >= L) break;
                if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)acc * NH;
                float v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty(acc));
                if (++acc == nacc) { acc = 0; accphase ^= 1; }
                const float *wl = myw + l * NH;
                float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll
                for (int h = 0; h < 32; h += 4) {
                    const float4 wa = *(const float4 *)(wl + h);
                    const float4 wb = *(const float4 *)(wl + 32 + h);
                    x0 = fmaf(wa.x, fmaxf(v0[h], 0.f), x0);
                    x1 = fmaf(wa.y, fmaxf(v0[h + 1], 0.f), x1);
                    x2 = fmaf(wa.z, fmaxf(v0[h + 2], 0.f), x2);
                    x3 = fmaf(wa.w, fmaxf(v0[h + 3], 0.f), x3);
                    x0 = fmaf(wb.x, fmaxf(v1[h], 0.f), x0);
                    x1 = fmaf(wb.y, fmaxf(v1[h + 1], 0.f), x1);
                    x2 = fmaf(wb.z, fmaxf(v1[h + 2], 0.f), x2);
                    x3 = fmaf(wb.w, fmaxf(v1[h + 3], 0.f), x3);
                }
                float x = (x0 + x1) + (x2 + x3);
                if (valid) {
                    if (FP8) {
                        const float sc = sc_cur[l];
                        if (!(sc >= 0.f)) flag(ERRF_SCALE);
                        x *= sc;  // ReLU(sc * d) = sc * ReLU(d) for sc >= 0
                    }
                    if (p.scores_out) p.scores_out[(int64_t)l * T + row] = 1.f / (1.f + expf(-x));
                    fetched |= (x >= p.thr);
                }
            }
            if (!ok) break;
            const unsigned m = __ballot_sync(0xffffffffu, fetched);
            if (lane == 0) p.tile_mask[(int64_t)t * 4 + quarter] = m;
        }
    } else if (FP8) {
        // ------------------------------------------------------------- E4M3 -> f16 converters
        const int quarter = warp & 3;            // this warp may only touch TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;       // tile row (entry) converted by this thread
        const int half = (warp - 6) >> 2;        // which 64 of the row's 128 codes (16-byte units 4h .. 4h+3)
        int stage = 0, as = 0;
        uint32_t phase = 0, aphase = 0;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; t++) {
            for (int l = 0; l < L; l++) {
                if (!mbar_wait_warp(full(stage), phase, abort_flag)) { ok = false; break; }
                if (!mbar_wait_warp(aempty(as), aphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t src = kraw + (uint32_t)stage * 128 * 128 + (uint32_t)r * 128;
                const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) +
                                    (uint32_t)(NACC_FP8 * NH + as * 64 + 32 * half);
                uint4 v[4];
#pragma unroll
                for (int uu = 0; uu < 4; uu++) {
                    const int u = 4 * half + uu;  // 16-byte unit of the row (codes 16u .. 16u+15)
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(v[uu].x), "=r"(v[uu].y), "=r"(v[uu].z), "=r"(v[uu].w)
                                 : "r"(src + (uint32_t)((u ^ (r & 7)) * 16)));
                }
                uint32_t o[32];
#pragma unroll
                for (int uu = 0; uu < 4; uu++) {
                    e4m3x4_to_f16_scaled(v[uu].x, o[8 * uu + 0], o[8 * uu + 1]);
                    e4m3x4_to_f16_scaled(v[uu].y, o[8 * uu + 2], o[8 * uu + 3]);
                    e4m3x4_to_f16_scaled(v[uu].z, o[8 * uu + 4], o[8 * uu + 5]);
                    e4m3x4_to_f16_scaled(v[uu].w, o[8 * uu + 6], o[8 * uu + 7]);
                }
                tmem_st32(ta, o);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(empty(stage));
                    mbar_arrive(afull(as));
                }
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
                if (++as == p.astages) { as = 0; aphase ^= 1; }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

}  // namespace tc

// ------------------------------------------------------------------------------------ host side

inline bool tc_score_available() { return tc_available(); }

// qh_ws / wh_ws: workspace for the f16 queries and scaled head weights of the E4M3 path
// ([L*B*64][128] f16 and [L*B*64] fp32).  *launches counts the kernels started.
inline lsa_status launch_score_tc(const void *q, const float *w, const void *K, const float *kscale, int kdt,
                                  const int64_t *offs, const int *tile_start, int B, int64_t T, int L,
                                  float thr, float *scores_out, uint32_t *tile_mask, void *qh_ws, float *wh_ws,
                                  int sms, cudaStream_t st, int *launches)
{
    using namespace tc;
    *launches = 0;
    if (L < 1 || L > MAX_L_TC) return LSA_ERR_UNSUPPORTED;
    const bool fp8 = (kdt == DT_FP8);
    if (fp8) {
        const int R = L * B * NH;
        k_q_to_f16<<<(R + 7) / 8, 256, 0, st>>>((const __nv_bfloat16 *)q, w, (__half *)qh_ws, wh_ws, R);
        (*launches)++;
        q = qh_ws;
        w = wh_ws;
    }
    CUtensorMap kmap, qmap;
    const uint64_t rows = (uint64_t)L * (uint64_t)T;
    if (rows == 0) return LSA_OK;
    bool ok = fp8 ? make_map_2d(&kmap, K, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, DI, 128, 128)
                  : make_map_2d(&kmap, K, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, DI, 64, 128);
    ok = ok && make_map_2d(&qmap, q, fp8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                           (uint64_t)L * B * NH, DI, 64, NH);
    if (!ok) return LSA_ERR_CUDA;
    Params p;
    p.w = w;
    p.kscale = kscale;
    p.offs = offs;
    p.tile_start = tile_start;
    p.scores_out = scores_out;
    p.tile_mask = tile_mask;
    p.T = T;
    p.B = B;
    p.L = L;
    p.thr = thr;
    // Shared memory goes first to key stages (bytes in flight hide the HBM latency); one query slot
    // (reloaded at each sequence change, a rare event for a CTA's contiguous tile range) leaves room
    // for more stages than two.
    const int max_smem = 227 * 1024;
    p.astages = fp8 ? ASLOTS : 0;
    p.qslots = 1;
    p.stages = MAX_STAGES;
    while (p.stages > 2 && Smem::plan(fp8, L, p.stages, p.astages, p.qslots).total > (uint32_t)max_smem) p.stages--;
    const uint32_t smem = Smem::plan(fp8, L, p.stages, p.astages, p.qslots).total;
    if (smem > (uint32_t)max_smem) return LSA_ERR_UNSUPPORTED;
    cudaError_t e;
    if (fp8) {
        e = cudaFuncSetAttribute(k_score_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return LSA_ERR_CUDA;
        k_score_tc<true><<<sms, 192 + 32 * CONV_WARPS, smem, st>>>(kmap, qmap, p);
        (*launches)++;
    } else {
        e = cudaFuncSetAttribute(k_score_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return LSA_ERR_CUDA;
        k_score_tc<false><<<sms, 192, smem, st>>>(kmap, qmap, p);
        (*launches)++;
    }
    e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa
