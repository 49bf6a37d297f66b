// Tensor-core (tcgen05 + TMEM + TMA) Memory-Indexer index score for n_h = 64, d_I = 128
// (blog review "FlashMemory-DeepSeek-V4", section 3.1; OR rule: section 4.2):
//     x_{l,s} = sum_h w_{l,h} ReLU(scale_s * (q_{l,h} . K_{l,s})),   fetched if x >= logit(thr) in any l.
//
// MMA orientation: one job = one 128-entry tile of one sequence in one layer.  The tile's keys are
// the A operand (M = 128 rows = TMEM lanes, K = d_I = 128) and the head queries are the B operand,
// so the accumulator row of entry s holds its head dot products and the ReLU-weighted head sum
// runs inside one thread (one TMEM lane per entry).  The threshold, the OR over the layers of a
// tile (consecutive jobs) and the ballot into fetch words are fused in the epilogue.
//
//   bf16 keys  kind::f16, N = 64 heads, 8 MMAs of K = 16 per job.
//   E4M3 keys  kind::f8f6f4 straight from the TMA tile (no conversion), K = 32.  The bf16 queries
//              are split by k_q_split_e4m3 into two E4M3 parts, q_h 2^s_h = hi_h + lo_h (s_h puts
//              the head's largest element in [2^7, 2^8)), stored as 128 rows (hi heads, then lo
//              heads); a job runs 8 MMAs of N = 64 into one 64-column accumulator, the 4 over the
//              hi rows and then the 4 over the lo rows of the same key tile, so the sum of the
//              two partial dot products comes out of the tensor core; w_h is pre-multiplied by
//              2^-s_h.  hi + lo is the query exactly (8 significant bits = 4 + 4) for every
//              element at least 2^-9 times its head's largest; smaller elements fall into the
//              E4M3 subnormal range and keep an absolute error below 2^-17 of the head's largest.
//              Each E4M3 x E4M3 product is exact and accumulates in fp32.
// The epilogue's weighted ReLU sum runs as packed fp32 pairs (fma.rn.f32x2), two heads per
// instruction.  Timings that led here: hi | lo as N = 128 columns with the sum in the epilogue
// 696 us, the same with a packed epilogue 676 us, accumulated in the MMA with a packed epilogue
// 656 us (1M x 32 entries x 3 layers).
//
// Warp roles (persistent CTA per SM, contiguous range of tiles; every role's warp runs converged):
//   warps 0, 11 TMA producers, one per parity group (an elected lane issues): key tiles; warp 0
//               also loads the queries of each sequence
//   warps 1, 10 MMA issuers taking alternate tiles (an elected lane issues the MMAs and commits;
//               warp 1 also allocates TMEM).  tcgen05.mma issue blocks while the tensor core is
//               busy, so with one issuer the tensor core idled during the issuer's waits and
//               bookkeeping; two issuers overlap one's bookkeeping with the other's MMAs.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator, score, threshold, OR, ballot; two warps per
//               TMEM lane quarter take alternate tiles (the epilogue is latency-bound per warp)
// Tiles alternate between two parity groups (producer and issuer m = 0/1 and 4 epilogue warps).  Each group
// owns half of the key stages and half of the accumulator slots, so every barrier ring is consumed
// in order by one group: a waiter can never be two phases ahead of a barrier (its parity would
// then alias the preceding, completed phase).  Within a group, job k (k-th job of the group's
// tiles, layer-major per tile) uses stage k % S and slot k % A of the group's halves.
// Every wait is bounded (about 2 s of global time): on time-out the CTA flags ERRF_TIMEOUT,
// stops issuing work, waits (bounded) for its own copies in flight, frees TMEM and returns.
#pragma once
#include "tc_common.cuh"

namespace lsa {

namespace tc {

constexpr int NH = 64;           // heads
constexpr int MAX_STAGES = 12;
constexpr int MAX_L_TC = 3;      // indexer layers handled by one launch
constexpr int NACC_BF16 = 8;     // TMEM accumulator slots: 8 x 64 columns (bf16 keys)
constexpr int NACC_E4M3 = 8;     //                         8 x 64 columns (E4M3 keys: hi + lo accumulated)
constexpr uint32_t IDESC_BF16 = idesc_bf16(128, NH);
constexpr uint32_t IDESC_E4M3 = idesc_f16(128, NH);  // format code 0 is E4M3 under kind::f8f6f4

__device__ __forceinline__ void mma_e4m3(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// Queries for the E4M3 MMA (see the header comment); one warp per head row (l, b, h), four
// consecutive elements per lane.  The last block of the launch does the tile setup of the select
// instead (one launch less on the stage).  q [R][128] bf16, w [R] fp32, R = L * B * 64 ->
// qs [(R/64)][128][128] E4M3 (rows 0..63 hi of heads 0..63, rows 64..127 lo), ws [R] fp32.
__global__ void __launch_bounds__(256) k_q_split_e4m3(const __nv_bfloat16 *__restrict__ q,
                                                      const float *__restrict__ w, uint8_t *__restrict__ qs,
                                                      float *__restrict__ ws, int R, const int64_t *__restrict__ offs,
                                                      int B, int64_t T, int *__restrict__ tile_start,
                                                      int *__restrict__ chunk_start, int32_t *__restrict__ count_out)
{
    if (blockIdx.x == gridDim.x - 1) {
        tile_setup_body(offs, B, T, tile_start, chunk_start, count_out);
        return;
    }
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= R) return;
    float v[4];
    float mx = 0.f;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        v[k] = __bfloat162float(q[(int64_t)row * DI + 4 * lane + k]);
        mx = fmaxf(mx, fabsf(v[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    if (mx > 0.f) {
        const int E = (int)((__float_as_uint(mx) >> 23) & 0xff) - 127;  // bf16 values are fp32-normal
        e = 7 - E;
        e = e < -100 ? -100 : (e > 100 ? 100 : e);
    }
    const float up = __uint_as_float((uint32_t)(127 + e) << 23);    // 2^e, exact
    const float down = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
    const int lb = row / NH, h = row % NH;
    uint32_t hi4 = 0, lo4 = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const float a = v[k] * up;                                   // exact (power-of-two scale)
        const __nv_fp8_storage_t hb = __nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
        const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(hb, __NV_E4M3)));
        const __nv_fp8_storage_t lbits = __nv_cvt_float_to_fp8(a - hv, __NV_SATFINITE, __NV_E4M3);  // a - hv exact
        hi4 |= (uint32_t)hb << (8 * k);
        lo4 |= (uint32_t)lbits << (8 * k);
    }
    uint8_t *base = qs + (int64_t)lb * 128 * DI;
    *(uint32_t *)(base + (int64_t)h * DI + 4 * lane) = hi4;
    *(uint32_t *)(base + (int64_t)(NH + h) * DI + 4 * lane) = lo4;
    if (lane == 0) ws[row] = w[row] * down;
}

// d = a * b + c on two fp32 lanes at once (one fma.rn.f32x2; each lane rounds as fmaf).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

struct Params {
    const float *w;          // [L][B][64]  (E4M3: pre-multiplied by 2^-s_h)
    const float *kscale;     // [L][T] or null
    const int64_t *offs;     // [B+1]
    const int *tile_start;   // [B+1]
    float *scores_out;       // [L][T] or null
    uint32_t *tile_mask;     // [tiles][4]
    int64_t T;
    int B, L, stages;
    float thr;
};

struct SeqTracker {
    // Sequence b owning tile t (t < tile_start[B]), found by walking forward from the previous
    // answer.  The per-sequence values are loaded once per sequence and kept in registers:
    // next = tile_start[b + 1], first = tile_start[b], off = offs[b], S = offs[b + 1] - offs[b].
    // (Entry offsets fit in 32 bits: the total is below 2^31.)
    int b = 0, next = -1, first = 0, off = 0, S = 0;
    __device__ __forceinline__ int of(const int *tile_start, const int64_t *offs, int t)
    {
        if (next < 0 || next <= t) {
            if (next < 0) next = __ldg(tile_start + 1);  // b = 0
            while (next <= t) next = __ldg(tile_start + (++b) + 1);
            first = __ldg(tile_start + b);
            off = (int)__ldg(offs + b);
            S = (int)(__ldg(offs + b + 1) - __ldg(offs + b));
        }
        return b;
    }
};

// Stage (or accumulator slot) and phase of the successive jobs of one parity group.
struct Ring {
    int i = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n)
    {
        if (++i == n) {
            i = 0;
            phase ^= 1;
        }
    }
};

// Shared-memory plan (offsets from a 1024-byte aligned base).  One query slot per launch
// (reloaded at each sequence change, a rare event for a CTA's contiguous tile range).
struct Smem {
    uint32_t kraw, qbuf, sw, bars, misc, total;
    __host__ __device__ static Smem plan(bool fp8, int L, int stages)
    {
        Smem s;
        const uint32_t kstage = fp8 ? 128 * 128 : 128 * 256;
        s.kraw = 0;
        s.qbuf = s.kraw + kstage * stages;
        s.sw = s.qbuf + L * 16384;  // per layer: 64 x 128 bf16, or 128 x 128 E4M3
        s.bars = s.sw + 8 * L * NH * 4;  // one copy of w per epilogue warp
        s.misc = s.bars + 8 * (2 * MAX_STAGES + 2 + 2 * NACC_BF16);
        s.total = s.misc + 64 + 1024;  // + alignment slack
        return s;
    }
};

constexpr int EPI_WARPS = 8;
constexpr int MMA_WARP2 = 2 + EPI_WARPS;          // the second MMA issuer
constexpr int PROD_WARP2 = MMA_WARP2 + 1;         // the second TMA producer
constexpr int THREADS = 32 * (PROD_WARP2 + 1);

template <bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
    k_score_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap, Params p)
{
    constexpr int nacc = FP8 ? NACC_E4M3 : NACC_BF16;
    constexpr int ncol = NH;                          // accumulator columns per job
    constexpr int AP = nacc / 2;                       // accumulator slots per parity group
    const int SP = p.stages / 2;                       // key stages per parity group
    constexpr uint32_t kbytes = FP8 ? 128 * 128 : 128 * 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Smem sp = Smem::plan(FP8, p.L, p.stages);
    const uint32_t sbase = smem_u32(base);
    const uint32_t kraw = sbase + sp.kraw, qbuf = sbase + sp.qbuf;
    float *sw = (float *)(base + sp.sw);
    const uint32_t bars = sbase + sp.bars;
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    const uint32_t qfull = bars + 8u * (2 * MAX_STAGES), qempty = qfull + 8u;
    auto tfull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + i); };
    auto tempty = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + NACC_BF16 + i); };
    uint32_t *tmem_holder = (uint32_t *)(base + sp.misc);
    volatile int *abort_flag = (volatile int *)(base + sp.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = p.L, B = p.B;
    const int64_t T = p.T;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; i++) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, 2);  // both MMA issuers release the query slot
        for (int i = 0; i < nacc; i++) {
            mbar_init(tfull(i), 1);
            mbar_init(tempty(i), 4);  // the 4 warps (one per lane quarter) that own the job's tile
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

    if (warp == 0 || warp == PROD_WARP2) {
        // ------------------------------------------------------------- TMA producers
        // Producer m loads the keys of its group's tiles t_begin + m, + m + 2, ... so that one
        // group's full ring never holds back the other's loads.  Producer 0 also loads the queries:
        // it walks every tile to see the sequence changes.
        const int m = warp == 0 ? 0 : 1;
        const bool leader = elect_one();
        if (leader) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&kmap) : "memory");
            if (m == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&qmap) : "memory");
        }
        SeqTracker tr;
        Ring ring;
        uint32_t quse = 0;
        int prev_b = -1;
        uint32_t last_phase[MAX_STAGES / 2];
        bool issued[MAX_STAGES / 2];
        for (int i = 0; i < MAX_STAGES / 2; i++) issued[i] = false;
        bool ok = true;
        for (int t = t_begin + (m == 0 ? 0 : 1); t < t_end && ok; t += (m == 0 ? 1 : 2)) {
            const int b = tr.of(p.tile_start, p.offs, t);
            if (m == 0 && b != prev_b) {
                if (!mbar_wait_warp(qempty, (quse & 1) ^ 1, abort_flag)) { ok = false; break; }
                quse++;
                if (leader) {
                    mbar_expect_tx(qfull, (uint32_t)L * 16384);
                    for (int l = 0; l < L; l++) {
                        const uint32_t qd = qbuf + (uint32_t)l * 16384;
                        if (FP8) {
                            tma_load_2d(qd, &qmap, 0, (l * B + b) * 2 * NH, qfull);
                        } else {
                            tma_load_2d(qd, &qmap, 0, (l * B + b) * NH, qfull);
                            tma_load_2d(qd + NH * 128, &qmap, 64, (l * B + b) * NH, qfull);
                        }
                    }
                }
                __syncwarp();
                prev_b = b;
            }
            if (((t - t_begin) & 1) != m) continue;
            const int64_t row0 = tr.off + (int64_t)(t - tr.first) * TILE;
            for (int l = 0; l < L; l++) {
                const int ls = ring.i;
                const int stage = m * SP + ls;
                const uint32_t phase = ring.phase;
                ring.next(SP);
                if (!mbar_wait_warp(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                if (leader) {
                    mbar_expect_tx(full(stage), kbytes);
                    const uint32_t dst = kraw + (uint32_t)stage * kbytes;
                    const int y = (int)(l * T + row0);
                    tma_load_2d(dst, &kmap, 0, y, full(stage));
                    if (!FP8) tma_load_2d(dst + 128 * 128, &kmap, 64, y, full(stage));
                }
                __syncwarp();
                issued[ls] = true;
                last_phase[ls] = phase;
            }
        }
        if (*abort_flag && leader) {
            // let the copies this warp started land before the CTA exits
            volatile int never = 0;
            for (int i = 0; i < SP; i++)
                if (issued[i]) mbar_wait(full(m * SP + i), last_phase[i], &never);
            if (m == 0 && quse > 0) mbar_wait(qfull, (quse - 1) & 1, &never);
        }
        __syncwarp();
    } else if (warp == 1 || warp == MMA_WARP2) {
        // ------------------------------------------------------------- MMA issuers
        // Issuer m takes the tiles t_begin + m, + m + 2, ... (its group's rings, see the header).
        // Both walk every tile to track sequences: at the last tile of a sequence each releases the
        // query slot, by a commit after its own MMAs of that sequence, or a plain arrive if none.
        const int m = warp == 1 ? 0 : 1;
        SeqTracker tr;
        Ring kring, aring;
        uint32_t quse = 0;
        int prev_b = -1;
        bool used_q = false;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; t++) {
            const int b = tr.of(p.tile_start, p.offs, t);
            if (b != prev_b) {
                // every issuer waits for every sequence's query load in order (also for sequences it
                // has no tile of), so that it is never two phases ahead of the query barrier
                quse++;  // sequence number within this CTA's range (1-based)
                if (!mbar_wait_warp(qfull, (quse - 1) & 1, abort_flag)) { ok = false; break; }
                prev_b = b;
                used_q = false;
            }
            const bool mine = ((t - t_begin) & 1) == m;
            if (mine) {
                used_q = true;
                for (int l = 0; l < L; l++) {
                    const int stage = m * SP + kring.i, acc = m * AP + aring.i;
                    const uint32_t kphase = kring.phase, aphase = aring.phase;
                    kring.next(SP);
                    aring.next(AP);
                    if (!mbar_wait_warp(full(stage), kphase, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_warp(tempty(acc), aphase ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = kraw + (uint32_t)stage * kbytes;
                    const uint32_t b_base = qbuf + (uint32_t)l * 16384;
                    const uint32_t d = tmem + (uint32_t)(acc * ncol);
                    if (elect_one()) {
                        if (FP8) {
#pragma unroll
                            for (int kk = 0; kk < DI / 32; kk++)  // hi rows (bytes 0 .. 8191 of the query tile)
                                mma_e4m3(d, sdesc(a_base + 32 * kk), sdesc(b_base + 32 * kk), IDESC_E4M3, kk > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < DI / 32; kk++)  // lo rows, accumulated into the same columns
                                mma_e4m3(d, sdesc(a_base + 32 * kk), sdesc(b_base + 8192 + 32 * kk), IDESC_E4M3, 1u);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < DI / 16; kk++) {
                                const uint32_t off = (uint32_t)(kk >> 2) * (128 * 128) + (uint32_t)(kk & 3) * 32;
                                const uint32_t boff = (uint32_t)(kk >> 2) * (NH * 128) + (uint32_t)(kk & 3) * 32;
                                mma_bf16(d, sdesc(a_base + off), sdesc(b_base + boff), IDESC_BF16, kk > 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(empty(stage));
                        mma_commit(tfull(acc));
                    }
                    __syncwarp();
                }
                if (!ok) break;
            }
            const bool last_of_seq = (t + 1 == t_end) || (tr.next <= t + 1);
            if (last_of_seq) {
                if (elect_one()) {
                    if (used_q) mma_commit(qempty);
                    else mbar_arrive(qempty);
                }
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue (warps 2..9)
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int parity = (warp - 2) >> 2;      // this warp takes the tiles t_begin + parity + 2i
        float *myw = sw + (size_t)(warp - 2) * L * NH;
        SeqTracker tr, trn;
        Ring aring;
        int prev_b = -1;
        bool ok = true;
        // E4M3 scales are per entry and layer: load them one tile ahead so that the global-load
        // latency overlaps the previous tile instead of stalling every job.
        float sc_nxt0 = 1.f, sc_nxt1 = 1.f, sc_nxt2 = 1.f;
        auto load_scales = [&](int tt) {
            trn.of(p.tile_start, p.offs, tt);
            const int64_t SS = trn.S;
            const int64_t ss = (int64_t)(tt - trn.first) * TILE + quarter * 32 + lane;
            const int64_t rr = trn.off + ss;
            const bool in = ss < SS;
            sc_nxt0 = in ? __ldg(p.kscale + rr) : 1.f;
            sc_nxt1 = (in && L > 1) ? __ldg(p.kscale + T + rr) : 1.f;
            sc_nxt2 = (in && L > 2) ? __ldg(p.kscale + 2 * T + rr) : 1.f;
        };
        if (FP8 && t_begin + parity < t_end) load_scales(t_begin + parity);
        for (int t = t_begin + parity; t < t_end && ok; t += 2) {
            const int b = tr.of(p.tile_start, p.offs, t);
            if (b != prev_b) {
                __syncwarp();
                for (int i = lane; i < L * NH; i += 32) {
                    const int l = i / NH, h = i % NH;
                    myw[i] = __ldg(p.w + ((int64_t)l * B + b) * NH + h);
                }
                __syncwarp();
                prev_b = b;
            }
            const float sc0 = sc_nxt0, sc1 = sc_nxt1, sc2 = sc_nxt2;
            if (FP8 && t + 2 < t_end) load_scales(t + 2);
            const int64_t S = tr.S;
            const int64_t s = (int64_t)(t - tr.first) * TILE + quarter * 32 + lane;
            const bool valid = s < S;
            const int64_t row = tr.off + s;
            bool fetched = false;
#pragma unroll 1
            for (int l = 0; l < L; l++) {
                const int acc = parity * AP + aring.i;
                const uint32_t accphase = aring.phase;
                aring.next(AP);
                if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * ncol);
                const float *wl = myw + l * NH;
                float2 xa = make_float2(0.f, 0.f), xb = make_float2(0.f, 0.f);
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {  // heads 32*hh .. 32*hh + 31
                    float v[32];
                    tmem_ld32(taddr + 32 * hh, v);
                    tmem_wait_ld();
                    if (hh == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty(acc));
                    }
#pragma unroll
                    for (int h = 0; h < 32; h += 4) {
                        const float4 wa = *(const float4 *)(wl + 32 * hh + h);
                        xa = fma2(make_float2(wa.x, wa.y), make_float2(fmaxf(v[h], 0.f), fmaxf(v[h + 1], 0.f)), xa);
                        xb = fma2(make_float2(wa.z, wa.w), make_float2(fmaxf(v[h + 2], 0.f), fmaxf(v[h + 3], 0.f)), xb);
                    }
                }
                float x = (xa.x + xa.y) + (xb.x + xb.y);
                if (valid) {
                    if (FP8) {
                        const float sc = l == 0 ? sc0 : (l == 1 ? sc1 : sc2);
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

// qs_ws / ws_ws: workspace for the split E4M3 queries and the scaled head weights of the E4M3
// path ([L*B][128][128] bytes and [L*B*64] fp32).  *launches counts the kernels started.
// For E4M3 keys the query split also runs the tile setup (chunk_start, count_out: see k_tile_setup);
// for bf16 keys the caller has run k_tile_setup before.
inline lsa_status launch_score_tc(const void *q, const float *w, const void *K, const float *kscale, int kdt,
                                  const int64_t *offs, int *tile_start, int *chunk_start, int32_t *count_out, int B,
                                  int64_t T, int L, float thr, float *scores_out, uint32_t *tile_mask, void *qs_ws,
                                  float *ws_ws, int sms, cudaStream_t st, int *launches)
{
    using namespace tc;
    *launches = 0;
    if (L < 1 || L > MAX_L_TC) return LSA_ERR_UNSUPPORTED;
    const bool fp8 = (kdt == DT_FP8);
    if (fp8) {
        const int R = L * B * NH;
        k_q_split_e4m3<<<(R + 7) / 8 + 1, 256, 0, st>>>((const __nv_bfloat16 *)q, w, (uint8_t *)qs_ws, ws_ws, R, offs, B, T,
                                                        tile_start, chunk_start, count_out);
        (*launches)++;
        q = qs_ws;
        w = ws_ws;
    }
    CUtensorMap kmap, qmap;
    const uint64_t rows = (uint64_t)L * (uint64_t)T;
    if (rows == 0) return LSA_OK;
    bool ok = fp8 ? make_map_2d(&kmap, K, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, DI, 128, 128)
                  : make_map_2d(&kmap, K, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, DI, 64, 128);
    ok = ok && (fp8 ? make_map_2d(&qmap, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L * B * 2 * NH, DI, 128, 2 * NH)
                    : make_map_2d(&qmap, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L * B * NH, DI, 64, NH));
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
    // Shared memory goes to key stages: bytes in flight hide the HBM latency.
    const int max_smem = 227 * 1024;
    p.stages = MAX_STAGES;  // even: each parity group owns half
    while (p.stages > 2 && Smem::plan(fp8, L, p.stages).total > (uint32_t)max_smem) p.stages -= 2;
    const uint32_t smem = Smem::plan(fp8, L, p.stages).total;
    if (smem > (uint32_t)max_smem) return LSA_ERR_UNSUPPORTED;
    cudaError_t e;
    if (fp8) {
        e = cudaFuncSetAttribute(k_score_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return LSA_ERR_CUDA;
        k_score_tc<true><<<sms, THREADS, smem, st>>>(kmap, qmap, p);
    } else {
        e = cudaFuncSetAttribute(k_score_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return LSA_ERR_CUDA;
        k_score_tc<false><<<sms, THREADS, smem, st>>>(kmap, qmap, p);
    }
    (*launches)++;
    e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa
