// Stage 5 on tensor cores: native Lightning-Indexer scores over the fetched entries
// (blog review "FlashMemory-DeepSeek-V4", sections 2.2 and 3.2):
//     y_{b,i,j} = sum_h w'_{b,i,h} ReLU(scale_j q'_{b,i,h} . hot_K_j),   j < count[b].
//
// MMA orientation: the hot keys of sequence b are the A operand (M = 128 keys per tile,
// K = d_I = 128); the queries of a group of nq decode steps are the B operand (N = nq x 64 heads:
// 256 for the batched call, nq = 4; 64 for one decode step, nq = 1), so each TMEM lane (one key)
// holds its head dot products and the weighted head sums of the group's queries run inside one
// thread.  Scores go to Y[tau*off_b + i*S_b + j].  With nq = 1 the query buffers shrink to a
// quarter and the freed shared memory holds more key stages (the one-query call has no key reuse
// and is bound by keys in flight, not by the tensor core).
//
// Work item = (sequence b, chunk of ch key tiles, query group g); items of one chunk are
// consecutive so that CTAs working at the same time share the chunk's keys in L2.  CTAs claim
// items from a global counter (not a fixed share each), so that CTAs slowed by other kernels on
// their SM (the host-link row gather runs beside this kernel) take fewer items instead of setting
// the finish time.  The producer claims; the claimed item numbers reach the MMA and epilogue warps
// through a ring of NRING entries in shared memory that every consumer reads in order.
// Hot keys are bf16 (E4M3 keys were decoded exactly to bf16 by the fetch, their per-entry scale
// is applied here in the epilogue).
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2..9 epilogue (two warps per TMEM
// lane quarter, two queries each).  All waits are bounded as in the index-score kernel.
#pragma once
#include "tc_common.cuh"

namespace lsa {

// A work item as the planner writes it, so that a claim costs one table read (two 16-byte loads).
struct __align__(16) ItemInfo {
    int b, g, t0, t1;  // sequence, query group, key tiles [t0, t1)
    int F, S;          // fetched entries and length of the sequence
    long long off;     // its first entry
};

namespace li {

constexpr int NQ = 4;              // decode queries per MMA (batched call; one decode step: 1)
constexpr int NH = 64;             // heads
constexpr int NCOL = NQ * NH;      // MMA N = 256 (TMEM columns per accumulator slot)
// accumulator slots in the 512 TMEM columns: 2 of 256 columns (4-query groups) or 8 of 64 (one
// query: more tiles between the MMA and the epilogue, whose two warp halves take alternate tiles)
template <int NQV> struct Acc {
    static constexpr int N = NQV == 1 ? 8 : 2;
    static constexpr uint32_t COLS = NQV == 1 ? NH : NCOL;
};
constexpr int CH = 16;             // key tiles per work item (batched call; one decode step: CH_STEP)
constexpr int CH_STEP = 8;
constexpr int MAX_STAGES = 8;
constexpr int NRING = 4;           // claimed items in flight inside a CTA
constexpr int HIST_SHIFT = 18;     // one decode step's score histogram: the top 14 bits of the
constexpr int HIST_BINS = 1 << (32 - HIST_SHIFT);  // order-preserving score key (sign, exponent, 5 bits)

struct Params {
    const float *wd;         // [B][tau][64]
    const float *hsc;        // [T] or null
    const int32_t *count;    // [B]
    const int64_t *offs;     // [B+1]
    const int *item_start;   // [B+1]
    const ItemInfo *items;   // [items] the planner's table
    int *item_counter;       // next unclaimed item, zeroed by k_li_items
    float *Y;                // [tau*T]
    int *hist;               // one decode step (nq = 1): per sequence b, HIST_BINS counters of the
                             // score keys' top bits (hist[b*HIST_BINS + (key >> HIST_SHIFT)]);
                             // null: not counted
    int64_t T;
    int B, tau, groups, stages;
    int ch;                  // key tiles per work item
};

struct Smem {
    uint32_t kraw, qbuf, sw, bars, misc, total;
    __host__ __device__ static Smem plan(int stages, int nq)
    {
        Smem s;
        s.kraw = 0;
        s.qbuf = s.kraw + 128 * 256 * stages;
        s.sw = s.qbuf + 2 * nq * NH * tc::DI * 2;
        s.bars = s.sw + 8 * 2 * NH * 4;
        s.misc = s.bars + 8 * (4 * MAX_STAGES + 8 + 2 * NRING);
        s.total = s.misc + 64 + 1024;
        return s;
    }
};


// Table entries of sequence b's items (items it0 ..): chunk c of ch key tiles and query group g at
// it0 + c groups + g.  nt threads write them, thread t every nt-th.
__device__ __forceinline__ void write_items(ItemInfo *items, int it0, int b, int F, int S, int64_t off, int groups,
                                           int ch, int t, int nt)
{
    const int tiles = (F + TILE - 1) / TILE, nch = (tiles + ch - 1) / ch;
    for (int r = t; r < nch * groups; r += nt) {
        const int c = r / groups;
        ItemInfo x;
        x.b = b;
        x.g = r % groups;
        x.t0 = c * ch;
        x.t1 = min(tiles, (c + 1) * ch);
        x.F = F;
        x.S = S;
        x.off = off;
        items[it0 + r] = x;
    }
}

__device__ __forceinline__ ItemInfo load_item(const ItemInfo *items, int it)
{
    const int4 a = __ldg((const int4 *)(items + it)), c = __ldg((const int4 *)(items + it) + 1);
    ItemInfo x;
    x.b = a.x;
    x.g = a.y;
    x.t0 = a.z;
    x.t1 = a.w;
    x.F = c.x;
    x.S = c.y;
    x.off = (long long)(((unsigned long long)(uint32_t)c.w << 32) | (uint32_t)c.z);
    return x;
}

// Work items per sequence: ceil(ceil(F/128)/ch) chunks x groups, and their table.  One block per
// sequence: it sums the items of the sequences before it (its first item), writes item_start[b + 1]
// and its table entries; block 0 also writes item_start[0] and zeroes the claim counter.
__device__ __forceinline__ int items_of(const int32_t *count, const int64_t *offs, int s, int groups, int ch, int &F,
                                        int64_t &S)
{
    S = offs[s + 1] - offs[s];
    F = count[s];
    F = F < 0 ? 0 : (F > S ? (int)S : F);
    const int tiles = (F + TILE - 1) / TILE;
    return ((tiles + ch - 1) / ch) * groups;
}

__global__ void __launch_bounds__(256) k_li_items(const int32_t *__restrict__ count, const int64_t *__restrict__ offs,
                                                  int B, int groups, int ch, int *__restrict__ item_start,
                                                  int *__restrict__ item_counter, ItemInfo *__restrict__ items)
{
    __shared__ int red[8];
    const int b = blockIdx.x;
    int part = 0, F;
    int64_t S;
    for (int s = threadIdx.x; s < b; s += 256) part += items_of(count, offs, s, groups, ch, F, S);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    int start = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) start += red[w];
    const int n = items_of(count, offs, b, groups, ch, F, S);
    if (threadIdx.x == 0) {
        const int F0 = count[b];
        if (F0 < 0 || F0 > S) flag(ERRF_COUNT);
        item_start[b + 1] = start + n;
        if (b == 0) {
            item_start[0] = 0;
            *item_counter = 0;
        }
    }
    write_items(items, start, b, F, (int)S, offs[b], groups, ch, threadIdx.x, 256);
}

template <int NQV>  // queries per group: NQ (batched call) or 1 (one decode step)
__global__ void __launch_bounds__(320, 1)
    k_li_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap, Params p)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Smem sp = Smem::plan(p.stages, NQV);
    constexpr int ncol = NQV * NH;                          // MMA N
    constexpr uint32_t qbytes = (uint32_t)ncol * DI * 2;    // one query slot
    constexpr uint32_t idesc = tc::idesc_bf16(128, ncol);
    const uint32_t sbase = smem_u32(base);
    const uint32_t kraw = sbase + sp.kraw, qbuf = sbase + sp.qbuf;
    float *sw = (float *)(base + sp.sw);
    const uint32_t bars = sbase + sp.bars;
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    auto qfull = [&](int i) { return bars + 8u * (4 * MAX_STAGES + i); };
    auto qempty = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 2 + i); };
    auto tfull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + i); };    // i < MAX_STAGES (8)
    auto tempty = [&](int i) { return bars + 8u * (3 * MAX_STAGES + i); };
    auto ifull = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 8 + i); };
    auto iempty = [&](int i) { return bars + 8u * (4 * MAX_STAGES + 8 + NRING + i); };
    uint32_t *tmem_holder = (uint32_t *)(base + sp.misc);
    volatile int *abort_flag = (volatile int *)(base + sp.misc + 8);
    volatile int *ring = (volatile int *)(base + sp.misc + 16);  // NRING claimed item numbers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.B;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; i++) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(qfull(i), 1);
            mbar_init(qempty(i), 1);
        }
        for (int i = 0; i < Acc<NQV>::N; i++) {
            mbar_init(tfull(i), 1);
            mbar_init(tempty(i), NQV == 1 ? 4 : 8);  // one query: the 4 warps of the tile's half
        }
        for (int i = 0; i < NRING; i++) {
            mbar_init(ifull(i), 1);
            mbar_init(iempty(i), 9);  // the MMA warp and the 8 epilogue warps
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
    const int NI = __ldg(p.item_start + B);

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&kmap) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&qmap) : "memory");
            int stage = 0, qslot = 1;
            uint32_t phase = 0;
            uint32_t quse[2] = {0, 0};
            uint32_t last_phase[MAX_STAGES];
            bool issued[MAX_STAGES];
            for (int i = 0; i < MAX_STAGES; i++) issued[i] = false;
            const uint32_t kbytes = 128 * 256;
            bool ok = true;
            int islot = 0;
            uint32_t iphase = 0;
            int claim = atomicAdd(p.item_counter, 1);
            while (ok) {
                const int it = claim < NI ? claim : -1;  // -1: no work left, the consumers stop
                if (!mbar_wait(iempty(islot), iphase ^ 1, abort_flag)) { ok = false; break; }
                ring[islot] = it;
                mbar_arrive(ifull(islot));  // release: the ring entry is visible to the waiters
                if (++islot == NRING) { islot = 0; iphase ^= 1; }
                if (it < 0) break;
                const ItemInfo w = load_item(p.items, it);
                claim = atomicAdd(p.item_counter, 1);  // the next claim, in flight while this item's loads go out
                const int t0 = w.t0, t1 = w.t1;
                qslot ^= 1;
                if (!mbar_wait(qempty(qslot), (quse[qslot] & 1) ^ 1, abort_flag)) { ok = false; break; }
                quse[qslot]++;
                mbar_expect_tx(qfull(qslot), qbytes);
                const uint32_t qd = qbuf + (uint32_t)qslot * qbytes;
                const int qrow = (w.b * p.tau + NQV * w.g) * NH;
                tma_load_2d(qd, &qmap, 0, qrow, qfull(qslot));
                tma_load_2d(qd + (uint32_t)ncol * 128, &qmap, 64, qrow, qfull(qslot));
                const int64_t off = w.off;
                for (int kt = t0; kt < t1; kt++) {
                    if (!mbar_wait(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(full(stage), kbytes);
                    const uint32_t dst = kraw + (uint32_t)stage * kbytes;
                    const int y = (int)(off + (int64_t)kt * TILE);
                    tma_load_2d(dst, &kmap, 0, y, full(stage));
                    tma_load_2d(dst + 128 * 128, &kmap, 64, y, full(stage));
                    issued[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort_flag) {
                volatile int never = 0;
                for (int i = 0; i < p.stages; i++)
                    if (issued[i]) mbar_wait(full(i), last_phase[i], &never);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0, qslot = 1;
            uint32_t phase = 0, accphase = 0;
            uint32_t quse[2] = {0, 0};
            bool ok = true;
            int islot = 0;
            uint32_t iphase = 0;
            while (ok) {
                if (!mbar_wait(ifull(islot), iphase, abort_flag)) { ok = false; break; }
                const int it = ring[islot];
                mbar_arrive(iempty(islot));
                if (++islot == NRING) { islot = 0; iphase ^= 1; }
                if (it < 0) break;
                const ItemInfo w = load_item(p.items, it);
                const int t0 = w.t0, t1 = w.t1;
                qslot ^= 1;
                if (!mbar_wait(qfull(qslot), quse[qslot] & 1, abort_flag)) { ok = false; break; }
                quse[qslot]++;
                const uint32_t b_base = qbuf + (uint32_t)qslot * qbytes;
                for (int kt = t0; kt < t1; kt++) {
                    if (!mbar_wait(full(stage), phase, abort_flag)) { ok = false; break; }
                    const uint32_t a_base = kraw + (uint32_t)stage * 128 * 256;
                    if (!mbar_wait(tempty(acc), accphase ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)acc * Acc<NQV>::COLS;
#pragma unroll
                    for (int kk = 0; kk < DI / 16; kk++) {
                        const uint32_t ka = a_base + (uint32_t)(kk >> 2) * (128 * 128) + (uint32_t)(kk & 3) * 32;
                        const uint32_t kb = b_base + (uint32_t)(kk >> 2) * ((uint32_t)ncol * 128) + (uint32_t)(kk & 3) * 32;
                        mma_bf16(d, sdesc(ka), sdesc(kb), idesc, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(empty(stage));
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                    mma_commit(tfull(acc));
                    if (kt == t1 - 1) mma_commit(qempty(qslot));
                    if (++acc == Acc<NQV>::N) { acc = 0; accphase ^= 1; }
                }
                if (ok && t1 <= t0) mma_commit(qempty(qslot));  // an item without tiles still frees its slot
            }
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------------------- epilogue
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int half = (warp - 2) >> 2;        // queries 2*half, 2*half+1 of the group (one query:
                                                 // the half that takes alternate tiles)
        const int nqw = NQV >= 4 ? 2 : NQV;      // this warp's queries of the group
        float *myw = sw + (size_t)(warp - 2) * 2 * NH;
        int acc = 0, tseq = 0;
        uint32_t accphase = 0;
        bool ok = true;
        int islot = 0;
        uint32_t iphase = 0;
        while (ok) {
            if (!mbar_wait_warp(ifull(islot), iphase, abort_flag)) { ok = false; break; }
            const int it = ring[islot];
            __syncwarp();
            if (lane == 0) mbar_arrive(iempty(islot));
            if (++islot == NRING) { islot = 0; iphase ^= 1; }
            if (it < 0) break;
            const ItemInfo w = load_item(p.items, it);
            const int64_t S = w.S;
            const int F = w.F;
            const int t0 = w.t0, t1 = w.t1;
            const int i0 = NQV * w.g + (NQV >= 4 ? 2 * half : 0);  // first of this warp's queries
            __syncwarp();
            for (int t = lane; t < nqw * NH; t += 32)
                myw[t] = __ldg(p.wd + ((int64_t)w.b * p.tau + i0 + t / NH) * NH + (t % NH));
            __syncwarp();
            const int64_t off = w.off;
            float *Yb = p.Y + (int64_t)p.tau * off;
            for (int kt = t0; kt < t1; kt++) {
                if (NQV == 1 && ((tseq++ & 1) != half)) {  // the other half's tile
                    if (++acc == Acc<NQV>::N) { acc = 0; accphase ^= 1; }
                    continue;
                }
                const int64_t j = (int64_t)kt * TILE + quarter * 32 + lane;
                const bool valid = j < F;
                float sc = 1.f;
                if (p.hsc && valid) sc = __ldg(p.hsc + off + j);  // issued before the wait: its latency hides there
                if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (p.hsc && valid && !(sc >= 0.f)) flag(ERRF_SCALE);
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)acc * Acc<NQV>::COLS +
                                       (NQV >= 4 ? 128 * half : 0);
                float y[2] = {0.f, 0.f};
                if (nqw == 0) {  // nothing of this warp in the slot: release it at once
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty(acc));
                }
#pragma unroll
                for (int qq = 0; qq < 2; qq++) {
                    if (qq >= nqw) break;
                    float v0[32], v1[32];
                    tmem_ld32(taddr + qq * NH, v0);
                    tmem_ld32(taddr + qq * NH + 32, v1);
                    tmem_wait_ld();
                    if (qq == nqw - 1) {  // the slot's last read by this warp
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty(acc));
                    }
                    const float *wq = myw + qq * NH;
                    float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll
                    for (int h = 0; h < 32; h += 4) {
                        const float4 wa = *(const float4 *)(wq + h);
                        const float4 wb = *(const float4 *)(wq + 32 + h);
                        x0 = fmaf(wa.x, fmaxf(v0[h], 0.f), x0);
                        x1 = fmaf(wa.y, fmaxf(v0[h + 1], 0.f), x1);
                        x2 = fmaf(wa.z, fmaxf(v0[h + 2], 0.f), x2);
                        x3 = fmaf(wa.w, fmaxf(v0[h + 3], 0.f), x3);
                        x0 = fmaf(wb.x, fmaxf(v1[h], 0.f), x0);
                        x1 = fmaf(wb.y, fmaxf(v1[h + 1], 0.f), x1);
                        x2 = fmaf(wb.z, fmaxf(v1[h + 2], 0.f), x2);
                        x3 = fmaf(wb.w, fmaxf(v1[h + 3], 0.f), x3);
                    }
                    y[qq] = ((x0 + x1) + (x2 + x3)) * sc;  // ReLU(sc d) = sc ReLU(d) for sc >= 0
                }
                if (++acc == Acc<NQV>::N) { acc = 0; accphase ^= 1; }
                if (valid) {
                    if (nqw > 0) Yb[(int64_t)i0 * S + j] = y[0];
                    if (nqw > 1) Yb[(int64_t)(i0 + 1) * S + j] = y[1];
                }
                if (NQV == 1 && p.hist && nqw > 0) {  // the step's histogram, one atomic per bin per warp
                    const uint32_t bin = valid ? float_to_ordered(y[0]) >> HIST_SHIFT : 0xFFFFFFFFu;
                    const unsigned grp = __match_any_sync(0xffffffffu, bin);
                    if (valid && lane == __ffs(grp) - 1)
                        atomicAdd(p.hist + (int64_t)w.b * HIST_BINS + bin, __popc(grp));
                }
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

}  // namespace li

// ------------------------------------------------------------------------------------ host side

// nq: decode queries per MMA group, li::NQ for the batched call, 1 for one decode step.
inline bool li_tc_supported(int n_h, int d_I, int tau, int kdt, int nq = li::NQ)
{
    return n_h == li::NH && d_I == tc::DI && (nq == li::NQ || nq == 1) && tau % nq == 0 &&
           (kdt == DT_BF16 || kdt == DT_FP8) && tc_available();
}

// hotK: bf16 [T][128] (decoded E4M3 codes when hsc is given).  item_start: device [B+1];
// item_counter: one device int (zeroed by the planner).
// nq: queries per MMA group (li_tc_supported).  Launches the item planner and the scoring kernel;
// *launches counts them.
// planned: item_start and item_counter were already written for this call (ch = li_item_tiles(nq)),
// so the planner is not launched.  hist (nq = 1 only; nullable, zeroed): per sequence b, HIST_BINS
// counters of the scores' top key bits.
inline int li_item_tiles(int nq) { return nq == li::NQ ? li::CH : li::CH_STEP; }

// Upper bound on the work items of a call (sum over sequences of ceil(ceil(F_b/128)/ch) x groups).
inline int64_t li_max_items(int B, int64_t T, int tau, int nq)
{
    const int ch = li_item_tiles(nq);
    return (T / ((int64_t)TILE * ch) + B + 1) * (int64_t)(tau / nq);
}

inline lsa_status launch_li_tc(const void *qd, const float *wd, const void *hotK, const float *hsc,
                               const int32_t *count, const int64_t *offs, int B, int64_t T, int tau, int nq, float *Y,
                               int *item_start, int *item_counter, ItemInfo *items, int sms, cudaStream_t st,
                               int *launches, bool planned = false, int *hist = nullptr)
{
    using namespace li;
    *launches = 0;
    if (nq != NQ && nq != 1) return LSA_ERR_UNSUPPORTED;
    const int ch = li_item_tiles(nq);
    if (!planned) {
        k_li_items<<<(unsigned)B, 256, 0, st>>>(count, offs, B, tau / nq, ch, item_start, item_counter, items);
        (*launches)++;
    }
    if (T == 0) return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
    CUtensorMap kmap, qmap;
    bool ok = make_map_2d(&kmap, hotK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)T, tc::DI, 64, 128);
    ok = ok && make_map_2d(&qmap, qd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)B * tau * NH, tc::DI, 64, nq * NH);
    if (!ok) return LSA_ERR_CUDA;
    Params p;
    p.wd = wd;
    p.hsc = hsc;
    p.count = count;
    p.offs = offs;
    p.item_start = item_start;
    p.items = items;
    p.item_counter = item_counter;
    p.Y = Y;
    p.hist = hist;
    p.T = T;
    p.B = B;
    p.tau = tau;
    p.groups = tau / nq;
    p.ch = ch;
    const int max_smem = 227 * 1024;
    p.stages = MAX_STAGES;
    while (p.stages > 2 && Smem::plan(p.stages, nq).total > (uint32_t)max_smem) p.stages--;
    const uint32_t smem = Smem::plan(p.stages, nq).total;
    if (smem > (uint32_t)max_smem) return LSA_ERR_UNSUPPORTED;
    auto kern = nq == NQ ? k_li_tc<NQ> : k_li_tc<1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    kern<<<sms, 320, smem, st>>>(kmap, qmap, p);
    (*launches)++;
    e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa
