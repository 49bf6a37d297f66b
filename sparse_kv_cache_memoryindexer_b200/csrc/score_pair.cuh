// The E4M3 index score on CTA pairs (blog review "FlashMemory-DeepSeek-V4", section 3.1; OR rule:
// section 4.2), the same result as k_score_tc<true> (score_tc.cuh) with half the MMA instructions
// per key:
//     x_{l,s} = sum_h w_{l,h} ReLU(scale_s * (q_{l,h} . K_{l,s})),   fetched if x >= logit(thr) in any l.
//
// A cluster of two CTAs on one pair of SMs shares each MMA (tcgen05 cta_group::2, M = 256): a job is
// two consecutive 128-entry tiles of one sequence in one layer, the leader CTA's tile as rows 0..127
// and the peer's as rows 128..255.  Each CTA loads its own key tile and its half of the query
// columns (heads 32 r .. 32 r + 31 of the hi rows and of the lo rows, r = its rank) into its own
// shared memory; the leader issues the 8 MMAs (K = 32, N = 64) of the job and each CTA's TMEM
// receives its own tile's 128 rows x 64 heads.  A sequence with an odd number of tiles ends in a job
// whose peer tile does not exist: the peer loads nothing and its rows are not read.
//
// Synchronisation across the pair:
//   key and query loads  both CTAs' TMA copies complete on the leader's barriers (the leader alone
//                        expects the transaction bytes of both);
//   stage / slot release the leader's MMA commits arrive on the barrier of the same offset in both
//                        CTAs (multicast commit);
//   accumulator release  each CTA's epilogue warps arrive on the leader's barrier (remote arrive);
//   start and end        cluster barriers (the end one keeps each CTA alive until its partner's
//                        last remote arrivals have landed).
// Roles, parity groups and bounded waits are those of k_score_tc (score_tc.cuh); the peer's MMA
// warps issue nothing.  No TMA load here uses cluster multicast.
#pragma once
#include "score_tc.cuh"

namespace lsa {

namespace pair {

using tc::DI;
using tc::NH;
constexpr int MAX_STAGES = tc::MAX_STAGES;
constexpr int NACC = 8;                                   // 8 x 64 TMEM columns, 4 per parity group
constexpr uint32_t IDESC = tc::idesc_f16(256, NH);        // format code 0 is E4M3 under kind::f8f6f4
constexpr uint32_t KBYTES = 128 * 128;                    // one CTA's key tile (E4M3)
constexpr uint32_t QHALF = 32 * DI;                       // 32 query rows (hi or lo) of one layer
constexpr uint32_t QBYTES = 2 * QHALF;                    // one CTA's query half of one layer
constexpr int MAX_B = 1024;                               // sequences per launch (the pair prefix in shared memory)

__device__ __forceinline__ uint32_t cta_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// the address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory, completing on a barrier of either CTA of the pair
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"((uint64_t)map), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// arrive on the barrier at this offset in both CTAs of the pair once the leader's MMAs are done
__device__ __forceinline__ void commit_pair(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(bar), "h"((uint16_t)3) : "memory");
}

struct Params {
    tc::Params p;            // as k_score_tc (w pre-multiplied by 2^-s_h; the E4M3 query split)
};

// Sequence b of pair job j (jobs numbered over the sequences: ceil(tiles_b / 2) each, prefix in
// shared memory), walking forward from the previous answer.
struct PairTracker {
    int b = 0, next = -1, first = 0, tfirst = 0, ntiles = 0, off = 0, S = 0;
    __device__ __forceinline__ int of(const int *pstart, const int *tile_start, const int64_t *offs, int j)
    {
        if (next < 0 || next <= j) {
            if (next < 0) next = pstart[1];
            while (next <= j) next = pstart[(++b) + 1];
            first = pstart[b];
            tfirst = __ldg(tile_start + b);
            ntiles = __ldg(tile_start + b + 1) - tfirst;
            off = (int)__ldg(offs + b);
            S = (int)(__ldg(offs + b + 1) - __ldg(offs + b));
        }
        return b;
    }
};

struct Smem {
    uint32_t kraw, qbuf, sw, pstart, bars, misc, total;
    __host__ __device__ static Smem plan(int L, int stages, int B)
    {
        Smem s;
        s.kraw = 0;
        s.qbuf = s.kraw + KBYTES * stages;
        s.sw = s.qbuf + L * QBYTES;
        s.pstart = s.sw + 8 * L * NH * 4;                  // one copy of w per epilogue warp
        s.bars = s.pstart + ((4 * (B + 1) + 15) & ~15);
        s.misc = s.bars + 8 * (2 * MAX_STAGES + 2 + 2 * NACC);
        s.total = s.misc + 64 + 1024;                      // + alignment slack
        return s;
    }
};

constexpr int EPI_WARPS = 8;
constexpr int MMA_WARP2 = 2 + EPI_WARPS;
constexpr int PROD_WARP2 = MMA_WARP2 + 1;
constexpr int THREADS = 32 * (PROD_WARP2 + 1);

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_score_pair(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap, Params pp)
{
    using namespace tc;
    const tc::Params &p = pp.p;
    constexpr int AP = NACC / 2;
    const int SP = p.stages / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Smem sp = Smem::plan(p.L, p.stages, p.B);
    const uint32_t sbase = smem_u32(base);
    const uint32_t kraw = sbase + sp.kraw, qbuf = sbase + sp.qbuf;
    float *sw = (float *)(base + sp.sw);
    int *pstart = (int *)(base + sp.pstart);
    const uint32_t bars = sbase + sp.bars;
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    const uint32_t qfull = bars + 8u * (2 * MAX_STAGES), qempty = qfull + 8u;
    auto tfull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + i); };
    auto tempty = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + NACC + i); };
    uint32_t *tmem_holder = (uint32_t *)(base + sp.misc);
    volatile int *abort_flag = (volatile int *)(base + sp.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = p.L, B = p.B;
    const int64_t T = p.T;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; i++) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, 2);  // both MMA issuers of the leader release the query slot
        for (int i = 0; i < NACC; i++) {
            mbar_init(tfull(i), 1);
            mbar_init(tempty(i), 8);  // the job's 4 epilogue warps in each CTA (used in the leader)
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // jobs per sequence: ceil(tiles / 2), their prefix (every CTA keeps its own copy)
    if (warp == 2) {
        int carry = 0;
        if (lane == 0) pstart[0] = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            const int n = b < B ? (__ldg(p.tile_start + b + 1) - __ldg(p.tile_start + b) + 1) / 2 : 0;
            const int inc = warp_incl_scan(n);
            if (b < B) pstart[b + 1] = carry + inc;
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers initialised before any remote arrival or copy
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int NJ = pstart[B];
    const int npair = gridDim.x >> 1, pi = blockIdx.x >> 1;
    const int j_begin = (int)((int64_t)pi * NJ / npair);
    const int j_end = (int)((int64_t)(pi + 1) * NJ / npair);

    if (warp == 0 || warp == PROD_WARP2) {
        // ------------------------------------------------------------- TMA producers (both CTAs)
        const int m = warp == 0 ? 0 : 1;
        const bool el = elect_one();
        if (el) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&kmap) : "memory");
            if (m == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&qmap) : "memory");
        }
        PairTracker tr;
        Ring ring;
        uint32_t quse = 0;
        int prev_b = -1;
        bool ok = true;
        for (int j = j_begin + (m == 0 ? 0 : 1); j < j_end && ok; j += (m == 0 ? 1 : 2)) {
            const int b = tr.of(pstart, p.tile_start, p.offs, j);
            if (m == 0 && b != prev_b) {
                if (!mbar_wait_warp(qempty, (quse & 1) ^ 1, abort_flag)) { ok = false; break; }
                quse++;
                if (el) {
                    if (leader) mbar_expect_tx(qfull, (uint32_t)L * 2 * QBYTES);
                    const uint32_t qbar = mapa(qfull, 0);
                    for (int l = 0; l < L; l++) {
                        const uint32_t qd = qbuf + (uint32_t)l * QBYTES;
                        const int row = (l * B + b) * 2 * NH + 32 * (int)rank;
                        tma_load_2d_pair(qd, &qmap, 0, row, qbar);               // hi rows of my heads
                        tma_load_2d_pair(qd + QHALF, &qmap, 0, row + NH, qbar);  // lo rows of my heads
                    }
                }
                __syncwarp();
                prev_b = b;
            }
            if (((j - j_begin) & 1) != m) continue;
            const int tl = 2 * (j - tr.first) + (int)rank;  // this CTA's tile within the sequence
            const bool mine = tl < tr.ntiles;
            const bool both = 2 * (j - tr.first) + 1 < tr.ntiles;
            const int64_t row0 = tr.off + (int64_t)tl * TILE;
            for (int l = 0; l < L; l++) {
                const int stage = m * SP + ring.i;
                const uint32_t phase = ring.phase;
                ring.next(SP);
                if (!mbar_wait_warp(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                if (el) {
                    if (leader) mbar_expect_tx(full(stage), KBYTES * (both ? 2u : 1u));
                    if (mine)
                        tma_load_2d_pair(kraw + (uint32_t)stage * KBYTES, &kmap, 0, (int)(l * T + row0),
                                         mapa(full(stage), 0));
                }
                __syncwarp();
            }
        }
        __syncwarp();
    } else if (warp == 1 || warp == MMA_WARP2) {
        // ------------------------------------------------------------- MMA issuers (the leader)
        if (leader) {
            const int m = warp == 1 ? 0 : 1;
            PairTracker tr;
            Ring kring, aring;
            uint32_t quse = 0;
            int prev_b = -1;
            bool used_q = false;
            bool ok = true;
            for (int j = j_begin; j < j_end && ok; j++) {
                const int b = tr.of(pstart, p.tile_start, p.offs, j);
                if (b != prev_b) {
                    quse++;
                    if (!mbar_wait_warp(qfull, (quse - 1) & 1, abort_flag)) { ok = false; break; }
                    prev_b = b;
                    used_q = false;
                }
                if (((j - j_begin) & 1) == m) {
                    used_q = true;
                    for (int l = 0; l < L; l++) {
                        const int stage = m * SP + kring.i, acc = m * AP + aring.i;
                        const uint32_t kphase = kring.phase, aphase = aring.phase;
                        kring.next(SP);
                        aring.next(AP);
                        if (!mbar_wait_warp(full(stage), kphase, abort_flag)) { ok = false; break; }
                        if (!mbar_wait_warp(tempty(acc), aphase ^ 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_base = kraw + (uint32_t)stage * KBYTES;
                        const uint32_t b_base = qbuf + (uint32_t)l * QBYTES;
                        const uint32_t d = tmem + (uint32_t)(acc * NH);
                        if (elect_one()) {
#pragma unroll
                            for (int kk = 0; kk < DI / 32; kk++)  // hi rows
                                mma_pair(d, sdesc(a_base + 32 * kk), sdesc(b_base + 32 * kk), IDESC, kk > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < DI / 32; kk++)  // lo rows, accumulated into the same columns
                                mma_pair(d, sdesc(a_base + 32 * kk), sdesc(b_base + QHALF + 32 * kk), IDESC, 1u);
                            commit_pair(empty(stage));
                            commit_pair(tfull(acc));
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                }
                const bool last_of_seq = (j + 1 == j_end) || (tr.next <= j + 1);
                if (last_of_seq) {
                    if (elect_one()) {
                        if (used_q) {
                            commit_pair(qempty);
                        } else {
                            mbar_arrive(qempty);
                            remote_arrive(mapa(qempty, 1));
                        }
                    }
                    __syncwarp();
                }
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue (warps 2..9, both CTAs)
        const int quarter = warp & 3;
        const int parity = (warp - 2) >> 2;
        float *myw = sw + (size_t)(warp - 2) * L * NH;
        PairTracker tr, trn;
        Ring aring;
        int prev_b = -1;
        bool ok = true;
        float sc_nxt0 = 1.f, sc_nxt1 = 1.f, sc_nxt2 = 1.f;
        auto load_scales = [&](int jj) {
            trn.of(pstart, p.tile_start, p.offs, jj);
            const int tl = 2 * (jj - trn.first) + (int)rank;
            const int64_t ss = (int64_t)tl * TILE + quarter * 32 + lane;
            const int64_t rr = trn.off + ss;
            const bool in = tl < trn.ntiles && ss < trn.S;
            sc_nxt0 = in ? __ldg(p.kscale + rr) : 1.f;
            sc_nxt1 = (in && L > 1) ? __ldg(p.kscale + T + rr) : 1.f;
            sc_nxt2 = (in && L > 2) ? __ldg(p.kscale + 2 * T + rr) : 1.f;
        };
        if (j_begin + parity < j_end) load_scales(j_begin + parity);
        for (int j = j_begin + parity; j < j_end && ok; j += 2) {
            const int b = tr.of(pstart, p.tile_start, p.offs, j);
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
            if (j + 2 < j_end) load_scales(j + 2);
            const int tl = 2 * (j - tr.first) + (int)rank;
            const bool mine = tl < tr.ntiles;
            const int64_t s = (int64_t)tl * TILE + quarter * 32 + lane;
            const bool valid = mine && s < tr.S;
            const int64_t row = tr.off + s;
            bool fetched = false;
#pragma unroll 1
            for (int l = 0; l < L; l++) {
                const int acc = parity * AP + aring.i;
                const uint32_t accphase = aring.phase;
                aring.next(AP);
                if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NH);
                const float *wl = myw + l * NH;
                float2 xa = make_float2(0.f, 0.f), xb = make_float2(0.f, 0.f);
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    float v[32];
                    tmem_ld32(taddr + 32 * hh, v);
                    tmem_wait_ld();
                    if (hh == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (leader) mbar_arrive(tempty(acc));
                            else remote_arrive(mapa(tempty(acc), 0));
                        }
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
                    const float sc = l == 0 ? sc0 : (l == 1 ? sc1 : sc2);
                    if (!(sc >= 0.f)) flag(ERRF_SCALE);
                    x *= sc;  // ReLU(sc * d) = sc * ReLU(d) for sc >= 0
                    if (p.scores_out) p.scores_out[(int64_t)l * T + row] = 1.f / (1.f + expf(-x));
                    fetched |= (x >= p.thr);
                }
            }
            if (!ok) break;
            const unsigned fm = __ballot_sync(0xffffffffu, fetched);
            if (mine && lane == 0) p.tile_mask[(int64_t)(tr.tfirst + tl) * 4 + quarter] = fm;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the partner's last remote arrivals and copies have landed
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

}  // namespace pair

// ------------------------------------------------------------------------------------ host side

inline bool score_pair_supported(int kdt, int B, int sms) { return kdt == DT_FP8 && B <= pair::MAX_B && sms >= 2; }

// The score launch of the E4M3 path on CTA pairs (after k_q_split_e4m3 wrote qs / ws and the tile
// setup); grid: the largest even number of CTAs not above the SM count.
inline lsa_status launch_score_pair(const void *qs, const float *ws, const void *K, const float *kscale,
                                    const int64_t *offs, int *tile_start, int B, int64_t T, int L, float thr,
                                    float *scores_out, uint32_t *tile_mask, int sms, cudaStream_t st)
{
    using namespace pair;
    CUtensorMap kmap, qmap;
    const uint64_t rows = (uint64_t)L * (uint64_t)T;
    if (rows == 0) return LSA_OK;
    bool ok = make_map_2d(&kmap, K, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, DI, 128, 128);
    ok = ok && make_map_2d(&qmap, qs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L * B * 2 * NH, DI, 128, 32);
    if (!ok) return LSA_ERR_CUDA;
    Params pp;
    pp.p.w = ws;
    pp.p.kscale = kscale;
    pp.p.offs = offs;
    pp.p.tile_start = tile_start;
    pp.p.scores_out = scores_out;
    pp.p.tile_mask = tile_mask;
    pp.p.T = T;
    pp.p.B = B;
    pp.p.L = L;
    pp.p.thr = thr;
    const int max_smem = 227 * 1024;
    pp.p.stages = MAX_STAGES;  // even: each parity group owns half
    while (pp.p.stages > 2 && Smem::plan(L, pp.p.stages, B).total > (uint32_t)max_smem) pp.p.stages -= 2;
    const uint32_t smem = Smem::plan(L, pp.p.stages, B).total;
    if (smem > (uint32_t)max_smem) return LSA_ERR_UNSUPPORTED;
    cudaError_t e = cudaFuncSetAttribute(k_score_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    k_score_pair<<<(unsigned)(sms & ~1), THREADS, smem, st>>>(kmap, qmap, pp);
    e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa
