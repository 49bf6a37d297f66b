// Stage 1 on tensor cores: the indexer projections of the trigger token (blog review
// "FlashMemory-DeepSeek-V4", section 3.1; hyper.ai summary, "Method"):
//     c = h W^DQ,   q = c W^IUQ,   w = h W^w     for every layer l and sequence b.
// Each is Y[l][b][o] = sum_k X[l][b][k] W[l][o][k] with the weights stored as rows of outputs
// (K contiguous).  The weights dominate the bytes (B is a batch of sequences, at most 256), so
// the weight rows are the MMA A operand (M = 128 output rows per tile, streamed once by TMA) and
// the batch is the B operand (N = B rounded up to 16; the small X tiles are re-read from L2 by
// every CTA).
//
// A launch serves one or two problems with the same X (c and w both read h).  Its work units are
// (problem, 128-row tile, range of K): a problem whose tiles alone would leave SMs idle is split
// along K into at most KSPLIT_MAX ranges, each unit storing its fp32 partial sums into a slice of
// its own (no atomics, nothing to zero); k_proj_reduce then adds the slices in a fixed order and
// rounds (c to bf16; w stays fp32).  A problem with enough tiles takes all of K per unit and its
// epilogue rounds to the output type (bf16 nearest-even, or fp32) and stores.  Either way every
// output is an fp32 sum of its K products, rounded once, and the same on every run.
//
// Launches of one projection follow each other as programmatic dependents: every kernel here lets
// its dependents start at once, and a dependent waits for its predecessor (griddepcontrol.wait)
// before it touches what the predecessor writes.  The tensor-core kernel issues the weight boxes
// of its first stages before that wait (the weights are inputs of the call, not results of the
// previous launch), so its weight stream starts while the previous launch drains; the X boxes
// follow the wait.
//
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2..5 epilogue (one TMEM lane
// quarter each).  Two accumulators, so a unit's epilogue overlaps the next unit's MMAs.  Every
// ring is consumed in order by one consumer (group); waits are bounded as in the other
// tensor-core kernels.
#pragma once
#include "pdl.cuh"
#include "tc_common.cuh"

namespace lsa {

namespace proj {

constexpr int KB = 64;              // K elements per box (one 128-byte swizzle atom of bf16)
constexpr int MAX_BOX = 2;          // boxes per stage: 256 contiguous bytes of every weight row
constexpr int KSPLIT_MAX = 8;       // K ranges of a split problem (partial slices)
constexpr int MAX_STAGES = 8;
constexpr int THREADS = 6 * 32;
constexpr uint32_t A_BYTES = 128 * KB * 2;

struct Prob {
    void *out;          // [L][B][R] bf16 or fp32; split: fp32 partial slices [ksplit][L][B][R]
    int R;              // output rows
    int out_f32;
    int partial;        // split along K: store fp32 partial sums into slice ks
    int mtiles;         // 128-row tiles per layer
    int ksplit;         // K ranges per tile
    int nkb_per;        // K blocks per range
    int units;          // L * mtiles * ksplit
};

struct Params {
    Prob pr[2];
    int nprob;
    int L, B, K;        // layers, batch, reduction length
    int NB;             // MMA N = B rounded up to 16
    int stages;
    int nbox;           // K boxes per stage
};

struct Unit {
    int prob, l, m0, kb0, kb1, ks;
    void *out;
    int R, out_f32, partial;
};

// The problem fields are picked with selects (no dynamic index into the kernel parameters).
__device__ __forceinline__ Unit unit_of(const Params &p, int u, int nkb)
{
    Unit x;
    x.prob = u < p.pr[0].units ? 0 : 1;
    const bool one = x.prob == 1;
    const int ksplit = one ? p.pr[1].ksplit : p.pr[0].ksplit;
    const int mtiles = one ? p.pr[1].mtiles : p.pr[0].mtiles;
    const int nkb_per = one ? p.pr[1].nkb_per : p.pr[0].nkb_per;
    const int v = u - (one ? p.pr[0].units : 0);
    const int t = v / ksplit, ks = v % ksplit;
    x.l = t / mtiles;
    x.m0 = (t % mtiles) * 128;
    x.kb0 = ks * nkb_per;
    x.kb1 = min(nkb, x.kb0 + nkb_per);
    x.ks = ks;
    x.out = one ? p.pr[1].out : p.pr[0].out;
    x.R = one ? p.pr[1].R : p.pr[0].R;
    x.out_f32 = one ? p.pr[1].out_f32 : p.pr[0].out_f32;
    x.partial = one ? p.pr[1].partial : p.pr[0].partial;
    return x;
}

__host__ __device__ inline uint32_t b_bytes(int NB) { return (uint32_t)NB * KB * 2; }
// a stage: nbox weight boxes (128 rows x 64 K each), then nbox X boxes (NB rows x 64 K each)
__host__ __device__ inline uint32_t stage_bytes(int NB, int nbox) { return (uint32_t)nbox * (A_BYTES + b_bytes(NB)); }
__host__ __device__ inline uint32_t smem_total(int NB, int stages, int nbox)
{
    return stage_bytes(NB, nbox) * stages + 8 * (2 * MAX_STAGES + 4) + 64 + 1024;
}
// TMEM columns per accumulator: N rounded up to 32, so that 32-column loads stay inside it.
__host__ __device__ inline uint32_t acc_cols(int NB) { return (uint32_t)(NB + 31) / 32 * 32; }
__host__ __device__ inline uint32_t tmem_cols(int NB)  // two accumulators, a power of two >= 32
{
    uint32_t c = 32;
    while (c < 2 * acc_cols(NB)) c <<= 1;
    return c;
}

__global__ void __launch_bounds__(THREADS)
    k_proj_tc(const __grid_constant__ CUtensorMap wmap0, const __grid_constant__ CUtensorMap wmap1,
              const __grid_constant__ CUtensorMap xmap, Params p)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t sbytes = stage_bytes(p.NB, p.nbox), bbox = b_bytes(p.NB);
    const uint32_t bars = sbase + sbytes * p.stages;
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    auto tfull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + i); };
    auto tempty = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + i); };
    uint8_t *misc = base + sbytes * p.stages + 8 * (2 * MAX_STAGES + 4);
    uint32_t *tmem_holder = (uint32_t *)misc;
    volatile int *abort_flag = (volatile int *)(misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nunits = p.pr[0].units + (p.nprob > 1 ? p.pr[1].units : 0);
    const int nkb = (p.K + KB - 1) / KB;
    const uint32_t ncols = tmem_cols(p.NB), acol = acc_cols(p.NB);
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; i++) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(tfull(i), 1);
            mbar_init(tempty(i), 4);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------- TMA producer
        const bool leader = elect_one();
        if (leader) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&wmap0) : "memory");
            if (p.nprob > 1) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&wmap1) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&xmap) : "memory");
        }
        int stage = 0;
        uint32_t phase = 0;
        uint32_t last_phase[MAX_STAGES];
        bool issued[MAX_STAGES];
        for (int i = 0; i < MAX_STAGES; i++) issued[i] = false;
        // stages whose weight boxes went out before the wait for the previous launch: their X boxes
        // (K block, count, X row) follow the wait
        int pend_kb[MAX_STAGES], pend_nb[MAX_STAGES], pend_row[MAX_STAGES];
        int pending = 0;
        bool waited = false;
        auto x_boxes = [&](int st_i, int kb, int nb, int xrow) {
            const uint32_t dst = sbase + (uint32_t)st_i * sbytes + (uint32_t)p.nbox * A_BYTES;
            for (int i = 0; i < nb; i++) tma_load_2d(dst + (uint32_t)i * bbox, &xmap, (kb + i) * KB, xrow, full(st_i));
        };
        auto release = [&]() {  // wait for the previous launch, then the X boxes of the pending stages
            pdl_wait();
            if (leader)
                for (int j = 0; j < pending; j++) x_boxes(j, pend_kb[j], pend_nb[j], pend_row[j]);
            __syncwarp();
            waited = true;
        };
        bool ok = true;
        for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
            const Unit x = unit_of(p, u, nkb);
            const CUtensorMap *wm = x.prob == 0 ? &wmap0 : &wmap1;
            for (int kb = x.kb0; kb < x.kb1; kb += p.nbox) {
                const int nb = min(p.nbox, x.kb1 - kb);
                if (!waited && pending == p.stages) release();  // every stage holds weights: nothing more before X
                if (!mbar_wait_warp(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                if (leader) {
                    mbar_expect_tx(full(stage), (uint32_t)nb * (A_BYTES + bbox));
                    const uint32_t dst = sbase + (uint32_t)stage * sbytes;
                    for (int i = 0; i < nb; i++)  // the boxes of a stage back to back: row segments of 256 bytes
                        tma_load_2d(dst + (uint32_t)i * A_BYTES, wm, (kb + i) * KB, x.l * x.R + x.m0, full(stage));
                    if (waited) x_boxes(stage, kb, nb, x.l * p.B);
                }
                if (!waited) {  // (the first stages, in order: stage == pending)
                    pend_kb[pending] = kb;
                    pend_nb[pending] = nb;
                    pend_row[pending] = x.l * p.B;
                    pending++;
                }
                __syncwarp();
                issued[stage] = true;
                last_phase[stage] = phase;
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
            }
        }
        if (!waited) release();  // (also on an abort: every issued stage gets its X bytes)
        if (*abort_flag && leader) {
            volatile int never = 0;
            for (int i = 0; i < p.stages; i++)
                if (issued[i]) mbar_wait(full(i), last_phase[i], &never);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        const uint32_t idesc = idesc_bf16(128, p.NB);
        int stage = 0, acc = 0;
        uint32_t phase = 0, accphase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
            const Unit x = unit_of(p, u, nkb);
            if (!mbar_wait_warp(tempty(acc), accphase ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)acc * acol;
            for (int kb = x.kb0; kb < x.kb1; kb += p.nbox) {
                const int nb = min(p.nbox, x.kb1 - kb);
                if (!mbar_wait_warp(full(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_base = sbase + (uint32_t)stage * sbytes;
                const uint32_t b_base = a_base + (uint32_t)p.nbox * A_BYTES;
                if (elect_one()) {
                    for (int i = 0; i < nb; i++) {
#pragma unroll
                        for (int kk = 0; kk < KB / 16; kk++)
                            mma_bf16(d, sdesc(a_base + (uint32_t)i * A_BYTES + 32 * kk), sdesc(b_base + (uint32_t)i * bbox + 32 * kk),
                                     idesc, (kb > x.kb0 || i > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(empty(stage));
                    if (kb + nb >= x.kb1) mma_commit(tfull(acc));
                }
                __syncwarp();
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
            }
            if (++acc == 2) { acc = 0; accphase ^= 1; }
        }
    } else {
        // ------------------------------------------------------------- epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        int acc = 0;
        uint32_t accphase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
            const Unit x = unit_of(p, u, nkb);
            if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const int o = x.m0 + quarter * 32 + lane;
            const bool valid = o < x.R;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)acc * acol;
            for (int b0 = 0; b0 < p.NB; b0 += 32) {
                float v[32];
                tmem_ld32(taddr + b0, v);  // columns past N (up to the accumulator's end) are not stored
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int b = b0 + i;
                    if (valid && b < p.B) {
                        const int64_t at = ((int64_t)x.l * p.B + b) * x.R + o;
                        if (x.partial) ((float *)x.out)[(int64_t)x.ks * p.L * p.B * x.R + at] = v[i];
                        else if (x.out_f32) ((float *)x.out)[at] = v[i];
                        else ((__nv_bfloat16 *)x.out)[at] = __float2bfloat16_rn(v[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(acc));
            if (++acc == 2) { acc = 0; accphase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

}  // namespace proj

// ------------------------------------------------------------------------------------ host side

inline bool proj_tc_supported(int dt, int B, int K) { return dt == DT_BF16 && B >= 1 && B <= 256 && K % 8 == 0 && tc_available(); }

// One problem of a launch: out[l][b][o] = sum_k X[l][b][k] W[l][o][k], W bf16 [L][R][K].
struct ProjProblem {
    const void *W;
    void *out;          // split along K: fp32 partial slices [KSPLIT_MAX][L][B][R]; else bf16 or fp32
    int R;
    bool out_f32;
};

// Boxes per stage and stages of a launch with batch B (the shared memory decides).
struct ProjShape {
    int NB, nbox, stages;
    uint32_t smem;
};
inline ProjShape proj_shape(int B)
{
    using namespace proj;
    ProjShape s;
    s.NB = (B + 15) / 16 * 16;
    const uint32_t max_smem = 227 * 1024 - 1024;
    s.nbox = MAX_BOX;
    while (s.nbox > 1 && smem_total(s.NB, 2, s.nbox) > max_smem) s.nbox >>= 1;
    s.stages = MAX_STAGES;
    while (s.stages > 2 && smem_total(s.NB, s.stages, s.nbox) > max_smem) s.stages--;
    s.smem = smem_total(s.NB, s.stages, s.nbox);
    if (s.smem > max_smem) s.smem = 0;  // unsupported
    return s;
}

// K ranges for `tiles` 128-row tiles over K of `nst` stages: the count (at most KSPLIT_MAX, whole
// stages each) whose units fill `sms` CTAs best (1: no split).
inline int proj_ksplit(int64_t tiles, int nst, int sms)
{
    int ks = 1;
    double best = -1.0;
    for (int c = 1; c <= proj::KSPLIT_MAX && c <= nst; c++) {
        const int spc = (nst + c - 1) / c;  // stages per range
        const int ranges = (nst + spc - 1) / spc;
        if (ranges != c) continue;
        const int64_t units = tiles * c;
        const int64_t waves = (units + sms - 1) / sms;
        const double eff = (double)units / (double)(waves * sms);
        if (eff > best + 1e-9) {
            best = eff;
            ks = c;
        }
    }
    return ks;
}

// Stages of all of K for a launch of batch B.
inline int proj_stages_of_k(int B, int K)
{
    const ProjShape sh = proj_shape(B);
    const int nkb = (K + proj::KB - 1) / proj::KB;
    return (nkb + sh.nbox - 1) / sh.nbox;
}

// One launch over one or two problems sharing X bf16 [L][B][K]; a split problem's units store
// partial slices, and ksplit_out[i] (nullable) reports how many.  One CTA per SM; a stage holds up
// to MAX_BOX boxes of K so that every weight row is read in segments of 256 bytes.  Split problems
// take the number of K ranges (proj_ksplit) that balances the units best over the CTAs.  pdl: the
// launch is a programmatic dependent of the previous one on the stream.
inline lsa_status launch_proj_tc(const void *X, const ProjProblem *pb, const bool *split, int nprob, int L, int B,
                                 int K, int sms, cudaStream_t st, int *ksplit_out = nullptr, bool pdl = false)
{
    using namespace proj;
    CUtensorMap wmap[2], xmap;
    proj::Params p;
    p.nprob = nprob;
    p.L = L;
    p.B = B;
    p.K = K;
    const ProjShape sh = proj_shape(B);
    if (sh.smem == 0) return LSA_ERR_UNSUPPORTED;
    p.NB = sh.NB;
    p.nbox = sh.nbox;
    p.stages = sh.stages;
    const uint32_t smem = sh.smem;
    const int nkb = (K + KB - 1) / KB;
    const int nst = (nkb + p.nbox - 1) / p.nbox;  // stages of all of K
    int tiles = 0;
    for (int i = 0; i < nprob; i++) tiles += L * ((pb[i].R + 127) / 128);
    bool any_split = false;
    for (int i = 0; i < nprob; i++) any_split = any_split || split[i];
    const int ks = any_split ? proj_ksplit(tiles, nst, sms) : 1;
    bool ok = make_map_2d(&xmap, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L * B, (uint64_t)K, KB, (uint32_t)p.NB);
    int total = 0;
    for (int i = 0; i < 2; i++) {
        const ProjProblem &q = pb[i < nprob ? i : 0];
        Prob &r = p.pr[i];
        r.out = q.out;
        r.R = q.R;
        r.out_f32 = q.out_f32 ? 1 : 0;
        r.mtiles = (q.R + 127) / 128;
        const bool sp = i < nprob && split[i];
        r.partial = sp ? 1 : 0;
        const int spc = (nst + (sp ? ks : 1) - 1) / (sp ? ks : 1);
        r.nkb_per = spc * p.nbox;
        r.ksplit = (nkb + r.nkb_per - 1) / r.nkb_per;
        if (ksplit_out && i < nprob) ksplit_out[i] = r.ksplit;
        r.units = i < nprob ? L * r.mtiles * r.ksplit : 0;
        total += r.units;
        ok = ok && make_map_2d(&wmap[i], q.W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L * q.R, (uint64_t)K, KB, 128);
    }
    if (!ok) return LSA_ERR_CUDA;
    cudaError_t e = cudaFuncSetAttribute(k_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    const int grid = total < sms ? total : sms;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(dim3((unsigned)grid), dim3(THREADS), smem, st, attr);
    if (!pdl) cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, k_proj_tc, wmap[0], wmap[1], xmap, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

// The partial slices of the split problems summed in slice order: c = sum of pc's k0 slices of n0
// elements, rounded to bf16; w = sum of pw's k1 slices of n1 elements (fp32).
__global__ void __launch_bounds__(256) k_proj_reduce(const float *__restrict__ pc, int k0, int64_t n0,
                                                     __nv_bfloat16 *__restrict__ c, const float *__restrict__ pw,
                                                     int k1, int64_t n1, float *__restrict__ w)
{
    pdl_trigger();
    pdl_wait();  // the partial slices of the previous launch
    // every slice's value loaded before the sum (the loads in flight together), summed in slice order
    auto sum = [](const float *src, int ks, int64_t n, int64_t at) {
        float v[proj::KSPLIT_MAX];
#pragma unroll
        for (int k = 0; k < proj::KSPLIT_MAX; k++) v[k] = k < ks ? __ldg(src + (int64_t)k * n + at) : 0.f;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < proj::KSPLIT_MAX; k++)
            if (k < ks) s += v[k];
        return s;
    };
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n0 + n1; i += (int64_t)gridDim.x * 256) {
        if (i < n0) c[i] = __float2bfloat16_rn(sum(pc, k0, n0, i));
        else w[i - n0] = sum(pw, k1, n1, i - n0);
    }
}

// k_proj_reduce as a programmatic dependent of the previous launch on the stream.
inline cudaError_t launch_proj_reduce(const float *pc, int k0, int64_t n0, __nv_bfloat16 *c, const float *pw, int k1,
                                      int64_t n1, float *w, int sms, cudaStream_t st)
{
    cudaLaunchAttribute attr[1];
    // few enough CTAs to sit beside the previous launch's CTAs while they wait for it
    cudaLaunchConfig_t cfg =
        pdl_config(dim3((unsigned)std::min<int64_t>((n0 + n1 + 255) / 256, (int64_t)sms * 4)), dim3(256), 0, st, attr);
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_proj_reduce, pc, k0, n0, c, pw, k1, n1, w);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace lsa
