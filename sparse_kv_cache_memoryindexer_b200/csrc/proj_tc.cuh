// Stage 1 on tensor cores: the indexer projections of the trigger token (blog review
// "FlashMemory-DeepSeek-V4", section 3.1; hyper.ai summary, "Method"):
//     c = h W^DQ,   q = c W^IUQ,   w = h W^w     for every layer l and sequence b.
// Each is Y[l][b][o] = sum_k X[l][b][k] W[l][o][k] with the weights stored as rows of outputs
// (K contiguous).  The weights dominate the bytes (B is a batch of sequences, at most 256), so
// the weight rows are the MMA A operand (M = 128 output rows per tile, streamed once by TMA) and
// the batch is the B operand (N = B rounded up to 16; the small X tiles are re-read from L2 by
// every CTA).  A tile covers all of K: its accumulator (N fp32 columns of TMEM) is complete when
// the epilogue reads it, which rounds to the output type (bf16 nearest-even, or fp32) and writes
// Y[l][b][o] with consecutive lanes on consecutive o.
//
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2..5 epilogue (one TMEM lane
// quarter each).  Two accumulators, so a tile's epilogue overlaps the next tile's MMAs.  Every
// ring is consumed in order by one consumer (group); waits are bounded as in the other
// tensor-core kernels.
#pragma once
#include "tc_common.cuh"

namespace lsa {

namespace proj {

constexpr int KB = 64;              // K elements per stage (one 128-byte swizzle atom of bf16)
constexpr int MAX_STAGES = 8;
constexpr int THREADS = 6 * 32;
constexpr uint32_t A_BYTES = 128 * KB * 2;

struct Params {
    void *out;          // [L][B][R] bf16 or fp32
    int L, B, R, K;     // layers, batch, output rows, reduction length
    int NB;             // MMA N = B rounded up to 16
    int stages;
    int out_f32;
};

__host__ __device__ inline uint32_t b_bytes(int NB) { return (uint32_t)NB * KB * 2; }
__host__ __device__ inline uint32_t stage_bytes(int NB) { return A_BYTES + b_bytes(NB); }
__host__ __device__ inline uint32_t smem_total(int NB, int stages) { return stage_bytes(NB) * stages + 8 * (2 * MAX_STAGES + 4) + 64 + 1024; }
// TMEM columns per accumulator: N rounded up to 32, so that 32-column loads stay inside it.
__host__ __device__ inline uint32_t acc_cols(int NB) { return (uint32_t)(NB + 31) / 32 * 32; }
__host__ __device__ inline uint32_t tmem_cols(int NB)  // two accumulators, a power of two >= 32
{
    uint32_t c = 32;
    while (c < 2 * acc_cols(NB)) c <<= 1;
    return c;
}

__global__ void __launch_bounds__(THREADS, 1)
    k_proj_tc(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, Params p)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t sbytes = stage_bytes(p.NB);
    const uint32_t bars = sbase + sbytes * p.stages;
    auto full = [&](int i) { return bars + 8u * i; };
    auto empty = [&](int i) { return bars + 8u * (MAX_STAGES + i); };
    auto tfull = [&](int i) { return bars + 8u * (2 * MAX_STAGES + i); };
    auto tempty = [&](int i) { return bars + 8u * (2 * MAX_STAGES + 2 + i); };
    uint8_t *misc = base + sbytes * p.stages + 8 * (2 * MAX_STAGES + 4);
    uint32_t *tmem_holder = (uint32_t *)misc;
    volatile int *abort_flag = (volatile int *)(misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mtiles = (p.R + 127) / 128;
    const int ntiles = p.L * mtiles;
    const int nkb = (p.K + KB - 1) / KB;
    const uint32_t ncols = tmem_cols(p.NB), acol = acc_cols(p.NB);

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
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&wmap) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&xmap) : "memory");
        }
        int stage = 0;
        uint32_t phase = 0;
        uint32_t last_phase[MAX_STAGES];
        bool issued[MAX_STAGES];
        for (int i = 0; i < MAX_STAGES; i++) issued[i] = false;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int l = t / mtiles, m0 = (t % mtiles) * 128;
            for (int kb = 0; kb < nkb; kb++) {
                if (!mbar_wait_warp(empty(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                if (leader) {
                    mbar_expect_tx(full(stage), sbytes);
                    const uint32_t dst = sbase + (uint32_t)stage * sbytes;
                    tma_load_2d(dst, &wmap, kb * KB, l * p.R + m0, full(stage));
                    tma_load_2d(dst + A_BYTES, &xmap, kb * KB, l * p.B, full(stage));
                }
                __syncwarp();
                issued[stage] = true;
                last_phase[stage] = phase;
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
            }
        }
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
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            if (!mbar_wait_warp(tempty(acc), accphase ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)acc * acol;
            for (int kb = 0; kb < nkb; kb++) {
                if (!mbar_wait_warp(full(stage), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_base = sbase + (uint32_t)stage * sbytes;
                const uint32_t b_base = a_base + A_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < KB / 16; kk++)
                        mma_bf16(d, sdesc(a_base + 32 * kk), sdesc(b_base + 32 * kk), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(empty(stage));
                    if (kb == nkb - 1) mma_commit(tfull(acc));
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
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int l = t / mtiles, m0 = (t % mtiles) * 128;
            if (!mbar_wait_warp(tfull(acc), accphase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const int o = m0 + quarter * 32 + lane;
            const bool valid = o < p.R;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)acc * acol;
            for (int b0 = 0; b0 < p.NB; b0 += 32) {
                float v[32];
                tmem_ld32(taddr + b0, v);  // columns past N (up to the accumulator's end) are not stored
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int b = b0 + i;
                    if (valid && b < p.B) {
                        const int64_t at = ((int64_t)l * p.B + b) * p.R + o;
                        if (p.out_f32) ((float *)p.out)[at] = v[i];
                        else ((__nv_bfloat16 *)p.out)[at] = __float2bfloat16_rn(v[i]);
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

// out[l][b][o] = sum_k X[l][b][k] W[l][o][k]; X bf16 [L][B][K], W bf16 [L][R][K], out bf16 or fp32.
inline lsa_status launch_proj_tc(const void *X, const void *W, void *out, bool out_f32, int L, int B, int R, int K,
                                 int sms, cudaStream_t st)
{
    using namespace proj;
    CUtensorMap wmap, xmap;
    proj::Params p;
    p.out = out;
    p.L = L;
    p.B = B;
    p.R = R;
    p.K = K;
    p.NB = (B + 15) / 16 * 16;
    p.out_f32 = out_f32 ? 1 : 0;
    bool ok = make_map_2d(&wmap, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L * R, (uint64_t)K, KB, 128);
    ok = ok && make_map_2d(&xmap, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L * B, (uint64_t)K, KB, (uint32_t)p.NB);
    if (!ok) return LSA_ERR_CUDA;
    const uint32_t max_smem = 227 * 1024;
    p.stages = MAX_STAGES;
    while (p.stages > 2 && smem_total(p.NB, p.stages) > max_smem) p.stages--;
    const uint32_t smem = smem_total(p.NB, p.stages);
    if (smem > max_smem) return LSA_ERR_UNSUPPORTED;
    cudaError_t e = cudaFuncSetAttribute(k_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    const int ntiles = L * ((R + 127) / 128);
    k_proj_tc<<<ntiles < sms ? ntiles : sms, THREADS, smem, st>>>(wmap, xmap, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa
