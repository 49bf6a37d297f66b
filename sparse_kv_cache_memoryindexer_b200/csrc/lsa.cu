// C ABI of the LSA indexer hot path (declared in include/lsa.h).  Host-side validation and
// dispatch; every stage runs in the kernels included below (one translation unit).
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/lsa.h"
#include "common.cuh"
#include "gather.cuh"
#include "project.cuh"
#include "score_select.cuh"
#include "score_tc.cuh"
#include "score_pair.cuh"
#include "li_tc.cuh"
#include "proj_tc.cuh"
#include "golden.cuh"
#include "train.cuh"
#include "train_tc.cuh"
#include "step_select.cuh"
#include "topk.cuh"
#include "selftest.cuh"

using namespace lsa;

namespace {

thread_local char g_msg[512] = "";
std::atomic<uint64_t> g_launches{0};

lsa_status fail(lsa_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return st;
}

lsa_status ok()
{
    g_msg[0] = '\0';
    return LSA_OK;
}

// After a launch: count it and turn a launch error into LSA_ERR_CUDA.
lsa_status launched(const char *what)
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return LSA_OK;
}

#define LSA_TRY(x)                            \
    do {                                      \
        lsa_status _st = (x);                 \
        if (_st != LSA_OK) return _st;        \
    } while (0)

#define LSA_REQUIRE(cond, ...)                                        \
    do {                                                              \
        if (!(cond)) return fail(LSA_ERR_INVALID_ARG, __VA_ARGS__);   \
    } while (0)

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t elem_bytes(int dt) { return dt == DT_F32 ? 4 : (dt == DT_BF16 ? 2 : 1); }

int num_sms()
{
    static thread_local int cached_dev = -1, cached_sms = 148;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != cached_dev) {
        cudaDeviceGetAttribute(&cached_sms, cudaDevAttrMultiProcessorCount, dev);
        cached_dev = dev;
    }
    return cached_sms;
}

// Workspace layout of lsa_memindex_score_select:
//   tile_start [B+1] int, chunk_start [B+1] int | tile_mask [max_tiles][4] u32 |
//   qh [L*B][128][128] E4M3 | wh [L*B*64] fp32
// (qh / wh: the split queries and scaled head weights of the E4M3 tensor-core path).
struct ScoreWs {
    int *tile_start;
    int *chunk_start;
    uint32_t *tile_mask;
    void *qh;
    float *wh;
};

int64_t max_tiles(int B, int64_t T) { return T / TILE + B + 1; }

size_t score_ws_parts(int L, int B, int64_t T, size_t part[4])
{
    part[0] = align_up(sizeof(int) * (size_t)(2 * B + 2), 256);  // tile starts, compaction chunk starts
    part[1] = align_up((size_t)max_tiles(B, T) * 16, 256);
    part[2] = align_up((size_t)L * B * 64 * 128 * 2, 256);
    part[3] = align_up((size_t)L * B * 64 * 4, 256);
    return part[0] + part[1] + part[2] + part[3];
}

size_t score_ws_bytes(int L, int B, int64_t T)
{
    size_t part[4];
    return score_ws_parts(L, B, T, part);
}

ScoreWs score_ws(void *ws, int L, int B, int64_t T)
{
    size_t part[4];
    score_ws_parts(L, B, T, part);
    char *p = (char *)ws;
    ScoreWs w;
    w.tile_start = (int *)p;
    w.chunk_start = (int *)p + (B + 1);
    w.tile_mask = (uint32_t *)(p + part[0]);
    w.qh = (void *)(p + part[0] + part[1]);
    w.wh = (float *)(p + part[0] + part[1] + part[2]);
    return w;
}

// Dynamic shared memory of a launch: the limit is set explicitly (static plus dynamic above 48 KB
// needs it even when the dynamic part alone is below 48 KB).
template <typename K>
lsa_status set_smem(K kernel, size_t bytes)
{
    if (bytes > 0) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    return LSA_OK;
}

// ---------------------------------------------------------------- SIMT score dispatch
template <int D, int KDT, int QDT>
lsa_status launch_score_simt(const void *q, const float *w, const void *K, const float *ks, const int64_t *offs,
                             const int *tile_start, int B, int64_t T, int L, int n_h, float thr,
                             float *scores, uint32_t *tile_mask, cudaStream_t st)
{
    const size_t smem = sizeof(float) * (size_t)(n_h * D + n_h);
    LSA_TRY(set_smem(k_score_simt<D, KDT, QDT>, smem));
    const int64_t grid = max_tiles(B, T);
    k_score_simt<D, KDT, QDT><<<(unsigned)grid, TILE, smem, st>>>(q, w, K, ks, offs, tile_start, B, T, L, n_h, thr,
                                                                  scores, tile_mask);
    return launched("score (SIMT)");
}

template <int D>
lsa_status score_simt_d(int kdt, const void *q, const float *w, const void *K, const float *ks, const int64_t *offs,
                        const int *tile_start, int B, int64_t T, int L, int n_h, float thr, float *scores,
                        uint32_t *tile_mask, cudaStream_t st)
{
    switch (kdt) {
    case DT_F32:
        return launch_score_simt<D, DT_F32, DT_F32>(q, w, K, ks, offs, tile_start, B, T, L, n_h, thr, scores,
                                                    tile_mask, st);
    case DT_BF16:
        return launch_score_simt<D, DT_BF16, DT_BF16>(q, w, K, ks, offs, tile_start, B, T, L, n_h, thr, scores,
                                                      tile_mask, st);
    default:
        return launch_score_simt<D, DT_FP8, DT_BF16>(q, w, K, ks, offs, tile_start, B, T, L, n_h, thr, scores,
                                                     tile_mask, st);
    }
}

template <int D, int KDT, int QDT>
lsa_status launch_li_simt(const void *qd, const float *wd, const void *hotK, const float *hotsc,
                          const int32_t *count, const int64_t *offs, int B, int64_t T, int tau, int n_h, float *Y,
                          cudaStream_t st)
{
    const size_t smem = sizeof(float) * (size_t)(n_h * D + n_h);
    LSA_TRY(set_smem(k_li_score_simt<D, KDT, QDT>, smem));
    int64_t gx = (T + TILE - 1) / TILE;
    int64_t cap = (int64_t)num_sms() * 8 / (B > 0 ? B : 1) + 1;
    if (gx > cap) gx = cap;
    if (gx < 1) gx = 1;
    dim3 grid((unsigned)gx, (unsigned)B);
    k_li_score_simt<D, KDT, QDT><<<grid, TILE, smem, st>>>(qd, wd, hotK, hotsc, count, offs, tau, n_h, Y);
    return launched("lightning score (SIMT)");
}

template <int D>
lsa_status li_simt_d(int kdt, const void *qd, const float *wd, const void *hotK, const float *hotsc,
                     const int32_t *count, const int64_t *offs, int B, int64_t T, int tau, int n_h, float *Y,
                     cudaStream_t st)
{
    switch (kdt) {
    case DT_F32: return launch_li_simt<D, DT_F32, DT_F32>(qd, wd, hotK, hotsc, count, offs, B, T, tau, n_h, Y, st);
    default:
        return launch_li_simt<D, DT_BF16, DT_BF16>(qd, wd, hotK, hotsc, count, offs, B, T, tau, n_h, Y, st);
    }
}

// The E4M3 score runs on CTA pairs unless LSA_SCORE_PAIR=0 (the one-CTA kernel, k_score_tc, the
// same result; read at every call, so the two kernels can be cross-checked in one process).
bool score_pair_enabled()
{
    const char *v = getenv("LSA_SCORE_PAIR");
    return !(v && v[0] == '0');
}

bool valid_dtype(int dt) { return dt == DT_F32 || dt == DT_BF16 || dt == DT_FP8; }

}  // namespace

extern "C" {

const char *lsa_last_error(void) { return g_msg; }

const char *lsa_version(void) { return "lsa-b200 0.1 (sm_100a)"; }

uint64_t lsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

lsa_status lsa_check_device(lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    unsigned int word = 0;
    e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof(word));
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    if (word == 0) return ok();
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "clearing the device error word: %s", cudaGetErrorString(e));
    return fail(LSA_ERR_DEVICE_CHECK, "device check flags 0x%x:%s%s%s%s%s", word,
                (word & ERRF_OFFSETS) ? " bad-seq-offsets" : "", (word & ERRF_INDEX) ? " index-out-of-range" : "",
                (word & ERRF_COUNT) ? " count-out-of-range" : "", (word & ERRF_SCALE) ? " bad-key-scale" : "",
                (word & ERRF_TIMEOUT) ? " pipeline-wait-timeout" : "");
}

lsa_status lsa_selftest_wait_timeout(int32_t *status_out, lsa_stream_t stream)
{
    LSA_REQUIRE(status_out, "lsa_selftest_wait_timeout: null pointer");
    k_selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>(status_out);
    LSA_TRY(launched("self-test: bounded wait"));
    return ok();
}

// ------------------------------------------------------------------------------ stage 1

// Workspace of lsa_project: c in the storage type [L][B][r], then its fp32 sums [L][B][r] (the
// tensor-core path adds the partial sums of its K ranges there before rounding c once).
size_t lsa_project_workspace_size(int L, int B, int d, int r, int n_h, int d_I, lsa_dtype dt)
{
    (void)d;
    if (L <= 0 || B <= 0 || r <= 0 || n_h <= 0 || d_I <= 0) return 0;
    // c in its storage type, then the fp32 partial slices of c and w (K split in at most KSPLIT_MAX),
    // which the partial slices of q reuse once c and w are summed
    const size_t cw = align_up((size_t)proj::KSPLIT_MAX * L * B * r * 4, 256) +
                      align_up((size_t)proj::KSPLIT_MAX * L * B * n_h * 4, 256);
    const size_t qs = align_up((size_t)proj::KSPLIT_MAX * L * B * n_h * d_I * 4, 256);
    return align_up((size_t)L * B * r * elem_bytes(dt), 256) + (cw > qs ? cw : qs);
}

lsa_status lsa_project(const void *h, const void *W_dq, const void *W_iuq, const void *W_w, lsa_dtype dt,
                       int L, int B, int d, int r, int n_h, int d_I, void *q_out, float *w_out, void *workspace,
                       size_t workspace_bytes, lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(h && W_dq && W_iuq && W_w && q_out && w_out, "lsa_project: null pointer");
    LSA_REQUIRE(L > 0 && B > 0 && d > 0 && r > 0 && n_h > 0 && d_I > 0, "lsa_project: sizes must be positive");
    if (dt != LSA_F32 && dt != LSA_BF16) return fail(LSA_ERR_UNSUPPORTED, "lsa_project: dt must be F32 or BF16");
    LSA_REQUIRE(d % 8 == 0 && r % 8 == 0, "lsa_project: d and r must be multiples of 8");
    LSA_REQUIRE(aligned(h, 16) && aligned(W_dq, 16) && aligned(W_iuq, 16) && aligned(W_w, 16),
                "lsa_project: h and weights must be 16-byte aligned");
    const size_t need = lsa_project_workspace_size(L, B, d, r, n_h, d_I, dt);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_project: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_project: workspace must be 256-byte aligned");
    const int nq = n_h * d_I;
    void *c = workspace;
    if (proj_tc_supported(dt, B, d) && proj_tc_supported(dt, B, r)) {
        // c and w in one launch, split along d so that every SM streams weights (fp32 partial sums
        // in slices of their own); the slices summed in order, c rounded to bf16 once; then q,
        // split along r the same way when it has fewer tiles than SMs.  Every launch after the
        // first is a programmatic dependent of the one before (the q launch streams its first
        // weight stages while c is summed).
        const int sms = num_sms();
        const int64_t nc = (int64_t)L * B * r, nw = (int64_t)L * B * n_h, nqt = (int64_t)L * B * nq;
        float *pc = (float *)((char *)workspace + align_up((size_t)nc * elem_bytes(dt), 256));
        float *pw = (float *)((char *)pc + align_up((size_t)proj::KSPLIT_MAX * nc * 4, 256));
        const ProjProblem cw[2] = {{W_dq, pc, r, true}, {W_w, pw, n_h, true}};
        const bool split[2] = {true, true};
        int ks[2] = {1, 1};
        lsa_status s = launch_proj_tc(h, cw, split, 2, L, B, d, sms, st, ks);
        if (s == LSA_OK) s = launched("project c and w (tensor cores)");
        if (s == LSA_OK && launch_proj_reduce(pc, ks[0], nc, (__nv_bfloat16 *)c, pw, ks[1], nw, w_out, sms, st) !=
                               cudaSuccess)
            s = LSA_ERR_CUDA;
        if (s == LSA_OK) s = launched("project: reduce c and w");
        // (q is split only when its tiles leave SMs idle: measured at 192 tiles on 148 SMs, the split's
        // better balance did not pay for the slice sums)
        const int64_t qtiles = (int64_t)L * ((nq + 127) / 128);
        const bool qsplit = qtiles < sms && proj_ksplit(qtiles, proj_stages_of_k(B, r), sms) > 1;
        const ProjProblem qp = {W_iuq, qsplit ? (void *)pc : q_out, nq, false};  // (pc: summed already)
        int kq = 1;
        if (s == LSA_OK) s = launch_proj_tc(c, &qp, &qsplit, 1, L, B, r, sms, st, &kq, true);
        if (s == LSA_OK) s = launched("project q (tensor cores)");
        if (s == LSA_OK && qsplit &&
            launch_proj_reduce(pc, kq, nqt, (__nv_bfloat16 *)q_out, nullptr, 0, 0, nullptr, sms, st) != cudaSuccess)
            s = LSA_ERR_CUDA;
        if (s == LSA_OK && qsplit) s = launched("project: reduce q");
        if (s != LSA_OK) return fail(s, "lsa_project: tensor-core launch failed (%s)", cudaGetErrorString(cudaGetLastError()));
    } else if (dt == LSA_BF16) {
        k_rowdot<DT_BF16, DT_BF16><<<dim3((r + 7) / 8, L), 256, 0, st>>>(h, W_dq, c, B, d, r);
        LSA_TRY(launched("project c"));
        k_rowdot<DT_BF16, DT_F32><<<dim3((n_h + 7) / 8, L), 256, 0, st>>>(h, W_w, w_out, B, d, n_h);
        LSA_TRY(launched("project w"));
        k_rowdot<DT_BF16, DT_BF16><<<dim3((nq + 7) / 8, L), 256, 0, st>>>(c, W_iuq, q_out, B, r, nq);
        LSA_TRY(launched("project q"));
    } else {
        k_rowdot<DT_F32, DT_F32><<<dim3((r + 7) / 8, L), 256, 0, st>>>(h, W_dq, c, B, d, r);
        LSA_TRY(launched("project c"));
        k_rowdot<DT_F32, DT_F32><<<dim3((n_h + 7) / 8, L), 256, 0, st>>>(h, W_w, w_out, B, d, n_h);
        LSA_TRY(launched("project w"));
        k_rowdot<DT_F32, DT_F32><<<dim3((nq + 7) / 8, L), 256, 0, st>>>(c, W_iuq, q_out, B, r, nq);
        LSA_TRY(launched("project q"));
    }
    return ok();
}

// ------------------------------------------------------------------------------ stages 2-4a

size_t lsa_score_select_workspace_size(int L, int B, int64_t total_S)
{
    if (L <= 0 || B <= 0 || total_S < 0) return 0;
    return score_ws_bytes(L, B, total_S);
}

lsa_status lsa_memindex_score_select(const void *q, const float *w, const void *K, const float *k_scale,
                                     lsa_dtype kdt, const int64_t *seq_offsets, int64_t total_S, int L, int B,
                                     int n_h, int d_I, float threshold, float *scores_out, uint8_t *mask_out,
                                     int32_t *idx_out, int32_t *count_out, void *workspace,
                                     size_t workspace_bytes, lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(q && w && K && seq_offsets && idx_out && count_out, "lsa_memindex_score_select: null pointer");
    LSA_REQUIRE(L > 0 && B > 0 && n_h > 0 && d_I > 0 && total_S >= 0,
                "lsa_memindex_score_select: sizes must be positive");
    LSA_REQUIRE(total_S < (int64_t)1 << 31, "lsa_memindex_score_select: total_S must be below 2^31");
    if (!valid_dtype(kdt)) return fail(LSA_ERR_UNSUPPORTED, "lsa_memindex_score_select: unknown key dtype");
    LSA_REQUIRE((kdt == LSA_FP8_E4M3) == (k_scale != nullptr),
                "lsa_memindex_score_select: k_scale is required for FP8 keys and must be NULL otherwise");
    LSA_REQUIRE(threshold > 0.f && threshold < 1.f, "lsa_memindex_score_select: threshold must be in (0, 1)");
    const size_t need = score_ws_bytes(L, B, total_S);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_memindex_score_select: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_memindex_score_select: workspace must be 256-byte aligned");
    const float thr_logit = (float)log((double)threshold / (1.0 - (double)threshold));
    ScoreWs ws = score_ws(workspace, L, B, total_S);

    const bool tc = (n_h == 64 && d_I == 128 && L <= tc::MAX_L_TC && (kdt == LSA_BF16 || kdt == LSA_FP8_E4M3) &&
                     tc_score_available());
    if (tc) LSA_REQUIRE(aligned(q, 16) && aligned(K, 16), "lsa_memindex_score_select: q and K must be 16-byte aligned");
    if (!(tc && kdt == LSA_FP8_E4M3)) {  // (the E4M3 tensor-core path does the setup in its query split)
        k_tile_setup<<<1, 1024, 0, st>>>(seq_offsets, B, total_S, ws.tile_start, ws.chunk_start, count_out);
        LSA_TRY(launched("tile setup"));
    }
    if (tc && kdt == LSA_FP8_E4M3 && score_pair_enabled() && score_pair_supported(DT_FP8, B, num_sms())) {
        // E4M3 keys on CTA pairs (score_pair.cuh): the query split (with the tile setup), then the score
        const int R = L * B * tc::NH;
        tc::k_q_split_e4m3<<<(R + 7) / 8 + 1, 256, 0, st>>>((const __nv_bfloat16 *)q, w, (uint8_t *)ws.qh, ws.wh, R,
                                                            seq_offsets, B, total_S, ws.tile_start, ws.chunk_start,
                                                            count_out);
        LSA_TRY(launched("E4M3 query split"));
        const lsa_status s = launch_score_pair(ws.qh, ws.wh, K, k_scale, seq_offsets, ws.tile_start, B, total_S, L,
                                               thr_logit, scores_out, ws.tile_mask, num_sms(), st);
        if (s != LSA_OK) return fail(s, "lsa_memindex_score_select: CTA-pair launch failed (%s)",
                                     cudaGetErrorString(cudaGetLastError()));
        LSA_TRY(launched("index score (CTA pairs)"));
    } else if (tc) {
        int n = 0;
        const lsa_status s = launch_score_tc(q, w, K, k_scale, kdt, seq_offsets, ws.tile_start, ws.chunk_start,
                                             count_out, B, total_S, L, thr_logit, scores_out, ws.tile_mask, ws.qh,
                                             ws.wh, num_sms(), st, &n);
        g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed);
        if (s != LSA_OK) return fail(s, "lsa_memindex_score_select: tensor-core launch failed (%s)",
                                     cudaGetErrorString(cudaGetLastError()));
    } else {
        if (n_h > 128) return fail(LSA_ERR_UNSUPPORTED, "lsa_memindex_score_select: n_h must be <= 128");
        switch (d_I) {
        case 32: LSA_TRY(score_simt_d<32>(kdt, q, w, K, k_scale, seq_offsets, ws.tile_start, B, total_S, L, n_h,
                                          thr_logit, scores_out, ws.tile_mask, st)); break;
        case 64: LSA_TRY(score_simt_d<64>(kdt, q, w, K, k_scale, seq_offsets, ws.tile_start, B, total_S, L, n_h,
                                          thr_logit, scores_out, ws.tile_mask, st)); break;
        case 128: LSA_TRY(score_simt_d<128>(kdt, q, w, K, k_scale, seq_offsets, ws.tile_start, B, total_S, L, n_h,
                                            thr_logit, scores_out, ws.tile_mask, st)); break;
        default: return fail(LSA_ERR_UNSUPPORTED, "lsa_memindex_score_select: d_I must be 32, 64 or 128");
        }
    }
    const int64_t chunks = (max_tiles(B, total_S) + COMPACT_TILES - 1) / COMPACT_TILES + B;
    k_compact<<<(unsigned)chunks, COMPACT_THREADS, 0, st>>>(ws.tile_mask, ws.tile_start, ws.chunk_start, seq_offsets,
                                                          B, idx_out, count_out, mask_out);
    LSA_TRY(launched("compact"));
    return ok();
}

// ------------------------------------------------------------------------------ stage 4b

lsa_status lsa_fetch_gather(const int32_t *idx, const int32_t *count, const int64_t *seq_offsets, int64_t total_S,
                            int B, const void *pool, size_t row_bytes, void *hot_kv, const void *K_sel,
                            const float *k_scale_sel, lsa_dtype kdt, int d_I, void *hot_K, float *hot_scale,
                            lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(idx && count && seq_offsets, "lsa_fetch_gather: null pointer");
    LSA_REQUIRE((pool == nullptr) == (hot_kv == nullptr), "lsa_fetch_gather: pool and hot_kv are given together");
    LSA_REQUIRE(pool || K_sel, "lsa_fetch_gather: nothing to gather (pool and K_sel are both NULL)");
    LSA_REQUIRE(B > 0 && total_S >= 0, "lsa_fetch_gather: sizes must be positive");
    void *dpool = nullptr;
    if (pool) {
        LSA_REQUIRE(row_bytes > 0 && row_bytes % 16 == 0,
                    "lsa_fetch_gather: row_bytes must be a positive multiple of 16");
        if (row_bytes > 16 * 32 * GATHER_MAX_CHUNKS)
            return fail(LSA_ERR_UNSUPPORTED, "lsa_fetch_gather: row_bytes above %d", 16 * 32 * GATHER_MAX_CHUNKS);
        LSA_REQUIRE(aligned(pool, 16) && aligned(hot_kv, 16),
                    "lsa_fetch_gather: pool and hot_kv must be 16-byte aligned");
        cudaError_t e = cudaHostGetDevicePointer(&dpool, const_cast<void *>(pool), 0);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(LSA_ERR_INVALID_ARG, "lsa_fetch_gather: pool is not mapped page-locked host memory (%s)",
                        cudaGetErrorString(e));
        }
    }
    int krow16 = 0;
    if (K_sel) {
        if (!valid_dtype(kdt)) return fail(LSA_ERR_UNSUPPORTED, "lsa_fetch_gather: unknown key dtype");
        LSA_REQUIRE(hot_K && d_I > 0, "lsa_fetch_gather: hot_K and d_I are required with K_sel");
        LSA_REQUIRE((kdt == LSA_FP8_E4M3) == (k_scale_sel != nullptr) && (!k_scale_sel || hot_scale),
                    "lsa_fetch_gather: scales are required for FP8 keys (and only for them)");
        const size_t kb = (size_t)d_I * elem_bytes(kdt);
        LSA_REQUIRE(kb % 16 == 0 && aligned(K_sel, 16) && aligned(hot_K, 16),
                    "lsa_fetch_gather: key rows must be whole 16-byte chunks, 16-byte aligned");
        krow16 = (int)(kb / 16);
        if (kdt == LSA_FP8_E4M3 && krow16 > 32)
            return fail(LSA_ERR_UNSUPPORTED, "lsa_fetch_gather: E4M3 key rows above 512 bytes");
    }
    const int row16 = pool ? (int)(row_bytes / 16) : 0;
    if (pool && !K_sel && B <= GATHER_ROWS_MAX_B) {
        // rows only: a small launch meant to run beside other work (see k_gather_rows)
        const size_t smem = sizeof(int) * (size_t)(B + 1);
        const dim3 grid(GATHER_LINK_CTAS);
        const uint8_t *src = (const uint8_t *)dpool;
        if (row16 <= 32) k_gather_rows<1><<<grid, link_threads<1>(), smem, st>>>(idx, count, seq_offsets, B, src, row16, (uint8_t *)hot_kv);
        else if (row16 <= 64) k_gather_rows<2><<<grid, link_threads<2>(), smem, st>>>(idx, count, seq_offsets, B, src, row16, (uint8_t *)hot_kv);
        else k_gather_rows<4><<<grid, link_threads<4>(), smem, st>>>(idx, count, seq_offsets, B, src, row16, (uint8_t *)hot_kv);
        LSA_TRY(launched("gather rows"));
        return ok();
    }
    if (!pool && B <= GATHER_ROWS_MAX_B) {
        // keys only: one thread per 16-byte chunk of every fetched key row
        const size_t smem = sizeof(int) * (size_t)(B + 1);
        k_gather_keys<<<num_sms() * 8, 128, smem, st>>>(idx, count, seq_offsets, B, (const uint8_t *)K_sel, k_scale_sel,
                                                        krow16, kdt == LSA_FP8_E4M3, (uint8_t *)hot_K, hot_scale);
        LSA_TRY(launched("gather keys"));
        return ok();
    }
    const int warps_per_block = 8;
    int64_t gx = ((total_S / (B > 0 ? B : 1)) + warps_per_block * GATHER_ROWS_PER_WARP - 1) /
                 (warps_per_block * GATHER_ROWS_PER_WARP);
    const int64_t cap = (int64_t)num_sms() * 4 / B + 1;
    if (gx > cap) gx = cap;
    if (gx < 1) gx = 1;
    k_gather<<<dim3((unsigned)gx, (unsigned)B), 32 * warps_per_block, 0, st>>>(
        idx, count, seq_offsets, (const uint8_t *)dpool, row16, (uint8_t *)hot_kv,
        (const uint8_t *)K_sel, k_scale_sel, krow16, kdt == LSA_FP8_E4M3, (uint8_t *)hot_K, hot_scale);
    LSA_TRY(launched("gather"));
    return ok();
}

// ------------------------------------------------------------------------------ stage 4b, incremental

// Workspace of lsa_fetch_gather_incremental: [map: total_S int32][miss: total_S int32][miss count].
size_t lsa_fetch_incremental_workspace_size(int B, int64_t total_S)
{
    if (B <= 0 || total_S < 0) return 0;
    return 2 * align_up(sizeof(int32_t) * (size_t)(total_S > 0 ? total_S : 1), 256) + 256;
}

lsa_status lsa_fetch_gather_incremental(const int32_t *idx, const int32_t *count, const int64_t *seq_offsets,
                                        int64_t total_S, int B, const int32_t *prev_idx, const int32_t *prev_count,
                                        const int64_t *prev_seq_offsets, int64_t prev_total_S,
                                        const void *prev_hot_kv, const void *pool, size_t row_bytes, void *hot_kv,
                                        int32_t *host_rows_out, void *workspace, size_t workspace_bytes,
                                        lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(idx && count && seq_offsets && prev_idx && prev_count && prev_seq_offsets && prev_hot_kv && pool &&
                    hot_kv,
                "lsa_fetch_gather_incremental: null pointer");
    LSA_REQUIRE(B > 0 && total_S >= 0 && prev_total_S >= 0, "lsa_fetch_gather_incremental: sizes must be positive");
    LSA_REQUIRE(total_S < (int64_t)1 << 31, "lsa_fetch_gather_incremental: total_S must be below 2^31");
    if (B > GATHER_ROWS_MAX_B)
        return fail(LSA_ERR_UNSUPPORTED, "lsa_fetch_gather_incremental: at most %d sequences", GATHER_ROWS_MAX_B);
    LSA_REQUIRE(row_bytes > 0 && row_bytes % 16 == 0 && row_bytes <= 16 * 32 * GATHER_MAX_CHUNKS,
                "lsa_fetch_gather_incremental: row_bytes must be a multiple of 16, at most %d",
                16 * 32 * GATHER_MAX_CHUNKS);
    LSA_REQUIRE(aligned(pool, 16) && aligned(hot_kv, 16) && aligned(prev_hot_kv, 16),
                "lsa_fetch_gather_incremental: row buffers must be 16-byte aligned");
    {
        const uintptr_t a0 = (uintptr_t)hot_kv, a1 = a0 + (uintptr_t)total_S * row_bytes;
        const uintptr_t b0 = (uintptr_t)prev_hot_kv, b1 = b0 + (uintptr_t)prev_total_S * row_bytes;
        LSA_REQUIRE(a1 <= b0 || b1 <= a0, "lsa_fetch_gather_incremental: hot_kv and prev_hot_kv overlap");
    }
    const size_t need = lsa_fetch_incremental_workspace_size(B, total_S);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_fetch_gather_incremental: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_fetch_gather_incremental: workspace must be 256-byte aligned");
    void *dpool = nullptr;
    cudaError_t e = cudaHostGetDevicePointer(&dpool, const_cast<void *>(pool), 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(LSA_ERR_INVALID_ARG, "lsa_fetch_gather_incremental: pool is not mapped page-locked host memory (%s)",
                    cudaGetErrorString(e));
    }
    const size_t part = align_up(sizeof(int32_t) * (size_t)(total_S > 0 ? total_S : 1), 256);
    int32_t *map = (int32_t *)workspace;
    int32_t *miss = (int32_t *)((char *)workspace + part);
    int *nmiss = (int *)((char *)workspace + 2 * part);
    e = cudaMemsetAsync(nmiss, 0, sizeof(int), st);
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "lsa_fetch_gather_incremental: %s", cudaGetErrorString(e));
    const size_t smem = sizeof(int) * (size_t)(B + 1);
    const int row16 = (int)(row_bytes / 16);
    const int sms = num_sms();
    k_incr_map<<<sms * 4, 128, smem, st>>>(idx, count, seq_offsets, B, prev_idx, prev_count, prev_seq_offsets, map, miss,
                                           nmiss);
    LSA_TRY(launched("incremental fetch: lookup"));
    // the host rows first: their launch takes its few SMs before the other stream's kernels fill the rest
    const uint8_t *src = (const uint8_t *)dpool;
    if (row16 <= 32)
        k_incr_fetch<1><<<GATHER_LINK_CTAS, link_threads<1>(), smem, st>>>(idx, count, seq_offsets, B, miss, nmiss, src, row16,
                                                             (uint8_t *)hot_kv, host_rows_out);
    else if (row16 <= 64)
        k_incr_fetch<2><<<GATHER_LINK_CTAS, link_threads<2>(), smem, st>>>(idx, count, seq_offsets, B, miss, nmiss, src, row16,
                                                             (uint8_t *)hot_kv, host_rows_out);
    else
        k_incr_fetch<4><<<GATHER_LINK_CTAS, link_threads<4>(), smem, st>>>(idx, count, seq_offsets, B, miss, nmiss, src, row16,
                                                             (uint8_t *)hot_kv, host_rows_out);
    LSA_TRY(launched("incremental fetch: host rows"));
        if (row16 <= 32)
        k_incr_copy<1><<<sms * 4, 256, smem, st>>>(count, seq_offsets, B, prev_seq_offsets, map, (const uint8_t *)prev_hot_kv,
                                                   row16, (uint8_t *)hot_kv);
    else if (row16 <= 64)
        k_incr_copy<2><<<sms * 4, 256, smem, st>>>(count, seq_offsets, B, prev_seq_offsets, map, (const uint8_t *)prev_hot_kv,
                                                   row16, (uint8_t *)hot_kv);
    else
        k_incr_copy<4><<<sms * 4, 256, smem, st>>>(count, seq_offsets, B, prev_seq_offsets, map, (const uint8_t *)prev_hot_kv,
                                                   row16, (uint8_t *)hot_kv);
    LSA_TRY(launched("incremental fetch: device copy"));
return ok();
}

// ------------------------------------------------------------------------------ stage 5

// Workspace of lsa_lightning_topk: [item_start: B+1 ints, item counter: 1 int][item table]
// [Y: tau * total_S floats].
static size_t topk_items_bytes(int B, int tau, int64_t total_S)
{
    return align_up(sizeof(ItemInfo) * (size_t)li_max_items(B, total_S, tau < li::NQ ? li::NQ : tau, li::NQ), 256);
}

size_t lsa_lightning_topk_workspace_size(int B, int tau, int64_t total_S, int k)
{
    (void)k;
    if (B <= 0 || tau <= 0 || total_S < 0) return 0;
    return align_up(sizeof(int) * (size_t)(B + 2), 256) + topk_items_bytes(B, tau, total_S) +
           align_up(sizeof(float) * (size_t)tau * (size_t)total_S, 256);
}

lsa_status lsa_lightning_topk(const void *q_dec, const float *w_dec, const void *hot_K, const float *hot_scale,
                              lsa_dtype kdt, const int32_t *idx, const int32_t *count, const int64_t *seq_offsets,
                              int64_t total_S, int B, int tau, int n_h, int d_I, int k, int32_t *topk_idx,
                              float *topk_score, void *workspace, size_t workspace_bytes, lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(q_dec && w_dec && hot_K && idx && count && seq_offsets && topk_idx, "lsa_lightning_topk: null pointer");
    LSA_REQUIRE(B > 0 && tau > 0 && n_h > 0 && d_I > 0 && total_S >= 0, "lsa_lightning_topk: sizes must be positive");
    LSA_REQUIRE(k >= 1 && k <= LSA_MAX_TOPK, "lsa_lightning_topk: k must be in [1, %d]", LSA_MAX_TOPK);
    if (!valid_dtype(kdt)) return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk: unknown key dtype");
    LSA_REQUIRE((kdt == LSA_FP8_E4M3) == (hot_scale != nullptr),
                "lsa_lightning_topk: hot_scale is required for FP8 keys and must be NULL otherwise");
    const size_t need = lsa_lightning_topk_workspace_size(B, tau, total_S, k);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_lightning_topk: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_lightning_topk: workspace must be 256-byte aligned");
    LSA_REQUIRE((int64_t)tau * total_S < ((int64_t)1 << 40), "lsa_lightning_topk: tau * total_S too large");
    if (n_h > 128) return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk: n_h must be <= 128");
    int *item_start = (int *)workspace;
    int *item_counter = item_start + B + 1;
    ItemInfo *items = (ItemInfo *)((char *)workspace + align_up(sizeof(int) * (size_t)(B + 2), 256));
    float *Y = (float *)((char *)items + topk_items_bytes(B, tau, total_S));
    // E4M3 keys arrive here decoded to bf16 by lsa_fetch_gather (scales in hot_scale)
    const int hdt = (kdt == LSA_FP8_E4M3) ? (int)DT_BF16 : (int)kdt;
    if (li_tc_supported(n_h, d_I, tau, kdt)) {
        LSA_REQUIRE(aligned(q_dec, 16) && aligned(hot_K, 16), "lsa_lightning_topk: q_dec and hot_K must be 16-byte aligned");
        int n = 0;
        const lsa_status s = launch_li_tc(q_dec, w_dec, hot_K, hot_scale, count, seq_offsets, B, total_S, tau, li::NQ,
                                          Y, item_start, item_counter, items, num_sms(), st, &n);
        g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed);
        if (s != LSA_OK) return fail(s, "lsa_lightning_topk: tensor-core launch failed (%s)", cudaGetErrorString(cudaGetLastError()));
    } else {
        switch (d_I) {
        case 32: LSA_TRY(li_simt_d<32>(hdt, q_dec, w_dec, hot_K, hot_scale, count, seq_offsets, B, total_S, tau, n_h, Y, st)); break;
        case 64: LSA_TRY(li_simt_d<64>(hdt, q_dec, w_dec, hot_K, hot_scale, count, seq_offsets, B, total_S, tau, n_h, Y, st)); break;
        case 128: LSA_TRY(li_simt_d<128>(hdt, q_dec, w_dec, hot_K, hot_scale, count, seq_offsets, B, total_S, tau, n_h, Y, st)); break;
        default: return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk: d_I must be 32, 64 or 128");
        }
    }
    int kpow2 = 64;  // the block sort works on at least 64 keys
    while (kpow2 < k) kpow2 <<= 1;
    const size_t smem = topk_select_smem(kpow2);
    LSA_TRY(set_smem(k_topk_select, smem));
    k_topk_select<<<(unsigned)((int64_t)B * tau), SEL_THREADS, smem, st>>>(Y, idx, count, seq_offsets, tau, k, kpow2,
                                                                  topk_idx, topk_score);
    LSA_TRY(launched("top-k select"));
    return ok();
}

// ------------------------------------------------------------------------------ stage 5, one decode step

// Workspace of lsa_lightning_topk_step: [item_start B+1, counter][item table][Y: total_S]
// [tail: B * W][queries: B * n_h * d_I (4-byte elements)][weights: B * n_h][select: histograms
// B * HB, chunk starts B+1, the query of each chunk, state B * NS, the selections B * LSA_MAX_TOPK,
// the stages total_S + B * W].
static int64_t step_max_chunks(int B, int64_t total_S, int W)
{
    return (total_S + (int64_t)B * W) / stepsel::CH + B + 1;
}

static size_t step_sel_parts(int B, int64_t total_S, int W, size_t sp[6])
{
    sp[0] = align_up(sizeof(int) * (size_t)B * stepsel::HB, 256);
    sp[1] = align_up(sizeof(int) * (size_t)(B + 1), 256);
    sp[2] = align_up(sizeof(int) * (size_t)step_max_chunks(B, total_S, W), 256);
    sp[3] = align_up(sizeof(uint32_t) * stepsel::NS * (size_t)B, 256);
    sp[4] = align_up(sizeof(unsigned long long) * (size_t)B * LSA_MAX_TOPK, 256);
    sp[5] = align_up(sizeof(unsigned long long) * (size_t)(total_S + (int64_t)B * W + 1), 256);
    return sp[0] + sp[1] + sp[2] + sp[3] + sp[4] + sp[5];
}

static size_t step_ws_parts(int B, int64_t total_S, int n_h, int d_I, int W, size_t part[6])
{
    part[0] = align_up(sizeof(int) * (size_t)(B + 2), 256) +
              align_up(sizeof(ItemInfo) * (size_t)li_max_items(B, total_S, 1, 1), 256);
    part[1] = align_up(sizeof(float) * (size_t)(total_S > 0 ? total_S : 1), 256);
    part[2] = align_up(sizeof(float) * (size_t)B * (W > 0 ? W : 1), 256);
    part[3] = align_up((size_t)4 * B * n_h * d_I, 256);
    part[4] = align_up(sizeof(float) * (size_t)B * n_h, 256);
    size_t sp[6];
    part[5] = step_sel_parts(B, total_S, W, sp);
    return part[0] + part[1] + part[2] + part[3] + part[4] + part[5];
}

size_t lsa_lightning_topk_step_workspace_size(int B, int64_t total_S, int n_h, int d_I, int W)
{
    if (B <= 0 || total_S < 0 || n_h <= 0 || d_I <= 0 || W < 0) return 0;
    size_t part[6];
    return step_ws_parts(B, total_S, n_h, d_I, W, part);
}

lsa_status lsa_lightning_topk_step(const void *q_step, int64_t q_batch_stride, const float *w_step,
                                   int64_t w_batch_stride, const void *hot_K, const float *hot_scale, lsa_dtype kdt,
                                   const int32_t *idx, const int32_t *count, const int64_t *seq_offsets,
                                   int64_t total_S, const void *win_K, const float *win_scale,
                                   const int32_t *win_count, int W, int B, int n_h, int d_I, int k,
                                   int32_t *topk_idx, float *topk_score, void *workspace, size_t workspace_bytes,
                                   lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(q_step && w_step && hot_K && idx && count && seq_offsets && topk_idx,
                "lsa_lightning_topk_step: null pointer");
    LSA_REQUIRE(B > 0 && n_h > 0 && d_I > 0 && total_S >= 0 && W >= 0, "lsa_lightning_topk_step: sizes must be positive");
    LSA_REQUIRE(W == 0 || (win_K && win_count), "lsa_lightning_topk_step: W > 0 needs win_K and win_count");
    LSA_REQUIRE(q_batch_stride >= (int64_t)n_h * d_I && w_batch_stride >= n_h,
                "lsa_lightning_topk_step: batch strides below one query");
    LSA_REQUIRE(k >= 1 && k <= LSA_MAX_TOPK, "lsa_lightning_topk_step: k must be in [1, %d]", LSA_MAX_TOPK);
    LSA_REQUIRE(total_S < (int64_t)1 << 31, "lsa_lightning_topk_step: total_S must be below 2^31");
    if (!valid_dtype(kdt)) return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk_step: unknown key dtype");
    LSA_REQUIRE((kdt == LSA_FP8_E4M3) == (hot_scale != nullptr),
                "lsa_lightning_topk_step: hot_scale is required for FP8 keys and must be NULL otherwise");
    if (n_h > 128) return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk_step: n_h must be <= 128");
    if (d_I != 32 && d_I != 64 && d_I != 128)
        return fail(LSA_ERR_UNSUPPORTED, "lsa_lightning_topk_step: d_I must be 32, 64 or 128");
    size_t part[6];
    const size_t need = step_ws_parts(B, total_S, n_h, d_I, W, part);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_lightning_topk_step: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_lightning_topk_step: workspace must be 256-byte aligned");
    char *p = (char *)workspace;
    int *item_start = (int *)p;
    int *item_counter = item_start + B + 1;
    ItemInfo *items = (ItemInfo *)(p + align_up(sizeof(int) * (size_t)(B + 2), 256));
    float *Y = (float *)(p + part[0]);
    float *tail = (float *)(p + part[0] + part[1]);
    void *qw = (void *)(p + part[0] + part[1] + part[2]);
    float *ww = (float *)(p + part[0] + part[1] + part[2] + part[3]);
    const int hdt = (kdt == LSA_FP8_E4M3) ? (int)DT_BF16 : (int)kdt;  // hot keys: E4M3 arrives decoded to bf16
    // one query per sequence: the tensor-core scorer runs with one-query groups (MMA N = n_h)
    const bool tc = li_tc_supported(n_h, d_I, 1, kdt, 1);
    const int TQ = 1;
    size_t sp[6];
    step_sel_parts(B, total_S, W, sp);
    char *sb = p + part[0] + part[1] + part[2] + part[3] + part[4];
    int *ghist = (int *)sb;
    int *chunk_start = (int *)(sb + sp[0]);
    int *chunk_query = (int *)(sb + sp[0] + sp[1]);
    uint32_t *state = (uint32_t *)(sb + sp[0] + sp[1] + sp[2]);
    unsigned long long *sel = (unsigned long long *)(sb + sp[0] + sp[1] + sp[2] + sp[3]);
    unsigned long long *stage = (unsigned long long *)(sb + sp[0] + sp[1] + sp[2] + sp[3] + sp[4]);
    const int32_t *tcnt = W > 0 ? win_count : nullptr;
    // first launch: the scorer's items and their table, cleared histograms, the dense query copy and
    // the window entries' scores
    {
        stepsel::FrontParams fp;
        fp.count = count;
        fp.offs = seq_offsets;
        fp.win_count = tcnt;
        fp.W = W;
        fp.B = B;
        fp.k = k;
        fp.chunk_start = chunk_start;
        fp.chunk_query = chunk_query;
        fp.state = state;
        fp.n_h = n_h;
        fp.d_I = d_I;
        fp.dt = hdt;
        fp.ch = li_item_tiles(1);
        fp.item_start = item_start;
        fp.item_counter = item_counter;
        fp.items = items;
        fp.ghist = ghist;
        fp.qs = q_step;
        fp.q_bstride = q_batch_stride;
        fp.ws = w_step;
        fp.w_bstride = w_batch_stride;
        fp.q_out = qw;
        fp.w_out = ww;
        fp.winK = win_K;
        fp.winsc = win_scale;
        fp.tail = tail;
        fp.nclear = stepsel::front_clear_ctas(B);
        const unsigned grid = (unsigned)(1 + fp.nclear + B);
        const bool f32 = hdt == (int)DT_F32;
        const size_t fsm = stepsel::front_smem(n_h, d_I, hdt);
#define LSA_STEP_FRONT(E, F)                                                                   \
    do {                                                                                       \
        LSA_TRY(set_smem(stepsel::k_step_front<E, F>, fsm));                                   \
        stepsel::k_step_front<E, F><<<grid, stepsel::FRONT_TH, fsm, st>>>(fp);                 \
    } while (0)
        if (d_I == 32) { if (f32) LSA_STEP_FRONT(1, true); else LSA_STEP_FRONT(1, false); }
        else if (d_I == 64) { if (f32) LSA_STEP_FRONT(2, true); else LSA_STEP_FRONT(2, false); }
        else { if (f32) LSA_STEP_FRONT(4, true); else LSA_STEP_FRONT(4, false); }
#undef LSA_STEP_FRONT
        LSA_TRY(launched("decode step: front"));
    }
    if (tc) {
        LSA_REQUIRE(aligned(hot_K, 16), "lsa_lightning_topk_step: hot_K must be 16-byte aligned");
        int n = 0;
        const lsa_status s = launch_li_tc(qw, ww, hot_K, hot_scale, count, seq_offsets, B, total_S, TQ, 1, Y, item_start,
                                          item_counter, items, num_sms(), st, &n, /*planned=*/true, ghist);
        g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed);
        if (s != LSA_OK)
            return fail(s, "lsa_lightning_topk_step: tensor-core launch failed (%s)", cudaGetErrorString(cudaGetLastError()));
    } else {
        switch (d_I) {
        case 32: LSA_TRY(li_simt_d<32>(hdt, qw, ww, hot_K, hot_scale, count, seq_offsets, B, total_S, 1, n_h, Y, st)); break;
        case 64: LSA_TRY(li_simt_d<64>(hdt, qw, ww, hot_K, hot_scale, count, seq_offsets, B, total_S, 1, n_h, Y, st)); break;
        default: LSA_TRY(li_simt_d<128>(hdt, qw, ww, hot_K, hot_scale, count, seq_offsets, B, total_S, 1, n_h, Y, st)); break;
        }
        // the SIMT scorer does not count the histogram
        stepsel::k_step_hist<<<dim3(16, (unsigned)B), 256, 0, st>>>(Y, count, seq_offsets, ghist);
        LSA_TRY(launched("decode step: histogram"));
    }
    // the select: the k-th key's bin per query, then the chunks of candidates, the query's last chunk
    // completing it
    {
        const size_t hsm = sizeof(int) * (size_t)stepsel::HB;
        LSA_TRY(set_smem(stepsel::k_ss_beta, hsm));
        stepsel::k_ss_beta<<<(unsigned)B, stepsel::SEL_TH, hsm, st>>>(Y, count, seq_offsets, tail, tcnt, W, state, ghist,
                                                                      k);
        LSA_TRY(launched("decode step: bin of the k-th key"));
    }
    int kpow2 = 64;  // the block sort works on at least 64 keys
    while (kpow2 < k) kpow2 <<= 1;
    const size_t smem = stepsel::write_smem(kpow2);
    LSA_TRY(set_smem(stepsel::k_ss_write, smem));
    // (the chunks are counted on the device: one CTA per SM walks them)
    const int64_t mc = std::min<int64_t>(step_max_chunks(B, total_S, W), (int64_t)num_sms());
    stepsel::k_ss_write<<<(unsigned)mc, stepsel::SEL_TH, smem, st>>>(Y, count, seq_offsets, tail, tcnt, W, B, chunk_start,
                                                                     chunk_query, state, ghist, LSA_MAX_TOPK, sel, stage,
                                                                     idx, k, kpow2, topk_idx, topk_score);
    LSA_TRY(launched("decode step: select"));
    return ok();
}

// ------------------------------------------------------------------------------ golden labels

size_t lsa_golden_labels_workspace_size(int tau, int Lc, int64_t total_S)
{
    if (tau <= 0 || Lc <= 0 || total_S < 0) return 0;
    return align_up(sizeof(uint32_t) * (size_t)tau * Lc * (size_t)((total_S + 31) / 32 + 1), 256);
}

lsa_status lsa_golden_labels(const float *z, const int64_t *seq_offsets, int64_t total_S, int B, int tau, int Lc,
                             double p, int theta, uint8_t *label_out, int32_t *nsize_out, void *workspace,
                             size_t workspace_bytes, lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(z && seq_offsets && label_out, "lsa_golden_labels: null pointer");
    LSA_REQUIRE(B > 0 && tau > 0 && Lc > 0 && total_S >= 0, "lsa_golden_labels: sizes must be positive");
    LSA_REQUIRE(p > 0.0 && p <= 1.0, "lsa_golden_labels: p must be in (0, 1]");
    LSA_REQUIRE(theta >= 1, "lsa_golden_labels: theta must be at least 1");
    LSA_REQUIRE(Lc <= 255, "lsa_golden_labels: at most 255 layers");
    LSA_REQUIRE(total_S < ((int64_t)1 << 31), "lsa_golden_labels: total_S must be below 2^31");
    LSA_REQUIRE((int64_t)B * tau * Lc < ((int64_t)1 << 31), "lsa_golden_labels: too many rows");
    const size_t need = lsa_golden_labels_workspace_size(tau, Lc, total_S);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_golden_labels: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_golden_labels: workspace must be 256-byte aligned");
    if (total_S == 0) return ok();
    const int64_t W32 = (total_S + 31) / 32;
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t) * (size_t)tau * Lc * W32, st);
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "lsa_golden_labels: %s", cudaGetErrorString(e));
    uint32_t *bits = (uint32_t *)workspace;
    golden::k_golden_nucleus<<<(unsigned)((int64_t)B * tau * Lc), golden::THREADS, 0, st>>>(
        z, seq_offsets, total_S, B, tau, Lc, p, bits, W32, nsize_out);
    LSA_TRY(launched("golden labels: nucleus"));
    golden::k_golden_vote<<<(unsigned)((W32 + 31) / 32), golden::VOTE_THREADS, 0, st>>>(bits, W32, total_S, tau, Lc,
                                                                                      theta, label_out);
    LSA_TRY(launched("golden labels: vote"));
    return ok();
}

// ------------------------------------------------------------------------------ training step

// Workspace of lsa_indexer_train_step: c, q (dt), w, dq, dw, dc (fp32), tile and chunk starts, counts.
static size_t train_ws_parts(int L, int B, int64_t T, int d, int r, int n_h, int d_I, lsa_dtype dt, size_t part[8])
{
    const size_t eb = elem_bytes(dt), LB = (size_t)L * B, nq = (size_t)n_h * d_I;
    (void)T;
    part[0] = lsa_project_workspace_size(L, B, d, r, n_h, d_I, dt);  // c (the projection's workspace)
    part[1] = align_up(LB * nq * eb, 256);              // q
    part[2] = align_up(LB * n_h * 4, 256);              // w
    part[3] = align_up(LB * nq * 4, 256);               // dq
    part[4] = align_up(LB * n_h * 4, 256);              // dw
    part[5] = align_up(LB * r * 4, 256);                // dc
    part[6] = align_up(sizeof(int) * (size_t)(3 * B + 3), 256);  // tile starts, chunk starts, counts
    part[7] = 256;                                      // loss (double)
    size_t t = 0;
    for (int i = 0; i < 8; i++) t += part[i];
    return t;
}

size_t lsa_indexer_train_workspace_size(int L, int B, int64_t total_S, int d, int r, int n_h, int d_I, lsa_dtype dt)
{
    if (L <= 0 || B <= 0 || total_S < 0 || d <= 0 || r <= 0 || n_h <= 0 || d_I <= 0) return 0;
    size_t part[8];
    return train_ws_parts(L, B, total_S, d, r, n_h, d_I, dt, part);
}

lsa_status lsa_indexer_train_step(const void *h, const void *W_dq, const void *W_iuq, const void *W_w, lsa_dtype dt,
                                  const void *K, const float *k_scale, lsa_dtype kdt, const uint8_t *labels,
                                  const int64_t *seq_offsets, int64_t total_S, int L, int B, int d, int r, int n_h,
                                  int d_I, float gamma, float alpha, double *loss_out, float *g_Wdq, float *g_Wiuq,
                                  float *g_Ww, void *workspace, size_t workspace_bytes, lsa_stream_t stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    LSA_REQUIRE(h && W_dq && W_iuq && W_w && K && labels && seq_offsets && loss_out && g_Wdq && g_Wiuq && g_Ww,
                "lsa_indexer_train_step: null pointer");
    LSA_REQUIRE(L > 0 && B > 0 && total_S > 0 && d > 0 && r > 0 && n_h > 0 && d_I > 0,
                "lsa_indexer_train_step: sizes must be positive");
    LSA_REQUIRE(total_S < (int64_t)1 << 31, "lsa_indexer_train_step: total_S must be below 2^31");
    LSA_REQUIRE(gamma >= 0.f && alpha <= 1.f, "lsa_indexer_train_step: gamma >= 0 and alpha <= 1 (alpha < 0: no weighting)");
    LSA_REQUIRE((kdt == LSA_FP8_E4M3) == (k_scale != nullptr),
                "lsa_indexer_train_step: k_scale is required for FP8 keys and must be NULL otherwise");
    const bool combo = (dt == LSA_F32 && kdt == LSA_F32) || (dt == LSA_BF16 && (kdt == LSA_BF16 || kdt == LSA_FP8_E4M3));
    if (!combo) return fail(LSA_ERR_UNSUPPORTED, "lsa_indexer_train_step: dtypes F32/F32, BF16/BF16 or BF16/FP8 only");
    if (n_h > train::NHMAX || d_I > train::DMAX)
        return fail(LSA_ERR_UNSUPPORTED, "lsa_indexer_train_step: n_h <= 64 and d_I <= 128");
    if (B > train::DC_BMAX) return fail(LSA_ERR_UNSUPPORTED, "lsa_indexer_train_step: at most %d sequences", train::DC_BMAX);
    LSA_REQUIRE(d % 8 == 0 && r % 8 == 0, "lsa_indexer_train_step: d and r must be multiples of 8");
    size_t part[8];
    const size_t need = train_ws_parts(L, B, total_S, d, r, n_h, d_I, dt, part);
    if (!workspace || workspace_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "lsa_indexer_train_step: workspace needs %zu bytes", need);
    LSA_REQUIRE(aligned(workspace, 256), "lsa_indexer_train_step: workspace must be 256-byte aligned");
    char *p = (char *)workspace;
    void *c = p;
    void *q = p + part[0];
    float *w = (float *)(p + part[0] + part[1]);
    float *dq = (float *)(p + part[0] + part[1] + part[2]);
    float *dw = (float *)(p + part[0] + part[1] + part[2] + part[3]);
    float *dc = (float *)(p + part[0] + part[1] + part[2] + part[3] + part[4]);
    int *tile_start = (int *)(p + part[0] + part[1] + part[2] + part[3] + part[4] + part[5]);
    int *chunk_start = tile_start + (B + 1);
    int32_t *cnt = chunk_start + (B + 1);
    const int nq = n_h * d_I;
    cudaError_t e = cudaMemsetAsync(dq, 0, part[3] + part[4] + part[5], st);  // dq, dw and dc are adjacent
    if (e == cudaSuccess) e = cudaMemsetAsync(loss_out, 0, sizeof(double), st);
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "lsa_indexer_train_step: %s", cudaGetErrorString(e));
    LSA_TRY(lsa_project(h, W_dq, W_iuq, W_w, dt, L, B, d, r, n_h, d_I, q, w, c, part[0], stream));
    k_tile_setup<<<1, 1024, 0, st>>>(seq_offsets, B, total_S, tile_start, chunk_start, cnt);
    LSA_TRY(launched("training step: tiles"));
    const double invN = 1.0 / ((double)L * (double)total_S);
    if (train_tc::supported(dt, kdt, n_h, d_I)) {
        const dim3 grid((unsigned)((total_S / train_tc::TT + B + 1 + train_tc::TPC - 1) / train_tc::TPC), (unsigned)L);
#define LSA_TRAIN_ENTRIES_TC(KD)                                                                                   \
        do {                                                                                                       \
            LSA_TRY(set_smem(train_tc::k_train_entries_tc<KD>, train_tc::SMEM_BYTES));                            \
            train_tc::k_train_entries_tc<KD><<<grid, train_tc::THREADS, train_tc::SMEM_BYTES, st>>>(              \
                (const __nv_bfloat16 *)q, w, (const uint8_t *)K, k_scale, labels, seq_offsets, tile_start, B,       \
                total_S, gamma, alpha, invN, dq, dw, loss_out);                                                    \
        } while (0)
        if (kdt == LSA_BF16) LSA_TRAIN_ENTRIES_TC(DT_BF16);
        else LSA_TRAIN_ENTRIES_TC(DT_FP8);
#undef LSA_TRAIN_ENTRIES_TC
        LSA_TRY(launched("training step: entries (tensor cores)"));
    } else {
    const size_t smem = train::entries_smem();
    const dim3 grid((unsigned)((total_S / train::TT + B + 1 + train::TPC - 1) / train::TPC), (unsigned)L);
#define LSA_TRAIN_ENTRIES(QD, KD)                                                                                  \
    do {                                                                                                           \
        LSA_TRY(set_smem(train::k_train_entries<QD, KD>, smem));                                                   \
        train::k_train_entries<QD, KD><<<grid, train::THREADS, smem, st>>>(q, w, K, k_scale, labels, seq_offsets,  \
                                                                           tile_start, B, total_S, n_h, d_I, gamma,  \
                                                                           alpha, invN, dq, dw, loss_out);         \
    } while (0)
    if (dt == LSA_F32) LSA_TRAIN_ENTRIES(DT_F32, DT_F32);
    else if (kdt == LSA_BF16) LSA_TRAIN_ENTRIES(DT_BF16, DT_BF16);
    else LSA_TRAIN_ENTRIES(DT_BF16, DT_FP8);
#undef LSA_TRAIN_ENTRIES
    LSA_TRY(launched("training step: entries"));
    }
    const dim3 gdc((unsigned)((r + train::DC_COLS - 1) / train::DC_COLS), (unsigned)((nq + train::DC_OCH - 1) / train::DC_OCH),
                   (unsigned)L);
    auto gout = [&](int M, int N) {
        return dim3((unsigned)((N / 4 + 255) / 256), (unsigned)((M + train::OUT_MR - 1) / train::OUT_MR), (unsigned)L);
    };
#define LSA_OUTER3(VD, BM)                                                                                   \
    do {                                                                                                     \
        train::k_outer<VD, BM><<<gout(nq, r), 256, 0, st>>>(dq, c, L, B, nq, r, g_Wiuq);                     \
        train::k_outer<VD, BM><<<gout(r, d), 256, 0, st>>>(dc, h, L, B, r, d, g_Wdq);                        \
        train::k_outer<VD, BM><<<gout(n_h, d), 256, 0, st>>>(dw, h, L, B, n_h, d, g_Ww);                     \
    } while (0)
    if (dt == LSA_F32) {
        if (B <= 8) train::k_train_dc<DT_F32, 8><<<gdc, 256, 0, st>>>(dq, W_iuq, L, B, nq, r, dc);
        else train::k_train_dc<DT_F32, train::DC_BMAX><<<gdc, 256, 0, st>>>(dq, W_iuq, L, B, nq, r, dc);
        if (B <= 8) LSA_OUTER3(DT_F32, 8);
        else LSA_OUTER3(DT_F32, train::DC_BMAX);
    } else {
        if (B <= 8) train::k_train_dc<DT_BF16, 8><<<gdc, 256, 0, st>>>(dq, W_iuq, L, B, nq, r, dc);
        else train::k_train_dc<DT_BF16, train::DC_BMAX><<<gdc, 256, 0, st>>>(dq, W_iuq, L, B, nq, r, dc);
        if (B <= 8) LSA_OUTER3(DT_BF16, 8);
        else LSA_OUTER3(DT_BF16, train::DC_BMAX);
    }
#undef LSA_OUTER3
    LSA_TRY(launched("training step: weight gradients"));
    g_launches.fetch_add(3, std::memory_order_relaxed);
    return ok();
}

// ------------------------------------------------------------------------------ pool helpers

lsa_status lsa_pool_alloc(size_t bytes, void **ptr)
{
    LSA_REQUIRE(ptr && bytes > 0, "lsa_pool_alloc: bad arguments");
    *ptr = nullptr;
    cudaError_t e = cudaHostAlloc(ptr, bytes, cudaHostAllocMapped | cudaHostAllocPortable);
    if (e != cudaSuccess) {
        *ptr = nullptr;
        return fail(LSA_ERR_CUDA, "cudaHostAlloc(%zu): %s", bytes, cudaGetErrorString(e));
    }
    return ok();
}

lsa_status lsa_pool_free(void *ptr)
{
    if (!ptr) return ok();
    cudaError_t e = cudaFreeHost(ptr);
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "cudaFreeHost: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"

// ------------------------------------------------------------ score/select without a workspace
// lsa_memindex_score_select_static: the same computation as lsa_memindex_score_select, with its
// scratch in a fixed array of device memory that the library owns (declared below, reserved when
// the library's device code is loaded), so that a call performs no allocation of any kind.

namespace {

// The scratch of the allocation-free entry point: one copy per device.  Nothing in it needs to
// hold any value before a call: every byte the call reads is written earlier in the same call.
static __device__ __align__(256) unsigned char g_score_scratch[LSA_STATIC_SCORE_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxScratchDevices];  // device address of g_score_scratch, per device

// The device address of the scratch on the current device, looked up once per device.
lsa_status static_scratch(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(LSA_ERR_CUDA, "lsa_memindex_score_select_static: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxScratchDevices)
        return fail(LSA_ERR_UNSUPPORTED, "lsa_memindex_score_select_static: device %d beyond the %d supported", dev,
                    kMaxScratchDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_score_scratch);
        if (e != cudaSuccess || !p)
            return fail(LSA_ERR_CUDA, "lsa_memindex_score_select_static: cudaGetSymbolAddress on device %d: %s", dev,
                        cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" {

lsa_status lsa_memindex_score_select_static(const void *q, const float *w, const void *K, const float *k_scale,
                                            lsa_dtype kdt, const int64_t *seq_offsets, int64_t total_S, int L,
                                            int B, int n_h, int d_I, float threshold, float *scores_out,
                                            uint8_t *mask_out, int32_t *idx_out, int32_t *count_out,
                                            lsa_stream_t stream)
{
    LSA_REQUIRE(L > 0 && B > 0 && total_S >= 0 && total_S < (int64_t)1 << 31,
                "lsa_memindex_score_select_static: L and B must be positive, total_S in [0, 2^31)");
    const size_t need = score_ws_bytes(L, B, total_S);
    if (need > (size_t)LSA_STATIC_SCORE_SCRATCH_BYTES)
        return fail(LSA_ERR_WORKSPACE,
                    "lsa_memindex_score_select_static: L=%d, B=%d, total_S=%lld need %zu bytes of scratch, more than "
                    "the %zu-byte static scratch; use lsa_memindex_score_select with a workspace",
                    L, B, (long long)total_S, need, (size_t)LSA_STATIC_SCORE_SCRATCH_BYTES);
    void *scratch = nullptr;
    LSA_TRY(static_scratch(&scratch));
    return lsa_memindex_score_select(q, w, K, k_scale, kdt, seq_offsets, total_S, L, B, n_h, d_I, threshold,
                                     scores_out, mask_out, idx_out, count_out, scratch,
                                     (size_t)LSA_STATIC_SCORE_SCRATCH_BYTES, stream);
}

}  // extern "C"
