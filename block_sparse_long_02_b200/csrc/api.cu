// The C-ABI of libqsa.so (declared in include/qsa.h): host-side validation,
// workspace layout and stream-ordered launches. No allocation, no sync except
// in qsa_workspace_status.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/qsa.h"
#include "kernels.h"

namespace qsa {
static std::atomic<uint64_t> g_launches{0};
static std::atomic<int> g_attention_kernel{0};  // 0: warp-level tiles, 1: tensor-core tiles
static std::atomic<int> g_decode_kernel{1};     // 0: one persistent step kernel, 1: three kernels
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace qsa

namespace {

thread_local std::string g_err;

qsa_status fail(qsa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

}  // namespace

int qsa::report_error(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return status;
}

namespace {

qsa_status cuda_check(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return QSA_OK;
    return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

qsa_status make_dims(const qsa_config* c, qsa::LayerDims* L) {
    if (!c) return fail(QSA_ERR_INVALID_ARG, "cfg is NULL");
    if (c->r < 1 || c->r > 64) return fail(QSA_ERR_UNSUPPORTED, "r=%d outside [1, 64]", c->r);
    if (c->K < 1) return fail(QSA_ERR_INVALID_ARG, "K=%d must be positive", c->K);
    const int kB = (c->K + c->r - 1) / c->r;
    if (kB > qsa::kMaxKB) return fail(QSA_ERR_UNSUPPORTED, "k_B=%d above %d", kB, qsa::kMaxKB);
    if (c->idx_heads != qsa::kIdxHeads || c->idx_dim != qsa::kIdxDim)
        return fail(QSA_ERR_UNSUPPORTED, "indexer must be 4 heads x 128 dims (got %d x %d)",
                    c->idx_heads, c->idx_dim);
    if (c->rope_dims < 0 || c->rope_dims > qsa::kIdxDim || c->rope_dims % 8 != 0)
        return fail(QSA_ERR_UNSUPPORTED, "rope_dims=%d must be a multiple of 8 in [0, 128]",
                    c->rope_dims);
    if (!(c->rope_base > 0.0)) return fail(QSA_ERR_INVALID_ARG, "rope_base must be > 0");
    if (!(c->rms_eps >= 0.0)) return fail(QSA_ERR_INVALID_ARG, "rms_eps must be >= 0");
    if (c->head_dim != qsa::kHeadDim)
        return fail(QSA_ERR_UNSUPPORTED, "head_dim=%d (only 128)", c->head_dim);
    if (c->q_heads < 1 || c->kv_heads < 1 || c->q_heads % c->kv_heads != 0)
        return fail(QSA_ERR_UNSUPPORTED, "q_heads=%d must be a multiple of kv_heads=%d",
                    c->q_heads, c->kv_heads);
    if (c->q_heads / c->kv_heads > 16)
        return fail(QSA_ERR_UNSUPPORTED, "q_heads/kv_heads=%d above 16", c->q_heads / c->kv_heads);
    if (!(c->kv_heads == 1 || c->kv_heads == 2 || c->kv_heads == 4 || c->kv_heads == 8))
        return fail(QSA_ERR_UNSUPPORTED, "kv_heads=%d not in {1, 2, 4, 8}", c->kv_heads);
    L->r = c->r;
    L->K = c->K;
    L->kB = kB;
    L->rope_dims = c->rope_dims;
    L->rope_base = c->rope_base;
    L->rms_eps = c->rms_eps;
    L->q_heads = c->q_heads;
    L->kv_heads = c->kv_heads;
    L->head_dim = c->head_dim;
    L->sm_scale = c->sm_scale > 0.0 ? (float)c->sm_scale : (float)(1.0 / std::sqrt((double)c->head_dim));
    L->rope.half = c->rope_dims / 2;
    for (int j = 0; j < 64; ++j)
        L->rope.theta[j] = j < L->rope.half ? std::pow(c->rope_base, -2.0 * j / c->rope_dims) : 0.0;
    return QSA_OK;
}

// ---------------------------------------------------------------- workspaces
// Every workspace: [0, 256) status header, then the op's regions (256-aligned).
struct TopkWs {
    size_t qrot, scores, total;
    int64_t chunk_rows, ld;
    bool fused;
};

int64_t visible_ld(const qsa::LayerDims& L, int64_t q_begin, int64_t nq) {
    return std::max<int64_t>(1, (q_begin + nq - 1) / L.r);
}

// Row chunk of the materialised score matrix: at most ~1 GiB of fp32 scores.
TopkWs topk_layout(const qsa::LayerDims& L, int batch, int64_t cap, int64_t nq) {
    TopkWs w;
    const int64_t ld = std::max<int64_t>(1, cap / L.r);
    int64_t rows = std::max<int64_t>(32, ((int64_t)1 << 28) / std::max<int64_t>(1, (int64_t)batch * ld));
    rows = std::min<int64_t>(rows, std::max<int64_t>(nq, 1));
    rows = (rows + 31) / 32 * 32;
    w.ld = ld;
    w.chunk_rows = rows;
    w.qrot = qsa::kWsHeader;
    w.scores = w.qrot + align_up((size_t)batch * std::max<int64_t>(nq, 1) * qsa::kIdxHeads * qsa::kIdxDim * 2);
    w.fused = qsa::fused_topk_supported(L);
    // Fused path: the region after the rotated queries holds the tile counter and
    // candidate buffers; otherwise it holds one row chunk of materialised scores.
    w.total = w.scores + align_up(w.fused ? qsa::fused_topk_ws_bytes(batch, nq, L.kB) : (size_t)batch * rows * ld * 4);
    return w;
}

struct DecodeWs {
    size_t scores, sel, nsel, hist, counters, sync, est, winners, cand, part, pre, total;
};

DecodeWs decode_layout(const qsa::LayerDims& L, int batch, int64_t cap) {
    // The selection state (histograms, counters) comes first, right after the
    // status header: it must be zero when a step starts, and every step leaves
    // it zero.
    DecodeWs w;
    w.hist = qsa::kWsHeader;
    w.counters = w.hist + align_up((size_t)batch * 2048 * 4);
    w.sync = w.counters + align_up((size_t)batch * 4 * 4);
    w.est = w.sync + align_up((size_t)batch * qsa::step_sync_words(L.kv_heads) * 4);
    w.scores = w.est + align_up((size_t)batch * 8);
    // (w.scores == qsa::decode_state_bytes(batch, L.kv_heads))
    w.sel = w.scores + align_up((size_t)batch * std::max<int64_t>(1, cap / L.r) * 4);
    w.nsel = w.sel + align_up((size_t)batch * L.kB * 4);
    w.winners = w.nsel + align_up((size_t)batch * 4);
    w.cand = w.winners + align_up((size_t)batch * L.kB * 4);
    w.part = w.cand + align_up((size_t)batch * qsa::kDecodeCand * 8);
    const size_t G = (size_t)(L.q_heads / L.kv_heads);
    w.pre = w.part + align_up((size_t)batch * L.kv_heads * qsa::kStepSplitCap * (G * L.head_dim + 2 * G) * 4);
    w.total = w.pre + align_up((size_t)batch * qsa::kDecodePre * 8);
    return w;
}

size_t index_scores_ws(int batch, int64_t nq) {
    return qsa::kWsHeader + align_up((size_t)batch * std::max<int64_t>(nq, 1) * qsa::kIdxHeads * qsa::kIdxDim * 2);
}

qsa_status check_ws(void* ws, size_t have, size_t need) {
    if (have < need)
        return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", have, need);
    if (need && !ws) return fail(QSA_ERR_WORKSPACE, "workspace is NULL");
    if (ws && !aligned16(ws)) return fail(QSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    return QSA_OK;
}

#define REQUIRE_PTR(p)                                                                   \
    do {                                                                                 \
        if (!(p)) return fail(QSA_ERR_INVALID_ARG, "%s is NULL", #p);                    \
        if (!aligned16(p)) return fail(QSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

#define TRY(x)                              \
    do {                                    \
        qsa_status st_ = (x);               \
        if (st_ != QSA_OK) return st_;      \
    } while (0)

}  // namespace

extern "C" {

const char* qsa_last_error(void) { return g_err.c_str(); }

uint64_t qsa_launch_count(void) { return qsa::g_launches.load(std::memory_order_relaxed); }

qsa_status qsa_set_fault_injection(int32_t mode, double wait_seconds) {
    if (mode < 0 || mode > 4) return fail(QSA_ERR_INVALID_ARG, "fault injection mode %d", mode);
    if (mode != 0 && !(wait_seconds > 0.0 && wait_seconds <= 10.0))
        return fail(QSA_ERR_INVALID_ARG, "fault injection wait of %g s (want (0, 10])", wait_seconds);
    const uint64_t ns = mode ? (uint64_t)(wait_seconds * 1e9) : 0;
    qsa::set_fault_injection(mode == 1 || mode == 2 ? mode : 0, ns);
    qsa::set_attention_fault_injection(mode == 3 ? 3 : 0, ns);
    qsa::set_decode_fault_injection(mode == 4 ? 1 : 0, ns);
    return QSA_OK;
}

qsa_status qsa_set_decode_kernel(int32_t kernel) {
    if (kernel != 0 && kernel != 1) return fail(QSA_ERR_INVALID_ARG, "decode kernel %d (0 or 1)", kernel);
    qsa::g_decode_kernel.store(kernel, std::memory_order_relaxed);
    return QSA_OK;
}

qsa_status qsa_set_attention_kernel(int32_t kernel) {
    if (kernel != 0 && kernel != 1) return fail(QSA_ERR_INVALID_ARG, "attention kernel %d (0 or 1)", kernel);
    qsa::g_attention_kernel.store(kernel, std::memory_order_relaxed);
    return QSA_OK;
}

qsa_status qsa_workspace_size(const qsa_config* cfg, int32_t op, int32_t batch, int64_t cap,
                              int64_t nq, size_t* bytes) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    if (!bytes) return fail(QSA_ERR_INVALID_ARG, "bytes is NULL");
    if (batch < 1 || cap < 1 || nq < 0) return fail(QSA_ERR_INVALID_ARG, "bad batch/cap/nq");
    switch (op) {
        case QSA_OP_INDEX_SCORES: *bytes = index_scores_ws(batch, nq); break;
        case QSA_OP_TOPK_BLOCKS: *bytes = topk_layout(L, batch, cap, nq).total; break;
        case QSA_OP_SPARSE_ATTENTION: *bytes = qsa::kWsHeader; break;
        case QSA_OP_DECODE_STEP: *bytes = decode_layout(L, batch, cap).total; break;
        case QSA_OP_DISTILL_TARGET: *bytes = qsa::distill_target_ws_bytes(batch, nq, L.q_heads); break;
        default: return fail(QSA_ERR_INVALID_ARG, "unknown op %d", op);
    }
    return QSA_OK;
}

qsa_status qsa_compress_keys(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_k,
                             int64_t cap, const float* rms_w, int64_t blk_begin, int64_t blk_end,
                             qsa_bf16* pooled, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(idx_k);
    REQUIRE_PTR(pooled);
    if (rms_w && !aligned16(rms_w)) return fail(QSA_ERR_INVALID_ARG, "rms_w not 16-byte aligned");
    if (batch < 1 || cap < 1) return fail(QSA_ERR_INVALID_ARG, "batch=%d cap=%lld", batch, (long long)cap);
    if (blk_begin < 0 || blk_end < blk_begin)
        return fail(QSA_ERR_INVALID_ARG, "block range [%lld, %lld)", (long long)blk_begin, (long long)blk_end);
    if (blk_end * L.r > cap)
        return fail(QSA_ERR_CAPACITY, "block %lld needs %lld rows, cap=%lld", (long long)blk_end - 1,
                    (long long)(blk_end * L.r), (long long)cap);
    return cuda_check(qsa::launch_compress(L, batch, idx_k, cap, rms_w, blk_begin, blk_end, pooled,
                                           (cudaStream_t)stream),
                      "qsa_compress_keys launch");
}

qsa_status qsa_index_scores(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                            int64_t q_begin, int64_t nq, const qsa_bf16* pooled, int64_t cap,
                            float* scores, int64_t ld, void* ws, size_t ws_bytes,
                            qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(idx_q);
    REQUIRE_PTR(pooled);
    if (!scores || ((uintptr_t)scores & 3u)) return fail(QSA_ERR_INVALID_ARG, "scores NULL or misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap) return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    if (nq == 0) return QSA_OK;
    if (ld < visible_ld(L, q_begin, nq))
        return fail(QSA_ERR_INVALID_ARG, "ld=%lld below %lld visible blocks", (long long)ld, (long long)visible_ld(L, q_begin, nq));
    TRY(check_ws(ws, ws_bytes, index_scores_ws(batch, nq)));
    uint16_t* qrot = reinterpret_cast<uint16_t*>((char*)ws + qsa::kWsHeader);
    cudaStream_t st = (cudaStream_t)stream;
    TRY(cuda_check(qsa::launch_rotate_queries(L, batch, idx_q, q_begin, nq, qrot, st), "rotate"));
    return cuda_check(qsa::launch_index_scores(L, batch, qrot, nq, q_begin, 0, nq, pooled, cap,
                                               scores, ld, true, st),
                      "index scores");
}

qsa_status qsa_topk_blocks(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                           int64_t q_begin, int64_t nq, const qsa_bf16* pooled, int64_t cap,
                           const float* scores, int64_t ld, int32_t* sel, int32_t* nsel, void* ws,
                           size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(sel);
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap) return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    if (nq == 0) return QSA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    if (scores) {
        if ((uintptr_t)scores & 3u) return fail(QSA_ERR_INVALID_ARG, "scores misaligned");
        if (ld < visible_ld(L, q_begin, nq)) return fail(QSA_ERR_INVALID_ARG, "ld below visible blocks");
        return cuda_check(qsa::launch_select_rows(L, batch, scores, ld, q_begin, 0, nq, nq, sel, nsel, st),
                          "select rows");
    }
    REQUIRE_PTR(idx_q);
    REQUIRE_PTR(pooled);
    const TopkWs w = topk_layout(L, batch, cap, nq);
    TRY(check_ws(ws, ws_bytes, w.total));
    uint16_t* qrot = reinterpret_cast<uint16_t*>((char*)ws + w.qrot);
    float* chunk = reinterpret_cast<float*>((char*)ws + w.scores);
    const int64_t vld = visible_ld(L, q_begin, nq);
    TRY(cuda_check(qsa::launch_rotate_queries(L, batch, idx_q, q_begin, nq, qrot, st), "rotate"));
    if (w.fused)
        return cuda_check(qsa::launch_fused_topk(L, batch, qrot, nq, q_begin, pooled, cap, sel, nsel,
                                                 (char*)ws + w.scores, reinterpret_cast<int32_t*>(ws), st),
                          "fused top-k");
    for (int64_t j0 = 0; j0 < nq; j0 += w.chunk_rows) {
        const int64_t rows = std::min<int64_t>(w.chunk_rows, nq - j0);
        TRY(cuda_check(qsa::launch_index_scores(L, batch, qrot, nq, q_begin, j0, rows, pooled, cap,
                                                chunk, vld, false, st),
                       "index scores (chunk)"));
        TRY(cuda_check(qsa::launch_select_rows(L, batch, chunk, vld, q_begin, j0, rows, nq, sel, nsel, st),
                       "select rows (chunk)"));
    }
    return QSA_OK;
}

qsa_status qsa_sparse_attention(const qsa_config* cfg, int32_t batch, const qsa_bf16* q,
                                int64_t q_begin, int64_t nq, const qsa_bf16* k_cache,
                                const qsa_bf16* v_cache, int64_t cap, const int32_t* sel,
                                const int32_t* nsel, qsa_bf16* out, float* lse, void* ws,
                                size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_cache);
    REQUIRE_PTR(v_cache);
    REQUIRE_PTR(sel);
    REQUIRE_PTR(out);
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    if (lse && ((uintptr_t)lse & 3u)) return fail(QSA_ERR_INVALID_ARG, "lse misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap) return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    if (ws && (ws_bytes < (size_t)qsa::kWsHeader || !aligned16(ws)))
        return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes (%d needed) or misaligned", ws_bytes, qsa::kWsHeader);
    if (nq == 0) return QSA_OK;
    if (qsa::g_attention_kernel.load(std::memory_order_relaxed) == 1 && qsa::attention_tc_supported(L, batch, cap, nq))
        return cuda_check(qsa::launch_sparse_attention_tc(L, batch, q, q_begin, nq, k_cache, v_cache, cap, sel, nsel,
                                                          out, lse, reinterpret_cast<int32_t*>(ws),
                                                          (cudaStream_t)stream),
                          "sparse attention");
    return cuda_check(qsa::launch_sparse_attention(L, batch, q, q_begin, nq, k_cache, v_cache, cap,
                                                   sel, nsel, out, lse, (cudaStream_t)stream),
                      "sparse attention");
}

// ---- Variable-length batches: one call over sequences with their own query
// ranges. Every argument of every sequence is checked first; then each
// sequence runs through the single-sequence path on `stream`, in order,
// sharing the workspace (the launches on one stream never overlap).
}  // extern "C"

namespace {
struct VarlenPlan {
    int64_t total = 0, max_nq = 0, max_vis = 0;
};

qsa_status varlen_plan(const qsa::LayerDims& L, int32_t batch, const int64_t* q_begin, const int64_t* nq,
                       int64_t cap, VarlenPlan* plan) {
    if (batch < 1 || cap < 1) return fail(QSA_ERR_INVALID_ARG, "batch=%d cap=%lld", batch, (long long)cap);
    if (!q_begin || !nq) return fail(QSA_ERR_INVALID_ARG, "q_begin and nq must be host arrays of batch entries");
    VarlenPlan p;
    for (int32_t s = 0; s < batch; ++s) {
        if (q_begin[s] < 0 || nq[s] < 0)
            return fail(QSA_ERR_INVALID_ARG, "sequence %d: q_begin=%lld nq=%lld", s, (long long)q_begin[s],
                        (long long)nq[s]);
        if (q_begin[s] + nq[s] > cap)
            return fail(QSA_ERR_CAPACITY, "sequence %d: queries end at %lld > cap %lld", s,
                        (long long)(q_begin[s] + nq[s]), (long long)cap);
        p.total += nq[s];
        p.max_nq = std::max(p.max_nq, nq[s]);
        if (nq[s] > 0) p.max_vis = std::max(p.max_vis, visible_ld(L, q_begin[s], nq[s]));
    }
    *plan = p;
    return QSA_OK;
}
}  // namespace

extern "C" {

qsa_status qsa_index_scores_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                                   const int64_t* q_begin, const int64_t* nq, const qsa_bf16* pooled, int64_t cap,
                                   float* scores, int64_t ld, void* ws, size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    VarlenPlan plan;
    TRY(varlen_plan(L, batch, q_begin, nq, cap, &plan));
    REQUIRE_PTR(idx_q);
    REQUIRE_PTR(pooled);
    if (!scores || ((uintptr_t)scores & 3u)) return fail(QSA_ERR_INVALID_ARG, "scores NULL or misaligned");
    if (plan.total && ld < plan.max_vis)
        return fail(QSA_ERR_INVALID_ARG, "ld=%lld below %lld visible blocks", (long long)ld, (long long)plan.max_vis);
    TRY(check_ws(ws, ws_bytes, index_scores_ws(1, plan.max_nq)));
    int64_t off = 0;
    for (int32_t s = 0; s < batch; ++s) {
        if (nq[s] > 0)
            TRY(qsa_index_scores(cfg, 1, idx_q + off * qsa::kIdxHeads * qsa::kIdxDim, q_begin[s], nq[s],
                                 pooled + (size_t)s * (cap / L.r) * qsa::kIdxDim, cap, scores + off * ld, ld, ws,
                                 ws_bytes, stream));
        off += nq[s];
    }
    return QSA_OK;
}

qsa_status qsa_topk_blocks_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                                  const int64_t* q_begin, const int64_t* nq, const qsa_bf16* pooled, int64_t cap,
                                  int32_t* sel, int32_t* nsel, void* ws, size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    VarlenPlan plan;
    TRY(varlen_plan(L, batch, q_begin, nq, cap, &plan));
    REQUIRE_PTR(idx_q);
    REQUIRE_PTR(pooled);
    REQUIRE_PTR(sel);
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    TRY(check_ws(ws, ws_bytes, topk_layout(L, 1, cap, plan.max_nq).total));
    int64_t off = 0;
    for (int32_t s = 0; s < batch; ++s) {
        if (nq[s] > 0)
            TRY(qsa_topk_blocks(cfg, 1, idx_q + off * qsa::kIdxHeads * qsa::kIdxDim, q_begin[s], nq[s],
                                pooled + (size_t)s * (cap / L.r) * qsa::kIdxDim, cap, nullptr, 0, sel + off * L.kB,
                                nsel + off, ws, ws_bytes, stream));
        off += nq[s];
    }
    return QSA_OK;
}

qsa_status qsa_sparse_attention_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* q,
                                       const int64_t* q_begin, const int64_t* nq, const qsa_bf16* k_cache,
                                       const qsa_bf16* v_cache, int64_t cap, const int32_t* sel, const int32_t* nsel,
                                       qsa_bf16* out, float* lse, void* ws, size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    VarlenPlan plan;
    TRY(varlen_plan(L, batch, q_begin, nq, cap, &plan));
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_cache);
    REQUIRE_PTR(v_cache);
    REQUIRE_PTR(sel);
    REQUIRE_PTR(out);
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    if (lse && ((uintptr_t)lse & 3u)) return fail(QSA_ERR_INVALID_ARG, "lse misaligned");
    if (ws && (ws_bytes < (size_t)qsa::kWsHeader || !aligned16(ws)))
        return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes (%d needed) or misaligned", ws_bytes, qsa::kWsHeader);
    const size_t row = (size_t)L.q_heads * L.head_dim;
    const size_t seq = (size_t)cap * L.kv_heads * L.head_dim;
    int64_t off = 0;
    for (int32_t s = 0; s < batch; ++s) {
        if (nq[s] > 0)
            TRY(qsa_sparse_attention(cfg, 1, q + off * row, q_begin[s], nq[s], k_cache + s * seq, v_cache + s * seq,
                                     cap, sel + off * L.kB, nsel + off, out + off * row,
                                     lse ? lse + off * L.q_heads : nullptr, ws, ws_bytes, stream));
        off += nq[s];
    }
    return QSA_OK;
}

qsa_status qsa_sparse_attention_backward(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin,
                                         int64_t nq, const qsa_bf16* k_cache, const qsa_bf16* v_cache, int64_t cap,
                                         const int32_t* sel, const int32_t* nsel, const qsa_bf16* out,
                                         const float* lse, const qsa_bf16* dout, float* dq, float* dk, float* dv,
                                         qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_cache);
    REQUIRE_PTR(v_cache);
    REQUIRE_PTR(sel);
    REQUIRE_PTR(out);
    REQUIRE_PTR(dout);
    REQUIRE_PTR(dq);
    REQUIRE_PTR(dk);
    REQUIRE_PTR(dv);
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    if (!lse || ((uintptr_t)lse & 3u)) return fail(QSA_ERR_INVALID_ARG, "lse NULL or misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap)
        return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    if (nq == 0) return QSA_OK;
    return cuda_check(qsa::launch_attention_backward(L, batch, q, q_begin, nq, k_cache, v_cache, cap, sel, nsel, out,
                                                     lse, dout, dq, dk, dv, (cudaStream_t)stream),
                      "sparse attention backward");
}

qsa_status qsa_distill_target(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin, int64_t nq,
                              const qsa_bf16* k_cache, int64_t cap, float* target, int64_t ld, void* ws,
                              size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    if (!qsa::distill_target_supported(L))
        return fail(QSA_ERR_UNSUPPORTED, "distillation target: q_heads <= 32, q_heads/kv_heads dividing or "
                                         "divisible by 8, r in {1, 2, 4, 8, 16}");
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_cache);
    if (!target || ((uintptr_t)target & 3u)) return fail(QSA_ERR_INVALID_ARG, "target NULL or misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap)
        return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    if (nq > 0 && ld < (q_begin + nq - 1) / L.r)
        return fail(QSA_ERR_INVALID_ARG, "ld=%lld < floor((q_begin + nq - 1) / r)", (long long)ld);
    if ((int64_t)batch * cap >= INT32_MAX || (int64_t)batch * nq >= INT32_MAX)  // 32-bit TMA row coordinates
        return fail(QSA_ERR_UNSUPPORTED, "batch x cap and batch x nq must stay below 2^31");
    if (nq == 0) return QSA_OK;
    const size_t need = qsa::distill_target_ws_bytes(batch, nq, L.q_heads);
    if (!ws || !aligned16(ws) || ws_bytes < need)
        return fail(QSA_ERR_WORKSPACE, "workspace %zu bytes < %zu (or NULL / misaligned)", ws_bytes, need);
    return cuda_check(qsa::launch_distill_target(L, batch, q, q_begin, nq, k_cache, cap, target, ld, ws,
                                                 (cudaStream_t)stream),
                      "distillation target");
}

qsa_status qsa_distill_kl(const qsa_config* cfg, int32_t batch, int64_t q_begin, int64_t nq, const float* target,
                          const float* scores, int64_t ld, float* kl, float* dscores, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    if (!target || ((uintptr_t)target & 3u)) return fail(QSA_ERR_INVALID_ARG, "target NULL or misaligned");
    if (!scores || ((uintptr_t)scores & 3u)) return fail(QSA_ERR_INVALID_ARG, "scores NULL or misaligned");
    if (!kl || ((uintptr_t)kl & 3u)) return fail(QSA_ERR_INVALID_ARG, "kl NULL or misaligned");
    if (dscores && ((uintptr_t)dscores & 3u)) return fail(QSA_ERR_INVALID_ARG, "dscores misaligned");
    if (batch < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (nq > 0 && ld < (q_begin + nq - 1) / L.r)
        return fail(QSA_ERR_INVALID_ARG, "ld=%lld < floor((q_begin + nq - 1) / r)", (long long)ld);
    if (nq == 0) return QSA_OK;
    return cuda_check(qsa::launch_distill_kl(L, batch, q_begin, nq, target, scores, ld, kl, dscores,
                                             (cudaStream_t)stream),
                      "distillation KL");
}

qsa_status qsa_quantize_rows(const qsa_bf16* x, int64_t rows, int32_t dim, uint8_t* codes, float* scales,
                             qsa_stream stream) {
    REQUIRE_PTR(x);
    REQUIRE_PTR(codes);
    if (!scales || ((uintptr_t)scales & 3u)) return fail(QSA_ERR_INVALID_ARG, "scales NULL or misaligned");
    if (rows < 0) return fail(QSA_ERR_INVALID_ARG, "rows=%lld", (long long)rows);
    if (dim != 64 && dim != 128 && dim != 256) return fail(QSA_ERR_UNSUPPORTED, "dim=%d (64, 128 or 256)", dim);
    if (rows == 0) return QSA_OK;
    return cuda_check(qsa::launch_quantize_rows(x, rows, dim, codes, scales, (cudaStream_t)stream),
                      "quantize rows");
}

qsa_status qsa_sparse_attention_q8(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin,
                                   int64_t nq, const uint8_t* k_codes, const float* k_scales,
                                   const uint8_t* v_codes, const float* v_scales, int64_t cap,
                                   const int32_t* sel, const int32_t* nsel, qsa_bf16* out, float* lse,
                                   void* ws, size_t ws_bytes, qsa_stream stream) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_codes);
    REQUIRE_PTR(v_codes);
    REQUIRE_PTR(sel);
    REQUIRE_PTR(out);
    if (!k_scales || !v_scales || ((uintptr_t)k_scales & 3u) || ((uintptr_t)v_scales & 3u))
        return fail(QSA_ERR_INVALID_ARG, "k_scales/v_scales NULL or misaligned");
    if (!nsel || ((uintptr_t)nsel & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel NULL or misaligned");
    if (lse && ((uintptr_t)lse & 3u)) return fail(QSA_ERR_INVALID_ARG, "lse misaligned");
    if (batch < 1 || cap < 1 || nq < 0 || q_begin < 0) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q_begin + nq > cap) return fail(QSA_ERR_CAPACITY, "queries end at %lld > cap %lld", (long long)(q_begin + nq), (long long)cap);
    (void)ws;
    (void)ws_bytes;
    if (nq == 0) return QSA_OK;
    return cuda_check(qsa::launch_sparse_attention_q8(L, batch, q, q_begin, nq, k_codes, k_scales, v_codes,
                                                      v_scales, cap, sel, nsel, out, lse, (cudaStream_t)stream),
                      "sparse attention (fp8 caches)");
}

}  // extern "C"

namespace {
// The decode step's launches; q8 non-null: fp8 K/V and pooled-key caches.
qsa_status decode_step_impl(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                            const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                            qsa_bf16* k_cache, qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled,
                            int64_t cap, const float* rms_w, qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out,
                            void* ws, size_t ws_bytes, qsa_stream stream, const qsa::Q8Caches* q8,
                            qsa::HotCache* hot = nullptr, bool clear_state = false) {
    qsa::LayerDims L;
    TRY(make_dims(cfg, &L));
    REQUIRE_PTR(pos);
    REQUIRE_PTR(q);
    REQUIRE_PTR(k);
    REQUIRE_PTR(v);
    REQUIRE_PTR(idx_q);
    REQUIRE_PTR(idx_k);
    if (!q8) {
        REQUIRE_PTR(k_cache);
        REQUIRE_PTR(v_cache);
    }
    REQUIRE_PTR(idx_k_cache);
    REQUIRE_PTR(pooled);
    REQUIRE_PTR(out);
    if (rms_w && !aligned16(rms_w)) return fail(QSA_ERR_INVALID_ARG, "rms_w not 16-byte aligned");
    if (sel_out && ((uintptr_t)sel_out & 3u)) return fail(QSA_ERR_INVALID_ARG, "sel_out misaligned");
    if (nsel_out && ((uintptr_t)nsel_out & 3u)) return fail(QSA_ERR_INVALID_ARG, "nsel_out misaligned");
    if (batch < 1 || cap < 1) return fail(QSA_ERR_INVALID_ARG, "bad sizes");
    if (q8 && L.head_dim != 128) return fail(QSA_ERR_UNSUPPORTED, "fp8 caches need head_dim 128");
    const DecodeWs w = decode_layout(L, batch, cap);
    TRY(check_ws(ws, ws_bytes, w.total));
    char* base = (char*)ws;
    int32_t* status = reinterpret_cast<int32_t*>(base);
    float* scores = reinterpret_cast<float*>(base + w.scores);
    int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(base + w.sel);
    int32_t* nsel = nsel_out ? nsel_out : reinterpret_cast<int32_t*>(base + w.nsel);
    qsa::DecodeSelWs sw;
    sw.hist = reinterpret_cast<uint32_t*>(base + w.hist);
    sw.counters = reinterpret_cast<int32_t*>(base + w.counters);
    sw.winners = reinterpret_cast<int32_t*>(base + w.winners);
    sw.cand = reinterpret_cast<uint2*>(base + w.cand);
    sw.est = reinterpret_cast<float2*>(base + w.est);
    sw.pre = reinterpret_cast<uint2*>(base + w.pre);
    cudaStream_t st = (cudaStream_t)stream;
    // Every argument is valid from here on. A caller whose scratch may hold
    // another call's state asks for the status header and the selection state
    // to be cleared first.
    if (clear_state)
        TRY(cuda_check(cudaMemsetAsync(ws, 0, qsa::decode_state_bytes(batch, L.kv_heads), st), "decode state clear"));
    if (qsa::g_decode_kernel.load(std::memory_order_relaxed) == 0 && qsa::decode_step_supported(L)) {
        qsa::StepSync sy{};
        sy.arrive = reinterpret_cast<int32_t*>(base + w.sync);
        sy.ready = sy.arrive + batch;
        sy.fin = sy.ready + batch;
        sy.done = sy.fin + batch;
        sy.part = reinterpret_cast<float*>(base + w.part);
        TRY(cuda_check(qsa::launch_decode_step(L, batch, pos, q, k, v, idx_q, idx_k, k_cache, v_cache, idx_k_cache,
                                               pooled, cap, rms_w, scores, sw, sy, sel, nsel, out, status, q8, hot,
                                               st),
                       "decode step"));
        if (!hot) return QSA_OK;
        return cuda_check(qsa::launch_install_hot(L, batch, pos, cap, sel, nsel, k_cache, v_cache, hot->k, hot->v,
                                                  hot->tags, hot->blocks, st),
                          "hot-cache install");
    }
    TRY(cuda_check(qsa::launch_decode_score(L, batch, pos, k, v, idx_q, idx_k, k_cache, v_cache, idx_k_cache,
                                            pooled, cap, rms_w, scores, sw, status, q8, hot, st),
                   "decode score"));
    TRY(cuda_check(qsa::launch_decode_select(L, batch, pos, cap, scores, sw, sel, nsel, status, st),
                   "decode select"));
    if (!hot)
        return cuda_check(qsa::launch_decode_attention(L, batch, pos, q, k_cache, v_cache, cap, sel, nsel, out, q8,
                                                       nullptr, st),
                          "decode attention");
    TRY(cuda_check(qsa::launch_decode_attention(L, batch, pos, q, k_cache, v_cache, cap, sel, nsel, out, nullptr, hot,
                                                st),
                   "decode attention"));
    return cuda_check(qsa::launch_install_hot(L, batch, pos, cap, sel, nsel, k_cache, v_cache, hot->k, hot->v,
                                              hot->tags, hot->blocks, st),
                      "hot-cache install");
}

// The device address of pinned host memory that is mapped into the device's
// address space, or NULL (then the caller returns an error: the library never
// hands a kernel a host pointer it cannot read).
void* mapped_host(void* p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}
}  // namespace

extern "C" {

qsa_status qsa_decode_step(const qsa_config* cfg, int32_t batch, const int64_t* pos,
                           const qsa_bf16* q, const qsa_bf16* k, const qsa_bf16* v,
                           const qsa_bf16* idx_q, const qsa_bf16* idx_k, qsa_bf16* k_cache,
                           qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap,
                           const float* rms_w, qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out,
                           void* ws, size_t ws_bytes, qsa_stream stream) {
    return decode_step_impl(cfg, batch, pos, q, k, v, idx_q, idx_k, k_cache, v_cache, idx_k_cache, pooled, cap,
                            rms_w, out, sel_out, nsel_out, ws, ws_bytes, stream, nullptr);
}

qsa_status qsa_decode_step_offload(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                                   const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q,
                                   const qsa_bf16* idx_k, qsa_bf16* host_k_cache, qsa_bf16* host_v_cache,
                                   qsa_bf16* hot_k, qsa_bf16* hot_v, int32_t* hot_tags, int64_t hot_blocks,
                                   qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap, const float* rms_w,
                                   qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out, void* ws, size_t ws_bytes,
                                   qsa_stream stream) {
    REQUIRE_PTR(host_k_cache);
    REQUIRE_PTR(host_v_cache);
    REQUIRE_PTR(hot_k);
    REQUIRE_PTR(hot_v);
    if (!hot_tags || ((uintptr_t)hot_tags & 3u)) return fail(QSA_ERR_INVALID_ARG, "hot_tags NULL or misaligned");
    if (hot_blocks < 1 || hot_blocks >= INT32_MAX)
        return fail(QSA_ERR_INVALID_ARG, "hot_blocks=%lld", (long long)hot_blocks);
    void* hk = mapped_host(host_k_cache);
    void* hv = mapped_host(host_v_cache);
    if (!hk || !hv)
        return fail(QSA_ERR_INVALID_ARG, "host K/V caches must be pinned host memory mapped into the device");
    qsa::HotCache hot{reinterpret_cast<uint16_t*>(hot_k), reinterpret_cast<uint16_t*>(hot_v), hot_tags, hot_blocks};
    return decode_step_impl(cfg, batch, pos, q, k, v, idx_q, idx_k, static_cast<qsa_bf16*>(hk),
                            static_cast<qsa_bf16*>(hv), idx_k_cache, pooled, cap, rms_w, out, sel_out, nsel_out, ws,
                            ws_bytes, stream, nullptr, &hot);
}

qsa_status qsa_decode_step_q8(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                              const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                              uint8_t* k_codes, float* k_scales, uint8_t* v_codes, float* v_scales,
                              qsa_bf16* idx_k_cache, qsa_bf16* pooled, uint8_t* pooled_codes,
                              float* pooled_scales, int64_t cap, const float* rms_w, qsa_bf16* out,
                              int32_t* sel_out, int32_t* nsel_out, void* ws, size_t ws_bytes, qsa_stream stream) {
    REQUIRE_PTR(k_codes);
    REQUIRE_PTR(v_codes);
    REQUIRE_PTR(pooled_codes);
    for (const float* p : {k_scales, v_scales, pooled_scales})
        if (!p || ((uintptr_t)p & 3u)) return fail(QSA_ERR_INVALID_ARG, "a scale array is NULL or misaligned");
    const qsa::Q8Caches q8{k_codes, k_scales, v_codes, v_scales, pooled_codes, pooled_scales};
    return decode_step_impl(cfg, batch, pos, q, k, v, idx_q, idx_k, nullptr, nullptr, idx_k_cache, pooled, cap,
                            rms_w, out, sel_out, nsel_out, ws, ws_bytes, stream, &q8);
}

qsa_status qsa_workspace_status(void* ws, qsa_stream stream, int32_t* status) {
    if (!ws || !status) return fail(QSA_ERR_INVALID_ARG, "ws or status is NULL");
    cudaStream_t st = (cudaStream_t)stream;
    TRY(cuda_check(cudaStreamSynchronize(st), "stream sync"));
    int32_t v = 0;
    TRY(cuda_check(cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost), "status read"));
    TRY(cuda_check(cudaMemset(ws, 0, sizeof(v)), "status clear"));
    *status = v;
    return QSA_OK;
}

}  // extern "C"

namespace qsa {
int decode_step_cleared(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                        const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                        qsa_bf16* k_cache, qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap,
                        const float* rms_w, qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out, void* ws,
                        size_t ws_bytes, void* stream) {
    return decode_step_impl(cfg, batch, pos, q, k, v, idx_q, idx_k, k_cache, v_cache, idx_k_cache, pooled, cap,
                            rms_w, out, sel_out, nsel_out, ws, ws_bytes, stream, nullptr, nullptr, true);
}

size_t decode_state_bytes(int batch, int kv_heads) {
    return kWsHeader + align_up((size_t)batch * 2048 * 4) + align_up((size_t)batch * 4 * 4) +
           align_up((size_t)batch * step_sync_words(kv_heads) * 4) + align_up((size_t)batch * 8);
}
}  // namespace qsa
