/*
 * qsa.h: C-ABI of libqsa.so, the B200 (sm_100a) hot path of the QSA (Qwen
 * Sparse Attention) layer.
 *
 * The layer, as the pages state it:
 *   "QSA (Qwen Sparse Attention)" concept page, "Key math / How it works":
 *     (A) compressed lightweight indexer: 4 query heads + 1 shared key head of
 *         128 dims; keys average-pooled into blocks of r tokens, RMSNorm'd,
 *         partial RoPE on 64 of 128 dims after compression; block importance
 *         I_ib = sum_h ReLU(<q_i^h, k_b>) under block-causal masking; keep the
 *         k_B = ceil(K/r) best blocks, expand them to tokens, always add the
 *         tail of the current block;
 *     (B) sparse core attention: full scaled-dot-product attention restricted
 *         to the selected tokens. "Config": K = 2048, r = 4.
 *   "Qwen Sparse Attention" gallery page, "How block selection works": pooled
 *     keys are normalised, then rotated at the first position of each block.
 *
 * Conventions (all entry points):
 *   - bf16 tensors are passed as qsa_bf16 (the 16-bit pattern); all tensor
 *     pointers are DEVICE pointers unless stated, 16-byte aligned, contiguous,
 *     row-major in the layouts given. The caller owns every buffer.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream). Arguments are validated on the host before any launch;
 *     a bad argument returns an error status and launches nothing.
 *   - The library never allocates device memory: scratch comes from a caller
 *     workspace sized by qsa_workspace_size(). The first 256 bytes of a
 *     workspace hold a device status word and must be zero before first use
 *     (qsa_workspace_status reads and re-clears it). A decode-step workspace
 *     must be all zero before its first use, and again whenever batch or cap
 *     change; each step leaves it ready for the next.
 *   - No exceptions cross the ABI; qsa_last_error() returns a thread-local
 *     message for the last non-OK status of the calling thread.
 *   - Positions are 0-based. Query i sees complete blocks b < floor(i/r) and
 *     the tail tokens r*floor(i/r) .. i. Prefill queries are the consecutive
 *     positions [q_begin, q_begin + nq); every sequence of a batch shares them
 *     (the *_varlen calls take a range per sequence).
 *   - Supported shapes: idx_heads = 4, idx_dim = 128, rope_dims even and
 *     <= 128, head_dim = 128, q_heads % kv_heads == 0 with q_heads/kv_heads <= 16,
 *     kv_heads <= 8, 1 <= r <= 64, k_B = ceil(K/r) <= 4096. Others return
 *     QSA_ERR_UNSUPPORTED.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qsa_bf16; /* bfloat16 bit pattern */
typedef void* qsa_stream;  /* cudaStream_t */

typedef enum {
    QSA_OK = 0,
    QSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative or inconsistent size */
    QSA_ERR_UNSUPPORTED = 2,  /* shape outside the supported set above */
    QSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than qsa_workspace_size() */
    QSA_ERR_CAPACITY = 4,     /* a position does not fit the cache capacity */
    QSA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    QSA_ERR_TIMEOUT = 6,      /* a bounded device wait expired */
    QSA_ERR_DEVICE_CHECK = 7  /* a device-side check failed (see qsa_workspace_status) */
} qsa_status;

/* Layer configuration (the pages' statement of the layer). */
typedef struct {
    int32_t r;          /* block size (micro-block tokens), 4 */
    int32_t K;          /* token budget, 2048; k_B = ceil(K / r) blocks */
    int32_t idx_heads;  /* indexer query heads, 4 (one shared key head) */
    int32_t idx_dim;    /* indexer head dim, 128 */
    int32_t rope_dims;  /* dims [0, rope_dims) rotated, 64; pairs (j, j + rope_dims/2) */
    double rope_base;   /* 10000 */
    double rms_eps;     /* 1e-6 */
    int32_t q_heads;    /* core query heads (32) */
    int32_t kv_heads;   /* core kv heads (4); q head h reads kv head h / (q_heads/kv_heads) */
    int32_t head_dim;   /* 128 */
    double sm_scale;    /* softmax scale; <= 0 means 1/sqrt(head_dim) */
} qsa_config;

/* Operations that take a workspace. */
typedef enum {
    QSA_OP_INDEX_SCORES = 0,     /* qsa_index_scores */
    QSA_OP_TOPK_BLOCKS = 1,      /* qsa_topk_blocks (both modes) */
    QSA_OP_SPARSE_ATTENTION = 2, /* qsa_sparse_attention */
    QSA_OP_DECODE_STEP = 3,      /* qsa_decode_step */
    QSA_OP_DISTILL_TARGET = 4    /* qsa_distill_target */
} qsa_op;

/* Bytes of workspace `op` needs for `batch` sequences of capacity `cap` and
 * `nq` queries per sequence (nq is ignored by QSA_OP_DECODE_STEP). Writes
 * *bytes; never launches anything. */
qsa_status qsa_workspace_size(const qsa_config* cfg, int32_t op, int32_t batch, int64_t cap,
                              int64_t nq, size_t* bytes);

/* a1-a3 (concept page (A) "Block compression" and "Partial RoPE"; gallery page
 * "How block selection works"): for every sequence and every complete block b
 * in [blk_begin, blk_end):
 *   kbar = mean of idx_k rows r*b .. r*b+r-1;
 *   kn   = kbar * (mean_j kbar_j^2 + rms_eps)^-1/2 * rms_w;
 *   pooled[b] = RoPE at position r*b of kn on dims [0, rope_dims), as bf16 (RNE).
 * idx_k:  [batch][cap][idx_dim] raw indexer keys.
 * rms_w:  [idx_dim] fp32 RMSNorm weight, or NULL for all ones.
 * pooled: [batch][cap / r][idx_dim], written for blocks [blk_begin, blk_end) only.
 * Errors: blk_end * r > cap -> QSA_ERR_CAPACITY. */
qsa_status qsa_compress_keys(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_k,
                             int64_t cap, const float* rms_w, int64_t blk_begin, int64_t blk_end,
                             qsa_bf16* pooled, qsa_stream stream);

/* a3'+a4 materialised (concept page (A) "Block importance"): for query j of
 * sequence s, at position i = q_begin + j, with q^h = RoPE_i(idx_q[s][j][h]) as bf16:
 *   scores[s][j][b] = sum_h max(0, <q^h, pooled[s][b]>)  (fp32 accumulation)
 *                                 for b < floor(i / r),
 *   scores[s][j][b] = -inf        for floor(i / r) <= b < ld.
 * idx_q:  [batch][nq][idx_heads][idx_dim] un-rotated indexer queries.
 * pooled: [batch][cap / r][idx_dim] from qsa_compress_keys.
 * scores: [batch][nq][ld] fp32; ld >= floor((q_begin + nq - 1) / r).
 * ws:     qsa_workspace_size(QSA_OP_INDEX_SCORES, batch, cap, nq) bytes (holds the
 *         rotated queries).
 * Errors: q_begin + nq > cap -> QSA_ERR_CAPACITY. */
qsa_status qsa_index_scores(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                            int64_t q_begin, int64_t nq, const qsa_bf16* pooled, int64_t cap,
                            float* scores, int64_t ld, void* ws, size_t ws_bytes,
                            qsa_stream stream);

/* a5 (concept page (A) "Top-k_B block selection"; gallery page pseudo-code
 * top_k(scores, k=512)): for every query, the min(k_B, floor(i/r)) visible
 * blocks ranked first by (score descending, block index ascending).
 *   scores == NULL: fused a3'+a4+a5 from idx_q and pooled (the prefill path;
 *                   the score matrix is never materialised in full);
 *   scores != NULL: select from given scores laid out as qsa_index_scores
 *                   writes them ([batch][nq][ld]); idx_q and pooled are unused.
 * sel:  [batch][nq][k_B] int32, the selected blocks in ascending order; slots
 *       past nsel hold -1.
 * nsel: [batch][nq] int32.
 * ws:   workspace of qsa_workspace_size(QSA_OP_TOPK_BLOCKS, batch, cap, nq). */
qsa_status qsa_topk_blocks(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                           int64_t q_begin, int64_t nq, const qsa_bf16* pooled, int64_t cap,
                           const float* scores, int64_t ld, int32_t* sel, int32_t* nsel, void* ws,
                           size_t ws_bytes, qsa_stream stream);

/* a6+a7 (concept page (B) "Sparse core attention"; gallery page
 * attention_input = flatten(selected_blocks) + current_incomplete_block): for
 * query i and core head h (kv head g = h / (q_heads / kv_heads)), over the
 * tokens T_i = {r*b .. r*b+r-1 : b in sel} U {r*floor(i/r) .. i}:
 *   out[h] = sum_t softmax_t(sm_scale * <q[h], k_cache[t][g]>) v_cache[t][g].
 * Logits, softmax and accumulation are fp32; probabilities are rounded to bf16
 * for the P.V product.
 * q:       [batch][nq][q_heads][head_dim]  (already position-encoded)
 * k_cache, v_cache: [batch][cap][kv_heads][head_dim]
 * sel, nsel: as written by qsa_topk_blocks; entries outside [0, floor(i/r)) are
 *          skipped (never read out of bounds).
 * out:     [batch][nq][q_heads][head_dim] bf16.
 * lse:     [batch][nq][q_heads] fp32 natural-log sum-exp of the scaled logits,
 *          or NULL.
 * ws:      qsa_workspace_size(QSA_OP_SPARSE_ATTENTION, ...) bytes (its status
 *          header), or NULL. The tensor-core kernel's bounded waits record
 *          QSA_ERR_TIMEOUT there (qsa_workspace_status); without a workspace a
 *          timeout goes unreported.
 * Kernels (qsa_set_attention_kernel): the default runs warp-level tensor-core
 * tiles (mma.sync) over 16-token chunks gathered by each warp; the other runs
 * tcgen05 tiles in TMEM fed by TMA block gathers, for q_heads / kv_heads in
 * {1, 2, 4, 8, 16} (and batch x cap, batch x nq x q_heads below 2^31; other
 * shapes keep the default). Both compute the same values up to fp32 summation
 * order. */
qsa_status qsa_sparse_attention(const qsa_config* cfg, int32_t batch, const qsa_bf16* q,
                                int64_t q_begin, int64_t nq, const qsa_bf16* k_cache,
                                const qsa_bf16* v_cache, int64_t cap, const int32_t* sel,
                                const int32_t* nsel, qsa_bf16* out, float* lse, void* ws,
                                size_t ws_bytes, qsa_stream stream);

/* Which kernel runs qsa_sparse_attention on bf16 caches (process-wide):
 *   0 (default): warp-level tiles: every warp gathers its own 16-token chunks
 *      with cp.async and runs mma.sync; the faster of the two on the
 *      measured workloads (128K and 1M prefill);
 *   1: tcgen05 tiles with TMEM accumulators, fed by TMA boxes of whole blocks
 *      (a persistent, warp-specialised kernel; its bounded waits report
 *      QSA_ERR_TIMEOUT in the attention workspace).
 * Returns QSA_ERR_INVALID_ARG for another value. Launches nothing. */
qsa_status qsa_set_attention_kernel(int32_t kernel);

/* ---- Variable-length batches ----
 * One call over `batch` sequences whose queries are different ranges: query j
 * (0 <= j < nq[s]) of sequence s sits at position q_begin[s] + j, and the
 * queries of all sequences are packed one after another (sequence 0's first;
 * total = sum of nq). This is the serving pattern of the "QSA" knowledge page's
 * timeline (prefills of requests at different lengths, serial or interleaved
 * with decoding), for the calls of a prefill. Caches, pooled keys and the
 * workspace are as for the single-range calls (per sequence, capacity cap).
 * q_begin, nq: HOST arrays of batch int64 each; q_begin[s] >= 0, nq[s] >= 0
 * (0 skips the sequence), q_begin[s] + nq[s] <= cap (else QSA_ERR_CAPACITY).
 * Packed layouts (total rows): idx_q [total][idx_heads][idx_dim], q and out
 * [total][q_heads][head_dim], sel [total][k_B], nsel [total], lse
 * [total][q_heads], scores [total][ld].
 * Workspace: the single-range size for one sequence with the largest nq,
 * qsa_workspace_size(op, 1, cap, max nq[s]).
 * Every argument of every sequence is checked before anything is launched;
 * then the sequences run in order on `stream` (a sequence's launches are the
 * single-range call's), so the results equal those calls' bit for bit. */
qsa_status qsa_index_scores_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                                   const int64_t* q_begin, const int64_t* nq, const qsa_bf16* pooled, int64_t cap,
                                   float* scores, int64_t ld, void* ws, size_t ws_bytes, qsa_stream stream);
/* The fused selection (qsa_topk_blocks with scores == NULL) of each range. */
qsa_status qsa_topk_blocks_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* idx_q,
                                  const int64_t* q_begin, const int64_t* nq, const qsa_bf16* pooled, int64_t cap,
                                  int32_t* sel, int32_t* nsel, void* ws, size_t ws_bytes, qsa_stream stream);
qsa_status qsa_sparse_attention_varlen(const qsa_config* cfg, int32_t batch, const qsa_bf16* q,
                                       const int64_t* q_begin, const int64_t* nq, const qsa_bf16* k_cache,
                                       const qsa_bf16* v_cache, int64_t cap, const int32_t* sel, const int32_t* nsel,
                                       qsa_bf16* out, float* lse, void* ws, size_t ws_bytes, qsa_stream stream);

/* Gradient of qsa_sparse_attention (concept page, "Native trainability via
 * 2-stage continued pretraining": stage 2 trains the model and the indexer
 * together under the sparse selection, so the attention over the selected
 * tokens is differentiated). For query i, core head h (kv head g) and the
 * forward's token set T_i, with L = sum <dout, out>:
 *   P[h][t]   = exp(sm_scale <q[h], k_cache[t][g]> - lse[h]);
 *   dv[t][g] += sum over g's heads h of P[h][t] dout[h];
 *   dS[h][t]  = P[h][t] (<dout[h], v_cache[t][g]> - <dout[h], out[h]>);
 *   dq[h]     = sm_scale sum_t dS[h][t] k_cache[t][g];
 *   dk[t][g] += sm_scale sum over g's heads h of dS[h][t] q[h].
 * q, k_cache, v_cache, sel, nsel: as given to qsa_sparse_attention.
 * out, lse: its outputs for them (lse is required here).
 * dout: [batch][nq][q_heads][head_dim] bf16, the loss gradient w.r.t. out.
 * dq:   [batch][nq][q_heads][head_dim] fp32, written.
 * dk, dv: [batch][cap][kv_heads][head_dim] fp32, ADDED to (zero them before
 *       the first call; calls over several query ranges accumulate).
 * Probabilities are recomputed in fp32; P and dS are rounded to bf16 for the
 * tile products, which accumulate in fp32; dk and dv take fp32 atomic adds, so
 * their summation order (and last bits) may differ from run to run.
 * Errors: q_begin + nq > cap -> QSA_ERR_CAPACITY. No workspace. */
qsa_status qsa_sparse_attention_backward(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin,
                                         int64_t nq, const qsa_bf16* k_cache, const qsa_bf16* v_cache, int64_t cap,
                                         const int32_t* sel, const int32_t* nsel, const qsa_bf16* out,
                                         const float* lse, const qsa_bf16* dout, float* dq, float* dk, float* dv,
                                         qsa_stream stream);

/* ---- Stage-1 indexer distillation ----
 * Concept page, "Native trainability via 2-stage continued pretraining",
 * stage 1: the indexer scores are trained to match a block-max-pooled version
 * of the dense teacher attention distribution through a KL loss, while the
 * model still runs dense attention. The page names the pieces, not their
 * arithmetic; this library's reading: the teacher distribution of query i is
 * the dense causal softmax of every core head over tokens j <= i, averaged
 * over the heads; block b's pooled value is the largest of its r tokens'
 * probabilities; only the blocks the indexer scores (b < floor(i/r)) are kept,
 * normalised to sum to 1; the loss is KL(target || softmax of the scores). */

/* target[s][j][b] = max over j' in block b of p_i(j') / sum over b' < floor(i/r)
 *                   of the same maximum, for b < floor(i/r); 0 for
 *                   floor(i/r) <= b < ld  (i = q_begin + j);
 *   p_i(j') = (1/q_heads) sum_h softmax over j'' <= i of sm_scale <q[h], k_cache[j''][g(h)]>.
 * q:       [batch][nq][q_heads][head_dim] bf16 (position-encoded, as the core
 *          attention takes it); k_cache: [batch][cap][kv_heads][head_dim].
 * target:  [batch][nq][ld] fp32; ld >= floor((q_begin + nq - 1) / r).
 * ws:      qsa_workspace_size(QSA_OP_DISTILL_TARGET, batch, cap, nq) bytes (the
 *          heads' log-sum-exps); a smaller one returns QSA_ERR_WORKSPACE. A
 *          bounded device wait that runs out records QSA_ERR_TIMEOUT in its
 *          status word (qsa_workspace_status); the target is then incomplete.
 * Logits on the tensor cores (bf16 in, fp32 accumulate), softmax in fp32: two
 * passes over the keys (every head's log-sum-exp, then the probabilities).
 * Supported: q_heads <= 32, q_heads/kv_heads in {1, 2, 4, 8, 16}, r in
 * {1, 2, 4, 8, 16}, batch x cap and batch x nq below 2^31; else
 * QSA_ERR_UNSUPPORTED. */
qsa_status qsa_distill_target(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin, int64_t nq,
                              const qsa_bf16* k_cache, int64_t cap, float* target, int64_t ld, void* ws,
                              size_t ws_bytes, qsa_stream stream);

/* Per query i = q_begin + j, over its n = floor(i/r) visible blocks:
 *   kl[s][j]         = sum_b t_b (log t_b - log softmax_b(scores)), 0 log 0 = 0
 *                      (0 when n = 0);
 *   dscores[s][j][b] = (sum_b' t_b') softmax_b(scores) - t_b for b < n, 0 for
 *                      n <= b < ld (the gradient of kl; may be NULL).
 * target: as qsa_distill_target writes it; scores: as qsa_index_scores writes
 * them ([batch][nq][ld] fp32; entries from n on are not read).
 * kl: [batch][nq] fp32. fp32 arithmetic. */
qsa_status qsa_distill_kl(const qsa_config* cfg, int32_t batch, int64_t q_begin, int64_t nq, const float* target,
                          const float* scores, int64_t ld, float* kl, float* dscores, qsa_stream stream);

/* ---- Low-precision (fp8) caches ----
 * The "Qwen Sparse Attention" gallery page ("Community Quantized Version")
 * reports a quantized variant but not its format. This library's reading: a
 * row of dim bf16 values is stored as dim FP8 E4M3 codes (the OCP format: 1
 * sign bit, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448)
 * and one fp32 scale,
 *   scale = fl32(max|x| / 448),  code = E4M3(fl32(x / scale)) rounded to
 *   nearest even, magnitudes beyond 448 saturating,  value = E4M3(code)*scale;
 * an all-zero row has scale 0 and codes 0. */

/* Quantizes rows: x [rows][dim] bf16 -> codes [rows][dim] uint8 and scales
 * [rows] fp32. dim is 64, 128 or 256 (QSA_ERR_UNSUPPORTED otherwise). Device
 * pointers; x and codes 16-byte aligned, scales 4-byte aligned. Asynchronous
 * on `stream`. Used for the core K/V cache rows (one row per token and kv
 * head) and for the pooled keys (one row per block). */
qsa_status qsa_quantize_rows(const qsa_bf16* x, int64_t rows, int32_t dim, uint8_t* codes, float* scales,
                             qsa_stream stream);

/* a6+a7 as qsa_sparse_attention, on fp8 core K/V caches:
 * k_codes, v_codes: [batch][cap][kv_heads][head_dim] uint8, 16-byte aligned;
 * k_scales, v_scales: [batch][cap][kv_heads] fp32, one per (token, kv head) row.
 * The key codes enter the logit product exactly (as f16, with the query
 * converted to f16: exact for |q| below 65504) and each logit is multiplied by
 * its key row's scale in fp32; the values enter the P.V product as f16
 * (code times its row's scale, rounded to f16: full precision between 6e-5 and
 * 65504 in magnitude) with the probabilities as f16. Other arguments, errors
 * and the workspace as for qsa_sparse_attention. */
qsa_status qsa_sparse_attention_q8(const qsa_config* cfg, int32_t batch, const qsa_bf16* q, int64_t q_begin,
                                   int64_t nq, const uint8_t* k_codes, const float* k_scales,
                                   const uint8_t* v_codes, const float* v_scales, int64_t cap,
                                   const int32_t* sel, const int32_t* nsel, qsa_bf16* out, float* lse,
                                   void* ws, size_t ws_bytes, qsa_stream stream);

/* qsa_decode_step on fp8 caches: the core K/V caches are k_codes/k_scales and
 * v_codes/v_scales (layouts as for qsa_sparse_attention_q8; the appended
 * token's rows are quantized as qsa_quantize_rows would), and the decode score
 * stream reads pooled_codes [batch][cap/r][128] uint8 (16-byte aligned) with
 * pooled_scales [batch][cap/r] fp32: I_b = scale_b * sum_h ReLU(<q_h, codes_b>)
 * in fp32 (the query in f16, exact for its bf16 values inside the f16 range).
 * A block the token completes is pooled into `pooled` (bf16, as in
 * qsa_decode_step) and quantized from it into pooled_codes/pooled_scales. The
 * attention is that of qsa_sparse_attention_q8. Other arguments, the workspace
 * and the errors as for qsa_decode_step; head_dim must be 128. */
qsa_status qsa_decode_step_q8(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                              const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                              uint8_t* k_codes, float* k_scales, uint8_t* v_codes, float* v_scales,
                              qsa_bf16* idx_k_cache, qsa_bf16* pooled, uint8_t* pooled_codes,
                              float* pooled_scales, int64_t cap, const float* rms_w, qsa_bf16* out,
                              int32_t* sel_out, int32_t* nsel_out, void* ws, size_t ws_bytes, qsa_stream stream);

/* qsa_decode_step with the core K/V caches in host memory. A step reads only
 * the selected blocks' tokens and the tail (concept page, (B)), so the cache
 * can outgrow HBM when each step fetches just those blocks (the KV-offloading
 * port on the "QSA" knowledge page: history in host memory, hot data and the
 * indexer's caches on the GPU).
 * host_k_cache, host_v_cache: [batch][cap][kv_heads][head_dim] bf16 in pinned
 *   host memory mapped into the device address space (cudaHostAlloc or a
 *   torch pinned tensor); anything else returns QSA_ERR_INVALID_ARG. The
 *   step appends the new token's K/V there and reads the tail and the blocks
 *   missing from the hot cache from there (over the host link).
 * hot_k, hot_v: [batch][hot_blocks + 1][r][kv_heads][head_dim] bf16 (HBM),
 *   an HBM cache of blocks; hot_tags [batch][hot_blocks + 1] int32: the block
 *   each slot holds, or -1 (initialise to -1, and again whenever the host
 *   caches change other than by these steps). Block b may only sit in slot
 *   b % hot_blocks; 1 <= hot_blocks < INT32_MAX, else QSA_ERR_INVALID_ARG.
 *   After the attention, every selected block that missed is installed (of
 *   several selected blocks sharing a slot, the lowest). Slot hot_blocks is
 *   the tail slot: the step writes its token to row p % r there as well and
 *   tags the slot with block p / r when p opens that block or the tag already
 *   names it (else -1); the tail is read from there when the tag names the
 *   current block, from host memory otherwise.
 * The outputs equal qsa_decode_step's on the same caches bit for bit (the
 * same arithmetic on the same values). Other arguments and the workspace as
 * for qsa_decode_step. */
qsa_status qsa_decode_step_offload(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                                   const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q,
                                   const qsa_bf16* idx_k, qsa_bf16* host_k_cache, qsa_bf16* host_v_cache,
                                   qsa_bf16* hot_k, qsa_bf16* hot_v, int32_t* hot_tags, int64_t hot_blocks,
                                   qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap, const float* rms_w,
                                   qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out, void* ws, size_t ws_bytes,
                                   qsa_stream stream);

/* One decode step for every sequence s, at p = pos[s] (its current length):
 *   a8: append k, v (-> k_cache/v_cache row p) and idx_k (-> idx_k_cache row p);
 *   a3'..a7: the new token is query p: score blocks b < floor(p/r), select,
 *       attend over the selection and the tail r*floor(p/r) .. p;
 *   then, if (p + 1) % r == 0, pool block floor(p/r) into `pooled` (a1-a3), so
 *       the next step sees it (gallery page: only the attention layers grow the
 *       KV cache; the pooling time is a reading).
 * pos:  DEVICE [batch] int64 (not modified; the caller advances it).
 * q: [batch][q_heads][head_dim]; k, v: [batch][kv_heads][head_dim];
 * idx_q: [batch][idx_heads][idx_dim]; idx_k: [batch][idx_dim].
 * Caches as above with capacity cap; pooled [batch][cap/r][idx_dim].
 * out: [batch][q_heads][head_dim] bf16; sel_out: [batch][k_B] int32 or NULL
 * (ascending, -1 padded); nsel_out: [batch] int32 or NULL.
 * A sequence with pos >= cap or pos < 0 is skipped and flags
 * QSA_ERR_CAPACITY in the workspace status (qsa_workspace_status). */
qsa_status qsa_decode_step(const qsa_config* cfg, int32_t batch, const int64_t* pos,
                           const qsa_bf16* q, const qsa_bf16* k, const qsa_bf16* v,
                           const qsa_bf16* idx_q, const qsa_bf16* idx_k, qsa_bf16* k_cache,
                           qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap,
                           const float* rms_w, qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out,
                           void* ws, size_t ws_bytes, qsa_stream stream);

/* Which kernels run a decode step (qsa_decode_step, _q8, _offload, _noalloc;
 * process-wide):
 *   0: one persistent kernel per step, one CTA of 512 threads per
 *      SM, X = max(1, SMs / batch) CTAs per sequence. Each sequence's CTAs
 *      append the token and score their slices of the pooled keys, also
 *      listing the blocks at or above a threshold estimated from the previous
 *      step (kept per batch slot in the workspace). CTA 0 waits for the others
 *      and, when the list holds between k_B and 4096 blocks (then it holds
 *      every top-k_B block), picks from it alone; otherwise every CTA runs the
 *      histogram selection. The pick is published with a release flag, then
 *      the CTAs attend their splits of the selection and combine them. The
 *      estimate affects speed only, never the result. CTAs only wait for CTAs
 *      of the same sequence, all resident at once; every wait is bounded (10 s)
 *      and reports QSA_ERR_TIMEOUT in the workspace status. Runs
 *      q_heads / kv_heads <= 8; larger groups use 1.
 *   1 (default): three kernels per step (scores, selection, attention).
 * Both give the same selection; outputs agree up to fp32 summation order.
 * Returns QSA_ERR_INVALID_ARG for another value. Launches nothing. */
qsa_status qsa_set_decode_kernel(int32_t kernel);

/* Bytes of the fixed device scratch array behind qsa_decode_step_noalloc. */
#define QSA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* qsa_decode_step without a workspace. The pages have no counterpart: this is
 * a property of the library, not of the layer.
 *
 * For callers that cannot allocate device memory: serving engines that carve
 * all device memory into their own pool and forbid allocations outside it,
 * plugin hosts that pass a stream and tensors but no allocator or workspace,
 * and latency-critical loops that cannot afford the device-wide
 * synchronisation cudaMalloc/cudaFree may cause. It allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine). Its scratch is one
 * fixed array of QSA_NOALLOC_SCRATCH_BYTES (16 MiB) in the library's device
 * memory, which every GPU that loads the library holds until the process exits.
 *
 * Arguments and results are those of qsa_decode_step, minus ws/ws_bytes. The
 * caller still owns and passes every input, output and cache.
 * Limits and rules:
 *   - If qsa_workspace_size(QSA_OP_DECODE_STEP, batch, cap) exceeds
 *     QSA_NOALLOC_SCRATCH_BYTES the call returns QSA_ERR_WORKSPACE and launches
 *     nothing (e.g. batch 8 x 256K cached tokens fits; batch 64 x 4M does not).
 *   - Every call looks up the array's device address in the current context;
 *     the first call in a context also loads the library's device code there,
 *     so make that first call before any stream capture.
 *   - Every argument is checked before anything is queued: a bad argument
 *     returns its error status and leaves the stream untouched.
 *   - Every call shares the one array and it keeps the last call's contents:
 *     calls whose work overlaps on the GPU (other streams, other threads) race
 *     and corrupt each other's results. Order them on one stream.
 *   - The device status word lives in the array, is cleared at each call and
 *     cannot be read back, so every status the step can flag on the device is
 *     lost: QSA_ERR_CAPACITY (a position outside [0, cap) is skipped) and
 *     QSA_ERR_DEVICE_CHECK (the selection's internal consistency check; out
 *     and sel_out may then be wrong). Callers that need them use
 *     qsa_decode_step with a workspace. */
qsa_status qsa_decode_step_noalloc(const qsa_config* cfg, int32_t batch, const int64_t* pos,
                                   const qsa_bf16* q, const qsa_bf16* k, const qsa_bf16* v,
                                   const qsa_bf16* idx_q, const qsa_bf16* idx_k, qsa_bf16* k_cache,
                                   qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled,
                                   int64_t cap, const float* rms_w, qsa_bf16* out,
                                   int32_t* sel_out, int32_t* nsel_out, qsa_stream stream);

/* Device-side status recorded in a workspace by the calls that used it:
 * QSA_OK, or the first error a kernel flagged (QSA_ERR_CAPACITY,
 * QSA_ERR_DEVICE_CHECK, QSA_ERR_TIMEOUT). Synchronises `stream`, copies the
 * word to *status and clears it. */
qsa_status qsa_workspace_status(void* ws, qsa_stream stream, int32_t* status);

/* Thread-local message describing the last non-OK status ("" if none). */
const char* qsa_last_error(void);

/* Number of kernel launches this library has issued in this process (all
 * threads, all entry points). Used to count device work in benchmarks. */
uint64_t qsa_launch_count(void);

/* Fault injection, for tests of the failure path (the pages have no
 * counterpart; such a test needs a bounded device wait that runs out without
 * faulting the GPU). Process-wide, off by default.
 *   mode 0: normal operation (every bounded device wait gives up after 10 s).
 *   mode 1: the fused qsa_topk_blocks path (k_B <= 512) withholds the pooled-key
 *           tiles of each CTA's first unit of work, so the MMA's bounded wait
 *           runs out after wait_seconds (0 < wait_seconds <= 10): the kernel
 *           records QSA_ERR_TIMEOUT in the workspace status, drains its own
 *           copies and MMAs, frees its tensor memory and returns; the selection
 *           it leaves is incomplete, and the CUDA context stays usable.
 *   mode 2: the same for qsa_distill_target: both of its kernels withhold
 *           every key tile; each CTA records QSA_ERR_TIMEOUT after
 *           wait_seconds, drains, frees its tensor memory and returns (the
 *           target it leaves is incomplete).
 *   mode 3: the same for qsa_sparse_attention (its tensor-core kernel): the
 *           key tiles of each CTA's first group of queries are withheld; the
 *           timeout is recorded in the workspace passed to that call (none is
 *           recorded without one) and the outputs it leaves are incomplete.
 *   mode 4: the same for the decode steps' one-kernel path (qsa_decode_step,
 *           _q8, _offload with qsa_set_decode_kernel(0)): the last CTA of
 *           sequence 0 withholds its arrival after the score stream, so that
 *           sequence's CTAs (when it has more than one and the step scores,
 *           p / r > k_B) wait until wait_seconds have passed, record
 *           QSA_ERR_TIMEOUT and skip the rest of the step. The outputs of
 *           sequence 0 are then incomplete, and the workspace must be zeroed
 *           before its next step.
 * Returns QSA_ERR_INVALID_ARG for another mode or wait. */
qsa_status qsa_set_fault_injection(int32_t mode, double wait_seconds);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H_ */
