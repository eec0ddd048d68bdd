// Internal launchers (host side) of the QSA kernels. The C-ABI in api.cu
// validates arguments and calls these; each returns cudaGetLastError().
#pragma once

#include <atomic>
#include <utility>

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/qsa.h"
#include "common.cuh"

namespace qsa {

// Launch with programmatic stream serialization: the kernel may begin
// launching while the previous kernel in the stream finishes; it must call
// pdl_wait() before touching memory (the decode kernels do so first thing).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Counts one kernel launch (see qsa_launch_count).
void note_launch(int n = 1);
// Sets the calling thread's qsa_last_error message; returns `status`.
int report_error(int status, const char* fmt, ...);

struct LayerDims {
    int r, K, kB;
    int rope_dims;
    double rope_base, rms_eps;
    int q_heads, kv_heads, head_dim;
    float sm_scale;  // resolved (> 0)
    RopeTable rope;
};

// compress.cu
cudaError_t launch_compress(const LayerDims& L, int batch, const uint16_t* idx_k, int64_t cap,
                            const float* rms_w, int64_t blk_begin, int64_t blk_end,
                            uint16_t* pooled, cudaStream_t st);
cudaError_t launch_rotate_queries(const LayerDims& L, int batch, const uint16_t* idx_q,
                                  int64_t q_begin, int64_t nq, uint16_t* qrot, cudaStream_t st);

// scores.cu: fp32 scores [batch][nq][ld] from rotated queries. Queries [j0, j0+nrows)
// of each sequence are written to rows 0..nrows-1 of `scores` (per sequence stride
// nrows*ld). Entries b >= floor(i/r) get -inf when fill_masked, else are left.
cudaError_t launch_index_scores(const LayerDims& L, int batch, const uint16_t* qrot, int64_t nq,
                                int64_t q_begin, int64_t j0, int64_t nrows, const uint16_t* pooled,
                                int64_t cap, float* scores, int64_t ld, bool fill_masked,
                                cudaStream_t st);

// indexer_tc.cu: fused tcgen05 score + streaming top-k (prefill), k_B <= 512.
bool fused_topk_supported(const LayerDims& L);
size_t fused_topk_ws_bytes(int batch, int64_t nq, int kB);
// Tests of the failure path: mode 1 makes the fused indexer's TMA producer
// withhold the key tiles of each CTA's first unit, mode 2 the stage-1 target
// kernels' producers their key tiles, so the MMA warp's bounded wait runs out
// after wait_ns; mode 0 restores normal operation. The state (defined with the
// fused indexer) is read by the kernels' launchers.
void set_fault_injection(int mode, uint64_t wait_ns);
extern std::atomic<int> g_fault_mode;
extern std::atomic<uint64_t> g_fault_wait_ns;
// Merge of the per-split top-k lists of the fused indexer (topk.cu): for query
// j of sequence s, the lists of its query tile's `splits` key ranges hold
// (score bits, block) entries in split_out[(unit * QT + j % QT) * k_B ...],
// unit = ((nqt - 1 - j / QT) * batch + s) * splits + split, with counts in
// split_cnt; the top k_B of their union goes to sel/nsel, ascending.
cudaError_t launch_split_merge(const LayerDims& L, int batch, int64_t nq, int64_t q_begin, int qt_rows,
                               int splits, const uint2* split_out, const int32_t* split_cnt, int32_t* sel,
                               int32_t* nsel, cudaStream_t st);
cudaError_t launch_fused_topk(const LayerDims& L, int batch, const uint16_t* qrot, int64_t nq,
                              int64_t q_begin, const uint16_t* pooled, int64_t cap, int32_t* sel,
                              int32_t* nsel, void* ws, int32_t* status, cudaStream_t st);

// topk.cu: row selection. Row (s, j) has position i = q_begin + j0 + j and
// floor(i/r) visible entries starting at scores + ((s*nrows + j) * ld).
cudaError_t launch_select_rows(const LayerDims& L, int batch, const float* scores, int64_t ld,
                               int64_t q_begin, int64_t j0, int64_t nrows, int64_t nq_total,
                               int32_t* sel, int32_t* nsel, cudaStream_t st);
// attention.cu
cudaError_t launch_sparse_attention(const LayerDims& L, int batch, const uint16_t* q,
                                    int64_t q_begin, int64_t nq, const uint16_t* kc,
                                    const uint16_t* vc, int64_t cap, const int32_t* sel,
                                    const int32_t* nsel, uint16_t* out, float* lse,
                                    cudaStream_t st);
cudaError_t launch_sparse_attention_q8(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin,
                                       int64_t nq, const uint8_t* k8, const float* ks, const uint8_t* v8,
                                       const float* vs, int64_t cap, const int32_t* sel, const int32_t* nsel,
                                       uint16_t* out, float* lse, cudaStream_t st);
// An HBM cache of K/V blocks in front of caches held in host memory:
// k, v [batch][blocks + 1][r][kv_heads][128] bf16; tags [batch][blocks + 1] =
// the block a slot holds, or -1; block b may only sit in slot b % blocks.
// Slot `blocks` is the tail slot: when its tag is the current block, its rows
// hold that block's tokens up to the step's position (each step appends its
// token there as well, and claims the slot when its token opens a block).
struct HotCache {
    uint16_t* k;
    uint16_t* v;
    int32_t* tags;
    int64_t blocks;
};
// q8 non-null: the K/V caches are q8's fp8 codes and scales (kc, vc unused).
// hot non-null: kc, vc are (device-mapped) host memory with hot in front.
cudaError_t launch_decode_attention(const LayerDims& L, int batch, const int64_t* pos,
                                    const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                    int64_t cap, const int32_t* sel, const int32_t* nsel,
                                    uint16_t* out, const struct Q8Caches* q8, const HotCache* hot,
                                    cudaStream_t st);
// offload.cu: after the attention, installs each selected block that missed
// into its hot slot (the lowest selected block of a slot wins); blocks is the
// number of slots before the tail slot.
cudaError_t launch_install_hot(const LayerDims& L, int batch, const int64_t* pos, int64_t cap, const int32_t* sel,
                               const int32_t* nsel, const uint16_t* host_k, const uint16_t* host_v, uint16_t* hot_k,
                               uint16_t* hot_v, int32_t* tags, int64_t blocks, cudaStream_t st);

// attention_bwd.cu: gradient of launch_sparse_attention (dq written; dk, dv
// accumulated with atomics).
cudaError_t launch_attention_backward(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                      const uint16_t* kc, const uint16_t* vc, int64_t cap, const int32_t* sel,
                                      const int32_t* nsel, const uint16_t* out, const float* lse,
                                      const uint16_t* dout, float* dq, float* dk, float* dv, cudaStream_t st);

// distill.cu: stage-1 distillation target (block-max-pooled, head-averaged
// dense attention distribution over the visible blocks, normalised; zero from
// floor(i/r) to ld) and the KL loss with its gradient w.r.t. the scores.
bool distill_target_supported(const LayerDims& L);
// distill_tc.cu: the target on tcgen05; ws = status header + the heads'
// log-sum-exps [batch][nq][q_heads] fp32.
size_t distill_target_ws_bytes(int batch, int64_t nq, int q_heads);
cudaError_t launch_distill_target(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                  const uint16_t* kc, int64_t cap, float* target, int64_t ld, void* ws,
                                  cudaStream_t st);
cudaError_t launch_distill_kl(const LayerDims& L, int batch, int64_t q_begin, int64_t nq, const float* target,
                              const float* scores, int64_t ld, float* kl, float* dscores, cudaStream_t st);

// quant.cu: FP8 E4M3 rows with one fp32 scale per row (dim 64, 128 or 256).
cudaError_t launch_quantize_rows(const uint16_t* x, int64_t rows, int dim, uint8_t* codes, float* scales,
                                 cudaStream_t st);

// fp8 decode caches: core K/V codes [batch][cap][kv_heads][128] with row scales
// [batch][cap][kv_heads], and the pooled keys' codes [batch][cap/r][128] with
// block scales [batch][cap/r].
struct Q8Caches {
    uint8_t* k8;
    float* ks;
    uint8_t* v8;
    float* vs;
    uint8_t* pooled8;
    float* pscale;
};

// decode.cu. Per-sequence selection state in the decode workspace.
constexpr int kDecodeCand = 4096;  // candidates of the threshold digit kept for the final pick
constexpr int kDecodePre = 4096;  // blocks the step kernel's score pass can list per sequence
struct DecodeSelWs {
    uint32_t* hist;     // [batch][2048] histogram of the scores' level-1 key digit
    int32_t* counters;  // [batch][4]: sure winners, candidates, finished CTAs, listed blocks
    int32_t* winners;   // [batch][k_B]
    uint2* cand;        // [batch][kDecodeCand] (key, block)
    float2* est;        // [batch] (last k-th score / its query's summed head norms, this query's sum)
    uint2* pre;         // [batch][kDecodePre] (key, block) of the blocks listed by the score pass
};
int decode_select_ctas(int batch);
// Sparse attention (a6 + a7) on tcgen05 with TMA block gathers; `status` (a
// workspace header, may be NULL) receives QSA_ERR_TIMEOUT if a bounded wait
// runs out.
bool attention_tc_supported(const LayerDims& L, int batch, int64_t cap, int64_t nq);
cudaError_t launch_sparse_attention_tc(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                       const uint16_t* kc, const uint16_t* vc, int64_t cap, const int32_t* sel,
                                       const int32_t* nsel, uint16_t* out, float* lse, int32_t* status,
                                       cudaStream_t st);
void set_attention_fault_injection(int mode, uint64_t wait_ns);
// Bytes at the start of a decode workspace (status header, histograms,
// counters, step synchronisation) that must be zero when a decode step
// starts; each step leaves them zero.
size_t decode_state_bytes(int batch, int kv_heads);
// qsa_decode_step on a workspace whose state bytes may hold anything (another
// call's leftovers): checks every argument first, then clears the state bytes
// on `stream`, then launches the step. A bad argument returns its error status
// and queues nothing.
int decode_step_cleared(const qsa_config* cfg, int32_t batch, const int64_t* pos, const qsa_bf16* q,
                        const qsa_bf16* k, const qsa_bf16* v, const qsa_bf16* idx_q, const qsa_bf16* idx_k,
                        qsa_bf16* k_cache, qsa_bf16* v_cache, qsa_bf16* idx_k_cache, qsa_bf16* pooled, int64_t cap,
                        const float* rms_w, qsa_bf16* out, int32_t* sel_out, int32_t* nsel_out, void* ws,
                        size_t ws_bytes, void* stream);
cudaError_t launch_decode_score(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* k,
                                const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                                uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled,
                                int64_t cap, const float* rms_w, float* scores, DecodeSelWs sw,
                                int32_t* status, const Q8Caches* q8, const HotCache* hot, cudaStream_t st);
cudaError_t launch_decode_select(const LayerDims& L, int batch, const int64_t* pos, int64_t cap,
                                 const float* scores, DecodeSelWs sw, int32_t* sel, int32_t* nsel,
                                 int32_t* status, cudaStream_t st);

// The decode step as one persistent kernel (decode.cu): inter-CTA state in the
// decode workspace, zero between steps.
constexpr int kStepSplitCap = 16;  // attention CTAs per (sequence, kv head)
struct StepSync {
    int32_t* arrive;  // [batch] CTAs whose histogram counts are in
    int32_t* ready;   // [batch] 1 once the sequence's selection is written
    int32_t* fin;     // [batch] CTAs done with the step
    int32_t* done;    // [batch][kv_heads] attention CTAs whose partial state is written
    float* part;      // [batch][kv_heads][kStepSplitCap][G * 128 + 2 G] partial states (o, m, l)
    uint64_t wait_ns; // bound of every inter-CTA wait
    int32_t inject;   // fault injection: CTA (0, 0) withholds its arrival
};
// int32 words of StepSync state per sequence (arrive, ready, fin, done[kv_heads]).
inline size_t step_sync_words(int kv_heads) { return 3 + (size_t)kv_heads; }
bool decode_step_supported(const LayerDims& L);
cudaError_t launch_decode_step(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* q,
                               const uint16_t* k, const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                               uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled, int64_t cap,
                               const float* rms_w, float* scores, DecodeSelWs sw, StepSync sy, int32_t* sel,
                               int32_t* nsel, uint16_t* out, int32_t* status, const Q8Caches* q8,
                               const HotCache* hot, cudaStream_t st);
void set_decode_fault_injection(int mode, uint64_t wait_ns);

}  // namespace qsa
