// Decode step pieces ("QSA (Qwen Sparse Attention)" concept page, (A)-(B), for
// one new token per sequence): a8 (cache append, block pooling) with a3' (query
// rotation), the a4 score stream over every pooled key of a sequence, and the
// a5 selection.
//
// The score stream is the hot spot: 256 bytes of pooled key per block and
// 4 x 128 multiply-adds, an L2/HBM stream. A half-warp scores four blocks per
// step from 16-byte loads (prefetched one step ahead); the 16 per-lane partial
// sums (4 blocks x 4 heads) are reduced across the half-warp with a transpose
// reduction (15 shuffles for 16 sums), then ReLU and the head sum take two more.
// The same pass builds a histogram of the scores' top 11 key bits per sequence,
// so the selection needs one more pass over the score row, not a sort:
// every CTA finds the threshold digit from the histogram, appends the sure
// winners and the threshold-digit candidates, and the last CTA of the sequence
// finishes the exact pick among the candidates (ties to the lower block index)
// and sorts the k_B winners (select.cuh).
#include <algorithm>

#include "kernels.h"
#include "rope.cuh"
#include "select.cuh"

namespace qsa {
namespace {

constexpr int SC_THREADS = 512;  // score and select CTAs
constexpr int SC_WARPS = SC_THREADS / 32;

__global__ void __launch_bounds__(128) decode_prepare_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, double eps, RopeTable rt,
    uint16_t* __restrict__ qrot, DecodeSelWs sw, int32_t* __restrict__ status) {
    const int s = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Selection state of this step starts empty.
    for (int b = tid; b < 2048; b += blockDim.x) sw.hist[(size_t)s * 2048 + b] = 0u;
    if (tid < 4) sw.counters[s * 4 + tid] = 0;
    const int64_t p = pos[s];
    if (p < 0 || p >= cap) {
        if (tid == 0) flag_status(status, 4 /* QSA_ERR_CAPACITY */);
        return;
    }
    const int row16 = kv_heads * kHeadDim / 8;  // 16-byte chunks per kv row
    const uint4* ks = reinterpret_cast<const uint4*>(k + (size_t)s * kv_heads * kHeadDim);
    const uint4* vs = reinterpret_cast<const uint4*>(v + (size_t)s * kv_heads * kHeadDim);
    uint4* kd = reinterpret_cast<uint4*>(kc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
    uint4* vd = reinterpret_cast<uint4*>(vc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
    for (int c = tid; c < row16; c += blockDim.x) {
        kd[c] = ks[c];
        vd[c] = vs[c];
    }
    if (tid < kIdxDim / 8)
        reinterpret_cast<uint4*>(idx_k_cache + ((size_t)s * cap + p) * kIdxDim)[tid] =
            reinterpret_cast<const uint4*>(idx_k + (size_t)s * kIdxDim)[tid];
    // a3': the new indexer query, rotated at its own position.
    rotate_head_warp(idx_q + ((size_t)s * kIdxHeads + warp) * kIdxDim, p, rt,
                     qrot + ((size_t)s * kIdxHeads + warp) * kIdxDim, lane);
    // a8: the token closes its block -> pool it for the following steps. The
    // block's last raw key is read from the input (the append above is by
    // other threads of this CTA).
    if (warp == 0 && (p + 1) % r == 0) {
        const int64_t b = p / r;
        pool_block_warp(idx_k_cache + ((size_t)s * cap + (size_t)b * r) * kIdxDim,
                        idx_k + (size_t)s * kIdxDim, r, rms_w, eps, b * r, rt,
                        pooled + ((size_t)s * (cap / r) + b) * kIdxDim, lane);
    }
}

// Blocks [lo, hi) of a sequence's nvis visible blocks handled by CTA x of X.
__device__ __forceinline__ void cta_range(int64_t nvis, int x, int X, int64_t& lo, int64_t& hi) {
    const int64_t chunk = (nvis + X - 1) / X;
    lo = min(nvis, (int64_t)x * chunk);
    hi = min(nvis, lo + chunk);
}

__device__ __forceinline__ void load4(const uint16_t* ks, int64_t b0, int64_t hi, int hl, uint4 (&w)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t b = b0 + i;
        w[i] = b < hi ? *reinterpret_cast<const uint4*>(ks + (size_t)b * kIdxDim + hl * 8)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
}

__global__ void __launch_bounds__(SC_THREADS) decode_scores_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ qrot,
    const uint16_t* __restrict__ pooled, int64_t cap, int r, float* __restrict__ scores,
    uint32_t* __restrict__ hist_g) {
    __shared__ uint32_t hist[2048];
    const int s = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hl = lane & 15, half = lane >> 4;
    const int64_t p = pos[s];
    if (p < 0 || p >= cap) return;
    const int64_t pcap = cap / r;
    int64_t lo, hi;
    cta_range(p / r, blockIdx.x, gridDim.x, lo, hi);
    if (lo >= hi) return;
    for (int b = tid; b < 2048; b += SC_THREADS) hist[b] = 0u;
    // This lane's 8 dims of the 4 rotated query heads.
    float qv[kIdxHeads][8];
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) {
        const uint4 w = *reinterpret_cast<const uint4*>(qrot + ((size_t)s * kIdxHeads + h) * kIdxDim + hl * 8);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qv[h][2 * e] = bf16_lo(ws[e]);
            qv[h][2 * e + 1] = bf16_hi(ws[e]);
        }
    }
    __syncthreads();
    const uint16_t* ks = pooled + (size_t)s * pcap * kIdxDim;
    float* dst = scores + (size_t)s * pcap;
    // Warp step: 8 blocks, half-warp `half` takes blocks b0 + 4*half + (0..3).
    const int64_t stride = (int64_t)SC_WARPS * 8;
    int64_t b0 = lo + (int64_t)warp * 8;
    uint4 cur[4];
    load4(ks, b0 + half * 4, hi, hl, cur);
    for (; b0 < hi; b0 += stride) {
        uint4 nxt[4];
        load4(ks, b0 + stride + half * 4, hi, hl, nxt);  // prefetch the next step
        float v[16];  // v[4*i + h]: block i, head h (partial over this lane's 8 dims)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t ws[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    a = fmaf(qv[h][2 * e], bf16_lo(ws[e]), a);
                    a = fmaf(qv[h][2 * e + 1], bf16_hi(ws[e]), a);
                }
                v[4 * i + h] = a;
            }
        }
        // Transpose reduction over the 16 lanes: lane hl ends with sum index hl.
#pragma unroll
        for (int m = 8, n = 8; m >= 1; m >>= 1, n >>= 1) {
            const bool up = (hl & m) != 0;
#pragma unroll
            for (int j = 0; j < n; ++j) {
                const float send = up ? v[j] : v[j + n];
                const float keep = up ? v[j + n] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        float sc = fmaxf(v[0], 0.f);  // block hl >> 2, head hl & 3
        sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        sc += __shfl_xor_sync(0xffffffffu, sc, 2);
        const int64_t b = b0 + half * 4 + (hl >> 2);
        if ((hl & 3) == 0 && b < hi) {
            dst[b] = sc;
            atomicAdd(&hist[float_key(sc) >> 21], 1u);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    }
    __syncthreads();
    for (int b = tid; b < 2048; b += SC_THREADS)
        if (hist[b]) atomicAdd(&hist_g[(size_t)s * 2048 + b], hist[b]);
}

// Block-aggregated append: the CTA's flagged entries get consecutive slots of a
// per-sequence global list (one atomic per CTA round). Returns this thread's
// slot or -1. All threads must call it.
__device__ __forceinline__ int cta_append(SelSmem& sm, bool flag, int32_t* counter, int* base_slot) {
    uint32_t pre;
    const uint32_t tot = cta_scan(sm, flag, pre);
    if (threadIdx.x == 0) *base_slot = tot ? atomicAdd(counter, (int)tot) : 0;
    __syncthreads();
    const int slot = flag ? *base_slot + (int)pre : -1;
    __syncthreads();
    return slot;
}

__global__ void __launch_bounds__(SC_THREADS) decode_select_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int r, int kB, const float* __restrict__ scores,
    DecodeSelWs sw, int32_t* __restrict__ sel, int32_t* __restrict__ nsel) {
    extern __shared__ __align__(16) uint8_t raw[];
    SelSmem& sm = *reinterpret_cast<SelSmem*>(raw);
    __shared__ int base_slot, last;
    const int s = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t p = pos[s];
    const int64_t nvis = (p >= 0 && p < cap) ? p / r : 0;
    int32_t* out = sel + (size_t)s * kB;
    if (nvis <= kB) {  // every visible block is selected
        if (blockIdx.x == 0) {
            for (int k2 = tid; k2 < kB; k2 += SC_THREADS) out[k2] = k2 < nvis ? k2 : -1;
            if (tid == 0) nsel[s] = (int32_t)nvis;
        }
        return;
    }
    const float* row = scores + (size_t)s * (cap / r);
    // Threshold digit from the sequence's histogram.
    for (int b = tid; b < 2048; b += SC_THREADS) sm.hist[b] = __ldcg(&sw.hist[(size_t)s * 2048 + b]);
    find_bin(sm, 2048, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;
    int32_t* cnt = sw.counters + s * 4;
    int32_t* winners = sw.winners + (size_t)s * kB;
    uint2* cand = sw.cand + (size_t)s * kDecodeCand;
    int64_t lo, hi;
    cta_range(nvis, blockIdx.x, gridDim.x, lo, hi);
    for (int64_t b0 = lo; b0 < hi; b0 += SC_THREADS) {
        const int64_t b = b0 + tid;
        const uint32_t key = b < hi ? float_key(__ldcg(row + b)) : 0u;
        const bool win = b < hi && (key >> 21) > b1;
        const bool tie = b < hi && (key >> 21) == b1;
        const int ws = cta_append(sm, win, cnt + 0, &base_slot);
        if (ws >= 0) winners[ws] = (int32_t)b;
        const int cs = cta_append(sm, tie, cnt + 1, &base_slot);
        if (cs >= 0 && cs < kDecodeCand) cand[cs] = make_uint2(key, (uint32_t)b);
    }
    // The last CTA of the sequence finishes the pick.
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(cnt + 2, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int n_win = __ldcg(cnt + 0);
    const int nc = __ldcg(cnt + 1);
    if (n_win != (int)(kB - need1) || nc > CAND || nc > kDecodeCand) {
        // Candidates overflow (e.g. thousands of equal scores): exact pick from the row.
        select_row(sm, row, nvis, kB, out, nsel + s);
        return;
    }
    for (int k2 = tid; k2 < n_win; k2 += SC_THREADS) sm.out[k2] = __ldcg(winners + k2);
    for (int c = tid; c < nc; c += SC_THREADS) {
        const uint2 e = __ldcg(cand + c);
        sm.cand_key[c] = e.x;
        sm.cand_idx[c] = (int32_t)e.y;
    }
    if (tid == 0) sm.n_out = n_win;
    __syncthreads();
    finish_from_candidates(sm, nc, b1, need1, kB, out);
    if (tid == 0) nsel[s] = kB;
}

}  // namespace

int decode_select_ctas(int batch) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return std::max(1, 2 * sms / std::max(batch, 1));
}

cudaError_t launch_decode_prepare(const LayerDims& L, int batch, const int64_t* pos,
                                  const uint16_t* k, const uint16_t* v, const uint16_t* idx_q,
                                  const uint16_t* idx_k, uint16_t* kc, uint16_t* vc,
                                  uint16_t* idx_k_cache, uint16_t* pooled, int64_t cap,
                                  const float* rms_w, uint16_t* qrot, DecodeSelWs sw,
                                  int32_t* status, cudaStream_t st) {
    note_launch();
    decode_prepare_kernel<<<batch, 128, 0, st>>>(pos, k, v, idx_q, idx_k, kc, vc, idx_k_cache,
                                                 pooled, cap, rms_w, L.kv_heads, L.r, L.rms_eps,
                                                 L.rope, qrot, sw, status);
    return cudaGetLastError();
}

cudaError_t launch_decode_scores(const LayerDims& L, int batch, const int64_t* pos,
                                 const uint16_t* qrot, const uint16_t* pooled, int64_t cap,
                                 float* scores, DecodeSelWs sw, cudaStream_t st) {
    note_launch();
    decode_scores_kernel<<<dim3((unsigned)decode_select_ctas(batch), (unsigned)batch), SC_THREADS, 0, st>>>(
        pos, qrot, pooled, cap, L.r, scores, sw.hist);
    return cudaGetLastError();
}

cudaError_t launch_decode_select(const LayerDims& L, int batch, const int64_t* pos, int64_t cap,
                                 const float* scores, DecodeSelWs sw, int32_t* sel, int32_t* nsel,
                                 cudaStream_t st) {
    const int smem = (int)sizeof(SelSmem);
    cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch();
    decode_select_kernel<<<dim3((unsigned)decode_select_ctas(batch), (unsigned)batch), SC_THREADS, smem, st>>>(
        pos, cap, L.r, L.kB, scores, sw, sel, nsel);
    return cudaGetLastError();
}

}  // namespace qsa
