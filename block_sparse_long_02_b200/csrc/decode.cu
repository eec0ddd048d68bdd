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

constexpr int DS_THREADS = 256;  // fused score CTAs
constexpr int DS_WARPS = DS_THREADS / 32;

// Blocks [lo, hi) of a sequence's nvis visible blocks handled by CTA x of X.
__device__ __forceinline__ void cta_range(int64_t nvis, int x, int X, int64_t& lo, int64_t& hi) {
    const int64_t chunk = (nvis + X - 1) / X;
    lo = min(nvis, (int64_t)x * chunk);
    hi = min(nvis, lo + chunk);
}

// One decode step's cache update, query rotation and score stream, fused.
//
// CTA (0, s) appends the new token's K, V and raw indexer key to the caches
// and, when the token closes its block, pools that block for later steps (a8;
// the block is not visible at this position, so no CTA of this step reads
// it); with more than one CTA per sequence it scores nothing, so the slow
// fp64 rotation of the pooling never delays a score slice. The other CTAs
// rotate the new indexer query themselves (a3', fp64, from one shared table
// of the position's angles) and score their slices of the visible pooled
// keys (a4) on the tensor cores:
// mma.sync m16n8k16 with A = 16 pooled keys x 16 dims and B = 16 dims x
// (4 heads + 4 zero columns). The 128 dims are taken in a fixed permutation
// (the same for keys and query, so every dot product is unchanged) chosen so
// that lane (g, t) of a warp reads its A fragments for all 8 k-steps of rows
// g and g + 8 with four 16-byte loads per row: chunk i of lane t is bytes
// [64 i + 16 t, +16) of the row, and k-step j uses its pairs 2 (j % 2) and
// 2 (j % 2) + 1 of chunk j / 2 as the low and high column pairs. The ReLU
// head sum takes one shuffle; the scores go to `scores` and their top 11 key
// bits to the sequence's histogram (zeroed by the selection after use).
__global__ void __launch_bounds__(DS_THREADS) decode_score_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, int kB, double eps, RopeTable rt,
    float* __restrict__ scores, uint32_t* __restrict__ hist_g, int32_t* __restrict__ status) {
    __shared__ uint32_t hist[2048];
    __shared__ __align__(16) uint16_t qs[kIdxHeads * kIdxDim];
    __shared__ double2 cs[kIdxDim / 2];  // (sin, cos) of the query position's angles
    pdl_wait();
    pdl_trigger();
    const int s = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t p = pos[s];
    if (p < 0 || p >= cap) {
        if (blockIdx.x == 0 && tid == 0) flag_status(status, 4 /* QSA_ERR_CAPACITY */);
        return;
    }
    if (blockIdx.x == 0) {
        const int row16 = kv_heads * kHeadDim / 8;  // 16-byte chunks per kv row
        const uint4* ks = reinterpret_cast<const uint4*>(k + (size_t)s * kv_heads * kHeadDim);
        const uint4* vs = reinterpret_cast<const uint4*>(v + (size_t)s * kv_heads * kHeadDim);
        uint4* kd = reinterpret_cast<uint4*>(kc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
        uint4* vd = reinterpret_cast<uint4*>(vc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
        for (int c = tid; c < row16; c += DS_THREADS) {
            kd[c] = ks[c];
            vd[c] = vs[c];
        }
        if (tid < kIdxDim / 8)
            reinterpret_cast<uint4*>(idx_k_cache + ((size_t)s * cap + p) * kIdxDim)[tid] =
                reinterpret_cast<const uint4*>(idx_k + (size_t)s * kIdxDim)[tid];
        // The block's last raw key is read from the input (its cache row is
        // written by another thread of this CTA).
        if (warp == kIdxHeads && (p + 1) % r == 0) {
            const int64_t b = p / r;
            pool_block_warp(idx_k_cache + ((size_t)s * cap + (size_t)b * r) * kIdxDim,
                            idx_k + (size_t)s * kIdxDim, r, rms_w, eps, b * r, rt,
                            pooled + ((size_t)s * (cap / r) + b) * kIdxDim, lane);
        }
    }
    const int64_t pcap = cap / r;
    if (p / r <= kB) return;  // every visible block is selected: no scores needed
    const int X = gridDim.x > 1 ? (int)gridDim.x - 1 : 1;  // scoring CTAs
    const int x = gridDim.x > 1 ? (int)blockIdx.x - 1 : 0;
    if (x < 0) return;                                     // CTA 0 only appends and pools
    int64_t lo, hi;
    cta_range(p / r, x, X, lo, hi);
    if (lo >= hi) return;
    // The rope_dims / 2 angles of position p once per CTA (an fp64 sincos of a
    // large argument is slow), then the 4 heads rotate from the table.
    if (tid < rt.half) {
        double sn, cn;
        sincos(__dmul_rn((double)p, rt.theta[tid]), &sn, &cn);
        cs[tid] = make_double2(sn, cn);
    }
    for (int b = tid; b < 2048; b += DS_THREADS) hist[b] = 0u;
    __syncthreads();
    if (warp < kIdxHeads)
        rotate_head_warp_tab(idx_q + ((size_t)s * kIdxHeads + warp) * kIdxDim, rt.half, cs, qs + warp * kIdxDim,
                             lane);
    __syncthreads();
    const int g = lane >> 2, t = lane & 3;
    // B fragments: column g (head g, zero for g >= 4), k-step j.
    uint32_t bq0[8], bq1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d = 32 * (j >> 1) + 8 * t + 4 * (j & 1);
        bq0[j] = g < kIdxHeads ? *reinterpret_cast<const uint32_t*>(qs + g * kIdxDim + d) : 0u;
        bq1[j] = g < kIdxHeads ? *reinterpret_cast<const uint32_t*>(qs + g * kIdxDim + d + 2) : 0u;
    }
    const uint16_t* keys = pooled + (size_t)s * pcap * kIdxDim;
    float* dst = scores + (size_t)s * pcap;
    auto load = [&](int64_t base, uint4 (&ra)[4], uint4 (&rb)[4]) {
        const int64_t b0 = base + g, b1 = b0 + 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ra[i] = b0 < hi ? __ldg(reinterpret_cast<const uint4*>(keys + (size_t)b0 * kIdxDim + 32 * i + 8 * t))
                            : make_uint4(0u, 0u, 0u, 0u);
            rb[i] = b1 < hi ? __ldg(reinterpret_cast<const uint4*>(keys + (size_t)b1 * kIdxDim + 32 * i + 8 * t))
                            : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    const int64_t step = 16 * DS_WARPS;
    int64_t base = lo + 16 * warp;
    uint4 ca[4], cb[4];
    load(base, ca, cb);
    for (; base < hi; base += step) {
        uint4 na[4], nb[4];
        load(base + step, na, nb);  // the next group, in flight during this one
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mma_bf16_16816(c, ca[i].x, cb[i].x, ca[i].y, cb[i].y, bq0[2 * i], bq1[2 * i]);
            mma_bf16_16816(c, ca[i].z, cb[i].z, ca[i].w, cb[i].w, bq0[2 * i + 1], bq1[2 * i + 1]);
        }
        // Lane t = 0 holds heads 0, 1 and lane t = 1 heads 2, 3 of rows g, g + 8.
        float sa = fmaxf(c[0], 0.f) + fmaxf(c[1], 0.f);
        float sb = fmaxf(c[2], 0.f) + fmaxf(c[3], 0.f);
        sa += __shfl_xor_sync(0xffffffffu, sa, 1);
        sb += __shfl_xor_sync(0xffffffffu, sb, 1);
        if (t == 0) {
            const int64_t b0 = base + g, b1 = b0 + 8;
            if (b0 < hi) {
                dst[b0] = sa;
                atomicAdd(&hist[float_key(sa) >> 21], 1u);
            }
            if (b1 < hi) {
                dst[b1] = sb;
                atomicAdd(&hist[float_key(sb) >> 21], 1u);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ca[i] = na[i];
            cb[i] = nb[i];
        }
    }
    __syncthreads();
    for (int b = tid; b < 2048; b += DS_THREADS)
        if (hist[b]) atomicAdd(&hist_g[(size_t)s * 2048 + b], hist[b]);
}

// The sequence's histogram and counters back to zero for the next step (the
// score kernel only adds to them). Called by the last CTA, after every CTA
// of the sequence has read them.
__device__ __forceinline__ void reset_state(DecodeSelWs& sw, int s) {
    for (int b = threadIdx.x; b < 2048; b += blockDim.x) sw.hist[(size_t)s * 2048 + b] = 0u;
    if (threadIdx.x < 4) sw.counters[s * 4 + threadIdx.x] = 0;
}

// Exclusive prefix over the CTA (thread order) of a per-thread packed count;
// returns the CTA total. All threads must call it.
__device__ __forceinline__ uint32_t cta_prefix(SelSmem& sm, uint32_t v, uint32_t& prefix) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) sm.wsum[w] = inc;
    __syncthreads();
    uint32_t base = 0, total = 0;
    for (int k = 0; k < NW; ++k) {
        const uint32_t x = sm.wsum[k];
        if (k < w) base += x;
        total += x;
    }
    __syncthreads();
    prefix = base + inc - v;
    return total;
}

__global__ void __launch_bounds__(SC_THREADS) decode_select_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int r, int kB, const float* __restrict__ scores,
    DecodeSelWs sw, int32_t* __restrict__ sel, int32_t* __restrict__ nsel) {
    extern __shared__ __align__(16) uint8_t raw[];
    SelSmem& sm = *reinterpret_cast<SelSmem*>(raw);
    __shared__ unsigned long long slot_base;  // (candidates << 32) | winners before this round
    __shared__ int last;
    pdl_wait();
    pdl_trigger();
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
    reinterpret_cast<uint4*>(sm.hist)[tid] = __ldcg(reinterpret_cast<const uint4*>(sw.hist + (size_t)s * 2048) + tid);
    find_bin(sm, 2048, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;
    int32_t* cnt = sw.counters + s * 4;
    int32_t* winners = sw.winners + (size_t)s * kB;
    uint2* cand = sw.cand + (size_t)s * kDecodeCand;
    // Sure winners (digit above b1) and candidates (digit b1) of this CTA's
    // slice, 8 entries per thread per round (coalesced: entry e of thread t
    // is r0 + e T + t); one scan and one 64-bit atomic on (winners,
    // candidates) place a round's entries.
    int64_t lo, hi;
    cta_range(nvis, blockIdx.x, gridDim.x, lo, hi);
    constexpr int E = 8;
    for (int64_t r0 = lo; r0 < hi; r0 += (int64_t)E * SC_THREADS) {
        uint32_t key[E];
        uint32_t nw = 0, ncand = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int64_t b = r0 + (int64_t)e * SC_THREADS + tid;
            key[e] = b < hi ? float_key(__ldcg(row + b)) : 0u;
            nw += (b < hi && (key[e] >> 21) > b1) ? 1u : 0u;
            ncand += (b < hi && (key[e] >> 21) == b1) ? 1u : 0u;
        }
        uint32_t pre;
        const uint32_t tot = cta_prefix(sm, (ncand << 16) | nw, pre);
        if (tid == 0) {
            const unsigned long long add = ((unsigned long long)(tot >> 16) << 32) | (tot & 0xFFFFu);
            slot_base = tot ? atomicAdd(reinterpret_cast<unsigned long long*>(cnt), add) : 0ull;
        }
        __syncthreads();
        int ws_ = (int)(uint32_t)slot_base + (int)(pre & 0xFFFFu);
        int cs = (int)(uint32_t)(slot_base >> 32) + (int)(pre >> 16);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int64_t b = r0 + (int64_t)e * SC_THREADS + tid;
            if (b >= hi) break;
            const uint32_t d = key[e] >> 21;
            if (d > b1) {
                if (ws_ < kB) winners[ws_] = (int32_t)b;  // < k_B by the histogram
                ++ws_;
            } else if (d == b1) {
                if (cs < kDecodeCand) cand[cs] = make_uint2(key[e], (uint32_t)b);
                ++cs;
            }
        }
        __syncthreads();
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
        reset_state(sw, s);
        return;
    }
    for (int k2 = tid; k2 < n_win; k2 += SC_THREADS) sm.out[k2] = __ldcg(winners + k2);
    for (int c = tid; c < nc; c += SC_THREADS) {
        const uint2 e = __ldcg(cand + c);
        sm.cand_key[c] = e.x;
        sm.cand_idx[c] = (int32_t)e.y;
    }
    if (tid == 0) sm.n_out = n_win;
    __syncthreads();  // (counters read by every thread before the reset)
    reset_state(sw, s);
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

// One wave: as many CTAs as fit on the GPU at once, split over the batch.
int decode_score_ctas(int batch) {
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_score_kernel, DS_THREADS, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return std::max(1, per_sm * sms / std::max(batch, 1));
}

cudaError_t launch_decode_score(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* k,
                                const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                                uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled,
                                int64_t cap, const float* rms_w, float* scores, DecodeSelWs sw,
                                int32_t* status, cudaStream_t st) {
    note_launch();
    return launch_pdl(decode_score_kernel, dim3((unsigned)decode_score_ctas(batch), (unsigned)batch),
                      dim3(DS_THREADS), 0, st, pos, k, v, idx_q, idx_k, kc, vc, idx_k_cache, pooled, cap, rms_w,
                      L.kv_heads, L.r, L.kB, L.rms_eps, L.rope, scores, sw.hist, status);
}

cudaError_t launch_decode_select(const LayerDims& L, int batch, const int64_t* pos, int64_t cap,
                                 const float* scores, DecodeSelWs sw, int32_t* sel, int32_t* nsel,
                                 cudaStream_t st) {
    const int smem = (int)sizeof(SelSmem);
    cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch();
    return launch_pdl(decode_select_kernel, dim3((unsigned)decode_select_ctas(batch), (unsigned)batch),
                      dim3(SC_THREADS), (size_t)smem, st, pos, cap, L.r, L.kB, scores, sw, sel, nsel);
}

}  // namespace qsa
