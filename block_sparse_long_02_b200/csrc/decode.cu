// Decode step pieces: a8 (cache append and block pooling) with a3' (query
// rotation), and the a4 score stream over all pooled keys of a sequence.
// The score stream is the decode hot spot: it reads 256 bytes of pooled key
// per block and does 4 x 128 multiply-adds, so it is an HBM (or L2) stream;
// half-warps read one 256-byte block each with 16-byte loads.
#include <algorithm>

#include "kernels.h"
#include "rope.cuh"

namespace qsa {
namespace {

__global__ void __launch_bounds__(128) decode_prepare_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, double eps, RopeTable rt,
    uint16_t* __restrict__ qrot, int32_t* __restrict__ status) {
    const int s = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

__global__ void __launch_bounds__(256) decode_scores_kernel(const int64_t* __restrict__ pos,
                                                            const uint16_t* __restrict__ qrot,
                                                            const uint16_t* __restrict__ pooled,
                                                            int64_t cap, int r,
                                                            float* __restrict__ scores) {
    const int s = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int hl = lane & 15, hsel = lane >> 4;
    const int64_t p = pos[s];
    if (p < 0 || p >= cap) return;
    const int64_t pcap = cap / r;
    const int64_t nvis = p / r;
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
    const uint16_t* ks = pooled + (size_t)s * pcap * kIdxDim;
    float* dst = scores + (size_t)s * pcap;
    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t b0 = warp_id * 2; b0 < nvis; b0 += nwarps * 2) {
        const int64_t b = b0 + hsel;
        float d[kIdxHeads] = {0.f, 0.f, 0.f, 0.f};
        if (b < nvis) {
            const uint4 w = *reinterpret_cast<const uint4*>(ks + (size_t)b * kIdxDim + hl * 8);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = bf16_lo(ws[e]), x1 = bf16_hi(ws[e]);
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) {
                    d[h] = fmaf(qv[h][2 * e], x0, d[h]);
                    d[h] = fmaf(qv[h][2 * e + 1], x1, d[h]);
                }
            }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) d[h] += __shfl_xor_sync(0xffffffffu, d[h], o);
        if (hl == 0 && b < nvis)
            dst[b] = fmaxf(d[0], 0.f) + fmaxf(d[1], 0.f) + fmaxf(d[2], 0.f) + fmaxf(d[3], 0.f);
    }
}

}  // namespace

cudaError_t launch_decode_prepare(const LayerDims& L, int batch, const int64_t* pos,
                                  const uint16_t* k, const uint16_t* v, const uint16_t* idx_q,
                                  const uint16_t* idx_k, uint16_t* kc, uint16_t* vc,
                                  uint16_t* idx_k_cache, uint16_t* pooled, int64_t cap,
                                  const float* rms_w, uint16_t* qrot, int32_t* status,
                                  cudaStream_t st) {
    note_launch();
    decode_prepare_kernel<<<batch, 128, 0, st>>>(pos, k, v, idx_q, idx_k, kc, vc, idx_k_cache,
                                                 pooled, cap, rms_w, L.kv_heads, L.r, L.rms_eps,
                                                 L.rope, qrot, status);
    return cudaGetLastError();
}

cudaError_t launch_decode_scores(const LayerDims& L, int batch, const int64_t* pos,
                                 const uint16_t* qrot, const uint16_t* pooled, int64_t cap,
                                 float* scores, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t pcap = cap / L.r;
    // 16 blocks per CTA per sweep; cap the grid at ~8 CTAs per SM over the batch.
    int64_t x = (pcap + 15) / 16;
    const int64_t maxx = std::max<int64_t>(1, (int64_t)sms * 8 / batch);
    x = std::max<int64_t>(1, std::min<int64_t>(x, maxx));
    note_launch();
    decode_scores_kernel<<<dim3((unsigned)x, (unsigned)batch), 256, 0, st>>>(pos, qrot, pooled, cap,
                                                                            L.r, scores);
    return cudaGetLastError();
}

}  // namespace qsa
