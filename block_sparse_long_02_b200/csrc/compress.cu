// a1-a3 (pool, RMSNorm, partial RoPE of the indexer keys) and a3' (rotation of
// the indexer queries). Memory-bound streams: one warp per block or per head,
// 8-byte coalesced loads, fp64 arithmetic (see rope.cuh).
#include "kernels.h"
#include "rope.cuh"

namespace qsa {
namespace {

__global__ void __launch_bounds__(256) compress_kernel(const uint16_t* __restrict__ idx_k,
                                                       int64_t cap, int batch,
                                                       const float* __restrict__ w,
                                                       int64_t blk_begin, int64_t nblk, int r,
                                                       double eps, RopeTable rt,
                                                       uint16_t* __restrict__ pooled) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t total = (int64_t)batch * nblk;
    const int64_t pcap = cap / r;
    for (int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; item < total;
         item += nwarps) {
        const int64_t s = item / nblk;
        const int64_t b = blk_begin + item % nblk;
        const uint16_t* rows = idx_k + ((size_t)s * cap + (size_t)b * r) * kIdxDim;
        pool_block_warp(rows, rows + (size_t)(r - 1) * kIdxDim, r, w, eps, b * r, rt,
                        pooled + ((size_t)s * pcap + b) * kIdxDim, lane);
    }
}

__global__ void __launch_bounds__(256) rotate_queries_kernel(const uint16_t* __restrict__ idx_q,
                                                             int64_t q_begin, int64_t nq,
                                                             int64_t total, RopeTable rt,
                                                             uint16_t* __restrict__ qrot) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; item < total;
         item += nwarps) {
        // item = (s * nq + j) * 4 + h
        const int64_t j = (item / kIdxHeads) % nq;
        rotate_head_warp(idx_q + (size_t)item * kIdxDim, q_begin + j, rt,
                         qrot + (size_t)item * kIdxDim, lane);
    }
}

int grid_for(int64_t warps) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (warps + 7) / 8;  // 8 warps per 256-thread CTA
    const int64_t cap = (int64_t)sms * 8;
    return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_compress(const LayerDims& L, int batch, const uint16_t* idx_k, int64_t cap,
                            const float* rms_w, int64_t blk_begin, int64_t blk_end,
                            uint16_t* pooled, cudaStream_t st) {
    const int64_t nblk = blk_end - blk_begin;
    if (nblk <= 0 || batch <= 0) return cudaSuccess;
    note_launch();
    compress_kernel<<<grid_for(nblk * batch), 256, 0, st>>>(idx_k, cap, batch, rms_w, blk_begin,
                                                            nblk, L.r, L.rms_eps, L.rope, pooled);
    return cudaGetLastError();
}

cudaError_t launch_rotate_queries(const LayerDims& L, int batch, const uint16_t* idx_q,
                                  int64_t q_begin, int64_t nq, uint16_t* qrot, cudaStream_t st) {
    const int64_t total = (int64_t)batch * nq * kIdxHeads;
    if (total <= 0) return cudaSuccess;
    note_launch();
    rotate_queries_kernel<<<grid_for(total), 256, 0, st>>>(idx_q, q_begin, nq, total, L.rope,
                                                           qrot);
    return cudaGetLastError();
}

}  // namespace qsa
