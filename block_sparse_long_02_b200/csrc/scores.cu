// a4 materialised: I[i][b] = sum_h ReLU(<q_i^h, k_b>) for b < floor(i/r)
// ("QSA (Qwen Sparse Attention)" concept page, (A) block importance with
// block-causal masking). Used by qsa_index_scores and by the row-select path
// of qsa_topk_blocks when scores are given.
//
// Warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32 accumulation).
// A CTA keeps 32 queries x 4 heads of rotated indexer queries resident in
// shared memory and streams 128-block tiles of pooled keys through a
// double-buffered cp.async ring. Each warp owns 16 queries x 32 blocks; its
// four m16 tiles are the four heads of the same 16 queries, so the ReLU-sum
// over heads happens inside each thread's accumulators with no shuffles.
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int QT = 32;    // queries per CTA
constexpr int BT = 128;   // blocks per tile
constexpr int THREADS = 256;
constexpr int A_BYTES = QT * kIdxHeads * 256;  // 32 KB
constexpr int B_BYTES = BT * 256;              // 32 KB per stage
constexpr int SMEM = A_BYTES + 2 * B_BYTES;

__device__ __forceinline__ void load_b_tile(uint32_t sb, const uint16_t* pooled_s, int64_t pcap,
                                            int64_t b0, int tid) {
#pragma unroll
    for (int k = 0; k < (BT * 16) / THREADS; ++k) {
        const int idx = tid + k * THREADS;  // chunk id
        const int row = idx >> 4, c = idx & 15;
        const int64_t b = b0 + row;
        const bool ok = b < pcap;
        const uint16_t* src = pooled_s + (size_t)(ok ? b : 0) * kIdxDim + c * 8;
        cp_async16_zfill(sb + swz256(row, c), src, ok);
    }
}

__global__ void __launch_bounds__(THREADS) index_scores_kernel(
    const uint16_t* __restrict__ qrot, int64_t nq, int64_t q_begin, int64_t j0, int64_t nrows,
    const uint16_t* __restrict__ pooled, int64_t pcap, float* __restrict__ scores, int64_t ld,
    int r, bool fill_masked) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sA = smem_u32(smem);
    const uint32_t sB = sA + A_BYTES;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qsub = warp >> 2, bsub = warp & 3;
    const int s = blockIdx.y;
    const int64_t row0 = (int64_t)blockIdx.x * QT;  // first row (relative to j0)
    const int64_t rows_here = (nrows - row0) < QT ? (nrows - row0) : QT;
    // Visible blocks of the last query of the tile bound the tiles to visit.
    const int64_t vis_max = (q_begin + j0 + row0 + rows_here - 1) / r;
    const int64_t limit = fill_masked ? ld : (vis_max < ld ? vis_max : ld);
    const int64_t ntiles = (limit + BT - 1) / BT;
    const uint16_t* pooled_s = pooled + (size_t)s * pcap * kIdxDim;

    int64_t tile = blockIdx.z;
    if (tile >= ntiles) return;

    // Resident A: row (h*32 + q) holds head h of query q.
#pragma unroll
    for (int k = 0; k < (QT * kIdxHeads * 16) / THREADS; ++k) {
        const int idx = tid + k * THREADS;
        const int q = idx >> 6, h = (idx >> 4) & 3, c = idx & 15;
        const bool ok = q < rows_here;
        const uint16_t* src =
            qrot + (((size_t)s * nq + (ok ? j0 + row0 + q : 0)) * kIdxHeads + h) * kIdxDim + c * 8;
        cp_async16_zfill(sA + swz256(h * QT + q, c), src, ok);
    }
    load_b_tile(sB, pooled_s, pcap, tile * BT, tid);
    cp_async_commit();

    const int g = lane >> 2, tig = lane & 3;
    int stage = 0;
    for (; tile < ntiles; tile += gridDim.z) {
        const int64_t next = tile + gridDim.z;
        if (next < ntiles) {
            load_b_tile(sB + (stage ^ 1) * B_BYTES, pooled_s, pcap, next * BT, tid);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t sb = sB + stage * B_BYTES;

        float acc[kIdxHeads][4][4];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][nt][e] = 0.f;

#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t bfr[4][2];
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                const int nrow = bsub * 32 + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
                const int c = ks * 2 + ((lane >> 3) & 1);
                ldmatrix_x4(sb + swz256(nrow, c), bfr[2 * np][0], bfr[2 * np][1],
                            bfr[2 * np + 1][0], bfr[2 * np + 1][1]);
            }
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) {
                uint32_t a0, a1, a2, a3;
                const int q = qsub * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = ks * 2 + (lane >> 4);
                ldmatrix_x4(sA + swz256(h * QT + q, c), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    mma_bf16_16816(acc[h][nt], a0, a1, a2, a3, bfr[nt][0], bfr[nt][1]);
            }
        }

        // Epilogue: ReLU-sum over the four heads, block-causal mask, store.
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int64_t rrow = row0 + qsub * 16 + g + half * 8;
            if (rrow >= nrows) continue;
            const int64_t vis = (q_begin + j0 + rrow) / r;
            float* dst = scores + ((size_t)s * nrows + rrow) * ld;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int64_t b = tile * BT + bsub * 32 + nt * 8 + 2 * tig + e;
                    if (b >= ld) continue;
                    float v = 0.f;
#pragma unroll
                    for (int h = 0; h < kIdxHeads; ++h) v += fmaxf(acc[h][nt][half * 2 + e], 0.f);
                    if (b < vis)
                        dst[b] = v;
                    else if (fill_masked)
                        dst[b] = -INFINITY;
                }
        }
        __syncthreads();
        stage ^= 1;
    }
}

}  // namespace

cudaError_t launch_index_scores(const LayerDims& L, int batch, const uint16_t* qrot, int64_t nq,
                                int64_t q_begin, int64_t j0, int64_t nrows, const uint16_t* pooled,
                                int64_t cap, float* scores, int64_t ld, bool fill_masked,
                                cudaStream_t st) {
    if (nrows <= 0 || batch <= 0 || ld <= 0) return cudaSuccess;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(index_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        attr = true;
    }
    const int64_t qtiles = (nrows + QT - 1) / QT;
    const int64_t limit = fill_masked ? ld : std::min<int64_t>(ld, (q_begin + j0 + nrows - 1) / L.r);
    const int64_t ntiles = std::max<int64_t>(1, (limit + BT - 1) / BT);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Enough CTAs for ~4 waves; each CTA walks a strided subset of the block tiles.
    int64_t z = (4LL * sms * 2 + qtiles * batch - 1) / (qtiles * batch);
    z = std::max<int64_t>(1, std::min<int64_t>(z, ntiles));
    z = std::min<int64_t>(z, 65535);
    dim3 grid((unsigned)qtiles, (unsigned)batch, (unsigned)z);
    note_launch();
    index_scores_kernel<<<grid, THREADS, SMEM, st>>>(qrot, nq, q_begin, j0, nrows, pooled,
                                                     cap / L.r, scores, ld, L.r, fill_masked);
    return cudaGetLastError();
}

}  // namespace qsa
