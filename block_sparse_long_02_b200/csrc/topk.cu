// a5: top-k_B block selection over a materialised score row
// ("QSA (Qwen Sparse Attention)" concept page, (A) "Top-k_B block selection";
// "Qwen Sparse Attention" gallery page pseudo-code top_k(scores, k=512)).
// One CTA per row; the exact selection routine is in select.cuh.
#include <algorithm>

#include "kernels.h"
#include "select.cuh"

namespace qsa {
namespace {

__global__ void __launch_bounds__(T) select_rows_kernel(const float* __restrict__ scores, int64_t ld,
                                                        int64_t q_begin, int64_t j0, int64_t nrows,
                                                        int64_t nq_total, int batch, int r, int kB,
                                                        int32_t* __restrict__ sel,
                                                        int32_t* __restrict__ nsel) {
    extern __shared__ __align__(16) uint8_t raw[];
    SelSmem& sm = *reinterpret_cast<SelSmem*>(raw);
    const int64_t rows = (int64_t)batch * nrows;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t s = row / nrows, jr = row % nrows;
        const int64_t i = q_begin + j0 + jr;
        const int64_t out_row = s * nq_total + j0 + jr;
        select_row(sm, scores + (size_t)row * ld, i / r, kB, sel + (size_t)out_row * kB,
                   nsel + out_row);
        __syncthreads();
    }
}

// Exact top k_B (by score desc, block asc) of n <= CAND entries already in
// sm.cand_key (order-preserving keys) / sm.cand_idx, written ascending to sel.
// Level 1 here (winners above the threshold digit to sm.out, the digit's
// entries compacted in place to the front), the rest in finish_from_candidates.
__device__ void select_smem(SelSmem& sm, int n, int kB, int32_t* sel) {
    const int tid = threadIdx.x;
    clear_hist(sm);
    for (int c = tid; c < n; c += T) atomicAdd(&sm.hist[sm.cand_key[c] >> 21], 1u);
    find_bin(sm, BINS, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;
    if (tid == 0) sm.n_out = 0;
    __syncthreads();
    uint32_t nc = 0;
    for (int c0 = 0; c0 < n; c0 += T) {  // same trip count in every thread
        const int c = c0 + tid;
        const uint32_t key = c < n ? sm.cand_key[c] : 0u;
        const int32_t idx = c < n ? sm.cand_idx[c] : 0;
        const uint32_t d = key >> 21;
        warp_push(sm, c < n && d > b1, idx);
        const bool is_c = c < n && d == b1;
        uint32_t pre;
        const uint32_t tot = cta_scan(sm, is_c, pre);  // every read of this round is done
        if (is_c) {  // position nc + pre <= c: only entries already read are overwritten
            sm.cand_key[nc + pre] = key;
            sm.cand_idx[nc + pre] = idx;
        }
        nc += tot;
        __syncthreads();
    }
    finish_from_candidates(sm, (int)nc, b1, need1, kB, sel);
}

// Merge of the fused indexer's per-split top-k lists: one CTA per query row.
__global__ void __launch_bounds__(T) split_merge_kernel(const uint2* __restrict__ split_out,
                                                        const int32_t* __restrict__ split_cnt, int splits,
                                                        int64_t nq, int64_t q_begin, int batch, int r, int kB,
                                                        int qt_rows, int32_t* __restrict__ sel,
                                                        int32_t* __restrict__ nsel) {
    extern __shared__ __align__(16) uint8_t raw[];
    SelSmem& sm = *reinterpret_cast<SelSmem*>(raw);
    __shared__ int offs[CAND / 64 + 1];
    const int64_t j = blockIdx.x;
    const int s = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t row = (int64_t)s * nq + j;
    const int64_t c = (q_begin + j) / r;
    int32_t* out = sel + (size_t)row * kB;
    if (c <= kB) {  // every visible block is selected
        for (int k = tid; k < kB; k += T) out[k] = k < c ? k : -1;
        if (tid == 0) nsel[row] = (int32_t)c;
        return;
    }
    const int64_t nqt = (nq + qt_rows - 1) / qt_rows;
    const int64_t tu = (nqt - 1 - j / qt_rows) * batch + s;
    const int q = (int)(j % qt_rows);
    if (tid == 0) {
        int acc = 0;
        for (int sp = 0; sp < splits; ++sp) {
            offs[sp] = acc;
            acc += split_cnt[((size_t)tu * splits + sp) * qt_rows + q];
        }
        offs[splits] = acc;
    }
    __syncthreads();
    const int n = offs[splits];  // >= k_B (each split holds min(k_B, its visible blocks))
    for (int sp = 0; sp < splits; ++sp) {
        const uint2* src = split_out + (((size_t)tu * splits + sp) * qt_rows + q) * kB;
        const int o = offs[sp], cnt = offs[sp + 1] - o;
        for (int k = tid; k < cnt; k += T) {
            const uint2 e = src[k];
            sm.cand_key[o + k] = float_key(__uint_as_float(e.x));
            sm.cand_idx[o + k] = (int32_t)e.y;
        }
    }
    __syncthreads();
    select_smem(sm, n, kB, out);
    if (tid == 0) nsel[row] = kB;
}

int sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace

cudaError_t launch_select_rows(const LayerDims& L, int batch, const float* scores, int64_t ld,
                               int64_t q_begin, int64_t j0, int64_t nrows, int64_t nq_total,
                               int32_t* sel, int32_t* nsel, cudaStream_t st) {
    if (nrows <= 0 || batch <= 0) return cudaSuccess;
    const int smem = (int)sizeof(SelSmem);
    cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int64_t rows = (int64_t)batch * nrows;
    const int grid = (int)std::min<int64_t>(rows, (int64_t)sms() * 4);
    note_launch();
    select_rows_kernel<<<grid, T, smem, st>>>(scores, ld, q_begin, j0, nrows, nq_total, batch, L.r,
                                              L.kB, sel, nsel);
    return cudaGetLastError();
}

cudaError_t launch_split_merge(const LayerDims& L, int batch, int64_t nq, int64_t q_begin, int qt_rows,
                               int splits, const uint2* split_out, const int32_t* split_cnt, int32_t* sel,
                               int32_t* nsel, cudaStream_t st) {
    if (nq <= 0 || batch <= 0) return cudaSuccess;
    if ((int64_t)splits * L.kB > CAND) return cudaErrorInvalidValue;
    const int smem = (int)sizeof(SelSmem);
    cudaFuncSetAttribute(split_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch();
    split_merge_kernel<<<dim3((unsigned)nq, (unsigned)batch), T, smem, st>>>(
        split_out, split_cnt, splits, nq, q_begin, batch, L.r, L.kB, qt_rows, sel, nsel);
    return cudaGetLastError();
}

}  // namespace qsa
