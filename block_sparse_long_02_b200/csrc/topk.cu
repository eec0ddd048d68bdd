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

}  // namespace qsa
