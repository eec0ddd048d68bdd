// Low-precision caches: FP8 E4M3 codes with one fp32 scale per row. The
// "Qwen Sparse Attention" gallery page ("Community Quantized Version") reports
// a quantized variant without its format; this library's reading is the OCP
// E4M3 format with scale = fl32(max|x| / 448) and code = E4M3(fl32(x / scale))
// rounded to nearest even, magnitudes beyond 448 saturating; an all-zero row
// has scale 0 and codes 0.
//
// One warp per row (rows of 64, 128 or 256 values): the row's maximum magnitude
// by a warp reduction, both divisions correctly rounded in fp32, the codes by
// the hardware conversion. HBM stream: 2 bytes read and 1 written per value.
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

template <int E>  // values per lane
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const uint16_t* xr = x + (size_t)r * (32 * E) + lane * E;
        float v[E];
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            v[e] = bf16f(xr[e]);
            amax = fmaxf(amax, fabsf(v[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
        uint8_t* cr = codes + (size_t)r * (32 * E) + lane * E;
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const uint16_t c2 = scale > 0.f ? f32x2_to_e4m3x2(__fdiv_rn(v[e], scale), __fdiv_rn(v[e + 1], scale))
                                            : (uint16_t)0;
            cr[e] = (uint8_t)(c2 & 0xFF);
            cr[e + 1] = (uint8_t)(c2 >> 8);
        }
        if (lane == 0) scales[r] = scale;
    }
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t* x, int64_t rows, int dim, uint8_t* codes, float* scales,
                                 cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)sms * 8);
    note_launch();
    switch (dim) {
        case 64: quantize_rows_kernel<2><<<(unsigned)blocks, 256, 0, st>>>(x, rows, codes, scales); break;
        case 128: quantize_rows_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(x, rows, codes, scales); break;
        case 256: quantize_rows_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(x, rows, codes, scales); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace qsa
