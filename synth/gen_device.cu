// Seeded synthetic inputs, device side: the same counter-based generator as
// gen_host.c, drawn on the GPU so that multi-GB inputs need no host pass.
// Holds none of the layer's arithmetic. Bit-identical to the host generator
// (integer arithmetic, one exact int->fp32 conversion, explicit RNE to bf16).
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t sm64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint16_t draw(uint64_t key, uint64_t e) {
    int32_t s = 0;
#pragma unroll
    for (int w = 0; w < 3; ++w) {
        uint64_t r = sm64(key + 3ull * e + (uint64_t)w);
        s += (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF) +
             (int32_t)((r >> 32) & 0xFFFF) + (int32_t)(r >> 48);
    }
    s -= 393210;
    float f = (float)s * (1.0f / 65536.0f);
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void fill_kernel(uint64_t key, uint64_t e0, uint64_t count, uint16_t* __restrict__ out) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
        out[i] = draw(key, e0 + i);
}

uint64_t host_sm64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

}  // namespace

// out[i] = value(e0 + i) for i < count, on `stream`. Returns a cudaError_t code.
extern "C" int synth_fill_device(uint64_t seed, uint64_t tensor_id, uint64_t e0, uint64_t count,
                                 uint16_t* out, void* stream) {
    if (count == 0) return 0;
    uint64_t key = host_sm64(seed ^ host_sm64(tensor_id + 0x632BE59BD9B4E019ull));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t want = (count + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    unsigned grid = (unsigned)(want < cap ? want : cap);
    fill_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(key, e0, count, out);
    return (int)cudaGetLastError();
}
