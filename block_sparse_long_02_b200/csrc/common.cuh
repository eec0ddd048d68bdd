// Internal helpers shared by the QSA kernels (not part of the C-ABI).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace qsa {

constexpr int kIdxDim = 128;   // indexer head dim (one shared key head)
constexpr int kIdxHeads = 4;   // indexer query heads
constexpr int kHeadDim = 128;  // core head dim
constexpr int kMaxKB = 4096;   // largest supported k_B
constexpr int kWsHeader = 256; // every workspace starts with this many bytes of status

// theta_j = base^(-2j/rope_dims) for j < half, computed on the host in fp64.
struct RopeTable {
    double theta[64];
    int half;
};

// ---------------------------------------------------------------- bf16 / floats
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// fp64 -> bf16 bits, round to nearest even in a single rounding: clear all but
// the top 7 explicit significand bits of the double with RNE, then narrow
// (exactly) to fp32 and keep the high half.
__device__ __forceinline__ uint16_t f64_to_bf16(double x) {
    unsigned long long u = (unsigned long long)__double_as_longlong(x);
    const unsigned long long half_ulp = 1ull << 44, mask = (1ull << 45) - 1ull;
    u = (u + (half_ulp - 1ull) + ((u >> 45) & 1ull)) & ~mask;
    float f = __double2float_rn(__longlong_as_double((long long)u));
    return (uint16_t)(__float_as_uint(f) >> 16);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
    uint32_t u = __float_as_uint(x);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16(lo) | ((uint32_t)f32_to_bf16(hi) << 16);
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz;
// relative error about 2^-22, subnormal results flushed to zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Order-preserving map of fp32 onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// First error wins.
__device__ __forceinline__ void flag_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before
// the previous kernel in the stream has finished; pdl_wait() blocks until
// every earlier grid has completed and its writes are visible (a no-op for a
// normal launch), and pdl_trigger() lets the next such kernel start launching.
// Decode kernels call both first thing, so they read nothing early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------ thread-block clusters (DSMEM)
// Barrier over every thread of every CTA of the cluster, with release/acquire
// ordering of shared-memory writes before it and reads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_dsmem(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Split cluster barrier: arrive early (no ordering), wait before the first
// access to another CTA's shared memory (every CTA of the cluster has started).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// --------------------------------------------------------------- cp.async / mma
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
    int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A(16x16, row) * B(16x8, col), f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4-byte asynchronous copy; zero-fill when !valid.
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, bool valid) {
    int sz = valid ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}

// Two FP8 E4M3 codes (low byte = first) -> two f16 (low half = first); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes) {
    uint32_t d;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(codes));
    return d;
}
// Two fp32 -> two FP8 E4M3 codes (low byte = lo), round to nearest even,
// magnitudes beyond 448 saturating.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}
// Two fp32 -> f16x2 (low half = lo), round to nearest even.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
// f16x2 a * b, round to nearest even.
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// One warp quantizes a 128-value bf16 row to FP8 E4M3 codes and an fp32
// scale: scale = fl32(max|x| / 448) (0 for an all-zero row), code =
// E4M3(fl32(x / scale)) rounded to nearest even, saturating. Lane l handles
// values 4 l .. 4 l + 3.
__device__ __forceinline__ void quantize_row128_warp(const uint16_t* x, uint8_t* codes, float* scale_out,
                                                     int lane) {
    const uint2 raw = *reinterpret_cast<const uint2*>(x + lane * 4);
    const float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
    uint32_t packed = 0u;
    if (scale > 0.f)
        packed = (uint32_t)f32x2_to_e4m3x2(__fdiv_rn(v[0], scale), __fdiv_rn(v[1], scale)) |
                 ((uint32_t)f32x2_to_e4m3x2(__fdiv_rn(v[2], scale), __fdiv_rn(v[3], scale)) << 16);
    *reinterpret_cast<uint32_t*>(codes + lane * 4) = packed;
    if (lane == 0) *scale_out = scale;
}

// Byte offset of 16-byte chunk `c` (0..15) of 256-byte row `row` in a
// row-swizzled tile: conflict-free ldmatrix over 8 consecutive rows.
__device__ __forceinline__ uint32_t swz256(int row, int c) {
    return (uint32_t)(row * 256 + ((c ^ (row & 7)) << 4));
}

}  // namespace qsa
