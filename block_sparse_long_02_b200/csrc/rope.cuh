// Partial RoPE and key pooling for one warp (lane l owns dims 4l .. 4l+3).
//
// "QSA (Qwen Sparse Attention)" concept page, (A): keys are average-pooled into
// blocks of r tokens, k_b = RMSNorm(AvgPool), and RoPE is applied to 64 of the
// 128 dims after compression; "Qwen Sparse Attention" gallery page, "How block
// selection works": normalisation first, then RoPE at the block's first
// position. The indexer query gets the same rotation at its own position.
//
// The arithmetic here is fp64 (the work is a few hundred bytes per block and
// memory-bound), with explicit IEEE operations so that the stored bf16 values
// are the correctly rounded results; at positions near 2^20 an fp32 angle
// would be off by ~0.06 rad.
#pragma once

#include "common.cuh"

namespace qsa {

// Rotates pairs (j, j + half), j < half = rope_dims/2, of the fp64 values
// x[0..3] = dims 4*lane .. 4*lane+3 at position pos. Requires half % 4 == 0.
// Every lane of the warp must call it (it shuffles).
__device__ __forceinline__ void rope_lane4(double (&x)[4], int lane, int64_t pos,
                                           const RopeTable& rt) {
    const int half = rt.half;
    const int d0 = lane * 4;
    const int qh = half >> 2;
    const int src = (d0 < half) ? lane + qh : (d0 < 2 * half ? lane - qh : lane);
    double y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = __shfl_sync(0xffffffffu, x[e], src);
    if (d0 < 2 * half) {
        const bool first = d0 < half;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = first ? d0 + e : d0 + e - half;
            const double a = __dmul_rn((double)pos, rt.theta[j]);
            double s, c;
            sincos(a, &s, &c);
            // first half:  x_j' = x_j cos - x_{j+half} sin
            // second half: x_{j+half}' = x_j sin + x_{j+half} cos
            x[e] = first ? __dsub_rn(__dmul_rn(x[e], c), __dmul_rn(y[e], s))
                         : __dadd_rn(__dmul_rn(y[e], s), __dmul_rn(x[e], c));
        }
    }
}

// rope_lane4 with the sines and cosines of the position's angles precomputed
// (cs[j] = (sin, cos) of pos * theta[j], j < half, the same operations as
// rope_lane4 uses, so the results are identical).
__device__ __forceinline__ void rope_lane4_tab(double (&x)[4], int lane, int half, const double2* cs) {
    const int d0 = lane * 4;
    const int qh = half >> 2;
    const int src = (d0 < half) ? lane + qh : (d0 < 2 * half ? lane - qh : lane);
    double y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = __shfl_sync(0xffffffffu, x[e], src);
    if (d0 < 2 * half) {
        const bool first = d0 < half;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = first ? d0 + e : d0 + e - half;
            const double s = cs[j].x, c = cs[j].y;
            x[e] = first ? __dsub_rn(__dmul_rn(x[e], c), __dmul_rn(y[e], s))
                         : __dadd_rn(__dmul_rn(y[e], s), __dmul_rn(x[e], c));
        }
    }
}

// Loads 4 bf16 dims (8 bytes) of a row as fp64.
__device__ __forceinline__ void load4(const uint16_t* p, double (&v)[4]) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    v[0] = (double)bf16_lo(w.x);
    v[1] = (double)bf16_hi(w.x);
    v[2] = (double)bf16_lo(w.y);
    v[3] = (double)bf16_hi(w.y);
}

__device__ __forceinline__ void store4(uint16_t* p, const double (&v)[4]) {
    uint2 w;
    w.x = (uint32_t)f64_to_bf16(v[0]) | ((uint32_t)f64_to_bf16(v[1]) << 16);
    w.y = (uint32_t)f64_to_bf16(v[2]) | ((uint32_t)f64_to_bf16(v[3]) << 16);
    *reinterpret_cast<uint2*>(p) = w;
}

// a1-a3 for one complete block, by one warp. rows: the block's first r-1 raw
// keys (consecutive 128-dim rows); last: its final raw key (may live
// elsewhere, as in decode where it is the token being appended).
__device__ __forceinline__ void pool_block_warp(const uint16_t* rows, const uint16_t* last, int r,
                                                const float* w, double eps, int64_t pos,
                                                const RopeTable& rt, uint16_t* out, int lane) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int t = 0; t < r; ++t) {
        double v[4];
        load4((t == r - 1 ? last : rows + (size_t)t * kIdxDim) + lane * 4, v);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = __dadd_rn(acc[e], v[e]);
    }
    double x[4], ss = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[e] = __ddiv_rn(acc[e], (double)r);
        ss = __dadd_rn(ss, __dmul_rn(x[e], x[e]));
    }
    ss = warp_sum(ss);
    const double rms = __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)kIdxDim), eps));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[e] = __ddiv_rn(x[e], rms);
        if (w) x[e] = __dmul_rn(x[e], (double)w[lane * 4 + e]);
    }
    rope_lane4(x, lane, pos, rt);
    store4(out + lane * 4, x);
}

// a3': rotate one 128-dim indexer query head at position pos, store as bf16.
__device__ __forceinline__ void rotate_head_warp(const uint16_t* in, int64_t pos,
                                                 const RopeTable& rt, uint16_t* out, int lane) {
    double x[4];
    load4(in + lane * 4, x);
    rope_lane4(x, lane, pos, rt);
    store4(out + lane * 4, x);
}

// rotate_head_warp with a precomputed (sin, cos) table of the position.
__device__ __forceinline__ void rotate_head_warp_tab(const uint16_t* in, int half, const double2* cs,
                                                     uint16_t* out, int lane) {
    double x[4];
    load4(in + lane * 4, x);
    rope_lane4_tab(x, lane, half, cs);
    store4(out + lane * 4, x);
}

}  // namespace qsa
