// Stage-1 indexer distillation ("QSA (Qwen Sparse Attention)" concept page,
// "Native trainability via 2-stage continued pretraining", stage 1): the
// indexer scores are trained to match a block-max-pooled version of the dense
// teacher attention distribution through a KL loss. This library's reading:
//   p_i(j)  = (1/q_heads) sum_h softmax over j' <= i of (sm_scale <q_h, k_j'>)
//             (the dense causal distribution of every core head, averaged);
//   t_i(b)  = max over the r tokens j of block b of p_i(j), for the blocks the
//             indexer scores (b < floor(i/r)), normalised to sum to 1;
//   KL_i    = sum_b t_i(b) (log t_i(b) - log softmax_b(I_i)), and its gradient
//             dKL_i / dI_ib = (sum_b t_i(b)) softmax_b(I_i) - t_i(b).
//
// The target's kernels are in distill_tc.cu (tcgen05).
// distill_kl_kernel: one CTA per query row, three passes over the row (maximum,
// sum of exponentials and KL, gradient).
#include <algorithm>
#include <cmath>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int KLT = 256;  // threads per KL row

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, w) : v + w;
    }
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = red[0];
    for (int w = 1; w < KLT / 32; ++w) v = is_max ? fmaxf(v, red[w]) : v + red[w];
    return v;
}

__global__ void __launch_bounds__(KLT) distill_kl_kernel(int64_t q_begin, int64_t nq, const float* __restrict__ target,
                                                         const float* __restrict__ scores, int64_t ld, int r,
                                                         float* __restrict__ kl, float* __restrict__ dscores) {
    __shared__ float red[KLT / 32];
    const int64_t row = blockIdx.x;  // s * nq + j
    const int64_t i = q_begin + row % nq;
    const int64_t n = i / r;
    const float* tr = target + (size_t)row * ld;
    const float* sr = scores + (size_t)row * ld;
    float* dr = dscores ? dscores + (size_t)row * ld : nullptr;
    float mx = -INFINITY;
    for (int64_t b = threadIdx.x; b < n; b += KLT) mx = fmaxf(mx, sr[b]);
    mx = block_reduce(mx, red, true);
    float den = 0.f, tsum = 0.f, cross = 0.f, ent = 0.f;
    for (int64_t b = threadIdx.x; b < n; b += KLT) {
        const float x = sr[b] - mx;
        const float tb = tr[b];
        den += expf(x);
        tsum += tb;
        if (tb > 0.f) {
            cross += tb * x;
            ent += tb * logf(tb);
        }
    }
    den = block_reduce(den, red, false);
    tsum = block_reduce(tsum, red, false);
    cross = block_reduce(cross, red, false);
    ent = block_reduce(ent, red, false);
    const float log_den = logf(den);
    // sum_b t_b (log t_b - (s_b - max - log_den))
    if (threadIdx.x == 0) kl[row] = n > 0 ? ent - cross + tsum * log_den : 0.f;
    if (dr) {
        const float inv = 1.f / den;
        for (int64_t b = threadIdx.x; b < ld; b += KLT) dr[b] = b < n ? tsum * expf(sr[b] - mx) * inv - tr[b] : 0.f;
    }
}

}  // namespace

bool distill_target_supported(const LayerDims& L) {
    const int G = L.q_heads / L.kv_heads;
    const bool groups_tile = G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
    return L.q_heads <= 32 && groups_tile && (L.r == 1 || L.r == 2 || L.r == 4 || L.r == 8 || L.r == 16);
}

cudaError_t launch_distill_kl(const LayerDims& L, int batch, int64_t q_begin, int64_t nq, const float* target,
                              const float* scores, int64_t ld, float* kl, float* dscores, cudaStream_t st) {
    if (batch <= 0 || nq <= 0) return cudaSuccess;
    note_launch();
    distill_kl_kernel<<<(unsigned)(batch * nq), KLT, 0, st>>>(q_begin, nq, target, scores, ld, L.r, kl, dscores);
    return cudaGetLastError();
}

}  // namespace qsa
