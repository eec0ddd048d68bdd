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
// distill_target_kernel: one CTA per 8 consecutive queries of a sequence, one
// warp per query. Key chunks of 16 tokens (every kv head's rows) stream through
// a 2-stage cp.async ring shared by the CTA's warps. Each warp computes
// S^T = K Q^T on the tensor cores (mma.sync m16n8k16: the chunk's 16 tokens as
// the m16 rows, its query's heads as the n8 columns, query fragments held in
// registers for the whole sweep), so the head average of a token is a sum over
// the warp's own columns. Sweep 1 keeps a running sum of exponentials of every
// head over tokens <= i (its log-sum-exp); sweep 2 recomputes the logits,
// averages the probabilities over the heads, takes each block's maximum with
// shuffles, writes it and sums it; the warp then normalises its row.
// distill_kl_kernel: one CTA per query row, three passes over the row (maximum,
// sum of exponentials and KL, gradient).
#include <algorithm>
#include <cmath>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int DQ = 8;        // queries (warps) per CTA
constexpr int DCT = 16;      // tokens per key chunk
constexpr float LOG2E_D = 1.4426950408889634f;

template <int NTQ, int G>  // n8 head tiles per query; query heads per kv head (1, 2, 4, 8 or 16)
__global__ void __launch_bounds__(DQ * 32) distill_target_kernel(
    const uint16_t* __restrict__ q, int64_t q_begin, int64_t nq, const uint16_t* __restrict__ kc, int64_t cap,
    float* __restrict__ target, int64_t ld, int q_heads, int kv_heads, int r, float scale_log2) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int s = blockIdx.y;
    const int64_t j0 = (int64_t)blockIdx.x * DQ;
    const int64_t j = j0 + warp;
    const bool live = j < nq;
    const int64_t i = q_begin + (live ? j : j0);
    const int64_t n_vis = live ? i / r : 0;
    const int stage_bytes = kv_heads * DCT * 256;
    const uint32_t ring_s = smem_u32(smem);

    // Query fragments (B operand): column = head 8 k + gq, rows = dims.
    uint32_t qb[NTQ][8][2];
    const uint16_t* qrow = q + ((size_t)s * nq + (size_t)(live ? j : j0)) * q_heads * kHeadDim;
#pragma unroll
    for (int k = 0; k < NTQ; ++k) {
        const int h = 8 * k + gq;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[k][ks][0] = h < q_heads ? *reinterpret_cast<const uint32_t*>(qrow + h * kHeadDim + ks * 16 + 2 * t) : 0u;
            qb[k][ks][1] =
                h < q_heads ? *reinterpret_cast<const uint32_t*>(qrow + h * kHeadDim + ks * 16 + 8 + 2 * t) : 0u;
        }
    }

    // Chunk range: sweep 1 covers tokens <= the tile's last query, sweep 2 the
    // tokens of the tile's visible blocks.
    const int64_t i_last = q_begin + (j0 + DQ < nq ? j0 + DQ : nq) - 1;
    const int n1 = (int)((i_last + 1 + DCT - 1) / DCT);
    const int n2 = (int)(((i_last / r) * r + DCT - 1) / DCT);
    const size_t seq = (size_t)s * cap;
    // A chunk is 16 consecutive token rows of kv_heads x 256 bytes (contiguous
    // in the cache), copied as 16-byte pieces: piece x is (token x / (16 kv),
    // kv head (x / 16) % kv, 16-byte column x % 16).
    const int pieces = kv_heads * DCT * 16;
    auto issue = [&](int c, int stg) {
        const uint32_t base = ring_s + stg * stage_bytes;
        const uint16_t* src0 = kc + (seq + (size_t)c * DCT) * kv_heads * kHeadDim;
        for (int x = threadIdx.x; x < pieces; x += DQ * 32) {
            const int rw = (x >> 4) / kv_heads, kvh = (x >> 4) - rw * kv_heads, ch = x & 15;
            const bool ok = (int64_t)c * DCT + rw <= i_last;
            cp_async16_zfill(base + kvh * DCT * 256 + swz256(rw, ch), ok ? src0 + (size_t)x * 8 : kc, ok);
        }
    };

    // S^T of chunk c in stage stg: rows = tokens gq, gq + 8; columns = heads
    // 8 k + 2 t (+1). G >= 8: n8 tile k belongs to kv head k / (G / 8). G < 8:
    // tile k holds the 8 / G kv heads 8 k / G ..; one mma per kv head, with the
    // other heads' columns of B zeroed (column gq belongs to sub-group gq / G).
    const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kch = lane >> 4;
    auto scores = [&](int stg, float (&sc)[NTQ][4]) {
        const uint32_t base = ring_s + stg * stage_bytes;
#pragma unroll
        for (int k = 0; k < NTQ; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[k][e] = 0.f;
        if constexpr (G >= 8) {
            constexpr int TPG = G / 8;  // tiles per kv head
#pragma unroll
            for (int gg = 0; gg < NTQ / TPG; ++gg)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(base + gg * DCT * 256 + swz256(krow, ks * 2 + kch), a0, a1, a2, a3);
#pragma unroll
                    for (int tt = 0; tt < TPG; ++tt)
                        mma_bf16_16816(sc[gg * TPG + tt], a0, a1, a2, a3, qb[gg * TPG + tt][ks][0],
                                       qb[gg * TPG + tt][ks][1]);
                }
        } else {
            constexpr int GPT = 8 / G;  // kv heads per tile
            const int my_sub = gq / G;
#pragma unroll
            for (int k = 0; k < NTQ; ++k)
#pragma unroll
                for (int sub = 0; sub < GPT; ++sub) {
                    const int gg = k * GPT + sub;
                    if (gg >= kv_heads) break;
                    const bool mine = my_sub == sub;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        uint32_t a0, a1, a2, a3;
                        ldmatrix_x4(base + gg * DCT * 256 + swz256(krow, ks * 2 + kch), a0, a1, a2, a3);
                        mma_bf16_16816(sc[k], a0, a1, a2, a3, mine ? qb[k][ks][0] : 0u, mine ? qb[k][ks][1] : 0u);
                    }
                }
        }
    };

    // Sweep 1: online max / sum per column (log2 domain).
    float m[NTQ][2], l[NTQ][2];
#pragma unroll
    for (int k = 0; k < NTQ; ++k)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            m[k][e] = -INFINITY;
            l[k][e] = 0.f;
        }
    issue(0, 0);
    cp_async_commit();
    for (int c = 0; c < n1; ++c) {
        if (c + 1 < n1) issue(c + 1, (c + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float sc[NTQ][4];
        scores(c & 1, sc);
        const int64_t t0 = (int64_t)c * DCT + gq, t1 = t0 + 8;
        // Lane-local running sums (merged over the 8 lanes of a column after
        // the sweep). The reference maximum is raised only when a logit exceeds
        // it by more than 8 (log2 units), so terms stay below 2^8 and most
        // chunks take one exponential per logit and no rescaling.
#pragma unroll
        for (int k = 0; k < NTQ; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool hv = 8 * k + 2 * t + e < q_heads;
                const float x0 = (hv && t0 <= i) ? sc[k][e] * scale_log2 : -INFINITY;
                const float x1 = (hv && t1 <= i) ? sc[k][2 + e] * scale_log2 : -INFINITY;
                const float mx = fmaxf(x0, x1);
                if (mx > m[k][e] + 8.f) {
                    l[k][e] *= ex2_approx(m[k][e] - mx);  // (0 while m is -inf)
                    m[k][e] = mx;
                }
                if (mx != -INFINITY) l[k][e] += ex2_approx(x0 - m[k][e]) + ex2_approx(x1 - m[k][e]);
            }
        __syncthreads();  // the stage is refilled next iteration
    }
    cp_async_wait<0>();
    // lse per column (log2 domain): merge the 8 lanes that share t.
    float lse2[NTQ][2];
#pragma unroll
    for (int k = 0; k < NTQ; ++k)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mc = m[k][e];
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 4));
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 8));
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 16));
            float sum = m[k][e] == -INFINITY ? 0.f : l[k][e] * ex2_approx(m[k][e] - mc);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            sum += __shfl_xor_sync(0xffffffffu, sum, 8);
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
            lse2[k][e] = mc + log2f(sum);
        }

    // Sweep 2: head-averaged probabilities, block maxima, their sum.
    float* trow = target + ((size_t)s * nq + (size_t)(live ? j : j0)) * ld;
    const float inv_h = 1.f / (float)q_heads;
    float mass = 0.f;
    __syncthreads();
    if (n2 > 0) issue(0, 0);
    cp_async_commit();
    for (int c = 0; c < n2; ++c) {
        if (c + 1 < n2) issue(c + 1, (c + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float sc[NTQ][4];
        scores(c & 1, sc);
        float a0 = 0.f, a1 = 0.f;  // rows gq, gq + 8: sum over this lane's heads
#pragma unroll
        for (int k = 0; k < NTQ; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (8 * k + 2 * t + e >= q_heads) continue;
                a0 += ex2_approx(sc[k][e] * scale_log2 - lse2[k][e]);
                a1 += ex2_approx(sc[k][2 + e] * scale_log2 - lse2[k][e]);
            }
        a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
        a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
        a0 *= inv_h;
        a1 *= inv_h;
        // Block maxima: rows of one block are consecutive tokens, i.e. lanes
        // whose gq differ in the low log2(r) bits (and, for r = 16, both rows).
        const int rb = r < 8 ? r : 8;  // rows of a block among the 8 lanes gq
        for (int o = 4; o < 4 * rb; o <<= 1) {
            a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, o));
            a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, o));
        }
        if (r == 16) a0 = a1 = fmaxf(a0, a1);
        if (t == 0 && gq % rb == 0 && live) {
            const int64_t b0 = ((int64_t)c * DCT + gq) / r, b1 = ((int64_t)c * DCT + gq + 8) / r;
            if (b0 < n_vis) {
                trow[b0] = a0;
                mass += a0;
            }
            if (r < 16 && b1 < n_vis) {
                trow[b1] = a1;
                mass += a1;
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    if (!live) return;
    mass = warp_sum(mass);
    __syncwarp();
    const float inv = mass > 0.f ? 1.f / mass : 0.f;
    for (int64_t b = lane; b < ld; b += 32) trow[b] = b < n_vis ? trow[b] * inv : 0.f;
}

constexpr int KT = 256;  // threads per KL row

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
    for (int w = 1; w < KT / 32; ++w) v = is_max ? fmaxf(v, red[w]) : v + red[w];
    return v;
}

__global__ void __launch_bounds__(KT) distill_kl_kernel(int64_t q_begin, int64_t nq, const float* __restrict__ target,
                                                         const float* __restrict__ scores, int64_t ld, int r,
                                                         float* __restrict__ kl, float* __restrict__ dscores) {
    __shared__ float red[KT / 32];
    const int64_t row = blockIdx.x;  // s * nq + j
    const int64_t i = q_begin + row % nq;
    const int64_t n = i / r;
    const float* tr = target + (size_t)row * ld;
    const float* sr = scores + (size_t)row * ld;
    float* dr = dscores ? dscores + (size_t)row * ld : nullptr;
    float mx = -INFINITY;
    for (int64_t b = threadIdx.x; b < n; b += KT) mx = fmaxf(mx, sr[b]);
    mx = block_reduce(mx, red, true);
    float den = 0.f, tsum = 0.f, cross = 0.f, ent = 0.f;
    for (int64_t b = threadIdx.x; b < n; b += KT) {
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
        for (int64_t b = threadIdx.x; b < ld; b += KT) dr[b] = b < n ? tsum * expf(sr[b] - mx) * inv - tr[b] : 0.f;
    }
}

template <int NTQ, int G>
cudaError_t launch_target_t(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                            const uint16_t* kc, int64_t cap, float* target, int64_t ld, cudaStream_t st) {
    auto kern = distill_target_kernel<NTQ, G>;
    const int smem = 2 * L.kv_heads * DCT * 256;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const dim3 grid((unsigned)((nq + DQ - 1) / DQ), (unsigned)batch);
    note_launch();
    kern<<<grid, DQ * 32, smem, st>>>(q, q_begin, nq, kc, cap, target, ld, L.q_heads, L.kv_heads, L.r,
                                      L.sm_scale * LOG2E_D);
    return cudaGetLastError();
}

}  // namespace

bool distill_target_supported(const LayerDims& L) {
    const int G = L.q_heads / L.kv_heads;
    const bool groups_tile = G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
    return L.q_heads <= 32 && groups_tile && (L.r == 1 || L.r == 2 || L.r == 4 || L.r == 8 || L.r == 16);
}

cudaError_t launch_distill_target(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                  const uint16_t* kc, int64_t cap, float* target, int64_t ld, cudaStream_t st) {
    if (batch <= 0 || nq <= 0) return cudaSuccess;
    const int G = L.q_heads / L.kv_heads;
#define QSA_TGT(NTQ_, G_) \
    if ((L.q_heads + 7) / 8 == NTQ_ && G == G_) return launch_target_t<NTQ_, G_>(L, batch, q, q_begin, nq, kc, cap, target, ld, st)
    // The (tiles, G) pairs that kv_heads <= 8 allows.
    QSA_TGT(1, 1);
    QSA_TGT(1, 2);
    QSA_TGT(1, 4);
    QSA_TGT(1, 8);
    QSA_TGT(2, 2);
    QSA_TGT(2, 4);
    QSA_TGT(2, 8);
    QSA_TGT(2, 16);
    QSA_TGT(3, 4);
    QSA_TGT(3, 8);
    QSA_TGT(4, 4);
    QSA_TGT(4, 8);
    QSA_TGT(4, 16);
#undef QSA_TGT
    return cudaErrorInvalidValue;
}

cudaError_t launch_distill_kl(const LayerDims& L, int batch, int64_t q_begin, int64_t nq, const float* target,
                              const float* scores, int64_t ld, float* kl, float* dscores, cudaStream_t st) {
    if (batch <= 0 || nq <= 0) return cudaSuccess;
    note_launch();
    distill_kl_kernel<<<(unsigned)(batch * nq), KT, 0, st>>>(q_begin, nq, target, scores, ld, L.r, kl, dscores);
    return cudaGetLastError();
}

}  // namespace qsa
