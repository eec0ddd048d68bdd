// a6 + a7: expansion of the selected blocks (plus the current tail) and the
// sparse core attention over those tokens ("QSA (Qwen Sparse Attention)"
// concept page, (B) sparse core attention; "Qwen Sparse Attention" gallery
// page: attention_input = flatten(selected_blocks) + current_incomplete_block).
//
// The stage is a gather: per query and kv head, ~2K random 256-byte key and
// value rows feed G = q_heads/kv_heads query heads (8 flop per byte). One warp
// owns one (query, kv head) pair (or a slice of its units); tokens stream
// through a 2-stage cp.async ring of 16-token chunks in row-swizzled shared
// memory (two stages leave room for three 4-warp CTAs per SM, which hides the
// gather latency better than a deeper ring). The tiles are transposed so that
// no row is padding: in S^T = K Q^T the 16 tokens of a chunk are the m16 rows
// and the query heads the n8 columns (one n8 tile per 8 heads), and in
// O^T += V^T P^T the 128 dims are eight m16 tiles and the heads again the
// columns; the probabilities move from the S^T accumulator to the P^T operand
// with one movmatrix transpose per 8x8 block. Logits, the online (running max) softmax and the
// accumulation are fp32; probabilities are rounded to bf16 for the P.V
// product. Invalid selections are skipped, never read.
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int WARPS = 4;
constexpr int CT = 16;                    // tokens per chunk
constexpr int STAGES = 2;
constexpr int STAGE_BYTES = CT * 256 * 2; // K and V rows
constexpr int WARP_SMEM = STAGES * STAGE_BYTES + STAGES * CT * 8 + 64;
constexpr int SMEM = WARPS * WARP_SMEM;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct Work {
    const uint16_t* q;     // first query head of the group: [G][128]
    const uint16_t* kc;    // sequence base of k_cache
    const uint16_t* vc;
    const int32_t* sel;    // selection row
    int64_t i;             // query position
    int nsel;              // valid count (clamped)
    int u0, u1;            // unit range, units [0, nsel) = selected blocks, nsel = tail
    int g;                 // kv head
    int G;                 // query heads per kv head
    int kv_heads;
    int r;
    float scale_log2;      // sm_scale * log2(e)
};

// Per-warp attention state for NT tiles of 8 query heads. Lane (g, t) =
// (lane / 4, lane % 4) holds, for head h = 8 nt + 2 t + e (e = 0, 1):
// o[nt][i][e] and o[nt][i][2 + e] = unnormalised output dims 16 i + g and
// 16 i + g + 8; m[nt][e] = running maximum (log2 domain), l[nt][e] = sum of
// probabilities (after warp_attend: over the whole warp).
template <int NT>
struct WarpState {
    float o[NT][8][4];
    float m[NT][2], l[NT][2];
};
template <int NT>
constexpr int park_floats() {
    return NT * 36;  // o (32), m (2), l (2) per n8 tile
}

// 8x8 b16 matrix transpose in the mma fragment layout (lane l holds row l/4,
// columns 2 (l % 4) and 2 (l % 4) + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
    return d;
}

template <int NT>
__device__ __forceinline__ void warp_attend(const Work& w, uint8_t* wsm, int lane, WarpState<NT>& st) {
    uint16_t* ring = reinterpret_cast<uint16_t*>(wsm);
    int64_t* tok = reinterpret_cast<int64_t*>(wsm + STAGES * STAGE_BYTES);  // [STAGES][CT]
    uint32_t* vmask = reinterpret_cast<uint32_t*>(wsm + STAGES * STAGE_BYTES + STAGES * CT * 8);
    const uint32_t ring_s = smem_u32(ring);
    const int g = lane >> 2, t = lane & 3;

    // Query fragments (B operand of S^T = K Q^T): column = head 8 nt + g,
    // k rows = dims 16 ks + 2 t (+1) and 16 ks + 8 + 2 t (+1).
    uint32_t qb[NT][8][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = 8 * nt + g;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[nt][ks][0] = h < w.G ? *reinterpret_cast<const uint32_t*>(w.q + h * kHeadDim + ks * 16 + 2 * t) : 0u;
            qb[nt][ks][1] = h < w.G ? *reinterpret_cast<const uint32_t*>(w.q + h * kHeadDim + ks * 16 + 8 + 2 * t) : 0u;
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) st.o[nt][i][e] = 0.f;
        st.m[nt][0] = st.m[nt][1] = -INFINITY;
        st.l[nt][0] = st.l[nt][1] = 0.f;
    }

    const int64_t ntok = (int64_t)(w.u1 - w.u0) * w.r;
    const int nchunks = (int)((ntok + CT - 1) / CT);
    const int64_t cur = w.i / w.r;
    const int64_t row_stride = (int64_t)w.kv_heads * kHeadDim;
    // The warp's first 32 selection entries in one round trip (lane u holds
    // unit u0 + u); later units, if any, are read when their chunk is issued.
    const int32_t sel_lane = (w.u0 + lane < w.u1 && w.u0 + lane < w.nsel) ? w.sel[w.u0 + lane] : -1;

    auto issue = [&](int c) {
        const int stg = c % STAGES;
        {
            const int64_t p = (int64_t)c * CT + (lane & (CT - 1));  // lanes >= CT mirror lanes < CT
            const int u = w.u0 + (int)(p / w.r);
            const int32_t b_pre = __shfl_sync(0xffffffffu, sel_lane, (u - w.u0) & 31);
            int64_t tk = -1;
            if (p < ntok) {
                const int e = (int)(p % w.r);
                if (u < w.nsel) {
                    const int32_t b = u - w.u0 < 32 ? b_pre : w.sel[u];
                    if (b >= 0 && (int64_t)b < cur) tk = (int64_t)b * w.r + e;
                } else {
                    const int64_t tt = cur * w.r + e;
                    if (tt <= w.i) tk = tt;
                }
            }
            if (lane < CT) tok[stg * CT + lane] = tk;
        }
        __syncwarp();
        if (lane == 0) {
            uint32_t m = 0;
            for (int k = 0; k < CT; ++k) m |= (tok[stg * CT + k] >= 0 ? 1u : 0u) << k;
            vmask[stg] = m;
        }
        const uint32_t kbase = ring_s + stg * STAGE_BYTES;
        const uint32_t vbase = kbase + CT * 256;
#pragma unroll
        for (int k = 0; k < (CT * 16) / 32; ++k) {
            const int idx = lane + k * 32;
            const int row = idx >> 4, ch = idx & 15;
            const int64_t tk = tok[stg * CT + row];
            const bool ok = tk >= 0;
            const size_t off = (size_t)(ok ? tk : 0) * row_stride + (size_t)w.g * kHeadDim + ch * 8;
            cp_async16_zfill(kbase + swz256(row, ch), w.kc + off, ok);
            cp_async16_zfill(vbase + swz256(row, ch), w.vc + off, ok);
        }
    };

#pragma unroll
    for (int c = 0; c < STAGES - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    // ldmatrix row addresses: K as the A operand (token rows, dims in chunk
    // pairs), V^T as the A operand (transposed 8x8 loads of token rows).
    const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kch = lane >> 4;
    const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8, vch = (lane >> 3) & 1;
    for (int c = 0; c < nchunks; ++c) {
        if (c + STAGES - 1 < nchunks) issue(c + STAGES - 1);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const int stg = c % STAGES;
        const uint32_t kbase = ring_s + stg * STAGE_BYTES;
        const uint32_t vbase = kbase + CT * 256;
        const uint32_t valid = vmask[stg];

        // S^T = K Q^T: rows = tokens g, g + 8; columns = heads 8 nt + 2 t (+1).
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(kbase + swz256(krow, ks * 2 + kch), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
        // Online softmax per head (log2 domain); a head's 16 tokens sit in the
        // 8 lanes with the same t.
        const bool v0 = (valid >> g) & 1u, v1 = (valid >> (g + 8)) & 1u;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float x0 = v0 ? s[nt][e] * w.scale_log2 : -INFINITY;
                const float x1 = v1 ? s[nt][2 + e] * w.scale_log2 : -INFINITY;
                float mx = fmaxf(x0, x1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(st.m[nt][e], mx);
                const float corr = (m_new == -INFINITY) ? 1.f : exp2f(st.m[nt][e] - m_new);
                const float p0 = (x0 == -INFINITY) ? 0.f : exp2f(x0 - m_new);
                const float p1 = (x1 == -INFINITY) ? 0.f : exp2f(x1 - m_new);
                st.l[nt][e] = st.l[nt][e] * corr + (p0 + p1);
                st.m[nt][e] = m_new;
                s[nt][e] = p0;
                s[nt][2 + e] = p1;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    st.o[nt][i][e] *= corr;
                    st.o[nt][i][2 + e] *= corr;
                }
            }
            // P^T operand: the two 8x8 blocks (tokens 0-7, 8-15) of this tile,
            // rounded to bf16 and transposed.
            pb[nt][0] = movmatrix_trans(pack_bf16x2(s[nt][0], s[nt][1]));
            pb[nt][1] = movmatrix_trans(pack_bf16x2(s[nt][2], s[nt][3]));
        }
        // O^T += V^T P^T: rows = dims 16 i + g (+8), columns = heads.
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(vbase + swz256(vrow, 2 * i + vch), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(st.o[nt][i], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // Full sums over the 16-token rows (the 8 lanes with the same t).
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            st.l[nt][e] += __shfl_xor_sync(0xffffffffu, st.l[nt][e], 4);
            st.l[nt][e] += __shfl_xor_sync(0xffffffffu, st.l[nt][e], 8);
            st.l[nt][e] += __shfl_xor_sync(0xffffffffu, st.l[nt][e], 16);
        }
}

// Parks a state in the lane-strided layout: slot k of lane l at k * 32 + l.
template <int NT>
__device__ __forceinline__ void park_state(const WarpState<NT>& st, float* dst, int lane) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[(nt * 36 + i * 4 + e) * 32 + lane] = st.o[nt][i][e];
        dst[(nt * 36 + 32) * 32 + lane] = st.m[nt][0];
        dst[(nt * 36 + 33) * 32 + lane] = st.m[nt][1];
        dst[(nt * 36 + 34) * 32 + lane] = st.l[nt][0];
        dst[(nt * 36 + 35) * 32 + lane] = st.l[nt][1];
    }
}

// Merges a parked state (same lanes, same heads) into `a`.
template <int NT>
__device__ __forceinline__ void merge_parked(WarpState<NT>& a, const float* src, int lane) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float bm = src[(nt * 36 + 32 + e) * 32 + lane];
            const float bl = src[(nt * 36 + 34 + e) * 32 + lane];
            const float m = fmaxf(a.m[nt][e], bm);
            const float ca = (m == -INFINITY) ? 0.f : exp2f(a.m[nt][e] - m);
            const float cb = (m == -INFINITY) ? 0.f : exp2f(bm - m);
            a.l[nt][e] = a.l[nt][e] * ca + bl * cb;
            a.m[nt][e] = m;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                a.o[nt][i][e] = a.o[nt][i][e] * ca + src[(nt * 36 + i * 4 + e) * 32 + lane] * cb;
                a.o[nt][i][2 + e] = a.o[nt][i][2 + e] * ca + src[(nt * 36 + i * 4 + 2 + e) * 32 + lane] * cb;
            }
        }
    }
}

// Writes the G normalised output rows (bf16) and, if asked, their LSE.
template <int NT>
__device__ __forceinline__ void write_out(const WarpState<NT>& st, int G, uint16_t* out_rows, float* lse_rows,
                                          int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nt + 2 * t + e;
            if (h >= G) continue;
            const float inv = st.l[nt][e] > 0.f ? 1.f / st.l[nt][e] : 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                out_rows[h * kHeadDim + 16 * i + g] = f32_to_bf16(st.o[nt][i][e] * inv);
                out_rows[h * kHeadDim + 16 * i + g + 8] = f32_to_bf16(st.o[nt][i][2 + e] * inv);
            }
            if (lse_rows && g == 0)
                lse_rows[h] = st.l[nt][e] > 0.f ? (st.m[nt][e] + log2f(st.l[nt][e])) * LN2 : -INFINITY;
        }
}

// Prefill: CTA = one query; warp w -> kv head kv0 + (w % GH), unit split w / GH.
template <int NT>
__global__ void __launch_bounds__(WARPS * 32) prefill_attention_kernel(
    const uint16_t* __restrict__ q, int64_t q_begin, int64_t nq, const uint16_t* __restrict__ kc,
    const uint16_t* __restrict__ vc, int64_t cap, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ nsel, uint16_t* __restrict__ out, float* __restrict__ lse,
    int q_heads, int kv_heads, int r, int kB, float scale_log2) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t j = blockIdx.x;
    const int s = blockIdx.y;
    const int GH = kv_heads < WARPS ? kv_heads : WARPS;  // kv heads per CTA
    const int NS = WARPS / GH;                            // unit splits per kv head
    const int g = blockIdx.z * GH + warp % GH;
    const int split = warp / GH;
    const int G = q_heads / kv_heads;
    const int64_t row = (int64_t)s * nq + j;
    const int64_t i = q_begin + j;

    int ns = nsel[row];
    ns = ns < 0 ? 0 : (ns > kB ? kB : ns);
    const int units = ns + 1;
    Work w;
    w.q = q + ((size_t)row * q_heads + (size_t)g * G) * kHeadDim;
    w.kc = kc + (size_t)s * cap * kv_heads * kHeadDim;
    w.vc = vc + (size_t)s * cap * kv_heads * kHeadDim;
    w.sel = sel + (size_t)row * kB;
    w.i = i;
    w.nsel = ns;
    w.u0 = (int)((int64_t)units * split / NS);
    w.u1 = (int)((int64_t)units * (split + 1) / NS);
    w.g = g;
    w.G = G;
    w.kv_heads = kv_heads;
    w.r = r;
    w.scale_log2 = scale_log2;

    uint8_t* wsm = smem + warp * WARP_SMEM;
    WarpState<NT> st;
    warp_attend<NT>(w, wsm, lane, st);

    if (NS > 1) {
        // Splits > 0 park their state in their own smem; split 0 merges.
        __syncthreads();
        if (split > 0) park_state<NT>(st, reinterpret_cast<float*>(wsm), lane);
        __syncthreads();
        if (split == 0)
            for (int sp = 1; sp < NS; ++sp)
                merge_parked<NT>(st, reinterpret_cast<const float*>(smem + (warp + sp * GH) * WARP_SMEM), lane);
    }
    if (split == 0)
        write_out<NT>(st, G, out + ((size_t)row * q_heads + (size_t)g * G) * kHeadDim,
                      lse ? lse + (size_t)row * q_heads + (size_t)g * G : nullptr, lane);
}

// Decode: one warp per (sequence, kv head, split); partial states to `part`
// laid out [batch][q_heads][S][132] = (o[128], m, l, pad, pad), log2 domain.
template <int NT>
__global__ void __launch_bounds__(WARPS * 32) decode_attention_kernel(
    const uint16_t* __restrict__ q, const int64_t* __restrict__ pos,
    const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc, int64_t cap,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel, float* __restrict__ part,
    int batch, int q_heads, int kv_heads, int r, int kB, int S, float scale_log2) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t item = (int64_t)blockIdx.x * WARPS + warp;
    if (item >= (int64_t)batch * kv_heads * S) return;
    const int split = (int)(item % S);
    const int g = (int)((item / S) % kv_heads);
    const int s = (int)(item / ((int64_t)S * kv_heads));
    const int G = q_heads / kv_heads;
    const int64_t p = pos[s];
    float* dst = part + (((size_t)s * q_heads + (size_t)g * G) * S + split) * 132;
    if (p < 0 || p >= cap) {
        // Skipped sequence: an empty partial (m = -inf, l = 0).
        for (int row = 0; row < G; ++row) {
            float* d = dst + (size_t)row * S * 132;
            for (int k = lane; k < 132; k += 32) d[k] = k == 128 ? -INFINITY : 0.f;
        }
        return;
    }
    int ns = nsel[s];
    ns = ns < 0 ? 0 : (ns > kB ? kB : ns);
    const int units = ns + 1;
    Work w;
    w.q = q + ((size_t)s * q_heads + (size_t)g * G) * kHeadDim;
    w.kc = kc + (size_t)s * cap * kv_heads * kHeadDim;
    w.vc = vc + (size_t)s * cap * kv_heads * kHeadDim;
    w.sel = sel + (size_t)s * kB;
    w.i = p;
    w.nsel = ns;
    w.u0 = (int)((int64_t)units * split / S);
    w.u1 = (int)((int64_t)units * (split + 1) / S);
    w.g = g;
    w.G = G;
    w.kv_heads = kv_heads;
    w.r = r;
    w.scale_log2 = scale_log2;
    WarpState<NT> st;
    warp_attend<NT>(w, smem + warp * WARP_SMEM, lane, st);
    const int gq = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nt + 2 * t + e;
            if (h >= G) continue;
            float* d = dst + (size_t)h * S * 132;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                d[16 * i + gq] = st.o[nt][i][e];
                d[16 * i + gq + 8] = st.o[nt][i][2 + e];
            }
            if (gq == 0) {
                d[128] = st.m[nt][e];
                d[129] = st.l[nt][e];
            }
        }
}

// Combine the S partials of each (sequence, head): one CTA of 4 warps per
// head; every warp finds the partials' maximum itself (two loads per lane),
// warp w sums partials w, w + 4, ... for all 128 dims (lane: dims lane + 32 j),
// with every load of the warp issued before the first use, and the four warp
// sums meet in shared memory.
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part, int S,
                                                            uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    __shared__ float so[4][128];
    __shared__ float sl[4];
    const int row = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float* src = part + (size_t)row * S * 132;
    float m = -INFINITY;
    for (int k = lane; k < S; k += 32) m = fmaxf(m, src[(size_t)k * 132 + 128]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, l = 0.f;
#pragma unroll 4
    for (int k = w; k < S; k += 4) {
        const float* pk = src + (size_t)k * 132;
        const float c = (m == -INFINITY) ? 0.f : exp2f(pk[128] - m);
        l = fmaf(pk[129], c, l);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(pk[lane + 32 * j], c, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) so[w][lane + 32 * j] = acc[j];
    if (lane == 0) sl[w] = l;
    __syncthreads();
    const int d = threadIdx.x;
    const float lt = sl[0] + sl[1] + sl[2] + sl[3];
    const float o = so[0][d] + so[1][d] + so[2][d] + so[3][d];
    out[(size_t)row * kHeadDim + d] = f32_to_bf16(lt > 0.f ? o / lt : 0.f);
}

}  // namespace

cudaError_t launch_sparse_attention(const LayerDims& L, int batch, const uint16_t* q,
                                    int64_t q_begin, int64_t nq, const uint16_t* kc,
                                    const uint16_t* vc, int64_t cap, const int32_t* sel,
                                    const int32_t* nsel, uint16_t* out, float* lse,
                                    cudaStream_t st) {
    if (nq <= 0 || batch <= 0) return cudaSuccess;
    const int GH = L.kv_heads < WARPS ? L.kv_heads : WARPS;
    dim3 grid((unsigned)nq, (unsigned)batch, (unsigned)(L.kv_heads / GH));
    const int G = L.q_heads / L.kv_heads;
    auto kern = G > 8 ? prefill_attention_kernel<2> : prefill_attention_kernel<1>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    note_launch();
    kern<<<grid, WARPS * 32, SMEM, st>>>(q, q_begin, nq, kc, vc, cap, sel, nsel, out, lse, L.q_heads, L.kv_heads,
                                         L.r, L.kB, L.sm_scale * LOG2E);
    return cudaGetLastError();
}

int decode_attention_splits(const LayerDims& L) {
    const int units = L.kB + 1;
    int S = (units + 7) / 8;
    return S < 1 ? 1 : (S > 64 ? 64 : S);
}

cudaError_t launch_decode_attention(const LayerDims& L, int batch, const int64_t* pos,
                                    const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                    int64_t cap, const int32_t* sel, const int32_t* nsel,
                                    float* part, uint16_t* out, cudaStream_t st) {
    if (batch <= 0) return cudaSuccess;
    const int G = L.q_heads / L.kv_heads;
    auto kern = G > 8 ? decode_attention_kernel<2> : decode_attention_kernel<1>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    const int S = decode_attention_splits(L);
    const int64_t items = (int64_t)batch * L.kv_heads * S;
    note_launch();
    cudaError_t e = launch_pdl(kern, dim3((unsigned)((items + WARPS - 1) / WARPS)), dim3(WARPS * 32), (size_t)SMEM,
                               st, q, pos, kc, vc, cap, sel, nsel, part, batch, L.q_heads, L.kv_heads, L.r, L.kB,
                               S, L.sm_scale * LOG2E);
    if (e != cudaSuccess) return e;
    const int rows = batch * L.q_heads;
    note_launch();
    return launch_pdl(decode_combine_kernel, dim3((unsigned)rows), dim3(128), 0, st, (const float*)part, S, out);
}

}  // namespace qsa
