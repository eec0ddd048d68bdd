// a6 + a7: expansion of the selected blocks (plus the current tail) and the
// sparse core attention over those tokens ("QSA (Qwen Sparse Attention)"
// concept page, (B) sparse core attention; "Qwen Sparse Attention" gallery
// page: attention_input = flatten(selected_blocks) + current_incomplete_block).
//
// The stage is a gather: per query and kv head, ~2K random 256-byte key and
// value rows feed 8 query heads (8 flop per byte), so it is bound by memory,
// not by the tensor pipe. One warp owns one (query, kv head) pair (or a slice
// of its units): the G = q_heads/kv_heads query heads are the rows of an
// m16n8k16 tile (padded to 16), tokens stream through a 3-stage cp.async ring
// of 16-token chunks in row-swizzled shared memory, logits/softmax/accumulation
// are fp32 with an online (running max) softmax, and probabilities are rounded
// to bf16 for the P.V product. Invalid selections are skipped, never read.
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int WARPS = 4;
constexpr int CT = 16;                    // tokens per chunk
constexpr int STAGES = 3;
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

struct WarpState {
    float o[16][4];
    float m[2], l[2];
};

__device__ __forceinline__ void warp_attend(const Work& w, uint8_t* wsm, int lane, WarpState& st) {
    uint16_t* ring = reinterpret_cast<uint16_t*>(wsm);
    int64_t* tok = reinterpret_cast<int64_t*>(wsm + STAGES * STAGE_BYTES);  // [STAGES][CT]
    uint32_t* vmask = reinterpret_cast<uint32_t*>(wsm + STAGES * STAGE_BYTES + STAGES * CT * 8);
    const uint32_t ring_s = smem_u32(ring);
    const int gq = lane >> 2, tig = lane & 3;

    // Query fragments (A operand, rows = query heads of the group).
    uint32_t qa[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
                const int row = gq + hf * 8;
                const int col = ks * 16 + kh * 8 + 2 * tig;
                uint32_t v = 0;
                if (row < w.G) v = *reinterpret_cast<const uint32_t*>(w.q + row * kHeadDim + col);
                qa[ks][kh * 2 + hf] = v;
            }
        }
    }
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[nd][e] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;

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
            int64_t t = -1;
            if (p < ntok) {
                const int e = (int)(p % w.r);
                if (u < w.nsel) {
                    const int32_t b = u - w.u0 < 32 ? b_pre : w.sel[u];
                    if (b >= 0 && (int64_t)b < cur) t = (int64_t)b * w.r + e;
                } else {
                    const int64_t tt = cur * w.r + e;
                    if (tt <= w.i) t = tt;
                }
            }
            if (lane < CT) tok[stg * CT + lane] = t;
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
            const int64_t t = tok[stg * CT + row];
            const bool ok = t >= 0;
            const size_t off = (size_t)(ok ? t : 0) * row_stride + (size_t)w.g * kHeadDim + ch * 8;
            cp_async16_zfill(kbase + swz256(row, ch), w.kc + off, ok);
            cp_async16_zfill(vbase + swz256(row, ch), w.vc + off, ok);
        }
    };

#pragma unroll
    for (int c = 0; c < STAGES - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        if (c + STAGES - 1 < nchunks) issue(c + STAGES - 1);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const int stg = c % STAGES;
        const uint32_t kbase = ring_s + stg * STAGE_BYTES;
        const uint32_t vbase = kbase + CT * 256;
        const uint32_t valid = vmask[stg];

        // S = Q K^T over 16 tokens (two n8 tiles).
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t b00, b01, b10, b11;
            const int nrow = (lane & 7) + ((lane >> 4) & 1) * 8;
            const int ch = ks * 2 + ((lane >> 3) & 1);
            ldmatrix_x4(kbase + swz256(nrow, ch), b00, b01, b10, b11);
            mma_bf16_16816(s[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
            mma_bf16_16816(s[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10, b11);
        }
        // Online softmax (log2 domain), rows gq (hf=0) and gq+8 (hf=1).
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + 2 * tig + e;
                    float v = s[nt][hf * 2 + e] * w.scale_log2;
                    v = ((valid >> col) & 1u) ? v : -INFINITY;
                    s[nt][hf * 2 + e] = v;
                    mx = fmaxf(mx, v);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(st.m[hf], mx);
            const float corr = (m_new == -INFINITY) ? 1.f : exp2f(st.m[hf] - m_new);
            float psum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float v = s[nt][hf * 2 + e];
                    const float p = (v == -INFINITY) ? 0.f : exp2f(v - m_new);
                    s[nt][hf * 2 + e] = p;
                    psum += p;
                }
            st.l[hf] = st.l[hf] * corr + psum;
            st.m[hf] = m_new;
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                st.o[nd][hf * 2] *= corr;
                st.o[nd][hf * 2 + 1] *= corr;
            }
        }
        // O += P V (P rounded to bf16).
        const uint32_t pa0 = pack_bf16x2(s[0][0], s[0][1]);
        const uint32_t pa1 = pack_bf16x2(s[0][2], s[0][3]);
        const uint32_t pa2 = pack_bf16x2(s[1][0], s[1][1]);
        const uint32_t pa3 = pack_bf16x2(s[1][2], s[1][3]);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            uint32_t b0, b1, b2, b3;
            const int trow = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int ch = np * 2 + (lane >> 4);
            ldmatrix_x4_trans(vbase + swz256(trow, ch), b0, b1, b2, b3);
            mma_bf16_16816(st.o[2 * np], pa0, pa1, pa2, pa3, b0, b1);
            mma_bf16_16816(st.o[2 * np + 1], pa0, pa1, pa2, pa3, b2, b3);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // Full row sums across the quad.
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        st.l[hf] += __shfl_xor_sync(0xffffffffu, st.l[hf], 1);
        st.l[hf] += __shfl_xor_sync(0xffffffffu, st.l[hf], 2);
    }
}

// Merge state `b` into `a` (same rows).
__device__ __forceinline__ void merge_state(WarpState& a, const float* bo, const float* bm,
                                            const float* bl) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const float m = fmaxf(a.m[hf], bm[hf]);
        const float ca = (m == -INFINITY) ? 0.f : exp2f(a.m[hf] - m);
        const float cb = (m == -INFINITY) ? 0.f : exp2f(bm[hf] - m);
        a.l[hf] = a.l[hf] * ca + bl[hf] * cb;
        a.m[hf] = m;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            a.o[nd][hf * 2] = a.o[nd][hf * 2] * ca + bo[nd * 4 + hf * 2] * cb;
            a.o[nd][hf * 2 + 1] = a.o[nd][hf * 2 + 1] * ca + bo[nd * 4 + hf * 2 + 1] * cb;
        }
    }
}

__device__ __forceinline__ void write_out(const WarpState& st, int G, uint16_t* out_rows,
                                          float* lse_rows, int lane) {
    const int gq = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int row = gq + hf * 8;
        if (row >= G) continue;
        const float inv = st.l[hf] > 0.f ? 1.f / st.l[hf] : 0.f;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            const uint32_t v = pack_bf16x2(st.o[nd][hf * 2] * inv, st.o[nd][hf * 2 + 1] * inv);
            *reinterpret_cast<uint32_t*>(out_rows + row * kHeadDim + nd * 8 + 2 * tig) = v;
        }
        if (lse_rows && tig == 0)
            lse_rows[row] = st.l[hf] > 0.f ? (st.m[hf] + log2f(st.l[hf])) * LN2 : -INFINITY;
    }
}

// Prefill: CTA = one query; warp w -> kv head kv0 + (w % GH), unit split w / GH.
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
    WarpState st;
    warp_attend(w, wsm, lane, st);

    if (NS > 1) {
        // Splits > 0 park their state in their own smem; split 0 merges.
        float* park = reinterpret_cast<float*>(wsm);
        __syncthreads();
        if (split > 0) {
#pragma unroll
            for (int nd = 0; nd < 16; ++nd)
#pragma unroll
                for (int e = 0; e < 4; ++e) park[(nd * 4 + e) * 32 + lane] = st.o[nd][e];
            park[64 * 32 + lane] = st.m[0];
            park[65 * 32 + lane] = st.m[1];
            park[66 * 32 + lane] = st.l[0];
            park[67 * 32 + lane] = st.l[1];
        }
        __syncthreads();
        if (split == 0) {
            for (int sp = 1; sp < NS; ++sp) {
                const float* src = reinterpret_cast<const float*>(smem + (warp + sp * GH) * WARP_SMEM);
                float bo[64], bm[2], bl[2];
#pragma unroll
                for (int k = 0; k < 64; ++k) bo[k] = src[k * 32 + lane];
                bm[0] = src[64 * 32 + lane];
                bm[1] = src[65 * 32 + lane];
                bl[0] = src[66 * 32 + lane];
                bl[1] = src[67 * 32 + lane];
                merge_state(st, bo, bm, bl);
            }
        }
    }
    if (split == 0)
        write_out(st, G, out + ((size_t)row * q_heads + (size_t)g * G) * kHeadDim,
                  lse ? lse + (size_t)row * q_heads + (size_t)g * G : nullptr, lane);
}

// Decode: one warp per (sequence, kv head, split); partial states to `part`
// laid out [batch][q_heads][S][132] = (o[128], m, l, pad, pad), log2 domain.
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
    WarpState st;
    warp_attend(w, smem + warp * WARP_SMEM, lane, st);
    const int gq = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int row = gq + hf * 8;
        if (row >= G) continue;
        float* d = dst + (size_t)row * S * 132;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            d[nd * 8 + 2 * tig] = st.o[nd][hf * 2];
            d[nd * 8 + 2 * tig + 1] = st.o[nd][hf * 2 + 1];
        }
        if (tig == 0) {
            d[128] = st.m[hf];
            d[129] = st.l[hf];
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
    cudaFuncSetAttribute(prefill_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SMEM);
    const int GH = L.kv_heads < WARPS ? L.kv_heads : WARPS;
    dim3 grid((unsigned)nq, (unsigned)batch, (unsigned)(L.kv_heads / GH));
    note_launch();
    prefill_attention_kernel<<<grid, WARPS * 32, SMEM, st>>>(
        q, q_begin, nq, kc, vc, cap, sel, nsel, out, lse, L.q_heads, L.kv_heads, L.r, L.kB,
        L.sm_scale * LOG2E);
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
    cudaFuncSetAttribute(decode_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SMEM);
    const int S = decode_attention_splits(L);
    const int64_t items = (int64_t)batch * L.kv_heads * S;
    note_launch();
    cudaError_t e = launch_pdl(decode_attention_kernel, dim3((unsigned)((items + WARPS - 1) / WARPS)),
                               dim3(WARPS * 32), (size_t)SMEM, st, q, pos, kc, vc, cap, sel, nsel, part, batch,
                               L.q_heads, L.kv_heads, L.r, L.kB, S, L.sm_scale * LOG2E);
    if (e != cudaSuccess) return e;
    const int rows = batch * L.q_heads;
    note_launch();
    return launch_pdl(decode_combine_kernel, dim3((unsigned)rows), dim3(128), 0, st, (const float*)part, S, out);
}

}  // namespace qsa
