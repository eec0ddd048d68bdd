// Gradient of the sparse core attention. The "QSA (Qwen Sparse Attention)"
// concept page ("Native trainability via 2-stage continued pretraining") trains
// the model and the indexer together under the sparse selection in stage 2, so
// the attention over the selected tokens (section (B)) is differentiated:
// for query i, core head h of kv head g, the token set T_i of the forward and
// the upstream gradient dO_h,
//   P_ht  = exp(scale <q_h, k_t> - lse_h)            (lse from the forward)
//   dV_t += sum over the heads h of g of P_ht dO_h
//   dS_ht = P_ht (<dO_h, v_t> - <dO_h, O_h>)
//   dQ_h  = scale sum_t dS_ht k_t,   dK_t += scale sum over g's heads dS_ht q_h.
//
// One warp owns one (query, kv head) pair and streams the same 16-token chunks
// as the forward (2-stage cp.async ring of K and V rows, row-swizzled). Per
// chunk, on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   S^T  = K Q^T and dP^T = V dO^T  (tokens as m16 rows, heads as n8 columns);
//   dQ^T += K^T dS^T                (dims as m16 rows, like O^T in the forward);
//   dV   = P dO and dK = dS Q       (tokens as rows, dims as 16 n8 tiles, heads
//                                    as the k16 dimension: the S^T accumulator
//                                    layout is already the A-operand layout).
// P and dS are rounded to bf16 for the products. dQ rows belong to one warp and
// are written once; dK and dV rows are shared by every query that selected the
// token, so each chunk's tiles are added with 16-byte fp32 vector atomics (the
// order of the additions is not fixed).
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int BW = 4;                            // warps per CTA (kv heads of one query)
constexpr int CT = 16;                           // tokens per chunk
constexpr int STAGES = 2;
constexpr int STAGE_BYTES = CT * 256 * 2;        // K and V rows
constexpr int OPND_BYTES = 16 * kHeadDim * 2;    // Q or dO rows of up to 16 heads (swizzled)
constexpr int WARP_SMEM = STAGES * STAGE_BYTES + 2 * OPND_BYTES + STAGES * CT * 4 + 64;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
    return d;
}

// B fragments (S^T = K X^T) of the G rows of X (Q or dO) in the swizzled
// operand tile: column = head 8 nt + g, k rows = dims 16 ks + 2 t (+1), +8.
template <int NT>
__device__ __forceinline__ void b_frags(const uint8_t* tile, int lane, uint32_t (&b)[NT][8][2]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int h = 8 * nt + g;
            b[nt][ks][0] = *reinterpret_cast<const uint32_t*>(tile + swz256(h, 2 * ks) + 4 * t);
            b[nt][ks][1] = *reinterpret_cast<const uint32_t*>(tile + swz256(h, 2 * ks + 1) + 4 * t);
        }
}

template <int NT>
__global__ void __launch_bounds__(BW * 32) attention_backward_kernel(
    const uint16_t* __restrict__ q, int64_t q_begin, int64_t nq, const uint16_t* __restrict__ kc,
    const uint16_t* __restrict__ vc, int64_t cap, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ nsel, const uint16_t* __restrict__ out, const float* __restrict__ lse,
    const uint16_t* __restrict__ dout, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
    int q_heads, int kv_heads, int r, int kB, float scale) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int64_t j = blockIdx.x;
    const int s = blockIdx.y;
    const int GH = (int)blockDim.x / 32;
    const int g = blockIdx.z * GH + warp;
    const int G = q_heads / kv_heads;
    const int64_t row = (int64_t)s * nq + j;
    const int64_t i = q_begin + j;
    const int64_t cur = i / r;
    const float scale_log2 = scale * LOG2E;

    uint8_t* wsm = smem + warp * WARP_SMEM;
    uint8_t* qtile = wsm + STAGES * STAGE_BYTES;
    uint8_t* gtile = qtile + OPND_BYTES;
    int32_t* toks = reinterpret_cast<int32_t*>(gtile + OPND_BYTES);  // [STAGES][CT]
    float* dsm = reinterpret_cast<float*>(toks + STAGES * CT);        // [16] <dO_h, O_h>

    // Q and dO rows of the group into swizzled tiles (rows >= G zero), and
    // D_h = <dO_h, O_h> in fp32 (from the forward's bf16 output).
    const size_t head0 = ((size_t)row * q_heads + (size_t)g * G) * kHeadDim;
    for (int h = 0; h < 16; ++h) {
        const bool live = h < G;
        if (lane < 16) {
            uint4 qv = make_uint4(0, 0, 0, 0), gv = make_uint4(0, 0, 0, 0);
            if (live) {
                qv = *reinterpret_cast<const uint4*>(q + head0 + (size_t)h * kHeadDim + lane * 8);
                gv = *reinterpret_cast<const uint4*>(dout + head0 + (size_t)h * kHeadDim + lane * 8);
            }
            *reinterpret_cast<uint4*>(qtile + swz256(h, lane)) = qv;
            *reinterpret_cast<uint4*>(gtile + swz256(h, lane)) = gv;
        }
        if (live) {
            const uint2 o2 = *reinterpret_cast<const uint2*>(out + head0 + (size_t)h * kHeadDim + lane * 4);
            const uint2 g2 = *reinterpret_cast<const uint2*>(dout + head0 + (size_t)h * kHeadDim + lane * 4);
            float d = bf16_lo(o2.x) * bf16_lo(g2.x) + bf16_hi(o2.x) * bf16_hi(g2.x) + bf16_lo(o2.y) * bf16_lo(g2.y) +
                      bf16_hi(o2.y) * bf16_hi(g2.y);
            d = warp_sum(d);
            if (lane == 0) dsm[h] = d;
        } else if (lane == 0) {
            dsm[h] = 0.f;
        }
    }
    __syncwarp();
    uint32_t qb[NT][8][2], gb[NT][8][2];
    b_frags<NT>(qtile, lane, qb);
    b_frags<NT>(gtile, lane, gb);
    // Per column (head 8 nt + 2 t + e): lse in the log2 domain and D.
    float lse2[NT][2], dd[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nt + 2 * t + e;
            lse2[nt][e] = h < G ? lse[(size_t)row * q_heads + (size_t)g * G + h] * LOG2E : 0.f;
            dd[nt][e] = dsm[h];
        }

    int ns = nsel[row];
    ns = ns < 0 ? 0 : (ns > kB ? kB : ns);
    const int32_t* srow = sel + (size_t)row * kB;
    const int ntok = (ns + 1) * r;  // selection entries, then the tail unit
    const int nchunks = (ntok + CT - 1) / CT;
    const size_t seq = (size_t)s * cap;
    const int64_t row_stride = (int64_t)kv_heads * kHeadDim;
    const uint32_t ring_s = smem_u32(wsm);

    auto issue = [&](int c) {
        const int stg = c % STAGES;
        const int pl = c * CT + (lane & (CT - 1));
        int32_t tk = -1;
        if (pl < ntok) {
            const int u = pl / r, e = pl % r;
            if (u == ns) {
                const int64_t tt = cur * r + e;
                if (tt <= i) tk = (int32_t)tt;
            } else {
                const int32_t b = srow[u];
                if (b >= 0 && (int64_t)b < cur) tk = b * r + e;
            }
        }
        if (lane < CT) toks[stg * CT + lane] = tk;
        const uint32_t kbase = ring_s + stg * STAGE_BYTES, vbase = kbase + CT * 256;
#pragma unroll
        for (int k = 0; k < (CT * 16) / 32; ++k) {
            const int idx = lane + k * 32;
            const int rw = idx >> 4, ch = idx & 15;
            const int32_t tkr = __shfl_sync(0xffffffffu, tk, rw);
            const bool ok = tkr >= 0;
            const size_t off = (seq + (size_t)(ok ? tkr : 0)) * row_stride + (size_t)g * kHeadDim + ch * 8;
            cp_async16_zfill(kbase + swz256(rw, ch), kc + off, ok);
            cp_async16_zfill(vbase + swz256(rw, ch), vc + off, ok);
        }
    };

    float acc[NT][8][4];  // dQ^T: rows dims 16 i + gq (+8), columns heads
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][a][e] = 0.f;

#pragma unroll
    for (int c = 0; c < STAGES - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kch = lane >> 4;
    const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8, vch = (lane >> 3) & 1;
    // ldmatrix.trans rows of the operand tiles for the dims-as-columns B fragments:
    // matrix m = lane / 8 covers heads 8 (m & 1) .. +7 and dims 8 (m >> 1) .. +7
    // of a 16-dim pair of n8 tiles.
    const int orow = (lane & 7) + 8 * ((lane >> 3) & 1), och = lane >> 4;
    const uint32_t qtile_s = smem_u32(qtile), gtile_s = smem_u32(gtile);
    float* dk_seq = dk + (seq * kv_heads + g) * kHeadDim;
    float* dv_seq = dv + (seq * kv_heads + g) * kHeadDim;

    for (int c = 0; c < nchunks; ++c) {
        if (c + STAGES - 1 < nchunks) issue(c + STAGES - 1);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const int stg = c % STAGES;
        const uint32_t kbase = ring_s + stg * STAGE_BYTES, vbase = kbase + CT * 256;
        const int32_t tk0 = toks[stg * CT + gq], tk1 = toks[stg * CT + gq + 8];

        // S^T = K Q^T and dP^T = V dO^T.
        float sc[NT][4], dp[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a0, a1, a2, a3, v0, v1, v2, v3;
            ldmatrix_x4(kbase + swz256(krow, ks * 2 + kch), a0, a1, a2, a3);
            ldmatrix_x4(vbase + swz256(krow, ks * 2 + kch), v0, v1, v2, v3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(sc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
                mma_bf16_16816(dp[nt], v0, v1, v2, v3, gb[nt][ks][0], gb[nt][ks][1]);
            }
        }
        // P and dS (rows gq, gq + 8; columns 8 nt + 2 t + e); invalid rows and
        // heads beyond G are zero.
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool hv = 8 * nt + 2 * t + e < G;
                const float p0 = (hv && tk0 >= 0) ? ex2_approx(sc[nt][e] * scale_log2 - lse2[nt][e]) : 0.f;
                const float p1 = (hv && tk1 >= 0) ? ex2_approx(sc[nt][2 + e] * scale_log2 - lse2[nt][e]) : 0.f;
                sc[nt][e] = p0;
                sc[nt][2 + e] = p1;
                dp[nt][e] = p0 * (dp[nt][e] - dd[nt][e]);
                dp[nt][2 + e] = p1 * (dp[nt][2 + e] - dd[nt][e]);
            }
        // dQ^T += K^T dS^T.
        uint32_t db[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            db[nt][0] = movmatrix_trans(pack_bf16x2(dp[nt][0], dp[nt][1]));
            db[nt][1] = movmatrix_trans(pack_bf16x2(dp[nt][2], dp[nt][3]));
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(kbase + swz256(vrow, 2 * a + vch), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt][a], a0, a1, a2, a3, db[nt][0], db[nt][1]);
        }
        // dV = P dO and dK = scale dS Q: A operands from the accumulators
        // (heads 0-7 from tile 0, heads 8-15 from tile 1 or zero).
        const uint32_t pa0 = pack_bf16x2(sc[0][0], sc[0][1]), pa1 = pack_bf16x2(sc[0][2], sc[0][3]);
        const uint32_t pa2 = NT > 1 ? pack_bf16x2(sc[NT - 1][0], sc[NT - 1][1]) : 0u;
        const uint32_t pa3 = NT > 1 ? pack_bf16x2(sc[NT - 1][2], sc[NT - 1][3]) : 0u;
        const uint32_t sa0 = pack_bf16x2(dp[0][0], dp[0][1]), sa1 = pack_bf16x2(dp[0][2], dp[0][3]);
        const uint32_t sa2 = NT > 1 ? pack_bf16x2(dp[NT - 1][0], dp[NT - 1][1]) : 0u;
        const uint32_t sa3 = NT > 1 ? pack_bf16x2(dp[NT - 1][2], dp[NT - 1][3]) : 0u;
        // Atomics as float4: lanes t and t ^ 1 swap halves so that an even-t
        // lane owns dims 2 t .. 2 t + 3 of row gq and an odd-t lane dims
        // 2 t - 2 .. 2 t + 1 of row gq + 8.
        const bool odd = t & 1;
        const int32_t tkm = odd ? tk1 : tk0;
        float* dvm = dv_seq + (size_t)(tkm >= 0 ? tkm : 0) * row_stride + 2 * (t & ~1);
        float* dkm = dk_seq + (size_t)(tkm >= 0 ? tkm : 0) * row_stride + 2 * (t & ~1);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {  // dims 16 jj .. 16 jj + 15 (two n8 tiles)
            uint32_t g0, g1, g2, g3, q0, q1, q2, q3;
            ldmatrix_x4_trans(gtile_s + swz256(orow, 2 * jj + och), g0, g1, g2, g3);
            ldmatrix_x4_trans(qtile_s + swz256(orow, 2 * jj + och), q0, q1, q2, q3);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float vt[4] = {0.f, 0.f, 0.f, 0.f}, kt[4] = {0.f, 0.f, 0.f, 0.f};
                mma_bf16_16816(vt, pa0, pa1, pa2, pa3, half ? g2 : g0, half ? g3 : g1);
                mma_bf16_16816(kt, sa0, sa1, sa2, sa3, half ? q2 : q0, half ? q3 : q1);
                const int dim = 16 * jj + 8 * half;
                const float v0 = __shfl_xor_sync(0xffffffffu, odd ? vt[0] : vt[2], 1);
                const float v1 = __shfl_xor_sync(0xffffffffu, odd ? vt[1] : vt[3], 1);
                const float k0 = __shfl_xor_sync(0xffffffffu, odd ? kt[0] : kt[2], 1);
                const float k1 = __shfl_xor_sync(0xffffffffu, odd ? kt[1] : kt[3], 1);
                if (tkm >= 0) {
                    atomicAdd(reinterpret_cast<float4*>(dvm + dim),
                              odd ? make_float4(v0, v1, vt[2], vt[3]) : make_float4(vt[0], vt[1], v0, v1));
                    atomicAdd(reinterpret_cast<float4*>(dkm + dim),
                              odd ? make_float4(k0 * scale, k1 * scale, kt[2] * scale, kt[3] * scale)
                                  : make_float4(kt[0] * scale, kt[1] * scale, k0 * scale, k1 * scale));
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // dQ rows: head 8 nt + 2 t + e, dims 16 a + gq (+8).
    float* dqr = dq + head0;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nt + 2 * t + e;
            if (h >= G) continue;
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                dqr[(size_t)h * kHeadDim + 16 * a + gq] = acc[nt][a][e] * scale;
                dqr[(size_t)h * kHeadDim + 16 * a + gq + 8] = acc[nt][a][2 + e] * scale;
            }
        }
}

// Warps (kv heads) per CTA: the largest divisor of kv_heads up to BW.
int warps_per_query(int kv_heads) {
    int gh = std::min(kv_heads, BW);
    while (kv_heads % gh) --gh;
    return gh;
}

template <int NT>
cudaError_t launch_bwd_t(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                         const uint16_t* kc, const uint16_t* vc, int64_t cap, const int32_t* sel,
                         const int32_t* nsel, const uint16_t* out, const float* lse, const uint16_t* dout,
                         float* dq, float* dk, float* dv, cudaStream_t st) {
    const int GH = warps_per_query(L.kv_heads);
    const int smem = GH * WARP_SMEM;
    auto kern = attention_backward_kernel<NT>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const dim3 grid((unsigned)nq, (unsigned)batch, (unsigned)(L.kv_heads / GH));
    note_launch();
    kern<<<grid, GH * 32, smem, st>>>(q, q_begin, nq, kc, vc, cap, sel, nsel, out, lse, dout, dq, dk, dv,
                                      L.q_heads, L.kv_heads, L.r, L.kB, L.sm_scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_backward(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                      const uint16_t* kc, const uint16_t* vc, int64_t cap, const int32_t* sel,
                                      const int32_t* nsel, const uint16_t* out, const float* lse,
                                      const uint16_t* dout, float* dq, float* dk, float* dv, cudaStream_t st) {
    if (batch <= 0 || nq <= 0) return cudaSuccess;
    const int G = L.q_heads / L.kv_heads;
    return G > 8 ? launch_bwd_t<2>(L, batch, q, q_begin, nq, kc, vc, cap, sel, nsel, out, lse, dout, dq, dk, dv, st)
                 : launch_bwd_t<1>(L, batch, q, q_begin, nq, kc, vc, cap, sel, nsel, out, lse, dout, dq, dk, dv, st);
}

}  // namespace qsa
