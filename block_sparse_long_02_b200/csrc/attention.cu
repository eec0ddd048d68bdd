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
//
// Variants: on fp8 caches (Q8) each chunk is gathered as E4M3 code rows with
// their row scales and converted into f16 tiles before the same tile products
// (in f16); the decode kernel runs one thread-block cluster per (sequence, kv
// head) and merges its split states over distributed shared memory.
#include <algorithm>

#include "attend.cuh"
#include "kernels.h"

namespace qsa {
namespace {

constexpr int WARPS = 4;
constexpr int SMEM = WARPS * WARP_SMEM;
constexpr int kMaxCluster = 16;           // decode CTAs per (sequence, kv head)

// Prefill: CTA = one query; warp w -> kv head kv0 + (w % GH), unit split w / GH.
// Q8: fp8 caches (codes with row scales ks, vs [batch][cap][kv_heads]).
template <int NT, bool Q8>
__global__ void __launch_bounds__(WARPS * 32) prefill_attention_kernel(
    const uint16_t* __restrict__ q, int64_t q_begin, int64_t nq, const void* __restrict__ kc,
    const void* __restrict__ vc, const float* __restrict__ ks, const float* __restrict__ vs, int64_t cap,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel, uint16_t* __restrict__ out,
    float* __restrict__ lse, int q_heads, int kv_heads, int r, int kB, float scale_log2) {
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
    const size_t seq_elems = (size_t)s * cap * kv_heads * kHeadDim;  // elements (bf16) or bytes (fp8)
    w.kc = Q8 ? (const void*)(static_cast<const uint8_t*>(kc) + seq_elems)
              : (const void*)(static_cast<const uint16_t*>(kc) + seq_elems);
    w.vc = Q8 ? (const void*)(static_cast<const uint8_t*>(vc) + seq_elems)
              : (const void*)(static_cast<const uint16_t*>(vc) + seq_elems);
    w.ks = Q8 ? ks + (size_t)s * cap * kv_heads : nullptr;
    w.vs = Q8 ? vs + (size_t)s * cap * kv_heads : nullptr;
    w.sel = sel + (size_t)row * kB;
    w.i = i;
    w.cur = i / r;
    w.nsel = ns;
    w.tail_unit = ns;
    w.u0 = (int)((int64_t)units * split / NS);
    w.u1 = (int)((int64_t)units * (split + 1) / NS);
    w.g = g;
    w.G = G;
    w.kv_heads = kv_heads;
    w.r = r;
    w.scale_log2 = scale_log2;

    uint8_t* wsm = smem + warp * WARP_SMEM;
    uint32_t qb[NT][8][2];
    if (Q8)
        load_q_frags_f16<NT>(w.q, G, lane, qb);
    else
        load_q_frags<NT>(w.q, G, lane, qb);
    const int32_t sel_lane = (w.u0 + lane < w.u1 && w.u0 + lane < ns) ? w.sel[w.u0 + lane] : -1;
    WarpState<NT> st;
    warp_attend<NT, Q8>(w, wsm, lane, qb, sel_lane, st);

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

// Writes a warp state in the head-major layout: o[h][128] (unnormalised),
// then m[h], then l[h] (log2 domain), heads h < G.

// Bytes of the decode kernel's receive area: C slices of the G x 128 outputs
// plus every CTA's m and l per head.
__host__ __device__ constexpr int decode_recv_bytes(int G, int C) { return (G * kHeadDim + 2 * G * C) * 4; }

// Decode: one thread-block cluster of C CTAs of DW warps per (sequence, kv
// head); warp w of CTA c takes unit split DW c + w of S = DW C. The units are the k_B
// selection entries (entry u counts if u < nsel) and, as unit k_B, the tail,
// so a split's entries are known before nsel is: the query and the position
// (inputs of the step) are read before the dependency wait, and nsel and the
// selection entries right after it, in one round trip. The four warp states
// of a CTA are merged element-wise by all its threads; CTA c then owns the
// outputs [c E / C, (c + 1) E / C) of the E = G x 128 and every CTA pushes its
// merged slice for them into c's shared memory (remote stores, no remote
// loads); after one cluster barrier each CTA finishes its slice locally.
// Q8: fp8 K/V caches (codes kc, vc with row scales ks, vs). HOT: kc, vc are
// host memory and hot holds an HBM cache of blocks (see HotCache).
template <int NT, int DW, bool Q8, bool HOT = false>
__global__ void __launch_bounds__(DW * 32) decode_attention_kernel(
    const uint16_t* __restrict__ q, const int64_t* __restrict__ pos,
    const void* __restrict__ kc, const void* __restrict__ vc, const float* __restrict__ ks,
    const float* __restrict__ vs, int64_t cap,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel, uint16_t* __restrict__ out,
    int q_heads, int kv_heads, int r, int kB, float scale_log2, HotCache hot) {
    extern __shared__ __align__(128) uint8_t smem[];
    cluster_arrive_relaxed();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = (int)gridDim.x;        // the cluster spans the grid's x dimension
    const int rank = (int)blockIdx.x;    // = rank in the cluster
    const int g = (int)blockIdx.y, s = (int)blockIdx.z;
    const int G = q_heads / kv_heads;
    const int S = C * DW, split = rank * DW + warp;
    const int units = kB + 1;
    Work w;
    w.q = q + ((size_t)s * q_heads + (size_t)g * G) * kHeadDim;
    const size_t seq_elems = (size_t)s * cap * kv_heads * kHeadDim;  // elements (bf16) or bytes (fp8)
    w.kc = Q8 ? (const void*)(static_cast<const uint8_t*>(kc) + seq_elems)
              : (const void*)(static_cast<const uint16_t*>(kc) + seq_elems);
    w.vc = Q8 ? (const void*)(static_cast<const uint8_t*>(vc) + seq_elems)
              : (const void*)(static_cast<const uint16_t*>(vc) + seq_elems);
    w.ks = Q8 ? ks + (size_t)s * cap * kv_heads : nullptr;
    w.vs = Q8 ? vs + (size_t)s * cap * kv_heads : nullptr;
    const size_t hot_seq = (size_t)s * (hot.blocks + 1) * r * kv_heads * kHeadDim;
    w.hot_k = HOT ? hot.k + hot_seq : nullptr;
    w.hot_v = HOT ? hot.v + hot_seq : nullptr;
    w.tags = HOT ? hot.tags + (size_t)s * (hot.blocks + 1) : nullptr;
    w.hot_blocks = (int32_t)hot.blocks;
    w.tail_hrow0 = -1;
    w.sel = sel + (size_t)s * kB;
    w.tail_unit = kB;
    w.u0 = (int)((int64_t)units * split / S);
    w.u1 = (int)((int64_t)units * (split + 1) / S);
    w.g = g;
    w.G = G;
    w.kv_heads = kv_heads;
    w.r = r;
    w.scale_log2 = scale_log2;
    // Inputs of the step: the kernels before this one in the step do not
    // write them, and they were complete before the step's first kernel ran.
    const int64_t p = pos[s];
    uint32_t qb[NT][8][2];
    if (Q8)
        load_q_frags_f16<NT>(w.q, G, lane, qb);
    else
        load_q_frags<NT>(w.q, G, lane, qb);
    uint8_t* wsm = smem + warp * WARP_SMEM;
    WarpState<NT> st;
    w.cur = p / r;
    pdl_wait();
    pdl_trigger();
    const int u_sel = w.u0 + lane;
    const int32_t sel_lane = (u_sel < w.u1 && u_sel < kB) ? __ldcg(w.sel + u_sel) : -1;
    int ns = __ldcg(nsel + s);
    ns = ns < 0 ? 0 : (ns > kB ? kB : ns);
    w.nsel = ns;
    w.i = p;
    if (p < 0 || p >= cap) w.u1 = w.u0;  // skipped sequence: zero output
    int32_t hot_lane = -1;  // HOT: the hot slot holding this lane's selected block
    if (HOT) {
        if (sel_lane >= 0) {
            const int32_t slot = sel_lane % w.hot_blocks;
            if (__ldcg(w.tags + slot) == sel_lane) hot_lane = slot;
        }
        if (__ldcg(w.tags + w.hot_blocks) == (int32_t)w.cur) w.tail_hrow0 = w.hot_blocks * r;
    }

    warp_attend<NT, Q8, HOT>(w, wsm, lane, qb, sel_lane, st, hot_lane);

    const int E = G * kHeadDim, per = E / C;
    store_state_hd<NT>(st, G, reinterpret_cast<float*>(wsm), lane);
    __syncthreads();
    float* recv = reinterpret_cast<float*>(smem + DW * WARP_SMEM);  // [C][per] o, [C][G] m, [C][G] l
    const uint32_t recv_s = smem_u32(recv);
    cluster_wait();  // every CTA of the cluster runs: its receive area exists
    for (int x = threadIdx.x; x < E; x += DW * 32) {
        const int h = x / kHeadDim;
        float mw[DW], M = -INFINITY;
#pragma unroll
        for (int k = 0; k < DW; ++k) {
            mw[k] = reinterpret_cast<const float*>(smem + k * WARP_SMEM)[E + h];
            M = fmaxf(M, mw[k]);
        }
        float o = 0.f;
#pragma unroll
        for (int k = 0; k < DW; ++k)
            o = fmaf(reinterpret_cast<const float*>(smem + k * WARP_SMEM)[x], M == -INFINITY ? 0.f : exp2f(mw[k] - M), o);
        const int owner = x / per;
        st_dsmem(dsmem_addr(recv_s + (uint32_t)(rank * per + x - owner * per) * 4u, (uint32_t)owner), o);
    }
    for (int h = threadIdx.x; h < G; h += DW * 32) {
        float mw[DW], M = -INFINITY, L = 0.f;
#pragma unroll
        for (int k = 0; k < DW; ++k) {
            mw[k] = reinterpret_cast<const float*>(smem + k * WARP_SMEM)[E + h];
            M = fmaxf(M, mw[k]);
        }
#pragma unroll
        for (int k = 0; k < DW; ++k)
            L = fmaf(reinterpret_cast<const float*>(smem + k * WARP_SMEM)[E + G + h],
                     M == -INFINITY ? 0.f : exp2f(mw[k] - M), L);
        for (int c2 = 0; c2 < C; ++c2) {
            st_dsmem(dsmem_addr(recv_s + (uint32_t)(E + rank * G + h) * 4u, (uint32_t)c2), M);
            st_dsmem(dsmem_addr(recv_s + (uint32_t)(E + C * G + rank * G + h) * 4u, (uint32_t)c2), L);
        }
    }
    cluster_sync();  // every push has landed
    for (int xi = threadIdx.x; xi < per; xi += DW * 32) {
        const int x = rank * per + xi, h = x / kHeadDim;
        float M = -INFINITY;
        for (int j = 0; j < C; ++j) M = fmaxf(M, recv[E + j * G + h]);
        float num = 0.f, den = 0.f;
        for (int j = 0; j < C; ++j) {
            const float c = M == -INFINITY ? 0.f : exp2f(recv[E + j * G + h] - M);
            num = fmaf(recv[j * per + xi], c, num);
            den = fmaf(recv[E + C * G + j * G + h], c, den);
        }
        out[((size_t)s * q_heads + (size_t)g * G) * kHeadDim + x] = f32_to_bf16(den > 0.f ? num / den : 0.f);
    }
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
    auto kern = G > 8 ? prefill_attention_kernel<2, false> : prefill_attention_kernel<1, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    note_launch();
    kern<<<grid, WARPS * 32, SMEM, st>>>(q, q_begin, nq, kc, vc, nullptr, nullptr, cap, sel, nsel, out, lse,
                                         L.q_heads, L.kv_heads, L.r, L.kB, L.sm_scale * LOG2E);
    return cudaGetLastError();
}

cudaError_t launch_sparse_attention_q8(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin,
                                       int64_t nq, const uint8_t* k8, const float* ks, const uint8_t* v8,
                                       const float* vs, int64_t cap, const int32_t* sel, const int32_t* nsel,
                                       uint16_t* out, float* lse, cudaStream_t st) {
    if (nq <= 0 || batch <= 0) return cudaSuccess;
    const int GH = L.kv_heads < WARPS ? L.kv_heads : WARPS;
    dim3 grid((unsigned)nq, (unsigned)batch, (unsigned)(L.kv_heads / GH));
    const int G = L.q_heads / L.kv_heads;
    auto kern = G > 8 ? prefill_attention_kernel<2, true> : prefill_attention_kernel<1, true>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    note_launch();
    kern<<<grid, WARPS * 32, SMEM, st>>>(q, q_begin, nq, k8, v8, ks, vs, cap, sel, nsel, out, lse, L.q_heads,
                                         L.kv_heads, L.r, L.kB, L.sm_scale * LOG2E);
    return cudaGetLastError();
}

// Launch shape of the decode attention: DW warps per CTA and C CTAs per
// cluster (one cluster per (sequence, kv head)). More warps per CTA shorten the
// per-warp chain of chunks when the batch leaves SMs idle; otherwise the
// largest of 16, 8, 4, 2, 1 CTAs per cluster whose grid runs in one wave and
// whose cluster the device can place.
namespace {

struct DecodeShape {
    int dw, c;
};

template <int NT, int DW>
int decode_cluster_for(const LayerDims& L, int batch, int G) {
    auto kern = decode_attention_kernel<NT, DW, false>;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int base = DW * WARP_SMEM;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, base + decode_recv_bytes(G, kMaxCluster));
    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    for (int C = kMaxCluster; C > 1; C >>= 1) {
        const int smem = base + decode_recv_bytes(G, C);
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, DW * 32, smem) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        if ((int64_t)batch * L.kv_heads * C > (int64_t)sms * per_sm) continue;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)C, (unsigned)L.kv_heads, (unsigned)batch);
        cfg.blockDim = dim3(DW * 32);
        cfg.dynamicSmemBytes = (size_t)smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0) return C;
        cudaGetLastError();  // clear a refused size
    }
    return 1;
}

template <int NT>
DecodeShape decode_shape(const LayerDims& L, int batch, int G) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if ((int64_t)batch * L.kv_heads * kMaxCluster <= sms) {
        const int c = decode_cluster_for<NT, 8>(L, batch, G);
        if (c == kMaxCluster) return {8, c};
    }
    return {4, decode_cluster_for<NT, 4>(L, batch, G)};
}

template <int NT, int DW, bool Q8, bool HOT>
cudaError_t launch_decode_attention_t(const LayerDims& L, int batch, int C, const int64_t* pos, const uint16_t* q,
                                      const void* kc, const void* vc, const float* ks, const float* vs, int64_t cap,
                                      const int32_t* sel, const int32_t* nsel, uint16_t* out, const HotCache& hot,
                                      cudaStream_t st) {
    auto kern = decode_attention_kernel<NT, DW, Q8, HOT>;
    const int G = L.q_heads / L.kv_heads;
    const int smem = DW * WARP_SMEM + decode_recv_bytes(G, C);
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (C > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)L.kv_heads, (unsigned)batch);
    cfg.blockDim = dim3(DW * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    note_launch();
    return cudaLaunchKernelEx(&cfg, kern, q, pos, kc, vc, ks, vs, cap, sel, nsel, out, L.q_heads, L.kv_heads, L.r,
                              L.kB, L.sm_scale * LOG2E, hot);
}

template <int NT>
cudaError_t launch_decode_attention_nt(const LayerDims& L, int batch, const DecodeShape& sh, const int64_t* pos,
                                       const uint16_t* q, const void* kc, const void* vc, const float* ks,
                                       const float* vs, bool q8, int64_t cap, const int32_t* sel, const int32_t* nsel,
                                       uint16_t* out, const HotCache& hot, cudaStream_t st) {
#define QSA_DA(DW_, Q8_, HOT_) \
    launch_decode_attention_t<NT, DW_, Q8_, HOT_>(L, batch, sh.c, pos, q, kc, vc, ks, vs, cap, sel, nsel, out, hot, st)
    if (hot.k) return sh.dw == 8 ? QSA_DA(8, false, true) : QSA_DA(4, false, true);
    if (q8) return sh.dw == 8 ? QSA_DA(8, true, false) : QSA_DA(4, true, false);
    return sh.dw == 8 ? QSA_DA(8, false, false) : QSA_DA(4, false, false);
#undef QSA_DA
}

}  // namespace

cudaError_t launch_decode_attention(const LayerDims& L, int batch, const int64_t* pos,
                                    const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                    int64_t cap, const int32_t* sel, const int32_t* nsel,
                                    uint16_t* out, const Q8Caches* q8, const HotCache* hot, cudaStream_t st) {
    if (batch <= 0) return cudaSuccess;
    const int G = L.q_heads / L.kv_heads;
    // The launch shape is chosen once per problem shape (and thread).
    static thread_local int cached_key[4] = {-1, -1, -1, -1};
    static thread_local DecodeShape cached = {4, 1};
    const int key[4] = {batch, L.q_heads, L.kv_heads, L.kB};
    if (!std::equal(key, key + 4, cached_key)) {
        cached = G > 8 ? decode_shape<2>(L, batch, G) : decode_shape<1>(L, batch, G);
        std::copy(key, key + 4, cached_key);
    }
    const DecodeShape sh = cached;
    const void* k = q8 ? (const void*)q8->k8 : (const void*)kc;
    const void* v = q8 ? (const void*)q8->v8 : (const void*)vc;
    const float* ks = q8 ? q8->ks : nullptr;
    const float* vs = q8 ? q8->vs : nullptr;
    const HotCache hc = hot ? *hot : HotCache{nullptr, nullptr, nullptr, 1};
    if (G > 8)
        return launch_decode_attention_nt<2>(L, batch, sh, pos, q, k, v, ks, vs, q8 != nullptr, cap, sel, nsel, out, hc,
                                             st);
    return launch_decode_attention_nt<1>(L, batch, sh, pos, q, k, v, ks, vs, q8 != nullptr, cap, sel, nsel, out, hc,
                                         st);
}

}  // namespace qsa
