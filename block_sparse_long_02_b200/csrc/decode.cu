// Decode step pieces ("QSA (Qwen Sparse Attention)" concept page, (A)-(B), for
// one new token per sequence): a8 (cache append, block pooling) with a3' (query
// rotation), the a4 score stream over every pooled key of a sequence, and the
// a5 selection; and the whole step as one persistent kernel.
//
// The score stream is the hot spot: 256 bytes of pooled key per block and
// 4 x 128 multiply-adds, an L2/HBM stream spread over one wave of CTAs, each
// scoring its slice on the tensor cores (mma.sync) from 16-byte loads issued a
// group ahead (streaming, evict-first loads when the batch's keys outsize L2).
// The same pass builds a per-sequence histogram of a level-1 key digit of the
// scores, so the selection reads the score row once more and never sorts it:
// every CTA of the selection grid finds the threshold digit, collects the sure
// winners and the threshold-digit candidates of its slice, and reserves room
// for them in the sequence's global lists; the last CTA to finish resolves the
// exact pick among the candidates (ties to the lower block index) and writes
// the k_B winners in ascending order.
//
// decode_step_kernel runs append, scores, selection and attention in one
// launch (see its comment); the attention there is the warp-level code of
// attend.cuh, and the three-kernel path's attention is in attention.cu.
#include <algorithm>
#include <atomic>

#include "attend.cuh"
#include "kernels.h"
#include "rope.cuh"
#include "select.cuh"

namespace qsa {
namespace {

constexpr int DS_THREADS = 256;  // fused score CTAs
constexpr int DS_WARPS = DS_THREADS / 32;

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// cp.async of 16 bytes (zero-filled when !valid) with an L2 cache policy.
__device__ __forceinline__ void cp_async16_zfill_hint(uint32_t dst, const void* src, bool valid, uint64_t pol) {
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src), "r"(sz),
                 "l"(pol));
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Inter-CTA signalling at GPU scope. A CTA publishes its threads' writes by a
// __syncthreads() followed by one release (or acq_rel) operation of thread 0;
// a reader acquires with thread 0 and then __syncthreads().
__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int32_t* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_release(int32_t* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_add_acq_rel(int32_t* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

constexpr int kScoreRing = 3;       // cp.async stages per warp of the step kernel's score stream (bf16 keys)
constexpr float kPreFactor = 0.8f;  // pre-filter threshold: this fraction of the estimated k-th score
constexpr int kCtaList = 1024;      // listed blocks a step CTA gathers in shared memory

// Blocks [lo, hi) of a sequence's nvis visible blocks handled by CTA x of X.
__device__ __forceinline__ void cta_range(int64_t nvis, int x, int X, int64_t& lo, int64_t& hi) {
    const int64_t chunk = (nvis + X - 1) / X;
    lo = min(nvis, (int64_t)x * chunk);
    hi = min(nvis, lo + chunk);
}

// Level-1 digit of a decode score's key: bits 30..20 (8 exponent and 3
// mantissa bits). Decode scores are sums of ReLUs, never negative, so the sign
// bit carries nothing; a negative key (impossible here) maps to digit 0, which
// the selection treats as "refine from the row".
__device__ __forceinline__ uint32_t dec_digit1(uint32_t key) {
    return key >= 0x80000000u ? (key >> 20) & 2047u : 0u;
}
// Level-2 digit inside a level-1 bin: bits 19..9.
__device__ __forceinline__ uint32_t dec_digit2(uint32_t key) { return (key >> 9) & 2047u; }

// One decode step's cache update, query rotation and score stream, fused.
//
// CTA (0, s) appends the new token's K, V and raw indexer key to the caches
// and, when the token closes its block, pools that block for later steps (a8;
// the block is not visible at this position, so no CTA of this step reads
// it); with more than one CTA per sequence it scores nothing, so the slow
// fp64 rotation of the pooling never delays a score slice. The other CTAs
// rotate the new indexer query themselves (a3', fp64, from one shared table
// of the position's angles) and score their slices of the visible pooled
// keys (a4) on the tensor cores:
// mma.sync m16n8k16 with A = 16 pooled keys x 16 dims and B = 16 dims x
// (4 heads + 4 zero columns). The 128 dims are taken in a fixed permutation
// (the same for keys and query, so every dot product is unchanged) chosen so
// that lane (g, t) of a warp reads its A fragments for all 8 k-steps of rows
// g and g + 8 with four 16-byte loads per row: chunk i of lane t is bytes
// [64 i + 16 t, +16) of the row, and k-step j uses its pairs 2 (j % 2) and
// 2 (j % 2) + 1 of chunk j / 2 as the low and high column pairs. The ReLU
// head sum takes one shuffle; the scores go to `scores` and their top 11 key
// bits to the sequence's histogram (zeroed by the selection after use).
//
// Q8 (fp8 caches): the appended K and V rows are quantized (one warp per row),
// a block closed by the token is pooled into the bf16 pooled keys and then
// quantized into the fp8 pooled keys, and the stream reads those: 128-byte
// code rows (each lane's 16-byte pieces hold 16 dims, so the fixed dimension
// permutation maps virtual chunk 2 i' + c of lane t to dims 64 i' + 16 t + 8 c),
// converted to f16 (exact) for an f16 mma.sync; a block's ReLU head sum is
// multiplied by its scale (scales are non-negative, so ReLU commutes).
// (The body, for CTAs of NWARPS warps; the step kernel below runs it too.
// RING > 0, bf16 keys: each warp streams its groups of 16 keys through RING
// 4 KB stages of shared memory at `ring` with cp.async (RING - 1 groups in
// flight without holding registers) instead of a register double buffer.)
template <bool Q8, int NWARPS, int RING = 0, bool STREAM = true>
__device__ __forceinline__ void score_body(uint8_t* ring, float2* est, uint2* pre, int32_t* pre_count,
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, int kB, double eps, RopeTable rt,
    float* __restrict__ scores, uint32_t* __restrict__ hist_g, int32_t* __restrict__ status, Q8Caches q8,
    HotCache hot) {
    constexpr int DS_THREADS = NWARPS * 32, DS_WARPS = NWARPS;
    __shared__ uint32_t hist[2048];
    __shared__ __align__(16) uint16_t qs[kIdxHeads * kIdxDim];
    __shared__ double2 cs[kIdxDim / 2];  // (sin, cos) of the query position's angles
    __shared__ float qnorm[kIdxHeads];
    __shared__ int n_clist, clist_at;  // blocks this CTA listed; their place in the sequence's list
    const int s = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // The position and the indexer query are inputs of the step (complete
    // before the step's first kernel could start), so the query rotation runs
    // before the dependency wait, overlapping the end of the previous step.
    const int64_t p = pos[s];
    const bool valid = p >= 0 && p < cap;
    const int X = gridDim.x > 1 ? (int)gridDim.x - 1 : 1;  // scoring CTAs
    const int x = gridDim.x > 1 ? (int)blockIdx.x - 1 : 0;  // CTA 0 only appends and pools
    int64_t lo = 0, hi = 0;
    if (valid && p / r > kB && x >= 0) cta_range(p / r, x, X, lo, hi);
    const bool scoring = lo < hi;  // (uniform over the CTA)
    if (scoring) {
        // The rope_dims / 2 angles of position p once per CTA (an fp64 sincos of
        // a large argument is slow), then the 4 heads rotate from the table.
        if (tid < rt.half) {
            double sn, cn;
            sincos(__dmul_rn((double)p, rt.theta[tid]), &sn, &cn);
            cs[tid] = make_double2(sn, cn);
        }
        for (int b = tid; b < 2048; b += DS_THREADS) hist[b] = 0u;
        __syncthreads();
        if (warp < kIdxHeads)
            rotate_head_warp_tab(idx_q + ((size_t)s * kIdxHeads + warp) * kIdxDim, rt.half, cs,
                                 qs + warp * kIdxDim, lane);
        if (est && warp < kIdxHeads) {  // |q_h| of the rotated (stored) query, for the pre-filter
            __syncwarp();
            float ss = 0.f;
            for (int j = lane; j < kIdxDim; j += 32) {
                const float q = bf16f(qs[warp * kIdxDim + j]);
                ss = fmaf(q, q, ss);
            }
            ss = warp_sum(ss);
            if (lane == 0) qnorm[warp] = sqrtf(ss);
        }
        __syncthreads();
    }
    pdl_wait();
    pdl_trigger();
    if (!valid) {
        if (blockIdx.x == 0 && tid == 0) flag_status(status, 4 /* QSA_ERR_CAPACITY */);
        return;
    }
    if (blockIdx.x == 0) {
        if constexpr (Q8) {
            for (int row = warp; row < 2 * kv_heads; row += DS_WARPS) {  // K rows, then V rows
                const bool isk = row < kv_heads;
                const int h = isk ? row : row - kv_heads;
                const size_t cr = ((size_t)s * cap + p) * kv_heads + h;  // (token, kv head) row of the cache
                quantize_row128_warp((isk ? k : v) + ((size_t)s * kv_heads + h) * kHeadDim,
                                     (isk ? q8.k8 : q8.v8) + cr * kHeadDim, (isk ? q8.ks : q8.vs) + cr, lane);
            }
        } else {
            const int row16 = kv_heads * kHeadDim / 8;  // 16-byte chunks per kv row
            const uint4* ks = reinterpret_cast<const uint4*>(k + (size_t)s * kv_heads * kHeadDim);
            const uint4* vs = reinterpret_cast<const uint4*>(v + (size_t)s * kv_heads * kHeadDim);
            uint4* kd = reinterpret_cast<uint4*>(kc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
            uint4* vd = reinterpret_cast<uint4*>(vc + ((size_t)s * cap + p) * kv_heads * kHeadDim);
            for (int c = tid; c < row16; c += DS_THREADS) {
                kd[c] = ks[c];
                vd[c] = vs[c];
            }
            if (hot.k) {
                // Host caches: the token also goes to row p % r of the tail slot,
                // which holds the current block's tokens once its tag names it.
                const size_t tail = (((size_t)s * (hot.blocks + 1) + hot.blocks) * r + p % r) * row16;
                uint4* tk = reinterpret_cast<uint4*>(hot.k) + tail;
                uint4* tv = reinterpret_cast<uint4*>(hot.v) + tail;
                for (int c = tid; c < row16; c += DS_THREADS) {
                    tk[c] = ks[c];
                    tv[c] = vs[c];
                }
                if (tid == 0) {
                    int32_t* tag = hot.tags + (size_t)s * (hot.blocks + 1) + hot.blocks;
                    const int32_t cur = (int32_t)(p / r);
                    // Rows before p are there when the tag already names the block.
                    *tag = (p % r == 0 || *tag == cur) ? cur : -1;
                }
            }
        }
        if (tid < kIdxDim / 8)
            reinterpret_cast<uint4*>(idx_k_cache + ((size_t)s * cap + p) * kIdxDim)[tid] =
                reinterpret_cast<const uint4*>(idx_k + (size_t)s * kIdxDim)[tid];
        // The block's last raw key is read from the input (its cache row is
        // written by another thread of this CTA).
        if (warp == kIdxHeads && (p + 1) % r == 0) {
            const int64_t b = p / r;
            uint16_t* prow = pooled + ((size_t)s * (cap / r) + b) * kIdxDim;
            pool_block_warp(idx_k_cache + ((size_t)s * cap + (size_t)b * r) * kIdxDim,
                            idx_k + (size_t)s * kIdxDim, r, rms_w, eps, b * r, rt, prow, lane);
            if constexpr (Q8) {
                __syncwarp();  // each lane reads back the values it stored
                const size_t pr = (size_t)s * (cap / r) + b;
                quantize_row128_warp(prow, q8.pooled8 + pr * kIdxDim, q8.pscale + pr, lane);
            }
        }
    }
    if (!scoring) return;  // (also: every visible block is selected, no scores needed)
    const int64_t pcap = cap / r;
    const int g = lane >> 2, t = lane & 3;
    // B fragments: column g (head g, zero for g >= 4), k-step j.
    uint32_t bq0[8], bq1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = j >> 1;
        const int d = Q8 ? 64 * (i >> 1) + 16 * t + 8 * (i & 1) + 4 * (j & 1) : 32 * i + 8 * t + 4 * (j & 1);
        bq0[j] = g < kIdxHeads ? *reinterpret_cast<const uint32_t*>(qs + g * kIdxDim + d) : 0u;
        bq1[j] = g < kIdxHeads ? *reinterpret_cast<const uint32_t*>(qs + g * kIdxDim + d + 2) : 0u;
        if (Q8) {  // the query in f16 (exact for its bf16 values inside the f16 range)
            bq0[j] = pack_f16x2(bf16_lo(bq0[j]), bf16_hi(bq0[j]));
            bq1[j] = pack_f16x2(bf16_lo(bq1[j]), bf16_hi(bq1[j]));
        }
    }
    const uint16_t* keys = pooled + (size_t)s * pcap * kIdxDim;
    const uint8_t* keys8 = Q8 ? q8.pooled8 + (size_t)s * pcap * kIdxDim : nullptr;
    const float* kscale = Q8 ? q8.pscale + (size_t)s * pcap : nullptr;
    float* dst = scores + (size_t)s * pcap;
    // bf16: four 16-byte pieces of each row; fp8: two (16 codes each), and the
    // rows' scales.
    // STREAM: the batch's pooled keys outsize the L2, so they are read with
    // streaming loads (ld.global.cs, evict-first) and what the selection and
    // the attention reuse, their code included, stays in L2; otherwise plain
    // loads, which let the keys stay in L2 for the next step.
    auto ldk = [](const void* a) {
        return STREAM ? __ldcs(reinterpret_cast<const uint4*>(a)) : __ldg(reinterpret_cast<const uint4*>(a));
    };
    auto load = [&](int64_t base, uint4 (&ra)[4], uint4 (&rb)[4], float& sa_, float& sb_) {
        const int64_t b0 = base + g, b1 = b0 + 8;
        if constexpr (Q8) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                ra[i] = b0 < hi ? ldk(keys8 + (size_t)b0 * kIdxDim + 64 * i + 16 * t) : make_uint4(0u, 0u, 0u, 0u);
                rb[i] = b1 < hi ? ldk(keys8 + (size_t)b1 * kIdxDim + 64 * i + 16 * t) : make_uint4(0u, 0u, 0u, 0u);
            }
            sa_ = (t == 0 && b0 < hi) ? __ldg(kscale + b0) : 0.f;
            sb_ = (t == 0 && b1 < hi) ? __ldg(kscale + b1) : 0.f;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ra[i] = b0 < hi ? ldk(keys + (size_t)b0 * kIdxDim + 32 * i + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
                rb[i] = b1 < hi ? ldk(keys + (size_t)b1 * kIdxDim + 32 * i + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // fp8: 16 codes -> two virtual bf16-layout pieces of f16 pairs.
    auto widen = [&](const uint4& c, uint4& lo4, uint4& hi4) {
        const uint32_t w4[4] = {c.x, c.y, c.z, c.w};
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[2 * j] = e4m3x2_to_f16x2((uint16_t)(w4[j] & 0xFFFFu));
            h[2 * j + 1] = e4m3x2_to_f16x2((uint16_t)(w4[j] >> 16));
        }
        lo4 = make_uint4(h[0], h[1], h[2], h[3]);
        hi4 = make_uint4(h[4], h[5], h[6], h[7]);
    };
    const int64_t step = 16 * DS_WARPS;
    int64_t base = lo + 16 * warp;
    // Scores of rows g, g + 8 of the group at `gb` (lanes t = 0) to the row and
    // the histogram.
    auto emit = [&](int64_t gb, float sa, float sb) {
        if (t == 0) {
            const int64_t b0 = gb + g, b1 = b0 + 8;
            if (b0 < hi) {
                dst[b0] = sa;
                atomicAdd(&hist[dec_digit1(float_key(sa))], 1u);
            }
            if (b1 < hi) {
                dst[b1] = sb;
                atomicAdd(&hist[dec_digit1(float_key(sb))], 1u);
            }
        }
    };
    // The pre-filter threshold tau: the last step's k-th score per unit of its
    // query's summed head norms, times this query's sum, times kPreFactor.
    // Blocks scoring at least tau are also listed (key, block); when the list
    // holds at least k_B of them it holds every top-k_B block, ties included,
    // whatever tau was. The CTA's listed blocks gather in shared memory (after
    // the ring, if any) and go to the sequence's list with one reservation.
    float tau = 0.f;
    if (est) {
        const float qsum = (qnorm[0] + qnorm[1]) + (qnorm[2] + qnorm[3]);
        const float ratio = __ldcg(&est[s].x);
        tau = ratio > 0.f ? ratio * qsum * kPreFactor : 0.f;
        if (x == 0 && tid == 0) est[s].y = qsum;  // (the first scoring CTA)
    }
    const bool listing = est && tau > 0.f;  // (NaN: no list; est is null without a list in shared memory)
    uint2* clist = est ? reinterpret_cast<uint2*>(ring + NWARPS * RING * 4096) : nullptr;
    if (tid == 0) n_clist = 0;
    __syncthreads();
    auto list = [&](int64_t gb, float sa, float sb) {  // warp-aggregated appends (every lane calls)
        const int64_t b0 = gb + g, b1 = b0 + 8;
        const bool ha = t == 0 && b0 < hi && sa >= tau, hb = t == 0 && b1 < hi && sb >= tau;
        const uint32_t ba = __ballot_sync(0xffffffffu, ha), bb = __ballot_sync(0xffffffffu, hb);
        if (ba | bb) {
            int at0 = 0;
            if (lane == 0) at0 = atomicAdd(&n_clist, __popc(ba) + __popc(bb));
            at0 = __shfl_sync(0xffffffffu, at0, 0);
            const uint32_t below = (1u << lane) - 1u;
            const int aa = at0 + __popc(ba & below), ab = at0 + __popc(ba) + __popc(bb & below);
            if (ha && aa < kCtaList) clist[aa] = make_uint2(float_key(sa), (uint32_t)b0);
            if (hb && ab < kCtaList) clist[ab] = make_uint2(float_key(sb), (uint32_t)b1);
        }
    };
    // After the stream: the CTA's histogram counts, and its list with one
    // reservation (a CTA list that overflowed marks the sequence's list
    // overflowed: the full selection runs).
    auto finish = [&]() {
        __syncthreads();
        for (int b = tid; b < 2048; b += DS_THREADS)
            if (hist[b]) atomicAdd(&hist_g[(size_t)s * 2048 + b], hist[b]);
        if (listing) {
            const int n = n_clist;
            if (tid == 0) clist_at = n > kCtaList ? -1 : (n ? atomicAdd(pre_count, n) : 0);
            __syncthreads();
            const int at = clist_at;
            if (at < 0) {
                if (tid == 0) atomicAdd(pre_count, kDecodePre + 1);
            } else {
                uint2* plist = pre + (size_t)s * kDecodePre;
                for (int i = tid; i < n && at + i < kDecodePre; i += DS_THREADS) plist[at + i] = clist[i];
            }
        }
    };
    if constexpr (RING > 0 && !Q8) {
        // Stage layout: piece i (0..7) of lane l at i * 512 + l * 16 (conflict-free
        // 16-byte accesses); each lane reads back only the pieces it copied.
        const uint32_t wring = smem_u32(ring) + (uint32_t)(warp * RING * 4096 + lane * 16);
        // The pooled keys are read once per step: first out of L2, so that what
        // the selection and the attention reuse (their code included) stays.
        const uint64_t pol = l2_evict_first_policy();
        auto issue = [&](int64_t gb, int stage) {
            const int64_t b0 = gb + g, b1 = b0 + 8;
            const uint16_t* ra = keys + (size_t)(b0 < hi ? b0 : 0) * kIdxDim + 8 * t;
            const uint16_t* rb = keys + (size_t)(b1 < hi ? b1 : 0) * kIdxDim + 8 * t;
            const uint32_t d = wring + (uint32_t)(stage * 4096);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cp_async16_zfill_hint(d + i * 512, ra + 32 * i, b0 < hi, pol);
                cp_async16_zfill_hint(d + (4 + i) * 512, rb + 32 * i, b1 < hi, pol);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int st = 0; st < RING; ++st) issue(base + st * step, st);
        int stage = 0;
        for (; base < hi; base += step) {
            cp_async_wait<RING - 1>();
            uint4 ca[4], cb[4];
            const uint32_t d = wring + (uint32_t)(stage * 4096);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ca[i] = ld_shared_v4(d + i * 512);
                cb[i] = ld_shared_v4(d + (4 + i) * 512);
            }
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mma_bf16_16816(c, ca[i].x, cb[i].x, ca[i].y, cb[i].y, bq0[2 * i], bq1[2 * i]);
                mma_bf16_16816(c, ca[i].z, cb[i].z, ca[i].w, cb[i].w, bq0[2 * i + 1], bq1[2 * i + 1]);
            }
            // (the stage's values are in registers, consumed above: refill it)
            issue(base + RING * step, stage);
            stage = stage + 1 == RING ? 0 : stage + 1;
            float sa = fmaxf(c[0], 0.f) + fmaxf(c[1], 0.f);
            float sb = fmaxf(c[2], 0.f) + fmaxf(c[3], 0.f);
            sa += __shfl_xor_sync(0xffffffffu, sa, 1);
            sb += __shfl_xor_sync(0xffffffffu, sb, 1);
            emit(base, sa, sb);
            if (listing) list(base, sa, sb);
        }
        cp_async_wait<0>();
        finish();
        return;
    }
    uint4 ca[4], cb[4];
    float psa = 0.f, psb = 0.f;
    load(base, ca, cb, psa, psb);
    for (; base < hi; base += step) {
        uint4 na[4], nb[4];
        float nsa = 0.f, nsb = 0.f;
        load(base + step, na, nb, nsa, nsb);  // the next group, in flight during this one
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (Q8) {
            uint4 wa[4], wb[4];
            widen(ca[0], wa[0], wa[1]);
            widen(ca[1], wa[2], wa[3]);
            widen(cb[0], wb[0], wb[1]);
            widen(cb[1], wb[2], wb[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mma_f16_16816(c, wa[i].x, wb[i].x, wa[i].y, wb[i].y, bq0[2 * i], bq1[2 * i]);
                mma_f16_16816(c, wa[i].z, wb[i].z, wa[i].w, wb[i].w, bq0[2 * i + 1], bq1[2 * i + 1]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mma_bf16_16816(c, ca[i].x, cb[i].x, ca[i].y, cb[i].y, bq0[2 * i], bq1[2 * i]);
                mma_bf16_16816(c, ca[i].z, cb[i].z, ca[i].w, cb[i].w, bq0[2 * i + 1], bq1[2 * i + 1]);
            }
        }
        // Lane t = 0 holds heads 0, 1 and lane t = 1 heads 2, 3 of rows g, g + 8.
        float sa = fmaxf(c[0], 0.f) + fmaxf(c[1], 0.f);
        float sb = fmaxf(c[2], 0.f) + fmaxf(c[3], 0.f);
        sa += __shfl_xor_sync(0xffffffffu, sa, 1);
        sb += __shfl_xor_sync(0xffffffffu, sb, 1);
        if constexpr (Q8) {
            sa *= psa;
            sb *= psb;
            psa = nsa;
            psb = nsb;
        }
        emit(base, sa, sb);
        if (listing) list(base, sa, sb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ca[i] = na[i];
            cb[i] = nb[i];
        }
    }
    finish();
}

template <bool Q8, bool STREAM>
__global__ void __launch_bounds__(DS_THREADS) decode_score_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, int kB, double eps, RopeTable rt,
    float* __restrict__ scores, uint32_t* __restrict__ hist_g, int32_t* __restrict__ status, Q8Caches q8,
    HotCache hot) {
    score_body<Q8, DS_WARPS, 0, STREAM>(nullptr, nullptr, nullptr, nullptr, pos, k, v, idx_q, idx_k, kc, vc,
                                        idx_k_cache, pooled, cap, rms_w, kv_heads, r, kB, eps, rt, scores, hist_g,
                                        status, q8, hot);
}

constexpr int SEL_E = 8;                 // scores per thread per round of the scan
constexpr int SEL_BITMAP_WORDS = 10240;  // ordered output by bitmap for up to 327680 blocks
static_assert(SEL_BITMAP_WORDS % (4 * 512) == 0, "T threads x 4-word multiples cover the bitmap exactly");

struct DecSelSmem {
    uint32_t hist[BINS];     // level-1, then level-2 histogram
    uint32_t cand_key[CAND]; // candidates (threshold digit): this CTA's, then all
    int32_t cand_idx[CAND];
    int32_t l3[T];           // candidate slots in the level-2 threshold bin
    union {
        int32_t out[kMaxKB];                // winners as a list
        uint32_t bitmap[SEL_BITMAP_WORDS];  // winners as a bitmap over the blocks
    } u;
    uint32_t wsum[NW];
    unsigned long long base;
    int32_t n_win, n_cand, n_l3, bin, above, last;
    uint32_t kth_key;  // key of the k_B-th selected block (0: not known)
};
static_assert(sizeof(SelSmem) <= sizeof(DecSelSmem), "the row-selection fallback reuses this shared memory");

// Exclusive prefix of v over the CTA in thread order; returns the total.
template <typename Sm>
__device__ __forceinline__ uint32_t cta_prefix(Sm& sm, uint32_t v, uint32_t& prefix) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) sm.wsum[w] = inc;
    __syncthreads();
    uint32_t base = 0, total = 0;
    for (int k = 0; k < NW; ++k) {
        const uint32_t x = sm.wsum[k];
        if (k < w) base += x;
        total += x;
    }
    __syncthreads();
    prefix = base + inc - v;
    return total;
}

// Warp-aggregated append of `value` to list[*count] (every lane calls it).
__device__ __forceinline__ void warp_append(int32_t* count, bool flag, int32_t* list, int32_t value, int cap) {
    const int lane = threadIdx.x & 31;
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    int base = 0;
    if (lane == 0 && bal) base = atomicAdd(count, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    const int at = base + __popc(bal & ((1u << lane) - 1u));
    if (flag && at < cap) list[at] = value;
}

// The sequence's histogram and counters back to zero for the next step.
__device__ __forceinline__ void reset_state(DecodeSelWs sw, int s) {
    for (int b = threadIdx.x; b < BINS; b += T) sw.hist[(size_t)s * BINS + b] = 0u;
    if (threadIdx.x < 4) sw.counters[s * 4 + threadIdx.x] = 0;
}

// Exact selection from the whole row (degenerate inputs only), in the last CTA.
__device__ __noinline__ void decode_select_fallback(uint8_t* raw, const float* row, int64_t nvis, int kB,
                                                    int32_t* out, int32_t* nsel_s) {
    select_row(*reinterpret_cast<SelSmem*>(raw), row, nvis, kB, out, nsel_s);
}

// The exact pick among the nc candidates (the level-1 threshold digit's
// blocks, need1 of them to be taken; in sm.cand_key / sm.cand_idx) with the
// sure winners already in the bitmap (use_bm) or in sm.u.out (sm.n_win of
// them), sm.hist zero and sm.n_l3 zero: a level-2 histogram on the next 11 key
// bits, a rank by (key descending, block ascending) inside the level-2
// threshold bin, then the k_B winners in ascending block order to out and
// *nsel_s. Ends with all the CTA's writes done.
__device__ __noinline__ void select_tail(uint8_t* raw, const float* row, int64_t nvis, int kB, int nc,
                                         uint32_t need1, bool use_bm, int per, int32_t* out, int32_t* nsel_s,
                                         int32_t* status) {
    DecSelSmem& sm = *reinterpret_cast<DecSelSmem*>(raw);
    const int tid = threadIdx.x;
    if (tid == 0) sm.kth_key = 0u;
    for (int c = tid; c < nc; c += T) atomicAdd(&sm.hist[dec_digit2(sm.cand_key[c])], 1u);
    find_bin(sm, BINS, need1);
    const uint32_t b2 = sm.bin;
    const uint32_t need2 = need1 - (uint32_t)sm.above;
    for (int c0 = 0; c0 < nc; c0 += T) {
        const int c = c0 + tid;
        const uint32_t d2 = c < nc ? dec_digit2(sm.cand_key[c]) : 0u;
        if (c < nc && d2 > b2) {
            const int32_t id = sm.cand_idx[c];
            if (use_bm) {
                atomicOr(&sm.u.bitmap[id >> 5], 1u << (id & 31));
            } else {
                const int at = atomicAdd(&sm.n_win, 1);
                if (at < kMaxKB) sm.u.out[at] = id;
            }
        }
        warp_append(&sm.n_l3, c < nc && d2 == b2, sm.l3, c, T);
    }
    __syncthreads();
    const int n3 = sm.n_l3;
    if (n3 > T) {  // thousands of equal keys
        __syncthreads();
        decode_select_fallback(raw, row, nvis, kB, out, nsel_s);
        __syncthreads();
        return;
    }
    if (tid < n3) {  // rank inside the level-2 threshold bin: (key desc, block asc)
        const int x = sm.l3[tid];
        const uint32_t kx = sm.cand_key[x];
        const int32_t ix = sm.cand_idx[x];
        uint32_t rk = 0;
        for (int u = 0; u < n3; ++u) {
            const int y = sm.l3[u];
            const uint32_t ky = sm.cand_key[y];
            rk += (ky > kx || (ky == kx && sm.cand_idx[y] < ix)) ? 1u : 0u;
        }
        if (rk + 1 == need2) sm.kth_key = kx;  // the last one taken: the k-th largest
        if (rk < need2) {
            if (use_bm) {
                atomicOr(&sm.u.bitmap[ix >> 5], 1u << (ix & 31));
            } else {
                const int at = atomicAdd(&sm.n_win, 1);
                if (at < kMaxKB) sm.u.out[at] = ix;
            }
        }
    }
    __syncthreads();
    if (use_bm) {
        // Ordered compaction: thread t owns words [t per, (t + 1) per), read
        // as 16-byte vectors.
        const int w0 = tid * per;
        uint32_t n = 0;
        for (int w = w0; w < w0 + per; w += 4) {
            const uint4 x = *reinterpret_cast<const uint4*>(&sm.u.bitmap[w]);
            n += __popc(x.x) + __popc(x.y) + __popc(x.z) + __popc(x.w);
        }
        uint32_t at;
        const uint32_t total = cta_prefix(sm, n, at);
        if (total != (uint32_t)kB && tid == 0) flag_status(status, 7 /* QSA_ERR_DEVICE_CHECK */);
        for (int w = w0; n && w < w0 + per; w += 4) {
            const uint4 x = *reinterpret_cast<const uint4*>(&sm.u.bitmap[w]);
            const uint32_t m4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t m = m4[j];
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    if (at < (uint32_t)kB) out[at] = (w + j) * 32 + bit;
                    ++at;
                }
            }
        }
    } else {
        if (sm.n_win != kB && tid == 0) flag_status(status, 7 /* QSA_ERR_DEVICE_CHECK */);
        sort_ints(sm.u.out, kB);
        for (int k2 = tid; k2 < kB; k2 += T) out[k2] = sm.u.out[k2];
    }
    if (tid == 0) *nsel_s = kB;
    __syncthreads();
}

// The decode selection (a5) of each sequence by X CTAs: every CTA reads the
// sequence's level-1 histogram (built by the score pass) and finds the
// threshold digit b1 with above(b1) < k_B <= above(b1) + hist[b1], scans its
// slice of the scores into shared-memory lists of sure winners (digit > b1)
// and candidates (digit == b1), reserves room in the sequence's global lists
// with one atomic and copies them there. The last CTA to finish resolves the
// exact pick among the candidates (a level-2 histogram on the next 11 key
// bits, then a rank by (key descending, block ascending) inside the level-2
// threshold bin) and writes the k_B winners in ascending block order through a
// bitmap over the blocks. The code is kept small and nearly barrier-free: it
// runs once per step on cold instruction caches.
//
// (The body, after the dependency wait; it returns true in the one CTA that
// wrote the sequence's selection, after all its threads' writes.)
__device__ __forceinline__ bool select_body(uint8_t* raw, const int64_t* __restrict__ pos, int64_t cap, int r,
                                            int kB, const float* __restrict__ scores, DecodeSelWs sw,
                                            int32_t* __restrict__ sel, int32_t* __restrict__ nsel,
                                            int32_t* __restrict__ status) {
    DecSelSmem& sm = *reinterpret_cast<DecSelSmem*>(raw);
    const int s = blockIdx.y, tid = threadIdx.x;
    const int64_t p = pos[s];  // an input of the step
    const int64_t nvis = (p >= 0 && p < cap) ? p / r : 0;
    int32_t* out = sel + (size_t)s * kB;
    if (nvis <= kB) {  // every visible block is selected
        if (blockIdx.x != 0) return false;
        for (int k2 = tid; k2 < kB; k2 += T) out[k2] = k2 < nvis ? k2 : -1;
        if (tid == 0) nsel[s] = (int32_t)nvis;
        __syncthreads();
        return true;
    }
    const float* row = scores + (size_t)s * (cap / r);
    reinterpret_cast<uint4*>(sm.hist)[tid] = __ldcg(reinterpret_cast<const uint4*>(sw.hist + (size_t)s * BINS) + tid);
    if (tid == 0) {
        sm.n_win = 0;
        sm.n_cand = 0;
        sm.n_l3 = 0;
    }
    find_bin(sm, BINS, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;

    // Scan this CTA's slice; hits are rare, so their appends sit behind a vote.
    int64_t lo, hi;
    cta_range(nvis, blockIdx.x, gridDim.x, lo, hi);
    for (int64_t r0 = lo; r0 < hi; r0 += (int64_t)SEL_E * T) {
        uint32_t key[SEL_E];
#pragma unroll
        for (int e = 0; e < SEL_E; ++e) {
            const int64_t b = r0 + (int64_t)e * T + tid;
            key[e] = b < hi ? float_key(__ldcg(row + b)) : 0u;
        }
#pragma unroll
        for (int e = 0; e < SEL_E; ++e) {
            const int64_t b = r0 + (int64_t)e * T + tid;
            const uint32_t d = dec_digit1(key[e]);
            const bool w = b < hi && d > b1, c = b < hi && d == b1;
            if (__any_sync(0xffffffffu, w || c)) {
                warp_append(&sm.n_win, w, sm.u.out, (int32_t)b, kMaxKB);
                const uint32_t bal = __ballot_sync(0xffffffffu, c);
                int cb = 0;
                if ((tid & 31) == 0 && bal) cb = atomicAdd(&sm.n_cand, __popc(bal));
                cb = __shfl_sync(0xffffffffu, cb, 0) + __popc(bal & ((1u << (tid & 31)) - 1u));
                if (c && cb < CAND) {
                    sm.cand_key[cb] = key[e];
                    sm.cand_idx[cb] = (int32_t)b;
                }
            }
        }
    }
    __syncthreads();
    int32_t* cnt = sw.counters + s * 4;  // [0] sure winners, [1] candidates, [2] finished CTAs
    if (tid == 0) {
        const unsigned long long add = ((unsigned long long)(uint32_t)sm.n_cand << 32) | (uint32_t)sm.n_win;
        sm.base = add ? atomicAdd(reinterpret_cast<unsigned long long*>(cnt), add) : 0ull;
    }
    __syncthreads();
    {
        const int wb = (int)(uint32_t)sm.base, cb = (int)(uint32_t)(sm.base >> 32);
        const int nw = sm.n_win, nc = min(sm.n_cand, CAND);
        int32_t* winners = sw.winners + (size_t)s * kB;
        uint2* cand = sw.cand + (size_t)s * kDecodeCand;
        for (int k = tid; k < nw; k += T)
            if (wb + k < kB) winners[wb + k] = sm.u.out[k];  // (< k_B by the histogram)
        for (int k = tid; k < nc; k += T)
            if (cb + k < kDecodeCand) cand[cb + k] = make_uint2(sm.cand_key[k], (uint32_t)sm.cand_idx[k]);
    }
    __syncthreads();
    if (tid == 0) sm.last = atom_add_acq_rel(cnt + 2, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!sm.last) return false;

    // ---- the last CTA of the sequence (it acquired every CTA's lists) ----
    if (tid == 0) sm.kth_key = 0u;
    const int n_win = __ldcg(cnt + 0), nc = __ldcg(cnt + 1);
    if (b1 == 0u || nc > kDecodeCand || nc > CAND || n_win != kB - (int)need1) {
        __syncthreads();
        decode_select_fallback(raw, row, nvis, kB, out, nsel + s);
        __syncthreads();
        reset_state(sw, s);
        __syncthreads();
        return true;
    }
    const bool use_bm = nvis <= (int64_t)SEL_BITMAP_WORDS * 32;
    const int words = use_bm ? (int)((nvis + 31) / 32) : 0;
    // Bitmap words per thread for the ordered output, a multiple of 4 (read as
    // 16-byte vectors); every word a thread reads is cleared here.
    const int per = (((words + T - 1) / T) + 3) & ~3;
    for (int b = tid; b < BINS; b += T) sm.hist[b] = 0u;
    for (int w = tid; w < T * per; w += T) sm.u.bitmap[w] = 0u;
    if (tid == 0) {
        sm.n_l3 = 0;
        sm.n_win = n_win;
    }
    const uint2* cand = sw.cand + (size_t)s * kDecodeCand;
    for (int c = tid; c < nc; c += T) {
        const uint2 e = __ldcg(cand + c);
        sm.cand_key[c] = e.x;
        sm.cand_idx[c] = (int32_t)e.y;
    }
    __syncthreads();
    const int32_t* winners = sw.winners + (size_t)s * kB;
    for (int k = tid; k < n_win; k += T) {
        const int32_t id = __ldcg(winners + k);
        if (use_bm)
            atomicOr(&sm.u.bitmap[id >> 5], 1u << (id & 31));
        else
            sm.u.out[k] = id;
    }
    select_tail(raw, row, nvis, kB, nc, need1, use_bm, per, out, nsel + s, status);
    reset_state(sw, s);
    __syncthreads();
    return true;
}

// The pre-filter estimate for the sequence's next step: this step's k-th
// largest score (sm.kth_key, left by select_tail) per unit of this step's
// summed indexer-query head norms; zero (no list next step) unless both are
// positive. Thread 0 only.
__device__ __forceinline__ void record_estimate(const DecSelSmem& sm, float2* est) {
    const uint32_t key = sm.kth_key;
    const float kth = __uint_as_float(key & 0x80000000u ? key & 0x7fffffffu : ~key);  // (float_key inverted)
    const float y = __ldcg(&est->y);
    est->x = (key != 0u && kth > 0.f && kth < INFINITY && y > 0.f) ? kth / y : 0.f;
}

constexpr int kListPerThread = kDecodePre / T;  // listed entries a thread of select_listed holds
static_assert(kListPerThread * T == kDecodePre, "select_listed holds the whole list in registers");

// The exact pick from the npre >= k_B listed blocks (every block at or above
// the score pass's threshold, hence every top-k_B block), by one CTA: a
// level-1 histogram of their keys' top digits, the sure winners above the
// threshold digit, that digit's blocks as the candidates, then select_tail.
// Returns false, having written nothing, when the candidates do not fit.
__device__ __noinline__ bool select_listed(uint8_t* raw, const float* row, int64_t nvis, int kB, int npre,
                                           const uint2* pre, int32_t* out, int32_t* nsel_s, int32_t* status) {
    DecSelSmem& sm = *reinterpret_cast<DecSelSmem*>(raw);
    const int tid = threadIdx.x, lane = tid & 31;
    for (int b = tid; b < BINS; b += T) sm.hist[b] = 0u;
    if (tid == 0) {
        sm.n_win = 0;
        sm.n_cand = 0;
        sm.n_l3 = 0;
    }
    // The list (npre <= T x kListPerThread) in registers: all loads in flight at once.
    uint2 e[kListPerThread];
#pragma unroll
    for (int j = 0; j < kListPerThread; ++j) {
        const int i = tid + j * T;
        e[j] = i < npre ? __ldcg(pre + i) : make_uint2(0u, 0u);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kListPerThread; ++j)
        if (tid + j * T < npre) atomicAdd(&sm.hist[dec_digit1(e[j].x)], 1u);
    find_bin(sm, BINS, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;
    const bool use_bm = nvis <= (int64_t)SEL_BITMAP_WORDS * 32;
    const int words = use_bm ? (int)((nvis + 31) / 32) : 0;
    const int per = (((words + T - 1) / T) + 3) & ~3;
    for (int b = tid; b < BINS; b += T) sm.hist[b] = 0u;
    for (int w = tid; w < T * per; w += T) sm.u.bitmap[w] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kListPerThread; ++j) {
        const int i = tid + j * T;
        const uint32_t d = dec_digit1(e[j].x);
        const bool w = i < npre && d > b1, c = i < npre && d == b1;
        if (w && use_bm) atomicOr(&sm.u.bitmap[e[j].y >> 5], 1u << (e[j].y & 31));
        warp_append(&sm.n_win, w, sm.u.out, (int32_t)e[j].y, use_bm ? 0 : kMaxKB);  // (cap 0: count only)
        const uint32_t bal = __ballot_sync(0xffffffffu, c);
        int cb = 0;
        if (lane == 0 && bal) cb = atomicAdd(&sm.n_cand, __popc(bal));
        cb = __shfl_sync(0xffffffffu, cb, 0) + __popc(bal & ((1u << lane) - 1u));
        if (c && cb < CAND) {
            sm.cand_key[cb] = e[j].x;
            sm.cand_idx[cb] = (int32_t)e[j].y;
        }
    }
    __syncthreads();
    const int nc = sm.n_cand;
    const bool fits = b1 != 0u && nc <= CAND && sm.n_win == kB - (int)need1;
    __syncthreads();
    if (!fits) return false;
    select_tail(raw, row, nvis, kB, nc, need1, use_bm, per, out, nsel_s, status);
    return true;
}

__global__ void __launch_bounds__(T) decode_select_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int r, int kB, const float* __restrict__ scores,
    DecodeSelWs sw, int32_t* __restrict__ sel, int32_t* __restrict__ nsel, int32_t* __restrict__ status) {
    extern __shared__ __align__(16) uint8_t raw[];
    pdl_wait();
    pdl_trigger();
    select_body(raw, pos, cap, r, kB, scores, sw, sel, nsel, status);
}

// ---------------------------------------------------------------------------
// The decode step as one persistent kernel: grid (X, batch) of 512-thread
// CTAs, one per SM, with the X CTAs of a sequence running its three phases
// back to back and meeting only through counters in the workspace.
//   1. a8, a3', a4: the score body above (CTA 0 appends and pools, the others
//      score their slices and add their histogram counts).
//   2. a5: each CTA arrives at the sequence's counter and waits for all X, so
//      the histogram is complete; then the selection body above (every CTA
//      scans its slice; the last to finish resolves the pick), whose resolver
//      publishes the selection with a release store of the ready flag.
//   3. a6, a7: after an acquire of the ready flag, CTA x takes kv head
//      x % kv_heads and split x / kv_heads (at most kStepSplitCap splits per
//      head); its first FA_WARPS warps attend their slices of the k_B + 1
//      units (the selection entries, then the tail), their states are merged
//      in shared memory into the CTA's partial (o, m, l) in the workspace, and
//      the last split of a head to finish combines the partials into the
//      output rows.
// A sequence's CTAs only ever wait for each other, and all of them are
// resident at once when batch x X CTAs fit on the GPU (X is chosen so); with
// X = 1 nothing waits at all. Every wait is bounded by %globaltimer: one that
// runs out flags QSA_ERR_TIMEOUT, and the CTA skips the rest of the step.
constexpr int FS_WARPS = T / 32;  // warps of a step CTA: the score stream and the selection
constexpr int FA_WARPS = 12;      // of which attend (each owns a WARP_SMEM ring)
constexpr uint64_t kStepWaitNs = 10000000000ull;  // 10 s: the bound of every wait in normal use



// Thread 0 waits (bounded) until *p >= target (acquire); every thread gets
// the value it read, or 0 (and QSA_ERR_TIMEOUT flagged) when the wait ran out.
__device__ int cta_wait_at_least(const int32_t* p, int target, uint64_t wait_ns, int* flag, int32_t* status) {
    if (threadIdx.x == 0) {
        int v = ld_acquire(p);
        if (v < target) {
            const uint64_t t0 = global_ns();
            while ((v = ld_acquire(p)) < target && global_ns() - t0 < wait_ns) __nanosleep(100);
        }
        if (v < target) {
            flag_status(status, 6 /* QSA_ERR_TIMEOUT */);
            v = 0;
        }
        *flag = v;
    }
    __syncthreads();
    const int v = *flag;
    __syncthreads();
    return v;
}

// One warp's slice [split of S] of the units of (sequence s, kv head g),
// attended and stored head-major at wsm (o[G][128], m[G], l[G]).
template <int NT, bool Q8, bool HOT>
__device__ __forceinline__ void attend_slice(uint8_t* wsm, int lane, int s, int g, int split, int S, int64_t p,
                                             const uint16_t* __restrict__ q, const void* kc, const void* vc,
                                             const float* ks, const float* vs, int64_t cap,
                                             const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel,
                                             int q_heads, int kv_heads, int r, int kB, float scale_log2,
                                             const HotCache& hot) {
    const int G = q_heads / kv_heads;
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
    w.cur = p / r;
    w.i = p;
    uint32_t qb[NT][8][2];
    if (Q8)
        load_q_frags_f16<NT>(w.q, G, lane, qb);
    else
        load_q_frags<NT>(w.q, G, lane, qb);
    const int u_sel = w.u0 + lane;
    const int32_t sel_lane = (u_sel < w.u1 && u_sel < kB) ? __ldcg(w.sel + u_sel) : -1;
    int ns = __ldcg(nsel + s);
    w.nsel = ns < 0 ? 0 : (ns > kB ? kB : ns);
    if (p < 0 || p >= cap) w.u1 = w.u0;  // skipped sequence: zero output
    int32_t hot_lane = -1;
    if (HOT) {
        if (sel_lane >= 0) {
            const int32_t slot = sel_lane % w.hot_blocks;
            if (__ldcg(w.tags + slot) == sel_lane) hot_lane = slot;
        }
        if (__ldcg(w.tags + w.hot_blocks) == (int32_t)w.cur) w.tail_hrow0 = w.hot_blocks * r;
    }
    WarpState<NT> st;
    warp_attend<NT, Q8, HOT>(w, wsm, lane, qb, sel_lane, st, hot_lane);
    store_state_hd<NT>(st, G, reinterpret_cast<float*>(wsm), lane);
}

template <int NT, bool Q8, bool HOT>
__global__ void __launch_bounds__(T, 1) decode_step_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const uint16_t* __restrict__ v, const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k,
    uint16_t* __restrict__ kc, uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache,
    uint16_t* __restrict__ pooled, int64_t cap, const float* __restrict__ rms_w, int q_heads, int kv_heads, int r,
    int kB, double eps, RopeTable rt, float scale_log2, float* __restrict__ scores, DecodeSelWs sw, StepSync sy,
    int32_t* __restrict__ sel, int32_t* __restrict__ nsel, uint16_t* __restrict__ out, int32_t* __restrict__ status,
    Q8Caches q8, HotCache hot) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ int s_wait, s_done;  // (each written by thread 0, read by all after a barrier)
    const int s = blockIdx.y, x = blockIdx.x, X = (int)gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // 1. Append, rotate, score this CTA's slice, count its histogram digits.
    score_body<Q8, FS_WARPS, kScoreRing>(dsm, sw.est, sw.pre, sw.counters + 4 * s + 3, pos, k, v, idx_q, idx_k, kc,
                                         vc, idx_k_cache, pooled, cap, rms_w, kv_heads, r, kB, eps, rt, scores,
                                         sw.hist, status, q8, hot);
    const int64_t p = pos[s];
    const int64_t nvis = (p >= 0 && p < cap) ? p / r : 0;
    const float* row = scores + (size_t)s * (cap / r);
    int32_t* cnt = sw.counters + 4 * s;
    // 2. The selection. ready: 1 = picked from the listed blocks (or every
    // block is visible and selected), 2 = the full selection is needed, 3 =
    // picked by the full selection.
    int ready;
    if (nvis > kB) {
        // The scoring CTAs arrive; CTA 0 (it scores only when alone) waits for
        // them and picks from the list when it holds the answer, else asks
        // every CTA for the full selection. (CTA 0 of every step is the same
        // kind of CTA, so the pick's code tends to be warm in its caches.)
        __syncthreads();
        if (x > 0 && tid == 0 && !(sy.inject && s == 0 && x == X - 1)) red_add_release(sy.arrive + s, 1);
        if (x == 0 && (X == 1 || cta_wait_at_least(sy.arrive + s, X - 1, sy.wait_ns, &s_wait, status))) {
            const int npre = __ldcg(cnt + 3);
            bool picked = false;
            if (npre >= kB && npre <= kDecodePre)
                picked = select_listed(dsm, row, nvis, kB, npre, sw.pre + (size_t)s * kDecodePre, sel + (size_t)s * kB,
                                       nsel + s, status);
            if (picked) {
                if (tid == 0) {
                    record_estimate(*reinterpret_cast<const DecSelSmem*>(dsm), sw.est + s);
                    cnt[3] = 0;  // (the other counters are untouched: zero)
                }
                for (int b = tid; b < BINS; b += T) sw.hist[(size_t)s * BINS + b] = 0u;
                __syncthreads();
            }
            if (tid == 0) st_release(sy.ready + s, picked ? 1 : 2);
        }
        ready = cta_wait_at_least(sy.ready + s, 1, sy.wait_ns, &s_wait, status);
        if (ready == 2) {  // every CTA scans its slice; the last to finish resolves
            if (select_body(dsm, pos, cap, r, kB, scores, sw, sel, nsel, status)) {
                if (tid == 0) {
                    record_estimate(*reinterpret_cast<const DecSelSmem*>(dsm), sw.est + s);
                    st_release(sy.ready + s, 3);
                }
            }
            __syncthreads();
            ready = cta_wait_at_least(sy.ready + s, 3, sy.wait_ns, &s_wait, status);
        }
    } else {
        if (select_body(dsm, pos, cap, r, kB, scores, sw, sel, nsel, status) && tid == 0)
            st_release(sy.ready + s, 1);  // (CTA 0: every visible block)
        __syncthreads();
        ready = cta_wait_at_least(sy.ready + s, 1, sy.wait_ns, &s_wait, status);
    }
    bool ok = ready == 1 || ready == 3;
    __syncthreads();  // (the selection's shared memory is free again)

    // 3. The attention, split over the sequence's CTAs, and the combine.
    const int G = q_heads / kv_heads, E = G * kHeadDim, PW = E + 2 * G;
    const int xg = max(1, min(kStepSplitCap, X / kv_heads));  // splits (CTAs) per kv head
    const int tasks = kv_heads * xg;
    const void* kv_k = Q8 ? (const void*)q8.k8 : (const void*)kc;
    const void* kv_v = Q8 ? (const void*)q8.v8 : (const void*)vc;
    for (int t = x; ok && t < tasks; t += X) {
        const int g = t % kv_heads, j = t / kv_heads;
        if (warp < FA_WARPS)
            attend_slice<NT, Q8, HOT>(dsm + warp * WARP_SMEM, lane, s, g, j * FA_WARPS + warp, xg * FA_WARPS, p, q,
                                      kv_k, kv_v, q8.ks, q8.vs, cap, sel, nsel, q_heads, kv_heads, r, kB, scale_log2,
                                      hot);
        __syncthreads();
        // The FA_WARPS warp states merged into this split's partial.
        float* part = sy.part + ((size_t)(s * kv_heads + g) * kStepSplitCap + j) * PW;
        for (int e = tid; e < E + G; e += T) {
            const int h = e < E ? e / kHeadDim : e - E;
            float M = -INFINITY;
#pragma unroll
            for (int w2 = 0; w2 < FA_WARPS; ++w2)
                M = fmaxf(M, reinterpret_cast<const float*>(dsm + w2 * WARP_SMEM)[E + h]);
            float acc = 0.f;
            const int src = e < E ? e : E + G + h;  // o element, or the head's l
#pragma unroll
            for (int w2 = 0; w2 < FA_WARPS; ++w2) {
                const float* ws = reinterpret_cast<const float*>(dsm + w2 * WARP_SMEM);
                acc = fmaf(ws[src], M == -INFINITY ? 0.f : exp2f(ws[E + h] - M), acc);
            }
            if (e < E) {
                part[e] = acc;
            } else {
                part[E + h] = M;
                part[E + G + h] = acc;
            }
        }
        __syncthreads();
        if (tid == 0) s_done = atom_add_acq_rel(sy.done + s * kv_heads + g, 1) == xg - 1;
        __syncthreads();
        if (s_done) {  // the last split of this kv head: combine all xg partials
            const float* base = sy.part + (size_t)(s * kv_heads + g) * kStepSplitCap * PW;
            uint16_t* orow = out + ((size_t)s * q_heads + (size_t)g * G) * kHeadDim;
            for (int e = tid; e < E; e += T) {
                const int h = e / kHeadDim;
                // Every split's (m, l, o) loaded at once (one round trip), then combined.
                float mj[kStepSplitCap], lj[kStepSplitCap], oj[kStepSplitCap];
#pragma unroll
                for (int jj = 0; jj < kStepSplitCap; ++jj) {
                    const bool in = jj < xg;
                    mj[jj] = in ? __ldcg(base + jj * PW + E + h) : -INFINITY;
                    lj[jj] = in ? __ldcg(base + jj * PW + E + G + h) : 0.f;
                    oj[jj] = in ? __ldcg(base + jj * PW + e) : 0.f;
                }
                float M = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < kStepSplitCap; ++jj) M = fmaxf(M, mj[jj]);
                float num = 0.f, den = 0.f;
#pragma unroll
                for (int jj = 0; jj < kStepSplitCap; ++jj) {
                    const float c = M == -INFINITY ? 0.f : exp2f(mj[jj] - M);
                    num = fmaf(oj[jj], c, num);
                    den = fmaf(lj[jj], c, den);
                }
                orow[e] = f32_to_bf16(den > 0.f ? num / den : 0.f);
            }
        }
        __syncthreads();  // (the rings are reused by the next task)
    }

    // The sequence's step state back to zero, by its last CTA.
    if (tid == 0) {
        if (atom_add_acq_rel(sy.fin + s, 1) == X - 1) {
            sy.arrive[s] = 0;
            sy.ready[s] = 0;
            for (int g = 0; g < kv_heads; ++g) sy.done[s * kv_heads + g] = 0;
            sy.fin[s] = 0;
        }
    }
}

}  // namespace

// CTAs per sequence of the decode selection: one wave over the batch, on the
// current device (each device's figure is computed once).
int decode_select_ctas(int batch) {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cached[kMaxDev];  // 0: not yet known
    int dev = 0;
    cudaGetDevice(&dev);
    int wave = (dev >= 0 && dev < kMaxDev) ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (wave <= 0) {
        const int smem = (int)sizeof(DecSelSmem);
        cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        int sms = 148, per_sm = 1;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_select_kernel, T, smem) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        wave = sms * per_sm;
        if (dev >= 0 && dev < kMaxDev) cached[dev].store(wave, std::memory_order_relaxed);
    }
    return std::max(1, wave / std::max(batch, 1));
}

// One wave: as many CTAs as fit on the GPU at once, split over the batch.
// CTAs per sequence: one wave of the variant that runs (the bf16 and fp8
// variants use different register counts, so their occupancies differ).
int decode_score_ctas(int batch, bool q8) {
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const cudaError_t e = q8 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_score_kernel<true, true>,
                                                                             DS_THREADS, 0)
                             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_score_kernel<false, true>,
                                                                             DS_THREADS, 0);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    return std::max(1, per_sm * sms / std::max(batch, 1));
}

// Pooled-key bytes of a batch at its capacity above which the score stream
// reads them as a stream (evict-first) rather than letting them stay in L2.
constexpr double kStreamKeyBytes = 96e6;

cudaError_t launch_decode_score(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* k,
                                const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                                uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled,
                                int64_t cap, const float* rms_w, float* scores, DecodeSelWs sw,
                                int32_t* status, const Q8Caches* q8, const HotCache* hot, cudaStream_t st) {
    const dim3 grid((unsigned)decode_score_ctas(batch, q8 != nullptr), (unsigned)batch);
    const bool stream = (double)batch * (double)(cap / L.r) * kIdxDim * (q8 ? 1 : 2) > kStreamKeyBytes;
    note_launch();
#define QSA_SCORE(Q8_, S_, Q8C_, HOT_)                                                                                \
    launch_pdl(decode_score_kernel<Q8_, S_>, grid, dim3(DS_THREADS), 0, st, pos, k, v, idx_q, idx_k, kc, vc,          \
               idx_k_cache, pooled, cap, rms_w, L.kv_heads, L.r, L.kB, L.rms_eps, L.rope, scores, sw.hist, status,    \
               Q8C_, HOT_)
    const HotCache hc = hot ? *hot : HotCache{};
    if (q8) return stream ? QSA_SCORE(true, true, *q8, HotCache{}) : QSA_SCORE(true, false, *q8, HotCache{});
    return stream ? QSA_SCORE(false, true, Q8Caches{}, hc) : QSA_SCORE(false, false, Q8Caches{}, hc);
#undef QSA_SCORE
}

cudaError_t launch_decode_select(const LayerDims& L, int batch, const int64_t* pos, int64_t cap,
                                 const float* scores, DecodeSelWs sw, int32_t* sel, int32_t* nsel,
                                 int32_t* status, cudaStream_t st) {
    const int smem = (int)sizeof(DecSelSmem);
    const int X = decode_select_ctas(batch);
    cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch();
    return launch_pdl(decode_select_kernel, dim3((unsigned)X, (unsigned)batch), dim3(T), (size_t)smem, st, pos, cap,
                      L.r, L.kB, scores, sw, sel, nsel, status);
}

// The step kernel takes G <= 8 query heads per kv head (one n8 tile of heads,
// within the register budget of a 512-thread CTA).
bool decode_step_supported(const LayerDims& L) { return L.q_heads / L.kv_heads <= 8; }

namespace {
std::atomic<int> g_step_fault_mode{0};
std::atomic<uint64_t> g_step_fault_wait_ns{kStepWaitNs};

constexpr size_t kStepSmem = std::max(std::max(sizeof(DecSelSmem), (size_t)FA_WARPS * WARP_SMEM),
                                      (size_t)FS_WARPS * kScoreRing * 4096 + kCtaList * sizeof(uint2));

template <bool Q8, bool HOT>
int step_ctas_per_sm() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cached[kMaxDev];  // 0: not yet known
    int dev = 0;
    cudaGetDevice(&dev);
    int per = (dev >= 0 && dev < kMaxDev) ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (per <= 0) {
        auto kern = decode_step_kernel<1, Q8, HOT>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStepSmem);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, T, kStepSmem) != cudaSuccess || per < 1) {
            cudaGetLastError();
            per = 1;
        }
        if (dev >= 0 && dev < kMaxDev) cached[dev].store(per, std::memory_order_relaxed);
    }
    return per;
}
}  // namespace

void set_decode_fault_injection(int mode, uint64_t wait_ns) {
    g_step_fault_wait_ns.store(mode ? wait_ns : kStepWaitNs, std::memory_order_relaxed);
    g_step_fault_mode.store(mode, std::memory_order_relaxed);
}

cudaError_t launch_decode_step(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* q,
                               const uint16_t* k, const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                               uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled, int64_t cap,
                               const float* rms_w, float* scores, DecodeSelWs sw, StepSync sy, int32_t* sel,
                               int32_t* nsel, uint16_t* out, int32_t* status, const Q8Caches* q8,
                               const HotCache* hot, cudaStream_t st) {
    if (batch <= 0) return cudaSuccess;
    if (!decode_step_supported(L)) return cudaErrorNotSupported;
    const int mode = g_step_fault_mode.load(std::memory_order_relaxed);
    sy.inject = mode != 0;
    sy.wait_ns = g_step_fault_wait_ns.load(std::memory_order_relaxed);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per = q8 ? step_ctas_per_sm<true, false>() : hot ? step_ctas_per_sm<false, true>()
                                                               : step_ctas_per_sm<false, false>();
    // One wave: batch x X CTAs resident at once (X = 1 when the batch alone
    // fills the GPU; then no CTA waits for another).
    const int X = std::max(1, sms * per / batch);
    const dim3 grid((unsigned)X, (unsigned)batch);
    const HotCache hc = hot ? *hot : HotCache{nullptr, nullptr, nullptr, 1};
    const Q8Caches qc = q8 ? *q8 : Q8Caches{};
    const float scale_log2 = L.sm_scale * LOG2E;
#define QSA_STEP(Q8_, HOT_)                                                                                          \
    launch_pdl(decode_step_kernel<1, Q8_, HOT_>, grid, dim3(T), kStepSmem, st, pos, q, k, v, idx_q, idx_k, kc, vc,   \
               idx_k_cache, pooled, cap, rms_w, L.q_heads, L.kv_heads, L.r, L.kB, L.rms_eps, L.rope, scale_log2,     \
               scores, sw, sy, sel, nsel, out, status, qc, hc)
    note_launch();
    if (q8) return QSA_STEP(true, false);
    if (hot) return QSA_STEP(false, true);
    return QSA_STEP(false, false);
#undef QSA_STEP
}

}  // namespace qsa
