// Decode step pieces ("QSA (Qwen Sparse Attention)" concept page, (A)-(B), for
// one new token per sequence): a8 (cache append, block pooling) with a3' (query
// rotation), the a4 score stream over every pooled key of a sequence, and the
// a5 selection.
//
// The score stream is the hot spot: 256 bytes of pooled key per block and
// 4 x 128 multiply-adds, an L2/HBM stream spread over one wave of CTAs, each
// scoring its slice on the tensor cores (mma.sync) from 16-byte loads issued a
// group ahead. The same pass builds a per-sequence histogram of a level-1 key
// digit of the scores, so the selection reads the score row once more and never
// sorts it: one thread-block cluster per sequence finds the threshold digit,
// collects the sure winners and the threshold-digit candidates of each CTA's
// slice in shared memory, resolves the exact pick among all candidates over
// distributed shared memory (ties to the lower block index), and writes the
// k_B winners in ascending order.
#include <algorithm>
#include <atomic>

#include "kernels.h"
#include "rope.cuh"
#include "select.cuh"

namespace qsa {
namespace {

constexpr int DS_THREADS = 256;  // fused score CTAs
constexpr int DS_WARPS = DS_THREADS / 32;

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
template <bool Q8>
__global__ void __launch_bounds__(DS_THREADS) decode_score_kernel(
    const int64_t* __restrict__ pos, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ idx_q, const uint16_t* __restrict__ idx_k, uint16_t* __restrict__ kc,
    uint16_t* __restrict__ vc, uint16_t* __restrict__ idx_k_cache, uint16_t* __restrict__ pooled,
    int64_t cap, const float* __restrict__ rms_w, int kv_heads, int r, int kB, double eps, RopeTable rt,
    float* __restrict__ scores, uint32_t* __restrict__ hist_g, int32_t* __restrict__ status, Q8Caches q8,
    HotCache hot) {
    __shared__ uint32_t hist[2048];
    __shared__ __align__(16) uint16_t qs[kIdxHeads * kIdxDim];
    __shared__ double2 cs[kIdxDim / 2];  // (sin, cos) of the query position's angles
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
    auto load = [&](int64_t base, uint4 (&ra)[4], uint4 (&rb)[4], float& sa_, float& sb_) {
        const int64_t b0 = base + g, b1 = b0 + 8;
        if constexpr (Q8) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                ra[i] = b0 < hi ? __ldg(reinterpret_cast<const uint4*>(keys8 + (size_t)b0 * kIdxDim + 64 * i + 16 * t))
                                : make_uint4(0u, 0u, 0u, 0u);
                rb[i] = b1 < hi ? __ldg(reinterpret_cast<const uint4*>(keys8 + (size_t)b1 * kIdxDim + 64 * i + 16 * t))
                                : make_uint4(0u, 0u, 0u, 0u);
            }
            sa_ = (t == 0 && b0 < hi) ? __ldg(kscale + b0) : 0.f;
            sb_ = (t == 0 && b1 < hi) ? __ldg(kscale + b1) : 0.f;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ra[i] = b0 < hi ? __ldg(reinterpret_cast<const uint4*>(keys + (size_t)b0 * kIdxDim + 32 * i + 8 * t))
                                : make_uint4(0u, 0u, 0u, 0u);
                rb[i] = b1 < hi ? __ldg(reinterpret_cast<const uint4*>(keys + (size_t)b1 * kIdxDim + 32 * i + 8 * t))
                                : make_uint4(0u, 0u, 0u, 0u);
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
        if (t == 0) {
            const int64_t b0 = base + g, b1 = b0 + 8;
            if (b0 < hi) {
                dst[b0] = sa;
                atomicAdd(&hist[dec_digit1(float_key(sa))], 1u);
            }
            if (b1 < hi) {
                dst[b1] = sb;
                atomicAdd(&hist[dec_digit1(float_key(sb))], 1u);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ca[i] = na[i];
            cb[i] = nb[i];
        }
    }
    __syncthreads();
    for (int b = tid; b < 2048; b += DS_THREADS)
        if (hist[b]) atomicAdd(&hist_g[(size_t)s * 2048 + b], hist[b]);
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
__global__ void __launch_bounds__(T) decode_select_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int r, int kB, const float* __restrict__ scores,
    DecodeSelWs sw, int32_t* __restrict__ sel, int32_t* __restrict__ nsel, int32_t* __restrict__ status) {
    extern __shared__ __align__(16) uint8_t raw[];
    DecSelSmem& sm = *reinterpret_cast<DecSelSmem*>(raw);
    const int s = blockIdx.y, tid = threadIdx.x;
    const int64_t p = pos[s];  // an input of the step
    pdl_wait();
    pdl_trigger();
    const int64_t nvis = (p >= 0 && p < cap) ? p / r : 0;
    int32_t* out = sel + (size_t)s * kB;
    if (nvis <= kB) {  // every visible block is selected
        if (blockIdx.x == 0) {
            for (int k2 = tid; k2 < kB; k2 += T) out[k2] = k2 < nvis ? k2 : -1;
            if (tid == 0) nsel[s] = (int32_t)nvis;
        }
        return;
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
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = atomicAdd(cnt + 2, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!sm.last) return;

    // ---- the last CTA of the sequence ----
    __threadfence();
    const int n_win = __ldcg(cnt + 0), nc = __ldcg(cnt + 1);
    if (b1 == 0u || nc > kDecodeCand || nc > CAND || n_win != kB - (int)need1) {
        __syncthreads();
        decode_select_fallback(raw, row, nvis, kB, out, nsel + s);
        __syncthreads();
        reset_state(sw, s);
        return;
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
        decode_select_fallback(raw, row, nvis, kB, out, nsel + s);
        __syncthreads();
        reset_state(sw, s);
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
    if (tid == 0) nsel[s] = kB;
    reset_state(sw, s);
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
    const cudaError_t e = q8 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_score_kernel<true>,
                                                                             DS_THREADS, 0)
                             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_score_kernel<false>,
                                                                             DS_THREADS, 0);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    return std::max(1, per_sm * sms / std::max(batch, 1));
}

cudaError_t launch_decode_score(const LayerDims& L, int batch, const int64_t* pos, const uint16_t* k,
                                const uint16_t* v, const uint16_t* idx_q, const uint16_t* idx_k,
                                uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache, uint16_t* pooled,
                                int64_t cap, const float* rms_w, float* scores, DecodeSelWs sw,
                                int32_t* status, const Q8Caches* q8, const HotCache* hot, cudaStream_t st) {
    const dim3 grid((unsigned)decode_score_ctas(batch, q8 != nullptr), (unsigned)batch);
    if (q8)
        return launch_pdl(decode_score_kernel<true>, grid, dim3(DS_THREADS), 0, st, pos, k, v, idx_q, idx_k, kc, vc,
                          idx_k_cache, pooled, cap, rms_w, L.kv_heads, L.r, L.kB, L.rms_eps, L.rope, scores, sw.hist,
                          status, *q8, HotCache{});
    return launch_pdl(decode_score_kernel<false>, grid, dim3(DS_THREADS), 0, st, pos, k, v, idx_q, idx_k, kc, vc,
                      idx_k_cache, pooled, cap, rms_w, L.kv_heads, L.r, L.kB, L.rms_eps, L.rope, scores, sw.hist,
                      status, Q8Caches{}, hot ? *hot : HotCache{});
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

}  // namespace qsa
