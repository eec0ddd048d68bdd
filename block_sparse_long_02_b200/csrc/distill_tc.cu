// Stage-1 distillation target on the 5th-generation tensor cores ("QSA (Qwen
// Sparse Attention)" concept page, "Native trainability via 2-stage continued
// pretraining", stage 1; the reading of the target is stated with
// launch_distill_target in kernels.h and in distill.cu).
//
// Two passes over the keys, each a tcgen05 kernel with the same roles: warp 0
// issues TMA tile loads (SWIZZLE_128B) into a 4-stage key ring, warp 1 issues
// tcgen05.mma (kind::f16, fp32 accumulators in TMEM, double-buffered against
// the epilogue) and warps 2-9 are the epilogue (two warps per TMEM lane
// quadrant, each taking half of the quadrant's columns).
//   distill_lse_kernel:  rows (M = 128) = the query heads of one kv head for
//     128 / G queries, columns (N = 128) = keys. Each epilogue thread owns one
//     (query, head) row for half the key columns and keeps a running sum of
//     exponentials of its logits over keys <= i (raising its reference maximum
//     only when a logit exceeds it by more than 2^8); the two halves merge
//     into the head's log-sum-exp, written to the workspace.
//   distill_pool_kernel: rows (M = 128) = keys, columns = (query, head) for
//     8 queries (16 when G = 1) and every head, one MMA per kv head. Each
//     thread owns one key and half of the queries: the head average of its
//     probabilities for a query is a sum over its own columns, the block
//     maximum a shuffle over
//     the r lanes of the block; the block values are written and summed, and
//     each row is normalised at the end.
// Every wait is bounded (10 s of %globaltimer); on expiry the kernel records
// QSA_ERR_TIMEOUT in the workspace status, drains its own copies and MMAs,
// frees TMEM and returns.
#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "tc.cuh"

namespace qsa {
namespace {

constexpr int TC_THREADS = 320;      // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int EPI = 256;             // epilogue threads: two warps per TMEM lane quadrant
constexpr int KT = 128;              // keys per tile
constexpr int HALF = 128 * 128;      // one 64-dim half of a 128-row bf16 tile
constexpr int TILE = 2 * HALF;       // 128 rows x 128 dims
constexpr int RING = 4;              // key-tile stages
constexpr uint64_t WAIT_NS = 10000000000ull;
constexpr float LOG2E_TC = 1.4426950408889634f;

struct Bars {
    uint64_t full[RING], empty[RING], q_full, acc_full[2], acc_empty[2], done;
    uint32_t tmem;
    int abort;
    float mass[16];
};

__device__ __forceinline__ uint32_t bar_s(const uint64_t& b) { return smem_u32(&b); }

__device__ __forceinline__ void init_bars(Bars& b) {
    for (int k = 0; k < RING; ++k) {
        tc::mbar_init(bar_s(b.full[k]), 1);
        tc::mbar_init(bar_s(b.empty[k]), 1);
    }
    tc::mbar_init(bar_s(b.q_full), 1);
    for (int h = 0; h < 2; ++h) {
        tc::mbar_init(bar_s(b.acc_full[h]), 1);
        tc::mbar_init(bar_s(b.acc_empty[h]), EPI / 32);
    }
    tc::mbar_init(bar_s(b.done), 1);
    b.abort = 0;
    for (int q = 0; q < 16; ++q) b.mass[q] = 0.f;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// After an abort: wait (bounded, ignoring the flag) for the copies this CTA
// issued and for its MMAs, so that no transfer lands after the CTA exits.
__device__ __forceinline__ void drain(Bars& b, int warp, int lane, const int (&issued)[RING]) {
    volatile int no_abort = 0;
    if (warp == 0 && lane == 0)
        for (int k = 0; k < RING; ++k)
            if (issued[k] >= 0) tc::mbar_wait(bar_s(b.full[k]), issued[k] & 1, &no_abort, WAIT_NS);
    if (warp == 1 && lane == 0) {
        tc::umma_commit(bar_s(b.done));
        tc::mbar_wait(bar_s(b.done), 0, &no_abort, WAIT_NS);
    }
}

template <int G>
__global__ void __launch_bounds__(TC_THREADS, 1) distill_lse_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int64_t q_begin, int64_t nq,
    int64_t cap, int batch, int q_heads, int kv_heads, float scale_log2, float* __restrict__ lse2_out,
    int32_t* __restrict__ status, uint64_t wait_ns, int fault_mode) {
    constexpr int QA = 128 / G;  // queries per tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t sQ = base_s, sK = base_s + TILE;
    Bars& bars = *reinterpret_cast<Bars*>(base + TILE + RING * TILE);
    volatile int* abort_flag = &bars.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Unit: deepest query tiles first (the most keys).
    const int64_t nqt = (nq + QA - 1) / QA;
    const int per = kv_heads * batch;
    const int64_t qt = nqt - 1 - (int64_t)blockIdx.x / per;
    const int g = (int)(blockIdx.x % per) % kv_heads;
    const int s = (int)(blockIdx.x % per) / kv_heads;
    const int64_t j0 = qt * QA;
    const int nrows = (int)(nq - j0 < QA ? nq - j0 : QA);
    const int64_t i_last = q_begin + j0 + nrows - 1;
    const int ntiles = (int)((i_last + KT) / KT);  // keys 0 .. i_last

    if (tid == 0) init_bars(bars);
    if (warp == 1) tc::tmem_alloc(smem_u32(&bars.tmem), 256);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars.tmem;
    int issued[RING];  // producer: last round issued on each stage (-1: none)
#pragma unroll
    for (int k = 0; k < RING; ++k) issued[k] = -1;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_expect_tx(bar_s(bars.q_full), TILE);
            for (int hf = 0; hf < 2; ++hf)
                tc::tma_load_3d(sQ + hf * HALF, &tm_q, bar_s(bars.q_full), hf * 64, g * G, (int)(s * nq + j0));
            const int kz0 = (int)(s * cap);
            for (int t = 0; t < ntiles; ++t) {
                const int stg = t % RING;
                if (!tc::mbar_wait(bar_s(bars.empty[stg]), ((t / RING) & 1) ^ 1, abort_flag, wait_ns)) break;
                if (fault_mode == 2) continue;  // tests of the failure path: the tile never arrives
                tc::mbar_expect_tx(bar_s(bars.full[stg]), TILE);
                for (int hf = 0; hf < 2; ++hf)
                    tc::tma_load_3d(sK + stg * TILE + hf * HALF, &tm_k, bar_s(bars.full[stg]), hf * 64, g,
                                    kz0 + t * KT);
                issued[stg] = t / RING;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID = tc::idesc_bf16(128, KT);
            bool ok = tc::mbar_wait(bar_s(bars.q_full), 0, abort_flag, wait_ns);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int stg = t % RING, buf = t & 1;
                if (!(ok = tc::mbar_wait(bar_s(bars.full[stg]), (t / RING) & 1, abort_flag, wait_ns))) break;
                if (!(ok = tc::mbar_wait(bar_s(bars.acc_empty[buf]), ((t >> 1) & 1) ^ 1, abort_flag, wait_ns)))
                    break;
                tc::fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
                    tc::umma_bf16(tmem + buf * KT, tc::desc_sw128(sQ + off), tc::desc_sw128(sK + stg * TILE + off),
                                  ID, kk > 0 ? 1u : 0u);
                }
                tc::umma_commit(bar_s(bars.acc_full[buf]));
                tc::umma_commit(bar_s(bars.empty[stg]));
            }
        }
    } else {
        // Epilogue: thread = TMEM lane = row (query qi, head h) of the tile; the
        // two warps of a quadrant take key columns [0, 64) and [64, 128).
        const int ew = warp - 2, hc = ew >> 2;
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const int qi = row / G, h = row % G;
        const bool live = qi < nrows;
        const int64_t i = q_begin + j0 + (live ? qi : 0);
        float m = -INFINITY, l = 0.f;
        for (int t = 0; t < ntiles; ++t) {
            const int buf = t & 1;
            const bool ok = __all_sync(0xffffffffu,
                                       tc::mbar_wait(bar_s(bars.acc_full[buf]), (t >> 1) & 1, abort_flag, wait_ns));
            if (!ok) break;
            tc::fence_after();
            constexpr int HC = KT / 2;
            float v[HC];
            const uint32_t a = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(buf * KT + hc * HC);
#pragma unroll
            for (int c = 0; c < HC / 16; ++c) tc::tmem_ld16(a + c * 16, v + c * 16);
            tc::tmem_wait_ld();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar_s(bars.acc_empty[buf]));
            const int64_t nvalid = i - ((int64_t)t * KT + hc * HC) + 1;  // columns whose key is <= i
            if (!live || nvalid <= 0) continue;
            float vmax = -INFINITY;
            if (nvalid >= HC) {
#pragma unroll
                for (int c = 0; c < HC; ++c) vmax = fmaxf(vmax, v[c]);
            } else {
#pragma unroll
                for (int c = 0; c < HC; ++c) {
                    v[c] = c < nvalid ? v[c] : -INFINITY;
                    vmax = fmaxf(vmax, v[c]);
                }
            }
            const float tmax = vmax * scale_log2;  // (the scale is positive)
            if (tmax > m + 8.f) {
                l *= ex2_approx(m - tmax);  // (0 while m is -inf)
                m = tmax;
            }
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int c = 0; c < HC; c += 2) {
                acc0 += ex2_approx(fmaf(v[c], scale_log2, -m));
                acc1 += ex2_approx(fmaf(v[c + 1], scale_log2, -m));
            }
            l += acc0 + acc1;
        }
        // Merge the two column halves of each row.
        __shared__ float red_m[128], red_l[128];
        if (hc == 1) {
            red_m[row] = m;
            red_l[row] = l;
        }
        tc::named_sync(1, EPI);
        if (hc == 0 && live && !*abort_flag) {
            const float m1 = red_m[row], l1 = red_l[row];
            const float mm = fmaxf(m, m1);
            const float ll = (m == -INFINITY ? 0.f : l * ex2_approx(m - mm)) +
                             (m1 == -INFINITY ? 0.f : l1 * ex2_approx(m1 - mm));
            lse2_out[((size_t)s * nq + (size_t)(j0 + qi)) * q_heads + (size_t)g * G + h] = mm + log2f(ll);
        }
    }

    if (!*abort_flag && warp == 0 && lane == 0)
        for (int k = 0; k < RING; ++k)  // the last commits on the ring land before shared memory goes away
            if (issued[k] >= 0) tc::mbar_wait(bar_s(bars.empty[k]), issued[k] & 1, abort_flag, wait_ns);
    if (*abort_flag) {
        if (tid == 0) flag_status(status, 6 /* QSA_ERR_TIMEOUT */);
        drain(bars, warp, lane, issued);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

template <int G>
__global__ void __launch_bounds__(TC_THREADS, 1) distill_pool_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int64_t q_begin, int64_t nq,
    int64_t cap, int batch, int q_heads, int kv_heads, int r, float scale_log2, const float* __restrict__ lse2,
    float* __restrict__ target, int64_t ld, int32_t* __restrict__ status, uint64_t wait_ns, int fault_mode) {
    constexpr int QB = G == 1 ? 16 : 8;  // queries per tile
    constexpr int NG = QB * G;           // columns per kv head (a multiple of 16)
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const int q_bytes = kv_heads * NG * 256;
    const uint32_t sQ = base_s, sK = base_s + q_bytes;
    float* lse_s = reinterpret_cast<float*>(base + q_bytes + RING * TILE);  // [QB][q_heads]
    Bars& bars = *reinterpret_cast<Bars*>(base + q_bytes + RING * TILE + QB * 32 * 4);
    volatile int* abort_flag = &bars.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NC = NG * kv_heads;                // accumulator columns per key tile
    const int bstride = NC <= 128 ? 128 : 256;  // TMEM columns per buffer

    const int64_t nqt = (nq + QB - 1) / QB;
    const int64_t qt = nqt - 1 - (int64_t)blockIdx.x / batch;
    const int s = (int)(blockIdx.x % batch);
    const int64_t j0 = qt * QB;
    const int nrows = (int)(nq - j0 < QB ? nq - j0 : QB);
    const int64_t nvis_max = (q_begin + j0 + nrows - 1) / r;
    const int ntiles = (int)((nvis_max * r + KT - 1) / KT);
    float* trow0 = target + ((size_t)s * nq + (size_t)j0) * ld;
    if (ntiles == 0) {  // no visible block for any query of the tile
        for (int q = 0; q < nrows; ++q)
            for (int64_t b = tid; b < ld; b += TC_THREADS) trow0[(size_t)q * ld + b] = 0.f;
        return;
    }

    if (tid == 0) init_bars(bars);
    if (warp == 1) tc::tmem_alloc(smem_u32(&bars.tmem), 2 * bstride);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars.tmem;
    int issued[RING];
#pragma unroll
    for (int k = 0; k < RING; ++k) issued[k] = -1;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_expect_tx(bar_s(bars.q_full), q_bytes);
            for (int gg = 0; gg < kv_heads; ++gg)
                for (int hf = 0; hf < 2; ++hf)
                    tc::tma_load_3d(sQ + gg * NG * 256 + hf * NG * 128, &tm_q, bar_s(bars.q_full), hf * 64, gg * G,
                                    (int)(s * nq + j0));
            const int kz0 = (int)(s * cap);
            for (int t = 0, idx = 0; t < ntiles; ++t)
                for (int gg = 0; gg < kv_heads; ++gg, ++idx) {
                    const int stg = idx % RING;
                    if (!tc::mbar_wait(bar_s(bars.empty[stg]), ((idx / RING) & 1) ^ 1, abort_flag, wait_ns)) {
                        t = ntiles;
                        break;
                    }
                    if (fault_mode == 2) continue;  // tests of the failure path: the tile never arrives
                    tc::mbar_expect_tx(bar_s(bars.full[stg]), TILE);
                    for (int hf = 0; hf < 2; ++hf)
                        tc::tma_load_3d(sK + stg * TILE + hf * HALF, &tm_k, bar_s(bars.full[stg]), hf * 64, gg,
                                        kz0 + t * KT);
                    issued[stg] = idx / RING;
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID = tc::idesc_bf16(128, NG);
            bool ok = tc::mbar_wait(bar_s(bars.q_full), 0, abort_flag, wait_ns);
            for (int t = 0, idx = 0; ok && t < ntiles; ++t) {
                const int buf = t & 1;
                if (!(ok = tc::mbar_wait(bar_s(bars.acc_empty[buf]), ((t >> 1) & 1) ^ 1, abort_flag, wait_ns)))
                    break;
                for (int gg = 0; gg < kv_heads; ++gg, ++idx) {
                    const int stg = idx % RING;
                    if (!(ok = tc::mbar_wait(bar_s(bars.full[stg]), (idx / RING) & 1, abort_flag, wait_ns))) break;
                    tc::fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t koff = (kk >> 2) * HALF + (kk & 3) * 32;
                        const uint32_t qoff = gg * NG * 256 + (kk >> 2) * NG * 128 + (kk & 3) * 32;
                        tc::umma_bf16(tmem + buf * bstride + gg * NG, tc::desc_sw128(sK + stg * TILE + koff),
                                      tc::desc_sw128(sQ + qoff), ID, kk > 0 ? 1u : 0u);
                    }
                    tc::umma_commit(bar_s(bars.empty[stg]));
                }
                if (!ok) break;
                tc::umma_commit(bar_s(bars.acc_full[buf]));
            }
        }
    } else {
        // Epilogue: thread = TMEM lane = key row of the tile; the two warps of a
        // quadrant take queries [0, QB / 2) and [QB / 2, QB).
        constexpr int QH = QB / 2;       // queries per thread
        constexpr int NH = QH * G;       // columns per kv head and thread (a multiple of 8)
        const int et = tid - 64, ew = warp - 2, qh = ew >> 2;
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        for (int x = et; x < QB * q_heads; x += EPI) {
            const int q = x / q_heads;
            lse_s[x] = q < nrows ? lse2[((size_t)s * nq + (size_t)(j0 + q)) * q_heads + x % q_heads] : 0.f;
        }
        int64_t nvis[QH];
        float mass[QH];
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            const int qq = qh * QH + q;
            nvis[q] = qq < nrows ? (q_begin + j0 + qq) / r : 0;
            mass[q] = 0.f;
        }
        tc::named_sync(1, EPI);
        const float inv_h = 1.f / (float)q_heads;
        for (int t = 0; t < ntiles; ++t) {
            const int buf = t & 1;
            const bool ok =
                __all_sync(0xffffffffu, tc::mbar_wait(bar_s(bars.acc_full[buf]), (t >> 1) & 1, abort_flag, wait_ns));
            if (!ok) break;
            tc::fence_after();
            float sum[QH];
#pragma unroll
            for (int q = 0; q < QH; ++q) sum[q] = 0.f;
            const uint32_t a = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(buf * bstride + qh * NH);
            for (int gg = 0; gg < kv_heads; ++gg) {
                float v[NH];
                if constexpr (NH % 16 == 0) {
#pragma unroll
                    for (int c = 0; c < NH / 16; ++c) tc::tmem_ld16(a + gg * NG + c * 16, v + c * 16);
                } else {
#pragma unroll
                    for (int c = 0; c < NH / 8; ++c) tc::tmem_ld8(a + gg * NG + c * 8, v + c * 8);
                }
                tc::tmem_wait_ld();
                const float* lg = lse_s + (qh * QH) * q_heads + gg * G;
#pragma unroll
                for (int c = 0; c < NH; ++c)
                    sum[c / G] += ex2_approx(fmaf(v[c], scale_log2, -lg[(c / G) * q_heads + c % G]));
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar_s(bars.acc_empty[buf]));
            const int64_t b = ((int64_t)t * KT + row) / r;
#pragma unroll
            for (int q = 0; q < QH; ++q) {
                const bool vis = b < nvis[q];
                float val = vis ? sum[q] * inv_h : -INFINITY;
                for (int o = 1; o < r; o <<= 1) val = fmaxf(val, __shfl_xor_sync(0xffffffffu, val, o));
                if (vis && (lane & (r - 1)) == 0) {
                    trow0[(size_t)(qh * QH + q) * ld + b] = val;
                    mass[q] += val;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            const float w = warp_sum(mass[q]);
            if (lane == 0) atomicAdd(&bars.mass[qh * QH + q], w);
        }
        tc::named_sync(1, EPI);
        if (!*abort_flag)
            for (int q = 0; q < nrows; ++q) {
                const float inv = bars.mass[q] > 0.f ? 1.f / bars.mass[q] : 0.f;
                const int64_t nv = (q_begin + j0 + q) / r;
                float* tr = trow0 + (size_t)q * ld;
                for (int64_t bb = et; bb < ld; bb += EPI) tr[bb] = bb < nv ? tr[bb] * inv : 0.f;
            }
    }

    if (!*abort_flag && warp == 0 && lane == 0)
        for (int k = 0; k < RING; ++k)  // the last commits on the ring land before shared memory goes away
            if (issued[k] >= 0) tc::mbar_wait(bar_s(bars.empty[k]), issued[k] & 1, abort_flag, wait_ns);
    if (*abort_flag) {
        if (tid == 0) flag_status(status, 6 /* QSA_ERR_TIMEOUT */);
        drain(bars, warp, lane, issued);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, 2 * bstride);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D bf16 map over [rows][mid][128] (row stride mid x 256 bytes), box
// 64 x box_mid x box_rows, 128-byte swizzle; out-of-range rows read as zero.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t mid, uint64_t rows, uint32_t box_mid,
                 uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, mid, rows};
    cuuint64_t strides[2] = {256, mid * 256};
    cuuint32_t box[3] = {64, box_mid, box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
cudaError_t launch_target_tc_g(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                               const uint16_t* kc, int64_t cap, float* target, int64_t ld, float* lse2,
                               int32_t* status, cudaStream_t st) {
    constexpr int QA = 128 / G, QB = G == 1 ? 16 : 8;
    CUtensorMap tq_a, tq_b, tk;
    if (!make_map_3d(&tq_a, q, L.q_heads, (uint64_t)batch * nq, G, QA) ||
        !make_map_3d(&tq_b, q, L.q_heads, (uint64_t)batch * nq, G, QB) ||
        !make_map_3d(&tk, kc, L.kv_heads, (uint64_t)batch * cap, 1, KT))
        return cudaErrorInvalidValue;
    const float sl2 = L.sm_scale * LOG2E_TC;
    const int smem_a = TILE + RING * TILE + (int)sizeof(Bars) + 1024;
    auto ka = distill_lse_kernel<G>;
    cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_a);
    const int64_t grid_a = ((nq + QA - 1) / QA) * L.kv_heads * batch;
    note_launch();
    const int fmode = g_fault_mode.load(std::memory_order_relaxed);
    const uint64_t wait_ns = fmode == 2 ? g_fault_wait_ns.load(std::memory_order_relaxed) : WAIT_NS;
    ka<<<(unsigned)grid_a, TC_THREADS, smem_a, st>>>(tq_a, tk, q_begin, nq, cap, batch, L.q_heads, L.kv_heads, sl2,
                                                     lse2, status, wait_ns, fmode);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int smem_b = L.kv_heads * QB * G * 256 + RING * TILE + QB * 32 * 4 + (int)sizeof(Bars) + 1024;
    auto kb = distill_pool_kernel<G>;
    cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_b);
    const int64_t grid_b = ((nq + QB - 1) / QB) * batch;
    note_launch();
    kb<<<(unsigned)grid_b, TC_THREADS, smem_b, st>>>(tq_b, tk, q_begin, nq, cap, batch, L.q_heads, L.kv_heads, L.r,
                                                     sl2, lse2, target, ld, status, wait_ns, fmode);
    return cudaGetLastError();
}

}  // namespace

size_t distill_target_ws_bytes(int batch, int64_t nq, int q_heads) {
    return (size_t)kWsHeader + (size_t)batch * (size_t)nq * (size_t)q_heads * sizeof(float);
}

cudaError_t launch_distill_target(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                  const uint16_t* kc, int64_t cap, float* target, int64_t ld, void* ws,
                                  cudaStream_t st) {
    if (batch <= 0 || nq <= 0) return cudaSuccess;
    int32_t* status = reinterpret_cast<int32_t*>(ws);
    float* lse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeader);
    switch (L.q_heads / L.kv_heads) {
        case 1: return launch_target_tc_g<1>(L, batch, q, q_begin, nq, kc, cap, target, ld, lse2, status, st);
        case 2: return launch_target_tc_g<2>(L, batch, q, q_begin, nq, kc, cap, target, ld, lse2, status, st);
        case 4: return launch_target_tc_g<4>(L, batch, q, q_begin, nq, kc, cap, target, ld, lse2, status, st);
        case 8: return launch_target_tc_g<8>(L, batch, q, q_begin, nq, kc, cap, target, ld, lse2, status, st);
        case 16: return launch_target_tc_g<16>(L, batch, q, q_begin, nq, kc, cap, target, ld, lse2, status, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qsa
