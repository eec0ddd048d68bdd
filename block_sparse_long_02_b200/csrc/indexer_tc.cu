// Fused prefill indexer: a3'..a5 ("QSA (Qwen Sparse Attention)" concept page,
// (A) block importance I_ib = sum_h ReLU(<q_i^h, k_b>) under block-causal
// masking, then top-k_B; "Qwen Sparse Attention" gallery page pseudo-code
// scores = sum(relu(query_head @ block_key)), top_k(scores, k=512)).
//
// The score matrix (1.4e11 entries at 1M tokens) is never materialised. One
// persistent CTA per SM owns a tile of 128 consecutive queries (512 rotated
// indexer rows = 128 KB of bf16, resident in shared memory) and sweeps every
// visible 128-block tile of pooled keys:
//   warp 0      TMA producer: pooled-key tiles (SWIZZLE_128B) into a 3-stage ring;
//   warp 1      MMA issuer: tcgen05.mma kind::f16, M = 128 blocks x N = 256
//               (query, head) columns x K = 128, fp32 accumulators in TMEM; the
//               512 TMEM columns hold two halves (queries 0-63 / 64-127) that
//               are double-buffered against the epilogue;
//   warps 2-9   epilogue: tcgen05.ld of 32 columns per thread-lane (a block
//               row), ReLU-sum over the 4 heads in registers, block-causal
//               mask, and a streaming top-k: a score enters the query's
//               candidate buffer (global, 1024 entries) only if it beats the
//               query's threshold tau; when a buffer could overflow, one warp
//               keeps its k_B best entries (radix select over the 32-bit
//               order-preserving keys, ties to the lower block index) and
//               raises tau to the k_B-th score. Since blocks arrive in
//               ascending order, a later block that ties tau loses the tie.
// At the end of the sweep each query keeps exactly min(k_B, visible) entries,
// which are sorted ascending and written out.
//
// Every wait is bounded (10 s of %globaltimer); on expiry the kernel records
// QSA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int QT = 128;                // queries per CTA tile
constexpr int BT = 128;                // pooled-key blocks per MMA tile (M)
constexpr int NHALF = 256;             // TMEM columns per half = 64 queries x 4 heads
constexpr int STAGES = 2;
constexpr int CAP = 1024;              // candidate entries per query
constexpr int NSEG = 4;                // one segment per TMEM lane quadrant (epilogue warp)
constexpr int SAMPLE = 16;             // estimate phase: every SAMPLE-th pooled-key tile
constexpr int SEG = CAP / NSEG;        // entries per segment
constexpr int KMAX_FUSED = 512;        // largest k_B handled here
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int THREADS = 64 + EPI_THREADS;
static_assert(QT / EPI_WARPS <= 32, "one lane per query of a warp in the compaction check");
constexpr int Q_BYTES = QT * kIdxHeads * 256;  // 131072
constexpr int KT_BYTES = BT * 256;             // 32768
constexpr uint64_t WAIT_NS = 10000000000ull;  // 10 s: the limit of every wait in normal use

struct Ctl {
    uint64_t full[STAGES], empty[STAGES];
    uint64_t q_full, acc_full[2], acc_empty[2], cta_bar, mma_done;
    uint32_t tmem_base;
    int abort;
    int tile[2];        // query tile of the next two iterations (double-buffered)
    int redo[2];        // 1: repeat the tile in exact mode for the queries that failed
    float tau_est[QT];  // threshold estimated from the sample phase (-inf: none)
    uint8_t failed[QT]; // query's candidates did not prove the top-k in estimate mode
    alignas(16) float tau[QT];
    int seg[QT][NSEG];  // entries in each segment of a query's candidate buffer
    alignas(16) int cvis[QT];
};
// Per epilogue warp: 16 scores x 32 lanes of append staging, which is also
// the warp's 256-bin radix histogram while it compacts.
constexpr int STAGE_FLOATS = 16 * 32;
constexpr int STAGE_BYTES = EPI_WARPS * STAGE_FLOATS * 4;
constexpr int SMEM = Q_BYTES + STAGES * KT_BYTES + STAGE_BYTES + (int)sizeof(Ctl) + 1024;
static_assert(SMEM <= 232448, "shared memory per CTA");

// ------------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t gtime() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase of parity `parity` to complete. Returns false (and sets
// the CTA's abort flag) after limit_ns, or at once if another warp aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
    if (mbar_try(a, parity)) return true;
    const uint64_t t0 = gtime();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(a, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (gtime() - t0 > limit_ns) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Barrier over the 256 epilogue threads (named barrier 1) that also ANDs a
// predicate across them, so a timeout seen by any warp ends all of them alike.
__device__ __forceinline__ bool epi_sync_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 256, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Barrier over the 256 epilogue threads that counts the threads whose
// predicate is true.
__device__ __forceinline__ int epi_sync_count(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n bar.red.popc.u32 %0, 1, 256, p;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return (int)r;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t mbar,
                                            int x, int y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"((uint64_t)map), "r"(mbar), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// UMMA shared-memory descriptor: K-major, SWIZZLE_128B (rows of 128 bytes,
// 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;             // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;   // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;             // descriptor version
    d |= (uint64_t)2u << 61;             // SWIZZLE_128B
    return d;
}
// Instruction descriptor: D f32, A/B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NHALF >> 3) << 17) |
                           ((uint32_t)(BT >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc) {
    const uint32_t z = 0;
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(IDESC), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z));
}
__device__ __forceinline__ void umma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
          "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(addr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ------------------------------------------------------- candidate compaction
// Keeps the k best of the n = sum(segn) (k <= n <= CAP) entries (score bits,
// block) of one query's segmented candidate buffer, ranked by (score desc,
// block asc). The kept entries are either written back round-robin over the
// segments (entry p of the kept list to segment p % 4, slot p / 4; in no
// particular order) or, if out_idx is given, their block indices are written
// to out_idx[0, k). Returns the
// order-preserving key of the smallest kept score. One warp; `hist` is its
// 256-bin scratch.
//
// Radix select over the 32-bit keys with 8-bit digits, starting at the highest
// bit where the buffer's keys differ (all keys above it are equal); each digit
// level is one shared-memory histogram pass over the entries still tied with
// the threshold prefix. It stops as soon as every entry matching the prefix is
// needed; exact ties beyond that go to the lowest block indices.
__device__ uint32_t warp_keep_best(uint2* qbuf, const int* segn, int k, int lane, uint32_t* hist,
                                   int32_t* out_idx) {
    uint32_t key[32];
    uint32_t ix[32];
    uint32_t valid = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
    int n = 0;
#pragma unroll
    for (int sg = 0; sg < NSEG; ++sg) n += segn[sg];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        // Register slot j of this lane: segment j / 8, entry ((j % 8) * 32 + lane).
        const int e = ((j & 7) << 5) | lane;
        if (e < segn[j >> 3]) {
            const uint2 v = qbuf[(j >> 3) * SEG + e];
            key[j] = float_key(__uint_as_float(v.x));
            ix[j] = v.y;
            valid |= 1u << j;
            kmin = min(kmin, key[j]);
            kmax = max(kmax, key[j]);
        } else {
            key[j] = 0u;
            ix[j] = 0xFFFFFFFFu;
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const uint32_t diff = kmin ^ kmax;
    int hi = diff ? 31 - __clz(diff) : -1;  // highest bit where keys differ
    uint32_t mask = hi >= 0 ? ~((2u << hi) - 1u) : 0xFFFFFFFFu;
    uint32_t prefix = kmin & mask;
    int need = k, rem = n;
    while (rem != need && hi >= 0) {
        const int lo = hi >= 7 ? hi - 7 : 0;
        const uint32_t dmask = (1u << (hi - lo + 1)) - 1u;
#pragma unroll
        for (int t = 0; t < 8; ++t) hist[lane * 8 + t] = 0u;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (((valid >> j) & 1u) && (key[j] & mask) == prefix) atomicAdd(&hist[(key[j] >> lo) & dmask], 1u);
        __syncwarp();
        uint32_t h[8], sum = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            h[t] = hist[lane * 8 + t];
            sum += h[t];
        }
        uint32_t suf = sum;  // inclusive suffix sum over lanes (bins from the top)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += v;
        }
        const uint32_t above = suf - sum;
        const bool mine = above < (uint32_t)need && (uint32_t)need <= suf;
        const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
        int digit = 0, acc_above = 0, dcount = 0;
        if (mine) {
            uint32_t acc = above;
#pragma unroll
            for (int t = 7; t >= 0; --t) {
                if (acc + h[t] >= (uint32_t)need && digit == 0 && dcount == 0) {
                    digit = lane * 8 + t;
                    acc_above = (int)acc;
                    dcount = (int)h[t];
                }
                acc += h[t];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        acc_above = __shfl_sync(0xffffffffu, acc_above, src);
        dcount = __shfl_sync(0xffffffffu, dcount, src);
        need -= acc_above;
        rem = dcount;
        prefix |= (uint32_t)digit << lo;
        mask |= dmask << lo;
        hi = lo - 1;
        __syncwarp();
    }
    // Ties at the threshold (keys exactly equal): the `need` lowest block indices.
    uint32_t iprefix = 0xFFFFFFFFu, imask = 0;
    if (rem != need) {
        iprefix = 0;
        int ineed = need, irem = rem;
        for (int bit = 31; bit >= 0 && irem != ineed; --bit) {
            const uint32_t m2 = imask | (1u << bit);
            int c0 = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                c0 += (((valid >> j) & 1u) && ((key[j] & mask) == prefix) && ((ix[j] & m2) == iprefix)) ? 1 : 0;
            c0 = (int)__reduce_add_sync(0xffffffffu, (unsigned)c0);
            if (c0 >= ineed) {
                irem = c0;
            } else {
                ineed -= c0;
                irem -= c0;
                iprefix |= 1u << bit;
            }
            imask = m2;
        }
    }
    uint32_t keep = 0, minkey = 0xFFFFFFFFu;
    int kc = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t km = key[j] & mask;
        const bool tie_ok = (imask == 0) || ((ix[j] & imask) <= iprefix);
        if (((valid >> j) & 1u) && (km > prefix || (km == prefix && tie_ok))) {
            keep |= 1u << j;
            ++kc;
            minkey = min(minkey, key[j]);
        }
    }
    int incl = kc;  // exclusive prefix of the per-lane counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int pos = incl - kc;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if ((keep >> j) & 1u) {
            if (out_idx)
                out_idx[pos] = (int32_t)ix[j];
            else
                qbuf[(pos % NSEG) * SEG + pos / NSEG] = make_uint2(__float_as_uint(key_to_float(key[j])), ix[j]);
            ++pos;
        }
    }
    __syncwarp();
    return __reduce_min_sync(0xffffffffu, minkey);
}

// Number of entries of a segmented buffer whose score is strictly above thr.
__device__ int warp_count_above(const uint2* qbuf, const int* segn, float thr, int lane) {
    int c = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int e = ((j & 7) << 5) | lane;
        if (e < segn[j >> 3] && __uint_as_float(qbuf[(j >> 3) * SEG + e].x) > thr) ++c;
    }
    return (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
}

__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
    float2 c;
    asm("{\n .reg .b64 ra, rb, rc;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " add.rn.f32x2 rc, ra, rb;\n mov.b64 {%0, %1}, rc;\n}\n"
        : "=f"(c.x), "=f"(c.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return c;
}

// An append whose slot is reserved but whose store is still to be issued.
struct Pending {
    uint2* p;  // nullptr: none
    float val;
    uint32_t b;
};
__device__ __forceinline__ void retire(Pending& x) {
    if (x.p) *x.p = make_uint2(__float_as_uint(x.val), x.b);
    x.p = nullptr;
}

// Scores of 16 queries (q0 .. q0 + 15) x this lane's block b from 64
// accumulator words (4 heads each). The kernel works with twice the score,
// 2 s = sum_h (x_h + |x_h|): every term is exactly 2 ReLU(x_h), so the order
// of all scores (and ties) is that of s, and the additions run on the FMA
// pipe. A score enters query q's candidate segment of this warp if
// 2 s >= tau[q] (tau is kept in the same units) and, on the diagonal tile,
// b < cvis[q].
//
// Appends are software-pipelined: a lane's first two takes of a call reserve
// their slots (shared atomic on the segment fill) and fetch their values from
// the lane's staging row now, and their stores are issued by the next call,
// after its scoring has covered those latencies (`retire`); further takes of
// the same call (only while tau is still low) are stored at once.
template <bool MASKED>
__device__ __forceinline__ void score16(const uint32_t* v, int q0, uint32_t b, Ctl& ctl, int qd,
                                        uint2* cand_q0, float* stage, int lane, Pending& pa, Pending& pb) {
    float sc[16];
    uint32_t m = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 t4 = *reinterpret_cast<const float4*>(&ctl.tau[q0 + 4 * g]);
        const float tq[4] = {t4.x, t4.y, t4.z, t4.w};
        int cq[4] = {0, 0, 0, 0};
        if (MASKED) {
            const int4 c4 = *reinterpret_cast<const int4*>(&ctl.cvis[q0 + 4 * g]);
            cq[0] = c4.x, cq[1] = c4.y, cq[2] = c4.z, cq[3] = c4.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int qq = 4 * g + i;
            const float x0 = __uint_as_float(v[4 * qq]), x1 = __uint_as_float(v[4 * qq + 1]);
            const float x2 = __uint_as_float(v[4 * qq + 2]), x3 = __uint_as_float(v[4 * qq + 3]);
            const float2 p = add_f32x2(make_float2(x0 + fabsf(x0), x1 + fabsf(x1)),
                                       make_float2(x2 + fabsf(x2), x3 + fabsf(x3)));
            sc[qq] = p.x + p.y;
            bool t = sc[qq] >= tq[i];
            if (MASKED) t = t && (int)b < cq[i];
            if (t) m |= 1u << qq;
        }
    }
    retire(pa);
    retire(pb);
    if (m) {
        // 16-byte chunks of the lane's 16 scores, rotated so that 8 consecutive
        // lanes hit distinct bank groups.
        const int rot = (lane >> 1) & 3;
        float4* st = reinterpret_cast<float4*>(stage) + lane * 4;
#pragma unroll
        for (int g = 0; g < 4; ++g) st[g ^ rot] = make_float4(sc[4 * g], sc[4 * g + 1], sc[4 * g + 2], sc[4 * g + 3]);
        int qq = __ffs(m) - 1;
        m &= m - 1;
        pa.val = stage[lane * 16 + (((qq >> 2) ^ rot) << 2) + (qq & 3)];
        pa.b = b;
        pa.p = cand_q0 + (size_t)qq * CAP + atomicAdd(&ctl.seg[q0 + qq][qd], 1);
        if (m) {
            qq = __ffs(m) - 1;
            m &= m - 1;
            pb.val = stage[lane * 16 + (((qq >> 2) ^ rot) << 2) + (qq & 3)];
            pb.b = b;
            pb.p = cand_q0 + (size_t)qq * CAP + atomicAdd(&ctl.seg[q0 + qq][qd], 1);
            while (m) {
                qq = __ffs(m) - 1;
                m &= m - 1;
                const float val = stage[lane * 16 + (((qq >> 2) ^ rot) << 2) + (qq & 3)];
                const int pos = atomicAdd(&ctl.seg[q0 + qq][qd], 1);
                cand_q0[(size_t)qq * CAP + pos] = make_uint2(__float_as_uint(val), b);
            }
        }
    }
}

// Sorts a[0, m) (m <= 32 R, shared memory, 16-byte aligned) ascending in
// place, one warp: bitonic network over 32 R values held in registers, element
// lane * R + r in register r of `lane` (strides below R stay in a lane, larger
// ones are shuffles); slots past m are padded with INT_MAX and come out last.
template <int R>
__device__ void warp_sort_regs(int32_t* a, int m, int lane) {
    int32_t v[R];
    if constexpr (R >= 4) {
#pragma unroll
        for (int r = 0; r < R; r += 4) {
            const int4 x = *reinterpret_cast<const int4*>(a + lane * R + r);
            v[r] = x.x, v[r + 1] = x.y, v[r + 2] = x.z, v[r + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) v[r] = a[lane * R + r];
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (lane * R + r >= m) v[r] = 0x7fffffff;
#pragma unroll
    for (int k = 2; k <= 32 * R; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= R) {
                const int lj = j / R;
                const bool lower = (lane & lj) == 0;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const bool up = ((lane * R + r) & k) == 0;
                    const int32_t o = __shfl_xor_sync(0xffffffffu, v[r], lj);
                    v[r] = (lower == up) ? min(v[r], o) : max(v[r], o);
                }
            } else {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if ((r & j) == 0) {
                        const bool up = ((lane * R + r) & k) == 0;
                        const int32_t x = v[r], y = v[r | j];
                        v[r] = up ? min(x, y) : max(x, y);
                        v[r | j] = up ? max(x, y) : min(x, y);
                    }
                }
            }
        }
    }
    __syncwarp();
    if constexpr (R >= 4) {
#pragma unroll
        for (int r = 0; r < R; r += 4)
            *reinterpret_cast<int4*>(a + lane * R + r) = make_int4(v[r], v[r + 1], v[r + 2], v[r + 3]);
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) a[lane * R + r] = v[r];
    }
    __syncwarp();
}

__device__ void warp_sort(int32_t* a, int m, int kB, int lane) {
    if (kB <= 32)
        warp_sort_regs<1>(a, m, lane);
    else if (kB <= 64)
        warp_sort_regs<2>(a, m, lane);
    else if (kB <= 128)
        warp_sort_regs<4>(a, m, lane);
    else if (kB <= 256)
        warp_sort_regs<8>(a, m, lane);
    else
        warp_sort_regs<16>(a, m, lane);
}

// Sweep order of the pooled-key tiles: with nsamp > 0, first the sample tiles
// 0, SAMPLE, 2*SAMPLE, ... then the others in ascending order.
__device__ __forceinline__ int tile_at(int t, int nsamp) {
    if (t < nsamp) return t * SAMPLE;
    if (nsamp == 0) return t;
    const int i = t - nsamp;
    return i + i / (SAMPLE - 1) + 1;
}

// --------------------------------------------------------------------- kernel
__global__ void __launch_bounds__(THREADS, 1) fused_topk_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int batch,
    int64_t nq, int64_t q_begin, int64_t pcap, int r, int kB, int* __restrict__ tile_counter,
    uint2* __restrict__ cand, int32_t* __restrict__ sel, int32_t* __restrict__ nsel,
    int32_t* __restrict__ status, int splits, uint2* __restrict__ split_out, int32_t* __restrict__ split_cnt,
    uint64_t wait_ns, int fault_mode) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t sQ = base_s;
    const uint32_t sK = base_s + Q_BYTES;
    float* stage_all = reinterpret_cast<float*>(base + Q_BYTES + STAGES * KT_BYTES);
    Ctl& ctl = *reinterpret_cast<Ctl*>(base + Q_BYTES + STAGES * KT_BYTES + STAGE_BYTES);
    volatile int* abort_flag = &ctl.abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t nqt = (nq + QT - 1) / QT;
    const int64_t total_tiles = nqt * batch * splits;  // work units: (query tile, key split)

    auto bar = [&](const uint64_t& b) { return smem_u32(&b); };

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(ctl.full[s]), 1);
            mbar_init(bar(ctl.empty[s]), 1);
        }
        mbar_init(bar(ctl.q_full), 1);
        for (int h = 0; h < 2; ++h) {
            mbar_init(bar(ctl.acc_full[h]), 1);
            mbar_init(bar(ctl.acc_empty[h]), EPI_WARPS);
        }
        mbar_init(bar(ctl.cta_bar), THREADS);
        mbar_init(bar(ctl.mma_done), 1);
        ctl.abort = 0;
        ctl.tile[0] = atomicAdd(tile_counter, 1);
        ctl.redo[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctl.tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;

    // Per-role pipeline state (continues across query tiles).
    uint32_t kring = 0;       // pooled-key tiles produced / consumed
    uint32_t acc_iter = 0;    // MMA tiles (both halves) issued / drained
    uint32_t q_iter = 0;      // query tiles with a sweep
    uint32_t cta_phase = 0;
    uint32_t produced_last[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) produced_last[i] = 0xFFFFFFFFu;
    const uint64_t pol_k = policy_evict_last();
    const uint64_t pol_q = policy_evict_first();

    for (int iter = 0;; ++iter) {
        // ---- CTA-wide: this iteration's query tile (chosen by the previous one) ----
        mbar_arrive(bar(ctl.cta_bar));
        // Warp-uniform outcome (warp collectives follow); for the epilogue warps
        // also uniform across the group, which meets at named barriers.
        const bool waited = __all_sync(0xffffffffu, mbar_wait(bar(ctl.cta_bar), cta_phase, abort_flag, wait_ns));
        cta_phase ^= 1;
        const int64_t u = waited ? (int64_t)ctl.tile[iter & 1] : total_tiles;
        const bool redo = waited && ctl.redo[iter & 1] != 0;
        bool go = waited && u < total_tiles && !*abort_flag;
        if (warp >= 2) go = epi_sync_and(go);
        if (!go) break;
        // Unit u: query tile tu = u / splits (deepest first) and key split sp, the
        // pooled-key tiles [kt0, kt0 + ntiles) of the tile's visible range.
        const int64_t tu = u / splits;
        const int sp = (int)(u % splits);
        const int s = (int)(tu % batch);
        const int64_t qt = nqt - 1 - tu / batch;
        const int64_t j0 = qt * QT;
        const int nrows = (int)std::min<int64_t>(QT, nq - j0);
        const int64_t c_min = (q_begin + j0) / r;
        const int64_t c_max = (q_begin + j0 + nrows - 1) / r;
        const int ntiles_all = c_max > kB ? (int)((c_max + BT - 1) / BT) : 0;
        const int kt0 = (int)((int64_t)ntiles_all * sp / splits);
        const int ntiles = (int)((int64_t)ntiles_all * (sp + 1) / splits) - kt0;
        const int64_t c_range = std::min<int64_t>((int64_t)(kt0 + ntiles) * BT, c_max) - (int64_t)kt0 * BT;
        // Estimate mode (sample first) when the sweep is long enough to need it;
        // exact mode (ascending sweep, running threshold) otherwise and on a redo.
        const int nsamp = (!redo && c_range > CAP) ? (ntiles + SAMPLE - 1) / SAMPLE : 0;
        // Sample entries kept: about 2 k_B candidates expected over the whole sweep.
        int kA = nsamp ? (int)((2LL * kB * nsamp * BT + c_range - 1) / c_range) : kB;
        kA = max(kA, min(16, kB));

        if (warp == 0) {
            // ------------------------------------------------ TMA producer
            if (lane == 0 && ntiles > 0) {
                const uint32_t qb = bar(ctl.q_full);
                mbar_expect_tx(qb, Q_BYTES);
                const int qrow = (int)(((int64_t)s * nq + j0) * kIdxHeads);
                for (int kh = 0; kh < 2; ++kh)
                    for (int rh = 0; rh < 2; ++rh)
                        tma_load_2d(sQ + kh * (Q_BYTES / 2) + rh * (Q_BYTES / 4), &tm_q, qb, kh * 64,
                                    qrow + rh * 256, pol_q);
                const int krow0 = (int)((int64_t)s * pcap);
                // Fault injection (tests of the failure path only): the CTA's first
                // unit gets no key tiles, so the MMA warp's wait runs out.
                const bool withhold = fault_mode == 1 && iter == 0;
                for (int t = 0; t < ntiles; ++t, ++kring) {
                    const int stg = (int)(kring % STAGES);
                    const uint32_t round = kring / STAGES;
                    if (!mbar_wait(bar(ctl.empty[stg]), (round & 1u) ^ 1u, abort_flag, wait_ns)) break;
                    if (withhold) continue;
                    const uint32_t fb = bar(ctl.full[stg]);
                    mbar_expect_tx(fb, KT_BYTES);
                    for (int kh = 0; kh < 2; ++kh)
                        tma_load_2d(sK + stg * KT_BYTES + kh * (KT_BYTES / 2), &tm_k, fb, kh * 64,
                                    krow0 + (kt0 + tile_at(t, nsamp)) * BT, pol_k);
                    produced_last[stg] = round;
                }
            }
        } else if (warp == 1) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0 && ntiles > 0) {
                bool ok = mbar_wait(bar(ctl.q_full), q_iter & 1u, abort_flag, wait_ns);
                for (int t = 0; ok && t < ntiles; ++t, ++kring, ++acc_iter) {
                    const int stg = (int)(kring % STAGES);
                    if (!(ok = mbar_wait(bar(ctl.full[stg]), (kring / STAGES) & 1u, abort_flag, wait_ns))) break;
                    tc_fence_after();
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = mbar_wait(bar(ctl.acc_empty[h]), (acc_iter & 1u) ^ 1u, abort_flag, wait_ns))) break;
                        tc_fence_after();
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t koff = (kk >> 2) * (KT_BYTES / 2) + (kk & 3) * 32;
                            const uint32_t qoff = (kk >> 2) * (Q_BYTES / 2) + h * (NHALF * 128) + (kk & 3) * 32;
                            umma_bf16(tmem + h * NHALF, desc_sw128(sK + stg * KT_BYTES + koff),
                                      desc_sw128(sQ + qoff), kk > 0 ? 1u : 0u);
                        }
                        umma_commit(bar(ctl.acc_full[h]));
                    }
                    if (!ok) break;
                    umma_commit(bar(ctl.empty[stg]));
                }
            }
            if (ntiles > 0) ++q_iter;
        } else {
            // ------------------------------------------------ epilogue
            const int et = tid - 64, ew = et >> 5;
            const int qd = warp & 3;          // TMEM lane quadrant of this warp
            const int ch = ew >> 2;           // which 128-column half of a TMEM half
            for (int q = et; q < QT; q += EPI_THREADS) {
                ctl.tau[q] = q < nrows ? -INFINITY : INFINITY;  // rows past nq never enter
                ctl.tau_est[q] = -INFINITY;
                for (int sg = 0; sg < NSEG; ++sg) ctl.seg[q][sg] = 0;
                ctl.cvis[q] = q < nrows ? (int)((q_begin + j0 + q) / r) : 0;
                if (!redo) ctl.failed[q] = 0;
            }
            bool ok = epi_sync_and(true);
            const size_t slot0 = (size_t)blockIdx.x * QT;
            const uint32_t tlane = tmem + ((uint32_t)(qd * 32) << 16);
            float* stage = stage_all + ew * STAGE_FLOATS;
            uint32_t* hist = reinterpret_cast<uint32_t*>(stage);
            Pending pa{nullptr, 0.f, 0u}, pb{nullptr, 0.f, 0u};
            for (int t = 0; ok && t < ntiles; ++t, ++acc_iter) {
                const int tt = kt0 + tile_at(t, nsamp);
                const uint32_t b = (uint32_t)(tt * BT + qd * 32 + lane);
                const bool masked = (int64_t)(tt + 1) * BT > c_min;
                bool okt = true;
                for (int h = 0; h < 2; ++h) {
                    const bool okh =
                        __all_sync(0xffffffffu, mbar_wait(bar(ctl.acc_full[h]), acc_iter & 1u, abort_flag, wait_ns));
                    if (okh) {  // warp-uniform
                        uint32_t v[128];
                        tc_fence_after();
                        const uint32_t col = tlane + h * NHALF + ch * 128;
                        tmem_ld32(col, v);
                        tmem_ld32(col + 32, v + 32);
                        tmem_ld32(col + 64, v + 64);
                        tmem_ld32(col + 96, v + 96);
                        tmem_wait_ld();
                        tc_fence_before();
                        // The accumulators are in registers: hand the TMEM half back to
                        // the MMA warp before scoring.
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(ctl.acc_empty[h]));
                        const int q0 = h * 64 + ch * 32;
                        uint2* cq = cand + (slot0 + q0) * CAP + qd * SEG;
                        if (masked) {
                            score16<true>(v, q0, b, ctl, qd, cq, stage, lane, pa, pb);
                            score16<true>(v + 64, q0 + 16, b, ctl, qd, cq + (size_t)16 * CAP, stage, lane, pa, pb);
                        } else {
                            score16<false>(v, q0, b, ctl, qd, cq, stage, lane, pa, pb);
                            score16<false>(v + 64, q0 + 16, b, ctl, qd, cq + (size_t)16 * CAP, stage, lane, pa, pb);
                        }
                    } else {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(ctl.acc_empty[h]));
                    }
                    okt = okt && okh;
                }
                // All appends of tile t are in. A buffer is compacted when one of its
                // segments could overflow on the next tile (a tile adds at most 32
                // entries to a segment), and at the end of the sample phase; the
                // check and the compaction barriers run only when some warp needs them.
                __syncwarp();
                const bool boundary = t + 1 == nsamp;
                const bool near_full =
                    ctl.seg[ch * 32 + lane][qd] > SEG - 32 || ctl.seg[64 + ch * 32 + lane][qd] > SEG - 32;
                if (epi_sync_count(near_full || !okt) == 0 && !boundary) continue;
                retire(pa);  // compaction reads every segment: all stores first
                retire(pb);
                // Sample phase (t < nsamp): keep the k_A best; at its last tile every
                // buffer is cut to k_A and tau becomes the estimate tau_est. Afterwards:
                // keep the k_B best on overflow. Every warp reads the same counts and
                // takes every 8th query of the list, so the work is spread evenly; the
                // list is topped up to a multiple of 8 with queries that are close to
                // their own trigger (those warps would otherwise wait at the barrier).
                const int target = t < nsamp ? kA : kB;
                uint32_t needm[QT / 32], optm[QT / 32];
                int fill = 0;
#pragma unroll
                for (int wd = 0; wd < QT / 32; ++wd) {
                    const int* sq = ctl.seg[wd * 32 + lane];
                    const int n = sq[0] + sq[1] + sq[2] + sq[3];
                    const int mx = max(max(sq[0], sq[1]), max(sq[2], sq[3]));
                    needm[wd] = __ballot_sync(0xffffffffu, mx > SEG - 32 || (boundary && n > target));
                    optm[wd] = __ballot_sync(0xffffffffu, mx > SEG - 96 && n > target + 64) & ~needm[wd];
                    fill -= __popc(needm[wd]);
                }
                fill &= EPI_WARPS - 1;
#pragma unroll
                for (int wd = 0; wd < QT / 32; ++wd) {
                    for (uint32_t o = optm[wd]; fill > 0 && o; o &= o - 1, --fill) needm[wd] |= o & (0u - o);
                }
                if (!(ok = epi_sync_and(okt))) break;  // counts read by all before any changes
                int rank = 0;
#pragma unroll 1
                for (int wd = 0; wd < QT / 32; ++wd) {
                    for (uint32_t msk = needm[wd]; msk; msk &= msk - 1) {
                        if ((rank++ & (EPI_WARPS - 1)) != ew) continue;
                        const int q = wd * 32 + __ffs(msk) - 1;
                        int* sq = ctl.seg[q];
                        const int n = sq[0] + sq[1] + sq[2] + sq[3];
                        // Keep the best `target` and raise tau to the smallest kept score.
                        // (With fewer entries, only rebalance the segments.)
                        const int kk = n < target ? n : target;
                        const uint32_t tk = warp_keep_best(cand + (slot0 + q) * CAP, sq, kk, lane, hist, nullptr);
                        if (lane == 0) {
                            if (kk == target) ctl.tau[q] = key_to_float(tk);
                            for (int sg = 0; sg < NSEG; ++sg) sq[sg] = (kk + NSEG - 1 - sg) / NSEG;
                        }
                        __syncwarp();
                    }
                }
                if (!(ok = epi_sync_and(true))) break;
                if (boundary && lane < QT / EPI_WARPS)
                    ctl.tau_est[ew + EPI_WARPS * lane] = ctl.tau[ew + EPI_WARPS * lane];
            }
            // The last reserved appends, then every warp's stores before the reads.
            retire(pa);
            retire(pb);
            if (ok) ok = epi_sync_and(true);
            // Final selection and ascending output (the pooled-key ring is idle now:
            // use it as sort scratch, 2 KB per warp).
            if (ok) {
                int32_t* scratch = reinterpret_cast<int32_t*>(base + Q_BYTES) + ew * KMAX_FUSED;
                for (int q = ew; q < nrows; q += EPI_WARPS) {
                    // Visible blocks of query q inside this unit's key range.
                    const int cq = max(0, min(ctl.cvis[q], (kt0 + ntiles) * BT) - kt0 * BT);
                    const int kq = cq < kB ? cq : kB;
                    const size_t orow = (size_t)s * nq + j0 + q;
                    int32_t* out = sel + orow * kB;
                    const size_t slot = ((size_t)tu * splits + sp) * QT + q;  // split result slot
                    if (splits > 1 && ntiles == 0) {
                        if (lane == 0) split_cnt[slot] = 0;
                        continue;
                    }
                    if (ntiles == 0) {  // every visible block is selected
                        const int kv = min(ctl.cvis[q], kB);
                        for (int k2 = lane; k2 < kB; k2 += 32) out[k2] = k2 < kv ? k2 : -1;
                        if (lane == 0) nsel[orow] = kv;
                        continue;
                    }
                    if (redo && !ctl.failed[q]) continue;  // written by the estimate pass
                    const int* sq = ctl.seg[q];
                    const int n = sq[0] + sq[1] + sq[2] + sq[3];
                    if (nsamp > 0) {
                        // Every entry above tau_est was admitted and kept; if at least k_q
                        // of them exist, the exact top k_q is among the candidates.
                        // Otherwise this query is redone in exact mode.
                        const float te = ctl.tau_est[q];
                        const int above = te == -INFINITY ? n
                                                          : warp_count_above(cand + (slot0 + q) * CAP, sq, te, lane);
                        if (above < kq) {
                            if (lane == 0) ctl.failed[q] = 1;
                            __syncwarp();
                            continue;
                        }
                    }
                    const int m = n < kq ? n : kq;
                    if (m != kq && lane == 0) flag_status(status, 7 /* QSA_ERR_DEVICE_CHECK */);
                    if (splits > 1) {
                        // The exact top k_q of this key range, with scores, for the merge.
                        uint2* qb = cand + (slot0 + q) * CAP;
                        warp_keep_best(qb, sq, m, lane, hist, nullptr);
                        __syncwarp();
                        uint2* dst = split_out + slot * kB;
                        for (int k2 = lane; k2 < m; k2 += 32) dst[k2] = qb[(k2 % NSEG) * SEG + k2 / NSEG];
                        if (lane == 0) split_cnt[slot] = m;
                        __syncwarp();
                        continue;
                    }
                    warp_keep_best(cand + (slot0 + q) * CAP, sq, m, lane, hist, scratch);
                    __syncwarp();
                    warp_sort(scratch, m, kB, lane);
                    for (int k2 = lane; k2 < kB; k2 += 32) out[k2] = k2 < m ? scratch[k2] : -1;
                    if (lane == 0) nsel[orow] = m;
                    __syncwarp();
                }
            }
            // Next iteration: this tile again in exact mode if a query failed its
            // check, otherwise the next tile from the queue.
            bool mine_ok = true;
            for (int q = ew; q < nrows; q += EPI_WARPS) mine_ok = mine_ok && !ctl.failed[q];
            const bool all_ok = epi_sync_and(mine_ok || redo);
            if (et == 0) {
                const int nx = (iter + 1) & 1;
                ctl.redo[nx] = all_ok ? 0 : 1;
                ctl.tile[nx] = all_ok ? atomicAdd(tile_counter, 1) : (int)u;
            }
        }
    }

    // ---- shutdown: drain what this CTA started, then free TMEM ----
    if (!*abort_flag && warp == 0 && lane == 0) {
        // The MMA warp's last commits release the ring stages; let them land
        // before the CTA's shared memory goes away.
        for (int stg = 0; stg < STAGES; ++stg)
            if (produced_last[stg] != 0xFFFFFFFFu)
                mbar_wait(smem_u32(&ctl.empty[stg]), produced_last[stg] & 1u, abort_flag, wait_ns);
    }
    if (*abort_flag) {
        if (tid == 0) flag_status(status, 6 /* QSA_ERR_TIMEOUT */);
        if (warp == 0 && lane == 0) {
            // Outstanding TMA copies complete on their stage barriers.
            volatile int no_abort = 0;
            for (int stg = 0; stg < STAGES; ++stg)
                if (produced_last[stg] != 0xFFFFFFFFu)
                    mbar_wait(smem_u32(&ctl.full[stg]), produced_last[stg] & 1u, &no_abort, wait_ns);
        }
        if (warp == 1 && lane == 0) {
            volatile int no_abort = 0;
            umma_commit(smem_u32(&ctl.mma_done));
            mbar_wait(smem_u32(&ctl.mma_done), 0, &no_abort, wait_ns);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
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

// 2D bf16 map over `rows` rows of 128 elements, box = 64 elements x box_rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace

bool fused_topk_supported(const LayerDims& L) { return L.kB <= KMAX_FUSED; }

// When there are fewer query tiles than SMs (a short chunk against a long
// context), each tile's key range is split over several CTAs; every split
// keeps the exact top-k of its range (with scores) and a merge selects the
// top k_B of their union, which is the top k_B of the whole range: an entry
// of the overall top k_B is beaten by fewer than k_B entries in its own split.
constexpr int kMaxSplits = 8;

// Fault injection for tests of the failure path (off unless a test sets it).
std::atomic<int> g_fault_mode{0};
std::atomic<uint64_t> g_fault_wait_ns{WAIT_NS};

void set_fault_injection(int mode, uint64_t wait_ns) {
    g_fault_wait_ns.store(wait_ns, std::memory_order_relaxed);
    g_fault_mode.store(mode, std::memory_order_relaxed);
}

int fused_topk_max_splits(int batch, int64_t nq) {
    const int64_t tiles = ((nq + QT - 1) / QT) * batch;
    const int sms = sm_count();
    if (tiles >= sms) return 1;
    return (int)std::min<int64_t>(kMaxSplits, (sms + tiles - 1) / tiles);
}

static size_t split_slots(int batch, int64_t nq) {
    return (size_t)((nq + QT - 1) / QT) * batch * fused_topk_max_splits(batch, nq) * QT;
}

size_t fused_topk_ws_bytes(int batch, int64_t nq, int kB) {
    // tile counter (256 B) + candidate buffers of one CTA per SM (+ split results).
    size_t bytes = 256 + (size_t)sm_count() * QT * CAP * sizeof(uint2);
    if (fused_topk_max_splits(batch, nq) > 1) bytes += split_slots(batch, nq) * ((size_t)kB * sizeof(uint2) + 4);
    return bytes;
}

cudaError_t launch_fused_topk(const LayerDims& L, int batch, const uint16_t* qrot, int64_t nq,
                              int64_t q_begin, const uint16_t* pooled, int64_t cap, int32_t* sel,
                              int32_t* nsel, void* ws, int32_t* status, cudaStream_t st) {
    if (nq <= 0 || batch <= 0) return cudaSuccess;
    const int64_t pcap = cap / L.r;
    CUtensorMap tm_q, tm_k;
    if (!make_map(&tm_q, qrot, (uint64_t)batch * nq * kIdxHeads, 256) ||
        !make_map(&tm_k, pooled, (uint64_t)batch * std::max<int64_t>(pcap, 1), BT))
        return cudaErrorInvalidValue;
    const int grid_max = sm_count();
    const int64_t tiles = ((nq + QT - 1) / QT) * batch;
    // Splits: the count that minimises the makespan estimate (rounds of units
    // over the CTAs) x (key tiles per unit of the deepest query tile), fewer
    // splits on a tie, at least 16 key tiles per split.
    int splits = 1;
    const int smax = fused_topk_max_splits(batch, nq);
    if (smax > 1) {
        const int64_t cdeep = (q_begin + nq - 1) / L.r;
        const int64_t kt = cdeep > L.kB ? (cdeep + BT - 1) / BT : 0;
        int64_t best = -1;
        for (int S = 1; S <= smax && (S == 1 || kt / S >= 16); ++S) {
            const int64_t est = ((tiles * S + grid_max - 1) / grid_max) * ((kt + S - 1) / S);
            if (best < 0 || est < best) {
                best = est;
                splits = S;
            }
        }
    }
    const int grid = (int)std::min<int64_t>(grid_max, tiles * splits);
    int* counter = reinterpret_cast<int*>(ws);
    uint2* cand = reinterpret_cast<uint2*>((char*)ws + 256);
    uint2* split_out = nullptr;
    int32_t* split_cnt = nullptr;
    if (splits > 1) {
        split_out = cand + (size_t)grid_max * QT * CAP;
        split_cnt = reinterpret_cast<int32_t*>(split_out + split_slots(batch, nq) * L.kB);
    }
    cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(fused_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    note_launch();
    const int fmode = g_fault_mode.load(std::memory_order_relaxed);
    const uint64_t wait_ns = fmode ? g_fault_wait_ns.load(std::memory_order_relaxed) : WAIT_NS;
    fused_topk_kernel<<<grid, THREADS, SMEM, st>>>(tm_q, tm_k, batch, nq, q_begin, pcap, L.r, L.kB, counter,
                                                   cand, sel, nsel, status, splits, split_out, split_cnt, wait_ns,
                                                   fmode);
    e = cudaGetLastError();
    if (e != cudaSuccess || splits == 1) return e;
    return launch_split_merge(L, batch, nq, q_begin, QT, splits, split_out, split_cnt, sel, nsel, st);
}

}  // namespace qsa
