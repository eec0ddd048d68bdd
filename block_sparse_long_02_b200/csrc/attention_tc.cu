// a6 + a7 on the fifth-generation tensor cores: expansion of the selected
// blocks (plus the current tail) and the sparse core attention over them
// ("QSA (Qwen Sparse Attention)" concept page, (B) sparse core attention;
// "Qwen Sparse Attention" gallery page, "How block selection works":
// attention_input = flatten(selected_blocks) + current_incomplete_block).
//
// Shape of the work. Query i attends, for every core head h, over the tokens
// of its selected blocks and its tail; every kv head's K/V rows of a block are
// r x kv_heads x 256 bytes, contiguous in the token-major caches. A tile is 128
// (token, kv head) rows of gathered keys; with the GQA group of q head h being
// kv head h / G, the tile products are
//     S^T = K_tile . Q^T          M = 128 rows, N = q_heads (padded to 16), K = 128 dims
//     O^T += V_tile^T . P^T       M = 128 dims, N = q_heads, K = 128 rows
// where P^T[row][h] is zero unless the row's kv head is h's group. A row's
// logits against the other groups' heads are computed and ignored: the MMA has
// capacity to spare here (8 flop per gathered byte), and a block of every kv
// head is then one contiguous stretch of the cache (4 KB per tensor at r = 4,
// kv_heads = 4) that lands as consecutive tile rows.
//
// Pieces. A piece is up to PT = min(r, 128 / kv_heads) consecutive tokens of
// one block with all their kv heads, in a slot of PR rows (PT x kv_heads
// rounded up to 8, whole 1024-byte swizzle atoms). A tile holds PPT = 128 / PR
// pieces. Query i's pieces are its valid selection entries' blocks, then its
// tail r*floor(i/r) .. i; only counting rows are loaded (rows never loaded hold
// zeros or earlier tiles' finite values, and their probabilities are 0).
//
// Pipeline (one CTA per SM, persistent; warp-specialised):
//   warp 0     schedules the tile stream: for each tile it publishes the
//              pieces' cache rows and the counting rows in a shared-memory
//              ring; it loads each group's Q^T tiles by TMA;
//   warps 1, 3 gather the K and V tiles: 16-byte cp.async copies of each
//              piece's contiguous rows into the 128B-swizzled layout the MMA
//              reads, every thread arriving on the stage's mbarrier when its
//              copies land. (Block-sized TMA boxes - 2 KB per instruction -
//              were measured first: the issuing warp, not the memory system,
//              became the limit at about 5 TB/s.)
//   warp 2     issues the tcgen05.mma (one thread): S^T into TMEM (double
//              buffered), then, once the epilogue has written P, O^T += V^T P^T
//              into the query's TMEM accumulator;
//   warps 4-7  the softmax: each thread owns one TMEM lane (a tile row for S,
//              a head dimension for O).
// A CTA processes QS consecutive query rows at once, their tiles interleaved
// round-robin, so that about QS x 148 queries walk their (ascending) block
// lists together and share fetched blocks through L2.
// Softmax. Logits are fp32 in the log2 domain (scale folded in). Each query
// head keeps a reference maximum m; a tile whose logits stay below m + 8 adds
// exp2(s - m) (at most 2^8) without any cross-thread reduction; otherwise the
// 128 threads agree on the new maxima and the accumulator columns are rescaled
// in TMEM (the first tile of every query does this). Probabilities enter P.V
// rounded to bf16; the row sums are fp32. Output = O / l, LSE = (m + log2 l) ln 2.
//
// Every wait is bounded (%globaltimer); a wait that runs out records
// QSA_ERR_TIMEOUT in the status word, the CTA drains its copies and MMAs, frees
// TMEM and returns.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "kernels.h"
#include "tc.cuh"

namespace qsa {
namespace {

using namespace tc;

constexpr int ROWS = 128;                  // tile rows (the MMA's M)
constexpr int HALF_BYTES = ROWS * 128;     // one 64-dim half of a tile
constexpr int TILE_BYTES = 2 * HALF_BYTES; // K or V tile: 32 KB
constexpr int INFO_DEPTH = 8;              // tile descriptions in flight
constexpr int MAX_PIECES = 16;             // pieces per tile (slots of >= 8 rows)
constexpr int NG = 1;                      // softmax groups of 4 warps
constexpr int THREADS = 128 + 128 * NG;    // scheduler, V loader, MMA, K loader; the softmax warps
constexpr int EPI_WARP0 = 4;
constexpr int MAX_STAGES = 4;
constexpr int MAX_NPAD = 128;
constexpr uint64_t WAIT_NS = 10ull * 1000000000ull;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_AT = 8.0f;         // log2 headroom before the maxima are raised

enum : int32_t { F_FIRST = 1, F_LAST = 2, F_GROUP_FIRST = 4, F_GROUP_LAST = 8, F_END = 16, F_WITHHOLD = 32 };

// One tile of the stream, as the scheduler publishes it.
struct TileInfo {
    int32_t coord[MAX_PIECES];  // piece slot p: first row of its box in the [batch*cap] token axis, -1: not loaded
    uint32_t valid[4];          // bit rho: tile row rho takes part in the softmax
    uint32_t vzero[4];          // bit rho: row rho was loaded but is masked (its V row is cleared)
    int32_t row;                // query row (sequence * nq + j)
    int32_t slot;               // the query's slot in the CTA (0 .. QS-1)
    int32_t flags;
    int32_t pad[5];
};
static_assert(sizeof(TileInfo) == 128, "tile description size");

struct Ctl {
    uint64_t k_full[MAX_STAGES], k_empty[MAX_STAGES], v_full[MAX_STAGES], v_empty[MAX_STAGES];
    uint64_t s_full[4], s_empty[4], p_full[2], p_empty[2];
    uint64_t q_full, q_empty, drain;
    uint64_t i_full[INFO_DEPTH], i_empty[INFO_DEPTH];
    uint32_t tmem;
    int abort;
    // Per softmax group: per-warp partial maxima / sums of each head (word
    // [w][h] is read back only by thread h, which then leaves a per-head result
    // there for all: the rescale factors in row 1, the final sums in row 0).
    float red[NG][4][MAX_NPAD];
    float mst[NG][4][MAX_NPAD];  // per slot of the group: each head's reference maximum (log2 domain)
    int64_t srow[4], sseq[4], spos[4], scur[4];  // the scheduler's current group of query rows
    int snsel[4], spieces[4], stiles[4];
};

struct Params {
    const int32_t* sel;
    const int32_t* nsel;
    uint16_t* out;
    float* lse;
    int32_t* status;
    int64_t rows;   // batch * nq
    int64_t nq, q_begin, cap;
    int r, kB, kvh, q_heads, n_pad;
    int pt, npb, pr, ppt;  // piece tokens, pieces per block, rows per piece slot, pieces per tile
    int kst, vst;          // K and V ring stages
    int tmem_cols;
    int ns_bufs;  // S^T buffers in TMEM (up to 4)
    float scale_log2;
    uint64_t wait_ns;
    int fault_mode;
    uint32_t off_v, off_q, off_p, off_sel, off_info, off_ctl;  // from the 1024-aligned base (K ring at 0)
    int stage_sel;  // the group's selection rows are copied to shared memory (else read per tile)
};

__device__ __forceinline__ uint32_t bar_addr(const uint64_t& b) { return smem_u32(&b); }
#define WAIT_AT(site, idx, bar, parity, ab, ns) wait_at(bar, parity, ab, ns, P.status, site, (int)(idx))

// Shared-memory matrix descriptor of an MN-major operand in SWIZZLE_128B atoms
// (8 rows of the K dimension x 128 bytes of 64 M elements): atoms along K every
// 1024 bytes, the second 64-element half of M `lbo` bytes further.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

__device__ __forceinline__ void tma_load_2d_nocache(uint32_t dst, const CUtensorMap* map, uint32_t mbar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"((uint64_t)map), "r"(mbar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const float* v) {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            addr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]), "r"(u[9]),
        "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Barrier over one softmax group's 128 threads (named barrier `id`) that also
// ORs a predicate across them.
__device__ __forceinline__ bool epi_sync_or(int id, bool p) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred a, b;\n setp.ne.u32 a, %2, 0;\n bar.red.or.pred b, %1, 128, a;\n selp.u32 %0, 1, 0, b;\n}\n"
        : "=r"(r)
        : "r"(id), "r"((uint32_t)p)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void epi_sync(int id) { named_sync(id, 128); }

// Bits [a, b) of a 128-bit row mask that fall in its 32-bit word w.
__device__ __forceinline__ uint32_t range_bits(int w, int a, int b) {
    const int lo = max(a - 32 * w, 0), hi = min(b - 32 * w, 32);
    if (hi <= lo) return 0u;
    const uint32_t width = (uint32_t)(hi - lo);
    return (width == 32u ? 0xFFFFFFFFu : ((1u << width) - 1u)) << lo;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}

// A bounded wait that, when it gives up (its own limit or another thread's),
// records where: status[1] = site, status[2] = tile index, status[3] = CTA of
// the first failure; status[4 + w] = (site << 16 | tile) of warp w's (warps
// 4-7 share word 8).
__device__ __forceinline__ bool wait_at(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint64_t ns,
                                        int32_t* status, int site, int n) {
    if (mbar_wait(bar, parity, abort_flag, ns)) return true;
    if (status) {
        if (atomicCAS(status + 1, 0, site) == 0) {
            status[2] = n;
            status[3] = (int32_t)blockIdx.x;
        }
        const int w = min((int)(threadIdx.x >> 5), 4);
        status[4 + w] = (site << 16) | (n & 0xFFFF);
    }
    return false;
}

// Slot bookkeeping of one group of QS query rows (every role derives the same).
// Slot k of group g (query row g * QS + k), computed by lane k of the
// scheduler into shared memory; returns the group's deepest tile count.
template <int QS>
__device__ __forceinline__ int group_slots(const Params& P, int64_t g, Ctl& ctl, int lane) {
    int tiles = 0;
    if (lane < QS) {
        const int k = lane;
        const int64_t row = g * QS + k;
        int64_t s = 0, i = 0;
        int ns = 0, pieces = 0;
        if (row < P.rows) {
            s = row / P.nq;
            i = P.q_begin + (row - s * P.nq);
            ns = P.nsel[row];
            ns = ns < 0 ? 0 : (ns > P.kB ? P.kB : ns);
            const int ell = (int)(i % P.r) + 1;
            pieces = ns * P.npb + (ell + P.pt - 1) / P.pt;
            tiles = (pieces + P.ppt - 1) / P.ppt;
        }
        ctl.srow[k] = row;
        ctl.sseq[k] = s;
        ctl.spos[k] = i;
        ctl.scur[k] = i / P.r;
        ctl.snsel[k] = ns;
        ctl.spieces[k] = pieces;
        ctl.stiles[k] = tiles;
    }
    __syncwarp();
    int maxT = tiles;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) maxT = max(maxT, __shfl_xor_sync(0xffffffffu, maxT, o));
    return maxT;
}

template <int G, int QS>
__global__ void __launch_bounds__(THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const Params P) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    Ctl& ctl = *reinterpret_cast<Ctl*>(base + P.off_ctl);
    TileInfo* info = reinterpret_cast<TileInfo*>(base + P.off_info);
    volatile int* abort_flag = &ctl.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ngroups = (P.rows + QS - 1) / QS;
    const uint32_t q_slot_bytes = (uint32_t)P.n_pad * 256u;

    // ---- set-up: clear the tile, query and probability buffers (rows that are
    // never loaded must hold finite values: zero), the barriers, TMEM.
    {
        uint4* z = reinterpret_cast<uint4*>(base);
        const uint32_t n16 = P.off_info / 16u;
        for (uint32_t x = tid; x < n16; x += THREADS) z[x] = make_uint4(0u, 0u, 0u, 0u);
        for (int x = tid; x < NG * 4 * MAX_NPAD; x += THREADS) (&ctl.red[0][0][0])[x] = -INFINITY;
        for (int x = tid; x < NG * 4 * MAX_NPAD; x += THREADS) (&ctl.mst[0][0][0])[x] = -INFINITY;
        fence_async_smem();
    }
    if (tid == 0) {
        for (int s = 0; s < MAX_STAGES; ++s) {
            mbar_init(bar_addr(ctl.k_full[s]), 1);
            mbar_init(bar_addr(ctl.k_empty[s]), 1);
            mbar_init(bar_addr(ctl.v_full[s]), 1);
            mbar_init(bar_addr(ctl.v_empty[s]), 1);
        }
        for (int b = 0; b < 4; ++b) {
            mbar_init(bar_addr(ctl.s_full[b]), 1);
            mbar_init(bar_addr(ctl.s_empty[b]), 128);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_addr(ctl.p_full[b]), 128);
            mbar_init(bar_addr(ctl.p_empty[b]), 1);
        }
        mbar_init(bar_addr(ctl.q_full), 1);
        mbar_init(bar_addr(ctl.q_empty), 1);
        mbar_init(bar_addr(ctl.drain), 1);
        for (int d = 0; d < INFO_DEPTH; ++d) {
            mbar_init(bar_addr(ctl.i_full[d]), 1);
            mbar_init(bar_addr(ctl.i_empty[d]), 3 + 4 * NG);  // K and V loaders, the MMA thread, the softmax warps
        }
        ctl.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 3) tmem_alloc(smem_u32(&ctl.tmem), (uint32_t)P.tmem_cols);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = ctl.tmem;
    const uint64_t wait_ns = P.wait_ns;

    // Stages the producers issued last (for the drain after an abort).
    int q_issued = 0, kv_issued = 0;  // copies this thread issued (drained after an abort)

    if (warp == 0) {
        // ------------------------------------------------ scheduler + Q loads
        int n = 0, gcount = 0;
        bool ok = true;
        for (int64_t gi = blockIdx.x; gi < ngroups && ok; gi += gridDim.x) {
            const int64_t g = ngroups - 1 - gi;  // longest queries first
            const int maxT = group_slots<QS>(P, g, ctl, lane);
            // This group's queries: Q^T tiles (rows past q_heads stay zero).
            if (lane == 0) {
                ok = WAIT_AT(1, gcount, bar_addr(ctl.q_empty), (uint32_t)(gcount & 1) ^ 1u, abort_flag, wait_ns);
                if (ok) {
                    int act = 0;
                    for (int k = 0; k < QS; ++k) act += ctl.stiles[k] > 0;
                    mbar_expect_tx(bar_addr(ctl.q_full), (uint32_t)(act * 2 * P.q_heads * 128));
                    for (int k = 0; k < QS; ++k)
                        if (ctl.stiles[k] > 0)
                            for (int h = 0; h < 2; ++h)
                                tma_load_2d_nocache(base_s + P.off_q + k * q_slot_bytes + h * (q_slot_bytes / 2),
                                                    &tm_q, bar_addr(ctl.q_full), h * 64,
                                                    (int)(ctl.srow[k] * P.q_heads));
                    q_issued = gcount + 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            ++gcount;
            // The group's selection rows, read once (the next group's are
            // already on their way to L2).
            int32_t* ssel = reinterpret_cast<int32_t*>(base + P.off_sel);
            if (P.stage_sel) {
                for (int k = 0; k < QS; ++k) {
                    const int32_t* src = P.sel + ctl.srow[k] * P.kB;
#pragma unroll 8
                    for (int x = lane; x < ctl.snsel[k]; x += 32) ssel[k * P.kB + x] = src[x];
                }
                __syncwarp();
            }
            if (gi + gridDim.x < ngroups) {
                const int64_t gn = ngroups - 1 - (gi + gridDim.x);
                const int64_t r0 = gn * QS, r1 = min(P.rows, r0 + QS);
                const char* s0 = reinterpret_cast<const char*>(P.sel + r0 * P.kB);
                const int64_t lines = ((r1 - r0) * P.kB * 4 + 127) / 128;
                for (int64_t x = lane; x < lines; x += 32) prefetch_l2(s0 + x * 128);
                if (lane == 0) prefetch_l2(P.nsel + r0);
            }
            const int32_t withhold = (P.fault_mode == 3 && gi == blockIdx.x) ? F_WITHHOLD : 0;
            bool first_in_group = true;
            for (int t = 0; t < maxT && ok; ++t) {
                for (int k = 0; k < QS && ok; ++k) {
                    if (t >= ctl.stiles[k]) continue;
                    bool last_in_group = (t == maxT - 1);
                    for (int k2 = k + 1; k2 < QS; ++k2) last_in_group = last_in_group && ctl.stiles[k2] < maxT;
                    // This lane's piece: its first cache row and how many of its
                    // tokens count (only those are loaded).
                    int32_t coord = -1;
                    int nvalid = 0;
                    if (lane < P.ppt) {
                        const int p = t * P.ppt + lane;
                        if (p < ctl.spieces[k]) {
                            const int64_t c = ctl.scur[k];
                            if (p < ctl.snsel[k] * P.npb) {
                                const int e = P.npb == 1 ? p : p / P.npb, sub = p - e * P.npb;
                                const int32_t b = P.stage_sel ? ssel[k * P.kB + e] : P.sel[ctl.srow[k] * P.kB + e];
                                if (b >= 0 && (int64_t)b < c) {
                                    coord = (int32_t)(ctl.sseq[k] * P.cap + (int64_t)b * P.r + sub * P.pt);
                                    nvalid = min(P.pt, P.r - sub * P.pt);
                                }
                            } else {
                                const int sub = p - ctl.snsel[k] * P.npb;
                                const int ell = (int)(ctl.spos[k] - c * P.r) + 1;
                                coord = (int32_t)(ctl.sseq[k] * P.cap + c * P.r + sub * P.pt);
                                nvalid = min(P.pt, ell - sub * P.pt);
                            }
                        }
                    }
                    // Rows of this piece slot ([lane*pr, lane*pr + pr)): the first
                    // nvalid*kvh count; the rest of the loaded box is masked.
                    const int r0 = lane * P.pr;
                    const int rv = coord >= 0 ? r0 + nvalid * P.kvh : r0;
                    const int rl = coord >= 0 ? r0 + P.pt * P.kvh : r0;
                    uint32_t vm[4], zm[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        vm[w] = __reduce_or_sync(0xffffffffu, range_bits(w, r0, rv));
                        zm[w] = __reduce_or_sync(0xffffffffu, range_bits(w, rv, rl));
                    }
                    // Publish the tile's description.
                    const int is = n % INFO_DEPTH;
                    if (lane == 0)
                        ok = WAIT_AT(2, n, bar_addr(ctl.i_empty[is]), (uint32_t)((n / INFO_DEPTH) & 1) ^ 1u, abort_flag,
                                       wait_ns);
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                    TileInfo& ti = info[is];
                    if (lane < MAX_PIECES) ti.coord[lane] = coord;
                    if (lane == 0) {
                        for (int w = 0; w < 4; ++w) {
                            ti.valid[w] = vm[w];
                            ti.vzero[w] = zm[w];
                        }
                        ti.row = (int32_t)ctl.srow[k];
                        ti.slot = k;
                        ti.flags = (t == 0 ? F_FIRST : 0) | (t == ctl.stiles[k] - 1 ? F_LAST : 0) |
                                   (first_in_group ? F_GROUP_FIRST : 0) | (last_in_group ? F_GROUP_LAST : 0) |
                                   withhold;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_addr(ctl.i_full[is]));
                    first_in_group = false;
                    ++n;
                }
            }
        }
        if (ok) {  // end of the stream
            const int is = n % INFO_DEPTH;
            if (lane == 0 &&
                WAIT_AT(3, n, bar_addr(ctl.i_empty[is]), (uint32_t)((n / INFO_DEPTH) & 1) ^ 1u, abort_flag, wait_ns)) {
                info[is].flags = F_END;
                mbar_arrive(bar_addr(ctl.i_full[is]));
            }
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------ K (warp 3) / V (warp 1) loads
        // One TMA box per piece and 64-dim half: pt tokens x kv_heads rows of
        // 128 bytes, landing on the piece slot's swizzle atoms.
        const int tensor = warp == 3 ? 0 : 1;
        const int nst = tensor == 0 ? P.kst : P.vst;
        uint64_t* full = tensor == 0 ? ctl.k_full : ctl.v_full;
        uint64_t* empty = tensor == 0 ? ctl.k_empty : ctl.v_empty;
        const CUtensorMap* map = tensor == 0 ? &tm_k : &tm_v;
        const uint32_t region = base_s + (tensor == 0 ? 0u : P.off_v);
        const uint32_t box_bytes = (uint32_t)(P.pt * P.kvh * 128);
        for (int n = 0;; ++n) {
            const int is = n % INFO_DEPTH;
            if (!WAIT_AT(4, n, bar_addr(ctl.i_full[is]), (uint32_t)((n / INFO_DEPTH) & 1), abort_flag, wait_ns)) break;
            const TileInfo& ti = info[is];
            const int32_t flags = ti.flags;
            const int32_t coord = lane < P.ppt ? ti.coord[lane] : -1;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_addr(ctl.i_empty[is]));
            if (flags & F_END) break;
            const uint32_t bytes = __reduce_add_sync(0xffffffffu, coord >= 0 ? 2u * box_bytes : 0u);
            const int st = n % nst;
            bool ok = true;
            if (lane == 0) {
                ok = WAIT_AT(5, n, bar_addr(empty[st]), (uint32_t)((n / nst) & 1) ^ 1u, abort_flag, wait_ns);
                if (ok) mbar_expect_tx(bar_addr(full[st]), bytes);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            if (coord >= 0 && !(flags & F_WITHHOLD)) {
                const uint32_t dst = region + (uint32_t)st * TILE_BYTES + (uint32_t)(lane * P.pr) * 128u;
                tma_load_3d(dst, map, bar_addr(full[st]), 0, 0, coord);
                tma_load_3d(dst + HALF_BYTES, map, bar_addr(full[st]), 64, 0, coord);
            }
            kv_issued = n + 1;
        }
    } else if (warp == 2) {
        // ------------------------------------------------ MMA issue (one thread)
        // Per tile n: S^T_n as soon as its K tile and S buffer are there, then
        // O^T += V^T P^T of tile n - 1 once its P is written.
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(ROWS, P.n_pad);
            const uint32_t idesc_pv = idesc_bf16(ROWS, P.n_pad) | (1u << 15);  // A (V^T) MN-major
            const uint32_t p_half = (uint32_t)P.n_pad * 128u;
            const int NS = P.ns_bufs;
            int gq = 0;
            bool ok = true;
            auto issue_pv = [&](int m, int slot, bool first) -> bool {
                if (!WAIT_AT(6, m, bar_addr(ctl.p_full[m & 1]), (uint32_t)((m >> 1) & 1), abort_flag, wait_ns))
                    return false;
                if (!WAIT_AT(7, m, bar_addr(ctl.v_full[m % P.vst]), (uint32_t)((m / P.vst) & 1), abort_flag, wait_ns))
                    return false;
                fence_after();
                const uint32_t d = tmem + (uint32_t)(NS * P.n_pad + slot * P.n_pad);
                const uint32_t va = base_s + P.off_v + (uint32_t)(m % P.vst) * TILE_BYTES;
                const uint32_t pa = base_s + P.off_p + (uint32_t)(m & 1) * (2u * p_half);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16(d, desc_mn_sw128(va + ks * 2048u, HALF_BYTES),
                              desc_sw128(pa + (ks >> 2) * p_half + (ks & 3) * 32u), idesc_pv,
                              (ks > 0 || !first) ? 1u : 0u);
                umma_commit(bar_addr(ctl.p_empty[m & 1]));
                umma_commit(bar_addr(ctl.v_empty[m % P.vst]));
                return true;
            };
            // P.V lags S by one tile: tile n-1 waits for it.
            int prev = -1, prev_slot = 0;
            bool prev_first = false;
            for (int n = 0;; ++n) {
                const int is = n % INFO_DEPTH;
                if (!(ok = WAIT_AT(8, n, bar_addr(ctl.i_full[is]), (uint32_t)((n / INFO_DEPTH) & 1), abort_flag,
                                   wait_ns)))
                    break;
                const int32_t flags = info[is].flags;
                const int slot = info[is].slot;
                mbar_arrive(bar_addr(ctl.i_empty[is]));
                if (flags & F_END) break;
                if (flags & F_GROUP_FIRST) {
                    if (!(ok = WAIT_AT(9, gq, bar_addr(ctl.q_full), (uint32_t)(gq & 1), abort_flag, wait_ns))) break;
                    ++gq;
                }
                const int st = n % P.kst;
                if (!(ok = WAIT_AT(10, n, bar_addr(ctl.k_full[st]), (uint32_t)((n / P.kst) & 1), abort_flag, wait_ns)))
                    break;
                if (!(ok = WAIT_AT(11, n, bar_addr(ctl.s_empty[n % NS]), (uint32_t)((n / NS) & 1) ^ 1u, abort_flag,
                                   wait_ns)))
                    break;
                fence_after();
                const uint32_t d = tmem + (uint32_t)((n % NS) * P.n_pad);
                const uint32_t ka = base_s + (uint32_t)st * TILE_BYTES;
                const uint32_t qa = base_s + P.off_q + (uint32_t)slot * q_slot_bytes;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16(d, desc_sw128(ka + (ks >> 2) * HALF_BYTES + (ks & 3) * 32u),
                              desc_sw128(qa + (ks >> 2) * (q_slot_bytes / 2) + (ks & 3) * 32u), idesc_s,
                              ks > 0 ? 1u : 0u);
                umma_commit(bar_addr(ctl.s_full[n % NS]));
                umma_commit(bar_addr(ctl.k_empty[st]));
                if (flags & F_GROUP_LAST) umma_commit(bar_addr(ctl.q_empty));
                if (prev >= 0 && !(ok = issue_pv(prev, prev_slot, prev_first))) break;
                prev = n;
                prev_slot = slot;
                prev_first = (flags & F_FIRST) != 0;
            }
            if (ok && prev >= 0) issue_pv(prev, prev_slot, prev_first);
        }
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------ softmax and output
        // Each thread owns TMEM lane rho (its warp's quadrant). With NG > 1
        // groups of four warps, group gid would own the query slots congruent to
        // gid mod NG (kept at NG = 1: the groups would share the P.V completion
        // barriers, and a group that falls two phases behind on ragged query
        // groups reads the wrong phase).
        const int gid = (warp - EPI_WARP0) >> 2;
        const int ew = warp & 3;
        const int bar_id = 1 + gid;
        const int rho = 32 * ew + lane;
        const int qrow = rho % P.pr;
        const int gq = qrow % P.kvh;                                  // the row's kv head
        const bool in_piece = qrow < P.pt * P.kvh && rho / P.pr < P.ppt;
        const int cstar = (gq * G) >> 4, coff = (gq * G) & 15;       // its G columns: chunk, offset
        const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
        const int nch = P.n_pad >> 4;
        const uint32_t p_half = (uint32_t)P.n_pad * 128u;
        constexpr int QL = QS / NG;  // slots of this group: NG kk + gid
        float(&red)[4][MAX_NPAD] = ctl.red[gid];
        float m[QL][G], l[QL][G];
        int64_t slot_row[QL];
        bool slot_on[QL];
#pragma unroll
        for (int kk = 0; kk < QL; ++kk) {
            slot_on[kk] = false;
            slot_row[kk] = 0;
#pragma unroll
            for (int x = 0; x < G; ++x) {
                m[kk][x] = -INFINITY;
                l[kk][x] = 0.f;
            }
        }
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int is = n % INFO_DEPTH;
            if (!(ok = WAIT_AT(12, n, bar_addr(ctl.i_full[is]), (uint32_t)((n / INFO_DEPTH) & 1), abort_flag, wait_ns)))
                break;
            const TileInfo& ti = info[is];
            const int32_t flags = ti.flags;
            const int slot = ti.slot;
            const int64_t row = ti.row;
            const bool valid = (ti.valid[rho >> 5] >> (rho & 31)) & 1u;
            const bool vzero = (ti.vzero[rho >> 5] >> (rho & 31)) & 1u;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_addr(ctl.i_empty[is]));
            if (flags & F_END) break;
            if (slot % NG == gid) {
                // S^T row of this thread: its group's G logits.
                const int sb = n % P.ns_bufs;
                if (!(ok = WAIT_AT(13, n, bar_addr(ctl.s_full[sb]), (uint32_t)((n / P.ns_bufs) & 1), abort_flag,
                                   wait_ns)))
                    break;
                fence_after();
                float kept[16];
                for (int c = 0; c < nch; ++c) {
                    float v[16];
                    tmem_ld16(tmem + lane_off + (uint32_t)(sb * P.n_pad + 16 * c), v);
                    tmem_wait_ld();
                    if (c == cstar) {
#pragma unroll
                        for (int x = 0; x < 16; ++x) kept[x] = v[x];
                    }
                }
                fence_before();
                mbar_arrive(bar_addr(ctl.s_empty[sb]));
                float s[G];
#pragma unroll
                for (int x = 0; x < G; ++x) {
                    float vx = kept[x];
#pragma unroll
                    for (int o = G; o < 16; o += G)
                        if (coff == o) vx = kept[o + x];
                    s[x] = valid ? vx * P.scale_log2 : -INFINITY;
                }
                // This slot's softmax state, in working registers.
                const int kk = slot / NG;
                float mw[G], lw[G];
#pragma unroll
                for (int x = 0; x < G; ++x) {
                    mw[x] = m[0][x];
                    lw[x] = l[0][x];
                }
#pragma unroll
                for (int q = 1; q < QL; ++q)
                    if (q == kk)
#pragma unroll
                        for (int x = 0; x < G; ++x) {
                            mw[x] = m[q][x];
                            lw[x] = l[q][x];
                        }
                do {
                if (flags & F_FIRST) {
#pragma unroll
                    for (int q = 0; q < QL; ++q)
                        if (q == kk) {
                            slot_on[q] = true;
                            slot_row[q] = row;
                        }
#pragma unroll
                    for (int x = 0; x < G; ++x) {
                        mw[x] = -INFINITY;
                        lw[x] = 0.f;
                    }
                    if (rho < P.n_pad) ctl.mst[gid][kk][rho] = -INFINITY;
                }
                bool need = false;
#pragma unroll
                for (int x = 0; x < G; ++x) need = need || (s[x] > mw[x] + RESCALE_AT);
                need = epi_sync_or(bar_id, need);
                if (need) {
                    // New reference maxima: the tile's per-head maximum, raised only.
                    float tm[G];
#pragma unroll
                    for (int x = 0; x < G; ++x) tm[x] = s[x];
                    for (int off = P.kvh; off < 32; off <<= 1)
#pragma unroll
                        for (int x = 0; x < G; ++x)
                            tm[x] = fmaxf(tm[x], __shfl_xor_sync(0xffffffffu, tm[x], off));
                    if (lane < P.kvh)
#pragma unroll
                        for (int x = 0; x < G; ++x) red[ew][lane * G + x] = tm[x];
                    epi_sync(bar_id);
                    if (rho < P.n_pad) {
                        const float mo = ctl.mst[gid][kk][rho];
                        const float mx = fmaxf(fmaxf(red[0][rho], red[1][rho]), fmaxf(red[2][rho], red[3][rho]));
                        const float mn = fmaxf(mo, mx);
                        red[1][rho] = (mn == mo) ? 1.f : ex2_approx(mo - mn);  // after reading red[*][rho]
                        ctl.mst[gid][kk][rho] = mn;
                    }
                    epi_sync(bar_id);
#pragma unroll
                    for (int x = 0; x < G; ++x) {
                        const int h = gq * G + x;
                        lw[x] *= red[1][h];
                        mw[x] = ctl.mst[gid][kk][h];
                    }
                    if (!(flags & F_FIRST)) {
                        // Rescale this query's accumulator once its last P.V is done.
                        if (!(ok = WAIT_AT(14, n, bar_addr(ctl.p_empty[(n - 1) & 1]),
                                           (uint32_t)(((n - 1) >> 1) & 1), abort_flag, wait_ns)))
                            break;
                        fence_after();
                        for (int c = 0; c < nch; ++c) {
                            float v[16];
                            const uint32_t a =
                                tmem + lane_off + (uint32_t)(P.ns_bufs * P.n_pad + slot * P.n_pad + 16 * c);
                            tmem_ld16(a, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 16; ++x) v[x] *= red[1][16 * c + x];
                            tmem_st16(a, v);
                        }
                        tmem_wait_st();
                    }
                }
                float p[G];
#pragma unroll
                for (int x = 0; x < G; ++x) {
                    p[x] = valid ? ex2_approx(s[x] - mw[x]) : 0.f;
                    lw[x] += p[x];
                }
                // Masked rows that were loaded (the tail past i): clear their V rows.
                if (vzero) {
                    const int vs = n % P.vst;
                    if (!(ok = WAIT_AT(17, n, bar_addr(ctl.v_full[vs]), (uint32_t)((n / P.vst) & 1), abort_flag,
                                       wait_ns)))
                        break;
                    uint4* vr0 = reinterpret_cast<uint4*>(base + P.off_v + vs * TILE_BYTES + rho * 128);
                    uint4* vr1 =
                        reinterpret_cast<uint4*>(base + P.off_v + vs * TILE_BYTES + HALF_BYTES + rho * 128);
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        vr0[x] = make_uint4(0u, 0u, 0u, 0u);
                        vr1[x] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                // P^T (K-major, 128B-swizzled: head rows of 64 tile rows per half).
                if (!(ok = WAIT_AT(15, n, bar_addr(ctl.p_empty[n & 1]), (uint32_t)((n >> 1) & 1) ^ 1u,
                                   abort_flag, wait_ns)))
                    break;
                if (in_piece) {
                    uint8_t* pb = base + P.off_p + (n & 1) * (2 * p_half) + (rho >> 6) * p_half;
                    const int ch = (rho & 63) >> 3;
#pragma unroll
                    for (int x = 0; x < G; ++x) {
                        const int h = gq * G + x;
                        *reinterpret_cast<uint16_t*>(pb + h * 128 + ((ch ^ (h & 7)) << 4) + (rho & 7) * 2) =
                            f32_to_bf16(p[x]);
                    }
                }
                fence_async_smem();
                fence_before();
                mbar_arrive(bar_addr(ctl.p_full[n & 1]));
                            } while (false);
#pragma unroll
                for (int q = 0; q < QL; ++q)
                    if (q == kk)
#pragma unroll
                        for (int x = 0; x < G; ++x) {
                            m[q][x] = mw[x];
                            l[q][x] = lw[x];
                        }
                if (!ok) break;
            }
            if (flags & F_GROUP_LAST) {
                // Every P.V of the group is done once this tile's is.
                if (!(ok = WAIT_AT(16, n, bar_addr(ctl.p_empty[n & 1]), (uint32_t)((n >> 1) & 1), abort_flag,
                                   wait_ns)))
                    break;
                fence_after();
                epi_sync(bar_id);  // every thread is past its last reads of the reduction rows
#pragma unroll
                for (int kk = 0; kk < QL; ++kk) {
                    if (!slot_on[kk]) continue;
                    const int slot_k = NG * kk + gid;
                    float lr[G];
#pragma unroll
                    for (int x = 0; x < G; ++x) lr[x] = l[kk][x];
                    for (int off = P.kvh; off < 32; off <<= 1)
#pragma unroll
                        for (int x = 0; x < G; ++x) lr[x] += __shfl_xor_sync(0xffffffffu, lr[x], off);
                    if (lane < P.kvh)
#pragma unroll
                        for (int x = 0; x < G; ++x) red[ew][lane * G + x] = lr[x];
                    epi_sync(bar_id);
                    if (rho < P.q_heads) {
                        const float lh = red[0][rho] + red[1][rho] + red[2][rho] + red[3][rho];
                        red[0][rho] = lh;  // after reading red[*][rho]
                        if (P.lse)
                            P.lse[slot_row[kk] * P.q_heads + rho] = (ctl.mst[gid][kk][rho] + log2f(lh)) * LN2;
                    }
                    epi_sync(bar_id);
                    uint16_t* orow = P.out + (size_t)slot_row[kk] * P.q_heads * 128 + rho;
                    for (int c = 0; c < nch; ++c) {
                        float v[16];
                        tmem_ld16(tmem + lane_off + (uint32_t)(P.ns_bufs * P.n_pad + slot_k * P.n_pad + 16 * c), v);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const int h = 16 * c + x;
                            if (h < P.q_heads) orow[(size_t)h * 128] = f32_to_bf16(v[x] / red[0][h]);
                        }
                    }
                    epi_sync(bar_id);
                    slot_on[kk] = false;
                }
                fence_before();
            }
        }
    }

    // ---- shutdown: drain what this CTA started, then free TMEM ----
    __syncwarp();
    if (*abort_flag) {
        if (tid == 0) flag_status(P.status, 6 /* QSA_ERR_TIMEOUT */);
        volatile int no_abort = 0;
        const uint64_t drain_ns = wait_ns < 1000000000ull ? wait_ns : 1000000000ull;
        if (warp == 0 && lane == 0 && q_issued > 0)  // the last query tiles' copy
            mbar_wait(bar_addr(ctl.q_full), (uint32_t)((q_issued - 1) & 1), &no_abort, drain_ns);
        if ((warp == 1 || warp == 3) && lane == 0) {  // the last tiles' copies, stage by stage
            const int nst = warp == 3 ? P.kst : P.vst;
            const uint64_t* full = warp == 3 ? ctl.k_full : ctl.v_full;
            for (int j = kv_issued > nst ? kv_issued - nst : 0; j < kv_issued; ++j)
                mbar_wait(bar_addr(full[j % nst]), (uint32_t)((j / nst) & 1), &no_abort, drain_ns);
        }
        if (warp == 2 && lane == 0) {
            umma_commit(bar_addr(ctl.drain));
            mbar_wait(bar_addr(ctl.drain), 0, &no_abort, drain_ns);
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 3) tmem_dealloc(tmem, (uint32_t)P.tmem_cols);
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

// K or V cache [tokens][kv_heads][128] bf16 as a 3-D map (dims, kv head,
// token); box = 64 dims x kv_heads x pt tokens, 128-byte swizzle.
bool make_kv_map(CUtensorMap* m, const void* base, uint64_t tokens, int kvh, int pt) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)kvh, tokens};
    cuuint64_t strides[2] = {256, (cuuint64_t)kvh * 256};
    cuuint32_t box[3] = {64, (cuuint32_t)kvh, (cuuint32_t)pt};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries [rows][128] bf16; box = 64 dims x q_heads rows.
bool make_q_map(CUtensorMap* m, const void* base, uint64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count_now() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

std::atomic<int> g_attn_fault_mode{0};
std::atomic<uint64_t> g_attn_fault_wait_ns{WAIT_NS};

template <int G, int QS>
cudaError_t launch_g(Params p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, size_t smem,
                     int grid, cudaStream_t st) {
    auto kern = attention_tc_kernel<G, QS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    note_launch();
    kern<<<grid, THREADS, smem, st>>>(tk, tv, tq, p);
    return cudaGetLastError();
}

}  // namespace

void set_attention_fault_injection(int mode, uint64_t wait_ns) {
    g_attn_fault_wait_ns.store(wait_ns, std::memory_order_relaxed);
    g_attn_fault_mode.store(mode, std::memory_order_relaxed);
}

// Shapes the tensor-core attention takes: a power-of-two GQA group (a row's G
// logit columns then sit inside one 16-column TMEM chunk), at most 128 query
// heads, and 32-bit TMA row coordinates.
bool attention_tc_supported(const LayerDims& L, int batch, int64_t cap, int64_t nq) {
    const int G = L.q_heads / L.kv_heads;
    return (G == 1 || G == 2 || G == 4 || G == 8 || G == 16) && L.q_heads <= MAX_NPAD &&
           L.head_dim == 128 && (int64_t)batch * cap < INT32_MAX &&
           (int64_t)batch * nq * L.q_heads < INT32_MAX;
}

cudaError_t launch_sparse_attention_tc(const LayerDims& L, int batch, const uint16_t* q, int64_t q_begin, int64_t nq,
                                       const uint16_t* kc, const uint16_t* vc, int64_t cap, const int32_t* sel,
                                       const int32_t* nsel, uint16_t* out, float* lse, int32_t* status,
                                       cudaStream_t st) {
    if (nq <= 0 || batch <= 0) return cudaSuccess;
    const int kvh = L.kv_heads, G = L.q_heads / kvh;
    Params p{};
    p.sel = sel;
    p.nsel = nsel;
    p.out = out;
    p.lse = lse;
    p.status = status;
    p.rows = (int64_t)batch * nq;
    p.nq = nq;
    p.q_begin = q_begin;
    p.cap = cap;
    p.r = L.r;
    p.kB = L.kB;
    p.kvh = kvh;
    p.q_heads = L.q_heads;
    p.n_pad = (L.q_heads + 15) / 16 * 16;
    p.pt = std::min(L.r, ROWS / kvh);
    p.npb = (L.r + p.pt - 1) / p.pt;
    p.pr = (p.pt * kvh + 7) / 8 * 8;
    p.ppt = ROWS / p.pr;
    p.scale_log2 = L.sm_scale * LOG2E;
    const int QS = G == 16 ? 2 : 4;
    p.ns_bufs = 2;  // with P.V one tile behind S, more buffers do not help (measured)
    int cols = (p.ns_bufs + QS) * p.n_pad, tc = 32;
    while (tc < cols) tc <<= 1;
    p.tmem_cols = tc;
    // Shared memory: K ring, V ring, Q slots, two P buffers, tile descriptions, control.
    const size_t qb = (size_t)QS * p.n_pad * 256, pb = 2 * (size_t)p.n_pad * 256;
    const size_t fixed = qb + pb + INFO_DEPTH * sizeof(TileInfo) + sizeof(Ctl) + 1024;
    const size_t limit = 227 * 1024;
    // Ring depths: V tiles wait for the softmax before they are consumed, so
    // their ring is the deeper one. Then the selection rows, if they fit.
    int kst = 2, vst = 3;
    while (fixed + (size_t)(kst + vst) * TILE_BYTES > limit) {
        if (vst > kst) --vst;
        else --kst;
    }
    if (kst < 1 || vst < 1) return cudaErrorInvalidConfiguration;
    const size_t selb = ((size_t)QS * L.kB * 4 + 127) / 128 * 128;
    p.stage_sel = fixed + (size_t)(kst + vst) * TILE_BYTES + selb <= limit ? 1 : 0;
    p.kst = kst;
    p.vst = vst;
    p.off_v = (uint32_t)(kst * TILE_BYTES);
    p.off_q = p.off_v + (uint32_t)(vst * TILE_BYTES);
    p.off_p = p.off_q + (uint32_t)qb;
    p.off_sel = p.off_p + (uint32_t)pb;
    p.off_info = p.off_sel + (uint32_t)(p.stage_sel ? selb : 0);
    p.off_ctl = p.off_info + (uint32_t)(INFO_DEPTH * sizeof(TileInfo));
    const size_t smem = (size_t)p.off_ctl + sizeof(Ctl) + 1024;
    const int fmode = g_attn_fault_mode.load(std::memory_order_relaxed);
    p.fault_mode = fmode;
    p.wait_ns = fmode ? g_attn_fault_wait_ns.load(std::memory_order_relaxed) : WAIT_NS;

    CUtensorMap tk, tv, tq;
    const uint64_t tokens = (uint64_t)batch * cap;
    if (!make_kv_map(&tk, kc, tokens, kvh, p.pt) || !make_kv_map(&tv, vc, tokens, kvh, p.pt) ||
        !make_q_map(&tq, q, (uint64_t)batch * nq * L.q_heads, L.q_heads))
        return cudaErrorInvalidValue;
    const int64_t ngroups = (p.rows + QS - 1) / QS;
    const int grid = (int)std::min<int64_t>(sm_count_now(), ngroups);
    switch (G) {
        case 1: return launch_g<1, 4>(p, tk, tv, tq, smem, grid, st);
        case 2: return launch_g<2, 4>(p, tk, tv, tq, smem, grid, st);
        case 4: return launch_g<4, 4>(p, tk, tv, tq, smem, grid, st);
        case 8: return launch_g<8, 4>(p, tk, tv, tq, smem, grid, st);
        case 16: return launch_g<16, 2>(p, tk, tv, tq, smem, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qsa
