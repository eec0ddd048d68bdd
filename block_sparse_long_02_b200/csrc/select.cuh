// Exact top-k selection over scores, shared by the row-select kernels (topk.cu)
// and the decode step (decode.cu). Rank = (score descending, index ascending).
// Scores map to order-preserving 32-bit keys; a radix select finds the k-th key
// in three digit levels (11, 11, 10 bits): a shared-memory histogram of the top
// digit, collection of the entries above it (sure winners) and in it
// (candidates), then refinement on the candidates in shared memory; ties at the
// threshold take the lowest indices; the winners are bitonic-sorted ascending.
// If the candidates overflow shared memory, the digits are refined by re-reading
// the row and an order-preserving compaction pass writes the output.
#pragma once

#include "common.cuh"

namespace qsa {
namespace {

constexpr int T = 512;           // threads per CTA of the select routines
constexpr int NW = T / 32;
constexpr int BINS = 2048;
constexpr int CAND = 4096;
static_assert(T * 4 == BINS, "find_bin: 4 bins per thread");

struct SelSmem {
    uint32_t hist[BINS];
    uint32_t cand_key[CAND];
    int32_t cand_idx[CAND];
    int32_t out[kMaxKB];
    uint32_t wsum[NW];
    int32_t n_out, n_cand, bin, above, ties;
};

// Finds bin B (counting from the top) with above(B) < need <= above(B) + hist[B].
// Result in sm.bin / sm.above. Must be called by all T threads; nbins is 1024
// or 2048. Thread t owns bins [t * per, (t + 1) * per) (one vector load, no
// bank conflicts); a suffix scan over the threads gives every thread the
// count above its bins, and the one thread whose bins hold the need-th key
// walks them.
template <int PER, typename Sm>
__device__ __forceinline__ void find_bin_per(Sm& sm, uint32_t need) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    uint32_t h[4];
    if (PER == 4) {
        const uint4 x = reinterpret_cast<const uint4*>(sm.hist)[tid];
        h[0] = x.x, h[1] = x.y, h[2] = x.z, h[3] = x.w;
    } else {
        const uint2 x = reinterpret_cast<const uint2*>(sm.hist)[tid];
        h[0] = x.x, h[1] = x.y, h[2] = 0u, h[3] = 0u;
    }
    const uint32_t sum = h[0] + h[1] + h[2] + h[3];
    uint32_t suf = sum;  // inclusive suffix over this warp's lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
    }
    if (lane == 0) sm.wsum[w] = suf;
    __syncthreads();
    uint32_t above_w = 0;
    for (int k = w + 1; k < NW; ++k) above_w += sm.wsum[k];
    const uint32_t incl = suf + above_w;  // keys in bins >= my first bin
    const uint32_t above = incl - sum;    // keys in bins above mine
    if (above < need && need <= incl) {
        uint32_t acc = above;
#pragma unroll
        for (int b = PER - 1; b >= 0; --b) {
            if (acc + h[b] >= need) {
                sm.bin = tid * PER + b;
                sm.above = (int32_t)acc;
                break;
            }
            acc += h[b];
        }
    }
    __syncthreads();
}

template <typename Sm>
__device__ void find_bin(Sm& sm, int nbins, uint32_t need) {
    __syncthreads();
    if (nbins == 2048)
        find_bin_per<4>(sm, need);
    else
        find_bin_per<2>(sm, need);
}

template <typename Sm>
__device__ void clear_hist(Sm& sm) {
    for (int b = threadIdx.x; b < BINS; b += T) sm.hist[b] = 0;
    __syncthreads();
}

// Exclusive prefix of `flag` over the CTA in thread order; returns the CTA total.
__device__ uint32_t cta_scan(SelSmem& sm, bool flag, uint32_t& prefix) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
    const uint32_t wpre = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) sm.wsum[w] = __popc(ballot);
    __syncthreads();
    uint32_t base = 0, total = 0;
    for (int k = 0; k < NW; ++k) {
        const uint32_t v = sm.wsum[k];
        if (k < w) base += v;
        total += v;
    }
    __syncthreads();
    prefix = base + wpre;
    return total;
}

// Slow general path: exact digits by re-reading the row, then an
// order-preserving compaction that writes the sorted selection.
__device__ void select_general(SelSmem& sm, const float* x, int64_t n, int kB, uint32_t b1,
                               uint32_t need1, int32_t* sel) {
    const int tid = threadIdx.x;
    // Level 2.
    clear_hist(sm);
    for (int64_t i = tid; i < n; i += T) {
        const uint32_t k = float_key(x[i]);
        if ((k >> 21) == b1) atomicAdd(&sm.hist[(k >> 10) & 2047u], 1u);
    }
    find_bin(sm, 2048, need1);
    const uint32_t b2 = sm.bin;
    const uint32_t need2 = need1 - sm.above;
    clear_hist(sm);
    const uint32_t p2 = (b1 << 11) | b2;
    for (int64_t i = tid; i < n; i += T) {
        const uint32_t k = float_key(x[i]);
        if ((k >> 10) == p2) atomicAdd(&sm.hist[k & 1023u], 1u);
    }
    find_bin(sm, 1024, need2);
    const uint32_t key_t = (p2 << 10) | (uint32_t)sm.bin;
    const uint32_t need_t = need2 - sm.above;  // ties at key_t to take, lowest index first
    // Ordered compaction.
    uint32_t taken = 0, ties = 0;
    for (int64_t base = 0; base < n; base += T) {
        const int64_t i = base + tid;
        uint32_t k = 0;
        if (i < n) k = float_key(x[i]);
        const bool is_tie = i < n && k == key_t;
        uint32_t tie_pre;
        const uint32_t tie_tot = cta_scan(sm, is_tie, tie_pre);
        const bool take = i < n && (k > key_t || (is_tie && ties + tie_pre < need_t));
        uint32_t pre;
        const uint32_t tot = cta_scan(sm, take, pre);
        if (take) sel[taken + pre] = (int32_t)i;
        taken += tot;
        ties += tie_tot;
    }
    for (int k = (int)taken + tid; k < kB; k += T) sel[k] = -1;
}

__device__ void finish_from_candidates(SelSmem& sm, int nc, uint32_t b1, uint32_t need1, int kB,
                                       int32_t* sel);

// Sorts sm.out[0, kB) ascending (bitonic network, padded with INT_MAX to a
// power of two). For up to T keys each thread holds one key; compare-exchange
// steps with a partner in the same warp use shuffles, the others go through
// shared memory.
__device__ void sort_out(SelSmem& sm, int kB) {
    const int tid = threadIdx.x;
    int P = 1;
    while (P < kB) P <<= 1;
    if (P <= T) {
        int32_t v = tid < kB ? sm.out[tid] : 0x7fffffff;
        for (int k = 2; k <= T; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                int32_t o;
                if (j >= 32) {
                    __syncthreads();
                    sm.out[tid] = v;
                    __syncthreads();
                    o = sm.out[tid ^ j];
                } else {
                    o = __shfl_xor_sync(0xffffffffu, v, j);
                }
                const bool up = (tid & k) == 0, lower = (tid & j) == 0;
                v = (lower == up) ? min(v, o) : max(v, o);
            }
        }
        __syncthreads();
        sm.out[tid] = v;
        __syncthreads();
        return;
    }
    for (int k = kB + tid; k < P; k += T) sm.out[k] = 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += T) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const int32_t a = sm.out[i], b = sm.out[ixj];
                    const bool up = (i & k) == 0;
                    if ((a > b) == up) {
                        sm.out[i] = b;
                        sm.out[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Sorts a[0, n) (shared memory, room for max(n, T) entries) ascending: the
// bitonic network of sort_out over the next power of two above n only.
__device__ void sort_ints(int32_t* a, int n) {
    const int tid = threadIdx.x;
    int P = 1;
    while (P < n) P <<= 1;
    if (P <= T) {
        int32_t v = tid < n ? a[tid] : 0x7fffffff;
        for (int k = 2; k <= P; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                int32_t o;
                if (j >= 32) {
                    __syncthreads();
                    a[tid] = v;
                    __syncthreads();
                    o = a[tid ^ j];
                } else {
                    o = __shfl_xor_sync(0xffffffffu, v, j);
                }
                const bool up = (tid & k) == 0, lower = (tid & j) == 0;
                v = (lower == up) ? min(v, o) : max(v, o);
            }
        }
        __syncthreads();
        if (tid < n) a[tid] = v;
        __syncthreads();
        return;
    }
    for (int k = n + tid; k < P; k += T) a[k] = 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += T) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const int32_t x = a[i], y = a[ixj];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) {
                        a[i] = y;
                        a[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Exact top-k_B of one row of n scores (x[i] = score of block i), written
// ascending to sel, nsel = min(n, k_B). One CTA of T threads.
__device__ void select_row(SelSmem& sm, const float* x, int64_t n, int kB, int32_t* sel,
                           int32_t* nsel) {
    const int tid = threadIdx.x;
    if (n <= kB) {
        for (int k = tid; k < kB; k += T) sel[k] = k < n ? k : -1;
        if (tid == 0) *nsel = (int32_t)(n > 0 ? n : 0);
        return;
    }
    if (tid == 0) *nsel = kB;
    // Level 1.
    clear_hist(sm);
    for (int64_t i = tid; i < n; i += T) atomicAdd(&sm.hist[float_key(x[i]) >> 21], 1u);
    find_bin(sm, BINS, (uint32_t)kB);
    const uint32_t b1 = sm.bin;
    const uint32_t need1 = (uint32_t)kB - (uint32_t)sm.above;
    if (tid == 0) {
        sm.n_out = 0;
        sm.n_cand = 0;
    }
    __syncthreads();
    for (int64_t i = tid; i < n; i += T) {
        const uint32_t k = float_key(x[i]);
        const uint32_t b = k >> 21;
        if (b > b1) {
            sm.out[atomicAdd(&sm.n_out, 1)] = (int32_t)i;
        } else if (b == b1) {
            const int p = atomicAdd(&sm.n_cand, 1);
            if (p < CAND) {
                sm.cand_key[p] = k;
                sm.cand_idx[p] = (int32_t)i;
            }
        }
    }
    __syncthreads();
    const int nc = sm.n_cand;
    if (nc > CAND) {
        select_general(sm, x, n, kB, b1, need1, sel);
        return;
    }
    finish_from_candidates(sm, nc, b1, need1, kB, sel);
}

// Completes a selection whose sure winners (keys above the threshold digit b1)
// are already in sm.out[0, sm.n_out) and whose nc <= CAND candidates (keys in
// digit b1) are in sm.cand_key / sm.cand_idx: refines the threshold on the
// remaining 21 key bits, takes ties at the threshold by lowest index, sorts the
// k_B winners ascending and writes them to sel. need1 = k_B - sm.n_out.
// Warp-aggregated append to a shared-memory list: one atomic per warp.
// Every lane of the warp must call it.
__device__ __forceinline__ void warp_push(SelSmem& sm, bool flag, int32_t value) {
    const int lane = threadIdx.x & 31;
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    int base = 0;
    if (lane == 0 && bal) base = atomicAdd(&sm.n_out, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (flag) sm.out[base + __popc(bal & ((1u << lane) - 1u))] = value;
}

__device__ void finish_from_candidates(SelSmem& sm, int nc, uint32_t b1, uint32_t need1, int kB,
                                       int32_t* sel) {
    const int tid = threadIdx.x;
    // Level 2 on the candidates. (Loops run the same trip count in every
    // thread, so the warp-wide appends see full warps.)
    clear_hist(sm);
    for (int c = tid; c < nc; c += T) atomicAdd(&sm.hist[(sm.cand_key[c] >> 10) & 2047u], 1u);
    find_bin(sm, 2048, need1);
    const uint32_t b2 = sm.bin;
    const uint32_t need2 = need1 - sm.above;
    for (int c0 = 0; c0 < nc; c0 += T) {
        const int c = c0 + tid;
        const bool f = c < nc && ((sm.cand_key[c] >> 10) & 2047u) > b2;
        warp_push(sm, f, f ? sm.cand_idx[c] : 0);
    }
    // Level 3.
    clear_hist(sm);
    for (int c = tid; c < nc; c += T)
        if (((sm.cand_key[c] >> 10) & 2047u) == b2) atomicAdd(&sm.hist[sm.cand_key[c] & 1023u], 1u);
    find_bin(sm, 1024, need2);
    const uint32_t key_t = (b1 << 21) | (b2 << 10) | (uint32_t)sm.bin;
    const uint32_t need_t = need2 - sm.above;
    if (tid == 0) sm.ties = 0;
    __syncthreads();
    int my_ties = 0;
    for (int c0 = 0; c0 < nc; c0 += T) {
        const int c = c0 + tid;
        const uint32_t k = c < nc ? sm.cand_key[c] : 0u;
        const bool f = c < nc && (k >> 10) == (key_t >> 10) && k > key_t;
        warp_push(sm, f, f ? sm.cand_idx[c] : 0);
        my_ties += (c < nc && k == key_t) ? 1 : 0;
    }
    my_ties = (int)warp_sum((uint32_t)my_ties);
    if ((tid & 31) == 0 && my_ties) atomicAdd(&sm.ties, my_ties);
    __syncthreads();
    const int nties = sm.ties;
    for (int c0 = 0; c0 < nc; c0 += T) {
        const int c = c0 + tid;
        bool take = c < nc && sm.cand_key[c] == key_t;
        if (take && (uint32_t)nties != need_t) {
            const int32_t me = sm.cand_idx[c];
            uint32_t rank = 0;
            for (int d = 0; d < nc; ++d)
                rank += (sm.cand_key[d] == key_t && sm.cand_idx[d] < me) ? 1u : 0u;
            take = rank < need_t;
        }
        warp_push(sm, take, take ? sm.cand_idx[c] : 0);
    }
    __syncthreads();
    sort_out(sm, kB);
    for (int k = tid; k < kB; k += T) sel[k] = sm.out[k];
}

}  // namespace
}  // namespace qsa
