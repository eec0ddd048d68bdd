// Warp-level sparse attention over selected blocks (shared by the prefill
// and decode kernels): one warp attends one query's G heads of one kv head
// over a range of units (selection entries and the current block's tail),
// with K/V tokens streamed through a 2-stage cp.async ring of 16-token
// chunks; per-warp online-softmax state and the helpers that park, merge,
// store and write it.
#pragma once
#include "kernels.h"

namespace qsa {
namespace {

constexpr int CT = 16;                    // tokens per chunk
constexpr int STAGES = 2;
constexpr int STAGE_BYTES = CT * 256 * 2; // K and V rows
constexpr int WARP_SMEM = STAGES * STAGE_BYTES + STAGES * CT * 8 + 64;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct Work {
    const uint16_t* q;     // first query head of the group: [G][128]
    const void* kc;        // sequence base of the K cache (bf16, or fp8 codes)
    const void* vc;
    const float* ks;       // fp8 caches: sequence base of the row scales [cap][kv_heads]
    const float* vs;
    const uint16_t* hot_k; // host-offloaded caches: sequence base of the HBM hot blocks
    const uint16_t* hot_v; //   [hot_blocks + 1][r][kv_heads][128] (the last one the tail slot)
    const int32_t* tags;   //   and of their tags [hot_blocks + 1]
    int32_t hot_blocks;
    int32_t tail_hrow0;    //   first hot row of the tail slot when it holds the tail, else -1
    const int32_t* sel;    // selection row
    int64_t i;             // query position
    int64_t cur;           // its block, i / r
    int nsel;              // valid selection entries (clamped)
    int tail_unit;         // the unit that stands for the current block's tail
    int u0, u1;            // unit range; unit u != tail_unit is selection entry u if u < nsel, else empty
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

// 8x8 b16 matrix transpose in the mma fragment layout (lane l holds row l/4,
// columns 2 (l % 4) and 2 (l % 4) + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
    return d;
}

// Query fragments (B operand of S^T = K Q^T) of the G heads at q: column =
// head 8 nt + g, k rows = dims 16 ks + 2 t (+1) and 16 ks + 8 + 2 t (+1).
template <int NT>
__device__ __forceinline__ void load_q_frags(const uint16_t* q, int G, int lane, uint32_t (&qb)[NT][8][2]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = 8 * nt + g;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[nt][ks][0] = h < G ? *reinterpret_cast<const uint32_t*>(q + h * kHeadDim + ks * 16 + 2 * t) : 0u;
            qb[nt][ks][1] = h < G ? *reinterpret_cast<const uint32_t*>(q + h * kHeadDim + ks * 16 + 8 + 2 * t) : 0u;
        }
    }
}

// As load_q_frags, converted to f16 (exact while |q| < 65504, the f16 range).
template <int NT>
__device__ __forceinline__ void load_q_frags_f16(const uint16_t* q, int G, int lane, uint32_t (&qb)[NT][8][2]) {
    load_q_frags<NT>(q, G, lane, qb);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int k = 0; k < 2; ++k) qb[nt][ks][k] = pack_f16x2(bf16_lo(qb[nt][ks][k]), bf16_hi(qb[nt][ks][k]));
}

// fp8 caches, per warp: an f16 tile (K rows then V rows, 256-byte swizzled
// rows as in the bf16 ring) and STAGES staging slots of codes and scales.
constexpr int Q8_TILE = CT * 256 * 2;
constexpr int Q8_STAGE = CT * 128 * 2 + CT * 8;  // K codes, V codes, K scales, V scales
static_assert(Q8_TILE + STAGES * Q8_STAGE + 8 <= WARP_SMEM, "fp8 layout fits the warp's area");

// The warp's units [u0, u1) against the query fragments qb. sel_lane: lane l
// holds selection entry u0 + l when that unit is a selection entry (any
// value otherwise); later entries are read when their chunk is issued.
// Q8: the caches hold FP8 E4M3 codes with per-row scales; each chunk is
// gathered as codes, then converted into the warp's f16 tile (values times
// their row scale), the logits take the key rows' scales, and both products
// run in f16 (qb then holds f16 fragments).
// HOT: the caches kc, vc are in host memory and the HBM hot cache holds some
// blocks: hot_lane (lane l, for the warp's unit u0 + l) is the hot slot of that
// selection entry's block, or -1 (read from host memory); entries past the
// warp's first 32 units look their slot's tag up when issued, and the tail
// comes from the tail slot when w.tail_hrow0 >= 0.
template <int NT, bool Q8 = false, bool HOT = false>
__device__ __forceinline__ void warp_attend(const Work& w, uint8_t* wsm, int lane, const uint32_t (&qb)[NT][8][2],
                                            int32_t sel_lane, WarpState<NT>& st, int32_t hot_lane = -1) {
    uint16_t* ring = reinterpret_cast<uint16_t*>(wsm);
    uint32_t* vmask = reinterpret_cast<uint32_t*>(
        Q8 ? wsm + Q8_TILE + STAGES * Q8_STAGE : wsm + STAGES * STAGE_BYTES + STAGES * CT * 8);
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t q8_stage_s = ring_s + Q8_TILE;  // stage k at q8_stage_s + k * Q8_STAGE
    const int g = lane >> 2;
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
    const int64_t cur = w.cur;
    const int64_t row_stride = (int64_t)w.kv_heads * kHeadDim;

    const int ntok_i = (int)ntok;
    // Chunk c: lane l (and l + 16) resolves token l of the chunk; the valid
    // mask is a ballot and the row addresses come by shuffle.
    auto issue = [&](int c) {
        const int stg = c % STAGES;
        const int pl = c * CT + (lane & (CT - 1));  // lanes >= CT mirror lanes < CT
        const int u = w.u0 + pl / w.r;
        const int32_t b_pre = __shfl_sync(0xffffffffu, sel_lane, (u - w.u0) & 31);
        const int32_t hot_pre = HOT ? __shfl_sync(0xffffffffu, hot_lane, (u - w.u0) & 31) : -1;
        int32_t tk = -1;  // token (the cache capacity is below 2^31 tokens)
        int32_t hrow = -1;  // HOT: the token's row in the hot cache, or -1
        if (pl < ntok_i) {
            const int e = pl % w.r;
            if (u == w.tail_unit) {
                const int64_t tt = cur * w.r + e;
                if (tt <= w.i) {
                    tk = (int32_t)tt;
                    if (HOT && w.tail_hrow0 >= 0) hrow = w.tail_hrow0 + e;
                }
            } else if (u < w.nsel) {
                const int32_t b = u - w.u0 < 32 ? b_pre : w.sel[u];
                if (b >= 0 && (int64_t)b < cur) {
                    tk = b * w.r + e;
                    if (HOT) {
                        int32_t slot = hot_pre;
                        if (u - w.u0 >= 32) {
                            slot = b % w.hot_blocks;
                            if (__ldcg(w.tags + slot) != b) slot = -1;
                        }
                        if (slot >= 0) hrow = slot * w.r + e;
                    }
                }
            }
        }
        const uint32_t valid = __ballot_sync(0xffffffffu, tk >= 0) & ((1u << CT) - 1u);
        if (lane == 0) vmask[stg] = valid;
        if (Q8) {
            // Codes: 16 rows x 128 bytes per cache, 16-byte pieces; scales: lanes
            // 0-15 fetch the K row scales, lanes 16-31 the V row scales.
            const uint32_t kb8 = q8_stage_s + stg * Q8_STAGE, vb8 = kb8 + CT * 128;
            const uint8_t* kc8 = static_cast<const uint8_t*>(w.kc);
            const uint8_t* vc8 = static_cast<const uint8_t*>(w.vc);
#pragma unroll
            for (int k = 0; k < (CT * 8) / 32; ++k) {
                const int idx = lane + k * 32;
                const int row = idx >> 3, ch = idx & 7;
                const int32_t tkr = __shfl_sync(0xffffffffu, tk, row);
                const bool ok = tkr >= 0;
                const size_t off = (size_t)(ok ? tkr : 0) * row_stride + (size_t)w.g * kHeadDim + ch * 16;
                cp_async16_zfill(kb8 + row * 128 + ch * 16, kc8 + off, ok);
                cp_async16_zfill(vb8 + row * 128 + ch * 16, vc8 + off, ok);
            }
            const int row = lane & (CT - 1);
            const int32_t tkr = __shfl_sync(0xffffffffu, tk, row);
            const bool ok = tkr >= 0;
            const size_t so = (size_t)(ok ? tkr : 0) * w.kv_heads + w.g;
            cp_async4_zfill(kb8 + 2 * CT * 128 + (lane < CT ? 0 : CT * 4) + row * 4, (lane < CT ? w.ks : w.vs) + so, ok);
        } else {
            const uint32_t kbase = ring_s + stg * STAGE_BYTES;
            const uint32_t vbase = kbase + CT * 256;
            const uint16_t* kc16 = static_cast<const uint16_t*>(w.kc);
            const uint16_t* vc16 = static_cast<const uint16_t*>(w.vc);
#pragma unroll
            for (int k = 0; k < (CT * 16) / 32; ++k) {
                const int idx = lane + k * 32;
                const int row = idx >> 4, ch = idx & 15;
                const int32_t tkr = __shfl_sync(0xffffffffu, tk, row);
                const bool ok = tkr >= 0;
                const uint16_t* ksrc = kc16;
                const uint16_t* vsrc = vc16;
                int32_t src_row = ok ? tkr : 0;
                if (HOT) {
                    const int32_t hr = __shfl_sync(0xffffffffu, hrow, row);
                    if (hr >= 0) {
                        ksrc = w.hot_k;
                        vsrc = w.hot_v;
                        src_row = hr;
                    }
                }
                const size_t off = (size_t)src_row * row_stride + (size_t)w.g * kHeadDim + ch * 8;
                cp_async16_zfill(kbase + swz256(row, ch), ksrc + off, ok);
                cp_async16_zfill(vbase + swz256(row, ch), vsrc + off, ok);
            }
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
        uint32_t kbase = ring_s + stg * STAGE_BYTES;
        float ksc0 = 1.f, ksc1 = 1.f;  // fp8: the key rows' scales of tokens g, g + 8
        if (Q8) {
            // Codes -> f16 tiles: K exact, V times its row scale (rounded to
            // f16); lane handles 16-byte code pieces (16 values) of rows idx / 8.
            kbase = ring_s;
            const uint8_t* st8 = wsm + Q8_TILE + stg * Q8_STAGE;
            const float* ksc = reinterpret_cast<const float*>(st8 + 2 * CT * 128);
            const float* vsc = ksc + CT;
#pragma unroll
            for (int k = 0; k < (CT * 8) / 32; ++k) {
                const int idx = lane + k * 32;
                const int row = idx >> 3, ch = idx & 7;
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {
                    const uint4 c16 = *reinterpret_cast<const uint4*>(st8 + kv * CT * 128 + row * 128 + ch * 16);
                    const uint32_t w4[4] = {c16.x, c16.y, c16.z, c16.w};
                    uint32_t h[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        h[2 * j] = e4m3x2_to_f16x2((uint16_t)(w4[j] & 0xFFFFu));
                        h[2 * j + 1] = e4m3x2_to_f16x2((uint16_t)(w4[j] >> 16));
                    }
                    if (kv == 1) {  // V: times the row's scale, in f16
                        const uint32_t s2 = pack_f16x2(vsc[row], vsc[row]);
#pragma unroll
                        for (int j = 0; j < 8; ++j) h[j] = hmul2(h[j], s2);
                    }
                    uint8_t* tile = wsm + kv * CT * 256;
                    *reinterpret_cast<uint4*>(tile + swz256(row, 2 * ch)) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4*>(tile + swz256(row, 2 * ch + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
                }
            }
            ksc0 = ksc[g];
            ksc1 = ksc[g + 8];
            __syncwarp();
        }
        const uint32_t vbase = kbase + CT * 256;
        const uint32_t valid = vmask[stg];

        // S^T = K Q^T: rows = tokens g, g + 8; columns = heads 8 nt + 2 t (+1).
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
        // (two independent accumulation chains over the k-steps, summed after)
        float s2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s2[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(kbase + swz256(krow, ks * 2 + kch), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (Q8)
                    mma_f16_16816((ks & 1) ? s2[nt] : s[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
                else
                    mma_bf16_16816((ks & 1) ? s2[nt] : s[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
        // Online softmax per head (log2 domain); a head's 16 tokens sit in the
        // 8 lanes with the same t.
        const bool v0 = (valid >> g) & 1u, v1 = (valid >> (g + 8)) & 1u;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float x0 = v0 ? s[nt][e] * ksc0 * w.scale_log2 : -INFINITY;
                const float x1 = v1 ? s[nt][2 + e] * ksc1 * w.scale_log2 : -INFINITY;
                float mx = fmaxf(x0, x1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(st.m[nt][e], mx);
                const float corr = (m_new == -INFINITY) ? 1.f : ex2_approx(st.m[nt][e] - m_new);
                const float p0 = (x0 == -INFINITY) ? 0.f : ex2_approx(x0 - m_new);
                const float p1 = (x1 == -INFINITY) ? 0.f : ex2_approx(x1 - m_new);
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
            pb[nt][0] = movmatrix_trans(Q8 ? pack_f16x2(s[nt][0], s[nt][1]) : pack_bf16x2(s[nt][0], s[nt][1]));
            pb[nt][1] = movmatrix_trans(Q8 ? pack_f16x2(s[nt][2], s[nt][3]) : pack_bf16x2(s[nt][2], s[nt][3]));
        }
        // O^T += V^T P^T: rows = dims 16 i + g (+8), columns = heads.
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(vbase + swz256(vrow, 2 * i + vch), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (Q8)
                    mma_f16_16816(st.o[nt][i], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                else
                    mma_bf16_16816(st.o[nt][i], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
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

template <int NT>
__device__ __forceinline__ void store_state_hd(const WarpState<NT>& st, int G, float* dst, int lane) {
    const int gq = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nt + 2 * t + e;
            if (h >= G) continue;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                dst[h * kHeadDim + 16 * i + gq] = st.o[nt][i][e];
                dst[h * kHeadDim + 16 * i + gq + 8] = st.o[nt][i][2 + e];
            }
            if (gq == 0) {
                dst[G * kHeadDim + h] = st.m[nt][e];
                dst[G * kHeadDim + G + h] = st.l[nt][e];
            }
        }
}

}  // namespace
}  // namespace qsa
