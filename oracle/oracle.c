/*
 * QSA layer oracle: a plain, slow, single-threaded CPU statement of what the
 * QSA layer computes, written from the method's description.
 *
 * TEST INFRASTRUCTURE ONLY. It is used by tests/, by __graft_entry__.smoke()
 * and by bench.py's CPU-baseline leg, nothing else. It shares no code with the
 * CUDA path (block_sparse_long_02_b200/); both take their inputs from synth/.
 *
 * Sources (page title, section):
 *   [P1] "QSA (Qwen Sparse Attention)" concept page, "Key math / How it works":
 *        (A) compressed lightweight indexer, (B) sparse core attention, "Config";
 *        "Native trainability via 2-stage continued pretraining" (training section).
 *   [P2] "Qwen Sparse Attention" (LLM architecture gallery), "How block selection
 *        works" (prose and pseudo-code) and the selection-unit / budget table.
 *
 * Arithmetic: bf16 inputs are widened exactly; every sum is taken in fp64; the
 * only roundings are the ones the layer's storage implies: pooled keys and
 * rotated indexer queries are stored as bf16 (round-to-nearest-even, directly
 * from fp64), indexer scores are returned as fp32. Attention is fp64 end to end.
 *
 * Readings where the pages are silent:
 *   - order pool -> RMSNorm -> RoPE; RMSNorm is x * (mean x^2 + eps)^-1/2 * w;
 *   - RoPE pairs dim j with dim j + rope_dims/2 for j < rope_dims/2 ("rotate
 *     half"), theta_j = base^(-2j/rope_dims), angle = pos * theta_j;
 *   - the indexer query is rotated at its own position i;
 *   - block-causal mask: query i scores blocks b < floor(i/r) only;
 *   - ties in the top-k go to the lower block index; the selection is returned
 *     in ascending block order;
 *   - the tail {r*floor(i/r) .. i} is added on top of the k_B blocks;
 *   - one selection per query token, shared by every core head; GQA maps q head
 *     h to kv head floor(h / (q_heads / kv_heads)); softmax scale 1/sqrt(d).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t r, K;             /* block size, token budget              */
    int32_t idx_heads, idx_dim;
    int32_t rope_dims;
    double rope_base;
    double rms_eps;
    int32_t q_heads, kv_heads, head_dim;
    double sm_scale;          /* 0 -> 1/sqrt(head_dim)                 */
} qsa_oracle_cfg;

/* ------------------------------------------------------------------ scalars */
static double bf(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp64 -> bf16 bits: the bf16 value nearest to x, ties to the even significand
 * (IEEE round-to-nearest-even), in one rounding from the exact value.
 * bf16 keeps 8 significant bits with fp32's exponent range: a normal value in
 * [2^e, 2^(e+1)) sits on the grid 2^(e-7); below 2^-126 the grid is the
 * subnormal step 2^-133. A result beyond the largest finite bf16
 * ((2 - 2^-7) * 2^127) is an infinity. */
static uint16_t to_bf16(double x) {
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e); /* a = m * 2^e, m in [0.5, 1): a lies in [2^(e-1), 2^e) */
    const int q = (e - 1 >= -126) ? (e - 1) - 7 : -133;
    const double k = ldexp(a, -q);        /* exact: a scaled by a power of two */
    const double kr = nearbyint(k);       /* nearest integer, ties to even */
    const double y = ldexp(kr, q);        /* exact: at most 9 significant bits */
    if (y > ldexp(255.0, 120)) return (uint16_t)(sign | 0x7F80u);
    const float f = (float)y; /* exact: y is on the bf16 grid, inside fp32's range */
    uint32_t v;
    memcpy(&v, &f, 4);
    return (uint16_t)(sign | ((v >> 16) & 0x7FFFu));
}

/* The storage rounding above, exposed for the pins. */
void qsa_oracle_round_bf16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(x[i]);
}

int64_t qsa_oracle_k_blocks(const qsa_oracle_cfg* c) {
    /* [P1] top-k_B: k_B = ceil(K / r); [P2] budget table: 2,048 / 4 = 512 blocks. */
    return ((int64_t)c->K + c->r - 1) / c->r;
}

/* -------------------------------------------------------------------- RoPE */
/* [P1] (A) "Partial RoPE: RoPE on 64 of 128 dims": rotates dims [0, rope_dims)
 * of x by the angles of position `pos`; dims >= rope_dims pass through. */
void qsa_oracle_rope(const double* x, int dim, int rope_dims, double base, int64_t pos,
                     double* out) {
    const int half = rope_dims / 2;
    for (int j = 0; j < dim; ++j) out[j] = x[j];
    for (int j = 0; j < half; ++j) {
        const double theta = pow(base, -2.0 * (double)j / (double)rope_dims);
        const double a = (double)pos * theta;
        const double c = cos(a), s = sin(a);
        out[j] = x[j] * c - x[j + half] * s;
        out[j + half] = x[j] * s + x[j + half] * c;
    }
}

/* ------------------------------------------------------- a1-a3 key pooling */
/* One complete block. `keys` holds its r raw indexer keys (bf16, [r][dim]);
 * `pos` is the block's first position.
 *   a1 [P1] (A) block compression; [P2] "averages the keys within each complete
 *      block":                      kbar  = (1/r) sum_t k_t
 *   a2 [P1] khat_b = RMSNorm(AvgPool); [P2] "a normalization step for these
 *      pooled keys":                knorm = kbar * (mean_j kbar_j^2 + eps)^-1/2 * w
 *   a3 [P1] partial RoPE after compression; [P2] "RoPE (using the first position
 *      in each block)":             krot  = RoPE_pos(knorm), stored as bf16.
 * Optional outputs expose the intermediate fp64 values for the pins. */
void qsa_oracle_pool_block(const qsa_oracle_cfg* c, const uint16_t* keys, const float* w,
                           int64_t pos, double* kbar_out, double* knorm_out, double* krot_out,
                           uint16_t* out) {
    const int dim = c->idx_dim;
    double* kbar = (double*)malloc(sizeof(double) * 3 * (size_t)dim);
    double* knorm = kbar + dim;
    double* krot = knorm + dim;
    for (int j = 0; j < dim; ++j) {
        double s = 0.0;
        for (int t = 0; t < c->r; ++t) s += bf(keys[(size_t)t * dim + j]);
        kbar[j] = s / (double)c->r;
    }
    double ms = 0.0;
    for (int j = 0; j < dim; ++j) ms += kbar[j] * kbar[j];
    ms /= (double)dim;
    const double rms = sqrt(ms + c->rms_eps);
    for (int j = 0; j < dim; ++j) knorm[j] = kbar[j] / rms * (w ? (double)w[j] : 1.0);
    qsa_oracle_rope(knorm, dim, c->rope_dims, c->rope_base, pos, krot);
    for (int j = 0; j < dim; ++j) {
        if (kbar_out) kbar_out[j] = kbar[j];
        if (knorm_out) knorm_out[j] = knorm[j];
        if (krot_out) krot_out[j] = krot[j];
        if (out) out[j] = to_bf16(krot[j]);
    }
    free(kbar);
}

/* Blocks [0, n_blocks) of one sequence: idx_k is [n >= r*n_blocks][dim]. */
void qsa_oracle_compress(const qsa_oracle_cfg* c, const uint16_t* idx_k, int64_t n_blocks,
                         const float* w, uint16_t* pooled) {
    for (int64_t b = 0; b < n_blocks; ++b)
        qsa_oracle_pool_block(c, idx_k + (size_t)b * c->r * c->idx_dim, w, b * c->r, NULL, NULL,
                              NULL, pooled + (size_t)b * c->idx_dim);
}

/* a3' (reading): the indexer query heads of position `pos` get the same partial
 * rotation at their own position, then are stored as bf16. q: [idx_heads][dim]. */
void qsa_oracle_rotate_query(const qsa_oracle_cfg* c, const uint16_t* q, int64_t pos,
                             uint16_t* out) {
    const int dim = c->idx_dim;
    double* x = (double*)malloc(sizeof(double) * 2 * (size_t)dim);
    double* y = x + dim;
    for (int h = 0; h < c->idx_heads; ++h) {
        for (int j = 0; j < dim; ++j) x[j] = bf(q[(size_t)h * dim + j]);
        qsa_oracle_rope(x, dim, c->rope_dims, c->rope_base, pos, y);
        for (int j = 0; j < dim; ++j) out[(size_t)h * dim + j] = to_bf16(y[j]);
    }
    free(x);
}

/* ---------------------------------------------------------------- a4 score */
/* [P1] (A) block importance: I_ib = sum_h ReLU(<q_i^h, khat_b>), 4 query heads
 * against the 1 shared key head; [P2] pseudo-code "sum(relu(query_head @
 * block_key) for each indexer head)". Block-causal masking is the caller's
 * n_vis = floor(i/r): only blocks b < n_vis are scored. qrot: [idx_heads][dim]. */
void qsa_oracle_scores(const qsa_oracle_cfg* c, const uint16_t* qrot, const uint16_t* pooled,
                       int64_t n_vis, float* scores) {
    const int dim = c->idx_dim;
    for (int64_t b = 0; b < n_vis; ++b) {
        double I = 0.0;
        for (int h = 0; h < c->idx_heads; ++h) {
            double dot = 0.0;
            for (int j = 0; j < dim; ++j)
                dot += bf(qrot[(size_t)h * dim + j]) * bf(pooled[(size_t)b * dim + j]);
            if (dot > 0.0) I += dot;
        }
        scores[b] = (float)I;
    }
}

/* --------------------------------------------------------------- a5 select */
typedef struct {
    float s;
    int32_t b;
} rank_entry;

/* Higher score first; equal scores: lower block index first. */
static int by_rank(const void* pa, const void* pb) {
    const rank_entry* a = (const rank_entry*)pa;
    const rank_entry* b = (const rank_entry*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->b > b->b) - (a->b < b->b);
}

static int by_value(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* [P1] (A) "keep the k_B = ceil(K/r) highest-scoring blocks"; [P2] top_k(scores,
 * k=512). Fewer visible blocks than k_B: all of them ([P1] Config "<= 512").
 * Returns nsel; sel[0..nsel) ascending. */
int64_t qsa_oracle_select(const float* scores, int64_t n_vis, int64_t k_b, int32_t* sel) {
    const int64_t m = n_vis < k_b ? n_vis : k_b;
    if (m <= 0) return 0;
    rank_entry* e = (rank_entry*)malloc(sizeof(rank_entry) * (size_t)n_vis);
    for (int64_t b = 0; b < n_vis; ++b) {
        e[b].s = scores[b];
        e[b].b = (int32_t)b;
    }
    qsort(e, (size_t)n_vis, sizeof(rank_entry), by_rank);
    for (int64_t k = 0; k < m; ++k) sel[k] = e[k].b;
    qsort(sel, (size_t)m, sizeof(int32_t), by_value);
    free(e);
    return m;
}

/* --------------------------------------------------------------- a6 expand */
/* [P1] (A) "expand them back to tokens, and always include the tail of the
 * current block"; [P2] attention_input = flatten(selected_blocks) +
 * current_incomplete_block. Returns |T_i|; tokens ascending. */
int64_t qsa_oracle_token_set(const qsa_oracle_cfg* c, const int32_t* sel, int64_t nsel, int64_t i,
                             int64_t* tokens) {
    int64_t n = 0;
    for (int64_t k = 0; k < nsel; ++k)
        for (int t = 0; t < c->r; ++t) tokens[n++] = (int64_t)sel[k] * c->r + t;
    const int64_t cur = i / c->r;
    for (int64_t t = cur * c->r; t <= i; ++t) tokens[n++] = t;
    return n;
}

/* ----------------------------------------------------- a7 sparse attention */
/* [P1] (B) "Full scaled-dot-product attention restricted to the selected
 * blocks' tokens". q: [q_heads][d]; kc, vc: [>= max token + 1][kv_heads][d].
 * out: [q_heads][d] fp64; lse: [q_heads] natural-log sum of exp (may be NULL). */
void qsa_oracle_attention(const qsa_oracle_cfg* c, const uint16_t* q, const uint16_t* kc,
                          const uint16_t* vc, const int64_t* tokens, int64_t ntok, double* out,
                          double* lse) {
    const int d = c->head_dim, hkv = c->kv_heads, g = c->q_heads / c->kv_heads;
    const double scale = c->sm_scale > 0.0 ? c->sm_scale : 1.0 / sqrt((double)d);
    double* logit = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
    for (int h = 0; h < c->q_heads; ++h) {
        const int kvh = h / g;
        double m = -INFINITY;
        for (int64_t t = 0; t < ntok; ++t) {
            const uint16_t* kr = kc + ((size_t)tokens[t] * hkv + kvh) * d;
            double dot = 0.0;
            for (int j = 0; j < d; ++j) dot += bf(q[(size_t)h * d + j]) * bf(kr[j]);
            logit[t] = dot * scale;
            if (logit[t] > m) m = logit[t];
        }
        double z = 0.0;
        for (int j = 0; j < d; ++j) out[(size_t)h * d + j] = 0.0;
        for (int64_t t = 0; t < ntok; ++t) {
            const double p = exp(logit[t] - m);
            z += p;
            const uint16_t* vr = vc + ((size_t)tokens[t] * hkv + kvh) * d;
            for (int j = 0; j < d; ++j) out[(size_t)h * d + j] += p * bf(vr[j]);
        }
        for (int j = 0; j < d; ++j) out[(size_t)h * d + j] /= z;
        if (lse) lse[h] = m + log(z);
    }
    free(logit);
}

/* ---------------------------------------------------- one query, a3'..a7 */
/* Everything the layer does for query position i of one sequence, given the
 * sequence's pooled keys for the blocks before i. Optional outputs: the scores
 * of the visible blocks ([floor(i/r)] fp32) and the selection. Returns nsel. */
int64_t qsa_oracle_row(const qsa_oracle_cfg* c, int64_t i, const uint16_t* idx_q_row,
                       const uint16_t* pooled, const uint16_t* q_row, const uint16_t* kc,
                       const uint16_t* vc, float* scores_out, int32_t* sel_out, double* out,
                       double* lse) {
    const int64_t n_vis = i / c->r;
    const int64_t k_b = qsa_oracle_k_blocks(c);
    uint16_t* qrot = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)c->idx_heads * c->idx_dim);
    float* scores = (float*)malloc(sizeof(float) * (size_t)(n_vis > 0 ? n_vis : 1));
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k_b > 0 ? k_b : 1));
    int64_t* tokens = (int64_t*)malloc(sizeof(int64_t) * (size_t)(k_b * c->r + c->r));
    qsa_oracle_rotate_query(c, idx_q_row, i, qrot);
    qsa_oracle_scores(c, qrot, pooled, n_vis, scores);
    const int64_t nsel = qsa_oracle_select(scores, n_vis, k_b, sel);
    const int64_t ntok = qsa_oracle_token_set(c, sel, nsel, i, tokens);
    if (out) qsa_oracle_attention(c, q_row, kc, vc, tokens, ntok, out, lse);
    if (scores_out) memcpy(scores_out, scores, sizeof(float) * (size_t)n_vis);
    if (sel_out) memcpy(sel_out, sel, sizeof(int32_t) * (size_t)nsel);
    free(qrot);
    free(scores);
    free(sel);
    free(tokens);
    return nsel;
}

/* ------------------------------------------------------- decode (a8 + row) */
/* One new token at position p (= current length) of one sequence.
 * a8: the new k, v and raw indexer key are appended at p ([P2] "only the QSA
 * layers contribute to the growing KV cache"); the token is then the query p
 * (so its own block's visible part, up to p, is its tail); when p closes a
 * block ((p+1) % r == 0) that block is pooled for the steps that follow
 * (reading: a block is pooled once its last token has been the query).
 * Caches: kc, vc [cap][kv_heads][d]; idx_k_cache [cap][idx_dim];
 * pooled [cap/r][idx_dim]. Returns nsel. */
int64_t qsa_oracle_decode_step(const qsa_oracle_cfg* c, int64_t p, const uint16_t* q_new,
                               const uint16_t* k_new, const uint16_t* v_new,
                               const uint16_t* idx_q_new, const uint16_t* idx_k_new,
                               uint16_t* kc, uint16_t* vc, uint16_t* idx_k_cache,
                               uint16_t* pooled, const float* w, int32_t* sel_out, double* out,
                               double* lse) {
    const size_t kvrow = (size_t)c->kv_heads * c->head_dim;
    memcpy(kc + (size_t)p * kvrow, k_new, sizeof(uint16_t) * kvrow);
    memcpy(vc + (size_t)p * kvrow, v_new, sizeof(uint16_t) * kvrow);
    memcpy(idx_k_cache + (size_t)p * c->idx_dim, idx_k_new, sizeof(uint16_t) * (size_t)c->idx_dim);
    const int64_t nsel =
        qsa_oracle_row(c, p, idx_q_new, pooled, q_new, kc, vc, NULL, sel_out, out, lse);
    if ((p + 1) % c->r == 0) {
        const int64_t b = p / c->r;
        qsa_oracle_pool_block(c, idx_k_cache + (size_t)b * c->r * c->idx_dim, w, b * c->r, NULL,
                              NULL, NULL, pooled + (size_t)b * c->idx_dim);
    }
    return nsel;
}

/* ================================================ low-precision (fp8) caches */
/* Reading (the "Community Quantized Version" section of the "Qwen Sparse
 * Attention" gallery page reports a quantized variant but not its format): K,
 * V and pooled-key rows stored as FP8 E4M3 codes (the OCP 8-bit format: 1 sign
 * bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
 * finite 448, code S.1111.111 = NaN) with one fp32 scale per row:
 *   scale = fl32(max_j |x_j| / 448),  code_j = E4M3_rne_sat(fl32(x_j / scale)),
 *   value_j = E4M3(code_j) * scale;  an all-zero row has scale 0 and codes 0.
 * Both divisions are done in fp64 and rounded once to fp32; since the quotient
 * of two fp32 values rounded to 53 bits and then to 24 bits equals the
 * correctly rounded fp32 quotient (53 >= 2*24 + 2), this is the fp32 division. */

/* The value of an E4M3 code, from the format definition. */
double qsa_oracle_e4m3_value(uint8_t code) {
    const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6); /* subnormal: 0.m * 2^(1 - 7) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* The E4M3 code nearest to y (ties to the even code, i.e. even mantissa),
 * magnitudes above 448 saturating to 448. y must not be NaN. */
uint8_t qsa_oracle_e4m3_encode(double y) {
    const uint8_t sign = y < 0.0 ? 0x80 : 0x00;
    const double a = fabs(y);
    /* Walk the 127 non-negative finite codes (values increase with the code). */
    uint8_t best = 0;
    for (int c = 1; c <= 126; ++c) {
        const double lo = qsa_oracle_e4m3_value((uint8_t)(c - 1)), hi = qsa_oracle_e4m3_value((uint8_t)c);
        if (a >= hi) {
            best = (uint8_t)c;
            continue;
        }
        /* lo <= a < hi */
        const double mid = 0.5 * (lo + hi);
        if (a > mid || (a == mid && (c & 1) == 0)) best = (uint8_t)c;
        else best = (uint8_t)(c - 1);
        return sign | best;
    }
    return sign | best; /* a >= 448: saturate */
}

static float fl32_div(double a, double b) { return (float)(a / b); }

/* Quantizes `rows` rows of `dim` bf16 values. codes: [rows][dim]; scales: [rows]. */
void qsa_oracle_quant_rows(const uint16_t* x, int64_t rows, int dim, uint8_t* codes, float* scales) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + (size_t)r * dim;
        double amax = 0.0;
        for (int j = 0; j < dim; ++j) {
            const double a = fabs(bf(xr[j]));
            if (a > amax) amax = a;
        }
        const float scale = amax > 0.0 ? fl32_div(amax, 448.0) : 0.0f;
        scales[r] = scale;
        for (int j = 0; j < dim; ++j)
            codes[(size_t)r * dim + j] = scale > 0.0f ? qsa_oracle_e4m3_encode(fl32_div(bf(xr[j]), scale)) : 0;
    }
}

/* a7 on fp8 caches: as qsa_oracle_attention with K and V values
 * E4M3(code) * scale (exact in fp64). kc, vc: codes [tokens][kv_heads][d];
 * ks, vs: scales [tokens][kv_heads]. */
void qsa_oracle_attention_q8(const qsa_oracle_cfg* c, const uint16_t* q, const uint8_t* kc, const float* ks,
                             const uint8_t* vc, const float* vs, const int64_t* tokens, int64_t ntok,
                             double* out, double* lse) {
    const int d = c->head_dim, hkv = c->kv_heads, group = c->q_heads / c->kv_heads;
    const double sm = c->sm_scale > 0.0 ? c->sm_scale : 1.0 / sqrt((double)d);
    double* lg = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
    for (int h = 0; h < c->q_heads; ++h) {
        const int kv = h / group;  /* GQA: contiguous groups of q heads */
        double mx = -INFINITY;
        for (int64_t t = 0; t < ntok; ++t) {
            const size_t row = (size_t)tokens[t] * hkv + kv;
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += (qsa_oracle_e4m3_value(kc[row * d + j]) * ks[row]) * bf(q[(size_t)h * d + j]);
            lg[t] = sm * acc;
            if (lg[t] > mx) mx = lg[t];
        }
        double z = 0.0;
        double* o = out + (size_t)h * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (int64_t t = 0; t < ntok; ++t) {
            const double w = exp(lg[t] - mx);
            z += w;
            const size_t row = (size_t)tokens[t] * hkv + kv;
            for (int j = 0; j < d; ++j) o[j] += w * (qsa_oracle_e4m3_value(vc[row * d + j]) * vs[row]);
        }
        for (int j = 0; j < d; ++j) o[j] /= z;
        if (lse) lse[h] = mx + log(z);
    }
    free(lg);
}

/* a4 on fp8 pooled keys: I_ib = sum_h ReLU(<q_i^h, E4M3(code_b) * scale_b>). */
void qsa_oracle_scores_q8(const qsa_oracle_cfg* c, const uint16_t* qrot, const uint8_t* pooled,
                          const float* pscale, int64_t n_vis, float* scores) {
    const int dim = c->idx_dim;
    for (int64_t b = 0; b < n_vis; ++b) {
        double sum = 0.0;
        for (int h = 0; h < c->idx_heads; ++h) {
            double acc = 0.0;
            for (int j = 0; j < dim; ++j)
                acc += (qsa_oracle_e4m3_value(pooled[(size_t)b * dim + j]) * pscale[b]) * bf(qrot[(size_t)h * dim + j]);
            sum += acc > 0.0 ? acc : 0.0; /* ReLU */
        }
        scores[b] = (float)sum;
    }
}

/* ============================================================ training (f3) */
/* [P1] "Native trainability via 2-stage continued pretraining": stage 1 trains
 * the indexer scores to match a block-max-pooled version of the dense teacher
 * attention distribution through a KL loss; stage 2 trains the model and the
 * indexer together under the sparse selection, which needs the gradient of the
 * sparse core attention. Readings (the page names the pieces, not their
 * arithmetic):
 *   - the teacher distribution of query i is the dense causal attention
 *     probability of every token j <= i, averaged over the core heads;
 *   - block-max-pooling keeps, for each block the indexer scores (b < floor(i/r)),
 *     the largest probability among its r tokens; the kept values are then
 *     normalised to sum to 1 so that they form a distribution;
 *   - the loss of query i is KL(target || softmax of the indexer scores over
 *     the same blocks).                                                       */

/* Sparse attention of one query on fp64 operands: q [q_heads][d]; kt, vt
 * [ntok][kv_heads][d] are the rows of the listed tokens in list order. The
 * same arithmetic as qsa_oracle_attention (which widens bf16 exactly). */
void qsa_oracle_attention_f64(const qsa_oracle_cfg* c, const double* q, const double* kt, const double* vt,
                              int64_t ntok, double* out, double* lse) {
    const int d = c->head_dim, hkv = c->kv_heads, g = c->q_heads / c->kv_heads;
    const double scale = c->sm_scale > 0.0 ? c->sm_scale : 1.0 / sqrt((double)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
    for (int h = 0; h < c->q_heads; ++h) {
        const int kvh = h / g;
        double mx = -INFINITY;
        for (int64_t t = 0; t < ntok; ++t) {
            double dot = 0.0;
            for (int j = 0; j < d; ++j) dot += q[(size_t)h * d + j] * kt[((size_t)t * hkv + kvh) * d + j];
            z[t] = dot * scale;
            if (z[t] > mx) mx = z[t];
        }
        double den = 0.0;
        for (int j = 0; j < d; ++j) out[(size_t)h * d + j] = 0.0;
        for (int64_t t = 0; t < ntok; ++t) {
            const double e = exp(z[t] - mx);
            den += e;
            for (int j = 0; j < d; ++j) out[(size_t)h * d + j] += e * vt[((size_t)t * hkv + kvh) * d + j];
        }
        for (int j = 0; j < d; ++j) out[(size_t)h * d + j] /= den;
        if (lse) lse[h] = mx + log(den);
    }
    free(z);
}

/* Gradient of that attention for the upstream gradient dout [q_heads][d], i.e.
 * of L = sum_h <dout_h, out_h>, from out_h = sum_t p_ht v_t, p_ht = softmax over
 * t of z_ht, z_ht = scale <q_h, k_t>:
 *   dL/dv_t   = sum over the heads h of v_t's group of p_ht dout_h;
 *   dL/dz_ht  = p_ht (<dout_h, v_t> - <dout_h, out_h>)   (softmax Jacobian);
 *   dL/dq_h   = scale sum_t dL/dz_ht k_t;
 *   dL/dk_t   = scale sum over the group's heads of dL/dz_ht q_h.
 * dq: [q_heads][d]; dk, dv: [ntok][kv_heads][d], one row per listed token (a
 * token listed twice gets two rows; the caller adds rows of the same token). */
void qsa_oracle_attention_backward_f64(const qsa_oracle_cfg* c, const double* q, const double* kt,
                                       const double* vt, int64_t ntok, const double* dout, double* dq,
                                       double* dk, double* dv) {
    const int d = c->head_dim, hkv = c->kv_heads, g = c->q_heads / c->kv_heads;
    const double scale = c->sm_scale > 0.0 ? c->sm_scale : 1.0 / sqrt((double)d);
    const size_t n_out = (size_t)c->q_heads * d;
    double* out = (double*)malloc(sizeof(double) * n_out);
    double* lse = (double*)malloc(sizeof(double) * (size_t)c->q_heads);
    qsa_oracle_attention_f64(c, q, kt, vt, ntok, out, lse);
    memset(dq, 0, sizeof(double) * n_out);
    memset(dk, 0, sizeof(double) * (size_t)(ntok > 0 ? ntok : 0) * hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)(ntok > 0 ? ntok : 0) * hkv * d);
    for (int h = 0; h < c->q_heads; ++h) {
        const int kvh = h / g;
        const double* qh = q + (size_t)h * d;
        const double* gh = dout + (size_t)h * d;
        double delta = 0.0; /* <dout_h, out_h> */
        for (int j = 0; j < d; ++j) delta += gh[j] * out[(size_t)h * d + j];
        for (int64_t t = 0; t < ntok; ++t) {
            const double* kr = kt + ((size_t)t * hkv + kvh) * d;
            const double* vr = vt + ((size_t)t * hkv + kvh) * d;
            double qk = 0.0, gv = 0.0;
            for (int j = 0; j < d; ++j) {
                qk += qh[j] * kr[j];
                gv += gh[j] * vr[j];
            }
            const double p = exp(qk * scale - lse[h]);
            const double dz = p * (gv - delta);
            double* dkr = dk + ((size_t)t * hkv + kvh) * d;
            double* dvr = dv + ((size_t)t * hkv + kvh) * d;
            for (int j = 0; j < d; ++j) {
                dvr[j] += p * gh[j];
                dq[(size_t)h * d + j] += scale * dz * kr[j];
                dkr[j] += scale * dz * qh[j];
            }
        }
    }
    free(out);
    free(lse);
}

/* The same gradient on the layer's bf16 operands: q, dout [q_heads][d]; kc, vc
 * [>= max token + 1][kv_heads][d]; tokens as for qsa_oracle_attention. */
void qsa_oracle_attention_backward(const qsa_oracle_cfg* c, const uint16_t* q, const uint16_t* kc,
                                   const uint16_t* vc, const int64_t* tokens, int64_t ntok, const uint16_t* dout,
                                   double* dq, double* dk, double* dv) {
    const int d = c->head_dim, hkv = c->kv_heads;
    const size_t row = (size_t)hkv * d, nq = (size_t)c->q_heads * d;
    double* qd = (double*)malloc(sizeof(double) * nq);
    double* gd = (double*)malloc(sizeof(double) * nq);
    double* kt = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1) * row);
    double* vt = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1) * row);
    for (size_t j = 0; j < nq; ++j) {
        qd[j] = bf(q[j]);
        gd[j] = bf(dout[j]);
    }
    for (int64_t t = 0; t < ntok; ++t)
        for (size_t j = 0; j < row; ++j) {
            kt[(size_t)t * row + j] = bf(kc[(size_t)tokens[t] * row + j]);
            vt[(size_t)t * row + j] = bf(vc[(size_t)tokens[t] * row + j]);
        }
    qsa_oracle_attention_backward_f64(c, qd, kt, vt, ntok, gd, dq, dk, dv);
    free(qd);
    free(gd);
    free(kt);
    free(vt);
}

/* Stage-1 target of query i: q [q_heads][d] (position-encoded, as the core
 * attention takes it), kc [>= i + 1][kv_heads][d]. Writes t[b] for the
 * floor(i/r) blocks the indexer scores (nothing when there are none). */
void qsa_oracle_distill_target(const qsa_oracle_cfg* c, int64_t i, const uint16_t* q, const uint16_t* kc,
                               double* t) {
    const int64_t n_vis = i / c->r;
    if (n_vis <= 0) return;
    const int d = c->head_dim, hkv = c->kv_heads, g = c->q_heads / c->kv_heads;
    const double scale = c->sm_scale > 0.0 ? c->sm_scale : 1.0 / sqrt((double)d);
    double* avg = (double*)calloc((size_t)(i + 1), sizeof(double));
    double* z = (double*)malloc(sizeof(double) * (size_t)(i + 1));
    for (int h = 0; h < c->q_heads; ++h) {
        /* dense causal softmax of head h over tokens 0..i */
        double mx = -INFINITY;
        for (int64_t j = 0; j <= i; ++j) {
            const uint16_t* kr = kc + ((size_t)j * hkv + h / g) * d;
            double dot = 0.0;
            for (int e = 0; e < d; ++e) dot += bf(q[(size_t)h * d + e]) * bf(kr[e]);
            z[j] = dot * scale;
            if (z[j] > mx) mx = z[j];
        }
        double den = 0.0;
        for (int64_t j = 0; j <= i; ++j) den += exp(z[j] - mx);
        for (int64_t j = 0; j <= i; ++j) avg[j] += exp(z[j] - mx) / den;
    }
    for (int64_t j = 0; j <= i; ++j) avg[j] /= (double)c->q_heads;
    double mass = 0.0;
    for (int64_t b = 0; b < n_vis; ++b) {
        double best = avg[b * c->r];
        for (int e = 1; e < c->r; ++e)
            if (avg[b * c->r + e] > best) best = avg[b * c->r + e];
        t[b] = best;
        mass += best;
    }
    for (int64_t b = 0; b < n_vis; ++b) t[b] /= mass;
    free(avg);
    free(z);
}

/* KL(t || softmax(s)) over n blocks, with 0 log 0 = 0, and its gradient with
 * respect to the scores: d/ds_b = (sum_b' t_b') softmax(s)_b - t_b. ds may be
 * NULL. Returns 0 for n = 0. */
double qsa_oracle_distill_kl(const double* t, const float* s, int64_t n, double* ds) {
    if (n <= 0) return 0.0;
    double mx = -INFINITY;
    for (int64_t b = 0; b < n; ++b)
        if ((double)s[b] > mx) mx = (double)s[b];
    double den = 0.0, tsum = 0.0;
    for (int64_t b = 0; b < n; ++b) {
        den += exp((double)s[b] - mx);
        tsum += t[b];
    }
    const double log_den = mx + log(den);
    double kl = 0.0;
    for (int64_t b = 0; b < n; ++b) {
        const double log_soft = (double)s[b] - log_den;
        if (t[b] > 0.0) kl += t[b] * (log(t[b]) - log_soft);
        if (ds) ds[b] = tsum * exp(log_soft) - t[b];
    }
    return kl;
}
