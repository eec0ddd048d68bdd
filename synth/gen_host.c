/*
 * Seeded synthetic inputs, host side.
 *
 * This module is shared by the CPU oracle and the CUDA path as the ONLY common
 * piece: it draws input tensors and holds none of the layer's arithmetic.
 *
 * Generator (defined here, mirrored bit for bit by gen_device.cu):
 *   key(seed, tensor)  = splitmix64(seed ^ splitmix64(tensor + 0x632BE59BD9B4E019))
 *   word(e, w)         = splitmix64(key + 3*e + w),   w = 0, 1, 2
 *   s(e)               = sum of the twelve 16-bit fields of word(e,0..2) - 393210
 *   x(e)               = s(e) * 2^-16            (Irwin-Hall(12) - 6, approx N(0,1))
 *   value(e)           = x(e) rounded to bf16, round-to-nearest-even
 * s(e) is an integer of at most 19 bits, so x(e) is exact in fp32 and every
 * value is a multiple of 2^-16 with |value| <= 6.
 * splitmix64 is Vigna's public SplitMix64 finaliser.
 *
 * e is the row-major LOGICAL element index of the tensor (see synth/__init__.py
 * for the logical shapes), so a row can be drawn without drawing the others.
 */
#include <stdint.h>
#include <string.h>

static inline uint64_t sm64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

uint64_t synth_key(uint64_t seed, uint64_t tensor_id) {
    return sm64(seed ^ sm64(tensor_id + 0x632BE59BD9B4E019ull));
}

static inline uint16_t draw(uint64_t key, uint64_t e) {
    int32_t s = 0;
    for (int w = 0; w < 3; ++w) {
        uint64_t r = sm64(key + 3ull * e + (uint64_t)w);
        s += (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF) +
             (int32_t)((r >> 32) & 0xFFFF) + (int32_t)(r >> 48);
    }
    s -= 393210;
    return f32_to_bf16_rne((float)s * (1.0f / 65536.0f));
}

/* out[i] = value(e0 + i), i < count. */
void synth_fill_host(uint64_t seed, uint64_t tensor_id, uint64_t e0, uint64_t count,
                     uint16_t* out) {
    const uint64_t key = synth_key(seed, tensor_id);
#pragma omp parallel for schedule(static) if (count > (1u << 20))
    for (int64_t i = 0; i < (int64_t)count; ++i) out[i] = draw(key, e0 + (uint64_t)i);
}

/* Rows of a tensor whose logical rows are row_len elements long:
 * out[k*row_len + j] = value(rows[k]*row_len + j). */
void synth_fill_rows_host(uint64_t seed, uint64_t tensor_id, const int64_t* rows, int64_t nrows,
                          int64_t row_len, uint16_t* out) {
    const uint64_t key = synth_key(seed, tensor_id);
#pragma omp parallel for schedule(static) if (nrows * row_len > (1 << 20))
    for (int64_t k = 0; k < nrows; ++k)
        for (int64_t j = 0; j < row_len; ++j)
            out[k * row_len + j] = draw(key, (uint64_t)(rows[k] * row_len + j));
}
