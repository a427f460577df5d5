/* Host-side twin of the seeded input generator in synth/__init__.py.
 *
 * Produces the same bits as the torch version: splitmix64 streams (Steele,
 * Lea & Flood 2014), twelve 16-bit uniforms summed for a normal deviate, an
 * independent Bernoulli lane for outliers, round-to-nearest-even to bf16.
 * It holds no part of the optimizer step's arithmetic.
 */
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static uint64_t lane(uint64_t key, int64_t idx) {
    return mix64(key + (uint64_t)(idx + 1) * GAMMA);
}

static float normal_at(uint64_t k0, uint64_t k1, uint64_t k2, int64_t idx, float scale) {
    uint64_t u[3] = {lane(k0, idx), lane(k1, idx), lane(k2, idx)};
    int64_t total = 0;
    for (int l = 0; l < 3; ++l)
        for (int sh = 0; sh < 64; sh += 16) total += (int64_t)((u[l] >> sh) & 0xFFFFu);
    float centred = (float)(total - 393210);
    return centred * scale;
}

/* fp32 -> bf16 bits, round to nearest even; NaN kept quiet with its sign. */
static uint16_t to_bf16(float x) {
    uint32_t b;
    memcpy(&b, &x, 4);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu) != 0u)
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t keep = b >> 16, drop = b & 0xFFFFu;
    if (drop > 0x8000u || (drop == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

void csynth_grad_range(uint64_t k0, uint64_t k1, uint64_t k2, uint64_t k_outlier,
                       int64_t start, int64_t n, int64_t n_valid, float scale,
                       uint32_t outlier_threshold, float outlier_scale, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        int64_t idx = start + i;
        if (idx >= n_valid) { out[i] = 0; continue; }
        float x = normal_at(k0, k1, k2, idx, scale);
        if (outlier_threshold != 0u) {
            uint32_t top = (uint32_t)(lane(k_outlier, idx) >> 32);
            if (top < outlier_threshold) x = x * outlier_scale;
        }
        out[i] = to_bf16(x);
    }
}

void csynth_normal_range(uint64_t k0, uint64_t k1, uint64_t k2, int64_t start, int64_t n,
                         int64_t n_valid, float scale, float* out) {
    for (int64_t i = 0; i < n; ++i) {
        int64_t idx = start + i;
        out[i] = idx >= n_valid ? 0.0f : normal_at(k0, k1, k2, idx, scale);
    }
}
