/* Host implementation of the seeded input generator defined in gen.h. */
#include "gen.h"

#include <math.h>

static const uint64_t GOLDEN = 0x9E3779B97F4A7C15ull;

static uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xbf58476d1ce4e5b9ull;
    z ^= z >> 27;
    z *= 0x94d049bb133111ebull;
    z ^= z >> 31;
    return z;
}

/* fp64 -> bf16 bits, round to nearest even, for finite normal-range z. */
static uint16_t bf16_rne_from_double(double z) {
    if (z == 0.0) return signbit(z) ? 0x8000u : 0u;
    int e = ilogb(z);                   /* |z| in [2^e, 2^(e+1)) */
    double scaled = ldexp(z, 7 - e);    /* 8 significant bits left of the point; exact */
    double r = nearbyint(scaled);       /* default rounding mode: ties to even */
    double y = ldexp(r, e - 7);         /* exact, and representable in bf16 */
    float f = (float)y;                 /* exact */
    union { float f; uint32_t u; } c;
    c.f = f;
    return (uint16_t)(c.u >> 16);
}

static double normal_from_counter(uint64_t base, uint64_t i) {
    uint64_t r = mix64(base + (i + 1) * GOLDEN);
    double u1 = (double)((r >> 40) + 1) * (1.0 / 16777216.0);
    double u2 = (double)((r >> 16) & 0xFFFFFFull) * (1.0 / 16777216.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

static uint64_t tensor_base(uint64_t seed, uint64_t tensor_id) {
    return mix64(seed * GOLDEN + tensor_id);
}

uint16_t gqa_gen_bf16_one(uint64_t seed, uint64_t tensor_id, uint64_t i) {
    return bf16_rne_from_double(normal_from_counter(tensor_base(seed, tensor_id), i));
}

void gqa_gen_bf16_range(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count,
                        uint16_t* out) {
    const uint64_t base = tensor_base(seed, tensor_id);
    long long n = (long long)count;
#pragma omp parallel for schedule(static)
    for (long long t = 0; t < n; ++t)
        out[t] = bf16_rne_from_double(normal_from_counter(base, start + (uint64_t)t));
}

void gqa_gen_bf16_strided(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t inner,
                          uint64_t outer, uint64_t outer_stride, uint16_t* out) {
    const uint64_t base = tensor_base(seed, tensor_id);
    long long no = (long long)outer;
#pragma omp parallel for schedule(static)
    for (long long o = 0; o < no; ++o)
        for (uint64_t n = 0; n < inner; ++n)
            out[(uint64_t)o * inner + n] = bf16_rne_from_double(
                normal_from_counter(base, offset + (uint64_t)o * outer_stride + n));
}

uint8_t gqa_e4m3_rne_from_double(double t) {
    const uint8_t sign = signbit(t) ? 0x80u : 0u;
    const double a = fabs(t);
    if (a == 0.0) return sign;
    if (!(a < 448.0)) return (uint8_t)(sign | 0x7Eu); /* 448 and above (and NaN): +-448 */
    int e = ilogb(a);                                   /* a in [2^e, 2^(e+1)) */
    if (e < -6) {                                       /* subnormal: m * 2^-9, m in [0, 8] */
        const double m = nearbyint(ldexp(a, 9));        /* exact scaling; ties to even */
        return (uint8_t)(sign | (uint8_t)m);            /* m = 8 is the smallest normal */
    }
    double q = nearbyint(ldexp(a, 3 - e));              /* 4 significant bits: [8, 16] */
    if (q == 16.0) {
        q = 8.0;
        ++e;
    }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8)));
}

void gqa_gen_e4m3_range(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count,
                        double scale, uint8_t* out) {
    const uint64_t base = tensor_base(seed, tensor_id);
    long long n = (long long)count;
#pragma omp parallel for schedule(static)
    for (long long t = 0; t < n; ++t)
        out[t] = gqa_e4m3_rne_from_double(normal_from_counter(base, start + (uint64_t)t) / scale);
}
