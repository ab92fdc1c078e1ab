/*
 * Seeded, counter-based generator of the synthetic attention inputs.
 *
 * This module is shared input infrastructure: the fp64 oracle, the tests and the
 * benchmark all draw Q, K and V from it, so both sides of a parity check see the
 * same numbers.  It holds none of the attention arithmetic.
 *
 * Definition (each element independent of every other, so any slice can be
 * regenerated without materialising the whole tensor):
 *
 *   mix(z)   = the splitmix64 finaliser: z ^= z>>30; z *= 0xbf58476d1ce4e5b9;
 *              z ^= z>>27; z *= 0x94d049bb133111eb; z ^= z>>31
 *   base     = mix(seed * G + tensor_id)                   G = 0x9E3779B97F4A7C15
 *   r        = mix(base + (i + 1) * G)                     i = linear element index
 *   u1       = ((r >> 40) + 1) * 2^-24                     in (0, 1]
 *   u2       = ((r >> 16) & 0xFFFFFF) * 2^-24              in [0, 1)
 *   z        = sqrt(-2 ln u1) * cos(2 pi u2)               Box-Muller, fp64 -> N(0,1)
 *   element  = z rounded to bfloat16, round-to-nearest-even, directly from fp64
 *
 * The rounding step is exact integer/ldexp arithmetic (no double rounding through
 * fp32).  Only log and cos are libm calls; a 1-ulp fp64 difference between two libm
 * implementations changes the bf16 result only when z lies within an ulp of a bf16
 * rounding midpoint (probability ~2^-44 per element).
 *
 * Tensor ids used by the tests and the benchmark: Q = 1, K = 2, V = 3.
 *
 * e4m3 variant (for 8-bit inputs): element = e4m3(z / scale), where e4m3(t) rounds t to
 * the OCP FP8 E4M3 format (4 exponent bits, bias 7, 3 mantissa bits, subnormals m * 2^-9,
 * no infinities, largest finite 448) to nearest even, saturating at +-448; again exact
 * integer/ldexp arithmetic from fp64.  The value it stands for is e4m3_value(bits) * scale.
 */
#ifndef GQA_INPUTS_GEN_H
#define GQA_INPUTS_GEN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 bit pattern of element i of tensor (seed, tensor_id). */
uint16_t gqa_gen_bf16_one(uint64_t seed, uint64_t tensor_id, uint64_t i);

/* out[n] = element (start + n), n < count.  Multithreaded (OpenMP). */
void gqa_gen_bf16_range(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count,
                        uint16_t* out);

/* Strided slice: out[o*inner + n] = element (offset + o*outer_stride + n),
 * n < inner, o < outer.  Used to regenerate one head's K/V rows of a BSHD tensor. */
void gqa_gen_bf16_strided(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t inner,
                          uint64_t outer, uint64_t outer_stride, uint16_t* out);

/* e4m3 bit pattern of t (round to nearest even, saturating at +-448). */
uint8_t gqa_e4m3_rne_from_double(double t);

/* out[n] = e4m3(z_(start + n) / scale), n < count.  Multithreaded (OpenMP). */
void gqa_gen_e4m3_range(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count,
                        double scale, uint8_t* out);

#ifdef __cplusplus
}
#endif

#endif
