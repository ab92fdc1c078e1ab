// Division by a run-time invariant divisor with a multiply and a shift.
//
// Granlund & Montgomery, "Division by Invariant Integers using Multiplication"
// (PLDI 1994), unsigned case: with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, the quotient of any 32-bit n < 2^31 is
// (mulhi(n, m) + n) >> l.  Used to turn a packed tile row into (position, head):
// the pages call for precomputing the q-head -> kv-head mapping with a fast divmod
// ("优化GQA在Flash-Attention中的批量敏感性", section "Flash-Attention的PackGQA优化",
// item 3).  This is an own implementation of the published method.
#pragma once

#include <cstdint>

namespace gqa {

struct FastDiv {
    uint32_t d;      // divisor (>= 1)
    uint32_t magic;  // m
    uint32_t shift;  // l
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.shift = l;
    f.magic = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    return f;
}

__host__ __device__ inline uint32_t fastdiv(uint32_t n, const FastDiv& f) {
#if defined(__CUDA_ARCH__)
    uint32_t hi = __umulhi(n, f.magic);
#else
    uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(n) * f.magic) >> 32);
#endif
    return static_cast<uint32_t>((static_cast<uint64_t>(hi) + n) >> f.shift);
}

__host__ __device__ inline void fastdivmod(uint32_t n, const FastDiv& f, uint32_t& q, uint32_t& r) {
    q = fastdiv(n, f);
    r = n - q * f.d;
}

}  // namespace gqa
