/*
 * Device implementation of the seeded input generator defined in gen.h, for inputs
 * too large to generate on the host and copy (e.g. tens of GB of K/V for long-context
 * decode).  Same definition, element for element; it holds no attention arithmetic.
 */
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xbf58476d1ce4e5b9ull;
    z ^= z >> 27;
    z *= 0x94d049bb133111ebull;
    z ^= z >> 31;
    return z;
}

__device__ __forceinline__ uint16_t bf16_rne_from_double(double z) {
    if (z == 0.0) return signbit(z) ? 0x8000u : 0u;
    int e = ilogb(z);
    double scaled = ldexp(z, 7 - e);
    double r = rint(scaled);  // ties to even
    double y = ldexp(r, e - 7);
    float f = __double2float_rn(y);  // exact: y has 8 significant bits
    return (uint16_t)(__float_as_uint(f) >> 16);
}

__global__ void gen_bf16_kernel(uint64_t base, uint64_t start, uint64_t count, uint16_t* out) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < count; t += stride) {
        uint64_t r = mix64(base + (start + t + 1) * kGolden);
        double u1 = (double)((r >> 40) + 1) * (1.0 / 16777216.0);
        double u2 = (double)((r >> 16) & 0xFFFFFFull) * (1.0 / 16777216.0);
        double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
        out[t] = bf16_rne_from_double(z);
    }
}

__device__ __forceinline__ uint8_t e4m3_rne_from_double(double t) {
    const uint8_t sign = signbit(t) ? 0x80u : 0u;
    const double a = fabs(t);
    if (a == 0.0) return sign;
    if (!(a < 448.0)) return (uint8_t)(sign | 0x7Eu);
    int e = ilogb(a);
    if (e < -6) return (uint8_t)(sign | (uint8_t)rint(ldexp(a, 9)));
    double q = rint(ldexp(a, 3 - e));
    if (q == 16.0) {
        q = 8.0;
        ++e;
    }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8)));
}

__global__ void gen_e4m3_kernel(uint64_t base, uint64_t start, uint64_t count, double scale,
                                uint8_t* out) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < count; t += stride) {
        uint64_t r = mix64(base + (start + t + 1) * kGolden);
        double u1 = (double)((r >> 40) + 1) * (1.0 / 16777216.0);
        double u2 = (double)((r >> 16) & 0xFFFFFFull) * (1.0 / 16777216.0);
        double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
        out[t] = e4m3_rne_from_double(z / scale);
    }
}

uint64_t tensor_base(uint64_t seed, uint64_t tensor_id) {
    uint64_t base = seed * kGolden + tensor_id;
    base ^= base >> 30;
    base *= 0xbf58476d1ce4e5b9ull;
    base ^= base >> 27;
    base *= 0x94d049bb133111ebull;
    base ^= base >> 31;
    return base;
}

unsigned grid_for(uint64_t count) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (count + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    return (unsigned)(blocks > cap ? cap : blocks);
}

}  // namespace

extern "C" int gqa_gen_e4m3_device(uint64_t seed, uint64_t tensor_id, uint64_t start,
                                   uint64_t count, double scale, uint8_t* out,
                                   cudaStream_t stream) {
    if (count == 0) return 0;
    if (out == nullptr) return 1;
    gen_e4m3_kernel<<<grid_for(count), 256, 0, stream>>>(tensor_base(seed, tensor_id), start,
                                                         count, scale, out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int gqa_gen_bf16_device(uint64_t seed, uint64_t tensor_id, uint64_t start,
                                   uint64_t count, uint16_t* out, cudaStream_t stream) {
    if (count == 0) return 0;
    if (out == nullptr) return 1;
    uint64_t base = seed * kGolden + tensor_id;
    // host-side copy of mix64 for the per-tensor base
    base ^= base >> 30;
    base *= 0xbf58476d1ce4e5b9ull;
    base ^= base >> 27;
    base *= 0x94d049bb133111ebull;
    base ^= base >> 31;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (count + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    gen_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(base, start, count, out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
