// Per-group arithmetic of the RT-Lynx sparsify step (RT-Lynx summary page,
// four-step pipeline paragraph, step 1), shared by the prologue kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rtlynx {

__device__ __forceinline__ double mag_to_double(uint32_t mag15) {
    return static_cast<double>(__uint_as_float(mag15 << 16));
}

// Adds sum(x^2) and the sum of the two largest squares of one group (bf16
// bits in two words) to the token's double accumulators.  A bf16 square has
// at most 16 significant bits, so every product here is exact and the sums
// carry double rounding only (the fp32 squares of tiny bf16 values would
// underflow, doubles do not).
__device__ __forceinline__ void group_energy(uint32_t w01, uint32_t w23, double& all, double& kept) {
    const uint32_t a0 = w01 & 0x7FFFu, a1 = (w01 >> 16) & 0x7FFFu;
    const uint32_t a2 = w23 & 0x7FFFu, a3 = (w23 >> 16) & 0x7FFFu;
    const uint32_t h01 = max(a0, a1), l01 = min(a0, a1), h23 = max(a2, a3), l23 = min(a2, a3);
    const uint32_t t1 = max(h01, h23);                        // largest magnitude
    const uint32_t t2 = max(min(h01, h23), max(l01, l23));    // second largest
    const uint32_t u1 = min(max(l01, l23), min(h01, h23));    // third
    const uint32_t u2 = min(l01, l23);                        // smallest
    const double d1 = mag_to_double(t1), d2 = mag_to_double(t2);
    const double d3 = mag_to_double(u1), d4 = mag_to_double(u2);
    const double k = fma(d2, d2, d1 * d1);
    kept += k;
    all += fma(d4, d4, fma(d3, d3, k));
}

// bf16 nearest-even of the exact product s*x (one rounding, like the definition).
__device__ __forceinline__ uint32_t mul_round_bf16(float s, float x) {
    const float p = __fmul_rn(s, x);
    const float e = __fmaf_rn(s, x, -p);  // s*x - p, exact
    const uint32_t u = __float_as_uint(p);
    if ((u & 0xFFFFu) == 0x8000u && e != 0.0f) {
        const uint32_t t = u & 0xFFFF0000u;
        const bool away = (e > 0.0f) == (p > 0.0f);
        return (away ? t + 0x10000u : t) >> 16;
    }
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(p)));
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// One group of four bf16 (bits packed in two words): kept indices by the
// 2-of-4 rule (magnitude, ties to the lower index); returns the nibble
// i0 | (i1 << 2) and the two rounded, scaled kept values packed as bf16x2.
// Entry j beats entry i when |x_j| > |x_i|, or |x_j| == |x_i| and j < i;
// an entry is kept when fewer than two others beat it.  Magnitudes compare
// as integers (bits & 0x7FFF), which orders finite bf16 values exactly.
__device__ __forceinline__ uint32_t compress_group(uint32_t w01, uint32_t w23, float s, uint32_t& packed) {
    const uint32_t m0 = w01 & 0x7FFFu, m1 = (w01 >> 16) & 0x7FFFu;
    const uint32_t m2 = w23 & 0x7FFFu, m3 = (w23 >> 16) & 0x7FFFu;
    const uint32_t c01 = m0 >= m1, c02 = m0 >= m2, c03 = m0 >= m3;  // lower index wins ties
    const uint32_t c12 = m1 >= m2, c13 = m1 >= m3, c23 = m2 >= m3;
    const uint32_t b0 = (c01 ^ 1u) + (c02 ^ 1u) + (c03 ^ 1u);
    const uint32_t b1 = c01 + (c12 ^ 1u) + (c13 ^ 1u);
    const uint32_t b2 = c02 + c12 + (c23 ^ 1u);
    const uint32_t b3 = c03 + c13 + c23;
    const uint32_t kept = (b0 < 2u) | ((b1 < 2u) << 1) | ((b2 < 2u) << 2) | ((b3 < 2u) << 3);
    // kept-mask -> nibble: 0b0011->0x4, 0b0101->0x8, 0b1001->0xC, 0b0110->0x9, 0b1010->0xD, 0b1100->0xE
    constexpr uint64_t kNibble = (0x4ull << 12) | (0x8ull << 20) | (0xCull << 36) | (0x9ull << 24) |
                                 (0xDull << 40) | (0xEull << 48);
    const uint32_t nib = static_cast<uint32_t>(kNibble >> (4u * kept)) & 0xFu;
    const uint32_t i0 = nib & 3u, i1 = nib >> 2;
    const uint32_t x0 = ((i0 & 2u) ? w23 : w01) >> (16u * (i0 & 1u));
    const uint32_t x1 = ((i1 & 2u) ? w23 : w01) >> (16u * (i1 & 1u));
    const uint32_t v0 = mul_round_bf16(s, bf16_bits_to_float(x0 & 0xFFFFu));
    const uint32_t v1 = mul_round_bf16(s, bf16_bits_to_float(x1 & 0xFFFFu));
    packed = v0 | (v1 << 16);
    return nib;
}

}  // namespace rtlynx
