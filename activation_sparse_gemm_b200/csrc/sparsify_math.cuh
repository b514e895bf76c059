// Per-group arithmetic of the RT-Lynx sparsify step (RT-Lynx summary page,
// four-step pipeline paragraph, step 1), shared by the prologue kernels.
//
// A group is four consecutive bf16 entries held in two 32-bit words.  The
// 2-of-4 rule keeps the two largest magnitudes, equal magnitudes going to the
// lower index.  Both prologue passes rank the group by the unique key
// (|x| bits << 2) | (3 - index): integer order of the keys is magnitude order
// with the lower index winning ties, so the two largest keys are the kept
// entries.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rtlynx {

struct GroupKeys {
    uint32_t k1, k2;  // largest and second-largest key (the kept entries)
    uint32_t k3, k4;  // the two dropped keys
};

__device__ __forceinline__ GroupKeys rank_group(uint32_t w01, uint32_t w23) {
    const uint32_t a0 = ((w01 & 0x7FFFu) << 2) | 3u;
    const uint32_t a1 = ((w01 >> 14) & (0x7FFFu << 2)) | 2u;
    const uint32_t a2 = ((w23 & 0x7FFFu) << 2) | 1u;
    const uint32_t a3 = (w23 >> 14) & (0x7FFFu << 2);
    const uint32_t h01 = max(a0, a1), l01 = min(a0, a1), h23 = max(a2, a3), l23 = min(a2, a3);
    GroupKeys g;
    g.k1 = max(h01, h23);
    const uint32_t mh = min(h01, h23), ml = max(l01, l23);
    g.k2 = max(mh, ml);
    g.k3 = min(mh, ml);
    g.k4 = min(l01, l23);
    return g;
}

// |x| of a key as a float (exact).
__device__ __forceinline__ float key_mag(uint32_t key) { return __uint_as_float((key >> 2) << 16); }

// A normal bf16 magnitude (exponent field 1..254) as a double, built from its
// bits: same significand, exponent rebiased from 127 to 1023.  Exact.
__device__ __forceinline__ double bf16_mag_to_double(uint32_t mag15) {
    return __hiloint2double(static_cast<int>((mag15 << 13) + ((1023u - 127u) << 20)), 0);
}

// Adds sum(x^2) and the sum of the two largest squares of one group to the
// token's double accumulators.  Products of bf16 values are exact in double
// and each fused multiply-add rounds once, so the sums carry double rounding
// only.  Zero and subnormal entries take the (rare) converting path.
__device__ __forceinline__ void group_energy(uint32_t w01, uint32_t w23, double& all, double& kept) {
    const uint32_t m0 = w01 & 0x7FFFu, m1 = (w01 >> 16) & 0x7FFFu;
    const uint32_t m2 = w23 & 0x7FFFu, m3 = (w23 >> 16) & 0x7FFFu;
    const uint32_t h01 = max(m0, m1), l01 = min(m0, m1), h23 = max(m2, m3), l23 = min(m2, m3);
    const uint32_t mh = min(h01, h23), ml = max(l01, l23);
    const uint32_t t1 = max(h01, h23), t2 = max(mh, ml);  // kept: the two largest
    const uint32_t t3 = min(mh, ml), t4 = min(l01, l23);  // dropped
    double e1, e2, e3, e4;
    if (t4 >= 0x80u) {
        e1 = bf16_mag_to_double(t1);
        e2 = bf16_mag_to_double(t2);
        e3 = bf16_mag_to_double(t3);
        e4 = bf16_mag_to_double(t4);
    } else {  // zero or subnormal entries
        e1 = __uint_as_float(t1 << 16);
        e2 = __uint_as_float(t2 << 16);
        e3 = __uint_as_float(t3 << 16);
        e4 = __uint_as_float(t4 << 16);
    }
    const double k = fma(e2, e2, e1 * e1);
    kept += k;
    all += fma(e4, e4, fma(e3, e3, k));
}

// bf16 nearest-even of the exact product s*x (one rounding, like the
// definition).  The float product is correctly rounded, so only a product
// that lands exactly on a bf16 midpoint needs the sign of the remainder.
__device__ __forceinline__ uint32_t mul_round_bf16(float s, float x) {
    const float p = __fmul_rn(s, x);
    const uint32_t u = __float_as_uint(p);
    if ((u & 0xFFFFu) == 0x8000u) {
        const float e = __fmaf_rn(s, x, -p);  // s*x - p, exact
        if (e != 0.0f) {
            const uint32_t t = u & 0xFFFF0000u;
            const bool away = (e > 0.0f) == (p > 0.0f);
            return (away ? t + 0x10000u : t) >> 16;
        }
    }
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(p)));
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Rounds the exact products s*x0 and s*x1 to bf16 (nearest even, one
// rounding each) and packs them (x0 low).
__device__ __forceinline__ uint32_t mul_round_bf16x2(float s, float x0, float x1) {
    const float p0 = __fmul_rn(s, x0), p1 = __fmul_rn(s, x1);
    __nv_bfloat162 r = __floats2bfloat162_rn(p0, p1);
    uint32_t packed = *reinterpret_cast<uint32_t*>(&r);
    const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
    if ((u0 & 0xFFFFu) == 0x8000u || (u1 & 0xFFFFu) == 0x8000u)  // a float product on a bf16 midpoint (rare)
        packed = mul_round_bf16(s, x0) | (mul_round_bf16(s, x1) << 16);
    return packed;
}

// One group: returns the metadata nibble i0 | (i1 << 2) (i0 < i1, the kept
// indices) and the two kept values, rounded s*x, packed as bf16x2 (i0 low).
__device__ __forceinline__ uint32_t compress_group(uint32_t w01, uint32_t w23, float s, uint32_t& packed) {
    const GroupKeys g = rank_group(w01, w23);
    const uint32_t ia = (~g.k1) & 3u, ib = (~g.k2) & 3u;  // 3 - (key & 3)
    const uint32_t i0 = min(ia, ib), i1 = max(ia, ib);
    // byte selector picking half-words i0 and i1 out of {w01, w23}
    const uint32_t sel = (i0 * 0x22u + 0x10u) | ((i1 * 0x22u + 0x10u) << 8);
    const uint32_t xx = __byte_perm(w01, w23, sel);
    packed = mul_round_bf16x2(s, __uint_as_float(xx << 16), __uint_as_float(xx & 0xFFFF0000u));
    return i0 | (i1 << 2);
}

}  // namespace rtlynx
