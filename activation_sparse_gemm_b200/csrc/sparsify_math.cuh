// Per-group arithmetic of the RT-Lynx sparsify step (RT-Lynx summary page,
// four-step pipeline paragraph, step 1), used by the prologue kernels.
//
// A group is four consecutive bf16 entries held in two 32-bit words.  The
// 2-of-4 rule keeps the two largest magnitudes, equal magnitudes going to the
// lower index.  The prologue ranks each group by the unique key
// (|x| bits << 16) | (3 - index): integer order of the keys is magnitude order
// with the lower index winning ties, so the two largest keys are the kept
// entries.  The magnitude sits where it sits in the high half of the input
// word, so the keys of odd entries are one mask away from the input.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rtlynx {

struct GroupKeys {
    uint32_t k1, k2;  // largest and second-largest key (the kept entries)
    uint32_t k3, k4;  // the two dropped keys
};

__device__ __forceinline__ GroupKeys rank_group(uint32_t w01, uint32_t w23) {
    const uint32_t a0 = ((w01 << 16) & 0x7FFF0000u) | 3u;
    const uint32_t a1 = (w01 & 0x7FFF0000u) | 2u;
    const uint32_t a2 = ((w23 << 16) & 0x7FFF0000u) | 1u;
    const uint32_t a3 = w23 & 0x7FFF0000u;
    const uint32_t h01 = max(a0, a1), l01 = min(a0, a1), h23 = max(a2, a3), l23 = min(a2, a3);
    GroupKeys g;
    g.k1 = max(h01, h23);
    const uint32_t mh = min(h01, h23), ml = max(l01, l23);
    g.k2 = max(mh, ml);
    g.k3 = min(mh, ml);
    g.k4 = min(l01, l23);
    return g;
}

// A normal bf16 magnitude (exponent field 1..254) as a double, built from its
// bits: same significand, exponent rebiased from 127 to 1023.  Exact.
// From a key (|x| bits << 16 | tag) the high word's significand and exponent
// bits, mag15 << 13, equal key >> 3 (the tag shifts out); a multiply-high
// with an added constant forms them on the multiply-add pipe, leaving the
// integer ALU, which bounds the prologue, to the ranking.
__device__ __forceinline__ double key_mag_to_double(uint32_t key) {
    return __hiloint2double(static_cast<int>(__umulhi(key, 1u << 29) + ((1023u - 127u) << 20)), 0);
}

// The metadata nibble i0 | (i1 << 2) of a ranked group (i0 < i1, the kept
// indices), and its two kept entries, unscaled, packed as bf16x2 (i0 in the
// low half).
__device__ __forceinline__ uint32_t pick_kept(const GroupKeys& g, uint32_t w01, uint32_t w23, uint32_t& kept) {
    const uint32_t ia = (~g.k1) & 3u, ib = (~g.k2) & 3u;  // 3 - (key & 3)
    const uint32_t i0 = min(ia, ib), i1 = max(ia, ib);
    // byte selector picking half-words i0 and i1 out of {w01, w23}
    // multiply-adds (the fields do not overlap, so + is |), off the integer ALU
    const uint32_t sel = i1 * 0x2200u + (i0 * 0x22u + 0x1010u);
    kept = __byte_perm(w01, w23, sel);
    return i1 * 4u + i0;
}

// True when the smallest entry of the group is a normal number (so are the others).
__device__ __forceinline__ bool group_all_normal(const GroupKeys& g) { return g.k4 >= (0x80u << 16); }

// Adds sum(x^2) of a ranked group whose entries are all normal numbers to
// `all` and the sum of its two largest squares to `top`.  Each entry is
// rebuilt as a double from its bits; products of bf16 values are exact in
// double and each fused multiply-add rounds once.
__device__ __forceinline__ void group_energy_normal(const GroupKeys& g, double& all, double& top) {
    const double e1 = key_mag_to_double(g.k1), e2 = key_mag_to_double(g.k2);
    const double e3 = key_mag_to_double(g.k3), e4 = key_mag_to_double(g.k4);
    const double k = fma(e2, e2, e1 * e1);
    top += k;
    all += fma(e4, e4, fma(e3, e3, k));
}

// The same sums for a group that may hold zero or subnormal entries (they go
// through float, which holds every bf16 value exactly).  Kept out of line:
// it runs only for the rare tiles that need it, so the common path never pays
// for its conversions.  Returns (sum of all four squares, sum of the top two).
static __device__ __noinline__ double2 group_energy_any(uint32_t k1, uint32_t k2, uint32_t k3, uint32_t k4) {
    const double e1 = __uint_as_float(k1 & 0x7FFF0000u), e2 = __uint_as_float(k2 & 0x7FFF0000u);
    const double e3 = __uint_as_float(k3 & 0x7FFF0000u), e4 = __uint_as_float(k4 & 0x7FFF0000u);
    const double k = fma(e2, e2, e1 * e1);
    return make_double2(fma(e4, e4, fma(e3, e3, k)), k);
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

// Rescales a packed pair of kept bf16 entries by s: each product s*x rounded
// once to bf16 (nearest even).
__device__ __forceinline__ uint32_t scale_pair(float s, uint32_t packed) {
    return mul_round_bf16x2(s, __uint_as_float(packed << 16), __uint_as_float(packed & 0xFFFF0000u));
}

}  // namespace rtlynx
