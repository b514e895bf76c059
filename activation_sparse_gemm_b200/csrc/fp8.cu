// The FP8 (E4M3) form of the RT-Lynx layer: weight preparation and the debug
// unpack of the prologue's FP8 outputs.  The layer itself runs the shared
// prologue (sparsify.cu, FP8 mode) and the pair GEMM (gemm.cu, FP8 variant).
//
// The pages name FP8 as future work that stacks with the method and give no
// recipe.  The reading: E4M3 without infinities (largest finite 448), round
// to nearest even, saturating; W per output channel with scale max|W_n| / 448;
// S(X) per token with scale max|S(X)| / 448, whose codes are those of
// x~ * 448 / max|x| because s scales the whole token and the largest entry is
// always kept.  The quantisation decisions are float32 operations.
#include <cuda_fp8.h>

#include "internal.h"
#include "sparsify_math.cuh"

namespace rtlynx {

// One CTA per output channel n: B = max_k |W[n,k]|; codes of W * (448 / B)
// (float32 product, nearest even, saturating); qw[n] = B / 448; and the row
// of L_A divided by qw[n] (by 1 for an all-zero channel, whose codes are all
// zero) for the LoRA stages that share the FP8 accumulator, which the
// epilogue multiplies by q_x qw[n].
__global__ void __launch_bounds__(256) rtlynx_quantize_weight_fp8_kernel(const uint16_t* __restrict__ W,
                                                                         const uint16_t* __restrict__ L_A,
                                                                         uint8_t* __restrict__ W8,
                                                                         float* __restrict__ qw,
                                                                         uint16_t* __restrict__ L_A8, int64_t K,
                                                                         int64_t R) {
    __shared__ float red[8];
    const int64_t n = blockIdx.x;
    const uint16_t* w = W + n * K;
    float b = 0.0f;
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) b = fmaxf(b, fabsf(bf16_bits_to_float(w[k])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = b;
    __syncthreads();
    b = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) b = fmaxf(b, red[i]);
    const float r = b > 0.0f ? __fdiv_rn(448.0f, b) : 0.0f;
    uint16_t* out = reinterpret_cast<uint16_t*>(W8 + n * K);  // K is even: two codes per store
    for (int64_t k = 2 * threadIdx.x; k < K; k += 2 * blockDim.x) {
        const float lo = __fmul_rn(bf16_bits_to_float(w[k]), r);
        const float hi = __fmul_rn(bf16_bits_to_float(w[k + 1]), r);
        out[k >> 1] = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    }
    const float q = __fdiv_rn(b, 448.0f);
    if (threadIdx.x == 0) qw[n] = q;
    if (L_A && L_A8) {
        const float qe = q > 0.0f ? q : 1.0f;
        for (int64_t j = threadIdx.x; j < R; j += blockDim.x)
            L_A8[n * R + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(bf16_bits_to_float(L_A[n * R + j]), qe)));
    }
}

int launch_quantize_weight_fp8(const void* W, const void* L_A, void* W8, float* qw, void* L_A8, int64_t N,
                               int64_t K, int64_t R, cudaStream_t stream) {
    if (N <= 0) return 0;
    rtlynx_quantize_weight_fp8_kernel<<<static_cast<unsigned>(N), 256, 0, stream>>>(
        static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(L_A), static_cast<uint8_t*>(W8), qw,
        static_cast<uint16_t*>(L_A8), K, R);
    return static_cast<int>(cudaGetLastError());
}

// Plain layouts of the FP8 prologue's outputs: codes [M, K/2] (kept entries'
// codes in channel order), meta [M, K/4] (one nibble per byte, from the 8-bit
// chunk layout: token m of a block at byte 16 m, group g of a chunk at nibble
// g), qx [M].
__global__ void rtlynx_unpack_fp8_kernel(const Dims d, const uint8_t* __restrict__ codes_ws,
                                         const uint8_t* __restrict__ meta_ws, const float* __restrict__ qx_ws,
                                         uint8_t* codes, uint8_t* meta, float* qx) {
    const int64_t G = d.K / 4;
    const int64_t total = d.M * G;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / G, g = i % G;
        const int64_t mb = row / kBM, m = row % kBM;
        const int64_t kc = g / 32, gg = g % 32;  // 32 groups (128 channels) per chunk
        const uint8_t byte = meta_ws[(mb * d.k_chunks + kc) * kChunkBytes + 16 * m + gg / 2];
        if (meta) meta[i] = static_cast<uint8_t>((byte >> (4 * (gg & 1))) & 0xF);
        if (codes) {
            codes[row * (d.K / 2) + 2 * g] = codes_ws[row * d.Kc_pad + 2 * g];
            codes[row * (d.K / 2) + 2 * g + 1] = codes_ws[row * d.Kc_pad + 2 * g + 1];
        }
        if (g == 0 && qx) qx[row] = qx_ws[row];
    }
}

int launch_unpack_fp8_debug(const Dims& d, const Workspace& ws, void* codes, void* meta, void* qx,
                            cudaStream_t stream) {
    const int64_t total = d.M * (d.K / 4);
    const int blocks = static_cast<int>((total + 255) / 256 < 8192 ? (total + 255) / 256 : 8192);
    rtlynx_unpack_fp8_kernel<<<blocks > 0 ? blocks : 1, 256, 0, stream>>>(
        d, ws.codes, ws.meta, ws.qx, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(meta),
        static_cast<float*>(qx));
    return static_cast<int>(cudaGetLastError());
}

}  // namespace rtlynx
