// The RT-Lynx sparsify prologue on sm_100a (RT-Lynx summary page, four-step
// pipeline paragraph, step 1 "Norm-Compensated Activation Sparsification" and
// step 4 items (1)-(3): mask decision, Top-K, compression to the sparse tensor
// core layout), plus the LoRA down-projection T = X L_B^T of step 2.
//
// Pass 1  norms_lora_down   grid (row block of 128 tokens, K-split).
//         TMA streams 128 x 64 tiles of X (128B swizzle) and 64-wide tiles of
//         L_B.  Four warps read each X tile from shared memory, one token per
//         thread, and accumulate sum(x^2) and sum(x~^2) in double from exact
//         squares (the kept entries are the two largest magnitudes of each
//         group; ties do not change the sum).
//         From the SAME shared-memory tile one thread issues dense tcgen05.mma
//         (M = 128, N = R) for the partial T.  Partial sums go to the workspace.
// Pass 2  compress          grid (16-token slab, 256-wide K block).
//         Sums the partial norms in a fixed order, s = ||x|| / (||x~|| + 1e-8),
//         applies the exact 2-of-4 rule (integer magnitude compares, ties to the
//         lower index), rounds s*x once to bf16, and writes the kept values
//         row-major and the metadata in the order tcgen05.cp copies it into
//         tensor memory.
// Pass 3  finalize_T        sums the partial T in a fixed order and rounds to bf16.
//
// Metadata chunk (128 tokens x 128 logical K, 2048 bytes), for token m in the
// row block (m0 = m % 8, m1 = (m / 8) % 2, m2 = m / 16) and logical k in the
// chunk (k0 = k % 16, k1 = (k / 16) % 2, k2 = k / 32):
//     tensor-memory lane dp = m0 + 8*k1 + 16*m2, column k2,
//     byte offset 16*dp + 4*k2, bit 16*m1 + 4*(k0 / 4) within that 32-bit word,
// and the nibble of a group is i0 | (i1 << 2) with i0 < i1 the kept indices.
#include "internal.h"
#include "ptx.cuh"
#include "sparsify_math.cuh"

namespace rtlynx {

// ---------------------------------------------------------------- pass 1
struct NormArgs {
    int M;
    int64_t M_pad;
    int k_tiles, tiles_per_split, R_pad;
    double* part_norm;
    float* part_T;
    int* err;
};

constexpr int kNormStages = 4;
constexpr int kNormThreads = 192;
constexpr int kXTileBytes = kBM * kBK * 2;  // 16 KB

__host__ __device__ inline int norm_stage_bytes(int R_pad) {
    return ((kXTileBytes + R_pad * kBK * 2 + 1023) / 1024) * 1024;
}

template <bool LORA>
__global__ void __launch_bounds__(kNormThreads, 1)
    rtlynx_norms_lora_down_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmLB,
                                  const NormArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = norm_stage_bytes(LORA ? a.R_pad : 0);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kNormStages * stage_bytes);
    uint64_t* empty = full + kNormStages;
    uint64_t* done_bar = empty + kNormStages;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done_bar + 1);
    int* consumed_holder = reinterpret_cast<int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int* err = a.err;
    const int mb = blockIdx.x;
    const int split = blockIdx.y;
    const int kt0 = split * a.tiles_per_split;
    const int kt1 = min(kt0 + a.tiles_per_split, a.k_tiles);
    const int ntiles = kt1 - kt0;
    uint32_t tmem_cols = 32;
    while (tmem_cols < static_cast<uint32_t>(a.R_pad)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNormStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], LORA ? 5 : 4);
        }
        mbar_init(done_bar, 1);
        *consumed_holder = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        if (LORA) prefetch_tmap(&tmLB);
    }
    if (LORA && warp == 1) {
        tmem_alloc(tmem_holder, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = LORA ? *tmem_holder : 0u;
    int issued = 0;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint32_t bytes = kXTileBytes + (LORA ? a.R_pad * kBK * 2 : 0);
            for (int i = 0; i < ntiles; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, err)) break;
                uint8_t* sX = smem + stage * stage_bytes;
                mbar_arrive_expect_tx(&full[stage], bytes);
                tma_load_2d(sX, &tmX, &full[stage], (kt0 + i) * kBK, mb * kBM);
                if (LORA) tma_load_2d(sX + kXTileBytes, &tmLB, &full[stage], (kt0 + i) * kBK, 0);
                ++issued;
                if (++stage == kNormStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (LORA && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(kBM, a.R_pad, false);
            int stage = 0;
            uint32_t phase = 0;
            int consumed = 0;
            for (int i = 0; i < ntiles; ++i) {
                if (!mbar_wait(&full[stage], phase, err)) break;
                tc_fence_after();
                const uint32_t sX = smem_u32(smem + stage * stage_bytes);
                const uint32_t sL = sX + kXTileBytes;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t ad = make_sdesc(sX + j * 32, 16, 1024, kSw128);
                    const uint64_t bd = make_sdesc(sL + j * 32, 16, 1024, kSw128);
                    mma_f16(tmem_base, ad, bd, idesc, (i | j) != 0);
                }
                tc_commit(&empty[stage]);
                ++consumed;
                if (++stage == kNormStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            tc_commit(done_bar);
            mbar_wait(done_bar, 0, nullptr);
            *consumed_holder = consumed;
        }
    } else {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // token row within the block
        double nx = 0.0, nt = 0.0;
        int stage = 0;
        uint32_t phase = 0;
        int consumed = 0;
        for (int i = 0; i < ntiles; ++i) {
            if (!mbar_wait(&full[stage], phase, err)) break;
            const uint8_t* row = smem + stage * stage_bytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
                group_energy(v.x, v.y, nx, nt);
                group_energy(v.z, v.w, nx, nt);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            ++consumed;
            if (++stage == kNormStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!LORA && warp == 2 && lane == 0) *consumed_holder = consumed;
        const int64_t grow = static_cast<int64_t>(mb) * kBM + r;
        double* pn = a.part_norm + (static_cast<int64_t>(split) * a.M_pad + grow) * 2;
        pn[0] = nx;
        pn[1] = nt;
        if (LORA) {
            if (mbar_wait(done_bar, 0, err)) {
                tc_fence_after();
                float* pt = a.part_T + (static_cast<int64_t>(split) * a.M_pad + grow) * a.R_pad;
                const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
                for (int c = 0; c < a.R_pad; c += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(c), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 f4 = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                        *reinterpret_cast<float4*>(pt + c + 4 * q) = f4;
                    }
                }
                tc_fence_before();
            }
        }
    }

    __syncthreads();
    if (warp == 0 && lane == 0) {
        for (int q = *consumed_holder; q < issued; ++q)
            mbar_wait(&full[q % kNormStages], (q / kNormStages) & 1, nullptr);
    }
    if (LORA && warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

// ---------------------------------------------------------------- pass 2
struct CompressArgs {
    int M, K;
    int64_t M_pad, Kc_pad;
    int k_chunks, nsplit;
    const double* part_norm;
    uint16_t* vals;
    uint8_t* meta;
    float* s_out;
};

__global__ void __launch_bounds__(256) rtlynx_compress_kernel(const uint16_t* __restrict__ X, const CompressArgs a) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = warp, m1 = lane >> 4, p = lane & 15;
    const int64_t slab = blockIdx.x;
    const int64_t mb = slab >> 3;
    const int m2 = static_cast<int>(slab & 7);
    const int64_t row = slab * 16 + m1 * 8 + m0;
    const int64_t k = static_cast<int64_t>(blockIdx.y) * 256 + p * 16;
    const int64_t kc = k >> 7;
    const bool chunk_ok = kc < a.k_chunks;

    float s = 0.f;
    if (row < a.M) {
        double nx = 0.0, nt = 0.0;
        for (int j = 0; j < a.nsplit; ++j) {
            const double* pn = a.part_norm + (static_cast<int64_t>(j) * a.M_pad + row) * 2;
            nx += pn[0];
            nt += pn[1];
        }
        s = static_cast<float>(sqrt(nx) / (sqrt(nt) + 1e-8));
    }
    uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
    if (row < a.M && chunk_ok) {
        const uint16_t* xr = X + row * a.K;
        if (k < a.K) lo = *reinterpret_cast<const uint4*>(xr + k);
        if (k + 8 < a.K) hi = *reinterpret_cast<const uint4*>(xr + k + 8);
    }
    uint4 out;
    uint32_t nib = 0;
    nib |= compress_group(lo.x, lo.y, s, out.x);
    nib |= compress_group(lo.z, lo.w, s, out.y) << 4;
    nib |= compress_group(hi.x, hi.y, s, out.z) << 8;
    nib |= compress_group(hi.z, hi.w, s, out.w) << 12;
    if (chunk_ok && (k >> 1) < a.Kc_pad)
        *reinterpret_cast<uint4*>(a.vals + row * a.Kc_pad + (k >> 1)) = out;
    const uint32_t partner = __shfl_xor_sync(0xFFFFFFFFu, nib, 16);
    if (m1 == 0 && chunk_ok) {
        const int kk = static_cast<int>(k & 127);
        const int k2 = kk >> 5, k1 = (kk >> 4) & 1;
        const int dp = m0 + 8 * k1 + 16 * m2;
        uint32_t* w = reinterpret_cast<uint32_t*>(a.meta + (mb * a.k_chunks + kc) * kChunkBytes + dp * 16 + k2 * 4);
        *w = (nib & 0xFFFFu) | (partner << 16);
    }
    if (blockIdx.y == 0 && p == 0) a.s_out[row] = s;
}

// ---------------------------------------------------------------- pass 3
__global__ void rtlynx_finalize_T_kernel(const float* __restrict__ part_T, uint16_t* __restrict__ T, int64_t n,
                                         int64_t split_stride, int nsplit) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < nsplit; ++j) acc += part_T[j * split_stride + i];
        T[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
    }
}

// ---------------------------------------------------------------- debug unpack
__global__ void rtlynx_unpack_kernel(const Dims d, const uint16_t* __restrict__ vals_ws,
                                     const uint8_t* __restrict__ meta_ws, const float* __restrict__ s_ws,
                                     const uint16_t* __restrict__ T_ws, uint16_t* vals, uint8_t* meta, float* s,
                                     uint16_t* T) {
    const int64_t G = d.K / 4;
    const int64_t total = d.M * G;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / G, g = i % G;
        const int64_t mb = row / kBM;
        const int m = static_cast<int>(row % kBM);
        const int m0 = m & 7, m1 = (m >> 3) & 1, m2 = m >> 4;
        const int64_t k = 4 * g;
        const int64_t kc = k >> 7;
        const int kk = static_cast<int>(k & 127);
        const int k2 = kk >> 5, k1 = (kk >> 4) & 1, nibble = (kk & 15) >> 2;
        const int dp = m0 + 8 * k1 + 16 * m2;
        const uint32_t w =
            *reinterpret_cast<const uint32_t*>(meta_ws + (mb * d.k_chunks + kc) * kChunkBytes + dp * 16 + k2 * 4);
        if (meta) meta[i] = static_cast<uint8_t>((w >> (16 * m1 + 4 * nibble)) & 0xFu);
        if (vals) {
            vals[row * (d.K / 2) + 2 * g] = vals_ws[row * d.Kc_pad + 2 * g];
            vals[row * (d.K / 2) + 2 * g + 1] = vals_ws[row * d.Kc_pad + 2 * g + 1];
        }
        if (g == 0 && s) s[row] = s_ws[row];
        if (g == 0 && T && d.R > 0)
            for (int64_t r = 0; r < d.R; ++r) T[row * d.R + r] = T_ws[row * d.R_pad + r];
    }
}

// ---------------------------------------------------------------- launchers
int launch_norms_lora_down(const Dims& d, const void* X, const void* L_B, const Workspace& ws, int* err,
                           cudaStream_t stream) {
    const bool lora = d.R > 0 && L_B != nullptr;
    CUtensorMap tmX, tmLB;
    int rc = encode_tmap_bf16_2d(&tmX, X, d.K, d.M, d.K * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    if (lora) {
        rc = encode_tmap_bf16_2d(&tmLB, L_B, d.K, d.R, d.K * 2, kBK, static_cast<uint32_t>(d.R_pad),
                                 CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    } else {
        tmLB = tmX;
    }
    NormArgs a;
    a.M = static_cast<int>(d.M);
    a.M_pad = d.M_pad;
    a.k_tiles = static_cast<int>(d.k_tiles);
    a.tiles_per_split = static_cast<int>((d.k_tiles + d.nsplit - 1) / d.nsplit);
    a.R_pad = lora ? static_cast<int>(d.R_pad) : 0;
    a.part_norm = ws.part_norm;
    a.part_T = ws.part_T;
    a.err = err;
    const int smem = kNormStages * norm_stage_bytes(a.R_pad) + 256 + 1024;
    dim3 grid(static_cast<unsigned>(d.m_blocks), static_cast<unsigned>(d.nsplit));
    cudaError_t e;
    if (lora) {
        e = cudaFuncSetAttribute(rtlynx_norms_lora_down_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
        if (e != cudaSuccess) return e;
        rtlynx_norms_lora_down_kernel<true><<<grid, kNormThreads, smem, stream>>>(tmX, tmLB, a);
    } else {
        e = cudaFuncSetAttribute(rtlynx_norms_lora_down_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        rtlynx_norms_lora_down_kernel<false><<<grid, kNormThreads, smem, stream>>>(tmX, tmLB, a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || !lora) return e;
    const int64_t n = d.M_pad * d.R_pad;
    const int blocks = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    rtlynx_finalize_T_kernel<<<blocks, 256, 0, stream>>>(ws.part_T, ws.T, n, d.M_pad * d.R_pad,
                                                          static_cast<int>(d.nsplit));
    return cudaGetLastError();
}

int launch_compress(const Dims& d, const void* X, const Workspace& ws, cudaStream_t stream) {
    CompressArgs a;
    a.M = static_cast<int>(d.M);
    a.K = static_cast<int>(d.K);
    a.M_pad = d.M_pad;
    a.Kc_pad = d.Kc_pad;
    a.k_chunks = static_cast<int>(d.k_chunks);
    a.nsplit = static_cast<int>(d.nsplit);
    a.part_norm = ws.part_norm;
    a.vals = ws.vals;
    a.meta = ws.meta;
    a.s_out = ws.s;
    dim3 grid(static_cast<unsigned>(d.M_pad / 16), static_cast<unsigned>((d.k_chunks * kChunkK + 255) / 256));
    rtlynx_compress_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(X), a);
    return cudaGetLastError();
}

int launch_unpack_debug(const Dims& d, const Workspace& ws, void* vals, void* meta, void* s, void* T,
                        cudaStream_t stream) {
    const int64_t total = d.M * (d.K / 4);
    const int blocks = static_cast<int>((total + 255) / 256 < 8192 ? (total + 255) / 256 : 8192);
    rtlynx_unpack_kernel<<<blocks > 0 ? blocks : 1, 256, 0, stream>>>(
        d, ws.vals, ws.meta, ws.s, ws.T, static_cast<uint16_t*>(vals), static_cast<uint8_t*>(meta),
        static_cast<float*>(s), static_cast<uint16_t*>(T));
    return cudaGetLastError();
}

}  // namespace rtlynx
