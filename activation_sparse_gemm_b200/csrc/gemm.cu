// Persistent tcgen05 GEMM for the RT-Lynx linear layer on sm_100a.
//
//   sparse mode:      Y = S(X) W^T + T L_A^T      (RT-Lynx summary page, four-step
//                     pipeline paragraph: step 2 gives Y = Y_s + Y_r; step 4 asks
//                     for Y_s and Y_r to be summed on chip)
//   dense-skip mode:  Y = X W^T                   (step 3, Selective Layer Skipping)
//
// One CTA per SM walks output tiles of 128 x 256.  Warp roles:
//   warp 0      TMA producer: A tile (compressed S(X) or dense X), W tile and, in
//               sparse mode, one 2 KB metadata chunk every second stage; then
//               the LoRA stages (T tile and L_A tile).
//   warp 1      TMEM owner and single-thread MMA issuer.  Sparse stages issue
//               tcgen05.mma.sp (K = 32 logical per instruction) with the
//               metadata copied into tensor memory by tcgen05.cp; the LoRA
//               stages issue dense tcgen05.mma into the SAME accumulator, so
//               T L_A^T never exists outside tensor memory.
//   warps 2-5   epilogue: tcgen05.ld, round to bf16, 16-byte stores.
//
// Shared memory per stage (1024-byte aligned):
//   A  sparse: 128 rows x 32 kept values (64 B rows, 64B swizzle)  8 KB
//      dense:  128 rows x 64 values      (128 B rows, 128B swizzle) 16 KB
//   B  256 rows of W x 64 values (128B swizzle)                    32 KB
//   E  metadata chunk, 128 lanes x 16 B, no swizzle                  2 KB (sparse)
// LoRA stages reuse the slots: T 128 x 32 (64B swizzle) in A, L_A 256 x 32
// (64B swizzle) in B.
//
// Tensor memory: columns [0, 256) hold the f32 accumulator (lane = tile row),
// columns [256, 260) the metadata of the current 128-wide K chunk.
#include "internal.h"
#include "ptx.cuh"

namespace rtlynx {

template <bool SPARSE>
struct GemmShape {
    static constexpr int A_BYTES = SPARSE ? kBM * (kBK / 2) * 2 : kBM * kBK * 2;
    static constexpr int B_BYTES = kBN * kBK * 2;
    static constexpr int E_BYTES = SPARSE ? kChunkBytes : 0;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + E_BYTES + 1023) / 1024) * 1024;
    static constexpr int STAGES = 4;
    static constexpr int LORA_A_BYTES = kBM * 32 * 2;
    static constexpr int LORA_B_BYTES = kBN * 32 * 2;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    static_assert(LORA_A_BYTES <= A_BYTES || !SPARSE, "T tile must fit the A slot");
    static_assert(LORA_B_BYTES <= B_BYTES, "L_A tile must fit the B slot");
};

struct GemmArgs {
    int M, N;
    int m_blocks, n_blocks, k_tiles, lora_tiles, k_chunks;
    const uint8_t* meta;
    __nv_bfloat16* Y;
    int64_t ldy;
    int* err;
};

constexpr int kGemmThreads = 192;
constexpr uint32_t kTmemCols = 512;

template <bool SPARSE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    rtlynx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmLA,
                       const GemmArgs args) {
    using G = GemmShape<SPARSE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES);
    uint64_t* empty = full + G::STAGES;
    uint64_t* acc_full = empty + G::STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* done_bar = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done_bar + 1);
    int* consumed_holder = reinterpret_cast<int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int* err = args.err;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(done_bar, 1);
        *consumed_holder = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (args.lora_tiles > 0) {
            prefetch_tmap(&tmT);
            prefetch_tmap(&tmLA);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t tmem_acc = tmem_base;
    const uint32_t tmem_meta = tmem_base + 256;

    const int num_tiles = args.m_blocks * args.n_blocks;
    const int total_k = args.k_tiles + args.lora_tiles;
    int issued = 0;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile % args.m_blocks;
                const int nb = tile / args.m_blocks;
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + stage * G::STAGE_BYTES;
                    uint8_t* sB = sA + G::A_BYTES;
                    uint8_t* sE = sB + G::B_BYTES;
                    if (kt < args.k_tiles) {
                        const bool with_meta = SPARSE && ((kt & 1) == 0);
                        mbar_arrive_expect_tx(&full[stage], G::A_BYTES + G::B_BYTES + (with_meta ? G::E_BYTES : 0));
                        tma_load_2d(sA, &tmA, &full[stage], kt * (SPARSE ? kBK / 2 : kBK), mb * kBM);
                        tma_load_2d(sB, &tmB, &full[stage], kt * kBK, nb * kBN);
                        if (with_meta) {
                            const uint8_t* src =
                                args.meta + (static_cast<size_t>(mb) * args.k_chunks + (kt >> 1)) * kChunkBytes;
                            bulk_load(sE, src, kChunkBytes, &full[stage]);
                        }
                    } else {
                        const int j = kt - args.k_tiles;
                        mbar_arrive_expect_tx(&full[stage], G::LORA_A_BYTES + G::LORA_B_BYTES);
                        tma_load_2d(sA, &tmT, &full[stage], j * 32, mb * kBM);
                        tma_load_2d(sB, &tmLA, &full[stage], j * 32, nb * kBN);
                    }
                    ++issued;
                    if (++stage == G::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc_main = make_idesc_bf16(kBM, kBN, SPARSE);
            const uint32_t idesc_dense = make_idesc_bf16(kBM, kBN, false);
            int stage = 0;
            uint32_t phase = 0;
            int consumed = 0;
            int local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                if (!mbar_wait(acc_empty, (local & 1) ^ 1u, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&full[stage], phase, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sA = smem_u32(smem + stage * G::STAGE_BYTES);
                    const uint32_t sB = sA + G::A_BYTES;
                    const uint32_t sE = sB + G::B_BYTES;
                    if (kt < args.k_tiles) {
                        if constexpr (SPARSE) {
                            if ((kt & 1) == 0) tmem_cp_128x128b(tmem_meta, make_sdesc(sE, 128, 128, kSwNone));
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const uint64_t a = make_sdesc(sA + j * 32, 16, 512, kSw64);
                                const uint64_t b = make_sdesc(sB + j * 64, 16, 1024, kSw128);
                                const uint32_t e = tmem_meta + static_cast<uint32_t>((kt & 1) * 2 + j);
                                mma_sp_f16(tmem_acc, a, b, e & ~1u, idesc_main | (e & 1u), (kt | j) != 0);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint64_t a = make_sdesc(sA + j * 32, 16, 1024, kSw128);
                                const uint64_t b = make_sdesc(sB + j * 32, 16, 1024, kSw128);
                                mma_f16(tmem_acc, a, b, idesc_main, (kt | j) != 0);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const uint64_t a = make_sdesc(sA + j * 32, 16, 512, kSw64);
                            const uint64_t b = make_sdesc(sB + j * 32, 16, 512, kSw64);
                            mma_f16(tmem_acc, a, b, idesc_dense, 1u);
                        }
                    }
                    tc_commit(&empty[stage]);
                    ++consumed;
                    if (++stage == G::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(acc_full);
            }
            // Every MMA this thread issued has finished before tensor memory is freed.
            tc_commit(done_bar);
            mbar_wait(done_bar, 0, nullptr);
            *consumed_holder = consumed;
        }
    } else {
        const int quad = warp & 3;                 // warps 2..5 own TMEM lane quadrants 2,3,0,1
        const int row_in_tile = quad * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            if (!mbar_wait(acc_full, local & 1, err)) break;
            tc_fence_after();
            const int mb = tile % args.m_blocks;
            const int nb = tile / args.m_blocks;
            const int64_t m = static_cast<int64_t>(mb) * kBM + row_in_tile;
            const int n0 = nb * kBN;
#pragma unroll 1
            for (int c = 0; c < kBN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_acc + lane_addr + static_cast<uint32_t>(c), r);
                tmem_ld_wait();
                if (m < args.M) {
                    __nv_bfloat16* yrow = args.Y + m * args.ldy + n0 + c;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (n0 + c + v * 8 < args.N) {
                            uint4 pk;
                            pk.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                            pk.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                            pk.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                            pk.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                            *reinterpret_cast<uint4*>(yrow + v * 8) = pk;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
        }
    }

    __syncthreads();
    if (warp == 0 && lane == 0) {
        // After an abort, wait for copies still in flight into this CTA's shared memory.
        for (int q = *consumed_holder; q < issued; ++q)
            mbar_wait(&full[q % G::STAGES], (q / G::STAGES) & 1, nullptr);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <bool SPARSE>
static int launch_gemm_impl(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmT,
                            const CUtensorMap& tmLA, const GemmArgs& args, int num_sms, cudaStream_t stream) {
    using G = GemmShape<SPARSE>;
    auto kernel = rtlynx_gemm_kernel<SPARSE>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int tiles = args.m_blocks * args.n_blocks;
    const int grid = tiles < num_sms ? tiles : num_sms;
    kernel<<<grid, kGemmThreads, G::SMEM_BYTES, stream>>>(tmA, tmB, tmT, tmLA, args);
    return cudaGetLastError();
}

int launch_gemm(const Dims& d, bool sparse, const void* A, const void* W, const void* L_A, const Workspace& ws,
                void* Y, int num_sms, int* err, cudaStream_t stream) {
    CUtensorMap tmA, tmB, tmT, tmLA;
    int rc;
    if (sparse) {
        rc = encode_tmap_bf16_2d(&tmA, ws.vals, d.Kc_pad, d.M_pad, d.Kc_pad * 2, kBK / 2, kBM,
                                 CU_TENSOR_MAP_SWIZZLE_64B);
    } else {
        rc = encode_tmap_bf16_2d(&tmA, A, d.K, d.M, d.K * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (rc) return rc;
    rc = encode_tmap_bf16_2d(&tmB, W, d.K, d.N, d.K * 2, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const bool lora = sparse && d.R > 0 && L_A != nullptr;
    if (lora) {
        rc = encode_tmap_bf16_2d(&tmT, ws.T, d.R_pad, d.M_pad, d.R_pad * 2, 32, kBM, CU_TENSOR_MAP_SWIZZLE_64B);
        if (rc) return rc;
        rc = encode_tmap_bf16_2d(&tmLA, L_A, d.R, d.N, d.R * 2, 32, kBN, CU_TENSOR_MAP_SWIZZLE_64B);
        if (rc) return rc;
    } else {
        tmT = tmA;
        tmLA = tmB;
    }
    GemmArgs args;
    args.M = static_cast<int>(d.M);
    args.N = static_cast<int>(d.N);
    args.m_blocks = static_cast<int>(sparse ? d.m_blocks : (d.M + kBM - 1) / kBM);
    args.n_blocks = static_cast<int>((d.N + kBN - 1) / kBN);
    args.k_tiles = static_cast<int>(d.k_tiles);
    args.lora_tiles = lora ? static_cast<int>(d.R_pad / 32) : 0;
    args.k_chunks = static_cast<int>(d.k_chunks);
    args.meta = ws.meta;
    args.Y = static_cast<__nv_bfloat16*>(Y);
    args.ldy = d.N;
    args.err = err;
    return sparse ? launch_gemm_impl<true>(tmA, tmB, tmT, tmLA, args, num_sms, stream)
                  : launch_gemm_impl<false>(tmA, tmB, tmT, tmLA, args, num_sms, stream);
}

}  // namespace rtlynx
