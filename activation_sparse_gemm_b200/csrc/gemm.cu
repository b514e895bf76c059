// Persistent CTA-pair tcgen05 GEMM for the RT-Lynx linear layer on sm_100a.
//
//   sparse mode:      Y = S(X) W^T + T L_A^T      (RT-Lynx summary page, four-step
//                     pipeline paragraph: step 2 gives Y = Y_s + Y_r; step 4 asks
//                     for Y_s and Y_r to be summed on chip)
//   dense-skip mode:  Y = X W^T                   (step 3, Selective Layer Skipping)
//
// A cluster of two CTAs on neighbouring SMs computes one 256 x BN output tile
// with cta_group::2 MMAs: each CTA holds 128 rows of A and BN/2 rows of W in
// its own shared memory and 128 rows x BN columns of the f32 accumulator in
// its own tensor memory, so each SM streams only half of the W tile.
//
// Warp roles in each CTA:
//   warp 0      TMA producer.  Both CTAs load their halves; the completion of
//               both is counted on the leader CTA's "full" barrier.  Sparse
//               stages carry the compressed S(X) tile, the W tile and, every
//               second stage, one 2 KB metadata chunk; then come the LoRA
//               stages (T tile and L_A tile).
//   warp 1      tensor-memory owner; in the leader CTA one thread issues every
//               MMA of the pair: tcgen05.mma.sp (K = 32 logical per instruction)
//               with the metadata moved into tensor memory by tcgen05.cp, and
//               dense tcgen05.mma for the LoRA stages into the SAME accumulator,
//               so T L_A^T never leaves the chip.  Its commits arrive on the
//               barriers of both CTAs.
//   warps 2-5   epilogue: tcgen05.ld, round to bf16, swizzled staging in shared
//               memory, TMA store (clips the ragged M and N edges).
// The accumulator is double-buffered in tensor memory, so the epilogue of one
// tile overlaps the main loop of the next.
//
// Shared memory per CTA and stage (1024-byte aligned, 128B swizzle):
//   sparse stage, 128 logical K:
//     A  128 rows x 64 kept values                                  16 KB
//     B  BN/2 rows of W x 128 values, two 64-wide column blocks     BN*128 B
//     E  the metadata chunk of these 128 K, 128 lanes x 16 B         2 KB
//   dense stage, 64 logical K:  A 128 x 64 (16 KB), B BN/2 x 64 (BN*64 B)
// LoRA stages reuse the slots: T 128 x 64 in A, L_A BN/2 x 64 in B, four
// dense K = 16 MMAs per stage.
// The single MMA-issuing thread is latency bound on its own instruction
// chain, so its loop only adds precomputed offsets to precomputed
// descriptors and every stage carries four MMAs per barrier round trip.
//
// BN = 240 keeps two accumulators and the metadata inside 512 columns; the
// epilogue writes it as seven 32-column chunks and one 16-column chunk.
//
// Tensor memory (per CTA, 512 columns): accumulators at [0, BN) and
// [BN, 2 BN); metadata of the current 128-wide K chunk at [2 BN, 2 BN + 4).
#include "internal.h"
#include "ptx.cuh"

namespace rtlynx {

constexpr int kPairThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiBufBytes = 32 * 64;  // one warp's 32 rows x 32 bf16 columns

template <bool SPARSE, int BN>
struct PairShape {
    static constexpr int BN_HALF = BN / 2;
    static constexpr int BK = SPARSE ? 128 : 64;                 // logical K per stage
    static constexpr int A_BYTES = kBM * 64 * 2;                  // 128 rows x 128 B
    static constexpr int B_ATOM_BYTES = BN_HALF * 64 * 2;        // BN/2 rows x 128 B
    static constexpr int B_BYTES = (BK / 64) * B_ATOM_BYTES;
    static constexpr int E_BYTES = SPARSE ? kChunkBytes : 0;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + E_BYTES + 1023) / 1024) * 1024;
    static constexpr int STAGES = SPARSE ? 4 : 6;
    static constexpr int LORA_A_BYTES = kBM * 64 * 2;
    static constexpr int LORA_B_BYTES = BN_HALF * 64 * 2;
    static constexpr int EPI_BYTES = 4 * 2 * kEpiBufBytes;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
    static_assert(BN % 16 == 0 && BN >= 64 && 2 * BN + 4 <= 512, "two accumulators and the metadata must fit");
    static_assert(B_ATOM_BYTES % 1024 == 0, "operand tiles must stay 1024-byte aligned");
    static_assert(LORA_A_BYTES <= A_BYTES && LORA_B_BYTES <= B_BYTES, "LoRA tiles must fit the operand slots");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct PairArgs {
    int M, N;
    int m_pairs, n_tiles;
    int k_stages;      // main-loop stages per tile (128-wide K chunks when sparse, 64-wide when dense)
    int lora_stages;   // 64-wide LoRA stages per tile
    int k_chunks;      // metadata chunks per 128-row block
    int* err;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* err) {
    uint32_t ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err) ? 1u : 0u;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <bool SPARSE, int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    rtlynx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmLA,
                            const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                            const __grid_constant__ CUtensorMap tmY16, const PairArgs args) {
    using G = PairShape<SPARSE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi = smem + G::STAGES * G::STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + G::EPI_BYTES);
    uint64_t* empty = full + G::STAGES;
    uint64_t* acc_full = empty + G::STAGES;   // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2], used in the leader only
    uint64_t* done_bar = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done_bar + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    int* err = args.err;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmY);
        if (BN % 32) prefetch_tmap(&tmY16);
        if (SPARSE) prefetch_tmap(&tmE);
        if (args.lora_stages > 0) {
            prefetch_tmap(&tmT);
            prefetch_tmap(&tmLA);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t tmem_meta = tmem_base + 2 * BN;

    const int num_tiles = args.m_pairs * args.n_tiles;
    const int total_k = args.k_stages + args.lora_stages;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                const int mp = tile % args.m_pairs;
                const int nt = tile / args.m_pairs;
                const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;
                const int col0 = nt * BN + static_cast<int>(rank) * G::BN_HALF;
                const int chunk0 = (row0 / kBM) * args.k_chunks;
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + stage * G::STAGE_BYTES;
                    uint8_t* sB = sA + G::A_BYTES;
                    const uint32_t fbar = full0 + static_cast<uint32_t>(stage) * 8u;
                    if (kt < args.k_stages) {
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (G::A_BYTES + G::B_BYTES + G::E_BYTES));
                        tma_load_2d_pair(sA, &tmA, fbar, kt * 64, row0);
                        tma_load_2d_pair(sB, &tmB, fbar, kt * G::BK, col0);
                        if constexpr (SPARSE) {
                            tma_load_2d_pair(sB + G::B_ATOM_BYTES, &tmB, fbar, kt * G::BK + 64, col0);
                            tma_load_2d_pair(sB + G::B_BYTES, &tmE, fbar, 0, (chunk0 + kt) * 4);
                        }
                    } else {
                        const int j = kt - args.k_stages;
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (G::LORA_A_BYTES + G::LORA_B_BYTES));
                        tma_load_2d_pair(sA, &tmT, fbar, j * 64, row0);
                        tma_load_2d_pair(sB, &tmLA, fbar, j * 64, col0);
                    }
                    if (++stage == G::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Wait until the leader's MMAs have released every stage this CTA
            // filled, so no commit arrival is still on its way to this CTA.
            for (int i = 0; i < G::STAGES && ok; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, err)) break;
                if (++stage == G::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            const uint32_t idesc_main = make_idesc_bf16(2 * kBM, BN, SPARSE);
            const uint32_t idesc_dense = make_idesc_bf16(2 * kBM, BN, false);
            // Descriptors of stage 0; stage s adds s * STAGE_BYTES / 16 to the
            // start-address field, operand offsets inside a stage likewise.
            const uint32_t smem0 = smem_u32(smem);
            const uint64_t descA0 = make_sdesc(smem0, 16, 1024, kSw128);
            const uint64_t descB0 = make_sdesc(smem0 + G::A_BYTES, 16, 1024, kSw128);
            const uint64_t descE0 = make_sdesc(smem0 + G::A_BYTES + G::B_BYTES, 128, 128, kSwNone);
            constexpr uint64_t kStageStep = G::STAGE_BYTES >> 4;
            constexpr uint64_t kAtomStep = G::B_ATOM_BYTES >> 4;
            // metadata column of sparse MMA j: (tmem_meta + j) with bit 0 moved to the selector
            const uint32_t e01 = tmem_meta & ~1u, e23 = (tmem_meta + 2u) & ~1u;
            const uint32_t id0 = idesc_main | (tmem_meta & 1u), id1 = idesc_main | ((tmem_meta + 1u) & 1u);
            int stage = 0;
            uint32_t phase = 0;
            uint64_t off = 0;  // stage offset in 16-byte units
            int local = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++local) {
                const int buf = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&full[stage], phase, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a = descA0 + off;
                    const uint64_t b = descB0 + off;
                    if (kt < args.k_stages) {
                        const uint32_t acc = kt != 0;
                        if constexpr (SPARSE) {
                            tmem_cp_128x128b_pair(tmem_meta, descE0 + off);
                            mma_sp_f16_pair(d, a, b, e01, id0, acc);
                            mma_sp_f16_pair(d, a + 2, b + 4, e01, id1, 1u);
                            mma_sp_f16_pair(d, a + 4, b + kAtomStep, e23, id0, 1u);
                            mma_sp_f16_pair(d, a + 6, b + kAtomStep + 4, e23, id1, 1u);
                        } else {
                            mma_f16_pair(d, a, b, idesc_main, acc);
                            mma_f16_pair(d, a + 2, b + 2, idesc_main, 1u);
                            mma_f16_pair(d, a + 4, b + 4, idesc_main, 1u);
                            mma_f16_pair(d, a + 6, b + 6, idesc_main, 1u);
                        }
                    } else {
                        mma_f16_pair(d, a, b, idesc_dense, 1u);
                        mma_f16_pair(d, a + 2, b + 2, idesc_dense, 1u);
                        mma_f16_pair(d, a + 4, b + 4, idesc_dense, 1u);
                        mma_f16_pair(d, a + 6, b + 6, idesc_dense, 1u);
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);
                    off += kStageStep;
                    if (++stage == G::STAGES) {
                        stage = 0;
                        off = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair_mc(&acc_full[buf], 0x3);
            }
            // Every MMA of the pair has finished before tensor memory is freed.
            tc_commit_pair_mc(done_bar, 0x1);
            mbar_wait(done_bar, 0, nullptr);
        }
    } else {
        const int quad = warp & 3;  // warps 2..5 own tensor-memory lane quadrants 2,3,0,1
        const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
        uint8_t* stage_buf = epi + (warp - 2) * 2 * kEpiBufBytes;
        int sbuf = 0;
        int local = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
            const int buf = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            if (!warp_wait(&acc_full[buf], use & 1u, err)) break;
            tc_fence_after();
            const int mp = tile % args.m_pairs;
            const int nt = tile / args.m_pairs;
            const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM + quad * 32;
            const int col0 = nt * BN;
            const uint32_t acc = tmem_base + static_cast<uint32_t>(buf * BN) + lane_addr;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                const bool half = (BN - c) < 32;  // 16-column tail chunk
                uint32_t r[32];
                if (half) {
                    uint32_t h[16];
                    tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c), h);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) r[q] = h[q];
                } else {
                    tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(c), r);
                    tmem_ld_wait();
                }
                uint8_t* sb = stage_buf + sbuf * kEpiBufBytes;
                if (lane == 0) bulk_wait_group_read<1>();  // the store that last used sb has read it
                __syncwarp();
                if (!half) {
                    // 32 rows x 64 B, 64B swizzle: 16-byte unit q of row i at q ^ ((i / 2) % 4)
                    uint8_t* row = sb + lane * 64;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
                        pk.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
                        pk.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
                        pk.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
                        *reinterpret_cast<uint4*>(row + ((q ^ ((lane >> 1) & 3)) << 4)) = pk;
                    }
                } else {
                    // 32 rows x 32 B, 32B swizzle: 16-byte unit q of row i at q ^ ((i / 4) % 2)
                    uint8_t* row = sb + lane * 32;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
                        pk.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
                        pk.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
                        pk.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
                        *reinterpret_cast<uint4*>(row + ((q ^ ((lane >> 2) & 1)) << 4)) = pk;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(half ? &tmY16 : &tmY, sb, col0 + c, row0);
                    bulk_commit_group();
                }
                sbuf ^= 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[buf]), 0));
        }
        if (lane == 0) bulk_wait_all();
    }

    __syncwarp();  // reconverge the role warps before the cluster barrier
    // After an abort, give copies still in flight time to land before the
    // shared memory they target is released.
    if (error_seen(err)) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <bool SPARSE, int BN>
static int launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmT,
                       const CUtensorMap& tmLA, const CUtensorMap& tmE, const CUtensorMap& tmY,
                       const CUtensorMap& tmY16, const PairArgs& args, int num_sms, cudaStream_t stream) {
    using G = PairShape<SPARSE, BN>;
    auto kernel = rtlynx_gemm_pair_kernel<SPARSE, BN>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int tiles = args.m_pairs * args.n_tiles;
    const int max_pairs = num_sms / 2;
    const int pairs = tiles < max_pairs ? tiles : max_pairs;
    kernel<<<2 * pairs, kPairThreads, G::SMEM_BYTES, stream>>>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args);
    return cudaGetLastError();
}

constexpr int kPairBN = 240;

int launch_gemm(const Dims& d, bool sparse, const void* A, const void* W, const void* L_A, const Workspace& ws,
                void* Y, int num_sms, int* err, cudaStream_t stream) {
    constexpr int BN = kPairBN;
    CUtensorMap tmA, tmB, tmT, tmLA, tmE, tmY, tmY16;
    int rc;
    if (sparse) {
        rc = encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.vals, d.Kc_pad, d.M_pad, d.Kc_pad * 2,
                            64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        // metadata chunks viewed as rows of 256 16-bit words, four rows per chunk
        rc = encode_tmap_2d(&tmE, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, ws.meta, 256, d.m_blocks * d.k_chunks * 4, 512,
                            256, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc) return rc;
    } else {
        rc = encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, d.K, d.M, d.K * 2, kBK, kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        tmE = tmA;
    }
    rc = encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, d.K, d.N, d.K * 2, kBK, BN / 2,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    rc = encode_tmap_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, d.N, d.M, d.N * 2, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
    rc = encode_tmap_2d(&tmY16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, d.N, d.M, d.N * 2, 16, 32,
                        CU_TENSOR_MAP_SWIZZLE_32B);
    if (rc) return rc;
    const bool lora = sparse && d.R > 0 && L_A != nullptr;
    if (lora) {
        rc = encode_tmap_2d(&tmT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.T, d.R_pad, d.M_pad, d.R_pad * 2, 64, kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        rc = encode_tmap_2d(&tmLA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L_A, d.R, d.N, d.R * 2, 64, BN / 2,
                            CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    } else {
        tmT = tmA;
        tmLA = tmB;
    }
    PairArgs args;
    args.M = static_cast<int>(d.M);
    args.N = static_cast<int>(d.N);
    args.m_pairs = static_cast<int>((d.M + 2 * kBM - 1) / (2 * kBM));
    args.n_tiles = static_cast<int>((d.N + BN - 1) / BN);
    args.k_stages = static_cast<int>(sparse ? d.k_chunks : d.k_tiles);
    args.lora_stages = lora ? static_cast<int>(d.R_pad / 64) : 0;
    args.k_chunks = static_cast<int>(d.k_chunks);
    args.err = err;
    return sparse ? launch_pair<true, BN>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream)
                  : launch_pair<false, BN>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream);
}

}  // namespace rtlynx
