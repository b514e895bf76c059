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
//               stages carry the compressed S(X) tile, the W tile and the 2 KB
//               metadata chunk of their 128 K; then come the LoRA stages (T
//               tile and L_A tile).
//   warp 1      tensor-memory owner; in the leader CTA the warp runs the issue
//               loop and one elected lane issues every MMA of the pair:
//               tcgen05.mma.sp (K = 32 logical per instruction)
//               with the metadata moved into tensor memory by tcgen05.cp, and
//               dense tcgen05.mma for the LoRA stages into the SAME accumulator,
//               so T L_A^T never leaves the chip.  Its commits arrive on the
//               barriers of both CTAs.
//   warps 2-5   epilogue: tcgen05.ld, optional GELU (a template parameter,
//               used by the feed-forward block's up-projection), round to
//               bf16; sparse mode stages in swizzled shared memory and stores
//               by TMA (clipping the ragged M and N edges), dense-skip stores
//               16-byte pieces straight to Y.
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
// Sparse tiles: BN = 240 keeps two accumulators and the metadata inside 512
// columns; the epilogue writes a tile as seven 32-column chunks and one
// 16-column chunk.  Dense-skip tiles: BN = 256, two accumulators filling the
// 512 columns.
//
// FP8 variant (E4M3 operands, tcgen05.mma.sp kind::f8f6f4, K = 64 logical
// per instruction): BN = 224 (the instruction wants N a multiple of 32); a
// stage carries 256 logical K in the bf16 stage's A and B bytes plus two
// metadata chunks, which tcgen05.cp moves into eight tensor-memory columns,
// two per MMA.  The LoRA stages stay bf16 (T / q_x and L_A / q_w) and add
// into the same accumulator, and the epilogue multiplies it by q_x q_w.
//
// Tensor memory (per CTA, 512 columns): accumulators at [0, BN) and
// [BN, 2 BN); in sparse mode the metadata of the current 128-wide K chunk at
// [2 BN, 2 BN + 4).
//
// Every launch is a programmatic dependent of the preceding kernel: the setup
// (barriers, tensor memory, tensor-map prefetch) overlaps that kernel's tail,
// and operands are read after the grid-dependency wait.
#include "internal.h"
#include "ptx.cuh"

namespace rtlynx {

constexpr int kPairThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiBufBytes = 32 * 64;  // one warp's 32 rows x 32 bf16 columns

// FP8: E4M3 operands; a stage of 256 logical K has the bf16 sparse stage's
// A and B bytes (128-byte rows) and two metadata chunks.
template <bool SPARSE, int BN, bool FP8 = false>
struct PairShape {
    static constexpr int BN_HALF = BN / 2;
    static constexpr int BK = FP8 ? kFp8StageK : (SPARSE ? 128 : 64);  // logical K per stage
    static constexpr int A_BYTES = kBM * 64 * 2;                  // 128 rows x 128 B
    static constexpr int B_ATOM_BYTES = BN_HALF * 64 * 2;        // BN/2 rows x 128 B
    static constexpr int B_BYTES = (FP8 ? 2 : BK / 64) * B_ATOM_BYTES;
    static constexpr int E_CHUNKS = SPARSE ? (FP8 ? 2 : 1) : 0;  // metadata chunks (128 logical K each) per stage
    static constexpr int E_BYTES = E_CHUNKS * kChunkBytes;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + E_BYTES + 1023) / 1024) * 1024;
    static constexpr int STAGES = SPARSE ? 4 : 6;
    static constexpr int LORA_A_BYTES = kBM * 64 * 2;
    static constexpr int LORA_B_BYTES = BN_HALF * 64 * 2;
    static constexpr int EPI_BYTES = 4 * 2 * kEpiBufBytes;
    static constexpr int QW_BYTES = FP8 ? 4 * BN * 4 : 0;  // FP8: each epilogue warp's copy of the tile's q_w
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + QW_BYTES + BAR_BYTES + 1024;
    static_assert(BN % (FP8 ? 32 : 16) == 0 && BN >= 64 && 2 * BN + 4 * E_CHUNKS <= 512,
                  "two accumulators (and, when sparse, the metadata) must fit");
    static_assert(B_ATOM_BYTES % 1024 == 0, "operand tiles must stay 1024-byte aligned");
    static_assert(LORA_A_BYTES <= A_BYTES && LORA_B_BYTES <= B_BYTES, "LoRA tiles must fit the operand slots");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct PairArgs {
    int M, N;
    int m_pairs, n_tiles;
    int group_n;       // column tiles per raster group (see tile_coords)
    int k_stages;      // main-loop stages per tile (128-wide K chunks when sparse, 64-wide when dense)
    int lora_stages;   // 64-wide LoRA stages per tile
    int k_chunks;      // metadata chunks per 128-row block
    // schedule: tiles [0, full_tiles) round-robin over the pairs; tile
    // full_tiles + u / tail_split is cut along K, part u % tail_split going to
    // pair u (u < tail_units)
    int full_tiles, tail_split, tail_units;
    float* split_part;  // fp32 partial tile of each part, per CTA of the pair
    int* split_cnt;     // arrival ticket of each split tile, per CTA of the pair (zeroed by the prologue)
    uint16_t* Y;        // [M, N] bf16 output, row-major (the dense-skip epilogue stores to it directly)
    const float* qx;    // FP8: [M_pad] per-token scale
    const float* qw;    // FP8: [N] per-channel scale (0 for an all-zero channel, applied as 1)
    int* err;
};

// GELU, erf form: x * Phi(x) = x/2 (1 + erf(x / sqrt 2)), in float.
// erfc(z) for z = |x| / sqrt 2 >= 0 comes from Hastings' rational
// approximation as printed in Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26: erfc(z) ~ (a1 t + ... + a5 t^5) exp(-z^2) with
// t = 1 / (1 + p z), absolute error at most 1.5e-7.  Working with erfc
// avoids the cancellation of 1 + erf for negative x:
//   x >= 0:  GELU = x (1 - erfc(z) / 2),    x < 0:  GELU = x erfc(z) / 2.
// About fifteen instructions (one reciprocal, one exponential), so the GEMM
// epilogue stays cheaper than the main loop it overlaps.
__device__ __forceinline__ float gelu_erf(float x) {
    const float z = fabsf(x) * 0.70710678118654752f;
    const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
    float poly = fmaf(t, 1.061405429f, -1.453152027f);
    poly = fmaf(t, poly, 1.421413741f);
    poly = fmaf(t, poly, -0.284496736f);
    poly = fmaf(t, poly, 0.254829592f);
    poly *= t;
    const float half_erfc = 0.5f * poly * __expf(-z * z);
    return x >= 0.0f ? fmaf(-x, half_erfc, x) : x * half_erfc;
}

// Raster order of the tiles: column tiles are taken in groups of group_n; a
// group's tiles are numbered row pair by row pair, so a wave of consecutive
// tiles covers a few row pairs across group_n column tiles, and the group's
// slice of W stays in L2 while all row pairs sweep past it.  The last group
// may be narrower.
__device__ __forceinline__ void tile_coords(int tile, const PairArgs& a, int& mp, int& nt) {
    const int per_group = a.m_pairs * a.group_n;
    const int g = tile / per_group;
    const int width = min(a.group_n, a.n_tiles - g * a.group_n);
    const int local = tile - g * per_group;
    mp = local / width;
    nt = g * a.group_n + local % width;
}

// One work item of a pair: output tile `tile` over stages [kb, ke) of its
// k_stages + lora_stages stages; `unit` >= 0 marks a part of a split tile.
struct PairWork {
    int tile, kb, ke, unit;
};

__device__ __forceinline__ bool pair_work(int idx, int pair, int num_pairs, const PairArgs& a, PairWork& w) {
    const int n_iter = a.k_stages + a.lora_stages;
    const int ndp = pair < a.full_tiles ? (a.full_tiles - pair + num_pairs - 1) / num_pairs : 0;
    if (idx < ndp) {
        w.tile = pair + idx * num_pairs;
        w.kb = 0;
        w.ke = n_iter;
        w.unit = -1;
        return true;
    }
    if (idx == ndp && pair < a.tail_units) {
        const int j = pair % a.tail_split;
        w.tile = a.full_tiles + pair / a.tail_split;
        w.kb = j * n_iter / a.tail_split;
        w.ke = (j + 1) * n_iter / a.tail_split;
        w.unit = pair;
        return true;
    }
    return false;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* err) {
    uint32_t ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err) ? 1u : 0u;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// One 32-column chunk of the accumulator (16 columns when `half`) into r,
// waited for.  `half` must be the same in the whole warp.
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, bool half, uint32_t (&r)[32]) {
    if (half) {
        uint32_t h[16];
        tmem_ld_32x32b_x16(taddr, h);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) r[q] = h[q];
    } else {
        tmem_ld_32x32b_x32(taddr, r);
        tmem_ld_wait();
    }
}

// Rounds 32 (or 16, when `half`) fp32 values of row `row`, columns col ..,
// to bf16 and stores them straight to Y in 16-byte pieces.  Rows >= M and
// columns >= N (the ragged edges) are skipped; N is a multiple of 8, so every
// 8-column piece is wholly inside or wholly outside.  Dense-skip mode writes Y
// this way: plain stores leave the TMA unit to the producer's loads and
// measured faster there; the sparse mode measured faster with staged TMA
// stores.
__device__ __forceinline__ void store_row_bf16(const PairArgs& a, int row, int col, bool half, const uint32_t (&r)[32]) {
    if (row >= a.M) return;
    uint4* dst = reinterpret_cast<uint4*>(a.Y + static_cast<size_t>(row) * a.N + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if ((!half || q < 2) && col + 8 * q < a.N) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
            pk.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
            pk.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
            pk.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
            dst[q] = pk;
        }
    }
}

template <bool SPARSE, int BN, int ACT, bool FP8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    rtlynx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmLA,
                            const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                            const __grid_constant__ CUtensorMap tmY16, const PairArgs args) {
    using G = PairShape<SPARSE, BN, FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi = smem + G::STAGES * G::STAGE_BYTES;
    float* qw_sh = reinterpret_cast<float*>(epi + G::EPI_BYTES);  // FP8 only: [4 warps][BN]
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + G::EPI_BYTES + G::QW_BYTES);
    uint64_t* empty = full + G::STAGES;
    uint64_t* acc_full = empty + G::STAGES;   // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2], used in the leader only
    uint64_t* done_bar = acc_empty + 2;
    uint64_t* epi_done = done_bar + 1;  // split tile: the four epilogue warps stored their partials
    uint64_t* epi_dec = epi_done + 1;   // split tile: the ticket has been read
    uint64_t* fix_full = epi_dec + 1;   // [8] split fix-up: a chunk of the other parts has landed
    uint64_t* fix_empty = fix_full + 8; // [8] split fix-up: the four epilogue warps are done with it
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fix_empty + 8);
    uint32_t* epi_last = tmem_holder + 1;  // split tile: this CTA sums the parts

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
        mbar_init(epi_done, 4);
        mbar_init(epi_dec, 1);
        for (int b = 0; b < 8; ++b) {
            mbar_init(&fix_full[b], 1);
            mbar_init(&fix_empty[b], 4);
        }
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
    // The GEMM is launched as a programmatic dependent of the preceding kernel
    // (the prologue in sparse mode): the setup above overlaps its tail, the
    // operands are read after this.
    grid_dependency_wait();

    PairWork w;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int idx = 0; ok && pair_work(idx, pair, num_pairs, args, w); ++idx) {
                int mp, nt;
                tile_coords(w.tile, args, mp, nt);
                const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;
                const int col0 = nt * BN + static_cast<int>(rank) * G::BN_HALF;
                const int chunk0 = (row0 / kBM) * args.k_chunks;
                for (int kt = w.kb; kt < w.ke; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + stage * G::STAGE_BYTES;
                    uint8_t* sB = sA + G::A_BYTES;
                    const uint32_t fbar = full0 + static_cast<uint32_t>(stage) * 8u;
                    if (kt < args.k_stages) {
                        if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (G::A_BYTES + G::B_BYTES + G::E_BYTES));
                        // A and B coordinates count elements: 128-byte rows hold 64 bf16 or 128 E4M3
                        constexpr int kRowElems = FP8 ? 128 : 64;
                        tma_load_2d_pair(sA, &tmA, fbar, kt * kRowElems, row0);
                        tma_load_2d_pair(sB, &tmB, fbar, kt * G::BK, col0);
                        if constexpr (SPARSE) {
                            tma_load_2d_pair(sB + G::B_ATOM_BYTES, &tmB, fbar, kt * G::BK + kRowElems, col0);
                            tma_load_2d_pair(sB + G::B_BYTES, &tmE, fbar, 0, (chunk0 + kt * G::E_CHUNKS) * 4);
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
        if (leader) {
            // The whole warp runs the issue loop, so its descriptors and counters
            // are warp-uniform values; one elected lane (always the same one, so
            // its commits track all of its MMAs) issues the tcgen05 instructions.
            // Measured against lane 0 running the loop alone: 2-4% faster GEMMs
            // (qkv sparse 105.4 -> 102.0 us, dense-skip 146.9 -> 141.3 us).
            const uint32_t idesc_main = FP8 ? make_idesc_e4m3(2 * kBM, BN, true) : make_idesc_bf16(2 * kBM, BN, SPARSE);
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
            bool ok = true;
            for (int local = 0; ok && pair_work(local, pair, num_pairs, args, w); ++local) {
                const int buf = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kt = w.kb; kt < w.ke; ++kt) {
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[stage], phase, err))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a = descA0 + off;
                    const uint64_t b = descB0 + off;
                    const uint32_t acc = kt != w.kb;  // the item's first stage starts the accumulator
                    if (!elect_one()) {
                        // the other lanes only keep the loop's state
                    } else if (kt < args.k_stages) {
                        if constexpr (FP8) {
                            // two metadata chunks -> columns [meta, meta + 8); MMA j reads columns meta + 2j, + 2j + 1
                            tmem_cp_128x128b_pair(tmem_meta, descE0 + off);
                            tmem_cp_128x128b_pair(tmem_meta + 4u, descE0 + off + (kChunkBytes >> 4));
                            mma_sp_f8_pair(d, a, b, tmem_meta, idesc_main, acc);
                            mma_sp_f8_pair(d, a + 2, b + 4, tmem_meta + 2u, idesc_main, 1u);
                            mma_sp_f8_pair(d, a + 4, b + kAtomStep, tmem_meta + 4u, idesc_main, 1u);
                            mma_sp_f8_pair(d, a + 6, b + kAtomStep + 4, tmem_meta + 6u, idesc_main, 1u);
                        } else if constexpr (SPARSE) {
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
                        mma_f16_pair(d, a, b, idesc_dense, acc);
                        mma_f16_pair(d, a + 2, b + 2, idesc_dense, 1u);
                        mma_f16_pair(d, a + 4, b + 4, idesc_dense, 1u);
                        mma_f16_pair(d, a + 6, b + 6, idesc_dense, 1u);
                    }
                    if (elect_one()) tc_commit_pair_mc(&empty[stage], 0x3);
                    off += kStageStep;
                    if (++stage == G::STAGES) {
                        stage = 0;
                        off = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (elect_one()) tc_commit_pair_mc(&acc_full[buf], 0x3);
            }
            // Every MMA of the pair has finished before tensor memory is freed.
            if (elect_one()) tc_commit_pair_mc(done_bar, 0x1);
            mbar_wait(done_bar, 0, nullptr);
        }
        __syncwarp();
    } else {
        const int quad = warp & 3;  // warps 2..5 own tensor-memory lane quadrants 2,3,0,1
        const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
        const int row_in_cta = quad * 32 + lane;
        uint8_t* stage_buf = epi + (warp - 2) * 2 * kEpiBufBytes;
        int sbuf = 0;
        for (int local = 0; pair_work(local, pair, num_pairs, args, w); ++local) {
            const int buf = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            int mp, nt;
            tile_coords(w.tile, args, mp, nt);
            const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM + quad * 32;
            const int col0 = nt * BN;
            const uint32_t acc = tmem_base + static_cast<uint32_t>(buf * BN) + lane_addr;
            const bool split = w.unit >= 0;
            float* qw_w = qw_sh + (warp - 2) * BN;  // FP8: this warp's copy of the tile's q_w
            float qxr = 0.0f;                        // FP8: q_x of this lane's token, loaded once per tile
            if constexpr (FP8) {
                qxr = __ldg(args.qx + row0 + lane);
                // one coalesced pass per tile, every load in flight before the
                // first store (the stores go through a generic pointer, so loads
                // interleaved with them would each wait out their own latency);
                // zero scales (all-zero channels) and columns past N apply as 1
                constexpr int kQw = (BN + 31) / 32;
                float qv[kQw];
#pragma unroll
                for (int i = 0; i < kQw; ++i) {
                    const int j = lane + 32 * i;
                    qv[i] = (j < BN && col0 + j < args.N) ? __ldg(args.qw + col0 + j) : 1.0f;
                }
#pragma unroll
                for (int i = 0; i < kQw; ++i) {
                    const int j = lane + 32 * i;
                    if (j < BN) qw_w[j] = qv[i] > 0.0f ? qv[i] : 1.0f;
                }
                __syncwarp();
            }
            // the scales above do not depend on the accumulator: their loads
            // overlap the main loop of this tile
            if (!warp_wait(&acc_full[buf], use & 1u, err)) break;
            tc_fence_after();
            bool write_y = true;
            const int S = args.tail_split;
            const int tt = w.tile - args.full_tiles;  // index among the split tiles
            const int my_j = split ? w.unit % S : 0;
            // fp32 partial slot of part j of this split tile, this CTA's half
            auto slot = [&](int j) {
                return args.split_part + (static_cast<size_t>(tt * S + j) * 2 + rank) * kSplitSlotFloats;
            };
            // Fix-up buffers: the pipeline stages, idle once the accumulator of
            // the pair's last work item (the split part) is complete.  They
            // form a ring of `nslot` slots; slot b holds chunk c (c % nslot ==
            // b) of the S - 1 other parts, 16 KB each.  With two parts every
            // chunk has its own slot and all of them are requested at once.
            constexpr uint32_t kFixChunk = kBM * 32 * 4;
            constexpr int kChunks = (BN + 31) / 32;
            const int per_slot = (S > 1 ? S - 1 : 1) * static_cast<int>(kFixChunk);
            int nslot = (G::STAGES * G::STAGE_BYTES) / per_slot;
            nslot = nslot < kChunks ? nslot : kChunks;
            auto fix_issue = [&](int c) {  // one thread
                const int b = c % nslot;
                uint8_t* dst = smem + b * per_slot;
                const uint32_t bytes = (BN - c * 32) < 32 ? kFixChunk / 2 : kFixChunk;
                mbar_arrive_expect_tx(&fix_full[b], bytes * static_cast<uint32_t>(S - 1));
                for (int j = 0, jj = 0; j < S; ++j) {
                    if (j == my_j) continue;
                    bulk_load(dst + jj * kFixChunk, slot(j) + c * (kFixChunk / 4), bytes, &fix_full[b]);
                    ++jj;
                }
            };
            if (split) {
                // This CTA's fp32 partial goes to its slot; the last of the
                // tile's parts to arrive sums all of them in part order.
                float* own = slot(my_j);
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t r[32];
                    const bool half = (BN - c) < 32;
                    tmem_ld_chunk(acc + static_cast<uint32_t>(c), half, r);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (!half || q < 4)
                            reinterpret_cast<float4*>(own)[((c / 32) * 8 + q) * kBM + row_in_cta] =
                                make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                            __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) mbar_arrive(epi_done);
                if (warp == 2) {
                    const bool stored = warp_wait(epi_done, 0, err);
                    if (lane == 0) {
                        uint32_t last = 0;
                        if (stored) {
                            const int old = atomicAdd(&args.split_cnt[tt * 2 + rank], 1);
                            last = old == S - 1;
                            if (last) {
                                __threadfence();
                                args.split_cnt[tt * 2 + rank] = 0;
                                for (int c = 0; c < nslot; ++c) fix_issue(c);
                            }
                        }
                        *epi_last = last;
                        mbar_arrive(epi_dec);
                    }
                    __syncwarp();
                }
                if (!warp_wait(epi_dec, 0, err)) break;
                write_y = *reinterpret_cast<volatile uint32_t*>(epi_last) != 0;
            }
            if (write_y) {
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    const bool half = (BN - c) < 32;  // 16-column tail chunk
                    const int ci = c / 32;
                    uint32_t r[32];
                    if (!split) {
                        tmem_ld_chunk(acc + static_cast<uint32_t>(c), half, r);
                    } else {
                        const int b = ci % nslot;
                        const uint32_t round = static_cast<uint32_t>(ci / nslot);
                        if (!warp_wait(&fix_full[b], round & 1u, err)) break;
                        const uint8_t* fb = smem + b * per_slot;
                        float sum[32];
#pragma unroll
                        for (int q = 0; q < 32; ++q) sum[q] = 0.f;
                        for (int j = 0, jj = 0; j < S; ++j) {
                            uint32_t t[32];
                            if (j == my_j) {
                                tmem_ld_chunk(acc + static_cast<uint32_t>(c), half, t);
                            } else {
                                const float4* src = reinterpret_cast<const float4*>(fb + jj * kFixChunk);
#pragma unroll
                                for (int q = 0; q < 8; ++q) {
                                    if (!half || q < 4) {
                                        const float4 v = src[q * kBM + row_in_cta];
                                        t[4 * q] = __float_as_uint(v.x);
                                        t[4 * q + 1] = __float_as_uint(v.y);
                                        t[4 * q + 2] = __float_as_uint(v.z);
                                        t[4 * q + 3] = __float_as_uint(v.w);
                                    }
                                }
                                ++jj;
                            }
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                if (!half || q < 16) sum[q] += __uint_as_float(t[q]);
                        }
#pragma unroll
                        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(sum[q]);
                        __syncwarp();
                        if (ci + nslot < kChunks) {  // refill this slot with chunk ci + nslot
                            if (lane == 0) mbar_arrive(&fix_empty[b]);
                            if (warp == 2) {
                                const bool free_slot = warp_wait(&fix_empty[b], round & 1u, err);
                                if (lane == 0 && free_slot) fix_issue(ci + nslot);
                                __syncwarp();
                            }
                        }
                    }
                    if constexpr (FP8) {  // dequantise: q_x of the token times q_w of the column
                        const float4* w4 = reinterpret_cast<const float4*>(qw_w + c);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 w = w4[q];  // the same address in every lane: a broadcast
                            r[4 * q + 0] = __float_as_uint(__uint_as_float(r[4 * q + 0]) * (qxr * w.x));
                            r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) * (qxr * w.y));
                            r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) * (qxr * w.z));
                            r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) * (qxr * w.w));
                        }
                    }
                    if constexpr (ACT == 1) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(gelu_erf(__uint_as_float(r[q])));
                    }
                    if constexpr (!SPARSE) {
                        store_row_bf16(args, row0 + lane, col0 + c, half, r);
                        continue;
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

template <bool SPARSE, int BN, int ACT, bool FP8 = false>
static int launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmT,
                       const CUtensorMap& tmLA, const CUtensorMap& tmE, const CUtensorMap& tmY,
                       const CUtensorMap& tmY16, const PairArgs& args, int num_sms, cudaStream_t stream) {
    using G = PairShape<SPARSE, BN, FP8>;
    auto kernel = rtlynx_gemm_pair_kernel<SPARSE, BN, ACT, FP8>;
    static std::atomic<uint64_t> smem_set{0};
    const int e = allow_max_dynamic_smem(kernel, smem_set);
    if (e) return e;
    const int tiles = args.m_pairs * args.n_tiles;
    const int max_pairs = num_sms / 2;
    const int pairs = tiles < max_pairs ? tiles : max_pairs;
    // A programmatic dependent of whatever ran before (the prologue in sparse
    // mode): the setup overlaps that kernel's tail, the operands are read
    // after grid_dependency_wait.
    return launch_dependent(kernel, dim3(2 * pairs), dim3(kPairThreads), G::SMEM_BYTES, stream, tmA, tmB, tmT, tmLA,
                            tmE, tmY, tmY16, args);
}

int launch_gemm(const Dims& d, bool sparse, const void* A, const void* W, const void* L_A, const Workspace& ws,
                void* Y, int act, int num_sms, int* err, cudaStream_t stream, const float* qw) {
    // Sparse tiles are 240 wide so that two accumulators and the metadata fit
    // in 512 tensor-memory columns; dense-skip tiles carry no metadata and are
    // 256 wide (two accumulators fill the 512 columns).
    const bool fp8 = sparse && d.fp8;
    if (fp8 && (act != 0 || !qw || d.K % kFp8StageK)) return static_cast<int>(cudaErrorInvalidValue);
    const int BN = fp8 ? kFp8BN : (sparse ? kPairBN : kDenseBN);
    CUtensorMap tmA, tmB, tmT, tmLA, tmE, tmY, tmY16;
    int rc;
    if (fp8) {
        // E4M3 codes of the kept entries and of W (one byte each), 128-byte boxes
        rc = encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws.codes, d.Kc_pad, d.M_pad, d.Kc_pad, 128, kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        // two metadata chunks per stage: eight rows of 256 16-bit words
        rc = encode_tmap_2d(&tmE, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, ws.meta, 256, d.m_blocks * d.k_chunks * 4, 512,
                            256, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc) return rc;
    } else if (sparse) {
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
    rc = fp8 ? encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, W, d.K, d.N, d.K, 128, BN / 2,
                              CU_TENSOR_MAP_SWIZZLE_128B)
             : encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, d.K, d.N, d.K * 2, kBK, BN / 2,
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
    args.k_stages = static_cast<int>(sparse ? sparse_k_stages(d) : d.k_tiles);
    args.lora_stages = lora ? static_cast<int>(sparse_lora_stages(d)) : 0;
    args.k_chunks = static_cast<int>(d.k_chunks);
    {
        // While both operands fit in L2 (126 MB) the row-pair-fastest order
        // (group width 1) serves each W tile to many pairs of one wave.  When
        // they do not, column tiles are grouped so that a group's W slice,
        // about 48 MiB, stays in L2 while the row pairs sweep past it.
        const double a_bytes = static_cast<double>(d.M_pad) * static_cast<double>(d.K) * (sparse ? 1.125 : 2.0);
        const double w_bytes = static_cast<double>(d.N) * static_cast<double>(d.K) * 2.0;
        int gn = 1;
        if (a_bytes + w_bytes > 192.0 * (1 << 20)) {
            const double w_tile_bytes = static_cast<double>(BN) * static_cast<double>(d.K) * 2.0;
            gn = static_cast<int>((48.0 * (1 << 20)) / w_tile_bytes);
            gn = gn < 1 ? 1 : (gn > args.n_tiles ? args.n_tiles : gn);
        }
        args.group_n = gn;
    }
    if (sparse) {
        args.full_tiles = static_cast<int>(d.tail_full);
        args.tail_split = static_cast<int>(d.tail_split);
        args.tail_units = static_cast<int>(d.tail_units);
    } else {  // dense-skip has no workspace: every tile whole, round-robin
        args.full_tiles = args.m_pairs * args.n_tiles;
        args.tail_split = 1;
        args.tail_units = 0;
    }
    args.split_part = ws.split_part;
    args.split_cnt = ws.split_cnt;
    args.Y = static_cast<uint16_t*>(Y);
    args.qx = ws.qx;
    args.qw = qw;
    args.err = err;
    if (fp8) return launch_pair<true, kFp8BN, 0, true>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream);
    // the epilogue activation is a template parameter, so the plain kernels carry no GELU code
    if (act == 1)
        return sparse ? launch_pair<true, kPairBN, 1>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream)
                      : launch_pair<false, kDenseBN, 1>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream);
    return sparse ? launch_pair<true, kPairBN, 0>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream)
                  : launch_pair<false, kDenseBN, 0>(tmA, tmB, tmT, tmLA, tmE, tmY, tmY16, args, num_sms, stream);
}

}  // namespace rtlynx
