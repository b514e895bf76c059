// The RT-Lynx linear layer for small problems in one kernel (RT-Lynx summary
// page, four-step pipeline paragraph: step 1, the 2-of-4 mask and the
// norm-compensating scale s; step 2, Y = S(X) W^T + X (L_A L_B)^T; step 4,
// mask, Top-K and compression fused with the sparse GEMM, Y_s and Y_r summed
// on chip).
//
// Where a problem is one wave of output tiles and a 128-token block of X fits
// in shared memory whole (D_in <= 256), the three launches of the general path
// (two sparsify passes and the GEMM) cost more than their work: every kernel
// moves well under a megabyte and pays its own launch, setup and drain.  Here
// each CTA pair sparsifies its own 256 tokens in shared memory and computes one
// 256 x 240 output tile:
//   - thread 0 loads the CTA's 128 tokens of X, its 32 rows of L_B, its 120
//     rows of the W tile and of L_A, all at once (TMA, 128-byte swizzle),
//     before the pair's set-up so the loads overlap it;
//   - warps 2-17 rank every group of four (the integer keys of sparsify_math.cuh); a token is
//     held whole, so the exact sums of x^2 and of the kept x^2 give s in the
//     same pass, and the kept entries go straight into shared memory as
//     bf16(s x), in the swizzled layout of the sparse MMA's A operand, with
//     their metadata bytes in tensor-memory order;
//   - warp 1 (leader CTA) issues T = X L_B^T on tcgen05 from the X tiles
//     while they rank; warps 0, 1, 18 and 19 (one per tensor-memory lane
//     quadrant) round T to bf16 into shared memory, and warp 1 issues
//     T L_A^T into the accumulator, all before S(X) is ready; the sparse
//     MMAs over the W tile then accumulate onto it (the order of the two
//     fp32 sums differs from the general path's, within the same bar);
//   - warps 2-9 write Y as the general GEMM's epilogue does, staging in the
//     X tiles (free once the accumulator is complete).
// The CTA pairs of column tile 0 also copy the kept values, metadata and T
// out of shared memory to the workspace in the general path's layout (what
// the parity checks and the debug export read), and s.  Rows past M and
// channels past D_in are zeros: their groups keep entries 0 and 1 (metadata
// 0x4) with zero values, as in the general path, without being ranked.
#include "internal.h"
#include "ptx.cuh"
#include "sparsify_math.cuh"

namespace rtlynx {

namespace {

// warp 0 TMA, warp 1 MMA, warps 2-17 sparsify (2-9 also the epilogue), warps 0, 1, 18, 19 round T
constexpr int kSmallThreads = 640;
constexpr int kSparsifyWarps = 16;
constexpr int kSmallBN = kPairBN;   // 240 output columns per CTA pair
constexpr int kSmallMaxK = 256;
constexpr int kXTile = kBM * 64 * 2;         // 16 KB: 128 tokens x 64 channels
constexpr int kLBTile = 32 * 64 * 2;         // 4 KB: 32 rows of L_B x 64 channels
constexpr int kWAtom = (kSmallBN / 2) * 128; // 15 KB: 120 rows of W x 64 channels
constexpr int kSTile = kBM * 128;            // 16 KB: 128 tokens x 64 kept values
constexpr int kEpiBuf = 32 * 64;             // one warp's 32 rows x 32 bf16 columns

// Shared-memory map (offsets from the 1024-aligned base), for D_in <= 256.
constexpr int kOffX = 0;                                   // 4 X tiles
constexpr int kOffLB = kOffX + 4 * kXTile;                 // 4 L_B tiles
constexpr int kOffW = kOffLB + 4 * kLBTile;                // 2 chunks x 2 W atoms
constexpr int kOffLA = kOffW + 4 * kWAtom;                 // L_A: 120 rows x 64
constexpr int kOffS = kOffLA + kWAtom;                     // 2 S(X) tiles
constexpr int kOffT = kOffS + 2 * kSTile;                  // T: 128 x 64 bf16
constexpr int kOffE = kOffT + kXTile;                      // 2 metadata chunks
constexpr int kOffBar = kOffE + 2 * kChunkBytes;
// The epilogue's staging buffers (8 warps x 2) reuse the X tiles, which the
// last MMA has read before the accumulator is complete.
constexpr int kOffEpi = kOffX;
constexpr int kEpiWarps = 8;
static_assert(kEpiWarps * 2 * kEpiBuf <= 4 * kXTile, "staging fits in the X tiles");
constexpr int kSmallSmem = kOffBar + 1024 + 1024;
static_assert(kSmallSmem <= 232448, "shared memory budget");
static_assert(kOffS % 1024 == 0 && kOffT % 1024 == 0 && kOffLA % 1024 == 0 && kOffW % 1024 == 0,
              "swizzled operands must be 1024-byte aligned");

// Tensor-memory columns: the accumulator, T, the metadata of both chunks.
constexpr uint32_t kColT = kSmallBN;
constexpr uint32_t kColE = kSmallBN + 64;

struct SmallArgs {
    int M, K, N, R_pad;
    int k_chunks;        // 1 or 2
    int m_pairs, n_tiles;
    int lora;            // 1: T L_A^T is added
    // column tile 0 writes these (the general path's workspace layout)
    uint16_t* vals;      // [M_pad, Kc_pad]
    uint8_t* meta;       // [m_blocks, k_chunks, 2048]
    float* s;            // [M_pad]
    uint16_t* T;         // [M_pad, 64]
    int Kc_pad;
    int* err;
};

// T (fp32, tensor memory) -> the bf16 rows of the swizzled shared-memory tile
// that the LoRA-up MMA reads as its A operand: one warp per tensor-memory lane
// quadrant, then an arrive on the leader's t_ready.  In column tile 0 the
// tile is also copied to the workspace, by the `issuer` warp, after the arrive.
__device__ __forceinline__ void round_t(uint8_t* smem, uint32_t tmem_base, int quad, int lane, uint64_t* t_done,
                                        uint64_t* t_ready, bool writer, bool issuer, const CUtensorMap* tmT, int row0,
                                        int* err) {
    uint32_t okw = 0;
    if (lane == 0) okw = mbar_wait(t_done, 0, err) ? 1u : 0u;
    if (__shfl_sync(0xFFFFFFFFu, okw, 0)) {
        tc_fence_after();
        const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
        const int trow = quad * 32 + lane;  // this lane's token within the CTA
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_base + lane_addr + kColT + 32 * half, v);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 pk;
                pk.x = pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1]));
                pk.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                pk.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                pk.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                const int unit = 4 * half + q;  // 16-byte unit of the 128-byte row
                *reinterpret_cast<uint4*>(smem + kOffT + trow * 128 + ((unit ^ (trow & 7)) << 4)) = pk;
            }
        }
        tc_fence_before();
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(t_ready), 0));
    if (writer) {
        if (issuer) {
            named_barrier(2, 128);
            if (lane == 0) {
                tma_store_2d(tmT, smem + kOffT, 0, row0);
                bulk_commit_group();
                bulk_wait_group_read<0>();  // the CTA may exit once shared memory has been read
            }
            __syncwarp();
        } else {
            named_barrier_arrive(2, 128);
        }
    }
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSmallThreads, 1)
    rtlynx_small_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmLB,
                        const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmLA,
                        const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmY16,
                        const __grid_constant__ CUtensorMap tmVals, const __grid_constant__ CUtensorMap tmT,
                        const __grid_constant__ SmallArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* x_full = bars + 0;    // this CTA's X and L_B have landed
    uint64_t* w_full = bars + 1;    // this CTA's W and L_A have landed
    uint64_t* t_go = bars + 2;      // leader: both CTAs' X and L_B landed (2 arrivals)
    uint64_t* w_go = bars + 3;      // leader: both CTAs' W and L_A landed (2)
    uint64_t* s_ready = bars + 4;   // leader: both CTAs' S(X) and metadata written (2 x 16 warps)
    uint64_t* t_ready = bars + 5;   // leader: both CTAs' T rounded into shared memory (8 warps)
    uint64_t* t_done = bars + 6;    // T's MMAs are complete (commit, both CTAs)
    uint64_t* acc_full = bars + 7;  // the accumulator is complete (commit, both CTAs)
    uint64_t* done_bar = bars + 8;  // leader: every MMA of the pair is done
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 9);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int mp = pair / a.n_tiles, nt = pair - mp * a.n_tiles;
    const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;  // this CTA's first token
    const int col0 = nt * kSmallBN;
    int* err = a.err;
    const int n_xt = 2 * a.k_chunks;  // 64-wide X tiles (a padding tile reads as zeros)

    if (threadIdx.x == 0) {  // the descriptors are kernel parameters: fetch them while the grid waits
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
        if (a.lora) {
            prefetch_tmap(&tmLB);
            prefetch_tmap(&tmLA);
        }
    }
    // wait for the kernel before this one (programmatic dependent launch) before any global access
    grid_dependency_wait();

    if (threadIdx.x == 0) {
        mbar_init(x_full, 1);
        mbar_init(w_full, 1);
        mbar_init(t_go, 2);
        mbar_init(w_go, 2);
        mbar_init(s_ready, 2 * kSparsifyWarps);
        mbar_init(t_ready, 8);
        mbar_init(t_done, 1);
        mbar_init(acc_full, 1);
        mbar_init(done_bar, 1);
        fence_mbar_init();
        fence_proxy_async_smem();  // the initialised barriers are visible to the copy engine
        // this CTA's operands land on its own barriers: the loads start before the
        // pair's set-up (tensor-memory allocation, cluster barrier) so the two overlap
        mbar_arrive_expect_tx(x_full, n_xt * (kXTile + (a.lora ? kLBTile : 0)));
        for (int kt = 0; kt < n_xt; ++kt) {
            tma_load_2d(smem + kOffX + kt * kXTile, &tmX, x_full, kt * 64, row0);
            if (a.lora) tma_load_2d(smem + kOffLB + kt * kLBTile, &tmLB, x_full, kt * 64, 32 * static_cast<int>(rank));
        }
        const uint32_t wb = a.k_chunks * 2 * kWAtom + (a.lora ? kWAtom : 0);
        mbar_arrive_expect_tx(w_full, wb);
        const int wrow = col0 + static_cast<int>(rank) * (kSmallBN / 2);
        for (int c = 0; c < a.k_chunks; ++c)
            for (int h = 0; h < 2; ++h)
                tma_load_2d(smem + kOffW + (2 * c + h) * kWAtom, &tmW, w_full, c * 128 + h * 64, wrow);
        if (a.lora) tma_load_2d(smem + kOffLA, &tmLA, w_full, 0, wrow);
        prefetch_tmap(&tmY);
        prefetch_tmap(&tmY16);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // the leader's barriers are initialised before the peer arrives on them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const bool writer = nt == 0;  // column tile 0 writes the workspace copy
    if (warp == 0) {
        // ------------------------------------------------------------ operand arrival
        if (lane == 0) {
            // tell the leader once this CTA's operands are in
            if (mbar_wait(x_full, 0, err) && a.lora) mbar_arrive_cluster(mapa_shared(smem_u32(t_go), 0));
            if (mbar_wait(w_full, 0, err)) mbar_arrive_cluster(mapa_shared(smem_u32(w_go), 0));
        }
        __syncwarp();
        if (a.lora) round_t(smem, tmem_base, 0, lane, t_done, t_ready, writer, false, &tmT, row0, err);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue (leader)
        const uint32_t s0 = smem_u32(smem);
        bool ok = true;
        if (a.lora) {
            if (leader && lane == 0) {
                ok = mbar_wait_cluster(t_go, 0, err);
                if (ok) {
                    tc_fence_after();
                    const uint32_t idesc_T = make_idesc_bf16(2 * kBM, 64, false);
                    for (int kt = 0; kt < n_xt; ++kt) {
                        const uint64_t da = make_sdesc(s0 + kOffX + kt * kXTile, 16, 1024, kSw128);
                        const uint64_t db = make_sdesc(s0 + kOffLB + kt * kLBTile, 16, 1024, kSw128);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_f16_pair(tmem_base + kColT, da + 2 * j, db + 2 * j, idesc_T, (kt | j) != 0);
                    }
                    tc_commit_pair_mc(t_done, 0x3);
                }
            }
            __syncwarp();
            // the whole warp rounds quadrant 1 of T while the sparsify warps rank
            round_t(smem, tmem_base, 1, lane, t_done, t_ready, writer, false, &tmT, row0, err);
        }
        if (leader && lane == 0) {
            const uint32_t idesc_sp = make_idesc_bf16(2 * kBM, kSmallBN, true);
            const uint32_t idesc_d = make_idesc_bf16(2 * kBM, kSmallBN, false);
            if (ok) ok = mbar_wait_cluster(w_go, 0, err);
            // T L_A^T first: T is rounded while the sparsify warps still rank, so
            // these MMAs run before S(X) is ready; the sparse ones accumulate onto them
            if (ok && a.lora) {
                ok = mbar_wait_cluster(t_ready, 0, err);
                if (ok) {
                    tc_fence_after();
                    const uint64_t da = make_sdesc(s0 + kOffT, 16, 1024, kSw128);
                    const uint64_t db = make_sdesc(s0 + kOffLA, 16, 1024, kSw128);
#pragma unroll
                    for (int j = 0; j < 4; ++j) mma_f16_pair(tmem_base, da + 2 * j, db + 2 * j, idesc_d, j != 0);
                }
            }
            if (ok) ok = mbar_wait_cluster(s_ready, 0, err);
            if (ok) {
                tc_fence_after();
                const uint64_t de = make_sdesc(s0 + kOffE, 128, 128, kSwNone);
                for (int c = 0; c < a.k_chunks; ++c)
                    tmem_cp_128x128b_pair(tmem_base + kColE + 4 * c, de + ((c * kChunkBytes) >> 4));
                for (int c = 0; c < a.k_chunks; ++c) {
                    const uint64_t da = make_sdesc(s0 + kOffS + c * kSTile, 16, 1024, kSw128);
                    const uint64_t db = make_sdesc(s0 + kOffW + 2 * c * kWAtom, 16, 1024, kSw128);
                    constexpr uint64_t kAtom = kWAtom >> 4;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t ecol = tmem_base + kColE + 4 * c + j;  // metadata of MMA j
                        const uint64_t b = db + (j >> 1) * kAtom + 4 * (j & 1);
                        mma_sp_f16_pair(tmem_base, da + 2 * j, b, ecol & ~1u, idesc_sp | (ecol & 1u),
                                        a.lora || (c | j) != 0);
                    }
                }
                tc_commit_pair_mc(acc_full, 0x3);
            }
            tc_commit_pair_mc(done_bar, 0x1);
            mbar_wait(done_bar, 0, nullptr);
        }
        __syncwarp();
    } else if (warp >= 2 + kSparsifyWarps) {
        // ------------------------------------------------------------ T rounding, quadrants 2 and 3
        if (a.lora) round_t(smem, tmem_base, warp & 3, lane, t_done, t_ready, writer, warp == 2 + kSparsifyWarps, &tmT,
                            row0, err);
    } else {
        // ------------------------------------------------------------ sparsify (warps 2-17)
        // thread: token r of this CTA, quarter h of its channels (64 each)
        const int tid = threadIdx.x - 64;
        const int r = tid >> 2, h = tid & 3;
        const int units = a.k_chunks * 4;  // 8-channel units in each quarter
        const int m0 = r & 7, m1 = (r >> 3) & 1, m2 = r >> 4;
        const int64_t grow = row0 + r;
        uint32_t kept[8][2];               // unscaled kept pairs of each unit (units <= 8)
        uint32_t nib[8];
        double nx = 0.0, ntop = 0.0;
        float s = 0.0f;
        {
            const bool live = grow < a.M;  // rows past M are padding: zeros
            mbar_wait(x_full, 0, err);  // a timeout sets the error word: the result is then void
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < units) {
                    const int u = h * units + i;  // unit of the token (8 channels)
                    if (live && 8 * u < a.K) {
                        const int kt = u >> 3, q = u & 7;  // X tile, 16-byte unit in its 128-byte row
                        const uint4 x = *reinterpret_cast<const uint4*>(smem + kOffX + kt * kXTile + r * 128 +
                                                                       ((q ^ (r & 7)) << 4));
                        const GroupKeys g0 = rank_group(x.x, x.y), g1 = rank_group(x.z, x.w);
                        nib[i] = pick_kept(g0, x.x, x.y, kept[i][0]) | (pick_kept(g1, x.z, x.w, kept[i][1]) << 4);
                        if (group_all_normal(g0) && group_all_normal(g1)) {
                            group_energy_normal(g0, nx, ntop);
                            group_energy_normal(g1, nx, ntop);
                        } else {
                            double2 e = group_energy_any(g0.k1, g0.k2, g0.k3, g0.k4);
                            nx += e.x;
                            ntop += e.y;
                            e = group_energy_any(g1.k1, g1.k2, g1.k3, g1.k4);
                            nx += e.x;
                            ntop += e.y;
                        }
                    } else {  // padding: both groups keep entries 0 and 1, values zero
                        nib[i] = 0x44u;
                        kept[i][0] = kept[i][1] = 0u;
                    }
                }
            }
        }
        {
            // the token's four quarters are neighbouring lanes (summed in a fixed order)
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                nx += __shfl_xor_sync(0xFFFFFFFFu, nx, o);
                ntop += __shfl_xor_sync(0xFFFFFFFFu, ntop, o);
            }
            s = static_cast<float>(sqrt(nx) / (sqrt(ntop) + 1e-8));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < units) {
                    const int u = h * units + i;
                    uint2 v;
                    v.x = scale_pair(s, kept[i][0]);
                    v.y = scale_pair(s, kept[i][1]);
                    // A operand: chunk u / 16, kept values 4 (u % 16) .. + 3 of the row
                    const int c = u >> 4, uc = u & 15;
                    *reinterpret_cast<uint2*>(smem + kOffS + c * kSTile + r * 128 + (((uc >> 1) ^ (r & 7)) << 4) +
                                              8 * (uc & 1)) = v;
                    // metadata byte of the unit's two groups in the chunk's tensor-memory order
                    const int k1 = (uc >> 1) & 1, k2 = uc >> 2;
                    const int dp = m0 + 8 * k1 + 16 * m2;
                    const int byte = 16 * dp + 4 * k2 + 2 * m1 + (uc & 1);
                    smem[kOffE + c * kChunkBytes + byte] = static_cast<uint8_t>(nib[i]);
                }
            }
        }
        // S(X) and the metadata are read by the tensor cores and the bulk copies (async proxy)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(s_ready), 0));
        if (writer && warp == 1 + kSparsifyWarps) {
            // the workspace copy, by the last sparsify warp (not a T or epilogue warp):
            // the S(X) tiles are already in the TMA's 128-byte swizzle, the metadata
            // chunks in the workspace's byte order.  It is issued after the arrive:
            // a release waits for the thread's bulk copies in flight.
            named_barrier(1, 32 * kSparsifyWarps);
            if (lane == 0) {
                for (int c = 0; c < a.k_chunks; ++c) {
                    tma_store_2d(&tmVals, smem + kOffS + c * kSTile, c * 64, row0);
                    bulk_store(a.meta + (static_cast<int64_t>(row0 / kBM) * a.k_chunks + c) * kChunkBytes,
                               smem + kOffE + c * kChunkBytes, kChunkBytes);
                }
                bulk_commit_group();
                bulk_wait_group_read<0>();  // the CTA may exit once shared memory has been read
            }
            __syncwarp();
        } else if (writer) {
            named_barrier_arrive(1, 32 * kSparsifyWarps);
        }
        // s goes to the workspace after the release-arrive: a release waits until
        // the thread's earlier global stores are acknowledged
        if (writer && h == 0) a.s[grow] = s;

        if (warp < 2 + kEpiWarps) {
            const int quad = warp & 3;  // warps 2..9 own tensor-memory lane quadrants 2,3,0,1,2,3,0,1
            const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
            // ---- the epilogue: 32-column chunks -> bf16 -> swizzled staging -> TMA store;
            // warps 2..5 take columns 0..127 of the tile, warps 6..9 the rest
            const int c_begin = warp < 6 ? 0 : 128, c_end = warp < 6 ? 128 : kSmallBN;
            uint32_t okw = 0;
            if (lane == 0) okw = mbar_wait(acc_full, 0, err) ? 1u : 0u;
            if (__shfl_sync(0xFFFFFFFFu, okw, 0)) {
                tc_fence_after();
                uint8_t* stage_buf = smem + kOffEpi + (warp - 2) * 2 * kEpiBuf;
                const int yrow = row0 + quad * 32;
                int sbuf = 0;
#pragma unroll 1
                for (int c = c_begin; c < c_end; c += 32) {
                    const bool half = (kSmallBN - c) < 32;
                    uint32_t r32[32];
                    if (half) {
                        uint32_t h16[16];
                        tmem_ld_32x32b_x16(tmem_base + lane_addr + c, h16);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 16; ++q) r32[q] = h16[q];
                    } else {
                        tmem_ld_32x32b_x32(tmem_base + lane_addr + c, r32);
                        tmem_ld_wait();
                    }
                    uint8_t* sb = stage_buf + sbuf * kEpiBuf;
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    const int n16 = half ? 2 : 4;  // 16-byte units of the row
                    uint8_t* row = sb + lane * (half ? 32 : 64);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (q < n16) {
                            uint4 pk;
                            pk.x = pack_bf16x2(__uint_as_float(r32[8 * q + 0]), __uint_as_float(r32[8 * q + 1]));
                            pk.y = pack_bf16x2(__uint_as_float(r32[8 * q + 2]), __uint_as_float(r32[8 * q + 3]));
                            pk.z = pack_bf16x2(__uint_as_float(r32[8 * q + 4]), __uint_as_float(r32[8 * q + 5]));
                            pk.w = pack_bf16x2(__uint_as_float(r32[8 * q + 6]), __uint_as_float(r32[8 * q + 7]));
                            // 64B swizzle: unit q of row i at q ^ ((i / 2) % 4); 32B: q ^ ((i / 4) % 2)
                            const int sw = half ? (q ^ ((lane >> 2) & 1)) : (q ^ ((lane >> 1) & 3));
                            *reinterpret_cast<uint4*>(row + (sw << 4)) = pk;
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(half ? &tmY16 : &tmY, sb, col0 + c, yrow);
                        bulk_commit_group();
                    }
                    sbuf ^= 1;
                }
                // the CTA may exit once the copies have read shared memory
                if (lane == 0) bulk_wait_group_read<0>();
            }
        }
    }

    __syncwarp();
    if (error_seen(err)) {  // after an abort, let copies in flight land before shared memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

bool small_path_fits(const Dims& d, int num_sms) {
    if (d.fp8 || d.K > kSmallMaxK || (d.R_pad != 0 && d.R_pad != 64)) return false;
    const int64_t pairs = (d.M_pad / (2 * kBM)) * ((d.N + kSmallBN - 1) / kSmallBN);
    return pairs <= (num_sms > 0 ? num_sms : 148) / 2;
}

int launch_small(const Dims& d, const void* X, const void* W, const void* L_A, const void* L_B,
                 const Workspace& ws, void* Y, int* err, cudaStream_t stream) {
    const bool lora = d.R_pad == 64 && L_A && L_B;
    CUtensorMap tmX, tmLB, tmW, tmLA, tmY, tmY16, tmVals, tmT;
    int rc = encode_tmap_bf16_2d(&tmX, X, d.K, d.M, d.K * 2, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    rc = encode_tmap_bf16_2d(&tmW, W, d.K, d.N, d.K * 2, 64, kSmallBN / 2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    if (lora) {
        rc = encode_tmap_bf16_2d(&tmLB, L_B, d.K, d.R, d.K * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        rc = encode_tmap_bf16_2d(&tmLA, L_A, d.R, d.N, d.R * 2, 64, kSmallBN / 2, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    } else {
        tmLB = tmX;
        tmLA = tmW;
    }
    rc = encode_tmap_bf16_2d(&tmY, Y, d.N, d.M, d.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
    rc = encode_tmap_bf16_2d(&tmY16, Y, d.N, d.M, d.N * 2, 16, 32, CU_TENSOR_MAP_SWIZZLE_32B);
    if (rc) return rc;
    // the workspace copy of the kept values and of T (column tile 0)
    rc = encode_tmap_bf16_2d(&tmVals, ws.vals, d.Kc_pad, d.M_pad, d.Kc_pad * 2, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    if (lora) {
        rc = encode_tmap_bf16_2d(&tmT, ws.T, 64, d.M_pad, 128, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    } else {
        tmT = tmVals;
    }
    SmallArgs a;
    a.M = static_cast<int>(d.M);
    a.K = static_cast<int>(d.K);
    a.N = static_cast<int>(d.N);
    a.R_pad = lora ? 64 : 0;
    a.k_chunks = static_cast<int>(d.k_chunks);
    a.m_pairs = static_cast<int>(d.M_pad / (2 * kBM));
    a.n_tiles = static_cast<int>((d.N + kSmallBN - 1) / kSmallBN);
    a.lora = lora ? 1 : 0;
    a.vals = ws.vals;
    a.meta = ws.meta;
    a.s = ws.s;
    a.T = ws.T;
    a.Kc_pad = static_cast<int>(d.Kc_pad);
    a.err = err;
    static std::atomic<uint64_t> smem_set{0};
    rc = allow_max_dynamic_smem(rtlynx_small_kernel, smem_set);
    if (rc) return rc;
    return launch_dependent(rtlynx_small_kernel, dim3(2 * a.m_pairs * a.n_tiles), dim3(kSmallThreads), kSmallSmem,
                            stream, tmX, tmLB, tmW, tmLA, tmY, tmY16, tmVals, tmT, a);
}

}  // namespace rtlynx
