// The RT-Lynx sparsify prologue on sm_100a (RT-Lynx summary page, four-step
// pipeline paragraph, step 1 "Norm-Compensated Activation Sparsification" and
// step 4 items (1)-(3): mask decision, Top-K, compression to the sparse tensor
// core layout), plus the LoRA down-projection T = X L_B^T of step 2.
//
// Pass 1  sparsify_stream   persistent, one CTA per SM.
//         The (row block of 128 tokens) x (64-wide K tile) grid of X is cut
//         into equal contiguous runs, one per CTA.  A TMA producer streams the
//         CTA's tiles (and the matching 64-wide tiles of L_B) through a ring of
//         shared-memory stages.  Sixteen math warps rank every group of four
//         once: the 2-of-4 rule (integer magnitude compares, ties to the lower
//         index) gives the metadata nibble and the two kept entries, which are
//         written unscaled; the same ranking gives the exact squares for
//         sum(x^2) and sum(x~^2), accumulated in double (a tile holding zero
//         or subnormal entries takes a converting path, chosen per warp).  One thread issues
//         dense tcgen05.mma (M = 128, N = R) from the same shared-memory tiles
//         into one of two tensor-memory accumulators.  Where a run crosses a
//         row block, the partial norms and the partial T of the finished
//         segment go to the workspace.
// Pass 2  scale             eight tokens per CTA, one warp per token for the sums.
//         Sums each token's partial norms in segment order,
//         s = ||x|| / (||x~|| + 1e-8) in float, and sums the partial T in
//         segment order, rounded to bf16; then all threads of the CTA rescale
//         the kept entries in place (s*x rounded once to bf16, nearest even).
// FP8 mode (the layer's E4M3 form): pass 1 writes the metadata in the 8-bit
//         operand order (token m of a block at byte 16 m of a chunk, group g
//         at nibble g) and each segment's max |x| per token; pass 2 forms
//         q_x = s * max|x| / 448, stores T / q_x, and converts the kept
//         entries to E4M3 codes of x * (448 / max|x|) in a separate buffer
//         instead of rescaling them.
// Both passes and the GEMM launch as programmatic dependents: each one's setup
// overlaps the previous kernel's tail, and it touches memory only after the
// grid-dependency wait.
// Every reduction runs in a fixed order, so results are deterministic.
//
// Metadata chunk (128 tokens x 128 logical K, 2048 bytes), for token m in the
// row block (m0 = m % 8, m1 = (m / 8) % 2, m2 = m / 16) and logical k in the
// chunk (k0 = k % 16, k1 = (k / 16) % 2, k2 = k / 32):
//     tensor-memory lane dp = m0 + 8*k1 + 16*m2, column k2,
//     byte offset 16*dp + 4*k2, bit 16*m1 + 4*(k0 / 4) within that 32-bit word,
// and the nibble of a group is i0 | (i1 << 2) with i0 < i1 the kept indices.
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"
#include "sparsify_math.cuh"

namespace rtlynx {

constexpr int kStreamThreads = 576;  // warp 0 TMA, warp 1 MMA, warps 2-17 math
constexpr int kMathWarps = 16;
constexpr int kXTileBytes = kBM * kBK * 2;  // 16 KB

struct StreamArgs {
    int64_t M_pad, Kc_pad, total_tiles, grid;
    int kt2, k_chunks, R_pad, stages;
    uint16_t* vals;
    uint8_t* meta;
    double* part_norm;
    float* part_T;
    float* part_amax;  // FP8 form: [max_segs, M_pad] partial max |x|
    int* split_cnt;  // arrival tickets of the GEMM's split tiles, zeroed here for the GEMM that follows
    int n_split_cnt;
    int* err;
};

// Bytes of one ring stage: a 128 x 64 tile of X and, with LoRA, a R_pad x 64
// tile of L_B (both multiples of 1024, as the 128-byte swizzle wants).
__host__ __device__ inline int stream_stage_bytes(int R_pad) { return kXTileBytes + R_pad * kBK * 2; }

// Every lane of the warp waits; the warp goes on only if all of them saw the
// phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* err) {
    const bool ok = mbar_wait(bar, parity, err);
    return __all_sync(0xFFFFFFFFu, ok);
}

// stream_owner with a 32-bit division whenever the operands fit.
__device__ __forceinline__ int64_t stream_owner_dev(int64_t t, int64_t total, int64_t grid) {
    const uint64_t num = static_cast<uint64_t>(t + 1) * static_cast<uint64_t>(grid) - 1u;
    if (num < (1ull << 32) && static_cast<uint64_t>(total) < (1ull << 32))
        return static_cast<uint32_t>(num) / static_cast<uint32_t>(total);
    return static_cast<int64_t>(num / static_cast<uint64_t>(total));
}

// FP8: the metadata goes out in the 8-bit layout (token m of the block at
// byte 16 m of each chunk, group g of the chunk at nibble g), and each
// segment's max |x| per token goes to part_amax.
template <bool LORA, bool FP8>
__global__ void __launch_bounds__(kStreamThreads, 1)
    rtlynx_sparsify_stream_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmLB,
                                  const StreamArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.stages;
    const int stage_bytes = stream_stage_bytes(LORA ? a.R_pad : 0);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;  // [2] accumulator ready for draining
    uint64_t* tempty = tfull + 2; // [2] accumulator drained
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int* err = a.err;
    const int64_t cta = blockIdx.x;
    const int64_t t0 = stream_begin(cta, a.total_tiles, a.grid);
    const int64_t t1 = stream_begin(cta + 1, a.total_tiles, a.grid);
    const int64_t kt2 = a.kt2;
    uint32_t tmem_cols = 32;
    while (tmem_cols < static_cast<uint32_t>(2 * a.R_pad)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMathWarps + (LORA ? 1 : 0));
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(mma_done, 1);
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
    // Launched as a programmatic dependent: the setup above overlaps the tail
    // of whatever ran before in the stream (the previous layer's GEMM, say),
    // and nothing before this wait touches memory that kernel may still use.
    grid_dependency_wait();
    launch_dependents();  // the scale pass may be scheduled; it waits for this grid to finish
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.n_split_cnt; i += blockDim.x) a.split_cnt[i] = 0;

    // Role warps run their loops with all 32 lanes (waits by every lane, the
    // single-thread actions predicated on lane 0), so every warp reaches the
    // block-wide barriers converged.  Tile t is row block mb = t / kt2, K tile
    // kt = t % kt2; the loops step (mb, kt) without dividing.
    const int64_t mb0 = t0 / kt2;
    const int kt0 = static_cast<int>(t0 - mb0 * kt2);
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        int stage = 0, issued = 0;
        uint32_t phase = 0;
        int64_t mb = mb0;
        int kt = kt0;
        for (int64_t t = t0; t < t1; ++t) {
            if (!warp_wait(&empty[stage], phase ^ 1u, err)) break;
            if (lane == 0) {
                uint8_t* sX = smem + stage * stage_bytes;
                mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(stage_bytes));
                tma_load_2d(sX, &tmX, &full[stage], kt * kBK, static_cast<int>(mb * kBM));
                if (LORA) tma_load_2d(sX + kXTileBytes, &tmLB, &full[stage], kt * kBK, 0);
            }
            __syncwarp();
            ++issued;
            if (++stage == S) {
                stage = 0;
                phase ^= 1u;
            }
            if (++kt == a.kt2) {
                kt = 0;
                ++mb;
            }
        }
        // every issued copy has landed before the CTA may exit
        for (int q = issued > S ? issued - S : 0; q < issued; ++q)
            mbar_wait(&full[q % S], static_cast<uint32_t>((q / S) & 1), nullptr);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ LoRA-down MMA issuer
        if (LORA) {
            const uint32_t idesc = make_idesc_bf16(kBM, a.R_pad, false);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t n = 0;  // segments so far: accumulator n & 1, its use (n >> 1)
            bool ok = true;
            int64_t t = t0;
            int64_t seg_end = min(t1, (mb0 + 1) * kt2);
            while (ok && t < t1) {
                const uint32_t b = n & 1u;
                if (!warp_wait(&tempty[b], ((n >> 1) & 1u) ^ 1u, err)) break;
                tc_fence_after();
                const uint32_t acc = tmem_base + static_cast<uint32_t>(b * a.R_pad);
                for (bool first = true; t < seg_end; ++t, first = false) {
                    if (!warp_wait(&full[stage], phase, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t sX = smem_u32(smem + stage * stage_bytes);
                        const uint32_t sL = sX + kXTileBytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_f16(acc, make_sdesc(sX + j * 32, 16, 1024, kSw128),
                                    make_sdesc(sL + j * 32, 16, 1024, kSw128), idesc, !(first && j == 0));
                        tc_commit(&empty[stage]);
                    }
                    __syncwarp();
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) tc_commit(&tfull[b]);
                __syncwarp();
                ++n;
                seg_end = min(t1, seg_end + kt2);
            }
            if (lane == 0) tc_commit(mma_done);
            __syncwarp();
            mbar_wait(mma_done, 0, nullptr);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ math warps
        // Thread (row pair, 16-byte unit): rows rA = m0 + 16*m2 and rB = rA + 8
        // of the block, channels 8u .. 8u+7 of each 64-wide tile.  The eight
        // lanes of a quarter warp read the eight units of one row (no bank
        // conflict), and rows rA, rB fill the two halves of the same metadata
        // word.
        const int wi = threadIdx.x - 64;
        const int u = wi & 7, rp = wi >> 3;
        const int m0 = rp & 7, m2 = rp >> 3;
        const int rA = m0 + 16 * m2;
        const uint32_t offA = static_cast<uint32_t>(rA * 128 + ((u ^ m0) << 4));
        const uint32_t offB = offA + 8 * 128;
        const int dp = m0 + 8 * ((u >> 1) & 1) + 16 * m2;
        const bool even = (u & 1) == 0;
        const bool drain = LORA && warp >= 4 && warp < 8;  // warps reaching tensor-memory lanes 0-127
        int stage = 0;
        uint32_t phase = 0;
        uint32_t n = 0;  // segments so far (accumulator n & 1)
        int64_t t = t0;
        for (int64_t mb = mb0; t < t1; ++mb) {
            const int64_t seg_end = min(t1, (mb + 1) * kt2);
            const int64_t seg = cta - stream_owner_dev(mb * kt2, a.total_tiles, a.grid);
            const int64_t growA = mb * kBM + rA;
            uint16_t* vA = a.vals + growA * a.Kc_pad + u * 4;
            uint16_t* vB = vA + 8 * a.Kc_pad;
            uint8_t* mrow = a.meta + mb * a.k_chunks * kChunkBytes + dp * 16;
            double nxA = 0.0, ntA = 0.0, nxB = 0.0, ntB = 0.0;
            uint32_t mkA = 0u, mkB = 0u;  // FP8: the largest key of each token's entries in this segment
            uint8_t* mchunk8 = a.meta + mb * a.k_chunks * kChunkBytes;
            bool ok = true;
            for (int kt = static_cast<int>(t - mb * kt2); t < seg_end; ++t, ++kt) {
                if (!warp_wait(&full[stage], phase, err)) {
                    ok = false;
                    break;
                }
                const uint8_t* sX = smem + stage * stage_bytes;
                const uint4 xa = *reinterpret_cast<const uint4*>(sX + offA);
                const uint4 xb = *reinterpret_cast<const uint4*>(sX + offB);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
                // rank each group once: metadata, kept entries and the energies
                const GroupKeys g0 = rank_group(xa.x, xa.y), g1 = rank_group(xa.z, xa.w);
                const GroupKeys g2 = rank_group(xb.x, xb.y), g3 = rank_group(xb.z, xb.w);
                uint2 ka, kb;
                const uint32_t na = pick_kept(g0, xa.x, xa.y, ka.x) | (pick_kept(g1, xa.z, xa.w, ka.y) << 4);
                const uint32_t nb = pick_kept(g2, xb.x, xb.y, kb.x) | (pick_kept(g3, xb.z, xb.w, kb.y) << 4);
                const bool normal = group_all_normal(g0) && group_all_normal(g1) && group_all_normal(g2) &&
                                    group_all_normal(g3);
                if (__all_sync(0xFFFFFFFFu, normal)) {
                    group_energy_normal(g0, nxA, ntA);
                    group_energy_normal(g1, nxA, ntA);
                    group_energy_normal(g2, nxB, ntB);
                    group_energy_normal(g3, nxB, ntB);
                } else {  // zero or subnormal entries somewhere in the warp's tile (rare)
                    double2 e = group_energy_any(g0.k1, g0.k2, g0.k3, g0.k4);
                    nxA += e.x;
                    ntA += e.y;
                    e = group_energy_any(g1.k1, g1.k2, g1.k3, g1.k4);
                    nxA += e.x;
                    ntA += e.y;
                    e = group_energy_any(g2.k1, g2.k2, g2.k3, g2.k4);
                    nxB += e.x;
                    ntB += e.y;
                    e = group_energy_any(g3.k1, g3.k2, g3.k3, g3.k4);
                    nxB += e.x;
                    ntB += e.y;
                }
                *reinterpret_cast<uint2*>(vA + kt * 32) = ka;
                *reinterpret_cast<uint2*>(vB + kt * 32) = kb;
                if constexpr (FP8) {
                    mkA = max(mkA, max(g0.k1, g1.k1));
                    mkB = max(mkB, max(g2.k1, g3.k1));
                    // one byte (groups 2u and 2u + 1 of this 64-wide tile) per token
                    uint8_t* c8 = mchunk8 + (kt >> 1) * kChunkBytes + (kt & 1) * 8 + u;
                    c8[16 * rA] = static_cast<uint8_t>(na);
                    c8[16 * (rA + 8)] = static_cast<uint8_t>(nb);
                } else {
                    // metadata word: bytes (rA, u even), (rA, u odd), (rB, u even), (rB, u odd)
                    const uint32_t mine = na | (nb << 8);
                    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, mine, 1);
                    if (even)
                        *reinterpret_cast<uint32_t*>(mrow + (kt >> 1) * kChunkBytes + (2 * (kt & 1) + (u >> 2)) * 4) =
                            __byte_perm(mine, other, 0x5140);
                }
            }
            if (!ok) break;
            // the token's totals over the eight units, in a fixed order
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                nxA += __shfl_xor_sync(0xFFFFFFFFu, nxA, o);
                ntA += __shfl_xor_sync(0xFFFFFFFFu, ntA, o);
                nxB += __shfl_xor_sync(0xFFFFFFFFu, nxB, o);
                ntB += __shfl_xor_sync(0xFFFFFFFFu, ntB, o);
            }
            if constexpr (FP8) {
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    mkA = max(mkA, __shfl_xor_sync(0xFFFFFFFFu, mkA, o));
                    mkB = max(mkB, __shfl_xor_sync(0xFFFFFFFFu, mkB, o));
                }
                if (u == 0) {  // the key's high half is the bf16 magnitude: as a float, |x| exactly
                    a.part_amax[seg * a.M_pad + growA] = __uint_as_float(mkA & 0x7FFF0000u);
                    a.part_amax[seg * a.M_pad + growA + 8] = __uint_as_float(mkB & 0x7FFF0000u);
                }
            }
            if (u == 0) {
                double* pn = a.part_norm + (seg * a.M_pad + growA) * 2;
                pn[0] = nxA;
                pn[1] = ntA;
                pn[16] = nxB;  // row rB = rA + 8
                pn[17] = ntB;
            }
            if (drain) {
                const uint32_t b = n & 1u;
                if (!warp_wait(&tfull[b], (n >> 1) & 1u, err)) break;
                tc_fence_after();
                const int q = warp & 3;
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * a.R_pad);
                float* pt = a.part_T + (seg * a.M_pad + mb * kBM + q * 32 + lane) * a.R_pad;
                for (int c = 0; c < a.R_pad; c += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        *reinterpret_cast<float4*>(pt + c + 4 * q4) =
                            make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                        __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[b]);
            }
            ++n;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (LORA && warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

// ---------------------------------------------------------------- pass 2
struct ScaleArgs {
    int64_t M_pad, Kc_pad, total_tiles, grid;
    int64_t trigger_from;  // CTAs from this index on (the last wave) let the GEMM launch
    int kt2, R_pad;
    const double* part_norm;
    const float* part_T;
    uint16_t* vals;
    float* s_out;
    uint16_t* T;
    // FP8 form
    const float* part_amax;
    uint8_t* codes;
    float* qx;
};

// Eight tokens per CTA (all in one row block, so they share the segment
// split).  Every global load the CTA needs is issued before anything waits
// on one: the CTA's kept values (one contiguous span of 8 rows), each warp's
// token's partial norms (one segment per lane) and partial T (up to four
// segments at a time).  Warp w then forms token w's s and T; after one CTA
// barrier all 256 threads rescale the span.
// FP8: instead of the in-place rescale, the kept entries become E4M3 codes of
// x * (448 / max|x|) (float32 product, nearest even, saturating), the token's
// dequantisation scale q_x = s * max|x| / 448 is stored, and T is stored as
// T / q_x (the GEMM multiplies its accumulator by q_x q_w).
template <bool FP8>
__global__ void __launch_bounds__(256, 4) rtlynx_scale_kernel(const ScaleArgs a) {
    constexpr int kRows = 8;  // tokens per CTA
    constexpr int kU = 8;     // 16-byte value vectors in flight per thread
    constexpr int kSegU = 4;  // partial-T segments loaded at once
    __shared__ float s_sh[kRows];  // s, or with FP8 the code scale 448 / max|x|
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRows;  // M_pad is a multiple of kRows
    const int64_t row = row0 + w;
    const int64_t first = (row0 / kBM) * a.kt2;
    grid_dependency_wait();  // everything pass 1 wrote is visible from here on
    // Only the last wave lets the GEMM launch (the CTAs before it count once
    // they exit): a GEMM CTA placed on an SM early would halve the room for
    // the scale pass's later waves there.
    if (static_cast<int64_t>(blockIdx.x) >= a.trigger_from) launch_dependents();
    const int64_t c0 = stream_owner_dev(first, a.total_tiles, a.grid);
    const int nseg = static_cast<int>(stream_owner_dev(first + a.kt2 - 1, a.total_tiles, a.grid) - c0 + 1);
    uint4* v = reinterpret_cast<uint4*>(a.vals + row0 * a.Kc_pad);
    const int n16 = static_cast<int>(a.Kc_pad / 8);
    const int total = kRows * n16;
    uint4 q[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u)
        if (static_cast<int>(threadIdx.x) + 256 * u < total) q[u] = v[threadIdx.x + 256 * u];
    double2 part = make_double2(0.0, 0.0);
    if (lane < nseg) part = *reinterpret_cast<const double2*>(a.part_norm + (lane * a.M_pad + row) * 2);
    float amax = 0.0f, inv_q = 1.0f, code_scale = 0.0f;
    if constexpr (FP8) {
        for (int j = lane; j < nseg; j += 32) amax = fmaxf(amax, a.part_amax[j * a.M_pad + row]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        // s first: q_x needs it before T is stored
        double nx = 0.0, nt = 0.0;
        for (int j0 = 0; j0 < nseg; j0 += 32) {
            double2 p2 = part;
            if (j0 > 0) {
                p2 = make_double2(0.0, 0.0);
                if (j0 + lane < nseg)
                    p2 = *reinterpret_cast<const double2*>(a.part_norm + ((j0 + lane) * a.M_pad + row) * 2);
            }
            const int m = nseg - j0 < 32 ? nseg - j0 : 32;
            for (int j = 0; j < m; ++j) {
                nx += __shfl_sync(0xFFFFFFFFu, p2.x, j);
                nt += __shfl_sync(0xFFFFFFFFu, p2.y, j);
            }
        }
        const float s = static_cast<float>(sqrt(nx) / (sqrt(nt) + 1e-8));
        const float q = __fdiv_rn(__fmul_rn(s, amax), 448.0f);
        inv_q = q > 0.0f ? __fdiv_rn(1.0f, q) : 0.0f;
        code_scale = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
        if (lane == 0) {
            s_sh[w] = code_scale;
            a.s_out[row] = s;
            a.qx[row] = q;
        }
    }
    // T: partial sums in segment order, rounded once to bf16 (with FP8, T / q_x)
    for (int c = 2 * lane; c < a.R_pad; c += 64) {
        float t0 = 0.f, t1 = 0.f;
        for (int j0 = 0; j0 < nseg; j0 += kSegU) {
            float2 p[kSegU];
#pragma unroll
            for (int j = 0; j < kSegU; ++j)
                if (j0 + j < nseg)
                    p[j] = *reinterpret_cast<const float2*>(a.part_T + ((j0 + j) * a.M_pad + row) * a.R_pad + c);
#pragma unroll
            for (int j = 0; j < kSegU; ++j) {
                if (j0 + j < nseg) {
                    t0 += p[j].x;
                    t1 += p[j].y;
                }
            }
        }
        if (FP8) {
            t0 *= inv_q;
            t1 *= inv_q;
        }
        *reinterpret_cast<__nv_bfloat162*>(a.T + row * a.R_pad + c) = __floats2bfloat162_rn(t0, t1);
    }
    if constexpr (FP8) {
        __syncthreads();
        // codes of the CTA's span: 8 kept entries (one 16-byte vector) -> 8 bytes
        uint2* out = reinterpret_cast<uint2*>(a.codes + row0 * a.Kc_pad);
        for (int i0 = static_cast<int>(threadIdx.x);;) {
            int r0 = i0 / n16;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int idx = i0 + 256 * u;
                while (r0 < kRows - 1 && idx >= (r0 + 1) * n16) ++r0;
                if (idx < total) {
                    const float cs = s_sh[r0];
                    const uint32_t wv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
                    uint32_t pk[2] = {0u, 0u};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float lo = __fmul_rn(__uint_as_float(wv[h] << 16), cs);
                        const float hi = __fmul_rn(__uint_as_float(wv[h] & 0xFFFF0000u), cs);
                        const uint32_t c2 = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
                        pk[h >> 1] |= c2 << (16 * (h & 1));
                    }
                    out[idx] = make_uint2(pk[0], pk[1]);
                }
            }
            i0 += 256 * kU;
            if (i0 >= total) break;
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (i0 + 256 * u < total) q[u] = v[i0 + 256 * u];
        }
        return;
    }
    // partial norms, one segment per lane, added in segment order (every lane
    // forms the same s)
    double nx = 0.0, nt = 0.0;
    for (int j0 = 0; j0 < nseg; j0 += 32) {
        if (j0 > 0) {
            part = make_double2(0.0, 0.0);
            if (j0 + lane < nseg)
                part = *reinterpret_cast<const double2*>(a.part_norm + ((j0 + lane) * a.M_pad + row) * 2);
        }
        const int m = nseg - j0 < 32 ? nseg - j0 : 32;
        for (int j = 0; j < m; ++j) {
            nx += __shfl_sync(0xFFFFFFFFu, part.x, j);
            nt += __shfl_sync(0xFFFFFFFFu, part.y, j);
        }
    }
    const float s = static_cast<float>(sqrt(nx) / (sqrt(nt) + 1e-8));
    if (lane == 0) {
        s_sh[w] = s;
        a.s_out[row] = s;
    }
    __syncthreads();
    for (int i0 = static_cast<int>(threadIdx.x);;) {
        int r0 = i0 / n16;  // row of the first vector of this round; later ones step it
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int idx = i0 + 256 * u;
            while (r0 < kRows - 1 && idx >= (r0 + 1) * n16) ++r0;
            if (idx < total) {
                const float sr = s_sh[r0];
                q[u].x = scale_pair(sr, q[u].x);
                q[u].y = scale_pair(sr, q[u].y);
                q[u].z = scale_pair(sr, q[u].z);
                q[u].w = scale_pair(sr, q[u].w);
                v[idx] = q[u];
            }
        }
        i0 += 256 * kU;
        if (i0 >= total) break;
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (i0 + 256 * u < total) q[u] = v[i0 + 256 * u];
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
int launch_sparsify(const Dims& d, const void* X, const void* L_B, const Workspace& ws, int* err,
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
    StreamArgs a;
    a.part_amax = ws.part_amax;
    a.M_pad = d.M_pad;
    a.Kc_pad = d.Kc_pad;
    a.total_tiles = d.m_blocks * d.kt2;
    a.grid = d.grid1;
    a.kt2 = static_cast<int>(d.kt2);
    a.k_chunks = static_cast<int>(d.k_chunks);
    a.R_pad = lora ? static_cast<int>(d.R_pad) : 0;
    const int stage_bytes = stream_stage_bytes(a.R_pad);
    a.stages = 200 * 1024 / stage_bytes < 6 ? 200 * 1024 / stage_bytes : 6;
    a.vals = ws.vals;
    a.meta = ws.meta;
    a.part_norm = ws.part_norm;
    a.part_T = ws.part_T;
    a.split_cnt = ws.split_cnt;
    a.n_split_cnt = static_cast<int>(2 * (d.gemm_tiles - d.tail_full));
    a.err = err;
    const int smem = a.stages * stage_bytes + 256 + 1024;
    const dim3 grid(static_cast<unsigned>(d.grid1));
    cudaError_t e;
    static std::atomic<uint64_t> smem_set[4];
    auto kernel = d.fp8 ? (lora ? rtlynx_sparsify_stream_kernel<true, true> : rtlynx_sparsify_stream_kernel<false, true>)
                        : (lora ? rtlynx_sparsify_stream_kernel<true, false> : rtlynx_sparsify_stream_kernel<false, false>);
    const int rc2 = allow_max_dynamic_smem(kernel, smem_set[(lora ? 1 : 0) + (d.fp8 ? 2 : 0)]);
    if (rc2) return rc2;
    e = static_cast<cudaError_t>(launch_dependent(kernel, grid, dim3(kStreamThreads), smem, stream, tmX, tmLB, a));
    if (e != cudaSuccess) return e;

    ScaleArgs b;
    b.M_pad = d.M_pad;
    {
        const int64_t ctas = d.M_pad / 8, wave = 4 * d.grid1;  // four scale CTAs fit on an SM
        b.trigger_from = ctas > wave ? ctas - wave : 0;
    }
    b.Kc_pad = d.Kc_pad;
    b.total_tiles = a.total_tiles;
    b.grid = d.grid1;
    b.kt2 = a.kt2;
    b.R_pad = a.R_pad;
    b.part_norm = ws.part_norm;
    b.part_T = ws.part_T;
    b.vals = ws.vals;
    b.s_out = ws.s;
    b.T = ws.T;
    b.part_amax = ws.part_amax;
    b.codes = ws.codes;
    b.qx = ws.qx;
    return launch_dependent(d.fp8 ? rtlynx_scale_kernel<true> : rtlynx_scale_kernel<false>, dim3(static_cast<unsigned>(d.M_pad / 8)), dim3(256), 0, stream, b);
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
