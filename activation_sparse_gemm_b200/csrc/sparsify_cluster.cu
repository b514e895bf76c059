// One-pass RT-Lynx sparsify prologue on sm_100a (RT-Lynx summary page,
// four-step pipeline paragraph, step 1 and step 4 items (1)-(3); the LoRA
// down-projection T = X L_B^T of step 2).
//
// A cluster of CS CTAs owns 64 tokens; CTA r of the cluster owns a contiguous
// range of 128-wide K chunks and keeps its whole 64 x K_r slice of X resident
// in shared memory (TMA, 128B swizzle), so X is read from HBM exactly once:
//   1. per token, sum(x^2) and sum of the two largest squares per group
//      (exact squares, double sums) over the CTA's slice;  one thread issues
//      dense tcgen05.mma for the partial T = X_r L_B,r^T from the same
//      shared-memory tiles (M = 128, of which lanes 0-63 are these tokens);
//   2. the partial norms are exchanged through distributed shared memory and
//      summed in rank order: s = ||x|| / (||x~|| + 1e-8), identical in every
//      CTA of the cluster;
//   3. every CTA compresses its slice straight from shared memory: exact 2-of-4
//      rule, s*x rounded once to bf16, values row-major, metadata nibbles in
//      tensor-memory order (see sparsify.cu for the mapping);
//   4. the partial T tiles are summed across the cluster through distributed
//      shared memory, each CTA producing a slice of the columns, and rounded
//      to bf16.
// Every reduction runs in a fixed order, so the results are deterministic.
#include "internal.h"
#include "ptx.cuh"
#include "sparsify_math.cuh"

namespace rtlynx {

constexpr int kRB = 64;                   // tokens per cluster
constexpr int kCThreads = 576;             // 2 role warps + 16 worker warps
constexpr int kXTile = kRB * 128;         // one 64 x 64 bf16 tile (128 B rows): 8 KB
constexpr int kMaxTiles = 64;

struct ClusterArgs {
    int M, K;
    int64_t M_pad, Kc_pad;
    int k_chunks, chunks_per_cta, R_pad;
    int lb_slots;  // L_B tiles resident at once (the whole slice when it fits)
    uint16_t* vals;
    uint8_t* meta;
    float* s_out;
    uint16_t* T;
    int* err;
};

// Shared-memory bytes the kernel needs for a given split and L_B ring.
__host__ __device__ inline int cluster_body_bytes(int chunks_per_cta, int R_pad, int lb_slots) {
    const int x = 2 * chunks_per_cta * kXTile;
    const int lb = R_pad > 0 ? lb_slots * R_pad * 128 : 0;
    // the T MMA reads 128 rows from the last 64-row X tile: keep 8 KB after it
    const int tail = (R_pad > 0 && lb < kXTile) ? kXTile - lb : 0;
    const int tpart = kRB * (R_pad + 1) * 4;
    const int body = x + lb + tail;
    return tpart > body ? tpart : body;
}

__host__ __device__ inline int cluster_smem_bytes(int chunks_per_cta, int R_pad, int lb_slots) {
    return cluster_body_bytes(chunks_per_cta, R_pad, lb_slots) + kRB * 16 + kRB * 4 + 2048 /*barriers*/ +
           1024 /*align*/;
}

template <bool LORA>
__global__ void __launch_bounds__(kCThreads, 1)
    rtlynx_sparsify_cluster_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmLB,
                                   const ClusterArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t csize = cluster_nctarank();
    const int row0 = blockIdx.y * kRB;

    const int c_begin = static_cast<int>(rank) * a.chunks_per_cta;
    const int c_end = min(c_begin + a.chunks_per_cta, a.k_chunks);
    const int ntiles = c_end > c_begin ? 2 * (c_end - c_begin) : 0;
    const int k_begin = c_begin * kChunkK;

    const int x_bytes = 2 * a.chunks_per_cta * kXTile;
    const int lb_slot = LORA ? a.R_pad * 128 : 0;
    const int LBS = a.lb_slots;
    uint8_t* sX = smem;
    uint8_t* sLB = smem + x_bytes;
    const int body = cluster_body_bytes(a.chunks_per_cta, LORA ? a.R_pad : 0, LBS);
    float* sTpart = reinterpret_cast<float*>(smem);  // reuses X / L_B after compression
    double* sPart = reinterpret_cast<double*>(smem + body);          // [kRB][2]
    float* sS = reinterpret_cast<float*>(smem + body + kRB * 16);     // [kRB]
    uint64_t* full_x = reinterpret_cast<uint64_t*>(smem + body + kRB * 16 + kRB * 4);
    uint64_t* full_lb = full_x + kMaxTiles;
    uint64_t* empty_lb = full_lb + kMaxTiles;
    uint64_t* t_done = empty_lb + kMaxTiles;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(t_done + 1);

    uint32_t tmem_cols = 32;
    while (tmem_cols < static_cast<uint32_t>(a.R_pad)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < ntiles; ++i) mbar_init(&full_x[i], 1);
        for (int i = 0; i < LBS; ++i) {
            mbar_init(&full_lb[i], 1);
            mbar_init(&empty_lb[i], 1);
        }
        mbar_init(t_done, 1);
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
    int* err = a.err;

    // ---------------------------------------------------------------- loads and T MMAs
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < ntiles; ++i) {
            mbar_arrive_expect_tx(&full_x[i], kXTile);
            tma_load_2d(sX + i * kXTile, &tmX, &full_x[i], k_begin + i * 64, row0);
        }
        if (LORA) {
            for (int i = 0; i < ntiles; ++i) {
                const int slot = i % LBS, pass = i / LBS;
                if (!mbar_wait(&empty_lb[slot], (pass & 1) ^ 1u, err)) break;
                mbar_arrive_expect_tx(&full_lb[slot], lb_slot);
                tma_load_2d(sLB + slot * lb_slot, &tmLB, &full_lb[slot], k_begin + i * 64, 0);
            }
        }
    } else if (LORA && warp == 1 && lane == 0) {
        const uint32_t idesc = make_idesc_bf16(128, a.R_pad, false);
        const uint64_t dX = make_sdesc(smem_u32(sX), 16, 1024, kSw128);
        const uint64_t dL = make_sdesc(smem_u32(sLB), 16, 1024, kSw128);
        for (int i = 0; i < ntiles; ++i) {
            const int slot = i % LBS, pass = i / LBS;
            if (!mbar_wait(&full_x[i], 0, err)) break;
            if (!mbar_wait(&full_lb[slot], pass & 1, err)) break;
            tc_fence_after();
            const uint64_t ax = dX + static_cast<uint64_t>((i * kXTile) >> 4);
            const uint64_t bl = dL + static_cast<uint64_t>((slot * lb_slot) >> 4);
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_f16(tmem_base, ax + 2 * j, bl + 2 * j, idesc, (i | j) != 0);
            tc_commit(&empty_lb[slot]);
        }
        tc_commit(t_done);
    }
    __syncwarp();  // reconverge the role warps before any block-wide barrier

    // ---------------------------------------------------------------- partial norms (worker warps 2..17)
    // worker w handles token r = w / 8 and the 16-byte unit u = w % 8 of each
    // 128-byte tile row (two groups of four channels per tile)
    const int wr = (threadIdx.x - 64) >> 3;
    const int wu = (threadIdx.x - 64) & 7;
    const uint32_t unit_off = static_cast<uint32_t>(wr * 128 + ((wu ^ (wr & 7)) << 4));
    if (warp >= 2) {
        double nx = 0.0, nt = 0.0;
        for (int i = 0; i < ntiles; ++i) {
            uint32_t ok = 1;
            if (lane == 0) ok = mbar_wait(&full_x[i], 0, err) ? 1u : 0u;
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            const uint4 v = *reinterpret_cast<const uint4*>(sX + i * kXTile + unit_off);
            group_energy(v.x, v.y, nx, nt);
            group_energy(v.z, v.w, nx, nt);
        }
        // fixed-order combine of the eight units of the token (every lane ends with the same sums)
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            nx += __shfl_xor_sync(0xFFFFFFFFu, nx, o);
            nt += __shfl_xor_sync(0xFFFFFFFFu, nt, o);
        }
        if (wu == 0) {
            sPart[2 * wr] = nx;
            sPart[2 * wr + 1] = nt;
        }
    }
    cluster_sync();

    // ---------------------------------------------------------------- s, summed over the cluster in rank order
    if (threadIdx.x >= 64 && threadIdx.x < 64 + kRB) {
        const int r = threadIdx.x - 64;
        const uint32_t base = smem_u32(&sPart[2 * r]);
        double nx = 0.0, nt = 0.0;
        for (uint32_t j = 0; j < csize; ++j) {
            const uint32_t addr = mapa_shared(base, j);
            nx += ld_shared_cluster_f64(addr);
            nt += ld_shared_cluster_f64(addr + 8);
        }
        const float s = static_cast<float>(sqrt(nx) / (sqrt(nt) + 1e-8));
        sS[r] = s;
        if (rank == 0) a.s_out[row0 + r] = s;
    }
    __syncthreads();

    // ---------------------------------------------------------------- compress from shared memory
    if (warp >= 2) {
        const float s = sS[wr];
        const int64_t grow = row0 + wr;
        // metadata: token m of its 128-token block, 8 channels per unit = two nibbles = one byte
        const int m = static_cast<int>(grow & 127);
        const int m0 = m & 7, m1 = (m >> 3) & 1, m2 = m >> 4;
        uint8_t* meta_blk = a.meta + (grow >> 7) * a.k_chunks * kChunkBytes;
        uint2* vrow = reinterpret_cast<uint2*>(a.vals + grow * a.Kc_pad + (k_begin >> 1));
        for (int i = 0; i < ntiles; ++i) {
            const uint4 v = *reinterpret_cast<const uint4*>(sX + i * kXTile + unit_off);
            uint2 out;
            uint32_t nib = compress_group(v.x, v.y, s, out.x);
            nib |= compress_group(v.z, v.w, s, out.y) << 4;
            vrow[i * 8 + wu] = out;  // 4 kept values of channels k_begin + 64 i + 8 wu ...
            const int k = k_begin + i * 64 + wu * 8;  // first channel of the unit
            const int kk = k & 127;
            const int dp = m0 + 8 * ((kk >> 4) & 1) + 16 * m2;
            meta_blk[(k >> 7) * kChunkBytes + dp * 16 + (kk >> 5) * 4 + m1 * 2 + ((kk >> 3) & 1)] =
                static_cast<uint8_t>(nib);
        }
    }

    // ---------------------------------------------------------------- T: partials through distributed shared memory
    if (LORA) {
        bool have = ntiles > 0;
        if (have && warp < 2) {
            uint32_t ok = 1;
            if (lane == 0) ok = mbar_wait(t_done, 0, err) ? 1u : 0u;
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            have = ok != 0;
        }
        tc_fence_after();
        __syncthreads();  // every thread is done with X in shared memory
        if (warp < 2) {
            // warps 0 and 1 own tensor-memory lanes 0-63 = the cluster's tokens
            const int r = warp * 32 + lane;
            const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
            for (int c = 0; c < a.R_pad; c += 32) {
                uint32_t v[32];
                if (ntiles > 0) {
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(c), v);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) sTpart[r * (a.R_pad + 1) + c + q] = have ? __uint_as_float(v[q]) : 0.0f;
            }
        }
        tc_fence_before();
        cluster_sync();
        const int cols = a.R_pad / static_cast<int>(csize);
        const int c0 = static_cast<int>(rank) * cols;
        for (int idx = threadIdx.x; idx < kRB * cols; idx += kCThreads) {
            const int r = idx / cols;
            const int c = c0 + (idx - r * cols);
            const uint32_t base = smem_u32(&sTpart[r * (a.R_pad + 1) + c]);
            float acc = 0.f;
            for (uint32_t j = 0; j < csize; ++j) acc += ld_shared_cluster_f32(mapa_shared(base, j));
            a.T[(row0 + r) * static_cast<int64_t>(a.R_pad) + c] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
        }
    }
    // no CTA leaves while a peer may still read its shared memory
    cluster_sync();
    if (LORA && warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

// Picks the cluster split: the smallest power-of-two number of CTAs per 64
// tokens whose slice fits in shared memory and that puts at least two CTAs
// on every SM.  Returns 0 when no split fits (callers use the two-pass path).
int pick_cluster_split(const Dims& d, int num_sms, int* chunks_per_cta, int* lb_slots) {
    const int row_blocks = static_cast<int>(d.M_pad / kRB);
    const int R_pad = static_cast<int>(d.R_pad);
    constexpr int kBudget = 220 * 1024;
    // Largest L_B ring (up to the whole slice) that fits next to the X slice.
    auto fit = [&](int cs, int* cpc, int* lbs) {
        *cpc = static_cast<int>((d.k_chunks + cs - 1) / cs);
        if (2 * *cpc > kMaxTiles) return false;
        if (R_pad > 0 && R_pad % cs != 0) return false;
        if (R_pad == 0) {
            *lbs = 1;
            return cluster_smem_bytes(*cpc, 0, 1) <= kBudget;
        }
        for (int l = 2 * *cpc; l >= 2; --l) {
            if (cluster_smem_bytes(*cpc, R_pad, l) <= kBudget) {
                *lbs = l;
                return true;
            }
        }
        return false;
    };
    int best = 0;
    for (int pass = 0; pass < 2 && !best; ++pass) {
        for (int cs = 1; cs <= 16; cs *= 2) {
            int cpc = 0, lbs = 0;
            if (!fit(cs, &cpc, &lbs)) continue;
            if (pass == 0 && R_pad > 0 && lbs < 2 * cpc) continue;  // first try: whole L_B slice resident
            const bool enough = static_cast<int64_t>(cs) * row_blocks >= 2LL * num_sms;
            if (enough || cs >= d.k_chunks || cs == 16) {
                *chunks_per_cta = cpc;
                *lb_slots = lbs;
                best = cs;
                break;
            }
        }
    }
    return best;
}

int launch_sparsify_cluster(const Dims& d, int cs, int chunks_per_cta, int lb_slots, const void* X, const void* L_B,
                            const Workspace& ws, int* err, cudaStream_t stream) {
    const bool lora = d.R > 0 && L_B != nullptr;
    CUtensorMap tmX, tmLB;
    int rc = encode_tmap_bf16_2d(&tmX, X, d.K, d.M, d.K * 2, 64, kRB, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    if (lora) {
        rc = encode_tmap_bf16_2d(&tmLB, L_B, d.K, d.R, d.K * 2, 64, static_cast<uint32_t>(d.R_pad),
                                 CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    } else {
        tmLB = tmX;
    }
    ClusterArgs a;
    a.M = static_cast<int>(d.M);
    a.K = static_cast<int>(d.K);
    a.M_pad = d.M_pad;
    a.Kc_pad = d.Kc_pad;
    a.k_chunks = static_cast<int>(d.k_chunks);
    a.chunks_per_cta = chunks_per_cta;
    a.lb_slots = lb_slots;
    a.R_pad = lora ? static_cast<int>(d.R_pad) : 0;
    a.vals = ws.vals;
    a.meta = ws.meta;
    a.s_out = ws.s;
    a.T = ws.T;
    a.err = err;
    const int smem = cluster_smem_bytes(chunks_per_cta, a.R_pad, lb_slots);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cs), static_cast<unsigned>(d.M_pad / kRB), 1);
    cfg.blockDim = dim3(kCThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (lora) {
        auto k = rtlynx_sparsify_cluster_kernel<true>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess && cs > 8) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k, tmX, tmLB, a);
    } else {
        auto k = rtlynx_sparsify_cluster_kernel<false>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess && cs > 8) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k, tmX, tmLB, a);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace rtlynx
