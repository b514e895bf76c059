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
constexpr int kCThreads = 256;
constexpr int kXTile = kRB * 128;         // one 64 x 64 bf16 tile (128 B rows): 8 KB
constexpr int kMaxTiles = 64;

struct ClusterArgs {
    int M, K;
    int64_t M_pad, Kc_pad;
    int k_chunks, chunks_per_cta, R_pad;
    uint16_t* vals;
    uint8_t* meta;
    float* s_out;
    uint16_t* T;
    int* err;
};

// Shared-memory bytes the kernel needs for a given split.
__host__ __device__ inline int cluster_smem_bytes(int chunks_per_cta, int R_pad) {
    const int x = 2 * chunks_per_cta * kXTile;
    const int lb = R_pad > 0 ? 2 * R_pad * 128 : 0;
    // the T MMA reads 128 rows from the last 64-row X tile: keep 8 KB after it
    const int tail = (R_pad > 0 && lb < kXTile) ? kXTile - lb : 0;
    int tpart = kRB * R_pad * 4;
    int body = x + lb + tail;
    if (tpart > body) body = tpart;
    return body + kRB * 16 + kRB * 4 + 1024 /*barriers*/ + 1024 /*align*/;
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
    uint8_t* sX = smem;
    uint8_t* sLB = smem + x_bytes;
    const int lb_bytes = 2 * lb_slot;
    const int tail = (LORA && lb_bytes < kXTile) ? kXTile - lb_bytes : 0;
    int body = x_bytes + lb_bytes + tail;
    if (kRB * a.R_pad * 4 > body) body = kRB * a.R_pad * 4;
    float* sTpart = reinterpret_cast<float*>(smem);  // reuses X / L_B after compression
    double* sPart = reinterpret_cast<double*>(smem + body);          // [kRB][2]
    float* sS = reinterpret_cast<float*>(smem + body + kRB * 16);     // [kRB]
    uint64_t* full_x = reinterpret_cast<uint64_t*>(smem + body + kRB * 16 + kRB * 4);
    uint64_t* full_lb = full_x + kMaxTiles;
    uint64_t* empty_lb = full_lb + 2;
    uint64_t* t_done = empty_lb + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(t_done + 1);

    uint32_t tmem_cols = 32;
    while (tmem_cols < static_cast<uint32_t>(a.R_pad)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < ntiles; ++i) mbar_init(&full_x[i], 1);
        mbar_init(&full_lb[0], 1);
        mbar_init(&full_lb[1], 1);
        mbar_init(&empty_lb[0], 1);
        mbar_init(&empty_lb[1], 1);
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
                const int slot = i & 1;
                if (!mbar_wait(&empty_lb[slot], ((i >> 1) & 1) ^ 1u, err)) break;
                mbar_arrive_expect_tx(&full_lb[slot], lb_slot);
                tma_load_2d(sLB + slot * lb_slot, &tmLB, &full_lb[slot], k_begin + i * 64, 0);
            }
        }
    } else if (LORA && warp == 1 && lane == 0) {
        const uint32_t idesc = make_idesc_bf16(128, a.R_pad, false);
        const uint64_t dX = make_sdesc(smem_u32(sX), 16, 1024, kSw128);
        const uint64_t dL = make_sdesc(smem_u32(sLB), 16, 1024, kSw128);
        for (int i = 0; i < ntiles; ++i) {
            const int slot = i & 1;
            if (!mbar_wait(&full_x[i], 0, err)) break;
            if (!mbar_wait(&full_lb[slot], (i >> 1) & 1, err)) break;
            tc_fence_after();
            const uint64_t ax = dX + static_cast<uint64_t>((i * kXTile) >> 4);
            const uint64_t bl = dL + static_cast<uint64_t>((slot * lb_slot) >> 4);
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_f16(tmem_base, ax + 2 * j, bl + 2 * j, idesc, (i | j) != 0);
            tc_commit(&empty_lb[slot]);
        }
        tc_commit(t_done);
    }

    // ---------------------------------------------------------------- partial norms (all threads)
    {
        const int r = threadIdx.x >> 2;  // token within the cluster's 64
        const int q = threadIdx.x & 3;   // quarter of each 64-wide tile row
        double nx = 0.0, nt = 0.0;
        for (int i = 0; i < ntiles; ++i) {
            uint32_t ok = 1;
            if (lane == 0) ok = mbar_wait(&full_x[i], 0, err) ? 1u : 0u;
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            const uint8_t* row = sX + i * kXTile + r * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 2 * q + h;
                const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
                group_energy(v.x, v.y, nx, nt);
                group_energy(v.z, v.w, nx, nt);
            }
        }
        // fixed-order combine of the four quarters of the row
        nx += __shfl_xor_sync(0xFFFFFFFFu, nx, 1);
        nt += __shfl_xor_sync(0xFFFFFFFFu, nt, 1);
        nx += __shfl_xor_sync(0xFFFFFFFFu, nx, 2);
        nt += __shfl_xor_sync(0xFFFFFFFFu, nt, 2);
        if (q == 0) {
            sPart[2 * r] = nx;
            sPart[2 * r + 1] = nt;
        }
    }
    cluster_sync();

    // ---------------------------------------------------------------- s, summed over the cluster in rank order
    if (threadIdx.x < kRB) {
        const uint32_t base = smem_u32(&sPart[2 * threadIdx.x]);
        double nx = 0.0, nt = 0.0;
        for (uint32_t j = 0; j < csize; ++j) {
            const uint32_t addr = mapa_shared(base, j);
            nx += ld_shared_cluster_f64(addr);
            nt += ld_shared_cluster_f64(addr + 8);
        }
        const float s = static_cast<float>(sqrt(nx) / (sqrt(nt) + 1e-8));
        sS[threadIdx.x] = s;
        if (rank == 0) a.s_out[row0 + threadIdx.x] = s;
    }
    __syncthreads();

    // ---------------------------------------------------------------- compress from shared memory
    {
        const int pieces = 4 * ntiles;  // 16-wide K pieces per token
        for (int idx = threadIdx.x; idx < kRB * pieces; idx += kCThreads) {
            const int r = idx / pieces;
            const int p = idx - r * pieces;
            const int tile = p >> 2, pp = p & 3;
            const uint8_t* row = sX + tile * kXTile + r * 128;
            const uint4 lo = *reinterpret_cast<const uint4*>(row + (((2 * pp) ^ (r & 7)) << 4));
            const uint4 hi = *reinterpret_cast<const uint4*>(row + (((2 * pp + 1) ^ (r & 7)) << 4));
            const float s = sS[r];
            uint4 out;
            uint32_t nib = compress_group(lo.x, lo.y, s, out.x);
            nib |= compress_group(lo.z, lo.w, s, out.y) << 4;
            nib |= compress_group(hi.x, hi.y, s, out.z) << 8;
            nib |= compress_group(hi.z, hi.w, s, out.w) << 12;
            const int64_t grow = row0 + r;
            const int64_t k = k_begin + p * 16;
            *reinterpret_cast<uint4*>(a.vals + grow * a.Kc_pad + (k >> 1)) = out;
            const int m = static_cast<int>(grow & 127);
            const int m0 = m & 7, m1 = (m >> 3) & 1, m2 = m >> 4;
            const int kk = static_cast<int>(k & 127);
            const int k2 = kk >> 5, k1 = (kk >> 4) & 1;
            const int dp = m0 + 8 * k1 + 16 * m2;
            uint16_t* w = reinterpret_cast<uint16_t*>(a.meta + ((grow >> 7) * a.k_chunks + (k >> 7)) * kChunkBytes +
                                                      dp * 16 + k2 * 4 + m1 * 2);
            *w = static_cast<uint16_t>(nib);
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
                for (int q = 0; q < 32; ++q) sTpart[r * a.R_pad + c + q] = have ? __uint_as_float(v[q]) : 0.0f;
            }
        }
        tc_fence_before();
        cluster_sync();
        const int cols = a.R_pad / static_cast<int>(csize);
        const int c0 = static_cast<int>(rank) * cols;
        for (int idx = threadIdx.x; idx < kRB * cols; idx += kCThreads) {
            const int r = idx / cols;
            const int c = c0 + (idx - r * cols);
            const uint32_t base = smem_u32(&sTpart[r * a.R_pad + c]);
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
int pick_cluster_split(const Dims& d, int num_sms, int* chunks_per_cta) {
    const int row_blocks = static_cast<int>(d.M_pad / kRB);
    auto fits = [&](int cs, int* cpc) {
        *cpc = static_cast<int>((d.k_chunks + cs - 1) / cs);
        if (2 * *cpc > kMaxTiles) return false;
        if (cluster_smem_bytes(*cpc, static_cast<int>(d.R_pad)) > 225 * 1024) return false;
        return d.R_pad == 0 || d.R_pad % cs == 0;
    };
    // portable cluster sizes first; 16 only when nothing smaller fits
    for (int cs = 1; cs <= 8; cs *= 2) {
        int cpc = 0;
        if (!fits(cs, &cpc)) continue;
        const bool enough = static_cast<int64_t>(cs) * row_blocks >= 2LL * num_sms;
        if (enough || cs >= d.k_chunks || cs == 8) {
            *chunks_per_cta = cpc;
            return cs;
        }
    }
    int cpc = 0;
    if (fits(16, &cpc)) {
        *chunks_per_cta = cpc;
        return 16;
    }
    return 0;
}

int launch_sparsify_cluster(const Dims& d, int cs, int chunks_per_cta, const void* X, const void* L_B,
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
    a.R_pad = lora ? static_cast<int>(d.R_pad) : 0;
    a.vals = ws.vals;
    a.meta = ws.meta;
    a.s_out = ws.s;
    a.T = ws.T;
    a.err = err;
    const int smem = cluster_smem_bytes(chunks_per_cta, a.R_pad);
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
