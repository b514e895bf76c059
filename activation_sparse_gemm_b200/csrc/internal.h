// Declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace rtlynx {

// Tile geometry shared by the prologue and the GEMM.
constexpr int kBM = 128;          // rows (tokens) per tile
constexpr int kBK = 64;           // logical K per pipeline stage
constexpr int kChunkK = 128;      // logical K per metadata chunk (4 sparse MMAs of K = 32)
constexpr int kChunkBytes = 2048; // 128 lanes x 16 bytes of metadata per chunk
constexpr int kPairBN = 240;      // output columns per sparse GEMM tile (one CTA pair)
constexpr int kDenseBN = 256;     // output columns per dense-skip GEMM tile
// FP8 (E4M3) sparse tiles: the f8f6f4 sparse MMA of a CTA pair wants N a
// multiple of 32, and two accumulators plus eight metadata columns must fit
// in 512; a stage carries 256 logical K (the same bytes as a bf16 stage).
constexpr int kFp8BN = 224;
constexpr int kFp8StageK = 256;
// fp32 partial of one CTA's 128 x 240 tile: [32-column chunk 8][4-column group 8][row 128][4]
constexpr int kSplitSlotFloats = 8 * kBM * 32;
constexpr int kMaxSplit = 6;  // parts of one split tile (the fix-up holds two chunks of the others in shared memory)

// Sizes derived from one problem.
struct Dims {
    int64_t M, K, N, R;
    int64_t M_pad;        // M rounded up to 2 * kBM (one CTA pair of the GEMM)
    int64_t m_blocks;     // M_pad / kBM
    int64_t k_tiles;      // ceil(K / kBK)
    int64_t k_chunks;     // ceil(K / kChunkK)
    int64_t Kc_pad;       // compressed row length in elements = k_chunks * kChunkK / 2
    int64_t R_pad;        // R rounded up to 64 (0 when R == 0)
    int64_t kt2;          // 64-wide K tiles per row block in the prologue = 2 * k_chunks
    int64_t grid1;        // CTAs of the streaming prologue pass
    int64_t max_segs;     // most CTAs whose tile runs meet one row block (partial-sum slots)
    // Sparse GEMM schedule: `gemm_pairs` persistent CTA pairs take the first
    // `tail_full` tiles round-robin; each of the remaining tiles is cut along K
    // into `tail_split` parts, one per pair (`tail_units` parts in all).
    int64_t gemm_pairs, gemm_tiles, tail_full, tail_split, tail_units;
    bool fp8;             // the FP8 form: E4M3 codes, 224-wide tiles, 256-K stages
};

// The streaming prologue cuts the m_blocks * kt2 tiles into `grid` contiguous
// runs: CTA c takes tiles [stream_begin(c), stream_begin(c + 1)), and tile t
// belongs to CTA stream_owner(t).
__host__ __device__ inline int64_t stream_begin(int64_t c, int64_t total, int64_t grid) { return c * total / grid; }
__host__ __device__ inline int64_t stream_owner(int64_t t, int64_t total, int64_t grid) {
    return ((t + 1) * grid - 1) / total;
}

// Byte offsets of the sparse-mode workspace regions (each 256-byte aligned).
struct WsLayout {
    size_t vals, meta, s, T, part_norm, part_T, split_part, split_cnt;
    size_t codes, qx, part_amax;  // FP8 form only (empty otherwise)
    size_t total;
};

// Main-loop and LoRA stages of one sparse GEMM tile (the split of the last
// wave and the kernel's schedule use the same counts): a bf16 stage covers
// one 128-wide metadata chunk, an FP8 stage two; a LoRA-up stage 64 of R.
inline int64_t sparse_k_stages(const Dims& d) { return d.fp8 ? d.k_chunks / 2 : d.k_chunks; }
inline int64_t sparse_lora_stages(const Dims& d) { return d.R_pad / 64; }

Dims make_dims(int64_t M, int64_t K, int64_t N, int64_t R, int num_sms, bool fp8 = false);
WsLayout make_ws_layout(const Dims& d);

struct Workspace {
    uint16_t* vals;       // [M_pad, Kc_pad] bf16, compressed kept values (rows >= M are zero)
    uint8_t* meta;        // [m_blocks, k_chunks, 2048] metadata chunks in tensor-memory order
    float* s;             // [M_pad] per-token scale
    uint16_t* T;          // [M_pad, R_pad] bf16, X L_B^T
    double* part_norm;    // [max_segs, M_pad, 2] partial sums of x^2 and of kept x^2
    float* part_T;        // [max_segs, M_pad, R_pad] partial X L_B^T
    float* split_part;    // [tail_units, 2, kSplitSlotFloats] fp32 partial tiles of the split tail
    int* split_cnt;       // [2 * (gemm_tiles - tail_full)] arrival tickets of the split tiles
    // FP8 form: metadata in the 8-bit layout (row m of a 128-token block at
    // byte 16 m of each 2 KB chunk, group g at nibble g of the row's 16 bytes)
    uint8_t* codes;       // [M_pad, Kc_pad] E4M3 codes of the kept entries
    float* qx;            // [M_pad] per-token dequantisation scale s * max|x| / 448
    float* part_amax;     // [max_segs, M_pad] partial max |x|
};

// Tensor-map encoding through the driver entry point (no libcuda link needed).
int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle);
inline int encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                               uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                               CUtensorMapSwizzle swizzle) {
    return encode_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, outer, row_stride_bytes, box_inner,
                          box_outer, swizzle);
}

// Launches `kernel` as a programmatic dependent of the preceding kernel in
// the stream: it may be scheduled while that kernel drains and must call
// grid_dependency_wait before reading what the preceding kernel wrote.
template <typename... KArgs, typename... Args>
int launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    return e != cudaSuccess ? static_cast<int>(e) : static_cast<int>(cudaGetLastError());
}

// Raises `kernel`'s dynamic shared-memory limit to the most a CTA may use,
// once per device (the attribute is kept by the runtime; setting it on every
// launch is host work the GPU may end up waiting for).  `done` is the
// kernel's own per-device record.
template <typename Kernel>
int allow_max_dynamic_smem(Kernel kernel, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return static_cast<int>(cudaErrorInvalidDevice);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return 0;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return static_cast<int>(e);
}

// Launchers; each returns a cudaError_t value (0 on success).
// The sparsify prologue: two launches (streaming pass, then per-token scale).
int launch_sparsify(const Dims& d, const void* X, const void* L_B, const Workspace& ws, int* err,
                    cudaStream_t stream);
// act: 0 none, 1 GELU (erf form) applied to the output before its bf16 rounding.
int launch_gemm(const Dims& d, bool sparse, const void* A, const void* W, const void* L_A, const Workspace& ws,
                void* Y, int act, int num_sms, int* err, cudaStream_t stream, const float* qw = nullptr);
// FP8 weight preparation: W8 = E4M3(W * 448 / max|W_n|), qw = max|W_n| / 448,
// L_A8 = L_A / qw (rows of all-zero channels divided by 1).
int launch_quantize_weight_fp8(const void* W, const void* L_A, void* W8, float* qw, void* L_A8, int64_t N,
                               int64_t K, int64_t R, cudaStream_t stream);
int launch_unpack_fp8_debug(const Dims& d, const Workspace& ws, void* codes, void* meta, void* qx,
                            cudaStream_t stream);
// Shared by the entry points (api.cu).
// Argument checks of one layer call; returns an rtlynx_status (nothing is
// launched).  Y must not share a byte with X, W, L_A or L_B.
int validate(const void* X, const void* W, const void* L_A, const void* L_B, const void* Y, int64_t M,
             int64_t K, int64_t N, int64_t R, int mode);
// The current device's SM count and the device address of the library's
// error word on it; an rtlynx_status.  Allocates nothing.
int device_info(int* num_sms, int** err_word);
bool ensure_tmap_encoder();
Workspace carve(void* base, const WsLayout& l);
int run_prologue(const Dims& d, const void* X, const void* L_B, const Workspace& ws, int* err, int num_sms,
                 cudaStream_t stream);

// Small problems in one kernel (small.cu): one wave of 256 x 240 tiles,
// D_in <= 256, R = 0 or R <= 64, bf16, no epilogue activation.
bool small_path_fits(const Dims& d, int num_sms);
int launch_small(const Dims& d, const void* X, const void* W, const void* L_A, const void* L_B,
                 const Workspace& ws, void* Y, int* err, cudaStream_t stream);

int launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t stream);
int launch_unpack_debug(const Dims& d, const Workspace& ws, void* vals, void* meta, void* s, void* T,
                        cudaStream_t stream);

}  // namespace rtlynx
