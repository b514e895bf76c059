/*
 * rtlynx.h - C ABI of the B200 (sm_100a) RT-Lynx activation-sparse linear layer.
 *
 * The operation (RT-Lynx summary page, paper.rainbus.top for arXiv 2605.26632,
 * "four-step pipeline" paragraph):
 *   step 1  X~ keeps, for every token, the 2 largest-magnitude entries of each
 *           group of 4 consecutive input channels (ties go to the lower
 *           channel); s = ||X||_2 / (||X~||_2 + 1e-8) per token; S(X) = s * X~.
 *   step 2  Y = S(X) W^T + X (L_A L_B)^T, the LoRA branch fed with the dense X.
 *   step 3  layers chosen for skipping run dense: Y = X W^T.
 *   step 4  mask, Top-K, compression to the sparse tensor-core layout and the
 *           sparse GEMM run in fused GPU kernels; the sparse and LoRA products
 *           are accumulated on chip.
 *
 * Conventions for every entry point:
 *   - Tensors are row-major bf16 (IEEE binary16-brain, little endian):
 *       X [M, D_in], W [D_out, D_in] (nn.Linear layout), L_A [D_out, R],
 *       L_B [R, D_in], Y [M, D_out].
 *   - Pointers are device memory owned by the caller unless a name ends in
 *     _host.  Inputs are only read.  Y is overwritten; a Y that shares a byte
 *     with an input is rejected with RTLYNX_ERR_INVALID_ARG.  Every pointer
 *     must be 16-byte aligned.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream; nothing synchronizes the host
 *     unless stated.
 *   - Return value: an rtlynx_status.  Argument errors return before anything
 *     is launched.
 *   - No kernel traps.  Every device-side wait is bounded; a wait that runs
 *     out records RTLYNX_ERR_DEVICE_TIMEOUT in a per-device error word that
 *     rtlynx_stream_status() reads and clears.
 */
#ifndef RTLYNX_H
#define RTLYNX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RTLYNX_MODE_SPARSE = 0,     /* Y = S(X) W^T + X (L_A L_B)^T  (steps 1-2) */
    RTLYNX_MODE_DENSE_SKIP = 1  /* Y = X W^T                     (step 3)    */
} rtlynx_mode;

typedef enum {
    RTLYNX_OK = 0,
    RTLYNX_ERR_INVALID_ARG = 1,    /* bad size, pointer, alignment or mode        */
    RTLYNX_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. R > 256, not sm_100) */
    RTLYNX_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed           */
    RTLYNX_ERR_OOM = 4,            /* workspace allocation failed                 */
    RTLYNX_ERR_DEVICE_TIMEOUT = 5  /* a bounded device-side wait ran out          */
} rtlynx_status;

/*
 * rtlynx_linear - the fused RT-Lynx linear layer (steps 1-4).
 *   M      tokens (> 0)            D_in   input channels, > 0, multiple of 8
 *   D_out  output channels, > 0, multiple of 8
 *   R      LoRA rank: 0 (no LoRA branch) or a multiple of 8 up to 256; with
 *          R = 0, or L_A / L_B NULL, sparse mode computes Y = S(X) W^T only
 *   mode   rtlynx_mode; DENSE_SKIP ignores L_A, L_B and R
 * Uses a workspace cached per (device, stream), grown with cudaMalloc when a
 * larger problem arrives (the stream is synchronized before the old buffer is
 * freed); call once outside any stream capture for each new size.
 */
int rtlynx_linear(const void* X, const void* W, const void* L_A, const void* L_B, void* Y, int64_t M,
                  int64_t D_in, int64_t D_out, int64_t R, int mode, void* stream);

/* Workspace bytes rtlynx_linear_ws needs for these sizes (0 for DENSE_SKIP;
 * 0 also when the arguments are invalid). */
size_t rtlynx_workspace_size(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode);

/* rtlynx_linear with a caller-owned device workspace of ws_bytes bytes
 * (>= rtlynx_workspace_size, 256-byte aligned).  Allocates nothing (the
 * device error word is a module variable of the library). */
int rtlynx_linear_ws(const void* X, const void* W, const void* L_A, const void* L_B, void* Y, int64_t M,
                     int64_t D_in, int64_t D_out, int64_t R, int mode, void* workspace, size_t ws_bytes,
                     void* stream);

/* rtlynx_linear_ws that also records caller-created CUDA events (cudaEvent_t
 * passed as void*, any may be NULL) on stream: ev_start before the first
 * kernel, ev_mid after the sparsify prologue (right before the GEMM kernel),
 * ev_end after the GEMM kernel.  Used to time the two phases separately. */
int rtlynx_linear_ws_events(const void* X, const void* W, const void* L_A, const void* L_B, void* Y,
                            int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, void* workspace,
                            size_t ws_bytes, void* ev_start, void* ev_mid, void* ev_end, void* stream);

/* Where the sparse-mode intermediates sit inside the workspace (byte offsets),
 * for tests that inspect them:
 *   vals       [M_pad, Kc_pad] bf16 kept values, rows >= M zero, Kc_pad >= D_in/2
 *   meta       [M_pad/128, k_chunks, 2048] bytes, metadata in tensor-memory order:
 *              for token m of a 128-token block (m0 = m%8, m1 = (m/8)%2,
 *              m2 = m/16) and channel k of a 128-channel chunk (k0 = k%16,
 *              k1 = (k/16)%2, k2 = k/32) the group nibble i0 | (i1<<2) sits in
 *              the 32-bit word at byte 16*(m0 + 8*k1 + 16*m2) + 4*k2, bits
 *              16*m1 + 4*(k0/4) ... +3
 *   s          [M_pad] float
 *   T          [M_pad, R_pad] bf16, X L_B^T */
typedef struct {
    int64_t M_pad, Kc_pad, k_chunks, R_pad;
    size_t vals, meta, s, T, total;
} rtlynx_ws_layout;
int rtlynx_workspace_layout(int64_t M, int64_t D_in, int64_t D_out, int64_t R, rtlynx_ws_layout* out);

/* Step 1 and the LoRA down-projection alone, written in plain layouts:
 *   vals [M, D_in/2] bf16 (kept values in channel order), meta [M, D_in/4]
 *   uint8 (one nibble i0 | (i1<<2) per byte), s [M] float, T [M, R] bf16.
 * Any output pointer may be NULL.  Uses the cached workspace of rtlynx_linear. */
int rtlynx_sparsify_debug(const void* X, const void* L_B, int64_t M, int64_t D_in, int64_t R, void* vals,
                          void* meta, void* s, void* T, void* stream);

/* ---------------------------------------------------------------- FP8 form
 * The layer with E4M3 operands (the pages name FP8 as future work that
 * stacks with the method; the recipe is this library's reading):
 *   - W per output channel: qw[n] = max_k |W[n,k]| / 448 and codes
 *     W8 = E4M3(W * 448 / max|W_n|), float32 product, nearest even,
 *     saturating at 448; all-zero channels get qw = 0 and zero codes;
 *   - S(X) per token: q_x = s * max|x| / 448, codes of the kept entries
 *     E4M3(x~ * 448 / max|x|) (the largest |x| of a token is always kept);
 *   - Y = q_x qw[n] sum(x8 w8) + X L_B^T L_A^T, rounded to bf16.
 * The GEMM accumulates x8 w8 and the LoRA product of T / q_x and
 * L_A8 = L_A / qw (bf16) in one accumulator and multiplies it by q_x qw[n].
 * Validation, before anything is launched: a size <= 0, D_in not a multiple
 * of 256 (whole 256-K stages), D_out not a multiple of 8, a NULL or
 * misaligned pointer, or R > 0 without the LoRA factors give
 * RTLYNX_ERR_INVALID_ARG; R not a multiple of 8, or above 256, gives
 * RTLYNX_ERR_UNSUPPORTED.  Device-side timeouts are reported as for the
 * bf16 layer (rtlynx_stream_status).
 */

/* Weight preparation, once per layer: W [D_out, D_in] bf16 -> W8 [D_out, D_in]
 * E4M3 codes (bytes), qw [D_out] float, L_A8 [D_out, R] bf16 = L_A / qw (a
 * zero qw divides by 1).  L_A and L_A8 may be NULL when R == 0. */
int rtlynx_quantize_weight_fp8(const void* W, const void* L_A, void* W8, void* qw, void* L_A8, int64_t D_out,
                               int64_t D_in, int64_t R, void* stream);

/* The FP8 layer, sparse mode: X [M, D_in] bf16, W8 / qw / L_A8 from
 * rtlynx_quantize_weight_fp8, L_B [R, D_in] bf16, Y [M, D_out] bf16.  Uses
 * the cached workspace of rtlynx_linear. */
int rtlynx_linear_fp8(const void* X, const void* W8, const void* qw, const void* L_A8, const void* L_B, void* Y,
                      int64_t M, int64_t D_in, int64_t D_out, int64_t R, void* stream);

/* rtlynx_linear_fp8 that also records caller-created CUDA events (any may
 * be NULL): before the prologue, between prologue and GEMM, after the GEMM. */
int rtlynx_linear_fp8_events(const void* X, const void* W8, const void* qw, const void* L_A8, const void* L_B,
                             void* Y, int64_t M, int64_t D_in, int64_t D_out, int64_t R, void* ev_start,
                             void* ev_mid, void* ev_end, void* stream);

/* Step 1 of the FP8 form alone, in plain layouts: codes [M, D_in/2] E4M3 of
 * the kept entries in channel order, meta [M, D_in/4] (one nibble per byte),
 * qx [M] float.  Any output pointer may be NULL. */
int rtlynx_sparsify_fp8_debug(const void* X, int64_t M, int64_t D_in, void* codes, void* meta, void* qx,
                              void* stream);

/* End-to-end form for callers whose activations live in host memory:
 * copies X_host to X_dev, runs rtlynx_linear into Y_dev, copies Y_dev to
 * Y_host.  The work is cut into up to eight token chunks (of at least 512
 * tokens) and pipelined: uploads run on one helper stream, each chunk's layer
 * on `stream` once its upload has landed, downloads on a second helper stream
 * once its layer is done, so copies in both directions overlap the compute.
 * The helper streams belong to the library (one pair per device, created on
 * the first call; make it outside any stream capture).  Everything is ordered
 * after the work already queued on `stream`, and later work queued on
 * `stream` waits for all of it; synchronize `stream` before reading Y_host.
 * X_host and Y_host should be pinned (page-locked) for the copies to overlap.
 * W, L_A, L_B, X_dev and Y_dev are device pointers; X_dev and Y_dev must not
 * overlap.  Concurrent calls from several host threads are serialized while
 * they enqueue. */
int rtlynx_linear_host(const void* X_host, const void* W, const void* L_A, const void* L_B, void* Y_host,
                       int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, void* X_dev, void* Y_dev,
                       void* stream);

/*
 * rtlynx_mlp_block - the feed-forward part of a DiT block built from two
 * RT-Lynx linear layers (RT-Lynx summary page, four-step pipeline paragraph:
 * steps 1-2 for each layer, step 3 for layers chosen for skipping):
 *   H = GELU(layer_up(X))      [M, D_ff], GELU in its erf form,
 *                              x/2 (1 + erf(x/sqrt 2)), applied in the
 *                              up-projection's epilogue before the bf16
 *                              rounding of H (no separate pass)
 *   Y = layer_down(H)          [M, D]
 * Each layer runs as rtlynx_linear with its own mode (mode_up, mode_down:
 * RTLYNX_MODE_SPARSE or RTLYNX_MODE_DENSE_SKIP, selective layer skipping)
 * and LoRA pair; both pairs have rank R.
 *   X [M, D], W_up [D_ff, D], LA_up [D_ff, R], LB_up [R, D],
 *   W_down [D, D_ff], LA_down [D, R], LB_down [R, D_ff], all bf16, device.
 *   H  caller-owned [M, D_ff] bf16 device buffer that receives the GELU
 *      activations (the down-projection's input); it must not overlap X or Y.
 *   D and D_ff multiples of 8.
 * Uses the workspace cache of rtlynx_linear (sized for the larger layer).
 * Argument errors of either layer return before anything is launched.
 */
int rtlynx_mlp_block(const void* X, const void* W_up, const void* LA_up, const void* LB_up, const void* W_down,
                     const void* LA_down, const void* LB_down, void* H, void* Y, int64_t M, int64_t D, int64_t D_ff,
                     int64_t R, int mode_up, int mode_down, void* stream);

/* Largest workspace rtlynx_linear_noalloc can use (32 MiB). */
#define RTLYNX_NOALLOC_MAX_BYTES (32u << 20)

/*
 * rtlynx_linear_noalloc - rtlynx_linear for callers that cannot allocate
 * device memory.  (The RT-Lynx pages have no counterpart: this is a
 * deployment entry point.)
 *
 * Some callers cannot call cudaMalloc where they run the layer: a serving
 * engine that has handed all device memory to its own pool, code whose
 * allocations must go through an allocator this library does not see, or a
 * latency-critical path where cudaMalloc, which may synchronize the device,
 * is not acceptable.  This entry point allocates nothing.  Its workspace is a
 * static device array of RTLYNX_NOALLOC_MAX_BYTES that every GPU using this
 * entry point holds until the process exits; problems whose workspace
 * (rtlynx_workspace_size) is larger are rejected with RTLYNX_ERR_UNSUPPORTED
 * before anything is launched.
 *   dev_status  a caller-owned, 4-byte-aligned device int, or NULL.  A
 *               bounded device-side wait that runs out stores a nonzero code
 *               (1) there, the kernels of the call then stop early, and Y is
 *               incomplete; the caller zeroes the int beforehand and reads it
 *               after synchronizing.  With NULL the code goes to the library's
 *               own per-device error word (a module variable, no allocation),
 *               which rtlynx_stream_status reports as RTLYNX_ERR_DEVICE_TIMEOUT
 *               and clears, exactly as for rtlynx_linear.
 * Other arguments as rtlynx_linear.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) and reads device properties;
 * make it outside any stream capture.  Every call shares the one array and
 * rewrites every part it reads, so nothing needs clearing between calls, but
 * calls that overlap on the GPU (other streams or host threads on the same
 * device) race on it and must be serialized by the caller.
 */
int rtlynx_linear_noalloc(const void* X, const void* W, const void* L_A, const void* L_B, void* Y, int64_t M,
                          int64_t D_in, int64_t D_out, int64_t R, int mode, int* dev_status, void* stream);

/* The work split one sparse-mode call uses on a GPU with num_sms SMs (2 ..
 * 1024), computed on the host alone (no GPU needed):
 *   prologue_ctas      CTAs of the streaming sparsify pass; CTA c takes the
 *                      tiles [c T / G, (c + 1) T / G) of the T = prologue_tiles
 *                      (row block x 64-wide K tile) tiles, G = prologue_ctas,
 *                      row block b owning tiles [b k, (b + 1) k), k =
 *                      k_tiles_per_block
 *   prologue_max_segs  the most CTAs whose tiles meet one row block (the
 *                      partial-sum slots the workspace holds per token)
 *   gemm_pairs, gemm_tiles  persistent CTA pairs and 256 x 240 output tiles
 *   tail_full, tail_split, tail_units  tiles [0, tail_full) run whole; each
 *                      later tile is cut along its stages into tail_split
 *                      parts (tail_units parts in all, one per pair)
 *   k_stages, lora_stages  pipeline stages of one tile (main loop, LoRA-up)
 *   small_path         1 when the problem is one wave of 256 x 240 tiles with
 *                      D_in <= 256 and R = 0 or R <= 64: the call is then one
 *                      kernel whose CTA pairs sparsify their own tokens in
 *                      shared memory (the fields above describe the general
 *                      form it replaces)
 * RTLYNX_ERR_INVALID_ARG for invalid sizes or a NULL out. */
typedef struct {
    int64_t prologue_ctas, prologue_tiles, prologue_max_segs, row_blocks, k_tiles_per_block;
    int64_t gemm_pairs, gemm_tiles, tail_full, tail_split, tail_units, k_stages, lora_stages;
    int64_t small_path;  /* 1: the call runs as one kernel (small problems, see above) */
} rtlynx_schedule;
int rtlynx_schedule_info(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int num_sms, rtlynx_schedule* out);

/* Number of kernels one rtlynx_linear call with these sizes launches on the
 * current device (0 for invalid sizes): the sparse path launches its two
 * sparsify kernels and the GEMM, or one kernel where the problem takes the
 * small path (rtlynx_schedule.small_path); the dense-skip path the GEMM alone. */
int rtlynx_kernel_launches(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode);

/* Self-test of the device-side failure detection: launches one thread that
 * waits on a barrier nothing arrives on.  The wait gives up after limit_ns
 * (1 .. 1e9), records RTLYNX_ERR_DEVICE_TIMEOUT in the device error word and
 * returns; the next rtlynx_stream_status() on the stream reports it. */
int rtlynx_wait_selftest(int64_t limit_ns, void* stream);

/* Synchronizes stream, then returns and clears the current device's error
 * word (RTLYNX_OK or RTLYNX_ERR_DEVICE_TIMEOUT), or RTLYNX_ERR_CUDA. */
int rtlynx_stream_status(void* stream);

/* Static text for a status code. */
const char* rtlynx_status_string(int status);

/* Frees every cached workspace and error word (synchronizes the device). */
void rtlynx_release(void);

#ifdef __cplusplus
}
#endif

#endif /* RTLYNX_H */
