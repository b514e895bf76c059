// C ABI of the RT-Lynx linear layer: argument checks, workspace management,
// tensor-map encoding and the launch sequence.  See include/rtlynx.h.
#include <mutex>
#include <unordered_map>

#include "../../include/rtlynx.h"
#include "internal.h"

namespace rtlynx {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    bool supported = false;
    int num_sms = 0;
    int* err_word = nullptr;  // device address of g_err_word on this device
};

// The per-device error word: a module variable, so that every device that
// loads the library has its own copy and no call has to allocate one.
__device__ int g_err_word;

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];

struct WsEntry {
    void* ptr = nullptr;
    size_t bytes = 0;
};
struct WsKey {
    int dev;
    cudaStream_t stream;
    bool operator==(const WsKey& o) const { return dev == o.dev && stream == o.stream; }
};
struct WsKeyHash {
    size_t operator()(const WsKey& k) const {
        return std::hash<void*>()(static_cast<void*>(k.stream)) ^ (static_cast<size_t>(k.dev) << 1);
    }
};
std::unordered_map<WsKey, WsEntry, WsKeyHash> g_ws;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RTLYNX_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& di = g_dev[dev];
    if (!di.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return RTLYNX_ERR_CUDA;
        di.supported = (major == 10 && minor == 0);
        di.num_sms = sms;
        if (di.supported) {
            void* word = nullptr;
            if (cudaGetSymbolAddress(&word, g_err_word) != cudaSuccess || word == nullptr) {
                cudaGetLastError();
                return RTLYNX_ERR_CUDA;
            }
            di.err_word = static_cast<int*>(word);
            if (cudaMemset(di.err_word, 0, sizeof(int)) != cudaSuccess) return RTLYNX_ERR_CUDA;
        }
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return RTLYNX_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        di.init = true;
    }
    if (!di.supported) return RTLYNX_ERR_UNSUPPORTED;
    *out = &di;
    return RTLYNX_OK;
}

// The host-buffer entry point pipelines its copies over token chunks on two
// helper streams per device (uploads, downloads), created on first use.
constexpr int kHostChunks = 8;
struct HostPipe {
    bool ready = false;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join_up = nullptr, ev_join_down = nullptr;
    cudaEvent_t ev_h2d[kHostChunks] = {}, ev_comp[kHostChunks] = {};
};
std::mutex g_host_mutex;
HostPipe g_host[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
    HostPipe& hp = g_host[dev];
    if (!hp.ready) {
        auto ev = [](cudaEvent_t* e) { return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess; };
        bool ok = cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking) == cudaSuccess && ev(&hp.ev_fork) &&
                  ev(&hp.ev_join_up) && ev(&hp.ev_join_down);
        for (int i = 0; ok && i < kHostChunks; ++i) ok = ev(&hp.ev_h2d[i]) && ev(&hp.ev_comp[i]);
        if (!ok) {
            cudaGetLastError();
            return RTLYNX_ERR_CUDA;
        }
        hp.ready = true;
    }
    *out = &hp;
    return RTLYNX_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// True when the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, uint64_t na, const void* b, uint64_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace

int validate(const void* X, const void* W, const void* L_A, const void* L_B, const void* Y, int64_t M,
             int64_t K, int64_t N, int64_t R, int mode) {
    if (mode != RTLYNX_MODE_SPARSE && mode != RTLYNX_MODE_DENSE_SKIP) return RTLYNX_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0 || N <= 0 || R < 0) return RTLYNX_ERR_INVALID_ARG;
    if (K % 8 != 0 || N % 8 != 0) return RTLYNX_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) - 2 * kBM || K > (int64_t(1) << 30) || N > (int64_t(1) << 30))
        return RTLYNX_ERR_UNSUPPORTED;
    if (!X || !W || !Y) return RTLYNX_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y)) return RTLYNX_ERR_INVALID_ARG;
    const bool lora = mode == RTLYNX_MODE_SPARSE && R > 0;
    if (lora) {
        if (!L_A || !L_B) return RTLYNX_ERR_INVALID_ARG;
        if (!aligned16(L_A) || !aligned16(L_B)) return RTLYNX_ERR_INVALID_ARG;
        if (R % 8 != 0 || R > 256) return RTLYNX_ERR_UNSUPPORTED;
    }
    // Y is written while the inputs are still being read: it must not share a
    // byte with any of them.
    const uint64_t m = static_cast<uint64_t>(M), k = static_cast<uint64_t>(K), n = static_cast<uint64_t>(N),
                   r = static_cast<uint64_t>(R);
    const uint64_t y_bytes = 2 * m * n;
    if (overlaps(Y, y_bytes, X, 2 * m * k) || overlaps(Y, y_bytes, W, 2 * n * k)) return RTLYNX_ERR_INVALID_ARG;
    if (lora && (overlaps(Y, y_bytes, L_A, 2 * n * r) || overlaps(Y, y_bytes, L_B, 2 * r * k)))
        return RTLYNX_ERR_INVALID_ARG;
    return RTLYNX_OK;
}

int device_info(int* num_sms, int** err_word) {
    DeviceInfo* di = nullptr;
    const int rc = current_device(&di);
    if (rc) return rc;
    *num_sms = di->num_sms;
    *err_word = di->err_word;
    return RTLYNX_OK;
}

bool ensure_tmap_encoder() {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return false;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return true;
}

namespace {

// A layer call encodes the same handful of tensor maps every time it runs on
// the same buffers; encoding is host work that can leave the GPU waiting.
// Each host thread keeps the last kTmapCacheSize maps it encoded, keyed by
// every argument of the encode, and hands back an identical copy.
struct TmapKey {
    const void* base;
    uint64_t inner, outer, stride;
    uint32_t box_inner, box_outer;
    int dtype, swizzle;
    bool operator==(const TmapKey& o) const {
        return base == o.base && inner == o.inner && outer == o.outer && stride == o.stride &&
               box_inner == o.box_inner && box_outer == o.box_outer && dtype == o.dtype && swizzle == o.swizzle;
    }
};
constexpr int kTmapCacheSize = 16;
struct TmapCache {
    TmapKey key[kTmapCacheSize];
    CUtensorMap map[kTmapCacheSize];
    int count = 0, next = 0;
};
thread_local TmapCache t_tmap_cache;

}  // namespace

int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle) {
    (void)elem_bytes;
    if (!g_encode) return cudaErrorInitializationError;
    const TmapKey key{base, inner, outer, row_stride_bytes, box_inner, box_outer, static_cast<int>(dtype),
                      static_cast<int>(swizzle)};
    TmapCache& c = t_tmap_cache;
    for (int i = 0; i < c.count; ++i) {
        if (c.key[i] == key) {
            *map = c.map[i];
            return 0;
        }
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return static_cast<int>(cudaErrorInvalidValue);
    c.key[c.next] = key;
    c.map[c.next] = *map;
    c.next = (c.next + 1) % kTmapCacheSize;
    if (c.count < kTmapCacheSize) ++c.count;
    return 0;
}

Dims make_dims(int64_t M, int64_t K, int64_t N, int64_t R, int num_sms, bool fp8) {
    Dims d;
    d.fp8 = fp8;
    d.M = M;
    d.K = K;
    d.N = N;
    d.R = R;
    d.M_pad = (M + 2 * kBM - 1) / (2 * kBM) * (2 * kBM);
    d.m_blocks = d.M_pad / kBM;
    d.k_tiles = (K + kBK - 1) / kBK;
    d.k_chunks = (K + kChunkK - 1) / kChunkK;
    d.Kc_pad = d.k_chunks * (kChunkK / 2);
    d.R_pad = R > 0 ? (R + 63) / 64 * 64 : 0;
    // Streaming prologue: one CTA per SM over the row-block x K-tile grid.
    d.kt2 = 2 * d.k_chunks;
    const int64_t total = d.m_blocks * d.kt2;
    const int64_t sms = num_sms > 0 ? num_sms : 148;
    // Four tiles a CTA or more once that still leaves 32 CTAs: with fewer, a
    // row block splits into so many segments that summing their partials
    // dominates the scale pass.  Very small problems keep a CTA per tile.
    int64_t by_work = (total + 3) / 4;
    const int64_t floor_ctas = total < 32 ? total : 32;
    if (by_work < floor_ctas) by_work = floor_ctas;
    d.grid1 = by_work < sms ? by_work : sms;
    // A row block's kt2 tiles meet at most (kt2 - 2) / L + 2 runs when every
    // run holds at least L = floor(total / grid1) tiles.
    const int64_t run = total / d.grid1;
    d.max_segs = (d.kt2 - 2) / run + 2;
    // Sparse GEMM: full rounds of tiles over the pairs, then the remainder
    // tiles cut along K so that every pair has a part (3 to kMaxSplit parts a
    // tile, each at least two stages long).
    const int64_t m_pairs = d.M_pad / (2 * kBM);
    const int64_t bn = fp8 ? kFp8BN : kPairBN;
    const int64_t n_tiles = (N + bn - 1) / bn;
    d.gemm_tiles = m_pairs * n_tiles;
    const int64_t max_pairs = (num_sms > 0 ? num_sms : 148) / 2;
    d.gemm_pairs = d.gemm_tiles < max_pairs ? d.gemm_tiles : max_pairs;
    const int64_t rem = d.gemm_tiles % d.gemm_pairs;
    const int64_t n_iter = sparse_k_stages(d) + sparse_lora_stages(d);
    int64_t split = rem > 0 ? d.gemm_pairs / rem : 1;
    if (split > kMaxSplit) split = kMaxSplit;
    if (split > n_iter / 2) split = n_iter / 2;
    // A split tile pays for a partial store, a ticket and a fix-up; two parts
    // save less than that costs.
    if (split < 3) {
        d.tail_full = d.gemm_tiles;
        d.tail_split = 1;
        d.tail_units = 0;
    } else {
        d.tail_full = d.gemm_tiles - rem;
        d.tail_split = split;
        d.tail_units = rem * split;
    }
    return d;
}

WsLayout make_ws_layout(const Dims& d) {
    WsLayout l;
    size_t off = 0;
    l.vals = off;
    off = align256(off + static_cast<size_t>(d.M_pad) * d.Kc_pad * 2);
    l.meta = off;
    off = align256(off + static_cast<size_t>(d.m_blocks) * d.k_chunks * kChunkBytes);
    l.s = off;
    off = align256(off + static_cast<size_t>(d.M_pad) * 4);
    l.T = off;
    off = align256(off + static_cast<size_t>(d.M_pad) * d.R_pad * 2);
    l.part_norm = off;
    off = align256(off + static_cast<size_t>(d.max_segs) * d.M_pad * 2 * 8);
    l.part_T = off;
    off = align256(off + static_cast<size_t>(d.max_segs) * d.M_pad * d.R_pad * 4);
    l.split_part = off;
    off = align256(off + static_cast<size_t>(d.tail_units) * 2 * kSplitSlotFloats * 4);
    l.split_cnt = off;
    off = align256(off + static_cast<size_t>(d.gemm_tiles - d.tail_full) * 2 * 4);
    const int64_t f = d.fp8 ? 1 : 0;
    l.codes = off;
    off = align256(off + static_cast<size_t>(f * d.M_pad * d.Kc_pad));
    l.qx = off;
    off = align256(off + static_cast<size_t>(f * d.M_pad * 4));
    l.part_amax = off;
    off = align256(off + static_cast<size_t>(f * d.max_segs * d.M_pad * 4));
    l.total = off;
    return l;
}

Workspace carve(void* base, const WsLayout& l) {
    uint8_t* b = static_cast<uint8_t*>(base);
    Workspace w;
    w.vals = reinterpret_cast<uint16_t*>(b + l.vals);
    w.meta = b + l.meta;
    w.s = reinterpret_cast<float*>(b + l.s);
    w.T = reinterpret_cast<uint16_t*>(b + l.T);
    w.part_norm = reinterpret_cast<double*>(b + l.part_norm);
    w.part_T = reinterpret_cast<float*>(b + l.part_T);
    w.split_part = reinterpret_cast<float*>(b + l.split_part);
    w.split_cnt = reinterpret_cast<int*>(b + l.split_cnt);
    w.codes = b + l.codes;
    w.qx = reinterpret_cast<float*>(b + l.qx);
    w.part_amax = reinterpret_cast<float*>(b + l.part_amax);
    return w;
}

// Grow (or create) the cached workspace of (device, stream).
static int cached_workspace(int dev, cudaStream_t stream, size_t bytes, void** out) {
    std::lock_guard<std::mutex> lock(g_mutex);
    WsEntry& e = g_ws[WsKey{dev, stream}];
    if (e.bytes < bytes) {
        if (e.ptr) {
            if (cudaStreamSynchronize(stream) != cudaSuccess) return RTLYNX_ERR_CUDA;
            cudaFree(e.ptr);
            e.ptr = nullptr;
            e.bytes = 0;
        }
        if (cudaMalloc(&e.ptr, bytes) != cudaSuccess) {
            cudaGetLastError();
            return RTLYNX_ERR_OOM;
        }
        e.bytes = bytes;
    }
    *out = e.ptr;
    return RTLYNX_OK;
}

// One linear layer on a validated problem: the sparse path (prologue, then
// the GEMM with LoRA) or the dense-skip GEMM; `act` selects the epilogue
// activation.  Events (any may be null) are recorded before the first kernel,
// between prologue and GEMM, and after the GEMM.
static int run_layer(DeviceInfo* di, const void* X, const void* W, const void* L_A, const void* L_B, void* Y,
                     int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, int act, void* workspace,
                     size_t ws_bytes, void* ev_start, void* ev_mid, void* ev_end, cudaStream_t stream) {
    const bool lora = (mode == RTLYNX_MODE_SPARSE) && R > 0 && L_A && L_B;
    const Dims d = make_dims(M, D_in, D_out, lora ? R : 0, di->num_sms);
    auto record = [&](void* ev) {
        return ev == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(ev), stream) == cudaSuccess;
    };
    if (mode == RTLYNX_MODE_DENSE_SKIP) {
        Workspace none{};
        if (!record(ev_start) || !record(ev_mid)) return RTLYNX_ERR_CUDA;
        if (launch_gemm(d, false, X, W, nullptr, none, Y, act, di->num_sms, di->err_word, stream))
            return RTLYNX_ERR_CUDA;
        return record(ev_end) ? RTLYNX_OK : RTLYNX_ERR_CUDA;
    }
    const WsLayout l = make_ws_layout(d);
    if (!workspace || ws_bytes < l.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return RTLYNX_ERR_INVALID_ARG;
    const Workspace ws = carve(workspace, l);
    if (!record(ev_start)) return RTLYNX_ERR_CUDA;
    if (act == 0 && small_path_fits(d, di->num_sms)) {
        // one kernel: each CTA pair sparsifies its tokens in shared memory
        if (!record(ev_mid)) return RTLYNX_ERR_CUDA;
        if (launch_small(d, X, W, lora ? L_A : nullptr, lora ? L_B : nullptr, ws, Y, di->err_word, stream))
            return RTLYNX_ERR_CUDA;
        return record(ev_end) ? RTLYNX_OK : RTLYNX_ERR_CUDA;
    }
    int rc = run_prologue(d, X, lora ? L_B : nullptr, ws, di->err_word, di->num_sms, stream);
    if (rc) return rc;
    if (!record(ev_mid)) return RTLYNX_ERR_CUDA;
    if (launch_gemm(d, true, nullptr, W, lora ? L_A : nullptr, ws, Y, act, di->num_sms, di->err_word, stream))
        return RTLYNX_ERR_CUDA;
    return record(ev_end) ? RTLYNX_OK : RTLYNX_ERR_CUDA;
}

// The sparsify prologue: pass 1 and pass 2 (the partition over CTAs is fixed
// in make_dims).
int run_prologue(const Dims& d, const void* X, const void* L_B, const Workspace& ws, int* err, int num_sms,
                 cudaStream_t stream) {
    (void)num_sms;  // the split is fixed in make_dims
    return launch_sparsify(d, X, L_B, ws, err, stream) ? RTLYNX_ERR_CUDA : RTLYNX_OK;
}

}  // namespace rtlynx

using namespace rtlynx;

extern "C" {

size_t rtlynx_workspace_size(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode) {
    if (mode == RTLYNX_MODE_DENSE_SKIP) return 0;
    if (mode != RTLYNX_MODE_SPARSE || M <= 0 || D_in <= 0 || D_out <= 0 || R < 0 || D_in % 8 || D_out % 8)
        return 0;
    DeviceInfo* di = nullptr;
    const int sms = current_device(&di) == RTLYNX_OK ? di->num_sms : 148;
    return make_ws_layout(make_dims(M, D_in, D_out, R, sms)).total;
}

int rtlynx_workspace_layout(int64_t M, int64_t D_in, int64_t D_out, int64_t R, rtlynx_ws_layout* out) {
    if (!out || M <= 0 || D_in <= 0 || D_out <= 0 || R < 0 || D_in % 8 || D_out % 8) return RTLYNX_ERR_INVALID_ARG;
    DeviceInfo* di = nullptr;
    const int sms = current_device(&di) == RTLYNX_OK ? di->num_sms : 148;
    const Dims d = make_dims(M, D_in, D_out, R, sms);
    const WsLayout l = make_ws_layout(d);
    out->M_pad = d.M_pad;
    out->Kc_pad = d.Kc_pad;
    out->k_chunks = d.k_chunks;
    out->R_pad = d.R_pad;
    out->vals = l.vals;
    out->meta = l.meta;
    out->s = l.s;
    out->T = l.T;
    out->total = l.total;
    return RTLYNX_OK;
}

int rtlynx_linear_ws_events(const void* X, const void* W, const void* L_A, const void* L_B, void* Y,
                            int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, void* workspace,
                            size_t ws_bytes, void* ev_start, void* ev_mid, void* ev_end, void* stream_) {
    int rc = validate(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode);
    if (rc) return rc;
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    return run_layer(di, X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, 0, workspace, ws_bytes, ev_start, ev_mid, ev_end,
                     static_cast<cudaStream_t>(stream_));
}

int rtlynx_linear_ws(const void* X, const void* W, const void* L_A, const void* L_B, void* Y, int64_t M,
                     int64_t D_in, int64_t D_out, int64_t R, int mode, void* workspace, size_t ws_bytes,
                     void* stream_) {
    return rtlynx_linear_ws_events(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, workspace, ws_bytes, nullptr,
                                   nullptr, nullptr, stream_);
}

int rtlynx_linear(const void* X, const void* W, const void* L_A, const void* L_B, void* Y, int64_t M,
                  int64_t D_in, int64_t D_out, int64_t R, int mode, void* stream_) {
    int rc = validate(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode);
    if (rc) return rc;
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    if (mode == RTLYNX_MODE_DENSE_SKIP)
        return rtlynx_linear_ws(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, nullptr, 0, stream_);
    int dev = 0;
    cudaGetDevice(&dev);
    const bool lora = R > 0 && L_A && L_B;
    const size_t bytes = make_ws_layout(make_dims(M, D_in, D_out, lora ? R : 0, di->num_sms)).total;
    void* ws = nullptr;
    rc = cached_workspace(dev, static_cast<cudaStream_t>(stream_), bytes, &ws);
    if (rc) return rc;
    return rtlynx_linear_ws(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, ws, bytes, stream_);
}

int rtlynx_mlp_block(const void* X, const void* W_up, const void* LA_up, const void* LB_up, const void* W_down,
                     const void* LA_down, const void* LB_down, void* H, void* Y, int64_t M, int64_t D, int64_t D_ff,
                     int64_t R, int mode_up, int mode_down, void* stream_) {
    int rc = validate(X, W_up, LA_up, LB_up, H, M, D, D_ff, R, mode_up);
    if (rc) return rc;
    rc = validate(H, W_down, LA_down, LB_down, Y, M, D_ff, D, R, mode_down);
    if (rc) return rc;
    if (H == X || H == Y || Y == X) return RTLYNX_ERR_INVALID_ARG;
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    auto ws_bytes = [&](int64_t K, int64_t N, const void* la, const void* lb, int mode) -> size_t {
        if (mode == RTLYNX_MODE_DENSE_SKIP) return 0;
        const bool lora = R > 0 && la && lb;
        return make_ws_layout(make_dims(M, K, N, lora ? R : 0, di->num_sms)).total;
    };
    const size_t b_up = ws_bytes(D, D_ff, LA_up, LB_up, mode_up);
    const size_t b_dn = ws_bytes(D_ff, D, LA_down, LB_down, mode_down);
    const size_t bytes = b_up > b_dn ? b_up : b_dn;
    void* ws = nullptr;
    if (bytes > 0) {
        rc = cached_workspace(dev, stream, bytes, &ws);
        if (rc) return rc;
    }
    // up-projection with GELU in its epilogue, then the down-projection; the
    // two layers use the workspace one after the other in stream order
    rc = run_layer(di, X, W_up, LA_up, LB_up, H, M, D, D_ff, R, mode_up, 1, ws, bytes, nullptr, nullptr, nullptr,
                   stream);
    if (rc) return rc;
    return run_layer(di, H, W_down, LA_down, LB_down, Y, M, D_ff, D, R, mode_down, 0, ws, bytes, nullptr, nullptr,
                     nullptr, stream);
}

int rtlynx_sparsify_debug(const void* X, const void* L_B, int64_t M, int64_t D_in, int64_t R, void* vals,
                          void* meta, void* s, void* T, void* stream_) {
    if (!X || M <= 0 || D_in <= 0 || D_in % 8 || R < 0 || !aligned16(X)) return RTLYNX_ERR_INVALID_ARG;
    if (R > 0 && (!L_B || !aligned16(L_B))) return RTLYNX_ERR_INVALID_ARG;
    if (R % 8 != 0 || R > 256) return RTLYNX_ERR_UNSUPPORTED;
    DeviceInfo* di = nullptr;
    int rc = current_device(&di);
    if (rc) return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int dev = 0;
    cudaGetDevice(&dev);
    const Dims d = make_dims(M, D_in, 8, R, di->num_sms);
    const WsLayout l = make_ws_layout(d);
    void* base = nullptr;
    rc = cached_workspace(dev, stream, l.total, &base);
    if (rc) return rc;
    const Workspace ws = carve(base, l);
    rc = run_prologue(d, X, R > 0 ? L_B : nullptr, ws, di->err_word, di->num_sms, stream);
    if (rc) return rc;
    if (launch_unpack_debug(d, ws, vals, meta, s, R > 0 ? T : nullptr, stream)) return RTLYNX_ERR_CUDA;
    return RTLYNX_OK;
}

// ---------------------------------------------------------------- FP8 form
static int validate_fp8(int64_t M, int64_t K, int64_t N, int64_t R) {
    if (M <= 0 || K <= 0 || N <= 0 || R < 0) return RTLYNX_ERR_INVALID_ARG;
    if (K % kFp8StageK != 0 || N % 8 != 0) return RTLYNX_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) - kBM || K > (int64_t(1) << 30) || N > (int64_t(1) << 30))
        return RTLYNX_ERR_UNSUPPORTED;
    if (R % 8 != 0 || R > 256) return RTLYNX_ERR_UNSUPPORTED;
    return RTLYNX_OK;
}

int rtlynx_quantize_weight_fp8(const void* W, const void* L_A, void* W8, void* qw, void* L_A8, int64_t D_out,
                               int64_t D_in, int64_t R, void* stream_) {
    int rc = validate_fp8(1, D_in, D_out, R);
    if (rc) return rc;
    if (!W || !W8 || !qw || !aligned16(W) || !aligned16(W8) || !aligned16(qw)) return RTLYNX_ERR_INVALID_ARG;
    if (R > 0 && (!L_A || !L_A8 || !aligned16(L_A) || !aligned16(L_A8))) return RTLYNX_ERR_INVALID_ARG;
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    return launch_quantize_weight_fp8(W, R > 0 ? L_A : nullptr, W8, static_cast<float*>(qw), R > 0 ? L_A8 : nullptr,
                                      D_out, D_in, R, static_cast<cudaStream_t>(stream_))
               ? RTLYNX_ERR_CUDA
               : RTLYNX_OK;
}

int rtlynx_linear_fp8_events(const void* X, const void* W8, const void* qw, const void* L_A8, const void* L_B,
                             void* Y, int64_t M, int64_t D_in, int64_t D_out, int64_t R, void* ev_start,
                             void* ev_mid, void* ev_end, void* stream_) {
    int rc = validate_fp8(M, D_in, D_out, R);
    if (rc) return rc;
    if (!X || !W8 || !qw || !Y || !aligned16(X) || !aligned16(W8) || !aligned16(qw) || !aligned16(Y))
        return RTLYNX_ERR_INVALID_ARG;
    if (R > 0 && (!L_A8 || !L_B || !aligned16(L_A8) || !aligned16(L_B))) return RTLYNX_ERR_INVALID_ARG;
    {
        const uint64_t m = static_cast<uint64_t>(M), k = static_cast<uint64_t>(D_in), n = static_cast<uint64_t>(D_out),
                       r = static_cast<uint64_t>(R);
        const uint64_t yb = 2 * m * n;
        if (overlaps(Y, yb, X, 2 * m * k) || overlaps(Y, yb, W8, n * k) || overlaps(Y, yb, qw, 4 * n) ||
            (R > 0 && (overlaps(Y, yb, L_A8, 2 * n * r) || overlaps(Y, yb, L_B, 2 * r * k))))
            return RTLYNX_ERR_INVALID_ARG;
    }
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const Dims d = make_dims(M, D_in, D_out, R, di->num_sms, true);
    const WsLayout l = make_ws_layout(d);
    void* base = nullptr;
    rc = cached_workspace(dev, stream, l.total, &base);
    if (rc) return rc;
    const Workspace ws = carve(base, l);
    const bool lora = R > 0;
    auto record = [&](void* ev) {
        return ev == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(ev), stream) == cudaSuccess;
    };
    if (!record(ev_start)) return RTLYNX_ERR_CUDA;
    if (launch_sparsify(d, X, lora ? L_B : nullptr, ws, di->err_word, stream)) return RTLYNX_ERR_CUDA;
    if (!record(ev_mid)) return RTLYNX_ERR_CUDA;
    if (launch_gemm(d, true, nullptr, W8, lora ? L_A8 : nullptr, ws, Y, 0, di->num_sms, di->err_word, stream,
                    static_cast<const float*>(qw)))
        return RTLYNX_ERR_CUDA;
    return record(ev_end) ? RTLYNX_OK : RTLYNX_ERR_CUDA;
}

int rtlynx_linear_fp8(const void* X, const void* W8, const void* qw, const void* L_A8, const void* L_B, void* Y,
                      int64_t M, int64_t D_in, int64_t D_out, int64_t R, void* stream_) {
    return rtlynx_linear_fp8_events(X, W8, qw, L_A8, L_B, Y, M, D_in, D_out, R, nullptr, nullptr, nullptr, stream_);
}

int rtlynx_sparsify_fp8_debug(const void* X, int64_t M, int64_t D_in, void* codes, void* meta, void* qx,
                              void* stream_) {
    int rc = validate_fp8(M, D_in, 8, 0);
    if (rc) return rc;
    if (!X || !aligned16(X)) return RTLYNX_ERR_INVALID_ARG;
    DeviceInfo* di = nullptr;
    rc = current_device(&di);
    if (rc) return rc;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const Dims d = make_dims(M, D_in, 8, 0, di->num_sms, true);
    const WsLayout l = make_ws_layout(d);
    void* base = nullptr;
    rc = cached_workspace(dev, stream, l.total, &base);
    if (rc) return rc;
    const Workspace ws = carve(base, l);
    if (launch_sparsify(d, X, nullptr, ws, di->err_word, stream)) return RTLYNX_ERR_CUDA;
    return launch_unpack_fp8_debug(d, ws, codes, meta, qx, stream) ? RTLYNX_ERR_CUDA : RTLYNX_OK;
}

int rtlynx_linear_host(const void* X_host, const void* W, const void* L_A, const void* L_B, void* Y_host,
                       int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, void* X_dev, void* Y_dev,
                       void* stream_) {
    if (!X_host || !Y_host) return RTLYNX_ERR_INVALID_ARG;
    int rc = validate(X_dev, W, L_A, L_B, Y_dev, M, D_in, D_out, R, mode);
    if (rc) return rc;
    if (X_dev == Y_dev) return RTLYNX_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RTLYNX_ERR_CUDA;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // At most kHostChunks token chunks of at least 512 rows; every chunk but
    // the last is a whole number of 256-row blocks, so all of them fit the
    // workspace the first one sizes.
    int64_t n = M / 512;
    n = n < 1 ? 1 : (n > kHostChunks ? kHostChunks : n);
    const int64_t chunk = ((M + n - 1) / n + 255) / 256 * 256;
    n = (M + chunk - 1) / chunk;
    std::lock_guard<std::mutex> lock(g_host_mutex);  // the helper streams and events are shared per device
    HostPipe* hp = nullptr;
    rc = host_pipe(dev, &hp);
    if (rc) return rc;
    if (cudaEventRecord(hp->ev_fork, stream) != cudaSuccess || cudaStreamWaitEvent(hp->up, hp->ev_fork, 0) != cudaSuccess)
        return RTLYNX_ERR_CUDA;
    auto first = [&](int64_t i) { return i * chunk; };
    auto rows = [&](int64_t i) { return (i + 1 < n ? chunk : M - i * chunk); };
    const uint8_t* xh = static_cast<const uint8_t*>(X_host);
    uint8_t* yh = static_cast<uint8_t*>(Y_host);
    uint8_t* xd = static_cast<uint8_t*>(X_dev);
    uint8_t* yd = static_cast<uint8_t*>(Y_dev);
    const size_t xrow = static_cast<size_t>(D_in) * 2, yrow = static_cast<size_t>(D_out) * 2;
    for (int64_t i = 0; i < n && rc == RTLYNX_OK; ++i) {
        const size_t off = static_cast<size_t>(first(i)) * xrow, bytes = static_cast<size_t>(rows(i)) * xrow;
        if (cudaMemcpyAsync(xd + off, xh + off, bytes, cudaMemcpyHostToDevice, hp->up) != cudaSuccess ||
            cudaEventRecord(hp->ev_h2d[i], hp->up) != cudaSuccess)
            rc = RTLYNX_ERR_CUDA;
    }
    int64_t issued = 0;  // chunks whose compute is queued
    for (int64_t i = 0; i < n && rc == RTLYNX_OK; ++i) {
        if (cudaStreamWaitEvent(stream, hp->ev_h2d[i], 0) != cudaSuccess) {
            rc = RTLYNX_ERR_CUDA;
            break;
        }
        rc = rtlynx_linear(xd + static_cast<size_t>(first(i)) * xrow, W, L_A, L_B,
                           yd + static_cast<size_t>(first(i)) * yrow, rows(i), D_in, D_out, R, mode, stream_);
        if (rc) break;
        if (cudaEventRecord(hp->ev_comp[i], stream) != cudaSuccess ||
            cudaStreamWaitEvent(hp->down, hp->ev_comp[i], 0) != cudaSuccess ||
            cudaMemcpyAsync(yh + static_cast<size_t>(first(i)) * yrow, yd + static_cast<size_t>(first(i)) * yrow,
                            static_cast<size_t>(rows(i)) * yrow, cudaMemcpyDeviceToHost, hp->down) != cudaSuccess) {
            rc = RTLYNX_ERR_CUDA;
            break;
        }
        ++issued;
    }
    // join: whatever was queued on the helper streams finishes before later work on `stream`
    if (cudaEventRecord(hp->ev_join_up, hp->up) != cudaSuccess ||
        cudaEventRecord(hp->ev_join_down, hp->down) != cudaSuccess ||
        cudaStreamWaitEvent(stream, hp->ev_join_up, 0) != cudaSuccess ||
        cudaStreamWaitEvent(stream, hp->ev_join_down, 0) != cudaSuccess)
        return RTLYNX_ERR_CUDA;
    (void)issued;
    return rc;
}

int rtlynx_schedule_info(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int num_sms, rtlynx_schedule* out) {
    if (!out || M <= 0 || D_in <= 0 || D_out <= 0 || R < 0 || D_in % 8 || D_out % 8 || num_sms < 2 ||
        num_sms > 1024)
        return RTLYNX_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) - 2 * kBM || D_in > (int64_t(1) << 30) || D_out > (int64_t(1) << 30))
        return RTLYNX_ERR_UNSUPPORTED;
    const Dims d = make_dims(M, D_in, D_out, R, num_sms);
    out->prologue_ctas = d.grid1;
    out->prologue_tiles = d.m_blocks * d.kt2;
    out->prologue_max_segs = d.max_segs;
    out->row_blocks = d.m_blocks;
    out->k_tiles_per_block = d.kt2;
    out->gemm_pairs = d.gemm_pairs;
    out->gemm_tiles = d.gemm_tiles;
    out->tail_full = d.tail_full;
    out->tail_split = d.tail_split;
    out->tail_units = d.tail_units;
    out->k_stages = sparse_k_stages(d);
    out->lora_stages = sparse_lora_stages(d);
    out->small_path = small_path_fits(d, num_sms) ? 1 : 0;
    return RTLYNX_OK;
}

int rtlynx_kernel_launches(int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode) {
    if (mode == RTLYNX_MODE_DENSE_SKIP) return (M > 0 && D_in > 0 && D_out > 0) ? 1 : 0;
    if (mode != RTLYNX_MODE_SPARSE || M <= 0 || D_in <= 0 || D_out <= 0 || R < 0 || D_in % 8 || D_out % 8) return 0;
    DeviceInfo* di = nullptr;
    const int sms = current_device(&di) == RTLYNX_OK ? di->num_sms : 148;
    // one kernel for small problems; else the streaming sparsify pass, the scale pass and the GEMM
    return small_path_fits(make_dims(M, D_in, D_out, R, sms), sms) ? 1 : 3;
}

int rtlynx_wait_selftest(int64_t limit_ns, void* stream_) {
    if (limit_ns <= 0 || limit_ns > 1000000000) return RTLYNX_ERR_INVALID_ARG;
    DeviceInfo* di = nullptr;
    int rc = current_device(&di);
    if (rc) return rc;
    return launch_wait_selftest(di->err_word, static_cast<uint64_t>(limit_ns), static_cast<cudaStream_t>(stream_))
               ? RTLYNX_ERR_CUDA
               : RTLYNX_OK;
}

int rtlynx_stream_status(void* stream_) {
    DeviceInfo* di = nullptr;
    int rc = current_device(&di);
    if (rc) return rc;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream_)) != cudaSuccess) return RTLYNX_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, di->err_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RTLYNX_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(di->err_word, 0, sizeof(int)) != cudaSuccess) return RTLYNX_ERR_CUDA;
        return RTLYNX_ERR_DEVICE_TIMEOUT;
    }
    return RTLYNX_OK;
}

const char* rtlynx_status_string(int status) {
    switch (status) {
        case RTLYNX_OK: return "ok";
        case RTLYNX_ERR_INVALID_ARG: return "invalid argument";
        case RTLYNX_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case RTLYNX_ERR_CUDA: return "CUDA call failed";
        case RTLYNX_ERR_OOM: return "out of device memory";
        case RTLYNX_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

void rtlynx_release(void) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto& kv : g_ws) {
        if (kv.second.ptr) {
            cudaSetDevice(kv.first.dev);
            cudaDeviceSynchronize();
            cudaFree(kv.second.ptr);
        }
    }
    g_ws.clear();
    {
        std::lock_guard<std::mutex> hl(g_host_mutex);
        for (int i = 0; i < kMaxDevices; ++i) {
            HostPipe& hp = g_host[i];
            if (!hp.ready) continue;
            cudaSetDevice(i);
            cudaStreamSynchronize(hp.up);
            cudaStreamSynchronize(hp.down);
            cudaStreamDestroy(hp.up);
            cudaStreamDestroy(hp.down);
            cudaEventDestroy(hp.ev_fork);
            cudaEventDestroy(hp.ev_join_up);
            cudaEventDestroy(hp.ev_join_down);
            for (int c = 0; c < kHostChunks; ++c) {
                cudaEventDestroy(hp.ev_h2d[c]);
                cudaEventDestroy(hp.ev_comp[c]);
            }
            hp = HostPipe{};
        }
    }
    // the error words are module variables: nothing to free
    for (int i = 0; i < kMaxDevices; ++i) g_dev[i] = DeviceInfo{};
    cudaSetDevice(cur);
}

}  // extern "C"
