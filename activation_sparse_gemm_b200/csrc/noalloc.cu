// rtlynx_linear_noalloc: the linear layer for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// a serving engine that has already handed the whole device memory to its own
// pool, code whose allocations must go through an allocator this library does
// not see, or a latency-critical path where cudaMalloc (which may synchronize
// the device) is not acceptable.  This entry point allocates nothing.  Its
// scratch workspace is a file-scope device array of kNoAllocBytes; every GPU
// that loads this part of the library holds it until the process exits.
//
// The array's name is only a host-side stand-in in host code.  Its device
// address is looked up once per device with cudaGetSymbolAddress, with that
// device current, the first time this entry point runs on the device; make
// that first call outside any stream capture.  All calls share the one array
// and it keeps the last call's contents: every region the kernels read is
// rewritten by the same call before it is read, so nothing needs clearing,
// but calls that overlap on the GPU (different streams, or different host
// threads on the same device) race on the array and must be serialized by the
// caller.
#include <mutex>

#include "../../include/rtlynx.h"
#include "internal.h"

namespace rtlynx {
namespace {

constexpr size_t kNoAllocBytes = RTLYNX_NOALLOC_MAX_BYTES;
constexpr int kMaxNoAllocDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

struct NoAllocDevice {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};

std::mutex g_noalloc_mutex;
NoAllocDevice g_noalloc_dev[kMaxNoAllocDevices];

int noalloc_device(NoAllocDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoAllocDevices) return RTLYNX_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocDevice& nd = g_noalloc_dev[dev];
    if (!nd.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return RTLYNX_ERR_CUDA;
        nd.supported = (major == 10 && minor == 0);
        nd.num_sms = sms;
        if (nd.supported) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
                cudaGetLastError();
                return RTLYNX_ERR_CUDA;
            }
            nd.scratch = ptr;
        }
        nd.ready = true;
    }
    if (!nd.supported) return RTLYNX_ERR_UNSUPPORTED;
    *out = &nd;
    return RTLYNX_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace rtlynx

using namespace rtlynx;

extern "C" int rtlynx_linear_noalloc(const void* X, const void* W, const void* L_A, const void* L_B, void* Y,
                                     int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, int* dev_status,
                                     void* stream_) {
    // argument checks (same rules as rtlynx_linear)
    if (mode != RTLYNX_MODE_SPARSE && mode != RTLYNX_MODE_DENSE_SKIP) return RTLYNX_ERR_INVALID_ARG;
    if (M <= 0 || D_in <= 0 || D_out <= 0 || R < 0 || D_in % 8 || D_out % 8) return RTLYNX_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) - 256 || D_in > (int64_t(1) << 30) || D_out > (int64_t(1) << 30))
        return RTLYNX_ERR_UNSUPPORTED;
    if (!X || !W || !Y || !aligned16(X) || !aligned16(W) || !aligned16(Y)) return RTLYNX_ERR_INVALID_ARG;
    if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return RTLYNX_ERR_INVALID_ARG;
    const bool lora = mode == RTLYNX_MODE_SPARSE && R > 0;
    if (lora) {
        if (!L_A || !L_B || !aligned16(L_A) || !aligned16(L_B)) return RTLYNX_ERR_INVALID_ARG;
        if (R % 8 != 0 || R > 256) return RTLYNX_ERR_UNSUPPORTED;
    }
    NoAllocDevice* nd = nullptr;
    int rc = noalloc_device(&nd);
    if (rc) return rc;
    if (!ensure_tmap_encoder()) return RTLYNX_ERR_CUDA;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const Dims d = make_dims(M, D_in, D_out, lora ? R : 0, nd->num_sms);
    if (mode == RTLYNX_MODE_DENSE_SKIP) {
        Workspace none{};
        return launch_gemm(d, false, X, W, nullptr, none, Y, 0, nd->num_sms, dev_status, stream) ? RTLYNX_ERR_CUDA
                                                                                              : RTLYNX_OK;
    }
    const WsLayout l = make_ws_layout(d);
    if (l.total > kNoAllocBytes) return RTLYNX_ERR_UNSUPPORTED;  // workspace larger than the static array
    const Workspace ws = carve(nd->scratch, l);
    rc = run_prologue(d, X, lora ? L_B : nullptr, ws, dev_status, nd->num_sms, stream);
    if (rc) return rc;
    if (launch_gemm(d, true, nullptr, W, lora ? L_A : nullptr, ws, Y, 0, nd->num_sms, dev_status, stream))
        return RTLYNX_ERR_CUDA;
    return RTLYNX_OK;
}
