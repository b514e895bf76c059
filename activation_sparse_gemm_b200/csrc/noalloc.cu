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
// rewritten by the same call before it is read (the prologue zeroes the split
// tiles' arrival tickets before the GEMM takes them), so nothing needs
// clearing between calls, but calls that overlap on the GPU (different
// streams, or different host threads on the same device) race on the array
// and must be serialized by the caller.
#include <mutex>

#include "../../include/rtlynx.h"
#include "internal.h"

namespace rtlynx {
namespace {

constexpr size_t kNoAllocBytes = RTLYNX_NOALLOC_MAX_BYTES;
constexpr int kMaxNoAllocDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxNoAllocDevices];  // device address of g_noalloc_scratch, per device

// The scratch array's device address on the current device (looked up once).
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoAllocDevices) return RTLYNX_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return RTLYNX_ERR_CUDA;
        }
        g_noalloc_addr[dev] = ptr;
    }
    *out = g_noalloc_addr[dev];
    return RTLYNX_OK;
}

}  // namespace
}  // namespace rtlynx

using namespace rtlynx;

extern "C" int rtlynx_linear_noalloc(const void* X, const void* W, const void* L_A, const void* L_B, void* Y,
                                     int64_t M, int64_t D_in, int64_t D_out, int64_t R, int mode, int* dev_status,
                                     void* stream_) {
    int rc = validate(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode);
    if (rc) return rc;
    if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return RTLYNX_ERR_INVALID_ARG;
    // the library's own error word when the caller passes none (a module variable: no allocation)
    int num_sms = 0;
    int* lib_err = nullptr;
    rc = device_info(&num_sms, &lib_err);
    if (rc) return rc;
    int* err = dev_status ? dev_status : lib_err;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    if (!ensure_tmap_encoder()) return RTLYNX_ERR_CUDA;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool lora = mode == RTLYNX_MODE_SPARSE && R > 0;
    const Dims d = make_dims(M, D_in, D_out, lora ? R : 0, num_sms);
    if (mode == RTLYNX_MODE_DENSE_SKIP) {
        Workspace none{};
        return launch_gemm(d, false, X, W, nullptr, none, Y, 0, num_sms, err, stream) ? RTLYNX_ERR_CUDA : RTLYNX_OK;
    }
    const WsLayout l = make_ws_layout(d);
    if (l.total > kNoAllocBytes) return RTLYNX_ERR_UNSUPPORTED;  // workspace larger than the static array
    const Workspace ws = carve(scratch, l);
    if (small_path_fits(d, num_sms))
        return launch_small(d, X, W, lora ? L_A : nullptr, lora ? L_B : nullptr, ws, Y, err, stream) ? RTLYNX_ERR_CUDA
                                                                                                  : RTLYNX_OK;
    rc = run_prologue(d, X, lora ? L_B : nullptr, ws, err, num_sms, stream);
    if (rc) return rc;
    if (launch_gemm(d, true, nullptr, W, lora ? L_A : nullptr, ws, Y, 0, num_sms, err, stream))
        return RTLYNX_ERR_CUDA;
    return RTLYNX_OK;
}
