// linear_forward_fp8 for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they run the
// forward pass.  Examples: plug-ins embedded in a host application that owns the
// device-memory budget and gives them no allocator, and services that must keep a fixed
// device footprint after start-up.  This entry point takes the same arguments as
// linear_forward_fp8 except the workspace: its scratch (the x8 / w8 operand buffers and the
// amax scratch) lives in one file-scope __device__ array of FP8DSA_NOALLOC_WORKSPACE_BYTES,
// which every GPU that loads the library holds until the process exits.
//
// Set-up: the first call on each device looks up that array's device address with
// cudaGetSymbolAddress, with that device current, and caches it for the life of the process;
// make that first call before any stream capture.  The cached address belongs to the device
// context that first call saw: after cudaDeviceReset (or a primary context released and
// created again) the library must not be called again in the same process.
//
// Afterwards the call enqueues what linear_forward_fp8 enqueues, except that its GEMM never
// splits K (the array holds only the operand buffers and the scale scratch), and it
// allocates nothing.  Every call shares the one array, which keeps the last call's contents:
// the operand buffers are rewritten in full by each call and the dynamic-scaling amax scratch
// is cleared by each call, but calls that overlap on the GPU (different streams without
// ordering between them) race on the array.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "internal.h"

namespace fp8dsa {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_workspace[FP8DSA_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices];

// Device address of the array on the current device (looked up once per device).
int noalloc_workspace(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(FP8DSA_ERR_DEVICE, "device index out of range");
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
        if (e != cudaSuccess || p == nullptr)
            return fail(FP8DSA_ERR_CUDA, std::string("cudaGetSymbolAddress(no-alloc workspace): ") + cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return FP8DSA_OK;
}

}  // namespace
}  // namespace fp8dsa

using namespace fp8dsa;

extern "C" int linear_forward_fp8_noalloc(const void* x, const void* w, int w_is_fp8, const float* w_step,
                                          const void* bias, const float* bias_scale, int64_t m, int64_t k,
                                          int64_t n, fp8_fmt_t fmt, const fp8_ring_t* x_ring,
                                          const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                                          float* sw_used, void* y, cudaStream_t stream) {
    clear_error();
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    // m * k and n * k must not wrap before they are compared with the array's size
    constexpr int64_t kCap = static_cast<int64_t>(FP8DSA_NOALLOC_WORKSPACE_BYTES);
    if (k > 0 && (m > kCap / k || n > kCap / k))
        return fail(FP8DSA_ERR_WORKSPACE, "linear_forward_fp8_noalloc: m * k or n * k exceeds the built-in array (" +
                                              std::to_string(kCap) + " bytes)");
    const size_t need = linear_forward_base_workspace(m, k, n);
    if (need > static_cast<size_t>(FP8DSA_NOALLOC_WORKSPACE_BYTES))
        return fail(FP8DSA_ERR_WORKSPACE, "linear_forward_fp8_noalloc: this shape needs " + std::to_string(need) +
                                              " bytes of scratch; the built-in array holds " +
                                              std::to_string(static_cast<size_t>(FP8DSA_NOALLOC_WORKSPACE_BYTES)));
    int rc = check_device();
    if (rc) return rc;
    void* ws = nullptr;
    rc = noalloc_workspace(&ws);
    if (rc) return rc;
    // the GEMM runs without split-K: the built-in array holds only the operand buffers
    return linear_forward_impl(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                               sx_used, sw_used, nullptr, nullptr, nullptr, nullptr, fmt, ws,
                               static_cast<size_t>(FP8DSA_NOALLOC_WORKSPACE_BYTES), false, y, stream);
}
