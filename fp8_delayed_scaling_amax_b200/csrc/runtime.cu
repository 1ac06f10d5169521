// Library runtime: thread-local error messages, device checks, the device status word that
// bounded waits report into, the wait timeout, optional per-kernel CUDA-event timing, and
// the stalled-wait test hook.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace fp8dsa {

namespace {

thread_local std::string t_last_error;

std::mutex g_mutex;
int g_cc_major[kMaxDevices];      // 0 = not queried yet
int g_sms[kMaxDevices];
int* g_status_ptr[kMaxDevices];   // device address of g_status on each device
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_pdl{1};

// Per-kernel timing.
struct TimedLaunch {
    cudaEvent_t start, stop;
    double work;
};
std::atomic<bool> g_profile{false};
std::vector<TimedLaunch> g_timed[kNumKinds];
std::vector<cudaEvent_t> g_event_pool;
thread_local cudaEvent_t t_pending_start = nullptr;

cudaEvent_t take_event() {
    // caller holds g_mutex
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

// The status word bounded waits report into (one per device, one per loaded module).
__device__ int g_status;

bool pdl_enabled() { return g_pdl.load() != 0; }

std::atomic<int> g_fold_in_call{1};
bool ring_fold_in_call() { return g_fold_in_call.load() != 0; }

int fail(int code, const std::string& msg) {
    t_last_error = msg;
    return code;
}

void clear_error() { t_last_error.clear(); }

int check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(FP8DSA_ERR_DEVICE, "device index out of range");
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_cc_major[dev] == 0) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess)
            return fail(FP8DSA_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
        g_cc_major[dev] = prop.major;
        g_sms[dev] = prop.multiProcessorCount;
    }
    if (g_cc_major[dev] != 10)
        return fail(FP8DSA_ERR_DEVICE, "fp8dsa kernels are built for sm_100a (compute capability 10.x)");
    return FP8DSA_OK;
}

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    return dev < 0 ? 0 : (dev >= kMaxDevices ? kMaxDevices - 1 : dev);
}

int sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_mutex);
    return g_sms[dev] > 0 ? g_sms[dev] : 148;
}

int wait_ctl(WaitCtl* ctl) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, "cudaGetDevice failed");
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_status_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status);
        if (e != cudaSuccess)
            return fail(FP8DSA_ERR_CUDA, std::string("cudaGetSymbolAddress(status): ") + cudaGetErrorString(e));
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    ctl->status = g_status_ptr[dev];
    ctl->timeout_ns = g_timeout_ns.load();
    return FP8DSA_OK;
}

// Record `e` on `stream`.  Inside a stream capture the record becomes an external event-record
// node of the graph, so every replay of the graph timestamps it again.
void record_event(cudaEvent_t e, cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(e, stream);
}

void launch_begin(int kind, cudaStream_t stream) {
    (void)kind;
    if (!g_profile.load()) return;
    std::lock_guard<std::mutex> lock(g_mutex);
    t_pending_start = take_event();
    record_event(t_pending_start, stream);
}

void launch_end(int kind, cudaStream_t stream, double work) {
    if (!g_profile.load() || t_pending_start == nullptr) return;
    std::lock_guard<std::mutex> lock(g_mutex);
    cudaEvent_t stop = take_event();
    record_event(stop, stream);
    g_timed[kind].push_back({t_pending_start, stop, work});
    t_pending_start = nullptr;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}
}  // namespace

int encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner,
                      int64_t outer, int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_outer,
                      CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (fn == nullptr) return fail(FP8DSA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                                static_cast<cuuint64_t>(batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld), static_cast<cuuint64_t>(bstride)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FP8DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
    return FP8DSA_OK;
}

int check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return FP8DSA_OK;
}

// One block, one thread: wait on a barrier that nothing arrives at.  The bounded wait gives
// up after the timeout and records kStatusWaitDebug.
__global__ void stalled_wait_kernel(WaitCtl ctl) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_wait_bounded(&bar, 0, ctl, &abort_flag, kStatusWaitDebug);
        mbar_arrive(&bar);  // complete the phase so the barrier is left quiescent
    }
    __syncthreads();
}

}  // namespace fp8dsa

using namespace fp8dsa;

extern "C" {

const char* fp8_last_error(void) { return t_last_error.c_str(); }

const char* fp8dsa_version(void) { return "fp8dsa 0.1.0 (sm_100a)"; }

int fp8_set_wait_timeout_ns(uint64_t ns) {
    if (ns == 0) return fail(FP8DSA_ERR_INVALID_ARG, "timeout must be > 0");
    g_timeout_ns.store(ns);
    return FP8DSA_OK;
}

int fp8_get_device_status(cudaStream_t stream, int* status) {
    clear_error();
    if (status == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "status is NULL");
    int rc = check_device();
    if (rc) return rc;
    WaitCtl ctl;
    rc = wait_ctl(&ctl);
    if (rc) return rc;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("sync: ") + cudaGetErrorString(e));
    int v = 0;
    e = cudaMemcpy(&v, ctl.status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("read status: ") + cudaGetErrorString(e));
    const int zero = 0;
    e = cudaMemcpy(ctl.status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("clear status: ") + cudaGetErrorString(e));
    *status = v;
    return FP8DSA_OK;
}

int fp8_debug_stalled_wait(cudaStream_t stream) {
    clear_error();
    int rc = check_device();
    if (rc) return rc;
    WaitCtl ctl;
    rc = wait_ctl(&ctl);
    if (rc) return rc;
    stalled_wait_kernel<<<1, 32, 0, stream>>>(ctl);
    return check_launch("stalled_wait_kernel");
}

int fp8_set_ring_fold_mode(int mode) {
    clear_error();
    if (mode != 0 && mode != 1) return fail(FP8DSA_ERR_INVALID_ARG, "mode must be 0 (fold in the call) or 1 (defer)");
    g_fold_in_call.store(mode == 0 ? 1 : 0);
    return FP8DSA_OK;
}

int fp8_set_gemm_split_k(int splits) {
    clear_error();
    return gemm_set_split_mode(splits);
}

int fp8_set_pdl(int enabled) {
    g_pdl.store(enabled != 0 ? 1 : 0);
    return FP8DSA_OK;
}

int fp8_profiler_enable(int on) {
    g_profile.store(on != 0);
    return FP8DSA_OK;
}

int fp8_profiler_read(int kind, double* total_ms, int64_t* launches, double* work) {
    clear_error();
    if (kind < 0 || kind >= kNumKinds) return fail(FP8DSA_ERR_INVALID_ARG, "kind must be 0 .. 4");
    std::lock_guard<std::mutex> lock(g_mutex);
    double ms_sum = 0.0, work_sum = 0.0;
    int64_t count = 0;
    int rc = FP8DSA_OK;
    const int kinds[2] = {kind == kKindGemm ? kKindGemmPair : kind, kind == kKindGemm ? kKindGemmSingle : -1};
    for (int kk : kinds) {
        if (kk < 0) continue;
        for (auto& t : g_timed[kk]) {
            cudaError_t e = cudaEventSynchronize(t.stop);
            float ms = 0.f;
            if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, t.start, t.stop);
            if (e != cudaSuccess && rc == FP8DSA_OK)
                rc = fail(FP8DSA_ERR_CUDA, std::string("profiler event: ") + cudaGetErrorString(e));
            ms_sum += ms;
            work_sum += t.work;
            ++count;
            g_event_pool.push_back(t.start);
            g_event_pool.push_back(t.stop);
        }
        g_timed[kk].clear();
    }
    if (total_ms) *total_ms = ms_sum;
    if (launches) *launches = count;
    if (work) *work = work_sum;
    return rc;
}

}  // extern "C"
