// q4_gemv_noalloc: the decode GEMV for callers that cannot provide a workspace.
//
// q4_gemv splits K across thread blocks for skinny shapes and needs a
// caller-allocated workspace for the partial sums and arrival counters.  Some
// callers have no way to get one: inference runtimes that own all device memory
// through their own pool and give plugins no allocation hook, real-time or
// safety-certified hosts that forbid allocation after start-up, and code that
// runs while another thread captures a CUDA graph in global capture mode, where
// cudaMalloc is an illegal call.  This entry point takes the same inputs and
// outputs but keeps its scratch in one file-scope device array, so it never
// allocates.
//
// Costs and limits:
//  * every GPU that loads this library holds kScratchBytes (1 MiB) of device
//    memory for the array until the process exits;
//  * every call on a device shares the one array and it keeps the last call's
//    contents, so calls that overlap on the GPU (concurrent streams, or the same
//    work from several host threads) race and give wrong results;
//  * shapes whose split needs more scratch than kScratchBytes are rejected with
//    Q4_ERR_WORKSPACE (with 148 SMs no shape with M <= 16 comes near it).
//
// The first call on each device does a one-time set-up with that device
// current: it looks up the array's device address (in host code the array's
// name is only a host-side stand-in, not a device address) and zero-fills it,
// then waits for the device.  That first call must therefore come before any
// stream capture on the device.  A set-up that fails (the call returns
// Q4_ERR_CUDA) is not remembered: the next call on the device tries it again.
#include <mutex>

#include "q4_common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
__device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex[kMaxDevices];
bool g_setup_done[kMaxDevices];          // set only by a set-up that succeeded
void* g_scratch_addr[kMaxDevices];

// Looks up and clears the array on device `dev` (current) unless an earlier call did;
// returns the array's device address, or nullptr when the set-up failed.
void* scratch_of(int dev)
{
    std::lock_guard<std::mutex> lock(g_setup_mutex[dev]);
    if (g_setup_done[dev]) return g_scratch_addr[dev];
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_gemv_scratch);
    if (e == cudaSuccess) e = cudaMemset(p, 0, kScratchBytes);   // the arrival counters must start at zero
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    g_scratch_addr[dev] = p;
    g_setup_done[dev] = true;
    return p;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

}  // namespace

extern "C" q4_status q4_gemv_noalloc(const void* x, q4_dtype x_dtype, int64_t M, int64_t K,
                                     const uint8_t* packed, const uint16_t* scales, int64_t N, float* y,
                                     void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    if (N < 0 || K < 32 || (K % 32) != 0 || N > INT32_MAX || K > INT32_MAX || N > (INT64_C(1) << 62) / K)
        return Q4_ERR_SHAPE;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !packed || !scales || !y) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || misaligned(packed, 16) || misaligned(scales, 2) || misaligned(y, 4))
        return Q4_ERR_ALIGN;

    q4::DeviceInfo dev;
    q4_status st = q4::current_device(&dev);
    if (st != Q4_OK) return st;
    if (dev.device < 0 || dev.device >= kMaxDevices) return Q4_ERR_UNSUPPORTED_DEVICE;
    void* scratch = scratch_of(dev.device);
    if (!scratch) return Q4_ERR_CUDA;

    const q4_weight w = {packed, scales, N, y};
    q4::GemvPlan plan;
    if (!q4::plan_gemv(M, &w, 1, K, x_dtype, dev, false, &plan)) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    if (plan.workspace_bytes > kScratchBytes) return Q4_ERR_WORKSPACE;
    return q4::launch_gemv(x, x_dtype, M, K, &w, 1, 0u, scratch, plan,
                           static_cast<cudaStream_t>(stream));
}
