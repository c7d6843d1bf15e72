// Host-side runtime pieces shared by the kernels: TMA descriptor encoding through
// the driver entry point, and the library's device error word.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "tma.cuh"

namespace q4 {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode()
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
        cudaGetLastError();
}

// Bit 0: a bounded wait inside a kernel ran out (the kernel gave up and returned).
__device__ unsigned g_device_error = 0;

constexpr int kMaxDevices = 64;
std::mutex g_err_mutex;
unsigned* g_err_addr[kMaxDevices];      // set once the lookup has succeeded on the device

// Limit of the kernels' waits for their own TMA copies (see q4_set_consumer_wait_limit).
std::atomic<uint64_t> g_consumer_wait_ns{kWaitLimitNs};

// Occupancy answers already obtained (a handful of kernels x shapes per process).
struct OccEntry {
    int device;
    const void* fn;
    int threads;
    size_t smem;
    int blocks;
};
constexpr int kOccSlots = 256;
OccEntry g_occ[kOccSlots];
int g_occ_used = 0;
std::mutex g_occ_mutex;

// Largest dynamic shared memory each kernel has been opted into, per device.
struct OptIn {
    int device;
    const void* fn;
    size_t smem;
};
OptIn g_optin[kOccSlots];
int g_optin_used = 0;

}  // namespace

int blocks_per_sm(const void* fn, int threads, size_t smem)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(g_occ_mutex);
    for (int i = 0; i < g_occ_used; ++i)
        if (g_occ[i].device == dev && g_occ[i].fn == fn && g_occ[i].threads == threads && g_occ[i].smem == smem)
            return g_occ[i].blocks;
    int o = 0;
    while (o < g_optin_used && !(g_optin[o].device == dev && g_optin[o].fn == fn)) ++o;
    if (o == g_optin_used || g_optin[o].smem < smem) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        if (o == g_optin_used) {
            if (g_optin_used == kOccSlots) return 0;
            g_optin[g_optin_used++] = {dev, fn, smem};
        } else {
            g_optin[o].smem = smem;
        }
    }
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, threads, smem) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (g_occ_used < kOccSlots) g_occ[g_occ_used++] = {dev, fn, threads, smem, blocks};
    return blocks;
}

bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle)
{
    std::call_once(g_encode_once, load_encode);
    if (!g_encode) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

unsigned* device_error_word()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_err_mutex);
    if (!g_err_addr[dev]) {                // a failed lookup is retried by the next call
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_err_addr[dev] = static_cast<unsigned*>(p);
    }
    return g_err_addr[dev];
}

uint64_t consumer_wait_ns() { return g_consumer_wait_ns.load(std::memory_order_relaxed); }

}  // namespace q4

extern "C" uint64_t q4_set_consumer_wait_limit(uint64_t ns)
{
    return q4::g_consumer_wait_ns.exchange(ns);
}

extern "C" q4_status q4_device_error(uint32_t* out, int clear)
{
    if (!out) return Q4_ERR_INVALID_ARG;
    unsigned* p = q4::device_error_word();
    if (!p) return Q4_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    if (clear && v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) {
            cudaGetLastError();
            return Q4_ERR_CUDA;
        }
    }
    *out = v;
    return Q4_OK;
}
