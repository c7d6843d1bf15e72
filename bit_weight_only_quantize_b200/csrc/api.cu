// C ABI of the library (declared in include/q4.h): argument validation, device
// checks and dispatch to the kernels.  Every argument check happens before the
// first CUDA call, so a bad call returns its status without touching the device.
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "q4_common.cuh"

namespace q4 {

namespace {
constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
DeviceInfo g_info[kMaxDevices];
q4_status g_info_status[kMaxDevices];

void query(int dev)
{
    DeviceInfo d = {};
    d.device = dev;
    q4_status st = Q4_OK;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.l2_bytes, cudaDevAttrL2CacheSize, dev) != cudaSuccess) {
        cudaGetLastError();
        st = Q4_ERR_CUDA;
    } else if (d.cc_major != 10 || d.cc_minor != 0) {
        st = Q4_ERR_UNSUPPORTED_DEVICE;    // the kernels are built for sm_100a only
    }
    g_info[dev] = d;
    g_info_status[dev] = st;
}
}  // namespace

q4_status current_device(DeviceInfo* out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return Q4_ERR_UNSUPPORTED_DEVICE;
    std::call_once(g_once[dev], query, dev);
    *out = g_info[dev];
    return g_info_status[dev];
}

bool pdl_enabled()
{
    static const bool on = [] {
        const char* v = getenv("Q4_NO_PDL");
        return !(v && v[0] != '\0' && strcmp(v, "0") != 0);
    }();
    return on;
}

}  // namespace q4

namespace {

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

// K: positive multiple of 32; N >= 0; both small enough for 32-bit row/group indices.
q4_status check_nk(int64_t N, int64_t K)
{
    if (N < 0 || K < 32 || (K % 32) != 0) return Q4_ERR_SHAPE;
    if (N > INT32_MAX || K > INT32_MAX || N > (INT64_C(1) << 62) / K) return Q4_ERR_SHAPE;
    return Q4_OK;
}

}  // namespace

extern "C" {

int q4_abi_version(void) { return 1; }

const char* q4_status_string(q4_status status)
{
    switch (status) {
    case Q4_OK: return "Q4_OK";
    case Q4_ERR_INVALID_ARG: return "Q4_ERR_INVALID_ARG: a required pointer is NULL or an enum is out of range";
    case Q4_ERR_SHAPE: return "Q4_ERR_SHAPE: K must be a positive multiple of 32, N >= 0, M in range";
    case Q4_ERR_ALIGN: return "Q4_ERR_ALIGN: a pointer violates its documented alignment";
    case Q4_ERR_DTYPE: return "Q4_ERR_DTYPE: unsupported data type";
    case Q4_ERR_WORKSPACE: return "Q4_ERR_WORKSPACE: workspace missing or too small";
    case Q4_ERR_CUDA: return "Q4_ERR_CUDA: a CUDA call or kernel launch failed";
    case Q4_ERR_UNSUPPORTED_DEVICE: return "Q4_ERR_UNSUPPORTED_DEVICE: the current device is not sm_100";
    }
    return "Q4_ERR_UNKNOWN";
}

q4_status q4_quantize(const float* W, int64_t N, int64_t K, uint8_t* packed, uint16_t* scales,
                      uint32_t* flags, void* stream)
{
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (N == 0) return Q4_OK;
    if (!W || !packed || !scales) return Q4_ERR_INVALID_ARG;
    if (misaligned(W, 16) || misaligned(packed, 16) || misaligned(scales, 2) || (flags && misaligned(flags, 4)))
        return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    return q4::launch_quantize(W, N, K, packed, scales, flags, static_cast<cudaStream_t>(stream), dev);
}

namespace {

// Validates a matrix list and keeps the matrices with N > 0.
q4_status collect(const q4_weight* mats, int count, int64_t K, q4_weight* out, int* kept, bool need_pointers)
{
    if (!mats || count < 1 || count > Q4_MULTI_MAX) return Q4_ERR_INVALID_ARG;
    int n = 0;
    for (int i = 0; i < count; ++i) {
        q4_status st = check_nk(mats[i].N, K);
        if (st != Q4_OK) return st;
        if (mats[i].N == 0) continue;
        if (need_pointers) {
            if (!mats[i].packed || !mats[i].scales || !mats[i].y) return Q4_ERR_INVALID_ARG;
            if (misaligned(mats[i].packed, 16) || misaligned(mats[i].scales, 2) || misaligned(mats[i].y, 4))
                return Q4_ERR_ALIGN;
        }
        out[n++] = mats[i];
    }
    *kept = n;
    return Q4_OK;
}

size_t workspace_for(int64_t M, int64_t K, const q4_weight* mats, int count)
{
    q4::DeviceInfo dev;
    if (q4::current_device(&dev) != Q4_OK) return 0;
    size_t need = 0;
    for (q4_dtype t : {Q4_BF16, Q4_F32}) {
        q4::GemvPlan plan;
        if (!q4::plan_gemv(M, mats, count, K, t, dev, true, &plan)) return 0;
        if (plan.workspace_bytes > need) need = plan.workspace_bytes;
    }
    return need;
}

// Validated and planned GEMV call (nothing enqueued yet); n == 0 means nothing to do.
struct GemvCall {
    q4_weight kept[Q4_MULTI_MAX];
    int n;
    q4::GemvPlan plan;
};

q4_status gemv_prepare(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const q4_weight* mats, int count,
                       uint32_t flags, void* workspace, size_t workspace_bytes, GemvCall* call)
{
    call->n = 0;
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    if (K < 32 || (K % 32) != 0 || K > INT32_MAX) return Q4_ERR_SHAPE;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    int n = 0;
    q4_status st = collect(mats, count, K, call->kept, &n, M > 0);
    if (st != Q4_OK) return st;
    if (M == 0 || n == 0) return Q4_OK;
    if (!x) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || (workspace && misaligned(workspace, 16))) return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    if (!q4::plan_gemv(M, call->kept, n, K, x_dtype, dev, false, &call->plan)) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    if (call->plan.workspace_bytes > 0 && (!workspace || workspace_bytes < call->plan.workspace_bytes))
        return Q4_ERR_WORKSPACE;
    call->n = n;
    return Q4_OK;
}

q4_status gemv_common(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const q4_weight* mats, int count,
                      uint32_t flags, void* workspace, size_t workspace_bytes, void* stream)
{
    GemvCall call;
    const q4_status st = gemv_prepare(x, x_dtype, M, K, mats, count, flags, workspace, workspace_bytes, &call);
    if (st != Q4_OK || call.n == 0) return st;
    return q4::launch_gemv(x, x_dtype, M, K, call.kept, call.n, flags, workspace, call.plan,
                           static_cast<cudaStream_t>(stream));
}

}  // namespace

size_t q4_gemv_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || M > Q4_GEMV_MAX_M || N < 1 || check_nk(N, K) != Q4_OK) return 0;
    const q4_weight w = {nullptr, nullptr, N, nullptr};
    return workspace_for(M, K, &w, 1);
}

size_t q4_gemv_multi_workspace_size(int64_t M, int64_t K, const int64_t* Ns, int count)
{
    if (M < 1 || M > Q4_GEMV_MAX_M || !Ns || count < 1 || count > Q4_MULTI_MAX) return 0;
    q4_weight mats[Q4_MULTI_MAX];
    int n = 0;
    for (int i = 0; i < count; ++i) {
        if (check_nk(Ns[i], K) != Q4_OK) return 0;
        if (Ns[i] > 0) mats[n++] = q4_weight{nullptr, nullptr, Ns[i], nullptr};
    }
    return n ? workspace_for(M, K, mats, n) : 0;
}

q4_status q4_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                  const uint16_t* scales, int64_t N, float* y, void* workspace, size_t workspace_bytes,
                  void* stream)
{
    const q4_weight w = {packed, scales, N, y};
    return gemv_common(x, x_dtype, M, K, &w, 1, 0u, workspace, workspace_bytes, stream);
}

q4_status q4_gemv_multi(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const q4_weight* mats, int count,
                        uint32_t flags, void* workspace, size_t workspace_bytes, void* stream)
{
    return gemv_common(x, x_dtype, M, K, mats, count, flags, workspace, workspace_bytes, stream);
}

q4_status q4_gemv_host(const void* x_host, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                       const uint16_t* scales, int64_t N, float* y_host, void* x_dev, float* y_dev, uint32_t flags,
                       void* workspace, size_t workspace_bytes, void* stream)
{
    const q4_weight w = {packed, scales, N, y_dev};
    GemvCall call;
    q4_status st = gemv_prepare(x_dev, x_dtype, M, K, &w, 1, flags, workspace, workspace_bytes, &call);
    if (st != Q4_OK || call.n == 0) return st;
    if (!x_host || !y_host) return Q4_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t x_bytes = (size_t)M * (size_t)K * (x_dtype == Q4_F32 ? 4 : 2);
    const size_t y_bytes = (size_t)M * (size_t)N * sizeof(float);
    if (cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    st = q4::launch_gemv(x_dev, x_dtype, M, K, call.kept, call.n, flags, workspace, call.plan, s);
    if (st != Q4_OK) return st;
    if (cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return Q4_ERR_CUDA;
    }
    return Q4_OK;
}

q4_status q4_gemv_gate_up(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* gate_packed,
                          const uint16_t* gate_scales, const uint8_t* up_packed, const uint16_t* up_scales,
                          int64_t N, float* y, uint32_t flags, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !gate_packed || !gate_scales || !up_packed || !up_scales || !y) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || misaligned(gate_packed, 16) || misaligned(up_packed, 16) ||
        misaligned(gate_scales, 16) || misaligned(up_scales, 16) || misaligned(y, 4))
        return Q4_ERR_ALIGN;
    if (K % 256 != 0 || (M > 1 && x_dtype != Q4_BF16)) return Q4_ERR_SHAPE;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    const q4_weight mats[2] = {{gate_packed, gate_scales, N, y}, {up_packed, up_scales, N, y}};
    const int64_t Ns[2] = {N, N};
    q4::GemvPlan plan;
    if (!q4::plan_gemv_tma(M, Ns, 2, K, x_dtype, dev, &plan, q4::kGemvFuse)) {
        cudaGetLastError();
        return Q4_ERR_SHAPE;                      // x of this K does not fit beside the rings
    }
    return q4::launch_gemv_tma(x, x_dtype, M, K, mats, 2, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0, nullptr, plan,
                               static_cast<cudaStream_t>(stream), q4::kGemvFuse);
}

size_t q4_gemv_argmax_workspace_size(void) { return 256; }   // Q4_GEMV_MAX_M keys, then the counter

q4_status q4_gemv_argmax(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                         const uint16_t* scales, int64_t N, float* y, int64_t* index, float* value,
                         uint32_t flags, void* workspace, size_t workspace_bytes, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !packed || !scales || !index) return Q4_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < q4_gemv_argmax_workspace_size()) return Q4_ERR_WORKSPACE;
    if (misaligned(x, 16) || misaligned(packed, 16) || misaligned(scales, 16) || (y && misaligned(y, 4)) ||
        misaligned(index, 8) || (value && misaligned(value, 4)) || misaligned(workspace, 16))
        return Q4_ERR_ALIGN;
    if (K % 256 != 0 || (M > 1 && x_dtype != Q4_BF16)) return Q4_ERR_SHAPE;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    const q4_weight w = {packed, scales, N, y};
    q4::GemvPlan plan;
    if (!q4::plan_gemv_tma(M, &N, 1, K, x_dtype, dev, &plan, q4::kGemvArgmax)) {
        cudaGetLastError();
        return Q4_ERR_SHAPE;
    }
    q4::ArgmaxOut am;
    am.key = static_cast<unsigned long long*>(workspace);
    am.done = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + Q4_GEMV_MAX_M * 8);
    am.index = reinterpret_cast<long long*>(index);
    am.value = value;
    am.cand = nullptr;
    am.floor = nullptr;
    am.k = 1;
    am.row_base = 0u;
    return q4::launch_gemv_tma(x, x_dtype, M, K, &w, 1, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0, nullptr, plan,
                               static_cast<cudaStream_t>(stream), q4::kGemvArgmax, &am);
}

// Top-k workspace: the block counter at 0, the published k-th key at 8 (both zero at
// rest), then from byte 256 the blocks' lists [M][grid_x][k].
static constexpr size_t kTopkFloorOffset = 8;
static constexpr size_t kTopkListsOffset = 256;

static bool topk_shape(int64_t M, int64_t N, int64_t K, int64_t k, q4_dtype x_dtype)
{
    return M >= 1 && M <= Q4_GEMV_MAX_M && k >= 1 && k <= Q4_TOPK_MAX && N >= 1 && check_nk(N, K) == Q4_OK &&
           K % 256 == 0 && (x_dtype == Q4_BF16 || (x_dtype == Q4_F32 && M == 1));
}

static bool topk_plan(int64_t M, int64_t N, int64_t K, q4_dtype x_dtype, q4::DeviceInfo* dev, q4::GemvPlan* plan)
{
    if (q4::current_device(dev) != Q4_OK) return false;
    if (!q4::plan_gemv_tma(M, &N, 1, K, x_dtype, *dev, plan, q4::kGemvTopk)) {
        cudaGetLastError();
        return false;
    }
    return true;
}

size_t q4_gemv_topk_workspace_size(int64_t M, int64_t N, int64_t K, int64_t k, q4_dtype x_dtype)
{
    q4::DeviceInfo dev;
    q4::GemvPlan plan;
    if (!topk_shape(M, N, K, k, x_dtype) || !topk_plan(M, N, K, x_dtype, &dev, &plan)) return 0;
    return kTopkListsOffset + (size_t)M * (size_t)plan.grid_x * (size_t)k * sizeof(unsigned long long);
}

q4_status q4_gemv_topk(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                       const uint16_t* scales, int64_t N, int64_t k, int64_t row_base, float* y, int64_t* index,
                       float* value, uint32_t flags, void* workspace, size_t workspace_bytes, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (k < 1 || k > Q4_TOPK_MAX || row_base < 0 || row_base > INT32_MAX - N) return Q4_ERR_SHAPE;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !packed || !scales || !index) return Q4_ERR_INVALID_ARG;
    if (!workspace) return Q4_ERR_WORKSPACE;
    if (misaligned(x, 16) || misaligned(packed, 16) || misaligned(scales, 16) || (y && misaligned(y, 4)) ||
        misaligned(index, 8) || (value && misaligned(value, 4)) || misaligned(workspace, 16))
        return Q4_ERR_ALIGN;
    if (!topk_shape(M, N, K, k, x_dtype)) return Q4_ERR_SHAPE;
    q4::DeviceInfo dev;
    q4::GemvPlan plan;
    if (!topk_plan(M, N, K, x_dtype, &dev, &plan)) return Q4_ERR_SHAPE;
    if (workspace_bytes < kTopkListsOffset + (size_t)M * (size_t)plan.grid_x * (size_t)k * 8) return Q4_ERR_WORKSPACE;
    const q4_weight w = {packed, scales, N, y};
    q4::ArgmaxOut am;
    am.key = nullptr;
    am.done = static_cast<unsigned*>(workspace);
    am.index = reinterpret_cast<long long*>(index);
    am.value = value;
    am.cand = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + kTopkListsOffset);
    am.floor = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + kTopkFloorOffset);
    am.k = (int)k;
    am.row_base = (unsigned)row_base;
    return q4::launch_gemv_tma(x, x_dtype, M, K, &w, 1, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0, nullptr, plan,
                               static_cast<cudaStream_t>(stream), q4::kGemvTopk, &am);
}

q4_status q4_topk_merge(const float* values, const int64_t* indices, int64_t S, int64_t M, int64_t k,
                        int64_t* index, float* value, void* stream)
{
    if (S < 1 || S > (1 << 20) || M < 0 || M > INT32_MAX / 4 || k < 1 || k > Q4_TOPK_MAX) return Q4_ERR_SHAPE;
    if (M == 0) return Q4_OK;
    if (!values || !indices || !index) return Q4_ERR_INVALID_ARG;
    if (misaligned(values, 4) || misaligned(indices, 8) || misaligned(index, 8) || (value && misaligned(value, 4)))
        return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    const q4_status st = q4::current_device(&dev);
    if (st != Q4_OK) return st;
    return q4::launch_topk_merge(values, indices, S, M, k, index, value, static_cast<cudaStream_t>(stream));
}

q4_status q4_int8_quantize(const float* W, int64_t N, int64_t K, int8_t* codes, uint16_t* scales,
                           uint32_t* flags, void* stream)
{
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (N == 0) return Q4_OK;
    if (!W || !codes || !scales) return Q4_ERR_INVALID_ARG;
    if (misaligned(W, 16) || misaligned(codes, 16) || misaligned(scales, 2) || (flags && misaligned(flags, 4)))
        return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    return q4::launch_int8_quantize(W, N, K, codes, scales, flags, static_cast<cudaStream_t>(stream), dev);
}

q4_status q4_int8_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const int8_t* codes,
                       const uint16_t* scales, int64_t N, float* y, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !codes || !scales || !y) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || misaligned(codes, 16) || misaligned(scales, 2) || misaligned(y, 4)) return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // M = 1: the TMA kernel's integer path (codes straight into the tensor cores), K whole
    if (M == 1 && K % 256 == 0 && !misaligned(scales, 16)) {
        const int fmt = 1;
        const q4_weight w = {reinterpret_cast<const uint8_t*>(codes), scales, N, y};
        q4::GemvPlan plan;
        if (q4::plan_gemv_tma(M, &N, 1, K, x_dtype, dev, &plan, q4::kGemvPlain, &fmt, false))
            return q4::launch_gemv_tma(x, x_dtype, M, K, &w, 1, 0, nullptr, plan, s, q4::kGemvPlain, nullptr, &fmt);
        cudaGetLastError();
    }
    if ((size_t)M * (size_t)K * sizeof(float) > (size_t)dev.max_smem_optin) return Q4_ERR_SHAPE;
    return q4::launch_int8_gemv(x, x_dtype, M, K, codes, scales, N, y, s, dev);
}

namespace {

// Validates a mixed matrix list: N >= 0, bits 4 or 8, pointers and alignment of the kept
// (N > 0) matrices.
q4_status collect_mixed(const q4_mixed_weight* mats, int count, int64_t K, q4_mixed_weight* out, int* kept)
{
    if (!mats || count < 1 || count > Q4_MULTI_MAX) return Q4_ERR_INVALID_ARG;
    int n = 0;
    for (int i = 0; i < count; ++i) {
        q4_status st = check_nk(mats[i].N, K);
        if (st != Q4_OK) return st;
        if ((mats[i].bits != 4 && mats[i].bits != 8) || mats[i].reserved != 0) return Q4_ERR_INVALID_ARG;
        if (mats[i].N == 0) continue;
        if (!mats[i].codes || !mats[i].scales || !mats[i].y) return Q4_ERR_INVALID_ARG;
        if (misaligned(mats[i].codes, 16) || misaligned(mats[i].scales, 2) || misaligned(mats[i].y, 4))
            return Q4_ERR_ALIGN;
        out[n++] = mats[i];
    }
    *kept = n;
    return Q4_OK;
}

// One launch for every matrix: M == 1, K % 256 == 0, 16-byte aligned x and scales.
bool mixed_single_launch(int64_t M, int64_t K, const void* x, const q4_mixed_weight* mats, int n)
{
    if (M != 1 || K % 256 != 0 || misaligned(x, 16)) return false;
    for (int i = 0; i < n; ++i)
        if (misaligned(mats[i].scales, 16)) return false;
    return true;
}

}  // namespace

size_t q4_gemv_mixed_workspace_size(int64_t M, int64_t K, const q4_mixed_weight* mats, int count)
{
    if (M < 1 || M > Q4_GEMV_MAX_M || !mats || count < 1 || count > Q4_MULTI_MAX) return 0;
    q4::DeviceInfo dev;
    if (q4::current_device(&dev) != Q4_OK) return 0;
    int64_t Ns[Q4_MULTI_MAX];
    int fmts[Q4_MULTI_MAX];
    q4_weight q4m[Q4_MULTI_MAX];
    int n = 0, nq = 0;
    for (int i = 0; i < count; ++i) {
        if (check_nk(mats[i].N, K) != Q4_OK) return 0;
        if (mats[i].N == 0) continue;
        Ns[n] = mats[i].N;
        fmts[n++] = mats[i].bits == 8 ? 1 : 0;
        if (mats[i].bits != 8) q4m[nq++] = q4_weight{nullptr, nullptr, mats[i].N, nullptr};
    }
    size_t need = 0;
    q4::GemvPlan plan;
    if (n && M == 1 && K % 256 == 0 && q4::plan_gemv_tma(M, Ns, n, K, Q4_BF16, dev, &plan, q4::kGemvPlain, fmts))
        need = plan.workspace_bytes;
    if (n && M == 1 && K % 256 == 0 && q4::plan_gemv_tma(M, Ns, n, K, Q4_F32, dev, &plan, q4::kGemvPlain, fmts) &&
        plan.workspace_bytes > need)
        need = plan.workspace_bytes;
    if (nq) {                                  // the Q4 matrices in their own launch
        const size_t q = workspace_for(M, K, q4m, nq);
        if (q > need) need = q;
    }
    return need;
}

q4_status q4_gemv_mixed(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const q4_mixed_weight* mats,
                        int count, uint32_t flags, void* workspace, size_t workspace_bytes, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M) return Q4_ERR_SHAPE;
    if (K < 32 || (K % 32) != 0 || K > INT32_MAX) return Q4_ERR_SHAPE;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    q4_mixed_weight kept[Q4_MULTI_MAX];
    int n = 0;
    q4_status st = collect_mixed(mats, count, K, kept, &n);
    if (st != Q4_OK) return st;
    if (M == 0 || n == 0) return Q4_OK;
    if (!x) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || (workspace && misaligned(workspace, 16))) return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    q4_weight w[Q4_MULTI_MAX];
    int64_t Ns[Q4_MULTI_MAX];
    int fmts[Q4_MULTI_MAX];
    for (int i = 0; i < n; ++i) {
        w[i] = q4_weight{reinterpret_cast<const uint8_t*>(kept[i].codes), kept[i].scales, kept[i].N, kept[i].y};
        Ns[i] = kept[i].N;
        fmts[i] = kept[i].bits == 8 ? 1 : 0;
    }
    if (mixed_single_launch(M, K, x, kept, n)) {
        q4::GemvPlan plan;
        if (q4::plan_gemv_tma(M, Ns, n, K, x_dtype, dev, &plan, q4::kGemvPlain, fmts)) {
            if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes))
                return Q4_ERR_WORKSPACE;
            return q4::launch_gemv_tma(x, x_dtype, M, K, w, n, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0, workspace, plan,
                                       s, q4::kGemvPlain, nullptr, fmts);
        }
        cudaGetLastError();
    }
    // Otherwise: the Q4 matrices in one q4_gemv_multi launch, each INT8 matrix on its own.
    q4_weight q4m[Q4_MULTI_MAX];
    int nq = 0;
    for (int i = 0; i < n; ++i)
        if (!fmts[i]) q4m[nq++] = w[i];
    for (int i = 0; i < n; ++i)           // argument checks of every launch before the first
        if (fmts[i] && (size_t)M * (size_t)K * sizeof(float) > (size_t)dev.max_smem_optin) return Q4_ERR_SHAPE;
    if (nq) {
        GemvCall call;
        st = gemv_prepare(x, x_dtype, M, K, q4m, nq, flags, workspace, workspace_bytes, &call);
        if (st != Q4_OK) return st;
        st = q4::launch_gemv(x, x_dtype, M, K, call.kept, call.n, flags, workspace, call.plan, s);
        if (st != Q4_OK) return st;
    }
    for (int i = 0; i < n; ++i) {
        if (!fmts[i]) continue;
        st = q4_int8_gemv(x, x_dtype, M, K, reinterpret_cast<const int8_t*>(kept[i].codes), kept[i].scales, kept[i].N,
                          kept[i].y, stream);
        if (st != Q4_OK) return st;
    }
    return Q4_OK;
}

q4_status q4_f16_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint16_t* w, int64_t N, float* y,
                      uint32_t flags, void* stream)
{
    if (x_dtype != Q4_F32 && x_dtype != Q4_BF16) return Q4_ERR_DTYPE;
    if (M < 0 || M > Q4_GEMV_MAX_M || (M > 1 && x_dtype != Q4_BF16)) return Q4_ERR_SHAPE;
    if (K < 8 || K % 8 != 0 || K > INT32_MAX || N < 0 || N > INT32_MAX) return Q4_ERR_SHAPE;
    if (flags & ~Q4_WEIGHTS_STATIC) return Q4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !w || !y) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || misaligned(w, 16) || misaligned(y, 4)) return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    q4_status st = q4::current_device(&dev);
    if (st != Q4_OK) return st;
    return q4::launch_f16_gemv(x, x_dtype, M, K, w, N, y, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0,
                               static_cast<cudaStream_t>(stream), dev);
}

q4_status q4_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed, const uint16_t* scales,
                  int64_t N, uint16_t* y, void* stream)
{
    if (M < 0 || M > INT32_MAX) return Q4_ERR_SHAPE;
    q4_status st = check_nk(N, K);
    if (st != Q4_OK) return st;
    if (M == 0 || N == 0) return Q4_OK;
    if (!x || !packed || !scales || !y) return Q4_ERR_INVALID_ARG;
    if (misaligned(x, 16) || misaligned(packed, 16) || misaligned(scales, 2) || misaligned(y, 2))
        return Q4_ERR_ALIGN;
    q4::DeviceInfo dev;
    if ((st = q4::current_device(&dev)) != Q4_OK) return st;
    return q4::launch_gemm(x, M, K, packed, scales, N, y, static_cast<cudaStream_t>(stream), dev);
}

}  // extern "C"
