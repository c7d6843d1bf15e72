// Shared declarations of the CUDA library (internal; not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "q4.h"

namespace q4 {

struct DeviceInfo {
    int device;
    int sm_count;
    int cc_major;
    int cc_minor;
    int max_smem_optin;     // bytes of dynamic shared memory one block may opt into
    int l2_bytes;
};

// Attributes of the current device, cached per device id.  Returns Q4_ERR_CUDA on
// failure and Q4_ERR_UNSUPPORTED_DEVICE when the device is not sm_100.
q4_status current_device(DeviceInfo* out);

// Launch wrappers (defined next to their kernels).  Arguments are already
// validated by the ABI layer.
q4_status launch_quantize(const float* W, int64_t N, int64_t K, uint8_t* packed, uint16_t* scales,
                          uint32_t* flags, cudaStream_t stream, const DeviceInfo& dev);

struct GemvPlan {
    int kernel;             // which GEMV kernel family serves the shape
    int splits;             // K splits across thread blocks (1 = none)
    int groups_per_split;   // 32-wide groups of K each split covers
    int row_blocks;         // blocks of rows
    int grid_x;             // thread blocks per split
    int chunk;              // groups per work unit
    int xcap;               // groups of x staged in shared memory at once
    int smem_bytes;         // dynamic shared memory per block
    size_t workspace_bytes; // partial sums + counters (0 when splits == 1)
    int has_int8;           // TMA kernel: some matrix holds INT8 codes
    int block_warps;        // TMA kernel: warps per block (>= chunk * xcap; the rest only stage x)
};

// Chooses the kernels for one or more weight matrices sharing x (all N > 0).
// With sizing_only the pointers are not looked at: the plan assumes pointers the TMA
// kernels accept and reports the largest workspace either kernel family may need.
bool plan_gemv(int64_t M, const q4_weight* mats, int count, int64_t K, q4_dtype xt, const DeviceInfo& dev,
               bool sizing_only, GemvPlan* plan);
q4_status launch_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const q4_weight* mats, int count,
                      uint32_t flags, void* workspace, const GemvPlan& plan, cudaStream_t stream);

bool tma_gemv_eligible(int64_t M, int64_t K, q4_dtype xt, const void* packed, const void* scales);
// Row-block epilogues of the TMA GEMV.  Fuse: mats are gate and up of equal N and the
// kernel writes silu(x.gate^T) * (x.up^T) into mats[0].y.  Argmax / top-k: one matrix
// (mats[0].y may be null), greedy argmax or the k largest logits per x row.  Every
// epilogue but the plain one needs whole sums, so K is never split for them.
enum GemvEpilogue { kGemvPlain = 0, kGemvFuse = 1, kGemvArgmax = 2, kGemvTopk = 3 };

// Argmax / top-k outputs of a TMA GEMV launch (see q4_gemv_argmax, q4_gemv_topk).
struct ArgmaxOut {
    unsigned long long* key;   // argmax: [M] workspace, zero at rest
    unsigned* done;            // workspace block counter, zero at rest
    long long* index;          // [M] (top-k: [M][k])
    float* value;              // [M] (top-k: [M][k]) or null
    unsigned long long* cand;  // top-k: [M][grid_x][k] workspace
    unsigned long long* floor; // top-k: one key of workspace, zero at rest
    int k;                     // top-k list length (1..32)
    unsigned row_base;         // added to every reported row
};

// fmts: per matrix 1 = INT8 codes [N][K] (M == 1, plain epilogue only), 0 = Q4; null = all
// Q4.  allow_split = false keeps K whole (no workspace).
bool plan_gemv_tma(int64_t M, const int64_t* Ns, int count, int64_t K, q4_dtype xt, const DeviceInfo& dev,
                   GemvPlan* plan, int epi = kGemvPlain, const int* fmts = nullptr, bool allow_split = true);
// am: non-null for an argmax or top-k launch.  For an INT8 matrix, mats[i].packed holds its codes.
q4_status launch_gemv_tma(const void* x, q4_dtype xt, int64_t M, int64_t K, const q4_weight* mats, int count,
                          int prefetch, void* workspace, const GemvPlan& plan, cudaStream_t stream,
                          int epi = kGemvPlain, const ArgmaxOut* am = nullptr, const int* fmts = nullptr);

q4_status launch_topk_merge(const float* values, const int64_t* indices, int64_t S, int64_t M, int64_t k,
                            int64_t* out_index, float* out_value, cudaStream_t stream);

q4_status launch_int8_quantize(const float* W, int64_t N, int64_t K, int8_t* codes, uint16_t* scales,
                               uint32_t* flags, cudaStream_t stream, const DeviceInfo& dev);
q4_status launch_int8_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const int8_t* codes,
                           const uint16_t* scales, int64_t N, float* y, cudaStream_t stream, const DeviceInfo& dev);

q4_status launch_f16_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const uint16_t* w, int64_t N, float* y,
                          int prefetch, cudaStream_t stream, const DeviceInfo& dev);

q4_status launch_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed, const uint16_t* scales,
                      int64_t N, uint16_t* y, cudaStream_t stream, const DeviceInfo& dev);

// Resident blocks per SM of kernel `fn` launched with `threads` threads and `smem` bytes
// of dynamic shared memory, after opting the kernel into that much shared memory on the
// current device.  Both the opt-in and the occupancy answer are cached per (device,
// kernel, threads, smem), so a call that repeats a shape makes no CUDA API calls.
// Returns 0 when the configuration cannot run.
int blocks_per_sm(const void* fn, int threads, size_t smem);

// Programmatic dependent launch is on unless the environment sets Q4_NO_PDL=1
// (read once per process; useful under tools that do not follow such launches).
bool pdl_enabled();

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start before its predecessor finishes;
// pdl_wait() blocks until the predecessor has completed and its writes are
// visible, and must precede every global read or write of the kernel.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace q4
