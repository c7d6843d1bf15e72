// Merge of top-k lists (QORA-LLM-0.8B model card, section "Sampling Defaults": top_k 20):
// the k best (value, row) entries over S lists per x row, ordered as the fused LM-head
// top-k orders them.  With an LM head split by rows across devices, each device's
// q4_gemv_topk reports global rows; after the lists are gathered (S = devices) this
// kernel selects the global top k, so only S * k entries per x row cross the links.
#include "q4_common.cuh"
#include "topk.cuh"

namespace q4 {
namespace {

constexpr int kMergeWarps = 4;

// One warp per x row m: candidates (s, j) of lists [S][M][k], 32 per step.  Entries whose
// row lies outside [0, 2^31 - 1) are padding and take no place.
__global__ void __launch_bounds__(kMergeWarps * 32)
topk_merge_kernel(const float* __restrict__ values, const int64_t* __restrict__ indices, int S, int M, int k,
                  int64_t* __restrict__ out_index, float* __restrict__ out_value)
{
    const int lane = threadIdx.x & 31;
    const int m = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    if (m >= M) return;                                   // whole warps leave together
    const int n = S * k;
    unsigned long long list = 0ull;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        unsigned long long key = 0ull;
        if (i < n) {
            const int s = i / k, j = i - s * k;
            const size_t at = ((size_t)s * M + m) * k + j;
            const int64_t r = indices[at];
            if (r >= 0 && r < INT32_MAX) key = argmax_key(values[at], (uint32_t)r);
        }
        topk_insert(list, key, true, k, lane);
    }
    if (lane < k) {
        out_index[(size_t)m * k + lane] = list ? (int64_t)(0xFFFFFFFFu - (uint32_t)list) : -1;
        if (out_value) out_value[(size_t)m * k + lane] = list ? argmax_value(list) : __int_as_float(0x7FC00000);
    }
}

}  // namespace

q4_status launch_topk_merge(const float* values, const int64_t* indices, int64_t S, int64_t M, int64_t k,
                            int64_t* out_index, float* out_value, cudaStream_t stream)
{
    const unsigned blocks = (unsigned)((M + kMergeWarps - 1) / kMergeWarps);
    topk_merge_kernel<<<blocks, kMergeWarps * 32, 0, stream>>>(values, indices, (int)S, (int)M, (int)k, out_index,
                                                               out_value);
    return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
