// INT8 weights, the other half of a mixed INT8/INT4 model (QKV-Core thread, section
// "自适应混合量化": the precision-sensitive attention layers in INT8, the feed-forward
// layers in INT4).  The page gives no encoding; the library's format is the Q4 one with
// 8-bit codes, as include/q4.h states:
//   s = binary16(f32(amax) / 127), q = clamp(rint(w / f32(s)), -128, 127) as int8 [N,K],
//   zero group -> codes 0 and scale 0, the same flags as q4_quantize.
//
// int8_quantize_kernel: the Q4 quantiser's layout (one float4 per thread, the 8 lanes of
// a group reduce |w|max with xor shuffles, IEEE divisions, cvt.rn.f16, cvt.rni), writing
// four codes as one 32-bit word.
//
// int8_gemv_kernel: one warp per output row.  Lane l reads the 16 codes
// k = 512 i + 16 l .. +15 with one 16-byte load; a code becomes an exact f32 by placing
// its biased byte (q + 128) under the exponent of 2^23 (one PRMT) and subtracting
// 2^23 + 128 (one FADD); each group of 16 is dotted with x in f32 and scaled by the
// group's scale.  x is staged in shared memory as f32 in the order lane l reads it, so
// the 16-byte shared loads of a warp hit distinct banks.
#include "q4_common.cuh"

namespace q4 {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;
constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

__device__ __forceinline__ float4 load_stream_f4(const float4* p)
{
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 load_stream_u4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t code8(float w, float sf)
{
    int q = __float2int_rn(__fdiv_rn(w, sf));
    q = min(max(q, -128), 127);
    return (uint32_t)q & 0xFFu;
}

__global__ void __launch_bounds__(kQuantThreads)
int8_quantize_kernel(const float4* __restrict__ W, long long nvec, uint32_t* __restrict__ codes32,
                     uint16_t* __restrict__ scales, uint32_t* __restrict__ flags)
{
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long v0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
         v0 - lane < nvec;                                  // warp-uniform trip count
         v0 += stride * kQuantUnroll) {
        float4 w[kQuantUnroll];
        bool act[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const long long v = v0 + u * stride;
            act[u] = v < nvec;                              // uniform within each 8-lane group
            w[u] = act[u] ? load_stream_f4(W + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const float4 e = w[u];
            float amax = fmaxf(fmaxf(fabsf(e.x), fabsf(e.y)), fmaxf(fabsf(e.z), fabsf(e.w)));
            int bad = !(isfinite(e.x) && isfinite(e.y) && isfinite(e.z) && isfinite(e.w));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                bad |= __shfl_xor_sync(0xffffffffu, bad, o);
            }
            const __half hs = __float2half_rn(__fdiv_rn(amax, 127.0f));
            const uint16_t sbits = __half_as_ushort(hs);
            const bool overflow = (sbits & 0x7FFFu) == 0x7C00u;
            const bool zero_group = bad || overflow || (sbits & 0x7FFFu) == 0;
            uint32_t out = 0u;
            if (!zero_group) {
                const float sf = __half2float(hs);
                out = code8(e.x, sf) | (code8(e.y, sf) << 8) | (code8(e.z, sf) << 16) | (code8(e.w, sf) << 24);
            }
            const long long v = v0 + u * stride;
            if (act[u]) {
                codes32[v] = out;
                if ((lane & 7) == 0) {
                    scales[v >> 3] = zero_group ? (uint16_t)0 : sbits;
                    if (flags && (bad || overflow))
                        atomicOr(flags, bad ? Q4_FLAG_NONFINITE : Q4_FLAG_SCALE_OVERFLOW);
                }
            }
        }
    }
}

// Code j (0..3) of the 32-bit word t of biased codes (q + 128), as an exact f32.
__device__ __forceinline__ float code_f32(uint32_t t, int j)
{
    return __uint_as_float(__byte_perm(t, 0x4B000000u, 0x7650u + j)) - 8388736.0f;   // 2^23 + 128
}

// x staged as f32 [M][4][K/16]: float4 (c, b) holds x[m][16 b + 4 c .. + 3], so lane l's
// c-th float4 of its 16 values sits at c * (K/16) + (32 i + l).
template <int MAXM>
__global__ void __launch_bounds__(kGemvThreads)
int8_gemv_kernel(const void* __restrict__ x, int x_bf16, int M, int K, const int8_t* __restrict__ codes,
                 const uint16_t* __restrict__ scales, int N, float* __restrict__ y)
{
    extern __shared__ float4 xs[];
    const int K16 = K >> 4;
    for (int i = threadIdx.x; i < M * K16 * 4; i += blockDim.x) {
        const int m = i / (K16 * 4), r = i - m * K16 * 4;
        const int c = r / K16, b = r - c * K16;
        const size_t k = (size_t)m * K + 16 * b + 4 * c;
        float4 v;
        if (x_bf16) {
            const uint16_t* xb = reinterpret_cast<const uint16_t*>(x) + k;
            v = make_float4(__uint_as_float((uint32_t)xb[0] << 16), __uint_as_float((uint32_t)xb[1] << 16),
                            __uint_as_float((uint32_t)xb[2] << 16), __uint_as_float((uint32_t)xb[3] << 16));
        } else {
            const float* xf = reinterpret_cast<const float*>(x) + k;
            v = make_float4(xf[0], xf[1], xf[2], xf[3]);
        }
        xs[i] = v;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = K >> 5;
    for (int n = blockIdx.x * kGemvWarps + warp; n < N; n += gridDim.x * kGemvWarps) {
        float acc[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        const int8_t* row = codes + (size_t)n * K;
        for (int b = lane; b < K16; b += 32) {                       // b: this lane's block of 16 codes
            const uint4 w = load_stream_u4(row + 16 * b);
            const float s = __half2float(__ushort_as_half(__ldg(scales + (size_t)n * G + (b >> 1))));
            const uint32_t words[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
            float q[16];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j) q[4 * c + j] = code_f32(words[c], j);
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M) {
                    float d = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float4 xv = xs[(size_t)m * K16 * 4 + (size_t)c * K16 + b];
                        d = fmaf(q[4 * c + 0], xv.x, d);
                        d = fmaf(q[4 * c + 1], xv.y, d);
                        d = fmaf(q[4 * c + 2], xv.z, d);
                        d = fmaf(q[4 * c + 3], xv.w, d);
                    }
                    acc[m] = fmaf(s, d, acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m < M) {
                float v = acc[m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) y[(size_t)m * N + n] = v;
            }
        }
    }
}

template <int MAXM>
q4_status launch_int8_gemv_t(const void* x, int x_bf16, int64_t M, int64_t K, const int8_t* codes,
                             const uint16_t* scales, int64_t N, float* y, cudaStream_t stream,
                             const DeviceInfo& dev)
{
    const size_t smem = (size_t)M * K * sizeof(float);
    const void* fn = reinterpret_cast<const void*>(&int8_gemv_kernel<MAXM>);
    const int per_sm = blocks_per_sm(fn, kGemvThreads, smem);
    if (per_sm < 1) return Q4_ERR_SHAPE;
    long long blocks = (N + kGemvWarps - 1) / kGemvWarps;
    const long long cap = (long long)dev.sm_count * per_sm;
    if (blocks > cap) blocks = cap;
    int8_gemv_kernel<MAXM><<<(unsigned)blocks, kGemvThreads, smem, stream>>>(x, x_bf16, (int)M, (int)K, codes,
                                                                             scales, (int)N, y);
    return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace

q4_status launch_int8_quantize(const float* W, int64_t N, int64_t K, int8_t* codes, uint16_t* scales,
                               uint32_t* flags, cudaStream_t stream, const DeviceInfo& dev)
{
    const long long nvec = (long long)N * (K / 4);
    long long blocks = (nvec + (long long)kQuantThreads * kQuantUnroll - 1) / ((long long)kQuantThreads * kQuantUnroll);
    const long long cap = (long long)dev.sm_count * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    int8_quantize_kernel<<<(unsigned)blocks, kQuantThreads, 0, stream>>>(
        reinterpret_cast<const float4*>(W), nvec, reinterpret_cast<uint32_t*>(codes), scales, flags);
    return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

q4_status launch_int8_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const int8_t* codes,
                           const uint16_t* scales, int64_t N, float* y, cudaStream_t stream, const DeviceInfo& dev)
{
    const int bf = xt == Q4_BF16 ? 1 : 0;
    if (M == 1) return launch_int8_gemv_t<1>(x, bf, M, K, codes, scales, N, y, stream, dev);
    if (M <= 4) return launch_int8_gemv_t<4>(x, bf, M, K, codes, scales, N, y, stream, dev);
    if (M <= 8) return launch_int8_gemv_t<8>(x, bf, M, K, codes, scales, N, y, stream, dev);
    return launch_int8_gemv_t<16>(x, bf, M, K, codes, scales, N, y, stream, dev);
}

}  // namespace q4
