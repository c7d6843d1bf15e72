// q4_quantize kernel: f32 W[N,K] -> 4-bit codes + binary16 group scales.
//
// Format (QORA-4B thread, section "量化与内存管理"; QORA-LLM-0.8B model card,
// section "Weight Format": 4-bit symmetric, group size 32, one scale per group;
// divisor 7, ties-to-even rounding, code + 8, low nibble = even k as q4.h states).
//
// Work layout.  Because K % 32 == 0, the flat f32 index space splits into whole
// groups, so a group's flat index equals its scale index and float4 number v
// owns packed bytes 2v and 2v+1.  One thread takes one float4 (4 weights); the
// 8 consecutive lanes holding one group reduce |w|max and the non-finite flag
// with three xor shuffles.  A warp reads 512 contiguous bytes per load and
// writes 64 contiguous bytes of codes.  Each thread handles UNROLL float4s per
// iteration of a grid-stride loop so that several 16-byte loads are in flight.
//
// Bit-exactness: the amax is exact; amax/7 and w/scale use the IEEE
// round-to-nearest division (__fdiv_rn); the binary16 cast is cvt.rn.f16.f32
// (round to nearest even, subnormals kept); the code uses cvt.rni (ties to even).
// The library is compiled without flush-to-zero or fast-math.
#include "q4_common.cuh"

namespace q4 {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ float4 load_stream(const float4* p)
{
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t code_of(float w, float sf)
{
    int q = __float2int_rn(__fdiv_rn(w, sf));
    q = min(max(q, -8), 7);
    return (uint32_t)(q + 8);
}

__global__ void __launch_bounds__(kThreads)
quantize_kernel(const float4* __restrict__ W, long long nvec, uint16_t* __restrict__ packed16,
                uint16_t* __restrict__ scales, uint32_t* __restrict__ flags)
{
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long v0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
         v0 - lane < nvec;                                  // warp-uniform trip count
         v0 += stride * kUnroll) {
        float4 w[kUnroll];
        bool act[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long v = v0 + u * stride;
            act[u] = v < nvec;                              // uniform within each 8-lane group
            w[u] = act[u] ? load_stream(W + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float4 e = w[u];
            float amax = fmaxf(fmaxf(fabsf(e.x), fabsf(e.y)), fmaxf(fabsf(e.z), fabsf(e.w)));
            int bad = !(isfinite(e.x) && isfinite(e.y) && isfinite(e.z) && isfinite(e.w));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                bad |= __shfl_xor_sync(0xffffffffu, bad, o);
            }
            const __half hs = __float2half_rn(__fdiv_rn(amax, 7.0f));
            const uint16_t sbits = __half_as_ushort(hs);
            const bool overflow = (sbits & 0x7FFFu) == 0x7C00u;
            const bool zero_group = bad || overflow || (sbits & 0x7FFFu) == 0;
            uint32_t out = 0x8888u;
            if (!zero_group) {
                const float sf = __half2float(hs);
                out = code_of(e.x, sf) | (code_of(e.y, sf) << 4) | (code_of(e.z, sf) << 8) |
                      (code_of(e.w, sf) << 12);
            }
            const long long v = v0 + u * stride;
            if (act[u]) {
                packed16[v] = (uint16_t)out;
                if ((lane & 7) == 0) {
                    scales[v >> 3] = zero_group ? (uint16_t)0 : sbits;
                    if (flags && (bad || overflow))
                        atomicOr(flags, bad ? Q4_FLAG_NONFINITE : Q4_FLAG_SCALE_OVERFLOW);
                }
            }
        }
    }
}

}  // namespace

q4_status launch_quantize(const float* W, int64_t N, int64_t K, uint8_t* packed, uint16_t* scales,
                          uint32_t* flags, cudaStream_t stream, const DeviceInfo& dev)
{
    const long long nvec = (long long)N * (K / 4);
    long long blocks = (nvec + (long long)kThreads * kUnroll - 1) / ((long long)kThreads * kUnroll);
    const long long cap = (long long)dev.sm_count * 8;      // 8 resident blocks of 256 per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, quantize_kernel, reinterpret_cast<const float4*>(W), nvec,
                                         reinterpret_cast<uint16_t*>(packed), scales, flags);
    return err == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
