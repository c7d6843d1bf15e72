// q4_gemv, M = 1, for shapes the TMA path serves (K % 256 == 0, scales 16-byte aligned).
//
// Same arithmetic as the generic kernel in gemv.cu (exact code expansion through
// the float mantissa, packed f32x2 FMAs, per-group scale, f32 accumulation), with
// the data movement rebuilt around the Tensor Memory Accelerator:
//
//  * Weights stream as TMA boxes of 16 rows x 8 groups: 2 KiB of codes (128-byte
//    swizzled) plus 256 B of binary16 scales, into a per-warp ring of kStages
//    stages guarded by mbarriers.  Every warp issues its own boxes (lane 0), so a
//    block keeps warps * kStages boxes in flight without a producer warp.
//  * Two lanes per row: lane r and lane r+16 take words 0-1 and 2-3 of every group
//    of row r, so the 16 lanes of each half work on the same group at the same time
//    and their x values are shared-memory broadcasts (x is staged once per block
//    as f32); the codes come from the swizzled box without bank conflicts.
//  * Work is split into teams of P warps.  A team owns a sequence of 16-row
//    blocks; its P warps take disjoint K ranges of each block and add their
//    partial sums through shared memory in a fixed order.  P = 1 (huge N, e.g. an
//    LM head) needs no barrier at all; skinny N uses larger P and, if needed, a
//    K split across blocks with the last-arriver reduction of gemv.cu.
//  * Every mbarrier wait is bounded.  If one runs out, the kernel records
//    kErrWaitTimeout in the library error word, stops issuing and computing, waits
//    (bounded) for its own copies still in flight and returns; the host reads the
//    word through q4_device_error().
#include "tma.cuh"

namespace q4 {
namespace {

constexpr int kRows = 16;                    // rows per row block; two lanes per row
constexpr int kMaxWarps = 16;
constexpr int kStages = 2;
constexpr uint32_t kCodeBox = kRows * 128;   // bytes of codes per box (8 groups)
constexpr uint32_t kScaleBox = kRows * 16;   // bytes of scales per box
constexpr uint64_t kWaitLimit = kWaitLimitNs;
constexpr int kCounterSlots = 1024;          // must match the generic kernel's workspace layout
constexpr size_t kCounterBytes = kCounterSlots * sizeof(unsigned);

struct TmaGemvArgs {
    const void* x;
    float* y;
    float* partial;        // [splits][N]
    unsigned* counters;    // [row_blocks]
    unsigned* err;
    int N, G;
    int ksg;               // groups per split (multiple of 8)
    int splits;
    int row_blocks;
    int P;                 // warps per team
    int teams;             // teams per block
};

__device__ __forceinline__ void team_sync(int team, int P)
{
    if (P == 1) {
        __syncwarp();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(P * 32) : "memory");
    }
}

// A value the compiler must keep in a register (it cannot rematerialise it as an
// immediate); used for the packed-add constants so they are not rebuilt per use.
__device__ __forceinline__ float pinned(float v)
{
    float r;
    asm volatile("mov.b32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

struct ExpandConsts {
    float2 c01, c23, c45, c67;
};

// Eight codes of one word (nibble p holds weight p) dotted with eight x values:
// nibble p OR-ed into the mantissa of 2^(23-4p) is exactly 2^(23-4p) + code, and one
// packed add of -(2^(23-4p) + 8) leaves code - 8 exactly.
__device__ __forceinline__ float2 word_dot(uint32_t v, const float4* xw, const ExpandConsts& k)
{
    const uint32_t u = v >> 12;
    const float f0 = __uint_as_float((v & 0x0000000Fu) | 0x4B000000u);   // 2^23 + c0
    const float f1 = __uint_as_float((v & 0x000000F0u) | 0x49000000u);   // 2^19 + c1
    const float f2 = __uint_as_float((v & 0x00000F00u) | 0x47000000u);   // 2^15 + c2
    const float f3 = __uint_as_float((v & 0x0000F000u) | 0x45000000u);   // 2^11 + c3
    const float f4 = __uint_as_float((v & 0x000F0000u) | 0x43000000u);   // 2^7  + c4
    const float f5 = __uint_as_float((u & 0x00000F00u) | 0x47000000u);   // 2^15 + c5
    const float f6 = __uint_as_float((u & 0x0000F000u) | 0x45000000u);   // 2^11 + c6
    const float f7 = __uint_as_float((u & 0x000F0000u) | 0x43000000u);   // 2^7  + c7
    const float2 d01 = __fadd2_rn(make_float2(f0, f1), k.c01);
    const float2 d23 = __fadd2_rn(make_float2(f2, f3), k.c23);
    const float2 d45 = __fadd2_rn(make_float2(f4, f5), k.c45);
    const float2 d67 = __fadd2_rn(make_float2(f6, f7), k.c67);
    const float4 xa = xw[0];
    const float4 xb = xw[1];
    float2 acc = __fmul2_rn(make_float2(xa.x, xa.y), d01);
    acc = __ffma2_rn(make_float2(xa.z, xa.w), d23, acc);
    acc = __ffma2_rn(make_float2(xb.x, xb.y), d45, acc);
    acc = __ffma2_rn(make_float2(xb.z, xb.w), d67, acc);
    return acc;
}

// d = a * b + c with bfloat16 a, b (exact product) and f32 c, d: one rounding.
__device__ __forceinline__ float fma_bf16(uint16_t a, uint16_t b, float c)
{
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// bf16 x: sum_j x_j * (128 + code_j) over the 8 weights of one word.  OR-ing the
// nibble pair (j, j+4) into 0x4300 gives the bf16 pair (128 + c_j, 128 + c_{j+4});
// xp holds the matching x pairs (x_j, x_{j+4}).  Every product is exact in f32.
__device__ __forceinline__ float word_dot_bf16(uint32_t v, uint4 xp, float acc)
{
    const uint32_t xs[4] = {xp.x, xp.y, xp.z, xp.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t t = ((v >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
        acc = fma_bf16((uint16_t)(t & 0xFFFFu), (uint16_t)(xs[j] & 0xFFFFu), acc);
        acc = fma_bf16((uint16_t)(t >> 16), (uint16_t)(xs[j] >> 16), acc);
    }
    return acc;
}

template <bool XBF16>
__global__ void __launch_bounds__(kMaxWarps * 32, 2)
gemv_tma_m1_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
                   const TmaGemvArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    __shared__ int s_last[kMaxWarps];
    const int W = blockDim.x >> 5;
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* codes = smem;                                          // [warp][stage][2048]
    unsigned char* scl = codes + W * kStages * kCodeBox;                  // [warp][stage][256]
    uint64_t* bars = reinterpret_cast<uint64_t*>(scl + W * kStages * kScaleBox);   // [warp][stage]
    float* red = reinterpret_cast<float*>(bars + W * kStages);            // [warp][16]
    float* xs = red + W * kRows;                                          // [boxes * 8 groups][32]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane & 15, h = lane >> 4;                              // row of the block, half of each group
    const int P = a.P;
    const int team = warp / P, wt = warp - team * P;
    const bool active = team < a.teams;
    const int split = blockIdx.y;
    const int g0 = split * a.ksg;
    const int ng = min(a.G - g0, a.ksg);
    const int nb = (ng + 7) >> 3;                                         // boxes of this split
    const int b0 = wt * nb / P, nbw = (wt + 1) * nb / P - b0;             // this warp's boxes
    const int first_rb = blockIdx.x * a.teams + team;
    const int rb_stride = gridDim.x * a.teams;
    const int nrb = (active && first_rb < a.row_blocks) ? (a.row_blocks - first_rb + rb_stride - 1) / rb_stride : 0;
    const int njobs = nrb * nbw;
    uint64_t* my_bars = bars + warp * kStages;

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
        if (warp == 0) {
            tma_prefetch_desc(&tm_codes);
            tma_prefetch_desc(&tm_scales);
        }
    }
    __syncwarp();
    const ExpandConsts kc = {make_float2(pinned(-8388616.0f), pinned(-524296.0f)),
                             make_float2(pinned(-32776.0f), pinned(-2056.0f)),
                             make_float2(pinned(-136.0f), pinned(-32776.0f)),
                             make_float2(pinned(-2056.0f), pinned(-136.0f))};

    pdl_launch_dependents();
    pdl_wait();

    auto issue = [&](int j) {
        const int s = j % kStages;
        const int rb = first_rb + (j / nbw) * rb_stride;
        const int b = b0 + j % nbw;
        mbar_arrive_expect_tx(&my_bars[s], kCodeBox + kScaleBox);
        tma_load_2d(codes + (warp * kStages + s) * kCodeBox, &tm_codes, (g0 + 8 * b) * 16, rb * kRows, &my_bars[s]);
        tma_load_2d(scl + (warp * kStages + s) * kScaleBox, &tm_scales, g0 + 8 * b, rb * kRows, &my_bars[s]);
    };
    int issued = min(kStages, njobs);
    if (lane == 0)
        for (int j = 0; j < issued; ++j) issue(j);

    // Stage x for this split while the boxes fly (zero past the split / past K).
    //  f32 x : as f32, [group][32].
    //  bf16 x: as bf16 pairs (x_j, x_{j+4}) per 8-element word, [group][4 words][4 pairs],
    //          plus the f32 sum of each half group (16 values, added in f64, rounded once).
    if constexpr (XBF16) {
        uint4* xp = reinterpret_cast<uint4*>(xs);
        for (int i = threadIdx.x; i < nb * 32; i += blockDim.x) {
            const int lg = i >> 2, wd = i & 3;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (lg < ng) {
                const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x) +
                                                                  (size_t)(g0 + lg) * 32 + wd * 8);
                // raw holds x_0..x_7 as (x0,x1)(x2,x3)(x4,x5)(x6,x7); regroup to (x_j, x_{j+4})
                v.x = __byte_perm(raw.x, raw.z, 0x5410);
                v.y = __byte_perm(raw.x, raw.z, 0x7632);
                v.z = __byte_perm(raw.y, raw.w, 0x5410);
                v.w = __byte_perm(raw.y, raw.w, 0x7632);
            }
            xp[i] = v;
        }
        float* xsum = xs + nb * 8 * 16;
        for (int i = threadIdx.x; i < nb * 16; i += blockDim.x) {
            const int lg = i >> 1, hh = i & 1;
            double sum = 0.0;
            if (lg < ng) {
                const uint16_t* src = reinterpret_cast<const uint16_t*>(a.x) + (size_t)(g0 + lg) * 32 + hh * 16;
                for (int e = 0; e < 16; ++e) sum += (double)__uint_as_float((uint32_t)src[e] << 16);
            }
            xsum[i] = (float)sum;
        }
    } else {
        for (int i = threadIdx.x; i < nb * 64; i += blockDim.x) {
            const int lg = i >> 3, c = i & 7;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lg < ng) v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) +
                                                              (size_t)(g0 + lg) * 32 + c * 4);
            reinterpret_cast<float4*>(xs)[i] = v;
        }
    }
    __syncthreads();

    bool ok = true;
    int consumed = 0;
    for (int rbi = 0; rbi < nrb; ++rbi) {
        const int rb = first_rb + rbi * rb_stride;
        float yacc = 0.f;
        for (int jb = 0; jb < nbw; ++jb) {
            const int j = rbi * nbw + jb;
            const int s = j % kStages;
            if (ok) ok = mbar_wait_bounded(&my_bars[s], (uint32_t)(j / kStages) & 1u, kWaitLimit);
            if (ok) {
                consumed = j + 1;
                const unsigned char* cb = codes + (warp * kStages + s) * kCodeBox + r * 128 + h * 8;
                const uint4 sc8 = *reinterpret_cast<const uint4*>(scl + (warp * kStages + s) * kScaleBox + r * 16);
                if constexpr (XBF16) {
                    const uint4* xpb = reinterpret_cast<const uint4*>(xs) + (b0 + jb) * 32 + h * 2;
                    const float* xsum = xs + nb * 8 * 16 + (b0 + jb) * 16 + h;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(cb + ((c ^ (r & 7)) << 4));
                        const float a0 = word_dot_bf16(w2.x, xpb[c * 4], 0.f);
                        const float a1 = word_dot_bf16(w2.y, xpb[c * 4 + 1], 0.f);
                        const float part = fmaf(-136.0f, xsum[c * 2], a0 + a1);   // remove 128 + 8
                        const uint32_t sw = c < 2 ? sc8.x : c < 4 ? sc8.y : c < 6 ? sc8.z : sc8.w;
                        const float sf = __half2float(__ushort_as_half((unsigned short)((c & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
                        yacc = fmaf(sf, part, yacc);
                    }
                } else {
                    const float4* xb = reinterpret_cast<const float4*>(xs) + (b0 + jb) * 64 + h * 4;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(cb + ((c ^ (r & 7)) << 4));
                        const float4* xg = xb + c * 8;
                        const float2 q = __fadd2_rn(word_dot(w2.x, xg, kc), word_dot(w2.y, xg + 2, kc));
                        const uint32_t sw = c < 2 ? sc8.x : c < 4 ? sc8.y : c < 6 ? sc8.z : sc8.w;
                        const float sf = __half2float(__ushort_as_half((unsigned short)((c & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
                        yacc = fmaf(sf, q.x + q.y, yacc);
                    }
                }
            }
            __syncwarp();
            if (ok && j + kStages < njobs) {
                if (lane == 0) {
                    fence_proxy_async_smem();      // our reads of this stage precede the refill
                    issue(j + kStages);
                }
                issued = j + kStages + 1;
            }
        }
        yacc += __shfl_xor_sync(0xffffffffu, yacc, 16);   // the two halves of each row

        // The team's P partial sums for row block rb, added in warp order.
        const int row = rb * kRows + r;
        float total = yacc;
        if (P > 1) {
            if (h == 0) red[warp * kRows + r] = yacc;
            team_sync(team, P);
            if (wt == 0) {
                total = 0.f;
                for (int w = 0; w < P; ++w) total += red[(team * P + w) * kRows + r];
            }
        }
        if (a.splits == 1) {
            if (wt == 0 && h == 0 && row < a.N) a.y[row] = total;
        } else {
            if (wt == 0) {
                if (h == 0 && row < a.N) a.partial[(size_t)split * a.N + row] = total;
                __threadfence();
                __syncwarp();
                if (lane == 0) s_last[team] = atomicAdd(&a.counters[rb], 1u) == (unsigned)(a.splits - 1);
                __syncwarp();
                if (s_last[team]) {
                    __threadfence();
                    if (h == 0 && row < a.N) {
                        float sum = 0.f;
                        for (int sp = 0; sp < a.splits; ++sp) sum += __ldcg(&a.partial[(size_t)sp * a.N + row]);
                        a.y[row] = sum;
                    }
                    if (lane == 0) a.counters[rb] = 0u;
                }
            }
        }
        if (P > 1) team_sync(team, P);           // red[] may be rewritten for the next block
    }

    if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrWaitTimeout);
        for (int j = consumed; j < issued; ++j)   // copies still in flight into this warp's ring
            mbar_wait_bounded(&my_bars[j % kStages], (uint32_t)(j / kStages) & 1u, kWaitLimit);
    }
}

size_t smem_bytes_for(int warps, int nb)
{
    return 1024 + (size_t)warps * kStages * (kCodeBox + kScaleBox) + warps * kStages * sizeof(uint64_t) +
           warps * kRows * sizeof(float) + (size_t)nb * 8 * 32 * sizeof(float);
}

}  // namespace

bool tma_gemv_eligible(int64_t M, int64_t K, const void* packed, const void* scales)
{
    return M == 1 && K % 256 == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(packed) & 15) == 0;
}

bool plan_gemv_tma(int64_t M, int64_t N, int64_t K, q4_dtype xt, const DeviceInfo& dev, GemvPlan* p)
{
    (void)M;
    const int G = (int)(K / 32);
    const int row_blocks = (int)((N + kRows - 1) / kRows);
    const int boxes = (G + 7) / 8;
    const long long warp_slots = (long long)dev.sm_count * 2 * kMaxWarps;
    // Team size: enough warps per row block to fill the SMs, at most one per box.
    int P = 1;
    if ((long long)row_blocks < warp_slots) {
        const long long want = (warp_slots + row_blocks - 1) / row_blocks;
        P = (int)(want < boxes ? want : boxes);
        if (P > kMaxWarps) P = kMaxWarps;
        if (P < 1) P = 1;
    }
    // Still short of work: split K across blocks (each warp keeps >= 1 box).
    int splits = 1;
    while ((long long)row_blocks * P * splits < warp_slots / 2 && boxes / (splits + 1) >= P &&
           row_blocks <= kCounterSlots)
        ++splits;
    int ksg = ((G + splits - 1) / splits + 7) / 8 * 8;
    splits = (G + ksg - 1) / ksg;
    const int nb = (ksg + 7) / 8;
    const int teams = P == 1 ? kMaxWarps : (kMaxWarps / P > 0 ? kMaxWarps / P : 1);
    const int warps = P * teams;
    const size_t smem = smem_bytes_for(warps, nb);
    if (smem > (size_t)dev.max_smem_optin) return false;
    const void* fn = xt == Q4_BF16 ? reinterpret_cast<const void*>(&gemv_tma_m1_kernel<true>)
                                   : reinterpret_cast<const void*>(&gemv_tma_m1_kernel<false>);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, warps * 32, smem) != cudaSuccess || per_sm < 1) {
        cudaGetLastError();
        return false;
    }
    const long long blocks_needed = ((long long)row_blocks + teams - 1) / teams;
    long long gx = ((long long)dev.sm_count * per_sm + splits - 1) / splits;
    if (gx > blocks_needed) gx = blocks_needed;
    if (gx < 1) gx = 1;
    p->kernel = 1;
    p->splits = splits;
    p->groups_per_split = ksg;
    p->row_blocks = row_blocks;
    p->grid_x = (int)gx;
    p->chunk = P;                 // the TMA kernel reuses `chunk` for its team size
    p->xcap = teams;              // ... and `xcap` for teams per block
    p->smem_bytes = (int)smem;
    p->workspace_bytes = splits > 1 ? kCounterBytes + (size_t)splits * (size_t)N * sizeof(float) : 0;
    return true;
}

q4_status launch_gemv_tma(const void* x, q4_dtype xt, int64_t K, const uint8_t* packed, const uint16_t* scales,
                          int64_t N, float* y, void* workspace, const GemvPlan& plan, cudaStream_t stream)
{
    CUtensorMap tm_codes, tm_scales;
    const uint64_t G = (uint64_t)(K / 32);
    if (!encode_tma_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N,
                       (uint64_t)K / 2, 128, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tma_2d(&tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, scales, G, (uint64_t)N, G * 2, 8, kRows,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return Q4_ERR_CUDA;

    TmaGemvArgs a;
    a.x = x;
    a.y = y;
    a.partial = nullptr;
    a.counters = nullptr;
    if (plan.splits > 1) {
        a.counters = reinterpret_cast<unsigned*>(workspace);
        a.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + kCounterBytes);
    }
    a.err = err;
    a.N = (int)N;
    a.G = (int)G;
    a.ksg = plan.groups_per_split;
    a.splits = plan.splits;
    a.row_blocks = plan.row_blocks;
    a.P = plan.chunk;
    a.teams = plan.xcap;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid_x, (unsigned)plan.splits);
    cfg.blockDim = dim3((unsigned)(a.P * a.teams * 32));
    cfg.dynamicSmemBytes = (size_t)plan.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = xt == Q4_BF16
                              ? cudaLaunchKernelEx(&cfg, gemv_tma_m1_kernel<true>, tm_codes, tm_scales, a)
                              : cudaLaunchKernelEx(&cfg, gemv_tma_m1_kernel<false>, tm_codes, tm_scales, a);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
