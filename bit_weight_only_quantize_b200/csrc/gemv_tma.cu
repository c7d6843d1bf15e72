// q4_gemv / q4_gemv_multi for the shapes the TMA path serves (K % 256 == 0, scales
// 16-byte aligned; M = 1 with f32 or bf16 x, M = 2..16 with bf16 x).
//
// Decode streams every weight once, so the kernels are built around keeping HBM busy
// and spending few instructions per weight (QORA-LLM-0.8B model card, section "AVX-512
// SIMD Acceleration": a Q4 GEMV whose nibbles go through a 16-entry table; QORA-4B
// thread, section "量化与内存管理": GEMV over Q4 weights on a thread pool):
//
//  * Weights stream as TMA boxes of 16 rows x 8 groups: 2 KiB of codes (128-byte
//    swizzled) plus 256 B of binary16 scales, into a per-warp ring of kStages stages
//    guarded by mbarriers.  Each warp issues its own boxes (lane 0), so no producer
//    warp is needed and a block keeps warps * kStages boxes in flight.
//  * Work is cut into row blocks of 16 rows, enumerated over one or more weight
//    matrices that share x (one launch for a set of projections of the same token).
//    Teams of P warps own sequences of row blocks; the P warps of a team take
//    disjoint K ranges of each block and add their partial sums in a fixed order.
//    Skinny shapes also split K across blocks (last-arriver reduction, no waiting).
//  * Arithmetic per mode:
//      f32 x, M = 1:  nibble p OR-ed into the mantissa of 2^(23-4p) is exactly
//                     2^(23-4p) + code; a packed f32x2 add leaves code - 8; packed
//                     f32x2 FMAs accumulate each group in f32.  Two lanes per row.
//      bf16 x, M = 1: nibble pair (j, j+4) OR-ed into 0x4300 is the bf16 pair
//                     (128 + c_j, 128 + c_{j+4}); fma.rn.f32.bf16 multiplies it by the
//                     bf16 x pair exactly and accumulates in f32; 136 * sum(x) of the
//                     half group (an f64 sum rounded once) is subtracted afterwards.
//      bf16 x, M = 2..16: the same bf16 pairs are the A operand of
//                     mma.sync.m16n8k16 (f32 accumulate), x rows the B operand, in a
//                     permuted k order that matches the pairs; 136 * sum(x) per group
//                     and x row is subtracted from each group's MMA result.
//    In every mode each group's sum is scaled by its binary16 scale and added in f32.
//  * Every mbarrier wait is bounded.  If one runs out the kernel records
//    kErrWaitTimeout in the library error word, stops issuing and computing, waits
//    (bounded) for its own copies still in flight and returns (see q4_device_error).
#include "tma.cuh"

namespace q4 {
namespace {

constexpr int kRows = 16;                    // rows per row block
constexpr int kMaxWarps = 16;
constexpr int kStages = 2;
constexpr uint32_t kCodeBox = kRows * 128;   // bytes of codes per box (8 groups)
constexpr uint32_t kScaleBox = kRows * 16;   // bytes of scales per box
constexpr uint64_t kWaitLimit = kWaitLimitNs;
constexpr int kCounterSlots = 1024;          // same workspace layout as the generic kernel
constexpr size_t kCounterBytes = kCounterSlots * sizeof(unsigned);

enum Mode { kF32M1 = 0, kBf16M1 = 1, kMma8 = 2, kMma16 = 3 };

struct TmaMaps {
    CUtensorMap codes[Q4_MULTI_MAX];
    CUtensorMap scales[Q4_MULTI_MAX];
};

struct TmaGemvArgs {
    const void* x;
    float* y[Q4_MULTI_MAX];
    int N[Q4_MULTI_MAX];
    int rb_begin[Q4_MULTI_MAX + 1];   // first row block of each matrix; [count] = total
    int count;
    int M;
    float* partial;                   // [splits][M][row_blocks * 16]
    unsigned* counters;               // [row_blocks]
    unsigned* err;
    int G;
    int ksg;                          // groups per split (multiple of 8)
    int splits;
    int row_blocks;
    int P;                            // warps per team
    int teams;                        // teams per block
    int prefetch;                     // weights may be read before the dependency wait
};

__device__ __forceinline__ void team_sync(int team, int P)
{
    if (P == 1) {
        __syncwarp();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(P * 32) : "memory");
    }
}

__device__ __forceinline__ int matrix_of(const TmaGemvArgs& a, int rb)
{
    int m = 0;
    while (m + 1 < a.count && rb >= a.rb_begin[m + 1]) ++m;
    return m;
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

// f32 x: eight codes of one word dotted with eight x values (exact code - 8).
__device__ __forceinline__ float2 word_dot_f32(uint32_t v, const float4* xw, const ExpandConsts& k)
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

// Nibble pair (j, j+4) of a word as the bf16 pair (128 + c_j, 128 + c_{j+4}).
__device__ __forceinline__ uint32_t nib_pair(uint32_t v, int j)
{
    return ((v >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
}

// bf16 x: sum_j x_j * (128 + c_j) over the 8 weights of one word; xp holds the x pairs
// (x_j, x_{j+4}) matching nib_pair.  Every product is exact in f32.
__device__ __forceinline__ float word_dot_bf16(uint32_t v, uint4 xp, float acc)
{
    const uint32_t xs[4] = {xp.x, xp.y, xp.z, xp.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t t = nib_pair(v, j);
        acc = fma_bf16((uint16_t)(t & 0xFFFFu), (uint16_t)(xs[j] & 0xFFFFu), acc);
        acc = fma_bf16((uint16_t)(t >> 16), (uint16_t)(xs[j] >> 16), acc);
    }
    return acc;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f), "f"(0.f), "f"(0.f), "f"(0.f));
}

__device__ __forceinline__ float scale_at(const uint4& s8, int c)
{
    const uint32_t sw = c < 2 ? s8.x : c < 4 ? s8.y : c < 6 ? s8.z : s8.w;
    return __half2float(__ushort_as_half((unsigned short)((c & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
}

__device__ __forceinline__ uint4 pairs_of(const uint4 raw)
{
    // raw holds x_0..x_7 as (x0,x1)(x2,x3)(x4,x5)(x6,x7); regroup to (x_j, x_{j+4}).
    return make_uint4(__byte_perm(raw.x, raw.z, 0x5410), __byte_perm(raw.x, raw.z, 0x7632),
                      __byte_perm(raw.y, raw.w, 0x5410), __byte_perm(raw.y, raw.w, 0x7632));
}

__device__ __forceinline__ double sum8_bf16(const uint4 raw)
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        s += (double)__uint_as_float(w[i] << 16) + (double)__uint_as_float(w[i] & 0xFFFF0000u);
    return s;
}

template <int MODE>
struct ModeCfg {
    static constexpr int MP = MODE == kMma16 ? 16 : MODE == kMma8 ? 8 : 1;   // padded x rows
    static constexpr int NT = MP >= 8 ? MP / 8 : 1;                          // n-tiles of 8 x rows
    static constexpr int kMinBlocks = MODE <= kBf16M1 ? 2 : 1;
};

template <int MODE>
__global__ void __launch_bounds__(kMaxWarps * 32, ModeCfg<MODE>::kMinBlocks)
gemv_tma_kernel(const __grid_constant__ TmaMaps maps, const TmaGemvArgs a)
{
    constexpr int MP = ModeCfg<MODE>::MP;
    constexpr int NT = ModeCfg<MODE>::NT;
    extern __shared__ unsigned char smem_raw[];
    __shared__ int s_last[kMaxWarps];
    const int W = blockDim.x >> 5;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* codes = smem;                                          // [warp][stage][2048]
    unsigned char* scl = codes + W * kStages * kCodeBox;                  // [warp][stage][256]
    uint64_t* bars = reinterpret_cast<uint64_t*>(scl + W * kStages * kScaleBox);   // [warp][stage]
    float* red = reinterpret_cast<float*>(bars + W * kStages);            // [warp][16 rows][MP]
    unsigned char* xst = reinterpret_cast<unsigned char*>(red + W * kRows * MP);   // staged x (16-byte aligned)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = a.P;
    const int team = warp / P, wt = warp - team * P;
    const bool active = team < a.teams;
    const int split = blockIdx.y;
    const int g0 = split * a.ksg;
    const int ng = min(a.G - g0, a.ksg);
    const int nb = (ng + 7) >> 3;                                         // boxes of this split
    const int ngp = nb * 8;                                               // groups, padded
    const int b0 = wt * nb / P, nbw = (wt + 1) * nb / P - b0;             // this warp's boxes
    const int first_rb = blockIdx.x * a.teams + team;
    const int rb_stride = gridDim.x * a.teams;
    const int nrb = (active && first_rb < a.row_blocks) ? (a.row_blocks - first_rb + rb_stride - 1) / rb_stride : 0;
    const int njobs = nrb * nbw;
    uint64_t* my_bars = bars + warp * kStages;
    const size_t K = (size_t)a.G * 32;

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const ExpandConsts kc = {make_float2(pinned(-8388616.0f), pinned(-524296.0f)),
                             make_float2(pinned(-32776.0f), pinned(-2056.0f)),
                             make_float2(pinned(-136.0f), pinned(-32776.0f)),
                             make_float2(pinned(-2056.0f), pinned(-136.0f))};

    auto issue = [&](int j) {
        const int s = j % kStages;
        const int rb = first_rb + (j / nbw) * rb_stride;
        const int b = b0 + j % nbw;
        const int mi = matrix_of(a, rb);
        const int lrow = (rb - a.rb_begin[mi]) * kRows;
        mbar_arrive_expect_tx(&my_bars[s], kCodeBox + kScaleBox);
        tma_load_2d(codes + (warp * kStages + s) * kCodeBox, &maps.codes[mi], (g0 + 8 * b) * 16, lrow, &my_bars[s]);
        tma_load_2d(scl + (warp * kStages + s) * kScaleBox, &maps.scales[mi], g0 + 8 * b, lrow, &my_bars[s]);
    };
    int issued = min(kStages, njobs);
    // Weights that no kernel still in flight writes may stream before the dependency
    // wait; x and every output only after it.
    if (a.prefetch && lane == 0)
        for (int j = 0; j < issued; ++j) issue(j);
    pdl_launch_dependents();
    pdl_wait();
    if (!a.prefetch && lane == 0)
        for (int j = 0; j < issued; ++j) issue(j);

    // ---- stage x for this split (zero past the split, past K and past M) ----
    //  kF32M1 : f32 [group][32]
    //  kBf16M1: bf16 pairs [group][word][4] + f32 sums of each half group
    //  kMma*  : bf16 pairs [m][group][word][4] + f32 sums [group][m]
    // Sums are of the bf16 values in f64, rounded once; neighbouring lanes combine words.
    float* xsum = nullptr;
    if constexpr (MODE == kF32M1) {
        float4* xf = reinterpret_cast<float4*>(xst);
        for (int i = threadIdx.x; i < ngp * 8; i += blockDim.x) {
            const int lg = i >> 3, c = i & 7;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lg < ng)
                v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + (size_t)(g0 + lg) * 32 + c * 4);
            xf[i] = v;
        }
    } else {
        uint4* xp = reinterpret_cast<uint4*>(xst);
        xsum = reinterpret_cast<float*>(xp + MP * ngp * 4);
        const int total = MP * ngp * 4;
        for (int i0 = threadIdx.x - lane; i0 < total; i0 += blockDim.x) {    // warp-uniform trips
            const int i = i0 + lane;
            const int m = i / (ngp * 4);
            const int rem = i - m * ngp * 4;
            const int lg = rem >> 2, wd = rem & 3;
            uint4 raw = make_uint4(0u, 0u, 0u, 0u);
            if (i < total && m < a.M && lg < ng)
                raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x) + (size_t)m * K +
                                                      (size_t)(g0 + lg) * 32 + wd * 8);
            if (i < total) xp[i] = pairs_of(raw);
            double sum = sum8_bf16(raw);
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);                    // words (0,1) and (2,3)
            if constexpr (MODE == kBf16M1) {
                if (i < total && (wd & 1) == 0) xsum[lg * 2 + (wd >> 1)] = (float)sum;
            } else {
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);                // all four words
                if (i < total && wd == 0) xsum[lg * MP + m] = (float)sum;
            }
        }
    }
    __syncthreads();

    bool ok = true;
    int consumed = 0;
    for (int rbi = 0; rbi < nrb; ++rbi) {
        const int rb = first_rb + rbi * rb_stride;
        float yacc = 0.f;     // M = 1 modes: row (lane & 15), half (lane >> 4)
        float acc[NT][4];     // MMA modes: rows g, g+8; x rows n*8 + 2t, +1
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

        for (int jb = 0; jb < nbw; ++jb) {
            const int j = rbi * nbw + jb;
            const int s = j % kStages;
            if (ok) ok = mbar_wait_bounded(&my_bars[s], (uint32_t)(j / kStages) & 1u, kWaitLimit);
            if (ok) {
                consumed = j + 1;
                const unsigned char* cb = codes + (warp * kStages + s) * kCodeBox;
                const unsigned char* sb = scl + (warp * kStages + s) * kScaleBox;
                const int gb = (b0 + jb) * 8;                                 // first group of the box
                if constexpr (MODE == kF32M1 || MODE == kBf16M1) {
                    const int r = lane & 15, h = lane >> 4;
                    const unsigned char* rowp = cb + r * 128 + h * 8;
                    const uint4 s8 = *reinterpret_cast<const uint4*>(sb + r * 16);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(rowp + ((c ^ (r & 7)) << 4));
                        float part;
                        if constexpr (MODE == kF32M1) {
                            const float4* xg = reinterpret_cast<const float4*>(xst) + (gb + c) * 8 + h * 4;
                            const float2 q = __fadd2_rn(word_dot_f32(w2.x, xg, kc), word_dot_f32(w2.y, xg + 2, kc));
                            part = q.x + q.y;
                        } else {
                            const uint4* xpg = reinterpret_cast<const uint4*>(xst) + (gb + c) * 4 + h * 2;
                            const float a0 = word_dot_bf16(w2.x, xpg[0], 0.f);
                            const float a1 = word_dot_bf16(w2.y, xpg[1], 0.f);
                            part = fmaf(-136.0f, xsum[(gb + c) * 2 + h], a0 + a1);   // remove 128 + 8
                        }
                        yacc = fmaf(scale_at(s8, c), part, yacc);
                    }
                } else {
                    const int g = lane >> 2, t = lane & 3;
                    const uint4 sg = *reinterpret_cast<const uint4*>(sb + g * 16);
                    const uint4 sg8 = *reinterpret_cast<const uint4*>(sb + (g + 8) * 16);
                    const uint4* xp = reinterpret_cast<const uint4*>(xst);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int off = ((c ^ g) << 4) + 4 * t;                 // (g & 7) == g
                        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(cb + g * 128 + off);
                        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(cb + (g + 8) * 128 + off);
                        const uint32_t A0 = nib_pair(w0, 0), A1 = nib_pair(w1, 0), A2 = nib_pair(w0, 1),
                                       A3 = nib_pair(w1, 1);
                        const uint32_t A4 = nib_pair(w0, 2), A5 = nib_pair(w1, 2), A6 = nib_pair(w0, 3),
                                       A7 = nib_pair(w1, 3);
                        const float s0 = scale_at(sg, c), s1 = scale_at(sg8, c);
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint4 bx = xp[((n * 8 + g) * ngp + gb + c) * 4 + t];
                            float d0[4], d1[4];
                            mma_bf16_16816(d0, A0, A1, A2, A3, bx.x, bx.y);
                            mma_bf16_16816(d1, A4, A5, A6, A7, bx.z, bx.w);
                            const float2 xs2 = *reinterpret_cast<const float2*>(xsum + (gb + c) * MP + n * 8 + 2 * t);
                            acc[n][0] = fmaf(s0, fmaf(-136.0f, xs2.x, d0[0] + d1[0]), acc[n][0]);
                            acc[n][1] = fmaf(s0, fmaf(-136.0f, xs2.y, d0[1] + d1[1]), acc[n][1]);
                            acc[n][2] = fmaf(s1, fmaf(-136.0f, xs2.x, d0[2] + d1[2]), acc[n][2]);
                            acc[n][3] = fmaf(s1, fmaf(-136.0f, xs2.y, d0[3] + d1[3]), acc[n][3]);
                        }
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

        // ---- row block rb complete: partials -> red[warp][row][m], team sum in warp order ----
        float* my_red = red + warp * kRows * MP;
        if constexpr (MODE == kF32M1 || MODE == kBf16M1) {
            yacc += __shfl_xor_sync(0xffffffffu, yacc, 16);           // the two halves of each row
            if (lane < 16) my_red[lane] = yacc;
        } else {
            const int g = lane >> 2, t = lane & 3;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                my_red[g * MP + n * 8 + 2 * t] = acc[n][0];
                my_red[g * MP + n * 8 + 2 * t + 1] = acc[n][1];
                my_red[(g + 8) * MP + n * 8 + 2 * t] = acc[n][2];
                my_red[(g + 8) * MP + n * 8 + 2 * t + 1] = acc[n][3];
            }
        }
        team_sync(team, P);
        if (wt == 0) {
            const int mi = matrix_of(a, rb);
            const int nrow = a.N[mi];
            const int lrow0 = (rb - a.rb_begin[mi]) * kRows;
            const size_t vrows = (size_t)a.row_blocks * kRows;            // padded rows over all matrices
            for (int e = lane; e < kRows * MP; e += 32) {
                const int rr = e / MP, m = e - rr * MP;
                float total = 0.f;
                for (int w = 0; w < P; ++w) total += red[(team * P + w) * kRows * MP + e];
                if (m < a.M && lrow0 + rr < nrow) {
                    if (a.splits == 1) a.y[mi][(size_t)m * nrow + lrow0 + rr] = total;
                    else a.partial[((size_t)split * a.M + m) * vrows + (size_t)rb * kRows + rr] = total;
                }
            }
            if (a.splits > 1) {
                __threadfence();
                __syncwarp();
                if (lane == 0) s_last[team] = atomicAdd(&a.counters[rb], 1u) == (unsigned)(a.splits - 1);
                __syncwarp();
                if (s_last[team]) {
                    __threadfence();
                    for (int e = lane; e < kRows * a.M; e += 32) {
                        const int m = e / kRows, rr = e - m * kRows;
                        if (lrow0 + rr < nrow) {
                            float sum = 0.f;
                            for (int sp = 0; sp < a.splits; ++sp)
                                sum += __ldcg(&a.partial[((size_t)sp * a.M + m) * vrows + (size_t)rb * kRows + rr]);
                            a.y[mi][(size_t)m * nrow + lrow0 + rr] = sum;
                        }
                    }
                    if (lane == 0) a.counters[rb] = 0u;
                }
            }
        }
        team_sync(team, P);                        // red[] may be rewritten for the next block
    }

    if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrWaitTimeout);
        for (int j = consumed; j < issued; ++j)    // copies still in flight into this warp's ring
            mbar_wait_bounded(&my_bars[j % kStages], (uint32_t)(j / kStages) & 1u, kWaitLimit);
    }
}

size_t smem_bytes(int mode, int warps, int nb)
{
    const int mp = mode == kMma16 ? 16 : mode == kMma8 ? 8 : 1;
    const size_t ring = (size_t)warps * kStages * (kCodeBox + kScaleBox) + warps * kStages * sizeof(uint64_t);
    const size_t red = (size_t)warps * kRows * mp * sizeof(float);
    const size_t ngp = (size_t)nb * 8;
    const size_t xs = mode == kF32M1 ? ngp * 32 * sizeof(float)
                                     : (size_t)mp * ngp * 64 + ngp * (mode == kBf16M1 ? 2 : mp) * sizeof(float);
    return 1024 + ring + red + xs;
}

int mode_for(int64_t M, q4_dtype xt)
{
    if (M == 1) return xt == Q4_BF16 ? kBf16M1 : kF32M1;
    return M <= 8 ? kMma8 : kMma16;
}

const void* kernel_for(int mode)
{
    switch (mode) {
    case kF32M1: return reinterpret_cast<const void*>(&gemv_tma_kernel<kF32M1>);
    case kBf16M1: return reinterpret_cast<const void*>(&gemv_tma_kernel<kBf16M1>);
    case kMma8: return reinterpret_cast<const void*>(&gemv_tma_kernel<kMma8>);
    default: return reinterpret_cast<const void*>(&gemv_tma_kernel<kMma16>);
    }
}

}  // namespace

bool tma_gemv_eligible(int64_t M, int64_t K, q4_dtype xt, const void* packed, const void* scales)
{
    const bool shape = M == 1 || (M >= 2 && M <= Q4_GEMV_MAX_M && xt == Q4_BF16);
    return shape && K % 256 == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(packed) & 15) == 0;
}

bool plan_gemv_tma(int64_t M, const int64_t* Ns, int count, int64_t K, q4_dtype xt, const DeviceInfo& dev,
                   GemvPlan* p)
{
    const int mode = mode_for(M, xt);
    const int G = (int)(K / 32);
    long long rbl = 0;
    for (int i = 0; i < count; ++i) rbl += (Ns[i] + kRows - 1) / kRows;
    if (rbl < 1 || rbl > INT32_MAX / kRows) return false;
    const int row_blocks = (int)rbl;
    const int boxes = (G + 7) / 8;
    const long long warp_slots = (long long)dev.sm_count * (mode <= kBf16M1 ? 2 : 1) * kMaxWarps;
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
    const int ksg = ((G + splits - 1) / splits + 7) / 8 * 8;
    splits = (G + ksg - 1) / ksg;
    const int nb = (ksg + 7) / 8;
    const int teams = P == 1 ? kMaxWarps : (kMaxWarps / P > 0 ? kMaxWarps / P : 1);
    const int warps = P * teams;
    const size_t smem = smem_bytes(mode, warps, nb);
    if (smem > (size_t)dev.max_smem_optin) return false;
    const void* fn = kernel_for(mode);
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
    p->chunk = P;                 // the TMA kernels reuse `chunk` for their team size
    p->xcap = teams;              // ... and `xcap` for teams per block
    p->smem_bytes = (int)smem;
    p->workspace_bytes =
        splits > 1 ? kCounterBytes + (size_t)splits * (size_t)M * (size_t)row_blocks * kRows * sizeof(float) : 0;
    return true;
}

q4_status launch_gemv_tma(const void* x, q4_dtype xt, int64_t M, int64_t K, const q4_weight* mats, int count,
                          int prefetch, void* workspace, const GemvPlan& plan, cudaStream_t stream)
{
    TmaMaps maps;
    TmaGemvArgs a;
    const uint64_t G = (uint64_t)(K / 32);
    int rb = 0;
    for (int i = 0; i < count; ++i) {
        if (!encode_tma_2d(&maps.codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, mats[i].packed, (uint64_t)K / 2,
                           (uint64_t)mats[i].N, (uint64_t)K / 2, 128, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_tma_2d(&maps.scales[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, mats[i].scales, G, (uint64_t)mats[i].N,
                           G * 2, 8, kRows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
        a.y[i] = mats[i].y;
        a.N[i] = (int)mats[i].N;
        a.rb_begin[i] = rb;
        rb += (int)((mats[i].N + kRows - 1) / kRows);
    }
    for (int i = count; i < Q4_MULTI_MAX; ++i) {
        maps.codes[i] = maps.codes[0];
        maps.scales[i] = maps.scales[0];
        a.y[i] = nullptr;
        a.N[i] = 0;
        a.rb_begin[i] = rb;
    }
    a.rb_begin[Q4_MULTI_MAX] = rb;
    unsigned* err = device_error_word();
    if (!err) return Q4_ERR_CUDA;
    a.x = x;
    a.count = count;
    a.M = (int)M;
    a.partial = nullptr;
    a.counters = nullptr;
    if (plan.splits > 1) {
        a.counters = reinterpret_cast<unsigned*>(workspace);
        a.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + kCounterBytes);
    }
    a.err = err;
    a.G = (int)G;
    a.ksg = plan.groups_per_split;
    a.splits = plan.splits;
    a.row_blocks = plan.row_blocks;
    a.P = plan.chunk;
    a.teams = plan.xcap;
    a.prefetch = prefetch;

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
    void* args[] = {&maps, &a};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, kernel_for(mode_for(M, xt)), args);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
