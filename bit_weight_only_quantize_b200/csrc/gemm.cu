// q4_gemm: y[M,N] = bf16( x[M,K] . dequant(W)^T ), prefill shapes, on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// The pages batch every prefill projection across the prompt's tokens into GEMMs
// (QORA-4B thread, section "GPU 预填充优化"; QORA-LLM-0.8B model card, section
// "Performance": batched prefill "processes all GEMM projections in parallel across
// tokens").  Here each weight is dequantised once per tile into shared memory as
// bf16 and fed to tcgen05.mma with f32 accumulation:
//
//   w_bf16 = bf16_rn((code - 8) * f32(scale))      (the f32 product is exact, one rounding)
//
// One persistent block per SM, warp-specialised:
//   warp 0      TMA producer: x tiles (128 rows x 64 k, 128-byte swizzle), the raw
//               codes of the weight tile (BN rows x 32 bytes) and, when K % 256 == 0,
//               the 16-byte row of scales around the stage's two groups into a ring of
//               kStages.
//   warp 1      allocates tensor memory; one thread issues the MMAs (128 x BN x 16
//               per instruction, MA accumulators of 128 rows per tile) and commits.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator lanes, f32 -> bf16, stores.
//   warps 6..21 dequantise: codes -> bf16 in the K-major 128-byte-swizzled layout the
//               MMA descriptor expects, scales from the stage (or, for other K, read
//               from global two k-blocks ahead), then fence.proxy.async and arrive.
// Accumulators are double-buffered in tensor memory, so the epilogue of one tile
// overlaps the MMAs of the next.  Every mbarrier wait is bounded; on a timeout the
// block records kErrWaitTimeout, all roles stop, outstanding copies and MMAs are
// waited for (bounded) and tensor memory is freed before the block exits.
#include <algorithm>
#include <mutex>

#include "tma.cuh"

namespace q4 {
namespace {

constexpr int kBK = 64;                       // k per stage: one 128-byte swizzle row of bf16
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;                  // warps 2..5
constexpr int kDeqWarp0 = 6;                  // warps 6..21
constexpr int kDeqWarps = 16;
constexpr int kDeqGroups = 2;                 // CTA-pair kernel: dequantising warp groups taking alternate stages
constexpr int kThreads = (kDeqWarp0 + kDeqWarps) * 32;   // 704
constexpr uint64_t kWaitLimit = kWaitLimitNs;

struct GemmArgs {
    const uint16_t* scales;
    int scale_tma;                    // scales arrive by TMA with each stage (needs K % 256 == 0)
    uint16_t* y;
    unsigned* err;
    int M, N, K, G;
    int tiles_m, tiles_n;
    int kblocks;
};

// ---- tcgen05 wrappers (inline PTX) ----
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// 32 consecutive f32 columns of this warp's 32 accumulator lanes.
// 16 consecutive f32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: bf16 x bf16 -> f32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t instr_desc(int m, int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// (a & m) | c as one LOP3 with all three operands in registers (the instruction takes a
// single immediate, so constant masks and magics are kept in registers by the caller).
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(m), "r"(c));
    return r;
}

__device__ __forceinline__ uint32_t pinned_u32(uint32_t v)
{
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

// Constants of dequant8 held in registers: nibble masks 0xF << 4i and the exponents
// 2^(23-4i) whose mantissa a nibble at bit 4i lands in.
struct DequantConsts {
    uint32_t mask[5], magic[5];
    __device__ __forceinline__ DequantConsts()
    {
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            mask[i] = pinned_u32(0xFu << (4 * i));
            magic[i] = pinned_u32((uint32_t)(150 - 4 * i) << 23);
        }
    }
};

// Eight codes of one word -> eight bf16 values (code - 8) * s in k order, rounded once.
// Nibble i OR-ed into the mantissa of 2^(23-4i) is exactly 2^(23-4i) + code; a packed
// add removes 2^(23-4i) + 8 exactly, the packed multiply by s is exact (a 4-bit integer
// times a binary16 value fits in f32), and cvt.rn.bf16x2 rounds once.
__device__ __forceinline__ uint4 dequant8(uint32_t v, float s, const DequantConsts& k)
{
    const uint32_t u = v >> 12;
    const float f0 = __uint_as_float(and_or(v, k.mask[0], k.magic[0]));   // 2^23 + c0
    const float f1 = __uint_as_float(and_or(v, k.mask[1], k.magic[1]));   // 2^19 + c1
    const float f2 = __uint_as_float(and_or(v, k.mask[2], k.magic[2]));   // 2^15 + c2
    const float f3 = __uint_as_float(and_or(v, k.mask[3], k.magic[3]));   // 2^11 + c3
    const float f4 = __uint_as_float(and_or(v, k.mask[4], k.magic[4]));   // 2^7  + c4
    const float f5 = __uint_as_float(and_or(u, k.mask[2], k.magic[2]));   // 2^15 + c5
    const float f6 = __uint_as_float(and_or(u, k.mask[3], k.magic[3]));   // 2^11 + c6
    const float f7 = __uint_as_float(and_or(u, k.mask[4], k.magic[4]));   // 2^7  + c7
    const float2 ss = make_float2(s, s);
    const float2 d01 = __fmul2_rn(__fadd2_rn(make_float2(f0, f1), make_float2(-8388616.0f, -524296.0f)), ss);
    const float2 d23 = __fmul2_rn(__fadd2_rn(make_float2(f2, f3), make_float2(-32776.0f, -2056.0f)), ss);
    const float2 d45 = __fmul2_rn(__fadd2_rn(make_float2(f4, f5), make_float2(-136.0f, -32776.0f)), ss);
    const float2 d67 = __fmul2_rn(__fadd2_rn(make_float2(f6, f7), make_float2(-2056.0f, -136.0f)), ss);
    return make_uint4(pack_bf16x2(d01.x, d01.y), pack_bf16x2(d23.x, d23.y), pack_bf16x2(d45.x, d45.y),
                      pack_bf16x2(d67.x, d67.y));
}

template <int MA, int BN>
struct GemmCfg {
    static constexpr int kStages = MA == 2 ? 4 : (BN == 128 ? 5 : 7);
    static constexpr uint32_t kABytes = 128 * kBK * 2;            // one 128-row x tile: 16 KiB
    static constexpr uint32_t kBBytes = BN * kBK * 2;             // dequantised weight tile
    static constexpr uint32_t kRawBytes = BN * (kBK / 2);         // raw codes
    static constexpr uint32_t kScaleBytes = BN * 16;              // scales: 8 groups x BN rows
    static constexpr uint32_t kStageBytes = MA * kABytes + kBBytes + kRawBytes + kScaleBytes;
    static constexpr uint32_t kTxBytes = MA * kABytes + kRawBytes;
    static constexpr uint32_t kTmemCols = 2 * MA * BN;            // double-buffered accumulators
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 256;
    static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "tensor memory columns");
};

template <int MA, int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
               const __grid_constant__ CUtensorMap tm_scales, const GemmArgs a)
{
    using C = GemmCfg<MA, BN>;
    constexpr int S = C::kStages;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Per stage: [MA x A tile][B tile][raw codes][scales]; A and B tiles are 1024-byte
    // aligned.  The scale box holds the 8 groups around the stage's 2 (a 16-byte row).
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
    uint64_t* full = bars;               // producer -> dequant   (TMA bytes)
    uint64_t* bready = bars + S;         // dequant -> MMA        (kDeqWarps arrivals)
    uint64_t* empty = bars + 2 * S;      // MMA -> producer       (commit)
    uint64_t* accfull = bars + 3 * S;    // MMA -> epilogue, 2 buffers (commit)
    uint64_t* accempty = accfull + 2;    // epilogue -> MMA, 2 buffers (4 warp arrivals)
    uint64_t* drain = accempty + 2;      // final commit on abort
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = a.tiles_m * a.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bready[s], kDeqWarps);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_codes);
        if (a.scale_tma) tma_prefetch_desc(&tm_scales);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_launch_dependents();
    pdl_wait();

    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.err, kErrWaitTimeout);
    };

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int it = 0;
            int last_phase[16];
            for (int s = 0; s < S; ++s) last_phase[s] = -1;
            for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
                const int m0 = (t % a.tiles_m) * (128 * MA);
                const int n0 = (t / a.tiles_m) * BN;
                for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (uint32_t)(it / S) & 1u;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, kWaitLimit)) { fail(); break; }
                    if (*abort_flag) break;
                    unsigned char* st = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], C::kTxBytes + (a.scale_tma ? C::kScaleBytes : 0u));
                    for (int am = 0; am < MA; ++am)
                        tma_load_2d(st + am * C::kABytes, &tm_x, kb * kBK, m0 + am * 128, &full[s]);
                    tma_load_2d(st + MA * C::kABytes + C::kBBytes, &tm_codes, kb * (kBK / 2), n0, &full[s]);
                    if (a.scale_tma)           // 16-byte aligned: group (2 kb) rounded down to 8
                        tma_load_2d(st + MA * C::kABytes + C::kBBytes + C::kRawBytes, &tm_scales, (kb * 2) & ~7, n0,
                                    &full[s]);
                    last_phase[s] = (int)ph;
                }
            }
            if (*abort_flag)      // copies still in flight land before the block can exit
                for (int s = 0; s < S; ++s)
                    if (last_phase[s] >= 0) mbar_wait_bounded(&full[s], (uint32_t)last_phase[s], kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc(128, BN);
            int it = 0, tcount = 0;
            bool issued_any = false;
            for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++tcount) {
                const int buf = tcount & 1;
                if (!mbar_wait_bounded(&accempty[buf], ((uint32_t)(tcount >> 1) & 1u) ^ 1u, kWaitLimit)) { fail(); break; }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait_bounded(&bready[s], (uint32_t)(it / S) & 1u, kWaitLimit)) { fail(); ok = false; break; }
                    if (*abort_flag) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * C::kStageBytes);
                    const uint32_t b_addr = st + MA * C::kABytes;
#pragma unroll
                    for (int am = 0; am < MA; ++am) {
                        const uint32_t d = tmem_base + (uint32_t)((buf * MA + am) * BN);
                        const uint32_t a_addr = st + am * C::kABytes;
#pragma unroll
                        for (int j = 0; j < kBK / 16; ++j)
                            mma_bf16(d, sw128_desc(a_addr + j * 32), sw128_desc(b_addr + j * 32), idesc,
                                     (kb > 0 || j > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[s]);     // stage reusable once these MMAs have read it
                    issued_any = true;
                }
                if (!ok) break;
                mma_commit(&accfull[buf]);     // accumulator complete
            }
            if (*abort_flag && issued_any) {   // every MMA issued so far completes before tensor memory is freed
                mma_commit(drain);
                mbar_wait_bounded(drain, 0, kWaitLimit);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        const int quad = warp & 3;             // tensor-memory lanes 32*quad .. 32*quad+31
        int tcount = 0;
        const bool vec_ok = (a.N % 8) == 0 && (reinterpret_cast<uintptr_t>(a.y) & 15) == 0;
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++tcount) {
            const int buf = tcount & 1;
            if (!mbar_wait_bounded(&accfull[buf], (uint32_t)(tcount >> 1) & 1u, kWaitLimit)) { fail(); break; }
            tc_fence_after();
            const int m0 = (t % a.tiles_m) * (128 * MA);
            const int n0 = (t / a.tiles_m) * BN;
#pragma unroll 1
            for (int am = 0; am < MA; ++am) {
                const int row = m0 + am * 128 + quad * 32 + lane;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)((buf * MA + am) * BN + c0), r);
                    const int col = n0 + c0;
                    if (row < a.M) {
                        uint16_t* dst = a.y + (size_t)row * a.N + col;
                        if (vec_ok && col + 32 <= a.N) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint4 o;
                                o.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
                                o.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
                                o.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
                                o.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
                                *reinterpret_cast<uint4*>(dst + 8 * q) = o;
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                if (col + q < a.N) dst[q] = (uint16_t)(pack_bf16x2(__uint_as_float(r[q]), 0.f) & 0xFFFFu);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[buf]);
        }
    } else {
        // Dequantise: each thread owns BN*8/256 chunks (row n, 16-byte k chunk c) of every stage.
        const int dt = threadIdx.x - kDeqWarp0 * 32;
        constexpr int kChunks = BN * 8 / (kDeqWarps * 32);
        const DequantConsts dk;
        int it = 0;
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
            const int n0 = (t / a.tiles_m) * BN;
            // Scales for k-blocks kb+1 and kb+2 are in flight while kb is dequantised.
            float sc0[kChunks], sc1[kChunks], sc2[kChunks];
            auto load_scales = [&](int kb, float (&dst)[kChunks]) {
#pragma unroll
                for (int q = 0; q < kChunks; ++q) {
                    const int idx = dt + q * kDeqWarps * 32;
                    const int n = n0 + idx / 8, g = kb * 2 + (idx & 7) / 4;
                    dst[q] = (kb < a.kblocks && n < a.N && g < a.G)
                                 ? __half2float(__ushort_as_half(__ldg(a.scales + (size_t)n * a.G + g)))
                                 : 0.f;
                }
            };
            if (!a.scale_tma) {
                load_scales(0, sc0);
                load_scales(1, sc1);
            }
            bool ok = true;
            for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                if (!a.scale_tma) load_scales(kb + 2, sc2);
                const int s = it % S;
                if (!mbar_wait_bounded(&full[s], (uint32_t)(it / S) & 1u, kWaitLimit)) { fail(); ok = false; break; }
                if (*abort_flag) { ok = false; break; }
                unsigned char* st = smem + s * C::kStageBytes;
                unsigned char* bt = st + MA * C::kABytes;
                const unsigned char* raw = bt + C::kBBytes;
                const __half* sst = reinterpret_cast<const __half*>(raw + C::kRawBytes);
#pragma unroll
                for (int q = 0; q < kChunks; ++q) {
                    const int idx = dt + q * kDeqWarps * 32;
                    const int n = idx >> 3, c = idx & 7;
                    const uint32_t v = *reinterpret_cast<const uint32_t*>(raw + n * 32 + c * 4);
                    const float sc = a.scale_tma ? __half2float(sst[n * 8 + ((kb * 2 + c / 4) & 7)]) : sc0[q];
                    *reinterpret_cast<uint4*>(bt + n * 128 + ((c ^ (n & 7)) << 4)) = dequant8(v, sc, dk);
                }
                fence_proxy_async_smem();      // generic-proxy writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) mbar_arrive(&bready[s]);
#pragma unroll
                for (int q = 0; q < kChunks; ++q) {
                    sc0[q] = sc1[q];
                    sc1[q] = sc2[q];
                }
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ------------------------------------------------------------------------------------
// CTA-pair kernel (cta_group::2).  Two CTAs of a cluster share one 256 x BNP output tile:
// CTA r holds x rows m0 + 128 r .. + 127 and dequantises weight rows n0 + (BNP/2) r ..
// + BNP/2 - 1; one thread of CTA 0 issues tcgen05.mma.cta_group::2 (M = 256, N = BNP),
// which reads the A and B halves from both CTAs' shared memory, and each CTA's tensor
// memory receives its 128 rows x BNP f32 accumulators.  Per SM this halves the
// shared-memory operand traffic and the dequantisation per flop of a single-CTA tile.
// Both CTAs' dequantise warps arrive on CTA 0's "B ready" barrier and both CTAs'
// epilogue warps on its "accumulator empty" barrier; MMA completion is committed to the
// barriers of both CTAs by one commit addressed to the pair.  Every tensor copy is a plain
// one: each CTA loads its own x and code tiles.

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared::cluster address of `p` (this CTA's shared memory) in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

// Arrive on an mbarrier of a CTA of this cluster (address from peer_addr).  The writes
// the arrival publishes are the dequantised tiles (ordered for the tensor cores by
// fence.proxy.async before the arrive) and completed tensor-memory loads.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Waits on barriers the peer CTA arrives on use the plain bounded wait.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns)
{
    return mbar_wait_bounded(bar, parity, limit_ns);
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n barrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier at the same offset in both CTAs of the pair (the cluster
// ranks set in `mask`) when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_addr(bar)),
        "h"(mask)
        : "memory");
}

// Bulk copy of `bytes` from this CTA's shared memory into another CTA's of this cluster
// (cluster addresses from peer_addr); completion counts on the destination's mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, const void* src, uint32_t bytes,
                                                  uint32_t bar_cluster)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst_cluster),
                 "r"(smem_addr(src)), "r"(bytes), "r"(bar_cluster)
                 : "memory");
}


// Arrive on an mbarrier of a CTA of this cluster, releasing this thread's earlier writes
// (to any CTA's shared memory) at cluster scope.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bounded wait on one of this CTA's mbarriers that acquires, at cluster scope, the writes
// the arriving threads of other CTAs released.
__device__ __forceinline__ bool mbar_wait_acquire_cluster_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns)
{
    auto try_wait = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (try_wait()) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (try_wait()) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

template <int BNP>
struct PairCfg {
    static constexpr int BH = BNP / 2;                            // weight rows per CTA
    static constexpr int kStages = BNP == 256 ? 5 : 7;
    static constexpr uint32_t kABytes = 128 * kBK * 2;            // this CTA's 128 x rows
    static constexpr uint32_t kBBytes = BH * kBK * 2;             // this CTA's dequantised weight rows
    static constexpr uint32_t kRawBytes = BH * (kBK / 2);
    static constexpr uint32_t kScaleBytes = BH * 16;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes + kRawBytes + kScaleBytes;
    static constexpr uint32_t kTxBytes = kABytes + kRawBytes;
    static constexpr uint32_t kTmemCols = 2 * BNP;                // double-buffered 128 x BNP f32
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 256;
    static_assert(kTmemCols == 256 || kTmemCols == 512, "tensor memory columns");
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

// SPL == 2: a cluster of two pairs computes one pair tile, pair j over the j-th half of the
// k range, and owns columns [j, j + 1) * BNP / 2 of the tile.  After its last MMA each CTA
// stages the other pair's column slice of its f32 partial tile in its own (then idle) stage
// ring and, once the other pair announces that its ring is idle too, sends it there with one
// bulk copy (same half of the pair); it then sums its own slice over both partials, in pair
// order, and stores it as bf16.  One tile per cluster: the launch has one cluster per tile.
template <int BNP, int SPL>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_scales, const GemmArgs a)
{
    using C = PairCfg<BNP>;
    constexpr int S = C::kStages;
    constexpr int BH = C::BH;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Per stage: [A tile][B tile][raw codes][scales]; the layout is the same in both CTAs,
    // so one descriptor names the operand halves of both.
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
    uint64_t* full = bars;               // producer -> dequant (own TMA bytes)
    uint64_t* bready = bars + S;         // dequant of both CTAs -> MMA (CTA 0's copy is used)
    uint64_t* empty = bars + 2 * S;      // MMA -> producers of both CTAs (one commit to the pair)
    uint64_t* accfull = bars + 3 * S;    // MMA -> epilogues of both CTAs, 2 buffers
    uint64_t* accempty = accfull + 2;    // epilogues of both CTAs -> MMA (CTA 0's copy)
    uint64_t* drain = accempty + 2;      // final commit on abort
    uint64_t* ring_free = drain + 1;     // SPL == 2: the other pair's ring is idle (4 arrivals)
    uint64_t* recv_full = ring_free + 1; // SPL == 2: the other pair's slice has arrived (bulk copy bytes)
    uint64_t* staged = recv_full + 1;    // SPL == 2: the four epilogue warps staged their rows (4)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(staged + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_rank();
    const uint32_t rank = crank & 1u;                    // half of the pair
    const uint32_t lead = crank & ~1u;                   // cluster rank of the pair's MMA CTA
    const uint16_t pair_mask = (uint16_t)(3u << lead);
    const int ks = (int)(crank >> 1);                    // k range of this pair
    const int kb0 = ks * a.kblocks / SPL, kb1 = (ks + 1) * a.kblocks / SPL;
    const int cluster = blockIdx.x / (2 * SPL), nclusters = gridDim.x / (2 * SPL);
    const int tiles = a.tiles_m * a.tiles_n;
    // SPL == 2, in the idle ring: the slice the other pair sends [128 rows][kRS], then the
    // slice this CTA sends it, staged the same way
    static_assert(SPL == 1 || SPL == 2, "K splits over one or two pairs");
    constexpr int kCols = BNP / SPL;                     // columns a pair owns
    constexpr int kRS = kCols + 4;                       // floats per staged row (spreads the banks)
    constexpr uint32_t kSliceBytes = 128u * kRS * 4u;
    float* rcv = reinterpret_cast<float*>(smem);
    float* snd = rcv + 128 * kRS;
    static_assert(SPL == 1 || 2 * kSliceBytes <= S * C::kStageBytes, "both slices fit the ring");

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bready[s], 2 * kDeqWarps / kDeqGroups);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 8);
        }
        mbar_init(drain, 1);
        mbar_init(ring_free, 4);
        mbar_init(recv_full, 1);
        mbar_init(staged, 4);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_codes);
        if (a.scale_tma) tma_prefetch_desc(&tm_scales);
    }
    if (warp == kMmaWarp) {
        tmem_alloc2(tmem_slot, C::kTmemCols);
        tmem_relinquish2();
    }
    tc_fence_before();
    cluster_sync_all();                  // both CTAs' barriers initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_launch_dependents();
    pdl_wait();

    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.err, kErrWaitTimeout);
    };

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int it = 0;
            int last_phase[16];
            for (int s = 0; s < S; ++s) last_phase[s] = -1;
            for (int t = cluster; t < tiles && !*abort_flag; t += nclusters) {
                const int m0 = (t % a.tiles_m) * 256 + (int)rank * 128;
                const int n0 = (t / a.tiles_m) * BNP + (int)rank * BH;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (uint32_t)(it / S) & 1u;
                    if (!mbar_wait_cluster_bounded(&empty[s], ph ^ 1u, kWaitLimit)) { fail(); break; }
                    if (*abort_flag) break;
                    unsigned char* st = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], C::kTxBytes + (a.scale_tma ? C::kScaleBytes : 0u));
                    tma_load_2d(st, &tm_x, kb * kBK, m0, &full[s]);
                    tma_load_2d(st + C::kABytes + C::kBBytes, &tm_codes, kb * (kBK / 2), n0, &full[s]);
                    if (a.scale_tma)
                        tma_load_2d(st + C::kABytes + C::kBBytes + C::kRawBytes, &tm_scales, (kb * 2) & ~7, n0,
                                    &full[s]);
                    last_phase[s] = (int)ph;
                }
            }
            if (*abort_flag)
                for (int s = 0; s < S; ++s)
                    if (last_phase[s] >= 0) mbar_wait_bounded(&full[s], (uint32_t)last_phase[s], kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        if (rank == 0 && lane == 0) {                      // the pair's even CTA issues its MMAs
            constexpr uint32_t idesc = instr_desc(256, BNP);
            int it = 0, tcount = 0;
            bool issued_any = false;
            for (int t = cluster; t < tiles && !*abort_flag; t += nclusters, ++tcount) {
                const int buf = tcount & 1;
                if (!mbar_wait_cluster_bounded(&accempty[buf], ((uint32_t)(tcount >> 1) & 1u) ^ 1u, kWaitLimit)) {
                    fail();
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait_cluster_bounded(&bready[s], (uint32_t)(it / S) & 1u, kWaitLimit)) {
                        fail();
                        ok = false;
                        break;
                    }
                    if (*abort_flag) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * C::kStageBytes);
                    const uint32_t d = tmem_base + (uint32_t)(buf * BNP);
#pragma unroll
                    for (int j = 0; j < kBK / 16; ++j)
                        mma_bf16_pair(d, sw128_desc(st + j * 32), sw128_desc(st + C::kABytes + j * 32), idesc,
                                      (kb > kb0 || j > 0) ? 1u : 0u);
                    mma_commit_pair(&empty[s], pair_mask);   // both CTAs' stages reusable once read
                    issued_any = true;
                }
                if (!ok) break;
                mma_commit_pair(&accfull[buf], pair_mask);
            }
            if (*abort_flag && issued_any) {
                mma_commit_pair(drain, pair_mask);
                mbar_wait_bounded(drain, 0, kWaitLimit);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        const int quad = warp & 3;             // tensor-memory lanes 32*quad .. 32*quad+31
        int tcount = 0;
        const bool vec_ok = (a.N % 8) == 0 && (reinterpret_cast<uintptr_t>(a.y) & 15) == 0;
        const uint32_t accempty0 = peer_addr(accempty, lead);  // the MMA CTA's accempty[0]; buffer b at + 8 b
        for (int t = cluster; t < tiles && !*abort_flag; t += nclusters, ++tcount) {
            const int buf = tcount & 1;
            if (!mbar_wait_cluster_bounded(&accfull[buf], (uint32_t)(tcount >> 1) & 1u, kWaitLimit)) { fail(); break; }
            tc_fence_after();
            const int row = (t % a.tiles_m) * 256 + (int)rank * 128 + quad * 32 + lane;
            const int n0 = (t / a.tiles_m) * BNP;
            if constexpr (SPL > 1) {
                // This pair's MMAs are done, so its ring is idle: tell the other pair (same
                // half), stage its slice here, and send it once its ring is idle too.
                const int lrow = quad * 32 + lane;             // this thread's row of the CTA's 128
                const int jd = 1 - ks;                          // the other pair
                const uint32_t peer = 2u * (uint32_t)jd + rank;
                if (lane == 0) mbar_arrive_release_cluster(peer_addr(ring_free, peer));
                if (quad == 0 && lane == 0) mbar_arrive_expect_tx(recv_full, kSliceBytes);
#pragma unroll 1
                for (int c0 = 0; c0 < kCols; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BNP + jd * kCols + c0), r);
                    float4* d = reinterpret_cast<float4*>(snd + lrow * kRS + c0);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        d[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                           __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                }
                fence_proxy_async_smem();                       // staged writes -> the bulk copy's reads
                __syncwarp();
                if (lane == 0) mbar_arrive(staged);
                if (quad == 0 && lane == 0) {
                    bool go = mbar_wait_bounded(staged, 0, kWaitLimit);
                    go = go && mbar_wait_acquire_cluster_bounded(ring_free, 0, kWaitLimit);
                    if (go) bulk_copy_to_peer(peer_addr(rcv, peer), snd, kSliceBytes, peer_addr(recv_full, peer));
                    else fail();
                }
                // The other pair issues its copy only after two bounded waits of its own, so
                // this wait is bounded by three limits: no copy into this CTA can still be
                // under way when it gives up.
                if (!mbar_wait_bounded(recv_full, 0, 3 * kWaitLimit)) fail();
                // own slice: the partials in pair order (this pair's from tensor memory)
                const int col0 = n0 + ks * kCols;
                const bool vec_own = (a.N % 8) == 0 && (reinterpret_cast<uintptr_t>(a.y) & 15) == 0;
#pragma unroll 1
                for (int c0 = 0; c0 < kCols; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BNP + ks * kCols + c0), r);
                    float v[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) v[q] = 0.f;
#pragma unroll
                    for (int js = 0; js < SPL; ++js) {
                        if (js == ks) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) v[q] += __uint_as_float(r[q]);
                        } else {
                            const float4* src = reinterpret_cast<const float4*>(rcv + lrow * kRS + c0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 w = src[q];
                                v[4 * q] += w.x;
                                v[4 * q + 1] += w.y;
                                v[4 * q + 2] += w.z;
                                v[4 * q + 3] += w.w;
                            }
                        }
                    }
                    const int col = col0 + c0;
                    if (row < a.M) {
                        uint16_t* dst = a.y + (size_t)row * a.N + col;
                        if (vec_own && col + 16 <= a.N) {
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                uint4 o;
                                o.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
                                o.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
                                o.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
                                o.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
                                *reinterpret_cast<uint4*>(dst + 8 * q) = o;
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                if (col + q < a.N) dst[q] = (uint16_t)(pack_bf16x2(v[q], 0.f) & 0xFFFFu);
                        }
                    }
                }
            }
#pragma unroll 1
            for (int c0 = 0; c0 < (SPL > 1 ? 0 : BNP); c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BNP + c0), r);
                const int col = n0 + c0;
                if (row < a.M) {
                    uint16_t* dst = a.y + (size_t)row * a.N + col;
                    if (vec_ok && col + 32 <= a.N) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
                            o.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
                            o.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
                            o.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
                            *reinterpret_cast<uint4*>(dst + 8 * q) = o;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            if (col + q < a.N) dst[q] = (uint16_t)(pack_bf16x2(__uint_as_float(r[q]), 0.f) & 0xFFFFu);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(accempty0 + 8u * (uint32_t)buf);
        }
    } else {
        // Dequantise this CTA's BH weight rows.  The dequantising warps form kDeqGroups
        // groups that take alternate stages, so a group has kDeqGroups stage periods for
        // the latency of one stage (shared-memory reads, the proxy fence and the remote
        // arrival); each thread owns BH*8/(threads of a group) chunks (row n, 16-byte k
        // chunk c) of its stages.
        constexpr int kGroupThreads = kDeqWarps * 32 / kDeqGroups;
        const int dq = threadIdx.x - kDeqWarp0 * 32;
        const int grp = dq / kGroupThreads, dt = dq - grp * kGroupThreads;
        constexpr int kChunks = BH * 8 / kGroupThreads;
        const DequantConsts dk;
        const uint32_t bready0 = peer_addr(bready, lead);      // the MMA CTA's bready[0]; stage s at + 8 s
        int it = 0;
        for (int t = cluster; t < tiles && !*abort_flag; t += nclusters) {
            const int n0 = (t / a.tiles_m) * BNP + (int)rank * BH;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                if (it % kDeqGroups != grp) continue;
                float scv[kChunks];
                if (!a.scale_tma) {                // issued before the wait, which hides their latency
#pragma unroll
                    for (int q = 0; q < kChunks; ++q) {
                        const int idx = dt + q * kGroupThreads;
                        const int n = n0 + idx / 8, g = kb * 2 + (idx & 7) / 4;
                        scv[q] = (n < a.N && g < a.G)
                                     ? __half2float(__ushort_as_half(__ldg(a.scales + (size_t)n * a.G + g)))
                                     : 0.f;
                    }
                }
                const int s = it % S;
                if (!mbar_wait_bounded(&full[s], (uint32_t)(it / S) & 1u, kWaitLimit)) { fail(); ok = false; break; }
                if (*abort_flag) { ok = false; break; }
                unsigned char* st = smem + s * C::kStageBytes;
                unsigned char* bt = st + C::kABytes;
                const unsigned char* raw = bt + C::kBBytes;
                const __half* sst = reinterpret_cast<const __half*>(raw + C::kRawBytes);
#pragma unroll
                for (int q = 0; q < kChunks; ++q) {
                    const int idx = dt + q * kGroupThreads;
                    const int n = idx >> 3, c = idx & 7;
                    const uint32_t v = *reinterpret_cast<const uint32_t*>(raw + n * 32 + c * 4);
                    const float sc = a.scale_tma ? __half2float(sst[n * 8 + ((kb * 2 + c / 4) & 7)]) : scv[q];
                    *reinterpret_cast<uint4*>(bt + n * 128 + ((c ^ (n & 7)) << 4)) = dequant8(v, sc, dk);
                }
                fence_proxy_async_smem();      // generic-proxy writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(bready0 + 8u * (uint32_t)s);
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                  // no CTA leaves while the pair's MMAs may read its shared memory
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc2(tmem_base, C::kTmemCols);
}

template <int BNP, int SPL>
bool setup_pair_kernel(size_t* smem)
{
    *smem = PairCfg<BNP>::kSmem;
    const void* fn = reinterpret_cast<const void*>(&gemm_pair_kernel<BNP, SPL>);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess) {
        cudaGetLastError();
    }
    return blocks_per_sm(fn, kThreads, *smem) >= 1;
}

template <int MA, int BN>
bool setup_kernel(size_t* smem)
{
    *smem = GemmCfg<MA, BN>::kSmem;
    return blocks_per_sm(reinterpret_cast<const void*>(&gemm_tc_kernel<MA, BN>), kThreads, *smem) >= 1;
}

}  // namespace

namespace {

std::mutex g_cluster_mutex;
struct ClusterCap {
    int device;
    const void* fn;
    int capacity;
};
ClusterCap g_cluster_cap[16];
int g_cluster_cap_used = 0;

// How many clusters of the pair kernel <BNP, SPL> (2 * SPL CTAs each) can be resident
// at once on the current device (0 when none can, or the query fails); cached.
template <int BNP, int SPL>
int pair_cluster_capacity(const DeviceInfo& dev)
{
    const void* fn = reinterpret_cast<const void*>(&gemm_pair_kernel<BNP, SPL>);
    {
        std::lock_guard<std::mutex> lock(g_cluster_mutex);
        for (int i = 0; i < g_cluster_cap_used; ++i)
            if (g_cluster_cap[i].device == dev.device && g_cluster_cap[i].fn == fn) return g_cluster_cap[i].capacity;
    }
    size_t smem = 0;
    int capacity = 0;
    if (setup_pair_kernel<BNP, SPL>(&smem)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * SPL));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2 * SPL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&capacity, gemm_pair_kernel<BNP, SPL>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            capacity = 0;
        }
    }
    std::lock_guard<std::mutex> lock(g_cluster_mutex);
    if (g_cluster_cap_used < 16) g_cluster_cap[g_cluster_cap_used++] = {dev.device, fn, capacity};
    return capacity;
}

// The CTA-pair kernel with BNP output columns per pair tile; SPL pairs per cluster split
// K (one tile per cluster), SPL == 1 is persistent over the tiles.
template <int BNP, int SPL>
q4_status launch_gemm_pair(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed, const uint16_t* scales,
                           int64_t N, uint16_t* y, cudaStream_t stream, const DeviceInfo& dev)
{
    constexpr int BH = BNP / 2;
    CUtensorMap tm_x, tm_codes;
    if (!encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, kBK, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tma_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                       kBK / 2, (uint32_t)BH, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    CUtensorMap tm_scales = tm_codes;
    const bool scale_tma = (K / 32) % 8 == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
    if (scale_tma && !encode_tma_2d(&tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, scales, (uint64_t)(K / 32),
                                    (uint64_t)N, (uint64_t)(K / 32) * 2, 8, (uint32_t)BH, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return Q4_ERR_CUDA;
    GemmArgs a;
    a.scales = scales;
    a.scale_tma = scale_tma ? 1 : 0;
    a.y = y;
    a.err = err;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.G = (int)(K / 32);
    a.tiles_m = (int)((M + 255) / 256);
    a.tiles_n = (int)((N + BNP - 1) / BNP);
    a.kblocks = (int)((K + kBK - 1) / kBK);
    const long long tiles = (long long)a.tiles_m * a.tiles_n;
    size_t smem = 0;
    if (!setup_pair_kernel<BNP, SPL>(&smem)) return Q4_ERR_CUDA;
    const long long clusters = SPL > 1 ? tiles : std::min<long long>(tiles, dev.sm_count / 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * SPL * clusters));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2 * SPL;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<BNP, SPL>, tm_x, tm_codes, tm_scales, a);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace

q4_status launch_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed, const uint16_t* scales,
                      int64_t N, uint16_t* y, cudaStream_t stream, const DeviceInfo& dev)
{
    // CTA pairs (256-row tiles) from M = 256 on.  A pair's k-block takes about the same
    // time with 128 output columns as with 256 (measured on B200: 0.45-0.5 us against
    // 0.55-0.6 us), so 256 x 256 tiles are used throughout; when they leave at least half
    // of the SM pairs idle, two pairs share each tile's K range (clusters of 4 CTAs, each
    // pair at least 4 k-blocks) as long as every cluster can be resident at once; else
    // 256 x 128 tiles when 256 x 256 ones would occupy fewer than half of the pairs.
    if (M >= 256 && dev.sm_count >= 2) {
        const long long p256 = ((M + 255) / 256) * ((N + 255) / 256);
        const long long pairs = dev.sm_count / 2;
        const long long kblocks = (K + kBK - 1) / kBK;
        if (p256 * 2 <= pairs && kblocks >= 8 && pair_cluster_capacity<256, 2>(dev) >= p256)
            return launch_gemm_pair<256, 2>(x, M, K, packed, scales, N, y, stream, dev);
        if (2 * p256 >= pairs) return launch_gemm_pair<256, 1>(x, M, K, packed, scales, N, y, stream, dev);
        return launch_gemm_pair<128, 1>(x, M, K, packed, scales, N, y, stream, dev);
    }
    // Tile shape: 256 x 128 when that still gives every SM a tile, else 128 x 128, else 128 x 64.
    const long long t256 = ((M + 255) / 256) * ((N + 127) / 128);
    const long long t128 = ((M + 127) / 128) * ((N + 127) / 128);
    int MA = 1, BN = 64;
    if (t256 >= dev.sm_count) { MA = 2; BN = 128; }
    else if (t128 >= dev.sm_count) { MA = 1; BN = 128; }

    CUtensorMap tm_x, tm_codes;
    if (!encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, kBK, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tma_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                       kBK / 2, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    // Scales by TMA when a row of them is a whole number of 16-byte units and 16-byte aligned.
    CUtensorMap tm_scales = tm_codes;
    const bool scale_tma = (K / 32) % 8 == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
    if (scale_tma && !encode_tma_2d(&tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, scales, (uint64_t)(K / 32),
                                    (uint64_t)N, (uint64_t)(K / 32) * 2, 8, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return Q4_ERR_CUDA;

    GemmArgs a;
    a.scales = scales;
    a.scale_tma = scale_tma ? 1 : 0;
    a.y = y;
    a.err = err;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.G = (int)(K / 32);
    a.tiles_m = (int)((M + 128 * MA - 1) / (128 * MA));
    a.tiles_n = (int)((N + BN - 1) / BN);
    a.kblocks = (int)((K + kBK - 1) / kBK);
    const int tiles = a.tiles_m * a.tiles_n;

    size_t smem = 0;
    bool ok = MA == 2 ? setup_kernel<2, 128>(&smem) : BN == 128 ? setup_kernel<1, 128>(&smem)
                                                                : setup_kernel<1, 64>(&smem);
    if (!ok) return Q4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles < dev.sm_count ? tiles : dev.sm_count));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (MA == 2) e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<2, 128>, tm_x, tm_codes, tm_scales, a);
    else if (BN == 128) e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<1, 128>, tm_x, tm_codes, tm_scales, a);
    else e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<1, 64>, tm_x, tm_codes, tm_scales, a);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
