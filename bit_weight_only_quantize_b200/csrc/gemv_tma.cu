// q4_gemv / q4_gemv_multi for the shapes the TMA path serves (K % 256 == 0, scales
// 16-byte aligned; M = 1 with f32 or bf16 x, M = 2..16 with bf16 x).
//
// Decode streams every weight once, so the kernels are built around keeping HBM busy
// and spending few instructions per weight (QORA-LLM-0.8B model card, section "AVX-512
// SIMD Acceleration": a Q4 GEMV whose nibbles go through a 16-entry table; QORA-4B
// thread, section "量化与内存管理": GEMV over Q4 weights on a thread pool):
//
//  * Weights stream as TMA boxes of 16 rows x 8 groups (2 KiB of codes, 128-byte
//    swizzled); a ring stage holds kBoxesPerStage consecutive boxes plus one box of
//    their binary16 scales under one mbarrier.  Each warp keeps its own ring of kStages
//    stages and issues its own copies (lane 0), so every warp has about 9 KiB in flight.
//  * Work is cut into row blocks of 16 rows, enumerated over one or more weight
//    matrices that share x (one launch for a set of projections of the same token).
//    Teams of P warps own sequences of row blocks; the P warps of a team take
//    disjoint K ranges of each block and add their partial sums in a fixed order.
//    Skinny shapes may also split K across blocks (last-arriver reduction, no
//    waiting).  The plan picks splits, P and teams per block with a small cost model.
//  * Arithmetic per mode:
//      M = 1 (kImma1, f32 or bf16 x): no code becomes a float.  Each box of 256 x values
//          (8 groups) is scaled by a power of two 2^F (max |x| of the box * 2^F < 2^30),
//          rounded once to integers and cut into four balanced base-256 digit planes;
//          the codes stay bytes (even k as is, odd k at 16 x code, one AND each) and
//          mma.sync.m16n8k32 (u8 codes x s8 digits) sums code x digit exactly in int32,
//          the eight B columns being (plane, even/odd half).  The C operand, a bias
//          0x4B400000 minus 8 (or 128) x the digit sum, removes the code offset 8 and
//          makes the int32 result the bit pattern of the exact float 1.5 * 2^23 + sum.
//          Each group's sum is multiplied by its scale, the box's sums by 2^-F, and
//          accumulated in f32 per plane; the planes are combined at the end.
//      M = 2..16 (bf16 x): byte j of a code word (codes 2j, 2j+1) placed by one PRMT
//          and OR-ed into 0x4300 (one LOP3) is the bf16 pair (128 + c_2j, 128 + c_2j+1);
//          one exact bf16x2 subtraction of 136 makes it (c_2j - 8, c_2j+1 - 8).  Such
//          pairs, read with ldmatrix, are the A operand of mma.sync.m16n8k16 and x rows,
//          as they arrive, the B operand (both in k order); every product is exact and
//          the group's sum is accumulated in f32 from zero.
//    In every mode each group's sum is scaled by its binary16 scale and added in f32.
//  * Every mbarrier wait is bounded.  If one runs out the kernel records
//    kErrWaitTimeout in the library error word, stops issuing and computing, waits
//    (bounded) for its own copies still in flight and returns (see q4_device_error).
#include <algorithm>

#include "tma.cuh"
#include "topk.cuh"

namespace q4 {
namespace {

constexpr int kRows = 16;                    // rows per row block
constexpr int kMaxWarps = 16;
constexpr int kStages = 2;
constexpr int kBoxesPerStage = 2;            // code boxes per ring stage (one mbarrier)
constexpr uint32_t kCodeBox = kRows * 128;   // bytes of codes per box (8 groups)
constexpr uint32_t kScaleBox = kRows * 16;   // bytes of scales per box
constexpr uint32_t kStageCodes = kBoxesPerStage * kCodeBox;
constexpr uint32_t kStageScales = kBoxesPerStage * kScaleBox;   // one box of 8 * kBoxesPerStage groups
constexpr uint64_t kWaitLimit = kWaitLimitNs;
constexpr int kCounterSlots = 1024;          // same workspace layout as the generic kernel
// Plan cost model, in units of the time one warp takes for a stage unit when 16 warps
// share the SM (measured on B200: about 2.7 us).  A warp with fewer neighbours is
// faster only down to the pace of kMinWarpShare warps (its own dependency chains and
// memory latency bound it); the row-block epilogue (team reduction, stores) and the
// split-K reduction (partials through L2 and an atomic per row block) add fixed costs.
constexpr double kMinWarpShare = 12.0;
constexpr double kEpilogueCost = 0.1;
constexpr double kSplitCost = 0.9;
constexpr int kStagingWarps = 8;              // fewest warps per block (extra ones only stage x)
constexpr size_t kCounterBytes = kCounterSlots * sizeof(unsigned);

// kImma1: one x row on the integer tensor cores; kMma8 / kMma16: 2..8 / 9..16 bf16 x rows.
enum Mode { kMma8 = 1, kMma16 = 2, kImma1 = 4 };

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
    int x_f32;                        // kImma1: x is f32 (else bf16)
    int fmt[Q4_MULTI_MAX];            // kImma1: 1 = matrix i holds INT8 codes [N][K], 0 = Q4
    int has_int8;                     // some matrix is INT8 (the natural-order digits are staged)
    uint64_t wait_ns;                 // limit of the waits for this warp's copies (0: give up at once)
    // kEpiArgmax (greedy argmax over the rows of matrix 0, splits == 1): per x row, the
    // largest logit and its row; keys and the block counter live in a workspace that is
    // zero at rest.  (kEpiFuse: matrices 0 and 1 are gate and up, y = silu(y0) * y1 into y[0].)
    // kEpiTopk (the k largest logits of matrix 0, splits == 1): each team keeps a sorted
    // list per x row, each block merges its teams' lists into tk_cand [M][gridDim.x][k],
    // and the last block merges those.  Rows are reported as row_base + row.
    unsigned long long* am_key;       // [M] (value order, then lowest row)
    unsigned* am_done;                // blocks finished
    long long* am_index;              // [M] output ([M][k] for top-k)
    float* am_value;                  // [M] output ([M][k]), may be null
    unsigned long long* tk_cand;      // top-k: per-block lists
    unsigned long long* tk_floor;     // top-k, M == 1: the largest k-th key any team has published
    int tk_k;                         // top-k: list length, 1..32
    unsigned row_base;                // argmax / top-k: added to every reported row
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

// (a & m) | c as one LOP3; m and c are kept in registers (pinned) by the callers, since the
// instruction takes a single immediate.
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

// Nibble pair (j, j+4) of a word as the bf16 pair (128 + c_j, 128 + c_{j+4}); mask and
// magic are the registers holding 0x000F000F and 0x43004300.
// Byte j of a code word as the bf16 pair (128 + low nibble, 128 + high nibble): codes
// 2j and 2j + 1 of the word in k order.  v4 = v >> 4 puts each high nibble where PRMT
// can take it (byte j of v into the low half, byte j of v4 into the high half).
__device__ __forceinline__ uint32_t byte_pair(uint32_t v, uint32_t v4, int j, uint32_t mask, uint32_t magic)
{
    return and_or(__byte_perm(v, v4, (uint32_t)(j | ((4 + j) << 8))), mask, magic);
}

// (128 + c) - 136 = c - 8 for both bf16 halves; exact (small integers).
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// d = A . B for one m16n8k16 tile (bf16 inputs, f32 accumulate from zero).
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Four 8x8 b16 matrices from shared memory; lane 8i + r supplies the address of row r of
// matrix i and lane (g, t) receives the 32-bit word (row g, columns 2t, 2t+1) of each.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// d = A . B + c for one m16n8k16 tile (bf16 inputs, f32 accumulate).
// d += A . B for one m16n8k16 tile (bf16 inputs, f32 accumulate).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A . B + c for one m16n8k32 tile: A unsigned 8-bit, B signed 8-bit, exact int32
// accumulation.
__device__ __forceinline__ void imma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1, int c0, int c1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1));
}

// d = A . B + c for one m16n8k32 tile of signed 8-bit operands, exact int32 accumulation.
__device__ __forceinline__ void imma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1, int c0, int c1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1));
}

// Integer MMA results are read as f32 through a bias: the bit pattern 0x4B400000 is
// 1.5 * 2^23, and adding an integer |v| < 2^22 to it gives the float 1.5 * 2^23 + v.
constexpr int kBiasBits = 0x4B400000;
// A lo-nibble column holds bias + T_lo and its hi-nibble column bias + 16 T_hi, so
// hi * (1/16) + lo = (17/16) * 1.5 * 2^23 + T_lo + T_hi, an integer below 2^24 (exact).
constexpr float kBias17 = 13369344.0f;
constexpr float kBiasF = 12582912.0f;          // 1.5 * 2^23, the float of kBiasBits

__device__ __forceinline__ float scale_at(const uint4& s8, int c)
{
    const uint32_t sw = c < 2 ? s8.x : c < 4 ? s8.y : c < 6 ? s8.z : s8.w;
    return __half2float(__ushort_as_half((unsigned short)((c & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
}

// Eight x values (k = 8t .. 8t+7 of a group) as balanced base-256 digit planes of
// X = rint(v * x_scale) (|X| < 2^30): X = d0 2^24 + d1 2^16 + d2 2^8 + d3, d1..d3 in
// [-128, 127].  The digits' bytes are bytes of X plus carries: d3 = byte 0 of X, d2 = byte
// 1 of X + 0x80, d1 = byte 2 of X + 0x8080, d0 = byte 3 of X + 0x808080 (each read as a
// signed byte).  word[p][h] packs plane p's digits of k = 8t + h, + 2, + 4, + 6 (byte i =
// k 8t + 2i + h); dsum[p][h] is their sum.
__device__ __forceinline__ void digits8(const float (&v)[8], float x_scale, uint32_t (&word)[4][2], int (&dsum)[4][2],
                                        uint32_t (*nat)[2] = nullptr)
{
    int X[8], Y1[8], Y2[8], Y3[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        X[e] = __float2int_rn(__fmul_rn(v[e], x_scale));
        Y1[e] = (int)((uint32_t)X[e] + 0x80u);        // wraps (defined) only for non-finite x
        Y2[e] = (int)((uint32_t)X[e] + 0x8080u);
        Y3[e] = (int)((uint32_t)X[e] + 0x808080u);
    }
    if (nat) {        // natural k order: nat[p][0] = plane p of k 8t .. 8t+3, nat[p][1] = 8t+4 .. 8t+7
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = 4 * h;
            nat[3][h] = __byte_perm(__byte_perm(X[e], X[e + 1], 0x0040), __byte_perm(X[e + 2], X[e + 3], 0x0040), 0x5410);
            nat[2][h] = __byte_perm(__byte_perm(Y1[e], Y1[e + 1], 0x0051), __byte_perm(Y1[e + 2], Y1[e + 3], 0x0051), 0x5410);
            nat[1][h] = __byte_perm(__byte_perm(Y2[e], Y2[e + 1], 0x0062), __byte_perm(Y2[e + 2], Y2[e + 3], 0x0062), 0x5410);
            nat[0][h] = __byte_perm(__byte_perm(Y3[e], Y3[e + 1], 0x0073), __byte_perm(Y3[e + 2], Y3[e + 3], 0x0073), 0x5410);
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        word[3][h] = __byte_perm(__byte_perm(X[h], X[h + 2], 0x0040), __byte_perm(X[h + 4], X[h + 6], 0x0040), 0x5410);
        word[2][h] = __byte_perm(__byte_perm(Y1[h], Y1[h + 2], 0x0051), __byte_perm(Y1[h + 4], Y1[h + 6], 0x0051), 0x5410);
        word[1][h] = __byte_perm(__byte_perm(Y2[h], Y2[h + 2], 0x0062), __byte_perm(Y2[h + 4], Y2[h + 6], 0x0062), 0x5410);
        word[0][h] = __byte_perm(__byte_perm(Y3[h], Y3[h + 2], 0x0073), __byte_perm(Y3[h + 4], Y3[h + 6], 0x0073), 0x5410);
        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
        for (int e = h; e < 8; e += 2) {
            const int x1 = Y1[e] >> 8, x2 = Y2[e] >> 16, x3 = Y3[e] >> 24;   // arithmetic shifts
            s3 += (int)((uint32_t)X[e] - ((uint32_t)x1 << 8));
            s2 += (int)((uint32_t)x1 - ((uint32_t)x2 << 8));
            s1 += (int)((uint32_t)x2 - ((uint32_t)x3 << 8));
            s0 += x3;
        }
        dsum[0][h] = s0;
        dsum[1][h] = s1;
        dsum[2][h] = s2;
        dsum[3][h] = s3;
    }
}

template <int MODE>
struct ModeCfg {
    static constexpr int MP = MODE == kMma16 ? 16 : MODE == kMma8 ? 8 : 1;   // x rows in red[]
    static constexpr int NT = MP >= 8 ? MP / 8 : 1;                          // n-tiles of 8 x rows
    static constexpr int kMinBlocks = 1;
};

// Row-block epilogues: plain stores, fused gate+up, greedy argmax (compile-time, so the
// plain GEMV carries none of the others' code or registers).
enum Epi { kEpiPlain = kGemvPlain, kEpiFuse = kGemvFuse, kEpiArgmax = kGemvArgmax, kEpiTopk = kGemvTopk };

template <int MODE, int EPI>
__global__ void __launch_bounds__(kMaxWarps * 32, ModeCfg<MODE>::kMinBlocks)
gemv_tma_kernel(const __grid_constant__ TmaMaps maps, const TmaGemvArgs a)
{
    constexpr int MP = ModeCfg<MODE>::MP;
    constexpr int NT = ModeCfg<MODE>::NT;
    constexpr bool kFuse = EPI == kEpiFuse;
    constexpr bool kArgmax = EPI == kEpiArgmax;
    constexpr bool kTopk = EPI == kEpiTopk;
    constexpr int kTkM = MODE == kImma1 ? 1 : MP;                         // x rows of a top-k list set
    extern __shared__ unsigned char smem_raw[];
    __shared__ int s_last[kMaxWarps];
    __shared__ unsigned long long s_best[kArgmax ? kMaxWarps : 1];        // argmax, one x row
    __shared__ uint64_t s_xbar;                                            // kMma*: x rows in flight
    const int W = blockDim.x >> 5;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* codes = smem;                                          // [warp][stage][box][2048]
    unsigned char* scl = codes + W * kStages * kStageCodes;               // [warp][stage][16 rows][8 * boxes]
    uint64_t* bars = reinterpret_cast<uint64_t*>(scl + W * kStages * kStageScales);   // [warp][stage]
    float* red = reinterpret_cast<float*>(bars + W * kStages);            // [warp][16 rows][MP]
    unsigned char* xst = reinterpret_cast<unsigned char*>(                 // staged x, 16-byte aligned
        (reinterpret_cast<uintptr_t>(red + W * kRows * MP) + 15) & ~uintptr_t(15));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = a.P;
    const int team = warp / P, wt = warp - team * P;
    const bool active = team < a.teams;
    const int split = blockIdx.y;
    const int g0 = split * a.ksg;
    const int ng = min(a.G - g0, a.ksg);
    const int nb = (ng + 7) >> 3;                                         // boxes of this split
    const int ngp = nb * 8;                                               // groups, padded
    const int nu = (nb + kBoxesPerStage - 1) / kBoxesPerStage;            // stage units of this split
    const int u0 = wt * nu / P, nbw = (wt + 1) * nu / P - u0;             // this warp's units
    // INT8 matrices (kImma1): a box holds 4 groups (16 rows x 128 bytes), so a split has
    // twice the boxes and units of a Q4 matrix.
    const int nb8 = (ng + 3) >> 2;
    const int nu8 = (nb8 + kBoxesPerStage - 1) / kBoxesPerStage;
    const int u08 = wt * nu8 / P, nbw8 = (wt + 1) * nu8 / P - u08;
    const bool mixed = MODE == kImma1 && a.has_int8;
    // A team walks row blocks first_rb, first_rb + rb_stride, ...  With fuse it walks the
    // row-block pairs of the gate and up matrices instead, visiting gate block p and then
    // up block p (= p + the gate's block count) of each pair in turn.
    const int first_rb = blockIdx.x * a.teams + team;
    const int rb_stride = gridDim.x * a.teams;
    const int walk = kFuse ? a.rb_begin[1] : a.row_blocks;
    const int nwalk = (active && first_rb < walk) ? (walk - first_rb + rb_stride - 1) / rb_stride : 0;
    const int nrb = kFuse ? 2 * nwalk : nwalk;                           // row-block visits
    auto rb_of = [&](int i) {
        return kFuse ? first_rb + (i >> 1) * rb_stride + (i & 1) * a.rb_begin[1] : first_rb + i * rb_stride;
    };
    // INT8 row block: the matrix of row block rb holds INT8 codes
    auto is_int8 = [&](int rb) { return mixed && a.fmt[matrix_of(a, rb)] != 0; };
    int njobs = nrb * nbw;
    if (mixed) {
        njobs = 0;
        for (int i = 0; i < nrb; ++i) njobs += is_int8(rb_of(i)) ? nbw8 : nbw;
    }
    uint64_t* my_bars = bars + warp * kStages;
    const size_t K = (size_t)a.G * 32;

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // Job j: unit (u0 + j % nbw) of the warp's (j / nbw)-th row block; a unit is up to
    // kBoxesPerStage consecutive code boxes plus one scale box spanning all of them.  Jobs
    // are issued in order, so a cursor (unit, row block and its matrix) replaces the
    // division and the matrix lookup.
    // A row block in which this warp has no unit (possible when a team's warps split an
    // INT8 and a Q4 row block differently) is skipped.
    int iss_u = 0, iss_vis = 0, iss_mi = 0, iss_lrow = 0, iss_i8 = 0;
    auto locate = [&]() {
        while (true) {
            const int rb = rb_of(iss_vis);
            iss_mi = matrix_of(a, rb);
            iss_lrow = (rb - a.rb_begin[iss_mi]) * kRows;
            iss_i8 = mixed && a.fmt[iss_mi] != 0;
            if ((iss_i8 ? nbw8 : nbw) > 0 || iss_vis + 1 >= nrb) break;
            ++iss_vis;
        }
    };
    if (lane == 0 && njobs > 0) locate();
    auto issue = [&](int j) {
        const int s = j % kStages;
        const int bf = ((iss_i8 ? u08 : u0) + iss_u) * kBoxesPerStage;
        const int nbox = min(kBoxesPerStage, (iss_i8 ? nb8 : nb) - bf);
        const int gpb = iss_i8 ? 4 : 8;                                   // groups per box
        uint64_t* bar = &my_bars[s];
        const CUtensorMap* cmap = &maps.codes[iss_mi];
        unsigned char* dst = codes + (warp * kStages + s) * kStageCodes;
        mbar_arrive_expect_tx(bar, nbox * kCodeBox + (iss_i8 ? kStageScales / 2 : kStageScales));
        for (int q = 0; q < nbox; ++q)
            tma_load_2d(dst + q * kCodeBox, cmap, (g0 + gpb * (bf + q)) * (iss_i8 ? 32 : 16), iss_lrow, bar);
        tma_load_2d(scl + (warp * kStages + s) * kStageScales, &maps.scales[iss_mi], g0 + gpb * bf, iss_lrow, bar);
        if (++iss_u == (iss_i8 ? nbw8 : nbw)) {
            iss_u = 0;
            ++iss_vis;
            if (j + 1 < njobs) locate();
        }
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

    // ---- stage x for this split (zero past the split and past K) ----
    //  kMma* : x rows [m][group][32 bf16] in k order for m < M, then one zero row that
    //          lanes of x rows >= M read; each row is padded by one group so that lanes
    //          of neighbouring x rows fall on different banks.
    //  kImma1: each box of 8 groups (256 x values) is scaled by 2^F (the largest F with
    //          max |x| of the box * 2^F < 2^30, at most 100), rounded to integers X and
    //          cut into four balanced base-256 digits X = d0 2^24 + d1 2^16 + d2 2^8 + d3,
    //          d1..d3 in [-128, 127].  The MMA's eight B columns are (digit plane p,
    //          nibble half h) = column 2p + h: half 0 holds the digits of the even k of
    //          the group (the low nibbles), half 1 those of the odd k (the high nibbles,
    //          which the A operand keeps at 16 x code).  [group pair][column g][t] uint4
    //          holds the two B registers of lane (g, t) for both groups of the pair, the
    //          slots of the other half zero.  Then [group pair][plane][4] int: the C
    //          operand per group and plane, bias - 8 sum(d of even k) for half 0 and
    //          bias - 128 sum(d of odd k) for half 1, which removes the code offset 8.
    //          Then [box] float: 2^-F.  One pass: the 32 lanes that stage a box find its
    //          maximum with five shuffles, so no block-wide reduction is needed.
    const int rs = (ngp + 1) * 4;                                         // uint4 per staged x row
    bool x_ok = true;                                                     // kMma*: x rows arrived
    if constexpr (MODE == kImma1) {
        const int items = ngp * 4;                                        // (group, k = 8t .. 8t+7)
        uint2* xq = reinterpret_cast<uint2*>(xst);
        int2* xc = reinterpret_cast<int2*>(xst + (size_t)ngp * 256);
        float* xf = reinterpret_cast<float*>(xst + (size_t)ngp * 288);
#pragma unroll 2
        for (int i0 = threadIdx.x - lane; i0 < items; i0 += blockDim.x) {    // warp-uniform trips
            const int i = i0 + lane;
            const int lg = i >> 2, t = i & 3;
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
            if (i < items && lg < ng) {
                const size_t k0 = (size_t)(g0 + lg) * 32 + t * 8;
                if (a.x_f32) {
                    const float4 p = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + k0);
                    const float4 q = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + k0 + 4);
                    v[0] = p.x; v[1] = p.y; v[2] = p.z; v[3] = p.w; v[4] = q.x; v[5] = q.y; v[6] = q.z; v[7] = q.w;
                } else {
                    const uint4 r = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x) + k0);
                    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[2 * e] = __uint_as_float(w[e] << 16);
                        v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                    }
                }
            }
            // the group's max |x| (bit patterns of non-negative floats order as the values)
            uint32_t mx = 0u;
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = max(mx, __float_as_uint(v[e]) & 0x7FFFFFFFu);
            // the warp's 32 items are the 8 groups of one box: one exponent per box
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            // F: 100 for a zero or subnormal maximum, 0 for a non-finite one (the product
            // is then undefined, but every step stays defined)
            const int ex = (int)(mx >> 23);
            const int F = ex == 0 ? 100 : ex >= 255 ? 0 : min(29 - (ex - 127), 100);
            uint32_t word[4][2];
            int dsum[4][2];
            uint32_t nat[4][2];
            digits8(v, __uint_as_float((uint32_t)(F + 127) << 23), word, dsum, mixed ? nat : nullptr);
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    dsum[p][h] += __shfl_xor_sync(0xffffffffu, dsum[p][h], 1);
                    dsum[p][h] += __shfl_xor_sync(0xffffffffu, dsum[p][h], 2);
                }
            if (i < items) {
                const int gp = lg >> 1, half = lg & 1;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    xq[(((gp * 8 + 2 * p) * 4 + t) << 1) + half] = make_uint2(word[p][0], 0u);
                    xq[(((gp * 8 + 2 * p + 1) * 4 + t) << 1) + half] = make_uint2(0u, word[p][1]);
                    if (t == 0)
                        xc[((gp * 4 + p) << 1) + half] = make_int2(kBiasBits - 8 * dsum[p][0], kBiasBits - 128 * dsum[p][1]);
                }
                if (lane == 0) xf[lg >> 3] = __uint_as_float((uint32_t)(127 - F) << 23);
                if (mixed) {
                    // INT8 operands, natural k order: [group][column g][t'] uint2 = (k 4t'..4t'+3,
                    // k 16 + 4t' .. 16 + 4t'+3) of plane g for g < 4, zero for g >= 4; this
                    // item's k = 8t .. 8t+7 are the chunks 2t and 2t+1 of 4.
                    uint32_t* x8 = reinterpret_cast<uint32_t*>(xst + (size_t)ngp * 292);
                    const int hf = t >> 1;
#pragma unroll
                    for (int p = 0; p < 4; ++p)
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const int tq = (2 * t + c) & 3;
                            x8[((lg * 8 + p) * 4 + tq) * 2 + hf] = nat[p][c];
                            x8[((lg * 8 + p + 4) * 4 + tq) * 2 + hf] = 0u;
                        }
                }
            }
        }
    } else {
        uint4* xp = reinterpret_cast<uint4*>(xst);
        // The split's part of each x row arrives by one bulk copy, in k order, where the
        // MMAs read it (all rows in flight at once); the groups past the split's end
        // and the zero row are cleared meanwhile.
        if (threadIdx.x == 0) {
            mbar_init(&s_xbar, 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(&s_xbar, (uint32_t)(a.M * ng * 64));
            for (int m = 0; m < a.M; ++m)
                bulk_load(xp + m * rs, reinterpret_cast<const uint16_t*>(a.x) + (size_t)m * K + (size_t)g0 * 32,
                          (uint32_t)(ng * 64), &s_xbar);
        }
        const int tail = (ngp - ng) * 4;                                  // uint4 past the split per row
        for (int i = threadIdx.x; i < a.M * tail + ngp * 4; i += blockDim.x) {
            const int m = i < a.M * tail ? i / tail : a.M;
            const int w = i < a.M * tail ? ng * 4 + (i - m * tail) : i - a.M * tail;
            xp[m * rs + w] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncthreads();
        x_ok = mbar_wait_bounded(&s_xbar, 0, kWaitLimit);
    }
    __syncthreads();

    const uint32_t kmask = pinned_u32(0x000F000Fu), kmagic = pinned_u32(0x43004300u);
    const uint32_t k136 = pinned_u32(0x43084308u);                        // bf16x2 (136, 136)
    // MMA modes: lane (g, t) supplies the B operand of x row n * 8 + g (the zero row past M).
    const uint4* xrow[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) xrow[n] = reinterpret_cast<const uint4*>(xst) + min(n * 8 + (lane >> 2), a.M) * rs;

    bool ok = x_ok;
    int consumed = 0;
    float gsave[kFuse ? kRows * Q4_GEMV_MAX_M / 32 : 1];   // fuse: the gate totals of the current pair
    unsigned long long tk[kTopk ? kTkM + 1 : 1];           // top-k: the team's list per x row
#pragma unroll
    for (int i = 0; i < (kTopk ? kTkM + 1 : 1); ++i) tk[i] = 0ull;
    // Top-k with one x row: every team's k-th key is at most the whole head's k-th largest,
    // so the largest one published so far (tk_floor) is a bar no row below it can pass.
    // A team reads it when it starts a row block and publishes its own when it rises.
    constexpr bool kFloor = kTopk && kTkM == 1;
    unsigned long long floor_now = 0ull, floor_pub = 0ull, tk_last = 0ull;   // tk_last: the list's k-th key
    // Argmax with one x row: the best key of the rows this lane has reported so far; the
    // block reduces them once at the end (a global atomic per row block would queue on
    // one L2 address).
    unsigned long long am_best = 0ull;
    int jnext = 0;                                         // this warp's next job
    for (int rbi = 0; rbi < nrb; ++rbi) {
        const int rb = rb_of(rbi);
        if constexpr (kFloor) floor_now = load_key_relaxed(a.tk_floor);   // used in this block's epilogue
        float yacc = 0.f;     // kImma1: row g, plane t
        float yacc8 = 0.f;    // kImma1: row g + 8, plane t
        float acc[NT][4];     // MMA modes: rows g, g+8; x rows n*8 + 2t, +1
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

        const bool i8 = is_int8(rb);
        const int nbw_c = i8 ? nbw8 : nbw;
        for (int jb = 0; jb < nbw_c; ++jb) {
            const int j = jnext++;
            const int s = j % kStages;
            if (ok) ok = a.wait_ns != 0 && mbar_wait_bounded(&my_bars[s], (uint32_t)(j / kStages) & 1u, a.wait_ns);
            if (ok) {
                consumed = j + 1;
                const int bf = ((i8 ? u08 : u0) + jb) * kBoxesPerStage;
                const int nbox = min(kBoxesPerStage, (i8 ? nb8 : nb) - bf);
#pragma unroll
                for (int q = 0; q < kBoxesPerStage; ++q) {
                    if (q >= nbox) break;
                    if (MODE == kImma1 && i8) {
                        // INT8 box: 4 groups of 32 signed codes per row.  ldmatrix at the
                        // Q4 addresses gives the A operand as is (a0/a2: k 4t .. 4t+3 and
                        // 16 + 4t .. of row g, a1/a3 the same of row g+8); B column g < 4 is
                        // digit plane g in natural k order, columns 4..7 are zero, and the
                        // C operand is the bias alone (the codes carry no offset).  Lane t of
                        // rows g, g+8 gets planes 2t, 2t+1 (t < 2): scaled onto the plane-t
                        // accumulator they are u(2t) 2^(-8t) + u(2t+1) 2^(-8t-8) (t = 0, 1).
                        const unsigned char* cb = codes + ((warp * kStages + s) * kBoxesPerStage + q) * kCodeBox;
                        const unsigned char* sb = scl + (warp * kStages + s) * kStageScales + q * 8;
                        const int g = lane >> 2, t = lane & 3;
                        const int gb = (bf + q) * 4;                     // first group of the box
                        const uint2 sg = *reinterpret_cast<const uint2*>(sb + g * 16);
                        const uint2 sg8 = *reinterpret_cast<const uint2*>(sb + (g + 8) * 16);
                        const int lr = lane & 7, li = lane >> 3;
                        const uint32_t abase = smem_addr(cb) + ((li & 1) * 8 + lr) * 128 + (((li >> 1) ^ lr) << 4);
                        const uint2* x8 = reinterpret_cast<const uint2*>(xst + (size_t)ngp * 292) + ((size_t)gb * 8 + g) * 4 + t;
                        const float fb = reinterpret_cast<const float*>(xst + (size_t)ngp * 288)[gb >> 3];
                        float part = 0.f, part8 = 0.f;
                        const float lc0 = t == 0 ? 1.0f : t == 1 ? 0.00390625f : 0.0f;
                        const float lc1 = t == 0 ? 0.00390625f : t == 1 ? 1.52587890625e-05f : 0.0f;
#pragma unroll
                        for (int cg = 0; cg < 4; ++cg) {
                            uint32_t r0, r1, r2, r3;
                            ldmatrix_x4(abase ^ (uint32_t)(cg << 5), r0, r1, r2, r3);
                            const uint2 bq = x8[cg * 32];
                            int d[4];
                            imma_s8s8(d, r0, r1, r2, r3, bq.x, bq.y, kBiasBits, kBiasBits);
                            const float v0 = (__int_as_float(d[0]) - kBiasF) * lc0 + (__int_as_float(d[1]) - kBiasF) * lc1;
                            const float v1 = (__int_as_float(d[2]) - kBiasF) * lc0 + (__int_as_float(d[3]) - kBiasF) * lc1;
                            const uint32_t sw = cg < 2 ? sg.x : sg.y, sw8 = cg < 2 ? sg8.x : sg8.y;
                            const float s0 = __half2float(__ushort_as_half((unsigned short)((cg & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
                            const float s1 = __half2float(__ushort_as_half((unsigned short)((cg & 1) ? (sw8 >> 16) : (sw8 & 0xFFFFu))));
                            part = fmaf(s0, v0, part);
                            part8 = fmaf(s1, v1, part8);
                        }
                        yacc = fmaf(fb, part, yacc);
                        yacc8 = fmaf(fb, part8, yacc8);
                        continue;
                    }
                    {
                        const unsigned char* cb = codes + ((warp * kStages + s) * kBoxesPerStage + q) * kCodeBox;
                        const unsigned char* sb = scl + (warp * kStages + s) * kStageScales + q * 16;
                        constexpr int kScaleRow = 16 * kBoxesPerStage;   // bytes per row of the scale box
                        const int gb = (bf + q) * 8;                     // first group of the box
                        if constexpr (MODE == kImma1) {
                            const int g = lane >> 2, t = lane & 3;
                            const uint4 sg = *reinterpret_cast<const uint4*>(sb + g * kScaleRow);
                            const uint4 sg8 = *reinterpret_cast<const uint4*>(sb + (g + 8) * kScaleRow);
                            // ldmatrix as in the bf16 modes: r0/r1 = word t of rows g/g+8 of group
                            // 2 cp, r2/r3 the same of group 2 cp + 1 (codes 8t .. 8t+7 of each row)
                            const int lr = lane & 7, li = lane >> 3;
                            const uint32_t abase =
                                smem_addr(cb) + ((li & 1) * 8 + lr) * 128 + (((li >> 1) ^ lr) << 4);
                            const uint4* xq = reinterpret_cast<const uint4*>(xst) + ((gb >> 1) * 8 + g) * 4 + t;
                            const int4* xc = reinterpret_cast<const int4*>(xst + (size_t)ngp * 256) + (gb >> 1) * 4 + t;
                            // the box's sums are scaled and added here, then once by 2^-F
                            const float fb = reinterpret_cast<const float*>(xst + (size_t)ngp * 288)[gb >> 3];
                            float part = 0.f, part8 = 0.f;
#pragma unroll
                            for (int cp = 0; cp < 4; ++cp) {
                                uint32_t r0, r1, r2, r3;
                                ldmatrix_x4(abase ^ (uint32_t)(cp << 5), r0, r1, r2, r3);
                                const uint4 bq = xq[cp * 32];
                                const int4 cq = xc[cp * 4];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int c = 2 * cp + h;
                                    const uint32_t w0 = h ? r2 : r0, w1 = h ? r3 : r1;
                                    // A: slot 4t + i holds code 8t + 2i (low nibble), slot
                                    // 16 + 4t + i holds 16 x code 8t + 2i + 1 (high nibble in place)
                                    int d[4];
                                    imma_u8s8(d, w0 & 0x0F0F0F0Fu, w1 & 0x0F0F0F0Fu, w0 & 0xF0F0F0F0u,
                                              w1 & 0xF0F0F0F0u, h ? bq.z : bq.x, h ? bq.w : bq.y, h ? cq.z : cq.x,
                                              h ? cq.w : cq.y);
                                    // d[0], d[2]: bias + sum over even k of (code - 8) d_t for rows
                                    // g, g+8; d[1], d[3]: bias + 16 x the same over odd k
                                    const float u0 =
                                        fmaf(__int_as_float(d[1]), 0.0625f, __int_as_float(d[0])) - kBias17;
                                    const float u1 =
                                        fmaf(__int_as_float(d[3]), 0.0625f, __int_as_float(d[2])) - kBias17;
                                    part = fmaf(scale_at(sg, c), u0, part);
                                    part8 = fmaf(scale_at(sg8, c), u1, part8);
                                }
                            }
                            yacc = fmaf(fb, part, yacc);
                            yacc8 = fmaf(fb, part8, yacc8);
                        } else {
                            const int g = lane >> 2, t = lane & 3;
                            const uint4 sg = *reinterpret_cast<const uint4*>(sb + g * kScaleRow);
                            const uint4 sg8 = *reinterpret_cast<const uint4*>(sb + (g + 8) * kScaleRow);
                            // ldmatrix rows: lane 8i + r -> weight row 8 (i & 1) + r of group
                            // 2 cp + (i >> 1); with the 128-byte swizzle the chunk of group c in
                            // row r sits at (c ^ (r & 7)) * 16, so group pair cp is one XOR away.
                            const int lr = lane & 7, li = lane >> 3;
                            const uint32_t abase =
                                smem_addr(cb) + ((li & 1) * 8 + lr) * 128 + (((li >> 1) ^ lr) << 4);
                            // All MMAs of a batch of groups are issued before any result is
                            // read, so the tensor-core latency overlaps across groups.
                            constexpr int GB = 2;            // groups per batch
#pragma unroll
                            for (int c0 = 0; c0 < 8; c0 += GB) {
                                float d[GB][NT][4];
#pragma unroll
                                for (int cp = c0 / 2; cp < (c0 + GB) / 2; ++cp) {
                                    uint32_t r0, r1, r2, r3;  // word t of rows g, g+8 for groups 2cp, 2cp+1
                                    ldmatrix_x4(abase ^ (uint32_t)(cp << 5), r0, r1, r2, r3);
#pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        const int c = 2 * cp + h;
                                        const uint32_t w0 = h ? r2 : r0, w1 = h ? r3 : r1;
                                        // codes 8t .. 8t+7 of rows g, g+8 in k order: MMA 1 takes
                                        // bytes 0, 1 (k 8t .. 8t+3), MMA 2 bytes 2, 3
                                        const uint32_t v0 = w0 >> 4, v1 = w1 >> 4;
                                        const uint32_t A0 = sub_bf16x2(byte_pair(w0, v0, 0, kmask, kmagic), k136);
                                        const uint32_t A1 = sub_bf16x2(byte_pair(w1, v1, 0, kmask, kmagic), k136);
                                        const uint32_t A2 = sub_bf16x2(byte_pair(w0, v0, 1, kmask, kmagic), k136);
                                        const uint32_t A3 = sub_bf16x2(byte_pair(w1, v1, 1, kmask, kmagic), k136);
                                        const uint32_t A4 = sub_bf16x2(byte_pair(w0, v0, 2, kmask, kmagic), k136);
                                        const uint32_t A5 = sub_bf16x2(byte_pair(w1, v1, 2, kmask, kmagic), k136);
                                        const uint32_t A6 = sub_bf16x2(byte_pair(w0, v0, 3, kmask, kmagic), k136);
                                        const uint32_t A7 = sub_bf16x2(byte_pair(w1, v1, 3, kmask, kmagic), k136);
#pragma unroll
                                        for (int n = 0; n < NT; ++n) {
                                            const uint4 bx = xrow[n][(gb + c) * 4 + t];
                                            mma_bf16_16816_z(d[c - c0][n], A0, A1, A2, A3, bx.x, bx.y);
                                            mma_bf16_16816(d[c - c0][n], A4, A5, A6, A7, bx.z, bx.w);
                                        }
                                    }
                                }
#pragma unroll
                                for (int c = c0; c < c0 + GB; ++c) {
                                    const float s0 = scale_at(sg, c), s1 = scale_at(sg8, c);
#pragma unroll
                                    for (int n = 0; n < NT; ++n) {
                                        acc[n][0] = fmaf(s0, d[c - c0][n][0], acc[n][0]);
                                        acc[n][2] = fmaf(s1, d[c - c0][n][2], acc[n][2]);
                                        acc[n][1] = fmaf(s0, d[c - c0][n][1], acc[n][1]);
                                        acc[n][3] = fmaf(s1, d[c - c0][n][3], acc[n][3]);
                                    }
                                }
                            }
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
        if constexpr (MODE == kImma1) {
            // planes t = 0..3 of rows g and g+8 scaled by 2^(8 (3 - t)) and summed (the
            // groups' 2^-F_g went in with their scales)
            const float plane_factor = __uint_as_float((uint32_t)(24 - 8 * (lane & 3) + 127) << 23);
            float v0 = yacc * plane_factor, v1 = yacc8 * plane_factor;
            v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
            v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
            if ((lane & 3) == 0) {
                my_red[lane >> 2] = v0;
                my_red[(lane >> 2) + 8] = v1;
            }
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
        // Plain stores without split-K: every warp of the team stores a share of the
        // block's (x row, row) outputs; otherwise the team's first warp does the epilogue.
        const bool share = EPI == kEpiPlain && a.splits == 1;
        if (wt == 0 || share) {
            const int mi = matrix_of(a, rb);
            const int nrow = a.N[mi];
            const int lrow0 = (rb - a.rb_begin[mi]) * kRows;
            const size_t vrows = (size_t)a.row_blocks * kRows;            // padded rows over all matrices
            if constexpr (kFuse) {                       // splits == 1: gate totals wait in registers
#pragma unroll
                for (int it = 0; it < kRows * Q4_GEMV_MAX_M / 32; ++it) {
                    const int e = lane + 32 * it;
                    if (e < kRows * a.M) {
                        const int m = e / kRows, rr = e - m * kRows;
                        float total = 0.f;
                        for (int w = 0; w < P; ++w) total += red[(team * P + w) * kRows * MP + rr * MP + m];
                        if (mi == 0) {
                            gsave[it] = total;
                        } else if (lrow0 + rr < nrow) {
                            const float g = gsave[it];
                            a.y[0][(size_t)m * nrow + lrow0 + rr] = g / (1.0f + expf(-g)) * total;
                        }
                    }
                }
            }
            // Lanes cover 32 (x row, row) pairs from e0 on, x row major (coalesced y); the
            // key of each live total orders it for argmax and top-k (0 when not live).
            auto rows_out = [&](int e0) {
                const int e = e0 + lane;
                const int m = e / kRows, rr = e - m * kRows;
                const bool live = e < kRows * a.M && lrow0 + rr < nrow;
                float total = 0.f;
                if (e < kRows * a.M)
                    for (int w = 0; w < P; ++w) total += red[(team * P + w) * kRows * MP + rr * MP + m];
                if (live) {
                    if (a.splits > 1) a.partial[((size_t)split * a.M + m) * vrows + (size_t)rb * kRows + rr] = total;
                    else if (a.y[mi]) a.y[mi][(size_t)m * nrow + lrow0 + rr] = total;
                }
                return live ? argmax_key(total, a.row_base + (uint32_t)(lrow0 + rr)) : 0ull;
            };
            if constexpr (kFloor) {
                // One x row: lanes 0-15 hold the block's 16 rows.  Most blocks have no row
                // above the list's k-th key (tk_last) or the published floor, and skip the
                // insert after one vote.
                const unsigned long long key = rows_out(0);
                const unsigned long long bar = key_max(tk_last, floor_now);
                if (__any_sync(0xffffffffu, lane < 16 && key > bar)) {
                    topk_insert(tk[0], key, lane < 16, a.tk_k, lane, floor_now);
                    tk_last = __shfl_sync(0xffffffffu, tk[0], a.tk_k - 1);
                    if (tk_last > floor_pub && tk_last > floor_now) {       // the same on every lane
                        if (lane == 0) atomicMax(a.tk_floor, tk_last);
                        floor_pub = tk_last;
                    }
                }
            } else if constexpr (kTopk) {               // lanes 0-15: x row 2h, lanes 16-31: x row 2h + 1
#pragma unroll
                for (int h = 0; h < (kTkM + 1) / 2; ++h) {
                    if (h * 32 < kRows * a.M) {
                        const unsigned long long key = rows_out(h * 32);
                        topk_insert(tk[2 * h], key, lane < 16, a.tk_k, lane);
                        if (2 * h + 1 < kTkM) topk_insert(tk[2 * h + 1], key, lane >= 16, a.tk_k, lane);
                    }
                }
            } else {
                for (int e0 = share ? wt * 32 : 0; e0 < (kFuse ? 0 : kRows * a.M); e0 += share ? P * 32 : 32) {
                    unsigned long long key = rows_out(e0);
                    if constexpr (kArgmax && MODE == kImma1) {
                        am_best = key_max(am_best, key);
                    } else if constexpr (kArgmax) {     // the 16 lanes of one x row agree on its best row
                        const int m = (e0 + lane) / kRows;
#pragma unroll
                        for (int o = 1; o < kRows; o <<= 1) {
                            const unsigned long long k2 = __shfl_xor_sync(0xffffffffu, key, o);
                            key = k2 > key ? k2 : key;
                        }
                        if ((lane & (kRows - 1)) == 0 && m < a.M && key) atomicMax(&a.am_key[m], key);
                    }
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
            if (!mbar_wait_bounded(&my_bars[j % kStages], (uint32_t)(j / kStages) & 1u, kWaitLimit)) break;
    }
    if (!x_ok && threadIdx.x == 0) mbar_wait_bounded(&s_xbar, 0, kWaitLimit);   // x rows still in flight

    if constexpr (kArgmax) {                                // the last block to finish reports and resets
        if constexpr (MODE == kImma1) {                     // the warps' best keys, then one atomic
            unsigned long long k = am_best;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) k = key_max(k, __shfl_xor_sync(0xffffffffu, k, o));
            if (lane == 0) s_best[warp] = k;
            __syncthreads();
            if (threadIdx.x == 0) {
                unsigned long long b = 0ull;
                for (int w = 0; w < W; ++w) b = key_max(b, s_best[w]);
                if (b) atomicMax(&a.am_key[0], b);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            s_last[0] = atomicAdd(a.am_done, 1u) == gridDim.x - 1;
        }
        __syncthreads();
        if (s_last[0]) {
            __threadfence();
            if ((int)threadIdx.x < a.M) {
                const unsigned long long key = atomicExch(&a.am_key[threadIdx.x], 0ull);
                a.am_index[threadIdx.x] = key ? (long long)(0xFFFFFFFFu - (uint32_t)key) : -1;
                if (a.am_value) a.am_value[threadIdx.x] = key ? argmax_value(key) : __int_as_float(0x7FC00000);
            }
            if (threadIdx.x == 0) *a.am_done = 0u;
        }
    }

    if constexpr (kTopk) {
        // Every team is past its last row block, so the code rings are free: each team
        // leader parks its 32-key list of every x row in its own warp's ring (a team that
        // gave up parks empty lists), then a tree of warp merges reduces the teams' lists
        // of each x row to one, and the block writes its first k keys to the workspace.
        const int kk = a.tk_k;
        constexpr int kRingWords = kStages * kStageCodes / 8;          // u64 per warp ring
        unsigned long long* lists = reinterpret_cast<unsigned long long*>(codes);
        const size_t team_stride = (size_t)P * kRingWords;            // list of team t: t * team_stride
        __syncthreads();
        if (active && wt == 0) {
#pragma unroll
            for (int mm = 0; mm < kTkM; ++mm)
                if (mm < a.M) lists[(size_t)warp * kRingWords + mm * 32 + lane] = ok ? tk[mm] : 0ull;
        }
        __syncthreads();
        for (int step = 1; step < a.teams; step <<= 1) {               // merge team i + step into team i
            const int pairs = (a.teams + 2 * step - 1) / (2 * step);
            for (int job = warp; job < a.M * pairs; job += W) {
                const int m = job / pairs, t = (job - m * pairs) * 2 * step;
                if (t + step < a.teams) {
                    unsigned long long* dst = lists + (size_t)t * team_stride + m * 32;
                    const unsigned long long* src = lists + (size_t)(t + step) * team_stride + m * 32;
                    dst[lane] = warp_merge_desc(dst[lane], src[lane], lane);
                }
            }
            __syncthreads();
        }
        for (int m = warp; m < a.M; m += W) {
            if (lane < kk) a.tk_cand[((size_t)m * gridDim.x + blockIdx.x) * kk + lane] = lists[m * 32 + lane];
            __threadfence();
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            s_last[0] = atomicAdd(a.am_done, 1u) == gridDim.x - 1;
        }
        __syncthreads();
        if (s_last[0]) {
            // The last block: S warps per x row each merge the lists of every S-th block
            // (k keys each, padded with 0 to 32 lanes), with up to kDepth lists loaded at
            // once, then a tree of warp merges reduces the S slice lists of each x row to
            // the result.
            __threadfence();
            constexpr int kDepth = 12;
            const int S = max(1, W / a.M);
            for (int job = warp; job < a.M * S; job += W) {
                const int m = job / S, sl = job - m * S;
                const unsigned long long* src = a.tk_cand + (size_t)m * gridDim.x * kk;
                unsigned long long list = 0ull;
                for (int b0 = sl; b0 < (int)gridDim.x; b0 += kDepth * S) {
                    unsigned long long cur[kDepth];
#pragma unroll
                    for (int q = 0; q < kDepth; ++q) {
                        const int b = b0 + q * S;
                        cur[q] = (b < (int)gridDim.x && lane < kk) ? __ldcg(src + (size_t)b * kk + lane) : 0ull;
                    }
#pragma unroll
                    for (int q = 0; q < kDepth; ++q)
                        if (b0 + q * S < (int)gridDim.x) list = warp_merge_desc(list, cur[q], lane);   // warp-uniform
                }
                lists[(size_t)job * 32 + lane] = list;
            }
            __syncthreads();
            for (int step = 1; step < S; step <<= 1) {
                const int pairs = (S + 2 * step - 1) / (2 * step);
                for (int job = warp; job < a.M * pairs; job += W) {
                    const int m = job / pairs, i = (job - m * pairs) * 2 * step;
                    if (i + step < S) {
                        unsigned long long* dst = lists + ((size_t)m * S + i) * 32;
                        dst[lane] = warp_merge_desc(dst[lane], dst[(size_t)step * 32 + lane], lane);
                    }
                }
                __syncthreads();
            }
            for (int m = warp; m < a.M; m += W) {
                const unsigned long long key = lists[(size_t)m * S * 32 + lane];
                if (lane < kk) {
                    a.am_index[(size_t)m * kk + lane] = key ? (long long)(0xFFFFFFFFu - (uint32_t)key) : -1;
                    if (a.am_value) a.am_value[(size_t)m * kk + lane] = key ? argmax_value(key) : __int_as_float(0x7FC00000);
                }
            }
            if (threadIdx.x == 0) {
                *a.am_done = 0u;
                if (a.tk_floor) *a.tk_floor = 0ull;
            }
        }
    }
}

size_t per_warp_bytes(int mode)
{
    const int mp = mode == kMma16 ? 16 : mode == kMma8 ? 8 : 1;
    return (size_t)kStages * (kStageCodes + kStageScales + sizeof(uint64_t)) + (size_t)kRows * mp * sizeof(float);
}

// kImma1 per group: B operands 256 B, C operands 32 B, 4 B for the boxes' 2^-F (one
// float per box of 8 groups), and with INT8 matrices in the launch the natural-order B
// operands, 256 B more.  kMma*: the M x rows and one zero row, each padded by a group.
size_t x_stage_bytes(int mode, int nb, int64_t M, bool int8 = false)
{
    const size_t ngp = (size_t)nb * 8;
    if (mode == kImma1) return ngp * (int8 ? 548 : 292);
    return (size_t)(M + 1) * (ngp + 1) * 64;
}

size_t smem_bytes(int mode, int warps, int nb, int64_t M, bool int8 = false)
{
    return 1024 + 16 + (size_t)warps * per_warp_bytes(mode) + x_stage_bytes(mode, nb, M, int8);
}

int mode_for(int64_t M, q4_dtype xt)
{
    (void)xt;
    return M == 1 ? kImma1 : M <= 8 ? kMma8 : kMma16;
}

template <int EPI>
const void* kernel_for_epi(int mode)
{
    switch (mode) {
    case kMma8: return reinterpret_cast<const void*>(&gemv_tma_kernel<kMma8, EPI>);
    case kImma1: return reinterpret_cast<const void*>(&gemv_tma_kernel<kImma1, EPI>);
    default: return reinterpret_cast<const void*>(&gemv_tma_kernel<kMma16, EPI>);
    }
}

const void* kernel_for(int mode, int epi)
{
    switch (epi) {
    case kEpiFuse: return kernel_for_epi<kEpiFuse>(mode);
    case kEpiArgmax: return kernel_for_epi<kEpiArgmax>(mode);
    case kEpiTopk: return kernel_for_epi<kEpiTopk>(mode);
    default: return kernel_for_epi<kEpiPlain>(mode);
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
                   GemvPlan* p, int epi, const int* fmts, bool allow_split)
{
    const bool fuse = epi == kEpiFuse, whole_k = epi != kEpiPlain || !allow_split;
    if (fuse && (count != 2 || Ns[0] != Ns[1])) return false;
    const int mode = mode_for(M, xt);
    int n_int8 = 0;
    for (int i = 0; fmts && i < count; ++i) n_int8 += fmts[i] != 0;
    if (n_int8 && (mode != kImma1 || epi != kEpiPlain)) return false;
    const bool int8 = n_int8 > 0;
    // INT8 row blocks have twice the stage units of Q4 ones
    const double unit_scale = !int8 ? 1.0 : n_int8 == count ? 2.0 : 1.5;
    const int G = (int)(K / 32);
    long long rbl = 0;
    for (int i = 0; i < count; ++i) rbl += (Ns[i] + kRows - 1) / kRows;
    if (rbl < 1 || rbl > INT32_MAX / kRows) return false;
    const int row_blocks = (int)rbl;
    const int walk = fuse ? row_blocks / 2 : row_blocks;      // row blocks (gate+up: pairs) teams walk
    const int visits = fuse ? 2 : 1;                          // row blocks per walked item
    const int boxes = (G + 7) / 8;
    const int units = (boxes + kBoxesPerStage - 1) / kBoxesPerStage;
    const size_t pw = per_warp_bytes(mode);
    const size_t budget = (size_t)dev.max_smem_optin - 512;   // room for the kernel's static arrays
    // Boxes of the widest split when K is cut into `sp` splits of whole units.
    auto split_boxes = [&](int sp) {
        const int b = (units + sp - 1) / sp * kBoxesPerStage;
        return b < boxes ? b : boxes;
    };
    // Splits forced by shared memory: the staged x of one split leaves room for 4 warps.
    int splits_min = 1;
    while (1040 + 4 * pw + x_stage_bytes(mode, split_boxes(splits_min), M, int8) > budget) {
        if (split_boxes(splits_min) <= kBoxesPerStage) return false;
        ++splits_min;
    }
    // Choose the K splits, the team size P and the teams per block by a cost model of the
    // busiest block: rounds of row blocks x units per warp x warps sharing the SM, plus
    // the row-block epilogue and, for a split K, the reduction of partial sums.  Teams
    // per block are capped so that small problems spread over all SMs.
    int splits = 0, P = 0, teams = 0;
    double best = 0.0;
    if ((fuse || whole_k) && splits_min > 1) return false;   // fused epilogues need whole sums
    const int max_splits = (row_blocks <= kCounterSlots && !fuse && !whole_k) ? units : splits_min;
    for (int sp = splits_min; sp <= max_splits; ++sp) {
        const int nbs = split_boxes(sp);
        if ((boxes + nbs - 1) / nbs != sp) continue;                  // same cut as fewer splits
        const size_t xs = x_stage_bytes(mode, nbs, M, int8);
        if (1040 + pw + xs > budget) continue;
        const size_t fitw = (budget - 1040 - xs) / pw;
        const int wbs = (int)(fitw < (size_t)kMaxWarps ? fitw : (size_t)kMaxWarps);
        const int nus = (nbs + kBoxesPerStage - 1) / kBoxesPerStage;
        const long long sms = dev.sm_count / sp > 0 ? dev.sm_count / sp : 1;   // blocks of one split
        for (int pp = 1; pp <= nus && pp <= wbs; ++pp) {
            const int pwu = (nus + pp - 1) / pp;                          // units per warp per row block
            const long long spread = ((long long)walk + sms - 1) / sms;
            // Fewer teams than fit can finish sooner: the last round of row blocks is then
            // full (e.g. 15 teams of one warp cover 15,520 row blocks in 7 rounds on 148
            // SMs, 16 teams need 7 rounds of 16 warps each).
            for (long long tm = std::min<long long>(wbs / pp, spread); tm >= 1; --tm) {
                const long long gxs = std::min(((long long)walk + tm - 1) / tm, sms);
                const long long rounds = visits * (((long long)walk + gxs * tm - 1) / (gxs * tm));
                const double share = std::max((double)(tm * pp), kMinWarpShare) / 16.0;
                const double cost = (double)rounds * (pwu * unit_scale + kEpilogueCost) * share +
                                    (sp > 1 ? kSplitCost : 0.0);
                if (splits == 0 || cost < best - 1e-9) {
                    splits = sp;
                    P = pp;
                    teams = (int)tm;
                    best = cost;
                }
            }
        }
    }
    if (splits == 0) return false;
    const int ksg = split_boxes(splits) * 8;
    const int nb = ksg / 8;
    // A block with few warps stages x slowly (every block stages its split in full), so
    // small plans get warps that own no rows and only help with the staging.
    int warps = P * teams;
    if (warps < kStagingWarps) {
        const size_t sw = smem_bytes(mode, kStagingWarps, nb, M, int8);
        if (sw <= budget && blocks_per_sm(kernel_for(mode, epi), kStagingWarps * 32, sw) >= 1) warps = kStagingWarps;
    }
    const size_t smem = smem_bytes(mode, warps, nb, M, int8);
    if (smem > budget) return false;
    const int per_sm = blocks_per_sm(kernel_for(mode, epi), warps * 32, smem);
    if (per_sm < 1) return false;
    const long long blocks_needed = ((long long)walk + teams - 1) / teams;
    long long gx = (long long)dev.sm_count * per_sm / splits;
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
    p->has_int8 = int8 ? 1 : 0;
    p->block_warps = warps;
    return true;
}

q4_status launch_gemv_tma(const void* x, q4_dtype xt, int64_t M, int64_t K, const q4_weight* mats, int count,
                          int prefetch, void* workspace, const GemvPlan& plan, cudaStream_t stream, int epi,
                          const ArgmaxOut* am, const int* fmts)
{
    TmaMaps maps;
    TmaGemvArgs a;
    const uint64_t G = (uint64_t)(K / 32);
    int rb = 0;
    for (int i = 0; i < count; ++i) {
        // Q4: K/2 code bytes per row, a box is 8 groups; INT8: K bytes per row, 4 groups
        const bool i8 = fmts && fmts[i] != 0;
        const uint64_t row_bytes = i8 ? (uint64_t)K : (uint64_t)K / 2;
        if (!encode_tma_2d(&maps.codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, mats[i].packed, row_bytes,
                           (uint64_t)mats[i].N, row_bytes, 128, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_tma_2d(&maps.scales[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, mats[i].scales, G, (uint64_t)mats[i].N,
                           G * 2, (i8 ? 4 : 8) * kBoxesPerStage, kRows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
        a.fmt[i] = i8 ? 1 : 0;
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
        a.fmt[i] = 0;
    }
    a.has_int8 = plan.has_int8;
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
    a.x_f32 = xt == Q4_F32 ? 1 : 0;
    a.wait_ns = consumer_wait_ns();
    a.am_key = am ? am->key : nullptr;
    a.am_done = am ? am->done : nullptr;
    a.am_index = am ? am->index : nullptr;
    a.am_value = am ? am->value : nullptr;
    a.tk_cand = am ? am->cand : nullptr;
    a.tk_floor = am ? am->floor : nullptr;
    a.tk_k = am ? am->k : 1;
    a.row_base = am ? am->row_base : 0u;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid_x, (unsigned)plan.splits);
    cfg.blockDim = dim3((unsigned)(plan.block_warps * 32));
    cfg.dynamicSmemBytes = (size_t)plan.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&maps, &a};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, kernel_for(mode_for(M, xt), epi), args);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
