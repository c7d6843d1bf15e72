// q4_gemv: y[m,n] = sum_g s[n,g] * sum_{j<32} x[m,32g+j] * (code[n,32g+j] - 8), M = 1..16.
//
// The pages' decode kernel is an AVX-512 Q4 GEMV that expands nibbles through a
// 16-entry table (QORA-LLM-0.8B model card, section "AVX-512 SIMD Acceleration")
// and splits rows over a thread pool (QORA-4B thread, section "量化与内存管理").
// On sm_100a the product is bound by HBM: 0.5625 bytes per weight against one
// multiply-add per weight and row of x.  The kernel therefore spends as few
// instructions per weight as it can:
//
//  * Rows are served by 16-lane teams; a lane reads one whole 32-weight group of
//    its row with one 16-byte load, so a team reads 256 contiguous bytes.
//  * Nibble -> float without a table or a conversion instruction: OR-ing nibble p
//    of a 32-bit word (bits 4p..4p+3, p <= 4) into the mantissa of the float
//    2^(23-4p) gives the exact value 2^(23-4p) + code; one packed f32x2 add of
//    -(2^(23-4p) + 8) leaves code - 8 exactly.  Nibbles 5..7 are read from the
//    word shifted right by 12.  Per 8 weights: 1 shift, 8 LOP3, 4 FADD2.
//  * Products use packed f32x2 FMAs (sm_100), accumulating each group's 32
//    products in f32; the group sum is scaled by the binary16 scale and added to
//    the row's f32 accumulator; the 16 lanes of a team reduce with shuffles.
//  * x is staged once per block in shared memory as f32; the eight 16-byte chunks
//    of group g sit at slots c ^ (g & 7) so the 8 lanes of a load phase hit
//    distinct banks.
//  * Skinny shapes (fewer row blocks than SMs) split K across blocks (grid.y).
//    Each block writes f32 partial sums to the workspace, then bumps the row
//    block's arrival counter; the block that arrives last adds the partials in
//    split order (a fixed order, so the result does not depend on timing), writes
//    y and resets the counter.  Nobody waits on anybody.
//  * When x for a split does not fit the shared-memory budget it is staged in
//    pieces of whole chunks; the block restages when its work crosses a piece.
#include "q4_common.cuh"

namespace q4 {
namespace {

constexpr int kThreads = 256;
constexpr int kTeam = 16;                       // lanes per row
constexpr int kTeams = kThreads / kTeam;        // rows per row block
constexpr int kSlots = 5;                       // groups per lane per chunk
constexpr int kChunkGroups = kTeam * kSlots;    // 80 groups = 2560 weights per chunk

struct GemvArgs {
    const void* x;
    const uint8_t* packed;
    const uint16_t* scales;
    float* y;
    float* partial;        // [splits][M][N] (splits > 1)
    unsigned* counters;    // [row_blocks]   (splits > 1)
    int M, N, G;           // G = K / 32
    int ksg;               // groups per split
    int splits;
    int row_blocks;
    int chunk;             // groups per work unit (<= kSlots * kTeam)
    int xcap;              // groups of x held in shared memory at once (multiple of chunk)
};

// Workspace layout (shape independent, so one workspace serves every shape):
// [0, kCounterBytes) arrival counters, one per row block of a split launch; they
// must be zero before the first call and every call leaves them zero.  Splits
// are only used when there are fewer row blocks than SMs, so kCounterSlots
// bounds the count.  Partial sums follow.
constexpr int kCounterSlots = 1024;
constexpr size_t kCounterBytes = kCounterSlots * sizeof(unsigned);

__device__ __forceinline__ uint4 load_weights(const uint8_t* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Eight codes of one word (nibble p holds weight p) -> (code - 8) as exact floats.
__device__ __forceinline__ void expand8(uint32_t v, float2& d01, float2& d23, float2& d45, float2& d67)
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
    d01 = __fadd2_rn(make_float2(f0, f1), make_float2(-8388616.0f, -524296.0f));
    d23 = __fadd2_rn(make_float2(f2, f3), make_float2(-32776.0f, -2056.0f));
    d45 = __fadd2_rn(make_float2(f4, f5), make_float2(-136.0f, -32776.0f));
    d67 = __fadd2_rn(make_float2(f6, f7), make_float2(-2056.0f, -136.0f));
}

template <bool XBF16>
__device__ __forceinline__ float4 load_x4(const void* x, size_t idx)
{
    if constexpr (XBF16) {
        const uint2 b = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(x) + idx);
        return make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u),
                           __uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
    } else {
        return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + idx);
    }
}

// Loads of one work unit: row block rb, chunk ch (groups ch*chunk .. of this split).
__device__ __forceinline__ void load_unit(const GemvArgs& a, int rb, int ch, int g0, int ng, int team, int lane16,
                                          uint4 (&w)[kSlots], uint32_t (&sc)[kSlots])
{
    const int row = rb * kTeams + team;
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
        const int lg = ch * a.chunk + j * kTeam + lane16;
        if (row < a.N && j * kTeam < a.chunk && lg < ng) {
            const size_t gg = (size_t)row * a.G + g0 + lg;
            w[j] = load_weights(a.packed + gg * 16);
            sc[j] = a.scales[gg];
        }
    }
}

// x[:, 32*gbase .. 32*(gbase+n)) -> shared memory as f32; rows m >= M are zero.
template <int MT, bool XBF16>
__device__ __forceinline__ void stage_x(const GemvArgs& a, float4* xs, int gbase, int n, int per_m, size_t K)
{
    for (int i = threadIdx.x; i < MT * n * 8; i += kThreads) {
        const int m = i / (n * 8);
        const int r = i - m * (n * 8);
        const int lg = r >> 3, c = r & 7;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m < a.M) v = load_x4<XBF16>(a.x, (size_t)m * K + (size_t)(gbase + lg) * 32 + c * 4);
        xs[m * per_m + lg * 8 + (c ^ (lg & 7))] = v;
    }
}

template <int MT, bool XBF16>
__global__ void __launch_bounds__(kThreads, 2) gemv_ffma_kernel(const GemvArgs a)
{
    extern __shared__ float4 xs[];               // [MT][xcap][8] float4, chunk-swizzled per group
    __shared__ int s_last;

    const int tid = threadIdx.x;
    const int lane16 = tid & (kTeam - 1);
    const int team = tid / kTeam;
    const int split = blockIdx.y;
    const int g0 = split * a.ksg;
    const int ng = min(a.G - g0, a.ksg);
    const size_t K = (size_t)a.G * 32;
    const int nchunks = (ng + a.chunk - 1) / a.chunk;
    const int chunks_per_stage = a.xcap / a.chunk;
    const int per_m = min(ng, a.xcap) * 8;       // float4 per x row in shared memory

    pdl_launch_dependents();
    pdl_wait();
    int rb = blockIdx.x, ch = 0;
    if (rb >= a.row_blocks) return;

    // The first unit's weight loads go out before x is staged, so the two
    // latencies overlap; afterwards each unit's loads go out before the
    // previous unit is computed.
    uint4 w[kSlots];
    uint32_t sc[kSlots];
    load_unit(a, rb, ch, g0, ng, team, lane16, w, sc);
    int staged = -1;
    float yacc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m] = 0.f;

    while (true) {
        const int stage = ch / chunks_per_stage;
        if (stage != staged) {
            if (staged >= 0) __syncthreads();    // the previous stage is no longer read
            const int gb = stage * a.xcap;
            stage_x<MT, XBF16>(a, xs, g0 + gb, min(a.xcap, ng - gb), per_m, K);
            __syncthreads();
            staged = stage;
        }
        int nrb = rb, nch = ch + 1;
        if (nch == nchunks) {
            nch = 0;
            nrb += gridDim.x;
        }
        const bool has_next = nrb < a.row_blocks;
        uint4 wn[kSlots];
        uint32_t scn[kSlots];
        if (has_next) load_unit(a, nrb, nch, g0, ng, team, lane16, wn, scn);

        const int row = rb * kTeams + team;
        const bool row_ok = row < a.N;
#pragma unroll
        for (int j = 0; j < kSlots; ++j) {
            const int lg = ch * a.chunk + j * kTeam + lane16;        // group within the split
            if (row_ok && j * kTeam < a.chunk && lg < ng) {
                const int ls = lg - stage * a.xcap;                    // group within the stage
                const float s = __half2float(__ushort_as_half((unsigned short)sc[j]));
                const float4* xg = xs + ls * 8;
                const int sw = ls & 7;
                float2 acc[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.f, 0.f);
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    const uint32_t v = wd == 0 ? w[j].x : wd == 1 ? w[j].y : wd == 2 ? w[j].z : w[j].w;
                    float2 d01, d23, d45, d67;
                    expand8(v, d01, d23, d45, d67);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float4 xa = xg[m * per_m + ((2 * wd) ^ sw)];
                        const float4 xb = xg[m * per_m + ((2 * wd + 1) ^ sw)];
                        acc[m] = __ffma2_rn(make_float2(xa.x, xa.y), d01, acc[m]);
                        acc[m] = __ffma2_rn(make_float2(xa.z, xa.w), d23, acc[m]);
                        acc[m] = __ffma2_rn(make_float2(xb.x, xb.y), d45, acc[m]);
                        acc[m] = __ffma2_rn(make_float2(xb.z, xb.w), d67, acc[m]);
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) yacc[m] = fmaf(s, acc[m].x + acc[m].y, yacc[m]);
            }
        }

        if (nch == 0) {                          // row block rb is complete
            // Team reduction: after it every lane of the team holds the row's sums.
#pragma unroll
            for (int m = 0; m < MT; ++m) {
#pragma unroll
                for (int o = kTeam / 2; o > 0; o >>= 1) yacc[m] += __shfl_xor_sync(0xffffffffu, yacc[m], o);
            }
            float mine = 0.f;                    // lane m keeps output m
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m == lane16) mine = yacc[m];
                yacc[m] = 0.f;
            }
            if (a.splits == 1) {
                if (row_ok && lane16 < a.M) a.y[(size_t)lane16 * a.N + row] = mine;
            } else {
                if (row_ok && lane16 < a.M) a.partial[((size_t)split * a.M + lane16) * a.N + row] = mine;
                __threadfence();
                __syncthreads();
                if (tid == 0) s_last = atomicAdd(&a.counters[rb], 1u) == (unsigned)(a.splits - 1);
                __syncthreads();
                if (s_last) {
                    __threadfence();
                    for (int i = tid; i < kTeams * a.M; i += kThreads) {
                        const int m = i / kTeams;
                        const int r = rb * kTeams + (i - m * kTeams);
                        if (r < a.N) {
                            float sum = 0.f;
                            for (int sp = 0; sp < a.splits; ++sp)
                                sum += __ldcg(&a.partial[((size_t)sp * a.M + m) * a.N + r]);
                            a.y[(size_t)m * a.N + r] = sum;
                        }
                    }
                    if (tid == 0) a.counters[rb] = 0u;
                }
            }
        }
        if (!has_next) break;
        rb = nrb;
        ch = nch;
#pragma unroll
        for (int j = 0; j < kSlots; ++j) {
            w[j] = wn[j];
            sc[j] = scn[j];
        }
    }
}

template <int MT, bool XBF16>
const void* ffma_kernel_ptr() { return reinterpret_cast<const void*>(&gemv_ffma_kernel<MT, XBF16>); }

const void* pick_ffma(int mt, bool bf16)
{
    switch (mt) {
    case 1: return bf16 ? ffma_kernel_ptr<1, true>() : ffma_kernel_ptr<1, false>();
    case 2: return bf16 ? ffma_kernel_ptr<2, true>() : ffma_kernel_ptr<2, false>();
    case 4: return bf16 ? ffma_kernel_ptr<4, true>() : ffma_kernel_ptr<4, false>();
    case 8: return bf16 ? ffma_kernel_ptr<8, true>() : ffma_kernel_ptr<8, false>();
    default: return bf16 ? ffma_kernel_ptr<16, true>() : ffma_kernel_ptr<16, false>();
    }
}

int round_m(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

constexpr int kSmemBudget = 96 * 1024;          // x stage per block, keeps >= 2 blocks per SM

}  // namespace

namespace {
bool plan_gemv_generic(int64_t M, int64_t N, int64_t K, q4_dtype xt, const DeviceInfo& dev, GemvPlan* p)
{
    const int mt = round_m(M);
    const int G = (int)(K / 32);
    const int row_blocks = (int)((N + kTeams - 1) / kTeams);
    // Skinny shapes: split K until every SM has a block, keeping >= 16 groups per split.
    int splits = 1;
    while ((long long)row_blocks * splits < dev.sm_count && G / (splits + 1) >= kTeam) ++splits;
    const int ksg = (G + splits - 1) / splits;
    splits = (G + ksg - 1) / ksg;
    if (splits > 1 && row_blocks > kCounterSlots) splits = 1;   // cannot happen while SMs < 1024

    // x staging: as many groups as the shared-memory budget holds, in whole chunks.
    const int cap_raw = kSmemBudget / (mt * 128);
    int chunk = cap_raw >= kChunkGroups ? kChunkGroups : (cap_raw / kTeam) * kTeam;
    if (chunk < kTeam) chunk = kTeam;
    int xcap = (cap_raw / chunk) * chunk;
    if (xcap < chunk) xcap = chunk;
    const int held = ksg < xcap ? ksg : xcap;

    p->kernel = 0;
    p->splits = splits;
    p->groups_per_split = ksg;
    p->row_blocks = row_blocks;
    p->chunk = chunk;
    p->xcap = xcap;
    p->smem_bytes = mt * held * 128;
    const int per_sm = blocks_per_sm(pick_ffma(mt, xt == Q4_BF16), kThreads, (size_t)p->smem_bytes);
    if (per_sm < 1) return false;
    const long long resident = (long long)dev.sm_count * per_sm;
    long long gx = (resident + splits - 1) / splits;
    if (gx > row_blocks) gx = row_blocks;
    if (gx < 1) gx = 1;
    p->grid_x = (int)gx;
    p->workspace_bytes = 0;
    if (splits > 1) p->workspace_bytes = kCounterBytes + (size_t)splits * (size_t)M * (size_t)N * sizeof(float);
    return true;
}
}  // namespace

namespace {
q4_status launch_gemv_generic(const void* x, q4_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                              const uint16_t* scales, int64_t N, float* y, void* workspace,
                              const GemvPlan& plan, cudaStream_t stream)
{
    GemvArgs a;
    a.x = x;
    a.packed = packed;
    a.scales = scales;
    a.y = y;
    a.partial = nullptr;
    a.counters = nullptr;
    if (plan.splits > 1) {
        a.counters = reinterpret_cast<unsigned*>(workspace);
        a.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + kCounterBytes);
    }
    a.M = (int)M;
    a.N = (int)N;
    a.G = (int)(K / 32);
    a.ksg = plan.groups_per_split;
    a.splits = plan.splits;
    a.row_blocks = plan.row_blocks;
    a.chunk = plan.chunk;
    a.xcap = plan.xcap;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid_x, (unsigned)plan.splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)plan.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&a};
    const cudaError_t err = cudaLaunchKernelExC(&cfg, pick_ffma(round_m(M), xt == Q4_BF16), args);
    return err == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace

bool plan_gemv(int64_t M, const q4_weight* mats, int count, int64_t K, q4_dtype xt, const DeviceInfo& dev,
               bool sizing_only, GemvPlan* p)
{
    if (count < 1 || count > Q4_MULTI_MAX) return false;
    // Workspace the generic kernel needs for the largest of the matrices (it serves
    // them one launch each when the TMA kernels cannot).
    size_t generic_ws = 0;
    GemvPlan g = {};
    for (int i = 0; i < count; ++i) {
        if (!plan_gemv_generic(M, mats[i].N, K, xt, dev, &g)) return false;
        if (g.workspace_bytes > generic_ws) generic_ws = g.workspace_bytes;
    }
    bool eligible = true;
    for (int i = 0; i < count; ++i)
        eligible = eligible && (sizing_only ? tma_gemv_eligible(M, K, xt, nullptr, nullptr)
                                            : tma_gemv_eligible(M, K, xt, mats[i].packed, mats[i].scales));
    int64_t Ns[Q4_MULTI_MAX];
    for (int i = 0; i < count; ++i) Ns[i] = mats[i].N;
    if (eligible && plan_gemv_tma(M, Ns, count, K, xt, dev, p)) {
        if (sizing_only && generic_ws > p->workspace_bytes) p->workspace_bytes = generic_ws;
        return true;
    }
    *p = g;
    p->kernel = 0;
    p->workspace_bytes = generic_ws;
    return true;
}

q4_status launch_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const q4_weight* mats, int count,
                      uint32_t flags, void* workspace, const GemvPlan& plan, cudaStream_t stream)
{
    if (plan.kernel == 1)
        return launch_gemv_tma(x, xt, M, K, mats, count, (flags & Q4_WEIGHTS_STATIC) ? 1 : 0, workspace, plan,
                               stream);
    DeviceInfo dev;
    q4_status st = current_device(&dev);
    if (st != Q4_OK) return st;
    for (int i = 0; i < count; ++i) {        // one generic launch per matrix, in order on the stream
        GemvPlan g;
        if (!plan_gemv_generic(M, mats[i].N, K, xt, dev, &g)) return Q4_ERR_CUDA;
        st = launch_gemv_generic(x, xt, M, K, mats[i].packed, mats[i].scales, mats[i].N, mats[i].y, workspace, g,
                                 stream);
        if (st != Q4_OK) return st;
    }
    return Q4_OK;
}

}  // namespace q4
