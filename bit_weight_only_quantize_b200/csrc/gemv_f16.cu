// q4_f16_gemv: y[M,N] = x[M,K] . W^T for binary16 weights W[N,K] (2 bytes per weight),
// the pages' second weight format (QORA-LLM-0.8B model card, section "AVX-512 SIMD
// Acceleration": the F16 GEMV widens binary16 weights and multiply-adds them).
//
// The weights are already tensor-core operands, so the kernel has no decode step:
//  * W streams as TMA boxes of 16 rows x 64 k (128-byte rows, 128-byte swizzle); a ring
//    stage holds two boxes (16 rows x 128 k, 4 KiB) under one mbarrier, two stages per
//    warp, each warp issuing its own copies (as the Q4 kernel does).
//  * ldmatrix turns a box's 16 x 16 slices straight into the A operand of
//    mma.sync.m16n8k16 (binary16 in, f32 accumulate); the accumulators run over the
//    warp's whole K range, so nothing is read back until the row block ends.
//  * x becomes the B operand in binary16: bf16 x row m is multiplied by 2^-e_m (e_m puts
//    max |x| in [2^14, 2^15)), after which every bf16 value above max |x| * 2^-24 is
//    exact in binary16; y is multiplied back by 2^e_m.  f32 x (M == 1) is split into
//    two binary16 columns hi + lo (22 significant bits) whose results are added.
//  * Teams of P warps split the K range of a row block and add their sums in a fixed
//    order; the plan picks P and teams per block with the same cost model as the Q4
//    kernels.  Every mbarrier wait is bounded (see q4_device_error).
#include <algorithm>

#include "tma.cuh"

namespace q4 {
namespace {

constexpr int kRows = 16;
constexpr int kMaxWarps = 16;
constexpr int kStages = 2;
constexpr int kBoxK = 64;                         // k per box (128 bytes of binary16)
constexpr int kBoxBytes = kRows * kBoxK * 2;      // 2 KiB
constexpr int kUnitK = 2 * kBoxK;                 // k per ring stage
constexpr uint32_t kStageBytes = 2 * kBoxBytes;   // 4 KiB
constexpr uint64_t kWaitLimit = kWaitLimitNs;
constexpr double kMinWarpShare = 12.0;
constexpr double kEpilogueCost = 0.1;

struct F16Args {
    const void* x;
    float* y;
    int M, N, K;
    int xf32;                 // x is f32 (M == 1): columns 0, 1 = hi, lo
    int cols;                 // B columns staged (M, or 2 for f32 x)
    int nks;                  // k16 steps of x staged: ceil(K / 16)
    int row_blocks;
    int P, teams;
    int prefetch;
    unsigned* err;
};

__device__ __forceinline__ void team_sync_f16(int team, int P)
{
    if (P == 1) __syncwarp();
    else asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(P * 32) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += A . B, one m16n8k16 tile, binary16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint2 b)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
}

// 2^e as an exact f32 product of two factors, for e in [-140, 140].
__device__ __forceinline__ void pow2_pair(int e, float& a, float& b)
{
    const int h = e / 2;
    a = __int_as_float((127 + h) << 23);
    b = __int_as_float((127 + e - h) << 23);
}

__device__ __forceinline__ float x_at(const F16Args& a, int m, int k)
{
    if (k >= a.K) return 0.f;
    if (a.xf32) return reinterpret_cast<const float*>(a.x)[(size_t)m * a.K + k];
    const uint16_t b = reinterpret_cast<const uint16_t*>(a.x)[(size_t)m * a.K + k];
    return __uint_as_float((uint32_t)b << 16);
}

template <int NT>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
gemv_f16_kernel(const __grid_constant__ CUtensorMap wmap, const F16Args a)
{
    constexpr int MP = NT * 8;
    extern __shared__ unsigned char smem_raw[];
    __shared__ unsigned s_amax[16];
    const int W = blockDim.x >> 5;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* ring = smem;                                            // [warp][stage][2 boxes]
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring + W * kStages * kStageBytes);
    float* red = reinterpret_cast<float*>(bars + W * kStages);            // [warp][16 rows][MP]
    uint2* xb = reinterpret_cast<uint2*>(red + W * kRows * MP);            // [col][ks][t], then a zero column
    const int cstride = a.nks * 4 + 4;                                     // uint2 per column (padded)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = a.P;
    const int team = warp / P, wt = warp - team * P;
    const int nu = (a.K + kUnitK - 1) / kUnitK;
    const int u0 = wt * nu / P, nbw = (wt + 1) * nu / P - u0;
    const int first_rb = blockIdx.x * a.teams + team;
    const int rb_stride = gridDim.x * a.teams;
    const int nrb = (team < a.teams && first_rb < a.row_blocks)
                        ? (a.row_blocks - first_rb + rb_stride - 1) / rb_stride : 0;
    const int njobs = nrb * nbw;
    uint64_t* my_bars = bars + warp * kStages;

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // Job j: unit u0 + j % nbw (128 k) of the warp's (j / nbw)-th row block.
    int iss_u = 0, iss_rb = first_rb;
    auto issue = [&](int j) {
        const int s = j % kStages;
        const int k0 = (u0 + iss_u) * kUnitK;
        unsigned char* dst = ring + (warp * kStages + s) * kStageBytes;
        const int nbox = k0 + kBoxK < a.K ? 2 : 1;
        mbar_arrive_expect_tx(&my_bars[s], nbox * kBoxBytes);
        for (int q = 0; q < nbox; ++q)
            tma_load_2d(dst + q * kBoxBytes, &wmap, k0 + q * kBoxK, iss_rb * kRows, &my_bars[s]);
        if (++iss_u == nbw) {
            iss_u = 0;
            iss_rb += rb_stride;
        }
    };
    int issued = min(kStages, njobs);
    if (a.prefetch && lane == 0)
        for (int j = 0; j < issued; ++j) issue(j);
    pdl_launch_dependents();
    pdl_wait();
    if (!a.prefetch && lane == 0)
        for (int j = 0; j < issued; ++j) issue(j);

    // ---- stage x as binary16 B fragments: column c, k16 step ks, lane t holds
    //      (x[16 ks + 2t], x[16 ks + 2t + 1]) and (x[16 ks + 2t + 8], x[16 ks + 2t + 9]) ----
    const int xrows = a.xf32 ? 1 : a.M;
    if (threadIdx.x < 16) s_amax[threadIdx.x] = 0u;
    __syncthreads();
    for (int m = 0; m < xrows; ++m) {                                    // max |x| bits per row
        unsigned mx = 0u;
        for (int k = threadIdx.x; k < a.K; k += blockDim.x) mx = max(mx, __float_as_uint(fabsf(x_at(a, m, k))));
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0 && mx) atomicMax(&s_amax[m], mx);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (a.cols + 1) * a.nks * 4; i += blockDim.x) {
        const int c = i / (a.nks * 4), rem = i - c * a.nks * 4;
        const int ks = rem >> 2, t = rem & 3;
        uint32_t h[4] = {0u, 0u, 0u, 0u};
        if (c < a.cols) {
            const int m = a.xf32 ? 0 : c;
            const int eb = max((int)(s_amax[m] >> 23), 1);
            float sa, sb;
            pow2_pair(127 + 14 - eb, sa, sb);                               // 2^-e_m
            const int kk[4] = {16 * ks + 2 * t, 16 * ks + 2 * t + 1, 16 * ks + 2 * t + 8, 16 * ks + 2 * t + 9};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float v = x_at(a, m, kk[q]) * sa * sb;
                const __half hi = __float2half_rn(v);
                const __half val = (a.xf32 && c == 1) ? __float2half_rn(v - __half2float(hi)) : hi;
                h[q] = __half_as_ushort(val);
            }
        }
        xb[c * cstride + ks * 4 + t] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    }
    __syncthreads();

    // lane (g, t) supplies B column n * 8 + g (the zero column past the staged ones)
    const int g = lane >> 2, t = lane & 3;
    const uint2* xcol[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) xcol[n] = xb + min(n * 8 + g, a.cols) * cstride + t;
    // ldmatrix rows: lane 8i + r -> box row 8 (i & 1) + r, 16-byte chunk 2 ks + (i >> 1)
    const int lr = lane & 7, li = lane >> 3;
    const uint32_t lane_off = ((li & 1) * 8 + lr) * 128 + (((li >> 1) ^ lr) << 4);

    bool ok = true;
    int consumed = 0;
    for (int rbi = 0; rbi < nrb; ++rbi) {
        const int rb = first_rb + rbi * rb_stride;
        float acc[2][NT][4] = {};
        for (int jb = 0; jb < nbw; ++jb) {
            const int j = rbi * nbw + jb;
            const int s = j % kStages;
            if (ok) ok = mbar_wait_bounded(&my_bars[s], (uint32_t)(j / kStages) & 1u, kWaitLimit);
            if (ok) {
                consumed = j + 1;
                const int k0 = (u0 + jb) * kUnitK;
                const uint32_t st = smem_addr(ring + (warp * kStages + s) * kStageBytes) + lane_off;
#pragma unroll
                for (int kq = 0; kq < kUnitK / 16; ++kq) {              // 8 k16 steps per stage
                    const int ks = k0 / 16 + kq;
                    if (ks < a.nks) {
                        uint32_t ra[4];
                        // box kq / 4, chunk pair (kq % 4): the XOR reaches chunk 2 (kq % 4) + (i >> 1)
                        ldsm_x4((st + (kq >> 2) * kBoxBytes) ^ (uint32_t)((kq & 3) << 5), ra);
#pragma unroll
                        for (int n = 0; n < NT; ++n) mma_f16(acc[kq & 1][n], ra, xcol[n][ks * 4]);
                    }
                }
            }
            __syncwarp();
            if (ok && j + kStages < njobs) {
                if (lane == 0) {
                    fence_proxy_async_smem();
                    issue(j + kStages);
                }
                issued = j + kStages + 1;
            }
        }
        // ---- row block complete: team sum in warp order, then y (x scale undone) ----
        float* my_red = red + warp * kRows * MP;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            my_red[g * MP + n * 8 + 2 * t] = acc[0][n][0] + acc[1][n][0];
            my_red[g * MP + n * 8 + 2 * t + 1] = acc[0][n][1] + acc[1][n][1];
            my_red[(g + 8) * MP + n * 8 + 2 * t] = acc[0][n][2] + acc[1][n][2];
            my_red[(g + 8) * MP + n * 8 + 2 * t + 1] = acc[0][n][3] + acc[1][n][3];
        }
        team_sync_f16(team, P);
        if (wt == 0) {
            for (int e = lane; e < kRows * a.M; e += 32) {
                const int m = e / kRows, rr = e - m * kRows;
                float total = 0.f;
                for (int w = 0; w < P; ++w) {
                    const float* rw = red + (team * P + w) * kRows * MP + rr * MP;
                    total += a.xf32 ? rw[0] + rw[1] : rw[m];
                }
                const int row = rb * kRows + rr;
                if (row < a.N) {
                    float ya, yb;
                    pow2_pair(max((int)(s_amax[m] >> 23), 1) - 127 - 14, ya, yb);   // 2^e_m
                    a.y[(size_t)m * a.N + row] = total * ya * yb;
                }
            }
        }
        team_sync_f16(team, P);
    }

    if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrWaitTimeout);
        for (int j = consumed; j < issued; ++j)
            if (!mbar_wait_bounded(&my_bars[j % kStages], (uint32_t)(j / kStages) & 1u, kWaitLimit)) break;
    }
}

size_t f16_smem_bytes(int nt, int warps, int cols, int nks)
{
    const size_t ring = (size_t)warps * kStages * (kStageBytes + sizeof(uint64_t));
    const size_t red = (size_t)warps * kRows * nt * 8 * sizeof(float);
    const size_t xs = (size_t)(cols + 1) * (nks * 4 + 4) * sizeof(uint2);
    return 1024 + ring + red + xs;
}

const void* f16_kernel(int nt)
{
    return nt == 1 ? reinterpret_cast<const void*>(&gemv_f16_kernel<1>)
                   : reinterpret_cast<const void*>(&gemv_f16_kernel<2>);
}

}  // namespace

q4_status launch_f16_gemv(const void* x, q4_dtype xt, int64_t M, int64_t K, const uint16_t* w, int64_t N, float* y,
                          int prefetch, cudaStream_t stream, const DeviceInfo& dev)
{
    const bool xf32 = xt == Q4_F32;
    const int cols = xf32 ? 2 : (int)M;
    const int nt = cols <= 8 ? 1 : 2;
    const int nks = (int)((K + 15) / 16);
    const long long rbl = (N + kRows - 1) / kRows;
    if (rbl > INT32_MAX) return Q4_ERR_SHAPE;
    const int row_blocks = (int)rbl;
    const int units = (int)((K + kUnitK - 1) / kUnitK);
    const size_t budget = (size_t)dev.max_smem_optin - 512;
    const size_t per_warp = (size_t)kStages * (kStageBytes + sizeof(uint64_t)) + (size_t)kRows * nt * 8 * sizeof(float);
    const size_t xs = f16_smem_bytes(nt, 0, cols, nks) - 1024;
    if (1024 + xs + per_warp > budget) return Q4_ERR_SHAPE;          // x of this K does not fit
    const size_t fitw = (budget - 1024 - xs) / per_warp;
    const int wb = (int)std::min<size_t>(fitw, kMaxWarps);
    // Team size P and teams per block: the Q4 kernels' cost model (no K split here).
    int P = 0, teams = 0;
    double best = 0.0;
    const long long sms = dev.sm_count;
    for (int pp = 1; pp <= units && pp <= wb; ++pp) {
        const int pwu = (units + pp - 1) / pp;
        long long tm = wb / pp;
        const long long spread = ((long long)row_blocks + sms - 1) / sms;
        if (tm > spread) tm = spread;
        const long long gxs = std::min(((long long)row_blocks + tm - 1) / tm, sms);
        const long long rounds = ((long long)row_blocks + gxs * tm - 1) / (gxs * tm);
        const double share = std::max((double)(tm * pp), kMinWarpShare) / 16.0;
        const double cost = (double)rounds * (pwu + kEpilogueCost) * share;
        if (P == 0 || cost < best - 1e-9) {
            P = pp;
            teams = (int)tm;
            best = cost;
        }
    }
    const int warps = P * teams;
    const size_t smem = f16_smem_bytes(nt, warps, cols, nks);
    const int per_sm = blocks_per_sm(f16_kernel(nt), warps * 32, smem);
    if (per_sm < 1) return Q4_ERR_CUDA;
    long long gx = std::min<long long>(((long long)row_blocks + teams - 1) / teams, (long long)dev.sm_count * per_sm);
    if (gx < 1) gx = 1;

    CUtensorMap wmap;
    if (!encode_tma_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, kBoxK,
                       kRows, CU_TENSOR_MAP_SWIZZLE_128B))
        return Q4_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return Q4_ERR_CUDA;
    F16Args a;
    a.x = x;
    a.y = y;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.xf32 = xf32 ? 1 : 0;
    a.cols = cols;
    a.nks = nks;
    a.row_blocks = row_blocks;
    a.P = P;
    a.teams = teams;
    a.prefetch = prefetch;
    a.err = err;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx);
    cfg.blockDim = dim3((unsigned)(warps * 32));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&wmap, &a};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, f16_kernel(nt), args);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // namespace q4
