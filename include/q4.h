/*
 * q4.h - C ABI of the B200 (sm_100a) Q4 weight-only quantisation library.
 *
 * Weight format.  The QORA-4B thread (zingnex.cn, section "量化与内存管理") and
 * the QORA-LLM-0.8B model card (section "Weight Format") quantise weights to
 * 4 bits, symmetrically, in groups of 32 along the reduction axis K, with one
 * scale per group.  They leave the encoding details open; this library fixes
 * them as follows, for a weight matrix W[N,K] (row n = one output feature):
 *
 *   for every row n and group g (the 32 values W[n, 32g .. 32g+31]):
 *     amax = max |w|                               exact
 *     s    = binary16_rne( f32(amax) / 7 )         IEEE f32 division, then round to
 *                                                  nearest even into binary16
 *     if s == +0: every code is 8 (each byte 0x88) and the stored scale is 0x0000
 *     else:      code_k = clamp(rint_even(w_k / f32(s)), -8, 7) + 8   (f32 division)
 *   packed[n, k/2] = code_{2i} | code_{2i+1} << 4   (low nibble = even k)
 *   scales[n, g]   = s (binary16 bit pattern)
 *   dequantised weight w'[n,k] = (code - 8) * f32(s)
 *
 * A group holding a NaN or an infinity, or whose scale would round to binary16
 * infinity (amax/7 >= 65520), is stored as a zero group and reported through the
 * flag word (Q4_FLAG_NONFINITE, Q4_FLAG_SCALE_OVERFLOW).
 *
 * Products.  The pages run "multi-threaded GEMV/GEMM" against these weights
 * (model card, "Weight Format"; "File Structure": GEMV/GEMM kernels for Q4,
 * prefill).  Here:
 *   y[m, n] = sum_k x[m, k] * w'[n, k]        (x row-major [M,K], y row-major [M,N])
 * q4_gemv serves decode (M = 1..16: one token, or a few tokens verified together);
 * q4_gemm serves prefill (large M: projections batched across the prompt's tokens,
 * QORA-4B thread, section "GPU 预填充优化").
 *
 * Conventions for every entry point:
 *  - Pointers named d_* / documented as device pointers must point to device
 *    memory of the current CUDA device.  The caller allocates and owns every
 *    buffer; the library allocates nothing and keeps no state between calls
 *    except cached device attributes.
 *  - All matrices are dense, contiguous and row-major.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously; argument errors are returned synchronously before
 *    anything is enqueued; a launch failure returns Q4_ERR_CUDA.
 *  - No entry point traps, asserts or aborts.  Functions are thread-safe;
 *    calls that share an output or workspace buffer must not overlap in time.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum q4_status {
    Q4_OK = 0,
    Q4_ERR_INVALID_ARG = 1,        /* a required pointer is NULL, or an enum is out of range */
    Q4_ERR_SHAPE = 2,              /* K not a positive multiple of 32, N < 0, M out of range */
    Q4_ERR_ALIGN = 3,              /* a pointer violates its documented alignment */
    Q4_ERR_DTYPE = 4,              /* unsupported data type for this entry point */
    Q4_ERR_WORKSPACE = 5,          /* workspace missing or smaller than required */
    Q4_ERR_CUDA = 6,               /* a CUDA runtime call or kernel launch failed */
    Q4_ERR_UNSUPPORTED_DEVICE = 7  /* current device is not compute capability 10.0 */
} q4_status;

typedef enum q4_dtype {
    Q4_F32 = 0,
    Q4_BF16 = 1                    /* bfloat16, passed as its 16-bit pattern */
} q4_dtype;

#define Q4_FLAG_NONFINITE 1u
#define Q4_FLAG_SCALE_OVERFLOW 2u

#define Q4_GEMV_MAX_M 16
#define Q4_MULTI_MAX 4
#define Q4_WEIGHTS_STATIC 1u

/* Version of this ABI (incremented on any incompatible change). */
Q4_API int q4_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
Q4_API const char* q4_status_string(q4_status status);

#define Q4_DEVICE_ERR_WAIT_TIMEOUT 1u

/*
 * Kernels never trap: a kernel whose bounded wait (on a TMA transfer, through an
 * mbarrier) runs out records Q4_DEVICE_ERR_WAIT_TIMEOUT in a per-device error word,
 * drains its own transfers and returns; its output is then undefined.
 * q4_device_error reads that word for the current device into *out (synchronous,
 * after all previously issued work that wrote it) and clears it when `clear` is
 * non-zero.  Returns Q4_ERR_INVALID_ARG for a NULL out, Q4_ERR_CUDA on a failed copy.
 */
Q4_API q4_status q4_device_error(uint32_t* out, int clear);

/*
 * q4_set_consumer_wait_limit: sets, for every device and every later launch of the TMA
 * GEMV kernels (q4_gemv, q4_gemv_multi, q4_gemv_noalloc, q4_gemv_host, q4_gemv_gate_up,
 * q4_gemv_argmax, q4_gemv_topk), how long a warp waits for one of its own TMA transfers
 * before it gives up, in nanoseconds, and returns the previous limit.  The default is
 * 1,000,000,000 (1 s); every legitimate wait lasts microseconds.  0 makes each launch
 * give up at its first wait: the kernel then records Q4_DEVICE_ERR_WAIT_TIMEOUT, waits
 * (up to 1 s, a limit this call does not change) for the transfers it has in flight,
 * leaves any workspace it shares zero at rest as a completed call does, and returns
 * with an undefined output.  This exercises the failure path without any fault; it
 * exists for tests of that path.  Not synchronised with launches in flight: a launch
 * uses the value set when it was enqueued.
 */
Q4_API uint64_t q4_set_consumer_wait_limit(uint64_t ns);

/*
 * q4_quantize: encode W[N,K] (f32, device) into the Q4 format above.
 *   W       device, f32 [N,K], 16-byte aligned.
 *   N, K    N >= 0 (N == 0 enqueues nothing and returns Q4_OK);
 *           K >= 32 and K % 32 == 0.
 *   packed  device, uint8 [N, K/2], 16-byte aligned (output).
 *   scales  device, binary16 bits [N, K/32], 2-byte aligned (output).
 *   flags   device uint32 or NULL.  When given, the kernel ORs Q4_FLAG_* bits
 *           into *flags; the caller clears it beforehand if it wants only this
 *           call's flags.
 * The result is bit-identical to the definition above for every input.
 */
Q4_API q4_status q4_quantize(const float* W, int64_t N, int64_t K,
                      uint8_t* packed, uint16_t* scales, uint32_t* flags, void* stream);

/*
 * Bytes of workspace q4_gemv needs for this shape (0 when none).  When the
 * shape is split along K across thread blocks, the workspace holds the f32
 * partial sums and one arrival counter per block of rows.
 */
Q4_API size_t q4_gemv_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * q4_gemv: y = x . dequant(W)^T for M = 1..16 (decode).
 *   x          device, [M,K] f32 or bfloat16 (x_dtype), 16-byte aligned.
 *   M          0 .. Q4_GEMV_MAX_M (M == 0 or N == 0 enqueues nothing).
 *   K, N       as for q4_quantize.
 *   packed, scales  the Q4 encoding of W[N,K] (16-byte / 2-byte aligned).
 *   y          device, f32 [M,N], 4-byte aligned (output, overwritten).
 *   workspace  device, at least q4_gemv_workspace_size(M,N,K) bytes, 16-byte
 *              aligned; may be NULL when that size is 0.  It must be zero-filled
 *              before its first use.  Every completed call leaves the part that
 *              must start at zero (the arrival counters) at zero again, so the
 *              same workspace can be reused by later calls without clearing.
 *              Calls that share a workspace must not overlap on the GPU.
 * Arithmetic.  M = 1 (f32 or bf16 x): each box of 256 x values (8 groups) is scaled by a
 * power of two 2^F with max |x| * 2^F < 2^30, rounded once to integers and cut into four
 * base-256 digits; the codes times the digits are summed exactly on the integer tensor
 * cores per group, and each group's sum is multiplied by its scale, then by 2^-F, and
 * accumulated in f32 (per digit plane, combined at the end).  M >= 2 with bf16 x: the
 * codes become the bf16 values code - 8 exactly and multiply x on the bf16 tensor cores
 * (exact products, f32 sums), each group's sum scaled and accumulated in f32.  Other shapes (f32 x
 * with M >= 2, K % 256 != 0, scales not 16-byte aligned): exact expansion and f32 FMAs.
 */
Q4_API q4_status q4_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K,
                  const uint8_t* packed, const uint16_t* scales, int64_t N,
                  float* y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * q4_gemv_host: q4_gemv from and to host memory, for a caller whose activations live on
 * the host: copies x_host into x_dev, runs q4_gemv into y_dev, copies y_dev into y_host
 * and waits for the stream.  On return y_host holds the product.
 *   x_host   host, [M,K] f32 or bfloat16 (x_dtype); page-locked memory makes the copy
 *            asynchronous (pageable memory works, the runtime stages it).
 *   y_host   host, f32 [M,N] (output).
 *   x_dev    device staging buffer of M*K elements of x_dtype, 16-byte aligned.
 *   y_dev    device staging buffer, f32 [M,N], 4-byte aligned (overwritten).
 *   flags    0 or Q4_WEIGHTS_STATIC (as for q4_gemv_multi).
 *   Other arguments, the arithmetic and the errors as for q4_gemv; argument errors return
 *   before any copy is enqueued.  M == 0 or N == 0 is a no-op.  The call blocks the host
 *   until the stream's work up to and including the copy of y has finished.
 */
Q4_API q4_status q4_gemv_host(const void* x_host, q4_dtype x_dtype, int64_t M, int64_t K,
                              const uint8_t* packed, const uint16_t* scales, int64_t N,
                              float* y_host, void* x_dev, float* y_dev, uint32_t flags,
                              void* workspace, size_t workspace_bytes, void* stream);

/* One weight matrix of a q4_gemv_multi call and its output. */
typedef struct q4_weight {
    const uint8_t* packed;    /* device, codes [N, K/2], 16-byte aligned */
    const uint16_t* scales;   /* device, binary16 bits [N, K/32], 2-byte aligned */
    int64_t N;                /* output features (rows), >= 0 */
    float* y;                 /* device, f32 [M, N], 4-byte aligned (output, overwritten) */
} q4_weight;

/* Workspace bytes for q4_gemv_multi with these row counts (0 when none). */
Q4_API size_t q4_gemv_multi_workspace_size(int64_t M, int64_t K, const int64_t* Ns, int count);

/*
 * q4_gemv_multi: y_i = x . dequant(W_i)^T for up to Q4_MULTI_MAX weight matrices that
 * share x (the several projections of one token, e.g. query/key/value or gate/up, as in
 * the fused gate+up decode of the QORA-LLM-0.8B model card, section "AVX-512 SIMD
 * Acceleration"), in one launch.  Same arithmetic, layouts and alignment as q4_gemv,
 * which is the count == 1 case.  Matrices with N == 0 are skipped.
 *   mats     host array of `count` (1..Q4_MULTI_MAX) q4_weight; all share K.
 *   flags    0, or Q4_WEIGHTS_STATIC: the caller guarantees no kernel still in flight
 *            on `stream` writes any packed/scales buffer of `mats`, which lets the
 *            kernel stream the weights while its predecessor on the stream finishes
 *            (x and the outputs are only touched after the predecessor completes).
 *   workspace  as for q4_gemv, sized by q4_gemv_multi_workspace_size.
 */
Q4_API q4_status q4_gemv_multi(const void* x, q4_dtype x_dtype, int64_t M, int64_t K,
                               const q4_weight* mats, int count, uint32_t flags,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * q4_gemv_gate_up: the fused gate+up of an MLP decode step (QORA-LLM-0.8B model card,
 * section "AVX-512 SIMD Acceleration": "Fused gate+up", both projections decoded in one
 * pass over x).  The page names no activation; the model card's one activation is SiLU,
 * so the gated product is SwiGLU's:
 *     y[m, n] = silu(g[m, n]) * u[m, n],   silu(g) = g / (1 + exp(-g)),
 *     g = x . dequant(Wg)^T,  u = x . dequant(Wu)^T   (f32 accumulation, as q4_gemv),
 * g and u never leave the chip: one launch, one f32 output.
 *   x        device, f32 (M == 1) or bfloat16 (M = 1..16) [M,K], 16-byte aligned.
 *   K        a multiple of 256 (the kernel streams 256-wide boxes; other K: Q4_ERR_SHAPE).
 *   gate_*, up_*  Q4 encodings of Wg[N,K] and Wu[N,K]: packed 16-byte aligned, scales
 *            16-byte aligned (Q4_ERR_ALIGN otherwise).
 *   y        device, f32 [M,N], 4-byte aligned (output, overwritten).
 *   flags    0 or Q4_WEIGHTS_STATIC, as for q4_gemv_multi.
 * No workspace (K is never split).  M == 0 or N == 0 is a no-op.
 */
Q4_API q4_status q4_gemv_gate_up(const void* x, q4_dtype x_dtype, int64_t M, int64_t K,
                                 const uint8_t* gate_packed, const uint16_t* gate_scales,
                                 const uint8_t* up_packed, const uint16_t* up_scales, int64_t N,
                                 float* y, uint32_t flags, void* stream);

/*
 * q4_gemv_argmax: greedy decoding over an LM head in one launch: for each x row m,
 *     index[m] = the row n with the largest y[m, n] = x . dequant(W)^T (f32, as q4_gemv),
 *     the lowest such n on ties; a NaN logit counts as the largest value;
 *     value[m] = y[m, index[m]].
 * The logits need not leave the chip (QORA-4B thread, section "量化与内存管理": the LM head
 * is one of the parallel workloads; QORA-LLM-0.8B model card, section "CLI Flags":
 * --greedy, temperature 0).  Shapes, dtypes and alignment as for q4_gemv_gate_up
 * (K % 256 == 0; M == 1 with f32 x or M = 1..16 with bf16 x; scales 16-byte aligned).
 *   y        device f32 [M,N] or NULL: when given, the logits are written too.
 *   index    device int64 [M], 8-byte aligned (output).
 *   value    device f32 [M] or NULL (output).
 *   workspace  device, q4_gemv_argmax_workspace_size() bytes, 16-byte aligned, all zero
 *            before the first call; every call leaves it zero again, so one workspace
 *            serves every call on a stream (calls in flight at the same time on
 *            different streams need their own).
 * K is never split.  M == 0 or N == 0 is a no-op.
 */
Q4_API size_t q4_gemv_argmax_workspace_size(void);
Q4_API q4_status q4_gemv_argmax(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                                const uint16_t* scales, int64_t N, float* y, int64_t* index, float* value,
                                uint32_t flags, void* workspace, size_t workspace_bytes, void* stream);

/*
 * q4_gemv_topk: the k largest logits of an LM head per x row in one launch: for each x
 * row m, index[m][0..k-1] are the rows n of the k largest y[m, n] = x . dequant(W)^T (f32,
 * as q4_gemv), larger value first, the lower n among equal values, a NaN logit above
 * every number; value[m][i] = y[m, index[m][i]].  Rows are reported as row_base + n, so
 * that an LM head split by rows across devices reports global rows.  When N < k the
 * tail of each list holds index -1 and value NaN.
 * The list is what a top-k sampler draws from (QORA-LLM-0.8B model card, section
 * "Sampling Defaults": top_k 20); the logits need not leave the chip.  Shapes, dtypes and
 * alignment as for q4_gemv_argmax.
 *   k        1 .. Q4_TOPK_MAX.
 *   row_base >= 0, with row_base + N <= 2^31 - 1 (Q4_ERR_SHAPE otherwise).
 *   y        device f32 [M,N] or NULL: when given, the logits are written too.
 *   index    device int64 [M,k], 8-byte aligned (output).
 *   value    device f32 [M,k] or NULL (output).
 *   workspace  device, at least q4_gemv_topk_workspace_size(M, N, K, k, x_dtype) bytes
 *            (0 when the shape is not served or no device is current), 16-byte aligned;
 *            its first 16 bytes must be zero before the first call and every call leaves
 *            them zero again (one workspace per stream, as for q4_gemv_argmax).
 * K is never split.  M == 0 or N == 0 is a no-op (nothing is written).
 */
#define Q4_TOPK_MAX 32
Q4_API size_t q4_gemv_topk_workspace_size(int64_t M, int64_t N, int64_t K, int64_t k, q4_dtype x_dtype);
Q4_API q4_status q4_gemv_topk(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint8_t* packed,
                              const uint16_t* scales, int64_t N, int64_t k, int64_t row_base, float* y,
                              int64_t* index, float* value, uint32_t flags, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * q4_topk_merge: the k best entries per x row over S top-k lists, ordered as q4_gemv_topk
 * orders them (larger value first, the lower row among equal values, a NaN above every
 * number).  With an LM head split by rows across S devices, each device runs
 * q4_gemv_topk on its rows with row_base = its first row, the [M,k] lists are gathered
 * (S * M * k entries, the only exchange), and this call selects the global top k
 * (QORA-LLM-0.8B model card, section "Sampling Defaults": top_k 20; QORA-4B thread,
 * section "量化与内存管理": the LM head among the parallel workloads).
 *   values   device f32 [S,M,k], 4-byte aligned; indices device int64 [S,M,k], 8-byte
 *            aligned: list s of x row m at [s,m,:].  An index outside [0, 2^31 - 1)
 *            (such as the -1 of a short list) marks padding and is skipped.  Rows must be
 *            distinct across the lists of one x row (disjoint shards).
 *   S        1 .. 2^20 lists;  M >= 0 x rows (0: no-op);  k 1 .. Q4_TOPK_MAX.
 *   index    device int64 [M,k], 8-byte aligned (output); value f32 [M,k] or NULL.
 * When fewer than k entries exist the tail holds index -1 and value NaN.
 */
Q4_API q4_status q4_topk_merge(const float* values, const int64_t* indices, int64_t S, int64_t M, int64_t k,
                               int64_t* index, float* value, void* stream);

/*
 * INT8 weights, for models that mix INT8 and INT4 layers (QKV-Core thread, section
 * "自适应混合量化": precision-sensitive attention layers in INT8, feed-forward layers in
 * INT4).  The page gives no encoding; this library's INT8 format is the Q4 one with 8-bit
 * codes, per group of 32 consecutive k of a row:
 *   amax = max |w| (exact);  s = binary16_rne(f32_rn(amax / 127))
 *   s == 0 (or a non-finite group, or amax / 127 overflowing binary16): codes 0, scale 0,
 *     and the Q4_FLAG_* bit as for q4_quantize
 *   otherwise q = clamp(rint(w / f32(s)), -128, 127) (f32 division, ties to even),
 *     stored as a two's-complement int8; dequantised w' = q * f32(s).
 *
 * q4_int8_quantize: W f32 [N,K] (device, 16-byte aligned) -> codes int8 [N,K] (device,
 *   16-byte aligned) + scales binary16 bits [N,K/32] (2-byte aligned); flags as for
 *   q4_quantize.  N, K as for q4_quantize.  Bit-identical to the definition above.
 * q4_int8_gemv: y[M,N] (f32) = x[M,K] . dequant(W)^T for M = 1..16, x f32 or bfloat16
 *   (device, 16-byte aligned, the same contract as q4_gemv, so one x serves both formats),
 *   codes 16-byte aligned, scales 2-byte aligned, y 4-byte aligned.  M == 1 with
 *   K % 256 == 0 and 16-byte aligned scales runs on the Q4 GEMV's TMA kernel: x is cut
 *   into exact digit planes as for q4_gemv (per box of 256, max |x| * 2^F < 2^30) and
 *   the codes multiply them on the integer tensor cores with exact int32 group sums, each
 *   scaled by its binary16 scale and by 2^-F and accumulated in f32.  Other shapes stage
 *   x in shared memory as f32 (M*K*4 bytes; a shape whose x does not fit returns
 *   Q4_ERR_SHAPE) and form products in f32 per group of 16 k, scaled and accumulated in
 *   f32.  No workspace.  M == 0 or N == 0 is a no-op.
 */
Q4_API q4_status q4_int8_quantize(const float* W, int64_t N, int64_t K, int8_t* codes, uint16_t* scales,
                                  uint32_t* flags, void* stream);
Q4_API q4_status q4_int8_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const int8_t* codes,
                              const uint16_t* scales, int64_t N, float* y, void* stream);

/*
 * q4_gemv_mixed: the projections of one token against weights of mixed precision, INT8
 * and Q4 matrices side by side (QKV-Core thread, section "自适应混合量化": precision-
 * sensitive layers in INT8, the rest in INT4): y_i = x . dequant_i(W_i)^T for up to
 * Q4_MULTI_MAX matrices sharing x and K.
 *   mats[i].codes   device: Q4 packed codes [N, K/2] (bits == 4, the q4_quantize format) or
 *                   INT8 codes [N, K] (bits == 8, the q4_int8_quantize format), 16-byte aligned.
 *   mats[i].scales  device, binary16 bits [N, K/32], 2-byte aligned.
 *   mats[i].y       device, f32 [M, N], 4-byte aligned (output, overwritten).
 *   mats[i].bits    4 or 8; mats[i].reserved must be 0 (Q4_ERR_INVALID_ARG otherwise).
 *   x, M, K, flags  as for q4_gemv_multi (x 16-byte aligned).
 *   workspace  at least q4_gemv_mixed_workspace_size(M, K, mats, count) bytes, as for
 *              q4_gemv_multi (zero before its first use, left zero by every call).
 * With M == 1, K % 256 == 0 and 16-byte aligned scales every matrix streams through one
 * launch of the TMA kernel (the INT8 rows take the q4_int8_gemv arithmetic, the Q4 rows
 * the q4_gemv arithmetic); otherwise the Q4 matrices run in one q4_gemv_multi launch and
 * each INT8 matrix in its own q4_int8_gemv launch, in that order on the stream.
 * Matrices with N == 0 are skipped; M == 0 is a no-op.
 */
typedef struct q4_mixed_weight {
    const void* codes;        /* device: Q4 packed [N, K/2] or INT8 [N, K] codes */
    const uint16_t* scales;   /* device, binary16 bits [N, K/32] */
    int64_t N;                /* output features (rows), >= 0 */
    float* y;                 /* device, f32 [M, N] (output) */
    int32_t bits;             /* 4 or 8 */
    int32_t reserved;         /* 0 */
} q4_mixed_weight;

Q4_API size_t q4_gemv_mixed_workspace_size(int64_t M, int64_t K, const q4_mixed_weight* mats, int count);
Q4_API q4_status q4_gemv_mixed(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const q4_mixed_weight* mats,
                               int count, uint32_t flags, void* workspace, size_t workspace_bytes, void* stream);

/*
 * q4_f16_gemv: y[M,N] = x[M,K] . W^T for binary16 weights W (2 bytes per weight), the
 * pages' second weight format (QORA-LLM-0.8B model card, section "AVX-512 SIMD
 * Acceleration": "F16 GEMV").  Same roles as q4_gemv, without quantisation:
 *   x        device, f32 (M == 1) or bfloat16 (M = 1..16) [M,K], 16-byte aligned.
 *   K        a positive multiple of 8 (16-byte weight rows); any such K.
 *   w        device, binary16 bits [N,K] row-major, 16-byte aligned.
 *   y        device, f32 [M,N], 4-byte aligned (output, overwritten).
 *   flags    0 or Q4_WEIGHTS_STATIC, as for q4_gemv_multi.
 * Arithmetic: the products run on the tensor cores with binary16 operands and f32
 * accumulation.  bf16 x row m is scaled by a power of two 2^-e_m that puts max |x| in
 * [2^14, 2^15) and converted to binary16, exact for every value above max |x| * 2^-24;
 * f32 x is split into two binary16 parts (22 significant bits); y is scaled back by
 * 2^e_m.  No workspace.  M == 0 or N == 0 is a no-op; a K whose x does not fit in
 * shared memory returns Q4_ERR_SHAPE.
 */
Q4_API q4_status q4_f16_gemv(const void* x, q4_dtype x_dtype, int64_t M, int64_t K, const uint16_t* w, int64_t N,
                             float* y, uint32_t flags, void* stream);

/*
 * q4_gemm: y = bf16( x . dequant(W)^T ) for prefill (any M >= 0; tuned for M >= 512).
 * The pages batch the prefill projections across tokens into GEMMs (QORA-4B thread,
 * section "GPU 预填充优化"; QORA-LLM-0.8B model card, section "Performance").
 *   x        device, bfloat16 [M,K], 16-byte aligned.
 *   K, N     as for q4_quantize (K % 32 == 0, K >= 32; N >= 0).
 *   packed, scales  the Q4 encoding of W[N,K] (16-byte / 2-byte aligned).
 *   y        device, bfloat16 [M,N], 2-byte aligned (output, overwritten); stores are
 *            vectorised when y is 16-byte aligned and N % 8 == 0.
 * Arithmetic: each weight becomes bf16_rn((code - 8) * f32(scale)) (one rounding of an
 * exact product), products run on the tensor cores (tcgen05) with f32 accumulation,
 * and each f32 output is rounded to nearest-even bfloat16.  At small M the K range of a
 * tile may be split over the 2 CTA pairs of one cluster, whose f32 partial tiles are
 * summed in a fixed order before the rounding (results are repeatable bit for bit).
 * M == 0 or N == 0 is a no-op.  No workspace.
 */
Q4_API q4_status q4_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed,
                         const uint16_t* scales, int64_t N, uint16_t* y, void* stream);

/*
 * q4_gemv_noalloc: q4_gemv for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for hosts that
 * cannot hand the library a workspace (runtimes that own all device memory and
 * give plugins no allocation hook, hosts that forbid allocation after start-up,
 * code running while another thread captures a CUDA graph in global mode).
 * Same inputs, outputs, layouts, alignment and arithmetic as q4_gemv; the
 * split-K scratch is one library-owned device array of 1 MiB per device
 * (held by every GPU that loads the library until the process exits) instead
 * of a workspace argument.  It calls no cudaMalloc/cudaFree.
 *  - The first call on a device performs a one-time set-up (looks up the
 *    array's address, zero-fills it and waits for the device), so make that
 *    first call before any stream capture on the device.  If the set-up fails
 *    the call returns Q4_ERR_CUDA and the next call on that device retries it.
 *  - All calls on a device share the array, which keeps the last call's
 *    contents: calls that overlap on the GPU race.  Serialise them.
 *  - A shape whose split needs more than 1 MiB of scratch returns
 *    Q4_ERR_WORKSPACE (none with M <= 16 on a 148-SM B200).
 */
Q4_API q4_status q4_gemv_noalloc(const void* x, q4_dtype x_dtype, int64_t M, int64_t K,
                                 const uint8_t* packed, const uint16_t* scales, int64_t N,
                                 float* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
