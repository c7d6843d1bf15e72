// Ordering of (logit, row) pairs for argmax and top-k selection (internal).
#pragma once

#include <stdint.h>

namespace q4 {

// Orderable 64-bit key of (logit v, row r): larger v wins, then the lower row; every NaN
// counts as the largest value (a NaN logit is reported, as numpy's argmax does) and -0
// equals +0 (both are reported as +0).
__device__ __forceinline__ unsigned long long argmax_key(float v, uint32_t r)
{
    uint32_t b = __float_as_uint(v);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) b = 0x7FC00000u;
    if (b == 0x80000000u) b = 0u;
    const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)ord << 32) | (0xFFFFFFFFu - r);
}

__device__ __forceinline__ float argmax_value(unsigned long long key)
{
    const uint32_t ord = (uint32_t)(key >> 32);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}

// A relaxed load of a key other blocks raise with atomicMax (always a valid lower bound,
// however stale).
__device__ __forceinline__ unsigned long long load_key_relaxed(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long key_max(unsigned long long a, unsigned long long b)
{
    return a > b ? a : b;
}

__device__ __forceinline__ unsigned long long key_min(unsigned long long a, unsigned long long b)
{
    return a < b ? a : b;
}

// Warp lists of keys are held one key per lane, in descending order across the lanes
// (lane 0 the largest); 0 is padding, below every live key (the row field of a live key
// is never 0).  Live keys are distinct.  Every function below must be called by all 32
// lanes of the warp together, and none of their shuffles sits behind a condition that
// differs by lane.

// Sorts the warp's 32 keys into a descending list (a bitonic sorting network: blocks of
// 2, 4, .. 32 lanes are merged, alternately ascending and descending, into the next size).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long v, int lane)
{
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int d = size >> 1; d > 0; d >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, d);
            const bool keep_max = ((lane & d) == 0) == ((lane & size) == 0);
            v = keep_max ? key_max(v, o) : key_min(v, o);
        }
    }
    return v;
}

// The 32 largest keys of two descending lists a and b, as a descending list: a against b
// reversed, lane by lane, keeps the top 32 as one bitonic sequence, which five
// half-cleaning steps put in order.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a, unsigned long long b, int lane)
{
    unsigned long long v = key_max(a, __shfl_sync(0xffffffffu, b, 31 - lane));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, d);
        v = (lane & d) == 0 ? key_max(v, o) : key_min(v, o);
    }
    return v;
}

// Candidates beyond this many are sorted and merged instead of inserted one by one.
constexpr int kSortInsert = 4;

// Adds the keys of the lanes in `mine` to a descending list whose first kk lanes are the
// kk largest keys seen; a key that does not beat the kk-th entry cannot enter them and is
// skipped.  Few candidates are inserted one at a time (the list shifts down one lane from
// the insertion point), many are sorted and merged.
// `floor` is a key no candidate needs to beat, as well as the list's k-th entry (0: none).
__device__ __forceinline__ void topk_insert(unsigned long long& list, unsigned long long key, bool mine, int kk,
                                            int lane, unsigned long long floor = 0ull)
{
    const unsigned long long last = key_max(__shfl_sync(0xffffffffu, list, kk - 1), floor);
    const bool want = mine && key > last;
    unsigned mask = __ballot_sync(0xffffffffu, want);
    if (__popc(mask) > kSortInsert) {               // the same on every lane
        list = warp_merge_desc(list, warp_sort_desc(want ? key : 0ull, lane), lane);
        return;
    }
    while (mask) {                                  // the same on every lane
        const int src = __ffs(mask) - 1;
        mask &= mask - 1;
        const unsigned long long c = __shfl_sync(0xffffffffu, key, src);
        const unsigned long long now_last = key_max(__shfl_sync(0xffffffffu, list, kk - 1), floor);
        if (c > now_last) {
            const int pos = __popc(__ballot_sync(0xffffffffu, list > c));   // entries above c
            const unsigned long long up = __shfl_up_sync(0xffffffffu, list, 1);
            list = lane == pos ? c : lane > pos ? up : list;
        }
    }
}

}  // namespace q4
