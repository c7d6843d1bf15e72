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

// A warp's top-k list: lane i holds the i-th largest key, lanes >= kk hold 0, which is
// below every live key (the row field of a live key is never 0).  Keys are distinct, so
// the list is strictly decreasing.  Inserts the keys of the lanes in `mine` that beat
// the list's last entry, in lane order.  Every lane of the warp must call it, and every
// shuffle below runs on all 32 lanes (none sits behind a condition that differs by lane).
__device__ __forceinline__ void topk_insert(unsigned long long& list, unsigned long long key, bool mine, int kk,
                                            int lane)
{
    const unsigned long long last = __shfl_sync(0xffffffffu, list, kk - 1);
    unsigned mask = __ballot_sync(0xffffffffu, mine && key > last);
    while (mask) {                                  // the same on every lane
        const int src = __ffs(mask) - 1;
        mask &= mask - 1;
        const unsigned long long c = __shfl_sync(0xffffffffu, key, src);
        const unsigned long long now_last = __shfl_sync(0xffffffffu, list, kk - 1);
        if (c > now_last) {
            const int pos = __popc(__ballot_sync(0xffffffffu, list > c));   // entries above c
            const unsigned long long up = __shfl_up_sync(0xffffffffu, list, 1);
            if (lane < kk) list = lane == pos ? c : lane > pos ? up : list;
        }
    }
}

}  // namespace q4
