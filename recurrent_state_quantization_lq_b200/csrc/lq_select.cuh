// Top-n selection shared by the state codec kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lq {

// The indices of the `n` (<= 8) largest of the D (<= 128) non-negative
// scores, in order, ties to the lower index, packed one byte each (0xff when
// unused); every lane of every calling warp returns the same list.
// Non-negative floats order like their bit patterns, so each pick is one
// integer maximum over the warp and the lowest index holding it (a ballot per
// 32 scores); taken scores drop out of later picks.
template <int D>
__device__ __forceinline__ uint2 select_top(const float *score, int n) {
    static_assert(D <= 128, "indices are packed in bytes");
    uint2 sel = make_uint2(0xffffffffu, 0xffffffffu);
    const int lane = threadIdx.x & 31;
    uint32_t key[D / 32];
#pragma unroll
    for (int k = 0; k < D / 32; ++k) key[k] = __float_as_uint(score[k * 32 + lane]);
    uint32_t taken = 0;                        // bit k: this lane's score k is taken
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        if (c < n) {
            uint32_t mx = 0;
#pragma unroll
            for (int k = 0; k < D / 32; ++k) mx = max(mx, ((taken >> k) & 1u) ? 0u : key[k]);
            mx = __reduce_max_sync(0xffffffffu, mx);
            int idx = -1;
#pragma unroll
            for (int k = 0; k < D / 32; ++k) {
                const uint32_t hit = __ballot_sync(0xffffffffu, !((taken >> k) & 1u) && key[k] == mx);
                if (idx < 0 && hit != 0u) idx = k * 32 + __ffs(hit) - 1;
            }
            const uint32_t keep = ~(0xffu << (8 * (c & 3))), put = (uint32_t)idx << (8 * (c & 3));
            if (c < 4) sel.x = (sel.x & keep) | put;
            else sel.y = (sel.y & keep) | put;
            if (idx >= 0 && (idx & 31) == lane) taken |= 1u << (idx >> 5);
        }
    }
    return sel;
}

__device__ __forceinline__ int sel_at(uint2 sel, int c) {
    return (int)(((c < 4 ? sel.x : sel.y) >> (8 * (c & 3))) & 0xffu);
}

}  // namespace lq
