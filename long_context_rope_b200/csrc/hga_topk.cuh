// hga_topk.cuh -- warp-level exact top-k by radix select over 32-bit keys.
//
// Selection rule of the routing steps ("Kernmechanisme" item 2): higher score
// first, -0 equal to +0, NaN after every number, ties to the lower index;
// winners are reported in ascending index order, padded with -1.
#pragma once

#include "hga_common.cuh"

namespace hga {

// Order-preserving key of a candidate's score: a larger score gives a larger
// key; -0 and +0 give the same key; NaN gives 1 (below every number); 0 is
// reserved for "not a candidate".
__device__ __forceinline__ uint32_t score_key32(float s) {
    if (s != s) return 1u;
    s += 0.0f;
    const uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp: among keys[0..n) (0 = absent) keep the top k by (key desc,
// position asc) and write idx_of(x) of the winners in ascending position
// order to out[0..k_cap), padded with -1. hist: 256 words of shared memory
// private to this warp. Returns the number kept (in every lane).
template <typename IndexOf>
__device__ int warp_radix_topk(const uint32_t* keys, int n, int k, int k_cap, int32_t* out,
                               uint32_t* hist, IndexOf idx_of) {
    const int lane = threadIdx.x & 31;
    int n_cand = 0;
    for (int x0 = 0; x0 < n; x0 += 32) {
        const int x = x0 + lane;
        n_cand += __popc(__ballot_sync(0xffffffffu, x < n && keys[x] != 0u));
    }
    const int take = k < n_cand ? k : n_cand;
    uint32_t prefix = 0u, mask = 0u;
    int need = take;
    const bool all = take >= n_cand;
    if (!all) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int b = lane; b < 256; b += 32) hist[b] = 0u;
            __syncwarp();
            for (int x = lane; x < n; x += 32) {
                const uint32_t key = keys[x];
                if (key != 0u && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncwarp();
            // lane L owns digits 255-8L .. 248-8L (descending)
            uint32_t cnt[8];
            uint32_t lsum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = hist[255 - 8 * lane - i];
                lsum += cnt[i];
            }
            uint32_t incl = lsum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const uint32_t excl = incl - lsum;
            const bool here = excl < (uint32_t)need && (uint32_t)need <= incl;
            const unsigned hm = __ballot_sync(0xffffffffu, here);
            const int owner = hm ? __ffs(hm) - 1 : 0;
            uint32_t digit = 0u, above = 0u;
            if (lane == owner) {
                uint32_t run = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run + cnt[i] >= (uint32_t)need) {
                        digit = 255u - 8u * lane - i;
                        above = run;
                        break;
                    }
                    run += cnt[i];
                }
            }
            digit = __shfl_sync(0xffffffffu, digit, owner);
            above = __shfl_sync(0xffffffffu, above, owner);
            need -= (int)above;
            prefix |= digit << shift;
            mask |= 255u << shift;
            __syncwarp();
        }
    }
    // keys above the threshold are in; among keys equal to it the first
    // `need` positions are in
    int base = 0, ties = 0;
    for (int x0 = 0; x0 < n; x0 += 32) {
        const int x = x0 + lane;
        bool is = false, tie = false;
        if (x < n) {
            const uint32_t key = keys[x];
            if (key != 0u) {
                is = all || key > prefix;
                tie = !all && key == prefix;
            }
        }
        const unsigned tm = __ballot_sync(0xffffffffu, tie);
        is = is || (tie && ties + __popc(tm & ((1u << lane) - 1u)) < need);
        ties += __popc(tm);
        const unsigned m = __ballot_sync(0xffffffffu, is);
        if (is) out[base + __popc(m & ((1u << lane) - 1u))] = idx_of(x);
        base += __popc(m);
    }
    for (int s = base + lane; s < k_cap; s += 32) out[s] = -1;
    return base;
}

}  // namespace hga
