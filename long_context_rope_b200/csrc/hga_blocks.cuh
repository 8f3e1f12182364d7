// hga_blocks.cuh -- the bounded key set of one attention unit as 16-row blocks.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" items 2 and 4: the keys a query chunk j
// attends to are the tokens of its always-visible chunks (sinks, recent
// locals, current) and of the groups its router selected. Each group is
// 16 consecutive token rows, and every chunk is G such groups, so the set is
// a list of 16-row blocks. Each block records where its rows live (source
// and first row) and the position of its first token (for the causal rule).
#pragma once

#include "hga_common.cuh"

namespace hga {

constexpr int kSrcGathered = 1 << 30;  // flag in the row word: row is in the gathered buffer

// Validated group index of slot s of a selection list, or -1 (and the device
// error word is set). A valid entry lies in an earlier, non-forced chunk and
// is strictly above the previous entry.
__device__ __forceinline__ int checked_group_entry(const Params& p, int j, const int32_t* list,
                                                   int s) {
    const int gi = list[s];
    const int c = gi >= 0 ? gi / p.G : -1;
    const bool ok = gi >= 0 && c < j && !is_forced(p, j, c) && (s == 0 || gi > list[s - 1]);
    if (!ok) {
        raise_dev_error(p, kDevErrGroupIndex);
        return -1;
    }
    return gi;
}

// Fill blk_row / blk_pos for query chunk j and return the number of blocks
// (in every lane). Called by all 32 lanes of one warp. `list` holds the
// selection (top_k_groups slots) and `n_list_ptr` its count. Forced chunks
// come first in ascending order, then the routed groups in list order;
// blocks that start at or past L are dropped; invalid list entries are
// skipped (and recorded in the device error word). Rows of the resident
// store: the token position (HGA_KV_FULL) or slot * C + 16 * gamma
// (HGA_KV_WINDOWS). Rows of the gathered buffer: kSrcGathered | 16 * slot.
// The count and the first 128 list slots are loaded in one round trip. The
// caller guarantees the capacity (G * forced chunks + top_k_groups <= kMaxBlocks).
__device__ __forceinline__ int build_key_blocks_warp(const Params& p, int j, const int32_t* list,
                                                     const int32_t* n_list_ptr, bool gathered,
                                                     int* blk_row, int* blk_pos) {
    const int lane = threadIdx.x & 31;
    constexpr int kPre = 4;  // slots loaded ahead per lane (128 per warp)
    int n_list = n_list_ptr ? *n_list_ptr : 0;
    int pre[kPre];
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
        const int s = lane + 32 * u;
        pre[u] = (list != nullptr && s < p.kg) ? list[s] : -1;
    }
    const int s_end = p.n_sink < j + 1 ? p.n_sink : j + 1;
    const int l_begin = j - p.n_local > s_end ? j - p.n_local : s_end;
    const int nf = s_end + (j + 1 - l_begin);
    const bool windows = p.kv_layout == HGA_KV_WINDOWS;
    int nb = 0;
    for (int i0 = 0; i0 < nf * p.G; i0 += 32) {
        const int i = i0 + lane;
        int pos = 0, row = 0;
        bool ok = false;
        if (i < nf * p.G) {
            const int w = i / p.G, gm = i % p.G;
            const int c = w < s_end ? w : l_begin + (w - s_end);
            pos = c * p.C + kGroupRows * gm;
            row = windows ? w * p.C + kGroupRows * gm : pos;
            ok = pos < p.L;
        }
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const int at = nb + __popc(m & ((1u << lane) - 1u));
            blk_row[at] = row;
            blk_pos[at] = pos;
        }
        nb += __popc(m);
    }
    if (n_list < 0 || n_list > p.kg) {
        if (lane == 0) raise_dev_error(p, kDevErrCount);
        n_list = n_list < 0 ? 0 : p.kg;
    }
    int carry = -1;  // list[s0 - 1]
    for (int s0 = 0; s0 < n_list; s0 += 32) {
        const int s = s0 + lane;
        const int u = s0 >> 5;
        int gi = u < kPre ? pre[0] : -1;
#pragma unroll
        for (int v = 1; v < kPre; ++v)
            if (u == v) gi = pre[v];
        if (u >= kPre && s < n_list) gi = list[s];
        int prev = __shfl_up_sync(0xffffffffu, gi, 1);
        if (lane == 0) prev = carry;
        carry = __shfl_sync(0xffffffffu, gi, 31);
        if (s < n_list) {
            const int c = gi >= 0 ? gi / p.G : -1;
            const bool ok = gi >= 0 && c < j && !is_forced(p, j, c) && (s == 0 || gi > prev);
            if (!ok) {
                raise_dev_error(p, kDevErrGroupIndex);
                gi = -1;
            }
        } else {
            gi = -1;
        }
        const unsigned m = __ballot_sync(0xffffffffu, gi >= 0);
        if (gi >= 0) {
            const int at = nb + __popc(m & ((1u << lane) - 1u));
            const int pos = gi * kGroupRows;
            blk_row[at] = gathered ? (kSrcGathered | (kGroupRows * s)) : pos;
            blk_pos[at] = pos;
        }
        nb += __popc(m);
    }
    return nb;
}

}  // namespace hga
