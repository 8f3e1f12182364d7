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

// Fill blk_row / blk_pos for query chunk j (index jj within the span) and
// return the number of blocks. Forced chunks come first in ascending order,
// then the routed groups in list order. Blocks that start at or past L are
// dropped. Rows of the resident store: the token position (HGA_KV_FULL) or
// slot * C + 16 * gamma (HGA_KV_WINDOWS). Rows of the gathered buffer:
// kSrcGathered | 16 * slot. Run by one thread.
__device__ __forceinline__ int build_key_blocks(const Params& p, int j, const int32_t* list,
                                                int n_list, bool gathered, int* blk_row,
                                                int* blk_pos, int cap) {
    int forced[kMaxForced];
    const int nf = forced_chunks(p, j, forced);
    const bool windows = p.kv_layout == HGA_KV_WINDOWS;
    int nb = 0;
    for (int w = 0; w < nf; ++w) {
        const int c = forced[w];
        for (int gm = 0; gm < p.G; ++gm) {
            const int pos = c * p.C + kGroupRows * gm;
            if (pos >= p.L || nb >= cap) continue;
            blk_row[nb] = windows ? w * p.C + kGroupRows * gm : pos;
            blk_pos[nb] = pos;
            ++nb;
        }
    }
    if (n_list < 0 || n_list > p.kg) {
        raise_dev_error(p, kDevErrCount);
        n_list = n_list < 0 ? 0 : p.kg;
    }
    for (int s = 0; s < n_list; ++s) {
        const int gi = checked_group_entry(p, j, list, s);
        if (gi < 0 || nb >= cap) continue;
        const int pos = gi * kGroupRows;
        blk_row[nb] = gathered ? (kSrcGathered | (kGroupRows * s)) : pos;
        blk_pos[nb] = pos;
        ++nb;
    }
    return nb;
}

}  // namespace hga
