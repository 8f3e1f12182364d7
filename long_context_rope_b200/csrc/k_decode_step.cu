// k_decode_step.cu -- one decode step of hierarchical global attention in a
// single launch: q-bar, chunk routing, group routing and exact attention.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" items 2 and 4: the new token's query
// scores the chunk key summaries of all earlier chunks and keeps the top
// k_c; it scores the group summaries inside those chunks and keeps the top
// k_g groups; then it attends exactly (standard softmax) over the tokens of
// the selected groups and of the always-visible chunks (sinks, recent
// locals, current).
//
// One cluster of CL CTAs per (sequence, KV head). The always-visible blocks
// do not depend on routing, so the producer warp issues their TMA loads at
// the start and they land while routing runs. Routing needs one cluster
// exchange and no serial selection pass:
//   level 1  CTA r scores a contiguous slice of the candidate chunks and
//            ranks them locally (count of larger keys); its local top k_c
//            (the only ones that can be in the global top k_c) go, in
//            ascending chunk order, to every CTA's finalist table through
//            distributed shared memory; cluster barrier; every CTA ranks the
//            whole table (rank < k_c wins). Slices are contiguous, so the
//            table is in ascending chunk order and compacting the winners in
//            table order gives the sorted list without a sort.
//   level 2  every CTA scores all G groups of the selected chunks (at most
//            G x k_c rows, shared through L2) and ranks them exactly; the
//            candidates are already in ascending group order, so one warp
//            compacts the winners with ballots.
// Keys are 64-bit: the order-preserving 32-bit score key above, the index
// below (lower index wins a tie), 0 = not a candidate, so every rank is
// exact and unique. The scores are the same fp32 dot products, summed in the
// same order, as the separate routing kernels, so both paths select the same
// sets. Attention then runs as in the split-K decode kernel on CTA r's share
// of the forced blocks and of the routed blocks (hga_decode_core.cuh).
#include <cooperative_groups.h>

#include <mutex>

#include "hga_decode_core.cuh"
#include "hga_kernels.h"
#include "hga_tmap.h"
#include "hga_topk.cuh"

namespace cg = cooperative_groups;

namespace hga {

namespace {

using dec::kConsumers;
using dec::kD;
using dec::kMaxCluster;
using dec::kStagesMax;
using dec::kThreads;

constexpr int kMaxSlice = 512;   // level-1 candidates per CTA
constexpr int kMaxF1 = 512;      // level-1 finalist slots of the cluster
constexpr int kMaxCand2 = 512;   // level-2 candidates (G x k_c)
constexpr int kMaxKc = 64;
constexpr int kMaxKg = 512;
constexpr int kMaxLocal = 256;   // key blocks per CTA
constexpr int kRankThreads = kConsumers * 32;
constexpr int kL1Rows = 16;      // level-1 rows per consumer warp per batch

struct StepMaps {
    CUtensorMap k, v;
};

struct StepSmem {
    union {
        dec::Ring ring;
        dec::Partial warp_part[kConsumers];
    } u;
    dec::Owned owned;                            // partials of the heads this CTA finalises
    float wgt[kConsumers][8];                    // warp-merge weights
    uint16_t pt[kConsumers][8][16];
    uint64_t full[kStagesMax], empty[kStagesMax];
    alignas(16) uint64_t key1[kMaxSlice];     // own level-1 candidates
    uint64_t own1[kMaxKc];        // this CTA's level-1 finalists, ascending
    alignas(16) uint64_t f1[kMaxF1];          // level-1 finalists of all CTAs
    alignas(16) uint64_t key2[kMaxCand2];     // level-2 candidates (all of them, every CTA)
    int wcnt[2][kConsumers];      // rank_select's per-warp winner counts
    int win1[kMaxKc];             // selected chunks, ascending
    int routed[kMaxKg];           // selected groups, ascending
    int blk_pos[kMaxLocal];       // position of a local block's first key
    int blk_row[kMaxLocal];       // its first row in the resident store (TMA source)
    int n_win1, n_wl, bad;
};

__device__ __forceinline__ uint64_t rank_key(uint32_t key32, int idx) {
    return key32 ? ((uint64_t)key32 << 32) | (uint32_t)(0x7fffffff - idx) : 0ull;
}
__device__ __forceinline__ int index_of(uint64_t k) {
    return 0x7fffffff - (int)(uint32_t)(k & 0xffffffffu);
}

// Consumer threads (kRankThreads): the exact top k of the present keys
// a[0..na) (0 = absent, never selected, never counted) by rank = number of
// b[0..nb) larger; emit(pos, x) receives the winners (rank < k) with
// positions 0, 1, ... in candidate order, and the count is returned to every
// consumer thread. Two threads share a candidate and each streams every
// other pair of b through it with 16-byte loads (b 16-byte aligned); the two
// counts are summed with one shuffle. (Four candidates per thread over eight
// threads, with 8-byte loads, took twice as long.) The compaction is
// stable and parallel: a ballot per warp, the warps' counts through wcnt
// (2 x kConsumers ints, alternating per 128 candidates) and one named
// barrier of the consumer warps per 128 candidates.
constexpr int kRankTpc = 2;
constexpr int kRankBarrier = 1;  // named barrier id (0 is __syncthreads)
template <typename Emit>
__device__ __forceinline__ int rank_select(const uint64_t* a, int na, const uint64_t* b, int nb,
                                           int k, int (*wcnt)[kConsumers], Emit emit) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int sub = t & (kRankTpc - 1);
    const ulonglong2* b2 = reinterpret_cast<const ulonglong2*>(b);
    const int npairs = nb >> 1;
    int base = 0;
    for (int x0 = 0, it = 0; x0 < na; x0 += kRankThreads / kRankTpc, ++it) {
        const int x = x0 + t / kRankTpc;
        const uint64_t ax = x < na ? a[x] : 0ull;
        int c = 0;
#pragma unroll 8
        for (int yp = sub; yp < npairs; yp += kRankTpc) {
            const ulonglong2 by = b2[yp];
            c += (by.x > ax ? 1 : 0) + (by.y > ax ? 1 : 0);
        }
        if ((nb & 1) && sub == 0) c += b[nb - 1] > ax ? 1 : 0;
        c += __shfl_xor_sync(0xffffffffu, c, 1);
        const bool win = sub == 0 && x < na && ax != 0ull && c < k;
        const unsigned m = __ballot_sync(0xffffffffu, win);
        if (lane == 0) wcnt[it & 1][warp] = __popc(m);
        asm volatile("bar.sync %0, %1;" ::"n"(kRankBarrier), "n"(kRankThreads) : "memory");
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            const int cw = wcnt[it & 1][w];
            before += w < warp ? cw : 0;
            total += cw;
        }
        if (win) emit(base + before + __popc(m & ((1u << lane) - 1u)), x);
        base += total;
    }
    return base;
}

// Elements 4 * lane .. 4 * lane + 3 of a summary row as fp32 (fp32 or bf16
// tables; a bf16 value converts to fp32 exactly).
__device__ __forceinline__ float4 load4(const float* row, int lane) {
    return __ldg(reinterpret_cast<const float4*>(row) + lane);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* row, int lane) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(row) + lane);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Score rows [0, n) of a summary table for this warp's share and hand each
// (row, fp32 score) to emit. Same arithmetic and order as the routing kernels.
template <int kRowsInFlight, typename RowOf, typename Emit>
__device__ __forceinline__ void score_rows(const float* q, int n, RowOf row_of, Emit emit) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int x0 = warp * kRowsInFlight; x0 < n; x0 += kConsumers * kRowsInFlight) {
        float v[kRowsInFlight][4];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int x = x0 + u < n ? x0 + u : n - 1;
            const float4 t = load4(row_of(x), lane);
            v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
        }
        float sc[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) s = fmaf(q[e], v[u][e], s);
            sc[u] = warp_sum(s);
        }
        if (lane < kRowsInFlight) {
            float s = sc[0];
#pragma unroll
            for (int u = 1; u < kRowsInFlight; ++u)
                if (lane == u) s = sc[u];
            if (x0 + lane < n) emit(x0 + lane, s);
        }
    }
}

// Producer warp, host tier: the K and V rows of one routed group (16 rows of
// d = 128 elements each, contiguous in the full store) read over the host
// link with 16-byte loads (each lane 8 (bf16) or 4 (E4M3) of each tensor,
// 512 contiguous bytes per warp load) and stored into ring stage s in the
// layout the TMA tile loads write: 128-byte panels of 16 rows (two for bf16,
// one for E4M3), 16-byte chunk c of row r at c ^ (r % 8).
template <bool kF8>
__device__ __forceinline__ void copy_host_block(dec::Ring& ring, int s, const uint4* kh,
                                                const uint4* vh) {
    const int lane = threadIdx.x & 31;
    constexpr int kPieces = kF8 ? 4 : 8;             // per lane per tensor
    constexpr int kRowPieces = kF8 ? 8 : 16;         // 16-byte pieces per row
    uint4 kr[kPieces], vr[kPieces];
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
        kr[u] = kh[lane + 32 * u];
        vr[u] = vh[lane + 32 * u];
    }
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
        const int idx = lane + 32 * u;               // 16-byte piece of the block
        const int row = idx / kRowPieces, c16 = idx % kRowPieces;
        const int off = (c16 >> 3) * 2048 + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(dec::k_stage<kF8>(ring, s) + off) = kr[u];
        *reinterpret_cast<uint4*>(dec::v_stage<kF8>(ring, s) + off) = vr[u];
    }
    // a later tile load into this stage (async proxy) is ordered after these
    // stores
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// S: element type of the summary tables (float, or bf16 for bf16 tables).
// kF8: keys and values are E4M3 codes (else bf16).
// k_host / v_host: nullptr, or the full store [B, Hkv, L, d] in mapped host
// memory (the host tier); then the maps cover the resident windows of the
// forced chunks ([B, Hkv, W * C, d]) and the routed groups are read from the
// host by the producer warp.
template <typename S, bool kF8>
__global__ void __launch_bounds__(kThreads, 2) decode_step_kernel(
    const __grid_constant__ StepMaps maps, Params p, const __nv_bfloat16* __restrict__ q,
    const S* __restrict__ cs, const S* __restrict__ gs, float* __restrict__ qbar_out,
    int32_t* __restrict__ sel_c, int32_t* __restrict__ nsel_c, int32_t* __restrict__ sel_g,
    int32_t* __restrict__ nsel_g, __nv_bfloat16* __restrict__ out, int attend,
    const uint4* __restrict__ k_host, const uint4* __restrict__ v_host) {
    extern __shared__ uint8_t smem_raw[];
    StepSmem& sm = *reinterpret_cast<StepSmem*>(
        align_smem_1024(smem_raw));
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int64_t bh = blockIdx.y;  // routing unit: (sequence, KV head) or (sequence, query head)
    const int b = (int)(bh / p.Hu), h = (int)(bh % p.Hu);
    const int64_t kvh = (int64_t)b * p.Hkv + h / (p.Hu / p.Hkv);  // its K/V and summary row
    const int j = p.j0;
    const int64_t prob = bh;  // one query chunk per unit
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool consumer = warp < kConsumers;

    // ---- forced blocks: sinks, locals, current chunk (blocks starting < L)
    const int s_end = p.n_sink < j + 1 ? p.n_sink : j + 1;
    const int l_begin = j - p.n_local > s_end ? j - p.n_local : s_end;
    const int nf = s_end + (j + 1 - l_begin);
    const int cur_blocks = (p.L - j * p.C + kGroupRows - 1) / kGroupRows;
    const int n_fb = (nf - 1) * p.G + (cur_blocks < p.G ? cur_blocks : p.G);
    const int pf = (n_fb + CL - 1) / CL;
    const int f_lo = r * pf;
    int nf_loc = n_fb - f_lo < pf ? n_fb - f_lo : pf;
    nf_loc = nf_loc < 0 ? 0 : nf_loc;
    if (tid == 0) {
        sm.bad = 0;
        sm.n_win1 = 0;
        sm.n_wl = 0;
        for (int s = 0; s < kStagesMax; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        ptx::fence_mbar_init();
    }
    const bool host_tier = k_host != nullptr;
    for (int i = tid; i < nf_loc; i += blockDim.x) {
        const int fi = f_lo + i, w = fi / p.G, gm = fi % p.G;
        const int c = w < s_end ? w : l_begin + (w - s_end);
        sm.blk_pos[i] = c * p.C + kGroupRows * gm;
        // resident windows: forced chunk w of the list sits in slot w
        sm.blk_row[i] = host_tier ? w * p.C + kGroupRows * gm : sm.blk_pos[i];
    }
    __syncthreads();
    constexpr int kS = dec::ring_stages<kF8>();
    const int n_pre = nf_loc < kS ? nf_loc : kS;

    // ---- level-1 slice: the first batch of this warp's chunk-summary rows is
    // requested before q-bar, so the two memory latencies overlap
    const int per1 = (j + CL - 1) / CL;
    const int c_lo = r * per1;
    const int c_hi = c_lo + per1 < j ? c_lo + per1 : j;
    const int ns = c_hi > c_lo ? c_hi - c_lo : 0;
    const S* ctab = cs + kvh * (int64_t)p.nC * kD;
    float4 first[kL1Rows];
    if (consumer) {
#pragma unroll
        for (int u = 0; u < kL1Rows; ++u) {
            const int x = warp * kL1Rows + u;
            first[u] = x < ns ? load4(ctab + (int64_t)(c_lo + x) * kD, lane)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }

    // ---- q-bar of the new token over the KV head's gq query heads
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    {
        const int64_t row0 = ((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq) * kD;
        uint2 raw[8];
#pragma unroll
        for (int r2 = 0; r2 < 8; ++r2)
            raw[r2] = r2 < p.gq ? *reinterpret_cast<const uint2*>(q + row0 + (int64_t)r2 * kD + lane * 4)
                                : make_uint2(0u, 0u);
#pragma unroll
        for (int r2 = 0; r2 < 8; ++r2) {
            if (r2 < p.gq) {
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[r2]);
                const float2 lo = __bfloat1622float2(h2[0]), hi = __bfloat1622float2(h2[1]);
                qv[0] += lo.x;
                qv[1] += lo.y;
                qv[2] += hi.x;
                qv[3] += hi.y;
            }
        }
        const float inv_n = 1.0f / (float)p.gq;
#pragma unroll
        for (int e = 0; e < 4; ++e) qv[e] *= inv_n;
        if (qbar_out && r == 0 && warp == 0) {
#pragma unroll
            for (int e = 0; e < 4; ++e) qbar_out[prob * kD + lane * 4 + e] = qv[e];
        }
    }

    // ---- level 1: own slice of the candidate chunks [0, j)
    const int cap1 = p.kc < per1 ? p.kc : per1;
    if (consumer) {
        auto emit1 = [&](int x, float s) {
            const int c = c_lo + x;
            sm.key1[x] = is_forced(p, j, c) ? 0ull : rank_key(score_key32(s), c);
        };
        // the prefetched first batch (same dot products and order as score_rows)
        float sc[kL1Rows];
#pragma unroll
        for (int u = 0; u < kL1Rows; ++u) {
            float s = 0.f;
            s = fmaf(qv[0], first[u].x, s);
            s = fmaf(qv[1], first[u].y, s);
            s = fmaf(qv[2], first[u].z, s);
            s = fmaf(qv[3], first[u].w, s);
            sc[u] = warp_sum(s);
        }
        if (lane < kL1Rows) {
            float s = sc[0];
#pragma unroll
            for (int u = 1; u < kL1Rows; ++u)
                if (lane == u) s = sc[u];
            if (warp * kL1Rows + lane < ns) emit1(warp * kL1Rows + lane, s);
        }
        // rows beyond the first batch (slices longer than 8 x kL1Rows)
        const int rest0 = kConsumers * kL1Rows;
        if (ns > rest0)
            score_rows<kL1Rows>(qv, ns - rest0,
                                [&](int x) { return ctab + (int64_t)(c_lo + rest0 + x) * kD; },
                                [&](int x, float s) { emit1(rest0 + x, s); });
    }
    __syncthreads();
    // the forced blocks' loads are issued once the level-1 rows are in: they
    // are needed only after routing, and the chunk-summary reads above are
    // on the critical path
    if (attend && warp == kConsumers && lane == 0)
        for (int i = 0; i < n_pre; ++i)
            dec::issue_block<kF8>(sm.u.ring, sm.full, i, &maps.k, &maps.v, sm.blk_row[i], (int)kvh);
    // this CTA's winners, in candidate (= ascending chunk) order, padded
    // with 0 to cap1 entries. (Prefetching the winners' group rows into L2
    // here, with one bulk prefetch per winner, cost more in this phase than
    // it saved at level 2: +0.9 against -0.2 us; so did prefetching the
    // selected chunks' K/V rows after level 1: +4 us, the attention phase
    // being HBM-bound already.)
    if (consumer) {
        const int n1 = rank_select(sm.key1, ns, sm.key1, ns, cap1, sm.wcnt,
                                   [&](int pos, int x) { sm.own1[pos] = sm.key1[x]; });
        for (int x = n1 + tid; x < cap1; x += kRankThreads) sm.own1[x] = 0ull;
    }
    cluster.sync();
    // the finalist table: CTA t's winners at slots [t * cap1, (t + 1) * cap1),
    // read from its shared memory; ascending, as the slices are contiguous
    // and ordered by t
    for (int x = tid; x < CL * cap1; x += blockDim.x)
        sm.f1[x] = cluster.map_shared_rank(sm.own1, x / cap1)[x % cap1];
    __syncthreads();

    // ---- every CTA ranks the whole finalist table: the global top k_c,
    // compacted in table order, which is ascending chunk order
    const int nF1 = CL * cap1;
    if (consumer) {
        const int n = rank_select(sm.f1, nF1, sm.f1, nF1, p.kc, sm.wcnt,
                                  [&](int pos, int x) { sm.win1[pos] = index_of(sm.f1[x]); });
        if (tid == 0) sm.n_win1 = n;
    }
    __syncthreads();
    const int nsel1 = sm.n_win1;  // min(k_c, number of candidates)
    if (r == 0) {
        for (int i = tid; i < p.kc; i += blockDim.x) sel_c[prob * p.kc + i] = i < nsel1 ? sm.win1[i] : -1;
        if (tid == 0) nsel_c[prob] = nsel1;
    }

    // ---- level 2: every CTA scores all G groups of the selected chunks
    // (candidate x = group x % G of the (x / G)-th chunk: ascending group
    // index) and ranks them exactly; no second cluster exchange is needed
    const int n2 = nsel1 * p.G;
    const S* gtab = gs + kvh * (int64_t)p.nC * p.G * kD;
    if (consumer)
        score_rows<16>(qv, n2,
                       [&](int x) { return gtab + ((int64_t)sm.win1[x / p.G] * p.G + x % p.G) * kD; },
                       [&](int x, float s) {
                           sm.key2[x] = rank_key(score_key32(s), sm.win1[x / p.G] * p.G + x % p.G);
                       });
    __syncthreads();
    // winners (rank < k_g) in candidate order = ascending group index
    if (consumer) {
        const int n = rank_select(sm.key2, n2, sm.key2, n2, p.kg, sm.wcnt,
                                  [&](int pos, int x) { sm.routed[pos] = index_of(sm.key2[x]); });
        if (tid == 0) sm.n_wl = n;
    }
    __syncthreads();
    const int nw = sm.n_wl;
    if (r == 0) {
        for (int i = tid; i < p.kg; i += blockDim.x) sel_g[prob * p.kg + i] = i < nw ? sm.routed[i] : -1;
        if (tid == 0) nsel_g[prob] = nw;
    }
    if (!attend) {
        // peers read this CTA's finalist table (own1) after the first cluster
        // barrier; it stays valid until every CTA has passed this one
        cluster.sync();
        return;
    }

    // ---- attention over this CTA's forced share, then its routed share
    const int pr = (nw + CL - 1) / CL;
    const int r_lo = r * pr;
    int nr_loc = nw - r_lo < pr ? nw - r_lo : pr;
    nr_loc = nr_loc < 0 ? 0 : nr_loc;
    for (int i = tid; i < nr_loc; i += blockDim.x) {
        sm.blk_pos[nf_loc + i] = sm.routed[r_lo + i] * kGroupRows;
        sm.blk_row[nf_loc + i] = sm.routed[r_lo + i] * kGroupRows;
    }
    const int nloc = nf_loc + nr_loc;
    __syncthreads();
    if (warp == kConsumers) {
        // lane 0 waits for free stages and issues the tile loads of resident
        // blocks; a routed block of the host tier is copied by the whole warp
        // (its stage's barrier then completes on lane 0's plain arrival)
        int i = n_pre;
        bool ok = true;
        for (; i < nloc; ++i) {
            const int s = i % kS;
            if (i >= kS) {
                bool got = true;
                if (lane == 0)
                    got = ptx::mbar_wait_bounded(&sm.empty[s], ((i / kS) - 1) & 1, p.wait_ns);
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
            }
            if (host_tier && i >= nf_loc) {
                const int64_t row = kvh * (int64_t)p.L + sm.blk_row[i];
                constexpr int kRowVecs = kF8 ? kD / 16 : kD / 8;  // 16-byte pieces per row
                copy_host_block<kF8>(sm.u.ring, s, k_host + row * kRowVecs, v_host + row * kRowVecs);
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.full[s]);
            } else if (lane == 0) {
                dec::issue_block<kF8>(sm.u.ring, sm.full, s, &maps.k, &maps.v, sm.blk_row[i], (int)kvh);
            }
        }
        if (lane == 0) {
            if (!ok) {
                raise_timeout(p);
                sm.bad = 1;
            }
            // every issued load (the early forced blocks included) lands
            // before the ring's memory is reused
            if (!dec::drain_ring<kF8>(sm.full, i)) {
                raise_timeout(p);
                sm.bad = 1;
            }
        }
    }
    dec::WarpAcc acc;
    dec::acc_init(acc);
    if (consumer) {
        uint32_t qf[8][2];
        dec::load_q_frags<kF8>(p, q, b, h, qf);
        dec::consume_blocks<kF8>(p, qf, sm.u.ring, sm.full, sm.empty, sm.blk_pos, nloc, p.q_begin,
                            sm.pt[warp], acc, &sm.bad);
    }
    __syncthreads();
    if (consumer) dec::store_warp_partial<kF8>(acc, sm.u.warp_part[warp]);
    __syncthreads();
    dec::merge_warps_push(sm.u.warp_part, cluster, sm.owned, sm.wgt, p.gq);
    cluster.sync();  // every partial is in its owner's shared memory
    dec::merge_owned_and_store(p, (int)cluster.num_blocks(), (int)cluster.block_rank(), sm.owned, b,
                               h, out);
}

// Table sizes a cluster of cl CTAs needs; false if one is over its cap.
bool step_fits(const Params& p, int cl) {
    const int j = p.j0;
    const int per1 = (j + cl - 1) / cl;
    const int cap1 = p.kc < per1 ? p.kc : per1;
    const int n_fb_max = (p.n_sink + p.n_local + 1) * p.G;
    return per1 <= kMaxSlice && cl * cap1 <= kMaxF1 && cl * cap1 <= kMaxSlice &&
           p.G * p.kc <= kMaxCand2 &&
           (n_fb_max + cl - 1) / cl + (p.kg + cl - 1) / cl <= kMaxLocal;
}

std::mutex g_step_mu;
// per device, summary type and K/V type, 0 = not queried
int g_max_active[kMaxDevicesPerProcess][2][2][kMaxCluster + 1] = {};

template <typename S, bool kF8>
cudaError_t step_prepare(size_t smem) {
    cudaError_t e = set_func_attr_once((const void*)decode_step_kernel<S, kF8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = set_func_attr_once((const void*)decode_step_kernel<S, kF8>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

// Clusters of `cl` CTAs that can be resident at once on the current device
// (-1 if the query fails).
template <typename S, bool kF8>
int active_clusters(int cl, size_t smem) {
    int dev = 0;
    if (current_device_index(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(g_step_mu);
    int& slot = g_max_active[dev][sizeof(S) == 2 ? 1 : 0][kF8 ? 1 : 0][cl];
    if (slot == 0) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(cl, 1, 1);
        q.blockDim = dim3(kThreads);
        q.dynamicSmemBytes = smem;
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeClusterDimension;
        a[0].val.clusterDim.x = cl;
        a[0].val.clusterDim.y = 1;
        a[0].val.clusterDim.z = 1;
        q.attrs = a;
        q.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, decode_step_kernel<S, kF8>, &q) != cudaSuccess) {
            cudaGetLastError();
            n = -1;
        }
        slot = n;
    }
    return slot;
}

// Cluster size: two CTAs per SM over the whole grid if the tables fit and the
// clusters can all be resident at once; else the largest size that fits.
template <typename S, bool kF8>
int step_cluster(const Params& p, size_t smem) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int units = p.B * p.Hu;
    int cl = 2 * sms / units;
    cl = cl < 1 ? 1 : (cl > kMaxCluster ? kMaxCluster : cl);
    for (; cl >= 1; --cl) {
        if (!step_fits(p, cl)) continue;
        if (cl == 1) return 1;
        const int n = active_clusters<S, kF8>(cl, smem);
        if (n >= units || (n > 0 && cl <= 2)) return cl;
    }
    return 0;
}

}  // namespace

bool decode_step_supports(const Params& p) {
    if (!(p.dtype == HGA_BF16 && p.d == kD && p.q_len == 1 && p.gq <= 8 && p.L % kGroupRows == 0 &&
          p.kc <= kMaxKc && p.kg <= kMaxKg && p.nQC == 1))
        return false;
    for (int cl = 1; cl <= kMaxCluster; ++cl)
        if (step_fits(p, cl)) return true;
    return false;
}

namespace {

template <typename S, bool kF8>
cudaError_t launch_step(const Params& p, const void* q_rot, const S* chunk_sum,
                        const S* group_sum, const void* k_cache, const void* v_cache, float* qbar,
                        int32_t* sel_chunks, int32_t* n_sel_chunks, int32_t* sel_groups,
                        int32_t* n_sel_groups, void* out, const void* k_host, const void* v_host,
                        cudaStream_t st) {
    const bool attend = out != nullptr;
    StepMaps maps;
    if (attend) {
        const int64_t BH = (int64_t)p.B * p.Hkv;
        const int64_t rows = p.kv_layout == HGA_KV_WINDOWS
                                 ? (int64_t)(p.n_sink + p.n_local + 1) * p.C
                                 : (int64_t)p.L;
        const bool ok = kF8 ? make_rows_map_u8(&maps.k, k_cache, BH, rows, kD, kGroupRows) &&
                                  make_rows_map_u8(&maps.v, v_cache, BH, rows, kD, kGroupRows)
                            : make_rows_map(&maps.k, k_cache, BH, rows, kD, kGroupRows) &&
                                  make_rows_map(&maps.v, v_cache, BH, rows, kD, kGroupRows);
        if (!ok) return cudaErrorInvalidValue;
    } else {
        memset(&maps, 0, sizeof(maps));
    }
    const size_t smem = sizeof(StepSmem) + 1024;
    cudaError_t e = step_prepare<S, kF8>(smem);
    if (e != cudaSuccess) return e;
    const int cl = step_cluster<S, kF8>(p, smem);
    if (cl < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, (unsigned)(p.B * p.Hu), 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<S, kF8>, maps, p, (const __nv_bfloat16*)q_rot,
                              chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks, sel_groups,
                              n_sel_groups, (__nv_bfloat16*)out, attend ? 1 : 0,
                              (const uint4*)k_host, (const uint4*)v_host);
}

}  // namespace

cudaError_t launch_decode_step(const Params& p, const void* q_rot, const void* chunk_sum,
                               const void* group_sum, const void* k_cache, const void* v_cache,
                               float* qbar, int32_t* sel_chunks, int32_t* n_sel_chunks,
                               int32_t* sel_groups, int32_t* n_sel_groups, void* out,
                               cudaStream_t st, const void* k_host, const void* v_host) {
    using bf = __nv_bfloat16;
    const bf* cb = (const bf*)chunk_sum;
    const bf* gb = (const bf*)group_sum;
    const float* cf = (const float*)chunk_sum;
    const float* gf = (const float*)group_sum;
    if (p.sum_bf16 && p.kv_f8)
        return launch_step<bf, true>(p, q_rot, cb, gb, k_cache, v_cache, qbar, sel_chunks,
                                     n_sel_chunks, sel_groups, n_sel_groups, out, k_host, v_host, st);
    if (p.sum_bf16)
        return launch_step<bf, false>(p, q_rot, cb, gb, k_cache, v_cache, qbar, sel_chunks,
                                      n_sel_chunks, sel_groups, n_sel_groups, out, k_host, v_host, st);
    if (p.kv_f8)
        return launch_step<float, true>(p, q_rot, cf, gf, k_cache, v_cache, qbar, sel_chunks,
                                        n_sel_chunks, sel_groups, n_sel_groups, out, k_host, v_host,
                                        st);
    return launch_step<float, false>(p, q_rot, cf, gf, k_cache, v_cache, qbar, sel_chunks,
                                     n_sel_chunks, sel_groups, n_sel_groups, out, k_host, v_host, st);
}

}  // namespace hga
