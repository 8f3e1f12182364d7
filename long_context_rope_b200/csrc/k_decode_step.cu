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
// the start and they land while routing runs. Routing is split across the
// cluster and needs no serial selection pass:
//   level 1  CTA r scores a contiguous slice of the candidate chunks and
//            ranks them locally (count of larger keys); its local top k_c
//            (the only ones that can be in the global top k_c) go to every
//            CTA's finalist table through distributed shared memory;
//            cluster barrier; each CTA ranks its own finalists against the
//            table: rank < k_c is a winner.
//   level 2  each CTA scores the G groups of its own winning chunks, ranks
//            them locally, publishes its local top k_g; cluster barrier;
//            every CTA ranks the whole table and sorts the winners by
//            group index, so every CTA holds the routed list.
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
using dec::kStages;
using dec::kThreads;

constexpr int kMaxSlice = 512;   // level-1 candidates per CTA
constexpr int kMaxF1 = 512;      // level-1 finalist slots of the cluster
constexpr int kMaxCand2 = 512;   // level-2 candidates per CTA
constexpr int kMaxF2 = 1024;     // level-2 finalist slots of the cluster
constexpr int kMaxKc = 64;
constexpr int kMaxKg = 512;
constexpr int kMaxLocal = 256;   // key blocks per CTA
constexpr int kRowsInFlight = 8;
constexpr int kRankThreads = kConsumers * 32;

struct StepMaps {
    CUtensorMap k, v;
};

struct StepSmem {
    union {
        dec::Ring ring;
        dec::Partial warp_part[kConsumers];
    } u;
    dec::Partial cta_part;
    __nv_bfloat16 pt[kConsumers][8][16];
    uint64_t full[kStages], empty[kStages];
    uint64_t key1[kMaxSlice];     // own level-1 candidates
    uint64_t f1[kMaxF1];          // level-1 finalists of all CTAs
    uint64_t key2[kMaxCand2];     // own level-2 candidates
    uint64_t f2[kMaxF2];          // level-2 finalists of all CTAs
    int rank[kMaxF2];             // rank scratch
    int win1[kMaxKc];             // chunk winners by global rank (read in rank 0)
    int own_win[kMaxKc];          // this CTA's winning chunks
    int wl[kMaxKg];               // winning groups, unordered
    int routed[kMaxKg];           // winning groups, ascending
    int blk_pos[kMaxLocal];
    int n_own_win, n_wl, n_dense, bad;
};

__device__ __forceinline__ uint64_t rank_key(uint32_t key32, int idx) {
    return key32 ? ((uint64_t)key32 << 32) | (uint32_t)(0x7fffffff - idx) : 0ull;
}
__device__ __forceinline__ int index_of(uint64_t k) {
    return 0x7fffffff - (int)(uint32_t)(k & 0xffffffffu);
}

// Consumer threads (kRankThreads): rank[x] = number of b[0..nb) larger than
// a[x], for every present a[x] (0 = absent: not ranked, never counted).
__device__ __forceinline__ void count_greater(const uint64_t* a, int na, const uint64_t* b, int nb,
                                              int* rank) {
    const int t = threadIdx.x;
    int tpc = 1;
    while (tpc < 32 && na * tpc * 2 <= kRankThreads) tpc <<= 1;
    const int per_pass = kRankThreads / tpc;
    const int sub = t % tpc;
    for (int base = 0; base < na; base += per_pass) {
        const int x = base + t / tpc;
        const uint64_t ax = x < na ? a[x] : 0ull;
        int cnt = 0;
        if (ax != 0ull)
            for (int y = sub; y < nb; y += tpc) cnt += b[y] > ax ? 1 : 0;
        for (int off = 1; off < tpc; off <<= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
        if (sub == 0 && x < na && ax != 0ull) rank[x] = cnt;
    }
}

// Number of forced chunks (sinks, locals) below the current chunk j that
// fall in [lo, hi).
__device__ __forceinline__ int forced_below_in(const Params& p, int j, int lo, int hi) {
    const int s_hi = p.n_sink < j ? p.n_sink : j;
    const int s_end = p.n_sink < j + 1 ? p.n_sink : j + 1;
    const int l_lo = j - p.n_local > s_end ? j - p.n_local : s_end;
    auto overlap = [&](int a, int b) {
        const int x0 = a > lo ? a : lo, x1 = b < hi ? b : hi;
        return x1 > x0 ? x1 - x0 : 0;
    };
    return overlap(0, s_hi) + (l_lo < j ? overlap(l_lo, j) : 0);
}

// Score rows [0, n) of a summary table for this warp's share and hand each
// (row, fp32 score) to emit. Same arithmetic and order as the routing kernels.
template <typename RowOf, typename Emit>
__device__ __forceinline__ void score_rows(const float* q, int n, RowOf row_of, Emit emit) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int x0 = warp * kRowsInFlight; x0 < n; x0 += kConsumers * kRowsInFlight) {
        float v[kRowsInFlight][4];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int x = x0 + u < n ? x0 + u : n - 1;
            const float4 t = __ldg(reinterpret_cast<const float4*>(row_of(x)) + lane);
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

__global__ void __launch_bounds__(kThreads, 2) decode_step_kernel(
    const __grid_constant__ StepMaps maps, Params p, const __nv_bfloat16* __restrict__ q,
    const float* __restrict__ cs, const float* __restrict__ gs, float* __restrict__ qbar_out,
    int32_t* __restrict__ sel_c, int32_t* __restrict__ nsel_c, int32_t* __restrict__ sel_g,
    int32_t* __restrict__ nsel_g, __nv_bfloat16* __restrict__ out, int attend) {
    extern __shared__ uint8_t smem_raw[];
    StepSmem& sm = *reinterpret_cast<StepSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int64_t bh = blockIdx.y;
    const int b = (int)(bh / p.Hkv), h = (int)(bh % p.Hkv);
    const int j = p.j0;
    const int64_t prob = bh;  // one query chunk per (sequence, KV head)
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
        sm.n_own_win = 0;
        sm.n_wl = 0;
        sm.n_dense = 0;
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        ptx::fence_mbar_init();
    }
    for (int i = tid; i < nf_loc; i += blockDim.x) {
        const int fi = f_lo + i, w = fi / p.G, gm = fi % p.G;
        const int c = w < s_end ? w : l_begin + (w - s_end);
        sm.blk_pos[i] = c * p.C + kGroupRows * gm;
    }
    __syncthreads();
    const int n_pre = nf_loc < kStages ? nf_loc : kStages;
    if (attend && warp == kConsumers && lane == 0)
        for (int i = 0; i < n_pre; ++i)
            dec::issue_block(sm.u.ring, sm.full, i, &maps.k, &maps.v, sm.blk_pos[i], (int)bh);

    // ---- q-bar of the new token over the KV head's gq query heads
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    {
        const int64_t row0 = ((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq) * kD;
#pragma unroll 8
        for (int r2 = 0; r2 < p.gq; ++r2) {
            const __nv_bfloat16* qp = q + row0 + (int64_t)r2 * kD + lane * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) qv[e] += __bfloat162float(qp[e]);
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
    const int per1 = (j + CL - 1) / CL;
    const int c_lo = r * per1;
    const int c_hi = c_lo + per1 < j ? c_lo + per1 : j;
    const int ns = c_hi > c_lo ? c_hi - c_lo : 0;
    const int cap1 = p.kc < per1 ? p.kc : per1;
    const float* ctab = cs + bh * (int64_t)p.nC * kD;
    if (consumer)
        score_rows(qv, ns, [&](int x) { return ctab + (int64_t)(c_lo + x) * kD; },
                   [&](int x, float s) {
                       const int c = c_lo + x;
                       sm.key1[x] = is_forced(p, j, c) ? 0ull : rank_key(score_key32(s), c);
                   });
    __syncthreads();
    if (consumer) count_greater(sm.key1, ns, sm.key1, ns, sm.rank);
    __syncthreads();
    {
        const int present = ns - forced_below_in(p, j, c_lo, c_hi);
        const int filled = present < cap1 ? present : cap1;
        for (int x = tid; x < ns; x += blockDim.x) {
            const uint64_t k = sm.key1[x];
            if (k != 0ull && sm.rank[x] < cap1)
                for (int t = 0; t < CL; ++t)
                    cluster.map_shared_rank(sm.f1, t)[r * cap1 + sm.rank[x]] = k;
        }
        for (int x = filled + tid; x < cap1; x += blockDim.x)
            for (int t = 0; t < CL; ++t) cluster.map_shared_rank(sm.f1, t)[r * cap1 + x] = 0ull;
    }
    cluster.sync();

    // own finalists against all finalists: the global top k_c
    const int nF1 = CL * cap1;
    if (consumer) count_greater(sm.f1 + r * cap1, cap1, sm.f1, nF1, sm.rank);
    __syncthreads();
    {
        int* win1_0 = cluster.map_shared_rank(sm.win1, 0);
        for (int x = tid; x < cap1; x += blockDim.x) {
            const uint64_t k = sm.f1[r * cap1 + x];
            if (k != 0ull && sm.rank[x] < p.kc) {
                const int c = index_of(k);
                win1_0[sm.rank[x]] = c;
                sm.own_win[atomicAdd(&sm.n_own_win, 1)] = c;
            }
        }
    }
    __syncthreads();

    // ---- level 2: the G groups of this CTA's winning chunks
    const int n2 = sm.n_own_win * p.G;
    const int cap2_raw = p.G * (p.kc < cap1 ? p.kc : cap1);
    const int cap2 = p.kg < cap2_raw ? p.kg : cap2_raw;
    const float* gtab = gs + bh * (int64_t)p.nC * p.G * kD;
    if (consumer)
        score_rows(qv, n2,
                   [&](int x) {
                       return gtab + ((int64_t)sm.own_win[x / p.G] * p.G + x % p.G) * kD;
                   },
                   [&](int x, float s) {
                       sm.key2[x] = rank_key(score_key32(s), sm.own_win[x / p.G] * p.G + x % p.G);
                   });
    __syncthreads();
    if (consumer) count_greater(sm.key2, n2, sm.key2, n2, sm.rank);
    __syncthreads();
    {
        const int filled = n2 < cap2 ? n2 : cap2;
        for (int x = tid; x < n2; x += blockDim.x)
            if (sm.rank[x] < cap2)
                for (int t = 0; t < CL; ++t)
                    cluster.map_shared_rank(sm.f2, t)[r * cap2 + sm.rank[x]] = sm.key2[x];
        for (int x = filled + tid; x < cap2; x += blockDim.x)
            for (int t = 0; t < CL; ++t) cluster.map_shared_rank(sm.f2, t)[r * cap2 + x] = 0ull;
    }
    cluster.sync();

    // ---- selections
    const int n_cand1 = j - forced_below_in(p, j, 0, j);
    const int nsel1 = p.kc < n_cand1 ? p.kc : n_cand1;
    if (r == 0 && warp == 0) {
        int32_t* so = sel_c + prob * p.kc;
        for (int i = lane; i < p.kc; i += 32) {
            if (i < nsel1) {
                const int c = sm.win1[i];
                int pos = 0;
                for (int t = 0; t < nsel1; ++t) pos += sm.win1[t] < c ? 1 : 0;
                so[pos] = c;
            }
            if (i >= nsel1) so[i] = -1;
        }
        if (lane == 0) nsel_c[prob] = nsel1;
    }
    // the table's present entries (at most G * k_c) are packed into key2,
    // then ranked among themselves
    const int nF2 = CL * cap2;
    for (int x = tid; x < nF2; x += blockDim.x)
        if (sm.f2[x] != 0ull) sm.key2[atomicAdd(&sm.n_dense, 1)] = sm.f2[x];
    __syncthreads();
    const int n_dense = sm.n_dense;
    if (consumer) count_greater(sm.key2, n_dense, sm.key2, n_dense, sm.rank);
    __syncthreads();
    for (int x = tid; x < n_dense; x += blockDim.x)
        if (sm.rank[x] < p.kg) sm.wl[atomicAdd(&sm.n_wl, 1)] = index_of(sm.key2[x]);
    __syncthreads();
    const int nw = sm.n_wl;
    for (int i = tid; i < nw; i += blockDim.x) {
        const int gi = sm.wl[i];
        int pos = 0;
        for (int t = 0; t < nw; ++t) pos += sm.wl[t] < gi ? 1 : 0;
        sm.routed[pos] = gi;
    }
    __syncthreads();
    if (r == 0) {
        for (int i = tid; i < p.kg; i += blockDim.x) sel_g[prob * p.kg + i] = i < nw ? sm.routed[i] : -1;
        if (tid == 0) nsel_g[prob] = nw;
    }
    if (!attend) return;  // no distributed shared memory access is pending

    // ---- attention over this CTA's forced share, then its routed share
    const int pr = (nw + CL - 1) / CL;
    const int r_lo = r * pr;
    int nr_loc = nw - r_lo < pr ? nw - r_lo : pr;
    nr_loc = nr_loc < 0 ? 0 : nr_loc;
    for (int i = tid; i < nr_loc; i += blockDim.x)
        sm.blk_pos[nf_loc + i] = sm.routed[r_lo + i] * kGroupRows;
    const int nloc = nf_loc + nr_loc;
    __syncthreads();
    if (warp == kConsumers) {
        if (lane == 0) {
            for (int i = n_pre; i < nloc; ++i) {
                const int s = i % kStages;
                if (i >= kStages &&
                    !ptx::mbar_wait_bounded(&sm.empty[s], ((i / kStages) - 1) & 1, p.err)) {
                    raise_dev_error(p, kDevErrTimeout);
                    sm.bad = 1;
                    break;
                }
                dec::issue_block(sm.u.ring, sm.full, s, &maps.k, &maps.v, sm.blk_pos[i], (int)bh);
            }
        }
    }
    dec::WarpAcc acc;
    dec::acc_init(acc);
    if (consumer) {
        uint32_t qf[8][2];
        dec::load_q_frags(p, q, b, h, qf);
        dec::consume_blocks(p, qf, sm.u.ring, sm.full, sm.empty, sm.blk_pos, nloc, p.q_begin,
                            sm.pt[warp], acc, &sm.bad);
    }
    __syncthreads();
    if (consumer) dec::store_warp_partial(acc, sm.u.warp_part[warp]);
    __syncthreads();
    dec::merge_warps(sm.u.warp_part, sm.cta_part);
    cluster.sync();
    dec::merge_cluster_and_store(p, cluster, sm.cta_part, b, h, out);
    cluster.sync();
}

// Table sizes a cluster of cl CTAs needs; false if one is over its cap.
bool step_fits(const Params& p, int cl) {
    const int j = p.j0;
    const int per1 = (j + cl - 1) / cl;
    const int cap1 = p.kc < per1 ? p.kc : per1;
    const int cap2_raw = p.G * (p.kc < cap1 ? p.kc : cap1);
    const int cap2 = p.kg < cap2_raw ? p.kg : cap2_raw;
    const int n_fb_max = (p.n_sink + p.n_local + 1) * p.G;
    return per1 <= kMaxSlice && cl * cap1 <= kMaxF1 && cap2_raw <= kMaxCand2 &&
           cl * cap2 <= kMaxF2 && (n_fb_max + cl - 1) / cl + (p.kg + cl - 1) / cl <= kMaxLocal;
}

std::mutex g_step_mu;
int g_max_active[kMaxCluster + 1] = {};
bool g_attr_done = false;

cudaError_t step_prepare(size_t smem) {
    std::lock_guard<std::mutex> lock(g_step_mu);
    if (g_attr_done) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(decode_step_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_step_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                 1);
    if (e == cudaSuccess) g_attr_done = true;
    return e;
}

int active_clusters(int cl, size_t smem) {
    std::lock_guard<std::mutex> lock(g_step_mu);
    if (g_max_active[cl] == 0) {
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
        if (cudaOccupancyMaxActiveClusters(&n, decode_step_kernel, &q) != cudaSuccess) {
            cudaGetLastError();
            n = -1;
        }
        g_max_active[cl] = n;
    }
    return g_max_active[cl];
}

// Cluster size: two CTAs per SM over the whole grid if the tables fit and the
// clusters can all be resident at once; else the largest size that fits.
int step_cluster(const Params& p, size_t smem) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int units = p.B * p.Hkv;
    int cl = 2 * sms / units;
    cl = cl < 1 ? 1 : (cl > kMaxCluster ? kMaxCluster : cl);
    for (; cl >= 1; --cl) {
        if (!step_fits(p, cl)) continue;
        if (cl == 1) return 1;
        const int n = active_clusters(cl, smem);
        if (n >= units || (n > 0 && cl <= 2)) return cl;
    }
    return 0;
}

}  // namespace

bool decode_step_supports(const Params& p) {
    if (!(p.dtype == HGA_BF16 && p.d == kD && p.q_len == 1 && p.gq <= 8 && p.L % kGroupRows == 0 &&
          p.kv_layout == HGA_KV_FULL && p.kc <= kMaxKc && p.kg <= kMaxKg && p.nQC == 1))
        return false;
    for (int cl = 1; cl <= kMaxCluster; ++cl)
        if (step_fits(p, cl)) return true;
    return false;
}

cudaError_t launch_decode_step(const Params& p, const void* q_rot, const float* chunk_sum,
                               const float* group_sum, const void* k_cache, const void* v_cache,
                               float* qbar, int32_t* sel_chunks, int32_t* n_sel_chunks,
                               int32_t* sel_groups, int32_t* n_sel_groups, void* out,
                               cudaStream_t st) {
    const bool attend = out != nullptr;
    StepMaps maps;
    if (attend) {
        const int64_t BH = (int64_t)p.B * p.Hkv;
        if (!make_rows_map(&maps.k, k_cache, BH, p.L, kD, kGroupRows) ||
            !make_rows_map(&maps.v, v_cache, BH, p.L, kD, kGroupRows))
            return cudaErrorInvalidValue;
    } else {
        memset(&maps, 0, sizeof(maps));
    }
    const size_t smem = sizeof(StepSmem) + 1024;
    cudaError_t e = step_prepare(smem);
    if (e != cudaSuccess) return e;
    const int cl = step_cluster(p, smem);
    if (cl < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, (unsigned)(p.B * p.Hkv), 1);
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
    return cudaLaunchKernelEx(&cfg, decode_step_kernel, maps, p, (const __nv_bfloat16*)q_rot,
                              chunk_sum, group_sum, qbar, sel_chunks, n_sel_chunks, sel_groups,
                              n_sel_groups, (__nv_bfloat16*)out, attend ? 1 : 0);
}

}  // namespace hga
