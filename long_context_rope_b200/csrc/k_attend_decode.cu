// k_attend_decode.cu -- single-token (decode) exact attention over the routed
// set: a streaming split-K kernel whose splits merge inside a thread-block
// cluster.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4: standard softmax over the bounded
// exact token set. Decode is HBM-bound: every key/value row of the set is
// read once, and the query heads of a KV head share each load (GQA).
//
// One cluster of CL CTAs per (sequence, KV head), CL chosen so the grid
// fills every SM with two CTAs at once. CTA r owns a contiguous share of the
// unit's 16-row key blocks and streams them through a shared-memory ring
// (8 stages, or 16 of E4M3 blocks) filled by TMA (tensor-map tile loads,
// 128-byte swizzle; one producer thread). Eight consumer warps take every 8th block: S^T[16 keys x 8 heads]
// = K_blk Q^T and O^T[128 dims x 8 heads] += V^T P^T on warp-level bf16 MMA
// (m16n8k16, fp32 accumulate) with a per-warp online softmax in fp32. The
// 8 x CL warp partials (max, sum, O) merge through distributed shared memory:
// CTA r finalises heads r, r + CL, ... With E4M3 keys and values
// (HGA_KV_E4M3) the blocks are 2 KiB per tensor and the products run on fp16
// MMA (hga_decode_core.cuh).
#include <cooperative_groups.h>

#include <mutex>

#include "hga_blocks.cuh"
#include "hga_decode_core.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"
#include "hga_tmap.h"

namespace cg = cooperative_groups;

namespace hga {

namespace {

using dec::kBlkBytes;
using dec::kConsumers;
using dec::kD;
using dec::kMaxCluster;
using dec::kStagesMax;
using dec::kThreads;

struct DecodeMaps {
    CUtensorMap k_res, v_res, k_gat, v_gat;
};

struct DecodeSmem {
    union {
        dec::Ring ring;
        dec::Partial warp_part[kConsumers];      // reused once the ring is drained
    } u;
    dec::Owned owned;                            // partials of the heads this CTA finalises
    float wgt[kConsumers][8];                    // warp-merge weights
    uint16_t pt[kConsumers][8][16];              // per-warp P transpose buffer
    uint64_t full[kStagesMax], empty[kStagesMax];
    int blk_row[kMaxBlocks];
    int blk_pos[kMaxBlocks];
    int nb;
    int bad;
};

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 2) attend_decode_kernel(
    const __grid_constant__ DecodeMaps maps, Params p, const __nv_bfloat16* __restrict__ q,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel,
    __nv_bfloat16* __restrict__ out, int gathered) {
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        align_smem_1024(smem_raw));
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int64_t bh = blockIdx.y;  // routing unit: (sequence, KV head) or (sequence, query head)
    const int b = (int)(bh / p.Hu), h = (int)(bh % p.Hu);
    const int64_t kvh = (int64_t)b * p.Hkv + h / (p.Hu / p.Hkv);  // its K/V row
    const int j = p.j0;
    const int64_t prob = bh * p.nQC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (warp == 0) {
        const int nb_w = build_key_blocks_warp(p, j, sel + prob * p.kg, nsel + prob, gathered != 0,
                                               sm.blk_row, sm.blk_pos);
        if (lane == 0) {
            sm.nb = nb_w;
            sm.bad = 0;
            for (int s = 0; s < kStagesMax; ++s) {
                ptx::mbar_init(&sm.full[s], 1);
                ptx::mbar_init(&sm.empty[s], 1);
            }
            ptx::fence_mbar_init();
        }
    }
    __syncthreads();
    const int nb = sm.nb;
    const int per = (nb + CL - 1) / CL;
    const int lo = r * per;
    int nloc = nb - lo < per ? nb - lo : per;
    nloc = nloc < 0 ? 0 : nloc;

    if (warp == kConsumers) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int i = 0;
            for (; i < nloc; ++i) {
                constexpr int kS = dec::ring_stages<kF8>();
                const int s = i % kS;
                if (i >= kS &&
                    !ptx::mbar_wait_bounded(&sm.empty[s], ((i / kS) - 1) & 1, p.wait_ns)) {
                    raise_timeout(p);
                    sm.bad = 1;
                    break;
                }
                const int rw = sm.blk_row[lo + i];
                const bool gat = (rw & kSrcGathered) != 0;
                const int row = rw & ~kSrcGathered;
                dec::issue_block<kF8>(sm.u.ring, sm.full, s, gat ? &maps.k_gat : &maps.k_res,
                                 gat ? &maps.v_gat : &maps.v_res, row, (int)(gat ? prob : kvh));
            }
            // every issued load lands before the ring's memory is reused
            if (!dec::drain_ring<kF8>(sm.full, i)) {
                raise_timeout(p);
                sm.bad = 1;
            }
        }
    }

    // ------------------------------------------------------------ consumers
    dec::WarpAcc acc;
    dec::acc_init(acc);
    if (warp < kConsumers) {
        uint32_t qf[8][2];
        dec::load_q_frags<kF8>(p, q, b, h, qf);
        dec::consume_blocks<kF8>(p, qf, sm.u.ring, sm.full, sm.empty, sm.blk_pos + lo, nloc,
                            p.q_begin, sm.pt[warp], acc, &sm.bad);
    }
    __syncthreads();  // ring drained: every stage a consumer used was waited for

    // ---- per-warp partials -> shared memory (the ring's space is reused)
    if (warp < kConsumers) dec::store_warp_partial<kF8>(acc, sm.u.warp_part[warp]);
    __syncthreads();
    dec::merge_warps_push(sm.u.warp_part, cluster, sm.owned, sm.wgt, p.gq);
    cluster.sync();  // every partial is in its owner's shared memory
    dec::merge_owned_and_store(p, (int)cluster.num_blocks(), (int)cluster.block_rank(), sm.owned, b,
                               h, out);
}

std::mutex g_decode_mu;
// per device and K/V type: clusters of each size resident at once (0 = not
// queried) and the largest cluster size that co-schedules
int g_dec_active[kMaxDevicesPerProcess][2][kMaxCluster + 1] = {};
int g_dec_max_cluster[kMaxDevicesPerProcess][2] = {};

// Cluster size: as many CTAs per (sequence, KV head) as keep every unit's
// cluster resident at once (one wave), per the occupancy query for clusters.
template <bool kF8>
int pick_cluster(const Params& p, size_t smem, int dev) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int units = p.B * p.Hu;
    int cl = 2 * sms / units;  // two CTAs per SM
    cl = cl < 1 ? 1 : (cl > kMaxCluster ? kMaxCluster : cl);
    std::lock_guard<std::mutex> lock(g_decode_mu);
    int* max_active = g_dec_active[dev][kF8 ? 1 : 0];
    for (; cl > 1; --cl) {
        if (max_active[cl] == 0) {
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
            if (cudaOccupancyMaxActiveClusters(&n, attend_decode_kernel<kF8>, &q) != cudaSuccess) {
                cudaGetLastError();
                n = -1;
            }
            max_active[cl] = n;
        }
        if (max_active[cl] >= units) break;
    }
    return cl;
}

}  // namespace

namespace {

template <bool kF8>
cudaError_t launch_decode_t(const Params& p, const void* q_rot, const KvSources& kv,
                            const int32_t* sel_groups, const int32_t* n_sel_groups, void* out,
                            cudaStream_t st) {
    DecodeMaps maps;
    const bool gathered = kv.k_gat != nullptr;
    const int64_t res_rows = p.kv_layout == HGA_KV_WINDOWS
                                 ? (int64_t)(p.n_sink + p.n_local + 1) * p.C
                                 : (int64_t)p.L;
    const int64_t BH = (int64_t)p.B * p.Hkv;
    auto rows_map = [](CUtensorMap* m, const void* base, int64_t outer, int64_t rows) {
        return kF8 ? make_rows_map_u8(m, base, outer, rows, kD, kGroupRows)
                   : make_rows_map(m, base, outer, rows, kD, kGroupRows);
    };
    bool ok = rows_map(&maps.k_res, kv.k_res, BH, res_rows) &&
              rows_map(&maps.v_res, kv.v_res, BH, res_rows);
    if (gathered) {
        ok = ok && rows_map(&maps.k_gat, kv.k_gat, BH * p.nQC, (int64_t)p.kg * kGroupRows) &&
             rows_map(&maps.v_gat, kv.v_gat, BH * p.nQC, (int64_t)p.kg * kGroupRows);
    } else {
        maps.k_gat = maps.k_res;
        maps.v_gat = maps.v_res;
    }
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(DecodeSmem) + 1024;
    int dev = 0;
    cudaError_t e = current_device_index(&dev);
    if (e != cudaSuccess) return e;
    e = set_func_attr_once((const void*)attend_decode_kernel<kF8>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = set_func_attr_once((const void*)attend_decode_kernel<kF8>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    int max_cluster = 0;
    {
        std::lock_guard<std::mutex> lock(g_decode_mu);
        int& mc_slot = g_dec_max_cluster[dev][kF8 ? 1 : 0];
        if (mc_slot <= 0) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(kMaxCluster, 1, 1);
            q.blockDim = dim3(kThreads);
            q.dynamicSmemBytes = smem;
            int mc = 0;
            if (cudaOccupancyMaxPotentialClusterSize(&mc, attend_decode_kernel<kF8>, &q) !=
                cudaSuccess) {
                cudaGetLastError();
                return cudaErrorInvalidConfiguration;
            }
            mc_slot = mc < 1 ? 1 : mc;
        }
        max_cluster = mc_slot;
    }
    int cl = pick_cluster<kF8>(p, smem, dev);
    if (cl > max_cluster) cl = max_cluster;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, (unsigned)((int64_t)p.B * p.Hu), 1);
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
    const int gflag = gathered ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, attend_decode_kernel<kF8>, maps, p,
                              (const __nv_bfloat16*)q_rot, sel_groups, n_sel_groups,
                              (__nv_bfloat16*)out, gflag);
}

}  // namespace

cudaError_t launch_attend_decode(const Params& p, const void* q_rot, const KvSources& kv,
                                 const int32_t* sel_groups, const int32_t* n_sel_groups,
                                 void* out, cudaStream_t st) {
    if (p.kv_f8)
        return launch_decode_t<true>(p, q_rot, kv, sel_groups, n_sel_groups, out, st);
    return launch_decode_t<false>(p, q_rot, kv, sel_groups, n_sel_groups, out, st);
}

bool decode_kernel_supports(const Params& p) {
    return p.dtype == HGA_BF16 && p.d == kD && p.q_len == 1 && p.gq <= 8 &&
           p.L % kGroupRows == 0;
}

}  // namespace hga
