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
// unit's 16-row key blocks and streams them through an 8-stage shared-memory ring
// filled by TMA (tensor-map tile loads, 128-byte swizzle; one producer
// thread). Eight consumer warps take every 8th block: S^T[16 keys x 8 heads]
// = K_blk Q^T and O^T[128 dims x 8 heads] += V^T P^T on warp-level bf16 MMA
// (m16n8k16, fp32 accumulate) with a per-warp online softmax in fp32. The
// 8 x CL warp partials (max, sum, O) merge through distributed shared memory:
// CTA r finalises heads r, r + CL, ...
#include <cooperative_groups.h>

#include "hga_blocks.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"
#include "hga_tmap.h"

namespace cg = cooperative_groups;

namespace hga {

namespace {

constexpr int kD = 128;
constexpr int kStages = 8;                       // ring of key blocks
constexpr int kBlkBytes = kGroupRows * kD * 2;   // 4 KiB per block per tensor
constexpr int kConsumers = 8;                    // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;  // + one producer warp
constexpr int kMaxCluster = 16;

struct DecodeMaps {
    CUtensorMap k_res, v_res, k_gat, v_gat;
};

struct Partial {
    float m[8], l[8];          // per head
    float o[8][kD];            // per head, un-normalised
};

struct DecodeSmem {
    union {
        struct {
            alignas(1024) uint8_t k[kStages][kBlkBytes];
            alignas(1024) uint8_t v[kStages][kBlkBytes];
        } ring;
        Partial warp_part[kConsumers];           // reused once the ring is drained
    } u;
    Partial cta_part;
    __nv_bfloat16 pt[kConsumers][8][16];         // per-warp P transpose buffer
    uint64_t full[kStages], empty[kStages];
    int blk_row[kMaxBlocks];
    int blk_pos[kMaxBlocks];
    int nb;
    int bad;
};

__global__ void __launch_bounds__(kThreads, 2) attend_decode_kernel(
    const __grid_constant__ DecodeMaps maps, Params p, const __nv_bfloat16* __restrict__ q,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ nsel,
    __nv_bfloat16* __restrict__ out, int gathered) {
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int64_t bh = blockIdx.y;
    const int b = (int)(bh / p.Hkv), h = (int)(bh % p.Hkv);
    const int j = p.j0;
    const int64_t prob = bh * p.nQC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int qpos = p.q_begin;

    if (warp == 0) {
        const int nb_w = build_key_blocks_warp(p, j, sel + prob * p.kg, nsel + prob, gathered != 0,
                                               sm.blk_row, sm.blk_pos);
        if (lane == 0) {
            sm.nb = nb_w;
            sm.bad = 0;
            for (int s = 0; s < kStages; ++s) {
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
            for (int i = 0; i < nloc; ++i) {
                const int s = i % kStages;
                if (i >= kStages &&
                    !ptx::mbar_wait_bounded(&sm.empty[s], ((i / kStages) - 1) & 1, p.err)) {
                    raise_dev_error(p, kDevErrTimeout);
                    sm.bad = 1;
                    break;
                }
                const int rw = sm.blk_row[lo + i];
                const bool gat = (rw & kSrcGathered) != 0;
                const int row = rw & ~kSrcGathered;
                const CUtensorMap* mk = gat ? &maps.k_gat : &maps.k_res;
                const CUtensorMap* mv = gat ? &maps.v_gat : &maps.v_res;
                const int outer = (int)(gat ? prob : bh);
                ptx::mbar_arrive_expect_tx(&sm.full[s], 2 * kBlkBytes);
                for (int hf = 0; hf < 2; ++hf) {
                    ptx::tma_load_3d(sm.u.ring.k[s] + hf * 2048, mk, hf * 64, row, outer, &sm.full[s]);
                    ptx::tma_load_3d(sm.u.ring.v[s] + hf * 2048, mv, hf * 64, row, outer, &sm.full[s]);
                }
            }
        }
    }

    // ------------------------------------------------------------ consumers
    float acc_o[8][4];
    float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc_o[mt][e] = 0.f;
    if (warp < kConsumers) {
        // Q^T as MMA B fragments: lane (g, t4) holds Q[head g][16kk + 2t4 .. +1]
        // and Q[head g][16kk + 2t4 + 8 .. +9]; heads >= gq are zero.
        uint32_t qf[8][2];
        {
            const bool okh = g < p.gq;
            const __nv_bfloat16* qr =
                q + ((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq + (okh ? g : 0)) * kD;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                qf[kk][0] = okh ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4) : 0u;
                qf[kk][1] = okh ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4 + 8) : 0u;
            }
        }
        const float sc = 1.4426950408889634f / sqrtf((float)kD);
        const int mq = lane >> 3;
        const int krow = (mq & 1) * 8 + (lane & 7);      // K ldmatrix row
        const int vkey = (mq >> 1) * 8 + (lane & 7);     // V ldmatrix (trans) row
        for (int i = warp; i < nloc; i += kConsumers) {
            const int s = i % kStages;
            const bool got = __all_sync(
                0xffffffffu, ptx::mbar_wait_bounded(&sm.full[s], (i / kStages) & 1, p.err));
            if (!got) {
                if (lane == 0) {
                    raise_dev_error(p, kDevErrTimeout);
                    sm.bad = 1;
                }
                break;
            }
            // S^T = K Q^T for 16 keys x 8 heads (two accumulator chains)
            float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sacc2[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t kb = ptx::smem_u32(sm.u.ring.k[s]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int chunk = (kk & 3) * 2 + (mq >> 1);
                uint32_t a[4];
                ptx::ldsm_x4(kb + (kk >> 2) * 2048 + krow * 128 + ((chunk ^ (krow & 7)) << 4), a);
                ptx::mma_16816((kk & 1) ? sacc2 : sacc, a, qf[kk][0], qf[kk][1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[e] += sacc2[e];
            // this lane holds keys g, g+8 for heads 2t4, 2t4+1
            const int kp = sm.blk_pos[lo + i];
            const bool v0 = kp + g <= qpos, v1 = kp + g + 8 <= qpos;
            const float sv[4] = {v0 ? sacc[0] * sc : -INFINITY, v0 ? sacc[1] * sc : -INFINITY,
                                 v1 ? sacc[2] * sc : -INFINITY, v1 ? sacc[3] * sc : -INFINITY};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float mb = fmaxf(sv[hh], sv[hh + 2]);
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 4));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
                const float mn = fmaxf(m_run[hh], mb);
                float alpha = 1.f, p0 = 0.f, p1 = 0.f;
                if (mn != -INFINITY) {
                    alpha = m_run[hh] == -INFINITY ? 0.f : ptx::ex2_approx(m_run[hh] - mn);
                    p0 = ptx::ex2_approx(sv[hh] - mn);
                    p1 = ptx::ex2_approx(sv[hh + 2] - mn);
                }
                m_run[hh] = mn;
                // bf16 weights; the running sum uses the same rounded values
                const __nv_bfloat16 b0 = __float2bfloat16_rn(p0);
                const __nv_bfloat16 b1 = __float2bfloat16_rn(p1);
                l_part[hh] = l_part[hh] * alpha + __bfloat162float(b0) + __bfloat162float(b1);
                sm.pt[warp][2 * t4 + hh][g] = b0;
                sm.pt[warp][2 * t4 + hh][g + 8] = b1;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    acc_o[mt][hh] *= alpha;
                    acc_o[mt][hh + 2] *= alpha;
                }
            }
            __syncwarp();
            const uint32_t pb0 = *reinterpret_cast<const uint32_t*>(&sm.pt[warp][g][2 * t4]);
            const uint32_t pb1 = *reinterpret_cast<const uint32_t*>(&sm.pt[warp][g][2 * t4 + 8]);
            // O^T[16 dims x 8 heads] += V^T P^T, eight 16-dim tiles
            const uint32_t vb = ptx::smem_u32(sm.u.ring.v[s]);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int chunk = (mt & 3) * 2 + (mq & 1);
                uint32_t a[4];
                ptx::ldsm_x4_trans(vb + (mt >> 2) * 2048 + vkey * 128 + ((chunk ^ (vkey & 7)) << 4),
                                   a);
                ptx::mma_16816(acc_o[mt], a, pb0, pb1);
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.empty[s]);
        }
    }
    __syncthreads();  // ring drained: every stage a consumer used was waited for

    // ---- per-warp partials -> shared memory (the ring's space is reused)
    if (warp < kConsumers) {
        Partial& wp = sm.u.warp_part[warp];
        float lsum[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float v = l_part[hh];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            lsum[hh] = v;
        }
        if (g == 0) {
            wp.m[2 * t4] = m_run[0];
            wp.m[2 * t4 + 1] = m_run[1];
            wp.l[2 * t4] = lsum[0];
            wp.l[2 * t4 + 1] = lsum[1];
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d0 = mt * 16 + g;
            wp.o[2 * t4][d0] = acc_o[mt][0];
            wp.o[2 * t4 + 1][d0] = acc_o[mt][1];
            wp.o[2 * t4][d0 + 8] = acc_o[mt][2];
            wp.o[2 * t4 + 1][d0 + 8] = acc_o[mt][3];
        }
    }
    __syncthreads();
    // ---- merge the 8 warps into this CTA's partial
    for (int x = tid; x < 8 * kD; x += blockDim.x) {
        const int n = x / kD, d = x % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sm.u.warp_part[w].m[n]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) {
                const float mw = sm.u.warp_part[w].m[n];
                if (mw == -INFINITY) continue;
                const float wgt = ptx::ex2_approx(mw - M);
                num = fmaf(wgt, sm.u.warp_part[w].o[n][d], num);
                den = fmaf(wgt, sm.u.warp_part[w].l[n], den);
            }
        }
        sm.cta_part.o[n][d] = num;
        if (d == 0) {
            sm.cta_part.m[n] = M;
            sm.cta_part.l[n] = den;
        }
    }
    cluster.sync();
    // ---- merge the CL CTA partials of head n in CTA n % CL
    for (int n = r; n < p.gq; n += CL) {
        if (tid < kD) {
            float mc[kMaxCluster], lc[kMaxCluster], oc[kMaxCluster];
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) {
                if (c < CL) {
                    const Partial* rp = cluster.map_shared_rank(&sm.cta_part, c);
                    mc[c] = rp->m[n];
                    lc[c] = rp->l[n];
                    oc[c] = rp->o[n][tid];
                } else {
                    mc[c] = -INFINITY;
                    lc[c] = 0.f;
                    oc[c] = 0.f;
                }
            }
            float M = -INFINITY;
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) M = fmaxf(M, mc[c]);
            float num = 0.f, den = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int c = 0; c < kMaxCluster; ++c) {
                    if (mc[c] == -INFINITY) continue;
                    const float wgt = ptx::ex2_approx(mc[c] - M);
                    num = fmaf(wgt, oc[c], num);
                    den = fmaf(wgt, lc[c], den);
                }
            }
            const float o = den > 0.f ? num / den : 0.f;
            out[((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq + n) * kD + tid] =
                __float2bfloat16_rn(o);
        }
    }
    cluster.sync();
}

// Cluster size: as many CTAs per (sequence, KV head) as keep every unit's
// cluster resident at once (one wave), per the occupancy query for clusters.
int pick_cluster(const Params& p, size_t smem) {
    static int max_active[kMaxCluster + 1] = {};
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int units = p.B * p.Hkv;
    int cl = 2 * sms / units;  // two CTAs per SM
    cl = cl < 1 ? 1 : (cl > kMaxCluster ? kMaxCluster : cl);
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
            if (cudaOccupancyMaxActiveClusters(&n, attend_decode_kernel, &q) != cudaSuccess) n = -1;
            max_active[cl] = n;
        }
        if (max_active[cl] >= units) break;
    }
    return cl;
}

}  // namespace

cudaError_t launch_attend_decode(const Params& p, const void* q_rot, const KvSources& kv,
                                 const int32_t* sel_groups, const int32_t* n_sel_groups,
                                 void* out, cudaStream_t st) {
    DecodeMaps maps;
    const bool gathered = kv.k_gat != nullptr;
    const int64_t res_rows = p.kv_layout == HGA_KV_WINDOWS
                                 ? (int64_t)(p.n_sink + p.n_local + 1) * p.C
                                 : (int64_t)p.L;
    const int64_t BH = (int64_t)p.B * p.Hkv;
    bool ok = make_rows_map(&maps.k_res, kv.k_res, BH, res_rows, kD, kGroupRows) &&
              make_rows_map(&maps.v_res, kv.v_res, BH, res_rows, kD, kGroupRows);
    if (gathered) {
        ok = ok && make_rows_map(&maps.k_gat, kv.k_gat, BH * p.nQC, (int64_t)p.kg * kGroupRows, kD,
                                 kGroupRows) &&
             make_rows_map(&maps.v_gat, kv.v_gat, BH * p.nQC, (int64_t)p.kg * kGroupRows, kD,
                           kGroupRows);
    } else {
        maps.k_gat = maps.k_res;
        maps.v_gat = maps.v_res;
    }
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(DecodeSmem) + 1024;
    static int max_cluster = -1;
    if (max_cluster < 0) {
        cudaError_t e = cudaFuncSetAttribute(attend_decode_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(attend_decode_kernel,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(kMaxCluster, 1, 1);
        q.blockDim = dim3(kThreads);
        q.dynamicSmemBytes = smem;
        int mc = 0;
        if (cudaOccupancyMaxPotentialClusterSize(&mc, attend_decode_kernel, &q) != cudaSuccess)
            return cudaErrorInvalidConfiguration;
        max_cluster = mc < 1 ? 1 : mc;
    }
    int cl = pick_cluster(p, smem);
    if (cl > max_cluster) cl = max_cluster;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, (unsigned)BH, 1);
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
    return cudaLaunchKernelEx(&cfg, attend_decode_kernel, maps, p, (const __nv_bfloat16*)q_rot,
                              sel_groups, n_sel_groups, (__nv_bfloat16*)out, gflag);
}

bool decode_kernel_supports(const Params& p) {
    return p.dtype == HGA_BF16 && p.d == kD && p.q_len == 1 && p.gq <= 8 &&
           p.L % kGroupRows == 0;
}

}  // namespace hga
