// k_attend_decode.cu -- single-token (decode) exact attention over the routed
// set, split across a thread-block cluster.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4: standard softmax over the bounded
// exact token set. Decode is HBM-bound: every key/value row of the set is
// read once, and the 8 query heads of a KV head share each load (GQA).
//
// One cluster of CL CTAs per (sequence, KV head); CTA r owns a contiguous
// share of at most kMaxLoc 16-row key blocks. Each block's K and V arrive by
// TMA (tensor-map tile loads, 128-byte swizzle, one mbarrier for K and one
// for V). Scores S^T[16 keys x 8 heads] = K_blk Q^T and the output
// O^T[16 dims x 8 heads] += V^T P^T run on warp-level bf16 MMA (m16n8k16,
// fp32 accumulate) so the CUDA cores stay out of the critical path; the
// softmax between them is fp32. The CTAs' partial (max, sum, O) triples are
// merged through distributed shared memory: CTA r finalises heads r, r+CL...
#include <cooperative_groups.h>

#include "hga_blocks.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"
#include "hga_tmap.h"

namespace cg = cooperative_groups;

namespace hga {

namespace {

constexpr int kD = 128;
constexpr int kMaxLoc = 8;                 // key blocks per CTA
constexpr int kMaxCluster = 16;            // CTAs per (sequence, KV head)
constexpr int kBlkBytes = kGroupRows * kD * 2;  // 4 KiB per block per tensor
constexpr int kSP = kMaxLoc * 16 + 4;      // fp32 score row pitch
constexpr int kPP = kMaxLoc * 16 + 8;      // bf16 probability row pitch (conflict-free)

struct DecodeMaps {
    CUtensorMap k_res, v_res, k_gat, v_gat;
};

struct DecodeSmem {
    alignas(1024) uint8_t kbuf[kMaxLoc * kBlkBytes];
    alignas(1024) uint8_t vbuf[kMaxLoc * kBlkBytes];
    float s[8][kSP];
    __nv_bfloat16 pb[8][kPP];
    float opart[8][kD];
    float m[8], l[8];
    int blk_row[kMaxBlocks];
    int blk_pos[kMaxBlocks];
    int nb;
    int bad;
    uint64_t bar_k, bar_v;
};

__global__ void __launch_bounds__(256) attend_decode_kernel(const __grid_constant__ DecodeMaps maps,
                                                            Params p, const __nv_bfloat16* __restrict__ q,
                                                            const int32_t* __restrict__ sel,
                                                            const int32_t* __restrict__ nsel,
                                                            __nv_bfloat16* __restrict__ out,
                                                            int gathered) {
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
        const int nb_w = build_key_blocks_warp(p, j, sel + prob * p.kg, nsel[prob], gathered != 0,
                                               sm.blk_row, sm.blk_pos);
        if (lane == 0) sm.nb = nb_w;
    }
    if (tid == 0) {
        sm.bad = 0;
        ptx::mbar_init(&sm.bar_k, 1);
        ptx::mbar_init(&sm.bar_v, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    const int nb = sm.nb;
    const int per = (nb + CL - 1) / CL;
    const int lo = r * per;
    int nloc = nb - lo < per ? nb - lo : per;
    nloc = nloc < 0 ? 0 : (nloc > kMaxLoc ? kMaxLoc : nloc);

    if (tid == 0 && nloc > 0) {
        ptx::mbar_arrive_expect_tx(&sm.bar_k, (uint32_t)(nloc * kBlkBytes));
        ptx::mbar_arrive_expect_tx(&sm.bar_v, (uint32_t)(nloc * kBlkBytes));
        for (int i = 0; i < nloc; ++i) {
            const int rw = sm.blk_row[lo + i];
            const bool gat = (rw & kSrcGathered) != 0;
            const int row = rw & ~kSrcGathered;
            const CUtensorMap* mk = gat ? &maps.k_gat : &maps.k_res;
            const CUtensorMap* mv = gat ? &maps.v_gat : &maps.v_res;
            const int outer = (int)(gat ? prob : bh);
            for (int hf = 0; hf < 2; ++hf) {
                ptx::tma_load_3d(sm.kbuf + i * kBlkBytes + hf * 2048, mk, hf * 64, row, outer,
                                 &sm.bar_k);
                ptx::tma_load_3d(sm.vbuf + i * kBlkBytes + hf * 2048, mv, hf * 64, row, outer,
                                 &sm.bar_v);
            }
        }
    }

    // Q^T as MMA B fragments: lane (g, t4) holds Q[head g][16kk + 2t4 .. +1]
    // and Q[head g][16kk + 2t4 + 8 .. +9]; heads >= gq are zero.
    uint32_t qf[8][2];
    {
        const bool ok = g < p.gq;
        const __nv_bfloat16* qr =
            q + (((int64_t)b * p.q_len + 0) * p.Hq + (int64_t)h * p.gq + (ok ? g : 0)) * kD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4) : 0u;
            qf[kk][1] = ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4 + 8) : 0u;
        }
    }
    const float scale = 1.4426950408889634f / sqrtf((float)kD);

    if (nloc > 0 && tid == 0 && !ptx::mbar_wait_bounded(&sm.bar_k, 0, p.err)) {
        raise_dev_error(p, kDevErrTimeout);
        sm.bad = 1;
    }
    __syncthreads();
    if (nloc > 0 && !sm.bad) {
        // ---- scores: warp w handles local block w
        if (warp < nloc) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t kb = ptx::smem_u32(sm.kbuf + warp * kBlkBytes);
            const int mq = lane >> 3;
            const int row = (mq & 1) * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int chunk = (kk & 3) * 2 + (mq >> 1);
                const uint32_t addr = kb + (kk >> 2) * 2048 + row * 128 + ((chunk ^ (row & 7)) << 4);
                uint32_t a[4];
                ptx::ldsm_x4(addr, a);
                ptx::mma_16816(acc, a, qf[kk][0], qf[kk][1]);
            }
            const int kp = sm.blk_pos[lo + warp];
            const int x0 = warp * 16 + g;
            const bool v0 = kp + g <= qpos, v1 = kp + g + 8 <= qpos;
            sm.s[2 * t4][x0] = v0 ? acc[0] * scale : -INFINITY;
            sm.s[2 * t4 + 1][x0] = v0 ? acc[1] * scale : -INFINITY;
            sm.s[2 * t4][x0 + 8] = v1 ? acc[2] * scale : -INFINITY;
            sm.s[2 * t4 + 1][x0 + 8] = v1 ? acc[3] * scale : -INFINITY;
        }
        __syncthreads();
        // ---- softmax of each head over the local keys (warp n = head n)
        {
            const int n = warp;
            const int nk = nloc * 16;
            float mx = -INFINITY;
            for (int x = lane; x < nk; x += 32) mx = fmaxf(mx, n < p.gq ? sm.s[n][x] : -INFINITY);
            mx = warp_max(mx);
            float sum = 0.f;
            for (int x = lane; x < nk; x += 32) {
                float pv = 0.f;
                if (n < p.gq && mx != -INFINITY) pv = exp2f(sm.s[n][x] - mx);
                const __nv_bfloat16 pbv = __float2bfloat16_rn(pv);
                sm.pb[n][x] = pbv;
                sum += __bfloat162float(pbv);  // normalise by the rounded weights used below
            }
            sum = warp_sum(sum);
            if (lane == 0) {
                sm.m[n] = mx;
                sm.l[n] = sum;
            }
        }
    } else if (tid < 8) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.f;
    }
    if (nloc > 0 && tid == 0 && !sm.bad && !ptx::mbar_wait_bounded(&sm.bar_v, 0, p.err)) {
        raise_dev_error(p, kDevErrTimeout);
        sm.bad = 1;
    }
    __syncthreads();
    // ---- O^T tile of 16 dims per warp, accumulated over the local blocks
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (nloc > 0 && !sm.bad) {
            const int mq = lane >> 3;
            const int key = (mq >> 1) * 8 + (lane & 7);
            const int chunk = (warp & 3) * 2 + (mq & 1);
            const uint32_t voff = (warp >> 2) * 2048 + key * 128 + ((chunk ^ (key & 7)) << 4);
            for (int i = 0; i < nloc; ++i) {
                uint32_t a[4];
                ptx::ldsm_x4_trans(ptx::smem_u32(sm.vbuf + i * kBlkBytes) + voff, a);
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&sm.pb[g][i * 16 + 2 * t4]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&sm.pb[g][i * 16 + 2 * t4 + 8]);
                ptx::mma_16816(acc, a, b0, b1);
            }
        }
        const int d0 = warp * 16 + g;
        sm.opart[2 * t4][d0] = acc[0];
        sm.opart[2 * t4 + 1][d0] = acc[1];
        sm.opart[2 * t4][d0 + 8] = acc[2];
        sm.opart[2 * t4 + 1][d0 + 8] = acc[3];
    }
    cluster.sync();
    // ---- merge the CL partials of head n in CTA n % CL
    for (int n = r; n < p.gq; n += CL) {
        if (tid < kD) {
            // issue every remote (distributed shared memory) load first, then combine
            float mc[kMaxCluster], lc[kMaxCluster], oc[kMaxCluster];
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) {
                if (c < CL) {
                    const DecodeSmem* rs = cluster.map_shared_rank(&sm, c);
                    mc[c] = rs->m[n];
                    lc[c] = rs->l[n];
                    oc[c] = rs->opart[n][tid];
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
                    const float wgt = exp2f(mc[c] - M);
                    num = fmaf(wgt, oc[c], num);
                    den = fmaf(wgt, lc[c], den);
                }
            }
            const float o = den > 0.f ? num / den : 0.f;
            out[(((int64_t)b * p.q_len + 0) * p.Hq + (int64_t)h * p.gq + n) * kD + tid] =
                __float2bfloat16_rn(o);
        }
    }
    cluster.sync();
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
    const int nb_max = p.G * (p.n_sink + p.n_local + 1) + p.kg;
    int cl = (nb_max + kMaxLoc - 1) / kMaxLoc;
    cl = cl < 1 ? 1 : cl;
    const size_t smem = sizeof(DecodeSmem) + 1024;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(attend_decode_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(attend_decode_kernel,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    static int max_cluster = -1;
    cudaLaunchConfig_t cfg = {};
    if (max_cluster < 0) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(16, 1, 1);
        q.blockDim = dim3(256);
        q.dynamicSmemBytes = smem;
        int mc = 0;
        if (cudaOccupancyMaxPotentialClusterSize(&mc, attend_decode_kernel, &q) != cudaSuccess)
            return cudaErrorInvalidConfiguration;
        max_cluster = mc;
    }
    if (cl > max_cluster) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3(cl, (unsigned)BH, 1);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int g = gathered ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, attend_decode_kernel, maps, p,
                              (const __nv_bfloat16*)q_rot, sel_groups, n_sel_groups,
                              (__nv_bfloat16*)out, g);
}

bool decode_kernel_supports(const Params& p) {
    const int nb_max = p.G * (p.n_sink + p.n_local + 1) + p.kg;
    return p.dtype == HGA_BF16 && p.d == kD && p.q_len == 1 && p.gq <= 8 &&
           p.L % kGroupRows == 0 && nb_max <= kMaxCluster * kMaxLoc;
}

}  // namespace hga
