// k_attend_simt.cu -- exact softmax attention over the routed set, fp32 math
// on the CUDA cores.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4: standard softmax over the bounded
// exact token set, no synthetic summary values in the output.
//
// This kernel serves the fp32 workloads (whose 1e-4 tolerance rules out
// reduced-precision tensor-core inputs) and every shape the tensor-core
// kernels do not cover. One CTA = 16 query rows (token x query head) of one
// (sequence, KV head, query chunk) unit; 4 warps x 4 rows. Keys stream
// through shared memory 32 at a time (two 16-row blocks) as fp32; lane i of
// a warp scores key i, then the online-softmax state of the row is updated
// and each lane accumulates d/32 output columns.
#include "hga_blocks.cuh"
#include "hga_kernels.h"

namespace hga {

namespace {

constexpr int kRowsPerCta = 16;
constexpr int kRowsPerWarp = 4;
constexpr int kTileKeys = 32;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T, int D>
__global__ void __launch_bounds__(128) attend_simt_kernel(Params p, const T* __restrict__ q,
                                                          KvSources kv,
                                                          const int32_t* __restrict__ sel,
                                                          const int32_t* __restrict__ nsel,
                                                          T* __restrict__ out) {
    constexpr int DP = D + 4;          // padded fp32 row (conflict-free float4 reads)
    constexpr int NE = D / 32;         // output columns per lane
    __shared__ int blk_row[kMaxBlocks];
    __shared__ int blk_pos[kMaxBlocks];
    __shared__ int s_nb;
    __shared__ __align__(16) float sq[kRowsPerCta][D];
    __shared__ __align__(16) float sk[kTileKeys][DP];
    __shared__ __align__(16) float sv[kTileKeys][DP];

    const int rb = blockIdx.x, jj = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int b = (int)(bh / p.Hkv), h = (int)(bh % p.Hkv);
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const bool gathered = kv.k_gat != nullptr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int64_t span_end = (int64_t)p.q_begin + p.q_len;
    const int pos_lo = (int)((int64_t)j * p.C > p.q_begin ? (int64_t)j * p.C : p.q_begin);
    const int pos_hi = (int)((int64_t)(j + 1) * p.C < span_end ? (int64_t)(j + 1) * p.C : span_end);
    const int n_rows = (pos_hi - pos_lo) * p.gq;
    const int row0 = rb * kRowsPerCta;
    if (row0 >= n_rows) return;

    if (warp == 0) {
        const int32_t* list = sel ? sel + prob * p.kg : nullptr;
        const int nb_w = build_key_blocks_warp(p, j, list, sel ? nsel + prob : nullptr, gathered,
                                               blk_row, blk_pos);
        if (lane == 0) s_nb = nb_w;
    }
    for (int x = tid; x < kRowsPerCta * D; x += blockDim.x) {
        const int rr = x / D, e = x % D;
        const int r = row0 + rr;
        float v = 0.f;
        if (r < n_rows) {
            const int t = pos_lo + r / p.gq - p.q_begin;
            const int hq = h * p.gq + r % p.gq;
            v = to_f(q[(((int64_t)b * p.q_len + t) * p.Hq + hq) * D + e]);
        }
        sq[rr][e] = v;
    }
    __syncthreads();
    const int nb = s_nb;

    const int64_t res_slab = (int64_t)(p.kv_layout == HGA_KV_WINDOWS
                                           ? (int64_t)(p.n_sink + p.n_local + 1) * p.C
                                           : p.L);
    const T* kres = (const T*)kv.k_res + bh * res_slab * D;
    const T* vres = (const T*)kv.v_res + bh * res_slab * D;
    const T* kgat = gathered ? (const T*)kv.k_gat + prob * (int64_t)p.kg * kGroupRows * D : nullptr;
    const T* vgat = gathered ? (const T*)kv.v_gat + prob * (int64_t)p.kg * kGroupRows * D : nullptr;
    const float scale = 1.4426950408889634f / sqrtf((float)D);

    float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][NE];
    int qpos[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) acc[i][e] = 0.f;
        const int r = row0 + warp * kRowsPerWarp + i;
        qpos[i] = r < n_rows ? pos_lo + r / p.gq : -1;
    }

    for (int b0 = 0; b0 < nb; b0 += 2) {
        __syncthreads();
        // stage 32 keys (blocks b0, b0+1) as fp32
        for (int x = tid; x < kTileKeys * D; x += blockDim.x) {
            const int kr = x / D, e = x % D;
            const int bi = b0 + kr / kGroupRows;
            float kvk = 0.f, kvv = 0.f;
            if (bi < nb) {
                const int rw = blk_row[bi];
                const int pos = blk_pos[bi] + kr % kGroupRows;
                if (pos < p.L) {
                    int64_t off;
                    if (rw & kSrcGathered) {
                        off = (int64_t)((rw & ~kSrcGathered) + kr % kGroupRows) * D + e;
                        kvk = to_f(kgat[off]);
                        kvv = to_f(vgat[off]);
                    } else {
                        off = (int64_t)(rw + kr % kGroupRows) * D + e;
                        kvk = to_f(kres[off]);
                        kvv = to_f(vres[off]);
                    }
                }
            }
            sk[kr][e] = kvk;
            sv[kr][e] = kvv;
        }
        __syncthreads();
        const int bi = b0 + lane / kGroupRows;
        const int kpos = bi < nb ? blk_pos[bi] + lane % kGroupRows : 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            if (qpos[i] < 0) continue;
            const float* qr = sq[warp * kRowsPerWarp + i];
            float s = 0.f;
#pragma unroll 8
            for (int e = 0; e < D; e += 4) {
                const float4 a = *reinterpret_cast<const float4*>(qr + e);
                const float4 c = *reinterpret_cast<const float4*>(&sk[lane][e]);
                s = fmaf(a.x, c.x, s);
                s = fmaf(a.y, c.y, s);
                s = fmaf(a.z, c.z, s);
                s = fmaf(a.w, c.w, s);
            }
            const bool vis = kpos <= qpos[i] && kpos < p.L;
            s = vis ? s * scale : -INFINITY;
            const float mt = warp_max(s);
            const float mn = fmaxf(m[i], mt);
            float pr, alpha;
            if (mn == -INFINITY) {
                pr = 0.f;
                alpha = 1.f;
            } else {
                pr = vis ? exp2f(s - mn) : 0.f;
                alpha = exp2f(m[i] - mn);
            }
            m[i] = mn;
            l[i] = l[i] * alpha + warp_sum(pr);
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[i][e] *= alpha;
#pragma unroll 4
            for (int kk = 0; kk < kTileKeys; ++kk) {
                const float pk = __shfl_sync(0xffffffffu, pr, kk);
#pragma unroll
                for (int e = 0; e < NE; ++e) acc[i][e] = fmaf(pk, sv[kk][lane + 32 * e], acc[i][e]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        if (qpos[i] < 0) continue;
        const int r = row0 + warp * kRowsPerWarp + i;
        const int t = pos_lo + r / p.gq - p.q_begin;
        const int hq = h * p.gq + r % p.gq;
        const float inv = l[i] > 0.f ? 1.0f / l[i] : 0.f;
        T* orow = out + (((int64_t)b * p.q_len + t) * p.Hq + hq) * D;
#pragma unroll
        for (int e = 0; e < NE; ++e) orow[lane + 32 * e] = from_f<T>(acc[i][e] * inv);
    }
}

}  // namespace

cudaError_t launch_attend_simt(const Params& p, const void* q_rot, const KvSources& kv,
                               const int32_t* sel_groups, const int32_t* n_sel_groups,
                               void* out, cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    const int max_rows = (p.q_len < p.C ? p.q_len : p.C) * p.gq;
    dim3 grid((max_rows + kRowsPerCta - 1) / kRowsPerCta, p.nQC, p.B * p.Hkv);
    if (p.dtype == HGA_BF16) {
        if (p.d == 128)
            attend_simt_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(
                p, (const __nv_bfloat16*)q_rot, kv, sel_groups, n_sel_groups, (__nv_bfloat16*)out);
        else
            attend_simt_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(
                p, (const __nv_bfloat16*)q_rot, kv, sel_groups, n_sel_groups, (__nv_bfloat16*)out);
    } else {
        if (p.d == 128)
            attend_simt_kernel<float, 128><<<grid, 128, 0, st>>>(p, (const float*)q_rot, kv,
                                                                 sel_groups, n_sel_groups,
                                                                 (float*)out);
        else
            attend_simt_kernel<float, 64><<<grid, 128, 0, st>>>(p, (const float*)q_rot, kv,
                                                                sel_groups, n_sel_groups,
                                                                (float*)out);
    }
    return cudaGetLastError();
}

}  // namespace hga
