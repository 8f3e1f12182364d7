// k_gather.cu -- exact-token retrieval of the routed groups' K/V.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4 (the router fetches the original
// token-level K/V of the chosen groups into VRAM) and "Geheugenarchitectuur"
// (cold tier: the full K/V history in host RAM).
//
// HBM source: each 16-row group of K and of V is one contiguous block
// (16 * d elements); one thread issues bulk (TMA) copies global -> shared for
// SLOTS groups, waits on one mbarrier, then bulk-stores shared -> global.
// Host source: the pinned host store is read with 16-byte loads through its
// device mapping (zero-copy over the host link); every thread keeps several
// loads in flight.
#include "hga_blocks.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {

namespace {

constexpr int kSlotsPerCta = 8;

__device__ __forceinline__ int checked_count(const Params& p, const int32_t* n_sel, int64_t prob) {
    int n = n_sel[prob];
    if (n < 0 || n > p.kg) {
        raise_dev_error(p, kDevErrCount);
        n = n < 0 ? 0 : p.kg;
    }
    return n;
}

// Grid (ceil(kg / SLOTS), nQC, B*Hkv); one warp; lane 0 drives the copies.
__global__ void __launch_bounds__(32) gather_hbm_kernel(Params p, const char* __restrict__ k_src,
                                                        const char* __restrict__ v_src,
                                                        const int32_t* __restrict__ sel,
                                                        const int32_t* __restrict__ nsel,
                                                        char* __restrict__ k_dst,
                                                        char* __restrict__ v_dst) {
    extern __shared__ __align__(128) char buf[];
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const int jj = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const int es = p.dtype == HGA_BF16 ? 2 : 4;
    const uint32_t blk = (uint32_t)(kGroupRows * p.d * es);
    const int n = checked_count(p, nsel, prob);
    const int s_lo = blockIdx.x * kSlotsPerCta;
    const int s_hi = s_lo + kSlotsPerCta < n ? s_lo + kSlotsPerCta : n;
    if (s_lo >= s_hi) return;
    const int32_t* list = sel + prob * p.kg;
    int gi[kSlotsPerCta];
    uint32_t bytes = 0;
    for (int s = s_lo; s < s_hi; ++s) {
        gi[s - s_lo] = checked_group_entry(p, j, list, s);
        if (gi[s - s_lo] >= 0) bytes += 2 * blk;
    }
    if (bytes == 0) return;
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
    ptx::mbar_arrive_expect_tx(&bar, bytes);
    const int64_t src_base = bh * (int64_t)p.L * p.d * es;
    for (int s = s_lo; s < s_hi; ++s) {
        const int g = gi[s - s_lo];
        if (g < 0) continue;
        const int64_t off = src_base + (int64_t)g * blk;
        char* sk = buf + (size_t)(s - s_lo) * 2 * blk;
        ptx::bulk_g2s(sk, k_src + off, blk, &bar);
        ptx::bulk_g2s(sk + blk, v_src + off, blk, &bar);
    }
    if (!ptx::mbar_wait_bounded(&bar, 0, p.err)) {
        raise_dev_error(p, kDevErrTimeout);
        return;
    }
    const int64_t dst_base = prob * (int64_t)p.kg * blk;
    for (int s = s_lo; s < s_hi; ++s) {
        if (gi[s - s_lo] < 0) continue;
        char* sk = buf + (size_t)(s - s_lo) * 2 * blk;
        ptx::bulk_s2g(k_dst + dst_base + (int64_t)s * blk, sk, blk);
        ptx::bulk_s2g(v_dst + dst_base + (int64_t)s * blk, sk + blk, blk);
    }
    ptx::bulk_commit();
    ptx::bulk_wait_all();
}

constexpr int kHostSlots = 4;

// Grid (ceil(kg / kHostSlots), nQC, B*Hkv), 256 threads. Reads the mapped
// host store with 16-byte loads: each thread has 2 * kHostSlots loads in flight.
__global__ void __launch_bounds__(256) gather_host_kernel(Params p, const uint4* __restrict__ k_src,
                                                          const uint4* __restrict__ v_src,
                                                          const int32_t* __restrict__ sel,
                                                          const int32_t* __restrict__ nsel,
                                                          uint4* __restrict__ k_dst,
                                                          uint4* __restrict__ v_dst) {
    __shared__ int s_gi[kHostSlots];
    const int jj = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const int es = p.dtype == HGA_BF16 ? 2 : 4;
    const int vec_per_blk = kGroupRows * p.d * es / 16;
    const int s_lo = blockIdx.x * kHostSlots;
    if (threadIdx.x < kHostSlots) {
        const int n = checked_count(p, nsel, prob);
        const int s = s_lo + threadIdx.x;
        s_gi[threadIdx.x] = s < n ? checked_group_entry(p, j, sel + prob * p.kg, s) : -1;
    }
    __syncthreads();
    const int64_t src_base = bh * (int64_t)p.L * p.d * es / 16;
    const int64_t dst_base = prob * (int64_t)p.kg * vec_per_blk;
    for (int v0 = threadIdx.x; v0 < vec_per_blk; v0 += blockDim.x) {
        uint4 kk[kHostSlots], vv[kHostSlots];
#pragma unroll
        for (int u = 0; u < kHostSlots; ++u) {
            const int g = s_gi[u];
            if (g >= 0) {
                const int64_t off = src_base + (int64_t)g * vec_per_blk + v0;
                kk[u] = k_src[off];
                vv[u] = v_src[off];
            }
        }
#pragma unroll
        for (int u = 0; u < kHostSlots; ++u) {
            if (s_gi[u] >= 0) {
                const int64_t off = dst_base + (int64_t)(s_lo + u) * vec_per_blk + v0;
                k_dst[off] = kk[u];
                v_dst[off] = vv[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_gather(const Params& p, const void* k_src, const void* v_src, bool from_host,
                          const int32_t* sel_groups, const int32_t* n_sel_groups, void* k_dst,
                          void* v_dst, cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    const int es = p.dtype == HGA_BF16 ? 2 : 4;
    if (from_host) {
        dim3 grid((p.kg + kHostSlots - 1) / kHostSlots, p.nQC, p.B * p.Hkv);
        gather_host_kernel<<<grid, 256, 0, st>>>(p, (const uint4*)k_src, (const uint4*)v_src,
                                                 sel_groups, n_sel_groups, (uint4*)k_dst,
                                                 (uint4*)v_dst);
    } else {
        const size_t smem = (size_t)kSlotsPerCta * 2 * kGroupRows * p.d * es;
        static bool attr_set = false;
        if (!attr_set) {
            cudaError_t e = cudaFuncSetAttribute(
                gather_hbm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
            if (e != cudaSuccess) return e;
            attr_set = true;
        }
        dim3 grid((p.kg + kSlotsPerCta - 1) / kSlotsPerCta, p.nQC, p.B * p.Hkv);
        gather_hbm_kernel<<<grid, 32, smem, st>>>(p, (const char*)k_src, (const char*)v_src,
                                                  sel_groups, n_sel_groups, (char*)k_dst,
                                                  (char*)v_dst);
    }
    return cudaGetLastError();
}

}  // namespace hga
