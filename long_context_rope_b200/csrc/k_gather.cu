// k_gather.cu -- exact-token retrieval of the routed groups' K/V.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4 (the router fetches the original
// token-level K/V of the chosen groups into VRAM) and "Geheugenarchitectuur"
// (cold tier: the full K/V history in host RAM).
//
// HBM source: each 16-row group of K and of V is one contiguous block
// (16 * d elements); per CTA one thread streams its groups through a ring of
// shared-memory stages with bulk (TMA) loads and bulk stores.
// Host source: the pinned host store is read with 16-byte loads through its
// device mapping (zero-copy over the host link); every thread keeps several
// loads in flight.
#include "hga_blocks.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"
#include "hga_topk.cuh"

namespace hga {

namespace {

__device__ __forceinline__ int checked_count(const Params& p, const int32_t* n_sel, int64_t prob) {
    int n = n_sel[prob];
    if (n < 0 || n > p.kg) {
        raise_dev_error(p, kDevErrCount);
        n = n < 0 ? 0 : p.kg;
    }
    return n;
}

// HBM source. The copy units are the selection slots of all problems,
// flattened (unit = problem * kg + slot); CTA c takes the contiguous range
// [c * per, (c + 1) * per). Lanes first validate their units' selection
// entries in parallel; then lane 0 runs a ring of kGatherStages shared-memory
// stages: bulk (TMA) loads of a group's K and V block into a stage, counted
// on the stage's mbarrier, and bulk stores from the stage to the compact
// buffers, one bulk group per unit. kGatherStages - 1 loads are in flight
// while the oldest landed stage is stored; a stage is loaded again only
// after the store that last read it has finished reading.
constexpr int kGatherStages = 6;
constexpr int kGatherUnitsMax = 64;   // units of one CTA (per <= this)

__global__ void __launch_bounds__(32) gather_hbm_kernel(Params p, const char* __restrict__ k_src,
                                                        const char* __restrict__ v_src,
                                                        const int32_t* __restrict__ sel,
                                                        const int32_t* __restrict__ nsel,
                                                        char* __restrict__ k_dst,
                                                        char* __restrict__ v_dst, int per) {
    extern __shared__ __align__(128) char buf[];
    __shared__ __align__(8) uint64_t full[kGatherStages];
    __shared__ int64_t src_off[kGatherUnitsMax], dst_off[kGatherUnitsMax];
    const int lane = threadIdx.x;
    const int es = p.kv_es;
    const uint32_t blk = (uint32_t)(kGroupRows * p.d * es);
    const int64_t total = (int64_t)p.B * p.Hkv * p.nQC * p.kg;
    const int64_t u0 = (int64_t)blockIdx.x * per;
    // validate this CTA's units; compact the valid ones, in unit order
    int n = 0;
    for (int i0 = 0; i0 < per; i0 += 32) {
        const int64_t u = u0 + i0 + lane;
        bool ok = false;
        int64_t so = 0, dof = 0;
        if (i0 + lane < per && u < total) {
            const int64_t prob = u / p.kg;
            const int s = (int)(u % p.kg);
            const int64_t bh = prob / p.nQC;
            const int j = p.j0 + (int)(prob % p.nQC);
            // the count and the two list entries are independent loads (one
            // round trip); a bad count is recorded once, by the slot-0 unit
            const int32_t* list = sel + prob * p.kg;
            const int n_raw = nsel[prob];
            const int gi = list[s];
            const int prev = s > 0 ? list[s - 1] : -1;
            if (s == 0 && (n_raw < 0 || n_raw > p.kg)) raise_dev_error(p, kDevErrCount);
            const int cnt = min(max(n_raw, 0), p.kg);
            if (s < cnt) {
                const int c = gi >= 0 ? gi / p.G : -1;
                if (gi >= 0 && c < j && !is_forced(p, j, c) && (s == 0 || gi > prev)) {
                    ok = true;
                    so = bh * (int64_t)p.L * p.d * es + (int64_t)gi * blk;
                    dof = u * (int64_t)blk;
                } else {
                    raise_dev_error(p, kDevErrGroupIndex);
                }
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const int at = n + __popc(m & ((1u << lane) - 1u));
            src_off[at] = so;
            dst_off[at] = dof;
        }
        n += __popc(m);
    }
    __syncwarp();
    if (lane != 0 || n == 0) return;
    for (int s = 0; s < kGatherStages; ++s) ptx::mbar_init(&full[s], 1);
    ptx::fence_mbar_init();
    auto load = [&](int i) {
        char* st = buf + (size_t)(i % kGatherStages) * 2 * blk;
        uint64_t* bar = &full[i % kGatherStages];
        ptx::mbar_arrive_expect_tx(bar, 2 * blk);
        ptx::bulk_g2s(st, k_src + src_off[i], blk, bar);
        ptx::bulk_g2s(st + blk, v_src + src_off[i], blk, bar);
    };
    int loaded = 0;
    for (; loaded < kGatherStages - 1 && loaded < n; ++loaded) load(loaded);
    bool ok = true;
    for (int i = 0; i < n; ++i) {
        const int s = i % kGatherStages;
        if (!ptx::mbar_wait_bounded(&full[s], (uint32_t)(i / kGatherStages) & 1u, p.wait_ns)) {
            ok = false;
            break;
        }
        char* st = buf + (size_t)s * 2 * blk;
        ptx::bulk_s2g(k_dst + dst_off[i], st, blk);
        ptx::bulk_s2g(v_dst + dst_off[i], st + blk, blk);
        ptx::bulk_commit();
        if (loaded < n) {
            // the stage of unit `loaded` last held unit loaded - kGatherStages
            // = i - 1, whose store is the second newest bulk group
            if (loaded >= kGatherStages) ptx::bulk_wait_read<1>();
            load(loaded);
            ++loaded;
        }
    }
    if (!ok) {
        // gave up: every issued load lands before the CTA exits (the last
        // armed phase of each stage); stores were issued only from landed stages
        raise_timeout(p);
        for (int s = 0; s < kGatherStages && s < loaded; ++s) {
            const int last = s + ((loaded - 1 - s) / kGatherStages) * kGatherStages;
            ptx::mbar_drain(&full[s], last / kGatherStages);
        }
    }
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
    const int es = p.kv_es;
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

// ------------------------------------------------------------ warm tier
// "Geheugenarchitectuur": between the cold store in host RAM and attention,
// a bounded cache in VRAM keeps recently routed groups (least recently used
// out). Per (sequence, KV head) the caller owns n_slots pool slots of one
// group each, with the group index held (tag, -1 = empty) and the step of
// last use (last, -1 = never).

// Plan: one CTA per (sequence, KV head). Hits are found by a binary search
// of every slot's tag in the (ascending) selection list; the misses take the
// slots with the oldest last use that this step does not hit (ties to the
// lower slot), chosen exactly by the warp radix select. Writes the source of
// every selected group to src (slot for a hit, -2 - slot for a miss that
// fills that slot, -1 for an invalid entry) and updates tag / last.
constexpr int kMaxWarmSlots = 4096;

__global__ void __launch_bounds__(256) warm_plan_kernel(Params p, const int32_t* __restrict__ sel,
                                                        const int32_t* __restrict__ nsel,
                                                        int32_t* __restrict__ tag,
                                                        int32_t* __restrict__ last, int n_slots,
                                                        int step, int32_t* __restrict__ src,
                                                        int32_t* __restrict__ stats) {
    extern __shared__ uint32_t wsm[];
    uint32_t* key = wsm;                           // [n_slots] victim keys (0 = taken this step)
    uint32_t* hist = key + n_slots;                // [256]
    int* gi = reinterpret_cast<int*>(hist + 256);  // [kg] validated selection, -1 invalid
    int* hit = gi + p.kg;                          // [kg] slot holding the group, -1 none
    int* victim = hit + p.kg;                      // [kg] victim slots, ascending
    int* lst = victim + p.kg;                      // [kg] the list as given
    __shared__ int n_miss, n_valid;
    const int64_t bh = blockIdx.x;
    const int j = p.j0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t prob = bh * p.nQC;
    const int n = checked_count(p, nsel, prob);
    const int32_t* list = sel + prob * p.kg;
    for (int s = tid; s < p.kg; s += blockDim.x) {
        gi[s] = s < n ? checked_group_entry(p, j, list, s) : -1;
        lst[s] = s < n ? list[s] : -1;
        hit[s] = -1;
    }
    __syncthreads();
    int32_t* utag = tag + bh * n_slots;
    int32_t* ulast = last + bh * n_slots;
    for (int t = tid; t < n_slots; t += blockDim.x) {
        const int g = utag[t];
        int found = -1;
        if (g >= 0) {  // binary search in the ascending list (valid entries ascend)
            int lo = 0, hi = n - 1;
            while (lo <= hi) {
                const int mid = (lo + hi) >> 1;
                const int v = lst[mid];
                if (v == g) {
                    found = mid;
                    break;
                }
                if (v < g) lo = mid + 1; else hi = mid - 1;
            }
            if (found >= 0 && gi[found] < 0) found = -1;
        }
        if (found >= 0) hit[found] = t;
        // older last use -> larger key; never used -> largest; hit -> 0 (not a victim)
        key[t] = found >= 0 ? 0u : 0xffffffffu - (uint32_t)(ulast[t] + 1);
    }
    __syncthreads();
    if (warp == 0) {
        int m = 0, nv = 0;
        for (int s0 = 0; s0 < n; s0 += 32) {
            const int s = s0 + lane;
            m += __popc(__ballot_sync(0xffffffffu, s < n && gi[s] >= 0 && hit[s] < 0));
            nv += __popc(__ballot_sync(0xffffffffu, s < n && gi[s] >= 0));
        }
        warp_radix_topk(key, n_slots, m, m, victim, hist, [](int x) { return x; });
        if (lane == 0) {
            n_miss = m;
            n_valid = nv;
        }
    }
    __syncthreads();
    // the i-th miss in list order takes the i-th victim
    if (warp == 0) {
        int base = 0;
        for (int s0 = 0; s0 < p.kg; s0 += 32) {
            const int s = s0 + lane;
            const bool valid = s < n && gi[s] >= 0;
            const bool miss = valid && hit[s] < 0;
            const unsigned mm = __ballot_sync(0xffffffffu, miss);
            int out = -1;
            if (valid) out = miss ? -2 - victim[base + __popc(mm & ((1u << lane) - 1u))] : hit[s];
            if (s < p.kg) src[prob * p.kg + s] = out;
            if (valid) {
                const int slot = miss ? victim[base + __popc(mm & ((1u << lane) - 1u))] : hit[s];
                if (miss) utag[slot] = gi[s];
                ulast[slot] = step;
            }
            base += __popc(mm);
        }
        if (lane == 0 && stats) {
            stats[2 * bh] = n_valid - n_miss;  // hits (invalid entries count as neither)
            stats[2 * bh + 1] = n_miss;
        }
    }
}

// Copy: grid (ceil(kg / kHostSlots), 1, B*Hkv), 256 threads. A hit copies
// pool slot -> k_dst / v_dst (VRAM); a miss reads the mapped host store once
// and writes both k_dst / v_dst and its pool slot.
__global__ void __launch_bounds__(256) warm_copy_kernel(Params p, const uint4* __restrict__ k_host,
                                                        const uint4* __restrict__ v_host,
                                                        const int32_t* __restrict__ sel,
                                                        const int32_t* __restrict__ src,
                                                        uint4* __restrict__ pool_k,
                                                        uint4* __restrict__ pool_v, int n_slots,
                                                        uint4* __restrict__ k_dst,
                                                        uint4* __restrict__ v_dst) {
    __shared__ int s_src[kHostSlots], s_gi[kHostSlots];
    const int64_t bh = blockIdx.z;
    const int64_t prob = bh * p.nQC;
    const int es = p.kv_es;
    const int vec_per_blk = kGroupRows * p.d * es / 16;
    const int s_lo = blockIdx.x * kHostSlots;
    if (threadIdx.x < kHostSlots) {
        const int s = s_lo + threadIdx.x;
        s_src[threadIdx.x] = s < p.kg ? src[prob * p.kg + s] : -1;
        s_gi[threadIdx.x] = s < p.kg ? sel[prob * p.kg + s] : -1;
    }
    __syncthreads();
    const int64_t host_base = bh * (int64_t)p.L * p.d * es / 16;
    const int64_t pool_base = bh * (int64_t)n_slots * vec_per_blk;
    const int64_t dst_base = prob * (int64_t)p.kg * vec_per_blk;
    for (int v0 = threadIdx.x; v0 < vec_per_blk; v0 += blockDim.x) {
        uint4 kk[kHostSlots], vv[kHostSlots];
#pragma unroll
        for (int u = 0; u < kHostSlots; ++u) {
            const int sr = s_src[u];
            if (sr >= 0) {
                const int64_t off = pool_base + (int64_t)sr * vec_per_blk + v0;
                kk[u] = pool_k[off];
                vv[u] = pool_v[off];
            } else if (sr <= -2) {
                const int64_t off = host_base + (int64_t)s_gi[u] * vec_per_blk + v0;
                kk[u] = k_host[off];
                vv[u] = v_host[off];
            }
        }
#pragma unroll
        for (int u = 0; u < kHostSlots; ++u) {
            const int sr = s_src[u];
            if (sr == -1) continue;
            const int64_t off = dst_base + (int64_t)(s_lo + u) * vec_per_blk + v0;
            k_dst[off] = kk[u];
            v_dst[off] = vv[u];
            if (sr <= -2) {
                const int64_t po = pool_base + (int64_t)(-2 - sr) * vec_per_blk + v0;
                pool_k[po] = kk[u];
                pool_v[po] = vv[u];
            }
        }
    }
}

}  // namespace

bool gather_warm_supports(const Params& p, int n_slots) {
    return p.nQC == 1 && n_slots >= p.kg && n_slots <= kMaxWarmSlots;
}

cudaError_t launch_gather_warm(const Params& p, const void* k_host, const void* v_host,
                               const int32_t* sel_groups, const int32_t* n_sel_groups,
                               void* pool_k, void* pool_v, int32_t* pool_tag, int32_t* pool_last,
                               int n_slots, int step, int32_t* src_out, int32_t* stats_out,
                               void* k_dst, void* v_dst, cudaStream_t st) {
    const size_t smem = (size_t)(n_slots + 256) * sizeof(uint32_t) + (size_t)4 * p.kg * sizeof(int);
    {
        cudaError_t e = set_func_attr_once((const void*)warm_plan_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)((kMaxWarmSlots + 256) * 4 + 4 * kMaxBlocks * 4));
        if (e != cudaSuccess) return e;
    }
    warm_plan_kernel<<<p.B * p.Hkv, 256, smem, st>>>(p, sel_groups, n_sel_groups, pool_tag,
                                                     pool_last, n_slots, step, src_out, stats_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 grid((p.kg + kHostSlots - 1) / kHostSlots, 1, p.B * p.Hkv);
    warm_copy_kernel<<<grid, 256, 0, st>>>(p, (const uint4*)k_host, (const uint4*)v_host,
                                           sel_groups, src_out, (uint4*)pool_k, (uint4*)pool_v,
                                           n_slots, (uint4*)k_dst, (uint4*)v_dst);
    return cudaGetLastError();
}

cudaError_t launch_gather(const Params& p, const void* k_src, const void* v_src, bool from_host,
                          const int32_t* sel_groups, const int32_t* n_sel_groups, void* k_dst,
                          void* v_dst, cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    const int es = p.kv_es;
    if (from_host) {
        dim3 grid((p.kg + kHostSlots - 1) / kHostSlots, p.nQC, p.B * p.Hkv);
        gather_host_kernel<<<grid, 256, 0, st>>>(p, (const uint4*)k_src, (const uint4*)v_src,
                                                 sel_groups, n_sel_groups, (uint4*)k_dst,
                                                 (uint4*)v_dst);
    } else {
        const size_t smem = (size_t)kGatherStages * 2 * kGroupRows * p.d * es;
        cudaError_t e = set_func_attr_once((const void*)gather_hbm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kGatherStages * 2 * kGroupRows * 128 * 4);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cudaErrorInvalidValue;
        // one wave: four CTAs per SM fit (48 KB of stages each), each with
        // 4 .. kGatherUnitsMax units
        const int64_t total = (int64_t)p.B * p.Hkv * p.nQC * p.kg;
        int64_t per = (total + 4 * sms - 1) / (4 * sms);
        per = per < 4 ? 4 : (per > kGatherUnitsMax ? kGatherUnitsMax : per);
        const int64_t grid = (total + per - 1) / per;
        if (grid > INT32_MAX) return cudaErrorInvalidValue;
        gather_hbm_kernel<<<(unsigned)grid, 32, smem, st>>>(p, (const char*)k_src,
                                                           (const char*)v_src, sel_groups,
                                                           n_sel_groups, (char*)k_dst,
                                                           (char*)v_dst, (int)per);
    }
    return cudaGetLastError();
}

}  // namespace hga
