// k_route.cu -- two-level routing: q-bar, chunk top-k, group top-k.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 2: level 1 scores the current
// chunk's query against the table of chunk key summaries of earlier chunks
// and keeps the top-k; level 2 scores the group key summaries inside the
// chosen chunks and keeps the top-k groups; the current chunk, the sink
// chunks and the recent local chunks are always visible and never routed.
//
// Scoring is HBM/L2 streaming (one 16-byte load per lane per summary row,
// several rows in flight per warp). A thread-block cluster splits one
// routing problem's candidates across CTAs; every CTA writes its candidates'
// 64-bit rank keys straight into the leader CTA's shared memory (distributed
// shared memory), and after one cluster barrier the leader's warp 0 takes the
// top-k by repeated warp arg-max and compacts the winners in ascending order.
#include <cooperative_groups.h>


#include "hga_kernels.h"
#include "hga_topk.cuh"

namespace cg = cooperative_groups;

namespace hga {

namespace {

template <typename T>
struct QVec;
template <>
struct QVec<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void add(const __nv_bfloat16* ptr, float* acc) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(ptr), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
    }
};
template <>
struct QVec<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void add(const float* ptr, float* acc) {
        float4 v = *reinterpret_cast<const float4*>(ptr);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
    }
};

// q-bar of every (b, KV head, query chunk): mean of the rotated queries over
// the chunk's query tokens and the KV head's gq query heads. Grid (nQC, B);
// 128 threads, so one wave holds the whole grid (64K context: 1024 CTAs, ~7
// per SM at 48 registers) and no partial second wave trails the stream.
constexpr int kQbarThreads = 128;
template <typename T>
__global__ void __launch_bounds__(kQbarThreads) qbar_kernel(Params p, const T* __restrict__ q,
                                                   float* __restrict__ qbar) {
    constexpr int V = QVec<T>::N;
    extern __shared__ float red[];
    const int jj = blockIdx.x, b = blockIdx.y;
    const int j = p.j0 + jj;
    const int nv = p.d / V, ncol = p.Hkv * nv;
    const int TL = ncol >= (int)blockDim.x ? 1 : (int)blockDim.x / ncol;
    const int tid = threadIdx.x;
    const int64_t pos_lo = (int64_t)j * p.C > p.q_begin ? (int64_t)j * p.C : p.q_begin;
    const int64_t span_end = (int64_t)p.q_begin + p.q_len;
    const int64_t pos_hi = (int64_t)(j + 1) * p.C < span_end ? (int64_t)(j + 1) * p.C : span_end;
    const int tl = tid / (ncol < (int)blockDim.x ? ncol : (int)blockDim.x);
    if (tl < TL) {
        for (int col = tid % (ncol < (int)blockDim.x ? ncol : (int)blockDim.x); col < ncol;
             col += blockDim.x) {
            const int h = col / nv, v = col % nv;
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll 2
            for (int64_t pos = pos_lo + tl; pos < pos_hi; pos += TL) {
                const T* row = q + (((int64_t)b * p.q_len + (pos - p.q_begin)) * p.Hq +
                                    (int64_t)h * p.gq) * p.d + v * V;
#pragma unroll 8
                for (int r = 0; r < p.gq; ++r) QVec<T>::add(row + (int64_t)r * p.d, acc);
            }
#pragma unroll
            for (int e = 0; e < V; ++e) red[((int64_t)tl * ncol + col) * V + e] = acc[e];
        }
    }
    __syncthreads();
    const float inv_n = 1.0f / (float)((pos_hi - pos_lo) * p.gq);
    for (int x = tid; x < ncol * V; x += blockDim.x) {
        float s = 0.f;
        for (int l = 0; l < TL; ++l) s += red[(int64_t)l * ncol * V + x];
        const int col = x / V, e = x % V;
        const int h = col / nv, v = col % nv;
        qbar[(((int64_t)b * p.Hkv + h) * p.nQC + jj) * p.d + v * V + e] = s * inv_n;
    }
}

// Load DPL consecutive floats of a summary row for this lane.
template <int DPL>
__device__ __forceinline__ void load_row(const float* row, int lane, float* v) {
    if constexpr (DPL == 4) {
        float4 t = __ldg(reinterpret_cast<const float4*>(row) + lane);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
        float2 t = __ldg(reinterpret_cast<const float2*>(row) + lane);
        v[0] = t.x; v[1] = t.y;
    }
}

constexpr int kRowsInFlight = 8;

// Level 1. Grid (CL, nQC, B*Hkv), cluster (CL, 1, 1), 256 threads.
template <int DPL>
__global__ void __launch_bounds__(256) route_chunks_kernel(Params p, float* __restrict__ qbar,
                                                           const void* __restrict__ q_rot,
                                                           int fuse_qbar,
                                                           const float* __restrict__ cs,
                                                           int32_t* __restrict__ sel,
                                                           int32_t* __restrict__ nsel,
                                                           float* __restrict__ scores) {
    extern __shared__ uint32_t keys[];     // [nC] candidate keys, then 256 histogram words
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int jj = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t* lk = cluster.map_shared_rank(keys, 0);

    float q[DPL];
    if (fuse_qbar) {
        // few query tokens (decode): every CTA forms q-bar itself from the
        // rotated queries (a few KB), rank 0 publishes it for level 2
        const int64_t span_end = (int64_t)p.q_begin + p.q_len;
        const int64_t pos_lo = (int64_t)j * p.C > p.q_begin ? (int64_t)j * p.C : p.q_begin;
        const int64_t pos_hi = (int64_t)(j + 1) * p.C < span_end ? (int64_t)(j + 1) * p.C : span_end;
        const int hk = (int)(bh % p.Hkv);
        const int64_t b = bh / p.Hkv;
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] = 0.f;
        for (int64_t pos = pos_lo; pos < pos_hi; ++pos) {
            const int64_t row0 = ((b * p.q_len + (pos - p.q_begin)) * p.Hq + (int64_t)hk * p.gq) * p.d;
#pragma unroll 8
            for (int r2 = 0; r2 < p.gq; ++r2) {
                const int64_t off = row0 + (int64_t)r2 * p.d + lane * DPL;
                if (p.dtype == HGA_BF16) {
                    const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(q_rot) + off;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) q[e] += __bfloat162float(qp[e]);
                } else {
                    const float* qp = reinterpret_cast<const float*>(q_rot) + off;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) q[e] += qp[e];
                }
            }
        }
        const float inv_n = 1.0f / (float)((pos_hi - pos_lo) * p.gq);
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] *= inv_n;
        if (r == 0 && warp == 0) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) qbar[prob * p.d + lane * DPL + e] = q[e];
        }
    } else {
        const float* qr = qbar + prob * p.d;
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] = qr[lane * DPL + e];
    }
    const int per = (j + CL - 1) / CL;
    const int c_lo = r * per;
    const int c_hi = c_lo + per < j ? c_lo + per : j;
    const float* table = cs + bh * (int64_t)p.nC * p.d;
    for (int c0 = c_lo + warp * kRowsInFlight; c0 < c_hi; c0 += nw * kRowsInFlight) {
        float v[kRowsInFlight][DPL];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int c = c0 + u < c_hi ? c0 + u : c_hi - 1;
            load_row<DPL>(table + (int64_t)c * p.d, lane, v[u]);
        }
        float sc[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(q[e], v[u][e], s);
            sc[u] = warp_sum(s);
        }
        if (lane < kRowsInFlight) {
            float s = sc[0];
#pragma unroll
            for (int u = 1; u < kRowsInFlight; ++u)
                if (lane == u) s = sc[u];
            const int c = c0 + lane;
            if (c < c_hi) {
                const bool forced = is_forced(p, j, c);
                lk[c] = forced ? 0u : score_key32(s);
                if (scores) scores[prob * p.nC + c] = forced ? __int_as_float(0x7fc00000) : s;
            }
        }
    }
    if (scores && r == 0)
        for (int c = j + threadIdx.x; c < p.nC; c += blockDim.x)
            scores[prob * p.nC + c] = __int_as_float(0x7fc00000);
    cluster.sync();
    if (r != 0 || warp != 0) return;
    const int kept = warp_radix_topk(keys, j, p.kc, p.kc, sel + prob * p.kc, keys + p.nC,
                                     [](int x) { return x; });
    if (lane == 0) nsel[prob] = kept;
}

// Level 2. Grid (CL, nQC, B*Hkv), cluster (CL, 1, 1), 256 threads.
template <int DPL>
__global__ void __launch_bounds__(256) route_groups_kernel(
    Params p, const float* __restrict__ qbar, const float* __restrict__ gs,
    const int32_t* __restrict__ sel_chunks, const int32_t* __restrict__ n_sel_chunks,
    int32_t* __restrict__ sel_groups, int32_t* __restrict__ n_sel_groups,
    float* __restrict__ scores) {
    extern __shared__ uint32_t keys[];     // [kc*G] candidate keys, then 256 histogram words
    __shared__ int s_chunk[1024];  // validated chunk of each slot, -1 if invalid
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int jj = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t* lk = cluster.map_shared_rank(keys, 0);

    int n = n_sel_chunks[prob];
    if (n < 0 || n > p.kc) {
        if (threadIdx.x == 0 && r == 0) raise_dev_error(p, kDevErrCount);
        n = n < 0 ? 0 : p.kc;
    }
    const int32_t* sc_in = sel_chunks + prob * p.kc;
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
        const int c = sc_in[s];
        const bool ok = c >= 0 && c < j && !is_forced(p, j, c) && (s == 0 || c > sc_in[s - 1]);
        s_chunk[s] = ok ? c : -1;
        if (!ok && r == 0) raise_dev_error(p, kDevErrChunkIndex);
    }
    __syncthreads();

    float q[DPL];
    {
        const float* qr = qbar + prob * p.d;
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] = qr[lane * DPL + e];
    }
    const int ncand = n * p.G;
    const int per = (ncand + CL - 1) / CL;
    const int x_lo = r * per;
    const int x_hi = x_lo + per < ncand ? x_lo + per : ncand;
    const float* table = gs + bh * (int64_t)p.nC * p.G * p.d;
    for (int x0 = x_lo + warp * kRowsInFlight; x0 < x_hi; x0 += nw * kRowsInFlight) {
        float v[kRowsInFlight][DPL];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            int x = x0 + u < x_hi ? x0 + u : x_hi - 1;
            int c = s_chunk[x / p.G];
            int64_t gi = c < 0 ? 0 : (int64_t)c * p.G + x % p.G;
            load_row<DPL>(table + gi * p.d, lane, v[u]);
        }
        float sc[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(q[e], v[u][e], s);
            sc[u] = warp_sum(s);
        }
        if (lane < kRowsInFlight) {
            float s = sc[0];
#pragma unroll
            for (int u = 1; u < kRowsInFlight; ++u)
                if (lane == u) s = sc[u];
            const int x = x0 + lane;
            if (x < x_hi) {
                const int c = s_chunk[x / p.G];
                // ties break on the candidate position x: candidates are in
                // ascending global group order, so this equals breaking on gi
                lk[x] = c < 0 ? 0u : score_key32(s);
                if (scores)
                    scores[prob * p.kc * p.G + x] = c < 0 ? __int_as_float(0x7fc00000) : s;
            }
        }
    }
    if (scores && r == 0)
        for (int x = ncand + threadIdx.x; x < p.kc * p.G; x += blockDim.x)
            scores[prob * p.kc * p.G + x] = __int_as_float(0x7fc00000);
    cluster.sync();
    if (r != 0 || warp != 0) return;
    const int G = p.G;
    const int kept = warp_radix_topk(keys, ncand, p.kg, p.kg, sel_groups + prob * p.kg,
                                     keys + p.kc * p.G,
                                     [&](int x) { return s_chunk[x / G] * G + x % G; });
    if (lane == 0) n_sel_groups[prob] = kept;
}

// Level 2 when every query chunk has at most 256 candidate groups
// (top_k_chunks * G <= 256): grid (nQC, B*Hkv), 128 threads. A warp takes
// one selected chunk at a time and reads its G group rows (contiguous in the
// table) with coalesced 16-byte loads; lane L holds dims L*DPL.. of every
// row, so each score is the same per-lane partial dot product and butterfly
// sum as in route_groups_kernel and the decode step (bitwise identical
// scores and selections). Warp 0 then selects.
template <int DPL>
__global__ void __launch_bounds__(128) route_groups_small_kernel(
    Params p, const float* __restrict__ qbar, const float* __restrict__ gs,
    const int32_t* __restrict__ sel_chunks, const int32_t* __restrict__ n_sel_chunks,
    int32_t* __restrict__ sel_groups, int32_t* __restrict__ n_sel_groups,
    float* __restrict__ scores) {
    constexpr int kMaxCand = 256;
    __shared__ uint32_t keys[kMaxCand];
    __shared__ uint32_t hist[256];
    __shared__ int s_chunk[kMaxCand];
    const int jj = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int j = p.j0 + jj;
    const int64_t prob = bh * p.nQC + jj;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

    int n = n_sel_chunks[prob];
    if (n < 0 || n > p.kc) {
        if (t == 0) raise_dev_error(p, kDevErrCount);
        n = n < 0 ? 0 : p.kc;
    }
    const int32_t* sc_in = sel_chunks + prob * p.kc;
    for (int s = t; s < n; s += blockDim.x) {
        const int c = sc_in[s];
        const bool ok = c >= 0 && c < j && !is_forced(p, j, c) && (s == 0 || c > sc_in[s - 1]);
        s_chunk[s] = ok ? c : -1;
        if (!ok) raise_dev_error(p, kDevErrChunkIndex);
    }
    float q[DPL];
    {
        const float* qr = qbar + prob * p.d;
#pragma unroll
        for (int e = 0; e < DPL; ++e) q[e] = qr[lane * DPL + e];
    }
    __syncthreads();

    const int G = p.G;
    const float* table = gs + bh * (int64_t)p.nC * G * p.d;
    for (int s = warp; s < n; s += 4) {
        const int c = s_chunk[s];
        const float* rows = table + (int64_t)(c < 0 ? 0 : c) * G * p.d;
        float v[8][DPL];
#pragma unroll
        for (int g = 0; g < 8; ++g)
            if (g < G) load_row<DPL>(rows + (int64_t)g * p.d, lane, v[g]);
        float sc = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            if (g < G) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) a = fmaf(q[e], v[g][e], a);
                a = warp_sum(a);
                if (lane == g) sc = a;
            }
        }
        if (lane < G) {
            const int x = s * G + lane;
            keys[x] = c < 0 ? 0u : score_key32(sc);
            if (scores) scores[prob * p.kc * G + x] = c < 0 ? __int_as_float(0x7fc00000) : sc;
        }
    }
    const int ncand = n * G;
    if (scores)
        for (int x = ncand + t; x < p.kc * G; x += blockDim.x)
            scores[prob * p.kc * G + x] = __int_as_float(0x7fc00000);
    __syncthreads();
    if (warp != 0) return;
    const int kept = warp_radix_topk(keys, ncand, p.kg, p.kg, sel_groups + prob * p.kg, hist,
                                     [&](int x) { return s_chunk[x / G] * G + x % G; });
    if (lane == 0) n_sel_groups[prob] = kept;
}

// Raise a kernel's dynamic shared-memory limit (once per device and kernel).
cudaError_t allow_smem(const void* fn, size_t bytes) {
    return set_func_attr_once(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_cluster(const void* fn, dim3 grid, int block, size_t smem, int cl,
                           cudaStream_t st, void** args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

cudaError_t launch_qbar(const Params& p, const void* q_rot, float* qbar, cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    const int V = p.dtype == HGA_BF16 ? 8 : 4;
    const int ncol = p.Hkv * (p.d / V);
    const int TL = ncol >= kQbarThreads ? 1 : kQbarThreads / ncol;
    size_t smem = (size_t)TL * ncol * V * sizeof(float);
    dim3 grid(p.nQC, p.B);
    if (p.dtype == HGA_BF16) {
        auto fn = qbar_kernel<__nv_bfloat16>;
        if (smem > 48 * 1024) {
            cudaError_t e = set_func_attr_once((const void*)fn,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        fn<<<grid, kQbarThreads, smem, st>>>(p, (const __nv_bfloat16*)q_rot, qbar);
    } else {
        auto fn = qbar_kernel<float>;
        if (smem > 48 * 1024) {
            cudaError_t e = set_func_attr_once((const void*)fn,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        fn<<<grid, kQbarThreads, smem, st>>>(p, (const float*)q_rot, qbar);
    }
    return cudaGetLastError();
}

static int chunk_cluster(const Params& p) {
    return p.nC >= 256 ? 8 : (p.nC >= 64 ? 4 : 1);
}

bool route_chunks_fuses_qbar(const Params& p) {
    return !route_chunks_tiled_supports(p) && p.q_len <= 4;
}

cudaError_t launch_route_chunks(const Params& p, const void* q_rot, float* qbar,
                                const float* chunk_sum, int32_t* sel, int32_t* n_sel,
                                float* scores, cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    if (route_chunks_tiled_supports(p))
        return launch_route_chunks_tiled(p, qbar, chunk_sum, sel, n_sel, scores, st);
    int fuse = route_chunks_fuses_qbar(p) ? 1 : 0;
    const int cl = chunk_cluster(p);
    size_t smem = ((size_t)p.nC + 256) * sizeof(uint32_t);
    dim3 grid(cl, p.nQC, p.B * p.Hkv);
    Params pp = p;
    void* args[] = {&pp, (void*)&qbar, (void*)&q_rot, &fuse, (void*)&chunk_sum, &sel, &n_sel, &scores};
    const void* fn = p.d == 128 ? (const void*)route_chunks_kernel<4>
                                : (const void*)route_chunks_kernel<2>;
    cudaError_t e = allow_smem(fn, (kMaxChunks + 256) * sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    return launch_cluster(fn, grid, 256, smem, cl, st, args);
}

cudaError_t launch_route_groups(const Params& p, const float* qbar, const float* group_sum,
                                const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                                int32_t* sel_groups, int32_t* n_sel_groups, float* scores,
                                cudaStream_t st) {
    if (p.nQC == 0) return cudaSuccess;
    if (p.kc * p.G <= 256) {
        const dim3 grid(p.nQC, p.B * p.Hkv);
        if (p.d == 128)
            route_groups_small_kernel<4><<<grid, 128, 0, st>>>(
                p, qbar, group_sum, sel_chunks, n_sel_chunks, sel_groups, n_sel_groups, scores);
        else
            route_groups_small_kernel<2><<<grid, 128, 0, st>>>(
                p, qbar, group_sum, sel_chunks, n_sel_chunks, sel_groups, n_sel_groups, scores);
        return cudaGetLastError();
    }
    const int64_t problems = (int64_t)p.B * p.Hkv * p.nQC;
    const int cl = problems >= 1024 ? 1 : 4;
    size_t smem = ((size_t)p.kc * p.G + 256) * sizeof(uint32_t);
    dim3 grid(cl, p.nQC, p.B * p.Hkv);
    Params pp = p;
    void* args[] = {&pp, (void*)&qbar, (void*)&group_sum, (void*)&sel_chunks,
                    (void*)&n_sel_chunks, &sel_groups, &n_sel_groups, &scores};
    const void* fn = p.d == 128 ? (const void*)route_groups_kernel<4>
                                : (const void*)route_groups_kernel<2>;
    cudaError_t e = allow_smem(fn, (8192 + 256) * sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    return launch_cluster(fn, grid, 256, smem, cl, st, args);
}

}  // namespace hga
