// k_route_tiled.cu -- level-1 routing for many query chunks at once (prefill).
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 2, Niveau 1: every query chunk
// scores the table of chunk key summaries of its earlier chunks and keeps the
// top-k; sink, local and current chunks are always visible and never routed.
//
// In prefill all query chunks of one (sequence, KV head) score the same
// table, so a CTA takes 8 query chunks and streams the table through shared
// memory once for all of them: a register-blocked fp32 product (each of 256
// threads 4 query chunks x 2 table rows), with the next table slice loaded
// into registers while the current one is multiplied, writes the 8 score
// rows to shared memory. Each of the 8 warps then selects the top-k of one
// query chunk with a 4-pass radix select over the order-preserving score
// keys (hga_topk.cuh) and writes the winners in ascending chunk order. Ties
// go to the lower chunk index; NaN ranks last. Work grows with the query
// chunk index (more earlier chunks to score), so CTAs take the last query
// chunks first and the block scheduler fills in with the short ones.
//
// Level 2 in the same warp (hga_route, when a group table is given; Niveau
// 2 of the same item): the warp that selected a query chunk's chunks then
// scores all G group rows of each of them (read from L2 eight rows at a
// time) and selects the top-k groups with the same radix select. Lane L
// holds dims L*DPL.. of every row and each score is the same per-lane
// partial dot product and butterfly sum as in route_groups_small_kernel and
// the decode step, so the fused and the separate routing select the same
// groups, bitwise. This replaces a second launch of one short CTA per query
// chunk and its round trip of the chunk lists through global memory.
#include "hga_kernels.h"
#include "hga_topk.cuh"

namespace hga {

namespace {

constexpr int kQB = 8;           // query chunks per CTA (one selecting warp each)
constexpr int kCT = 256;         // table rows per tile
constexpr int kKS = 32;          // dims per k-slice
constexpr int kThreads = 256;
constexpr int kPerThread = kCT * kKS / 4 / kThreads;  // float4 per thread per slice
static_assert(kKS == 32 && kCT % 32 == 0, "a slice row is 8 float4, rows come in warps of 4");
static_assert(kThreads / 32 == kQB, "one warp per query chunk");
static_assert(kThreads / 32 * 256 <= kKS * kCT, "histograms fit in the tile buffer");

// Shared words of the tile buffer reused once the products are done: the
// radix histograms [8 warps][256], then (level 2) group keys [8][256] and
// the selected chunks [8][64].
constexpr int kGroupKeysAt = kQB * 256;
constexpr int kSelChunksAt = kGroupKeysAt + kQB * 256;
static_assert(kSelChunksAt + kQB * 64 <= kKS * kCT, "level-2 scratch fits in the tile buffer");

template <int D>
__global__ void __launch_bounds__(kThreads, 3) route_chunks_tiled_kernel(
    Params p, const float* __restrict__ qbar, const float* __restrict__ cs,
    int32_t* __restrict__ sel, int32_t* __restrict__ nsel, float* __restrict__ scores_out,
    const float* __restrict__ gs, int32_t* __restrict__ sel_g, int32_t* __restrict__ nsel_g) {
    extern __shared__ __align__(16) float smem_f[];
    float* qT = smem_f;                         // [D][kQB]   transposed q-bar
    float* tile = qT + D * kQB;                 // [kKS][kCT] transposed table slice
    float* sc = tile + kKS * kCT;               // [kQB][ncp] scores
    const int ncp = (p.nC + 3) & ~3;
    uint32_t* hist = reinterpret_cast<uint32_t*>(tile);  // [8 warps][256], after the products

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int jj0 = (gridDim.x - 1 - blockIdx.x) * kQB;  // longest first
    const int nq = p.nQC - jj0 < kQB ? p.nQC - jj0 : kQB;
    const int j_hi = p.j0 + jj0 + nq;           // chunks [0, j_hi - 1) are candidates at most

    for (int x = tid; x < D * kQB; x += kThreads) {
        const int q = x % kQB, k = x / kQB;
        qT[x] = q < nq ? qbar[((bh * p.nQC) + jj0 + q) * D + k] : 0.f;
    }
    const float* table = cs + bh * (int64_t)p.nC * D;
    const int qg = tid & 1;                     // query group: queries 4*qg .. 4*qg+3
    const int cg = tid >> 1;                    // rows 2*cg, 2*cg+1 of the tile
    // Loader: float4 e = tid + kThreads * v of the slice is row e / 8, dims
    // 4 * (e % 8) ..; a warp reads 4 whole 128-byte slice rows. The
    // transposed tile stores row r of dim kk at column r ^ (4 * (kk / 4 % 8)),
    // so those stores hit 32 distinct banks; the XOR keeps 2 * cg and
    // 2 * cg + 1 adjacent for the float2 reads of the product.
    constexpr int kSlices = D / kKS;
    const int n_steps = ((j_hi - 1 + kCT - 1) / kCT) * kSlices;
    float4 pf[kPerThread];
    auto load = [&](int step) {
        const int k0 = (step % kSlices) * kKS;
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int e = tid + kThreads * v;
            const int c = (step / kSlices) * kCT + (e >> 3);
            pf[v] = c < p.nC ? __ldg(reinterpret_cast<const float4*>(table + (int64_t)c * D + k0) +
                                     (e & 7))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    if (n_steps > 0) load(0);
    float acc[4][2];
    for (int step = 0; step < n_steps; ++step) {
        const int ks = step % kSlices;
        const int c0 = (step / kSlices) * kCT, k0 = ks * kKS;
        if (ks == 0) {
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = 0.f;
        }
        __syncthreads();  // the previous slice is no longer read
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int e = tid + kThreads * v;
            const int ch = e & 7, col = (e >> 3) ^ (ch << 2);
            tile[(4 * ch + 0) * kCT + col] = pf[v].x;
            tile[(4 * ch + 1) * kCT + col] = pf[v].y;
            tile[(4 * ch + 2) * kCT + col] = pf[v].z;
            tile[(4 * ch + 3) * kCT + col] = pf[v].w;
        }
        __syncthreads();
        if (step + 1 < n_steps) load(step + 1);  // lands while this slice is multiplied
#pragma unroll 8
        for (int k = 0; k < kKS; ++k) {
            const float4 qv = *reinterpret_cast<const float4*>(qT + (k0 + k) * kQB + 4 * qg);
            const float2 tv =
                *reinterpret_cast<const float2*>(tile + k * kCT + ((2 * cg) ^ (((k >> 2) & 7) << 2)));
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                acc[a][0] = fmaf(qa[a], tv.x, acc[a][0]);
                acc[a][1] = fmaf(qa[a], tv.y, acc[a][1]);
            }
        }
        if (ks == kSlices - 1) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int c = c0 + 2 * cg + bb;
                    if (c < ncp) sc[(4 * qg + a) * ncp + c] = acc[a][bb];
                }
        }
    }
    __syncthreads();

    // ---- per query chunk: radix top-k over its candidates (one warp each)
    uint32_t* h = hist + warp * 256;
    for (int q = warp; q < nq; q += kThreads / 32) {  // one pass: a warp per query chunk
        const int jj = jj0 + q, j = p.j0 + jj;
        const int64_t prob = bh * p.nQC + jj;
        float* srow = sc + q * ncp;
        if (scores_out) {
            float* so = scores_out + prob * p.nC;
            for (int c = lane; c < p.nC; c += 32)
                so[c] = (c < j && !is_forced(p, j, c)) ? srow[c] : __int_as_float(0x7fc00000);
        }
        // the score row becomes the key row in place (0 = not a candidate)
        uint32_t* krow = reinterpret_cast<uint32_t*>(srow);
        for (int c = lane; c < j; c += 32)
            krow[c] = is_forced(p, j, c) ? 0u : score_key32(srow[c]);
        __syncwarp();
        const int kept = warp_radix_topk(krow, j, p.kc, p.kc, sel + prob * p.kc, h,
                                         [](int x) { return x; });
        if (lane == 0) nsel[prob] = kept;
        if (gs == nullptr) continue;

        // ---- level 2: all G groups of the kept chunks, then their top k_g
        constexpr int DPL = D / 32;
        const int G = p.G;
        uint32_t* gkeys = reinterpret_cast<uint32_t*>(tile) + kGroupKeysAt + warp * 256;
        int32_t* s_chunk = reinterpret_cast<int32_t*>(tile) + kSelChunksAt + warp * 64;
        __syncwarp();  // this warp's lanes wrote the kept chunks
        for (int s = lane; s < kept; s += 32) s_chunk[s] = sel[prob * p.kc + s];
        float qv[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) qv[e] = qT[(lane * DPL + e) * kQB + q];
        __syncwarp();
        const float* gtab = gs + bh * (int64_t)p.nC * G * D;
        const int n_rows = kept * G;  // row x: group x % G of the (x / G)-th kept chunk
        for (int x0 = 0; x0 < n_rows; x0 += 8) {
            float v[8][DPL];  // eight group rows in flight
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int x = x0 + i < n_rows ? x0 + i : x0;
                const float* row = gtab + ((int64_t)s_chunk[x / G] * G + x % G) * D + lane * DPL;
                if constexpr (DPL == 4) {
                    const float4 t = __ldg(reinterpret_cast<const float4*>(row));
                    v[i][0] = t.x; v[i][1] = t.y; v[i][2] = t.z; v[i][3] = t.w;
                } else {
                    const float2 t = __ldg(reinterpret_cast<const float2*>(row));
                    v[i][0] = t.x; v[i][1] = t.y;
                }
            }
            float sc2 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) a = fmaf(qv[e], v[i][e], a);
                a = warp_sum(a);
                if (lane == i) sc2 = a;
            }
            if (lane < 8 && x0 + lane < n_rows) gkeys[x0 + lane] = score_key32(sc2);
        }
        __syncwarp();
        const int kept2 = warp_radix_topk(gkeys, kept * G, p.kg, p.kg, sel_g + prob * p.kg, h,
                                          [&](int x) { return s_chunk[x / G] * G + x % G; });
        if (lane == 0) nsel_g[prob] = kept2;
    }
}

}  // namespace

bool route_chunks_tiled_supports(const Params& p) {
    return p.nQC >= 8 && p.nC <= 2048 && (p.d == 128 || p.d == 64);
}

bool route_tiled_fuses_groups(const Params& p) {
    return route_chunks_tiled_supports(p) && p.G <= 8 && p.kc <= 64 && p.kc * p.G <= 256;
}

cudaError_t launch_route_chunks_tiled(const Params& p, const float* qbar, const float* chunk_sum,
                                      int32_t* sel, int32_t* n_sel, float* scores,
                                      cudaStream_t st, const float* group_sum, int32_t* sel_g,
                                      int32_t* n_sel_g) {
    const int ncp = (p.nC + 3) & ~3;
    const size_t smem = (size_t)(p.d * kQB + kKS * kCT + kQB * ncp) * sizeof(float);
    dim3 grid((p.nQC + kQB - 1) / kQB, p.B * p.Hkv);
    const void* fn = p.d == 128 ? (const void*)route_chunks_tiled_kernel<128>
                                : (const void*)route_chunks_tiled_kernel<64>;
    {
        const int max_smem = (int)((size_t)(128 * kQB + kKS * kCT + kQB * 2048) * sizeof(float));
        cudaError_t e = set_func_attr_once((const void*)route_chunks_tiled_kernel<128>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e == cudaSuccess)
            e = set_func_attr_once((const void*)route_chunks_tiled_kernel<64>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e != cudaSuccess) return e;
    }
    Params pp = p;
    void* args[] = {&pp,    (void*)&qbar,       (void*)&chunk_sum, &sel,   &n_sel,
                    &scores, (void*)&group_sum, &sel_g,            &n_sel_g};
    return cudaLaunchKernel(fn, grid, dim3(kThreads), args, smem, st);
}

}  // namespace hga
