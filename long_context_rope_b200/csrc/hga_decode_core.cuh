// hga_decode_core.cuh -- the attention half of single-token decode, shared by
// the split-K decode attention kernel and the fused decode step.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4: standard softmax over the bounded
// exact token set. One query token, gq <= 8 query heads of one KV head; the
// heads share every key/value load (GQA).
//
// A CTA streams its share of the unit's 16-row key blocks through a ring of
// shared-memory stages (TMA tile loads, 128-byte swizzle) and eight consumer
// warps take every 8th block: S^T[16 keys x 8 heads] = K_blk Q^T and
// O^T[128 dims x 8 heads] += V^T P^T on warp-level bf16 MMA (m16n8k16, fp32
// accumulate) with a per-warp online softmax in fp32. Partials (max, sum, O)
// merge first across the warps of a CTA, then across the CTAs of the cluster
// through distributed shared memory.
//
// FP8 (E4M3) keys and values: a 16-row block is 2 KiB per tensor (one
// 128-byte swizzled panel). The products run on fp16 MMA (m16n8k16, fp32
// accumulate): every E4M3 value converts to fp16 exactly, two codes per
// convert instruction; the scales multiply the scores (k_scale) and the
// normalised output (v_scale). Shared-memory reads are 8-byte loads; the
// MMA's k and m indices are permuted so that each lane's bytes are
// contiguous:
//   S = K Q^T   step kk = 2j + e of the head dimension: logical k 2t4 + {0,1}
//               is dim 32j + 8t4 + 4e + {0,1}, logical 2t4 + 8 + {0,1} is
//               dim 32j + 8t4 + 4e + {2,3} (queries permuted the same way);
//   O^T += V^T P^T  tile mt, output row g is dim 8g + mt and row g + 8 is
//               dim 64 + 8g + mt.
// Both are bijections of the 128 dims, so the results are the same dot
// products and output dims, in another summation order.
#pragma once

#include <cooperative_groups.h>

#include "hga_common.cuh"
#include "hga_ptx.cuh"

namespace hga {
namespace dec {

namespace cg = cooperative_groups;

constexpr int kD = 128;
constexpr int kStages = 8;                       // ring of key blocks (bf16)
constexpr int kStagesMax = 16;                   // E4M3: the same bytes hold 16 blocks
constexpr int kBlkBytes = kGroupRows * kD * 2;   // 4 KiB per block per tensor (bf16)
constexpr int kBlkBytesF8 = kGroupRows * kD;     // 2 KiB per block per tensor (E4M3)
constexpr int kConsumers = 8;                    // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;  // + one producer warp
constexpr int kMaxCluster = 16;

// Row stride of a partial's O: 132 floats, so the per-warp stores (lanes
// spread over 4 heads x 8 dims) fall in 32 distinct banks.
constexpr int kOStride = kD + 4;

struct Partial {
    float m[8], l[8];          // per head
    float o[8][kOStride];      // per head, un-normalised (dims 0..kD-1 used)
};

struct Ring {
    alignas(1024) uint8_t k[kStages][kBlkBytes];
    alignas(1024) uint8_t v[kStages][kBlkBytes];
};

// Ring geometry: 8 stages of 4 KiB per tensor (bf16), or 16 stages of 2 KiB
// (E4M3) in the same bytes, so twice as many E4M3 blocks are in flight.
// Every stage starts on a 1024-byte boundary (the 128-byte swizzle's period).
// The stage count must be a multiple of the consumer warps: block i goes to
// warp i % 8 and stage i % S, so every use of a stage then belongs to one
// warp, which waits for its phases in order. With another count two warps
// share a stage, and a warp that reaches its wait for phase k + 2 before
// phase k + 1 has completed passes the parity wait at once (a parity names
// only two phases) and reads a stage that is still being refilled.
template <bool kF8>
__host__ __device__ constexpr int ring_stages() { return kF8 ? kStagesMax : kStages; }
static_assert(kStages % kConsumers == 0 && kStagesMax % kConsumers == 0,
              "ring stages must be a multiple of the consumer warps");
static_assert(kStagesMax * kBlkBytesF8 == kStages * kBlkBytes, "E4M3 stages fill the ring");
template <bool kF8>
__device__ __forceinline__ uint8_t* k_stage(Ring& ring, int s) {
    return &ring.k[0][0] + s * (kF8 ? kBlkBytesF8 : kBlkBytes);
}
template <bool kF8>
__device__ __forceinline__ uint8_t* v_stage(Ring& ring, int s) {
    return &ring.v[0][0] + s * (kF8 ? kBlkBytesF8 : kBlkBytes);
}

// Per-warp accumulator state of the online softmax.
struct WarpAcc {
    float o[8][4];
    float m[2], l[2];
};

// Q^T as MMA B fragments; heads >= gq are zero. bf16: lane (g, t4) holds
// Q[head g][16kk + 2t4 .. +1] and Q[head g][16kk + 2t4 + 8 .. +9]. E4M3 path:
// fp16 pairs of dims 32j + 8t4 + {0,1}, {2,3} (step 2j) and {4,5}, {6,7}
// (step 2j + 1), the permutation the key fragments use.
template <bool kF8>
__device__ __forceinline__ void load_q_frags(const Params& p, const __nv_bfloat16* q, int b, int h,
                                             uint32_t (&qf)[8][2]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const bool okh = g < p.gq;
    const __nv_bfloat16* qr =
        q + ((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq + (okh ? g : 0)) * kD;
    if constexpr (kF8) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 raw = okh ? *reinterpret_cast<const uint4*>(qr + 32 * j + 8 * t4)
                                  : make_uint4(0u, 0u, 0u, 0u);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
            uint32_t f[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 v = __bfloat1622float2(h2[e]);
                const __half2 hv = __floats2half2_rn(v.x, v.y);
                f[e] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            qf[2 * j][0] = f[0];
            qf[2 * j][1] = f[1];
            qf[2 * j + 1][0] = f[2];
            qf[2 * j + 1][1] = f[3];
        }
    } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = okh ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4) : 0u;
            qf[kk][1] = okh ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4 + 8) : 0u;
        }
    }
}

// E4M3 path: the 16-bit word whose low byte is byte m of a and whose high
// byte is byte m of b (m = 0..3).
__device__ __forceinline__ uint16_t byte_pair(uint32_t a, uint32_t b, int m) {
    return (uint16_t)__byte_perm(a, b, (unsigned)(m | ((m + 4) << 4)));
}

__device__ __forceinline__ void acc_init(WarpAcc& a) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) a.o[mt][e] = 0.f;
    a.m[0] = a.m[1] = -INFINITY;
    a.l[0] = a.l[1] = 0.f;
}

// Consumer warp `warp` processes local blocks warp, warp + 8, ... < nloc of
// the ring. blk_pos[i] is the position of block i's first token. pt is the
// warp's 8 x 16 transpose buffer of P (bf16, or fp16 on the E4M3 path, as
// bits). Returns false (and sets *bad) if a wait gave up.
template <bool kF8>
__device__ __forceinline__ bool consume_blocks(const Params& p, const uint32_t (&qf)[8][2],
                                               Ring& ring, uint64_t* full, uint64_t* empty,
                                               const int* blk_pos, int nloc, int qpos,
                                               uint16_t (*pt)[16], WarpAcc& acc, int* bad) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const float sc0 = 1.4426950408889634f / sqrtf((float)kD);
    const float sc = kF8 ? sc0 * p.k_scale : sc0;
    const int mq = lane >> 3;
    const int krow = (mq & 1) * 8 + (lane & 7);      // K ldmatrix row
    const int vkey = (mq >> 1) * 8 + (lane & 7);     // V ldmatrix (trans) row
    constexpr int S = ring_stages<kF8>();
    for (int i = warp; i < nloc; i += kConsumers) {
        const int s = i % S;
        const bool got = __all_sync(
            0xffffffffu, ptx::mbar_wait_bounded(&full[s], (i / S) & 1, p.wait_ns));
        if (!got) {
            if (lane == 0) {
                raise_timeout(p);
                *bad = 1;
            }
            return false;
        }
        // S^T = K Q^T for 16 keys x 8 heads (two accumulator chains)
        float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sacc2[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (kF8) {
            // rows g and g + 8, dims 32j + 8t4 .. +7: 16-byte chunk 2j + t4/2
            // of the row, XOR-swizzled by the row (g and g + 8 alike)
            const uint8_t* kb = k_stage<true>(ring, s);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int off = (((2 * j + (t4 >> 1)) ^ g) << 4) + (t4 & 1) * 8;
                const uint2 w0 = *reinterpret_cast<const uint2*>(kb + g * 128 + off);
                const uint2 w1 = *reinterpret_cast<const uint2*>(kb + (g + 8) * 128 + off);
                uint32_t a[4] = {ptx::e4m3x2_to_f16x2((uint16_t)w0.x),
                                 ptx::e4m3x2_to_f16x2((uint16_t)w1.x),
                                 ptx::e4m3x2_to_f16x2((uint16_t)(w0.x >> 16)),
                                 ptx::e4m3x2_to_f16x2((uint16_t)(w1.x >> 16))};
                ptx::mma_16816_f16(sacc, a, qf[2 * j][0], qf[2 * j][1]);
                uint32_t a2[4] = {ptx::e4m3x2_to_f16x2((uint16_t)w0.y),
                                  ptx::e4m3x2_to_f16x2((uint16_t)w1.y),
                                  ptx::e4m3x2_to_f16x2((uint16_t)(w0.y >> 16)),
                                  ptx::e4m3x2_to_f16x2((uint16_t)(w1.y >> 16))};
                ptx::mma_16816_f16(sacc2, a2, qf[2 * j + 1][0], qf[2 * j + 1][1]);
            }
        } else {
            const uint32_t kb = ptx::smem_u32(k_stage<false>(ring, s));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int chunk = (kk & 3) * 2 + (mq >> 1);
                uint32_t a[4];
                ptx::ldsm_x4(kb + (kk >> 2) * 2048 + krow * 128 + ((chunk ^ (krow & 7)) << 4), a);
                ptx::mma_16816((kk & 1) ? sacc2 : sacc, a, qf[kk][0], qf[kk][1]);
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[e] += sacc2[e];
        // this lane holds keys g, g+8 for heads 2t4, 2t4+1
        const int kp = blk_pos[i];
        const bool v0 = kp + g <= qpos, v1 = kp + g + 8 <= qpos;
        const float sv[4] = {v0 ? sacc[0] * sc : -INFINITY, v0 ? sacc[1] * sc : -INFINITY,
                             v1 ? sacc[2] * sc : -INFINITY, v1 ? sacc[3] * sc : -INFINITY};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float mb = fmaxf(sv[hh], sv[hh + 2]);
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 4));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
            const float mn = fmaxf(acc.m[hh], mb);
            float alpha = 1.f, p0 = 0.f, p1 = 0.f;
            if (mn != -INFINITY) {
                alpha = acc.m[hh] == -INFINITY ? 0.f : ptx::ex2_approx(acc.m[hh] - mn);
                p0 = ptx::ex2_approx(sv[hh] - mn);
                p1 = ptx::ex2_approx(sv[hh + 2] - mn);
            }
            acc.m[hh] = mn;
            // bf16 weights (fp16 on the E4M3 path); the running sum uses the
            // same rounded values
            uint16_t b0, b1;
            float r0, r1;
            if constexpr (kF8) {
                const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
                b0 = __half_as_ushort(h0);
                b1 = __half_as_ushort(h1);
                r0 = __half2float(h0);
                r1 = __half2float(h1);
            } else {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
                b0 = __bfloat16_as_ushort(h0);
                b1 = __bfloat16_as_ushort(h1);
                r0 = __bfloat162float(h0);
                r1 = __bfloat162float(h1);
            }
            acc.l[hh] = acc.l[hh] * alpha + r0 + r1;
            pt[2 * t4 + hh][g] = b0;
            pt[2 * t4 + hh][g + 8] = b1;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                acc.o[mt][hh] *= alpha;
                acc.o[mt][hh + 2] *= alpha;
            }
        }
        __syncwarp();
        const uint32_t pb0 = *reinterpret_cast<const uint32_t*>(&pt[g][2 * t4]);
        const uint32_t pb1 = *reinterpret_cast<const uint32_t*>(&pt[g][2 * t4 + 8]);
        // O^T[16 dims x 8 heads] += V^T P^T, eight 16-dim tiles
        if constexpr (kF8) {
            // keys 2t4, 2t4 + 1, 2t4 + 8, 2t4 + 9; dims 8g .. +7 (rows g of
            // the tiles) and 64 + 8g .. +7 (rows g + 8): 16-byte chunk g/2
            // (or 4 + g/2) of the key's row, XOR-swizzled by the key
            const uint8_t* vb = v_stage<true>(ring, s);
            auto ldv = [&](int key, int hi) {
                const int off = (((hi * 4 + (g >> 1)) ^ (key & 7)) << 4) + (g & 1) * 8;
                return *reinterpret_cast<const uint2*>(vb + key * 128 + off);
            };
            const uint2 v0l = ldv(2 * t4, 0), v1l = ldv(2 * t4 + 1, 0);
            const uint2 v0h = ldv(2 * t4, 1), v1h = ldv(2 * t4 + 1, 1);
            const uint2 v8l = ldv(2 * t4 + 8, 0), v9l = ldv(2 * t4 + 9, 0);
            const uint2 v8h = ldv(2 * t4 + 8, 1), v9h = ldv(2 * t4 + 9, 1);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int m = mt & 3;
                const bool y = mt >= 4;
                uint32_t a[4] = {
                    ptx::e4m3x2_to_f16x2(byte_pair(y ? v0l.y : v0l.x, y ? v1l.y : v1l.x, m)),
                    ptx::e4m3x2_to_f16x2(byte_pair(y ? v0h.y : v0h.x, y ? v1h.y : v1h.x, m)),
                    ptx::e4m3x2_to_f16x2(byte_pair(y ? v8l.y : v8l.x, y ? v9l.y : v9l.x, m)),
                    ptx::e4m3x2_to_f16x2(byte_pair(y ? v8h.y : v8h.x, y ? v9h.y : v9h.x, m))};
                ptx::mma_16816_f16(acc.o[mt], a, pb0, pb1);
            }
        } else {
            const uint32_t vb = ptx::smem_u32(v_stage<false>(ring, s));
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int chunk = (mt & 3) * 2 + (mq & 1);
                uint32_t a[4];
                ptx::ldsm_x4_trans(vb + (mt >> 2) * 2048 + vkey * 128 + ((chunk ^ (vkey & 7)) << 4),
                                   a);
                ptx::mma_16816(acc.o[mt], a, pb0, pb1);
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
    return true;
}

// Consumer warp writes its partial (row max, row sum, O) to wp. Accumulator
// tile mt holds dims mt * 16 + {g, g + 8} (bf16 path) or 8g + mt and
// 64 + 8g + mt (E4M3 path).
template <bool kF8>
__device__ __forceinline__ void store_warp_partial(const WarpAcc& acc, Partial& wp) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    float lsum[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float v = acc.l[hh];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        lsum[hh] = v;
    }
    if (g == 0) {
        wp.m[2 * t4] = acc.m[0];
        wp.m[2 * t4 + 1] = acc.m[1];
        wp.l[2 * t4] = lsum[0];
        wp.l[2 * t4 + 1] = lsum[1];
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int d0 = kF8 ? 8 * g + mt : mt * 16 + g;
        const int d1 = kF8 ? 64 + 8 * g + mt : d0 + 8;
        wp.o[2 * t4][d0] = acc.o[mt][0];
        wp.o[2 * t4 + 1][d0] = acc.o[mt][1];
        wp.o[2 * t4][d1] = acc.o[mt][2];
        wp.o[2 * t4 + 1][d1] = acc.o[mt][3];
    }
}

// The heads a CTA finalises: CTA r of a cluster of CL owns heads r, r + CL,
// ... (below gq); every CTA of the cluster writes its merged partial of such
// a head into the owner's Owned buffer, slot src * owned_per_cta(CL) + n / CL.
// CL * ceil(8 / CL) <= kOwnSlots for every CL <= 16. The buffer must not
// share memory with the ring: a peer may write it while this CTA still
// consumes blocks.
constexpr int kOwnSlots = 16;
__host__ __device__ constexpr int owned_per_cta(int CL) { return (8 + CL - 1) / CL; }
__host__ __device__ constexpr bool owned_slots_fit(int cl = 1) {
    return cl > kMaxCluster || (cl * owned_per_cta(cl) <= kOwnSlots && owned_slots_fit(cl + 1));
}
static_assert(owned_slots_fit(), "owned slots for every cluster size");

struct Owned {
    float m[kOwnSlots], l[kOwnSlots];  // per slot: max, sum
    float o[kOwnSlots][kD];            // per slot: un-normalised O
};

// All threads of CTA r: merge the 8 warp partials of each head n < gq (max
// M, weights 2^(m_w - M), weighted sums of l and O) and write the result
// straight into the Owned buffer of the head's owner (CTA n % CL) through
// distributed shared memory. wgt is an 8 x 8 scratch. The caller's cluster
// barrier then publishes these writes to the owners.
__device__ __forceinline__ void merge_warps_push(const Partial* warp_part, cg::cluster_group& cluster,
                                                 Owned& owned, float (*wgt)[8], int gq) {
    const int t = threadIdx.x;
    const int CL = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    const int per = owned_per_cta(CL);
    if (t < gq) {
        const int n = t;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, warp_part[w].m[n]);
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            const float mw = warp_part[w].m[n];
            const float wt = (M == -INFINITY || mw == -INFINITY) ? 0.f : ptx::ex2_approx(mw - M);
            wgt[w][n] = wt;
            den = fmaf(wt, warp_part[w].l[n], den);
        }
        Owned* dst = cluster.map_shared_rank(&owned, n % CL);
        dst->m[r * per + n / CL] = M;
        dst->l[r * per + n / CL] = den;
    }
    __syncthreads();
    for (int x = t; x < gq * kD; x += blockDim.x) {
        const int n = x / kD, d = x % kD;
        float num = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) num = fmaf(wgt[w][n], warp_part[w].o[n][d], num);
        cluster.map_shared_rank(&owned, n % CL)->o[r * per + n / CL][d] = num;
    }
}

// After the cluster barrier that published merge_warps_push's writes: CTA r
// merges the CL partials of each head it owns and writes the normalised
// output rows (bf16). It reads only its own shared memory, so no CTA waits
// for another afterwards.
__device__ __forceinline__ void merge_owned_and_store(const Params& p, int CL, int r,
                                                      const Owned& owned, int b, int h,
                                                      __nv_bfloat16* out) {
    const int per = owned_per_cta(CL);
    const int nh = (p.gq - r + CL - 1) / CL;  // heads r, r + CL, ... below gq
    for (int x = threadIdx.x; x < nh * kD; x += blockDim.x) {
        const int k = x / kD, d = x % kD, n = r + k * CL;
        float M = -INFINITY;
        for (int c = 0; c < CL; ++c) M = fmaxf(M, owned.m[c * per + k]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
            for (int c = 0; c < CL; ++c) {
                const float mc = owned.m[c * per + k];
                const float wgt = mc == -INFINITY ? 0.f : ptx::ex2_approx(mc - M);
                num = fmaf(wgt, owned.o[c * per + k][d], num);
                den = fmaf(wgt, owned.l[c * per + k], den);
            }
        }
        float o = den > 0.f ? num / den : 0.f;
        if (p.kv_f8) o *= p.v_scale;
        out[((int64_t)b * p.q_len * p.Hq + (int64_t)h * p.gq + n) * kD + d] =
            __float2bfloat16_rn(o);
    }
}

// Issue the TMA loads of one 16-row block into ring stage s: K and V, two
// 64-column bf16 halves each, or one 128-byte-wide E4M3 panel each.
template <bool kF8>
__device__ __forceinline__ void issue_block(Ring& ring, uint64_t* full, int s,
                                            const CUtensorMap* mk, const CUtensorMap* mv, int row,
                                            int outer) {
    if constexpr (kF8) {
        ptx::mbar_arrive_expect_tx(&full[s], 2 * kBlkBytesF8);
        ptx::tma_load_3d(k_stage<true>(ring, s), mk, 0, row, outer, &full[s]);
        ptx::tma_load_3d(v_stage<true>(ring, s), mv, 0, row, outer, &full[s]);
    } else {
        ptx::mbar_arrive_expect_tx(&full[s], 2 * kBlkBytes);
        for (int hf = 0; hf < 2; ++hf) {
            ptx::tma_load_3d(k_stage<false>(ring, s) + hf * 2048, mk, hf * 64, row, outer, &full[s]);
            ptx::tma_load_3d(v_stage<false>(ring, s) + hf * 2048, mv, hf * 64, row, outer, &full[s]);
        }
    }
}

// Producer thread, before the ring's memory is reused or the CTA exits:
// waits (bounded) until every block load of the first n_issued ring slots
// has landed. Slot i used stage i % S in phase i / S (S = ring_stages), and a stage
// is armed again only after its previous phase completed, so the last armed
// phase of each stage covers all of that stage's copies. False if a copy did
// not land within the drain limit.
template <bool kF8>
__device__ __forceinline__ bool drain_ring(uint64_t* full, int n_issued) {
    constexpr int S = ring_stages<kF8>();
    bool ok = true;
    for (int s = 0; s < S && s < n_issued; ++s) {
        const int last = s + ((n_issued - 1 - s) / S) * S;
        ok &= ptx::mbar_drain(&full[s], last / S);
    }
    return ok;
}

}  // namespace dec
}  // namespace hga
