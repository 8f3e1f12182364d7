// k_attend_tc.cu -- prefill exact attention over the routed set on the
// 5th-generation tensor cores (tcgen05 MMA, TMEM accumulators, TMA).
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 4: standard softmax over the bounded
// exact token set of each query chunk. With 64-query chunks and 8 query
// heads per KV head, one (sequence, KV head, query chunk) unit is a real
// dense contraction: 512 query rows against up to ~1.8K keys.
//
// A persistent CTA per SM walks the units (query-token pair, query chunk,
// sequence x KV head) u = blockIdx.x, blockIdx.x + gridDim.x, ... Each unit
// is two M tiles (A, B) of 128 query rows (16 tokens x 8 heads) that share
// every K/V tile; 11 warps:
//   warp 10     builds the key-block list of the CTA's next units (double
//               buffered), so no unit waits for its selection list;
//   warp 0      TMA producer: a unit's Q tiles as soon as the previous unit's
//               last QK has completed, then K and V tiles of 128 keys
//               assembled from 16-row group boxes (two stages each; stages
//               and barrier phases follow a per-CTA tile counter across units);
//   warp 1      TMEM owner and MMA issuer. Issue order per key tile t:
//               PV_A(t), QK_A(t+1), PV_B(t), QK_B(t+1), so the tensor core
//               works on one M tile while the other's softmax runs; the next
//               unit's first QKs follow the last PVs on the same queue;
//   warps 2..5  softmax of tile A, warps 6..9 softmax of tile B: each thread
//               owns one query row (its TMEM lane); it loads its S row,
//               masks (causal / padding), keeps a lazily rescaled running max
//               (O is rescaled in TMEM only when the max grows by > 2^8),
//               writes P = 2^(S - max) as bf16 back into TMEM over its S row,
//               and at the end of a unit normalises O and writes it out
//               through a small per-warp staging area as coalesced rows.
// TMEM: S_A | S_B | O_A | O_B (128 columns each); P_X lives in the first 64
// columns of S_X and feeds the PV MMA directly from TMEM. The key set comes
// in arbitrary group order (forced chunks, then routed groups), so each
// 128-key tile is 8 independent TMA boxes of 16 rows x 64 columns (x2).
// Every wait is bounded; on a timeout the CTA records a device error, stops
// its roles, waits for the TMA loads and MMAs it has issued, frees TMEM and
// exits. The device error word is never read here, so an invalid selection
// entry only removes that entry's keys from its own unit.
#include "hga_blocks.cuh"
#include "hga_kernels.h"
#include "hga_ptx.cuh"
#include "hga_tmap.h"

namespace hga {

namespace {

constexpr int kD = 128;
constexpr int kRows = 128;                 // query rows per M tile
constexpr int kTileKeys = 128;             // keys per tile
constexpr int kBlocksPerTile = kTileKeys / kGroupRows;
constexpr int kPanel = 128 * 128;          // 128 rows x 128 bytes (64 bf16)
constexpr int kTile = 2 * kPanel;          // 128 x 128 bf16
constexpr int kThreads = 352;  // 11 warps
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

__host__ __device__ constexpr uint32_t col_s(int x) { return (uint32_t)(x * 128); }
__host__ __device__ constexpr uint32_t col_o(int x) { return (uint32_t)(256 + x * 128); }

struct TcMaps {
    CUtensorMap q, k, v;
};

struct TcSmem {
    alignas(1024) uint8_t q[2][kTile];
    alignas(1024) uint8_t k[2][kTile];
    alignas(1024) uint8_t v[2][kTile];
    uint64_t bar_q, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2];
    uint64_t s_full[2], p_full[2], o_done[2], list_full[2], list_empty[2], drain;
    uint32_t tmem_base;
    int abort;
    int nb[2];                                        // per list buffer
    int blk_row[2][kMaxBlocks];
    int blk_pos[2][kMaxBlocks];
    int tile_last[2][kMaxBlocks / kBlocksPerTile];    // last key position of a tile, INT_MAX if partial
    alignas(16) uint8_t stage[8][32 * 64];            // per softmax warp: 32 rows x 32 output dims
};

static_assert(sizeof(TcSmem) + 1024 <= 227 * 1024, "shared memory of one CTA");

// One unit = (query-token pair of M tiles, query chunk, sequence x KV head);
// false for a pair with no token in the query span.
struct Unit {
    int pair, jj, b, h, j, tok0;
    int64_t bh;
};

__device__ __forceinline__ bool unit_at(const Params& p, int u, Unit& un) {
    const int pairs = p.C / 32;
    un.pair = u % pairs;
    const int rest = u / pairs;
    un.jj = rest % p.nQC;
    un.bh = rest / p.nQC;
    un.b = (int)(un.bh / p.Hkv);
    un.h = (int)(un.bh % p.Hkv);
    un.j = p.j0 + un.jj;
    un.tok0 = un.j * p.C + un.pair * 32;
    return un.tok0 < p.q_begin + p.q_len && un.tok0 + 32 > p.q_begin;
}

// Bounded wait shared by the roles of one CTA: gives up after the launch's
// wait limit or when another role of this CTA gave up (*abort); a give-up
// sets *abort so the other roles stop. Both are checked every 8 polls. The
// device error word is not consulted: an invalid selection entry (of this
// unit or any other, in this launch or an earlier one) never stops a wait.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         uint64_t limit_ns) {
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 7u) == 7u && (*abort || ptx::globaltimer_ns() - t0 > limit_ns)) break;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_s, uint32_t k_s) {
    constexpr uint32_t id_qk = ptx::idesc_bf16_f32(kRows, kTileKeys, 0, 0);
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
        ptx::umma_f16(d_tmem, ptx::smem_desc_sw128(q_s + off, 16, 1024),
                      ptx::smem_desc_sw128(k_s + off, 16, 1024), id_qk, kk > 0);
    }
}

// O (+)= P V with P (bf16) in TMEM columns [p_tmem, p_tmem + 64).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_s,
                                         bool accumulate) {
    constexpr uint32_t id_pv = ptx::idesc_bf16_f32(kRows, kD, 0, 1);
#pragma unroll
    for (int kk = 0; kk < kTileKeys / 16; ++kk)
        ptx::umma_f16_ts(d_tmem, p_tmem + kk * 8,
                         ptx::smem_desc_sw128(v_s + kk * 2048, kPanel, 1024), id_pv,
                         (accumulate || kk > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const __grid_constant__ TcMaps maps,
                                                               Params p,
                                                               const int32_t* __restrict__ sel,
                                                               const int32_t* __restrict__ nsel,
                                                               __nv_bfloat16* __restrict__ out,
                                                               int n_units) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>(
        align_smem_1024(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int span_end = p.q_begin + p.q_len;

    if (warp == 0) {
        if (lane == 0) {
            sm.abort = 0;
            ptx::mbar_init(&sm.bar_q, 1);
            ptx::mbar_init(&sm.q_empty, 1);
            for (int s = 0; s < 2; ++s) {
                ptx::mbar_init(&sm.k_full[s], 1);
                ptx::mbar_init(&sm.k_empty[s], 1);
                ptx::mbar_init(&sm.v_full[s], 1);
                ptx::mbar_init(&sm.v_empty[s], 1);
                ptx::mbar_init(&sm.s_full[s], 1);
                ptx::mbar_init(&sm.p_full[s], 4);
                ptx::mbar_init(&sm.o_done[s], 1);
                ptx::mbar_init(&sm.list_full[s], 1);
                ptx::mbar_init(&sm.list_empty[s], 9);  // the producer and the 8 softmax warps
            }
            ptx::mbar_init(&sm.drain, 1);
            ptx::fence_mbar_init();
        }
    } else if (warp == 1) {
        ptx::tmem_alloc(&sm.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort = &sm.abort;
    auto n_tiles_of = [](int nb) { return (nb + kBlocksPerTile - 1) / kBlocksPerTile; };

    if (warp == 10) {
        // ------------------------------------------------------ block lists
        // builds the key-block list of this CTA's next units into a double buffer
        int k = 0;
        Unit un;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            if (!unit_at(p, u, un)) continue;
            const int bf = k & 1;
            if (k >= 2 &&
                !__all_sync(0xffffffffu, wait_bar(&sm.list_empty[bf], ((k >> 1) - 1) & 1, abort, p.wait_ns)))
                break;
            const int64_t prob = un.bh * p.nQC + un.jj;
            const int nb = build_key_blocks_warp(p, un.j, sel + prob * p.kg, nsel + prob, false,
                                                 sm.blk_row[bf], sm.blk_pos[bf]);
            __syncwarp();
            for (int t = lane; t * kBlocksPerTile < nb; t += 32) {
                int last = 0;
#pragma unroll
                for (int i = 0; i < kBlocksPerTile; ++i) {
                    const int blk = t * kBlocksPerTile + i;
                    last = blk < nb ? max(last, sm.blk_pos[bf][blk] + kGroupRows - 1) : INT_MAX;
                }
                sm.tile_last[bf][t] = last;
            }
            __syncwarp();
            if (lane == 0) {
                sm.nb[bf] = nb;
                ptx::mbar_arrive(&sm.list_full[bf]);
            }
            ++k;
        }
    } else if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int k = 0, g0 = 0, nq_armed = 0;
            int last_gk = -1, last_gv = -1;  // last tile whose K / V loads were issued
            Unit un;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                if (!unit_at(p, u, un)) continue;
                const int bf = k & 1;
                if (!wait_bar(&sm.list_full[bf], (k >> 1) & 1, abort, p.wait_ns)) break;
                const int nb = sm.nb[bf];
                const int n = n_tiles_of(nb);
                if (k >= 1 && !wait_bar(&sm.q_empty, (k - 1) & 1, abort, p.wait_ns)) break;
                const int tq = un.tok0 - p.q_begin;
                ptx::mbar_arrive_expect_tx(&sm.bar_q, 2 * kTile);
                ++nq_armed;
                for (int x = 0; x < 2; ++x) {
                    ptx::tma_load_4d(sm.q[x], &maps.q, 0, un.h * 8, tq + 16 * x, un.b, &sm.bar_q);
                    ptx::tma_load_4d(sm.q[x] + kPanel, &maps.q, 64, un.h * 8, tq + 16 * x, un.b,
                                     &sm.bar_q);
                }
                for (int t = 0; t < n; ++t) {
                    const int g = g0 + t, s = g & 1;
                    if (g >= 2 && !wait_bar(&sm.k_empty[s], ((g >> 1) - 1) & 1, abort, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&sm.k_full[s], kTile);
                    last_gk = g;
                    for (int i = 0; i < kBlocksPerTile; ++i) {
                        const int blk = t * kBlocksPerTile + i;
                        const int row = blk < nb ? sm.blk_row[bf][blk] : p.L;  // past the end: zero fill
                        ptx::tma_load_3d(sm.k[s] + i * 2048, &maps.k, 0, row, (int)un.bh, &sm.k_full[s]);
                        ptx::tma_load_3d(sm.k[s] + kPanel + i * 2048, &maps.k, 64, row, (int)un.bh,
                                         &sm.k_full[s]);
                    }
                    if (g >= 2 && !wait_bar(&sm.v_empty[s], ((g >> 1) - 1) & 1, abort, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&sm.v_full[s], kTile);
                    last_gv = g;
                    for (int i = 0; i < kBlocksPerTile; ++i) {
                        const int blk = t * kBlocksPerTile + i;
                        const int row = blk < nb ? sm.blk_row[bf][blk] : p.L;
                        ptx::tma_load_3d(sm.v[s] + i * 2048, &maps.v, 0, row, (int)un.bh, &sm.v_full[s]);
                        ptx::tma_load_3d(sm.v[s] + kPanel + i * 2048, &maps.v, 64, row, (int)un.bh,
                                         &sm.v_full[s]);
                    }
                }
                if (!ok) break;
                ptx::mbar_arrive(&sm.list_empty[bf]);
                g0 += n;
                ++k;
            }
            // Drain: every tile load issued above has landed before the CTA
            // can exit. Each barrier is armed again only after its previous
            // phase completed, so waiting for its last armed phase covers
            // all of its copies. (A no-op wait in a launch that did not abort.)
            bool drained = ptx::mbar_drain(&sm.bar_q, nq_armed - 1);
            for (int s = 0; s < 2; ++s) {
                const int gk = last_gk - ((last_gk - s) & 1);  // last tile of stage s
                const int gv = last_gv - ((last_gv - s) & 1);
                drained &= ptx::mbar_drain(&sm.k_full[s], gk >= 0 ? gk >> 1 : -1);
                drained &= ptx::mbar_drain(&sm.v_full[s], gv >= 0 ? gv >> 1 : -1);
            }
            if (!drained) *abort = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q_s[2] = {ptx::smem_u32(sm.q[0]), ptx::smem_u32(sm.q[1])};
            int k = 0, g0 = 0;
            Unit un;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                if (!unit_at(p, u, un)) continue;
                const int bf = k & 1;
                ok = wait_bar(&sm.list_full[bf], (k >> 1) & 1, abort, p.wait_ns);
                if (!ok) break;
                const int n = n_tiles_of(sm.nb[bf]);
                const int s0 = g0 & 1;
                ok = wait_bar(&sm.bar_q, k & 1, abort, p.wait_ns) &&
                     wait_bar(&sm.k_full[s0], (g0 >> 1) & 1, abort, p.wait_ns);
                if (!ok) break;
                ptx::tc_fence_after();
                // S_x of the previous unit was read and its P consumed by the PV
                // issued before on this in-order queue
                const uint32_t k0 = ptx::smem_u32(sm.k[s0]);
                issue_qk(tmem + col_s(0), q_s[0], k0);
                ptx::umma_commit(&sm.s_full[0]);
                issue_qk(tmem + col_s(1), q_s[1], k0);
                ptx::umma_commit(&sm.s_full[1]);
                if (n == 1) ptx::umma_commit(&sm.q_empty);
                ptx::umma_commit(&sm.k_empty[s0]);
                for (int t = 0; ok && t < n; ++t) {
                    const int g = g0 + t, s = g & 1, s1 = (g + 1) & 1;
                    const bool more = t + 1 < n;
                    if (!wait_bar(&sm.v_full[s], (g >> 1) & 1, abort, p.wait_ns)) { ok = false; break; }
                    if (more && !wait_bar(&sm.k_full[s1], ((g + 1) >> 1) & 1, abort, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t v_s = ptx::smem_u32(sm.v[s]);
                    const uint32_t k_s1 = ptx::smem_u32(sm.k[s1]);
                    for (int x = 0; x < 2; ++x) {
                        // P_x of this tile; for t == 0 this also orders the
                        // PV that overwrites O_x after the same warps' epilogue
                        // of the previous unit read it
                        if (!wait_bar(&sm.p_full[x], g & 1, abort, p.wait_ns)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        issue_pv(tmem + col_o(x), tmem + col_s(x), v_s, t > 0);
                        if (more) {
                            issue_qk(tmem + col_s(x), q_s[x], k_s1);
                            ptx::umma_commit(&sm.s_full[x]);
                        } else {
                            ptx::umma_commit(&sm.o_done[x]);
                        }
                    }
                    if (!ok) break;
                    if (more && t + 2 == n) ptx::umma_commit(&sm.q_empty);  // last QK issued
                    ptx::umma_commit(&sm.v_empty[s]);
                    if (more) ptx::umma_commit(&sm.k_empty[s1]);
                }
                g0 += n;
                ++k;
            }
            // drain: every MMA issued above has completed before TMEM is freed
            ptx::umma_commit(&sm.drain);
            const uint64_t t0 = ptx::globaltimer_ns();
            while (!ptx::mbar_try_wait(&sm.drain, 0) &&
                   ptx::globaltimer_ns() - t0 < ptx::kDrainLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------ softmax
        const int x = (warp - 2) >> 2;                  // M tile of this warpgroup
        const int q4 = warp & 3;                        // TMEM lane quarter
        const int r = q4 * 32 + lane;                   // row = TMEM lane
        const int head = r & 7;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + col_s(x);
        const uint32_t o_addr = tmem + lane_off + col_o(x);
        const float sc = 1.4426950408889634f / sqrtf((float)kD);
        int k = 0, g0 = 0;
        Unit un;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            if (!unit_at(p, u, un)) continue;
            const int bf = k & 1;
            if (!__all_sync(0xffffffffu, wait_bar(&sm.list_full[bf], (k >> 1) & 1, abort, p.wait_ns))) {
                ok = false;
                break;
            }
            const int nb = sm.nb[bf];
            const int n = n_tiles_of(nb);
            const int tokx = un.tok0 + 16 * x;
            const int qpos = tokx + (r >> 3);
            const bool row_ok = qpos >= p.q_begin && qpos < span_end;
            float m_used = -INFINITY, l = 0.f;
            for (int t = 0; t < n; ++t) {
                const int g = g0 + t;
                if (!__all_sync(0xffffffffu, wait_bar(&sm.s_full[x], g & 1, abort, p.wait_ns))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                float sx[kTileKeys];
                {
                    uint32_t* xr = reinterpret_cast<uint32_t*>(sx);
                    ptx::tmem_ld64(s_addr, xr);
                    ptx::tmem_ld64(s_addr + 64, xr + 64);
                    ptx::tmem_wait_ld();
                    ptx::reg_fence<kTileKeys>(xr);
                }
                // mask (causal within the current chunk; padding past the set)
                const int blk0 = t * kBlocksPerTile;
                const bool need_mask = sm.tile_last[bf][t] > tokx;
                float mraw = -INFINITY;
                if (need_mask) {
#pragma unroll
                    for (int i = 0; i < kBlocksPerTile; ++i) {
                        const int kp = blk0 + i < nb ? sm.blk_pos[bf][blk0 + i] : 0x7fffffff - 64;
#pragma unroll
                        for (int e = 0; e < kGroupRows; ++e) {
                            const int c = i * kGroupRows + e;
                            sx[c] = (kp + e <= qpos) ? sx[c] : -INFINITY;
                            mraw = fmaxf(mraw, sx[c]);
                        }
                    }
                } else {
                    // four independent three-input chains
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < kTileKeys; c += 8) {
#pragma unroll
                        for (int uu = 0; uu < 4; ++uu)
                            m4[uu] = ptx::fmax3(m4[uu], sx[c + 2 * uu], sx[c + 2 * uu + 1]);
                    }
                    mraw = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                }
                const float m_new = fmaxf(m_used, mraw * sc);
                bool rescale = false;
                float alpha = 1.f;
                if (m_new != -INFINITY) {
                    if (m_used == -INFINITY) {
                        m_used = m_new;
                    } else if (m_new > m_used + kRescaleLog2) {
                        alpha = ptx::ex2_approx(m_used - m_new);
                        m_used = m_new;
                        rescale = true;
                    }
                }
                // P = 2^(S*sc - m), rounded to bf16; the row sum uses the rounded values
                uint32_t pk[kTileKeys / 2];
                float lsum0 = 0.f, lsum1 = 0.f;
                const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
#pragma unroll
                for (int c = 0; c < kTileKeys; c += 2) {
                    float a0, a1;
                    ptx::fma2_bc(sx[c], sx[c + 1], sc, neg_m, a0, a1);
                    const float p0 = ptx::ex2_approx(a0);
                    const float p1 = ptx::ex2_approx(a1);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    pk[c / 2] = *reinterpret_cast<uint32_t*>(&b2);
                    ptx::add_bf16x2_f32(pk[c / 2], lsum0, lsum1);
                }
                const float lsum = lsum0 + lsum1;
                // tcgen05.ld/st are warp-collective: the whole warp rescales its
                // rows when any row needs it (rows that do not use alpha = 1).
                // PV of the previous tile has completed: S of this tile was issued
                // after it on the same (in-order) tensor-core queue.
                if (__any_sync(0xffffffffu, rescale && t >= 1)) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        ptx::tmem_ld32(o_addr + 32 * c, o);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence<32>(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        ptx::tmem_st32(o_addr + 32 * c, o);
                    }
                }
                l = l * alpha + lsum;
                ptx::tmem_st32(s_addr, pk);
                ptx::tmem_st32(s_addr + 32, pk + 32);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.p_full[x]);
            }
            if (!ok) break;
            if (lane == 0) ptx::mbar_arrive(&sm.list_empty[bf]);
            if (!__all_sync(0xffffffffu, wait_bar(&sm.o_done[x], k & 1, abort, p.wait_ns))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const float inv = l > 0.f ? 1.0f / l : 0.f;
            // all of O in one round trip
            uint32_t o[kD];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(o_addr + 32 * c, o + 32 * c);
            ptx::tmem_wait_ld();
            ptx::reg_fence<kD>(o);
            ptx::tc_fence_before();
            // Coalesced output: four rounds of 32 dims; each row's 64 bytes go
            // through this warp's staging area (16-byte chunks XOR-swizzled by
            // (row / 2) % 4) and come back as 8 rows x 4 chunks per store.
            uint8_t* stg = sm.stage[warp - 2];
            const int rr = lane >> 2, cc = lane & 3;   // read-back: row within 8, chunk
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float f[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) f[z] = __uint_as_float(o[32 * qd + 8 * c + z]) * inv;
                    *reinterpret_cast<uint4*>(stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                        f32x8_to_bf16(f);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int R = 8 * i + rr;                       // row within the warp
                    const int rq = q4 * 32 + R;                     // row of the M tile
                    const int qp = tokx + (rq >> 3);
                    const uint4 v = *reinterpret_cast<const uint4*>(stg + R * 64 + ((cc ^ ((R >> 1) & 3)) << 4));
                    if (qp >= p.q_begin && qp < span_end) {
                        __nv_bfloat16* dst = out + (((int64_t)un.b * p.q_len + (qp - p.q_begin)) * p.Hq +
                                                    (int64_t)un.h * 8 + (rq & 7)) * kD + 32 * qd + 8 * cc;
                        *reinterpret_cast<uint4*>(dst) = v;
                    }
                }
                __syncwarp();
            }
            g0 += n;
            ++k;
        }
        ptx::tc_fence_before();
    }
    __syncthreads();
    if (*abort && tid == 0) raise_timeout(p);
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool tc_kernel_supports(const Params& p, bool gathered) {
    return p.dtype == HGA_BF16 && p.d == kD && p.gq == 8 && p.q_len > 1 && !gathered &&
           p.kv_layout == HGA_KV_FULL && p.C % 32 == 0;
}

cudaError_t launch_attend_tc(const Params& p, const void* q_rot, const KvSources& kv,
                             const int32_t* sel_groups, const int32_t* n_sel_groups, void* out,
                             cudaStream_t st) {
    TcMaps maps;
    const int64_t BH = (int64_t)p.B * p.Hkv;
    bool ok = make_query_map(&maps.q, q_rot, p.B, p.q_len, p.Hq, kD, 8, 16) &&
              make_rows_map(&maps.k, kv.k_res, BH, p.L, kD, kGroupRows) &&
              make_rows_map(&maps.v, kv.v_res, BH, p.L, kD, kGroupRows);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(TcSmem) + 1024;
    cudaError_t e = set_func_attr_once((const void*)attend_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidValue;
    const int64_t n_units = (int64_t)(p.C / 32) * p.nQC * BH;
    const int grid = (int)(n_units < sms ? n_units : sms);
    attend_tc_kernel<<<grid, kThreads, smem, st>>>(maps, p, sel_groups, n_sel_groups,
                                                   (__nv_bfloat16*)out, (int)n_units);
    return cudaGetLastError();
}

}  // namespace hga
