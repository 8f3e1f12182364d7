// k_summaries.cu -- RoPE and the RoPE-aware chunk / group key summaries.
//
// "Technische Samenvatting: Hierarchical Global Attention (HGA)"
// (gist.science), "Kernmechanisme" item 3: high-frequency RoPE pairs are
// rotated per token before averaging; low-frequency pairs are averaged in the
// raw-key space and rotated to the representative position (mean position)
// of the chunk or group. Built from the existing projected keys; no weights.
//
// One CTA per (sequence, KV head, chunk). HBM-streaming: each key row is read
// once with 16-byte vector loads and (optionally) its rotated copy written
// once. Thread (u, k, s) owns pair slice u (VEC pairs: dims u*VEC.. and
// d/2 + u*VEC..), group k, and the 4 tokens 16k + 4s + {0..3}; group sums
// are reduced across s and chunk sums across k with warp shuffles.
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    using Raw = uint4;  // one 16-byte vector as loaded
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const uint4*>(p));
    }
    static __device__ __forceinline__ void unpack(const Raw& r, float* f) { bf16x8_to_f32(r, f); }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* f) {
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* f) {
        *reinterpret_cast<uint4*>(p) = f32x8_to_bf16(f);
    }
};
template <>
struct Vec<float> {
    static constexpr int N = 4;
    using Raw = float4;
    static __device__ __forceinline__ Raw load_raw(const float* p) {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
    static __device__ __forceinline__ void unpack(const Raw& r, float* f) {
        f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
    }
    static __device__ __forceinline__ void load(const float* p, float* f) {
        float4 v = *reinterpret_cast<const float4*>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* f) {
        *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};

// ------------------------------------------------------------------ RoPE
// One thread per (row, pair slice); rows are [n_outer, n_tokens, n_heads].
template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(Params p, const T* __restrict__ x,
                                                   T* __restrict__ y, int64_t n_rows,
                                                   int64_t n_tokens, int n_heads, int64_t pos0) {
    constexpr int V = Vec<T>::N;
    const int half = p.d / 2, ns = half / V;
    const int64_t total = n_rows * ns;
    for (int64_t it = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; it < total;
         it += (int64_t)gridDim.x * blockDim.x) {
        int64_t row = it / ns;
        int u = (int)(it % ns);
        int64_t t = (row / n_heads) % n_tokens;
        double pos = (double)(pos0 + t);
        const T* xr = x + row * p.d;
        float a[V], b[V], ra[V], rb[V];
        Vec<T>::load(xr + u * V, a);
        Vec<T>::load(xr + half + u * V, b);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            float c, s;
            rope_cs(pos, p.inv_freq[u * V + e], c, s);
            ra[e] = a[e] * c - b[e] * s;
            rb[e] = a[e] * s + b[e] * c;
        }
        T* yr = y + row * p.d;
        Vec<T>::store(yr + u * V, ra);
        Vec<T>::store(yr + half + u * V, rb);
    }
}

// ------------------------------------------------------------- summaries
// n consecutive summary values (n = 4 or 8) written as fp32, or rounded to
// bf16 (nearest even) for bf16 summary tables.
__device__ __forceinline__ void store_sum(float* out, const float* v, int n) {
    for (int i = 0; i < n; i += 4)
        *reinterpret_cast<float4*>(out + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
__device__ __forceinline__ void store_sum(__nv_bfloat16* out, const float* v, int n) {
    if (n == 8) {
        *reinterpret_cast<uint4*>(out) = f32x8_to_bf16(v);
    } else {
        __nv_bfloat162 h[2] = {__floats2bfloat162_rn(v[0], v[1]), __floats2bfloat162_rn(v[2], v[3])};
        *reinterpret_cast<uint2*>(out) = *reinterpret_cast<const uint2*>(h);
    }
}

template <typename T, typename S>
__global__ void summaries_kernel(Params p, const T* __restrict__ k_raw, S* __restrict__ cs,
                                 S* __restrict__ gs, T* __restrict__ k_rot, int chunk_begin) {
    constexpr int V = Vec<T>::N;
    const int half = p.d / 2;
    const int G = p.G;
    const int tid = threadIdx.x;
    const int s = tid & 3;             // token lane within the group
    const int k = (tid >> 2) % G;      // group within the chunk
    const int u = tid / (4 * G);       // pair slice
    const int ch = chunk_begin + blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t c0 = (int64_t)ch * p.C;
    const T* base = k_raw + bh * (int64_t)p.L * p.d;

    float acc0[V], acc1[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc0[e] = acc1[e] = 0.f;

    // every row load of this thread is issued before any arithmetic
    typename Vec<T>::Raw raw_a[4], raw_b[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int64_t t = c0 + 16 * k + 4 * s + m;
        if (t < p.L) {
            const T* row = base + t * p.d;
            raw_a[m] = Vec<T>::load_raw(row + u * V);
            raw_b[m] = Vec<T>::load_raw(row + half + u * V);
        }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        int64_t t = c0 + 16 * k + 4 * s + m;
        if (t < p.L) {
            float a[V], b[V], ra[V], rb[V];
            Vec<T>::unpack(raw_a[m], a);
            Vec<T>::unpack(raw_b[m], b);
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const int i = u * V + e;
                float c, sn;
                rope_cs((double)t, p.inv_freq[i], c, sn);
                ra[e] = a[e] * c - b[e] * sn;
                rb[e] = a[e] * sn + b[e] * c;
                if (i < p.F) {
                    acc0[e] += ra[e];
                    acc1[e] += rb[e];
                } else {
                    acc0[e] += a[e];
                    acc1[e] += b[e];
                }
            }
            if (k_rot != nullptr) {
                T* orow = k_rot + bh * (int64_t)p.L * p.d + t * p.d;
                Vec<T>::store(orow + u * V, ra);
                Vec<T>::store(orow + half + u * V, rb);
            }
        }
    }

    // group sums: reduce over the 4 token lanes s
#pragma unroll
    for (int e = 0; e < V; ++e) {
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            acc0[e] += __shfl_xor_sync(0xffffffffu, acc0[e], off);
            acc1[e] += __shfl_xor_sync(0xffffffffu, acc1[e], off);
        }
    }
    auto finish = [&](const float* s0, const float* s1, int64_t first, int n, S* out) {
        float o0[V], o1[V];
        if (n <= 0) {
#pragma unroll
            for (int e = 0; e < V; ++e) o0[e] = o1[e] = 0.f;
        } else {
            const float inv_n = 1.0f / (float)n;
            const double pbar = (double)first + 0.5 * (double)(n - 1);
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const int i = u * V + e;
                float m0 = s0[e] * inv_n, m1 = s1[e] * inv_n;
                if (i < p.F) {
                    o0[e] = m0;
                    o1[e] = m1;
                } else {
                    float c, sn;
                    rope_cs(pbar, p.inv_freq[i], c, sn);
                    o0[e] = m0 * c - m1 * sn;
                    o1[e] = m0 * sn + m1 * c;
                }
            }
        }
        store_sum(out + u * V, o0, V);
        store_sum(out + half + u * V, o1, V);
    };
    if (s == 0) {
        int64_t g0 = c0 + 16 * k;
        int64_t left = (int64_t)p.L - g0;
        int n = left <= 0 ? 0 : (left >= 16 ? 16 : (int)left);
        S* out = gs + ((bh * p.nC + ch) * G + k) * (int64_t)p.d;
        finish(acc0, acc1, g0, n, out);
    }
    // chunk sums: reduce the group sums over k (lanes 4, 8, ...)
#pragma unroll
    for (int e = 0; e < V; ++e) {
        for (int off = 4; off < 4 * G; off <<= 1) {
            acc0[e] += __shfl_xor_sync(0xffffffffu, acc0[e], off);
            acc1[e] += __shfl_xor_sync(0xffffffffu, acc1[e], off);
        }
    }
    if (s == 0 && k == 0) {
        int64_t left = (int64_t)p.L - c0;
        int n = left <= 0 ? 0 : (left >= p.C ? p.C : (int)left);
        S* out = cs + (bh * p.nC + ch) * (int64_t)p.d;
        finish(acc0, acc1, c0, n, out);
    }
}

// ------------------------------------------------ streaming summaries
// Form for bf16 keys with d = 128, 4 groups of 16 rows per chunk and F a
// multiple of 4 (every bf16 workload here). Persistent CTAs walk the
// (sequence x KV head, chunk) items in order; one thread issues each chunk's
// rows (64 x 256 contiguous bytes) as one bulk copy into a ring of
// kSumStages shared-memory stages, so the next chunk's read is in flight
// while this one is rotated and summed; the rotated rows leave as plain
// coalesced 8-byte stores. Warp k owns group k; lane (r = lane / 16,
// u = lane % 16) owns pairs 4u .. 4u+3 of tokens 16k + 2i + r (i = 0..7), so
// one warp-wide 8-byte shared load reads two whole 128-byte half-rows (no
// bank conflict).
//
// Angles by the angle-addition formulas, so that no double-precision
// reduction or special-function op runs per element: a lane's first token
// is rotated by R((c0 + 16k) theta) R(r theta) and each next one by a further
// R(2 theta). R(r theta) and R(2 theta) are per-lane constants, and R(m theta)
// for m = 16, 32, 48 (group bases from the chunk bases) and m = 7.5, 31.5
// (mean positions of a full group and chunk) a per-CTA table, all from
// cs_accurate (about one fp32 ulp). Per item only R(c0 theta) and
// R((c0 + 32) theta) come from rope_cs (within 2^-21.4 absolute); the other
// bases are one complex product each. Along a lane's 8 tokens the rotation
// then stays within about 1.5e-6 of the exact one, far below one bf16 ulp of
// the rotated key (2^-8 relative).
constexpr int kSumStages = 2;
constexpr int kSumCtasPerSm = 5;
constexpr int kSumG = 4;                                  // groups per chunk = warps per CTA
constexpr int kSumRows = kSumG * kGroupRows;              // 64 rows per chunk
constexpr int kSumChunkBytes = kSumRows * 128 * 2;        // 16 KiB of bf16 key rows
constexpr int kSumThreads = 32 * kSumG;

// Rotations (cos, sin) of the 64 pairs, laid out [q][u] as float4
// (cos e, cos e+1, sin e, sin e+1) of the pairs e = 4u + 2q and e + 1, ready
// for the packed fp32x2 operations: lane u's slots are [0][u] and [1][u].
struct __align__(16) PairRot {
    float4 s[2][16];
};
enum SumExtra { kX16 = 0, kX32, kX48, kXGroupMean, kXChunkMean, kSumExtras };

struct __align__(16) SumShared {
    PairRot ext[kSumExtras];       // R(16 theta), R(32 theta), R(48 theta), R(7.5 theta), R(31.5 theta)
    PairRot base[2][kSumG];        // per item parity, group k: R((c0 + 16k) theta)
    float gsum[2][kSumG][128];     // per item parity: raw group sums (chunk-sum input)
    uint64_t full[kSumStages];
    int abort;
};
constexpr int kSumSmemBytes = kSumStages * kSumChunkBytes + (int)sizeof(SumShared);
static_assert(kSumCtasPerSm * (kSumSmemBytes + 1024) <= 228 * 1024, "CTAs per SM");

bool summaries_stream_supports(const Params& p) {
    // F a multiple of 4: each lane's 4 pairs are all high- or all low-frequency
    return p.dtype == HGA_BF16 && p.d == 128 && p.G == kSumG && p.C == kSumRows && p.F % 4 == 0;
}

__device__ __forceinline__ float2 get_cs(const PairRot& t, int pr) {
    const float* v = reinterpret_cast<const float*>(&t.s[(pr & 3) >> 1][pr >> 2]);
    return make_float2(v[pr & 1], v[2 + (pr & 1)]);
}
__device__ __forceinline__ void put_cs(PairRot& t, int pr, float2 cs) {
    float* v = reinterpret_cast<float*>(&t.s[(pr & 3) >> 1][pr >> 2]);
    v[pr & 1] = cs.x;
    v[2 + (pr & 1)] = cs.y;
}
// R(x) R(y) = R(x + y) on (cos, sin) pairs
__device__ __forceinline__ float2 rot_mul(float2 x, float2 y) {
    return make_float2(x.x * y.x - x.y * y.y, x.y * y.x + x.x * y.y);
}
// (cos, sin) of a small angle a (|a| < 2^20): reduced to [-pi, pi] in double,
// split into a float head and the float remainder, the library sincosf of
// the head corrected to first order by the remainder (the remainder's square,
// below 2^-44, is dropped), so the cast to float costs no accuracy.
__device__ __forceinline__ float2 cs_accurate(double a) {
    const double red = fma(-rint(a * 0.15915494309189535), 6.283185307179586, a);
    const float hi = (float)red, lo = (float)(red - (double)hi);
    float c, sn;
    sincosf(hi, &sn, &c);
    return make_float2(fmaf(-sn, lo, c), fmaf(c, lo, sn));
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t x) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
}
__device__ __forceinline__ uint32_t f2_to_bf16x2(float2 v) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void store_pair2(float* out, float x0, float x1) {
    *reinterpret_cast<float2*>(out) = make_float2(x0, x1);
}
__device__ __forceinline__ void store_pair2(__nv_bfloat16* out, float x0, float x1) {
    *reinterpret_cast<__nv_bfloat162*>(out) = __floats2bfloat162_rn(x0, x1);
}
__device__ __forceinline__ void store_one(float* out, float x) { *out = x; }
__device__ __forceinline__ void store_one(__nv_bfloat16* out, float x) {
    *out = __float2bfloat16_rn(x);
}

// Summary value of pair pr from its raw sums (times 1/n): the mean; the
// low-frequency pairs (pr >= F) are then rotated by `mean_rot`, the rotation
// to the mean position.
__device__ __forceinline__ void summary_pair(const Params& p, int pr, float sa, float sb,
                                             float inv_n, float2 mean_rot, float& oa,
                                             float& ob) {
    const float ma = sa * inv_n, mb = sb * inv_n;
    if (pr < p.F) {
        oa = ma;
        ob = mb;
    } else {
        oa = ma * mean_rot.x - mb * mean_rot.y;
        ob = ma * mean_rot.y + mb * mean_rot.x;
    }
}

// Rotation to the mean position of n tokens from `first`: from the table
// for a full group / chunk, else from rope_cs (only the ragged last chunk).
__device__ __forceinline__ float2 mean_rotation(const Params& p, int pr, int64_t first, int n,
                                                int full_n, float2 base, float2 ext) {
    if (n == full_n) return rot_mul(base, ext);
    float c, sn;
    rope_cs((double)first + 0.5 * (double)(n - 1), p.inv_freq[pr], c, sn);
    return make_float2(c, sn);
}

template <typename S>
__global__ void __launch_bounds__(kSumThreads, kSumCtasPerSm) summaries_stream_kernel(
    Params p, const __nv_bfloat16* __restrict__ k_raw, S* __restrict__ cs, S* __restrict__ gs,
    __nv_bfloat16* __restrict__ k_rot, int chunk_begin, int n_chunks) {
    using namespace ptx;
    extern __shared__ __align__(16) uint8_t stages[];  // bulk copies need 16-byte alignment
    SumShared& sh = *reinterpret_cast<SumShared*>(stages + kSumStages * kSumChunkBytes);
    const int tid = threadIdx.x, lane = tid & 31, k = tid >> 5;
    const int r = lane >> 4, u = lane & 15;
    // item cursor (sequence x KV head, chunk offset), stepped by the grid
    // size without a division per item (B * Hkv * n_chunks < 2^31)
    struct Cursor {
        int bh, off;
    };
    const int n_bh = p.B * p.Hkv;
    const int g_div = (int)gridDim.x / n_chunks, g_mod = (int)gridDim.x % n_chunks;
    auto advance = [&](Cursor c) -> Cursor {
        c.off += g_mod;
        c.bh += g_div;
        if (c.off >= n_chunks) {
            c.off -= n_chunks;
            ++c.bh;
        }
        return c;
    };
    auto rows_of = [&](int ch) -> int {
        const int64_t left = (int64_t)p.L - (int64_t)ch * kSumRows;
        return left >= kSumRows ? kSumRows : (int)left;  // >= 1: ch < nC
    };
    // one bulk copy per item (local index j): its rows are contiguous in [B*Hkv, L, d]
    auto issue = [&](Cursor c, int j) {
        if (c.bh >= n_bh) return;
        const int ch = chunk_begin + c.off;
        const uint32_t bytes = (uint32_t)rows_of(ch) * 256u;
        uint64_t* bar = &sh.full[j % kSumStages];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stages + (j % kSumStages) * kSumChunkBytes,
                 k_raw + ((int64_t)c.bh * p.L + (int64_t)ch * kSumRows) * 128, bytes, bar);
    };
    // group bases of an item: thread (pair pr, half h) forms R((c0 + 32h) theta)
    // and its product with R(16 theta)
    auto make_base = [&](Cursor c, int parity) {
        if (c.bh >= n_bh) return;
        const int ch = chunk_begin + c.off;
        const int pr = tid & 63, h = tid >> 6;
        float c_, sn;
        rope_cs((double)((int64_t)ch * kSumRows + 2 * kGroupRows * h), p.inv_freq[pr], c_, sn);
        const float2 b0 = make_float2(c_, sn);
        put_cs(sh.base[parity][2 * h], pr, b0);
        put_cs(sh.base[parity][2 * h + 1], pr, rot_mul(b0, get_cs(sh.ext[kX16], pr)));
    };

    const Cursor first = {(int)blockIdx.x / n_chunks, (int)blockIdx.x % n_chunks};
    Cursor iss = first;  // thread 0: the next item to issue
    if (tid == 0) {
        for (int s = 0; s < kSumStages; ++s) mbar_init(&sh.full[s], 1);
        fence_mbar_init();
        sh.abort = 0;
        for (int j = 0; j < kSumStages; ++j) {
            issue(iss, j);
            iss = advance(iss);
        }
    }
    // the first copies are in flight while the constants are formed
    for (int i = tid; i < kSumExtras * 64; i += kSumThreads) {
        const int x = i >> 6, pr = i & 63;
        const double m = x <= kX48 ? 16.0 * (x + 1) : (x == kXGroupMean ? 7.5 : 31.5);
        put_cs(sh.ext[x], pr, cs_accurate(m * p.inv_freq[pr]));
    }
    // this lane's step R(2 theta) and first-token offset R(r theta), pairs
    // (4u, 4u+1) in [0] and (4u+2, 4u+3) in [1]
    float2 stc[2], sts[2], ofc[2], ofs[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const float2 s0 = cs_accurate(2.0 * p.inv_freq[4 * u + 2 * q]);
        const float2 s1 = cs_accurate(2.0 * p.inv_freq[4 * u + 2 * q + 1]);
        const float2 o0 = cs_accurate((double)r * p.inv_freq[4 * u + 2 * q]);
        const float2 o1 = cs_accurate((double)r * p.inv_freq[4 * u + 2 * q + 1]);
        stc[q] = make_float2(s0.x, s1.x);
        sts[q] = make_float2(s0.y, s1.y);
        ofc[q] = make_float2(o0.x, o1.x);
        ofs[q] = make_float2(o0.y, o1.y);
    }
    __syncthreads();  // ext (make_base reads it)
    make_base(first, 0);
    __syncthreads();

    const bool write_rot = k_rot != nullptr;
    const bool hi = 4 * u < p.F;  // all 4 of this lane's pairs rotate before averaging
    Cursor cur = first, nxt = advance(first);
    for (int j = 0; cur.bh < n_bh; ++j, cur = nxt, nxt = advance(nxt)) {
        const int64_t bh = cur.bh;
        const int ch = chunk_begin + cur.off;
        const int64_t c0 = (int64_t)ch * kSumRows;
        const int nrows = rows_of(ch);
        const int st = j % kSumStages;
        const bool ok = mbar_wait_bounded(&sh.full[st], (uint32_t)(j / kSumStages) & 1u,
                                          p.wait_ns);
        if (!ok) {
            *reinterpret_cast<volatile int*>(&sh.abort) = 1;
            raise_timeout(p);
        }
        make_base(nxt, (j + 1) & 1);

        float2 acc0[2], acc1[2];  // raw sums of pairs (4u + 2q, +1): a half, b half
#pragma unroll
        for (int q = 0; q < 2; ++q) acc0[q] = acc1[q] = make_float2(0.f, 0.f);
        const PairRot& bk = sh.base[j & 1][k];
        if (ok) {
            const uint8_t* sb = stages + st * kSumChunkBytes;
            // rotation of this lane's first token: R((c0 + 16k) theta) R(r theta)
            float2 rc[2], rs[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float4 b4 = bk.s[q][u];
                const float2 bc = make_float2(b4.x, b4.y), bs = make_float2(b4.z, b4.w);
                rc[q] = sub2(mul2(bc, ofc[q]), mul2(bs, ofs[q]));
                rs[q] = fma2(bs, ofc[q], mul2(bc, ofs[q]));
            }
            __nv_bfloat16* orow = k_rot + (bh * p.L + c0 + kGroupRows * k + r) * 128 + 4 * u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int o = kGroupRows * k + 2 * i + r;
                if (o < nrows) {
                    const uint2 va = *reinterpret_cast<const uint2*>(sb + o * 256 + u * 8);
                    const uint2 vb = *reinterpret_cast<const uint2*>(sb + o * 256 + 128 + u * 8);
                    const float2 av[2] = {bf16x2_to_f2(va.x), bf16x2_to_f2(va.y)};
                    const float2 bv[2] = {bf16x2_to_f2(vb.x), bf16x2_to_f2(vb.y)};
                    float2 xa[2], xb[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        xa[q] = sub2(mul2(av[q], rc[q]), mul2(bv[q], rs[q]));
                        xb[q] = fma2(av[q], rs[q], mul2(bv[q], rc[q]));
                        if (hi) {
                            acc0[q] = add2(acc0[q], xa[q]);
                            acc1[q] = add2(acc1[q], xb[q]);
                        } else {
                            acc0[q] = add2(acc0[q], av[q]);
                            acc1[q] = add2(acc1[q], bv[q]);
                        }
                    }
                    if (write_rot) {
                        *reinterpret_cast<uint2*>(orow + 2 * 128 * i) =
                            make_uint2(f2_to_bf16x2(xa[0]), f2_to_bf16x2(xa[1]));
                        *reinterpret_cast<uint2*>(orow + 2 * 128 * i + 64) =
                            make_uint2(f2_to_bf16x2(xb[0]), f2_to_bf16x2(xb[1]));
                    }
                }
                if (i < 7) {  // on to token o + 2
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float2 nc = sub2(mul2(rc[q], stc[q]), mul2(rs[q], sts[q]));
                        rs[q] = fma2(rs[q], stc[q], mul2(rc[q], sts[q]));
                        rc[q] = nc;
                    }
                }
            }
        }
        // group sums: reduce-scatter over r (lane bit 4); lane (r, u) ends
        // with the pairs 4u + 2r and 4u + 2r + 1
        const float2 ka = r ? acc0[1] : acc0[0], sa_ = r ? acc0[0] : acc0[1];
        const float2 kb = r ? acc1[1] : acc1[0], sb_ = r ? acc1[0] : acc1[1];
        const float2 ya = add2(ka, make_float2(__shfl_xor_sync(0xffffffffu, sa_.x, 16),
                                               __shfl_xor_sync(0xffffffffu, sa_.y, 16)));
        const float2 yb = add2(kb, make_float2(__shfl_xor_sync(0xffffffffu, sb_.x, 16),
                                               __shfl_xor_sync(0xffffffffu, sb_.y, 16)));
        {
            const int pr = 4 * u + 2 * r;
            const int left = nrows - kGroupRows * k;
            const int n = left <= 0 ? 0 : (left >= kGroupRows ? kGroupRows : left);
            float oa0 = 0.f, ob0 = 0.f, oa1 = 0.f, ob1 = 0.f;
            if (n > 0) {
                const float inv_n = __frcp_rn((float)n);
                const int64_t g0 = c0 + kGroupRows * k;
                const float4 bb = bk.s[r][u], xx = sh.ext[kXGroupMean].s[r][u];
                summary_pair(p, pr, ya.x, yb.x, inv_n,
                             mean_rotation(p, pr, g0, n, kGroupRows, make_float2(bb.x, bb.z),
                                           make_float2(xx.x, xx.z)),
                             oa0, ob0);
                summary_pair(p, pr + 1, ya.y, yb.y, inv_n,
                             mean_rotation(p, pr + 1, g0, n, kGroupRows, make_float2(bb.y, bb.w),
                                           make_float2(xx.y, xx.w)),
                             oa1, ob1);
            }
            S* out = gs + ((bh * p.nC + ch) * kSumG + k) * (int64_t)128;
            store_pair2(out + pr, oa0, oa1);
            store_pair2(out + 64 + pr, ob0, ob1);
            *reinterpret_cast<float2*>(&sh.gsum[j & 1][k][pr]) = ya;
            *reinterpret_cast<float2*>(&sh.gsum[j & 1][k][64 + pr]) = yb;
        }
        __syncthreads();  // stage st read; gsum[j & 1] and base[(j + 1) & 1] written
        if (*reinterpret_cast<volatile int*>(&sh.abort)) {
            // every thread saw the flag after the same barrier: retire the
            // copies still in flight (this item's and the ones issued ahead)
            if (tid == 0) {
                Cursor c = cur;
                for (int jj = j; jj < j + kSumStages && c.bh < n_bh; ++jj, c = advance(c))
                    mbar_drain(&sh.full[jj % kSumStages], jj / kSumStages);
            }
            return;
        }
        if (tid == 0) {
            issue(iss, j + kSumStages);
            iss = advance(iss);
        }
        if (tid < 64) {
            float sa = 0.f, sb2 = 0.f;
#pragma unroll
            for (int kk = 0; kk < kSumG; ++kk) {
                sa += sh.gsum[j & 1][kk][tid];
                sb2 += sh.gsum[j & 1][kk][64 + tid];
            }
            float oa, ob;
            summary_pair(p, tid, sa, sb2, __frcp_rn((float)nrows),
                         mean_rotation(p, tid, c0, nrows, kSumRows, get_cs(sh.base[j & 1][0], tid),
                                       get_cs(sh.ext[kXChunkMean], tid)),
                         oa, ob);
            S* out = cs + (bh * p.nC + ch) * (int64_t)128;
            store_one(out + tid, oa);
            store_one(out + 64 + tid, ob);
        }
    }
}

cudaError_t launch_rope(const Params& p, const void* x, void* y, int64_t n_outer,
                        int64_t n_tokens, int n_heads, int64_t pos0, cudaStream_t st) {
    int64_t rows = n_outer * n_tokens * n_heads;
    if (rows == 0) return cudaSuccess;
    const int V = p.dtype == HGA_BF16 ? 8 : 4;
    int64_t work = rows * (p.d / 2 / V);
    int64_t blocks = (work + 255) / 256;
    int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
    if (p.dtype == HGA_BF16)
        rope_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            p, (const __nv_bfloat16*)x, (__nv_bfloat16*)y, rows, n_tokens, n_heads, pos0);
    else
        rope_kernel<float><<<grid, 256, 0, st>>>(p, (const float*)x, (float*)y, rows, n_tokens,
                                                  n_heads, pos0);
    return cudaGetLastError();
}

cudaError_t launch_summaries(const Params& p, const void* k_raw, void* chunk_sum,
                             void* group_sum, void* k_rot, int chunk_begin, int chunk_end,
                             cudaStream_t st) {
    int n = chunk_end - chunk_begin;
    if (n <= 0) return cudaSuccess;
    using bf = __nv_bfloat16;
    const int64_t items = (int64_t)p.B * p.Hkv * n;
    if (summaries_stream_supports(p) && items <= INT32_MAX) {
        const void* fn = p.sum_bf16 ? (const void*)summaries_stream_kernel<bf>
                                    : (const void*)summaries_stream_kernel<float>;
        cudaError_t e =
            set_func_attr_once(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSumSmemBytes);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cudaErrorInvalidValue;
        // kSumCtasPerSm CTAs per SM (their shared memory fits); each walks its items
        const int64_t slots = (int64_t)kSumCtasPerSm * sms;
        const int grid = (int)(items < slots ? items : slots);
        if (p.sum_bf16)
            summaries_stream_kernel<bf><<<grid, kSumThreads, kSumSmemBytes, st>>>(
                p, (const bf*)k_raw, (bf*)chunk_sum, (bf*)group_sum, (bf*)k_rot, chunk_begin, n);
        else
            summaries_stream_kernel<float><<<grid, kSumThreads, kSumSmemBytes, st>>>(
                p, (const bf*)k_raw, (float*)chunk_sum, (float*)group_sum, (bf*)k_rot,
                chunk_begin, n);
        return cudaGetLastError();
    }
    const int V = p.dtype == HGA_BF16 ? 8 : 4;
    int threads = (p.d / 2 / V) * 4 * p.G;
    dim3 grid(n, p.B * p.Hkv);
    if (p.dtype == HGA_BF16) {
        if (p.sum_bf16)
            summaries_kernel<bf, bf><<<grid, threads, 0, st>>>(
                p, (const bf*)k_raw, (bf*)chunk_sum, (bf*)group_sum, (bf*)k_rot, chunk_begin);
        else
            summaries_kernel<bf, float><<<grid, threads, 0, st>>>(
                p, (const bf*)k_raw, (float*)chunk_sum, (float*)group_sum, (bf*)k_rot, chunk_begin);
    } else {
        if (p.sum_bf16)
            summaries_kernel<float, bf><<<grid, threads, 0, st>>>(
                p, (const float*)k_raw, (bf*)chunk_sum, (bf*)group_sum, (float*)k_rot, chunk_begin);
        else
            summaries_kernel<float, float><<<grid, threads, 0, st>>>(
                p, (const float*)k_raw, (float*)chunk_sum, (float*)group_sum, (float*)k_rot,
                chunk_begin);
    }
    return cudaGetLastError();
}

}  // namespace hga
