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
    const int V = p.dtype == HGA_BF16 ? 8 : 4;
    int threads = (p.d / 2 / V) * 4 * p.G;
    dim3 grid(n, p.B * p.Hkv);
    using bf = __nv_bfloat16;
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
