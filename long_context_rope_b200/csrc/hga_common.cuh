// hga_common.cuh -- shared device helpers of the HGA kernels (sm_100a).
//
// The kernel-side view of an hga_config (Params), the forced-chunk rule of
// "Kernmechanisme" item 2 (Deterministische Zichtbaarheid), RoPE angles, the
// orderable key used by every top-k, and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hga.h"

namespace hga {

constexpr int kMaxHalfDim = 64;      // head_dim <= 128
constexpr int kGroupRows = 16;       // g = C / G: one group = 16 token rows
constexpr int kMaxForced = 64;       // n_sink + n_local + 1 chunks at most

// Kernel-side copy of the configuration, passed by value.
struct Params {
    int B, L, Hq, Hkv, d, C, G, g, gq;
    int n_sink, n_local, kc, kg, F;
    int nC, q_begin, q_len, j0, nQC;
    int dtype, kv_layout;
    int sum_bf16;                  // summary tables stored as bf16 (else fp32)
    int Hu;                        // routing units per sequence: Hkv, or Hq (per query head);
                                   // gq = query heads per unit; unit h reads KV head
                                   // h / (Hu / Hkv)
    int kv_f8;                     // K/V stored as E4M3 codes (else dtype)
    int kv_es;                     // bytes per K/V element
    float k_scale, v_scale;        // E4M3 code scales (1 otherwise)
    int* err;                      // device error word, never NULL
    unsigned long long wait_ns;    // limit of each bounded device wait
    double inv_freq[kMaxHalfDim];  // rope_theta^(-2i/d), computed on the host in double
};

// Codes written to the device error word. An invalid-entry code (1..3) is
// recorded only while the word is 0 (the first one wins); a timeout (4)
// always overwrites it, so a launch that gave up reports that.
enum DevError : int {
    kDevErrNone = 0,
    kDevErrChunkIndex = 1,   // a chunk selection entry out of range / forced / not ascending
    kDevErrGroupIndex = 2,   // a group selection entry out of range / forced / not ascending
    kDevErrCount = 3,        // a selection count above its k
    kDevErrTimeout = 4,      // a bounded wait gave up
};

__device__ __forceinline__ void raise_dev_error(const Params& p, int code) {
    atomicCAS(p.err, 0, code);
}

__device__ __forceinline__ void raise_timeout(const Params& p) {
    atomicExch(p.err, (int)kDevErrTimeout);
}

// Forced chunks of query chunk j in ascending order without duplicates:
// sinks [0, min(n_sink, j+1)) then locals [max(end of sinks, j - n_local), j].
__host__ __device__ __forceinline__ int forced_chunks(const Params& p, int j, int* out) {
    int n = 0;
    int s_end = p.n_sink < j + 1 ? p.n_sink : j + 1;
    for (int c = 0; c < s_end; ++c) out[n++] = c;
    int l_begin = j - p.n_local > s_end ? j - p.n_local : s_end;
    for (int c = l_begin; c <= j; ++c) out[n++] = c;
    return n;
}

__host__ __device__ __forceinline__ bool is_forced(const Params& p, int j, int c) {
    return c == j || (c >= 0 && c < p.n_sink && c <= j) || (c < j && c >= j - p.n_local);
}

// cos / sin of position * inv_freq. The product is formed and reduced to
// [-pi, pi] in double (Cody-Waite style reduction by 2*pi); the fast
// hardware __sincosf of the reduced angle is then within 2^-21.4 absolute
// (its documented bound on [-pi, pi]), a few 1e-7 of a rotated value.
__device__ __forceinline__ void rope_cs(double pos, double inv_freq, float& c, float& s) {
    double a = pos * inv_freq;
    double k = rint(a * 0.15915494309189535);
    double r = fma(-k, 6.283185307179586, a);
    __sincosf((float)r, &s, &c);
}

// The first 1024-byte-aligned shared address at or after p (dynamic shared
// memory), formed by pointer arithmetic on p so that the compiler still knows
// every access through the result is a shared-memory access (a round trip
// through an integer would make them generic accesses).
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// 8 bf16 <-> 8 floats through one 16-byte vector.
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

}  // namespace hga
