// hga_api.cu -- the C ABI of libhga.so: host-side validation and dispatch.
//
// Every entry point validates its arguments on the host, builds the
// kernel-side Params, and enqueues kernels on the caller's stream. Nothing
// is allocated. State: per device, the error word (a file-scope __device__
// int) and the fixed scratch array of hga_gather_kv_warm_noalloc, whose
// addresses are looked up once per device; on the host, which kernel
// attributes have been set on which device.
#include <math.h>
#include <stddef.h>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

#include "hga.h"
#include "hga_kernels.h"

namespace hga {
namespace {

__device__ int g_error_word = 0;

constexpr int kMaxDevices = 64;
int* g_err_addr[kMaxDevices] = {};
std::mutex g_err_mutex;

// Address of this device's error word (looked up once per device).
hga_status error_word(int** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_err_mutex);
    if (g_err_addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return HGA_ERR_CUDA;
        g_err_addr[dev] = static_cast<int*>(ptr);
    }
    *out = g_err_addr[dev];
    return HGA_OK;
}

// Scratch of hga_gather_kv_warm_noalloc: the source list that the warm
// tier's plan kernel writes and its copy kernel reads, one int32 per
// (sequence, KV head, selection slot). 65536 entries (256 KiB), held by every
// GPU that loads the library until exit. Each call writes every entry it
// reads first, so nothing here needs a starting value. In host code the name
// g_warm_scratch is only a handle for the runtime, never a pointer to give a
// kernel: warm_scratch() returns the device address.
constexpr int64_t kWarmScratchEntries = 65536;
static __device__ __align__(256) int32_t g_warm_scratch[kWarmScratchEntries];
int32_t* g_warm_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_warm_scratch on the current device (looked up once per
// device, with that device current).
hga_status warm_scratch(int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_warm_scratch_addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_warm_scratch) != cudaSuccess) return HGA_ERR_CUDA;
        g_warm_scratch_addr[dev] = static_cast<int32_t*>(ptr);
    }
    *out = g_warm_scratch_addr[dev];
    return HGA_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Limit of every bounded device wait of later launches (hga_set_wait_limit_ns).
std::atomic<unsigned long long> g_wait_ns{1000000000ull};


// Checks shared by every call; fills p.
hga_status make_params(const hga_config* c, Params* p) {
    if (c == nullptr) return HGA_ERR_NULL;
    if (c->dtype != HGA_BF16 && c->dtype != HGA_F32) return HGA_ERR_CONFIG;
    if (c->batch < 1 || c->seq_len < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1)
        return HGA_ERR_SHAPE;
    if (c->n_q_heads % c->n_kv_heads) return HGA_ERR_SHAPE;
    if (c->head_dim != 64 && c->head_dim != 128) return HGA_ERR_UNSUPPORTED;
    if (c->groups_per_chunk < 1 || c->groups_per_chunk > 8) return HGA_ERR_UNSUPPORTED;
    if (c->chunk_size != kGroupRows * c->groups_per_chunk) return HGA_ERR_UNSUPPORTED;
    {
        const int v = c->dtype == HGA_BF16 ? 8 : 4;
        if (((c->head_dim / 2 / v) * 4 * c->groups_per_chunk) % 32) return HGA_ERR_UNSUPPORTED;
    }
    if (c->n_sink < 0 || c->n_local < 0 || c->n_sink + c->n_local + 1 > kMaxForced)
        return HGA_ERR_CONFIG;
    if (c->top_k_chunks < 1 || c->top_k_chunks > 1024) return HGA_ERR_CONFIG;
    if (c->top_k_groups < 1) return HGA_ERR_CONFIG;
    if ((int64_t)c->groups_per_chunk * (c->n_sink + c->n_local + 1) + c->top_k_groups > kMaxBlocks)
        return HGA_ERR_UNSUPPORTED;
    if (c->n_high_freq_pairs < 0 || c->n_high_freq_pairs > c->head_dim / 2) return HGA_ERR_CONFIG;
    if (!(c->rope_theta > 1.0) || !isfinite(c->rope_theta)) return HGA_ERR_CONFIG;
    if (c->kv_layout != HGA_KV_FULL && c->kv_layout != HGA_KV_WINDOWS) return HGA_ERR_CONFIG;
    if (c->summary_type != HGA_SUMMARY_F32 && c->summary_type != HGA_SUMMARY_BF16)
        return HGA_ERR_CONFIG;
    if (c->kv_type != HGA_KV_AS_DTYPE && c->kv_type != HGA_KV_E4M3) return HGA_ERR_CONFIG;
    if (c->routing != HGA_ROUTE_PER_KV_HEAD && c->routing != HGA_ROUTE_PER_Q_HEAD)
        return HGA_ERR_CONFIG;
    if (c->kv_type == HGA_KV_E4M3) {
        if (!(c->k_scale > 0.0f) || !isfinite(c->k_scale) || !(c->v_scale > 0.0f) ||
            !isfinite(c->v_scale))
            return HGA_ERR_CONFIG;
        if (c->dtype != HGA_BF16 || c->head_dim != 128) return HGA_ERR_UNSUPPORTED;
    }
    if (c->q_begin < 0 || c->q_len < 0 || (int64_t)c->q_begin + c->q_len > c->seq_len)
        return HGA_ERR_SHAPE;
    const int64_t nC = ((int64_t)c->seq_len + c->chunk_size - 1) / c->chunk_size;
    if (nC > kMaxChunks) return HGA_ERR_UNSUPPORTED;

    p->B = c->batch;
    p->L = c->seq_len;
    p->Hq = c->n_q_heads;
    p->Hkv = c->n_kv_heads;
    p->d = c->head_dim;
    p->C = c->chunk_size;
    p->G = c->groups_per_chunk;
    p->g = kGroupRows;
    const bool per_q = c->routing == HGA_ROUTE_PER_Q_HEAD;
    p->Hu = per_q ? c->n_q_heads : c->n_kv_heads;
    p->gq = per_q ? 1 : c->n_q_heads / c->n_kv_heads;
    p->n_sink = c->n_sink;
    p->n_local = c->n_local;
    p->kc = c->top_k_chunks;
    p->kg = c->top_k_groups;
    p->F = c->n_high_freq_pairs;
    p->nC = (int)nC;
    p->q_begin = c->q_begin;
    p->q_len = c->q_len;
    p->j0 = c->q_begin / c->chunk_size;
    p->nQC = c->q_len > 0 ? (c->q_begin + c->q_len - 1) / c->chunk_size - p->j0 + 1 : 0;
    p->dtype = c->dtype;
    p->kv_layout = c->kv_layout;
    p->sum_bf16 = c->summary_type == HGA_SUMMARY_BF16 ? 1 : 0;
    p->kv_f8 = c->kv_type == HGA_KV_E4M3 ? 1 : 0;
    p->kv_es = p->kv_f8 ? 1 : (c->dtype == HGA_BF16 ? 2 : 4);
    p->k_scale = p->kv_f8 ? c->k_scale : 1.0f;
    p->v_scale = p->kv_f8 ? c->v_scale : 1.0f;
    for (int i = 0; i < kMaxHalfDim; ++i)
        p->inv_freq[i] = i < c->head_dim / 2
                             ? pow(c->rope_theta, -2.0 * (double)i / (double)c->head_dim)
                             : 0.0;
    p->err = nullptr;
    p->wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    return HGA_OK;
}

// The last failed CUDA call of this thread that made a call return HGA_ERR_CUDA.
thread_local int g_last_cuda_error = 0;

hga_status cuda_failed(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return HGA_ERR_CUDA;
}

hga_status launched(cudaError_t e) { return e == cudaSuccess ? HGA_OK : cuda_failed(e); }

// Last step before any launch: attach the current device's error word. (A
// call's stream must belong to the current device; that is the caller's
// rule, not checked here: a stream query is not allowed while the stream is
// being captured into a CUDA graph.)
#define HGA_ATTACH_ERR(p)                                  \
    do {                                                   \
        hga_status es_ = error_word(&(p).err);             \
        if (es_ != HGA_OK) return es_;                     \
    } while (0)

}  // namespace
}  // namespace hga

namespace hga {

cudaError_t current_device_index(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return cudaErrorInvalidDevice;
    return (*dev >= 0 && *dev < kMaxDevicesPerProcess) ? cudaSuccess : cudaErrorInvalidDevice;
}

cudaError_t set_func_attr_once(const void* fn, cudaFuncAttribute attr, int value) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, int>, int> done;
    int dev = 0;
    cudaError_t e = current_device_index(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_tuple(dev, fn, (int)attr);
    std::lock_guard<std::mutex> lock(mu);
    const auto it = done.find(key);
    if (it != done.end() && it->second == value) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, attr, value);
    if (e == cudaSuccess) done[key] = value;
    return e;
}

}  // namespace hga

using namespace hga;

static_assert(sizeof(hga_config) == 96, "hga_config layout is part of the ABI");
static_assert(offsetof(hga_config, routing) == 88, "hga_config layout is part of the ABI");
static_assert(offsetof(hga_config, summary_type) == 72, "hga_config layout is part of the ABI");
static_assert(offsetof(hga_config, kv_type) == 76, "hga_config layout is part of the ABI");
static_assert(offsetof(hga_config, v_scale) == 84, "hga_config layout is part of the ABI");
static_assert(offsetof(hga_config, rope_theta) == 48, "hga_config layout is part of the ABI");

extern "C" {

int32_t hga_version(void) { return 10800; }

int32_t hga_last_cuda_error(void) { return g_last_cuda_error; }

const char* hga_cuda_error_string(int32_t cuda_error) {
    const char* s = cudaGetErrorString((cudaError_t)cuda_error);
    return s != nullptr ? s : "unknown CUDA error";
}

void hga_set_wait_limit_ns(uint64_t limit_ns) {
    g_wait_ns.store(limit_ns == 0 ? 1000000000ull : (unsigned long long)limit_ns,
                    std::memory_order_relaxed);
}

const char* hga_status_string(hga_status s) {
    switch (s) {
        case HGA_OK: return "HGA_OK";
        case HGA_ERR_NULL: return "HGA_ERR_NULL: a required pointer is NULL";
        case HGA_ERR_SHAPE: return "HGA_ERR_SHAPE: sizes inconsistent or out of range";
        case HGA_ERR_ALIGN: return "HGA_ERR_ALIGN: a data pointer is not 16-byte aligned";
        case HGA_ERR_CONFIG: return "HGA_ERR_CONFIG: routing or RoPE parameters invalid";
        case HGA_ERR_CUDA: return "HGA_ERR_CUDA: a CUDA call failed";
        case HGA_ERR_DEVICE_INDEX:
            return "HGA_ERR_DEVICE_INDEX: a kernel met an invalid selection entry";
        case HGA_ERR_TIMEOUT: return "HGA_ERR_TIMEOUT: a bounded device wait gave up";
        case HGA_ERR_UNSUPPORTED: return "HGA_ERR_UNSUPPORTED: combination not implemented";
        case HGA_ERR_MEMORY: return "HGA_ERR_MEMORY: pointer not in the required memory space";
        case HGA_ERR_SCRATCH_LIMIT:
            return "HGA_ERR_SCRATCH_LIMIT: larger than the library's fixed scratch array";
    }
    return "HGA_ERR_UNKNOWN";
}

hga_status hga_apply_rope(const hga_config* cfg, const void* x, void* x_rot, int64_t n_outer,
                          int64_t n_tokens, int32_t n_heads, int64_t pos0, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (n_outer < 0 || n_tokens < 0 || n_heads < 1 || pos0 < 0 || pos0 + n_tokens > INT32_MAX)
        return HGA_ERR_SHAPE;
    if (n_outer * n_tokens * n_heads == 0) return HGA_OK;
    if (x == nullptr || x_rot == nullptr) return HGA_ERR_NULL;
    if (!aligned16(x) || !aligned16(x_rot)) return HGA_ERR_ALIGN;
    HGA_ATTACH_ERR(p);
    return launched(launch_rope(p, x, x_rot, n_outer, n_tokens, n_heads, pos0,
                                (cudaStream_t)stream));
}

hga_status hga_build_summaries(const hga_config* cfg, const void* k_raw, void* chunk_sum,
                               void* group_sum, void* k_rot_out, int32_t chunk_begin,
                               int32_t chunk_end, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (chunk_begin < 0 || chunk_end < chunk_begin || chunk_end > p.nC) return HGA_ERR_SHAPE;
    if (chunk_end == chunk_begin) return HGA_OK;
    if (k_raw == nullptr || chunk_sum == nullptr || group_sum == nullptr) return HGA_ERR_NULL;
    if (!aligned16(k_raw) || !aligned16(chunk_sum) || !aligned16(group_sum) ||
        (k_rot_out && !aligned16(k_rot_out)))
        return HGA_ERR_ALIGN;
    if (k_rot_out && p.kv_f8) return HGA_ERR_UNSUPPORTED;  // rotated keys are written in dtype
    HGA_ATTACH_ERR(p);
    return launched(launch_summaries(p, k_raw, chunk_sum, group_sum, k_rot_out, chunk_begin,
                                     chunk_end, (cudaStream_t)stream));
}

hga_status hga_route_chunks(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                            float* qbar_out, int32_t* sel_chunks, int32_t* n_sel_chunks,
                            float* scores_out, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!q_rot || !chunk_sum || !qbar_out || !sel_chunks || !n_sel_chunks) return HGA_ERR_NULL;
    if (!aligned16(q_rot) || !aligned16(chunk_sum) || !aligned16(qbar_out) ||
        !aligned16(sel_chunks) || !aligned16(n_sel_chunks) || (scores_out && !aligned16(scores_out)))
        return HGA_ERR_ALIGN;
    if (p.sum_bf16) return HGA_ERR_UNSUPPORTED;  // bf16 tables: the one-launch decode path only
    if (p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;  // per query head: the decode step only
    HGA_ATTACH_ERR(p);
    cudaStream_t st = (cudaStream_t)stream;
    if (!route_chunks_fuses_qbar(p)) {
        cudaError_t e = launch_qbar(p, q_rot, qbar_out, st);
        if (e != cudaSuccess) return cuda_failed(e);
    }
    return launched(launch_route_chunks(p, q_rot, qbar_out, (const float*)chunk_sum, sel_chunks,
                                        n_sel_chunks, scores_out, st));
}

hga_status hga_route_groups(const hga_config* cfg, const float* qbar, const void* group_sum,
                            const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                            int32_t* sel_groups, int32_t* n_sel_groups, float* scores_out,
                            void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!qbar || !group_sum || !sel_chunks || !n_sel_chunks || !sel_groups || !n_sel_groups)
        return HGA_ERR_NULL;
    if (!aligned16(qbar) || !aligned16(group_sum) || !aligned16(sel_chunks) ||
        !aligned16(n_sel_chunks) || !aligned16(sel_groups) || !aligned16(n_sel_groups) ||
        (scores_out && !aligned16(scores_out)))
        return HGA_ERR_ALIGN;
    if (p.sum_bf16) return HGA_ERR_UNSUPPORTED;  // bf16 tables: the one-launch decode path only
    if (p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;  // per query head: the decode step only
    HGA_ATTACH_ERR(p);
    return launched(launch_route_groups(p, qbar, (const float*)group_sum, sel_chunks, n_sel_chunks,
                                        sel_groups, n_sel_groups, scores_out,
                                        (cudaStream_t)stream));
}

// Shared checks of hga_route / hga_decode_step (routing outputs).
static hga_status check_route_args(const Params& p, const void* q_rot, const void* chunk_sum,
                                   const void* group_sum, const float* qbar_out,
                                   const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                                   const int32_t* sel_groups, const int32_t* n_sel_groups) {
    (void)p;
    if (!q_rot || !chunk_sum || !group_sum || !qbar_out || !sel_chunks || !n_sel_chunks ||
        !sel_groups || !n_sel_groups)
        return HGA_ERR_NULL;
    if (!aligned16(q_rot) || !aligned16(chunk_sum) || !aligned16(group_sum) ||
        !aligned16(qbar_out) || !aligned16(sel_chunks) || !aligned16(n_sel_chunks) ||
        !aligned16(sel_groups) || !aligned16(n_sel_groups))
        return HGA_ERR_ALIGN;
    return HGA_OK;
}

// The two routing levels as separate kernels.
static hga_status route_separate(const Params& p, const void* q_rot, const void* chunk_sum,
                                 const void* group_sum, float* qbar_out, int32_t* sel_chunks,
                                 int32_t* n_sel_chunks, int32_t* sel_groups,
                                 int32_t* n_sel_groups, cudaStream_t st) {
    if (p.sum_bf16 || p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;  // one-launch path only
    cudaError_t e = route_chunks_fuses_qbar(p) ? cudaSuccess : launch_qbar(p, q_rot, qbar_out, st);
    if (e != cudaSuccess) return cuda_failed(e);
    if (route_tiled_fuses_groups(p))  // prefill: both levels in one launch after q-bar
        return launched(launch_route_chunks_tiled(p, qbar_out, (const float*)chunk_sum, sel_chunks,
                                                  n_sel_chunks, nullptr, st,
                                                  (const float*)group_sum, sel_groups,
                                                  n_sel_groups));
    e = launch_route_chunks(p, q_rot, qbar_out, (const float*)chunk_sum, sel_chunks, n_sel_chunks,
                            nullptr, st);
    if (e != cudaSuccess) return cuda_failed(e);
    return launched(launch_route_groups(p, qbar_out, (const float*)group_sum, sel_chunks,
                                        n_sel_chunks, sel_groups, n_sel_groups, nullptr, st));
}

hga_status hga_route(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                     const void* group_sum, float* qbar_out, int32_t* sel_chunks,
                     int32_t* n_sel_chunks, int32_t* sel_groups, int32_t* n_sel_groups,
                     void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    s = check_route_args(p, q_rot, chunk_sum, group_sum, qbar_out, sel_chunks, n_sel_chunks,
                         sel_groups, n_sel_groups);
    if (s != HGA_OK) return s;
    HGA_ATTACH_ERR(p);
    cudaStream_t st = (cudaStream_t)stream;
    if (decode_step_supports(p))
        return launched(launch_decode_step(p, q_rot, chunk_sum, group_sum, nullptr, nullptr,
                                           qbar_out, sel_chunks, n_sel_chunks, sel_groups,
                                           n_sel_groups, nullptr, st));
    return route_separate(p, q_rot, chunk_sum, group_sum, qbar_out, sel_chunks, n_sel_chunks,
                          sel_groups, n_sel_groups, st);
}

hga_status hga_decode_step(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                           const void* group_sum, const void* k_cache, const void* v_cache,
                           float* qbar_out, int32_t* sel_chunks, int32_t* n_sel_chunks,
                           int32_t* sel_groups, int32_t* n_sel_groups, void* out, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    s = check_route_args(p, q_rot, chunk_sum, group_sum, qbar_out, sel_chunks, n_sel_chunks,
                         sel_groups, n_sel_groups);
    if (s != HGA_OK) return s;
    if (!k_cache || !v_cache || !out) return HGA_ERR_NULL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return HGA_ERR_ALIGN;
    if (p.kv_layout != HGA_KV_FULL) return HGA_ERR_UNSUPPORTED;
    HGA_ATTACH_ERR(p);
    cudaStream_t st = (cudaStream_t)stream;
    if (decode_step_supports(p))
        return launched(launch_decode_step(p, q_rot, chunk_sum, group_sum, k_cache, v_cache,
                                           qbar_out, sel_chunks, n_sel_chunks, sel_groups,
                                           n_sel_groups, out, st));
    if (p.kv_f8 && !decode_kernel_supports(p)) return HGA_ERR_UNSUPPORTED;
    if (p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;  // per query head: one-launch path only
    s = route_separate(p, q_rot, chunk_sum, group_sum, qbar_out, sel_chunks, n_sel_chunks,
                       sel_groups, n_sel_groups, st);
    if (s != HGA_OK) return s;
    KvSources kv{k_cache, v_cache, nullptr, nullptr};
    if (p.kv_f8)
        return launched(launch_attend_decode(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    if (tc_kernel_supports(p, false))
        return launched(launch_attend_tc(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    if (decode_kernel_supports(p))
        return launched(launch_attend_decode(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    return launched(launch_attend_simt(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
}

static hga_status device_view(const void* ptr, bool want_host, const void** dev_ptr);

hga_status hga_decode_step_tiered(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                                  const void* group_sum, const void* k_win, const void* v_win,
                                  const void* k_host, const void* v_host, float* qbar_out,
                                  int32_t* sel_chunks, int32_t* n_sel_chunks, int32_t* sel_groups,
                                  int32_t* n_sel_groups, void* out, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    s = check_route_args(p, q_rot, chunk_sum, group_sum, qbar_out, sel_chunks, n_sel_chunks,
                         sel_groups, n_sel_groups);
    if (s != HGA_OK) return s;
    if (!k_win || !v_win || !k_host || !v_host || !out) return HGA_ERR_NULL;
    if (!aligned16(k_win) || !aligned16(v_win) || !aligned16(k_host) || !aligned16(v_host) ||
        !aligned16(out))
        return HGA_ERR_ALIGN;
    if (p.kv_layout != HGA_KV_WINDOWS || p.q_len != 1 || p.q_begin != p.L - 1 ||
        !decode_step_supports(p))
        return HGA_ERR_UNSUPPORTED;
    HGA_ATTACH_ERR(p);
    const void* kd = nullptr;
    const void* vd = nullptr;
    if ((s = device_view(k_host, true, &kd)) != HGA_OK) return s;
    if ((s = device_view(v_host, true, &vd)) != HGA_OK) return s;
    return launched(launch_decode_step(p, q_rot, chunk_sum, group_sum, k_win, v_win, qbar_out,
                                       sel_chunks, n_sel_chunks, sel_groups, n_sel_groups, out,
                                       (cudaStream_t)stream, kd, vd));
}

static hga_status device_view(const void* ptr, bool want_host, const void** dev_ptr) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();  // clear the error raised for an unknown pointer
        return HGA_ERR_MEMORY;
    }
    if (want_host) {
        if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return HGA_ERR_MEMORY;
        *dev_ptr = a.devicePointer;
    } else {
        if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return HGA_ERR_MEMORY;
        *dev_ptr = ptr;
    }
    return HGA_OK;
}

hga_status hga_gather_kv(const hga_config* cfg, const void* k_src, const void* v_src,
                         int32_t src_is_host, const int32_t* sel_groups,
                         const int32_t* n_sel_groups, void* k_dst, void* v_dst, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!k_src || !v_src || !sel_groups || !n_sel_groups || !k_dst || !v_dst) return HGA_ERR_NULL;
    if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(sel_groups) ||
        !aligned16(n_sel_groups) || !aligned16(k_dst) || !aligned16(v_dst))
        return HGA_ERR_ALIGN;
    if (p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;  // gathers follow per-KV-head lists
    HGA_ATTACH_ERR(p);
    const void* kd = nullptr;
    const void* vd = nullptr;
    if ((s = device_view(k_src, src_is_host != 0, &kd)) != HGA_OK) return s;
    if ((s = device_view(v_src, src_is_host != 0, &vd)) != HGA_OK) return s;
    return launched(launch_gather(p, kd, vd, src_is_host != 0, sel_groups, n_sel_groups, k_dst,
                                  v_dst, (cudaStream_t)stream));
}

hga_status hga_gather_kv_warm(const hga_config* cfg, const void* k_host, const void* v_host,
                              const int32_t* sel_groups, const int32_t* n_sel_groups,
                              void* pool_k, void* pool_v, int32_t* pool_tag, int32_t* pool_last,
                              int32_t n_slots, int32_t step, int32_t* src_out,
                              int32_t* stats_out, void* k_dst, void* v_dst, void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!k_host || !v_host || !sel_groups || !n_sel_groups || !pool_k || !pool_v || !pool_tag ||
        !pool_last || !src_out || !k_dst || !v_dst)
        return HGA_ERR_NULL;
    if (!aligned16(k_host) || !aligned16(v_host) || !aligned16(sel_groups) ||
        !aligned16(n_sel_groups) || !aligned16(pool_k) || !aligned16(pool_v) ||
        !aligned16(pool_tag) || !aligned16(pool_last) || !aligned16(src_out) ||
        !aligned16(k_dst) || !aligned16(v_dst) || (stats_out && !aligned16(stats_out)))
        return HGA_ERR_ALIGN;
    if (p.q_len != 1 || p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;
    if (n_slots < p.kg || step < 0) return HGA_ERR_SHAPE;
    if (!gather_warm_supports(p, n_slots)) return HGA_ERR_UNSUPPORTED;
    HGA_ATTACH_ERR(p);
    const void* kd = nullptr;
    const void* vd = nullptr;
    if ((s = device_view(k_host, true, &kd)) != HGA_OK) return s;
    if ((s = device_view(v_host, true, &vd)) != HGA_OK) return s;
    return launched(launch_gather_warm(p, kd, vd, sel_groups, n_sel_groups, pool_k, pool_v,
                                       pool_tag, pool_last, n_slots, step, src_out, stats_out,
                                       k_dst, v_dst, (cudaStream_t)stream));
}

hga_status hga_gather_kv_warm_noalloc(const hga_config* cfg, const void* k_host,
                                      const void* v_host, const int32_t* sel_groups,
                                      const int32_t* n_sel_groups, void* pool_k, void* pool_v,
                                      int32_t* pool_tag, int32_t* pool_last, int32_t n_slots,
                                      int32_t step, int32_t* stats_out, void* k_dst, void* v_dst,
                                      void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!k_host || !v_host || !sel_groups || !n_sel_groups || !pool_k || !pool_v || !pool_tag ||
        !pool_last || !k_dst || !v_dst)
        return HGA_ERR_NULL;
    if (!aligned16(k_host) || !aligned16(v_host) || !aligned16(sel_groups) ||
        !aligned16(n_sel_groups) || !aligned16(pool_k) || !aligned16(pool_v) ||
        !aligned16(pool_tag) || !aligned16(pool_last) || !aligned16(k_dst) ||
        !aligned16(v_dst) || (stats_out && !aligned16(stats_out)))
        return HGA_ERR_ALIGN;
    if (p.q_len != 1 || p.Hu != p.Hkv) return HGA_ERR_UNSUPPORTED;
    if (n_slots < p.kg || step < 0) return HGA_ERR_SHAPE;
    if (!gather_warm_supports(p, n_slots)) return HGA_ERR_UNSUPPORTED;
    if ((int64_t)p.B * p.Hkv * p.kg > kWarmScratchEntries) return HGA_ERR_SCRATCH_LIMIT;
    HGA_ATTACH_ERR(p);
    int32_t* src = nullptr;
    if ((s = warm_scratch(&src)) != HGA_OK) return s;
    const void* kd = nullptr;
    const void* vd = nullptr;
    if ((s = device_view(k_host, true, &kd)) != HGA_OK) return s;
    if ((s = device_view(v_host, true, &vd)) != HGA_OK) return s;
    return launched(launch_gather_warm(p, kd, vd, sel_groups, n_sel_groups, pool_k, pool_v,
                                       pool_tag, pool_last, n_slots, step, src, stats_out, k_dst,
                                       v_dst, (cudaStream_t)stream));
}

hga_status hga_attend(const hga_config* cfg, const void* q_rot, const void* k_res,
                      const void* v_res, const void* k_gat, const void* v_gat,
                      const int32_t* sel_groups, const int32_t* n_sel_groups, void* out,
                      void* stream) {
    Params p;
    hga_status s = make_params(cfg, &p);
    if (s != HGA_OK) return s;
    if (p.nQC == 0) return HGA_OK;
    if (!q_rot || !k_res || !v_res || !sel_groups || !n_sel_groups || !out) return HGA_ERR_NULL;
    if ((k_gat == nullptr) != (v_gat == nullptr)) return HGA_ERR_NULL;
    if (!aligned16(q_rot) || !aligned16(k_res) || !aligned16(v_res) || !aligned16(sel_groups) ||
        !aligned16(n_sel_groups) || !aligned16(out) || (k_gat && !aligned16(k_gat)) ||
        (v_gat && !aligned16(v_gat)))
        return HGA_ERR_ALIGN;
    if (p.kv_layout == HGA_KV_WINDOWS &&
        (p.q_len != 1 || p.q_begin != p.L - 1 || k_gat == nullptr))
        return HGA_ERR_UNSUPPORTED;
    if (p.kv_f8 && !decode_kernel_supports(p)) return HGA_ERR_UNSUPPORTED;  // decode only
    if (p.Hu != p.Hkv && (!decode_kernel_supports(p) || k_gat != nullptr))
        return HGA_ERR_UNSUPPORTED;  // per query head: decode, index mode
    HGA_ATTACH_ERR(p);
    KvSources kv{k_res, v_res, k_gat, v_gat};
    cudaStream_t st = (cudaStream_t)stream;
    if (p.kv_f8 || p.Hu != p.Hkv)
        return launched(launch_attend_decode(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    if (tc_kernel_supports(p, k_gat != nullptr))
        return launched(launch_attend_tc(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    if (decode_kernel_supports(p))
        return launched(launch_attend_decode(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
    return launched(launch_attend_simt(p, q_rot, kv, sel_groups, n_sel_groups, out, st));
}

hga_status hga_get_device_error(void* stream, int32_t* detail_out) {
    if (detail_out) *detail_out = 0;
    cudaError_t se = cudaStreamSynchronize((cudaStream_t)stream);
    if (se != cudaSuccess) return cuda_failed(se);
    int* addr = nullptr;
    hga_status s = error_word(&addr);
    if (s != HGA_OK) return s;
    int v = 0;
    cudaError_t ce = cudaMemcpy(&v, addr, sizeof(int), cudaMemcpyDeviceToHost);
    if (ce != cudaSuccess) return cuda_failed(ce);
    if (v == 0) return HGA_OK;
    const int zero = 0;
    ce = cudaMemcpy(addr, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (ce != cudaSuccess) return cuda_failed(ce);
    if (detail_out) *detail_out = v;
    return v == kDevErrTimeout ? HGA_ERR_TIMEOUT : HGA_ERR_DEVICE_INDEX;
}

}  // extern "C"
