// hga_kernels.h -- internal launchers behind the C ABI (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hga_common.cuh"

namespace hga {

// Largest number of 16-row key blocks one attention unit may hold:
// G * (n_sink + n_local + 1) forced blocks plus top_k_groups routed ones.
constexpr int kMaxBlocks = 512;
// Largest number of chunks the routing kernels keep in shared memory.
constexpr int kMaxChunks = 16384;
// Devices a process may drive (per-device caches of the launchers).
constexpr int kMaxDevicesPerProcess = 64;

// Set attribute `attr` of kernel `fn` to `value` on the current device, once
// per (device, kernel, attribute, value): kernel attributes belong to the
// kernel as loaded on each device, and a driver call on every launch would
// add host latency to every decode step.
cudaError_t set_func_attr_once(const void* fn, cudaFuncAttribute attr, int value);
// Current device as an index into per-device caches (< kMaxDevicesPerProcess).
cudaError_t current_device_index(int* dev);

cudaError_t launch_rope(const Params& p, const void* x, void* y, int64_t n_outer,
                        int64_t n_tokens, int n_heads, int64_t pos0, cudaStream_t st);

// chunk_sum / group_sum: fp32, or bf16 when p.sum_bf16.
cudaError_t launch_summaries(const Params& p, const void* k_raw, void* chunk_sum,
                             void* group_sum, void* k_rot, int chunk_begin, int chunk_end,
                             cudaStream_t st);

cudaError_t launch_qbar(const Params& p, const void* q_rot, float* qbar, cudaStream_t st);

// Level-1 routing. q-bar must already be in `qbar` unless
// route_chunks_fuses_qbar(p), in which case the kernel forms it from q_rot
// and writes it to `qbar` (few query tokens: decode).
bool route_chunks_fuses_qbar(const Params& p);
cudaError_t launch_route_chunks(const Params& p, const void* q_rot, float* qbar,
                                const float* chunk_sum, int32_t* sel, int32_t* n_sel,
                                float* scores, cudaStream_t st);

// Prefill form of level-1 routing: 8 query chunks per CTA share one pass
// over the chunk-summary table (needs nQC >= 8 and nC <= 2048). With a group
// table (group_sum != nullptr; route_tiled_fuses_groups(p)) the same launch
// also runs level 2 and writes sel_g / n_sel_g, bitwise as launch_route_groups.
bool route_chunks_tiled_supports(const Params& p);
bool route_tiled_fuses_groups(const Params& p);
cudaError_t launch_route_chunks_tiled(const Params& p, const float* qbar, const float* chunk_sum,
                                      int32_t* sel, int32_t* n_sel, float* scores,
                                      cudaStream_t st, const float* group_sum = nullptr,
                                      int32_t* sel_g = nullptr, int32_t* n_sel_g = nullptr);

cudaError_t launch_route_groups(const Params& p, const float* qbar, const float* group_sum,
                                const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                                int32_t* sel_groups, int32_t* n_sel_groups, float* scores,
                                cudaStream_t st);

cudaError_t launch_gather(const Params& p, const void* k_src, const void* v_src, bool from_host,
                          const int32_t* sel_groups, const int32_t* n_sel_groups, void* k_dst,
                          void* v_dst, cudaStream_t st);

// Warm tier for one-token decode: the selected groups into k_dst / v_dst,
// from a VRAM pool of n_slots groups per (sequence, KV head) where present,
// else from the mapped host store (also filling the least recently used
// pool slot). Needs nQC == 1 and top_k_groups <= n_slots <= 4096.
bool gather_warm_supports(const Params& p, int n_slots);
cudaError_t launch_gather_warm(const Params& p, const void* k_host, const void* v_host,
                               const int32_t* sel_groups, const int32_t* n_sel_groups,
                               void* pool_k, void* pool_v, int32_t* pool_tag, int32_t* pool_last,
                               int n_slots, int step, int32_t* src_out, int32_t* stats_out,
                               void* k_dst, void* v_dst, cudaStream_t st);

// Where an attention unit finds its keys.
struct KvSources {
    const void* k_res;  // full store [B,Hkv,L,d] or forced windows [B,Hkv,W*C,d]
    const void* v_res;
    const void* k_gat;  // gathered [B,Hkv,nQC,kg*16,d] or nullptr (index mode)
    const void* v_gat;
};

cudaError_t launch_attend_simt(const Params& p, const void* q_rot, const KvSources& kv,
                               const int32_t* sel_groups, const int32_t* n_sel_groups,
                               void* out, cudaStream_t st);

// True when the tcgen05 prefill kernel covers this configuration (bf16,
// d = 128, 8 query heads per KV head, prefill, full resident store, index mode).
bool tc_kernel_supports(const Params& p, bool gathered);

cudaError_t launch_attend_tc(const Params& p, const void* q_rot, const KvSources& kv,
                             const int32_t* sel_groups, const int32_t* n_sel_groups, void* out,
                             cudaStream_t st);

// True when the cluster / MMA decode kernel covers this configuration
// (bf16, d = 128, one query token, gq <= 8, L % 16 == 0, <= 128 key blocks).
bool decode_kernel_supports(const Params& p);

cudaError_t launch_attend_decode(const Params& p, const void* q_rot, const KvSources& kv,
                                 const int32_t* sel_groups, const int32_t* n_sel_groups,
                                 void* out, cudaStream_t st);

// One-launch decode step (q-bar, both routing levels, attention): bf16,
// d = 128, one query token, gq <= 8, L % 16 == 0, top_k_chunks <= 64,
// top_k_groups <= 512, and routing tables that fit one cluster's shared
// memory. With out == nullptr it stops after routing. The keys come from
// k_cache / v_cache in p.kv_layout: the full resident store, or (with
// k_host / v_host, the full store in mapped host memory) the resident
// windows of the forced chunks, the routed groups then read from the host.
bool decode_step_supports(const Params& p);
// Summary tables fp32, or bf16 when p.sum_bf16.
cudaError_t launch_decode_step(const Params& p, const void* q_rot, const void* chunk_sum,
                               const void* group_sum, const void* k_cache, const void* v_cache,
                               float* qbar, int32_t* sel_chunks, int32_t* n_sel_chunks,
                               int32_t* sel_groups, int32_t* n_sel_groups, void* out,
                               cudaStream_t st, const void* k_host = nullptr,
                               const void* v_host = nullptr);

}  // namespace hga
