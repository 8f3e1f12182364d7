/*
 * hga.h -- C ABI of libhga.so, the B200 (sm_100a) hot path of Hierarchical
 * Global Attention (HGA).
 *
 * The operations follow the statement of the method in "Technische
 * Samenvatting: Hierarchical Global Attention (HGA)" (gist.science), section
 * "Methodologie", subsection "Kernmechanisme", items 1-4, and section
 * "Geheugenarchitectuur" (hot/cold K/V tiers). Where that page is silent the
 * readings are the same as the CPU oracle's:
 *   - RoPE uses half-split pairing: pair i = (dim i, dim i + d/2), frequency
 *     theta_i = rope_theta^(-2i/d), angle = position * theta_i. Pairs
 *     0..n_high_freq_pairs-1 are the high-frequency pairs.
 *   - A token set's representative position is the mean of its positions.
 *   - The routing query of (sequence, KV head, query chunk) is the mean of the
 *     rotated queries over the chunk's query tokens and the KV head's query
 *     heads ("q-bar"); scores are plain fp32 dot products.
 *   - Top-k counts only the non-forced earlier chunks (clamped to what is
 *     available); the group top-k is global over all groups of the chosen
 *     chunks. Ties: higher score first, then lower index; NaN ranks last.
 *     Lists are returned in ascending index order, padded with -1.
 *   - A query at position p attends to the keys of its set at positions <= p.
 *
 * Conventions for every call:
 *   - All pointers are device pointers unless stated otherwise. The caller owns
 *     every buffer and keeps it alive until the stream has passed the call.
 *     Inputs are never modified. The library allocates no memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is only enqueued; nothing blocks the host except
 *     hga_get_device_error. The stream must belong to the current device:
 *     the library's per-device state (error word, scratch array) is looked
 *     up for the current device, and the stream is not queried (a query is
 *     not allowed while the stream is being captured into a CUDA graph).
 *   - Arguments are validated on the host before anything is launched; a call
 *     that returns an error has launched nothing. Every data pointer must be
 *     16-byte aligned.
 *   - Index lists produced by the library are device-side and never copied to
 *     the host. Kernels that read a caller-supplied list check every entry;
 *     an entry out of range, an entry naming a forced chunk, or a list that is
 *     not strictly ascending sets the device error word (read it with
 *     hga_get_device_error) and the entry is skipped: the unit computes over
 *     its remaining keys, and every other unit of the launch, and every later
 *     launch, computes exactly as if the word were clear (the word is only
 *     written by kernels, never read by them). No kernel traps.
 *   - Every device-side wait (a pipeline stage of the attention and gather
 *     kernels) is bounded, by default by 1 s (hga_set_wait_limit_ns). A wait
 *     that runs out records HGA_ERR_TIMEOUT in the device error word (it
 *     overrides an invalid-entry code there), the CTA stops its work, waits
 *     (again bounded) for the copies and tensor-core operations it has
 *     already issued, frees its tensor memory and exits; the output rows of
 *     the units it did not finish are undefined (not written, or computed
 *     from part of the key set).
 *   - Layouts (row-major, innermost last):
 *       queries / outputs   [B, q_len, Hq, d]       (token q_begin + t at row t)
 *       keys / values       [B, Hkv, L, d]          (full store, HGA_KV_FULL)
 *       chunk summaries     [B, Hkv, nC, d]         nC = ceil(L / C)
 *       group summaries     [B, Hkv, nC * G, d]     (fp32 or bf16: summary_type)
 *       q-bar               [B, Hkv, nQC, d] fp32   query chunks of the span
 *       chunk selections    [B, Hkv, nQC, top_k_chunks] int32
 *       group selections    [B, Hkv, nQC, top_k_groups] int32 (global group
 *                           index = chunk * G + group within the chunk)
 *       selection counts    [B, Hkv, nQC] int32
 *       gathered K / V      [B, Hkv, nQC, top_k_groups * g, d], g = C / G
 *     nQC counts the chunks touched by the query span [q_begin, q_begin+q_len).
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HGA_OK = 0,
    HGA_ERR_NULL = -1,         /* a required pointer is NULL */
    HGA_ERR_SHAPE = -2,        /* sizes inconsistent or out of the supported range */
    HGA_ERR_ALIGN = -3,        /* a data pointer is not 16-byte aligned */
    HGA_ERR_CONFIG = -4,       /* routing or RoPE parameters invalid */
    HGA_ERR_CUDA = -5,         /* a CUDA call failed (this launch or an earlier async error) */
    HGA_ERR_DEVICE_INDEX = -6, /* a kernel met an invalid entry in a caller-supplied list */
    HGA_ERR_TIMEOUT = -7,      /* a bounded device-side wait gave up */
    HGA_ERR_UNSUPPORTED = -8,  /* valid arguments, combination not implemented */
    HGA_ERR_MEMORY = -9,       /* a pointer is not in the memory space the call needs */
    HGA_ERR_SCRATCH_LIMIT = -10 /* larger than the library's fixed scratch array */
} hga_status;

typedef enum { HGA_BF16 = 0, HGA_F32 = 1 } hga_dtype;

/* Where hga_attend finds the forced (always visible) chunks.
 * HGA_KV_FULL:    k_res / v_res are the full store [B, Hkv, L, d].
 * HGA_KV_WINDOWS: k_res / v_res hold only the forced chunks of the decode
 *                 query chunk j = (L-1)/C, packed in ascending chunk order:
 *                 [B, Hkv, W * C, d] with W = n_sink + n_local + 1 slots
 *                 (the hot tier of "Geheugenarchitectuur"). Decode only. */
typedef enum { HGA_KV_FULL = 0, HGA_KV_WINDOWS = 1 } hga_kv_layout;

/* Storage type of the chunk and group summary tables (chunk_sum, group_sum).
 * HGA_SUMMARY_F32:  fp32.
 * HGA_SUMMARY_BF16: the fp32 summaries rounded to bf16 (nearest even); half
 *                   the bytes the decode step reads for routing. Routing
 *                   scores are still fp32 dot products (of the rounded
 *                   values). Written by hga_build_summaries; read by
 *                   hga_route and hga_decode_step on their one-launch decode
 *                   path (one query token, bf16, d = 128, gq <= 8, L % 16 ==
 *                   0, top_k_chunks <= 64); every other routing call returns
 *                   HGA_ERR_UNSUPPORTED for it. */
typedef enum { HGA_SUMMARY_F32 = 0, HGA_SUMMARY_BF16 = 1 } hga_summary_type;

/* Storage type of the attention keys and values: the stores (k_res / v_res,
 * k_cache / v_cache, k_win / v_win, k_src / v_src, k_host / v_host), the
 * gathered buffers and the warm-tier pools.
 * HGA_KV_AS_DTYPE: cfg->dtype, like the queries.
 * HGA_KV_E4M3:     one byte per element, an 8-bit floating-point code of the
 *                  E4M3 kind (bit 7 sign, bits 6..3 exponent with bias 7,
 *                  bits 2..0 mantissa; no infinities; 0x7F / 0xFF are NaN):
 *                  the FP8 K/V cache of an FP8 deployment (the setting of
 *                  "Probleemstelling"). An element's value is its code's
 *                  value times cfg->k_scale (keys) or cfg->v_scale (values);
 *                  layouts are the same, with 1-byte elements. Needs dtype
 *                  HGA_BF16 and head_dim 128; queries must lie in the fp16
 *                  range (|q| < 65504: the products run on fp16 tensor-core
 *                  inputs, which hold every E4M3 value exactly). Read by the
 *                  decode calls (hga_attend with q_len == 1, hga_decode_step,
 *                  hga_decode_step_tiered) and moved by the gathers
 *                  (hga_gather_kv, hga_gather_kv_warm[_noalloc]). Prefill
 *                  attention (q_len > 1) and a rotated-key output of
 *                  hga_build_summaries return HGA_ERR_UNSUPPORTED. */
typedef enum { HGA_KV_AS_DTYPE = 0, HGA_KV_E4M3 = 1 } hga_kv_type;

/* Which heads route.
 * HGA_ROUTE_PER_KV_HEAD: one routing query per (sequence, KV head, query
 *     chunk), the q-bar of the conventions above; the KV head's query heads
 *     attend over one shared selection.
 * HGA_ROUTE_PER_Q_HEAD:  one routing query per (sequence, query head, query
 *     chunk): the mean of that head's own rotated queries over the chunk's
 *     query tokens. It scores its KV head's summaries (KV head h / (Hq/Hkv))
 *     and the head attends over its own selection. q-bar, the selection
 *     lists and their counts then have Hq rows where the layouts above say
 *     Hkv ([B, Hq, nQC, ...]). Decode (q_len == 1) only: hga_route,
 *     hga_decode_step and hga_decode_step_tiered on their one-launch path,
 *     and hga_attend in index mode; every other call returns
 *     HGA_ERR_UNSUPPORTED. */
typedef enum { HGA_ROUTE_PER_KV_HEAD = 0, HGA_ROUTE_PER_Q_HEAD = 1 } hga_routing;

typedef struct {
    int32_t batch;             /* B */
    int32_t seq_len;           /* L: tokens in the K/V history (context length) */
    int32_t n_q_heads;         /* Hq */
    int32_t n_kv_heads;        /* Hkv; Hq % Hkv == 0 (GQA) */
    int32_t head_dim;          /* d: 64 or 128 */
    int32_t chunk_size;        /* C ("Kernmechanisme" item 1: fixed chunks, e.g. C=64) */
    int32_t groups_per_chunk;  /* G; group size g = C / G must be 16 */
    int32_t n_sink;            /* initial chunks always visible */
    int32_t n_local;           /* recent chunks before the current one, always visible */
    int32_t top_k_chunks;      /* level-1 k (>= 1) */
    int32_t top_k_groups;      /* level-2 k (>= 1) */
    int32_t n_high_freq_pairs; /* F: pairs 0..F-1 are rotated per token, then averaged */
    double rope_theta;         /* RoPE base (> 1) */
    int32_t dtype;             /* hga_dtype of queries, keys, values and outputs */
    int32_t q_begin;           /* first query position */
    int32_t q_len;             /* number of query tokens (1 = decode) */
    int32_t kv_layout;         /* hga_kv_layout, read by hga_attend only */
    int32_t summary_type;      /* hga_summary_type of the summary tables (0 = fp32) */
    int32_t kv_type;           /* hga_kv_type of keys and values (0 = cfg->dtype) */
    float k_scale;             /* HGA_KV_E4M3: scale of the key codes (finite, > 0) */
    float v_scale;             /* HGA_KV_E4M3: scale of the value codes (finite, > 0) */
    int32_t routing;           /* hga_routing (0 = per KV head) */
} hga_config;

/* Rotate x by RoPE (standard rotary position embedding; the summaries of
 * "Kernmechanisme" item 3 are built on it). x, x_rot: [n_outer, n_tokens,
 * n_heads, d] of cfg->dtype; token t sits at position pos0 + t. x_rot may
 * equal x (in place). Uses cfg->head_dim, rope_theta and dtype only. Typical
 * uses: queries [B, q_len, Hq, d] with pos0 = q_begin; keys [B*Hkv, L, 1, d]
 * with pos0 = 0. */
hga_status hga_apply_rope(const hga_config* cfg, const void* x, void* x_rot, int64_t n_outer,
                          int64_t n_tokens, int32_t n_heads, int64_t pos0, void* stream);

/* RoPE-aware chunk and group key summaries ("Kernmechanisme" item 3) of the
 * chunks [chunk_begin, chunk_end) from the pre-RoPE projected keys k_raw
 * [B, Hkv, L, d]. For a token set S (a group, or a whole chunk) with mean
 * position pbar: pairs i < F get mean_{t in S} R(p_t theta_i) k_t,i; pairs
 * i >= F get R(pbar theta_i) mean_{t in S} k_t,i. Only tokens < L count; an
 * empty group is zero. Writes chunk_sum [B,Hkv,nC,d] and group_sum
 * [B,Hkv,nC*G,d] (fp32) rows of those chunks and, if k_rot_out is not NULL,
 * the rotated keys R(p_t) k_t [B,Hkv,L,d] of their tokens in cfg->dtype (the
 * attention cache). Building chunk by chunk gives bitwise the same result as
 * building all chunks at once. The tables are fp32, or bf16 (each value the
 * fp32 summary rounded to nearest even) when cfg->summary_type is
 * HGA_SUMMARY_BF16. */
hga_status hga_build_summaries(const hga_config* cfg, const void* k_raw, void* chunk_sum,
                               void* group_sum, void* k_rot_out, int32_t chunk_begin,
                               int32_t chunk_end, void* stream);

/* Level-1 routing ("Kernmechanisme" item 2, Niveau 1, and Deterministische
 * Zichtbaarheid). For every (b, KV head, query chunk j of the span): q-bar
 * from q_rot [B, q_len, Hq, d] (written to qbar_out [B,Hkv,nQC,d] fp32), the
 * scores q-bar . chunk_sum[c] of the candidates c in [0, j) that are not
 * forced (forced = sinks c < n_sink, locals j-n_local <= c < j, current j),
 * and the top-min(top_k_chunks, #candidates) of them. Writes sel_chunks and
 * n_sel_chunks. scores_out (NULL or [B,Hkv,nQC,nC] fp32) receives every
 * candidate's score and NaN elsewhere. */
hga_status hga_route_chunks(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                            float* qbar_out, int32_t* sel_chunks, int32_t* n_sel_chunks,
                            float* scores_out, void* stream);

/* Level-2 routing ("Kernmechanisme" item 2, Niveau 2): inside the chunks
 * chosen by hga_route_chunks, score all G groups of every chosen chunk
 * against q-bar (qbar [B,Hkv,nQC,d] from hga_route_chunks) and keep the
 * top-min(top_k_groups, G * n_sel) globally. Writes sel_groups and
 * n_sel_groups. scores_out (NULL or [B,Hkv,nQC,top_k_chunks*G] fp32) holds the
 * score of group gamma of the s-th chosen chunk at s*G + gamma, NaN where
 * unused. */
hga_status hga_route_groups(const hga_config* cfg, const float* qbar, const void* group_sum,
                            const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                            int32_t* sel_groups, int32_t* n_sel_groups, float* scores_out,
                            void* stream);

/* Both routing levels in one call ("Kernmechanisme" item 2, Niveau 1 and 2):
 * the same q-bar and bitwise the same selections as hga_route_chunks
 * followed by hga_route_groups on these arguments, without the score
 * outputs. For a one-token query span (decode) in bf16 with d = 128 and
 * top_k_chunks <= 64 this is one launch (both levels split across a
 * thread-block cluster). For a prefill span of at least 8 query chunks with
 * nC <= 2048, groups_per_chunk <= 8, top_k_chunks <= 64 and
 * top_k_chunks * groups_per_chunk <= 256 it is two launches: q-bar, then both
 * levels in one kernel (each level-1 warp goes on to the groups of its query
 * chunk). Otherwise the two calls' kernels run in sequence.
 * qbar_out [B,Hkv,nQC,d] fp32, sel_chunks / n_sel_chunks, sel_groups /
 * n_sel_groups as for the two calls; all required. */
hga_status hga_route(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                     const void* group_sum, float* qbar_out, int32_t* sel_chunks,
                     int32_t* n_sel_chunks, int32_t* sel_groups, int32_t* n_sel_groups,
                     void* stream);

/* One routed attention step over a resident cache: hga_route, then
 * hga_attend in index mode over the full store k_cache / v_cache
 * [B, Hkv, L, d] (cfg->kv_layout must be HGA_KV_FULL; the host tier goes
 * through hga_route, hga_gather_kv and hga_attend). Writes q-bar, both
 * selections (as hga_route) and out [B, q_len, Hq, d]. For a one-token query
 * span (decode) in bf16, d = 128, gq <= 8, L % 16 == 0, top_k_chunks <= 64
 * this is a single launch: the always-visible blocks are fetched while the
 * routing runs; the attention result equals hga_attend's within fp32
 * summation order. Other configurations run the separate kernels. */
hga_status hga_decode_step(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                           const void* group_sum, const void* k_cache, const void* v_cache,
                           float* qbar_out, int32_t* sel_chunks, int32_t* n_sel_chunks,
                           int32_t* sel_groups, int32_t* n_sel_groups, void* out, void* stream);

/* One decode step over the tiered store of "Geheugenarchitectuur" in a
 * single launch: the hot tier (summary tables and the forced chunks'
 * windows) in device memory, the cold tier (the full K/V history) in host
 * memory. Routing as hga_route; then exact attention ("Kernmechanisme" item
 * 4) over the forced chunks, read from the resident windows k_win / v_win
 * [B, Hkv, W * C, d] (W = n_sink + n_local + 1 slots in ascending chunk
 * order, as for HGA_KV_WINDOWS), and over the selected groups, whose rows
 * are read from k_host / v_host [B, Hkv, L, d] (page-locked host memory
 * mapped into the device address space) inside the same kernel, so the
 * host-link reads overlap the attention over the resident windows and
 * nothing is staged in a gathered buffer. Writes q-bar, both selections (as
 * hga_route) and out [B, 1, Hq, d]; the result equals hga_route +
 * hga_gather_kv (host) + hga_attend in HGA_KV_WINDOWS within fp32 summation
 * order. Needs cfg->kv_layout == HGA_KV_WINDOWS, a one-token query at
 * q_begin == L - 1, and the one-launch configuration of hga_decode_step;
 * else HGA_ERR_UNSUPPORTED. HGA_ERR_MEMORY if a host pointer is not mapped. */
hga_status hga_decode_step_tiered(const hga_config* cfg, const void* q_rot, const void* chunk_sum,
                                  const void* group_sum, const void* k_win, const void* v_win,
                                  const void* k_host, const void* v_host, float* qbar_out,
                                  int32_t* sel_chunks, int32_t* n_sel_chunks, int32_t* sel_groups,
                                  int32_t* n_sel_groups, void* out, void* stream);

/* Exact-token retrieval ("Kernmechanisme" item 4; "Geheugenarchitectuur"
 * cold tier): copy the K and V rows of every selected group into compact
 * buffers k_dst, v_dst [B, Hkv, nQC, top_k_groups * g, d]; slot s holds the
 * g rows of the s-th selected group. Slots past n_sel_groups are not written.
 * k_src, v_src are the full store [B, Hkv, L, d]: device memory when
 * src_is_host == 0, page-locked host memory mapped into the device address
 * space (cudaHostAlloc / cudaHostRegister) when src_is_host == 1, read over
 * the host link. HGA_ERR_MEMORY if a host pointer is not mapped. */
hga_status hga_gather_kv(const hga_config* cfg, const void* k_src, const void* v_src,
                         int32_t src_is_host, const int32_t* sel_groups,
                         const int32_t* n_sel_groups, void* k_dst, void* v_dst, void* stream);

/* Warm tier ("Geheugenarchitectuur": a bounded LRU cache in VRAM keeps
 * recently routed groups between the cold host store and attention). Same
 * result in k_dst / v_dst as hga_gather_kv with src_is_host = 1 for a
 * one-token query span (decode): every selected group's K and V rows. A group
 * already in the caller's VRAM pool is copied from there; a missing group is
 * read once over the host link and also stored in the pool slot whose last
 * use is oldest among the slots this call does not hit (ties: lower slot;
 * empty slots first), so only misses cross the host link.
 *   k_host, v_host     full store [B, Hkv, L, d] in mapped page-locked host
 *                      memory (as for hga_gather_kv).
 *   pool_k, pool_v     [B, Hkv, n_slots, g, d] device memory, cfg->dtype.
 *   pool_tag           [B, Hkv, n_slots] int32: group index held, -1 = empty.
 *   pool_last          [B, Hkv, n_slots] int32: step of last use, -1 = never.
 *                      Initialise both to -1 once; the call updates them.
 *   n_slots            top_k_groups <= n_slots <= 4096.
 *   step               this call's step number, increasing over calls.
 *   src_out            [B, Hkv, top_k_groups] int32, written: the source of
 *                      each selected group (pool slot for a hit, -2 - slot for
 *                      a miss that filled that slot, -1 for an unused entry).
 *   stats_out          NULL or [B, Hkv, 2] int32: hits, misses.
 * Calls on one pool must not overlap (each reads and updates its tags).
 * HGA_ERR_UNSUPPORTED unless q_len == 1; HGA_ERR_MEMORY if a host pointer
 * is not mapped. */
hga_status hga_gather_kv_warm(const hga_config* cfg, const void* k_host, const void* v_host,
                              const int32_t* sel_groups, const int32_t* n_sel_groups,
                              void* pool_k, void* pool_v, int32_t* pool_tag, int32_t* pool_last,
                              int32_t n_slots, int32_t step, int32_t* src_out,
                              int32_t* stats_out, void* k_dst, void* v_dst, void* stream);

/* hga_gather_kv_warm without a caller scratch buffer. The pages have no
 * counterpart of this call: it exists for callers that may not allocate
 * device memory, e.g. a serving engine that reserves nearly all of HBM for
 * its KV pools at start-up and hands out only fixed buffers, or a decode loop
 * that cannot afford the device-wide synchronisation cudaFree implies. Same
 * arguments and results as hga_gather_kv_warm minus src_out: the per-selection
 * source list that the plan kernel hands to the copy kernel lives in a static
 * device array of 65536 int32 (256 KiB) inside the library, which every GPU
 * that loads the library holds until the process exits. The call allocates
 * nothing (no cudaMalloc, no allocating library routine).
 *   - HGA_ERR_SCRATCH_LIMIT if batch * n_kv_heads * top_k_groups > 65536.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (that device current) before enqueueing anything;
 *     make that first call before any stream capture.
 *   - Nothing in the array needs a starting value: each call writes every
 *     entry it reads before reading it. The array keeps the last call's
 *     contents.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (unordered streams, or several host threads) race and corrupt each
 *     other's results. Order them, e.g. on one stream. */
hga_status hga_gather_kv_warm_noalloc(const hga_config* cfg, const void* k_host,
                                      const void* v_host, const int32_t* sel_groups,
                                      const int32_t* n_sel_groups, void* pool_k, void* pool_v,
                                      int32_t* pool_tag, int32_t* pool_last, int32_t n_slots,
                                      int32_t step, int32_t* stats_out, void* k_dst, void* v_dst,
                                      void* stream);

/* Exact softmax attention over the bounded set ("Kernmechanisme" item 4):
 * for each query token at position p in chunk j and each query head, softmax
 * (scale 1/sqrt(d), fp32 accumulation) over the keys at positions <= p of
 * the forced chunks of j and of the selected groups, then the weighted sum of
 * their values. q_rot [B, q_len, Hq, d]; out [B, q_len, Hq, d].
 * Forced chunks come from k_res / v_res in cfg->kv_layout. Selected groups
 * come from k_gat / v_gat (the gathered buffers of hga_gather_kv) when those
 * are not NULL, else from k_res / v_res (HGA_KV_FULL only) by index. */
hga_status hga_attend(const hga_config* cfg, const void* q_rot, const void* k_res,
                      const void* v_res, const void* k_gat, const void* v_gat,
                      const int32_t* sel_groups, const int32_t* n_sel_groups, void* out,
                      void* stream);

/* Human-readable name of a status. Never NULL. */
const char* hga_status_string(hga_status status);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device. Returns HGA_OK, HGA_ERR_TIMEOUT (a wait gave up),
 * HGA_ERR_DEVICE_INDEX (an invalid entry; detail_out, if not NULL, receives
 * the code of the first one recorded: 1 chunk entry, 2 group entry, 3 count;
 * 4 = timeout) or HGA_ERR_CUDA. */
hga_status hga_get_device_error(void* stream, int32_t* detail_out);

/* Limit, in nanoseconds, of every bounded device-side wait in the launches
 * enqueued after this call, process-wide (0 restores the default, 1 s). A
 * healthy wait lasts microseconds; a watchdog that must report a stalled
 * launch sooner sets a shorter limit. The drain after a give-up always uses
 * the default limit. */
void hga_set_wait_limit_ns(uint64_t limit_ns);

/* The cudaError_t (as an int) of the last failed CUDA call that made a
 * library call of this host thread return HGA_ERR_CUDA; 0 if there was none. */
int32_t hga_last_cuda_error(void);

/* CUDA's description of a cudaError_t value (hga_last_cuda_error). Never NULL. */
const char* hga_cuda_error_string(int32_t cuda_error);

/* Library version as major * 10000 + minor * 100 + patch. */
int32_t hga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H */
