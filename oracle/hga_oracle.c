/*
 * hga_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, double-precision CPU oracle for the hot path of Hierarchical
 * Global Attention (HGA). Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it; the product path never does. It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Source of the method: "Technische Samenvatting: Hierarchical Global
 * Attention (HGA)" (gist.science/nl/paper/2606.30709), section
 * "Methodologie", subsection "Kernmechanisme":
 *   item 1 (Partitionering)            fixed chunks of C tokens, split in groups
 *   item 2 (Hierarchische Routing)     level-1 chunk routing over a table of
 *                                      chunk key summaries of earlier chunks,
 *                                      level-2 group routing inside the chosen
 *                                      chunks, and always-visible current,
 *                                      sink and recent local chunks
 *   item 3 (RoPE-bewuste Summaries)    high-frequency RoPE pairs rotated per
 *                                      token then averaged; low-frequency pairs
 *                                      averaged raw then rotated to the chunk's
 *                                      representative position; built from the
 *                                      existing projected keys
 *   item 4 (Exact-Token Attention)     standard softmax over the bounded exact
 *                                      token set
 * The arxivlens explanation ("Hierarchical Global Attention (HGA)", Key
 * Takeaways) restates the two-level chunk-then-group retrieval.
 *
 * The pages give no formulas. Readings taken here where they are silent:
 *   - RoPE: half-split pairing, pair i = (dim i, dim i + d/2), frequency
 *     theta_i = base^(-2i/d), angle p * theta_i; "high frequency" = small i,
 *     so pairs 0..F-1 are the high-frequency ones.
 *   - representative position of a token set = mean of its positions.
 *   - summaries are plain means (no length normalisation); the same mixed
 *     rule is applied at group scope and at chunk scope.
 *   - the routing query of (sequence, KV head, query chunk) is the mean of the
 *     rotated queries over the chunk's query tokens and the KV head's query
 *     heads; scores are plain dot products (no 1/sqrt(d): rank-invariant).
 *   - top-k counts only non-forced earlier chunks and is clamped to what is
 *     available; group top-k is global over all groups of the chosen chunks.
 *   - ties: higher score first, then lower index; a NaN score ranks last.
 *     Selections are returned in ascending index order, padded with -1.
 *   - routing decisions are taken on scores rounded to float (fp32), the
 *     precision in which the kernels take them.
 *   - the attention cache and the queries are bf16 in the bf16 workloads; the
 *     oracle rounds its own rotated keys/queries to bf16 (nearest-even) when
 *     asked, and computes everything else in double.
 *   - causal rule: a query at position p sees keys at positions <= p.
 *   - FP8 K/V caches (the FP8 deployment the pages motivate the method with,
 *     "Probleemstelling"): each cache entry is an E4M3 code times a per-tensor
 *     scale; attention runs on those decoded values exactly as on any other.
 *
 * Parity unpinned: the pairing, the representative position and the routing
 * query's aggregation are choices the pages cannot decide, so no test pins
 * them to the pages; they are fixed as above and taken identically on the
 * GPU side. The rest is pinned by closed forms, invariants and brute force
 * (tests/test_oracle_pins.py).
 *
 * Arithmetic is double throughout; loops follow the definitions with no
 * blocking or reordering. Independent units may run in parallel (OpenMP);
 * that changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t batch, seq_len, n_q_heads, n_kv_heads, head_dim;
    int32_t chunk_size, groups_per_chunk, n_sink, n_local;
    int32_t top_k_chunks, top_k_groups, n_high_freq_pairs;
    double rope_theta;
    int32_t q_begin, q_len;
} hgaref_cfg;

/* ------------------------------------------------------------------ RoPE */

/* Rotation angle of pair i at (possibly fractional) position p. */
static double ref_angle(const hgaref_cfg* c, int i, double p) {
    double freq = pow(c->rope_theta, -2.0 * (double)i / (double)c->head_dim);
    return p * freq;
}

/* out = R(p) x for one head vector of length d (half-split pairing). */
static void ref_rotate(const hgaref_cfg* c, const double* x, double p, double* out) {
    int h = c->head_dim / 2;
    for (int i = 0; i < h; ++i) {
        double a = ref_angle(c, i, p);
        double cs = cos(a), sn = sin(a);
        double x0 = x[i], x1 = x[i + h];
        out[i] = x0 * cs - x1 * sn;
        out[i + h] = x0 * sn + x1 * cs;
    }
}

/* bf16 round-to-nearest-even of a double, returned as a double. */
double hgaref_round_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (double)f; /* inf / nan */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    u &= 0xffff0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* out[i] = hgaref_round_bf16(in[i]) for i < n (bf16 summary tables). */
void hgaref_round_bf16_n(const double* in, double* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = hgaref_round_bf16(in[i]);
}

/* Value of one 8-bit floating-point code of the E4M3 kind (the FP8 format of
 * FP8 K/V caches): bit 7 the sign, bits 6..3 the exponent e with bias 7, bits
 * 2..0 the mantissa m. e = 0 is subnormal, (m / 8) * 2^-6; otherwise
 * (1 + m / 8) * 2^(e - 7). The one all-ones pattern below the sign (e = 15,
 * m = 7) is NaN; there are no infinities, so the largest finite value is
 * 1.75 * 2^8 = 448. */
double hgaref_e4m3_value(uint8_t code) {
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* out[i] = hgaref_e4m3_value(codes[i]) * scale for i < n: an FP8 K or V
 * cache entry with its per-tensor scale, as the attention reads it. */
void hgaref_e4m3_decode_n(const uint8_t* codes, int64_t n, double scale, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = hgaref_e4m3_value(codes[i]) * scale;
}

/* Rotate rows x[n_tok][n_heads][d] where token t sits at position pos0 + t.
 * round_bf16 != 0 rounds each result to bf16 (the storage type of the cache). */
void hgaref_rope(const hgaref_cfg* c, const float* x, int64_t n_tok, int n_heads,
                 int64_t pos0, int round_bf16, double* out) {
    int d = c->head_dim;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t) {
        double xin[512], xo[512];
        for (int hh = 0; hh < n_heads; ++hh) {
            const float* row = x + (t * n_heads + hh) * (int64_t)d;
            for (int k = 0; k < d; ++k) xin[k] = row[k];
            ref_rotate(c, xin, (double)(pos0 + t), xo);
            double* o = out + (t * n_heads + hh) * (int64_t)d;
            for (int k = 0; k < d; ++k) o[k] = round_bf16 ? hgaref_round_bf16(xo[k]) : xo[k];
        }
    }
}

/* ------------------------------------------------------------ summaries */

/* Mixed RoPE-aware summary of the n keys krow[0..n) at positions
 * first_pos..first_pos+n-1 ("Kernmechanisme" item 3). Zero when n == 0. */
static void ref_summary(const hgaref_cfg* c, const float* krow, int64_t first_pos, int n,
                        double* out) {
    int d = c->head_dim, h = d / 2, F = c->n_high_freq_pairs;
    for (int k = 0; k < d; ++k) out[k] = 0.0;
    if (n <= 0) return;
    double pbar = 0.0;
    for (int t = 0; t < n; ++t) pbar += (double)(first_pos + t);
    pbar /= (double)n;
    for (int i = 0; i < h; ++i) {
        if (i < F) {
            /* high frequency: rotate each token to its own position, then average */
            double s0 = 0.0, s1 = 0.0;
            for (int t = 0; t < n; ++t) {
                double a = ref_angle(c, i, (double)(first_pos + t));
                double x0 = krow[(int64_t)t * d + i], x1 = krow[(int64_t)t * d + i + h];
                s0 += x0 * cos(a) - x1 * sin(a);
                s1 += x0 * sin(a) + x1 * cos(a);
            }
            out[i] = s0 / n;
            out[i + h] = s1 / n;
        } else {
            /* low frequency: average the raw keys, then rotate to pbar */
            double m0 = 0.0, m1 = 0.0;
            for (int t = 0; t < n; ++t) {
                m0 += krow[(int64_t)t * d + i];
                m1 += krow[(int64_t)t * d + i + h];
            }
            m0 /= n;
            m1 /= n;
            double a = ref_angle(c, i, pbar);
            out[i] = m0 * cos(a) - m1 * sin(a);
            out[i + h] = m0 * sin(a) + m1 * cos(a);
        }
    }
}

static int64_t ref_n_chunks(const hgaref_cfg* c) {
    return (c->seq_len + c->chunk_size - 1) / c->chunk_size;
}

/* k_raw [B,Hkv,L,d] pre-RoPE keys -> chunk_sum [B,Hkv,nC,d], group_sum
 * [B,Hkv,nC*G,d]. Chunks and groups cover only the tokens that exist. */
void hgaref_build_summaries(const hgaref_cfg* c, const float* k_raw, double* chunk_sum,
                            double* group_sum) {
    int64_t L = c->seq_len, nC = ref_n_chunks(c);
    int d = c->head_dim, C = c->chunk_size, G = c->groups_per_chunk, g = C / G;
    int64_t BH = (int64_t)c->batch * c->n_kv_heads;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t ch = 0; ch < nC; ++ch) {
            const float* base = k_raw + bh * L * d;
            int64_t c0 = ch * C;
            int64_t c1 = c0 + C < L ? c0 + C : L;
            ref_summary(c, base + c0 * d, c0, (int)(c1 - c0), chunk_sum + (bh * nC + ch) * d);
            for (int gr = 0; gr < G; ++gr) {
                int64_t g0 = c0 + (int64_t)gr * g;
                int64_t g1 = g0 + g < L ? g0 + g : L;
                int n = g1 > g0 ? (int)(g1 - g0) : 0;
                ref_summary(c, base + g0 * d, g0, n,
                            group_sum + ((bh * nC + ch) * G + gr) * d);
            }
        }
    }
}

/* ------------------------------------------------------------- routing */

/* Query chunks touched by the span [q_begin, q_begin + q_len). */
static int64_t ref_first_qchunk(const hgaref_cfg* c) { return c->q_begin / c->chunk_size; }
static int64_t ref_n_qchunks(const hgaref_cfg* c) {
    if (c->q_len <= 0) return 0;
    return (c->q_begin + c->q_len - 1) / c->chunk_size - ref_first_qchunk(c) + 1;
}

/* q_rot [B,q_len,Hq,d] (rotated queries) -> qbar [B,Hkv,nQC,d]: mean over
 * the chunk's query tokens (ascending) and the KV head's query heads. */
void hgaref_qbar(const hgaref_cfg* c, const float* q_rot, double* qbar) {
    int d = c->head_dim, Hq = c->n_q_heads, Hkv = c->n_kv_heads, gq = Hq / Hkv;
    int C = c->chunk_size;
    int64_t nQC = ref_n_qchunks(c), j0 = ref_first_qchunk(c);
#pragma omp parallel for collapse(3) schedule(static)
    for (int b = 0; b < c->batch; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int64_t jj = 0; jj < nQC; ++jj) {
                int64_t j = j0 + jj;
                int64_t t0 = j * C > c->q_begin ? j * C : c->q_begin;
                int64_t t1 = (j + 1) * C < (int64_t)c->q_begin + c->q_len ? (j + 1) * C
                                                                     : (int64_t)c->q_begin + c->q_len;
                double* o = qbar + (((int64_t)b * Hkv + hk) * nQC + jj) * d;
                for (int k = 0; k < d; ++k) o[k] = 0.0;
                int64_t n = 0;
                for (int64_t t = t0; t < t1; ++t)
                    for (int hq = hk * gq; hq < (hk + 1) * gq; ++hq) {
                        const float* row =
                            q_rot + (((int64_t)b * c->q_len + (t - c->q_begin)) * Hq + hq) * d;
                        for (int k = 0; k < d; ++k) o[k] += row[k];
                        ++n;
                    }
                for (int k = 0; k < d; ++k) o[k] /= (double)n;
            }
}

/* Is chunk ch always visible to query chunk j (sink, recent local, current)? */
int hgaref_is_forced(const hgaref_cfg* c, int64_t j, int64_t ch) {
    if (ch < 0 || ch > j) return 0;
    if (ch == j) return 1;
    if (ch < c->n_sink) return 1;
    if (ch >= j - c->n_local) return 1;
    return 0;
}

typedef struct {
    float score;
    int32_t index;
} ref_cand;

/* Order: higher score first, NaN last, then lower index first. */
static int ref_cand_cmp(const void* pa, const void* pb) {
    const ref_cand* a = (const ref_cand*)pa;
    const ref_cand* b = (const ref_cand*)pb;
    int an = isnan(a->score), bn = isnan(b->score);
    if (an != bn) return an ? 1 : -1;
    if (!an) {
        if (a->score > b->score) return -1;
        if (a->score < b->score) return 1;
    }
    return (a->index > b->index) - (a->index < b->index);
}

static int ref_int_cmp(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Keep the first k of cand[0..n) in the order above; write them ascending
 * into sel[0..k_cap), padded with -1. Returns the number kept. */
static int ref_topk(ref_cand* cand, int n, int k, int32_t* sel, int k_cap) {
    qsort(cand, (size_t)n, sizeof(ref_cand), ref_cand_cmp);
    int kept = k < n ? k : n;
    for (int s = 0; s < kept; ++s) sel[s] = cand[s].index;
    qsort(sel, (size_t)kept, sizeof(int32_t), ref_int_cmp);
    for (int s = kept; s < k_cap; ++s) sel[s] = -1;
    return kept;
}

static float ref_dot_f32(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += a[k] * b[k];
    return (float)s;
}

/* Level-1 routing. qbar [B,Hkv,nQC,d], chunk_sum [B,Hkv,nC,d] ->
 * sel [B,Hkv,nQC,k_c], n_sel [B,Hkv,nQC]; scores (nullable) [B,Hkv,nQC,nC]
 * holds the fp32 score of every candidate and NaN for non-candidates. */
void hgaref_route_chunks(const hgaref_cfg* c, const double* qbar, const double* chunk_sum,
                         int32_t* sel, int32_t* n_sel, float* scores) {
    int d = c->head_dim, Hkv = c->n_kv_heads, kc = c->top_k_chunks;
    int64_t nC = ref_n_chunks(c), nQC = ref_n_qchunks(c), j0 = ref_first_qchunk(c);
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < c->batch; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int64_t jj = 0; jj < nQC; ++jj) {
                int64_t j = j0 + jj, prob = ((int64_t)b * Hkv + hk) * nQC + jj;
                const double* q = qbar + prob * d;
                ref_cand* cand = (ref_cand*)malloc(sizeof(ref_cand) * (size_t)(j > 0 ? j : 1));
                int n = 0;
                if (scores)
                    for (int64_t ch = 0; ch < nC; ++ch) scores[prob * nC + ch] = NAN;
                for (int64_t ch = 0; ch < j; ++ch) {
                    if (hgaref_is_forced(c, j, ch)) continue;
                    const double* s = chunk_sum + (((int64_t)b * Hkv + hk) * nC + ch) * d;
                    cand[n].score = ref_dot_f32(q, s, d);
                    cand[n].index = (int32_t)ch;
                    if (scores) scores[prob * nC + ch] = cand[n].score;
                    ++n;
                }
                n_sel[prob] = ref_topk(cand, n, kc, sel + prob * kc, kc);
                free(cand);
            }
}

/* Level-2 routing inside the chosen chunks. Candidates are all G groups of
 * every selected chunk (global group index ch*G + gamma); top-k_g globally.
 * scores (nullable) [B,Hkv,nQC,k_c*G] in candidate order (selected chunk s,
 * group gamma at s*G + gamma), NaN where unused. */
void hgaref_route_groups(const hgaref_cfg* c, const double* qbar, const double* group_sum,
                         const int32_t* sel_chunks, const int32_t* n_sel_chunks,
                         int32_t* sel_groups, int32_t* n_sel_groups, float* scores) {
    int d = c->head_dim, Hkv = c->n_kv_heads, kc = c->top_k_chunks, kg = c->top_k_groups;
    int G = c->groups_per_chunk;
    int64_t nC = ref_n_chunks(c), nQC = ref_n_qchunks(c);
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < c->batch; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int64_t jj = 0; jj < nQC; ++jj) {
                int64_t prob = ((int64_t)b * Hkv + hk) * nQC + jj;
                const double* q = qbar + prob * d;
                int ns = n_sel_chunks[prob];
                ref_cand* cand = (ref_cand*)malloc(sizeof(ref_cand) * (size_t)(ns * G + 1));
                int n = 0;
                if (scores)
                    for (int s = 0; s < kc * G; ++s) scores[prob * kc * G + s] = NAN;
                for (int s = 0; s < ns; ++s) {
                    int32_t ch = sel_chunks[prob * kc + s];
                    for (int gr = 0; gr < G; ++gr) {
                        int64_t gi = (int64_t)ch * G + gr;
                        const double* gs = group_sum + (((int64_t)b * Hkv + hk) * nC * G + gi) * d;
                        cand[n].score = ref_dot_f32(q, gs, d);
                        cand[n].index = (int32_t)gi;
                        if (scores) scores[prob * kc * G + s * G + gr] = cand[n].score;
                        ++n;
                    }
                }
                n_sel_groups[prob] = ref_topk(cand, n, kg, sel_groups + prob * kg, kg);
                free(cand);
            }
}

/* ------------------------------------------------------------ attention */

/* Exact softmax attention over the bounded set ("Kernmechanisme" item 4).
 * q_rot [B,q_len,Hq,d]; k_rot, v [B,Hkv,L,d]; sel_groups [B,Hkv,nQC,k_g].
 * The key set of query chunk j is the union of the tokens of its forced
 * chunks and of its selected groups; a query at position p sees the keys of
 * that set at positions <= p. units: n_units triples (b, kv head, query
 * chunk index jj) to compute, or NULL for all. out [B,q_len,Hq,d]; rows of
 * units not computed are left untouched. Two-pass softmax, scale 1/sqrt(d). */
void hgaref_attend(const hgaref_cfg* c, const float* q_rot, const float* k_rot, const float* v,
                   const int32_t* sel_groups, const int32_t* n_sel_groups,
                   const int32_t* units, int64_t n_units, double* out) {
    int d = c->head_dim, Hq = c->n_q_heads, Hkv = c->n_kv_heads, gq = Hq / Hkv;
    int C = c->chunk_size, G = c->groups_per_chunk, g = C / G, kg = c->top_k_groups;
    int64_t L = c->seq_len, nQC = ref_n_qchunks(c), j0 = ref_first_qchunk(c);
    int64_t total = units ? n_units : (int64_t)c->batch * Hkv * nQC;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic)
    for (int64_t u = 0; u < total; ++u) {
        int b, hk;
        int64_t jj;
        if (units) {
            b = units[3 * u];
            hk = units[3 * u + 1];
            jj = units[3 * u + 2];
        } else {
            b = (int)(u / (Hkv * nQC));
            hk = (int)((u / nQC) % Hkv);
            jj = u % nQC;
        }
        int64_t j = j0 + jj, prob = ((int64_t)b * Hkv + hk) * nQC + jj;
        /* membership of every key position in the set */
        unsigned char* in_set = (unsigned char*)calloc((size_t)L, 1);
        for (int64_t ch = 0; ch <= j; ++ch)
            if (hgaref_is_forced(c, j, ch))
                for (int64_t t = ch * C; t < (ch + 1) * C && t < L; ++t) in_set[t] = 1;
        for (int s = 0; s < n_sel_groups[prob]; ++s) {
            int64_t gi = sel_groups[prob * kg + s];
            for (int64_t t = gi * g; t < (gi + 1) * g && t < L; ++t) in_set[t] = 1;
        }
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
        double* sc = (double*)malloc(sizeof(double) * (size_t)L);
        int64_t t0 = j * C > c->q_begin ? j * C : c->q_begin;
        int64_t t1 = (j + 1) * C < (int64_t)c->q_begin + c->q_len ? (j + 1) * C
                                                             : (int64_t)c->q_begin + c->q_len;
        const float* kb = k_rot + ((int64_t)b * Hkv + hk) * L * d;
        const float* vb = v + ((int64_t)b * Hkv + hk) * L * d;
        for (int64_t t = t0; t < t1; ++t) {
            int64_t nk = 0;
            for (int64_t p = 0; p <= t; ++p)
                if (in_set[p]) keys[nk++] = p;
            for (int hq = hk * gq; hq < (hk + 1) * gq; ++hq) {
                const float* q = q_rot + (((int64_t)b * c->q_len + (t - c->q_begin)) * Hq + hq) * d;
                double m = -INFINITY;
                for (int64_t s = 0; s < nk; ++s) {
                    const float* kr = kb + keys[s] * d;
                    double dot = 0.0;
                    for (int k = 0; k < d; ++k) dot += (double)q[k] * (double)kr[k];
                    sc[s] = dot * scale;
                    if (sc[s] > m) m = sc[s];
                }
                double l = 0.0;
                for (int64_t s = 0; s < nk; ++s) {
                    sc[s] = exp(sc[s] - m);
                    l += sc[s];
                }
                double* o = out + (((int64_t)b * c->q_len + (t - c->q_begin)) * Hq + hq) * d;
                for (int k = 0; k < d; ++k) o[k] = 0.0;
                for (int64_t s = 0; s < nk; ++s) {
                    const float* vr = vb + keys[s] * d;
                    for (int k = 0; k < d; ++k) o[k] += sc[s] * (double)vr[k];
                }
                for (int k = 0; k < d; ++k) o[k] /= l;
            }
        }
        free(sc);
        free(keys);
        free(in_set);
    }
}

/* Number of threads the parallel loops above use. */
int hgaref_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void hgaref_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
