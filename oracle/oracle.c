/*
 * oracle.c -- plain fp64 CPU restatement of the paged-KV decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA path.
 *
 * Pages followed (cited by title and section):
 *   [源码解析]  "vLLM 源码解析：PagedAttention 如何让大模型推理提速 10 倍"
 *   [深度解析]  "vLLM 核心源码深度解析：PagedAttention 的 KV Cache 管理、Scheduler
 *               调度引擎与 Continuous Batching 实现全解"
 *   [论文专题]  "论文专题讲解：vLLM / PagedAttention：为什么 KV cache 需要分页管理"
 *               (a digest of Kwon et al., arXiv 2309.06180)
 *
 * Conventions (all arrays row-major, caller-owned):
 *   bf16 values arrive as their raw 16-bit patterns (uint16_t) and are widened
 *   exactly to double; all arithmetic is double.
 *   key_cache / value_cache: [num_blocks, block_size, num_kv_heads, head_dim]
 *     -- the layout of [源码解析 §四] (its `num_heads` read as the KV heads).
 *   block_tables: int32 [num_seqs, max_blocks]; seq_lens: int32 [num_seqs].
 *   slot_mapping: int64 [num_tokens]; a negative slot means "skip" (padding).
 *
 * Every function here is pinned by tests/test_oracle_pins.py against values
 * the pages print, closed forms, invariants and an independent library routine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Address translation, [深度解析 «Block Table 数据结构»]:
 *   block_number = position // block_size
 *   offset       = position %  block_size
 *   physical     = block_table[block_number]
 * and the flat slot index of that token in the cache is physical*bs + offset.
 * Returns 0, or -1 if a position is negative or falls outside its table row.
 */
int oracle_slot_mapping(const int32_t *block_tables, int max_blocks,
                        const int32_t *seq_ids, const int64_t *positions,
                        int num_tokens, int block_size, int64_t *slots)
{
    for (int t = 0; t < num_tokens; ++t) {
        int64_t pos = positions[t];
        if (pos < 0) { slots[t] = -1; continue; }
        int64_t block_number = pos / block_size;
        int64_t offset = pos % block_size;
        if (block_number >= max_blocks) return -1;
        int64_t physical = block_tables[(int64_t)seq_ids[t] * max_blocks + block_number];
        if (physical < 0) return -1;
        slots[t] = physical * block_size + offset;
    }
    return 0;
}

/*
 * Cache write: each new token's K and V go to its slot ([论文专题 «Continuous
 * batching 为什么离不开内存管理»]: generated K/V are written back into the
 * corresponding block; [深度解析 «Copy-on-Write 与 Prefix Caching»]: 写入新值).
 * key/value: [num_tokens, num_kv_heads, head_dim].  A plain element loop.
 */
void oracle_reshape_and_cache(const uint16_t *key, const uint16_t *value,
                              uint16_t *key_cache, uint16_t *value_cache,
                              const int64_t *slot_mapping, int num_tokens,
                              int num_kv_heads, int head_dim, int block_size)
{
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim + d;
                int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim + d;
                key_cache[dst] = key[src];
                value_cache[dst] = value[src];
            }
        }
    }
}

/*
 * Block copy for copy-on-write, [源码解析 §五] (allocate_or_get_cow: allocate a
 * new physical block and copy the old data into it).  Pairs are applied in
 * order; each copies a whole physical block of K and of V.
 */
void oracle_copy_blocks(uint16_t *key_cache, uint16_t *value_cache,
                        const int64_t *src_dst_pairs, int num_pairs,
                        int num_kv_heads, int head_dim, int block_size)
{
    int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = src_dst_pairs[2 * i];
        int64_t dst = src_dst_pairs[2 * i + 1];
        for (int64_t e = 0; e < block_elems; ++e) {
            key_cache[dst * block_elems + e] = key_cache[src * block_elems + e];
            value_cache[dst * block_elems + e] = value_cache[src * block_elems + e];
        }
    }
}

/*
 * Swap of whole blocks between two caches (GPU cache and host cache), the copy
 * behind the GPU/CPU swap of "vLLM 核心源码深度解析 …", «BlockAllocator 源码核心»:
 * pair i copies block src of (src_k, src_v) into block dst of (dst_k, dst_v).
 */
void oracle_swap_blocks(uint16_t *dst_k, uint16_t *dst_v, const uint16_t *src_k, const uint16_t *src_v,
                        const int64_t *src_dst_pairs, int num_pairs, int num_kv_heads, int head_dim,
                        int block_size)
{
    int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = src_dst_pairs[2 * i];
        int64_t dst = src_dst_pairs[2 * i + 1];
        for (int64_t e = 0; e < block_elems; ++e) {
            dst_k[dst * block_elems + e] = src_k[src * block_elems + e];
            dst_v[dst * block_elems + e] = src_v[src * block_elems + e];
        }
    }
}

/*
 * Gather of one sequence's logical K (or V) rows for one KV head into a
 * contiguous [len, head_dim] double array, walking the block table exactly as
 * [论文专题 «PagedAttention：逻辑连续，物理不必连续»] describes: logical block j
 * holds positions j*B .. j*B+B-1 (the K_j, V_j equation), found at physical
 * block block_table[j].
 */
static void gather_rows(double *dst, const uint16_t *cache, const int32_t *table,
                        int first_pos, int len, int kv_head, int num_kv_heads,
                        int head_dim, int block_size)
{
    for (int i = 0; i < len; ++i) {
        int pos = first_pos + i;
        int64_t physical = table[pos / block_size];
        int offset = pos % block_size;
        const uint16_t *row = cache + ((physical * block_size + offset) * num_kv_heads + kv_head) * (int64_t)head_dim;
        for (int d = 0; d < head_dim; ++d) dst[(int64_t)i * head_dim + d] = widen_bf16(row[d]);
    }
}

/*
 * Partial attention of one (sequence, query head) over positions
 * [first_pos, first_pos+len): the per-block local result that [源码解析 §四]
 * computes before merging.  With x_p = scale * <q, k_p>:
 *   m = max_p x_p,  l = sum_p exp(x_p - m),  o[d] = sum_p exp(x_p - m) v_p[d]
 * (o is NOT normalised).  len == 0 gives m = -inf, l = 0, o = 0.
 */
static void partial_attention(double *m_out, double *l_out, double *o_out,
                              const double *q, const double *k, const double *v,
                              int len, int head_dim, double scale, double *x)
{
    double m = -INFINITY;
    for (int p = 0; p < len; ++p) {
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d) dot += q[d] * k[(int64_t)p * head_dim + d];
        x[p] = scale * dot;
        if (x[p] > m) m = x[p];
    }
    double l = 0.0;
    for (int d = 0; d < head_dim; ++d) o_out[d] = 0.0;
    for (int p = 0; p < len; ++p) {
        double w = exp(x[p] - m);
        l += w;
        for (int d = 0; d < head_dim; ++d) o_out[d] += w * v[(int64_t)p * head_dim + d];
    }
    *m_out = m;
    *l_out = l;
}

/*
 * Single-query paged decode, [源码解析 §四] paged_attention(query, key_cache,
 * value_cache, page_table) and [论文专题 «PagedAttention：逻辑连续，物理不必连续»]:
 * the query of sequence s attends to all of its cached positions 0..L_s-1
 * (the formula is the ordinary one; only where K/V are read from changes):
 *   out[s,h,:] = sum_p softmax_p(scale * q[s,h]·k_p) v_p
 * Query head h reads KV head h / (num_heads / num_kv_heads).  L_s == 0 gives a
 * zero output.  query: bf16 [num_seqs, num_heads, head_dim]; out: double, same
 * shape.  Parallel over (s, h) with nthreads OpenMP threads (<= 0: all).
 */
void oracle_paged_decode(double *out, const uint16_t *query,
                         const uint16_t *key_cache, const uint16_t *value_cache,
                         const int32_t *block_tables, const int32_t *seq_lens,
                         double scale, int block_size, int num_kv_heads,
                         int num_seqs, int num_heads, int head_dim,
                         int max_blocks, int nthreads)
{
    int group = num_heads / num_kv_heads;
    int64_t units = (int64_t)num_seqs * num_heads;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / num_heads);
        int h = (int)(u % num_heads);
        int len = seq_lens[s];
        double *o = out + u * head_dim;
        if (len <= 0) {
            for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
            continue;
        }
        int kv_head = h / group;
        double *q = malloc(sizeof(double) * head_dim);
        double *k = malloc(sizeof(double) * (size_t)len * head_dim);
        double *v = malloc(sizeof(double) * (size_t)len * head_dim);
        double *x = malloc(sizeof(double) * (size_t)len);
        const uint16_t *qrow = query + u * head_dim;
        for (int d = 0; d < head_dim; ++d) q[d] = widen_bf16(qrow[d]);
        const int32_t *table = block_tables + (int64_t)s * max_blocks;
        gather_rows(k, key_cache, table, 0, len, kv_head, num_kv_heads, head_dim, block_size);
        gather_rows(v, value_cache, table, 0, len, kv_head, num_kv_heads, head_dim, block_size);
        double m, l;
        partial_attention(&m, &l, o, q, k, v, len, head_dim, scale, x);
        for (int d = 0; d < head_dim; ++d) o[d] /= l;
        free(q); free(k); free(v); free(x);
    }
}

/*
 * The split form of the same computation ("逐块计算局部 Attention，最后合并结果",
 * [源码解析 §四]): positions are cut into partitions of partition_size tokens;
 * partition p of (s, h) yields m, l and the unnormalised o over its positions.
 * Outputs: m, l: double [num_seqs, num_heads, max_parts];
 *          o:    double [num_seqs, num_heads, max_parts, head_dim].
 * Partitions at or beyond ceil(L/partition_size) get m=-inf, l=0, o=0.
 */
void oracle_paged_decode_partials(double *m_out, double *l_out, double *o_out,
                                  const uint16_t *query,
                                  const uint16_t *key_cache, const uint16_t *value_cache,
                                  const int32_t *block_tables, const int32_t *seq_lens,
                                  double scale, int block_size, int num_kv_heads,
                                  int num_seqs, int num_heads, int head_dim,
                                  int max_blocks, int partition_size, int max_parts)
{
    int group = num_heads / num_kv_heads;
    double *q = malloc(sizeof(double) * head_dim);
    double *k = malloc(sizeof(double) * (size_t)partition_size * head_dim);
    double *v = malloc(sizeof(double) * (size_t)partition_size * head_dim);
    double *x = malloc(sizeof(double) * (size_t)partition_size);
    for (int s = 0; s < num_seqs; ++s) {
        const int32_t *table = block_tables + (int64_t)s * max_blocks;
        for (int h = 0; h < num_heads; ++h) {
            int kv_head = h / group;
            const uint16_t *qrow = query + ((int64_t)s * num_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d) q[d] = widen_bf16(qrow[d]);
            for (int p = 0; p < max_parts; ++p) {
                int64_t idx = ((int64_t)s * num_heads + h) * max_parts + p;
                int first = p * partition_size;
                int len = seq_lens[s] - first;
                if (len > partition_size) len = partition_size;
                if (len < 0) len = 0;
                gather_rows(k, key_cache, table, first, len, kv_head, num_kv_heads, head_dim, block_size);
                gather_rows(v, value_cache, table, first, len, kv_head, num_kv_heads, head_dim, block_size);
                partial_attention(&m_out[idx], &l_out[idx], o_out + idx * head_dim,
                                  q, k, v, len, head_dim, scale, x);
            }
        }
    }
    free(q); free(k); free(v); free(x);
}

/*
 * Merge of partition results (the "最后合并结果" step of [源码解析 §四]) by the
 * log-sum-exp rule: with M = max_p m_p and w_p = exp(m_p - M),
 *   out = (sum_p w_p o_p) / (sum_p w_p l_p).
 * Partitions with m_p = -inf (empty) carry weight 0.  All partitions empty
 * gives a zero output.  Shapes as oracle_paged_decode_partials; out is
 * double [num_seqs*num_heads, head_dim] with rows = num_seqs*num_heads.
 */
void oracle_lse_merge(double *out, const double *m, const double *l, const double *o,
                      int rows, int max_parts, int head_dim)
{
    for (int r = 0; r < rows; ++r) {
        const double *mr = m + (int64_t)r * max_parts;
        const double *lr = l + (int64_t)r * max_parts;
        const double *orow = o + (int64_t)r * max_parts * head_dim;
        double *dst = out + (int64_t)r * head_dim;
        double big = -INFINITY;
        for (int p = 0; p < max_parts; ++p) if (mr[p] > big) big = mr[p];
        for (int d = 0; d < head_dim; ++d) dst[d] = 0.0;
        if (big == -INFINITY) continue;
        double denom = 0.0;
        for (int p = 0; p < max_parts; ++p) {
            if (mr[p] == -INFINITY) continue;
            double w = exp(mr[p] - big);
            denom += w * lr[p];
            for (int d = 0; d < head_dim; ++d) dst[d] += w * orow[(int64_t)p * head_dim + d];
        }
        for (int d = 0; d < head_dim; ++d) dst[d] /= denom;
    }
}

/*
 * FP8 KV cache ("vLLM 核心源码深度解析 …", milestone list: FP8 KV Cache).  The
 * stored byte is an OCP FP8 E4M3 code: sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no
 * infinities; the largest finite magnitude is 448.  A stored code c stands for
 * e4m3(c) * scale (one scale per cache tensor).
 */
double oracle_e4m3_to_f64(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest E4M3 code to x (ties to the even code, the sign kept, zero included),
 * magnitudes beyond 448 clamped
 * to +-448 (infinities included: the format has none, and a saturating
 * conversion keeps the sign and takes the largest finite value), NaN to 0x7F:
 * a linear scan over the 127 non-negative finite codes. */
uint8_t oracle_f64_to_e4m3(double x)
{
    if (x != x) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;   /* -0 and negative underflows keep the sign */
    double a = fabs(x);
    if (a > 448.0) return (uint8_t)(sign | 0x7E);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 126; ++c) {
        double err = fabs(oracle_e4m3_to_f64((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* Cache write with quantisation: code = e4m3(fp32(fp32(x) * inv_scale)), the
 * product taken in fp32 (as the kernel takes it) and then rounded to E4M3. */
void oracle_reshape_and_cache_fp8(const uint16_t *key, const uint16_t *value, uint8_t *key_cache,
                                  uint8_t *value_cache, const int64_t *slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_dim, int block_size, float k_inv_scale,
                                  float v_inv_scale)
{
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim + d;
                int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim + d;
                float kx = (float)widen_bf16(key[src]) * k_inv_scale;
                float vx = (float)widen_bf16(value[src]) * v_inv_scale;
                key_cache[dst] = oracle_f64_to_e4m3((double)kx);
                value_cache[dst] = oracle_f64_to_e4m3((double)vx);
            }
        }
    }
}

/* Paged decode over an FP8 cache: K and V rows are e4m3(code) * k_scale and
 * e4m3(code) * v_scale; otherwise exactly oracle_paged_decode. */
void oracle_paged_decode_fp8(double *out, const uint16_t *query, const uint8_t *key_cache,
                             const uint8_t *value_cache, const int32_t *block_tables,
                             const int32_t *seq_lens, double scale, double k_scale, double v_scale,
                             int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                             int max_blocks, int nthreads)
{
    int group = num_heads / num_kv_heads;
    int64_t units = (int64_t)num_seqs * num_heads;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / num_heads);
        int h = (int)(u % num_heads);
        int len = seq_lens[s];
        double *o = out + u * head_dim;
        if (len <= 0) {
            for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
            continue;
        }
        int kv_head = h / group;
        double *q = malloc(sizeof(double) * head_dim);
        double *k = malloc(sizeof(double) * (size_t)len * head_dim);
        double *v = malloc(sizeof(double) * (size_t)len * head_dim);
        double *x = malloc(sizeof(double) * (size_t)len);
        const uint16_t *qrow = query + u * head_dim;
        for (int d = 0; d < head_dim; ++d) q[d] = widen_bf16(qrow[d]);
        const int32_t *table = block_tables + (int64_t)s * max_blocks;
        for (int i = 0; i < len; ++i) {
            int64_t physical = table[i / block_size];
            int64_t row = ((physical * block_size + i % block_size) * num_kv_heads + kv_head) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                k[(int64_t)i * head_dim + d] = oracle_e4m3_to_f64(key_cache[row + d]) * k_scale;
                v[(int64_t)i * head_dim + d] = oracle_e4m3_to_f64(value_cache[row + d]) * v_scale;
            }
        }
        double m, l;
        partial_attention(&m, &l, o, q, k, v, len, head_dim, scale, x);
        for (int d = 0; d < head_dim; ++d) o[d] /= l;
        free(q); free(k); free(v); free(x);
    }
}

/*
 * Multi-query paged prefill over the block table: the chunked-prefill step
 * ("vLLM 核心源码深度解析 …", milestone list: v0.5 Chunked Prefill -- a long
 * prompt is fed in chunks so that it does not hold up the decodes) with the
 * causal rule of [论文专题] (the query at position i attends to positions up to
 * and including i).  Sequence s holds seq_lens[s] cached positions; the last
 * q_lens[s] of them are this chunk's new tokens, whose K/V rows are already in
 * the cache.  New token i of s sits at position p = seq_lens[s] - q_lens[s] + i
 * and its query row is q_start[s] + i (q_start: int32 [num_seqs + 1],
 * q_start[s+1] - q_start[s] = q_lens[s]):
 *   out[row, h, :] = sum_{j <= p} softmax_j(scale * q[row, h] . k_j) v_j
 * query / out: [num_tokens, num_heads, head_dim] (out double).  Query head h
 * reads KV head h / (num_heads / num_kv_heads).  Parallel over (row, head).
 */
void oracle_paged_prefill(double *out, const uint16_t *query, const uint16_t *key_cache,
                          const uint16_t *value_cache, const int32_t *block_tables,
                          const int32_t *seq_lens, const int32_t *q_start, double scale,
                          int block_size, int num_kv_heads, int num_seqs, int num_heads,
                          int head_dim, int max_blocks, int nthreads)
{
    int group = num_heads / num_kv_heads;
    int64_t rows = q_start[num_seqs];
    int64_t units = rows * num_heads;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int64_t row = u / num_heads;
        int h = (int)(u % num_heads);
        int s = 0;
        while (q_start[s + 1] <= row) ++s;   /* the sequence owning this row */
        int q_len = q_start[s + 1] - q_start[s];
        int pos = seq_lens[s] - q_len + (int)(row - q_start[s]);
        int len = pos + 1;                   /* positions 0..pos */
        int kv_head = h / group;
        double *o = out + u * head_dim;
        double *q = malloc(sizeof(double) * head_dim);
        double *k = malloc(sizeof(double) * (size_t)len * head_dim);
        double *v = malloc(sizeof(double) * (size_t)len * head_dim);
        double *x = malloc(sizeof(double) * (size_t)len);
        const uint16_t *qrow = query + u * head_dim;
        for (int d = 0; d < head_dim; ++d) q[d] = widen_bf16(qrow[d]);
        const int32_t *table = block_tables + (int64_t)s * max_blocks;
        gather_rows(k, key_cache, table, 0, len, kv_head, num_kv_heads, head_dim, block_size);
        gather_rows(v, value_cache, table, 0, len, kv_head, num_kv_heads, head_dim, block_size);
        double m, l;
        partial_attention(&m, &l, o, q, k, v, len, head_dim, scale, x);
        for (int d = 0; d < head_dim; ++d) o[d] /= l;
        free(q); free(k); free(v); free(x);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
