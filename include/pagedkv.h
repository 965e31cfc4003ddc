/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged-KV decode attention for B200 (sm_100a).
 *
 * Pages cited (by title and section):
 *   [源码解析]  "vLLM 源码解析：PagedAttention 如何让大模型推理提速 10 倍"
 *   [深度解析]  "vLLM 核心源码深度解析：PagedAttention 的 KV Cache 管理、Scheduler
 *               调度引擎与 Continuous Batching 实现全解"
 *   [论文专题]  "论文专题讲解：vLLM / PagedAttention：为什么 KV cache 需要分页管理"
 *
 * Common conventions
 * ------------------
 * - Every pointer argument named *_cache, query, key, value, out, block_tables,
 *   seq_lens, slot_mapping, src_dst_pairs, positions, seq_ids or workspace is
 *   DEVICE memory owned by the caller.  The library allocates no device memory
 *   and keeps no per-call state; all launches are asynchronous on `stream`
 *   (a cudaStream_t passed as void*, NULL = the legacy default stream).
 * - bf16 tensors are passed as void* and hold IEEE bfloat16 bit patterns.
 * - KV cache layout ([源码解析 §四]): key_cache and value_cache are each
 *   bf16 [num_blocks, block_size, num_kv_heads, head_dim], row-major; the page's
 *   `num_heads` is read as the number of KV heads.
 * - Block tables ([深度解析 «Block Table 数据结构»], [源码解析 §三]): int32
 *   [num_seqs, max_blocks_per_seq], row s lists the physical block of each of
 *   sequence s's logical blocks in order; entries past ceil(seq_len/block_size)
 *   are never read.  A position pos lives in physical block
 *   block_tables[s][pos / block_size] at offset pos % block_size.
 * - Supported shapes: head_dim in {64, 128}; block_size in {4, 8, 16};
 *   num_heads = G * num_kv_heads with G in 1..16.  Query head h reads KV head
 *   h / G.
 * - Return value: PA_OK (0) on success, a negative PA_ERR_* code otherwise.
 *   Argument errors are detected on the host before any launch and nothing is
 *   launched.  A launch failure returns PA_ERR_CUDA (pa_last_cuda_error() gives
 *   the cudaError_t).  The library never aborts the process and never traps on
 *   the device.
 * - Every kernel is launched with programmatic dependent launch and lets the
 *   next kernel of the stream start early.  The decode kernels read seq_lens,
 *   block_tables and query, and the pa_append_decode_kv* kernels seq_lens,
 *   block_tables, cow_src and the new key / value rows, before waiting for the
 *   previous kernel of the stream to finish (everything else after it); no
 *   kernel of this library writes those, and a kernel launched without that
 *   attribute (or one that never triggers its dependents early) is waited for
 *   as usual.
 * - Preconditions NOT checked in the launch path (pa_validate_tables checks
 *   them on the device): table entries below num_blocks for the blocks a
 *   sequence uses; ceil(seq_len/block_size) <= max_blocks_per_seq;
 *   0 <= seq_len <= max_seq_len; copy pairs with distinct destinations that are
 *   not also sources.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_OK 0
#define PA_ERR_NULL_POINTER (-1)   /* a required pointer is NULL                     */
#define PA_ERR_BAD_SHAPE (-2)      /* a size is <= 0, inconsistent or too large      */
#define PA_ERR_UNSUPPORTED (-3)    /* head_dim / block_size / group not compiled in  */
#define PA_ERR_WORKSPACE (-4)      /* workspace missing or smaller than required     */
#define PA_ERR_CUDA (-5)           /* a CUDA runtime or driver call failed           */
#define PA_ERR_POOL_EXHAUSTED (-6) /* the host block pool has too few free blocks    */
#define PA_ERR_BAD_BLOCK (-7)      /* a block id outside the pool / not allocated    */
#define PA_ERR_ALIGNMENT (-8)      /* a device pointer is not 16-byte aligned         */
#define PA_ERR_DEVICE_TIMEOUT (-9) /* a bounded on-device wait gave up (see below)   */
#define PA_ERR_SCRATCH_TOO_SMALL (-10) /* the built-in scratch of the no-allocation call is too small */
#define PA_ERR_NOT_DEVICE_ACCESSIBLE (-11) /* a pointer the kernel would read is not device-accessible */
#define PA_ERR_VALUE_RANGE (-12)   /* a kernel met a value outside its operand range (see pa_prefill) */

/* Human-readable name of a status code (static string, never NULL). */
const char *pa_status_string(int status);

/* cudaError_t of the last failing CUDA call in this thread (0 if none). */
int pa_last_cuda_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int pa_version(void);

/* --------------------------------------------------------------------------
 * a1. Address translation / slot mapping ([深度解析 «Block Table 数据结构»]):
 *     slot_mapping[t] = block_tables[seq][pos / block_size] * block_size
 *                       + pos % block_size
 * for token t of sequence seq at logical position pos.
 *   seq_ids   int32 [num_tokens] or NULL (token t belongs to sequence t);
 *   positions int64 [num_tokens] or NULL (decode: pos = seq_lens[seq] - 1);
 *   seq_lens  int32 [num_seqs], read only when positions is NULL.
 * block_tables has num_seqs rows.  A negative position, a seq_id outside
 * [0, num_seqs), a position past the table row, a negative table entry, or
 * seq_len == 0 in decode form yields slot -1.  Without seq_ids, num_tokens
 * must not exceed num_seqs.
 * Output slot_mapping: int64 [num_tokens].
 * ------------------------------------------------------------------------ */
int pa_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables, int num_seqs,
                    int max_blocks_per_seq, const int32_t *seq_ids, const int64_t *positions,
                    const int32_t *seq_lens, int num_tokens, int block_size, void *stream);

/* --------------------------------------------------------------------------
 * a2. Cache write ("reshape_and_cache"): the new tokens' K and V rows are
 * stored at their slots ([论文专题 «Continuous batching 为什么离不开内存管理»]:
 * generated K/V are written back into the owning block).
 *   key, value: bf16 [num_tokens, num_kv_heads, head_dim], contiguous;
 *   key_cache[slot / bs][slot % bs][h][:] = key[t][h][:] (same for value);
 *   slot_mapping: int64 [num_tokens]; a negative slot skips the token.
 * Slots must be < num_blocks * block_size and distinct among non-negative ones.
 * ------------------------------------------------------------------------ */
int pa_reshape_and_cache(const void *key, const void *value, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, void *stream);

/* --------------------------------------------------------------------------
 * a1 + a2 in one launch, decode form: for each sequence s, its newest position
 * pos = seq_lens[s] - 1 is translated to a slot exactly as pa_slot_mapping does
 * (slot -1 when seq_lens[s] == 0, the position falls past the table row, or
 * the table entry is negative) and key[s] / value[s] (bf16 [num_seqs,
 * num_kv_heads, head_dim]) are stored there as pa_reshape_and_cache stores
 * them.  slot_mapping (int64 [num_seqs], device) receives the slots, or is
 * NULL.  The same result as pa_slot_mapping followed by pa_reshape_and_cache,
 * one kernel instead of two.  num_kv_heads * head_dim must be a multiple of 8.
 * ------------------------------------------------------------------------ */
int pa_append_decode_kv(const void *key, const void *value, void *key_cache, void *value_cache,
                        const int32_t *block_tables, const int32_t *seq_lens, int64_t *slot_mapping,
                        int num_seqs, int max_blocks_per_seq, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, void *stream);

/* --------------------------------------------------------------------------
 * a3 + a1 + a2 in one launch: the decode step's copy-on-write copies and cache
 * write ([源码解析 §五] allocate_or_get_cow: a write into a shared block goes to
 * a new block that first receives the old block's contents; [论文专题
 * «共享前缀和 copy-on-write»]).  As pa_append_decode_kv, sequence s stores
 * key[s] / value[s] at its newest position pos = seq_lens[s] - 1, in block
 * dst = block_tables[s][pos / block_size] (the table already names the new
 * block), row pos % block_size.  cow_src (int32 [num_seqs], device, or NULL =
 * no copies): when cow_src[s] >= 0, dst first receives a copy of block
 * cow_src[s] -- every row but the new token's, which gets the new K/V.  The
 * caches end up byte for byte as after pa_copy_blocks of the pairs
 * (cow_src[s], dst) followed by pa_append_decode_kv, in one kernel instead of
 * two.  cow_src entries outside [0, num_blocks) or equal to dst copy nothing;
 * a sequence whose slot is -1 (see pa_append_decode_kv) writes nothing.
 * Precondition: the destinations of sequences with a copy are distinct and are
 * not copy sources.  pa_cow_sources turns the pool's (src, dst) pairs and the
 * step's slots into cow_src.  num_seqs <= 65535.
 * ------------------------------------------------------------------------ */
int pa_append_decode_kv_cow(const void *key, const void *value, void *key_cache, void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cow_src,
                            int64_t *slot_mapping, int num_seqs, int max_blocks_per_seq, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks, void *stream);

/* --------------------------------------------------------------------------
 * a3. Copy-on-write block copy ([源码解析 §五] allocate_or_get_cow: a new block
 * receives a copy of the shared one; [深度解析 «Copy-on-Write 与 Prefix Caching»]).
 *   src_dst_pairs: int64 [num_pairs, 2] (device), pair i copies the whole
 *   physical block src -> dst in both caches (all heads, all slots).
 * num_pairs == 0 is a no-op.  Destinations must be distinct and not sources;
 * a pair naming a block outside [0, num_blocks) is skipped.
 * ------------------------------------------------------------------------ */
int pa_copy_blocks(void *key_cache, void *value_cache, const int64_t *src_dst_pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, void *stream);

/* --------------------------------------------------------------------------
 * Swap of whole blocks between two caches in different memories -- the GPU
 * cache and a cache in pinned host memory -- for a two-level GPU/CPU block
 * allocator that swaps cold blocks out to host memory when the GPU runs short
 * and back in when they are needed ([深度解析 «BlockAllocator 源码核心»],
 * CpuGpuBlockAllocator).  Pair i copies src block src_dst_pairs[i][0] of
 * (src_key_cache, src_value_cache) to dst block src_dst_pairs[i][1] of
 * (dst_key_cache, dst_value_cache); both caches are [num_blocks, block_size,
 * num_kv_heads, head_dim] bf16 with their own block counts.  A device kernel
 * does the gather/scatter, so host-side caches and the pairs must be
 * device-accessible: device memory or pinned, mapped host memory
 * (cudaHostAlloc / cudaMallocHost / cudaHostRegister).  Pageable host memory
 * is rejected with PA_ERR_NOT_DEVICE_ACCESSIBLE before any launch.  Pairs with
 * ids outside their cache are skipped.
 * ------------------------------------------------------------------------ */
int pa_swap_blocks(void *dst_key_cache, void *dst_value_cache, const void *src_key_cache,
                   const void *src_value_cache, const int64_t *src_dst_pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int src_num_blocks,
                   int dst_num_blocks, void *stream);

/* --------------------------------------------------------------------------
 * a4-a6. Single-query paged decode attention ([源码解析 §四] paged_attention;
 * [论文专题 «PagedAttention：逻辑连续，物理不必连续»]): for sequence s and query
 * head h, with L = seq_lens[s] and K_s, V_s read block by block through the
 * table,
 *     out[s][h] = sum_{p<L} softmax_p(scale * query[s][h] . K_s[p]) V_s[p].
 * query, out: bf16 [num_seqs, num_heads, head_dim]; accumulation in fp32,
 * output rounded to bf16 (round to nearest even).  L == 0 gives zeros.
 * max_seq_len: a host-known upper bound of seq_lens (sizes the grid; no
 * device-to-host read).
 *
 * pa_decode picks the one-pass kernel or the split form by max_seq_len and the
 * number of (sequence, KV head) units.  It takes a workspace of at least
 * pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len, 0)
 * bytes, or none (workspace NULL: one pass, work handed out round-robin).
 *
 * Workspace contract (all decode entry points that take one): caller-owned
 * device memory, 16-byte aligned.  Its first 256 bytes hold the counters of
 * the kernels' dynamic work scheduler: ZERO-FILL THE WORKSPACE ONCE after
 * allocating it (e.g. cudaMemsetAsync); every call leaves those bytes zero
 * again when it completes.  The rest is scratch (no initialisation needed).
 * Calls that may run concurrently must not share a workspace.  After
 * pa_device_status() has reported a timeout, zero the workspace again.
 *
 * The decode kernel is persistent: (resident CTAs per SM) x (SMs) CTAs loop
 * over (sequence, partition, KV head) work items.  Sequence count limit: the
 * per-CTA enumeration tables (10 bytes per sequence) must fit in shared memory
 * next to the pipeline (num_seqs up to about 11000); beyond that the call
 * returns PA_ERR_BAD_SHAPE.
 * ------------------------------------------------------------------------ */
int pa_decode(void *out, const void *query, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
              int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
              int num_blocks, int max_seq_len, void *workspace, size_t workspace_bytes,
              void *stream);

/* The plan pa_decode follows for these sizes: 0 = one pass (one launch),
 * otherwise the partition size of the split form (partition kernel + reduce
 * kernel, two launches).  One pass when max_seq_len <= 4096 and the
 * (sequence, KV head) units give every SM several items; else partitions of
 * 1024 positions (2048 beyond 16384), halved while the batch is too small to
 * give every SM several items.  A workspace smaller than the split form needs
 * gives one pass.  No device work. */
int pa_decode_plan(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_seq_len,
                   size_t workspace_bytes);

/* Workspace bytes pa_decode / pa_decode_split need.  partition_size <= 0 means
 * the plan pa_decode would choose for these sizes (256 bytes when that plan is
 * one pass).  0 for invalid sizes. */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                int max_seq_len, int partition_size);

/* a4 alone: each (sequence, KV head) work item walks all of the sequence's
 * blocks with an online softmax ("逐块计算局部 Attention，最后合并结果",
 * [源码解析 §四]).  No workspace: items are handed out round-robin. */
int pa_decode_one_pass(void *out, const void *query, const void *key_cache,
                       const void *value_cache, const int32_t *block_tables,
                       const int32_t *seq_lens, float scale, int block_size, int num_kv_heads,
                       int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                       int num_blocks, int max_seq_len, void *stream);

/* a5 + a6: positions are cut into partitions of partition_size tokens (a
 * multiple of 16, >= 16); each (sequence, partition, KV head) work item
 * computes the partition's local result, and a log-sum-exp reduce kernel
 * merges them.  A sequence that fits in one partition is written directly. */
int pa_decode_split(void *out, const void *query, const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *seq_lens, float scale,
                    int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                    int max_blocks_per_seq, int num_blocks, int max_seq_len, int partition_size,
                    void *workspace, size_t workspace_bytes, void *stream);

/* a5 + a6 with shared prefixes read once per group of sequences.  When
 * several sequences' tables start with the same blocks -- the prompt blocks
 * that parallel sampling or a fork leaves shared ([论文专题 «共享前缀和
 * copy-on-write»]: the samples reference the prompt's blocks; [深度解析
 * «Copy-on-Write 与 Prefix Caching»]) -- the decode reads those blocks once per
 * KV head for several sequences at a time instead of once per sequence.
 * Groups (device arrays, e.g. from pa_prefix_groups): group g is sequences
 * group_start[g] .. group_start[g+1]-1 (int32 [num_groups + 1]); its first
 * group_parts[g] partitions (int32 [num_groups]) are computed once for up to
 * 16 / G of its sequences per work item (G = num_heads / num_kv_heads) and
 * every later partition per sequence.  The result is that of pa_decode_split
 * with the same partition_size (same workspace size).  Preconditions: groups
 * cover sequences 0 .. num_seqs-1 in order; within group g every sequence's
 * table entries for the first group_parts[g] * partition_size positions equal
 * those of the group's first sequence, and every sequence's length is at
 * least group_parts[g] * partition_size (pa_prefix_groups builds such groups).
 * bf16 caches only (G <= 16). */
int pa_decode_shared(void *out, const void *query, const void *key_cache, const void *value_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                     int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                     int num_blocks, int max_seq_len, int partition_size, const int32_t *group_start,
                     const int32_t *group_parts, int num_groups, void *workspace, size_t workspace_bytes,
                     void *stream);

/* a5 alone, for inspection: every partition p < ceil(max_seq_len/partition_size)
 * of every (s, h) writes its local result into the workspace, laid out as
 *   the 256-byte scheduler header,
 *   float o[num_seqs][num_heads][max_parts][head_dim]  at byte 256,
 *   float m[num_seqs][num_heads][max_parts]           after o (256-B aligned),
 *   float l[num_seqs][num_heads][max_parts]           after m (256-B aligned),
 * with max_parts = ceil(max_seq_len / partition_size) (at least 1):
 *   m = max_p scale*q.k_p (natural-log units), l = sum_p exp(x_p - m),
 *   o = sum_p exp(x_p - m) v_p (not normalised).
 * Partitions holding no position of their sequence get m = -inf, l = 0, o = 0. */
int pa_decode_partitions(const void *query, const void *key_cache, const void *value_cache,
                         const int32_t *block_tables, const int32_t *seq_lens, float scale,
                         int block_size, int num_kv_heads, int num_seqs, int num_heads,
                         int head_dim, int max_blocks_per_seq, int num_blocks, int max_seq_len,
                         int partition_size, void *workspace, size_t workspace_bytes,
                         void *stream);

/* a6 alone: merge the partitions that pa_decode_partitions wrote
 * (out = sum_p e^{m_p-M} o_p / sum_p e^{m_p-M} l_p, M = max_p m_p) into bf16 out. */
int pa_lse_reduce(void *out, const void *workspace, const int32_t *seq_lens, int num_seqs,
                  int num_heads, int head_dim, int max_seq_len, int partition_size,
                  void *stream);

/* --------------------------------------------------------------------------
 * FP8 KV cache ([深度解析], milestone list: "FP8 KV Cache" -- one byte per
 * cached K/V element).  key_cache and value_cache hold OCP FP8 E4M3 codes
 * (uint8 [num_blocks, block_size, num_kv_heads, head_dim]: sign, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent 0 subnormal; S.1111.111 NaN;
 * largest finite magnitude 448).  A code c stands for e4m3(c) * k_scale in the
 * key cache and e4m3(c) * v_scale in the value cache: one positive, finite
 * fp32 scale per cache tensor (otherwise PA_ERR_BAD_SHAPE).
 *
 * pa_reshape_and_cache_fp8: pa_reshape_and_cache with quantisation.  key and
 * value are bf16 [num_tokens, num_kv_heads, head_dim]; each element x becomes
 * the code nearest to fp32(x * fp32(1 / scale)) (the inverse scale rounded to
 * fp32 once; ties to the even code; magnitudes beyond 448, infinities
 * included, saturate to +-448; NaN gives 0x7F).  num_kv_heads * head_dim must
 * be a multiple of 16 (PA_ERR_UNSUPPORTED otherwise).  Slot rules as in
 * pa_reshape_and_cache.
 * ------------------------------------------------------------------------ */
int pa_reshape_and_cache_fp8(const void *key, const void *value, void *key_cache,
                             void *value_cache, const int64_t *slot_mapping, int num_tokens,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                             float k_scale, float v_scale, void *stream);

/* pa_append_decode_kv into FP8 caches: the slot rules of pa_append_decode_kv,
 * the quantisation of pa_reshape_and_cache_fp8 (num_kv_heads * head_dim a
 * multiple of 16). */
int pa_append_decode_kv_fp8(const void *key, const void *value, void *key_cache, void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens,
                            int64_t *slot_mapping, int num_seqs, int max_blocks_per_seq,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            float k_scale, float v_scale, void *stream);

/* pa_decode over an FP8 cache: the same result with K = e4m3(code) * k_scale
 * and V = e4m3(code) * v_scale.  query and out stay bf16.  Supported: head_dim
 * 128, block_size 8 or 16, G = num_heads / num_kv_heads in 1..16
 * (PA_ERR_UNSUPPORTED otherwise).  The logits are E4M3 x E4M3 tensor-core
 * products accumulated in fp32: each query head is scaled by a power of two
 * (its largest |q| into [128, 256)) and split into two E4M3 terms whose sum is
 * the bf16 query exactly for every element within 2^9 of the head's largest
 * (smaller elements are off by less than 2^-17 of the largest).  The value
 * product widens the codes to fp16 (exact) and takes the softmax weights as
 * fp16.  Same plan, workspace contract and workspace size as pa_decode. */
int pa_decode_fp8(void *out, const void *query, const void *key_cache, const void *value_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, float scale, float k_scale,
                  float v_scale, int block_size, int num_kv_heads, int num_seqs, int num_heads,
                  int head_dim, int max_blocks_per_seq, int num_blocks, int max_seq_len,
                  void *workspace, size_t workspace_bytes, void *stream);

/* pa_decode_fp8 with an explicit plan: partition_size 0 = one pass (workspace
 * optional: NULL hands items out round-robin), otherwise the split form of
 * pa_decode_split with that partition size (workspace required). */
int pa_decode_fp8_split(void *out, const void *query, const void *key_cache,
                        const void *value_cache, const int32_t *block_tables,
                        const int32_t *seq_lens, float scale, float k_scale, float v_scale,
                        int block_size, int num_kv_heads, int num_seqs, int num_heads,
                        int head_dim, int max_blocks_per_seq, int num_blocks, int max_seq_len,
                        int partition_size, void *workspace, size_t workspace_bytes,
                        void *stream);

/* --------------------------------------------------------------------------
 * Multi-query paged prefill: the chunked-prefill step ([深度解析], milestone
 * list: v0.5 "Chunked Prefill" -- a long prompt is fed in chunks so that it
 * does not hold up decodes) with the causal rule of [论文专题] (the query at
 * position i attends to positions up to and including i).
 *   seq_lens  int32 [num_seqs]: cached positions of each sequence, this
 *             chunk's tokens included (their K/V rows are already in the cache,
 *             e.g. written by pa_reshape_and_cache);
 *   q_start   int32 [num_seqs + 1] (device): the chunk of sequence s is query
 *             rows q_start[s] .. q_start[s+1]-1, in position order, and holds
 *             its last q_len = q_start[s+1] - q_start[s] positions;
 *   query, out: bf16 [num_tokens, num_heads, head_dim], num_tokens = q_start[num_seqs].
 * Row q_start[s] + i (position p = seq_len - q_len + i) gets
 *     out = sum_{j <= p} softmax_j(scale * q . k_j) v_j,
 * with K/V read block by block through the table.  Sequences with q_len <= 0
 * or q_len > seq_len are skipped (their rows are not written).
 * Supported: head_dim 64 or 128, block_size 8, 16 or 32, G = num_heads /
 * num_kv_heads in 1..16; scale > 0 (the kernel takes a row's max logit before
 * scaling it, so a non-positive scale is outside the contract).  fp32 accumulation on the tensor cores (tcgen05):
 * q . k in bf16; P V in fp16 -- the softmax weights rounded to fp16 and the
 * value rows converted to fp16 in shared memory, exact for 2^-17 <= |v| <=
 * 65504.  A value entry of larger magnitude that a row reads saturates to
 * +-65504 and sets PA_ERR_VALUE_RANGE in the device status (pa_device_status);
 * the output rows that attend to it are then not exact.  Output rounded to
 * bf16.  No workspace; one launch.
 * ------------------------------------------------------------------------ */
int pa_prefill(void *out, const void *query, const void *key_cache, const void *value_cache,
               const int32_t *block_tables, const int32_t *seq_lens, const int32_t *q_start,
               float scale, int block_size, int num_kv_heads, int num_seqs, int num_heads,
               int head_dim, int max_blocks_per_seq, int num_blocks, int num_tokens, void *stream);

/* --------------------------------------------------------------------------
 * Precondition check on the device: counts, into *bad_count (device int32,
 * overwritten), the sequences whose seq_len is negative or above max_seq_len,
 * whose ceil(seq_len/block_size) exceeds max_blocks_per_seq, or whose used
 * table entries fall outside [0, num_blocks).
 * ------------------------------------------------------------------------ */
int pa_validate_tables(const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                       int max_blocks_per_seq, int block_size, int num_blocks, int max_seq_len,
                       int32_t *bad_count, void *stream);

/* --------------------------------------------------------------------------
 * Split-form decode that allocates nothing and takes no workspace.
 * (The pages have no counterpart of this call; it exists for callers of this
 * library, not for the method.)
 *
 * Some callers cannot hand the library a workspace: code that must not call
 * cudaMalloc on its decode path (cudaMalloc can synchronise the device and
 * stall a latency-critical serving loop), code that runs inside another
 * framework's memory arena with no way to allocate from it, or plugin hosts
 * that fix the device memory a component may own up front.  This call keeps
 * the split form's scratch -- the scheduler counters and the per-partition
 * partial results -- in one fixed array inside the library instead:
 * PA_NOALLOC_SCRATCH_BYTES of device memory that every GPU which loads the
 * library holds until the process exits.
 *
 * Arguments and results are those of pa_decode_split without the workspace;
 * the caller still owns and passes query, caches, tables, lengths and out.
 * A problem whose split workspace (pa_decode_workspace_size with the same
 * sizes and partition_size) exceeds PA_NOALLOC_SCRATCH_BYTES is rejected with
 * PA_ERR_SCRATCH_TOO_SMALL before any launch; a larger partition_size shrinks it.
 * The call allocates no device memory and calls no allocating routine.
 * The first call on each device looks up the array's device address on that
 * device (with the device current); make that first call before any stream
 * capture.  The address is kept per CUDA context (by the context's
 * process-unique id): after cudaDeviceReset, or any other end of the context
 * the array was found in, the next call looks it up again in the new context
 * -- again a set-up call, to be made outside stream capture.  Each call clears the scheduler counters (an asynchronous memset on
 * `stream`) and leaves its partial results in the array.  All calls share the
 * one array: calls that may overlap on the GPU (different streams, or other
 * host threads) race on it and must be serialised by the caller.
 * ------------------------------------------------------------------------ */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)
int pa_decode_split_noalloc(void *out, const void *query, const void *key_cache,
                            const void *value_cache, const int32_t *block_tables,
                            const int32_t *seq_lens, float scale, int block_size,
                            int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                            int max_blocks_per_seq, int num_blocks, int max_seq_len,
                            int partition_size, void *stream);

/* Bounded waits.  Every wait inside the kernels (on TMA completion or on a
 * pipeline stage being released) gives up after about one second, records a
 * nonzero code in a device word and lets the kernel return.  This call reads
 * and clears that word for the current device (synchronising the device);
 * 0 means no wait ever gave up and no kernel met an out-of-range value;
 * otherwise PA_ERR_DEVICE_TIMEOUT, or PA_ERR_VALUE_RANGE when pa_prefill read
 * a value-cache entry of magnitude above 65504 (its P.V operand is fp16). */
int pa_device_status(void);

/* Self-test of the bounded-wait path: launches one thread that waits on an
 * mbarrier nothing ever arrives on.  The wait gives up after its limit (about
 * one second), records the timeout in the device status word and the kernel
 * returns; pa_device_status() then reports PA_ERR_DEVICE_TIMEOUT (and clears
 * it), and the context stays usable.  Returns PA_OK or PA_ERR_CUDA (launch). */
int pa_selftest_bounded_wait(void *stream);

/* --------------------------------------------------------------------------
 * a7. Host block pool (host memory only; it generates block tables, slots and
 * copy pairs, it never touches the GPU):
 *   - a free list popped from its end in O(1) ([深度解析 «内存分配与回收流程»,
 *     «核心方法 allocate»]; [源码解析 §三] allocate / free / get_num_free_blocks);
 *   - per-block reference counts; fork() adds an owner to every block of a
 *     table (parallel sampling / beam search share prompt blocks,
 *     [论文专题 «共享前缀和 copy-on-write»]);
 *   - copy-on-write: a write into a block with reference count > 1 takes a
 *     fresh block, records (src, dst) and decrements src ([源码解析 §五]);
 *   - on-demand growth: a new block only when the last one is full
 *     ([源码解析 §六]; [论文专题 «Block table：为什么它能减少碎片»], Figure 6).
 * Not thread-safe: one pool per host thread, or external locking.
 * ------------------------------------------------------------------------ */
typedef struct pa_pool pa_pool;

/* free_order: int32 [num_blocks] permutation giving the initial free list
 * (the LAST entry is handed out first), or NULL for 0..num_blocks-1.
 * Returns NULL on bad arguments or out of host memory. */
pa_pool *pa_pool_create(int num_blocks, int block_size, const int32_t *free_order);
void pa_pool_destroy(pa_pool *pool);
int pa_pool_num_free(const pa_pool *pool);
int pa_pool_num_blocks(const pa_pool *pool);
/* Reference count of a block (0 = free), or PA_ERR_BAD_BLOCK. */
int pa_pool_refcount(const pa_pool *pool, int block);
/* Take n blocks (refcount 1 each) into out_ids[n]; PA_ERR_POOL_EXHAUSTED and
 * no change if fewer than n are free. */
int pa_pool_allocate(pa_pool *pool, int n, int32_t *out_ids);
/* Drop one owner; the block returns to the free list at refcount 0. */
int pa_pool_free(pa_pool *pool, int block);
/* Add one owner to each of ids[0..n). */
int pa_pool_fork(pa_pool *pool, const int32_t *ids, int n);
/* Copy-on-write decision for a write into `block`: *out_block is the block to
 * write; *copied is 1 if a fresh block was taken (then copy block -> *out_block). */
int pa_pool_cow(pa_pool *pool, int block, int32_t *out_block, int32_t *copied);
/* Adopt existing tables (host int32 [num_seqs, max_blocks], first
 * num_table_blocks[s] entries of row s valid): every reference adds an owner and
 * referenced blocks leave the free list (the others keep their order). */
int pa_pool_import(pa_pool *pool, const int32_t *block_tables, int num_seqs, int max_blocks,
                   const int32_t *num_table_blocks);
/* One decode step's host work for a batch (all arrays host memory):
 * sequence s has context_lens[s] cached tokens and appends one at position
 * context_lens[s].  If that position opens a new logical block, a fresh block is
 * appended to row s (num_table_blocks[s] += 1); otherwise the copy-on-write
 * decision is taken for the block being written.  Outputs slot_mapping[s] and
 * the (src, dst) pairs (int64 [num_seqs, 2], *num_pairs of them).  Returns
 * PA_ERR_POOL_EXHAUSTED if the pool runs dry (sequences before the failing
 * one keep their updates) or PA_ERR_BAD_SHAPE if a row would overflow. */
int pa_pool_prepare_decode(pa_pool *pool, int num_seqs, int32_t *block_tables, int max_blocks,
                           int32_t *num_table_blocks, const int32_t *context_lens,
                           int64_t *slot_mapping, int64_t *src_dst_pairs, int *num_pairs);
/* Release every block of the first n entries of a table row. */
int pa_pool_free_table(pa_pool *pool, const int32_t *table, int n);
/* Shared-prefix groups for pa_decode_shared (host arrays): runs of
 * consecutive sequences whose tables start with the same blocks.  A run starts
 * at sequence s and takes s+1, s+2, ... while each one shares at least one
 * whole partition (partition_size positions, a multiple of block_size) with
 * the run's first sequence: identical table entries over it, and both lengths
 * covering it.  group_parts[g] = the partitions every member of group g shares
 * with the first (the minimum over the members; 0 for a sequence shared with
 * no neighbour).  Outputs group_start (int32 [num_seqs + 1]: group g is
 * sequences group_start[g] .. group_start[g+1]-1), group_parts (int32
 * [num_seqs]) and *num_groups; block_tables int32 [num_seqs, max_blocks],
 * seq_lens int32 [num_seqs]. */
int pa_prefix_groups(const int32_t *block_tables, int num_seqs, int max_blocks, const int32_t *seq_lens,
                     int block_size, int partition_size, int32_t *group_start, int32_t *group_parts,
                     int *num_groups);
/* Per-sequence copy sources for pa_append_decode_kv_cow (host arrays):
 * cow_src[s] = the src of the pair (src, dst) of src_dst_pairs (int64
 * [num_pairs, 2]) whose dst is the block of slot_mapping[s] (slot / block_size),
 * or -1 when no pair writes that block or the slot is negative.  Returns
 * PA_ERR_BAD_SHAPE if two pairs share a destination. */
int pa_cow_sources(const int64_t *slot_mapping, int num_seqs, int block_size, const int64_t *src_dst_pairs,
                   int num_pairs, int32_t *cow_src);


/* Swap planning between two pools (GPU pool and host pool): every distinct
 * block of table[0..n) gets a block in `dst` (reference count = its number of
 * entries in the table), the table is rewritten to the dst ids, each source
 * block loses those references (returning to src's free list at zero), and
 * one (src, dst) pair per distinct block is written to src_dst_pairs
 * (int64 [n, 2], host) for pa_swap_blocks.  PA_ERR_POOL_EXHAUSTED and no
 * change if dst has too few free blocks. */
int pa_pool_swap_plan(pa_pool *src, pa_pool *dst, int32_t *table, int n, int64_t *src_dst_pairs,
                      int *num_pairs);

/* --------------------------------------------------------------------------
 * Prefix caching in the host block pool ([深度解析 «Copy-on-Write 与 Prefix
 * Caching»]: a block is recognised by hash(token_ids[0:block_size]); a prompt
 * that starts with the same tokens references the existing blocks, an O(1)
 * lookup).  The hash of a full block is chained with its parent's, so equal
 * blocks behind different prefixes do not match:
 *   pa_block_hash(parent, tokens, n) = FNV-1a-64 over the 8 little-endian bytes
 *   of `parent` followed by the 4 little-endian bytes of each token id;
 *   the first block of a prompt has parent 0.
 * pa_pool_allocate_prompt_cached builds the table of a prompt of num_tokens
 * tokens: the leading run of full blocks whose chained hashes are registered
 * (and alive) is referenced (refcount + 1, *num_cached_tokens = their tokens,
 * whose K/V need no recomputation); every later block is taken from the free
 * list, and the full ones among them are registered under their hashes.  A
 * partly filled last block is never registered (it will be written).  A block
 * leaves the cache when its reference count returns to 0.  PA_ERR_POOL_EXHAUSTED
 * (no change) if the free list is too short, PA_ERR_BAD_SHAPE if the table
 * needs more than max_blocks entries.
 * ------------------------------------------------------------------------ */
uint64_t pa_block_hash(uint64_t parent_hash, const int32_t *token_ids, int num_tokens);
int pa_pool_allocate_prompt_cached(pa_pool *pool, const int32_t *token_ids, int num_tokens,
                                   int32_t *table_out, int max_blocks, int *num_table_blocks,
                                   int *num_cached_tokens);
/* Number of blocks currently registered in the prefix cache. */
int pa_pool_num_cached_blocks(const pa_pool *pool);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
