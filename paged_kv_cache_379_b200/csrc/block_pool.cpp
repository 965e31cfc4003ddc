// block_pool.cpp -- host-side KV block pool behind the pa_pool_* C ABI.
//
// The pool owns no device memory: it hands out physical block ids, keeps their
// reference counts and decides copy-on-write, so that a serving loop (or the
// benchmark) can build the block tables, slot mappings and copy pairs that the
// kernels consume.
//
// Pages followed:
//   "vLLM 源码解析：PagedAttention 如何让大模型推理提速 10 倍", §三 (BlockAllocator:
//     allocate / free / get_num_free_blocks), §五 (allocate_or_get_cow), §六 (only
//     the next page is reserved, when the last one is full);
//   "vLLM 核心源码深度解析 …", «内存分配与回收流程» (free_list with O(1) pop and
//     push), «核心方法 allocate» (free_list.pop()), «Copy-on-Write 与 Prefix Caching»
//     (shared prompt blocks carry a reference count; a write copies the block,
//     writes the new value and decrements the count);
//   "论文专题讲解：vLLM / PagedAttention …", «共享前缀和 copy-on-write» and
//     «Block table：为什么它能减少碎片» (Figure 6).
//
// The free list is a vector used as a stack: the last entry is handed out first,
// freed blocks are pushed on the end.  Both are O(1).

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pagedkv.h"

struct pa_pool {
    int num_blocks;
    int block_size;
    std::vector<int32_t> free_stack;   // top = back()
    std::vector<int32_t> refcount;
    // prefix cache: chained hash of a full block's tokens -> the block holding them
    std::unordered_map<uint64_t, int32_t> cache;
    std::vector<uint64_t> block_hash;  // hash a block is registered under
    std::vector<char> registered;
};

namespace {

// 64-bit FNV-1a (offset basis 14695981039346656037, prime 1099511628211).
constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv1a(uint64_t h, const unsigned char *bytes, size_t n)
{
    for (size_t i = 0; i < n; ++i) {
        h ^= bytes[i];
        h *= kFnvPrime;
    }
    return h;
}

// Drop a block's prefix-cache entry (when it returns to the free list).
void unregister_block(pa_pool *pool, int32_t b)
{
    if (!pool->registered[b]) return;
    auto it = pool->cache.find(pool->block_hash[b]);
    if (it != pool->cache.end() && it->second == b) pool->cache.erase(it);
    pool->registered[b] = 0;
}

}  // namespace

extern "C" {

pa_pool *pa_pool_create(int num_blocks, int block_size, const int32_t *free_order)
{
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pa_pool *p = new (std::nothrow) pa_pool;
    if (!p) return nullptr;
    try {
        p->num_blocks = num_blocks;
        p->block_size = block_size;
        p->refcount.assign(num_blocks, 0);
        p->block_hash.assign(num_blocks, 0);
        p->registered.assign(num_blocks, 0);
        p->free_stack.resize(num_blocks);
        if (free_order) {
            std::vector<char> seen(num_blocks, 0);
            for (int i = 0; i < num_blocks; ++i) {
                int32_t b = free_order[i];
                if (b < 0 || b >= num_blocks || seen[b]) { delete p; return nullptr; }
                seen[b] = 1;
                p->free_stack[i] = b;
            }
        } else {
            for (int i = 0; i < num_blocks; ++i) p->free_stack[i] = i;
        }
    } catch (...) {
        delete p;
        return nullptr;
    }
    return p;
}

void pa_pool_destroy(pa_pool *pool) { delete pool; }

int pa_pool_num_free(const pa_pool *pool)
{
    if (!pool) return PA_ERR_NULL_POINTER;
    return (int)pool->free_stack.size();
}

int pa_pool_num_blocks(const pa_pool *pool)
{
    if (!pool) return PA_ERR_NULL_POINTER;
    return pool->num_blocks;
}

int pa_pool_refcount(const pa_pool *pool, int block)
{
    if (!pool) return PA_ERR_NULL_POINTER;
    if (block < 0 || block >= pool->num_blocks) return PA_ERR_BAD_BLOCK;
    return pool->refcount[block];
}

int pa_pool_allocate(pa_pool *pool, int n, int32_t *out_ids)
{
    if (!pool || (n > 0 && !out_ids)) return PA_ERR_NULL_POINTER;
    if (n < 0) return PA_ERR_BAD_SHAPE;
    if ((size_t)n > pool->free_stack.size()) return PA_ERR_POOL_EXHAUSTED;
    for (int i = 0; i < n; ++i) {
        int32_t b = pool->free_stack.back();
        pool->free_stack.pop_back();
        pool->refcount[b] = 1;
        out_ids[i] = b;
    }
    return PA_OK;
}

int pa_pool_free(pa_pool *pool, int block)
{
    if (!pool) return PA_ERR_NULL_POINTER;
    if (block < 0 || block >= pool->num_blocks || pool->refcount[block] <= 0) return PA_ERR_BAD_BLOCK;
    if (--pool->refcount[block] == 0) {
        unregister_block(pool, block);
        pool->free_stack.push_back(block);
    }
    return PA_OK;
}

int pa_pool_fork(pa_pool *pool, const int32_t *ids, int n)
{
    if (!pool || (n > 0 && !ids)) return PA_ERR_NULL_POINTER;
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= pool->num_blocks || pool->refcount[ids[i]] <= 0) return PA_ERR_BAD_BLOCK;
    for (int i = 0; i < n; ++i) ++pool->refcount[ids[i]];
    return PA_OK;
}

int pa_pool_cow(pa_pool *pool, int block, int32_t *out_block, int32_t *copied)
{
    if (!pool || !out_block || !copied) return PA_ERR_NULL_POINTER;
    if (block < 0 || block >= pool->num_blocks || pool->refcount[block] <= 0) return PA_ERR_BAD_BLOCK;
    if (pool->refcount[block] > 1) {
        if (pool->free_stack.empty()) return PA_ERR_POOL_EXHAUSTED;
        int32_t fresh = pool->free_stack.back();
        pool->free_stack.pop_back();
        pool->refcount[fresh] = 1;
        --pool->refcount[block];
        *out_block = fresh;
        *copied = 1;
    } else {
        *out_block = block;
        *copied = 0;
    }
    return PA_OK;
}

int pa_pool_import(pa_pool *pool, const int32_t *block_tables, int num_seqs, int max_blocks,
                   const int32_t *num_table_blocks)
{
    if (!pool || (num_seqs > 0 && (!block_tables || !num_table_blocks))) return PA_ERR_NULL_POINTER;
    if (num_seqs < 0 || max_blocks < 0) return PA_ERR_BAD_SHAPE;
    for (int s = 0; s < num_seqs; ++s) {
        if (num_table_blocks[s] < 0 || num_table_blocks[s] > max_blocks) return PA_ERR_BAD_SHAPE;
        for (int j = 0; j < num_table_blocks[s]; ++j) {
            int32_t b = block_tables[(int64_t)s * max_blocks + j];
            if (b < 0 || b >= pool->num_blocks) return PA_ERR_BAD_BLOCK;
        }
    }
    for (int s = 0; s < num_seqs; ++s)
        for (int j = 0; j < num_table_blocks[s]; ++j) ++pool->refcount[block_tables[(int64_t)s * max_blocks + j]];
    std::vector<int32_t> kept;
    kept.reserve(pool->free_stack.size());
    for (int32_t b : pool->free_stack)
        if (pool->refcount[b] == 0) kept.push_back(b);
    pool->free_stack.swap(kept);
    return PA_OK;
}

int pa_pool_prepare_decode(pa_pool *pool, int num_seqs, int32_t *block_tables, int max_blocks,
                           int32_t *num_table_blocks, const int32_t *context_lens,
                           int64_t *slot_mapping, int64_t *src_dst_pairs, int *num_pairs)
{
    if (!pool || !num_pairs) return PA_ERR_NULL_POINTER;
    if (num_seqs > 0 && (!block_tables || !num_table_blocks || !context_lens || !slot_mapping || !src_dst_pairs))
        return PA_ERR_NULL_POINTER;
    if (num_seqs < 0 || max_blocks <= 0) return PA_ERR_BAD_SHAPE;
    const int bs = pool->block_size;
    *num_pairs = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t pos = context_lens[s];
        if (pos < 0) return PA_ERR_BAD_SHAPE;
        int64_t logical = pos / bs;
        int64_t offset = pos % bs;
        int32_t *row = block_tables + (int64_t)s * max_blocks;
        int32_t have = num_table_blocks[s];
        if (logical == have) {
            // the last page is full (or there is none): reserve the next page
            if (offset != 0) return PA_ERR_BAD_SHAPE;
            if (have >= max_blocks) return PA_ERR_BAD_SHAPE;
            int32_t fresh;
            int rc = pa_pool_allocate(pool, 1, &fresh);
            if (rc != PA_OK) return rc;
            row[have] = fresh;
            num_table_blocks[s] = have + 1;
        } else if (logical < have) {
            int32_t target, copied;
            int rc = pa_pool_cow(pool, row[logical], &target, &copied);
            if (rc != PA_OK) return rc;
            if (copied) {
                src_dst_pairs[2 * (*num_pairs)] = row[logical];
                src_dst_pairs[2 * (*num_pairs) + 1] = target;
                ++*num_pairs;
                row[logical] = target;
            }
        } else {
            return PA_ERR_BAD_SHAPE;
        }
        slot_mapping[s] = (int64_t)row[logical] * bs + offset;
    }
    return PA_OK;
}

int pa_prefix_groups(const int32_t *block_tables, int num_seqs, int max_blocks, const int32_t *seq_lens,
                     int block_size, int partition_size, int32_t *group_start, int32_t *group_parts,
                     int *num_groups)
{
    if (num_seqs < 0 || max_blocks <= 0 || block_size <= 0 || partition_size <= 0 ||
        partition_size % block_size != 0)
        return PA_ERR_BAD_SHAPE;
    if (!num_groups || (num_seqs > 0 && (!block_tables || !seq_lens || !group_start || !group_parts)))
        return PA_ERR_NULL_POINTER;
    const int bpp = partition_size / block_size;  // blocks per partition
    // whole partitions that sequences a and b share: equal leading table
    // entries, within both lengths and both table rows
    auto shared_parts = [&](int a, int b) -> int {
        const int64_t la = std::max(seq_lens[a], 0), lb = std::max(seq_lens[b], 0);
        const int64_t parts = std::min(std::min(la, lb) / partition_size, (int64_t)max_blocks / bpp);
        const int32_t *ra = block_tables + (int64_t)a * max_blocks;
        const int32_t *rb = block_tables + (int64_t)b * max_blocks;
        int64_t blk = 0;
        while (blk < parts * bpp && ra[blk] == rb[blk] && ra[blk] >= 0) ++blk;
        return (int)(blk / bpp);
    };
    int g = 0, s = 0;
    while (s < num_seqs) {
        int parts = INT32_MAX, e = s + 1;
        while (e < num_seqs) {
            const int k = shared_parts(s, e);
            if (k < 1) break;
            parts = std::min(parts, k);
            ++e;
        }
        group_start[g] = s;
        group_parts[g] = e > s + 1 ? parts : 0;
        ++g;
        s = e;
    }
    group_start[g] = num_seqs;
    *num_groups = g;
    return PA_OK;
}

int pa_cow_sources(const int64_t *slot_mapping, int num_seqs, int block_size, const int64_t *src_dst_pairs,
                   int num_pairs, int32_t *cow_src)
{
    if (num_seqs < 0 || num_pairs < 0 || block_size <= 0) return PA_ERR_BAD_SHAPE;
    if ((num_seqs > 0 && (!slot_mapping || !cow_src)) || (num_pairs > 0 && !src_dst_pairs))
        return PA_ERR_NULL_POINTER;
    std::unordered_map<int64_t, int64_t> src_of;  // dst block -> src block
    src_of.reserve((size_t)num_pairs * 2);
    for (int p = 0; p < num_pairs; ++p)
        if (!src_of.emplace(src_dst_pairs[2 * p + 1], src_dst_pairs[2 * p]).second) return PA_ERR_BAD_SHAPE;
    for (int s = 0; s < num_seqs; ++s) {
        cow_src[s] = -1;
        if (slot_mapping[s] < 0) continue;
        const auto it = src_of.find(slot_mapping[s] / block_size);
        if (it != src_of.end()) cow_src[s] = (int32_t)it->second;
    }
    return PA_OK;
}

int pa_pool_free_table(pa_pool *pool, const int32_t *table, int n)
{
    if (!pool || (n > 0 && !table)) return PA_ERR_NULL_POINTER;
    for (int i = 0; i < n; ++i) {
        int rc = pa_pool_free(pool, table[i]);
        if (rc != PA_OK) return rc;
    }
    return PA_OK;
}

// Swap planning between two pools (the GPU pool and a host-memory pool, as in
// the GPU/CPU two-level allocator with swap of "vLLM 核心源码深度解析 …",
// «BlockAllocator 源码核心»): every distinct block of `table` gets a block in
// `dst`, the table is rewritten to the new ids, the source blocks lose the
// table's reference, and one (src, dst) pair per distinct block is emitted.
int pa_pool_swap_plan(pa_pool *src, pa_pool *dst, int32_t *table, int n, int64_t *src_dst_pairs, int *num_pairs)
{
    if (!src || !dst || !num_pairs || (n > 0 && (!table || !src_dst_pairs))) return PA_ERR_NULL_POINTER;
    if (n < 0) return PA_ERR_BAD_SHAPE;
    if (src->block_size != dst->block_size) return PA_ERR_BAD_SHAPE;
    std::unordered_map<int32_t, int32_t> moved;
    for (int i = 0; i < n; ++i) {
        const int32_t b = table[i];
        if (b < 0 || b >= src->num_blocks || src->refcount[b] <= 0) return PA_ERR_BAD_BLOCK;
        moved.emplace(b, -1);
    }
    if (moved.size() > dst->free_stack.size()) return PA_ERR_POOL_EXHAUSTED;
    int np = 0;
    for (int i = 0; i < n; ++i) {
        const int32_t b = table[i];
        int32_t &d = moved[b];
        if (d < 0) {
            d = dst->free_stack.back();
            dst->free_stack.pop_back();
            dst->refcount[d] = 0;
            src_dst_pairs[2 * np] = b;
            src_dst_pairs[2 * np + 1] = d;
            ++np;
        }
        ++dst->refcount[d];
        table[i] = d;
        pa_pool_free(src, b);
    }
    *num_pairs = np;
    return PA_OK;
}

// Prefix caching ("vLLM 核心源码深度解析 …", «Copy-on-Write 与 Prefix Caching»: a
// block is identified by the hash of its tokens, so a request whose prompt
// starts with the same tokens references the existing blocks -- an O(1)
// lookup).  The hash is chained with the previous block's, so two equal blocks
// behind different prefixes do not match.
uint64_t pa_block_hash(uint64_t parent_hash, const int32_t *token_ids, int num_tokens)
{
    unsigned char buf[8];
    for (int i = 0; i < 8; ++i) buf[i] = (unsigned char)(parent_hash >> (8 * i));
    uint64_t h = fnv1a(kFnvOffset, buf, 8);
    for (int t = 0; t < num_tokens; ++t) {
        const uint32_t v = (uint32_t)token_ids[t];
        unsigned char tb[4] = {(unsigned char)v, (unsigned char)(v >> 8), (unsigned char)(v >> 16),
                               (unsigned char)(v >> 24)};
        h = fnv1a(h, tb, 4);
    }
    return h;
}

int pa_pool_allocate_prompt_cached(pa_pool *pool, const int32_t *token_ids, int num_tokens, int32_t *table_out,
                                   int max_blocks, int *num_table_blocks, int *num_cached_tokens)
{
    if (!pool || !table_out || !num_table_blocks || !num_cached_tokens || (num_tokens > 0 && !token_ids))
        return PA_ERR_NULL_POINTER;
    if (num_tokens < 0) return PA_ERR_BAD_SHAPE;
    const int bs = pool->block_size;
    const int n_full = num_tokens / bs;
    const int n_all = (num_tokens + bs - 1) / bs;
    if (n_all > max_blocks) return PA_ERR_BAD_SHAPE;
    // blocks this prompt must take from the free list: everything after the leading cached run
    std::vector<uint64_t> hashes(n_full);
    uint64_t parent = 0;
    int hits = 0;
    for (int j = 0; j < n_full; ++j) {
        hashes[j] = pa_block_hash(parent, token_ids + (int64_t)j * bs, bs);
        parent = hashes[j];
        if (hits == j) {
            auto it = pool->cache.find(hashes[j]);
            if (it != pool->cache.end() && pool->refcount[it->second] > 0) ++hits;
        }
    }
    if ((size_t)(n_all - hits) > pool->free_stack.size()) return PA_ERR_POOL_EXHAUSTED;
    for (int j = 0; j < hits; ++j) {
        const int32_t b = pool->cache.find(hashes[j])->second;
        ++pool->refcount[b];
        table_out[j] = b;
    }
    for (int j = hits; j < n_all; ++j) {
        const int32_t b = pool->free_stack.back();
        pool->free_stack.pop_back();
        pool->refcount[b] = 1;
        table_out[j] = b;
        if (j < n_full) {  // a full block: later prompts with this prefix may reuse it
            auto it = pool->cache.find(hashes[j]);
            if (it != pool->cache.end()) pool->registered[it->second] = 0;
            pool->cache[hashes[j]] = b;
            pool->block_hash[b] = hashes[j];
            pool->registered[b] = 1;
        }
    }
    *num_table_blocks = n_all;
    *num_cached_tokens = hits * bs;
    return PA_OK;
}

int pa_pool_num_cached_blocks(const pa_pool *pool)
{
    if (!pool) return PA_ERR_NULL_POINTER;
    return (int)pool->cache.size();
}

}  // extern "C"
