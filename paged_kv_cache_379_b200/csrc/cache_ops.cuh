// cache_ops.cuh -- the integer / byte-moving kernels of the decode step:
//   slot mapping   (address translation of a new token's position),
//   reshape_and_cache (write the new K/V rows at their slots),
//   copy_blocks    (copy-on-write block copies),
//   validate_tables (device-side precondition check).
// All of them are HBM- or launch-bound copies: 16-byte vector accesses, grid
// sized from the work, no shared memory.  Included once, by pagedkv.cu.
#pragma once

#include "common.cuh"

namespace pakv {

// Address translation ("vLLM 核心源码深度解析 …", «Block Table 数据结构»):
//   block_number = pos / block_size, offset = pos % block_size,
//   slot = block_table[block_number] * block_size + offset.
__global__ void slot_mapping_kernel(int64_t *__restrict__ slots, const int32_t *__restrict__ block_tables,
                                    int num_seqs, int max_blocks, const int32_t *__restrict__ seq_ids,
                                    const int64_t *__restrict__ positions,
                                    const int32_t *__restrict__ seq_lens, int num_tokens, int block_size)
{
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= num_tokens) return;
    const int seq = seq_ids ? seq_ids[t] : t;
    int64_t slot = -1;
    if (seq < 0 || seq >= num_seqs) {  // out-of-range sequence id: treated as padding
        slots[t] = slot;
        return;
    }
    const int64_t pos = positions ? positions[t] : (int64_t)seq_lens[seq] - 1;
    if (pos >= 0) {
        const int64_t block_number = pos / block_size;
        const int64_t offset = pos - block_number * block_size;
        if (block_number < max_blocks) {
            const int32_t physical = block_tables[(int64_t)seq * max_blocks + block_number];
            if (physical >= 0) slot = (int64_t)physical * block_size + offset;
        }
    }
    slots[t] = slot;
}

// One thread per 16-byte chunk of a token's [num_kv_heads, head_dim] row (the
// row is contiguous both in `key` and at its slot in the cache, because the
// cache is [num_blocks, block_size, num_kv_heads, head_dim]).
__global__ void reshape_and_cache_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                                         uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                                         const int64_t *__restrict__ slot_mapping, int num_tokens,
                                         int chunks_per_token, int64_t num_slots)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)num_tokens * chunks_per_token) return;
    const int64_t t = i / chunks_per_token;
    const int64_t c = i - t * chunks_per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0 || slot >= num_slots) return;
    const int64_t dst = slot * chunks_per_token + c;
    const uint4 k = key[i];
    const uint4 v = value[i];
    key_cache[dst] = k;
    value_cache[dst] = v;
}

// FP8 cache write: one thread per 16 values of a token's [num_kv_heads, head_dim]
// row (32 bytes of bf16 in, one 16-byte chunk of E4M3 codes out); each code is
// e4m3(x * inv_scale) with the product taken in fp32, rounded to nearest even,
// finite overflow saturating to +-448.
__device__ __forceinline__ uint4 quantise16(uint4 a, uint4 b, float inv)
{
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f0 = unpack_bf16x2(w[2 * i]);
        const float2 f1 = unpack_bf16x2(w[2 * i + 1]);
        const uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv));
        const uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv));
        out[i] = lo | (hi << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void reshape_and_cache_fp8_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                                             uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                                             const int64_t *__restrict__ slot_mapping, int num_tokens,
                                             int chunks_per_token, int64_t num_slots, float k_inv_scale,
                                             float v_inv_scale)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)num_tokens * chunks_per_token) return;
    const int64_t t = i / chunks_per_token;
    const int64_t c = i - t * chunks_per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0 || slot >= num_slots) return;
    const int64_t dst = slot * chunks_per_token + c;
    const uint4 k0 = key[2 * i], k1 = key[2 * i + 1];
    const uint4 v0 = value[2 * i], v1 = value[2 * i + 1];
    key_cache[dst] = quantise16(k0, k1, k_inv_scale);
    value_cache[dst] = quantise16(v0, v1, v_inv_scale);
}

// The decode step's cache write with its own address translation, in one
// launch: token s is sequence s's newest position seq_lens[s] - 1; its slot is
// computed as slot_mapping_kernel does (optionally written to slots_out) and
// its K/V row stored there -- copied (bf16) or quantised (FP8: one thread per 16
// codes).  chunks_per_token counts 16-byte chunks of the destination row.
template <bool FP8>
__global__ void append_kv_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                                 uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                                 const int32_t *__restrict__ block_tables, const int32_t *__restrict__ seq_lens,
                                 int64_t *__restrict__ slots_out, int num_seqs, int max_blocks,
                                 int chunks_per_token, int block_size, int64_t num_slots, float k_inv, float v_inv)
{
    // The lengths, the table and the new rows are inputs no kernel of this
    // library writes: they are read before waiting for the previous kernel of
    // the stream; the slot output and the cache are written after it.
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool live = i < (int64_t)num_seqs * chunks_per_token;
    int s = 0, c = 0;
    int64_t slot = -1;
    uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0, v0 = k0, v1 = k0;
    if (live) {
        s = (int)(i / chunks_per_token);
        c = (int)(i - (int64_t)s * chunks_per_token);
        if constexpr (FP8) {
            k0 = key[2 * i];
            k1 = key[2 * i + 1];
            v0 = value[2 * i];
            v1 = value[2 * i + 1];
        } else {
            k0 = key[i];
            v0 = value[i];
        }
        const int64_t pos = (int64_t)seq_lens[s] - 1;
        if (pos >= 0) {
            const int64_t block_number = pos / block_size;
            if (block_number < max_blocks) {
                const int32_t physical = block_tables[(int64_t)s * max_blocks + block_number];
                if (physical >= 0) slot = (int64_t)physical * block_size + (pos - block_number * block_size);
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (!live) return;
    if (c == 0 && slots_out) slots_out[s] = slot;
    if (slot < 0 || slot >= num_slots) return;
    const int64_t dst = slot * chunks_per_token + c;
    if constexpr (FP8) {
        key_cache[dst] = quantise16(k0, k1, k_inv);
        value_cache[dst] = quantise16(v0, v1, v_inv);
    } else {
        key_cache[dst] = k0;
        value_cache[dst] = v0;
    }
}

// The decode step's copy-on-write and cache write in one launch
// ("vLLM 源码解析 …", §五: a write into a shared block goes to a new block that
// first receives a copy of the old one; "论文专题讲解 …", «共享前缀和
// copy-on-write»).  Sequence s writes its newest position pos = seq_lens[s] - 1
// into block dst = block_tables[s][pos / bs] at row o = pos % bs.  When
// cow_src[s] >= 0, dst is a fresh block that must first hold a copy of block
// cow_src[s]: every row of cow_src[s] but row o is copied into dst, and row o
// receives the new K/V -- the bytes that a block copy followed by the cache
// write leave, with no ordering between the two needed, as no byte is written
// twice.  Grid: (row slices of the block, sequence); a CTA covers rows
// [r0, r0 + rows_per_cta) of both caches, one thread per 16-byte chunk with four
// chunks per cache in flight.  Sequences without a copy only run the CTA that
// holds row o.
__global__ void __launch_bounds__(256) append_kv_cow_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value, uint4 *__restrict__ key_cache,
    uint4 *__restrict__ value_cache, const int32_t *__restrict__ block_tables, const int32_t *__restrict__ seq_lens,
    const int32_t *__restrict__ cow_src, int64_t *__restrict__ slots_out, int max_blocks, int chunks_per_token,
    int block_size, int rows_per_cta, int64_t num_blocks)
{
    // The lengths, the table and the copy sources are inputs no kernel of this
    // library writes: they are read before waiting for the previous kernel of
    // the stream; the caches and the slot output are touched after it.
    const int s = blockIdx.y;
    const int r0 = blockIdx.x * rows_per_cta;
    const int r1 = min(block_size, r0 + rows_per_cta);
    const int32_t src = cow_src ? cow_src[s] : -1;
    const int64_t pos = (int64_t)seq_lens[s] - 1;
    int64_t dst = -1, slot = -1;
    int o = -1;
    if (pos >= 0) {
        const int64_t block_number = pos / block_size;
        if (block_number < max_blocks) {
            const int32_t physical = block_tables[(int64_t)s * max_blocks + block_number];
            if (physical >= 0 && physical < num_blocks) {
                dst = physical;
                o = (int)(pos - block_number * block_size);
                slot = dst * block_size + o;
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0 && threadIdx.x == 0 && slots_out) slots_out[s] = slot;
    if (dst < 0) return;
    const bool copy = src >= 0 && src < num_blocks && src != dst;
    const bool has_row = o >= r0 && o < r1;
    if (!copy && !has_row) return;
    const int64_t chunks_per_block = (int64_t)block_size * chunks_per_token;
    uint4 *kd = key_cache + dst * chunks_per_block;
    uint4 *vd = value_cache + dst * chunks_per_block;
    const int64_t c_begin = (int64_t)(copy ? r0 : o) * chunks_per_token;
    const int64_t c_end = (int64_t)(copy ? r1 : o + 1) * chunks_per_token;
    const int64_t row_begin = (int64_t)o * chunks_per_token;
    // copy source (only read when copying) and the new row
    const uint4 *ks = copy ? key_cache + (int64_t)src * chunks_per_block : kd;
    const uint4 *vs = copy ? value_cache + (int64_t)src * chunks_per_block : vd;
    const uint4 *kn = key + (int64_t)s * chunks_per_token;
    const uint4 *vn = value + (int64_t)s * chunks_per_token;
    constexpr int U = 4;
    int64_t c = c_begin + threadIdx.x;
    for (; c + (U - 1) * blockDim.x < c_end; c += U * blockDim.x) {
        uint4 k[U], v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t cc = c + u * blockDim.x;
            const int64_t rc = cc - row_begin;  // chunk within the new row, if it is in it
            const bool nr = rc >= 0 && rc < chunks_per_token;
            k[u] = nr ? kn[rc] : ks[cc];
            v[u] = nr ? vn[rc] : vs[cc];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            kd[c + u * blockDim.x] = k[u];
            vd[c + u * blockDim.x] = v[u];
        }
    }
    for (; c < c_end; c += blockDim.x) {
        const int64_t rc = c - row_begin;
        const bool nr = rc >= 0 && rc < chunks_per_token;
        kd[c] = nr ? kn[rc] : ks[c];
        vd[c] = nr ? vn[rc] : vs[c];
    }
}

// One CTA per (pair, slice): copies `per_cta` 16-byte chunks of the source block
// into the destination block, in both caches, with 16 loads in flight per thread.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ key_cache,
                                                          uint4 *__restrict__ value_cache,
                                                          const int64_t *__restrict__ pairs,
                                                          int64_t chunks_per_block, int slices, int64_t num_blocks)
{
    pdl_wait();
    pdl_launch_dependents();
    const int pair = blockIdx.x / slices;
    const int slice = blockIdx.x - pair * slices;
    const int64_t src = pairs[2 * pair];
    const int64_t dst = pairs[2 * pair + 1];
    if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) return;  // ids outside the pool
    const int64_t per_cta = (chunks_per_block + slices - 1) / slices;
    const int64_t begin = slice * per_cta;
    const int64_t end = min(chunks_per_block, begin + per_cta);
    const uint4 *ks = key_cache + src * chunks_per_block;
    const uint4 *vs = value_cache + src * chunks_per_block;
    uint4 *kd = key_cache + dst * chunks_per_block;
    uint4 *vd = value_cache + dst * chunks_per_block;
    constexpr int U = 8;
    int64_t c = begin + threadIdx.x;
    for (; c + (U - 1) * blockDim.x < end; c += U * blockDim.x) {
        uint4 k[U], v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            k[u] = ks[c + u * blockDim.x];
            v[u] = vs[c + u * blockDim.x];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            kd[c + u * blockDim.x] = k[u];
            vd[c + u * blockDim.x] = v[u];
        }
    }
    for (; c < end; c += blockDim.x) {
        kd[c] = ks[c];
        vd[c] = vs[c];
    }
}

// Block copies between two caches that may live in different memories (device
// memory and pinned, mapped host memory): swap-out / swap-in.  One CTA per
// (pair, slice), 16-byte accesses, two loads in flight per cache per thread.
__global__ void __launch_bounds__(256) swap_blocks_kernel(uint4 *__restrict__ dst_key, uint4 *__restrict__ dst_value,
                                                          const uint4 *__restrict__ src_key,
                                                          const uint4 *__restrict__ src_value,
                                                          const int64_t *__restrict__ pairs, int64_t chunks_per_block,
                                                          int slices, int64_t src_blocks, int64_t dst_blocks)
{
    pdl_wait();
    pdl_launch_dependents();
    const int pair = blockIdx.x / slices;
    const int slice = blockIdx.x - pair * slices;
    const int64_t src = pairs[2 * pair];
    const int64_t dst = pairs[2 * pair + 1];
    if (src < 0 || dst < 0 || src >= src_blocks || dst >= dst_blocks) return;  // ids outside the caches
    const int64_t per_cta = (chunks_per_block + slices - 1) / slices;
    const int64_t begin = slice * per_cta;
    const int64_t end = min(chunks_per_block, begin + per_cta);
    const uint4 *ks = src_key + src * chunks_per_block;
    const uint4 *vs = src_value + src * chunks_per_block;
    uint4 *kd = dst_key + dst * chunks_per_block;
    uint4 *vd = dst_value + dst * chunks_per_block;
    constexpr int U = 2;
    int64_t c = begin + threadIdx.x;
    for (; c + (U - 1) * blockDim.x < end; c += U * blockDim.x) {
        uint4 k[U], v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            k[u] = ks[c + u * blockDim.x];
            v[u] = vs[c + u * blockDim.x];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            kd[c + u * blockDim.x] = k[u];
            vd[c + u * blockDim.x] = v[u];
        }
    }
    for (; c < end; c += blockDim.x) {
        kd[c] = ks[c];
        vd[c] = vs[c];
    }
}

// Counts sequences that break a precondition of the decode kernels.
__global__ void validate_tables_kernel(const int32_t *__restrict__ block_tables,
                                       const int32_t *__restrict__ seq_lens, int num_seqs, int max_blocks,
                                       int block_size, int num_blocks, int max_seq_len, int32_t *bad_count)
{
    pdl_wait();
    const int s = blockIdx.x;
    if (s >= num_seqs) return;
    const int L = seq_lens[s];
    __shared__ int bad;
    if (threadIdx.x == 0) bad = (L < 0 || L > max_seq_len) ? 1 : 0;
    __syncthreads();
    const int64_t used = L > 0 ? ((int64_t)L + block_size - 1) / block_size : 0;
    if (used > max_blocks) {
        if (threadIdx.x == 0) bad = 1;
    } else {
        for (int64_t j = threadIdx.x; j < used; j += blockDim.x) {
            const int32_t b = block_tables[(int64_t)s * max_blocks + j];
            if (b < 0 || b >= num_blocks) bad = 1;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && bad) atomicAdd(bad_count, 1);
}

}  // namespace pakv
