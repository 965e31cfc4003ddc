// decode.cuh -- single-query paged decode attention for sm_100a.
//
// What is computed ("vLLM 源码解析：PagedAttention 如何让大模型推理提速 10 倍", §四;
// "论文专题讲解：vLLM / PagedAttention …", «PagedAttention：逻辑连续，物理不必连续»):
// for sequence s and query head h, with L = seq_lens[s],
//     out[s][h] = sum_{p<L} softmax_p(scale * q[s][h] . k_p) v_p,
// where k_p, v_p live in physical block block_tables[s][p / bs] at offset p % bs
// of the cache [num_blocks, bs, num_kv_heads, head_dim].  The kernel walks the
// sequence block by block and merges the per-block results with an online
// softmax -- the "compute locally per block, merge at the end" pattern of §四.
//
// Work item: (sequence, partition, KV head).  All G = Hq/Hkv query heads of the
// KV head are handled together, so every K/V byte crosses HBM once.  A
// partition is a run of `part_tokens` positions; the one-pass form has one
// partition per sequence.
//
// Persistent kernel: a grid of (CTAs per SM) x (SM count) CTAs loops over the
// work items.  The items of a launch are enumerated compactly (a prefix sum of
// partitions per sequence, in shared memory), sequence-major with the KV head
// fastest, and handed out by an atomic counter in the workspace (or round-robin
// when there is no workspace).  A CTA is six warps:
//  * Scheduler warp: takes the next item, decodes it, bulk-copies the item's G
//    query rows into an item slot, and loads the item's block-table entries in
//    chunks of 32 into a chunk queue -- running ahead of the other warps, so
//    their latency is hidden.
//  * Producer warp: for each chunk, four lanes take four consecutive tiles at
//    once (their ring waits, transaction counts and copies share each warp
//    instruction) and issue TMA tile loads of the K and V blocks (one box
//    {64 d, 1 head, bs tokens} per 64-wide d-plane, or one box per block with
//    both planes, 128B-swizzled) into a shared-memory ring guarded by
//    mbarriers.  The ring runs continuously across items.
//  * 4 consumer warps: 16-token tile i of an item goes to warp i % 4.  Every warp
//    keeps its own running max m, sum l and fp32 accumulator; the four states
//    are merged through shared memory at the end of the item (consumer-only
//    named barriers, so the loads of the next item keep flowing meanwhile).
//    - G >= 3 (grouped heads: a dense [16 x D] . [D x G] contraction per tile):
//      bf16 mma.sync m16n8k16 in transposed form, S^T = K Q^T with the K tile as
//      the A operand (rows = tokens, via ldmatrix) and Q^T in registers, then
//      O^T += V^T P^T with V^T through ldmatrix.trans and P^T moved out of the
//      S^T accumulators by movmatrix.trans; P goes in as bf16 hi + residual
//      (an FP8 cache: E4M3 key products and fp16 P, see below).
//    - G <= 2 (MHA-like, a matrix-vector product): CUDA cores, 16-byte shared
//      loads, warp-shuffle reductions for the dot products, max and sum.
//  * Masking selects (-inf logits, zeroed V rows) instead of multiplying by 0,
//    so stale or NaN data in unused slots of a partial block is never mixed in.
//  * Every mbarrier wait is bounded in time (about 1 s); on expiry the kernel
//    records a code in the device status word, drains its own TMA copies and
//    returns.
// Split form: a partition's (m, l, o) go to the workspace and lse_reduce_kernel
// merges them, one warp per (sequence, head); a sequence with a single
// partition is finished in place.
#pragma once

#include "common.cuh"

namespace pakv {

struct DecodeParams {
    __nv_bfloat16 *out;               // [B, Hq, D]
    const __nv_bfloat16 *query;       // [B, Hq, D]
    const int32_t *block_tables;      // [B, max_blocks]
    const int32_t *seq_lens;          // [B]
    float *ws_o;                      // [B, Hq, max_parts, D]   (split form)
    float *ws_m;                      // [B, Hq, max_parts]      natural-log units
    float *ws_l;                      // [B, Hq, max_parts]
    int *sched;                       // [2] item counter, finished-CTA counter; nullptr = round robin
    float scale_log2;                 // scale * log2(e) (times the K scale of an FP8 cache)
    float v_scale;                    // value scale of an FP8 cache (1 for bf16)
    int num_seqs, num_heads, num_kv_heads, group, max_blocks;
    int part_tokens;                  // positions per partition (multiple of 16); 0 = one pass
    int max_parts;                    // partitions per sequence (workspace stride); 1 = one pass
    int direct_single;                // a sequence with one partition writes `out`
    // Shared-prefix groups (split form, tensor-core consumers): group g is
    // sequences grp_start[g] .. grp_start[g+1]-1, whose first grp_parts[g]
    // partitions are the same blocks; those partitions are computed once per
    // KV head for up to ROWS / G sequences of the group at a time.
    const int32_t *grp_start;         // [num_groups + 1] or nullptr
    const int32_t *grp_parts;         // [num_groups]
    int num_groups;                   // 0: no groups
};

struct ReduceParams {
    __nv_bfloat16 *out;
    const float *ws_o, *ws_m, *ws_l;
    const int32_t *seq_lens;
    int num_seqs, num_heads, head_dim, part_tokens, max_parts;
    int skip_single;                  // sequences with one partition are already done
};

constexpr int kConsumerWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kSchedulerWarp = 5;
constexpr int kDecodeThreads = 6 * 32;
constexpr int kRingBudget = 80 * 1024;  // shared memory budget for the K/V ring per CTA (2 CTAs per SM)
constexpr int kTileTokens = 16;
constexpr int kItemSlots = 2;
constexpr int kChunkSlots = 4;
constexpr int kChunkBlocks = 32;
constexpr int kProducerLanes = 4;  // producer lanes issuing consecutive tiles together
constexpr int kSortKeys = 256;  // size classes (16-token tiles) of the largest-first item order
constexpr float kLn2 = 0.693147180559945309f;
// A column's softmax reference max moves only when a logit exceeds it by more
// than this (log2 units), so unnormalised weights stay below 2^8.
constexpr float kRescaleSlack = 8.f;

template <int D, int BS>
struct TileGeom {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 4 || BS == 8 || BS == 16, "block_size");
    // A K (or V) tile of 16 tokens is stored as D/64 planes; plane h holds
    // d in [64h, 64h+64) of every token as one 128-byte row per token.  TMA
    // writes one box {64 elements, 1, 1 head, bs tokens} per (block, plane),
    // 128B-swizzled, at a 1024-byte aligned slot.  With bs >= 8, 8 consecutive
    // tokens occupy 8 consecutive rows, so every ldmatrix phase touches 8
    // distinct swizzle rows: no bank conflicts.
    static constexpr int kHalves = D / 64;
    static constexpr int kBlkBytes = BS * D * 2;                  // bytes TMA delivers per block
    static constexpr int kSlotRows = BS < 8 ? 8 : BS;             // 128-B rows reserved per block per plane
    static constexpr int kBlocksPerTile = kTileTokens / BS;
    static constexpr int kPlaneSmem = kBlocksPerTile * kSlotRows * 128;
    static constexpr int kTileSmem = kHalves * kPlaneSmem;
    static constexpr int kStageSmem = 2 * kTileSmem;              // K tile, then V tile
    // Ring depth: as many stages as the budget holds, rounded down to a multiple
    // of the consumer-warp count (8 at head_dim 128, bs 16).  The multiple is
    // required: tile j of an item goes to warp j % 4 and sits at ring position
    // base + j, so a stage's previous tile (position - kStages) then belongs to
    // the same warp, which has consumed it before it waits on the stage again.
    // Otherwise a warp could wait on a stage whose previous phase is still
    // pending, and an mbarrier parity wait cannot tell that phase from the next.
    static constexpr int kStagesRaw = kRingBudget / kStageSmem > 16 ? 16 : kRingBudget / kStageSmem;
    static constexpr int kStages = kStagesRaw / kConsumerWarps * kConsumerWarps;
    static_assert(kStages >= kConsumerWarps && kStages % kConsumerWarps == 0, "ring depth");
    static constexpr int kPipeSmem = kStages * kStageSmem;

    // Offset, inside a plane, of token t's 128-byte row.
    __device__ static __forceinline__ uint32_t row_offset(int t)
    {
        return (uint32_t)((t / BS) * kSlotRows * 128 + (t % BS) * 128);
    }
    // Offset inside a tile of the 16-byte chunk c (0..D/8-1) of token t (0..15):
    // chunk index XOR (row index mod 8), the 128-byte swizzle.
    __device__ static __forceinline__ uint32_t chunk_offset(int t, int c)
    {
        const uint32_t ro = row_offset(t);
        return (uint32_t)((c >> 3) * kPlaneSmem) + ro + ((((uint32_t)c & 7u) ^ ((ro >> 7) & 7u)) << 4);
    }
    // Destination of the TMA box of block k (within the tile), plane h.
    __device__ static __forceinline__ uint32_t box_offset(int k, int h)
    {
        return (uint32_t)(h * kPlaneSmem + k * kSlotRows * 128);
    }
};

// Ring tiles of an FP8 (E4M3) cache, head_dim 128: one 128-byte row per token
// (one swizzle row), TMA box {128 codes, 1, 1 head, bs tokens}, 1024-byte
// aligned block slots, 128-byte swizzle.  The consumers read the codes with
// 16-byte loads straight into MMA fragments (no widened copy in shared memory).
template <int D, int BS>
struct TileGeom8 {
    static_assert(D == 128, "FP8 cache: head_dim 128");
    static_assert(BS == 8 || BS == 16, "FP8 cache: block_size 8 or 16");
    static constexpr int kHalves = 1;
    static constexpr int kBlkBytes = BS * D;                      // bytes TMA delivers per block
    static constexpr int kSlotRows = BS;
    static constexpr int kBlocksPerTile = kTileTokens / BS;
    static constexpr int kTileSmem = kBlocksPerTile * kSlotRows * 128;
    static constexpr int kPlaneSmem = kTileSmem;
    static constexpr int kStageSmem = 2 * kTileSmem;
    static constexpr int kStages = 16;                            // a multiple of the consumer warps
    static_assert(kStages % kConsumerWarps == 0, "ring depth");
    static constexpr int kPipeSmem = kStages * kStageSmem;

    __device__ static __forceinline__ uint32_t row_offset(int t) { return (uint32_t)(t * 128); }
    // 16-byte chunk c (codes 16c .. 16c+15) of token t
    __device__ static __forceinline__ uint32_t chunk_offset(int t, int c)
    {
        const uint32_t ro = row_offset(t);
        return ro + ((((uint32_t)c & 7u) ^ ((ro >> 7) & 7u)) << 4);
    }
    __device__ static __forceinline__ uint32_t box_offset(int k, int) { return (uint32_t)(k * kSlotRows * 128); }
};

// Per-item merge scratch: each consumer warp's running max (log2 units), sum
// and accumulator of up to ROWS heads.
template <int D, int ROWS>
struct MergeScratch {
    float o[kConsumerWarps][ROWS][D + 4];  // +4: the heads a warp writes at once land in distinct banks
    float m[kConsumerWarps][ROWS];         // reference max that o and l are relative to (log2 units)
    float mt[kConsumerWarps][ROWS];        // true max of the logits seen (log2 units), >= m
    float l[kConsumerWarps][ROWS];
};

// A work item as the scheduler publishes it.
struct ItemInfo {
    int s, g, part, nparts;
    int t_begin, t_end, n_tiles;
    int ring_base;                    // ring position of the item's first tile
    int stop;                         // 1: no more items
    int nseq;                         // sequences s .. s+nseq-1 of a shared-prefix item; 0 otherwise
    int ncols;                        // query rows (MMA columns) of the item: nseq * G, or G
    int single_mask;                  // shared-prefix item: bit i = sequence s+i has this one partition only
};

// A run of up to 32 blocks of one item for the producer.
struct ChunkInfo {
    int g, n_blocks, stop, pad;
    int phys[kChunkBlocks];
};

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Named barrier over the 4 consumer warps that also ORs a predicate across them,
// so every consumer warp takes the same decision after it.
__device__ __forceinline__ bool consumer_bar_or(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

// Bulk copy global -> this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Whether the decode loads a block with one TMA box covering its 64-wide
// d-planes (planes as the box's outer dimension) instead of one box per plane:
// only where a tile is one block, so the box lands plane-major.
__host__ __device__ constexpr bool decode_block_box(int D, int BS, bool FP8) { return !FP8 && D == 128 && BS == 16; }

template <int D, int BS, int MODE, int GC, bool FP8>
struct DecodeSmem {
    static constexpr int ROWS = MODE == 0 ? GC : (MODE == 1 ? 8 : 16);
    using Ring = std::conditional_t<FP8, TileGeom8<D, BS>, TileGeom<D, BS>>;
    using Merge = MergeScratch<D, ROWS>;
    static_assert(ROWS <= 32, "one query row per scheduler lane");
    static constexpr int kMergeOff = Ring::kPipeSmem;
    static constexpr int kQOff = (kMergeOff + (int)sizeof(Merge) + 127) & ~127;
    // one item's query rows, each padded by 16 bytes: the MMA consumers' fragment
    // loads (8 rows x 4 words per instruction) then fall in 32 distinct banks
    static constexpr int kQRow = D * 2 + 16;
    static constexpr int kQBytes = ROWS * kQRow;
    static constexpr int kItemOff = kQOff + kItemSlots * kQBytes;
    static constexpr int kChunkOff = kItemOff + kItemSlots * (int)sizeof(ItemInfo);
    static constexpr int kBarOff = (kChunkOff + kChunkSlots * (int)sizeof(ChunkInfo) + 7) & ~7;
    // barriers: full[kStages], empty[kStages], item_full, item_empty, chunk_full, chunk_empty
    static constexpr int kNumBars = 2 * Ring::kStages + 2 * kItemSlots + 2 * kChunkSlots;
    static constexpr int kFlagOff = kBarOff + kNumBars * 8;
    static constexpr int kPrefixOff = kFlagOff + 16;
    // bytes of dynamic shared memory for a launch over num_seqs sequences and
    // num_groups shared-prefix groups (enumeration tables: pf[B + 1],
    // rest_order[B], sort bases, gf[num_groups + 1], int16 keys[B], int16
    // kshared[B])
    static constexpr int bytes(int num_seqs, int num_groups = 0)
    {
        return 1024 + kPrefixOff + 4 * (2 * num_seqs + 1 + kSortKeys + 2 * (num_groups + 1)) +
               2 * ((2 * num_seqs + 3) & ~3);
    }
};

template <int D, int BS, int MODE, int GC, bool FP8>
__global__ void __launch_bounds__(kDecodeThreads, 2)
    paged_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v)
{
    static_assert(!FP8 || MODE != 0, "FP8 caches use the tensor-core consumers");
    // MODE 0: CUDA cores, GC (1 or 2) query heads per KV head.
    // MODE 1: tensor cores, up to 8 query heads per KV head (one 8-head tile).
    // MODE 2: tensor cores, up to 16 query heads per KV head (two 8-head tiles).
    using Lay = DecodeSmem<D, BS, MODE, GC, FP8>;
    using Geo = typename Lay::Ring;                                         // ring tiles
    using Merge = typename Lay::Merge;
    constexpr int kStages = Geo::kStages;
    // bf16, head_dim 128, bs 16: a block's two planes are one tile's two planes,
    // so one TMA box (planes as its outer dimension) loads the whole block
    constexpr bool kBlockBox = decode_block_box(D, BS, FP8);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    Merge *const ms = reinterpret_cast<Merge *>(base_ptr + Lay::kMergeOff);
    ItemInfo *const items = reinterpret_cast<ItemInfo *>(base_ptr + Lay::kItemOff);
    ChunkInfo *const chunks = reinterpret_cast<ChunkInfo *>(base_ptr + Lay::kChunkOff);
    const uint32_t full_bar = base + Lay::kBarOff;
    const uint32_t empty_bar = full_bar + kStages * 8;
    const uint32_t ifull_bar = empty_bar + kStages * 8;
    const uint32_t iempty_bar = ifull_bar + kItemSlots * 8;
    const uint32_t cfull_bar = iempty_bar + kItemSlots * 8;
    const uint32_t cempty_bar = cfull_bar + kChunkSlots * 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base_ptr + Lay::kFlagOff);
    // ring position up to which the producer has issued tile loads (a hint for
    // the scheduler's timing only; written by producer lane 0)
    volatile int *prod_ring = reinterpret_cast<volatile int *>(base_ptr + Lay::kFlagOff + 4);
    int *const prefix = reinterpret_cast<int *>(base_ptr + Lay::kPrefixOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = (MODE == 0) ? GC : p.group;
    const int B = p.num_seqs;
    const int Hkv = p.num_kv_heads;
    const bool split = p.max_parts > 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full_bar + 8 * i, 1);
            mbar_init(empty_bar + 8 * i, 1);
        }
        for (int i = 0; i < kItemSlots; ++i) {
            mbar_init(ifull_bar + 8 * i, 1);
            mbar_init(iempty_bar + 8 * i, 1);
        }
        for (int i = 0; i < kChunkSlots; ++i) {
            mbar_init(cfull_bar + 8 * i, 1);
            mbar_init(cempty_bar + 8 * i, 1);
        }
        *abort_flag = 0;
        *prod_ring = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x == kProducerWarp * 32) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
    }
    // Programmatic dependent launch: this grid may start while the previous
    // kernel of the stream still runs.  The enumeration below reads only the
    // lengths (and the scheduler the tables and queries), which no kernel of
    // this library writes, so it runs before griddepcontrol.wait; every
    // access to the caches, the outputs, the workspace and its counters comes
    // after it (producer before its first load, scheduler before its first
    // counter access, all threads before the partitions-only fill and the
    // counter reset).
    pdl_launch_dependents();

    // ---- enumeration of the work items, largest first.  Per sequence (length L
    // clamped to its table): f = number of full partitions of part_tokens
    // positions, plus one "rest" pair for the remainder (or for an empty
    // sequence, whose output is zeros).  Pair order: every full partition first
    // (sequence-major), then the rest pairs by size, largest first (a stable,
    // deterministic counting sort, so every CTA derives the same order; the
    // tail of the launch is made of the smallest items).  One pass: no full
    // partitions, every sequence is a rest pair, so sequences go longest first.
    // Item = pair * Hkv + KV head.  pf[s] = full partitions before sequence s.
    const int NG = p.num_groups;
    int *const pf = prefix;                    // [B + 1]
    int *const rest_order = prefix + B + 1;    // [B]
    int *const sort_base = rest_order + B;     // [kSortKeys]
    int *const gf = sort_base + kSortKeys;     // [NG + 1] shared-prefix pairs before group g
    int *const gstart = gf + NG + 1;           // [NG + 1] first sequence of group g
    int16_t *const keys = reinterpret_cast<int16_t *>(gstart + NG + 1);  // [B] rest keys
    int16_t *const kshared = keys + ((B + 1) & ~1);                 // [B] partitions computed by groups
    constexpr int kColsMax = Lay::ROWS;        // query rows one item holds
    const int spi = MODE == 0 ? 1 : max(1, kColsMax / max(G, 1));  // sequences per shared-prefix item
    const int Lcap = p.max_blocks * BS;
    auto full_of = [&](int L) {
        return (split && L > 0) ? min(L / p.part_tokens, p.max_parts) : 0;
    };
    auto rest_key = [&](int L) -> int {        // -1: no rest pair
        const int f = full_of(L);
        if (split && L > 0 && (f == p.max_parts || L == f * p.part_tokens)) return -1;
        const int r = max(L, 0) - f * (split ? p.part_tokens : 0);
        return min((r + kTileTokens - 1) / kTileTokens, kSortKeys - 1);
    };
    __shared__ int warp_tot[kDecodeThreads / 32];
    __shared__ int rest_count;
    // block-wide exclusive scan of arr[0..n) in place; arr[n] = the total
    auto block_scan = [&](int *arr, int n) {
        const int per = (n + kDecodeThreads - 1) / kDecodeThreads;
        const int i0 = min(n, (int)threadIdx.x * per);
        const int i1 = min(n, i0 + per);
        int local = 0;
        for (int i = i0; i < i1; ++i) local += arr[i];
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int run = incl - local;
        for (int w = 0; w < warp; ++w) run += warp_tot[w];
        for (int i = i0; i < i1; ++i) {
            const int f = arr[i];
            arr[i] = run;
            run += f;
        }
        if (threadIdx.x == kDecodeThreads - 1) arr[n] = run;
        __syncthreads();
    };
    // one coalesced pass over the lengths: each sequence's rest key, and its
    // full-partition count parked in pf[s] for the scan below
    if (threadIdx.x == 0) rest_count = 0;
    for (int k = threadIdx.x; k < kSortKeys; k += kDecodeThreads) sort_base[k] = 0;
    // shared-prefix groups: the partitions each sequence's group computes
    // (kshared), each group's item pairs (partitions x column blocks) and first
    // sequence -- read together with the lengths below, one round of loads
    const bool groups = split && NG > 0;
    for (int s = threadIdx.x; s < B; s += kDecodeThreads) kshared[s] = 0;
    __syncthreads();
    if (groups) {
        for (int gi = threadIdx.x; gi <= NG; gi += kDecodeThreads) {
            const int s0 = p.grp_start[gi];
            gstart[gi] = s0;
            if (gi == NG) continue;
            const int s1 = p.grp_start[gi + 1];
            const int k = p.grp_parts[gi];
            for (int s = s0; s < s1; ++s) kshared[s] = (int16_t)k;
            gf[gi] = k * ((s1 - s0 + spi - 1) / spi);
        }
    }
    {
        // ... and the histogram of the rest keys, for the largest-first order
        int nrest = 0;
        for (int s = threadIdx.x; s < B; s += kDecodeThreads) {
            // the start of every table row into L2: the first items' table
            // loads come right after the enumeration
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.block_tables + (int64_t)s * p.max_blocks));
            const int L = min(p.seq_lens[s], Lcap);
            const int key = rest_key(L);
            keys[s] = (int16_t)key;
            if (key >= 0) atomicAdd(&sort_base[key], 1);
            nrest += key >= 0;
            pf[s] = full_of(L);
        }
        if (nrest) atomicAdd(&rest_count, nrest);
    }
    __syncthreads();
    if (groups)  // the partitions a sequence's group computes are not its own
        for (int s = threadIdx.x; s < B; s += kDecodeThreads) pf[s] = max(0, pf[s] - kshared[s]);
    __syncthreads();
    if (split) block_scan(pf, B);                 // full partitions before sequence s
    if (split && NG > 0) block_scan(gf, NG);      // shared-prefix pairs before group g
    __syncthreads();
    const int total_full = split ? pf[B] : 0;
    const int total_group = (split && NG > 0) ? gf[NG] : 0;   // shared-prefix pairs come first
    const int total_rest = rest_count;

    if (warp == kSchedulerWarp) {
        // ------------------------------------------------------------ scheduler
        // Rest pairs sorted by size, largest first: a counting sort over
        // kSortKeys tile-count keys (histogram taken in the pass over the
        // lengths), stable in sequence order.  The CTA's first item needs only
        // its own rank, so it is selected from the scanned histogram right away
        // (its key's bin, then the n-th sequence of that key by ballots) and the
        // full order is scattered after that item has been handed to the
        // producer, off the path to the first loads.
        const int total_items = (total_group + total_full + total_rest) * Hkv;
        int first_rest = -1;   // sequence of this CTA's first item, if that is a rest pair
        {
            // exclusive scan in descending key order; lane owns kSortKeys/32 keys
            constexpr int KPL = kSortKeys / 32;
            int cnt[KPL], sum = 0;
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                cnt[i] = sort_base[kSortKeys - 1 - (lane * KPL + i)];
                sum += cnt[i];
            }
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            int run = incl - sum;
            const int r = (int)blockIdx.x / Hkv - total_group - total_full;   // rest rank of the first item
            int sel_key = -1, sel_off = 0;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int k = kSortKeys - 1 - (lane * KPL + i);
                if (r >= run && r < run + cnt[i]) {
                    sel_key = k;
                    sel_off = r - run;
                }
                sort_base[k] = run;
                run += cnt[i];
            }
            __syncwarp();
            const unsigned who = __ballot_sync(0xffffffffu, sel_key >= 0);
            if (who) {
                const int src = __ffs(who) - 1;
                sel_key = __shfl_sync(0xffffffffu, sel_key, src);
                sel_off = __shfl_sync(0xffffffffu, sel_off, src);
                for (int c = 0; c < B; c += 32) {
                    const int key = c + lane < B ? keys[c + lane] : -1;
                    const unsigned m = __ballot_sync(0xffffffffu, key == sel_key);
                    const int n = __popc(m);
                    if (sel_off < n) {
                        const int pre = __popc(m & ((1u << lane) - 1u));
                        const unsigned hit = __ballot_sync(0xffffffffu, key == sel_key && pre == sel_off);
                        first_rest = c + __ffs(hit) - 1;
                        break;
                    }
                    sel_off -= n;
                }
            }
        }
        // stable scatter of the rest pairs into rest_order (match_any ranks lanes)
        auto scatter_rest = [&]() {
            for (int c = 0; c < B; c += 32) {
                const int key = c + lane < B ? keys[c + lane] : -1;
                const unsigned peers = __match_any_sync(0xffffffffu, key);
                const int rank = __popc(peers & ((1u << lane) - 1u));
                if (key >= 0) rest_order[sort_base[key] + rank] = c + lane;
                __syncwarp();
                if (key >= 0 && rank == 0) sort_base[key] += __popc(peers);
                __syncwarp();
            }
            __syncwarp();
        };
        bool sorted = false;

        // Each CTA starts on item blockIdx.x; later items come from the atomic
        // counter (offset by the grid size) or round-robin without a workspace.
        int rr_next = blockIdx.x;
        bool first_grab = true;
        auto grab = [&]() -> int {
            int v = 0;
            if (lane == 0) {
                if (first_grab || !p.sched) {
                    v = rr_next;
                    rr_next += gridDim.x;
                } else {
                    v = (int)gridDim.x + atomicAdd(&p.sched[0], 1);
                }
            }
            first_grab = false;
            return __shfl_sync(0xffffffffu, v, 0);
        };
        // An item is taken only once its slot is free, i.e. when the item two
        // before it has been consumed: one item ahead of the consumers (so the
        // producer runs on across items) and no earlier, so the largest-first
        // order still decides what runs at the tail of the launch.
        int idx = 0;
        int item_seq = 0, chunk_seq = 0, ring_base = 0;
        while (true) {
            // item slot
            const int islot = item_seq % kItemSlots;
            bool ok = true;
            if (lane == 0) {
                if (*abort_flag || !mbar_wait_bounded(iempty_bar + 8 * islot, ((item_seq / kItemSlots) & 1) ^ 1)) {
                    if (!*abort_flag) record_timeout(kTimeoutEmptyBarrier);
                    *abort_flag = 1;
                    ok = false;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (item_seq == 1) pdl_wait();  // the counters belong to the previous grid until here
            idx = grab();
            const bool have = idx < total_items;
            ItemInfo it = {};
            int first_blk = 0, end_blk = 0;
            if (have && idx / Hkv < total_group) {
                // a shared-prefix pair: partition `part` of group gi for the
                // sequences of one column block (pairs of a group: partition-major,
                // so the column blocks of a partition run together)
                const int gp = idx / Hkv;
                it.g = idx - gp * Hkv;
                int lo = 0, hi = NG;  // largest group with gf[g] <= gp
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (gf[mid] <= gp) lo = mid; else hi = mid;
                }
                const int s0 = gstart[lo], n = gstart[lo + 1] - s0;
                const int nblk = (n + spi - 1) / spi;
                const int local = gp - gf[lo];
                const int cbk = local % nblk;
                it.part = local / nblk;
                it.s = s0 + cbk * spi;
                it.nseq = min(spi, n - cbk * spi);
                it.ncols = it.nseq * G;
                it.nparts = 0;
                it.single_mask = 0;  // members whose only partition this is write `out` directly
                for (int i = 0; i < it.nseq; ++i) {
                    const int si = it.s + i;   // partitions: the group's, its own full ones, its rest
                    if (kshared[si] + (pf[si + 1] - pf[si]) + (keys[si] >= 0 ? 1 : 0) == 1) it.single_mask |= 1 << i;
                }
                it.t_begin = it.part * p.part_tokens;
                it.t_end = it.t_begin + p.part_tokens;   // every member covers the group's partitions
                it.n_tiles = p.part_tokens / kTileTokens;
                it.ring_base = ring_base;
                it.stop = 0;
                first_blk = it.t_begin / BS;
                end_blk = (it.t_end + BS - 1) / BS;
            } else if (have) {
                const int sp = idx / Hkv - total_group;
                it.g = idx - (sp + total_group) * Hkv;
                if (sp < total_full) {
                    int lo = 0, hi = B;  // largest s with pf[s] <= sp
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (pf[mid] <= sp) lo = mid; else hi = mid;
                    }
                    it.s = lo;
                    it.part = kshared[lo] + sp - pf[lo];   // after the partitions its group computes
                } else {
                    // before the scatter, the only rest pair taken is the CTA's first item
                    it.s = sorted ? rest_order[sp - total_full] : first_rest;
                    it.part = -1;  // the rest pair: after the full partitions
                }
                it.nseq = 0;
                it.ncols = G;
                it.single_mask = 0;
                const int L = min(p.seq_lens[it.s], Lcap);
                const int f = full_of(L);
                it.nparts = f + (rest_key(L) >= 0 ? 1 : 0);
                if (it.part < 0) it.part = f;
                it.t_begin = split ? it.part * p.part_tokens : 0;
                it.t_end = split ? min(L, it.t_begin + p.part_tokens) : max(L, 0);
                it.n_tiles = it.t_end > it.t_begin ? (it.t_end - it.t_begin + kTileTokens - 1) / kTileTokens : 0;
                it.ring_base = ring_base;
                it.stop = 0;
                first_blk = it.t_begin / BS;
                end_blk = it.n_tiles > 0 ? (it.t_end + BS - 1) / BS : first_blk;
            } else {
                it.stop = 1;
            }
            {
                // the G query rows of each of the item's sequences, one after another,
                // one row per lane into the padded rows of the item's query slot
                const uint32_t bar = ifull_bar + 8 * islot;
                const int rows = it.stop ? 0 : (it.nseq > 0 ? it.nseq : 1) * G;
                if (lane == 0) {
                    items[islot] = it;
                    if (rows > 0)
                        mbar_arrive_expect_tx(bar, (uint32_t)(rows * D * 2));
                    else
                        mbar_arrive(bar);
                }
                __syncwarp();
                if (lane < rows)
                    bulk_load(base + Lay::kQOff + islot * Lay::kQBytes + (uint32_t)(lane * Lay::kQRow),
                              p.query + ((int64_t)(it.s + lane / G) * p.num_heads + (int64_t)it.g * G + lane % G) * D,
                              (uint32_t)(D * 2), bar);
            }
            // chunks of the item's block table (and a stop marker after the last item)
            for (int cb = first_blk; ok && (cb < end_blk || it.stop); cb += kChunkBlocks) {
                const int cslot = chunk_seq % kChunkSlots;
                bool cok = true;
                if (lane == 0) {
                    if (*abort_flag ||
                        !mbar_wait_bounded(cempty_bar + 8 * cslot, ((chunk_seq / kChunkSlots) & 1) ^ 1)) {
                        if (!*abort_flag) record_timeout(kTimeoutEmptyBarrier);
                        *abort_flag = 1;
                        cok = false;
                    }
                }
                cok = __shfl_sync(0xffffffffu, cok, 0);
                if (!cok) {
                    ok = false;
                    break;
                }
                ChunkInfo *c = chunks + cslot;
                if (it.stop) {
                    if (lane == 0) c->stop = 1;
                } else {
                    const int n = min(kChunkBlocks, end_blk - cb);
                    c->phys[lane] = lane < n ? __ldg(p.block_tables + (int64_t)it.s * p.max_blocks + cb + lane) : 0;
                    if (lane == 0) {
                        c->g = it.g;
                        c->n_blocks = n;
                        c->stop = 0;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(cfull_bar + 8 * cslot);
                ++chunk_seq;
                if (it.stop) break;
            }
            if (!ok || it.stop) break;
            if (!sorted) {  // before the next item can be a rest pair
                scatter_rest();
                sorted = true;
            }
            // The next item is taken only when the producer is within a ring's
            // depth (kStages tiles) of this item's end -- with the ring full, about
            // two rings' worth of tiles before the consumers finish it: late
            // enough that an item is not reserved long before it runs (a CTA that
            // starts on one of the largest items would otherwise end the launch
            // with the medium item it took at the start), so the largest-first
            // order decides what runs last; early enough that the next item's
            // queries and table entries arrive before the ring drains.  Items
            // shorter than the lookahead keep their successor one item ahead.
            {
                const int target = ring_base + it.n_tiles - kStages;
                bool gok = true;
                if (lane == 0 && *prod_ring < target) {
                    const unsigned long long t0 = global_timer_ns();
                    while (*prod_ring < target) {
                        if (*abort_flag) {
                            gok = false;
                            break;
                        }
                        if (global_timer_ns() - t0 > kWaitLimitNs) {
                            record_timeout(kTimeoutEmptyBarrier);
                            *abort_flag = 1;
                            gok = false;
                            break;
                        }
                        __nanosleep(64);
                    }
                }
                if (!__shfl_sync(0xffffffffu, gok, 0)) break;
            }
            ring_base += it.n_tiles;
            ++item_seq;
        }
    } else if (warp == kProducerWarp) {
        // ------------------------------------------------------------- producer
        pdl_wait();  // the caches may still be written by the previous grid until here
        int chunk_seq = 0, ring = 0;
        while (true) {
            const int cslot = chunk_seq % kChunkSlots;
            bool ok = true;
            if (lane == 0 && (*abort_flag || !mbar_wait_bounded(cfull_bar + 8 * cslot, (chunk_seq / kChunkSlots) & 1))) {
                if (!*abort_flag) record_timeout(kTimeoutFullBarrier);
                *abort_flag = 1;
                ok = false;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const ChunkInfo *c = chunks + cslot;
            if (c->stop) break;
            {
                // kProducerLanes lanes take consecutive tiles of the chunk at once:
                // their ring waits, transaction counts and TMA issues go out as
                // one instruction each, so the per-tile handoff latency is shared.
                const int n = c->n_blocks;
                const int g = c->g;
                const int ntiles = (n + Geo::kBlocksPerTile - 1) / Geo::kBlocksPerTile;
                for (int t0 = 0; t0 < ntiles; t0 += kProducerLanes) {
                    const int t = t0 + lane;
                    const bool mine = lane < kProducerLanes && t < ntiles;
                    const int r = ring + lane;  // ring position of tile t
                    const int stage = r % kStages;
                    bool w_ok = true;
                    if (mine) w_ok = !*abort_flag && mbar_wait_bounded(empty_bar + 8 * stage, ((r / kStages) & 1) ^ 1);
                    if (!__all_sync(0xffffffffu, w_ok)) {
                        if (lane == 0) {
                            if (!*abort_flag) record_timeout(kTimeoutEmptyBarrier);
                            *abort_flag = 1;
                        }
                        ok = false;
                        break;
                    }
                    if (mine) {
                        const int j = t * Geo::kBlocksPerTile;
                        const int valid = min(Geo::kBlocksPerTile, n - j);
                        const uint32_t kdst = base + stage * Geo::kStageSmem;
                        const uint32_t vdst = kdst + Geo::kTileSmem;
                        const uint32_t bar = full_bar + 8 * stage;
                        mbar_arrive_expect_tx(bar, (uint32_t)(valid * Geo::kBlkBytes * 2));
#pragma unroll
                        for (int k = 0; k < Geo::kBlocksPerTile; ++k) {
                            if (k < valid) {
                                const int row = c->phys[j + k] * BS;
                                if constexpr (kBlockBox) {
                                    // one box per block: both 64-wide planes, plane-major
                                    tma_load_4d(kdst + Geo::box_offset(k, 0), &tmap_k, bar, 0, row, 0, g);
                                    tma_load_4d(vdst + Geo::box_offset(k, 0), &tmap_v, bar, 0, row, 0, g);
                                } else {
#pragma unroll
                                    for (int h = 0; h < Geo::kHalves; ++h) {
                                        tma_load_4d(kdst + Geo::box_offset(k, h), &tmap_k, bar, 0, h, g, row);
                                        tma_load_4d(vdst + Geo::box_offset(k, h), &tmap_v, bar, 0, h, g, row);
                                    }
                                }
                            }
                        }
                    }
                    ring += min(kProducerLanes, ntiles - t0);
                    if (lane == 0) *prod_ring = ring;
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(cempty_bar + 8 * cslot);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ring = __shfl_sync(0xffffffffu, ring, 0);
            if (!ok) break;
            ++chunk_seq;
        }
        // On an abort, wait for the copies already in flight before the CTA exits.
        if (lane == 0 && *abort_flag && ring > 0) {
            for (int st = 0; st < kStages && st < ring; ++st) {
                const int last = ring - 1 - ((ring - 1 - st) % kStages);
                if (!mbar_wait_bounded(full_bar + 8 * st, (last / kStages) & 1)) record_timeout(kTimeoutDrain);
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        pdl_wait();  // outputs and partials may still be touched by the previous grid until here
        // Zero the V rows of tokens [valid, 16) so masked positions contribute
        // exactly 0 (stale or NaN data is never multiplied).
        auto zero_tail = [&](uint32_t vt, int valid) {
            constexpr int kChunksPerTok = Geo::kHalves * 8;
            for (int i = lane; i < (kTileTokens - valid) * kChunksPerTok; i += 32) {
                const int t = valid + i / kChunksPerTok;
                const int c = i % kChunksPerTok;  // whole rows are zeroed, so the swizzle does not matter
                *reinterpret_cast<uint4 *>(base_ptr + (vt - base) + (c >> 3) * Geo::kPlaneSmem +
                                           Geo::row_offset(t) + (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        };
        // Wait for a ring stage; false (and the abort flag set) if the wait gave up.
        auto wait_full = [&](int ring) -> bool {
            if (*abort_flag) return false;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar + 8 * (ring % kStages), (ring / kStages) & 1));
            if (!ok && lane == 0) {
                record_timeout(kTimeoutFullBarrier);
                *abort_flag = 1;
            }
            return ok;
        };
        auto release = [&](int ring, int valid) {
            if (valid < kTileTokens) fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar + 8 * (ring % kStages));
        };

        int item_seq = 0;
        while (true) {
            const int islot = item_seq % kItemSlots;
            bool ok = !*abort_flag;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(ifull_bar + 8 * islot, (item_seq / kItemSlots) & 1));
            if (!ok && lane == 0 && !*abort_flag) {
                record_timeout(kTimeoutFullBarrier);
                *abort_flag = 1;
            }
            // all four consumer warps leave together, or none does
            if (consumer_bar_or(!ok || *abort_flag)) break;
            const ItemInfo it = items[islot];
            if (it.stop) break;
            const uint8_t *qsm = base_ptr + Lay::kQOff + islot * Lay::kQBytes;

            if constexpr (MODE == 0) {
                constexpr int CPT = D / 8;              // lanes per token in the dot products
                constexpr int TPP = 32 / CPT;           // tokens per pass
                constexpr int PASSES = kTileTokens / TPP;
                constexpr int DPL = D / 32;             // accumulator columns per lane
                const int qc = lane % CPT;
                const int qt = lane / CPT;
                float q[GC][8];
#pragma unroll
                for (int h = 0; h < GC; ++h) {
                    const uint4 rq = *reinterpret_cast<const uint4 *>(qsm + h * Lay::kQRow + qc * 16);
                    const uint32_t w[4] = {rq.x, rq.y, rq.z, rq.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = unpack_bf16x2(w[e]);
                        q[h][2 * e] = f.x * p.scale_log2;
                        q[h][2 * e + 1] = f.y * p.scale_log2;
                    }
                }
                float o[GC][DPL];
                float m[GC], l[GC];
#pragma unroll
                for (int h = 0; h < GC; ++h) {
                    m[h] = -INFINITY;
                    l[h] = 0.f;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[h][e] = 0.f;
                }
                for (int j = warp; j < it.n_tiles; j += kConsumerWarps) {
                    const int ring = it.ring_base + j;
                    if (!wait_full(ring)) break;
                    const uint32_t kt = base + (ring % kStages) * Geo::kStageSmem;
                    const uint32_t vt = kt + Geo::kTileSmem;
                    const int valid = min(kTileTokens, it.t_end - (it.t_begin + j * kTileTokens));
                    if (valid < kTileTokens) zero_tail(vt, valid);

                    float sv[GC][PASSES];
#pragma unroll
                    for (int jj = 0; jj < PASSES; ++jj) {
                        const int tok = jj * TPP + qt;
                        const uint4 kr = *reinterpret_cast<const uint4 *>(base_ptr + (kt - base) + Geo::chunk_offset(tok, qc));
                        const uint32_t w[4] = {kr.x, kr.y, kr.z, kr.w};
                        float kf[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = unpack_bf16x2(w[e]);
                            kf[2 * e] = f.x;
                            kf[2 * e + 1] = f.y;
                        }
#pragma unroll
                        for (int h = 0; h < GC; ++h) {
                            float dot = 0.f;
#pragma unroll
                            for (int e = 0; e < 8; ++e) dot = fmaf(q[h][e], kf[e], dot);
#pragma unroll
                            for (int off = CPT / 2; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                            sv[h][jj] = tok < valid ? dot : -INFINITY;
                        }
                    }
                    float pr[GC][PASSES];
#pragma unroll
                    for (int h = 0; h < GC; ++h) {
                        float mx = sv[h][0];
#pragma unroll
                        for (int jj = 1; jj < PASSES; ++jj) mx = fmaxf(mx, sv[h][jj]);
#pragma unroll
                        for (int off = CPT; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                        const float m_new = fmaxf(m[h], mx);
                        const float corr = exp2f(m[h] - m_new);
                        m[h] = m_new;
                        float sum = 0.f;
#pragma unroll
                        for (int jj = 0; jj < PASSES; ++jj) {
                            pr[h][jj] = exp2f(sv[h][jj] - m_new);
                            sum += pr[h][jj];
                        }
#pragma unroll
                        for (int off = CPT; off < 32; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                        l[h] = l[h] * corr + sum;
#pragma unroll
                        for (int e = 0; e < DPL; ++e) o[h][e] *= corr;
                    }
#pragma unroll
                    for (int tok = 0; tok < kTileTokens; ++tok) {
                        const int c = (DPL * lane) >> 3;
                        const uint32_t off = Geo::chunk_offset(tok, c) + ((DPL * lane) & 7) * 2;
                        float vf[DPL];
                        if constexpr (DPL == 4) {
                            const uint2 vr = *reinterpret_cast<const uint2 *>(base_ptr + (vt - base) + off);
                            const float2 a = unpack_bf16x2(vr.x), b = unpack_bf16x2(vr.y);
                            vf[0] = a.x; vf[1] = a.y; vf[2] = b.x; vf[3] = b.y;
                        } else {
                            const uint32_t vr = *reinterpret_cast<const uint32_t *>(base_ptr + (vt - base) + off);
                            const float2 a = unpack_bf16x2(vr);
                            vf[0] = a.x; vf[1] = a.y;
                        }
#pragma unroll
                        for (int h = 0; h < GC; ++h) {
                            const float pt = __shfl_sync(0xffffffffu, pr[h][tok / TPP], (tok % TPP) * CPT);
#pragma unroll
                            for (int e = 0; e < DPL; ++e) o[h][e] = fmaf(pt, vf[e], o[h][e]);
                        }
                    }
                    release(ring, valid);
                }
#pragma unroll
                for (int h = 0; h < GC; ++h) {
#pragma unroll
                    for (int e = 0; e < DPL; ++e) ms->o[warp][h][DPL * lane + e] = o[h][e];
                    if (lane == 0) {
                        ms->m[warp][h] = m[h];
                        ms->mt[warp][h] = m[h];
                        ms->l[warp][h] = l[h];
                    }
                }
            } else {
                // Tensor cores, transposed form: S^T[16 tokens x 8*NH heads] = K Q^T,
                // then O^T[D x heads] += V^T P^T.  Tokens are the MMA's M dimension,
                // so no accumulator row is wasted when G <= 8; P^T is taken from the
                // S^T accumulators by an in-register 8x8 transpose (movmatrix).
                // The body is compiled once per count of 8-column tiles (NH): an item
                // of at most 8 query rows runs the one-tile body even in the
                // 16-row kernel, with half the accumulators and no second softmax.
                auto mma_item = [&](auto nh_tag) {
                constexpr int NH = decltype(nh_tag)::value;  // 8-head column tiles
                constexpr int KSTEPS = D / 16;           // k-steps of S^T = K Q^T
                constexpr int MT = D / 16;               // 16-row d tiles of O^T
                const int gq = lane >> 2;                // MMA groupID
                const int tq = lane & 3;                 // MMA thread-in-group
                // B operand of S^T = K Q^T: b0 = Q[head][d 16kk+2tq..+1], b1 = Q[head][d 16kk+8+2tq..+1].
                uint32_t qb[NH][FP8 ? 1 : KSTEPS][2];
                // FP8 cache: S^T = K Q^T runs on E4M3 MMAs (m16n8k32) straight from the
                // codes.  Q is scaled by a power of two per head (max |q| into
                // [128, 256)) and split into two E4M3 terms, q1 = e4m3(q) and
                // q2 = e4m3(q - q1), whose sum is the bf16 value exactly for every
                // element within 2^9 of the head's largest (smaller ones are off by
                // less than 2^-17 of the largest); the logit scale divides the power
                // of two out again.  The contraction order over head_dim is
                // permuted so that a lane's k-slots 4tq..4tq+3 and 16+4tq..16+4tq+3
                // of k-step kk are words 2(kk&1) and 2(kk&1)+1 of code chunk
                // tq + 4(kk>>1) of its key row.
                uint32_t q8[NH][FP8 ? 4 : 1][2][2];  // [head tile][k-step][term][b0/b1]
                float qscale[NH][2];       // logit scale of accumulator columns 2tq, 2tq+1
                if constexpr (FP8) {
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh) {
                        const int head = nh * 8 + gq;
                        float v[4][2][4];
                        float amax = 0.f;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const int col = 16 * (tq + 4 * (kk >> 1)) + 8 * (kk & 1) + 4 * hh;
                                uint2 w = make_uint2(0u, 0u);
                                if (head < it.ncols) w = *reinterpret_cast<const uint2 *>(qsm + head * Lay::kQRow + col * 2);
                                const float2 f0 = unpack_bf16x2(w.x), f1 = unpack_bf16x2(w.y);
                                v[kk][hh][0] = f0.x;
                                v[kk][hh][1] = f0.y;
                                v[kk][hh][2] = f1.x;
                                v[kk][hh][3] = f1.y;
#pragma unroll
                                for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[kk][hh][e]));
                            }
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                        // sigma = 2^(8 - e) for amax = m 2^e, m in [0.5, 1): sigma amax in [128, 256)
                        int e2 = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 126;
                        int se = 8 - e2;
                        se = amax > 0.f ? min(max(se, -126), 127) : 0;
                        const float sigma = __uint_as_float((uint32_t)(se + 127) << 23);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                float a[4], r[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) a[e] = v[kk][hh][e] * sigma;
                                const uint16_t c01 = f32x2_to_e4m3x2(a[0], a[1]);
                                const uint16_t c23 = f32x2_to_e4m3x2(a[2], a[3]);
                                const float2 d01 = f16x2_to_float2(e4m3x2_to_f16x2(c01));
                                const float2 d23 = f16x2_to_float2(e4m3x2_to_f16x2(c23));
                                r[0] = a[0] - d01.x;
                                r[1] = a[1] - d01.y;
                                r[2] = a[2] - d23.x;
                                r[3] = a[3] - d23.y;
                                q8[nh][kk][0][hh] = (uint32_t)c01 | ((uint32_t)c23 << 16);
                                q8[nh][kk][1][hh] = (uint32_t)f32x2_to_e4m3x2(r[0], r[1]) |
                                                    ((uint32_t)f32x2_to_e4m3x2(r[2], r[3]) << 16);
                            }
                        // accumulator column 2tq + jj of this head tile is head nh*8 + 2tq + jj,
                        // whose sigma the lanes of group 2tq + jj computed
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const float sg = __shfl_sync(0xffffffffu, sigma, (2 * tq + jj) * 4);
                            qscale[nh][jj] = p.scale_log2 / sg;
                        }
                    }
                } else {
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh) {
                        const int head = nh * 8 + gq;
#pragma unroll
                        for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const int col = kk * 16 + hh * 8 + tq * 2;
                                qb[nh][kk][hh] =
                                    head < it.ncols ? *reinterpret_cast<const uint32_t *>(qsm + head * Lay::kQRow + col * 2) : 0u;
                            }
                        }
                        qscale[nh][0] = qscale[nh][1] = p.scale_log2;
                    }
                }
                float o[MT][NH][4];
                float m[NH][2], mtrue[NH][2], l[NH][2];
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) {
                    m[nh][0] = m[nh][1] = -INFINITY;
                    mtrue[nh][0] = mtrue[nh][1] = -INFINITY;
                    l[nh][0] = l[nh][1] = 0.f;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) o[mt][nh][0] = o[mt][nh][1] = o[mt][nh][2] = o[mt][nh][3] = 0.f;
                }
                // ldmatrix lane roles: K as the A operand (rows = tokens), V^T as the A
                // operand through the transposing load (rows = d)
                const int ktok = (lane & 7) + (((lane >> 3) & 1) << 3);
                const int kpar = lane >> 4;
                const int vtok = (lane & 7) + ((lane >> 4) << 3);
                const int vpar = (lane >> 3) & 1;
                (void)qb, (void)q8, (void)ktok, (void)kpar, (void)vtok, (void)vpar;  // each form uses some

                for (int j = warp; j < it.n_tiles; j += kConsumerWarps) {
                    const int ring = it.ring_base + j;
                    if (!wait_full(ring)) break;
                    const int valid = min(kTileTokens, it.t_end - (it.t_begin + j * kTileTokens));
                    const uint32_t kt = base + (ring % kStages) * Geo::kStageSmem;
                    const uint32_t vt = kt + Geo::kTileSmem;
                    if constexpr (!FP8) {
                        if (valid < kTileTokens) zero_tail(vt, valid);
                    }

                    // S^T[token][head] = K Q^T, as two independent MMA chains (even and
                    // odd k-steps) summed at the end: half the dependent latency
                    float sc[NH][4], sd[NH][4];
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
                        for (int c = 0; c < 4; ++c) sc[nh][c] = sd[nh][c] = 0.f;
                    if constexpr (FP8) {
                        // key rows gq and gq+8, code chunks tq (set 0) and tq + 4 (set 1); the
                        // lanes of odd gq load set 1 first so that each 8-lane phase of a
                        // 16-byte load touches 8 distinct swizzled chunks
                        const bool odd = gq & 1;
                        uint4 kr[2][2];  // [row gq / gq+8][set]
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int tok = gq + 8 * r;
                            const uint4 x = lds128(kt + Geo::chunk_offset(tok, tq + (odd ? 4 : 0)));
                            const uint4 y = lds128(kt + Geo::chunk_offset(tok, tq + (odd ? 0 : 4)));
                            kr[r][0] = odd ? y : x;
                            kr[r][1] = odd ? x : y;
                        }
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t a0 = u4_word(kr[0][kk >> 1], 2 * (kk & 1));
                            const uint32_t a2 = u4_word(kr[0][kk >> 1], 2 * (kk & 1) + 1);
                            const uint32_t a1 = u4_word(kr[1][kk >> 1], 2 * (kk & 1));
                            const uint32_t a3 = u4_word(kr[1][kk >> 1], 2 * (kk & 1) + 1);
#pragma unroll
                            for (int nh = 0; nh < NH; ++nh) {
                                mma_e4m3_16832(sc[nh], a0, a1, a2, a3, q8[nh][kk][0][0], q8[nh][kk][0][1]);
                                mma_e4m3_16832(sd[nh], a0, a1, a2, a3, q8[nh][kk][1][0], q8[nh][kk][1][1]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < KSTEPS; ++kk) {
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4(kt + Geo::chunk_offset(ktok, 2 * kk + kpar), a0, a1, a2, a3);
#pragma unroll
                            for (int nh = 0; nh < NH; ++nh)
                                mma_bf16_16816((kk & 1) ? sd[nh] : sc[nh], a0, a1, a2, a3, qb[nh][kk][0], qb[nh][kk][1]);
                        }
                    }
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
                        for (int c = 0; c < 4; ++c) sc[nh][c] += sd[nh][c];
                    // Online softmax per head column; this lane holds tokens gq and gq+8
                    // of heads 2tq and 2tq+1.  The reference max m of a column moves
                    // only when a logit exceeds it by more than kRescaleSlack (log2
                    // units): weights stay <= 2^kRescaleSlack, and o and l keep one
                    // common reference, so the result is the same softmax while the
                    // rescale of o is almost never taken.  P enters the PV product as a
                    // bf16 high part plus a bf16 residual (two MMAs): ~16 significant bits.
                    const bool in0 = gq < valid, in1 = gq + 8 < valid;
                    uint32_t bh[NH][2], bl[NH][2];
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh) {
                        // Each lane tests its own two logits per column against the
                        // column's reference; the column max (3 shuffles) is formed
                        // only when some lane's logit passes it by the slack.  The
                        // true max is kept per lane and reduced once per item.
                        float x[2][2], lv[2];  // [head j][token row]
                        bool bump = false;
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            x[jj][0] = in0 ? sc[nh][jj] * qscale[nh][jj] : -INFINITY;
                            x[jj][1] = in1 ? sc[nh][2 + jj] * qscale[nh][jj] : -INFINITY;
                            lv[jj] = fmaxf(x[jj][0], x[jj][1]);
                            mtrue[nh][jj] = fmaxf(mtrue[nh][jj], lv[jj]);
                            bump |= lv[jj] > m[nh][jj] + kRescaleSlack;
                        }
                        if (__any_sync(0xffffffffu, bump)) {
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                float v = lv[jj];
                                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                                const float m_new = v > m[nh][jj] + kRescaleSlack ? v : m[nh][jj];
                                const float corr = fast_exp2(m[nh][jj] - m_new);  // 1 for an unmoved column
                                m[nh][jj] = m_new;
                                l[nh][jj] *= corr;
#pragma unroll
                                for (int mt = 0; mt < MT; ++mt) {
                                    o[mt][nh][jj] *= corr;
                                    o[mt][nh][2 + jj] *= corr;
                                }
                            }
                        }
                        float pr[2][2];
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            pr[jj][0] = fast_exp2(x[jj][0] - m[nh][jj]);
                            pr[jj][1] = fast_exp2(x[jj][1] - m[nh][jj]);
                            l[nh][jj] += pr[jj][0] + pr[jj][1];
                        }
#pragma unroll
                        for (int row = 0; row < 2; ++row) {
                            if constexpr (FP8) {  // fp16 weights: 11 significant bits, one MMA
                                bh[nh][row] = movmatrix_trans(pack_f16x2(pr[0][row], pr[1][row]));
                                bl[nh][row] = 0u;
                            } else {
                                const uint32_t hi = pack_bf16x2(pr[0][row], pr[1][row]);
                                const float2 hf = unpack_bf16x2(hi);
                                const uint32_t lo = pack_bf16x2(pr[0][row] - hf.x, pr[1][row] - hf.y);
                                bh[nh][row] = movmatrix_trans(hi);
                                bl[nh][row] = movmatrix_trans(lo);
                            }
                        }
                    }
                    // O^T[d][head] += V^T P^T
                    if constexpr (FP8) {
                        // FP8 cache: the rows of O^T are permuted so that this lane's rows
                        // gq and gq+8 of d-tile mt are d = 16gq + 2mt and 16gq + 2mt + 1,
                        // i.e. code chunk gq of value rows 2tq, 2tq+1, 2tq+8, 2tq+9 (one
                        // 16-byte load each, 8 distinct swizzled chunks per phase).  Rows
                        // past the sequence end are zeroed here: stale codes may be NaN.
                        uint4 vr[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int tok = 2 * tq + (r & 1) + 8 * (r >> 1);
                            vr[r] = tok < valid ? lds128(vt + Geo::chunk_offset(tok, gq)) : make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            // bytes 2mt, 2mt+1 of each row, token pairs interleaved
                            const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                            const uint32_t lo = prmt(u4_word(vr[0], mt >> 1), u4_word(vr[1], mt >> 1), sel);
                            const uint32_t hi = prmt(u4_word(vr[2], mt >> 1), u4_word(vr[3], mt >> 1), sel);
                            uint32_t a0, a1, a2, a3;
                            e4m3x4_to_f16x2x2(lo, a0, a1);
                            e4m3x4_to_f16x2x2(hi, a2, a3);
#pragma unroll
                            for (int nh = 0; nh < NH; ++nh) mma_f16_16816(o[mt][nh], a0, a1, a2, a3, bh[nh][0], bh[nh][1]);
                        }
                    } else {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4_trans(vt + Geo::chunk_offset(vtok, 2 * mt + vpar), a0, a1, a2, a3);
#pragma unroll
                            for (int nh = 0; nh < NH; ++nh) {
                                mma_bf16_16816(o[mt][nh], a0, a1, a2, a3, bh[nh][0], bh[nh][1]);
                                mma_bf16_16816(o[mt][nh], a0, a1, a2, a3, bl[nh][0], bl[nh][1]);
                            }
                        }
                    }
                    release(ring, valid);
                }
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        l[nh][jj] += __shfl_xor_sync(0xffffffffu, l[nh][jj], 4);
                        l[nh][jj] += __shfl_xor_sync(0xffffffffu, l[nh][jj], 8);
                        l[nh][jj] += __shfl_xor_sync(0xffffffffu, l[nh][jj], 16);
                        mtrue[nh][jj] = fmaxf(mtrue[nh][jj], __shfl_xor_sync(0xffffffffu, mtrue[nh][jj], 4));
                        mtrue[nh][jj] = fmaxf(mtrue[nh][jj], __shfl_xor_sync(0xffffffffu, mtrue[nh][jj], 8));
                        mtrue[nh][jj] = fmaxf(mtrue[nh][jj], __shfl_xor_sync(0xffffffffu, mtrue[nh][jj], 16));
                    }
                }
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int head = nh * 8 + 2 * tq + jj;
                        if (head < it.ncols) {
#pragma unroll
                            for (int mt = 0; mt < MT; ++mt) {
                                const int d0 = FP8 ? 16 * gq + 2 * mt : mt * 16 + gq;
                                const int d1 = FP8 ? d0 + 1 : d0 + 8;
                                ms->o[warp][head][d0] = o[mt][nh][jj];
                                ms->o[warp][head][d1] = o[mt][nh][2 + jj];
                            }
                            if (gq == 0) {
                                ms->m[warp][head] = m[nh][jj];
                                ms->mt[warp][head] = mtrue[nh][jj];
                                ms->l[warp][head] = l[nh][jj];
                            }
                        }
                    }
                }
                };
                if constexpr (MODE == 2) {
                    if (it.ncols > 8)
                        mma_item(std::integral_constant<int, 2>{});
                    else
                        mma_item(std::integral_constant<int, 1>{});
                } else {
                    mma_item(std::integral_constant<int, 1>{});
                }
            }
            consumer_bar();  // every warp's state is in the merge scratch
            // the item's slot (its description and query rows) is read no more
            if (threadIdx.x == 0) mbar_arrive(iempty_bar + 8 * islot);
            // ---- merge the four warps of this item (after an abort the values are
            // meaningless but harmless; the next item check stops every warp)
            const bool direct = p.direct_single && it.nparts == 1;
            const int ncols = MODE == 0 ? G : it.ncols;
            // weighted sum of the four accumulators, 4 columns per thread; each
            // thread forms its row's weights itself: the combined true max is the
            // common reference (every warp's own reference is <= it, so the
            // weights are <= 1)
            constexpr int D4 = D / 4;
            for (int idx = threadIdx.x; idx < ncols * D4; idx += kConsumerWarps * 32) {
                const int row = idx / D4;
                const int d = (idx - row * D4) * 4;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ms->mt[w][row]);
                float den = 0.f;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float mw = ms->m[w][row];
                    const float c = (M != -INFINITY && mw != -INFINITY) ? exp2f(mw - M) : 0.f;
                    den = fmaf(c, ms->l[w][row], den);
                    const float4 v = *reinterpret_cast<const float4 *>(&ms->o[w][row][d]);
                    acc.x = fmaf(c, v.x, acc.x);
                    acc.y = fmaf(c, v.y, acc.y);
                    acc.z = fmaf(c, v.z, acc.z);
                    acc.w = fmaf(c, v.w, acc.w);
                }
                // query row: column `row` of a shared-prefix item is head row % G of
                // its sequence row / G
                const int64_t hrow = (int64_t)(it.s + row / G) * p.num_heads + (int64_t)it.g * G + row % G;
                const bool direct_row = direct || (p.direct_single && ((it.single_mask >> (row / G)) & 1));
                acc.x *= p.v_scale;
                acc.y *= p.v_scale;
                acc.z *= p.v_scale;
                acc.w *= p.v_scale;
                if (direct_row) {
                    const float inv = den > 0.f ? 1.f / den : 0.f;
                    uint2 packed;
                    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
                    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
                    *reinterpret_cast<uint2 *>(p.out + hrow * D + d) = packed;
                } else {
                    const int64_t wi = hrow * p.max_parts + it.part;
                    *reinterpret_cast<float4 *>(p.ws_o + wi * D + d) = acc;
                    if (d == 0) {
                        p.ws_m[wi] = M == -INFINITY ? -INFINITY : M * kLn2;
                        p.ws_l[wi] = den;
                    }
                }
            }
            consumer_bar();  // the merge scratch may be reused
            ++item_seq;
        }
    }

    // Partitions-only form: partitions that hold no position (past the end of
    // their sequence) report m = -inf, l = 0, o = 0.  Grid-strided over all
    // (sequence, head, partition) triples, after the CTA's items.
    pdl_wait();
    if (split && !p.direct_single) {
        const int64_t triples = (int64_t)B * p.num_heads * p.max_parts;
        for (int64_t t = (int64_t)blockIdx.x * kDecodeThreads + threadIdx.x; t < triples;
             t += (int64_t)gridDim.x * kDecodeThreads) {
            const int part = (int)(t % p.max_parts);
            const int s = (int)(t / ((int64_t)p.num_heads * p.max_parts));
            const int L = min(p.seq_lens[s], Lcap);
            if (part < full_of(L) + (rest_key(L) >= 0 ? 1 : 0)) continue;
            p.ws_m[t] = -INFINITY;
            p.ws_l[t] = 0.f;
            for (int d = 0; d < D; ++d) p.ws_o[t * D + d] = 0.f;
        }
    }

    __syncthreads();
    // The last CTA to finish leaves the scheduler counters at zero for the next launch.
    if (threadIdx.x == 0 && p.sched) {
        __threadfence();
        if (atomicAdd(&p.sched[1], 1) == (int)gridDim.x - 1) {
            atomicExch(&p.sched[0], 0);
            atomicExch(&p.sched[1], 0);
        }
    }
}

// Log-sum-exp merge of the partitions of one (sequence, head) row:
//   M = max_p m_p,  out = sum_p e^{m_p - M} o_p / sum_p e^{m_p - M} l_p.
// The partials were just written and sit in L2; the kernel is bound by load
// latency, so it keeps many loads in flight.  WPR warps share a row (a CTA of
// kReduceWarps warps serves kReduceWarps / WPR rows): warp w of a row takes
// partitions w, w + WPR, ...; lane i reads m and l of every 32nd of them (one
// round), then the o rows of 8 of its partitions are read together, each as one
// coalesced 16-byte (D = 128) or 8-byte (D = 64) vector per lane.  Each warp
// merges its partitions against its own maximum; the WPR warp states of a row
// are then merged through shared memory the same way.  WPR = 1 for rows of a
// few partitions, 8 for rows of many (a 128K-position sequence in 512-token
// partitions has 256: 4 rounds of 8 loads per warp instead of 32).
constexpr int kReduceWarps = 8;

template <int D, int WPR>
__global__ void __launch_bounds__(kReduceWarps * 32) lse_reduce_kernel(const ReduceParams r)
{
    static_assert(kReduceWarps % WPR == 0, "warps per row");
    constexpr int VEC = D / 32;
    constexpr int U = 8;  // partitions whose o rows are in flight together, per warp
    __shared__ float sh_acc[kReduceWarps][D];
    __shared__ float sh_m[kReduceWarps], sh_den[kReduceWarps];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int wr = warp % WPR;  // this warp's share of its row
    const int64_t row = (int64_t)blockIdx.x * (kReduceWarps / WPR) + warp / WPR;
    const bool live = row < (int64_t)r.num_seqs * r.num_heads;
    int nparts = 0;
    if (live) {
        const int L = r.seq_lens[row / r.num_heads];
        nparts = L > 0 ? (L + r.part_tokens - 1) / r.part_tokens : 1;
        nparts = min(nparts, r.max_parts);
    }
    const bool skip = !live || (r.skip_single && nparts == 1);
    float Mw = -INFINITY, den = 0.f;
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    if (!skip) {
        const float *m = r.ws_m + row * r.max_parts;
        const float *l = r.ws_l + row * r.max_parts;
        const float *o = r.ws_o + row * r.max_parts * D + lane * VEC;
        // this warp's partitions: j = wr + WPR * k, k = 0 .. mine - 1
        const int mine = nparts > wr ? (nparts - wr + WPR - 1) / WPR : 0;
        for (int k = lane; k < mine; k += 32) Mw = fmaxf(Mw, m[wr + WPR * k]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) Mw = fmaxf(Mw, __shfl_xor_sync(0xffffffffu, Mw, off));
        if (Mw != -INFINITY) {
            for (int k = lane; k < mine; k += 32) {
                const int j = wr + WPR * k;
                const float mj = m[j];
                if (mj != -INFINITY) den = fmaf(expf(mj - Mw), l[j], den);  // an empty partition weighs 0
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
            for (int k0 = 0; k0 < mine; k0 += U) {
                float v[U][VEC], w[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int k = k0 + u;
                    w[u] = 0.f;
#pragma unroll
                    for (int e = 0; e < VEC; ++e) v[u][e] = 0.f;
                    if (k < mine) {
                        const int j = wr + WPR * k;
                        const float mj = m[j];
                        w[u] = mj != -INFINITY ? expf(mj - Mw) : 0.f;
                        const float *src = o + (int64_t)j * D;
                        if constexpr (VEC == 4) {
                            const float4 f = *reinterpret_cast<const float4 *>(src);
                            v[u][0] = f.x; v[u][1] = f.y; v[u][2] = f.z; v[u][3] = f.w;
                        } else {
                            const float2 f = *reinterpret_cast<const float2 *>(src);
                            v[u][0] = f.x; v[u][1] = f.y;
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] = fmaf(w[u], v[u][e], acc[e]);
            }
        }
    }
    if constexpr (WPR > 1) {
        // merge the row's warp states: M = max_w M_w, weights e^{M_w - M}
#pragma unroll
        for (int e = 0; e < VEC; ++e) sh_acc[warp][lane * VEC + e] = acc[e];
        if (lane == 0) {
            sh_m[warp] = Mw;
            sh_den[warp] = den;
        }
        __syncthreads();
        if (skip || wr != 0) return;
        const int w0 = warp;  // first warp of this row
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WPR; ++w) M = fmaxf(M, sh_m[w0 + w]);
        den = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < WPR; ++w) {
                const float mw = sh_m[w0 + w];
                const float c = mw != -INFINITY ? expf(mw - M) : 0.f;
                den = fmaf(c, sh_den[w0 + w], den);
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] = fmaf(c, sh_acc[w0 + w][lane * VEC + e], acc[e]);
            }
        }
    } else if (skip) {
        return;
    }
    __nv_bfloat16 *dst = r.out + row * D + lane * VEC;
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[e] = __float2bfloat16_rn(den > 0.f ? acc[e] / den : 0.f);
}

}  // namespace pakv
