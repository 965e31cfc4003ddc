// prefill.cuh -- multi-query paged prefill attention (chunked prefill, causal
// within the chunk) on the fifth-generation tensor cores.
//
// "vLLM 核心源码深度解析 …", milestone list (v0.5 Chunked Prefill): a long
// prompt is processed in chunks so that it does not hold up decodes; with the
// causal rule of "论文专题讲解：vLLM / PagedAttention …" (the query at position i
// attends to positions up to i), new token i of a chunk that starts at
// position ctx attends to positions 0 .. ctx + i, read through the block table.
//
// One CTA per work item (sequence s, KV head g, pair of query tiles).  A query
// tile is 128 MMA rows = tq tokens x G query heads (row r = token r / G, head
// r % G), so every K/V tile read from the cache feeds all G heads of the KV
// head -- and, as the CTA holds two consecutive query tiles A and B, both of
// them.  Keys are processed in tiles of 64.  Fifteen warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: warp w owns TMEM
//              lanes 32(w % 4) .. +31, one row per thread; it reads S from
//              TMEM (which frees the S buffer for the next S), keeps a lazily
//              moved reference max, writes P as fp16 (rounded to nearest: 11
//              significant bits) into one of two P buffers, rescales O in
//              TMEM when a reference moves, and finally normalises O and
//              stores the output rows;
//   warp 8     producer: TMA loads of the two query tiles and of 64-key K and
//              V tiles, block by block through the table, into a 4-stage ring
//              (a stage frees once both query tiles' S and P V have read it);
//   warps 9-10 MMA: warp 9 allocates TMEM -- per query tile a 64-column S
//              buffer and two 32-column P buffers (A: columns 0..127, B:
//              128..255), O of A from 256, O of B from 256 + D.  One thread of
//              warp 9 issues both tiles' S products, one of warp 10 both
//              tiles' P V products:
//                S_X = Q_X K_j^T    (SS form, bf16: M 128, N 64, K D)
//                O_X += P V_j       (TS form, fp16: P read from TMEM; V an
//                                    MN-major shared-memory operand)
//              so S_X(j+1) is issued as soon as the softmax has read S_X(j) and
//              is never queued behind a P V that waits for P; completion is
//              tracked by tcgen05.commit on mbarriers;
//   warps 11-14 convert every V tile in shared memory from bf16 to fp16 in
//              place as soon as it lands (16 keys each), zeroing rows past the
//              sequence end; the four quarters meet on a per-stage mbarrier
//              that both tiles' P V wait for.
// P V runs on fp16 operands: a bf16 P (8 significant bits) is too coarse for
// the attention tolerance, and a bf16 high part + residual pair costs a second
// P V product.  A bf16 value converts to fp16 exactly for 2^-17 <= |v| <= 65504
// (smaller magnitudes round by at most 2^-25; larger ones saturate and record
// kStatusValueRange in the device status word).
// Every wait is bounded in time; after a timeout the CTA drains its own TMA
// loads and MMAs (bounded again), frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "tc05.cuh"

namespace pakv {

struct PrefillParams {
    __nv_bfloat16 *out;               // [T, Hq, D]
    const int32_t *block_tables;      // [B, max_blocks]
    const int32_t *seq_lens;          // [B]   cached positions, the chunk included
    const int32_t *q_start;           // [B+1] first query row of each sequence
    float scale_log2;                 // scale * log2(e)
    int num_seqs, num_heads, num_kv_heads, group, max_blocks;
    int tq;                           // tokens per query tile (tq * group <= 128)
    int q_box;                        // tokens per query TMA box: min(tq, total query rows)
};

constexpr int kPfProducerWarp = 8;
constexpr int kPfMmaWarp = 9;         // tile A's MMAs; warp 10 issues tile B's
constexpr int kPfConvWarp = 11;       // first of the 4 V-conversion warps
constexpr int kPfThreads = 480;
constexpr int kPfRows = 128;          // MMA M: query rows per tile
constexpr int kPfKeys = 64;           // keys per K/V tile
constexpr int kPfStages = 4;          // K/V ring stages
constexpr int kPfQBufs = 1;           // query buffers (pairs of query tiles)
constexpr uint32_t kPfTmemCols = 512;
// A row's softmax reference max moves only when a logit exceeds it by more
// than this (log2 units), so unnormalised weights stay below 2^8.
constexpr float kPfRescaleSlack = 8.f;
// Weights are computed as 2^(logit - reference + kPfP16Shift), i.e. in
// (0, 2^15]: inside the fp16 range, and 2^7 further from fp16's subnormals.
// The factor cancels between O and the row sum.
constexpr float kPfP16Shift = 7.f;

// Packed fp32 pairs (one 64-bit register pair, two lanes of one instruction).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f32x2_split(uint64_t v)
{
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
// a * b + c on both lanes
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// bf16x2 -> f16x2 (round to nearest), tracking the largest magnitude seen.
// Magnitudes beyond the fp16 range saturate to +-65504 rather than becoming
// infinite, so a zero weight times such an entry stays 0 for the other rows.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float &amax)
{
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    amax = max3f(amax, fabsf(lo), fabsf(hi));
    uint32_t d;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

template <int D>
struct PfLayout {
    static constexpr int kQPlane = kPfRows * 128;          // 128 query rows x 128 bytes (64 bf16)
    static constexpr int kKPlane = kPfKeys * 128;          // 64 key rows x 128 bytes
    static constexpr int kPlanes = D / 64;
    static constexpr int kQTile = kPlanes * kQPlane;
    static constexpr int kKTile = kPlanes * kKPlane;       // K or V tile
    static constexpr int kQ = 0;                           // Q buffer qb: tile A, then tile B
    static constexpr int kQBuf = 2 * kQTile;
    static constexpr int kStage0 = kPfQBufs * kQBuf;       // stage st: K tile, then V tile
    static constexpr int kStageBytes = 2 * kKTile;
    static constexpr int kBar = kStage0 + kPfStages * kStageBytes;
    // q_full[2], q_free[2], drain[2], kv_full[S], kv_empty[S], then per query
    // tile s_full[2], s_free[2], o_free[2], and per query tile and P buffer
    // p_full[2][2], o_done[2][2]; then v16[S] (the V tile of a stage in fp16)
    static constexpr int kNumBars = 6 + 3 * kPfStages + 6 + 8;
    static constexpr int kMisc = kBar + kNumBars * 8;      // TMEM base, abort flag, item count
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
    // TMEM columns of query tile x: S at x * kTmemTile (kPfKeys columns), its
    // two fp16 P buffers after it (kPfKeys / 2 columns each); O_A at kTmemO,
    // O_B at kTmemO + D
    static constexpr uint32_t kTmemTile = 2 * kPfKeys;
    static constexpr uint32_t kTmemO = 2 * kTmemTile;
};

// One work item: a pair of consecutive query tiles (A and B) of one sequence
// and one KV head.
struct PfItem {
    int s, g, q0, q_len, L, ctx, tA;
    bool hasB;
    int endA, endB, nkA, nk;  // causal: key tiles of tile A, of the pair (>= nkA)
};

// Persistent: each CTA takes one work item of every round of gridDim.x items,
// in snake order (see item_of).  Item w = (r, s, g) with the KV head fastest,
// then the sequence, then r: the r-th pair of sequence s counted from its end
// (its longest), so every sequence's longest pairs come first and the CTAs
// share each length class.  Consecutive items of a CTA overlap: the next
// item's first K/V tile loads while the current item runs, its queries as
// soon as the current item's last S products have completed, and its first S
// is issued once the softmax has read the last S of the previous item, under
// that item's epilogue.
template <int D, int BS>
__global__ void __launch_bounds__(kPfThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v)
{
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    using Lay = PfLayout<D>;
    constexpr int kQPlane = Lay::kQPlane;
    constexpr int kKPlane = Lay::kKPlane;
    constexpr int kPlanes = Lay::kPlanes;
    constexpr int S = kPfStages;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + Lay::kBar;
    auto q_full = [&](int qb) { return bar0 + 8u * qb; };
    auto q_free = [&](int qb) { return bar0 + 8u * (2 + qb); };
    auto drain = [&](int x) { return bar0 + 8u * (4 + x); };
    auto kv_full = [&](int st) { return bar0 + 8u * (6 + st); };
    auto kv_empty = [&](int st) { return bar0 + 8u * (6 + S + st); };
    auto s_full = [&](int x) { return bar0 + 8u * (6 + 2 * S + x); };
    auto s_free = [&](int x) { return bar0 + 8u * (8 + 2 * S + x); };
    auto o_free = [&](int x) { return bar0 + 8u * (10 + 2 * S + x); };
    auto p_full = [&](int x, int b) { return bar0 + 8u * (12 + 2 * S + 2 * x + b); };
    auto o_done = [&](int x, int b) { return bar0 + 8u * (16 + 2 * S + 2 * x + b); };
    auto v16 = [&](int st) { return bar0 + 8u * (20 + 2 * S + st); };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(base_ptr + Lay::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 4);
    volatile int *rmax = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 8);

    pdl_wait();
    pdl_launch_dependents();

    const int G = p.group;
    const int B = p.num_seqs;
    const int Hkv = p.num_kv_heads;
    // pairs of query tiles of sequence s (0: nothing to do)
    auto pairs_of = [&](int q_len, int L) { return (q_len > 0 && q_len <= L) ? ((q_len + p.tq - 1) / p.tq + 1) / 2 : 0; };
    // ---- the most pairs any sequence has: the items are w < rmax * B * Hkv
    if (warp == 0) {
        int r = 0;
        for (int s = lane; s < B; s += 32) r = max(r, pairs_of(p.q_start[s + 1] - p.q_start[s], p.seq_lens[s]));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) r = max(r, __shfl_xor_sync(0xffffffffu, r, o));
        if (lane == 0) *rmax = r;
    }
    if (threadIdx.x == 32) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(q_full(b), 1);
            mbar_init(q_free(b), 1);  // the S warp's commit after its last S of the item
            mbar_init(drain(b), 1);
        }
        for (int i = 0; i < S; ++i) {
            mbar_init(kv_full(i), 1);
            mbar_init(kv_empty(i), 2);  // one commit from each MMA warp (K read by S, V by P V)
            mbar_init(v16(i), 4);       // one arrival per conversion warp
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full(x), 1);
            mbar_init(s_free(x), 128);  // every softmax thread of the tile has read S
            mbar_init(o_free(x), 128);  // every softmax thread of the tile has read O (epilogue)
            for (int b = 0; b < 2; ++b) {
                mbar_init(p_full(x, b), 128);
                mbar_init(o_done(x, b), 1);
            }
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const int64_t W = (int64_t)(*rmax) * B * Hkv;
    if (W == 0 || (int64_t)blockIdx.x >= W) return;  // no work: the whole CTA leaves before any TMEM use

    if (warp == kPfMmaWarp) {
        tmem_alloc(base + Lay::kMisc, kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The CTA's kr-th item: rounds of gridDim.x items, taken in snake order
    // (odd rounds reversed), so that the CTAs that take a round's longer items
    // take the next round's shorter ones
    auto item_of = [&](int64_t kr) -> int64_t {
        const int64_t b = (kr & 1) ? (int64_t)gridDim.x - 1 - blockIdx.x : (int64_t)blockIdx.x;
        return kr * gridDim.x + b;
    };
    // item w, or false if it holds no pair
    auto decode = [&](int64_t w, PfItem &it) -> bool {
        const int64_t per_r = (int64_t)B * Hkv;
        const int r = (int)(w / per_r);
        const int rem = (int)(w - (int64_t)r * per_r);
        it.s = rem / Hkv;
        it.g = rem - it.s * Hkv;
        it.q0 = p.q_start[it.s];
        it.q_len = p.q_start[it.s + 1] - it.q0;
        it.L = p.seq_lens[it.s];
        const int qp = pairs_of(it.q_len, it.L) - 1 - r;
        if (qp < 0) return false;
        it.ctx = it.L - it.q_len;
        it.tA = 2 * qp * p.tq;                             // first token of tile A (tile B follows)
        it.hasB = it.tA + p.tq < it.q_len;
        it.endA = min(it.q_len, it.tA + p.tq);
        it.endB = it.hasB ? min(it.q_len, it.tA + 2 * p.tq) : it.endA;
        it.nkA = (it.ctx + it.endA + kPfKeys - 1) / kPfKeys;
        it.nk = (it.ctx + it.endB + kPfKeys - 1) / kPfKeys;
        return true;
    };

    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait_bounded(bar, parity)) return true;
        record_timeout(kTimeoutFullBarrier);
        *abort_flag = 1;
        return false;
    };

    if (warp == kPfProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        int k = 0;         // items taken
        int kq_issued = 0; // query loads issued
        int64_t T = 0;     // ring tiles issued
        bool ok = true;
        for (int64_t kr = 0; ok && kr * gridDim.x < W; ++kr) {
            const int64_t w = item_of(kr);
            if (w >= W) break;
            PfItem it;
            if (!decode(w, it)) continue;
            const int qb = k % kPfQBufs;
            // the item's queries: the buffer is free once both MMA warps' last S of
            // item k - kPfQBufs completed; issued after the item's first K/V tile, so
            // that tile's load does not wait for the previous item's last S
            auto load_q = [&]() -> bool {
                if (k >= kPfQBufs &&
                    !__all_sync(0xffffffffu, wait(q_free(qb), (uint32_t)((k / kPfQBufs - 1) & 1))))
                    return false;
                if (lane == 0) {
                    mbar_arrive_expect_tx(q_full(qb), (uint32_t)(2 * kPlanes * G * p.q_box * 128));
                    for (int x = 0; x < 2; ++x)
                        for (int pl = 0; pl < kPlanes; ++pl)
                            tma_load_4d(base + Lay::kQ + qb * Lay::kQBuf + x * Lay::kQTile + pl * kQPlane,
                                        &tmap_q, q_full(qb), 0, pl, it.g * G, it.q0 + it.tA + x * p.tq);
                }
                __syncwarp();
                ++kq_issued;
                return true;
            };
            bool q_done = false;
            const int32_t *table = p.block_tables + (int64_t)it.s * p.max_blocks;
            for (int t = 0; t < it.nk; ++t, ++T) {
                if (t == 1) {
                    if (!load_q()) {
                        ok = false;
                        break;
                    }
                    q_done = true;
                }
                const int st = (int)(T % S);
                const int key0 = t * kPfKeys;
                const int nblk = min(kPfKeys / BS, (it.L - key0 + BS - 1) / BS);
                const int phys = lane < nblk ? table[key0 / BS + lane] : 0;
                if (T >= S && !__all_sync(0xffffffffu, wait(kv_empty(st), ((T / S) - 1) & 1))) {
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(kv_full(st), (uint32_t)(nblk * BS * D * 2 * 2));
                const uint32_t kdst = base + Lay::kStage0 + st * Lay::kStageBytes;
                const uint32_t vdst = kdst + Lay::kKTile;
                for (int kb = 0; kb < nblk; ++kb) {
                    const int row = __shfl_sync(0xffffffffu, phys, kb) * BS;
                    if (lane == 0) {
#pragma unroll
                        for (int pl = 0; pl < kPlanes; ++pl) {
                            tma_load_4d(kdst + pl * kKPlane + kb * BS * 128, &tmap_k, kv_full(st), 0, pl, it.g, row);
                            tma_load_4d(vdst + pl * kKPlane + kb * BS * 128, &tmap_v, kv_full(st), 0, pl, it.g, row);
                        }
                    }
                }
            }
            if (ok && !q_done && !load_q()) ok = false;   // an item of one key tile
            if (!ok) break;
            ++k;
        }
        if (lane == 0 && *abort_flag) {
            // let the loads this CTA issued land before it exits: the last two
            // query loads and each stage's last tile
            for (int kq = max(0, kq_issued - kPfQBufs); kq < kq_issued; ++kq)
                mbar_wait_bounded(q_full(kq % kPfQBufs), (uint32_t)((kq / kPfQBufs) & 1));
            for (int st = 0; st < S; ++st)
                if (st < T) {
                    const int64_t last = T - 1 - (T - 1 - st) % S;
                    mbar_wait_bounded(kv_full(st), (uint32_t)((last / S) & 1));
                }
        }
    } else if (warp == kPfMmaWarp) {
        // ------------------------------------------------------------ S products
        // Warp 9 issues both query tiles' S = Q K^T: S_X(j) as soon as K/V tile j
        // has landed and the softmax has read S_X(j-1), never behind a P V
        // product (those come from warp 10), so the next S is ready when the
        // softmax finishes the current tile.  After tile j's S products it
        // commits once to the stage's release (the K half of its reads), and
        // after the item's last S to the query buffer's.
        constexpr uint32_t kIdS = idesc_bf16_f32(kPfRows, kPfKeys, false, false);
        int k = 0;          // items taken
        int64_t T = 0;      // ring tiles consumed
        int64_t n[2] = {0, 0};  // S products issued per query tile
        bool ok = true;
        for (int64_t kr = 0; ok && kr * gridDim.x < W; ++kr) {
            const int64_t w = item_of(kr);
            if (w >= W) break;
            PfItem it;
            if (!decode(w, it)) continue;
            const int qb = k % kPfQBufs;
            ok = __all_sync(0xffffffffu, wait(q_full(qb), (uint32_t)((k / kPfQBufs) & 1)));
            for (int j = 0; ok && j < it.nk; ++j) {
                const int64_t tr = T + j;
                const int st = (int)(tr % S);
                ok = __all_sync(0xffffffffu, wait(kv_full(st), (uint32_t)((tr / S) & 1)));
                for (int x = 0; ok && x < 2; ++x) {
                    if (j >= (x == 0 ? it.nkA : (it.hasB ? it.nk : 0))) continue;
                    const int64_t nn = n[x] + j;
                    if (nn >= 1 && !__all_sync(0xffffffffu, wait(s_free(x), (uint32_t)((nn - 1) & 1)))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t q_lo = desc_lo_sw128(base + Lay::kQ + qb * Lay::kQBuf + x * Lay::kQTile, 16);
                        const uint32_t k_lo = desc_lo_sw128(base + Lay::kStage0 + st * Lay::kStageBytes, 16);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            tc_mma_lo(tmem + x * Lay::kTmemTile, q_lo + (uint32_t)(((kk >> 2) * kQPlane + (kk & 3) * 32) >> 4),
                                      k_lo + (uint32_t)(((kk >> 2) * kKPlane + (kk & 3) * 32) >> 4), kIdS, kk > 0);
                        }
                        tc_commit(s_full(x));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc_commit(kv_empty(st));
                __syncwarp();
            }
            if (!ok) break;
            // every S of the item was issued before this commit: the query buffer
            // frees when they complete
            if (lane == 0) tc_commit(q_free(qb));
            __syncwarp();
            T += it.nk;
            n[0] += it.nkA;
            if (it.hasB) n[1] += it.nk;
            ++k;
        }
    } else if (warp == kPfMmaWarp + 1) {
        // ------------------------------------------------------------ P V products
        // Warp 10 issues both query tiles' O += P V_j once the softmax has written
        // P_X(j) and V_j is fp16 (which also means tile j has landed), the first
        // of an item once the previous item's epilogue has read O; then commits
        // once to the stage's release (the V half of its reads).
        constexpr uint32_t kIdO = idesc_f16_f32(kPfRows, D, false, true);
        int64_t T = 0;          // ring tiles consumed
        int64_t n[2] = {0, 0};  // P V products issued per query tile
        int kx[2] = {0, 0};     // items with query tile x active
        bool ok = true;
        for (int64_t kr = 0; ok && kr * gridDim.x < W; ++kr) {
            const int64_t w = item_of(kr);
            if (w >= W) break;
            PfItem it;
            if (!decode(w, it)) continue;
            for (int j = 0; ok && j < it.nk; ++j) {
                const int64_t tr = T + j;
                const int st = (int)(tr % S);
                ok = __all_sync(0xffffffffu, wait(v16(st), (uint32_t)((tr / S) & 1)));
                for (int x = 0; ok && x < 2; ++x) {
                    if (j >= (x == 0 ? it.nkA : (it.hasB ? it.nk : 0))) continue;
                    const int64_t nj = n[x] + j;
                    const int b = (int)(nj & 1);
                    ok = __all_sync(0xffffffffu, wait(p_full(x, b), (uint32_t)((nj >> 1) & 1)));
                    // O of the previous item must have been read by its epilogue
                    if (ok && j == 0 && kx[x] >= 1)
                        ok = __all_sync(0xffffffffu, wait(o_free(x), (uint32_t)((kx[x] - 1) & 1)));
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t v_lo = desc_lo_sw128(base + Lay::kStage0 + st * Lay::kStageBytes + Lay::kKTile, kKPlane);
                        // P of the tile's 64 keys: fp16 pairs in kPfKeys / 2 columns; a K
                        // step of 16 keys is 8 columns
#pragma unroll
                        for (int kk = 0; kk < kPfKeys / 16; ++kk) {
                            tc_mma_ts_lo(tmem + Lay::kTmemO + x * D,
                                         tmem + x * Lay::kTmemTile + kPfKeys + b * (kPfKeys / 2) + kk * 8,
                                         v_lo + (uint32_t)(kk * 16 * 128 / 16), kIdO, j > 0 || kk > 0);
                        }
                        tc_commit(o_done(x, b));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc_commit(kv_empty(st));
                __syncwarp();
            }
            if (!ok) break;
            T += it.nk;
            n[0] += it.nkA;
            ++kx[0];
            if (it.hasB) {
                n[1] += it.nk;
                ++kx[1];
            }
        }
    } else if (warp >= kPfConvWarp) {
        // ------------------------------------------------------------ V to fp16
        // Warp 11 + c converts keys 16c .. 16c + 15 of every V tile (every
        // plane) in place as soon as the tile lands; rows past the sequence end
        // become 0 (they may hold stale or foreign data, even NaN, and P = 0
        // there would still give 0 * NaN = NaN).  The stage cannot be reloaded
        // before the P V that waits for this conversion has completed.
        const int c = warp - kPfConvWarp;
        float amax = 0.f;
        int64_t T = 0;
        bool ok = true;
        for (int64_t kr = 0; ok && kr * gridDim.x < W; ++kr) {
            const int64_t w = item_of(kr);
            if (w >= W) break;
            PfItem it;
            if (!decode(w, it)) continue;
            for (int t = 0; t < it.nk; ++t, ++T) {
                const int st = (int)(T % S);
                if (!__all_sync(0xffffffffu, wait(kv_full(st), (uint32_t)((T / S) & 1)))) {
                    ok = false;
                    break;
                }
                const int kv_valid = min(kPfKeys, it.L - t * kPfKeys);
                uint8_t *vt = base_ptr + Lay::kStage0 + st * Lay::kStageBytes + Lay::kKTile;
                uint4 v[kPlanes][4];
#pragma unroll
                for (int pl = 0; pl < kPlanes; ++pl)
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        v[pl][kq] = reinterpret_cast<const uint4 *>(vt + pl * kKPlane + c * 16 * 128)[lane + 32 * kq];
#pragma unroll
                for (int pl = 0; pl < kPlanes; ++pl)
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq) {
                        const int key = 16 * c + 4 * kq + (lane >> 3);  // 8 chunks of 16 bytes per 128-byte row
                        uint4 o = make_uint4(0, 0, 0, 0);
                        if (key < kv_valid) {
                            o.x = bf16x2_to_f16x2(v[pl][kq].x, amax);
                            o.y = bf16x2_to_f16x2(v[pl][kq].y, amax);
                            o.z = bf16x2_to_f16x2(v[pl][kq].z, amax);
                            o.w = bf16x2_to_f16x2(v[pl][kq].w, amax);
                        }
                        reinterpret_cast<uint4 *>(vt + pl * kKPlane + c * 16 * 128)[lane + 32 * kq] = o;
                    }
                fence_proxy_async_smem();  // the tensor cores read it through the async proxy
                __syncwarp();
                if (lane == 0) mbar_arrive(v16(st));
            }
        }
        if (amax > 65504.f) record_status(kStatusValueRange);
    } else {
        // ------------------------------------------------------------ softmax
        const int x = warp >> 2;                 // query tile: 0 = A, 1 = B
        const int r = threadIdx.x & 127;         // MMA row = TMEM lane
        const int tok = r / G;
        const int gi = r - tok * G;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t o_addr = lane_addr + Lay::kTmemO + x * D;
        const uint32_t s_addr = lane_addr + x * Lay::kTmemTile;
        int64_t n = 0;      // S tiles of this query tile consumed (= P tiles written)
        bool ok = true;
        for (int64_t kr = 0; ok && kr * gridDim.x < W; ++kr) {
            const int64_t w = item_of(kr);
            if (w >= W) break;
            PfItem it;
            if (!decode(w, it)) continue;
            const bool active = x == 0 || it.hasB;
            if (!active) continue;
            const int nkx = x == 0 ? it.nkA : it.nk;
            const int i = it.tA + x * p.tq + tok;
            const int endx = x == 0 ? it.endA : it.endB;
            const bool row_ok = tok < p.tq && i < endx;
            const int pos = row_ok ? it.ctx + i : it.L - 1;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < nkx; ++j) {
                const int64_t nj = n + j;
                const int b = (int)(nj & 1);
                const uint32_t p_addr = s_addr + kPfKeys + b * (kPfKeys / 2);
                ok = __all_sync(0xffffffffu, wait(s_full(x), (uint32_t)(nj & 1)));
                if (!ok) break;
                tc_fence_after();
                float xs[kPfKeys];
                tmem_ld32(s_addr, xs);
                tmem_ld32(s_addr + 32, xs + 32);
                // S is in registers: the next S product may overwrite the buffer
                tc_fence_before();
                mbar_arrive(s_free(x));
                // causal mask, only in tiles that reach past some row's position
                const int lim = pos - j * kPfKeys;  // keys c <= lim are visible
                if (!__all_sync(0xffffffffu, lim >= kPfKeys - 1)) {
#pragma unroll
                    for (int c = 0; c < kPfKeys; ++c) xs[c] = c <= lim ? xs[c] : -INFINITY;
                }
                // row max: four chains of three-input maxima
                float pm[4] = {xs[0], xs[1], xs[2], xs[3]};
#pragma unroll
                for (int c = 4; c < kPfKeys; c += 8) {
                    pm[0] = max3f(pm[0], xs[c], xs[c + 1]);
                    pm[1] = max3f(pm[1], xs[c + 2], xs[c + 3]);
                    pm[2] = max3f(pm[2], xs[c + 4], xs[c + 5]);
                    pm[3] = max3f(pm[3], xs[c + 6], xs[c + 7]);
                }
                const float mx = fmaxf(max3f(pm[0], pm[1], pm[2]), pm[3]) * p.scale_log2;  // scale > 0: the max commutes with it
                // lazily moved reference max (log2 units): weights stay <= 2^kPfRescaleSlack
                const bool bump = mx > m + kPfRescaleSlack;
                float corr = 1.f;
                if (bump) {
                    corr = fast_exp2(m - mx);  // 0 on the first tile (m = -inf)
                    m = mx;
                }
                // weights (scaled by 2^kPfP16Shift) as fp16 pairs, the lower key in
                // the low half: (logit scale, shift) on key pairs by packed fp32 FMAs;
                // the row sum in four packed fp32 accumulators
                const float mneg = kPfP16Shift - m;
                const uint64_t scale2 = f32x2(p.scale_log2, p.scale_log2), shift2 = f32x2(mneg, mneg);
                uint64_t ps[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) ps[u] = 0ull;
                float pw[kPfKeys / 2];
#pragma unroll
                for (int e = 0; e < kPfKeys / 2; ++e) {
                    const float2 y = f32x2_split(fma_f32x2(f32x2(xs[2 * e], xs[2 * e + 1]), scale2, shift2));
                    const float p0 = fast_exp2(y.x);
                    const float p1 = fast_exp2(y.y);
                    ps[e & 3] = add_f32x2(ps[e & 3], f32x2(p0, p1));
                    pw[e] = __uint_as_float(pack_f16x2(p0, p1));
                }
                const float2 q01 = f32x2_split(add_f32x2(ps[0], ps[1])), q23 = f32x2_split(add_f32x2(ps[2], ps[3]));
                l = l * corr + ((q01.x + q01.y) + (q23.x + q23.y));
                if (j >= 1 && __any_sync(0xffffffffu, bump)) {
                    // O holds P_{<j} V: rescale it once P_{j-1} V has completed
                    const int64_t jp = nj - 1;
                    ok = __all_sync(0xffffffffu, wait(o_done(x, (int)(jp & 1)), (uint32_t)((jp >> 1) & 1)));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        float o[32];
                        tmem_ld32(o_addr + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= corr;
                        tmem_st32(o_addr + c * 32, o);
                    }
                }
                // P into buffer b, once the P V product two tiles back has read it
                if (nj >= 2) {
                    ok = __all_sync(0xffffffffu, wait(o_done(x, b), (uint32_t)(((nj - 2) >> 1) & 1)));
                    if (!ok) break;
                    tc_fence_after();
                }
                tmem_st32(p_addr, pw);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full(x, b));
            }
            if (!ok) break;
            // epilogue: O / l once the item's last P V has completed
            const int64_t nl = n + nkx - 1;
            ok = __all_sync(0xffffffffu, wait(o_done(x, (int)(nl & 1)), (uint32_t)((nl >> 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst =
                p.out + ((int64_t)(it.q0 + (row_ok ? i : 0)) * p.num_heads + (int64_t)it.g * G + gi) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tmem_ld32(o_addr + c * 32, o);
                if (row_ok) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 v;
                        v.x = pack_bf16x2(o[8 * q4 + 0] * inv, o[8 * q4 + 1] * inv);
                        v.y = pack_bf16x2(o[8 * q4 + 2] * inv, o[8 * q4 + 3] * inv);
                        v.z = pack_bf16x2(o[8 * q4 + 4] * inv, o[8 * q4 + 5] * inv);
                        v.w = pack_bf16x2(o[8 * q4 + 6] * inv, o[8 * q4 + 7] * inv);
                        *reinterpret_cast<uint4 *>(dst + c * 32 + 8 * q4) = v;
                    }
                }
            }
            // O is in registers (and stored): the next item's first P V may overwrite it
            tc_fence_before();
            mbar_arrive(o_free(x));
            n += nkx;
        }
    }

    // ---- teardown: every role has left its loop (done or aborted)
    tc_fence_before();
    __syncthreads();
    if (warp >= kPfMmaWarp && warp < kPfConvWarp) {
        tc_fence_after();
        // all MMAs this CTA issued (by either MMA warp) have completed before
        // TMEM is released
        const uint32_t dr = drain(warp - kPfMmaWarp);
        if (lane == 0) tc_commit(dr);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(dr, 0)) && lane == 0) record_timeout(kTimeoutDrain);
        asm volatile("bar.sync 2, 64;" ::: "memory");  // both MMA warps drained
        if (warp == kPfMmaWarp) tmem_dealloc(tmem, kPfTmemCols);
    }
}

}  // namespace pakv
