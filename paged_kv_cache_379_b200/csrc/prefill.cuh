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
//              TMEM, keeps a lazily moved reference max, writes P back over S
//              as fp16 (rounded to nearest: 11 significant bits),
//              rescales O in TMEM when a reference moves, and finally
//              normalises O and stores the output rows;
//   warp 8     producer: TMA loads of the two query tiles (once) and of 64-key
//              K and V tiles, block by block through the table, into a 4-stage
//              ring (a stage frees once both query tiles' P V have read it);
//   warps 9-10 MMA: warp 9 allocates TMEM -- two 64-column S/P buffers per
//              query tile (A: columns 0..127, B: 128..255), O of A from 256, O
//              of B from 256 + D; one thread of warp 9 issues tile A's
//              tcgen05.mma, one of warp 10 tile B's:
//                S_X = Q_X K_j^T    (SS form, bf16: M 128, N 64, K D)
//                O_X += P V_j       (TS form, fp16: P read from TMEM; V an
//                                    MN-major shared-memory operand)
//              S_X(j) goes to buffer j % 2, so it overlaps the softmax of
//              S_X(j-1); completion is tracked by tcgen05.commit on mbarriers,
//              one per buffer.  The two tiles' chains run independently;
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
    static constexpr int kQ = 0;                           // Q_A, then Q_B
    static constexpr int kStage0 = 2 * kQTile;             // stage st: K tile, then V tile
    static constexpr int kStageBytes = 2 * kKTile;
    static constexpr int kBar = kStage0 + kPfStages * kStageBytes;
    // q_full, drain[2], kv_full[4], kv_empty[4], then per query tile:
    // s_full[2], s_free[2], and per query tile and P buffer p_full[2][2],
    // o_done[2][2]; then v16[4] (the V tile of a stage converted to fp16)
    static constexpr int kNumBars = 3 + 3 * kPfStages + 12;
    static constexpr int kMisc = kBar + kNumBars * 8;      // TMEM base, abort flag, item
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
    // TMEM columns of query tile x: S at x * kTmemTile (kPfKeys columns), its
    // two fp16 P buffers after it (kPfKeys / 2 columns each); O_A at kTmemO,
    // O_B at kTmemO + D
    static constexpr uint32_t kTmemTile = 2 * kPfKeys;
    static constexpr uint32_t kTmemO = 2 * kTmemTile;
};

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

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + Lay::kBar;
    const uint32_t q_full = bar0;
    auto drain = [&](int x) { return bar0 + 8u * (1 + x); };
    auto kv_full = [&](int st) { return bar0 + 8u * (3 + st); };
    auto kv_empty = [&](int st) { return bar0 + 8u * (3 + kPfStages + st); };
    auto s_full = [&](int x) { return bar0 + 8u * (3 + 2 * kPfStages + x); };
    auto s_free = [&](int x) { return bar0 + 8u * (5 + 2 * kPfStages + x); };
    auto p_full = [&](int x, int b) { return bar0 + 8u * (7 + 2 * kPfStages + 2 * x + b); };
    auto o_done = [&](int x, int b) { return bar0 + 8u * (11 + 2 * kPfStages + 2 * x + b); };
    auto v16 = [&](int st) { return bar0 + 8u * (15 + 2 * kPfStages + st); };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(base_ptr + Lay::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 4);
    volatile int *item = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 16);

    pdl_wait();
    pdl_launch_dependents();

    // ---- which (sequence, pair of query tiles) this CTA takes: blockIdx.x
    // enumerates the tile pairs of all sequences, each sequence's last (longest)
    // pair first.
    if (warp == 0) {
        const int x = blockIdx.x;
        int found_s = -1, found_qp = 0, running = 0;
        for (int s0 = 0; s0 < p.num_seqs && found_s < 0; s0 += 32) {
            const int s = s0 + lane;
            int pairs = 0;
            if (s < p.num_seqs) {
                const int ql = p.q_start[s + 1] - p.q_start[s];
                if (ql > 0 && ql <= p.seq_lens[s]) pairs = ((ql + p.tq - 1) / p.tq + 1) / 2;
            }
            int incl = pairs;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = running + incl - pairs;
            const unsigned hit = __ballot_sync(0xffffffffu, pairs > 0 && x >= excl && x < excl + pairs);
            if (hit) {
                const int src = __ffs(hit) - 1;
                const int e = __shfl_sync(0xffffffffu, excl, src);
                const int np = __shfl_sync(0xffffffffu, pairs, src);
                found_s = s0 + src;
                found_qp = np - 1 - (x - e);
            }
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            item[0] = found_s;
            item[1] = found_qp;
        }
    }
    if (threadIdx.x == 32) {
        mbar_init(q_full, 1);
        for (int x = 0; x < 2; ++x) mbar_init(drain(x), 1);
        for (int i = 0; i < kPfStages; ++i) {
            mbar_init(kv_full(i), 1);
            mbar_init(kv_empty(i), 2);  // one commit from each MMA warp
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full(x), 1);
            mbar_init(s_free(x), 128);  // every softmax thread of the tile has read S
            for (int b = 0; b < 2; ++b) {
                mbar_init(p_full(x, b), 128);
                mbar_init(o_done(x, b), 1);
            }
        }
        for (int st = 0; st < kPfStages; ++st) mbar_init(v16(st), 4);  // one arrival per conversion warp
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const int s = item[0];
    if (s < 0) return;  // past the last pair: the whole CTA leaves before any TMEM use
    const int qp = item[1];

    if (warp == kPfMmaWarp) {
        tmem_alloc(base + Lay::kMisc, kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int G = p.group;
    const int g = blockIdx.y;
    const int q0 = p.q_start[s];
    const int q_len = p.q_start[s + 1] - q0;
    const int L = p.seq_lens[s];
    const int ctx = L - q_len;
    const int tA = 2 * qp * p.tq;                     // first token of tile A (tile B follows)
    const bool hasB = tA + p.tq < q_len;
    const int endA = min(q_len, tA + p.tq);
    const int endB = hasB ? min(q_len, tA + 2 * p.tq) : endA;
    const int nkA = (ctx + endA + kPfKeys - 1) / kPfKeys;  // causal: keys below ctx + end
    const int nk = (ctx + endB + kPfKeys - 1) / kPfKeys;   // key tiles of the pair (>= nkA)

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
            mbar_arrive_expect_tx(q_full, (uint32_t)(2 * kPlanes * G * p.q_box * 128));
            for (int x = 0; x < 2; ++x)
                for (int pl = 0; pl < kPlanes; ++pl)
                    tma_load_4d(base + Lay::kQ + x * Lay::kQTile + pl * kQPlane, &tmap_q, q_full, 0, pl, g * G,
                                q0 + tA + x * p.tq);
        }
        const int32_t *table = p.block_tables + (int64_t)s * p.max_blocks;
        int issued = 0;  // key tiles whose loads were issued
        for (int t = 0; t < nk; ++t) {
            const int st = t % kPfStages;
            const int key0 = t * kPfKeys;
            const int nblk = min(kPfKeys / BS, (L - key0 + BS - 1) / BS);
            const int phys = lane < nblk ? table[key0 / BS + lane] : 0;
            if (t >= kPfStages && !__all_sync(0xffffffffu, wait(kv_empty(st), (t / kPfStages - 1) & 1))) break;
            if (lane == 0) mbar_arrive_expect_tx(kv_full(st), (uint32_t)(nblk * BS * D * 2 * 2));
            const uint32_t kdst = base + Lay::kStage0 + st * Lay::kStageBytes;
            const uint32_t vdst = kdst + Lay::kKTile;
            for (int k = 0; k < nblk; ++k) {
                const int row = __shfl_sync(0xffffffffu, phys, k) * BS;
                if (lane == 0) {
#pragma unroll
                    for (int pl = 0; pl < kPlanes; ++pl) {
                        tma_load_4d(kdst + pl * kKPlane + k * BS * 128, &tmap_k, kv_full(st), 0, pl, g, row);
                        tma_load_4d(vdst + pl * kKPlane + k * BS * 128, &tmap_v, kv_full(st), 0, pl, g, row);
                    }
                }
            }
            issued = t + 1;
        }
        if (lane == 0 && *abort_flag) {  // let the loads this CTA issued land before it exits
            mbar_wait_bounded(q_full, 0);
            for (int st = 0; st < kPfStages; ++st)
                if (st < issued) {  // the stage's last tile: the largest t < issued with t % kPfStages == st
                    const int last = issued - 1 - (issued - 1 - st) % kPfStages;
                    mbar_wait_bounded(kv_full(st), (last / kPfStages) & 1);
                }
        }
    } else if (warp >= kPfMmaWarp && warp < kPfConvWarp) {
        // ------------------------------------------------------------ MMA issue
        // Warp 9 issues tile A's products, warp 10 tile B's.  Per key tile j:
        // S_X(j+1) into buffer (j+1) % 2 (after P_X(j-1) V has read it), then
        // P_X(j) V once the softmax has written P and V(j) is fp16.  Each warp
        // releases the K/V stage with its own commit, also for key tiles its
        // query tile skips.
        const int x = warp - kPfMmaWarp;
        const bool act = x == 0 || hasB;
        const int nkx = x == 0 ? nkA : nk;
        constexpr uint32_t kIdS = idesc_bf16_f32(kPfRows, kPfKeys, false, false);
        constexpr uint32_t kIdO = idesc_f16_f32(kPfRows, D, false, true);
        bool ok = __all_sync(0xffffffffu, wait(q_full, 0));
        const uint32_t qt = base + Lay::kQ + x * Lay::kQTile;
        // S_X(j) for key tile j into the tile's S buffer, as soon as the softmax
        // has read S_X(j-1) out of it (P goes to separate buffers, so S does not
        // wait for any P V product)
        auto issue_s = [&](int j) -> bool {
            const int st = j % kPfStages;
            if (!__all_sync(0xffffffffu, wait(kv_full(st), (j / kPfStages) & 1))) return false;
            if (j >= 1 && !__all_sync(0xffffffffu, wait(s_free(x), (j - 1) & 1))) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kt = base + Lay::kStage0 + st * Lay::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    tc_mma_bf16(tmem + x * Lay::kTmemTile,
                                desc_kmajor_sw128(qt + (kk >> 2) * kQPlane + (kk & 3) * 32),
                                desc_kmajor_sw128(kt + (kk >> 2) * kKPlane + (kk & 3) * 32), kIdS, kk > 0);
                }
                tc_commit(s_full(x));
            }
            __syncwarp();
            return true;
        };
        // The S product of the next key tile is issued before waiting for this
        // tile's P, so the softmax always finds its next S ready.
        if (ok && act && nkx > 0) ok = issue_s(0);
        for (int j = 0; ok && j < nk; ++j) {
            const int st = j % kPfStages;
            const int b = j & 1;
            const bool work = act && j < nkx;
            if (work) {
                if (j + 1 < nkx) {
                    ok = issue_s(j + 1);
                    if (!ok) break;
                }
                ok = __all_sync(0xffffffffu, wait(p_full(x, b), (j >> 1) & 1));
                if (ok) ok = __all_sync(0xffffffffu, wait(v16(st), (j / kPfStages) & 1));
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t vt = base + Lay::kStage0 + st * Lay::kStageBytes + Lay::kKTile;
                    // P of the tile's 64 keys: fp16 pairs in columns [0, 32); a K
                    // step of 16 keys is 8 columns
#pragma unroll
                    for (int kk = 0; kk < kPfKeys / 16; ++kk) {
                        tc_mma_bf16_ts(tmem + Lay::kTmemO + x * D,
                                       tmem + x * Lay::kTmemTile + kPfKeys + b * (kPfKeys / 2) + kk * 8,
                                       desc_mnmajor_sw128(vt + kk * 16 * 128, kKPlane), kIdO, j > 0 || kk > 0);
                    }
                    tc_commit(o_done(x, b));
                }
                __syncwarp();
            } else {
                // a key tile this query tile does not need: wait for it to land so the
                // release below cannot run ahead of the load
                ok = __all_sync(0xffffffffu, wait(kv_full(st), (j / kPfStages) & 1));
                if (!ok) break;
            }
            if (lane == 0) tc_commit(kv_empty(st));
            __syncwarp();
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
        for (int t = 0; t < nk; ++t) {
            const int st = t % kPfStages;
            if (!__all_sync(0xffffffffu, wait(kv_full(st), (t / kPfStages) & 1))) break;
            const int kv_valid = min(kPfKeys, L - t * kPfKeys);
            uint8_t *vt = base_ptr + Lay::kStage0 + st * Lay::kStageBytes + Lay::kKTile;
            uint4 v[kPlanes][4];
#pragma unroll
            for (int pl = 0; pl < kPlanes; ++pl)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[pl][k] = reinterpret_cast<const uint4 *>(vt + pl * kKPlane + c * 16 * 128)[lane + 32 * k];
#pragma unroll
            for (int pl = 0; pl < kPlanes; ++pl)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int key = 16 * c + 4 * k + (lane >> 3);  // 8 chunks of 16 bytes per 128-byte row
                    uint4 o = make_uint4(0, 0, 0, 0);
                    if (key < kv_valid) {
                        o.x = bf16x2_to_f16x2(v[pl][k].x, amax);
                        o.y = bf16x2_to_f16x2(v[pl][k].y, amax);
                        o.z = bf16x2_to_f16x2(v[pl][k].z, amax);
                        o.w = bf16x2_to_f16x2(v[pl][k].w, amax);
                    }
                    reinterpret_cast<uint4 *>(vt + pl * kKPlane + c * 16 * 128)[lane + 32 * k] = o;
                }
            fence_proxy_async_smem();  // the tensor cores read it through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(v16(st));
        }
        if (amax > 65504.f) record_status(kStatusValueRange);
    } else {
        // ------------------------------------------------------------ softmax
        const int x = warp >> 2;                 // query tile: 0 = A, 1 = B
        const int r = threadIdx.x & 127;         // MMA row = TMEM lane
        const bool active = x == 0 || hasB;
        const int nkx = x == 0 ? nkA : nk;
        const int tok = r / G;
        const int gi = r - tok * G;
        const int i = tA + x * p.tq + tok;
        const int endx = x == 0 ? endA : endB;
        const bool row_ok = active && tok < p.tq && i < endx;
        const int pos = row_ok ? ctx + i : L - 1;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t o_addr = lane_addr + Lay::kTmemO + x * D;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; active && j < nkx; ++j) {
            const int b = j & 1;
            const uint32_t s_addr = lane_addr + x * Lay::kTmemTile;
            const uint32_t p_addr = s_addr + kPfKeys + b * (kPfKeys / 2);
            ok = __all_sync(0xffffffffu, wait(s_full(x), j & 1));
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
            // weights (scaled by 2^kPfP16Shift) and their sum (8 partial sums);
            // P as fp16 pairs, the lower key in the low half
            // (logit scale, shift) on key pairs by packed fp32 FMAs; the row sum
            // in four packed fp32 accumulators
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
                const int jp = j - 1;
                ok = __all_sync(0xffffffffu, wait(o_done(x, jp & 1), (jp >> 1) & 1));
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
            // P into buffer b, once P_{j-2} V has read it
            if (j >= 2) {
                ok = __all_sync(0xffffffffu, wait(o_done(x, b), ((j >> 1) - 1) & 1));
                if (!ok) break;
                tc_fence_after();
            }
            tmem_st32(p_addr, pw);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full(x, b));
        }
        if (active && ok) {
            const int jl = nkx - 1;
            ok = __all_sync(0xffffffffu, wait(o_done(x, jl & 1), (jl >> 1) & 1));
        }
        if (active && ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst =
                p.out + ((int64_t)(q0 + (row_ok ? i : 0)) * p.num_heads + (int64_t)g * G + gi) * D;
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
