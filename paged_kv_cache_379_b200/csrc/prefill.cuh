// prefill.cuh -- multi-query paged prefill attention (chunked prefill, causal
// within the chunk) on the fifth-generation tensor cores.
//
// "vLLM 核心源码深度解析 …", milestone list (v0.5 Chunked Prefill): a long
// prompt is processed in chunks so that it does not hold up decodes; with the
// causal rule of "论文专题讲解：vLLM / PagedAttention …" (the query at position i
// attends to positions up to i), new token i of a chunk that starts at
// position ctx attends to positions 0 .. ctx + i, read through the block table.
//
// One CTA per work item (sequence s, KV head g, query tile).  A query tile is
// 128 MMA rows = tq tokens x G query heads (row r = token r / G, head r % G),
// so every K/V tile read from the cache feeds all G heads of the KV head.
//   warps 0-3  softmax: warp w owns TMEM lanes 32w..32w+31, i.e. one row per
//              thread; reads S_j from TMEM, online softmax with a lazily moved
//              reference max, and writes P_j back over S_j in TMEM as a bf16
//              high part and a bf16 residual (each truncated); rescales O in
//              TMEM when a reference moves; finally normalises O and stores the
//              output rows;
//   warp 4     producer: TMA loads of the query tile (once) and of 128-key K/V
//              tiles, block by block through the table, into a 3-stage ring;
//   warp 5     MMA: allocates TMEM -- three S/P buffers in columns 0..383, O in
//              384..384+D -- and one thread issues tcgen05.mma:
//                S_j = Q K_j^T              (SS form: M 128, N 128, K D)
//                O  += P_hi V_j + P_lo V_j  (TS form, P read from TMEM; V an
//                                            MN-major shared-memory operand)
//              with completion tracked by tcgen05.commit on mbarriers.  S_j
//              reuses buffer j % 3 once P_{j-3} V has completed.
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

constexpr int kPfThreads = 192;
constexpr int kPfProducerWarp = 4;
constexpr int kPfMmaWarp = 5;
constexpr int kPfRows = 128;          // MMA M: query rows per tile
constexpr int kPfKeys = 128;          // keys per K/V tile
constexpr int kPfStages = 3;          // K/V ring stages = TMEM S/P buffers
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kPfTmemO = 384;    // first TMEM column of O
// A row's softmax reference max moves only when a logit exceeds it by more
// than this (log2 units), so unnormalised weights stay below 2^8.
constexpr float kPfRescaleSlack = 8.f;

template <int D>
struct PfLayout {
    static constexpr int kPlane = kPfRows * 128;           // 128 rows x 128 bytes (64 bf16)
    static constexpr int kPlanes = D / 64;
    static constexpr int kQ = 0;
    static constexpr int kTile = kPlanes * kPlane;         // Q, K or V tile
    static constexpr int kStage0 = kQ + kTile;
    static constexpr int kStageBytes = 2 * kTile;          // K tile then V tile
    static constexpr int kBar = kStage0 + kPfStages * kStageBytes;
    // q_full, then per stage: kv_full, kv_empty, s_full, p_full, o_done; drain
    static constexpr int kNumBars = 2 + 5 * kPfStages;
    static constexpr int kMisc = kBar + kNumBars * 8;      // TMEM base, abort flag, item
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
};

template <int D, int BS>
__global__ void __launch_bounds__(kPfThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v)
{
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    using Lay = PfLayout<D>;
    constexpr int kPlane = Lay::kPlane;
    constexpr int kPlanes = Lay::kPlanes;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + Lay::kBar;
    const uint32_t q_full = bar0;
    const uint32_t drain = bar0 + 8;
    auto kv_full = [&](int st) { return bar0 + 8u * (2 + st); };
    auto kv_empty = [&](int st) { return bar0 + 8u * (2 + kPfStages + st); };
    auto s_full = [&](int b) { return bar0 + 8u * (2 + 2 * kPfStages + b); };
    auto p_full = [&](int b) { return bar0 + 8u * (2 + 3 * kPfStages + b); };
    auto o_done = [&](int b) { return bar0 + 8u * (2 + 4 * kPfStages + b); };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(base_ptr + Lay::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 4);
    volatile int *item = reinterpret_cast<volatile int *>(base_ptr + Lay::kMisc + 16);

    pdl_wait();
    pdl_launch_dependents();

    // ---- which (sequence, query tile) this CTA takes: blockIdx.x enumerates
    // the tiles of all sequences, each sequence's last (longest) tile first.
    if (warp == 0) {
        const int x = blockIdx.x;
        int found_s = -1, found_qt = 0, running = 0;
        for (int s0 = 0; s0 < p.num_seqs && found_s < 0; s0 += 32) {
            const int s = s0 + lane;
            int tiles = 0;
            if (s < p.num_seqs) {
                const int ql = p.q_start[s + 1] - p.q_start[s];
                if (ql > 0 && ql <= p.seq_lens[s]) tiles = (ql + p.tq - 1) / p.tq;
            }
            int incl = tiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = running + incl - tiles;
            const unsigned hit = __ballot_sync(0xffffffffu, tiles > 0 && x >= excl && x < excl + tiles);
            if (hit) {
                const int src = __ffs(hit) - 1;
                const int e = __shfl_sync(0xffffffffu, excl, src);
                const int tl = __shfl_sync(0xffffffffu, tiles, src);
                found_s = s0 + src;
                found_qt = tl - 1 - (x - e);
            }
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            item[0] = found_s;
            item[1] = found_qt;
        }
    }
    if (threadIdx.x == 32) {
        mbar_init(q_full, 1);
        mbar_init(drain, 1);
        for (int i = 0; i < kPfStages; ++i) {
            mbar_init(kv_full(i), 1);
            mbar_init(kv_empty(i), 1);
            mbar_init(s_full(i), 1);
            mbar_init(p_full(i), 128);
            mbar_init(o_done(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const int s = item[0];
    if (s < 0) return;  // past the last tile: the whole CTA leaves before any TMEM use
    const int qt = item[1];

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
    const int t_begin = qt * p.tq;
    const int t_end = min(q_len, t_begin + p.tq);
    const int nk = (ctx + t_end + kPfKeys - 1) / kPfKeys;  // causal: keys below ctx + t_end

    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait_bounded(bar, parity)) return true;
        record_timeout(kTimeoutFullBarrier);
        *abort_flag = 1;
        return false;
    };

    if (warp == kPfProducerWarp) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the tiles (lane k reads table entry k of a tile);
        // lane 0 issues the TMA loads.
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            mbar_arrive_expect_tx(q_full, (uint32_t)(kPlanes * G * p.q_box * 128));
            for (int pl = 0; pl < kPlanes; ++pl)
                tma_load_4d(base + Lay::kQ + pl * kPlane, &tmap_q, q_full, 0, pl, g * G, q0 + t_begin);
        }
        const int32_t *table = p.block_tables + (int64_t)s * p.max_blocks;
        int last[kPfStages] = {-1, -1, -1};
        for (int j = 0; j < nk; ++j) {
            const int st = j % kPfStages;
            const int key0 = j * kPfKeys;
            const int nblk = min(kPfKeys / BS, (L - key0 + BS - 1) / BS);
            const int phys = lane < nblk ? table[key0 / BS + lane] : 0;
            if (j >= kPfStages &&
                !__all_sync(0xffffffffu, wait(kv_empty(st), (j / kPfStages - 1) & 1)))
                break;
            if (lane == 0) mbar_arrive_expect_tx(kv_full(st), (uint32_t)(nblk * BS * D * 2 * 2));
            const uint32_t kdst = base + Lay::kStage0 + st * Lay::kStageBytes;
            const uint32_t vdst = kdst + Lay::kTile;
            for (int k = 0; k < nblk; ++k) {
                const int row = __shfl_sync(0xffffffffu, phys, k) * BS;
                if (lane == 0) {
#pragma unroll
                    for (int pl = 0; pl < kPlanes; ++pl) {
                        tma_load_4d(kdst + pl * kPlane + k * BS * 128, &tmap_k, kv_full(st), 0, pl, g, row);
                        tma_load_4d(vdst + pl * kPlane + k * BS * 128, &tmap_v, kv_full(st), 0, pl, g, row);
                    }
                }
            }
            last[st] = j;
        }
        if (lane == 0 && *abort_flag) {  // let the loads this CTA issued land before it exits
            mbar_wait_bounded(q_full, 0);
            for (int st = 0; st < kPfStages; ++st)
                if (last[st] >= 0) mbar_wait_bounded(kv_full(st), (last[st] / kPfStages) & 1);
        }
    } else if (warp == kPfMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        constexpr uint32_t kIdS = idesc_bf16_f32(kPfRows, kPfKeys, false, false);
        constexpr uint32_t kIdO = idesc_bf16_f32(kPfRows, D, false, true);
        bool ok = __all_sync(0xffffffffu, wait(q_full, 0));
        for (int j = 0; ok && j <= nk; ++j) {
            if (j < nk) {
                const int st = j % kPfStages;  // ring stage and TMEM S/P buffer
                ok = __all_sync(0xffffffffu, wait(kv_full(st), (j / kPfStages) & 1));
                if (!ok) break;
                // value rows past the sequence end hold stale or foreign data (maybe
                // NaN); P is 0 there, but 0 * NaN is NaN in the MMA: zero them
                const int kv_valid = min(kPfKeys, L - j * kPfKeys);
                if (kv_valid < kPfKeys) {
                    uint8_t *vt = base_ptr + Lay::kStage0 + st * Lay::kStageBytes + Lay::kTile;
                    const int chunks = (kPfKeys - kv_valid) * 8;
                    for (int i = lane; i < kPlanes * chunks; i += 32) {
                        const int pl = i / chunks, c = i - pl * chunks;
                        *reinterpret_cast<uint4 *>(vt + pl * kPlane + kv_valid * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (j >= kPfStages) {  // buffer st is free once P_{j-3} V has completed
                    ok = __all_sync(0xffffffffu, wait(o_done(st), (j / kPfStages - 1) & 1));
                    if (!ok) break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kt = base + Lay::kStage0 + st * Lay::kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kPlane + (kk & 3) * 32;
                        tc_mma_bf16(tmem + st * kPfKeys, desc_kmajor_sw128(base + Lay::kQ + off),
                                    desc_kmajor_sw128(kt + off), kIdS, kk > 0);
                    }
                    tc_commit(s_full(st));
                }
                __syncwarp();
            }
            if (j >= 1) {
                const int jp = j - 1, bp = jp % kPfStages;
                ok = __all_sync(0xffffffffu, wait(p_full(bp), (jp / kPfStages) & 1));
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t vt = base + Lay::kStage0 + bp * Lay::kStageBytes + Lay::kTile;
                    // P_hi in columns [0, 64) of the buffer, P_lo in [64, 128); a K step
                    // of 16 keys is 8 columns
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int kk = 0; kk < kPfKeys / 16; ++kk) {
                            tc_mma_bf16_ts(tmem + kPfTmemO, tmem + bp * kPfKeys + half * 64 + kk * 8,
                                           desc_mnmajor_sw128(vt + kk * 16 * 128, kPlane), kIdO,
                                           jp > 0 || half > 0 || kk > 0);
                        }
                    }
                    tc_commit(kv_empty(bp));
                    tc_commit(o_done(bp));
                }
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int r = threadIdx.x;  // MMA row = TMEM lane
        const int tok = r / G;
        const int gi = r - tok * G;
        const int i = t_begin + tok;
        const bool row_ok = tok < p.tq && i < t_end;
        const int pos = row_ok ? ctx + i : L - 1;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const int b = j % kPfStages;
            ok = __all_sync(0xffffffffu, wait(s_full(b), (j / kPfStages) & 1));
            if (!ok) break;
            tc_fence_after();
            float x[kPfKeys];
            tmem_ld128(lane_addr + b * kPfKeys, x);
            // causal mask, only in tiles that reach past some row's position
            const int lim = pos - j * kPfKeys;  // keys c <= lim are visible
            if (!__all_sync(0xffffffffu, lim >= kPfKeys - 1)) {
#pragma unroll
                for (int c = 0; c < kPfKeys; ++c) x[c] = c <= lim ? x[c] : -INFINITY;
            }
            // row max as a tree over 8 independent partial maxima
            float pm[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pm[u] = x[u];
#pragma unroll
            for (int c = 8; c < kPfKeys; ++c) pm[c & 7] = fmaxf(pm[c & 7], x[c]);
            const float mx =
                fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) *
                p.scale_log2;  // scale > 0: the max commutes with it
            // lazily moved reference max (log2 units): weights stay <= 2^kPfRescaleSlack
            const bool bump = mx > m + kPfRescaleSlack;
            float corr = 1.f;
            if (bump) {
                corr = fast_exp2(m - mx);  // 0 on the first tile (m = -inf)
                m = mx;
            }
            // weights, their sum (8 independent partial sums), and P split into a
            // bf16 high part and a bf16 residual, both by truncation (the pair
            // keeps 16 significant bits: relative error below 2^-15)
            float ps[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) ps[u] = 0.f;
            uint32_t hl[kPfKeys];  // [0, 64): high parts, [64, 128): residuals
#pragma unroll
            for (int e = 0; e < kPfKeys / 2; ++e) {
                const float p0 = fast_exp2(fmaf(x[2 * e], p.scale_log2, -m));
                const float p1 = fast_exp2(fmaf(x[2 * e + 1], p.scale_log2, -m));
                ps[e & 7] += p0 + p1;
                const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                hl[e] = prmt(b0, b1, 0x7632u);  // high halves: bf16(p0) | bf16(p1) << 16
                const float r0 = p0 - __uint_as_float(b0 & 0xFFFF0000u);
                const float r1 = p1 - __uint_as_float(b1 & 0xFFFF0000u);
                hl[kPfKeys / 2 + e] = prmt(__float_as_uint(r0), __float_as_uint(r1), 0x7632u);
            }
            l = l * corr + (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7])));
            if (j >= 1 && __any_sync(0xffffffffu, bump)) {
                // O holds P_{<j} V: rescale it once P_{j-1} V has completed
                const int jp = j - 1;
                ok = __all_sync(0xffffffffu, wait(o_done(jp % kPfStages), (jp / kPfStages) & 1));
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float o[32];
                    tmem_ld32(lane_addr + kPfTmemO + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= corr;
                    tmem_st32(lane_addr + kPfTmemO + c * 32, o);
                }
            }
            // P over S in this buffer's columns
            tmem_st64(lane_addr + b * kPfKeys, hl);
            tmem_st64(lane_addr + b * kPfKeys + 64, hl + 64);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full(b));
        }
        if (ok) ok = __all_sync(0xffffffffu, wait(o_done((nk - 1) % kPfStages), ((nk - 1) / kPfStages) & 1));
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst =
                p.out + ((int64_t)(q0 + (row_ok ? i : 0)) * p.num_heads + (int64_t)g * G + gi) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tmem_ld32(lane_addr + kPfTmemO + c * 32, o);
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
    if (warp == kPfMmaWarp) {
        tc_fence_after();
        // all MMAs this CTA issued have completed before TMEM is released
        if (lane == 0) tc_commit(drain);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(drain, 0)) && lane == 0) record_timeout(kTimeoutDrain);
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

}  // namespace pakv
