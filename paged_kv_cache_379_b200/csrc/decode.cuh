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
// Work unit: one CTA per (sequence, KV head, partition).  All G = Hq/Hkv query
// heads of the KV head are handled by the same CTA, so every K/V byte crosses
// HBM once.  A partition is a run of `part_tokens` positions; the one-pass form
// is a single partition covering the whole sequence.
//
// CTA = 4 consumer warps + 1 producer warp.
//  * Producer: one coalesced warp load of up to 32 table entries, then for each
//    16-token tile one elected lane issues TMA tile loads of the tile's K and V
//    blocks (box = [bs tokens x 1 head x head_dim], 128B-swizzled) into an
//    8-stage shared-memory ring guarded by mbarriers.  Nothing else touches HBM.
//  * Consumers: tile i goes to warp i % 4 (each warp owns 2 stages).  Every warp
//    keeps its own running max m, sum l and fp32 accumulator; the four states
//    are merged through shared memory at the end.
//    - G >= 3 (grouped heads: a dense [16 x D] . [D x G] contraction per tile):
//      bf16 mma.sync m16n8k16 in transposed form, S^T = K Q^T with the K tile as
//      the A operand (rows = tokens, via ldmatrix) and Q^T in registers, then
//      O^T += V^T P^T with V^T through ldmatrix.trans and P^T moved out of the
//      S^T accumulators by movmatrix.trans; P goes in as bf16 hi + residual.
//    - G <= 2 (MHA-like, a matrix-vector product): CUDA cores, 16-byte shared
//      loads, warp-shuffle reductions for the dot products, max and sum.
//  * Masking selects (-inf logits, zeroed V rows) instead of multiplying by 0,
//    so stale or NaN data in unused slots of a partial block is never mixed in.
//  * Every mbarrier wait is bounded in time (about 1 s); on expiry the kernel
//    records a code in the device status word, drains its own TMA copies and
//    returns.
// Split form: a partition's (m, l, o) go to a workspace and lse_reduce_kernel
// merges them; a sequence with a single partition is finished in place.
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
    float scale_log2;                 // scale * log2(e)
    int num_seqs, num_heads, num_kv_heads, group, max_blocks;
    int part_tokens;                  // positions per partition (multiple of 16)
    int max_parts;                    // partitions per sequence in the grid; 1 = one pass
    int direct_single;                // a sequence with one partition writes `out`
};

struct ReduceParams {
    __nv_bfloat16 *out;
    const float *ws_o, *ws_m, *ws_l;
    const int32_t *seq_lens;
    int num_seqs, num_heads, head_dim, part_tokens, max_parts;
    int skip_single;                  // sequences with one partition are already done
};

constexpr int kConsumerWarps = 4;
constexpr int kStages = 8;
constexpr int kTileTokens = 16;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr float kLn2 = 0.693147180559945309f;

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
    static constexpr int kPipeSmem = kStages * kStageSmem;
    static constexpr int kSmemBytes = kPipeSmem + 1024 /* alignment slack */ + 2 * kStages * 8 + 16;

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

// Merge scratch (reuses the drained pipeline ring): per consumer warp, the
// running max (log2 units), sum and accumulator of up to 16 heads.
template <int D>
struct MergeScratch {
    float o[kConsumerWarps][16][D + 4];  // +4: heads 2tq+j land in distinct banks
    float m[kConsumerWarps][16];
    float l[kConsumerWarps][16];
};

template <int D, int BS, int MODE, int GC>
__global__ void __launch_bounds__(kDecodeThreads, 2)
    paged_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v)
{
    // MODE 0: CUDA cores, GC (1 or 2) query heads per KV head.
    // MODE 1: tensor cores, up to 8 query heads per KV head (one 8-head tile).
    // MODE 2: tensor cores, up to 16 query heads per KV head (two 8-head tiles).
    using Geo = TileGeom<D, BS>;
    static_assert(sizeof(MergeScratch<D>) <= Geo::kPipeSmem, "merge scratch must fit the ring");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const uint32_t full_bar = base + Geo::kPipeSmem;
    const uint32_t empty_bar = full_bar + kStages * 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base_ptr + Geo::kPipeSmem + 2 * kStages * 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int bid = blockIdx.x;
    const int g = bid % p.num_kv_heads;
    bid /= p.num_kv_heads;
    const int s = bid % p.num_seqs;
    const int part = bid / p.num_seqs;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full_bar + 8 * i, 1);
            mbar_init(empty_bar + 8 * i, 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x == kConsumerWarps * 32) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    const int L = min(p.seq_lens[s], p.max_blocks * BS);
    int nparts = 1;
    int t_begin = 0, t_end = L;
    if (p.max_parts > 1) {
        nparts = L > 0 ? min((L + p.part_tokens - 1) / p.part_tokens, p.max_parts) : 1;
        t_begin = part * p.part_tokens;
        t_end = min(L, t_begin + p.part_tokens);
    }
    const int G = (MODE == 0) ? GC : p.group;
    if (part >= nparts) {  // uniform over the CTA
        if (!p.direct_single) {
            // partitions-only form: an empty partition reports m = -inf, l = 0, o = 0
            for (int idx = threadIdx.x; idx < G * D; idx += kDecodeThreads) {
                const int row = idx / D;
                const int64_t wi = ((int64_t)s * p.num_heads + (int64_t)g * G + row) * p.max_parts + part;
                p.ws_o[wi * D + (idx - row * D)] = 0.f;
                if (idx - row * D == 0) {
                    p.ws_m[wi] = -INFINITY;
                    p.ws_l[wi] = 0.f;
                }
            }
        }
        return;
    }
    const int n_tiles = t_end > t_begin ? (t_end - t_begin + kTileTokens - 1) / kTileTokens : 0;
    const bool direct = p.direct_single && nparts == 1;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        const int32_t *table = p.block_tables + (int64_t)s * p.max_blocks;
        const int first_blk = t_begin / BS;
        const int end_blk = (t_end + BS - 1) / BS;
        int issued = 0;
        bool stop = false;
        for (int cb = first_blk; cb < end_blk && !stop; cb += 32) {
            const int nchunk = min(32, end_blk - cb);
            const int my = lane < nchunk ? __ldg(table + cb + lane) : 0;
            for (int j = 0; j < nchunk; j += Geo::kBlocksPerTile) {
                int phys[Geo::kBlocksPerTile];
#pragma unroll
                for (int k = 0; k < Geo::kBlocksPerTile; ++k) phys[k] = __shfl_sync(0xffffffffu, my, (j + k) & 31);
                const int valid = min(Geo::kBlocksPerTile, nchunk - j);
                if (lane == 0) {
                    const int stage = issued % kStages;
                    const uint32_t parity = ((issued / kStages) & 1) ^ 1;
                    if (*abort_flag) {
                        stop = true;
                    } else if (!mbar_wait_bounded(empty_bar + 8 * stage, parity)) {
                        record_timeout(kTimeoutEmptyBarrier);
                        *abort_flag = 1;
                        stop = true;
                    } else {
                        const uint32_t kdst = base + stage * Geo::kStageSmem;
                        const uint32_t vdst = kdst + Geo::kTileSmem;
                        const uint32_t bar = full_bar + 8 * stage;
                        mbar_arrive_expect_tx(bar, (uint32_t)(valid * Geo::kBlkBytes * 2));
#pragma unroll
                        for (int k = 0; k < Geo::kBlocksPerTile; ++k) {
                            if (k < valid) {
#pragma unroll
                                for (int h = 0; h < Geo::kHalves; ++h) {
                                    tma_load_4d(kdst + Geo::box_offset(k, h), &tmap_k, bar, 0, h, g, phys[k] * BS);
                                    tma_load_4d(vdst + Geo::box_offset(k, h), &tmap_v, bar, 0, h, g, phys[k] * BS);
                                }
                            }
                        }
                        ++issued;
                    }
                }
                stop = __shfl_sync(0xffffffffu, stop, 0);
                if (stop) break;
            }
        }
        // On an abort, wait for the copies already in flight before the ring is
        // reused or the CTA exits.
        if (lane == 0 && *abort_flag && issued > 0) {
            for (int st = 0; st < kStages && st < issued; ++st) {
                const int last = issued - 1 - ((issued - 1 - st) % kStages);
                if (!mbar_wait_bounded(full_bar + 8 * st, (last / kStages) & 1)) record_timeout(kTimeoutDrain);
            }
        }
    } else {
        // ----------------------------------------------------------- consumers
        MergeScratch<D> *ms = reinterpret_cast<MergeScratch<D> *>(base_ptr);
        const int64_t q_off = ((int64_t)s * p.num_heads + (int64_t)g * G) * D;

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
                const uint4 raw_q = *reinterpret_cast<const uint4 *>(p.query + q_off + (int64_t)h * D + qc * 8);
                const uint32_t w[4] = {raw_q.x, raw_q.y, raw_q.z, raw_q.w};
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
            for (int tile = warp; tile < n_tiles; tile += kConsumerWarps) {
                const int stage = tile % kStages;
                if (*abort_flag) break;
                const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar + 8 * stage, (tile / kStages) & 1));
                if (!ok) {
                    if (lane == 0) { record_timeout(kTimeoutFullBarrier); *abort_flag = 1; }
                    break;
                }
                const uint32_t kt = base + stage * Geo::kStageSmem;
                const uint32_t vt = kt + Geo::kTileSmem;
                const int valid = min(kTileTokens, t_end - (t_begin + tile * kTileTokens));
                if (valid < kTileTokens) zero_tail(vt, valid);

                float sv[GC][PASSES];
#pragma unroll
                for (int j = 0; j < PASSES; ++j) {
                    const int tok = j * TPP + qt;
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
                        sv[h][j] = tok < valid ? dot : -INFINITY;
                    }
                }
                float pr[GC][PASSES];
#pragma unroll
                for (int h = 0; h < GC; ++h) {
                    float mx = sv[h][0];
#pragma unroll
                    for (int j = 1; j < PASSES; ++j) mx = fmaxf(mx, sv[h][j]);
#pragma unroll
                    for (int off = CPT; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    const float m_new = fmaxf(m[h], mx);
                    const float corr = exp2f(m[h] - m_new);
                    m[h] = m_new;
                    float sum = 0.f;
#pragma unroll
                    for (int j = 0; j < PASSES; ++j) {
                        pr[h][j] = exp2f(sv[h][j] - m_new);
                        sum += pr[h][j];
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
                if (valid < kTileTokens) fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar + 8 * stage);
            }
            __syncthreads();  // ring drained (all consumers and the producer are past it)
#pragma unroll
            for (int h = 0; h < GC; ++h) {
#pragma unroll
                for (int e = 0; e < DPL; ++e) ms->o[warp][h][DPL * lane + e] = o[h][e];
                if (lane == 0) {
                    ms->m[warp][h] = m[h];
                    ms->l[warp][h] = l[h];
                }
            }
        } else {
            // Tensor cores, transposed form: S^T[16 tokens x 8*NH heads] = K Q^T,
            // then O^T[D x heads] += V^T P^T.  Tokens are the MMA's M dimension,
            // so no accumulator row is wasted when G <= 8; P^T is taken from the
            // S^T accumulators by an in-register 8x8 transpose (movmatrix).
            constexpr int NH = (MODE == 2) ? 2 : 1;  // 8-head column tiles
            constexpr int KSTEPS = D / 16;           // k-steps of S^T = K Q^T
            constexpr int MT = D / 16;               // 16-row d tiles of O^T
            const int gq = lane >> 2;                // MMA groupID
            const int tq = lane & 3;                 // MMA thread-in-group
            // B operand of S^T = K Q^T: b0 = Q[head][d 16kk+2tq..+1], b1 = Q[head][d 16kk+8+2tq..+1]
            uint32_t qb[NH][KSTEPS][2];
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
                const int head = nh * 8 + gq;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int col = kk * 16 + hh * 8 + tq * 2;
                        qb[nh][kk][hh] = head < G
                                             ? *reinterpret_cast<const uint32_t *>(p.query + q_off + (int64_t)head * D + col)
                                             : 0u;
                    }
                }
            }
            float o[MT][NH][4];
            float m[NH][2], l[NH][2];
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
                m[nh][0] = m[nh][1] = -INFINITY;
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

            for (int tile = warp; tile < n_tiles; tile += kConsumerWarps) {
                const int stage = tile % kStages;
                if (*abort_flag) break;
                const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar + 8 * stage, (tile / kStages) & 1));
                if (!ok) {
                    if (lane == 0) { record_timeout(kTimeoutFullBarrier); *abort_flag = 1; }
                    break;
                }
                const uint32_t kt = base + stage * Geo::kStageSmem;
                const uint32_t vt = kt + Geo::kTileSmem;
                const int valid = min(kTileTokens, t_end - (t_begin + tile * kTileTokens));
                if (valid < kTileTokens) zero_tail(vt, valid);

                // S^T[token][head] = K Q^T
                float sc[NH][4];
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) sc[nh][0] = sc[nh][1] = sc[nh][2] = sc[nh][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(kt + Geo::chunk_offset(ktok, 2 * kk + kpar), a0, a1, a2, a3);
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh) mma_bf16_16816(sc[nh], a0, a1, a2, a3, qb[nh][kk][0], qb[nh][kk][1]);
                }
                // online softmax per head column; this lane holds tokens gq and gq+8
                // of heads 2tq and 2tq+1.  P enters the PV product as a bf16 high
                // part plus a bf16 residual (two MMAs): ~16 significant bits.
                const bool in0 = gq < valid, in1 = gq + 8 < valid;
                uint32_t bh[NH][2], bl[NH][2];
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) {
                    float pr[2][2];  // [head j][token row]
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float x0 = in0 ? sc[nh][j] * p.scale_log2 : -INFINITY;
                        const float x1 = in1 ? sc[nh][2 + j] * p.scale_log2 : -INFINITY;
                        float mx = fmaxf(x0, x1);
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        const float m_new = fmaxf(m[nh][j], mx);
                        const float corr = exp2f(m[nh][j] - m_new);
                        m[nh][j] = m_new;
                        pr[j][0] = exp2f(x0 - m_new);
                        pr[j][1] = exp2f(x1 - m_new);
                        l[nh][j] = l[nh][j] * corr + (pr[j][0] + pr[j][1]);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            o[mt][nh][j] *= corr;
                            o[mt][nh][2 + j] *= corr;
                        }
                    }
#pragma unroll
                    for (int row = 0; row < 2; ++row) {
                        const uint32_t hi = pack_bf16x2(pr[0][row], pr[1][row]);
                        const float2 hf = unpack_bf16x2(hi);
                        const uint32_t lo = pack_bf16x2(pr[0][row] - hf.x, pr[1][row] - hf.y);
                        bh[nh][row] = movmatrix_trans(hi);
                        bl[nh][row] = movmatrix_trans(lo);
                    }
                }
                // O^T[d][head] += V^T P^T
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
                if (valid < kTileTokens) fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar + 8 * stage);
            }
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    l[nh][j] += __shfl_xor_sync(0xffffffffu, l[nh][j], 4);
                    l[nh][j] += __shfl_xor_sync(0xffffffffu, l[nh][j], 8);
                    l[nh][j] += __shfl_xor_sync(0xffffffffu, l[nh][j], 16);
                }
            }
            __syncthreads();  // ring drained
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int head = nh * 8 + 2 * tq + j;
                    if (head < G) {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            ms->o[warp][head][mt * 16 + gq] = o[mt][nh][j];
                            ms->o[warp][head][mt * 16 + gq + 8] = o[mt][nh][2 + j];
                        }
                        if (gq == 0) {
                            ms->m[warp][head] = m[nh][j];
                            ms->l[warp][head] = l[nh][j];
                        }
                    }
                }
            }
        }
    }
    if (warp == kConsumerWarps) __syncthreads();  // pairs with the consumers' "ring drained"
    __syncthreads();                              // merge scratch written

    // ------------------------------------------------ merge the four warps
    if (*abort_flag) return;
    const MergeScratch<D> *ms = reinterpret_cast<const MergeScratch<D> *>(base_ptr);
    for (int idx = threadIdx.x; idx < G * D; idx += kDecodeThreads) {
        const int row = idx / D;
        const int d = idx - row * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ms->m[w][row]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float mw = ms->m[w][row];
                if (mw != -INFINITY) {
                    const float c = exp2f(mw - M);
                    num = fmaf(c, ms->o[w][row][d], num);
                    den = fmaf(c, ms->l[w][row], den);
                }
            }
        }
        const int64_t hrow = (int64_t)s * p.num_heads + (int64_t)g * G + row;
        if (direct) {
            p.out[hrow * D + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
        } else {
            const int64_t wi = hrow * p.max_parts + part;
            p.ws_o[wi * D + d] = num;
            if (d == 0) {
                p.ws_m[wi] = M == -INFINITY ? -INFINITY : M * kLn2;
                p.ws_l[wi] = den;
            }
        }
    }
}

// Log-sum-exp merge of the partitions of one (sequence, head) per warp:
//   M = max_p m_p,  out = sum_p e^{m_p - M} o_p / sum_p e^{m_p - M} l_p.
// Lane p computes the weight of partition p; the weighted sum over partitions
// reads each partition's o row as one coalesced 16-byte (D = 128) or 8-byte
// (D = 64) vector per lane.
constexpr int kReduceWarps = 8;

template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32) lse_reduce_kernel(const ReduceParams r)
{
    constexpr int VEC = D / 32;
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kReduceWarps + (threadIdx.x >> 5);
    if (row >= (int64_t)r.num_seqs * r.num_heads) return;
    const int s = (int)(row / r.num_heads);
    const int L = r.seq_lens[s];
    int nparts = L > 0 ? (L + r.part_tokens - 1) / r.part_tokens : 1;
    nparts = min(nparts, r.max_parts);
    if (r.skip_single && nparts == 1) return;
    const float *m = r.ws_m + row * r.max_parts;
    const float *l = r.ws_l + row * r.max_parts;
    const float *o = r.ws_o + row * r.max_parts * D + lane * VEC;

    float M = -INFINITY;
    for (int i = lane; i < nparts; i += 32) M = fmaxf(M, m[i]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int i0 = 0; i0 < nparts; i0 += 32) {
            const int i = i0 + lane;
            const float w = (i < nparts) ? expf(m[i] - M) : 0.f;  // an empty partition has m = -inf: weight 0
            den += (i < nparts) ? w * l[i] : 0.f;
            const int cnt = min(32, nparts - i0);
            int j = 0;
            for (; j + 4 <= cnt; j += 4) {
                float wj[4], v[4][VEC];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    wj[u] = __shfl_sync(0xffffffffu, w, j + u);
                    const float *src = o + (int64_t)(i0 + j + u) * D;
                    if constexpr (VEC == 4) {
                        const float4 f = *reinterpret_cast<const float4 *>(src);
                        v[u][0] = f.x; v[u][1] = f.y; v[u][2] = f.z; v[u][3] = f.w;
                    } else {
                        const float2 f = *reinterpret_cast<const float2 *>(src);
                        v[u][0] = f.x; v[u][1] = f.y;
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] = fmaf(wj[u], v[u][e], acc[e]);
            }
            for (; j < cnt; ++j) {
                const float wj = __shfl_sync(0xffffffffu, w, j);
                const float *src = o + (int64_t)(i0 + j) * D;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] = fmaf(wj, src[e], acc[e]);
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    }
    __nv_bfloat16 *dst = r.out + row * D + lane * VEC;
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[e] = __float2bfloat16_rn(den > 0.f ? acc[e] / den : 0.f);
}

}  // namespace pakv
