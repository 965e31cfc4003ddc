// pagedkv.cu -- the C ABI of libpagedkv.so (declared in include/pagedkv.h):
// argument checks, TMA tensor-map encoding, kernel selection and launch.
// The kernels themselves are in cache_ops.cuh and decode.cuh.
#include <algorithm>
#include <atomic>
#include <climits>
#include <mutex>
#include <tuple>
#include <vector>

#include "cache_ops.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"

namespace pakv {

static thread_local int t_last_cuda_error = 0;
void set_last_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

// ----------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// The cache [num_blocks, bs, Hkv, D] seen by TMA as 4-D (innermost first):
//   {64 elements = 128 B, D/64, Hkv, num_blocks*bs slots}
// with a box of one 64-wide d-plane of one block of one head: {64, 1, 1, bs},
// 128-byte swizzle.
// An FP8 cache (1-byte codes, head_dim 128) is {128 codes = 128 B, 1, Hkv, slots}
// with a box {128, 1, 1, bs}: one 128-byte row per token.
// With block_box the dimensions are ordered {64 elements, slots, D/64 planes,
// Hkv} (strides Hkv*D*2, 128, D*2 bytes) and the box is {64, bs, D/64, 1}: one
// block of one head, both planes, landing plane-major.
static int make_cache_map(CUtensorMap *map, const void *cache, int64_t num_blocks, int bs, int hkv, int d,
                          bool fp8 = false, bool block_box = false)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return check_cuda(cudaErrorNotSupported);
    const int esize = fp8 ? 1 : 2;
    const int inner = 128 / esize;  // elements per 128-byte row
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)(d / inner), (cuuint64_t)hkv,
                          (cuuint64_t)(num_blocks * bs)};
    cuuint64_t strides[3] = {128, (cuuint64_t)d * esize, (cuuint64_t)hkv * d * esize};
    cuuint32_t box[4] = {(cuuint32_t)inner, 1, 1, (cuuint32_t)bs};
    if (block_box) {
        dims[1] = (cuuint64_t)(num_blocks * bs);
        dims[2] = (cuuint64_t)(d / inner);
        dims[3] = (cuuint64_t)hkv;
        strides[0] = (cuuint64_t)hkv * d * esize;
        strides[1] = 128;
        strides[2] = (cuuint64_t)d * esize;
        box[1] = (cuuint32_t)bs;
        box[2] = (cuuint32_t)(d / inner);
        box[3] = 1;
    }
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                          const_cast<void *>(cache), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_last_cuda_error(cudaErrorInvalidValue);
        return PA_ERR_CUDA;
    }
    return PA_OK;
}

// The queries [T, Hq, D] as {64 elements, D/64, Hq, T} with a box of one
// 64-wide d-plane of G heads x q_box tokens: rows token-major, head-minor.
static int make_query_map(CUtensorMap *map, const void *query, int64_t tokens, int hq, int d, int g, int q_box)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return check_cuda(cudaErrorNotSupported);
    const cuuint64_t dims[4] = {64, (cuuint64_t)(d / 64), (cuuint64_t)hq, (cuuint64_t)tokens};
    const cuuint64_t strides[3] = {128, (cuuint64_t)d * 2, (cuuint64_t)hq * d * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)g, (cuuint32_t)q_box};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(query), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_last_cuda_error(cudaErrorInvalidValue);
        return PA_ERR_CUDA;
    }
    return PA_OK;
}

// --------------------------------------------------------------- decode launch

// Raises a kernel's dynamic shared-memory limit (per device) when a launch
// needs more than was set before.
static int ensure_smem(const void *kernel, size_t bytes)
{
    static std::mutex mu;
    static std::vector<std::tuple<const void *, int, size_t>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_cuda(e);
    std::lock_guard<std::mutex> lock(mu);
    for (auto &t : done)
        if (std::get<0>(t) == kernel && std::get<1>(t) == dev && std::get<2>(t) >= bytes) return PA_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return check_cuda(e);
    done.emplace_back(kernel, dev, bytes);
    return PA_OK;
}

static int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const int slot = dev & 63;
    int n = cache[slot].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[slot].store(n, std::memory_order_relaxed);
    return n;
}

// Persistent launch: (resident CTAs per SM) x (SM count) CTAs, at most one per item.
template <int D, int BS, int MODE, int GC, bool FP8 = false>
static int launch_decode_t(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int64_t max_items,
                           cudaStream_t st)
{
    using Lay = DecodeSmem<D, BS, MODE, GC, FP8>;
    auto kernel = paged_decode_kernel<D, BS, MODE, GC, FP8>;
    const size_t smem = (size_t)Lay::bytes(p.num_seqs, p.num_groups);
    if (smem > 227 * 1024) return PA_ERR_BAD_SHAPE;  // too many sequences for the enumeration tables
    int rc = ensure_smem(reinterpret_cast<const void *>(kernel), smem);
    if (rc != PA_OK) return rc;
    int occ = 0;
    rc = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kDecodeThreads, smem));
    if (rc != PA_OK) return rc;
    const int sms = sm_count();
    if (occ < 1 || sms < 1) return check_cuda(cudaErrorInvalidConfiguration);
    const int64_t grid = std::min<int64_t>(max_items, (int64_t)occ * sms);
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kDecodeThreads), smem, st, p, tk, tv);
}

template <int D, int BS>
static int launch_decode_bs(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int64_t grid,
                            cudaStream_t st)
{
    const int G = p.group;
    // shared-prefix groups: 16-column tensor-core items, ROWS / G sequences each
    if (p.num_groups > 0) return G <= 16 ? launch_decode_t<D, BS, 2, 0>(p, tk, tv, grid, st) : PA_ERR_UNSUPPORTED;
    if (G == 1) return launch_decode_t<D, BS, 0, 1>(p, tk, tv, grid, st);
    if (G == 2) return launch_decode_t<D, BS, 0, 2>(p, tk, tv, grid, st);
    if (G <= 8) return launch_decode_t<D, BS, 1, 0>(p, tk, tv, grid, st);
    if (G <= 16) return launch_decode_t<D, BS, 2, 0>(p, tk, tv, grid, st);
    return PA_ERR_UNSUPPORTED;
}

// FP8 cache (head_dim 128, bs 8 or 16): always the tensor-core consumers.
template <int BS>
static int launch_decode_fp8_bs(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int64_t grid,
                                cudaStream_t st)
{
    if (p.group <= 8) return launch_decode_t<128, BS, 1, 0, true>(p, tk, tv, grid, st);
    if (p.group <= 16) return launch_decode_t<128, BS, 2, 0, true>(p, tk, tv, grid, st);
    return PA_ERR_UNSUPPORTED;
}

template <int D>
static int launch_decode_d(int bs, const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv,
                           int64_t grid, cudaStream_t st)
{
    switch (bs) {
    case 4: return launch_decode_bs<D, 4>(p, tk, tv, grid, st);
    case 8: return launch_decode_bs<D, 8>(p, tk, tv, grid, st);
    case 16: return launch_decode_bs<D, 16>(p, tk, tv, grid, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

// Rows of more than 32 partitions are merged by a whole CTA (8 warps) each,
// the others by one warp each.
static int launch_reduce(const ReduceParams &r, cudaStream_t st)
{
    const int64_t rows = (int64_t)r.num_seqs * r.num_heads;
    const bool wide = r.max_parts > 32;
    const int rows_per_cta = wide ? 1 : kReduceWarps;
    if (cdiv64(rows, rows_per_cta) > INT_MAX) return PA_ERR_BAD_SHAPE;
    const dim3 grid((unsigned)cdiv64(rows, rows_per_cta)), block(kReduceWarps * 32);
    if (r.head_dim == 64)
        return wide ? launch_pdl(lse_reduce_kernel<64, kReduceWarps>, grid, block, 0, st, r)
                    : launch_pdl(lse_reduce_kernel<64, 1>, grid, block, 0, st, r);
    return wide ? launch_pdl(lse_reduce_kernel<128, kReduceWarps>, grid, block, 0, st, r)
                : launch_pdl(lse_reduce_kernel<128, 1>, grid, block, 0, st, r);
}

struct DecodeArgs {
    void *out;
    const void *query, *key_cache, *value_cache;
    const int32_t *block_tables, *seq_lens;
    float scale;
    int block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks, num_blocks, max_seq_len;
    bool fp8 = false;             // caches hold E4M3 codes
    float k_scale = 1.f, v_scale = 1.f;
    const int32_t *grp_start = nullptr, *grp_parts = nullptr;  // shared-prefix groups (device)
    int num_groups = 0;
};

static int check_decode_args(const DecodeArgs &a, bool need_out)
{
    if ((need_out && !a.out) || !a.query || !a.key_cache || !a.value_cache || !a.block_tables || !a.seq_lens)
        return PA_ERR_NULL_POINTER;
    if (a.num_seqs < 0 || a.num_heads <= 0 || a.num_kv_heads <= 0 || a.head_dim <= 0 || a.block_size <= 0 ||
        a.max_blocks <= 0 || a.num_blocks <= 0 || a.max_seq_len < 0)
        return PA_ERR_BAD_SHAPE;
    if (a.num_heads % a.num_kv_heads != 0) return PA_ERR_BAD_SHAPE;
    if (a.head_dim != 64 && a.head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (a.block_size != 4 && a.block_size != 8 && a.block_size != 16) return PA_ERR_UNSUPPORTED;
    if (a.num_heads / a.num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
    if (a.fp8 && (a.head_dim != 128 || a.block_size < 8)) return PA_ERR_UNSUPPORTED;
    if (a.fp8 && !(a.k_scale > 0.f && a.v_scale > 0.f && a.k_scale < INFINITY && a.v_scale < INFINITY))
        return PA_ERR_BAD_SHAPE;
    if ((int64_t)a.num_blocks * a.block_size > INT_MAX) return PA_ERR_BAD_SHAPE;
    if ((int64_t)a.max_blocks * a.block_size > INT_MAX) return PA_ERR_BAD_SHAPE;
    if (!aligned16(a.query) || !aligned16(a.key_cache) || !aligned16(a.value_cache) ||
        (need_out && !aligned16(a.out)))
        return PA_ERR_ALIGNMENT;
    return PA_OK;
}

static constexpr size_t kSchedBytes = 256;  // workspace header: the scheduler counters
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static int max_parts_for(int max_seq_len, int part) { return max_seq_len > 0 ? (int)cdiv64(max_seq_len, part) : 1; }

// Split-form workspace: [scheduler counters, 256 B][partial results o, m, l],
// every section 256-byte aligned.
static size_t workspace_bytes_for(int num_seqs, int num_heads, int head_dim, int max_parts)
{
    const size_t rows = (size_t)num_seqs * num_heads * max_parts;
    return kSchedBytes + align256(rows * head_dim * sizeof(float)) + 2 * align256(rows * sizeof(float));
}

struct WsLayout {
    float *o, *m, *l;
};
static WsLayout ws_layout(void *ws, int num_seqs, int num_heads, int head_dim, int max_parts)
{
    const size_t rows = (size_t)num_seqs * num_heads * max_parts;
    char *w = static_cast<char *>(ws) + kSchedBytes;
    const size_t ob = align256(rows * head_dim * sizeof(float)), mb = align256(rows * sizeof(float));
    WsLayout L;
    L.o = reinterpret_cast<float *>(w);
    L.m = reinterpret_cast<float *>(w + ob);
    L.l = reinterpret_cast<float *>(w + ob + mb);
    return L;
}

// mode: 0 = one pass, 1 = split (direct singles + reduce), 2 = partitions only.
// A workspace (when given) supplies the scheduler counters for every mode and
// the partial results for modes 1 and 2.
static int run_decode(const DecodeArgs &a, int mode, int part, void *ws, size_t ws_bytes, cudaStream_t st)
{
    int rc = check_decode_args(a, mode != 2);
    if (rc != PA_OK) return rc;
    if (a.num_seqs == 0) return PA_OK;
    DecodeParams p = {};
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.query = static_cast<const __nv_bfloat16 *>(a.query);
    p.block_tables = a.block_tables;
    p.seq_lens = a.seq_lens;
    p.scale_log2 = a.scale * (a.fp8 ? a.k_scale : 1.f) * 1.4426950408889634f;
    p.v_scale = a.fp8 ? a.v_scale : 1.f;
    p.num_seqs = a.num_seqs;
    p.num_heads = a.num_heads;
    p.num_kv_heads = a.num_kv_heads;
    p.group = a.num_heads / a.num_kv_heads;
    p.max_blocks = a.max_blocks;
    if (ws && (!aligned16(ws) || ws_bytes < kSchedBytes)) return PA_ERR_WORKSPACE;
    p.sched = ws ? static_cast<int *>(ws) : nullptr;
    if (mode == 0) {
        p.part_tokens = 0;
        p.max_parts = 1;
        p.direct_single = 1;
    } else {
        if (part < kTileTokens || part % kTileTokens != 0) return PA_ERR_BAD_SHAPE;
        p.part_tokens = part;
        p.max_parts = max_parts_for(a.max_seq_len, part);
        p.direct_single = mode == 1 ? 1 : 0;
        const size_t need = workspace_bytes_for(a.num_seqs, a.num_heads, a.head_dim, p.max_parts);
        if (!ws || ws_bytes < need) return PA_ERR_WORKSPACE;
        const WsLayout L = ws_layout(ws, a.num_seqs, a.num_heads, a.head_dim, p.max_parts);
        p.ws_o = L.o;
        p.ws_m = L.m;
        p.ws_l = L.l;
        p.grp_start = a.grp_start;
        p.grp_parts = a.grp_parts;
        p.num_groups = a.num_groups;
    }
    const int64_t max_items = (int64_t)p.max_parts * a.num_seqs * a.num_kv_heads;
    if (max_items > INT_MAX) return PA_ERR_BAD_SHAPE;
    CUtensorMap tk, tv;
    const bool bb = decode_block_box(a.head_dim, a.block_size, a.fp8);
    rc = make_cache_map(&tk, a.key_cache, a.num_blocks, a.block_size, a.num_kv_heads, a.head_dim, a.fp8, bb);
    if (rc != PA_OK) return rc;
    rc = make_cache_map(&tv, a.value_cache, a.num_blocks, a.block_size, a.num_kv_heads, a.head_dim, a.fp8, bb);
    if (rc != PA_OK) return rc;
    if (a.fp8)
        rc = a.block_size == 8 ? launch_decode_fp8_bs<8>(p, tk, tv, max_items, st)
                               : launch_decode_fp8_bs<16>(p, tk, tv, max_items, st);
    else
        rc = a.head_dim == 64 ? launch_decode_d<64>(a.block_size, p, tk, tv, max_items, st)
                              : launch_decode_d<128>(a.block_size, p, tk, tv, max_items, st);
    if (rc != PA_OK || mode != 1) return rc;
    ReduceParams r = {};
    r.out = p.out;
    r.ws_o = p.ws_o;
    r.ws_m = p.ws_m;
    r.ws_l = p.ws_l;
    r.seq_lens = a.seq_lens;
    r.num_seqs = a.num_seqs;
    r.num_heads = a.num_heads;
    r.head_dim = a.head_dim;
    r.part_tokens = part;
    r.max_parts = p.max_parts;
    r.skip_single = 1;
    return launch_reduce(r, st);
}

// pa_decode's plan: 0 = one pass, else the partition size of the split form.
// Chosen from measurements on B200 (head_dim 128, bs 16, largest-first item
// order, items taken when their slot frees): one pass wins when no sequence is
// longer than 4096 and the (sequence, KV head) units alone give every SM
// several items -- GQA batch, max 4096: 99.4 us one pass vs 101.4 us at 1024
// and 100.3 us at 2048 (FP8 cache: 60.9 vs 66.0 and 63.2 us); MHA batch, max
// 2048: 182.2 vs 185.4 us -- as the one pass needs no partials and no reduce.
// (A batch whose sequences share 1024-token prompts runs faster split at 1024,
// 123.1 vs 134.2 us, because the shared parts are then read together; lengths
// alone do not show sharing.)  Otherwise 1024-token partitions up to 16K
// positions and 2048-token ones beyond (128K context: 412.8 us vs 430.3 us at
// 1024); partitions shrink until a small batch still yields several items per
// resident CTA.
static constexpr int kOnePassMaxLen = 4096;

static int choose_plan(int num_seqs, int num_kv_heads, int max_seq_len)
{
    const int64_t units = (int64_t)num_seqs * num_kv_heads;
    const int64_t target = 8LL * std::max(1, sm_count());  // ~4 items per resident CTA
    if (max_seq_len <= kOnePassMaxLen && units >= target / 2) return 0;
    int part = max_seq_len > 16384 ? 2048 : 1024;
    while (part > 64 && units * std::max<int64_t>(1, max_seq_len / (2 * part)) < target) part /= 2;
    return part;
}

template <int D, int BS>
static int launch_prefill_t(const PrefillParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, int64_t tiles, cudaStream_t st)
{
    auto kernel = paged_prefill_kernel<D, BS>;
    const size_t smem = (size_t)PfLayout<D>::kAlloc;
    int rc = ensure_smem(reinterpret_cast<const void *>(kernel), smem);
    if (rc != PA_OK) return rc;
    return launch_pdl(kernel, dim3((unsigned)tiles), dim3(kPfThreads), smem, st, p, tq, tk, tv);
}

template <int D>
static int launch_prefill_d(int bs, const PrefillParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, int64_t tiles, cudaStream_t st)
{
    switch (bs) {
    case 8: return launch_prefill_t<D, 8>(p, tq, tk, tv, tiles, st);
    case 16: return launch_prefill_t<D, 16>(p, tq, tk, tv, tiles, st);
    case 32: return launch_prefill_t<D, 32>(p, tq, tk, tv, tiles, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

// A wait that nothing satisfies, for testing the bounded-wait path: one
// thread waits on an mbarrier that no one arrives on; at the wait limit it
// records kTimeoutFullBarrier in the device status word and the kernel returns.
__global__ void bounded_wait_selftest_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbarrier_init();
    if (!mbar_wait_bounded(b, 0)) record_timeout(kTimeoutFullBarrier);
}

}  // namespace pakv

using namespace pakv;

extern "C" {

const char *pa_status_string(int status)
{
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_NULL_POINTER: return "null pointer";
    case PA_ERR_BAD_SHAPE: return "bad shape";
    case PA_ERR_UNSUPPORTED: return "unsupported head_dim / block_size / group";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_POOL_EXHAUSTED: return "block pool exhausted";
    case PA_ERR_BAD_BLOCK: return "bad block id";
    case PA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case PA_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case PA_ERR_VALUE_RANGE: return "an input value outside the range a kernel's arithmetic represents";
    case PA_ERR_NOT_DEVICE_ACCESSIBLE: return "memory not accessible from the device (pageable host memory?)";
    case PA_ERR_SCRATCH_TOO_SMALL:
        return "split workspace exceeds the built-in scratch of pa_decode_split_noalloc (use a larger "
               "partition_size, or pa_decode_split with a caller workspace)";
    default: return "unknown status";
    }
}

int pa_last_cuda_error(void) { return t_last_cuda_error; }

int pa_version(void) { return 10000; }

int pa_selftest_bounded_wait(void *stream)
{
    return launch_pdl(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream));
}

int pa_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables, int num_seqs, int max_blocks_per_seq,
                    const int32_t *seq_ids, const int64_t *positions, const int32_t *seq_lens, int num_tokens,
                    int block_size, void *stream)
{
    if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0) return PA_ERR_BAD_SHAPE;
    if (!seq_ids && num_tokens > num_seqs) return PA_ERR_BAD_SHAPE;
    if (num_tokens == 0) return PA_OK;
    if (!slot_mapping || !block_tables || (!positions && !seq_lens)) return PA_ERR_NULL_POINTER;
    const int threads = 256;
    return launch_pdl(slot_mapping_kernel, dim3((unsigned)cdiv64(num_tokens, threads)), dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), slot_mapping, block_tables, num_seqs, max_blocks_per_seq, seq_ids,
                      positions, seq_lens, num_tokens, block_size);
}

int pa_reshape_and_cache(const void *key, const void *value, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL_POINTER;
    if (((int64_t)num_kv_heads * head_dim) % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGNMENT;
    const int chunks = (int)((int64_t)num_kv_heads * head_dim / 8);
    const int64_t total = (int64_t)num_tokens * chunks;
    const int threads = 256;
    if (cdiv64(total, threads) > INT_MAX) return PA_ERR_BAD_SHAPE;
    return launch_pdl(reshape_and_cache_kernel, dim3((unsigned)cdiv64(total, threads)), dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), static_cast<const uint4 *>(key),
                      static_cast<const uint4 *>(value), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), slot_mapping, num_tokens, chunks,
                      (int64_t)num_blocks * block_size);
}

int pa_reshape_and_cache_fp8(const void *key, const void *value, void *key_cache, void *value_cache,
                             const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, float k_scale, float v_scale, void *stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (!(k_scale > 0.f && v_scale > 0.f && k_scale < INFINITY && v_scale < INFINITY)) return PA_ERR_BAD_SHAPE;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL_POINTER;
    if (((int64_t)num_kv_heads * head_dim) % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGNMENT;
    const int chunks = (int)((int64_t)num_kv_heads * head_dim / 16);
    const int64_t total = (int64_t)num_tokens * chunks;
    const int threads = 256;
    if (cdiv64(total, threads) > INT_MAX) return PA_ERR_BAD_SHAPE;
    // the inverse scales are rounded to fp32 once, here
    const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
    return launch_pdl(reshape_and_cache_fp8_kernel, dim3((unsigned)cdiv64(total, threads)), dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), static_cast<const uint4 *>(key),
                      static_cast<const uint4 *>(value), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), slot_mapping, num_tokens, chunks,
                      (int64_t)num_blocks * block_size, k_inv, v_inv);
}

static int append_kv(bool fp8, const void *key, const void *value, void *key_cache, void *value_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, int64_t *slot_mapping, int num_seqs,
                     int max_blocks_per_seq, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     float k_scale, float v_scale, void *stream)
{
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f && k_scale < INFINITY && v_scale < INFINITY))
        return PA_ERR_BAD_SHAPE;
    if (num_seqs == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !block_tables || !seq_lens) return PA_ERR_NULL_POINTER;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (row % (fp8 ? 16 : 8) != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGNMENT;
    const int chunks = (int)(row / (fp8 ? 16 : 8));
    const int64_t total = (int64_t)num_seqs * chunks;
    const int threads = 256;
    if (cdiv64(total, threads) > INT_MAX) return PA_ERR_BAD_SHAPE;
    const dim3 grid((unsigned)cdiv64(total, threads));
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t slots = (int64_t)num_blocks * block_size;
    if (fp8)
        return launch_pdl(append_kv_kernel<true>, grid, dim3(threads), 0, st, static_cast<const uint4 *>(key),
                          static_cast<const uint4 *>(value), static_cast<uint4 *>(key_cache),
                          static_cast<uint4 *>(value_cache), block_tables, seq_lens, slot_mapping, num_seqs,
                          max_blocks_per_seq, chunks, block_size, slots, 1.0f / k_scale, 1.0f / v_scale);
    return launch_pdl(append_kv_kernel<false>, grid, dim3(threads), 0, st, static_cast<const uint4 *>(key),
                      static_cast<const uint4 *>(value), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), block_tables, seq_lens, slot_mapping, num_seqs,
                      max_blocks_per_seq, chunks, block_size, slots, 1.f, 1.f);
}

int pa_append_decode_kv(const void *key, const void *value, void *key_cache, void *value_cache,
                        const int32_t *block_tables, const int32_t *seq_lens, int64_t *slot_mapping, int num_seqs,
                        int max_blocks_per_seq, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        void *stream)
{
    return append_kv(false, key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, num_seqs,
                     max_blocks_per_seq, num_kv_heads, head_dim, block_size, num_blocks, 1.f, 1.f, stream);
}

int pa_append_decode_kv_fp8(const void *key, const void *value, void *key_cache, void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens, int64_t *slot_mapping,
                            int num_seqs, int max_blocks_per_seq, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float k_scale, float v_scale, void *stream)
{
    return append_kv(true, key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, num_seqs,
                     max_blocks_per_seq, num_kv_heads, head_dim, block_size, num_blocks, k_scale, v_scale, stream);
}

int pa_append_decode_kv_cow(const void *key, const void *value, void *key_cache, void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cow_src,
                            int64_t *slot_mapping, int num_seqs, int max_blocks_per_seq, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks, void *stream)
{
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (num_seqs == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !block_tables || !seq_lens) return PA_ERR_NULL_POINTER;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (row % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_seqs > 65535) return PA_ERR_BAD_SHAPE;  // one grid row per sequence
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGNMENT;
    const int cpt = (int)(row / 8);
    // about 1024 chunks (16 KB) of each cache per CTA, whole rows
    const int rows_per_cta = std::max(1, std::min(block_size, 1024 / std::max(cpt, 1)));
    const dim3 grid((unsigned)((block_size + rows_per_cta - 1) / rows_per_cta), (unsigned)num_seqs);
    return launch_pdl(append_kv_cow_kernel, grid, dim3(256), 0, static_cast<cudaStream_t>(stream),
                      static_cast<const uint4 *>(key), static_cast<const uint4 *>(value),
                      static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), block_tables, seq_lens,
                      cow_src, slot_mapping, max_blocks_per_seq, cpt, block_size, rows_per_cta,
                      (int64_t)num_blocks);
}

int pa_copy_blocks(void *key_cache, void *value_cache, const int64_t *src_dst_pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, void *stream)
{
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !src_dst_pairs) return PA_ERR_NULL_POINTER;
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    if (block_elems % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_ALIGNMENT;
    const int64_t chunks = block_elems / 8;
    // 2048 chunks (32 KB) per CTA slice keeps ~16 KB of loads in flight per CTA.
    const int slices = (int)std::max<int64_t>(1, std::min<int64_t>(64, cdiv64(chunks, 2048)));
    if ((int64_t)num_pairs * slices > INT_MAX) return PA_ERR_BAD_SHAPE;
    return launch_pdl(copy_blocks_kernel, dim3((unsigned)(num_pairs * slices)), dim3(256), 0,
                      static_cast<cudaStream_t>(stream), static_cast<uint4 *>(key_cache),
                      static_cast<uint4 *>(value_cache), src_dst_pairs, chunks, slices, (int64_t)num_blocks);
}

// Device-accessible memory: device allocations, or host memory that is pinned
// and mapped into the device's address space (cudaHostAlloc / registered).
static bool device_accessible(const void *ptr)
{
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) return true;
    return attr.type == cudaMemoryTypeHost && attr.devicePointer == ptr;
}

int pa_swap_blocks(void *dst_key_cache, void *dst_value_cache, const void *src_key_cache,
                   const void *src_value_cache, const int64_t *src_dst_pairs, int num_pairs, int num_kv_heads,
                   int head_dim, int block_size, int src_num_blocks, int dst_num_blocks, void *stream)
{
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || src_num_blocks <= 0 ||
        dst_num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (num_pairs == 0) return PA_OK;
    if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || !src_dst_pairs)
        return PA_ERR_NULL_POINTER;
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    if (block_elems % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(dst_key_cache) || !aligned16(dst_value_cache) || !aligned16(src_key_cache) ||
        !aligned16(src_value_cache))
        return PA_ERR_ALIGNMENT;
    if (!device_accessible(dst_key_cache) || !device_accessible(dst_value_cache) ||
        !device_accessible(src_key_cache) || !device_accessible(src_value_cache) ||
        !device_accessible(src_dst_pairs))
        return PA_ERR_NOT_DEVICE_ACCESSIBLE;
    const int64_t chunks = block_elems / 8;
    const int slices = (int)std::max<int64_t>(1, std::min<int64_t>(64, cdiv64(chunks, 2048)));
    if ((int64_t)num_pairs * slices > INT_MAX) return PA_ERR_BAD_SHAPE;
    return launch_pdl(swap_blocks_kernel, dim3((unsigned)(num_pairs * slices)), dim3(256), 0,
                      static_cast<cudaStream_t>(stream), static_cast<uint4 *>(dst_key_cache),
                      static_cast<uint4 *>(dst_value_cache), static_cast<const uint4 *>(src_key_cache),
                      static_cast<const uint4 *>(src_value_cache), src_dst_pairs, chunks, slices,
                      (int64_t)src_num_blocks, (int64_t)dst_num_blocks);
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_seq_len,
                                int partition_size)
{
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_seq_len < 0) return 0;
    const int part = partition_size > 0 ? partition_size : choose_plan(num_seqs, num_kv_heads, max_seq_len);
    if (part == 0) return kSchedBytes;  // one pass: the scheduler counters only
    return workspace_bytes_for(num_seqs, num_heads, head_dim, max_parts_for(max_seq_len, part));
}

int pa_decode_plan(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int max_seq_len,
                   size_t workspace_bytes)
{
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_seq_len < 0) return 0;
    const int part = choose_plan(num_seqs, num_kv_heads, max_seq_len);
    if (part == 0) return 0;
    const size_t need = workspace_bytes_for(num_seqs, num_heads, head_dim, max_parts_for(max_seq_len, part));
    return workspace_bytes >= need ? part : 0;
}

int pa_decode(void *out, const void *query, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size, int num_kv_heads,
              int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq, int num_blocks, int max_seq_len,
              void *workspace, size_t workspace_bytes, void *stream)
{
    const DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                          num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int part = workspace ? pa_decode_plan(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len,
                                                workspace_bytes)
                               : 0;
    if (part > 0) return run_decode(a, 1, part, workspace, workspace_bytes, st);
    const bool counters = workspace && workspace_bytes >= kSchedBytes;
    return run_decode(a, 0, 0, counters ? workspace : nullptr, counters ? workspace_bytes : 0, st);
}

int pa_decode_one_pass(void *out, const void *query, const void *key_cache, const void *value_cache,
                       const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                       int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                       int num_blocks, int max_seq_len, void *stream)
{
    const DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                          num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    return run_decode(a, 0, 0, nullptr, 0, static_cast<cudaStream_t>(stream));
}

int pa_decode_split(void *out, const void *query, const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                    int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                    int num_blocks, int max_seq_len, int partition_size, void *workspace, size_t workspace_bytes,
                    void *stream)
{
    const DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                          num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    return run_decode(a, 1, partition_size, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pa_decode_shared(void *out, const void *query, const void *key_cache, const void *value_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                     int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                     int num_blocks, int max_seq_len, int partition_size, const int32_t *group_start,
                     const int32_t *group_parts, int num_groups, void *workspace, size_t workspace_bytes,
                     void *stream)
{
    DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                    num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    if (num_groups < 0 || num_groups > num_seqs) return PA_ERR_BAD_SHAPE;
    if (num_groups > 0 && (!group_start || !group_parts)) return PA_ERR_NULL_POINTER;
    a.grp_start = group_start;
    a.grp_parts = group_parts;
    a.num_groups = num_groups;
    return run_decode(a, 1, partition_size, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pa_decode_fp8(void *out, const void *query, const void *key_cache, const void *value_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, float scale, float k_scale, float v_scale,
                  int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                  int max_blocks_per_seq, int num_blocks, int max_seq_len, void *workspace, size_t workspace_bytes,
                  void *stream)
{
    DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                    num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    a.fp8 = true;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int part = workspace ? pa_decode_plan(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len,
                                                workspace_bytes)
                               : 0;
    if (part > 0) return run_decode(a, 1, part, workspace, workspace_bytes, st);
    const bool counters = workspace && workspace_bytes >= kSchedBytes;
    return run_decode(a, 0, 0, counters ? workspace : nullptr, counters ? workspace_bytes : 0, st);
}

int pa_decode_fp8_split(void *out, const void *query, const void *key_cache, const void *value_cache,
                        const int32_t *block_tables, const int32_t *seq_lens, float scale, float k_scale,
                        float v_scale, int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                        int max_blocks_per_seq, int num_blocks, int max_seq_len, int partition_size,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                    num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    a.fp8 = true;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (partition_size == 0) return run_decode(a, 0, 0, workspace, workspace ? workspace_bytes : 0, st);
    return run_decode(a, 1, partition_size, workspace, workspace_bytes, st);
}

int pa_prefill(void *out, const void *query, const void *key_cache, const void *value_cache,
               const int32_t *block_tables, const int32_t *seq_lens, const int32_t *q_start, float scale,
               int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
               int num_blocks, int num_tokens, void *stream)
{
    if (num_seqs < 0 || num_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
        return PA_ERR_BAD_SHAPE;
    if (num_heads % num_kv_heads != 0) return PA_ERR_BAD_SHAPE;
    // the softmax takes the row max of the unscaled logits: only a finite,
    // positive scale keeps that max the max of the scaled ones
    if (!(scale > 0.f && scale < INFINITY)) return PA_ERR_BAD_SHAPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != 8 && block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
    const int G = num_heads / num_kv_heads;
    if (G > 16) return PA_ERR_UNSUPPORTED;
    if ((int64_t)num_blocks * block_size > INT_MAX || (int64_t)max_blocks_per_seq * block_size > INT_MAX)
        return PA_ERR_BAD_SHAPE;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !q_start)
        return PA_ERR_NULL_POINTER;
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGNMENT;
    PrefillParams p = {};
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.q_start = q_start;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = G;
    p.max_blocks = max_blocks_per_seq;
    p.tq = kPfRows / G;
    p.q_box = std::min(p.tq, num_tokens);
    // persistent: one CTA per SM (shared memory and TMEM hold one), at most one
    // per work item; the items are (pair of query tiles, KV head), at most
    // (T / (2 tq) + B) * num_kv_heads of them
    const int64_t items = ((int64_t)num_tokens / (2 * p.tq) + num_seqs + 1) * num_kv_heads;
    const int64_t tiles = std::min<int64_t>(items, std::max(1, sm_count()));
    CUtensorMap tq, tk, tv;
    int rc = make_query_map(&tq, query, num_tokens, num_heads, head_dim, G, p.q_box);
    if (rc != PA_OK) return rc;
    rc = make_cache_map(&tk, key_cache, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc != PA_OK) return rc;
    rc = make_cache_map(&tv, value_cache, num_blocks, block_size, num_kv_heads, head_dim);
    if (rc != PA_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    return head_dim == 64 ? launch_prefill_d<64>(block_size, p, tq, tk, tv, tiles, st)
                          : launch_prefill_d<128>(block_size, p, tq, tk, tv, tiles, st);
}

// Scratch of pa_decode_split_noalloc: one fixed array per device, part of the
// library image, so that the call needs no allocation by anyone.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  The address is
// looked up once per context (with the context's device current) and cached
// under the context's process-unique id: after a device reset the runtime
// loads the library's module again in a new primary context, where the array
// may sit elsewhere, and a new id makes the next call look it up again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

static int current_context_id(unsigned long long *id)
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<CtxGetCurrentFn>(a);
            get_id = reinterpret_cast<CtxGetIdFn>(b);
        }
    });
    if (!get_current || !get_id) return check_cuda(cudaErrorNotSupported);
    CUcontext ctx = nullptr;
    *id = 0;  // 0: no context is current yet
    if (get_current(&ctx) != CUDA_SUCCESS) return check_cuda(cudaErrorDeviceUninitialized);
    if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return check_cuda(cudaErrorDeviceUninitialized);
    return PA_OK;
}

static int noalloc_scratch(void **ptr)
{
    static std::mutex mu;
    static unsigned long long ctx_of[64] = {};
    static void *addr[64] = {};
    int dev = 0;
    int rc = check_cuda(cudaGetDevice(&dev));
    if (rc != PA_OK) return rc;
    if (dev < 0 || dev >= 64) return check_cuda(cudaErrorInvalidDevice);
    unsigned long long ctx = 0;
    rc = current_context_id(&ctx);
    if (rc != PA_OK) return rc;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx == 0 || ctx_of[dev] != ctx) {
        // the lookup makes the device's primary context current if none was
        void *p = nullptr;
        rc = check_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        if (rc != PA_OK) return rc;
        rc = current_context_id(&ctx);
        if (rc != PA_OK) return rc;
        if (ctx == 0) return check_cuda(cudaErrorDeviceUninitialized);
        addr[dev] = p;
        ctx_of[dev] = ctx;
    }
    *ptr = addr[dev];
    return PA_OK;
}

int pa_decode_split_noalloc(void *out, const void *query, const void *key_cache, const void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                            int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                            int num_blocks, int max_seq_len, int partition_size, void *stream)
{
    const DecodeArgs a = {out, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                          num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    int rc = check_decode_args(a, true);
    if (rc != PA_OK) return rc;
    if (partition_size < kTileTokens || partition_size % kTileTokens != 0) return PA_ERR_BAD_SHAPE;
    if (num_seqs == 0) return PA_OK;
    const size_t need =
        workspace_bytes_for(num_seqs, num_heads, head_dim, max_parts_for(max_seq_len, partition_size));
    if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_SCRATCH_TOO_SMALL;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != PA_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the scheduler counters must start at zero; the array keeps whatever the last call left
    rc = check_cuda(cudaMemsetAsync(scratch, 0, kSchedBytes, st));
    if (rc != PA_OK) return rc;
    return run_decode(a, 1, partition_size, scratch, PA_NOALLOC_SCRATCH_BYTES, st);
}

int pa_decode_partitions(const void *query, const void *key_cache, const void *value_cache,
                         const int32_t *block_tables, const int32_t *seq_lens, float scale, int block_size,
                         int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                         int num_blocks, int max_seq_len, int partition_size, void *workspace,
                         size_t workspace_bytes, void *stream)
{
    const DecodeArgs a = {nullptr, query, key_cache, value_cache, block_tables, seq_lens, scale, block_size,
                          num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len};
    return run_decode(a, 2, partition_size, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int pa_lse_reduce(void *out, const void *workspace, const int32_t *seq_lens, int num_seqs, int num_heads,
                  int head_dim, int max_seq_len, int partition_size, void *stream)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_seq_len < 0) return PA_ERR_BAD_SHAPE;
    if (partition_size < kTileTokens || partition_size % kTileTokens != 0) return PA_ERR_BAD_SHAPE;
    if (num_seqs == 0) return PA_OK;
    if (!out || !workspace || !seq_lens) return PA_ERR_NULL_POINTER;
    const int max_parts = max_parts_for(max_seq_len, partition_size);
    const WsLayout L = ws_layout(const_cast<void *>(workspace), num_seqs, num_heads, head_dim, max_parts);
    ReduceParams r = {};
    r.out = static_cast<__nv_bfloat16 *>(out);
    r.ws_o = L.o;
    r.ws_m = L.m;
    r.ws_l = L.l;
    r.seq_lens = seq_lens;
    r.num_seqs = num_seqs;
    r.num_heads = num_heads;
    r.head_dim = head_dim;
    r.part_tokens = partition_size;
    r.max_parts = max_parts;
    r.skip_single = 0;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!aligned16(workspace) || !aligned16(out)) return PA_ERR_ALIGNMENT;
    return launch_reduce(r, static_cast<cudaStream_t>(stream));
}

int pa_validate_tables(const int32_t *block_tables, const int32_t *seq_lens, int num_seqs, int max_blocks_per_seq,
                       int block_size, int num_blocks, int max_seq_len, int32_t *bad_count, void *stream)
{
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0) return PA_ERR_BAD_SHAPE;
    if (!bad_count || (num_seqs > 0 && (!block_tables || !seq_lens))) return PA_ERR_NULL_POINTER;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = check_cuda(cudaMemsetAsync(bad_count, 0, sizeof(int32_t), st));
    if (rc != PA_OK || num_seqs == 0) return rc;
    return launch_pdl(validate_tables_kernel, dim3((unsigned)num_seqs), dim3(128), 0, st, block_tables, seq_lens,
                      num_seqs, max_blocks_per_seq, block_size, num_blocks, max_seq_len, bad_count);
}

int pa_device_status(void)
{
    int rc = check_cuda(cudaDeviceSynchronize());
    if (rc != PA_OK) return rc;
    int v = 0;
    rc = check_cuda(cudaMemcpyFromSymbol(&v, g_pa_device_status, sizeof(int)));
    if (rc != PA_OK) return rc;
    if (v != 0) {
        const int zero = 0;
        rc = check_cuda(cudaMemcpyToSymbol(g_pa_device_status, &zero, sizeof(int)));
        if (rc != PA_OK) return rc;
        return v == pakv::kStatusValueRange ? PA_ERR_VALUE_RANGE : PA_ERR_DEVICE_TIMEOUT;
    }
    return PA_OK;
}

}  // extern "C"
