// tc05.cuh -- fifth-generation tensor-core (tcgen05) building blocks for sm_100a:
// tensor-memory allocation, shared-memory matrix descriptors, the instruction
// descriptor of a bf16 MMA with fp32 accumulation, MMA issue and completion
// tracking, and tensor-memory loads/stores.  All inline PTX; single CTA
// (cta_group::1) forms only.
#pragma once

#include "common.cuh"

namespace pakv {

// ---- tensor memory (TMEM) ------------------------------------------------------
// Allocation is warp-collective: the whole warp executes it; the base address
// (lane 0, first column) is written to the shared word at `dst_smem`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Ordering of tcgen05 operations against thread synchronisation (barriers,
// mbarriers): `before` ahead of the signal, `after` behind the wait.
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- shared-memory matrix descriptors --------------------------------------------
// 64-bit descriptor: start address >> 4 in bits [0,14), leading-dimension byte
// offset >> 4 in [16,30), stride-dimension byte offset >> 4 in [32,46), the
// value 1 in [46,48), base offset 0 in [49,52), layout type in [61,64)
// (2 = 128-byte swizzle).  Operand tiles are stored as 1024-byte aligned
// swizzle atoms of 8 rows x 128 bytes, the 16-byte chunk index of row r XORed
// with r % 8 -- the layout TMA writes with 128-byte swizzling.
constexpr uint64_t kDescSw128 = 2ull << 61;
constexpr uint64_t kDescVersion = 1ull << 46;

// K-major operand (rows = M or N, 64 contiguous K elements per 128-byte row):
// 8-row groups 1024 bytes apart (stride byte offset); the leading byte offset
// is unused by swizzled K-major layouts and set to 16 bytes.  A K step of 16
// bf16 elements inside the atom advances the start address by 32 bytes.
__host__ __device__ constexpr uint64_t desc_kmajor_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | kDescVersion |
           kDescSw128;
}

// MN-major operand (rows = K, 64 contiguous MN elements per 128-byte row):
// atoms of 8 K-rows 1024 bytes apart along K (stride byte offset), atoms along
// MN `lbo` bytes apart (leading byte offset).
__host__ __device__ constexpr uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t lbo)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | kDescVersion | kDescSw128;
}

// The two words of those descriptors apart: the high word (stride byte offset,
// version, swizzle mode) is the same for every operand here, and the low word
// (start address, leading byte offset) of an address plus a multiple of 16
// bytes is the low word of the address plus that multiple / 16 (shared-memory
// addresses stay below 2^18).  An MMA loop then derives each k-step's
// descriptor with one add instead of rebuilding it.
constexpr uint32_t kDescHiSw128 = (uint32_t)((((uint64_t)(1024 >> 4) << 32) | kDescVersion | kDescSw128) >> 32);
__host__ __device__ constexpr uint32_t desc_lo_sw128(uint32_t saddr, uint32_t lbo)
{
    return ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
}

static_assert(desc_kmajor_sw128(0x1C400u) == (((uint64_t)kDescHiSw128 << 32) | desc_lo_sw128(0x1C400u, 16)) &&
                  desc_kmajor_sw128(0x1C400u + 96) == (((uint64_t)kDescHiSw128 << 32) | (desc_lo_sw128(0x1C400u, 16) + 6)) &&
                  desc_mnmajor_sw128(0x30000u + 3 * 2048, 8192) ==
                      (((uint64_t)kDescHiSw128 << 32) | (desc_lo_sw128(0x30000u, 8192) + 3 * 128)),
              "split descriptor words");

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 D, dense:
// D format (1 = f32) in bits [4,6), A format (1 = bf16) in [7,10), B format in
// [10,13), A major in bit 15, B major in bit 16 (0 = K-major, 1 = MN-major),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n, bool a_mn_major, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// The same for fp16 A and B (kind::f16, a_format = b_format = 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n, bool a_mn_major, bool b_mn_major)
{
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], issued by one thread, both descriptors given
// by their low words over kDescHiSw128.
__device__ __forceinline__ void tc_mma_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                          bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.u32 p, %4, 0;\n\t"
        "mov.b64 da, {%1, %5};\n\t"
        "mov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"((uint32_t)accumulate), "r"(kDescHiSw128)
        : "memory");
}

// The mbarrier at `bar` receives one arrive when every tcgen05 operation this
// thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// ---- TMEM <-> registers ------------------------------------------------------------
// Warp w of a warpgroup reaches TMEM lanes 32(w % 4) .. 32(w % 4) + 31; lane i
// of the warp reads / writes its TMEM lane, 32 consecutive 32-bit columns.
// The load and its wait are one asm statement, so no use of the registers can
// be scheduled ahead of the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x 16, K-major) read from TMEM -- lane =
// row, two 16-bit K elements per 32-bit column, the lower K index in the low
// half; B's descriptor given by its low word over kDescHiSw128; issued by one
// thread.
__device__ __forceinline__ void tc_mma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc,
                                             bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "setp.ne.u32 p, %4, 0;\n\t"
        "mov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"((uint32_t)accumulate), "r"(kDescHiSw128)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace pakv
