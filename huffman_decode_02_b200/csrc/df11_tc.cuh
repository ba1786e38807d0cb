// df11_tc.cuh -- tensor-core and TMA building blocks for sm_100a shared by
// the consumer GEMM (df11_gemm.cu) and the fused decode -> GEMM kernel
// (df11_decode.cu): UMMA shared-memory and instruction descriptors,
// tcgen05.mma / commit, 2-D TMA tile loads (no multicast) and bounded
// mbarrier waits.  Private to libdf11.
//
// Layout these helpers assume: K-major BF16 tiles whose rows are 64 elements
// (128 bytes) long, stored with the 128-byte swizzle -- the 16-byte piece j of
// row r sits at piece position (j XOR (r mod 8)) of the row, and the tile
// starts on a 1024-byte boundary, so 8-row groups are 1024 bytes apart.  A
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes exactly this layout, and the
// fused kernel's decoder writes it with plain shared-memory stores.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace df11 {
namespace tc {

constexpr uint32_t kSpin = 1u << 24;  // bounded waits: iterations of try_wait

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Bounded wait for the phase with the given parity of an mbarrier; false if
// it did not complete within the iteration limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t spin = kSpin) {
    uint32_t done = 0;
    for (uint32_t it = 0; it < spin && !done; ++it) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
    }
    return done != 0;
}

// One probe of the phase with the given parity that may suspend the thread
// for up to `hint_ns` nanoseconds while the phase is incomplete (the thread
// resumes when it completes): a waiter that does not spin.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One arrival plus `bytes` more expected transaction bytes for this phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// `bytes` of expected transactions done (the writer's own shared-memory
// stores, made visible to the async proxy first with fence.proxy.async).
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle
// layout above (start address, stride of 8-row groups = 1024 bytes).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);  // start address
    d |= (uint64_t)1u << 16;                 // leading byte offset (unused with swizzle)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                 // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                 // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: BF16 x BF16 -> FP32, both operands K-major.
__device__ __forceinline__ uint32_t instr_desc_bf16(uint32_t n, uint32_t m) {
    return (1u << 4)            // D format F32
           | (1u << 7)          // A format BF16
           | (1u << 10)         // B format BF16
           | ((n >> 3) << 17)   // N / 8
           | ((m >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives on the mbarrier once every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 16 consecutive FP32 accumulator columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t v[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Host: a 2-D TMA map over a row-major [rows, cols] BF16 matrix with box
// [box_rows, 64] and the 128-byte swizzle (rows past the end read as zero).
// Defined in df11_gemm.cu; false if the driver's encoder is unavailable or
// refuses the map (e.g. a misaligned pointer or stride).
bool make_bf16_tile_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

}  // namespace tc
}  // namespace df11
