// df11_decode.cu -- the DF11 decode kernel for sm_100a and its launchers
// (df11_decode, df11_decode_block), and the row-gather kernel that decodes
// only the thread blocks covering requested rows (df11_decode_rows).
//
// Sources: "DFloat11 : compression sans perte pour l'inference GPU qui reduit
// les LLM a 70 % de leur taille" (fr.news.hada.io):
//  << Noyau GPU en deux etapes et metadonnees auxiliaires >> -- each thread
//     owns n = 8 bytes of EncodedExponent and decodes the codes that start
//     there; Gaps gives its first code's bit offset; only the output index
//     of each thread block's first element is stored; a first pass counts,
//     a block prefix sum gives each thread its write position, a second
//     pass writes the exponents into an on-chip buffer, and the block's
//     output is written to HBM in one coalesced sweep.
//  << Decodage fonde sur des LUT hierarchiques >> -- lookup tables resident
//     in on-chip memory instead of a bit-by-bit tree walk.
//  << Decompression par bloc transformer >> -- all matrices of a block are
//     decoded in one launch.
//
// B200 design (what differs from the pages' own kernel):
//  * Persistent CTAs, one per SM (1024 threads = 8 groups of 128).  Each
//    group decodes one format block (256 format threads x 8 bytes) at a
//    time and strides over the blocks.  The compact decode tables arrive by
//    one TMA bulk copy (cp.async.bulk, no multicast); the count table is
//    kept in two interleaved copies (lane l reads copy l mod 2), the symbol
//    table in two or one (per instance).
//  * Per group, bulk copies on mbarriers bring the next block's inputs
//    (stream bytes, gaps, block starts) and the current block's whole
//    sign/mantissa range into shared memory, so the merge reads nothing
//    from global memory and no register holds prefetched data across the
//    decode loops.
//  * The exponent buffer holds 7152 symbols per group when every block of
//    the tensor fits (LLM-like weights: the room left gives the symbol table
//    its second copy), else 8192; tensors whose blocks hold more codes
//    (average code under 2 bits) use an instance with 4 groups of 16 KB
//    buffers.
//  * Every CUDA thread runs two format threads side by side (two
//    independent decode chains in one loop): each lookup is a dependent
//    shift -> index -> shared load chain, and two chains per thread hide
//    its latency twice over.
//  * Each chain holds its 8 bytes plus the next chain's first 4 bytes in a
//    96-bit shift register (three funnel shifts per step).  Bits at and
//    after the thread's last code end (known exactly from the next thread's
//    gap) are set to 1: a run of ones shorter than the longest code is never
//    a whole code of a canonical code, so a table lookup can never take a
//    code that belongs to the next thread.
//  * Pass 1 counts with a 12-bit count table (several codes per lookup);
//    one add per lookup updates both the code count and the bits taken,
//    and the entry's low bits are the shift amount.
//  * Pass 2 decodes with a 12-bit table of up to four symbols per entry and
//    stops on the code count pass 1 found; the symbol bytes are OR-ed into
//    the clear buffer (a word is touched only when it receives a symbol).
//    Codes longer than the window fall back to canonical limits.
//  * Warp shuffle scan + one cross-warp step (named barrier per group).
//    Two group barriers per block: the merge clears the buffer chunks it
//    reads, so the next block needs no barrier of its own before decoding.
//  * Exponents are kept rotated by one bit, so the merge with the
//    sign/mantissa bytes is two bit-selects and two byte-permutes per four
//    weights; stores are 32 bytes per thread (whole sectors per warp).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "df11.h"
#include "df11_internal.h"
#include "df11_tc.cuh"

namespace {

using namespace df11;

// Shared memory layout of one CTA:
//   [0, 768)                 table header, canonical limits, symbol list
//   kOffCountRep             count table, kCountCopies copies interleaved:
//                            entry i of copy c at word (i * kCountCopies + c)
//   kOffSymRep               symbol table, C::kSymCopies copies interleaved:
//                            entry i of copy c at u64 (i * copies + c)
//   kOffGroups               per group: exponent buffer, warp totals, staged
//                            inputs of the next block, this block's
//                            sign/mantissa bytes, 2 mbarriers
//   table mbarrier
// Lane l reads copy (l mod copies).  Random lookups still meet bank
// conflicts (a warp's lookup costs several wavefronts); more copies cut
// them little and take the room the staged sign/mantissa bytes need.
#ifndef DF11_COUNT_COPIES
#define DF11_COUNT_COPIES 2
#endif
constexpr uint32_t kCountCopies = DF11_COUNT_COPIES;
constexpr uint32_t log2u(uint32_t x) { return x <= 1u ? 0u : 1u + log2u(x >> 1); }
constexpr uint32_t kCountShift = log2u(4u * kCountCopies);  // byte stride of one replicated entry
static_assert((1u << kCountShift) == 4u * kCountCopies, "power of two");
constexpr uint32_t kOffCountRep = 768;
constexpr uint32_t kEncStage = kThreadsPerBlockFmt * kBytesPerThread + 16u;  // + next block's first 16
constexpr uint32_t kGapStage = kThreadsPerBlockFmt * 5u / 8u + 16u;          // + next block's first gaps
constexpr uint32_t kFull = 0xFFFFFFFFu;
#ifndef DF11_LOOP_CAP
#define DF11_LOOP_CAP 128
#endif
constexpr uint32_t kLoopCap = DF11_LOOP_CAP;  // lookups per decode loop (95 suffice)
constexpr uint32_t kKernErrTimeout = 0x10u;  // an asynchronous copy did not complete in time
static_assert(kGroupThreads == 128, "group scan assumes four warps");

// Debug builds (DF11_DEBUG_CHECKS, libdf11_debug.so) check every
// data-dependent shared-memory index and global store address against its
// array before the access; a failed check skips the access and is counted in
// a device word the host reads back.  In the product build the checks are
// the constant `true` and generate no code.
#ifdef DF11_DEBUG_CHECKS
__device__ uint32_t g_df11_bounds_errors;
#define DF11_BOUNDS_OK(cond) ((cond) || (atomicAdd(&g_df11_bounds_errors, 1u), false))
#else
#define DF11_BOUNDS_OK(cond) true
#endif
static_assert(kLutBytes % 16 == 0, "bulk copy size");

// Per-instance layout: G groups per CTA, buffers of S symbols (+ 16: the
// 16-element chunk alignment of the block start is at most 15), SC copies of
// the symbol table.  CT: the instance runs the count pass and keeps the count
// table (tensors without stored per-thread counts); without it, the counts
// come from the tensor's `counts` array, staged per block, and the 32 KB of
// the count table are free for buffers and table copies.
template <int G, int S, int SC, bool CT = true, bool SMS = true>
struct Cfg {
    static constexpr bool kCountTable = CT;
    static constexpr bool kStageSm = SMS;  // the block's sign/mantissa bytes are staged in shared memory
    static constexpr uint32_t kSymCopies = SC;  // symbol-table copies (lane l reads copy l mod SC)
    static constexpr uint32_t kOffSymRep = CT ? kOffCountRep + 4u * kCountCopies * (1u << kW1Max) : kOffCountRep;
    static constexpr uint32_t kOffGroups = kOffSymRep + 8u * SC * (1u << kW2Max);
    static constexpr uint32_t kGroups = G;
    static constexpr uint32_t kBufSyms = S;
    static constexpr uint32_t kCtaThreads = G * kGroupThreads;
    static constexpr uint32_t kSbufBytes = S + 16u;  // + the word after the last one
    static constexpr uint32_t kGrpWtot = kSbufBytes;
    static constexpr uint32_t kGrpEnc = kGrpWtot + 16u;
    static constexpr uint32_t kGrpGap = kGrpEnc + kEncStage;
    static constexpr uint32_t kGrpBs = kGrpGap + kGapStage;
    static constexpr uint32_t kGrpCnt = kGrpBs + 32u;  // the block's stored counts (instances without CT)
    static constexpr uint32_t kCntStage = CT ? 0u : (uint32_t)kThreadsPerBlockFmt;
    static constexpr uint32_t kGrpSm = kGrpCnt + kCntStage;  // the block's sign/mantissa bytes
    static constexpr uint32_t kSmBytes = SMS ? S + 16u : 0u;
    static constexpr uint32_t kGrpMbar = kGrpSm + kSmBytes;
    static constexpr uint32_t kGrpAux = kGrpMbar + 16u;  // row gather: the row's block range
    static constexpr uint32_t kGroupBytes = kGrpAux + 16u;
    static constexpr uint32_t kSmemBytes = kOffGroups + G * kGroupBytes + 16u;
    static_assert(S % 16 == 0, "whole chunks");
    static_assert(((S + 19u) >> 4) * 16u <= kSbufBytes, "zeroing stays inside the buffer");
    static_assert(SC >= 1 && SC <= 4, "one to four symbol-table copies");
    static_assert(kGroupBytes % 16 == 0 && kGrpEnc % 16 == 0 && kGrpGap % 16 == 0 && kGrpBs % 16 == 0 &&
                      kGrpCnt % 16 == 0 && kGrpSm % 16 == 0,
                  "bulk copy destinations are 16-byte aligned");
    // where the staged symbol LUT lands (right after the header when the count
    // LUT is not staged) and how many bytes the staging takes
    static constexpr uint32_t kStageSym = CT ? kOffSymLut : kOffCountLut;
    static constexpr uint32_t kStageBytes = kStageSym + (kLutBytes - kOffSymLut);
    static_assert(kStageBytes <= G * kGroupBytes, "tables stage in the group area");
    static_assert(kSmemBytes <= 227u * 1024u, "fits one CTA's shared memory");
};
// (SMS = false: the merge reads the sign/mantissa bytes from global memory;
// only the fused decode -> GEMM kernel, which needs the room for its operand
// tiles, does so)
// (S = 7152 is the largest buffer with which 8 groups and two symbol-table
// copies fit beside the count table: 232,336 of the 232,448 bytes a CTA may
// use)
using CfgTypical = Cfg<8, 7152, 2>;  // blocks of up to 7152 - 15 codes: two symbol-table copies fit
using CfgWide = Cfg<8, 8192, 1>;     // blocks of up to 8192 - 15 codes (any LLM-like data)
using CfgDense = Cfg<4, 16400, 1>;   // any block (1-bit codes: 16384 per block)
// Stored counts (no count pass, no count table).
#ifndef DF11_TYPICAL_C_SYMS
#define DF11_TYPICAL_C_SYMS 7152
#endif
#ifndef DF11_TYPICAL_C_COPIES
#define DF11_TYPICAL_C_COPIES 2
#endif
using CfgTypicalC = Cfg<8, DF11_TYPICAL_C_SYMS, DF11_TYPICAL_C_COPIES, false>;
using CfgWideC = Cfg<8, 8192, 2, false>;
using CfgDenseC = Cfg<4, 16400, 2, false>;
// The fused decode -> GEMM kernel's decoder: stored counts, one symbol-table
// copy, 6 or 4 groups (the rest of the shared memory holds the operand tiles;
// the largest X tiles leave no room to stage the sign/mantissa bytes).
using CfgFused6 = Cfg<6, 7152, 1, false>;          // T <= 64
using CfgFused4 = Cfg<4, 7152, 1, false>;          // T <= 128
using CfgFused4U = Cfg<4, 7152, 1, false, false>;  // T <= 256: no sign/mantissa staging
using CfgFused6U = Cfg<6, 7152, 1, false, false>;

struct DecodeArgs {
    const uint8_t *enc;
    const uint8_t *counts;  // per-thread code counts (instances without the count pass)
    const uint8_t *sm;
    const uint8_t *gaps;
    const uint32_t *bstart;
    const uint8_t *lut;
    uint16_t *out;
    uint32_t *err;
    uint64_t n_elems;
    uint64_t total_bits;
    uint64_t n_threads;
    uint64_t n_blocks;
    uint32_t out_al32;  // out is 32-byte aligned: whole-chunk stores are 32 bytes
};

// ----------------------------------------------------------------- PTX
// 32-byte store (sm_100): one warp instruction writes 1 KB of whole sectors.
__device__ __forceinline__ void st_u8x32(void *p, const uint32_t o[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                 "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                 : "memory");
}
__device__ __forceinline__ void st_u4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
// Shared memory through 32-bit shared-window addresses.  Volatile keeps them
// ordered with the barriers (also volatile asm).
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint64_t lds_u64(uint32_t a) {
    uint64_t v;
    asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ void sts_zero16(uint32_t a) { sts_u4(a, 0u, 0u, 0u, 0u); }
__device__ __forceinline__ void red_or(uint32_t a, uint32_t v) {
    asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void group_barrier(uint32_t group) {
    asm volatile("bar.sync %0, %1;" ::"r"(group + 1u), "r"((uint32_t)kGroupThreads) : "memory");
}
__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0u, 0x0123u); }
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Bounded wait for the given phase of an mbarrier.  Returns false if the
// phase did not complete within the iteration limit.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t phase) {
    uint32_t done = 0;
    for (uint32_t it = 0; it < (1u << 22) && !done; ++it) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(phase)
            : "memory");
    }
    return done != 0;
}
__device__ __forceinline__ void mbar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// One-dimensional bulk copy global -> shared (TMA engine), completion counted
// on the mbarrier.  Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, a multiple of
// 16 bytes); no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Length of a code longer than the table window, from the canonical limits
// in shared memory (non-decreasing in l): the smallest l in [from, max_len]
// with window < lim[l], by binary search.  0 if none.
__device__ __forceinline__ uint32_t long_code_length(uint32_t x, uint32_t lim_addr, uint32_t from, uint32_t max_len) {
    if (from > max_len || (uint64_t)x >= lds_u64(lim_addr + 8u * max_len)) return 0u;
    uint32_t lo = from, hi = max_len;  // answer in [lo, hi]
    while (lo < hi) {
        const uint32_t mid = (lo + hi) >> 1;
        if ((uint64_t)x < lds_u64(lim_addr + 8u * mid)) hi = mid;
        else lo = mid + 1u;
    }
    return lo;
}

// Shifts a 96-bit window left by n bits (n <= 32), filling with ones.
__device__ __forceinline__ void shift_window_clamped(uint32_t &hi, uint32_t &lo, uint32_t &fl, uint32_t n) {
    hi = __funnelshift_lc(lo, hi, n);
    lo = __funnelshift_lc(fl, lo, n);
    fl = __funnelshift_lc(kFull, fl, n);
}

// Merges 16 rotated exponents with their 16 sign/mantissa bytes into 16
// BF16 words (8 u32): per 4 weights two bit-selects and two byte-permutes.
__device__ __forceinline__ void merge16(const uint4 smv, const uint4 ex, uint32_t o[8]) {
    const uint32_t S[4] = {smv.x, smv.y, smv.z, smv.w};
    const uint32_t R[4] = {ex.x, ex.y, ex.z, ex.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t hi8 = (S[q] & 0x80808080u) | (R[q] & 0x7F7F7F7Fu);
        const uint32_t lo8 = (R[q] & 0x80808080u) | (S[q] & 0x7F7F7F7Fu);
        o[2 * q] = __byte_perm(lo8, hi8, 0x5140u);
        o[2 * q + 1] = __byte_perm(lo8, hi8, 0x7362u);
    }
}

// Sign/mantissa byte of element g of a block whose output starts at element
// `base`: from the block's staged bytes at shared address sm_s0 (chunk 0 on),
// or from global memory when they are not staged (sm_s0 = 0).
__device__ __forceinline__ uint32_t sm_byte(const uint8_t *sm, uint32_t sm_s0, uint32_t g, uint32_t base) {
    return sm_s0 ? lds_u8(sm_s0 + (g - base)) : (uint32_t)__ldg(sm + g);
}

// The chunks holding the block's first and last elements, by one warp:
// lanes 0..15 take the first chunk, lanes 16..31 the last one, one element
// each (only elements inside [s, e) are written).
__device__ __forceinline__ void merge_edges(const uint8_t *sm, uint32_t sm_s0, uint16_t *out, uint32_t sb,
                                            uint32_t base, uint32_t c_full, uint32_t span, uint32_t s, uint32_t e,
                                            uint32_t lane) {
    const bool head = s != base;
    const bool tail = (span & 15u) != 0u && !(head && c_full == 0u);
    const uint32_t c = (lane < 16u) ? 0u : c_full;
    const bool mine = (lane < 16u) ? head : tail;
    const uint32_t g = base + 16u * c + (lane & 15u);
    if (mine && g >= s && g < e && DF11_BOUNDS_OK(g - base < kMaxCodesPerBlock + 16u)) {
        const uint32_t sm8 = sm_byte(sm, sm_s0, g, base);
        const uint32_t r = lds_u8(sb + (g - base));
        // r = rotated exponent: high byte (s & 0x80) | (r & 0x7F), low byte (r & 0x80) | (s & 0x7F)
        const uint32_t hi8 = (sm8 & 0x80u) | (r & 0x7Fu);
        const uint32_t lo8 = (r & 0x80u) | (sm8 & 0x7Fu);
        out[g] = (uint16_t)(lo8 | (hi8 << 8));
    }
}
// merge_edges, then clears the two edge chunks (whole warp, converged).
__device__ __forceinline__ void merge_edges_clear(const uint8_t *sm, uint32_t sm_s0, uint16_t *out, uint32_t sb,
                                                  uint32_t base, uint32_t c_full, uint32_t span, uint32_t s,
                                                  uint32_t e, uint32_t lane) {
    merge_edges(sm, sm_s0, out, sb, base, c_full, span, s, e, lane);
    __syncwarp();
    const bool head = s != base;
    const bool tail = (span & 15u) != 0u && !(head && c_full == 0u);
    if ((lane == 0u && head) || (lane == 16u && tail)) sts_zero16(sb + 16u * (lane == 0u ? 0u : c_full));
}

// One decode chain: the 96-bit window (hi, lo, fl) of a format thread and
// the bits it must consume.
struct Chain {
    uint32_t hi, lo, fl;
    int32_t rem0;
};

// Builds a chain from its three big-endian stream words, its first code's
// bit offset and the end of its last code; bits at/after the end become 1.
__device__ __forceinline__ Chain make_chain(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t gap, int32_t end,
                                            uint32_t &err) {
    Chain c;
    int32_t rem0 = end - (int32_t)gap;
    if (rem0 < 0) {
        err |= DF11_KERR_OVERRUN;
        rem0 = 0;
        end = (int32_t)gap;
    }
    x0 |= __funnelshift_rc(kFull, 0u, (uint32_t)max(end, 0));
    x1 |= __funnelshift_rc(kFull, 0u, (uint32_t)max(end - 32, 0));
    x2 |= __funnelshift_rc(kFull, 0u, (uint32_t)max(end - 64, 0));
    c.hi = __funnelshift_lc(x1, x0, gap);
    c.lo = __funnelshift_lc(x2, x1, gap);
    c.fl = __funnelshift_lc(kFull, x2, gap);
    c.rem0 = rem0;
    return c;
}

// Long code at the top of a chain's window (its table entry was the escape):
// shifts the window past it and returns the count-table style entry that
// accounts for it (1 code, l bits) with a zero shift amount.  An invalid
// pattern stops the chain: the entry then brings the accumulator to `lim`.
__device__ __forceinline__ uint32_t count_long_code(uint32_t acc, uint32_t lim, uint32_t &hi, uint32_t &lo,
                                                    uint32_t &fl, uint32_t s_lim, uint32_t from, uint32_t max_len,
                                                    uint32_t &err) {
    const uint32_t l = long_code_length(hi, s_lim, from, max_len);
    if (l == 0u) {
        err |= DF11_KERR_BAD_CODE;
        return (lim - acc + 31u) & ~31u;  // reaches lim; low bits clear: no window shift
    }
    shift_window_clamped(hi, lo, fl, l);
    return (1u << 8) | (l << 24);
}

// Same for the decoding pass: ORs the long code's symbol into the buffer at
// index p, shifts the window and returns the meta word of 1 code with a
// zero shift amount (its length is added to `lbits`); an invalid pattern
// stops the chain at pend.
template <uint32_t kBufBytes>
__device__ __forceinline__ uint32_t decode_long_code(uint32_t pacc, uint32_t pend, uint32_t &hi, uint32_t &lo,
                                                     uint32_t &fl, uint32_t &lbits, uint32_t sb, uint32_t s_lim,
                                                     uint32_t s_offs, uint32_t s_symrot, uint32_t from,
                                                     uint32_t max_len) {
    const uint32_t l = long_code_length(hi, s_lim, from, max_len);
    if (l == 0u) {
        lbits += 0x100u;  // no code: the bit check below fails
        return (pend - pacc + 31u) & ~31u;
    }
    const uint32_t idx = (hi >> (32u - l)) + lds_u32(s_offs + 4u * l);
    const uint32_t p = pacc >> 8;
    if (DF11_BOUNDS_OK((p & ~3u) + 4u <= kBufBytes))
        red_or(sb + (p & ~3u), lds_u8(s_symrot + (idx & 255u)) << (8u * (p & 3u)));
    shift_window_clamped(hi, lo, fl, l);
    lbits += l;
    return 1u << 8;
}

// Count pass for both chains of a thread (count table, fused accumulator).
// Long codes are resolved in place (a short divergent branch), so all lanes
// keep looping together.  Table reads are plain C++ shared-memory loads so
// the compiler may schedule and predicate freely; `cnt` points at this
// lane's copy of the count table (entry i at cnt[i * kCountCopies]).
template <bool kLong>
__device__ __forceinline__ void count_pass(const Chain &A, const Chain &B, const uint32_t *cnt, uint32_t sh1,
                                           uint32_t s_lim, uint32_t from, uint32_t max_len, uint32_t &cA,
                                           uint32_t &cB, uint32_t &err) {
    uint32_t hA = A.hi, lA = A.lo, fA = A.fl, hB = B.hi, lB = B.lo, fB = B.fl;
    uint32_t aA = 0, aB = 0;
    const uint32_t limA = (uint32_t)A.rem0 << 24, limB = (uint32_t)B.rem0 << 24;
    // A valid chain needs at most 95 lookups; the cap only guards against a
    // malformed table or stream (reported as an overrun below).
    uint32_t guard = kLoopCap;
    while (((aA < limA) | (aB < limB)) && guard != 0u) {
        --guard;
        uint32_t eA = DF11_BOUNDS_OK((hA >> sh1) < (1u << kW1Max)) ? cnt[(hA >> sh1) * kCountCopies] : kEscape;
        uint32_t eB = DF11_BOUNDS_OK((hB >> sh1) < (1u << kW1Max)) ? cnt[(hB >> sh1) * kCountCopies] : kEscape;
        eA = (aA < limA) ? eA : 0u;
        eB = (aB < limB) ? eB : 0u;
        // Long codes exist only when the code is longer than the window; an
        // escape entry reaching the short-code instance (a corrupt table)
        // sets bit 31 of the accumulator and stops that chain.
        if (kLong && (eA | eB) >= kEscape) {  // rare: a long code
            if (eA == kEscape) eA = count_long_code(aA, limA, hA, lA, fA, s_lim, from, max_len, err);
            if (eB == kEscape) eB = count_long_code(aB, limB, hB, lB, fB, s_lim, from, max_len, err);
        }
        aA += eA;
        aB += eB;
        hA = __funnelshift_l(lA, hA, eA);
        lA = __funnelshift_l(fA, lA, eA);
        fA = __funnelshift_l(kFull, fA, eA);
        hB = __funnelshift_l(lB, hB, eB);
        lB = __funnelshift_l(fB, lB, eB);
        fB = __funnelshift_l(kFull, fB, eB);
    }
    cA = (aA >> 8) & 0xFFFFu;
    cB = (aB >> 8) & 0xFFFFu;
    if ((aA >> 24) != (uint32_t)A.rem0 || (aB >> 24) != (uint32_t)B.rem0) err |= DF11_KERR_OVERRUN;
}

// Decoding pass for both chains of a thread: writes each code's rotated
// exponent into the group buffer `buf` (word-addressed).  Symbol bytes are
// OR-ed into the (zeroed) buffer, one or two aligned words per lookup;
// unused symbol bytes of a table entry are zero.  Stops on the code counts
// (of the count pass, or stored with the tensor).  `sym` points at this
// lane's copy of the symbol table (entry i at sym[i * kSymCopies]).
// kCheck (stored counts, no count pass to check the stream): after the
// loop each chain must stand exactly on its code count and have taken
// exactly its bits (the low byte of the position accumulator sums the bits
// of the table entries, long codes are summed apart); else DF11_KERR_OVERRUN.
template <bool kLong, bool kCheck, uint32_t kSymCopies, uint32_t kBufBytes>
__device__ __forceinline__ void decode_pass(const Chain &A, const Chain &B, uint32_t startA, uint32_t cA,
                                            uint32_t startB, uint32_t cB, uint32_t *buf, uint32_t sb,
                                            const uint2 *sym, uint32_t sh2, uint32_t s_lim, uint32_t s_offs,
                                            uint32_t s_symrot, uint32_t from, uint32_t max_len, uint32_t &err) {
    uint32_t hA = A.hi, lA = A.lo, fA = A.fl, hB = B.hi, lB = B.lo, fB = B.fl;
    uint32_t pA = startA << 8, pB = startB << 8;
    uint32_t lbA = 0, lbB = 0;  // bits of long codes
    const uint32_t endPA = (startA + cA) << 8, endPB = (startB + cB) << 8;
    uint32_t guard = kLoopCap;  // as in the count pass
    while (((pA < endPA) | (pB < endPB)) && guard != 0u) {
        --guard;
        const uint2 eA = DF11_BOUNDS_OK((hA >> sh2) < (1u << kW2Max)) ? sym[(hA >> sh2) * kSymCopies]
                                                                      : make_uint2(0u, kEscape);
        const uint2 eB = DF11_BOUNDS_OK((hB >> sh2) < (1u << kW2Max)) ? sym[(hB >> sh2) * kSymCopies]
                                                                      : make_uint2(0u, kEscape);
        const bool actA = pA < endPA, actB = pB < endPB;
        uint32_t mA = actA ? eA.y : 0u;
        uint32_t mB = actB ? eB.y : 0u;
        if (kLong && (mA | mB) >= kEscape) {  // rare: a long code
            if (mA == kEscape)
                mA = decode_long_code<kBufBytes>(pA, endPA, hA, lA, fA, lbA, sb, s_lim, s_offs, s_symrot, from,
                                                 max_len);
            if (mB == kEscape)
                mB = decode_long_code<kBufBytes>(pB, endPB, hB, lB, fB, lbB, sb, s_lim, s_offs, s_symrot, from,
                                                 max_len);
        }
        const uint32_t bA = pA >> 8, bB = pB >> 8;
        const uint32_t shA = (bA & 3u) << 3, shB = (bB & 3u) << 3;
        uint32_t *wA = buf + (bA >> 2), *wB = buf + (bB >> 2);
        // (an escape entry has no symbol bytes: its stores OR zero)
        // the second word only when symbol bytes reach it (OR with zero is a no-op)
        const uint32_t hiA = __funnelshift_l(eA.x, 0u, shA), hiB = __funnelshift_l(eB.x, 0u, shB);
        if (actA && DF11_BOUNDS_OK(4u * ((bA >> 2) + 2u) <= kBufBytes)) {
            atomicOr(wA, eA.x << shA);
            if (hiA) atomicOr(wA + 1, hiA);
        }
        if (actB && DF11_BOUNDS_OK(4u * ((bB >> 2) + 2u) <= kBufBytes)) {
            atomicOr(wB, eB.x << shB);
            if (hiB) atomicOr(wB + 1, hiB);
        }
        pA += mA;
        pB += mB;
        hA = __funnelshift_l(lA, hA, mA);
        lA = __funnelshift_l(fA, lA, mA);
        fA = __funnelshift_l(kFull, fA, mA);
        hB = __funnelshift_l(lB, hB, mB);
        lB = __funnelshift_l(fB, lB, mB);
        fB = __funnelshift_l(kFull, fB, mB);
    }
    if (kCheck && (pA != endPA + (uint32_t)A.rem0 - lbA || pB != endPB + (uint32_t)B.rem0 - lbB))
        err |= DF11_KERR_OVERRUN;
}

// Merges chunks c_first, c_first + 128, ... < c_end (chunk c covers output
// elements base + 16c .. +16, at buffer offset 16c) with their sign/mantissa
// bytes, staged in shared memory from chunk c_lo on at `sm_s`, and clears
// each buffer chunk it reads (the decoding pass ORs into a clear buffer).
// Stores are 32 bytes per thread when `out` is 32-byte aligned (one warp
// instruction writes 1 KB of whole sectors), else two 16-byte stores.
template <uint32_t kBufBytes>
__device__ __forceinline__ void merge_chunks(uint16_t *out, uint32_t sb, uint32_t base, uint32_t c_first,
                                             uint32_t c_end, uint32_t sm_s, uint32_t c_lo, uint32_t al32,
                                             uint64_t n_elems) {
    for (uint32_t c = c_first; c < c_end; c += kGroupThreads) {
        if (!DF11_BOUNDS_OK(16u * (c + 1u) <= kBufBytes && (uint64_t)base + 16ull * (c + 1u) <= n_elems &&
                            c >= c_lo && 16u * (c - c_lo + 1u) <= kBufBytes))
            continue;
        const uint4 smv = lds_u4(sm_s + 16u * (c - c_lo));
        const uint4 ex = lds_u4(sb + 16u * c);
        sts_zero16(sb + 16u * c);
        uint32_t o[8];
        merge16(smv, ex, o);
        uint16_t *dst = out + (uint64_t)base + 16ull * c;
        if (al32) {
            st_u8x32(dst, o);
        } else
        {
            st_u4(dst, o[0], o[1], o[2], o[3]);
            st_u4(dst + 8, o[4], o[5], o[6], o[7]);
        }
    }
}

// Issues the bulk copies of block `blk`'s inputs into the group's staging
// area: its 2048 stream bytes plus the next block's first 16 (the last
// thread's look-ahead), its 160 gap bytes (+16: the next block's first
// gaps), and the 32-byte aligned window holding block_start[blk], [blk + 1].
template <class C>
__device__ __forceinline__ void issue_inputs(const DecodeArgs &a, uint64_t blk, uint32_t grp, uint32_t mbar) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect(mbar, kEncStage + kGapStage + 32u + C::kCntStage);
    bulk_g2s(grp + C::kGrpEnc, a.enc + blk * (uint64_t)(kThreadsPerBlockFmt * kBytesPerThread), kEncStage, mbar);
    bulk_g2s(grp + C::kGrpGap, a.gaps + blk * (uint64_t)(kThreadsPerBlockFmt * 5u / 8u), kGapStage, mbar);
    bulk_g2s(grp + C::kGrpBs, reinterpret_cast<const uint8_t *>(a.bstart) + ((4ull * blk) & ~15ull), 32u, mbar);
    if (!C::kCountTable)  // the block's 256 stored counts (one byte per thread)
        bulk_g2s(grp + C::kGrpCnt, a.counts + blk * (uint64_t)kThreadsPerBlockFmt, C::kCntStage, mbar);
}

// The two chains' code counts: from the count pass, or from the stored
// counts staged with the block's inputs.
template <class C, bool kLong>
__device__ __forceinline__ void chain_counts(const Chain &A, const Chain &B, uint32_t grp, uint32_t lt,
                                             const uint32_t *cnt_lane, uint32_t sh1, uint32_t s_lim, uint32_t from,
                                             uint32_t max_len, uint32_t &cA, uint32_t &cB, uint32_t &err) {
    if (C::kCountTable) {
        count_pass<kLong>(A, B, cnt_lane, sh1, s_lim, from, max_len, cA, cB, err);
    } else {
        uint32_t v;
        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(grp + C::kGrpCnt + 2u * lt));
        cA = v & 0xFFu;
        cB = v >> 8;
    }
}

// Stages the decode tables by one bulk copy, validates every entry and
// replicates them (whole CTA).  Returns false, uniformly over the CTA and with
// the error reported, when they did not arrive in time or are malformed;
// nothing has been written to global memory then.
// Issues the bulk copy of the compact tables (thread 0; nothing else of the
// CTA may write the group area until finish_tables): the CTA can do other
// work (a block search) while they travel.
template <class C>
__device__ __forceinline__ void issue_tables(const uint8_t *lut, uint32_t s_base, uint32_t tid) {
    const uint32_t s_tmbar = s_base + C::kOffGroups + C::kGroups * C::kGroupBytes;
    const uint32_t s_stage = s_base + C::kOffGroups;  // compact tables land here first
    if (tid == 0) {
        mbar_init(s_tmbar);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (C::kCountTable) {
            mbar_expect(s_tmbar, kLutBytes);
            bulk_g2s(s_stage, lut, kLutBytes, s_tmbar);
        } else {  // header, limits and symbols; then the symbol LUT (the count LUT is not used)
            mbar_expect(s_tmbar, C::kStageBytes);
            bulk_g2s(s_stage, lut, kOffCountLut, s_tmbar);
            bulk_g2s(s_stage + C::kStageSym, lut + kOffSymLut, kLutBytes - kOffSymLut, s_tmbar);
        }
    }
}

// Waits for the tables issue_tables requested, validates every entry and
// replicates them (whole CTA; the same contract as load_tables).
template <class C>
__device__ __forceinline__ bool finish_tables(const uint8_t *lut, uint32_t *err_out, uint8_t *smem, uint32_t s_base,
                                              uint32_t tid) {
    constexpr uint32_t kOffGroups = C::kOffGroups;
    constexpr uint32_t kSymCopies = C::kSymCopies;
    const uint32_t s_tmbar = s_base + kOffGroups + C::kGroups * C::kGroupBytes;
    const uint32_t s_stage = s_base + kOffGroups;
    __syncthreads();  // the barrier's initialisation is visible to every waiter
    const bool staged = wait_phase(s_tmbar, 0u);
    if (__syncthreads_or(!staged)) {
        // Uniform over the CTA.  One more bounded wait so no copy is left in
        // flight into this CTA's shared memory, then report and stop.
        if (tid == 0) {
            wait_phase(s_tmbar, 0u);
            if (err_out) atomicOr(err_out, kKernErrTimeout);
        }
        __syncthreads();
        return false;
    }
    const LutHeader *hdr = reinterpret_cast<const LutHeader *>(smem + kOffGroups + kOffHeader);
    const uint32_t w1 = hdr->w1, w2 = hdr->w2, max_len = hdr->max_len;
    {
        bool bad = !(hdr->magic == kMagic && w1 >= 1u && w1 <= (uint32_t)kW1Max && w2 >= 1u &&
                     w2 <= (uint32_t)kW2Max && max_len <= 32u);
        // header, limits and symbol list go to the front
        for (uint32_t i = tid; i < kOffCountLut / 16u; i += blockDim.x) {
            const uint4 v = lds_u4(s_stage + 16u * i);
            sts_u4(s_base + 16u * i, v.x, v.y, v.z, v.w);
        }
        // each store writes kCW copies of a count entry / kSW of a symbol
        // entry; the loops cover every (entry, copy), so every copy a lane can
        // read is written and validated here
        constexpr uint32_t kCW = kCountCopies < 4u ? kCountCopies : 4u;
        constexpr uint32_t kSW = kSymCopies % 2u == 0u ? 2u : 1u;
        static_assert(kCountCopies % kCW == 0u && kSymCopies % kSW == 0u, "copies fill whole stores");
        for (uint32_t i = tid; C::kCountTable && i < (1u << kW1Max) * (kCountCopies / kCW); i += blockDim.x) {
            const uint32_t ent = lds_u32(s_stage + kOffCountLut + 4u * (i / (kCountCopies / kCW)));
            const uint32_t nb = count_entry_bits(ent), nc = count_entry_codes(ent);
            bad |= ent != kEscape && (ent != count_entry(nb, nc) || nb == 0u || nb > w1 || nc == 0u || nc > nb);
            const uint32_t dst = s_base + kOffCountRep + 4u * kCW * i;
            if (kCW == 4u) sts_u4(dst, ent, ent, ent, ent);
            else if (kCW == 2u) asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(dst), "r"(ent) : "memory");
            else sts_u32(dst, ent);
        }
        for (uint32_t i = tid; i < (1u << kW2Max) * (kSymCopies / kSW); i += blockDim.x) {
            const uint2 ent = lds_u2(s_stage + C::kStageSym + 8u * (i / (kSymCopies / kSW)));
            const uint32_t nb = sym_entry_bits(ent.y), nc = sym_entry_codes(ent.y);
            bad |= ent.y != kEscape && (ent.y != sym_entry_meta(nb, nc) || nb == 0u || nb > w2 || nc == 0u ||
                                        nc > (uint32_t)kSymsPerEntry || nc > nb);
            const uint32_t dst = s_base + C::kOffSymRep + 8u * kSW * i;
            if (kSW == 2u) sts_u4(dst, ent.x, ent.y, ent.x, ent.y);
            else asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(dst), "r"(ent.x), "r"(ent.y) : "memory");
        }
        // Every entry is the escape flag or takes 1..W bits for 1..(bits)
        // codes, so each lookup makes progress: the decode loops then end
        // after at most 95 lookups plus 95 long codes whatever the stream.
        if (__syncthreads_or(bad)) {
            if (tid == 0 && err_out) atomicOr(err_out, DF11_KERR_BAD_CODE);
            return false;  // uniform over the CTA: nothing was written to global memory
        }
    }
    __syncthreads();  // the replicated tables are complete before any lookup
    return true;
}

template <class C>
__device__ __forceinline__ bool load_tables(const uint8_t *lut, uint32_t *err_out, uint8_t *smem, uint32_t s_base,
                                            uint32_t tid) {
    issue_tables<C>(lut, s_base, tid);
    return finish_tables<C>(lut, err_out, smem, s_base, tid);
}

// Where a decoded block goes: StoreSink writes it as BF16 (the decoder);
// the fused matrix-vector product below multiplies it into y instead, and
// the fused GEMM writes it into tensor-core operand tiles.  A sink takes the
// whole chunks of a block (`chunks`, every thread of the group) and its two
// edge chunks (`edges`, warp 0), and clears every buffer chunk it reads.
// Hooks let a sink publish what it wrote: `begin_block(s, e)` before a
// block's merge and `block_done(s, e, ok, range_ok)` after it (every thread;
// the block's element range, whether it decoded and whether its range was
// even plausible), `published(lt)`
// right after the next group barrier (every thread of the group has then
// finished that merge), `plan(s, e, lt)` right after it too (the block about
// to be decoded: a sink may prepare its merge there), and `finish(group, lt)`
// after the group's last block.
struct NoHooks {
    __device__ __forceinline__ void plan(uint32_t, uint32_t, uint32_t) {}
    __device__ __forceinline__ void begin_block(uint32_t, uint32_t) {}
    __device__ __forceinline__ void block_done(uint32_t, uint32_t, bool, bool) {}
    __device__ __forceinline__ void published(uint32_t) {}
    __device__ __forceinline__ void finish(uint32_t, uint32_t) {}
};

struct StoreSink : NoHooks {
    uint16_t *out;
    const uint8_t *sm;
    uint64_t n_elems;
    uint32_t al32;
    template <uint32_t kBufBytes>
    __device__ __forceinline__ void chunks(uint32_t sb, uint32_t base, uint32_t c_first, uint32_t c_end,
                                           uint32_t sm_s, uint32_t c_lo) {
        merge_chunks<kBufBytes>(out, sb, base, c_first, c_end, sm_s, c_lo, al32, n_elems);
    }
    __device__ __forceinline__ void edges(uint32_t sb, uint32_t base, uint32_t c_full, uint32_t span, uint32_t s,
                                          uint32_t e, uint32_t lane, uint32_t sm_s0) {
        merge_edges_clear(sm, sm_s0, out, sb, base, c_full, span, s, e, lane);
    }
};

// The persistent decode loop of one group (the tables are loaded): the group
// decodes format blocks blk, blk + stride, ... below blk_end and hands every
// decoded block to the sink.  With `counter` (the shared-memory address of a
// u32 holding the CTA's next block; 0: the fixed stride) the groups instead
// take the CTA's blocks in order from that counter, whichever group is free
// first (the group's leader takes one at each first barrier and passes it on
// through the group's aux word, which the others read after the second).
// kLong: compiled with the long-code path (codes longer than the table
// windows); without it the loops carry no escape handling at all.
template <class C, bool kLong, class Sink>
__device__ __forceinline__ void decode_loop(const DecodeArgs &a, Sink &sink, uint64_t blk, uint64_t stride,
                                            uint64_t blk_end, uint32_t counter = 0u) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_lim = s_base + kOffLim;
    const uint32_t s_offs = s_base + kOffOffs;
    const uint32_t s_symrot = s_base + kOffSymRot;
    const uint32_t tid = threadIdx.x;
    const uint32_t group = tid / kGroupThreads;
    const uint32_t lt = tid % kGroupThreads;  // thread within the group
    const uint32_t lane = tid & 31u;
    const uint32_t warp = lt >> 5;            // warp within the group
    const uint32_t grp = s_base + C::kOffGroups + group * C::kGroupBytes;
    const uint32_t sb = grp;                  // exponent buffer
    const uint32_t wtot = grp + C::kGrpWtot;  // 4 warp totals
    const uint32_t mb_in = grp + C::kGrpMbar, mb_sm = grp + C::kGrpMbar + 8u;
    const uint32_t *cnt_lane = reinterpret_cast<const uint32_t *>(smem + kOffCountRep) + (lane % kCountCopies);
    const uint2 *sym_lane = reinterpret_cast<const uint2 *>(smem + C::kOffSymRep) + (lane % C::kSymCopies);
    uint32_t *buf = reinterpret_cast<uint32_t *>(smem + C::kOffGroups + group * C::kGroupBytes);
    uint32_t my_err = 0;

    const LutHeader *hdr = reinterpret_cast<const LutHeader *>(smem + kOffHeader);
    const uint32_t w1 = hdr->w1, w2 = hdr->w2, max_len = hdr->max_len;
    const uint32_t sh1 = 32u - w1, sh2 = 32u - w2;

    // The exponent buffer starts clear; the merge clears what it reads.
    for (uint32_t c = lt; c < C::kSbufBytes / 16u; c += kGroupThreads) sts_zero16(sb + 16u * c);

    // ---- the group's mbarriers (inputs of the next block; first
    // sign/mantissa vectors of this one) and its first block's inputs
    const uint32_t aux = grp + C::kGrpAux;
    if (lt == 0) {
        mbar_init(mb_in);
        mbar_init(mb_sm);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (counter) {
            blk = atomicAdd(reinterpret_cast<uint32_t *>(smem + (counter - s_base)), 1u);
            sts_u32(aux, (uint32_t)blk);
        }
        if (blk < blk_end) issue_inputs<C>(a, blk, grp, mb_in);
    }
    group_barrier(group);
    if (counter) blk = lds_u32(aux);
    uint32_t ph_in = 0, ph_sm = 0;

    while (blk < blk_end) {
        if (!wait_phase(mb_in, ph_in)) my_err |= kKernErrTimeout;
        ph_in ^= 1u;
        const uint64_t tA = blk * (uint64_t)kThreadsPerBlockFmt + 2u * lt;
        const uint32_t bs_off = (uint32_t)((4ull * blk) & 15ull);
        const uint32_t s = lds_u32(grp + C::kGrpBs + bs_off), e = lds_u32(grp + C::kGrpBs + bs_off + 4u);
        const uint32_t base = s & ~15u;  // first 16-element chunk of the block's output
        // buffer index of output element g is g - base (< span)
        const bool range_ok = (e >= s) && ((uint64_t)e <= a.n_elems) && (e - base <= C::kBufSyms);
        const uint32_t span = range_ok ? e - base : 0u;
        const uint32_t c_lo = (s != base) ? 1u : 0u;
        const uint32_t c_full = span >> 4;  // chunks [c_lo, c_full) lie wholly inside [s, e)
        const uint32_t c0 = c_lo + lt;
        // ---- the two chains: format threads tA and tA + 1
        const uint4 v = lds_u4(grp + C::kGrpEnc + 16u * lt);
        const uint32_t nextw = lds_u32(grp + C::kGrpEnc + 16u * lt + 16u);
        // gaps are an MSB-first bit string: bits [10 lt, 10 lt + 15) of the
        // block's gap bytes hold the gaps of tA, tA + 1 and tA + 2
        const uint32_t gq = (10u * lt) >> 5;
        const uint32_t g_hi = lds_u32(grp + C::kGrpGap + 4u * gq), g_lo = lds_u32(grp + C::kGrpGap + 4u * gq + 4u);
        const uint32_t gb = __funnelshift_l(bswap32(g_lo), bswap32(g_hi), (10u * lt) & 31u);
        uint32_t gapA = gb >> 27, gapB = (gb >> 22) & 31u;
        const uint32_t gapC = (gb >> 17) & 31u;
        int32_t endA, endB;
        if (tA >= a.n_threads) { gapA = 0; endA = 0; }
        else if (tA + 1 == a.n_threads) endA = (int32_t)(a.total_bits - 64ull * tA);
        else endA = 64 + (int32_t)gapB;
        if (tA + 1 >= a.n_threads) { gapB = 0; endB = 0; }
        else if (tA + 2 == a.n_threads) endB = (int32_t)(a.total_bits - 64ull * (tA + 1));
        else endB = 64 + (int32_t)gapC;
        const Chain A = make_chain(bswap32(v.x), bswap32(v.y), bswap32(v.z), gapA, endA, my_err);
        const Chain B = make_chain(bswap32(v.z), bswap32(v.w), bswap32(nextw), gapB, endB, my_err);

        // ---- pass 1: count the codes of both chains (or read the stored counts)
        uint32_t cA, cB;
        chain_counts<C, kLong>(A, B, grp, lt, cnt_lane, sh1, s_lim, w1 + 1u, max_len, cA, cB, my_err);

        // ---- block scan: warp inclusive scan, then across the group's warps
        const uint32_t cnt = cA + cB;
        uint32_t incl = cnt;
#pragma unroll
        for (uint32_t d = 1; d < 32; d <<= 1) {
            const uint32_t x = __shfl_up_sync(kFull, incl, d);
            if (lane >= d) incl += x;
        }
        constexpr uint32_t kWarps = kGroupThreads / 32;
        if (lane == 31u) sts_u32(wtot + 4u * warp, incl);
        group_barrier(group);
        // every thread has read this block's staged inputs: fetch the next
        uint64_t nxt = blk + stride;
        if (lt == 0) {
            if (counter) {
                nxt = atomicAdd(reinterpret_cast<uint32_t *>(smem + (counter - s_base)), 1u);
                sts_u32(aux, (uint32_t)nxt);  // read by the group after the next barrier
            }
            if (nxt < blk_end) issue_inputs<C>(a, nxt, grp, mb_in);
        }
        sink.published(lt);  // the previous block's merge is done by the whole group
        sink.plan(s, e, lt);
        // and this block's sign/mantissa bytes (chunks 0 .. the block's last
        // chunk, at most kBufSyms bytes: the edge chunks are read from there
        // too; always at least 16 bytes).  Every thread of the group has
        // passed its previous merge, so the staging area is free.
        if (lt == 0) {
            // (64-bit: the end of the last chunk passes 2^32 when the tensor
            // holds nearly 2^32 elements)
            const uint64_t from = range_ok ? (uint64_t)base : 0u;
            const uint64_t upto = range_ok ? (((uint64_t)e + 15u) & ~15ull) : 16u;
            const uint32_t bytes =
                upto > from ? (uint32_t)min((uint64_t)(C::kStageSm ? C::kSmBytes : C::kSbufBytes), upto - from) : 16u;
            const uint64_t src = upto > from ? from : (range_ok ? base : 0u);
            if (C::kStageSm) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect(mb_sm, bytes);
                bulk_g2s(grp + C::kGrpSm, a.sm + src, bytes, mb_sm);
            } else {
                // unstaged (the merge reads them from global memory): bring
                // them into L2 while the block decodes
                bulk_prefetch_l2(a.sm + src, bytes);
            }
        }

        uint32_t wsum = (lane < kWarps) ? lds_u32(wtot + 4u * lane) : 0u;
#pragma unroll
        for (uint32_t d = 1; d < kWarps; d <<= 1) {
            const uint32_t x = __shfl_up_sync(kFull, wsum, d);
            if (lane >= d) wsum += x;
        }
        const uint32_t total = __shfl_sync(kFull, wsum, kWarps - 1u);
        const uint32_t wpre = __shfl_sync(kFull, wsum, (warp + kWarps - 1u) % kWarps) * (warp != 0u ? 1u : 0u);
        const bool ok = range_ok && (total == e - s);
        if (!ok && lt == 0) my_err |= range_ok ? DF11_KERR_COUNT_MISMATCH : DF11_KERR_BAD_BLOCK;

        // ---- pass 2: decode both chains again into the buffer
        if (ok) {
            const uint32_t startA = (s - base) + wpre + incl - cnt;  // buffer index of A's first code
            decode_pass<kLong, !C::kCountTable, C::kSymCopies, C::kSbufBytes>(
                A, B, startA, cA, startA + cA, cB, buf, sb, sym_lane, sh2, s_lim, s_offs, s_symrot, w2 + 1u, max_len,
                my_err);
        }
        group_barrier(group);

        // ---- merge with sign/mantissa and store, 16 weights per step
        if (C::kStageSm) {
            if (!wait_phase(mb_sm, ph_sm)) my_err |= kKernErrTimeout;
            ph_sm ^= 1u;
        }
        sink.begin_block(s, e);
        if (ok) {
            // (the staged bytes start at chunk 0; the chunk merges index them from c_lo)
            sink.template chunks<C::kSbufBytes>(sb, base, c0, c_full, grp + C::kGrpSm + 16u * c_lo, c_lo);
            if (warp == 0) sink.edges(sb, base, c_full, span, s, e, lane, C::kStageSm ? grp + C::kGrpSm : 0u);
        }
        sink.block_done(s, e, ok, range_ok);
        // No barrier here: the next block's buffer writes and staging copies
        // come after its scan barrier, which every thread reaches only after
        // this merge.
        blk = counter ? (uint64_t)lds_u32(aux) : blk + stride;
    }
    sink.finish(group, lt);
    if (my_err && a.err) atomicOr(a.err, my_err);
}

// Loads the tables (whole CTA), then runs the decode loop of this thread's
// group over blocks blk_first + (CTA + group * grid) + k * (grid * groups)
// below blk_end: the first blocks go to every CTA's group 0 before any
// CTA's group 1, so a tensor of few blocks is spread over all the SMs (one
// block per SM decodes faster than eight on one).
template <class C, bool kLong, class Sink>
__device__ __forceinline__ void decode_blocks(const DecodeArgs &a, Sink &sink, uint64_t blk_first, uint64_t blk_end,
                                              bool tables_issued = false) {
    extern __shared__ __align__(128) uint8_t smem[];
    if (tables_issued ? !finish_tables<C>(a.lut, a.err, smem, smem_addr(smem), threadIdx.x)
                      : !load_tables<C>(a.lut, a.err, smem, smem_addr(smem), threadIdx.x))
        return;
    const uint32_t group = threadIdx.x / kGroupThreads;
    decode_loop<C, kLong>(a, sink, blk_first + blockIdx.x + (uint64_t)group * gridDim.x,
                          (uint64_t)gridDim.x * C::kGroups, blk_end);
}

template <class C, bool kLong>
__global__ void __launch_bounds__(C::kCtaThreads, 1) df11_decode_kernel(const DecodeArgs a) {
    StoreSink sink{{}, a.out, a.sm, a.n_elems, a.out_al32};
    decode_blocks<C, kLong>(a, sink, 0u, a.n_blocks);
}


// ----------------------------------------------------------------- row gather
struct GatherArgs {
    DecodeArgs d;           // the compressed matrix (d.out unused)
    const uint32_t *rows;   // requested row indices
    uint16_t *out;          // n_rows x row_len
    uint64_t row_len;
    uint64_t n_rows_total;  // n_elems / row_len
    uint32_t n_rows;
};

// Largest b in [lo, hi) with bs[b] <= x (lo if none), by one warp (32-way
// search, ceil(log32 (hi - lo)) rounds of one load per lane).  bs[0] is 0 for
// valid data; with corrupt starts the result is still some block in range
// (the per-block range checks then catch the inconsistency).
__device__ __forceinline__ uint64_t find_block_in(const uint32_t *bs, uint64_t lo, uint64_t hi, uint64_t x,
                                                 uint32_t lane) {
    while (hi - lo > 1u) {
        const uint64_t step = (hi - lo + 31u) / 32u;
        const uint64_t p = lo + (uint64_t)lane * step;
        const bool le = p < hi && (uint64_t)__ldg(bs + p) <= x;
        const uint32_t m = __ballot_sync(kFull, le) | 1u;  // lane 0 probes lo itself
        const uint64_t j = 31u - __clz(m);
        lo += j * step;
        hi = min(hi, lo + step);
    }
    return lo;
}
__device__ __forceinline__ uint64_t find_block(const uint32_t *bs, uint64_t n_blocks, uint64_t x, uint32_t lane) {
    return find_block_in(bs, 0u, n_blocks, x, lane);
}
// The same answer, probing the 32 blocks from `hint` first (one load per
// lane): the 32-way search runs only when the answer lies outside them.
__device__ __forceinline__ uint64_t find_block_near(const uint32_t *bs, uint64_t n_blocks, uint64_t hint, uint64_t x,
                                                    uint32_t lane) {
    if (n_blocks == 0u) return 0u;
    hint = min(hint, n_blocks - 1u);
    const uint64_t p = hint + lane;
    const uint32_t m = __ballot_sync(kFull, p < n_blocks && (uint64_t)__ldg(bs + p) <= x);
    if (m == 0u) return find_block_in(bs, 0u, hint, x, lane);  // (hint = 0: block 0)
    const uint32_t j = 31u - __clz(m);
    if (j < 31u || hint + 32u >= n_blocks) return hint + j;
    return find_block_in(bs, hint + 31u, n_blocks, x, lane);
}

// One group per requested row (grid-stride over rows): the format blocks
// covering the row are staged, decoded as in df11_decode_kernel and merged
// element by element into the output row.  Three group barriers per block
// (inputs and buffer are reused synchronously; this path decodes a few
// blocks per row, not the whole tensor).
template <class C, bool kLong>
__global__ void __launch_bounds__(C::kCtaThreads, 1) df11_gather_kernel(const GatherArgs ga) {
    const DecodeArgs &a = ga.d;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_lim = s_base + kOffLim;
    const uint32_t s_offs = s_base + kOffOffs;
    const uint32_t s_symrot = s_base + kOffSymRot;
    const uint32_t tid = threadIdx.x;
    const uint32_t group = tid / kGroupThreads;
    const uint32_t lt = tid % kGroupThreads;
    const uint32_t lane = tid & 31u;
    const uint32_t warp = lt >> 5;
    const uint32_t grp = s_base + C::kOffGroups + group * C::kGroupBytes;
    const uint32_t sb = grp;
    const uint32_t wtot = grp + C::kGrpWtot;
    const uint32_t mb_in = grp + C::kGrpMbar;
    const uint32_t aux = grp + C::kGrpAux;
    const uint32_t *cnt_lane = reinterpret_cast<const uint32_t *>(smem + kOffCountRep) + (lane % kCountCopies);
    const uint2 *sym_lane = reinterpret_cast<const uint2 *>(smem + C::kOffSymRep) + (lane % C::kSymCopies);
    uint32_t *buf = reinterpret_cast<uint32_t *>(smem + C::kOffGroups + group * C::kGroupBytes);
    uint32_t my_err = 0;

    if (!load_tables<C>(a.lut, a.err, smem, s_base, tid)) return;
    const LutHeader *hdr = reinterpret_cast<const LutHeader *>(smem + kOffHeader);
    const uint32_t w1 = hdr->w1, w2 = hdr->w2, max_len = hdr->max_len;
    const uint32_t sh1 = 32u - w1, sh2 = 32u - w2;

    for (uint32_t c = lt; c < C::kSbufBytes / 16u; c += kGroupThreads) sts_zero16(sb + 16u * c);
    if (lt == 0) {
        mbar_init(mb_in);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    group_barrier(group);
    uint32_t ph_in = 0;

    for (uint64_t i = (uint64_t)blockIdx.x * C::kGroups + group; i < ga.n_rows;
         i += (uint64_t)gridDim.x * C::kGroups) {
        const uint64_t row = __ldg(ga.rows + i);
        const bool row_ok = row < ga.n_rows_total;
        const uint64_t lo = row * ga.row_len, hi = lo + ga.row_len;
        if (warp == 0 && row_ok) {
            const uint64_t b0 = find_block(a.bstart, a.n_blocks, lo, lane);
            const uint64_t b1 = find_block(a.bstart, a.n_blocks, hi - 1u, lane);
            if (lane == 0) {
                sts_u32(aux, (uint32_t)b0);
                sts_u32(aux + 4u, (uint32_t)b1);
            }
        }
        group_barrier(group);
        const uint32_t b0 = lds_u32(aux), b1 = lds_u32(aux + 4u);
        if (!row_ok || b1 < b0) {
            if (lt == 0) my_err |= row_ok ? DF11_KERR_BAD_BLOCK : DF11_KERR_BAD_ROW;
            group_barrier(group);  // the range words are read before the next row writes them
            continue;
        }
        uint16_t *orow = ga.out + i * ga.row_len;
        for (uint64_t blk = b0; blk <= b1; ++blk) {
            if (lt == 0) issue_inputs<C>(a, blk, grp, mb_in);
            if (!wait_phase(mb_in, ph_in)) my_err |= kKernErrTimeout;
            ph_in ^= 1u;
            const uint64_t tA = blk * (uint64_t)kThreadsPerBlockFmt + 2u * lt;
            const uint32_t bs_off = (uint32_t)((4ull * blk) & 15ull);
            const uint32_t s = lds_u32(grp + C::kGrpBs + bs_off), e = lds_u32(grp + C::kGrpBs + bs_off + 4u);
            const uint32_t base = s & ~15u;
            const bool range_ok = (e >= s) && ((uint64_t)e <= a.n_elems) && (e - base <= C::kBufSyms);
            const uint32_t span = range_ok ? e - base : 0u;

            const uint4 v = lds_u4(grp + C::kGrpEnc + 16u * lt);
            const uint32_t nextw = lds_u32(grp + C::kGrpEnc + 16u * lt + 16u);
            const uint32_t gq = (10u * lt) >> 5;
            const uint32_t g_hi = lds_u32(grp + C::kGrpGap + 4u * gq), g_lo = lds_u32(grp + C::kGrpGap + 4u * gq + 4u);
            const uint32_t gb = __funnelshift_l(bswap32(g_lo), bswap32(g_hi), (10u * lt) & 31u);
            uint32_t gapA = gb >> 27, gapB = (gb >> 22) & 31u;
            const uint32_t gapC = (gb >> 17) & 31u;
            int32_t endA, endB;
            if (tA >= a.n_threads) { gapA = 0; endA = 0; }
            else if (tA + 1 == a.n_threads) endA = (int32_t)(a.total_bits - 64ull * tA);
            else endA = 64 + (int32_t)gapB;
            if (tA + 1 >= a.n_threads) { gapB = 0; endB = 0; }
            else if (tA + 2 == a.n_threads) endB = (int32_t)(a.total_bits - 64ull * (tA + 1));
            else endB = 64 + (int32_t)gapC;
            const Chain A = make_chain(bswap32(v.x), bswap32(v.y), bswap32(v.z), gapA, endA, my_err);
            const Chain B = make_chain(bswap32(v.z), bswap32(v.w), bswap32(nextw), gapB, endB, my_err);

            uint32_t cA, cB;
            chain_counts<C, kLong>(A, B, grp, lt, cnt_lane, sh1, s_lim, w1 + 1u, max_len, cA, cB, my_err);
            const uint32_t cnt = cA + cB;
            uint32_t incl = cnt;
#pragma unroll
            for (uint32_t d = 1; d < 32; d <<= 1) {
                const uint32_t x = __shfl_up_sync(kFull, incl, d);
                if (lane >= d) incl += x;
            }
            constexpr uint32_t kWarps = kGroupThreads / 32;
            if (lane == 31u) sts_u32(wtot + 4u * warp, incl);
            group_barrier(group);
            uint32_t wsum = (lane < kWarps) ? lds_u32(wtot + 4u * lane) : 0u;
#pragma unroll
            for (uint32_t d = 1; d < kWarps; d <<= 1) {
                const uint32_t x = __shfl_up_sync(kFull, wsum, d);
                if (lane >= d) wsum += x;
            }
            const uint32_t total = __shfl_sync(kFull, wsum, kWarps - 1u);
            const uint32_t wpre = __shfl_sync(kFull, wsum, (warp + kWarps - 1u) % kWarps) * (warp != 0u ? 1u : 0u);
            const bool ok = range_ok && (total == e - s);
            if (!ok && lt == 0) my_err |= range_ok ? DF11_KERR_COUNT_MISMATCH : DF11_KERR_BAD_BLOCK;
            if (ok) {
                const uint32_t startA = (s - base) + wpre + incl - cnt;
                decode_pass<kLong, !C::kCountTable, C::kSymCopies, C::kSbufBytes>(
                    A, B, startA, cA, startA + cA, cB, buf, sb, sym_lane, sh2, s_lim, s_offs, s_symrot, w2 + 1u,
                    max_len, my_err);
            }
            group_barrier(group);
            if (ok) {  // the row's part of this block, element by element
                const uint64_t g0 = max((uint64_t)s, lo), g1 = min((uint64_t)e, hi);
                for (uint64_t g = g0 + lt; g < g1; g += kGroupThreads) {
                    if (!DF11_BOUNDS_OK(g - lo < ga.row_len && g - base < C::kSbufBytes && g < a.n_elems)) continue;
                    const uint32_t sm8 = __ldg(a.sm + g);
                    const uint32_t r = lds_u8(sb + (uint32_t)(g - base));
                    const uint32_t hi8 = (sm8 & 0x80u) | (r & 0x7Fu);
                    const uint32_t lo8 = (r & 0x80u) | (sm8 & 0x7Fu);
                    orow[g - lo] = (uint16_t)(lo8 | (hi8 << 8));
                }
            }
            group_barrier(group);  // every read of the buffer and the staged inputs is done
            for (uint32_t c = lt; c < (span + 19u) >> 4; c += kGroupThreads) sts_zero16(sb + 16u * c);
        }
        group_barrier(group);  // the range words are read before the next row writes them
    }
    if (my_err && a.err) atomicOr(a.err, my_err);
}

// ------------------------------------------------- fused decode -> matrix-vector
// Decompressing a matrix right before its multiplication ("Decompression
// adaptee a l'inference GPU") taken to the end for small batches: the merge
// multiplies each decoded chunk by the activations instead of storing it, so
// the BF16 weights never reach global memory.  For T <= 4 the product is a
// matrix-vector stream (at most 8 flops per weight), which fits in the merge
// on the CUDA cores.  Each listed matrix j of the tensor gets
// y_j[t][r] += sum_c W_j[r][c] * x_j[t][c] (FP32; each warp reduces its
// partial sums per row and adds them with FP32 atomics).
constexpr uint32_t kMaxGemvMats = 16;
constexpr uint32_t kNoRow = 0xFFFFFFFFu;

struct GemvMat {
    uint32_t off, end;      // elements [off, end) of the tensor; both multiples of 16
    uint32_t rows, cols;    // cols a multiple of 16
    uint32_t magic, shift;  // chunk q = (g - off) / 16 (< 2^28) lies in row (q * magic) >> shift
    const uint16_t *x;      // [T][cols] BF16
    float *y;               // [T][rows] FP32, accumulated into
};

struct GemvArgs {
    DecodeArgs d;
    GemvMat m[kMaxGemvMats];  // ordered by offset, not overlapping
    uint32_t n_mats, T;
    uint32_t e_first, e_last;  // first and last element of the matrices
};

// lo += w.lo * x.lo and hi += w.hi * x.hi for two BF16 pairs, with FP32
// accumulators (mixed-precision FMA: the product is exact, one rounding).
__device__ __forceinline__ void fma2_bf16(float &lo, float &hi, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(w), "r"(x));
}

// Accumulates 16 BF16 weights (8 words, element order) times 16 BF16
// activations into (lo, hi).
__device__ __forceinline__ void dot16(const uint32_t w[8], const uint4 xa, const uint4 xb, float &lo, float &hi) {
    const uint32_t X[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) fma2_bf16(lo, hi, w[i], X[i]);
}

__device__ __forceinline__ uint32_t gemv_row(uint32_t local, uint32_t magic, uint32_t shift) {
    return (uint32_t)(((uint64_t)(local >> 4) * magic) >> shift);
}

// Adds a warp's per-lane sums into y: one atomic per run of lanes holding the
// same key (the row), at that run's `yrow` (y + row) for each t (stride
// `rows`).  Equal keys must sit in contiguous lanes (the caller's element
// order guarantees it); a lane with key kNoRow holds nothing.  Whole warp,
// converged.
template <uint32_t TM>
__device__ __forceinline__ void flush_runs(const float (&lo)[TM], const float (&hi)[TM], uint32_t key,
                                           float *const yrow, uint32_t rows, uint32_t T, uint32_t lane) {
    const uint32_t k0 = __shfl_sync(kFull, key, 0);
    if (__all_sync(kFull, key == k0)) {  // the common case: one run
        if (k0 == kNoRow) return;
#pragma unroll
        for (uint32_t t = 0; t < TM; ++t) {
            float v = lo[t] + hi[t];
#pragma unroll
            for (uint32_t d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
            if (lane == 0 && t < T) atomicAdd(yrow + (uint64_t)t * rows, v);
        }
        return;
    }
    // suffix sums inside each run, then the run's first lane adds
    uint32_t same = 0;  // bit k: lane + 2^k holds the same key
#pragma unroll
    for (uint32_t k = 0; k < 5; ++k) {
        const uint32_t o = __shfl_down_sync(kFull, key, 1u << k);
        if (lane + (1u << k) < 32u && o == key) same |= 1u << k;
    }
    const uint32_t prev = __shfl_up_sync(kFull, key, 1);
    const bool first = (lane == 0 || prev != key) && key != kNoRow;
#pragma unroll
    for (uint32_t t = 0; t < TM; ++t) {
        float v = lo[t] + hi[t];
#pragma unroll
        for (uint32_t k = 0; k < 5; ++k) {
            const float o = __shfl_down_sync(kFull, v, 1u << k);
            if (same & (1u << k)) v += o;
        }
        if (first && t < T) atomicAdd(yrow + (uint64_t)t * rows, v);
    }
}

// The fused sink: decoded chunks are multiplied into y instead of stored.
// Each warp takes a contiguous quarter of the block's whole chunks (lane l
// the chunk at l + 32 i), so its successive 512-weight pieces mostly stay in
// one row: lanes accumulate until some lane's row changes, then the warp
// adds its sums into y.  `m` is the first matrix that can still hold the
// warp's elements (they only grow: chunks within a block, then blocks by
// stride).
template <uint32_t TM>
struct GemvSink : NoHooks {
    const GemvArgs &g;
    uint32_t m;

    template <uint32_t kBufBytes>
    __device__ __forceinline__ void chunks(uint32_t sb, uint32_t base, uint32_t /*c_first*/, uint32_t c_end,
                                           uint32_t sm_s, uint32_t c_lo) {
        const uint32_t lane = threadIdx.x & 31u, warp = (threadIdx.x >> 5) % (kGroupThreads / 32u);
        const uint32_t n = c_end > c_lo ? c_end - c_lo : 0u;
        const uint32_t per = ((n + 3u) / 4u + 31u) & ~31u;  // whole warp iterations
        const uint32_t w_lo = c_lo + min(n, warp * per), w_hi = c_lo + min(n, (warp + 1u) * per);
        if (w_lo >= w_hi) return;  // warp-uniform
        const uint32_t g_lo = base + 16u * w_lo, g_hi = base + 16u * w_hi;
        while (m < g.n_mats && g_lo >= g.m[m].end) ++m;
        if (m < g.n_mats && g_lo >= g.m[m].off && g_hi <= g.m[m].end)
            one_matrix<kBufBytes>(sb, base, w_lo, w_hi, sm_s, c_lo, lane);
        else
            any_matrices<kBufBytes>(sb, base, w_lo, w_hi, sm_s, c_lo, lane);
    }

    // All of the warp's chunks lie in matrix m (the common case).
    template <uint32_t kBufBytes>
    __device__ __forceinline__ void one_matrix(uint32_t sb, uint32_t base, uint32_t w_lo, uint32_t w_hi,
                                               uint32_t sm_s, uint32_t c_lo, uint32_t lane) {
        const GemvMat &M = g.m[m];
        const uint32_t off = M.off, cols = M.cols, magic = M.magic, shift = M.shift, rows = M.rows, T = g.T;
        const uint16_t *const x = M.x;
        float lo[TM], hi[TM];
#pragma unroll
        for (uint32_t t = 0; t < TM; ++t) lo[t] = hi[t] = 0.f;
        uint32_t held = kNoRow;  // row of the sums this lane holds
        for (uint32_t cw = w_lo; cw < w_hi; cw += 32u) {  // warp-uniform trip count
            const uint32_t c = cw + lane;
            const bool act = c < w_hi && DF11_BOUNDS_OK(16u * (c + 1u) <= kBufBytes &&
                                                        (uint64_t)base + 16ull * (c + 1u) <= g.d.n_elems &&
                                                        c >= c_lo && 16u * (c - c_lo + 1u) <= kBufBytes);
            uint4 smv, ex;
            uint32_t local = 0, row = kNoRow;
            if (act) {
                smv = lds_u4(sm_s + 16u * (c - c_lo));
                ex = lds_u4(sb + 16u * c);
                sts_zero16(sb + 16u * c);
                local = base + 16u * c - off;
                row = gemv_row(local, magic, shift);
            }
            // Rows grow with the lane within a step and from step to step, and
            // a lane that is idle once stays idle: so after this flush rule the
            // lanes holding one row are always contiguous.
            if (__any_sync(kFull, act && held != kNoRow && row != held)) {
                flush_runs<TM>(lo, hi, held, M.y + (held == kNoRow ? 0u : held), rows, T, lane);
#pragma unroll
                for (uint32_t t = 0; t < TM; ++t) lo[t] = hi[t] = 0.f;
                held = kNoRow;
            }
            if (act) {
                uint32_t w[8];
                merge16(smv, ex, w);
                const uint16_t *xp = x + (local - row * cols);
#pragma unroll
                for (uint32_t t = 0; t < TM; ++t) {
                    if (t < T) {
                        const uint4 *xv = reinterpret_cast<const uint4 *>(xp + (uint64_t)t * cols);
                        dot16(w, __ldg(xv), __ldg(xv + 1), lo[t], hi[t]);
                    }
                }
                held = row;
            }
        }
        flush_runs<TM>(lo, hi, held, M.y + (held == kNoRow ? 0u : held), rows, T, lane);
    }

    // The warp's chunks meet a matrix boundary or elements of no matrix:
    // each chunk finds its matrix, and the warp adds its sums every step.
    template <uint32_t kBufBytes>
    __device__ __forceinline__ void any_matrices(uint32_t sb, uint32_t base, uint32_t w_lo, uint32_t w_hi,
                                                 uint32_t sm_s, uint32_t c_lo, uint32_t lane) {
        uint32_t mm = m;
        for (uint32_t cw = w_lo; cw < w_hi; cw += 32u) {  // warp-uniform trip count
            const uint32_t c = cw + lane;
            float lo[TM], hi[TM];
#pragma unroll
            for (uint32_t t = 0; t < TM; ++t) lo[t] = hi[t] = 0.f;
            uint32_t key = kNoRow, rows = 0;
            float *yrow = nullptr;
            if (c < w_hi && DF11_BOUNDS_OK(16u * (c + 1u) <= kBufBytes &&
                                           (uint64_t)base + 16ull * (c + 1u) <= g.d.n_elems && c >= c_lo &&
                                           16u * (c - c_lo + 1u) <= kBufBytes)) {
                const uint4 smv = lds_u4(sm_s + 16u * (c - c_lo));
                const uint4 ex = lds_u4(sb + 16u * c);
                sts_zero16(sb + 16u * c);
                const uint32_t g0 = base + 16u * c;
                while (mm < g.n_mats && g0 >= g.m[mm].end) ++mm;
                if (mm < g.n_mats && g0 >= g.m[mm].off) {
                    const GemvMat &M = g.m[mm];
                    uint32_t w[8];
                    merge16(smv, ex, w);
                    const uint32_t local = g0 - M.off;
                    const uint32_t row = gemv_row(local, M.magic, M.shift);
                    const uint16_t *xp = M.x + (local - row * M.cols);
#pragma unroll
                    for (uint32_t t = 0; t < TM; ++t) {
                        if (t < g.T) {
                            const uint4 *xv = reinterpret_cast<const uint4 *>(xp + (uint64_t)t * M.cols);
                            dot16(w, __ldg(xv), __ldg(xv + 1), lo[t], hi[t]);
                        }
                    }
                    // the key orders (matrix, row) pairs as the elements do
                    key = M.off / 16u + row;
                    rows = M.rows;
                    yrow = M.y + row;
                }
            }
            // (a lane's y row and row stride travel with its key)
            flush_any<TM>(lo, hi, key, yrow, rows, lane);
        }
    }

    // flush_runs for lanes whose runs may belong to different matrices: the
    // run's first lane adds with its own row pointer and stride.
    template <uint32_t TM2>
    __device__ __forceinline__ void flush_any(const float (&lo)[TM2], const float (&hi)[TM2], uint32_t key,
                                              float *yrow, uint32_t rows, uint32_t lane) {
        uint32_t same = 0;
#pragma unroll
        for (uint32_t k = 0; k < 5; ++k) {
            const uint32_t o = __shfl_down_sync(kFull, key, 1u << k);
            if (lane + (1u << k) < 32u && o == key) same |= 1u << k;
        }
        const uint32_t prev = __shfl_up_sync(kFull, key, 1);
        const bool first = (lane == 0 || prev != key) && key != kNoRow;
#pragma unroll
        for (uint32_t t = 0; t < TM2; ++t) {
            float v = lo[t] + hi[t];
#pragma unroll
            for (uint32_t k = 0; k < 5; ++k) {
                const float o = __shfl_down_sync(kFull, v, 1u << k);
                if (same & (1u << k)) v += o;
            }
            if (first && t < g.T) atomicAdd(yrow + (uint64_t)t * rows, v);
        }
    }

    // The block's two edge chunks (warp 0, converged): lanes 0..15 the first,
    // 16..31 the last, one element each; each half-warp's sum is added once
    // (a chunk lies in one row of one matrix or in none).
    __device__ __forceinline__ void edges(uint32_t sb, uint32_t base, uint32_t c_full, uint32_t span, uint32_t s,
                                          uint32_t e, uint32_t lane, uint32_t sm_s0) {
        const bool head = s != base;
        const bool tail = (span & 15u) != 0u && !(head && c_full == 0u);
        const uint32_t c = (lane < 16u) ? 0u : c_full;
        const bool mine = (lane < 16u) ? head : tail;
        const uint32_t gc = base + 16u * c;  // the chunk's first element
        uint32_t mm = 0;
        while (mm < g.n_mats && gc >= g.m[mm].end) ++mm;
        const bool in_mat = mine && mm < g.n_mats && gc >= g.m[mm].off;
        float p[TM];
#pragma unroll
        for (uint32_t t = 0; t < TM; ++t) p[t] = 0.f;
        uint32_t row = 0;
        if (in_mat) {
            const GemvMat &M = g.m[mm];
            row = gemv_row(gc - M.off, M.magic, M.shift);
            const uint32_t gel = gc + (lane & 15u);
            if (gel >= s && gel < e && DF11_BOUNDS_OK(gel - base < kMaxCodesPerBlock + 16u)) {
                const uint32_t sm8 = sm_byte(g.d.sm, sm_s0, gel, base);
                const uint32_t r = lds_u8(sb + (gel - base));
                const uint32_t hi8 = (sm8 & 0x80u) | (r & 0x7Fu);
                const uint32_t lo8 = (r & 0x80u) | (sm8 & 0x7Fu);
                const float wv = __uint_as_float((lo8 | (hi8 << 8)) << 16);
                const uint32_t col = (gel - M.off) - row * M.cols;
#pragma unroll
                for (uint32_t t = 0; t < TM; ++t)
                    if (t < g.T) p[t] = wv * __uint_as_float((uint32_t)__ldg(M.x + (uint64_t)t * M.cols + col) << 16);
            }
        }
#pragma unroll
        for (uint32_t t = 0; t < TM; ++t) {
#pragma unroll
            for (uint32_t d = 8; d >= 1; d >>= 1) p[t] += __shfl_xor_sync(kFull, p[t], d);
            if ((lane & 15u) == 0u && in_mat && t < g.T)
                atomicAdd(g.m[mm].y + (uint64_t)t * g.m[mm].rows + row, p[t]);
        }
        __syncwarp();
        if ((lane == 0u && head) || (lane == 16u && tail)) sts_zero16(sb + 16u * (lane == 0u ? 0u : c_full));
    }
};

// TM: the largest batch the instance handles (1, 2, or 4 for T = 3..4).
template <class C, bool kLong, uint32_t TM>
__global__ void __launch_bounds__(C::kCtaThreads, 1) df11_decode_gemv_kernel(const __grid_constant__ GemvArgs g) {
    // the format blocks that hold the matrices' elements (each warp finds them)
    // (probed first near the blocks the elements' positions suggest: blocks
    // hold about n_elems / n_blocks elements each)
    extern __shared__ __align__(128) uint8_t smem[];
    issue_tables<C>(g.d.lut, smem_addr(smem), threadIdx.x);  // in flight during the search
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t nb = g.d.n_blocks, ne = g.d.n_elems ? g.d.n_elems : 1u;
    const uint64_t h0 = (uint64_t)((double)g.e_first / (double)ne * (double)nb), h1 = (uint64_t)((double)g.e_last / (double)ne * (double)nb);
    const uint64_t b0 = find_block_near(g.d.bstart, nb, h0 > 16u ? h0 - 16u : 0u, g.e_first, lane);
    const uint64_t b1 = find_block_near(g.d.bstart, nb, h1 > 16u ? h1 - 16u : 0u, g.e_last, lane) + 1u;
    GemvSink<TM> sink{{}, g, 0u};
    decode_blocks<C, kLong>(g.d, sink, b0, b1, true);
}

// ------------------------------------------------- fused decode -> tcgen05 GEMM
// Decompressing each matrix right before its multiplication ("Decompression
// adaptee a l'inference GPU") taken to the tensor cores for batches T > 4:
// the decoder's merge writes the BF16 weights straight into shared-memory
// operand tiles of tcgen05.mma instead of global memory, so a block's weights
// never reach HBM (only the compressed arrays are read).
//
// The matrices must be encoded in tile order: a [rows, cols] matrix (rows a
// multiple of 128, cols of 64) as its 128 x 64 tiles, row tiles in order and
// the 64-column k-tiles of a row tile in order, each tile row-major (the
// format itself is unchanged; only the order of the elements is).  Then every
// k-tile is 8192 consecutive elements of the stream, and a range of k-tiles is
// a range of the stream.
//
// Work: the listed matrices' k-tiles, numbered in stream order, are split
// evenly over the CTAs.  A CTA decodes the format blocks covering its range
// (groups take them in turn, as in the decode kernel) and its decoder groups
// merge each block into a ring of 128 x 64 BF16 tiles in the UMMA layout
// (128-byte swizzle): element (r, c) of a tile at byte r * 128 + ((c / 8) XOR
// (r mod 8)) * 16 + (c mod 8) * 2.  Each group makes its stores visible to the
// async proxy, and after its next group barrier one thread counts the bytes
// into the tile's mbarrier (complete_tx; a tile completes at 16384 bytes).  One
// more warp consumes the tiles in order: one thread loads each k-tile's
// activations X [n_pad x 64] by TMA (no multicast) and issues four UMMAs
// (M = 128 rows of W, N = n_pad, K = 16) into an FP32 accumulator in tensor
// memory, then releases the tile slot with tcgen05.commit; at the end of a
// run of k-tiles of one row tile (a segment) four epilogue warps read the
// accumulator (two buffers, so the next segment's MMAs need not wait) and add
// it into Y with FP32 atomics.  Every wait is bounded; a timeout sets the
// error bit 0x20 and lets the CTA finish without further waits.
constexpr uint32_t kFusedMaxMats = 16;
constexpr uint32_t kTileElems = 8192;   // 128 rows x 64 columns
constexpr uint32_t kTileBytes = 16384;  // as BF16
static_assert(kTileBytes == 1u << 14, "slot offset >> 11 = slot index x 8 (mbarrier bytes)");
constexpr uint32_t kFusedErrTimeout = 0x20u;

struct FusedMat {
    uint32_t off;    // first element in the tensor (a multiple of 16)
    uint32_t end;    // off + rows * cols
    uint32_t kt;     // k-tiles per row tile: cols / 64
    uint32_t rows;   // out features (a multiple of 128)
    uint32_t tbase;  // number of k-tiles of the matrices before this one
    float *y;        // [T][rows] FP32, accumulated into
};

struct FusedArgs {
    DecodeArgs d;
    FusedMat m[kFusedMaxMats];  // ordered by offset, not overlapping
    uint32_t n_mats, T, n_pad;  // n_pad: T rounded up to 16 (UMMA N)
    uint32_t n_tiles;           // k-tiles of all listed matrices
    uint32_t ring, xring;       // W-tile and X-tile slots
    uint32_t look;              // X tiles are loaded `look` tiles ahead (xring - look >= 2 tiles back are reused)
    uint32_t tmem_cols;         // power of two >= 2 * n_pad
};

struct FusedMaps {
    CUtensorMap x[kFusedMaxMats];  // X_j [T, cols_j], box [n_pad, 64], 128-byte swizzle
};

// The shared-memory area after the decoder's: ring slots, barriers, flags.
struct FusedSmem {
    uint32_t wring, xring;  // 1024-aligned slot arrays
    uint32_t xbytes;        // bytes of one X slot
    uint32_t full0, empty0, xfull0, xempty0, accfull0, accempty0, final_bar;
    uint32_t tmem_slot, abort_flag, next_block, block_end;
    uint32_t plan0;  // per decoder group 32 bytes: the tiles of its current block (TileSink::plan)
};

__device__ __forceinline__ FusedSmem fused_layout(const FusedArgs &f, uint32_t dec_end) {
    FusedSmem L;
    L.wring = (dec_end + 1023u) & ~1023u;
    L.xbytes = f.n_pad * 128u;
    L.xring = L.wring + f.ring * kTileBytes;
    uint32_t b = L.xring + f.xring * L.xbytes;
    L.full0 = b;
    L.empty0 = b + 8u * f.ring;
    L.xfull0 = b + 16u * f.ring;
    L.xempty0 = L.xfull0 + 8u * f.xring;
    L.accfull0 = L.xempty0 + 8u * f.xring;
    L.accempty0 = L.accfull0 + 16u;
    L.final_bar = L.accempty0 + 16u;
    L.tmem_slot = L.final_bar + 8u;
    L.abort_flag = L.tmem_slot + 4u;
    L.next_block = L.abort_flag + 4u;  // the decoder groups' block counter
    L.block_end = L.next_block + 4u;   // and the end of the CTA's blocks
    L.plan0 = L.block_end + 4u;
    return L;
}

// Bounded wait that gives up, for good, once any wait of the CTA timed out or
// a block could not be placed (the CTA's abort flag, checked between probes).
// Each probe suspends the thread for up to `hint_ns` while the phase is
// incomplete (it resumes when the phase completes), so waiters leave the
// issue slots to the decoder warps instead of spinning; the number of probes
// bounds the wait at about two seconds even if no probe suspends for long.
__device__ __forceinline__ bool fused_wait(uint32_t bar, uint32_t parity, uint32_t abort_flag, uint32_t &err,
                                           uint32_t hint_ns) {
    const uint32_t rounds = 2000000000u / (hint_ns + 100u);
    for (uint32_t round = 0; round < rounds; ++round) {
        if (df11::tc::mbar_try_wait_hint(bar, parity, hint_ns)) return true;
        if (lds_u32(abort_flag)) return false;
    }
    err |= kFusedErrTimeout;
    sts_u32(abort_flag, 1u);
    return false;
}

// The number of listed k-tiles that start before stream element E (k-tiles
// are numbered in stream order; a matrix's tiles start at off + 8192 k).
__device__ __forceinline__ uint32_t tiles_before(const FusedArgs &f, uint64_t E) {
    for (uint32_t j = 0; j < f.n_mats; ++j) {
        const FusedMat &M = f.m[j];
        if (E <= M.off) return M.tbase;
        if (E < M.end) return M.tbase + (uint32_t)((E - M.off + kTileElems - 1u) / kTileElems);
    }
    return f.n_tiles;
}

// The k-tile at a global k-tile index: matrix, row tile and k-tile column.
struct TileAt {
    uint32_t j, rt, kt;
};
__device__ __forceinline__ TileAt tile_at(const FusedArgs &f, uint32_t K) {
    uint32_t j = 0;
    while (j + 1u < f.n_mats && K >= f.m[j + 1u].tbase) ++j;
    const uint32_t lk = K - f.m[j].tbase;
    return TileAt{j, lk / f.m[j].kt, lk % f.m[j].kt};
}

// Walks the k-tiles in stream order: matrix j, row tile rt, k-tile column kt
// (KT k-tiles per row tile, RT row tiles in matrix j).
struct TileCursor {
    uint32_t j, rt, kt, KT, RT;
    __device__ __forceinline__ void start(const FusedArgs &f, uint32_t K) {
        const TileAt a = tile_at(f, K);
        j = a.j;
        rt = a.rt;
        kt = a.kt;
        KT = f.m[j].kt;
        RT = f.m[j].rows / 128u;
    }
    __device__ __forceinline__ void next(const FusedArgs &f) {
        if (++kt < KT) return;
        kt = 0;
        if (++rt < RT) return;
        rt = 0;
        if (++j < f.n_mats) {
            KT = f.m[j].kt;
            RT = f.m[j].rows / 128u;
        }
    }
};

// The decoder side: the merge of a decoded block writes into the tile ring.
// kStaged: the block's sign/mantissa bytes are staged in shared memory (else
// read from global memory, prefetched into L2 while the block decodes).
// A block (at most 7152 elements) meets at most two k-tiles (8192 elements
// each, consecutive in the stream, 16-aligned) and each of them holds the
// block's first or last element; they are located once per block, so the
// per-chunk work is two range tests and two swizzled stores.
template <bool kStaged>
struct TileSink {
    static constexpr uint32_t kNoTile = 0xFFFFFFFFu;
    const FusedArgs &f;
    FusedSmem L;
    uint32_t K0, NT;     // this CTA's k-tiles [K0, K0 + NT)
    uint32_t avail;      // local tiles [0, avail) are known to have a free slot
    uint32_t ta, tb;     // the local tiles of the block's first and last elements (kNoTile: none)
    uint32_t ga, gb;     // the stream index of their first elements
    uint32_t sa, sb_;    // their slots' shared-memory addresses
    uint32_t ba, bb;     // bytes this thread wrote into them
    uint32_t err;

    // Local tile index of element g and its position in the tile; false if
    // g is in no listed matrix or in another CTA's tiles.
    __device__ __forceinline__ bool locate(uint32_t g, uint32_t &i, uint32_t &p) const {
        uint32_t mm = 0;
        while (mm < f.n_mats && g >= f.m[mm].end) ++mm;
        if (mm >= f.n_mats || g < f.m[mm].off) return false;
        const uint32_t q = g - f.m[mm].off;
        const uint32_t K = f.m[mm].tbase + q / kTileElems;
        if (K < K0 || K - K0 >= NT) return false;
        i = K - K0;
        p = q % kTileElems;
        return true;
    }
    // Waits until local tile i's slot no longer holds an unconsumed tile;
    // false once the CTA has aborted (then nothing more is written or counted:
    // a count that lands in a phase that never completes would push the tile
    // mbarrier's transaction count out of its range).
    __device__ __forceinline__ bool ensure(uint32_t i) {
        if (i < avail) return true;
        const uint32_t r = i / f.ring;
        if (r > 0u && !fused_wait(L.empty0 + 8u * (i % f.ring), (r - 1u) & 1u, L.abort_flag, err, 2000u))
            return false;
        avail = i + 1u;
        return true;
    }
    // The tile-complete mbarrier of the slot at shared-memory address `slot`.
    __device__ __forceinline__ uint32_t full_bar(uint32_t slot) const { return L.full0 + ((slot - L.wring) >> 11); }
    // Shared-memory address of position p (a multiple of 8: a 16-byte piece)
    // of the tile whose slot starts at `slot` (UMMA 128-byte swizzle).
    __device__ __forceinline__ static uint32_t piece(uint32_t slot, uint32_t p) {
        const uint32_t r = p >> 6, j = (p & 63u) >> 3;
        return slot + r * 128u + ((j ^ (r & 7u)) << 4);
    }
    // The tile holding element g (a chunk's first element): slot address and
    // position; false if g is in neither of the block's tiles.
    __device__ __forceinline__ bool which(uint32_t g, bool &in_a, uint32_t &slot, uint32_t &p) {
        in_a = ta != kNoTile && g - ga < kTileElems;
        if (in_a) {
            p = g - ga;
            slot = sa;
        } else if (tb != kNoTile && g - gb < kTileElems) {
            p = g - gb;
            slot = sb_;
        } else {
            return false;
        }
        return ensure(in_a ? ta : tb);
    }

    // Two threads of the group, after the scan barrier: the tiles of the
    // block's first element (thread 64) and last element (thread 96) into the
    // group's plan words (tile, first element, slot address), read by the
    // whole group after the next barrier.  (The previous block's plan was read
    // before its merge, which every thread finished before the scan barrier.)
    __device__ __forceinline__ void plan(uint32_t s, uint32_t e, uint32_t lt) {
        if (lt != 64u && lt != 96u) return;
        const uint32_t at = L.plan0 + 32u * (threadIdx.x / kGroupThreads) + (lt == 64u ? 0u : 12u);
        const uint32_t g = lt == 64u ? s : e - 1u;
        uint32_t i, p;
        if (e > s && locate(g, i, p)) {
            sts_u32(at, i);
            sts_u32(at + 4u, g - p);
            sts_u32(at + 8u, L.wring + (i % f.ring) * kTileBytes);
        } else {
            sts_u32(at, kNoTile);
        }
    }
    // Every thread of the group, before the block's merge.
    __device__ __forceinline__ void begin_block(uint32_t, uint32_t) {
        const uint32_t at = L.plan0 + 32u * (threadIdx.x / kGroupThreads);
        ba = bb = 0u;
        ta = lds_u32(at);
        ga = lds_u32(at + 4u);
        sa = lds_u32(at + 8u);
        tb = lds_u32(at + 12u);
        gb = lds_u32(at + 16u);
        sb_ = lds_u32(at + 20u);
        if (tb == ta) tb = kNoTile;
    }

    __device__ __forceinline__ void put16(const uint4 smv, const uint4 ex, uint32_t g) {
        bool in_a;
        uint32_t slot, p;
        if (!which(g, in_a, slot, p)) return;
        uint32_t o[8];
        merge16(smv, ex, o);
        // 16 weights = two 16-byte pieces of one tile row (p is a multiple of 16)
        sts_u4(piece(slot, p), o[0], o[1], o[2], o[3]);
        sts_u4(piece(slot, p + 8u), o[4], o[5], o[6], o[7]);
        if (in_a) ba += 32u;
        else bb += 32u;
    }

    template <uint32_t kBufBytes>
    __device__ __forceinline__ void chunks(uint32_t sbuf, uint32_t base, uint32_t c_first, uint32_t c_end,
                                           uint32_t sm_s, uint32_t c_lo) {
        if (kStaged) {
            for (uint32_t c = c_first; c < c_end; c += kGroupThreads) {
                if (!DF11_BOUNDS_OK(16u * (c + 1u) <= kBufBytes && c >= c_lo &&
                                    (uint64_t)base + 16u * (c + 1u) <= f.d.n_elems &&
                                    16u * (c - c_lo + 1u) <= kBufBytes))
                    continue;
                const uint4 smv = lds_u4(sm_s + 16u * (c - c_lo));
                const uint4 ex = lds_u4(sbuf + 16u * c);
                sts_zero16(sbuf + 16u * c);
                put16(smv, ex, base + 16u * c);
            }
        } else {
            // the thread's (at most four per round) 16-byte loads from global
            // memory are all issued before the first is used
            constexpr uint32_t kRound = 4;
            for (uint32_t c1 = c_first; c1 < c_end; c1 += kRound * kGroupThreads) {
                uint4 v[kRound];
#pragma unroll
                for (uint32_t q = 0; q < kRound; ++q) {
                    const uint32_t c = c1 + q * kGroupThreads;
                    if (c < c_end && DF11_BOUNDS_OK((uint64_t)base + 16u * (c + 1u) <= f.d.n_elems))
                        v[q] = __ldg(reinterpret_cast<const uint4 *>(f.d.sm + base + 16u * c));
                }
#pragma unroll
                for (uint32_t q = 0; q < kRound; ++q) {
                    const uint32_t c = c1 + q * kGroupThreads;
                    if (!(c < c_end) || !DF11_BOUNDS_OK(16u * (c + 1u) <= kBufBytes && c >= c_lo &&
                                                       (uint64_t)base + 16u * (c + 1u) <= f.d.n_elems))
                        continue;
                    const uint4 ex = lds_u4(sbuf + 16u * c);
                    sts_zero16(sbuf + 16u * c);
                    put16(v[q], ex, base + 16u * c);
                }
            }
        }
        // (the stores are made visible to the async proxy in block_done,
        // one fence per thread for the chunks and the edges together)
    }
    __device__ __forceinline__ void edges(uint32_t sbuf, uint32_t base, uint32_t c_full, uint32_t span, uint32_t s,
                                          uint32_t e, uint32_t lane, uint32_t sm_s0) {
        const bool head = s != base;
        const bool tail = (span & 15u) != 0u && !(head && c_full == 0u);
        const uint32_t c = (lane < 16u) ? 0u : c_full;
        const bool mine = (lane < 16u) ? head : tail;
        const uint32_t g = base + 16u * c + (lane & 15u);
        bool in_a;
        uint32_t slot, p;
        if (mine && g >= s && g < e && DF11_BOUNDS_OK(g - base < kMaxCodesPerBlock + 16u) &&
            which(g & ~15u, in_a, slot, p)) {
            const uint32_t sm8 = sm_byte(f.d.sm, sm_s0, g, base);
            const uint32_t rr = lds_u8(sbuf + (g - base));
            const uint32_t hi8 = (sm8 & 0x80u) | (rr & 0x7Fu);
            const uint32_t lo8 = (rr & 0x80u) | (sm8 & 0x7Fu);
            const uint32_t pe = p + (g & 15u);  // the element's own position (same row as the chunk's)
            const uint32_t r = pe >> 6, cc = pe & 63u;
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(slot + r * 128u + (((cc >> 3) ^ (r & 7u)) << 4) +
                                                         (cc & 7u) * 2u),
                         "h"((uint16_t)(lo8 | (hi8 << 8)))
                         : "memory");
            if (in_a) ba += 2u;
            else bb += 2u;
        }
        __syncwarp();  // every lane has read the edge chunks before they are cleared
        if ((lane == 0u && head) || (lane == 16u && tail)) sts_zero16(sbuf + 16u * (lane == 0u ? 0u : c_full));
    }
    // After the block's merge (every thread of the group): each warp counts
    // the bytes it wrote into the tiles' mbarriers right away (lane 0; the
    // writers' stores were made visible to the async proxy, the warp sync
    // gathers them, and the fence orders them before the relaxed count).  A
    // block that failed its checks wrote nothing but still counts its range,
    // so its tiles complete and the CTA finishes (the error word says the
    // product is garbage); a block whose range cannot even be placed aborts the
    // CTA's waits instead.
    __device__ __forceinline__ void block_done(uint32_t s, uint32_t e, bool ok, bool range_ok) {
        const uint32_t lane = threadIdx.x & 31u;
        if (!range_ok) {
            if ((threadIdx.x % kGroupThreads) == 0u) sts_u32(L.abort_flag, 1u);
            return;
        }
        if (ok) {
            // this thread's tile stores (chunks and edges) become visible to
            // the tensor cores' async proxy; the warp sync gathers them
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            const uint32_t a = __reduce_add_sync(0xFFFFFFFFu, ba), b = __reduce_add_sync(0xFFFFFFFFu, bb);
            if (lane == 0u && (a | b) != 0u && !lds_u32(L.abort_flag)) {
                asm volatile("fence.acq_rel.cta;" ::: "memory");
                if (a) df11::tc::mbar_complete_tx(full_bar(sa), a);
                if (b) df11::tc::mbar_complete_tx(full_bar(sb_), b);
            }
        } else if ((threadIdx.x % kGroupThreads) == 0u && e > s) {
            for (uint32_t q = 0; q < 2u; ++q) {
                const uint32_t i = q == 0u ? ta : tb;
                if (i == kNoTile || !ensure(i)) continue;  // the count must land in this round of the slot
                const uint32_t ts = q == 0u ? ga : gb, te = ts + kTileElems;
                const uint32_t lo = s > ts ? s : ts, hi = e < te ? e : te;
                if (lds_u32(L.abort_flag)) break;
                asm volatile("fence.acq_rel.cta;" ::: "memory");
                df11::tc::mbar_complete_tx(full_bar(q == 0u ? sa : sb_), 2u * (hi - lo));
            }
        }
    }
    __device__ __forceinline__ void published(uint32_t) {}
    __device__ __forceinline__ void finish(uint32_t, uint32_t) {}
};

// four epilogue warps (a warp reads the TMEM lanes of its rank in its
// warpgroup; the decoder threads are a multiple of 128, so the four are one
// warpgroup) and the MMA warp, which never reads TMEM itself (a variant whose
// MMA warp also drained a quarter of the accumulators stopped completing
// MMAs on B200: every wait then ran into its limit)
constexpr uint32_t kFusedExtraThreads = 160;

// One warp's share of a finished segment (the k-tiles of row tile rt of
// matrix j, accumulated in buffer seg & 1): TMEM lanes 32 q .. 32 q + 31 are
// rows rt * 128 + 32 q + lane, added into Y with FP32 atomics; then the warp
// arrives on the buffer's accempty barrier.  The wait for the segment is
// bounded; after an abort the accumulators are read but nothing is added.
__device__ __forceinline__ void drain_segment(const FusedArgs &f, const FusedSmem &L, uint32_t tmem, uint32_t j,
                                              uint32_t rt, uint32_t seg, uint32_t q, uint32_t &err) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t abuf = seg & 1u;
    // (every lane waits; the warp is converged again before the
    // .sync.aligned loads)
    const bool have = fused_wait(L.accfull0 + 8u * abuf, (seg >> 1) & 1u, L.abort_flag, err, 20000u);
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const FusedMat &M = f.m[j];
    const uint32_t row = rt * 128u + q * 32u + lane;
    for (uint32_t c0 = 0; c0 < f.n_pad; c0 += 16u) {
        uint32_t v[16];
        df11::tc::tmem_ld16(tmem + ((q * 32u) << 16) + abuf * f.n_pad + c0, v);
        if (have) {
#pragma unroll
            for (uint32_t k = 0; k < 16u; ++k)
                if (c0 + k < f.T) atomicAdd(M.y + (uint64_t)(c0 + k) * M.rows + row, __uint_as_float(v[k]));
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncwarp();
    if (lane == 0u) df11::tc::mbar_arrive(L.accempty0 + 8u * abuf);
}

template <class C, bool kLong>
__global__ void __launch_bounds__(C::kCtaThreads + kFusedExtraThreads, 1)
    df11_decode_gemm_kernel(const __grid_constant__ FusedArgs f, const __grid_constant__ FusedMaps maps) {
    extern __shared__ __align__(128) uint8_t smem[];  // the tile rings are aligned to 1024 by hand
    const uint32_t s_base = smem_addr(smem);
    const uint32_t tid = threadIdx.x;
    constexpr uint32_t kDec = C::kCtaThreads;  // decoder threads; then 4 epilogue warps and the MMA warp
    static_assert(C::kGroups <= 6u, "the shared-memory tail holds six groups' tile plans");
    const FusedSmem L = fused_layout(f, s_base + C::kSmemBytes);
    // The work split follows the decoding, the larger share of the work: CTA
    // c takes the format blocks [Bc, Bn) = the c-th of gridDim.x equal shares
    // and owns the k-tiles that start inside their elements [Ec, En) (the
    // elements per block vary with the matrices' statistics, so equal tile
    // shares would not be equal decode work).  Valid block starts increase,
    // so the shares partition the tiles; a CTA whose boundaries are out of
    // order reports it (the product is then incomplete).
    const uint64_t nbk = f.d.n_blocks;
    const uint64_t Bc = nbk * blockIdx.x / gridDim.x, Bn = nbk * (blockIdx.x + 1u) / gridDim.x;
    const uint64_t Ec = blockIdx.x == 0u ? 0u : (uint64_t)__ldg(f.d.bstart + Bc);
    const uint64_t En = blockIdx.x + 1u == gridDim.x ? ~0ull : (uint64_t)__ldg(f.d.bstart + Bn);
    const uint32_t K0 = tiles_before(f, Ec), K1 = tiles_before(f, En);
    if (K1 <= K0) {  // uniform over the CTA
        if (K1 < K0 && tid == 0u && f.d.err) atomicOr(f.d.err, (uint32_t)DF11_KERR_BAD_BLOCK);
        return;
    }
    const uint32_t NT = K1 - K0;
    uint32_t err = 0;

    issue_tables<C>(f.d.lut, s_base, tid);  // in flight during the search
    // warp 0: the format blocks covering the elements of k-tiles [K0, K1),
    // searched near the share's ends
    if (tid < 32u) {
        const TileAt a0 = tile_at(f, K0), a1 = tile_at(f, K1 - 1u);
        const FusedMat &m0 = f.m[a0.j], &m1 = f.m[a1.j];
        const uint64_t e_first = m0.off + (uint64_t)(K0 - m0.tbase) * kTileElems;
        const uint64_t e_last = m1.off + (uint64_t)(K1 - m1.tbase) * kTileElems - 1u;
        const uint64_t b0 = find_block_near(f.d.bstart, nbk, Bc, e_first, tid);
        const uint64_t b1 = find_block_near(f.d.bstart, nbk, Bn > 0u ? Bn - 1u : 0u, e_last, tid) + 1u;
        if (tid == 0u) {
            sts_u32(L.next_block, (uint32_t)b0);  // n_blocks < 2^32 (n_elems < 2^32)
            sts_u32(L.block_end, (uint32_t)b1);
        }
    }
    if (!finish_tables<C>(f.d.lut, f.d.err, smem, s_base, tid)) return;  // uniform over the CTA
    if (tid == 0) {
        for (uint32_t s = 0; s < f.ring; ++s) {
            df11::tc::mbar_init(L.full0 + 8u * s, 1);
            df11::tc::mbar_init(L.empty0 + 8u * s, 1);
        }
        for (uint32_t s = 0; s < f.xring; ++s) {
            df11::tc::mbar_init(L.xfull0 + 8u * s, 1);
            df11::tc::mbar_init(L.xempty0 + 8u * s, 1);
        }
        for (uint32_t a = 0; a < 2u; ++a) {
            df11::tc::mbar_init(L.accfull0 + 8u * a, 1);
            df11::tc::mbar_init(L.accempty0 + 8u * a, 4);  // one arrival per draining warp
        }
        df11::tc::mbar_init(L.final_bar, 1);
        sts_u32(L.abort_flag, 0u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid >= kDec && tid < kDec + 32u) {  // the first epilogue warp allocates the accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(L.tmem_slot),
                     "r"(f.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = lds_u32(L.tmem_slot);

    if (tid < kDec) {
        // ---- decoders: the CTA's blocks, taken in order from the counter
        // (tiles are consumed in order, so a group that ran ahead would only
        // wait for a slot; a free group takes the next block instead)
        TileSink<C::kStageSm> sink{f, L, K0, NT, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // (tiles set per block)
        decode_loop<C, kLong>(f.d, sink, 0u, 1u, lds_u32(L.block_end), L.next_block);
        err |= sink.err;
    } else if (tid < kDec + 128u) {
        // ---- epilogue warps 0..3: TMEM lanes 32 q .. 32 q + 31 of each segment
        const uint32_t q = (tid - kDec) >> 5;
        uint32_t seg = 0;
        TileCursor ce;  // the first k-tile of each segment
        ce.start(f, K0);
        for (uint32_t i = 0; i < NT;) {
            const uint32_t n = min(ce.KT - ce.kt, NT - i);  // the segment's k-tiles
            const uint32_t j = ce.j, rt = ce.rt;
            i += n;
            ce.kt += n - 1u;
            ce.next(f);
            drain_segment(f, L, tmem, j, rt, seg, q, err);
            ++seg;
        }
    } else {
        // ---- the MMA warp: one thread loads X and issues the MMAs (the
        // others wait at the end; a loop run by the whole warp with one lane
        // doing the work measured slower)
        if ((tid & 31u) == 0u) {
            const uint32_t idesc = df11::tc::instr_desc_bf16(f.n_pad, 128u);
            // descriptors of slot 0; a slot (and a K = 16 step, 32 bytes along
            // the swizzled row) adds its byte offset / 16 to the address field
            const uint64_t dw0 = df11::tc::smem_desc_sw128(L.wring), dx0 = df11::tc::smem_desc_sw128(L.xring);
            // X tile of the next local k-tile to load (its slot and the slot's
            // round), walked by its own cursor
            TileCursor cx;
            cx.start(f, K0);
            uint32_t xl_slot = 0, xl_round = 0;
            auto load_x = [&]() {
                if (xl_round == 0u ||
                    fused_wait(L.xempty0 + 8u * xl_slot, (xl_round - 1u) & 1u, L.abort_flag, err, 2000u)) {
                    df11::tc::mbar_arrive_expect_tx(L.xfull0 + 8u * xl_slot, L.xbytes);
                    df11::tc::tma_load_2d(L.xring + xl_slot * L.xbytes, &maps.x[cx.j], L.xfull0 + 8u * xl_slot,
                                          (int32_t)(cx.kt * 64u), 0);
                }
                cx.next(f);
                if (++xl_slot == f.xring) {
                    xl_slot = 0;
                    ++xl_round;
                }
            };
            // X tiles are loaded `look` tiles ahead, each into the slot of the
            // tile xring - look before the current one: its MMA has had that
            // many tiles' time to finish (waiting on the MMA of the tile just
            // before would tie the loop to the MMAs' latency)
            const uint32_t look = f.look;
            for (uint32_t i = 0; i < look && i < NT; ++i) load_x();
            TileCursor ct;
            ct.start(f, K0);
            uint32_t seg = 0;          // segments started
            uint32_t s = 0, sph = 0;   // W slot of tile i and the parity of its round
            uint32_t xs = 0, xph = 0;  // X slot of tile i and the parity of its round
            for (uint32_t i = 0; i < NT; ++i) {
                // once aborted, arm no more phases (a second arrival on a phase
                // that never completed is not allowed)
                if (lds_u32(L.abort_flag)) break;
                if (i + look < NT) load_x();
                const bool first = (i == 0u) || ct.kt == 0u;
                const bool last = (i + 1u == NT) || ct.kt + 1u == ct.KT;
                const uint32_t abuf = seg & 1u;
                // the accumulator buffer's previous segment has been drained
                if (first && seg >= 2u)
                    fused_wait(L.accempty0 + 8u * abuf, ((seg >> 1) - 1u) & 1u, L.abort_flag, err, 2000u);
                df11::tc::mbar_arrive_expect_tx(L.full0 + 8u * s, kTileBytes);  // this round's tile
                const bool ok = fused_wait(L.full0 + 8u * s, sph, L.abort_flag, err, 2000u) &&
                                fused_wait(L.xfull0 + 8u * xs, xph, L.abort_flag, err, 2000u);
                if (ok) {
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint64_t dw = dw0 + ((s * kTileBytes) >> 4), dx = dx0 + ((xs * L.xbytes) >> 4);
#pragma unroll
                    for (uint32_t kk = 0; kk < 4u; ++kk)
                        df11::tc::umma_bf16(tmem + abuf * f.n_pad, dw + 2u * kk, dx + 2u * kk, idesc,
                                            (first && kk == 0u) ? 0u : 1u);
                }
                df11::tc::umma_commit(L.empty0 + 8u * s);
                df11::tc::umma_commit(L.xempty0 + 8u * xs);
                if (last) {
                    df11::tc::umma_commit(L.accfull0 + 8u * abuf);
                    ++seg;
                }
                ct.next(f);
                if (++s == f.ring) {
                    s = 0;
                    sph ^= 1u;
                }
                if (++xs == f.xring) {
                    xs = 0;
                    xph ^= 1u;
                }
            }
            // every issued MMA has completed before the accumulators are freed
            // (not skipped on abort: issued MMAs finish on their own)
            df11::tc::umma_commit(L.final_bar);
            if (!df11::tc::mbar_wait(L.final_bar, 0u)) err |= kFusedErrTimeout;
        }
        __syncwarp();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid >= kDec && tid < kDec + 32u) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(f.tmem_cols)
                     : "memory");
    }
    if (err && f.d.err) atomicOr(f.d.err, err);
}

// ----------------------------------------------------------------- host
std::atomic<int> g_sm_count[64];
std::atomic<int> g_attr_set[64];

template <class C, bool kLong>
cudaError_t set_smem_attr() {
    const cudaFuncAttribute kAttr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(df11_decode_kernel<C, kLong>, kAttr, (int)C::kSmemBytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(df11_gather_kernel<C, kLong>, kAttr, (int)C::kSmemBytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(df11_decode_gemv_kernel<C, kLong, 1>, kAttr, (int)C::kSmemBytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(df11_decode_gemv_kernel<C, kLong, 2>, kAttr, (int)C::kSmemBytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(df11_decode_gemv_kernel<C, kLong, 4>, kAttr, (int)C::kSmemBytes);
    return e;
}

df11_status prepare_device(int *sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
    if (dev < 0 || dev >= 64) return DF11_ERR_UNSUPPORTED;
    int sms = g_sm_count[dev].load(std::memory_order_relaxed);
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
    }
    if (!g_attr_set[dev].load(std::memory_order_acquire)) {
        if (set_smem_attr<CfgTypical, false>() != cudaSuccess || set_smem_attr<CfgTypical, true>() != cudaSuccess ||
            set_smem_attr<CfgWide, false>() != cudaSuccess || set_smem_attr<CfgWide, true>() != cudaSuccess ||
            set_smem_attr<CfgDense, false>() != cudaSuccess || set_smem_attr<CfgDense, true>() != cudaSuccess ||
            set_smem_attr<CfgTypicalC, false>() != cudaSuccess || set_smem_attr<CfgTypicalC, true>() != cudaSuccess ||
            set_smem_attr<CfgWideC, false>() != cudaSuccess || set_smem_attr<CfgWideC, true>() != cudaSuccess ||
            set_smem_attr<CfgDenseC, false>() != cudaSuccess || set_smem_attr<CfgDenseC, true>() != cudaSuccess)
            return DF11_ERR_CUDA;
        g_attr_set[dev].store(1, std::memory_order_release);
    }
    *sm_count = sms;
    return DF11_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

template <class C, bool kLong>
void launch(const DecodeArgs &a, uint64_t n_blocks, int sms, cudaStream_t stream) {
    // one CTA per SM, or one per block when there are fewer blocks
    const unsigned grid = (unsigned)(n_blocks < (uint64_t)sms ? (n_blocks ? n_blocks : 1u) : (uint64_t)sms);
    df11_decode_kernel<C, kLong><<<grid, C::kCtaThreads, C::kSmemBytes, stream>>>(a);
}

struct DecodeLaunch {
    const DecodeArgs &a;
    uint64_t n_blocks;
    int sms;
    cudaStream_t s;
    template <class C, bool kLong>
    void go() { launch<C, kLong>(a, n_blocks, sms, s); }
};

// Checks a device tensor for a decode launch and fills the kernel arguments.
df11_status prepare_args(const df11_tensor *t, DecodeArgs &a) {
    if (!t->enc || !t->sm || !t->gaps || !t->block_start || !t->lut) return DF11_ERR_INVALID_ARG;
    if (!aligned16(t->enc) || !aligned16(t->sm) || !aligned16(t->gaps) || !aligned16(t->lut) ||
        !aligned16(t->block_start) || !aligned16(t->counts))
        return DF11_ERR_INVALID_ARG;
    a.enc = t->enc;
    a.counts = t->counts;  // NULL: the kernel runs the count pass
    a.sm = t->sm;
    a.gaps = t->gaps;
    a.bstart = t->block_start;
    a.lut = t->lut;
    a.out = nullptr;
    a.err = nullptr;
    a.n_elems = t->n_elems;
    a.total_bits = t->total_bits;
    a.n_threads = t->n_threads;
    a.n_blocks = t->n_blocks;
    a.out_al32 = 0;
    return DF11_OK;
}

// Which instance decodes a tensor: codes no longer than both table windows
// never take the long-code path; a block's buffer span is at most its code
// count + 15, and the instance with the smallest buffers that holds it is
// taken (smaller buffers leave room for a second symbol-table copy); a
// tensor with stored per-thread counts takes the instances without the
// count pass.
enum class Inst { kTypical, kWide, kDense, kTypicalC, kWideC, kDenseC };
void pick_instance(const df11_tensor *t, Inst &inst, bool &lng) {
    uint32_t max_len = 0;
    for (int k = 0; k < 256; ++k) max_len = t->code_len[k] > max_len ? t->code_len[k] : max_len;
    lng = max_len > (uint32_t)(kW1Max < kW2Max ? kW1Max : kW2Max);
    const uint64_t need = (uint64_t)t->max_block_codes + 15u;
    if (t->counts)
        inst = need <= CfgTypicalC::kBufSyms ? Inst::kTypicalC : need <= CfgWideC::kBufSyms ? Inst::kWideC
                                                                                          : Inst::kDenseC;
    else
        inst = need <= CfgTypical::kBufSyms ? Inst::kTypical : need <= CfgWide::kBufSyms ? Inst::kWide
                                                                                       : Inst::kDense;
}

// Calls f.go<C, kLong>() for the picked instance.
template <class F>
void dispatch(Inst inst, bool lng, F f) {
    switch (inst) {
        case Inst::kTypical: lng ? f.template go<CfgTypical, true>() : f.template go<CfgTypical, false>(); break;
        case Inst::kWide: lng ? f.template go<CfgWide, true>() : f.template go<CfgWide, false>(); break;
        case Inst::kDense: lng ? f.template go<CfgDense, true>() : f.template go<CfgDense, false>(); break;
        case Inst::kTypicalC: lng ? f.template go<CfgTypicalC, true>() : f.template go<CfgTypicalC, false>(); break;
        case Inst::kWideC: lng ? f.template go<CfgWideC, true>() : f.template go<CfgWideC, false>(); break;
        case Inst::kDenseC: lng ? f.template go<CfgDenseC, true>() : f.template go<CfgDenseC, false>(); break;
    }
}

df11_status launch_decode(const df11_tensor *t, uint16_t *out, uint32_t *err_word, void *stream) {
    if (!t) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (t->n_elems == 0) return DF11_OK;  // nothing to write; out may be NULL
    if (!out || !aligned16(out)) return DF11_ERR_INVALID_ARG;
    DecodeArgs a;
    st = prepare_args(t, a);
    if (st != DF11_OK) return st;
    int sms = 0;
    st = prepare_device(&sms);
    if (st != DF11_OK) return st;
    a.out = out;
    a.err = err_word;
    a.out_al32 = ((uintptr_t)out & 31u) == 0 ? 1u : 0u;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Inst inst;
    bool lng;
    pick_instance(t, inst, lng);
    dispatch(inst, lng, DecodeLaunch{a, t->n_blocks, sms, s});
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}

template <class C, bool kLong>
void launch_gather(const GatherArgs &g, int sms, cudaStream_t stream) {
    const uint64_t ctas_needed = (g.n_rows + C::kGroups - 1) / C::kGroups;
    const unsigned grid = (unsigned)(ctas_needed < (uint64_t)sms ? ctas_needed : (uint64_t)sms);
    df11_gather_kernel<C, kLong><<<grid, C::kCtaThreads, C::kSmemBytes, stream>>>(g);
}

struct GatherLaunch {
    const GatherArgs &g;
    int sms;
    cudaStream_t s;
    template <class C, bool kLong>
    void go() { launch_gather<C, kLong>(g, sms, s); }
};

df11_status launch_rows(const df11_tensor *t, uint64_t row_len, const uint32_t *rows, uint32_t n_rows, uint16_t *out,
                        uint32_t *err_word, void *stream) {
    if (!t) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (row_len == 0 || t->n_elems % row_len != 0) return DF11_ERR_INVALID_ARG;
    if (n_rows == 0) return DF11_OK;
    if (!rows || !out || ((uintptr_t)out & 1u) || ((uintptr_t)rows & 3u) || t->n_elems == 0)
        return DF11_ERR_INVALID_ARG;
    GatherArgs g;
    st = prepare_args(t, g.d);
    if (st != DF11_OK) return st;
    int sms = 0;
    st = prepare_device(&sms);
    if (st != DF11_OK) return st;
    g.d.err = err_word;
    g.rows = rows;
    g.out = out;
    g.row_len = row_len;
    g.n_rows_total = t->n_elems / row_len;
    g.n_rows = n_rows;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Inst inst;
    bool lng;
    pick_instance(t, inst, lng);
    dispatch(inst, lng, GatherLaunch{g, sms, s});
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}

template <class C, bool kLong, uint32_t TM>
void launch_gemv_inst(const GemvArgs &g, uint64_t blocks_est, int sms, cudaStream_t stream) {
    const unsigned grid = (unsigned)(blocks_est < (uint64_t)sms ? (blocks_est ? blocks_est : 1u) : (uint64_t)sms);
    df11_decode_gemv_kernel<C, kLong, TM><<<grid, C::kCtaThreads, C::kSmemBytes, stream>>>(g);
}

template <uint32_t TM>
struct GemvLaunch {
    const GemvArgs &g;
    uint64_t blocks_est;
    int sms;
    cudaStream_t s;
    template <class C, bool kLong>
    void go() { launch_gemv_inst<C, kLong, TM>(g, blocks_est, sms, s); }
};

template <uint32_t TM>
void launch_gemv_tm(const GemvArgs &g, Inst inst, bool lng, uint64_t blocks_est, int sms, cudaStream_t s) {
    dispatch(inst, lng, GemvLaunch<TM>{g, blocks_est, sms, s});
}

// Multiply-shift division by d (1 <= d < 2^28) for dividends q < 2^28: with
// l = ceil(log2 d), shift = 28 + l and magic = ceil(2^shift / d) (< 2^29),
// the error magic * d - 2^shift is below d <= 2^l, so q times it stays below
// 2^shift and floor(q * magic / 2^shift) = floor(q / d) (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994).
void div_magic(uint32_t d, uint32_t &magic, uint32_t &shift) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    shift = 28u + l;
    magic = (uint32_t)(((1ull << shift) + d - 1u) / d);
}

df11_status launch_gemv(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                        uint32_t *err_word, void *stream) {
    if (!t) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (n_mats == 0) return DF11_OK;
    if (!mats) return DF11_ERR_INVALID_ARG;
    if (n_mats > kMaxGemvMats || T < 1u || T > 4u) return DF11_ERR_UNSUPPORTED;
    GemvArgs g;
    st = prepare_args(t, g.d);
    if (st != DF11_OK) return st;
    uint64_t prev_end = 0;
    for (uint32_t j = 0; j < n_mats; ++j) {
        const df11_gemv_mat &mj = mats[j];
        if (mj.rows == 0 || mj.cols == 0 || (mj.cols & 15u) || (mj.elem_offset & 15u) || !mj.x || !mj.y ||
            !aligned16(mj.x) || ((uintptr_t)mj.y & 3u))
            return DF11_ERR_INVALID_ARG;
        const uint64_t size = (uint64_t)mj.rows * mj.cols;
        if (mj.elem_offset < prev_end || mj.elem_offset > t->n_elems || size > t->n_elems - mj.elem_offset)
            return DF11_ERR_INVALID_ARG;
        GemvMat &M = g.m[j];
        M.off = (uint32_t)mj.elem_offset;  // n_elems < 2^32 (df11_validate)
        M.end = (uint32_t)(mj.elem_offset + size);
        M.x = mj.x;
        M.y = mj.y;
        M.rows = mj.rows;
        M.cols = mj.cols;
        div_magic(mj.cols / 16u, M.magic, M.shift);
        prev_end = mj.elem_offset + size;
    }
    for (uint32_t j = n_mats; j < kMaxGemvMats; ++j) g.m[j] = GemvMat{};
    g.n_mats = n_mats;
    g.T = T;
    g.e_first = g.m[0].off;
    g.e_last = g.m[n_mats - 1].end - 1u;
    g.d.err = err_word;
    int sms = 0;
    st = prepare_device(&sms);
    if (st != DF11_OK) return st;
    // blocks the matrices span, estimated from the mean block size (the
    // persistent CTAs stride over the exact range the kernel finds)
    const uint64_t span = (uint64_t)g.e_last + 1u - g.e_first;
    const uint64_t blocks_est =
        (uint64_t)((double)span * (double)t->n_blocks / (double)t->n_elems) + 2u;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Inst inst;
    bool lng;
    pick_instance(t, inst, lng);
    if (T == 1u) launch_gemv_tm<1>(g, inst, lng, blocks_est, sms, s);
    else if (T == 2u) launch_gemv_tm<2>(g, inst, lng, blocks_est, sms, s);
    else launch_gemv_tm<4>(g, inst, lng, blocks_est, sms, s);
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}

// ---- fused decode -> GEMM launcher
constexpr uint32_t kSmemLimit = 227u * 1024u;
// alignment slack of the rings (1024), barriers and flags (at most 276 bytes)
// and the decoder groups' tile plans (32 bytes per group)
constexpr uint32_t kFusedTail = 1024u + 512u;
static_assert(16u * 8u + 16u * 6u + 56u + 6u * 32u <= 512u, "ring <= 8, xring <= 6, <= 6 groups");

// Shared memory of an instance with `xring` X slots: true if at least
// `min_ring` operand-tile slots fit (then as many as fit, at most 8).
template <class C>
bool fused_fit(uint32_t n_pad, uint32_t xring, uint32_t min_ring, uint32_t &ring, uint32_t &smem) {
    const uint32_t xbytes = 128u * n_pad;
    if (C::kSmemBytes + kFusedTail + xring * xbytes + min_ring * kTileBytes > kSmemLimit) return false;
    ring = (kSmemLimit - C::kSmemBytes - kFusedTail - xring * xbytes) / kTileBytes;
    if (ring > 8u) ring = 8u;
    smem = C::kSmemBytes + kFusedTail + xring * xbytes + ring * kTileBytes;
    return true;
}

template <class C, bool kLong>
cudaError_t fused_launch(const FusedArgs &f, const FusedMaps &maps, uint32_t smem, unsigned grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(df11_decode_gemm_kernel<C, kLong>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    df11_decode_gemm_kernel<C, kLong><<<grid, C::kCtaThreads + kFusedExtraThreads, smem, s>>>(f, maps);
    return cudaGetLastError();
}

df11_status launch_fused(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                         uint32_t *err_word, void *stream) {
    if (!t) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (n_mats == 0) return DF11_OK;
    if (!mats) return DF11_ERR_INVALID_ARG;
    if (n_mats > kFusedMaxMats || T < 1u || T > 256u || !t->counts) return DF11_ERR_UNSUPPORTED;
    FusedArgs f;
    st = prepare_args(t, f.d);
    if (st != DF11_OK) return st;
    Inst inst;
    bool lng;
    pick_instance(t, inst, lng);
    if (inst != Inst::kTypicalC) return DF11_ERR_UNSUPPORTED;  // blocks larger than the fused kernel's buffers
    uint64_t prev_end = 0, tiles = 0;
    for (uint32_t j = 0; j < n_mats; ++j) {
        const df11_gemv_mat &mj = mats[j];
        if (mj.rows == 0 || mj.cols == 0 || !mj.x || !mj.y || !aligned16(mj.x) || ((uintptr_t)mj.y & 3u) ||
            (mj.elem_offset & 15u))
            return DF11_ERR_INVALID_ARG;
        if (mj.rows % 128u || mj.cols % 64u) return DF11_ERR_UNSUPPORTED;
        const uint64_t size = (uint64_t)mj.rows * mj.cols;
        if (mj.elem_offset < prev_end || mj.elem_offset > t->n_elems || size > t->n_elems - mj.elem_offset)
            return DF11_ERR_INVALID_ARG;
        FusedMat &M = f.m[j];
        M.off = (uint32_t)mj.elem_offset;  // n_elems < 2^32 (df11_validate)
        M.end = (uint32_t)(mj.elem_offset + size);
        M.kt = mj.cols / 64u;
        M.rows = mj.rows;
        M.tbase = (uint32_t)tiles;
        M.y = mj.y;
        tiles += size / kTileElems;
        prev_end = mj.elem_offset + size;
    }
    for (uint32_t j = n_mats; j < kFusedMaxMats; ++j) f.m[j] = FusedMat{};
    f.n_mats = n_mats;
    f.T = T;
    f.n_pad = (T + 15u) & ~15u;
    f.n_tiles = (uint32_t)tiles;
    f.tmem_cols = 32u;
    while (f.tmem_cols < 2u * f.n_pad) f.tmem_cols <<= 1;
    f.d.err = err_word;
    FusedMaps maps;
    for (uint32_t j = 0; j < n_mats; ++j)
        if (!df11::tc::make_bf16_tile_map(&maps.x[j], mats[j].x, T, mats[j].cols, f.n_pad)) return DF11_ERR_CUDA;
    for (uint32_t j = n_mats; j < kFusedMaxMats; ++j) maps.x[j] = maps.x[0];
    int sms = 0;
    st = prepare_device(&sms);
    if (st != DF11_OK) return st;
    const unsigned grid = (unsigned)(f.n_tiles < (uint32_t)sms ? f.n_tiles : (uint32_t)sms);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t smem = 0;
    cudaError_t e;
    // Prefer six X slots (loads 3 tiles ahead, slots reused 3 tiles later),
    // then the most decode groups (staging the sign/mantissa bytes if there is
    // room) whose ring still holds 4 operand tiles; with the largest X tiles,
    // four unstaged groups and fewer X slots.  (Seven groups do not fit: with
    // the five warps of the MMA side they pass 1024 threads.)
#ifndef DF11_FUSED_CFG
#define DF11_FUSED_CFG 0  // 0: by the rule above; 1..4: 6 staged, 6 unstaged, 4 staged, 4 unstaged groups
#endif
    const int forced = DF11_FUSED_CFG;
    f.xring = 6u;
    f.look = 3u;
    if ((forced == 0 || forced == 1) && fused_fit<CfgFused6>(f.n_pad, f.xring, forced ? 2u : 4u, f.ring, smem)) {
        e = lng ? fused_launch<CfgFused6, true>(f, maps, smem, grid, s)
                : fused_launch<CfgFused6, false>(f, maps, smem, grid, s);
    } else if ((forced == 0 || forced == 2) &&
               fused_fit<CfgFused6U>(f.n_pad, f.xring, forced ? 2u : 4u, f.ring, smem)) {
        e = lng ? fused_launch<CfgFused6U, true>(f, maps, smem, grid, s)
                : fused_launch<CfgFused6U, false>(f, maps, smem, grid, s);
    } else if ((forced == 0 || forced == 3) &&
               fused_fit<CfgFused4>(f.n_pad, f.xring, forced ? 2u : 4u, f.ring, smem)) {
        e = lng ? fused_launch<CfgFused4, true>(f, maps, smem, grid, s)
                : fused_launch<CfgFused4, false>(f, maps, smem, grid, s);
    } else {
        // four unstaged groups; fewer X slots until a ring of 3 fits
        bool fit = false;
        for (f.xring = 6u; f.xring >= 3u && !fit; --f.xring)
            fit = fused_fit<CfgFused4U>(f.n_pad, f.xring, 3u, f.ring, smem);
        if (!fit) return DF11_ERR_UNSUPPORTED;
        ++f.xring;  // (the loop stepped past the one that fit)
        f.look = f.xring / 2u;
        e = lng ? fused_launch<CfgFused4U, true>(f, maps, smem, grid, s)
                : fused_launch<CfgFused4U, false>(f, maps, smem, grid, s);
    }
    return e == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

}  // namespace

extern "C" {

df11_status df11_decode_gemm(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                             uint32_t *err_word, void *stream) {
    return launch_fused(t, mats, n_mats, T, err_word, stream);
}

df11_status df11_decode(const df11_tensor *t, uint16_t *out, uint32_t *err_word, void *stream) {
    return launch_decode(t, out, err_word, stream);
}

df11_status df11_decode_block(const df11_tensor *blk, const uint64_t *mat_offsets, uint32_t k,
                              uint16_t *scratch, uint32_t *err_word, void *stream) {
    if (!blk || !mat_offsets || k == 0) return DF11_ERR_INVALID_ARG;
    if (mat_offsets[0] != 0 || mat_offsets[k] != blk->n_elems) return DF11_ERR_INVALID_ARG;
    for (uint32_t j = 0; j < k; ++j)
        if (mat_offsets[j + 1] < mat_offsets[j]) return DF11_ERR_INVALID_ARG;
    return launch_decode(blk, scratch, err_word, stream);
}

df11_status df11_decode_rows(const df11_tensor *t, uint64_t row_len, const uint32_t *rows, uint32_t n_rows,
                             uint16_t *out, uint32_t *err_word, void *stream) {
    return launch_rows(t, row_len, rows, n_rows, out, err_word, stream);
}

df11_status df11_decode_gemv(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                             uint32_t *err_word, void *stream) {
    return launch_gemv(t, mats, n_mats, T, err_word, stream);
}

#ifdef DF11_DEBUG_CHECKS
// Debug builds only (not part of the product ABI): the number of failed
// bounds checks since the last reset; synchronises the device.
uint32_t df11_debug_bounds_errors(int reset) {
    uint32_t v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyFromSymbol(&v, g_df11_bounds_errors, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (reset) {
        const uint32_t z = 0;
        if (cudaMemcpyToSymbol(g_df11_bounds_errors, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    }
    return v;
}
#endif

df11_status df11_read_error(const uint32_t *err_word, void *stream, uint32_t *host_value) {
    if (!err_word || !host_value) return DF11_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(host_value, err_word, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return DF11_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DF11_ERR_CUDA;
    return *host_value ? DF11_ERR_CORRUPT : DF11_OK;
}

df11_status df11_device_sm_count(int *sm_count) {
    if (!sm_count) return DF11_ERR_INVALID_ARG;
    return prepare_device(sm_count);
}

}  // extern "C"
