// df11_decode.cu -- the DF11 decode kernel for sm_100a and its launchers
// (df11_decode, df11_decode_block).
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
//    time and strides over the blocks; the decode tables are staged into
//    shared memory once per CTA with one TMA bulk copy (cp.async.bulk, no
//    multicast).
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
//  * Pass 1 counts with a 14-bit count table (several codes per lookup);
//    one add per lookup updates both the code count and the bits taken,
//    the entry's low bits are the shift amount, and a code longer than the
//    window leaves the loop through its condition (flag bit), so the loop
//    body is a lookup, an add, three funnel shifts and a compare.
//  * Pass 2 decodes with a 12-bit table of up to four symbols per entry and
//    stops on the code count pass 1 found.  Codes longer than the window
//    fall back to canonical limits.
//  * Warp shuffle scan + one cross-warp step (named barrier per group).
//  * Exponents are kept rotated by one bit, so the merge with the
//    sign/mantissa bytes is two bit-selects and two byte-permutes per four
//    weights; loads and stores are 128-bit.  The next block's stream words,
//    gaps and block starts, and this block's first sign/mantissa vectors,
//    are loaded before the decode loops so their latency hides behind the
//    arithmetic.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "df11.h"
#include "df11_internal.h"

namespace {

using namespace df11;

constexpr uint32_t kSbufBytes = (uint32_t)kMaxCodesPerBlock + 64u;  // + head offset (<16) + slack
constexpr uint32_t kGroupBytes = kSbufBytes + 32u;                    // + 8 warp totals
constexpr uint32_t kSmemBytes = kLutBytes + kGroupsPerCta * kGroupBytes + 16u;  // + mbarrier
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint32_t kKernErrTimeout = 0x10u;  // table staging did not complete
static_assert(kGroupBytes % 16 == 0, "group stride keeps 16-byte alignment");
static_assert(kLutBytes % 16 == 0, "bulk copy size");
static_assert(kSmemBytes <= 227u * 1024u, "fits one CTA's shared memory");

struct DecodeArgs {
    const uint8_t *enc;
    const uint8_t *sm;
    const uint32_t *gaps32;
    const uint32_t *bstart;
    const uint8_t *lut;
    uint16_t *out;
    uint32_t *err;
    uint64_t n_elems;
    uint64_t total_bits;
    uint64_t n_threads;
    uint64_t n_blocks;
};

// ----------------------------------------------------------------- PTX
__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
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
__device__ __forceinline__ void sts_zero16(uint32_t a) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
}
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

// Bounded wait for phase 0 of the table mbarrier.  Returns false if the
// copy did not complete within the iteration limit.
__device__ __forceinline__ bool wait_tables(uint32_t bar) {
    uint32_t done = 0;
    for (uint32_t it = 0; it < (1u << 22) && !done; ++it) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar)
            : "memory");
    }
    return done != 0;
}

// Bulk copy of the decode tables into shared memory (TMA engine, one
// thread), completion tracked by an mbarrier that every thread waits on.
__device__ __forceinline__ bool stage_tables(uint32_t dst, const uint8_t *src, uint32_t bytes, uint32_t bar) {
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
            "l"(src), "r"(bytes), "r"(bar)
            : "memory");
    }
    return wait_tables(bar);
}

// Length of a code longer than the table window, from the canonical limits
// in shared memory: the smallest l with window < lim[l].  0 if none.
__device__ __noinline__ uint32_t long_code_length(uint32_t x, uint32_t lim_addr, uint32_t from, uint32_t max_len) {
    for (uint32_t l = from; l <= max_len; ++l) {
        const uint64_t lim = lds_u64(lim_addr + 8u * l);
        if ((uint64_t)x < lim) return l;
    }
    return 0u;
}

// Shifts the 96-bit window left by n bits (n <= 32), filling with ones.
__device__ __forceinline__ void shift_window_clamped(uint32_t &hi, uint32_t &lo, uint32_t &fl, uint32_t n) {
    hi = __funnelshift_lc(lo, hi, n);
    lo = __funnelshift_lc(fl, lo, n);
    fl = __funnelshift_lc(kFull, fl, n);
}

struct BlockInputs {
    uint4 v;              // 16 stream bytes: chain A's 8, then chain B's 8
    uint32_t wn;          // lane 31 only: the next thread's first 4 bytes
    uint32_t g_hi, g_lo;  // the two 32-bit gap words holding bits [5tA, 5tA + 15)
    uint32_t s, e;        // block_start[b], block_start[b + 1]
};

__device__ __forceinline__ void load_block_inputs(const DecodeArgs &a, uint64_t blk, uint32_t lt,
                                                  uint32_t lane, BlockInputs &in) {
    const uint64_t tA = blk * (uint64_t)kThreadsPerBlockFmt + 2u * lt;
    in.v = ld_stream_u4(a.enc + 8ull * tA);  // 16-byte aligned: tA is even
    in.wn = (lane == 31u) ? __ldg(reinterpret_cast<const uint32_t *>(a.enc + 8ull * tA + 16ull)) : 0u;
    const uint64_t word = (5ull * tA) >> 5;
    in.g_hi = __ldg(a.gaps32 + word);
    in.g_lo = __ldg(a.gaps32 + word + 1);
    in.s = __ldg(a.bstart + blk);
    in.e = __ldg(a.bstart + blk + 1);
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

// The chunks holding the block's first and last elements, by one warp:
// lanes 0..15 take the first chunk, lanes 16..31 the last one, one element
// each (only elements inside [s, e) are written).
__device__ __forceinline__ void merge_edges(const uint8_t *sm, uint16_t *out, uint32_t sb, uint32_t base,
                                            uint32_t c_full, uint32_t span, uint32_t s, uint32_t e,
                                            uint32_t lane) {
    const bool head = s != base;
    const bool tail = (span & 15u) != 0u && !(head && c_full == 0u);
    const uint32_t c = (lane < 16u) ? 0u : c_full;
    const bool mine = (lane < 16u) ? head : tail;
    const uint32_t g = base + 16u * c + (lane & 15u);
    if (mine && g >= s && g < e) {
        const uint32_t sm8 = __ldg(sm + g);
        const uint32_t r = lds_u8(sb + (g - base));
        // r = rotated exponent: high byte (s & 0x80) | (r & 0x7F), low byte (r & 0x80) | (s & 0x7F)
        const uint32_t hi8 = (sm8 & 0x80u) | (r & 0x7Fu);
        const uint32_t lo8 = (r & 0x80u) | (sm8 & 0x7Fu);
        out[g] = (uint16_t)(lo8 | (hi8 << 8));
    }
}

// One decode chain: the 96-bit window (hi, lo, fl) of a format thread, the
// bits it must consume (rem0), and a running accumulator.
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

// Long-code step of the count pass for one chain whose accumulator carries
// the escape flag.  Returns true if the chain still has bits to consume.
__device__ __forceinline__ bool count_long_code(uint32_t &acc, uint32_t lim, uint32_t &hi, uint32_t &lo,
                                                uint32_t &fl, uint32_t s_lim, uint32_t from, uint32_t max_len,
                                                uint32_t &err) {
    acc -= kEscape;
    const uint32_t l = long_code_length(hi, s_lim, from, max_len);
    if (l == 0u) {
        err |= DF11_KERR_BAD_CODE;
        acc = lim;  // stop this chain
        return false;
    }
    acc += (l << 24) | (1u << 8);
    shift_window_clamped(hi, lo, fl, l);
    return acc < lim;
}

// Long-code step of the decoding pass: writes the symbol, advances.
__device__ __forceinline__ bool decode_long_code(uint32_t &pacc, uint32_t pend, uint32_t &hi, uint32_t &lo,
                                                 uint32_t &fl, uint32_t sb, uint32_t s_lim, uint32_t s_offs,
                                                 uint32_t s_symrot, uint32_t from, uint32_t max_len) {
    pacc -= kEscape;
    const uint32_t l = long_code_length(hi, s_lim, from, max_len);
    if (l == 0u) {  // reported by the count pass
        pacc = pend;
        return false;
    }
    const uint32_t idx = (hi >> (32u - l)) + lds_u32(s_offs + 4u * l);
    const uint32_t p = pacc >> 8;
    red_or(sb + (p & ~3u), lds_u8(s_symrot + (idx & 255u)) << (8u * (p & 3u)));
    pacc += 1u << 8;
    shift_window_clamped(hi, lo, fl, l);
    return pacc < pend;
}

__global__ void __launch_bounds__(kCtaThreads, 1) df11_decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_lim = s_base + kOffLim;
    const uint32_t s_offs = s_base + kOffOffs;
    const uint32_t s_symrot = s_base + kOffSymRot;
    const uint32_t s_clut = s_base + kOffCountLut;
    const uint32_t s_slut = s_base + kOffSymLut;
    const uint32_t s_mbar = s_base + kLutBytes + kGroupsPerCta * kGroupBytes;

    const uint32_t tid = threadIdx.x;
    const uint32_t group = tid / kGroupThreads;
    const uint32_t lt = tid % kGroupThreads;  // thread within the group
    const uint32_t lane = tid & 31u;
    const uint32_t warp = lt >> 5;            // warp within the group
    const uint32_t sb = s_base + kLutBytes + group * kGroupBytes;  // this group's exponent buffer
    const uint32_t wtot = sb + kSbufBytes;                          // per-warp totals
    uint32_t my_err = 0;

    const uint64_t stride = (uint64_t)gridDim.x * kGroupsPerCta;
    uint64_t blk = (uint64_t)blockIdx.x * kGroupsPerCta + group;

    // Prefetch the first block's inputs while the tables stream in.
    BlockInputs cur{};
    if (blk < a.n_blocks) load_block_inputs(a, blk, lt, lane, cur);

    const bool staged = stage_tables(s_base, a.lut, kLutBytes, s_mbar);
    if (__syncthreads_or(!staged)) {
        // Uniform over the CTA.  One more bounded wait so no copy is left in
        // flight into this CTA's shared memory, then report and stop.
        if (tid == 0) {
            wait_tables(s_mbar);
            if (a.err) atomicOr(a.err, kKernErrTimeout);
        }
        __syncthreads();
        return;
    }

    const LutHeader *hdr = reinterpret_cast<const LutHeader *>(smem + kOffHeader);
    const uint32_t w1 = hdr->w1, w2 = hdr->w2, max_len = hdr->max_len;
    if (hdr->magic != kMagic || w1 < 1u || w1 > (uint32_t)kW1Max || w2 < 1u || w2 > (uint32_t)kW2Max ||
        max_len > 32u) {
        if (tid == 0 && a.err) atomicOr(a.err, DF11_KERR_BAD_CODE);
        return;  // uniform over the CTA: nothing was written yet
    }
    // Every table entry must be the escape flag or take 1..W bits for
    // 1..(bits) codes, so each lookup makes progress: the decode loops then
    // end after at most 95 lookups plus 95 long codes whatever the stream.
    {
        bool bad = false;
        for (uint32_t i = tid; i < (1u << w1); i += kCtaThreads) {
            const uint32_t ent = lds_u32(s_clut + 4u * i);
            const uint32_t nb = count_entry_bits(ent), nc = count_entry_codes(ent);
            bad |= ent != kEscape && (ent != count_entry(nb, nc) || nb == 0u || nb > w1 || nc == 0u || nc > nb);
        }
        for (uint32_t i = tid; i < (1u << w2); i += kCtaThreads) {
            const uint2 ent = lds_u2(s_slut + 8u * i);
            const uint32_t nb = sym_entry_bits(ent.y), nc = sym_entry_codes(ent.y);
            bad |= ent.y != kEscape && (ent.y != sym_entry_meta(nb, nc) || nb == 0u || nb > w2 || nc == 0u ||
                                        nc > (uint32_t)kSymsPerEntry || nc > nb);
        }
        if (__syncthreads_or(bad)) {
            if (tid == 0 && a.err) atomicOr(a.err, DF11_KERR_BAD_CODE);
            return;
        }
    }
    const uint32_t sh1 = 32u - w1, sh2 = 32u - w2;

    for (; blk < a.n_blocks; blk += stride) {
        const BlockInputs in = cur;
        const uint64_t nxt = blk + stride;
        if (nxt < a.n_blocks) load_block_inputs(a, nxt, lt, lane, cur);

        const uint64_t tA = blk * (uint64_t)kThreadsPerBlockFmt + 2u * lt;
        const uint32_t s = in.s, e = in.e;
        const uint32_t base = s & ~15u;  // first 16-element chunk of the block's output
        const bool range_ok = (e >= s) && ((uint64_t)e <= a.n_elems) && (e - s <= (uint32_t)kMaxCodesPerBlock);
        // chunks [c_lo, c_full) lie wholly inside [s, e)
        const uint32_t span = range_ok ? e - base : 0u;
        const uint32_t c_lo = (s != base) ? 1u : 0u;
        const uint32_t c_full = span >> 4;
        const uint32_t c0 = c_lo + lt;
        uint4 smv0 = make_uint4(0, 0, 0, 0);
        if (c0 < c_full) smv0 = ld_stream_u4(a.sm + (uint64_t)base + 16ull * c0);

        // ---- the two chains: format threads tA and tA + 1
        // gaps are an MSB-first bit string: bits [5tA, 5tA + 15) hold the
        // gaps of tA, tA + 1 and tA + 2
        const uint32_t gb = __funnelshift_l(bswap32(in.g_lo), bswap32(in.g_hi), (uint32_t)((5ull * tA) & 31u));
        uint32_t gapA = gb >> 27, gapB = (gb >> 22) & 31u;
        const uint32_t gapC = (gb >> 17) & 31u;
        int32_t endA, endB;
        if (tA >= a.n_threads) { gapA = 0; endA = 0; }
        else if (tA + 1 == a.n_threads) endA = (int32_t)(a.total_bits - 64ull * tA);
        else endA = 64 + (int32_t)gapB;
        if (tA + 1 >= a.n_threads) { gapB = 0; endB = 0; }
        else if (tA + 2 == a.n_threads) endB = (int32_t)(a.total_bits - 64ull * (tA + 1));
        else endB = 64 + (int32_t)gapC;
        uint32_t nextw = __shfl_down_sync(kFull, in.v.x, 1);
        if (lane == 31u) nextw = in.wn;
        const Chain A = make_chain(bswap32(in.v.x), bswap32(in.v.y), bswap32(in.v.z), gapA, endA, my_err);
        const Chain B = make_chain(bswap32(in.v.z), bswap32(in.v.w), bswap32(nextw), gapB, endB, my_err);

        // ---- pass 1: count the codes of both chains
        uint32_t cA, cB;
        {
            uint32_t hA = A.hi, lA = A.lo, fA = A.fl, hB = B.hi, lB = B.lo, fB = B.fl;
            uint32_t aA = 0, aB = 0;
            const uint32_t limA = (uint32_t)A.rem0 << 24, limB = (uint32_t)B.rem0 << 24;
            for (;;) {
                while ((aA < limA) | (aB < limB)) {
                    uint32_t eA = lds_u32(s_clut + ((hA >> sh1) << 2));
                    uint32_t eB = lds_u32(s_clut + ((hB >> sh1) << 2));
                    eA = (aA < limA) ? eA : 0u;
                    eB = (aB < limB) ? eB : 0u;
                    aA += eA;
                    aB += eB;
                    hA = __funnelshift_l(lA, hA, eA);
                    lA = __funnelshift_l(fA, lA, eA);
                    fA = __funnelshift_l(kFull, fA, eA);
                    hB = __funnelshift_l(lB, hB, eB);
                    lB = __funnelshift_l(fB, lB, eB);
                    fB = __funnelshift_l(kFull, fB, eB);
                }
                bool more = false;
                if (aA >= kEscape) more |= count_long_code(aA, limA, hA, lA, fA, s_lim, w1 + 1u, max_len, my_err);
                if (aB >= kEscape) more |= count_long_code(aB, limB, hB, lB, fB, s_lim, w1 + 1u, max_len, my_err);
                if (!more) break;
            }
            cA = (aA >> 8) & 0xFFFFu;
            cB = (aB >> 8) & 0xFFFFu;
            if ((aA >> 24) != (uint32_t)A.rem0 || (aB >> 24) != (uint32_t)B.rem0) my_err |= DF11_KERR_OVERRUN;
        }

        // ---- clear the exponent buffer span this block uses (the decoding
        // pass ORs symbols into it); the scan barrier orders this before it
        for (uint32_t c = lt; c < ((span + 15u) >> 4) + 1u; c += kGroupThreads) sts_zero16(sb + 16u * c);

        // ---- block scan: warp inclusive scan, then across the group's warps
        const uint32_t cnt = cA + cB;
        uint32_t incl = cnt;
#pragma unroll
        for (uint32_t d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, d);
            if (lane >= d) incl += v;
        }
        constexpr uint32_t kWarps = kGroupThreads / 32;
        if (lane == 31u) sts_u32(wtot + 4u * warp, incl);
        group_barrier(group);
        uint32_t wsum = (lane < kWarps) ? lds_u32(wtot + 4u * lane) : 0u;
#pragma unroll
        for (uint32_t d = 1; d < kWarps; d <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, wsum, d);
            if (lane >= d) wsum += v;
        }
        const uint32_t total = __shfl_sync(kFull, wsum, kWarps - 1u);
        const uint32_t wpre = __shfl_sync(kFull, wsum, (warp + kWarps - 1u) % kWarps) * (warp != 0u ? 1u : 0u);
        const bool ok = range_ok && (total == e - s);
        if (!ok && lt == 0) my_err |= range_ok ? DF11_KERR_COUNT_MISMATCH : DF11_KERR_BAD_BLOCK;

        // ---- pass 2: decode both chains again into the exponent buffer
        if (ok) {
            uint32_t hA = A.hi, lA = A.lo, fA = A.fl, hB = B.hi, lB = B.lo, fB = B.fl;
            const uint32_t startA = (s - base) + wpre + incl - cnt;  // buffer index of A's first code
            const uint32_t startB = startA + cA;
            uint32_t pA = startA << 8, pB = startB << 8;
            const uint32_t endPA = (startA + cA) << 8, endPB = (startB + cB) << 8;
            for (;;) {
                while ((pA < endPA) | (pB < endPB)) {
                    const uint2 eA = lds_u2(s_slut + ((hA >> sh2) << 3));
                    const uint2 eB = lds_u2(s_slut + ((hB >> sh2) << 3));
                    const bool actA = pA < endPA, actB = pB < endPB;
                    const int32_t mA = actA ? (int32_t)eA.y : 0;
                    const int32_t mB = actB ? (int32_t)eB.y : 0;
                    // up to four symbol bytes land in the word holding byte p
                    // and the next one; unused symbol bytes are zero
                    const uint32_t bA = pA >> 8, bB = pB >> 8;
                    const uint32_t shA = (bA & 3u) << 3, shB = (bB & 3u) << 3;
                    const uint32_t wA = sb + (bA & ~3u), wB = sb + (bB & ~3u);
                    if (actA) {
                        red_or(wA, eA.x << shA);
                        if (shA) red_or(wA + 4u, __funnelshift_l(eA.x, 0u, shA));
                    }
                    if (actB) {
                        red_or(wB, eB.x << shB);
                        if (shB) red_or(wB + 4u, __funnelshift_l(eB.x, 0u, shB));
                    }
                    pA += (uint32_t)mA;
                    pB += (uint32_t)mB;
                    hA = __funnelshift_l(lA, hA, (uint32_t)mA);
                    lA = __funnelshift_l(fA, lA, (uint32_t)mA);
                    fA = __funnelshift_l(kFull, fA, (uint32_t)mA);
                    hB = __funnelshift_l(lB, hB, (uint32_t)mB);
                    lB = __funnelshift_l(fB, lB, (uint32_t)mB);
                    fB = __funnelshift_l(kFull, fB, (uint32_t)mB);
                }
                bool more = false;
                if (pA >= kEscape)
                    more |= decode_long_code(pA, endPA, hA, lA, fA, sb, s_lim, s_offs, s_symrot, w2 + 1u, max_len);
                if (pB >= kEscape)
                    more |= decode_long_code(pB, endPB, hB, lB, fB, sb, s_lim, s_offs, s_symrot, w2 + 1u, max_len);
                if (!more) break;
            }
        }
        group_barrier(group);

        // ---- merge with sign/mantissa and store, 16 weights per step
        if (ok) {
            if (c0 < c_full) {
                const uint8_t *smp = a.sm + (uint64_t)base + 16ull * c0;
                uint16_t *dst = a.out + (uint64_t)base + 16ull * c0;
                uint32_t ex_addr = sb + 16u * c0;
                uint4 smv = smv0;
                for (uint32_t c = c0;;) {
                    const uint4 ex = lds_u4(ex_addr);
                    uint32_t o[8];
                    merge16(smv, ex, o);
                    st_u4(dst, o[0], o[1], o[2], o[3]);
                    st_u4(dst + 8, o[4], o[5], o[6], o[7]);
                    c += kGroupThreads;
                    if (c >= c_full) break;
                    smp += 16u * kGroupThreads;
                    dst += 16u * kGroupThreads;
                    ex_addr += 16u * kGroupThreads;
                    smv = ld_stream_u4(smp);
                }
            }
            if (warp == 0) merge_edges(a.sm, a.out, sb, base, c_full, span, s, e, lane);
        }
        group_barrier(group);
    }
    if (my_err && a.err) atomicOr(a.err, my_err);
}

// ----------------------------------------------------------------- host
std::atomic<int> g_sm_count[64];
std::atomic<int> g_attr_set[64];

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
        if (cudaFuncSetAttribute(df11_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_attr_set[dev].store(1, std::memory_order_release);
    }
    *sm_count = sms;
    return DF11_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

df11_status launch_decode(const df11_tensor *t, uint16_t *out, uint32_t *err_word, void *stream) {
    if (!t) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (t->n_elems == 0) return DF11_OK;  // nothing to write; out may be NULL
    if (!out || !t->enc || !t->sm || !t->gaps || !t->block_start || !t->lut) return DF11_ERR_INVALID_ARG;
    if (!aligned16(t->enc) || !aligned16(t->sm) || !aligned16(t->gaps) || !aligned16(t->lut) ||
        !aligned16(t->block_start) || !aligned16(out))
        return DF11_ERR_INVALID_ARG;
    int sms = 0;
    st = prepare_device(&sms);
    if (st != DF11_OK) return st;
    DecodeArgs a;
    a.enc = t->enc;
    a.sm = t->sm;
    a.gaps32 = reinterpret_cast<const uint32_t *>(t->gaps);
    a.bstart = t->block_start;
    a.lut = t->lut;
    a.out = out;
    a.err = err_word;
    a.n_elems = t->n_elems;
    a.total_bits = t->total_bits;
    a.n_threads = t->n_threads;
    a.n_blocks = t->n_blocks;
    const uint64_t ctas_needed = (t->n_blocks + kGroupsPerCta - 1) / kGroupsPerCta;
    const unsigned grid = (unsigned)(ctas_needed < (uint64_t)sms ? ctas_needed : (uint64_t)sms);
    df11_decode_kernel<<<grid, kCtaThreads, kSmemBytes, reinterpret_cast<cudaStream_t>(stream)>>>(a);
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}

}  // namespace

extern "C" {

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
