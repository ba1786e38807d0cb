// df11_internal.h -- layout of the decode tables (the `lut` array of a
// df11_tensor) shared by the host planner (df11_host.cpp) and the decode
// kernel (df11_decode.cu).  Private to libdf11.
//
// The pages decode with lookup tables instead of walking the Huffman tree,
// and split the 2^L-entry table (L = longest code, 24..32 for LLMs) into
// small tables that fit in on-chip memory ("Decodage fonde sur des LUT
// hierarchiques").  This library keeps that idea with its own layout:
//
//   level 1a  count LUT, 2^W1 u32: for a W1-bit window, how many whole codes
//             it holds from its first bit on and how many bits they take
//             (used by the counting pass);
//   level 1b  symbol LUT, 2^W2 pairs of u32: for a W2-bit window, up to four
//             whole codes: their symbols, count and total bits (decoding
//             pass);
//   level 2   for a code longer than the window, canonical limits: the
//             length is the smallest l with window < lim[l], and the symbol
//             index is (window >> (32 - l)) + offs[l].
//
// No entry of any table is an exponent value reused as a pointer (the
// pages reuse exponents 240..255 that way); codes longer than a window are
// marked by a flag entry, so every one of the 256 exponents stays legal.
#pragma once

#include <stdint.h>

#include "df11.h"

#if defined(__CUDACC__)
#define DF11_HD __host__ __device__
#else
#define DF11_HD
#endif

namespace df11 {

constexpr uint32_t kMagic = 0x33314644u;  // "DF13": table layout version 3
#ifndef DF11_COUNT_WINDOW
#define DF11_COUNT_WINDOW 12
#endif
#ifndef DF11_SYM_WINDOW
#define DF11_SYM_WINDOW 12
#endif
constexpr int kW1Max = DF11_COUNT_WINDOW;  // count LUT window (bits)
constexpr int kW2Max = DF11_SYM_WINDOW;    // symbol LUT window (bits)
constexpr int kSymsPerEntry = 4;          // codes per symbol-LUT entry

// Byte offsets inside the lut array (the compact tables; the decode kernel
// replicates them in shared memory, see df11_decode.cu).
constexpr uint32_t kOffHeader = 0;
constexpr uint32_t kOffLim = 64;                     // uint64_t[33]
constexpr uint32_t kOffOffs = kOffLim + 33 * 8 + 8;  // uint32_t[33] (336)
constexpr uint32_t kOffSymRot = 480;                 // uint8_t[256]
constexpr uint32_t kOffCountLut = 768;               // uint32_t[1 << kW1Max]
constexpr uint32_t kOffSymLut = kOffCountLut + 4u * (1u << kW1Max);  // uint2[1 << kW2Max]
constexpr uint32_t kLutBytes = kOffSymLut + 8u * (1u << kW2Max);
struct LutHeader {
    uint32_t magic;
    uint32_t w1;       // effective count-LUT window: min(kW1Max, max_len)
    uint32_t w2;       // effective symbol-LUT window: min(kW2Max, max_len)
    uint32_t max_len;  // longest code length
    uint32_t min_len;  // shortest code length
    uint32_t n_syms;   // exponent values with a code
    uint32_t w1_max;   // entries in the count LUT: 2^w1_max
    uint32_t w2_max;   // entries in the symbol LUT: 2^w2_max
    uint32_t pad[8];
};
static_assert(sizeof(LutHeader) == 64, "header is 64 bytes");

// Count-LUT entry (u32) for a window whose first code fits:
//   nb | (nc << 8) | (nb << 24), nb = bits taken (1..W1), nc = codes (1..nb).
// The low five bits are the shift amount for the window, a running sum of
// entries counts codes in bits 8..23 and bits in bits 24..30, and the sum
// stays below 2^31 for any thread (at most 95 + W1 bits, 95 codes).  kEscape marks a
// window whose first code is longer than W1 bits (or is no code): it shifts
// by 0 and sets bit 31, which ends the lookup loop.
constexpr uint32_t kEscape = 0x80000000u;
DF11_HD constexpr inline uint32_t count_entry(uint32_t nb, uint32_t nc) {
    return nb | (nc << 8) | (nb << 24);
}
DF11_HD constexpr inline uint32_t count_entry_bits(uint32_t e) { return e & 31u; }
DF11_HD constexpr inline uint32_t count_entry_codes(uint32_t e) { return (e >> 8) & 0xFFu; }

// Symbol-LUT entry: two u32, (S, M).  S holds up to four symbols (byte i =
// symbol i, as a rotated exponent, see below); M = nb | (nc << 8) with
// nb = bits taken (1..W2) and nc = codes (1..4), so nc >= k <=> M >= k << 8
// (compared as signed ints).  A long first code is S = 0, M = kEscape, which
// is negative as a signed int and so stores nothing.
DF11_HD constexpr inline uint32_t sym_entry_meta(uint32_t nb, uint32_t nc) { return nb | (nc << 8); }
DF11_HD constexpr inline uint32_t sym_entry_bits(uint32_t m) { return m & 31u; }
DF11_HD constexpr inline uint32_t sym_entry_codes(uint32_t m) { return (m >> 8) & 0xFFu; }

// Exponents are kept rotated right by one bit inside the decoder:
// rot(e) = (e >> 1) | ((e & 1) << 7).  With r = rot(e) and the sign/mantissa
// byte s = (sign << 7) | mantissa, the BF16 word is
//   high byte = (s & 0x80) | (r & 0x7F),  low byte = (r & 0x80) | (s & 0x7F),
// i.e. two bit-selects and a byte interleave per four weights.
DF11_HD constexpr inline uint32_t rotate_exponent(uint32_t e) {
    return ((e >> 1) | (e << 7)) & 0xFFu;
}

// Decode-kernel configuration.
constexpr int kThreadsPerBlockFmt = 256;  // T: threads sharing one block_start
constexpr int kBytesPerThread = 8;        // n
constexpr int kChainsPerThread = 2;       // format threads decoded by one CUDA thread
constexpr int kGroupThreads = kThreadsPerBlockFmt / kChainsPerThread;  // CUDA threads per format block
constexpr int kGroupsPerCta = 8;          // format blocks decoded side by side by one CTA
constexpr int kCtaThreads = kGroupThreads * kGroupsPerCta;
// Worst case codes per format block: every code 1 bit long.
constexpr int kMaxCodesPerBlock = kThreadsPerBlockFmt * kBytesPerThread * 8;

// Host planner pieces shared by the host and device encoders (df11_host.cpp).
df11_status plan_from_histogram(const uint64_t count[256], uint64_t n, const df11_params &p, df11_tensor *t);
void host_build_luts(const uint8_t len[256], uint8_t *lut);
void host_canonical_codes(const uint8_t len[256], uint32_t code[256]);

}  // namespace df11
