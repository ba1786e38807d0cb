// df11_internal.h -- layout of the decode tables (the `lut` array of a
// df11_tensor) shared by the host planner (df11_host.cpp) and the decode
// kernel (df11_decode.cu).  Private to libdf11.
//
// The pages decode with lookup tables instead of walking the Huffman tree,
// and split the 2^L-entry table (L = longest code, 24..32 for LLMs) into
// small tables that fit in on-chip memory ("Decodage fonde sur des LUT
// hierarchiques").  This library keeps that idea with its own layout:
//
//   level 1a  count LUT, 2^W1 bytes: for a W1-bit window, how many whole
//             codes it holds from its first bit on, and how many bits they
//             take (used by the counting pass);
//   level 1b  symbol LUT, 2^W2 u32: for a W2-bit window, up to three whole
//             codes: their symbols, count and total bits (decoding pass);
//   level 2   for a code longer than the window, canonical limits: the
//             length is the smallest l with window < lim[l], and the symbol
//             index is (window >> (32 - l)) + offs[l].
//
// No entry of any table is an exponent value reused as a pointer (the
// pages reuse exponents 240..255 that way); codes longer than a window are
// marked by a zero entry, so every one of the 256 exponents stays legal.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define DF11_HD __host__ __device__
#else
#define DF11_HD
#endif

namespace df11 {

constexpr uint32_t kMagic = 0x31314644u;  // "DF11"
constexpr int kW1Max = 14;                // count LUT window (bits)
constexpr int kW2Max = 12;                // symbol LUT window (bits)
constexpr int kSymsPerEntry = 3;          // codes per symbol-LUT entry

// Byte offsets inside the lut array.
constexpr uint32_t kOffHeader = 0;
constexpr uint32_t kOffLim = 64;                     // uint64_t[33]
constexpr uint32_t kOffOffs = kOffLim + 33 * 8 + 8;  // uint32_t[33] (336)
constexpr uint32_t kOffSymRot = 480;                 // uint8_t[256]
constexpr uint32_t kOffCountLut = 768;               // uint8_t[1 << kW1Max]
constexpr uint32_t kOffSymLut = kOffCountLut + (1u << kW1Max);  // uint32_t[1 << kW2Max]
constexpr uint32_t kLutBytes = kOffSymLut + 4u * (1u << kW2Max);
static_assert(kOffOffs + 33 * 4 <= kOffSymRot, "lut layout");
static_assert(kOffSymRot + 256 <= kOffCountLut, "lut layout");
static_assert(kLutBytes % 16 == 0, "lut must be a whole number of 16-byte units");

struct LutHeader {
    uint32_t magic;
    uint32_t w1;       // effective count-LUT window: min(kW1Max, max_len)
    uint32_t w2;       // effective symbol-LUT window: min(kW2Max, max_len)
    uint32_t max_len;  // longest code length
    uint32_t min_len;  // shortest code length
    uint32_t n_syms;   // exponent values with a code
    uint32_t pad[10];
};
static_assert(sizeof(LutHeader) == 64, "header is 64 bytes");

// Count-LUT entry: bits 0..3 = bits taken, bits 4..7 = codes.  0 = the first
// code is longer than the window.
DF11_HD constexpr inline uint32_t count_entry_bits(uint32_t e) { return e & 15u; }
DF11_HD constexpr inline uint32_t count_entry_codes(uint32_t e) { return e >> 4; }

// Symbol-LUT entry: bits 0..23 = up to three symbols (byte i = symbol i, as
// a rotated exponent, see below), bits 24..28 = bits taken, bits 29..30 =
// number of codes (1..3).  0 = the first code is longer than the window.
DF11_HD constexpr inline uint32_t sym_entry_bits(uint32_t e) { return (e >> 24) & 31u; }
DF11_HD constexpr inline uint32_t sym_entry_codes(uint32_t e) { return (e >> 29) & 3u; }

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
constexpr int kGroupsPerCta = 4;          // format blocks decoded side by side by one CTA
constexpr int kCtaThreads = kThreadsPerBlockFmt * kGroupsPerCta;
// Worst case codes per format block: every code 1 bit long.
constexpr int kMaxCodesPerBlock = kThreadsPerBlockFmt * kBytesPerThread * 8;

}  // namespace df11
