/*
 * df11_oracle.c -- the oracle for the DFloat11 exponent codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg may load or run this code.  It
 * shares no source, header, table or constant generator with the GPU
 * library, and it never calls into it.
 *
 * Everything here is written to be checked by eye against the method text,
 * not to be fast: plain loops, one bit at a time, explicit binary trees.
 *
 * Sources followed (web pages on DFloat11):
 *  [P4] "DFloat11 : compression sans perte pour l'inference GPU qui reduit
 *       les LLM a 70 % de leur taille" (fr.news.hada.io), sections
 *       << La marge de compression restante dans l'exposant BFloat16 >>,
 *       << Le format DFloat11 >>, << Decompression adaptee a l'inference GPU >>,
 *       << Noyau GPU en deux etapes et metadonnees auxiliaires >>.
 *  [P2] "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *       Inference via Dynamic-Length Float" (chatpaper.ai), abstract.
 * Published algorithms restated here from their definitions:
 *  - Huffman's construction (merge the two lightest subtrees, repeat).
 *  - Package-merge for length-limited optimal codes (Larmore & Hirschberg,
 *    "A fast algorithm for optimal length-limited Huffman codes", JACM 1990).
 *  - Canonical code assignment by (length, symbol) as defined in RFC 1951
 *    section 3.2.2.
 *
 * Readings of points the pages leave open:
 *  - Exponent bits are packed MSB-first inside each byte, bytes in increasing
 *    address order; the last partial byte is zero-filled.
 *  - The sign/mantissa byte of a weight is (sign << 7) | mantissa.
 *  - Only exponents that occur get a code; all 256 values are legal symbols.
 *    A one-symbol alphabet gets the 1-bit code "0".
 *  - Thread t owns bits [8n*t, 8n*(t+1)) of the exponent stream and decodes
 *    the codes that start there.  Its gap is the offset of the first code
 *    start at or after 8n*t, where the end of the stream counts as a start.
 *  - Gaps are 5-bit fields packed MSB-first in thread order; threads past the
 *    last one of the stream (padding up to a whole block) have gap 0.
 *  - block_start[b] is the index of the first element decoded by thread
 *    block b, with a final sentinel equal to the element count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_CAP (-2)     /* length cap too small for the alphabet */
#define ORC_ERR_CORRUPT (-3) /* stream does not decode */
#define ORC_ERR_NOMEM (-4)
#define ORC_ERR_NOT_PREFIX_FREE (-5)

/* ---------------------------------------------------------------------
 * BF16 fields [P4 << La marge de compression restante dans l'exposant
 * BFloat16 >>]: 1 sign bit, 8 exponent bits, 7 mantissa bits.
 * ------------------------------------------------------------------- */
static unsigned bf16_sign(uint16_t w) { return (w >> 15) & 1u; }
static unsigned bf16_exponent(uint16_t w) { return (w >> 7) & 0xFFu; }
static unsigned bf16_mantissa(uint16_t w) { return w & 0x7Fu; }
static uint16_t bf16_from_fields(unsigned s, unsigned e, unsigned m) {
    return (uint16_t)((s << 15) | (e << 7) | m);
}

/* Exponent histogram [P4 << Le format DFloat11 >>: the tree is built from
 * the distribution of the exponents]. */
int orc_histogram(const uint16_t *w, uint64_t n, uint64_t count[256]) {
    if (!count || (n && !w)) return ORC_ERR_ARG;
    for (int s = 0; s < 256; ++s) count[s] = 0;
    for (uint64_t i = 0; i < n; ++i) count[bf16_exponent(w[i])] += 1;
    return ORC_OK;
}

/* Statistics the pages quote: Shannon entropy of the exponent (bits),
 * number of exponent values in use, and the average code length. */
void orc_exponent_stats(const uint64_t count[256], const uint8_t len[256],
                        double *entropy_bits, int *distinct, double *mean_len) {
    uint64_t total = 0;
    for (int s = 0; s < 256; ++s) total += count[s];
    double h = 0.0, bits = 0.0;
    int k = 0;
    for (int s = 0; s < 256; ++s) {
        if (!count[s]) continue;
        ++k;
        double p = (double)count[s] / (double)total;
        h -= p * log2(p);
        if (len) bits += (double)count[s] * (double)len[s];
    }
    if (entropy_bits) *entropy_bits = h;
    if (distinct) *distinct = k;
    if (mean_len) *mean_len = total ? bits / (double)total : 0.0;
}

/* ---------------------------------------------------------------------
 * Code lengths.  An "item" is a weight plus, for every symbol, how many
 * times that symbol's leaf lies inside the item.
 * ------------------------------------------------------------------- */
typedef struct {
    uint64_t weight;
    uint16_t mult[256];
} orc_item;

/* Plain Huffman (no cap): repeatedly merge the two lightest nodes; every
 * merge adds one bit to the code of each symbol inside the merged nodes.
 * Ties are broken by the lower node index (any choice is optimal). */
int orc_huffman_lengths(const uint64_t count[256], uint8_t len[256]) {
    orc_item *nodes = (orc_item *)calloc(256, sizeof(orc_item));
    int alive[256];
    int k = 0;
    if (!nodes) return ORC_ERR_NOMEM;
    for (int s = 0; s < 256; ++s) len[s] = 0;
    for (int s = 0; s < 256; ++s) {
        if (!count[s]) continue;
        nodes[k].weight = count[s];
        nodes[k].mult[s] = 1;
        alive[k] = 1;
        ++k;
    }
    if (k == 1) {
        for (int s = 0; s < 256; ++s) if (count[s]) len[s] = 1;
    }
    int remaining = k;
    while (remaining > 1) {
        int a = -1, b = -1;
        for (int i = 0; i < k; ++i) {
            if (!alive[i]) continue;
            if (a < 0 || nodes[i].weight < nodes[a].weight) { b = a; a = i; }
            else if (b < 0 || nodes[i].weight < nodes[b].weight) { b = i; }
        }
        /* merge b into a */
        nodes[a].weight += nodes[b].weight;
        for (int s = 0; s < 256; ++s) nodes[a].mult[s] += nodes[b].mult[s];
        alive[b] = 0;
        for (int s = 0; s < 256; ++s)
            if (nodes[a].mult[s]) len[s] += 1;
        --remaining;
    }
    free(nodes);
    return ORC_OK;
}

/* Package-merge (coin collector): every used symbol contributes one coin of
 * each denomination 2^-1 .. 2^-cap whose value is its count.  Starting from
 * the smallest denomination, adjacent items are paired into packages of the
 * next denomination and merged with that denomination's coins.  In the final
 * (2^-1) list the 2K-2 cheapest items are taken; a symbol's code length is
 * the number of its coins among them.  This gives a prefix code of minimum
 * total length among those with every length <= cap. */
int orc_package_merge_lengths(const uint64_t count[256], int cap, uint8_t len[256]) {
    int k = 0;
    for (int s = 0; s < 256; ++s) { len[s] = 0; if (count[s]) ++k; }
    if (k == 0) return ORC_OK;
    if (cap < 1 || cap > 32) return ORC_ERR_ARG;
    if (k == 1) {
        for (int s = 0; s < 256; ++s) if (count[s]) len[s] = 1;
        return ORC_OK;
    }
    if (cap < 32 && (uint64_t)k > ((uint64_t)1 << cap)) return ORC_ERR_CAP;
    if (k > 256) return ORC_ERR_ARG;

    orc_item *leaves = (orc_item *)calloc((size_t)k, sizeof(orc_item));
    orc_item *list = (orc_item *)calloc((size_t)(2 * k), sizeof(orc_item));
    orc_item *packs = (orc_item *)calloc((size_t)k, sizeof(orc_item));
    if (!leaves || !list || !packs) { free(leaves); free(list); free(packs); return ORC_ERR_NOMEM; }
    int j = 0;
    for (int s = 0; s < 256; ++s) {
        if (!count[s]) continue;
        leaves[j].weight = count[s];
        leaves[j].mult[s] = 1;
        ++j;
    }
    /* leaves were filled in symbol order; a stable sort keeps that order
     * among equal weights (qsort is not stable, so insertion sort). */
    for (int a = 1; a < k; ++a) {
        orc_item t = leaves[a];
        int b = a - 1;
        while (b >= 0 && leaves[b].weight > t.weight) { leaves[b + 1] = leaves[b]; --b; }
        leaves[b + 1] = t;
    }

    /* list for denomination 2^-cap: the coins themselves */
    int n_list = k;
    for (int i = 0; i < k; ++i) list[i] = leaves[i];
    for (int level = cap - 1; level >= 1; --level) {
        /* package adjacent pairs */
        int n_pack = n_list / 2;
        for (int p = 0; p < n_pack; ++p) {
            packs[p].weight = list[2 * p].weight + list[2 * p + 1].weight;
            for (int s = 0; s < 256; ++s)
                packs[p].mult[s] = (uint16_t)(list[2 * p].mult[s] + list[2 * p + 1].mult[s]);
        }
        /* merge coins of this denomination with the packages (coins first
         * on equal weight) */
        int a = 0, b = 0, o = 0;
        orc_item *merged = (orc_item *)calloc((size_t)(k + n_pack), sizeof(orc_item));
        if (!merged) { free(leaves); free(list); free(packs); return ORC_ERR_NOMEM; }
        while (a < k || b < n_pack) {
            if (b >= n_pack || (a < k && leaves[a].weight <= packs[b].weight)) merged[o++] = leaves[a++];
            else merged[o++] = packs[b++];
        }
        /* a list never reaches 2K items: it holds K coins plus fewer than
         * K packages */
        if (o >= 2 * k) { free(merged); free(leaves); free(list); free(packs); return ORC_ERR_ARG; }
        n_list = o;
        for (int i = 0; i < n_list; ++i) list[i] = merged[i];
        free(merged);
    }
    for (int i = 0; i < 2 * k - 2; ++i)
        for (int s = 0; s < 256; ++s) len[s] = (uint8_t)(len[s] + list[i].mult[s]);
    free(leaves);
    free(list);
    free(packs);
    return ORC_OK;
}

/* Canonical codes (RFC 1951 section 3.2.2, restated): walk symbols in order
 * of (length, symbol value); the first gets code 0, each next one gets the
 * previous code plus one, shifted left by the increase in length. */
int orc_canonical_codes(const uint8_t len[256], uint32_t code[256]) {
    uint64_t next = 0;
    int prev_len = 0, first = 1;
    for (int s = 0; s < 256; ++s) code[s] = 0;
    for (int l = 1; l <= 32; ++l) {
        for (int s = 0; s < 256; ++s) {
            if (len[s] != l) continue;
            if (first) { next = 0; first = 0; }
            else next = (next + 1) << (l - prev_len);
            if (next >> l) return ORC_ERR_NOT_PREFIX_FREE; /* Kraft sum > 1 */
            code[s] = (uint32_t)next;
            prev_len = l;
        }
    }
    for (int s = 0; s < 256; ++s) if (len[s] > 32) return ORC_ERR_ARG;
    return ORC_OK;
}

/* Kraft sum scaled by 2^32: sum over symbols of 2^(32 - len). */
uint64_t orc_kraft_sum_2p32(const uint8_t len[256]) {
    uint64_t k = 0;
    for (int s = 0; s < 256; ++s)
        if (len[s]) k += (uint64_t)1 << (32 - len[s]);
    return k;
}

/* ---------------------------------------------------------------------
 * Encoding [P4 << Le format DFloat11 >>]: exponent codes bit-packed into
 * EncodedExponent, sign and mantissa kept as one byte per weight in
 * PackedSignMantissa.
 * ------------------------------------------------------------------- */
static void put_bit(uint8_t *buf, uint64_t pos, unsigned bit) {
    if (bit) buf[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
}
static unsigned get_bit(const uint8_t *buf, uint64_t pos) {
    return (buf[pos >> 3] >> (7 - (pos & 7))) & 1u;
}

/* Total bits of the exponent stream for the given lengths. */
uint64_t orc_total_bits(const uint16_t *w, uint64_t n, const uint8_t len[256]) {
    uint64_t bits = 0;
    for (uint64_t i = 0; i < n; ++i) bits += len[bf16_exponent(w[i])];
    return bits;
}

/* enc must hold at least ceil(total_bits / 8) bytes; it is zeroed first. */
int orc_encode(const uint16_t *w, uint64_t n, const uint8_t len[256],
               uint8_t *enc, uint64_t enc_cap, uint8_t *sm, uint64_t *total_bits) {
    uint32_t code[256];
    int rc = orc_canonical_codes(len, code);
    if (rc) return rc;
    uint64_t bits = orc_total_bits(w, n, len);
    if ((bits + 7) / 8 > enc_cap) return ORC_ERR_ARG;
    memset(enc, 0, (size_t)enc_cap);
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; ++i) {
        unsigned e = bf16_exponent(w[i]);
        if (!len[e]) return ORC_ERR_ARG; /* exponent without a code */
        for (int b = len[e] - 1; b >= 0; --b) put_bit(enc, pos++, (code[e] >> b) & 1u);
        sm[i] = (uint8_t)((bf16_sign(w[i]) << 7) | bf16_mantissa(w[i]));
    }
    *total_bits = pos;
    return ORC_OK;
}

/* ---------------------------------------------------------------------
 * Decoding: the classic Huffman decode the pages contrast the GPU kernel
 * with [P4 << Decompression adaptee a l'inference GPU >>] -- walk the code
 * tree one bit at a time from the root; at a leaf, emit its symbol and
 * return to the root.
 * ------------------------------------------------------------------- */
typedef struct {
    int32_t child[2 * 256 * 33][2]; /* generous bound on internal nodes */
    int32_t leaf_symbol[2 * 256 * 33];
    int n_nodes;
} orc_tree;

/* Inserts every code into a binary tree, one bit at a time from its most
 * significant bit.  A code set is prefix-free exactly when no insertion
 * walks through a node that is already a leaf, and no code ends on a node
 * that is already a leaf or already has children. */
static orc_tree *build_tree_from_codes(const uint32_t code[256], const uint8_t len[256], int *rc) {
    for (int s = 0; s < 256; ++s)
        if (len[s] > 32) { *rc = ORC_ERR_ARG; return NULL; }
    orc_tree *t = (orc_tree *)malloc(sizeof(orc_tree));
    if (!t) { *rc = ORC_ERR_NOMEM; return NULL; }
    t->n_nodes = 1;
    t->child[0][0] = t->child[0][1] = -1;
    t->leaf_symbol[0] = -1;
    for (int s = 0; s < 256; ++s) {
        if (!len[s]) continue;
        int node = 0;
        for (int b = len[s] - 1; b >= 0; --b) {
            if (t->leaf_symbol[node] >= 0) { free(t); *rc = ORC_ERR_NOT_PREFIX_FREE; return NULL; }
            unsigned bit = (code[s] >> b) & 1u;
            if (t->child[node][bit] < 0) {
                int m = t->n_nodes++;
                t->child[m][0] = t->child[m][1] = -1;
                t->leaf_symbol[m] = -1;
                t->child[node][bit] = m;
            }
            node = t->child[node][bit];
        }
        if (t->leaf_symbol[node] >= 0 || t->child[node][0] >= 0 || t->child[node][1] >= 0) {
            free(t); *rc = ORC_ERR_NOT_PREFIX_FREE; return NULL;
        }
        t->leaf_symbol[node] = s;
    }
    *rc = ORC_OK;
    return t;
}

/* The decoding tree of the canonical code the lengths define. */
static orc_tree *build_tree(const uint8_t len[256], int *rc) {
    uint32_t code[256];
    *rc = orc_canonical_codes(len, code);
    if (*rc) return NULL;
    return build_tree_from_codes(code, len, rc);
}

/* Prefix-freeness of an explicit code set (code[s] holds len[s] bits, most
 * significant first; len[s] == 0: no code), by tree insertion. */
int orc_codes_prefix_free(const uint32_t code[256], const uint8_t len[256]) {
    int rc;
    orc_tree *t = build_tree_from_codes(code, len, &rc);
    if (t) free(t);
    return rc == ORC_OK;
}

/* Prefix-freeness of the canonical code of the given lengths: false when
 * the lengths admit no prefix code (Kraft sum above 1, or a length above
 * 32), else the tree-insertion check of the canonical codes. */
int orc_is_prefix_free(const uint8_t len[256]) {
    int rc;
    orc_tree *t = build_tree(len, &rc);
    if (t) free(t);
    return rc == ORC_OK;
}

/* Decodes n weights whose codes occupy bits [first_bit, end_bit) of the
 * stream.  Exponents come from the bit-serial tree walk, sign and mantissa
 * from their byte, and the BF16 word is reassembled.  Fails if the stream
 * hits a missing branch or does not end exactly at end_bit.  (A piece of a
 * stream that starts at a thread block's first code -- its bit offset is
 * the block's first bit plus its first thread's gap -- decodes on its own,
 * which is what lets the GPU kernel's thread blocks work independently.) */
int orc_decode_range(const uint8_t *enc, uint64_t first_bit, uint64_t end_bit, const uint8_t *sm, uint64_t n,
                     const uint8_t len[256], uint16_t *out) {
    int rc;
    if (n == 0) return end_bit == first_bit ? ORC_OK : ORC_ERR_CORRUPT;
    if (end_bit < first_bit) return ORC_ERR_ARG;
    orc_tree *t = build_tree(len, &rc);
    if (!t) return rc;
    const uint64_t total_bits = end_bit;
    uint64_t pos = first_bit, i = 0;
    int node = 0;
    while (i < n) {
        if (pos >= total_bits) { free(t); return ORC_ERR_CORRUPT; }
        node = t->child[node][get_bit(enc, pos++)];
        if (node < 0) { free(t); return ORC_ERR_CORRUPT; }
        if (t->leaf_symbol[node] >= 0) {
            unsigned e = (unsigned)t->leaf_symbol[node];
            out[i] = bf16_from_fields(sm[i] >> 7, e, sm[i] & 0x7Fu);
            ++i;
            node = 0;
        }
    }
    free(t);
    return pos == total_bits ? ORC_OK : ORC_ERR_CORRUPT;
}

/* Decodes a whole stream: n weights from bits [0, total_bits). */
int orc_decode(const uint8_t *enc, uint64_t total_bits, const uint8_t *sm, uint64_t n,
               const uint8_t len[256], uint16_t *out) {
    return orc_decode_range(enc, 0, total_bits, sm, n, len, out);
}

/* ---------------------------------------------------------------------
 * Auxiliary data [P4 << Noyau GPU en deux etapes et metadonnees
 * auxiliaires >>]: thread t owns n bytes of EncodedExponent; Gaps[t] is the
 * bit offset of the first code starting in its range; only the output index
 * of the first element of every thread block is stored.
 *
 * Recomputed here from the stream alone, by walking it bit by bit.
 * gaps: n_blocks * threads_per_block bytes (one value per thread, unpacked)
 * counts: same length, codes starting in each thread's range
 * block_start: n_blocks + 1 entries.
 * ------------------------------------------------------------------- */
int orc_aux(const uint8_t *enc, uint64_t total_bits, uint64_t n, const uint8_t len[256],
            uint32_t bytes_per_thread, uint32_t threads_per_block,
            uint8_t *gaps, uint32_t *counts, uint32_t *block_start,
            uint64_t *n_threads_out, uint64_t *n_blocks_out) {
    int rc;
    const uint64_t span = 8ull * bytes_per_thread; /* bits per thread */
    const uint64_t n_threads = (total_bits + span - 1) / span;
    const uint64_t n_blocks = (n_threads + threads_per_block - 1) / threads_per_block;
    if (n_threads_out) *n_threads_out = n_threads;
    if (n_blocks_out) *n_blocks_out = n_blocks;
    if (!gaps || !counts || !block_start) return ORC_OK; /* size query */
    const uint64_t padded = n_blocks * threads_per_block;
    for (uint64_t t = 0; t < padded; ++t) { gaps[t] = 0; counts[t] = 0; }
    uint64_t need_gap = 0; /* next thread whose gap is not known yet */
    if (n) {
        orc_tree *tr = build_tree(len, &rc);
        if (!tr) return rc;
        uint64_t pos = 0, start = 0, produced = 0;
        int node = 0;
        while (produced < n) {
            if (node == 0) {
                start = pos; /* a code starts here */
                while (need_gap < n_threads && need_gap * span <= start) {
                    gaps[need_gap] = (uint8_t)(start - need_gap * span);
                    ++need_gap;
                }
                counts[start / span] += 1;
            }
            if (pos >= total_bits) { free(tr); return ORC_ERR_CORRUPT; }
            node = tr->child[node][get_bit(enc, pos++)];
            if (node < 0) { free(tr); return ORC_ERR_CORRUPT; }
            if (tr->leaf_symbol[node] >= 0) { ++produced; node = 0; }
        }
        free(tr);
        if (pos != total_bits) return ORC_ERR_CORRUPT;
    }
    /* the end of the stream counts as a code start */
    while (need_gap < n_threads) {
        gaps[need_gap] = (uint8_t)(total_bits - need_gap * span);
        ++need_gap;
    }
    uint64_t acc = 0;
    for (uint64_t b = 0; b < n_blocks; ++b) {
        block_start[b] = (uint32_t)acc;
        for (uint64_t t = b * threads_per_block; t < (b + 1) * threads_per_block; ++t) acc += counts[t];
    }
    block_start[n_blocks] = (uint32_t)acc;
    return acc == n ? ORC_OK : ORC_ERR_CORRUPT;
}

/* Gaps packed as 5-bit fields, MSB-first, in thread order. */
void orc_pack_gaps(const uint8_t *gaps, uint64_t count, uint8_t *out, uint64_t out_bytes) {
    memset(out, 0, (size_t)out_bytes);
    for (uint64_t t = 0; t < count; ++t)
        for (int b = 4; b >= 0; --b)
            put_bit(out, 5 * t + (uint64_t)(4 - b), (gaps[t] >> b) & 1u);
}

/* Reads one 5-bit gap field back (used to check a packed array). */
unsigned orc_read_gap(const uint8_t *packed, uint64_t t) {
    unsigned v = 0;
    for (int b = 0; b < 5; ++b) v = (v << 1) | get_bit(packed, 5 * t + (uint64_t)b);
    return v;
}
