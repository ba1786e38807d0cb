// df11_host.cpp -- host side of libdf11: the encoder/packer and the aux
// planner (exponent histogram, length-limited optimal canonical code,
// EncodedExponent / PackedSignMantissa packing, Gaps, per-block output
// positions, decode tables).
//
// Sources: "DFloat11 : compression sans perte pour l'inference GPU qui reduit
// les LLM a 70 % de leur taille" (fr.news.hada.io), sections
// << Le format DFloat11 >> (Huffman code of the exponent, built from the
// exponent distribution; exponents bit-packed into EncodedExponent; sign
// and mantissa kept apart in PackedSignMantissa), << Noyau GPU en deux
// etapes et metadonnees auxiliaires >> (n bytes per thread, Gaps in 5 bits,
// output position stored per thread block only) and << Decodage fonde sur
// des LUT hierarchiques >> (small lookup tables instead of one 2^L table).
//
// The work is split over host threads: the histogram, the packing and the
// aux positions are all computed per chunk of elements, with chunk bit
// offsets from a prefix sum.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

#include "df11.h"
#include "df11_internal.h"

namespace {

using df11::kBytesPerThread;
using df11::kThreadsPerBlockFmt;

unsigned worker_count() {
    unsigned n = std::thread::hardware_concurrency();
    if (n == 0) n = 1;
    const char *env = std::getenv("DF11_HOST_THREADS");
    if (env) {
        long v = std::strtol(env, nullptr, 10);
        if (v >= 1 && v <= 1024) n = (unsigned)v;
    }
    return std::min(n, 128u);
}

// Runs fn(i) for i in [0, n) on up to worker_count() threads.
template <class F>
void parallel_tasks(size_t n, F fn) {
    if (n == 0) return;
    unsigned nw = std::min<size_t>(worker_count(), n);
    if (nw <= 1) {
        for (size_t i = 0; i < n; ++i) fn(i);
        return;
    }
    std::atomic<size_t> next{0};
    std::vector<std::thread> pool;
    pool.reserve(nw);
    for (unsigned w = 0; w < nw; ++w)
        pool.emplace_back([&] {
            for (size_t i = next++; i < n; i = next++) fn(i);
        });
    for (auto &t : pool) t.join();
}

// k matrices seen as one sequence of BF16 words.
struct Sequence {
    const uint16_t *const *mats;
    const uint64_t *sizes;
    uint32_t k;
    std::vector<uint64_t> start;  // start[j] = first global index of matrix j
    uint64_t n = 0;

    Sequence(const uint16_t *const *m, const uint64_t *s, uint32_t kk) : mats(m), sizes(s), k(kk) {
        start.resize(kk + 1);
        for (uint32_t j = 0; j < kk; ++j) {
            start[j] = n;
            n += s[j];
        }
        start[kk] = n;
    }
    // Calls fn(ptr, global_index, count) for the pieces of [lo, hi).
    template <class F>
    void segments(uint64_t lo, uint64_t hi, F fn) const {
        if (lo >= hi) return;
        uint32_t j = (uint32_t)(std::upper_bound(start.begin(), start.end(), lo) - start.begin()) - 1;
        while (lo < hi && j < k) {
            uint64_t end = std::min(hi, start[j + 1]);
            if (end > lo) fn(mats[j] + (lo - start[j]), lo, end - lo);
            lo = end;
            ++j;
        }
    }
};

constexpr uint64_t kChunk = 1ull << 20;  // elements per host work item

inline unsigned exponent_of(uint16_t w) { return (w >> 7) & 0xFFu; }

// ------------------------------------------------------------ histogram
void histogram(const Sequence &seq, uint64_t count[256]) {
    size_t n_chunks = (size_t)((seq.n + kChunk - 1) / kChunk);
    std::vector<uint64_t> part(n_chunks * 256, 0);
    parallel_tasks(n_chunks, [&](size_t c) {
        uint64_t local[4][256] = {};
        seq.segments(c * kChunk, std::min<uint64_t>(seq.n, (c + 1) * kChunk),
                     [&](const uint16_t *p, uint64_t, uint64_t cnt) {
                         uint64_t i = 0;
                         for (; i + 4 <= cnt; i += 4) {
                             local[0][exponent_of(p[i])]++;
                             local[1][exponent_of(p[i + 1])]++;
                             local[2][exponent_of(p[i + 2])]++;
                             local[3][exponent_of(p[i + 3])]++;
                         }
                         for (; i < cnt; ++i) local[0][exponent_of(p[i])]++;
                     });
        for (int s = 0; s < 256; ++s)
            part[c * 256 + s] = local[0][s] + local[1][s] + local[2][s] + local[3][s];
    });
    for (int s = 0; s < 256; ++s) count[s] = 0;
    for (size_t c = 0; c < n_chunks; ++c)
        for (int s = 0; s < 256; ++s) count[s] += part[c * 256 + s];
}

// ------------------------------------------------------------ code lengths
// Huffman with the two-queue method: leaves sorted by (count, symbol), merged
// nodes appended to a second queue in non-decreasing weight order.
void huffman_lengths(const uint64_t count[256], uint8_t len[256]) {
    struct Leaf { uint64_t w; int sym; };
    std::vector<Leaf> leaves;
    for (int s = 0; s < 256; ++s)
        if (count[s]) leaves.push_back({count[s], s});
    std::memset(len, 0, 256);
    if (leaves.empty()) return;
    if (leaves.size() == 1) { len[leaves[0].sym] = 1; return; }
    std::stable_sort(leaves.begin(), leaves.end(), [](const Leaf &a, const Leaf &b) { return a.w < b.w; });
    const int nl = (int)leaves.size();
    // node ids: 0..nl-1 leaves, nl.. internal
    std::vector<uint64_t> weight(2 * nl);
    std::vector<int> parent(2 * nl, -1);
    for (int i = 0; i < nl; ++i) weight[i] = leaves[i].w;
    int qa = 0;            // next unused leaf
    int qb = nl, qe = nl;  // internal queue [qb, qe)
    auto pop_min = [&]() {
        if (qa < nl && (qb >= qe || weight[qa] <= weight[qb])) return qa++;
        return qb++;
    };
    while ((nl - qa) + (qe - qb) > 1) {
        int a = pop_min(), b = pop_min();
        weight[qe] = weight[a] + weight[b];
        parent[a] = parent[b] = qe;
        ++qe;
    }
    const int root = qe - 1;
    std::vector<int> depth(2 * nl, 0);
    for (int v = root - 1; v >= 0; --v) depth[v] = depth[parent[v]] + 1;  // parents have larger ids
    for (int i = 0; i < nl; ++i) len[leaves[i].sym] = (uint8_t)std::min(depth[i], 255);
}

// Length-limited optimal lengths by package-merge (Larmore & Hirschberg):
// coins of denominations 2^-1..2^-cap per symbol; packages built bottom-up
// from the smallest denomination; the 2K-2 cheapest items of the 2^-1 list
// are selected and a symbol's length is the number of its coins selected.
// Items are kept in a node pool (leaf coin or package of two items) and the
// selection is expanded by walking packages.
bool package_merge_lengths(const uint64_t count[256], int cap, uint8_t len[256]) {
    struct Item { uint64_t w; int sym; int a; int b; };  // sym >= 0: coin; else package (a, b)
    std::vector<int> syms;
    for (int s = 0; s < 256; ++s)
        if (count[s]) syms.push_back(s);
    std::memset(len, 0, 256);
    const int k = (int)syms.size();
    if (k == 0) return true;
    if (k == 1) { len[syms[0]] = 1; return true; }
    if (cap < 32 && (uint64_t)k > (1ull << cap)) return false;
    std::stable_sort(syms.begin(), syms.end(), [&](int x, int y) { return count[x] < count[y]; });
    std::vector<Item> pool;
    pool.reserve((size_t)cap * 2 * k + k);
    std::vector<int> cur;
    for (int s : syms) { cur.push_back((int)pool.size()); pool.push_back({count[s], s, -1, -1}); }
    for (int level = cap - 1; level >= 1; --level) {
        std::vector<int> packs;
        for (size_t i = 0; i + 1 < cur.size(); i += 2) {
            packs.push_back((int)pool.size());
            pool.push_back({pool[cur[i]].w + pool[cur[i + 1]].w, -1, cur[i], cur[i + 1]});
        }
        std::vector<int> merged;
        merged.reserve(k + packs.size());
        size_t ia = 0, ib = 0;
        while (ia < (size_t)k || ib < packs.size()) {
            bool take_coin = ib >= packs.size() ||
                             (ia < (size_t)k && count[syms[ia]] <= pool[packs[ib]].w);
            if (take_coin) { merged.push_back((int)pool.size()); pool.push_back({count[syms[ia]], syms[ia], -1, -1}); ++ia; }
            else merged.push_back(packs[ib++]);
        }
        cur.swap(merged);
    }
    std::vector<int> stack;
    for (int i = 0; i < 2 * k - 2; ++i) {
        stack.push_back(cur[i]);
        while (!stack.empty()) {
            int v = stack.back();
            stack.pop_back();
            if (pool[v].sym >= 0) ++len[pool[v].sym];
            else { stack.push_back(pool[v].a); stack.push_back(pool[v].b); }
        }
    }
    return true;
}

// Canonical codes by (length, symbol), via per-length counts (RFC 1951
// section 3.2.2: bl_count, then next_code[l] = (next_code[l-1] +
// bl_count[l-1]) << 1).
void canonical_codes(const uint8_t len[256], uint32_t code[256], uint64_t first_out[34],
                     uint32_t cnt_out[34]) {
    uint32_t bl_count[34] = {};
    for (int s = 0; s < 256; ++s) bl_count[len[s]]++;
    bl_count[0] = 0;
    uint64_t next[34] = {};
    uint64_t c = 0;
    for (int l = 1; l <= 33; ++l) {
        c = (c + bl_count[l - 1]) << 1;
        next[l] = c;
    }
    // RFC 1951 starts at code 0 for the shortest length: next[1] = 0.
    for (int l = 1; l <= 33; ++l) {
        first_out[l] = next[l];
        cnt_out[l] = bl_count[l];
    }
    first_out[0] = 0;
    cnt_out[0] = 0;
    for (int s = 0; s < 256; ++s)
        code[s] = len[s] ? (uint32_t)(next[len[s]]++) : 0u;
}

// ------------------------------------------------------------ decode tables
struct FirstCode { int len; int sym_index; };

// Length of the code at the top of a left-aligned 32-bit window, or -1 if
// no code matches (possible only for an incomplete code).
inline int code_length(uint32_t x, const uint64_t lim[33], int max_len) {
    for (int l = 1; l <= max_len; ++l)
        if ((uint64_t)x < lim[l]) return l;
    return -1;
}

void build_luts(const uint8_t len[256], uint8_t *lut) {
    std::memset(lut, 0, df11::kLutBytes);
    uint32_t code[256];
    uint64_t first[34];
    uint32_t cnt[34];
    canonical_codes(len, code, first, cnt);
    int max_len = 0, min_len = 33, n_syms = 0;
    for (int s = 0; s < 256; ++s)
        if (len[s]) { max_len = std::max(max_len, (int)len[s]); min_len = std::min(min_len, (int)len[s]); ++n_syms; }
    if (n_syms == 0) { max_len = 1; min_len = 1; }
    df11::LutHeader h{};
    h.magic = df11::kMagic;
    h.w1 = (uint32_t)std::min(df11::kW1Max, max_len);
    h.w2 = (uint32_t)std::min(df11::kW2Max, max_len);
    h.max_len = (uint32_t)max_len;
    h.min_len = (uint32_t)min_len;
    h.n_syms = (uint32_t)n_syms;
    h.w1_max = (uint32_t)df11::kW1Max;
    h.w2_max = (uint32_t)df11::kW2Max;
    std::memcpy(lut + df11::kOffHeader, &h, sizeof(h));

    uint64_t lim[33] = {};
    uint32_t offs[33] = {};
    uint32_t base = 0;  // symbols with a shorter code
    for (int l = 1; l <= 32; ++l) {
        lim[l] = (first[l] + cnt[l]) << (32 - l);
        offs[l] = (uint32_t)(base - (uint32_t)first[l]);
        base += cnt[l];
    }
    std::memcpy(lut + df11::kOffLim, lim, sizeof(lim));
    std::memcpy(lut + df11::kOffOffs, offs, sizeof(offs));
    // symbols in canonical order, stored rotated
    uint8_t *sym_rot = lut + df11::kOffSymRot;
    int idx = 0;
    for (int l = 1; l <= 32; ++l)
        for (int s = 0; s < 256; ++s)
            if (len[s] == l) sym_rot[idx++] = (uint8_t)df11::rotate_exponent((uint32_t)s);

    auto symbol_at = [&](uint32_t x, int l) -> uint32_t {
        uint32_t i = (x >> (32 - l)) + offs[l];
        return sym_rot[i & 255];
    };
    // count LUT (entries past 2^w1 are never indexed; they hold the escape)
    uint32_t *clut = reinterpret_cast<uint32_t *>(lut + df11::kOffCountLut);
    for (uint32_t v = 0; v < (1u << df11::kW1Max); ++v) clut[v] = df11::kEscape;
    for (uint32_t v = 0; v < (1u << h.w1); ++v) {
        const uint32_t x = v << (32 - h.w1);
        uint32_t pos = 0, n = 0;
        while (pos < h.w1) {
            int l = code_length(x << pos, lim, max_len);
            if (l < 0 || (uint32_t)l > h.w1 - pos) break;
            pos += (uint32_t)l;
            ++n;
        }
        clut[v] = n ? df11::count_entry(pos, n) : df11::kEscape;
    }
    // symbol LUT (same for entries past 2^w2)
    uint32_t *slut = reinterpret_cast<uint32_t *>(lut + df11::kOffSymLut);
    for (uint32_t v = 0; v < (1u << df11::kW2Max); ++v) {
        slut[2 * v] = 0u;
        slut[2 * v + 1] = df11::kEscape;
    }
    for (uint32_t v = 0; v < (1u << h.w2); ++v) {
        const uint32_t x = v << (32 - h.w2);
        uint32_t pos = 0, n = 0, syms = 0;
        while (pos < h.w2 && n < (uint32_t)df11::kSymsPerEntry) {
            int l = code_length(x << pos, lim, max_len);
            if (l < 0 || (uint32_t)l > h.w2 - pos) break;
            syms |= symbol_at(x << pos, l) << (8 * n);
            pos += (uint32_t)l;
            ++n;
        }
        slut[2 * v] = n ? syms : 0u;
        slut[2 * v + 1] = n ? df11::sym_entry_meta(pos, n) : df11::kEscape;
    }
}

// ------------------------------------------------------------ sizes
df11_status fill_sizes(const Sequence &seq, const df11_params *params, df11_tensor *t) {
    df11_params p;
    df11_default_params(&p);
    if (params) p = *params;
    if (p.max_code_len < 1 || p.max_code_len > 32 || p.reserved != 0) return DF11_ERR_INVALID_ARG;
    if (p.bytes_per_thread != (uint32_t)kBytesPerThread || p.threads_per_block != (uint32_t)kThreadsPerBlockFmt)
        return DF11_ERR_UNSUPPORTED;
    if (seq.n > 0xFFFFFFFFull) return DF11_ERR_TOO_LARGE;
    uint64_t count[256];
    histogram(seq, count);
    return df11::plan_from_histogram(count, seq.n, p, t);
}

}  // namespace

// Code lengths, sizes and scalar fields of a tensor from its exponent
// histogram (shared by the host encoder and the device encoder).
df11_status df11::plan_from_histogram(const uint64_t count[256], uint64_t n, const df11_params &p, df11_tensor *t) {
    uint64_t total = 0;
    for (int s = 0; s < 256; ++s) total += count[s];
    if (total != n) return DF11_ERR_INVALID_ARG;
    uint8_t len[256];
    huffman_lengths(count, len);
    int mx = 0;
    for (int s = 0; s < 256; ++s) mx = std::max(mx, (int)len[s]);
    if (mx > (int)p.max_code_len) {
        if (!package_merge_lengths(count, (int)p.max_code_len, len)) return DF11_ERR_INVALID_ARG;
    }
    uint64_t bits = 0;
    for (int s = 0; s < 256; ++s) bits += count[s] * len[s];
    const uint64_t span = 8ull * kBytesPerThread;
    std::memset(t, 0, offsetof(df11_tensor, enc));
    t->n_elems = n;
    t->total_bits = bits;
    t->n_threads = (bits + span - 1) / span;
    t->n_blocks = (t->n_threads + kThreadsPerBlockFmt - 1) / kThreadsPerBlockFmt;
    t->params = p;
    std::memcpy(t->code_len, len, 256);
    const uint64_t padded_threads = t->n_blocks * kThreadsPerBlockFmt;
    t->enc_bytes = padded_threads * kBytesPerThread + 16;
    t->sm_bytes = ((n + 15) / 16) * 16 + 16;
    t->gaps_bytes = ((padded_threads * 5 + 7) / 8 + 15) / 16 * 16 + 16;
    t->block_start_bytes = ((t->n_blocks + 1) * 4 + 15) / 16 * 16 + 16;
    t->lut_bytes = df11::kLutBytes;
    t->counts_bytes = padded_threads + 16;
    return DF11_OK;
}

void df11::host_build_luts(const uint8_t len[256], uint8_t *lut) { build_luts(len, lut); }
void df11::host_canonical_codes(const uint8_t len[256], uint32_t code[256]) {
    uint64_t first[34];
    uint32_t cnt[34];
    canonical_codes(len, code, first, cnt);
}

namespace {

// ------------------------------------------------------------ packing
df11_status fill_arrays(const Sequence &seq, df11_tensor *t) {
    if (!t || !t->enc || !t->sm || !t->gaps || !t->block_start || !t->lut) return DF11_ERR_INVALID_ARG;
    if (t->n_elems != seq.n) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    uint32_t code[256];
    uint64_t first[34];
    uint32_t cnt[34];
    canonical_codes(t->code_len, code, first, cnt);
    const uint8_t *len = t->code_len;
    const uint64_t n = seq.n;
    const uint64_t span = 8ull * kBytesPerThread;
    const uint64_t block_span = span * kThreadsPerBlockFmt;
    const uint64_t n_threads = t->n_threads, n_blocks = t->n_blocks;

    // pass 1: bits per chunk (and a check that every exponent has a code)
    const size_t n_chunks = (size_t)((n + kChunk - 1) / kChunk);
    std::vector<uint64_t> chunk_bits(n_chunks + 1, 0);
    std::atomic<bool> missing{false};
    parallel_tasks(n_chunks, [&](size_t c) {
        uint64_t b = 0;
        seq.segments(c * kChunk, std::min<uint64_t>(n, (c + 1) * kChunk),
                     [&](const uint16_t *p, uint64_t, uint64_t m) {
                         for (uint64_t i = 0; i < m; ++i) {
                             unsigned l = len[exponent_of(p[i])];
                             if (!l) missing = true;
                             b += l;
                         }
                     });
        chunk_bits[c + 1] = b;
    });
    if (missing) return DF11_ERR_INVALID_ARG;
    for (size_t c = 0; c < n_chunks; ++c) chunk_bits[c + 1] += chunk_bits[c];
    if (chunk_bits[n_chunks] != t->total_bits) return DF11_ERR_INVALID_ARG;

    // pass 2: write codes, sign/mantissa bytes, gaps and block starts
    std::vector<uint8_t> gaps((size_t)(n_blocks * kThreadsPerBlockFmt), 0);
    // Bytes a chunk shares with its neighbours are kept aside and OR-ed in
    // afterwards: head = first byte when the chunk starts mid-byte, tail =
    // last partial byte when it ends mid-byte.
    std::vector<uint8_t> head(n_chunks, 0), tail(n_chunks, 0), head_set(n_chunks, 0);
    // Per-thread code counts (when asked for): a chunk writes the counts of
    // the threads only it starts codes in; its first and last runs (threads
    // it may share with its neighbours) are kept aside and added afterwards.
    uint8_t *counts = t->counts;
    if (counts) std::memset(counts, 0, (size_t)t->counts_bytes);
    constexpr uint64_t kNoThread = ~0ull;
    std::vector<uint64_t> run_first_t(n_chunks, kNoThread), run_last_t(n_chunks, kNoThread);
    std::vector<uint32_t> run_first_n(n_chunks, 0), run_last_n(n_chunks, 0);
    uint8_t *enc = t->enc;
    uint8_t *sm = t->sm;
    uint32_t *bstart = t->block_start;
    parallel_tasks(n_chunks, [&](size_t c) {
        const uint64_t lo = c * kChunk, hi = std::min<uint64_t>(n, (c + 1) * kChunk);
        const uint64_t b0 = chunk_bits[c], b1 = chunk_bits[c + 1];
        uint64_t tn = (b0 + span - 1) / span;              // next thread needing a gap
        uint64_t bn = (b0 + block_span - 1) / block_span;  // next block needing a start
        uint64_t pos = b0;
        uint64_t acc = 0;
        unsigned nacc = (unsigned)(b0 & 7);
        uint8_t *dst = enc + (b0 >> 3);
        bool at_head = (b0 & 7) != 0;
        uint64_t run_t = kNoThread;  // thread of the current run of code starts
        uint32_t run_n = 0;
        seq.segments(lo, hi, [&](const uint16_t *p, uint64_t g0, uint64_t m) {
            for (uint64_t i = 0; i < m; ++i) {
                const uint16_t w = p[i];
                const unsigned e = exponent_of(w);
                const unsigned l = len[e];
                if (counts) {
                    const uint64_t th = pos / span;
                    if (th != run_t) {
                        if (run_t != kNoThread) {
                            if (run_first_t[c] == kNoThread) { run_first_t[c] = run_t; run_first_n[c] = run_n; }
                            else counts[run_t] = (uint8_t)run_n;
                        }
                        run_t = th;
                        run_n = 0;
                    }
                    ++run_n;
                }
                while (tn < n_threads && tn * span <= pos) { gaps[tn] = (uint8_t)(pos - tn * span); ++tn; }
                while (bn < n_blocks && bn * block_span <= pos) { bstart[bn] = (uint32_t)(g0 + i); ++bn; }
                sm[g0 + i] = (uint8_t)(((w >> 8) & 0x80u) | (w & 0x7Fu));
                acc = (acc << l) | code[e];
                nacc += l;
                pos += l;
                while (nacc >= 8) {
                    nacc -= 8;
                    const uint8_t byte = (uint8_t)(acc >> nacc);
                    if (at_head) { head[c] = byte; head_set[c] = 1; at_head = false; ++dst; }
                    else *dst++ = byte;
                }
            }
        });
        // threads / blocks whose first code start is the next chunk's first code
        while (tn < n_threads && tn * span < b1) { gaps[tn] = (uint8_t)(b1 - tn * span); ++tn; }
        while (bn < n_blocks && bn * block_span < b1) { bstart[bn] = (uint32_t)hi; ++bn; }
        if (nacc) tail[c] = (uint8_t)(acc << (8 - nacc));
        else tail[c] = 0;
        if (counts && run_t != kNoThread) {
            if (run_first_t[c] == kNoThread) { run_first_t[c] = run_t; run_first_n[c] = run_n; }
            else { run_last_t[c] = run_t; run_last_n[c] = run_n; }
        }
        (void)dst;
    });
    if (counts)
        for (size_t c = 0; c < n_chunks; ++c) {
            if (run_first_t[c] != kNoThread) counts[run_first_t[c]] = (uint8_t)(counts[run_first_t[c]] + run_first_n[c]);
            if (run_last_t[c] != kNoThread) counts[run_last_t[c]] = (uint8_t)(counts[run_last_t[c]] + run_last_n[c]);
        }
    // Shared bytes are never written whole by any chunk: clear them, then OR
    // in every partial contribution (a chunk that never completed its first
    // byte has all of its bits in its tail).
    for (size_t c = 0; c < n_chunks; ++c) {
        const uint64_t b0 = chunk_bits[c], b1 = chunk_bits[c + 1];
        if (b0 & 7) enc[b0 >> 3] = 0;
        if (b1 & 7) enc[b1 >> 3] = 0;
    }
    for (size_t c = 0; c < n_chunks; ++c) {
        const uint64_t b0 = chunk_bits[c], b1 = chunk_bits[c + 1];
        if ((b0 & 7) && head_set[c]) enc[b0 >> 3] |= head[c];
        if (b1 & 7) enc[b1 >> 3] |= tail[c];
    }
    const uint64_t used = (t->total_bits + 7) / 8;
    std::memset(enc + used, 0, (size_t)(t->enc_bytes - used));
    std::memset(sm + n, 0, (size_t)(t->sm_bytes - n));
    bstart[n_blocks] = (uint32_t)n;
    uint32_t most = 0;
    for (uint64_t b = 0; b < n_blocks; ++b) most = std::max(most, bstart[b + 1] - bstart[b]);
    t->max_block_codes = most;
    std::memset(bstart + n_blocks + 1, 0, (size_t)(t->block_start_bytes - 4 * (n_blocks + 1)));

    // gaps: eight 5-bit fields = five bytes, MSB-first
    uint8_t *pg = t->gaps;
    std::memset(pg, 0, (size_t)t->gaps_bytes);
    const uint64_t n_groups = (uint64_t)gaps.size() / 8;
    parallel_tasks((size_t)((n_groups + 65535) / 65536), [&](size_t c) {
        const uint64_t g_lo = (uint64_t)c * 65536, g_hi = std::min<uint64_t>(n_groups, g_lo + 65536);
        for (uint64_t g = g_lo; g < g_hi; ++g) {
            uint64_t v = 0;
            for (int j = 0; j < 8; ++j) v = (v << 5) | (gaps[8 * g + j] & 31u);
            uint8_t *o = pg + 5 * g;
            o[0] = (uint8_t)(v >> 32); o[1] = (uint8_t)(v >> 24); o[2] = (uint8_t)(v >> 16);
            o[3] = (uint8_t)(v >> 8); o[4] = (uint8_t)v;
        }
    });
    build_luts(len, t->lut);
    return DF11_OK;
}

}  // namespace

extern "C" {

uint32_t df11_abi_version(void) { return DF11_ABI_VERSION; }
size_t df11_sizeof_tensor(void) { return sizeof(df11_tensor); }

void df11_default_params(df11_params *p) {
    if (!p) return;
    p->max_code_len = 12;
    p->bytes_per_thread = (uint32_t)kBytesPerThread;
    p->threads_per_block = (uint32_t)kThreadsPerBlockFmt;
    p->reserved = 0;
}

const char *df11_status_str(df11_status s) {
    switch (s) {
        case DF11_OK: return "ok";
        case DF11_ERR_INVALID_ARG: return "invalid argument";
        case DF11_ERR_UNSUPPORTED: return "unsupported parameter";
        case DF11_ERR_TOO_LARGE: return "tensor too large (more than 2^32-1 elements)";
        case DF11_ERR_CORRUPT: return "corrupt compressed data";
        case DF11_ERR_CUDA: return "CUDA error";
        case DF11_ERR_NOMEM: return "out of host memory";
    }
    return "unknown status";
}

df11_status df11_exponent_histogram(const uint16_t *const *mats, const uint64_t *sizes, uint32_t k,
                                    uint64_t count[256]) {
    if (!count || (k && (!mats || !sizes))) return DF11_ERR_INVALID_ARG;
    for (uint32_t j = 0; j < k; ++j)
        if (sizes[j] && !mats[j]) return DF11_ERR_INVALID_ARG;
    try {
        Sequence seq(mats, sizes, k);
        histogram(seq, count);
    } catch (...) {
        return DF11_ERR_NOMEM;
    }
    return DF11_OK;
}

df11_status df11_encode_multi_size(const uint16_t *const *mats, const uint64_t *sizes, uint32_t k,
                                   const df11_params *params, df11_tensor *t) {
    if (!t || (k && (!mats || !sizes))) return DF11_ERR_INVALID_ARG;
    for (uint32_t j = 0; j < k; ++j)
        if (sizes[j] && !mats[j]) return DF11_ERR_INVALID_ARG;
    try {
        Sequence seq(mats, sizes, k);
        return fill_sizes(seq, params, t);
    } catch (...) {
        return DF11_ERR_NOMEM;
    }
}

df11_status df11_encode_multi(const uint16_t *const *mats, const uint64_t *sizes, uint32_t k,
                              df11_tensor *t) {
    if (!t || (k && (!mats || !sizes))) return DF11_ERR_INVALID_ARG;
    for (uint32_t j = 0; j < k; ++j)
        if (sizes[j] && !mats[j]) return DF11_ERR_INVALID_ARG;
    try {
        Sequence seq(mats, sizes, k);
        return fill_arrays(seq, t);
    } catch (...) {
        return DF11_ERR_NOMEM;
    }
}

df11_status df11_encode_size(const uint16_t *bf16, uint64_t n, const df11_params *params,
                             df11_tensor *t) {
    const uint16_t *mats[1] = {bf16};
    uint64_t sizes[1] = {n};
    return df11_encode_multi_size(mats, sizes, 1, params, t);
}

df11_status df11_encode(const uint16_t *bf16, uint64_t n, df11_tensor *t) {
    const uint16_t *mats[1] = {bf16};
    uint64_t sizes[1] = {n};
    return df11_encode_multi(mats, sizes, 1, t);
}

// Tile order (the fused decode -> GEMM's element order): 128 x 64 tiles, row
// tiles in order, the k-tiles of a row tile in order, each tile row-major.
df11_status df11_to_tile_order(const uint16_t *w, uint32_t rows, uint32_t cols, uint16_t *out) {
    if (!w || !out) return DF11_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0 || rows % 128u || cols % 64u) return DF11_ERR_UNSUPPORTED;
    const uint32_t kt = cols / 64u;
    parallel_tasks(rows / 128u, [&](size_t rt) {
        for (uint32_t k = 0; k < kt; ++k) {
            uint16_t *dst = out + ((uint64_t)rt * kt + k) * 8192u;
            for (uint32_t r = 0; r < 128u; ++r)
                std::memcpy(dst + 64u * r, w + ((uint64_t)rt * 128u + r) * cols + 64u * k, 128);
        }
    });
    return DF11_OK;
}

df11_status df11_from_tile_order(const uint16_t *tiled, uint32_t rows, uint32_t cols, uint16_t *out) {
    if (!tiled || !out) return DF11_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0 || rows % 128u || cols % 64u) return DF11_ERR_UNSUPPORTED;
    const uint32_t kt = cols / 64u;
    parallel_tasks(rows / 128u, [&](size_t rt) {
        for (uint32_t k = 0; k < kt; ++k) {
            const uint16_t *src = tiled + ((uint64_t)rt * kt + k) * 8192u;
            for (uint32_t r = 0; r < 128u; ++r)
                std::memcpy(out + ((uint64_t)rt * 128u + r) * cols + 64u * k, src + 64u * r, 128);
        }
    });
    return DF11_OK;
}

df11_status df11_validate(const df11_tensor *t) {
    if (!t) return DF11_ERR_INVALID_ARG;
    const df11_params &p = t->params;
    if (p.bytes_per_thread != (uint32_t)kBytesPerThread || p.threads_per_block != (uint32_t)kThreadsPerBlockFmt)
        return DF11_ERR_UNSUPPORTED;
    if (p.max_code_len < 1 || p.max_code_len > 32) return DF11_ERR_INVALID_ARG;
    if (t->n_elems > 0xFFFFFFFFull) return DF11_ERR_TOO_LARGE;
    const uint64_t span = 8ull * kBytesPerThread;
    if (t->n_threads != (t->total_bits + span - 1) / span) return DF11_ERR_CORRUPT;
    if (t->n_blocks != (t->n_threads + kThreadsPerBlockFmt - 1) / kThreadsPerBlockFmt) return DF11_ERR_CORRUPT;
    if (t->total_bits > 32ull * t->n_elems || t->total_bits < (t->n_elems ? t->n_elems : 0))
        return DF11_ERR_CORRUPT;
    const uint64_t padded = t->n_blocks * kThreadsPerBlockFmt;
    if (t->enc_bytes < padded * kBytesPerThread + 16) return DF11_ERR_INVALID_ARG;
    if (t->sm_bytes < ((t->n_elems + 15) / 16) * 16 + 16) return DF11_ERR_INVALID_ARG;
    if (t->gaps_bytes < (padded * 5 + 7) / 8 + 16) return DF11_ERR_INVALID_ARG;
    if (t->block_start_bytes < ((t->n_blocks + 1) * 4 + 15) / 16 * 16 + 16) return DF11_ERR_INVALID_ARG;
    if (t->lut_bytes < df11::kLutBytes) return DF11_ERR_INVALID_ARG;
    if (t->counts && t->counts_bytes < padded + 16) return DF11_ERR_INVALID_ARG;
    if (t->max_block_codes > (uint32_t)df11::kMaxCodesPerBlock || t->reserved2 != 0) return DF11_ERR_CORRUPT;
    // Kraft: sum 2^-len <= 1 and lengths within the cap
    uint64_t kraft = 0;
    int k = 0;
    for (int s = 0; s < 256; ++s) {
        if (!t->code_len[s]) continue;
        if (t->code_len[s] > p.max_code_len) return DF11_ERR_CORRUPT;
        kraft += 1ull << (32 - t->code_len[s]);
        ++k;
    }
    if (kraft > (1ull << 32)) return DF11_ERR_CORRUPT;
    if (t->n_elems && k == 0) return DF11_ERR_CORRUPT;
    return DF11_OK;
}

}  // extern "C"
