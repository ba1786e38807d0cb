// df11_encode.cu -- the encoder on the GPU: exponent histogram, then the
// packing of EncodedExponent, PackedSignMantissa, Gaps and the per-block
// output positions, for weights already in device memory.  Only the code
// lengths (at most 256 symbols) and the decode tables are computed on the
// host, between the two steps, by the same planner as the host encoder, so
// both encoders produce byte-identical arrays.
//
// Sources: "DFloat11 : compression sans perte pour l'inference GPU qui reduit
// les LLM a 70 % de leur taille" (fr.news.hada.io): << Le format DFloat11 >>
// (a Huffman code of the exponent built from the exponent frequencies;
// exponents bit-packed in element order into EncodedExponent; sign and
// mantissa kept apart, one byte per weight, in PackedSignMantissa) and
// << Noyau GPU en deux etapes et metadonnees auxiliaires >> (a thread owns
// n = 8 bytes of the bitstream; Gaps holds, in 5 bits, the offset of the
// first code that starts in each thread's bytes; each thread block of 256
// threads stores the index of its first output element).
//
// Layout of the work: tiles of 8192 elements, one CTA of 256 threads per
// tile, 32 consecutive elements per thread.  The bit offset of every element
// is the tile's offset (an exclusive prefix sum over tiles) plus an in-tile
// prefix sum.  A thread appends its codes MSB-first into 64-bit words kept in
// a register and ORs each finished word into the bitstream (big-endian byte
// order), so only the words it shares with its neighbours see more than one
// writer.  An element whose code start is the first at or after a thread's
// (block's) bit boundary writes that thread's gap (that block's first output
// index); the end of the stream counts as a code start, as in the format.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "df11.h"
#include "df11_internal.h"

namespace {

constexpr uint32_t kTile = 8192;                  // elements per tile
constexpr uint32_t kEncThreads = 256;             // threads per tile
constexpr uint32_t kPer = kTile / kEncThreads;    // elements per thread
constexpr uint64_t kThreadBits = 8ull * df11::kBytesPerThread;                  // 64
constexpr uint64_t kBlockBits = kThreadBits * (uint64_t)df11::kThreadsPerBlockFmt;  // 16384
static_assert(kThreadBits == 64 && kBlockBits == 16384, "bit boundaries are shifts by 6 and 14");

struct CodeTables {
    uint32_t code[256];  // canonical code of each exponent (right-aligned)
    uint8_t len[256];    // its length in bits, 0 = exponent absent
};

// Scratch layout: exponent counts (256 x u64), tile offsets (n_tiles + 1 x
// u64), the largest block's code count (u32) and the total bits (u64).
constexpr uint64_t n_tiles_of(uint64_t n) { return (n + kTile - 1) / kTile; }
constexpr uint64_t kOffCounts = 0;
constexpr uint64_t kOffTiles = 2048;
constexpr uint64_t off_tail(uint64_t n) { return kOffTiles + 8u * (n_tiles_of(n) + 1u); }
constexpr uint64_t scratch_need(uint64_t n) { return ((off_tail(n) + 16u + 15u) / 16u) * 16u; }

__device__ __forceinline__ uint32_t exponent_of(uint32_t w) { return (w >> 7) & 0xFFu; }

// ---------------------------------------------------------------- kernels
// Exponent histogram: 8 sub-histograms per CTA in shared memory (warp w
// adds into sub-histogram w mod 8), then one 64-bit add per bin.
__global__ void __launch_bounds__(256) hist_kernel(const uint16_t *w, uint64_t n, unsigned long long *count) {
    __shared__ uint32_t h[8][256];
    for (uint32_t i = threadIdx.x; i < 8u * 256u; i += blockDim.x) (&h[0][0])[i] = 0u;
    __syncthreads();
    uint32_t *mine = h[(threadIdx.x >> 5) & 7u];
    const uint64_t n8 = n / 8u;
    const uint4 *w8 = reinterpret_cast<const uint4 *>(w);
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(w8 + i);
        const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            atomicAdd(&mine[exponent_of(q[k])], 1u);
            atomicAdd(&mine[exponent_of(q[k] >> 16)], 1u);
        }
    }
    if (blockIdx.x == 0)
        for (uint64_t i = 8u * n8 + threadIdx.x; i < n; i += blockDim.x) atomicAdd(&mine[exponent_of(w[i])], 1u);
    __syncthreads();
    for (uint32_t b = threadIdx.x; b < 256u; b += blockDim.x) {
        uint32_t s = 0;
        for (int k = 0; k < 8; ++k) s += h[k][b];
        if (s) atomicAdd(count + b, (unsigned long long)s);
    }
}

// Block-wide exclusive scan of one value per thread (256 threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t &total) {
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (uint32_t d = 1; d < 32; d <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += x;
    }
    if (lane == 31u) warp_sums[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
    for (uint32_t k = 0; k < kEncThreads / 32u; ++k) {
        const uint32_t s = warp_sums[k];
        if (k < warp) before += s;
        total += s;
    }
    return before + incl - v;
}

// Bits of each tile (written at tile_off[tile + 1]; the scan makes them offsets).
__global__ void __launch_bounds__(kEncThreads) tile_bits_kernel(const uint16_t *w, uint64_t n, const CodeTables ct,
                                                               unsigned long long *tile_off) {
    __shared__ uint8_t len[256];
    __shared__ uint32_t warp_sums[kEncThreads / 32u];
    len[threadIdx.x] = ct.len[threadIdx.x];
    __syncthreads();
    const uint64_t i0 = (uint64_t)blockIdx.x * kTile + (uint64_t)threadIdx.x * kPer;
    uint32_t s = 0;
    for (uint32_t j = 0; j < kPer; ++j)
        if (i0 + j < n) s += len[exponent_of(w[i0 + j])];
    uint32_t total;
    (void)block_exclusive_scan(s, warp_sums, total);
    if (threadIdx.x == 0) tile_off[blockIdx.x + 1u] = total;
}

// In-place inclusive scan of tile_off[1 .. n_tiles] by one CTA of 1024
// threads, chunk by chunk with a running carry (tile_off[0] is 0).
__global__ void __launch_bounds__(1024) scan_tiles_kernel(unsigned long long *tile_off, uint64_t n_tiles) {
    __shared__ unsigned long long warp_sums[32];
    __shared__ unsigned long long carry_s;
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (uint64_t base = 1; base <= n_tiles; base += 1024u) {
        const uint64_t i = base + threadIdx.x;
        unsigned long long v = i <= n_tiles ? tile_off[i] : 0ull;
#pragma unroll
        for (uint32_t d = 1; d < 32; d <<= 1) {
            const unsigned long long x = __shfl_up_sync(0xFFFFFFFFu, v, d);
            if (lane >= d) v += x;
        }
        if (lane == 31u) warp_sums[warp] = v;
        __syncthreads();
        unsigned long long before = carry_s;
        for (uint32_t k = 0; k < warp; ++k) before += warp_sums[k];
        if (i <= n_tiles) tile_off[i] = before + v;
        __syncthreads();
        if (threadIdx.x == 1023u) carry_s = before + v;
        __syncthreads();
    }
}

__device__ __forceinline__ void or_word64(uint8_t *enc, uint64_t enc_words, uint64_t word, uint64_t v) {
    if (v == 0ull || word >= enc_words) return;
    const uint32_t hi = (uint32_t)(v >> 32), lo = (uint32_t)v;
    // big-endian byte order: the most significant byte first in memory
    const unsigned long long be =
        ((unsigned long long)__byte_perm(lo, 0u, 0x0123u) << 32) | (unsigned long long)__byte_perm(hi, 0u, 0x0123u);
    atomicOr(reinterpret_cast<unsigned long long *>(enc + 8u * word), be);
}

// Gap of thread t (5 bits, MSB-first fields) OR-ed into the gaps array.
__device__ __forceinline__ void put_gap(uint8_t *gaps, uint64_t t, uint32_t g) {
    if (g == 0u) return;
    const uint64_t q = 5u * t;  // first bit of the field
    const uint64_t wi = q >> 5;
    const uint32_t o = (uint32_t)(q & 31u);
    uint32_t *gw = reinterpret_cast<uint32_t *>(gaps);
    if (o <= 27u) {
        atomicOr(gw + wi, __byte_perm(g << (27u - o), 0u, 0x0123u));
    } else {
        const uint32_t r = o - 27u;  // bits spilling into the next word
        atomicOr(gw + wi, __byte_perm(g >> r, 0u, 0x0123u));
        atomicOr(gw + wi + 1u, __byte_perm(g << (32u - r), 0u, 0x0123u));
    }
}

struct PackArgs {
    const uint16_t *w;
    uint64_t n;
    uint64_t enc_words;  // 64-bit words of the enc array (writes stay below)
    const unsigned long long *tile_off;
    uint64_t n_threads, n_blocks;
    uint8_t *enc, *sm, *gaps;
    uint32_t *bstart;
    uint32_t *counts;  // per-thread code counts, 4 per word (NULL: not written)
};

// Adds a run of n code starts in format thread t to its count byte (a count
// never passes 64, so the bytes of a word never carry into each other).
__device__ __forceinline__ void add_count(uint32_t *counts, uint64_t t, uint32_t n) {
    if (counts && n) atomicAdd(counts + (t >> 2), n << (8u * (uint32_t)(t & 3u)));
}

__global__ void __launch_bounds__(kEncThreads) pack_kernel(const PackArgs a, const CodeTables ct) {
    __shared__ uint32_t code[256];
    __shared__ uint8_t len[256];
    __shared__ uint32_t warp_sums[kEncThreads / 32u];
    code[threadIdx.x] = ct.code[threadIdx.x];
    len[threadIdx.x] = ct.len[threadIdx.x];
    __syncthreads();
    const uint64_t i0 = (uint64_t)blockIdx.x * kTile + (uint64_t)threadIdx.x * kPer;
    const uint32_t cnt = i0 < a.n ? (a.n - i0 < kPer ? (uint32_t)(a.n - i0) : kPer) : 0u;
    uint32_t wv[kPer];
    uint32_t s = 0;
#pragma unroll
    for (uint32_t j = 0; j < kPer; ++j) {
        wv[j] = j < cnt ? (uint32_t)a.w[i0 + j] : 0u;
        s += j < cnt ? (uint32_t)len[exponent_of(wv[j])] : 0u;
    }
    uint32_t total;
    const uint32_t off = block_exclusive_scan(s, warp_sums, total);
    if (cnt == 0u) return;
    uint64_t p = a.tile_off[blockIdx.x] + off;  // bit offset of this thread's first code
    // start of the previous element's code (the boundary test of the first one)
    uint64_t p_prev = i0 == 0 ? 0ull : p - len[exponent_of(a.w[i0 - 1u])];
    bool first_elem = i0 == 0;

    uint64_t cur = 0, word = p >> 6;
    uint32_t used = (uint32_t)(p & 63u);
    uint64_t run_t = p >> 6;  // format thread of the current run of code starts
    uint32_t run_n = 0;
#pragma unroll
    for (uint32_t j = 0; j < kPer; ++j) {
        if (j >= cnt) break;
        const uint32_t e = exponent_of(wv[j]);
        const uint32_t l = len[e], c = code[e];
        if ((p >> 6) != run_t) {
            add_count(a.counts, run_t, run_n);
            run_t = p >> 6;
            run_n = 0;
        }
        ++run_n;
        // the first code starting at or after a thread / block boundary
        if ((first_elem || (p >> 6) > (p_prev >> 6)) && (p >> 6) < a.n_threads)
            put_gap(a.gaps, p >> 6, (uint32_t)(p & 63u));
        if ((first_elem || (p >> 14) > (p_prev >> 14)) && (p >> 14) < a.n_blocks)
            a.bstart[p >> 14] = (uint32_t)(i0 + j);
        first_elem = false;
        a.sm[i0 + j] = (uint8_t)(((wv[j] >> 8) & 0x80u) | (wv[j] & 0x7Fu));
        if (used + l <= 64u) {
            cur |= (uint64_t)c << (64u - used - l);
            used += l;
            if (used == 64u) {
                or_word64(a.enc, a.enc_words, word, cur);
                ++word;
                cur = 0;
                used = 0;
            }
        } else {
            const uint32_t r = used + l - 64u;  // bits of the code in the next word
            cur |= (uint64_t)c >> r;
            or_word64(a.enc, a.enc_words, word, cur);
            ++word;
            cur = (uint64_t)c << (64u - r);
            used = r;
        }
        p_prev = p;
        p += l;
    }
    if (used) or_word64(a.enc, a.enc_words, word, cur);
    add_count(a.counts, run_t, run_n);
    if (i0 + cnt == a.n) {
        // the end of the stream counts as a code start; then the sentinel
        if ((p >> 6) > (p_prev >> 6) && (p >> 6) < a.n_threads) put_gap(a.gaps, p >> 6, (uint32_t)(p & 63u));
        if ((p >> 14) > (p_prev >> 14) && (p >> 14) < a.n_blocks) a.bstart[p >> 14] = (uint32_t)a.n;
        a.bstart[a.n_blocks] = (uint32_t)a.n;
    }
}

// Largest block's code count, and the stream's total bits (the last tile offset).
__global__ void __launch_bounds__(256) finish_kernel(const uint32_t *bstart, uint64_t n_blocks,
                                                     const unsigned long long *tile_off, uint64_t n_tiles,
                                                     uint32_t *most, unsigned long long *total) {
    uint32_t m = 0;
    for (uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks; b += (uint64_t)gridDim.x * blockDim.x)
        m = max(m, bstart[b + 1u] - bstart[b]);
#pragma unroll
    for (uint32_t d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
    if ((threadIdx.x & 31u) == 0u && m) atomicMax(most, m);
    if (blockIdx.x == 0 && threadIdx.x == 0) *total = tile_off[n_tiles];
}

df11_status check_params(const df11_params *params, df11_params &p) {
    df11_default_params(&p);
    if (params) p = *params;
    if (p.max_code_len < 1 || p.max_code_len > 32 || p.reserved != 0) return DF11_ERR_INVALID_ARG;
    if (p.bytes_per_thread != (uint32_t)df11::kBytesPerThread ||
        p.threads_per_block != (uint32_t)df11::kThreadsPerBlockFmt)
        return DF11_ERR_UNSUPPORTED;
    return DF11_OK;
}

// The weights must live on the current device: the kernels launch there and
// would otherwise read another device's memory (a fault without peer access).
df11_status check_on_current_device(const void *w) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, w) != cudaSuccess) {
        (void)cudaGetLastError();  // clear the (non-sticky) error so later launch checks do not see it
        return DF11_ERR_INVALID_ARG;
    }
    if ((at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) || at.device != dev)
        return DF11_ERR_INVALID_ARG;
    return DF11_OK;
}

int sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

}  // namespace

extern "C" {

uint64_t df11_encode_device_scratch_bytes(uint64_t n) { return scratch_need(n); }

df11_status df11_encode_device_size(const uint16_t *w, uint64_t n, const df11_params *params, df11_tensor *hdr,
                                    void *scratch, uint64_t scratch_bytes, void *stream) {
    if (!hdr || (n > 0 && (!w || !scratch))) return DF11_ERR_INVALID_ARG;
    df11_params p;
    df11_status st = check_params(params, p);
    if (st != DF11_OK) return st;
    if (n > 0xFFFFFFFFull) return DF11_ERR_TOO_LARGE;
    uint64_t count[256] = {0};
    if (n > 0) {
        if (((uintptr_t)w & 15u) || ((uintptr_t)scratch & 15u) || scratch_bytes < scratch_need(n))
            return DF11_ERR_INVALID_ARG;
        st = check_on_current_device(w);
        if (st != DF11_OK) return st;
        const int sms = sm_count();
        if (sms <= 0) return DF11_ERR_CUDA;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        unsigned long long *cnt = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(scratch) + kOffCounts);
        if (cudaMemsetAsync(cnt, 0, 256 * sizeof(unsigned long long), s) != cudaSuccess) return DF11_ERR_CUDA;
        const uint64_t want = (n / 8u + 255u) / 256u;
        const unsigned grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>(want, 4u * (uint64_t)sms));
        hist_kernel<<<grid, 256, 0, s>>>(w, n, cnt);
        if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
        if (cudaMemcpyAsync(count, cnt, sizeof(count), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DF11_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return DF11_ERR_CUDA;
    }
    st = df11::plan_from_histogram(count, n, p, hdr);
    if (st != DF11_OK) return st;
    hdr->enc = hdr->sm = hdr->gaps = hdr->lut = hdr->counts = nullptr;
    hdr->block_start = nullptr;
    return DF11_OK;
}

df11_status df11_encode_device(const uint16_t *w, uint64_t n, df11_tensor *io, void *scratch, uint64_t scratch_bytes,
                               void *stream) {
    if (!io || io->n_elems != n) return DF11_ERR_INVALID_ARG;
    if (!io->enc || !io->sm || !io->gaps || !io->block_start || !io->lut) return DF11_ERR_INVALID_ARG;
    if (((uintptr_t)io->enc & 15u) || ((uintptr_t)io->sm & 15u) || ((uintptr_t)io->gaps & 15u) ||
        ((uintptr_t)io->block_start & 15u) || ((uintptr_t)io->lut & 15u) || ((uintptr_t)io->counts & 15u))
        return DF11_ERR_INVALID_ARG;
    // the scalar fields must be those df11_encode_device_size planned
    {
        df11_tensor chk = *io;
        chk.max_block_codes = 0;
        const df11_status vst = df11_validate(&chk);
        if (vst != DF11_OK) return vst;
    }
    if (n > 0) {  // before anything is enqueued
        if (!w || ((uintptr_t)w & 15u) || !scratch || ((uintptr_t)scratch & 15u) || scratch_bytes < scratch_need(n))
            return DF11_ERR_INVALID_ARG;
        const df11_status dst = check_on_current_device(w);
        if (dst != DF11_OK) return dst;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(io->enc, 0, io->enc_bytes, s) != cudaSuccess ||
        cudaMemsetAsync(io->sm, 0, io->sm_bytes, s) != cudaSuccess ||
        cudaMemsetAsync(io->gaps, 0, io->gaps_bytes, s) != cudaSuccess ||
        cudaMemsetAsync(io->block_start, 0, io->block_start_bytes, s) != cudaSuccess ||
        (io->counts && cudaMemsetAsync(io->counts, 0, io->counts_bytes, s) != cudaSuccess))
        return DF11_ERR_CUDA;
    std::vector<uint8_t> lut(io->lut_bytes);
    df11::host_build_luts(io->code_len, lut.data());
    if (cudaMemcpyAsync(io->lut, lut.data(), io->lut_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return DF11_ERR_CUDA;
    uint32_t most = 0;
    uint64_t total = 0;
    if (n > 0) {
        const int sms = sm_count();
        if (sms <= 0) return DF11_ERR_CUDA;
        CodeTables ct;
        df11::host_canonical_codes(io->code_len, ct.code);
        for (int k = 0; k < 256; ++k) ct.len[k] = io->code_len[k];
        uint8_t *sc = static_cast<uint8_t *>(scratch);
        unsigned long long *tile_off = reinterpret_cast<unsigned long long *>(sc + kOffTiles);
        uint32_t *most_d = reinterpret_cast<uint32_t *>(sc + off_tail(n));
        unsigned long long *total_d = reinterpret_cast<unsigned long long *>(sc + off_tail(n) + 8u);
        const uint64_t n_tiles = n_tiles_of(n);
        if (cudaMemsetAsync(tile_off, 0, 8u * (n_tiles + 1u), s) != cudaSuccess ||
            cudaMemsetAsync(most_d, 0, 16u, s) != cudaSuccess)
            return DF11_ERR_CUDA;
        tile_bits_kernel<<<(unsigned)n_tiles, kEncThreads, 0, s>>>(w, n, ct, tile_off);
        scan_tiles_kernel<<<1, 1024, 0, s>>>(tile_off, n_tiles);
        PackArgs a;
        a.w = w;
        a.n = n;
        a.enc_words = io->enc_bytes / 8u;
        a.tile_off = tile_off;
        a.n_threads = io->n_threads;
        a.n_blocks = io->n_blocks;
        a.enc = io->enc;
        a.sm = io->sm;
        a.gaps = io->gaps;
        a.bstart = io->block_start;
        a.counts = reinterpret_cast<uint32_t *>(io->counts);
        pack_kernel<<<(unsigned)n_tiles, kEncThreads, 0, s>>>(a, ct);
        const uint64_t fb = std::max<uint64_t>(1, std::min<uint64_t>((io->n_blocks + 255u) / 256u, 4u * (uint64_t)sms));
        finish_kernel<<<(unsigned)fb, 256, 0, s>>>(io->block_start, io->n_blocks, tile_off, n_tiles, most_d, total_d);
        if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
        if (cudaMemcpyAsync(&most, most_d, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(&total, total_d, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return DF11_ERR_CUDA;
    }
    if (cudaStreamSynchronize(s) != cudaSuccess) return DF11_ERR_CUDA;  // also keeps `lut` alive for its copy
    if (total != io->total_bits) return DF11_ERR_INVALID_ARG;  // the input changed since the size pass
    io->max_block_codes = most;
    return DF11_OK;
}

}  // extern "C"

// ------------------------------------------------------------ no-alloc entry points
// The same encoder with its scratch in a fixed array of this library
// instead of caller memory, for callers that must not allocate device memory
// (see df11.h).  Inputs of up to kNoAllocMaxElems weights.
namespace {

constexpr uint64_t kNoAllocMaxElems = 1ull << 28;
constexpr uint64_t kNoAllocScratchBytes = scratch_need(kNoAllocMaxElems);
static_assert(kNoAllocScratchBytes == 264224u, "the size the header states");
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the fixed scratch in the current device's context.  In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with cudaGetSymbolAddress, with the device current, on every
// call: a device reset or a re-created primary context reloads the module and
// may move the array, and a cached address would then point at freed memory.
// (The lookup is a host-side table query; the first one on a device loads
// the library's device code, which is why the first call must come before
// any stream capture.)
df11_status noalloc_scratch(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DF11_ERR_CUDA;
    *out = p;
    return DF11_OK;
}

}  // namespace

extern "C" {

uint64_t df11_encode_device_noalloc_max_elems(void) { return kNoAllocMaxElems; }

df11_status df11_encode_device_size_noalloc(const uint16_t *w, uint64_t n, const df11_params *params,
                                            df11_tensor *hdr, void *stream) {
    if (n > kNoAllocMaxElems) return DF11_ERR_TOO_LARGE;
    void *scratch = nullptr;
    const df11_status st = noalloc_scratch(&scratch);
    if (st != DF11_OK) return st;
    return df11_encode_device_size(w, n, params, hdr, scratch, kNoAllocScratchBytes, stream);
}

df11_status df11_encode_device_noalloc(const uint16_t *w, uint64_t n, df11_tensor *io, void *stream) {
    if (n > kNoAllocMaxElems) return DF11_ERR_TOO_LARGE;
    void *scratch = nullptr;
    const df11_status st = noalloc_scratch(&scratch);
    if (st != DF11_OK) return st;
    return df11_encode_device(w, n, io, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
