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
//  * Persistent CTAs, one per SM (1024 threads = 4 groups of 256).  Each
//    group decodes one format block (256 threads x 8 bytes) at a time and
//    strides over the blocks; the decode tables are staged into shared
//    memory once per CTA with one TMA bulk copy (cp.async.bulk, no
//    multicast).
//  * Each thread holds its 8 bytes plus the next thread's first 4 bytes in
//    a 96-bit shift register (three funnel shifts per step).  Bits at and
//    after the thread's last code end (known exactly from the next thread's
//    gap) are set to 1: a run of ones shorter than the longest code is never
//    a whole code of a canonical code, so a table lookup can never take a
//    code that belongs to the next thread.
//  * Pass 1 counts with a 14-bit count table (several codes per lookup);
//    pass 2 decodes with a 12-bit table holding up to three symbols per
//    entry.  Codes longer than the window fall back to canonical limits.
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
__device__ __forceinline__ uint2 ld_stream_u2(const void *p) {
    uint2 r;
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
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
__device__ __forceinline__ void group_barrier(uint32_t group) {
    asm volatile("bar.sync %0, %1;" ::"r"(group + 1u), "r"((uint32_t)kThreadsPerBlockFmt) : "memory");
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
__device__ __forceinline__ bool stage_tables(uint8_t *dst, const uint8_t *src, uint32_t bytes,
                                             uint64_t *mbar) {
    const uint32_t bar = smem_addr(mbar);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_addr(dst)),
            "l"(src), "r"(bytes), "r"(bar)
            : "memory");
    }
    return wait_tables(bar);
}

// Length of a code longer than the table window, from the canonical limits:
// the smallest l with window < lim[l].  0 if no code matches.
__device__ __forceinline__ uint32_t long_code_length(uint32_t x, const uint64_t *lim, uint32_t from,
                                                     uint32_t max_len) {
    for (uint32_t l = from; l <= max_len; ++l)
        if ((uint64_t)x < lim[l]) return l;
    return 0u;
}

struct BlockInputs {
    uint32_t w0, w1, w2;   // this thread's 8 bytes and the next 4 (big-endian words)
    uint32_t g_hi, g_lo;   // the two 32-bit gap words holding bits [5t, 5t + 10)
    uint32_t s, e;         // block_start[b], block_start[b + 1]
};

__device__ __forceinline__ void load_block_inputs(const DecodeArgs &a, uint64_t blk, uint32_t gt,
                                                  uint32_t lane, BlockInputs &in) {
    const uint64_t t = blk * (uint64_t)kThreadsPerBlockFmt + gt;
    const uint2 v = ld_stream_u2(a.enc + 8ull * t);
    in.w0 = v.x;
    in.w1 = v.y;
    // the next thread's first word: from the neighbour lane, or a load for lane 31
    in.w2 = (lane == 31u) ? __ldg(reinterpret_cast<const uint32_t *>(a.enc + 8ull * t + 8ull)) : 0u;
    const uint64_t bit = 5ull * t;
    const uint64_t word = bit >> 5;
    in.g_hi = __ldg(a.gaps32 + word);
    in.g_lo = __ldg(a.gaps32 + word + 1);
    in.s = __ldg(a.bstart + blk);
    in.e = __ldg(a.bstart + blk + 1);
}

__global__ void __launch_bounds__(kCtaThreads, 1) df11_decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *s_lut = smem;
    uint64_t *s_mbar = reinterpret_cast<uint64_t *>(smem + kLutBytes + kGroupsPerCta * kGroupBytes);

    const uint32_t tid = threadIdx.x;
    const uint32_t group = tid / kThreadsPerBlockFmt;
    const uint32_t gt = tid % kThreadsPerBlockFmt;  // thread within the format block
    const uint32_t lane = tid & 31u;
    const uint32_t warp = gt >> 5;                   // warp within the group
    uint8_t *sbuf = smem + kLutBytes + group * kGroupBytes;
    uint32_t *wtot = reinterpret_cast<uint32_t *>(sbuf + kSbufBytes);
    uint32_t my_err = 0;

    const uint64_t stride = (uint64_t)gridDim.x * kGroupsPerCta;
    uint64_t blk = (uint64_t)blockIdx.x * kGroupsPerCta + group;

    // Prefetch the first block's inputs while the tables stream in.
    BlockInputs cur{};
    if (blk < a.n_blocks) load_block_inputs(a, blk, gt, lane, cur);

    const bool staged = stage_tables(s_lut, a.lut, kLutBytes, s_mbar);
    if (__syncthreads_or(!staged)) {
        // Uniform over the CTA.  One more bounded wait so no copy is left in
        // flight into this CTA's shared memory, then report and stop.
        if (tid == 0) {
            wait_tables(smem_addr(s_mbar));
            if (a.err) atomicOr(a.err, kKernErrTimeout);
        }
        __syncthreads();
        return;
    }

    const LutHeader *hdr = reinterpret_cast<const LutHeader *>(s_lut + kOffHeader);
    const uint64_t *s_lim = reinterpret_cast<const uint64_t *>(s_lut + kOffLim);
    const uint32_t *s_offs = reinterpret_cast<const uint32_t *>(s_lut + kOffOffs);
    const uint8_t *s_symrot = s_lut + kOffSymRot;
    const uint8_t *s_clut = s_lut + kOffCountLut;
    const uint32_t *s_slut = reinterpret_cast<const uint32_t *>(s_lut + kOffSymLut);
    const uint32_t w1 = hdr->w1, w2 = hdr->w2, max_len = hdr->max_len;
    if (hdr->magic != kMagic || w1 < 1u || w1 > (uint32_t)kW1Max || w2 < 1u || w2 > (uint32_t)kW2Max ||
        max_len > 32u) {
        if (tid == 0 && a.err) atomicOr(a.err, DF11_KERR_BAD_CODE);
        return;  // uniform over the CTA: nothing was written yet
    }
    // Every non-zero table entry must take at least one bit and stay inside
    // its window, so each decode step makes progress: the per-thread loops
    // then end after at most 95 steps whatever the stream holds.
    {
        bool bad = false;
        for (uint32_t i = tid; i < (1u << w1); i += kCtaThreads) {
            const uint32_t ent = s_clut[i];
            bad |= ent != 0u && (count_entry_bits(ent) == 0u || count_entry_bits(ent) > w1 ||
                                 count_entry_codes(ent) == 0u);
        }
        for (uint32_t i = tid; i < (1u << w2); i += kCtaThreads) {
            const uint32_t ent = s_slut[i];
            bad |= ent != 0u && (sym_entry_bits(ent) == 0u || sym_entry_bits(ent) > w2 ||
                                 sym_entry_codes(ent) == 0u);
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
        if (nxt < a.n_blocks) load_block_inputs(a, nxt, gt, lane, cur);

        const uint64_t t = blk * (uint64_t)kThreadsPerBlockFmt + gt;
        const uint32_t s = in.s, e = in.e;
        const uint32_t base = s & ~15u;  // first 16-element chunk of the block's output
        const bool range_ok = (e >= s) && ((uint64_t)e <= a.n_elems) && (e - s <= (uint32_t)kMaxCodesPerBlock);
        const uint32_t n_chunks = range_ok ? (e - base + 15u) >> 4 : 0u;

        // First two sign/mantissa vectors this thread will merge.
        uint4 smv0 = make_uint4(0, 0, 0, 0), smv1 = make_uint4(0, 0, 0, 0);
        if (gt < n_chunks) smv0 = ld_stream_u4(a.sm + (uint64_t)base + 16ull * gt);
        if (gt + kThreadsPerBlockFmt < n_chunks)
            smv1 = ld_stream_u4(a.sm + (uint64_t)base + 16ull * (gt + kThreadsPerBlockFmt));

        // ---- this thread's bits: [gap, end) of its 96-bit window
        uint32_t w0 = bswap32(in.w0), w1v = bswap32(in.w1);
        uint32_t w2v = __shfl_down_sync(kFull, in.w0, 1);
        if (lane == 31u) w2v = in.w2;
        w2v = bswap32(w2v);
        // gaps are an MSB-first bit string: bits [5t, 5t + 10) hold this
        // thread's gap and the next thread's
        const uint32_t gb = __funnelshift_l(bswap32(in.g_lo), bswap32(in.g_hi), (uint32_t)((5ull * t) & 31u));
        uint32_t gap = gb >> 27;
        const uint32_t gap_next = (gb >> 22) & 31u;
        int32_t end;
        if (t >= a.n_threads) { gap = 0; end = 0; }
        else if (t + 1 == a.n_threads) end = (int32_t)(a.total_bits - 64ull * t);
        else end = 64 + (int32_t)gap_next;
        int32_t rem0 = end - (int32_t)gap;
        if (rem0 < 0) { my_err |= DF11_KERR_OVERRUN; rem0 = 0; }
        // set every bit at or after `end` to 1
        {
            const int32_t v0 = min(max(end, 0), 32), v1 = min(max(end - 32, 0), 32),
                          v2 = min(max(end - 64, 0), 32);
            w0 |= (v0 >= 32) ? 0u : (kFull >> v0);
            w1v |= (v1 >= 32) ? 0u : (kFull >> v1);
            w2v |= (v2 >= 32) ? 0u : (kFull >> v2);
        }
        // 96-bit window starting at the first code
        const uint32_t r_hi = __funnelshift_lc(w1v, w0, gap);
        const uint32_t r_lo = __funnelshift_lc(w2v, w1v, gap);
        const uint32_t r_fl = __funnelshift_lc(kFull, w2v, gap);

        // ---- pass 1: count the codes
        uint32_t cnt = 0;
        {
            uint32_t hi = r_hi, lo = r_lo, fl = r_fl;
            int32_t rem = rem0;
            while (rem > 0) {
                const uint32_t ent = s_clut[hi >> sh1];
                uint32_t nb = count_entry_bits(ent);
                uint32_t nc = count_entry_codes(ent);
                if (ent == 0u) {
                    nb = long_code_length(hi, s_lim, w1 + 1u, max_len);
                    nc = 1u;
                    if (nb == 0u) { my_err |= DF11_KERR_BAD_CODE; break; }
                }
                cnt += nc;
                rem -= (int32_t)nb;
                hi = __funnelshift_lc(lo, hi, nb);
                lo = __funnelshift_lc(fl, lo, nb);
                fl = __funnelshift_lc(kFull, fl, nb);
            }
            if (rem < 0) my_err |= DF11_KERR_OVERRUN;
        }

        // ---- block scan: warp inclusive scan, then across the 8 warps
        uint32_t incl = cnt;
#pragma unroll
        for (uint32_t d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, d);
            if (lane >= d) incl += v;
        }
        if (lane == 31u) wtot[warp] = incl;
        group_barrier(group);
        uint32_t wpre = 0, total = 0;
        {
            const uint4 ta = *reinterpret_cast<const uint4 *>(wtot);
            const uint4 tb = *reinterpret_cast<const uint4 *>(wtot + 4);
            const uint32_t tw[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
            for (uint32_t w = 0; w < 8; ++w) {
                wpre += (w < warp) ? tw[w] : 0u;
                total += tw[w];
            }
        }
        const bool ok = range_ok && (total == e - s);
        if (!ok && gt == 0) my_err |= range_ok ? DF11_KERR_COUNT_MISMATCH : DF11_KERR_BAD_BLOCK;

        // ---- pass 2: decode again, write rotated exponents to the buffer
        if (ok) {
            uint32_t hi = r_hi, lo = r_lo, fl = r_fl;
            int32_t rem = rem0;
            uint32_t p = (s - base) + wpre + incl - cnt;  // buffer index of this thread's first code
            while (rem > 0) {
                p = min(p, kSbufBytes - 3u);  // keeps a corrupt table inside this group's buffer
                const uint32_t ent = s_slut[hi >> sh2];
                uint32_t nb, nc;
                if (ent != 0u) {
                    nb = sym_entry_bits(ent);
                    nc = sym_entry_codes(ent);
                    sbuf[p] = (uint8_t)ent;
                    if (nc > 1u) sbuf[p + 1] = (uint8_t)(ent >> 8);
                    if (nc > 2u) sbuf[p + 2] = (uint8_t)(ent >> 16);
                } else {
                    nb = long_code_length(hi, s_lim, w2 + 1u, max_len);
                    if (nb == 0u) break;  // reported by pass 1
                    nc = 1u;
                    sbuf[p] = s_symrot[((hi >> (32u - nb)) + s_offs[nb]) & 255u];
                }
                p += nc;
                rem -= (int32_t)nb;
                hi = __funnelshift_lc(lo, hi, nb);
                lo = __funnelshift_lc(fl, lo, nb);
                fl = __funnelshift_lc(kFull, fl, nb);
            }
        }
        group_barrier(group);

        // ---- merge with sign/mantissa and store, 16 weights per step
        if (ok) {
            for (uint32_t c = gt; c < n_chunks; c += kThreadsPerBlockFmt) {
                uint4 smv;
                if (c == gt) smv = smv0;
                else if (c == gt + kThreadsPerBlockFmt) smv = smv1;
                else smv = ld_stream_u4(a.sm + (uint64_t)base + 16ull * c);
                const uint4 ex = *reinterpret_cast<const uint4 *>(sbuf + 16u * c);
                const uint32_t S[4] = {smv.x, smv.y, smv.z, smv.w};
                const uint32_t R[4] = {ex.x, ex.y, ex.z, ex.w};
                uint32_t o[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t hi8 = (S[q] & 0x80808080u) | (R[q] & 0x7F7F7F7Fu);
                    const uint32_t lo8 = (R[q] & 0x80808080u) | (S[q] & 0x7F7F7F7Fu);
                    o[2 * q] = __byte_perm(lo8, hi8, 0x5140u);
                    o[2 * q + 1] = __byte_perm(lo8, hi8, 0x7362u);
                }
                const uint32_t g0 = base + 16u * c;
                uint16_t *dst = a.out + g0;
                if (g0 >= s && g0 + 16u <= e) {
                    st_u4(dst, o[0], o[1], o[2], o[3]);
                    st_u4(dst + 8, o[4], o[5], o[6], o[7]);
                } else {
#pragma unroll
                    for (uint32_t j = 0; j < 16; ++j) {
                        const uint32_t g = g0 + j;
                        if (g >= s && g < e) dst[j] = (uint16_t)(o[j >> 1] >> (16u * (j & 1u)));
                    }
                }
            }
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
    if (!t || !out) return DF11_ERR_INVALID_ARG;
    df11_status st = df11_validate(t);
    if (st != DF11_OK) return st;
    if (t->n_elems == 0) return DF11_OK;
    if (!t->enc || !t->sm || !t->gaps || !t->block_start || !t->lut) return DF11_ERR_INVALID_ARG;
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
