// df11_gemm.cu -- the consumer of the decoded weights: Y = X * W^T in BF16
// with FP32 accumulation on the 5th-generation tensor cores (tcgen05),
// reading W straight from the decode scratch buffer.
//
// Sources: "DFloat11 : compression sans perte pour l'inference GPU qui reduit
// les LLM a 70 % de leur taille" (fr.news.hada.io), << Decompression adaptee
// a l'inference GPU >>: the weight matrix is decompressed to BF16 right
// before its matrix multiplication and discarded after it.
//
// Shapes: X [T, in] (activations, row-major), W [out, in] (nn.Linear weight,
// row-major), Y [T, out] FP32.  T is small (1..256 tokens), so the product
// is computed transposed (Y^T = W X^T): the UMMA M dimension is 128 rows of
// W, N is T rounded up to 16, K advances 16 per instruction.
//
// One CTA computes a 128-row tile of W over a range of K (split-K when there
// are too few row tiles to fill the SMs; partial tiles are added into Y,
// which the launcher zeroes first).  A stage holds one or two 64-wide K
// sub-tiles: two when T <= 128, so that each W row is read 256 contiguous
// bytes at a time (better DRAM locality for the weight stream), one when
// the X tiles are large (a deeper ring).  128 threads: one thread issues TMA
// loads (W and X tiles, 128-byte swizzle, no multicast) into a ring of
// shared-memory stages, one thread issues tcgen05.mma into an FP32
// accumulator in tensor memory and releases each stage with tcgen05.commit,
// and all four warps read the accumulator back (tcgen05.ld) and write Y.
// Every wait is bounded; a timed-out wait sets an error bit and the CTA
// still frees its tensor memory before leaving.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "df11.h"
#include "df11_tc.cuh"

namespace {

constexpr uint32_t kBlockM = 128;      // rows of W per tile (UMMA M)
constexpr uint32_t kBlockK = 64;       // K per sub-tile: 64 BF16 = one 128-byte swizzle row
constexpr uint32_t kUmmaK = 16;        // K per tcgen05.mma (kind::f16)
constexpr uint32_t kThreads = 128;
constexpr uint32_t kMaxStages = 8;
constexpr uint32_t kSmemBudget = 200u * 1024u;
constexpr uint32_t kGemmErrTimeout = 0x20u;

struct GemmArgs {
    float *y;
    uint32_t *err;
    uint32_t T, out, in;
    uint32_t n_pad;      // UMMA N: T rounded up to 16
    uint32_t sub;        // 64-wide K sub-tiles per stage (1 or 2)
    uint32_t k_tiles;    // K stages: in / (64 sub)
    uint32_t splits;     // CTAs per row tile along K
    uint32_t stages;
    uint32_t tmem_cols;  // power of two >= 32 and >= n_pad
    uint32_t atomic_out; // 1: add into Y (split-K), 0: store
};

using namespace df11::tc;

__global__ void __launch_bounds__(kThreads, 1)
    df11_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                     const GemmArgs g) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t a_sub = kBlockM * kBlockK * 2u, b_sub = g.n_pad * kBlockK * 2u;
    const uint32_t a_bytes = g.sub * a_sub;
    const uint32_t b_bytes = g.sub * b_sub;
    const uint32_t stage_bytes = (a_bytes + b_bytes + 1023u) & ~1023u;
    // smem: [stages x (A | B)] [full[S]] [empty[S]] [acc_full] [tmem address]
    const uint32_t base = (smem_u32(smem) + 1023u) & ~1023u;
    const uint32_t bars = base + g.stages * stage_bytes;
    const uint32_t full0 = bars, empty0 = bars + 8u * kMaxStages, acc_full = bars + 16u * kMaxStages;
    const uint32_t tmem_slot = acc_full + 8u;
    uint8_t *tmem_slot_ptr = smem + (tmem_slot - smem_u32(smem));

    const uint32_t m_tile = blockIdx.x / g.splits, split = blockIdx.x % g.splits;
    const uint32_t kt_per = (g.k_tiles + g.splits - 1u) / g.splits;
    const uint32_t kt0 = split * kt_per;
    const uint32_t kt1 = min(g.k_tiles, kt0 + kt_per);
    uint32_t err = 0;

    if (tid == 0) {
        for (uint32_t s = 0; s < g.stages; ++s) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8u * s) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(empty0 + 8u * s) : "memory");
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(acc_full) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {  // one full warp allocates the accumulator columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(g.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem_d = *reinterpret_cast<volatile uint32_t *>(tmem_slot_ptr);
    const uint32_t n_kt = kt1 > kt0 ? kt1 - kt0 : 0u;

    if (warp == 0 && lane == 0) {
        // ---- producer: TMA loads of W (128 x 64) and X (n_pad x 64) tiles
        for (uint32_t i = 0; i < n_kt; ++i) {
            const uint32_t s = i % g.stages, use = i / g.stages;
            if (!mbar_wait(empty0 + 8u * s, (use & 1u) ^ 1u)) { err |= kGemmErrTimeout; break; }
            const uint32_t sa = base + s * stage_bytes, sbb = sa + a_bytes;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full0 + 8u * s),
                         "r"(a_bytes + b_bytes)
                         : "memory");
            for (uint32_t j = 0; j < g.sub; ++j) {
                const int32_t k = (int32_t)(((kt0 + i) * g.sub + j) * kBlockK);
                tma_load_2d(sa + j * a_sub, &map_w, full0 + 8u * s, k, (int32_t)(m_tile * kBlockM));
                tma_load_2d(sbb + j * b_sub, &map_x, full0 + 8u * s, k, 0);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: 4 UMMAs of K = 16 per stage, then release the stage
        const uint32_t idesc = instr_desc_bf16(g.n_pad, kBlockM);
        for (uint32_t i = 0; i < n_kt; ++i) {
            const uint32_t s = i % g.stages, use = i / g.stages;
            if (!mbar_wait(full0 + 8u * s, use & 1u)) { err |= kGemmErrTimeout; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sa = base + s * stage_bytes, sbb = sa + a_bytes;
            for (uint32_t j = 0; j < g.sub; ++j) {
#pragma unroll
                for (uint32_t kk = 0; kk < kBlockK / kUmmaK; ++kk) {
                    // advancing K by 16 BF16 = 32 bytes inside the swizzled row
                    umma_bf16(tmem_d, smem_desc_sw128(sa + j * a_sub + kk * 32u),
                              smem_desc_sw128(sbb + j * b_sub + kk * 32u), idesc, (i | j | kk) != 0u ? 1u : 0u);
                }
            }
            umma_commit(empty0 + 8u * s);
        }
        umma_commit(acc_full);  // fires once every issued MMA has completed
    }
    __syncwarp();

    // ---- epilogue: warp w owns accumulator lanes 32w..32w+31 (rows of W)
    const bool have = n_kt > 0 && mbar_wait(acc_full, 0u);
    if (n_kt > 0 && !have) err |= kGemmErrTimeout;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t row = m_tile * kBlockM + warp * 32u + lane;
    for (uint32_t c0 = 0; c0 < g.n_pad; c0 += 16u) {
        uint32_t v[16];
        tmem_ld16(tmem_d + ((warp * 32u) << 16) + c0, v);
        if (have) {
#pragma unroll
            for (uint32_t j = 0; j < 16; ++j) {
                const uint32_t t = c0 + j;
                if (t < g.T) {
                    float *dst = g.y + (uint64_t)t * g.out + row;
                    if (g.atomic_out) atomicAdd(dst, __uint_as_float(v[j]));
                    else *dst = __uint_as_float(v[j]);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 2) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(g.tmem_cols)
                     : "memory");
    }
    if (err && g.err) atomicOr(g.err, err);
}

// ---------------------------------------------------------------- grouped
// Several products Y_j = X_j W_j^T in one persistent launch (e.g. the seven
// matrices of a decoded transformer block).  The 128 x 64 k-tiles of all the
// matrices, numbered matrix by matrix, row tile by row tile and along K,
// are split evenly over the CTAs: no launch leaves a tail and every SM
// streams the same number of weight bytes.  Warp 0 loads the W and X tiles
// of each k-tile by TMA (128-byte swizzle, no multicast) into a ring of
// stages; warp 1 issues four tcgen05.mma (K = 16 each) per k-tile into one
// of two FP32 accumulators in tensor memory, which alternate between
// segments (a segment = the k-tiles of one row tile in this CTA); warps 2..5
// read each finished segment (tcgen05.ld, TMEM lanes of their rank in the
// warpgroup) and add it into Y with FP32 atomics (a row tile split between
// two CTAs gets two partial sums; the launcher zeroes Y).  Every wait is
// bounded and suspends on the mbarrier instead of spinning.
constexpr uint32_t kMultiMax = 16;
constexpr uint32_t kMultiThreads = 192;
constexpr uint32_t kMultiStagesMax = 16;
constexpr uint32_t kTileW = kBlockM * kBlockK * 2u;  // one W k-tile: 16 KB

struct MultiMat {
    float *y;
    uint32_t rows;   // out
    uint32_t kt;     // k-tiles per row tile: in / 64
    uint32_t rt;     // row tiles: out / 128
    uint32_t tbase;  // first k-tile of this matrix in the numbering
};
struct MultiArgs {
    MultiMat m[kMultiMax];
    uint32_t *err;
    uint32_t n_mats, T, n_pad, n_tiles, stages, xbytes, tmem_cols;
    uint32_t sub;  // k-tiles per stage (1 or 2; every matrix's k-tiles per row tile are a multiple)
};
struct MultiMaps {
    CUtensorMap w[kMultiMax];  // W_j [out, in], box [128, 64]
    CUtensorMap x[kMultiMax];  // X_j [T, in], box [n_pad, 64]
};

// k-tile cursor: matrix j, row tile r, k-tile column k
struct MultiCursor {
    uint32_t j, r, k;
    __device__ __forceinline__ void start(const MultiArgs &g, uint32_t K) {
        j = 0;
        while (j + 1u < g.n_mats && K >= g.m[j + 1u].tbase) ++j;
        const uint32_t l = K - g.m[j].tbase;
        r = l / g.m[j].kt;
        k = l % g.m[j].kt;
    }
    __device__ __forceinline__ void next(const MultiArgs &g) {
        if (++k < g.m[j].kt) return;
        k = 0;
        if (++r < g.m[j].rt) return;
        r = 0;
        ++j;
    }
};

// Bounded wait (about two seconds at most) that gives up once the CTA's
// abort flag is set.  hint_ns > 0: each probe suspends up to hint_ns while
// the phase is incomplete (for waiters off the critical path); 0: plain
// probes (the producer and the MMA issuer, whose wake-up latency sets the
// pipeline's pace).
__device__ __forceinline__ bool multi_wait(uint32_t bar, uint32_t parity, uint32_t abort_flag, uint32_t &err,
                                           uint32_t hint_ns) {
    const uint32_t rounds = 2000000000u / (hint_ns + 100u);
    for (uint32_t i = 0; i < rounds; ++i) {
        if (hint_ns ? mbar_try_wait_hint(bar, parity, hint_ns) : mbar_wait(bar, parity, 1u)) return true;
        uint32_t a;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a) : "r"(abort_flag) : "memory");
        if (a) return false;
    }
    err |= kGemmErrTimeout;
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_flag), "r"(1u) : "memory");
    return false;
}

// Zeroes every product's Y [T, out] (one launch for all of them; 16-byte
// stores where the buffer allows, else 4-byte ones).
__global__ void zero_y_kernel(const __grid_constant__ MultiArgs g) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint32_t j = 0; j < g.n_mats; ++j) {
        float *y = g.m[j].y;
        const uint64_t n = (uint64_t)g.T * g.m[j].rows;
        const uint64_t i0 = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
        if (((uintptr_t)y & 15u) == 0u) {
            for (uint64_t i = i0; i < n / 4u; i += stride) reinterpret_cast<float4 *>(y)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint64_t i = (n / 4u) * 4u + i0; i < n; i += stride) y[i] = 0.f;
        } else {
            for (uint64_t i = i0; i < n; i += stride) y[i] = 0.f;
        }
    }
}

__global__ void __launch_bounds__(kMultiThreads, 1)
    df11_gemm_multi_kernel(const __grid_constant__ MultiArgs g, const __grid_constant__ MultiMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t stage_bytes = g.sub * (kTileW + g.xbytes);  // multiples of 1024 (n_pad is a multiple of 16)
    const uint32_t base = (smem_u32(smem) + 1023u) & ~1023u;
    const uint32_t full0 = base + g.stages * stage_bytes, empty0 = full0 + 8u * kMultiStagesMax;
    const uint32_t accfull0 = empty0 + 8u * kMultiStagesMax, accempty0 = accfull0 + 16u;
    const uint32_t final_bar = accempty0 + 16u, tmem_slot = final_bar + 8u, abort_flag = tmem_slot + 4u;
    // whole stages per CTA (n_tiles is a multiple of sub)
    const uint32_t n_st = g.n_tiles / g.sub;
    const uint32_t K0 = g.sub * (uint32_t)((uint64_t)n_st * blockIdx.x / gridDim.x);
    const uint32_t NT = g.sub * (uint32_t)((uint64_t)n_st * (blockIdx.x + 1u) / gridDim.x) - K0;
    uint32_t err = 0;

    if (tid == 0) {
        for (uint32_t s = 0; s < g.stages; ++s) {
            mbar_init(full0 + 8u * s, 1);
            mbar_init(empty0 + 8u * s, 1);
        }
        for (uint32_t a = 0; a < 2u; ++a) {
            mbar_init(accfull0 + 8u * a, 1);
            mbar_init(accempty0 + 8u * a, 4);  // one arrival per epilogue warp
        }
        mbar_init(final_bar, 1);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_flag), "r"(0u) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(g.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");

    if (warp == 0) {
        if (lane == 0) {  // ---- producer
            MultiCursor c;
            c.start(g, K0);
            uint32_t s = 0, use = 0;
            for (uint32_t i = 0; i < NT; i += g.sub) {
                if (use > 0u && !multi_wait(empty0 + 8u * s, (use - 1u) & 1u, abort_flag, err, 0u)) break;
                const uint32_t a = base + s * stage_bytes;
                mbar_arrive_expect_tx(full0 + 8u * s, stage_bytes);
                for (uint32_t u = 0; u < g.sub; ++u) {
                    tma_load_2d(a + u * kTileW, &maps.w[c.j], full0 + 8u * s, (int32_t)(c.k * kBlockK),
                                (int32_t)(c.r * kBlockM));
                    tma_load_2d(a + g.sub * kTileW + u * g.xbytes, &maps.x[c.j], full0 + 8u * s,
                                (int32_t)(c.k * kBlockK), 0);
                    c.next(g);
                }
                if (++s == g.stages) {
                    s = 0;
                    ++use;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {  // ---- MMA issuer
            const uint32_t idesc = instr_desc_bf16(g.n_pad, kBlockM);
            const uint64_t d0 = smem_desc_sw128(base);
            MultiCursor c;
            c.start(g, K0);
            uint32_t s = 0, use = 0, seg = 0;
            bool stop = false;
            for (uint32_t i = 0; i < NT && !stop; i += g.sub) {
                if (!multi_wait(full0 + 8u * s, use & 1u, abort_flag, err, 0u)) break;
                const uint64_t da0 = d0 + ((s * stage_bytes) >> 4), db0 = da0 + ((g.sub * kTileW) >> 4);
                for (uint32_t u = 0; u < g.sub; ++u) {  // (segments start and end on stage boundaries)
                    const bool first = i + u == 0u || c.k == 0u;
                    const bool last = i + u + 1u == NT || c.k + 1u == g.m[c.j].kt;
                    const uint32_t abuf = seg & 1u;
                    if (first && seg >= 2u &&
                        !multi_wait(accempty0 + 8u * abuf, ((seg >> 1) - 1u) & 1u, abort_flag, err, 0u)) {
                        stop = true;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint64_t da = da0 + ((u * kTileW) >> 4), db = db0 + ((u * g.xbytes) >> 4);
#pragma unroll
                    for (uint32_t kk = 0; kk < kBlockK / kUmmaK; ++kk)  // K = 16: 32 bytes along the swizzled row
                        umma_bf16(tmem + abuf * g.n_pad, da + 2u * kk, db + 2u * kk, idesc,
                                  (first && kk == 0u) ? 0u : 1u);
                    if (last) {
                        umma_commit(accfull0 + 8u * abuf);
                        ++seg;
                    }
                    c.next(g);
                }
                umma_commit(empty0 + 8u * s);
                if (++s == g.stages) {
                    s = 0;
                    ++use;
                }
            }
            // every issued MMA has completed before the accumulators are freed
            umma_commit(final_bar);
            if (!mbar_wait(final_bar, 0u)) err |= kGemmErrTimeout;
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp rank q in its warpgroup reads TMEM lanes 32q..32q+31
        const uint32_t q = warp & 3u;
        MultiCursor c;
        c.start(g, K0);
        uint32_t seg = 0;
        for (uint32_t i = 0; i < NT;) {
            const uint32_t n = min(g.m[c.j].kt - c.k, NT - i);  // the segment's k-tiles
            const uint32_t j = c.j, rtile = c.r;
            i += n;
            c.k += n - 1u;
            c.next(g);
            const uint32_t abuf = seg & 1u;
            const bool have = multi_wait(accfull0 + 8u * abuf, (seg >> 1) & 1u, abort_flag, err, 2000u);
            __syncwarp();
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const MultiMat &M = g.m[j];
            const uint32_t row = rtile * kBlockM + q * 32u + lane;
            for (uint32_t c0 = 0; c0 < g.n_pad; c0 += 16u) {
                uint32_t v[16];
                tmem_ld16(tmem + ((q * 32u) << 16) + abuf * g.n_pad + c0, v);
                if (have) {
#pragma unroll
                    for (uint32_t t = 0; t < 16u; ++t)
                        if (c0 + t < g.T) atomicAdd(M.y + (uint64_t)(c0 + t) * M.rows + row, __uint_as_float(v[t]));
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0u) mbar_arrive(accempty0 + 8u * abuf);
            ++seg;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 2) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(g.tmem_cols)
                     : "memory");
    }
    if (err && g.err) atomicOr(g.err, err);
}

// ---------------------------------------------------------------- T <= 4
// With T <= 4 tokens every weight feeds at most 8 flops: the product is a
// matrix-vector stream bound by reading W, and the tensor-core tiling (128
// rows x 64 columns per load) reads W with poor DRAM locality.  This kernel
// streams W along contiguous rows instead: a CTA of 8 warps takes R = 1 or
// 2 rows, S = 8 / R warps share a row's K range, each lane loads 16 bytes (8 weights)
// per step with several loads in flight, multiplies them by X (read through
// the cache: X is small and shared by every CTA) in FP32, and the partial sums
// are reduced by warp shuffles and then across the row's warps in shared
// memory.  One writer per output: no atomics, no zeroing, deterministic.
constexpr uint32_t kGemvThreads = 256;

__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// lo += a.lo * b.lo and hi += a.hi * b.hi for two BF16 pairs, with FP32
// accumulators (mixed-precision FMA: the product is exact, one rounding).
__device__ __forceinline__ void fma2_bf16(float &lo, float &hi, uint32_t a, uint32_t b) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %2;\n\t"
        "mov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %1, ah, bh, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(a), "r"(b));
}

// 8 BF16 products (two per 32-bit word) added into (lo, hi): with the
// mixed-precision FMA (kMixed), else by widening each BF16 to FP32 with a
// shift or a mask before an FP32 FMA.  Over a block's seven matrices the
// mixed form was faster at T = 3 and 4 (118 vs 139, 145 vs 167 us) and
// slower at T = 1 and 2, so the kernel takes it for T >= 3.
template <bool kMixed>
__device__ __forceinline__ void dot8(const uint4 a, const uint4 b, float &lo, float &hi) {
    const uint32_t A[4] = {a.x, a.y, a.z, a.w}, B[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (kMixed) {
            fma2_bf16(lo, hi, A[i], B[i]);
        } else {
            lo = fmaf(__uint_as_float(A[i] << 16), __uint_as_float(B[i] << 16), lo);
            hi = fmaf(__uint_as_float(A[i] & 0xFFFF0000u), __uint_as_float(B[i] & 0xFFFF0000u), hi);
        }
    }
}

template <int T, int R>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const uint16_t *x, const uint16_t *w, float *y,
                                                            uint32_t out, uint32_t in) {
    constexpr uint32_t S = 8 / R;  // warps per row
    __shared__ float part[8][T];
    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
    const uint32_t row = blockIdx.x * R + (warp % R);
    const uint32_t split = warp / R;
    const uint32_t n8 = in / (8u * S);  // 16-byte chunks in this warp's K range
    const uint32_t k0 = split * n8;     // first chunk
    const uint4 *wr = reinterpret_cast<const uint4 *>(w + (uint64_t)row * in) + k0;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x) + k0;
    const uint32_t xstride = in / 8u;   // chunks per token row of X
    float lo[T], hi[T];
#pragma unroll
    for (int t = 0; t < T; ++t) lo[t] = hi[t] = 0.f;
    uint32_t c = lane;
    for (; c + 96u < n8; c += 128u) {  // four loads of W in flight per lane
        const uint4 w0 = ld_stream_u4(wr + c), w1 = ld_stream_u4(wr + c + 32u);
        const uint4 w2 = ld_stream_u4(wr + c + 64u), w3 = ld_stream_u4(wr + c + 96u);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const uint4 *xt = xr + (uint64_t)t * xstride + c;
            dot8<(T >= 3)>(w0, __ldg(xt), lo[t], hi[t]);
            dot8<(T >= 3)>(w1, __ldg(xt + 32u), lo[t], hi[t]);
            dot8<(T >= 3)>(w2, __ldg(xt + 64u), lo[t], hi[t]);
            dot8<(T >= 3)>(w3, __ldg(xt + 96u), lo[t], hi[t]);
        }
    }
    for (; c < n8; c += 32u) {
        const uint4 w0 = ld_stream_u4(wr + c);
#pragma unroll
        for (int t = 0; t < T; ++t) dot8<(T >= 3)>(w0, __ldg(xr + (uint64_t)t * xstride + c), lo[t], hi[t]);
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
        float v = lo[t] + hi[t];
#pragma unroll
        for (uint32_t d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, d);
        if (lane == 0) part[warp][t] = v;
    }
    __syncthreads();
    if (threadIdx.x < (uint32_t)(R * T)) {
        const uint32_t r = threadIdx.x % R, t = threadIdx.x / R;
        float v = 0.f;
#pragma unroll
        for (uint32_t sp = 0; sp < S; ++sp) v += part[sp * R + r][t];
        y[(uint64_t)t * out + blockIdx.x * R + r] = v;
    }
}

template <int T>
void launch_gemv(const uint16_t *x, const uint16_t *w, float *y, uint32_t out, uint32_t in, int sms,
                 cudaStream_t s) {
    // rows per CTA: one when there are few rows (about 6 CTAs per SM), else
    // two, so that at least four warps share a row's K range (measured:
    // 4 or 8 rows per CTA, i.e. fewer warps per row, stream W more slowly)
    const uint32_t r = out >= 12u * (uint32_t)sms ? 2u : 1u;
    const unsigned grid = out / r;
    if (r == 2u) gemv_kernel<T, 2><<<grid, kGemvThreads, 0, s>>>(x, w, y, out, in);
    else gemv_kernel<T, 1><<<grid, kGemvThreads, 0, s>>>(x, w, y, out, in);
}

// ---------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
std::atomic<int> g_gemm_attr[64];

bool get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return df11::tc::make_bf16_tile_map(m, ptr, rows, cols, box_rows);
}

}  // namespace

// 2-D BF16 tensor map over a row-major [rows, cols] matrix, box [box_rows, 64]
// with the 128-byte swizzle; rows past the end read as zero.
bool df11::tc::make_bf16_tile_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    if (!get_encoder()) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2u};
    const cuuint32_t box[2] = {kBlockK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

extern "C" df11_status df11_gemm_bf16(const uint16_t *x, const uint16_t *w, float *y, uint32_t T, uint32_t out,
                                      uint32_t in, uint32_t *err_word, void *stream) {
    if (!x || !w || !y) return DF11_ERR_INVALID_ARG;
    if (T == 0 || T > 256 || out == 0 || out % kBlockM != 0 || in == 0 || in % kBlockK != 0)
        return DF11_ERR_UNSUPPORTED;
    if (((uintptr_t)x & 15u) || ((uintptr_t)w & 15u) || ((uintptr_t)y & 3u)) return DF11_ERR_INVALID_ARG;
    if (!get_encoder()) return DF11_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DF11_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DF11_ERR_CUDA;

    if (T <= 4u) {  // matrix-vector stream on the CUDA cores
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (T == 1u) launch_gemv<1>(x, w, y, out, in, sms, s);
        else if (T == 2u) launch_gemv<2>(x, w, y, out, in, sms, s);
        else if (T == 3u) launch_gemv<3>(x, w, y, out, in, sms, s);
        else launch_gemv<4>(x, w, y, out, in, sms, s);
        if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
        return DF11_OK;
    }

    GemmArgs g;
    g.y = y;
    g.err = err_word;
    g.T = T;
    g.out = out;
    g.in = in;
    g.n_pad = (T + 15u) & ~15u;
    g.sub = (g.n_pad <= 128u && in % (2u * kBlockK) == 0u) ? 2u : 1u;
    g.k_tiles = in / (g.sub * kBlockK);
    g.tmem_cols = 32;
    while (g.tmem_cols < g.n_pad) g.tmem_cols <<= 1;
    const uint32_t m_tiles = out / kBlockM;
    uint32_t splits = (uint32_t)sms / m_tiles;
    if (splits < 1) splits = 1;
    if (splits > g.k_tiles) splits = g.k_tiles;
    // no empty split: every CTA gets at least one K tile
    const uint32_t kt_per = (g.k_tiles + splits - 1) / splits;
    splits = (g.k_tiles + kt_per - 1) / kt_per;
    g.splits = splits;
    g.atomic_out = splits > 1 ? 1u : 0u;
    const uint32_t stage_bytes = (g.sub * (kBlockM + g.n_pad) * kBlockK * 2u + 1023u) & ~1023u;
    g.stages = kSmemBudget / stage_bytes;
    if (g.stages > kMaxStages) g.stages = kMaxStages;
    if (g.stages < 2) return DF11_ERR_UNSUPPORTED;
    const uint32_t smem = 1024u + g.stages * stage_bytes + 8u * (2u * kMaxStages + 2u);

    CUtensorMap mw, mx;
    if (!make_map(&mw, w, out, in, kBlockM) || !make_map(&mx, x, T, in, g.n_pad)) return DF11_ERR_CUDA;
    if (!g_gemm_attr[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(df11_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(1024u + kSmemBudget + 8u * (2u * kMaxStages + 2u))) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_gemm_attr[dev].store(1, std::memory_order_release);
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (g.atomic_out && cudaMemsetAsync(y, 0, (size_t)T * out * sizeof(float), s) != cudaSuccess)
        return DF11_ERR_CUDA;
    df11_gemm_kernel<<<m_tiles * splits, kThreads, smem, s>>>(mw, mx, g);
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}

extern "C" df11_status df11_gemm_bf16_multi(const df11_gemm_mat *mats, uint32_t n_mats, uint32_t T,
                                            uint32_t *err_word, void *stream) {
    if (n_mats == 0) return DF11_OK;
    if (!mats) return DF11_ERR_INVALID_ARG;
    if (n_mats > kMultiMax || T == 0 || T > 256) return DF11_ERR_UNSUPPORTED;
    for (uint32_t j = 0; j < n_mats; ++j) {
        const df11_gemm_mat &m = mats[j];
        if (!m.x || !m.w || !m.y) return DF11_ERR_INVALID_ARG;
        if (m.out == 0 || m.out % kBlockM != 0 || m.in == 0 || m.in % kBlockK != 0) return DF11_ERR_UNSUPPORTED;
        if (((uintptr_t)m.x & 15u) || ((uintptr_t)m.w & 15u) || ((uintptr_t)m.y & 3u)) return DF11_ERR_INVALID_ARG;
    }
    if (T <= 4u) {  // matrix-vector streams (one launch per matrix)
        for (uint32_t j = 0; j < n_mats; ++j) {
            const df11_status st = df11_gemm_bf16(mats[j].x, mats[j].w, mats[j].y, T, mats[j].out, mats[j].in,
                                                  err_word, stream);
            if (st != DF11_OK) return st;
        }
        return DF11_OK;
    }
    if (!get_encoder()) return DF11_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DF11_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DF11_ERR_CUDA;
    MultiArgs g;
    MultiMaps maps;
    g.err = err_word;
    g.n_mats = n_mats;
    g.T = T;
    g.n_pad = (T + 15u) & ~15u;
    g.xbytes = g.n_pad * kBlockK * 2u;
    g.tmem_cols = 32u;
    while (g.tmem_cols < 2u * g.n_pad) g.tmem_cols <<= 1;
    // two k-tiles per stage (each W row read 256 contiguous bytes at a time)
    // when the X tiles are small and every row tile has an even k-tile count
    g.sub = g.n_pad <= 128u ? 2u : 1u;
    for (uint32_t j = 0; j < n_mats; ++j)
        if ((mats[j].in / kBlockK) % 2u) g.sub = 1u;
    uint64_t tiles = 0;
    for (uint32_t j = 0; j < n_mats; ++j) {
        const df11_gemm_mat &m = mats[j];
        g.m[j] = MultiMat{m.y, m.out, m.in / kBlockK, m.out / kBlockM, (uint32_t)tiles};
        tiles += (uint64_t)(m.out / kBlockM) * (m.in / kBlockK);
        if (!make_map(&maps.w[j], m.w, m.out, m.in, kBlockM) || !make_map(&maps.x[j], m.x, T, m.in, g.n_pad))
            return DF11_ERR_CUDA;
    }
    if (tiles >= (1ull << 32)) return DF11_ERR_UNSUPPORTED;
    for (uint32_t j = n_mats; j < kMultiMax; ++j) {
        g.m[j] = MultiMat{nullptr, 0u, 1u, 1u, (uint32_t)tiles};
        maps.w[j] = maps.w[0];
        maps.x[j] = maps.x[0];
    }
    g.n_tiles = (uint32_t)tiles;
    // the deepest ring that fits: stages of one W k-tile and one X k-tile
    constexpr uint32_t kMultiSmem = 227u * 1024u;
    constexpr uint32_t kTail = 1024u + 8u * (2u * kMultiStagesMax + 5u) + 16u;  // alignment, barriers, flags
    const uint32_t stage_bytes = g.sub * (kTileW + g.xbytes);
    g.stages = (kMultiSmem - kTail) / stage_bytes;
    if (g.stages > kMultiStagesMax) g.stages = kMultiStagesMax;
    if (g.stages < 2u) return DF11_ERR_UNSUPPORTED;
    const uint32_t smem = kTail + g.stages * stage_bytes;
    static std::atomic<int> attr_set[64];
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(df11_gemm_multi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kMultiSmem) != cudaSuccess)
            return DF11_ERR_CUDA;
        attr_set[dev].store(1, std::memory_order_release);
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    zero_y_kernel<<<2u * (unsigned)sms, 256, 0, s>>>(g);  // partial sums are added into Y
    const uint32_t n_st = g.n_tiles / g.sub;  // every CTA gets at least one stage
    const unsigned grid = (unsigned)(n_st < (uint32_t)sms ? n_st : (uint32_t)sms);
    df11_gemm_multi_kernel<<<grid, kMultiThreads, smem, s>>>(g, maps);
    if (cudaGetLastError() != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
}
