// IF4 x IF4 linear for B200 (sm_100a): decode both IF4 operands to fp16 with
// the tensor scales factored out, then one dense tcgen05 GEMM with fp32
// accumulation in tensor memory and the two tensor scales applied in the
// epilogue.
//
// The pages' IF4 MAC routes every operand pair by its group's sign bit into
// an FP4 or a 6/7-scaled INT4 decoder before multiplying (episode companion
// "Adaptive Block-Scaled Data Types for FP4 Training", section "MAC Unit:
// Decoding Two Formats from One Sign Bit").  B200 tensor cores have no IF4
// type, so both decoders run once per operand element ahead of the GEMM: the
// decoded value q * E4M3(scale) is exact in fp16 for FP4 groups and rounded
// to 11 bits for INT4 groups, and the per-tensor scales (one float each)
// factor out of the whole sum.
//
// GEMM structure (one CTA per SM, persistent over 128 x 256 output tiles;
// large problems use the CTA-pair kernel further down, 256 x 256 tiles):
//   warp 0      TMA producer: 128B-swizzled 64-wide K slabs of A and B into a
//               4-stage shared-memory ring (no multicast)
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators)
//               and one thread issues tcgen05.mma (M=128, N=256, K=16)
//   warps 2-5   epilogue: tcgen05.ld of the finished accumulator, scale,
//               bf16 RNE, global stores; the next tile's MMAs run meanwhile.
//               With the IF4 output (QOUT) they also encode each row's
//               16-column groups with the quantizer's group encoder.
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the kernel
// sets IF4_DEV_TIMEOUT in the error word, stops issuing work, drains what is
// in flight (bounded), frees its tensor memory and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/if4.h"
#include "if4_decode.cuh"
#include "if4_encode.cuh"
#include "if4_internal.h"

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                       // fp16: one 128-byte swizzle row
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;            // two accumulators
constexpr int NUM_THREADS = 192;             // 6 warps
constexpr int EPI_WARP0 = 2;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
                           512 /*inverse block scales of the IF4 output*/;
constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;   // 1 s per wait
// mbarrier.try_wait suspends the thread until the phase completes or this
// many ns pass, instead of returning at once; a waiting warp then takes no
// issue slots from the warps beside it on its scheduler.
constexpr int WAIT_HINT_NS = 20000;

// instruction descriptor, kind::f16: D f32, A f16, B f16, both K-major,
// N = 256, M = 128
constexpr uint32_t IDESC = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

// ------------------------------------------------------------ PTX glue ----

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "n"(WAIT_HINT_NS) : "memory");
    return ok != 0;
}

// Same, with cluster-scope acquire: for barriers that threads of the peer CTA
// arrive on with release.cluster.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "n"(WAIT_HINT_NS) : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `parity` to complete.  Returns false (and
// raises the CTA's abort flag) when the wall-clock limit runs out or another
// role already aborted.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    auto try_once = [&] {
        return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    };
    if (try_once()) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (try_once()) return true;
        if ((i & 255u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > WAIT_LIMIT_NS) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core-matrix groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);          // start address
    d |= (uint64_t)1u << 16;                          // leading byte offset (unused)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                          // SWIZZLE_128B
    return d;
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"
                 " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}


// ------------------------------------------------- IF4 output epilogue ----
//
// With the IF4 output, each epilogue thread holds one row of a 32-column
// chunk of C, i.e. two whole groups of 16 along N, the contiguous dimension.
// It rounds them to bf16 (the values a separate if4_quantize of the bf16 C
// would read) and encodes them with the quantizer's own group encoder under
// the given tensor scale, so the codes equal those of that separate call.

struct OutQ {
    uint8_t *codes;         // [M, N/2]
    uint8_t *scales;        // [M, N/16]
    float ts, rts;          // tensor scale of C and its reciprocal
    const float *inv_tab;   // fl(1 / fl(E4M3(c) * ts)), shared memory
};

// Inverse block-scale table of the IF4 output and the check of its tensor
// scale, by threads 0..127 of a CTA.
__device__ __forceinline__ void out_inv_table(float *inv_tab, const float *c_ts, int *err)
{
    if (threadIdx.x < 128) {
        const float ts = *c_ts;
        const float eff = __fmul_rn(f32_from_e4m3(threadIdx.x), ts);
        inv_tab[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __frcp_rn(eff);
        if (threadIdx.x == 0 && blockIdx.x == 0 && !(ts >= 0x1p-117f && ts <= 0x1p117f) && err)
            atomicOr(err, IF4_DEV_BAD_SCALE);
    }
}

// One output group of 16 bf16 values (8 words, element 2j in the low half of
// word j): IF4 codes and scale byte to codes_p / scale_p.  True on Inf/NaN.
__device__ __forceinline__ bool quantize_out_group(const uint32_t *w, const OutQ &oq,
                                                   uint8_t *codes_p, uint8_t *scale_p)
{
    uint32_t m = 0;
    f2_t xv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        m = absmax_bf16x2(m, w[j]);
        xv[j] = f2_from_bf16x2(w[j]);
    }
    const uint32_t m16 = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
    const float amax = __uint_as_float(m16 << 16);
    const If4Fast f = if4_fast(xv, amax, oq.ts, oq.rts, oq.inv_tab);
    const GroupCode out = if4_finish(f, amax, oq.ts, oq.rts, oq.inv_tab, [&](float (&y)[16]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) f2_unpack(xv[j], y[2 * j], y[2 * j + 1]);
    });
    st_v2(codes_p, out.c0, out.c1);
    st_u8(scale_p, out.scale);
    return m16 >= 0x7F80u;
}

// Store one row's 32-column chunk (raw fp32 accumulators r, scaled by
// `scale`): bf16 to C when c is given, IF4 when QOUT.  True on Inf/NaN.
template <bool QOUT>
__device__ __forceinline__ bool store_chunk(const uint32_t (&r)[32], float scale, int row, int M,
                                            int N, int col0, __nv_bfloat16 *c, const OutQ &oq)
{
    if (row >= M) return false;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        w[i] = bf16x2(__fmul_rn(__uint_as_float(r[2 * i]), scale),
                      __fmul_rn(__uint_as_float(r[2 * i + 1]), scale));
    if (c != nullptr) {
        __nv_bfloat16 *crow = c + (int64_t)row * N;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (col0 + q * 8 < N)
                st_v4(crow + col0 + q * 8, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
    bool nonfinite = false;
    if constexpr (QOUT) {
        const int64_t gpr = N / 16;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int col = col0 + 16 * h;
            if (col < N) {
                const int64_t gi = (int64_t)row * gpr + col / 16;
                nonfinite |= quantize_out_group(w + 8 * h, oq, oq.codes + gi * 8, oq.scales + gi);
            }
        }
    }
    return nonfinite;
}

// ------------------------------------------------------------- kernel ----

struct TileIter {
    int m_blocks, n_blocks, tiles;
    __device__ void coords(int t, int &m0, int &n0) const
    {
        // consecutive tiles walk down M inside one column of N tiles, so the
        // CTAs resident at one time share B slabs in L2
        m0 = (t % m_blocks) * BM;
        n0 = (t / m_blocks) * BN;
    }
};

template <bool QOUT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_f16_tcgen05(const __grid_constant__ CUtensorMap tmap_a,
                 const __grid_constant__ CUtensorMap tmap_b,
                 const float *__restrict__ a_ts, const float *__restrict__ b_ts,
                 __nv_bfloat16 *__restrict__ c, int M, int N, int K, int *err,
                 uint8_t *__restrict__ c_codes, uint8_t *__restrict__ c_scales,
                 const float *__restrict__ c_ts)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + STAGES * A_STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                    // [STAGES]
    uint64_t *empty = bars + STAGES;          // [STAGES]
    uint64_t *acc_full = bars + 2 * STAGES;   // [2]
    uint64_t *acc_empty = acc_full + 2;       // [2]
    uint64_t *drain = acc_empty + 2;          // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *inv_tab = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + 256);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const TileIter it{(M + BM - 1) / BM, (N + BN - 1) / BN,
                      ((M + BM - 1) / BM) * ((N + BN - 1) / BN)};
    const int k_blocks = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 4 * 32);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // programmatic launch: nothing above reads a kernel input; wait here
    // until the kernel before this one (the operand decode) has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if constexpr (QOUT) {
        out_inv_table(inv_tab, c_ts, err);
        __syncthreads();
    }

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------- TMA producer
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < it.tiles && ok; t += gridDim.x) {
            int m0, n0;
            it.coords(t, m0, n0);
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_expect_tx(fb, STAGE_BYTES);
                tma_load_2d(smem_u32(smem_a + stage * A_STAGE_BYTES), &tmap_a, kb * BK, m0, fb);
                tma_load_2d(smem_u32(smem_b + stage * B_STAGE_BYTES), &tmap_b, kb * BK, n0, fb);
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // every copy this thread issued must land before the CTA can exit:
        // wait (bounded) for the last min(issued, STAGES) stages to fill
        const int pending = issued < STAGES ? issued : STAGES;
        for (int i = 0; i < pending; ++i) {
            if (--stage < 0) { stage = STAGES - 1; phase ^= 1u; }
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(smem_u32(&full[stage]), phase))
                if (globaltimer() - t0 > WAIT_LIMIT_NS) break;
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < it.tiles && ok; t += gridDim.x) {
            if (!mbar_wait(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem_a + stage * A_STAGE_BYTES);
                const uint32_t b0 = smem_u32(smem_b + stage * B_STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                    umma_f16(d_tmem, smem_desc_sw128(a0 + kk * UMMA_K * 2),
                             smem_desc_sw128(b0 + kk * UMMA_K * 2), (kb | kk) != 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            umma_commit(smem_u32(&acc_full[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        // all MMAs this thread issued complete before tensor memory is freed
        umma_commit(smem_u32(drain));
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(drain), 0))
            if (globaltimer() - t0 > WAIT_LIMIT_NS) break;
    } else if (warp >= EPI_WARP0) {
        // -------------------------------------------------------- epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may read
        const int row_in_tile = quarter * 32 + lane;
        const float scale = __fmul_rn(*a_ts, *b_ts);
        OutQ oq{c_codes, c_scales, 1.0f, 1.0f, inv_tab};
        if constexpr (QOUT) {
            oq.ts = *c_ts;
            oq.rts = __frcp_rn(oq.ts);
        }
        bool nonfinite = false;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < it.tiles; t += gridDim.x) {
            int m0, n0;
            it.coords(t, m0, n0);
            // tcgen05.ld is warp-collective: every lane must take the same path
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&acc_full[acc]), acc_phase,
                                                              abort_flag));
            if (!ok) break;
            tc_fence_after();
            const int row = m0 + row_in_tile;
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t r[32];
                tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) +
                              (uint32_t)(acc * BN + chunk * 32), r);
                nonfinite |= store_chunk<QOUT>(r, scale, row, M, N, n0 + chunk * 32, c, oq);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&acc_empty[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (nonfinite && err) atomicOr(err, IF4_DEV_NONFINITE);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag && err) atomicOr(err, IF4_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem_base), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------ two-SM (CTA pair) GEMM ----
//
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): CTA r loads rows r*128..+127
// of the tile's A slab and of its B slab into its own shared memory, and the
// even CTA (the leader) issues MMAs that read both CTAs' halves, so each SM
// receives 32 KB per 64-wide K step instead of 48 KB.  The leader's full
// barrier counts both CTAs' copies (cp.async.bulk.tensor.cta_group::2 lets a
// copy complete on the peer's barrier); its tcgen05.commit is multicast to the
// same barrier in both CTAs, which frees a stage in both rings and announces
// a finished accumulator to both epilogues; each epilogue thread then arrives
// on the leader's accumulator-free barrier.  No load uses multicast.

namespace pair {

constexpr int PBM = 128;                 // rows per CTA (256 per pair)
constexpr int PBN = 256;                 // output columns per pair
constexpr int PBNH = PBN / 2;             // B rows loaded per CTA
constexpr int PSTAGES = 6;
constexpr int PA_BYTES = PBM * BK * 2;    // 16 KB
constexpr int PB_BYTES = PBNH * BK * 2;   // 16 KB
constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;
constexpr int PSMEM_BYTES = PSTAGES * PSTAGE_BYTES + 1024 + 256 + 512;
constexpr uint32_t PIDESC = (1u << 4) | ((uint32_t)(PBN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cta_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 :: "r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar_cluster)
{
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
                 : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(PIDESC), "r"(accumulate));
}

// arrive on barrier `bar` (same offset) in both CTAs when the MMAs complete
__device__ __forceinline__ void umma_commit_both(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
                 " [%0], %1;" :: "r"(bar), "h"((uint16_t)0x3) : "memory");
}

}  // namespace pair

template <bool QOUT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_f16_tcgen05_2sm(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const float *__restrict__ a_ts, const float *__restrict__ b_ts,
                     __nv_bfloat16 *__restrict__ c, int M, int N, int K, int *err,
                     uint8_t *__restrict__ c_codes, uint8_t *__restrict__ c_scales,
                     const float *__restrict__ c_ts)
{
    using namespace pair;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + PSTAGES * PA_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + PSTAGES * PSTAGE_BYTES);
    uint64_t *full = bars;                    // [PSTAGES], used in the leader
    uint64_t *empty = bars + PSTAGES;          // [PSTAGES], both CTAs
    uint64_t *acc_full = bars + 2 * PSTAGES;   // [2], both CTAs
    uint64_t *acc_empty = acc_full + 2;       // [2], used in the leader
    uint64_t *drain = acc_empty + 2;          // [1], leader
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *inv_tab = reinterpret_cast<float *>(smem + PSTAGES * PSTAGE_BYTES + 256);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const int m_tiles = (M + 2 * PBM - 1) / (2 * PBM);
    const int n_tiles = (N + PBN - 1) / PBN;
    const int tiles = m_tiles * n_tiles;
    const int pair_id = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const int k_blocks = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int st = 0; st < PSTAGES; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 2 * 4 * 32);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                      // peer barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // programmatic launch: nothing above reads a kernel input
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if constexpr (QOUT) {
        out_inv_table(inv_tab, c_ts, err);
        __syncthreads();
    }

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------- TMA producer
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = pair_id; t < tiles && ok; t += num_pairs) {
            const int m0 = (t % m_tiles) * 2 * PBM + (int)rank * PBM;
            const int n0 = (t / m_tiles) * PBN + (int)rank * PBNH;
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t fb = map_to(smem_u32(&full[stage]), 0);
                if (leader) mbar_expect_tx(smem_u32(&full[stage]), 2 * PSTAGE_BYTES);
                tma_load_2d_pair(smem_u32(smem_a + stage * PA_BYTES), &tmap_a, kb * BK, m0, fb);
                tma_load_2d_pair(smem_u32(smem_b + stage * PB_BYTES), &tmap_b, kb * BK, n0, fb);
                if (++stage == PSTAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // every copy issued here has been consumed by the leader's MMAs when
        // the loops end normally; after an abort, give them a bounded time
        const unsigned long long t0 = globaltimer();
        if (*abort_flag)
            while (globaltimer() - t0 < 2000000ull) { }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------- MMA issuer (leader)
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = pair_id; t < tiles && ok; t += num_pairs) {
            // both CTAs' epilogue threads arrive here, the peer's remotely
            if (!mbar_wait<true>(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PBN);
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem_a + stage * PA_BYTES);
                const uint32_t b0 = smem_u32(smem_b + stage * PB_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / UMMA_K; ++kk)
                    umma_f16_pair(d_tmem, smem_desc_sw128(a0 + kk * UMMA_K * 2),
                                  smem_desc_sw128(b0 + kk * UMMA_K * 2), (kb | kk) != 0 ? 1u : 0u);
                umma_commit_both(smem_u32(&empty[stage]));
                if (++stage == PSTAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            umma_commit_both(smem_u32(&acc_full[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                     :: "r"(smem_u32(drain)) : "memory");
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(drain), 0))
            if (globaltimer() - t0 > WAIT_LIMIT_NS) break;
    } else if (warp >= EPI_WARP0) {
        // -------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row_in_cta = quarter * 32 + lane;
        const float scale = __fmul_rn(*a_ts, *b_ts);
        OutQ oq{c_codes, c_scales, 1.0f, 1.0f, inv_tab};
        if constexpr (QOUT) {
            oq.ts = *c_ts;
            oq.rts = __frcp_rn(oq.ts);
        }
        bool nonfinite = false;
        const uint32_t acc_empty_leader0 = map_to(smem_u32(&acc_empty[0]), 0);
        const uint32_t acc_empty_leader1 = map_to(smem_u32(&acc_empty[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = pair_id; t < tiles; t += num_pairs) {
            const int m0 = (t % m_tiles) * 2 * PBM + (int)rank * PBM;
            const int n0 = (t / m_tiles) * PBN;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&acc_full[acc]), acc_phase,
                                                              abort_flag));
            if (!ok) break;
            tc_fence_after();
            const int row = m0 + row_in_cta;
#pragma unroll 1
            for (int chunk = 0; chunk < PBN / 32; ++chunk) {
                uint32_t r[32];
                tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) +
                              (uint32_t)(acc * PBN + chunk * 32), r);
                nonfinite |= store_chunk<QOUT>(r, scale, row, M, N, n0 + chunk * 32, c, oq);
            }
            tc_fence_before();
            arrive_remote(acc ? acc_empty_leader1 : acc_empty_leader0);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (nonfinite && err) atomicOr(err, IF4_DEV_NONFINITE);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                      // the peer's MMAs and copies are done
    if (threadIdx.x == 0 && *abort_flag && err) atomicOr(err, IF4_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem_base), "r"(TMEM_COLS));
    }
}

// ------------------------------------------- fused-decode CTA-pair GEMM ----
//
// The CTA-pair GEMM above with its TMA producer replaced by decoder warps,
// so the IF4 operands are decoded inside the GEMM (the MAC of the companion
// page "MAC Unit: Decoding Two Formats from One Sign Bit" routes each operand
// through its group's decoder before the multiply) and no fp16 workspace is
// needed.  Two sets of decoder warps take the K steps in turn.  Within a
// set, the decoder threads (TPR per row) split the CTA's operand slab (rows
// 0-127: A, 128-255: B) of a 64-wide K step.  Each copies its part of a row's
// 32 code bytes, and the row's 4 scale bytes, into its set's raw ring in
// shared memory with cp.async, two of the set's steps ahead (L2 serves the
// re-reads across tiles).  It decodes them as if4_decode_f16 does (the
// byte-permute decode with the same roundings, so the fp16 operands, and with
// the same MMA order the product, equal if4_linear's bit for bit), and writes
// its part of the row into the stage in the 128-byte swizzled layout the MMA
// descriptors read (16-byte chunk j of row r at position j ^ (r & 7)).  A
// proxy fence makes those generic stores visible to the tensor cores; then
// one lane per warp arrives on the CTA's own decoder barrier, and one
// forwarder thread per CTA relays the completed stage to the leader CTA's MMA
// barrier (release.cluster).

namespace fused {

constexpr int DEC_WARP0 = 6;                          // after TMA-less warp 0, MMA, epilogue
// Two sets of 8 decoder warps, each decoding whole slab rows of every other
// K step.  Measured at 8192 x 4096 x 4096 (with the wait hint): one set of 8
// warps 533 us; one set of 16 sharing rows, 522 us (without the hint); two
// sets of 8, 418 us.  A K step's decode is latency-bound, so two steps in
// flight help where more warps on the same step do not.
constexpr int DEC_WARPS = 16;
constexpr int FNUM_THREADS = (DEC_WARP0 + DEC_WARPS) * 32;
// NPAR sets of decoder warps take the K steps in turn (set p: steps p,
// p + NPAR, ...), so NPAR steps are decoded at once; within a set, TPR
// threads share each slab row.
constexpr int NPAR = 2;
constexpr int TPR = DEC_WARPS * 32 / (2 * pair::PBM * NPAR);
constexpr int SET_THREADS = 2 * pair::PBM * TPR;      // decoder threads per set
constexpr int GPT = 4 / TPR;                          // groups per thread per K step
static_assert(TPR == 1 || TPR == 2, "one or two decoder threads per slab row");
static_assert(NPAR == 1 || NPAR == 2, "one or two sets of decoder warps");
constexpr int FSTAGES = NPAR == 1 ? pair::PSTAGES : 5;  // operand stages (32 KB each)
// Raw ring: per K step, the slab's code bytes as two 4 KB planes (16 bytes
// of each row per plane, so a warp's 16-byte loads are conflict-free) and
// the row's 4 scale bytes once per decoder thread.  Each decoder thread
// fills and reads back its own part only, so cp.async's per-thread
// wait_group is the only ordering needed.  One ring per set.
constexpr int RAW_STAGES = 3;
constexpr int RAW_SCALE_OFF = 2 * 4096;
constexpr int RAW_STAGE_BYTES = RAW_SCALE_OFF + TPR * 1024;
constexpr int RAW_OFFSET = FSTAGES * pair::PSTAGE_BYTES + 1024;   // after barriers, table
constexpr int FSMEM_BYTES = RAW_OFFSET + NPAR * RAW_STAGES * RAW_STAGE_BYTES + 1024;
static_assert(FSMEM_BYTES <= 227 * 1024, "fused linear shared memory");

// cp.async of 16 (or 4) bytes with zero fill of the bytes past src_bytes
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
                 :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

__device__ __forceinline__ void lds_v4(uint32_t addr, uint32_t *w)
{
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr) : "memory");
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// 16 fp16 values of one group (code words w0, w1, scale byte sb), scaled by
// E4M3(sb) only, as if4_decode_f16 computes them: eight f16x2 words.
__device__ __forceinline__ void decode_group_f16(uint32_t w0, uint32_t w1, uint32_t sb,
                                                 uint32_t lut_addr, uint32_t (&o)[8])
{
    const float e4 = f32_from_e4m3(sb);
    const uint32_t base = lut_addr + ((sb >> 1) & 0x40u);
    float qa[8], qb[8];
    decode_word(w0, base, qa);
    decode_word(w1, base, qb);
    const f2_t EFF = f2_pack(e4, e4);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f2_unpack(f2_mul(f2_pack(qa[2 * j], qa[2 * j + 1]), EFF), lo, hi);
        o[j] = f16x2_from_f32(lo, hi);
        f2_unpack(f2_mul(f2_pack(qb[2 * j], qb[2 * j + 1]), EFF), lo, hi);
        o[4 + j] = f16x2_from_f32(lo, hi);
    }
}

__device__ __forceinline__ void sts_v4(uint32_t addr, const uint32_t *w)
{
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};"
                 :: "r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
}

}  // namespace fused

__global__ void __launch_bounds__(fused::FNUM_THREADS, 1)
gemm_if4_fused_2sm(const uint8_t *__restrict__ a_codes, const uint8_t *__restrict__ a_scales,
                   const uint8_t *__restrict__ b_codes, const uint8_t *__restrict__ b_scales,
                   const float *__restrict__ a_ts, const float *__restrict__ b_ts,
                   __nv_bfloat16 *__restrict__ c, int M, int N, int K, int *err)
{
    using namespace pair;
    using namespace fused;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + FSTAGES * PA_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + FSTAGES * PSTAGE_BYTES);
    uint64_t *full = bars;                    // [FSTAGES], used in the leader
    uint64_t *empty = bars + FSTAGES;          // [FSTAGES], both CTAs
    uint64_t *acc_full = bars + 2 * FSTAGES;   // [2], both CTAs
    uint64_t *acc_empty = acc_full + 2;       // [2], used in the leader
    uint64_t *drain = acc_empty + 2;          // [1], leader
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint64_t *dec_full = drain + 2;           // [FSTAGES], both CTAs: this CTA's decoders
    float *lut = reinterpret_cast<float *>(smem + FSTAGES * PSTAGE_BYTES + 256);
    uint8_t *raw = smem + RAW_OFFSET;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const int m_tiles = (M + 2 * PBM - 1) / (2 * PBM);
    const int n_tiles = (N + PBN - 1) / PBN;
    const int tiles = m_tiles * n_tiles;
    const int pair_id = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const int k_blocks = K / BK;

    if (threadIdx.x == 0) {
        for (int st = 0; st < FSTAGES; ++st) {
            mbar_init(smem_u32(&full[st]), 2);           // one forwarder per CTA
            mbar_init(smem_u32(&dec_full[st]), DEC_WARPS / NPAR);
            mbar_init(smem_u32(&empty[st]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 2 * 4 * 32);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x < 32) lut[threadIdx.x] = code_value(threadIdx.x);
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                      // peer barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // programmatic launch: nothing above reads a kernel input
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp >= DEC_WARP0) {
        // ------------------------------------------------------- decoders
        // thread td: set p = td / SET_THREADS takes the K steps i = p, p +
        // NPAR, ...; within the set, part h (GPT of the 4 groups) of slab row
        // srow (rows 0-127 A, 128-255 B)
        const int td = threadIdx.x - DEC_WARP0 * 32;
        const int par = td / SET_THREADS, tp = td % SET_THREADS;
        const int srow = tp & 255, h = tp >> 8;
        const bool is_a = srow < PBM;
        const int rloc = is_a ? srow : srow - PBM;              // row in this CTA's slab
        const uint8_t *codes = is_a ? a_codes : b_codes;
        const uint8_t *scales = is_a ? a_scales : b_scales;
        const int rows_total = is_a ? M : N;
        const uint32_t slab0 = smem_u32(is_a ? smem_a : smem_b) + (uint32_t)rloc * 128u;
        const uint32_t sw = (uint32_t)(rloc & 7);
        const uint32_t lut_addr = smem_u32(lut);
        const uint32_t raw0 = smem_u32(raw) + (uint32_t)(par * RAW_STAGES * RAW_STAGE_BYTES);
        // this thread's 16-byte code chunks c = h * (2 / TPR) + j (plane c, row
        // srow) and its scale word
        const uint32_t chunk0 = (uint32_t)h * (2u / TPR);
        const uint32_t code_off = chunk0 * 4096u + (uint32_t)srow * 16u;
        const uint32_t scale_off = RAW_SCALE_OFF + (uint32_t)tp * 4u;
        const int64_t code_stride = K / 2, scale_stride = K / 16;
        const int my_tiles = pair_id < tiles ? (tiles - pair_id + num_pairs - 1) / num_pairs : 0;
        const int64_t steps = (int64_t)my_tiles * k_blocks;
        const int64_t my_steps = steps > par ? (steps - par + NPAR - 1) / NPAR : 0;
        // Fetch side of the raw ring: copies the code bytes of this thread's
        // part of the set's fi-th step, and the row's 4 scale bytes
        // (zero-filled past the matrix), into slot fslot, one commit group per
        // step (an empty group past the end).  (ft, fkb): tile and K step.
        int ft = pair_id, fkb = par, fslot = 0;
        while (fkb >= k_blocks) { fkb -= k_blocks; ft += num_pairs; }
        int64_t fi = 0;
        auto fetch_next = [&]() {
            if (fi < my_steps) {
                const int row = (is_a ? (ft % m_tiles) * 2 * PBM + (int)rank * PBM
                                      : (ft / m_tiles) * PBN + (int)rank * PBNH) + rloc;
                const bool in = row < rows_total;
                const int rr = in ? row : 0;
                const uint8_t *src = codes + (int64_t)rr * code_stride + (int64_t)fkb * 32 +
                                     16 * chunk0;
                const uint32_t slot = raw0 + (uint32_t)fslot * RAW_STAGE_BYTES;
#pragma unroll
                for (int j = 0; j < 2 / TPR; ++j)
                    cp_async16(slot + code_off + (uint32_t)j * 4096u, src + 16 * j, in ? 16u : 0u);
                cp_async4(slot + scale_off,
                          scales + (int64_t)rr * scale_stride + (int64_t)fkb * 4, in ? 4u : 0u);
                fkb += NPAR;
                while (fkb >= k_blocks) { fkb -= k_blocks; ft += num_pairs; }
                ++fi;
                if (++fslot == RAW_STAGES) fslot = 0;
            }
            cp_async_commit();
        };
#pragma unroll 1
        for (int s = 0; s < RAW_STAGES - 1; ++s) fetch_next();
        // operand stage and phase of step i = par + NPAR * j: stage i % FSTAGES,
        // phase (i / FSTAGES) & 1
        int stage = par, rslot = 0;
        uint32_t phase = 0;
#pragma unroll 1
        for (int64_t j = 0; j < my_steps; ++j) {
            fetch_next();
            cp_async_wait<RAW_STAGES - 1>();             // this thread's bytes of the step landed
            const uint32_t slot = raw0 + (uint32_t)rslot * RAW_STAGE_BYTES;
            if (++rslot == RAW_STAGES) rslot = 0;
            uint32_t w[2 * GPT];
#pragma unroll
            for (int c = 0; c < 2 / TPR; ++c) lds_v4(slot + code_off + (uint32_t)c * 4096u, w + 4 * c);
            const uint32_t sc = lds_u32(slot + scale_off);
            // the stage is free once the MMAs that read it have completed
            bool freed = true;
            if (lane == 0) freed = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag);
            if (!__shfl_sync(0xFFFFFFFFu, freed ? 1 : 0, 0)) break;
            const uint32_t dst = slab0 + (uint32_t)stage * (uint32_t)PA_BYTES;
#pragma unroll
            for (uint32_t q = 0; q < (uint32_t)GPT; ++q) {
                const uint32_t g = (uint32_t)h * GPT + q;      // group in the 64-wide step
                uint32_t o[8];
                const uint32_t sb = (sc >> (8 * g)) & 0xFFu;
                const float e4 = f32_from_e4m3(sb);
                const uint32_t im = 0u - (sb >> 7);
                const BytePlanes P = group_planes<false>(lut_addr + ((sb >> 1) & 0x40u), e4);
                const uint32_t bad = decode_word16(w[2 * q], im, P, o) |
                                     decode_word16(w[2 * q + 1], im, P, o + 4);
                if (bad != 0u) decode_group_f16(w[2 * q], w[2 * q + 1], sb, lut_addr, o);
                sts_v4(dst + (((2u * g) ^ sw) << 4), o);
                sts_v4(dst + (((2u * g + 1u) ^ sw) << 4), o + 4);
            }
            // generic-proxy stores, then the MMA (async proxy) may read
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&dec_full[stage]));
            stage += NPAR;
            if (stage >= FSTAGES) { stage -= FSTAGES; phase ^= 1u; }
        }
        cp_async_wait<0>();                              // no copy in flight at exit
    } else if (warp == 0 && lane == 0) {
        // ------------------------------------------------------- forwarder
        // Relays each stage from this CTA's decoders (CTA-scope barrier) to
        // the leader's MMA barrier with one cluster-scope release, so the
        // decoder threads, whose prefetches are in flight, never issue one.
        const int my_tiles = pair_id < tiles ? (tiles - pair_id + num_pairs - 1) / num_pairs : 0;
        const int64_t steps = (int64_t)my_tiles * k_blocks;
        const uint32_t full_leader0 = map_to(smem_u32(&full[0]), 0);
        int stage = 0;
        uint32_t phase = 0;
        for (int64_t i = 0; i < steps; ++i) {
            if (!mbar_wait(smem_u32(&dec_full[stage]), phase, abort_flag)) break;
            arrive_remote(full_leader0 + (uint32_t)stage * 8u);
            if (++stage == FSTAGES) { stage = 0; phase ^= 1u; }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------- MMA issuer (leader)
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = pair_id; t < tiles && ok; t += num_pairs) {
            if (!mbar_wait<true>(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PBN);
            for (int kb = 0; kb < k_blocks; ++kb) {
                // both CTAs' decoder warps arrive here with release.cluster
                if (!mbar_wait<true>(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem_a + stage * PA_BYTES);
                const uint32_t b0 = smem_u32(smem_b + stage * PB_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / UMMA_K; ++kk)
                    umma_f16_pair(d_tmem, smem_desc_sw128(a0 + kk * UMMA_K * 2),
                                  smem_desc_sw128(b0 + kk * UMMA_K * 2), (kb | kk) != 0 ? 1u : 0u);
                umma_commit_both(smem_u32(&empty[stage]));
                if (++stage == FSTAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            umma_commit_both(smem_u32(&acc_full[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                     :: "r"(smem_u32(drain)) : "memory");
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(drain), 0))
            if (globaltimer() - t0 > WAIT_LIMIT_NS) break;
    } else if (warp >= EPI_WARP0) {
        // -------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row_in_cta = quarter * 32 + lane;
        const float scale = __fmul_rn(*a_ts, *b_ts);
        const OutQ oq{nullptr, nullptr, 1.0f, 1.0f, nullptr};
        const uint32_t acc_empty_leader0 = map_to(smem_u32(&acc_empty[0]), 0);
        const uint32_t acc_empty_leader1 = map_to(smem_u32(&acc_empty[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = pair_id; t < tiles; t += num_pairs) {
            const int m0 = (t % m_tiles) * 2 * PBM + (int)rank * PBM;
            const int n0 = (t / m_tiles) * PBN;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&acc_full[acc]), acc_phase,
                                                              abort_flag));
            if (!ok) break;
            tc_fence_after();
            const int row = m0 + row_in_cta;
#pragma unroll 1
            for (int chunk = 0; chunk < PBN / 32; ++chunk) {
                uint32_t r[32];
                tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) +
                              (uint32_t)(acc * PBN + chunk * 32), r);
                store_chunk<false>(r, scale, row, M, N, n0 + chunk * 32, c, oq);
            }
            tc_fence_before();
            arrive_remote(acc ? acc_empty_leader1 : acc_empty_leader0);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                      // the peer's MMAs and stores are done
    if (threadIdx.x == 0 && *abort_flag && err) atomicOr(err, IF4_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem_base), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------------ host side ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// K-major fp16 matrix [rows, K] -> tensor map with a (64 x box_rows) box.
bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count_checked(int &sms)
{
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return IF4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return IF4_ERR_CUDA;
    if (major != 10) return IF4_ERR_DEVICE;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return IF4_ERR_CUDA;
    return IF4_OK;
}

int check_gemm_args(const void *a, const void *b, const float *a_ts, const float *b_ts,
                    int64_t M, int64_t N, int64_t K, const void *c, const int *err)
{
    if (!a || !b || !a_ts || !b_ts || !c || !err) return IF4_ERR_NULL;
    if (M < 1 || N < 1 || K < 16 || K % 16 != 0 || N % 8 != 0) return IF4_ERR_SHAPE;
    if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return IF4_ERR_SHAPE;
    for (const void *p : {a, b, c})
        if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return IF4_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(a_ts) % 4 || reinterpret_cast<uintptr_t>(b_ts) % 4 ||
        reinterpret_cast<uintptr_t>(err) % 4)
        return IF4_ERR_ALIGN;
    return IF4_OK;
}

// Output of a launch: bf16 C (may be null when QOUT) and, when QOUT, the
// IF4 codes and scales of C under the tensor scale *c_ts.
struct GemmOut {
    void *c;
    uint8_t *c_codes, *c_scales;
    const float *c_ts;
};

template <bool QOUT>
int launch_gemm_t(const void *a, const void *b, const float *a_ts, const float *b_ts, int64_t M,
                  int64_t N, int64_t K, const GemmOut &o, int *err, cudaStream_t st)
{
    int sms = 0;
    int rc = sm_count_checked(sms);
    if (rc != IF4_OK) return rc;
    __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(o.c);
    // A CTA pair per 256 x 256 tile when both dimensions fill a pair tile,
    // otherwise one CTA per 128 x 256 tile.
    const bool use_pair = M >= 256 && N >= 256 && sms >= 2;
    CUtensorMap ma, mb;
    if (use_pair) {
        auto kernel = gemm_f16_tcgen05_2sm<QOUT>;
        if (!make_map(&ma, a, M, K, pair::PBM) || !make_map(&mb, b, N, K, pair::PBNH))
            return IF4_ERR_CUDA;
        static std::once_flag attr2_once;
        static cudaError_t attr2_rc = cudaSuccess;
        std::call_once(attr2_once, [&kernel] {
            attr2_rc = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            pair::PSMEM_BYTES);
        });
        if (attr2_rc != cudaSuccess) return IF4_ERR_CUDA;
        const int64_t tiles = ((M + 2 * pair::PBM - 1) / (2 * pair::PBM)) *
                              ((N + pair::PBN - 1) / pair::PBN);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * (sms / 2)), 1, 1);
        cfg.blockDim = dim3(NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = pair::PSMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // persistent: as many pairs as can be resident at once (SM pairs
        // must share a GPC, so this can be below sms / 2)
        static std::once_flag clusters_once;
        static int resident_pairs = 0;
        std::call_once(clusters_once, [&cfg, &kernel] {
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess)
                resident_pairs = n;
            else
                (void)cudaGetLastError();
        });
        int64_t pairs = resident_pairs > 0 ? resident_pairs : sms / 2;
        if (pairs > sms / 2) pairs = sms / 2;
        if (tiles < pairs) pairs = tiles;
        cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
        cfg.numAttrs = 2;                  // the cluster shape, then programmatic launch
        if (cudaLaunchKernelEx(&cfg, kernel, ma, mb, a_ts, b_ts, c, (int)M, (int)N, (int)K, err,
                               o.c_codes, o.c_scales, o.c_ts) != cudaSuccess)
            return IF4_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? IF4_OK : IF4_ERR_CUDA;
    }
    auto kernel = gemm_f16_tcgen05<QOUT>;
    if (!make_map(&ma, a, M, K, BM) || !make_map(&mb, b, N, K, BN)) return IF4_ERR_CUDA;
    static std::once_flag attr_once;
    static cudaError_t attr_rc = cudaSuccess;
    std::call_once(attr_once, [&kernel] {
        attr_rc = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
    });
    if (attr_rc != cudaSuccess) return IF4_ERR_CUDA;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, ma, mb, a_ts, b_ts, c, (int)M, (int)N, (int)K, err,
                           o.c_codes, o.c_scales, o.c_ts) != cudaSuccess)
        return IF4_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? IF4_OK : IF4_ERR_CUDA;
}

int launch_gemm(const void *a, const void *b, const float *a_ts, const float *b_ts, int64_t M,
                int64_t N, int64_t K, void *c, int *err, cudaStream_t st)
{
    const GemmOut o{c, nullptr, nullptr, nullptr};
    return launch_gemm_t<false>(a, b, a_ts, b_ts, M, N, K, o, err, st);
}

// The fused-decode linear: CTA pairs persistent over 256 x 256 tiles.
int launch_fused(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *b_codes,
                 const uint8_t *b_scales, const float *a_ts, const float *b_ts, int64_t M,
                 int64_t N, int64_t K, void *c, int *err, cudaStream_t st)
{
    int sms = 0;
    int rc = sm_count_checked(sms);
    if (rc != IF4_OK) return rc;
    if (sms < 2) return IF4_ERR_DEVICE;
    auto kernel = gemm_if4_fused_2sm;
    static std::once_flag attr_once;
    static cudaError_t attr_rc = cudaSuccess;
    std::call_once(attr_once, [&kernel] {
        attr_rc = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       fused::FSMEM_BYTES);
    });
    if (attr_rc != cudaSuccess) return IF4_ERR_CUDA;
    const int64_t tiles = ((M + 2 * pair::PBM - 1) / (2 * pair::PBM)) *
                          ((N + pair::PBN - 1) / pair::PBN);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * (sms / 2)), 1, 1);
    cfg.blockDim = dim3(fused::FNUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = fused::FSMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::once_flag clusters_once;
    static int resident_pairs = 0;
    std::call_once(clusters_once, [&cfg, &kernel] {
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess)
            resident_pairs = n;
        else
            (void)cudaGetLastError();
    });
    int64_t pairs = resident_pairs > 0 ? resident_pairs : sms / 2;
    if (pairs > sms / 2) pairs = sms / 2;
    if (tiles < pairs) pairs = tiles;
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kernel, a_codes, a_scales, b_codes, b_scales, a_ts, b_ts,
                           static_cast<__nv_bfloat16 *>(c), (int)M, (int)N, (int)K, err) !=
        cudaSuccess)
        return IF4_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? IF4_OK : IF4_ERR_CUDA;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" {

int if4_gemm_f16(const void *a, const void *b, const float *a_ts, const float *b_ts, int64_t M,
                 int64_t N, int64_t K, void *c, int *err_flag, void *stream)
{
    int rc = check_gemm_args(a, b, a_ts, b_ts, M, N, K, c, err_flag);
    if (rc != IF4_OK) return rc;
    return launch_gemm(a, b, a_ts, b_ts, M, N, K, c, err_flag, static_cast<cudaStream_t>(stream));
}

size_t if4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 16 || K % 16 != 0) return 0;
    return align_up((size_t)M * (size_t)K * 2, 256) + (size_t)N * (size_t)K * 2;
}

int if4_linear(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
               const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts, int64_t M,
               int64_t N, int64_t K, void *workspace, size_t ws_bytes, void *c, int *err_flag,
               void *stream)
{
    if (!a_codes || !a_scales || !b_codes || !b_scales) return IF4_ERR_NULL;
    int rc = check_gemm_args(a_codes, b_codes, a_ts, b_ts, M, N, K, c, err_flag);
    if (rc != IF4_OK) return rc;
    const size_t need = if4_linear_workspace_bytes(M, N, K);
    if (workspace == nullptr || ws_bytes < need) return IF4_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return IF4_ERR_ALIGN;
    uint8_t *wa = static_cast<uint8_t *>(workspace);
    uint8_t *wb = wa + align_up((size_t)M * (size_t)K * 2, 256);
    rc = internal_decode_f16_pair(a_codes, a_scales, M, wa, b_codes, b_scales, N, wb, K, stream);
    if (rc != IF4_OK) return rc;
    return launch_gemm(wa, wb, a_ts, b_ts, M, N, K, c, err_flag, static_cast<cudaStream_t>(stream));
}

int if4_linear_fused(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
                     const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts, int64_t M,
                     int64_t N, int64_t K, void *c, int *err_flag, void *stream)
{
    if (!a_codes || !a_scales || !b_codes || !b_scales) return IF4_ERR_NULL;
    int rc = check_gemm_args(a_codes, b_codes, a_ts, b_ts, M, N, K, c, err_flag);
    if (rc != IF4_OK) return rc;
    if (K % 64 != 0) return IF4_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(a_codes) % 32 || reinterpret_cast<uintptr_t>(b_codes) % 32 ||
        reinterpret_cast<uintptr_t>(a_scales) % 4 || reinterpret_cast<uintptr_t>(b_scales) % 4)
        return IF4_ERR_ALIGN;
    return launch_fused(a_codes, a_scales, b_codes, b_scales, a_ts, b_ts, M, N, K, c, err_flag,
                        static_cast<cudaStream_t>(stream));
}

int if4_linear_quantized(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
                         const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts,
                         int64_t M, int64_t N, int64_t K, void *workspace, size_t ws_bytes,
                         void *c, uint8_t *c_codes, uint8_t *c_scales, const float *c_ts,
                         int *err_flag, void *stream)
{
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c_codes || !c_scales || !c_ts)
        return IF4_ERR_NULL;
    // c is optional here; the shared checks see the codes pointer in its place
    int rc = check_gemm_args(a_codes, b_codes, a_ts, b_ts, M, N, K, c ? c : c_codes, err_flag);
    if (rc != IF4_OK) return rc;
    if (N % 16 != 0) return IF4_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(c_codes) % 16 != 0 || reinterpret_cast<uintptr_t>(c_ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    const size_t need = if4_linear_workspace_bytes(M, N, K);
    if (workspace == nullptr || ws_bytes < need) return IF4_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return IF4_ERR_ALIGN;
    uint8_t *wa = static_cast<uint8_t *>(workspace);
    uint8_t *wb = wa + align_up((size_t)M * (size_t)K * 2, 256);
    rc = internal_decode_f16_pair(a_codes, a_scales, M, wa, b_codes, b_scales, N, wb, K, stream);
    if (rc != IF4_OK) return rc;
    const GemmOut o{c, c_codes, c_scales, c_ts};
    return launch_gemm_t<true>(wa, wb, a_ts, b_ts, M, N, K, o, err_flag,
                               static_cast<cudaStream_t>(stream));
}

}  // extern "C"
