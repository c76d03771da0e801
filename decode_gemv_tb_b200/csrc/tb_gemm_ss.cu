// tb_gemm_ss.cu -- Y = X W^T for prefill batches (64 < M <= 65536 rows) on
// the fifth-generation tensor cores (tcgen05), straight from the packed 2-
// and 3-bit codewords, with both MMA operands in shared memory.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나: w = c * s with
// one bf16 scale per 128 input weights; per output row n, batch row m and
// 128-group g
//     Y[m][n] += s[n][g] * sum_k c[n][k] X[m][k].
// Section 무엇인가: the weights are read once for all batch rows, so the
// product turns from memory-bound (a few rows) into a dense contraction.
//
// Work.  A unit is (tile of 128 weight rows, block of 128 batch rows); the
// call's work is the sequence of (unit, group) chunks, units in tile order
// (the batch blocks of a tile are neighbours, so the tile's packed bytes are
// re-read from L2), groups in k order.  One CTA per SM owns an equal
// contiguous range of chunks; a unit split between CTAs is finished by the
// CTA that holds its first chunk (for it the unit is the last segment of its
// range): each later CTA writes its partial sums and releases a flag, the
// finishing CTA acquires the flags (and clears them) and adds the sums in
// CTA order (bitwise deterministic).
//
// Pipeline of a CTA (19 warps), per chunk:
//   * producer warp: the block's activations of the group (128 rows x 128
//     bf16, rows past M read as zero) as two tensor copies (no multicast)
//     with 128-byte swizzle -- the MMA's K-major B layout -- into a ring of
//     activation stages;
//   * 8 decoder warps: each thread reads half a row's packed group from
//     global memory (four groups ahead, in registers), decodes it to the
//     signed codeword, exactly, as bf16 (tb_device.cuh) and stores it into
//     one of four A stages in the same swizzled K-major layout;
//   * MMA warps (the even chunks, the odd chunks): eight 128 x 128 x 16 MMAs
//     (kind::f16, bf16 in, fp32 out) into accumulator d = chunk mod 2 of
//     tensor memory, committed to three
//     mbarriers: the A stage and the activation stage are free, the
//     accumulator is ready;
//   * 8 epilogue warps (two per 32 TMEM lanes = 32 rows, each half of the
//     batch columns): read the accumulator back, release it, and add  s * D
//     to the row's running sums, kept in the last 128 columns of tensor
//     memory.  Every product c * x is exact;
//     the sums over a group (8 MMAs) and over groups are fp32.
// Every wait is bounded.  A wait that gives up is counted
// (g_ss_timeouts), raises the CTA's abort flag -- every other wait of the
// CTA then gives up at once -- and the CTA writes NaN to the outputs of its
// range, waits (bounded) for its copies and MMAs in flight, frees its tensor
// memory and exits.
#include "tb_device.cuh"
#include "tb_internal.h"

#include <algorithm>
#include <cstring>

namespace tb {

__device__ unsigned int g_ss_timeouts = 0;

namespace {

constexpr int kSSRows = 128;        // weight rows per tile (the MMA's M)
constexpr int kSSStages = 4;        // decoded A operands in shared memory
constexpr int kSSNP = 128;          // batch rows per unit: the MMA's N (two 64-row blocks share a decode)
constexpr int kSSDecWarps = 8;      // a thread per half of a row's group
constexpr int kSSEpiWarps = 8;      // two per 32 TMEM lanes, half the columns each
constexpr int kSSWarpDec0 = 2;                            // warps 2 .. 9 decode
constexpr int kSSWarpEpi0 = kSSWarpDec0 + kSSDecWarps;   // warps 10 .. 17 finish
// warps 1 and 18 issue the MMAs of the even and the odd chunks: an MMA
// holds its issuing thread for about 150 cycles, so one warp cannot keep
// pace with the decoders
constexpr int kSSWarpMma1 = kSSWarpEpi0 + kSSEpiWarps;
constexpr int kSSThreads = (kSSWarpMma1 + 1) * 32;
constexpr int kSSABytes = kSSRows * kGroup * 2;  // decoded group, bf16
constexpr uint64_t kSSMaxCtas = 256;             // bound of the grid (one CTA per SM)
constexpr int kSSPrefetch = 4;                   // groups of packed codes in flight per decoder thread

__host__ __device__ constexpr int ss_xbytes(int np) { return np * kGroup * 2; }
// activation stages (as many as fit beside the four A stages)
// (stage and accumulator counts are even: each is then waited on by one MMA warp, in order)
__host__ __device__ constexpr int ss_xstages(int np) { return np <= 32 ? 8 : (np <= 64 ? 4 : 2); }
// accumulators in tensor memory: its 512 columns less the running sums' NP
__host__ __device__ constexpr int ss_dbufs(int np) { return (512 / np - 1) & ~1; }
__host__ __device__ constexpr int ss_smem_bytes(int np) {
    return kSSStages * kSSABytes + ss_xstages(np) * ss_xbytes(np) + 1024;
}
static_assert(ss_smem_bytes(kSSNP) + 512 <= 227 * 1024, "shared memory");
static_assert(kSSStages == 4 && kSSPrefetch % kSSStages == 0, "the decoders' ring is unrolled by its depth");

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---- mbarriers ---------------------------------------------------------------
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void bar_arrive_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// true once the phase with this parity has completed; false when the CTA has
// aborted or after `limit` cycles (which aborts the CTA and is counted)
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, long long limit, volatile int* abort,
                                         uint32_t sleep_ns = 0) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity), "r"(20000u)
            : "memory");
        if (done) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            atomicAdd(&g_ss_timeouts, 1u);
            *abort = 1;
            return false;
        }
        if (sleep_ns) __nanosleep(sleep_ns);  // roles off the critical path leave the issue slots to the decoders
    }
}
// the same wait without abort checks (draining what is in flight before exit)
__device__ __forceinline__ void bar_drain(uint32_t bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done || clock64() - t0 > limit) return;
    }
}

// ---- tensor copies (no multicast) -----------------------------------------------
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// global -> registers, not kept in L1; L2 fetches the surrounding 256 bytes
// (the next groups of the same row)
__device__ __forceinline__ uint4 ldg_nc16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---- tcgen05 -------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory descriptor of a K-major operand in the 128-byte swizzle
// layout a tensor copy with CU_TENSOR_MAP_SWIZZLE_128B writes: rows of 128 bytes (64 bf16),
// 8-row atoms of 1 KB (stride 1024), 16-byte chunks XOR'ed with the row in
// the atom; a k offset inside the row is added to the start address.
__device__ __forceinline__ uint64_t kdesc_sw128(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
// kind::f16 instruction descriptor: fp32 D, bf16 A and B, both K-major, M = 128, N = np
__host__ __device__ constexpr uint32_t ss_idesc(int np) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(np >> 3) << 17) | ((uint32_t)(kSSRows >> 4) << 24);
}
// D[tmem d] (+)= A[smem] B[smem], issued by one elected lane of a converged warp
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred e, p;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// the MMAs issued so far by this thread, once complete, arrive on bar
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}" ::"r"(bar)
        : "memory");
}
// 16 consecutive columns of this thread's TMEM lane (complete after tmem_ld_wait)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// the registers of a tcgen05.ld, tied to a point after tmem_ld_wait (the wait
// names no register, so without this the compiler may use them before it)
__device__ __forceinline__ void tmem_regs_after_wait(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]));
}

// ---- partial sums between CTAs: a release flag per CTA --------------------------------
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

constexpr float kNaN = __builtin_nanf("");

// Waits (acquire) until a later CTA has released its flag, then clears it
// for the next call; gives up when the CTA has aborted or after `limit`
// cycles (which aborts the CTA and is counted).
__device__ __forceinline__ void take_flag(uint32_t* f, long long limit, volatile int* abort) {
    const long long t0 = clock64();
    while (ld_acquire(f) == 0u) {
        if (*abort) return;
        if (clock64() - t0 > limit) {
            atomicAdd(&g_ss_timeouts, 1u);
            *abort = 1;
            return;
        }
        __nanosleep(64);
    }
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(0u) : "memory");
}

}  // namespace

struct SSArgs {
    CUtensorMap xmap;         // X: bf16 {K, M} (row stride 2 ldx bytes), box {64, NP}, 128-byte swizzle
    const uint8_t* packed;    // [N][rb] packed codes
    const uint16_t* scales;   // [N][G] bf16
    void* Y;                  // [M][ldy]
    uint32_t* pflag;          // [ctas] release flags of published partial sums (zero between calls)
    float* pdata;             // [ctas][128][NP] published partial sums
    int64_t N, ldy, rb;
    uint64_t Q;               // chunks: T * MB * G
    long long wait_cycles;
    int32_t M, G, MB, ydt, ctas;
    int32_t xrows;            // rows of an activation box: min(NP, M) (the MMA's other columns are never stored)
};

namespace {

// first chunk of CTA c: floor(c Q / P)
__device__ __forceinline__ uint64_t ss_first(uint64_t c, uint64_t Q, uint64_t P) { return c * Q / P; }
// the CTA whose range holds chunk x
__device__ __forceinline__ uint64_t ss_owner(uint64_t x, uint64_t Q, uint64_t P) { return ((x + 1) * P - 1) / Q; }

template <int NP, int KIND>
__global__ void __launch_bounds__(kSSThreads, 1) k_gemm_ss(const __grid_constant__ SSArgs A) {
    constexpr int XB = ss_xbytes(NP);
    constexpr int XS = ss_xstages(NP);
    constexpr int kSSDBufs = ss_dbufs(NP);
    constexpr int kSSBlockM = NP;  // batch rows per unit
    constexpr int GB = KIND ? 48 : 32;  // packed bytes of one row's group
    constexpr uint32_t kIdesc = ss_idesc(NP);
    constexpr uint32_t kTmemCols = 512;  // kSSDBufs accumulators of NP columns, then NP columns of running sums
    static_assert(NP * (kSSDBufs + 1) <= (int)kTmemCols, "tensor memory");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t afull[kSSStages], aempty[kSSStages], xfull[XS], xempty[XS];
    __shared__ __align__(8) uint64_t dfull[kSSDBufs], dfree[kSSDBufs];
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_sh;
    volatile int* abort = &abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = saddr(smem_raw);
    uint8_t* const base = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // A stages, then X stages
    const uint32_t base_s = saddr(base);
    const uint32_t xbase_s = base_s + kSSStages * kSSABytes;
    const uint64_t P = (uint64_t)gridDim.x, cta = blockIdx.x;
    const uint64_t q0 = ss_first(cta, A.Q, P), q1 = ss_first(cta + 1, A.Q, P);
    const int n = (int)(q1 - q0);
    const uint32_t G = (uint32_t)A.G, MB = (uint32_t)A.MB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSSStages; ++s) {
            bar_init(saddr(&afull[s]), kSSDecWarps);
            bar_init(saddr(&aempty[s]), 1);
        }
        for (int s = 0; s < XS; ++s) {
            bar_init(saddr(&xfull[s]), 1);
            bar_init(saddr(&xempty[s]), 1);
        }
        for (int d = 0; d < kSSDBufs; ++d) {
            bar_init(saddr(&dfull[d]), 1);
            bar_init(saddr(&dfree[d]), kSSEpiWarps);
        }
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&tmem_sh)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;
    int issued = 0, committed = 0;  // producer: chunks requested; MMA warp: its last chunk committed, plus one

    if (warp == 0) {
        // ---------------- producer: the activations of every chunk, XS ahead ----------------
        if (lane == 0) {
            uint32_t u = (uint32_t)(q0 / G), g = (uint32_t)(q0 % G);
            for (int k = 0; k < n; ++k) {
                const int s = k % XS;
                if (k >= XS && !bar_wait(saddr(&xempty[s]), (uint32_t)(k / XS - 1) & 1u, A.wait_cycles, abort, 64))
                    break;
                const uint32_t b = u % MB;  // the unit's batch block
                const uint32_t st = xbase_s + s * XB, bar = saddr(&xfull[s]);
                bar_arrive_expect(bar, (uint32_t)(2 * 128 * A.xrows));
                tma_2d(st, &A.xmap, (int)(g * kGroup), (int)(b * kSSBlockM), bar);
                tma_2d(st + NP * 128, &A.xmap, (int)(g * kGroup + 64), (int)(b * kSSBlockM), bar);
                issued = k + 1;
                if (++g == G) {
                    g = 0;
                    ++u;
                }
            }
        }
    } else if (warp == 1 || warp == kSSWarpMma1) {
        // ---------------- MMA issuers: chunk k by warp 1 (k even) or kSSWarpMma1 (k odd) ----------------
        static_assert(kSSStages % 2 == 0 && XS % 2 == 0 && kSSDBufs % 2 == 0, "one waiting warp per stage");
        for (int k = warp == 1 ? 0 : 1; k < n; k += 2) {
            const int s = k % kSSStages, x = k % XS, d = k % kSSDBufs;
            if (!__all_sync(0xffffffffu, bar_wait(saddr(&afull[s]), (uint32_t)(k / kSSStages) & 1u, A.wait_cycles,
                                                  abort)))
                break;
            if (!__all_sync(0xffffffffu, bar_wait(saddr(&xfull[x]), (uint32_t)(k / XS) & 1u, A.wait_cycles, abort)))
                break;
            if (k >= kSSDBufs && !__all_sync(0xffffffffu, bar_wait(saddr(&dfree[d]), (uint32_t)(k / kSSDBufs - 1) & 1u,
                                                                   A.wait_cycles, abort)))
                break;
            tc_fence_after();
            const uint32_t sa = base_s + s * kSSABytes, sx = xbase_s + x * XB;
            const uint32_t dcol = tmem + (uint32_t)(d * NP);
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // k slice j: bytes 32 (j % 4) of the rows of 64-k column j / 4, A and X
                const uint64_t ad = kdesc_sw128(sa + (uint32_t)((j >> 2) * kSSRows * 128 + (j & 3) * 32));
                const uint64_t bd = kdesc_sw128(sx + (uint32_t)((j >> 2) * NP * 128 + (j & 3) * 32));
                mma_ss(dcol, ad, bd, kIdesc, j > 0 ? 1u : 0u);
            }
            mma_commit(saddr(&aempty[s]));
            mma_commit(saddr(&xempty[x]));
            mma_commit(saddr(&dfull[d]));
            committed = k + 1;
        }
    } else if (warp < kSSWarpEpi0) {
        // ---------------- decoders: row r, k half h (64 codes) of every group ----------------
        // The packed codes come straight from global memory into registers,
        // kSSPrefetch groups ahead of the decode.  A quarter warp covers 8
        // consecutive rows (distinct 16-byte bank groups in the swizzled A).
        constexpr int HW = KIND ? 6 : 4;  // packed words of half a row's group
        const int dw = warp - kSSWarpDec0;
        const int r = 16 * dw + (lane & 15), h = lane >> 4;
        uint32_t pg = (uint32_t)(q0 % G), pt = (uint32_t)(q0 / G / MB), pbk = (uint32_t)(q0 / G % MB);  // next load
        auto load = [&](uint32_t (&w)[HW]) {
            const int64_t row = (int64_t)pt * kSSRows + r;
            if (row < A.N) {
                if constexpr (KIND == 0) {
                    const uint4 v = ldg_nc16(A.packed + row * A.rb + (int64_t)pg * GB + 16 * h);
                    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
                } else {
                    // 48 bytes = three 16-byte pieces; half 0 takes words 0-5 (pieces 0, 1), half 1 words 6-11
                    // (pieces 1, 2): two aligned 16-byte loads each
                    const uint8_t* p = A.packed + row * A.rb + (int64_t)pg * GB + 16 * h;
                    const uint4 v0 = ldg_nc16(p), v1 = ldg_nc16(p + 16);
                    if (h == 0) w[0] = v0.x, w[1] = v0.y, w[2] = v0.z, w[3] = v0.w, w[4] = v1.x, w[5] = v1.y;
                    else w[0] = v0.z, w[1] = v0.w, w[2] = v1.x, w[3] = v1.y, w[4] = v1.z, w[5] = v1.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < HW; ++i) w[i] = 0u;
            }
            if (++pg == G) {
                pg = 0;
                if (++pbk == MB) {
                    pbk = 0;
                    ++pt;
                }
            }
        };
        // ring of PF groups' codes: buffer j % PF holds group j until its
        // decode starts, then is refilled with group j + PF (the index is a
        // compile-time constant in the unrolled body, so no load is waited
        // for before its turn)
        constexpr int PF = kSSPrefetch;
        uint32_t pb[PF][HW];
#pragma unroll
        for (int j = 0; j < PF; ++j)
            if (j < n) load(pb[j]);
        // row r of the swizzled A (64-k column h): 16-byte chunk c at (c ^ (r % 8)) * 16
        const uint32_t arow = (uint32_t)(h * (kSSRows * 128) + r * 128);
        const int sw = r & 7;
        bool stop = false;
#pragma unroll 1
        for (int k0 = 0; k0 < n && !stop; k0 += PF) {
#pragma unroll
            for (int j = 0; j < PF; ++j) {
                const int k = k0 + j;
                if (k >= n || stop) break;
                const int s = j % kSSStages;  // k % kSSStages
                // the A operand of stage s: the MMAs of chunk k - 4 have read it
                if (k >= kSSStages &&
                    !__all_sync(0xffffffffu, bar_wait(saddr(&aempty[s]), (uint32_t)(k / kSSStages - 1) & 1u,
                                                      A.wait_cycles, abort))) {
                    stop = true;
                    break;
                }
                uint32_t ws[HW];
#pragma unroll
                for (int i = 0; i < HW; ++i) ws[i] = pb[j][i];
                if (k + PF < n) load(pb[j]);
                uint8_t* a = base + s * kSSABytes + arow;
                if constexpr (KIND == 0) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {  // word i: codes 16 i .. 16 i + 15 of the half, chunks 2 i, 2 i + 1
                        uint32_t c[8];
                        decode2_signed<2>(ws[i], c);
                        *reinterpret_cast<uint4*>(a + (((2 * i) ^ sw) << 4)) = make_uint4(c[0], c[1], c[2], c[3]);
                        *reinterpret_cast<uint4*>(a + (((2 * i + 1) ^ sw) << 4)) = make_uint4(c[4], c[5], c[6], c[7]);
                    }
                } else {
#pragma unroll
                    for (int bl = 0; bl < 2; ++bl) {  // block bl: codes 32 bl .. 32 bl + 31 of the half, chunks 4 bl ..
                        uint32_t c[16];
                        decode3_signed(ws[3 * bl], ws[3 * bl + 1], ws[3 * bl + 2], c);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4*>(a + (((4 * bl + q) ^ sw) << 4)) =
                                make_uint4(c[4 * q], c[4 * q + 1], c[4 * q + 2], c[4 * q + 3]);
                    }
                }
                // the tensor cores read the stage through the async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) bar_arrive(saddr(&afull[s]));
            }
        }
    } else {
        // ---------------- epilogue: rows 32 (warp % 4) .. + 31, columns NH eh .. NH eh + NH - 1 ----------------
        // The row's running sums of a segment live in tensor memory (the
        // columns after the accumulators), 16 columns at a time in registers.
        constexpr int NH = NP / 2, W = 16;
        static_assert(NH % (2 * W) == 0, "epilogue columns");
        const int qd = warp & 3, eh = (warp - kSSWarpEpi0) >> 2;
        const int r = 32 * qd + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(eh * NH);
        const uint32_t scol = lane_base + (uint32_t)(kSSDBufs * NP);  // running sums
        // scales four chunks ahead (cursor pt, pbk, pg)
        uint32_t pg = (uint32_t)(q0 % G), pt = (uint32_t)(q0 / G / MB), pbk = (uint32_t)(q0 / G % MB);
        float sq[4] = {0.f, 0.f, 0.f, 0.f};  // the scales of the next block of four chunks
        auto next_scale = [&]() -> float {
            const int64_t row = (int64_t)pt * kSSRows + r;
            const float v = row < A.N ? bf16_bits_to_float(__ldg(A.scales + row * G + pg)) : 0.f;
            if (++pg == G) {
                pg = 0;
                if (++pbk == MB) {
                    pbk = 0;
                    ++pt;
                }
            }
            return v;
        };
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < n) sq[j] = next_scale();
        uint32_t u = (uint32_t)(q0 / G), g = (uint32_t)(q0 % G);
        uint64_t seg0 = q0;  // first chunk of the current segment
        bool failed = false;
        auto zero_sums = [&]() {
            uint32_t z[W];
#pragma unroll
            for (int i = 0; i < W; ++i) z[i] = 0u;
#pragma unroll
            for (int cc = 0; cc < NH; cc += W) tmem_st16(scol + cc, z);
            tmem_st_wait();
        };
        zero_sums();
#pragma unroll 1
        for (int k0 = 0; k0 < n; k0 += 4) {
          // this block's four scales (requested during the previous block); request the next block's
          const float c0 = sq[0], c1 = sq[1], c2 = sq[2], c3 = sq[3];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
              if (k0 + 4 + jj < n) sq[jj] = next_scale();
#pragma unroll 1
          for (int jj = 0; jj < 4; ++jj) {
            const int k = k0 + jj;
            if (k >= n) break;
            const int d = k % kSSDBufs;
            const float sc = jj == 0 ? c0 : (jj == 1 ? c1 : (jj == 2 ? c2 : c3));
            if (!failed)
                failed = !__all_sync(0xffffffffu, bar_wait(saddr(&dfull[d]), (uint32_t)(k / kSSDBufs) & 1u,
                                                           A.wait_cycles, abort, 128));
            if (!failed) {
                tc_fence_after();
                const uint32_t col = lane_base + (uint32_t)(d * NP);
#pragma unroll 1
                for (int cc = 0; cc < NH; cc += 2 * W) {  // sums += s * D, 32 columns (one wait) at a time
                    uint32_t v[2][W], a[2][W];
                    tmem_ld16(col + cc, v[0]);
                    tmem_ld16(col + cc + W, v[1]);
                    tmem_ld16(scol + cc, a[0]);
                    tmem_ld16(scol + cc + W, a[1]);
                    tmem_ld_wait();
                    tmem_regs_after_wait(v[0]);
                    tmem_regs_after_wait(v[1]);
                    tmem_regs_after_wait(a[0]);
                    tmem_regs_after_wait(a[1]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int i = 0; i < W; ++i)
                            a[h][i] = __float_as_uint(fmaf(sc, __uint_as_float(v[h][i]), __uint_as_float(a[h][i])));
                        tmem_st16(scol + cc + h * W, a[h]);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) bar_arrive(saddr(&dfree[d]));
            }
            // end of the unit or of the range: finish the segment
            const uint64_t q = q0 + (uint64_t)k;
            if (g + 1 == G || k + 1 == n) {
                const uint64_t ustart = (uint64_t)u * G, uend = ustart + G;
                const uint32_t t = u / MB, b = u - t * MB;
                const bool publish = seg0 > ustart;  // a later part of a unit begun by an earlier CTA
                const uint64_t c1 = (!publish && uend > q1) ? ss_owner(uend - 1, A.Q, P) : cta;
                const int64_t row = (int64_t)t * kSSRows + r;
                auto sums = [&](int cc, float (&acc)[W]) {  // this segment's sums, columns cc .. cc + 15
                    if (!failed) {
                        uint32_t a[W];
                        tmem_ld16(scol + cc, a);
                        tmem_ld_wait();
                        tmem_regs_after_wait(a);
#pragma unroll
                        for (int i = 0; i < W; ++i) acc[i] = __uint_as_float(a[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < W; ++i) acc[i] = kNaN;
                    }
                };
                if (publish) {
                    // the partial sums, then (all epilogue threads done) one release of this CTA's flag
                    float* pd = A.pdata + ((uint64_t)cta * kSSRows + r) * NP + eh * NH;
#pragma unroll 1
                    for (int cc = 0; cc < NH; cc += W) {
                        float acc[W];
                        sums(cc, acc);
#pragma unroll
                        for (int i = 0; i < W; i += 4)
                            *reinterpret_cast<float4*>(pd + cc + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
                    }
                    __threadfence();  // each thread's own sums, before the barrier that precedes the release
                    named_sync(1, kSSEpiWarps * 32);
                    if (warp == kSSWarpEpi0 && lane == 0) {
                        __threadfence();
                        st_release(A.pflag + cta, 1u);
                    }
                } else {
                    if (c1 > cta) {  // one thread acquires the later CTAs' flags (and clears them), then all read
                        if (warp == kSSWarpEpi0 && lane == 0)
                            for (uint64_t c = cta + 1; c <= c1; ++c) take_flag(A.pflag + c, A.wait_cycles, abort);
                        named_sync(1, kSSEpiWarps * 32);
                    }
                    const bool lost = *abort != 0;
#pragma unroll 1
                    for (int cc = 0; cc < NH; cc += W) {
                        float acc[W];
                        sums(cc, acc);
#pragma unroll 1
                        for (uint64_t c = cta + 1; c <= c1; ++c) {  // the later CTAs' sums, in CTA order
                            const float4* pd =
                                reinterpret_cast<const float4*>(A.pdata + (c * kSSRows + r) * NP + eh * NH + cc);
#pragma unroll
                            for (int i = 0; i < W / 4; ++i) {
                                const float4 v = __ldcg(pd + i);
                                acc[4 * i] += v.x;
                                acc[4 * i + 1] += v.y;
                                acc[4 * i + 2] += v.z;
                                acc[4 * i + 3] += v.w;
                            }
                        }
                        if (lost) {
#pragma unroll
                            for (int i = 0; i < W; ++i) acc[i] = kNaN;
                        }
                        if (row < A.N) {
#pragma unroll
                            for (int i = 0; i < W; ++i) {
                                const int64_t m = (int64_t)b * kSSBlockM + eh * NH + cc + i;
                                if (m < A.M) {
                                    if (A.ydt == kF32) static_cast<float*>(A.Y)[m * A.ldy + row] = acc[i];
                                    else
                                        static_cast<__nv_bfloat16*>(A.Y)[m * A.ldy + row] = __float2bfloat16_rn(acc[i]);
                                }
                            }
                        }
                    }
                }
                if (!failed) zero_sums();
                seg0 = q + 1;
            }
            if (++g == G) {
                g = 0;
                ++u;
            }
          }
        }
        tc_fence_before();
    }

    // ---------------- drain and exit ----------------
    const bool aborted = __syncthreads_or(*abort) != 0;
    if (aborted) {
        if (warp == 0 && lane == 0)  // the newest copy of each stage (older ones landed before it was refilled)
            for (int k = issued > XS ? issued - XS : 0; k < issued; ++k)
                bar_drain(saddr(&xfull[k % XS]), (uint32_t)(k / XS) & 1u, A.wait_cycles);
        if ((warp == 1 || warp == kSSWarpMma1) && committed > 0)  // each warp's commits complete in order
            bar_drain(saddr(&dfull[(committed - 1) % kSSDBufs]), (uint32_t)((committed - 1) / kSSDBufs) & 1u,
                      A.wait_cycles);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

template <int NP, int KIND>
const void* ss_kernel() {
    return reinterpret_cast<const void*>(&k_gemm_ss<NP, KIND>);
}

const void* pick_kernel(int kind) { return kind ? ss_kernel<kSSNP, 1>() : ss_kernel<kSSNP, 0>(); }

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn ss_encoder() {
    static EncodeFn fn = []() -> EncodeFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeFn>(p);
    }();
    return fn;
}

int ss_sms() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 0;
        sms[dev] = v;
    }
    return sms[dev];
}

}  // namespace

// batch rows per unit (the MMA's N)
int gemm_ss_np(int64_t) { return kSSNP; }

// bytes of the published partial sums' flags (control: zero between calls)
// and of the sums themselves (data), for a grid of at most 256 CTAs
SSSpace gemm_ss_space(int64_t M, int64_t N, int64_t K) {
    const int np = gemm_ss_np(M);
    const uint64_t T = (uint64_t)((N + kSSRows - 1) / kSSRows), MB = (uint64_t)((M + np - 1) / np);
    const uint64_t Q = T * MB * (uint64_t)(K / kGroup);
    const uint64_t ctas = std::min<uint64_t>(kSSMaxCtas, Q);
    SSSpace sp;
    sp.control = (size_t)((4 * ctas + 255) / 256 * 256);
    sp.data = (size_t)((ctas * kSSRows * (uint64_t)np * 4 + 255) / 256 * 256);
    return sp;
}

cudaError_t launch_gemm_ss(const void* packed, int grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                           void* Y, int ydt, int64_t ldy, int64_t M, int64_t N, int64_t K, void* ws,
                           size_t ws_bytes, long long wait_cycles, cudaStream_t st) {
    EncodeFn enc = ss_encoder();
    const int sms = ss_sms();
    if (!enc || sms <= 0) return cudaErrorInitializationError;
    const int np = gemm_ss_np(M), kind = grid == kInt3 ? 1 : 0;
    SSArgs A;
    std::memset(&A, 0, sizeof(A));
    {  // X: boxes of 64 k x NP batch rows, 128-byte swizzle (the MMA's B layout); rows past M read as zero
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)(ldx * 2)};
        const cuuint32_t box[2] = {64, (cuuint32_t)std::min<int64_t>(np, M)};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&A.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const uint64_t T = (uint64_t)((N + kSSRows - 1) / kSSRows), MB = (uint64_t)((M + np - 1) / np);
    const uint64_t G = (uint64_t)(K / kGroup);
    A.packed = static_cast<const uint8_t*>(packed);
    A.rb = row_bytes(grid, K);
    A.scales = scales;
    A.Y = Y;
    // flags at the front of the workspace, the sums at its back
    const SSSpace sp = gemm_ss_space(M, N, K);
    A.pflag = static_cast<uint32_t*>(ws);
    A.pdata = reinterpret_cast<float*>(static_cast<char*>(ws) + (ws_bytes & ~size_t(255)) - sp.data);
    A.N = N;
    A.ldy = ldy;
    A.Q = T * MB * G;
    A.wait_cycles = wait_cycles;
    A.M = (int32_t)M;
    A.G = (int32_t)G;
    A.MB = (int32_t)MB;
    A.ydt = ydt;
    A.xrows = (int32_t)std::min<int64_t>(np, M);
    const uint64_t ctas = std::min<uint64_t>(std::min<uint64_t>((uint64_t)sms, kSSMaxCtas), A.Q);
    A.ctas = (int32_t)ctas;
    const void* fn = pick_kernel(kind);
    const int smem = ss_smem_bytes(np);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    void* args[] = {&A};
    return cudaLaunchKernel(fn, dim3((unsigned)ctas), dim3(kSSThreads), args, (size_t)smem, st);
}

unsigned int take_ss_timeouts() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_ss_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyToSymbol(g_ss_timeouts, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

}  // namespace tb
