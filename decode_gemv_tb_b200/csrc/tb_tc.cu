// tb_tc.cu -- small-batch GEMM  Y = X W^T  on the fifth-generation tensor
// cores (tcgen05), straight from the packed 2- and 3-bit codewords.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나: w = c * s with
// one bf16 scale per 128 input weights; the product per output row n, batch
// row m and 128-group g is
//     Y[m][n] += s[n][g] * sum_k c[n][k] X[m][k].
//
// Data flow of one CTA (a 128-row tile of W and a contiguous range of its
// 128-groups; 256 decoder threads, two per weight row, and one producer
// warp):
//   * each decoder streams its half of the row's packed group through a
//     private cp.async ring six groups deep and decodes it to the signed
//     codeword itself, exactly, as bf16 (tb_device.cuh: the stored field
//     OR'ed into the mantissa of 2^(7-p), minus 2^(7-p) + offset); the pairs
//     go to tensor memory (tcgen05.st), one TMEM lane per row, k in natural
//     order along the columns -- the A operand;
//   * the preparation kernel has copied X per group into the K-major
//     core-matrix layout the MMA reads from shared memory (rows M .. NP - 1
//     zero) and transposed the group scales per tile; the producer brings a
//     group's X and the tile's 128 scales in with two bulk copies, two groups
//     ahead -- the B operand;
//   * the producer warp issues the group's eight 128 x NP x 16 MMAs (bf16
//     in, fp32 accumulate in tensor memory; one elected lane of the
//     converged warp, so the operands stay warp-uniform) and commits them to
//     an mbarrier; every product c * x is exact and a zero codeword
//     contributes nothing;
//   * while they run, each decoder reads its half of the previous group's
//     accumulator row back (tcgen05.ld) and applies the group scale:
//         acc[m] += s * D[m]
//     A and D are double-buffered in tensor memory (2 x 64 + 2 x NP
//     columns of the 256 a CTA allocates; two CTAs per SM).
// K-splits of one tile are combined by the last CTA to finish, in split
// order (deterministic).  Every wait is bounded: a wait that gives up
// counts itself in g_wait_timeouts, the CTA stops issuing work, waits
// (bounded) for what it already issued, writes NaN outputs, frees its
// tensor memory and exits.
#include "tb_device.cuh"
#include "tb_internal.h"

#include <algorithm>

namespace tb {

// bounded waits that gave up since the last tb_wait_timeouts() call
__device__ unsigned int g_wait_timeouts = 0;

namespace {

constexpr int kTCRows = 128;      // weight rows per tile (one decoder thread each)
constexpr int kTCStages = 3;      // prepared X groups (with the tile's scales) in shared memory
constexpr uint32_t kTmemCols = 256;
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr int kTCTargetCtas = 296;               // 2 CTAs on each of 148 SMs
constexpr int kTCMaxSplits = 16;
constexpr size_t kTCMinSmem = 80 * 1024;         // at most two CTAs (2 x 256 TMEM columns) per SM

// one prepared group: NP rows x 128 bf16 activations in the K-major
// core-matrix layout (16 chunks of 8 k per 8 rows: 2048 bytes per 8 rows)
__host__ __device__ constexpr int tc_group_bytes(int np) { return np * 256; }
constexpr int kTCBRowGroupB = 16 * 128;  // stride between 8-row core-matrix groups of B

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---- mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
// true once the phase with this parity has completed; false after about
// kWaitCycles (counted in g_wait_timeouts).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > kWaitCycles) {
            atomicAdd(&g_wait_timeouts, 1u);
            return false;
        }
    }
}
// The same for a converged warp: every lane waits (measured faster than one
// waiting lane and a broadcast), the result is warp-uniform.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
}

// 1-D bulk copy global -> shared, completion counted on bar (no multicast)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// ---- tensor memory -----------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16 consecutive columns of this thread's lane, complete on return
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&d)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) d[i] = __uint_as_float(r[i]);
}

// D[tmem d] (+)= A[tmem a] x B[smem desc b], issued by a whole converged
// warp: one elected lane issues, so the operands stay warp-uniform (a single
// divergent thread issuing costs about three times as many cycles per MMA).
__device__ __forceinline__ void mma_ts_warp(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred e, p;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}
// commit by the same elected lane (the lowest active one) that issued the MMAs
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}" ::"r"(smem_addr(bar))
        : "memory");
}

// Shared-memory descriptor of a K-major operand without swizzle: core
// matrices of 8 rows x 16 bytes, the next 8 k (16 bytes) 128 bytes on
// (leading byte offset), the next 8 rows sbo bytes on (stride byte offset).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
           (1ull << 46);
}

// kind::f16 instruction descriptor: fp32 D, bf16 A and B, both K-major, M = 128, N = np
__host__ __device__ constexpr uint32_t idesc_bf16(int np) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(np >> 3) << 17) | ((uint32_t)(kTCRows >> 4) << 24);
}

// ---- decode: a row's half group into 32 bf16 pairs (TMEM columns) ---------
// 2-bit container: word i holds codes 16i .. 16i+15 -> columns 8i .. 8i+7.
__device__ __forceinline__ void decode2_pair(uint32_t w0, uint32_t w1, uint32_t (&r)[16]) {
    uint32_t a[8], b[8];
    decode2_signed<2>(w0, a);
    decode2_signed<2>(w1, b);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        r[m] = a[m];
        r[8 + m] = b[m];
    }
}

}  // namespace

struct TCArgs {
    const uint8_t* packed;
    const uint16_t* scales;
    const uint16_t* X;  // [M][ldx] bf16
    uint8_t* bprep;     // G prepared groups of tc_group_bytes(NP)
    uint16_t* sprep;    // group scales per tile: [tiles][G][128] bf16 (0 past row N)
    void* Y;            // [M][ldy]
    float* partials;    // [tiles][splits][NP][128] when splits > 1
    int32_t* counters;  // [tiles]
    int64_t N, K, ldx, ldy;
    int32_t M, NP, grid, ydt, G, tiles, splits;
};

namespace {

// ---- preparation: one CTA per group g -----------------------------------------
// Rows m < M of X for group g are copied into the K-major core-matrix
// layout the MMA reads (rows M .. NP - 1 zero).  The CTAs also clear the
// tile counters and transpose the group scales per 128-row tile.
__global__ void __launch_bounds__(256) k_prep_tc(const __grid_constant__ TCArgs A) {
    for (int i = blockIdx.x * 256 + threadIdx.x; i < A.tiles; i += gridDim.x * 256) A.counters[i] = 0;
    // scales transposed per 128-row tile, so that one bulk copy brings a tile's 128 scales of a group
    // (element i: tile-group pair i / 128 = t * G + g, row t * 128 + i % 128)
    const int64_t n_sprep = (int64_t)A.tiles * A.G * kTCRows;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n_sprep; i += (int64_t)gridDim.x * 256) {
        const uint32_t tg = (uint32_t)(i >> 7), t = tg / (uint32_t)A.G, g = tg - t * (uint32_t)A.G;
        const int64_t row = (int64_t)t * kTCRows + (i & (kTCRows - 1));
        A.sprep[i] = row < A.N ? A.scales[row * A.G + g] : (uint16_t)0;
    }
    const int g = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (g >= A.G) return;  // uniform over the CTA
    uint8_t* gb = A.bprep + (int64_t)g * tc_group_bytes(A.NP);
    for (int m = warp; m < A.NP; m += 8) {
        uint8_t* rowb = gb + (m >> 3) * kTCBRowGroupB + (m & 7) * 16;  // chunk c of row m at rowb + 128 c
        uint2 v = make_uint2(0u, 0u);
        if (m < A.M) v = *reinterpret_cast<const uint2*>(A.X + (int64_t)m * A.ldx + (int64_t)g * kGroup + 4 * lane);
        // elements k = 4 lane .. 4 lane + 3: chunk lane / 2, bytes 8 (lane % 2)
        *reinterpret_cast<uint2*>(rowb + (lane >> 1) * 128 + 8 * (lane & 1)) = v;
    }
}

// ---- main kernel -------------------------------------------------------------
// 288 threads.  Warps 0-7 are decoders: two threads per weight row, thread
// t on row t % 128 and half h = t / 128 of the row's group (TMEM columns
// 32h .. 32h + 31; warps w and w + 4 share TMEM lanes 32 (w % 4) ..), and
// half h of the batch columns in the epilogue.  Each streams its part of
// the row's packed groups through a private cp.async ring, decodes it into
// the tensor-memory A buffer and runs the scale epilogue of the previous
// group.  Thread 256 (warp 8) is the producer: it brings the prepared X
// and the tile's scales of each group in with bulk copies and issues the
// MMAs.  Hand-offs, each an mbarrier:
//   afull[b]  decoders -> producer: A buffer b holds group i (256 arrivals)
//   mma[b]    producer -> decoders: the MMAs of group i are done (commit)
//   dfree[b]  decoders -> producer: D buffer b of group i has been read and
//             the group's shared-memory stage may be refilled (256 arrivals)
//   full[s]   bulk copies -> producer, decoders: stage s holds group i
// A waiter is never more than one phase behind a barrier, so parity waits
// are unambiguous: every next phase needs an action that comes after the
// wait in the other role's program order.
constexpr int kTCDecoders = 2 * kTCRows;
constexpr int kTCBlock = kTCDecoders + 32;
constexpr int kTCWStages = 6;   // per-thread ring of packed groups
constexpr int kTCWStride = 32;  // ring bytes per decoder thread and stage (two 16-byte chunks)

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* d) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = __uint_as_float(r[i]);
}
// NH consecutive columns (NH = 8, 16, 24 or 32) of this thread's lane
template <int NH>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&d)[NH]) {
    if constexpr (NH == 8) {
        tmem_ld8(taddr, d);
    } else if constexpr (NH == 16) {
        tmem_ld16(taddr, d);
    } else if constexpr (NH == 24) {
        float a[16];
        tmem_ld16(taddr, a);
        tmem_ld8(taddr + 16, d + 16);
#pragma unroll
        for (int i = 0; i < 16; ++i) d[i] = a[i];
    } else {
        float a[16], b[16];
        tmem_ld16(taddr, a);
        tmem_ld16(taddr + 16, b);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            d[i] = a[i];
            d[16 + i] = b[i];
        }
    }
}

// Half H of a row's group from the thread's ring slot into TMEM columns
// 32H .. 32H + 31.  2-bit: the slot holds words 4H .. 4H + 3.  3-bit: it
// holds words 4H .. 4H + 7, of which blocks 2H and 2H + 1 (words 6H ..
// 6H + 5) are this half's.
template <int KIND, int H>
__device__ __forceinline__ void decode_half(const uint4* src, uint32_t acol) {
    if constexpr (KIND == 0) {
        const uint4 c = src[0];
        uint32_t r[16];
        decode2_pair(c.x, c.y, r);
        tmem_st16(acol, r);
        decode2_pair(c.z, c.w, r);
        tmem_st16(acol + 16, r);
    } else {
        const uint4 c0 = src[0], c1 = src[1];
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        constexpr int o = 2 * H;
        uint32_t r[16];
        decode3_signed(w[o], w[o + 1], w[o + 2], r);
        tmem_st16(acol, r);
        decode3_signed(w[o + 3], w[o + 4], w[o + 5], r);
        tmem_st16(acol + 16, r);
    }
}

template <int NP, int KIND>
__global__ void __launch_bounds__(kTCBlock, 2) k_gemm_tc(const __grid_constant__ TCArgs A) {
    constexpr int GB = tc_group_bytes(NP);  // prepared X of one group (a multiple of 16 bytes)
    constexpr int SB = GB + 256;      // + the tile's 128 scales of that group
    constexpr int WQ = KIND ? 3 : 2;  // 16-byte packed chunks per row and group
    constexpr int WH = KIND ? 2 : 1;  // chunks one half-row thread loads (chunks h .. h + WH - 1)
    constexpr int NH = NP / 2;        // batch columns per half
    constexpr uint32_t kIdesc = idesc_bf16(NP);
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* const wring = smem + kTCStages * SB;  // [kTCWStages][256][kTCWStride]
    __shared__ __align__(8) uint64_t bar_full[kTCStages];
    __shared__ __align__(8) uint64_t bar_afull[2], bar_dfree[2], bar_mma[2];
    __shared__ uint32_t tmem_sh;
    __shared__ int last_sh;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = tid & (kTCRows - 1), h = (tid >> 7) & 1;  // decoders: row in tile, half
    const int tile = blockIdx.x / A.splits, split = blockIdx.x - tile * A.splits;
    const int g0 = (int)((int64_t)split * A.G / A.splits);
    const int ng = (int)((int64_t)(split + 1) * A.G / A.splits) - g0;
    const int64_t row = (int64_t)tile * kTCRows + r;
    const bool row_ok = tid < kTCDecoders && row < A.N;

    if (tid == 0) {
        for (int s = 0; s < kTCStages; ++s) mbar_init(&bar_full[s], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_afull[b], kTCDecoders);
            mbar_init(&bar_dfree[b], kTCDecoders);
            mbar_init(&bar_mma[b], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_sh)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;

    float acc[NH];
#pragma unroll
    for (int m = 0; m < NH; ++m) acc[m] = 0.f;
    bool fail = false;   // a bounded wait of this thread gave up
    int issued = 0;      // producer: groups whose bulk copies are issued
    int committed = 0;   // producer: groups whose MMAs are committed

    if (warp == kTCDecoders / 32) {
        // ---------------- producer (one converged warp) ----------------
        const int lane = tid & 31;
        auto issue = [&](int i) {
            if (lane == 0) {
                const int s = i % kTCStages;
                uint8_t* st = smem + s * SB;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect_tx(&bar_full[s], SB);
                bulk_g2s(st, A.bprep + (int64_t)(g0 + i) * GB, GB, &bar_full[s]);
                bulk_g2s(st + GB, A.sprep + ((int64_t)tile * A.G + g0 + i) * kTCRows, 256, &bar_full[s]);
            }
            __syncwarp();
        };
        for (; issued < min(kTCStages - 1, ng); ++issued) issue(issued);
        for (int i = 0; i < ng; ++i) {
            const int b = i & 1, s = i % kTCStages;
            // D buffer b was released (dfree of group i - 2) in the previous iteration
            if (!mbar_wait_warp(&bar_afull[b], (uint32_t)(i >> 1) & 1u)) { fail = true; break; }
            if (!mbar_wait_warp(&bar_full[s], (uint32_t)(i / kTCStages) & 1u)) { fail = true; break; }
            tc_fence_after();
            const uint64_t bdesc = kmajor_desc(smem_addr(smem + s * SB), kTCBRowGroupB);
            const uint32_t dcol = tmem + 128u + (uint32_t)(b * NP), acol = tmem + (uint32_t)(b * 64);
#pragma unroll
            for (int j = 0; j < 8; ++j)  // K slice j: 8 TMEM columns of A, 256 bytes (16 descriptor units) of B
                mma_ts_warp(dcol, acol + 8u * j, bdesc + 16u * j, kIdesc, j > 0 ? 1u : 0u);
            mma_commit_warp(&bar_mma[b]);
            committed = i + 1;
            // the next stage to fill, (i + kTCStages - 1) % kTCStages, last held group i - 1
            if (i >= 1 && !mbar_wait_warp(&bar_dfree[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u)) {
                fail = true;
                break;
            }
            if (issued < ng) issue(issued++);
        }
    } else if (tid < kTCDecoders) {
        // ---------------- decoders ----------------
        const int64_t rbytes = KIND ? 3 * A.K / 8 : A.K / 4;
        const uint8_t* rowp = A.packed + (row_ok ? row : 0) * rbytes + (int64_t)g0 * (16 * WQ) + 16 * h;
        const uint32_t wbase = smem_addr(wring) + (uint32_t)(tid * kTCWStride);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // this warp's 32 TMEM lanes
        auto load = [&](int i) {  // one commit group per call, empty past the end
            if (i < ng) {
                const uint32_t dst = wbase + (uint32_t)((i % kTCWStages) * kTCDecoders * kTCWStride);
#pragma unroll
                for (int q = 0; q < WH; ++q)
                    cp_async16_zfill(dst + 16 * q, rowp + (int64_t)i * (16 * WQ) + 16 * q, row_ok ? 16u : 0u);
            }
            cp_commit();
        };
#pragma unroll
        for (int j = 0; j < kTCWStages - 1; ++j) load(j);
        for (int i = 0; i <= ng; ++i) {
            const int b = i & 1;
            if (i < ng) {
                load(i + kTCWStages - 1);
                cp_wait<kTCWStages - 1>();  // this thread's copies of group i have landed
                const uint4* src = reinterpret_cast<const uint4*>(wring + (i % kTCWStages) * kTCDecoders * kTCWStride +
                                                                  tid * kTCWStride);
                // A buffer b: the MMAs of group i - 2 that read it finished before
                // this thread's epilogue of group i - 2 (previous iteration)
                const uint32_t acol = tmem + lane_base + (uint32_t)(b * 64 + 32 * h);
                if (h == 0) decode_half<KIND, 0>(src, acol);
                else decode_half<KIND, 1>(src, acol);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar_afull[b]);
            }
            if (i >= 1) {  // epilogue of group i - 1 (warp-uniform: tcgen05.ld is a warp instruction)
                const int bp = (i - 1) & 1, sp = (i - 1) % kTCStages;
                bool ok = mbar_wait_warp(&bar_mma[bp], (uint32_t)((i - 1) >> 1) & 1u);
                if (ok) ok = mbar_wait_warp(&bar_full[sp], (uint32_t)((i - 1) / kTCStages) & 1u);
                if (!ok) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                const uint8_t* st = smem + sp * SB;
                // D = sum c x: one factor, the group scale s, per row and group
                const float f = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(st + GB + 2 * r));
                float d[NH];
                tmem_ld_cols<NH>(tmem + lane_base + 128u + (uint32_t)(bp * NP + h * NH), d);
#pragma unroll
                for (int q = 0; q < NH; ++q) acc[q] = fmaf(f, d[q], acc[q]);
                // D buffer read and the stage's scale and exponent consumed
                tc_fence_before();
                mbar_arrive(&bar_dfree[bp]);
            }
        }
        cp_wait<0>();
    }

    const bool aborted = __syncthreads_or(fail ? 1 : 0) != 0;
    if (aborted && tid == kTCDecoders) {
        // wait (bounded) for what is still in flight: the newest copy of each
        // stage (older ones completed before their stage was refilled) and the
        // newest MMA commit (commits complete in order)
        for (int i = max(0, issued - kTCStages); i < issued; ++i)
            mbar_wait(&bar_full[i % kTCStages], (uint32_t)(i / kTCStages) & 1u);
        if (committed > 0) mbar_wait(&bar_mma[(committed - 1) & 1], (uint32_t)((committed - 1) >> 1) & 1u);
    }
    if (aborted) {
#pragma unroll
        for (int m = 0; m < NH; ++m) acc[m] = __int_as_float(0x7FC00000);
    }

    // ---- output: decoder (r, h) holds batch columns h NH .. h NH + NH - 1 of its row ----
    auto store = [&](int m, float v) {
        if (A.ydt == kF32)
            static_cast<float*>(A.Y)[(int64_t)m * A.ldy + row] = v;
        else
            static_cast<__nv_bfloat16*>(A.Y)[(int64_t)m * A.ldy + row] = __float2bfloat16_rn(v);
    };
    const int m0 = h * NH;
    if (A.splits == 1) {
        if (row_ok) {
#pragma unroll
            for (int j = 0; j < NH; ++j)
                if (m0 + j < A.M) store(m0 + j, acc[j]);
        }
    } else {
        if (tid < kTCDecoders) {
            float* slot = A.partials + ((int64_t)(tile * A.splits + split) * NP) * kTCRows;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                if (m0 + j < A.M) __stcg(slot + (m0 + j) * kTCRows + r, acc[j]);
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) last_sh = atomicAdd(A.counters + tile, 1) == A.splits - 1;
        __syncthreads();
        if (last_sh && row_ok) {
            __threadfence();
            const float* base = A.partials + (int64_t)tile * A.splits * NP * kTCRows;
            for (int j = 0; j < NH; ++j) {
                const int m = m0 + j;
                if (m >= A.M) break;
                float v = 0.f;
                for (int s = 0; s < A.splits; ++s) v += __ldcg(base + ((int64_t)s * NP + m) * kTCRows + r);
                store(m, v);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

int tc_np(int M) { return (M + 15) / 16 * 16; }

int tc_splits(int64_t N, int64_t K) {
    const int64_t tiles = (N + kTCRows - 1) / kTCRows, G = K / kGroup;
    int64_t s = (kTCTargetCtas + tiles / 2) / tiles;  // nearest to one wave of kTCTargetCtas
    s = std::min<int64_t>(std::min<int64_t>(s, kTCMaxSplits), G);
    return (int)std::max<int64_t>(s, 1);
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t tc_smem_bytes(int np) {
    return std::max(kTCMinSmem, (size_t)kTCStages * (tc_group_bytes(np) + 256) +
                                    (size_t)kTCWStages * kTCDecoders * kTCWStride + 1024);
}

template <int NP, int KIND>
cudaError_t launch_tc_main(const TCArgs& A, cudaStream_t st) {
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const size_t smem = tc_smem_bytes(NP);
    if (!ready[dev]) {
        e = cudaFuncSetAttribute((const void*)k_gemm_tc<NP, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        ready[dev] = true;
    }
    k_gemm_tc<NP, KIND><<<A.tiles * A.splits, kTCBlock, smem, st>>>(A);
    return cudaGetLastError();
}

template <int KIND>
cudaError_t launch_tc_np(const TCArgs& A, cudaStream_t st) {
    switch (A.NP) {
        case 16: return launch_tc_main<16, KIND>(A, st);
        case 32: return launch_tc_main<32, KIND>(A, st);
        case 48: return launch_tc_main<48, KIND>(A, st);
        default: return launch_tc_main<64, KIND>(A, st);
    }
}

}  // namespace

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    const int np = tc_np((int)M);
    const int64_t tiles = (N + kTCRows - 1) / kTCRows, G = K / kGroup;
    const int splits = tc_splits(N, K);
    size_t b = align256((size_t)G * tc_group_bytes(np)) + align256((size_t)tiles * G * kTCRows * 2) +
               align256((size_t)tiles * 4);
    if (splits > 1) b += align256((size_t)tiles * splits * np * kTCRows * 4);
    return b;
}

cudaError_t launch_gemm_tc(const void* packed, int grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                           void* Y, int ydt, int64_t ldy, int M, int64_t N, int64_t K, void* ws, cudaStream_t st) {
    TCArgs A;
    A.packed = static_cast<const uint8_t*>(packed);
    A.scales = scales;
    A.X = X;
    A.Y = Y;
    A.N = N;
    A.K = K;
    A.ldx = ldx;
    A.ldy = ldy;
    A.M = M;
    A.NP = tc_np(M);
    A.grid = grid;
    A.ydt = ydt;
    A.G = (int32_t)(K / kGroup);
    A.tiles = (int32_t)((N + kTCRows - 1) / kTCRows);
    A.splits = tc_splits(N, K);
    char* w = static_cast<char*>(ws);
    A.bprep = reinterpret_cast<uint8_t*>(w);
    w += align256((size_t)A.G * tc_group_bytes(A.NP));
    A.sprep = reinterpret_cast<uint16_t*>(w);
    w += align256((size_t)A.tiles * A.G * kTCRows * 2);
    A.counters = reinterpret_cast<int32_t*>(w);
    w += align256((size_t)A.tiles * 4);
    A.partials = A.splits > 1 ? reinterpret_cast<float*>(w) : nullptr;
    // one CTA per group at least, and about 8 transposed scales per thread
    const int64_t n_sprep = (int64_t)A.tiles * A.G * kTCRows;
    const int prep_ctas = (int)std::max<int64_t>(
        std::max<int64_t>(A.G, (A.tiles + 255) / 256), std::min<int64_t>((n_sprep + 2047) / 2048, 1184));
    k_prep_tc<<<prep_ctas, 256, 0, st>>>(A);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return grid == kInt3 ? launch_tc_np<1>(A, st) : launch_tc_np<0>(A, st);
}

unsigned int take_wait_timeouts() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_wait_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyToSymbol(g_wait_timeouts, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

}  // namespace tb
