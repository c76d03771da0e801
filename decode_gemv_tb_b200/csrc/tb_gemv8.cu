// tb_gemv8.cu -- batch-1 y = W x straight from the packed 2- and 3-bit
// codewords, on the integer tensor path (mma.sync m16n8k32, u8 x s8 -> s32).
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416): section 어떻게 동작하나 -- w = c * s with
// an integer codeword c on the layer's grid and one bf16 scale per 128
// weights; section 무엇인가 -- decoding a token reads every weight once, so
// this product is bound by memory bandwidth; section 전제와 한계 -- no kernel
// read the 2- and 3-bit codewords directly.
//
// Arithmetic.  Per output row n and 128-group g the kernel forms the group
// dot product  sum_k c[n][k] x[k]  EXACTLY, in integers, and scales it once:
//   * the stored code u = c + offset goes into the MMA as an unsigned byte
//     without conversion: one LOP3 mask yields four codes (the four bytes of
//     a register), each at its own bit position, i.e. multiplied by a power
//     of two 2^cls (its "class");
//   * the activations of the group become fixed-point integers
//     X_k = trunc(|x_k| 2^(F - cls_k)) (F from the group's largest |x|, so
//     that X < 2^56) split into eight signed 7-bit digit columns, the B
//     operand's eight columns (built per chunk in shared memory, below);
//   * the MMA sums u * 2^cls * digit exactly in int32, and starting its
//     accumulator at -offset * sum_k 2^cls_k digit_k subtracts the offset
//     exactly, so a zero codeword contributes exactly nothing however large
//     its activation is;
//   * digit columns 2t and 2t+1 (held by lane t of a quad) are joined in
//     int32, converted to float once and scaled by s * 2^(14 t - F).
// The only roundings are that conversion and the fp32 accumulation over
// groups and digit pairs: |error| <= (G + 4) 2^-24 sum_k |x_k c_k s| plus
// the truncation of activations more than 2^42 below their group's largest
// (include/tb.h states the bound).
//
// Data flow.  Two kernels per call, the second a programmatic dependent of
// the first:
//   * k_g8_records: one warp per (record set, group) builds the group's
//     record (1088 bytes: the eight digit columns in MMA fragment order and
//     the offset sums) into the workspace.  Projections that read the same x
//     with the same code width share a record set.  x is requested into L2
//     at once and read once the previous kernel in the stream has finished.
//   * k_gemv8 in one of two layouts, chosen per call by its chunks per
//     SM: one CTA per SM with sixteen consumer warps, a producer warp and
//     four stages (calls of a few chunks per SM), or two CTAs per SM, each
//     eight consumer warps, a producer and two stages (two independent
//     rings per SM; calls of many chunks per SM).
//     The work of a call is the sequence of chunks (item, tile of 256 rows,
//     C consecutive groups: C = 4 for the 2-bit container, 2 for 3 bits) in
//     item, tile, group order; each CTA owns a contiguous range of equal
//     cost (tb_partition.h: a 3-bit group costs twice a 2-bit one, so every
//     chunk costs the same).
//   * Stages.  Each chunk passes through a ring of shared-memory stages
//     per CTA.  The producer copies the packed weights (a 2-D tensor copy of
//     256 rows x 128 or 96 bytes, no multicast) and the scales (256 rows x 8
//     groups) into the stage -- inputs no earlier kernel writes, so both
//     first stages are requested at once, before the record kernel has finished --
//     and, once it has, the chunk's records (one bulk copy).
//   * Consumer warp w decodes the rows of row block w mod R of the tile
//     (R = 8 blocks of 32 rows, or 4 of 64 rows in the two-CTA layout),
//     for half of the chunk's groups (w / R), with LOP3 masks, runs four MMAs
//     per 16 rows and group and accumulates in fp32; the two halves of a row
//     block meet in shared memory at the end of a segment.  (Sixteen
//     consumer warps per SM hide more of the decode's fixed latencies than
//     eight; on long ranges two CTAs with independent rings more than one
//     with sixteen warps, on short ones the deeper ring of one CTA wins.
//     The record kernel's CTAs are one warp, so that waiting ones
//     never keep the next call's main CTAs off their SM.)
// A stage is full when its copies have landed and the producer has
// arrived; empty when all consumers have.  A tile whose groups are
// split between CTAs is combined by the CTA that reads its first chunk --
// for which it is the last segment of its range, so the others have long
// finished theirs: each later CTA publishes its partial sum of the tile's
// rows as (fp32 bits, flag) in one 64-bit store, and the combining CTA adds
// them in CTA order (results are bitwise deterministic) and clears them.
// Every wait is bounded; a wait that gives up is counted, the warp stops
// waiting and writes NaN for the rest of its range.
#include "tb_device.cuh"
#include "tb_internal.h"
#include "tb_partition.h"

#include <algorithm>

namespace tb {

__device__ unsigned int g_g8_timeouts = 0;  // bounded waits of this file's kernels that gave up

namespace {

constexpr int kSOff = 32768;                       // scales box: 256 rows x 8 bf16
constexpr int kROff = kSOff + 4096;                // records copied from the workspace: up to 4 x 1088 bytes
constexpr int kStageBytes = 41984;                 // >= kROff + 4 * kG8RecBytes, a multiple of 1 KB

// The two layouts of k_gemv8, chosen per call by its chunks per SM (host):
//   G8One: one CTA per SM, sixteen consumer warps of 32 rows, four stages
//     (calls with few chunks per SM: deep rings, few split tiles);
//   G8Two: two CTAs per SM, each eight consumer warps of 64 rows and two
//     stages (calls with many chunks per SM: two independent rings).
template <int WR, int NS, int MINB>
struct G8Cfg {
    static constexpr int kRB = WR;                    // rows of a consumer warp's row block
    static constexpr int kNRB = kG8TileRows / WR;     // row blocks of a tile (a warp pair each)
    static constexpr int kRT = WR / 16;               // 16-row MMA tiles of a warp
    static constexpr int kBL = WR / 32;               // 8-row blocks a lane finishes (kBL t .. kBL t + kBL - 1)
    static constexpr int kCWarps = 2 * kNRB;          // consumer warps
    static constexpr int kProducer = kCWarps;         // the producer warp
    static constexpr int kThreads = (kCWarps + 1) * 32;
    static constexpr int kStages = NS;
    static constexpr int kEarly = NS;                 // stages filled before the previous kernel has finished
    static constexpr int kMinBlocks = MINB;           // CTAs per SM
    static constexpr int kSmem = NS * kStageBytes + 1024;  // + alignment slack (swizzled boxes: 1 KB)
    static_assert(kSmem * MINB <= 227 * 1024, "shared memory");
};
using G8One = G8Cfg<32, 4, 1>;
using G8Two = G8Cfg<64, 2, 2>;
constexpr int kRecWarps = 1;                       // warps of a CTA of the record kernel (small: see above)

static_assert(kROff + 4 * kG8RecBytes <= kStageBytes, "stage layout");

// ---- small PTX helpers ------------------------------------------------------
__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// raises the transaction count of the current phase (no arrival)
__device__ __forceinline__ void bar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// true once the phase with this parity has completed; false after `limit`
// cycles.  Each try suspends the thread until the phase completes or about
// 20 us pass, so a waiting warp takes no issue slots from the working ones.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity), "r"(20000u)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit) return false;
    }
}
// 2-D tiled tensor copy global -> shared (no multicast): box at (x, y) of map
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// 1-D bulk copy global -> shared (no multicast): bytes a multiple of 16, both addresses 16-byte aligned
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// 64-bit words read and written whole (single-copy atomic)
__device__ __forceinline__ void st_word(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_word(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t flagged(float v) { return (1ull << 32) | __float_as_uint(v); }
// the value of a flagged word once its flag is set; false after `limit` cycles
__device__ __forceinline__ bool wait_word(const uint64_t* p, long long limit, float* v) {
    const long long t0 = clock64();
    for (;;) {
        const uint64_t w = ld_word(p);
        if (w >> 32) {
            *v = __uint_as_float((uint32_t)w);
            return true;
        }
        if (clock64() - t0 > limit) return false;
        __nanosleep(64);
    }
}
// hints: bring bytes of global memory into L2; fetch a tensor map's descriptor
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_map(const void* p) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(p) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// d += A B, A 16 x 32 unsigned bytes (row), B 32 x 8 signed bytes (col), int32 accumulate
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- the code -> MMA slot map ----------------------------------------------
// Lane t of a quad decodes codes 32t .. 32t+31 of a group (two 2-bit words
// or one 3-bit plane triple) of each of its rows into registers R[0..7] of
// four bytes; MMA kk (0..3) takes R[2kk] as a0/a1 (k slots 4t .. 4t+3) and
// R[2kk+1] as a2/a3 (k slots 16+4t .. 16+4t+3).  Byte b of R[r] holds the
// code code_of(r, b) (relative to 32t) multiplied by 2^cls_of(r).
//   2-bit, R[4w+q] = word w & (0x03030303 << 2q): bits 8b + 2q of word w,
//     i.e. codes 16w + {2q, 8+2q, 2q+1, 9+2q}[b], class 2q.
//   3-bit, R[i]: the fields whose plane bits sit at bit i of each byte of
//     the planes, i.e. codes {2i, 16+2i, 2i+1, 17+2i}[b]; the field lands at
//     bits i..i+2 of its byte for i <= 5 (class i), at 4..6 for i = 6
//     (class 4) and at 5..7 for i = 7 (class 5).
__device__ __forceinline__ int slot_code(bool three, int r, int b) {
    if (three) {
        const int base = (b & 1) ? 16 : 0;
        return base + 2 * r + ((b >> 1) & 1);  // b: 0 -> 2r, 1 -> 16+2r, 2 -> 2r+1, 3 -> 17+2r
    }
    const int w = r >> 2, q = r & 3;
    return 16 * w + ((b & 1) ? 8 : 0) + 2 * q + ((b >> 1) & 1);
}
__device__ __forceinline__ int slot_class(bool three, int r) { return three ? (r <= 5 ? r : r - 2) : 2 * (r & 3); }

// 2-bit word pair -> R[8]
__device__ __forceinline__ void decode2(uint32_t w0, uint32_t w1, uint32_t (&R)[8]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        R[q] = w0 & (0x03030303u << (2 * q));
        R[4 + q] = w1 & (0x03030303u << (2 * q));
    }
}
// 3-bit plane triple -> R[8]
__device__ __forceinline__ void decode3(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t (&R)[8]) {
    const uint32_t q1 = p1 << 1, q2 = p2 << 2;  // plane 1 (2) bit i at i + 1 (i + 2), inside the byte for i <= 6 (5)
    const uint32_t z0 = bit_mux(bit_mux(p0, q1, 0x12121212u), q2, 0x24242424u);  // fields at bits 0 and 3
    const uint32_t z1 = bit_mux(bit_mux(p0, q1, 0x24242424u), q2, 0x48484848u);  // fields at bits 1 and 4
    const uint32_t z2 = bit_mux(bit_mux(p0, q1, 0x48484848u), q2, 0x90909090u);  // fields at bits 2 and 5
    R[0] = z0 & 0x07070707u;
    R[3] = z0 & 0x38383838u;
    R[1] = z1 & 0x0E0E0E0Eu;
    R[4] = z1 & 0x70707070u;
    R[2] = z2 & 0x1C1C1C1Cu;
    R[5] = z2 & 0xE0E0E0E0u;
    const uint32_t r0 = p0 >> 2, r1 = p1 >> 1;  // plane bits 6, 7 realigned to stay inside the byte
    R[6] = bit_mux(bit_mux(r0, r1, 0x20202020u), p2, 0x40404040u) & 0x70707070u;  // bit 6 fields at 4..6
    R[7] = bit_mux(bit_mux(r0, r1, 0x40404040u), p2, 0x80808080u) & 0xE0E0E0E0u;  // bit 7 fields at 5..7
}

// ---- activation records ---------------------------------------------------
// Record of a group (kG8RecBytes), built by one warp:
//   bytes [512 h + 16 L + 8 (kk & 1) + 4 hf + b], h = kk >> 1, lane L = 4 j + t:
//     digit j of the activation in MMA kk, slot 16 hf + 4 t + b;
//   bytes 1024 + 16 t: int32 -offset * O_{2t}, -offset * O_{2t+1}, float 2^(14 t - F), 0,
//     O_j = sum over the group's slots of 2^cls * digit j.
// F = min(55 - E, 149), E the exponent of the group's largest |x| (a zero or
// subnormal group counts as 2^-126), so every X = trunc(|x| 2^(F - cls)) is
// below 2^56 and every scale factor 2^(14 t - F) is a float.  The eight
// bits of an activation's mantissa fill at most two consecutive 7-bit
// digits.  The offset sums come from four MMAs of the record's own B
// fragments against A = 2^cls in every byte (a group of codes u = 1).
// `raw` holds x[4 lane .. 4 lane + 3] of the group.
__device__ __noinline__ void make_record(const uint2 raw, bool three, uint8_t* rec) {
    const int lane = threadIdx.x & 31;
    int e = max(max((int)((raw.x >> 7) & 0xFFu), (int)((raw.x >> 23) & 0xFFu)),
                max((int)((raw.y >> 7) & 0xFFu), (int)((raw.y >> 23) & 0xFFu)));
#pragma unroll
    for (int o = 16; o; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
    const int E = max(e, 1) - 127;
    const int F = min(55 - E, 149);
    const int gq = lane >> 2, tq = lane & 3;
    const int kk = gq >> 1, hf = gq & 1, r = 2 * kk + hf;
    const int cls = slot_class(three, r);
    uint32_t lo[4], hi[4];  // digit bytes 0-3 / 4-7 of the lane's four slots
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int code = 32 * tq + slot_code(three, r, b);
        const uint32_t vx = __shfl_sync(0xffffffffu, raw.x, code >> 2), vy = __shfl_sync(0xffffffffu, raw.y, code >> 2);
        const uint32_t v2 = (code & 2) ? vy : vx;
        const uint32_t h = (code & 1) ? (v2 >> 16) : (v2 & 0xFFFFu);
        const int eb = (int)((h >> 7) & 0xFFu);
        uint32_t m = (h & 0x7Fu) | (eb ? 0x80u : 0u);  // |x| = m 2^(max(eb,1) - 134)
        int sh = max(eb, 1) - 134 + F - cls;           // <= 48 - cls
        if (sh < 0) {
            m = -sh >= 8 ? 0u : m >> -sh;  // truncated below 2^0
            sh = 0;
        }
        const int j0 = (sh * 37) >> 8;  // sh / 7 for 0 <= sh <= 48
        const uint32_t v = m << (sh - 7 * j0);           // < 2^14: digits j0 and j0 + 1
        uint64_t mag = (uint64_t)((v & 127u) | ((v >> 7) << 8)) << (8 * j0);
        if (h >> 15) mag = (0x8080808080808080ull - mag) ^ 0x8080808080808080ull;  // bytewise negation
        lo[b] = (uint32_t)mag;
        hi[b] = (uint32_t)(mag >> 32);
    }
    // digit column j of the four slots as one word, stored where lane (j, tq) reads its B fragment
    uint8_t* dst = rec + (kk >> 1) * 512 + tq * 16 + (kk & 1) * 8 + hf * 4;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t* src = j < 4 ? lo : hi;
        const uint32_t sel = (uint32_t)(j & 3) | ((uint32_t)(4 + (j & 3)) << 4);
        const uint32_t p01 = __byte_perm(src[0], src[1], sel), p23 = __byte_perm(src[2], src[3], sel);
        *reinterpret_cast<uint32_t*>(dst + 64 * j) = __byte_perm(p01, p23, 0x5410);
    }
    __syncwarp();
    // offset sums: D[.][j] = sum over slots of 2^cls * digit j
    const uint4 B0 = *reinterpret_cast<const uint4*>(rec + 16 * lane);
    const uint4 B1 = *reinterpret_cast<const uint4*>(rec + 512 + 16 * lane);
    uint32_t A[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) A[q] = 0x01010101u << slot_class(three, q);
    int d[4] = {0, 0, 0, 0};
    mma_u8s8(d, A[0], A[0], A[1], A[1], B0.x, B0.y);
    mma_u8s8(d, A[2], A[2], A[3], A[3], B0.z, B0.w);
    mma_u8s8(d, A[4], A[4], A[5], A[5], B1.x, B1.y);
    mma_u8s8(d, A[6], A[6], A[7], A[7], B1.z, B1.w);
    if (lane < 4) {  // g = 0, t = lane: columns 2t, 2t+1
        const int off = three ? 4 : 2, v = 14 * lane - F;  // v in [-149, 114]
        const uint32_t ebits = v >= -126 ? (uint32_t)(v + 127) << 23 : 1u << (v + 149);
        *reinterpret_cast<uint4*>(rec + 1024 + 16 * lane) =
            make_uint4((uint32_t)(-off * d[0]), (uint32_t)(-off * d[1]), ebits, 0u);
    }
}

// The records of a call: warp b of the grid builds record b of the call's
// build order (set o, group g) in shared memory and writes it to the
// workspace.  x is requested into L2 at once and read once the previous
// kernel in the stream has finished; the main kernel, a programmatic
// dependent of this one, reads the records after this kernel completes.
__global__ void __launch_bounds__(kRecWarps * 32) k_g8_records(const __grid_constant__ G8Launch L) {
    __shared__ __align__(16) uint8_t scratch[kRecWarps][kG8RecBytes];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * kRecWarps + warp;
    if (b >= L.n_build) {
        pdl_wait();
        return;
    }
    int o = 0;
    while (o + 1 < L.n_own && b >= L.own[o + 1].build_base) ++o;
    const G8Owner& O = L.own[o];
    const int g = b - O.build_base;
    const uint16_t* xg = O.x + (int64_t)g * kGroup;
    if (lane == 0) prefetch_l2(xg, kGroup * 2);
    pdl_wait();  // x may come from the previous kernel in the stream
    make_record(__ldcg(reinterpret_cast<const uint2*>(xg) + lane), O.three != 0, scratch[warp]);
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(O.rec + (int64_t)g * kG8RecBytes);
    for (int i = lane; i < kG8RecBytes / 16; i += 32) dst[i] = reinterpret_cast<const uint4*>(scratch[warp])[i];
}

// ---- consumer layout --------------------------------------------------------------
// Consumer warp w works on the kRB rows kRB rb .. kRB rb + kRB - 1 of every
// tile (rb = w mod kNRB) and on half of every chunk's groups (gh = w / kNRB:
// local groups gh C/2 .. gh C/2 + C/2 - 1), so that each record is read by
// half of the warps.  Lane (g, t) takes part in MMA rows g and g + 8 of the
// warp's kRT 16-row MMA tiles rt: 8-row blocks i = 2 rt (rows g) and
// i = 2 rt + 1 (rows g + 8), tile row kRB rb + 8 i + k7 with
// k7 = 2 (g & 3) + (g >> 2).  The eight lane groups of a block differ in
// row & 7 = k7, which keeps the 128-byte-swizzled weight loads free of bank
// conflicts, and block i of a lane is block 0 plus i x 8 rows: a constant
// offset.
__device__ __forceinline__ int lane_k7(int g) { return 2 * (g & 3) + (g >> 2); }

// Byte offsets of block 0 of a consumer lane's rows inside a stage.
struct LaneOff {
    uint32_t w2[2];  // 2-bit: local group 2 gh + q (128-byte swizzle applied), + 8 (t & 1)
    uint32_t w3;     // 3-bit: local group gh, + 12 t
    uint32_t sc;     // scales, column 0
};

template <class Cfg>
__device__ __forceinline__ LaneOff lane_offsets(int rb, int gh, int g, int t) {
    LaneOff o;
    const int k7 = lane_k7(g), r = Cfg::kRB * rb + k7;
#pragma unroll
    for (int q = 0; q < 2; ++q)
        o.w2[q] = (uint32_t)(r * 128 + (((2 * (2 * gh + q) + (t >> 1)) ^ k7) << 4) + 8 * (t & 1));
    o.w3 = (uint32_t)(r * 96 + 48 * gh + 12 * t);
    o.sc = (uint32_t)(kSOff + r * 16);
    return o;
}

// The warp's groups of one chunk (geff groups present; `recs` holds the
// chunk's records in order) for the lane's 2 kRT row blocks.
template <class Cfg, int KIND>
__device__ __forceinline__ void g8_chunk(const uint8_t* stage, const uint8_t* recs, const LaneOff& o, int geff,
                                         int gh, int scol, int lane, int t, float (&acc)[2 * Cfg::kRT]) {
    constexpr int C = KIND ? 2 : 4, CW = C / 2, WROW = KIND ? 96 * 8 : 128 * 8;
    const int gl0 = gh * CW;
    if (gl0 >= geff) return;  // the ragged end of a row: this half has no group
    // the scales of the warp's groups, per row block (2-bit: two bf16 in one word; 3-bit: one, as fp32 bits)
    uint32_t sv[2 * Cfg::kRT];
#pragma unroll
    for (int i = 0; i < 2 * Cfg::kRT; ++i) {
        const uint8_t* p = stage + o.sc + 128 * i + 2 * (scol + gl0);
        sv[i] = KIND ? (uint32_t)*reinterpret_cast<const uint16_t*>(p) << 16 : *reinterpret_cast<const uint32_t*>(p);
    }
#pragma unroll
    for (int q = 0; q < CW; ++q) {
        if (gl0 + q >= geff) break;
        const uint8_t* rec = recs + (gl0 + q) * kG8RecBytes;
        const uint4 B0 = *reinterpret_cast<const uint4*>(rec + 16 * lane);
        const uint4 B1 = *reinterpret_cast<const uint4*>(rec + 512 + 16 * lane);
        const uint4 H = *reinterpret_cast<const uint4*>(rec + 1024 + 16 * t);
        const float et = __uint_as_float(H.z);
        const uint8_t* wb = stage + (KIND ? o.w3 : o.w2[q]);
#pragma unroll
        for (int rt = 0; rt < Cfg::kRT; ++rt) {
            uint32_t R[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint8_t* p = wb + (2 * rt + h) * WROW;
                if (KIND == 0) {
                    const uint2 v = *reinterpret_cast<const uint2*>(p);
                    decode2(v.x, v.y, R[h]);
                } else {
                    const uint32_t* w = reinterpret_cast<const uint32_t*>(p);
                    decode3(w[0], w[1], w[2], R[h]);
                }
            }
            int d[4] = {(int)H.x, (int)H.y, (int)H.x, (int)H.y};
            mma_u8s8(d, R[0][0], R[1][0], R[0][1], R[1][1], B0.x, B0.y);
            mma_u8s8(d, R[0][2], R[1][2], R[0][3], R[1][3], B0.z, B0.w);
            mma_u8s8(d, R[0][4], R[1][4], R[0][5], R[1][5], B1.x, B1.y);
            mma_u8s8(d, R[0][6], R[1][6], R[0][7], R[1][7], B1.z, B1.w);
            // digit columns 2t, 2t+1 joined (|value| < 2^30), converted once
            const float p0 = (float)(d[0] + 128 * d[1]), p1 = (float)(d[2] + 128 * d[3]);
            const uint32_t w0 = sv[2 * rt], w1 = sv[2 * rt + 1];
            const float s0 = __uint_as_float(KIND || q == 0 ? w0 << (KIND ? 0 : 16) : w0 & 0xFFFF0000u);
            const float s1 = __uint_as_float(KIND || q == 0 ? w1 << (KIND ? 0 : 16) : w1 & 0xFFFF0000u);
            acc[2 * rt] = fmaf(s0 * et, p0, acc[2 * rt]);
            acc[2 * rt + 1] = fmaf(s1 * et, p1, acc[2 * rt + 1]);
        }
    }
}

__device__ __forceinline__ void store_y(const G8Item& I, int64_t row, float v) {
    if (row >= I.N) return;
    if (I.ydt == kF32) static_cast<float*>(I.Y)[row] = v;
    else static_cast<__nv_bfloat16*>(I.Y)[row] = __float2bfloat16_rn(v);
}

// The gated MLP input for one row of the gate/up pair: the gate's final
// value is published as a flagged word; the up item's, once final, waits for
// it and writes h = bf16(silu(gate) * up), then clears the word.
__device__ __forceinline__ void pair_epilogue(const G8Launch& L, int item, int64_t row, float v) {
    const int which = item - L.pair_first;  // 0: gate, 1: up
    if (L.pair_first < 0 || which < 0 || which > 1 || row >= L.it[item].N) return;
    uint64_t* slot = L.pair_slots + row;
    if (which == 0) {
        st_word(slot, flagged(v));
        return;
    }
    float g;
    if (!wait_word(slot, L.wait_cycles, &g)) {
        atomicAdd(&g_g8_timeouts, 1u);
        g = __int_as_float(0x7FC00000);
    }
    st_word(slot, 0);
    L.h[row] = __bfloat16_as_ushort(__float2bfloat16_rn(g / (1.f + expf(-g)) * v));
}

// How a range's segment of a tile ends: the whole tile (write y); a later
// part of a tile begun by an earlier range (publish); or the beginning of a
// tile that later ranges finish (combine).
enum SegKind { kWhole = 0, kPublish = 1, kCombine = 2 };

// Rows rin + 8 b (b < kBL) at the end of a segment (sums over this range's
// chunks of the tile): publish them, or add the later ranges' words in CTA
// order (the words of the lane's rows and two ranges in flight at a time),
// then write y.
template <class Cfg>
__device__ __forceinline__ void finish_rows(const G8Launch& L, int cta, int item, uint32_t tile, int kind, int rin,
                                            uint32_t c1, float (&s)[Cfg::kBL]) {
    constexpr int kBL = Cfg::kBL;
    if (kind == kPublish) {
#pragma unroll
        for (int b = 0; b < kBL; ++b) st_word(L.pslots + (int64_t)cta * kG8TileRows + rin + 8 * b, flagged(s[b]));
        return;
    }
    if (kind == kCombine) {  // the later ranges that read this tile, in order
        for (uint32_t c = (uint32_t)cta + 1; c <= c1; c += 2) {
            uint64_t* slot[2 * kBL];
            uint64_t wv[2 * kBL];
#pragma unroll
            for (int q = 0; q < 2 * kBL; ++q) {  // q: range c + q / kBL, row rin + 8 (q % kBL)
                slot[q] = L.pslots + (int64_t)(c + q / kBL) * kG8TileRows + rin + 8 * (q % kBL);
                wv[q] = c + q / kBL <= c1 ? ld_word(slot[q]) : 0;
            }
#pragma unroll
            for (int q = 0; q < 2 * kBL; ++q) {
                if (c + q / kBL > c1) break;
                float p = __uint_as_float((uint32_t)wv[q]);
                if (!(wv[q] >> 32) && !wait_word(slot[q], L.wait_cycles, &p)) {
                    atomicAdd(&g_g8_timeouts, 1u);
                    p = __int_as_float(0x7FC00000);
                }
                st_word(slot[q], 0);
                s[q % kBL] += p;
            }
        }
    }
    const int64_t row = (int64_t)tile * kG8TileRows + rin;
#pragma unroll
    for (int b = 0; b < kBL; ++b) store_y(L.it[item], row + 8 * b, s[b]);
#pragma unroll
    for (int b = 0; b < kBL; ++b) pair_epilogue(L, item, row + 8 * b, s[b]);
}

// End of a warp's segment of a tile: the quad's digit pairs are summed, the
// group half gh = 1 hands its sums to gh = 0 through shared memory (double
// buffered by `flip`), which adds them (gh 0 + gh 1) and finishes the rows.
template <class Cfg>
struct AccT {
    float v[2 * Cfg::kRT];
};

template <class Cfg>
__device__ __noinline__ void g8_flush(const G8Launch& L, int cta, int rb, int gh, int item, uint32_t tile, int kind,
                                      const AccT<Cfg> acc, float* pairbuf, int flip) {
    constexpr int kRT = Cfg::kRT, kBL = Cfg::kBL, kRB = Cfg::kRB;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float v[2 * kRT];
#pragma unroll
    for (int i = 0; i < 2 * kRT; ++i) {  // the same sum in all four lanes of the quad
        v[i] = acc.v[i] + __shfl_xor_sync(0xffffffffu, acc.v[i], 1);
        v[i] += __shfl_xor_sync(0xffffffffu, v[i], 2);
    }
    // lane t keeps blocks kBL t .. kBL t + kBL - 1
    float m[kBL];
#pragma unroll
    for (int b = 0; b < kBL; ++b) m[b] = v[b];
#pragma unroll
    for (int q = 1; q < 4; ++q)
        if (t == q) {
#pragma unroll
            for (int b = 0; b < kBL; ++b) m[b] = v[kBL * q + b];
        }
    float* pb = pairbuf + flip * kG8TileRows + rb * kRB + kBL * lane;
    if (gh == 1) {
#pragma unroll
        for (int b = 0; b < kBL; ++b) pb[b] = m[b];
    }
    named_sync(2 + rb, 64);
    if (gh == 1) return;
#pragma unroll
    for (int b = 0; b < kBL; ++b) m[b] += pb[b];
    const G8Item& I = L.it[item];
    uint32_t c1 = 0;
    if (kind == kCombine) {
        const uint32_t uc = (uint32_t)I.unit_cost;
        c1 = part_owner((uint32_t)I.cost_base + tile * (uint32_t)I.G * uc + (uint32_t)(I.cpt - 1) * (uint32_t)I.C * uc,
                        L.Q);
    }
    const int rin = kRB * rb + 8 * kBL * t + lane_k7(g);  // block kBL t; the next ones 8 rows on each
    finish_rows<Cfg>(L, cta, item, tile, kind, rin, c1, m);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, Cfg::kMinBlocks) k_gemv8(const __grid_constant__ G8Launch L) {
    constexpr int kStages = Cfg::kStages, kEarly = Cfg::kEarly, kCWarps = Cfg::kCWarps, kProducer = Cfg::kProducer;
    constexpr int kNRB = Cfg::kNRB, kRT = Cfg::kRT;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    __shared__ int producer_failed;  // set before the producer completes stages it could not fill
    __shared__ float pairbuf[2 * kG8TileRows];  // row sums handed between the two halves of a row block
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const uint32_t raw = saddr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // stages on 1 KB boundaries
    const uint32_t base_s = saddr(base);
    const uint32_t cb = L.range[cta].cb, ce = L.range[cta].ce;
    const int32_t n = cb < ce ? (int32_t)(ce - cb) : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(saddr(&full[s]), 1);  // the producer's arrival (after its byte counts)
            bar_init(saddr(&empty[s]), kCWarps);
        }
        producer_failed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();  // the only CTA-wide barrier

    // cursor over the chunks of [cb, ce)
    struct Cur {
        int item;
        uint32_t tile;
        int32_t j;
    };
    auto first_cur = [&]() { return Cur{L.range[cta].item, (uint32_t)L.range[cta].tile, L.range[cta].j}; };
    auto advance = [&](Cur& c) {
        if (++c.j == L.it[c.item].cpt) {
            c.j = 0;
            if (++c.tile == (uint32_t)L.it[c.item].T) {
                c.tile = 0;
                ++c.item;
            }
        }
    };

    if (warp == kProducer) {
        // ---------------- producer warp ----------------
        const bool active = n > 0 && !L.stall;
        auto weights = [&](const Cur& c, int s) {  // lane 0: the chunk's weights (and scales) into stage s
            const G8Item& I = L.it[c.item];
            const uint32_t st = base_s + s * kStageBytes, bar = saddr(&full[s]);
            const int wb = I.grid == kInt3 ? 96 : 128;
            bar_expect(bar, (uint32_t)(kG8TileRows * wb + (I.stage_scales ? 0 : kG8TileRows * 16)));
            tma_box(st, &L.wmap[c.item], c.j * wb, (int)(c.tile * kG8TileRows), bar);
            if (!I.stage_scales) tma_box(st + kSOff, &L.smap[c.item], (c.j * I.C) & ~7, (int)(c.tile * kG8TileRows), bar);
        };
        // The weights and scales are inputs no earlier kernel in the stream
        // writes: the first kEarly stages are requested at once, before the
        // previous kernel has finished (when the call may overlap it), the
        // rest of the ring and the records (workspace) once the record kernel
        // has completed.
        Cur pf = first_cur();  // next chunk whose weights are requested
        int pf_k = 0;
        if (active && lane == 0) {
            for (int i = 0; i < L.n_items; ++i) {
                prefetch_map(&L.wmap[i]);
                if (!L.it[i].stage_scales) prefetch_map(&L.smap[i]);
            }
            for (; pf_k < n && pf_k < kEarly; ++pf_k, advance(pf)) weights(pf, pf_k);
        }
        pdl_wait();  // the records: written by the record kernel, the previous one in the stream
        // they were written through the generic proxy; the bulk copies read them through the async one
        asm volatile("fence.proxy.async.global;" ::: "memory");
        if (active && lane == 0)
            for (; pf_k < n && pf_k < kStages; ++pf_k, advance(pf)) weights(pf, pf_k);
        int issued = 0;
        bool ok = active;
        if (active) {
            Cur c = first_cur();
            for (int k = 0; k < n; ++k, advance(c)) {
                const int s = k % kStages;
                const G8Item& I = L.it[c.item];
                int go = 1;
                if (lane == 0) {
                    if (k >= kStages) {
                        go = bar_wait(saddr(&empty[s]), (uint32_t)((k / kStages) - 1) & 1u, L.wait_cycles);
                        if (go) weights(c, s);
                    }
                    if (go) {
                        const G8Owner& O = L.own[I.owner];
                        const int geff = min(I.C, I.G - c.j * I.C);
                        const uint32_t bar = saddr(&full[s]);
                        bar_expect(bar, (uint32_t)(geff * kG8RecBytes));
                        bulk_copy(base_s + s * kStageBytes + kROff, O.rec + (int64_t)c.j * I.C * kG8RecBytes,
                                  (uint32_t)(geff * kG8RecBytes), bar);
                    }
                }
                if (!__shfl_sync(0xffffffffu, go, 0)) {
                    if (lane == 0) atomicAdd(&g_g8_timeouts, 1u);
                    ok = false;
                    break;
                }
                if (I.stage_scales) {  // rows of the scales that a tensor copy cannot address: plain loads
                    uint16_t* sc = reinterpret_cast<uint16_t*>(base + s * kStageBytes + kSOff);
                    const int geff = min(I.C, I.G - c.j * I.C), scol = (c.j * I.C) & 7;
                    for (int rr = lane; rr < kG8TileRows; rr += 32) {
                        const int64_t row = (int64_t)c.tile * kG8TileRows + rr;
                        for (int gi = 0; gi < geff; ++gi)
                            sc[rr * 8 + scol + gi] =
                                row < I.N ? __ldg(I.scales + row * I.G + c.j * I.C + gi) : (uint16_t)0;
                    }
                    // a later tensor copy may overwrite what these generic stores wrote
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (lane == 0) bar_arrive(saddr(&full[s]));
                issued = k + 1;
            }
        }
        if (lane == 0) {
            // the copies requested (stages beyond `issued` may hold weights only) land before the CTA can exit
            const int req = active ? max(issued, min(n, kStages)) : 0;
            if (!ok) {  // complete the phases of the stages requested but not filled, marked as failed
                producer_failed = 1;
                for (int q = issued; q < req; ++q) bar_arrive(saddr(&full[q % kStages]));
            }
            for (int q = max(0, req - kStages); q < req; ++q)
                bar_wait(saddr(&full[q % kStages]), (uint32_t)(q / kStages) & 1u, L.wait_cycles);
        }
        return;
    }

    // ---------------- consumers: rows 64 rb .. 64 rb + 63 of every tile, half the groups ----------------
    pdl_wait();  // y and the workspace may still be in use by the previous kernels in the stream
    const int w = warp, g = lane >> 2, t = lane & 3;
    if (n == 0) return;
    const int rb = w % kNRB, gh = w / kNRB;
    const LaneOff off = lane_offsets<Cfg>(rb, gh, g, t);
    Cur c = first_cur();
    // the fields of the item under the cursor, in registers (re-read when it changes)
    int it_C = L.it[c.item].C, it_G = L.it[c.item].G, it_cpt = L.it[c.item].cpt, it_T = L.it[c.item].T;
    bool it_three = L.it[c.item].grid == kInt3;
    bool failed = false;
    int flip = 0;
    float acc[2 * kRT];
#pragma unroll
    for (int i = 0; i < 2 * kRT; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int32_t k = 0; k < n; ++k) {
        const int s = k % kStages;
        if (!failed) {  // one lane waits for the stage; the warp synchronizes with it
            int ok = 1;
            if (lane == 0) {
                ok = bar_wait(saddr(&full[s]), (uint32_t)(k / kStages) & 1u, L.wait_cycles);
                if (!ok) atomicAdd(&g_g8_timeouts, 1u);
                ok = ok && *reinterpret_cast<volatile int*>(&producer_failed) == 0;
            }
            // no result after a failed wait: the rest of the range is written as NaN, the ring is left alone
            failed = __shfl_sync(0xffffffffu, ok, 0) == 0;
        }
        if (!failed) {
            const uint8_t* stage = base + s * kStageBytes;
            const int geff = min(it_C, it_G - c.j * it_C);
            const int scol = (c.j * it_C) & 7;
            const uint8_t* recs = stage + kROff;
            if (it_three) g8_chunk<Cfg, 1>(stage, recs, off, geff, gh, scol, lane, t, acc);
            else g8_chunk<Cfg, 0>(stage, recs, off, geff, gh, scol, lane, t, acc);
            __syncwarp();
            if (lane == 0) bar_arrive(saddr(&empty[s]));
        } else {
#pragma unroll
            for (int i = 0; i < 2 * kRT; ++i) acc[i] = __int_as_float(0x7FC00000);
        }
        const bool more = k + 1 < n;
        if (c.j + 1 == it_cpt || !more) {  // end of the range's segment of this tile
            const uint32_t first = (uint32_t)L.it[c.item].chunk_base + c.tile * (uint32_t)it_cpt;
            const int kind = first < cb ? kPublish : (first + (uint32_t)it_cpt > ce ? kCombine : kWhole);
            AccT<Cfg> a8;
#pragma unroll
            for (int i = 0; i < 2 * kRT; ++i) a8.v[i] = acc[i];
            g8_flush<Cfg>(L, cta, rb, gh, c.item, c.tile, kind, a8, pairbuf, flip);
            flip ^= 1;
#pragma unroll
            for (int i = 0; i < 2 * kRT; ++i) acc[i] = 0.f;
        }
        // advance the cursor (the item's fields are reloaded only when it changes)
        if (++c.j == it_cpt) {
            c.j = 0;
            if (++c.tile == (uint32_t)it_T && more) {
                c.tile = 0;
                ++c.item;
                it_C = L.it[c.item].C;
                it_G = L.it[c.item].G;
                it_cpt = L.it[c.item].cpt;
                it_T = L.it[c.item].T;
                it_three = L.it[c.item].grid == kInt3;
            }
        }
    }
}

cudaError_t launch_with_pdl(const void* fn, void** args, unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                            bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, looked up once through the runtime
EncodeFn encoder() {
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

bool prepare_device(int dev) {
    static bool ready[64] = {false};
    if (dev < 0 || dev >= 64) return false;
    if (!ready[dev]) {
        if (cudaFuncSetAttribute((const void*)k_gemv8<G8One>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 G8One::kSmem) != cudaSuccess ||
            cudaFuncSetAttribute((const void*)k_gemv8<G8Two>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 G8Two::kSmem) != cudaSuccess)
            return false;
        ready[dev] = true;
    }
    return true;
}

}  // namespace

int g8_chunk_groups(int grid) { return grid == kInt3 ? 2 : 4; }

// Packed weights of one matrix: bytes x rows, box of one chunk (128 bytes =
// four 2-bit groups, 128-byte swizzled; 96 bytes = two 3-bit groups) x 256
// rows; rows past N read as zero.
bool encode_g8_wmap(CUtensorMap* map, const void* packed, int grid, int64_t N, int64_t K) {
    EncodeFn enc = encoder();
    if (!enc) return false;
    const bool three = grid == kInt3;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes(grid, K), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes(grid, K)};
    const cuuint32_t box[2] = {three ? 96u : 128u, (cuuint32_t)kG8TileRows};
    const cuuint32_t es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(packed), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, three ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scales [N][G] bf16 (G a multiple of 8, 16-byte aligned base): box 8
// groups x 256 rows.
bool encode_g8_smap(CUtensorMap* map, const uint16_t* scales, int64_t N, int64_t Gp) {
    EncodeFn enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)Gp, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(Gp * 2)};
    const cuuint32_t box[2] = {8u, (cuuint32_t)kG8TileRows};
    const cuuint32_t es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemv8_ctas(bool two) {
    static int ctas[64][2] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int& c = ctas[dev][two ? 1 : 0];
    if (c == 0) {
        int sms = 0, per_sm = 0;
        if (!prepare_device(dev)) return 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        const cudaError_t e =
            two ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv8<G8Two>, G8Two::kThreads, G8Two::kSmem)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv8<G8One>, G8One::kThreads, G8One::kSmem);
        if (e != cudaSuccess || per_sm < 1) return 0;
        c = sms * per_sm;
    }
    return c;
}

// The record kernel, then the main kernel as its programmatic dependent
// (it streams weights while the records are built).  `overlap` lets the
// record kernel, in turn, start before the previous work in the stream ends.
cudaError_t launch_gemv8(const G8Launch& L, bool two, bool overlap, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!prepare_device(dev)) return cudaErrorInvalidDevice;
    void* args[] = {const_cast<G8Launch*>(&L)};
    const unsigned rec_ctas = (unsigned)((L.n_build + kRecWarps - 1) / kRecWarps);
    e = launch_with_pdl((const void*)k_g8_records, args, rec_ctas, kRecWarps * 32, 0, st, overlap);
    if (e != cudaSuccess) return e;
    if (two)
        return launch_with_pdl((const void*)k_gemv8<G8Two>, args, (unsigned)L.nctas, G8Two::kThreads, G8Two::kSmem,
                               st, true);
    return launch_with_pdl((const void*)k_gemv8<G8One>, args, (unsigned)L.nctas, G8One::kThreads, G8One::kSmem, st,
                           true);
}

unsigned int take_g8_timeouts() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_g8_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyToSymbol(g_g8_timeouts, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

}  // namespace tb
