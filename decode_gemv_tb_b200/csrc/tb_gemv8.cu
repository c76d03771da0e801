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
//     operand's eight columns (the preparation kernel below);
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
// Data flow.  One CTA per SM: a producer warp and eight consumer warps.  The
// work of a call is the sequence of chunks (item, tile of 256 rows, C
// consecutive groups: C = 4 for the 2-bit container, 2 for 3 bits) in item,
// tile, group order; each CTA owns a contiguous range of equal cost
// (tb_partition.h).  The producer streams each chunk into a ring of stages
// with three copies completing on the stage's mbarrier: a 2-D tensor copy of
// the packed weights (256 rows x 128 or 96 bytes; no multicast), a 2-D
// tensor copy of the scales (256 rows x 8 groups) and a bulk copy of the
// chunk's activation records, which every consumer warp shares.  Consumer
// warp w decodes rows 32w .. 32w+31 with LOP3 masks, runs eight MMAs per
// group and accumulates in fp32.  A tile whose groups are split between
// CTAs is combined by the last CTA to finish its part (per warp rows,
// arrival counter), in CTA order: results are bitwise deterministic.
// Every wait is bounded; a wait that gives up is counted, the warp stops
// waiting and writes NaN for the rest of its range.
#include "tb_device.cuh"
#include "tb_internal.h"
#include "tb_partition.h"

#include <algorithm>

namespace tb {

__device__ unsigned int g_g8_timeouts = 0;  // bounded waits of this file's kernels that gave up

namespace {

constexpr int kCWarps = 8;                         // consumer warps
constexpr int kG8Threads = (kCWarps + 1) * 32;     // + the producer warp
constexpr int kStages = 4;
constexpr int kSOff = 32768;                       // scales box: 256 rows x 8 bf16
constexpr int kROff = kSOff + 4096;                // records: up to 4 x 1088 bytes
constexpr int kStageBytes = 41984;                 // >= kROff + 4 * kG8RecBytes, a multiple of 1 KB
constexpr int kG8Smem = kStages * kStageBytes + 1024;  // + alignment slack (swizzled boxes: 1 KB)
constexpr int kPrepThreads = 256;

static_assert(kROff + 4 * kG8RecBytes <= kStageBytes, "stage layout");

// ---- small PTX helpers ------------------------------------------------------
__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// true once the phase with this parity has completed; false after `limit` cycles
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
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
// 1-D bulk copy global -> shared (no multicast)
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
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

// ---- preparation: one warp per (item, group) -----------------------------------
// Record of group g (kG8RecBytes):
//   bytes [512 h + 16 L + 8 (kk & 1) + 4 hf + b], h = kk >> 1, lane L = 4 j + t:
//     digit j of the activation in MMA kk, slot 16 hf + 4 t + b;
//   bytes 1024 + 16 t: int32 -offset * O_{2t}, -offset * O_{2t+1}, float 2^(14 t - F), 0,
//     O_j = sum over the group's slots of 2^cls * digit j.
// F = min(55 - E, 149), E the exponent of the group's largest |x| (a zero or
// subnormal group counts as 2^-126), so every X = trunc(|x| 2^(F - cls)) is
// below 2^56 and every scale factor 2^(14 t - F) is a float.
__global__ void __launch_bounds__(kPrepThreads) k_prep8(const __grid_constant__ G8Launch L) {
    pdl_trigger();  // the main kernel may start streaming weights now
    pdl_wait();     // x may come from the previous kernel, which may also still read the workspace
    const int tid = blockIdx.x * kPrepThreads + threadIdx.x, nthr = gridDim.x * kPrepThreads;
    for (int i = tid; i < L.n_counters; i += nthr) L.counters[i] = 0;  // arrival counters
    if (L.pair_first >= 0)
        for (int i = tid; i < L.it[L.pair_first].T * kCWarps; i += nthr) L.pair_counters[i] = 0;
    for (int ii = 0; ii < L.n_items; ++ii) {  // scale rows padded to a multiple of 8 groups (tensor-copy stride)
        const G8Item& I = L.it[ii];
        if (!I.spad) continue;
        const int64_t n = I.N * I.Gp;
        for (int64_t e = tid; e < n; e += nthr) {
            const int64_t row = e / I.Gp, col = e - row * I.Gp;
            I.spad[e] = col < I.G ? I.scales[row * I.G + col] : (uint16_t)0;
        }
    }
    const int wi = tid >> 5, lane = threadIdx.x & 31;
    if (wi >= L.prep_warps) return;
    int pi = 0;
    for (int i = 1; i < L.n_prep; ++i)
        if (wi >= L.prep[i].begin) pi = i;
    const G8Prep& P = L.prep[pi];
    const int64_t grp = wi - P.begin;
    const uint16_t* xg = P.x + grp * kGroup;
    uint8_t* rec = P.rec + grp * kG8RecBytes;

    const uint2 raw = *reinterpret_cast<const uint2*>(xg + 4 * lane);
    int e = max(max((int)((raw.x >> 7) & 0xFFu), (int)((raw.x >> 23) & 0xFFu)),
                max((int)((raw.y >> 7) & 0xFFu), (int)((raw.y >> 23) & 0xFFu)));
#pragma unroll
    for (int o = 16; o; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
    const int E = max(e, 1) - 127;
    const int F = min(55 - E, 149);

    const bool three = P.three != 0;
    const int gq = lane >> 2, tq = lane & 3;
    const int kk = gq >> 1, hf = gq & 1, r = 2 * kk + hf;
    const int cls = slot_class(three, r);
    uint32_t dig[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int osum[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t h = xg[32 * tq + slot_code(three, r, b)];
        const int eb = (int)((h >> 7) & 0xFFu);
        const uint64_t m = (h & 0x7Fu) | (eb ? 0x80u : 0u);  // |x| = m 2^(max(eb,1) - 134)
        const int sh = max(eb, 1) - 134 + F - cls;           // <= 48 - cls
        const uint64_t X = sh >= 0 ? (m << sh) : (-sh >= 64 ? 0ull : (m >> -sh));
        const bool neg = (h >> 15) != 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int d0 = (int)((X >> (7 * j)) & 127u), d = neg ? -d0 : d0;
            dig[j] |= (uint32_t)(d & 0xFF) << (8 * b);
            osum[j] += d;
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        *reinterpret_cast<uint32_t*>(rec + (kk >> 1) * 512 + (4 * j + tq) * 16 + (kk & 1) * 8 + hf * 4) = dig[j];
        int o = osum[j] * (1 << cls);  // |o| <= 4 * 127 * 2^6 per lane, the group total below 2^21
#pragma unroll
        for (int s = 16; s; s >>= 1) o += __shfl_xor_sync(0xffffffffu, o, s);
        osum[j] = o;
    }
    if (lane < 4) {
        const int off = three ? 4 : 2, t = lane, v = 14 * t - F;  // v in [-149, 114]
        const uint32_t ebits = v >= -126 ? (uint32_t)(v + 127) << 23 : 1u << (v + 149);
        *reinterpret_cast<uint4*>(rec + 1024 + 16 * t) =
            make_uint4((uint32_t)(-off * osum[2 * t]), (uint32_t)(-off * osum[2 * t + 1]), ebits, 0u);
    }
}

// ---- main kernel ------------------------------------------------------------------
// Row of the 256-row tile that MMA row (tile rt, half h: rows g / g+8) of
// lane group g in warp w reads: eight consecutive rows of a quarter differ in
// (row & 7) >> 1 within each half warp, which keeps the 128-byte-swizzled
// weight loads free of bank conflicts.
__device__ __forceinline__ int tile_row(int w, int rt, int h, int g) { return 32 * w + 8 * (2 * rt + h) + 2 * (g & 3) + (g >> 2); }

// Byte offsets of a consumer lane's data inside a stage, fixed for the
// whole kernel: its four rows i = 2 rt + h of the warp's 32.
struct LaneOff {
    uint32_t w2[4][4];  // 2-bit weights of row i, group gi (128-byte swizzle applied)
    uint32_t w3[4];     // 3-bit weights of row i, group 0 (group gi: + 48 gi)
    uint32_t sc[4];     // scales of row i, column 0
};

__device__ __forceinline__ LaneOff lane_offsets(int w, int g, int t) {
    LaneOff o;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = tile_row(w, i >> 1, i & 1, g);
#pragma unroll
        for (int gi = 0; gi < 4; ++gi)
            o.w2[i][gi] = (uint32_t)(r * 128 + (((2 * gi + (t >> 1)) ^ (r & 7)) << 4) + 8 * (t & 1));
        o.w3[i] = (uint32_t)(r * 96 + 12 * t);
        o.sc[i] = (uint32_t)(kSOff + r * 16);
    }
    return o;
}

// One chunk of C groups (geff of them present) for the lane's four rows.
template <int KIND>
__device__ __forceinline__ void g8_chunk(const uint8_t* stage, const LaneOff& o, int geff, int scol, int lane, int t,
                                         float (&acc)[4]) {
    constexpr int C = KIND ? 2 : 4;
    // the chunk's scales of the lane's rows: C consecutive bf16 of the staged 8 (aligned to C)
    uint32_t sv[4][C / 2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (C == 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(stage + o.sc[i] + 2 * scol);
            sv[i][0] = v.x;
            sv[i][C / 2 - 1] = v.y;
        } else {
            sv[i][0] = *reinterpret_cast<const uint32_t*>(stage + o.sc[i] + 2 * scol);
        }
    }
#pragma unroll
    for (int gi = 0; gi < C; ++gi) {
        if (gi >= geff) break;  // only the ragged end of a row has fewer groups
        const uint8_t* rec = stage + kROff + gi * kG8RecBytes;
        const uint4 B0 = *reinterpret_cast<const uint4*>(rec + 16 * lane);
        const uint4 B1 = *reinterpret_cast<const uint4*>(rec + 512 + 16 * lane);
        const uint4 H = *reinterpret_cast<const uint4*>(rec + 1024 + 16 * t);
        const float et = __uint_as_float(H.z);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            uint32_t R[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = 2 * rt + h;
                if (KIND == 0) {
                    const uint2 v = *reinterpret_cast<const uint2*>(stage + o.w2[i][gi]);
                    decode2(v.x, v.y, R[h]);
                } else {
                    const uint32_t* p = reinterpret_cast<const uint32_t*>(stage + o.w3[i] + 48 * gi);
                    decode3(p[0], p[1], p[2], R[h]);
                }
            }
            int d[4] = {(int)H.x, (int)H.y, (int)H.x, (int)H.y};
            mma_u8s8(d, R[0][0], R[1][0], R[0][1], R[1][1], B0.x, B0.y);
            mma_u8s8(d, R[0][2], R[1][2], R[0][3], R[1][3], B0.z, B0.w);
            mma_u8s8(d, R[0][4], R[1][4], R[0][5], R[1][5], B1.x, B1.y);
            mma_u8s8(d, R[0][6], R[1][6], R[0][7], R[1][7], B1.z, B1.w);
            // digit columns 2t, 2t+1 joined (|value| < 2^30), converted once
            const float p0 = (float)(d[0] + 128 * d[1]), p1 = (float)(d[2] + 128 * d[3]);
            const uint32_t w0 = sv[2 * rt][gi >> 1], w1 = sv[2 * rt + 1][gi >> 1];
            const float s0 = __uint_as_float((gi & 1) ? (w0 & 0xFFFF0000u) : (w0 << 16));
            const float s1 = __uint_as_float((gi & 1) ? (w1 & 0xFFFF0000u) : (w1 << 16));
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

// The gated MLP input for a warp's 32 rows of a tile of the gate/up pair:
// each of the two items, once its final values are written, publishes them
// in fp32; the second to arrive computes h = bf16(silu(gate) * up).
__device__ __forceinline__ void pair_epilogue(const G8Launch& L, int item, uint32_t tile, int w, int64_t row, float v) {
    const int which = item - L.pair_first;  // 0: gate, 1: up
    if (L.pair_first < 0 || which < 0 || which > 1) return;
    const int64_t N = L.it[item].N;
    const int lane = threadIdx.x & 31;
    if (row < N) __stcg(L.pair_vals + which * N + row, v);
    __threadfence();
    __syncwarp();
    int second = 0;
    if (lane == 0) second = atomicAdd(L.pair_counters + (int64_t)tile * kCWarps + w, 1) == 1;
    second = __shfl_sync(0xffffffffu, second, 0);
    if (!second) return;
    __threadfence();
    if (row < N) {
        const float other = __ldcg(L.pair_vals + (1 - which) * N + row);
        const float g = which == 0 ? v : other, u = which == 0 ? other : v;
        L.h[row] = __bfloat16_as_ushort(__float2bfloat16_rn(g / (1.f + expf(-g)) * u));
    }
}

// End of a warp's segment of a tile (its 32 rows): write y, or hand the
// partial sums over and combine them if this CTA arrives last.  The
// contributors are the owners of the tile's first and last chunk starts;
// every CTA between them owns at least one (the quota is at least one
// chunk's cost).
__device__ __noinline__ void g8_flush(const G8Launch& L, int cta, int w, int item, uint32_t tile, bool whole,
                                      bool first_seg, float a0, float a1, float a2, float a3) {
    const G8Item& I = L.it[item];
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float v[4] = {a0, a1, a2, a3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // the quad's digit pairs; the same sum in all four lanes
        v[i] += __shfl_xor_sync(0xffffffffu, v[i], 1);
        v[i] += __shfl_xor_sync(0xffffffffu, v[i], 2);
    }
    const float mine = t == 0 ? v[0] : (t == 1 ? v[1] : (t == 2 ? v[2] : v[3]));
    const int rin = tile_row(w, t >> 1, t & 1, g);  // 32 lanes, 32 distinct rows
    const int64_t row0 = (int64_t)tile * kG8TileRows;
    if (whole) {
        store_y(I, row0 + rin, mine);
        pair_epilogue(L, item, tile, w, row0 + rin, mine);
        return;
    }
    __stcg(L.partials + ((int64_t)cta * 2 + (first_seg ? 0 : 1)) * kG8TileRows + rin, mine);
    __threadfence();
    __syncwarp();
    const uint32_t uc = (uint32_t)I.unit_cost;
    const uint32_t pA = (uint32_t)I.cost_base + tile * (uint32_t)I.G * uc;
    const uint32_t pZ = pA + (uint32_t)(I.cpt - 1) * (uint32_t)I.C * uc;
    const uint32_t c0 = part_owner(pA, L.Q), c1 = part_owner(pZ, L.Q);
    int last = 0;
    if (lane == 0) last = atomicAdd(L.counters + ((int64_t)I.tile_base + tile) * kCWarps + w, 1) == (int)(c1 - c0);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    const uint32_t cA = (uint32_t)I.chunk_base + tile * (uint32_t)I.cpt;
    float sum = 0.f;
    for (uint32_t c = c0; c <= c1; ++c) {
        // a CTA that starts inside this tile has it as its first segment (slot 0), an earlier one as its last
        const uint32_t cb = part_first_chunk(L.it, L.n_items, c * L.Q);
        sum += __ldcg(L.partials + ((int64_t)c * 2 + (cb >= cA ? 0 : 1)) * kG8TileRows + 32 * w + lane);
    }
    store_y(I, row0 + 32 * w + lane, sum);
    pair_epilogue(L, item, tile, w, row0 + 32 * w + lane, sum);
}

__global__ void __launch_bounds__(kG8Threads, 1) k_gemv8(const __grid_constant__ G8Launch L) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const uint32_t raw = saddr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // stages on 1 KB boundaries
    const uint32_t base_s = saddr(base);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(saddr(&full[s]), 1);
            bar_init(saddr(&empty[s]), kCWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();  // the only CTA-wide barrier

    uint32_t cb, ce;
    part_chunk_range(L.it, L.n_items, (uint32_t)cta, L.Q, L.Ctot, &cb, &ce);
    const int32_t n = cb < ce ? (int32_t)(ce - cb) : 0;

    // cursor over the chunks of [cb, ce)
    struct Cur {
        int item;
        uint32_t tile;
        int32_t j;
    };
    auto first_cur = [&]() {
        Cur c{0, 0, 0};
        for (int i = 1; i < L.n_items; ++i)
            if (cb >= (uint32_t)L.it[i].chunk_base) c.item = i;
        const uint32_t local = cb - (uint32_t)L.it[c.item].chunk_base, cpt = (uint32_t)L.it[c.item].cpt;
        c.tile = local / cpt;
        c.j = (int32_t)(local - c.tile * cpt);
        return c;
    };
    auto advance = [&](Cur& c) {
        if (++c.j == L.it[c.item].cpt) {
            c.j = 0;
            if (++c.tile == (uint32_t)L.it[c.item].T) {
                c.tile = 0;
                ++c.item;
            }
        }
    };

    if (warp == kCWarps) {
        // ---------------- producer: one thread ----------------
        if (lane != 0 || n == 0 || L.stall) return;
        auto geff_of = [&](const Cur& c) { return min(L.it[c.item].C, L.it[c.item].G - c.j * L.it[c.item].C); };
        // The weights, and the caller's scales, are not written by earlier
        // work in flight, so they may be requested before the preparation
        // kernel is waited for; its records and padded scale copies after.
        auto issue_w = [&](const Cur& c, int k) {  // the stage's byte count, weights (+ caller's scales)
            const G8Item& I = L.it[c.item];
            const int s = k % kStages;
            const uint32_t st = base_s + s * kStageBytes, bar = saddr(&full[s]);
            const int wb = I.grid == kInt3 ? 96 : 128;
            const int geff = geff_of(c);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            bar_expect(bar, (uint32_t)(kG8TileRows * wb + kG8TileRows * 16 + geff * kG8RecBytes));
            tma_box(st, &L.wmap[c.item], c.j * wb, (int)(c.tile * kG8TileRows), bar);
            if (!I.spad) tma_box(st + kSOff, &L.smap[c.item], (c.j * I.C) & ~7, (int)(c.tile * kG8TileRows), bar);
        };
        auto issue_r = [&](const Cur& c, int k) {  // the chunk's activation records (+ padded scales)
            const G8Item& I = L.it[c.item];
            const int s = k % kStages;
            const uint32_t st = base_s + s * kStageBytes, bar = saddr(&full[s]);
            if (I.spad) tma_box(st + kSOff, &L.smap[c.item], (c.j * I.C) & ~7, (int)(c.tile * kG8TileRows), bar);
            bulk_copy(st + kROff, I.rec + (int64_t)c.j * I.C * kG8RecBytes, (uint32_t)(geff_of(c) * kG8RecBytes), bar);
        };
        const int npre = min(n, kStages);
        Cur c = first_cur();
        for (int k = 0; k < npre; ++k, advance(c)) issue_w(c, k);
        pdl_wait();  // records written and counters cleared by the preparation kernel past this point
        Cur r = first_cur();
        for (int k = 0; k < npre; ++k, advance(r)) issue_r(r, k);
        for (int k = npre; k < n; ++k, advance(c)) {
            const int s = k % kStages;
            if (!bar_wait(saddr(&empty[s]), (uint32_t)((k / kStages) - 1) & 1u, L.wait_cycles)) {
                atomicAdd(&g_g8_timeouts, 1u);
                // let the copies already issued land (bounded) before the CTA can exit
                for (int q = max(0, k - kStages); q < k; ++q)
                    bar_wait(saddr(&full[q % kStages]), (uint32_t)(q / kStages) & 1u, L.wait_cycles);
                return;
            }
            issue_w(c, k);
            issue_r(c, k);
        }
        return;
    }

    // ---------------- consumers: warp w owns rows 32w .. 32w+31 of every tile ----------------
    pdl_wait();  // arrival counters cleared past this point
    const int w = warp, g = lane >> 2, t = lane & 3;
    if (n == 0) return;
    const LaneOff off = lane_offsets(w, g, t);
    Cur c = first_cur();
    // the fields of the item under the cursor, in registers (re-read when it changes)
    int it_C = L.it[c.item].C, it_G = L.it[c.item].G, it_cpt = L.it[c.item].cpt, it_T = L.it[c.item].T;
    bool it_three = L.it[c.item].grid == kInt3;
    int32_t seg_j = c.j;
    bool first_seg = true, failed = false;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int32_t k = 0; k < n; ++k) {
        const int s = k % kStages;
        if (!failed) {
            if (!__all_sync(0xffffffffu, bar_wait(saddr(&full[s]), (uint32_t)(k / kStages) & 1u, L.wait_cycles))) {
                if (lane == 0) atomicAdd(&g_g8_timeouts, 1u);
                failed = true;  // no result: the rest of the range is written as NaN, the ring is left alone
            }
        }
        if (!failed) {
            const uint8_t* stage = base + s * kStageBytes;
            const int geff = min(it_C, it_G - c.j * it_C);
            const int scol = (c.j * it_C) & 7;
            if (it_three) g8_chunk<1>(stage, off, geff, scol, lane, t, acc);
            else g8_chunk<0>(stage, off, geff, scol, lane, t, acc);
            __syncwarp();
            if (lane == 0) bar_arrive(saddr(&empty[s]));
        } else {
            acc[0] = acc[1] = acc[2] = acc[3] = __int_as_float(0x7FC00000);
        }
        const int32_t cj_next = c.j + 1;
        const bool more = k + 1 < n;
        if (cj_next == it_cpt || !more) {
            g8_flush(L, cta, w, c.item, c.tile, seg_j == 0 && cj_next == it_cpt, first_seg, acc[0], acc[1], acc[2],
                     acc[3]);
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            first_seg = false;
            seg_j = 0;
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
        if (cudaFuncSetAttribute((const void*)k_gemv8, cudaFuncAttributeMaxDynamicSharedMemorySize, kG8Smem) !=
            cudaSuccess)
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

// Scales [N][Gp] bf16 (Gp a multiple of 8): box 8 groups x 256 rows.
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

int gemv8_ctas() {
    static int ctas[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (ctas[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (!prepare_device(dev)) return 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv8, kG8Threads, kG8Smem) != cudaSuccess ||
            per_sm < 1)
            return 0;
        ctas[dev] = sms * per_sm;
    }
    return ctas[dev];
}

cudaError_t launch_gemv8(const G8Launch& L, bool overlap, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!prepare_device(dev)) return cudaErrorInvalidDevice;
    {
        void* args[] = {const_cast<G8Launch*>(&L)};
        const int warps_per_cta = kPrepThreads / 32;
        const unsigned grid = (unsigned)std::max((L.prep_warps + warps_per_cta - 1) / warps_per_cta, 1);
        e = launch_with_pdl((const void*)k_prep8, args, grid, kPrepThreads, 0, st, overlap);
        if (e != cudaSuccess) return e;
    }
    void* args[] = {const_cast<G8Launch*>(&L)};
    return launch_with_pdl((const void*)k_gemv8, args, (unsigned)L.nctas, kG8Threads, kG8Smem, st, true);
}

unsigned int take_g8_timeouts() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_g8_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyToSymbol(g_g8_timeouts, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

}  // namespace tb
