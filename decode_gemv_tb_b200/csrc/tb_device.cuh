// tb_device.cuh -- device-side pieces shared by the sm_100a kernels:
// grid constants, the packed layout, bf16 helpers and launch descriptors.
//
// Format (declared in include/tb.h): w = c * s, one bf16 scale per 128
// weights along K, per-layer grid ternary / 2-bit / 3-bit (ThinkBit page
// "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로 검증한다",
// onedev.kr/papers/1416, section 어떻게 동작하나).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tb {

constexpr int kGroup = 128;      // weights per scale
constexpr int kMaxItems = 16;    // grouped-launch capacity

enum Grid : int { kTernary = 0, kInt2 = 1, kInt3 = 2 };
enum DType : int { kF32 = 0, kBF16 = 1 };

__host__ __device__ inline int grid_qmin(int g) { return g == kTernary ? -1 : (g == kInt2 ? -2 : -4); }
__host__ __device__ inline int grid_qmax(int g) { return g == kInt3 ? 3 : 1; }
__host__ __device__ inline int grid_offset(int g) { return g == kInt3 ? 4 : 2; }
// bytes of one packed row of K weights
__host__ __device__ inline int64_t row_bytes(int g, int64_t K) { return g == kInt3 ? 3 * K / 8 : K / 4; }

// ---- one small-batch product inside a launch (tb_linear.cu) -----------------
struct Item {
    const uint8_t* packed;
    const uint16_t* scales;
    const uint16_t* X;   // [M][ldx] bf16 activations
    void* Y;             // [M][ldy] outputs
    int64_t N, K, ldx, ldy;
    int32_t grid, ydt, M;
    int32_t cta_begin;   // first CTA of this item in the launch
    int32_t ksplit;      // warps sharing one 32-row tile (1, 2, 4 or 8)
};

struct Launch {
    Item it[kMaxItems];
    int32_t n_items;
    int32_t scl_stride;  // scales staged per row per warp (>= groups per warp)
};

// ---- batch-1 launch on the integer tensor path (see tb_gemv8.cu) ----------
// The activation record of one 128-group, built once per call by the first
// CTA that needs it and copied into the stage of every chunk that needs it:
// the group's activations as eight signed 7-bit digit columns in the order
// the MMA B fragments are read (1024 bytes), then per digit pair t = 0..3
// the accumulator start values of digit columns 2t, 2t+1 and the float
// 2^(14 t - F) (64 bytes).
constexpr int kG8RecBytes = 1088;
constexpr int kG8TileRows = 256;  // rows of a tile

struct G8Item {
    const uint16_t* x;       // [K] bf16 activations
    const uint16_t* scales;  // [N][G] bf16
    void* Y;
    int64_t N;
    int64_t chunk_base, cost_base;  // ChunkItem fields (tb_partition.h)
    int32_t T, G, C, cpt, unit_cost;
    int32_t grid, ydt, tile_base;
    int32_t stage_scales;  // 1: the producer warp copies the scales (rows not 16-byte multiples); 0: a tensor copy
    int32_t owner;         // index of the activation-record set this item reads
};

// One set of activation records: those of one x at one code width (items
// reading the same x with the same width share it), built once per call by
// the record kernel into the workspace.
struct G8Owner {
    const uint16_t* x;  // [G * 128] bf16
    uint8_t* rec;       // [G] records of kG8RecBytes, 256-byte aligned
    int32_t G, three;
    int32_t build_base;  // index of its first record in the call's build order
};

// A CTA's range of chunks [cb, ce) and the (item, tile, chunk in tile) of cb.
struct G8Range {
    uint32_t cb, ce;
    int32_t item, tile, j;
};
constexpr int kMaxG8Ranges = 512;

struct G8Launch {
    CUtensorMap wmap[kMaxItems];  // packed weights: bytes x rows, box (C groups) x 256 rows
    CUtensorMap smap[kMaxItems];  // scales [N][G] bf16: box 8 groups x 256 rows (stage_scales == 0)
    G8Item it[kMaxItems];
    G8Owner own[kMaxItems];
    int32_t n_items, nctas, n_own, n_build;
    uint32_t Ctot, Q;      // total cost and cost quota per CTA (tb_partition.h)
    G8Range range[kMaxG8Ranges];  // per CTA, from the partition
    // [nctas][256] partial sums of split tiles as (fp32 bits, flag 1) words,
    // written by the CTA that reads the tile's end, cleared by the one that
    // reads its start: zero before the call, zero after it
    uint64_t* pslots;
    int32_t stall;         // test hook: the weights are never copied, every wait gives up
    long long wait_cycles; // bound of every wait
    // gated MLP input: items pair_first (gate) and pair_first + 1 (up) of equal
    // shape; once both results of a row are final, h = bf16(silu(gate) * up)
    // (-1: no pair)
    int32_t pair_first;
    uint64_t* pair_slots;  // [N] gate results as (fp32 bits, flag 1): zero before the call, zero after it
    uint16_t* h;           // [N] bf16
};

// ---- cache-controlled loads ----------------------------------------------
// Streamed weights: read once, keep them out of L1.
__device__ __forceinline__ uint2 ld_stream_u2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
// Activations: small, re-read by every CTA: cache in L1.
__device__ __forceinline__ uint4 ld_act_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float2 ld_act_f2(const void* p) {
    float2 v;
    asm volatile("ld.global.nc.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

// Programmatic dependent launch (sm_90+): wait for the grids this one
// depends on / let the dependent grid start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// bf16x2 a*b+c, one rounding (exact whenever the true result is a bf16)
__device__ __forceinline__ uint32_t hfma2_bf16(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// (a & b) | c  in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// bitwise select: (a & ~m) | (b & m); LOP3 table 0xCA is "x ? y : z"
__device__ __forceinline__ uint32_t bit_mux(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(b), "r"(a));
    return d;
}

// ---- exact signed decode to bf16 (the products with M >= 2) -----------------
// A stored code u (2 or 3 bits) at mantissa bit p <= 4 of each 16-bit half,
// OR'ed with the exponent field of 2^(7-p), is the bf16 value 2^(7-p) + u;
// one bf16x2 subtraction of 2^(7-p) + offset then leaves c = u - offset
// exactly (both operands lie in [2^(7-p), 2^(8-p)), the difference is a
// small integer).  So the tensor cores see the signed codeword itself: a
// zero codeword contributes exactly nothing.
__host__ __device__ constexpr uint32_t dec_exp(int p) { return ((uint32_t)(134 - p) << 7) * 0x00010001u; }
__host__ __device__ constexpr uint32_t dec_bias(int p, int off) { return dec_exp(p) | ((uint32_t)(off << p) * 0x00010001u); }

__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// the pair of fields of w selected by mask (at bit p), as exact signed bf16
template <int P, int OFF>
__device__ __forceinline__ uint32_t dec_pair(uint32_t w, uint32_t mask) {
    return sub_bf16x2(and_or(w, mask, dec_exp(P)), dec_bias(P, OFF));
}

// 2-bit word (codes 2m at bits 2m, 2m+1 at bits 16+2m): r[m] = the codes
// 2m, 2m+1 as a bf16 pair (natural order).  Fields 0-2 in place, 3-5 after
// >> 6, 6-7 after >> 12 (each lands at bit 0, 2 or 4).
template <int OFF>
__device__ __forceinline__ void decode2_signed(uint32_t w, uint32_t (&r)[8]) {
    const uint32_t w6 = w >> 6, w12 = w >> 12;
    r[0] = dec_pair<0, OFF>(w, 0x00030003u);
    r[1] = dec_pair<2, OFF>(w, 0x000C000Cu);
    r[2] = dec_pair<4, OFF>(w, 0x00300030u);
    r[3] = dec_pair<0, OFF>(w6, 0x00030003u);
    r[4] = dec_pair<2, OFF>(w6, 0x000C000Cu);
    r[5] = dec_pair<4, OFF>(w6, 0x00300030u);
    r[6] = dec_pair<0, OFF>(w12, 0x00030003u);
    r[7] = dec_pair<2, OFF>(w12, 0x000C000Cu);
}

// masks with a bit at first + 3i + shift (i < count) in both halves
__host__ __device__ constexpr uint32_t bits3_at(int first, int count, int shift) {
    uint32_t m = 0;
    for (int i = 0; i < count; ++i) m |= (1u << (first + 3 * i + shift)) | (1u << (16 + first + 3 * i + shift));
    return m;
}

// 3-bit block (bit f of plane p is bit p of code 2f, bit 16+f of code
// 2f+1): r[f] = the codes 2f, 2f+1 as a bf16 pair (natural order).  The
// planes are merged into 3-bit fields at bit f (planes 1 and 2 shifted up
// by 1 and 2), in three sets of every third field; shifts bring each field
// to bit p <= 4; fields 14 and 15 are assembled from the planes realigned
// to the right.
__device__ __forceinline__ void decode3_signed(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t (&r)[16]) {
    const uint32_t q1 = p1 << 1, q2 = p2 << 2;
    const uint32_t zA = bit_mux(bit_mux(p0, q1, bits3_at(0, 5, 1)), q2, bits3_at(0, 5, 2));  // fields 0,3,6,9,12
    const uint32_t zB = bit_mux(bit_mux(p0, q1, bits3_at(1, 5, 1)), q2, bits3_at(1, 5, 2));  // fields 1,4,7,10,13
    const uint32_t zC = bit_mux(bit_mux(p0, q1, bits3_at(2, 4, 1)), q2, bits3_at(2, 4, 2));  // fields 2,5,8,11
    const uint32_t a6 = zA >> 6, a12 = zA >> 12, b6 = zB >> 6, b12 = zB >> 12;
    const uint32_t c3 = zC >> 3, c6 = zC >> 6, c9 = zC >> 9;
    r[0] = dec_pair<0, 4>(zA, 0x00070007u);
    r[3] = dec_pair<3, 4>(zA, 0x00380038u);
    r[6] = dec_pair<0, 4>(a6, 0x00070007u);
    r[9] = dec_pair<3, 4>(a6, 0x00380038u);
    r[12] = dec_pair<0, 4>(a12, 0x00070007u);
    r[1] = dec_pair<1, 4>(zB, 0x000E000Eu);
    r[4] = dec_pair<4, 4>(zB, 0x00700070u);
    r[7] = dec_pair<1, 4>(b6, 0x000E000Eu);
    r[10] = dec_pair<4, 4>(b6, 0x00700070u);
    r[13] = dec_pair<1, 4>(b12, 0x000E000Eu);
    r[2] = dec_pair<2, 4>(zC, 0x001C001Cu);
    r[5] = dec_pair<2, 4>(c3, 0x001C001Cu);
    r[8] = dec_pair<2, 4>(c6, 0x001C001Cu);
    r[11] = dec_pair<2, 4>(c9, 0x001C001Cu);
    const uint32_t s0 = p0 >> 14, s1 = p1 >> 13, s2 = p2 >> 12;  // plane p of fields 14, 15 at bits p, p + 1
    r[14] = dec_pair<0, 4>(bit_mux(bit_mux(s0, s1, 0x00020002u), s2, 0x00040004u), 0x00070007u);
    r[15] = dec_pair<1, 4>(bit_mux(bit_mux(s0, s1, 0x00040004u), s2, 0x00080008u), 0x000E000Eu);
}

}  // namespace tb
