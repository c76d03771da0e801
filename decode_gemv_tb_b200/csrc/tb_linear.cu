// tb_linear.cu -- y = W x (and Y = X W^T for M <= 16) straight from the
// packed 2- and 3-bit codewords.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416): section 무엇인가 -- every decoded token
// reads every weight, so decode is bound by memory bandwidth; section
// 어떻게 동작하나 -- w = c * s, one bf16 scale per 128 weights, dequant is
// one multiply; section 전제와 한계 -- no kernel read the 2/3-bit codes
// directly, so checkpoints ship in 4-bit containers.
//
// Design (sm_100a):
//  * One CTA (8 warps) owns a 16-row tile of one matrix; its warps split K
//    by 128-groups (group g goes to warp g mod 8) and reduce through shared
//    memory in a fixed order: deterministic, no global scratch, no atomics.
//    The hardware block scheduler balances tiles of different cost; tiles
//    of the most expensive matrices come first in blockIdx order.
//  * Weights stream with 64-bit (2-bit container) or 32-bit (3-bit planes)
//    L1-bypassing loads, PF groups ahead per warp, so every lane keeps
//    several loads in flight.
//  * Codes are decoded to exact bf16 integers with one LOP3 (mask the
//    field, OR the exponent of 128.0) and one bf16x2 FMA (rescale the
//    field position and subtract 128 + offset) per PAIR of codes.  The
//    multiply-accumulate runs on the tensor pipe (mma.sync m16n8k16,
//    fp32 accumulate), which keeps the FP32 and integer pipes free for the
//    decode: at 2.125 bits/weight the SM issue budget is about 1.5
//    instructions per weight, less than a CUDA-core decode + FMA costs.
//  * Each 128-group is accumulated on its own (fp32, tensor pipe) and
//    multiplied by its scale once; groups are summed in fp32.
//
// Fragment mapping (m16n8k16, lane = 4 g + t): A rows are W rows
// tile*16 + g and + 8.  A k-slot pairs (2t, 2t+1) and (2t+8, 2t+9) carry
// one decoded code PAIR each; because the packed word keeps codes 2m and
// 2m+1 in the same field of the two half-words, every pair is two
// ADJACENT k, so the B fragment of one MMA is four consecutive x values:
// x is read in its natural layout, no shuffling.
#include "tb_device.cuh"
#include "tb_internal.h"

namespace tb {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kPF = 4;  // groups in flight per warp

// bf16 constants
constexpr uint32_t kMag = 0x43004300u;  // 128.0 | 128.0
constexpr uint32_t kOne = 0x3F803F80u, kHalf = 0x3F003F00u, kQuarter = 0x3E803E80u, kEighth = 0x3E003E00u,
                   kSixteenth = 0x3D803D80u;
// -(128 / 2^q + offset)
constexpr uint32_t kN130 = 0xC302C302u, kN34 = 0xC208C208u, kN10 = 0xC120C120u;              // offset 2
constexpr uint32_t kN132 = 0xC304C304u, kN68 = 0xC288C288u, kN36 = 0xC210C210u, kN20 = 0xC1A0C1A0u,
                   kN12 = 0xC140C140u;                                                         // offset 4

__device__ __forceinline__ uint32_t dq_field(uint32_t v, uint32_t mask, uint32_t mul, uint32_t add) {
    // (v & mask) | 128.0 = 128 + u * 2^q exactly; * 2^-q + add = c exactly
    return hfma2_bf16(and_or(v, mask, kMag), mul, add);
}

// 2-bit word -> o[m] = bf16x2 (c[2m], c[2m+1]), m = 0..7
__device__ __forceinline__ void dq_word2(uint32_t w, uint32_t (&o)[8]) {
    const uint32_t w6 = w >> 6, w12 = w >> 12;
    o[0] = dq_field(w, 0x00030003u, kOne, kN130);
    o[1] = dq_field(w, 0x000C000Cu, kQuarter, kN34);
    o[2] = dq_field(w, 0x00300030u, kSixteenth, kN10);
    o[3] = dq_field(w6, 0x00030003u, kOne, kN130);
    o[4] = dq_field(w6, 0x000C000Cu, kQuarter, kN34);
    o[5] = dq_field(w6, 0x00300030u, kSixteenth, kN10);
    o[6] = dq_field(w12, 0x00030003u, kOne, kN130);
    o[7] = dq_field(w12, 0x000C000Cu, kQuarter, kN34);
}

// bit masks with bits set at positions s + {0, 3, 6, ...} in both halves
constexpr uint32_t bits_at(int first, int count, int shift) {
    uint32_t m = 0;
    for (int i = 0; i < count; ++i) {
        m |= 1u << (first + 3 * i + shift);
        m |= 1u << (16 + first + 3 * i + shift);
    }
    return m;
}

// 3-bit block (planes p0, p1, p2) -> o[m] = bf16x2 (c[2m], c[2m+1]), m = 0..15.
// Field m of the block is bit m of each plane (low half) and bit 16+m (high
// half).  Shifting plane 1 left by 1 and plane 2 by 2 puts the three bits
// of field m at m, m+1, m+2; a bit-select of the three planes assembles
// every third field at once, and those fields are then cut out in pairs.
__device__ __forceinline__ void dq_block3(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t (&o)[16]) {
    const uint32_t q1 = p1 << 1, q2 = p2 << 2;
    // fields m = 0, 3, 6, 9, 12
    {
        const uint32_t z = bit_mux(bit_mux(p0, q1, bits_at(0, 5, 1)), q2, bits_at(0, 5, 2));
        const uint32_t z6 = z >> 6, z12 = z >> 12;
        o[0] = dq_field(z, 0x00070007u, kOne, kN132);
        o[3] = dq_field(z, 0x00380038u, kEighth, kN20);
        o[6] = dq_field(z6, 0x00070007u, kOne, kN132);
        o[9] = dq_field(z6, 0x00380038u, kEighth, kN20);
        o[12] = dq_field(z12, 0x00070007u, kOne, kN132);
    }
    // fields m = 1, 4, 7, 10, 13
    {
        const uint32_t z = bit_mux(bit_mux(p0, q1, bits_at(1, 5, 1)), q2, bits_at(1, 5, 2));
        const uint32_t z6 = z >> 6, z12 = z >> 12;
        o[1] = dq_field(z, 0x000E000Eu, kHalf, kN68);
        o[4] = dq_field(z, 0x00700070u, kSixteenth, kN12);
        o[7] = dq_field(z6, 0x000E000Eu, kHalf, kN68);
        o[10] = dq_field(z6, 0x00700070u, kSixteenth, kN12);
        o[13] = dq_field(z12, 0x000E000Eu, kHalf, kN68);
    }
    // fields m = 2, 5, 8, 11
    {
        const uint32_t z = bit_mux(bit_mux(p0, q1, bits_at(2, 4, 1)), q2, bits_at(2, 4, 2));
        const uint32_t z4 = z >> 4, z10 = z >> 10;
        o[2] = dq_field(z, 0x001C001Cu, kQuarter, kN36);
        o[5] = dq_field(z4, 0x000E000Eu, kHalf, kN68);
        o[8] = dq_field(z4, 0x00700070u, kSixteenth, kN12);
        o[11] = dq_field(z10, 0x000E000Eu, kHalf, kN68);
    }
    // fields m = 14, 15 (bits 14/15 and 30/31 of each plane)
    {
        const uint32_t r0 = p0 >> 14, r1 = p1 >> 13, r2 = p2 >> 12;
        const uint32_t z14 = bit_mux(bit_mux(r0, r1, 0x00020002u), r2, 0x00040004u);
        const uint32_t z15 = bit_mux(bit_mux(r0, r1, 0x00040004u), r2, 0x00080008u);
        o[14] = dq_field(z14, 0x00070007u, kOne, kN132);
        o[15] = dq_field(z15, 0x000E000Eu, kHalf, kN68);
    }
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Codes, scales of one 128-group for one lane (rows g and g + 8).
struct Slot {
    uint32_t a[3], b[3];  // 2-bit: words 2t, 2t+1 in a[0..1]; 3-bit: block t planes in a[0..2]
    uint32_t sa, sb;      // bf16 scale bits, rows g and g + 8
};

template <int KIND>  // 0: 2-bit container, 1: 3-bit planes
__device__ __forceinline__ void load_slot(Slot& s, const uint8_t* ra, const uint8_t* rb, const uint16_t* sa,
                                          const uint16_t* sb, int64_t grp, int t) {
    if (KIND == 0) {
        const uint2 va = ld_stream_u2(ra + 32 * grp + 8 * t);
        const uint2 vb = ld_stream_u2(rb + 32 * grp + 8 * t);
        s.a[0] = va.x; s.a[1] = va.y; s.a[2] = 0;
        s.b[0] = vb.x; s.b[1] = vb.y; s.b[2] = 0;
    } else {
        const uint8_t* pa = ra + 48 * grp + 12 * t;
        const uint8_t* pb = rb + 48 * grp + 12 * t;
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            s.a[p] = ld_stream_u32(pa + 4 * p);
            s.b[p] = ld_stream_u32(pb + 4 * p);
        }
    }
    s.sa = ld_stream_u16(sa + grp);
    s.sb = ld_stream_u16(sb + grp);
}

template <int KIND, int NT>
__device__ __forceinline__ void compute_slot(const Slot& s, float (&acc)[NT][4], const uint16_t* const (&xr)[NT],
                                             int64_t grp, int t) {
    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[nt][i] = 0.f;

    if (KIND == 0) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            // x for codes 16*(2t+w) .. +15 of this group: two 16-byte loads per column tile
            uint4 xv[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint16_t* xp = xr[nt] + 128 * grp + 32 * t + 16 * w;
                xv[nt][0] = ld_act_u4(xp);
                xv[nt][1] = ld_act_u4(xp + 8);
            }
            uint32_t qa[8], qb[8];
            dq_word2(s.a[w], qa);
            dq_word2(s.b[w], qb);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4 v = xv[nt][r >> 1];
                    const uint32_t b0 = (r & 1) ? v.z : v.x, b1 = (r & 1) ? v.w : v.y;
                    mma16816(d[nt], qa[2 * r], qb[2 * r], qa[2 * r + 1], qb[2 * r + 1], b0, b1);
                }
            }
        }
    } else {
        uint4 xv[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint16_t* xp = xr[nt] + 128 * grp + 32 * t;
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[nt][q] = ld_act_u4(xp + 8 * q);
        }
        uint32_t qa[16], qb[16];
        dq_block3(s.a[0], s.a[1], s.a[2], qa);
        dq_block3(s.b[0], s.b[1], s.b[2], qb);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint4 v = xv[nt][r >> 1];
                const uint32_t b0 = (r & 1) ? v.z : v.x, b1 = (r & 1) ? v.w : v.y;
                mma16816(d[nt], qa[2 * r], qb[2 * r], qa[2 * r + 1], qb[2 * r + 1], b0, b1);
            }
        }
    }
    const float fa = bf16_bits_to_float(s.sa), fb = bf16_bits_to_float(s.sb);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] = fmaf(fa, d[nt][0], acc[nt][0]);
        acc[nt][1] = fmaf(fa, d[nt][1], acc[nt][1]);
        acc[nt][2] = fmaf(fb, d[nt][2], acc[nt][2]);
        acc[nt][3] = fmaf(fb, d[nt][3], acc[nt][3]);
    }
}

template <int KIND, int NT>
__device__ __forceinline__ void run_tile(const Item& I, int64_t tile, float (*red)[NT * 4][32]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t N = I.N, K = I.K, G = K / kGroup;
    const int64_t rowA = tile * 16 + g, rowB = rowA + 8;
    const int64_t rA = rowA < N ? rowA : N - 1, rB = rowB < N ? rowB : N - 1;
    const int64_t rbytes = KIND == 0 ? K / 4 : 3 * K / 8;
    const uint8_t* pa = I.packed + rA * rbytes;
    const uint8_t* pb = I.packed + rB * rbytes;
    const uint16_t* sa = I.scales + rA * G;
    const uint16_t* sb = I.scales + rB * G;
    const uint16_t* xr[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + g;
        xr[nt] = I.X + (int64_t)(col < I.M ? col : I.M - 1) * I.ldx;
    }

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

    // this warp's groups: warp, warp + 8, warp + 16, ...
    const int64_t ng = G > warp ? (G - warp + kWarps - 1) / kWarps : 0;
    Slot buf[kPF];
#pragma unroll
    for (int i = 0; i < kPF; ++i)
        if (i < ng) load_slot<KIND>(buf[i], pa, pb, sa, sb, warp + (int64_t)kWarps * i, t);
    for (int64_t base = 0; base < ng; base += kPF) {
#pragma unroll
        for (int i = 0; i < kPF; ++i) {
            const int64_t step = base + i;
            if (step < ng) {
                const Slot cur = buf[i];
                if (step + kPF < ng) load_slot<KIND>(buf[i], pa, pb, sa, sb, warp + kWarps * (step + kPF), t);
                compute_slot<KIND, NT>(cur, acc, xr, warp + kWarps * step, t);
            }
        }
    }

    // cross-warp reduction in a fixed order
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][nt * 4 + i][lane] = acc[nt][i];
    __syncthreads();
    for (int e = threadIdx.x; e < NT * 4 * 32; e += kThreads) {
        const int nt = e / 128, i = (e / 32) & 3, ln = e & 31;
        const int64_t row = tile * 16 + (ln >> 2) + ((i >> 1) ? 8 : 0);
        const int col = nt * 8 + 2 * (ln & 3) + (i & 1);
        if (row < N && col < I.M) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += red[w][nt * 4 + i][ln];
            if (I.ydt == kF32) static_cast<float*>(I.Y)[(int64_t)col * I.ldy + row] = v;
            else static_cast<__nv_bfloat16*>(I.Y)[(int64_t)col * I.ldy + row] = __float2bfloat16_rn(v);
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 2) k_linear(const __grid_constant__ Launch L) {
    __shared__ float red[kWarps][NT * 4][32];
    const int u = blockIdx.x;
    int ii = 0;
    for (int i = 1; i < L.n_items; ++i)
        if (u >= L.it[i].unit_begin) ii = i;
    const Item& I = L.it[ii];
    const int64_t tile = u - I.unit_begin;
    if (I.grid == kInt3) run_tile<1, NT>(I, tile, red);
    else run_tile<0, NT>(I, tile, red);
}

}  // namespace

cudaError_t launch_linear(const Launch& L, int nt, int ctas, cudaStream_t st) {
    if (nt == 1) k_linear<1><<<ctas, kThreads, 0, st>>>(L);
    else k_linear<2><<<ctas, kThreads, 0, st>>>(L);
    return cudaGetLastError();
}

}  // namespace tb
